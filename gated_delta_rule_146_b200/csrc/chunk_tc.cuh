// chunk_tc.cuh -- the launcher of the fused tensor-core forward (chunk_tc.cu), shared by the
// forward's dispatch (api.cu) and the backward (chunk_bwd.cu).
#pragma once

#include "common.cuh"

namespace gdr {

// The backward's two passes on the fused kernel (fp32 outputs, see TcParams in chunk_tc.cu).
// Forward (adjoint = false): G ([token][head]), the state at every chunk start H
// ([chunk][head][128][128]) and V' ([token][head][128]).  Adjoint
// (adjoint = true; the launch's v is dO, S0 is dS_final and S_final is dS0): dH+ of every
// chunk in H and dV' in V.
struct TcSave {
    float *G, *H, *V;
    bool adjoint;
};

bool tc_supported(const gdr_chunk_args& a);
// `dependent`: launched as the programmatic dependent of the stream's previous grid;
// `g_rev`, `beta_rev`: the reverse direction's gates of a bidirectional pair (fp32 partials at
// `part_off` in the workspace); `save`: the saving instantiation (plain gates, head size 128,
// no output), for the backward
gdr_status launch_chunk_tc(const gdr_chunk_args& a, const void* q, const void* k, const void* v,
                           const void* g, const void* beta, const float* S0, void* o,
                           float* S_final, void* ws, const WsLayout& L, cudaStream_t st,
                           bool dependent = false, const void* g_rev = nullptr,
                           const void* beta_rev = nullptr, size_t part_off = 0,
                           const TcSave* save = nullptr);

}  // namespace gdr
