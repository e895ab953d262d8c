// chunk_bwd.cuh -- what the backward's CUDA-core kernels (chunk_bwd.cu) and its
// tensor-core per-chunk kernel (chunk_bwd_tc.cu) share: the kernel parameters and the
// (chunk, head) position of a block.
#pragma once

#include "common.cuh"

namespace gdr {

struct BwdParams {
    const void *q, *k, *v, *g, *beta, *dO;
    const float *S0, *dS_final;
    void *dq_out, *dk_out, *dv_out, *dg_out, *dbeta_out;
    float* dS0;
    const WsHeader* hdr; const int32_t *cu, *chunk_off, *chunk_seq;
    const float *W, *U, *G;         // from chunk_local_simt: [T][Hv][dk], [T][Hv][dv], [T][Hv]
    float *Hc, *dHc;                // [max_chunks][Hv][dk][dv]: H at chunk start, dH+
    float *Vp, *dVp;                // [T][Hv][dv]: V', dV'
    float *dW, *dKp, *dqh, *dkh;    // [T][Hv][dk]
    float* dGp;                     // [T][Hv]
    const float *Qt, *Kt;           // [T][Hv][dk]: s e^{G'} q^, e^{G_C - G} k^ (chunk_prep_simt)
    const float* Pc;                // [max_chunks][Hv][C][C]: P, zero off the mask
    int Hk, Hv, dk, dv, chunk, read_pre, qk_l2norm, reverse;
    gdr_dtype io, gt;
    float scale;
    int direct_out;  // tensor cores with Hv == Hk: dq, dk leave the per-chunk kernels in bf16
};

struct ChunkPos {
    int s, c, jc, p0, Cc;
    long long t0, t1;
};

__device__ __forceinline__ bool chunk_pos(const BwdParams& p, ChunkPos& cp) {
    cp.c = blockIdx.x;
    if (cp.c >= p.hdr->n_chunks) return false;
    cp.s = p.chunk_seq[cp.c];
    cp.t0 = p.cu[cp.s];
    cp.t1 = p.cu[cp.s + 1];
    cp.jc = cp.c - p.chunk_off[cp.s];
    cp.p0 = cp.jc * p.chunk;
    cp.Cc = (int)min((long long)p.chunk, (cp.t1 - cp.t0) - cp.p0);
    return true;
}

// The tensor-core per-chunk steps (dq / dK / dW, then the WY step): bf16 inputs,
// dk = dv = 128, chunk 64.
bool bwd_dqk_tc_supported(const gdr_chunk_args& a);
gdr_status launch_bwd_dqk_tc(const BwdParams& p, dim3 grid, cudaStream_t st);
gdr_status launch_bwd_wy_tc(const BwdParams& p, dim3 grid, cudaStream_t st);

}  // namespace gdr
