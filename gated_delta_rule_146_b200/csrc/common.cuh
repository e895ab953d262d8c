// common.cuh -- device helpers and the workspace layout shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr.h"

namespace gdr {

constexpr float kNormEps = 1e-6f;  // x / max(||x||, eps), as F.normalize(eps=1e-6)

// ---- element access ---------------------------------------------------------

__device__ __forceinline__ float load_elem(const void* p, size_t i, gdr_dtype dt) {
    return dt == GDR_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
                          : static_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_elem(void* p, size_t i, float x, gdr_dtype dt) {
    if (dt == GDR_BF16) static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    else static_cast<float*>(p)[i] = x;
}

// ---- fused gating prologue ---------------------------------------------------
// Raw per-token projections a, b -> g = A softplus(a + dt_bias), beta = beta_scale sigmoid(b)
// (sparse_delta_memory/layer.py compute_gates, with the doubled beta of tiny_gdn/fugue.py
// `project`); the identity when the gates are given.  `P` is a kernel's parameter block
// (fields gate_raw, gate_A, gate_dt_bias, beta_scale), read where used so that nothing stays
// live in registers, and the math is out of line, so that the kernels' register allocation
// does not carry a branch that plain gates never take.
static __device__ __noinline__ float gate_g_from_raw(float A, float dt, float a) {
    const float x = a + dt;
    return A * (x > 20.f ? x : log1pf(expf(x)));
}

static __device__ __noinline__ float gate_beta_from_raw(float scale, float b) {
    return scale / (1.f + expf(-b));
}

template <typename P>
__device__ __forceinline__ float xform_g(const P& p, int h, float a) {
    return p.gate_raw ? gate_g_from_raw(p.gate_A[h], p.gate_dt_bias[h], a) : a;
}

template <typename P>
__device__ __forceinline__ float xform_beta(const P& p, float b) {
    return p.gate_raw ? gate_beta_from_raw(p.beta_scale, b) : b;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---- workspace ----------------------------------------------------------------
//
// [header 256 B][cu (n_seqs+1) int32][chunk_off (n_seqs+1) int32][chunk_seq (max_chunks)
// int32][fp32 W [T_tot][Hv][dk]][fp32 U [T_tot][Hv][dv]][fp32 G [T_tot][Hv] (x dk for GDN-2)]
// [fp32 Q~, K~ [T_tot][Hv][dk]][fp32 P [max_chunks][Hv][C][C]]
// The fp32 arrays exist only for the CUDA-core (SIMT) path; Q~, K~, P only for its
// register-blocked scan.

struct WsHeader {
    int err;           // gdr_status recorded by a device-side check
    int n_chunks;      // total chunks over all sequences
    int pad[62];
};

struct WsLayout {
    size_t cu, chunk_off, chunk_seq, order, W, U, G, Qt, Kt, Pc, rec, total;
    long long max_chunks;
};

// Sequences a per-(sequence, head) kernel visits in order of decreasing length (varlen calls
// of at most this many sequences; otherwise, and without cu_seqlens, in index order), so
// that the longest sequences start in the first wave and none is left for the last.
constexpr int kOrderMaxSeqs = 1024;

// The register-blocked CUDA-core scan (chunk_scan_rb) splits a chunk's rows and the state's
// dk rows over 8 warps, the latter in float4s: chunk <= 64, dk a multiple of 32 up to 128.
// It reads the decayed, scaled Q~, K~ and P that chunk_prep_simt writes.
inline bool simt_rb(const gdr_chunk_args& a) {
    return a.chunk <= 64 && a.dk % 32 == 0 && a.dk <= 128 && a.dv % 32 == 0;
}

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bytes of one (chunk, head) record of the tensor-core GDN-2 path: the shared-memory image of
// the recursion's operands (q~, -W, K~, U~^T, P in fp16, e^{G_C} in fp32).
constexpr size_t kG2RecordBytes = 74240;

inline WsLayout ws_layout(const gdr_chunk_args& a, bool simt) {
    WsLayout L{};
    const long long T_tot = (long long)a.B * a.T;
    L.max_chunks = (T_tot + a.chunk - 1) / a.chunk + a.n_seqs;
    size_t off = sizeof(WsHeader);
    L.cu = off;        off = align_up(off + sizeof(int32_t) * (a.n_seqs + 1), 256);
    L.chunk_off = off; off = align_up(off + sizeof(int32_t) * (a.n_seqs + 1), 256);
    L.chunk_seq = off; off = align_up(off + sizeof(int32_t) * (size_t)L.max_chunks, 256);
    L.order = off;     off = align_up(off + sizeof(int32_t) * (size_t)a.n_seqs, 256);
    if (simt) {
        L.W = off; off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv * a.dk, 256);
        L.U = off; off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv * a.dv, 256);
        // in-chunk log decay: one per token and head, or one per key channel for GDN-2
        L.G = off;
        off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv * (a.gdn2 ? a.dk : 1), 256);
        if (simt_rb(a)) {  // operands of the register-blocked scan
            L.Qt = off; off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv * a.dk, 256);
            L.Kt = off; off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv * a.dk, 256);
            L.Pc = off;
            off = align_up(off + sizeof(float) * (size_t)L.max_chunks * a.Hv * a.chunk * a.chunk, 256);
        }
    }
    if (!simt && a.gdn2) {  // tensor-core GDN-2: one record per (chunk, head)
        L.rec = off;
        off = align_up(off + kG2RecordBytes * (size_t)L.max_chunks * a.Hv, 256);
    }
    L.total = off;
    return L;
}

// Device view of the chunk map built by plan_kernel.
struct ChunkMap {
    const WsHeader* hdr;
    const int32_t* cu;         // [n_seqs+1] token offsets (validated)
    const int32_t* chunk_off;  // [n_seqs+1] first global chunk of each sequence
    const int32_t* chunk_seq;  // [max_chunks] sequence of each global chunk
};

// Physical token index of logical position p of a sequence spanning [t0, t1).
__device__ __forceinline__ long long phys_token(long long t0, long long t1, int p, int reverse) {
    return reverse ? (t1 - 1 - p) : (t0 + p);
}

}  // namespace gdr

// Launchers implemented in the .cu files (host side).
namespace gdr {
cudaError_t launch_plan(const gdr_chunk_args& a, const int32_t* cu_in, void* ws, const WsLayout& L,
                        cudaStream_t st);
gdr_status launch_chunk_simt(const gdr_chunk_args& a, const void* q, const void* k,
                             const void* v, const void* g, const void* beta, const float* S0,
                             void* o, float* S_final, void* ws, const WsLayout& L,
                             cudaStream_t st);
bool simt_supported(const gdr_chunk_args& a);
// W, U~, G of every chunk (the CUDA-core forward's first kernel) into the given arrays.
gdr_status launch_wy_local_simt(const gdr_chunk_args& a, const void* k, const void* v,
                                const void* g, const void* beta, void* ws, const WsLayout& L,
                                float* W, float* U, float* G, cudaStream_t st);

// Q~, K~ and P of every chunk (scalar gates) into the workspace arrays of ws_layout.
gdr_status launch_prep_simt(const gdr_chunk_args& a, const void* q, const void* k, void* ws,
                            const WsLayout& L, cudaStream_t st);

// Backward pass (chunk_bwd.cu).
struct BwdLayout {
    WsLayout base;  // the forward's plan and CUDA-core arrays
    size_t G;       // the in-chunk log decay (the base layout's, or the backward's own)
    size_t Hc, dHc, Vp, dVp, dW, dKp, dqh, dkh, dGp, total;
};
struct BwdPtrs {
    const void *q, *k, *v, *g, *beta, *dO;
    const float *S0, *dS_final;
    void *dq, *dk, *dv, *dg, *dbeta;
    float* dS0;
};
BwdLayout bwd_layout(const gdr_chunk_args& a);
bool bwd_supported(const gdr_chunk_args& a);
gdr_status launch_chunk_bwd(const gdr_chunk_args& a, const BwdPtrs& x, void* ws,
                            const BwdLayout& B, cudaStream_t st);
gdr_status launch_decode(const gdr_decode_args& a, const void* q, const void* k, const void* v,
                         const void* g, const void* beta, float* S, void* o, cudaStream_t st);
bool decode_supported(const gdr_decode_args& a);
}  // namespace gdr
