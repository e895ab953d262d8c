// decode.cu -- one-token recurrent decode step, streaming the fp32 state once.
//
// Per (sequence n, value head h) and token (flashrt fused_layer.py `_decode_one`:
// the recurrent core reads the cached state and writes the new one each token;
// tiny_gdn/fugue.py `fused_recurrent_gdn2_fwd` call with an initial state):
//     s_k = H^T k,  s_q = H^T q
//     u   = beta (v - alpha s_k)
//     H  <- alpha H + k u^T                         (in place)
//     post: o = scale (alpha s_q + (k.q) u)   [= scale H_new^T q]
//     pre:  o = scale s_q
// and, when the output epilogue is fused (the decode chain's gated RMSNorm, flashrt
// fused_layer.py `_decode_one`), o <- o / sqrt(mean(o^2) + eps) * weight * silu(z) over
// the head's dv values; the blocks of one head's column slices then form a thread-block
// cluster and add their partial sums of squares through distributed shared memory, so the
// normalised variant keeps the plain one's slice size (and its registers and occupancy).
// GDN-2 (decoupled gates, tiny_gdn/fugue.py BidirectionalGatedDeltaNet2) in the same pass:
// with per-row decay e^{g_d} and erase gate b_d and per-column write gate w_j,
//     s_k = H^T (e^g . b . k),  u = w . v - s_k,  H <- e^g . H + k u^T,
//     post: o = scale (H^T (e^g . q) + (k.q) u),  pre: o = scale H^T q.
// The columns of H (dv) are independent, so a block owns a slice of DVS columns
// and every row of it: it loads the whole slice into registers with 16-byte
// streaming loads, reduces s_k and s_q over the dk rows (warp shuffles, then
// shared memory across warps), and writes the updated slice back from the same
// registers.  Each block reads all of its slice before writing any of it, so the
// update in place needs no scratch copy of the state.
#include <cooperative_groups.h>

#include "common.cuh"

namespace gdr {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct DecodeParams {
    const void* q; const void* k; const void* v; const void* g; const void* beta;
    float* S; void* o;
    int Hk, Hv, read_pre, qk_l2norm;
    gdr_dtype io, gt;
    float scale;
    int gate_raw;                 // fused gating prologue (see gate_xform)
    const float* gate_A; const float* gate_dt_bias;
    float beta_scale;
    const void* norm_z; const float* norm_weight;  // fused gated RMSNorm epilogue
    float norm_eps;
    const void* w;                // GDN-2 write gate [N][Hv][dv]; g, beta are then [N][Hv][dk]
};

template <int DK, int DV, int DVS, bool kNorm, bool kG2>
__global__ void __launch_bounds__(kThreads)
decode_kernel(DecodeParams p) {
    constexpr int CL = DV / DVS;           // blocks per head (the cluster, when kNorm)
    constexpr int CPR = DVS / 4;           // float4 column groups per row slice
    constexpr int RPW = 32 / CPR;          // rows a warp covers per pass
    constexpr int RPP = RPW * kWarps;      // rows per pass over the block
    constexpr int NP = DK / RPP;           // passes (float4 registers per thread)
    static_assert(DK % RPP == 0, "dk must be a multiple of the rows per pass");

    __shared__ float s_q[DK], s_k[DK];
    __shared__ float s_red[2][kWarps][DVS];
    __shared__ float s_u[DVS];
    __shared__ float s_alpha, s_beta;
    __shared__ float s_o[kNorm ? DVS : 1];        // recurrent output of the head (epilogue)
    __shared__ float s_eg[kG2 ? DK : 1], s_b[kG2 ? DK : 1];  // GDN-2: e^{g_d}, b_d per row
    __shared__ float s_ss[kWarps];
    __shared__ float s_part[CL];                  // the cluster's partial sums of o^2

    const int nh = blockIdx.x;                   // n * Hv + h
    const int J = blockIdx.y;                    // column slice
    const int n = nh / p.Hv, h = nh % p.Hv, hk = h / (p.Hv / p.Hk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int cg = lane % CPR, rw = lane / CPR;  // float4 column group, row within warp pass

    // issue the state loads first: they are the whole cost of the kernel
    float* Sblk = p.S + (size_t)nh * DK * DV + J * DVS + cg * 4;
    float4 hreg[NP];
#pragma unroll
    for (int m = 0; m < NP; ++m) {
        const int d = m * RPP + wid * RPW + rw;
        hreg[m] = __ldcs(reinterpret_cast<const float4*>(Sblk + (size_t)d * DV));
    }

    // q, k (normalised), gates
    const size_t qk_base = ((size_t)n * p.Hk + hk) * DK;
    for (int d = tid; d < DK; d += kThreads) {
        s_q[d] = load_elem(p.q, qk_base + d, p.io);
        s_k[d] = load_elem(p.k, qk_base + d, p.io);
    }
    if constexpr (kG2) {
        for (int d = tid; d < DK; d += kThreads) {
            s_eg[d] = expf(load_elem(p.g, (size_t)nh * DK + d, p.gt));
            s_b[d] = load_elem(p.beta, (size_t)nh * DK + d, p.gt);
        }
    } else if (tid == 0) {
        s_alpha = expf(xform_g(p, h, load_elem(p.g, (size_t)nh, p.gt)));
        s_beta = xform_beta(p, load_elem(p.beta, (size_t)nh, p.gt));
    }
    __syncthreads();
    if (wid < 3) {
        // warp 0: ||q||, warp 1: ||k||, warp 2: raw k.q
        float acc = 0.f;
        for (int d = lane; d < DK; d += 32)
            acc += wid == 0 ? s_q[d] * s_q[d] : (wid == 1 ? s_k[d] * s_k[d] : s_q[d] * s_k[d]);
        acc = warp_sum(acc);
        if (lane == 0) s_red[0][wid][0] = acc;
    }
    __syncthreads();
    float inv_q = 1.f, inv_k = 1.f;
    if (p.qk_l2norm) {
        inv_q = 1.f / fmaxf(sqrtf(s_red[0][0][0]), kNormEps);
        inv_k = 1.f / fmaxf(sqrtf(s_red[0][1][0]), kNormEps);
    }
    const float kq = s_red[0][2][0] * inv_q * inv_k;
    __syncthreads();

    // partial s_k, s_q over this thread's rows, 4 columns
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sq = sk;
    float kr[NP];  // normalised k, per held row
#pragma unroll
    for (int m = 0; m < NP; ++m) {
        const int d = m * RPP + wid * RPW + rw;
        float kd = s_k[d] * inv_k, qd = s_q[d] * inv_q;
        kr[m] = kd;
        if constexpr (kG2) {  // weights of this row in s_k and s_q
            const float e = s_eg[d];
            kd *= e * s_b[d];
            if (!p.read_pre) qd *= e;
        }
        sk.x = fmaf(hreg[m].x, kd, sk.x); sk.y = fmaf(hreg[m].y, kd, sk.y);
        sk.z = fmaf(hreg[m].z, kd, sk.z); sk.w = fmaf(hreg[m].w, kd, sk.w);
        sq.x = fmaf(hreg[m].x, qd, sq.x); sq.y = fmaf(hreg[m].y, qd, sq.y);
        sq.z = fmaf(hreg[m].z, qd, sq.z); sq.w = fmaf(hreg[m].w, qd, sq.w);
    }
    // reduce over the rows held by this warp (lanes sharing a column group)
#pragma unroll
    for (int o = CPR; o < 32; o <<= 1) {
        sk.x += __shfl_xor_sync(0xffffffffu, sk.x, o); sk.y += __shfl_xor_sync(0xffffffffu, sk.y, o);
        sk.z += __shfl_xor_sync(0xffffffffu, sk.z, o); sk.w += __shfl_xor_sync(0xffffffffu, sk.w, o);
        sq.x += __shfl_xor_sync(0xffffffffu, sq.x, o); sq.y += __shfl_xor_sync(0xffffffffu, sq.y, o);
        sq.z += __shfl_xor_sync(0xffffffffu, sq.z, o); sq.w += __shfl_xor_sync(0xffffffffu, sq.w, o);
    }
    if (rw == 0) {
        s_red[0][wid][cg * 4 + 0] = sk.x; s_red[0][wid][cg * 4 + 1] = sk.y;
        s_red[0][wid][cg * 4 + 2] = sk.z; s_red[0][wid][cg * 4 + 3] = sk.w;
        s_red[1][wid][cg * 4 + 0] = sq.x; s_red[1][wid][cg * 4 + 1] = sq.y;
        s_red[1][wid][cg * 4 + 2] = sq.z; s_red[1][wid][cg * 4 + 3] = sq.w;
    }
    __syncthreads();
    const float alpha = s_alpha, beta = s_beta;
    if (tid < DVS) {
        float tk = 0.f, tq = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) { tk += s_red[0][w][tid]; tq += s_red[1][w][tid]; }
        const int col = J * DVS + tid;
        const float vj = load_elem(p.v, (size_t)nh * DV + col, p.io);
        float u, oj;
        if constexpr (kG2) {
            u = load_elem(p.w, (size_t)nh * DV + col, p.gt) * vj - tk;
            oj = p.read_pre ? p.scale * tq : p.scale * fmaf(kq, u, tq);
        } else {
            u = beta * (vj - alpha * tk);
            oj = p.read_pre ? p.scale * tq : p.scale * fmaf(alpha, tq, kq * u);
        }
        s_u[tid] = u;
        if constexpr (kNorm) s_o[tid] = oj;
        else store_elem(p.o, (size_t)nh * DV + col, oj, p.io);
    }
    __syncthreads();
    if constexpr (kNorm) {
        // gated RMSNorm over the head: o_j / sqrt(mean(o^2) + eps) * weight_j * silu(z_j);
        // this block's slice gives a partial sum of o^2, which its first thread writes into
        // slot J of every block of the cluster (the head's slices, J = rank in the cluster)
        if (wid * 32 < DVS) {
            const float x = tid < DVS ? s_o[tid] : 0.f;
            const float ss = warp_sum(x * x);
            if (lane == 0) s_ss[wid] = ss;
        }
        __syncthreads();
        if (tid == 0) {
            float ss = 0.f;
#pragma unroll
            for (int w = 0; w < (DVS + 31) / 32; ++w) ss += s_ss[w];
            if constexpr (CL > 1) {
                cooperative_groups::cluster_group cl = cooperative_groups::this_cluster();
#pragma unroll
                for (int r = 0; r < CL; ++r) cl.map_shared_rank(s_part, r)[J] = ss;
            } else {
                s_part[0] = ss;
            }
        }
        // every block's partial has arrived (and nothing reads another block's memory after)
        if constexpr (CL > 1) cooperative_groups::this_cluster().sync();
        else __syncthreads();
        if (tid < DVS) {
            float ss = 0.f;
#pragma unroll
            for (int r = 0; r < CL; ++r) ss += s_part[r];
            const int col = J * DVS + tid;
            const float rr = rsqrtf(ss / DV + p.norm_eps);
            const float z = load_elem(p.norm_z, (size_t)nh * DV + col, p.io);
            const float silu = z / (1.f + expf(-z));
            store_elem(p.o, (size_t)nh * DV + col, s_o[tid] * rr * p.norm_weight[col] * silu, p.io);
        }
    }
    const float4 u4 = *reinterpret_cast<const float4*>(&s_u[cg * 4]);
#pragma unroll
    for (int m = 0; m < NP; ++m) {
        const int d = m * RPP + wid * RPW + rw;
        float4 r;
        const float a = kG2 ? s_eg[d] : alpha;  // the row's decay (re-read: fewer registers)
        r.x = fmaf(a, hreg[m].x, kr[m] * u4.x); r.y = fmaf(a, hreg[m].y, kr[m] * u4.y);
        r.z = fmaf(a, hreg[m].z, kr[m] * u4.z); r.w = fmaf(a, hreg[m].w, kr[m] * u4.w);
        __stcs(reinterpret_cast<float4*>(Sblk + (size_t)d * DV), r);
    }
}

// The normed epilogue reduces over the head's dv values: its slices of one head run as one
// thread-block cluster (DV / DVS blocks along y).
template <int DK, int DV, int DVS, bool kG2>
gdr_status launch_norm(const DecodeParams& p, dim3 grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = DV / DVS;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_kernel<DK, DV, DVS, true, kG2>, p) != cudaSuccess)
        return GDR_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

template <int DK, int DV>
gdr_status launch_dv(const gdr_decode_args& a, const DecodeParams& p, cudaStream_t st) {
    constexpr int DVS = DV >= 64 ? 64 : 32;
    const dim3 sliced((unsigned)(a.N * a.Hv), DV / DVS);
    if (a.out_norm && a.gdn2) return launch_norm<DK, DV, DVS, true>(p, sliced, st);
    if (a.out_norm) return launch_norm<DK, DV, DVS, false>(p, sliced, st);
    if (a.gdn2) decode_kernel<DK, DV, DVS, false, true><<<sliced, kThreads, 0, st>>>(p);
    else decode_kernel<DK, DV, DVS, false, false><<<sliced, kThreads, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

template <int DK>
gdr_status launch_dk(const gdr_decode_args& a, const DecodeParams& p, cudaStream_t st) {
    switch (a.dv) {
        case 32: return launch_dv<DK, 32>(a, p, st);
        case 64: return launch_dv<DK, 64>(a, p, st);
        case 128: return launch_dv<DK, 128>(a, p, st);
        default: return GDR_ERR_UNSUPPORTED;
    }
}

}  // namespace

bool decode_supported(const gdr_decode_args& a) {
    return (a.dk == 32 || a.dk == 64 || a.dk == 128) && (a.dv == 32 || a.dv == 64 || a.dv == 128);
}

gdr_status launch_decode(const gdr_decode_args& a, const void* q, const void* k, const void* v,
                         const void* g, const void* beta, float* S, void* o, cudaStream_t st) {
    DecodeParams p;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.S = S; p.o = o;
    p.Hk = a.Hk; p.Hv = a.Hv; p.read_pre = a.read_mode == GDR_READ_PRE;
    p.qk_l2norm = a.qk_l2norm; p.io = a.io_dtype; p.gt = a.gate_dtype; p.scale = a.scale;
    p.gate_raw = a.gate_raw; p.gate_A = a.gate_A; p.gate_dt_bias = a.gate_dt_bias;
    p.beta_scale = a.beta_scale;
    p.norm_z = a.norm_z; p.norm_weight = a.norm_weight; p.norm_eps = a.norm_eps;
    p.w = a.gdn2_w;
    switch (a.dk) {
        case 32: return launch_dk<32>(a, p, st);
        case 64: return launch_dk<64>(a, p, st);
        case 128: return launch_dk<128>(a, p, st);
        default: return GDR_ERR_UNSUPPORTED;
    }
}

}  // namespace gdr
