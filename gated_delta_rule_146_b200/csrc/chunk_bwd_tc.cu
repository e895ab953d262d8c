// chunk_bwd_tc.cu -- the backward's per-(chunk, head) dq / dK / dW step on the tensor cores.
//
// It computes what bwd_chunk_dqk (chunk_bwd.cu) computes, for bf16 inputs, dk = dv = 128 and
// chunk 64 (the gradient of the chunk form; Prizma "seq/delta.py", module docstring, asks the
// chunk-parallel form to agree with the per-token recurrence on the gradients too):
//     dP_ij = dO_i . V'_j,  D1_ij = s dP_ij e^{G'_i - G_j} on the causal mask,  E = D1 . (Q^ K^T)
//     dQ^   = D1 K^ + s diag(e^{G'}) dO H^T        -> dq by the normalisation's adjoint
//     dK^   = D1^T Q^ + diag(e^{G_C - G}) V' dH+^T (the P and carry parts)
//     dW    = -dV' H^T
// and the decay gradients that these terms carry (row and column sums of E, the inter read,
// the carry and <dH+, H> at the chunk's last position).
//
// Every product is one tcgen05 MMA of M = 128 rows, fp16 operands from 128-byte swizzled
// shared memory and an fp32 accumulator in tensor memory.  M = 128 comes from stacking two
// 64-row operands; where only one half of the result is used, the other is not read:
//     [dO; dV'] H^T    rows 0-63: X = dO H^T           rows 64-127: dV' H^T = -dW
//     [dV'; V'] dH+^T                                  rows 64-127: Z = V' dH+^T
//     [dO; dV'] V'^T   rows 0-63: dP
//     [q; k] k^T       rows 0-63: q_i . k_j (the norms are applied in fp32)
//     [D1k; D1q^T] k   rows 0-63: D1 K^          (D1k_ij  = D1_ij / |k_j|)
//     [D1k; D1q^T] q                                   rows 64-127: D1^T Q^ (D1q^T_ji = D1_ij / |q_i|)
// The q and k tiles serve as K-major A operands and as MN-major B operands, so no transposed
// copy is made.
//
// Range.  Gradients carry whatever scale the loss gives them, so every operand row is stored
// as fp16 times a power of two that brings its largest magnitude into [2^14, 2^15): rows of
// the stacked A operands, the rows of H and dH+ (the N index of their products, so their
// factors divide the result's columns) and the rows of q and k.  The epilogues divide the
// factors out exactly; along a K index (the rows of q and k in the D1 products) the factor is
// folded into the other operand.  fp16 keeps 11 significant bits against bf16's 8.
#include "chunk_bwd.cuh"
#include "tc_ptx.cuh"

namespace gdr {

namespace {

using namespace tc;

constexpr int kTh = 256;                 // 8 warps: warps w and w + 4 share TMEM lanes 32 (w & 3)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBarEpi = 1;               // named barrier of the four warps that hold rows 0-63

// shared memory: 128-byte swizzled rows of 64 fp16 (a "group"); K = 128 takes two groups
constexpr uint32_t OFF_E = 0;            // per group: dO rows 0-63 | dV' rows | V' rows
constexpr uint32_t E_GRP = 24576;
constexpr uint32_t OFF_H = 49152;        // H as B (rows d, K = e), two groups of 16 KB
constexpr uint32_t OFF_DH = 81920;       // dH+ as B, same
constexpr uint32_t OFF_QK = 114688;      // per group: q rows 0-63 | k rows (K = d)
constexpr uint32_t G16 = 16384;          // group stride of the H, dH+ and q/k regions
constexpr uint32_t OFF_D = 147456;       // D1k rows 0-63 (K = j) | D1q^T rows 64-127 (K = i)
constexpr uint32_t OFF_SMALL = 163840;

// tensor memory columns (fp32 accumulators, lane = row of the stacked product)
constexpr uint32_t TM_X = 0, TM_Z = 128, TM_P = 256, TM_S = 320, TM_DQ = 256, TM_DK = 384;

struct DqkSmall {
    float G[64], Gr[64], invq[64], invk[64], nq[64];
    // reciprocal row factors: 1 / (power of two) of each stored fp16 row
    float rq[64], rk[64], rdo[64], rv[64], rdv[64], rh[128], rdh[128], rd1[64], rd1t[64];
    float amax[2][64];  // largest |D1k| of row i, by column half
    float bmax[2][64];  // largest |D1q^T| of row j, by row warp
    float dGr[2][64];   // row sums of E, by column half
    float dGs[2][64];   // column sums of -E, by row warp
    float gsum[2][64];  // sum_d q_d X_d, by d half
    float projq[2][64]; // sum_d q_d acc_d, by d half
    float ck[2][64];    // sum_d k_d Z_d, by d half
    float c[64];        // the carry's decay gradient per position
    float hdot[8];      // <dH+, H> by warp
    float csum[2];
    uint64_t mbar[2];
    uint32_t tmem;
};
constexpr uint32_t SMEM_BYTES = OFF_SMALL + sizeof(DqkSmall) + 1024;
static_assert(OFF_SMALL + sizeof(DqkSmall) + 1024 <= 227 * 1024, "shared memory");

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }

// The power of two that maps a row whose largest magnitude is m into [2^14, 2^15): 2^(15 - e)
// for m in [2^(e-1), 2^e), built from the exponent bits; 1 for a zero or non-finite row.
__device__ __forceinline__ float pow2_scale(float m) {
    if (!(m > 0.f) || !(m <= 3.402823e38f)) return 1.f;
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 126;  // m < 2^e (normal m)
    const int x = min(max(15 - e, -126), 127);
    return __uint_as_float((uint32_t)(x + 127) << 23);
}

// largest magnitude (or sum) over the 16 lanes that hold one row (lanes 16 l .. 16 l + 15)
__device__ __forceinline__ float max16(float m) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}
__device__ __forceinline__ float sum16(float m) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) m += __shfl_xor_sync(0xffffffffu, m, o);
    return m;
}

__device__ __forceinline__ float amax8(const float (&f)[8]) {
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    return m;
}

// 8 values times s -> one 16-byte piece of fp16
__device__ __forceinline__ uint4 f16x8(const float (&f)[8], float s) {
    return make_uint4(pack_f16x2(f[0] * s, f[1] * s), pack_f16x2(f[2] * s, f[3] * s),
                      pack_f16x2(f[4] * s, f[5] * s), pack_f16x2(f[6] * s, f[7] * s));
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = unpack_bf16x2(w[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}

__device__ __forceinline__ void f16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = unpack_f16x2(w[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}

__device__ __forceinline__ void f4x2_to_f32(const float4& a, const float4& b, float (&f)[8]) {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// v[u] summed (or maximised) over the warp's 32 lanes for every u, left in lane u: a
// butterfly that halves the values each thread carries at every step.
template <bool kMax>
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int u = 0; u < s; ++u) {
            const float send = upper ? v[u] : v[u + s];
            const float keep = upper ? v[u + s] : v[u];
            const float got = __shfl_xor_sync(0xffffffffu, send, s);
            v[u] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(kTh, 1) bwd_chunk_dqk_tc(BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    DqkSmall& SS = *reinterpret_cast<DqkSmall*>(sm + OFF_SMALL);
    if (p.hdr->err != GDR_OK) return;
    ChunkPos cp;
    if (!chunk_pos(p, cp)) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, ch = warp >> 2;  // TMEM lane quarter; column half
    const int h = blockIdx.y, hk = h / (p.Hv / p.Hk), Cc = cp.Cc;
    const bool pre = p.read_pre != 0, on = p.qk_l2norm != 0;
    auto tok = [&](int i) { return phys_token(cp.t0, cp.t1, cp.p0 + i, p.reverse); };
    const uint4* qg = static_cast<const uint4*>(p.q);
    const uint4* kg = static_cast<const uint4*>(p.k);
    const uint4* dog = static_cast<const uint4*>(p.dO);

    if (warp == 0) {
        tmem_alloc(&SS.tmem, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    if (tid == 0) {
        mbar_init(&SS.mbar[0], 1);
        mbar_init(&SS.mbar[1], 1);
        mbar_init_fence();
    }
    if (tid < 64) SS.G[tid] = tid < Cc ? p.G[(size_t)tok(tid) * p.Hv + h] : 0.f;

    // ---- staging.  Each row of 128 values is 16 pieces of 8, held by 16 consecutive lanes,
    // which agree on the row's factor; rows past the chunk are zero.
    {
        // q (t = 0), k (t = 1) and dO (t = 2), bf16; the norms of q and k on the way
        uint4 raw[12];
#pragma unroll
        for (int it = 0; it < 12; ++it) {
            const int idx = tid + it * kTh, t = idx >> 10, i = (idx >> 4) & 63, c = idx & 15;
            raw[it] = make_uint4(0, 0, 0, 0);
            if (i < Cc) {
                const size_t row = t == 2 ? (size_t)tok(i) * p.Hv + h : (size_t)tok(i) * p.Hk + hk;
                raw[it] = __ldg((t == 2 ? dog : t ? kg : qg) + row * 16 + c);
            }
        }
#pragma unroll
        for (int it = 0; it < 12; ++it) {
            const int idx = tid + it * kTh, t = idx >> 10, i = (idx >> 4) & 63, c = idx & 15;
            float f[8];
            bf16x8_to_f32(raw[it], f);
            const float sc = pow2_scale(max16(amax8(f)));
            const uint32_t dst = t == 2 ? OFF_E + (c >> 3) * E_GRP + sw128(i, c & 7)
                                        : OFF_QK + (c >> 3) * G16 + t * 8192 + sw128(i, c & 7);
            *reinterpret_cast<uint4*>(sm + dst) = f16x8(f, sc);
            float ss = 0.f;
            if (t < 2) {
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
                ss = sum16(ss);
            }
            if (c == 0) {
                const float r = __frcp_rn(sc);
                if (t == 2) {
                    SS.rdo[i] = r;
                } else {
                    const float n = sqrtf(ss);
                    const float inv = on ? 1.f / fmaxf(n, kNormEps) : 1.f;
                    if (t) { SS.rk[i] = r; SS.invk[i] = inv; }
                    else { SS.rq[i] = r; SS.invq[i] = inv; SS.nq[i] = n; }
                }
            }
        }
    }
    {
        // V' (t = 0) and dV' (t = 1), fp32 from the state passes
#pragma unroll 1
        for (int it0 = 0; it0 < 8; it0 += 4) {
            float4 a[4][2];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int idx = tid + (it0 + u) * kTh, t = idx >> 10, i = (idx >> 4) & 63, c = idx & 15;
                a[u][0] = a[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < Cc) {
                    const float4* src = reinterpret_cast<const float4*>(
                        (t ? p.dVp : p.Vp) + ((size_t)tok(i) * p.Hv + h) * 128 + c * 8);
                    a[u][0] = __ldg(src);
                    a[u][1] = __ldg(src + 1);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int idx = tid + (it0 + u) * kTh, t = idx >> 10, i = (idx >> 4) & 63, c = idx & 15;
                float f[8];
                f4x2_to_f32(a[u][0], a[u][1], f);
                const float sc = pow2_scale(max16(amax8(f)));
                *reinterpret_cast<uint4*>(sm + OFF_E + (c >> 3) * E_GRP + (t ? 8192 : 16384) +
                                          sw128(i, c & 7)) = f16x8(f, sc);
                if (c == 0) (t ? SS.rdv : SS.rv)[i] = __frcp_rn(sc);
            }
        }
    }
    {
        // H and dH+ (row d, column e), fp32, and <dH+, H> in fp32 on the way
        const size_t cbase = ((size_t)cp.c * p.Hv + h) * 128 * 128;
        float hdot = 0.f;
#pragma unroll 1
        for (int it0 = 0; it0 < 8; it0 += 2) {
            float4 a[2][2], b[2][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int idx = tid + (it0 + u) * kTh, d = idx >> 4, c = idx & 15;
                const float4* hs = reinterpret_cast<const float4*>(p.Hc + cbase + (size_t)d * 128 + c * 8);
                const float4* gs = reinterpret_cast<const float4*>(p.dHc + cbase + (size_t)d * 128 + c * 8);
                a[u][0] = __ldg(hs);
                a[u][1] = __ldg(hs + 1);
                b[u][0] = __ldg(gs);
                b[u][1] = __ldg(gs + 1);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int idx = tid + (it0 + u) * kTh, d = idx >> 4, c = idx & 15;
                float fh[8], fg[8];
                f4x2_to_f32(a[u][0], a[u][1], fh);
                f4x2_to_f32(b[u][0], b[u][1], fg);
#pragma unroll
                for (int e = 0; e < 8; ++e) hdot = fmaf(fh[e], fg[e], hdot);
                const float sh = pow2_scale(max16(amax8(fh)));
                const float sg = pow2_scale(max16(amax8(fg)));
                const uint32_t off = (c >> 3) * G16 + sw128(d, c & 7);
                *reinterpret_cast<uint4*>(sm + OFF_H + off) = f16x8(fh, sh);
                *reinterpret_cast<uint4*>(sm + OFF_DH + off) = f16x8(fg, sg);
                if (c == 0) {
                    SS.rh[d] = __frcp_rn(sh);
                    SS.rdh[d] = __frcp_rn(sg);
                }
            }
        }
        hdot = warp_sum(hdot);
        if (lane == 0) SS.hdot[warp] = hdot;
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    if (tid < 64) SS.Gr[tid] = pre ? (tid > 0 ? SS.G[tid - 1] : 0.f) : SS.G[tid];
    const uint32_t tmem = SS.tmem;
    const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);  // this warp's TMEM lanes

    // ---- first products: X, Z, dP and q . k
    if (tid == 0) {
        const uint32_t i64 = idesc_f32acc(128, 64, false, false, false);
        const uint32_t i128 = idesc_f32acc(128, 128, false, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t eo = (kk >> 2) * E_GRP + (kk & 3) * 32, go = (kk >> 2) * G16 + (kk & 3) * 32;
            mma_f32acc_ss(tmem + TM_P, kdesc(sbase + OFF_E + eo), kdesc(sbase + OFF_E + 16384 + eo), i64, kk > 0);
            mma_f32acc_ss(tmem + TM_S, kdesc(sbase + OFF_QK + go), kdesc(sbase + OFF_QK + 8192 + go), i64, kk > 0);
            mma_f32acc_ss(tmem + TM_X, kdesc(sbase + OFF_E + eo), kdesc(sbase + OFF_H + go), i128, kk > 0);
            mma_f32acc_ss(tmem + TM_Z, kdesc(sbase + OFF_E + 8192 + eo), kdesc(sbase + OFF_DH + go), i128, kk > 0);
        }
        mma_commit(&SS.mbar[0]);
    }
    bool fail = !mbar_wait_bounded(&SS.mbar[0], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();

    // ---- D1 from dP and q . k (rows i = 0-63: warps 0, 1 and 4, 5; column half ch)
    float a1[32], b1[32];  // D1k of row i, D1q^T of column i (rows j), before their row factors
    if (!fail && sp < 2) {
        const int i = sp * 32 + lane;
        uint32_t rp[32], rs[32];
        tmem_ld32(tl + TM_P + ch * 32, rp);
        tmem_ld32(tl + TM_S + ch * 32, rs);
        tmem_wait_ld();
        const bool li = i < Cc;
        const float gri = SS.Gr[i], iq = SS.invq[i], rqi = SS.rq[i], rdoi = SS.rdo[i];
        float e[32], bm[32], rsum = 0.f, am = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            const bool m = li && j < Cc && (pre ? j < i : j <= i);
            const float ik = SS.invk[j], rkj = SS.rk[j];
            const float dp = u2f(rp[u]) * rdoi * SS.rv[j];
            const float d1 = m ? p.scale * dp * exp2f((gri - SS.G[j]) * kLog2e) : 0.f;
            const float ev = d1 * (u2f(rs[u]) * rqi * rkj * iq * ik);
            rsum += ev;
            e[u] = -ev;
            a1[u] = d1 * ik * rkj;
            b1[u] = d1 * iq * rqi;
            am = fmaxf(am, fabsf(a1[u]));
            bm[u] = fabsf(b1[u]);
        }
        SS.dGr[ch][i] = rsum;
        SS.amax[ch][i] = am;
        const float col = transpose_reduce32<false>(e, lane);
        SS.dGs[sp][ch * 32 + lane] = col;
        const float cmax = transpose_reduce32<true>(bm, lane);
        SS.bmax[sp][ch * 32 + lane] = cmax;
        named_bar(kBarEpi, 128);
        // D1k row i and D1q^T rows j in fp16, each with its row's factor
        const float sd = pow2_scale(fmaxf(SS.amax[0][i], SS.amax[1][i]));
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = a1[e8 * 8 + u];
            *reinterpret_cast<uint4*>(sm + OFF_D + sw128(i, ch * 4 + e8)) = f16x8(f, sd);
        }
        uint16_t* d1t = reinterpret_cast<uint16_t*>(sm + OFF_D);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            const float st = pow2_scale(fmaxf(SS.bmax[0][j], SS.bmax[1][j]));
            const __half hv = __float2half_rn(b1[u] * st);
            d1t[(sw128(64 + j, i >> 3) >> 1) + (i & 7)] = *reinterpret_cast<const uint16_t*>(&hv);
        }
        if (ch == 0) SS.rd1[i] = __frcp_rn(sd);
        if (sp == 0) {
            const int j = ch * 32 + lane;
            SS.rd1t[j] = __frcp_rn(pow2_scale(fmaxf(SS.bmax[0][j], SS.bmax[1][j])));
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- second products: D1 K^ and D1^T Q^ (B = the k or q tile, MN-major)
    if (tid == 0 && !fail) {
        const uint32_t ib = idesc_f32acc(128, 128, false, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            mma_f32acc_ss(tmem + TM_DK, kdesc(sbase + OFF_D + kk * 32),
                          sdesc_sw128(sbase + OFF_QK + 8192 + kk * 2048, G16, 1024), ib, kk > 0);
            mma_f32acc_ss(tmem + TM_DQ, kdesc(sbase + OFF_D + kk * 32),
                          sdesc_sw128(sbase + OFF_QK + kk * 2048, G16, 1024), ib, kk > 0);
        }
        mma_commit(&SS.mbar[1]);
    }
    // rows 64-127 (warps 2, 3, 6, 7): dW = -(dV' H^T) while the second products run.  The
    // TMEM loads are warp-wide instructions: every lane issues them, live row or not.
    const int j = (sp - 2) * 32 + lane;  // the row's position, for sp >= 2
    if (!fail && sp >= 2) {
        const float rdvj = SS.rdv[j & 63];
        float* dst = p.dW + ((size_t)(j < Cc ? tok(j) : 0) * p.Hv + h) * 128 + ch * 64;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t r[32];
            tmem_ld32(tl + TM_X + ch * 64 + s * 32, r);
            tmem_wait_ld();
            if (j < Cc) {
                const float* rh = SS.rh + ch * 64 + s * 32;
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4)
                    reinterpret_cast<float4*>(dst + s * 32)[e4] = make_float4(
                        -u2f(r[4 * e4]) * rdvj * rh[4 * e4], -u2f(r[4 * e4 + 1]) * rdvj * rh[4 * e4 + 1],
                        -u2f(r[4 * e4 + 2]) * rdvj * rh[4 * e4 + 2], -u2f(r[4 * e4 + 3]) * rdvj * rh[4 * e4 + 3]);
            }
        }
    }
    if (!fail) fail = !mbar_wait_bounded(&SS.mbar[1], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();

    // ---- rows 0-63: dQ^ = D1 K^ + s e^{G'} X, its inter-read decay gradient, then dq
    float acc[64];
    if (!fail && sp < 2) {
        const int i = sp * 32 + lane;
        const bool li = i < Cc;
        const float rd = li ? p.scale * exp2f(SS.Gr[i] * kLog2e) : 0.f;
        const float rdoi = SS.rdo[i], rqi = SS.rq[i], rd1i = SS.rd1[i];
        const uint8_t* qrow = sm + OFF_QK + ch * G16;
        float gs = 0.f, pq = 0.f;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t rx[32], rk[32];
            tmem_ld32(tl + TM_X + ch * 64 + s * 32, rx);
            tmem_ld32(tl + TM_DK + ch * 64 + s * 32, rk);
            tmem_wait_ld();
            const float* rh = SS.rh + ch * 64 + s * 32;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float qf[8];
                f16x8_to_f32(*reinterpret_cast<const uint4*>(qrow + sw128(i, s * 4 + c8)), qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = c8 * 8 + e;
                    const float x = u2f(rx[u]) * rdoi * rh[u];
                    const float a = fmaf(rd, x, u2f(rk[u]) * rd1i);
                    const float qv = qf[e] * rqi;
                    gs = fmaf(qv, x, gs);
                    pq = fmaf(qv, a, pq);
                    acc[s * 32 + u] = a;
                }
            }
        }
        SS.gsum[ch][i] = gs;
        SS.projq[ch][i] = pq;
    }
    // ---- rows 64-127: the P and carry parts of dK^, the carry's decay gradient
    if (!fail && sp >= 2) {
        const bool lj = j < Cc;
        const float kd = lj ? exp2f((SS.G[Cc - 1] - SS.G[j]) * kLog2e) : 0.f;
        const float rvj = SS.rv[j], rkj = SS.rk[j], rd1tj = SS.rd1t[j];
        const uint8_t* krow = sm + OFF_QK + ch * G16 + 8192;
        float* dst = p.dKp + ((size_t)(lj ? tok(j) : 0) * p.Hv + h) * 128 + ch * 64;
        float c = 0.f;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t rz[32], rq[32];
            tmem_ld32(tl + TM_Z + ch * 64 + s * 32, rz);
            tmem_ld32(tl + TM_DQ + ch * 64 + s * 32, rq);
            tmem_wait_ld();
            const float* rdh = SS.rdh + ch * 64 + s * 32;
            float out[32];
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float kf[8];
                f16x8_to_f32(*reinterpret_cast<const uint4*>(krow + sw128(j, s * 4 + c8)), kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = c8 * 8 + e;
                    const float z = u2f(rz[u]) * rvj * rdh[u];
                    c = fmaf(kf[e] * rkj, z, c);
                    out[u] = fmaf(kd, z, u2f(rq[u]) * rd1tj);
                }
            }
            if (lj) {
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4)
                    reinterpret_cast<float4*>(dst + s * 32)[e4] =
                        make_float4(out[4 * e4], out[4 * e4 + 1], out[4 * e4 + 2], out[4 * e4 + 3]);
            }
        }
        SS.ck[ch][j] = c;
    }
    __syncthreads();
    if (!fail && sp < 2) {
        const int i = sp * 32 + lane;
        if (i < Cc) {
            const float iq = SS.invq[i], rqi = SS.rq[i];
            // the CUDA-core kernel's projection sum_d q^_d acc_d = |q|^-1 sum_d q_d acc_d
            const float proj = iq * (SS.projq[0][i] + SS.projq[1][i]);
            const float n = SS.nq[i];
            const float rn = n > kNormEps ? 1.f / n : 1.f / kNormEps;
            const uint8_t* qrow = sm + OFF_QK + ch * G16;
            float* dst = p.dqh + ((size_t)tok(i) * p.Hv + h) * 128 + ch * 64;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                float qf[8];
                f16x8_to_f32(*reinterpret_cast<const uint4*>(qrow + sw128(i, c8)), qf);
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float a = acc[c8 * 8 + e];
                    o[e] = on ? (n > kNormEps ? (a - qf[e] * rqi * iq * proj) * rn : a * rn) : a;
                }
                reinterpret_cast<float4*>(dst)[2 * c8] = make_float4(o[0], o[1], o[2], o[3]);
                reinterpret_cast<float4*>(dst)[2 * c8 + 1] = make_float4(o[4], o[5], o[6], o[7]);
            }
        }
    }
    // ---- decay gradient per position, assembled as bwd_chunk_dqk does
    if (!fail && tid < 64) {
        const int t = tid;
        const bool lt = t < Cc;
        const float kd = lt ? exp2f((SS.G[Cc - 1] - SS.G[t]) * kLog2e) : 0.f;
        const float c = lt ? kd * SS.invk[t] * (SS.ck[0][t] + SS.ck[1][t]) : 0.f;
        SS.c[t] = c;
        const float cs = warp_sum(c);
        if (lane == 0) SS.csum[warp] = cs;
    }
    __syncthreads();
    if (!fail && tid < 64 && tid < Cc) {
        const int t = tid;
        auto dgr = [&](int i) {
            const float rd = p.scale * exp2f(SS.Gr[i] * kLog2e);
            return SS.dGr[0][i] + SS.dGr[1][i] + rd * SS.invq[i] * (SS.gsum[0][i] + SS.gsum[1][i]);
        };
        float g = SS.dGs[0][t] + SS.dGs[1][t] - SS.c[t];
        if (t == Cc - 1) {
            float hd = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) hd += SS.hdot[w];
            g += (SS.csum[0] + SS.csum[1]) + exp2f(SS.G[Cc - 1] * kLog2e) * hd;
        }
        if (!pre) g += dgr(t);
        else if (t + 1 < Cc) g += dgr(t + 1);
        p.dGp[(size_t)tok(t) * p.Hv + h] = g;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (fail && tid == 0) atomicExch(const_cast<int*>(&p.hdr->err), (int)GDR_ERR_TIMEOUT);
}

}  // namespace

bool bwd_dqk_tc_supported(const gdr_chunk_args& a) {
    return a.io_dtype == GDR_BF16 && a.dk == 128 && a.dv == 128 && a.chunk == 64;
}

gdr_status launch_bwd_dqk_tc(const BwdParams& p, dim3 grid, cudaStream_t st) {
    if (cudaFuncSetAttribute(bwd_chunk_dqk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES) != cudaSuccess)
        return GDR_ERR_CUDA;
    bwd_chunk_dqk_tc<<<grid, kTh, SMEM_BYTES, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
