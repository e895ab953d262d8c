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
#include "wy_solve.cuh"

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
constexpr uint32_t OFF_D = 147456;
// fp32 row tiles of the stores, over the first products' operands (E, H, dH+)
constexpr uint32_t OFF_TW = 0, OFF_TK = 32768, OFF_TQ = 65536;
static_assert(OFF_TQ + 32768 <= OFF_QK, "row tiles");       // D1k rows 0-63 (K = j) | D1q^T rows 64-127 (K = i)
constexpr uint32_t OFF_SMALL = 163840;

// tensor memory columns (fp32 accumulators, lane = row of the stacked product)
constexpr uint32_t TM_X = 0, TM_Z = 128, TM_P = 256, TM_S = 320, TM_DQ = 256, TM_DK = 384;

struct DqkSmall {
    float4 jf[64];      // per column j: |k_j|^-1 rk_j, rv_j, G_j
    float G[64], Gr[64], invq[64], invk[64], nq[64];
    // reciprocal row factors: 1 / (power of two) of each stored fp16 row
    float rq[64], rk[64], rdo[64], rv[64], rdv[64], rh[128], rdh[128], rd1[64], rd1t[64];
    float amax[2][64];  // largest |D1k| of row i, by column half
    float bmax[2][64];  // largest |D1q^T| of row j, by row warp
    float dGr[2][64];   // row sums of E, by column half
    float dGs[2][64];   // column sums of -E, by row warp
    float gsum[2][64];  // sum_d q_d X_d, by d half
    float ck[2][64];    // sum_d k_d Z_d, by d half
    float c[64];        // the carry's decay gradient per position
    float hdot[8];      // <dH+, H> by warp
    float csum[2];
    uint64_t mbar[2];
    uint32_t tmem;
};
constexpr uint32_t SMEM_BYTES = OFF_SMALL + sizeof(DqkSmall) + 1024;
static_assert(OFF_SMALL + sizeof(DqkSmall) + 1024 <= 227 * 1024, "shared memory");

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

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
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

// four values -> four bf16, rounded to nearest, as one 8-byte word
__device__ __forceinline__ uint2 bf16x4(const float (&o)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]), b = __floats2bfloat162_rn(o[2], o[3]);
    return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
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
        // the setup that no staged value needs goes after the first loads are in flight
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
    if (tid < 64) {
        SS.Gr[tid] = pre ? (tid > 0 ? SS.G[tid - 1] : 0.f) : SS.G[tid];
        SS.jf[tid] = make_float4(SS.invk[tid] * SS.rk[tid], SS.rv[tid], SS.G[tid], 0.f);
    }
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
        // columns inside the mask: j < Cc and j <= i (j < i for the pre-write read)
        const int jend = i < Cc ? min(Cc, pre ? i : i + 1) : 0;
        const float gri = SS.Gr[i], qi = SS.invq[i] * SS.rq[i], ci = p.scale * SS.rdo[i];
        float e[32], bm[32], rsum = 0.f, am = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            const float4 f = SS.jf[j];
            const float d1 = j < jend ? ci * u2f(rp[u]) * f.y * ex2((gri - f.z) * kLog2e) : 0.f;
            a1[u] = d1 * f.x;
            b1[u] = d1 * qi;
            const float ev = a1[u] * (u2f(rs[u]) * qi);
            rsum += ev;
            e[u] = -ev;
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
        // D1k row i and D1q^T rows j in fp16, each with its row's factor (lane u holds row
        // j = 32 ch + u's)
        const float sd = pow2_scale(fmaxf(SS.amax[0][i], SS.amax[1][i]));
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = a1[e8 * 8 + u];
            *reinterpret_cast<uint4*>(sm + OFF_D + sw128(i, ch * 4 + e8)) = f16x8(f, sd);
        }
        const float stl = pow2_scale(fmaxf(SS.bmax[0][ch * 32 + lane], SS.bmax[1][ch * 32 + lane]));
        uint16_t* d1t = reinterpret_cast<uint16_t*>(sm + OFF_D);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            const __half hv = __float2half_rn(b1[u] * __shfl_sync(0xffffffffu, stl, u));
            d1t[(sw128(64 + j, i >> 3) >> 1) + (i & 7)] = *reinterpret_cast<const uint16_t*>(&hv);
        }
        if (ch == 0) SS.rd1[i] = __frcp_rn(sd);
        if (sp == 0) SS.rd1t[ch * 32 + lane] = __frcp_rn(stl);
    }
    // dW, the P and carry parts of dK^ and dQ^ leave as fp32 rows [64][128] staged over the
    // operands the first products read (dO, dV', V', H, dH+); a row's 16-byte piece pc sits
    // at pc ^ (row & 7), so that 32 rows' same piece and one row's 32 pieces both spread over
    // the banks.  One warp per row stores them below.
    auto tile_at = [&](uint32_t off, int row, int pc) {
        return reinterpret_cast<float4*>(sm + off + row * 512 + ((pc ^ (row & 7)) << 4));
    };
    // rows 64-127 (warps 2, 3, 6, 7, idle in D1, which only rows 0-63 take): dW = -(dV' H^T).
    // The TMEM loads are warp-wide instructions: every lane issues them, live row or not.
    const int j = (sp - 2) * 32 + lane;  // the row's position, for sp >= 2
    if (!fail && sp >= 2) {
        const float rdvj = -SS.rdv[j & 63];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t r[32];
            tmem_ld32(tl + TM_X + ch * 64 + s * 32, r);
            tmem_wait_ld();
            const float* rh = SS.rh + ch * 64 + s * 32;
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4)
                *tile_at(OFF_TW, j, ch * 16 + s * 8 + e4) = make_float4(
                    u2f(r[4 * e4]) * rdvj * rh[4 * e4], u2f(r[4 * e4 + 1]) * rdvj * rh[4 * e4 + 1],
                    u2f(r[4 * e4 + 2]) * rdvj * rh[4 * e4 + 2], u2f(r[4 * e4 + 3]) * rdvj * rh[4 * e4 + 3]);
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
    if (!fail) fail = !mbar_wait_bounded(&SS.mbar[1], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();

    // ---- rows 0-63: dQ^ = D1 K^ + s e^{G'} X and its inter-read decay gradient
    if (!fail && sp < 2) {
        const int i = sp * 32 + lane;
        const bool li = i < Cc;
        const float rd = li ? p.scale * ex2(SS.Gr[i] * kLog2e) : 0.f;
        const float rdoi = SS.rdo[i], rqi = SS.rq[i], rd1i = SS.rd1[i];
        const uint8_t* qrow = sm + OFF_QK + ch * G16;
        float gs = 0.f;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t rx[32], rk[32];
            tmem_ld32(tl + TM_X + ch * 64 + s * 32, rx);
            tmem_ld32(tl + TM_DK + ch * 64 + s * 32, rk);
            tmem_wait_ld();
            const float* rh = SS.rh + ch * 64 + s * 32;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float qf[8], a[8];
                f16x8_to_f32(*reinterpret_cast<const uint4*>(qrow + sw128(i, s * 4 + c8)), qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = c8 * 8 + e;
                    const float x = u2f(rx[u]) * rdoi * rh[u];
                    a[e] = fmaf(rd, x, u2f(rk[u]) * rd1i);
                    gs = fmaf(qf[e] * rqi, x, gs);
                }
                *tile_at(OFF_TQ, i, ch * 16 + s * 8 + 2 * c8) = make_float4(a[0], a[1], a[2], a[3]);
                *tile_at(OFF_TQ, i, ch * 16 + s * 8 + 2 * c8 + 1) = make_float4(a[4], a[5], a[6], a[7]);
            }
        }
        SS.gsum[ch][i] = gs;
    }
    // ---- rows 64-127: the P and carry parts of dK^, the carry's decay gradient
    if (!fail && sp >= 2) {
        const bool lj = j < Cc;
        const float kd = lj ? ex2((SS.G[Cc - 1] - SS.G[j]) * kLog2e) : 0.f;
        const float rvj = SS.rv[j], rkj = SS.rk[j], rd1tj = SS.rd1t[j];
        const uint8_t* krow = sm + OFF_QK + ch * G16 + 8192;
        float c = 0.f;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t rz[32], rq[32];
            tmem_ld32(tl + TM_Z + ch * 64 + s * 32, rz);
            tmem_ld32(tl + TM_DQ + ch * 64 + s * 32, rq);
            tmem_wait_ld();
            const float* rdh = SS.rdh + ch * 64 + s * 32;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float kf[8], out[8];
                f16x8_to_f32(*reinterpret_cast<const uint4*>(krow + sw128(j, s * 4 + c8)), kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = c8 * 8 + e;
                    const float z = u2f(rz[u]) * rvj * rdh[u];
                    c = fmaf(kf[e] * rkj, z, c);
                    out[e] = fmaf(kd, z, u2f(rq[u]) * rd1tj);
                }
                *tile_at(OFF_TK, j, ch * 16 + s * 8 + 2 * c8) = make_float4(out[0], out[1], out[2], out[3]);
                *tile_at(OFF_TK, j, ch * 16 + s * 8 + 2 * c8 + 1) = make_float4(out[4], out[5], out[6], out[7]);
            }
        }
        SS.ck[ch][j] = c;
    }
    __syncthreads();
    // Row passes: warp w takes positions 8w .. 8w + 7, lane l the features 4l .. 4l + 3.
    // dq = (dQ^ - q^ (q^ . dQ^)) / |q| (plain 1 / max(|q|, eps) below eps, dQ^ without it)
    if (!fail) {
#pragma unroll 2
        for (int r = 0; r < 8; ++r) {
            const int i = warp * 8 + r;
            if (i >= Cc) break;
            const size_t row = ((size_t)tok(i) * p.Hv + h) * 128;
            reinterpret_cast<float4*>(p.dW + row)[lane] = *tile_at(OFF_TW, i, lane);
            reinterpret_cast<float4*>(p.dKp + row)[lane] = *tile_at(OFF_TK, i, lane);
            const float4 a4 = *tile_at(OFF_TQ, i, lane);
            const int x0 = 4 * lane;
            const uint2 raw = *reinterpret_cast<const uint2*>(
                sm + OFF_QK + (x0 >> 6) * G16 + sw128(i, (x0 >> 3) & 7) + (x0 & 7) * 2);
            const float f = SS.rq[i] * SS.invq[i];
            const float2 q01 = unpack_f16x2(raw.x), q23 = unpack_f16x2(raw.y);
            const float a[4] = {a4.x, a4.y, a4.z, a4.w};
            const float qh[4] = {q01.x * f, q01.y * f, q23.x * f, q23.y * f};
            const float proj = warp_sum(qh[0] * a[0] + qh[1] * a[1] + qh[2] * a[2] + qh[3] * a[3]);
            const float n = SS.nq[i];
            const float rn = n > kNormEps ? 1.f / n : 1.f / kNormEps;
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = on ? (n > kNormEps ? (a[e] - qh[e] * proj) * rn : a[e] * rn) : a[e];
            if (p.direct_out)  // one v-head per key head: dq itself, in bf16
                reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.dq_out) + row)[lane] = bf16x4(o);
            else
                reinterpret_cast<float4*>(p.dqh + row)[lane] = make_float4(o[0], o[1], o[2], o[3]);
        }
    }
    // ---- decay gradient per position, assembled as bwd_chunk_dqk does
    if (!fail && tid < 64) {
        const int t = tid;
        const bool lt = t < Cc;
        const float kd = lt ? ex2((SS.G[Cc - 1] - SS.G[t]) * kLog2e) : 0.f;
        const float c = lt ? kd * SS.invk[t] * (SS.ck[0][t] + SS.ck[1][t]) : 0.f;
        SS.c[t] = c;
        const float cs = warp_sum(c);
        if (lane == 0) SS.csum[warp] = cs;
    }
    __syncthreads();
    if (!fail && tid < 64 && tid < Cc) {
        const int t = tid;
        auto dgr = [&](int i) {
            const float rd = p.scale * ex2(SS.Gr[i] * kLog2e);
            return SS.dGr[0][i] + SS.dGr[1][i] + rd * SS.invq[i] * (SS.gsum[0][i] + SS.gsum[1][i]);
        };
        float g = SS.dGs[0][t] + SS.dGs[1][t] - SS.c[t];
        if (t == Cc - 1) {
            float hd = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) hd += SS.hdot[w];
            g += (SS.csum[0] + SS.csum[1]) + ex2(SS.G[Cc - 1] * kLog2e) * hd;
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


// ============================================================================================
// The WY step: what bwd_chunk_wy (chunk_bwd.cu) computes, on the tensor cores.
//     A     = strict_lower(diag(beta) (K^ K^T) . e^{G_i - G_j}),  T = (I + A)^-1 (blocked solve)
//     dR    = [dR_w | dR_u] = T^T [dW | dV']
//     dA    = -(dR_w W^T + dR_u U~^T) on the strict lower triangle, D = dA . e^{G_i - G_j}
//     dK^   = (beta D + (beta D)^T) K^ + diag(beta e^G) dR_w + (the P and carry parts)
//     dv    = diag(beta) dR_u,  dbeta, dg (reverse cumulative sum of dG within the chunk)
// Products (tcgen05, fp16 operands, fp32 accumulators):
//     P1  [k; -] k^T             rows 0-63: k_i . k_j
//     P2  [dW | dV']^T T         two M = 128 blocks: dR_w^T, dR_u^T (lane = feature, column = i)
//     P3  [dR; -] [W | U~]^T     rows 0-63: -dA
//     P4  K^T (beta D + (beta D)^T)^T     dK^T (lane = d, column = i)
// The solve is the forward's (wy_solve.cuh): the diagonal 16x16 inverses by substitution,
// the blocks below them by tf32 warp MMAs, T written as an fp16 tile.  [dW | dV'] and dR take
// one power-of-two factor per tile (their rows run along a K index); the rows of k and of
// [W | U~] and of the combined beta D take one each.

constexpr int kBarWy = 1, kBarSolve = 2;
constexpr uint32_t W_K = 0;         // k rows (K = d): 2 groups x 8 KB
constexpr uint32_t W_R = 16384;     // [dW | dV'] rows j: 4 groups x 8 KB (x = feature)
constexpr uint32_t W_WF = 49152;    // [W | U~] rows j: 4 groups x 8 KB
constexpr uint32_t W_T = 81920;     // T (fp16, [i][j]), a second copy 8 KB on
constexpr uint32_t W_DR = 98304;    // dR rows i (K = x): 4 groups x 8 KB
constexpr uint32_t W_AS = 131072;   // A below the diagonal (fp32), then beta D (fp32)
constexpr uint32_t W_TS = 147456;   // T (fp32) of the solve
constexpr uint32_t W_RS = 163840;   // the solve's diagonal blocks
constexpr uint32_t W_BS = 167936;   // (beta D + (beta D)^T) diag(1/|k|) rows i (K = j): 8 KB
constexpr uint32_t W_SMALL = 176128;
constexpr uint32_t WT_SK = 0, WT_DRW = 64, WT_DRU = 128, WT_DA = 192, WT_DK = 0;
constexpr uint32_t WT_W = WT_DRW, WT_U = WT_DRU;  // W^T, U~^T until P2 takes the columns
constexpr uint32_t W_V = W_DR;     // beta v rows (K = feature) until the dR epilogue
// the tail's fp32 rows [64][128], over regions no product reads by then: dR_u over the
// upper half of [W | U~] (v takes the lower) and T, dR_w over dR, the P4 part over A and
// the solve's T
constexpr uint32_t W_DRU_S = W_WF + 16384, W_DRW_S = W_DR, W_DK_S = W_AS;
static_assert(W_DRU_S + 32768 <= W_DR && W_DK_S + 32768 <= W_RS, "tail rows");

struct WySmall {
    float4 jf[64];                    // per column j: |k_j|^-1 rk_j, rw_j, G_j
    // column factors of T for W: beta e^G rk |k|^-1 2^16 (the solve reads column factors in
    // pairs, so this array and `ones` are 8-byte aligned)
    alignas(16) float sw[64];
    float G[64], beta[64], ones[64], invk[64], nk[64];
    float rk[64], rw[64], rbs[64];    // reciprocal row factors: k, [W | U~], beta D + ...
    float rr[2], rdr;                 // reciprocal tile factors: dW, dV' halves; dR
    float mx[8][3];                   // per-warp largest magnitudes (dW, dV'; dR)
    float bsmax[2][64];               // largest |Bs'| of row i, by column half
    float dgr[2][64], dgc[2][64], db[2][64];  // from dA: row sums, column sums, beta parts
    float rsum[64], vsum[64];         // k^ . dR_w, v . dR_u per position
    float dgf[64], dbf[64];           // dG and dbeta per position
    float wmx[4][64];                 // largest |W|, |U~| of row j, by feature quarter
    uint64_t mbar[5];
    uint32_t tmem;
    int range_bad;
};
constexpr uint32_t W_SMEM = W_SMALL + sizeof(WySmall) + 1024;
static_assert(offsetof(WySmall, sw) % 8 == 0 && offsetof(WySmall, ones) % 8 == 0, "pair loads");
static_assert(W_SMALL + sizeof(WySmall) + 1024 <= 227 * 1024, "shared memory");

__global__ void __launch_bounds__(kTh, 1) bwd_chunk_wy_tc(BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    WySmall& SS = *reinterpret_cast<WySmall*>(sm + W_SMALL);
    if (p.hdr->err != GDR_OK) return;
    ChunkPos cp;
    if (!chunk_pos(p, cp)) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, ch = warp >> 2;
    const int h = blockIdx.y, hk = h / (p.Hv / p.Hk), Cc = cp.Cc;
    const bool on = p.qk_l2norm != 0;
    auto tok = [&](int i) { return phys_token(cp.t0, cp.t1, cp.p0 + i, p.reverse); };
    float* As = reinterpret_cast<float*>(sm + W_AS);
    float* Ts = reinterpret_cast<float*>(sm + W_TS);

    // ---- staging
    {
        // k rows (bf16), with their norms
        uint4 raw[4];
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + it * kTh, i = idx >> 4, c = idx & 15;
            raw[it] = make_uint4(0, 0, 0, 0);
            if (i < Cc)
                raw[it] = __ldg(static_cast<const uint4*>(p.k) + ((size_t)tok(i) * p.Hk + hk) * 16 + c);
        }
        // the setup that no staged value needs goes after the first loads are in flight
        if (warp == 0) {
            tmem_alloc(&SS.tmem, 256);
            tmem_relinquish();
            tc_fence_before();
        }
        if (tid == 0) {
            for (int b = 0; b < 5; ++b) mbar_init(&SS.mbar[b], 1);
            mbar_init_fence();
            SS.range_bad = 0;
        }
        if (tid < 64) {
            const bool lt = tid < Cc;
            const size_t gi = lt ? (size_t)tok(tid) * p.Hv + h : 0;
            SS.G[tid] = lt ? p.G[gi] : 0.f;
            SS.beta[tid] = lt ? load_elem(p.beta, gi, p.gt) : 0.f;
            SS.ones[tid] = 1.f;
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + it * kTh, i = idx >> 4, c = idx & 15;
            float f[8];
            bf16x8_to_f32(raw[it], f);
            const float sc = pow2_scale(max16(amax8(f)));
            *reinterpret_cast<uint4*>(sm + W_K + (c >> 3) * 8192 + sw128(i, c & 7)) = f16x8(f, sc);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
            ss = sum16(ss);
            if (c == 0) {
                const float n = sqrtf(ss);
                SS.rk[i] = __frcp_rn(sc);
                SS.nk[i] = n;
                SS.invk[i] = on ? 1.f / fmaxf(n, kNormEps) : 1.f;
            }
        }
    }
    // v rows (bf16) in registers, converted to fp16 times beta once beta is visible: the
    // operand of U~ = T (diag(beta) V)
    uint4 vraw[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int idx = tid + it * kTh, i = idx >> 4, c = idx & 15;
        vraw[it] = make_uint4(0, 0, 0, 0);
        if (i < Cc) vraw[it] = __ldg(static_cast<const uint4*>(p.v) + ((size_t)tok(i) * p.Hv + h) * 16 + c);
    }
    // [dW | dV'] (fp32) held in registers until the tile's largest magnitudes are known
    float4 rv[4][2][2];  // [piece][dW, dV'][half]
    {
        float mw = 0.f, mv = 0.f;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + it * kTh, j = idx >> 4, c = idx & 15;
#pragma unroll
            for (int t = 0; t < 2; ++t) rv[it][t][0] = rv[it][t][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < Cc) {
                const size_t row = ((size_t)tok(j) * p.Hv + h) * 128 + c * 8;
                const float4* w4 = reinterpret_cast<const float4*>(p.dW + row);
                const float4* v4 = reinterpret_cast<const float4*>(p.dVp + row);
                rv[it][0][0] = __ldg(w4); rv[it][0][1] = __ldg(w4 + 1);
                rv[it][1][0] = __ldg(v4); rv[it][1][1] = __ldg(v4 + 1);
            }
            float f[8];
            f4x2_to_f32(rv[it][0][0], rv[it][0][1], f);
            mw = fmaxf(mw, amax8(f));
            f4x2_to_f32(rv[it][1][0], rv[it][1][1], f);
            mv = fmaxf(mv, amax8(f));
        }
        mw = warp_max(mw);
        mv = warp_max(mv);
        if (lane == 0) { SS.mx[warp][0] = mw; SS.mx[warp][1] = mv; }
    }
    __syncthreads();
    {
        float mw = 0.f, mv = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) { mw = fmaxf(mw, SS.mx[w][0]); mv = fmaxf(mv, SS.mx[w][1]); }
        const float sw = pow2_scale(mw), sv = pow2_scale(mv);
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + it * kTh, j = idx >> 4, c = idx & 15;
            float f[8];
            f4x2_to_f32(rv[it][0][0], rv[it][0][1], f);
            *reinterpret_cast<uint4*>(sm + W_R + (c >> 3) * 8192 + sw128(j, c & 7)) = f16x8(f, sw);
            f4x2_to_f32(rv[it][1][0], rv[it][1][1], f);
            *reinterpret_cast<uint4*>(sm + W_R + (2 + (c >> 3)) * 8192 + sw128(j, c & 7)) = f16x8(f, sv);
        }
        if (tid == 0) { SS.rr[0] = __frcp_rn(sw); SS.rr[1] = __frcp_rn(sv); }
        // beta v rows in fp16, laid out as the k tile (rows i, K = feature); a value beyond
        // the fp16 range is reported
        bool vbad = false;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + it * kTh, i = idx >> 4, c = idx & 15;
            float f[8];
            bf16x8_to_f32(vraw[it], f);
            const float bi = SS.beta[i];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= bi;
            vbad |= !(amax8(f) <= 65504.f);
            *reinterpret_cast<uint4*>(sm + W_V + (c >> 3) * 8192 + sw128(i, c & 7)) = f16x8(f, 1.f);
        }
        if (vbad) SS.range_bad = 1;
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = SS.tmem;
    const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
    if (tid < 64) {
        const float kf = SS.invk[tid] * SS.rk[tid];
        SS.jf[tid] = make_float4(kf, 0.f, SS.G[tid], 0.f);  // .y = rw once W, U~ are formed
        SS.sw[tid] = SS.beta[tid] * ex2(SS.G[tid] * kLog2e) * kf * 65536.f;
    }

    // ---- P1: k . k
    if (tid == 0) {
        const uint32_t id = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t o = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_f32acc_ss(tmem + WT_SK, kdesc(sbase + W_K + o), kdesc(sbase + W_K + o), id, kk > 0);
        }
        mma_commit(&SS.mbar[0]);
    }
    bool fail = !mbar_wait_bounded(&SS.mbar[0], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();

    // ---- A (rows i = 0-63: warps 0, 1 and 4, 5) and the solve T = (I + A)^-1
    if (!fail) {
        if (sp < 2) {
            const int i = sp * 32 + lane;
            uint32_t rs[32];
            tmem_ld32(tl + WT_SK + ch * 32, rs);
            tmem_wait_ld();
            const float f = SS.beta[i] * SS.rk[i] * SS.invk[i], gi = SS.G[i];
            const int jend = i < Cc ? i : 0;  // strictly lower: j < i
            float vals[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int j = ch * 32 + u;
                const float4 fj = SS.jf[j];
                vals[u] = j < jend ? f * u2f(rs[u]) * fj.x * ex2((gi - fj.z) * kLog2e) : 0.f;
            }
            // the solve's layout: warp 1 holds only blocks below the diagonal, warps 0 and 5 the
            // diagonal blocks (and A_10, A_32), warp 4 none that it reads
            if (warp == 1) {
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4)
                    *reinterpret_cast<float4*>(f32sw(As, i, e4 * 4)) =
                        make_float4(vals[e4 * 4], vals[e4 * 4 + 1], vals[e4 * 4 + 2], vals[e4 * 4 + 3]);
            } else if (warp == 0 || warp == 5) {
                wy_diag_stage0(vals, i, lane, ch, As, reinterpret_cast<float*>(sm + W_RS), Ts);
            }
        }
        // T at W_T (dR and U~), T diag(sw) 8 KB on (W)
        wy_solve_offdiag(As, Ts, reinterpret_cast<float*>(sm + W_RS), sm + W_T, SS.ones, SS.sw, tid,
                         kBarSolve, kTh, [](int) {});
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P1b: W^T = K^T (T diag(sw))^T 2^-16 and U~^T = (diag(beta) V)^T T^T (A = the k or
    //      beta v tile, MN-major; B = T rows j, K-major), into the dR columns
    if (tid == 0 && !fail) {
        const uint32_t id = idesc_f32acc(128, 64, true, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            mma_f32acc_ss(tmem + WT_W, sdesc_sw128(sbase + W_K + kk * 2048, 8192, 1024),
                          kdesc(sbase + W_T + 8192 + kk * 32), id, kk > 0);
            mma_f32acc_ss(tmem + WT_U, sdesc_sw128(sbase + W_V + kk * 2048, 8192, 1024),
                          kdesc(sbase + W_T + kk * 32), id, kk > 0);
        }
        mma_commit(&SS.mbar[4]);
    }
    if (!fail) fail = !mbar_wait_bounded(&SS.mbar[4], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();
    // [W | U~] rows j in fp16 with one factor per row, the B operand of P3 (every warp: lanes
    // = the feature within its quarter, columns = positions 32 ch .. 32 ch + 31)
    if (!fail) {
        uint32_t rwv[32], ruv[32];
        tmem_ld32(tl + WT_W + ch * 32, rwv);
        tmem_ld32(tl + WT_U + ch * 32, ruv);
        tmem_wait_ld();
        float m[32];
#pragma unroll
        for (int u = 0; u < 32; ++u)
            m[u] = max_abs_nan(max_abs_nan(0.f, u2f(rwv[u]) * 0x1p-16f), u2f(ruv[u]));
        bool bad = false;
#pragma unroll
        for (int u = 0; u < 32; ++u) bad |= !(m[u] <= 3.402823e38f);
        if (bad) SS.range_bad = 1;
        SS.wmx[sp][ch * 32 + lane] = transpose_reduce32<true>(m, lane);
        __syncthreads();
        const int jl = ch * 32 + lane;
        const float scl = pow2_scale(fmaxf(fmaxf(SS.wmx[0][jl], SS.wmx[1][jl]), fmaxf(SS.wmx[2][jl], SS.wmx[3][jl])));
        if (sp == 0) {
            SS.rw[jl] = __frcp_rn(scl);
            SS.jf[jl].y = __frcp_rn(scl);
        }
        uint16_t* wf = reinterpret_cast<uint16_t*>(sm + W_WF);
        const int x = sp * 32 + lane;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            const float sc = __shfl_sync(0xffffffffu, scl, u);
            const __half hw = __float2half_rn(u2f(rwv[u]) * 0x1p-16f * sc);
            const __half hu = __float2half_rn(u2f(ruv[u]) * sc);
            const int o = ((x >> 6) * 8192 + sw128(j, (x >> 3) & 7)) / 2 + (x & 7);
            wf[o] = *reinterpret_cast<const uint16_t*>(&hw);
            wf[o + 8192] = *reinterpret_cast<const uint16_t*>(&hu);
        }
    } else {
        __syncthreads();  // the barrier every thread of the branch above takes
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P2: dR^T = [dW | dV']^T T (A and B MN-major)
    if (tid == 0 && !fail) {
        const uint32_t id = idesc_f32acc(128, 64, true, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t b = sdesc_sw128(sbase + W_T + kk * 2048, 8192, 1024);
            mma_f32acc_ss(tmem + WT_DRW, sdesc_sw128(sbase + W_R + kk * 2048, 8192, 1024), b, id, kk > 0);
            mma_f32acc_ss(tmem + WT_DRU, sdesc_sw128(sbase + W_R + 16384 + kk * 2048, 8192, 1024), b, id, kk > 0);
        }
        mma_commit(&SS.mbar[1]);
    }
    if (!fail) fail = !mbar_wait_bounded(&SS.mbar[1], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();
    // dR into shared memory as rows i (K = feature x), one factor for the tile; every warp
    // (lanes: the feature within its block, columns: positions 32 ch .. 32 ch + 31)
    if (!fail) {
        uint32_t ra[32], rb[32];
        tmem_ld32(tl + WT_DRW + ch * 32, ra);
        tmem_ld32(tl + WT_DRU + ch * 32, rb);
        tmem_wait_ld();
        const float r0 = SS.rr[0], r1 = SS.rr[1];
        float m = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            m = max_abs_nan(m, u2f(ra[u]) * r0);
            m = max_abs_nan(m, u2f(rb[u]) * r1);
        }
        m = warp_max(m);
        if (lane == 0) SS.mx[warp][2] = m;
        __syncthreads();
        float mt = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) mt = max_abs_nan(mt, SS.mx[w][2]);
        if (!(mt <= 3.402823e38f) && tid == 0) SS.range_bad = 1;
        const float sd = pow2_scale(mt);
        uint16_t* dr = reinterpret_cast<uint16_t*>(sm + W_DR);
        const int xa = sp * 32 + lane;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int i = ch * 32 + u;
            const __half ha = __float2half_rn(u2f(ra[u]) * r0 * sd);
            const __half hb = __float2half_rn(u2f(rb[u]) * r1 * sd);
            dr[((xa >> 6) * 8192 + sw128(i, (xa >> 3) & 7)) / 2 + (xa & 7)] = *reinterpret_cast<const uint16_t*>(&ha);
            dr[((2 + (xa >> 6)) * 8192 + sw128(i, (xa >> 3) & 7)) / 2 + (xa & 7)] = *reinterpret_cast<const uint16_t*>(&hb);
        }
        if (tid == 0) SS.rdr = __frcp_rn(sd);
    } else {
        __syncthreads();  // the barrier every thread of the branch above takes
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P3: -dA = dR [W | U~]^T (K = 256)
    if (tid == 0 && !fail) {
        const uint32_t id = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            const uint32_t o = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_f32acc_ss(tmem + WT_DA, kdesc(sbase + W_DR + o), kdesc(sbase + W_WF + o), id, kk > 0);
        }
        mma_commit(&SS.mbar[2]);
    }
    if (!fail) fail = !mbar_wait_bounded(&SS.mbar[2], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();
    // the products have read [dW | dV'] and [W | U~]: their regions take the P and carry parts
    // of dK^ (fp32 rows of 512 bytes) and v (bf16 rows of 256 bytes), copied in while the
    // next steps run
    {
        const long long tok0 = tok(0);
#pragma unroll
        for (int it = 0; it < 12; ++it) {
            const int idx = tid + it * kTh;
            const bool isv = idx >= 2048;
            const int i = isv ? (idx - 2048) >> 4 : idx >> 5, c = isv ? idx & 15 : idx & 31;
            const bool valid = i < Cc;
            const size_t row = (size_t)(valid ? tok(i) : tok0) * p.Hv + h;
            const void* src = isv ? static_cast<const void*>(static_cast<const uint4*>(p.v) + row * 16 + c)
                                  : static_cast<const void*>(reinterpret_cast<const uint4*>(p.dKp) + row * 32 + c);
            cp_async16(sbase + (isv ? W_WF + i * 256 : W_R + i * 512) + c * 16, src, valid);
        }
        cp_async_commit();
    }
    // dA -> D, the decay and beta gradients it carries, beta D (rows i: warps 0, 1, 4, 5)
    if (!fail && sp < 2) {
        const int i = sp * 32 + lane;
        uint32_t rd[32], rs[32];
        tmem_ld32(tl + WT_DA + ch * 32, rd);
        tmem_ld32(tl + WT_SK + ch * 32, rs);
        tmem_wait_ld();
        const float bi = SS.beta[i], gi = SS.G[i], fk = SS.rk[i] * SS.invk[i], rdr = -SS.rdr;
        const int jend = i < Cc ? i : 0;  // strictly lower: j < i
        float col[32], bd[32], db = 0.f, dg = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            const float4 fj = SS.jf[j];
            const float dA = u2f(rd[u]) * rdr * fj.y;
            const float sk = u2f(rs[u]) * fk * fj.x;
            const float D = j < jend ? dA * ex2((gi - fj.z) * kLog2e) : 0.f;
            db = fmaf(D, sk, db);
            const float ga = bi * sk * D;
            dg += ga;
            col[u] = -ga;
            bd[u] = bi * D;
        }
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4)
            *reinterpret_cast<float4*>(f32sw(As, i, ch * 32 + e4 * 4)) =
                make_float4(bd[e4 * 4], bd[e4 * 4 + 1], bd[e4 * 4 + 2], bd[e4 * 4 + 3]);
        SS.db[ch][i] = db;
        SS.dgr[ch][i] = dg;
        const float cs = transpose_reduce32<false>(col, lane);
        SS.dgc[sp][ch * 32 + lane] = cs;
        named_bar(kBarWy, 128);
        // Bs'_ij = (beta_i D_ij + beta_j D_ji) / |k_j| / (k_j's factor): the B operand of P4
        float bm = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int j = ch * 32 + u;
            bd[u] = (bd[u] + *f32sw(As, j, i)) * SS.jf[j].x;
            bm = fmaxf(bm, fabsf(bd[u]));
        }
        SS.bsmax[ch][i] = bm;
        named_bar(kBarWy, 128);
        const float sb = pow2_scale(fmaxf(SS.bsmax[0][i], SS.bsmax[1][i]));
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = bd[e8 * 8 + u];
            *reinterpret_cast<uint4*>(sm + W_BS + sw128(i, ch * 4 + e8)) = f16x8(f, sb);
        }
        if (ch == 0) SS.rbs[i] = __frcp_rn(sb);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P4: dK^T = K^T Bs'^T (A = the k tile, MN-major; B = Bs' rows i)
    if (tid == 0 && !fail) {
        const uint32_t id = idesc_f32acc(128, 64, true, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_f32acc_ss(tmem + WT_DK, sdesc_sw128(sbase + W_K + kk * 2048, 8192, 1024),
                          kdesc(sbase + W_BS + kk * 32), id, kk > 0);
        mma_commit(&SS.mbar[3]);
    }
    // dR_w and dR_u (lane = feature, column = position) into shared memory as fp32 rows i
    // while P4 runs; the row passes below read them back one row per warp
    float* drw_s = reinterpret_cast<float*>(sm + W_DRW_S);
    float* dru_s = reinterpret_cast<float*>(sm + W_DRU_S);
    float* dk_s = reinterpret_cast<float*>(sm + W_DK_S);
    if (!fail) {
        const int x = sp * 32 + lane;  // feature: d of dR_w, e of dR_u
        uint32_t ra[32], rb[32];
        tmem_ld32(tl + WT_DRW + ch * 32, ra);
        tmem_ld32(tl + WT_DRU + ch * 32, rb);
        tmem_wait_ld();
        const float r0 = SS.rr[0], r1 = SS.rr[1];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            drw_s[(ch * 32 + u) * 128 + x] = u2f(ra[u]) * r0;
            dru_s[(ch * 32 + u) * 128 + x] = u2f(rb[u]) * r1;
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    // Row passes: warp w takes positions 8w .. 8w + 7, lane l the features 4l .. 4l + 3.
    // k^ of those features: four fp16 values of the staged k tile, times the row's factors.
    const uint16_t* kt = reinterpret_cast<const uint16_t*>(sm + W_K);
    auto khat4 = [&](int i, float (&kh)[4]) {
        const int x0 = 4 * lane;
        const uint2 raw = *reinterpret_cast<const uint2*>(
            kt + ((x0 >> 6) * 8192 + sw128(i, (x0 >> 3) & 7)) / 2 + (x0 & 7));
        const float f = SS.rk[i] * SS.invk[i];
        const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
        const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
        kh[0] = __low2float(h01) * f; kh[1] = __high2float(h01) * f;
        kh[2] = __low2float(h23) * f; kh[3] = __high2float(h23) * f;
    };
    // dv = beta dR_u; v . dR_u and k^ . dR_w per position
    if (!fail) {
        const __nv_bfloat16* vsm = reinterpret_cast<const __nv_bfloat16*>(sm + W_WF);
#pragma unroll 2
        for (int r = 0; r < 8; ++r) {
            const int i = warp * 8 + r;
            if (i >= Cc) break;
            const float4 du = reinterpret_cast<const float4*>(dru_s + i * 128)[lane];
            const float4 dr = reinterpret_cast<const float4*>(drw_s + i * 128)[lane];
            const uint2 vr = *reinterpret_cast<const uint2*>(vsm + i * 128 + 4 * lane);
            const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vr.x));
            const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vr.y));
            float kh[4];
            khat4(i, kh);
            const float bi = SS.beta[i];
            const __nv_bfloat162 o01 = __floats2bfloat162_rn(bi * du.x, bi * du.y);
            const __nv_bfloat162 o23 = __floats2bfloat162_rn(bi * du.z, bi * du.w);
            uint2 ov;
            ov.x = *reinterpret_cast<const uint32_t*>(&o01);
            ov.y = *reinterpret_cast<const uint32_t*>(&o23);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.dv_out) +
                                      ((size_t)tok(i) * p.Hv + h) * 128 + 4 * lane) = ov;
            float vs = v01.x * du.x + v01.y * du.y + v23.x * du.z + v23.y * du.w;
            float rs = kh[0] * dr.x + kh[1] * dr.y + kh[2] * dr.z + kh[3] * dr.w;
            vs = warp_sum(vs);
            rs = warp_sum(rs);
            if (lane == 0) { SS.vsum[i] = vs; SS.rsum[i] = rs; }
        }
    }
    if (!fail) fail = !mbar_wait_bounded(&SS.mbar[3], 0, kWaitNs);
    fail = __syncthreads_or(fail);
    tc_fence_after();
    // the P4 part of dK^ (lane = d, column = i) as fp32 rows i, times the rows' factors of Bs'
    if (!fail) {
        const int x = sp * 32 + lane;
        uint32_t rk4[32];
        tmem_ld32(tl + WT_DK + ch * 32, rk4);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) dk_s[(ch * 32 + u) * 128 + x] = u2f(rk4[u]) * SS.rbs[ch * 32 + u];
    }
    __syncthreads();
    // dK^ = P4 + beta e^G dR_w + (the P and carry parts), then the normalisation's adjoint
    // dk = (dK^ - k^ (k^ . dK^)) / |k| (plain 1 / max(|k|, eps) below eps, dK^ without it)
    if (!fail) {
        const float* dkp = reinterpret_cast<const float*>(sm + W_R);
#pragma unroll 2
        for (int r = 0; r < 8; ++r) {
            const int i = warp * 8 + r;
            if (i >= Cc) break;
            const float4 k4 = reinterpret_cast<const float4*>(dk_s + i * 128)[lane];
            const float4 dr = reinterpret_cast<const float4*>(drw_s + i * 128)[lane];
            const float4 cp4 = reinterpret_cast<const float4*>(dkp + i * 128)[lane];
            const float be = SS.beta[i] * ex2(SS.G[i] * kLog2e);
            float a[4] = {k4.x + be * dr.x + cp4.x, k4.y + be * dr.y + cp4.y,
                          k4.z + be * dr.z + cp4.z, k4.w + be * dr.w + cp4.w};
            float kh[4];
            khat4(i, kh);
            const float proj = warp_sum(kh[0] * a[0] + kh[1] * a[1] + kh[2] * a[2] + kh[3] * a[3]);
            const float n = SS.nk[i], rn = SS.invk[i];  // 1 / max(|k|, eps) when normalising
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = on ? (n > kNormEps ? (a[e] - kh[e] * proj) * rn : a[e] * rn) : a[e];
            const size_t row = ((size_t)tok(i) * p.Hv + h) * 128;
            if (p.direct_out)  // one v-head per key head: dk itself, in bf16
                reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.dk_out) + row)[lane] = bf16x4(o);
            else
                reinterpret_cast<float4*>(p.dkh + row)[lane] = make_float4(o[0], o[1], o[2], o[3]);
        }
    }
    // ---- dG, dbeta per position and dg = the reverse cumulative sum of dG within the chunk
    if (!fail && tid < 64) {
        const int t = tid;
        if (t < Cc) {
            const float r = SS.rsum[t];
            const float eg = ex2(SS.G[t] * kLog2e);
            SS.dgf[t] = p.dGp[(size_t)tok(t) * p.Hv + h] + (SS.dgr[0][t] + SS.dgr[1][t]) +
                        (SS.dgc[0][t] + SS.dgc[1][t]) + SS.beta[t] * eg * r;
            SS.dbf[t] = (SS.db[0][t] + SS.db[1][t]) + eg * r + SS.vsum[t];
        }
    }
    __syncthreads();
    if (!fail && warp == 0) {
        // lane l takes positions 2l and 2l + 1: a suffix sum of the pair sums over the lanes
        const int t0 = 2 * lane, t1 = 2 * lane + 1;
        const float a = t0 < Cc ? SS.dgf[t0] : 0.f, b = t1 < Cc ? SS.dgf[t1] : 0.f;
        float incl = a + b;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += y;
        }
        const float after = incl - (a + b);  // positions 2l + 2 on
        if (t0 < Cc) {
            const size_t gi = (size_t)tok(t0) * p.Hv + h;
            store_elem(p.dg_out, gi, after + b + a, p.gt);
            store_elem(p.dbeta_out, gi, SS.dbf[t0], p.gt);
        }
        if (t1 < Cc) {
            const size_t gi = (size_t)tok(t1) * p.Hv + h;
            store_elem(p.dg_out, gi, after + b, p.gt);
            store_elem(p.dbeta_out, gi, SS.dbf[t1], p.gt);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
    if (tid == 0) {
        if (fail) atomicExch(const_cast<int*>(&p.hdr->err), (int)GDR_ERR_TIMEOUT);
        else if (SS.range_bad) atomicCAS(const_cast<int*>(&p.hdr->err), (int)GDR_OK, (int)GDR_ERR_RANGE);
    }
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

gdr_status launch_bwd_wy_tc(const BwdParams& p, dim3 grid, cudaStream_t st) {
    if (cudaFuncSetAttribute(bwd_chunk_wy_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)W_SMEM) != cudaSuccess)
        return GDR_ERR_CUDA;
    bwd_chunk_wy_tc<<<grid, kTh, W_SMEM, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
