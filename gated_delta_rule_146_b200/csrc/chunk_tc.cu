// chunk_tc.cu -- fused chunk-wise WY/UT forward on the 5th-generation tensor cores.
//
// One CTA (128 threads) per (sequence, value head) walks the sequence's 64-token chunks
// in order.  The fp32 state lives in tensor memory for the whole sequence; nothing but
// q, k, v, g, beta (and S0) is read from HBM and nothing but o (and S_final) is written.
//
// Per chunk, with the in-chunk log decay G_i = g_1 + ... + g_i (Prizma "seq/delta.py",
// chunked_delta: cumulative decay in log space; flashrt fused_layer.py `_wy_core`:
// kkt -> triangular solve -> recompute W/U -> chunk state -> output):
//
//   [K;Q] K^T                        one M=128 MMA gives K K^T and Q K^T
//   A_ij = beta_i (k_i.k_j) e^(G_i-G_j), j<i         (fp32, CUDA cores)
//   T = (I + A)^-1                                  (fp32 forward substitution)
//   W = T diag(beta e^G) K,  U~ = T diag(beta) V     (MMA)
//   V' = U~ - W H                                   (MMA, accumulating onto U~)
//   o = diag(scale e^G') Q H + P V',  P = scale (Q K^T)(.)decay mask   (MMA x2)
//   H <- e^(G_C) H + (diag(e^(G_C - G)) K)^T V'     (MMA into the TMEM state)
//
// Orientation: every product is written transposed so that its M dimension is a head
// dimension (128): accumulators hold rows of W^T, U~^T, V'^T, O^T and H^T, one TMEM lane
// per dk or dv index, one column per token (or per dk for the state).  Every MMA is then
// M=128, N=64 or 128, and every TMEM->shared epilogue writes whole 128-byte rows.  A and
// B operands are 16-bit in shared memory in the 128-byte-swizzled canonical layouts
// (K-major or MN-major as each product needs); accumulation and the state are fp32.
//
// Operand precision: V and T diag(beta) are bf16 (V arrives in bf16); every other operand
// (normalised q and k, T diag(beta e^G), W, the state copy, V', P) is rounded to fp16,
// whose 11-bit significand keeps the chain of roundings well inside the bf16 parity bound
// at long sequence lengths where bf16 operands do not.  The fp16 range is checked wherever
// an operand is produced; a value beyond it sets GDR_ERR_RANGE.
//
// The state H is kept transposed in TMEM (lane = dv, column = dk).  After each chunk the
// epilogue reads it once, writes the fp16 copy the next chunk's MMAs consume, and scales
// it in place by the next chunk's total decay, so the next state update accumulates onto
// it directly.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdr {

namespace {

using namespace tc;

constexpr int C = 64;            // chunk length
constexpr int D = 128;           // dk = dv
constexpr int kThreads = 128;    // one thread per TMEM lane
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// shared memory map (bytes from a 1024-byte-aligned base)
constexpr uint32_t OFF_KQ0 = 0;        // 2 x 16 KB atoms (dk halves): K rows 0-63, Q rows 64-127
constexpr uint32_t OFF_KQ1 = 32768;    // second buffer (next chunk)
constexpr uint32_t OFF_V0 = 65536;     // 2 x 8 KB (dv halves): V rows 0-63
constexpr uint32_t OFF_V1 = 81920;
constexpr uint32_t OFF_TW = 98304;     // T diag(beta e^G), [i][j] fp16
constexpr uint32_t OFF_TU = 106496;    // T diag(beta), [i][j] bf16
constexpr uint32_t OFF_OS = 98304;     // output staging [tok][dv] bf16 (aliases TW, TU)
constexpr uint32_t OFF_P = 114688;     // P [i][j] fp16
constexpr uint32_t OFF_WN = 122880;    // -W^T as [dk][tok] fp16
constexpr uint32_t OFF_AS = 122880;    // A fp32 [64][64] (aliases WN; dead before WN is written)
constexpr uint32_t OFF_HB = 139264;    // H^T fp16 [dv][dk], 2 x 16 KB atoms (dk halves)
constexpr uint32_t OFF_VP = 172032;    // V'^T fp16 [dv][tok]
constexpr uint32_t OFF_SMALL = 188416;
constexpr uint32_t SMEM_BYTES = OFF_SMALL + 2048 + 1024;

// TMEM columns (fp32)
constexpr uint32_t TM_D0 = 0, TM_DW = 64, TM_DU = 128, TM_DO = 192, TM_HM = 256;
constexpr uint32_t TM_COLS = 512;

struct Small {
    float g[2][C];        // raw log decays of the current / next chunk
    float b[2][C];        // beta
    float G[C];           // in-chunk cumulative log decay
    float Kd[C];          // e^(G_last - G_i) for valid rows, 0 beyond the chunk
    float gsum_part[2];   // partial sums of the next chunk's g
    uint64_t mbar[4];
    uint32_t tmem_base;
};
static_assert(sizeof(Small) <= 2048, "small shared block");

struct TcParams {
    const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
    const void* g; const void* beta; const float* S0;
    __nv_bfloat16* o; float* S_final;
    WsHeader* hdr; const int32_t* cu;
    int Hk, Hv, read_pre, qk_l2norm, reverse, o_acc;
    gdr_dtype gt;
    float scale;
};

constexpr float kF16Max = 65000.f;  // operands at or beyond this (or NaN) raise GDR_ERR_RANGE

// fp16 pair with a range check: `bad` is set when either value is not finite or too large
__device__ __forceinline__ uint32_t h2(float a, float b, bool& bad) {
    bad |= !(fabsf(a) < kF16Max) || !(fabsf(b) < kF16Max);
    return pack_f16x2(a, b);
}

__device__ __forceinline__ uint4 h8(const float* f, bool& bad) {
    return make_uint4(h2(f[0], f[1], bad), h2(f[2], f[3], bad), h2(f[4], f[5], bad),
                      h2(f[6], f[7], bad));
}

// 8 fp16 scaled by f (|f| <= 1 at every call site, so the range cannot grow)
__device__ __forceinline__ uint4 scale_f16x8(uint4 u, float f) {
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = unpack_f16x2(w[e]);
        w[e] = pack_f16x2(x.x * f, x.y * f);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kThreads, 1) chunk_fused_tc(TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    Small& SS = *reinterpret_cast<Small*>(sm + OFF_SMALL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (p.hdr->err != GDR_OK) return;

    const int s = blockIdx.x, h = blockIdx.y;
    const int hk = h / (p.Hv / p.Hk);
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);
    const int nchunks = (L + C - 1) / C;
    const size_t sb = ((size_t)s * p.Hv + h) * D * D;

    if (nchunks == 0) {  // empty sequence: the state passes through
        if (p.S_final)
            for (int e = tid; e < D * D; e += kThreads)
                p.S_final[sb + e] = p.S0 ? p.S0[sb + e] : 0.f;
        return;
    }

    if (warp == 0) {
        tmem_alloc(&SS.tmem_base, TM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&SS.mbar[i], 1);
        mbar_init_fence();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = SS.tmem_base;
    const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's 32 lanes

    auto load_chunk = [&](int c, int buf) {
        const int Cc = min(C, L - c * C);
        const uint32_t kq = sbase + (buf ? OFF_KQ1 : OFF_KQ0);
        const uint32_t vv = sbase + (buf ? OFF_V1 : OFF_V0);
        for (int idx = tid; idx < 3 * C * 16; idx += kThreads) {
            const int tile = idx >> 10, rem = idx & 1023, i = rem >> 4, cd = rem & 15;
            const bool valid = i < Cc;
            const long long t = valid ? phys_token(t0, t1, c * C + i, p.reverse) : t0;
            const __nv_bfloat16* src;
            uint32_t dst;
            if (tile == 0) {
                src = p.k + ((size_t)t * p.Hk + hk) * D + cd * 8;
                dst = kq + (cd >> 3) * 16384 + sw128(i, cd & 7);
            } else if (tile == 1) {
                src = p.q + ((size_t)t * p.Hk + hk) * D + cd * 8;
                dst = kq + (cd >> 3) * 16384 + 8192 + sw128(i, cd & 7);
            } else {
                src = p.v + ((size_t)t * p.Hv + h) * D + cd * 8;
                dst = vv + (cd >> 3) * 8192 + sw128(i, cd & 7);
            }
            cp_async16(dst, src, valid);
        }
    };
    auto load_gates = [&](int c, float& gv, float& bv) {
        const int Cc = min(C, L - c * C);
        gv = 0.f;
        bv = 0.f;
        if (tid < Cc) {
            const long long t = phys_token(t0, t1, c * C + tid, p.reverse);
            gv = load_elem(p.g, (size_t)t * p.Hv + h, p.gt);
            bv = load_elem(p.beta, (size_t)t * p.Hv + h, p.gt);
        }
    };
    // every thread polls the barrier, then all agree (a timeout anywhere stops the CTA)
    auto wait_mma = [&](int idx, uint32_t parity) -> bool {
        const bool ok = mbar_wait_bounded(&SS.mbar[idx], parity, kWaitLimitNs);
        const int all = __syncthreads_and(ok ? 1 : 0);
        tc_fence_after();
        return all != 0;
    };

    // ---- prologue: chunk 0 in flight, initial state into TMEM (pre-scaled) and fp16 copy
    bool bad = false;  // an fp16 operand out of range
    float g_nx, b_nx;
    load_chunk(0, 0);
    cp_async_commit();
    load_gates(0, g_nx, b_nx);
    if (tid < C) { SS.g[0][tid] = g_nx; SS.b[0][tid] = b_nx; }
    {
        const float part = warp_sum(tid < C ? g_nx : 0.f);
        if (lane == 0 && warp < 2) SS.gsum_part[warp] = part;
    }
    __syncthreads();
    {
        const float gam = expf(SS.gsum_part[0] + SS.gsum_part[1]);
        const int j = tid;
        for (int d0 = 0; d0 < D; d0 += 32) {
            uint32_t r[32];
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
                float hv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int d = d0 + e8 * 8 + u;
                    hv[u] = p.S0 ? p.S0[sb + (size_t)d * D + j] : 0.f;
                    r[e8 * 8 + u] = __float_as_uint(hv[u] * gam);
                }
                const int cd = (d0 >> 3) + e8;
                *reinterpret_cast<uint4*>(sm + OFF_HB + (cd >> 3) * 16384 + sw128(j, cd & 7)) =
                    h8(hv, bad);
            }
            tmem_st32(tlane + TM_HM + d0, r);
        }
        tmem_wait_st();
    }

    bool failed = false;
    for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        const uint32_t par = (uint32_t)(c & 1);
        const int Cc = min(C, L - c * C);
        const uint32_t KQ = sbase + (buf ? OFF_KQ1 : OFF_KQ0);
        const uint32_t VV = sbase + (buf ? OFF_V1 : OFF_V0);
        uint8_t* KQp = sm + (buf ? OFF_KQ1 : OFF_KQ0);
        const bool has_next = c + 1 < nchunks;

        if (has_next) load_chunk(c + 1, buf ^ 1);
        cp_async_commit();
        if (has_next) load_gates(c + 1, g_nx, b_nx);
        cp_async_wait<1>();
        fence_proxy_async_smem();
        __syncthreads();

        // ---- A: the 128 rows of [K; Q]: bf16 -> (L2-normalised) fp16 in place; cumsum of g
        {
            uint4 vals[16];
            float ss = 0.f;
#pragma unroll
            for (int cd = 0; cd < 16; ++cd) {
                vals[cd] = *reinterpret_cast<const uint4*>(KQp + (cd >> 3) * 16384 +
                                                           sw128(tid, cd & 7));
                const uint32_t w[4] = {vals[cd].x, vals[cd].y, vals[cd].z, vals[cd].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16x2(w[e]);
                    ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
                }
            }
            const float inv = p.qk_l2norm ? 1.f / fmaxf(sqrtf(ss), kNormEps) : 1.f;
#pragma unroll
            for (int cd = 0; cd < 16; ++cd) {
                const uint32_t w[4] = {vals[cd].x, vals[cd].y, vals[cd].z, vals[cd].w};
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16x2(w[e]);
                    f[2 * e] = x.x * inv;
                    f[2 * e + 1] = x.y * inv;
                }
                *reinterpret_cast<uint4*>(KQp + (cd >> 3) * 16384 + sw128(tid, cd & 7)) =
                    h8(f, bad);
            }
        }
        if (warp == 0) {
            const float a0 = SS.g[buf][2 * lane], a1 = SS.g[buf][2 * lane + 1];
            const float pair = a0 + a1;
            float incl = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float excl = incl - pair;
            SS.G[2 * lane] = excl + a0;
            SS.G[2 * lane + 1] = excl + a0 + a1;
        }
        __syncthreads();
        if (tid < C) SS.Kd[tid] = tid < Cc ? expf(SS.G[Cc - 1] - SS.G[tid]) : 0.f;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- B: D0 = [K;Q] K^T  (M=128, N=64, K=128)
        if (tid == 0) {
            const uint32_t id = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_f32acc_ss(tmem + TM_D0, sdesc_sw128(KQ + off, 16, 1024),
                              sdesc_sw128(KQ + off, 16, 1024), id, kk > 0);
            }
            mma_commit(&SS.mbar[0]);
        }
        if (!wait_mma(0, par)) { failed = true; break; }

        // ---- C: A (fp32, rows 0-63) and P (fp16, rows 64-127) from D0; Q -> Q~ in place
        {
            const int i = tid & 63;
            const bool isK = tid < C;
            const float Gi = SS.G[i];
            const float Gr = p.read_pre ? (i > 0 ? SS.G[i - 1] : 0.f) : Gi;
            const float bi = SS.b[buf][i];
            float* As = reinterpret_cast<float*>(sm + OFF_AS);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tlane + TM_D0 + half * 32, r);
                tmem_wait_ld();
                if (isK) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        float a[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int j = half * 32 + e4 * 4 + u;
                            a[u] = j < i ? bi * __uint_as_float(r[e4 * 4 + u]) * expf(Gi - SS.G[j])
                                         : 0.f;
                        }
                        const int cj = half * 8 + e4;
                        *reinterpret_cast<float4*>(As + i * 64 + ((cj ^ (i & 15)) << 2)) =
                            make_float4(a[0], a[1], a[2], a[3]);
                    }
                } else {
#pragma unroll
                    for (int e8 = 0; e8 < 4; ++e8) {
                        float pv[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int j = half * 32 + e8 * 8 + u;
                            const bool on = p.read_pre ? (j < i) : (j <= i);
                            pv[u] = on ? p.scale * __uint_as_float(r[e8 * 8 + u]) * expf(Gr - SS.G[j])
                                       : 0.f;
                        }
                        *reinterpret_cast<uint4*>(sm + OFF_P + sw128(i, half * 4 + e8)) =
                            h8(pv, bad);
                    }
                }
            }
            if (!isK) {
                const float f = p.scale * expf(Gr);
#pragma unroll
                for (int cd = 0; cd < 16; ++cd) {
                    uint4* ptr = reinterpret_cast<uint4*>(KQp + (cd >> 3) * 16384 + 8192 +
                                                          sw128(i, cd & 7));
                    const uint4 u = *ptr;
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                    float fv[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = unpack_f16x2(w[e]);
                        fv[2 * e] = x.x * f;
                        fv[2 * e + 1] = x.y * f;
                    }
                    *ptr = h8(fv, bad);
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- D: T = (I + A)^-1 by forward substitution, one column per thread
        if (tid < C) {
            const int c0 = tid;
            const float* As = reinterpret_cast<const float*>(sm + OFF_AS);
            float x[C];
#pragma unroll
            for (int i = 0; i < C; ++i) x[i] = 0.f;
#pragma unroll
            for (int i = 0; i < C; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int j4 = 0; j4 < (i + 3) / 4; ++j4) {
                    const float4 a = *reinterpret_cast<const float4*>(As + i * 64 +
                                                                      ((j4 ^ (i & 15)) << 2));
                    acc = fmaf(a.x, x[4 * j4 + 0], acc);
                    acc = fmaf(a.y, x[4 * j4 + 1], acc);
                    acc = fmaf(a.z, x[4 * j4 + 2], acc);
                    acc = fmaf(a.w, x[4 * j4 + 3], acc);
                }
                x[i] = i < c0 ? 0.f : (i == c0 ? 1.f : -acc);
            }
            const float fu = SS.b[buf][c0];
            const float fw = fu * expf(SS.G[c0]);
            uint8_t* tw = sm + OFF_TW;
            uint8_t* tu = sm + OFF_TU;
#pragma unroll
            for (int i = 0; i < C; ++i) {
                const uint32_t off = sw128(i, c0 >> 3) + (c0 & 7) * 2;
                const float tw_v = x[i] * fw;
                bad |= !(fabsf(tw_v) < kF16Max);
                *reinterpret_cast<__half*>(tw + off) = __float2half_rn(tw_v);
                *reinterpret_cast<__nv_bfloat16*>(tu + off) = __float2bfloat16_rn(x[i] * fu);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- E: W^T = K^T T_w^T (fp16) and U~^T = V^T T_u^T (bf16)  (M=128, N=64, K=64)
        if (tid == 0) {
            const uint32_t idw = idesc_f32acc(128, 64, true, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f32acc_ss(tmem + TM_DW, sdesc_sw128(KQ + kk * 2048, 16384, 1024),
                              sdesc_sw128(sbase + OFF_TW + kk * 32, 16, 1024), idw, kk > 0);
            const uint32_t idu = idesc_f32acc(128, 64, true, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f32acc_ss(tmem + TM_DU, sdesc_sw128(VV + kk * 2048, 8192, 1024),
                              sdesc_sw128(sbase + OFF_TU + kk * 32, 16, 1024), idu, kk > 0);
            mma_commit(&SS.mbar[1]);
        }
        if (!wait_mma(1, par)) { failed = true; break; }

        // ---- F: -W^T rows -> WN (B operand, MN-major); K -> K~ = diag(Kd) K in place
        {
            const int d = tid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tlane + TM_DW + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = -__uint_as_float(r[e8 * 8 + u]);
                    *reinterpret_cast<uint4*>(sm + OFF_WN + sw128(d, half * 4 + e8)) = h8(f, bad);
                }
            }
            if (tid < C) {
                const float f = SS.Kd[tid];
#pragma unroll
                for (int cd = 0; cd < 16; ++cd) {
                    uint4* ptr = reinterpret_cast<uint4*>(KQp + (cd >> 3) * 16384 +
                                                          sw128(tid, cd & 7));
                    *ptr = scale_f16x8(*ptr, f);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- G: V'^T = U~^T + H^T (-W^T);  O^T = H^T Q~^T   (M=128, N=64, K=128)
        if (tid == 0) {
            const uint32_t id1 = idesc_f32acc(128, 64, false, true, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t hoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_f32acc_ss(tmem + TM_DU, sdesc_sw128(sbase + OFF_HB + hoff, 16, 1024),
                              sdesc_sw128(sbase + OFF_WN + kk * 2048, 8192, 1024), id1, 1);
            }
            const uint32_t id2 = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t hoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_f32acc_ss(tmem + TM_DO, sdesc_sw128(sbase + OFF_HB + hoff, 16, 1024),
                              sdesc_sw128(KQ + hoff + 8192, 16, 1024), id2, kk > 0);
            }
            mma_commit(&SS.mbar[2]);
        }
        if (!wait_mma(2, par)) { failed = true; break; }

        // ---- H: V'^T rows -> VP (fp16); stage the next chunk's gates
        {
            const int j = tid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tlane + TM_DU + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    const float* f = reinterpret_cast<const float*>(r + e8 * 8);
                    *reinterpret_cast<uint4*>(sm + OFF_VP + sw128(j, half * 4 + e8)) = h8(f, bad);
                }
            }
            if (has_next && tid < C) { SS.g[buf ^ 1][tid] = g_nx; SS.b[buf ^ 1][tid] = b_nx; }
            if (warp < 2) {
                const float part = warp_sum(has_next ? g_nx : 0.f);
                if (lane == 0) SS.gsum_part[warp] = part;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- I: O^T += V'^T P^T (N=64, K=64);  H^T += V'^T K~ (N=128, K=64, B MN-major)
        if (tid == 0) {
            const uint32_t id3 = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f32acc_ss(tmem + TM_DO, sdesc_sw128(sbase + OFF_VP + kk * 32, 16, 1024),
                              sdesc_sw128(sbase + OFF_P + kk * 32, 16, 1024), id3, 1);
            const uint32_t id4 = idesc_f32acc(128, 128, false, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f32acc_ss(tmem + TM_HM, sdesc_sw128(sbase + OFF_VP + kk * 32, 16, 1024),
                              sdesc_sw128(KQ + kk * 2048, 16384, 1024), id4, 1);
            mma_commit(&SS.mbar[3]);
        }
        if (!wait_mma(3, par)) { failed = true; break; }

        // ---- J: O^T -> staging -> global; state -> fp16 copy, pre-scaled for the next chunk
        {
            const int j = tid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tlane + TM_DO + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int tok = half * 32 + e;
                    *reinterpret_cast<__nv_bfloat16*>(sm + OFF_OS + tok * 256 +
                                                      (((j >> 3) ^ (tok & 15)) << 4) + (j & 7) * 2) =
                        __float2bfloat16_rn(__uint_as_float(r[e]));
                }
            }
            const float gam = has_next ? expf(SS.gsum_part[0] + SS.gsum_part[1]) : 1.f;
#pragma unroll
            for (int d0 = 0; d0 < D; d0 += 32) {
                uint32_t r[32];
                tmem_ld32(tlane + TM_HM + d0, r);
                tmem_wait_ld();
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    const float* f = reinterpret_cast<const float*>(r + e8 * 8);
                    const int cd = (d0 >> 3) + e8;
                    *reinterpret_cast<uint4*>(sm + OFF_HB + (cd >> 3) * 16384 + sw128(j, cd & 7)) =
                        h8(f, bad);
                }
                if (has_next) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * gam);
                    tmem_st32(tlane + TM_HM + d0, r);
                } else if (p.S_final) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        p.S_final[sb + (size_t)(d0 + e) * D + j] = __uint_as_float(r[e]);
                }
            }
            if (has_next) tmem_wait_st();
        }
        __syncthreads();
        for (int idx = tid; idx < Cc * 16; idx += kThreads) {
            const int tok = idx >> 4, cd = idx & 15;
            uint4 val = *reinterpret_cast<const uint4*>(sm + OFF_OS + tok * 256 +
                                                        ((cd ^ (tok & 15)) << 4));
            const long long t = phys_token(t0, t1, c * C + tok, p.reverse);
            uint4* dst = reinterpret_cast<uint4*>(p.o + ((size_t)t * p.Hv + h) * D + cd * 8);
            if (p.o_acc) {
                const uint4 old = *dst;
                const uint32_t a[4] = {val.x, val.y, val.z, val.w};
                const uint32_t b2[4] = {old.x, old.y, old.z, old.w};
                uint32_t out[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16x2(a[e]), y = unpack_bf16x2(b2[e]);
                    out[e] = pack_bf16x2(x.x + y.x, x.y + y.y);
                }
                val = make_uint4(out[0], out[1], out[2], out[3]);
            }
            *dst = val;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (failed) {
        if (tid == 0) atomicExch(&p.hdr->err, (int)GDR_ERR_TIMEOUT);
        cp_async_wait<0>();
    }
    if (__syncthreads_or(bad ? 1 : 0) && tid == 0)
        atomicCAS(&p.hdr->err, (int)GDR_OK, (int)GDR_ERR_RANGE);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

bool tc_supported(const gdr_chunk_args& a) {
    return a.io_dtype == GDR_BF16 && a.dk == D && a.dv == D && a.chunk == C;
}

gdr_status launch_chunk_tc(const gdr_chunk_args& a, const void* q, const void* k, const void* v,
                           const void* g, const void* beta, const float* S0, void* o,
                           float* S_final, void* ws, const WsLayout& L, cudaStream_t st) {
    char* base = static_cast<char*>(ws);
    TcParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.g = g; p.beta = beta; p.S0 = S0;
    p.o = static_cast<__nv_bfloat16*>(o); p.S_final = S_final;
    p.hdr = reinterpret_cast<WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.Hk = a.Hk; p.Hv = a.Hv; p.read_pre = a.read_mode == GDR_READ_PRE;
    p.qk_l2norm = a.qk_l2norm; p.reverse = a.reverse; p.o_acc = a.o_accumulate;
    p.gt = a.gate_dtype; p.scale = a.scale;
    if (cudaFuncSetAttribute(chunk_fused_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES) != cudaSuccess)
        return GDR_ERR_CUDA;
    dim3 grid((unsigned)a.n_seqs, (unsigned)a.Hv);
    chunk_fused_tc<<<grid, kThreads, SMEM_BYTES, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
