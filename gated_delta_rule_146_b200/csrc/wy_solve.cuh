// wy_solve.cuh -- the blocked unit-lower solve of the chunked WY/UT form, shared by the
// tensor-core kernels, and the small helpers it uses.
//
// T = (I + A)^-1 for a strictly lower 64x64 A (Prizma "seq/delta.py", _solve_unit_lower:
// the unit-lower system of one chunk; flashrt fused_layer.py `_wy_core`: the solve between
// kkt and the W/U recompute), by 16x16 blocks: the four diagonal blocks by column
// substitution, the blocks below them in three phases of tf32 warp MMAs.
#pragma once

#include <cuda_fp16.h>

#include "tc_ptx.cuh"

namespace gdr {

using namespace tc;

// fp16 pair, rounded to nearest.  A value beyond the fp16 range becomes infinite; every
// operand takes part in products that reach the outputs or the state, where it shows as a
// non-finite value (an infinity, or NaN from infinity times zero), and those are checked.
__device__ __forceinline__ uint32_t h2(float a, float b) {
    const __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint4 h8(const float* f) {
    return make_uint4(h2(f[0], f[1]), h2(f[2], f[3]), h2(f[4], f[5]), h2(f[6], f[7]));
}

// max(m, |x|) with NaN propagation: the running magnitude of the outputs and the final state,
// non-finite exactly when one of them is
__device__ __forceinline__ float max_abs_nan(float m, float x) {
    float y;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(m), "f"(fabsf(x)));
    return y;
}

// element (i, j) of a fp32 [64][64] matrix stored with 16-byte chunks XOR-swizzled by row
__device__ __forceinline__ float* f32sw(float* base, int i, int j) {
    return base + i * 64 + ((((j >> 2) ^ (i & 15)) << 2) | (j & 3));
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// Stage 0 of the blocked solve, by the two warps whose rows i (lanes 0-15 and 16-31: one
// diagonal 16x16 block b = i >> 4 each) hold the diagonal blocks of A in `vals` (columns
// 32 hf .. 32 hf + 31 of row i): the block's strictly lower part goes to RS transposed, each
// lane forms column i & 15 of the block's inverse by substitution into Ts, and lanes 16-31
// store the block left of their diagonal block (A_10 or A_32) into As.
__device__ __forceinline__ void wy_diag_stage0(const float (&vals)[32], int i, int lane, int hf,
                                               float* As, float* RS, float* Ts) {
    const bool hi = lane >= 16;
    const int il = i & 15;
    float* at = RS + (i >> 4) * 256;
#pragma unroll
    for (int u = 0; u < 16; ++u)
        at[u * 16 + il] = u < il ? (hi ? vals[16 + u] : vals[u]) : 0.f;
    __syncwarp();
    // P4 stage 0, column il of T_bb (b = i >> 4, one block per half warp):
    //   x_m = [m == il] - sum_{n<m} A_mn x_n, in registers
    {
        const int b0 = i & ~15;
        const float* __restrict__ atr = at;  // atr[j * 16 + m] = A_mj
        float acc[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) acc[m] = 0.f;
        // column jc + 1 of A is loaded while column jc is applied, so each step
        // waits only on its own short chain of FMAs, not on shared memory
        float4 col[2][4];
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4)
            col[0][i4] = *reinterpret_cast<const float4*>(atr + 4 * i4);
#pragma unroll
        for (int jc = 0; jc < 16; ++jc) {
            if (jc < 15) {
#pragma unroll
                for (int i4 = (jc + 2) >> 2; i4 < 4; ++i4)
                    col[(jc + 1) & 1][i4] =
                        *reinterpret_cast<const float4*>(atr + (jc + 1) * 16 + 4 * i4);
            }
            const float xj = jc < il ? 0.f : (jc == il ? 1.f : -acc[jc]);
            acc[jc] = xj;
#pragma unroll
            for (int i4 = (jc + 1) >> 2; i4 < 4; ++i4) {
                const float4 a4 = col[jc & 1][i4];
                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (4 * i4 + u > jc) acc[4 * i4 + u] = fmaf(av[u], xj, acc[4 * i4 + u]);
            }
        }
#pragma unroll
        for (int jc = 0; jc < 16; ++jc) *f32sw(Ts, b0 + jc, b0 + il) = acc[jc];
    }
    if (hi) {
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4)
            *reinterpret_cast<float4*>(f32sw(As, i, hf * 32 + e4 * 4)) =
                make_float4(vals[e4 * 4], vals[e4 * 4 + 1], vals[e4 * 4 + 2], vals[e4 * 4 + 3]);
    }
}

// The blocks of T = (I + A)^-1 below the diagonal, in three phases of tf32 warp MMAs over the
// 256 threads pt of a preparation group (barrier bar_id of bar_n threads), after stage 0:
// Ts holds the diagonal inverses, As the blocks of A below the diagonal, RS is free.  Every
// block of T_w = T diag(bg) and T_u = T diag(bb) goes to twu (fp16, [i][j] K-major 128-byte
// swizzled tiles, T_u 8 KB after T_w) as soon as it is complete; on_phase(1) runs after the
// barrier that completes block columns 3 and 2, on_phase(2) after block column 1; block
// column 0 is complete once the caller's next barrier has passed.
template <typename OnPhase>
__device__ __forceinline__ void wy_solve_offdiag(float* As, float* Ts, float* RS, uint8_t* twu,
                                                 const float* bg, const float* bb, int pt,
                                                 int bar_id, int bar_n, OnPhase&& on_phase) {
    const int lane = pt & 31, pw = pt >> 5;
    named_bar(bar_id, bar_n);
    const int gq = lane >> 2, tq = lane & 3;
    // 16x16 blocks in warp-MMA fragments (tf32, m16n8k8).  Each thread's two k slots
    // are paired with two adjacent columns, so an accumulator block (rows gq, gq + 8;
    // columns 8 nt + 2 tq, +1) is itself the A fragment of its own k half nt.
    using Frag = uint32_t[2][4];  // A fragments of the two k halves
    using Blk = float[2][4];      // accumulator block, by column half
    auto frag_smem = [&](Frag& a, const float* X, int xr, int xc) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int col = 16 * xc + 8 * ks + 2 * tq;
            const float2 lo = *reinterpret_cast<const float2*>(f32sw(const_cast<float*>(X), 16 * xr + gq, col));
            const float2 hi = *reinterpret_cast<const float2*>(f32sw(const_cast<float*>(X), 16 * xr + gq + 8, col));
            a[ks][0] = to_tf32(lo.x); a[ks][1] = to_tf32(hi.x);
            a[ks][2] = to_tf32(lo.y); a[ks][3] = to_tf32(hi.y);
        }
    };
    auto frag_reg = [&](Frag& a, const Blk& e) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            a[ks][0] = to_tf32(e[ks][0]); a[ks][1] = to_tf32(e[ks][2]);
            a[ks][2] = to_tf32(e[ks][1]); a[ks][3] = to_tf32(e[ks][3]);
        }
    };
    // R (+)= X Z, Z the 16x16 block (zr, zc) in shared memory; the four MMAs are
    // independent (one accumulator per k half) and summed at the end
    auto bprod = [&](Blk& R, const Frag& a, const float* Z, int zr, int zc, bool add) {
        float t[2][2][4];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int zrow = 16 * zr + 8 * ks + 2 * tq, zcol = 16 * zc + 8 * nt + gq;
                const uint32_t bf[2] = {to_tf32(*f32sw(const_cast<float*>(Z), zrow, zcol)),
                                        to_tf32(*f32sw(const_cast<float*>(Z), zrow + 1, zcol))};
#pragma unroll
                for (int e = 0; e < 4; ++e) t[ks][nt][e] = 0.f;
                mma_tf32_16x8x8(t[ks][nt], a[ks], bf);
            }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                R[nt][e] = (add ? R[nt][e] : 0.f) + (t[0][nt][e] + t[1][nt][e]);
    };
    // T_w = T diag(beta e^G) and T_u = T diag(beta) (fp16) as [i][j] K-major
    // tiles, the B operands of the W and U~ products, in the -W^T buffer of this
    // chunk (free from the chunk's start until the products have run); each block of
    // T is written there by the warp that completes it
    auto put_twu = [&](int yr, int yc, const Blk& acc) {  // block (yr, yc) = -acc
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int cc = 16 * yc + 8 * nt + 2 * tq;
            const float2 bgp = *reinterpret_cast<const float2*>(&bg[cc]);
            const float2 bp = *reinterpret_cast<const float2*>(&bb[cc]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float t0 = -acc[nt][2 * hh], t1 = -acc[nt][2 * hh + 1];
                const uint32_t off = sw128(16 * yr + gq + 8 * hh, cc >> 3) + (cc & 7) * 2;
                *reinterpret_cast<uint32_t*>(twu + off) = h2(t0 * bgp.x, t1 * bgp.y);
                *reinterpret_cast<uint32_t*>(twu + 8192 + off) = h2(t0 * bp.x, t1 * bp.y);
            }
        }
    };
    auto store_neg = [&](float* Y, int yr, int yc, const Blk& acc) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int rr = 16 * yr + gq, cc = 16 * yc + 8 * nt + 2 * tq;
            *reinterpret_cast<float2*>(f32sw(Y, rr, cc)) = make_float2(-acc[nt][0], -acc[nt][1]);
            *reinterpret_cast<float2*>(f32sw(Y, rr + 8, cc)) = make_float2(-acc[nt][2], -acc[nt][3]);
        }
    };
    // E_rl = T_rr A_rl (r > l);  T_rs = -sum_{l=s}^{r-1} E_rl T_ls.
    //   phase 1: T_10, T_21, T_32 (warps 0-2); Y_20 = E_20 T_00, Y_31 = E_31 T_11,
    //            Y_30 = E_30 T_00 (warps 3-5, which also form the E they need next)
    //   phase 2: T_20 = -(Y_20 + E_21 T_10), T_31 = -(Y_31 + E_32 T_21),
    //            Y_30 += E_31 T_10
    //   phase 3: T_30 = -(Y_30 + E_32 T_20)
    // Warps 6 and 7 write the diagonal and upper blocks of T_w, T_u in phase 1.
    {
        Frag a;
        Blk Y, E1, E2;  // E1, E2: the E blocks a warp keeps for phases 2 and 3
        // E_32 passes from warp 8 (which forms it) to warp 9 (which needs it in phase
        // 3) through the transposed-diagonal buffer, free after stage 0, one
        // accumulator block per lane
        float* e32 = RS + lane * 8;
        if (pw < 6) {
            const int r = pw < 3 ? pw + 1 : (pw == 3 ? 2 : 3);
            const int l = pw < 3 ? pw : (pw == 4 ? 1 : 0);
            Blk E;
            frag_smem(a, Ts, r, r);
            bprod(E, a, As, r, l, false);
            if (pw >= 3) bprod(E1, a, As, r, l + 1, false);  // E_21, E_32, E_31
            if (pw == 4) {
                *reinterpret_cast<float4*>(e32) = make_float4(E1[0][0], E1[0][1], E1[0][2], E1[0][3]);
                *reinterpret_cast<float4*>(e32 + 4) = make_float4(E1[1][0], E1[1][1], E1[1][2], E1[1][3]);
            }
            frag_reg(a, E);
            bprod(Y, a, Ts, l, l, false);
            if (pw < 2) store_neg(Ts, r, l, Y);  // T_10, T_21: read in phase 2
            if (pw < 3) put_twu(r, l, Y);
        } else {
            // row i: its diagonal block from the fp32 T, zeros to its right
            const int i = pt - 192, b = i >> 4;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int j0 = 16 * b + 8 * m;
                const float4 t0 = *reinterpret_cast<const float4*>(f32sw(Ts, i, j0));
                const float4 t1 = *reinterpret_cast<const float4*>(f32sw(Ts, i, j0 + 4));
                const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                const float4 g0 = *reinterpret_cast<const float4*>(&bg[j0]);
                const float4 g1 = *reinterpret_cast<const float4*>(&bg[j0 + 4]);
                const float4 b0 = *reinterpret_cast<const float4*>(&bb[j0]);
                const float4 b1 = *reinterpret_cast<const float4*>(&bb[j0 + 4]);
                const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                uint32_t w4[4], u4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    w4[e] = h2(tv[2 * e] * gv[2 * e], tv[2 * e + 1] * gv[2 * e + 1]);
                    u4[e] = h2(tv[2 * e] * bv[2 * e], tv[2 * e + 1] * bv[2 * e + 1]);
                }
                *reinterpret_cast<uint4*>(twu + sw128(i, 2 * b + m)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                *reinterpret_cast<uint4*>(twu + 8192 + sw128(i, 2 * b + m)) = make_uint4(u4[0], u4[1], u4[2], u4[3]);
            }
            for (int c8 = 2 * b + 2; c8 < 8; ++c8) {
                *reinterpret_cast<uint4*>(twu + sw128(i, c8)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(twu + 8192 + sw128(i, c8)) = make_uint4(0, 0, 0, 0);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(bar_id, bar_n);
        on_phase(1);  // block columns 3 and 2 of T_w, T_u are complete
        if (pw >= 3 && pw < 6) {
            frag_reg(a, E1);
            if (pw == 3) { bprod(Y, a, Ts, 1, 0, true); store_neg(Ts, 2, 0, Y); put_twu(2, 0, Y); }
            if (pw == 4) { bprod(Y, a, Ts, 2, 1, true); put_twu(3, 1, Y); }
            if (pw == 5) bprod(Y, a, Ts, 1, 0, true);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(bar_id, bar_n);
        on_phase(2);  // block column 1
        if (pw == 5) {
            const float4 x0 = *reinterpret_cast<const float4*>(e32);
            const float4 x1 = *reinterpret_cast<const float4*>(e32 + 4);
            E2[0][0] = x0.x; E2[0][1] = x0.y; E2[0][2] = x0.z; E2[0][3] = x0.w;
            E2[1][0] = x1.x; E2[1][1] = x1.y; E2[1][2] = x1.z; E2[1][3] = x1.w;
            frag_reg(a, E2);
            bprod(Y, a, Ts, 2, 0, true);
            put_twu(3, 0, Y);
        }
    }
}

}  // namespace gdr
