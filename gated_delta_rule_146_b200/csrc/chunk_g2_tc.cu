// chunk_g2_tc.cu -- GDN-2 (decoupled per-channel gates) chunked forward on the tensor cores.
//
// Rondo-Exp tiny_gdn/fugue.py, BidirectionalGatedDeltaNet2 docstring: per token,
//     S_t = (I - k_t (b_t . k_t)^T) Diag(e^{g_t}) S_{t-1} + k_t (w_t . v_t)^T,
// with a log decay g and an erase gate b per key channel and a write gate w per value
// channel.  With G_t the per-channel cumulative log decay of a chunk (G_{-1} = 0), H (= S^T)
// the state at its start and T = (I + A)^-1, the chunk's WY/UT form (derived as Prizma
// "seq/delta.py", chunked_delta, derives the scalar one) is
//     A_ts = sum_d b_td k_td k_sd e^{G_td - G_sd}       (s < t)
//     W = T (b . e^{G} . K),   U~ = T (w . V),   V' = U~ - W H
//     o_t = q~_t H + sum_{s <= t (post) / < t (pre)} P_ts V'_s,
//         q~_t = scale e^{G'_t} . q_t,   P_ts = scale sum_d q_td k_sd e^{G'_td - G_sd}
//     H <- e^{G_C} . H + K~^T V',   K~_s = e^{G_C - G_s} . k_s
// (G' = G_t for the post-write read, G_{t-1} for the pre-write read; q, k L2-normalised.)
//
// Two kernels.  chunk_g2_prep_tc: a grid over every (chunk, value head) item computes q~,
// -W, K~, U~^T, P (fp16) and e^{G_C} (fp32) into the workspace, laid out as the shared-memory
// image the second kernel consumes.  chunk_g2_chain_tc: one CTA per (sequence, value head)
// streams its items (one bulk copy each) and runs the state recursion on the tensor cores
// with the fp32 state resident in tensor memory.
//
// The decayed pair sums A and P take tf32 warp MMAs over 16-row blocks: for row block I,
// with the reference R_I = G_{16 I + 7} (per channel),
//     e^{G_td - G_sd} = e^{G_td - R_Id} e^{R_Id - G_sd},
// the row operand b_t k_t e^{G_t - R_I} (or q_t e^{G'_t - R_I}) against the column operand
// k_s e^{R_I - G_s} for every s <= 16 I + 15.  Both factors stay within the decay over eight
// tokens of 1 for the block's own columns and are <= 1 for the earlier blocks' while the
// decay does not grow; a chunk where one of these factors would exceed 2^100 (a decay that
// grows that much) is refused with GDR_ERR_RANGE, as the fp32 range could not hold it.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"

#include "tc_ptx.cuh"
#include "wy_solve.cuh"

namespace gdr {

namespace {

using namespace tc;

constexpr int C = 64;      // chunk length
constexpr int D = 128;     // dk = dv
constexpr int kPrepThreads = 256;
constexpr int kBarG2 = 1;  // the prep kernel's named barrier (all threads)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

// The item record: the chain kernel's shared-memory image of one (chunk, head).
//   q~, -W, K~ : [64 tokens][128] fp16, two [64][64] halves (8 KB each) in the 128-byte
//                swizzled K-major layout
//   U~^T       : [128 dv][64 tokens] fp16, 128-byte rows, swizzled
//   P          : [64][64] fp16, swizzled K-major
//   decay      : e^{G_C} [128] fp32
constexpr uint32_t REC_Q = 0, REC_W = 16384, REC_K = 32768, REC_U = 49152, REC_P = 65536,
                   REC_D = 73728;
constexpr uint32_t kRecBytes = 74240;
static_assert(kRecBytes == kG2RecordBytes, "record size");

struct G2Params {
    const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
    const __nv_bfloat16* g; const __nv_bfloat16* b; const __nv_bfloat16* w;
    const float* S0; float* S_final; __nv_bfloat16* o;
    WsHeader* hdr; const int32_t* cu; const int32_t* chunk_off; const int32_t* chunk_seq;
    const int32_t* order;
    uint8_t* rec;
    int Hk, Hv, read_pre, qk_l2norm, tma_store;
    float scale;
};

// byte offset of element (row r, column c) of a [rows][128] 16-bit tile held as two swizzled
// [rows][64] halves of `half_bytes` each
__device__ __forceinline__ uint32_t tile16(int r, int c, uint32_t half_bytes) {
    return (uint32_t)(c >> 6) * half_bytes + sw128(r, (c & 63) >> 3) + (uint32_t)(c & 7) * 2;
}

__device__ __forceinline__ float bf(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

// eight consecutive fp32 values (16-byte aligned) into registers
__device__ __forceinline__ void load_row8(float (&v)[8], const float* src) {
    const float4 a = reinterpret_cast<const float4*>(src)[0], b = reinterpret_cast<const float4*>(src)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ----------------------------------------------------------------------------------------
// chunk_g2_prep_tc: per (chunk, value head) item, 256 threads
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t P_Q = 0;         // q bf16, then q~ fp16 (record layout)
constexpr uint32_t P_K = 16384;     // k bf16, then K~ fp16
constexpr uint32_t P_V = 32768;     // v bf16, then w . v fp16 (MN-major A operand of U~^T)
constexpr uint32_t P_G = 49152;     // g bf16, then b . e^G . k^ fp16 (A operand of W^T)
constexpr uint32_t P_B = 65536;     // b bf16, then -W staging
constexpr uint32_t P_W = 81920;     // w bf16, then U~^T staging
constexpr uint32_t P_GF = 98304;    // G (log2 units) fp32 [64][128]
constexpr int kLdXY = 136;          // padded row of the tf32 operands (conflict-free fragments)
constexpr uint32_t P_X = 131072;    // row operands of one row block: A [16][136], P [16][136]
constexpr uint32_t P_Y = 148480;    // column operand [<= 64][136]; then T_w | T_u (fp16)
constexpr uint32_t P_A = 183296;    // A fp32 [64][64], swizzled
constexpr uint32_t P_T = 199680;    // T fp32
constexpr uint32_t P_RS = 216064;   // transposed diagonal blocks, then E_32
constexpr uint32_t P_SMALL = 220160;
constexpr uint32_t P_SMEM = P_SMALL + 2048 + 1024;

struct PrepSmall {
    float inv_q[C], inv_k[C];
    float dec[D];         // e^{G_C} per channel
    float ones[C];        // column scales of the solve's T tiles (1: T itself)
    float half_tot[D];    // the cumulative log decay over the first 32 tokens, per channel
    uint64_t mbar[3];     // q, k, b, w tiles landed; W^T and U~^T done; v, g tiles landed
    uint32_t tmem_base;
    int range_bad;
};
static_assert(sizeof(PrepSmall) <= 2048, "prep small block");

// One tf32 warp-MMA product of a 16-row block: acc (16 x 8, n-tile) = X (16 x 128) Y^T
// (8 x 128).  X and Y hold tf32 bit patterns in rows padded to kLdXY words, so a fragment's
// eight rows fall in distinct banks and every load is a fixed offset from the lane's base.
// Each thread's two k slots of a step are two adjacent columns (any pairing the A and B
// fragments share gives the same sum); even and odd steps accumulate separately.
__device__ __forceinline__ void rowblock_ntile(float (&acc)[4], const uint32_t* X,
                                               const uint32_t* Y, int n0, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t* x0p = X + gq * kLdXY + 2 * tq;
    const uint32_t* x1p = x0p + 8 * kLdXY;
    const uint32_t* yp = Y + (n0 + gq) * kLdXY + 2 * tq;
    float acc2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = acc2[e] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < D; k0 += 8) {
        const uint2 x0 = *reinterpret_cast<const uint2*>(x0p + k0);
        const uint2 x1 = *reinterpret_cast<const uint2*>(x1p + k0);
        const uint2 y = *reinterpret_cast<const uint2*>(yp + k0);
        const uint32_t a[4] = {x0.x, x1.x, x0.y, x1.y};
        const uint32_t bb[2] = {y.x, y.y};
        if ((k0 >> 3) & 1) mma_tf32_16x8x8(acc2, a, bb);
        else mma_tf32_16x8x8(acc, a, bb);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += acc2[e];
}

__global__ void __launch_bounds__(kPrepThreads, 1)
chunk_g2_prep_tc(G2Params p, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_w) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    PrepSmall& SS = *reinterpret_cast<PrepSmall*>(sm + P_SMALL);
    const int pt = threadIdx.x, pw = pt >> 5, lane = pt & 31;
    griddep_launch_dependents();
    if (p.hdr->err != GDR_OK) { griddep_wait(); return; }
    const long long n_items = (long long)p.hdr->n_chunks * p.Hv;
    if ((long long)blockIdx.x >= n_items) { griddep_wait(); return; }

    if (pw == 0) {
        tmem_alloc(&SS.tmem_base, 128);
        tmem_relinquish();
    }
    if (pt == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&SS.mbar[i], 1);
        mbar_init_fence();
        SS.range_bad = 0;
    }
    if (pt < C) SS.ones[pt] = 1.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = SS.tmem_base;
    float* GF = reinterpret_cast<float*>(sm + P_GF);
    uint32_t* Xa = reinterpret_cast<uint32_t*>(sm + P_X);
    uint32_t* Xp = Xa + 16 * kLdXY;
    uint32_t* Yc = reinterpret_cast<uint32_t*>(sm + P_Y);
    float* As = reinterpret_cast<float*>(sm + P_A);
    float* Ts = reinterpret_cast<float*>(sm + P_T);
    float* RS = reinterpret_cast<float*>(sm + P_RS);
    bool fail = false;

    // An item's tiles are loaded while the previous item finishes: q, k, b, w once its q~
    // and K~ are out, v and g once its W and U~ products have read them.
    struct ItemPos { int h, hk, last; long long t0; };
    auto decode = [&](long long item) -> ItemPos {
        ItemPos ip;
        const int cg = (int)(item / p.Hv);
        ip.h = (int)(item - (long long)cg * p.Hv);
        ip.hk = ip.h / (p.Hv / p.Hk);
        const int s = p.chunk_seq[cg];
        const int c = cg - p.chunk_off[s];
        ip.t0 = (long long)p.cu[s] + (long long)c * C;
        ip.last = (int)min((long long)C, (long long)p.cu[s + 1] - ip.t0) - 1;
        return ip;
    };
    auto load_qkbw = [&](const ItemPos& ip) {  // thread 0
        uint64_t* bar = &SS.mbar[0];
        mbar_expect_tx(bar, 8 * 8192);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            tma_load_3d(sbase + P_Q + hh * 8192, &tm_q, hh * 64, ip.hk, (int)ip.t0, bar);
            tma_load_3d(sbase + P_K + hh * 8192, &tm_k, hh * 64, ip.hk, (int)ip.t0, bar);
            tma_load_3d(sbase + P_B + hh * 8192, &tm_b, hh * 64, ip.h, (int)ip.t0, bar);
            tma_load_3d(sbase + P_W + hh * 8192, &tm_w, hh * 64, ip.h, (int)ip.t0, bar);
        }
    };
    auto load_vg = [&](const ItemPos& ip) {  // thread 0
        uint64_t* bar = &SS.mbar[2];
        mbar_expect_tx(bar, 4 * 8192);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            tma_load_3d(sbase + P_V + hh * 8192, &tm_v, hh * 64, ip.h, (int)ip.t0, bar);
            tma_load_3d(sbase + P_G + hh * 8192, &tm_g, hh * 64, ip.h, (int)ip.t0, bar);
        }
    };
    ItemPos cur = decode(blockIdx.x);
    if (pt == 0) {
        load_qkbw(cur);
        load_vg(cur);
    }
    int pend = pt == 0 ? 3 : 0;  // tile groups in flight that nobody has waited for (bits 0, 1)

    int it = 0;
    for (long long item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
        const int h = cur.h;
        const int last = cur.last;
        const long long nitem = item + gridDim.x;
        const bool has_next = nitem < n_items;
        ItemPos nx = cur;
        if (has_next) nx = decode(nitem);  // its loads resolve while this item runs

        // L: this item's six tiles (tokens t0 .. t0 + 63; rows past the chunk are masked)
        bool landed = mbar_wait_bounded(&SS.mbar[0], (uint32_t)(it & 1), kWaitNs);
        landed = mbar_wait_bounded(&SS.mbar[2], (uint32_t)(it & 1), kWaitNs) && landed;
        if (landed) pend = 0;
        if (__syncthreads_or(landed ? 0 : 1)) { fail = true; break; }

        // N: per-channel cumulative log decay (log2 units): thread (channel d, half hh) scans
        //    its 32 tokens, the second half then adds the first half's total
        {
            const int d = pt & 127, hh = pt >> 7;
            float gv[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int t = 32 * hh + u;
                gv[u] = t <= last ? bf(sm + P_G, tile16(t, d, 8192)) * kLog2e : 0.f;
            }
#pragma unroll
            for (int u = 1; u < 32; ++u) gv[u] += gv[u - 1];
            if (hh == 0) SS.half_tot[d] = gv[31];
            __syncthreads();
            const float add = hh ? SS.half_tot[d] : 0.f;
#pragma unroll
            for (int u = 0; u < 32; ++u) GF[(32 * hh + u) * D + d] = gv[u] + add;
        }
        // the q and k row norms: thread (row r of [q; k], half hf2) sums 64 squares, the two
        // halves of a row in lanes l and l ^ 8
        {
            const int r2 = ((pt >> 4) << 3) | (pt & 7), hf2 = (pt >> 3) & 1;  // row 0..127
            const int t = r2 & 63;
            const uint8_t* tile = sm + (r2 < C ? P_Q : P_K) + hf2 * 8192;
            float ss = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                const uint4 u = *reinterpret_cast<const uint4*>(tile + sw128(t, c8));
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16x2(wv[e]);
                    ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
                }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 8);
            const float inv = t > last ? 0.f : (p.qk_l2norm ? rsqrtf(fmaxf(ss, kNormEps * kNormEps)) : 1.f);
            if (hf2 == 0) {
                if (r2 < C) SS.inv_q[t] = inv; else SS.inv_k[t] = inv;
            }
        }
        __syncthreads();
        if (pt < D) {
            const int d = pt;
            SS.dec[d] = ex2(GF[last * D + d]);
            // the exponents of the pair-sum factors this channel will use: row factors
            // G_t - R_I over block I, column factors R_I - G_s over s <= 16 I + 15
            float worst = 0.f, lo = 0.f;   // lo: min of G_{-1} = 0, G_0, ..., G_{16 I + 15}
#pragma unroll
            for (int I = 0; I < 4; ++I) {
                const float R = GF[(16 * I + 7) * D + d];
#pragma unroll
                for (int t = 16 * I; t < 16 * I + 16; ++t) {
                    const float Gt = GF[t * D + d];
                    worst = fmaxf(worst, Gt - R);
                    lo = fminf(lo, Gt);
                }
                worst = fmaxf(worst, R - lo);
            }
            if (!(worst <= 100.f)) SS.range_bad = 1;
        }

        // O: the A operands of W^T and U~^T over the consumed g and the v tile:
        //    b . e^G . k^ (fp16) and w . v (fp16); eight elements (16 bytes) per step
        for (int e = pt; e < 2 * 1024; e += kPrepThreads) {
            const int which = e >> 10, idx = e & 1023;
            const int t = (idx >> 4) & 63, c16 = idx & 15;   // row, 8-column group
            const uint32_t off = (c16 >> 3) * 8192 + sw128(t, c16 & 7);
            uint32_t outw[4];
            if (which == 0) {
                const uint4 bk = *reinterpret_cast<const uint4*>(sm + P_K + off);
                const uint4 bb = *reinterpret_cast<const uint4*>(sm + P_B + off);
                const float ik = SS.inv_k[t];
                const uint32_t kw[4] = {bk.x, bk.y, bk.z, bk.w}, gw[4] = {bb.x, bb.y, bb.z, bb.w};
                float Gv[8];
                load_row8(Gv, GF + t * D + c16 * 8);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 kk = unpack_bf16x2(kw[u]), gb = unpack_bf16x2(gw[u]);
                    outw[u] = h2(gb.x * kk.x * ik * ex2(Gv[2 * u]), gb.y * kk.y * ik * ex2(Gv[2 * u + 1]));
                }
                *reinterpret_cast<uint4*>(sm + P_G + off) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
            } else {
                const uint4 bv = *reinterpret_cast<const uint4*>(sm + P_V + off);
                const uint4 bw = *reinterpret_cast<const uint4*>(sm + P_W + off);
                const uint32_t vw[4] = {bv.x, bv.y, bv.z, bv.w}, ww[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 vv = unpack_bf16x2(vw[u]), wg = unpack_bf16x2(ww[u]);
                    outw[u] = t <= last ? h2(wg.x * vv.x, wg.y * vv.y) : 0u;
                }
                *reinterpret_cast<uint4*>(sm + P_V + off) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
            }
        }
        // the P staging (over the consumed w tile): zero, so the blocks above the diagonal
        // and the rows past the chunk stay zero
        __syncthreads();
        for (int e = pt; e < 512; e += kPrepThreads)
            reinterpret_cast<uint4*>(sm + P_W)[e] = make_uint4(0, 0, 0, 0);

        // A, P by row blocks: row operands X (16 rows) and the column operand Y (rows
        // 0 .. 16 I + 15) scaled around R_I = G_{16 I + 7}, then tf32 warp MMAs
        for (int I = 0; I < 4; ++I) {
            const int ref = 16 * I + 7;
            const int nY = 16 * (I + 1);
            // eight channels per step: 16 bytes of the bf16 tiles, two float4 of G and R
            for (int e = pt; e < (32 + nY) * 16; e += kPrepThreads) {
                const int row = e >> 4, c16 = e & 15, d0 = c16 * 8;
                const uint32_t off = (c16 >> 3) * 8192 + sw128(row < 32 ? 16 * I + (row & 15) : row - 32, c16 & 7);
                float Rv[8], Gv[8], f[8];
                {
                    const float4* rp = reinterpret_cast<const float4*>(GF + ref * D + d0);
                    const float4 r0 = rp[0], r1 = rp[1];
                    Rv[0] = r0.x; Rv[1] = r0.y; Rv[2] = r0.z; Rv[3] = r0.w;
                    Rv[4] = r1.x; Rv[5] = r1.y; Rv[6] = r1.z; Rv[7] = r1.w;
                }
                uint32_t* ob;  // destination rows
                int orow;
                if (row < 16) {               // A rows: b_t k^_t e^{G_t - R}
                    const int t = 16 * I + row;
                    const float4* gp = reinterpret_cast<const float4*>(GF + t * D + d0);
                    const float4 g0 = gp[0], g1 = gp[1];
                    Gv[0] = g0.x; Gv[1] = g0.y; Gv[2] = g0.z; Gv[3] = g0.w;
                    Gv[4] = g1.x; Gv[5] = g1.y; Gv[6] = g1.z; Gv[7] = g1.w;
                    const uint4 kb = *reinterpret_cast<const uint4*>(sm + P_K + off);
                    const uint4 bb = *reinterpret_cast<const uint4*>(sm + P_B + off);
                    const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w}, bw[4] = {bb.x, bb.y, bb.z, bb.w};
                    const float ik = SS.inv_k[t];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 kk = unpack_bf16x2(kw[u]), gb = unpack_bf16x2(bw[u]);
                        f[2 * u] = gb.x * kk.x * ik * ex2(Gv[2 * u] - Rv[2 * u]);
                        f[2 * u + 1] = gb.y * kk.y * ik * ex2(Gv[2 * u + 1] - Rv[2 * u + 1]);
                    }
                    ob = Xa;
                    orow = row;
                } else if (row < 32) {        // P rows: q^_t e^{G'_t - R}
                    const int t = 16 * I + row - 16;
                    const int tg = p.read_pre ? t - 1 : t;
                    if (tg >= 0) {
                        const float4* gp = reinterpret_cast<const float4*>(GF + tg * D + d0);
                        const float4 g0 = gp[0], g1 = gp[1];
                        Gv[0] = g0.x; Gv[1] = g0.y; Gv[2] = g0.z; Gv[3] = g0.w;
                        Gv[4] = g1.x; Gv[5] = g1.y; Gv[6] = g1.z; Gv[7] = g1.w;
                    } else {
#pragma unroll
                        for (int u = 0; u < 8; ++u) Gv[u] = 0.f;
                    }
                    const uint4 qb = *reinterpret_cast<const uint4*>(sm + P_Q + off);
                    const uint32_t qw[4] = {qb.x, qb.y, qb.z, qb.w};
                    const float iq = SS.inv_q[t];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 qq = unpack_bf16x2(qw[u]);
                        f[2 * u] = qq.x * iq * ex2(Gv[2 * u] - Rv[2 * u]);
                        f[2 * u + 1] = qq.y * iq * ex2(Gv[2 * u + 1] - Rv[2 * u + 1]);
                    }
                    ob = Xp;
                    orow = row - 16;
                } else {                      // columns: k^_s e^{R - G_s}
                    const int sidx = row - 32;
                    const float4* gp = reinterpret_cast<const float4*>(GF + sidx * D + d0);
                    const float4 g0 = gp[0], g1 = gp[1];
                    Gv[0] = g0.x; Gv[1] = g0.y; Gv[2] = g0.z; Gv[3] = g0.w;
                    Gv[4] = g1.x; Gv[5] = g1.y; Gv[6] = g1.z; Gv[7] = g1.w;
                    const uint4 kb = *reinterpret_cast<const uint4*>(sm + P_K + off);
                    const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w};
                    const float ik = SS.inv_k[sidx];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 kk = unpack_bf16x2(kw[u]);
                        f[2 * u] = kk.x * ik * ex2(Rv[2 * u] - Gv[2 * u]);
                        f[2 * u + 1] = kk.y * ik * ex2(Rv[2 * u + 1] - Gv[2 * u + 1]);
                    }
                    ob = Yc;
                    orow = sidx;
                }
                uint32_t* op = ob + orow * kLdXY + d0;
                *reinterpret_cast<uint4*>(op) = make_uint4(to_tf32(f[0]), to_tf32(f[1]), to_tf32(f[2]), to_tf32(f[3]));
                *reinterpret_cast<uint4*>(op + 4) = make_uint4(to_tf32(f[4]), to_tf32(f[5]), to_tf32(f[6]), to_tf32(f[7]));
            }
            __syncthreads();
            const int ntA = 2 * (I + 1);
            for (int task = pw; task < 2 * ntA; task += kPrepThreads / 32) {
                const bool isA = task < ntA;
                const int n0 = 8 * (isA ? task : task - ntA);
                float acc[4];
                rowblock_ntile(acc, isA ? Xa : Xp, Yc, n0, lane);
                const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = 16 * I + gq + 8 * hh, s0 = n0 + 2 * tq;
                    const float a0 = acc[2 * hh], a1 = acc[2 * hh + 1];
                    if (isA) {
                        *reinterpret_cast<float2*>(f32sw(As, t, s0)) =
                            make_float2(s0 < t ? a0 : 0.f, s0 + 1 < t ? a1 : 0.f);
                    } else {
                        const bool on0 = p.read_pre ? s0 < t : s0 <= t;
                        const bool on1 = p.read_pre ? s0 + 1 < t : s0 + 1 <= t;
                        *reinterpret_cast<uint32_t*>(sm + P_W + sw128(t, s0 >> 3) + (s0 & 7) * 2) =
                            h2(on0 ? p.scale * a0 : 0.f, on1 ? p.scale * a1 : 0.f);
                    }
                }
            }
            __syncthreads();
        }
        // P to the record now: its staging area takes U~^T later
        uint8_t* rec = p.rec + (size_t)item * kRecBytes;
        for (int e = pt; e < 512; e += kPrepThreads)
            reinterpret_cast<uint4*>(rec + REC_P)[e] = reinterpret_cast<const uint4*>(sm + P_W)[e];

        // Q: q~ over q, K~ over k (fp16, record layout), rows past the chunk zero
        for (int e = pt; e < 2 * 1024; e += kPrepThreads) {
            const int which = e >> 10, idx = e & 1023;
            const int t = (idx >> 4) & 63, c16 = idx & 15;
            const uint32_t off = (c16 >> 3) * 8192 + sw128(t, c16 & 7);
            uint8_t* tile = sm + (which == 0 ? P_Q : P_K);
            const uint4 raw = *reinterpret_cast<const uint4*>(tile + off);
            const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t outw[4];
            float ev[8];  // exponents (log2)
            if (which == 0) {
                const int tg = p.read_pre ? t - 1 : t;
                if (tg >= 0) {
                    load_row8(ev, GF + tg * D + c16 * 8);
                } else {
#pragma unroll
                    for (int u = 0; u < 8; ++u) ev[u] = 0.f;
                }
            } else {
                float gl[8];
                load_row8(ev, GF + t * D + c16 * 8);
                load_row8(gl, GF + last * D + c16 * 8);
#pragma unroll
                for (int u = 0; u < 8; ++u) ev[u] = gl[u] - ev[u];
            }
            const float sc = which == 0 ? p.scale * SS.inv_q[t] : SS.inv_k[t];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 x = unpack_bf16x2(rw[u]);
                outw[u] = h2(x.x * sc * ex2(ev[2 * u]), x.y * sc * ex2(ev[2 * u + 1]));
            }
            *reinterpret_cast<uint4*>(rec + (which == 0 ? REC_Q : REC_K) + off) =
                make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
        // q, k, b, w are consumed: the next item's land there during the solve
        fence_proxy_async_smem();
        __syncthreads();

        // S: T = (I + A)^-1 (the blocked solve of the scalar kernel), T in fp16 over Y
        if (pw == 0 || pw == 5) {
            const int i = pw == 0 ? lane : 32 + lane, hf = pw == 0 ? 0 : 1;
            float vals[32];
#pragma unroll
            for (int u4 = 0; u4 < 8; ++u4) {
                const float4 x = *reinterpret_cast<const float4*>(f32sw(As, i, hf * 32 + 4 * u4));
                vals[4 * u4] = x.x; vals[4 * u4 + 1] = x.y; vals[4 * u4 + 2] = x.z; vals[4 * u4 + 3] = x.w;
            }
            wy_diag_stage0(vals, i, lane, hf, As, RS, Ts);
        }
        uint8_t* twu = sm + P_Y;
        // (the solve's first barrier also orders every read of the q, k, b, w tiles before
        // the next item's tensor loads into them, issued after it)
        wy_solve_offdiag(As, Ts, RS, twu, SS.ones, SS.ones, pt, kBarG2, kPrepThreads, [&](int phase) {
            if (phase == 1 && has_next && pt == 0) {
                load_qkbw(nx);
                pend |= 1;
            }
        });
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(kBarG2, kPrepThreads);  // block column 0 of T complete

        // M: W^T = (b e^G k^)^T T^T and U~^T = (w v)^T T^T (M = 128, N = 64, K = 64 tokens)
        if (pt == 0) {
            tc_fence_after();
            const uint32_t id = idesc_f32acc(128, 64, true, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bt = sdesc_sw128(sbase + P_Y + kk * 32, 16, 1024);
                mma_f32acc_ss(tmem, sdesc_sw128(sbase + P_G + kk * 2048, 8192, 1024), bt, id, kk > 0);
                mma_f32acc_ss(tmem + 64, sdesc_sw128(sbase + P_V + kk * 2048, 8192, 1024), bt, id,
                              kk > 0);
            }
            mma_commit(&SS.mbar[1]);
        }
        const bool mdone = mbar_wait_bounded(&SS.mbar[1], (uint32_t)(it & 1), kWaitNs);
        tc_fence_after();

        // E: -W^T rows (warps 0-3, lane = dk) to the [token][dk] staging over b; U~^T rows
        //    (warps 4-7, lane = dv) to the [dv][token] staging over w
        {
            const int j = pt & 127;
            const uint32_t tl = tmem + ((uint32_t)((pw & 3) * 32) << 16) + (pt < 128 ? 0u : 64u);
            uint32_t r2[2][32];
            tmem_ld32(tl, r2[0]);
            tmem_ld32(tl + 32, r2[1]);
            tmem_wait_ld();
            if (pt < 128) {
#pragma unroll
                for (int t = 0; t < C; ++t)
                    *reinterpret_cast<__half*>(rec + REC_W + tile16(t, j, 8192)) =
                        __float2half_rn(-u2f(r2[t >> 5][t & 31]));
            } else {
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = u2f(r2[c8 >> 2][(c8 & 3) * 8 + u]);
                    *reinterpret_cast<uint4*>(rec + REC_U + sw128(j, c8)) = h8(f);
                }
            }
        }
        tc_fence_before();
        if (__syncthreads_or(mdone ? 0 : 1)) { fail = true; break; }
        // the W and U~ products have read b e^G k^ and w v: the next item's v, g land there
        if (has_next && pt == 0) {
            load_vg(nx);
            pend |= 2;
        }
        // R: the per-channel decay of the chunk
        if (pt < 32) reinterpret_cast<float4*>(rec + REC_D)[pt] = reinterpret_cast<const float4*>(SS.dec)[pt];
        if (SS.range_bad && pt == 0) atomicCAS(&p.hdr->err, (int)GDR_OK, (int)GDR_ERR_RANGE);
        cur = nx;
    }

    if (fail && pt == 0) {
        atomicExch(&p.hdr->err, (int)GDR_ERR_TIMEOUT);
        // no tile may land after the CTA has left its shared memory (the groups in flight
        // belong to item `it`, or to `it + 1` when this item's were waited for)
        const uint32_t par = (uint32_t)(it & 1);
        if (pend & 1) mbar_wait_bounded(&SS.mbar[0], par, kWaitNs) || mbar_wait_bounded(&SS.mbar[0], par ^ 1u, kWaitNs);
        if (pend & 2) mbar_wait_bounded(&SS.mbar[2], par, kWaitNs) || mbar_wait_bounded(&SS.mbar[2], par ^ 1u, kWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (pw == 0) tmem_dealloc(tmem, 128);
    griddep_wait();
}

// ----------------------------------------------------------------------------------------
// chunk_g2_chain_tc: one CTA per (sequence, value head), in the plan's order.  Warps 0-3 run
// the state recursion (lane = dv row of the transposed state H^T in tensor memory), warp 4
// streams the sequence's item records into two buffers by chunk parity.
constexpr int kChainThreads = 160;
constexpr int kBarChain = 1;
constexpr uint32_t kRecStride = 74752;           // a record buffer, 1024-aligned
constexpr uint32_t Q_ST = 2 * kRecStride;        // output staging: two [64][64] bf16 halves
constexpr uint32_t Q_SMALL = Q_ST + 16384;
constexpr uint32_t Q_SMEM = Q_SMALL + 1024 + 1024;
constexpr uint32_t TM_V = 0, TM_O = 64, TM_H = 128, TM_HB = 256, TM_VP = 320, TM_ALLOC = 512;
enum { CB_FULL = 0, CB_FREE = 2, CB_M1 = 4, CB_M3 = 5, CB_COUNT = 6 };

struct ChainSmall {
    uint64_t mbar[CB_COUNT];
    uint32_t tmem_base;
    int gflag[2];
};

__global__ void __launch_bounds__(kChainThreads, 1)
chunk_g2_chain_tc(G2Params p, const __grid_constant__ CUtensorMap tm_o) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    ChainSmall& SS = *reinterpret_cast<ChainSmall*>(sm + Q_SMALL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_launch_dependents();
    // the prep grid has completed and its records are visible
    griddep_wait();
    if (p.hdr->err != GDR_OK) return;

    const int h = (int)(blockIdx.x % (unsigned)p.Hv);
    const int s = p.order[blockIdx.x / (unsigned)p.Hv];
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);
    const int nchunks = (L + C - 1) / C;
    const size_t sb = ((size_t)s * p.Hv + h) * D * D;
    if (nchunks == 0) {
        if (p.S_final)
            for (int e = tid; e < D * D; e += kChainThreads) p.S_final[sb + e] = p.S0 ? p.S0[sb + e] : 0.f;
        return;
    }
    const long long item0 = (long long)p.chunk_off[s] * p.Hv + h;

    if (warp == 0) {
        tmem_alloc(&SS.tmem_base, TM_ALLOC);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < CB_COUNT; ++i) mbar_init(&SS.mbar[i], 1);
        SS.gflag[0] = SS.gflag[1] = 0;
        mbar_init_fence();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = SS.tmem_base;
    bool fail = false;
    float omax = 0.f;

    if (warp == 4) {
        // ------------------------------------------------------------ record loads
        if (lane == 0) {
            int issued = -1;
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                if (c >= 2 && !mbar_wait_bounded(&SS.mbar[CB_FREE + b], (uint32_t)(((c >> 1) & 1) ^ 1), kWaitNs)) {
                    fail = true;
                    break;
                }
                mbar_expect_tx(&SS.mbar[CB_FULL + b], kRecBytes);
                bulk_load(sbase + b * kRecStride, p.rec + (size_t)(item0 + (long long)c * p.Hv) * kRecBytes,
                          kRecBytes, &SS.mbar[CB_FULL + b]);
                issued = c;
            }
            // no copy may land after the CTA has left its shared memory: wait for the last two
            for (int c = max(0, issued - 1); fail && c <= issued; ++c)
                mbar_wait_bounded(&SS.mbar[CB_FULL + (c & 1)], (uint32_t)((c >> 1) & 1), kWaitNs);
        }
    } else {
        // ------------------------------------------------------------ state recursion
        const int j = tid;  // dv row = TMEM lane
        const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);
        int wk = 0;
        auto agree = [&](bool ok) -> bool {
            volatile int* f = &SS.gflag[wk & 1];
            ++wk;
            if (!ok) *f = 1;
            named_bar(kBarChain, 128);
            return *f == 0;
        };
        auto wait_all = [&](int idx, uint32_t parity) -> bool {
            const bool ok = agree(mbar_wait_bounded(&SS.mbar[idx], parity, kWaitNs));
            tc_fence_after();
            return ok;
        };
        const bool check_o = !p.qk_l2norm || !(fabsf(p.scale) <= 1024.f);
        if (wait_all(CB_FULL, 0u)) {
            // initial state: fp16 copy, and the fp32 state pre-scaled by chunk 0's decay
            const float* dec = reinterpret_cast<const float*>(sm + REC_D);
#pragma unroll 1
            for (int d0 = 0; d0 < D; d0 += 32) {
                uint32_t r[32], hb[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float x0 = p.S0 ? p.S0[sb + (size_t)(d0 + e) * D + j] : 0.f;
                    const float x1 = p.S0 ? p.S0[sb + (size_t)(d0 + e + 1) * D + j] : 0.f;
                    r[e] = __float_as_uint(x0 * dec[d0 + e]);
                    r[e + 1] = __float_as_uint(x1 * dec[d0 + e + 1]);
                    hb[e >> 1] = h2(x0, x1);
                }
                tmem_st32(tlane + TM_H + d0, r);
                tmem_st16(tlane + TM_HB + d0 / 2, hb);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();
        } else {
            fail = true;
        }
        for (int c = 0; c < nchunks && !fail; ++c) {
            const int b = c & 1;
            const uint32_t rs = sbase + b * kRecStride;
            const uint8_t* rp = sm + b * kRecStride;
            const int Cc = min(C, L - c * C);
            const bool has_next = c + 1 < nchunks;

            // C1: V'^T = H^T (-W^T) into TM_V (committed on its own), O^T = H^T q~^T
            if (j == 0) {
                tc_fence_after();
                const uint32_t id = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f32acc_ts(tmem + TM_V, tmem + TM_HB + kk * 8,
                                  sdesc_sw128(rs + REC_W + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                  id, kk > 0);
                mma_commit(&SS.mbar[CB_M1]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f32acc_ts(tmem + TM_O, tmem + TM_HB + kk * 8,
                                  sdesc_sw128(rs + REC_Q + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                  id, kk > 0);
            }
            if (!wait_all(CB_M1, (uint32_t)(c & 1))) { fail = true; break; }

            // C2: V'^T + U~^T -> fp16 in TMEM (the A operand of the output and state products)
            {
                uint32_t rv[2][32];
                tmem_ld32(tlane + TM_V, rv[0]);
                tmem_ld32(tlane + TM_V + 32, rv[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        const uint4 u = *reinterpret_cast<const uint4*>(rp + REC_U + sw128(j, hh * 4 + c8));
                        const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = unpack_f16x2(uw[e]);
                            const int m = c8 * 8 + 2 * e;
                            pk[c8 * 4 + e] = h2(u2f(rv[hh][m]) + x.x, u2f(rv[hh][m + 1]) + x.y);
                        }
                    }
                    tmem_st16(tlane + TM_VP + hh * 16, pk);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();

            // C3: O^T += V'^T P^T;  H^T += V'^T K~ (N = 128, B MN-major)
            if (j == 0) {
                const uint32_t id3 = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f32acc_ts(tmem + TM_O, tmem + TM_VP + kk * 8,
                                  sdesc_sw128(rs + REC_P + kk * 32, 16, 1024), id3, 1);
                const uint32_t id4 = idesc_f32acc(128, 128, false, true, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f32acc_ts(tmem + TM_H, tmem + TM_VP + kk * 8,
                                  sdesc_sw128(rs + REC_K + kk * 2048, 8192, 1024), id4, 1);
                mma_commit(&SS.mbar[CB_M3]);
            }
            if (!wait_all(CB_M3, (uint32_t)(c & 1))) { fail = true; break; }
            if (j == 0) mbar_arrive(&SS.mbar[CB_FREE + b]);  // every read of record c is done

            // C4: O -> bf16 staging -> global (tensor stores for a full chunk, else 16-byte
            //     stores); the state -> fp16 copy, pre-scaled by the next chunk's decay
            {
                uint8_t* stage = sm + Q_ST;
                uint32_t ro[2][32];
                tmem_ld32(tlane + TM_O, ro[0]);
                tmem_ld32(tlane + TM_O + 32, ro[1]);
                tmem_wait_ld();
                uint8_t* stage_j = stage + (j >> 6) * 8192 + (j & 7) * 2;
                const int cj = (j & 63) >> 3;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int m = 0; m < 32; ++m)
                        *reinterpret_cast<__nv_bfloat16*>(stage_j + sw128(hh * 32 + m, cj)) =
                            __float2bfloat16_rn(u2f(ro[hh][m]));
                if (check_o) {
#pragma unroll
                    for (int m = 0; m < 64; ++m) omax = max_abs_nan(omax, u2f(ro[m >> 5][m & 31]));
                }
                fence_proxy_async_smem();
                named_bar(kBarChain, 128);
                if (p.tma_store && Cc == C) {
                    if (j == 0) {
                        const int z = (int)(t0 + (long long)c * C);
                        tma_store_3d(&tm_o, sbase + Q_ST, 0, h, z);
                        tma_store_3d(&tm_o, sbase + Q_ST + 8192, 64, h, z);
                        bulk_commit();
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int idx = m * 128 + j, row = idx >> 4, c16 = idx & 15;
                        if (row < Cc) {
                            const long long tok = t0 + (long long)c * C + row;
                            *reinterpret_cast<uint4*>(p.o + ((size_t)tok * p.Hv + h) * D + c16 * 8) =
                                *reinterpret_cast<const uint4*>(stage + (c16 >> 3) * 8192 + sw128(row, c16 & 7));
                        }
                    }
                }
                if (has_next) {
                    // the next record's decay (it is needed next anyway)
                    if (!wait_all(CB_FULL + (b ^ 1), (uint32_t)(((c + 1) >> 1) & 1))) { fail = true; break; }
                    const float* dec = reinterpret_cast<const float*>(sm + (b ^ 1) * kRecStride + REC_D);
#pragma unroll
                    for (int d0 = 0; d0 < D; d0 += 64) {
                        uint32_t r2[2][32];
                        tmem_ld32(tlane + TM_H + d0, r2[0]);
                        tmem_ld32(tlane + TM_H + d0 + 32, r2[1]);
                        tmem_wait_ld();
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t (&r)[32] = r2[hh];
                            const int dd = d0 + hh * 32;
                            uint32_t hb[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const float x0 = u2f(r[2 * e]), x1 = u2f(r[2 * e + 1]);
                                hb[e] = h2(x0, x1);
                                r[2 * e] = __float_as_uint(x0 * dec[dd + 2 * e]);
                                r[2 * e + 1] = __float_as_uint(x1 * dec[dd + 2 * e + 1]);
                            }
                            tmem_st16(tlane + TM_HB + dd / 2, hb);
                            tmem_st32(tlane + TM_H + dd, r);
                        }
                    }
                } else {
#pragma unroll 1
                    for (int d0 = 0; d0 < D; d0 += 32) {
                        uint32_t r[32];
                        tmem_ld32(tlane + TM_H + d0, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            omax = max_abs_nan(omax, u2f(r[e]));
                            if (p.S_final) p.S_final[sb + (size_t)(d0 + e) * D + j] = u2f(r[e]);
                        }
                    }
                }
                tmem_wait_st();
                if (j == 0) bulk_wait_read();  // the staging buffer is free for reuse
            }
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();
        }
    }

    if (tid == 0) bulk_wait_all();
    if (fail) atomicExch(&p.hdr->err, (int)GDR_ERR_TIMEOUT);
    tc_fence_before();
    if (__syncthreads_or(omax <= 3.4e38f ? 0 : 1) && tid == 0)
        atomicCAS(&p.hdr->err, (int)GDR_OK, (int)GDR_ERR_RANGE);
    if (warp == 0) tmem_dealloc(tmem, TM_ALLOC);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_g2() {
    static EncodeTiledFn fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
        looked = true;
    }
    return fn;
}

// [tokens][heads][128] bf16 as a 3-D tensor (128, heads, tokens); box 64 x 1 x 64, 128-byte
// swizzle: one [64][64] half of a tile
bool make_g2_map(CUtensorMap* m, const void* base, int heads, long long tokens) {
    EncodeTiledFn fn = encode_tiled_g2();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int g2_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return 148;
    return n;
}

}  // namespace

bool tc_g2_supported(const gdr_chunk_args& a) {
    return a.gdn2 && !a.gate_raw && a.io_dtype == GDR_BF16 && a.gate_dtype == GDR_BF16 &&
           a.dk == D && a.dv == D && a.chunk == C && !a.reverse && !a.o_accumulate;
}

size_t g2_record_bytes() { return kRecBytes; }

gdr_status launch_chunk_g2_tc(const gdr_chunk_args& a, const void* q, const void* k, const void* v,
                              const void* g, const void* b, const float* S0, void* o,
                              float* S_final, void* ws, const WsLayout& L, cudaStream_t st) {
    char* base = static_cast<char*>(ws);
    G2Params p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.g = static_cast<const __nv_bfloat16*>(g);
    p.b = static_cast<const __nv_bfloat16*>(b);
    p.w = static_cast<const __nv_bfloat16*>(a.gdn2_w);
    p.S0 = S0; p.S_final = S_final; p.o = static_cast<__nv_bfloat16*>(o);
    p.hdr = reinterpret_cast<WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.chunk_off = reinterpret_cast<const int32_t*>(base + L.chunk_off);
    p.chunk_seq = reinterpret_cast<const int32_t*>(base + L.chunk_seq);
    p.order = reinterpret_cast<const int32_t*>(base + L.order);
    p.rec = reinterpret_cast<uint8_t*>(base + L.rec);
    p.Hk = a.Hk; p.Hv = a.Hv; p.read_pre = a.read_mode == GDR_READ_PRE;
    p.qk_l2norm = a.qk_l2norm; p.scale = a.scale;
    const long long T_tot = (long long)a.B * a.T;
    if (T_tot == 0) {  // every sequence is empty: the state passes through
        p.tma_store = 0;
        CUtensorMap to;
        memset(&to, 0, sizeof(to));
        cudaFuncSetAttribute(chunk_g2_chain_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Q_SMEM);
        chunk_g2_chain_tc<<<(unsigned)a.n_seqs * (unsigned)a.Hv, kChainThreads, Q_SMEM, st>>>(p, to);
        return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
    }
    CUtensorMap tq, tk, tv, tg, tb, tw, to;
    if (!make_g2_map(&tq, q, a.Hk, T_tot) || !make_g2_map(&tk, k, a.Hk, T_tot) ||
        !make_g2_map(&tv, v, a.Hv, T_tot) || !make_g2_map(&tg, g, a.Hv, T_tot) ||
        !make_g2_map(&tb, b, a.Hv, T_tot) || !make_g2_map(&tw, a.gdn2_w, a.Hv, T_tot) ||
        !make_g2_map(&to, o, a.Hv, T_tot))
        return GDR_ERR_CUDA;
    p.tma_store = 1;
    if (cudaFuncSetAttribute(chunk_g2_prep_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)P_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(chunk_g2_chain_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Q_SMEM) != cudaSuccess)
        return GDR_ERR_CUDA;
    const long long items = L.max_chunks * a.Hv;
    const unsigned pgrid = (unsigned)std::min<long long>(items, (long long)g2_sm_count());
    chunk_g2_prep_tc<<<pgrid, kPrepThreads, P_SMEM, st>>>(p, tq, tk, tv, tg, tb, tw);
    if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    // the recursion starts as the prep grid's dependent and waits for it to complete
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.n_seqs * (unsigned)a.Hv);
    cfg.blockDim = dim3(kChainThreads);
    cfg.dynamicSmemBytes = Q_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, chunk_g2_chain_tc, p, to) != cudaSuccess) return GDR_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
