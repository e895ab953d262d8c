// chunk_tc.cu -- fused chunk-wise WY/UT forward on the 5th-generation tensor cores.
//
// One CTA per (sequence, value head) walks the sequence's 64-token chunks in order.  The
// fp32 state lives in tensor memory for the whole sequence; nothing but q, k, v, g, beta
// (and S0) is read from HBM and nothing but o (and S_final) is written.
//
// Per chunk, with the in-chunk log decay G_i = g_1 + ... + g_i (Prizma "seq/delta.py",
// chunked_delta: cumulative decay in log space; flashrt fused_layer.py `_wy_core`:
// kkt -> triangular solve -> recompute W/U -> chunk state -> output):
//
//   [K;Q] K^T                        one M=128 MMA gives K K^T and Q K^T
//   A_ij = beta_i (k_i.k_j) e^(G_i-G_j), j<i         (fp32, CUDA cores)
//   T = (I + A)^-1                                  (blocked: 16x16 diagonal inverses by
//                                                    substitution, off-diagonal blocks by
//                                                    tf32 warp MMAs)
//   W = T diag(beta e^G) K,  U~ = T diag(beta) V     (MMA)
//   V' = U~ - W H                                   (MMA, accumulating onto U~)
//   o = diag(scale e^G') Q H + P V',  P = scale (Q K^T)(.)decay mask   (MMA x2)
//   H <- e^(G_C) H + (diag(e^(G_C - G)) K)^T V'     (MMA into the TMEM state)
//
// Three warpgroups work on consecutive chunks at once.  The two "prep" warpgroups (warps
// 4-11, splitting each step by rows or column halves) load chunk c+1 and do everything that
// does not depend on the state: normalisation, [K;Q]K^T, the solve, W and U~.  The "chain"
// warpgroup (warps 0-3) runs the state recursion of chunk c: V', the output and the state
// update.  They hand chunks over
// through mbarriers; K/Q tiles are triple-buffered and every other per-chunk buffer is
// double-buffered by chunk parity.
//
// Orientation: every product is written transposed so that its M dimension is a head
// dimension (128): accumulators hold rows of W^T, U~^T, V'^T, O^T and H^T, one TMEM lane
// per dk or dv index, one column per token (or per dk for the state).  Every MMA is then
// M=128, N=64 or 128.  The state copy H^T and V'^T, the A operands of the chain's
// products, stay in tensor memory as packed fp16; the other operands are 16-bit tiles in
// shared memory in the 128-byte-swizzled canonical layouts (K-major or MN-major as each
// product needs).  Accumulation and the state are fp32.
//
// Operand precision: [K;Q] K^T is formed from the bf16 inputs as they arrive (exact
// products, fp32 sums) and the L2 norms are applied to its rows and columns in fp32.
// Every other operand (normalised k, Q~, V, T diag(beta), T diag(beta e^G), W, the state
// copy, V', P) is fp16, whose 11-bit significand keeps the chain of roundings well inside
// the bf16 parity bound at long sequence lengths where bf16 operands do not; V is
// converted to fp16 in shared memory, exactly for every bf16 value of the fp16 range.  A
// value beyond the fp16 range becomes infinite and makes an output or the final state
// non-finite; the chain checks both, and a non-finite one sets GDR_ERR_RANGE.  Decay
// factors are 2^(log2(e) (G_i - G_j)) by the hardware exp2 approximation (relative error
// ~2^-22).
//
// The state update uses V' with its rows scaled by e^(G_C - G_i) (a second fp16 copy in
// tensor memory) against the unscaled K, so K is never rewritten after normalisation.
//
// The state H is kept transposed in TMEM (lane = dv, column = dk).  After each chunk the
// chain reads it once, writes the fp16 copy the next chunk's MMAs consume, and scales it
// in place by the next chunk's total decay, so the next state update accumulates onto it.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "chunk_tc.cuh"
#include "common.cuh"

#include "tc_ptx.cuh"
#include "wy_solve.cuh"

namespace gdr {

namespace {

using namespace tc;

constexpr int C = 64;            // chunk length
constexpr int D = 128;           // dk = dv
constexpr int kThreads = 384;    // warpgroup 0: state chain; warpgroups 1-2: chunk preparation
constexpr int kPrep = 256;       // preparation threads
constexpr int kBarChain = 1, kBarPrep = 2;  // named barriers of the chain and of the preparation
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory map (bytes from a 1024-byte-aligned base)
constexpr uint32_t OFF_KQ = 0;         // 3 x 32 KB; per dk half (16 KB): K rows 0-63, Q rows 64-127
constexpr uint32_t KQ_STRIDE = 32768;
constexpr uint32_t OFF_V = 98304;      // 2 x 16 KB; per dv half (8 KB): V rows 0-63 (bf16)
constexpr uint32_t V_STRIDE = 16384;
constexpr uint32_t OFF_TWU = 131072;   // T fp32 [64][64] (the solve)
constexpr uint32_t OFF_AS = 147456;    // A fp32 [64][64]
constexpr uint32_t OFF_RS = 163840;    // the four diagonal 16x16 blocks of A, transposed (fp32)
constexpr uint32_t OFF_P = 167936;     // 2 x 8 KB: P fp16 [i][j]
constexpr uint32_t OFF_WN = 184320;    // 2 x 16 KB: T diag(beta e^G) fp16 | T diag(beta) fp16
                                       // during the solve, then -W^T fp16 [dk][tok]; output
                                       // staging
constexpr uint32_t OFF_SMALL = 217088;
constexpr uint32_t SMEM_BYTES = OFF_SMALL + 5120 + 1024;

// TMEM columns (32-bit each)
constexpr uint32_t TM_D0 = 0;     // [K;Q] K^T, then W^T (64)
constexpr uint32_t TM_DU = 64;    // 2 x 64: U~^T, then V'^T, by chunk parity
constexpr uint32_t TM_DO = 192;   // O^T (64)
constexpr uint32_t TM_HM = 256;   // state H^T, fp32 (128)
constexpr uint32_t TM_HB = 384;   // state H^T, fp16 packed (64): A operand
constexpr uint32_t TM_VP = 448;   // V'^T, fp16 packed (32): A operand of the output product
constexpr uint32_t TM_VS = 480;   // V'^T scaled by e^(G_C - G_i), fp16 packed (32): state update
constexpr uint32_t TM_COLS = 512;

// mbarriers
enum {
    MB_M0 = 0, MB_M1 = 2,  // (index 1 unused)
    MB_M3 = 3,    // x2: state update of a chunk done (by chunk parity)
    MB_PREP = 5,  // x2: chunk prepared (by chunk parity)
    MB_LD = 7,    // x3: K, Q, V tiles of a chunk landed (by K/Q buffer)
    MB_CD = 10,   // x2: chain finished with a chunk's buffers (by chunk parity)
    MB_MU = 12,   // W and U~ products of a chunk done (awaited by the chain)
    MB_D0F = 13,  // the chain has read W^T out of D0 (the next [K;Q]K^T may overwrite it)
    MB_COUNT = 14
};

struct Small {
    float b[2][C];           // beta by chunk parity (prep)
    float G[2][C];           // log2(e) x in-chunk cumulative log decay, by chunk parity (prep)
    float bg[C];             // beta_i e^(G_i)
    float Kd[2][C];          // e^(G_last - G_i), 0 beyond the chunk, by chunk parity (for the chain)
    float Er[C];             // 2^(G_i - G_ref): row factor of the decay (K rows)
    float Eq[C];             // 2^(G'_i - G_ref): row factor for the read (G' = G_i or G_{i-1})
    float ck[C];             // column factor of [K;Q]K^T: 1/||k_j|| (x 2^(G_ref - G_j) when split)
    float inv[128];          // 1 / ||row|| of [K;Q] (1 without normalisation)
    float gsum_part[2];      // chain: partial sums of the next chunk's g
    float gam_adj[2];        // adjoint: e^(G_last) of the chunk, by step parity
    uint64_t mbar[MB_COUNT];
    uint32_t tmem_base;
    int gflag[2][2];         // a bounded wait gave up: [chain, preparation][alternate waits]
    int split_ok[2];         // the chunk's decay factors factor into row x column exactly
    uint32_t pair_cnt;       // bidirectional pair: chunks the partner has left for this CTA
};
static_assert(sizeof(Small) <= 5120, "small shared block");

struct TcParams {
    const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
    const void* g; const void* beta; const float* S0;
    __nv_bfloat16* o; float* S_final;
    WsHeader* hdr; const int32_t* cu;
    const int32_t* order;  // sequences in visiting order (longest first for varlen calls)
    int Hk, Hv, read_pre, qk_l2norm, reverse, o_acc, use_tma;
    int tma_store;  // full output chunks leave through the output tensor map
    gdr_dtype gt;
    float scale;
    // bidirectional pairs: the reverse scan's gates, the chunk map's first chunk of every
    // sequence, and the fp32 output a pair's first scan of a chunk leaves for the second
    // ([chunk][head][64 rows][head size], rows in forward order)
    const void* g_rev; const void* beta_rev;
    const int32_t* chunk_off;
    float* part;
    // the saving instantiation (kSave) leaves what the backward reads, fp32: W and U~ by
    // token ([token][head][d]), the in-chunk cumulative log decay G ([token][head]), the state
    // at every chunk start ([chunk][head][dk][dv]) and V' ([token][head][dv]); no output
    float *sv_G, *sv_H, *sv_V;
};

// The fused gating prologue's per-head arrays, a kernel argument of its own that only the
// gated instantiation reads (the plain kernel's parameter block stays as it is).
struct GateParams {
    const float* A; const float* dt_bias;
    float beta_scale;
};

// Raw bits of a gate element (bf16 zero-extended, or fp32): loading without converting lets
// the load stay in flight until the value is consumed much later.
__device__ __forceinline__ uint32_t load_gate_bits(const void* p, size_t i, gdr_dtype dt) {
    return dt == GDR_BF16 ? (uint32_t)static_cast<const unsigned short*>(p)[i]
                          : static_cast<const uint32_t*>(p)[i];
}
__device__ __forceinline__ float gate_bits_to_float(uint32_t b, gdr_dtype dt) {
    return __uint_as_float(dt == GDR_BF16 ? b << 16 : b);
}

// kRaw: the fused gating prologue is compiled into this instantiation only, so the plain-gate
// kernel carries none of its code or register pressure.
// kDh: the head size dk = dv in memory, 128 or 64.  A 64-wide head runs in the same 128-wide
// tiles with feature columns 64-127 zero (never loaded): the normalisation is unchanged and
// the state's extra rows and columns receive only zero updates, so they stay zero.
// kSave: the forward of the backward pass (see TcParams); plain gates, head size 128, single
// scans only.
// kAdj: the backward's reverse state pass on the same preparation.  The chunks are visited
// last to first; the value tiles carry dO, the initial state is dS_final and the final one
// dS0; the chain keeps dH^T in tensor memory and leaves dH+ at every chunk and dV' (sv_H,
// sv_V).  Plain gates, head size 128, single scans.
template <bool kRaw, int kDh, bool kPair, bool kSave, bool kAdj>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fused_tc(TcParams p, const __grid_constant__ CUtensorMap tm_q,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_o, const GateParams gp) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, as a byte offset from the shared array so that every access
    // through it stays a shared-memory access (an integer round trip would make them generic)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    Small& SS = *reinterpret_cast<Small*>(sm + OFF_SMALL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = tid >> 7;     // 0: chain, 1-2: prep
    const int lt = tid & 127;    // index within the warpgroup = TMEM lane
    // a grid launched after this one as its dependent (the reverse direction of a
    // bidirectional call) may start on the SMs this grid leaves free; every CTA waits for the
    // grid it depends on before it exits, so a later ordinary launch sees both grids' results
    griddep_launch_dependents();
    // a bidirectional pair stops only on an error of the plan, which both of its CTAs see
    // alike (an error another CTA records while this grid runs must not split a pair)
    if (kPair ? p.hdr->err == GDR_ERR_DEVICE_CHECK : p.hdr->err != GDR_OK) {
        griddep_wait();
        return;
    }

    // one CTA per (sequence, value head), heads fastest, sequences in the plan's order; a
    // bidirectional pair is two CTAs of one cluster, the forward scan (rank 0) and the reverse
    // scan (rank 1) of one (sequence, head)
    const unsigned unit = kPair ? blockIdx.x >> 1 : blockIdx.x;
    const bool rev = kPair ? cluster_ctarank() == 1 : p.reverse != 0;
    const void* const gsrc = kPair && rev ? p.g_rev : p.g;
    const void* const bsrc = kPair && rev ? p.beta_rev : p.beta;
    const bool use_tma = p.use_tma && !rev;  // reversed scans gather rows with cp.async
    const int h = (int)(unit % (unsigned)p.Hv);
    const int s = p.order[unit / (unsigned)p.Hv];
    // the gates as the recurrence uses them (fused gating prologue when kRaw)
    auto XG = [&](float a) -> float {
        if constexpr (kRaw) return gate_g_from_raw(gp.A[h], gp.dt_bias[h], a);
        else return a;
    };
    auto XB = [&](float b) -> float {
        if constexpr (kRaw) return gate_beta_from_raw(gp.beta_scale, b);
        else return b;
    };
    const int hk = h / (p.Hv / p.Hk);
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int Lseq = (int)(t1 - t0);
    // The reverse scan of a pair aligns its chunks with the forward scan's, so both cover the
    // same 64 tokens per chunk: its chunk 0 holds the sequence's last Lseq mod 64 tokens in
    // rows rofs..63, and rows below rofs are empty (zero keys, queries, values and gates,
    // which leave the recurrence unchanged).  The chunked form is exact for any chunking.
    const int rofs = kPair && rev ? (C - Lseq % C) % C : 0;
    const int L = Lseq + rofs;  // positions of the (row-offset) scan
    const int nchunks = (L + C - 1) / C;
    auto row_lo = [&](int c) -> int { return c == 0 ? rofs : 0; };  // first live row of chunk c
    // the chunk taken at step `step` (the adjoint pass walks the chunks backwards)
    auto chunk_of = [&](int step) -> int { return kAdj ? nchunks - 1 - step : step; };
    static_assert(kDh == 64 || kDh == D, "head size");
    const size_t sb = ((size_t)s * p.Hv + h) * kDh * kDh;
    // physical token of logical position 0, and the step between consecutive positions
    const long long tstep = rev ? -1 : 1;
    const long long tokA = (rev ? t1 - 1 : t0) - tstep * rofs;

    if (nchunks == 0) {  // empty sequence: the state passes through
        if (p.S_final)
            for (int e = tid; e < kDh * kDh; e += kThreads)
                p.S_final[sb + e] = p.S0 ? p.S0[sb + e] : 0.f;
        griddep_wait();
        return;
    }

    if (warp == 0) {
        tmem_alloc(&SS.tmem_base, TM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < MB_COUNT; ++i)
            mbar_init(&SS.mbar[i], (i == MB_PREP || i == MB_PREP + 1)              ? kPrep
                                   : (i == MB_CD || i == MB_CD + 1 || i == MB_D0F) ? 128
                                                                                   : 1);
        SS.gflag[0][0] = SS.gflag[0][1] = SS.gflag[1][0] = SS.gflag[1][1] = 0;
        SS.pair_cnt = 0;
        mbar_init_fence();
    }
    if constexpr (kDh < D) {  // feature columns 64-127 of every K/Q and V tile stay zero
        for (int e = tid; e < 3 * 1024 + 2 * 512; e += kThreads) {
            const uint32_t off = e < 3072
                ? OFF_KQ + (e >> 10) * KQ_STRIDE + 16384 + (e & 1023) * 16
                : OFF_V + ((e - 3072) >> 9) * V_STRIDE + 8192 + ((e - 3072) & 511) * 16;
            *reinterpret_cast<uint4*>(sm + off) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    // a pair's counters start at zero before either CTA may advance its partner's
    if constexpr (kPair) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = SS.tmem_base;
    const uint32_t tlane = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's lanes
    float omax = 0.f;     // chain: running max |output| and |final state| (NaN sticks)
    bool fail = false;    // a bounded wait gave up

    auto gate_at = [&](const void* arr, int pos) -> float {
        return load_elem(arr, (size_t)(tokA + tstep * pos) * p.Hv + h, p.gt);
    };
    auto gate_bits_at = [&](const void* arr, int pos) -> uint32_t {
        return load_gate_bits(arr, (size_t)(tokA + tstep * pos) * p.Hv + h, p.gt);
    };
    // the warpgroup agrees that every thread's wait succeeded: a thread whose wait gave up
    // raises its group's flag before a plain barrier and every thread reads it after.  Flags
    // alternate between consecutive waits, so a thread that has passed this barrier and fails
    // its next wait never raises the flag a slower thread is still about to read; flags only
    // ever go up, and a raised one ends the group.
    int wk = 0;
    auto group_agree = [&](bool ok, int bar_id) -> bool {
        volatile int* f = &SS.gflag[bar_id == kBarPrep ? 1 : 0][wk & 1];
        ++wk;
        if (!ok) *f = 1;
        named_bar(bar_id, bar_id == kBarPrep ? kPrep : 128);
        return *f == 0;
    };
    // wait for a phase of an mbarrier; the whole warpgroup agrees on the outcome
    auto wg_wait = [&](int idx, uint32_t parity, int bar_id) -> bool {
        const bool ok = mbar_wait_bounded(&SS.mbar[idx], parity, kWaitLimitNs);
        const bool all = group_agree(ok, bar_id);
        tc_fence_after();
        return all;
    };

    if (wg >= 1) {
        // ============================ preparation warpgroups ===========================
        const int pt = tid - 128;      // 0..255
        const int r = pt & 127;        // TMEM lane / row of [K;Q] / dk or dv row
        const int hf = pt >> 7;        // which half of the columns this thread takes
        const int pw = pt >> 5;        // preparation warp 0..7
        // P2's split of the rows: the two halves of a row sit in lanes l and l ^ 8 of one warp
        // (eight rows per quarter warp, so the swizzled 16-byte accesses do not conflict)
        const int r2 = ((pt >> 4) << 3) | (pt & 7), hf2 = (pt >> 3) & 1;
        // cp.async plan: this thread copies 16-byte column chunk `cd` of rows r0 + 16 m
        const int cd = pt & 15, r0 = pt >> 4;
        const bool cd_in = cd < kDh / 8;  // column chunks past a 64-wide head are zero-filled
        const __nv_bfloat16* kbase = p.k + (size_t)hk * kDh + (cd_in ? cd : 0) * 8;
        const __nv_bfloat16* qbase = p.q + (size_t)hk * kDh + (cd_in ? cd : 0) * 8;
        const __nv_bfloat16* vbase = p.v + (size_t)h * kDh + (cd_in ? cd : 0) * 8;
        const long long kq_tok = (long long)p.Hk * kDh, v_tok = (long long)p.Hv * kDh;
        auto load_chunk = [&](int step) {  // buffers by step, positions by chunk
            const int c = chunk_of(step);
            if (use_tma) {  // forward scans: six 8 KB tensor tiles, issued by one thread (pt 128)
                uint64_t* bar = &SS.mbar[MB_LD + step % 3];
                const uint32_t kq = sbase + OFF_KQ + (step % 3) * KQ_STRIDE;
                const uint32_t vv = sbase + OFF_V + (step & 1) * V_STRIDE;
                const int z = (int)(t0 + (long long)c * C);
                mbar_expect_tx(bar, 3 * (kDh / 64) * 8192);
#pragma unroll
                for (int half = 0; half < kDh / 64; ++half) {
                    tma_load_3d(kq + half * 16384, &tm_k, half * 64, hk, z, bar);
                    tma_load_3d(kq + half * 16384 + 8192, &tm_q, half * 64, hk, z, bar);
                    tma_load_3d(vv + half * 8192, &tm_v, half * 64, h, z, bar);
                }
                return;
            }
            const int Cc = min(C, L - c * C);
            const uint32_t kq = sbase + OFF_KQ + (step % 3) * KQ_STRIDE + (cd >> 3) * 16384;
            const uint32_t vv = sbase + OFF_V + (step & 1) * V_STRIDE + (cd >> 3) * 8192;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = r0 + 16 * m;
                const bool valid = i >= row_lo(c) && i < Cc && cd_in;
                const long long tok = valid ? tokA + tstep * (c * C + i) : t0;
                const uint32_t off = sw128(i, cd & 7);
                cp_async16(kq + off, kbase + tok * kq_tok, valid);
                cp_async16(kq + 8192 + off, qbase + tok * kq_tok, valid);
                cp_async16(vv + off, vbase + tok * v_tok, valid);
            }
        };
        if (use_tma && pt == 128) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
        }
        if (!use_tma || pt == 128) load_chunk(0);
        // the chunk whose tensor loads this thread issued and nobody has waited for yet (-1:
        // none); on an early exit it waits for them, so no copy lands in released memory
        int ld_pending = use_tma && pt == 128 ? 0 : -1;
        if (!use_tma) cp_async_commit();
        // in-chunk cumulative log decay (log2 units) of one chunk from its gates, two per lane
        // (positions 2 lane, 2 lane + 1; 0 past the chunk), into G[par], and whether every
        // decay factor 2^(G_i - G_j) splits into 2^(G_i - G_ref) 2^(G_ref - G_j) inside the
        // normal fp32 range (true unless the log2 decay strays more than 110 from G_ref = G_31)
        auto chunk_cumsum = [&](float a0, float a1, int par) {
            a0 *= kLog2e;
            a1 *= kLog2e;
            const float pair = a0 + a1;
            float incl = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float excl = incl - pair;
            const float G0 = excl + a0, G1 = excl + a0 + a1;
            SS.G[par][2 * lane] = G0;
            SS.G[par][2 * lane + 1] = G1;
            const float Gref = __shfl_sync(0xffffffffu, G1, 15);  // G_31
            float dev = fmaxf(fabsf(G0 - Gref), fabsf(G1 - Gref));
            dev = fmaxf(dev, fabsf(excl - Gref));                // G_{i-1} of the pre-read
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
            if (lane == 0) SS.split_ok[par] = dev <= 110.f;
        };
        {
            const int p0 = chunk_of(0) * C, Cc0 = min(C, L - p0);
            auto live0 = [&](int i) { return i >= row_lo(chunk_of(0)) && i < Cc0; };
            if (pt < C) SS.b[0][pt] = live0(pt) ? XB(gate_at(bsrc, p0 + pt)) : 0.f;
            if (pw == 1)
                chunk_cumsum(live0(2 * lane) ? XG(gate_at(gsrc, p0 + 2 * lane)) : 0.f,
                             live0(2 * lane + 1) ? XG(gate_at(gsrc, p0 + 2 * lane + 1)) : 0.f, 0);
        }
        // P5, issued as the solve completes T's block columns: K-step kk of W^T = K^T T_w^T
        // (into D0) and of U~^T = V^T T_u^T (into DU) reads block column kk of T_w and T_u
        // only, so columns 3 and 2 go after phase 1, column 1 after phase 2 and column 0 (with
        // the commits) after phase 3; the first K-step issued (kk = 3) starts each accumulator
        auto issue_w = [&](uint32_t KQa, int pb_, int kk) {
            mma_f32acc_ss(tmem + TM_D0, sdesc_sw128(KQa + kk * 2048, 16384, 1024),
                          sdesc_sw128(sbase + OFF_WN + pb_ * 16384 + kk * 32, 16, 1024),
                          idesc_f32acc(128, 64, true, false, false), kk < 3);
        };
        auto issue_u = [&](uint32_t VVa, int pb_, int kk) {
            mma_f32acc_ss(tmem + TM_DU + pb_ * 64, sdesc_sw128(VVa + kk * 2048, 8192, 1024),
                          sdesc_sw128(sbase + OFF_WN + pb_ * 16384 + 8192 + kk * 32, 16, 1024),
                          idesc_f32acc(128, 64, true, false, false), kk < 3);
        };
        // raw bits of the next chunk's gates: beta (one per thread), g (two per lane, warp 5)
        uint32_t b_nx = 0, g_nx0 = 0, g_nx1 = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int pb = c & 1;
            const uint32_t KQ = sbase + OFF_KQ + (c % 3) * KQ_STRIDE;
            uint8_t* KQp = sm + OFF_KQ + (c % 3) * KQ_STRIDE;
            const uint32_t VV = sbase + OFF_V + pb * V_STRIDE;
            const int cc = chunk_of(c);  // the chunk of this step
            const int Cc = min(C, L - cc * C);
            const bool has_next = c + 1 < nchunks;

            // P0: the buffers of chunk c-2 are released once the chain is done with them (each
            //     thread sees it on the mbarrier before its own copies into them); the one
            //     group barrier below, after this chunk's tiles have landed, also publishes this
            //     chunk's beta and cumulative decay (stored during the previous chunk's
            //     preparation, or before the loop)
            bool ok = true;
            if (c >= 2) ok = mbar_wait_bounded(&SS.mbar[MB_CD + pb], ((c >> 1) & 1) ^ 1, kWaitLimitNs);
            int Cn = 0;
            if (has_next) {
                // the loads of step c + 1 rewrite the value tile of step c - 1: its last reader
                // (the U~ product, or in the adjoint the chain's first products) must be done
                if (!use_tma && ok && c >= 1)
                    ok = mbar_wait_bounded(&SS.mbar[kAdj ? MB_M1 : MB_MU], (uint32_t)((c - 1) & 1), kWaitLimitNs);
                if (!use_tma && ok) load_chunk(c + 1);  // reversed scans: every thread's row copies
                // in-bounds positions for every thread, masked only where the values are used
                // (a select on a just-loaded value would wait for the load right here)
                const int pn = chunk_of(c + 1) * C;
                Cn = min(C, L - pn);
                b_nx = gate_bits_at(bsrc, pn + min(pt & 63, Cn - 1));
                if (pw == 1) {
                    g_nx0 = gate_bits_at(gsrc, pn + min(2 * lane, Cn - 1));
                    g_nx1 = gate_bits_at(gsrc, pn + min(2 * lane + 1, Cn - 1));
                }
            }
            if (!use_tma) cp_async_commit();
            // P1: D0 = [K;Q] K^T straight from the bf16 tiles (M=128, N=64, K=128), issued by
            //     warp 11 once the tiles have landed.  The L2 norms scale D0's rows and columns
            //     afterwards, so the product runs while the operands are normalised.
            auto issue_mma0 = [&]() {
                tc_fence_after();
                const uint32_t id = idesc_f32acc(128, 64, false, false, true);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_f32acc_ss(tmem + TM_D0, sdesc_sw128(KQ + off, 16, 1024),
                                  sdesc_sw128(KQ + off, 16, 1024), id, kk > 0);
                }
                mma_commit(&SS.mbar[MB_M0]);
            };
            bool landed = true;
            if (use_tma)
                landed = mbar_wait_bounded(&SS.mbar[MB_LD + c % 3], (uint32_t)((c / 3) & 1),
                                           kWaitLimitNs);
            else
                cp_async_wait<1>();
            if (!use_tma) fence_proxy_async_smem();  // row copies land through the generic proxy
            if (landed && ld_pending == c) ld_pending = -1;
            if (!group_agree(ok && landed, kBarPrep)) {
                fail = true;
                break;
            }
            tc_fence_after();
            // D0 held the previous chunk's W^T until the chain read it out
            if (pt == kPrep - 32 &&
                (c == 0 || mbar_wait_bounded(&SS.mbar[MB_D0F], (uint32_t)((c - 1) & 1), kWaitLimitNs)))
                issue_mma0();
            // P2: half row of [K; Q] -> sum of squares -> fp16 operand in registers: K rows
            //     L2-normalised, Q rows as Q~ = scale e^(G') q / ||q||; rows past the chunk
            //     (tensor tiles carry the following tokens there) become 0.  Stored over the
            //     bf16 tile once the product has read it.
            uint32_t hv[32];
            uint8_t* rowp = KQp + hf2 * 16384;  // this thread's half of row r2
            {
                uint4 vals[8];
                float2 ssq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8)
                    vals[c8] = *reinterpret_cast<const uint4*>(rowp + sw128(r2, c8));
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const uint32_t w[4] = {vals[c8].x, vals[c8].y, vals[c8].z, vals[c8].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = unpack_bf16x2(w[e]);
                        ssq[e & 1] = __ffma2_rn(x, x, ssq[e & 1]);
                    }
                }
                float tot = (ssq[0].x + ssq[0].y) + (ssq[1].x + ssq[1].y);
                tot += __shfl_xor_sync(0xffffffffu, tot, 8);  // the row's other half
                const float inv = p.qk_l2norm ? rsqrtf(fmaxf(tot, kNormEps * kNormEps)) : 1.f;
                if (hf2 == 0) SS.inv[r2] = inv;
                if (hf2 == 0 && r2 < C) {  // per-token factors; the column factor of D0 (K rows)
                                           // is 1/||k_j||, times 2^(G_ref - G_j) when split
                    const int t = r2;
                    const float Gref = SS.G[pb][31];
                    const float Gi = SS.G[pb][t];
                    const float Gr = p.read_pre ? (t > 0 ? SS.G[pb][t - 1] : 0.f) : Gi;
                    SS.Kd[pb][t] = t >= row_lo(cc) && t < Cc ? ex2(SS.G[pb][Cc - 1] - Gi) : 0.f;
                    if (kAdj && t == 0) SS.gam_adj[pb] = ex2(SS.G[pb][Cc - 1]);
                    SS.bg[t] = SS.b[pb][t] * ex2(Gi);
                    SS.Er[t] = ex2(Gi - Gref);
                    SS.Eq[t] = ex2(Gr - Gref);
                    SS.ck[t] = SS.split_ok[pb] ? ex2(Gref - Gi) * inv : inv;
                    if constexpr (kSave) {
                        if (t >= row_lo(cc) && t < Cc)
                            p.sv_G[(size_t)(tokA + tstep * (cc * C + t)) * p.Hv + h] = Gi * (1.f / kLog2e);
                    }
                }
                const int i = r2 & 63;
                float f = inv;
                if (r2 >= C) {
                    const float Gr = p.read_pre ? (i > 0 ? SS.G[pb][i - 1] : 0.f) : SS.G[pb][i];
                    f = p.scale * ex2(Gr) * inv;
                }
                if (i < row_lo(cc) || i >= Cc) f = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const uint32_t w[4] = {vals[c8].x, vals[c8].y, vals[c8].z, vals[c8].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __fmul2_rn(unpack_bf16x2(w[e]), make_float2(f, f));
                        hv[c8 * 4 + e] = pack_f16x2(x.x, x.y);
                    }
                }
                // V to fp16 in place, four 16-byte pieces per thread (every bf16 value of the
                // fp16 range is exact in fp16), rows past the chunk to zero; the swizzle only
                // permutes the pieces within a row, so a piece's row is its offset / 128
                uint4* vt = reinterpret_cast<uint4*>(sm + OFF_V + pb * V_STRIDE);
                constexpr int kVPieces = (kDh / 64) * 512 / kPrep;
                uint4 vw[kVPieces];
#pragma unroll
                for (int m = 0; m < kVPieces; ++m) vw[m] = vt[pt + m * kPrep];
#pragma unroll
                for (int m = 0; m < kVPieces; ++m) {
                    const int idx = pt + m * kPrep;
                    const uint32_t wi[4] = {vw[m].x, vw[m].y, vw[m].z, vw[m].w};
                    uint32_t wo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 xv = unpack_bf16x2(wi[e]);
                        wo[e] = h2(xv.x, xv.y);
                    }
                    vt[idx] = ((idx & 511) >> 3) < Cc ? make_uint4(wo[0], wo[1], wo[2], wo[3])
                                                      : make_uint4(0, 0, 0, 0);
                }
            }
            if (!wg_wait(MB_M0, c & 1, kBarPrep)) { fail = true; break; }
            // P3: columns [32 hf, 32 hf + 32) of row r of D0, with the norms applied: A (fp32,
            //     rows 0-63) and P (fp16, rows 64-127); the fp16 operands go over the bf16 tile
            //     (read by the product) while the accumulator load is in flight
            {
                // warp 8 has no store here: it issues the next chunk's tensor loads
                if (use_tma && has_next && pt == 128) {
                    // (adjoint: the chain's first products of step c - 1 read the value tile)
                    if (!kAdj || c == 0 || mbar_wait_bounded(&SS.mbar[MB_M1], (uint32_t)((c - 1) & 1), kWaitLimitNs)) {
                        load_chunk(c + 1);
                        ld_pending = c + 1;
                    }
                }
                const int i = r & 63;
                const bool live = i >= row_lo(cc) && i < Cc;
                const bool split = SS.split_ok[pb];
                float* As = reinterpret_cast<float*>(sm + OFF_AS);
                uint32_t rr[32];
                tmem_ld32(tlane + TM_D0 + hf * 32, rr);
                float ckv[32];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 x = *reinterpret_cast<const float4*>(&SS.ck[hf * 32 + e4 * 4]);
                    ckv[e4 * 4] = x.x; ckv[e4 * 4 + 1] = x.y; ckv[e4 * 4 + 2] = x.z; ckv[e4 * 4 + 3] = x.w;
                }
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8)
                    *reinterpret_cast<uint4*>(rowp + sw128(r2, c8)) =
                        make_uint4(hv[c8 * 4], hv[c8 * 4 + 1], hv[c8 * 4 + 2], hv[c8 * 4 + 3]);
                // row factor (beta_i / ||k_i|| or scale / ||q_i||, times 2^(G'_i - G_ref) when
                // split) and, without the split, the per-element decay exponent's row part
                const float Gi = r < C ? SS.G[pb][i]
                                       : (p.read_pre ? (i > 0 ? SS.G[pb][i - 1] : 0.f) : SS.G[pb][i]);
                float fi = live ? (r < C ? SS.b[pb][i] : p.scale) * SS.inv[r] : 0.f;
                if (split) fi *= r < C ? SS.Er[i] : SS.Eq[i];
                tmem_wait_ld();
                float vals[32];
                if (split) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) vals[u] = fi * u2f(rr[u]) * ckv[u];
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        vals[u] = fi * u2f(rr[u]) * ckv[u] * ex2(Gi - SS.G[pb][hf * 32 + u]);
                }
                // The solve reads the 16x16 blocks of A below the diagonal and the diagonal
                // blocks (strictly lower part, transposed); the rest of A is never read.  Warp 5
                // (rows 32-63, columns 0-31) holds only blocks below the diagonal; warps 4 and
                // 9 hold the diagonal blocks (0, 1 and 2, 3), which they invert at once, and in
                // lanes 16-31 one block below them (A_10, A_32); warp 8 holds none of them.
                if (pw == 1) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4)
                        *reinterpret_cast<float4*>(f32sw(As, i, e4 * 4)) =
                            make_float4(vals[e4 * 4], vals[e4 * 4 + 1], vals[e4 * 4 + 2], vals[e4 * 4 + 3]);
                    // then the next chunk's cumulative decay, off the critical path
                    if (has_next)
                        chunk_cumsum(2 * lane < Cn ? XG(gate_bits_to_float(g_nx0, p.gt)) : 0.f,
                                     2 * lane + 1 < Cn ? XG(gate_bits_to_float(g_nx1, p.gt)) : 0.f,
                                     pb ^ 1);
                } else if (pw == 0 || pw == 5) {
                    wy_diag_stage0(vals, i, lane, hf, As, reinterpret_cast<float*>(sm + OFF_RS),
                                   reinterpret_cast<float*>(sm + OFF_TWU));
                } else if (r >= C) {
#pragma unroll
                    for (int e8 = 0; e8 < 4; ++e8) {
                        float pv[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int j = hf * 32 + e8 * 8 + u;
                            const bool on = p.read_pre ? (j < i) : (j <= i);
                            pv[u] = on ? vals[e8 * 8 + u] : 0.f;
                        }
                        *reinterpret_cast<uint4*>(sm + OFF_P + pb * 8192 + sw128(i, hf * 4 + e8)) =
                            h8(pv);
                    }
                }
            }

            // P4: T = (I + A)^-1 by 16-blocks.  Stage 0 (the four diagonal inverses, above,
            //     while the Q-row warps form P), then the blocks below the diagonal in three
            //     phases of tf32 warp MMAs, each K-step of W and U~ issued as its block column
            //     of T_w, T_u completes.
            wy_solve_offdiag(reinterpret_cast<float*>(sm + OFF_AS), reinterpret_cast<float*>(sm + OFF_TWU),
                             reinterpret_cast<float*>(sm + OFF_RS), sm + OFF_WN + pb * 16384, SS.bg,
                             SS.b[pb], pt, kBarPrep, kPrep, [&](int phase) {
                                 if (pt != 192) return;
                                 tc_fence_after();
                                 if (phase == 1) {
                                     issue_w(KQ, pb, 3);
                                     issue_w(KQ, pb, 2);
                                     if (!kAdj) {
                                         issue_u(VV, pb, 3);
                                         issue_u(VV, pb, 2);
                                     }
                                 } else {
                                     issue_w(KQ, pb, 1);
                                     if (!kAdj) issue_u(VV, pb, 1);
                                 }
                             });
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarPrep, kPrep);
            tc_fence_after();

            // P5, last step: block column 0; the commit covers every K-step issued before.  The
            // chain reads W^T out of D0 itself, so the chunk is handed over right away.
            if (pt == 192) {
                issue_w(KQ, pb, 0);
                if (!kAdj) issue_u(VV, pb, 0);
                mma_commit(&SS.mbar[MB_MU]);
            }
            if (has_next && pt < C)
                SS.b[pb ^ 1][pt] = pt < Cn ? XB(gate_bits_to_float(b_nx, p.gt)) : 0.f;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&SS.mbar[MB_PREP + pb]);
        }
        cp_async_wait<0>();
        if (ld_pending >= 0)
            mbar_wait_bounded(&SS.mbar[MB_LD + ld_pending % 3], (uint32_t)((ld_pending / 3) & 1),
                              kWaitLimitNs);
    } else {
        // =============================== chain warpgroup ===============================
        const int j = lt;  // dv column = TMEM lane

        if constexpr (kAdj) {
            // ---------------- adjoint chain: dH^T (lane = dv column e) from dS_final back
            // to dS0.  Per chunk (last to first), with dH+ the gradient of its final state:
            //   dV'^T = dO^T P + diag-free (dH+^T K^T) diag(Kd)     (dV' = P^T dO + K~ dH+)
            //   dH^T  = e^(G_last) dH+^T + dO^T Q~ + dV'^T (-W)
#pragma unroll 1
            for (int d0 = 0; d0 < D; d0 += 32) {
                uint32_t r[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    r[e] = __float_as_uint(p.S0 ? p.S0[sb + (size_t)(d0 + e) * D + j] : 0.f);
                tmem_st32(tlane + TM_HM + d0, r);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();
            for (int c = 0; c < nchunks; ++c) {
                const int pb = c & 1, cc = chunk_of(c);
                const uint32_t KQ = sbase + OFF_KQ + (c % 3) * KQ_STRIDE;
                const uint32_t VV = sbase + OFF_V + pb * V_STRIDE;
                const int Cc = min(C, L - cc * C);
                if (!wg_wait(MB_PREP + pb, (c >> 1) & 1, kBarChain)) { fail = true; break; }
                if (!wg_wait(MB_MU, c & 1, kBarChain)) { fail = true; break; }
                // -W^T into WN[pb] (rows d): the B operand of dV'^T (-W), K-major
                {
                    uint32_t rw[2][32];
                    tmem_ld32(tlane + TM_D0, rw[0]);
                    tmem_ld32(tlane + TM_D0 + 32, rw[1]);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&SS.mbar[MB_D0F]);
#pragma unroll
                    for (int half = 0; half < 2; ++half)
#pragma unroll
                        for (int e8 = 0; e8 < 4; ++e8) {
                            float f[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) f[u] = -u2f(rw[half][e8 * 8 + u]);
                            *reinterpret_cast<uint4*>(sm + OFF_WN + pb * 16384 + sw128(lt, half * 4 + e8)) =
                                h8(f);
                        }
                }
                // dH+ -> this chunk's slot of sv_H ([d][e]), an fp16 copy (A operand), and
                // e^(G_last) dH+ back into the accumulator
                {
                    const float gam = SS.gam_adj[pb];
                    float* hc = p.sv_H + ((size_t)(p.chunk_off[s] + cc) * p.Hv + h) * (D * D) + j;
#pragma unroll 1
                    for (int d0 = 0; d0 < D; d0 += 32) {
                        uint32_t r[32], hb[16];
                        tmem_ld32(tlane + TM_HM + d0, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float x0 = u2f(r[2 * e]), x1 = u2f(r[2 * e + 1]);
                            omax = max_abs_nan(omax, x0);
                            omax = max_abs_nan(omax, x1);
                            hc[(size_t)(d0 + 2 * e) * D] = x0;
                            hc[(size_t)(d0 + 2 * e + 1) * D] = x1;
                            hb[e] = h2(x0, x1);
                            r[2 * e] = __float_as_uint(x0 * gam);
                            r[2 * e + 1] = __float_as_uint(x1 * gam);
                        }
                        tmem_st16(tlane + TM_HB + d0 / 2, hb);
                        tmem_st32(tlane + TM_HM + d0, r);
                    }
                    tmem_wait_st();
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(kBarChain, 128);
                // dO^T P (DU half 0; A = the fp16 dO tile, MN-major; B = P, MN-major) and
                // dH+^T K^T (DU half 1; A = the fp16 dH+ copy; B = the K^ rows, K-major)
                if (lt == 0) {
                    tc_fence_after();
                    const uint32_t i1 = idesc_f32acc(128, 64, true, true, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f32acc_ss(tmem + TM_DU, sdesc_sw128(VV + kk * 2048, 8192, 1024),
                                      sdesc_sw128(sbase + OFF_P + pb * 8192 + kk * 2048, 8192, 1024), i1, kk > 0);
                    const uint32_t i2 = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_f32acc_ts(tmem + TM_DU + 64, tmem + TM_HB + kk * 8,
                                      sdesc_sw128(KQ + off, 16, 1024), i2, kk > 0);
                    }
                    // dH^T += dO^T Q~ (B = the Q~ rows, MN-major): the dO tile's last reader, so
                    // this commit also frees it for the preparation's next loads
                    const uint32_t i3 = idesc_f32acc(128, 128, true, true, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f32acc_ss(tmem + TM_HM, sdesc_sw128(VV + kk * 2048, 8192, 1024),
                                      sdesc_sw128(KQ + 8192 + kk * 2048, 16384, 1024), i3, 1);
                    mma_commit(&SS.mbar[MB_M1]);
                }
                if (!wg_wait(MB_M1, c & 1, kBarChain)) { fail = true; break; }
                // dV'^T = dO^T P + (dH+^T K^T) diag(Kd) -> sv_V and the fp16 copy TM_VP
                {
                    float* vrow = p.sv_V + ((size_t)(tokA + tstep * cc * C) * p.Hv + h) * D + j;
                    const long long rstep = tstep * (long long)p.Hv * D;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t r1[32], r2[32], pk[16];
                        tmem_ld32(tlane + TM_DU + half * 32, r1);
                        tmem_ld32(tlane + TM_DU + 64 + half * 32, r2);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int i0 = half * 32 + 2 * e;
                            const float a0 = fmaf(SS.Kd[pb][i0], u2f(r2[2 * e]), u2f(r1[2 * e]));
                            const float a1 = fmaf(SS.Kd[pb][i0 + 1], u2f(r2[2 * e + 1]), u2f(r1[2 * e + 1]));
                            omax = max_abs_nan(omax, a0);
                            omax = max_abs_nan(omax, a1);
                            if (i0 < Cc) vrow[rstep * i0] = a0;
                            if (i0 + 1 < Cc) vrow[rstep * (i0 + 1)] = a1;
                            pk[e] = h2(a0, a1);
                        }
                        tmem_st16(tlane + TM_VP + half * 16, pk);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                named_bar(kBarChain, 128);
                // dH^T += dV'^T (-W) (B = WN[pb], K-major)
                if (lt == 0) {
                    tc_fence_after();
                    const uint32_t i4 = idesc_f32acc(128, 128, false, false, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f32acc_ts(tmem + TM_HM, tmem + TM_VP + kk * 8,
                                      sdesc_sw128(sbase + OFF_WN + pb * 16384 + kk * 32, 16, 1024), i4, 1);
                    mma_commit(&SS.mbar[MB_M3 + pb]);
                }
                if (!wg_wait(MB_M3 + pb, (c >> 1) & 1, kBarChain)) { fail = true; break; }
                mbar_arrive(&SS.mbar[MB_CD + pb]);  // the step's buffers are free
                tc_fence_before();
                named_bar(kBarChain, 128);
                tc_fence_after();
            }
            // dS0: dH^T after the first chunk ([d][e])
            if (!fail) {
#pragma unroll 1
                for (int d0 = 0; d0 < D; d0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tlane + TM_HM + d0, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        omax = max_abs_nan(omax, u2f(r[e]));
                        if (p.S_final) p.S_final[sb + (size_t)(d0 + e) * D + j] = u2f(r[e]);
                    }
                }
            }
        } else {
        {
            // initial state -> TM_HM (pre-scaled by chunk 0's total decay), TM_HB (fp16)
            const float gv = lt >= rofs && lt < min(C, L) ? XG(gate_at(gsrc, lt)) : 0.f;
            const float part = warp_sum(gv);
            if (lane == 0 && warp < 2) SS.gsum_part[warp] = part;
            named_bar(kBarChain, 128);
            const float gam = ex2((SS.gsum_part[0] + SS.gsum_part[1]) * kLog2e);
#pragma unroll 1
            for (int d0 = 0; d0 < D; d0 += 32) {
                uint32_t r[32], hb[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const bool in = p.S0 && d0 + e < kDh && j < kDh;
                    const float x0 = in ? p.S0[sb + (size_t)(d0 + e) * kDh + j] : 0.f;
                    const float x1 = in ? p.S0[sb + (size_t)(d0 + e + 1) * kDh + j] : 0.f;
                    r[e] = __float_as_uint(x0 * gam);
                    r[e + 1] = __float_as_uint(x1 * gam);
                    hb[e >> 1] = h2(x0, x1);
                    if constexpr (kSave) {
                        float* hc = p.sv_H + ((size_t)p.chunk_off[s] * p.Hv + h) * (D * D) + j;
                        hc[(size_t)(d0 + e) * D] = x0;
                        hc[(size_t)(d0 + e + 1) * D] = x1;
                    }
                }
                tmem_st32(tlane + TM_HM + d0, r);
                tmem_st16(tlane + TM_HB + d0 / 2, hb);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();
        }
        const bool check_o = !p.qk_l2norm || !(fabsf(p.scale) <= 1024.f);
        // bidirectional pair: a chunk's fp32 output left for the partner and not announced yet
        bool sig_pending = false;
        auto pair_flush = [&]() {
            if (!sig_pending) return;
            named_bar(kBarChain, 128);  // every thread's stores of the chunk precede the release
            if (lt == 0) {
                __threadfence();
                cluster_add_release(cluster_map(smem_u32(&SS.pair_cnt), rev ? 0u : 1u), 1u);
            }
            sig_pending = false;
        };
        for (int c = 0; c < nchunks; ++c) {
            const int pb = c & 1;
            const uint32_t KQ = sbase + OFF_KQ + (c % 3) * KQ_STRIDE;
            const int Cc = min(C, L - c * C);
            const bool has_next = c + 1 < nchunks;
            const int Cn = has_next ? min(C, L - (c + 1) * C) : 0;
            // loaded unconditionally from an in-bounds position, masked when reduced in C2
            uint32_t g_raw = 0;
            if (has_next) g_raw = gate_bits_at(gsrc, (c + 1) * C + min(lt & 63, Cn - 1));

            if (!wg_wait(MB_PREP + pb, (c >> 1) & 1, kBarChain)) { fail = true; break; }
            // C0: -W^T (the preparation's W product, in D0; row = dk = this lane) into WN[pb] as
            //     the B operand of V' (MN-major), once the W and U~ products are done (they read
            //     T_w, T_u from the same buffer); D0 is then released for the next chunk
            if (!wg_wait(MB_MU, c & 1, kBarChain)) { fail = true; break; }
            {
                uint32_t rw[2][32];
                tmem_ld32(tlane + TM_D0, rw[0]);
                tmem_ld32(tlane + TM_D0 + 32, rw[1]);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&SS.mbar[MB_D0F]);
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int e8 = 0; e8 < 4; ++e8) {
                        float f[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) f[u] = -u2f(rw[half][e8 * 8 + u]);
                        *reinterpret_cast<uint4*>(sm + OFF_WN + pb * 16384 + sw128(lt, half * 4 + e8)) =
                            h8(f);
                    }
                fence_proxy_async_smem();
            }
            named_bar(kBarChain, 128);
            // C1: V'^T = U~^T + H^T (-W^T);  O^T = H^T Q~^T   (A = state copy in TMEM)
            if (lt == 0) {
                tc_fence_after();
                const uint32_t id1 = idesc_f32acc(128, 64, false, true, false);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f32acc_ts(tmem + TM_DU + pb * 64, tmem + TM_HB + kk * 8,
                                  sdesc_sw128(sbase + OFF_WN + pb * 16384 + kk * 2048, 8192, 1024),
                                  id1, 1);
                // V' is all C2 needs: its barrier fires before the output product runs; the
                // commit after C3 covers the output product
                mma_commit(&SS.mbar[MB_M1]);
                const uint32_t id2 = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_f32acc_ts(tmem + TM_DO, tmem + TM_HB + kk * 8,
                                  sdesc_sw128(KQ + off + 8192, 16, 1024), id2, kk > 0);
                }
            }
            if (!wg_wait(MB_M1, c & 1, kBarChain)) { fail = true; break; }

            // C2: V'^T -> fp16 packed in TMEM, plain (output) and scaled by Kd (state update)
            {
                uint32_t rv[2][32];
                tmem_ld32(tlane + TM_DU + pb * 64, rv[0]);
                tmem_ld32(tlane + TM_DU + pb * 64 + 32, rv[1]);
                tmem_wait_ld();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[16], ps[16];
                    const uint32_t* r = rv[half];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 kd = *reinterpret_cast<const float4*>(&SS.Kd[pb][half * 32 + 4 * e4]);
                        const float a0 = u2f(r[4 * e4]), b0 = u2f(r[4 * e4 + 1]);
                        const float a1 = u2f(r[4 * e4 + 2]), b1 = u2f(r[4 * e4 + 3]);
                        pk[2 * e4] = h2(a0, b0);
                        pk[2 * e4 + 1] = h2(a1, b1);
                        ps[2 * e4] = h2(a0 * kd.x, b0 * kd.y);
                        ps[2 * e4 + 1] = h2(a1 * kd.z, b1 * kd.w);
                    }
                    tmem_st16(tlane + TM_VP + half * 16, pk);
                    tmem_st16(tlane + TM_VS + half * 16, ps);
                }
                tmem_wait_st();
                if (warp < 2) {
                    const float part = warp_sum(lt < Cn ? XG(gate_bits_to_float(g_raw, p.gt)) : 0.f);
                    if (lane == 0) SS.gsum_part[warp] = part;
                }
            }
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();

            // C3: O^T += V'^T P^T (N=64, K=64);  H^T += (Kd V')^T K (N=128, K=64, B MN-major)
            if (lt == 0) {
                const uint32_t id3 = idesc_f32acc(128, 64, false, false, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f32acc_ts(tmem + TM_DO, tmem + TM_VP + kk * 8,
                                  sdesc_sw128(sbase + OFF_P + pb * 8192 + kk * 32, 16, 1024), id3, 1);
                const uint32_t id4 = idesc_f32acc(128, 128, false, true, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f32acc_ts(tmem + TM_HM, tmem + TM_VS + kk * 8,
                                  sdesc_sw128(KQ + kk * 2048, 16384, 1024), id4, 1);
                mma_commit(&SS.mbar[MB_M3 + pb]);
            }
            // Bidirectional pair: chunk u of the forward order.  The scan that reaches it first
            // (the forward one in the first half of the sequence, the reverse one in the second)
            // leaves its fp32 output in the workspace and advances its partner's counter; the
            // other adds it to its own and rounds the sum once.  Reverse row i is forward row
            // 63 - i.  The counter moves one chunk late (a fence right after the stores would
            // wait for all of them), always before this CTA waits for its partner.  Each waits
            // only for chunks its partner reached at an earlier step and announced by the start
            // of this step's wait, before which the partner waits for nothing from it, so the
            // two CTAs of the cluster (resident together) cannot wait on each other.
            const int u = kPair && rev ? nchunks - 1 - c : c;
            const bool second = kPair && (rev ? 2 * u <= nchunks - 1 : 2 * u > nchunks - 1);
            float* const part = kPair ? p.part + ((size_t)(p.chunk_off[s] + u) * p.Hv + h) * (C * kDh)
                                      : nullptr;
            if constexpr (kPair) pair_flush();
            if (!wg_wait(MB_M3 + pb, (c >> 1) & 1, kBarChain)) { fail = true; break; }

            // C4: O -> staged in WN[pb] -> global (two tensor stores for a full chunk, else
            //     coalesced 16-byte stores); state -> fp16 copy, pre-scaled for the next chunk
            {
                // staging: two [token][64] bf16 tiles (dv halves) in the 128-byte-swizzled
                // layout of the output tensor map's box
                uint8_t* stage = sm + OFF_WN + pb * 16384;
                uint8_t* stage_j = stage + (j >> 6) * 8192 + (j & 7) * 2;
                const int cj = (j & 63) >> 3;
                uint32_t ro[2][32];
                tmem_ld32(tlane + TM_DO, ro[0]);
                tmem_ld32(tlane + TM_DO + 32, ro[1]);
                tmem_wait_ld();
                // Output rows: this chunk's own (tok = tokA + tstep (64 c + row)), or in a
                // bidirectional pair the forward chunk u both scans cover, in forward order.
                const long long obase = kPair ? t0 + (long long)C * u : tokA + tstep * (long long)c * C;
                const long long ostep = kPair ? 1 : tstep;
                const int olo = kPair ? 0 : row_lo(c);
                const int ohi = kPair ? min(C, Lseq - C * u) : Cc;
                bool emit = !kSave;  // this CTA writes the chunk's output
                if constexpr (kPair) {
                    if (!second) {
                        if (j < kDh) {
#pragma unroll
                            for (int i = 0; i < C; ++i)
                                __stcg(part + (rev ? C - 1 - i : i) * kDh + j, u2f(ro[i >> 5][i & 31]));
                        }
                        sig_pending = true;
                        emit = false;
                    } else {
                        bool ok = true;
                        if (lt == 0)
                            ok = counter_wait_bounded(smem_u32(&SS.pair_cnt),
                                                      (uint32_t)(rev ? u + 1 : nchunks - u), kWaitLimitNs);
                        if (!group_agree(ok, kBarChain)) { fail = true; break; }
                        if (j < kDh) {
#pragma unroll
                            for (int i = 0; i < C; ++i)
                                ro[i >> 5][i & 31] = __float_as_uint(
                                    u2f(ro[i >> 5][i & 31]) + __ldcg(part + (rev ? C - 1 - i : i) * kDh + j));
                        }
                    }
                }
                if (emit) {
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int m = 0; m < 32; ++m) {
                        const int row = kPair && rev ? C - 1 - (half * 32 + m) : half * 32 + m;
                        *reinterpret_cast<__nv_bfloat16*>(stage_j + sw128(row, cj)) =
                            __float2bfloat16_rn(u2f(ro[half][m]));
                    }
                // with normalised q, k and |scale| <= 1024 the operands that reach only the
                // output (P, Q~) are bounded by |scale|; otherwise every output is checked
                if (check_o) {
#pragma unroll
                    for (int m = 0; m < 64; ++m) omax = max_abs_nan(omax, u2f(ro[m >> 5][m & 31]));
                }
                fence_proxy_async_smem();
                named_bar(kBarChain, 128);
                if (p.tma_store && olo == 0 && ohi == C) {
                    if (lt == 0) {
                        const int z = (int)obase;
                        const uint32_t src = sbase + OFF_WN + pb * 16384;
                        tma_store_3d(&tm_o, src, 0, h, z);
                        if (kDh > 64) tma_store_3d(&tm_o, src + 8192, 64, h, z);
                        bulk_commit();
                    }
                } else {
                // 16-byte chunks, consecutive threads on consecutive chunks of a row
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int idx = m * 128 + lt, row = idx >> 4, c16 = idx & 15;
                    if (row >= olo && row < ohi && c16 < kDh / 8) {
                        const long long tok = obase + ostep * row;
                        uint4* dp = reinterpret_cast<uint4*>(p.o + ((size_t)tok * p.Hv + h) * kDh + c16 * 8);
                        uint4 a = *reinterpret_cast<const uint4*>(stage + (c16 >> 3) * 8192 +
                                                                  sw128(row, c16 & 7));
                        if (p.o_acc) {
                            const uint4 b = *dp;
                            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
                            uint32_t ow[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 x = unpack_bf16x2(aw[e]), y = unpack_bf16x2(bw[e]);
                                ow[e] = pack_bf16x2(x.x + y.x, x.y + y.y);
                            }
                            a = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                        }
                        *dp = a;
                    }
                }
                }
                }
                const float gam = has_next ? ex2((SS.gsum_part[0] + SS.gsum_part[1]) * kLog2e) : 1.f;
                if (has_next) {
#pragma unroll
                    for (int d0 = 0; d0 < D; d0 += 64) {
                        uint32_t r2[2][32];
                        tmem_ld32(tlane + TM_HM + d0, r2[0]);
                        tmem_ld32(tlane + TM_HM + d0 + 32, r2[1]);
                        tmem_wait_ld();
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t (&r)[32] = r2[hh];
                            const int dd = d0 + hh * 32;
                            uint32_t hb[16];
                            // the saving forward's state leaves through the free staging slab WN[pb]
                            // by bulk stores (off the chain's path); the slab is rewritten once
                            // the previous slab's store has read it
                            if constexpr (kSave) {
                                if (dd > 0) {
                                    if (lt == 0) bulk_wait_read();
                                    named_bar(kBarChain, 128);
                                }
                            }
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const float2 x = make_float2(u2f(r[2 * e]), u2f(r[2 * e + 1]));
                                if constexpr (kSave) {
                                    float* stg = reinterpret_cast<float*>(sm + OFF_WN + pb * 16384);
                                    stg[(2 * e) * D + lt] = x.x;
                                    stg[(2 * e + 1) * D + lt] = x.y;
                                }
                                hb[e] = h2(x.x, x.y);
                                const float2 y = __fmul2_rn(x, make_float2(gam, gam));
                                r[2 * e] = __float_as_uint(y.x);
                                r[2 * e + 1] = __float_as_uint(y.y);
                            }
                            tmem_st16(tlane + TM_HB + dd / 2, hb);
                            tmem_st32(tlane + TM_HM + dd, r);
                            if constexpr (kSave) {  // rows dd .. dd + 31 of the state, 16 KB contiguous
                                fence_proxy_async_smem();
                                named_bar(kBarChain, 128);
                                if (lt == 0) {
                                    float* hc = p.sv_H + ((size_t)(p.chunk_off[s] + c + 1) * p.Hv + h) * (D * D) + (size_t)dd * D;
                                    bulk_store(hc, sbase + OFF_WN + pb * 16384, 16384u);
                                    bulk_commit();
                                }
                            }
                        }
                    }
                } else {
                    // the final state, once per sequence (column j of the transposed state);
                    // an operand that left the fp16 range on the state's path shows here
#pragma unroll 1
                    for (int d0 = 0; d0 < kDh; d0 += 32) {
                        uint32_t r[32];
                        tmem_ld32(tlane + TM_HM + d0, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            omax = max_abs_nan(omax, u2f(r[e]));
                            if (p.S_final && j < kDh)
                                p.S_final[sb + (size_t)(d0 + e) * kDh + j] = u2f(r[e]);
                        }
                    }
                }
                if constexpr (kSave) {
                    // V' (lane = e), after the state slabs' proxy fences: V'^T stays in DU[pb]
                    // until the release below lets the preparation's U~ product reuse it
                    float* vrow = p.sv_V + ((size_t)(tokA + tstep * c * C) * p.Hv + h) * D + lt;
                    const long long rstep = tstep * (long long)p.Hv * D;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t rv[32];
                        tmem_ld32(tlane + TM_DU + pb * 64 + half * 32, rv);
                        tmem_wait_ld();
#pragma unroll
                        for (int m = 0; m < 32; ++m) {
                            const int i = half * 32 + m;
                            if (i >= row_lo(c) && i < Cc) vrow[rstep * i] = u2f(rv[m]);
                        }
                    }
                    tc_fence_before();
                }
                tmem_wait_st();
                if (lt == 0) bulk_wait_read();  // the staging buffer is free for reuse
                mbar_arrive(&SS.mbar[MB_CD + pb]);
            }
            tc_fence_before();
            named_bar(kBarChain, 128);
            tc_fence_after();
        }
        if constexpr (kPair) pair_flush();  // the last chunk left for the partner
        }  // forward chain
    }

    if (tid == 0) bulk_wait_all();  // output tiles written before the CTA exits
    if (fail && (tid == 0 || tid == 128 || tid == 256)) atomicExch(&p.hdr->err, (int)GDR_ERR_TIMEOUT);
    tc_fence_before();
    // an fp16 operand that left its range shows as a non-finite output or final state
    if (__syncthreads_or(omax <= 3.4e38f ? 0 : 1) && tid == 0)
        atomicCAS(&p.hdr->err, (int)GDR_OK, (int)GDR_ERR_RANGE);
    // no CTA of a pair leaves while its partner may still advance its counter
    if constexpr (kPair) cluster_sync_all();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
    griddep_wait();
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda)
EncodeTiledFn encode_tiled() {
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

// [tokens][heads][dim] bf16 viewed as a 3-D tensor (dim, heads, tokens); box 64 x 1 x 64
// with the 128-byte swizzle, i.e. one 8 KB K-major atom stack of the kernel's layout.
bool make_tile_map(CUtensorMap* m, const void* base, int heads, long long tokens, int dim) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)dim * 2, (cuuint64_t)heads * dim * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(const gdr_chunk_args& a) {
    return a.io_dtype == GDR_BF16 && a.dk == a.dv && (a.dk == D || a.dk == 64) && a.chunk == C &&
           !a.gdn2;
}

gdr_status launch_chunk_tc(const gdr_chunk_args& a, const void* q, const void* k, const void* v,
                           const void* g, const void* beta, const float* S0, void* o,
                           float* S_final, void* ws, const WsLayout& L, cudaStream_t st,
                           bool dependent, const void* g_rev, const void* beta_rev,
                           size_t part_off, const TcSave* save) {
    const bool pair = g_rev != nullptr;  // bidirectional: both scans, one cluster per pair
    char* base = static_cast<char*>(ws);
    TcParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.g = g; p.beta = beta; p.S0 = S0;
    p.o = static_cast<__nv_bfloat16*>(o); p.S_final = S_final;
    p.hdr = reinterpret_cast<WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.order = reinterpret_cast<const int32_t*>(base + L.order);
    p.Hk = a.Hk; p.Hv = a.Hv; p.read_pre = a.read_mode == GDR_READ_PRE;
    p.qk_l2norm = a.qk_l2norm; p.reverse = a.reverse; p.o_acc = a.o_accumulate;
    p.gt = a.gate_dtype; p.scale = a.scale;
    p.g_rev = g_rev; p.beta_rev = beta_rev;
    p.chunk_off = reinterpret_cast<const int32_t*>(base + L.chunk_off);
    p.part = pair ? reinterpret_cast<float*>(base + part_off) : nullptr;
    p.sv_G = save ? save->G : nullptr;
    p.sv_H = save ? save->H : nullptr;
    p.sv_V = save ? save->V : nullptr;
    const GateParams gp{a.gate_A, a.gate_dt_bias, a.beta_scale};
    CUtensorMap tq, tk, tv, to;
    memset(&tq, 0, sizeof(tq));
    memset(&tk, 0, sizeof(tk));
    memset(&tv, 0, sizeof(tv));
    memset(&to, 0, sizeof(to));
    const long long T_tot = (long long)a.B * a.T;
    p.use_tma = 0;
    p.tma_store = 0;
    // tensor maps for forward scans (a pair's forward CTA included); reversed scans gather
    // rows with cp.async instead.  A pair writes whole forward chunks from either CTA.
    if ((!a.reverse || pair) && T_tot > 0) {
        if (!make_tile_map(&tq, q, a.Hk, T_tot, a.dk) || !make_tile_map(&tk, k, a.Hk, T_tot, a.dk) ||
            !make_tile_map(&tv, v, a.Hv, T_tot, a.dv))
            return GDR_ERR_CUDA;
        p.use_tma = 1;
        // accumulating outputs are read back, so they keep the plain stores
        p.tma_store = !save && !a.o_accumulate && make_tile_map(&to, o, a.Hv, T_tot, a.dv);
    }
    auto kernel = pair ? (a.dk == D ? (a.gate_raw ? chunk_fused_tc<true, D, true, false, false> : chunk_fused_tc<false, D, true, false, false>)
                                    : (a.gate_raw ? chunk_fused_tc<true, 64, true, false, false> : chunk_fused_tc<false, 64, true, false, false>))
                       : (a.dk == D ? (a.gate_raw ? chunk_fused_tc<true, D, false, false, false> : chunk_fused_tc<false, D, false, false, false>)
                                    : (a.gate_raw ? chunk_fused_tc<true, 64, false, false, false> : chunk_fused_tc<false, 64, false, false, false>));
    if (save) kernel = save->adjoint ? chunk_fused_tc<false, D, false, false, true>
                                     : chunk_fused_tc<false, D, false, true, false>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES) != cudaSuccess)
        return GDR_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.n_seqs * (unsigned)a.Hv * (pair ? 2u : 1u));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (dependent) {  // may start while the stream's previous grid finishes (see the kernel)
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (pair) {  // the two scans of a (sequence, head) run together on one cluster
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, kernel, p, tq, tk, tv, to, gp) != cudaSuccess) return GDR_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
