// chunk_simt.cu -- fp32 CUDA-core evaluation of the chunk-wise WY/UT forward.
//
// This path serves fp32 inputs (whose 1e-4 bound rules out bf16/tf32 tensor-core
// operands) and the shapes the tensor-core kernel does not cover.  Two kernels:
//
//  chunk_local_simt  one block per (chunk, value head), all chunks in parallel.
//     With the in-chunk log decay G_i = g_1 + ... + g_i (Prizma "seq/delta.py",
//     chunked_delta: cumulative decay kept in log space) it forms
//        A_ij = beta_i (k_i . k_j) exp(G_i - G_j),  j < i,
//     and solves the unit-lower system (I + A) X = R by forward substitution
//     (the page's _solve_unit_lower) for the two right-hand sides
//        W = (I + A)^-1 diag(beta exp(G)) K,   U~ = (I + A)^-1 diag(beta) V,
//     which do not depend on the chunk's initial state (flashrt fused_layer.py
//     `_wy_core`: recompute_wu before chunk_h).
//
//  chunk_scan_simt   one block per (sequence, value head, 32-column slice of dv),
//     walking the sequence's chunks in order with its slice of the state H = S^T
//     resident in shared memory.  Per chunk (state carry + output, flashrt
//     `_wy_core`: chunk_h then output_o; Prizma chunked_delta O_inter/O_intra):
//        V' = U~ - W H
//        post: o_i = scale (exp(G_i) q_i H + sum_{j<=i} exp(G_i - G_j)(q_i.k_j) V'_j)
//        pre:  o_i = scale (exp(G_{i-1}) q_i H + sum_{j<i} exp(G_{i-1} - G_j)(q_i.k_j) V'_j)
//        H  <- exp(G_C) H + sum_i exp(G_C - G_i) k_i V'_i^T
//     Every column slice of H evolves independently, so the slices need no
//     communication.  Every decay factor is exp of a log difference that is <= 0.
#include "common.cuh"

namespace gdr {

namespace {

constexpr int kThreads = 256;
constexpr int kSlice = 32;  // dv columns per scan block (one per lane)

struct SimtParams {
    const void* q; const void* k; const void* v; const void* g; const void* beta;
    const float* S0; void* o; float* S_final;
    const WsHeader* hdr; const int32_t* cu; const int32_t* chunk_off; const int32_t* chunk_seq;
    float* W; float* U; float* G;
    int Hk, Hv, dk, dv, chunk, read_pre, qk_l2norm, reverse, o_acc;
    gdr_dtype io, gt;
    float scale;
    int gate_raw;                 // fused gating prologue (see gate_xform)
    const float* gate_A; const float* gate_dt_bias;
    float beta_scale;
    const void* w;                // GDN-2 write gate [T][Hv][dv]; g, beta are then [T][Hv][dk]
    float *Qt, *Kt, *Pc;          // register-blocked scan operands (chunk_prep_simt)
    int g2_factor;                // GDN-2: factored off-diagonal blocks (see decayed_pairs)
};

// Normalise `rows` rows of length n (row stride ld) in shared memory, one warp per row.
__device__ void l2norm_rows(float* x, int rows, int n, int ld) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int i = wid; i < rows; i += kThreads / 32) {
        float ss = 0.f;
        for (int d = lane; d < n; d += 32) ss += x[i * ld + d] * x[i * ld + d];
        ss = warp_sum(ss);
        const float inv = 1.f / fmaxf(sqrtf(ss), kNormEps);
        for (int d = lane; d < n; d += 32) x[i * ld + d] *= inv;
    }
}

__global__ void __launch_bounds__(kThreads)
chunk_local_simt(SimtParams p) {
    extern __shared__ float sm[];
    const WsHeader* hdr = p.hdr;
    if (hdr->err != GDR_OK) return;
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= hdr->n_chunks) return;
    const int s = p.chunk_seq[c];
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int jc = c - p.chunk_off[s];
    const int p0 = jc * p.chunk;
    const int Cc = (int)min((long long)p.chunk, (t1 - t0) - p0);
    const int dk = p.dk, dv = p.dv, ld = dk + dv + 1, C = p.chunk;
    const int hk = h / (p.Hv / p.Hk);

    float* R = sm;                       // [C][ld]: K | V, then W | U~ in place
    float* A = R + C * ld;               // [C][C+1]
    float* Gs = A + C * (C + 1);         // [C]
    float* Bs = Gs + C;                  // [C]
    const int tid = threadIdx.x;

    for (int idx = tid; idx < Cc * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        R[i * ld + d] = load_elem(p.k, (size_t)(t * p.Hk + hk) * dk + d, p.io);
    }
    for (int idx = tid; idx < Cc * dv; idx += kThreads) {
        const int i = idx / dv, d = idx % dv;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        R[i * ld + dk + d] = load_elem(p.v, (size_t)(t * p.Hv + h) * dv + d, p.io);
    }
    for (int i = tid; i < Cc; i += kThreads) {
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Gs[i] = xform_g(p, h, load_elem(p.g, (size_t)t * p.Hv + h, p.gt));
        Bs[i] = xform_beta(p, load_elem(p.beta, (size_t)t * p.Hv + h, p.gt));
    }
    __syncthreads();
    if (p.qk_l2norm) l2norm_rows(R, Cc, dk, ld);
    if (tid == 0) {
        float run = 0.f;
        for (int i = 0; i < Cc; ++i) { run += Gs[i]; Gs[i] = run; }
    }
    __syncthreads();
    // A_ij = beta_i (k_i . k_j) exp(G_i - G_j), j < i
    for (int idx = tid; idx < Cc * Cc; idx += kThreads) {
        const int i = idx / Cc, j = idx % Cc;
        float val = 0.f;
        if (j < i) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot = fmaf(R[i * ld + d], R[j * ld + d], dot);
            val = Bs[i] * dot * expf(Gs[i] - Gs[j]);
        }
        A[i * (C + 1) + j] = val;
    }
    __syncthreads();
    // right-hand sides: rows of K scaled by beta_i exp(G_i), rows of V by beta_i
    for (int idx = tid; idx < Cc * (dk + dv); idx += kThreads) {
        const int i = idx / (dk + dv), col = idx % (dk + dv);
        const float f = col < dk ? Bs[i] * expf(Gs[i]) : Bs[i];
        R[i * ld + col] *= f;
    }
    __syncthreads();
    // forward substitution, one column per thread: x_i = r_i - sum_{j<i} A_ij x_j
    for (int col = tid; col < dk + dv; col += kThreads) {
        for (int i = 1; i < Cc; ++i) {
            float x = R[i * ld + col];
            for (int j = 0; j < i; ++j) x = fmaf(-A[i * (C + 1) + j], R[j * ld + col], x);
            R[i * ld + col] = x;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < Cc * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        p.W[(size_t)(t * p.Hv + h) * dk + d] = R[i * ld + d];
    }
    for (int idx = tid; idx < Cc * dv; idx += kThreads) {
        const int i = idx / dv, d = idx % dv;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        p.U[(size_t)(t * p.Hv + h) * dv + d] = R[i * ld + dk + d];
    }
    for (int i = tid; i < Cc; i += kThreads) {
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        p.G[(size_t)t * p.Hv + h] = Gs[i];
    }
}

__global__ void __launch_bounds__(kThreads)
chunk_scan_simt(SimtParams p) {
    extern __shared__ float sm[];
    if (p.hdr->err != GDR_OK) return;
    const int s = blockIdx.x, h = blockIdx.y, J = blockIdx.z;
    const int dk = p.dk, dv = p.dv, C = p.chunk, ldk = dk + 1;
    const int hk = h / (p.Hv / p.Hk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = J * kSlice + lane;  // this lane's dv column
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);

    float* Hs = sm;                    // [dk][32]
    float* Qs = Hs + dk * kSlice;      // [C][dk+1]
    float* Ks = Qs + C * ldk;          // [C][dk+1]
    float* Ws = Ks + C * ldk;          // [C][dk+1]
    float* Us = Ws + C * ldk;          // [C][33]  U~ then V'
    float* Os = Us + C * (kSlice + 1); // [C][33]  inter-chunk read
    float* P = Os + C * (kSlice + 1);  // [C][C+1]
    float* Gs = P + C * (C + 1);       // [C] in-chunk log decay G_i
    float* Rd = Gs + C;                // [C] read decay exp(G_i) (post) / exp(G_{i-1}) (pre)
    float* Kd = Rd + C;                // [C] carry decay exp(G_C - G_i)

    const size_t sbase = ((size_t)s * p.Hv + h) * dk * dv;
    for (int d = wid; d < dk; d += kThreads / 32)
        Hs[d * kSlice + lane] = p.S0 ? p.S0[sbase + (size_t)d * dv + col] : 0.f;

    for (int p0 = 0; p0 < L; p0 += C) {
        const int Cc = min(C, L - p0);
        __syncthreads();
        for (int idx = tid; idx < Cc * dk; idx += kThreads) {
            const int i = idx / dk, d = idx % dk;
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Qs[i * ldk + d] = load_elem(p.q, (size_t)(t * p.Hk + hk) * dk + d, p.io);
            Ks[i * ldk + d] = load_elem(p.k, (size_t)(t * p.Hk + hk) * dk + d, p.io);
            Ws[i * ldk + d] = p.W[(size_t)(t * p.Hv + h) * dk + d];
        }
        for (int i = wid; i < Cc; i += kThreads / 32) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Us[i * (kSlice + 1) + lane] = p.U[(size_t)(t * p.Hv + h) * dv + col];
            if (lane == 0) Gs[i] = p.G[(size_t)t * p.Hv + h];
        }
        __syncthreads();
        if (p.qk_l2norm) { l2norm_rows(Qs, Cc, dk, ldk); l2norm_rows(Ks, Cc, dk, ldk); }
        for (int i = tid; i < Cc; i += kThreads) {
            const float Gi = p.read_pre ? (i > 0 ? Gs[i - 1] : 0.f) : Gs[i];
            Rd[i] = expf(Gi);
            Kd[i] = expf(Gs[Cc - 1] - Gs[i]);
        }
        __syncthreads();
        // masked, decayed, scaled Q K^T
        for (int idx = tid; idx < Cc * Cc; idx += kThreads) {
            const int i = idx / Cc, j = idx % Cc;
            float val = 0.f;
            if (p.read_pre ? (j < i) : (j <= i)) {
                float dot = 0.f;
                for (int d = 0; d < dk; ++d) dot = fmaf(Qs[i * ldk + d], Ks[j * ldk + d], dot);
                const float Gi = p.read_pre ? (i > 0 ? Gs[i - 1] : 0.f) : Gs[i];
                val = p.scale * dot * expf(Gi - Gs[j]);
            }
            P[i * (C + 1) + j] = val;
        }
        // V' = U~ - W H and the inter-chunk read scale exp(G) q_i H, per (row, lane column)
        for (int i = wid; i < Cc; i += kThreads / 32) {
            float wh = 0.f, qh = 0.f;
            for (int d = 0; d < dk; ++d) {
                const float hv = Hs[d * kSlice + lane];
                wh = fmaf(Ws[i * ldk + d], hv, wh);
                qh = fmaf(Qs[i * ldk + d], hv, qh);
            }
            Us[i * (kSlice + 1) + lane] -= wh;
            Os[i * (kSlice + 1) + lane] = p.scale * Rd[i] * qh;
        }
        __syncthreads();
        // o_i = inter read + sum_j P_ij V'_j
        for (int i = wid; i < Cc; i += kThreads / 32) {
            float acc = Os[i * (kSlice + 1) + lane];
            const int jmax = p.read_pre ? i - 1 : i;
            for (int j = 0; j <= jmax; ++j)
                acc = fmaf(P[i * (C + 1) + j], Us[j * (kSlice + 1) + lane], acc);
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            const size_t oi = (size_t)(t * p.Hv + h) * dv + col;
            if (p.o_acc) acc += load_elem(p.o, oi, p.io);
            store_elem(p.o, oi, acc, p.io);
        }
        // H <- exp(G_C) H + sum_i exp(G_C - G_i) k_i V'_i^T  (H is not read above any more)
        const float gC = expf(Gs[Cc - 1]);
        for (int d = wid; d < dk; d += kThreads / 32) {
            float acc = 0.f;
            for (int i = 0; i < Cc; ++i)
                acc = fmaf(Kd[i] * Ks[i * ldk + d], Us[i * (kSlice + 1) + lane], acc);
            Hs[d * kSlice + lane] = fmaf(gC, Hs[d * kSlice + lane], acc);
        }
    }
    __syncthreads();
    if (p.S_final)
        for (int d = wid; d < dk; d += kThreads / 32)
            p.S_final[sbase + (size_t)d * dv + col] = Hs[d * kSlice + lane];
}

// ---- decayed pair sums over key channels (GDN-2's A and P) ----------------------------
//
//     out_ij = sum_d X_id Y_jd e^{GX_id - GY_jd}   for j <= i,  a [C x C] tile, C <= 64,
//
// thread (rg = tid / 16, cg = tid % 16) owning rows 4 rg + ii and columns cg + 16 jj.  In
// 16-row blocks the thread's rows lie in block I = rg / 4 (the same for both row groups of a
// warp, so branches on it are warp-uniform) and column jj in block J = jj.
//  - Diagonal blocks (J = I): one exp per term, only where j <= i (above, the factor may
//    overflow).
//  - Blocks below them (J < I), when `factor`: with the reference R_I = GY_{16 I - 1} (the
//    decay just before row block I), e^{GX_i - GY_j} = e^{GX_i - R_I} e^{R_I - GY_j}.  While the
//    decay never grows (every g <= 0), GX_i <= R_I <= GY_j, so both factors are <= 1 (no
//    overflow; a factor that underflows belongs to a term that is smaller still), and the
//    block is a plain product of rows scaled once: Xs (rows 16 .. C-1) and Ys (for each I,
//    the rows j < 16 I, stacked from row 8 I (I - 1)).  Without `factor` these blocks take
//    one exp per term as well.
constexpr int kSub = 16;
__host__ __device__ constexpr int ys_rows(int C) { return 8 * (C / kSub) * (C / kSub - 1); }

struct PairOps {
    const float *X, *Y, *GX, *GY;
    int ldx, ldy, lgx, lgy;
};

__device__ void build_factored(float* Xs, float* Ys, int lds, const PairOps& o, int C, int dk) {
    for (int idx = threadIdx.x; idx < (C - kSub) * dk; idx += kThreads) {
        const int i = kSub + idx / dk, d = idx % dk, ref = kSub * (i / kSub) - 1;
        Xs[(i - kSub) * lds + d] =
            o.X[i * o.ldx + d] * expf(o.GX[i * o.lgx + d] - o.GY[ref * o.lgy + d]);
    }
    for (int I = 1; I < C / kSub; ++I)
        for (int idx = threadIdx.x; idx < kSub * I * dk; idx += kThreads) {
            const int j = idx / dk, d = idx % dk, ref = kSub * I - 1;
            Ys[(8 * I * (I - 1) + j) * lds + d] =
                o.Y[j * o.ldy + d] * expf(o.GY[ref * o.lgy + d] - o.GY[j * o.lgy + d]);
        }
}

__device__ __forceinline__ void decayed_pairs(float (&acc)[4][4], const PairOps& o,
                                              const float* Xs, const float* Ys, int lds,
                                              bool factor, int C, int dk) {
    const int rg = threadIdx.x >> 4, cg = threadIdx.x & 15, I = rg >> 2;
    if (4 * rg >= C) return;
    const bool fac = factor && I > 0;
    const float* xs = Xs + (4 * rg - kSub) * lds;  // read only when fac
    const float* ys = Ys + 8 * I * (I - 1) * lds;
    for (int d = 0; d < dk; ++d) {
        float a[4], ga[4], xa[4];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            a[ii] = o.X[(4 * rg + ii) * o.ldx + d];
            ga[ii] = o.GX[(4 * rg + ii) * o.lgx + d];
            xa[ii] = fac ? xs[ii * lds + d] : 0.f;
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            if (jj > I) continue;
            const int j = cg + 16 * jj;
            if (fac && jj < I) {
                const float b = ys[j * lds + d];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) acc[ii][jj] = fmaf(xa[ii], b, acc[ii][jj]);
            } else {
                const float b = o.Y[j * o.ldy + d], gb = o.GY[j * o.lgy + d];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
                    if (j <= 4 * rg + ii) acc[ii][jj] = fmaf(a[ii] * b, expf(ga[ii] - gb), acc[ii][jj]);
            }
        }
    }
}

// ---- GDN-2: decoupled per-channel gates ------------------------------------------
// (tiny_gdn/fugue.py BidirectionalGatedDeltaNet2: S_t = (I - k_t (b_t . k_t)^T) Diag(e^{g_t})
// S_{t-1} + k_t (w_t . v_t)^T.)  With G_t the per-key-channel cumulative log decay of the
// chunk and H (= S^T) the state at its start, the chunk's u_t solve one unit-lower system
//     u_t + sum_{s<t} A_ts u_s = w_t . v_t - H^T (e^{G_t} . b_t . k_t),
//     A_ts = sum_d b_td k_td k_sd e^{G_td - G_sd},
// so W = T (e^{G} . b . K) and U~ = T (w . V) with T = (I + A)^-1, and then
//     o_t = q_t^T (e^{G'_t} . H) + sum_{s<=t} (sum_d q_td k_sd e^{G'_td - G_sd}) (U~ - W H)_s,
//     H  <- e^{G_C} . H + sum_s (e^{G_C - G_s} . k_s) (U~ - W H)_s^T.

__global__ void __launch_bounds__(kThreads)
chunk_local_simt_g2(SimtParams p) {
    extern __shared__ float sm[];
    const WsHeader* hdr = p.hdr;
    if (hdr->err != GDR_OK) return;
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= hdr->n_chunks) return;
    const int s = p.chunk_seq[c];
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int jc = c - p.chunk_off[s];
    const int p0 = jc * p.chunk;
    const int Cc = (int)min((long long)p.chunk, (t1 - t0) - p0);
    const int dk = p.dk, dv = p.dv, ld = dk + dv + 1, C = p.chunk;
    const int hk = h / (p.Hv / p.Hk);

    const int lg = dk + 1;               // padded rows: column reads hit distinct banks
    float* R = sm;                       // [C][ld]: K | V, then W | U~ in place
    float* A = R + C * ld;               // [C][C+1]
    float* Gc = A + C * (C + 1);         // [C][dk+1] cumulative log decay per key channel
    float* Bc = Gc + C * lg;             // [C][dk+1] erase gate, then b . k^
    float* Xs = Bc + C * lg;             // [C-16][dk+1]  factored rows (g2_factor)
    float* Ys = Xs + (C - kSub) * lg;    // [ys_rows(C)][dk+1]
    const int tid = threadIdx.x;

    bool grows = false;                  // some g > 0: the factored blocks do not apply
    for (int idx = tid; idx < C * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk;
        float kv = 0.f, gv = 0.f, bv = 0.f;
        if (i < Cc) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            kv = load_elem(p.k, (size_t)(t * p.Hk + hk) * dk + d, p.io);
            gv = load_elem(p.g, (size_t)(t * p.Hv + h) * dk + d, p.gt);
            bv = load_elem(p.beta, (size_t)(t * p.Hv + h) * dk + d, p.gt);
        }
        grows |= gv > 0.f;
        R[i * ld + d] = kv;
        Gc[i * lg + d] = gv;
        Bc[i * lg + d] = bv;
    }
    for (int idx = tid; idx < Cc * dv; idx += kThreads) {
        const int i = idx / dv, d = idx % dv;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        const size_t e = (size_t)(t * p.Hv + h) * dv + d;
        R[i * ld + dk + d] = load_elem(p.v, e, p.io) * load_elem(p.w, e, p.gt);  // w . v
    }
    const bool any_grows = __syncthreads_or(grows);  // also the barrier after the loads
    const bool factor = p.g2_factor && !any_grows;
    if (p.qk_l2norm) l2norm_rows(R, Cc, dk, ld);
    for (int d = tid; d < dk; d += kThreads) {
        float run = 0.f;
        for (int i = 0; i < Cc; ++i) { run += Gc[i * lg + d]; Gc[i * lg + d] = run; }
    }
    __syncthreads();
    {   // A_ij = sum_d (b . k^)_id k^_jd e^{G_id - G_jd}, j < i (chunk <= 64)
        for (int idx = tid; idx < C * dk; idx += kThreads) {
            const int i = idx / dk, d = idx % dk;
            Bc[i * lg + d] *= R[i * ld + d];
        }
        __syncthreads();
        const PairOps ops{Bc, R, Gc, Gc, lg, ld, lg, lg};
        if (factor) {
            build_factored(Xs, Ys, lg, ops, C, dk);
            __syncthreads();
        }
        float acc[4][4] = {};
        decayed_pairs(acc, ops, Xs, Ys, lg, factor, C, dk);
        const int rg = tid >> 4, cg = tid & 15;
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int i = 4 * rg + ii, j = cg + 16 * jj;
                if (i < C && j < C) A[i * (C + 1) + j] = (j < i && i < Cc) ? acc[ii][jj] : 0.f;
            }
        __syncthreads();
        for (int idx = tid; idx < Cc * dk; idx += kThreads) {  // K rows -> e^{G} . b . k
            const int i = idx / dk, d = idx % dk;
            R[i * ld + d] = Bc[i * lg + d] * expf(Gc[i * lg + d]);
        }
    }
    __syncthreads();
    for (int col = tid; col < dk + dv; col += kThreads) {
        for (int i = 1; i < Cc; ++i) {
            float x = R[i * ld + col];
            for (int j = 0; j < i; ++j) x = fmaf(-A[i * (C + 1) + j], R[j * ld + col], x);
            R[i * ld + col] = x;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < Cc * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        p.W[(size_t)(t * p.Hv + h) * dk + d] = R[i * ld + d];
        p.G[(size_t)(t * p.Hv + h) * dk + d] = Gc[i * lg + d];
    }
    for (int idx = tid; idx < Cc * dv; idx += kThreads) {
        const int i = idx / dv, d = idx % dv;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        p.U[(size_t)(t * p.Hv + h) * dv + d] = R[i * ld + dk + d];
    }
}

__global__ void __launch_bounds__(kThreads)
chunk_scan_simt_g2(SimtParams p) {
    extern __shared__ float sm[];
    if (p.hdr->err != GDR_OK) return;
    const int s = blockIdx.x, h = blockIdx.y, J = blockIdx.z;
    const int dk = p.dk, dv = p.dv, C = p.chunk, ldk = dk + 1;
    const int hk = h / (p.Hv / p.Hk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = J * kSlice + lane;  // this lane's dv column
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);

    float* Hs = sm;                    // [dk][32]
    float* Qs = Hs + dk * kSlice;      // [C][dk+1]
    float* Ks = Qs + C * ldk;          // [C][dk+1]
    float* Ws = Ks + C * ldk;          // [C][dk+1]
    float* Us = Ws + C * ldk;          // [C][33]  U~ then V'
    float* Os = Us + C * (kSlice + 1); // [C][33]  inter-chunk read
    float* P = Os + C * (kSlice + 1);  // [C][C+1]
    float* Gc = P + C * (C + 1);       // [C][dk] cumulative log decay per key channel

    const size_t sbase = ((size_t)s * p.Hv + h) * dk * dv;
    for (int d = wid; d < dk; d += kThreads / 32)
        Hs[d * kSlice + lane] = p.S0 ? p.S0[sbase + (size_t)d * dv + col] : 0.f;

    for (int p0 = 0; p0 < L; p0 += C) {
        const int Cc = min(C, L - p0);
        __syncthreads();
        for (int idx = tid; idx < Cc * dk; idx += kThreads) {
            const int i = idx / dk, d = idx % dk;
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Qs[i * ldk + d] = load_elem(p.q, (size_t)(t * p.Hk + hk) * dk + d, p.io);
            Ks[i * ldk + d] = load_elem(p.k, (size_t)(t * p.Hk + hk) * dk + d, p.io);
            Ws[i * ldk + d] = p.W[(size_t)(t * p.Hv + h) * dk + d];
            Gc[i * dk + d] = p.G[(size_t)(t * p.Hv + h) * dk + d];
        }
        for (int i = wid; i < Cc; i += kThreads / 32) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Us[i * (kSlice + 1) + lane] = p.U[(size_t)(t * p.Hv + h) * dv + col];
        }
        __syncthreads();
        if (p.qk_l2norm) { l2norm_rows(Qs, Cc, dk, ldk); l2norm_rows(Ks, Cc, dk, ldk); }
        __syncthreads();
        // the read decay G'_i: G_i (post-write) or G_{i-1} (pre-write, 0 for the first token)
        auto gread = [&](int i, int d) -> float {
            return p.read_pre ? (i > 0 ? Gc[(i - 1) * dk + d] : 0.f) : Gc[i * dk + d];
        };
        for (int idx = tid; idx < Cc * Cc; idx += kThreads) {
            const int i = idx / Cc, j = idx % Cc;
            float val = 0.f;
            if (p.read_pre ? (j < i) : (j <= i))
                for (int d = 0; d < dk; ++d)
                    val = fmaf(Qs[i * ldk + d] * Ks[j * ldk + d], expf(gread(i, d) - Gc[j * dk + d]),
                               val);
            P[i * (C + 1) + j] = p.scale * val;
        }
        for (int i = wid; i < Cc; i += kThreads / 32) {
            float wh = 0.f, qh = 0.f;
            for (int d = 0; d < dk; ++d) {
                const float hv = Hs[d * kSlice + lane];
                wh = fmaf(Ws[i * ldk + d], hv, wh);
                qh = fmaf(Qs[i * ldk + d] * expf(gread(i, d)), hv, qh);
            }
            Us[i * (kSlice + 1) + lane] -= wh;
            Os[i * (kSlice + 1) + lane] = p.scale * qh;
        }
        __syncthreads();
        for (int i = wid; i < Cc; i += kThreads / 32) {
            float acc = Os[i * (kSlice + 1) + lane];
            const int jmax = p.read_pre ? i - 1 : i;
            for (int j = 0; j <= jmax; ++j)
                acc = fmaf(P[i * (C + 1) + j], Us[j * (kSlice + 1) + lane], acc);
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            const size_t oi = (size_t)(t * p.Hv + h) * dv + col;
            if (p.o_acc) acc += load_elem(p.o, oi, p.io);
            store_elem(p.o, oi, acc, p.io);
        }
        for (int d = wid; d < dk; d += kThreads / 32) {
            const float Gl = Gc[(Cc - 1) * dk + d];
            float acc = 0.f;
            for (int i = 0; i < Cc; ++i)
                acc = fmaf(expf(Gl - Gc[i * dk + d]) * Ks[i * ldk + d], Us[i * (kSlice + 1) + lane],
                           acc);
            Hs[d * kSlice + lane] = fmaf(expf(Gl), Hs[d * kSlice + lane], acc);
        }
    }
    __syncthreads();
    if (p.S_final)
        for (int d = wid; d < dk; d += kThreads / 32)
            p.S_final[sbase + (size_t)d * dv + col] = Hs[d * kSlice + lane];
}

// ---- register-blocked scan -----------------------------------------------------------
//
// chunk_prep_simt (one block per (chunk, value head), all chunks in parallel) forms, from the
// normalised rows and the in-chunk log decays (per token, or per key channel for GDN-2),
//     Q~_i = scale e^{G'_i} . q^_i,   K~_i = e^{G_C - G_i} . k^_i,
//     P_ij = scale sum_d q^_id k^_jd e^{G'_id - G_jd}  on the causal mask (0 elsewhere),
// so that the sequential scan is three dense fp32 products per chunk and column slice:
//     V' = U~ - W H,   O = Q~ H + P V',   H <- e^{G_C} . H + K~^T V'.
// In chunk_scan_rb lane l owns column l of the slice; warp w owns chunk rows w*RP ..
// w*RP+RP-1 (RP = C/8) and state rows w*DR .. w*DR+DR-1 (DR = dk/8), with float4 broadcast
// reads of the row operands and RP or DR independent accumulators per lane.

template <bool kG2>
__global__ void __launch_bounds__(kThreads)
chunk_prep_simt(SimtParams p) {
    extern __shared__ float sm[];
    const WsHeader* hdr = p.hdr;
    if (hdr->err != GDR_OK) return;
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= hdr->n_chunks) return;
    const int s = p.chunk_seq[c];
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int p0 = (c - p.chunk_off[s]) * p.chunk;
    const int C = p.chunk, dk = p.dk, ldk = dk + 1;
    const int Cc = (int)min((long long)C, (t1 - t0) - p0);
    const int hk = h / (p.Hv / p.Hk);
    const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
    const int lg = kG2 ? ldk : 1;       // stride of a row of G: per channel or per token

    float* Qs = sm;                     // [C][dk+1] q^
    float* Ks = Qs + C * ldk;           // [C][dk+1] k^
    float* Gs = Ks + C * ldk;           // [C][lg] G
    float* Gr = Gs + C * lg;            // [C][lg] G' (read decay)
    float* Xs = Gr + C * lg;            // GDN-2, g2_factor: [C-16][dk+1] factored rows
    float* Ys = Xs + (C - kSub) * ldk;  //                    [ys_rows(C)][dk+1]

    for (int idx = tid; idx < C * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk;
        float qv = 0.f, kv = 0.f;
        if (i < Cc) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            qv = load_elem(p.q, (size_t)(t * p.Hk + hk) * dk + d, p.io);
            kv = load_elem(p.k, (size_t)(t * p.Hk + hk) * dk + d, p.io);
        }
        Qs[i * ldk + d] = qv;
        Ks[i * ldk + d] = kv;
    }
    for (int idx = tid; idx < C * (kG2 ? dk : 1); idx += kThreads) {
        const int i = kG2 ? idx / dk : idx, d = kG2 ? idx % dk : 0;
        float gv = 0.f;
        if (i < Cc) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            gv = kG2 ? p.G[(size_t)(t * p.Hv + h) * dk + d] : p.G[(size_t)t * p.Hv + h];
        }
        Gs[i * lg + d] = gv;
    }
    __syncthreads();
    if (p.qk_l2norm) { l2norm_rows(Qs, Cc, dk, ldk); l2norm_rows(Ks, Cc, dk, ldk); }
    for (int idx = tid; idx < C * (kG2 ? dk : 1); idx += kThreads) {
        const int i = kG2 ? idx / dk : idx, d = kG2 ? idx % dk : 0;
        Gr[i * lg + d] = p.read_pre ? (i > 0 ? Gs[(i - 1) * lg + d] : 0.f) : Gs[i * lg + d];
    }
    __syncthreads();
    for (int idx = tid; idx < Cc * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk, e = kG2 ? d : 0;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        const size_t o = (size_t)(t * p.Hv + h) * dk + d;
        p.Qt[o] = p.scale * expf(Gr[i * lg + e]) * Qs[i * ldk + d];
        p.Kt[o] = expf(Gs[(Cc - 1) * lg + e] - Gs[i * lg + e]) * Ks[i * ldk + d];
    }
    // P over this thread's rows 4 rg + ii and columns cg + 16 jj (C <= 64)
    float acc[4][4] = {};
    if constexpr (kG2) {  // the decay differs per channel (decayed_pairs)
        bool grows = false;  // the decay grows somewhere (some g > 0): no factored blocks
        for (int idx = tid; idx < Cc * dk; idx += kThreads) {
            const int i = idx / dk, d = idx % dk;
            grows |= Gs[i * lg + d] > (i > 0 ? Gs[(i - 1) * lg + d] : 0.f);
        }
        const bool any_grows = __syncthreads_or(grows);
        const bool factor = p.g2_factor && !any_grows;
        const PairOps ops{Qs, Ks, Gr, Gs, ldk, ldk, lg, lg};
        if (factor) {
            build_factored(Xs, Ys, ldk, ops, C, dk);
            __syncthreads();
        }
        decayed_pairs(acc, ops, Xs, Ys, ldk, factor, C, dk);
    } else {
        for (int d = 0; d < dk; ++d) {
            float a[4], b[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = 4 * rg + ii < C ? Qs[(4 * rg + ii) * ldk + d] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = cg + 16 * jj < C ? Ks[(cg + 16 * jj) * ldk + d] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[ii][jj] = fmaf(a[ii], b[jj], acc[ii][jj]);
        }
    }
    float* Pout = p.Pc + ((size_t)c * p.Hv + h) * C * C;
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int i = 4 * rg + ii, j = cg + 16 * jj;
            if (i >= C || j >= C) continue;
            const bool m = i < Cc && j < Cc && (p.read_pre ? j < i : j <= i);
            float v = 0.f;
            if (m) v = kG2 ? p.scale * acc[ii][jj] : p.scale * acc[ii][jj] * expf(Gr[i] - Gs[j]);
            Pout[i * C + j] = v;
        }
}

// Rows [0, rows) of a token-major fp32 array [T][Hv][n] into shared rows of stride n.
__device__ __forceinline__ void load_rows4(float* dst, const float* src, int rows, int n,
                                           const SimtParams& p, long long t0, long long t1,
                                           int p0, int h) {
    const int n4 = n / 4;
    // read-only global loads: they may all be issued before the shared stores
#pragma unroll 4
    for (int idx = threadIdx.x; idx < rows * n4; idx += kThreads) {
        const int i = idx / n4, d4 = idx % n4;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        reinterpret_cast<float4*>(dst + (size_t)i * n)[d4] =
            __ldg(reinterpret_cast<const float4*>(src + ((size_t)t * p.Hv + h) * n) + d4);
    }
}

template <int RP, int DR, bool kG2>
__global__ void __launch_bounds__(kThreads)
chunk_scan_rb(SimtParams p) {
    extern __shared__ __align__(16) float smr[];
    if (p.hdr->err != GDR_OK) return;
    const int s = blockIdx.x, h = blockIdx.y, J = blockIdx.z;
    const int dk = p.dk, dv = p.dv, C = p.chunk;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = J * kSlice + lane;
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);

    float* Hs = smr;                    // [dk][32] state slice
    float* Kt = Hs + dk * kSlice;       // [C][dk] K~
    float* Qt = Kt + C * dk;            // [C][dk] Q~
    float* Ws = Qt + C * dk;            // [C][dk] W
    float* Ps = Ws + C * dk;            // [C][C]  P
    float* Us = Ps + C * C;             // [C][33] U~ then V'

    const size_t sbase = ((size_t)s * p.Hv + h) * dk * dv;
    for (int d = wid; d < dk; d += kThreads / 32)
        Hs[d * kSlice + lane] = p.S0 ? p.S0[sbase + (size_t)d * dv + col] : 0.f;

    for (int p0 = 0, jc = 0; p0 < L; p0 += C, ++jc) {
        const int Cc = min(C, L - p0);
        const int c = p.chunk_off[s] + jc;
        __syncthreads();
        load_rows4(Kt, p.Kt, Cc, dk, p, t0, t1, p0, h);
        load_rows4(Qt, p.Qt, Cc, dk, p, t0, t1, p0, h);
        load_rows4(Ws, p.W, Cc, dk, p, t0, t1, p0, h);
        {
            const float4* src = reinterpret_cast<const float4*>(p.Pc + ((size_t)c * p.Hv + h) * C * C);
#pragma unroll 4
            for (int idx = tid; idx < C * C / 4; idx += kThreads)
                reinterpret_cast<float4*>(Ps)[idx] = __ldg(src + idx);
        }
        for (int i = wid; i < Cc; i += kThreads / 32) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Us[i * (kSlice + 1) + lane] = p.U[(size_t)(t * p.Hv + h) * dv + col];
        }
        // the carry's decay of this warp's state rows: e^{G_C} (per channel for GDN-2)
        float dc[DR];
        {
            const long long tl = phys_token(t0, t1, p0 + Cc - 1, p.reverse);
#pragma unroll
            for (int r = 0; r < DR; ++r)
                dc[r] = expf(kG2 ? p.G[(size_t)(tl * p.Hv + h) * dk + wid * DR + r]
                                 : p.G[(size_t)tl * p.Hv + h]);
        }
        __syncthreads();
        // V' = U~ - W H
        {
            float acc[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) acc[r] = 0.f;
            for (int d = 0; d < dk; d += 4) {
                const float h0 = Hs[(d + 0) * kSlice + lane], h1 = Hs[(d + 1) * kSlice + lane];
                const float h2 = Hs[(d + 2) * kSlice + lane], h3 = Hs[(d + 3) * kSlice + lane];
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const float4 w4 = *reinterpret_cast<const float4*>(Ws + (wid * RP + r) * dk + d);
                    acc[r] = fmaf(w4.x, h0, fmaf(w4.y, h1, fmaf(w4.z, h2, fmaf(w4.w, h3, acc[r]))));
                }
            }
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int i = wid * RP + r;
                if (i < Cc) Us[i * (kSlice + 1) + lane] -= acc[r];
            }
        }
        __syncthreads();
        // O = Q~ H + P V' and the new state, both from the old H
        float hacc[DR];
        {
            float acc[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) acc[r] = 0.f;
            for (int d = 0; d < dk; d += 4) {
                const float h0 = Hs[(d + 0) * kSlice + lane], h1 = Hs[(d + 1) * kSlice + lane];
                const float h2 = Hs[(d + 2) * kSlice + lane], h3 = Hs[(d + 3) * kSlice + lane];
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const float4 q4 = *reinterpret_cast<const float4*>(Qt + (wid * RP + r) * dk + d);
                    acc[r] = fmaf(q4.x, h0, fmaf(q4.y, h1, fmaf(q4.z, h2, fmaf(q4.w, h3, acc[r]))));
                }
            }
            for (int j = 0; j < Cc; ++j) {
                const float a = Us[j * (kSlice + 1) + lane];
#pragma unroll
                for (int r = 0; r < RP; ++r) acc[r] = fmaf(Ps[(wid * RP + r) * C + j], a, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int i = wid * RP + r;
                if (i < Cc) {
                    const long long t = phys_token(t0, t1, p0 + i, p.reverse);
                    const size_t oi = (size_t)(t * p.Hv + h) * dv + col;
                    float o = acc[r];
                    if (p.o_acc) o += load_elem(p.o, oi, p.io);
                    store_elem(p.o, oi, o, p.io);
                }
            }
#pragma unroll
            for (int r = 0; r < DR; ++r) hacc[r] = dc[r] * Hs[(wid * DR + r) * kSlice + lane];
            for (int i = 0; i < Cc; ++i) {
                const float v = Us[i * (kSlice + 1) + lane];
#pragma unroll
                for (int r = 0; r < DR; r += 4) {
                    const float4 k4 = *reinterpret_cast<const float4*>(Kt + i * dk + wid * DR + r);
                    hacc[r] = fmaf(k4.x, v, hacc[r]);
                    hacc[r + 1] = fmaf(k4.y, v, hacc[r + 1]);
                    hacc[r + 2] = fmaf(k4.z, v, hacc[r + 2]);
                    hacc[r + 3] = fmaf(k4.w, v, hacc[r + 3]);
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < DR; ++r) Hs[(wid * DR + r) * kSlice + lane] = hacc[r];
    }
    __syncthreads();
    if (p.S_final)
        for (int d = wid; d < dk; d += kThreads / 32)
            p.S_final[sbase + (size_t)d * dv + col] = Hs[d * kSlice + lane];
}

constexpr size_t kMaxSmem = 227 * 1024;

// GDN-2's factored blocks: rows of the Xs and Ys buffers, for 32 <= chunk <= 64
size_t g2_factor_rows(const gdr_chunk_args& a) {
    return (a.gdn2 && a.chunk >= 32 && a.chunk <= 64) ? (size_t)(a.chunk - kSub + ys_rows(a.chunk)) : 0;
}

size_t prep_smem_base(const gdr_chunk_args& a) {
    const size_t C = a.chunk, ldk = a.dk + 1;
    return sizeof(float) * (2 * C * ldk + 2 * C * (a.gdn2 ? ldk : 1));
}

size_t local_smem_base(const gdr_chunk_args& a) {
    const int C = a.chunk;
    return sizeof(float) * ((size_t)C * (a.dk + a.dv + 1) + (size_t)C * (C + 1) +
                            (a.gdn2 ? 2 * (size_t)C * (a.dk + 1) : 2 * (size_t)C));
}

// whether the factored blocks' buffers fit next to both kernels' own
bool g2_factor(const gdr_chunk_args& a) {
    const size_t extra = sizeof(float) * g2_factor_rows(a) * (a.dk + 1);
    return extra > 0 && local_smem_base(a) + extra <= kMaxSmem &&
           (!simt_rb(a) || prep_smem_base(a) + extra <= kMaxSmem);
}

size_t g2_extra(const gdr_chunk_args& a) {
    return g2_factor(a) ? sizeof(float) * g2_factor_rows(a) * (a.dk + 1) : 0;
}

size_t prep_smem(const gdr_chunk_args& a) { return prep_smem_base(a) + g2_extra(a); }

size_t scan_rb_smem(const gdr_chunk_args& a) {
    const size_t C = a.chunk;
    return sizeof(float) * ((size_t)a.dk * kSlice + 3 * C * a.dk + C * C + C * (kSlice + 1));
}

template <int RP, int DR>
gdr_status launch_scan_rb_t(const gdr_chunk_args& a, const SimtParams& p, cudaStream_t st) {
    auto kern = a.gdn2 ? chunk_scan_rb<RP, DR, true> : chunk_scan_rb<RP, DR, false>;
    const size_t smem = scan_rb_smem(a);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return GDR_ERR_CUDA;
    kern<<<dim3((unsigned)a.n_seqs, (unsigned)a.Hv, (unsigned)(a.dv / kSlice)), kThreads, smem,
           st>>>(p);
    return GDR_OK;
}

template <int RP>
gdr_status launch_scan_rb_dk(const gdr_chunk_args& a, const SimtParams& p, cudaStream_t st) {
    switch (a.dk) {
        case 32: return launch_scan_rb_t<RP, 4>(a, p, st);
        case 64: return launch_scan_rb_t<RP, 8>(a, p, st);
        case 96: return launch_scan_rb_t<RP, 12>(a, p, st);
        case 128: return launch_scan_rb_t<RP, 16>(a, p, st);
    }
    return GDR_ERR_UNSUPPORTED;
}

gdr_status launch_scan_rb(const gdr_chunk_args& a, const SimtParams& p, cudaStream_t st) {
    switch (a.chunk) {
        case 16: return launch_scan_rb_dk<2>(a, p, st);
        case 32: return launch_scan_rb_dk<4>(a, p, st);
        case 64: return launch_scan_rb_dk<8>(a, p, st);
    }
    return GDR_ERR_UNSUPPORTED;
}

gdr_status launch_prep(const gdr_chunk_args& a, const SimtParams& p, const WsLayout& L,
                       cudaStream_t st) {
    if (L.max_chunks == 0) return GDR_OK;
    auto kern = a.gdn2 ? chunk_prep_simt<true> : chunk_prep_simt<false>;
    const size_t smem = prep_smem(a);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return GDR_ERR_CUDA;
    kern<<<dim3((unsigned)L.max_chunks, (unsigned)a.Hv), kThreads, smem, st>>>(p);
    return GDR_OK;
}

size_t local_smem(const gdr_chunk_args& a) { return local_smem_base(a) + g2_extra(a); }

size_t scan_smem(const gdr_chunk_args& a) {
    const int C = a.chunk, ldk = a.dk + 1;
    return sizeof(float) * ((size_t)a.dk * kSlice + 3 * (size_t)C * ldk +
                            2 * (size_t)C * (kSlice + 1) + (size_t)C * (C + 1) +
                            (a.gdn2 ? (size_t)C * a.dk : 3 * (size_t)C));
}

}  // namespace

bool simt_supported(const gdr_chunk_args& a) {
    if (a.dv % kSlice != 0 || a.dk < 1 || a.dk > 256 || a.dv > 256) return false;
    if (a.gdn2 && a.chunk > 64) return false;  // the GDN-2 local kernel tiles 64 rows
    if (simt_rb(a) && (prep_smem(a) > kMaxSmem || scan_rb_smem(a) > kMaxSmem)) return false;
    return local_smem(a) <= kMaxSmem && scan_smem(a) <= kMaxSmem;
}

gdr_status launch_chunk_simt(const gdr_chunk_args& a, const void* q, const void* k,
                             const void* v, const void* g, const void* beta, const float* S0,
                             void* o, float* S_final, void* ws, const WsLayout& L,
                             cudaStream_t st) {
    char* base = static_cast<char*>(ws);
    SimtParams p;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.S0 = S0; p.o = o; p.S_final = S_final;
    p.hdr = reinterpret_cast<const WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.chunk_off = reinterpret_cast<const int32_t*>(base + L.chunk_off);
    p.chunk_seq = reinterpret_cast<const int32_t*>(base + L.chunk_seq);
    p.W = reinterpret_cast<float*>(base + L.W);
    p.U = reinterpret_cast<float*>(base + L.U);
    p.G = reinterpret_cast<float*>(base + L.G);
    p.Hk = a.Hk; p.Hv = a.Hv; p.dk = a.dk; p.dv = a.dv; p.chunk = a.chunk;
    p.read_pre = a.read_mode == GDR_READ_PRE; p.qk_l2norm = a.qk_l2norm; p.reverse = a.reverse;
    p.o_acc = a.o_accumulate; p.io = a.io_dtype; p.gt = a.gate_dtype; p.scale = a.scale;
    p.gate_raw = a.gate_raw; p.gate_A = a.gate_A; p.gate_dt_bias = a.gate_dt_bias;
    p.beta_scale = a.beta_scale;
    p.w = a.gdn2_w;
    p.g2_factor = g2_factor(a);
    const bool rb = simt_rb(a);
    if (rb) {
        p.Qt = reinterpret_cast<float*>(base + L.Qt);
        p.Kt = reinterpret_cast<float*>(base + L.Kt);
        p.Pc = reinterpret_cast<float*>(base + L.Pc);
    }

    auto local = a.gdn2 ? chunk_local_simt_g2 : chunk_local_simt;
    auto scan = a.gdn2 ? chunk_scan_simt_g2 : chunk_scan_simt;
    const size_t sm1 = local_smem(a), sm2 = scan_smem(a);
    if ((cudaFuncSetAttribute(local, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm1)) != cudaSuccess) return GDR_ERR_CUDA;
    if ((cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm2)) != cudaSuccess) return GDR_ERR_CUDA;
    if (L.max_chunks > 0) {
        dim3 g1((unsigned)L.max_chunks, (unsigned)a.Hv);
        local<<<g1, kThreads, sm1, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    }
    if (rb) {
        gdr_status s = launch_prep(a, p, L, st);
        if (s == GDR_OK) s = launch_scan_rb(a, p, st);
        if (s != GDR_OK) return s;
        return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
    }
    dim3 g2((unsigned)a.n_seqs, (unsigned)a.Hv, (unsigned)(a.dv / kSlice));
    scan<<<g2, kThreads, sm2, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    return GDR_OK;
}

gdr_status launch_prep_simt(const gdr_chunk_args& a, const void* q, const void* k, void* ws,
                            const WsLayout& L, cudaStream_t st) {
    if (a.gdn2 || !simt_rb(a)) return GDR_ERR_UNSUPPORTED;
    char* base = static_cast<char*>(ws);
    SimtParams p{};
    p.q = q; p.k = k;
    p.hdr = reinterpret_cast<const WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.chunk_off = reinterpret_cast<const int32_t*>(base + L.chunk_off);
    p.chunk_seq = reinterpret_cast<const int32_t*>(base + L.chunk_seq);
    p.G = reinterpret_cast<float*>(base + L.G);
    p.Qt = reinterpret_cast<float*>(base + L.Qt);
    p.Kt = reinterpret_cast<float*>(base + L.Kt);
    p.Pc = reinterpret_cast<float*>(base + L.Pc);
    p.Hk = a.Hk; p.Hv = a.Hv; p.dk = a.dk; p.dv = a.dv; p.chunk = a.chunk;
    p.read_pre = a.read_mode == GDR_READ_PRE; p.qk_l2norm = a.qk_l2norm; p.reverse = a.reverse;
    p.io = a.io_dtype; p.gt = a.gate_dtype; p.scale = a.scale;
    const gdr_status s = launch_prep(a, p, L, st);
    if (s != GDR_OK) return s;
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status launch_wy_local_simt(const gdr_chunk_args& a, const void* k, const void* v,
                                const void* g, const void* beta, void* ws, const WsLayout& L,
                                float* W, float* U, float* G, cudaStream_t st) {
    if (a.gdn2 || L.max_chunks == 0) return a.gdn2 ? GDR_ERR_UNSUPPORTED : GDR_OK;
    char* base = static_cast<char*>(ws);
    SimtParams p{};
    p.k = k; p.v = v; p.g = g; p.beta = beta;
    p.hdr = reinterpret_cast<const WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.chunk_off = reinterpret_cast<const int32_t*>(base + L.chunk_off);
    p.chunk_seq = reinterpret_cast<const int32_t*>(base + L.chunk_seq);
    p.W = W; p.U = U; p.G = G;
    p.Hk = a.Hk; p.Hv = a.Hv; p.dk = a.dk; p.dv = a.dv; p.chunk = a.chunk;
    p.qk_l2norm = a.qk_l2norm; p.reverse = a.reverse;
    p.io = a.io_dtype; p.gt = a.gate_dtype;
    p.gate_raw = a.gate_raw; p.gate_A = a.gate_A; p.gate_dt_bias = a.gate_dt_bias;
    p.beta_scale = a.beta_scale;
    const size_t sm1 = local_smem(a);
    if (cudaFuncSetAttribute(chunk_local_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm1) != cudaSuccess) return GDR_ERR_CUDA;
    chunk_local_simt<<<dim3((unsigned)L.max_chunks, (unsigned)a.Hv), kThreads, sm1, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
