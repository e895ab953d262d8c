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

    float* R = sm;                       // [C][ld]: K | V, then W | U~ in place
    float* A = R + C * ld;               // [C][C+1]
    float* Gc = A + C * (C + 1);         // [C][dk] cumulative log decay per key channel
    float* Bc = Gc + C * dk;             // [C][dk] erase gate
    const int tid = threadIdx.x;

    for (int idx = tid; idx < Cc * dk; idx += kThreads) {
        const int i = idx / dk, d = idx % dk;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        R[i * ld + d] = load_elem(p.k, (size_t)(t * p.Hk + hk) * dk + d, p.io);
        Gc[i * dk + d] = load_elem(p.g, (size_t)(t * p.Hv + h) * dk + d, p.gt);
        Bc[i * dk + d] = load_elem(p.beta, (size_t)(t * p.Hv + h) * dk + d, p.gt);
    }
    for (int idx = tid; idx < Cc * dv; idx += kThreads) {
        const int i = idx / dv, d = idx % dv;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        const size_t e = (size_t)(t * p.Hv + h) * dv + d;
        R[i * ld + dk + d] = load_elem(p.v, e, p.io) * load_elem(p.w, e, p.gt);  // w . v
    }
    __syncthreads();
    if (p.qk_l2norm) l2norm_rows(R, Cc, dk, ld);
    for (int d = tid; d < dk; d += kThreads) {
        float run = 0.f;
        for (int i = 0; i < Cc; ++i) { run += Gc[i * dk + d]; Gc[i * dk + d] = run; }
    }
    __syncthreads();
    for (int idx = tid; idx < Cc * Cc; idx += kThreads) {
        const int i = idx / Cc, j = idx % Cc;
        float val = 0.f;
        if (j < i)
            for (int d = 0; d < dk; ++d)
                val = fmaf(Bc[i * dk + d] * R[i * ld + d] * R[j * ld + d],
                           expf(Gc[i * dk + d] - Gc[j * dk + d]), val);
        A[i * (C + 1) + j] = val;
    }
    __syncthreads();
    for (int idx = tid; idx < Cc * dk; idx += kThreads) {  // K rows -> e^{G} . b . k
        const int i = idx / dk, d = idx % dk;
        R[i * ld + d] *= Bc[i * dk + d] * expf(Gc[i * dk + d]);
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
        p.G[(size_t)(t * p.Hv + h) * dk + d] = Gc[i * dk + d];
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

size_t local_smem(const gdr_chunk_args& a) {
    const int C = a.chunk;
    return sizeof(float) * ((size_t)C * (a.dk + a.dv + 1) + (size_t)C * (C + 1) +
                            (a.gdn2 ? 2 * (size_t)C * a.dk : 2 * (size_t)C));
}

size_t scan_smem(const gdr_chunk_args& a) {
    const int C = a.chunk, ldk = a.dk + 1;
    return sizeof(float) * ((size_t)a.dk * kSlice + 3 * (size_t)C * ldk +
                            2 * (size_t)C * (kSlice + 1) + (size_t)C * (C + 1) +
                            (a.gdn2 ? (size_t)C * a.dk : 3 * (size_t)C));
}

constexpr size_t kMaxSmem = 227 * 1024;

}  // namespace

bool simt_supported(const gdr_chunk_args& a) {
    if (a.dv % kSlice != 0 || a.dk < 1 || a.dk > 256 || a.dv > 256) return false;
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
    dim3 g2((unsigned)a.n_seqs, (unsigned)a.Hv, (unsigned)(a.dv / kSlice));
    scan<<<g2, kThreads, sm2, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    return GDR_OK;
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
