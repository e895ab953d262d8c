// chunk_bwd.cu -- backward pass of the chunk-wise WY/UT forward, fp32 on CUDA cores.
//
// The gradient is the one of the per-token recurrence (Prizma "seq/delta.py", module
// docstring: the chunk-parallel form agrees with the per-token recurrence on the forward
// and on the gradients), taken here through the chunk form of the forward.  Per (sequence,
// v-head) and chunk, with normalised rows Q^, K^, in-chunk log decay G (G' = G for the
// post-write read, G shifted by one token for the pre-write read), state H at the chunk's
// start and s = scale:
//     A  = strict_lower(diag(beta) (K^ K^T) . e^{G_i - G_j}),   T = (I + A)^-1
//     W  = T diag(beta e^G) K^,   U~ = T diag(beta) V,   V' = U~ - W H
//     O  = s (diag(e^{G'}) Q^ H + P V'),  P_ij = (q^_i . k^_j) e^{G'_i - G_j} (causal mask)
//     H+ = e^{G_C} H + (diag(e^{G_C - G}) K^)^T V'
// Given dO and dH+ (the gradient of the next chunk's starting state), the adjoint is
//     dV' = s P^T dO + diag(e^{G_C - G}) K^ dH+
//     dH  = e^{G_C} dH+ + s (diag(e^{G'}) Q^)^T dO - W^T dV'          (sequential over chunks)
//     dQ^ = s diag(e^{G'}) dO H^T + (dP . M) K^,   dP_ij = s (dO_i . V'_j) e^{G'_i - G_j}
//     dK^ = (dP . M)^T Q^ + diag(e^{G_C - G}) V' dH+^T + [A and W terms]
//     dW  = -dV' H^T,   [dR_w | dR_u] = T^T [dW | dV']   (a unit-upper solve)
//     dA  = -(dR_w W^T + dR_u U~^T) on the strict lower triangle
//     dV  = diag(beta) dR_u,   dbeta, dG from every factor that carries them,
//     dg  = reverse cumulative sum of dG within the chunk,
// and the L2 normalisation's adjoint (dx^ - x^ (x^ . dx^)) / |x| maps dQ^, dK^ to dq, dk,
// summed over the v-heads that share a key head.
//
// Kernels, in order on the stream:
//   plan_kernel            chunk map (shared with the forward)
//   chunk_local_simt       W, U~, G per chunk (shared with the forward's CUDA-core path)
//   chunk_prep_simt        per (chunk, head): s e^{G'} q^, e^{G_C - G} k^ and P (shared too)
//   bwd_states_fwd         per (sequence, head, 32-column slice): H at every chunk start, V'
//   bwd_states_bwd         same grid, chunks in reverse: dH+ at every chunk, dV', dS0
//   bwd_chunk_dqk          per (chunk, head): dq (normalised adjoint), the P and carry parts
//                          of dK^ and dG, dW
//   bwd_chunk_wy           per (chunk, head): the transposed solve, dA, dbeta, dv, dg, dk
//   bwd_reduce_heads4      dq, dk summed over each key head's v-heads
#include <algorithm>

#include "chunk_bwd.cuh"
#include "chunk_tc.cuh"

namespace gdr {

namespace {

constexpr int kThreads = 256;  // state passes and the head reduction
constexpr int kNT = 512;       // per-(chunk, head) kernels: 16 warps over 64 rows
constexpr int kSlice = 32;     // dv columns per state-pass block (one per lane)



// Normalise `rows` rows of length n (stride ld) in shared memory, one warp per row, and
// record each row's norm |x| (needed by the adjoint).
__device__ void l2norm_rows_keep(float* x, float* norms, int rows, int n, int ld, bool on) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int i = wid; i < rows; i += kNT / 32) {
        float ss = 0.f;
        for (int d = lane; d < n; d += 32) ss += x[i * ld + d] * x[i * ld + d];
        ss = warp_sum(ss);
        const float nrm = sqrtf(ss);
        if (lane == 0) norms[i] = nrm;
        if (on) {
            const float inv = 1.f / fmaxf(nrm, kNormEps);
            for (int d = lane; d < n; d += 32) x[i * ld + d] *= inv;
        }
    }
}

// Adjoint of x^ = x / max(|x|, eps) for one element, with proj = x^ . dx^ over the row.
__device__ __forceinline__ float norm_adjoint(float dxh, float xh, float proj, float nrm,
                                              bool on) {
    if (!on) return dxh;
    return nrm > kNormEps ? (dxh - xh * proj) / nrm : dxh / kNormEps;
}

// Register tiles of the per-chunk kernels (kNT threads): thread (rg = warp, cg = lane) owns
// rows i = 4 rg + ii (ii < 4) and columns c = cg + 32 jj (jj < 2 for a [C x C] product,
// jj < 4 for [C x dk]), so a warp reads 32 consecutive columns of a row (no bank
// conflicts), shares its rows (broadcast) and reduces a row with warp shuffles.
struct Tile {
    int rg, cg;
    __device__ Tile() : rg(threadIdx.x >> 5), cg(threadIdx.x & 31) {}
    __device__ int row(int ii) const { return 4 * rg + ii; }
    __device__ int col(int jj) const { return cg + 32 * jj; }
};


// ---- state passes: one block per (sequence, v-head, 32-column slice of dv) ---------------
//
// Lane l of every warp owns column l of the slice.  Warp w owns rows w*RP .. w*RP+RP-1 of
// the chunk's [C x 32] products (RP = C/8) and rows w*DR .. w*DR+DR-1 of the [dk x 32]
// state (DR = dk/8), so each lane keeps RP or DR independent accumulators and reads the
// row operands as float4 broadcasts.  K~ = e^{G_C - G} k^, Q~ = s e^{G'} q^ and P come from
// chunk_prep_simt, so the passes hold no normalisation or exponential.

__device__ __forceinline__ void load_rows4(float* dst, const float* src, size_t row_stride,
                                           int rows, int n, const BwdParams& p, long long t0,
                                           long long t1, int p0, int h) {
    const int n4 = n / 4;
    // read-only global loads: they may all be issued before the shared stores
#pragma unroll 4
    for (int idx = threadIdx.x; idx < rows * n4; idx += kThreads) {
        const int i = idx / n4, d4 = idx % n4;
        const long long t = phys_token(t0, t1, p0 + i, p.reverse);
        reinterpret_cast<float4*>(dst + (size_t)i * n)[d4] =
            __ldg(reinterpret_cast<const float4*>(src + ((size_t)t * p.Hv + h) * row_stride) + d4);
    }
}

template <int RP, int DR>
__global__ void __launch_bounds__(kThreads)
bwd_states_fwd(BwdParams p) {
    extern __shared__ __align__(16) float sm[];
    if (p.hdr->err != GDR_OK) return;
    const int s = blockIdx.x, h = blockIdx.y, J = blockIdx.z;
    const int dk = p.dk, dv = p.dv, C = p.chunk;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = J * kSlice + lane;
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);

    float* Hs = sm;                     // [dk][32]
    float* Kt = Hs + dk * kSlice;       // [C][dk] K~
    float* Ws = Kt + C * dk;            // [C][dk] W
    float* Us = Ws + C * dk;            // [C][33] U~ then V'

    const size_t sbase = ((size_t)s * p.Hv + h) * dk * dv;
    for (int d = wid; d < dk; d += kThreads / 32)
        Hs[d * kSlice + lane] = p.S0 ? p.S0[sbase + (size_t)d * dv + col] : 0.f;

    for (int p0 = 0, jc = 0; p0 < L; p0 += C, ++jc) {
        const int Cc = min(C, L - p0);
        const size_t cbase = ((size_t)(p.chunk_off[s] + jc) * p.Hv + h) * dk * dv;
        __syncthreads();
        for (int d = wid; d < dk; d += kThreads / 32)
            p.Hc[cbase + (size_t)d * dv + col] = Hs[d * kSlice + lane];
        load_rows4(Kt, p.Kt, dk, Cc, dk, p, t0, t1, p0, h);
        load_rows4(Ws, p.W, dk, Cc, dk, p, t0, t1, p0, h);
        for (int i = wid; i < Cc; i += kThreads / 32) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            Us[i * (kSlice + 1) + lane] = p.U[(size_t)(t * p.Hv + h) * dv + col];
        }
        const float gC = expf(p.G[(size_t)phys_token(t0, t1, p0 + Cc - 1, p.reverse) * p.Hv + h]);
        __syncthreads();
        // V' = U~ - W H, rows wid*RP + r
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
                if (i < Cc) {
                    const float vp = Us[i * (kSlice + 1) + lane] - acc[r];
                    Us[i * (kSlice + 1) + lane] = vp;
                    const long long t = phys_token(t0, t1, p0 + i, p.reverse);
                    p.Vp[(size_t)(t * p.Hv + h) * dv + col] = vp;
                }
            }
        }
        __syncthreads();
        // H <- e^{G_C} H + K~^T V', rows wid*DR + dr
        {
            float acc[DR];
#pragma unroll
            for (int r = 0; r < DR; ++r) acc[r] = gC * Hs[(wid * DR + r) * kSlice + lane];
            for (int i = 0; i < Cc; ++i) {
                const float v = Us[i * (kSlice + 1) + lane];
#pragma unroll
                for (int r = 0; r < DR; r += 4) {
                    const float4 k4 = *reinterpret_cast<const float4*>(Kt + i * dk + wid * DR + r);
                    acc[r] = fmaf(k4.x, v, acc[r]);
                    acc[r + 1] = fmaf(k4.y, v, acc[r + 1]);
                    acc[r + 2] = fmaf(k4.z, v, acc[r + 2]);
                    acc[r + 3] = fmaf(k4.w, v, acc[r + 3]);
                }
            }
#pragma unroll
            for (int r = 0; r < DR; ++r) Hs[(wid * DR + r) * kSlice + lane] = acc[r];
        }
    }
}

template <int RP, int DR>
__global__ void __launch_bounds__(kThreads)
bwd_states_bwd(BwdParams p) {
    extern __shared__ __align__(16) float sm[];
    if (p.hdr->err != GDR_OK) return;
    const int s = blockIdx.x, h = blockIdx.y, J = blockIdx.z;
    const int dk = p.dk, dv = p.dv, C = p.chunk;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = J * kSlice + lane;
    const long long t0 = p.cu[s], t1 = p.cu[s + 1];
    const int L = (int)(t1 - t0);
    const int nC = (L + C - 1) / C;

    float* dHs = sm;                    // [dk][32]
    float* Kt = dHs + dk * kSlice;      // [C][dk] K~
    float* Qt = Kt + C * dk;            // [C][dk] Q~
    float* Ws = Qt + C * dk;            // [C][dk] W
    float* Ps = Ws + C * dk;            // [C][C]  P (scaled, decayed, masked)
    float* dOs = Ps + C * C;            // [C][33]
    float* dVs = dOs + C * (kSlice + 1);// [C][33]

    const size_t sbase = ((size_t)s * p.Hv + h) * dk * dv;
    for (int d = wid; d < dk; d += kThreads / 32)
        dHs[d * kSlice + lane] = p.dS_final ? p.dS_final[sbase + (size_t)d * dv + col] : 0.f;

    for (int jc = nC - 1; jc >= 0; --jc) {
        const int p0 = jc * C, Cc = min(C, L - p0);
        const int c = p.chunk_off[s] + jc;
        const size_t cbase = ((size_t)c * p.Hv + h) * dk * dv;
        __syncthreads();
        for (int d = wid; d < dk; d += kThreads / 32)
            p.dHc[cbase + (size_t)d * dv + col] = dHs[d * kSlice + lane];
        load_rows4(Kt, p.Kt, dk, Cc, dk, p, t0, t1, p0, h);
        load_rows4(Qt, p.Qt, dk, Cc, dk, p, t0, t1, p0, h);
        load_rows4(Ws, p.W, dk, Cc, dk, p, t0, t1, p0, h);
        {
            const float4* src = reinterpret_cast<const float4*>(p.Pc + ((size_t)c * p.Hv + h) * C * C);
#pragma unroll 4
            for (int idx = tid; idx < C * C / 4; idx += kThreads)
                reinterpret_cast<float4*>(Ps)[idx] = __ldg(src + idx);
        }
        for (int i = wid; i < Cc; i += kThreads / 32) {
            const long long t = phys_token(t0, t1, p0 + i, p.reverse);
            dOs[i * (kSlice + 1) + lane] = load_elem(p.dO, (size_t)(t * p.Hv + h) * dv + col, p.io);
        }
        const float gC = expf(p.G[(size_t)phys_token(t0, t1, p0 + Cc - 1, p.reverse) * p.Hv + h]);
        __syncthreads();
        // dV'_j = sum_i P_ij dO_i + K~_j . dH+, rows j = wid*RP + r
        {
            float acc[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) acc[r] = 0.f;
            for (int i = 0; i < Cc; ++i) {
                const float a = dOs[i * (kSlice + 1) + lane];
#pragma unroll
                for (int r = 0; r < RP; ++r) acc[r] = fmaf(Ps[i * C + wid * RP + r], a, acc[r]);
            }
            for (int d = 0; d < dk; d += 4) {
                const float h0 = dHs[(d + 0) * kSlice + lane], h1 = dHs[(d + 1) * kSlice + lane];
                const float h2 = dHs[(d + 2) * kSlice + lane], h3 = dHs[(d + 3) * kSlice + lane];
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const float4 k4 = *reinterpret_cast<const float4*>(Kt + (wid * RP + r) * dk + d);
                    acc[r] = fmaf(k4.x, h0, fmaf(k4.y, h1, fmaf(k4.z, h2, fmaf(k4.w, h3, acc[r]))));
                }
            }
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int j = wid * RP + r;
                if (j < Cc) {
                    dVs[j * (kSlice + 1) + lane] = acc[r];
                    const long long t = phys_token(t0, t1, p0 + j, p.reverse);
                    p.dVp[(size_t)(t * p.Hv + h) * dv + col] = acc[r];
                }
            }
        }
        __syncthreads();
        // dH = e^{G_C} dH+ + Q~^T dO - W^T dV', rows wid*DR + dr
        {
            float acc[DR];
#pragma unroll
            for (int r = 0; r < DR; ++r) acc[r] = gC * dHs[(wid * DR + r) * kSlice + lane];
            for (int i = 0; i < Cc; ++i) {
                const float a = dOs[i * (kSlice + 1) + lane], b = dVs[i * (kSlice + 1) + lane];
#pragma unroll
                for (int r = 0; r < DR; r += 4) {
                    const float4 q4 = *reinterpret_cast<const float4*>(Qt + i * dk + wid * DR + r);
                    const float4 w4 = *reinterpret_cast<const float4*>(Ws + i * dk + wid * DR + r);
                    acc[r] = fmaf(q4.x, a, fmaf(-w4.x, b, acc[r]));
                    acc[r + 1] = fmaf(q4.y, a, fmaf(-w4.y, b, acc[r + 1]));
                    acc[r + 2] = fmaf(q4.z, a, fmaf(-w4.z, b, acc[r + 2]));
                    acc[r + 3] = fmaf(q4.w, a, fmaf(-w4.w, b, acc[r + 3]));
                }
            }
#pragma unroll
            for (int r = 0; r < DR; ++r) dHs[(wid * DR + r) * kSlice + lane] = acc[r];
        }
    }
    __syncthreads();
    if (p.dS0)
        for (int d = wid; d < dk; d += kThreads / 32)
            p.dS0[sbase + (size_t)d * dv + col] = dHs[d * kSlice + lane];
}

// ---- per-chunk kernels: one block per (chunk, v-head) --------------------------------------

// Load rows [0, Cc) of a token-major tensor into smem rows of stride ld, zero-filling rows
// [Cc, C) so that products over the chunk need no bounds.
template <typename F>
__device__ void load_rows(float* dst, int C, int Cc, int n, int ld, F&& get) {
    for (int idx = threadIdx.x; idx < C * n; idx += kNT) {
        const int i = idx / n, d = idx % n;
        dst[i * ld + d] = i < Cc ? get(i, d) : 0.f;
    }
}

__global__ void __launch_bounds__(kNT, 1)
bwd_chunk_dqk(BwdParams p) {
    extern __shared__ float sm[];
    if (p.hdr->err != GDR_OK) return;
    ChunkPos cp;
    if (!chunk_pos(p, cp)) return;
    const int h = blockIdx.y, hk = h / (p.Hv / p.Hk);
    const int dk = p.dk, dv = p.dv, C = p.chunk, ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    const int ldt = dk + 1, Cc = cp.Cc;
    const Tile tl;
    const bool on = p.qk_l2norm;

    float* Qs = sm;                     // [C][dk+1] q^
    float* Ks = Qs + C * ldk;           // [C][dk+1] k^
    float* dOs = Ks + C * ldk;          // [C][dv+1]
    float* Vps = dOs + C * ldv;         // [C][dv+1] V'
    float* D1 = Vps + C * ldv;          // [C][C+1] s dP e^{G'_i - G_j} on the mask
    float* Tl = D1 + C * ldc;           // [32][dk+1] a 32-column tile of H or dH+, transposed
    float* dVt = Tl + kSlice * ldt;     // [C][33] the matching tile of dV'
    float* Gs = dVt + C * (kSlice + 1); // [C]
    float* Gr = Gs + C;                 // [C] G'
    float* qn = Gr + C;                 // [C]
    float* kn = qn + C;                 // [C]
    float* dGr = kn + C;                // [C] gradient of G'
    float* dGs = dGr + C;               // [C] gradient of G
    float* red = dGs + C;               // [1] <dH+, H>

    auto tok = [&](int i) { return phys_token(cp.t0, cp.t1, cp.p0 + i, p.reverse); };
    load_rows(Qs, C, Cc, dk, ldk, [&](int i, int d) {
        return load_elem(p.q, (size_t)(tok(i) * p.Hk + hk) * dk + d, p.io); });
    load_rows(Ks, C, Cc, dk, ldk, [&](int i, int d) {
        return load_elem(p.k, (size_t)(tok(i) * p.Hk + hk) * dk + d, p.io); });
    load_rows(dOs, C, Cc, dv, ldv, [&](int i, int e) {
        return load_elem(p.dO, (size_t)(tok(i) * p.Hv + h) * dv + e, p.io); });
    load_rows(Vps, C, Cc, dv, ldv, [&](int i, int e) {
        return p.Vp[(size_t)(tok(i) * p.Hv + h) * dv + e]; });
    for (int i = threadIdx.x; i < C; i += kNT) {
        Gs[i] = i < Cc ? p.G[(size_t)tok(i) * p.Hv + h] : 0.f;
        dGr[i] = 0.f; dGs[i] = 0.f;
    }
    if (threadIdx.x == 0) red[0] = 0.f;
    __syncthreads();
    l2norm_rows_keep(Qs, qn, Cc, dk, ldk, on);
    l2norm_rows_keep(Ks, kn, Cc, dk, ldk, on);
    for (int i = threadIdx.x; i < C; i += kNT)
        Gr[i] = p.read_pre ? (i > 0 ? Gs[i - 1] : 0.f) : Gs[i];
    __syncthreads();

    // dP_ij = dO_i . V'_j and S_ij = q^_i . k^_j; D1 = s dP e^{G'_i - G_j} on the mask;
    // E = D1 S carries the decay gradient of the intra-chunk read.
    {
        float dP[4][2] = {}, S[4][2] = {};
        for (int e = 0; e < dv; ++e) {
            float a[4], b[2];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? dOs[tl.row(ii) * ldv + e] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) b[jj] = tl.col(jj) < C ? Vps[tl.col(jj) * ldv + e] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) dP[ii][jj] = fmaf(a[ii], b[jj], dP[ii][jj]);
        }
        for (int d = 0; d < dk; ++d) {
            float a[4], b[2];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? Qs[tl.row(ii) * ldk + d] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) b[jj] = tl.col(jj) < C ? Ks[tl.col(jj) * ldk + d] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) S[ii][jj] = fmaf(a[ii], b[jj], S[ii][jj]);
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = tl.row(ii);
            float rsum = 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = tl.col(jj);
                const bool m = i < Cc && j < Cc && (p.read_pre ? j < i : j <= i);
                const float d1 = m ? p.scale * dP[ii][jj] * expf(Gr[i] - Gs[j]) : 0.f;
                const float e = d1 * S[ii][jj];
                if (i < C && j < C) D1[i * ldc + j] = d1;
                rsum += e;
                if (m) atomicAdd(&dGs[j], -e);
            }
            rsum = warp_sum(rsum);
            if (tl.cg == 0 && i < Cc) dGr[i] += rsum;
        }
    }
    __syncthreads();

    // Phase A: dQ^ = D1 K^ + s e^{G'} dO H^T; the inter read's decay gradient.
    const size_t cbase = ((size_t)cp.c * p.Hv + h) * dk * dv;
    {
        float acc[4][4] = {}, X[4][4] = {};
        for (int j = 0; j < C; ++j) {
            float a[4], b[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? D1[tl.row(ii) * ldc + j] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = tl.col(jj) < dk ? Ks[j * ldk + tl.col(jj)] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[ii][jj] = fmaf(a[ii], b[jj], acc[ii][jj]);
        }
        for (int e0 = 0; e0 < dv; e0 += kSlice) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < dk * kSlice; idx += kNT) {
                const int d = idx / kSlice, e = idx % kSlice;
                Tl[e * ldt + d] = p.Hc[cbase + (size_t)d * dv + e0 + e];
            }
            __syncthreads();
            for (int e = 0; e < kSlice; ++e) {
                float a[4], b[4];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? dOs[tl.row(ii) * ldv + e0 + e] : 0.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = tl.col(jj) < dk ? Tl[e * ldt + tl.col(jj)] : 0.f;
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) X[ii][jj] = fmaf(a[ii], b[jj], X[ii][jj]);
            }
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = tl.row(ii);
            const bool live = i < Cc;
            const float rd = live ? p.scale * expf(Gr[i]) : 0.f;
            float gsum = 0.f, proj = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int d = tl.col(jj);
                if (d < dk && live) {
                    const float qh = Qs[i * ldk + d];
                    gsum = fmaf(qh, X[ii][jj], gsum);
                    acc[ii][jj] = fmaf(rd, X[ii][jj], acc[ii][jj]);
                    proj = fmaf(qh, acc[ii][jj], proj);
                }
            }
            gsum = warp_sum(gsum);
            proj = warp_sum(proj);
            if (tl.cg == 0 && live) dGr[i] += rd * gsum;
            if (live) {
                const size_t base = (size_t)(tok(i) * p.Hv + h) * dk;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int d = tl.col(jj);
                    if (d < dk)
                        p.dqh[base + d] = norm_adjoint(acc[ii][jj], Qs[i * ldk + d], proj, qn[i], on);
                }
            }
        }
    }

    // Phase B: dK^ (P and carry parts) = D1^T Q^ + e^{G_C - G} V' dH+^T; the carry's decay
    // gradient.
    const float GC = Gs[Cc - 1];
    {
        float acc[4][4] = {}, Z[4][4] = {};
        for (int j = 0; j < C; ++j) {
            float a[4], b[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? D1[j * ldc + tl.row(ii)] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = tl.col(jj) < dk ? Qs[j * ldk + tl.col(jj)] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[ii][jj] = fmaf(a[ii], b[jj], acc[ii][jj]);
        }
        float hdot = 0.f;
        for (int e0 = 0; e0 < dv; e0 += kSlice) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < dk * kSlice; idx += kNT) {
                const int d = idx / kSlice, e = idx % kSlice;
                const size_t gi = cbase + (size_t)d * dv + e0 + e;
                const float dh = p.dHc[gi];
                Tl[e * ldt + d] = dh;
                hdot = fmaf(dh, p.Hc[gi], hdot);
            }
            __syncthreads();
            for (int e = 0; e < kSlice; ++e) {
                float a[4], b[4];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? Vps[tl.row(ii) * ldv + e0 + e] : 0.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = tl.col(jj) < dk ? Tl[e * ldt + tl.col(jj)] : 0.f;
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) Z[ii][jj] = fmaf(a[ii], b[jj], Z[ii][jj]);
            }
        }
        hdot = warp_sum(hdot);
        if ((threadIdx.x & 31) == 0) atomicAdd(red, hdot);
        float csum = 0.f;
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = tl.row(ii);
            const bool live = i < Cc;
            const float kd = live ? expf(GC - Gs[i]) : 0.f;
            float c = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int d = tl.col(jj);
                if (d < dk && live) {
                    c = fmaf(Ks[i * ldk + d], Z[ii][jj], c);
                    acc[ii][jj] = fmaf(kd, Z[ii][jj], acc[ii][jj]);
                }
            }
            c = warp_sum(c) * kd;
            if (tl.cg == 0 && live) { atomicAdd(&dGs[i], -c); csum += c; }
            if (live) {
                const size_t base = (size_t)(tok(i) * p.Hv + h) * dk;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int d = tl.col(jj);
                    if (d < dk) p.dKp[base + d] = acc[ii][jj];
                }
            }
        }
        if (tl.cg == 0) atomicAdd(&dGs[Cc - 1], csum);
    }

    // Phase C: dW = -dV' H^T.
    {
        float acc[4][4] = {};
        for (int e0 = 0; e0 < dv; e0 += kSlice) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < dk * kSlice; idx += kNT) {
                const int d = idx / kSlice, e = idx % kSlice;
                Tl[e * ldt + d] = p.Hc[cbase + (size_t)d * dv + e0 + e];
            }
            for (int idx = threadIdx.x; idx < C * kSlice; idx += kNT) {
                const int i = idx / kSlice, e = idx % kSlice;
                dVt[i * (kSlice + 1) + e] =
                    i < Cc ? p.dVp[(size_t)(tok(i) * p.Hv + h) * dv + e0 + e] : 0.f;
            }
            __syncthreads();
            for (int e = 0; e < kSlice; ++e) {
                float a[4], b[4];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? dVt[tl.row(ii) * (kSlice + 1) + e] : 0.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) b[jj] = tl.col(jj) < dk ? Tl[e * ldt + tl.col(jj)] : 0.f;
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) acc[ii][jj] = fmaf(a[ii], b[jj], acc[ii][jj]);
            }
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = tl.row(ii);
            if (i >= Cc) continue;
            const size_t base = (size_t)(tok(i) * p.Hv + h) * dk;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int d = tl.col(jj);
                if (d < dk) p.dW[base + d] = -acc[ii][jj];
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        dGs[Cc - 1] += expf(GC) * red[0];
        // the read decay G'_i is G_i (post) or G_{i-1} (pre; constant 0 for the first token)
        for (int i = 0; i < Cc; ++i) {
            if (!p.read_pre) dGs[i] += dGr[i];
            else if (i > 0) dGs[i - 1] += dGr[i];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < Cc; i += kNT) p.dGp[(size_t)tok(i) * p.Hv + h] = dGs[i];
}

__global__ void __launch_bounds__(kNT, 1)
bwd_chunk_wy(BwdParams p) {
    extern __shared__ float sm[];
    if (p.hdr->err != GDR_OK) return;
    ChunkPos cp;
    if (!chunk_pos(p, cp)) return;
    const int h = blockIdx.y, hk = h / (p.Hv / p.Hk);
    const int dk = p.dk, dv = p.dv, C = p.chunk, ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    const int ldr = dk + dv + 1, Cc = cp.Cc;
    const Tile tl;
    const bool on = p.qk_l2norm;

    float* Ks = sm;                     // [C][dk+1] k^
    float* Ws = Ks + C * ldk;           // [C][dk+1] W
    float* Us = Ws + C * ldk;           // [C][dv+1] U~
    float* R = Us + C * ldv;            // [C][dk+dv+1] dW | dV', solved in place to dR_w | dR_u
    float* A = R + C * ldr;             // [C][C+1] A (strict lower)
    float* Sk = A + C * ldc;            // [C][C+1] k^_i . k^_j, then beta_i dA_ij e^{G_i-G_j}
    float* Gs = Sk + C * ldc;           // [C]
    float* Bs = Gs + C;                 // [C] beta
    float* kn = Bs + C;                 // [C]
    float* dGs = kn + C;                // [C]
    float* dBs = dGs + C;               // [C]

    auto tok = [&](int i) { return phys_token(cp.t0, cp.t1, cp.p0 + i, p.reverse); };
    load_rows(Ks, C, Cc, dk, ldk, [&](int i, int d) {
        return load_elem(p.k, (size_t)(tok(i) * p.Hk + hk) * dk + d, p.io); });
    load_rows(Ws, C, Cc, dk, ldk, [&](int i, int d) {
        return p.W[(size_t)(tok(i) * p.Hv + h) * dk + d]; });
    load_rows(Us, C, Cc, dv, ldv, [&](int i, int e) {
        return p.U[(size_t)(tok(i) * p.Hv + h) * dv + e]; });
    load_rows(R, C, Cc, dk + dv, ldr, [&](int i, int x) {
        const size_t t = (size_t)tok(i) * p.Hv + h;
        return x < dk ? p.dW[t * dk + x] : p.dVp[t * dv + (x - dk)]; });
    for (int i = threadIdx.x; i < C; i += kNT) {
        const bool live = i < Cc;
        Gs[i] = live ? p.G[(size_t)tok(i) * p.Hv + h] : 0.f;
        Bs[i] = live ? load_elem(p.beta, (size_t)tok(i) * p.Hv + h, p.gt) : 0.f;
        dGs[i] = live ? p.dGp[(size_t)tok(i) * p.Hv + h] : 0.f;
        dBs[i] = 0.f;
    }
    __syncthreads();
    l2norm_rows_keep(Ks, kn, Cc, dk, ldk, on);
    __syncthreads();
    // A_ij = beta_i (k^_i . k^_j) e^{G_i - G_j}, j < i
    {
        float S[4][2] = {};
        for (int d = 0; d < dk; ++d) {
            float a[4], b[2];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? Ks[tl.row(ii) * ldk + d] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) b[jj] = tl.col(jj) < C ? Ks[tl.col(jj) * ldk + d] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) S[ii][jj] = fmaf(a[ii], b[jj], S[ii][jj]);
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int i = tl.row(ii), j = tl.col(jj);
                if (i >= C || j >= C) continue;
                const bool m = i < Cc && j < i;
                Sk[i * ldc + j] = S[ii][jj];
                A[i * ldc + j] = m ? Bs[i] * S[ii][jj] * expf(Gs[i] - Gs[j]) : 0.f;
            }
    }
    __syncthreads();
    // [dR_w | dR_u] = (I + A)^-T [dW | dV']: x_i = r_i - sum_{j > i} A_ji x_j, from the last row
    for (int x = threadIdx.x; x < dk + dv; x += kNT) {
        for (int i = Cc - 2; i >= 0; --i) {
            float r = R[i * ldr + x];
            for (int j = i + 1; j < Cc; ++j) r = fmaf(-A[j * ldc + i], R[j * ldr + x], r);
            R[i * ldr + x] = r;
        }
    }
    __syncthreads();
    // dA_ij = -(dR_w,i . W_j + dR_u,i . U~_j) on j < i, and what it carries to beta, G, k^
    {
        float dA[4][2] = {};
        for (int x = 0; x < dk + dv; ++x) {
            float a[4], b[2];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) a[ii] = tl.row(ii) < C ? R[tl.row(ii) * ldr + x] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = tl.col(jj);
                b[jj] = j < C ? (x < dk ? Ws[j * ldk + x] : Us[j * ldv + (x - dk)]) : 0.f;
            }
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) dA[ii][jj] = fmaf(-a[ii], b[jj], dA[ii][jj]);
        }
        __syncthreads();  // every thread has read R, W, U~; Sk is rewritten below
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = tl.row(ii);
            float db = 0.f, dg = 0.f;
            float sk[2], dd[2];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = tl.col(jj);
                const bool m = i < Cc && j < i;
                sk[jj] = (i < C && j < C) ? Sk[i * ldc + j] : 0.f;
                const float D = m ? dA[ii][jj] * expf(Gs[i] - Gs[j]) : 0.f;
                dd[jj] = D;
                db = fmaf(D, sk[jj], db);
                const float ga = m ? dA[ii][jj] * A[i * ldc + j] : 0.f;
                dg += ga;
                if (m) atomicAdd(&dGs[j], -ga);
            }
            db = warp_sum(db);
            dg = warp_sum(dg);
            if (tl.cg == 0 && i < Cc) { atomicAdd(&dBs[i], db); atomicAdd(&dGs[i], dg); }
            const float bi = i < C ? Bs[i] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = tl.col(jj);
                if (i < C && j < C) Sk[i * ldc + j] = bi * dd[jj];
            }
        }
    }
    __syncthreads();
    // dK^ = (beta D) K^ + (beta D)^T K^ + diag(beta e^G) dR_w + the P and carry parts
    {
        float acc[4][4] = {};
        for (int j = 0; j < C; ++j) {
            float a1[4], a2[4], b[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int i = tl.row(ii);
                a1[ii] = i < C ? Sk[i * ldc + j] : 0.f;
                a2[ii] = i < C ? Sk[j * ldc + i] : 0.f;
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) b[jj] = tl.col(jj) < dk ? Ks[j * ldk + tl.col(jj)] : 0.f;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[ii][jj] = fmaf(a1[ii] + a2[ii], b[jj], acc[ii][jj]);
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = tl.row(ii);
            const bool live = i < Cc;
            const float eg = live ? expf(Gs[i]) : 0.f, be = live ? Bs[i] * eg : 0.f;
            const size_t base = live ? (size_t)(tok(i) * p.Hv + h) * dk : 0;
            float r = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int d = tl.col(jj);
                if (d < dk && live) {
                    const float rw = R[i * ldr + d];
                    r = fmaf(Ks[i * ldk + d], rw, r);
                    acc[ii][jj] = fmaf(be, rw, acc[ii][jj]) + p.dKp[base + d];
                }
            }
            r = warp_sum(r);
            if (tl.cg == 0 && live) { atomicAdd(&dBs[i], eg * r); atomicAdd(&dGs[i], be * r); }
            float proj = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int d = tl.col(jj);
                if (d < dk && live) proj = fmaf(Ks[i * ldk + d], acc[ii][jj], proj);
            }
            proj = warp_sum(proj);
            if (live) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int d = tl.col(jj);
                    if (d < dk)
                        p.dkh[base + d] = norm_adjoint(acc[ii][jj], Ks[i * ldk + d], proj, kn[i], on);
                }
            }
        }
    }
    // dv = beta dR_u; dbeta += v . dR_u (one warp per row)
    {
        const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
        for (int i = wid; i < Cc; i += kNT / 32) {
            const size_t base = (size_t)(tok(i) * p.Hv + h) * dv;
            float db = 0.f;
            for (int e = lane; e < dv; e += 32) {
                const float ru = R[i * ldr + dk + e];
                db = fmaf(load_elem(p.v, base + e, p.io), ru, db);
                store_elem(p.dv_out, base + e, Bs[i] * ru, p.io);
            }
            db = warp_sum(db);
            if (lane == 0) atomicAdd(&dBs[i], db);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // dg_j = sum_{i >= j} dG_i within the chunk
        float run = 0.f;
        for (int i = Cc - 1; i >= 0; --i) {
            run += dGs[i];
            const size_t t = (size_t)tok(i) * p.Hv + h;
            store_elem(p.dg_out, t, run, p.gt);
            store_elem(p.dbeta_out, t, dBs[i], p.gt);
        }
    }
}

// dq, dk per key head: the sum over the v-heads that read it.  Four consecutive features per
// thread (dk is a multiple of 32): 16-byte loads of the fp32 per-v-head parts, one 8- or
// 16-byte store of the io-dtype result.
__global__ void bwd_reduce_heads4(BwdParams p, long long n4) {
    const int group = p.Hv / p.Hk, dk4 = p.dk / 4;
    const float4* qh = reinterpret_cast<const float4*>(p.dqh);
    const float4* kh = reinterpret_cast<const float4*>(p.dkh);
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n4;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long d4 = idx % dk4, r = idx / dk4;  // r = t * Hk + hk
        const long long t = r / p.Hk, hk = r % p.Hk;
        float4 sq = make_float4(0.f, 0.f, 0.f, 0.f), sk = sq;
        const size_t src = ((size_t)t * p.Hv + hk * group) * dk4 + d4;
        for (int j = 0; j < group; ++j) {
            const float4 a = __ldcs(qh + src + (size_t)j * dk4), b = __ldcs(kh + src + (size_t)j * dk4);
            sq.x += a.x; sq.y += a.y; sq.z += a.z; sq.w += a.w;
            sk.x += b.x; sk.y += b.y; sk.z += b.z; sk.w += b.w;
        }
        if (p.io == GDR_BF16) {
            const __nv_bfloat162 q0 = __floats2bfloat162_rn(sq.x, sq.y), q1 = __floats2bfloat162_rn(sq.z, sq.w);
            const __nv_bfloat162 k0 = __floats2bfloat162_rn(sk.x, sk.y), k1 = __floats2bfloat162_rn(sk.z, sk.w);
            reinterpret_cast<uint2*>(p.dq_out)[idx] =
                make_uint2(*reinterpret_cast<const uint32_t*>(&q0), *reinterpret_cast<const uint32_t*>(&q1));
            reinterpret_cast<uint2*>(p.dk_out)[idx] =
                make_uint2(*reinterpret_cast<const uint32_t*>(&k0), *reinterpret_cast<const uint32_t*>(&k1));
        } else {
            reinterpret_cast<float4*>(p.dq_out)[idx] = sq;
            reinterpret_cast<float4*>(p.dk_out)[idx] = sk;
        }
    }
}

size_t states_fwd_smem(const gdr_chunk_args& a) {
    const int C = a.chunk;
    return sizeof(float) * ((size_t)a.dk * kSlice + 2 * (size_t)C * a.dk + (size_t)C * (kSlice + 1));
}

size_t states_bwd_smem(const gdr_chunk_args& a) {
    const int C = a.chunk;
    return sizeof(float) * ((size_t)a.dk * kSlice + 3 * (size_t)C * a.dk + (size_t)C * C +
                            2 * (size_t)C * (kSlice + 1));
}

size_t dqk_smem(const gdr_chunk_args& a) {
    const int C = a.chunk;
    return sizeof(float) * (2 * (size_t)C * (a.dk + 1) + 2 * (size_t)C * (a.dv + 1) +
                            (size_t)C * (C + 1) + (size_t)kSlice * (a.dk + 1) +
                            (size_t)C * (kSlice + 1) + 6 * (size_t)C + 1);
}

size_t wy_smem(const gdr_chunk_args& a) {
    const int C = a.chunk;
    return sizeof(float) * (2 * (size_t)C * (a.dk + 1) + (size_t)C * (a.dv + 1) +
                            (size_t)C * (a.dk + a.dv + 1) + 2 * (size_t)C * (C + 1) + 5 * (size_t)C);
}

constexpr size_t kMaxSmem = 227 * 1024;

template <int RP, int DR>
gdr_status launch_states_t(const gdr_chunk_args& a, const BwdParams& p, dim3 grid,
                           cudaStream_t st) {
    const size_t sf = states_fwd_smem(a), sb = states_bwd_smem(a);
    if (cudaFuncSetAttribute(bwd_states_fwd<RP, DR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sf) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_states_bwd<RP, DR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sb) != cudaSuccess)
        return GDR_ERR_CUDA;
    bwd_states_fwd<RP, DR><<<grid, kThreads, sf, st>>>(p);
    bwd_states_bwd<RP, DR><<<grid, kThreads, sb, st>>>(p);
    return GDR_OK;
}

template <int RP>
gdr_status launch_states_dk(const gdr_chunk_args& a, const BwdParams& p, dim3 grid,
                            cudaStream_t st) {
    switch (a.dk) {
        case 32: return launch_states_t<RP, 4>(a, p, grid, st);
        case 64: return launch_states_t<RP, 8>(a, p, grid, st);
        case 96: return launch_states_t<RP, 12>(a, p, grid, st);
        case 128: return launch_states_t<RP, 16>(a, p, grid, st);
    }
    return GDR_ERR_UNSUPPORTED;
}

// State passes for C rows per chunk (C/8 per warp) and dk state rows (dk/8 per warp).
gdr_status launch_states(const gdr_chunk_args& a, const BwdParams& p, dim3 grid,
                         cudaStream_t st) {
    switch (a.chunk) {
        case 16: return launch_states_dk<2>(a, p, grid, st);
        case 32: return launch_states_dk<4>(a, p, grid, st);
        case 64: return launch_states_dk<8>(a, p, grid, st);
    }
    return GDR_ERR_UNSUPPORTED;
}

}  // namespace

bool bwd_tc_path(const gdr_chunk_args& a);

// Backward workspace: the forward's plan and CUDA-core arrays, then the backward's own.  The
// tensor-core path reads none of the CUDA-core arrays (W, U~, and the scan's Q~, K~, P), so
// its own arrays, G first, start where those would.
BwdLayout bwd_layout(const gdr_chunk_args& a) {
    BwdLayout B{};
    B.base = ws_layout(a, true);
    const long long T_tot = (long long)a.B * a.T;
    const size_t tk = sizeof(float) * (size_t)T_tot * a.Hv * a.dk;
    const size_t tv = sizeof(float) * (size_t)T_tot * a.Hv * a.dv;
    const size_t st = sizeof(float) * (size_t)B.base.max_chunks * a.Hv * a.dk * a.dv;
    const bool tc = bwd_tc_path(a) && B.base.W > 0;
    size_t off = tc ? B.base.W : B.base.total;
    if (tc) {
        B.G = off; off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv, 256);
    } else {
        B.G = B.base.G;
    }
    B.Hc = off;  off = align_up(off + st, 256);
    B.dHc = off; off = align_up(off + st, 256);
    B.Vp = off;  off = align_up(off + tv, 256);
    B.dVp = off; off = align_up(off + tv, 256);
    B.dW = off;  off = align_up(off + tk, 256);
    B.dKp = off; off = align_up(off + tk, 256);
    B.dqh = off; off = align_up(off + tk, 256);
    B.dkh = off; off = align_up(off + tk, 256);
    B.dGp = off; off = align_up(off + sizeof(float) * (size_t)T_tot * a.Hv, 256);
    B.total = off;
    return B;
}

bool bwd_supported(const gdr_chunk_args& a) {
    if (a.gate_raw || a.gdn2 || a.o_accumulate) return false;
    // the state passes split C rows and dk state rows over 8 warps, the latter in float4s
    if (a.chunk > 64 || a.dk > 128 || a.dk % 32 != 0 || a.dv > 128 || a.dv % kSlice != 0)
        return false;
    return simt_supported(a) && simt_rb(a) && states_fwd_smem(a) <= kMaxSmem &&
           states_bwd_smem(a) <= kMaxSmem && dqk_smem(a) <= kMaxSmem && wy_smem(a) <= kMaxSmem;
}

// bf16, head size 128, chunk 64: the tensor-core kernels (both recurrences on the fused
// forward kernel, the per-chunk steps in chunk_bwd_tc.cu)
bool bwd_tc_path(const gdr_chunk_args& a) { return bwd_dqk_tc_supported(a) && tc_supported(a); }

gdr_status launch_chunk_bwd(const gdr_chunk_args& a, const BwdPtrs& x, void* ws,
                            const BwdLayout& B, cudaStream_t st) {
    char* base = static_cast<char*>(ws);
    const WsLayout& L = B.base;
    BwdParams p{};
    p.q = x.q; p.k = x.k; p.v = x.v; p.g = x.g; p.beta = x.beta; p.dO = x.dO;
    p.S0 = x.S0; p.dS_final = x.dS_final;
    p.dq_out = x.dq; p.dk_out = x.dk; p.dv_out = x.dv; p.dg_out = x.dg; p.dbeta_out = x.dbeta;
    p.dS0 = x.dS0;
    p.hdr = reinterpret_cast<const WsHeader*>(base);
    p.cu = reinterpret_cast<const int32_t*>(base + L.cu);
    p.chunk_off = reinterpret_cast<const int32_t*>(base + L.chunk_off);
    p.chunk_seq = reinterpret_cast<const int32_t*>(base + L.chunk_seq);
    float* W = reinterpret_cast<float*>(base + L.W);
    float* U = reinterpret_cast<float*>(base + L.U);
    float* G = reinterpret_cast<float*>(base + B.G);
    p.W = W; p.U = U; p.G = G;
    p.Hc = reinterpret_cast<float*>(base + B.Hc);
    p.dHc = reinterpret_cast<float*>(base + B.dHc);
    p.Vp = reinterpret_cast<float*>(base + B.Vp);
    p.dVp = reinterpret_cast<float*>(base + B.dVp);
    p.dW = reinterpret_cast<float*>(base + B.dW);
    p.dKp = reinterpret_cast<float*>(base + B.dKp);
    p.dqh = reinterpret_cast<float*>(base + B.dqh);
    p.dkh = reinterpret_cast<float*>(base + B.dkh);
    p.dGp = reinterpret_cast<float*>(base + B.dGp);
    p.Qt = reinterpret_cast<const float*>(base + L.Qt);
    p.Kt = reinterpret_cast<const float*>(base + L.Kt);
    p.Pc = reinterpret_cast<const float*>(base + L.Pc);
    p.Hk = a.Hk; p.Hv = a.Hv; p.dk = a.dk; p.dv = a.dv; p.chunk = a.chunk;
    p.read_pre = a.read_mode == GDR_READ_PRE; p.qk_l2norm = a.qk_l2norm; p.reverse = a.reverse;
    p.io = a.io_dtype; p.gt = a.gate_dtype; p.scale = a.scale;

    // bf16, head size 128, chunk 64: the tensor-core forward leaves G, H and V' (its saving
    // instantiation), and the per-chunk steps run on the tensor cores (the WY step forms W
    // and U~ again from its own T)
    const bool tc = bwd_tc_path(a);
    p.direct_out = tc && a.Hv == a.Hk;
    gdr_status s;
    if (tc) {
        // the forward, then the reverse state pass (dH+ per chunk, dV', dS0) on the same kernel
        const TcSave fw{G, p.Hc, p.Vp, false};
        const TcSave ad{nullptr, p.dHc, p.dVp, true};
        s = launch_chunk_tc(a, x.q, x.k, x.v, x.g, x.beta, x.S0, nullptr, nullptr, ws, L, st,
                            false, nullptr, nullptr, 0, &fw);
        if (s == GDR_OK)
            s = launch_chunk_tc(a, x.q, x.k, x.dO, x.g, x.beta, x.dS_final, nullptr, x.dS0, ws, L,
                                st, false, nullptr, nullptr, 0, &ad);
    } else {
        s = launch_wy_local_simt(a, x.k, x.v, x.g, x.beta, ws, L, W, U, G, st);
        if (s == GDR_OK) s = launch_prep_simt(a, x.q, x.k, ws, L, st);
    }
    if (s != GDR_OK) return s;
    const size_t sm_q = dqk_smem(a), sm_w = wy_smem(a);
    if (cudaFuncSetAttribute(bwd_chunk_dqk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_q) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_chunk_wy, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_w) != cudaSuccess)
        return GDR_ERR_CUDA;
    const dim3 gc((unsigned)L.max_chunks, (unsigned)a.Hv);
    const dim3 gs((unsigned)a.n_seqs, (unsigned)a.Hv, (unsigned)(a.dv / kSlice));
    if (!tc && (s = launch_states(a, p, gs, st)) != GDR_OK) return s;
    if (L.max_chunks > 0) {
        if (tc) {
            if ((s = launch_bwd_dqk_tc(p, gc, st)) != GDR_OK) return s;
            if ((s = launch_bwd_wy_tc(p, gc, st)) != GDR_OK) return s;
        } else {
            bwd_chunk_dqk<<<gc, kNT, sm_q, st>>>(p);
            bwd_chunk_wy<<<gc, kNT, sm_w, st>>>(p);
        }
        // with one v-head per key head there is nothing to sum: the tensor-core kernels
        // write dq and dk themselves
        const long long n4 = (long long)a.B * a.T * a.Hk * (a.dk / 4);
        const unsigned blocks = (unsigned)std::min<long long>((n4 + kThreads - 1) / kThreads, 148LL * 16);
        if (n4 > 0 && !p.direct_out) bwd_reduce_heads4<<<blocks, kThreads, 0, st>>>(p, n4);
    }
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr
