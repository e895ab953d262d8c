/*
 * gdr_oracle.c -- fp64 CPU oracle of the gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct ground
 * truth that the CUDA library is checked against.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark may load it.  It shares
 * no code, header or constant with the CUDA path.
 *
 * What it computes (plain definition, one token at a time, no chunking):
 *
 *   Prizma "seq/delta.py", module docstring and `_delta_reference`:
 *       S_t = alpha_t S_{t-1} + u_t k_t^T,
 *       u_t = beta_t (v_t - alpha_t S_{t-1} k_t),
 *       pre-write read o_t = S_{t-1} q_t.
 *   sparse_delta_memory/layer.py, `SparseDeltaMemory` docstring: the memory
 *     decays by the exponential of the gate, then takes the delta write of beta
 *     times k and the prediction error, i.e. alpha_t = exp(g_t).
 *   tiny_gdn/fugue.py, `BidirectionalGatedDeltaNet2` docstring: the forward
 *     scan reads q_t^T S_t (post-write read).
 *
 * The state is stored transposed, H = S^T with shape [dk][dv] (dv
 * contiguous), the layout the library uses for S0 / S_final.  In that form
 *       s_k   = H^T k_t                    (= S_{t-1} k_t)
 *       u_t   = beta_t (v_t - alpha_t s_k)
 *       H    <- alpha_t H + k_t u_t^T
 * and the read is o_t = scale * H^T q_t, taken before the update (PRE) or
 * after it (POST).  `scale` multiplies both read modes.
 *
 * Optional L2 normalisation of q and k (the `use_qk_l2norm_in_kernel` flag of
 * tiny_gdn/fugue.py `scan`, and `F.normalize(eps=1e-6)` of
 * nested_learning/titan/self_modifying.py): x <- x / max(||x||_2, 1e-6),
 * computed here in fp64.
 *
 * Layouts (all row-major, contiguous):
 *   q, k   [B, T, Hk, dk]      v, o  [B, T, Hv, dv]      g, beta [B, T, Hv]
 *   S0, S_final [n_seqs, Hv, dk, dv]
 * With cu_seqlens (varlen) B must be 1 and sequence s covers the packed tokens
 * [cu_seqlens[s], cu_seqlens[s+1]).  Without it, sequence s is row s (n_seqs=B).
 * v-head h reads q/k head h / (Hv/Hk)  (tiny_gdn/fugue.py `heads`, key heads
 * repeated to the value heads).
 * `reverse` != 0 scans every sequence from its last token to its first
 * (tiny_gdn/fugue.py `scan`, direction 1, in-place segment reversal); o is
 * still written at each token's own position.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, Hk, Hv, dk, dv;
    int n_seqs;
    int read_pre;   /* 0: o = scale*S_t q_t ; 1: o = scale*S_{t-1} q_t */
    int qk_l2norm;  /* 1: normalise q and k */
    int reverse;    /* 1: scan each sequence back to front */
    double scale;
} gdr_oracle_args;

enum { ORACLE_OK = 0, ORACLE_BAD_ARG = 1, ORACLE_NOMEM = 2 };

static void l2_normalise(double *x, int n) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double nrm = sqrt(ss);
    double den = nrm > 1e-6 ? nrm : 1e-6;
    for (int i = 0; i < n; ++i) x[i] /= den;
}

/* H^T x for H [dk][dv]: out[j] = sum_d H[d][j] x[d]. */
static void state_t_times(const double *H, const double *x, int dk, int dv, double *out) {
    for (int j = 0; j < dv; ++j) out[j] = 0.0;
    for (int d = 0; d < dk; ++d) {
        const double xd = x[d];
        const double *row = H + (size_t)d * dv;
        for (int j = 0; j < dv; ++j) out[j] += row[j] * xd;
    }
}

/* One token of the recurrence on one (sequence, v-head) state. */
static void token_step(double *H, const double *q, const double *k, const double *v,
                       double g, double beta, int dk, int dv, int read_pre, double scale,
                       double *o, double *sk, double *u) {
    const double alpha = exp(g);
    if (read_pre) {
        state_t_times(H, q, dk, dv, o);
        for (int j = 0; j < dv; ++j) o[j] *= scale;
    }
    state_t_times(H, k, dk, dv, sk);
    for (int j = 0; j < dv; ++j) u[j] = beta * (v[j] - alpha * sk[j]);
    for (int d = 0; d < dk; ++d) {
        double *row = H + (size_t)d * dv;
        const double kd = k[d];
        for (int j = 0; j < dv; ++j) row[j] = alpha * row[j] + kd * u[j];
    }
    if (!read_pre) {
        state_t_times(H, q, dk, dv, o);
        for (int j = 0; j < dv; ++j) o[j] *= scale;
    }
}

/*
 * Whole forward over all sequences and v-heads.  S0 may be NULL (zero initial
 * state); S_final may be NULL.  Returns ORACLE_OK or an error code.
 */
int gdr_oracle_forward(const gdr_oracle_args *a, const double *q, const double *k,
                       const double *v, const double *g, const double *beta,
                       const double *S0, const int32_t *cu_seqlens, double *o,
                       double *S_final) {
    if (!a || !q || !k || !v || !g || !beta || !o) return ORACLE_BAD_ARG;
    if (a->Hk <= 0 || a->Hv <= 0 || a->Hv % a->Hk != 0 || a->dk <= 0 || a->dv <= 0)
        return ORACLE_BAD_ARG;
    if (cu_seqlens && a->B != 1) return ORACLE_BAD_ARG;
    if (!cu_seqlens && a->n_seqs != a->B) return ORACLE_BAD_ARG;
    const int Hk = a->Hk, Hv = a->Hv, dk = a->dk, dv = a->dv;
    const int group = Hv / Hk;
    const long n_units = (long)a->n_seqs * Hv;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (long unit = 0; unit < n_units; ++unit) {
        const int s = (int)(unit / Hv), h = (int)(unit % Hv), hk = h / group;
        long t0, t1;
        if (cu_seqlens) { t0 = cu_seqlens[s]; t1 = cu_seqlens[s + 1]; }
        else { t0 = (long)s * a->T; t1 = t0 + a->T; }
        double *H = (double *)malloc(sizeof(double) * ((size_t)dk * dv + 2 * dk + 3 * dv));
        if (!H) { failed = 1; continue; }
        double *qb = H + (size_t)dk * dv, *kb = qb + dk, *sk = kb + dk, *u = sk + dv, *ob = u + dv;
        if (S0) memcpy(H, S0 + (size_t)unit * dk * dv, sizeof(double) * (size_t)dk * dv);
        else memset(H, 0, sizeof(double) * (size_t)dk * dv);
        const long n = t1 - t0;
        for (long i = 0; i < n; ++i) {
            const long t = a->reverse ? (t1 - 1 - i) : (t0 + i);
            memcpy(qb, q + ((size_t)t * Hk + hk) * dk, sizeof(double) * dk);
            memcpy(kb, k + ((size_t)t * Hk + hk) * dk, sizeof(double) * dk);
            if (a->qk_l2norm) { l2_normalise(qb, dk); l2_normalise(kb, dk); }
            const double *vt = v + ((size_t)t * Hv + h) * dv;
            token_step(H, qb, kb, vt, g[(size_t)t * Hv + h], beta[(size_t)t * Hv + h], dk, dv,
                       a->read_pre, a->scale, ob, sk, u);
            memcpy(o + ((size_t)t * Hv + h) * dv, ob, sizeof(double) * dv);
        }
        if (S_final) memcpy(S_final + (size_t)unit * dk * dv, H, sizeof(double) * (size_t)dk * dv);
        free(H);
    }
    return failed ? ORACLE_NOMEM : ORACLE_OK;
}

/*
 * One-token decode step on N independent sequences: the same token_step with
 * T = 1, the state updated in place (flashrt fused_layer.py `_decode_one`,
 * the recurrent core that carries `recurrent_states` from token to token).
 *   q, k [N, Hk, dk]; v, o [N, Hv, dv]; g, beta [N, Hv]; S_inout [N, Hv, dk, dv].
 */
int gdr_oracle_decode_step(int N, int Hk, int Hv, int dk, int dv, int read_pre,
                           int qk_l2norm, double scale, const double *q, const double *k,
                           const double *v, const double *g, const double *beta,
                           double *S_inout, double *o) {
    gdr_oracle_args a;
    a.B = N; a.T = 1; a.Hk = Hk; a.Hv = Hv; a.dk = dk; a.dv = dv; a.n_seqs = N;
    a.read_pre = read_pre; a.qk_l2norm = qk_l2norm; a.reverse = 0; a.scale = scale;
    /* the state is read from and written back to the same buffer: each
       (sequence, head) unit owns a disjoint slice and copies it in first */
    return gdr_oracle_forward(&a, q, k, v, g, beta, S_inout, NULL, o, S_inout);
}
