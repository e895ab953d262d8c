/*
 * gdr.h -- C ABI of the B200 gated delta-rule library (libgdr.so).
 *
 * The recurrence, per (sequence n, value head h), with the state held
 * transposed as H = S^T of shape [dk][dv] (dv contiguous):
 *
 *     u_t = beta_t (v_t - alpha_t H_{t-1}^T k_t)
 *     H_t = alpha_t H_{t-1} + k_t u_t^T,            alpha_t = exp(g_t)
 *     post-write read  o_t = scale * H_t^T q_t
 *     pre-write read   o_t = scale * H_{t-1}^T q_t
 *
 * (Prizma "seq/delta.py", module docstring: the same update on the untransposed
 * state, and the strictly causal read from the state before the token's write;
 * sparse_delta_memory/layer.py, SparseDeltaMemory docstring: the memory decays by
 * the gate's exponential, then takes a write of beta times the key and the
 * prediction error; tiny_gdn/fugue.py, BidirectionalGatedDeltaNet2 docstring: the
 * forward scan reads the state after the token's write.)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor argument is a DEVICE pointer owned by the caller.  The
 *   library never allocates, frees or synchronises; every call only enqueues
 *   kernels on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *   stream) and returns.  Calls hold no host state between them.
 * - All tensors are dense and row-major in the index order given.  Pointers
 *   must be 16-byte aligned (GDR_ERR_ALIGNMENT otherwise).
 * - Arguments are validated on the host before anything is enqueued; a call
 *   that returns anything but GDR_OK has enqueued nothing (except
 *   GDR_ERR_CUDA, returned when a launch itself fails).
 * - Inconsistencies only visible on the device (a cu_seqlens array that is not
 *   non-decreasing, does not start at 0 or does not end at T) are recorded in
 *   an error word inside the workspace; the kernels then skip the work.  Read
 *   it with gdr_read_device_error.  No kernel traps or waits without a bound
 *   (the one wait not on a timer: in gdr_chunk_fwd_bidir the two CTAs of a
 *   cluster meet at a cluster barrier before they exit, and each bounds every
 *   wait that could keep it from getting there).
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,   /* null pointer, bad size, Hv % Hk != 0, bad enum ... */
    GDR_ERR_UNSUPPORTED = 2,   /* valid, but no kernel for this (dk, dv, chunk, dtype) */
    GDR_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    GDR_ERR_WORKSPACE = 4,     /* workspace missing or smaller than the required size */
    GDR_ERR_CUDA = 5,          /* a CUDA launch failed (cudaGetLastError after launch) */
    GDR_ERR_DEVICE_CHECK = 6,  /* device-side check failed (bad cu_seqlens) */
    GDR_ERR_TIMEOUT = 7,       /* a bounded device-side wait gave up */
    GDR_ERR_RANGE = 8          /* tensor-core path: an internal operand left the fp16 range
                                  (|x| >= 65000 or not finite); the outputs are not valid */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

/* Read mode.  POST: o_t = scale * S_t q_t (tiny_gdn/fugue.py forward scan,
 * q_t^T S_t).  PRE: o_t = scale * S_{t-1} q_t (Prizma "seq/delta.py", the
 * strictly causal pre-write read). */
typedef enum { GDR_READ_POST = 0, GDR_READ_PRE = 1 } gdr_read_mode;

/*
 * Arguments of the chunk-parallel forward (training / prefill).
 *
 * The forward is evaluated in the exact chunk-wise WY/UT form (Prizma
 * "seq/delta.py", chunked_delta: per chunk a unit-lower-triangular solve
 * (I + A) U = ..., then the chunk-to-chunk state carry;
 * sparse_delta_memory/layer.py module docstring: the chunk size changes the
 * result only through floating-point rounding).
 */
typedef struct {
    int B;                 /* rows; with cu_seqlens B must be 1 */
    int T;                 /* tokens per row (with cu_seqlens: total packed tokens) */
    int Hk, Hv;            /* key/query heads and value heads, Hv % Hk == 0; value head h
                              reads key head h / (Hv / Hk)  (tiny_gdn/fugue.py `heads`) */
    int dk, dv;            /* head dims; GPU kernels: dk, dv in {32, 64, 128} */
    int n_seqs;            /* == B without cu_seqlens, else number of packed sequences */
    int chunk;             /* 16, 32, 64 or 128 (64: the contract of flashrt fused_layer.py
                              `_prefill_chain`); chunks restart at every sequence start */
    gdr_dtype io_dtype;    /* dtype of q, k, v and o */
    gdr_dtype gate_dtype;  /* dtype of g and beta */
    gdr_read_mode read_mode;
    float scale;           /* multiplies the read in both modes */
    int qk_l2norm;         /* 1: q, k <- x / max(||x||_2, 1e-6) in fp32 inside the kernels
                              (use_qk_l2norm_in_kernel of tiny_gdn/fugue.py `scan`) */
    int reverse;           /* 1: scan every sequence from its last token to its first, in
                              place (tiny_gdn/fugue.py `scan`, direction 1); o is written at
                              each token's own position, S_final is the state after the
                              sequence's FIRST token */
    int o_accumulate;      /* 1: o += result (o is read, the sum written back in io_dtype);
                              0: o = result */
    /* Fused gating prologue (sparse_delta_memory/layer.py `compute_gates`: A = -exp(A_log),
     * g = A * softplus(a + dt_bias), beta = sigmoid(b); tiny_gdn/fugue.py `project`: beta
     * doubled to allow negative eigenvalues; flashrt fused_layer.py `gdn_gating`).
     *   gate_raw = 0: g and beta are the gates themselves; the three fields below are unused.
     *   gate_raw = 1: the g and beta arguments hold the raw per-token projections a and b
     *                 (same shape and gate_dtype), and the kernels form, in fp32,
     *                   g    = gate_A[h] * softplus(a + gate_dt_bias[h])
     *                   beta = beta_scale * sigmoid(b)
     *                 with softplus(x) = x for x > 20 (as torch's softplus threshold). */
    int gate_raw;
    const float* gate_A;        /* [Hv] fp32 device array, A = -exp(A_log) (<= 0 for a decay);
                                   4-byte aligned; required when gate_raw */
    const float* gate_dt_bias;  /* [Hv] fp32 device array; 4-byte aligned; required when
                                   gate_raw */
    float beta_scale;           /* 1, or 2 for negative eigenvalues; must be finite */
    /* GDN-2 decoupled gates (tiny_gdn/fugue.py BidirectionalGatedDeltaNet2:
     * S_t = (I - k_t (b_t * k_t)^T) Diag(exp g_t) S_{t-1} + k_t (w_t * v_t)^T).
     *   gdn2 = 0: scalar gates, g and beta of one value per token and value head.
     *   gdn2 = 1: g is the per-key-channel log decay [.., Hv, dk], beta the per-key-channel
     *             erase gate b [.., Hv, dk], and gdn2_w the per-value-channel write gate
     *             [.., Hv, dv], all gate_dtype and 16-byte aligned.  With g = log(alpha),
     *             b = w = beta on every channel this is the scalar rule.  Not combined with
     *             gate_raw.  bf16 inputs and gates with dk = dv = 128, chunk 64 and forward
     *             scans take the tensor cores (a preparation kernel over every chunk and
     *             head, then the recursion); a chunk whose per-channel decay grows by more
     *             than 2^100 within 16 tokens is refused there with GDR_ERR_RANGE. */
    int gdn2;
    const void* gdn2_w;
    /* Optional device status word (NULL: none).  A device int owned by the caller, who
     * sets it to GDR_OK (0) before the call.  When a device-side check of the call fails
     * (GDR_ERR_DEVICE_CHECK, GDR_ERR_TIMEOUT, GDR_ERR_RANGE), the call's last kernel stores
     * that status here if the word still holds GDR_OK; the library never clears it.  The
     * caller reads it whenever it likes (e.g. cudaMemcpyAsync into pinned host memory on
     * the same stream), with no synchronisation inside the library, so one word can
     * collect the status of many calls.  4-byte aligned.  Serves every entry point that
     * takes these arguments, gdr_chunk_fwd_noalloc included. */
    int* status;
} gdr_chunk_args;

/* Bytes of device workspace gdr_chunk_fwd needs for these arguments (0 on invalid
 * arguments).  Depends on B, T, Hv, dk, dv, n_seqs, chunk and the dtypes only. */
size_t gdr_chunk_fwd_workspace_size(const gdr_chunk_args* args);

/*
 * Chunk-parallel forward over every sequence and value head.
 *
 *   q, k        [B, T, Hk, dk]   io_dtype
 *   v           [B, T, Hv, dv]   io_dtype
 *   g, beta     [B, T, Hv]       gate_dtype; g = log(alpha) (<= 0 for a decay), beta
 *                                 unrestricted (beta in (0, 2) gives negative
 *                                 eigenvalues, tiny_gdn/fugue.py `project`)
 *   S0          [n_seqs, Hv, dk, dv] fp32 initial state, or NULL for zero
 *   cu_seqlens  [n_seqs + 1] int32 device offsets into the packed row (B == 1), or
 *               NULL for B rows of T tokens (tiny_gdn/fugue.py `segment_layout`)
 *   o           [B, T, Hv, dv]   io_dtype output (rounded to nearest even for bf16)
 *   S_final     [n_seqs, Hv, dk, dv] fp32 final state, or NULL; may alias S0
 *               (each state is read completely before its final value is written)
 *   workspace   device scratch of at least gdr_chunk_fwd_workspace_size(args) bytes,
 *               256-byte aligned; its contents need no initialisation
 *
 * Empty sequences are allowed (their S_final is S0, or zero).
 */
gdr_status gdr_chunk_fwd(const gdr_chunk_args* args,
                         const void* q, const void* k, const void* v,
                         const void* g, const void* beta,
                         const float* S0, const int32_t* cu_seqlens,
                         void* o, float* S_final,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdr_chunk_fwd without a caller-provided workspace.  (No counterpart on the pages: this is
 * a convenience of this library.)
 *
 * For callers that cannot allocate device memory: a serving process whose GPU memory is
 * reserved up front by its own pool (cudaMalloc may fail there, and it synchronises the
 * device), code inside a framework hook or callback where the CUDA allocator may not be
 * called, or a plain-C caller without a device allocator.  The caller still passes the
 * inputs and outputs exactly as for gdr_chunk_fwd; the scratch is a static device array of
 * GDR_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds until exit.
 *
 * - Calls whose scratch need (gdr_chunk_fwd_workspace_size) exceeds the array return
 *   GDR_ERR_WORKSPACE and enqueue nothing.  The tensor-core path needs only
 *   256 + 8 (n_seqs + 1) + 4 (ceil(B*T / chunk) + n_seqs) bytes (with gdn2 another 74240
 *   bytes per chunk and value head); the CUDA-core path
 *   additionally 4 B*T Hv (dk + dv + 1) bytes (4 B*T Hv (2 dk + dv) with gdn2), and for
 *   chunk <= 64 with dk a multiple of 32 up to 128 another 8 B*T Hv dk +
 *   4 (ceil(B*T / chunk) + n_seqs) Hv chunk^2 bytes, so it fits only small problems.
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *   with that device current; make that first call before any stream capture.
 * - All calls on a device share the one array: calls that overlap on the GPU (different
 *   streams, or different host threads, without ordering between them) race and may
 *   corrupt each other's results.  Each call rewrites every scratch field it reads, so a
 *   previous call's contents never leak into the next.
 * - The device error word lives in the shared array: read it with
 *   gdr_noalloc_read_device_error (which synchronises), or give args->status a device word
 *   of the caller's to have it set without a synchronisation.
 * - The array's address is cached per device and CUDA context; a call made after the
 *   device's primary context was reset (cudaDeviceReset) looks it up again.
 * - Arguments that are valid but have no kernel path return GDR_ERR_UNSUPPORTED, invalid
 *   ones the status gdr_chunk_fwd would return; neither enqueues anything.
 */
#define GDR_NOALLOC_SCRATCH_BYTES (4u << 20)
gdr_status gdr_chunk_fwd_noalloc(const gdr_chunk_args* args,
                                 const void* q, const void* k, const void* v,
                                 const void* g, const void* beta,
                                 const float* S0, const int32_t* cu_seqlens,
                                 void* o, float* S_final, void* stream);

/* Test/diagnostic helper for gdr_chunk_fwd_noalloc, NOT for the hot path: copies the device
 * error word out of the static scratch array of the current device (as the last
 * gdr_chunk_fwd_noalloc call on `stream` left it), SYNCHRONISES `stream`, and returns GDR_OK
 * or the recorded device-side status. */
gdr_status gdr_noalloc_read_device_error(void* stream);

/* Name of the kernel path gdr_chunk_fwd takes for these arguments: "tc" (tcgen05
 * tensor-core kernels), "simt" (fp32 CUDA-core kernels) or NULL if unsupported. */
const char* gdr_chunk_fwd_path(const gdr_chunk_args* args);

/*
 * Bidirectional forward (Rondo-Exp tiny_gdn/fugue.py, the bidirectional token mixer): one
 * forward scan with (g_fwd, beta_fwd) and one scan over each sequence's tokens in reverse
 * order with (g_bwd, beta_bwd), both from a zero state with the same q, k, v, read mode and
 * scale, their outputs summed into o:  o = o_fwd + o_bwd  (o_bwd at each token's own
 * position).  No state is returned.
 *
 *   args        as for gdr_chunk_fwd, with reverse = 0 and o_accumulate = 0
 *   g_*, beta_* [B, T, Hv] gate_dtype, or the raw projections with gate_raw (both
 *               directions share gate_A, gate_dt_bias, beta_scale); GDN-2 layouts with gdn2
 *               (both directions share gdn2_w)
 *   o           [B, T, Hv, dv] io_dtype; on the tensor-core path the two directions are
 *               summed in fp32 and the sum rounded once (two gdr_chunk_fwd calls, the second
 *               with reverse and o_accumulate, round each direction first)
 *   workspace   at least gdr_chunk_fwd_bidir_workspace_size(args) bytes, 256-byte aligned
 *
 * On the tensor-core path one grid runs both scans: the two scans of a (sequence, head) are
 * the two CTAs of a thread-block cluster.  The reverse scan's 64-token chunks are aligned
 * with the forward scan's (its first chunk holds the sequence's last T mod 64 tokens), so
 * both produce the output of the same 64 tokens per chunk; the scan that gets to a chunk
 * first leaves its fp32 output there in the workspace, and the other adds it to its own and
 * writes o.  The two CTAs read the same q, k, v tiles within one residency, so the second
 * read is served mostly from L2.  The CUDA-core path runs the reverse scan after the forward
 * one, accumulating into o.  Errors: as gdr_chunk_fwd.
 */
size_t gdr_chunk_fwd_bidir_workspace_size(const gdr_chunk_args* args);
gdr_status gdr_chunk_fwd_bidir(const gdr_chunk_args* args,
                               const void* q, const void* k, const void* v,
                               const void* g_fwd, const void* beta_fwd,
                               const void* g_bwd, const void* beta_bwd,
                               const int32_t* cu_seqlens, void* o,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass of gdr_chunk_fwd: the gradients of
 *     L = <dO, o> + <dS_final, S_final>
 * with respect to q, k, v, g, beta and S0, for the same arguments (Prizma "seq/delta.py",
 * module docstring: the chunk-parallel form agrees with the per-token recurrence on the
 * forward and on the gradients; the gradient is the per-token recurrence's).  The forward's
 * intermediate values are recomputed from the inputs; nothing from a forward call is kept.
 *
 *   args        as for gdr_chunk_fwd, with gate_raw = 0, gdn2 = 0, o_accumulate = 0;
 *               kernels: chunk in {16, 32, 64}, dk <= 128, dv a multiple of 32 up to 128
 *   q .. cu_seqlens   the forward's inputs, layouts as for gdr_chunk_fwd
 *   dO          [B, T, Hv, dv]   io_dtype, gradient of o
 *   dS_final    [n_seqs, Hv, dk, dv] fp32 gradient of S_final, or NULL for zero
 *   dq, dk      [B, T, Hk, dk]   io_dtype outputs (summed over the v-heads of a key head)
 *   dv          [B, T, Hv, dv]   io_dtype output
 *   dg, dbeta   [B, T, Hv]       gate_dtype outputs (dg is the gradient of g = log alpha)
 *   dS0         [n_seqs, Hv, dk, dv] fp32 output, or NULL
 *   workspace   device scratch of at least gdr_chunk_bwd_workspace_size(args) bytes,
 *               256-byte aligned, no initialisation needed
 *
 * Kernels.  bf16, dk = dv = 128, chunk 64 ("tc"): the tensor-core forward kernel runs twice,
 * once leaving the in-chunk decay, the state at every chunk start and V', once as the adjoint
 * recurrence from dS_final back to dS0 (dH+ at every chunk, dV'); two per-(chunk, head)
 * tcgen05 kernels then form dq, dk, dv, dg and dbeta, the second forming W and U~ again from
 * its own solve.  With one v-head per key head they write dq and dk themselves; otherwise a
 * last kernel sums them over each key head's v-heads.  Their operands are fp16, each row
 * (or tile) scaled by a power of two; an fp16 operand of the recurrences that leaves its range
 * (|dO| or a gradient of the state beyond 65504) is reported as GDR_ERR_RANGE through the
 * workspace, as in gdr_chunk_fwd.  Other sizes and fp32 ("simt"): fp32 CUDA-core kernels.
 *
 * Outputs are written, never accumulated.  Errors: as gdr_chunk_fwd; GDR_ERR_UNSUPPORTED
 * for sizes or options outside the kernels' range.
 */
size_t gdr_chunk_bwd_workspace_size(const gdr_chunk_args* args);
gdr_status gdr_chunk_bwd(const gdr_chunk_args* args,
                         const void* q, const void* k, const void* v,
                         const void* g, const void* beta,
                         const float* S0, const int32_t* cu_seqlens,
                         const void* dO, const float* dS_final,
                         void* dq, void* dk, void* dv, void* dg, void* dbeta, float* dS0,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Name of the kernel path gdr_chunk_bwd takes for these arguments: "tc" (tcgen05
 * tensor-core kernels), "simt" (fp32 CUDA-core kernels) or NULL if unsupported. */
const char* gdr_chunk_bwd_path(const gdr_chunk_args* args);

/*
 * One-token recurrent decode step (flashrt fused_layer.py `_decode_one`, the
 * recurrent core that reads and writes the cached state once per token).
 */
typedef struct {
    int N;                 /* independent sequences, one token each */
    int Hk, Hv, dk, dv;    /* as in gdr_chunk_args; GPU kernel: dk in {32,64,128},
                              dv a multiple of 32 up to 128 */
    gdr_dtype io_dtype, gate_dtype;
    gdr_read_mode read_mode;
    float scale;
    int qk_l2norm;
    int gate_raw;               /* fused gating prologue, exactly as in gdr_chunk_args */
    const float* gate_A;
    const float* gate_dt_bias;
    float beta_scale;
    /* Fused output epilogue of the decode chain (flashrt fused_layer.py `_decode_one`:
     * rms_norm_gated_silu(core_out, z, norm.weight, eps) applied per head to the
     * recurrent core's output).
     *   out_norm = 0: o is the recurrent output itself; the three fields below are unused.
     *   out_norm = 1: o_j = c_j / sqrt(mean_j(c_j^2) + norm_eps) * norm_weight[j] * silu(z_j)
     *                 per (sequence, head), c the recurrent output in fp32, the mean over the
     *                 dv values of the head, silu(x) = x / (1 + e^-x). */
    int out_norm;
    const void* norm_z;         /* [N, Hv, dv] io_dtype; 16-byte aligned; required when
                                   out_norm */
    const float* norm_weight;   /* [dv] fp32, shared by the heads; 4-byte aligned; required
                                   when out_norm */
    float norm_eps;             /* >= 0, finite */
    /* GDN-2 decoupled gates (tiny_gdn/fugue.py BidirectionalGatedDeltaNet2:
     * S_t = (I - k_t (b_t * k_t)^T) Diag(exp g_t) S_{t-1} + k_t (w_t * v_t)^T).
     *   gdn2 = 0: scalar gates, g and beta of one value per token and value head.
     *   gdn2 = 1: g is the per-key-channel log decay [N, Hv, dk], beta the per-key-channel
     *             erase gate b [N, Hv, dk], and gdn2_w the per-value-channel write gate
     *             [N, Hv, dv], all gate_dtype and 16-byte aligned.  With g = log(alpha),
     *             b = w = beta on every channel this is the scalar rule.  Not combined with
     *             gate_raw. */
    int gdn2;
    const void* gdn2_w;
} gdr_decode_args;

/*
 *   q, k     [N, Hk, dk]  io_dtype      v, o  [N, Hv, dv]  io_dtype
 *   g, beta  [N, Hv]      gate_dtype
 *   S_inout  [N, Hv, dk, dv] fp32, updated in place: every block reads its whole slice
 *            of the state into registers before it writes any of it back, so no scratch
 *            state is needed.
 */
gdr_status gdr_decode_step(const gdr_decode_args* args,
                           const void* q, const void* k, const void* v,
                           const void* g, const void* beta,
                           float* S_inout, void* o, void* stream);

/* Human-readable name of a status. */
const char* gdr_status_string(gdr_status status);

/* Test/diagnostic helper, NOT for the hot path: copies the device error word out of a
 * workspace last used by gdr_chunk_fwd with `args`, SYNCHRONISES `stream`, and returns
 * GDR_OK or the recorded device-side status. */
gdr_status gdr_read_device_error(const gdr_chunk_args* args, const void* workspace,
                                 void* stream);

/* Library version string (also names the target architecture). */
const char* gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
