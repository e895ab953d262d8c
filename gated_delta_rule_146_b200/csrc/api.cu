// api.cu -- the C ABI declared in include/gdr.h: host-side validation and dispatch.
//
// Nothing here allocates device memory, synchronises (except the diagnostic
// gdr_read_device_error) or keeps state between calls; every entry point only
// checks its arguments and enqueues kernels on the caller's stream.
#include <cmath>
#include <cstring>

#include "chunk_tc.cuh"
#include "common.cuh"

namespace gdr {
bool bwd_tc_path(const gdr_chunk_args& a);  // chunk_bwd.cu
bool tc_g2_supported(const gdr_chunk_args& a);
gdr_status launch_chunk_g2_tc(const gdr_chunk_args& a, const void* q, const void* k, const void* v,
                              const void* g, const void* b, const float* S0, void* o,
                              float* S_final, void* ws, const WsLayout& L, cudaStream_t st);
}  // namespace gdr

using namespace gdr;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(gdr_dtype d) { return d == GDR_F32 || d == GDR_BF16; }

// Fused gating fields: flags, the scale, and (for a call) the per-head arrays.
template <typename Args>
gdr_status check_gating(const Args* a, bool pointers) {
    if ((a->gate_raw | a->gdn2) & ~1) return GDR_ERR_INVALID_ARG;
    if (a->gdn2) {
        if (a->gate_raw) return GDR_ERR_INVALID_ARG;  // the decoupled gates come as they are
        if (pointers && !a->gdn2_w) return GDR_ERR_INVALID_ARG;
        if (pointers && !aligned16(a->gdn2_w)) return GDR_ERR_ALIGNMENT;
        return GDR_OK;
    }
    if (!a->gate_raw) return GDR_OK;
    if (!std::isfinite(a->beta_scale)) return GDR_ERR_INVALID_ARG;
    if (pointers) {
        if (!a->gate_A || !a->gate_dt_bias) return GDR_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(a->gate_A) | reinterpret_cast<uintptr_t>(a->gate_dt_bias)) & 3u)
            return GDR_ERR_ALIGNMENT;
    }
    return GDR_OK;
}

// Shape/enum validation shared by workspace_size, path and chunk_fwd.
gdr_status check_chunk_args(const gdr_chunk_args* a) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->B < 1 || a->T < 0 || a->Hk < 1 || a->Hv < 1 || a->Hv % a->Hk != 0)
        return GDR_ERR_INVALID_ARG;
    if (a->dk < 1 || a->dv < 1 || a->n_seqs < 1) return GDR_ERR_INVALID_ARG;
    if (a->chunk != 16 && a->chunk != 32 && a->chunk != 64 && a->chunk != 128)
        return GDR_ERR_INVALID_ARG;
    if (!valid_dtype(a->io_dtype) || !valid_dtype(a->gate_dtype)) return GDR_ERR_INVALID_ARG;
    if (a->read_mode != GDR_READ_POST && a->read_mode != GDR_READ_PRE) return GDR_ERR_INVALID_ARG;
    if ((a->qk_l2norm | a->reverse | a->o_accumulate) & ~1) return GDR_ERR_INVALID_ARG;
    if (check_gating(a, false) != GDR_OK) return GDR_ERR_INVALID_ARG;
    const long long T_tot = (long long)a->B * a->T;
    if (T_tot * a->Hv * (a->dk > a->dv ? a->dk : a->dv) >= (1LL << 40)) return GDR_ERR_INVALID_ARG;
    if (T_tot > 0x7fffffffLL || (long long)a->n_seqs * a->Hv > 0x7fffffffLL)
        return GDR_ERR_INVALID_ARG;
    if (a->Hv > 65535) return GDR_ERR_UNSUPPORTED;
    return GDR_OK;
}

// The caller's optional device status word: 4-byte aligned when given.
gdr_status check_status_word(const gdr_chunk_args* a) {
    return (reinterpret_cast<uintptr_t>(a->status) & 3u) ? GDR_ERR_ALIGNMENT : GDR_OK;
}

// Copies a device-side status recorded in the workspace header into the caller's status
// word, unless that word already holds an error.  Enqueued after a call's last kernel, so
// it sees everything the call recorded.
__global__ void publish_status_kernel(const WsHeader* __restrict__ hdr, int* __restrict__ status) {
    const int e = hdr->err;
    if (e != GDR_OK) atomicCAS(status, (int)GDR_OK, e);
}

gdr_status publish_status(const gdr_chunk_args& a, const void* ws, cudaStream_t s) {
    if (!a.status) return GDR_OK;
    publish_status_kernel<<<1, 1, 0, s>>>(reinterpret_cast<const WsHeader*>(ws), a.status);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

enum class Path { None, Tc, TcG2, Simt };

Path choose_path(const gdr_chunk_args& a) {
    if (tc_supported(a)) return Path::Tc;
    if (tc_g2_supported(a)) return Path::TcG2;
    if (simt_supported(a)) return Path::Simt;
    return Path::None;
}

// The bidirectional call: GDN-2 gates take the CUDA-core scans (the tensor-core GDN-2 path
// runs forward scans only).
Path bidir_path(const gdr_chunk_args& a) {
    const Path p = choose_path(a);
    return p == Path::TcG2 ? Path::Simt : p;
}

}  // namespace

namespace gdr {
// Host-side status of a forward call's arguments alone: what gdr_chunk_fwd would return
// before looking at pointers, or GDR_ERR_UNSUPPORTED when no kernel path takes them.
gdr_status chunk_args_status(const gdr_chunk_args* a) {
    const gdr_status st = check_chunk_args(a);
    if (st != GDR_OK) return st;
    return choose_path(*a) == Path::None ? GDR_ERR_UNSUPPORTED : GDR_OK;
}
}  // namespace gdr

extern "C" {

size_t gdr_chunk_fwd_workspace_size(const gdr_chunk_args* a) {
    if (check_chunk_args(a) != GDR_OK) return 0;
    const Path path = choose_path(*a);
    if (path == Path::None) return 0;
    return ws_layout(*a, path == Path::Simt).total;
}

const char* gdr_chunk_fwd_path(const gdr_chunk_args* a) {
    if (check_chunk_args(a) != GDR_OK) return nullptr;
    switch (choose_path(*a)) {
        case Path::Tc: return "tc";
        case Path::TcG2: return "tc";
        case Path::Simt: return "simt";
        default: return nullptr;
    }
}

gdr_status gdr_chunk_fwd(const gdr_chunk_args* a, const void* q, const void* k, const void* v,
                         const void* g, const void* beta, const float* S0,
                         const int32_t* cu_seqlens, void* o, float* S_final, void* workspace,
                         size_t workspace_bytes, void* stream) {
    gdr_status st = check_chunk_args(a);
    if (st != GDR_OK) return st;
    if (cu_seqlens) {
        if (a->B != 1) return GDR_ERR_INVALID_ARG;
    } else if (a->n_seqs != a->B) {
        return GDR_ERR_INVALID_ARG;
    }
    const bool has_tokens = (long long)a->B * a->T > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !o)) return GDR_ERR_INVALID_ARG;
    if ((st = check_gating(a, true)) != GDR_OK) return st;
    if ((st = check_status_word(a)) != GDR_OK) return st;
    if (!workspace) return GDR_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, v, g, beta, S0, cu_seqlens, o, S_final, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDR_ERR_ALIGNMENT;
    const Path path = choose_path(*a);
    if (path == Path::None) return GDR_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(*a, path == Path::Simt);
    if (workspace_bytes < L.total) return GDR_ERR_WORKSPACE;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_plan(*a, cu_seqlens, workspace, L, s) != cudaSuccess) return GDR_ERR_CUDA;
    st = path == Path::Tc     ? launch_chunk_tc(*a, q, k, v, g, beta, S0, o, S_final, workspace, L, s)
         : path == Path::TcG2 ? launch_chunk_g2_tc(*a, q, k, v, g, beta, S0, o, S_final, workspace, L, s)
                              : launch_chunk_simt(*a, q, k, v, g, beta, S0, o, S_final, workspace, L, s);
    if (st != GDR_OK) return st;
    return publish_status(*a, workspace, s);
}


// Bidirectional forward: the plan, then the two scans.  On the tensor-core path both run in
// one grid, the two scans of a (sequence, head) as a cluster pair that sums the two outputs
// of every chunk in fp32 through the workspace (one fp32 [64][head size] tile per chunk and
// head) and rounds once; the CUDA-core path runs the reverse scan after the forward one and
// accumulates into o.
namespace {
size_t bidir_scratch_offset(const gdr_chunk_args& a, Path path) {
    return align_up(ws_layout(a, path == Path::Simt).total, 256);
}
size_t bidir_workspace(const gdr_chunk_args& a, Path path) {
    const size_t base = bidir_scratch_offset(a, path);
    if (path != Path::Tc) return base;
    const WsLayout L = ws_layout(a, false);
    return align_up(base + sizeof(float) * (size_t)L.max_chunks * a.Hv * a.chunk * a.dv, 256);
}
}  // namespace

size_t gdr_chunk_fwd_bidir_workspace_size(const gdr_chunk_args* a) {
    if (check_chunk_args(a) != GDR_OK || a->reverse || a->o_accumulate) return 0;
    const Path path = bidir_path(*a);
    if (path == Path::None) return 0;
    return bidir_workspace(*a, path);
}

gdr_status gdr_chunk_fwd_bidir(const gdr_chunk_args* a, const void* q, const void* k,
                               const void* v, const void* g_fwd, const void* beta_fwd,
                               const void* g_bwd, const void* beta_bwd,
                               const int32_t* cu_seqlens, void* o, void* workspace,
                               size_t workspace_bytes, void* stream) {
    gdr_status st = check_chunk_args(a);
    if (st != GDR_OK) return st;
    if (a->reverse || a->o_accumulate) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (a->B != 1) return GDR_ERR_INVALID_ARG;
    } else if (a->n_seqs != a->B) {
        return GDR_ERR_INVALID_ARG;
    }
    const bool has_tokens = (long long)a->B * a->T > 0;
    if (has_tokens && (!q || !k || !v || !g_fwd || !beta_fwd || !g_bwd || !beta_bwd || !o))
        return GDR_ERR_INVALID_ARG;
    if ((st = check_gating(a, true)) != GDR_OK) return st;
    if ((st = check_status_word(a)) != GDR_OK) return st;
    if (!workspace) return GDR_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, v, g_fwd, beta_fwd, g_bwd, beta_bwd, cu_seqlens, o, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDR_ERR_ALIGNMENT;
    const Path path = bidir_path(*a);
    if (path == Path::None) return GDR_ERR_UNSUPPORTED;
    if (workspace_bytes < bidir_workspace(*a, path)) return GDR_ERR_WORKSPACE;
    const WsLayout L = ws_layout(*a, path == Path::Simt);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_plan(*a, cu_seqlens, workspace, L, s) != cudaSuccess) return GDR_ERR_CUDA;
    gdr_chunk_args rev = *a;
    rev.reverse = 1;
    if (path == Path::Tc) {
        if ((st = launch_chunk_tc(*a, q, k, v, g_fwd, beta_fwd, nullptr, o, nullptr, workspace,
                                  L, s, false, g_bwd, beta_bwd, bidir_scratch_offset(*a, path))) !=
            GDR_OK)
            return st;
        return publish_status(*a, workspace, s);
    }
    if ((st = launch_chunk_simt(*a, q, k, v, g_fwd, beta_fwd, nullptr, o, nullptr, workspace, L,
                                s)) != GDR_OK)
        return st;
    rev.o_accumulate = 1;  // the CUDA-core scan adds the reverse direction into o itself
    if ((st = launch_chunk_simt(rev, q, k, v, g_bwd, beta_bwd, nullptr, o, nullptr, workspace, L,
                                s)) != GDR_OK)
        return st;
    return publish_status(*a, workspace, s);
}

size_t gdr_chunk_bwd_workspace_size(const gdr_chunk_args* a) {
    if (check_chunk_args(a) != GDR_OK || !bwd_supported(*a)) return 0;
    return bwd_layout(*a).total;
}

const char* gdr_chunk_bwd_path(const gdr_chunk_args* a) {
    if (check_chunk_args(a) != GDR_OK || !bwd_supported(*a)) return nullptr;
    return bwd_tc_path(*a) ? "tc" : "simt";
}

gdr_status gdr_chunk_bwd(const gdr_chunk_args* a, const void* q, const void* k, const void* v,
                         const void* g, const void* beta, const float* S0,
                         const int32_t* cu_seqlens, const void* dO, const float* dS_final,
                         void* dq, void* dk, void* dv, void* dg, void* dbeta, float* dS0,
                         void* workspace, size_t workspace_bytes, void* stream) {
    gdr_status st = check_chunk_args(a);
    if (st != GDR_OK) return st;
    if (cu_seqlens) {
        if (a->B != 1) return GDR_ERR_INVALID_ARG;
    } else if (a->n_seqs != a->B) {
        return GDR_ERR_INVALID_ARG;
    }
    if (a->gate_raw || a->gdn2 || a->o_accumulate) return GDR_ERR_UNSUPPORTED;
    const bool has_tokens = (long long)a->B * a->T > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta))
        return GDR_ERR_INVALID_ARG;
    if ((st = check_status_word(a)) != GDR_OK) return st;
    if (!workspace) return GDR_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, v, g, beta, S0, cu_seqlens, dO, dS_final, dq, dk, dv, dg, dbeta,
                          dS0, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDR_ERR_ALIGNMENT;
    if (!bwd_supported(*a)) return GDR_ERR_UNSUPPORTED;
    const BwdLayout B = bwd_layout(*a);
    if (workspace_bytes < B.total) return GDR_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_plan(*a, cu_seqlens, workspace, B.base, s) != cudaSuccess) return GDR_ERR_CUDA;
    const BwdPtrs x{q, k, v, g, beta, dO, S0, dS_final, dq, dk, dv, dg, dbeta, dS0};
    if ((st = launch_chunk_bwd(*a, x, workspace, B, s)) != GDR_OK) return st;
    return publish_status(*a, workspace, s);
}

gdr_status gdr_decode_step(const gdr_decode_args* a, const void* q, const void* k, const void* v,
                           const void* g, const void* beta, float* S_inout, void* o,
                           void* stream) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->N < 0 || a->Hk < 1 || a->Hv < 1 || a->Hv % a->Hk != 0 || a->dk < 1 || a->dv < 1)
        return GDR_ERR_INVALID_ARG;
    if (!valid_dtype(a->io_dtype) || !valid_dtype(a->gate_dtype)) return GDR_ERR_INVALID_ARG;
    if (a->read_mode != GDR_READ_POST && a->read_mode != GDR_READ_PRE) return GDR_ERR_INVALID_ARG;
    if (a->qk_l2norm & ~1) return GDR_ERR_INVALID_ARG;
    if (check_gating(a, false) != GDR_OK) return GDR_ERR_INVALID_ARG;
    if (a->out_norm & ~1) return GDR_ERR_INVALID_ARG;
    if (a->out_norm && !(std::isfinite(a->norm_eps) && a->norm_eps >= 0.f)) return GDR_ERR_INVALID_ARG;
    if ((long long)a->N * a->Hv > 0x7fffffffLL) return GDR_ERR_INVALID_ARG;
    if (!decode_supported(*a)) return GDR_ERR_UNSUPPORTED;
    if (a->N == 0) return GDR_OK;
    if (!q || !k || !v || !g || !beta || !S_inout || !o) return GDR_ERR_INVALID_ARG;
    if (const gdr_status gs = check_gating(a, true); gs != GDR_OK) return gs;
    if (a->out_norm) {
        if (!a->norm_z || !a->norm_weight) return GDR_ERR_INVALID_ARG;
        if (!aligned16(a->norm_z) || (reinterpret_cast<uintptr_t>(a->norm_weight) & 3u))
            return GDR_ERR_ALIGNMENT;
    }
    const void* ptrs[] = {q, k, v, g, beta, S_inout, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGNMENT;
    return launch_decode(*a, q, k, v, g, beta, S_inout, o, static_cast<cudaStream_t>(stream));
}

const char* gdr_status_string(gdr_status s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG: invalid argument";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED: no kernel for these sizes/dtypes";
        case GDR_ERR_ALIGNMENT: return "GDR_ERR_ALIGNMENT: pointer not 16-byte aligned";
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE: workspace missing or too small";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA: kernel launch failed";
        case GDR_ERR_DEVICE_CHECK: return "GDR_ERR_DEVICE_CHECK: device-side check failed (cu_seqlens)";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT: a bounded device wait gave up";
        case GDR_ERR_RANGE: return "GDR_ERR_RANGE: a tensor-core operand left the fp16 range";
    }
    return "unknown gdr_status";
}

gdr_status gdr_read_device_error(const gdr_chunk_args* a, const void* workspace, void* stream) {
    (void)a;
    if (!workspace) return GDR_ERR_INVALID_ARG;
    int err = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDR_ERR_CUDA;
    return static_cast<gdr_status>(err);
}

const char* gdr_version(void) { return "gdr-b200 0.1 (sm_100a)"; }

}  // extern "C"
