// plan.cu -- builds the chunk map of a forward call on the device.
//
// Chunks restart at every sequence start and the last chunk of a sequence may be short
// (Prizma "seq/delta.py", chunked_delta: the chunk loop clips each chunk's end at the
// sequence length; flashrt fused_layer.py, `_prefill_chain`: the same clipping of its
// 64-token spans).  Packed sequences are delimited by cu_seqlens (tiny_gdn/fugue.py
// `segment_layout`).  The map is built without any host synchronisation: grids downstream
// are sized by the upper bound ceil(T_total / chunk) + n_seqs and surplus blocks exit.
// It also holds the order in which per-(sequence, head) kernels visit the sequences:
// longest first for varlen calls, so the long ones do not end up in the last wave.
#include "common.cuh"

namespace gdr {

namespace {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t* __restrict__ cu_in, int n_seqs, int B, int T, int chunk,
            WsHeader* __restrict__ hdr, int32_t* __restrict__ cu, int32_t* __restrict__ chunk_off,
            int32_t* __restrict__ chunk_seq, int32_t* __restrict__ order, long long max_chunks) {
    __shared__ int s_bad;
    __shared__ int s_warp[kPlanThreads / 32];
    __shared__ int s_len[kOrderMaxSeqs];
    const int tid = threadIdx.x;
    if (tid == 0) s_bad = 0;
    __syncthreads();

    const long long T_tot = (long long)B * T;
    // 1. token offsets: copied and validated, or synthesised for B rows of T tokens
    for (int s = tid; s <= n_seqs; s += kPlanThreads) {
        long long val = cu_in ? (long long)cu_in[s] : (long long)s * T;
        cu[s] = (int32_t)val;
        if (cu_in) {
            if (s == 0 && val != 0) s_bad = 1;
            if (s == n_seqs && val != T_tot) s_bad = 1;
            if (s > 0 && cu_in[s] < cu_in[s - 1]) s_bad = 1;
        }
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) { hdr->err = GDR_ERR_DEVICE_CHECK; hdr->n_chunks = 0; }
        return;
    }

    // 2. chunks per sequence, exclusive scan over a contiguous range per thread
    const int per = (n_seqs + kPlanThreads - 1) / kPlanThreads;
    const int s_lo = min(n_seqs, tid * per), s_hi = min(n_seqs, s_lo + per);
    int local = 0;
    for (int s = s_lo; s < s_hi; ++s) local += (cu[s + 1] - cu[s] + chunk - 1) / chunk;
    // block-wide exclusive scan of `local`
    const int lane = tid & 31, wid = tid >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int run = (wid > 0 ? s_warp[wid - 1] : 0) + incl - local;
    for (int s = s_lo; s < s_hi; ++s) {
        chunk_off[s] = run;
        run += (cu[s + 1] - cu[s] + chunk - 1) / chunk;
    }
    const int total = s_warp[31];
    if (tid == 0) chunk_off[n_seqs] = total;
    __syncthreads();
    // 3. sequence of every chunk: the last sequence whose first chunk is <= c (empty
    //    sequences share their offset with the next non-empty one and lose the tie)
    for (int c = tid; c < total; c += kPlanThreads) {
        int lo = 0, hi = n_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
        }
        chunk_seq[c] = lo;
    }
    // 4. visiting order: by decreasing length, ties by index (a stable rank of each sequence
    //    among all of them), for varlen calls of at most kOrderMaxSeqs sequences
    if (cu_in && n_seqs <= kOrderMaxSeqs) {
        for (int s = tid; s < n_seqs; s += kPlanThreads) s_len[s] = cu[s + 1] - cu[s];
        __syncthreads();
        for (int s = tid; s < n_seqs; s += kPlanThreads) {
            const int ls = s_len[s];
            int rank = 0;
            for (int t = 0; t < n_seqs; ++t) {
                const int lt = s_len[t];
                rank += (lt > ls) | ((lt == ls) & (t < s));
            }
            order[rank] = s;
        }
    } else {
        for (int s = tid; s < n_seqs; s += kPlanThreads) order[s] = s;
    }
    if (tid == 0) {
        hdr->n_chunks = total;
        hdr->err = (total <= max_chunks) ? GDR_OK : GDR_ERR_DEVICE_CHECK;
    }
}

}  // namespace

cudaError_t launch_plan(const gdr_chunk_args& a, const int32_t* cu_in, void* ws, const WsLayout& L,
                        cudaStream_t st) {
    char* base = static_cast<char*>(ws);
    plan_kernel<<<1, kPlanThreads, 0, st>>>(
        cu_in, a.n_seqs, a.B, a.T, a.chunk, reinterpret_cast<WsHeader*>(base),
        reinterpret_cast<int32_t*>(base + L.cu), reinterpret_cast<int32_t*>(base + L.chunk_off),
        reinterpret_cast<int32_t*>(base + L.chunk_seq), reinterpret_cast<int32_t*>(base + L.order),
        L.max_chunks);
    return cudaGetLastError();
}

}  // namespace gdr
