// chunk_tc.cu -- tcgen05 tensor-core forward (bf16 operands, fp32 state).
#include "common.cuh"

namespace gdr {

bool tc_supported(const gdr_chunk_args& a) { (void)a; return false; }

gdr_status launch_chunk_tc(const gdr_chunk_args& a, const void*, const void*, const void*,
                           const void*, const void*, const float*, void*, float*, void*,
                           const WsLayout&, cudaStream_t) {
    (void)a;
    return GDR_ERR_UNSUPPORTED;
}

}  // namespace gdr
