// Placeholder until the tcgen05 kernels land: reports the tensor-core path as
// unavailable so that lcp_step uses the CUDA-core kernels.
#include "lcp_internal.cuh"

namespace lcp {
bool tc_available() { return false; }
static lcp_status none(const char* w) { return fail(LCP_ERR_ARG, "%s: tensor-core path not built", w); }
lcp_status launch_permute_mask_tc(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                  const __nv_bfloat16*, uint32_t*, __nv_bfloat16*, float*, int, int,
                                  int, int, int, cudaStream_t) { return none("permute_mask_tc"); }
lcp_status launch_calib_gemm_tc(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                float*, float*, int, int, int, cudaStream_t) { return none("calib_gemm_tc"); }
lcp_status launch_bwd_gemm_tc(const __nv_bfloat16*, const __nv_bfloat16*, __nv_bfloat16*, int, int,
                              int, cudaStream_t) { return none("bwd_gemm_tc"); }
lcp_status launch_block_bwd_tc(const __nv_bfloat16*, const __nv_bfloat16*, const uint32_t*,
                               const __nv_bfloat16*, const __nv_bfloat16*, float*, int, int, int,
                               int, cudaStream_t) { return none("block_bwd_tc"); }
int block_bwd_tc_splits(int, int, int) { return 1; }
}  // namespace lcp
