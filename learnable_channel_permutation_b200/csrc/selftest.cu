// Self-test of the bounded waits used by every tensor-core kernel of the
// library: one thread waits on an mbarrier phase that nothing completes.  The
// wait must give up after its time limit, record its site in this unit's error
// word and return, leaving the CUDA context usable.

#include "tc_common.cuh"

namespace lcp {
namespace {

constexpr int kSelftestSite = 901;

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int* completed) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);   // one arrival expected; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) completed[0] = mbar_wait(smem_u32(&bar), 0, &abort_flag, kSelftestSite) ? 1 : 0;
}

}  // namespace
}  // namespace lcp

extern "C" lcp_status lcp_selftest_bounded_wait(int* site) {
  using namespace lcp;
  if (!site) return fail(LCP_ERR_NULL, "site is NULL");
  int* d = nullptr;
  cudaError_t e = cudaMalloc(&d, sizeof(int));
  if (e != cudaSuccess) return fail(LCP_ERR_CUDA, "selftest: cudaMalloc: %s", cudaGetErrorString(e));
  int prev = 0;
  lcp_status s = read_tc_error(&prev, 1);                 // start from a clear word
  if (s == LCP_OK) {
    bounded_wait_selftest_kernel<<<1, 32>>>(d);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    int completed = -1;
    if (e == cudaSuccess) e = cudaMemcpy(&completed, d, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
      s = fail(LCP_ERR_CUDA, "selftest: %s", cudaGetErrorString(e));
    } else {
      s = read_tc_error(site, 1);
      if (s == LCP_OK && completed != 0) s = fail(LCP_ERR_CUDA, "selftest: the wait reported completion");
    }
  }
  cudaFree(d);
  return s;
}
