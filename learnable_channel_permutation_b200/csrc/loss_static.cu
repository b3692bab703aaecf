// lcp_loss_fwd_static: the token-averaged cosine loss with no device memory
// allocated by anyone.
//
// lcp_loss_fwd needs a caller-provided scratch buffer of 4 floats per token
// (the per-token dot product, squared norms and cosine).  Some callers cannot
// provide one: embedders whose device memory is owned by another allocator or
// reserved up front under a fixed budget, and latency-critical pipelines that
// must not call cudaMalloc because its implicit device synchronisation would
// stall work running on other streams.  This entry point keeps that scratch in
// a file-scope __device__ array instead: every GPU that loads the library holds
// LCP_STATIC_MAX_TOKENS * 16 bytes of it until the process exits.
//
// Host code cannot use the array's name as a device address (in host code it
// names a host-side shadow).  The device address is obtained with
// cudaGetSymbolAddress, with the device current, by the first call made on a
// device, and cached together with the unique ID of the CUDA context it
// belongs to; a call that finds another context current (after
// cudaDeviceReset, for example) repeats the lookup instead of launching with a
// stale address.  Make the first call on a device before any stream capture
// begins.
//
// Every call shares the one array.  The token kernel writes all 4 * tokens
// floats before the reduction reads them, so nothing has to start at zero and
// the previous call's contents never leak into a result; but calls whose
// kernels overlap on the GPU (different streams, no ordering between them)
// race on the array and must not be issued.

#include <cuda.h>
#include <mutex>

#include "lcp_internal.cuh"

static __device__ __align__(256) float g_lcp_static_loss_stats[LCP_STATIC_MAX_TOKENS * 4];

namespace lcp {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
float* g_static_ptr[kMaxDevices] = {};
unsigned long long g_static_ctx[kMaxDevices] = {};   // context ID the cached address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F> F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();   // our own lookup's error
    return nullptr;
  }
  return reinterpret_cast<F>(p);
}

// Unique ID of the calling thread's current CUDA context, 0 when there is none
// yet or the driver cannot tell.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

lcp_status static_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices) return fail(LCP_ERR_ARG, "device ordinal %d is out of range", dev);
  std::lock_guard<std::mutex> lk(g_static_mu);
  const unsigned long long ctx = current_ctx_id();
  if (!g_static_ptr[dev] || ctx == 0 || ctx != g_static_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lcp_static_loss_stats);   // set-up: also makes the context current
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return fail(LCP_ERR_CUDA, "cudaGetSymbolAddress of the static loss scratch on device %d: %s", dev,
                  cudaGetErrorString(e));
    }
    g_static_ptr[dev] = static_cast<float*>(p);
    g_static_ctx[dev] = current_ctx_id();
  }
  *out = g_static_ptr[dev];
  return LCP_OK;
}

}  // namespace
}  // namespace lcp

extern "C" lcp_status lcp_loss_fwd_static(const float* Yd, const float* Ys, float* loss, int cout,
                                          int tokens, cudaStream_t stream) {
  using namespace lcp;
  if (!Yd || !Ys || !loss) return fail(LCP_ERR_NULL, "Yd, Ys and loss are required");
  if (cout < 8 || cout % 8 || cout > (1 << 24))
    return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8", cout);
  if (tokens < 1) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  if (tokens > LCP_STATIC_MAX_TOKENS)
    return fail(LCP_ERR_SHAPE,
                "T = %d exceeds LCP_STATIC_MAX_TOKENS = %d, the size of the static scratch of "
                "lcp_loss_fwd_static; use lcp_loss_fwd with a caller-provided buffer",
                tokens, LCP_STATIC_MAX_TOKENS);
  if (((uintptr_t)Yd & 15u) || ((uintptr_t)Ys & 15u))
    return fail(LCP_ERR_ARG, "Yd and Ys must be 16-byte aligned");
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "cannot query the current device");
  }
  if (major != 10 || minor != 0)
    return fail(LCP_ERR_ARCH, "device %d is sm_%d%d, this library is built for sm_100a", dev, major, minor);
  const lcp_status s0 = check_pending();
  if (s0 != LCP_OK) return s0;
  float* stats = nullptr;
  const lcp_status s = static_scratch(&stats);
  if (s != LCP_OK) return s;
  const lcp_status s1 = launch_loss_token(Yd, Ys, stats, nullptr, LCP_F32, cout, tokens, tokens, stream);
  if (s1 != LCP_OK) return s1;
  return launch_loss_reduce(stats, loss, tokens, tokens, stream);
}
