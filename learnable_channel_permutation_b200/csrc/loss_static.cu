// lcp_loss_fwd_static: the token-averaged cosine loss with no device memory
// allocated by anyone.
//
// lcp_loss_fwd needs a caller-provided scratch buffer of 4 floats per token
// (the per-token dot product, squared norms and cosine).  Some callers cannot
// provide one: code that must not call cudaMalloc because it runs while a
// stream is being captured into a CUDA graph or inside a stream-ordered
// pipeline that cudaMalloc's implicit device synchronisation would stall, and
// embedders whose device memory is owned by another allocator or reserved up
// front under a fixed budget.  This entry point keeps that scratch in a
// file-scope __device__ array instead: every GPU that loads the library holds
// LCP_STATIC_MAX_TOKENS * 16 bytes of it until the process exits.
//
// Host code cannot use the array's name as a device address (in host code it
// names a host-side shadow).  The device address is obtained once per device
// with cudaGetSymbolAddress, with that device current, on the first call made
// on that device; make that first call before any stream capture begins.
//
// Every call shares the one array.  The token kernel writes all 4 * tokens
// floats before the reduction reads them, so nothing has to start at zero and
// the previous call's contents never leak into a result; but calls whose
// kernels overlap on the GPU (different streams, no ordering between them)
// race on the array and must not be issued.

#include <mutex>

#include "lcp_internal.cuh"

static __device__ __align__(256) float g_lcp_static_loss_stats[LCP_STATIC_MAX_TOKENS * 4];

namespace lcp {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
float* g_static_ptr[kMaxDevices] = {};

lcp_status static_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices) return fail(LCP_ERR_ARG, "device ordinal %d is out of range", dev);
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lcp_static_loss_stats);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return fail(LCP_ERR_CUDA, "cudaGetSymbolAddress of the static loss scratch on device %d: %s", dev,
                  cudaGetErrorString(e));
    }
    g_static_ptr[dev] = static_cast<float*>(p);
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
  float* stats = nullptr;
  const lcp_status s = static_scratch(&stats);
  if (s != LCP_OK) return s;
  cudaGetLastError();
  const lcp_status s1 = launch_loss_token(Yd, Ys, stats, nullptr, LCP_F32, cout, tokens, stream);
  if (s1 != LCP_OK) return s1;
  return launch_loss_reduce(stats, loss, tokens, stream);
}
