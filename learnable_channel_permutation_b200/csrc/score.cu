// Importance scores S of the weights (PermLLM summary, "integration with
// existing pruning methods": for an importance matrix S the mask is taken from
// S_hat = S P_B).  The pages name the one-shot metrics Wanda and RIA without
// defining them; their published definitions are used:
//   magnitude  S_ij = |W_ij|
//   Wanda      S_ij = |W_ij| ||X_j||
//   RIA        S_ij = (|W_ij| / sum_k |W_kj| + |W_ij| / sum_k |W_ik|) ||X_j||^(1/2)
// with ||X_j|| the 2-norm of input channel j over the T calibration tokens.
//
// Three passes over HBM-resident data: channel norms of X (one thread per
// column, rows walked in order), row and column sums of |W| (RIA only), then
// the elementwise score, stored in the element type of W.

#include "lcp_internal.cuh"

namespace lcp {
namespace {

#define LCP_TRY_LAUNCH(x)              \
  do {                                 \
    const lcp_status s_ = (x);         \
    if (s_ != LCP_OK) return s_;       \
  } while (0)

// ||X_j||^2 accumulated in float32 over the tokens in order; one thread per column
template <typename T>
__global__ void __launch_bounds__(256)
colnorm_kernel(const T* __restrict__ X, float* __restrict__ norm, int tokens, int cin) {
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= cin) return;
  float s = 0.f;
  for (int t = 0; t < tokens; ++t) {
    const float x = to_f32(X[(size_t)t * cin + j]);
    s = fmaf(x, x, s);
  }
  norm[j] = sqrtf(s);
}

// row sums of |W| (one warp per row, lanes over the columns, fixed-order tree)
template <typename T>
__global__ void __launch_bounds__(256)
rowsum_kernel(const T* __restrict__ W, float* __restrict__ rows, int cout, int cin) {
  const int r = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (r >= cout) return;
  float s = 0.f;
  for (int j = lane; j < cin; j += 32) s += fabsf(to_f32(W[(size_t)r * cin + j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) rows[r] = s;
}

// column sums of |W| (one thread per column, rows in order)
template <typename T>
__global__ void __launch_bounds__(256)
colsum_kernel(const T* __restrict__ W, float* __restrict__ cols, int cout, int cin) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= cin) return;
  float s = 0.f;
  for (int r = 0; r < cout; ++r) s += fabsf(to_f32(W[(size_t)r * cin + j]));
  cols[j] = s;
}

template <typename T>
__global__ void __launch_bounds__(256)
score_kernel(const T* __restrict__ W, const float* __restrict__ xnorm, const float* __restrict__ rows,
             const float* __restrict__ cols, T* __restrict__ S, int cout, int cin, int kind) {
  const long long n = (long long)cout * cin;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(q / cin), j = (int)(q % cin);
    const float a = fabsf(to_f32(W[q]));
    float s;
    if (kind == LCP_SCORE_WANDA) s = a * xnorm[j];
    else if (kind == LCP_SCORE_RIA) s = (a / cols[j] + a / rows[i]) * sqrtf(xnorm[j]);
    else s = a;
    S[q] = from_f32<T>(s);
  }
}

template <typename T>
lcp_status score_t(const T* W, const T* X, T* S, float* stats, int cout, int cin, int tokens, int kind,
                   cudaStream_t st) {
  float* xnorm = stats;
  float* cols = stats + cin;
  float* rows = stats + 2 * cin;
  const unsigned gc = (unsigned)((cin + 255) / 256);
  LCP_TRY_LAUNCH(launch_kernel(colnorm_kernel<T>, dim3(gc), dim3(256), 0, st, 1, true, "score colnorm", X, xnorm,
                               tokens, cin));
  if (kind == LCP_SCORE_RIA) {
    LCP_TRY_LAUNCH(launch_kernel(colsum_kernel<T>, dim3(gc), dim3(256), 0, st, 1, false, "score colsum", W, cols,
                                 cout, cin));
    LCP_TRY_LAUNCH(launch_kernel(rowsum_kernel<T>, dim3((unsigned)((cout + 7) / 8)), dim3(256), 0, st, 1, false,
                                 "score rowsum", W, rows, cout, cin));
  }
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long n = (long long)cout * cin;
  long long grid = (n + 255) / 256;
  if (grid > 16LL * sms) grid = 16LL * sms;
  return launch_kernel(score_kernel<T>, dim3((unsigned)grid), dim3(256), 0, st, 1, false, "score", W, xnorm, rows,
                       cols, S, cout, cin, kind);
}

}  // namespace

lcp_status launch_score(const void* W, const void* X, void* S, float* stats, int cout, int cin, int tokens, int kind,
                        lcp_dtype dt, cudaStream_t st) {
  if (dt == LCP_F32)
    return score_t(static_cast<const float*>(W), static_cast<const float*>(X), static_cast<float*>(S), stats, cout,
                   cin, tokens, kind, st);
  return score_t(static_cast<const __nv_bfloat16*>(W), static_cast<const __nv_bfloat16*>(X),
                 static_cast<__nv_bfloat16*>(S), stats, cout, cin, tokens, kind, st);
}

}  // namespace lcp
