// AdamW update of the logits (PermLLM summary, "Implementation details": the
// logits are trained with AdamW).  Decoupled weight decay as in Loshchilov &
// Hutter's AdamW, bias-corrected moments:
//
//   m <- b1 m + (1 - b1) g          v <- b2 v + (1 - b2) g^2
//   L <- L (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v / (1 - b2^t)) + eps)
//
// with g = dL and t the 1-based step count.  One pass over four float32
// arrays of the same length, 16-byte vectors, grid-stride.

#include <cmath>

#include "lcp_internal.cuh"

namespace lcp {
namespace {

struct AdamCoef {
  float b1, b2, c1, c2, eps, decay;   // c = 1 - b (formed in double), decay = 1 - lr wd
  float step;                 // lr / (1 - b1^t)
  float inv_sqrt_bc2;         // 1 / sqrt(1 - b2^t)
};

__device__ __forceinline__ void adam1(float& L, float g, float& m, float& v, const AdamCoef& c) {
  m = c.b1 * m + c.c1 * g;
  v = c.b2 * v + c.c2 * g * g;
  L = L * c.decay - c.step * m / (sqrtf(v) * c.inv_sqrt_bc2 + c.eps);
}

__global__ void __launch_bounds__(256)
adamw_kernel(float* __restrict__ L, const float* __restrict__ dL, float* __restrict__ m, float* __restrict__ v,
             long long quads, AdamCoef c) {
  pdl_wait();
  pdl_trigger();
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < quads;
       q += (long long)gridDim.x * blockDim.x) {
    float4 l = reinterpret_cast<float4*>(L)[q];
    const float4 g = reinterpret_cast<const float4*>(dL)[q];
    float4 mm = reinterpret_cast<float4*>(m)[q];
    float4 vv = reinterpret_cast<float4*>(v)[q];
    adam1(l.x, g.x, mm.x, vv.x, c);
    adam1(l.y, g.y, mm.y, vv.y, c);
    adam1(l.z, g.z, mm.z, vv.z, c);
    adam1(l.w, g.w, mm.w, vv.w, c);
    reinterpret_cast<float4*>(L)[q] = l;
    reinterpret_cast<float4*>(m)[q] = mm;
    reinterpret_cast<float4*>(v)[q] = vv;
  }
}

}  // namespace

lcp_status launch_adamw(float* L, const float* dL, float* m, float* v, long long n, double lr, double beta1,
                        double beta2, double eps, double weight_decay, int t, cudaStream_t st) {
  if (n == 0) return LCP_OK;
  // every coefficient in double, rounded once
  const double bc1 = 1.0 - std::pow(beta1, (double)t);
  const double bc2 = 1.0 - std::pow(beta2, (double)t);
  AdamCoef c;
  c.b1 = (float)beta1;
  c.b2 = (float)beta2;
  c.c1 = (float)(1.0 - beta1);
  c.c2 = (float)(1.0 - beta2);
  c.eps = (float)eps;
  c.decay = (float)(1.0 - lr * weight_decay);
  c.step = (float)(lr / bc1);
  c.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  const long long quads = n / 4;
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long grid = (quads + 255) / 256;
  if (grid > 8LL * sms) grid = 8LL * sms;
  return launch_kernel(adamw_kernel, dim3((unsigned)grid), dim3(256), 0, st, 1, true, "adamw", L, dL, m, v, quads, c);
}

}  // namespace lcp
