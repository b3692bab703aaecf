// N:M magnitude mask (blog page "PermLLM: dynamic channel permutation",
// section 2.1: split each row into groups of M, keep the N largest |w|;
// PermLLM summary, "integration with existing pruning methods": the mask is
// the best N of every group of M consecutive columns kM..(k+1)M-1).
//
// Equal magnitudes keep the lower column first, so the kept set is unique:
// element j of a group is kept iff fewer than N elements rank ahead of it,
// where k ranks ahead of j when |w_k| > |w_j|, or |w_k| == |w_j| and k < j.
//
// Each thread produces one 32-bit output word (32 consecutive columns) from
// 128-bit loads; a warp reads a contiguous 4 KB (fp32) or 2 KB (bf16) span.

#include "lcp_internal.cuh"

namespace lcp {
namespace {

// Each pair k < j is compared once: k ranks ahead of j exactly when
// |a_k| >= |a_j| (ties go to the lower index), otherwise j ranks ahead of k.
template <int M>
__device__ __forceinline__ uint32_t group_bits(const float* a, int n) {
  int ahead[M];
#pragma unroll
  for (int j = 0; j < M; ++j) ahead[j] = 0;
#pragma unroll
  for (int k = 0; k < M; ++k)
#pragma unroll
    for (int j = k + 1; j < M; ++j) {
      const int kj = a[k] >= a[j];
      ahead[j] += kj;
      ahead[k] += 1 - kj;
    }
  uint32_t bits = 0;
#pragma unroll
  for (int j = 0; j < M; ++j) bits |= (ahead[j] < n ? 1u : 0u) << j;
  return bits;
}

template <int M>
__device__ __forceinline__ uint32_t word_bits(const float (&v)[32], int n) {
  uint32_t w = 0;
#pragma unroll
  for (int g = 0; g < 32 / M; ++g) {
    float a[M];
#pragma unroll
    for (int j = 0; j < M; ++j) a[j] = fabsf(v[g * M + j]);
    w |= group_bits<M>(a, n) << (g * M);
  }
  return w;
}

template <typename T, int M>
__global__ void __launch_bounds__(256)
nm_mask_kernel(const T* __restrict__ Wp, uint32_t* __restrict__ bits, long long words, int n) {
  const long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= words) return;
  float v[32];
  if constexpr (sizeof(T) == 4) {
    const float4* src = reinterpret_cast<const float4*>(Wp) + w * 8;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 f = __ldg(src + q);
      v[4 * q + 0] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(Wp) + w * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(src + q);
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[8 * q + 2 * h + 0] = __uint_as_float(p[h] << 16);
        v[8 * q + 2 * h + 1] = __uint_as_float(p[h] & 0xffff0000u);
      }
    }
  }
  if constexpr (M == 4) {
    uint32_t u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(v[i]);
    bits[w] = nm4_keep<32>(u, n);
  } else {
    bits[w] = word_bits<M>(v, n);
  }
}

__global__ void __launch_bounds__(256)
apply_mask_kernel(const float* __restrict__ in, const uint32_t* __restrict__ bits,
                  float* __restrict__ out, long long quads) {
  const long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= quads) return;
  const uint32_t w = __ldg(bits + (q >> 3));
  const int sh = (int)(q & 7) * 4;
  float4 v = reinterpret_cast<const float4*>(in)[q];
  v.x = ((w >> (sh + 0)) & 1u) ? v.x : 0.f;
  v.y = ((w >> (sh + 1)) & 1u) ? v.y : 0.f;
  v.z = ((w >> (sh + 2)) & 1u) ? v.z : 0.f;
  v.w = ((w >> (sh + 3)) & 1u) ? v.w : 0.f;
  reinterpret_cast<float4*>(out)[q] = v;
}

}  // namespace

lcp_status launch_nm_mask(const void* Wp, uint32_t* bits, int rows, int cols, int n, int m,
                          lcp_dtype dt, cudaStream_t st) {
  const long long words = (long long)rows * (cols / 32);
  if (words == 0) return LCP_OK;
  const unsigned grid = (unsigned)((words + 255) / 256);
  if (dt == LCP_F32) {
    if (m == 4) nm_mask_kernel<float, 4><<<grid, 256, 0, st>>>((const float*)Wp, bits, words, n);
    else nm_mask_kernel<float, 8><<<grid, 256, 0, st>>>((const float*)Wp, bits, words, n);
  } else {
    if (m == 4)
      nm_mask_kernel<__nv_bfloat16, 4><<<grid, 256, 0, st>>>((const __nv_bfloat16*)Wp, bits, words, n);
    else
      nm_mask_kernel<__nv_bfloat16, 8><<<grid, 256, 0, st>>>((const __nv_bfloat16*)Wp, bits, words, n);
  }
  return check_launch("nm_mask");
}

lcp_status launch_apply_mask(const float* in, const uint32_t* bits, float* out, int rows,
                             int cols, cudaStream_t st) {
  const long long quads = (long long)rows * cols / 4;
  if (quads == 0) return LCP_OK;
  apply_mask_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, st>>>(in, bits, out, quads);
  return check_launch("apply_mask");
}

}  // namespace lcp
