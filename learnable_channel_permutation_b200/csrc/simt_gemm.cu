// Strided batched GEMM on CUDA cores (float32 accumulation), for the float32
// workloads and for the LCP_FLAG_SIMT path:
//   C[z](m, n) = alpha * sum_k A[z](m, k) B[z](k, n) + beta * C[z](m, n)
// Arbitrary element strides express every transpose the step needs.  64x64
// output tile per CTA, 16-deep k slices staged in shared memory, 4x4 outputs
// per thread.  Operand loads walk the unit-stride dimension across threads.

#include "lcp_internal.cuh"

namespace lcp {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(NT) simt_gemm_kernel(SimtGemm g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int z = blockIdx.z;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const TA* A = static_cast<const TA*>(g.A) + (long long)z * g.sAz;
  const TB* Bm = static_cast<const TB*>(g.B) + (long long)z * g.sBz;
  TC* Cm = static_cast<TC*>(g.C) + (long long)z * g.sCz;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  const bool a_k_fast = (g.sAk == 1);
  const bool b_n_fast = (g.sBn == 1);
  for (int k0 = 0; k0 < g.K; k0 += BK) {
    for (int e = threadIdx.x; e < BM * BK; e += NT) {
      int mm, kk;
      if (a_k_fast) { kk = e % BK; mm = e / BK; } else { mm = e % BM; kk = e / BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < g.M && gk < g.K) ? to_f32(A[gm * g.sAm + gk * g.sAk]) : 0.f;
    }
    for (int e = threadIdx.x; e < BN * BK; e += NT) {
      int nn, kk;
      if (b_n_fast) { nn = e % BN; kk = e / BN; } else { kk = e % BK; nn = e / BK; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < g.N && gk < g.K) ? to_f32(Bm[gk * g.sBk + gn * g.sBn]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= g.N) continue;
      TC* c = Cm + gm * g.sCm + gn * g.sCn;
      float v = g.alpha * acc[i][j];
      if (g.beta != 0.f) v += g.beta * to_f32(*c);
      *c = from_f32<TC>(v);
    }
  }
}

template <typename TA, typename TB>
lcp_status dispatch_c(const SimtGemm& g, lcp_dtype tc, dim3 grid, cudaStream_t st) {
  if (tc == LCP_F32) simt_gemm_kernel<TA, TB, float><<<grid, NT, 0, st>>>(g);
  else simt_gemm_kernel<TA, TB, __nv_bfloat16><<<grid, NT, 0, st>>>(g);
  return check_launch("simt_gemm");
}
template <typename TA>
lcp_status dispatch_b(const SimtGemm& g, lcp_dtype tb, lcp_dtype tc, dim3 grid, cudaStream_t st) {
  if (tb == LCP_F32) return dispatch_c<TA, float>(g, tc, grid, st);
  return dispatch_c<TA, __nv_bfloat16>(g, tc, grid, st);
}

}  // namespace

lcp_status launch_simt_gemm(const SimtGemm& g, lcp_dtype ta, lcp_dtype tb, lcp_dtype tc,
                            cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return LCP_OK;
  const dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM, g.batch);
  if (ta == LCP_F32) return dispatch_b<float>(g, tb, tc, grid, st);
  return dispatch_b<__nv_bfloat16>(g, tb, tc, grid, st);
}

}  // namespace lcp
