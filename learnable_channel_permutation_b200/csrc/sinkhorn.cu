// Block-wise log-domain Sinkhorn normalisation, forward and reverse.
//
// PermLLM ("Learnable Channel Permutation for N:M Sparse LLMs"), Method 1:
// S_0(X) = exp(X), S_i(X) = T_c(T_r(S_{i-1}(X))), P = S_L(W_P / tau), applied
// to every B x B diagonal block (Method 3).  The blog page's section 2.2
// gives the log-domain form: subtract each row's log-sum-exp, then each
// column's, `iters` times, then exponentiate.
//
// Every log-domain iterate has the form Z = Z_0 - R_i - C_j, so a row step
// only has to compute R_i = LSE_j(Z_0[i,j] - C_j) and a column step
// C_j = LSE_i(Z_0[i,j] - R_i).  Z_0 = L / tau stays resident in shared
// memory; the (R, C) pair of every iteration is the checkpoint the reverse
// pass replays (2 * iters * B floats per block instead of 2 * iters * B^2).
//
// One CTA owns one block (B <= 128).  For B = 256 the 256 KB fp32 tile does
// not fit one CTA's shared memory, so a cluster of CS CTAs splits the rows;
// column reductions combine per-CTA partials through distributed shared
// memory (fixed rank order, so every CTA gets bit-identical results).
// All reductions run in a fixed order: results are deterministic.

#include <cooperative_groups.h>
#include <math_constants.h>

#include "lcp_internal.cuh"

namespace cg = cooperative_groups;

namespace lcp {
namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int B> struct SkCfg {
  static constexpr int CS = (B == 256) ? 4 : 1;          // CTAs per block (row split)
  static constexpr int NT = (B <= 64) ? 256 : 512;       // threads per CTA
  static constexpr int R = B / CS;                       // rows per CTA
  static constexpr int G = NT / B;                       // row groups of the column pass
  static_assert(NT % B == 0 && R % G == 0, "bad Sinkhorn configuration");
};

template <int CS> __device__ __forceinline__ int cta_rank() {
  if constexpr (CS > 1) return (int)cg::this_cluster().block_rank();
  else return 0;
}
template <int CS> __device__ __forceinline__ void cluster_barrier() {
  if constexpr (CS > 1) cg::this_cluster().sync();
}
template <int CS> __device__ __forceinline__ const float* peer(float* p, int r) {
  if constexpr (CS > 1) return cg::this_cluster().map_shared_rank(p, r);
  else return p;
}

// Forward.  Shared memory (floats): z[R*B] rv[R] cv[B] pm[G*B] ps[G*B] xm[2*B] xs[2*B]
template <int B>
__global__ void __launch_bounds__(SkCfg<B>::NT)
sinkhorn_fwd_kernel(const float* __restrict__ L, float* __restrict__ P, float* __restrict__ ckpt,
                    __nv_bfloat16* __restrict__ pt_hi, __nv_bfloat16* __restrict__ pt_lo,
                    __nv_bfloat16* __restrict__ p_hi, float tau, int iters) {
  using C = SkCfg<B>;
  constexpr int R = C::R, G = C::G, NT = C::NT, NW = NT / 32, CS = C::CS;
  extern __shared__ __align__(16) float sm[];
  float* z = sm;
  float* rv = z + R * B;
  float* cv = rv + R;
  float* pm = cv + B;
  float* ps = pm + G * B;
  float* xm = ps + G * B;   // this CTA's column partials, double-buffered by iteration parity
  float* xs = xm + 2 * B;

  const int rank = cta_rank<CS>();
  const int blk = blockIdx.x / CS;
  const int row0 = rank * R;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const size_t base = (size_t)blk * B * B;

  for (int e = tid; e < R * B; e += NT) z[e] = L[base + (size_t)row0 * B + e] / tau;
  for (int j = tid; j < B; j += NT) cv[j] = 0.f;
  __syncthreads();

  for (int k = 0; k < iters; ++k) {
    // T_r: R_i = LSE_j(z_ij - C_j) -- one warp per row
    for (int r = warp; r < R; r += NW) {
      const float* zr = z + r * B;
      float mx = -CUDART_INF_F;
      for (int j = lane; j < B; j += 32) mx = fmaxf(mx, zr[j] - cv[j]);
      mx = warp_max(mx);
      float s = 0.f;
      for (int j = lane; j < B; j += 32) s += expf(zr[j] - cv[j] - mx);
      s = warp_sum(s);
      if (lane == 0) {
        const float v = mx + logf(s);
        rv[r] = v;
        if (ckpt) ckpt[((size_t)blk * iters + k) * 2 * B + row0 + r] = v;
      }
    }
    __syncthreads();
    // T_c: C_j = LSE_i(z_ij - R_i) over all B rows of the block
    {
      const int j = tid % B, g = tid / B;
      float mx = -CUDART_INF_F;
      for (int r = g; r < R; r += G) mx = fmaxf(mx, z[r * B + j] - rv[r]);
      float s = 0.f;
      for (int r = g; r < R; r += G) s += expf(z[r * B + j] - rv[r] - mx);
      pm[g * B + j] = mx;
      ps[g * B + j] = s;
    }
    __syncthreads();
    float* bm = xm + (k & 1) * B;
    float* bs = xs + (k & 1) * B;
    for (int j = tid; j < B; j += NT) {
      float mx = pm[j];
      for (int g = 1; g < G; ++g) mx = fmaxf(mx, pm[g * B + j]);
      float s = 0.f;
      for (int g = 0; g < G; ++g) s += ps[g * B + j] * expf(pm[g * B + j] - mx);
      bm[j] = mx;
      bs[j] = s;
    }
    cluster_barrier<CS>();
    if constexpr (CS == 1) __syncthreads();
    for (int j = tid; j < B; j += NT) {
      float mx = -CUDART_INF_F;
      for (int q = 0; q < CS; ++q) mx = fmaxf(mx, peer<CS>(bm, q)[j]);
      float s = 0.f;
      for (int q = 0; q < CS; ++q) s += peer<CS>(bs, q)[j] * expf(peer<CS>(bm, q)[j] - mx);
      const float v = mx + logf(s);
      cv[j] = v;
      if (ckpt && rank == 0) ckpt[(((size_t)blk * iters + k) * 2 + 1) * B + j] = v;
    }
    __syncthreads();
  }

  // Operand images for the tensor-core kernels, in tiles of BC = max(B, 64)
  // columns: tile t holds the BC x BC block-diagonal slice of P_B covering
  // channels [t*BC, (t+1)*BC) (for B = 32 two blocks share one tile and the
  // off-diagonal quadrants are written as zeros).
  constexpr int BC = B < 64 ? 64 : B;
  const int gcol0 = blk * B;
  const size_t tbase = (size_t)(gcol0 / BC) * BC * BC;
  const int q0 = gcol0 % BC;
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  for (int e = tid; e < R * B; e += NT) {
    const int r = e / B, j = e % B;
    const float p = expf(z[e] - rv[r] - cv[j]);
    const int i = row0 + r;
    P[base + (size_t)i * B + j] = p;
    if (pt_hi) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(p);
      const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
      pt_hi[tbase + (size_t)(q0 + j) * BC + q0 + i] = hi;
      pt_lo[tbase + (size_t)(q0 + j) * BC + q0 + i] = lo;
      p_hi[tbase + (size_t)(q0 + i) * BC + q0 + j] = hi;
      if constexpr (B < BC) {
        const int zc = (q0 == 0) ? B : 0;
        pt_hi[tbase + (size_t)(q0 + j) * BC + zc + i] = zero;
        pt_lo[tbase + (size_t)(q0 + j) * BC + zc + i] = zero;
        p_hi[tbase + (size_t)(q0 + i) * BC + zc + j] = zero;
      }
    }
  }
  // keep peers' shared memory alive until every CTA of the cluster is done reading it
  cluster_barrier<CS>();
}

// Reverse.  Shared memory (floats): z[R*B] d[R*B] rv[R] ck[B] ck1[B] pm[G*B] xs[2*B]
template <int B>
__global__ void __launch_bounds__(SkCfg<B>::NT)
sinkhorn_bwd_kernel(const float* __restrict__ L, const float* __restrict__ ckpt,
                    const float* __restrict__ dP, int splits, int nblocks,
                    float* __restrict__ dL, float tau, int iters) {
  using C = SkCfg<B>;
  constexpr int R = C::R, G = C::G, NT = C::NT, NW = NT / 32, CS = C::CS;
  extern __shared__ __align__(16) float sm[];
  float* z = sm;
  float* d = z + R * B;
  float* rv = d + R * B;
  float* ck = rv + R;      // C^(k)
  float* ck1 = ck + B;     // C^(k-1)
  float* pm = ck1 + B;
  float* xs = pm + G * B;

  const int rank = cta_rank<CS>();
  const int blk = blockIdx.x / CS;
  const int row0 = rank * R;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const size_t base = (size_t)blk * B * B;
  const size_t split_stride = (size_t)nblocks * B * B;
  const float* ckb = ckpt + (size_t)blk * iters * 2 * B;

  for (int e = tid; e < R * B; e += NT) {
    const size_t off = base + (size_t)row0 * B + e;
    z[e] = L[off] / tau;
    float g = dP[off];
    for (int s = 1; s < splits; ++s) g += dP[(size_t)s * split_stride + off];
    d[e] = g;
  }
  for (int r = tid; r < R; r += NT) rv[r] = ckb[(size_t)(iters - 1) * 2 * B + row0 + r];
  for (int j = tid; j < B; j += NT) ck[j] = ckb[(size_t)(iters - 1) * 2 * B + B + j];
  __syncthreads();
  // dZ = dP (.) P with P = exp(z - R^(K) - C^(K))
  for (int e = tid; e < R * B; e += NT) d[e] *= expf(z[e] - rv[e / B] - ck[e % B]);
  __syncthreads();

  for (int k = iters - 1; k >= 0; --k) {
    // rv = R^(k+1), ck = C^(k+1), ck1 = C^(k) (zero before the first iteration)
    for (int r = tid; r < R; r += NT) rv[r] = ckb[(size_t)k * 2 * B + row0 + r];
    for (int j = tid; j < B; j += NT) {
      ck[j] = ckb[(size_t)k * 2 * B + B + j];
      ck1[j] = (k > 0) ? ckb[(size_t)(k - 1) * 2 * B + B + j] : 0.f;
    }
    // column step: dZ -= exp(Z') * colsum(dZ), Z' = z - R^(k+1) - C^(k+1)
    {
      const int j = tid % B, g = tid / B;
      float s = 0.f;
      for (int r = g; r < R; r += G) s += d[r * B + j];
      pm[g * B + j] = s;
    }
    __syncthreads();
    float* bs = xs + (k & 1) * B;
    for (int j = tid; j < B; j += NT) {
      float s = 0.f;
      for (int g = 0; g < G; ++g) s += pm[g * B + j];
      bs[j] = s;
    }
    cluster_barrier<CS>();
    if constexpr (CS == 1) __syncthreads();
    for (int e = tid; e < R * B; e += NT) {
      const int r = e / B, j = e % B;
      float cs = 0.f;
      for (int q = 0; q < CS; ++q) cs += peer<CS>(bs, q)[j];
      d[e] -= expf(z[e] - rv[r] - ck[j]) * cs;
    }
    __syncthreads();
    // row step: dZ -= exp(Z') * rowsum(dZ), Z' = z - R^(k+1) - C^(k); one warp per row
    for (int r = warp; r < R; r += NW) {
      float* dr = d + r * B;
      const float* zr = z + r * B;
      float s = 0.f;
      for (int j = lane; j < B; j += 32) s += dr[j];
      s = warp_sum(s);
      for (int j = lane; j < B; j += 32) dr[j] -= expf(zr[j] - rv[r] - ck1[j]) * s;
    }
    __syncthreads();
  }
  for (int e = tid; e < R * B; e += NT) dL[base + (size_t)row0 * B + e] = d[e] / tau;
  cluster_barrier<CS>();
}

template <int B> constexpr size_t fwd_smem() {
  using C = SkCfg<B>;
  return sizeof(float) * (C::R * B + C::R + B + 2 * C::G * B + 4 * B);
}
template <int B> constexpr size_t bwd_smem() {
  using C = SkCfg<B>;
  return sizeof(float) * (2 * C::R * B + C::R + 2 * B + C::G * B + 2 * B);
}

template <typename K, typename... Args>
lcp_status launch_cluster(K kernel, int grid, int threads, size_t smem, int cs, cudaStream_t st,
                          const char* what, Args... args) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return check_launch(what);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  return check_launch(what);
}

template <int B>
lcp_status fwd_b(const float* L, float* P, float* ckpt, __nv_bfloat16* a, __nv_bfloat16* b,
                 __nv_bfloat16* c, int nblocks, float tau, int iters, cudaStream_t st) {
  using C = SkCfg<B>;
  return launch_cluster(sinkhorn_fwd_kernel<B>, nblocks * C::CS, C::NT, fwd_smem<B>(), C::CS, st,
                        "sinkhorn_fwd", L, P, ckpt, a, b, c, tau, iters);
}
template <int B>
lcp_status bwd_b(const float* L, const float* ckpt, const float* dP, int splits, float* dL,
                 int nblocks, float tau, int iters, cudaStream_t st) {
  using C = SkCfg<B>;
  return launch_cluster(sinkhorn_bwd_kernel<B>, nblocks * C::CS, C::NT, bwd_smem<B>(), C::CS, st,
                        "sinkhorn_bwd", L, ckpt, dP, splits, nblocks, dL, tau, iters);
}

}  // namespace

lcp_status launch_sinkhorn_fwd(const float* L, float* P, float* ckpt, __nv_bfloat16* img_pt_hi,
                               __nv_bfloat16* img_pt_lo, __nv_bfloat16* img_p_hi, int nblocks,
                               int B, float tau, int iters, cudaStream_t st) {
  switch (B) {
    case 32: return fwd_b<32>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, nblocks, tau, iters, st);
    case 64: return fwd_b<64>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, nblocks, tau, iters, st);
    case 128: return fwd_b<128>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, nblocks, tau, iters, st);
    case 256: return fwd_b<256>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, nblocks, tau, iters, st);
  }
  return fail(LCP_ERR_SHAPE, "sinkhorn_fwd: unsupported block size %d", B);
}

lcp_status launch_sinkhorn_bwd(const float* L, const float* ckpt, const float* dP, int splits,
                               float* dL, int nblocks, int B, float tau, int iters,
                               cudaStream_t st) {
  switch (B) {
    case 32: return bwd_b<32>(L, ckpt, dP, splits, dL, nblocks, tau, iters, st);
    case 64: return bwd_b<64>(L, ckpt, dP, splits, dL, nblocks, tau, iters, st);
    case 128: return bwd_b<128>(L, ckpt, dP, splits, dL, nblocks, tau, iters, st);
    case 256: return bwd_b<256>(L, ckpt, dP, splits, dL, nblocks, tau, iters, st);
  }
  return fail(LCP_ERR_SHAPE, "sinkhorn_bwd: unsupported block size %d", B);
}

}  // namespace lcp
