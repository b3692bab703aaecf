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
// C_j = LSE_i(Z_0[i,j] - R_i).  Z_0 = L / tau never changes, so each thread
// keeps its share of Z_0 in registers twice: a row slice (TPR adjacent lanes
// per row, interleaved columns) for the row steps and a column slice (TPC
// adjacent lanes per column, interleaved rows) for the column steps.  A step
// is then register arithmetic, a read of the other side's normaliser vector
// from shared memory and two or three shuffles; the (R, C) pair of every
// iteration is the checkpoint the reverse pass replays.
//
// One CTA owns one block for B <= 128.  For B = 256 a cluster of 4 CTAs
// splits the rows; column reductions combine the per-CTA partials through
// distributed shared memory in a fixed rank order, so every CTA gets
// bit-identical results.  Every reduction runs in a fixed order.  Exponentials
// and logarithms use the hardware approximations (__expf, __logf): about 1e-6
// relative error, well inside the 1e-5 tolerance on P.

#include <cooperative_groups.h>
#include <math_constants.h>

#include "lcp_internal.cuh"

namespace cg = cooperative_groups;

namespace lcp {
namespace {

template <int B> struct SkCfg {
  static constexpr int CS = (B == 256) ? 4 : 1;                   // CTAs per block
  static constexpr int NT = (B == 32) ? 256 : (B == 64 ? 512 : 1024);
  static constexpr int R = B / CS;                                 // rows per CTA
  static constexpr int TPR = NT / R;                               // lanes per row
  static constexpr int EPR = B / TPR;                              // elements per row slice
  static constexpr int TPC = NT / B;                               // lanes per column
  static constexpr int EPC = R / TPC;                              // elements per column slice
  static constexpr int NW = NT / 32;
  static constexpr int LD = B + 1;                                 // padded smem tile row
  static_assert(TPR >= 1 && TPR <= 32 && (32 % TPR) == 0, "row slices must sit inside a warp");
  static_assert(TPC >= 1 && TPC <= 32 && (32 % TPC) == 0, "column slices must sit inside a warp");
  static_assert(R * TPR == NT && B * TPC == NT, "bad Sinkhorn configuration");
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

// reductions over `W` adjacent lanes (W a power of two)
template <int W> __device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = 1; o < W; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
template <int W> __device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = 1; o < W; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// log-sum-exp of x[0..N) combined over W adjacent lanes
template <int N, int W> __device__ __forceinline__ void lse_parts(const float (&x)[N], float& m, float& s) {
  float mx = x[0];
#pragma unroll
  for (int e = 1; e < N; ++e) mx = fmaxf(mx, x[e]);
  m = group_max<W>(mx);
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < N; ++e) acc += __expf(x[e] - m);
  s = group_sum<W>(acc);
}

// Stage a R x B row-major slab of a float32 [*, B, B] tensor into the padded tile (coalesced).
template <int B, int NT, int R>
__device__ __forceinline__ void load_slab(float* tile, const float* __restrict__ src, float scale) {
  constexpr int Q = B / 4;
  for (int q = threadIdx.x; q < R * Q; q += NT) {
    const float4 v = reinterpret_cast<const float4*>(src)[q];
    const int r = q / Q, j = (q % Q) * 4;
    float* d = tile + r * (B + 1) + j;
    d[0] = v.x * scale; d[1] = v.y * scale; d[2] = v.z * scale; d[3] = v.w * scale;
  }
}

// Forward.  Shared memory (floats): tile[R*(B+1)] rv[R] cv[B] xm[2B] xs[2B]
template <int B>
__global__ void __launch_bounds__(SkCfg<B>::NT, 1)
sinkhorn_fwd_kernel(const float* __restrict__ L, float* __restrict__ P, float* __restrict__ ckpt,
                    __nv_bfloat16* __restrict__ pt_hi, __nv_bfloat16* __restrict__ pt_lo,
                    __nv_bfloat16* __restrict__ p_hi, unsigned* __restrict__ zero_word, float tau, int iters) {
  using C = SkCfg<B>;
  pdl_wait();
  pdl_trigger();
  if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0u;
  constexpr int R = C::R, NT = C::NT, CS = C::CS, TPR = C::TPR, EPR = C::EPR, TPC = C::TPC,
                EPC = C::EPC, LD = C::LD;
  extern __shared__ __align__(16) float sm[];
  float* tile = sm;
  float* rv = tile + R * LD;
  float* cv = rv + R;
  float* xm = cv + B;   // this CTA's column partials, double-buffered by iteration parity
  float* xs = xm + 2 * B;

  const int rank = cta_rank<CS>();
  const int blk = blockIdx.x / CS;
  const int row0 = rank * R;
  const int tid = threadIdx.x;
  const size_t base = (size_t)blk * B * B;
  const int r = tid / TPR, c = tid % TPR;     // row slice: row r, columns c + TPR*e
  const int j = tid / TPC, g = tid % TPC;     // column slice: column j, rows g + TPC*e

  // Z_0 = L / tau (as L times the correctly rounded 1 / tau: within an ulp)
  const float inv_tau = 1.0f / tau;
  for (int q = tid; q < R * (B / 4); q += NT) {
    const float4 v = reinterpret_cast<const float4*>(L + base + (size_t)row0 * B)[q];
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    float* d = tile + rr * LD + jj;
    d[0] = v.x * inv_tau; d[1] = v.y * inv_tau; d[2] = v.z * inv_tau; d[3] = v.w * inv_tau;
  }
  for (int jj = tid; jj < B; jj += NT) cv[jj] = 0.f;
  __syncthreads();
  float zr[EPR], zc[EPC];
#pragma unroll
  for (int e = 0; e < EPR; ++e) zr[e] = tile[r * LD + c + TPR * e];
#pragma unroll
  for (int e = 0; e < EPC; ++e) zc[e] = tile[(g + TPC * e) * LD + j];

  float myR = 0.f;
  for (int k = 0; k < iters; ++k) {
    // T_r: R_i = LSE_j(z_ij - C_j)
    {
      float x[EPR];
#pragma unroll
      for (int e = 0; e < EPR; ++e) x[e] = zr[e] - cv[c + TPR * e];
      float m, s;
      lse_parts<EPR, TPR>(x, m, s);
      myR = m + __logf(s);
      if (c == 0) {
        rv[r] = myR;
        if (ckpt) ckpt[((size_t)blk * iters + k) * 2 * B + row0 + r] = myR;
      }
    }
    __syncthreads();
    // T_c: C_j = LSE_i(z_ij - R_i) over all B rows of the block
    {
      float x[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) x[e] = zc[e] - rv[g + TPC * e];
      float m, s;
      lse_parts<EPC, TPC>(x, m, s);
      if constexpr (CS == 1) {
        if (g == 0) {
          const float v = m + __logf(s);
          cv[j] = v;
          if (ckpt) ckpt[(((size_t)blk * iters + k) * 2 + 1) * B + j] = v;
        }
        __syncthreads();
      } else {
        float* bm = xm + (k & 1) * B;
        float* bs = xs + (k & 1) * B;
        if (g == 0) { bm[j] = m; bs[j] = s; }
        cluster_barrier<CS>();
        if (g == 0) {
          float M = -CUDART_INF_F;
#pragma unroll
          for (int q = 0; q < CS; ++q) M = fmaxf(M, peer<CS>(bm, q)[j]);
          float S = 0.f;
#pragma unroll
          for (int q = 0; q < CS; ++q) S += peer<CS>(bs, q)[j] * __expf(peer<CS>(bm, q)[j] - M);
          const float v = M + __logf(S);
          cv[j] = v;
          if (ckpt && rank == 0) ckpt[(((size_t)blk * iters + k) * 2 + 1) * B + j] = v;
        }
        __syncthreads();
      }
    }
  }

  // P = exp(Z_0 - R - C), staged through the tile for coalesced stores
#pragma unroll
  for (int e = 0; e < EPR; ++e) tile[r * LD + c + TPR * e] = __expf(zr[e] - myR - cv[c + TPR * e]);
  __syncthreads();
  for (int q = tid; q < R * B; q += NT) {
    const int rr = q / B, jj = q % B;
    P[base + (size_t)(row0 + rr) * B + jj] = tile[rr * LD + jj];
  }
  if (pt_hi) {
    // Operand images for the tensor-core kernels, in tiles of BC = max(B, 64)
    // columns: tile t holds the BC x BC block-diagonal slice of P_B covering
    // channels [t*BC, (t+1)*BC) (for B = 32 two blocks share one tile and the
    // off-diagonal quadrants are written as zeros).
    constexpr int BC = B < 64 ? 64 : B;
    const int gcol0 = blk * B;
    const size_t tb = (size_t)(gcol0 / BC) * BC * BC;
    const int q0 = gcol0 % BC;
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
    // transposed images: consecutive threads take consecutive source rows i
    for (int q = tid; q < R * B; q += NT) {
      const int jj = q / R, rr = q % R, i = row0 + rr;
      const float p = tile[rr * LD + jj];
      const __nv_bfloat16 hi = __float2bfloat16_rn(p);
      pt_hi[tb + (size_t)(q0 + jj) * BC + q0 + i] = hi;
      pt_lo[tb + (size_t)(q0 + jj) * BC + q0 + i] = __float2bfloat16_rn(p - __bfloat162float(hi));
      if constexpr (B < BC) {
        const int zc0 = (q0 == 0) ? B : 0;
        pt_hi[tb + (size_t)(q0 + jj) * BC + zc0 + i] = zero;
        pt_lo[tb + (size_t)(q0 + jj) * BC + zc0 + i] = zero;
      }
    }
    for (int q = tid; q < R * B; q += NT) {
      const int rr = q / B, jj = q % B, i = row0 + rr;
      p_hi[tb + (size_t)(q0 + i) * BC + q0 + jj] = __float2bfloat16_rn(tile[rr * LD + jj]);
      if constexpr (B < BC) p_hi[tb + (size_t)(q0 + i) * BC + ((q0 == 0) ? B : 0) + jj] = zero;
    }
  }
  // keep peers' shared memory alive until every CTA of the cluster is done reading it
  cluster_barrier<CS>();
}

// Reverse.  dZ lives in registers in the row layout.  For B = 64 the kernel is
// held to 64 registers a thread so that two CTAs share an SM when many blocks
// are in flight (a whole model's logits in one launch).
// Shared memory (floats): tile[R*(B+1)] ck[B] ck1[B] part[NW*B] cs[B] xs[2B]
template <int B>
__global__ void __launch_bounds__(SkCfg<B>::NT, B == 64 ? 2 : 1)
sinkhorn_bwd_kernel(const float* __restrict__ L, const float* __restrict__ ckpt,
                    const float* __restrict__ dP, int splits, int nblocks,
                    float* __restrict__ dL, float tau, int iters) {
  using C = SkCfg<B>;
  pdl_wait();
  pdl_trigger();
  constexpr int R = C::R, NT = C::NT, CS = C::CS, TPR = C::TPR, EPR = C::EPR, NW = C::NW, LD = C::LD;
  constexpr int RPW = 32 / TPR;   // rows per warp
  extern __shared__ __align__(16) float sm[];
  float* tile = sm;
  float* ck = tile + R * LD;   // C^(k+1)
  float* ck1 = ck + B;         // C^(k)
  float* part = ck1 + B;       // per-warp column partial sums
  float* cs = part + NW * B;   // column sums of dZ
  float* xs = cs + B;          // this CTA's column sums for the cluster, double-buffered

  const int rank = cta_rank<CS>();
  const int blk = blockIdx.x / CS;
  const int row0 = rank * R;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const size_t base = (size_t)blk * B * B;
  const size_t split_stride = (size_t)nblocks * B * B;
  const float* ckb = ckpt + (size_t)blk * iters * 2 * B;
  const int r = tid / TPR, c = tid % TPR;

  float zr[EPR], dz[EPR];
  // Z_0 = L / tau, formed as in the forward kernel
  const float inv_tau = 1.0f / tau;
  for (int q = tid; q < R * (B / 4); q += NT) {
    const float4 v = reinterpret_cast<const float4*>(L + base + (size_t)row0 * B)[q];
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    float* d = tile + rr * LD + jj;
    d[0] = v.x * inv_tau; d[1] = v.y * inv_tau; d[2] = v.z * inv_tau; d[3] = v.w * inv_tau;
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < EPR; ++e) zr[e] = tile[r * LD + c + TPR * e];
  __syncthreads();
  // dP summed over the splits in index order
  for (int q = tid; q < R * (B / 4); q += NT) {
    float4 a = reinterpret_cast<const float4*>(dP + base + (size_t)row0 * B)[q];
    for (int s = 1; s < splits; ++s) {
      const float4 b = reinterpret_cast<const float4*>(dP + (size_t)s * split_stride + base + (size_t)row0 * B)[q];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    float* d = tile + rr * LD + jj;
    d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w;
  }
  for (int jj = tid; jj < B; jj += NT) ck[jj] = ckb[(size_t)(iters - 1) * 2 * B + B + jj];
  __syncthreads();
  float myR = ckb[(size_t)(iters - 1) * 2 * B + row0 + r];
  // dZ = dP (.) P with P = exp(z - R^(K) - C^(K))
#pragma unroll
  for (int e = 0; e < EPR; ++e) dz[e] = tile[r * LD + c + TPR * e] * __expf(zr[e] - myR - ck[c + TPR * e]);

  for (int k = iters - 1; k >= 0; --k) {
    __syncthreads();   // previous iteration done with ck, ck1, part, cs
    for (int jj = tid; jj < B; jj += NT) {
      ck[jj] = ckb[(size_t)k * 2 * B + B + jj];
      ck1[jj] = (k > 0) ? ckb[(size_t)(k - 1) * 2 * B + B + jj] : 0.f;
    }
    myR = ckb[(size_t)k * 2 * B + row0 + r];
    // column sums of dZ: over the rows of this warp (lanes with equal c), then over warps
#pragma unroll
    for (int e = 0; e < EPR; ++e) {
      float v = dz[e];
#pragma unroll
      for (int o = TPR; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane < TPR) part[warp * B + c + TPR * e] = v;
    }
    __syncthreads();
    float* bs = xs + (k & 1) * B;
    for (int jj = tid; jj < B; jj += NT) {
      float s = 0.f;
      for (int w = 0; w < NW; ++w) s += part[w * B + jj];
      if constexpr (CS == 1) cs[jj] = s;
      else bs[jj] = s;
    }
    if constexpr (CS > 1) {
      cluster_barrier<CS>();
      for (int jj = tid; jj < B; jj += NT) {
        float s = 0.f;
        for (int q = 0; q < CS; ++q) s += peer<CS>(bs, q)[jj];
        cs[jj] = s;
      }
    }
    __syncthreads();
    // column step: dZ -= exp(Z') colsum, Z' = z - R^(k+1) - C^(k+1)
#pragma unroll
    for (int e = 0; e < EPR; ++e) dz[e] -= __expf(zr[e] - myR - ck[c + TPR * e]) * cs[c + TPR * e];
    // row step: dZ -= exp(Z') rowsum, Z' = z - R^(k+1) - C^(k)
    float rs = 0.f;
#pragma unroll
    for (int e = 0; e < EPR; ++e) rs += dz[e];
    rs = group_sum<TPR>(rs);
#pragma unroll
    for (int e = 0; e < EPR; ++e) dz[e] -= __expf(zr[e] - myR - ck1[c + TPR * e]) * rs;
  }
  // dL = dZ_0 / tau, staged for coalesced stores
  __syncthreads();
#pragma unroll
  for (int e = 0; e < EPR; ++e) tile[r * LD + c + TPR * e] = dz[e] * inv_tau;
  __syncthreads();
  for (int q = tid; q < R * B; q += NT) {
    const int rr = q / B, jj = q % B;
    dL[base + (size_t)(row0 + rr) * B + jj] = tile[rr * LD + jj];
  }
  cluster_barrier<CS>();
  (void)RPW;
}

template <int B> constexpr size_t fwd_smem() {
  using C = SkCfg<B>;
  return sizeof(float) * (C::R * C::LD + C::R + B + 4 * B);
}
template <int B> constexpr size_t bwd_smem() {
  using C = SkCfg<B>;
  return sizeof(float) * (C::R * C::LD + 2 * B + C::NW * B + B + 2 * B);
}

template <int B>
lcp_status fwd_b(const float* L, float* P, float* ckpt, __nv_bfloat16* a, __nv_bfloat16* b,
                 __nv_bfloat16* c, unsigned* zero_word, int nblocks, float tau, int iters, cudaStream_t st) {
  using C = SkCfg<B>;
  const lcp_status s0 = ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_fwd_kernel<B>), (int)fwd_smem<B>(),
                                          "sinkhorn_fwd");
  if (s0 != LCP_OK) return s0;
  return launch_kernel(sinkhorn_fwd_kernel<B>, dim3(nblocks * C::CS), dim3(C::NT), fwd_smem<B>(), st, C::CS, true,
                       "sinkhorn_fwd", L, P, ckpt, a, b, c, zero_word, tau, iters);
}
template <int B>
lcp_status bwd_b(const float* L, const float* ckpt, const float* dP, int splits, float* dL,
                 int nblocks, float tau, int iters, cudaStream_t st) {
  using C = SkCfg<B>;
  const lcp_status s0 = ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_bwd_kernel<B>), (int)bwd_smem<B>(),
                                          "sinkhorn_bwd");
  if (s0 != LCP_OK) return s0;
  return launch_kernel(sinkhorn_bwd_kernel<B>, dim3(nblocks * C::CS), dim3(C::NT), bwd_smem<B>(), st, C::CS, true,
                       "sinkhorn_bwd", L, ckpt, dP, splits, nblocks, dL, tau, iters);
}

}  // namespace

lcp_status launch_sinkhorn_fwd(const float* L, float* P, float* ckpt, __nv_bfloat16* img_pt_hi,
                               __nv_bfloat16* img_pt_lo, __nv_bfloat16* img_p_hi, unsigned* zero_word,
                               int nblocks, int B, float tau, int iters, cudaStream_t st) {
  switch (B) {
    case 32: return fwd_b<32>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, zero_word, nblocks, tau, iters, st);
    case 64: return fwd_b<64>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, zero_word, nblocks, tau, iters, st);
    case 128: return fwd_b<128>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, zero_word, nblocks, tau, iters, st);
    case 256: return fwd_b<256>(L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, zero_word, nblocks, tau, iters, st);
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
