// Block-wise Sinkhorn normalisation, forward and reverse.
//
// PermLLM ("Learnable Channel Permutation for N:M Sparse LLMs"), Method 1:
// S_0(X) = exp(X), S_i(X) = T_c(T_r(S_{i-1}(X))), P = S_L(W_P / tau), applied
// to every B x B diagonal block (Method 3).  The blog page's section 2.2
// gives the log-domain form: subtract each row's log-sum-exp, then each
// column's, `iters` times, then exponentiate.
//
// Every iterate has the form Z = Z_0 - R_i - C_j, so a row step only has to
// compute R_i = LSE_j(Z_0[i,j] - C_j) and a column step C_j = LSE_i(Z_0[i,j] -
// R_i); (R, C) after every step is the checkpoint the reverse pass replays.
// Two arithmetics compute these, chosen per block from the range of Z_0 = L/tau:
//
//  * linear (max Z_0 - min Z_0 <= 64, every block of a run near its
//    initialisation): with K = exp(Z_0 - max Z_0) formed once per element
//    (entries in [e^-64, 1]), exp(Z) = a_i K_ij b_j with a = e^{max - R},
//    b = e^{-C}; a row step is a_i = 1 / sum_j K_ij b_j and a column step
//    b_j = 1 / sum_i a_i K_ij -- multiply-adds and one reciprocal per row or
//    column instead of two exponentials per element.  The checkpoint stores
//    R_i = max + log(sum_j K_ij b_j) and C_j = log(sum_i a_i K_ij), the same
//    normalisers as the log domain.  The scalings stay within e^{+-70}, inside
//    the float32 range.
//  * log domain (wider ranges, e.g. sharply peaked logits, where K would
//    underflow): the log-sum-exp steps themselves.
//
// The kernels are persistent: a CTA (cluster) walks blocks g, g + grid, ... of
// every layer of the launch, the next block's inputs loaded into registers
// while the current one runs (B <= 128), so a launch over a whole model's
// logits keeps its loads in flight.
//
// Z_0 never changes, so each thread keeps its share of Z_0 (or K) in registers
// twice: a row slice (TPR adjacent lanes per row) for the row steps and a
// column slice (TPC adjacent lanes per column, interleaved rows) for the column
// steps.  A step is then register arithmetic, a read of
// the other side's vector from shared memory and two or three shuffles.
//
// A CTA owns one block at a time for B <= 64; for B = 128 a cluster of 2 CTAs
// and for B = 256 a cluster of 4 splits the rows; column reductions combine the per-CTA partials through
// distributed shared memory in a fixed rank order, so every CTA gets
// bit-identical results (the range that picks the arithmetic is combined the
// same way).  Every reduction runs in a fixed order.  Exponentials and
// logarithms use the hardware approximations (__expf, __logf): about 1e-6
// relative error, well inside the 1e-5 tolerance on P.

#include <algorithm>
#include <type_traits>
#include <cooperative_groups.h>
#include <math_constants.h>

#include "lcp_internal.cuh"

namespace cg = cooperative_groups;

namespace lcp {
namespace {

// B = 64 launches with at least this many blocks in all run the forward pass
// one warp a block (sinkhorn_fwd_warp_kernel) and the reverse pass two warps a
// block (sinkhorn_bwd_pair_kernel); smaller ones one 512-thread CTA a block.
// The forward threshold is higher: below it the warp kernel's log-domain
// fallback is slower than the CTA kernel's.
#ifndef LCP_SINKHORN_WARP_MIN_BLOCKS
#define LCP_SINKHORN_WARP_MIN_BLOCKS 1024
#endif
#ifndef LCP_SINKHORN_PAIR_MIN_BLOCKS
#define LCP_SINKHORN_PAIR_MIN_BLOCKS 256
#endif

// CTAs (a cluster) per B = 128 block (tuning: 1 or 2) and per B = 256 block (4 or 8)
#ifndef LCP_SINKHORN_B128_CTAS
#define LCP_SINKHORN_B128_CTAS 2
#endif
#ifndef LCP_SINKHORN_B256_CTAS
#define LCP_SINKHORN_B256_CTAS 4
#endif

template <int B> struct SkCfg {
  static constexpr int CS = (B == 256) ? LCP_SINKHORN_B256_CTAS : (B == 128 ? LCP_SINKHORN_B128_CTAS : 1);  // CTAs per block
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

// The B <= 64 forward kernel's threads: a 128-thread CTA (one warp per SM sub-partition, 32
// elements of a row and 32 of a column a thread for B = 64: one shuffle per reduction and a
// four-warp barrier per step, the step's latency being what bounds a block).
template <int B> struct SkFwdCfg {
  static_assert(B <= 64, "the cluster sizes run sinkhorn_fwd_cluster_kernel");
  static constexpr int CS = 1;
  static constexpr int NT = 128;
  static constexpr int R = B;
  static constexpr int TPR = NT / R;
  static constexpr int EPR = B / TPR;
  static constexpr int TPC = NT / B;
  static constexpr int EPC = R / TPC;
  static constexpr int NW = NT / 32;
  static constexpr int MINB = 4;   // CTAs an SM (register bound 128)
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

// two floats -> packed bf16x2 (round to nearest even), low half first
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
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

// Widest range of Z_0 = L / tau over a block for which the linear arithmetic
// is used: K = exp(Z_0 - max Z_0) then lies in [e^-64, 1].
constexpr float kLinearRange = 64.f;

// Largest and smallest value over the CTA (and over the cluster for CS > 1),
// bit-identical on every thread of every CTA of the cluster.  red: 66 floats
// of shared memory, not reused afterwards.  Ends with a CTA (cluster) barrier.
template <int NT, int CS>
__device__ __forceinline__ void block_range(float mx, float mn, float* red, float& gmx, float& gmn) {
  constexpr int NW = NT / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  mx = group_max<32>(mx);
  mn = -group_max<32>(-mn);
  if (lane == 0) {
    red[warp] = mx;
    red[32 + warp] = mn;
  }
  __syncthreads();
  if (warp == 0) {
    float a = lane < NW ? red[lane] : -CUDART_INF_F;
    float b = lane < NW ? -red[32 + lane] : -CUDART_INF_F;
    a = group_max<32>(a);
    b = group_max<32>(b);
    if (lane == 0) {
      red[64] = a;
      red[65] = -b;
    }
  }
  if constexpr (CS == 1) {
    __syncthreads();
    gmx = red[64];
    gmn = red[65];
  } else {
    cluster_barrier<CS>();
    float a = -CUDART_INF_F, b = CUDART_INF_F;
#pragma unroll
    for (int q = 0; q < CS; ++q) {
      const float* pr = peer<CS>(red, q);
      a = fmaxf(a, pr[64]);
      b = fminf(b, pr[65]);
    }
    gmx = a;
    gmn = b;
  }
}

// Forward for B <= 64 (one CTA a block; the cluster sizes run sinkhorn_fwd_cluster_kernel).
// A thread's row slice is EPR consecutive columns c EPR .. c EPR + EPR - 1 of row r
// and its column slice EPC consecutive rows g EPC .. g EPC + EPC - 1 of column j, so both
// vectors are read with 16-byte loads, P and its row-major bf16 image are written from the
// row slice and the transposed images from the column slice, straight from registers (the same
// operands in the same order: the same values).  Z_0 is staged with a row pitch of B + 4
// (16-byte rows).  The range of Z_0 is reduced from the staged registers under the barrier
// that publishes the tile.
// Shared memory (floats): tile[B*(B+4)] rv[B] cv[B] red[66]
template <int B> __host__ __device__ constexpr int fwd_ld() { return B + 4; }
template <int B> constexpr size_t fwd_smem_base() {
  using C = SkFwdCfg<B>;
  return sizeof(float) * (C::R * fwd_ld<B>() + C::R + B + 66);
}

template <int B>
__global__ void __launch_bounds__(SkFwdCfg<B>::NT, SkFwdCfg<B>::MINB)
sinkhorn_fwd_kernel(const __grid_constant__ SkFwdBatch batch, float tau, int iters) {
  using C = SkFwdCfg<B>;
  pdl_wait();
  pdl_trigger();
  constexpr int R = C::R, NT = C::NT, CS = C::CS, TPR = C::TPR, EPR = C::EPR, TPC = C::TPC,
                EPC = C::EPC, NW = C::NW, LD = fwd_ld<B>();
  constexpr int NPRE = R * (B / 4) / NT;   // float4 of L a thread stages per block
  static_assert(NPRE * NT == R * (B / 4), "the L slab must split evenly over the threads");
  static_assert(EPR % 4 == 0 && LD % 4 == 0, "row slices are read and written as float4");
  extern __shared__ __align__(16) float sm[];
  float* tile = sm;
  float* rv = tile + R * LD;   // per row of this CTA: a_i (linear) or R_i (log domain)
  float* cv = rv + R;          // per column: b_j (linear) or C_j (log domain)
  float* red = cv + B;

  const int rank = cta_rank<CS>();
  const int row0 = rank * R;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r = tid / TPR, c = tid % TPR;     // row slice: row r, columns c EPR + e
  const int j = tid / TPC, g = tid % TPC;     // column slice: column j, rows g EPC + e
  const float inv_tau = 1.0f / tau;
  // The CTA (cluster) walks the blocks g = blockIdx.x / CS, + gridDim.x / CS, ...
  // of every layer; the next block's slab of L is loaded into registers while
  // the current one iterates.
  int total = 0;
  for (int i = 0; i < batch.n; ++i) total += batch.layer[i].blocks;
  const int gstride = gridDim.x / CS;
  auto locate = [&](int gb, int& li, int& blk) {
    blk = gb;
    li = 0;
    while (li + 1 < batch.n && blk >= batch.layer[li].blocks) blk -= batch.layer[li++].blocks;
  };
  float4 pre[NPRE];
  auto prefetch = [&](int gb) {
    int li, blk;
    locate(gb, li, blk);
    const float4* src = reinterpret_cast<const float4*>(batch.layer[li].L + (size_t)blk * B * B + (size_t)row0 * B);
#pragma unroll
    for (int k = 0; k < NPRE; ++k) pre[k] = src[tid + k * NT];
  };
  // the look-ahead needs NPRE more registers a thread: not for the 1024-thread B = 256 CTAs
  constexpr bool AHEAD = NPRE <= 2;
  if (AHEAD && blockIdx.x / CS < total) prefetch(blockIdx.x / CS);
  for (int gb = blockIdx.x / CS; gb < total; gb += gstride) {
  if constexpr (!AHEAD) prefetch(gb);
  int li, blk;
  locate(gb, li, blk);
  const SkFwdLayer& ly = batch.layer[li];
  float* __restrict__ P = ly.P;
  float* __restrict__ ckpt = ly.ckpt;
  __nv_bfloat16* __restrict__ pt_hi = ly.pt_hi;
  __nv_bfloat16* __restrict__ pt_lo = ly.pt_lo;
  __nv_bfloat16* __restrict__ p_hi = ly.p_hi;
  if (ly.zero_word && blk == 0 && rank == 0 && tid == 0) *ly.zero_word = 0u;
  const size_t base = (size_t)blk * B * B;
  const size_t ck0 = (size_t)blk * iters * 2 * B;

  // Z_0 = L / tau (as L times the correctly rounded 1 / tau: within an ulp) into the tile, and
  // the range of this thread's staged values, reduced per warp
  float lmx = -CUDART_INF_F, lmn = CUDART_INF_F;
#pragma unroll
  for (int k = 0; k < NPRE; ++k) {
    const int q = tid + k * NT;
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    const float4 z = make_float4(pre[k].x * inv_tau, pre[k].y * inv_tau, pre[k].z * inv_tau, pre[k].w * inv_tau);
    *reinterpret_cast<float4*>(tile + rr * LD + jj) = z;
    lmx = fmaxf(lmx, fmaxf(fmaxf(z.x, z.y), fmaxf(z.z, z.w)));
    lmn = fminf(lmn, fminf(fminf(z.x, z.y), fminf(z.z, z.w)));
  }
  if (AHEAD && gb + gstride < total) prefetch(gb + gstride);   // in flight while this block iterates
  lmx = group_max<32>(lmx);
  lmn = -group_max<32>(-lmn);
  if (lane == 0) {
    red[warp] = lmx;
    red[32 + warp] = lmn;
  }
  __syncthreads();
  float zmax = red[0], zmin = red[32];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    zmax = fmaxf(zmax, red[w]);
    zmin = fminf(zmin, red[32 + w]);
  }
  float zr[EPR], zc[EPC];
#pragma unroll
  for (int e = 0; e < EPR; e += 4) {
    const float4 v = *reinterpret_cast<const float4*>(tile + r * LD + c * EPR + e);
    zr[e] = v.x; zr[e + 1] = v.y; zr[e + 2] = v.z; zr[e + 3] = v.w;
  }
#pragma unroll
  for (int e = 0; e < EPC; ++e) zc[e] = tile[(g * EPC + e) * LD + j];
  const bool linear = (zmax - zmin) <= kLinearRange;
  // checkpoint value of row r / column j after step k, in the log form the reverse pass reads
  // (R_i = max + log s and C_j = log s in the linear arithmetic)
  auto ck_row = [&](int k, float v) { ckpt[ck0 + (size_t)k * 2 * B + row0 + r] = linear ? zmax + __logf(v) : v; };
  auto ck_col = [&](int k, float v) { ckpt[ck0 + ((size_t)k * 2 + 1) * B + j] = linear ? __logf(v) : v; };

  float myR = 0.f;   // this thread's row: a_i (linear) or R_i (log domain)
  float pv[EPR];     // P of this thread's row slice
  if (linear) {
#pragma unroll
    for (int e = 0; e < EPR; ++e) zr[e] = __expf(zr[e] - zmax);
#pragma unroll
    for (int e = 0; e < EPC; ++e) zc[e] = __expf(zc[e] - zmax);
    for (int jj = tid; jj < B; jj += NT) cv[jj] = 1.f;
    __syncthreads();
    for (int k = 0; k < iters; ++k) {
      // T_r: a_i = 1 / sum_j K_ij b_j   (R_i = max Z_0 + log of that sum)
      {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int e = 0; e < EPR; e += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(cv + c * EPR + e);
          s0 = fmaf(zr[e], b4.x, s0);
          s1 = fmaf(zr[e + 1], b4.y, s1);
          s2 = fmaf(zr[e + 2], b4.z, s2);
          s3 = fmaf(zr[e + 3], b4.w, s3);
        }
        const float s = group_sum<TPR>((s0 + s1) + (s2 + s3));
        myR = __fdividef(1.f, s);
        if (c == 0) {
          rv[r] = myR;
          if (ckpt) ck_row(k, s);
        }
      }
      __syncthreads();
      // T_c: b_j = 1 / sum_i a_i K_ij over all B rows   (C_j = log of that sum)
      {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int e = 0; e < EPC; e += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(rv + g * EPC + e);
          s0 = fmaf(zc[e], a4.x, s0);
          s1 = fmaf(zc[e + 1], a4.y, s1);
          s2 = fmaf(zc[e + 2], a4.z, s2);
          s3 = fmaf(zc[e + 3], a4.w, s3);
        }
        const float s = group_sum<TPC>((s0 + s1) + (s2 + s3));
        if (g == 0) {
          cv[j] = __fdividef(1.f, s);
          if (ckpt) ck_col(k, s);
        }
        __syncthreads();
      }
    }
    // P = a_i K_ij b_j
#pragma unroll
    for (int e = 0; e < EPR; e += 4) {
      const float4 b4 = *reinterpret_cast<const float4*>(cv + c * EPR + e);
      pv[e] = myR * zr[e] * b4.x;
      pv[e + 1] = myR * zr[e + 1] * b4.y;
      pv[e + 2] = myR * zr[e + 2] * b4.z;
      pv[e + 3] = myR * zr[e + 3] * b4.w;
    }
  } else {
    for (int jj = tid; jj < B; jj += NT) cv[jj] = 0.f;
    __syncthreads();
    for (int k = 0; k < iters; ++k) {
      // T_r: R_i = LSE_j(z_ij - C_j)
      {
        float x[EPR];
#pragma unroll
        for (int e = 0; e < EPR; e += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(cv + c * EPR + e);
          x[e] = zr[e] - b4.x; x[e + 1] = zr[e + 1] - b4.y; x[e + 2] = zr[e + 2] - b4.z; x[e + 3] = zr[e + 3] - b4.w;
        }
        float m, s;
        lse_parts<EPR, TPR>(x, m, s);
        myR = m + __logf(s);
        if (c == 0) {
          rv[r] = myR;
          if (ckpt) ck_row(k, myR);
        }
      }
      __syncthreads();
      // T_c: C_j = LSE_i(z_ij - R_i) over all B rows of the block
      {
        float x[EPC];
#pragma unroll
        for (int e = 0; e < EPC; e += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(rv + g * EPC + e);
          x[e] = zc[e] - a4.x; x[e + 1] = zc[e + 1] - a4.y; x[e + 2] = zc[e + 2] - a4.z; x[e + 3] = zc[e + 3] - a4.w;
        }
        float m, s;
        lse_parts<EPC, TPC>(x, m, s);
        if (g == 0) {
          const float v = m + __logf(s);
          cv[j] = v;
          if (ckpt) ck_col(k, v);
        }
        __syncthreads();
      }
    }
    // P = exp(Z_0 - R - C)
#pragma unroll
    for (int e = 0; e < EPR; e += 4) {
      const float4 b4 = *reinterpret_cast<const float4*>(cv + c * EPR + e);
      pv[e] = __expf(zr[e] - myR - b4.x);
      pv[e + 1] = __expf(zr[e + 1] - myR - b4.y);
      pv[e + 2] = __expf(zr[e + 2] - myR - b4.z);
      pv[e + 3] = __expf(zr[e + 3] - myR - b4.w);
    }
  }
  // P and its row-major bf16 image, straight from registers
  {
    float* prow = P + base + (size_t)(row0 + r) * B + c * EPR;
#pragma unroll
    for (int e = 0; e < EPR; e += 4)
      *reinterpret_cast<float4*>(prow + e) = make_float4(pv[e], pv[e + 1], pv[e + 2], pv[e + 3]);
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
    const int zc0 = (q0 == 0) ? B : 0;   // the zero quadrant's columns (B < BC)
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    // P_hi: image row q0 + row0 + r, columns q0 + c EPR .. (from registers)
    {
      __nv_bfloat16* prow = p_hi + tb + (size_t)(q0 + row0 + r) * BC;
#pragma unroll
      for (int e = 0; e < EPR; e += 8) {
        if constexpr (EPR % 8 == 0) {
          *reinterpret_cast<uint4*>(prow + q0 + c * EPR + e) =
              make_uint4(pack_bf16x2_rn(pv[e], pv[e + 1]), pack_bf16x2_rn(pv[e + 2], pv[e + 3]),
                         pack_bf16x2_rn(pv[e + 4], pv[e + 5]), pack_bf16x2_rn(pv[e + 6], pv[e + 7]));
          if constexpr (B < BC) *reinterpret_cast<uint4*>(prow + zc0 + c * EPR + e) = zero4;
        }
      }
      if constexpr (EPR == 4) {
        *reinterpret_cast<uint2*>(prow + q0 + c * EPR) =
            make_uint2(pack_bf16x2_rn(pv[0], pv[1]), pack_bf16x2_rn(pv[2], pv[3]));
        if constexpr (B < BC) *reinterpret_cast<uint2*>(prow + zc0 + c * EPR) = make_uint2(0u, 0u);
      }
    }
    // transposed images from the column slice: image row q0 + j, columns q0 + row0 + g EPC ..
    {
      const size_t at = tb + (size_t)(q0 + j) * BC + q0 + row0 + g * EPC;
      const float bj = cv[j];
#pragma unroll
      for (int e = 0; e < EPC; e += 8) {
        float hv[8], lv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float ai = rv[g * EPC + e + u];
          const float p = linear ? ai * zc[e + u] * bj : __expf(zc[e + u] - ai - bj);
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          hv[u] = __bfloat162float(hi);
          lv[u] = p - hv[u];
        }
        *reinterpret_cast<uint4*>(pt_hi + at + e) = make_uint4(pack_bf16x2_rn(hv[0], hv[1]), pack_bf16x2_rn(hv[2], hv[3]),
                                                               pack_bf16x2_rn(hv[4], hv[5]), pack_bf16x2_rn(hv[6], hv[7]));
        *reinterpret_cast<uint4*>(pt_lo + at + e) = make_uint4(pack_bf16x2_rn(lv[0], lv[1]), pack_bf16x2_rn(lv[2], lv[3]),
                                                               pack_bf16x2_rn(lv[4], lv[5]), pack_bf16x2_rn(lv[6], lv[7]));
        if constexpr (B < BC) {
          const size_t az = tb + (size_t)(q0 + j) * BC + zc0 + row0 + g * EPC + e;
          *reinterpret_cast<uint4*>(pt_hi + az) = zero4;
          *reinterpret_cast<uint4*>(pt_lo + az) = zero4;
        }
      }
    }
  }
  // every thread is done with this block's shared memory before the next block overwrites it
  __syncthreads();
  }
}

// Forward for the cluster sizes (B = 128, 256: 2 / 4 CTAs of 1024 threads a block): row slices
// interleaved over the TPR lanes of a row, P staged through the tile for coalesced stores and
// the transposed images (measured faster at these sizes than the B <= 64 kernel's layout).
// Shared memory (floats): tile[R*(B+1)] rv[R] cv[B] xm[2B] xs[2B] red[66]
template <int B>
__global__ void __launch_bounds__(SkCfg<B>::NT, 1024 / SkCfg<B>::NT)
sinkhorn_fwd_cluster_kernel(const __grid_constant__ SkFwdBatch batch, float tau, int iters) {
  using C = SkCfg<B>;
  pdl_wait();
  pdl_trigger();
  constexpr int R = C::R, NT = C::NT, CS = C::CS, TPR = C::TPR, EPR = C::EPR, TPC = C::TPC,
                EPC = C::EPC, LD = C::LD;
  constexpr int NPRE = R * (B / 4) / NT;   // float4 of L a thread stages per block
  static_assert(NPRE * NT == R * (B / 4), "the L slab must split evenly over the threads");
  extern __shared__ __align__(16) float sm[];
  float* tile = sm;
  float* rv = tile + R * LD;   // per row of this CTA: a_i (linear) or R_i (log domain)
  float* cv = rv + R;          // per column: b_j (linear) or C_j (log domain)
  float* xm = cv + B;          // this CTA's column partials, double-buffered by iteration parity
  float* xs = xm + 2 * B;
  float* red = xs + 2 * B;

  const int rank = cta_rank<CS>();
  const int row0 = rank * R;
  const int tid = threadIdx.x;
  const int r = tid / TPR, c = tid % TPR;     // row slice: row r, columns c + TPR*e
  const int j = tid / TPC, g = tid % TPC;     // column slice: column j, rows g + TPC*e
  const float inv_tau = 1.0f / tau;
  // The CTA (cluster) walks the blocks g = blockIdx.x / CS, + gridDim.x / CS, ...
  // of every layer; the next block's slab of L is loaded into registers while
  // the current one iterates.
  int total = 0;
  for (int i = 0; i < batch.n; ++i) total += batch.layer[i].blocks;
  const int gstride = gridDim.x / CS;
  auto locate = [&](int gb, int& li, int& blk) {
    blk = gb;
    li = 0;
    while (li + 1 < batch.n && blk >= batch.layer[li].blocks) blk -= batch.layer[li++].blocks;
  };
  float4 pre[NPRE];
  auto prefetch = [&](int gb) {
    int li, blk;
    locate(gb, li, blk);
    const float4* src = reinterpret_cast<const float4*>(batch.layer[li].L + (size_t)blk * B * B + (size_t)row0 * B);
#pragma unroll
    for (int k = 0; k < NPRE; ++k) pre[k] = src[tid + k * NT];
  };
  // the look-ahead needs NPRE more registers a thread: not for the 1024-thread B = 256 CTAs
  constexpr bool AHEAD = NPRE <= 2;
  if (AHEAD && blockIdx.x / CS < total) prefetch(blockIdx.x / CS);
  for (int gb = blockIdx.x / CS; gb < total; gb += gstride) {
  if constexpr (!AHEAD) prefetch(gb);
  int li, blk;
  locate(gb, li, blk);
  const SkFwdLayer& ly = batch.layer[li];
  float* __restrict__ P = ly.P;
  float* __restrict__ ckpt = ly.ckpt;
  __nv_bfloat16* __restrict__ pt_hi = ly.pt_hi;
  __nv_bfloat16* __restrict__ pt_lo = ly.pt_lo;
  __nv_bfloat16* __restrict__ p_hi = ly.p_hi;
  if (ly.zero_word && blk == 0 && rank == 0 && tid == 0) *ly.zero_word = 0u;
  const size_t base = (size_t)blk * B * B;
  const size_t ck0 = (size_t)blk * iters * 2 * B;

  // Z_0 = L / tau (as L times the correctly rounded 1 / tau: within an ulp)
#pragma unroll
  for (int k = 0; k < NPRE; ++k) {
    const int q = tid + k * NT;
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    float* d = tile + rr * LD + jj;
    d[0] = pre[k].x * inv_tau; d[1] = pre[k].y * inv_tau; d[2] = pre[k].z * inv_tau; d[3] = pre[k].w * inv_tau;
  }
  if (AHEAD && gb + gstride < total) prefetch(gb + gstride);   // in flight while this block iterates
  __syncthreads();
  float zr[EPR], zc[EPC];
#pragma unroll
  for (int e = 0; e < EPR; ++e) zr[e] = tile[r * LD + c + TPR * e];
#pragma unroll
  for (int e = 0; e < EPC; ++e) zc[e] = tile[(g + TPC * e) * LD + j];
  float lmx = zr[0], lmn = zr[0];
#pragma unroll
  for (int e = 1; e < EPR; ++e) {
    lmx = fmaxf(lmx, zr[e]);
    lmn = fminf(lmn, zr[e]);
  }
  float zmax, zmin;
  block_range<NT, CS>(lmx, lmn, red, zmax, zmin);
  const bool linear = (zmax - zmin) <= kLinearRange;

  float myR = 0.f;   // this thread's row: a_i (linear) or R_i (log domain)
  if (linear) {
#pragma unroll
    for (int e = 0; e < EPR; ++e) zr[e] = __expf(zr[e] - zmax);
#pragma unroll
    for (int e = 0; e < EPC; ++e) zc[e] = __expf(zc[e] - zmax);
    for (int jj = tid; jj < B; jj += NT) cv[jj] = 1.f;
    __syncthreads();
    for (int k = 0; k < iters; ++k) {
      // T_r: a_i = 1 / sum_j K_ij b_j   (R_i = max Z_0 + log of that sum)
      {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < EPR; ++e) s = fmaf(zr[e], cv[c + TPR * e], s);
        s = group_sum<TPR>(s);
        myR = __frcp_rn(s);
        if (c == 0) {
          rv[r] = myR;
          if (ckpt) ckpt[ck0 + (size_t)k * 2 * B + row0 + r] = zmax + __logf(s);
        }
      }
      __syncthreads();
      // T_c: b_j = 1 / sum_i a_i K_ij over all B rows   (C_j = log of that sum)
      {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < EPC; ++e) s = fmaf(zc[e], rv[g + TPC * e], s);
        s = group_sum<TPC>(s);
        if constexpr (CS == 1) {
          if (g == 0) {
            cv[j] = __frcp_rn(s);
            if (ckpt) ckpt[ck0 + ((size_t)k * 2 + 1) * B + j] = __logf(s);
          }
        } else {
          float* bs = xs + (k & 1) * B;
          if (g == 0) bs[j] = s;
          cluster_barrier<CS>();
          if (g == 0) {
            float S = 0.f;
#pragma unroll
            for (int q = 0; q < CS; ++q) S += peer<CS>(bs, q)[j];
            cv[j] = __frcp_rn(S);
            if (ckpt && rank == 0) ckpt[ck0 + ((size_t)k * 2 + 1) * B + j] = __logf(S);
          }
        }
        __syncthreads();
      }
    }
    // P = a_i K_ij b_j, staged through the tile for coalesced stores
#pragma unroll
    for (int e = 0; e < EPR; ++e) tile[r * LD + c + TPR * e] = myR * zr[e] * cv[c + TPR * e];
  } else {
    for (int jj = tid; jj < B; jj += NT) cv[jj] = 0.f;
    __syncthreads();
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
          if (ckpt) ckpt[ck0 + (size_t)k * 2 * B + row0 + r] = myR;
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
            if (ckpt) ckpt[ck0 + ((size_t)k * 2 + 1) * B + j] = v;
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
            if (ckpt && rank == 0) ckpt[ck0 + ((size_t)k * 2 + 1) * B + j] = v;
          }
          __syncthreads();
        }
      }
    }
    // P = exp(Z_0 - R - C), staged through the tile for coalesced stores
#pragma unroll
    for (int e = 0; e < EPR; ++e) tile[r * LD + c + TPR * e] = __expf(zr[e] - myR - cv[c + TPR * e]);
  }
  __syncthreads();
  // P, four consecutive columns a thread (16-byte stores)
  for (int q = tid; q < R * (B / 4); q += NT) {
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    const float* src = tile + rr * LD + jj;
    reinterpret_cast<float4*>(P + base + (size_t)(row0 + rr) * B)[jj / 4] = make_float4(src[0], src[1], src[2], src[3]);
  }
  if (pt_hi) {
    // Operand images for the tensor-core kernels, in tiles of BC = max(B, 64)
    // columns: tile t holds the BC x BC block-diagonal slice of P_B covering
    // channels [t*BC, (t+1)*BC) (for B = 32 two blocks share one tile and the
    // off-diagonal quadrants are written as zeros).  Eight consecutive bf16 a
    // thread (16-byte stores).
    constexpr int BC = B < 64 ? 64 : B;
    const int gcol0 = blk * B;
    const size_t tb = (size_t)(gcol0 / BC) * BC * BC;
    const int q0 = gcol0 % BC;
    const int zc0 = (q0 == 0) ? B : 0;   // the zero quadrant's columns (B < BC)
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    // transposed images: image row q0 + jj, source rows i = row0 + 8 g .. + 7
    for (int q = tid; q < B * (R / 8); q += NT) {
      const int jj = q / (R / 8), g8 = (q % (R / 8)) * 8;
      float hv[8], lv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float p = tile[(g8 + u) * LD + jj];
        const __nv_bfloat16 hi = __float2bfloat16_rn(p);
        hv[u] = __bfloat162float(hi);
        lv[u] = p - hv[u];
      }
      const size_t at = tb + (size_t)(q0 + jj) * BC + q0 + row0 + g8;
      *reinterpret_cast<uint4*>(pt_hi + at) = make_uint4(pack_bf16x2_rn(hv[0], hv[1]), pack_bf16x2_rn(hv[2], hv[3]),
                                                         pack_bf16x2_rn(hv[4], hv[5]), pack_bf16x2_rn(hv[6], hv[7]));
      *reinterpret_cast<uint4*>(pt_lo + at) = make_uint4(pack_bf16x2_rn(lv[0], lv[1]), pack_bf16x2_rn(lv[2], lv[3]),
                                                         pack_bf16x2_rn(lv[4], lv[5]), pack_bf16x2_rn(lv[6], lv[7]));
      if constexpr (B < BC) {
        const size_t az = tb + (size_t)(q0 + jj) * BC + zc0 + row0 + g8;
        *reinterpret_cast<uint4*>(pt_hi + az) = zero4;
        *reinterpret_cast<uint4*>(pt_lo + az) = zero4;
      }
    }
    // P_hi: image row q0 + i, columns q0 + 8 g .. + 7
    for (int q = tid; q < R * (B / 8); q += NT) {
      const int rr = q / (B / 8), g8 = (q % (B / 8)) * 8;
      const float* src = tile + rr * LD + g8;
      const size_t at = tb + (size_t)(q0 + row0 + rr) * BC;
      *reinterpret_cast<uint4*>(p_hi + at + q0 + g8) =
          make_uint4(pack_bf16x2_rn(src[0], src[1]), pack_bf16x2_rn(src[2], src[3]), pack_bf16x2_rn(src[4], src[5]),
                     pack_bf16x2_rn(src[6], src[7]));
      if constexpr (B < BC) *reinterpret_cast<uint4*>(p_hi + at + zc0 + g8) = zero4;
    }
  }
  // every thread (and every CTA of the cluster) is done with this block's shared
  // memory before the next block overwrites it
  if constexpr (CS > 1) cluster_barrier<CS>();
  else __syncthreads();
  }
}

// Reverse.  dZ lives in registers in the row layout.  The iterate after each
// normalisation is rebuilt from the checkpoint: exp(Z) = a_i K_ij b_j with
// a_i = e^{max - R_i}, b_j = e^{-C_j} in the linear arithmetic, exp(Z_0 - R_i -
// C_j) per element in the log domain; the forward kernel's choice is
// recomputed from the same Z_0.  STAGED: the block's whole checkpoint
// (iters x 2 x B floats, already turned into a and b in the linear
// arithmetic) is staged in shared memory once, so an iteration has no global
// load and two barriers; otherwise each iteration fetches its two vectors.
// It runs launches of fewer than LCP_SINKHORN_PAIR_MIN_BLOCKS blocks of 64 (larger ones take
// the two-warps-a-block kernel) and the cluster sizes, so for B <= 64 it takes one CTA an SM
// and the registers that leaves; the range of Z_0 is reduced from the staged registers under
// the barrier that publishes the tile, and the block's checkpoint values are loaded with L and
// dP.
// Shared memory (floats): tile[R*(B+1)] ck[B] ck1[B] part[NW*B] cs[B] xs[2B] red[66]
//                         (+ stage[iters*2*B] when STAGED)
template <int B, bool STAGED>
__global__ void __launch_bounds__(SkCfg<B>::NT, B <= 64 ? 1 : 1024 / SkCfg<B>::NT)
sinkhorn_bwd_kernel(const __grid_constant__ SkBwdBatch batch, float tau, int iters) {
  using C = SkCfg<B>;
  pdl_wait();
  pdl_trigger();
  constexpr int R = C::R, NT = C::NT, CS = C::CS, TPR = C::TPR, EPR = C::EPR, NW = C::NW, LD = C::LD;
  constexpr int NPRE = R * (B / 4) / NT;   // float4 of L and of dP a thread stages per block
  static_assert(NPRE * NT == R * (B / 4), "the slab must split evenly over the threads");
  extern __shared__ __align__(16) float sm[];
  float* tile = sm;
  float* ck = tile + R * LD;   // C^(k+1) (log domain) or b^(k+1) = e^{-C^(k+1)} (linear)
  float* ck1 = ck + B;         // C^(k) or b^(k)
  float* part = ck1 + B;       // per-warp column partial sums
  float* cs = part + NW * B;   // column sums of dZ
  float* xs = cs + B;          // this CTA's column sums for the cluster, double-buffered
  float* red = xs + 2 * B;
  float* stage = red + 66;     // STAGED: [iters][2][B] in the arithmetic's form

  const int rank = cta_rank<CS>();
  const int row0 = rank * R;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r = tid / TPR, c = tid % TPR;
  const float inv_tau = 1.0f / tau;
  // persistent over the blocks of every layer, as the forward kernel: the next
  // block's slabs of L and of dP (its splits summed in index order) are loaded
  // into registers while the current one runs
  int total = 0;
  for (int i = 0; i < batch.n; ++i) total += batch.layer[i].blocks;
  const int gstride = gridDim.x / CS;
  auto locate = [&](int gb, int& li, int& blk) {
    blk = gb;
    li = 0;
    while (li + 1 < batch.n && blk >= batch.layer[li].blocks) blk -= batch.layer[li++].blocks;
  };
  float4 preL[NPRE], preD[NPRE];
  auto prefetch = [&](int gb) {
    int li, blk;
    locate(gb, li, blk);
    const SkBwdLayer& y = batch.layer[li];
    const size_t off = (size_t)blk * B * B + (size_t)row0 * B;
    const size_t sstride = (size_t)y.blocks * B * B;
#pragma unroll
    for (int k = 0; k < NPRE; ++k) {
      const int q = tid + k * NT;
      preL[k] = reinterpret_cast<const float4*>(y.L + off)[q];
      float4 a = reinterpret_cast<const float4*>(y.dP + off)[q];
      for (int sp = 1; sp < y.splits; ++sp) {
        const float4 b = reinterpret_cast<const float4*>(y.dP + (size_t)sp * sstride + off)[q];
        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
      }
      preD[k] = a;
    }
  };
  constexpr bool AHEAD = NPRE <= 2;   // as in the forward kernel
  if (AHEAD && blockIdx.x / CS < total) prefetch(blockIdx.x / CS);
  for (int gb = blockIdx.x / CS; gb < total; gb += gstride) {
  if constexpr (!AHEAD) prefetch(gb);
  int li, blk;
  locate(gb, li, blk);
  const SkBwdLayer& ly = batch.layer[li];
  const float* __restrict__ ckpt = ly.ckpt;
  float* __restrict__ dL = ly.dL;
  const size_t base = (size_t)blk * B * B;
  const float* ckb = ckpt + (size_t)blk * iters * 2 * B;

  float zr[EPR], dz[EPR];
  // the block's checkpoint values this thread stages (STAGED), loaded now so that their latency
  // overlaps the staging of Z_0 and the range reduction
  constexpr int NCK = (STAGED && CS == 1) ? 2 : 0;   // (the cluster CTAs have no registers to spare)
  float ckr[NCK > 0 ? NCK : 1];
  if constexpr (NCK > 0) {
#pragma unroll
    for (int u = 0; u < NCK; ++u) {
      const int q = tid + u * NT;
      ckr[u] = q < iters * 2 * B ? ckb[q] : 0.f;
    }
  }
  float zmax, zmin;
  if constexpr (CS == 1) {
    // Z_0 = L / tau, formed as in the forward kernel, and the range of this thread's values
    // reduced per warp under the barrier that publishes the tile (the same values, so the same
    // range and arithmetic as the forward kernel)
    float lmx = -CUDART_INF_F, lmn = CUDART_INF_F;
#pragma unroll
    for (int k = 0; k < NPRE; ++k) {
      const int q = tid + k * NT;
      const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
      const float z0 = preL[k].x * inv_tau, z1 = preL[k].y * inv_tau, z2 = preL[k].z * inv_tau, z3 = preL[k].w * inv_tau;
      float* d = tile + rr * LD + jj;
      d[0] = z0; d[1] = z1; d[2] = z2; d[3] = z3;
      lmx = fmaxf(lmx, fmaxf(fmaxf(z0, z1), fmaxf(z2, z3)));
      lmn = fminf(lmn, fminf(fminf(z0, z1), fminf(z2, z3)));
    }
    lmx = group_max<32>(lmx);
    lmn = -group_max<32>(-lmn);
    if (lane == 0) {
      red[warp] = lmx;
      red[32 + warp] = lmn;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < EPR; ++e) zr[e] = tile[r * LD + c + TPR * e];
    zmax = red[0];
    zmin = red[32];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      zmax = fmaxf(zmax, red[w]);
      zmin = fminf(zmin, red[32 + w]);
    }
    __syncthreads();   // every thread has read its row slice: the tile is free again
  } else {
    // Z_0 = L / tau, formed as in the forward kernel
#pragma unroll
    for (int k = 0; k < NPRE; ++k) {
      const int q = tid + k * NT;
      const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
      float* d = tile + rr * LD + jj;
      d[0] = preL[k].x * inv_tau; d[1] = preL[k].y * inv_tau; d[2] = preL[k].z * inv_tau; d[3] = preL[k].w * inv_tau;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < EPR; ++e) zr[e] = tile[r * LD + c + TPR * e];
    float lmx = zr[0], lmn = zr[0];
#pragma unroll
    for (int e = 1; e < EPR; ++e) {
      lmx = fmaxf(lmx, zr[e]);
      lmn = fminf(lmn, zr[e]);
    }
    block_range<NT, CS>(lmx, lmn, red, zmax, zmin);   // ends with a barrier: the tile is free again
  }
  const bool linear = (zmax - zmin) <= kLinearRange;
  if (linear) {
#pragma unroll
    for (int e = 0; e < EPR; ++e) zr[e] = __expf(zr[e] - zmax);   // K
  }
  // dP (splits summed)
#pragma unroll
  for (int k = 0; k < NPRE; ++k) {
    const int q = tid + k * NT;
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    float* d = tile + rr * LD + jj;
    d[0] = preD[k].x; d[1] = preD[k].y; d[2] = preD[k].z; d[3] = preD[k].w;
  }
  if (AHEAD && gb + gstride < total) prefetch(gb + gstride);   // in flight while this block runs
  if constexpr (STAGED) {
    // every (R, C) pair in the form the loop uses: a_i = e^{max - R_i} and
    // b_j = e^{-C_j} (linear), R and C as they are (log domain)
#pragma unroll
    for (int u = 0; u < NCK; ++u) {
      const int q = tid + u * NT;
      if (q < iters * 2 * B) {
        const bool is_row = (q / B) % 2 == 0;
        stage[q] = linear ? __expf(is_row ? zmax - ckr[u] : -ckr[u]) : ckr[u];
      }
    }
    for (int q = tid + NCK * NT; q < iters * 2 * B; q += NT) {
      const float v = ckb[q];
      const bool is_row = (q / B) % 2 == 0;
      stage[q] = linear ? __expf(is_row ? zmax - v : -v) : v;
    }
    for (int jj = tid; jj < B; jj += NT) ck1[jj] = linear ? 1.f : 0.f;   // b^(0) = 1, C^(0) = 0
  } else {
    for (int jj = tid; jj < B; jj += NT) {
      const float v = ckb[(size_t)(iters - 1) * 2 * B + B + jj];
      ck[jj] = linear ? __expf(-v) : v;
    }
  }
  __syncthreads();
  // the vectors after iteration k + 1 (k = iters - 1 ... 0): row values of this thread's row,
  // column values, and the column values after iteration k
  auto rowv = [&](int k) -> float {
    if constexpr (STAGED) return stage[(size_t)k * 2 * B + row0 + r];
    else {
      const float v = ckb[(size_t)k * 2 * B + row0 + r];
      return linear ? __expf(zmax - v) : v;
    }
  };
  auto colv = [&](int k) -> const float* {
    if constexpr (STAGED) return stage + (size_t)k * 2 * B + B;
    else return ck;
  };
  auto colv1 = [&](int k) -> const float* {
    if constexpr (STAGED) return k > 0 ? stage + (size_t)(k - 1) * 2 * B + B : ck1;
    else return ck1;
  };
  // dZ = dP (.) P with P the final iterate
  {
    const float rv = rowv(iters - 1);
    const float* cvp = colv(iters - 1);
    if (linear) {
#pragma unroll
      for (int e = 0; e < EPR; ++e) dz[e] = tile[r * LD + c + TPR * e] * (rv * zr[e] * cvp[c + TPR * e]);
    } else {
#pragma unroll
      for (int e = 0; e < EPR; ++e) dz[e] = tile[r * LD + c + TPR * e] * __expf(zr[e] - rv - cvp[c + TPR * e]);
    }
  }

  for (int k = iters - 1; k >= 0; --k) {
    if constexpr (!STAGED) {
      __syncthreads();   // previous iteration done with ck, ck1, part, cs
      for (int jj = tid; jj < B; jj += NT) {
        const float v = ckb[(size_t)k * 2 * B + B + jj];
        const float v1 = (k > 0) ? ckb[(size_t)(k - 1) * 2 * B + B + jj] : 0.f;
        ck[jj] = linear ? __expf(-v) : v;
        ck1[jj] = linear ? __expf(-v1) : v1;
      }
    }
    const float rv = rowv(k);
    const float* cvp = colv(k);
    const float* cvp1 = colv1(k);
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
    if (linear) {
      // column step: dZ -= exp(Z') colsum with exp(Z') = a_i K_ij b_j^(k+1)
#pragma unroll
      for (int e = 0; e < EPR; ++e) dz[e] -= (rv * zr[e] * cvp[c + TPR * e]) * cs[c + TPR * e];
      // row step: dZ -= exp(Z') rowsum with exp(Z') = a_i K_ij b_j^(k)
      float rs = 0.f;
#pragma unroll
      for (int e = 0; e < EPR; ++e) rs += dz[e];
      rs = group_sum<TPR>(rs);
#pragma unroll
      for (int e = 0; e < EPR; ++e) dz[e] -= (rv * zr[e] * cvp1[c + TPR * e]) * rs;
    } else {
      // column step: dZ -= exp(Z') colsum, Z' = z - R^(k+1) - C^(k+1)
#pragma unroll
      for (int e = 0; e < EPR; ++e) dz[e] -= __expf(zr[e] - rv - cvp[c + TPR * e]) * cs[c + TPR * e];
      // row step: dZ -= exp(Z') rowsum, Z' = z - R^(k+1) - C^(k)
      float rs = 0.f;
#pragma unroll
      for (int e = 0; e < EPR; ++e) rs += dz[e];
      rs = group_sum<TPR>(rs);
#pragma unroll
      for (int e = 0; e < EPR; ++e) dz[e] -= __expf(zr[e] - rv - cvp1[c + TPR * e]) * rs;
    }
  }
  // dL = dZ_0 / tau, staged for coalesced stores
  __syncthreads();
#pragma unroll
  for (int e = 0; e < EPR; ++e) tile[r * LD + c + TPR * e] = dz[e] * inv_tau;
  __syncthreads();
  for (int q = tid; q < R * (B / 4); q += NT) {
    const int rr = q / (B / 4), jj = (q % (B / 4)) * 4;
    const float* src = tile + rr * LD + jj;
    reinterpret_cast<float4*>(dL + base + (size_t)(row0 + rr) * B)[jj / 4] = make_float4(src[0], src[1], src[2], src[3]);
  }
  // every thread (and every CTA of the cluster) is done with this block's shared
  // memory before the next block overwrites it
  if constexpr (CS > 1) cluster_barrier<CS>();
  else __syncthreads();
  }
}

// out = sum over s of parts[s] (n floats each, summed in index order), float4-wide.
__global__ void __launch_bounds__(256) sum_splits_kernel(const float4* __restrict__ parts, int splits, size_t n4,
                                                         float4* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float4 a = parts[i];
    for (int s = 1; s < splits; ++s) {
      const float4 b = parts[(size_t)s * n4 + i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    out[i] = a;
  }
}

template <int B> constexpr size_t fwd_cluster_smem() {
  using C = SkCfg<B>;
  return sizeof(float) * (C::R * C::LD + C::R + B + 4 * B + 66);
}
template <int B> constexpr size_t bwd_smem() {
  using C = SkCfg<B>;
  return sizeof(float) * (C::R * C::LD + 2 * B + C::NW * B + B + 2 * B + 66);
}

// the reverse kernel stages the checkpoint in shared memory up to this many bytes
constexpr size_t kStageBytes = 64 * 1024;

// Grid of a persistent Sinkhorn launch: one CTA (cluster) per block, at most
// as many as are resident at once (the kernels walk the remaining blocks).
// ------------------------------------------- forward, one warp per block ---
// B = 64, for launches with many blocks (a whole model's logits): the
// 512-thread kernel above keeps two blocks in flight per SM, and a block's
// iteration is a chain of barriers and short reductions, so at that size it
// runs far below the memory bandwidth.  Here one warp owns a block: lane l
// holds columns 2l and 2l + 1 of all 64 rows of Z_0 (or K) in registers, a
// column sum is the lane's own loop, a row sum a reduce-scatter across the
// warp after which lane l holds the sums of rows 2l and 2l + 1, and the row
// scalings reach every lane through 256 bytes of shared memory.  No barrier
// beyond the warp's own, and about a dozen blocks in flight per SM.  The
// arithmetic (linear or log domain, chosen by the same range test), the
// checkpoint and the outputs are those of sinkhorn_fwd_kernel; only the
// order of the sums differs.
constexpr int kSkWarpWarps = 4;   // warps (blocks in flight) per CTA

// One step of a reduce-scatter across the warp: of v[0, 2N) every lane keeps
// the half selected by `up` and adds the partner lane's copy of it (the
// partner keeps the other half).
template <int N>
__device__ __forceinline__ void rs_step(float (&v)[32], bool up, int o) {
#pragma unroll
  for (int q = 0; q < N; ++q) {
    const float send = up ? v[q] : v[q + N];
    const float keep = up ? v[q + N] : v[q];
    v[q] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}
// Row sums of a 64-row block: part(i) is this lane's partial sum of row i;
// returns the full sums of rows 2 lane and 2 lane + 1 (fixed order).  The
// first step pairs rows q and q + 32 as their partials are formed, so only 32
// partials are ever live.
template <typename F>
__device__ __forceinline__ float2 row_sums(F part, int lane) {
  float v[32];
  const bool up = lane & 16;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const float lo = part(q), hi = part(q + 32);
    v[q] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, 16);
  }
  rs_step<16>(v, lane & 8, 8);
  rs_step<8>(v, lane & 4, 4);
  rs_step<4>(v, lane & 2, 2);
  rs_step<2>(v, lane & 1, 1);
  return make_float2(v[0], v[1]);
}
// (max, sum of exponentials) pairs of a log-sum-exp, combined
__device__ __forceinline__ void lse_add(float& m, float& s, float m2, float s2) {
  const float M = fmaxf(m, m2);
  s = s * __expf(m - M) + s2 * __expf(m2 - M);
  m = M;
}
template <int N>
__device__ __forceinline__ void rs_step_lse(float (&m)[32], float (&s)[32], bool up, int o) {
#pragma unroll
  for (int q = 0; q < N; ++q) {
    const float sm = up ? m[q] : m[q + N], ss = up ? s[q] : s[q + N];
    m[q] = up ? m[q + N] : m[q];
    s[q] = up ? s[q + N] : s[q];
    lse_add(m[q], s[q], __shfl_xor_sync(0xffffffffu, sm, o), __shfl_xor_sync(0xffffffffu, ss, o));
  }
}

__global__ void __launch_bounds__(32 * kSkWarpWarps)
sinkhorn_fwd_warp_kernel(const __grid_constant__ SkFwdBatch batch, float tau, int iters) {
  constexpr int B = 64;
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float rowv[kSkWarpWarps][B];   // a_i (linear) or R_i (log domain)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  float* rv = rowv[warp];
  const float inv_tau = 1.0f / tau;
  int total = 0;
  for (int i = 0; i < batch.n; ++i) total += batch.layer[i].blocks;
  const int nw = gridDim.x * kSkWarpWarps;
  for (int gb = blockIdx.x * kSkWarpWarps + warp; gb < total; gb += nw) {
    int li = 0, blk = gb;
    while (li + 1 < batch.n && blk >= batch.layer[li].blocks) blk -= batch.layer[li++].blocks;
    const SkFwdLayer& ly = batch.layer[li];
    if (ly.zero_word && blk == 0 && lane == 0) *ly.zero_word = 0u;
    const size_t base = (size_t)blk * B * B;
    const size_t ck0 = (size_t)blk * iters * 2 * B;
    float* __restrict__ ckpt = ly.ckpt;
    // Z_0, columns 2 lane and 2 lane + 1 (as L times the correctly rounded 1 / tau)
    float z0[B], z1[B];
    const float2* src = reinterpret_cast<const float2*>(ly.L + base) + lane;
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const float2 x = __ldcs(src + i * (B / 2));
      z0[i] = x.x * inv_tau;
      z1[i] = x.y * inv_tau;
    }
    float mx = z0[0], mn = z0[0];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      mx = fmaxf(mx, fmaxf(z0[i], z1[i]));
      mn = fminf(mn, fminf(z0[i], z1[i]));
    }
    const float zmax = group_max<32>(mx), zmin = -group_max<32>(-mn);
    float b0, b1;   // the lane's columns: b_j (linear) or C_j (log domain)
    if (zmax - zmin <= kLinearRange) {
#pragma unroll
      for (int i = 0; i < B; ++i) {
        z0[i] = __expf(z0[i] - zmax);
        z1[i] = __expf(z1[i] - zmax);
      }
      b0 = b1 = 1.f;
      for (int k = 0; k < iters; ++k) {
        // T_r: a_i = 1 / sum_j K_ij b_j   (R_i = max Z_0 + log of that sum)
        const float2 rs = row_sums([&](int i) { return fmaf(z0[i], b0, z1[i] * b1); }, lane);
        __syncwarp();   // every lane has read the previous row scalings
        reinterpret_cast<float2*>(rv)[lane] = make_float2(__frcp_rn(rs.x), __frcp_rn(rs.y));
        if (ckpt)
          reinterpret_cast<float2*>(ckpt + ck0 + (size_t)k * 2 * B)[lane] =
              make_float2(zmax + __logf(rs.x), zmax + __logf(rs.y));
        __syncwarp();
        // T_c: b_j = 1 / sum_i a_i K_ij   (C_j = log of that sum); rows i = r (mod 4)
        // accumulate separately, then pairwise: four short chains instead of one long one
        float c0, c1;
        {
          float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int i = 0; i < B; i += 4) {
            const float4 a = reinterpret_cast<const float4*>(rv)[i / 4];
            p0[0] = fmaf(a.x, z0[i], p0[0]); p1[0] = fmaf(a.x, z1[i], p1[0]);
            p0[1] = fmaf(a.y, z0[i + 1], p0[1]); p1[1] = fmaf(a.y, z1[i + 1], p1[1]);
            p0[2] = fmaf(a.z, z0[i + 2], p0[2]); p1[2] = fmaf(a.z, z1[i + 2], p1[2]);
            p0[3] = fmaf(a.w, z0[i + 3], p0[3]); p1[3] = fmaf(a.w, z1[i + 3], p1[3]);
          }
          c0 = (p0[0] + p0[1]) + (p0[2] + p0[3]);
          c1 = (p1[0] + p1[1]) + (p1[2] + p1[3]);
        }
        b0 = __frcp_rn(c0);
        b1 = __frcp_rn(c1);
        if (ckpt)
          reinterpret_cast<float2*>(ckpt + ck0 + ((size_t)k * 2 + 1) * B)[lane] = make_float2(__logf(c0), __logf(c1));
      }
      // P = a_i K_ij b_j (a_i of the last row step, in shared memory)
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const float a = rv[i];
        z0[i] = a * z0[i] * b0;
        z1[i] = a * z1[i] * b1;
      }
    } else {
      // log domain (rare: sharply peaked logits).  Z_0 is read again from L (just loaded, so
      // cache-resident) instead of being kept, which leaves the registers to the reductions.
      auto zat = [&](int i, int e) {
        const float2 x = __ldg(src + i * (B / 2));
        return (e ? x.y : x.x) * inv_tau;
      };
      b0 = b1 = 0.f;
      for (int k = 0; k < iters; ++k) {
        // T_r: R_i = LSE_j(z_ij - C_j); the first step pairs rows q and q + 32
        float m[32], s[32];
        {
          const bool up = lane & 16;
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            float mq[2], sq[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float x0 = zat(q + 32 * h, 0) - b0, x1 = zat(q + 32 * h, 1) - b1;
              mq[h] = fmaxf(x0, x1);
              sq[h] = __expf(x0 - mq[h]) + __expf(x1 - mq[h]);
            }
            m[q] = up ? mq[1] : mq[0];
            s[q] = up ? sq[1] : sq[0];
            lse_add(m[q], s[q], __shfl_xor_sync(0xffffffffu, up ? mq[0] : mq[1], 16),
                    __shfl_xor_sync(0xffffffffu, up ? sq[0] : sq[1], 16));
          }
        }
        rs_step_lse<16>(m, s, lane & 8, 8);
        rs_step_lse<8>(m, s, lane & 4, 4);
        rs_step_lse<4>(m, s, lane & 2, 2);
        rs_step_lse<2>(m, s, lane & 1, 1);
        const float R0 = m[0] + __logf(s[0]), R1 = m[1] + __logf(s[1]);
        __syncwarp();
        reinterpret_cast<float2*>(rv)[lane] = make_float2(R0, R1);
        if (ckpt) reinterpret_cast<float2*>(ckpt + ck0 + (size_t)k * 2 * B)[lane] = make_float2(R0, R1);
        __syncwarp();
        // T_c: C_j = LSE_i(z_ij - R_i)
        float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F;
        for (int i = 0; i < B; ++i) {
          const float r = rv[i];
          m0 = fmaxf(m0, zat(i, 0) - r);
          m1 = fmaxf(m1, zat(i, 1) - r);
        }
        float s0 = 0.f, s1 = 0.f;
        for (int i = 0; i < B; ++i) {
          const float r = rv[i];
          s0 += __expf(zat(i, 0) - r - m0);
          s1 += __expf(zat(i, 1) - r - m1);
        }
        b0 = m0 + __logf(s0);
        b1 = m1 + __logf(s1);
        if (ckpt) reinterpret_cast<float2*>(ckpt + ck0 + ((size_t)k * 2 + 1) * B)[lane] = make_float2(b0, b1);
      }
      // P = exp(Z_0 - R - C)
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const float r = rv[i];
        z0[i] = __expf(zat(i, 0) - r - b0);
        z1[i] = __expf(zat(i, 1) - r - b1);
      }
    }
    __syncwarp();   // every lane has read the row vector before the next block rewrites it
    // P, row i: 256 contiguous bytes a warp store
    float2* dst = reinterpret_cast<float2*>(ly.P + base) + lane;
#pragma unroll
    for (int i = 0; i < B; ++i) dst[i * (B / 2)] = make_float2(z0[i], z1[i]);
    if (ly.pt_hi) {
      // operand images (one 64 x 64 tile per block): Pt[j][i] = P[i][j] as
      // bf16 high and low parts -- rows 2 lane and 2 lane + 1 are this lane's
      // columns -- and P_hi[i][j] = bf16(P[i][j])
      __nv_bfloat16* pth = ly.pt_hi + base;
      __nv_bfloat16* ptl = ly.pt_lo + base;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float* col = e ? z1 : z0;
        uint4* oh = reinterpret_cast<uint4*>(pth + (size_t)(2 * lane + e) * B);
        uint4* ol = reinterpret_cast<uint4*>(ptl + (size_t)(2 * lane + e) * B);
#pragma unroll
        for (int g8 = 0; g8 < B / 8; ++g8) {
          float hv[8], lv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float p = col[8 * g8 + u];
            hv[u] = __bfloat162float(__float2bfloat16_rn(p));
            lv[u] = p - hv[u];
          }
          oh[g8] = make_uint4(pack_bf16x2_rn(hv[0], hv[1]), pack_bf16x2_rn(hv[2], hv[3]),
                              pack_bf16x2_rn(hv[4], hv[5]), pack_bf16x2_rn(hv[6], hv[7]));
          ol[g8] = make_uint4(pack_bf16x2_rn(lv[0], lv[1]), pack_bf16x2_rn(lv[2], lv[3]),
                              pack_bf16x2_rn(lv[4], lv[5]), pack_bf16x2_rn(lv[6], lv[7]));
        }
      }
      uint32_t* ph = reinterpret_cast<uint32_t*>(ly.p_hi + base) + lane;
#pragma unroll
      for (int i = 0; i < B; ++i) ph[i * (B / 2)] = pack_bf16x2_rn(z0[i], z1[i]);
    }
  }
}

// ------------------------------------- reverse, two warps per block ---
// B = 64, for launches with many blocks: a pair of warps owns a block, warp h
// of the pair rows [32 h, 32 h + 32), lane l columns 2l and 2l + 1, so that
// both K = exp(Z_0 - max) (or Z_0) and dZ sit in registers (64 values each a
// lane).  A column sum is the lane's own loop plus the partner warp's
// partial, exchanged through shared memory with one 64-thread named barrier
// per column step; a row sum is a reduce-scatter over the warp (lane l ends
// with row 32 h + l), broadcast through 128 bytes of shared memory.  The
// block's checkpoint is staged once in the form the loop uses (a_i =
// e^{max - R_i}, b_j = e^{-C_j}, or R and C).  The steps are those of
// sinkhorn_bwd_kernel.
constexpr int kSkPairSlots = 2;   // blocks in flight per CTA (two warps each)
// shared memory of one slot (floats): checkpoint [iters][2][64], column partials [2 buffers][2 warps][64],
// row sums [2 warps][32], range [2 warps][2]
__host__ __device__ constexpr size_t skp_floats(int iters) { return (size_t)iters * 2 * 64 + 256 + 64 + 4; }

__device__ __forceinline__ void pair_sync(int slot) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + slot) : "memory");
}

// Sum over the warp of v[0, 32) per index -> lane l holds the sum of index l.
__device__ __forceinline__ float rows32_sum(float (&v)[32], int lane) {
  rs_step<16>(v, lane & 16, 16);
  rs_step<8>(v, lane & 8, 8);
  rs_step<4>(v, lane & 4, 4);
  rs_step<2>(v, lane & 2, 2);
  rs_step<1>(v, lane & 1, 1);
  return v[0];
}

template <bool LIN>
__device__ __forceinline__ void skp_steps(float (&d0)[32], float (&d1)[32], const float (&k0)[32],
                                          const float (&k1)[32], const float* stage, float* colp, float* rsum,
                                          int iters, int h, int lane, int slot) {
  constexpr int B = 64;
  for (int k = iters - 1; k >= 0; --k) {
    const float* av = stage + (size_t)k * 2 * B + 32 * h;   // this warp's rows
    const float2 bk = reinterpret_cast<const float2*>(stage + ((size_t)k * 2 + 1) * B)[lane];
    const float2 bk1 = k > 0 ? reinterpret_cast<const float2*>(stage + ((size_t)k * 2 - 1) * B)[lane]
                             : make_float2(LIN ? 1.f : 0.f, LIN ? 1.f : 0.f);
    // column sums of dZ: this warp's rows (rows i = r (mod 4) separately, then pairwise),
    // then both warps' partials in a fixed order
    float c0, c1;
    {
      float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        p0[i & 3] += d0[i];
        p1[i & 3] += d1[i];
      }
      c0 = (p0[0] + p0[1]) + (p0[2] + p0[3]);
      c1 = (p1[0] + p1[1]) + (p1[2] + p1[3]);
    }
    float* cp = colp + (k & 1) * 128;   // double-buffered by iteration
    reinterpret_cast<float2*>(cp + 64 * h)[lane] = make_float2(c0, c1);
    pair_sync(slot);
    const float2 p0 = reinterpret_cast<const float2*>(cp)[lane], p1 = reinterpret_cast<const float2*>(cp + 64)[lane];
    c0 = p0.x + p1.x;
    c1 = p0.y + p1.y;
    // column step: dZ -= exp(Z') colsum, Z' the iterate after the column step k;
    // linear: exp(Z') colsum = (a_i K_ij) (b_j colsum_j)
    const float g0 = bk.x * c0, g1 = bk.y * c1;
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 r4 = *reinterpret_cast<const float4*>(av + i);
      const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if constexpr (LIN) {
          d0[i + u] = fmaf(-(rr[u] * k0[i + u]), g0, d0[i + u]);
          d1[i + u] = fmaf(-(rr[u] * k1[i + u]), g1, d1[i + u]);
        } else {
          d0[i + u] -= __expf(k0[i + u] - rr[u] - bk.x) * c0;
          d1[i + u] -= __expf(k1[i + u] - rr[u] - bk.y) * c1;
        }
      }
    }
    // row step: dZ -= exp(Z'') rowsum, Z'' the iterate after the row step k;
    // linear: exp(Z'') rowsum = (K_ij b_j) (a_i rowsum_i), the row factor formed by the row's lane
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = d0[i] + d1[i];
    const float rs = rows32_sum(v, lane);
    __syncwarp();   // every lane has read the previous row factors
    rsum[lane] = LIN ? av[lane] * rs : rs;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 f4 = *reinterpret_cast<const float4*>(rsum + i);
      const float ff[4] = {f4.x, f4.y, f4.z, f4.w};
      float rr[4];
      if constexpr (!LIN) {
        const float4 r4 = *reinterpret_cast<const float4*>(av + i);
        rr[0] = r4.x; rr[1] = r4.y; rr[2] = r4.z; rr[3] = r4.w;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if constexpr (LIN) {
          d0[i + u] = fmaf(-(k0[i + u] * bk1.x), ff[u], d0[i + u]);
          d1[i + u] = fmaf(-(k1[i + u] * bk1.y), ff[u], d1[i + u]);
        } else {
          d0[i + u] -= __expf(k0[i + u] - rr[u] - bk1.x) * ff[u];
          d1[i + u] -= __expf(k1[i + u] - rr[u] - bk1.y) * ff[u];
        }
      }
    }
  }
}

__global__ void __launch_bounds__(64 * kSkPairSlots, 3)
sinkhorn_bwd_pair_kernel(const __grid_constant__ SkBwdBatch batch, float tau, int iters) {
  constexpr int B = 64;
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) float skp_smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int slot = warp >> 1, h = warp & 1;
  float* stage = skp_smem + (size_t)slot * skp_floats(iters);
  float* colp = stage + (size_t)iters * 2 * B;
  float* rsum = colp + 256 + 32 * h;
  float* rng = colp + 256 + 64;
  const float inv_tau = 1.0f / tau;
  int total = 0;
  for (int i = 0; i < batch.n; ++i) total += batch.layer[i].blocks;
  const int ns = gridDim.x * kSkPairSlots;
  for (int gb = blockIdx.x * kSkPairSlots + slot; gb < total; gb += ns) {
    int li = 0, blk = gb;
    while (li + 1 < batch.n && blk >= batch.layer[li].blocks) blk -= batch.layer[li++].blocks;
    const SkBwdLayer& ly = batch.layer[li];
    const size_t base = (size_t)blk * B * B + (size_t)32 * h * B;   // this warp's first row
    const float* ckb = ly.ckpt + (size_t)blk * iters * 2 * B;
    // Z_0 (as in the forward kernel) and its range over the block
    float k0[32], k1[32];
    const float2* lsrc = reinterpret_cast<const float2*>(ly.L + base) + lane;
    float mx = -CUDART_INF_F, mn = CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float2 x = __ldcs(lsrc + i * (B / 2));
      k0[i] = x.x * inv_tau;
      k1[i] = x.y * inv_tau;
      mx = fmaxf(mx, fmaxf(k0[i], k1[i]));
      mn = fminf(mn, fminf(k0[i], k1[i]));
    }
    mx = group_max<32>(mx);
    mn = -group_max<32>(-mn);
    if (lane == 0) {
      rng[2 * h] = mx;
      rng[2 * h + 1] = mn;
    }
    // dP of this warp's rows, splits summed in index order
    float d0[32], d1[32];
    {
      const size_t sstride = (size_t)ly.blocks * B * B;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float2 a = __ldcs(reinterpret_cast<const float2*>(ly.dP + base) + lane + i * (B / 2));
        for (int sp = 1; sp < ly.splits; ++sp) {
          const float2 bb = __ldcs(reinterpret_cast<const float2*>(ly.dP + (size_t)sp * sstride + base) + lane + i * (B / 2));
          a.x += bb.x;
          a.y += bb.y;
        }
        d0[i] = a.x;
        d1[i] = a.y;
      }
    }
    pair_sync(slot);   // both ranges written; the previous block's use of the slot is over
    const float zmax = fmaxf(rng[0], rng[2]), zmin = fminf(rng[1], rng[3]);
    const bool linear = zmax - zmin <= kLinearRange;
    if (linear) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        k0[i] = __expf(k0[i] - zmax);
        k1[i] = __expf(k1[i] - zmax);
      }
    }
    // the checkpoint, warp h its vectors q = h, h + 2, ... (lane l entries 2l and 2l + 1)
    for (int q = h; q < iters * 2; q += 2) {
      const float2 v = reinterpret_cast<const float2*>(ckb + (size_t)q * B)[lane];
      const bool is_row = (q & 1) == 0;
      reinterpret_cast<float2*>(stage + (size_t)q * B)[lane] =
          linear ? (is_row ? make_float2(__expf(zmax - v.x), __expf(zmax - v.y)) : make_float2(__expf(-v.x), __expf(-v.y)))
                 : v;
    }
    pair_sync(slot);
    // dZ = dP (.) P, P the final iterate
    {
      const float2 bL = reinterpret_cast<const float2*>(stage + ((size_t)(iters - 1) * 2 + 1) * B)[lane];
      const float* aL = stage + (size_t)(iters - 1) * 2 * B + 32 * h;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float ri = aL[i];
        d0[i] *= linear ? ri * k0[i] * bL.x : __expf(k0[i] - ri - bL.x);
        d1[i] *= linear ? ri * k1[i] * bL.y : __expf(k1[i] - ri - bL.y);
      }
    }
    if (linear) skp_steps<true>(d0, d1, k0, k1, stage, colp, rsum, iters, h, lane, slot);
    else skp_steps<false>(d0, d1, k0, k1, stage, colp, rsum, iters, h, lane, slot);
    // dL = dZ_0 / tau, row i: 256 contiguous bytes a warp store
    float2* dst = reinterpret_cast<float2*>(ly.dL + base) + lane;
#pragma unroll
    for (int i = 0; i < 32; ++i) dst[i * (B / 2)] = make_float2(d0[i] * inv_tau, d1[i] * inv_tau);
  }
}

template <typename K>
int grid_blocks(K kernel, int nt, size_t smem, int cs, int blocks) {
  int per_sm = 1, sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, nt, smem) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();   // this query's own error
    per_sm = 1;
  }
  const int resident = std::max(1, per_sm * sms / cs);
  return std::min(blocks, resident);
}

template <int B>
lcp_status fwd_b(const SkFwdBatch& batch, int blocks, float tau, int iters, cudaStream_t st) {
  if (B == 64 && blocks >= LCP_SINKHORN_WARP_MIN_BLOCKS) {
    // one warp a block: enough blocks to keep every SM's warps busy
    const int g = grid_blocks(sinkhorn_fwd_warp_kernel, 32 * kSkWarpWarps, 0, 1,
                              (blocks + kSkWarpWarps - 1) / kSkWarpWarps);
    return launch_kernel(sinkhorn_fwd_warp_kernel, dim3(g), dim3(32 * kSkWarpWarps), 0, st, 1, true, "sinkhorn_fwd",
                         batch, tau, iters);
  }
  if constexpr (SkCfg<B>::CS > 1) {
    using C = SkCfg<B>;
    const size_t smem = fwd_cluster_smem<B>();
    const lcp_status s0 = ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_fwd_cluster_kernel<B>),
                                            (int)smem, "sinkhorn_fwd");
    if (s0 != LCP_OK) return s0;
    const int g = grid_blocks(sinkhorn_fwd_cluster_kernel<B>, C::NT, smem, C::CS, blocks);
    return launch_kernel(sinkhorn_fwd_cluster_kernel<B>, dim3(g * C::CS), dim3(C::NT), smem, st, C::CS, true,
                         "sinkhorn_fwd", batch, tau, iters);
  } else {
    using C = SkFwdCfg<B>;
    const size_t smem = fwd_smem_base<B>();
    const lcp_status s0 =
        ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_fwd_kernel<B>), (int)smem, "sinkhorn_fwd");
    if (s0 != LCP_OK) return s0;
    const int g = grid_blocks(sinkhorn_fwd_kernel<B>, C::NT, smem, C::CS, blocks);
    return launch_kernel(sinkhorn_fwd_kernel<B>, dim3(g * C::CS), dim3(C::NT), smem, st, C::CS, true,
                         "sinkhorn_fwd", batch, tau, iters);
  }
}

template <int B>
lcp_status bwd_b(const SkBwdBatch& batch, int blocks, float tau, int iters, cudaStream_t st) {
  using C = SkCfg<B>;
  const size_t pbytes = kSkPairSlots * skp_floats(iters) * sizeof(float);
  if (B == 64 && blocks >= LCP_SINKHORN_PAIR_MIN_BLOCKS && pbytes <= 96 * 1024) {
    // two warps a block, everything in registers
    const lcp_status s0 =
        ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_bwd_pair_kernel), (int)pbytes, "sinkhorn_bwd");
    if (s0 != LCP_OK) return s0;
    const int g = grid_blocks(sinkhorn_bwd_pair_kernel, 64 * kSkPairSlots, pbytes, 1,
                              (blocks + kSkPairSlots - 1) / kSkPairSlots);
    return launch_kernel(sinkhorn_bwd_pair_kernel, dim3(g), dim3(64 * kSkPairSlots), pbytes, st, 1, true,
                         "sinkhorn_bwd", batch, tau, iters);
  }
  const size_t stage = (size_t)iters * 2 * B * sizeof(float);
  if (stage <= kStageBytes) {
    const size_t bytes = bwd_smem<B>() + stage;
    const lcp_status s0 = ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_bwd_kernel<B, true>), (int)bytes,
                                            "sinkhorn_bwd");
    if (s0 != LCP_OK) return s0;
    const int g = grid_blocks(sinkhorn_bwd_kernel<B, true>, C::NT, bytes, C::CS, blocks);
    return launch_kernel(sinkhorn_bwd_kernel<B, true>, dim3(g * C::CS), dim3(C::NT), bytes, st, C::CS, true,
                         "sinkhorn_bwd", batch, tau, iters);
  }
  const lcp_status s0 = ensure_smem_limit(reinterpret_cast<const void*>(sinkhorn_bwd_kernel<B, false>),
                                          (int)bwd_smem<B>(), "sinkhorn_bwd");
  if (s0 != LCP_OK) return s0;
  const int g = grid_blocks(sinkhorn_bwd_kernel<B, false>, C::NT, bwd_smem<B>(), C::CS, blocks);
  return launch_kernel(sinkhorn_bwd_kernel<B, false>, dim3(g * C::CS), dim3(C::NT), bwd_smem<B>(), st, C::CS,
                       true, "sinkhorn_bwd", batch, tau, iters);
}

// Launches `kernel_b` over `layers` in batches of up to kSkMaxLayers layers.
template <typename Layer, typename Batch, typename F>
lcp_status in_batches(const Layer* layers, int n, F launch) {
  for (int first = 0; first < n; first += kSkMaxLayers) {
    Batch b{};
    b.n = std::min(kSkMaxLayers, n - first);
    int blocks = 0;
    for (int i = 0; i < b.n; ++i) {
      b.layer[i] = layers[first + i];
      blocks += b.layer[i].blocks;
    }
    if (blocks == 0) continue;
    const lcp_status s = launch(b, blocks);
    if (s != LCP_OK) return s;
  }
  return LCP_OK;
}

}  // namespace

lcp_status launch_sinkhorn_fwd_batch(const SkFwdLayer* layers, int n, int B, float tau, int iters,
                                     cudaStream_t st) {
  return in_batches<SkFwdLayer, SkFwdBatch>(layers, n, [&](const SkFwdBatch& b, int blocks) -> lcp_status {
    switch (B) {
      case 32: return fwd_b<32>(b, blocks, tau, iters, st);
      case 64: return fwd_b<64>(b, blocks, tau, iters, st);
      case 128: return fwd_b<128>(b, blocks, tau, iters, st);
      case 256: return fwd_b<256>(b, blocks, tau, iters, st);
    }
    return fail(LCP_ERR_SHAPE, "sinkhorn_fwd: unsupported block size %d", B);
  });
}

lcp_status launch_sinkhorn_fwd(const float* L, float* P, float* ckpt, __nv_bfloat16* img_pt_hi,
                               __nv_bfloat16* img_pt_lo, __nv_bfloat16* img_p_hi, unsigned* zero_word,
                               int nblocks, int B, float tau, int iters, cudaStream_t st) {
  const SkFwdLayer one{L, P, ckpt, img_pt_hi, img_pt_lo, img_p_hi, zero_word, nblocks};
  return launch_sinkhorn_fwd_batch(&one, 1, B, tau, iters, st);
}

lcp_status launch_sum_splits(const float* parts, int splits, size_t n, float* out, cudaStream_t st) {
  const size_t n4 = n / 4;
  const int grid = (int)std::min<size_t>((n4 + 255) / 256, 148 * 8);
  return launch_kernel(sum_splits_kernel, dim3(grid > 0 ? grid : 1), dim3(256), 0, st, 1, true, "sum_splits",
                       reinterpret_cast<const float4*>(parts), splits, n4, reinterpret_cast<float4*>(out));
}

lcp_status launch_sinkhorn_bwd_batch(const SkBwdLayer* layers, int n, int B, float tau, int iters,
                                     cudaStream_t st) {
  return in_batches<SkBwdLayer, SkBwdBatch>(layers, n, [&](const SkBwdBatch& b, int blocks) -> lcp_status {
    switch (B) {
      case 32: return bwd_b<32>(b, blocks, tau, iters, st);
      case 64: return bwd_b<64>(b, blocks, tau, iters, st);
      case 128: return bwd_b<128>(b, blocks, tau, iters, st);
      case 256: return bwd_b<256>(b, blocks, tau, iters, st);
    }
    return fail(LCP_ERR_SHAPE, "sinkhorn_bwd: unsupported block size %d", B);
  });
}

lcp_status launch_sinkhorn_bwd(const float* L, const float* ckpt, const float* dP, int splits,
                               float* dL, int nblocks, int B, float tau, int iters,
                               cudaStream_t st) {
  const SkBwdLayer one{L, ckpt, dP, dL, splits, nblocks};
  return launch_sinkhorn_bwd_batch(&one, 1, B, tau, iters, st);
}

}  // namespace lcp
