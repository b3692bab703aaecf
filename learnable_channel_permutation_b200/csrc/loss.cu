// Token-averaged cosine loss between the dense and sparse outputs and its
// gradient with respect to the sparse output (PermLLM summary, "optimization
// objective": L_cos(y, y~) = 1 - y.y~ / (|y| |y~|)), averaged over tokens.
//
//   c_t  = <yd_t, ys_t> / max(|yd_t| |ys_t|, 1e-8)
//   loss = (1/T) sum_t (1 - c_t)
//   G_t  = -(1/T) (yd_t / (|yd_t||ys_t|) - c_t ys_t / |ys_t|^2)
//
// One CTA per token reads its two rows with 128-bit loads, reduces in a fixed
// order (deterministic), writes the four per-token statistics and optionally
// G; a one-CTA kernel then sums the T cosines in a fixed order.

#include "lcp_internal.cuh"

namespace lcp {
namespace {

constexpr float kCosEps = 1e-8f;
constexpr int NT = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename TG>
__device__ __forceinline__ void write_g(TG* G, size_t off, float4 g);
template <>
__device__ __forceinline__ void write_g<float>(float* G, size_t off, float4 g) {
  *reinterpret_cast<float4*>(G + off) = g;
}
template <>
__device__ __forceinline__ void write_g<__nv_bfloat16>(__nv_bfloat16* G, size_t off, float4 g) {
  __nv_bfloat162 a = __floats2bfloat162_rn(g.x, g.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(g.z, g.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(G + off) = u;
}

template <typename TG>
__device__ __forceinline__ void token_grad(const float4* yd, const float4* ys, TG* G, size_t row,
                                           int quads, float dot, float nd2, float ns2,
                                           float inv_T) {
  const float den = sqrtf(nd2) * sqrtf(ns2);
  const bool ok = den > kCosEps;
  const float c = dot / fmaxf(den, kCosEps);
  const float a = ok ? -inv_T / den : -inv_T / kCosEps;     // coefficient of yd
  const float b = ok ? inv_T * c / ns2 : 0.f;               // coefficient of ys
  for (int q = threadIdx.x; q < quads; q += NT) {
    const float4 d = yd[q], s = ys[q];
    float4 g;
    g.x = a * d.x + b * s.x;
    g.y = a * d.y + b * s.y;
    g.z = a * d.z + b * s.z;
    g.w = a * d.w + b * s.w;
    write_g<TG>(G, row + 4 * (size_t)q, g);
  }
}

template <typename TG, bool WRITE_G>
__global__ void __launch_bounds__(NT)
loss_token_kernel(const float* __restrict__ Yd, const float* __restrict__ Ys,
                  float* __restrict__ stats, TG* __restrict__ G, int cout, float inv_T) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[3][NT / 32];
  const int t = blockIdx.x;
  const size_t row = (size_t)t * cout;
  const float4* yd = reinterpret_cast<const float4*>(Yd + row);
  const float4* ys = reinterpret_cast<const float4*>(Ys + row);
  const int quads = cout / 4;
  float dot = 0.f, nd = 0.f, ns = 0.f;
  for (int q = threadIdx.x; q < quads; q += NT) {
    const float4 a = yd[q], b = ys[q];
    dot += a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
    nd += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    ns += b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
  }
  dot = warp_sum(dot);
  nd = warp_sum(nd);
  ns = warp_sum(ns);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) { red[0][warp] = dot; red[1][warp] = nd; red[2][warp] = ns; }
  __syncthreads();
  dot = 0.f; nd = 0.f; ns = 0.f;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) { dot += red[0][w]; nd += red[1][w]; ns += red[2][w]; }
  if (threadIdx.x == 0) {
    const float c = dot / fmaxf(sqrtf(nd) * sqrtf(ns), kCosEps);
    float4 s;
    s.x = dot; s.y = nd; s.z = ns; s.w = c;
    reinterpret_cast<float4*>(stats)[t] = s;
  }
  if constexpr (WRITE_G) token_grad<TG>(yd, ys, G, row, quads, dot, nd, ns, inv_T);
}

template <typename TG>
__global__ void __launch_bounds__(NT)
loss_grad_kernel(const float* __restrict__ Yd, const float* __restrict__ Ys,
                 const float* __restrict__ stats, TG* __restrict__ G, int cout, float inv_T) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const size_t row = (size_t)t * cout;
  const float4 s = reinterpret_cast<const float4*>(stats)[t];
  token_grad<TG>(reinterpret_cast<const float4*>(Yd + row), reinterpret_cast<const float4*>(Ys + row),
                 G, row, cout / 4, s.x, s.y, s.z, inv_T);
}

// Fused variant used inside a step.  Persistent CTAs walk the tokens
// t = blockIdx.x, blockIdx.x + gridDim.x, ...; each thread keeps QPT float4
// quads of the current token's two rows in registers and already holds the
// next token's rows (loaded while the current one is reduced), so Y is read
// from HBM once with the loads always in flight.  The CTA that finishes last
// (a counter zeroed by the caller before the launch) sums the T cosines in
// index order into the loss and re-zeroes the counter: deterministic.
template <typename TG, int NTH, int QPT, bool PREFETCH>
__global__ void __launch_bounds__(NTH, PREFETCH ? 2 : 1)
loss_fused_kernel(const float* __restrict__ Yd, const float* __restrict__ Ys, float* __restrict__ stats,
                  TG* __restrict__ G, float* __restrict__ loss, unsigned* __restrict__ counter, int cout,
                  int tokens, int norm, float inv_T) {
  pdl_wait();
  pdl_trigger();
  constexpr int NWARP = NTH / 32;
  __shared__ float red[2][3][NWARP];
  __shared__ double redd[NWARP];
  __shared__ int is_last;
  const int quads = cout / 4;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  float4 a[QPT], b[QPT], na[QPT], nb[QPT];
  auto load = [&](int t, float4 (&x)[QPT], float4 (&y)[QPT]) {
    const float4* yd = reinterpret_cast<const float4*>(Yd + (size_t)t * cout);
    const float4* ys = reinterpret_cast<const float4*>(Ys + (size_t)t * cout);
#pragma unroll
    for (int i = 0; i < QPT; ++i) {
      const int q = threadIdx.x + i * NTH;
      if (t < tokens && q < quads) { x[i] = __ldcs(yd + q); y[i] = __ldcs(ys + q); }
      else { x[i] = make_float4(0.f, 0.f, 0.f, 0.f); y[i] = x[i]; }
    }
  };
  int t = blockIdx.x;
  if constexpr (PREFETCH) load(t, na, nb);
  for (int it = 0; t < tokens; t += gridDim.x, ++it) {
    if constexpr (PREFETCH) {
#pragma unroll
      for (int i = 0; i < QPT; ++i) { a[i] = na[i]; b[i] = nb[i]; }
      load(t + gridDim.x, na, nb);          // next token, in flight during this one
    } else {
      load(t, a, b);
    }
    float dot = 0.f, nd = 0.f, ns = 0.f;
#pragma unroll
    for (int i = 0; i < QPT; ++i) {
      dot += a[i].x * b[i].x + a[i].y * b[i].y + a[i].z * b[i].z + a[i].w * b[i].w;
      nd += a[i].x * a[i].x + a[i].y * a[i].y + a[i].z * a[i].z + a[i].w * a[i].w;
      ns += b[i].x * b[i].x + b[i].y * b[i].y + b[i].z * b[i].z + b[i].w * b[i].w;
    }
    dot = warp_sum(dot);
    nd = warp_sum(nd);
    ns = warp_sum(ns);
    const int p = it & 1;   // double-buffered partials: one barrier per token
    if (lane == 0) { red[p][0][warp] = dot; red[p][1][warp] = nd; red[p][2][warp] = ns; }
    __syncthreads();
    dot = 0.f; nd = 0.f; ns = 0.f;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) { dot += red[p][0][w]; nd += red[p][1][w]; ns += red[p][2][w]; }
    const float den = sqrtf(nd) * sqrtf(ns);
    const float c = dot / fmaxf(den, kCosEps);
    if (threadIdx.x == 0) {
      float4 sv;
      sv.x = dot; sv.y = nd; sv.z = ns; sv.w = c;
      reinterpret_cast<float4*>(stats)[t] = sv;
    }
    const bool ok = den > kCosEps;
    const float ca = ok ? -inv_T / den : -inv_T / kCosEps;
    const float cb = ok ? inv_T * c / ns : 0.f;
    const size_t row = (size_t)t * cout;
#pragma unroll
    for (int i = 0; i < QPT; ++i) {
      const int q = threadIdx.x + i * NTH;
      if (q < quads) {
        float4 g;
        g.x = ca * a[i].x + cb * b[i].x;
        g.y = ca * a[i].y + cb * b[i].y;
        g.z = ca * a[i].z + cb * b[i].z;
        g.w = ca * a[i].w + cb * b[i].w;
        write_g<TG>(G, row + 4 * (size_t)q, g);
      }
    }
  }
  // last CTA: the loss.  Thread 0 wrote this CTA's statistics; its fence
  // orders those writes before its vote, so the last voter sees every token.
  if (threadIdx.x == 0) {
    __threadfence();
    is_last = (atomicAdd(counter, 1u) == gridDim.x - 1u);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double sum = 0.0;
  for (int u = threadIdx.x; u < tokens; u += NTH) sum += 1.0 - (double)__ldcg(stats + 4 * (size_t)u + 3);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) redd[warp] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < NWARP; ++w) tot += redd[w];
    *loss = (float)(tot / norm);
    *counter = 0u;
  }
}

// The loss and its gradient from the calibration GEMM's loss epilogue
// (gemm_tc.cu, LOSS mode): per token t, the float4 partial sums
// (<y_d, y_s>, |y_d|^2, |y_s|^2, 0) of its nslots 64-channel slots, and the
// pair D = Y_d - Y_s, Y_s in bf16.  One warp per token, warps persistent over
// the tokens, no barrier between them: the warp issues its first row loads,
// sums the slot partials (lane-strided, then a butterfly: a fixed order) into
// c_t, and streams the rows in steps of NS 16-byte chunks a lane, the next
// step's loads in flight, writing G_t = ca y_d + cb y_s with y_d = D + Y_s,
// y_s = Y_s and the coefficients of token_grad in bf16, and stats[t] as
// loss_token_kernel writes it.  The CTA that finishes last (counter zero at
// launch) sums the cosines in index order into the loss and re-zeroes the
// counter: deterministic.
constexpr int kPairThreads = 256;

template <int NS>
__global__ void __launch_bounds__(kPairThreads)
loss_pair_kernel(const __nv_bfloat16* __restrict__ D, const __nv_bfloat16* __restrict__ Ys,
                 const float4* __restrict__ part, int nslots, float* __restrict__ stats,
                 __nv_bfloat16* __restrict__ G, float* __restrict__ loss, unsigned* __restrict__ counter, int cout,
                 int tokens, int norm, float inv_T) {
  constexpr int NWARP = kPairThreads / 32, STEP = 32 * NS;   // chunks of one step
  pdl_wait();
  pdl_trigger();
  __shared__ double redd[NWARP];
  __shared__ int is_last;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // token t goes to CTA t % gridDim.x: every SM gets the same number of tokens to within one
  const int gw = warp * gridDim.x + blockIdx.x, nw = gridDim.x * NWARP;
  const int oct = cout / 8;   // 16-byte chunks of 8 bf16 per row
  for (int t = gw; t < tokens; t += nw) {
    const uint4* d8 = reinterpret_cast<const uint4*>(D + (size_t)t * cout);
    const uint4* y8 = reinterpret_cast<const uint4*>(Ys + (size_t)t * cout);
    uint4* g8 = reinterpret_cast<uint4*>(G + (size_t)t * cout);
    uint4 d[NS], y[NS], dn[NS], yn[NS];
    auto load = [&](int q0, uint4 (&dd)[NS], uint4 (&yy)[NS]) {
#pragma unroll
      for (int u = 0; u < NS; ++u) {
        const int q = q0 + lane + 32 * u;
        if (q < oct) {
          dd[u] = __ldcs(d8 + q);
          yy[u] = __ldcs(y8 + q);
        }
      }
    };
    load(0, dn, yn);
    float dot = 0.f, nd2 = 0.f, ns2 = 0.f;
    for (int k = lane; k < nslots; k += 32) {
      const float4 p = __ldcs(part + (size_t)t * nslots + k);
      dot += p.x;
      nd2 += p.y;
      ns2 += p.z;
    }
    dot = warp_sum(dot);
    nd2 = warp_sum(nd2);
    ns2 = warp_sum(ns2);
    const float den = sqrtf(nd2) * sqrtf(ns2);
    const float c = dot / fmaxf(den, kCosEps);
    if (lane == 0) {
      float4 sv;
      sv.x = dot; sv.y = nd2; sv.z = ns2; sv.w = c;
      reinterpret_cast<float4*>(stats)[t] = sv;
    }
    const bool ok = den > kCosEps;
    const float ca = ok ? -inv_T / den : -inv_T / kCosEps;   // coefficient of y_d
    const float cb = ok ? inv_T * c / ns2 : 0.f;             // coefficient of y_s
    for (int q0 = 0; q0 < oct; q0 += STEP) {
#pragma unroll
      for (int u = 0; u < NS; ++u) { d[u] = dn[u]; y[u] = yn[u]; }
      if (q0 + STEP < oct) load(q0 + STEP, dn, yn);   // the next step's chunks, in flight meanwhile
#pragma unroll
      for (int u = 0; u < NS; ++u) {
        const int q = q0 + lane + 32 * u;
        if (q < oct) {
          const uint32_t dw[4] = {d[u].x, d[u].y, d[u].z, d[u].w};
          const uint32_t yw[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
          uint32_t gwd[4];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const float2 df = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dw[v]));
            const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&yw[v]));
            const __nv_bfloat162 gv =
                __floats2bfloat162_rn(ca * (df.x + yf.x) + cb * yf.x, ca * (df.y + yf.y) + cb * yf.y);
            gwd[v] = *reinterpret_cast<const uint32_t*>(&gv);
          }
          g8[q] = make_uint4(gwd[0], gwd[1], gwd[2], gwd[3]);
        }
      }
    }
  }
  // last CTA: the loss (as in loss_fused_kernel).  Every lane 0 wrote its
  // warp's statistics; the barrier and thread 0's fence order them before the
  // CTA's vote.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    is_last = (atomicAdd(counter, 1u) == gridDim.x - 1u);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double sum = 0.0;
  for (int u = threadIdx.x; u < tokens; u += kPairThreads) sum += 1.0 - (double)__ldcg(stats + 4 * (size_t)u + 3);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) redd[warp] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < NWARP; ++w) tot += redd[w];
    *loss = (float)(tot / norm);
    *counter = 0u;
  }
}

__global__ void __launch_bounds__(1024)
loss_reduce_kernel(const float* __restrict__ stats, float* __restrict__ loss, int tokens, int norm) {
  pdl_wait();
  pdl_trigger();
  __shared__ double red[32];
  double s = 0.0;
  for (int t = threadIdx.x; t < tokens; t += 1024) s += 1.0 - (double)stats[4 * (size_t)t + 3];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 32; ++w) tot += red[w];
    *loss = (float)(tot / norm);
  }
}

}  // namespace

lcp_status launch_loss_token(const float* Yd, const float* Ys, float* stats, void* G,
                             lcp_dtype gdt, int cout, int tokens, int norm, cudaStream_t st) {
  const float inv_T = 1.0f / (float)norm;
  const dim3 grid(tokens), block(NT);
  if (!G)
    return launch_kernel(loss_token_kernel<float, false>, grid, block, 0, st, 1, true, "loss_token", Yd, Ys, stats,
                         (float*)nullptr, cout, inv_T);
  if (gdt == LCP_F32)
    return launch_kernel(loss_token_kernel<float, true>, grid, block, 0, st, 1, true, "loss_token", Yd, Ys, stats,
                         (float*)G, cout, inv_T);
  return launch_kernel(loss_token_kernel<__nv_bfloat16, true>, grid, block, 0, st, 1, true, "loss_token", Yd, Ys,
                       stats, (__nv_bfloat16*)G, cout, inv_T);
}

lcp_status launch_loss_grad(const float* Yd, const float* Ys, const float* stats, void* G,
                            lcp_dtype gdt, int cout, int tokens, int norm, cudaStream_t st) {
  const float inv_T = 1.0f / (float)norm;
  const dim3 grid(tokens), block(NT);
  if (gdt == LCP_F32)
    return launch_kernel(loss_grad_kernel<float>, grid, block, 0, st, 1, true, "loss_grad", Yd, Ys, stats,
                         (float*)G, cout, inv_T);
  return launch_kernel(loss_grad_kernel<__nv_bfloat16>, grid, block, 0, st, 1, true, "loss_grad", Yd, Ys, stats,
                       (__nv_bfloat16*)G, cout, inv_T);
}

bool loss_fused_supported(int cout) { return cout <= 8 * 4 * 512; }

lcp_status launch_loss_fused(const float* Yd, const float* Ys, float* stats, void* G, lcp_dtype gdt,
                             float* loss, unsigned* counter, int cout, int tokens, int norm, cudaStream_t st) {
  const float inv_T = 1.0f / (float)norm;
  const int quads = cout / 4;
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const dim3 grid(tokens < 2 * sms ? tokens : 2 * sms);
#define LCP_LOSS_FUSED(TG, NTH, QPT)                                                                             \
  return launch_kernel(loss_fused_kernel<TG, NTH, QPT, (QPT <= 4)>, grid, dim3(NTH), 0, st, 1, true, "loss_fused", \
                       Yd, Ys, stats, static_cast<TG*>(G), loss, counter, cout, tokens, norm, inv_T)
  if (gdt == LCP_F32) {
    if (quads <= 4 * 256) LCP_LOSS_FUSED(float, 256, 4);
    if (quads <= 8 * 256) LCP_LOSS_FUSED(float, 256, 8);
    LCP_LOSS_FUSED(float, 512, 8);
  }
  if (quads <= 4 * 256) LCP_LOSS_FUSED(__nv_bfloat16, 256, 4);
  if (quads <= 8 * 256) LCP_LOSS_FUSED(__nv_bfloat16, 256, 8);
  LCP_LOSS_FUSED(__nv_bfloat16, 512, 8);
#undef LCP_LOSS_FUSED
}

bool loss_pair_supported(int cout) { return cout <= 16384; }

// 16-byte chunks a lane streams per step of loss_pair_kernel (tuning)
#ifndef LCP_LOSS_PAIR_NS
#define LCP_LOSS_PAIR_NS 4
#endif

lcp_status launch_loss_pair(const __nv_bfloat16* D, const __nv_bfloat16* Ys, const float* partials, int nslots,
                            float* stats, __nv_bfloat16* G, float* loss, unsigned* counter, int cout, int tokens,
                            int norm, cudaStream_t st) {
  constexpr int NS = LCP_LOSS_PAIR_NS;
  int sms = 148, dev = 0, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, loss_pair_kernel<NS>, kPairThreads, 0) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();   // this query's own error
    per_sm = 1;
  }
  // every resident CTA (at most one a token), the tokens interleaved over them
  const int resident = per_sm * sms;
  return launch_kernel(loss_pair_kernel<NS>, dim3(tokens < resident ? tokens : resident), dim3(kPairThreads), 0, st, 1,
                       true, "loss_pair", D, Ys, reinterpret_cast<const float4*>(partials), nslots, stats, G, loss,
                       counter, cout, tokens, norm, 1.0f / (float)norm);
}

lcp_status launch_loss_reduce(const float* stats, float* loss, int tokens, int norm, cudaStream_t st) {
  return launch_kernel(loss_reduce_kernel, dim3(1), dim3(1024), 0, st, 1, true, "loss_reduce", stats, loss, tokens,
                       norm);
}

}  // namespace lcp
