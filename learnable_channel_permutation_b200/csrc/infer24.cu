// Inference side of a PermLLM layer (PermLLM summary, "Effect on inference
// acceleration": at run time the layer permutes its input channels with a
// custom kernel and multiplies by the 2:4 sparse weight).
//
// The deployed weight is A = M.(W P_B) for the hard block permutation P_B
// and a 2:4 mask M, in permuted column order, stored compressed:
//   values [C_out, C_in/2]  the two kept entries of every group of four
//                           columns, in column order;
//   meta   [C_out, C_in/32] 32-bit words, eight groups a word: group g's
//                           4-bit field at bits 4 (g % 8) of word g / 8 holds
//                           the first kept position (0..3) in its low two bits
//                           and the second in its high two.
// The input side is x_pi = P_B^T x: x_pi[bB + perm[b][i]] = x[bB + i], with
// perm the hardening's permutation (row i of block b goes to column perm[b][i]).
//
// Kernels:
//   pack24_kernel    A from W, perm and the mask bits -> values, meta (offline);
//   gather_kernel    x_pi for every token (the standalone permutation);
//   sp24_mm_kernel   Y = x_pi A^T for a tile of up to 16 tokens on the CUDA
//                    cores, the gather fused into the staging of the inputs:
//                    one warp per output row, 16-byte value loads, the inputs
//                    of the tile resident in shared memory.  Used for float32,
//                    for one token and for bf16 shapes the tensor-core variant
//                    (infer24_tc.cu: C_in a multiple of 256, at most 8192) does
//                    not take.

#include "lcp_internal.cuh"

namespace lcp {

__device__ int g_infer_error = 0;   // 301: group without exactly two kept; 302: perm entry out of range;
                                    // 303: perm not a permutation of its block

namespace {

__device__ __forceinline__ void infer_fail(int site) { atomicCAS(&g_infer_error, 0, site); }
inline int cdiv_int(int a, int b) { return (a + b - 1) / b; }
__device__ __forceinline__ int cdiv_dev(int a, int b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------- pack ---
// CTA (block column b, 64 rows): the inverse of block b's permutation in shared
// memory, then one thread per (row, mask word of the block): eight groups.
template <typename T>
__global__ void __launch_bounds__(256)
pack24_kernel(const T* __restrict__ W, const int32_t* __restrict__ perm, const uint32_t* __restrict__ mask,
              T* __restrict__ vals, uint32_t* __restrict__ meta, int cout, int cin, int B) {
  extern __shared__ int inv[];   // inv[j]: source channel (within the block) of slot j
  const int b = blockIdx.x, row0 = blockIdx.y * 64;
  for (int j = threadIdx.x; j < B; j += blockDim.x) inv[j] = perm ? -1 : j;
  __syncthreads();
  if (perm) {
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
      const int p = perm[(size_t)b * B + i];
      if (p < 0 || p >= B) infer_fail(302);
      else inv[p] = i;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < B; j += blockDim.x)
      if (inv[j] < 0) {
        infer_fail(303);
        inv[j] = j;
      }
    __syncthreads();
  }
  const int wpb = B / 32;                 // mask words per block row
  const int words = cin / 32;
  const int rows = min(64, cout - row0);
  for (int q = threadIdx.x; q < rows * wpb; q += blockDim.x) {
    const int o = row0 + q / wpb, w = q % wpb;
    const int gw = b * wpb + w;           // mask / meta word of the row
    const uint32_t mw = mask[(size_t)o * words + gw];
    const T* src = W + (size_t)o * cin + (size_t)b * B;
    T* dst = vals + (size_t)o * (cin / 2) + (size_t)gw * 16;
    uint32_t field = 0;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint32_t nib = (mw >> (4 * g)) & 0xFu;
      T v0 = from_f32<T>(0.f), v1 = from_f32<T>(0.f);
      uint32_t p0 = 0, p1 = 1;
      if (__popc(nib) == 2) {
        p0 = (uint32_t)(__ffs(nib) - 1);
        p1 = (uint32_t)(__ffs(nib & (nib - 1u)) - 1);
        v0 = src[inv[32 * w + 4 * g + (int)p0]];
        v1 = src[inv[32 * w + 4 * g + (int)p1]];
      } else {
        infer_fail(301);
      }
      dst[2 * g] = v0;
      dst[2 * g + 1] = v1;
      field |= (p0 | (p1 << 2)) << (4 * g);
    }
    meta[(size_t)o * words + gw] = field;
  }
}

// 16 bytes of elements, loaded and stored as one vector
template <typename T> struct __align__(16) Vec16 { T e[16 / sizeof(T)]; };

// ----------------------------------------------------------------- gather ---
// Items (token t, segment of `seg` channels = whole blocks): each thread loads
// 16-byte runs of source channels and their slots (every load of the item
// issued before any store), scatters them into shared memory at their slots,
// and after a barrier the segment leaves in coalesced 16-byte stores.
template <typename T>
__global__ void __launch_bounds__(256)
gather_kernel(const T* __restrict__ X, const int32_t* __restrict__ perm, T* __restrict__ Xp, int tokens,
              int cin, int bshift, int seg) {
  extern __shared__ __align__(16) uint8_t gsm[];
  T* buf = reinterpret_cast<T*>(gsm);
  constexpr int V = 16 / sizeof(T);
  constexpr int KC = 2;                 // 16-byte runs per thread in flight
  const int Bm = (1 << bshift) - 1;
  pdl_wait();
  pdl_trigger();
  const int nseg = cin / seg;
  const long long items = (long long)tokens * nseg;
  for (long long it = blockIdx.x; it < items; it += gridDim.x) {
    const int t = (int)(it / nseg), s0 = (int)(it % nseg) * seg;
    const Vec16<T>* src = reinterpret_cast<const Vec16<T>*>(X + (size_t)t * cin + s0);
    const int4* pv = reinterpret_cast<const int4*>(perm + s0);
    for (int base = threadIdx.x; base < seg / V; base += KC * blockDim.x) {
      Vec16<T> r[KC];
      int4 p[KC][V / 4];
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        const int q = base + k * (int)blockDim.x;
        if (q < seg / V) {
          r[k] = src[q];
#pragma unroll
          for (int h = 0; h < V / 4; ++h) p[k][h] = __ldg(pv + q * (V / 4) + h);
        }
      }
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        const int q = base + k * (int)blockDim.x;
        if (q >= seg / V) continue;
        const int* pk = reinterpret_cast<const int*>(&p[k][0]);
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const int i = q * V + v;
          if (pk[v] < 0 || pk[v] > Bm) infer_fail(302);
          else buf[(i & ~Bm) | pk[v]] = r[k].e[v];
        }
      }
    }
    __syncthreads();
    Vec16<T>* dst = reinterpret_cast<Vec16<T>*>(Xp + (size_t)t * cin + s0);
    for (int q = threadIdx.x; q < seg / V; q += blockDim.x) dst[q] = reinterpret_cast<const Vec16<T>*>(buf)[q];
    __syncthreads();
  }
}

// ------------------------------------------------------ sparse product ---
// Shared-memory image of the token tile: slot s of chunk c = s / 16 holds the TT
// inputs x_pi[t0 + t, s] (t < TT) contiguously, U = TT * sizeof(T) bytes; chunks
// are 16 U + PAD bytes apart, PAD making the chunk stride an odd number of the
// access width, so the 32 lanes (one chunk each) hit distinct banks.
//
// Persistent CTAs of 16 warps (8 for 16-token tiles); a warp takes rows o, o + WARPS G, ... and streams
// each row in batches of KP chunks (16 permuted columns, eight kept values)
// per lane, the next batch's loads issued before the current batch's
// arithmetic, so two batches per warp are in flight.
template <typename T, int TT> struct Sp24Cfg {
  static constexpr int U = TT * (int)sizeof(T);
  static constexpr int PAD = U < 4 ? 4 : (U > 16 ? 16 : U);
  static constexpr int CHUNK = 16 * U + PAD;
  static constexpr int WARPS = TT >= 16 ? 8 : 16;   // 16 tokens: registers for 255 a thread
  // chunks per lane per batch
  static constexpr int KP = 4;
  static constexpr int VU = (int)sizeof(T) / 2;    // 16-byte loads per chunk of values
};

// TT consecutive inputs of one slot from shared memory
template <typename T, int TT>
__device__ __forceinline__ void load_slot(const uint8_t* p, float (&x)[TT]) {
  constexpr int U = TT * (int)sizeof(T);
  if constexpr (U == 2) {
    x[0] = to_f32(*reinterpret_cast<const T*>(p));
  } else if constexpr (U == 4) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
    for (int t = 0; t < TT; ++t) x[t] = to_f32(e[t]);
  } else if constexpr (U == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
    for (int t = 0; t < TT; ++t) x[t] = to_f32(e[t]);
  } else {
#pragma unroll
    for (int h = 0; h < U / 16; ++h) {
      const uint4 w = reinterpret_cast<const uint4*>(p)[h];
      const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
      for (int t = 0; t < 16 / (int)sizeof(T); ++t) x[h * (16 / (int)sizeof(T)) + t] = to_f32(e[t]);
    }
  }
}

template <typename T, int TT> struct Batch {
  uint4 v[Sp24Cfg<T, TT>::KP][Sp24Cfg<T, TT>::VU];
  uint32_t m[Sp24Cfg<T, TT>::KP];
};

// loads of batch k of row o (chunks lane + 32 (KP k + j)); out-of-range chunks read nothing
template <typename T, int TT>
__device__ __forceinline__ void load_batch(Batch<T, TT>& b, const T* __restrict__ vals,
                                           const uint16_t* __restrict__ meta16, int o, int k, int nchunk,
                                           int lane) {
  using C = Sp24Cfg<T, TT>;
  const uint4* rv = reinterpret_cast<const uint4*>(vals + (size_t)o * (nchunk * 8));
  const uint16_t* rm = meta16 + (size_t)o * nchunk;
#pragma unroll
  for (int j = 0; j < C::KP; ++j) {
    const int c = lane + 32 * (C::KP * k + j);
    if (c < nchunk) {
#pragma unroll
      for (int h = 0; h < C::VU; ++h) b.v[j][h] = __ldg(rv + (size_t)c * C::VU + h);
      b.m[j] = __ldg(rm + c);
    } else {
#pragma unroll
      for (int h = 0; h < C::VU; ++h) b.v[j][h] = make_uint4(0u, 0u, 0u, 0u);
      b.m[j] = 0x4444u;   // positions (0, 1) of zero values
    }
  }
}

template <typename T, int TT>
__device__ __forceinline__ void mac_batch(const Batch<T, TT>& b, const uint8_t* xs, int k, int lane,
                                          int nchunk, float (&acc)[TT]) {
  using C = Sp24Cfg<T, TT>;
#pragma unroll
  for (int j = 0; j < C::KP; ++j) {
    const int c = lane + 32 * (C::KP * k + j);
    if (c >= nchunk) continue;
    const T* v8 = reinterpret_cast<const T*>(&b.v[j][0]);
    const uint8_t* base = xs + (size_t)c * C::CHUNK;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t f = (b.m[j] >> (4 * q)) & 0xFu;
      float x0[TT], x1[TT];
      load_slot<T, TT>(base + (4 * q + (int)(f & 3u)) * C::U, x0);
      load_slot<T, TT>(base + (4 * q + (int)(f >> 2)) * C::U, x1);
      const float a0 = to_f32(v8[2 * q]), a1 = to_f32(v8[2 * q + 1]);
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[t] = fmaf(a1, x1[t], fmaf(a0, x0[t], acc[t]));
    }
  }
}

template <typename T, int TT>
__global__ void __launch_bounds__(32 * Sp24Cfg<T, TT>::WARPS)
sp24_mm_kernel(const T* __restrict__ vals, const uint32_t* __restrict__ meta, const T* __restrict__ X,
               const int32_t* __restrict__ perm, float* __restrict__ Y, int cout, int cin, int tokens,
               int bshift) {
  using C = Sp24Cfg<T, TT>;
  extern __shared__ __align__(16) uint8_t xs[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nchunk = cin / 16;
  const int nbatch = cdiv_dev(nchunk, 32 * C::KP);
  const uint16_t* meta16 = reinterpret_cast<const uint16_t*>(meta);
  const int o0 = blockIdx.x * C::WARPS + warp, ostep = gridDim.x * C::WARPS;
  // the first batch of the warp's first row is in flight while the inputs are staged
  Batch<T, TT> cur;
  if (o0 < cout) load_batch<T, TT>(cur, vals, meta16, o0, 0, nchunk, lane);
  pdl_wait();
  pdl_trigger();
  // without a permutation every channel is its own slot: Bm spans the whole row
  const int Bm = perm ? (1 << bshift) - 1 : 0x7fffffff;
  for (int t0 = 0; t0 < tokens; t0 += TT) {
    // stage x_pi of tokens [t0, t0 + TT): source channels i = threadIdx.x + k
    // blockDim.x, KS of them (their slot and their TT inputs) loaded before any
    // is stored into the image at its slot
    constexpr int KS = TT >= 16 ? 2 : (TT >= 8 ? 4 : 8);
    for (int base = threadIdx.x; base < cin; base += KS * blockDim.x) {
      alignas(16) T e[KS][TT];
      int slot[KS];
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int i = base + k * (int)blockDim.x;
        slot[k] = i < cin ? (perm ? __ldg(perm + i) : (i & Bm)) : 0;
#pragma unroll
        for (int t = 0; t < TT; ++t)
          e[k][t] = (i < cin && t0 + t < tokens) ? __ldg(X + (size_t)(t0 + t) * cin + i) : from_f32<T>(0.f);
      }
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int i = base + k * (int)blockDim.x;
        if (i >= cin) continue;
        if (slot[k] < 0 || slot[k] > Bm) {
          infer_fail(302);
          continue;
        }
        const int s = (i & ~Bm) | slot[k];
        uint8_t* d = xs + (size_t)(s / 16) * C::CHUNK + (s % 16) * C::U;
        if constexpr (C::U % 16 == 0) {
#pragma unroll
          for (int h = 0; h < C::U / 16; ++h)
            reinterpret_cast<uint4*>(d)[h] = reinterpret_cast<const uint4*>(&e[k][0])[h];
        } else {
#pragma unroll
          for (int t = 0; t < TT; ++t) reinterpret_cast<T*>(d)[t] = e[k][t];
        }
      }
    }
    __syncthreads();
    for (int o = o0; o < cout; o += ostep) {
      float acc[TT];
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[t] = 0.f;
      for (int k = 0; k < nbatch; ++k) {
        // next batch: this row's, else the next row's first (this token tile),
        // else the first row's first batch of the next token tile
        Batch<T, TT> nxt;
        const bool more_row = k + 1 < nbatch;
        const int on = more_row ? o : o + ostep;
        if (more_row || on < cout) load_batch<T, TT>(nxt, vals, meta16, on, more_row ? k + 1 : 0, nchunk, lane);
        else if (t0 + TT < tokens && o0 < cout) load_batch<T, TT>(nxt, vals, meta16, o0, 0, nchunk, lane);
        mac_batch<T, TT>(cur, xs, k, lane, nchunk, acc);
        cur = nxt;
      }
#pragma unroll
      for (int t = 0; t < TT; ++t) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
      }
#pragma unroll
      for (int t = 0; t < TT; ++t)
        if (lane == t && t0 + t < tokens) Y[(size_t)(t0 + t) * cout + o] = acc[t];
    }
    __syncthreads();
  }
}

template <typename T, int TT>
lcp_status launch_sp24(const void* vals, const uint32_t* meta, const void* X, const int32_t* perm, float* Y,
                       int cout, int cin, int tokens, int bshift, cudaStream_t st) {
  using C = Sp24Cfg<T, TT>;
  const size_t smem = (size_t)(cin / 16) * C::CHUNK;
  auto k = sp24_mm_kernel<T, TT>;
  if (smem > 48 * 1024) {
    const lcp_status s = ensure_smem_limit(reinterpret_cast<const void*>(k), (int)smem, "sparse24_mm");
    if (s != LCP_OK) return s;
  }
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = (int)((227u * 1024u) / (smem + 1024));
  if (per_sm > 64 / C::WARPS) per_sm = 64 / C::WARPS;
  if (per_sm < 1) per_sm = 1;
  int grid = cdiv_int(cout, C::WARPS);
  if (grid > sms * per_sm) grid = sms * per_sm;
  return launch_kernel(k, dim3((unsigned)grid), dim3(32 * C::WARPS), smem, st, 1, true, "sparse24_mm",
                       static_cast<const T*>(vals), meta, static_cast<const T*>(X), perm, Y, cout, cin, tokens,
                       bshift);
}

template <typename T>
lcp_status sp24_dispatch(const void* vals, const uint32_t* meta, const void* X, const int32_t* perm, float* Y,
                         int cout, int cin, int tokens, int bshift, cudaStream_t st) {
  const int tt = sparse24_tile_tokens(cin, tokens, (int)sizeof(T));
  switch (tt) {
    case 16: return launch_sp24<T, 16>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
    case 8: return launch_sp24<T, 8>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
    case 4: return launch_sp24<T, 4>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
    case 2: return launch_sp24<T, 2>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
    case 1: return launch_sp24<T, 1>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
    default: return fail(LCP_ERR_SHAPE, "sparse24_mm: C_in = %d is too wide for the input tile", cin);
  }
}

int log2_block(int B) {
  int s = 0;
  while ((1 << s) < B) ++s;
  return s;
}

}  // namespace

// Tokens per tile: the power of two covering min(tokens, 16) whose input image
// fits in 200 KB of shared memory; 0 if not even one token fits.
int sparse24_tile_tokens(int cin, int tokens, int esize) {
  int tt = 1;
  while (tt < 16 && tt < tokens) tt *= 2;
  for (; tt >= 1; tt /= 2) {
    const int U = tt * esize, pad = U < 4 ? 4 : (U > 16 ? 16 : U);
    if ((long long)(cin / 16) * (16 * U + pad) <= 200 * 1024) return tt;
  }
  return 0;
}

lcp_status launch_pack24(const void* W, const int32_t* perm, const uint32_t* mask, void* vals, uint32_t* meta,
                         int cout, int cin, int B, lcp_dtype dt, cudaStream_t st) {
  const dim3 grid((unsigned)(cin / B), (unsigned)cdiv_int(cout, 64));
  const size_t smem = (size_t)B * sizeof(int);
  if (dt == LCP_F32)
    return launch_kernel(pack24_kernel<float>, grid, dim3(256), (int)smem, st, 1, false, "pack24",
                         static_cast<const float*>(W), perm, mask, static_cast<float*>(vals), meta, cout, cin, B);
  return launch_kernel(pack24_kernel<__nv_bfloat16>, grid, dim3(256), (int)smem, st, 1, false, "pack24",
                       static_cast<const __nv_bfloat16*>(W), perm, mask, static_cast<__nv_bfloat16*>(vals), meta,
                       cout, cin, B);
}

lcp_status launch_gather(const void* X, const int32_t* perm, void* Xp, int tokens, int cin, int B, lcp_dtype dt,
                         cudaStream_t st) {
  // segments of whole blocks, at most 4096 channels
  int seg = cin;
  while (seg > 4096 && seg % 2 == 0 && (seg / 2) % B == 0) seg /= 2;
  const int esize = dt == LCP_F32 ? 4 : 2;
  const size_t smem = (size_t)seg * esize;
  if (smem > 200 * 1024) return fail(LCP_ERR_SHAPE, "gather: C_in = %d does not split into segments of whole blocks", cin);
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = (long long)tokens * (cin / seg);
  long long grid = items < 8LL * sms ? items : 8LL * sms;
  const int bshift = log2_block(B);
  if (dt == LCP_F32) {
    auto k = gather_kernel<float>;
    if (smem > 48 * 1024) {
      const lcp_status s = ensure_smem_limit(reinterpret_cast<const void*>(k), (int)smem, "gather");
      if (s != LCP_OK) return s;
    }
    return launch_kernel(k, dim3((unsigned)grid), dim3(256), smem, st, 1, true, "gather",
                         static_cast<const float*>(X), perm, static_cast<float*>(Xp), tokens, cin, bshift, seg);
  }
  auto k = gather_kernel<__nv_bfloat16>;
  if (smem > 48 * 1024) {
    const lcp_status s = ensure_smem_limit(reinterpret_cast<const void*>(k), (int)smem, "gather");
    if (s != LCP_OK) return s;
  }
  return launch_kernel(k, dim3((unsigned)grid), dim3(256), smem, st, 1, true, "gather",
                       static_cast<const __nv_bfloat16*>(X), perm, static_cast<__nv_bfloat16*>(Xp), tokens, cin,
                       bshift, seg);
}

lcp_status launch_sparse24_mm(const void* vals, const uint32_t* meta, const void* X, const int32_t* perm, float* Y,
                              int cout, int cin, int tokens, int B, lcp_dtype dt, cudaStream_t st) {
  const int bshift = perm ? log2_block(B) : 0;
  // one token: the CUDA-core kernel (its per-row stream has the shorter dependency
  // chain); from 2 tokens on the sparse tensor-core kernel (its time hardly depends on
  // the token count up to 16)
  if (dt == LCP_BF16 && tokens >= 2 && sparse24_tc_splits(cout, cin) > 0)
    return launch_sparse24_tc(static_cast<const __nv_bfloat16*>(vals), meta, static_cast<const __nv_bfloat16*>(X),
                              perm, Y, cout, cin, tokens, bshift, st);
  if (dt == LCP_F32) return sp24_dispatch<float>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
  return sp24_dispatch<__nv_bfloat16>(vals, meta, X, perm, Y, cout, cin, tokens, bshift, st);
}

lcp_status infer_error(int* site, int reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_infer_error, sizeof(int));
  if (e == cudaSuccess && reset) {
    const int z = 0;
    e = cudaMemcpyToSymbol(g_infer_error, &z, sizeof(int));
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "reading the inference error word: %s", cudaGetErrorString(e));
  }
  *site = v;
  return LCP_OK;
}

}  // namespace lcp
