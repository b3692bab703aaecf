// Deployed 2:4 product on the tensor cores (PermLLM summary, "Effect on
// inference acceleration"): Y = x_pi A^T for up to 16 tokens, A kept in the
// compressed form of infer24.cu (values [C_out, C_in/2], 4-bit position fields
// [C_out, C_in/32]).
//
// The weight stays compressed in HBM (0.5625 of the dense bytes) and goes to
// the tensor cores compressed: tcgen05.mma.sp (kind::f16, M = 128, N = 16, 32
// channels a product) takes the two kept values of every group of four as its
// A operand and their positions as metadata in tensor memory.
//   - the CTA owns 128 output rows and a K range of C_in / S channels; the S
//     CTAs of a row tile form a cluster (S <= 4 with 16 staging warps, S <= 8
//     with 8 and two CTAs an SM);
//   - TMA brings the compressed values (128 rows x 64 values, 128-byte
//     swizzle: the A operand of four products as it lands) and the position
//     words (128 rows x 4 words) of each 128-channel stage into a 4-stage ring;
//   - four metadata warps (one per TMEM lane quadrant) write each stage's
//     position words into four TMEM columns (eight-column aligned) in the
//     layout the sparse product reads: per 16-row group b and j < 8, lane 16 b + j holds the 16-bit
//     position fields of channels 0-15 of rows 16 b + j (low half) and
//     16 b + 8 + j (high half), lane 16 b + 8 + j those of channels 16-31
//     (found with a probe on a B200: one sparse product on known inputs);
//   - an MMA warp issues the four products of a stage against the inputs
//     x_pi (the tokens zero-padded to 16), staged once per launch as K-major
//     tiles with the gather applied;
//   - the S partial accumulators are summed in rank order through distributed
//     shared memory, each rank writing 1/S of Y (deterministic, no workspace).

#include "tc_common.cuh"

namespace lcp {
namespace {

// Two configurations: 16 staging warps (one CTA an SM, up to 2048 channels and 4 splits), and 8
// (two CTAs an SM, up to 1024 channels and 8 splits: twice the weight streams in flight and half
// the staging a CTA, measured faster at 4 and 8 tokens on the 4096^2 layer), used whenever it
// takes the shape.
template <int EW> struct StCfgT {
  static constexpr int EXP_WARPS = EW;              // stage the inputs; warps 0-3 then write the metadata
  static constexpr int CTAS_PER_SM = EW <= 8 ? 2 : 1;
  static constexpr int MAX_SPLITS = EW <= 8 ? 8 : 4;
  static constexpr int PROD_WARP = EXP_WARPS, MMA_WARP = EXP_WARPS + 1;
  static constexpr int THREADS = 32 * (EXP_WARPS + 2);
  static constexpr int EXP_THREADS = 32 * EXP_WARPS;
  static constexpr int STG = 4;                     // ring stages of 128 channels
  static constexpr int NM = 2;                      // metadata buffers in TMEM (4 columns each)
  static constexpr int V_BYTES = 128 * 128;         // 128 rows x 64 bf16 values
  static constexpr int M_BYTES = 128 * 16;          // 128 rows x 4 position words
  static constexpr int RED_BYTES = 16 * 128 * 4;    // 16 tokens x 128 rows float32
  static constexpr int MAX_KR = 128 * EXP_WARPS;   // channels per CTA (input image up to 64 KB)
  // metadata of product k of buffer m at column TMEM_META + 8 (4 m + k): eight-column
  // aligned, the placement the probe used (the accumulator: columns 0-15)
  static constexpr int TMEM_META = 64, TMEM_COLS = 128;
  static constexpr int NBAR = 2 * STG + 2 * NM + 1;
  static int smem(int kr) { return STG * V_BYTES + (kr / 64) * 2048 + STG * M_BYTES + RED_BYTES + 256 + 1024; }
};

// tcgen05.mma.sp, kind::f16: D (+)= A B^T with A the 2:4-compressed M x 16 stored values of
// 32 channels and their positions at TMEM address `meta`
__device__ __forceinline__ void mma_bf16_sp(uint32_t d, uint64_t a, uint64_t b, uint32_t meta, uint32_t idesc,
                                            bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(meta), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Roles (EW + 2 warps): warp EW loads the ring (TMA), warp EW + 1 issues the products,
// warps 0 .. EW - 1 stage the inputs, then warps 0-3 write each stage's metadata into
// TMEM; they meet only through mbarriers:
//   full[q]   (TMA bytes)          ring slot q holds stage j        -> metadata warps, MMA warp
//   empty[q]  (MMA commit)         the products reading slot q done -> producer
//   mready[m] (4 warp arrivals)    TMEM metadata buffer m holds j   -> MMA warp
//   mfree[m]  (MMA commit)         the products reading m are done  -> metadata warps
//   fin       (MMA commit)         every product has landed         -> epilogue
template <int EW>
__global__ void __launch_bounds__(StCfgT<EW>::THREADS, StCfgT<EW>::CTAS_PER_SM)
sp24_tc_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
               const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm, float* __restrict__ Y,
               int cout, int cin, int tokens, int bshift, int kr) {
  using C = StCfgT<EW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sV = smem;                                   // STG x 16 KB
  uint8_t* sX = sV + C::STG * C::V_BYTES;               // kr / 64 blocks x 2 KB
  uint8_t* sM = sX + (kr / 64) * 2048;                  // STG x 2 KB
  float* sRed = reinterpret_cast<float*>(sM + C::STG * C::M_BYTES);   // [16][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRed + 16 * 128);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto full = [&](int q) { return smem_u32(bars + q); };
  auto empty = [&](int q) { return smem_u32(bars + C::STG + q); };
  auto mready = [&](int m) { return smem_u32(bars + 2 * C::STG + m); };
  auto mfree = [&](int m) { return smem_u32(bars + 2 * C::STG + C::NM + m); };
  const uint32_t fin = smem_u32(bars + 2 * C::STG + 2 * C::NM);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int S = (int)gridDim.x;                         // cluster = the S splits of a row tile
  const uint32_t rank = S > 1 ? cluster_rank() : 0u;
  const int row0 = blockIdx.y * 128, k0 = (int)rank * kr;
  const int nst = kr / 128;
  if (tid == 0) {
    for (int q = 0; q < C::STG; ++q) {
      mbar_init(full(q), 1);
      mbar_init(empty(q), 1);
    }
    for (int m = 0; m < C::NM; ++m) {
      mbar_init(mready(m), 4);
      mbar_init(mfree(m), 1);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) tmem_alloc(smem_u32(holder), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  bool ok = true;

  if (warp == C::PROD_WARP) {
    // the weight does not come from the previous kernel: the ring fills at once
    if (lane == 0) {
      int last_issued[C::STG];
#pragma unroll
      for (int q = 0; q < C::STG; ++q) last_issued[q] = -1;
      for (int j = 0; j < nst; ++j) {
        const int q = j % C::STG;
        if (j >= C::STG && !mbar_wait(empty(q), (uint32_t)((j - C::STG) / C::STG) & 1u, abort_flag, 311)) break;
        mbar_expect_tx(full(q), C::V_BYTES + C::M_BYTES);
        tma_load_2d(smem_u32(sV + q * C::V_BYTES), &tmV, full(q), (k0 + 128 * j) / 2, row0);
        tma_load_2d(smem_u32(sM + q * C::M_BYTES), &tmM, full(q), (k0 + 128 * j) / 32, row0);
        last_issued[q] = j;
      }
      // every copy started here lands before the CTA moves on
      for (int q = 0; q < C::STG; ++q)
        if (last_issued[q] >= 0) mbar_wait_drain(full(q), (uint32_t)(last_issued[q] / C::STG) & 1u, 314);
    }
    __syncwarp();
    pdl_wait();
    pdl_trigger();
  } else if (warp == C::MMA_WARP) {
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 16, false, false) | (1u << 2);   // sparse A
      int j = 0;
      for (; j < nst; ++j) {
        const int q = j % C::STG, m = j % C::NM;
        if (!mbar_wait(full(q), (uint32_t)(j / C::STG) & 1u, abort_flag, 312)) break;
        if (!mbar_wait(mready(m), (uint32_t)(j / C::NM) & 1u, abort_flag, 317)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sV + q * C::V_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // 32 channels: stored values k * 16 .. + 15 of the 64 a row; inputs of block
          // (128 j + 32 k) / 64, half k % 2 of its 128-byte rows
          const uint32_t b0 = smem_u32(sX + (2 * j + k / 2) * 2048) + (k & 1) * 64;
          mma_bf16_sp(tmem, sdesc(a0 + k * 32, 16, 1024), sdesc(b0, 16, 1024),
                      tmem + C::TMEM_META + 8 * (m * 4 + k), idesc, (j | k) != 0);
        }
        mma_commit(empty(q));
        mma_commit(mfree(m));
      }
      mma_commit(fin);                                  // arrives once every issued product is done
    }
    __syncwarp();
  } else {
    // inputs x_pi of this K range, tokens zero-padded to 16: source channel i goes
    // to slot s = (i & ~(B-1)) | perm[i]; element (t, s) of block (s - k0) / 64 at
    // row t, 16-byte chunk ((s - k0) % 64) / 8 (swizzled), position (s - k0) % 8.
    // Thread = (run c of 8 source channels, token group): the run's slots (two
    // 16-byte loads) and x of tokens g, g + G, ... (one 16-byte load each), every
    // load issued before the stores.
    {
      const int Bm = perm ? (1 << bshift) - 1 : 0x7fffffff;
      const int runs = kr / 8;                          // 32 .. 256
      const int G = C::EXP_THREADS / runs;              // token groups
      constexpr int TPT = 16 * C::MAX_KR / 8 / C::EXP_THREADS;   // tokens per thread at most (8)
      const int c = tid % runs, g = tid / runs;
      const int i0 = k0 + c * 8;
      int4 pv[2] = {make_int4(0, 0, 0, 0), make_int4(0, 0, 0, 0)};
      if (perm) {                                       // the permutation is no kernel's output
        pv[0] = __ldg(reinterpret_cast<const int4*>(perm + i0));
        pv[1] = __ldg(reinterpret_cast<const int4*>(perm + i0) + 1);
      }
      pdl_wait();
      pdl_trigger();
      uint4 xv[TPT];
#pragma unroll
      for (int m = 0; m < TPT; ++m) {
        const int t = g + m * G;
        xv[m] = make_uint4(0u, 0u, 0u, 0u);
        if (t < 16 && t < tokens) xv[m] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)t * cin + i0));
      }
      const int* pk = reinterpret_cast<const int*>(&pv[0]);
      int loc[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int i = i0 + v;
        const int p = perm ? pk[v] : (i & Bm);
        if (p < 0 || p > Bm) {
          atomicCAS(&g_tc_error, 0, 302);   // out-of-range permutation entry: skipped
          loc[v] = -1;
        } else {
          loc[v] = ((i & ~Bm) | p) - k0;
        }
      }
#pragma unroll
      for (int m = 0; m < TPT; ++m) {
        const int t = g + m * G;
        if (t >= 16) continue;
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&xv[m]);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          if (loc[v] < 0) continue;
          const int ch = (loc[v] & 63) >> 3, pos = loc[v] & 7;
          *reinterpret_cast<__nv_bfloat16*>(sX + (loc[v] >> 6) * 2048 + t * 128 + ((ch ^ (t & 7)) << 4) + pos * 2) =
              e[v];
        }
      }
    }
    fence_async_smem();
    // the inputs are in shared memory before the first product reads them: every
    // metadata warp arrives on mready only after this point, and the staging warps
    // 4-15 join the metadata warps at a named barrier
    asm volatile("bar.sync 1, %0;" ::"r"(C::EXP_THREADS) : "memory");

    if (warp < 4) {
      // metadata of stage j -> TMEM columns TMEM_META + 8 (4 (j % NM) + k), lanes of this
      // warp's quadrant: lane L = 32 warp + lane, rows r0 = 16 (L / 16) + L % 8 and r0 + 8
      const int L = warp * 32 + lane;
      const int r0 = (L & ~15) + (L & 7), r1 = r0 + 8;
      const bool hi = (L & 8) != 0;                     // channels 16-31 of each 32
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + C::TMEM_META;
      for (int j = 0; j < nst; ++j) {
        const int q = j % C::STG, m = j % C::NM;
        ok = ok && warp_all(mbar_wait(full(q), (uint32_t)(j / C::STG) & 1u, abort_flag, 315));
        if (j >= C::NM)
          ok = ok && warp_all(mbar_wait(mfree(m), (uint32_t)((j - C::NM) / C::NM) & 1u, abort_flag, 316));
        if (!ok) break;
        tc_fence_after();
        const uint4 w0 = *reinterpret_cast<const uint4*>(sM + q * C::M_BYTES + r0 * 16);
        const uint4 w1 = *reinterpret_cast<const uint4*>(sM + q * C::M_BYTES + r1 * 16);
        auto pick = [&](uint32_t a, uint32_t b) {
          return hi ? ((a >> 16) | (b & 0xFFFF0000u)) : ((a & 0xFFFFu) | (b << 16));
        };
        tmem_st1(taddr + 8 * (m * 4 + 0), pick(w0.x, w1.x));
        tmem_st1(taddr + 8 * (m * 4 + 1), pick(w0.y, w1.y));
        tmem_st1(taddr + 8 * (m * 4 + 2), pick(w0.z, w1.z));
        tmem_st1(taddr + 8 * (m * 4 + 3), pick(w0.w, w1.w));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(mready(m));
      }
      // epilogue: one warp per TMEM lane quadrant (warp w reads lanes 32 w ..)
      const bool got = ok && nst > 0 && warp_all(mbar_wait(fin, 0, abort_flag, 313));
      tc_fence_after();
      uint32_t acc[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), acc);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < 16; ++t) sRed[t * 128 + warp * 32 + lane] = got ? __uint_as_float(acc[t]) : 0.f;
    }
  }
  tc_fence_before();
  // the S partials are summed in rank order; rank q writes the outputs [q, q + 1) * 2048 / S
  if (S == 1) {
    __syncthreads();
    for (int idx = tid; idx < 16 * 128; idx += C::THREADS) {
      const int t = idx >> 7, rr = idx & 127;
      if (t < tokens && row0 + rr < cout) Y[(size_t)t * cout + row0 + rr] = sRed[idx];
    }
  } else {
    cluster_sync_all();                                 // partials visible cluster-wide
    const uint32_t red = smem_u32(sRed);
    const int per = 16 * 128 / S, base = (int)rank * per;
    for (int idx = base + tid; idx < base + per; idx += C::THREADS) {
      const int t = idx >> 7, rr = idx & 127;
      if (t >= tokens || row0 + rr >= cout) continue;
      float v = 0.f;
      for (int q = 0; q < S; ++q) v += ld_cluster_f32(mapa(red + idx * 4, (uint32_t)q));
      Y[(size_t)t * cout + row0 + rr] = v;
    }
    cluster_sync_all();                                 // peers keep their partials until read
  }
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// 2-D uint32 tensor map, no swizzle
lcp_status make_map_u32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t bx, uint32_t by,
                        const char* what) {
  EncodeFn fn = encode_fn();
  if (!fn) return fail(LCP_ERR_CUDA, "%s: cuTensorMapEncodeTiled is unavailable from the driver", what);
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 4};
  const cuuint32_t box[2] = {bx, by};
  const cuuint32_t es[2] = {1, 1};
  const CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (res != CUDA_SUCCESS) return fail(LCP_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)res);
  return LCP_OK;
}

}  // namespace

lcp_status tc_error_infer(int* site, int reset) { return read_tc_error(site, reset); }

// Splits of C_in for the tensor-core product (0: the shape is not supported):
// S in {1, 2, 4} with C_in / S a multiple of 256 and at most 2048, as many as
// keep the grid (S x row tiles) within one wave of the SMs.
// most C_in splits of a row tile (tuning: 1, 2 or 4)
// C_in splits S of a row tile for configuration EW: C_in / S a multiple of 256 and at most
// MAX_KR; the fewest that fit, then more while one wave of the SMs holds the grid.
template <int EW> int tc_splits(int cout, int cin) {
  using C = StCfgT<EW>;
  if (cin % 256) return 0;
  const int tiles = cdiv(cout, 128);
  int best = 0;
  for (int s = 1; s <= C::MAX_SPLITS; s *= 2) {
    if (cin % (256 * s) || cin / s > C::MAX_KR) continue;
    if (best == 0) best = s;
    else if (tiles * s <= num_sms() * C::CTAS_PER_SM) best = s;
  }
  return best;
}

template <int EW>
lcp_status launch_sp24(const CUtensorMap& mV, const CUtensorMap& mM, const __nv_bfloat16* X, const int32_t* perm,
                       float* Y, int cout, int cin, int tokens, int bshift, int S, cudaStream_t st) {
  using C = StCfgT<EW>;
  const int kr = cin / S;
  const int smem = C::smem(kr);
  TC_TRY(set_smem(sp24_tc_kernel<EW>, smem, "sparse24_tc"));
  const dim3 grid((unsigned)S, (unsigned)cdiv(cout, 128));
  for (int t0 = 0; t0 < tokens; t0 += 16) {
    const int tt = tokens - t0 < 16 ? tokens - t0 : 16;
    TC_TRY(launch_kernel(sp24_tc_kernel<EW>, grid, dim3(C::THREADS), smem, st, S, true, "sparse24_tc", mV, mM,
                         X + (size_t)t0 * cin, perm, Y + (size_t)t0 * cout, cout, cin, tt, bshift, kr));
  }
  return LCP_OK;
}

int sparse24_tc_splits(int cout, int cin) {
  const int s8 = tc_splits<8>(cout, cin);
  return s8 > 0 ? s8 : tc_splits<16>(cout, cin);
}

lcp_status launch_sparse24_tc(const __nv_bfloat16* vals, const uint32_t* meta, const __nv_bfloat16* X,
                              const int32_t* perm, float* Y, int cout, int cin, int tokens, int bshift,
                              cudaStream_t st) {
  const int s8 = tc_splits<8>(cout, cin), s16 = s8 > 0 ? 0 : tc_splits<16>(cout, cin);
  if (s8 == 0 && s16 == 0) return fail(LCP_ERR_SHAPE, "sparse24 tensor-core path: C_in = %d is not supported", cin);
  CUtensorMap mV, mM;
  TC_TRY(make_map(&mV, vals, (uint64_t)cin / 2, (uint64_t)cout, 64, 128, "sparse24 values"));
  TC_TRY(make_map_u32(&mM, meta, (uint64_t)cin / 32, (uint64_t)cout, 4, 128, "sparse24 positions"));
  if (s8 > 0) return launch_sp24<8>(mV, mM, X, perm, Y, cout, cin, tokens, bshift, s8, st);
  return launch_sp24<16>(mV, mM, X, perm, Y, cout, cin, tokens, bshift, s16, st);
}

}  // namespace lcp
