// Block backward on the tensor cores: dA = dAt P_B, dW' = M.dA and the
// gradient of every diagonal block, dP_b = dAt_b^T A_b + W_b^T dW'_b
// (reverse of PermLLM's Method 3 product and mask).

#include "tc_common.cuh"

namespace lcp {
namespace {

// ---------------------------------------- block backward, warp-specialised ---
// BC = 64 (B = 32 or 64).  One CTA per (channel tile, row segment).  Warp 0
// streams the (dAt, W) tiles of each 128-row chunk into a 4-stage ring; warp 1
// issues [W P_hi | W P_lo] (one N = 128 product: the two P images are adjacent
// in shared memory) and dA = dAt P_hi into one of two TMEM buffers; warp 2,
// once the epilogue has written A = M.W' and dW' = M.dA, issues the stacked dP
// product; warps 3-10 (two per TMEM lane quadrant, 32 columns each) form
// W' = W P_hi + W P_lo and turn W', dA and the mask into the bf16 operands.
// The two issuers sit on different SM sub-partitions: issuing a tcgen05.mma
// costs one thread about 60 cycles on an idle SM and more next to busy
// epilogue warps, and these products (16 a chunk) take about 70 cycles each
// on the tensor core, so one issuer would set the pace.  The dP accumulator
// stays in TMEM for the whole segment and is written once at the end.  TMEM
// columns: buffer a at 192 a (W P_hi, W P_lo, dA: 64 each), dP at 384.
template <int NSL> struct BwCfg {
  static constexpr int STAGES = 4;
  static constexpr int T_BYTES = 16384;                  // 128 rows x 64 bf16
  static constexpr int STAGE = 2 * T_BYTES;              // dAt | W (adjacent: stacked A operand)
  static constexpr int IMG_BYTES = 8192;
  static constexpr int SMEM = STAGES * STAGE + 2 * IMG_BYTES + 2 * (2 * T_BYTES) + 1024 + 256;
  static constexpr int EPI_WARPS = 4 * NSL;              // NSL column slices per TMEM lane quadrant
  static constexpr int COLS = 64 / NSL;
  static constexpr int CTRL_WARPS = 3;                   // producer, two MMA issuers
  static constexpr int THREADS = 32 * (CTRL_WARPS + EPI_WARPS);
  static constexpr int EPI = 32 * EPI_WARPS;
};

template <int B, int NSL>
__global__ void __launch_bounds__(BwCfg<NSL>::THREADS, 1)
block_bwd_ws_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmDAt,
                    const __grid_constant__ CUtensorMap tmPth, const __grid_constant__ CUtensorMap tmPtl,
                    const uint32_t* __restrict__ mask, float* __restrict__ dP, int cout, int cin,
                    int rows_per_split) {
  using C = BwCfg<NSL>;
  constexpr int NV = C::COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sStage = smem;
  uint8_t* sPth = smem + C::STAGES * C::STAGE;
  uint8_t* sPtl = sPth + C::IMG_BYTES;
  uint8_t* sAB = sPtl + C::IMG_BYTES;      // buffer a at + a * 2 * T_BYTES: A | dW' (adjacent)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sAB + 2 * 2 * C::T_BYTES);
  // bars: full[S] empty[S] wd[2] abf[2] abe[2] dpf drain img drain2
  constexpr int S = C::STAGES;
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 2 * S + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = S, WD = 2 * S, ABF = 2 * S + 2, ABE = 2 * S + 4, DPF = 2 * S + 6, DRAIN = 2 * S + 7,
            IMG = 2 * S + 8, DRAIN2 = 2 * S + 9;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x, sidx = blockIdx.y, col0 = t * 64;
  const int rbeg = sidx * rows_per_split;
  const int rend = min(cout, rbeg + rows_per_split);
  const int nchunk = cdiv(rend - rbeg, 128);
  const int words = cin / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(bar(FULL + i), 1); mbar_init(bar(EMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(WD + i), 1);
      mbar_init(bar(ABF + i), C::EPI_WARPS);
      mbar_init(bar(ABE + i), 1);
    }
    mbar_init(bar(DPF), 1);
    mbar_init(bar(DRAIN), 1);
    mbar_init(bar(DRAIN2), 1);
    mbar_init(bar(IMG), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  pdl_wait();
  pdl_trigger();
  const uint32_t tDP = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      bool img_ok = true;
      if (nchunk > 0) {
        mbar_expect_tx(bar(IMG), 2 * C::IMG_BYTES);
        tma_load_2d(smem_u32(sPth), &tmPth, bar(IMG), 0, col0);
        tma_load_2d(smem_u32(sPtl), &tmPtl, bar(IMG), 0, col0);
      }
      uint32_t issued = 0, par = 0;
      for (int c = 0; c < nchunk; ++c) {
        const int st = c % C::STAGES;
        const uint32_t use = (uint32_t)(c / C::STAGES) & 1u;
        if (!mbar_wait(bar(EMPTY + st), use ^ 1u, abort_flag, 71)) break;
        uint8_t* sg = sStage + st * C::STAGE;
        const int r0 = rbeg + c * 128;
        mbar_expect_tx(bar(FULL + st), C::STAGE);
        tma_load_2d(smem_u32(sg), &tmDAt, bar(FULL + st), col0, r0);
        tma_load_2d(smem_u32(sg + C::T_BYTES), &tmW, bar(FULL + st), col0, r0);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (use << st);
      }
      for (int st = 0; st < C::STAGES; ++st)
        if (issued & (1u << st)) mbar_wait_drain(bar(FULL + st), (par >> st) & 1u, 72);
      if (nchunk > 0) img_ok = mbar_wait_drain(bar(IMG), 0, 73);
      (void)img_ok;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_n = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_w = idesc_bf16(128, 128, false, false);
      bool ok = nchunk == 0 || mbar_wait(bar(IMG), 0, abort_flag, 74);
      // [W P_hi | W P_lo] and dA = dAt P_hi of chunk c into TMEM buffer c & 1
      auto mma1 = [&](int c) -> bool {
        const int st = c % C::STAGES, a = c & 1;
        const uint32_t use = (uint32_t)(c / C::STAGES) & 1u, ua = (uint32_t)(c >> 1) & 1u;
        if (!mbar_wait(bar(FULL + st), use, abort_flag, 75)) return false;
        // the epilogue has read buffer a of chunk c - 2 (it arrives on ABF after its loads)
        if (c >= 2 && !mbar_wait(bar(ABF + a), ua ^ 1u, abort_flag, 76)) return false;
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
        const uint32_t tW = tmem + a * 192, tDA = tmem + a * 192 + 128;
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint64_t pdesc = sdesc(smem_u32(sPth) + k16 * 32, 16, 1024);   // rows 64..127: P_lo image
          mma_bf16(tW, sdesc(sg + C::T_BYTES + k16 * 32, 16, 1024), pdesc, idesc_w, k16 != 0);
          mma_bf16(tDA, sdesc(sg + k16 * 32, 16, 1024), pdesc, idesc_n, k16 != 0);
        }
        mma_commit(bar(WD + a));
        return true;
      };
      for (int c = 0; c < nchunk && ok; ++c) ok = mma1(c);
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0, 78);
    }
    __syncwarp();
  } else if (warp == 2) {
    // dP issuer: the stage of chunk c (dAt | W) and buffer a (A | dW') once the epilogue has
    // written the latter; its completion also frees the stage (the W' / dA products of the
    // chunk completed before the epilogue could start)
    if (lane == 0) {
      constexpr uint32_t idesc_dp = idesc_bf16(128, 128, true, true);
      for (int c = 0; c < nchunk; ++c) {
        const int st = c % C::STAGES, a = c & 1;
        const uint32_t use = (uint32_t)(c / C::STAGES) & 1u, ua = (uint32_t)(c >> 1) & 1u;
        if (!mbar_wait(bar(FULL + st), use, abort_flag, 82)) break;
        if (!mbar_wait(bar(ABF + a), ua, abort_flag, 77)) break;
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
        const uint32_t sab = smem_u32(sAB + a * 2 * C::T_BYTES);
        // stacked: A operand [dAt | W] (M = 128), B operand [A | dW'] (N = 128), LBO = 16 KB
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_bf16(tDP, sdesc(sg + k16 * 2048, 16384, 1024), sdesc(sab + k16 * 2048, 16384, 1024), idesc_dp,
                   (c | k16) != 0);
        mma_commit(bar(ABE + a));
        mma_commit(bar(EMPTY + st));
      }
      mma_commit(bar(DPF));
      mma_commit(bar(DRAIN2));
      mbar_wait_drain(bar(DRAIN2), 0, 83);
    }
    __syncwarp();
  } else {
    const int e = warp - C::CTRL_WARPS, q = warp & 3, h = e >> 2;   // h: column slice of NV columns
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    bool ok = true;
    // mask bits of this thread's NV columns, one chunk ahead of the chunk being processed
    auto mask_bits = [&](int c) -> uint32_t {
      const int grow = rbeg + c * 128 + row;
      if (c >= nchunk || grow >= rend) return 0u;
      const uint32_t w = __ldg(mask + (size_t)grow * words + col0 / 32 + (h * NV) / 32);
      return NV == 32 ? w : (w >> ((h * NV) % 32)) & ((1u << NV) - 1u);
    };
    uint32_t next_bits = mask_bits(0);
    for (int c = 0; c < nchunk; ++c) {
      const int a = c & 1;
      const uint32_t ua = (uint32_t)(c >> 1) & 1u;
      const uint32_t bits = next_bits;
      next_bits = mask_bits(c + 1);
      ok = named_and(1, C::EPI, mbar_wait(bar(WD + a), ua, abort_flag, 79));
      if (!ok) break;
      tc_fence_after();
      uint32_t wv[NV], wl[NV], dv[NV];
      tmem_ld_cols<NV>(tmem + lane_off + a * 192 + h * NV, wv);
      tmem_ld_cols<NV>(tmem + lane_off + a * 192 + 64 + h * NV, wl);
      tmem_ld_cols<NV>(tmem + lane_off + a * 192 + 128 + h * NV, dv);
      tmem_ld_wait();
      // buffer a was last read by the dP product of chunk c - 2
      ok = named_and(1, C::EPI, c < 2 || mbar_wait(bar(ABE + a), ua ^ 1u, abort_flag, 80));
      if (!ok) break;
      uint8_t* rA = sAB + a * 2 * C::T_BYTES;
      uint8_t* rD = rA + C::T_BYTES;
#pragma unroll
      for (int c8 = 0; c8 < NV / 8; ++c8) {
        float fa[8], fd[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const bool keep = (bits >> (8 * c8 + x)) & 1u;
          fa[x] = keep ? __uint_as_float(wv[8 * c8 + x]) + __uint_as_float(wl[8 * c8 + x]) : 0.f;
          fd[x] = keep ? __uint_as_float(dv[8 * c8 + x]) : 0.f;
        }
        const int chunk = h * (NV / 8) + c8;
        st_sw128(rA, row, chunk, make_uint4(pack_bf16x2(fa[0], fa[1]), pack_bf16x2(fa[2], fa[3]),
                                            pack_bf16x2(fa[4], fa[5]), pack_bf16x2(fa[6], fa[7])));
        st_sw128(rD, row, chunk, make_uint4(pack_bf16x2(fd[0], fd[1]), pack_bf16x2(fd[2], fd[3]),
                                            pack_bf16x2(fd[4], fd[5]), pack_bf16x2(fd[6], fd[7])));
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ABF + a));
    }
    if (ok) ok = named_and(1, C::EPI, mbar_wait(bar(DPF), 0, abort_flag, 81));
    if (ok) {
      tc_fence_after();
      // rows 0..63 hold dAt^T A (columns 0..63), rows 64..127 W^T dW' (columns 64..127)
      uint32_t v[NV];
      const uint32_t cbase = (row < 64 ? 0u : 64u) + h * NV;
      tmem_ld_cols<NV>(tDP + lane_off + cbase, v);
      tmem_ld_wait();
      // 64 x 64 floats, row pitch 65 (a warp's 32 rows fall in distinct banks); every MMA is done
      float* scratch = reinterpret_cast<float*>(sAB);
      if (row >= 64) {
#pragma unroll
        for (int x = 0; x < NV; ++x) scratch[(row - 64) * 65 + h * NV + x] = __uint_as_float(v[x]);
      }
      named_sync(1, C::EPI);
      if (row < 64) {
        const int nb = cin / B;
        float* dPs = dP + (size_t)sidx * nb * B * B;
        const float* add = scratch + row * 65 + h * NV;
        if constexpr (B == 64) {
          float4* o = reinterpret_cast<float4*>(dPs + ((size_t)t * 64 + row) * 64 + h * NV);
#pragma unroll
          for (int qq = 0; qq < NV / 4; ++qq)
            o[qq] = make_float4(__uint_as_float(v[4 * qq]) + add[4 * qq], __uint_as_float(v[4 * qq + 1]) + add[4 * qq + 1],
                                __uint_as_float(v[4 * qq + 2]) + add[4 * qq + 2],
                                __uint_as_float(v[4 * qq + 3]) + add[4 * qq + 3]);
        } else {
          // B = 32: the tile holds blocks 2t (rows/columns 0..31) and 2t+1 (32..63);
          // keep only the diagonal quadrants
          const int qb = row / 32;
          if ((h * NV) / 32 == qb) {
            float* o = dPs + ((size_t)(2 * t + qb) * 32 + (row - 32 * qb)) * 32 + (h * NV) % 32;
#pragma unroll
            for (int x = 0; x < NV; ++x) o[x] = __uint_as_float(v[x]) + add[x];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------- block backward, warp-specialised, B = 128 ---
// One CTA per (128-channel block t, row segment), with the B <= 64 kernel's roles: warp 0
// streams the (dAt, W) tiles of each 128-row chunk (two 64-channel halves each, 64 KB a stage)
// into a 2-stage ring; warp 1 issues W' = W P_hi and dA = dAt P_hi (M = 128, N = 128, K = 128)
// into one TMEM buffer once the epilogue has read the previous chunk's; warp 2 issues
// dP += dAt^T A + W^T dW' (K = 128 rows, MN-major operands) once the epilogue has written A and
// dW'; warps 3..10 (two per TMEM lane quadrant, 64 columns each) load W' and dA, release the
// buffer, and write the bf16 operand tiles.  W' is formed from P_hi alone, as for B = 256: the
// ring, the operand tiles and a second P image would need 256 KB of shared memory.  TMEM: dP at
// columns 0..127, W' at 128, dA at 256.
struct Bw128Cfg {
  static constexpr int STAGES = 2;
  static constexpr int HALF = 16384;                 // 128 rows x 64 bf16
  static constexpr int STAGE = 4 * HALF;             // dAt (two channel halves) | W (two channel halves)
  static constexpr int IMG = 2 * HALF;               // transposed P_hi of the block, two K halves
  static constexpr int AB = 4 * HALF;                // A (two slot halves) | dW' (two slot halves)
  static constexpr int CTRL_WARPS = 3, EPI_WARPS = 8;
  static constexpr int THREADS = 32 * (CTRL_WARPS + EPI_WARPS);
  static constexpr int NBAR = 2 * STAGES + 8;
  static constexpr int SMEM = STAGES * STAGE + IMG + AB + NBAR * 8 + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

__global__ void __launch_bounds__(Bw128Cfg::THREADS, 1)
block_bwd_ws128_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmDAt,
                       const __grid_constant__ CUtensorMap tmPth, const uint32_t* __restrict__ mask,
                       float* __restrict__ dP, int cout, int cin, int rows_per_split) {
  using C = Bw128Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sStage = smem;
  uint8_t* sPth = sStage + C::STAGES * C::STAGE;
  uint8_t* sAB = sPth + C::IMG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sAB + C::AB);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  constexpr int S = C::STAGES;
  constexpr int FULL = 0, EMPTY = S, IMG = 2 * S, WD = IMG + 1, TF = WD + 1, ABF = TF + 1, ABE = ABF + 1,
                DPF = ABE + 1, DRAIN = DPF + 1, DRAIN2 = DRAIN + 1;
  static_assert(DRAIN2 + 1 == C::NBAR, "barrier count");

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x, sidx = blockIdx.y, col0 = t * 128;
  const int rbeg = sidx * rows_per_split;
  const int rend = min(cout, rbeg + rows_per_split);
  const int nchunk = cdiv(rend - rbeg, 128);
  const int words = cin / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(bar(FULL + i), 1); mbar_init(bar(EMPTY + i), 1); }
    mbar_init(bar(IMG), 1);
    mbar_init(bar(WD), 1);
    mbar_init(bar(TF), C::EPI_WARPS);
    mbar_init(bar(ABF), C::EPI_WARPS);
    mbar_init(bar(ABE), 1);
    mbar_init(bar(DPF), 1);
    mbar_init(bar(DRAIN), 1);
    mbar_init(bar(DRAIN2), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  pdl_wait();
  pdl_trigger();
  const uint32_t tDP = tmem, tW = tmem + 128, tDA = tmem + 256;
  auto wait_all = [&](int b, uint32_t parity, int site) {
    return __all_sync(0xffffffffu, mbar_wait(bar(b), parity, abort_flag, site));
  };

  if (warp == 0) {
    if (lane == 0) {
      if (nchunk > 0) {
        mbar_expect_tx(bar(IMG), C::IMG);
        for (int kc = 0; kc < 2; ++kc) tma_load_2d(smem_u32(sPth + kc * C::HALF), &tmPth, bar(IMG), kc * 64, col0);
      }
      uint32_t issued = 0, par = 0;
      for (int c = 0; c < nchunk; ++c) {
        const int st = c % S;
        const uint32_t use = (uint32_t)(c / S) & 1u;
        if (!mbar_wait(bar(EMPTY + st), use ^ 1u, abort_flag, 84)) break;
        uint8_t* sg = sStage + st * C::STAGE;
        const int r0 = rbeg + c * 128;
        mbar_expect_tx(bar(FULL + st), C::STAGE);
        for (int kc = 0; kc < 2; ++kc) {
          tma_load_2d(smem_u32(sg + kc * C::HALF), &tmDAt, bar(FULL + st), col0 + kc * 64, r0);
          tma_load_2d(smem_u32(sg + (2 + kc) * C::HALF), &tmW, bar(FULL + st), col0 + kc * 64, r0);
        }
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (use << st);
      }
      for (int st = 0; st < S; ++st)
        if (issued & (1u << st)) mbar_wait_drain(bar(FULL + st), (par >> st) & 1u, 85);
      if (nchunk > 0) mbar_wait_drain(bar(IMG), 0, 86);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
      bool ok = nchunk == 0 || mbar_wait(bar(IMG), 0, abort_flag, 87);
      for (int c = 0; c < nchunk && ok; ++c) {
        const int st = c % S;
        if (!mbar_wait(bar(FULL + st), (uint32_t)(c / S) & 1u, abort_flag, 88)) break;
        // the epilogue has loaded W' and dA of chunk c - 1
        if (c >= 1 && !mbar_wait(bar(TF), (uint32_t)(c - 1) & 1u, abort_flag, 89)) break;
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
#pragma unroll
        for (int kc = 0; kc < 2; ++kc)
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t pdesc = sdesc(smem_u32(sPth) + kc * C::HALF + k16 * 32, 16, 1024);
            mma_bf16(tW, sdesc(sg + (2 + kc) * C::HALF + k16 * 32, 16, 1024), pdesc, idesc, (kc | k16) != 0);
            mma_bf16(tDA, sdesc(sg + kc * C::HALF + k16 * 32, 16, 1024), pdesc, idesc, (kc | k16) != 0);
          }
        mma_commit(bar(WD));
      }
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0, 90);
    }
    __syncwarp();
  } else if (warp == 2) {
    // dP issuer; its completion also frees the stage (W' and dA of the chunk completed before
    // the epilogue could start)
    if (lane == 0) {
      constexpr uint32_t idesc_dp = idesc_bf16(128, 128, true, true);
      const uint32_t sab = smem_u32(sAB);
      for (int c = 0; c < nchunk; ++c) {
        const int st = c % S;
        if (!mbar_wait(bar(FULL + st), (uint32_t)(c / S) & 1u, abort_flag, 91)) break;
        if (!mbar_wait(bar(ABF), (uint32_t)c & 1u, abort_flag, 92)) break;
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
        // dAt^T A, then W^T dW' (M = 128 input channels, N = 128 slots, K = 128 rows)
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_bf16(tDP, sdesc(sg + k16 * 2048, C::HALF, 1024), sdesc(sab + k16 * 2048, C::HALF, 1024), idesc_dp,
                   (c | k16) != 0);
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_bf16(tDP, sdesc(sg + 2 * C::HALF + k16 * 2048, C::HALF, 1024),
                   sdesc(sab + 2 * C::HALF + k16 * 2048, C::HALF, 1024), idesc_dp, true);
        mma_commit(bar(ABE));
        mma_commit(bar(EMPTY + st));
      }
      mma_commit(bar(DPF));
      mma_commit(bar(DRAIN2));
      mbar_wait_drain(bar(DRAIN2), 0, 93);
    }
    __syncwarp();
  } else {
    const int e = warp - C::CTRL_WARPS, q = warp & 3, h = e >> 2;   // h: 64-column half
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint8_t* rA = sAB + h * C::HALF;
    uint8_t* rD = sAB + (2 + h) * C::HALF;
    // the two mask words of this thread's 64 columns, one chunk ahead
    auto mask_bits = [&](int c) -> uint2 {
      const int grow = rbeg + c * 128 + row;
      if (c >= nchunk || grow >= rend) return make_uint2(0u, 0u);
      return __ldg(reinterpret_cast<const uint2*>(mask + (size_t)grow * words + col0 / 32 + 2 * h));
    };
    // A = M.W' and dW' = M.dA of 32 columns, packed to bf16 pairs at pa / pd [base, base + 16)
    uint32_t pa[32], pd[32];
    auto pack32 = [&](const uint32_t (&wv)[32], const uint32_t (&dv)[32], uint32_t bits, int base) {
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const bool k0 = (bits >> (2 * x)) & 1u, k1 = (bits >> (2 * x + 1)) & 1u;
        pa[base + x] = pack_bf16x2(k0 ? __uint_as_float(wv[2 * x]) : 0.f, k1 ? __uint_as_float(wv[2 * x + 1]) : 0.f);
        pd[base + x] = pack_bf16x2(k0 ? __uint_as_float(dv[2 * x]) : 0.f, k1 ? __uint_as_float(dv[2 * x + 1]) : 0.f);
      }
    };
    bool ok = true;
    uint2 next_bits = mask_bits(0);
    for (int c = 0; c < nchunk; ++c) {
      const uint2 bits = next_bits;
      next_bits = mask_bits(c + 1);
      ok = wait_all(WD, (uint32_t)c & 1u, 94);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        uint32_t wv[32], dv[32];
        tmem_ld32(tW + lane_off + h * 64 + g * 32, wv);
        tmem_ld32(tDA + lane_off + h * 64 + g * 32, dv);
        tmem_ld_wait();
        pack32(wv, dv, g ? bits.y : bits.x, 16 * g);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(TF));
      // the operand tiles were last read by the dP product of chunk c - 1
      ok = c < 1 || wait_all(ABE, (uint32_t)(c - 1) & 1u, 95);
      if (!ok) break;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        st_sw128(rA, row, c8, make_uint4(pa[4 * c8], pa[4 * c8 + 1], pa[4 * c8 + 2], pa[4 * c8 + 3]));
        st_sw128(rD, row, c8, make_uint4(pd[4 * c8], pd[4 * c8 + 1], pd[4 * c8 + 2], pd[4 * c8 + 3]));
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ABF));
    }
    if (ok) ok = wait_all(DPF, 0, 96);
    if (ok) {
      tc_fence_after();
      // thread `row` holds dP row i = row of block t, columns j = 64 h .. 64 h + 63
      const int nb = cin / 128;
      float* o = dP + (size_t)sidx * nb * 128 * 128 + ((size_t)t * 128 + row) * 128 + h * 64;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t r[32];
        tmem_ld32(tDP + lane_off + h * 64 + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 8; ++x)
          reinterpret_cast<float4*>(o + cc * 32)[x] = make_float4(__uint_as_float(r[4 * x]), __uint_as_float(r[4 * x + 1]),
                                                                  __uint_as_float(r[4 * x + 2]),
                                                                  __uint_as_float(r[4 * x + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------ block backward, B = 256 ---
// The 256 x 256 dP_b does not fit one SM's tensor memory next to W' and dA,
// so four CTAs share a block, CTA (qr, qc) owning the dP quadrant of rows
// (input channels i) [128 qr, 128 qr + 128) and columns (permuted slots j)
// [128 qc, 128 qc + 128).  Per 128-row chunk o of the CTA's row segment:
//   W'[:, qc] = W_chunk P_hi[:, qc],  dA[:, qc] = dAt_chunk P_hi[:, qc]
//                    (M = 128, N = 128, K = 256: all of the block's columns)
//   A = M.W', dW' = M.dA -> bf16 operand tiles
//   dP[qr, qc] += dAt_chunk[:, qr]^T A + W_chunk[:, qr]^T dW'   (K = 128 rows)
// Shared memory: the chunk's W and dAt tiles over the block's 256 columns (four
// 16 KB column quarters each) and the 128 rows of the transposed P_hi image
// this CTA's columns need (64 KB): 192 KB.  Once the first two products have
// read the tiles, the two column quarters of W and of dAt outside the row half
// qr are free and receive the A and dW' operand tiles, which the dP product
// reads (MN-major) next to the qr quarters of dAt and W.
// W' uses P_hi alone here (the forward pass forms W' from P_hi + P_lo, which
// decides the mask; the mask bits are read from the forward): the two P
// images would not fit beside the tiles.  TMEM: W' 128 | dA 128 | dP 128.
constexpr int Q_T_BYTES = 16384;                  // 128 rows x 64 bf16: one column quarter
constexpr int Q_SMEM = 12 * Q_T_BYTES + 1024 + 128;
constexpr int Q_THREADS = 256;   // eight warps (two per TMEM lane quadrant)

__global__ void __launch_bounds__(Q_THREADS, 1)
block_bwd_q_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmDAt,
                   const __grid_constant__ CUtensorMap tmPth, const uint32_t* __restrict__ mask,
                   float* __restrict__ dP, int cout, int cin, int rows_per_split) {
  constexpr int B = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem;                       // 4 quarters
  uint8_t* sDAt = sW + 4 * Q_T_BYTES;       // 4 quarters
  uint8_t* sPth = sDAt + 4 * Q_T_BYTES;     // 4 K-quarters of the 128 image rows j
  uint64_t* bars = reinterpret_cast<uint64_t*>(sPth + 4 * Q_T_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  // bar_q[kc]: column quarter kc of the chunk's W and dAt (and, with the first chunk, of the
  // image) has landed, so the first products run on each quarter as it arrives
  const uint32_t bar_q0 = smem_u32(bars + 3), bar_mma1 = smem_u32(bars + 0), bar_mma2 = smem_u32(bars + 1);
  const uint32_t bar_drain = smem_u32(bars + 2);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t = blockIdx.x >> 2, qr = (blockIdx.x >> 1) & 1, qc = blockIdx.x & 1;
  const int s = blockIdx.y, col0 = t * B;
  const int rbeg = s * rows_per_split;
  const int rend = min(cout, rbeg + rows_per_split);
  const int nchunk = cdiv(rend - rbeg, 128);
  // the quarters of the row half qr (read by the dP product) and the free ones (operand tiles)
  uint8_t* wq = sW + 2 * qr * Q_T_BYTES;
  uint8_t* dq = sDAt + 2 * qr * Q_T_BYTES;
  uint8_t* sAb = sW + 2 * (1 - qr) * Q_T_BYTES;     // A = M.W'  [o][j], two 64-column regions
  uint8_t* sdWb = sDAt + 2 * (1 - qr) * Q_T_BYTES;  // dW' = M.dA
  if (tid == 0) {
    for (int kc = 0; kc < 4; ++kc) mbar_init(bar_q0 + 8 * kc, 1);
    mbar_init(bar_mma1, 1);
    mbar_init(bar_mma2, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  pdl_wait();
  pdl_trigger();
  // eight warps: two per TMEM lane quadrant, each taking 64 of the quadrant's 128 columns
  const int qd = warp & 3, h = warp >> 2;
  const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
  const int row = qd * 32 + lane;
  const int words = cin / 32;
  uint32_t pending = 0;   // thread 0: quarters with a load not yet seen complete (parity pending_par)
  uint32_t pending_par = 0;
  constexpr uint32_t idesc_n = idesc_bf16(128, 128, false, false);
  constexpr uint32_t idesc_dp = idesc_bf16(128, 128, true, true);
  const uint32_t tW = tmem, tDA = tmem + 128, tDP = tmem + 256;

  bool ok = true;
  for (int ch = 0; ch < nchunk && ok; ++ch) {
    const int r0 = rbeg + ch * 128;
    if (tid == 0) {
      // the previous chunk's dP product has read every tile this load overwrites
      bool go = (ch == 0) || mbar_wait(bar_mma2, (uint32_t)(ch - 1) & 1u, abort_flag, 41);
      if (go) {
        pending = 0xFu;
        pending_par = (uint32_t)ch & 1u;
        for (int kc = 0; kc < 4; ++kc) {
          const uint32_t bq = bar_q0 + 8 * kc;
          mbar_expect_tx(bq, 2 * Q_T_BYTES + (ch == 0 ? Q_T_BYTES : 0));
          tma_load_2d(smem_u32(sW + kc * Q_T_BYTES), &tmW, bq, col0 + kc * 64, r0);
          tma_load_2d(smem_u32(sDAt + kc * Q_T_BYTES), &tmDAt, bq, col0 + kc * 64, r0);
          if (ch == 0) tma_load_2d(smem_u32(sPth + kc * Q_T_BYTES), &tmPth, bq, kc * 64, col0 + qc * 128);
        }
        for (int kc = 0; kc < 4 && go; ++kc) {
          go = mbar_wait(bar_q0 + 8 * kc, (uint32_t)ch & 1u, abort_flag, 42);
          if (!go) break;
          pending &= ~(1u << kc);
          tc_fence_after();
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t pd = sdesc(smem_u32(sPth + kc * Q_T_BYTES) + k16 * 32, 16, 1024);
            mma_bf16(tW, sdesc(smem_u32(sW + kc * Q_T_BYTES) + k16 * 32, 16, 1024), pd, idesc_n, (kc | k16) != 0);
            mma_bf16(tDA, sdesc(smem_u32(sDAt + kc * Q_T_BYTES) + k16 * 32, 16, 1024), pd, idesc_n,
                     (kc | k16) != 0);
          }
        }
        if (go) mma_commit(bar_mma1);
      }
      if (!go) *abort_flag = 1;
    }
    ok = __syncthreads_and(mbar_wait(bar_mma1, (uint32_t)ch & 1u, abort_flag, 43));
    if (!ok) break;
    tc_fence_after();
    const int grow = r0 + row;
    const bool valid = grow < rend;
#pragma unroll 1
    for (int cc = 2 * h; cc < 2 * h + 2; ++cc) {
      uint32_t wv[32], dv[32];
      tmem_ld32(tW + lane_off + cc * 32, wv);
      tmem_ld32(tDA + lane_off + cc * 32, dv);
      tmem_ld_wait();
      const uint32_t bits = valid ? __ldg(mask + (size_t)grow * words + (col0 + qc * 128) / 32 + cc) : 0u;
      uint8_t* rA = sAb + (cc / 2) * Q_T_BYTES;
      uint8_t* rD = sdWb + (cc / 2) * Q_T_BYTES;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float fa[8], fd[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const bool keep = (bits >> (8 * q + e)) & 1u;
          fa[e] = keep ? __uint_as_float(wv[8 * q + e]) : 0.f;
          fd[e] = keep ? __uint_as_float(dv[8 * q + e]) : 0.f;
        }
        const int chunk16 = (cc & 1) * 4 + q;
        st_sw128(rA, row, chunk16, make_uint4(pack_bf16x2(fa[0], fa[1]), pack_bf16x2(fa[2], fa[3]),
                                              pack_bf16x2(fa[4], fa[5]), pack_bf16x2(fa[6], fa[7])));
        st_sw128(rD, row, chunk16, make_uint4(pack_bf16x2(fd[0], fd[1]), pack_bf16x2(fd[2], fd[3]),
                                              pack_bf16x2(fd[4], fd[5]), pack_bf16x2(fd[6], fd[7])));
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // dP[qr, qc] += dAt[:, qr]^T A + W[:, qr]^T dW', contracted over the chunk's 128 rows
#pragma unroll
      for (int k16 = 0; k16 < 8; ++k16)
        mma_bf16(tDP, sdesc(smem_u32(dq) + k16 * 2048, Q_T_BYTES, 1024),
                 sdesc(smem_u32(sAb) + k16 * 2048, Q_T_BYTES, 1024), idesc_dp, (ch | k16) != 0);
#pragma unroll
      for (int k16 = 0; k16 < 8; ++k16)
        mma_bf16(tDP, sdesc(smem_u32(wq) + k16 * 2048, Q_T_BYTES, 1024),
                 sdesc(smem_u32(sdWb) + k16 * 2048, Q_T_BYTES, 1024), idesc_dp, true);
      mma_commit(bar_mma2);
    }
  }
  if (ok && nchunk > 0) ok = __syncthreads_and(mbar_wait(bar_mma2, (uint32_t)(nchunk - 1) & 1u, abort_flag, 44));
  const int nb = cin / B;
  if (ok) {
    tc_fence_after();
    // thread `row` holds dP row i = 128 qr + row of the quadrant, columns 128 qc + (0..127)
    float* o = dP + (size_t)s * nb * B * B + ((size_t)t * B + qr * 128 + row) * B + qc * 128;
#pragma unroll 1
    for (int cc = 2 * h; cc < 2 * h + 2; ++cc) {
      uint32_t r[32];
      tmem_ld32(tDP + lane_off + cc * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 8; ++e)
        reinterpret_cast<float4*>(o + cc * 32)[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                                                __uint_as_float(r[4 * e + 2]),
                                                                __uint_as_float(r[4 * e + 3]));
    }
  }
  if (tid == 0) {
    for (int kc = 0; kc < 4; ++kc)
      if (pending & (1u << kc)) mbar_wait_drain(bar_q0 + 8 * kc, pending_par, 45);
    mma_commit(bar_drain);
    mbar_wait_drain(bar_drain, 0, 46);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int bb_rows_per_split(int cout, int cin, int B) {
  const int BC = B < 64 ? 64 : B;
  const int tiles = (cin / BC) * (B == 256 ? 4 : 1);   // CTAs of one row segment (B = 256: quadrants)
  const int chunks = cdiv(cout, 128);
  // one CTA per SM: as many row segments per channel tile as fill the SMs once
  int S = 148 / tiles;
  if (S < 1) S = 1;
  if (S > 64) S = 64;
  if (S > chunks) S = chunks;
  return cdiv(chunks, S) * 128;
}

}  // namespace

lcp_status tc_error_block_bwd(int* site, int reset) { return read_tc_error(site, reset); }

bool block_bwd_tc_supported(int B) { return B == 32 || B == 64 || B == 128 || B == 256; }

int block_bwd_tc_splits(int cout, int cin, int B) {
  if (!block_bwd_tc_supported(B)) return 1;
  return cdiv(cout, bb_rows_per_split(cout, cin, B));
}

lcp_status launch_block_bwd_tc(const __nv_bfloat16* W, const __nv_bfloat16* dAt, const uint32_t* mask,
                               const __nv_bfloat16* img_pt_hi, const __nv_bfloat16* img_pt_lo, float* dP_partials,
                               int splits, int cout, int cin, int B, cudaStream_t st) {
  if (!block_bwd_tc_supported(B)) return fail(LCP_ERR_SHAPE, "block_bwd_tc: B = %d is not supported", B);
  const int BC = B < 64 ? 64 : B;
  const int rows = bb_rows_per_split(cout, cin, B);
  if (cdiv(cout, rows) != splits) return fail(LCP_ERR_ARG, "block_bwd_tc: split count mismatch");
  CUtensorMap mW, mD, mPth, mPtl;
  TC_TRY(make_map(&mW, W, cin, cout, 64, 128, "block_bwd W"));
  TC_TRY(make_map(&mD, dAt, cin, cout, 64, 128, "block_bwd dAt"));
  if (B == 256) {
    // the 128 transposed-image rows of one quadrant's columns, in 64-column K quarters
    TC_TRY(make_map(&mPth, img_pt_hi, BC, cin, 64, 128, "block_bwd Pt_hi"));
    TC_TRY(set_smem(block_bwd_q_kernel, Q_SMEM, "block_bwd_q"));
    return launch_kernel(block_bwd_q_kernel, dim3((cin / 256) * 4, splits), dim3(Q_THREADS), Q_SMEM, st, 1, true,
                         "block_bwd_q", mW, mD, mPth, mask, dP_partials, cout, cin, rows);
  }
  TC_TRY(make_map(&mPth, img_pt_hi, BC, cin, 64, BC, "block_bwd Pt_hi"));
  TC_TRY(make_map(&mPtl, img_pt_lo, BC, cin, 64, BC, "block_bwd Pt_lo"));
  if (B <= 64) {
    constexpr int NSL = 2;
    using C = BwCfg<NSL>;
    auto k = (B == 32) ? block_bwd_ws_kernel<32, NSL> : block_bwd_ws_kernel<64, NSL>;
    TC_TRY(set_smem(k, C::SMEM, "block_bwd_tc"));
    return launch_kernel(k, dim3(cin / 64, splits), dim3(C::THREADS), C::SMEM, st, 1, true, "block_bwd_tc", mW, mD,
                         mPth, mPtl, mask, dP_partials, cout, cin, rows);
  }
  using C = Bw128Cfg;
  TC_TRY(set_smem(block_bwd_ws128_kernel, C::SMEM, "block_bwd_tc"));
  return launch_kernel(block_bwd_ws128_kernel, dim3(cin / 128, splits), dim3(C::THREADS), C::SMEM, st, 1, true,
                       "block_bwd_tc", mW, mD, mPth, mask, dP_partials, cout, cin, rows);
}

}  // namespace lcp
