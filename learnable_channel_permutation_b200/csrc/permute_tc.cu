// W' = W P_B (PermLLM, Method 3: the block-diagonal permutation applied to the
// weight's input channels), the N:M mask of |W'| (integration with pruning
// methods), A = M.W' and At = A P_B^T, fused per tile on the tensor cores.

#include "tc_common.cuh"

namespace lcp {
namespace {

// ------------------------------------------------------- permute + mask ---
// One CTA: rows [r0, r0+128) x channels [t*BC, (t+1)*BC) with BC = max(B, 64),
// in 64-column chunks c:
//   W'_c  = W_tile (P_hi + P_lo)[:, chunk c]          (TMEM, 64 columns)
//   mask bits and A_c = M.W'_c (bf16, shared memory, SW128 K-major)
//   At   += A_c P_hi[:, chunk c]^T                      (TMEM, BC columns)
// P enters through the tile-format images written by the Sinkhorn kernel:
// Pt[t][j][i] = P[i][j] (B operand of the first product, rows j of chunk c),
// Ph[t][i][j] = P[i][j] (B operand of the second product, columns of chunk c).
// The images of chunk c + 1 load while chunk c is finished: Pt once the first
// product of chunk c has completed (bar_pt), Ph once its second product has
// (bar_ph, waited for only before the second product of chunk c + 1).

template <int BC> struct PmCfg {
  static constexpr int NCH = BC / 64;
  static constexpr int W_BYTES = BC * 256;   // 128 rows x BC bf16
  static constexpr int PT_BYTES = BC * 128;  // 64 rows x BC bf16 (NCH regions of 8 KB)
  static constexpr int PH_BYTES = BC * 128;  // BC rows x 64 bf16
  static constexpr int A_BYTES = 16384;      // 128 rows x 64 bf16
  static constexpr uint32_t TMEM_COLS = (64 + BC <= 128) ? 128u : ((64 + BC <= 256) ? 256u : 512u);
  static constexpr int SMEM = W_BYTES + 2 * PT_BYTES + PH_BYTES + A_BYTES + 1024 + 128;
  // 8 warps: two per TMEM lane quadrant, each taking 32 of a chunk's 64 columns (and half of
  // At's BC columns at the end), so every SM sub-partition runs two independent epilogue warps
  static constexpr int THREADS = 256;
};

template <int BC, int MGROUP>
__global__ void __launch_bounds__(PmCfg<BC>::THREADS, 1)
permute_mask_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmPth,
                       const __grid_constant__ CUtensorMap tmPtl, const __grid_constant__ CUtensorMap tmPh,
                       uint32_t* __restrict__ mask, __nv_bfloat16* __restrict__ At,
                       float* __restrict__ Wp_out, int cout, int cin, int n) {
  using C = PmCfg<BC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem;
  uint8_t* sPth = sW + C::W_BYTES;
  uint8_t* sPtl = sPth + C::PT_BYTES;
  uint8_t* sPh = sPtl + C::PT_BYTES;
  uint8_t* sA = sPh + C::PH_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sA + C::A_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const uint32_t bar_pt = smem_u32(bars + 0), bar_mma1 = smem_u32(bars + 1), bar_mma2 = smem_u32(bars + 2);
  const uint32_t bar_drain = smem_u32(bars + 3), bar_ph = smem_u32(bars + 4);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r0 = blockIdx.x * 128, t = blockIdx.y, col0 = t * BC;
  if (tid == 0) {
    mbar_init(bar_pt, 1);
    mbar_init(bar_ph, 1);
    mbar_init(bar_mma1, 1);
    mbar_init(bar_mma2, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(holder), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  pdl_wait();
  pdl_trigger();
  const int q = warp & 3, h = warp >> 2;   // TMEM lane quadrant, column half
  const uint32_t lane_off = (uint32_t)(q * 32) << 16;
  const int row = q * 32 + lane, grow = r0 + row;
  const int words = cin / 32;
  constexpr uint32_t idesc1 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t idesc2 = idesc_bf16(128, BC, false, false);

  bool ok = true;
  // thread 0: parity of a load not yet seen complete (Pt, Ph), -1 if none
  int pending_pt = -1, pending_ph = -1;
  auto load_pt = [&](int c) {   // the transposed images of chunk c (and, for c = 0, the W tile)
    pending_pt = c & 1;
    mbar_expect_tx(bar_pt, (c == 0 ? C::W_BYTES : 0) + 2 * C::PT_BYTES);
    if (c == 0)
      for (int kc = 0; kc < C::NCH; ++kc) tma_load_2d(smem_u32(sW + kc * 16384), &tmW, bar_pt, col0 + kc * 64, r0);
    for (int kc = 0; kc < C::NCH; ++kc) {
      tma_load_2d(smem_u32(sPth + kc * 8192), &tmPth, bar_pt, kc * 64, col0 + c * 64);
      tma_load_2d(smem_u32(sPtl + kc * 8192), &tmPtl, bar_pt, kc * 64, col0 + c * 64);
    }
  };
  auto load_ph = [&](int c) {   // P_hi columns of chunk c
    pending_ph = c & 1;
    mbar_expect_tx(bar_ph, C::PH_BYTES);
    tma_load_2d(smem_u32(sPh), &tmPh, bar_ph, c * 64, col0);
  };
  if (tid == 0) {
    load_pt(0);
    load_ph(0);
  }
  for (int c = 0; c < C::NCH && ok; ++c) {
    if (tid == 0) {
      bool go = mbar_wait(bar_pt, (uint32_t)c & 1u, abort_flag, 22);
      if (go) pending_pt = -1;
      if (go) {
        tc_fence_after();
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          const uint8_t* sB = pass ? sPtl : sPth;
          for (int kc = 0; kc < C::NCH; ++kc)
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(tmem, sdesc(smem_u32(sW + kc * 16384) + k16 * 32, 16, 1024),
                       sdesc(smem_u32(sB + kc * 8192) + k16 * 32, 16, 1024), idesc1,
                       (pass | kc | k16) != 0);
        }
        mma_commit(bar_mma1);
        // the second product of chunk c - 1 has read the A tile and Ph: the epilogue below may
        // overwrite the former, and Ph takes chunk c (chunk 0's was loaded up front)
        if (c > 0) {
          go = mbar_wait(bar_mma2, (uint32_t)(c - 1) & 1u, abort_flag, 21);
          if (go) load_ph(c);
        }
      }
      if (!go) *abort_flag = 1;
    }
    ok = __syncthreads_and(mbar_wait(bar_mma1, (uint32_t)c & 1u, abort_flag, 23));
    if (!ok) break;
    // the first product of chunk c has read Pt: the next chunk's transposed images may load
    if (tid == 0 && c + 1 < C::NCH) load_pt(c + 1);
    tc_fence_after();
    // this thread's 32 columns h * 32 .. of the chunk
    uint32_t v[32];
    tmem_ld32(tmem + lane_off + h * 32, v);
    tmem_ld_wait();
    const uint32_t w = MGROUP == 4 ? nm4_keep<32>(v, n) : nm_word<MGROUP>(v, n);
    if (grow < cout) {
      mask[(size_t)grow * words + (col0 + c * 64) / 32 + h] = w;
      if (Wp_out) {
        float4* o = reinterpret_cast<float4*>(Wp_out + (size_t)grow * cin + col0 + c * 64 + h * 32);
#pragma unroll
        for (int qq = 0; qq < 8; ++qq)
          o[qq] = make_float4(__uint_as_float(v[4 * qq]), __uint_as_float(v[4 * qq + 1]),
                              __uint_as_float(v[4 * qq + 2]), __uint_as_float(v[4 * qq + 3]));
      }
    }
    // A_c = M . W'_c as bf16 into the K-major SW128 operand tile (16-byte chunks 4 h .. 4 h + 3)
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = ((w >> (8 * ch + e)) & 1u) ? __uint_as_float(v[8 * ch + e]) : 0.f;
      st_sw128(sA, row, 4 * h + ch, make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                               pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      bool go = mbar_wait(bar_ph, (uint32_t)c & 1u, abort_flag, 27);
      if (go) pending_ph = -1;
      if (!go) *abort_flag = 1;
      if (go) {
        tc_fence_after();
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(tmem + 64, sdesc(smem_u32(sA) + k16 * 32, 16, 1024), sdesc(smem_u32(sPh) + k16 * 32, 16, 1024),
                   idesc2, (c | k16) != 0);
        mma_commit(bar_mma2);
      }
    }
  }
  if (ok) ok = __syncthreads_and(mbar_wait(bar_mma2, (uint32_t)(C::NCH - 1) & 1u, abort_flag, 24));
  if (ok) {
    tc_fence_after();
    // At columns: this warp's half of the BC
#pragma unroll 1
    for (int cc = h * (BC / 64); cc < (h + 1) * (BC / 64); ++cc) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + 64 + cc * 32, r);
      tmem_ld_wait();
      if (grow < cout) {
        uint4* o = reinterpret_cast<uint4*>(At + (size_t)grow * cin + col0 + cc * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          o[q] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                            pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                            pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                            pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
      }
    }
  }
  if (tid == 0) {
    // no copy or MMA of ours may still be running when the CTA exits
    if (pending_pt >= 0) mbar_wait_drain(bar_pt, (uint32_t)pending_pt, 25);
    if (pending_ph >= 0) mbar_wait_drain(bar_ph, (uint32_t)pending_ph, 28);
    mma_commit(bar_drain);
    mbar_wait_drain(bar_drain, 0, 26);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------- permute + mask, warp-specialised ---
// BC = 64 (B = 32 or 64).  CTA c takes the contiguous run
// [c * total / G, (c + 1) * total / G) of the flat (channel tile t, row tile
// rt) list in t-major order, so a run walks down one or two channel strips
// (more only when C_out is short) and the three P images of its current
// channel tile stay resident in one of two shared-memory slots.  The ring then
// carries W tiles only and a stage is free as soon as W' of its tile is
// formed, so the loads run STAGES tiles ahead of the tensor core.
// Per tile k two products:
//   W'_k = W_k P_hi + W_k P_lo  both N = 64 products accumulate into one TMEM
//                              buffer (float32), so W' is read with one load
//   At_k = A_k P_hi^T          N = 64, with A = M.W'_k written by the mask warps
//                              straight into tensor memory (bf16 pairs, row r in
//                              lane r) and read from there as the MMA's A operand
// Issuing a tcgen05.mma takes one thread about 60 cycles on an idle SM and
// several times that when the other warps of its SM sub-partition are busy
// with ALU work, while these small-N products take about 70 cycles each on the
// tensor core.  So the MMAs are shared by three issuing threads on three
// sub-partitions, each owning its products' commits:
//   warp 0: TMA producer (W ring; the images of each channel tile once)
//   warp 1: W' of every tile into TMEM buffer k % 3
//   warps 2, 3: At of the even / odd tiles into TMEM buffer k % 2
//   warps 4..11: 8 mask warps (two per TMEM lane quadrant, 32 columns each):
//           W' of tile k -> the N:M keep bits (stored to the mask) and A (tcgen05.st)
//   warps 12..15: copy-out warps (one per quadrant, 64 columns each): At of
//           tile k -> swizzled staging tile -> TMA store
// Sixteen warps, four per sub-partition, leave each thread 128 registers.
// The P-image slot of a channel tile is free once every issuer that had a
// tile in it has committed; the producer arrives for the At issuer that had
// none, so each phase of that barrier counts all three.
#ifndef LCP_PERMUTE_STAGES
#define LCP_PERMUTE_STAGES 5
#endif
#ifndef LCP_PERMUTE_MASK_WARPS
#define LCP_PERMUTE_MASK_WARPS 8   // 8 or 16 (two or four per TMEM lane quadrant)
#endif
struct PwCfg {
  static constexpr int STAGES = LCP_PERMUTE_STAGES;
  static constexpr int NW = 3;                          // W' TMEM buffers (64 columns)
  static constexpr int NAT = 2;                         // At TMEM buffers (64 columns)
  static constexpr int NA = 3;                          // A TMEM buffers (32 columns of bf16 pairs)
  static constexpr int W_BYTES = 16384;                 // 128 rows x 64 bf16
  static constexpr int IMG_BYTES = 8192;                // 64 x 64 bf16
  static constexpr int SLOT = 3 * IMG_BYTES;            // Pt_hi | Pt_lo | P_hi
  static constexpr int A_BYTES = 16384;
  static constexpr int ISSUERS = 3, MASK_WARPS = LCP_PERMUTE_MASK_WARPS, COPY_WARPS = 4;
  static constexpr int MCOLS = 64 / (MASK_WARPS / 4);   // columns per mask thread
  static constexpr int MASK0 = 1 + ISSUERS, COPY0 = MASK0 + MASK_WARPS;   // first warp of each role
  static constexpr int THREADS = 32 * (COPY0 + COPY_WARPS);
  static constexpr int NBAR = 2 * STAGES + 2 * NW + 2 * NAT + 2 * NA + 8 + ISSUERS;
  static constexpr int SMEM = STAGES * W_BYTES + 2 * SLOT + 2 * A_BYTES + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t TM_AT = NW * 64, TM_A = TM_AT + NAT * 64;   // TMEM column bases
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(TM_A + NA * 32 <= 512, "tensor memory budget");
  static_assert(MCOLS == 32 || MCOLS == 16, "a mask thread stores MCOLS / 2 columns of bf16 pairs");
};

// position in the flat t-major tile list, advanced one tile at a time
struct TileIter {
  int t, rt, nrt;
  __device__ TileIter(int idx, int nrt_) : t(idx / nrt_), rt(idx % nrt_), nrt(nrt_) {}
  __device__ void next() {
    if (++rt == nrt) { rt = 0; ++t; }
  }
};

// MODE: kFull (W' -> mask, A, At), kMaskOnly (the ranked matrix -> mask only:
// no A, no At) or kGivenMask (W' -> A and At with the mask read from `mask`).
constexpr int kFull = 0, kMaskOnly = 1, kGivenMask = 2;

template <int MGROUP, int MODE>
__global__ void __launch_bounds__(PwCfg::THREADS, 1)
permute_mask_ws_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmPth,
                       const __grid_constant__ CUtensorMap tmPtl, const __grid_constant__ CUtensorMap tmPh,
                       const __grid_constant__ CUtensorMap tmAt, uint32_t* __restrict__ mask,
                       float* __restrict__ Wp_out, int cout, int cin, int n) {
  using C = PwCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sStage = smem;
  uint8_t* sSlot = sStage + C::STAGES * C::W_BYTES;     // 2 slots of P images
  uint8_t* sO = sSlot + 2 * C::SLOT;                    // 2 staging tiles for At
  uint64_t* bars = reinterpret_cast<uint64_t*>(sO + 2 * C::A_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  constexpr int S = C::STAGES, NW = C::NW, NAT = C::NAT, NA = C::NA;
  constexpr int FULL = 0, EMPTY = S, WF = 2 * S, TMW = WF + NW, ATF = TMW + NW, TMA = ATF + NAT, AF = TMA + NAT,
                AE = AF + NA, PREADY = AE + NA, PFREE = PREADY + 2, SFULL = PFREE + 2, SFREE = SFULL + 2,
                DRAIN = SFREE + 2;
  static_assert(DRAIN + C::ISSUERS == C::NBAR, "barrier count");
  constexpr bool HAS_AT = MODE != kMaskOnly;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nrt = cdiv(cout, 128), ntc = cin / 64;
  const int total = nrt * ntc;
  const int first = (int)((long long)blockIdx.x * total / gridDim.x);
  const int last = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
  const int nloc = last - first;
  const int t_first = first / nrt;
  const int nt = nloc > 0 ? (last - 1) / nrt - t_first + 1 : 0;   // channel tiles met by the run
  const int words = cin / 32;
  auto jt_of = [&](int k) { return (first + k) / nrt - t_first; };   // run-local channel tile of tile k
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(bar(FULL + i), 1); mbar_init(bar(EMPTY + i), 1); }
    for (int i = 0; i < NW; ++i) { mbar_init(bar(WF + i), 1); mbar_init(bar(TMW + i), C::MASK_WARPS); }
    for (int i = 0; i < NAT; ++i) { mbar_init(bar(ATF + i), 1); mbar_init(bar(TMA + i), C::COPY_WARPS); }
    for (int i = 0; i < NA; ++i) { mbar_init(bar(AF + i), C::MASK_WARPS); mbar_init(bar(AE + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(PREADY + i), 1);
      mbar_init(bar(PFREE + i), HAS_AT ? 3 : 1);   // the issuers that read the P images
      mbar_init(bar(SFULL + i), C::COPY_WARPS);
      mbar_init(bar(SFREE + i), 1);
    }
    for (int i = 0; i < C::ISSUERS; ++i) mbar_init(bar(DRAIN + i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  // the producer prefetches W (never written by a kernel of the step) before waiting
  if (warp != 0) {
    pdl_wait();
    pdl_trigger();
  }
  auto wait_all = [&](int b, uint32_t parity, int site) {
    return __all_sync(0xffffffffu, mbar_wait(bar(b), parity, abort_flag, site));
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, par = 0;   // per stage: outstanding load and its parity
      uint32_t img_issued = 0;        // per slot: images in flight
      int img_next = 0;               // next channel tile (run-local) whose images to load
      bool ok = true;
      // At issuers (even / odd tiles) without a tile in channel tile jt; the W' issuer has them all
      auto absent = [&](int jt) -> int {
        const int k0 = max(0, (t_first + jt) * nrt - first);
        const int k1 = min(nloc - 1, (t_first + jt + 1) * nrt - 1 - first);
        return HAS_AT && k1 == k0 ? 1 : 0;
      };
      // images of run-local channel tiles up to jt, each into slot jt & 1 once
      // the products of channel tile jt - 2 that read the slot have completed
      auto images_upto = [&](int jt) -> bool {
        for (; img_next <= jt && img_next < nt; ++img_next) {
          const int s = img_next & 1;
          if (!mbar_wait(bar(PFREE + s), ((uint32_t)(img_next >> 1) & 1u) ^ 1u, abort_flag, 60)) return false;
          const uint32_t d = smem_u32(sSlot + s * C::SLOT);
          const int t = t_first + img_next;
          mbar_expect_tx(bar(PREADY + s), C::SLOT);
          tma_load_2d(d, &tmPth, bar(PREADY + s), 0, t * 64);
          tma_load_2d(d + C::IMG_BYTES, &tmPtl, bar(PREADY + s), 0, t * 64);
          tma_load_2d(d + 2 * C::IMG_BYTES, &tmPh, bar(PREADY + s), 0, t * 64);
          img_issued |= 1u << s;
          // this phase of the slot's free barrier: one arrival for each issuer with no tile here
          for (int a = absent(img_next); a > 0; --a) mbar_arrive(bar(PFREE + s));
        }
        return true;
      };
      // first ring fill: W tiles at once, the P images (written by the
      // Sinkhorn kernel) once the previous kernel has completed
      const int pre = nloc < S ? nloc : S;
      TileIter it(first, nrt);
      for (int k = 0; k < pre; ++k, it.next()) {
        mbar_expect_tx(bar(FULL + k), C::W_BYTES);
        tma_load_2d(smem_u32(sStage + k * C::W_BYTES), &tmW, bar(FULL + k), it.t * 64, it.rt * 128);
        issued |= 1u << k;
      }
      pdl_wait();
      pdl_trigger();
      if (nloc > 0) {
        const int jt_pre = (first + pre - 1) / nrt - t_first;
        ok = images_upto(jt_pre > 1 ? jt_pre : (nt > 1 ? 1 : 0));
      }
      for (int k = pre; k < nloc && ok; ++k, it.next()) {
        const int st = k % S;
        const uint32_t use = (uint32_t)(k / S) & 1u;
        if (!mbar_wait(bar(EMPTY + st), use ^ 1u, abort_flag, 61)) break;
        if (!images_upto(it.t - t_first)) break;
        mbar_expect_tx(bar(FULL + st), C::W_BYTES);
        tma_load_2d(smem_u32(sStage + st * C::W_BYTES), &tmW, bar(FULL + st), it.t * 64, it.rt * 128);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (use << st);
      }
      // drain: every copy this thread started has landed before the CTA exits
      for (int st = 0; st < S; ++st)
        if (issued & (1u << st)) mbar_wait_drain(bar(FULL + st), (par >> st) & 1u, 62);
      for (int s = 0; s < 2; ++s)
        if (img_issued & (1u << s)) {
          const int lastj = (img_next - 1) - ((img_next - 1 - s) & 1);   // last run-local tile loaded into slot s
          mbar_wait_drain(bar(PREADY + s), (uint32_t)(lastj >> 1) & 1u, 59);
        }
    }
    __syncwarp();
  } else if (warp < C::MASK0) {
    // issuers: warp 1 issues W' of every tile, warp 2 + p At of the tiles k = p (mod 2)
    const int role = warp == 1 ? 0 : 1;
    const int k_first = warp == 1 ? 0 : warp - 2, k_step = warp == 1 ? 1 : 2;
    if (lane == 0 && (role == 0 || HAS_AT)) {
      int cur_jt = -1;
      for (int k = k_first; k < nloc; k += k_step) {
        const int jt = jt_of(k);
        // the products of this thread that read the previous channel tile's images are issued
        if (jt != cur_jt) {
          if (cur_jt >= 0) mma_commit(bar(PFREE + (cur_jt & 1)));
          cur_jt = jt;
        }
        if (!mbar_wait(bar(PREADY + (jt & 1)), (uint32_t)(jt >> 1) & 1u, abort_flag, 58)) break;
        const uint32_t sp = smem_u32(sSlot + (jt & 1) * C::SLOT);
        if (role == 0) {
          const int st = k % S, b = k % NW;
          if (!mbar_wait(bar(FULL + st), (uint32_t)(k / S) & 1u, abort_flag, 63)) break;
          if (!mbar_wait(bar(TMW + b), ((uint32_t)(k / NW) & 1u) ^ 1u, abort_flag, 64)) break;   // W' of k - NW read
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);
          const uint32_t sw = smem_u32(sStage + st * C::W_BYTES);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t wdesc = sdesc(sw + k16 * 32, 16, 1024);
            mma_bf16(tmem + b * 64, wdesc, sdesc(sp + k16 * 32, 16, 1024), idesc, k16 != 0);
            mma_bf16(tmem + b * 64, wdesc, sdesc(sp + C::IMG_BYTES + k16 * 32, 16, 1024), idesc, true);
          }
          mma_commit(bar(WF + b));
          mma_commit(bar(EMPTY + st));
        } else {
          const int a = k % NAT, c = k % NA;
          if (!mbar_wait(bar(AF + c), (uint32_t)(k / NA) & 1u, abort_flag, 65)) break;            // A of tile k
          if (!mbar_wait(bar(TMA + a), ((uint32_t)(k / NAT) & 1u) ^ 1u, abort_flag, 69)) break;  // At of k - NAT read
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);
          const uint32_t sph = sp + 2 * C::IMG_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_bf16_ts(tmem + C::TM_AT + a * 64, tmem + C::TM_A + c * 32 + k16 * 8, sdesc(sph + k16 * 32, 16, 1024),
                        idesc, k16 != 0);
          mma_commit(bar(ATF + a));
          mma_commit(bar(AE + c));   // A buffer c reusable
        }
      }
      if (cur_jt >= 0) mma_commit(bar(PFREE + (cur_jt & 1)));
      mma_commit(bar(DRAIN + warp - 1));
      mbar_wait_drain(bar(DRAIN + warp - 1), 0, 66);
    }
    __syncwarp();
  } else if (warp < C::COPY0) {
    constexpr int NV = C::MCOLS;
    const int e = warp - C::MASK0, q = warp & 3, h = e >> 2;   // h: NV-column slice of the tile
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    TileIter it(first, nrt);
    // W' of tile k + 1 is loaded from TMEM while tile k is processed
    // (tcgen05.wait::ld waits for every outstanding load of the thread, so the
    // next load is issued only after the current one has been waited for)
    uint32_t hn[NV];
    bool have_next = nloc > 0 && wait_all(WF + 0, 0u, 67);
    if (have_next) {
      tc_fence_after();
      tmem_ld_cols<NV>(tmem + lane_off + h * NV, hn);
    }
    for (int k = 0; k < nloc && have_next; ++k, it.next()) {
      const int b = k % NW;
      tmem_ld_wait();
      uint32_t v[NV];
#pragma unroll
      for (int x = 0; x < NV; ++x) v[x] = hn[x];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(TMW + b));
      have_next = false;
      if (k + 1 < nloc) {
        const int bn = (k + 1) % NW;
        if (!wait_all(WF + bn, (uint32_t)((k + 1) / NW) & 1u, 67)) break;
        tc_fence_after();
        tmem_ld_cols<NV>(tmem + lane_off + bn * 64 + h * NV, hn);
        have_next = true;
      }
      const int grow = it.rt * 128 + row;
      if (Wp_out && grow < cout) {
        float4* o = reinterpret_cast<float4*>(Wp_out + (size_t)grow * cin + it.t * 64 + h * NV);
#pragma unroll
        for (int qq = 0; qq < NV / 4; ++qq)
          o[qq] = make_float4(__uint_as_float(v[4 * qq]), __uint_as_float(v[4 * qq + 1]),
                              __uint_as_float(v[4 * qq + 2]), __uint_as_float(v[4 * qq + 3]));
      }
      // keep bits (computed, or given) of this thread's NV columns: a mask word (NV = 32) or
      // one 16-bit half of one (NV = 16)
      const size_t wi = (size_t)grow * words + 2 * it.t;
      uint32_t w;
      if constexpr (MODE == kGivenMask) {
        if constexpr (NV == 32) w = grow < cout ? mask[wi + h] : 0u;
        else w = grow < cout ? (uint32_t)reinterpret_cast<const uint16_t*>(mask)[wi * 2 + h] : 0u;
      } else {
        w = MGROUP == 4 ? nm4_keep<NV>(v, n) : nm_bits<MGROUP, NV>(v, n);
        if (grow < cout) {
          if constexpr (NV == 32) mask[wi + h] = w;
          else reinterpret_cast<uint16_t*>(mask)[wi * 2 + h] = (uint16_t)w;
        }
      }
      if constexpr (MODE == kMaskOnly) continue;
#pragma unroll
      for (int x = 0; x < NV; ++x) v[x] = ((w >> x) & 1u) ? v[x] : 0u;
      uint32_t pk[NV / 2];
#pragma unroll
      for (int x = 0; x < NV / 2; ++x) pk[x] = pack_bf16x2(__uint_as_float(v[2 * x]), __uint_as_float(v[2 * x + 1]));
      // A buffer k % NA was last read by At of tile k - NA
      if (!wait_all(AE + k % NA, ((uint32_t)(k / NA) & 1u) ^ 1u, 57)) break;
      tmem_st_cols<NV / 2>(tmem + lane_off + C::TM_A + (k % NA) * 32 + h * (NV / 2), pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(AF + k % NA));
    }
    tmem_ld_wait();   // no TMEM load of this thread is left outstanding
  } else {
    // copy-out warps: At of tile j -> staging tile j & 1 (refilled once the
    // store of tile j - 2 has read it: SFREE) -> TMA store by the first copy
    // warp once all four have written their rows (SFULL)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool storer = warp == C::COPY0;
    TileIter it(first, nrt);
    for (int j = 0; j < nloc && HAS_AT; ++j, it.next()) {
      const int a = j % NAT, s = j & 1;
      const uint32_t us = (uint32_t)(j >> 1) & 1u;
      if (!wait_all(ATF + a, (uint32_t)(j / NAT) & 1u, 68)) break;
      tc_fence_after();
      // the staging tile is free once the store of tile j - 2 has read it
      if (!wait_all(SFREE + s, us ^ 1u, 70)) break;
      uint8_t* so = sO + s * C::A_BYTES;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + C::TM_AT + a * 64 + hh * 32, u);
        tmem_ld_wait();
        if (hh == 1) {
          // the TMEM buffer may take At of tile j + NAT
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(TMA + a));
        }
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_sw128(so, row, 4 * hh + c8,
                   make_uint4(pack_bf16x2(__uint_as_float(u[8 * c8 + 0]), __uint_as_float(u[8 * c8 + 1])),
                              pack_bf16x2(__uint_as_float(u[8 * c8 + 2]), __uint_as_float(u[8 * c8 + 3])),
                              pack_bf16x2(__uint_as_float(u[8 * c8 + 4]), __uint_as_float(u[8 * c8 + 5])),
                              pack_bf16x2(__uint_as_float(u[8 * c8 + 6]), __uint_as_float(u[8 * c8 + 7]))));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(SFULL + s));
      if (storer) {
        if (!wait_all(SFULL + s, us, 71)) break;
        if (lane == 0) {
          tma_store_2d(&tmAt, smem_u32(so), it.t * 64, it.rt * 128);
          bulk_commit();
          // the store of tile j - 1 has read staging tile s ^ 1: it may be refilled
          if (j >= 1) {
            bulk_wait_read<1>();
            mbar_arrive(bar(SFREE + (s ^ 1)));
          }
        }
        __syncwarp();
      }
    }
    if (storer && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------- permute + mask, warp-specialised, B = 128 ---
// The B <= 64 kernel's scheme for 128-channel blocks.  Tile k = (channel tile t
// of 128 channels, row tile rt); each of its two 64-column chunks c needs all
// 128 input channels of the block:
//   W'_{k,c} = W_k [P_hi | P_lo]_{rows of chunk c}   N = 128 (the two transposed
//              images of the chunk stacked), K = 128 (two 64-channel W halves)
//   At_k     = A_k P_hi^T                              N = 128, K = 128
// Shared memory: a 2-stage ring of W tiles (128 rows x 128 channels, 32 KB),
// one slot with the channel tile's images (Pt_hi / Pt_lo pairs per chunk and
// K half, 4 x 16 KB, and P_hi, 2 x 16 KB) reloaded when the run moves to the
// next channel tile, and two A buffers (32 KB): 224 KB.  TMEM: two W' chunk
// buffers (hi | lo, 128 columns) and two At buffers (128 columns).  The copy-out
// warps write At straight from registers (16-byte stores).  Roles as in the
// B <= 64 kernel: warp 0 TMA producer; warp 1 issues W' of every chunk, warps
// 2 and 3 At of the even / odd tiles; warps 4..11 mask warps (two per TMEM lane
// quadrant, 32 columns of the chunk each); warps 12..15 copy-out.
struct Pw128Cfg {
  static constexpr int STAGES = 2;
  static constexpr int W_BYTES = 32768;                 // 128 rows x 128 bf16 (two 16 KB halves)
  static constexpr int SLOT = 6 * 16384;                // Pt pairs [c][kc] (hi 8 KB | lo 8 KB), then P_hi [kj]
  static constexpr int A_BYTES = 32768;                 // two 16 KB K halves
  static constexpr int ISSUERS = 3, MASK_WARPS = 8, COPY_WARPS = 4;
  static constexpr int MASK0 = 1 + ISSUERS, COPY0 = MASK0 + MASK_WARPS;
  static constexpr int THREADS = 32 * (COPY0 + COPY_WARPS);
  static constexpr int NBAR = 2 * STAGES + 2 + 2 * 2 + 2 * 2 + 2 * 2 + ISSUERS;
  static constexpr int SMEM = STAGES * W_BYTES + SLOT + 2 * A_BYTES + NBAR * 8 + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int MGROUP>
__global__ void __launch_bounds__(Pw128Cfg::THREADS, 1)
permute_mask_ws128_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmPth,
                          const __grid_constant__ CUtensorMap tmPtl, const __grid_constant__ CUtensorMap tmPh,
                          uint32_t* __restrict__ mask, __nv_bfloat16* __restrict__ At, float* __restrict__ Wp_out,
                          int cout, int cin, int n) {
  using C = Pw128Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sStage = smem;
  uint8_t* sSlot = sStage + C::STAGES * C::W_BYTES;
  uint8_t* sA = sSlot + C::SLOT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sA + 2 * C::A_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  constexpr int S = C::STAGES;
  constexpr int FULL = 0, EMPTY = S, PREADY = 2 * S, PFREE = PREADY + 1, WF = PFREE + 1, TMW = WF + 2,
                ATF = TMW + 2, TMA = ATF + 2, AF = TMA + 2, AE = AF + 2, DRAIN = AE + 2;
  static_assert(DRAIN + C::ISSUERS == C::NBAR, "barrier count");
  constexpr uint32_t TM_AT = 256;   // At buffers at columns 256 + 128 b

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nrt = cdiv(cout, 128), ntc = cin / 128;
  const int total = nrt * ntc;
  const int first = (int)((long long)blockIdx.x * total / gridDim.x);
  const int last = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
  const int nloc = last - first;
  const int t_first = first / nrt;
  const int nt = nloc > 0 ? (last - 1) / nrt - t_first + 1 : 0;
  const int words = cin / 32;
  auto jt_of = [&](int k) { return (first + k) / nrt - t_first; };
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(bar(FULL + i), 1); mbar_init(bar(EMPTY + i), 1); }
    mbar_init(bar(PREADY), 1);
    mbar_init(bar(PFREE), 3);   // the W' issuer and both At issuers
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(WF + i), 1);
      mbar_init(bar(TMW + i), C::MASK_WARPS);
      mbar_init(bar(ATF + i), 1);
      mbar_init(bar(TMA + i), C::COPY_WARPS);
      mbar_init(bar(AF + i), C::MASK_WARPS);
      mbar_init(bar(AE + i), 1);
    }
    for (int i = 0; i < C::ISSUERS; ++i) mbar_init(bar(DRAIN + i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  if (warp != 0) {
    pdl_wait();
    pdl_trigger();
  }
  auto wait_all = [&](int b, uint32_t parity, int site) {
    return __all_sync(0xffffffffu, mbar_wait(bar(b), parity, abort_flag, site));
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, par = 0;
      int img_next = 0;
      bool img_issued = false;
      bool ok = true;
      auto absent = [&](int jt) -> int {   // At issuers with no tile in channel tile jt
        const int k0 = max(0, (t_first + jt) * nrt - first);
        const int k1 = min(nloc - 1, (t_first + jt + 1) * nrt - 1 - first);
        return k1 == k0 ? 1 : 0;
      };
      // images of channel tile jt into the slot once every product of jt - 1 has completed
      auto images_upto = [&](int jt) -> bool {
        for (; img_next <= jt && img_next < nt; ++img_next) {
          if (!mbar_wait(bar(PFREE), ((uint32_t)img_next & 1u) ^ 1u, abort_flag, 160)) return false;
          const int t = t_first + img_next;
          const uint32_t d = smem_u32(sSlot);
          mbar_expect_tx(bar(PREADY), C::SLOT);
          for (int c = 0; c < 2; ++c)
            for (int kc = 0; kc < 2; ++kc) {
              const uint32_t pair = d + (c * 2 + kc) * 16384;
              tma_load_2d(pair, &tmPth, bar(PREADY), kc * 64, t * 128 + c * 64);
              tma_load_2d(pair + 8192, &tmPtl, bar(PREADY), kc * 64, t * 128 + c * 64);
            }
          for (int kj = 0; kj < 2; ++kj) tma_load_2d(d + (4 + kj) * 16384, &tmPh, bar(PREADY), kj * 64, t * 128);
          img_issued = true;
          for (int a = absent(img_next); a > 0; --a) mbar_arrive(bar(PFREE));
        }
        return true;
      };
      auto load_w = [&](int k, int st) {
        const int idx = first + k, t = idx / nrt, rt = idx % nrt;
        mbar_expect_tx(bar(FULL + st), C::W_BYTES);
        for (int kc = 0; kc < 2; ++kc)
          tma_load_2d(smem_u32(sStage + st * C::W_BYTES + kc * 16384), &tmW, bar(FULL + st), t * 128 + kc * 64,
                      rt * 128);
      };
      const int pre = nloc < S ? nloc : S;
      for (int k = 0; k < pre; ++k) {
        load_w(k, k);
        issued |= 1u << k;
      }
      pdl_wait();
      pdl_trigger();
      if (nloc > 0) ok = images_upto(0);
      for (int k = pre; k < nloc && ok; ++k) {
        const int st = k % S;
        const uint32_t use = (uint32_t)(k / S) & 1u;
        if (!mbar_wait(bar(EMPTY + st), use ^ 1u, abort_flag, 161)) break;
        if (!images_upto(jt_of(k))) break;
        load_w(k, st);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (use << st);
      }
      for (int st = 0; st < S; ++st)
        if (issued & (1u << st)) mbar_wait_drain(bar(FULL + st), (par >> st) & 1u, 162);
      if (img_issued) mbar_wait_drain(bar(PREADY), (uint32_t)(img_next - 1) & 1u, 163);
    }
    __syncwarp();
  } else if (warp < C::MASK0) {
    const int role = warp == 1 ? 0 : 1;
    const int k_first = warp == 1 ? 0 : warp - 2, k_step = warp == 1 ? 1 : 2;
    if (lane == 0) {
      int cur_jt = -1;
      const uint32_t slot = smem_u32(sSlot);
      for (int k = k_first; k < nloc; k += k_step) {
        const int jt = jt_of(k);
        if (jt != cur_jt) {
          if (cur_jt >= 0) mma_commit(bar(PFREE));
          cur_jt = jt;
        }
        if (!mbar_wait(bar(PREADY), (uint32_t)jt & 1u, abort_flag, 158)) break;
        bool ok = true;
        if (role == 0) {
          const int st = k % S;
          if (!mbar_wait(bar(FULL + st), (uint32_t)(k / S) & 1u, abort_flag, 163)) break;
          constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
          const uint32_t sw = smem_u32(sStage + st * C::W_BYTES);
          for (int c = 0; c < 2 && ok; ++c) {
            const int q = 2 * k + c, b = q & 1;
            if (!mbar_wait(bar(TMW + b), ((uint32_t)(q >> 1) & 1u) ^ 1u, abort_flag, 164)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kc = 0; kc < 2; ++kc)
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                mma_bf16(tmem + b * 128, sdesc(sw + kc * 16384 + k16 * 32, 16, 1024),
                         sdesc(slot + (c * 2 + kc) * 16384 + k16 * 32, 16, 1024), idesc, (kc | k16) != 0);
            mma_commit(bar(WF + b));
          }
          if (!ok) break;
          mma_commit(bar(EMPTY + st));
        } else {
          const int a = k & 1;
          if (!mbar_wait(bar(AF + a), (uint32_t)(k >> 1) & 1u, abort_flag, 165)) break;
          if (!mbar_wait(bar(TMA + a), ((uint32_t)(k >> 1) & 1u) ^ 1u, abort_flag, 169)) break;
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
          const uint32_t sa = smem_u32(sA + a * C::A_BYTES);
#pragma unroll
          for (int kj = 0; kj < 2; ++kj)
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(tmem + TM_AT + a * 128, sdesc(sa + kj * 16384 + k16 * 32, 16, 1024),
                       sdesc(slot + (4 + kj) * 16384 + k16 * 32, 16, 1024), idesc, (kj | k16) != 0);
          mma_commit(bar(ATF + a));
          mma_commit(bar(AE + a));
        }
      }
      if (cur_jt >= 0) mma_commit(bar(PFREE));
      mma_commit(bar(DRAIN + warp - 1));
      mbar_wait_drain(bar(DRAIN + warp - 1), 0, 166);
    }
    __syncwarp();
  } else if (warp < C::COPY0) {
    // mask warps: chunk q = 2 k + c of tile k.  W' of chunk q + 1 is waited for and loaded
    // only once chunk q is finished (its A half written, the A buffer released after chunk 1):
    // with one image slot, W' of the first chunk of the next channel tile waits for the images,
    // the images for every At product of this channel tile, and those for this tile's A.
    constexpr int NV = 32;
    const int e = warp - C::MASK0, qd = warp & 3, h = e >> 2;
    const int row = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const int nq = 2 * nloc;
    uint32_t hi[NV], lo[NV];
    bool have = nq > 0 && wait_all(WF + 0, 0u, 167);
    if (have) {
      tc_fence_after();
      tmem_ld32(tmem + lane_off + h * NV, hi);
      tmem_ld32(tmem + lane_off + 64 + h * NV, lo);
    }
    for (int q = 0; q < nq && have; ++q) {
      const int k = q >> 1, c = q & 1, b = q & 1;
      tmem_ld_wait();
      uint32_t v[NV];
#pragma unroll
      for (int x = 0; x < NV; ++x) v[x] = __float_as_uint(__uint_as_float(hi[x]) + __uint_as_float(lo[x]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(TMW + b));
      const int idx = first + k, t = idx / nrt, rt = idx % nrt;
      const int grow = rt * 128 + row;
      const int col = t * 128 + c * 64 + h * NV;
      if (Wp_out && grow < cout) {
        float4* o = reinterpret_cast<float4*>(Wp_out + (size_t)grow * cin + col);
#pragma unroll
        for (int qq = 0; qq < NV / 4; ++qq)
          o[qq] = make_float4(__uint_as_float(v[4 * qq]), __uint_as_float(v[4 * qq + 1]),
                              __uint_as_float(v[4 * qq + 2]), __uint_as_float(v[4 * qq + 3]));
      }
      const uint32_t w = MGROUP == 4 ? nm4_keep<NV>(v, n) : nm_bits<MGROUP, NV>(v, n);
      if (grow < cout) mask[(size_t)grow * words + col / 32] = w;
#pragma unroll
      for (int x = 0; x < NV; ++x) v[x] = ((w >> x) & 1u) ? v[x] : 0u;
      // A buffer k & 1 was last read by At of tile k - 2
      if (c == 0 && !wait_all(AE + (k & 1), ((uint32_t)(k >> 1) & 1u) ^ 1u, 157)) break;
      uint8_t* sa = sA + (k & 1) * C::A_BYTES + c * 16384;
#pragma unroll
      for (int c8 = 0; c8 < NV / 8; ++c8)
        st_sw128(sa, row, h * (NV / 8) + c8,
                 make_uint4(pack_bf16x2(__uint_as_float(v[8 * c8 + 0]), __uint_as_float(v[8 * c8 + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * c8 + 2]), __uint_as_float(v[8 * c8 + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * c8 + 4]), __uint_as_float(v[8 * c8 + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * c8 + 6]), __uint_as_float(v[8 * c8 + 7]))));
      if (c == 1) {
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(AF + (k & 1)));
      }
      have = false;
      if (q + 1 < nq) {
        const int bn = (q + 1) & 1;
        if (!wait_all(WF + bn, (uint32_t)((q + 1) >> 1) & 1u, 167)) break;
        tc_fence_after();
        tmem_ld32(tmem + lane_off + bn * 128 + h * NV, hi);
        tmem_ld32(tmem + lane_off + bn * 128 + 64 + h * NV, lo);
        have = true;
      }
    }
    tmem_ld_wait();
  } else {
    // copy-out warps: At of tile k (128 columns) -> 16-byte stores of the row
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    for (int k = 0; k < nloc; ++k) {
      const int a = k & 1;
      if (!wait_all(ATF + a, (uint32_t)(k >> 1) & 1u, 168)) break;
      tc_fence_after();
      const int idx = first + k, t = idx / nrt, rt = idx % nrt;
      const int grow = rt * 128 + row;
      uint4* o = reinterpret_cast<uint4*>(At + (size_t)grow * cin + t * 128);
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + TM_AT + a * 128 + cc * 32, u);
        tmem_ld_wait();
        if (cc == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(TMA + a));   // the buffer may take At of tile k + 2
        }
        if (grow < cout) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            o[cc * 4 + c8] =
                make_uint4(pack_bf16x2(__uint_as_float(u[8 * c8 + 0]), __uint_as_float(u[8 * c8 + 1])),
                           pack_bf16x2(__uint_as_float(u[8 * c8 + 2]), __uint_as_float(u[8 * c8 + 3])),
                           pack_bf16x2(__uint_as_float(u[8 * c8 + 4]), __uint_as_float(u[8 * c8 + 5])),
                           pack_bf16x2(__uint_as_float(u[8 * c8 + 6]), __uint_as_float(u[8 * c8 + 7])));
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

template <int BC, int MG>
lcp_status permute_mask_bc(const CUtensorMap& mW, const CUtensorMap& mPth, const CUtensorMap& mPtl,
                           const CUtensorMap& mPh, uint32_t* mask, __nv_bfloat16* At, float* Wp, int cout,
                           int cin, int n, cudaStream_t st) {
  auto k = permute_mask_tc_kernel<BC, MG>;
  TC_TRY(set_smem(k, PmCfg<BC>::SMEM, "permute_mask_tc"));
  const dim3 grid(cdiv(cout, 128), cin / BC);
  return launch_kernel(k, grid, dim3(PmCfg<BC>::THREADS), PmCfg<BC>::SMEM, st, 1, true, "permute_mask_tc", mW, mPth,
                       mPtl, mPh, mask,
                       At, Wp, cout, cin, n);
}

}  // namespace

lcp_status tc_error_permute(int* site, int reset) { return read_tc_error(site, reset); }

lcp_status launch_score_mask_tc(const __nv_bfloat16* S, const __nv_bfloat16* img_pt_hi,
                                const __nv_bfloat16* img_pt_lo, const __nv_bfloat16* img_p_hi, uint32_t* mask,
                                float* Shat_out, int cout, int cin, int B, int n, int m, cudaStream_t st) {
  if (B > 64) return fail(LCP_ERR_SHAPE, "score_mask_tc: B = %d (the tensor-core score path takes B <= 64)", B);
  CUtensorMap mS, mPth, mPtl, mPh;
  TC_TRY(make_map(&mS, S, cin, cout, 64, 128, "score_mask S"));
  TC_TRY(make_map(&mPth, img_pt_hi, 64, cin, 64, 64, "score_mask Pt_hi"));
  TC_TRY(make_map(&mPtl, img_pt_lo, 64, cin, 64, 64, "score_mask Pt_lo"));
  TC_TRY(make_map(&mPh, img_p_hi, 64, cin, 64, 64, "score_mask P_hi"));
  using C = PwCfg;
  auto k = (m == 4) ? permute_mask_ws_kernel<4, kMaskOnly> : permute_mask_ws_kernel<8, kMaskOnly>;
  TC_TRY(set_smem(k, C::SMEM, "score_mask_tc"));
  const int tiles = cdiv(cout, 128) * (cin / 64);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  // no At in this mode: the At map is never used (the S map stands in)
  return launch_kernel(k, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, true, "score_mask_tc", mS, mPth, mPtl, mPh,
                       mS, mask, Shat_out, cout, cin, n);
}

lcp_status launch_permute_mask_tc(const __nv_bfloat16* W, const __nv_bfloat16* img_pt_hi,
                                  const __nv_bfloat16* img_pt_lo, const __nv_bfloat16* img_p_hi, uint32_t* mask,
                                  __nv_bfloat16* At, float* Wp_out, int cout, int cin, int B, int n, int m,
                                  bool given_mask, cudaStream_t st) {
  const int BC = B < 64 ? 64 : B;
  CUtensorMap mW, mPth, mPtl, mPh;
  TC_TRY(make_map(&mW, W, cin, cout, 64, 128, "permute_mask W"));
  TC_TRY(make_map(&mPth, img_pt_hi, BC, cin, 64, 64, "permute_mask Pt_hi"));
  TC_TRY(make_map(&mPtl, img_pt_lo, BC, cin, 64, 64, "permute_mask Pt_lo"));
  TC_TRY(make_map(&mPh, img_p_hi, BC, cin, 64, BC == 64 ? 64 : BC, "permute_mask P_hi"));
  if (BC == 64) {
    CUtensorMap mAt;
    TC_TRY(make_map(&mAt, At, cin, cout, 64, 128, "permute_mask At"));
    using C = PwCfg;
    auto k = (m == 4) ? (given_mask ? permute_mask_ws_kernel<4, kGivenMask> : permute_mask_ws_kernel<4, kFull>)
                      : (given_mask ? permute_mask_ws_kernel<8, kGivenMask> : permute_mask_ws_kernel<8, kFull>);
    TC_TRY(set_smem(k, C::SMEM, "permute_mask_tc"));
    const int tiles = cdiv(cout, 128) * (cin / 64);
    const int grid = tiles < num_sms() ? tiles : num_sms();
    return launch_kernel(k, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, true, "permute_mask_tc", mW, mPth, mPtl,
                         mPh, mAt, mask, Wp_out, cout, cin, n);
  }
  if (given_mask) return fail(LCP_ERR_SHAPE, "permute_mask_tc: a given mask needs B <= 64 (B = %d)", B);
  if (BC == 128) {
    using C = Pw128Cfg;
    auto k = (m == 4) ? permute_mask_ws128_kernel<4> : permute_mask_ws128_kernel<8>;
    TC_TRY(set_smem(k, C::SMEM, "permute_mask_tc"));
    const int tiles = cdiv(cout, 128) * (cin / 128);
    const int grid = tiles < num_sms() ? tiles : num_sms();
    return launch_kernel(k, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, true, "permute_mask_tc", mW, mPth, mPtl,
                         mPh, mask, At, Wp_out, cout, cin, n);
  }
  if (m == 4) return permute_mask_bc<256, 4>(mW, mPth, mPtl, mPh, mask, At, Wp_out, cout, cin, n, st);
  return permute_mask_bc<256, 8>(mW, mPth, mPtl, mPh, mask, At, Wp_out, cout, cin, n, st);
}

}  // namespace lcp
