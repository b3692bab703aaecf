// Dense bf16 products of the LCP step on the tensor cores (tcgen05, CTA pairs):
// the calibration outputs Y_d = X W^T and Y_s = X At^T (PermLLM summary,
// "optimization objective": the dense and sparse outputs), and the weight
// gradient dAt = G^T X of the reverse pass.
//
// The calibration products can also run with the cosine-loss reduction in the
// epilogue (LOSS mode): both outputs of the same 256 tokens x 128 channels come
// out of one MMA, and the epilogue writes, instead of the two float32 outputs,
// per-token partial sums <y_d, y_s>, |y_d|^2, |y_s|^2 over each 64-channel
// slot and the pair D = Y_d - Y_s, Y_s in bf16 -- all the loss and its
// gradient G need (see loss.cu, loss_pair_kernel).

#include "tc_common.cuh"

namespace lcp {
namespace {

constexpr int GM_THREADS = 192;   // warp 0: TMA producer, warp 1: MMA issuer, warps 2-5: epilogue

// ------------------------------------------------------ GEMM, CTA pairs ---
// Same product as gemm_tc_kernel with 256 x 256 output tiles computed by a
// cluster of two CTAs on two SMs (tcgen05 cta_group::2): CTA r stages rows
// [128 r, 128 r + 128) of the tile's A block and of its B block; the leader
// (rank 0) issues M = 256, N = 256 MMAs that read both CTAs' operands, and each
// CTA holds its 128 x 256 half of the accumulator in its own tensor memory.
// Per SM this halves the B bytes per MMA cycle (32 KB of operands per 64-deep
// k-block instead of 48 KB), and seven stages fit in shared memory.
//
// Tiles go to pairs round-robin.  When the last round would leave more than half
// of the pairs idle, its tiles are split into two 256 x 128 halves (N = 128
// MMAs, 64 B rows per CTA), so the pairs that still work finish in about half a
// tile's time instead of a whole one.
constexpr int G2_BM = 256, G2_BN = 256, G2_BK = 64, G2_STAGES = 7;
constexpr int G2_HALF = 128 * G2_BK * 2;               // one 128-row operand half: 16 KB
constexpr int G2_SMEM = G2_STAGES * 2 * G2_HALF + 1024 + 256;

// Work items of the round-robin schedule: whole tiles [0, split_base), then the
// remaining tiles as two halves each.
struct PairSched {
  int items, split_base;
  __device__ PairSched(int total, int npairs) {
    const int rem = total % npairs;
    if (rem != 0 && 2 * rem <= npairs) {
      split_base = total - rem;
      items = split_base + 2 * rem;
    } else {
      split_base = total;
      items = total;
    }
  }
  // tile of item it; half -1 for the whole tile, else the 128-column half
  __device__ void at(int it, int& tile, int& half) const {
    if (it < split_base) {
      tile = it;
      half = -1;
    } else {
      tile = split_base + ((it - split_base) >> 1);
      half = (it - split_base) & 1;
    }
  }
};

// LOSS mode (calibration products only): item = 256 tokens x 128 channels of
// both problems.  CTA 0 of the pair stages the channels' rows of B0 = W, CTA 1
// the same rows of B1 = At, so the N = 256 MMA leaves accumulator columns
// [0, 128) = Y_d and [128, 256) = Y_s (a half item: 64 channels, N = 128,
// columns [0, 64) and [64, 128)).  D0 receives D = Y_d - Y_s and D1 Y_s, both
// bf16 [M, N] with row stride ldd; part[row * nslots + s] the float4
// (<y_d, y_s>, |y_d|^2, |y_s|^2, 0) of channels [64 s, 64 s + 64).
template <bool A_MN, bool B_MN, bool OUT_BF16, bool LOSS>
__global__ void __launch_bounds__(GM_THREADS, 1)
gemm_pair_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, void* __restrict__ D0, void* __restrict__ D1,
                    float4* __restrict__ part, int nslots, int M, int N, int K, int ldd, int nprob) {
  static_assert(!LOSS || (!A_MN && !B_MN && !OUT_BF16), "the loss epilogue belongs to the calibration products");
  constexpr int BNT = LOSS ? 128 : G2_BN;   // output channels per item (of each problem in LOSS mode)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + G2_STAGES * G2_HALF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + G2_STAGES * G2_HALF);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 2 * G2_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto full = [&](int s) { return smem_u32(bars + s); };               // leader's counts both halves
  auto empty = [&](int s) { return smem_u32(bars + G2_STAGES + s); };  // one per CTA
  auto tfull = [&](int a) { return smem_u32(bars + 2 * G2_STAGES + a); };
  auto tempty = [&](int a) { return smem_u32(bars + 2 * G2_STAGES + 2 + a); };  // leader: 8 warps
  const uint32_t drain = smem_u32(bars + 2 * G2_STAGES + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < G2_STAGES; ++s) {
      mbar_init(full(s), 2);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(holder), 512);
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem = *holder;
  pdl_wait();           // operands come from the previous kernel
  pdl_trigger();

  const int mtiles = cdiv(M, G2_BM), ntiles = cdiv(N, BNT);
  const int total = mtiles * ntiles * nprob;
  const int nk = cdiv(K, G2_BK);
  const PairSched sched(total, npairs);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_par = 0;
      for (int it = pair; it < sched.items; it += npairs) {
        int tile, half;
        sched.at(it, tile, half);
        const int mt = tile % mtiles, rest = tile / mtiles;
        const int nt = rest % ntiles, prob = rest / ntiles;
        const CUtensorMap* mb = (LOSS ? rank : prob) ? &tmB1 : &tmB0;
        // each CTA stages half of the tile's B rows: 128 of a whole tile, 64 of a half
        // (LOSS: CTA r stages all the item's channels of problem r)
        const int a_row = mt * G2_BM + (int)rank * 128;
        const int b_row = LOSS ? nt * BNT + (half < 0 ? 0 : half * 64)
                               : nt * G2_BN + (half < 0 ? (int)rank * 128 : half * 128 + (int)rank * 64);
        const uint32_t bytes = half < 0 ? 2 * G2_HALF : G2_HALF + G2_HALF / 2;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty(stage), ph ^ 1u, abort_flag, 91)) { ok = false; break; }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (ph << stage);
          const uint32_t fbar = mapa(full(stage), 0);
          mbar_expect_tx_cluster(fbar, bytes);
          const uint32_t a_dst = smem_u32(sA + stage * G2_HALF);
          const uint32_t b_dst = smem_u32(sB + stage * G2_HALF);
          if (!A_MN) {
            tma_load_2d_pair(a_dst, &tmA, fbar, kb * G2_BK, a_row);
          } else {
            tma_load_2d_pair(a_dst, &tmA, fbar, a_row, kb * G2_BK);
            tma_load_2d_pair(a_dst + 8192, &tmA, fbar, a_row + 64, kb * G2_BK);
          }
          // B in boxes of 64 rows (K-major) or 64 columns (MN-major), 8 KB each
          if (!B_MN) {
            tma_load_2d_pair(b_dst, mb, fbar, kb * G2_BK, b_row);
            if (half < 0) tma_load_2d_pair(b_dst + 8192, mb, fbar, kb * G2_BK, b_row + 64);
          } else {
            tma_load_2d_pair(b_dst, mb, fbar, b_row, kb * G2_BK);
            if (half < 0) tma_load_2d_pair(b_dst + 8192, mb, fbar, b_row + 64, kb * G2_BK);
          }
          if (++stage == G2_STAGES) { stage = 0; ph ^= 1u; }
        }
        if (!ok) break;
      }
      // our copies have landed once our own empty barrier shows the leader consumed
      // them, or (after an abort) once the leader's full barrier completed: wait for
      // every stage still outstanding on the leader's barrier
      if (rank == 0)
        for (int st = 0; st < G2_STAGES; ++st)
          if (issued & (1u << st)) mbar_wait_drain(full(st), (issued_par >> st) & 1u, 92);
      if (rank != 0)
        for (int st = 0; st < G2_STAGES; ++st)
          if (issued & (1u << st)) mbar_wait_drain(empty(st), (issued_par >> st) & 1u, 93);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_full = idesc_bf16(G2_BM, G2_BN, A_MN, B_MN);
      constexpr uint32_t idesc_half = idesc_bf16(G2_BM, G2_BN / 2, A_MN, B_MN);
      int stage = 0, lt = 0;
      uint32_t ph = 0;
      for (int it = pair; it < sched.items; it += npairs, ++lt) {
        int tile, half;
        sched.at(it, tile, half);
        const uint32_t idesc = half < 0 ? idesc_full : idesc_half;
        const int acc = lt & 1;
        const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
        if (!mbar_wait(tempty(acc), aph ^ 1u, abort_flag, 94)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * G2_BN);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full(stage), ph, abort_flag, 95)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * G2_HALF);
          const uint32_t b0 = smem_u32(sB + stage * G2_HALF);
#pragma unroll
          for (int k16 = 0; k16 < G2_BK / 16; ++k16) {
            const uint64_t ad = A_MN ? sdesc(a0 + k16 * 2048, 8192, 1024) : sdesc(a0 + k16 * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc(b0 + k16 * 2048, 8192, 1024) : sdesc(b0 + k16 * 32, 16, 1024);
            mma_bf16_pair(d, ad, bd, idesc, (kb | k16) != 0);
          }
          mma_commit_pair(empty(stage), 0x3);
          if (++stage == G2_STAGES) { stage = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(tfull(acc), 0x3);
      }
      mma_commit_pair(drain, 0x1);
      mbar_wait_drain(drain, 0, 96);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    const uint32_t tempty_leader0 = mapa(tempty(0), 0), tempty_leader1 = mapa(tempty(1), 0);
    int lt = 0;
    for (int it = pair; it < sched.items; it += npairs, ++lt) {
      int tile, half;
      sched.at(it, tile, half);
      const int acc = lt & 1;
      const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
      if (!warp_all(mbar_wait(tfull(acc), aph, abort_flag, 97))) break;
      tc_fence_after();
      const int mt = tile % mtiles, rest = tile / mtiles;
      const int nt = rest % ntiles, prob = rest / ntiles;
      if constexpr (LOSS) {
        const int row = mt * G2_BM + (int)rank * 128 + q * 32 + lane;
        const int ncol = half < 0 ? 128 : 64;             // channels of each problem in this item
        const int col_base = nt * BNT + (half < 0 ? 0 : half * 64);
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * G2_BN);
#pragma unroll 1
        for (int s64 = 0; s64 < ncol / 64; ++s64) {
          float dot = 0.f, nd = 0.f, ns = 0.f;
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            const int cc = s64 * 64 + h * 32;
            uint32_t rd[32], rs[32];
            tmem_ld32(tbase + (uint32_t)cc, rd);
            tmem_ld32(tbase + (uint32_t)(ncol + cc), rs);
            tmem_ld_wait();
#pragma unroll
            for (int v = 0; v < 32; ++v) {
              const float yd = __uint_as_float(rd[v]), ys = __uint_as_float(rs[v]);
              dot = fmaf(yd, ys, dot);
              nd = fmaf(yd, yd, nd);
              ns = fmaf(ys, ys, ns);
            }
            const int col0 = col_base + cc;
            if (row < M && col0 < N) {
              __nv_bfloat16* od = static_cast<__nv_bfloat16*>(D0) + (size_t)row * ldd + col0;
              __nv_bfloat16* os = static_cast<__nv_bfloat16*>(D1) + (size_t)row * ldd + col0;
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                if (col0 + 8 * v < N) {
                  float fd[8], fs[8];
#pragma unroll
                  for (int u = 0; u < 8; ++u) {
                    fs[u] = __uint_as_float(rs[8 * v + u]);
                    fd[u] = __uint_as_float(rd[8 * v + u]) - fs[u];
                  }
                  uint4 ud, us;
                  ud.x = pack_bf16x2(fd[0], fd[1]);
                  ud.y = pack_bf16x2(fd[2], fd[3]);
                  ud.z = pack_bf16x2(fd[4], fd[5]);
                  ud.w = pack_bf16x2(fd[6], fd[7]);
                  us.x = pack_bf16x2(fs[0], fs[1]);
                  us.y = pack_bf16x2(fs[2], fs[3]);
                  us.z = pack_bf16x2(fs[4], fs[5]);
                  us.w = pack_bf16x2(fs[6], fs[7]);
                  reinterpret_cast<uint4*>(od)[v] = ud;
                  reinterpret_cast<uint4*>(os)[v] = us;
                }
              }
            }
          }
          const int slot = (col_base + s64 * 64) / 64;
          if (row < M && slot < nslots) part[(size_t)row * nslots + slot] = make_float4(dot, nd, ns, 0.f);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        continue;
      }
      const int row = mt * G2_BM + (int)rank * 128 + q * 32 + lane;
      const int chunks = half < 0 ? G2_BN / 32 : G2_BN / 64;
      const int col_base = nt * G2_BN + (half < 0 ? 0 : half * (G2_BN / 2));
      void* Dp = prob ? D1 : D0;
#pragma unroll 1
      for (int c = 0; c < chunks; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * G2_BN + c * 32), r);
        tmem_ld_wait();
        const int col0 = col_base + c * 32;
        if (row < M && col0 < N) {
          if constexpr (OUT_BF16) {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(Dp) + (size_t)row * ldd + col0;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col0 + 8 * v < N) {
                uint4 u;
                u.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                u.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                u.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                u.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                reinterpret_cast<uint4*>(out)[v] = u;
              }
            }
          } else {
            float* out = static_cast<float*>(Dp) + (size_t)row * ldd + col0;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              if (col0 + 4 * v < N) {
                float4 f;
                f.x = __uint_as_float(r[4 * v + 0]);
                f.y = __uint_as_float(r[4 * v + 1]);
                f.z = __uint_as_float(r[4 * v + 2]);
                f.w = __uint_as_float(r[4 * v + 3]);
                reinterpret_cast<float4*>(out)[v] = f;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }
  tc_fence_before();
  cluster_sync_all();   // neither CTA leaves while the other may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

template <typename K>
lcp_status launch_pair(K kernel, int tiles, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       void* d0, void* d1, float4* part, int nslots, int M, int N, int Kd, int ldd, int nprob,
                       cudaStream_t st, const char* what) {
  TC_TRY(set_smem(kernel, G2_SMEM, what));
  const int max_pairs = num_sms() / 2;
  // few tiles: twice as many pairs, each taking one half tile
  const int pairs = 2 * tiles <= max_pairs ? 2 * tiles : (tiles < max_pairs ? tiles : max_pairs);
  return launch_kernel(kernel, dim3(2 * pairs), dim3(GM_THREADS), G2_SMEM, st, 2, true, what, a, b0, b1, d0, d1, part,
                       nslots, M, N, Kd, ldd, nprob);
}

}  // namespace

lcp_status tc_error_gemm(int* site, int reset) { return read_tc_error(site, reset); }

lcp_status launch_calib_gemm_tc(const __nv_bfloat16* X, const __nv_bfloat16* W, const __nv_bfloat16* At,
                                float* Yd, float* Ys, int tokens, int cout, int cin, cudaStream_t st) {
  // A in boxes of 128 rows, B in boxes of 64 rows: each CTA of a pair stages its own half
  CUtensorMap mA, mB0, mB1;
  const int nprob = Ys ? 2 : 1;
  TC_TRY(make_map(&mA, X, cin, tokens, 64, 128, "calib_gemm X"));
  TC_TRY(make_map(&mB0, W, cin, cout, 64, 64, "calib_gemm W"));
  TC_TRY(make_map(&mB1, Ys ? (const void*)At : (const void*)W, cin, cout, 64, 64, "calib_gemm At"));
  const int tiles = cdiv(tokens, G2_BM) * cdiv(cout, G2_BN) * nprob;
  return launch_pair(gemm_pair_tc_kernel<false, false, false, false>, tiles, mA, mB0, mB1, Yd, Ys, nullptr, 0, tokens,
                     cout, cin, cout, nprob, st, "calib_gemm");
}

int calib_loss_slots(int cout) { return cdiv(cout, 64); }

lcp_status launch_calib_loss_tc(const __nv_bfloat16* X, const __nv_bfloat16* W, const __nv_bfloat16* At,
                                __nv_bfloat16* D, __nv_bfloat16* Ys, float* partials, int tokens, int cout, int cin,
                                cudaStream_t st) {
  // A in boxes of 128 rows; B in boxes of 64 rows, CTA 0 of a pair from W, CTA 1 from At
  CUtensorMap mA, mB0, mB1;
  TC_TRY(make_map(&mA, X, cin, tokens, 64, 128, "calib_loss X"));
  TC_TRY(make_map(&mB0, W, cin, cout, 64, 64, "calib_loss W"));
  TC_TRY(make_map(&mB1, At, cin, cout, 64, 64, "calib_loss At"));
  const int tiles = cdiv(tokens, G2_BM) * cdiv(cout, 128);
  return launch_pair(gemm_pair_tc_kernel<false, false, false, true>, tiles, mA, mB0, mB1, D, Ys,
                     reinterpret_cast<float4*>(partials), calib_loss_slots(cout), tokens, cout, cin, cout, 1, st,
                     "calib_loss");
}

lcp_status launch_bwd_gemm_tc(const __nv_bfloat16* G, const __nv_bfloat16* X, __nv_bfloat16* dAt, int tokens,
                              int cout, int cin, cudaStream_t st) {
  CUtensorMap mA, mB;
  TC_TRY(make_map(&mA, G, cout, tokens, 64, 64, "grad_gemm G"));
  TC_TRY(make_map(&mB, X, cin, tokens, 64, 64, "grad_gemm X"));
  const int tiles = cdiv(cout, G2_BM) * cdiv(cin, G2_BN);
  return launch_pair(gemm_pair_tc_kernel<true, true, true, false>, tiles, mA, mB, mB, dAt, nullptr, nullptr, 0, cout,
                     cin, tokens, cin, 1, st, "grad_gemm");
}

}  // namespace lcp
