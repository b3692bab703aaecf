// Dense bf16 products of the LCP step on the tensor cores (tcgen05, CTA pairs):
// the calibration outputs Y_d = X W^T and Y_s = X At^T (PermLLM summary,
// "optimization objective": the dense and sparse outputs), and the weight
// gradient dAt = G^T X of the reverse pass.

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

template <bool A_MN, bool B_MN, bool OUT_BF16>
__global__ void __launch_bounds__(GM_THREADS, 1)
gemm_pair_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, void* __restrict__ D0, void* __restrict__ D1,
                    int M, int N, int K, int ldd, int nprob) {
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

  const int mtiles = cdiv(M, G2_BM), ntiles = cdiv(N, G2_BN);
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
        const CUtensorMap* mb = prob ? &tmB1 : &tmB0;
        // each CTA stages half of the tile's B rows: 128 of a whole tile, 64 of a half
        const int a_row = mt * G2_BM + (int)rank * 128;
        const int b_row = nt * G2_BN + (half < 0 ? (int)rank * 128 : half * 128 + (int)rank * 64);
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
                       void* d0, void* d1, int M, int N, int Kd, int ldd, int nprob, cudaStream_t st,
                       const char* what) {
  TC_TRY(set_smem(kernel, G2_SMEM, what));
  const int max_pairs = num_sms() / 2;
  // few tiles: twice as many pairs, each taking one half tile
  const int pairs = 2 * tiles <= max_pairs ? 2 * tiles : (tiles < max_pairs ? tiles : max_pairs);
  return launch_kernel(kernel, dim3(2 * pairs), dim3(GM_THREADS), G2_SMEM, st, 2, true, what, a, b0, b1, d0, d1, M, N,
                       Kd, ldd, nprob);
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
  return launch_pair(gemm_pair_tc_kernel<false, false, false>, tiles, mA, mB0, mB1, Yd, Ys, tokens, cout, cin,
                     cout, nprob, st, "calib_gemm");
}

lcp_status launch_bwd_gemm_tc(const __nv_bfloat16* G, const __nv_bfloat16* X, __nv_bfloat16* dAt, int tokens,
                              int cout, int cin, cudaStream_t st) {
  CUtensorMap mA, mB;
  TC_TRY(make_map(&mA, G, cout, tokens, 64, 64, "grad_gemm G"));
  TC_TRY(make_map(&mB, X, cin, tokens, 64, 64, "grad_gemm X"));
  const int tiles = cdiv(cout, G2_BM) * cdiv(cin, G2_BN);
  return launch_pair(gemm_pair_tc_kernel<true, true, true>, tiles, mA, mB, mB, dAt, nullptr, cout, cin, tokens, cin,
                     1, st, "grad_gemm");
}

}  // namespace lcp
