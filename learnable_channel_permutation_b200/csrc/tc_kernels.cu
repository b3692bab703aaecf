// Tensor-core (tcgen05 / TMEM / TMA) kernels of the LCP step, sm_100a only.
//
//  gemm_tc_kernel        D = A B^T, bf16 operands, float32 accumulation in TMEM.
//                        Used for the calibration outputs Y_d = X W^T and
//                        Y_s = X At^T (PermLLM summary, "optimization
//                        objective": the dense and sparse outputs) and for the
//                        weight gradient dAt = G^T X of the reverse pass.
//  permute_mask_tc_kernel  W' = W P_B (Method 3), the N:M mask of |W'|
//                        (integration with pruning methods), A = M.W' and
//                        At = A P_B^T, fused per 128-row x BC-column tile.
//  block_bwd_tc_kernel   dA = dAt P_B, dW' = M.dA and the block-diagonal
//                        gradient dP_b = dAt_b^T A_b + W_b^T dW'_b.
//
// Common machinery: operands are staged in shared memory by TMA with the
// 128-byte swizzle; one thread issues tcgen05.mma (kind::f16, bf16 inputs);
// accumulators live in tensor memory and are read back with tcgen05.ld; every
// mbarrier wait is bounded (2 s of %globaltimer): on expiry the kernel records
// the wait site in an error word (lcp_device_error), raises a CTA-wide abort
// flag, and all roles fall through to the teardown that frees tensor memory.

#include <cuda.h>
#include <mutex>

#include "lcp_internal.cuh"

namespace lcp {

__device__ int g_tc_error;  // first failing wait site, 0 if none

namespace {

// ------------------------------------------------------------------ PTX ---

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            int site) {
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitTimeoutNs) {
        *abort_flag = 1;
        atomicCAS(&g_tc_error, 0, site);
        return false;
      }
    }
  }
}
// Waits for the phase with the given parity to complete; false on timeout/abort.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, site);
}

// Drains this CTA's own asynchronous work before exit: ignores the abort flag,
// still bounded by the timeout.
__device__ __noinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, int site) {
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0 && globaltimer() - t0 > kWaitTimeoutNs) {
      atomicCAS(&g_tc_error, 0, site);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most N committed bulk groups still reading shared memory
template <int N> __device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// barrier over `n` threads on named barrier `id` that also ANDs a predicate
__device__ __forceinline__ bool named_and(int id, int n, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(v ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// --- CTA-pair (cluster of 2) helpers ---
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the object at shared::cta address `a` in CTA `rank`
__device__ __forceinline__ uint32_t mapa(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrivals on a barrier addressed through the cluster window (it may live in
// the peer CTA).  No cluster-scope release: the data these arrivals announce
// travels by TMA (counted by complete_tx) or lives in tensor memory (ordered by
// tcgen05.fence), and a cluster-scope release would make the arriving thread
// wait for its own outstanding bulk copies.
__device__ __forceinline__ void mbar_expect_tx_cluster(uint32_t bar_cluster, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(bar_cluster), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on a
// barrier that may live in the peer CTA of the pair
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// Arrives on the barrier at shared::cta offset `bar` of every CTA in `mask`
// once the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, f32 accumulate)
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// Arrives on `bar` once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// NV columns per epilogue thread: 32 (one tcgen05.ld x32) or 16 (x16)
template <int NV> __device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NV]) {
  if constexpr (NV == 32) tmem_ld32(taddr, r);
  else tmem_ld16(taddr, r);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format):
// start>>4 in [0,14), leading byte offset>>4 in [16,30), stride byte
// offset>>4 in [32,46), version 1 at bit 46, layout SWIZZLE_128B (2) at [61,64).
//  K-major:  rows of 128 B (64 bf16 along K), 8-row atoms SBO = 1024 apart.
//  MN-major: 128 B rows hold 64 elements along M/N, one row per K index;
//            8-K-row atoms SBO = 1024 apart; 64-element M/N groups LBO apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: D f32, A and B bf16, majorness, N>>3, M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Writes 8 consecutive bf16 (one 16-byte chunk) of row `row`, chunk `ch`
// (columns 8ch..8ch+7) of a [128 x 64] K-major SW128 region.
__device__ __forceinline__ void st_sw128(uint8_t* region, int row, int ch, uint4 v) {
  *reinterpret_cast<uint4*>(region + row * 128 + ((ch ^ (row & 7)) << 4)) = v;
}

// N:M keep bits of the 32 consecutive values in v (|v| compared as float32;
// equal magnitudes keep the lower column).  Element k ranks ahead of j when
// |v_k| > |v_j|, or the two are equal and k < j; j is kept when fewer than n
// elements rank ahead of it.  Each pair k < j is compared once: k ranks ahead
// of j exactly when |v_k| >= |v_j|, otherwise j ranks ahead of k.
template <int M, int NV>
__device__ __forceinline__ uint32_t nm_bits(const uint32_t (&v)[NV], int n) {
  uint32_t w = 0;
#pragma unroll
  for (int g = 0; g < NV / M; ++g) {
    float a[M];
    int ahead[M];
#pragma unroll
    for (int j = 0; j < M; ++j) { a[j] = fabsf(__uint_as_float(v[g * M + j])); ahead[j] = 0; }
#pragma unroll
    for (int k = 0; k < M; ++k)
#pragma unroll
      for (int j = k + 1; j < M; ++j) {
        const int kj = a[k] >= a[j];
        ahead[j] += kj;
        ahead[k] += 1 - kj;
      }
#pragma unroll
    for (int j = 0; j < M; ++j) w |= (ahead[j] < n ? 1u : 0u) << (g * M + j);
  }
  return w;
}
template <int M>
__device__ __forceinline__ uint32_t nm_word(const uint32_t (&v)[32], int n) {
  return nm_bits<M, 32>(v, n);
}

// --------------------------------------------------------------- GEMM -----
// D[M, N] (row-major, leading dimension ldd) = A B^T for up to two problems
// that share A (D0 = A B0^T, D1 = A B1^T).  A is [M, K] (K-major) or [K, M]
// (A_MN); B is [N, K] (K-major) or [K, N] (B_MN).  128 x 256 output tiles,
// 64-deep k-blocks, a 4-stage TMA ring, two TMEM accumulators so that the
// epilogue of one tile overlaps the main loop of the next.  Persistent CTAs
// walk the tiles with a grid stride.  Warp 0: TMA producer; warp 1: MMA
// issuer and TMEM owner; warps 2-5: epilogue (one TMEM lane quadrant each).

constexpr int GM_BM = 128, GM_BN = 256, GM_BK = 64, GM_STAGES = 4;
constexpr int GM_A_BYTES = GM_BM * GM_BK * 2;
constexpr int GM_B_BYTES = GM_BN * GM_BK * 2;
constexpr int GM_SMEM = GM_STAGES * (GM_A_BYTES + GM_B_BYTES) + 1024 + 256;
constexpr int GM_THREADS = 192;

template <bool A_MN, bool B_MN, bool OUT_BF16>
__global__ void __launch_bounds__(GM_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, void* __restrict__ D0, void* __restrict__ D1,
               int M, int N, int K, int ldd, int nprob) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + GM_STAGES * GM_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + GM_STAGES * GM_B_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 2 * GM_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const uint32_t drain = smem_u32(bars + 2 * GM_STAGES + 4);
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + GM_STAGES + s); };
  auto tfull = [&](int a) { return smem_u32(bars + 2 * GM_STAGES + a); };
  auto tempty = [&](int a) { return smem_u32(bars + 2 * GM_STAGES + 2 + a); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < GM_STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;

  const int mtiles = cdiv(M, GM_BM), ntiles = cdiv(N, GM_BN);
  const int total = mtiles * ntiles * nprob;
  const int nk = cdiv(K, GM_BK);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_par = 0;   // per stage: a load is outstanding / its phase parity
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int mt = tile % mtiles, rest = tile / mtiles;
        const int nt = rest % ntiles, prob = rest / ntiles;
        const CUtensorMap* mb = prob ? &tmB1 : &tmB0;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty(stage), ph ^ 1u, abort_flag, 11)) { ok = false; break; }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (ph << stage);
          mbar_expect_tx(full(stage), GM_A_BYTES + GM_B_BYTES);
          const uint32_t a_dst = smem_u32(sA + stage * GM_A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * GM_B_BYTES);
          if (!A_MN) {
            tma_load_2d(a_dst, &tmA, full(stage), kb * GM_BK, mt * GM_BM);
          } else {
            tma_load_2d(a_dst, &tmA, full(stage), mt * GM_BM, kb * GM_BK);
            tma_load_2d(a_dst + 8192, &tmA, full(stage), mt * GM_BM + 64, kb * GM_BK);
          }
          if (!B_MN) {
            tma_load_2d(b_dst, mb, full(stage), kb * GM_BK, nt * GM_BN);
          } else {
#pragma unroll
            for (int h = 0; h < 4; ++h) tma_load_2d(b_dst + h * 8192, mb, full(stage), nt * GM_BN + 64 * h, kb * GM_BK);
          }
          if (++stage == GM_STAGES) { stage = 0; ph ^= 1u; }
        }
        if (!ok) break;
      }
      // every TMA copy issued into this CTA's shared memory has landed before exit
      for (int st = 0; st < GM_STAGES; ++st)
        if (issued & (1u << st)) mbar_wait_drain(full(st), (issued_par >> st) & 1u, 15);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(GM_BM, GM_BN, A_MN, B_MN);
      int stage = 0, lt = 0;
      uint32_t ph = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++lt) {
        const int acc = lt & 1;
        const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
        if (!mbar_wait(tempty(acc), aph ^ 1u, abort_flag, 12)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * GM_BN);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full(stage), ph, abort_flag, 13)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * GM_A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * GM_B_BYTES);
#pragma unroll
          for (int k16 = 0; k16 < GM_BK / 16; ++k16) {
            const uint64_t ad = A_MN ? sdesc(a0 + k16 * 2048, 8192, 1024) : sdesc(a0 + k16 * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc(b0 + k16 * 2048, 8192, 1024) : sdesc(b0 + k16 * 32, 16, 1024);
            mma_bf16(d, ad, bd, idesc, (kb | k16) != 0);
          }
          mma_commit(empty(stage));
          if (++stage == GM_STAGES) { stage = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(tfull(acc));
      }
      // every MMA this thread issued is complete before the teardown frees TMEM
      mma_commit(drain);
      mbar_wait_drain(drain, 0, 16);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    int lt = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++lt) {
      const int acc = lt & 1;
      const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
      if (!warp_all(mbar_wait(tfull(acc), aph, abort_flag, 14))) break;
      tc_fence_after();
      const int mt = tile % mtiles, rest = tile / mtiles;
      const int nt = rest % ntiles, prob = rest / ntiles;
      const int row = mt * GM_BM + q * 32 + lane;
      void* Dp = prob ? D1 : D0;
#pragma unroll 1
      for (int c = 0; c < GM_BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * GM_BN + c * 32), r);
        tmem_ld_wait();
        const int col0 = nt * GM_BN + c * 32;
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
      if (lane == 0) mbar_arrive(tempty(acc));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------ GEMM, CTA pairs ---
// Same product as gemm_tc_kernel with 256 x 256 output tiles computed by a
// cluster of two CTAs on two SMs (tcgen05 cta_group::2): CTA r stages rows
// [128 r, 128 r + 128) of the tile's A block and of its B block; the leader
// (rank 0) issues M = 256, N = 256 MMAs that read both CTAs' operands, and each
// CTA holds its 128 x 256 half of the accumulator in its own tensor memory.
// Per SM this halves the B bytes per MMA cycle (32 KB of operands per 64-deep
// k-block instead of 48 KB), and six stages fit in shared memory.
constexpr int G2_BM = 256, G2_BN = 256, G2_BK = 64, G2_STAGES = 6;
constexpr int G2_HALF = 128 * G2_BK * 2;               // one 128-row operand half: 16 KB
constexpr int G2_SMEM = G2_STAGES * 2 * G2_HALF + 1024 + 256;

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

  const int mtiles = cdiv(M, G2_BM), ntiles = cdiv(N, G2_BN);
  const int total = mtiles * ntiles * nprob;
  const int nk = cdiv(K, G2_BK);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_par = 0;
      for (int tile = pair; tile < total; tile += npairs) {
        const int mt = tile % mtiles, rest = tile / mtiles;
        const int nt = rest % ntiles, prob = rest / ntiles;
        const CUtensorMap* mb = prob ? &tmB1 : &tmB0;
        const int a_row = mt * G2_BM + (int)rank * 128, b_row = nt * G2_BN + (int)rank * 128;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty(stage), ph ^ 1u, abort_flag, 91)) { ok = false; break; }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (ph << stage);
          const uint32_t fbar = mapa(full(stage), 0);
          mbar_expect_tx_cluster(fbar, 2 * G2_HALF);
          const uint32_t a_dst = smem_u32(sA + stage * G2_HALF);
          const uint32_t b_dst = smem_u32(sB + stage * G2_HALF);
          if (!A_MN) {
            tma_load_2d_pair(a_dst, &tmA, fbar, kb * G2_BK, a_row);
          } else {
            tma_load_2d_pair(a_dst, &tmA, fbar, a_row, kb * G2_BK);
            tma_load_2d_pair(a_dst + 8192, &tmA, fbar, a_row + 64, kb * G2_BK);
          }
          if (!B_MN) {
            tma_load_2d_pair(b_dst, mb, fbar, kb * G2_BK, b_row);
          } else {
            tma_load_2d_pair(b_dst, mb, fbar, b_row, kb * G2_BK);
            tma_load_2d_pair(b_dst + 8192, mb, fbar, b_row + 64, kb * G2_BK);
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
      constexpr uint32_t idesc = idesc_bf16(G2_BM, G2_BN, A_MN, B_MN);
      int stage = 0, lt = 0;
      uint32_t ph = 0;
      for (int tile = pair; tile < total; tile += npairs, ++lt) {
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
    for (int tile = pair; tile < total; tile += npairs, ++lt) {
      const int acc = lt & 1;
      const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
      if (!warp_all(mbar_wait(tfull(acc), aph, abort_flag, 97))) break;
      tc_fence_after();
      const int mt = tile % mtiles, rest = tile / mtiles;
      const int nt = rest % ntiles, prob = rest / ntiles;
      const int row = mt * G2_BM + (int)rank * 128 + q * 32 + lane;
      void* Dp = prob ? D1 : D0;
#pragma unroll 1
      for (int c = 0; c < G2_BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * G2_BN + c * 32), r);
        tmem_ld_wait();
        const int col0 = nt * G2_BN + c * 32;
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

// ------------------------------------------------------- permute + mask ---
// One CTA: rows [r0, r0+128) x channels [t*BC, (t+1)*BC) with BC = max(B, 64),
// in 64-column chunks c:
//   W'_c  = W_tile (P_hi + P_lo)[:, chunk c]          (TMEM, 64 columns)
//   mask bits and A_c = M.W'_c (bf16, shared memory, SW128 K-major)
//   At   += A_c P_hi[:, chunk c]^T                      (TMEM, BC columns)
// P enters through the tile-format images written by the Sinkhorn kernel:
// Pt[t][j][i] = P[i][j] (B operand of the first product, rows j of chunk c),
// Ph[t][i][j] = P[i][j] (B operand of the second product, columns of chunk c).

template <int BC> struct PmCfg {
  static constexpr int NCH = BC / 64;
  static constexpr int W_BYTES = BC * 256;   // 128 rows x BC bf16
  static constexpr int PT_BYTES = BC * 128;  // 64 rows x BC bf16 (NCH regions of 8 KB)
  static constexpr int PH_BYTES = BC * 128;  // BC rows x 64 bf16
  static constexpr int A_BYTES = 16384;      // 128 rows x 64 bf16
  static constexpr uint32_t TMEM_COLS = (64 + BC <= 128) ? 128u : ((64 + BC <= 256) ? 256u : 512u);
  static constexpr int SMEM = W_BYTES + 2 * PT_BYTES + PH_BYTES + A_BYTES + 1024 + 128;
};

template <int BC, int MGROUP>
__global__ void __launch_bounds__(128)
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
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const uint32_t bar_load = smem_u32(bars + 0), bar_mma1 = smem_u32(bars + 1), bar_mma2 = smem_u32(bars + 2);
  const uint32_t bar_drain = smem_u32(bars + 3);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r0 = blockIdx.x * 128, t = blockIdx.y, col0 = t * BC;
  if (tid == 0) {
    mbar_init(bar_load, 1);
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
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int row = warp * 32 + lane, grow = r0 + row;
  const int words = cin / 32;
  constexpr uint32_t idesc1 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t idesc2 = idesc_bf16(128, BC, false, false);

  bool ok = true;
  int pending_load = -1;   // thread 0: parity of a load not yet seen complete
  for (int c = 0; c < C::NCH && ok; ++c) {
    if (tid == 0) {
      bool go = (c == 0) || mbar_wait(bar_mma2, (uint32_t)(c - 1) & 1u, abort_flag, 21);
      if (go) {
        pending_load = c & 1;
        mbar_expect_tx(bar_load, (c == 0 ? C::W_BYTES : 0) + 2 * C::PT_BYTES + C::PH_BYTES);
        if (c == 0)
          for (int kc = 0; kc < C::NCH; ++kc)
            tma_load_2d(smem_u32(sW + kc * 16384), &tmW, bar_load, col0 + kc * 64, r0);
        for (int kc = 0; kc < C::NCH; ++kc) {
          tma_load_2d(smem_u32(sPth + kc * 8192), &tmPth, bar_load, kc * 64, col0 + c * 64);
          tma_load_2d(smem_u32(sPtl + kc * 8192), &tmPtl, bar_load, kc * 64, col0 + c * 64);
        }
        tma_load_2d(smem_u32(sPh), &tmPh, bar_load, c * 64, col0);
        go = mbar_wait(bar_load, (uint32_t)c & 1u, abort_flag, 22);
        if (go) pending_load = -1;
      }
      if (!go) *abort_flag = 1;
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
      }
    }
    ok = __syncthreads_and(mbar_wait(bar_mma1, (uint32_t)c & 1u, abort_flag, 23));
    if (!ok) break;
    tc_fence_after();
    uint32_t v0[32], v1[32];
    tmem_ld32(tmem + lane_off + 0, v0);
    tmem_ld32(tmem + lane_off + 32, v1);
    tmem_ld_wait();
    const uint32_t w0 = nm_word<MGROUP>(v0, n), w1 = nm_word<MGROUP>(v1, n);
    if (grow < cout) {
      const int wi = (col0 + c * 64) / 32;
      mask[(size_t)grow * words + wi] = w0;
      mask[(size_t)grow * words + wi + 1] = w1;
      if (Wp_out) {
        float4* o = reinterpret_cast<float4*>(Wp_out + (size_t)grow * cin + col0 + c * 64);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          o[q] = make_float4(__uint_as_float(v0[4 * q]), __uint_as_float(v0[4 * q + 1]),
                             __uint_as_float(v0[4 * q + 2]), __uint_as_float(v0[4 * q + 3]));
#pragma unroll
        for (int q = 0; q < 8; ++q)
          o[8 + q] = make_float4(__uint_as_float(v1[4 * q]), __uint_as_float(v1[4 * q + 1]),
                                 __uint_as_float(v1[4 * q + 2]), __uint_as_float(v1[4 * q + 3]));
      }
    }
    // A_c = M . W'_c as bf16 into the K-major SW128 operand tile
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint32_t* v = ch < 4 ? v0 : v1;
      const uint32_t w = ch < 4 ? w0 : w1;
      const int b0 = (ch & 3) * 8;
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = ((w >> (b0 + e)) & 1u) ? __uint_as_float(v[b0 + e]) : 0.f;
      st_sw128(sA, row, ch, make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                       pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k16 = 0; k16 < 4; ++k16)
        mma_bf16(tmem + 64, sdesc(smem_u32(sA) + k16 * 32, 16, 1024), sdesc(smem_u32(sPh) + k16 * 32, 16, 1024),
                 idesc2, (c | k16) != 0);
      mma_commit(bar_mma2);
    }
  }
  if (ok) ok = __syncthreads_and(mbar_wait(bar_mma2, (uint32_t)(C::NCH - 1) & 1u, abort_flag, 24));
  if (ok) {
    tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < BC / 32; ++cc) {
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
    if (pending_load >= 0) mbar_wait_drain(bar_load, (uint32_t)pending_load, 25);
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
// BC = 64 (B = 32 or 64).  Persistent CTAs walk a flat list of (channel tile,
// row tile) pairs.  Warp 0 streams each tile's W block together with its P
// images into a 3-stage ring; warp 1 issues W' = W (P_hi + P_lo) into one of
// two TMEM buffers and, once the epilogue has written A = M.W' to shared
// memory, At = A P_hi into the same buffer; warps 2-9 (two per TMEM lane
// quadrant, 32 columns each) compute the mask, write A, and copy At out
// through a swizzled staging tile with TMA stores.
template <int NSL> struct PwCfg {
  static constexpr int STAGES = 3;
  static constexpr int W_BYTES = 16384;                 // 128 rows x 64 bf16
  static constexpr int IMG_BYTES = 8192;                // 64 x 64 bf16
  static constexpr int STAGE = W_BYTES + 3 * IMG_BYTES; // W | Pt_hi | Pt_lo | P_hi
  static constexpr int A_BYTES = 16384;
  static constexpr int SMEM = STAGES * STAGE + 2 * A_BYTES + 2 * A_BYTES + 1024 + 256;
  static constexpr int EPI_WARPS = 4 * NSL;              // NSL column slices per TMEM lane quadrant
  static constexpr int COLS = 64 / NSL;                  // columns per epilogue thread
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int EPI = 32 * EPI_WARPS;
};

template <int MGROUP, int NSL>
__global__ void __launch_bounds__(PwCfg<NSL>::THREADS, 1)
permute_mask_ws_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmPth,
                       const __grid_constant__ CUtensorMap tmPtl, const __grid_constant__ CUtensorMap tmPh,
                       const __grid_constant__ CUtensorMap tmAt, uint32_t* __restrict__ mask,
                       float* __restrict__ Wp_out, int cout, int cin, int n) {
  using C = PwCfg<NSL>;
  constexpr int NV = C::COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sStage = smem;
  uint8_t* sA = smem + C::STAGES * C::STAGE;          // 2 buffers
  uint8_t* sO = sA + 2 * C::A_BYTES;                  // 2 staging tiles for At
  uint64_t* bars = reinterpret_cast<uint64_t*>(sO + 2 * C::A_BYTES);
  // bars: full[3] empty[3] wf[2] af[2] atf[2] tmw[2] tma[2] drain
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = 3, WF = 6, AF = 8, ATF = 10, TMW = 12, TMA = 14, DRAIN = 16;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nrt = cdiv(cout, 128), ntc = cin / 64;
  const int total = nrt * ntc;
  const int nloc = (int)blockIdx.x < total ? cdiv(total - (int)blockIdx.x, (int)gridDim.x) : 0;
  const int words = cin / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) { mbar_init(bar(FULL + i), 1); mbar_init(bar(EMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(WF + i), 1);
      mbar_init(bar(AF + i), C::EPI_WARPS);
      mbar_init(bar(ATF + i), 1);
      mbar_init(bar(TMW + i), C::EPI_WARPS);
      mbar_init(bar(TMA + i), C::EPI_WARPS);
    }
    mbar_init(bar(DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  auto tile_of = [&](int k, int& t, int& rt) {
    const int idx = (int)blockIdx.x + k * (int)gridDim.x;
    t = idx / nrt;
    rt = idx % nrt;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, par = 0;   // per stage: outstanding load and its parity
      for (int k = 0; k < nloc; ++k) {
        const int st = k % C::STAGES;
        const uint32_t use = (uint32_t)(k / C::STAGES) & 1u;
        if (!mbar_wait(bar(EMPTY + st), use ^ 1u, abort_flag, 61)) break;
        int t, rt;
        tile_of(k, t, rt);
        uint8_t* sg = sStage + st * C::STAGE;
        mbar_expect_tx(bar(FULL + st), C::STAGE);
        tma_load_2d(smem_u32(sg), &tmW, bar(FULL + st), t * 64, rt * 128);
        tma_load_2d(smem_u32(sg + C::W_BYTES), &tmPth, bar(FULL + st), 0, t * 64);
        tma_load_2d(smem_u32(sg + C::W_BYTES + C::IMG_BYTES), &tmPtl, bar(FULL + st), 0, t * 64);
        tma_load_2d(smem_u32(sg + C::W_BYTES + 2 * C::IMG_BYTES), &tmPh, bar(FULL + st), 0, t * 64);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (use << st);
      }
      for (int st = 0; st < C::STAGES; ++st)
        if (issued & (1u << st)) mbar_wait_drain(bar(FULL + st), (par >> st) & 1u, 62);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);
      // W' = W (P_hi + P_lo) of local tile k into the W' half of TMEM buffer k & 1
      auto mma1 = [&](int k) -> bool {
        const int st = k % C::STAGES, a = k & 1;
        const uint32_t use = (uint32_t)(k / C::STAGES) & 1u, ua = (uint32_t)(k >> 1) & 1u;
        if (!mbar_wait(bar(FULL + st), use, abort_flag, 63)) return false;
        if (!mbar_wait(bar(TMW + a), ua ^ 1u, abort_flag, 64)) return false;   // W' of tile k - 2 read
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
        const uint32_t dW = tmem + a * 128;
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint64_t ad = sdesc(sg + k16 * 32, 16, 1024);
          mma_bf16(dW, ad, sdesc(sg + C::W_BYTES + k16 * 32, 16, 1024), idesc, k16 != 0);
          mma_bf16(dW, ad, sdesc(sg + C::W_BYTES + C::IMG_BYTES + k16 * 32, 16, 1024), idesc, true);
        }
        mma_commit(bar(WF + a));
        return true;
      };
      // the next tile's first product is issued before waiting for this tile's
      // epilogue, so the tensor core and the epilogue warps overlap
      bool ok = nloc == 0 || mma1(0);
      for (int k = 0; k < nloc && ok; ++k) {
        const int st = k % C::STAGES, a = k & 1;
        const uint32_t ua = (uint32_t)(k >> 1) & 1u;
        if (k + 1 < nloc && !mma1(k + 1)) break;
        if (!mbar_wait(bar(AF + a), ua, abort_flag, 65)) break;        // A of tile k in shared memory
        if (!mbar_wait(bar(TMA + a), ua ^ 1u, abort_flag, 69)) break;  // At of tile k - 2 read
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
        const uint32_t sa = smem_u32(sA + a * C::A_BYTES);
        const uint32_t dAt = tmem + a * 128 + 64;
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(dAt, sdesc(sa + k16 * 32, 16, 1024), sdesc(sg + C::W_BYTES + 2 * C::IMG_BYTES + k16 * 32, 16, 1024),
                   idesc, k16 != 0);
        mma_commit(bar(ATF + a));
        mma_commit(bar(EMPTY + st));
      }
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0, 66);
    }
    __syncwarp();
  } else {
    // Software-pipelined epilogue: in step k the warps first turn W' of tile k
    // into the mask and A (so the MMA warp can start At of tile k), then copy
    // out At of tile k - 1, whose product ran meanwhile.
    const int e = warp - 2, q = warp & 3, h = e >> 2;   // h: column slice of NV columns
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool leader = (e == 0 && lane == 0);
    for (int k = 0; k <= nloc; ++k) {
      if (k < nloc) {
        const int a = k & 1;
        const uint32_t ua = (uint32_t)(k >> 1) & 1u;
        int t, rt;
        tile_of(k, t, rt);
        const int grow = rt * 128 + row;
        if (!named_and(1, C::EPI, mbar_wait(bar(WF + a), ua, abort_flag, 67))) break;
        tc_fence_after();
        uint32_t v[NV];
        tmem_ld_cols<NV>(tmem + lane_off + a * 128 + h * NV, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(TMW + a));
        const uint32_t w = nm_bits<MGROUP, NV>(v, n);
        if (grow < cout) {
          if constexpr (NV == 32) {
            mask[(size_t)grow * words + 2 * t + h] = w;
          } else {
            reinterpret_cast<uint16_t*>(mask)[((size_t)grow * words + 2 * t) * 2 + h] = (uint16_t)w;
          }
          if (Wp_out) {
            float4* o = reinterpret_cast<float4*>(Wp_out + (size_t)grow * cin + t * 64 + h * NV);
#pragma unroll
            for (int qq = 0; qq < NV / 4; ++qq)
              o[qq] = make_float4(__uint_as_float(v[4 * qq]), __uint_as_float(v[4 * qq + 1]),
                                  __uint_as_float(v[4 * qq + 2]), __uint_as_float(v[4 * qq + 3]));
          }
        }
        uint8_t* sa = sA + a * C::A_BYTES;
#pragma unroll
        for (int c8 = 0; c8 < NV / 8; ++c8) {
          float f[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) f[x] = ((w >> (8 * c8 + x)) & 1u) ? __uint_as_float(v[8 * c8 + x]) : 0.f;
          st_sw128(sa, row, h * (NV / 8) + c8, make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(AF + a));
      }
      if (k > 0) {
        const int kp = k - 1, a = kp & 1;
        const uint32_t ua = (uint32_t)(kp >> 1) & 1u;
        int t, rt;
        tile_of(kp, t, rt);
        const bool got = mbar_wait(bar(ATF + a), ua, abort_flag, 68);
        // the staging tile of two tiles ago must have been read out by its TMA store
        if (leader) bulk_wait_read<1>();
        if (!named_and(1, C::EPI, got)) break;
        tc_fence_after();
        uint32_t v[NV];
        tmem_ld_cols<NV>(tmem + lane_off + a * 128 + 64 + h * NV, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(TMA + a));
        uint8_t* so = sO + a * C::A_BYTES;
#pragma unroll
        for (int c8 = 0; c8 < NV / 8; ++c8)
          st_sw128(so, row, h * (NV / 8) + c8,
                   make_uint4(pack_bf16x2(__uint_as_float(v[8 * c8 + 0]), __uint_as_float(v[8 * c8 + 1])),
                              pack_bf16x2(__uint_as_float(v[8 * c8 + 2]), __uint_as_float(v[8 * c8 + 3])),
                              pack_bf16x2(__uint_as_float(v[8 * c8 + 4]), __uint_as_float(v[8 * c8 + 5])),
                              pack_bf16x2(__uint_as_float(v[8 * c8 + 6]), __uint_as_float(v[8 * c8 + 7]))));
        fence_async_smem();
        named_sync(1, C::EPI);
        if (leader) {
          tma_store_2d(&tmAt, smem_u32(so), t * 64, rt * 128);
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ----------------------------------------- permute + mask, row-streamed ---
// For BC <= 128 the P images of the CTA's channel tile stay resident and the
// CTA walks the row tiles rt = blockIdx.y, blockIdx.y + gridDim.y, ...; the W
// tile of the next-but-one row tile streams in (two buffers) while the current
// one is processed, so that HBM reads stay in flight across the whole launch.
template <int BC> struct Pm2Cfg {
  static constexpr int NCH = BC / 64;
  static constexpr int W_BYTES = BC * 256;        // 128 rows x BC
  static constexpr int PT_BYTES = BC * BC * 2;    // every chunk of one transposed image
  static constexpr int PH_BYTES = BC * BC * 2;
  static constexpr int A_BYTES = 16384;
  static constexpr uint32_t TMEM_COLS = (64 + BC <= 128) ? 128u : 256u;
  static constexpr int SMEM = 2 * W_BYTES + 2 * PT_BYTES + PH_BYTES + A_BYTES + 1024 + 128;
  static constexpr int CTAS_PER_SM = BC == 64 ? 3 : 1;
};

template <int BC, int MGROUP>
__global__ void __launch_bounds__(128)
permute_mask_tc2_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmPth,
                        const __grid_constant__ CUtensorMap tmPtl, const __grid_constant__ CUtensorMap tmPh,
                        uint32_t* __restrict__ mask, __nv_bfloat16* __restrict__ At,
                        float* __restrict__ Wp_out, int cout, int cin, int n) {
  using C = Pm2Cfg<BC>;
  constexpr int NCH = C::NCH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW0 = smem;
  uint8_t* sPth = sW0 + 2 * C::W_BYTES;
  uint8_t* sPtl = sPth + C::PT_BYTES;
  uint8_t* sPh = sPtl + C::PT_BYTES;
  uint8_t* sA = sPh + C::PH_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sA + C::A_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const uint32_t bar_full0 = smem_u32(bars + 0);          // +8 for buffer 1
  const uint32_t bar_mma1 = smem_u32(bars + 2), bar_mma2 = smem_u32(bars + 3), bar_drain = smem_u32(bars + 4);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t = blockIdx.x, col0 = t * BC;
  const int nrt = cdiv(cout, 128), first = blockIdx.y, step = gridDim.y;
  const int nloc = first < nrt ? cdiv(nrt - first, step) : 0;
  if (tid == 0) {
    mbar_init(bar_full0, 1);
    mbar_init(bar_full0 + 8, 1);
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
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int row = warp * 32 + lane;
  const int words = cin / 32;
  constexpr uint32_t idesc1 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t idesc2 = idesc_bf16(128, BC, false, false);

  auto load_w = [&](int k, int b) {   // thread 0: W rows of local tile k into buffer b
    const int r0 = (first + k * step) * 128;
    for (int kc = 0; kc < NCH; ++kc)
      tma_load_2d(smem_u32(sW0 + b * C::W_BYTES + kc * 16384), &tmW, bar_full0 + 8 * b, col0 + kc * 64, r0);
  };
  int issued = 0;   // thread 0: local tiles whose W load has been issued
  if (tid == 0 && nloc > 0) {
    mbar_expect_tx(bar_full0, C::W_BYTES + 2 * C::PT_BYTES + C::PH_BYTES);
    for (int c = 0; c < NCH; ++c) {
      for (int kc = 0; kc < NCH; ++kc) {
        tma_load_2d(smem_u32(sPth + (c * NCH + kc) * 8192), &tmPth, bar_full0, kc * 64, col0 + c * 64);
        tma_load_2d(smem_u32(sPtl + (c * NCH + kc) * 8192), &tmPtl, bar_full0, kc * 64, col0 + c * 64);
      }
      tma_load_2d(smem_u32(sPh + c * BC * 128), &tmPh, bar_full0, c * 64, col0);
    }
    load_w(0, 0);
    issued = 1;
    if (nloc > 1) {
      mbar_expect_tx(bar_full0 + 8, C::W_BYTES);
      load_w(1, 1);
      issued = 2;
    }
  }

  bool ok = true;
  uint32_t n1 = 0, n2 = 0;   // completed phases of bar_mma1 / bar_mma2
  int consumed = 0;          // thread 0: local tiles whose W load was seen complete
  for (int k = 0; k < nloc && ok; ++k) {
    const int b = k & 1;
    const int grow = (first + k * step) * 128 + row;
    const uint8_t* sW = sW0 + b * C::W_BYTES;
    if (tid == 0) {
      if (mbar_wait(bar_full0 + 8 * b, (uint32_t)(k >> 1) & 1u, abort_flag, 41)) consumed = k + 1;
      else *abort_flag = 1;
    }
    for (int c = 0; c < NCH; ++c) {
      if (tid == 0 && !*abort_flag) {
        tc_fence_after();
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          const uint8_t* sB = (pass ? sPtl : sPth) + c * NCH * 8192;
          for (int kc = 0; kc < NCH; ++kc)
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(tmem, sdesc(smem_u32(sW + kc * 16384) + k16 * 32, 16, 1024),
                       sdesc(smem_u32(sB + kc * 8192) + k16 * 32, 16, 1024), idesc1, (pass | kc | k16) != 0);
        }
        mma_commit(bar_mma1);
      }
      ok = __syncthreads_and(mbar_wait(bar_mma1, n1 & 1u, abort_flag, 42));
      ++n1;
      if (!ok) break;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(tmem + lane_off + 0, v0);
      tmem_ld32(tmem + lane_off + 32, v1);
      tmem_ld_wait();
      const uint32_t w0 = nm_word<MGROUP>(v0, n), w1 = nm_word<MGROUP>(v1, n);
      if (grow < cout) {
        const int wi = (col0 + c * 64) / 32;
        *reinterpret_cast<uint2*>(mask + (size_t)grow * words + wi) = make_uint2(w0, w1);
        if (Wp_out) {
          float4* o = reinterpret_cast<float4*>(Wp_out + (size_t)grow * cin + col0 + c * 64);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            o[q] = make_float4(__uint_as_float(v0[4 * q]), __uint_as_float(v0[4 * q + 1]),
                               __uint_as_float(v0[4 * q + 2]), __uint_as_float(v0[4 * q + 3]));
#pragma unroll
          for (int q = 0; q < 8; ++q)
            o[8 + q] = make_float4(__uint_as_float(v1[4 * q]), __uint_as_float(v1[4 * q + 1]),
                                   __uint_as_float(v1[4 * q + 2]), __uint_as_float(v1[4 * q + 3]));
        }
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t* v = ch < 4 ? v0 : v1;
        const uint32_t w = ch < 4 ? w0 : w1;
        const int b0 = (ch & 3) * 8;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = ((w >> (b0 + e)) & 1u) ? __uint_as_float(v[b0 + e]) : 0.f;
        st_sw128(sA, row, ch, make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                         pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(tmem + 64, sdesc(smem_u32(sA) + k16 * 32, 16, 1024),
                   sdesc(smem_u32(sPh + c * BC * 128) + k16 * 32, 16, 1024), idesc2, (c | k16) != 0);
        mma_commit(bar_mma2);
      }
    }
    if (!ok) break;
    n2 += NCH;
    // the W buffer of this tile is free once its MMAs are done: stream tile k + 2 into it
    if (tid == 0 && k + 2 < nloc) {
      if (mbar_wait(bar_mma2, (n2 - 1) & 1u, abort_flag, 43)) {
        mbar_expect_tx(bar_full0 + 8 * b, C::W_BYTES);
        load_w(k + 2, b);
        issued = k + 3;
      } else {
        *abort_flag = 1;
      }
    }
    ok = __syncthreads_and(mbar_wait(bar_mma2, (n2 - 1) & 1u, abort_flag, 44));
    if (!ok) break;
    tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < BC / 32; ++cc) {
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
    tc_fence_before();
    __syncthreads();   // the next tile's MMAs overwrite the accumulators just read
  }
  if (tid == 0) {
    for (int kk = consumed; kk < issued; ++kk)
      mbar_wait_drain(bar_full0 + 8 * (kk & 1), (uint32_t)(kk >> 1) & 1u, 45);
    mma_commit(bar_drain);
    mbar_wait_drain(bar_drain, 0, 46);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------- block backward, warp-specialised ---
// BC = 64 (B = 32 or 64).  One CTA per (channel tile, row segment).  Warp 0
// streams the (dAt, W) tiles of each 128-row chunk into a 3-stage ring; warp 1
// issues W' = W (P_hi + P_lo) and dA = dAt P_hi into one of two TMEM buffers,
// then, once the epilogue has written A = M.W' and dW' = M.dA, the stacked
// dP product; warps 2-9 (two per TMEM lane quadrant, 32 columns each) turn
// W', dA and the mask into the bf16 operands.  The dP accumulator stays in
// TMEM for the whole segment and is written once at the end.
template <int NSL> struct BwCfg {
  static constexpr int STAGES = 3;
  static constexpr int T_BYTES = 16384;                  // 128 rows x 64 bf16
  static constexpr int STAGE = 2 * T_BYTES;              // dAt | W (adjacent: stacked A operand)
  static constexpr int IMG_BYTES = 8192;
  static constexpr int SMEM = STAGES * STAGE + 2 * IMG_BYTES + 2 * (2 * T_BYTES) + 1024 + 256;
  static constexpr int EPI_WARPS = 4 * NSL;              // NSL column slices per TMEM lane quadrant
  static constexpr int COLS = 64 / NSL;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
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
  // bars: full[3] empty[3] wd[2] abf[2] abe[2] dpf drain img
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = 3, WD = 6, ABF = 8, ABE = 10, DPF = 12, DRAIN = 13, IMG = 14;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x, sidx = blockIdx.y, col0 = t * 64;
  const int rbeg = sidx * rows_per_split;
  const int rend = min(cout, rbeg + rows_per_split);
  const int nchunk = cdiv(rend - rbeg, 128);
  const int words = cin / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) { mbar_init(bar(FULL + i), 1); mbar_init(bar(EMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(WD + i), 1);
      mbar_init(bar(ABF + i), C::EPI_WARPS);
      mbar_init(bar(ABE + i), 1);
    }
    mbar_init(bar(DPF), 1);
    mbar_init(bar(DRAIN), 1);
    mbar_init(bar(IMG), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  const uint32_t tDP = tmem + 256;

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
      constexpr uint32_t idesc_dp = idesc_bf16(128, 128, true, true);
      bool ok = nchunk == 0 || mbar_wait(bar(IMG), 0, abort_flag, 74);
      // W' = W (P_hi + P_lo) and dA = dAt P_hi of chunk c into TMEM buffer c & 1
      auto mma1 = [&](int c) -> bool {
        const int st = c % C::STAGES, a = c & 1;
        const uint32_t use = (uint32_t)(c / C::STAGES) & 1u, ua = (uint32_t)(c >> 1) & 1u;
        if (!mbar_wait(bar(FULL + st), use, abort_flag, 75)) return false;
        // the epilogue has read buffer a of chunk c - 2 (it arrives on ABF after its loads)
        if (c >= 2 && !mbar_wait(bar(ABF + a), ua ^ 1u, abort_flag, 76)) return false;
        tc_fence_after();
        const uint32_t sg = smem_u32(sStage + st * C::STAGE);
        const uint32_t tW = tmem + a * 128, tDA = tmem + a * 128 + 64;
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint64_t wdesc = sdesc(sg + C::T_BYTES + k16 * 32, 16, 1024);
          mma_bf16(tW, wdesc, sdesc(smem_u32(sPth) + k16 * 32, 16, 1024), idesc_n, k16 != 0);
          mma_bf16(tW, wdesc, sdesc(smem_u32(sPtl) + k16 * 32, 16, 1024), idesc_n, true);
          mma_bf16(tDA, sdesc(sg + k16 * 32, 16, 1024), sdesc(smem_u32(sPth) + k16 * 32, 16, 1024), idesc_n,
                   k16 != 0);
        }
        mma_commit(bar(WD + a));
        return true;
      };
      if (ok && nchunk > 0) ok = mma1(0);
      for (int c = 0; c < nchunk && ok; ++c) {
        const int st = c % C::STAGES, a = c & 1;
        const uint32_t ua = (uint32_t)(c >> 1) & 1u;
        if (c + 1 < nchunk && !mma1(c + 1)) break;
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
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0, 78);
    }
    __syncwarp();
  } else {
    const int e = warp - 2, q = warp & 3, h = e >> 2;   // h: column slice of NV columns
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
      uint32_t wv[NV], dv[NV];
      tmem_ld_cols<NV>(tmem + lane_off + a * 128 + h * NV, wv);
      tmem_ld_cols<NV>(tmem + lane_off + a * 128 + 64 + h * NV, dv);
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
          fa[x] = keep ? __uint_as_float(wv[8 * c8 + x]) : 0.f;
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
      float* scratch = reinterpret_cast<float*>(sAB);   // 64 x 64 floats; every MMA is done
      if (row >= 64) {
#pragma unroll
        for (int x = 0; x < NV; ++x) scratch[(row - 64) * 64 + h * NV + x] = __uint_as_float(v[x]);
      }
      named_sync(1, C::EPI);
      if (row < 64) {
        const int nb = cin / B;
        float* dPs = dP + (size_t)sidx * nb * B * B;
        const float* add = scratch + row * 64 + h * NV;
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

// ------------------------------------------------------- block backward ---
// One CTA: channel tile t (BC columns) x a segment of C_out rows, in chunks of
// 128 rows o:
//   W'  = W_tile (P_hi + P_lo)          dA = dAt_tile P_hi          (TMEM)
//   A = M.W', dW' = M.dA  -> bf16 operand tiles in shared memory
//   dP += dAt_tile^T A + W_tile^T dW'   (contraction over the 128 rows: the
//         row-major tiles are read as MN-major operands)
// For BC = 64 the two products share one M = 128 MMA: the A operand stacks the
// dAt and W tiles (adjacent, LBO = 16 KB) and the B operand stacks A and dW',
// so the wanted sums are the two diagonal 64 x 64 quadrants of the result.
// The partial dP of each segment goes to dP[s] (summed by the Sinkhorn reverse).

template <int BC> struct BbCfg {
  static constexpr int NCH = BC / 64;
  static constexpr int T_BYTES = BC * 256;   // 128 rows x BC bf16
  static constexpr int P_BYTES = BC * BC * 2;
  static constexpr uint32_t TMEM_COLS = (2 * BC + 128 <= 256) ? 256u : 512u;
  // sDAt | sW | sPth | sPtl | sAb | sdWb
  static constexpr int SMEM = 4 * T_BYTES + 2 * P_BYTES + 1024 + 128;
};

template <int BC, int B>
__global__ void __launch_bounds__(128)
block_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmDAt,
                    const __grid_constant__ CUtensorMap tmPth, const __grid_constant__ CUtensorMap tmPtl,
                    const uint32_t* __restrict__ mask, float* __restrict__ dP, int cout, int cin,
                    int rows_per_split) {
  using C = BbCfg<BC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sDAt = smem;
  uint8_t* sW = sDAt + C::T_BYTES;
  uint8_t* sPth = sW + C::T_BYTES;
  uint8_t* sPtl = sPth + C::P_BYTES;
  uint8_t* sAb = sPtl + C::P_BYTES;
  uint8_t* sdWb = sAb + C::T_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdWb + C::T_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const uint32_t bar_load = smem_u32(bars + 0), bar_mma1 = smem_u32(bars + 1), bar_mma2 = smem_u32(bars + 2);
  const uint32_t bar_drain = smem_u32(bars + 3);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t = blockIdx.x, s = blockIdx.y, col0 = t * BC;
  const int rbeg = s * rows_per_split;
  const int rend = min(cout, rbeg + rows_per_split);
  const int nchunk = cdiv(rend - rbeg, 128);
  if (tid == 0) {
    mbar_init(bar_load, 1);
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
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int row = warp * 32 + lane;
  const int words = cin / 32;
  int pending_load = -1;
  constexpr uint32_t idesc_n = idesc_bf16(128, BC, false, false);
  constexpr uint32_t idesc_dp = idesc_bf16(128, 128, true, true);
  const uint32_t tW = tmem, tDA = tmem + BC, tDP = tmem + 2 * BC;

  bool ok = true;
  for (int ch = 0; ch < nchunk && ok; ++ch) {
    const int r0 = rbeg + ch * 128;
    if (tid == 0) {
      bool go = (ch == 0) || mbar_wait(bar_mma2, (uint32_t)(ch - 1) & 1u, abort_flag, 31);
      if (go) {
        pending_load = ch & 1;
        mbar_expect_tx(bar_load, 2 * C::T_BYTES + (ch == 0 ? 2 * C::P_BYTES : 0));
        for (int kc = 0; kc < C::NCH; ++kc) {
          tma_load_2d(smem_u32(sW + kc * 16384), &tmW, bar_load, col0 + kc * 64, r0);
          tma_load_2d(smem_u32(sDAt + kc * 16384), &tmDAt, bar_load, col0 + kc * 64, r0);
        }
        if (ch == 0)
          for (int kc = 0; kc < C::NCH; ++kc) {
            tma_load_2d(smem_u32(sPth + kc * BC * 128), &tmPth, bar_load, kc * 64, col0);
            tma_load_2d(smem_u32(sPtl + kc * BC * 128), &tmPtl, bar_load, kc * 64, col0);
          }
        go = mbar_wait(bar_load, (uint32_t)ch & 1u, abort_flag, 32);
        if (go) pending_load = -1;
      }
      if (!go) *abort_flag = 1;
      if (go) {
        tc_fence_after();
        for (int kc = 0; kc < C::NCH; ++kc)
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t a = sdesc(smem_u32(sW + kc * 16384) + k16 * 32, 16, 1024);
            mma_bf16(tW, a, sdesc(smem_u32(sPth + kc * BC * 128) + k16 * 32, 16, 1024), idesc_n,
                     (kc | k16) != 0);
            mma_bf16(tW, a, sdesc(smem_u32(sPtl + kc * BC * 128) + k16 * 32, 16, 1024), idesc_n, true);
            mma_bf16(tDA, sdesc(smem_u32(sDAt + kc * 16384) + k16 * 32, 16, 1024),
                     sdesc(smem_u32(sPth + kc * BC * 128) + k16 * 32, 16, 1024), idesc_n, (kc | k16) != 0);
          }
        mma_commit(bar_mma1);
      }
    }
    ok = __syncthreads_and(mbar_wait(bar_mma1, (uint32_t)ch & 1u, abort_flag, 33));
    if (!ok) break;
    tc_fence_after();
    const int grow = r0 + row;
    const bool valid = grow < rend;
#pragma unroll 1
    for (int cc = 0; cc < BC / 32; ++cc) {
      uint32_t wv[32], dv[32];
      tmem_ld32(tW + lane_off + cc * 32, wv);
      tmem_ld32(tDA + lane_off + cc * 32, dv);
      tmem_ld_wait();
      const uint32_t bits = valid ? __ldg(mask + (size_t)grow * words + col0 / 32 + cc) : 0u;
      uint8_t* rA = sAb + (cc / 2) * 16384;
      uint8_t* rD = sdWb + (cc / 2) * 16384;
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
      if constexpr (BC == 64) {
        // stacked: A = [dAt | W] (M = 128), B = [A | dW'] (N = 128), LBO = 16 KB
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_bf16(tDP, sdesc(smem_u32(sDAt) + k16 * 2048, 16384, 1024),
                   sdesc(smem_u32(sAb) + k16 * 2048, 16384, 1024), idesc_dp, (ch | k16) != 0);
      } else {
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_bf16(tDP, sdesc(smem_u32(sDAt) + k16 * 2048, 16384, 1024),
                   sdesc(smem_u32(sAb) + k16 * 2048, 16384, 1024), idesc_dp, (ch | k16) != 0);
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_bf16(tDP, sdesc(smem_u32(sW) + k16 * 2048, 16384, 1024),
                   sdesc(smem_u32(sdWb) + k16 * 2048, 16384, 1024), idesc_dp, true);
      }
      mma_commit(bar_mma2);
    }
  }
  if (ok && nchunk > 0) ok = __syncthreads_and(mbar_wait(bar_mma2, (uint32_t)(nchunk - 1) & 1u, abort_flag, 34));
  const int nb = cin / B;
  float* dPs = dP + (size_t)s * nb * B * B;
  if (ok) {
    tc_fence_after();
    if constexpr (BC == 64) {
      // rows 0..63: dAt^T A in columns 0..63; rows 64..127: W^T dW' in columns 64..127
      float* scratch = reinterpret_cast<float*>(sAb);   // 64 x 64 floats (free: last MMA done)
      uint32_t r0v[32], r1v[32];
      const uint32_t cbase = (row < 64) ? 0u : 64u;
      tmem_ld32(tDP + lane_off + cbase, r0v);
      tmem_ld32(tDP + lane_off + cbase + 32, r1v);
      tmem_ld_wait();
      if (row >= 64) {
        float* dst = scratch + (row - 64) * 64;
#pragma unroll
        for (int e = 0; e < 32; ++e) { dst[e] = __uint_as_float(r0v[e]); dst[32 + e] = __uint_as_float(r1v[e]); }
      }
      __syncthreads();
      if (row < 64) {
        const float* add = scratch + row * 64;
        float v[64];
#pragma unroll
        for (int e = 0; e < 32; ++e) { v[e] = __uint_as_float(r0v[e]) + add[e]; v[32 + e] = __uint_as_float(r1v[e]) + add[32 + e]; }
        if constexpr (B == 64) {
          float* o = dPs + ((size_t)t * 64 + row) * 64;
#pragma unroll
          for (int e = 0; e < 64; ++e) o[e] = v[e];
        } else {
          const int qb = row / 32;            // which 32-block of the tile
          float* o = dPs + ((size_t)(2 * t + qb) * 32 + (row - 32 * qb)) * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = v[32 * qb + e];
        }
      }
    } else {
      float* o = dPs + ((size_t)t * BC + row) * BC;
#pragma unroll 1
      for (int cc = 0; cc < BC / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tDP + lane_off + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[cc * 32 + e] = __uint_as_float(r[e]);
      }
    }
  }
  if (tid == 0) {
    if (pending_load >= 0) mbar_wait_drain(bar_load, (uint32_t)pending_load, 35);
    mma_commit(bar_drain);
    mbar_wait_drain(bar_drain, 0, 36);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host --

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [outer, inner] matrix, box {bx, by}, 128-byte swizzle.
lcp_status make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t bx,
                    uint32_t by, const char* what) {
  EncodeFn fn = encode_fn();
  if (!fn) return fail(LCP_ERR_CUDA, "%s: cuTensorMapEncodeTiled is unavailable from the driver", what);
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {bx, by};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LCP_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)r);
  return LCP_OK;
}

int num_sms() {
  static int n[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!n[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

template <typename K>
lcp_status set_smem(K kernel, int bytes, const char* what) {
  return ensure_smem_limit(reinterpret_cast<const void*>(kernel), bytes, what);
}

#define TC_TRY(x)                      \
  do {                                 \
    const lcp_status s_ = (x);         \
    if (s_ != LCP_OK) return s_;       \
  } while (0)

template <int BC, int MG>
lcp_status permute_mask2_bc(const CUtensorMap& mW, const CUtensorMap& mPth, const CUtensorMap& mPtl,
                            const CUtensorMap& mPh, uint32_t* mask, __nv_bfloat16* At, float* Wp, int cout,
                            int cin, int n, cudaStream_t st) {
  using C = Pm2Cfg<BC>;
  auto k = permute_mask_tc2_kernel<BC, MG>;
  TC_TRY(set_smem(k, C::SMEM, "permute_mask_tc"));
  const int ntiles = cin / BC, nrt = cdiv(cout, 128);
  int ry = cdiv(C::CTAS_PER_SM * num_sms(), ntiles);
  if (ry > nrt) ry = nrt;
  if (ry < 1) ry = 1;
  k<<<dim3(ntiles, ry), 128, C::SMEM, st>>>(mW, mPth, mPtl, mPh, mask, At, Wp, cout, cin, n);
  return check_launch("permute_mask_tc");
}

template <int BC, int MG>
lcp_status permute_mask_bc(const CUtensorMap& mW, const CUtensorMap& mPth, const CUtensorMap& mPtl,
                           const CUtensorMap& mPh, uint32_t* mask, __nv_bfloat16* At, float* Wp, int cout,
                           int cin, int n, cudaStream_t st) {
  auto k = permute_mask_tc_kernel<BC, MG>;
  TC_TRY(set_smem(k, PmCfg<BC>::SMEM, "permute_mask_tc"));
  const dim3 grid(cdiv(cout, 128), cin / BC);
  k<<<grid, 128, PmCfg<BC>::SMEM, st>>>(mW, mPth, mPtl, mPh, mask, At, Wp, cout, cin, n);
  return check_launch("permute_mask_tc");
}

template <int BC, int B>
lcp_status block_bwd_bc(const CUtensorMap& mW, const CUtensorMap& mD, const CUtensorMap& mPth,
                        const CUtensorMap& mPtl, const uint32_t* mask, float* dP, int splits, int rows,
                        int cout, int cin, cudaStream_t st) {
  auto k = block_bwd_tc_kernel<BC, B>;
  TC_TRY(set_smem(k, BbCfg<BC>::SMEM, "block_bwd_tc"));
  const dim3 grid(cin / BC, splits);
  k<<<grid, 128, BbCfg<BC>::SMEM, st>>>(mW, mD, mPth, mPtl, mask, dP, cout, cin, rows);
  return check_launch("block_bwd_tc");
}

int bb_rows_per_split(int cout, int cin, int B) {
  const int BC = B < 64 ? 64 : B;
  const int tiles = cin / BC;
  const int chunks = cdiv(cout, 128);
  // one CTA per SM: as many row segments per channel tile as fill the SMs once
  int S = 148 / tiles;
  if (S < 1) S = 1;
  if (S > 64) S = 64;
  if (S > chunks) S = chunks;
  return cdiv(chunks, S) * 128;
}

}  // namespace

bool tc_available() { return true; }

bool block_bwd_tc_supported(int B) { return B <= 128; }

int block_bwd_tc_splits(int cout, int cin, int B) {
  if (!block_bwd_tc_supported(B)) return 1;
  return cdiv(cout, bb_rows_per_split(cout, cin, B));
}

template <typename K>
lcp_status launch_pair(K kernel, int tiles, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       void* d0, void* d1, int M, int N, int Kd, int ldd, int nprob, cudaStream_t st,
                       const char* what) {
  TC_TRY(set_smem(kernel, G2_SMEM, what));
  const int max_pairs = num_sms() / 2;
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(GM_THREADS);
  cfg.dynamicSmemBytes = G2_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, a, b0, b1, d0, d1, M, N, Kd, ldd, nprob);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  return check_launch(what);
}

bool use_pair_gemm() { return true; }

lcp_status launch_calib_gemm_tc(const __nv_bfloat16* X, const __nv_bfloat16* W, const __nv_bfloat16* At,
                                float* Yd, float* Ys, int tokens, int cout, int cin, cudaStream_t st) {
  CUtensorMap mA, mB0, mB1;
  TC_TRY(make_map(&mA, X, cin, tokens, 64, 128, "calib_gemm X"));
  TC_TRY(make_map(&mB0, W, cin, cout, 64, 256, "calib_gemm W"));
  const int nprob = Ys ? 2 : 1;
  TC_TRY(make_map(&mB1, Ys ? (const void*)At : (const void*)W, cin, cout, 64, 256, "calib_gemm At"));
  if (use_pair_gemm()) {
    CUtensorMap pA, pB0, pB1;   // operand halves of 128 rows
    TC_TRY(make_map(&pA, X, cin, tokens, 64, 128, "calib_gemm X"));
    TC_TRY(make_map(&pB0, W, cin, cout, 64, 128, "calib_gemm W"));
    TC_TRY(make_map(&pB1, Ys ? (const void*)At : (const void*)W, cin, cout, 64, 128, "calib_gemm At"));
    const int tiles2 = cdiv(tokens, G2_BM) * cdiv(cout, G2_BN) * nprob;
    return launch_pair(gemm_pair_tc_kernel<false, false, false>, tiles2, pA, pB0, pB1, Yd, Ys, tokens, cout, cin,
                       cout, nprob, st, "calib_gemm");
  }
  auto k = gemm_tc_kernel<false, false, false>;
  TC_TRY(set_smem(k, GM_SMEM, "calib_gemm"));
  const int tiles = cdiv(tokens, GM_BM) * cdiv(cout, GM_BN) * nprob;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  k<<<grid, GM_THREADS, GM_SMEM, st>>>(mA, mB0, mB1, Yd, Ys, tokens, cout, cin, cout, nprob);
  return check_launch("calib_gemm");
}

lcp_status launch_bwd_gemm_tc(const __nv_bfloat16* G, const __nv_bfloat16* X, __nv_bfloat16* dAt, int tokens,
                              int cout, int cin, cudaStream_t st) {
  CUtensorMap mA, mB;
  TC_TRY(make_map(&mA, G, cout, tokens, 64, 64, "grad_gemm G"));
  TC_TRY(make_map(&mB, X, cin, tokens, 64, 64, "grad_gemm X"));
  if (use_pair_gemm()) {
    const int tiles2 = cdiv(cout, G2_BM) * cdiv(cin, G2_BN);
    return launch_pair(gemm_pair_tc_kernel<true, true, true>, tiles2, mA, mB, mB, dAt, nullptr, cout, cin, tokens, cin,
                       1, st, "grad_gemm");
  }
  auto k = gemm_tc_kernel<true, true, true>;
  TC_TRY(set_smem(k, GM_SMEM, "grad_gemm"));
  const int tiles = cdiv(cout, GM_BM) * cdiv(cin, GM_BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  k<<<grid, GM_THREADS, GM_SMEM, st>>>(mA, mB, mB, dAt, nullptr, cout, cin, tokens, cin, 1);
  return check_launch("grad_gemm");
}

lcp_status launch_permute_mask_tc(const __nv_bfloat16* W, const __nv_bfloat16* img_pt_hi,
                                  const __nv_bfloat16* img_pt_lo, const __nv_bfloat16* img_p_hi, uint32_t* mask,
                                  __nv_bfloat16* At, float* Wp_out, int cout, int cin, int B, int n, int m,
                                  cudaStream_t st) {
  const int BC = B < 64 ? 64 : B;
  CUtensorMap mW, mPth, mPtl, mPh;
  TC_TRY(make_map(&mW, W, cin, cout, 64, 128, "permute_mask W"));
  TC_TRY(make_map(&mPth, img_pt_hi, BC, cin, 64, 64, "permute_mask Pt_hi"));
  TC_TRY(make_map(&mPtl, img_pt_lo, BC, cin, 64, 64, "permute_mask Pt_lo"));
  TC_TRY(make_map(&mPh, img_p_hi, BC, cin, 64, BC == 64 ? 64 : BC, "permute_mask P_hi"));
  if (BC == 64) {
    CUtensorMap mAt;
    TC_TRY(make_map(&mAt, At, cin, cout, 64, 128, "permute_mask At"));
    constexpr int NSL = 2;
    using C = PwCfg<NSL>;
    auto k = (m == 4) ? permute_mask_ws_kernel<4, NSL> : permute_mask_ws_kernel<8, NSL>;
    TC_TRY(set_smem(k, C::SMEM, "permute_mask_tc"));
    const int tiles = cdiv(cout, 128) * (cin / 64);
    const int grid = tiles < num_sms() ? tiles : num_sms();
    k<<<grid, C::THREADS, C::SMEM, st>>>(mW, mPth, mPtl, mPh, mAt, mask, Wp_out, cout, cin, n);
    return check_launch("permute_mask_tc");
  }
  if (m == 4) {
    if (BC == 128) return permute_mask2_bc<128, 4>(mW, mPth, mPtl, mPh, mask, At, Wp_out, cout, cin, n, st);
    return permute_mask_bc<256, 4>(mW, mPth, mPtl, mPh, mask, At, Wp_out, cout, cin, n, st);
  }
  if (BC == 128) return permute_mask2_bc<128, 8>(mW, mPth, mPtl, mPh, mask, At, Wp_out, cout, cin, n, st);
  return permute_mask_bc<256, 8>(mW, mPth, mPtl, mPh, mask, At, Wp_out, cout, cin, n, st);
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
  TC_TRY(make_map(&mPth, img_pt_hi, BC, cin, 64, BC, "block_bwd Pt_hi"));
  TC_TRY(make_map(&mPtl, img_pt_lo, BC, cin, 64, BC, "block_bwd Pt_lo"));
  if (B <= 64) {
    constexpr int NSL = 2;
    using C = BwCfg<NSL>;
    auto k = (B == 32) ? block_bwd_ws_kernel<32, NSL> : block_bwd_ws_kernel<64, NSL>;
    TC_TRY(set_smem(k, C::SMEM, "block_bwd_tc"));
    k<<<dim3(cin / 64, splits), C::THREADS, C::SMEM, st>>>(mW, mD, mPth, mPtl, mask, dP_partials, cout, cin, rows);
    return check_launch("block_bwd_tc");
  }
  return block_bwd_bc<128, 128>(mW, mD, mPth, mPtl, mask, dP_partials, splits, rows, cout, cin, st);
}

}  // namespace lcp

extern "C" lcp_status lcp_device_error(int* site, int reset) {
  using namespace lcp;
  if (!site) return fail(LCP_ERR_NULL, "site is NULL");
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(int));
  if (e == cudaSuccess && reset) {
    const int z = 0;
    e = cudaMemcpyToSymbol(g_tc_error, &z, sizeof(int));
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
  }
  *site = v;
  return LCP_OK;
}
