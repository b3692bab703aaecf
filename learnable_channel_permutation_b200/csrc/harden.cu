// Hardening of the soft permutation (PermLLM, "Method", subsection 2): in the
// forward pass every diagonal block P_hat_b of the Sinkhorn output is replaced
// by the permutation pi maximising Tr(P^T P_hat_b) = sum_i P_hat_b[i, pi(i)],
// a linear assignment problem.  The backward pass is straight-through
// (dP / dP_hat = 1), which needs nothing here: the reverse kernels simply see
// the hard matrix in the operand images and hand their dP to the Sinkhorn
// reverse pass of the soft matrix.
//
// Two solvers, chosen by block size (measured on a B200: the single-warp search
// is the faster one for B = 32 and 64, the auction below for B = 128 and 256,
// where the search's step count grows with B^2).
//
// B = 32 and 64: the Hungarian method in its shortest-augmenting-path form,
// exact up to float32 rounding of the potentials.  Costs c[i][j] = -P_hat[i][j].  Start
// from v[j] = min_i c[i][j] (feasible), and match every column to the row of
// its minimum when no lower-numbered column claims that row (tight edges).
// Then each still-free row i0 runs a Dijkstra search over reduced costs with
// the potentials held fixed: tentative distances d[j] = c[i0][j] - v[j]; the
// nearest unscanned column is scanned, and if it is matched to row i, every
// unscanned column relaxes to d[j*] - u_i + c[i][j] - v[j], where the row
// potential u_i = c[i][j*] - v[j*] is implicit (matched edges are tight).
// Once a free column is reached at distance D, each scanned column's
// potential moves by d[j] - D and the matching flips along the path.
//
// One warp per block (B = 32 and 64).  Lane l owns columns l, l + 32, ...: their
// potential v, matched row, tentative distance, predecessor row and scanned flag
// live in registers; the row -> column matching sits in shared memory next to
// the block's costs.  A search step is one scan of the owned columns, one
// warp-wide argmin (ties: lowest column) and two shuffles from the scanned
// column's owner, so the result is deterministic.

#include <climits>

#include <math_constants.h>

#include "lcp_internal.cuh"

namespace lcp {
namespace {

__device__ int g_harden_error;   // 201 once a block's search overran (cannot happen), 0 otherwise

constexpr int kFree = -1;
constexpr int kRoot = -2;   // the virtual column the tree of the current row grows from

template <int B> struct HdCfg {
  static_assert(B <= 64, "the shortest-path solver serves B <= 64; larger blocks use the auction");
  static constexpr int CPL = B / 32;                        // columns per lane
  static constexpr int WARPS = 4;                           // blocks per CTA
  static constexpr int COST_FLOATS = B * B;
  static constexpr int PER_WARP = COST_FLOATS + 3 * B;      // costs, row -> column, match, claims (4-byte words)
  static constexpr size_t SMEM = (size_t)WARPS * PER_WARP * 4;
};

// Order-preserving map of a float to an unsigned key (no NaN): negative
// values reversed below the positive ones.
__device__ __forceinline__ unsigned sort_key(float x) {
  const unsigned u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// argmin over the warp of (value, column), ties to the lower column: two
// warp-wide integer minimum reductions (smallest key, then smallest column
// among the lanes holding it)
__device__ __forceinline__ void warp_argmin(float& v, int& j) {
  const unsigned k = __reduce_min_sync(0xffffffffu, sort_key(v));
  j = (int)__reduce_min_sync(0xffffffffu, sort_key(v) == k ? (unsigned)j : 0xffffffffu);
  v = key_value(k);
}

template <int B>
__global__ void __launch_bounds__(32 * HdCfg<B>::WARPS)
harden_kernel(const float* __restrict__ P, int* __restrict__ perm, float* __restrict__ P_hard,
              __nv_bfloat16* __restrict__ pt_hi, __nv_bfloat16* __restrict__ pt_lo, __nv_bfloat16* __restrict__ p_hi,
              int nblocks) {
  using C = HdCfg<B>;
  constexpr int CPL = C::CPL;
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) float hd_smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int blk = blockIdx.x * C::WARPS + warp;
  if (blk >= nblocks) return;
  float* cost = hd_smem + (size_t)warp * C::PER_WARP;       // c[i][j] = -P[i][j], rows [0, CROWS)
  float* u = cost + C::COST_FLOATS;                          // later the row -> column matching
  int* match = reinterpret_cast<int*>(u + B);                // column -> row, kFree if none
  int* way = match + B;                                      // row -> lowest claiming column
  const float* Pb = P + (size_t)blk * B * B;

  {
    for (int q = lane; q < B * B / 4; q += 32) {
      const float4 x = reinterpret_cast<const float4*>(Pb)[q];
      cost[4 * q + 0] = -x.x; cost[4 * q + 1] = -x.y; cost[4 * q + 2] = -x.z; cost[4 * q + 3] = -x.w;
    }
  }
  auto c_at = [&](int i, int j) -> float { return cost[i * B + j]; };
  for (int i = lane; i < B; i += 32) { u[i] = 0.f; match[i] = kFree; way[i] = kRoot; }
  __syncwarp();

  // column reduction: v[j] = min_i c[i][j]; column j claims the row of its
  // minimum (lowest row on ties) and the lowest claiming column gets the row
  float v[CPL];
  int claim[CPL];
#pragma unroll
  for (int s = 0; s < CPL; ++s) {
    const int j = lane + 32 * s;
    float best = c_at(0, j);
    int bi = 0;
    for (int i = 1; i < B; ++i) {
      const float x = c_at(i, j);
      if (x < best) { best = x; bi = i; }
    }
    v[s] = best;
    claim[s] = bi;
  }
  // way[] doubles as the row -> lowest claiming column table during the claim
  for (int i = lane; i < B; i += 32) way[i] = B;
  __syncwarp();
#pragma unroll
  for (int s = 0; s < CPL; ++s) atomicMin(&way[claim[s]], lane + 32 * s);
  __syncwarp();
#pragma unroll
  for (int s = 0; s < CPL; ++s) {
    const int j = lane + 32 * s;
    if (way[claim[s]] == j) match[j] = claim[s];
  }
  __syncwarp();
  // match[] -> registers: x[s] the row of column lane + 32 s; y[] (in the u slot) row -> column
  int* y = reinterpret_cast<int*>(u);
  for (int i = lane; i < B; i += 32) y[i] = kFree;
  __syncwarp();
  int x[CPL];
#pragma unroll
  for (int s = 0; s < CPL; ++s) {
    x[s] = match[lane + 32 * s];
    if (x[s] != kFree) y[x[s]] = lane + 32 * s;
  }
  __syncwarp();
  // each free row in increasing order: shortest augmenting path over reduced costs with the
  // potentials held fixed during the search (the row potentials stay implicit: a matched edge
  // is tight, u_i = c[i][col(i)] - v[col(i)]), then one update of the scanned columns'
  // potentials and a flip of the path
  bool ok = true;
  for (int i0 = 0; i0 < B && ok; ++i0) {
    if (y[i0] != kFree) continue;
    float d[CPL];
    int pred[CPL];
    bool sc[CPL];
#pragma unroll
    for (int s = 0; s < CPL; ++s) {
      d[s] = c_at(i0, lane + 32 * s) - v[s];
      pred[s] = i0;
      sc[s] = false;
    }
    int jend = -1;
    float D = 0.f;
    for (int steps = 0; steps < B; ++steps) {   // at most B columns get scanned
      float best = CUDART_INF_F;
      int bj = B;
#pragma unroll
      for (int s = 0; s < CPL; ++s) {
        const int j = lane + 32 * s;
        if (!sc[s] && (d[s] < best || (d[s] == best && j < bj))) { best = d[s]; bj = j; }
      }
      warp_argmin(best, bj);
      D = best;
      const int ol = bj & 31, os = bj >> 5;   // owner lane and slot of column bj
      int xo = x[0];
      float vo = v[0];
#pragma unroll
      for (int s = 1; s < CPL; ++s)
        if (os == s) { xo = x[s]; vo = v[s]; }
      const int xi = __shfl_sync(0xffffffffu, xo, ol);
      const float vj = __shfl_sync(0xffffffffu, vo, ol);
#pragma unroll
      for (int s = 0; s < CPL; ++s)
        if (s == os && lane == ol) sc[s] = true;
      if (xi == kFree) { jend = bj; break; }
      // through column bj to its row xi: distance of that row, less its implicit potential
      const float h = D - (c_at(xi, bj) - vj);
#pragma unroll
      for (int s = 0; s < CPL; ++s) {
        if (!sc[s]) {
          const float nd = h + (c_at(xi, lane + 32 * s) - v[s]);
          if (nd < d[s]) { d[s] = nd; pred[s] = xi; }
        }
      }
    }
    if (jend < 0) { ok = false; break; }   // cannot happen: a free column is always reachable
    // potentials: every scanned column moves by its distance short of D (the path becomes tight)
#pragma unroll
    for (int s = 0; s < CPL; ++s)
      if (sc[s]) v[s] += d[s] - D;
    // flip the path from column jend back to row i0
    int j = jend;
    for (int guard = 0; guard <= B; ++guard) {
      const int ol = j & 31, os = j >> 5;
      int po = pred[0];
#pragma unroll
      for (int s = 1; s < CPL; ++s)
        if (os == s) po = pred[s];
      const int i = __shfl_sync(0xffffffffu, po, ol);   // the row before column j on the path
      const int jn = y[i];                                // its column so far (free for i0)
      __syncwarp();
#pragma unroll
      for (int s = 0; s < CPL; ++s)
        if (s == os && lane == ol) x[s] = i;
      if (lane == 0) y[i] = j;
      __syncwarp();
      if (i == i0) break;
      if (guard == B) ok = false;                         // cannot happen: the path ends at i0
      j = jn;
    }
  }
  if (!__all_sync(0xffffffffu, ok)) {
    if (lane == 0) atomicCAS(&g_harden_error, 0, 201);
    return;
  }
#pragma unroll
  for (int s = 0; s < CPL; ++s) match[lane + 32 * s] = x[s];
  __syncwarp();

  // outputs: pi(i) = the column matched to row i, and the hard matrix
  int* pb = perm + (size_t)blk * B;
#pragma unroll
  for (int s = 0; s < CPL; ++s) {
    const int j = lane + 32 * s;
    pb[match[j]] = j;
  }
  if (P_hard) {
    float* H = P_hard + (size_t)blk * B * B;
    for (int q = lane; q < B * B; q += 32) H[q] = 0.f;
    __syncwarp();
#pragma unroll
    for (int s = 0; s < CPL; ++s) {
      const int j = lane + 32 * s;
      H[(size_t)match[j] * B + j] = 1.f;
    }
  }
  if (pt_hi) {
    // operand images in tiles of BC = max(B, 64) columns (the layout the
    // Sinkhorn kernel writes): Pt[j][i] = P[i][j] (high part exact, low part
    // zero), P_hi[i][j] = P[i][j]; with B = 32 two blocks share a tile and the
    // off-diagonal quadrants stay zero
    constexpr int BC = B < 64 ? 64 : B;
    const int gcol0 = blk * B;
    const size_t tb = (size_t)(gcol0 / BC) * BC * BC;
    const int q0 = gcol0 % BC;
    const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
    for (int q = lane; q < B * B; q += 32) {
      const int a = q / B, bcol = q % B;     // image row a, column bcol within the block
      pt_hi[tb + (size_t)(q0 + a) * BC + q0 + bcol] = zero;
      pt_lo[tb + (size_t)(q0 + a) * BC + q0 + bcol] = zero;
      p_hi[tb + (size_t)(q0 + a) * BC + q0 + bcol] = zero;
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < CPL; ++s) {
      const int j = lane + 32 * s, i = match[j];
      pt_hi[tb + (size_t)(q0 + j) * BC + q0 + i] = one;
      p_hi[tb + (size_t)(q0 + i) * BC + q0 + j] = one;
    }
  }
}

// ---------------------------------------------------------------------------
// B = 128 and 256: Bertsekas' forward auction with epsilon-scaling, in Jacobi
// rounds.  One CTA of 32 warps per block.  The benefits P_hat[i][j] are mapped
// onto integers a_ij = rint((P_hat[i][j] - min) 2^k) over the block's own range,
// 2^k the power of two with (max - min) 2^k in [2^28, 2^29).  Every unassigned row ("person") i bids for the column ("object")
// j* of largest value a_ij - p_j, raising its price to
// p_j* + (best - second best value) + eps; each column goes to its highest bid
// (lowest row on equal bids) and displaces its previous owner.  Phases run with
// eps a fixed fraction of the block's integer range, then divided by a fixed
// factor down to 1; between phases a row keeps its column only while it is
// within eps of its best value.  The final phase
// (eps = 1) ends with every row within one unit of its best value, so the
// assignment is within B units of the integer problem's maximum; with every
// a_ij within half a unit of (P_hat[i][j] - min) 2^k, it is within 2 B 2^-k
// <= B (max - min) 2^-27 of the maximum of P_hat itself.
//
// Each column's price and owner share one 64-bit word, price << 32 | (2^32 - 1
// - row), so a bid is a single shared-memory atomicMax and a row knows it still
// holds its column by reading that word.  A round reads (prices, owners) under
// one barrier and lands its bids under the next, so the result does not depend
// on the warps' timing.  Warp w handles rows w, w + WARPS, ...; lane l holds
// the CPL consecutive columns l CPL, ..., and a bid is one pass over them, two
// warp-wide integer maximum reductions and a ballot (ties: lowest column).
//
// Every thread tracks how many rows are free (a bid that finds its column
// without an owner leaves one fewer; a release one more).  When a single row
// is free, the rest of the phase is that row's chain of displacements: warp 0
// runs it alone, writing each bid directly (no barrier, no atomic), until a bid
// takes a column nobody holds -- the same bids the Jacobi rounds would make,
// one a round, without two CTA barriers each.
// ---------------------------------------------------------------------------

constexpr int kAuScaleLog2 = 29;               // benefits span [0, 2^29)
constexpr int kAuMaxRounds = 1 << 16;          // the sizes here need ~100 to ~1200
constexpr int kAuPriceLimit = 0x60000000;      // prices stayed below 2^29 in every case measured; checked

template <int B> struct AuCfg {
  static_assert(B == 64 || B == 128 || B == 256, "the auction serves B = 64, 128 and 256");
  static constexpr int WARPS = B == 64 ? 16 : 32;
  // epsilon schedule: the first phase at the block's integer range / EPS_DIV,
  // each next one THETA times smaller (the fastest of the schedules measured,
  // over near-uniform, intermediate and spread Sinkhorn outputs)
  static constexpr int EPS_DIV = B == 64 ? 256 : (B == 128 ? 128 : 512);
  static constexpr int THETA = B == 64 ? 64 : (B == 128 ? 16 : 32);
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int PPW = B / WARPS;                     // rows per warp
  static constexpr int CPL = B / 32;                        // columns per lane
  static constexpr int SROWS = B <= 128 ? B : 192;          // benefit rows in shared memory
  static constexpr int SSLOTS = SROWS / WARPS;              // a warp's rows k < SSLOTS read them there
  static constexpr int RSLOTS = PPW - SSLOTS;               // the rest live in registers
  static constexpr size_t BEN_BYTES = (size_t)SROWS * B * 4;
  // benefits, words, range scratch, row -> column table
  static constexpr size_t SMEM = BEN_BYTES + (size_t)B * 8 + 2 * 32 * 4 + (size_t)B * 4;
};

__device__ __forceinline__ unsigned au_code(int i) { return 0xffffffffu - (unsigned)i; }

// CPL consecutive ints / 64-bit words from shared memory, vectorised
template <int CPL> __device__ __forceinline__ void au_load_ints(const int* src, int (&v)[CPL]) {
  if constexpr (CPL == 2) {
    const int2 t = *reinterpret_cast<const int2*>(src);
    v[0] = t.x; v[1] = t.y;
    return;
  }
#pragma unroll
  for (int q = 0; q < CPL / 4; ++q) {
    const int4 t = reinterpret_cast<const int4*>(src)[q];
    v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
  }
}
template <int CPL> __device__ __forceinline__ void au_load_prices(const unsigned long long* w, int (&p)[CPL]) {
#pragma unroll
  for (int q = 0; q < CPL / 2; ++q) {
    const ulonglong2 t = reinterpret_cast<const ulonglong2*>(w)[q];
    p[2 * q] = (int)(t.x >> 32); p[2 * q + 1] = (int)(t.y >> 32);
  }
}

template <int B>
__global__ void __launch_bounds__(AuCfg<B>::THREADS)
harden_auction_kernel(const float* __restrict__ P, int* __restrict__ perm, float* __restrict__ P_hard,
                      __nv_bfloat16* __restrict__ pt_hi, __nv_bfloat16* __restrict__ pt_lo,
                      __nv_bfloat16* __restrict__ p_hi, int nblocks) {
  using C = AuCfg<B>;
  constexpr int CPL = C::CPL, PPW = C::PPW, NW = C::WARPS, NT = C::THREADS;
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char au_smem[];
  int* ben = reinterpret_cast<int*>(au_smem);                                        // [SROWS][B]
  unsigned long long* word = reinterpret_cast<unsigned long long*>(au_smem + C::BEN_BYTES);   // [B]
  unsigned* red = reinterpret_cast<unsigned*>(word + B);                              // [2][32]
  int* obj_of = reinterpret_cast<int*>(red + 64);                                     // [B]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int blk = blockIdx.x;
  if (blk >= nblocks) return;
  const float* Pb = P + (size_t)blk * B * B;

  // the block's range: order-preserving keys, minimum and maximum over the CTA
  unsigned kmin = 0xffffffffu, kmax = 0u;
  for (int q = threadIdx.x; q < B * B / 4; q += NT) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(Pb) + q);
    const unsigned k0 = sort_key(x.x), k1 = sort_key(x.y), k2 = sort_key(x.z), k3 = sort_key(x.w);
    kmin = min(kmin, min(min(k0, k1), min(k2, k3)));
    kmax = max(kmax, max(max(k0, k1), max(k2, k3)));
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) { red[warp] = kmin; red[32 + warp] = kmax; }
  for (int j = threadIdx.x; j < B; j += NT) word[j] = 0ull;   // price 0, no owner
  __syncthreads();
  kmin = __reduce_min_sync(0xffffffffu, lane < NW ? red[lane] : 0xffffffffu);
  kmax = __reduce_max_sync(0xffffffffu, lane < NW ? red[32 + lane] : 0u);
  // a_ij = rint((P_ij - min) 2^k), 2^k the power of two with (max - min) 2^k in
  // [2^28, 2^29): the difference of two floats is exact in double and so is the
  // scaling, so every benefit is within half a unit of the exact value
  const double lo = (double)key_value(kmin), hi = (double)key_value(kmax);
  int ex = 0;
  if (hi > lo) frexp(hi - lo, &ex);
  const double scale = hi > lo ? ldexp(1.0, kAuScaleLog2 - ex) : 0.0;
  auto quant = [&](float x) { return (int)rint(((double)x - lo) * scale); };
  for (int q = threadIdx.x; q < C::SROWS * B / 4; q += NT) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(Pb) + q);
    reinterpret_cast<int4*>(ben)[q] = make_int4(quant(x.x), quant(x.y), quant(x.z), quant(x.w));
  }
  int rben[C::RSLOTS > 0 ? C::RSLOTS : 1][CPL];
#pragma unroll
  for (int r = 0; r < C::RSLOTS; ++r) {
    const int i = warp + NW * (C::SSLOTS + r);
#pragma unroll
    for (int c = 0; c < CPL; ++c) rben[r][c] = quant(__ldg(Pb + (size_t)i * B + lane * CPL + c));
  }
  __syncthreads();

  auto benefits = [&](int k, int (&a)[CPL]) {
    if (k < C::SSLOTS) {
      au_load_ints<CPL>(ben + (size_t)(warp + NW * k) * B + lane * CPL, a);
    } else {
#pragma unroll
      for (int r = 0; r < C::RSLOTS; ++r)
        if (k == C::SSLOTS + r) {
#pragma unroll
          for (int c = 0; c < CPL; ++c) a[c] = rben[r][c];
        }
    }
  };

  auto any_row = [&](int i, int (&a)[CPL]) {   // rows past SROWS from global memory, quantised alike
    if (i < C::SROWS) {
      au_load_ints<CPL>(ben + (size_t)i * B + lane * CPL, a);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) a[c] = quant(__ldg(Pb + (size_t)i * B + lane * CPL + c));
    }
  };

  int myobj[PPW];
#pragma unroll
  for (int k = 0; k < PPW; ++k) myobj[k] = 0;   // word[0] has no owner yet: every row starts free
  int nfree = B;   // rows without a column, the same in every thread
  int eps = max(1, (int)rint((hi - lo) * scale) / C::EPS_DIV);
  int rounds = 0;
  bool ok = true;
  int over = 0;   // a bid reached the price limit (clamped; reported after the search)
  for (int phase = 0; ok; ++phase) {
    if (phase > 0) {
      // a row keeps its column only while its value there is within eps of its best value
      unsigned rel = 0;
#pragma unroll
      for (int k = 0; k < PPW; ++k) {
        const int i = warp + NW * k;
        const unsigned long long wo = word[myobj[k]];
        if ((unsigned)wo == au_code(i)) {
          int a[CPL], p[CPL];
          benefits(k, a);
          au_load_prices<CPL>(word + lane * CPL, p);
          int v1 = a[0] - p[0];
#pragma unroll
          for (int c = 1; c < CPL; ++c) v1 = max(v1, a[c] - p[c]);
          const int m1 = __reduce_max_sync(0xffffffffu, v1);
          const int ol = myobj[k] / CPL, oc = myobj[k] % CPL;
          int vo = a[0] - p[0];
#pragma unroll
          for (int c = 1; c < CPL; ++c)
            if (c == oc) vo = a[c] - p[c];
          vo = __shfl_sync(0xffffffffu, vo, ol);
          if (m1 - vo > eps) {
            if (lane == 0) word[myobj[k]] = wo & 0xffffffff00000000ull;   // release, price kept
            rel |= 1u << k;
          }
        }
      }
      nfree += __syncthreads_count(lane < PPW && ((rel >> lane) & 1u));
    }
    for (;;) {
      if (++rounds > kAuMaxRounds) { ok = false; break; }
      if (nfree == 0) break;
      if (nfree == 1) {
        // one free row: its chain of displacements runs on warp 0 alone, each bid
        // written directly (no barrier, no atomic), until a bid takes a free column
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < PPW; ++k) obj_of[warp + NW * k] = myobj[k];
        }
        if (threadIdx.x == 0) red[0] = 0u;
        __syncthreads();
        if (warp == 0) {
          int f = -1;
          for (int i0 = 0; i0 < B; i0 += 32) {
            const unsigned bal =
                __ballot_sync(0xffffffffu, (unsigned)word[obj_of[i0 + lane]] != au_code(i0 + lane));
            if (f < 0 && bal != 0u) f = i0 + __ffs(bal) - 1;
          }
          for (int chain = 0; f >= 0; ++chain) {
            if (chain >= kAuMaxRounds) {
              if (lane == 0) red[0] = 1u;
              break;
            }
            int a[CPL], p[CPL];
            unsigned own[CPL];
            any_row(f, a);
#pragma unroll
            for (int q = 0; q < CPL / 2; ++q) {
              const ulonglong2 t = reinterpret_cast<const ulonglong2*>(word + lane * CPL)[q];
              p[2 * q] = (int)(t.x >> 32); own[2 * q] = (unsigned)t.x;
              p[2 * q + 1] = (int)(t.y >> 32); own[2 * q + 1] = (unsigned)t.y;
            }
            int v1 = INT_MIN, v2 = INT_MIN, c1 = 0;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
              const int v = a[c] - p[c];
              if (v > v1) { v2 = v1; v1 = v; c1 = c; }
              else if (v > v2) v2 = v;
            }
            const int m1 = __reduce_max_sync(0xffffffffu, v1);
            const int wl = __ffs(__ballot_sync(0xffffffffu, v1 == m1)) - 1;
            const int m2 = __reduce_max_sync(0xffffffffu, lane == wl ? v2 : v1);
            int pc = p[0];
            unsigned oc = own[0];
#pragma unroll
            for (int c = 1; c < CPL; ++c)
              if (c == c1) { pc = p[c]; oc = own[c]; }
            const int cw = __shfl_sync(0xffffffffu, c1, wl);
            const int pw = __shfl_sync(0xffffffffu, pc, wl);
            const unsigned prev = __shfl_sync(0xffffffffu, oc, wl);
            const long long bid = (long long)pw + ((long long)m1 - m2) + eps;
            if (bid >= kAuPriceLimit) over = 1;
            const int j = wl * CPL + cw;
            if (lane == 0) {
              word[j] = ((unsigned long long)(unsigned)min(bid, (long long)kAuPriceLimit) << 32) | au_code(f);
              obj_of[f] = j;
            }
            __syncwarp();
            f = prev != 0u ? (int)(0xffffffffu - prev) : -1;   // the displaced owner bids next
          }
        }
        __syncthreads();
        if (red[0] != 0u) { ok = false; break; }
#pragma unroll
        for (int k = 0; k < PPW; ++k) myobj[k] = obj_of[warp + NW * k];
        nfree = 0;
        break;
      }
      unsigned pend = 0;
      int bidv[PPW];
      unsigned held[PPW];   // owner codes of the rows' columns, loaded together before any branch
#pragma unroll
      for (int k = 0; k < PPW; ++k) held[k] = (unsigned)word[myobj[k]];
#pragma unroll
      for (int k = 0; k < PPW; ++k) {
        const int i = warp + NW * k;
        bidv[k] = 0;
        if (held[k] != au_code(i)) {   // free: bid
          int a[CPL], p[CPL];
          benefits(k, a);
          au_load_prices<CPL>(word + lane * CPL, p);
          int v1 = INT_MIN, v2 = INT_MIN, c1 = 0;
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            const int v = a[c] - p[c];
            if (v > v1) { v2 = v1; v1 = v; c1 = c; }
            else if (v > v2) v2 = v;
          }
          const int m1 = __reduce_max_sync(0xffffffffu, v1);
          const int wl = __ffs(__ballot_sync(0xffffffffu, v1 == m1)) - 1;   // lowest column attaining it
          const int m2 = __reduce_max_sync(0xffffffffu, lane == wl ? v2 : v1);
          int pc = p[0];
#pragma unroll
          for (int c = 1; c < CPL; ++c)
            if (c == c1) pc = p[c];
          const int cw = __shfl_sync(0xffffffffu, c1, wl);
          const int pw = __shfl_sync(0xffffffffu, pc, wl);
          const long long bid = (long long)pw + ((long long)m1 - m2) + eps;
          if (bid >= kAuPriceLimit) over = 1;
          bidv[k] = (int)min(bid, (long long)kAuPriceLimit);
          myobj[k] = wl * CPL + cw;
          pend |= 1u << k;
        }
      }
      __syncthreads();   // every read of this round precedes every bid
      // lane k lands bid k; a bid that finds its column without an owner leaves one row
      // fewer free (exactly one bid on such a column sees that, whichever wins)
      bool took = false;
#pragma unroll
      for (int k = 0; k < PPW; ++k)
        if (lane == k && (pend & (1u << k))) {
          const unsigned long long old =
              atomicMax(&word[myobj[k]], ((unsigned long long)(unsigned)bidv[k] << 32) | au_code(warp + NW * k));
          took = (unsigned)old == 0u;
        }
      nfree -= __syncthreads_count(took);
    }
    if (eps == 1) break;
    eps = max(1, eps / C::THETA);
  }
  if (__syncthreads_or(over)) ok = false;
  if (!ok) {
    if (threadIdx.x == 0) atomicCAS(&g_harden_error, 0, 202);
    return;
  }

  // outputs: pi(i) = the column row i holds; the column -> row table for the matrices
  int* pb = perm + (size_t)blk * B;
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < PPW; ++k) pb[warp + NW * k] = myobj[k];
  }
  int* row_of = ben;   // the benefits are no longer read
  __syncthreads();
  for (int j = threadIdx.x; j < B; j += NT) row_of[j] = (int)(0xffffffffu - (unsigned)word[j]);
  __syncthreads();
  if (P_hard) {
    float* H = P_hard + (size_t)blk * B * B;
    for (int q = threadIdx.x; q < B * B / 4; q += NT) reinterpret_cast<float4*>(H)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    for (int j = threadIdx.x; j < B; j += NT)
      if ((unsigned)row_of[j] < (unsigned)B) H[(size_t)row_of[j] * B + j] = 1.f;
  }
  if (pt_hi) {
    constexpr int BC = B < 64 ? 64 : B;
    const int gcol0 = blk * B;
    const size_t tb = (size_t)(gcol0 / BC) * BC * BC;
    const int q0 = gcol0 % BC;
    const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
    for (int q = threadIdx.x; q < B * B; q += NT) {
      const int a = q / B, bcol = q % B;
      pt_hi[tb + (size_t)(q0 + a) * BC + q0 + bcol] = zero;
      pt_lo[tb + (size_t)(q0 + a) * BC + q0 + bcol] = zero;
      p_hi[tb + (size_t)(q0 + a) * BC + q0 + bcol] = zero;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < B; j += NT) {
      const int i = row_of[j];
      if ((unsigned)i >= (unsigned)B) continue;   // cannot happen: every column has an owner
      pt_hi[tb + (size_t)(q0 + j) * BC + q0 + i] = one;
      p_hi[tb + (size_t)(q0 + i) * BC + q0 + j] = one;
    }
  }
}

template <int B>
lcp_status harden_auction_b(const float* P, int* perm, float* P_hard, __nv_bfloat16* a, __nv_bfloat16* b,
                            __nv_bfloat16* c, int nblocks, cudaStream_t st) {
  using C = AuCfg<B>;
  const lcp_status s0 =
      ensure_smem_limit(reinterpret_cast<const void*>(harden_auction_kernel<B>), (int)C::SMEM, "harden");
  if (s0 != LCP_OK) return s0;
  return launch_kernel(harden_auction_kernel<B>, dim3(nblocks), dim3(C::THREADS), C::SMEM, st, 1, true, "harden",
                       P, perm, P_hard, a, b, c, nblocks);
}

template <int B>
lcp_status harden_b(const float* P, int* perm, float* P_hard, __nv_bfloat16* a, __nv_bfloat16* b,
                    __nv_bfloat16* c, int nblocks, cudaStream_t st) {
  using C = HdCfg<B>;
  const lcp_status s0 = ensure_smem_limit(reinterpret_cast<const void*>(harden_kernel<B>), (int)C::SMEM, "harden");
  if (s0 != LCP_OK) return s0;
  const int grid = (nblocks + C::WARPS - 1) / C::WARPS;
  return launch_kernel(harden_kernel<B>, dim3(grid), dim3(32 * C::WARPS), C::SMEM, st, 1, true, "harden", P, perm,
                       P_hard, a, b, c, nblocks);
}

}  // namespace

lcp_status launch_harden(const float* P, int* perm, float* P_hard, __nv_bfloat16* img_pt_hi,
                         __nv_bfloat16* img_pt_lo, __nv_bfloat16* img_p_hi, int nblocks, int B, cudaStream_t st) {
  if (nblocks == 0) return LCP_OK;
  switch (B) {   // shortest augmenting paths for the small blocks, the auction for the large ones
    case 32: return harden_b<32>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
#ifndef LCP_HARDEN_AUCTION_64
#define LCP_HARDEN_AUCTION_64 0   // 1: the auction at B = 64 (faster on spread P, slower near the initialisation)
#endif
    case 64:
      if (LCP_HARDEN_AUCTION_64) return harden_auction_b<64>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
      return harden_b<64>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
    case 128: return harden_auction_b<128>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
    case 256: return harden_auction_b<256>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
  }
  return fail(LCP_ERR_SHAPE, "harden: unsupported block size %d", B);
}

lcp_status harden_error(int* site, int reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_harden_error, sizeof(int));
  if (e == cudaSuccess && reset) {
    const int z = 0;
    e = cudaMemcpyToSymbol(g_harden_error, &z, sizeof(int));
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "reading the hardening error word: %s", cudaGetErrorString(e));
  }
  *site = v;
  return LCP_OK;
}

}  // namespace lcp
