// Hardening of the soft permutation (PermLLM, "Method", subsection 2): in the
// forward pass every diagonal block P_hat_b of the Sinkhorn output is replaced
// by the permutation pi maximising Tr(P^T P_hat_b) = sum_i P_hat_b[i, pi(i)],
// a linear assignment problem.  The backward pass is straight-through
// (dP / dP_hat = 1), which needs nothing here: the reverse kernels simply see
// the hard matrix in the operand images and hand their dP to the Sinkhorn
// reverse pass of the soft matrix.
//
// Solver: the Hungarian method in its shortest-augmenting-path form, exact up
// to float32 rounding of the potentials.  Costs c[i][j] = -P_hat[i][j].  Start
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
// One warp per block.  Lane l owns columns l, l + 32, ...: their potential v,
// matched row, tentative distance, predecessor row and scanned flag live in
// registers; the row -> column matching sits in shared memory next to the
// block's costs (B <= 128; for B = 256 the first 216 of its 256 rows, the rest
// read from global memory).  A
// search step is one scan of the owned columns, one warp-wide argmin (ties:
// lowest column) and two shuffles from the scanned column's owner, so the
// result is deterministic.

#include <math_constants.h>

#include "lcp_internal.cuh"

namespace lcp {
namespace {

__device__ int g_harden_error;   // 201 once a block's search overran (cannot happen), 0 otherwise

constexpr int kFree = -1;
constexpr int kRoot = -2;   // the virtual column the tree of the current row grows from

template <int B> struct HdCfg {
  static constexpr int CPL = B / 32;                        // columns per lane
  static constexpr bool SMEM_COST = B <= 128;
  // B = 256: the first CROWS cost rows in shared memory, the rest read from global memory
  static constexpr int CROWS = SMEM_COST ? B : 216;
  static constexpr int WARPS = B <= 64 ? 4 : 1;             // blocks per CTA
  static constexpr int COST_FLOATS = CROWS * B;
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
    for (int q = lane; q < C::CROWS * B / 4; q += 32) {
      const float4 x = reinterpret_cast<const float4*>(Pb)[q];
      cost[4 * q + 0] = -x.x; cost[4 * q + 1] = -x.y; cost[4 * q + 2] = -x.z; cost[4 * q + 3] = -x.w;
    }
  }
  auto c_at = [&](int i, int j) -> float {
    if constexpr (C::SMEM_COST) return cost[i * B + j];
    else return i < C::CROWS ? cost[i * B + j] : -__ldg(Pb + (size_t)i * B + j);
  };
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
  switch (B) {
    case 32: return harden_b<32>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
    case 64: return harden_b<64>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
    case 128: return harden_b<128>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
    case 256: return harden_b<256>(P, perm, P_hard, img_pt_hi, img_pt_lo, img_p_hi, nblocks, st);
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
