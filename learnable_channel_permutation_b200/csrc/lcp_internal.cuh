// Internal declarations shared by the CUDA translation units of liblcp.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/lcp.h"

namespace lcp {

// ---- error reporting (thread-local message, see lcp_last_error) ----------
void set_error(const char* fmt, ...);
lcp_status fail(lcp_status s, const char* fmt, ...);
// Checks cudaGetLastError() after a launch; returns LCP_ERR_CUDA with `what`.
lcp_status check_launch(const char* what);
// Before the first launch of an entry point: an error another caller left
// pending (cudaPeekAtLastError) is reported as LCP_ERR_CUDA and NOT cleared,
// so that neither is it blamed on this call's launches nor lost to its owner.
lcp_status check_pending();

// Raises `func`'s dynamic shared-memory limit to `bytes` on the current device
// unless an earlier call already did (the attribute persists for the process).
lcp_status ensure_smem_limit(const void* func, int bytes, const char* what);

// ---- programmatic dependent launch -------------------------------------
// A kernel launched with pdl = true (launch_kernel below) may start while the
// kernel before it on the stream is still finishing.  It calls pdl_wait()
// before touching any global memory that an earlier kernel writes or reads
// (the only exception: the permute kernels prefetch the weight W, which no
// kernel of a step writes), and pdl_trigger() after its own pdl_wait(), which
// lets the next kernel start its prologue.  Launched without the attribute,
// both are no-ops.  LCP_PDL=0 in the environment turns the attribute off.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
bool pdl_enabled();

// Launches `kernel` with an optional cluster size (x) and the PDL attribute.
template <typename... KArgs, typename... Args>
lcp_status launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         int cluster, bool pdl, const char* what, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl && pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  return check_launch(what);
}

// ---- element conversions -------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ---- N:4 keep bits --------------------------------------------------------
// Bit j of the result keeps element j of NV consecutive values (NV / 4 groups
// of M = 4 consecutive columns): the same bits as the pairwise count
// (nm_bits), computed bit-sliced.  For a pair a < b of a group, bit 4g of
// T_ab says that element b beats element a (|v_b| > |v_a|; equal magnitudes
// go to the lower index); it is the sign of the single-precision difference
// |v_a| - |v_b|, which is exact in sign (equal magnitudes give +0, distinct
// ones a nonzero difference; no flush to zero in this build).  Element j is
// kept when it beats at least 4 - n of the other three: all of them (n = 1,
// bitwise AND), two (n = 2, bitwise majority) or one (n = 3, OR); n = 4 keeps
// everything.  Six subtractions and bit moves per group, a few word-wide
// logic operations per 32 values.
__device__ __forceinline__ uint32_t sign_at(float d, int pos) {
  return (__float_as_uint(d) >> 31) << pos;
}
template <int NV>
__device__ __forceinline__ uint32_t nm4_keep(const uint32_t (&v)[NV], int n) {
  uint32_t T01 = 0, T02 = 0, T03 = 0, T12 = 0, T13 = 0, T23 = 0;
#pragma unroll
  for (int g = 0; g < NV / 4; ++g) {
    const float a0 = fabsf(__uint_as_float(v[4 * g])), a1 = fabsf(__uint_as_float(v[4 * g + 1]));
    const float a2 = fabsf(__uint_as_float(v[4 * g + 2])), a3 = fabsf(__uint_as_float(v[4 * g + 3]));
    const int p = 4 * g;
    T01 |= sign_at(a0 - a1, p);
    T02 |= sign_at(a0 - a2, p);
    T03 |= sign_at(a0 - a3, p);
    T12 |= sign_at(a1 - a2, p);
    T13 |= sign_at(a1 - a3, p);
    T23 |= sign_at(a2 - a3, p);
  }
  if (n >= 4) return NV == 32 ? 0xffffffffu : (1u << NV) - 1u;   // nothing pruned
  if (n <= 0) return 0u;
  constexpr uint32_t lo = NV == 32 ? 0x11111111u : 0x1111u;   // bit 0 of every group
  // what element j beats: 0 -> ~T01 ~T02 ~T03, 1 -> T01 ~T12 ~T13, 2 -> T02 T12 ~T23, 3 -> T03 T13 T23
  auto f = [n](uint32_t x, uint32_t y, uint32_t z) {
    return n == 1 ? (x & y & z) : (n == 2 ? ((x & y) | (x & z) | (y & z)) : (x | y | z));
  };
  const uint32_t k0 = f(~T01, ~T02, ~T03) & lo, k1 = f(T01, ~T12, ~T13) & lo;
  const uint32_t k2 = f(T02, T12, ~T23) & lo, k3 = f(T03, T13, T23) & lo;
  return k0 | (k1 << 1) | (k2 << 2) | (k3 << 3);
}

// ---- launchers (host side; each returns LCP_OK or LCP_ERR_CUDA) ----------

// Sinkhorn.  img_* are optional bf16 operand images for the tensor-core path,
// stored as C_in/BC tiles of BC x BC (BC = max(B, 64)); tile t is the slice of
// blockdiag(P) covering channels [t*BC, (t+1)*BC), so with local indices:
//   img_pt_hi[t][j][i] = bf16(P[i][j])          (transposed, high part)
//   img_pt_lo[t][j][i] = bf16(P[i][j] - hi)     (transposed, low part)
//   img_p_hi [t][i][j] = bf16(P[i][j])          (high part)
// zero_word (optional) is set to 0 by the first CTA: the counter of the
// layer's fused loss kernel, which runs later on the same stream.
// One launch over the blocks of several layers (same B, tau, iters): the
// layers' blocks follow each other in the grid, in layer order; more than
// kSkMaxLayers layers take several launches.
constexpr int kSkMaxLayers = 16;
struct SkFwdLayer {
  const float* L;
  float* P;
  float* ckpt;
  __nv_bfloat16* pt_hi;
  __nv_bfloat16* pt_lo;
  __nv_bfloat16* p_hi;
  unsigned* zero_word;
  int blocks;
};
struct SkFwdBatch {
  SkFwdLayer layer[kSkMaxLayers];
  int n;
};
struct SkBwdLayer {
  const float* L;
  const float* ckpt;
  const float* dP;   // [splits, blocks, B, B]
  float* dL;
  int splits;
  int blocks;
};
struct SkBwdBatch {
  SkBwdLayer layer[kSkMaxLayers];
  int n;
};
lcp_status launch_sinkhorn_fwd_batch(const SkFwdLayer* layers, int n, int B, float tau, int iters, cudaStream_t st);
lcp_status launch_sinkhorn_bwd_batch(const SkBwdLayer* layers, int n, int B, float tau, int iters, cudaStream_t st);
lcp_status launch_sinkhorn_fwd(const float* L, float* P, float* ckpt, __nv_bfloat16* img_pt_hi,
                               __nv_bfloat16* img_pt_lo, __nv_bfloat16* img_p_hi, unsigned* zero_word,
                               int nblocks, int B, float tau, int iters, cudaStream_t st);
lcp_status launch_sinkhorn_bwd(const float* L, const float* ckpt, const float* dP, int splits,
                               float* dL, int nblocks, int B, float tau, int iters,
                               cudaStream_t st);

// out[i] = sum over s < splits of parts[s * n + i] (float32, n a multiple of 4,
// summed in index order): the block backward's dP partials for a caller.
lcp_status launch_sum_splits(const float* parts, int splits, size_t n, float* out, cudaStream_t st);

// N:M mask of a [rows, cols] matrix (float or bf16) into packed bits.
lcp_status launch_nm_mask(const void* Wp, uint32_t* bits, int rows, int cols, int n, int m,
                          lcp_dtype dt, cudaStream_t st);
// out[o][j] = mask(o, j) ? in[o][j] : 0   (float32, [rows, cols])
lcp_status launch_apply_mask(const float* in, const uint32_t* bits, float* out, int rows,
                             int cols, cudaStream_t st);

// Generic strided batched GEMM on CUDA cores with float32 accumulation:
//   C[z](m, n) = alpha * sum_k A[z](m, k) * B[z](k, n) + beta * C[z](m, n)
struct SimtGemm {
  int M, N, K, batch;
  const void* A; long long sAz, sAm, sAk;
  const void* B; long long sBz, sBk, sBn;
  void* C;       long long sCz, sCm, sCn;
  float alpha, beta;
};
lcp_status launch_simt_gemm(const SimtGemm& g, lcp_dtype ta, lcp_dtype tb, lcp_dtype tc,
                            cudaStream_t st);

// Loss.  stats[t] = {<yd,ys>, |yd|^2, |ys|^2, cos}.  G (optional) in dtype.
// `norm` is the token count the mean is taken over: `tokens` for a whole
// batch, the global count for one shard of it (the shards' losses and
// gradients then add up to the whole batch's).
lcp_status launch_loss_token(const float* Yd, const float* Ys, float* stats, void* G,
                             lcp_dtype gdt, int cout, int tokens, int norm, cudaStream_t st);
lcp_status launch_loss_grad(const float* Yd, const float* Ys, const float* stats, void* G,
                            lcp_dtype gdt, int cout, int tokens, int norm, cudaStream_t st);
lcp_status launch_loss_reduce(const float* stats, float* loss, int tokens, int norm, cudaStream_t st);
// One launch: stats, G and the loss.  cout <= 16384.  `counter` must be zero
// at launch (an earlier kernel of the step clears it); the kernel leaves it zero.
bool loss_fused_supported(int cout);
lcp_status launch_loss_fused(const float* Yd, const float* Ys, float* stats, void* G, lcp_dtype gdt,
                             float* loss, unsigned* counter, int cout, int tokens, int norm, cudaStream_t st);

// Loss and G (bf16) from the calibration GEMM's loss epilogue: the pair
// D = Y_d - Y_s, Y_s (bf16 [tokens, cout]) and the per-token partials of the
// nslots 64-channel slots (float4 [tokens, nslots]).  cout <= 16384 (see
// loss_pair_supported).  `counter` as for launch_loss_fused.
bool loss_pair_supported(int cout);
lcp_status launch_loss_pair(const __nv_bfloat16* D, const __nv_bfloat16* Ys, const float* partials, int nslots,
                            float* stats, __nv_bfloat16* G, float* loss, unsigned* counter, int cout, int tokens,
                            int norm, cudaStream_t st);

// Tensor-core (tcgen05) kernels, bf16 operands, float32 accumulation.
// given_mask (B <= 64): the mask is read from `mask` instead of computed.
lcp_status launch_permute_mask_tc(const __nv_bfloat16* W, const __nv_bfloat16* img_pt_hi,
                                  const __nv_bfloat16* img_pt_lo, const __nv_bfloat16* img_p_hi,
                                  uint32_t* mask, __nv_bfloat16* At, float* Wp_out, int cout,
                                  int cin, int B, int n, int m, bool given_mask, cudaStream_t st);
// B <= 64: the N:M mask of S_hat = S P_B (an importance score permuted like W)
// into `mask`; Shat_out (optional) receives S_hat as float32.
lcp_status launch_score_mask_tc(const __nv_bfloat16* S, const __nv_bfloat16* img_pt_hi,
                                const __nv_bfloat16* img_pt_lo, const __nv_bfloat16* img_p_hi, uint32_t* mask,
                                float* Shat_out, int cout, int cin, int B, int n, int m, cudaStream_t st);
lcp_status launch_calib_gemm_tc(const __nv_bfloat16* X, const __nv_bfloat16* W,
                                const __nv_bfloat16* At, float* Yd, float* Ys, int tokens,
                                int cout, int cin, cudaStream_t st);
// The calibration products with the loss reduction in the epilogue: D = Y_d -
// Y_s and Ys (bf16 [tokens, cout]) and the slot partials (float4 [tokens,
// calib_loss_slots(cout)]) -- see gemm_tc.cu.
int calib_loss_slots(int cout);
lcp_status launch_calib_loss_tc(const __nv_bfloat16* X, const __nv_bfloat16* W, const __nv_bfloat16* At,
                                __nv_bfloat16* D, __nv_bfloat16* Ys, float* partials, int tokens, int cout, int cin,
                                cudaStream_t st);
lcp_status launch_bwd_gemm_tc(const __nv_bfloat16* G, const __nv_bfloat16* X,
                              __nv_bfloat16* dAt, int tokens, int cout, int cin,
                              cudaStream_t st);
lcp_status launch_block_bwd_tc(const __nv_bfloat16* W, const __nv_bfloat16* dAt,
                               const uint32_t* mask, const __nv_bfloat16* img_pt_hi,
                               const __nv_bfloat16* img_pt_lo, float* dP_partials, int splits,
                               int cout, int cin, int B, cudaStream_t st);
int block_bwd_tc_splits(int cout, int cin, int B);
bool block_bwd_tc_supported(int B);   // every B (B = 256: four CTAs per block, one dP quadrant each)

// Hardening (per-block maximum-weight assignment).  Writes perm [nblocks, B],
// optionally the 0/1 matrices P_hard and the bf16 operand images of P_hard in
// the Sinkhorn kernel's tile layout (all three image pointers or none).
lcp_status launch_harden(const float* P, int* perm, float* P_hard, __nv_bfloat16* img_pt_hi,
                         __nv_bfloat16* img_pt_lo, __nv_bfloat16* img_p_hi, int nblocks, int B, cudaStream_t st);
lcp_status harden_error(int* site, int reset);

// Importance scores (LCP_SCORE_*) of W into S; stats: 2 cin + cout floats.
lcp_status launch_score(const void* W, const void* X, void* S, float* stats, int cout, int cin, int tokens, int kind,
                        lcp_dtype dt, cudaStream_t st);

// AdamW over n float32 values (n a multiple of 4), t the 1-based step.
lcp_status launch_adamw(float* L, const float* dL, float* m, float* v, long long n, double lr, double beta1,
                        double beta2, double eps, double weight_decay, int t, cudaStream_t st);

// Inference side: the 2:4 compressed weight (values [cout, cin/2], meta
// [cout, cin/32]) from W, the hard permutation and the mask bits; the input
// gather x_pi = P_B^T x; the product Y = x_pi A^T ([tokens, cout] float32).
lcp_status launch_pack24(const void* W, const int32_t* perm, const uint32_t* mask, void* vals, uint32_t* meta,
                         int cout, int cin, int B, lcp_dtype dt, cudaStream_t st);
lcp_status launch_gather(const void* X, const int32_t* perm, void* Xp, int tokens, int cin, int B, lcp_dtype dt,
                         cudaStream_t st);
lcp_status launch_sparse24_mm(const void* vals, const uint32_t* meta, const void* X, const int32_t* perm, float* Y,
                              int cout, int cin, int tokens, int B, lcp_dtype dt, cudaStream_t st);
int sparse24_tile_tokens(int cin, int tokens, int esize);   // 0: C_in too wide for one token
// the same product on the tensor cores (bf16; C_in splits from sparse24_tc_splits, 0 = unsupported)
int sparse24_tc_splits(int cout, int cin);
lcp_status launch_sparse24_tc(const __nv_bfloat16* vals, const uint32_t* meta, const __nv_bfloat16* X,
                              const int32_t* perm, float* Y, int cout, int cin, int tokens, int bshift,
                              cudaStream_t st);
lcp_status tc_error_infer(int* site, int reset);
lcp_status infer_error(int* site, int reset);

// Device error words of the tensor-core translation units: the first wait
// site that timed out since the last reset, 0 if none (cleared when `reset`).
lcp_status tc_error_gemm(int* site, int reset);
lcp_status tc_error_permute(int* site, int reset);
lcp_status tc_error_block_bwd(int* site, int reset);

constexpr int kCkptPerIter = 2;  // R then C vectors per iteration

}  // namespace lcp
