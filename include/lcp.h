/*
 * lcp.h -- C ABI of the B200 (sm_100a) learnable-channel-permutation hot path.
 *
 * The method: PermLLM, "Learnable Channel Permutation for N:M Sparse Large
 * Language Models" (summary page of arXiv 2510.10136), section "Method".
 * For one linear layer W (C_out x C_in) with calibration activations X
 * (the pages' C_in x T matrix, stored here token-major as [T, C_in]):
 *
 *   P_b   = S_L(L_b / tau)                 block-wise log-domain Sinkhorn
 *   W'    = W * blockdiag(P_1..P_nb)       block-wise permutation
 *   M     = N:M magnitude mask of |W'|     (groups of M consecutive columns)
 *   y_s   = (M (.) W') (P_B^T X),  y_d = W X
 *   loss  = mean over tokens of 1 - cos(y_d, y_s)
 *   dL    = d loss / d L                   (mask held constant: straight-through)
 *
 * Conventions for every entry point:
 *  - Every pointer is a DEVICE pointer owned by the caller, unless stated.
 *    The library never allocates, frees or synchronises; it enqueues kernels
 *    on `stream` and returns.  Results are ready when the stream is.
 *  - Arguments are validated on the host before any launch.  On error nothing
 *    is enqueued and a status other than LCP_OK is returned; lcp_last_error()
 *    then holds a message for the calling thread.
 *  - A launch failure is reported as LCP_ERR_CUDA (message kept likewise).
 *    A CUDA error that earlier work left pending (cudaPeekAtLastError) is
 *    also reported as LCP_ERR_CUDA, before anything is enqueued, and is left
 *    pending for its owner (the library never clears another caller's error).
 *  - Matrices are row-major and densely packed:
 *      W  [C_out, C_in]    X  [T, C_in]      (dtype of the call: f32 or bf16)
 *      L, P, dL  [C_in/B, B, B] float32; P_b[i][j] moves source channel bB+i
 *                to permuted slot bB+j; row sums run over j.
 *      mask bits [C_out, C_in/32] uint32: bit (j % 32) of word j/32 of row o
 *                is set when W'[o][j] is kept.
 *      Yd, Ys, G [T, C_out] (token-major outputs).
 *  - Shapes: B in {32, 64, 128, 256}; C_in % B == 0 and C_in % 32 == 0;
 *    M in {4, 8} and 1 <= N <= M (N == M prunes nothing); B % M == 0;
 *    C_out >= 8 and C_out % 8 == 0; T >= 1 (any value, ragged tails allowed);
 *    1 <= iters <= 1000; tau > 0 and finite.
 *  - The device must be compute capability 10.0 (B200); otherwise LCP_ERR_ARCH.
 */
#ifndef LCP_H
#define LCP_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LCP_ABI_VERSION 4

#if defined(__GNUC__)
#define LCP_API __attribute__((visibility("default")))
#else
#define LCP_API
#endif

typedef enum {
  LCP_OK = 0,
  LCP_ERR_NULL = 1,       /* a required pointer is NULL                         */
  LCP_ERR_SHAPE = 2,      /* a size violates the shape rules above              */
  LCP_ERR_DTYPE = 3,      /* unknown dtype                                      */
  LCP_ERR_WORKSPACE = 4,  /* workspace too small or misaligned (256 B)          */
  LCP_ERR_ARCH = 5,       /* current device is not compute capability 10.0      */
  LCP_ERR_CUDA = 6,       /* a CUDA call or kernel launch failed                */
  LCP_ERR_ARG = 7         /* any other invalid argument (tau, iters, flags ...) */
} lcp_status;

typedef enum { LCP_F32 = 0, LCP_BF16 = 1 } lcp_dtype;

/* lcp_hparams.flags */
#define LCP_FLAG_WRITE_WPRIME 0x1u  /* also write W' (float32, [C_out, C_in]) to layer.Wp */
#define LCP_FLAG_SIMT         0x2u  /* run every contraction on the CUDA-core (SIMT) kernels
                                       instead of the tensor-core kernels (bf16 only; the
                                       f32 dtype always uses SIMT kernels)              */
#define LCP_FLAG_HARD         0x8u  /* harden P before use ("Method" 2): every block of the
                                       Sinkhorn output is replaced by the permutation
                                       maximising Tr(P^T P_hat) (lcp_harden); the backward
                                       pass is straight-through, dP_hat = dP.  layer.P
                                       still returns the soft P_hat                    */
#define LCP_FLAG_SCORE        0x10u /* take the N:M mask from S_hat = S P_B, S = layer.S an
                                       importance matrix ("integration with pruning
                                       methods"; see lcp_score), instead of |W'|.  With
                                       LCP_FLAG_WRITE_WPRIME, layer.Wp receives S_hat (the
                                       matrix the mask ranks).  Tensor-core path: B <= 64 */
#define LCP_FLAG_CACHED_DENSE 0x4u  /* read the dense output Y_d = X W^T from layer.Yd
                                       instead of computing it: the dense output depends
                                       on neither L nor P, so a loop over one calibration
                                       batch computes it once (the library's extension of
                                       the objective; the pages evaluate it per step)  */

typedef struct {
  int block;        /* B, the permutation block size                                */
  int n, m;         /* N:M pattern: keep n of every m consecutive input channels     */
  int iters;        /* Sinkhorn iterations (one = row then column normalisation)     */
  float tau;        /* temperature: Z_0 = L / tau                                    */
  lcp_dtype dtype;  /* element type of W and X (and of the bf16 intermediates)       */
  unsigned flags;   /* LCP_FLAG_*                                                    */
} lcp_hparams;

typedef struct {
  const void* W;    /* in  [C_out, C_in] dtype                                        */
  const void* X;    /* in  [T, C_in] dtype; may alias another layer's X               */
  const float* L;   /* in  [C_in/B, B, B] logits                                      */
  float* P;         /* out [C_in/B, B, B] soft permutation (required)                 */
  float* dL;        /* out [C_in/B, B, B] d loss / d L (required)                     */
  float* loss;      /* out one float: the layer's mean cosine loss (required)         */
  uint32_t* mask;   /* out [C_out, C_in/32] mask bits (optional, NULL = not returned) */
  float* Wp;        /* out [C_out, C_in] W' (only with LCP_FLAG_WRITE_WPRIME)         */
  int cout, cin, tokens;
  float* Yd;        /* [T, C_out] float32 dense output X W^T, optional: with
                       LCP_FLAG_CACHED_DENSE an input (required; it must hold X W^T for
                       this W and X, e.g. written by an earlier step), otherwise, when
                       non-NULL, an output the step fills                                */
  int32_t* perm;    /* out [C_in/B, B] optional: with LCP_FLAG_HARD, perm[b][i] = the
                       column of block b that row i is sent to                          */
  const void* S;    /* in  [C_out, C_in] dtype importance scores (with LCP_FLAG_SCORE)  */
} lcp_layer;

/* Bytes of workspace lcp_step needs for these layers (the layers run one after
 * another on the stream, so the workspace is the maximum over layers).
 * Cites: the whole of the "Method" section (every intermediate of the step). */
LCP_API lcp_status lcp_workspace_size(const lcp_layer* layers, int nlayers, const lcp_hparams* hp,
                              size_t* bytes);

/* One forward + backward step for each of `nlayers` independent layers
 * (each with its own W, L, P, dL and loss; X may be shared).  Cites: the whole
 * "Method" section and its "optimization objective" (the loss above and its
 * gradient to L).  `ws` is a device
 * buffer of at least lcp_workspace_size() bytes, 256-byte aligned, owned by the
 * caller and not used concurrently by another call.  nlayers == 0 is a no-op. */
LCP_API lcp_status lcp_step(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, void* ws,
                    size_t ws_bytes, cudaStream_t stream);

/* As lcp_step, and records events[k] (caller-created cudaEvent_t) on `stream`
 * at the stage boundaries of the FIRST layer: 0 before the Sinkhorn forward,
 * then after each stage (Sinkhorn fwd, permute+mask, calibration GEMM, loss,
 * backward GEMM, block backward, Sinkhorn bwd).  n_events must be 0,
 * LCP_TIMED_EVENTS, or LCP_TIMED_EVENTS * nlayers: then layer i records
 * events[LCP_TIMED_EVENTS * i + k] the same way.  Used to time each kernel
 * inside a real step. */
#define LCP_TIMED_EVENTS 8
LCP_API lcp_status lcp_step_timed(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, void* ws,
                          size_t ws_bytes, cudaStream_t stream, cudaEvent_t* events, int n_events);

/* One token shard of a token-parallel step (the loss is a mean over tokens, so
 * the calibration batch of T tokens can be split across GPUs: "Implementation
 * details" trains 7B on 4 GPUs and 13B on 8).  As lcp_step on this call's
 * layers, whose X hold this shard's layer.tokens tokens, except that
 *  - the mean over tokens is taken over `total_tokens` (the whole batch):
 *    layer.loss receives (1/total_tokens) * sum over the shard of (1 - c_t),
 *    and every gradient is scaled the same way, so the shards' losses and
 *    gradients add up to the whole batch's;
 *  - the step stops before the Sinkhorn reverse pass: dP[i] (float32
 *    [C_in/B, B, B], caller-owned) receives d loss / d P of layer i for the
 *    shard and ckpt[i] (float32 [C_in/B, iters, 2, B]) the Sinkhorn
 *    checkpoint of lcp_sinkhorn_fwd; layer.dL is not written.
 * Summing dP[i] and the losses over the shards (an all-reduce) and calling
 * lcp_sinkhorn_bwd(L, ckpt, dP_sum, 1, dL, ...) gives the whole batch's dL.
 * Every layer.tokens <= total_tokens; dP and ckpt 16-byte aligned. */
LCP_API lcp_status lcp_step_shard(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, int total_tokens,
                                  float* const* dP, float* const* ckpt, void* ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* Number of kernel launches lcp_step enqueues for these layers. */
LCP_API lcp_status lcp_step_launches(const lcp_layer* layers, int nlayers, const lcp_hparams* hp,
                             int* launches);

/* Block-wise log-domain Sinkhorn ("Method", 1: S_0 = exp, S_i = T_c(T_r(S_{i-1})),
 * P = S_L(L / tau); the blog page's section 2.2 fixes rows before columns).
 * L, P: [nblocks, B, B].  ckpt (optional, may be NULL): float32
 * [nblocks, iters, 2, B]; entry [b][k][0][i] is the row log-normaliser R_i and
 * [b][k][1][j] the column log-normaliser C_j after iteration k+1, so that the
 * iterate is Z = L/tau - R_i - C_j.  lcp_sinkhorn_bwd needs it. */
LCP_API lcp_status lcp_sinkhorn_fwd(const float* L, float* P, float* ckpt, int nblocks, int B, float tau,
                            int iters, cudaStream_t stream);

/* Reverse pass of lcp_sinkhorn_fwd ("Method", 1: the gradient flows back
 * through every row and column normalisation): dL = d loss / d L given
 * d loss / d P.
 * dP holds dP_splits partial gradients [dP_splits, nblocks, B, B] that are
 * summed in index order (deterministic).  ckpt from lcp_sinkhorn_fwd with the
 * same L, tau and iters. */
LCP_API lcp_status lcp_sinkhorn_bwd(const float* L, const float* ckpt, const float* dP, int dP_splits,
                            float* dL, int nblocks, int B, float tau, int iters,
                            cudaStream_t stream);

/* AdamW on the logits (summary page, "Implementation details": AdamW, learning
 * rate 1e-3 or 5e-3; the pages fix no betas, epsilon or decay: the usual
 * defaults are 0.9, 0.999, 1e-8, 0.01).  Decoupled weight decay, bias-corrected
 * moments, t = the 1-based step count:
 *   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2
 *   L = L (1 - lr wd) - lr / (1 - b1^t) * m / (sqrt(v / (1 - b2^t)) + eps)     */
typedef struct {
  double lr, beta1, beta2, eps, weight_decay;   /* host values; 1 - beta is formed in double */
} lcp_adamw_params;

/* Per-layer AdamW state: first and second moments, float32 [C_in/B, B, B]
 * each, zero before the first step, owned by the caller. */
typedef struct {
  float* m;
  float* v;
} lcp_adamw_state;

/* One AdamW update ("Implementation details": AdamW on the logits) of n float32
 * parameters in place (g = dL; n a multiple of 4;
 * every pointer 16-byte aligned).  t >= 1. */
LCP_API lcp_status lcp_adamw(float* L, const float* dL, float* m, float* v, long long n,
                             const lcp_adamw_params* opt, int t, cudaStream_t stream);

/* The training loop of one or more layers ("Implementation details": AdamW,
 * temperature decreasing linearly from 1 to 0.1): steps s = first, ...,
 * first + count - 1 of a run of `total` steps, each one lcp_step at
 * tau_s = tau_start + (tau_end - tau_start) * s / (total - 1) (tau_start when
 * total = 1) followed by the AdamW update of every layer's L in place (layer.L
 * is written: the const in lcp_layer does not hold for this call) with
 * t = s + 1.  hp->tau is ignored.  Enqueues everything on `stream` (capturable
 * in a CUDA graph); after the call, dL and loss hold step first + count - 1. */
LCP_API lcp_status lcp_train(const lcp_layer* layers, int nlayers, const lcp_hparams* hp,
                             const lcp_adamw_params* opt, const lcp_adamw_state* state, int first,
                             int count, int total, float tau_start, float tau_end, void* ws,
                             size_t ws_bytes, cudaStream_t stream);

/* Importance scores of W for the mask ("integration with existing pruning
 * methods"; the pages name Wanda and RIA without defining them, so their
 * published definitions are used), with ||X_j|| the 2-norm of input channel j
 * over the T tokens:
 *   LCP_SCORE_MAGNITUDE  S_ij = |W_ij|
 *   LCP_SCORE_WANDA      S_ij = |W_ij| ||X_j||
 *   LCP_SCORE_RIA        S_ij = (|W_ij| / sum_k |W_kj| + |W_ij| / sum_k |W_ik|) ||X_j||^(1/2)
 * W [C_out, C_in], X [T, C_in] and S [C_out, C_in] in `dtype` (S rounded to it);
 * stats: float32 scratch of 2 C_in + C_out values owned by the caller. */
#define LCP_SCORE_MAGNITUDE 0
#define LCP_SCORE_WANDA     1
#define LCP_SCORE_RIA       2
LCP_API lcp_status lcp_score(const void* W, const void* X, void* S, float* stats, int cout, int cin, int tokens,
                             int kind, lcp_dtype dtype, cudaStream_t stream);

/* Hardening ("Method" 2: P = argmax over permutations of Tr(P^T P_hat), the
 * Hungarian algorithm): for each of `nblocks` B x B blocks of P_hat (float32,
 * [nblocks, B, B]) the permutation maximising sum_i P_hat[i, perm[i]].  B = 32
 * and 64: solved exactly (shortest augmenting paths, float32 potentials).
 * B = 128 and 256: an epsilon-scaling auction on P_hat quantised to 2^28..2^29
 * levels of each block's range, whose result is within B (max - min) 2^-27 of
 * the maximum (max, min: the block's extreme values).  perm: int32
 * [nblocks, B] (required); P_hard: float32 [nblocks, B, B] 0/1 matrices
 * (optional, NULL = not written).  B in {32, 64, 128, 256}.  When several
 * permutations attain the maximum, the result is one of them (deterministic). */
LCP_API lcp_status lcp_harden(const float* P_hat, int32_t* perm, float* P_hard, int nblocks, int B,
                              cudaStream_t stream);

/* W' = W * blockdiag(P) ("Method", 3: W_hat_B = W P_B).  W [cout, cin] in
 * `dtype`, P [cin/B, B, B], Wp [cout, cin] float32. */
LCP_API lcp_status lcp_permute_weight(const void* W, const float* P, float* Wp, int cout, int cin, int B,
                              lcp_dtype dtype, cudaStream_t stream);

/* N:M magnitude mask (blog page section 2.1; "integration with existing
 * pruning methods": the best N of each group of M consecutive columns).
 * Keeps the n largest |Wp| of every m consecutive columns of each row; equal
 * magnitudes keep the lower column (+0 and -0 are equal).  Wp [rows, cols] in
 * `dtype`, compared in that precision; mask_bits [rows, cols/32].
 * cols % 32 == 0, m in {4, 8}, 1 <= n <= m.  NaN inputs give an unspecified mask. */
LCP_API lcp_status nm_mask(const void* Wp, uint32_t* mask_bits, int rows, int cols, int n, int m,
                   lcp_dtype dtype, cudaStream_t stream);

/* Token-averaged cosine loss ("optimization objective": 1 - y.y~ / (|y||y~|),
 * denominator clamped at 1e-8).  Yd, Ys [tokens, cout] float32; loss: one
 * float; stats: caller-provided scratch of 4*tokens floats that receives, per
 * token, <y_d,y_s>, |y_d|^2, |y_s|^2 and cos (lcp_loss_bwd reads it). */
LCP_API lcp_status lcp_loss_fwd(const float* Yd, const float* Ys, float* loss, float* stats, int cout,
                        int tokens, cudaStream_t stream);

/* G = d loss / d Ys for the loss above ("optimization objective": the gradient
 * of 1 - cos(y_d, y_s) with respect to y_s), written in `dtype` ([tokens, cout]);
 * stats from lcp_loss_fwd on the same Yd, Ys. */
LCP_API lcp_status lcp_loss_bwd(const float* Yd, const float* Ys, const float* stats, void* G, int cout,
                        int tokens, lcp_dtype dtype, cudaStream_t stream);

/* Calibration outputs on the tensor cores ("optimization objective": the dense
 * output y = W X and the sparse output y~ = At X with At = (M.W') P_B^T):
 * Yd = X W^T and, when At and Ys are given, Ys = X At^T.  X [T, C_in],
 * W and At [C_out, C_in] bf16; Yd, Ys [T, C_out] float32 (float32
 * accumulation).  C_out and C_in multiples of 8, T >= 1. */
LCP_API lcp_status lcp_calib_gemm(const void* X, const void* W, const void* At, float* Yd, float* Ys,
                                  int tokens, int cout, int cin, cudaStream_t stream);

/* The calibration outputs with the cosine-loss reduction in the GEMM's epilogue
 * ("optimization objective": the loss needs, per token, <y, y~>, |y|^2 and
 * |y~|^2, and its gradient G a combination of y and y~): y_d = X W^T and
 * y_s = X At^T come out of one tensor-core pass (float32 accumulation), and
 * instead of the two float32 outputs the call writes
 *   partials [T, ceil(C_out / 64), 4] float32: for token t and 64-channel
 *            slot s, (sum y_d y_s, sum y_d^2, sum y_s^2, 0) over channels
 *            [64 s, 64 s + 64) (a fixed summation order);
 *   D = Y_d - Y_s and Ys = Y_s, bf16 [T, C_out] (the difference is formed
 *            in float32 before rounding).
 * X [T, C_in], W and At [C_out, C_in] bf16.  C_out and C_in multiples of 8,
 * T >= 1.  lcp_step uses it for bf16 layers without layer.Yd. */
LCP_API lcp_status lcp_calib_gemm_loss(const void* X, const void* W, const void* At, void* D, void* Ys,
                                       float* partials, int tokens, int cout, int cin, cudaStream_t stream);

/* ("optimization objective") The token-averaged cosine loss and G = d loss / d Ys
 * (bf16 [T, C_out]) from
 * lcp_calib_gemm_loss's outputs: the slot partials of each token, summed in a
 * fixed order, give c_t = <y_d,y_s> / max(|y_d||y_s|, 1e-8) and the loss
 * (1/T) sum_t (1 - c_t); G_t = -(1/T)(y_d / (|y_d||y_s|) - c_t y_s / |y_s|^2)
 * with y_d = D + Ys and y_s = Ys.  stats [T, 4] receives what lcp_loss_fwd
 * writes there.  counter: one uint32 of device memory, zero before the call
 * and left zero by it (not shared by calls that may overlap).  C_out <= 16384. */
LCP_API lcp_status lcp_loss_pair(const void* D, const void* Ys, const float* partials, float* loss, float* stats,
                                 void* G, unsigned* counter, int cout, int tokens, cudaStream_t stream);

/* Weight gradient of the sparse output on the tensor cores ("optimization
 * objective" with "Method", 3: y_s = At x, so d loss / d At = G^T X): dAt = G^T X with
 * G [T, C_out] and X [T, C_in] bf16 and dAt [C_out, C_in] bf16 (float32
 * accumulation over the T tokens). */
LCP_API lcp_status lcp_grad_gemm(const void* G, const void* X, void* dAt, int tokens, int cout,
                                 int cin, cudaStream_t stream);

/* ---- Inference side ("Effect on inference acceleration": the deployed layer
 * permutes its input channels at run time and multiplies by the 2:4 sparse
 * weight).  The deployed weight is A = M.(W P_B) for a hard block permutation
 * P_B and a 2:4 mask M, in permuted column order, kept compressed:
 *   values [C_out, C_in/2] in `dtype`: the two kept entries of every group of
 *          four columns, in column order;
 *   meta   [C_out, C_in/32] uint32: group g's 4-bit field at bits 4 (g % 8) of
 *          word g / 8, first kept position (0..3) in the low two bits, second
 *          (larger) in the high two.
 * perm [C_in/B, B] int32 is the hardening's permutation (lcp_harden: row i of
 * block b goes to column perm[b][i]); the input side is x_pi = P_B^T x, i.e.
 * x_pi[bB + perm[b][i]] = x[bB + i].  A perm entry outside [0, B) is skipped
 * and recorded in lcp_device_error (302); a perm that is not a permutation of
 * its block gives unspecified (in-bounds) results. */

/* ("Effect on inference acceleration": the 2:4 weight stored for sparse
 * tensor cores) Compressed weight from W [C_out, C_in] (original column order, `dtype`), perm
 * (NULL: identity, B then only needs to divide C_in; 0 is accepted) and the
 * mask bits of M [C_out, C_in/32] in permuted order (as lcp_step writes them
 * for LCP_FLAG_HARD).  A group without exactly two kept bits is written as
 * positions (0, 1) with zero values and recorded in lcp_device_error (301); a
 * repeated perm entry is recorded as 303.  C_in % 32 == 0, C_in % B == 0,
 * B in {32, 64, 128, 256}. */
LCP_API lcp_status lcp_pack24(const void* W, const int32_t* perm, const uint32_t* mask, void* values,
                              uint32_t* meta, int cout, int cin, int B, lcp_dtype dtype, cudaStream_t stream);

/* The input gather (the pages' run-time channel permutation): Xp = x_pi for
 * every token, X and Xp [T, C_in] in `dtype`, out of place. */
LCP_API lcp_status lcp_gather(const void* X, const int32_t* perm, void* Xp, int tokens, int cin, int B,
                              lcp_dtype dtype, cudaStream_t stream);

/* ("Effect on inference acceleration": the permuted, 2:4-sparse layer at run
 * time) The deployed product Y = x_pi A^T for every token: X [T, C_in] in `dtype`
 * (original channel order when perm is given, already permuted when perm is
 * NULL), values / meta as above, Y [T, C_out] float32 (float32 accumulation).
 * Built for decode-sized T (tiles of up to 16 tokens; larger T runs tile by
 * tile, re-streaming the weight).  One token's inputs must fit in 200 KB of
 * shared memory: C_in <= 91008 (bf16) / 48160 (float32), else LCP_ERR_SHAPE. */
LCP_API lcp_status lcp_sparse24_mm(const void* values, const uint32_t* meta, const void* X, const int32_t* perm,
                                   float* Y, int cout, int cin, int tokens, int B, lcp_dtype dtype,
                                   cudaStream_t stream);

/* Diagnostic (synchronous: reads a device word).  Every wait inside the
 * tensor-core kernels is bounded; a wait that expires records its site here
 * (0 = none) and the kernel returns early with incomplete results.  With
 * reset != 0 the word is cleared after reading. */
LCP_API lcp_status lcp_device_error(int* site, int reset);

/* Self-test (synchronous; allocates and frees 4 bytes of device memory).  One
 * thread waits on a barrier phase that nothing completes, with the time limit
 * every wait of the tensor-core kernels uses (2 s); the wait must give up,
 * record its site and return.  On success *site is 901 and the CUDA context
 * stays usable.  Not for use while other work of the library is in flight. */
LCP_API lcp_status lcp_selftest_bounded_wait(int* site);

/* Allocation-free variant of lcp_loss_fwd (the paper has no counterpart; this
 * is a library convenience).  Same loss ("optimization objective"), same arguments minus the scratch
 * buffer: the per-token scratch lives in a static __device__ array of
 * LCP_STATIC_MAX_TOKENS * 4 floats (1 MiB) that every GPU loading the library
 * holds until exit.  For callers that cannot allocate device memory: embedders
 * whose device memory belongs to another allocator or is reserved up front
 * under a fixed budget, and latency-critical pipelines in which cudaMalloc's
 * implicit device synchronisation would stall work on other streams.
 * - tokens > LCP_STATIC_MAX_TOKENS is rejected with LCP_ERR_SHAPE.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and caches it with the
 *   ID of the current CUDA context; make that first call before any stream
 *   capture begins.  After cudaDeviceReset (any change of context) the next
 *   call repeats the lookup.
 * - All calls share the array (each call overwrites all of it that it reads,
 *   so nothing must be cleared); calls that overlap on the GPU race on it.
 * - Allocates and frees nothing, calls no allocating routine. */
#define LCP_STATIC_MAX_TOKENS 65536
LCP_API lcp_status lcp_loss_fwd_static(const float* Yd, const float* Ys, float* loss, int cout,
                                       int tokens, cudaStream_t stream);

LCP_API const char* lcp_status_string(lcp_status s);
/* Message of the last failed call made by this thread ("" if none). */
LCP_API const char* lcp_last_error(void);
LCP_API int lcp_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LCP_H */
