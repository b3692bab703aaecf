// C ABI of liblcp: argument validation, workspace planning and the ordering of
// the kernels of one learnable-channel-permutation step (see include/lcp.h).
//
// Step order (PermLLM summary, "Method"):
//   Sinkhorn (Method 1)  ->  W' = W P_B (Method 3)  ->  N:M mask of |W'|
//   (integration with pruning methods)  ->  y_d = W X, y_s = (M.W')(P_B^T X)
//   evaluated as (M.W' P_B^T) X  ->  token-mean cosine loss (objective)
//   ->  reverse pass to the logits with the mask held constant.

#include <cstdlib>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "lcp_internal.cuh"

namespace lcp {

static thread_local char g_msg[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

lcp_status fail(lcp_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

lcp_status ensure_smem_limit(const void* func, int bytes, const char* what) {
  struct Entry { const void* f; int dev; int bytes; };
  static std::mutex mu;
  static Entry seen[256];
  static int nseen = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < nseen; ++i)
    if (seen[i].f == func && seen[i].dev == dev && seen[i].bytes >= bytes) return LCP_OK;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "%s: cudaFuncSetAttribute: %s", what, cudaGetErrorString(e));
  }
  if (nseen < 256) seen[nseen++] = Entry{func, dev, bytes};
  return LCP_OK;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("LCP_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

lcp_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(LCP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return LCP_OK;
}

lcp_status check_pending() {
  const cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess)
    return fail(LCP_ERR_CUDA, "a CUDA error from earlier work is pending (%s); nothing was enqueued and the "
                "error is left for its owner", cudaGetErrorString(e));
  return LCP_OK;
}

namespace {

#define LCP_TRY(expr)                     \
  do {                                    \
    const lcp_status s_ = (expr);         \
    if (s_ != LCP_OK) return s_;          \
  } while (0)

constexpr int kMaxDim = 1 << 24;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

lcp_status check_arch() {
  static int cached[64];  // 0 unknown, 1 ok, 2 wrong
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  }
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= 0 && dev < 64 && cached[dev]) {
    if (cached[dev] == 1) return LCP_OK;
    return fail(LCP_ERR_ARCH, "device %d is not compute capability 10.0 (B200)", dev);
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(LCP_ERR_CUDA, "cannot query the compute capability of device %d", dev);
  }
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < 64) cached[dev] = ok ? 1 : 2;
  if (!ok) return fail(LCP_ERR_ARCH, "device %d is sm_%d%d, this library is built for sm_100a", dev, major, minor);
  return LCP_OK;
}

lcp_status check_hparams(const lcp_hparams* hp) {
  if (!hp) return fail(LCP_ERR_NULL, "hparams is NULL");
  if (hp->dtype != LCP_F32 && hp->dtype != LCP_BF16)
    return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)hp->dtype);
  const int B = hp->block;
  if (B != 32 && B != 64 && B != 128 && B != 256)
    return fail(LCP_ERR_SHAPE, "block size %d is not one of 32, 64, 128, 256", B);
  if (hp->m != 4 && hp->m != 8) return fail(LCP_ERR_SHAPE, "m = %d is not 4 or 8", hp->m);
  if (hp->n < 1 || hp->n > hp->m) return fail(LCP_ERR_SHAPE, "n = %d is not in [1, m]", hp->n);
  if (B % hp->m) return fail(LCP_ERR_SHAPE, "block %d is not a multiple of m = %d", B, hp->m);
  if (hp->iters < 1 || hp->iters > 1000)
    return fail(LCP_ERR_ARG, "iters = %d is not in [1, 1000]", hp->iters);
  if (!(hp->tau > 0.f) || !std::isfinite(hp->tau))
    return fail(LCP_ERR_ARG, "tau must be positive and finite");
  if (hp->flags & ~(LCP_FLAG_WRITE_WPRIME | LCP_FLAG_SIMT | LCP_FLAG_CACHED_DENSE | LCP_FLAG_HARD | LCP_FLAG_SCORE))
    return fail(LCP_ERR_ARG, "unknown flags 0x%x", hp->flags);
  return LCP_OK;
}

bool use_tc(const lcp_hparams& hp) {
  return hp.dtype == LCP_BF16 && !(hp.flags & LCP_FLAG_SIMT);
}

lcp_status check_layer(const lcp_layer& l, const lcp_hparams& hp, int idx) {
  if (!l.W || !l.X || !l.L || !l.P || !l.dL || !l.loss)
    return fail(LCP_ERR_NULL, "layer %d: W, X, L, P, dL and loss are required", idx);
  if ((hp.flags & LCP_FLAG_WRITE_WPRIME) && !l.Wp)
    return fail(LCP_ERR_NULL, "layer %d: LCP_FLAG_WRITE_WPRIME needs layer.Wp", idx);
  if ((hp.flags & LCP_FLAG_CACHED_DENSE) && !l.Yd)
    return fail(LCP_ERR_NULL, "layer %d: LCP_FLAG_CACHED_DENSE needs layer.Yd", idx);
  if ((hp.flags & LCP_FLAG_SCORE) && !l.S)
    return fail(LCP_ERR_NULL, "layer %d: LCP_FLAG_SCORE needs layer.S", idx);
  if ((hp.flags & LCP_FLAG_SCORE) && use_tc(hp) && hp.block > 64)
    return fail(LCP_ERR_ARG, "layer %d: LCP_FLAG_SCORE on the tensor-core path takes B <= 64 "
                "(B = %d: add LCP_FLAG_SIMT)", idx, hp.block);
  if (l.cout < 8 || l.cout % 8 || l.cout > kMaxDim)
    return fail(LCP_ERR_SHAPE, "layer %d: C_out = %d must be a positive multiple of 8", idx, l.cout);
  if (l.cin < hp.block || l.cin % hp.block || l.cin % 32 || l.cin > kMaxDim)
    return fail(LCP_ERR_SHAPE, "layer %d: C_in = %d must be a positive multiple of B = %d and of 32",
                idx, l.cin, hp.block);
  if (l.tokens < 1 || l.tokens > kMaxDim)
    return fail(LCP_ERR_SHAPE, "layer %d: T = %d must be >= 1", idx, l.tokens);
  if (use_tc(hp) && l.cin % 64)
    return fail(LCP_ERR_SHAPE,
                "layer %d: C_in = %d must be a multiple of 64 on the tensor-core path "
                "(LCP_FLAG_SIMT accepts multiples of 32)", idx, l.cin);
  const void* ptrs[] = {l.W, l.X, l.L, l.P, l.dL, l.mask, l.Wp, l.Yd, l.perm, l.S};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(LCP_ERR_ARG, "layer %d: every pointer must be 16-byte aligned", idx);
  return LCP_OK;
}


size_t esize(lcp_dtype d) { return d == LCP_F32 ? 4 : 2; }

// Workspace layout.  Each layer has a persistent region that lives for the
// whole call (its Sinkhorn checkpoint, the bf16 operand images of P, its dP
// partials and the loss counter: the Sinkhorn kernels run once over every
// layer, before and after the other stages), laid out layer after layer; one
// shared region after them holds everything else and is reused layer by layer.
struct Plan {
  size_t ckpt, img0, img1, img2, counter, dp;                                          // persistent
  size_t mask, wp, amask, at, yd, ys, stats, g, dat, da, perm, phard, shat;            // shared
  size_t persist, shared;   // bytes of this layer's persistent and shared parts
  int splits;
};

Plan make_plan(const lcp_layer& l, const lcp_hparams& hp, size_t pbase, size_t sbase) {
  const bool tc = use_tc(hp);
  const size_t B = hp.block, nb = l.cin / hp.block;
  const size_t oc = l.cout, ic = l.cin, T = l.tokens;
  const size_t es = esize(hp.dtype);
  Plan p{};
  size_t po = pbase, so = sbase;
  auto takep = [&](size_t bytes) {
    const size_t at = po;
    po += (bytes + 1023) & ~(size_t)1023;
    return at;
  };
  auto take = [&](size_t bytes) {
    const size_t at = so;
    so += (bytes + 1023) & ~(size_t)1023;
    return at;
  };
  p.splits = tc ? block_bwd_tc_splits(l.cout, l.cin, hp.block) : 1;
  p.ckpt = takep(nb * hp.iters * 2 * B * 4);
  const size_t BC = B < 64 ? 64 : B;   // tile width of the operand images
  p.img0 = takep(tc ? ic * BC * 2 : 0);
  p.img1 = takep(tc ? ic * BC * 2 : 0);
  p.img2 = takep(tc ? ic * BC * 2 : 0);
  p.counter = takep(256);
  p.dp = takep((size_t)p.splits * nb * B * B * 4);
  p.mask = take(oc * ic / 8);
  // the CUDA-core block backward (f32 or LCP_FLAG_SIMT) works on float32 W', A, dA
  const bool simt_bwd = !tc;
  p.wp = take(simt_bwd ? oc * ic * 4 : 0);
  p.amask = take(simt_bwd ? oc * ic * 4 : 0);
  p.at = take(oc * ic * es);
  p.yd = take(l.Yd ? 0 : T * oc * 4);   // the caller's Yd replaces the workspace copy
  p.ys = take(T * oc * 4);
  p.stats = take(T * 16);
  p.g = take(T * oc * es);
  p.dat = take(oc * ic * (tc ? 2 : 4));
  p.da = take(simt_bwd ? oc * ic * 4 : 0);
  const bool hard = (hp.flags & LCP_FLAG_HARD) != 0;
  p.perm = take(hard && !l.perm ? nb * B * 4 : 0);
  p.phard = take(hard && simt_bwd ? nb * B * B * 4 : 0);   // the CUDA-core products read P_hard as float32
  p.shat = take((hp.flags & LCP_FLAG_SCORE) && !tc ? oc * ic * 4 : 0);   // S_hat of the CUDA-core path
  p.persist = po - pbase;
  p.shared = so - sbase;
  return p;
}

// Every layer's plan; *total receives the workspace bytes the call needs.
std::vector<Plan> layout(const lcp_layer* layers, int nlayers, const lcp_hparams& hp, size_t* total) {
  std::vector<Plan> plans((size_t)nlayers);
  size_t persist = 0, shared = 0;
  for (int i = 0; i < nlayers; ++i) {
    const Plan q = make_plan(layers[i], hp, 0, 0);
    persist += q.persist;
    shared = std::max(shared, q.shared);
  }
  size_t pb = 0;
  for (int i = 0; i < nlayers; ++i) {
    plans[i] = make_plan(layers[i], hp, pb, persist);
    pb += plans[i].persist;
  }
  *total = persist + shared;
  return plans;
}

lcp_status validate_all(const lcp_layer* layers, int nlayers, const lcp_hparams* hp) {
  LCP_TRY(check_hparams(hp));
  if (nlayers < 0) return fail(LCP_ERR_ARG, "nlayers = %d is negative", nlayers);
  if (nlayers > 0 && !layers) return fail(LCP_ERR_NULL, "layers is NULL");
  for (int i = 0; i < nlayers; ++i) LCP_TRY(check_layer(layers[i], *hp, i));
  return LCP_OK;
}

template <typename T> T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// Loss stage of a step: the fused one-launch kernel when a token row fits its
// registers, else per-token statistics + gradient and a separate reduction.
lcp_status launch_loss(const float* Yd, const float* Ys, float* stats, void* G, lcp_dtype gdt, float* loss,
                       unsigned* counter, int cout, int tokens, int norm, cudaStream_t st) {
  if (loss_fused_supported(cout))
    return launch_loss_fused(Yd, Ys, stats, G, gdt, loss, counter, cout, tokens, norm, st);
  LCP_TRY(launch_loss_token(Yd, Ys, stats, G, gdt, cout, tokens, norm, st));
  return launch_loss_reduce(stats, loss, tokens, norm, st);
}
int loss_launches(int cout) { return loss_fused_supported(cout) ? 1 : 2; }

// The tensor-core step takes the loss from the calibration GEMM's epilogue
// unless the caller wants the float32 dense output (layer.Yd, as input or
// output) or C_out is wider than the pair kernel takes.
bool fused_loss(const lcp_layer& l, const lcp_hparams& hp) {
  return use_tc(hp) && !l.Yd && !(hp.flags & LCP_FLAG_CACHED_DENSE) && loss_pair_supported(l.cout);
}

// Stage events.  Under stream capture they become event-record nodes of the
// graph (external records), so a replayed graph still times every stage.
lcp_status record(cudaEvent_t* ev, int k, cudaStream_t st) {
  if (!ev) return LCP_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  const cudaError_t e = (cs == cudaStreamCaptureStatusActive)
                            ? cudaEventRecordWithFlags(ev[k], st, cudaEventRecordExternal)
                            : cudaEventRecord(ev[k], st);
  if (e != cudaSuccess) return fail(LCP_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(e));
  return LCP_OK;
}

// ---- one layer, CUDA-core path (float32, or bf16 with LCP_FLAG_SIMT) -------
// Options of a layer's step beyond lcp_step's: the token count the loss mean is
// taken over (norm), and, for one shard of a token-parallel step, caller-owned
// buffers for the Sinkhorn checkpoint and for dP, in which case the step stops
// before the Sinkhorn reverse pass.
struct LayerOpts {
  int norm;
  float* ckpt;
  float* dP;
};

lcp_status layer_simt(const lcp_layer& l, const lcp_hparams& hp, const Plan& p, void* ws,
                      cudaStream_t st, cudaEvent_t* ev, const LayerOpts& o) {
  const int B = hp.block, nb = l.cin / B;
  const lcp_dtype dt = hp.dtype;
  float* ckpt = o.ckpt ? o.ckpt : at<float>(ws, p.ckpt);
  uint32_t* mask = l.mask ? l.mask : at<uint32_t>(ws, p.mask);
  const bool score = (hp.flags & LCP_FLAG_SCORE) != 0, write_wp = (hp.flags & LCP_FLAG_WRITE_WPRIME) != 0;
  // W' (float32); with scores the ranked S_hat goes to layer.Wp when requested
  float* Wp = (write_wp && !score) ? l.Wp : at<float>(ws, p.wp);
  float* Shat = score ? (write_wp ? l.Wp : at<float>(ws, p.shat)) : nullptr;
  float* Am = at<float>(ws, p.amask);
  void* At = at<void>(ws, p.at);
  float* Yd = l.Yd ? l.Yd : at<float>(ws, p.yd);
  const bool cached = (hp.flags & LCP_FLAG_CACHED_DENSE) != 0;
  float* Ys = at<float>(ws, p.ys);
  float* stats = at<float>(ws, p.stats);
  void* G = at<void>(ws, p.g);
  float* dAt = at<float>(ws, p.dat);
  float* dA = at<float>(ws, p.da);
  float* dP = o.dP ? o.dP : at<float>(ws, p.dp);
  const long long ic = l.cin, oc = l.cout, BB = (long long)B * B;

  LCP_TRY(record(ev, 0, st));
  LCP_TRY(launch_sinkhorn_fwd(l.L, l.P, ckpt, nullptr, nullptr, nullptr, at<unsigned>(ws, p.counter), nb, B, hp.tau,
                              hp.iters, st));
  // the permutation every product below uses: P_hat, or its hardening (straight-through)
  const float* Pu = l.P;
  if (hp.flags & LCP_FLAG_HARD) {
    float* Ph = at<float>(ws, p.phard);
    LCP_TRY(launch_harden(l.P, l.perm ? l.perm : at<int>(ws, p.perm), Ph, nullptr, nullptr, nullptr, nb, B, st));
    Pu = Ph;
  }
  LCP_TRY(record(ev, 1, st));
  // W'_b = W_b P_b
  LCP_TRY(launch_simt_gemm({l.cout, B, B, nb, l.W, B, ic, 1, Pu, BB, B, 1, Wp, B, ic, 1, 1.f, 0.f},
                           dt, LCP_F32, LCP_F32, st));
  if (score) {   // S_hat_b = S_b P_b, ranked in place of |W'|
    LCP_TRY(launch_simt_gemm({l.cout, B, B, nb, l.S, B, ic, 1, Pu, BB, B, 1, Shat, B, ic, 1, 1.f, 0.f},
                             dt, LCP_F32, LCP_F32, st));
    LCP_TRY(launch_nm_mask(Shat, mask, l.cout, l.cin, hp.n, hp.m, LCP_F32, st));
  } else {
    LCP_TRY(launch_nm_mask(Wp, mask, l.cout, l.cin, hp.n, hp.m, LCP_F32, st));
  }
  LCP_TRY(launch_apply_mask(Wp, mask, Am, l.cout, l.cin, st));
  // At_b = A_b P_b^T
  LCP_TRY(launch_simt_gemm({l.cout, B, B, nb, Am, B, ic, 1, Pu, BB, 1, B, At, B, ic, 1, 1.f, 0.f},
                           LCP_F32, LCP_F32, dt, st));
  LCP_TRY(record(ev, 2, st));
  // Yd = X W^T, Ys = X At^T   ([T, C_out])
  if (!cached)
    LCP_TRY(launch_simt_gemm({l.tokens, l.cout, l.cin, 1, l.X, 0, ic, 1, l.W, 0, 1, ic, Yd, 0, oc, 1, 1.f, 0.f},
                             dt, dt, LCP_F32, st));
  LCP_TRY(launch_simt_gemm({l.tokens, l.cout, l.cin, 1, l.X, 0, ic, 1, At, 0, 1, ic, Ys, 0, oc, 1, 1.f, 0.f},
                           dt, dt, LCP_F32, st));
  LCP_TRY(record(ev, 3, st));
  LCP_TRY(launch_loss(Yd, Ys, stats, G, dt, l.loss, at<unsigned>(ws, p.counter), l.cout, l.tokens, o.norm, st));
  LCP_TRY(record(ev, 4, st));
  // dAt = G^T X   ([C_out, C_in], K = T)
  LCP_TRY(launch_simt_gemm({l.cout, l.cin, l.tokens, 1, G, 0, 1, oc, l.X, 0, ic, 1, dAt, 0, ic, 1, 1.f, 0.f},
                           dt, dt, LCP_F32, st));
  LCP_TRY(record(ev, 5, st));
  // dA_b = dAt_b P_b ; dW' = M . dA ; dP_b = dAt_b^T A_b + W_b^T dW'_b
  LCP_TRY(launch_simt_gemm({l.cout, B, B, nb, dAt, B, ic, 1, Pu, BB, B, 1, dA, B, ic, 1, 1.f, 0.f},
                           LCP_F32, LCP_F32, LCP_F32, st));
  LCP_TRY(launch_apply_mask(dA, mask, dA, l.cout, l.cin, st));
  LCP_TRY(launch_simt_gemm({B, B, l.cout, nb, dAt, B, 1, ic, Am, B, ic, 1, dP, BB, B, 1, 1.f, 0.f},
                           LCP_F32, LCP_F32, LCP_F32, st));
  LCP_TRY(launch_simt_gemm({B, B, l.cout, nb, l.W, B, 1, ic, dA, B, ic, 1, dP, BB, B, 1, 1.f, 1.f},
                           dt, LCP_F32, LCP_F32, st));
  LCP_TRY(record(ev, 6, st));
  if (!o.dP) LCP_TRY(launch_sinkhorn_bwd(l.L, ckpt, dP, 1, l.dL, nb, B, hp.tau, hp.iters, st));
  LCP_TRY(record(ev, 7, st));
  return LCP_OK;
}

// kernel launches per layer, not counting the loss stage (1 or 2 launches)
constexpr int kSimtLaunches = 13;
constexpr int kTcLaunches = 6;

int launches_per_layer(const lcp_layer& l, const lcp_hparams& hp) {
  const int loss = (fused_loss(l, hp) ? 1 : loss_launches(l.cout)) + ((hp.flags & LCP_FLAG_HARD) ? 1 : 0) +
                   ((hp.flags & LCP_FLAG_SCORE) ? 1 : 0);   // hardening; the score GEMM or score-mask pass
  if (!use_tc(hp)) return kSimtLaunches - ((hp.flags & LCP_FLAG_CACHED_DENSE) ? 1 : 0) + loss;
  return kTcLaunches - 2 + loss;   // the two Sinkhorn launches are shared by all layers
}

// ---- the tensor-core path (bf16 operands, float32 accumulation) -----------
// The Sinkhorn forward pass runs once over every layer's blocks, then each
// layer's middle stages run in turn, then the Sinkhorn reverse pass runs once
// over every layer (with stage events, layer 0's Sinkhorn forward stage holds
// the batched launch and the last layer's Sinkhorn reverse stage the other).

// the middle of one layer: hardening, permute + mask, calibration products +
// loss, gradient product, block backward (and, for a token shard, its dP out)
lcp_status layer_tc_middle(const lcp_layer& l, const lcp_hparams& hp, const Plan& p, void* ws,
                           cudaStream_t st, cudaEvent_t* ev, bool first, const LayerOpts& o) {
  const int B = hp.block, nb = l.cin / B;
  auto* pt_hi = at<__nv_bfloat16>(ws, p.img0);
  auto* pt_lo = at<__nv_bfloat16>(ws, p.img1);
  auto* p_hi = at<__nv_bfloat16>(ws, p.img2);
  uint32_t* mask = l.mask ? l.mask : at<uint32_t>(ws, p.mask);
  float* Wp = (hp.flags & LCP_FLAG_WRITE_WPRIME) ? l.Wp : nullptr;
  auto* At = at<__nv_bfloat16>(ws, p.at);
  float* Yd = l.Yd ? l.Yd : at<float>(ws, p.yd);
  const bool cached = (hp.flags & LCP_FLAG_CACHED_DENSE) != 0;
  float* Ys = at<float>(ws, p.ys);
  float* stats = at<float>(ws, p.stats);
  auto* G = at<__nv_bfloat16>(ws, p.g);
  auto* dAt = at<__nv_bfloat16>(ws, p.dat);
  float* dP = at<float>(ws, p.dp);
  const auto* W = static_cast<const __nv_bfloat16*>(l.W);
  const auto* X = static_cast<const __nv_bfloat16*>(l.X);

  if (!first) LCP_TRY(record(ev, 0, st));
  // with hardening the operand images are those of the hard permutation; the
  // Sinkhorn reverse pass still runs on the soft P_hat (straight-through)
  if (hp.flags & LCP_FLAG_HARD)
    LCP_TRY(launch_harden(l.P, l.perm ? l.perm : at<int>(ws, p.perm), nullptr, pt_hi, pt_lo, p_hi, nb, B, st));
  LCP_TRY(record(ev, 1, st));
  if (hp.flags & LCP_FLAG_SCORE) {
    // mask from S_hat = S P_B (exported to layer.Wp when requested), then A and At from W'
    LCP_TRY(launch_score_mask_tc(static_cast<const __nv_bfloat16*>(l.S), pt_hi, pt_lo, p_hi, mask, Wp, l.cout, l.cin,
                                 B, hp.n, hp.m, st));
    LCP_TRY(launch_permute_mask_tc(W, pt_hi, pt_lo, p_hi, mask, At, nullptr, l.cout, l.cin, B, hp.n, hp.m, true,
                                   st));
  } else {
    LCP_TRY(launch_permute_mask_tc(W, pt_hi, pt_lo, p_hi, mask, At, Wp, l.cout, l.cin, B, hp.n, hp.m, false, st));
  }
  LCP_TRY(record(ev, 2, st));
  if (fused_loss(l, hp)) {
    // the loss reduction in the calibration GEMM's epilogue: it leaves D = Y_d - Y_s
    // and Y_s in bf16 (in the Y_d slot) and per-token slot partials (in the Y_s slot)
    auto* Dq = at<__nv_bfloat16>(ws, p.yd);
    auto* Ysq = Dq + (size_t)l.tokens * l.cout;
    float* part = at<float>(ws, p.ys);
    LCP_TRY(launch_calib_loss_tc(X, W, At, Dq, Ysq, part, l.tokens, l.cout, l.cin, st));
    LCP_TRY(record(ev, 3, st));
    LCP_TRY(launch_loss_pair(Dq, Ysq, part, calib_loss_slots(l.cout), stats, G, l.loss, at<unsigned>(ws, p.counter),
                             l.cout, l.tokens, o.norm, st));
  } else {
    if (cached)   // Y_s = X At^T alone (one problem)
      LCP_TRY(launch_calib_gemm_tc(X, At, nullptr, Ys, nullptr, l.tokens, l.cout, l.cin, st));
    else
      LCP_TRY(launch_calib_gemm_tc(X, W, At, Yd, Ys, l.tokens, l.cout, l.cin, st));
    LCP_TRY(record(ev, 3, st));
    LCP_TRY(launch_loss(Yd, Ys, stats, G, LCP_BF16, l.loss, at<unsigned>(ws, p.counter), l.cout, l.tokens, o.norm,
                        st));
  }
  LCP_TRY(record(ev, 4, st));
  LCP_TRY(launch_bwd_gemm_tc(G, X, dAt, l.tokens, l.cout, l.cin, st));
  LCP_TRY(record(ev, 5, st));
  LCP_TRY(launch_block_bwd_tc(W, dAt, mask, pt_hi, pt_lo, dP, p.splits, l.cout, l.cin, B, st));
  LCP_TRY(record(ev, 6, st));
  if (o.dP) LCP_TRY(launch_sum_splits(dP, p.splits, (size_t)nb * B * B, o.dP, st));
  return LCP_OK;
}

lcp_status step_tc(const lcp_layer* layers, int n, const lcp_hparams& hp, const std::vector<Plan>& plans,
                   void* ws, cudaStream_t st, cudaEvent_t* (*evl)(void*, int), void* evctx,
                   const std::vector<LayerOpts>& opts) {
  const int B = hp.block;
  const bool shard = opts[0].dP != nullptr;
  std::vector<SkFwdLayer> fl((size_t)n);
  for (int i = 0; i < n; ++i) {
    const lcp_layer& l = layers[i];
    const Plan& p = plans[i];
    fl[i] = SkFwdLayer{l.L, l.P, opts[i].ckpt ? opts[i].ckpt : at<float>(ws, p.ckpt), at<__nv_bfloat16>(ws, p.img0),
                       at<__nv_bfloat16>(ws, p.img1), at<__nv_bfloat16>(ws, p.img2), at<unsigned>(ws, p.counter),
                       l.cin / B};
  }
  LCP_TRY(record(evl(evctx, 0), 0, st));
  LCP_TRY(launch_sinkhorn_fwd_batch(fl.data(), n, B, hp.tau, hp.iters, st));
  for (int i = 0; i < n; ++i) {
    cudaEvent_t* e = evl(evctx, i);
    LCP_TRY(layer_tc_middle(layers[i], hp, plans[i], ws, st, e, i == 0, opts[i]));
    if (i + 1 < n || shard) LCP_TRY(record(e, 7, st));
  }
  if (shard) return LCP_OK;
  std::vector<SkBwdLayer> bl((size_t)n);
  for (int i = 0; i < n; ++i) {
    const lcp_layer& l = layers[i];
    const Plan& p = plans[i];
    bl[i] = SkBwdLayer{l.L, fl[i].ckpt, at<float>(ws, p.dp), l.dL, p.splits, l.cin / B};
  }
  LCP_TRY(launch_sinkhorn_bwd_batch(bl.data(), n, B, hp.tau, hp.iters, st));
  return record(evl(evctx, n - 1), 7, st);
}

// total_tokens > 0, dP and ckpt: one token shard of a token-parallel step (see lcp_step_shard)
lcp_status step_impl(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, void* ws,
                     size_t ws_bytes, cudaStream_t st, cudaEvent_t* ev, int nev, int total_tokens = 0,
                     float* const* dP = nullptr, float* const* ckpt = nullptr) {
  LCP_TRY(validate_all(layers, nlayers, hp));
  if (total_tokens > 0) {
    if (!dP || !ckpt) return fail(LCP_ERR_NULL, "dP and ckpt are required");
    for (int i = 0; i < nlayers; ++i) {
      if (layers[i].tokens > total_tokens)
        return fail(LCP_ERR_SHAPE, "layer %d: its %d tokens exceed total_tokens = %d", i, layers[i].tokens,
                    total_tokens);
      if (!dP[i] || !ckpt[i]) return fail(LCP_ERR_NULL, "layer %d: dP and ckpt are required", i);
      if (!aligned16(dP[i]) || !aligned16(ckpt[i]))
        return fail(LCP_ERR_ARG, "layer %d: dP and ckpt must be 16-byte aligned", i);
    }
  }
  if (nev != 0 && nev != LCP_TIMED_EVENTS && !(nlayers > 0 && nev == LCP_TIMED_EVENTS * nlayers))
    return fail(LCP_ERR_ARG, "n_events must be 0, %d or %d x nlayers", LCP_TIMED_EVENTS, LCP_TIMED_EVENTS);
  if (nev && !ev) return fail(LCP_ERR_NULL, "events is NULL");
  if (nlayers == 0) return LCP_OK;
  size_t need = 0;
  const std::vector<Plan> plans = layout(layers, nlayers, *hp, &need);
  if (!ws) return fail(LCP_ERR_NULL, "workspace is NULL");
  if (((uintptr_t)ws & 255u) != 0) return fail(LCP_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(LCP_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  struct EvCtx { cudaEvent_t* ev; int nev, nlayers; } ectx{ev, nev, nlayers};
  auto evl = [](void* c, int i) -> cudaEvent_t* {
    const EvCtx& x = *static_cast<const EvCtx*>(c);
    if (!x.nev) return nullptr;
    if (x.nev == LCP_TIMED_EVENTS * x.nlayers) return x.ev + (size_t)LCP_TIMED_EVENTS * i;
    return i == 0 ? x.ev : nullptr;
  };
  std::vector<LayerOpts> opts((size_t)nlayers);
  for (int i = 0; i < nlayers; ++i)
    opts[i] = LayerOpts{total_tokens > 0 ? total_tokens : layers[i].tokens, total_tokens > 0 ? ckpt[i] : nullptr,
                        total_tokens > 0 ? dP[i] : nullptr};
  if (use_tc(*hp)) return step_tc(layers, nlayers, *hp, plans, ws, st, evl, &ectx, opts);
  for (int i = 0; i < nlayers; ++i) LCP_TRY(layer_simt(layers[i], *hp, plans[i], ws, st, evl(&ectx, i), opts[i]));
  return LCP_OK;
}

}  // namespace
}  // namespace lcp

using namespace lcp;

extern "C" {

int lcp_abi_version(void) { return LCP_ABI_VERSION; }

const char* lcp_last_error(void) { return g_msg; }

const char* lcp_status_string(lcp_status s) {
  switch (s) {
    case LCP_OK: return "LCP_OK";
    case LCP_ERR_NULL: return "LCP_ERR_NULL: a required pointer is NULL";
    case LCP_ERR_SHAPE: return "LCP_ERR_SHAPE: unsupported shape";
    case LCP_ERR_DTYPE: return "LCP_ERR_DTYPE: unknown dtype";
    case LCP_ERR_WORKSPACE: return "LCP_ERR_WORKSPACE: workspace too small or misaligned";
    case LCP_ERR_ARCH: return "LCP_ERR_ARCH: device is not sm_100 (B200)";
    case LCP_ERR_CUDA: return "LCP_ERR_CUDA: a CUDA call failed";
    case LCP_ERR_ARG: return "LCP_ERR_ARG: invalid argument";
  }
  return "unknown lcp_status";
}

lcp_status lcp_workspace_size(const lcp_layer* layers, int nlayers, const lcp_hparams* hp,
                              size_t* bytes) {
  if (!bytes) return fail(LCP_ERR_NULL, "bytes is NULL");
  LCP_TRY(validate_all(layers, nlayers, hp));
  size_t need = 0;
  layout(layers, nlayers, *hp, &need);
  *bytes = need;
  return LCP_OK;
}

lcp_status lcp_step_launches(const lcp_layer* layers, int nlayers, const lcp_hparams* hp,
                             int* launches) {
  if (!launches) return fail(LCP_ERR_NULL, "launches is NULL");
  LCP_TRY(validate_all(layers, nlayers, hp));
  int n = 0;
  for (int i = 0; i < nlayers; ++i) n += launches_per_layer(layers[i], *hp);
  if (use_tc(*hp) && nlayers > 0) n += 2 * ((nlayers + kSkMaxLayers - 1) / kSkMaxLayers);   // batched Sinkhorn
  *launches = n;
  return LCP_OK;
}

lcp_status lcp_step(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, void* ws,
                    size_t ws_bytes, cudaStream_t stream) {
  return step_impl(layers, nlayers, hp, ws, ws_bytes, stream, nullptr, 0);
}

lcp_status lcp_step_timed(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, void* ws,
                          size_t ws_bytes, cudaStream_t stream, cudaEvent_t* events,
                          int n_events) {
  return step_impl(layers, nlayers, hp, ws, ws_bytes, stream, events, n_events);
}

lcp_status lcp_step_shard(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, int total_tokens,
                          float* const* dP, float* const* ckpt, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (total_tokens < 1 || total_tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "total_tokens = %d", total_tokens);
  return step_impl(layers, nlayers, hp, ws, ws_bytes, stream, nullptr, 0, total_tokens, dP, ckpt);
}

lcp_status lcp_adamw(float* L, const float* dL, float* m, float* v, long long n, const lcp_adamw_params* opt,
                     int t, cudaStream_t stream) {
  if (!L || !dL || !m || !v || !opt) return fail(LCP_ERR_NULL, "L, dL, m, v and opt are required");
  if (n < 0 || n % 4) return fail(LCP_ERR_SHAPE, "n = %lld must be a non-negative multiple of 4", n);
  if (t < 1) return fail(LCP_ERR_ARG, "t = %d must be >= 1", t);
  if (!(opt->lr >= 0.0) || !(opt->beta1 >= 0.0 && opt->beta1 < 1.0) || !(opt->beta2 >= 0.0 && opt->beta2 < 1.0) ||
      !(opt->eps > 0.0) || !(opt->weight_decay >= 0.0) || !std::isfinite(opt->lr))
    return fail(LCP_ERR_ARG, "AdamW parameters out of range");
  if (!aligned16(L) || !aligned16(dL) || !aligned16(m) || !aligned16(v))
    return fail(LCP_ERR_ARG, "every pointer must be 16-byte aligned");
  if (n == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_adamw(L, dL, m, v, n, opt->lr, opt->beta1, opt->beta2, opt->eps, opt->weight_decay, t, stream);
}

lcp_status lcp_train(const lcp_layer* layers, int nlayers, const lcp_hparams* hp, const lcp_adamw_params* opt,
                     const lcp_adamw_state* state, int first, int count, int total, float tau_start, float tau_end,
                     void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!hp || !opt) return fail(LCP_ERR_NULL, "hp and opt are required");
  if (nlayers > 0 && !state) return fail(LCP_ERR_NULL, "state is required");
  if (!(opt->lr >= 0.0) || !(opt->beta1 >= 0.0 && opt->beta1 < 1.0) || !(opt->beta2 >= 0.0 && opt->beta2 < 1.0) ||
      !(opt->eps > 0.0) || !(opt->weight_decay >= 0.0) || !std::isfinite(opt->lr))
    return fail(LCP_ERR_ARG, "AdamW parameters out of range");
  if (total < 1 || first < 0 || count < 0 || first + count > total)
    return fail(LCP_ERR_ARG, "steps [%d, %d) outside a run of %d", first, first + count, total);
  if (!(tau_start > 0.f) || !(tau_end > 0.f) || !std::isfinite(tau_start) || !std::isfinite(tau_end))
    return fail(LCP_ERR_ARG, "temperatures must be positive and finite");
  for (int i = 0; i < nlayers; ++i) {
    if (!state[i].m || !state[i].v) return fail(LCP_ERR_NULL, "layer %d: AdamW moments are required", i);
    if (!aligned16(state[i].m) || !aligned16(state[i].v))
      return fail(LCP_ERR_ARG, "layer %d: AdamW moments must be 16-byte aligned", i);
  }
  lcp_hparams h = *hp;
  for (int s = first; s < first + count; ++s) {
    const double frac = total > 1 ? (double)s / (double)(total - 1) : 0.0;
    h.tau = (float)((double)tau_start + ((double)tau_end - (double)tau_start) * frac);
    LCP_TRY(step_impl(layers, nlayers, &h, ws, ws_bytes, stream, nullptr, 0));
    for (int i = 0; i < nlayers; ++i) {
      const long long n = (long long)layers[i].cin * h.block;
      LCP_TRY(launch_adamw(const_cast<float*>(layers[i].L), layers[i].dL, state[i].m, state[i].v, n, opt->lr,
                           opt->beta1, opt->beta2, opt->eps, opt->weight_decay, s + 1, stream));
    }
  }
  return LCP_OK;
}

lcp_status lcp_sinkhorn_fwd(const float* L, float* P, float* ckpt, int nblocks, int B, float tau,
                            int iters, cudaStream_t stream) {
  if (!L || !P) return fail(LCP_ERR_NULL, "L and P are required");
  if (B != 32 && B != 64 && B != 128 && B != 256)
    return fail(LCP_ERR_SHAPE, "block size %d is not one of 32, 64, 128, 256", B);
  if (nblocks < 0 || nblocks > kMaxDim) return fail(LCP_ERR_SHAPE, "nblocks = %d", nblocks);
  if (iters < 1 || iters > 1000) return fail(LCP_ERR_ARG, "iters = %d is not in [1, 1000]", iters);
  if (!(tau > 0.f) || !std::isfinite(tau)) return fail(LCP_ERR_ARG, "tau must be positive and finite");
  if (nblocks == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_sinkhorn_fwd(L, P, ckpt, nullptr, nullptr, nullptr, nullptr, nblocks, B, tau, iters, stream);
}

lcp_status lcp_sinkhorn_bwd(const float* L, const float* ckpt, const float* dP, int dP_splits,
                            float* dL, int nblocks, int B, float tau, int iters,
                            cudaStream_t stream) {
  if (!L || !ckpt || !dP || !dL) return fail(LCP_ERR_NULL, "L, ckpt, dP and dL are required");
  if (B != 32 && B != 64 && B != 128 && B != 256)
    return fail(LCP_ERR_SHAPE, "block size %d is not one of 32, 64, 128, 256", B);
  if (nblocks < 0 || nblocks > kMaxDim) return fail(LCP_ERR_SHAPE, "nblocks = %d", nblocks);
  if (dP_splits < 1 || dP_splits > 64) return fail(LCP_ERR_ARG, "dP_splits = %d is not in [1, 64]", dP_splits);
  if (iters < 1 || iters > 1000) return fail(LCP_ERR_ARG, "iters = %d is not in [1, 1000]", iters);
  if (!(tau > 0.f) || !std::isfinite(tau)) return fail(LCP_ERR_ARG, "tau must be positive and finite");
  if (nblocks == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_sinkhorn_bwd(L, ckpt, dP, dP_splits, dL, nblocks, B, tau, iters, stream);
}

lcp_status lcp_permute_weight(const void* W, const float* P, float* Wp, int cout, int cin, int B,
                              lcp_dtype dtype, cudaStream_t stream) {
  if (!W || !P || !Wp) return fail(LCP_ERR_NULL, "W, P and Wp are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  if (B != 32 && B != 64 && B != 128 && B != 256)
    return fail(LCP_ERR_SHAPE, "block size %d is not one of 32, 64, 128, 256", B);
  if (cout < 0 || cin < 0 || cin % B || cout > kMaxDim || cin > kMaxDim)
    return fail(LCP_ERR_SHAPE, "C_out = %d, C_in = %d (C_in must be a multiple of B)", cout, cin);
  if (cout == 0 || cin == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  const long long ic = cin, BB = (long long)B * B;
  return launch_simt_gemm({cout, B, B, cin / B, W, B, ic, 1, P, BB, B, 1, Wp, B, ic, 1, 1.f, 0.f},
                          dtype, LCP_F32, LCP_F32, stream);
}

lcp_status lcp_score(const void* W, const void* X, void* S, float* stats, int cout, int cin, int tokens, int kind,
                     lcp_dtype dtype, cudaStream_t stream) {
  if (!W || !X || !S || !stats) return fail(LCP_ERR_NULL, "W, X, S and stats are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  if (kind != LCP_SCORE_MAGNITUDE && kind != LCP_SCORE_WANDA && kind != LCP_SCORE_RIA)
    return fail(LCP_ERR_ARG, "unknown score kind %d", kind);
  if (cout < 0 || cin < 0 || tokens < 1 || cout > kMaxDim || cin > kMaxDim || tokens > kMaxDim)
    return fail(LCP_ERR_SHAPE, "C_out = %d, C_in = %d, T = %d", cout, cin, tokens);
  if (cout == 0 || cin == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_score(W, X, S, stats, cout, cin, tokens, kind, dtype, stream);
}

lcp_status lcp_harden(const float* P_hat, int32_t* perm, float* P_hard, int nblocks, int B, cudaStream_t stream) {
  if (!P_hat || !perm) return fail(LCP_ERR_NULL, "P_hat and perm are required");
  if (B != 32 && B != 64 && B != 128 && B != 256)
    return fail(LCP_ERR_SHAPE, "block size %d is not one of 32, 64, 128, 256", B);
  if (nblocks < 0 || nblocks > kMaxDim) return fail(LCP_ERR_SHAPE, "nblocks = %d", nblocks);
  if (!aligned16(P_hat) || (P_hard && !aligned16(P_hard)))
    return fail(LCP_ERR_ARG, "P_hat and P_hard must be 16-byte aligned");
  if (nblocks == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_harden(P_hat, perm, P_hard, nullptr, nullptr, nullptr, nblocks, B, stream);
}

static lcp_status check_infer_shape(int cout, int cin, int B, bool need_block) {
  if (cout < 1 || cout > kMaxDim) return fail(LCP_ERR_SHAPE, "C_out = %d", cout);
  if (cin < 32 || cin % 32 || cin > kMaxDim) return fail(LCP_ERR_SHAPE, "C_in = %d must be a positive multiple of 32", cin);
  if (need_block) {
    if (B != 32 && B != 64 && B != 128 && B != 256)
      return fail(LCP_ERR_SHAPE, "block size %d is not one of 32, 64, 128, 256", B);
    if (cin % B) return fail(LCP_ERR_SHAPE, "C_in = %d is not a multiple of B = %d", cin, B);
  }
  return LCP_OK;
}

lcp_status lcp_pack24(const void* W, const int32_t* perm, const uint32_t* mask, void* values, uint32_t* meta,
                      int cout, int cin, int B, lcp_dtype dtype, cudaStream_t stream) {
  if (!W || !mask || !values || !meta) return fail(LCP_ERR_NULL, "W, mask, values and meta are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  if (!perm && B == 0) B = 32;                       // no permutation: any block width of the columns
  LCP_TRY(check_infer_shape(cout, cin, B, true));
  if (!aligned16(W) || !aligned16(mask) || !aligned16(values) || !aligned16(meta) || (perm && !aligned16(perm)))
    return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_pack24(W, perm, mask, values, meta, cout, cin, B, dtype, stream);
}

lcp_status lcp_gather(const void* X, const int32_t* perm, void* Xp, int tokens, int cin, int B, lcp_dtype dtype,
                      cudaStream_t stream) {
  if (!X || !perm || !Xp) return fail(LCP_ERR_NULL, "X, perm and Xp are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  LCP_TRY(check_infer_shape(1, cin, B, true));
  if (tokens < 0 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d", tokens);
  if (X == Xp) return fail(LCP_ERR_ARG, "the gather is out of place: X and Xp must differ");
  if (!aligned16(X) || !aligned16(Xp) || !aligned16(perm)) return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  if (tokens == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_gather(X, perm, Xp, tokens, cin, B, dtype, stream);
}

lcp_status lcp_sparse24_mm(const void* values, const uint32_t* meta, const void* X, const int32_t* perm, float* Y,
                           int cout, int cin, int tokens, int B, lcp_dtype dtype, cudaStream_t stream) {
  if (!values || !meta || !X || !Y) return fail(LCP_ERR_NULL, "values, meta, X and Y are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  LCP_TRY(check_infer_shape(cout, cin, B, perm != nullptr));
  if (tokens < 0 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d", tokens);
  if (sparse24_tile_tokens(cin, tokens < 1 ? 1 : tokens, dtype == LCP_F32 ? 4 : 2) == 0)
    return fail(LCP_ERR_SHAPE, "C_in = %d: one token's inputs do not fit in shared memory", cin);
  if (!aligned16(values) || !aligned16(meta) || !aligned16(X) || (perm && !aligned16(perm)) || !aligned16(Y))
    return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  if (tokens == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_sparse24_mm(values, meta, X, perm, Y, cout, cin, tokens, B, dtype, stream);
}

lcp_status nm_mask(const void* Wp, uint32_t* mask_bits, int rows, int cols, int n, int m,
                   lcp_dtype dtype, cudaStream_t stream) {
  if (!Wp || !mask_bits) return fail(LCP_ERR_NULL, "Wp and mask_bits are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  if (m != 4 && m != 8) return fail(LCP_ERR_SHAPE, "m = %d is not 4 or 8", m);
  if (n < 1 || n > m) return fail(LCP_ERR_SHAPE, "n = %d is not in [1, m]", n);
  if (rows < 0 || cols < 0 || cols % 32 || rows > kMaxDim || cols > kMaxDim)
    return fail(LCP_ERR_SHAPE, "rows = %d, cols = %d (cols must be a multiple of 32)", rows, cols);
  if (!aligned16(Wp) || !aligned16(mask_bits)) return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  if (rows == 0 || cols == 0) return LCP_OK;
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_nm_mask(Wp, mask_bits, rows, cols, n, m, dtype, stream);
}

lcp_status lcp_calib_gemm(const void* X, const void* W, const void* At, float* Yd, float* Ys, int tokens,
                          int cout, int cin, cudaStream_t stream) {
  if (!X || !W || !Yd) return fail(LCP_ERR_NULL, "X, W and Yd are required");
  if ((At == nullptr) != (Ys == nullptr)) return fail(LCP_ERR_NULL, "At and Ys go together");
  if (cout < 8 || cout % 8 || cout > kMaxDim) return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8", cout);
  if (cin < 8 || cin % 8 || cin > kMaxDim) return fail(LCP_ERR_SHAPE, "C_in = %d must be a positive multiple of 8", cin);
  if (tokens < 1 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  const void* ptrs[] = {X, W, At, Yd, Ys};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_calib_gemm_tc(static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(W),
                              static_cast<const __nv_bfloat16*>(At), Yd, Ys, tokens, cout, cin, stream);
}

lcp_status lcp_calib_gemm_loss(const void* X, const void* W, const void* At, void* D, void* Ys, float* partials,
                               int tokens, int cout, int cin, cudaStream_t stream) {
  if (!X || !W || !At || !D || !Ys || !partials) return fail(LCP_ERR_NULL, "X, W, At, D, Ys and partials are required");
  if (cout < 8 || cout % 8 || cout > kMaxDim) return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8", cout);
  if (cin < 8 || cin % 8 || cin > kMaxDim) return fail(LCP_ERR_SHAPE, "C_in = %d must be a positive multiple of 8", cin);
  if (tokens < 1 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  const void* ptrs[] = {X, W, At, D, Ys, partials};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_calib_loss_tc(static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(W),
                              static_cast<const __nv_bfloat16*>(At), static_cast<__nv_bfloat16*>(D),
                              static_cast<__nv_bfloat16*>(Ys), partials, tokens, cout, cin, stream);
}

lcp_status lcp_loss_pair(const void* D, const void* Ys, const float* partials, float* loss, float* stats, void* G,
                         unsigned* counter, int cout, int tokens, cudaStream_t stream) {
  if (!D || !Ys || !partials || !loss || !stats || !G || !counter)
    return fail(LCP_ERR_NULL, "D, Ys, partials, loss, stats, G and counter are required");
  if (cout < 8 || cout % 8 || !loss_pair_supported(cout))
    return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8, at most 16384", cout);
  if (tokens < 1 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  if (!aligned16(D) || !aligned16(Ys) || !aligned16(partials) || !aligned16(stats) || !aligned16(G))
    return fail(LCP_ERR_ARG, "D, Ys, partials, stats and G must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_loss_pair(static_cast<const __nv_bfloat16*>(D), static_cast<const __nv_bfloat16*>(Ys), partials,
                          calib_loss_slots(cout), stats, static_cast<__nv_bfloat16*>(G), loss, counter, cout, tokens,
                          tokens, stream);
}

lcp_status lcp_grad_gemm(const void* G, const void* X, void* dAt, int tokens, int cout, int cin,
                         cudaStream_t stream) {
  if (!G || !X || !dAt) return fail(LCP_ERR_NULL, "G, X and dAt are required");
  if (cout < 8 || cout % 8 || cout > kMaxDim) return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8", cout);
  if (cin < 8 || cin % 8 || cin > kMaxDim) return fail(LCP_ERR_SHAPE, "C_in = %d must be a positive multiple of 8", cin);
  if (tokens < 1 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  if (!aligned16(G) || !aligned16(X) || !aligned16(dAt)) return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_bwd_gemm_tc(static_cast<const __nv_bfloat16*>(G), static_cast<const __nv_bfloat16*>(X),
                            static_cast<__nv_bfloat16*>(dAt), tokens, cout, cin, stream);
}

lcp_status lcp_loss_fwd(const float* Yd, const float* Ys, float* loss, float* stats, int cout,
                        int tokens, cudaStream_t stream) {
  if (!Yd || !Ys || !loss || !stats) return fail(LCP_ERR_NULL, "Yd, Ys, loss and stats are required");
  if (cout < 8 || cout % 8 || cout > kMaxDim) return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8", cout);
  if (tokens < 1 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  if (!aligned16(Yd) || !aligned16(Ys) || !aligned16(stats)) return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  LCP_TRY(launch_loss_token(Yd, Ys, stats, nullptr, LCP_F32, cout, tokens, tokens, stream));
  return launch_loss_reduce(stats, loss, tokens, tokens, stream);
}

lcp_status lcp_loss_bwd(const float* Yd, const float* Ys, const float* stats, void* G, int cout,
                        int tokens, lcp_dtype dtype, cudaStream_t stream) {
  if (!Yd || !Ys || !stats || !G) return fail(LCP_ERR_NULL, "Yd, Ys, stats and G are required");
  if (dtype != LCP_F32 && dtype != LCP_BF16) return fail(LCP_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  if (cout < 8 || cout % 8 || cout > kMaxDim) return fail(LCP_ERR_SHAPE, "C_out = %d must be a positive multiple of 8", cout);
  if (tokens < 1 || tokens > kMaxDim) return fail(LCP_ERR_SHAPE, "T = %d must be >= 1", tokens);
  if (!aligned16(Yd) || !aligned16(Ys) || !aligned16(stats) || !aligned16(G))
    return fail(LCP_ERR_ARG, "pointers must be 16-byte aligned");
  LCP_TRY(check_arch());
  LCP_TRY(check_pending());
  return launch_loss_grad(Yd, Ys, stats, G, dtype, cout, tokens, tokens, stream);
}

}  // extern "C"

extern "C" lcp_status lcp_device_error(int* site, int reset) {
  using namespace lcp;
  if (!site) return fail(LCP_ERR_NULL, "site is NULL");
  lcp_status (*const readers[])(int*, int) = {tc_error_gemm, tc_error_permute, tc_error_block_bwd, harden_error,
                                               infer_error, tc_error_infer};
  int first = 0;
  for (auto rd : readers) {
    int v = 0;
    const lcp_status s = rd(&v, reset);
    if (s != LCP_OK) return s;
    if (!first) first = v;
  }
  *site = first;
  return LCP_OK;
}
