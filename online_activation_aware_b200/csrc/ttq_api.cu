// C ABI of the TTQ hot path (declared in include/ttq.h): argument validation, workspace
// layout and the launch sequence of each entry point. Every check happens before any
// launch, so an argument error leaves the stream untouched.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "ttq.h"
#include "ttq_internal.h"

namespace ttq {

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}
}  // namespace

bool current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  if (ctx == nullptr) {
    // no context bound to this thread yet: make the runtime bind the current device's
    // primary context
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return false;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  }
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace ttq

namespace {

__device__ unsigned g_ttq_error_word;

constexpr int kMaxDevices = 64;
constexpr int32_t kMaxDecodeRequests = 4096;  // batched decode: requests per call
std::atomic<uint64_t> g_wait_ns{2000000000ull};
cudaEvent_t g_trace[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
bool g_trace_on = false;

inline cudaError_t trace(int i, cudaStream_t stream) {
  return g_trace_on ? cudaEventRecord(g_trace[i], stream) : cudaSuccess;
}

struct DeviceInfo {
  unsigned long long ctx_id = 0;  // context the cached addresses belong to (0: none yet)
  unsigned* err_word = nullptr;
  int num_sms = 148;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
thread_local DeviceInfo t_dev;  // this host thread's copy of the entry it last looked up

// Per-device facts of the current context: the device address of the error word (module
// symbols move when a context is rebuilt, e.g. after cudaDeviceReset, or differ in a
// caller's own driver-API context, so the cache is keyed on the context's id) and the SM
// count. The table is shared by every host thread and guarded by a mutex; the caller gets
// a pointer to its own thread's copy.
ttq_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTQ_ERR_CUDA;
  unsigned long long ctx = 0;
  if (!ttq::current_context_id(&ctx)) return TTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ttq_error_word) != cudaSuccess || p == nullptr) return TTQ_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TTQ_ERR_CUDA;
    di.err_word = static_cast<unsigned*>(p);
    di.num_sms = sms;
    di.ctx_id = ctx;
  }
  t_dev = di;
  *out = &t_dev;
  return TTQ_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

ttq_status check_qg(int32_t q, int32_t g, int64_t d) {
  if (q < 2 || q > 4) return TTQ_ERR_UNSUPPORTED;
  if (g != 32 && g != 64 && g != 128) return TTQ_ERR_UNSUPPORTED;
  if (d % g != 0) return TTQ_ERR_INVALID_ARG;
  return TTQ_OK;
}

ttq_status check_stats_args(float alpha, float lambda, int32_t p) {
  if (p != 1 && p != 2) return TTQ_ERR_UNSUPPORTED;
  if (!std::isfinite(alpha) || !std::isfinite(lambda) || alpha < 0.f || lambda < 0.f)
    return TTQ_ERR_INVALID_ARG;
  if (alpha > 0.f && !(lambda > 0.f)) return TTQ_ERR_INVALID_ARG;
  return TTQ_OK;
}

ttq_status check_dims(int64_t T, int64_t d, int64_t d_out) {
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (T < 1 || d < 1 || d_out < 1) return TTQ_ERR_INVALID_ARG;
  if (T > lim || d > lim || d_out > lim || T * d > (int64_t(1) << 40) || d_out * d > (int64_t(1) << 40))
    return TTQ_ERR_INVALID_ARG;
  if (d % 8 != 0) return TTQ_ERR_INVALID_ARG;
  return TTQ_OK;
}

ttq_status check_cfg(const ttq_config* cfg, int64_t d) {
  if (!cfg) return TTQ_ERR_INVALID_ARG;
  ttq_status st = check_qg(cfg->q, cfg->g, d);
  if (st != TTQ_OK) return st;
  st = check_stats_args(cfg->alpha, cfg->lambda, cfg->p);
  if (st != TTQ_OK) return st;
  if (cfg->r < 0 || cfg->r > 64) return TTQ_ERR_UNSUPPORTED;
  if (cfg->r % 8 != 0) return TTQ_ERR_UNSUPPORTED;
  return TTQ_OK;
}

struct WsLayout {
  size_t stats_off, stats_bytes;
  size_t xf_off, xf_bytes;
  size_t u_off, u_bytes;
  size_t part_off, part_bytes;
  size_t dec_off, dec_bytes;  // CUDA-core decode (b <= 2): x' and its unit sums
  size_t total;
  ttq::GemmPlan plan;
};

WsLayout ws_layout(int64_t T, int64_t d, int64_t d_out, int r, int q, int g, int num_sms) {
  WsLayout L{};
  L.stats_off = 0;
  // the statistic reduces on chip, except when it rides on the low-rank pass over X
  // (r > 0): then its per-token-block column sums take [ceil(T / 64), d] fp32
  L.stats_bytes = (d_out > 0 && r > 0 && T > ttq::lowrank_small_tokens())
                      ? round256(ttq::lowrank_stats_bytes(T, d))
                      : 0;
  L.xf_off = L.stats_off + L.stats_bytes;
  L.xf_bytes = d_out > 0 ? round256(static_cast<size_t>(T) * static_cast<size_t>(d) * 2) : 0;
  L.u_off = L.xf_off + L.xf_bytes;
  // U (bf16 [T, 64]) and the fp32 partial sums of its K splits
  L.u_bytes = (d_out > 0 && r > 0)
                  ? round256(static_cast<size_t>(T) * 64 * 2) + round256(ttq::lowrank_partial_bytes(T, d, r, num_sms))
                  : 0;
  L.part_off = L.u_off + L.u_bytes;
  if (d_out > 0) {
    L.plan = ttq::gemm_plan(T, d, d_out, q, g, num_sms);
    L.part_bytes = round256(ttq::gemm_partial_bytes(L.plan, T, d_out));
  }
  L.dec_off = L.part_off + L.part_bytes;
  if (d_out > 0 && ttq::decode_gemv_ok(T, d)) L.dec_bytes = round256(ttq::decode_gemv_ws_bytes(T, d));
  L.total = L.dec_off + L.dec_bytes;
  return L;
}

ttq::DevErr dev_err(const DeviceInfo* di) { return ttq::DevErr{di->err_word, g_wait_ns.load()}; }

thread_local int g_last_cuda_error = 0;

inline ttq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TTQ_OK;
  g_last_cuda_error = static_cast<int>(e);
  return TTQ_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t ttq_codes_words(int64_t d_out, int64_t d, int32_t q) {
  if (d_out < 0 || d < 0 || d % 32 != 0 || q < 2 || q > 4) return 0;
  return static_cast<size_t>(d_out) * static_cast<size_t>(d / 32) * static_cast<size_t>(q);
}

ttq_status ttq_workspace_size(int64_t T, int64_t d, int64_t d_out, const ttq_config* cfg,
                              size_t* bytes) {
  if (!bytes) return TTQ_ERR_INVALID_ARG;
  if (d_out < 0) return TTQ_ERR_INVALID_ARG;
  ttq_status st = check_dims(T, d, d_out > 0 ? d_out : 1);
  if (st != TTQ_OK) return st;
  const int r = cfg ? cfg->r : 0;
  if (cfg) {
    st = check_cfg(cfg, d);
    if (st != TTQ_OK) return st;
  }
  // the statistic's row split and the split-K plan depend on the SM count of the current
  // device (148 when no device can be queried)
  int num_sms = 148;
  DeviceInfo* di = nullptr;
  if (device_info(&di) == TTQ_OK) num_sms = di->num_sms;
  const int q = cfg ? cfg->q : 4;
  const int g = cfg ? cfg->g : 128;
  *bytes = ws_layout(T, d, d_out, r, q, g, num_sms).total;
  return TTQ_OK;
}

ttq_status ttq_workspace_folded_offset(int64_t T, int64_t d, int64_t d_out, const ttq_config* cfg,
                                       size_t* offset) {
  if (!offset || !cfg) return TTQ_ERR_INVALID_ARG;
  ttq_status st = check_dims(T, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  int num_sms = 148;
  DeviceInfo* di = nullptr;
  if (device_info(&di) == TTQ_OK) num_sms = di->num_sms;
  *offset = ws_layout(T, d, d_out, cfg->r, cfg->q, cfg->g, num_sms).xf_off;
  return TTQ_OK;
}

ttq_status ttq_act_stats(const void* X_bf16, int64_t T, int64_t d, int64_t ld_x, float alpha,
                         float lambda, int32_t p, float* s, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  ttq_status st = check_dims(T, d, 1);
  if (st != TTQ_OK) return st;
  if (ld_x < d || ld_x % 8 != 0) return TTQ_ERR_INVALID_ARG;
  st = check_stats_args(alpha, lambda, p);
  if (st != TTQ_OK) return st;
  if (!X_bf16 || !s) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(s) || (ws && !aligned16(ws))) return TTQ_ERR_MISALIGNED;
  (void)ws_bytes;  // the statistic reduces on chip and needs no workspace
  DeviceInfo* di = nullptr;
  ttq_status dst = device_info(&di);
  if (dst != TTQ_OK) return dst;
  return cuda_status(ttq::launch_act_stats(X_bf16, T, d, ld_x, alpha, lambda, p, s, di->num_sms, dev_err(di), stream));
}

ttq_status ttq_requant(const void* W_bf16, int64_t d_out, int64_t d, const float* s, int32_t q,
                       int32_t g, uint32_t* codes, void* scale_f16, void* zero_f16,
                       cudaStream_t stream) {
  ttq_status st = check_dims(1, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_qg(q, g, d);
  if (st != TTQ_OK) return st;
  if (!W_bf16 || !s || !codes || !scale_f16 || !zero_f16) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(W_bf16) || !aligned16(s) || !aligned16(codes) || !aligned16(scale_f16) ||
      !aligned16(zero_f16))
    return TTQ_ERR_MISALIGNED;
  return cuda_status(ttq::launch_requant(W_bf16, d_out, d, s, q, g, codes, scale_f16, zero_f16, false, stream));
}

ttq_status ttq_requant_batched(const void* W_bf16, int64_t d_out, int64_t d, const float* s, int32_t prompts,
                               int32_t q, int32_t g, uint32_t* codes, void* scale_f16, void* zero_f16,
                               cudaStream_t stream) {
  ttq_status st = check_dims(1, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_qg(q, g, d);
  if (st != TTQ_OK) return st;
  if (prompts < 1 || prompts > ttq::kRequantMaxPrompts) return TTQ_ERR_UNSUPPORTED;
  if (!W_bf16 || !s || !codes || !scale_f16 || !zero_f16) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(W_bf16) || !aligned16(s) || !aligned16(codes) || !aligned16(scale_f16) ||
      !aligned16(zero_f16))
    return TTQ_ERR_MISALIGNED;
  return cuda_status(
      ttq::launch_requant_batched(W_bf16, d_out, d, s, prompts, q, g, codes, scale_f16, zero_f16, stream));
}

static ttq_status check_lowrank(const ttq_config* cfg, const void* A, const void* B) {
  if (cfg->r > 0) {
    if (!A || !B) return TTQ_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B)) return TTQ_ERR_MISALIGNED;
  } else if (A || B) {
    return TTQ_ERR_INVALID_ARG;
  }
  return TTQ_OK;
}

ttq_status ttq_linear_prefill(const void* X_bf16, int64_t T, int64_t d, const void* W_bf16,
                              int64_t d_out, const void* A_bf16, const void* B_bf16,
                              const ttq_config* cfg, float* s, uint32_t* codes, void* scale_f16,
                              void* zero_f16, void* Y_bf16, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
  ttq_status st = check_dims(T, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  st = check_lowrank(cfg, A_bf16, B_bf16);
  if (st != TTQ_OK) return st;
  if (!X_bf16 || !W_bf16 || !s || !codes || !scale_f16 || !zero_f16 || !Y_bf16)
    return TTQ_ERR_INVALID_ARG;
  if (!ws) return TTQ_ERR_WORKSPACE;
  if (!aligned16(X_bf16) || !aligned16(W_bf16) || !aligned16(s) || !aligned16(codes) ||
      !aligned16(scale_f16) || !aligned16(zero_f16) || !aligned16(Y_bf16) || !aligned16(ws))
    return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  st = device_info(&di);
  if (st != TTQ_OK) return st;
  const WsLayout L = ws_layout(T, d, d_out, cfg->r, cfg->q, cfg->g, di->num_sms);
  if (ws_bytes < L.total) return TTQ_ERR_WORKSPACE;
  auto* base = static_cast<uint8_t*>(ws);
  void* Xf = base + L.xf_off;
  void* U = cfg->r > 0 ? base + L.u_off : nullptr;
  float* upart = cfg->r > 0 ? reinterpret_cast<float*>(base + L.u_off + round256(static_cast<size_t>(T) * 64 * 2))
                            : nullptr;
  float* gpart = L.part_bytes ? reinterpret_cast<float*>(base + L.part_off) : nullptr;

  // statistic -> (X A^T) -> fold of X fused with the requant of W -> projection; with a
  // low-rank side path the statistic comes out of the same pass over X as X A^T
  const bool stats_in_lowrank = L.stats_bytes > 0;
  cudaError_t e = trace(0, stream);
  if (e == cudaSuccess && !stats_in_lowrank)
    e = ttq::launch_act_stats(X_bf16, T, d, d, cfg->alpha, cfg->lambda, cfg->p, s, di->num_sms, dev_err(di), stream);
  if (e == cudaSuccess) e = trace(1, stream);
  if (e == cudaSuccess && stats_in_lowrank)
    e = ttq::launch_lowrank_u_stats(X_bf16, T, d, A_bf16, cfg->r, U, upart,
                                    reinterpret_cast<float*>(base + L.stats_off), cfg->alpha, cfg->lambda, cfg->p, s,
                                    di->num_sms, dev_err(di), stream);
  else if (e == cudaSuccess && cfg->r > 0)
    e = ttq::launch_lowrank_u(X_bf16, T, d, A_bf16, cfg->r, U, upart, di->num_sms, dev_err(di), stream);
  if (e == cudaSuccess) e = trace(2, stream);
  if (e == cudaSuccess)
    e = ttq::launch_fold_requant(X_bf16, T, Xf, W_bf16, d_out, d, s, cfg->q, cfg->g, codes, scale_f16, zero_f16,
                                 stream);
  if (e == cudaSuccess) e = trace(3, stream);
  if (e == cudaSuccess) {
    ttq::GemmArgs ga{Xf, codes, scale_f16, zero_f16, U, B_bf16, cfg->r, T, d, d_out, cfg->q, cfg->g,
                     Y_bf16, gpart};
    e = ttq::launch_gemm_mainloop(ga, L.plan, dev_err(di), stream);
    if (e == cudaSuccess) e = trace(4, stream);
    if (e == cudaSuccess) e = ttq::launch_gemm_reduce(ga, L.plan, stream);
  }
  if (e == cudaSuccess) e = trace(5, stream);
  return cuda_status(e);
}

ttq_status ttq_linear_decode(const void* X_bf16, int64_t b, int64_t d, int64_t d_out,
                             const float* s, const uint32_t* codes, const void* scale_f16,
                             const void* zero_f16, const void* A_bf16, const void* B_bf16,
                             const ttq_config* cfg, void* Y_bf16, void* ws, size_t ws_bytes,
                             cudaStream_t stream) {
  ttq_status st = check_dims(b, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  st = check_lowrank(cfg, A_bf16, B_bf16);
  if (st != TTQ_OK) return st;
  if (!X_bf16 || !s || !codes || !scale_f16 || !zero_f16 || !Y_bf16) return TTQ_ERR_INVALID_ARG;
  if (!ws) return TTQ_ERR_WORKSPACE;
  if (!aligned16(X_bf16) || !aligned16(s) || !aligned16(codes) || !aligned16(scale_f16) ||
      !aligned16(zero_f16) || !aligned16(Y_bf16) || !aligned16(ws))
    return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  st = device_info(&di);
  if (st != TTQ_OK) return st;
  const WsLayout L = ws_layout(b, d, d_out, cfg->r, cfg->q, cfg->g, di->num_sms);
  if (ws_bytes < L.total) return TTQ_ERR_WORKSPACE;
  auto* base = static_cast<uint8_t*>(ws);
  void* Xf = base + L.xf_off;
  void* U = cfg->r > 0 ? base + L.u_off : nullptr;
  float* upart = cfg->r > 0 ? reinterpret_cast<float*>(base + L.u_off + round256(static_cast<size_t>(b) * 64 * 2))
                            : nullptr;
  float* gpart = L.part_bytes ? reinterpret_cast<float*>(base + L.part_off) : nullptr;
  if (L.dec_bytes > 0) {
    // few tokens: the CUDA-core GEMV streams the codes once; its prep kernel also forms
    // U = X A^T for the low-rank side path
    ttq::DecodeArgs da{X_bf16, s, codes, scale_f16, zero_f16, U, B_bf16, cfg->r, b, d, d_out, cfg->q, cfg->g, Y_bf16,
                       1, dev_err(di)};
    da.A = cfg->r > 0 ? A_bf16 : nullptr;
    return cuda_status(ttq::launch_decode_gemv(da, base + L.dec_off, stream));
  }
  cudaError_t e = ttq::launch_fold(X_bf16, b, d, d, s, Xf, stream);
  if (e == cudaSuccess && cfg->r > 0)
    e = ttq::launch_lowrank_u(X_bf16, b, d, A_bf16, cfg->r, U, upart, di->num_sms, dev_err(di), stream);
  if (e == cudaSuccess) {
    ttq::GemmArgs ga{Xf, codes, scale_f16, zero_f16, U, B_bf16, cfg->r, b, d, d_out, cfg->q, cfg->g,
                     Y_bf16, gpart};
    e = ttq::launch_gemm(ga, L.plan, dev_err(di), stream);
  }
  return cuda_status(e);
}

// Workspace of a batched prefill: statistic partials (largest prompt), X' and U (with its
// K-split partials) for all prompts' tokens, and the split-K partials of the largest
// per-prompt projection (used when the prompts cannot share one grouped launch).
struct BatchLayout {
  size_t stats_off, xf_off, u_off, upart_off, gpart_off, total;
  int64_t tokens;
  bool grouped;
  ttq::GemmPlan plan;  // the grouped plan (tokens of all prompts), when grouped
};

static BatchLayout batch_layout(const int64_t* T, int32_t prompts, int64_t d, int64_t d_out, const ttq_config* cfg,
                                int num_sms) {
  BatchLayout L{};
  size_t stats = 0, gpart = 0;
  int64_t tokens = 0;
  for (int32_t p = 0; p < prompts; ++p) {
    tokens += T[p];
    const ttq::GemmPlan pp = ttq::gemm_plan(T[p], d, d_out, cfg->q, cfg->g, num_sms);
    gpart = std::max(gpart, ttq::gemm_partial_bytes(pp, T[p], d_out));
  }
  L.tokens = tokens;
  L.plan = ttq::gemm_plan(tokens, d, d_out, cfg->q, cfg->g, num_sms);
  L.grouped = L.plan.pair && prompts <= ttq::kGemmMaxGroups;
  if (L.grouped) {  // one launch over every prompt's tiles, no split-K
    L.plan.kb_per_split = L.plan.nkb;
    L.plan.ksplit = 1;
    gpart = 0;
  }
  L.stats_off = 0;
  L.xf_off = round256(stats);
  L.u_off = L.xf_off + round256(static_cast<size_t>(tokens) * static_cast<size_t>(d) * 2);
  const size_t ub = cfg->r > 0 ? round256(static_cast<size_t>(tokens) * 64 * 2) : 0;
  L.upart_off = L.u_off + ub;
  const size_t upb = cfg->r > 0 ? round256(ttq::lowrank_partial_bytes(tokens, d, cfg->r, num_sms)) : 0;
  L.gpart_off = L.upart_off + upb;
  L.total = L.gpart_off + round256(gpart);
  return L;
}

static ttq_status check_batch(const int64_t* T, int32_t prompts, int64_t d, int64_t d_out) {
  if (!T) return TTQ_ERR_INVALID_ARG;
  if (prompts < 1 || prompts > ttq::kRequantMaxPrompts) return TTQ_ERR_UNSUPPORTED;
  int64_t tokens = 0;
  for (int32_t p = 0; p < prompts; ++p) {
    if (T[p] < 1) return TTQ_ERR_INVALID_ARG;
    tokens += T[p];
  }
  return check_dims(tokens, d, d_out);
}

ttq_status ttq_prefill_batched_workspace_size(const int64_t* T, int32_t prompts, int64_t d, int64_t d_out,
                                              const ttq_config* cfg, size_t* bytes) {
  if (!bytes) return TTQ_ERR_INVALID_ARG;
  ttq_status st = check_batch(T, prompts, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  int num_sms = 148;
  DeviceInfo* di = nullptr;
  if (device_info(&di) == TTQ_OK) num_sms = di->num_sms;
  *bytes = batch_layout(T, prompts, d, d_out, cfg, num_sms).total;
  return TTQ_OK;
}

ttq_status ttq_linear_prefill_batched(const void* X_bf16, const int64_t* T, int32_t prompts, int64_t d,
                                      const void* W_bf16, int64_t d_out, const void* A_bf16, const void* B_bf16,
                                      const ttq_config* cfg, float* s, uint32_t* codes, void* scale_f16,
                                      void* zero_f16, void* Y_bf16, void* ws, size_t ws_bytes, cudaStream_t stream) {
  ttq_status st = check_batch(T, prompts, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  st = check_lowrank(cfg, A_bf16, B_bf16);
  if (st != TTQ_OK) return st;
  if (!X_bf16 || !W_bf16 || !s || !codes || !scale_f16 || !zero_f16 || !Y_bf16) return TTQ_ERR_INVALID_ARG;
  if (!ws) return TTQ_ERR_WORKSPACE;
  if (!aligned16(X_bf16) || !aligned16(W_bf16) || !aligned16(s) || !aligned16(codes) || !aligned16(scale_f16) ||
      !aligned16(zero_f16) || !aligned16(Y_bf16) || !aligned16(ws))
    return TTQ_ERR_MISALIGNED;
  const int64_t words = static_cast<int64_t>(ttq_codes_words(d_out, d, cfg->q));
  const int64_t metas = d_out * (d / cfg->g);
  if (d_out % 8 || words % 4 || metas % 8) return TTQ_ERR_MISALIGNED;  // every prompt's outputs 16-byte aligned
  DeviceInfo* di = nullptr;
  st = device_info(&di);
  if (st != TTQ_OK) return st;
  const BatchLayout L = batch_layout(T, prompts, d, d_out, cfg, di->num_sms);
  if (ws_bytes < L.total) return TTQ_ERR_WORKSPACE;
  auto* base = static_cast<uint8_t*>(ws);
  auto* Xf = reinterpret_cast<__nv_bfloat16*>(base + L.xf_off);
  void* U = cfg->r > 0 ? base + L.u_off : nullptr;
  float* upart = cfg->r > 0 ? reinterpret_cast<float*>(base + L.upart_off) : nullptr;
  float* gpart = reinterpret_cast<float*>(base + L.gpart_off);
  const auto* Xb = static_cast<const __nv_bfloat16*>(X_bf16);
  auto* Yb = static_cast<__nv_bfloat16*>(Y_bf16);
  auto* sc = static_cast<__half*>(scale_f16);
  auto* zr = static_cast<__half*>(zero_f16);
  cudaError_t e = cudaSuccess;
  // each prompt's statistic and folded activations
  int64_t off = 0;
  for (int32_t p = 0; p < prompts && e == cudaSuccess; ++p) {
    e = ttq::launch_act_stats(Xb + off * d, T[p], d, d, cfg->alpha, cfg->lambda, cfg->p, s + p * d, di->num_sms,
                              dev_err(di), stream);
    if (e == cudaSuccess) e = ttq::launch_fold(Xb + off * d, T[p], d, d, s + p * d, Xf + off * d, stream);
    off += T[p];
  }
  // the low-rank projection of every prompt's tokens at once (A is shared)
  if (e == cudaSuccess && cfg->r > 0)
    e = ttq::launch_lowrank_u(X_bf16, L.tokens, d, A_bf16, cfg->r, U, upart, di->num_sms, dev_err(di), stream);
  // one read of W re-quantized for every prompt
  if (e == cudaSuccess)
    e = ttq::launch_requant_batched(W_bf16, d_out, d, s, prompts, cfg->q, cfg->g, codes, scale_f16, zero_f16, stream);
  if (e == cudaSuccess) {
    if (L.grouped) {
      // one grouped launch over every prompt's output tiles
      ttq::GemmArgs ga{Xf, codes, scale_f16, zero_f16, U, B_bf16, cfg->r, L.tokens, d, d_out, cfg->q, cfg->g,
                       Y_bf16, nullptr};
      e = ttq::launch_gemm2sm(ga, L.plan, dev_err(di), 0, stream, prompts, T);
    } else {
      off = 0;
      for (int32_t p = 0; p < prompts && e == cudaSuccess; ++p) {
        const ttq::GemmPlan pp = ttq::gemm_plan(T[p], d, d_out, cfg->q, cfg->g, di->num_sms);
        ttq::GemmArgs ga{Xf + off * d, codes + p * words, sc + p * metas, zr + p * metas,
                         U != nullptr ? static_cast<__nv_bfloat16*>(U) + off * 64 : nullptr, B_bf16, cfg->r, T[p], d,
                         d_out, cfg->q, cfg->g, Yb + off * d_out, gpart};
        e = ttq::launch_gemm(ga, pp, dev_err(di), stream);
        off += T[p];
      }
    }
  }
  return cuda_status(e);
}

// Workspace of a batched decode whose requests run on the CUDA-core GEMV (b <= 2): U for
// all P * b rows and its K-split partials, then one GEMV slice per request.
static size_t decode_batched_gemv_bytes(int32_t requests, int64_t b, int64_t d, int r, int num_sms) {
  const int64_t rows = static_cast<int64_t>(requests) * b;
  size_t bytes = 0;
  if (r > 0)
    bytes += round256(static_cast<size_t>(rows) * 64 * 2) + round256(ttq::lowrank_partial_bytes(rows, d, r, num_sms));
  bytes += round256(static_cast<size_t>(requests) * ttq::decode_gemv_ws_bytes(b, d));
  return bytes;
}

ttq_status ttq_decode_batched_workspace_size(int32_t requests, int64_t b, int64_t d, int64_t d_out,
                                             const ttq_config* cfg, size_t* bytes) {
  if (!bytes) return TTQ_ERR_INVALID_ARG;
  if (requests < 1 || requests > kMaxDecodeRequests) return TTQ_ERR_UNSUPPORTED;
  ttq_status st = check_dims(b, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  int num_sms = 148;
  DeviceInfo* di = nullptr;
  if (device_info(&di) == TTQ_OK) num_sms = di->num_sms;
  if (ttq::decode_gemv_ok(b, d))
    *bytes = decode_batched_gemv_bytes(requests, b, d, cfg->r, num_sms);
  else
    *bytes = ws_layout(b, d, d_out, cfg->r, cfg->q, cfg->g, num_sms).total;  // requests one after another
  return TTQ_OK;
}

ttq_status ttq_linear_decode_batched(const void* X_bf16, int32_t requests, int64_t b, int64_t d, int64_t d_out,
                                     const float* s, const uint32_t* codes, const void* scale_f16,
                                     const void* zero_f16, const void* A_bf16, const void* B_bf16,
                                     const ttq_config* cfg, void* Y_bf16, void* ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  if (requests < 1 || requests > kMaxDecodeRequests) return TTQ_ERR_UNSUPPORTED;
  ttq_status st = check_dims(b, d, d_out);
  if (st != TTQ_OK) return st;
  st = check_cfg(cfg, d);
  if (st != TTQ_OK) return st;
  st = check_lowrank(cfg, A_bf16, B_bf16);
  if (st != TTQ_OK) return st;
  if (!X_bf16 || !s || !codes || !scale_f16 || !zero_f16 || !Y_bf16) return TTQ_ERR_INVALID_ARG;
  if (!ws) return TTQ_ERR_WORKSPACE;
  if (!aligned16(X_bf16) || !aligned16(s) || !aligned16(codes) || !aligned16(scale_f16) ||
      !aligned16(zero_f16) || !aligned16(Y_bf16) || !aligned16(ws))
    return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  st = device_info(&di);
  if (st != TTQ_OK) return st;
  const int64_t words = static_cast<int64_t>(ttq_codes_words(d_out, d, cfg->q));
  const int64_t metas = d_out * (d / cfg->g);
  if (!ttq::decode_gemv_ok(b, d)) {
    // more tokens per request: the tensor-core decode of each request in turn (the
    // per-request strides keep every operand 16-byte aligned when b * d, b * d_out, d,
    // the code words and d_out * d / g are multiples of 8 elements)
    if ((b * d) % 8 || (b * d_out) % 8 || words % 4 || metas % 8) return TTQ_ERR_MISALIGNED;
    for (int32_t p = 0; p < requests; ++p) {
      st = ttq_linear_decode(static_cast<const __nv_bfloat16*>(X_bf16) + p * b * d, b, d, d_out, s + p * d,
                             codes + p * words, static_cast<const __half*>(scale_f16) + p * metas,
                             static_cast<const __half*>(zero_f16) + p * metas, A_bf16, B_bf16, cfg,
                             static_cast<__nv_bfloat16*>(Y_bf16) + p * b * d_out, ws, ws_bytes, stream);
      if (st != TTQ_OK) return st;
    }
    return TTQ_OK;
  }
  if (ws_bytes < decode_batched_gemv_bytes(requests, b, d, cfg->r, di->num_sms)) return TTQ_ERR_WORKSPACE;
  auto* base = static_cast<uint8_t*>(ws);
  const int64_t rows = static_cast<int64_t>(requests) * b;
  void* U = nullptr;
  size_t off = 0;
  if (cfg->r > 0) {
    // U = X A^T of request p's tokens in rows p * b .. p * b + b - 1, formed by the GEMV's
    // prep kernel (A is shared)
    U = base;
    off = round256(static_cast<size_t>(rows) * 64 * 2) + round256(ttq::lowrank_partial_bytes(rows, d, cfg->r, di->num_sms));
  }
  ttq::DecodeArgs da{X_bf16, s, codes, scale_f16, zero_f16, U, B_bf16, cfg->r, b, d, d_out, cfg->q, cfg->g, Y_bf16,
                     requests, dev_err(di)};
  da.A = cfg->r > 0 ? A_bf16 : nullptr;
  return cuda_status(ttq::launch_decode_gemv(da, base + off, stream));
}

// ---------------------------------------------------------------- decoder layer

ttq_status ttq_rmsnorm(const void* y_bf16, void* residual_bf16, const void* w_bf16, int64_t rows, int64_t n,
                       float eps, void* out_bf16, cudaStream_t stream) {
  if (!y_bf16 || !w_bf16 || !out_bf16) return TTQ_ERR_INVALID_ARG;
  if (rows < 1 || rows > (int64_t(1) << 31) - 1 || n < 8 || n > 8192 || n % 8 != 0) return TTQ_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || !(eps > 0.f)) return TTQ_ERR_INVALID_ARG;
  if (out_bf16 == y_bf16 || (residual_bf16 && (residual_bf16 == y_bf16 || residual_bf16 == out_bf16)))
    return TTQ_ERR_INVALID_ARG;
  if (!aligned16(y_bf16) || !aligned16(w_bf16) || !aligned16(out_bf16) ||
      (residual_bf16 && !aligned16(residual_bf16)))
    return TTQ_ERR_MISALIGNED;
  return cuda_status(ttq::launch_rmsnorm(y_bf16, residual_bf16, w_bf16, rows, static_cast<int>(n), eps, out_bf16,
                                         stream));
}

ttq_status ttq_rope_table(int64_t positions, int64_t head_dim, double base, float* table, cudaStream_t stream) {
  if (!table) return TTQ_ERR_INVALID_ARG;
  if (positions < 1 || positions > (int64_t(1) << 24)) return TTQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return TTQ_ERR_UNSUPPORTED;
  if (!std::isfinite(base) || !(base > 1.0)) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(table)) return TTQ_ERR_MISALIGNED;
  return cuda_status(ttq::launch_rope_table(positions, static_cast<int>(head_dim), base, table, stream));
}

ttq_status ttq_qk_norm_rope(void* qkv_bf16, int64_t T, int64_t heads, int64_t kv_heads, int64_t head_dim,
                            const void* q_norm_bf16, const void* k_norm_bf16, float eps, const float* rope_table,
                            int64_t table_positions, int64_t pos0, const int64_t* pos0_dev, void* k_cache_bf16,
                            void* v_cache_bf16, int64_t cache_len, cudaStream_t stream) {
  if (!qkv_bf16 || !q_norm_bf16 || !k_norm_bf16 || !rope_table || !k_cache_bf16 || !v_cache_bf16)
    return TTQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return TTQ_ERR_UNSUPPORTED;
  if (T < 1 || heads < 1 || kv_heads < 1 || heads > 1024 || kv_heads > 1024) return TTQ_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 24) || cache_len < T || table_positions < T) return TTQ_ERR_INVALID_ARG;
  if (!pos0_dev && (pos0 < 0 || pos0 + T > cache_len || pos0 + T > table_positions)) return TTQ_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || !(eps > 0.f)) return TTQ_ERR_INVALID_ARG;
  if (k_cache_bf16 == v_cache_bf16) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(qkv_bf16) || !aligned16(q_norm_bf16) || !aligned16(k_norm_bf16) || !aligned16(rope_table) ||
      !aligned16(k_cache_bf16) || !aligned16(v_cache_bf16) || (pos0_dev && (reinterpret_cast<uintptr_t>(pos0_dev) & 7)))
    return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  ttq_status st = device_info(&di);
  if (st != TTQ_OK) return st;
  return cuda_status(ttq::launch_qk_norm_rope(qkv_bf16, T, static_cast<int>(heads), static_cast<int>(kv_heads),
                                              static_cast<int>(head_dim), q_norm_bf16, k_norm_bf16, eps, rope_table,
                                              pos0, pos0_dev, std::min(cache_len, table_positions), k_cache_bf16,
                                              v_cache_bf16, di->err_word, stream));
}

namespace {
ttq_status check_decode_attention(int64_t heads, int64_t kv_heads, int64_t head_dim, int64_t cache_len) {
  if (head_dim != 64 && head_dim != 128) return TTQ_ERR_UNSUPPORTED;
  if (heads < 1 || kv_heads < 1 || heads > 1024 || heads % kv_heads != 0) return TTQ_ERR_INVALID_ARG;
  const int64_t G = heads / kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TTQ_ERR_UNSUPPORTED;
  if (cache_len < 1 || cache_len > (int64_t(1) << 30)) return TTQ_ERR_INVALID_ARG;
  return TTQ_OK;
}
}  // namespace

ttq_status ttq_decode_attention_workspace_size(int64_t heads, int64_t kv_heads, int64_t head_dim, int64_t cache_len,
                                               size_t* bytes) {
  if (!bytes) return TTQ_ERR_INVALID_ARG;
  ttq_status st = check_decode_attention(heads, kv_heads, head_dim, cache_len);
  if (st != TTQ_OK) return st;
  const int splits = ttq::decode_attn_splits(cache_len, static_cast<int>(kv_heads));
  *bytes = round256(ttq::decode_attn_partial_bytes(static_cast<int>(heads), static_cast<int>(head_dim), splits));
  return TTQ_OK;
}

ttq_status ttq_decode_attention(const void* q_bf16, int64_t heads, int64_t kv_heads, int64_t head_dim,
                                const void* k_cache_bf16, const void* v_cache_bf16, int64_t cache_len, int64_t length,
                                const int64_t* pos_dev, void* out_bf16, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
  if (!q_bf16 || !k_cache_bf16 || !v_cache_bf16 || !out_bf16) return TTQ_ERR_INVALID_ARG;
  ttq_status st = check_decode_attention(heads, kv_heads, head_dim, cache_len);
  if (st != TTQ_OK) return st;
  if (!pos_dev && (length < 1 || length > cache_len)) return TTQ_ERR_INVALID_ARG;
  if (!ws) return TTQ_ERR_WORKSPACE;
  const int splits = ttq::decode_attn_splits(cache_len, static_cast<int>(kv_heads));
  if (ws_bytes < ttq::decode_attn_partial_bytes(static_cast<int>(heads), static_cast<int>(head_dim), splits))
    return TTQ_ERR_WORKSPACE;
  if (!aligned16(q_bf16) || !aligned16(k_cache_bf16) || !aligned16(v_cache_bf16) || !aligned16(out_bf16) ||
      !aligned16(ws) || (pos_dev && (reinterpret_cast<uintptr_t>(pos_dev) & 7)))
    return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  st = device_info(&di);
  if (st != TTQ_OK) return st;
  return cuda_status(ttq::launch_decode_attention(q_bf16, static_cast<int>(heads), static_cast<int>(kv_heads),
                                                  static_cast<int>(head_dim), k_cache_bf16, v_cache_bf16, cache_len,
                                                  length, pos_dev, out_bf16, static_cast<float*>(ws), splits,
                                                  di->err_word, stream));
}

ttq_status ttq_prompt_attention(const void* qkv_bf16, int64_t T, int64_t heads, int64_t kv_heads, int64_t head_dim,
                                const void* k_cache_bf16, const void* v_cache_bf16, int64_t cache_len, void* out_bf16,
                                cudaStream_t stream) {
  if (!qkv_bf16 || !k_cache_bf16 || !v_cache_bf16 || !out_bf16) return TTQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return TTQ_ERR_UNSUPPORTED;
  if (heads < 1 || kv_heads < 1 || heads > 1024 || heads % kv_heads != 0) return TTQ_ERR_INVALID_ARG;
  if (T < 1 || T > (int64_t(1) << 24) || cache_len < T) return TTQ_ERR_INVALID_ARG;
  if (out_bf16 == qkv_bf16 || k_cache_bf16 == v_cache_bf16) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(qkv_bf16) || !aligned16(k_cache_bf16) || !aligned16(v_cache_bf16) || !aligned16(out_bf16))
    return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  ttq_status st = device_info(&di);
  if (st != TTQ_OK) return st;
  return cuda_status(ttq::launch_prompt_attention(qkv_bf16, T, static_cast<int>(heads), static_cast<int>(kv_heads),
                                                  static_cast<int>(head_dim), k_cache_bf16, v_cache_bf16, out_bf16,
                                                  dev_err(di), stream));
}

ttq_status ttq_position_advance(int64_t* pos_dev, int64_t n, cudaStream_t stream) {
  if (!pos_dev || n < 0) return TTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(pos_dev) & 7) return TTQ_ERR_MISALIGNED;
  return cuda_status(ttq::launch_position_advance(pos_dev, n, stream));
}

ttq_status ttq_silu_mul(const void* gate_up_bf16, int64_t rows, int64_t inter, void* out_bf16, cudaStream_t stream) {
  if (!gate_up_bf16 || !out_bf16) return TTQ_ERR_INVALID_ARG;
  if (rows < 1 || inter < 8 || inter % 8 != 0 || rows * inter > (int64_t(1) << 40)) return TTQ_ERR_INVALID_ARG;
  if (gate_up_bf16 == out_bf16) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(gate_up_bf16) || !aligned16(out_bf16)) return TTQ_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  ttq_status st = device_info(&di);
  if (st != TTQ_OK) return st;
  return cuda_status(ttq::launch_silu_mul(gate_up_bf16, rows, inter, out_bf16, di->num_sms, stream));
}

ttq_status ttq_device_status(cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  ttq_status st = device_info(&di);
  if (st != TTQ_OK) return st;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TTQ_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpyFromSymbol(&word, g_ttq_error_word, sizeof(word)) != cudaSuccess) return TTQ_ERR_CUDA;
  if (word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_ttq_error_word, &zero, sizeof(zero)) != cudaSuccess) return TTQ_ERR_CUDA;
    return (word & ttq::kErrTimeout) ? TTQ_ERR_TIMEOUT : TTQ_ERR_INVALID_ARG;
  }
  return TTQ_OK;
}

ttq_status ttq_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns == 0 ? 2000000000ull : ns);
  return TTQ_OK;
}

int32_t ttq_last_cuda_error(void) { return g_last_cuda_error; }

const char* ttq_cuda_error_string(int32_t code) {
  return cudaGetErrorString(static_cast<cudaError_t>(code));
}

ttq_status ttq_debug_inject_stall(int32_t enable) {
  ttq::set_inject_stall(enable != 0);
  return TTQ_OK;
}

ttq_status ttq_set_trace_events(void* const* events, int32_t n) {
  if (n == 0 || events == nullptr) {
    g_trace_on = false;
    return TTQ_OK;
  }
  if (n < 6) return TTQ_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i) {
    if (!events[i]) return TTQ_ERR_INVALID_ARG;
  }
  for (int i = 0; i < 6; ++i) g_trace[i] = static_cast<cudaEvent_t>(events[i]);
  g_trace_on = true;
  return TTQ_OK;
}

const char* ttq_status_string(ttq_status status) {
  switch (status) {
    case TTQ_OK: return "TTQ_OK";
    case TTQ_ERR_INVALID_ARG: return "TTQ_ERR_INVALID_ARG";
    case TTQ_ERR_UNSUPPORTED: return "TTQ_ERR_UNSUPPORTED";
    case TTQ_ERR_MISALIGNED: return "TTQ_ERR_MISALIGNED";
    case TTQ_ERR_WORKSPACE: return "TTQ_ERR_WORKSPACE";
    case TTQ_ERR_CUDA: return "TTQ_ERR_CUDA";
    case TTQ_ERR_TIMEOUT: return "TTQ_ERR_TIMEOUT";
    case TTQ_ERR_TOO_LARGE: return "TTQ_ERR_TOO_LARGE";
  }
  return "TTQ_ERR_UNKNOWN";
}

}  // extern "C"
