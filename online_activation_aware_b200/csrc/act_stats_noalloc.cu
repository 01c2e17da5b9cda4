// ttq_act_stats_noalloc: the activation statistic for callers that cannot allocate
// device memory. The reduction's scratch (fp32 partial sums and the per-strip arrival
// counters) lives in one fixed array in the library's own device memory instead of a
// caller workspace. Host code reaches the array only through the device address that
// cudaGetSymbolAddress returns (the symbol itself is a host-side stand-in, not a device
// pointer), looked up with the device current on the first call in each CUDA context.
#include <mutex>

#include "ttq.h"
#include "ttq_internal.h"

namespace {

constexpr int64_t kMaxD = 65536;                   // channels
constexpr int64_t kPartialFloats = 262144;         // 1 MiB of fp32 partial sums
constexpr int64_t kCounterBytes = 1024;            // kMaxD / 256 column strips x 4 B
constexpr int64_t kScratchBytes = kPartialFloats * 4 + kCounterBytes;

static __device__ __align__(256) unsigned char g_act_stats_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  unsigned long long ctx_id = 0;  // context the address belongs to (0: not looked up yet)
  void* addr = nullptr;
};
std::mutex g_mu;
ScratchAddr g_scratch[kMaxDevices];

// Device address of the scratch array in the context current on this thread, looked up
// with cudaGetSymbolAddress on the first call in that context and cached per device
// ordinal together with the context's id. A module's symbols get new addresses when its
// context is rebuilt (cudaDeviceReset) and differ in a caller's own driver-API context,
// so a change of context id triggers a fresh lookup instead of reusing a dead address.
ttq_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTQ_ERR_CUDA;
  unsigned long long ctx = 0;
  if (!ttq::current_context_id(&ctx)) return TTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchAddr& e = g_scratch[dev];
  if (e.ctx_id != ctx || e.addr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_act_stats_scratch) != cudaSuccess || p == nullptr) return TTQ_ERR_CUDA;
    e.addr = p;
    e.ctx_id = ctx;
  }
  *out = e.addr;
  return TTQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" ttq_status ttq_act_stats_noalloc(const void* X_bf16, int64_t T, int64_t d, int64_t ld_x,
                                            float alpha, float lambda, int32_t p, float* s,
                                            cudaStream_t stream) {
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (T < 1 || d < 1 || T > lim || T * d > (int64_t(1) << 40) || d % 8 != 0) return TTQ_ERR_INVALID_ARG;
  if (ld_x < d || ld_x % 8 != 0) return TTQ_ERR_INVALID_ARG;
  if (p != 1 && p != 2) return TTQ_ERR_UNSUPPORTED;
  if (!(alpha >= 0.f) || !(lambda >= 0.f) || alpha > 3.0e38f || lambda > 3.0e38f) return TTQ_ERR_INVALID_ARG;
  if (alpha > 0.f && !(lambda > 0.f)) return TTQ_ERR_INVALID_ARG;
  if (d > kMaxD) return TTQ_ERR_TOO_LARGE;
  if (!X_bf16 || !s) return TTQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(s)) return TTQ_ERR_MISALIGNED;
  void* base = nullptr;
  ttq_status st = scratch_on_current_device(&base);
  if (st != TTQ_OK) return st;
  auto* partial = static_cast<float*>(base);
  auto* counters = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(base) + kPartialFloats * 4);
  const cudaError_t e = ttq::launch_act_stats_capped(X_bf16, T, d, ld_x, alpha, lambda, p, s, partial,
                                                     kPartialFloats, counters, stream);
  return e == cudaSuccess ? TTQ_OK : TTQ_ERR_CUDA;
}
