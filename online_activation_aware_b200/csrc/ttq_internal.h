// Internal launch interface between the C ABI (ttq_api.cu) and the kernel files.
// Every launcher enqueues on `stream` and returns the launch status; none allocates.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "ttq_common.cuh"

namespace ttq {

// Launches `kernel` with programmatic stream serialization: it may start launching while the
// kernel ahead in the stream finishes, so it must begin with pdl_enter() (or wait with
// grid_dep_wait() before it reads anything that kernel writes).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Identifier (cuCtxGetId) of the CUDA context current on this host thread; when none is,
// the current device's primary context is bound first. False when the driver refuses.
// Device addresses of module symbols are per context, so caches of them key on this.
bool current_context_id(unsigned long long* id);

// ---------------------------------------------------------------- act_stats / fold

// Column-split plan of the statistics kernels: blocks of 256 columns, T split in
// `nsplit` row ranges of `rows_per_split` rows.
struct StatsPlan {
  int col_blocks;
  int nsplit;
  int64_t rows_per_split;
};
// Plan of the single-kernel statistic with arrival counters (launch_act_stats_capped).
StatsPlan stats_plan(int64_t T, int64_t d);

// Row split of the single-launch statistic: blocks of 256 columns x rows_per_split rows,
// about two blocks per SM, the nsplit <= kStatsMaxSplit blocks of a column strip forming
// one thread-block cluster.
constexpr int kStatsMaxSplit = 16;
StatsPlan cluster_plan(int64_t T, int64_t d, int num_sms);

// s = (mean_t |x|^p + lambda)^(alpha/p) in one launch with no scratch memory (the row
// splits of a strip reduce through distributed shared memory); launched with programmatic
// stream serialization: it waits for the kernel ahead before it reads X, then lets the
// next kernel launch.
// X streams through a TMA ring in shared memory (every wait bounded by err.wait_ns).
cudaError_t launch_act_stats(const void* X, int64_t T, int64_t d, int64_t ld_x, float alpha, float lambda, int p,
                             float* s, int num_sms, const DevErr& err, cudaStream_t stream);

// Same statistic, with at most `max_partial_floats` fp32 partial sums: the row split is
// reduced until nsplit * d fits (used where the scratch has a fixed size).
cudaError_t launch_act_stats_capped(const void* X, int64_t T, int64_t d, int64_t ld_x, float alpha,
                                    float lambda, int p, float* s, float* partial,
                                    int64_t max_partial_floats, unsigned* counters,
                                    cudaStream_t stream);

// Xf[t, j] = bf16(X[t, j] * (1 / s[j])), Xf contiguous [T, d].
cudaError_t launch_fold(const void* X, int64_t T, int64_t d, int64_t ld_x, const float* s,
                        void* Xf, cudaStream_t stream);

// s_j from the column sum of |x_tj|^p over the prompt's T tokens (every statistic kernel
// finishes with this one step, so their results agree whenever their sums do).
__device__ __forceinline__ float finalize_scale(float colsum, float T, float alpha_over_p, float lambda) {
  const float m = __fdiv_rn(colsum, T);  // mean over the prompt's tokens
  return powf(__fadd_rn(m, lambda), alpha_over_p);
}

// U[t, :] = X[t, :] A^T in fp32 accumulation (tensor cores, K split over blocks, the
// splits added in a fixed order by a dependent kernel), stored bf16 with row stride 64
// (columns r..63 zero). Requires r % 8 == 0, r <= 64; `partial` holds
// lowrank_partial_bytes() of workspace.
int lowrank_splits(int64_t T, int64_t d, int num_sms);
size_t lowrank_partial_bytes(int64_t T, int64_t d, int r, int num_sms);
cudaError_t launch_lowrank_u(const void* X, int64_t T, int64_t d, const void* A, int r, void* U, float* partial,
                             int num_sms, const DevErr& err, cudaStream_t stream);

// The same pass over X also yielding the statistic s (p in {1, 2}): each block sums |x|^p
// over its 64 tokens for the channels of its K slice (fp32, fixed order) into `stats_part`
// ([ceil(T / 64), d] fp32, lowrank_stats_bytes() of workspace), and the dependent kernel
// that adds the K splits of U also adds those rows in token-block order and writes s.
// Only for T > lowrank_small_tokens() (fewer tokens take one block per output of U).
int lowrank_small_tokens();
size_t lowrank_stats_bytes(int64_t T, int64_t d);
cudaError_t launch_lowrank_u_stats(const void* X, int64_t T, int64_t d, const void* A, int r, void* U,
                                   float* partial, float* stats_part, float alpha, float lambda, int p, float* s,
                                   int num_sms, const DevErr& err, cudaStream_t stream);

// ---------------------------------------------------------------- decode

constexpr int kGemvMaxTokens = 2;  // larger decode batches run on the tensor cores
struct DecodeArgs {
  const void* X;          // bf16 [b, d] new tokens (not folded)
  const float* s;         // fp32 [d] the prefill's statistic
  const uint32_t* codes;  // packed codes [d_out, d*q/32]
  const void* scale;      // fp16 [d_out, d/g]
  const void* zero;       // fp16 [d_out, d/g]
  const void* U;          // bf16 [b, 64] = X A^T (r > 0) or null
  const void* Blr;        // bf16 [d_out, r] or null
  int r;
  int64_t b, d, d_out;
  int q, g;
  void* Y;                // bf16 [b, d_out]
  int requests;           // batched decode: requests stacked along every per-request operand
  DevErr err;             // device error word and wait limit
  const void* A = nullptr;  // bf16 [r, d]: when set, the prep kernel also forms U (b <= 8)
};
// True when the CUDA-core GEMV handles these decode sizes (b <= 2).
bool decode_gemv_ok(int64_t b, int64_t d);
// Workspace bytes of launch_decode_gemv for one request: x' (fp32, [d][B]) and its
// 32-input unit sums (a batched decode takes `requests` such slices back to back).
size_t decode_gemv_ws_bytes(int64_t b, int64_t d);
// The prep kernel and the GEMV (launched as its programmatic dependent).
cudaError_t launch_decode_gemv(const DecodeArgs& a, void* ws, cudaStream_t stream);

// ---------------------------------------------------------------- requant

// pdl: launch as the programmatic dependent of the kernel ahead in the stream (only where
// that kernel does not write W; the kernel waits for it before it reads s).
cudaError_t launch_requant(const void* W, int64_t d_out, int64_t d, const float* s, int q, int g,
                           uint32_t* codes, void* scale, void* zero, bool pdl, cudaStream_t stream);

// P prompts (1 <= P <= kRequantMaxPrompts) re-quantized from one read of W: s is [P, d],
// prompt p's codes / scale / zero start P strides into the outputs (strides of one
// prompt's output sizes).
constexpr int kRequantMaxPrompts = 8;
cudaError_t launch_requant_batched(const void* W, int64_t d_out, int64_t d, const float* s, int prompts, int q,
                                   int g, uint32_t* codes, void* scale, void* zero, cudaStream_t stream);

// The prefill's fused form: the re-quantization of W and, in the same launch (extra warps
// per CTA), the fold Xf = bf16(X * (1/s)) of the contiguous [T, d] activations. Launched
// as the programmatic dependent of the kernel ahead in the stream, which must write
// neither W nor X (it waits for that kernel before it reads s).
cudaError_t launch_fold_requant(const void* X, int64_t T, void* Xf, const void* W, int64_t d_out, int64_t d,
                                const float* s, int q, int g, uint32_t* codes, void* scale, void* zero,
                                cudaStream_t stream);

// ---------------------------------------------------------------- GEMM

struct GemmPlan {
  bool pair;        // 2-SM kernel (tcgen05 cta_group::2, 256-row tiles per CTA pair)
  int BN;           // tokens per tile (MMA N): 16, 32, 64, 128 or 256
  int m_tiles;      // ceil(d_out / 128), or ceil(d_out / 256) for the 2-SM kernel
  int n_tiles;      // ceil(T / BN)
  int nkb;          // K blocks of 64: ceil(d / 64)
  int ksplit;       // split-K factor (1 = direct bf16 epilogue)
  int kb_per_split;
  int ctas_per_sm;  // single-CTA kernel: 2 for 16-token tiles with TMA-loaded codes, else 1
  size_t smem_bytes;
};
GemmPlan gemm_plan(int64_t T, int64_t d, int64_t d_out, int q, int g, int num_sms);
// Codes and group scale/zero rows have 16-byte pitches, so TMA can load them.
bool tma_codes_ok(int64_t d, int q, int g);
size_t gemm_partial_bytes(const GemmPlan& p, int64_t T, int64_t d_out);

struct GemmArgs {
  const void* Xf;        // bf16 [T, d] folded activations
  const uint32_t* codes; // packed codes [d_out, d*q/32]
  const void* scale;     // fp16 [d_out, d/g]
  const void* zero;      // fp16 [d_out, d/g]
  const void* U;         // bf16 [T, 64] low-rank projection (r > 0) or null
  const void* Blr;       // bf16 [d_out, r] (r > 0) or null
  int r;
  int64_t T, d, d_out;
  int q, g;
  void* Y;               // bf16 [T, d_out]
  float* partial;        // fp32 [ksplit, T, d_out] when ksplit > 1
};

// The tensor-core kernel (writes Y directly, or fp32 partials when plan.ksplit > 1) and
// the split-K reduction (a no-op when plan.ksplit == 1); launch_gemm runs both.
cudaError_t launch_gemm_mainloop(const GemmArgs& a, const GemmPlan& plan, const DevErr& err,
                                 cudaStream_t stream);
cudaError_t launch_gemm_reduce(const GemmArgs& a, const GemmPlan& plan, cudaStream_t stream);
cudaError_t launch_gemm(const GemmArgs& a, const GemmPlan& plan, const DevErr& err,
                        cudaStream_t stream);

// Test hook: when on, the tensor-core kernel's MMA thread first waits on a barrier that
// nothing arrives at, so its bounded wait runs out (see ttq_debug_inject_stall).
void set_inject_stall(bool on);

// 2-D row-major tensor map of `elem_bytes`-sized elements with a {box_cols, box_rows}
// box and the given swizzle.
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, uint32_t elem_bytes, const void* base,
                    uint64_t rows, uint64_t cols, uint64_t row_stride_elems, uint32_t box_cols,
                    uint32_t box_rows, CUtensorMapSwizzle swz);
// The 2-SM tensor-core kernel (launched by launch_gemm_mainloop when plan.pair). Grouped
// form (groups > 1, at most kGemmMaxGroups, plan.ksplit == 1): group_T[p] tokens of prompt p
// stacked along the token axis of Xf, U and Y (a.T their sum), each prompt with its own
// codes / scale / zero stacked along the rows (p * d_out ..); one launch covers every
// prompt's tiles.
constexpr int kGemmMaxGroups = 8;
cudaError_t launch_gemm2sm(const GemmArgs& a, const GemmPlan& plan, const DevErr& err, int inject_stall,
                           cudaStream_t stream, int groups = 1, const int64_t* group_T = nullptr);

// 3-D bf16 tensor map (dims innermost first, byte strides of dims 1 and 2), 128-byte
// swizzle, zero fill outside the tensor.
bool encode_bf16_tmap_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2);

// Encodes a 2-D row-major bf16 tensor map with 128-byte swizzle and a box of
// {64 columns, box_rows rows}. Returns false when the driver refuses it.
bool encode_bf16_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint64_t row_stride_elems, uint32_t box_rows);

// ---------------------------------------------------------------- decoder layer (decoder.cu)

// r <- bf16(r + y) per row when `residual` is non-null, then out = bf16(h w / rms(h))
// over rows of n channels (n % 8 == 0, n <= 8192).
cudaError_t launch_rmsnorm(const void* y, void* residual, const void* w, int64_t rows, int n, float eps, void* out,
                           cudaStream_t stream);
// fp32 (cos, sin) pairs of pos * base^(-2i/D) for pos < positions, i < D/2.
cudaError_t launch_rope_table(int64_t positions, int head_dim, double base, float* table, cudaStream_t stream);
// Device error word bits: a position read from device memory was outside the cache; a
// kernel's shared-memory layout did not fit its allocation (it returned without work).
constexpr unsigned kErrRange = 2u;
constexpr unsigned kErrLayout = 4u;

// Per-head RMSNorm + rotary embedding of q (in place) and k (into k_cache), v copied into
// v_cache, for T tokens of the stacked projection at positions pos0 ... (pos0 = *pos_dev
// when pos_dev is given, checked against `limit` on the device); head_dim in {64, 128, 256}.
cudaError_t launch_qk_norm_rope(void* qkv, int64_t T, int heads, int kv_heads, int head_dim, const void* wq,
                                const void* wk, float eps, const float* table, int64_t pos0, const int64_t* pos_dev,
                                int64_t limit, void* k_cache, void* v_cache, unsigned* err, cudaStream_t stream);
// One token's attention over the first L cache positions (L = *pos_dev + 1 when pos_dev is
// given, else `length`): split over positions into `part` (decode_attn_partial_bytes), then
// merged per query head into out [heads * head_dim] bf16. head_dim in {64, 128};
// heads / kv_heads in {1, 2, 4, 8}.
int decode_attn_splits(int64_t cache_len, int kv_heads);
size_t decode_attn_partial_bytes(int heads, int head_dim, int splits);
cudaError_t launch_decode_attention(const void* q, int heads, int kv_heads, int head_dim, const void* k_cache,
                                    const void* v_cache, int64_t cache_len, int64_t length, const int64_t* pos_dev,
                                    void* out, float* part, int splits, unsigned* err, cudaStream_t stream);
// Causal grouped-query attention of a prompt at positions 0 .. T-1 on the tensor cores:
// q from the stacked projection (after ttq_qk_norm_rope), k and v from the caches' first T
// positions, out [T, heads * head_dim] bf16. head_dim 64 or 128.
cudaError_t launch_prompt_attention(const void* qkv, int64_t T, int heads, int kv_heads, int head_dim,
                                    const void* k_cache, const void* v_cache, void* out, const DevErr& err,
                                    cudaStream_t stream);
// *pos += n on the device (one thread).
cudaError_t launch_position_advance(int64_t* pos, int64_t n, cudaStream_t stream);
// out = bf16(silu(gate) * up) over rows of [gate | up] (inter channels each, inter % 8 == 0).
cudaError_t launch_silu_mul(const void* gu, int64_t rows, int64_t inter, void* out, int num_sms, cudaStream_t stream);

}  // namespace ttq
