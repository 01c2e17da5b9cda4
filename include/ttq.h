/*
 * ttq.h - C ABI of the TTQ hot path on NVIDIA B200 (sm_100a).
 *
 * TTQ, activation-aware test-time quantization, quantizes the weights of a linear
 * layer on the fly for every prompt, from that prompt's own activations.
 * Definitions come from the pages on "TTQ: Activation-Aware Test-Time Quantization to
 * Accelerate LLM Inference On The Fly":
 *   [DR]  paper-daily.com deep reading, section 2 (method) and section 6 (deployment);
 *   [NR]  nubint.ai review, section "proposed method";
 *   [GDE] gist.science German technical summary, section 2 (Methodik);
 *   [GFR] gist.science French technical summary, sections 2A and 2B.
 *
 * Conventions for every entry point
 *   - Layouts: X is [T, d] bf16 row-major (tokens by input channels); W is [d_out, d]
 *     bf16 row-major (the usual linear-layer layout); s is fp32 [d]; codes are uint32
 *     [d_out, d*q/32]; scale and zero are fp16 [d_out, d/g]; Y is [T, d_out] bf16.
 *   - Packed codes: groups run along d. q = 2 or 4: 32/q codes per word, code k of the
 *     word at bits [q*k, q*k+q). q = 3: every 32 consecutive codes occupy 3 words, word
 *     b holding bit b of each code (code k at bit k). Always exactly q/8 bytes a weight.
 *   - Ownership: the caller allocates and owns every buffer (device memory); the library
 *     allocates nothing, keeps no state between calls beyond one device error word, and
 *     never writes to its inputs.
 *   - Asynchrony: every compute call enqueues work on `stream` and returns. Argument
 *     errors are returned synchronously and nothing is launched. A failed launch returns
 *     TTQ_ERR_CUDA. A kernel that gives up on a bounded wait records TTQ_ERR_TIMEOUT in
 *     the device error word, which ttq_device_status() reports.
 *   - Alignment: every pointer must be 16-byte aligned (TTQ_ERR_MISALIGNED otherwise).
 *   - Supported settings: q in {2,3,4}; g in {32,64,128}; d % g == 0; p in {1,2};
 *     alpha >= 0; lambda > 0 when alpha > 0; 0 <= r <= 64 with A and B non-NULL
 *     exactly when r > 0.
 *   - Numerics: the quantizer runs in pinned IEEE fp32 and is reproducible bit for bit
 *     given the same s; statistics accumulate in fp32; the projection multiplies bf16
 *     operands on the tensor cores with fp32 accumulation and rounds Y to bf16.
 */
#ifndef TTQ_H_
#define TTQ_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define TTQ_API __attribute__((visibility("default")))
#else
#define TTQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTQ_OK = 0,
  TTQ_ERR_INVALID_ARG = -1,  /* a size, pointer or setting is out of range          */
  TTQ_ERR_UNSUPPORTED = -2,  /* q, g, p or r outside the supported set               */
  TTQ_ERR_MISALIGNED = -3,   /* a pointer (or leading dimension) is not 16-byte aligned */
  TTQ_ERR_WORKSPACE = -4,    /* ws is NULL or smaller than ttq_workspace_size()       */
  TTQ_ERR_CUDA = -5,         /* a CUDA runtime call or kernel launch failed            */
  TTQ_ERR_TIMEOUT = -6,      /* a kernel gave up on a bounded wait (device error word) */
  TTQ_ERR_TOO_LARGE = -7     /* a size exceeds a fixed internal capacity               */
} ttq_status;

/* TTQ settings. q: bits per weight; g: group size along d; alpha, lambda, p: the
 * statistic s_j = (mean_t |x_tj|^p + lambda)^(alpha/p) (p = 2 gives D^(1/2) with
 * D = diag[X X^T / T + lambda I]^alpha, [DR] section 2); r: rank of the static low-rank
 * factors B [d_out, r] and A [r, d] ([DR] section 2, [GFR] section 2B; 0 = none). */
typedef struct {
  int32_t q;
  int32_t g;
  float alpha;
  float lambda;
  int32_t p;
  int32_t r;
} ttq_config;

/* Number of uint32 words of packed codes for a [d_out, d] weight at q bits
 * (d_out * d * q / 32). Returns 0 when d is not a multiple of 32 or q is unsupported. */
TTQ_API size_t ttq_codes_words(int64_t d_out, int64_t d, int32_t q);

/* Bytes of scratch workspace that ttq_linear_prefill (and ttq_linear_decode with
 * T = b rows; and ttq_act_stats with d_out = 0) needs for these sizes. For the prefill
 * and decode it holds the folded activations X diag(1/s) in bf16, the low-rank
 * projection X A^T, split-K partial products and the decode GEMV's operands; for
 * ttq_act_stats (d_out = 0) nothing (0 bytes). Contents need not be initialised and are
 * not preserved. */
TTQ_API ttq_status ttq_workspace_size(int64_t T, int64_t d, int64_t d_out, const ttq_config* cfg,
                              size_t* bytes);

/* Where the folded activations sit in the workspace of ttq_linear_prefill (and of
 * ttq_linear_decode with T = b rows when b > 2). Once such a call has run (in stream
 * order), bytes [*offset, *offset + 2*T*d) of its workspace hold X diag(1/s) as bf16
 * [T, d] row-major, x'_tj = RN_bf16(x_tj * RN_fp32(1/s_j)): the pre-scaling of the
 * activations that [DR] section 5 suggests fusing, which the projection multiplies. They
 * stay there until the workspace is used again. Same arguments and errors as
 * ttq_workspace_size (d_out >= 1). For inspection and tests. */
TTQ_API ttq_status ttq_workspace_folded_offset(int64_t T, int64_t d, int64_t d_out, const ttq_config* cfg,
                                               size_t* offset);

/* Online activation statistics ([DR] section 2 online diagonal D of each prompt;
 * [GDE] section 2 D_ii from the norms of the input rows).
 *   X      device bf16 [T, ld_x] (first d columns used), ld_x >= d, ld_x % 8 == 0
 *   s      device fp32 [d] output: s_j = (mean_t |x_tj|^p + lambda)^(alpha/p)
 *   ws     scratch of ttq_workspace_size(T, d, 0, ...) bytes, which is 0: the reduction
 *          runs on chip (the row splits of each 256-channel strip form one thread-block
 *          cluster and add their partial sums in shared memory), so ws may be NULL and
 *          ws_bytes is ignored; a non-NULL ws must be 16-byte aligned
 * The column sums accumulate in fp32 in a fixed order, so results are deterministic. */
TTQ_API ttq_status ttq_act_stats(const void* X_bf16, int64_t T, int64_t d, int64_t ld_x, float alpha,
                         float lambda, int32_t p, float* s, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* Allocation-free variant of ttq_act_stats, for callers that cannot allocate device
 * memory: code running where cudaMalloc is unavailable or too costly (cudaMalloc can
 * synchronise the whole device, which a latency-bound serving loop cannot afford), or
 * code embedded in a program whose allocator has already reserved all device memory
 * (for example a serving engine that claims the free HBM for its KV cache at start-up)
 * and so cannot hand out a workspace. The paper has no counterpart: this is a
 * deployment convenience of this library.
 * Same inputs, output and numerics as ttq_act_stats, without the workspace argument:
 * the partial sums live in a fixed scratch array in the library's device memory (1 MiB
 * of fp32 partial sums plus 1 KiB of counters, held on every GPU that loads the library
 * until the process exits). Limits: d <= 65536 channels, else TTQ_ERR_TOO_LARGE and
 * nothing is launched (at most about 600 blocks of 256 channels are launched, so the
 * partial sums of any d up to that limit fit in the array).
 * The first call on a device looks up the scratch array's device address (with that
 * device current); make that first call before any stream capture. The address is cached
 * per CUDA context: the first call in a new context (after cudaDeviceReset, or under a
 * caller's own driver-API context) looks it up again. Every call on a
 * device shares the one array and overwrites it (its counters are cleared by each
 * call): calls whose kernels overlap on the GPU (other streams, other host threads)
 * race and must be serialised by the caller. */
TTQ_API ttq_status ttq_act_stats_noalloc(const void* X_bf16, int64_t T, int64_t d, int64_t ld_x,
                                         float alpha, float lambda, int32_t p, float* s,
                                         cudaStream_t stream);

/* Re-quantization of W diag(s) ([DR] section 2 W_hat = Q[W D^(1/2)] D^(-1/2); [NR]
 * group-wise round-to-nearest quantize-dequantize). For each output row i and each
 * group G of g consecutive input channels: v = fl32(w * s), sigma = smallest fp16 >=
 * fl32((max v - min v) / (2^q - 1)), z = rint(fl32(-min v / sigma)) clamped to
 * [-2048, 2048], c = clamp(rint(fl32(v / sigma)) + z, 0, 2^q - 1); a zero range is
 * replaced by |min v| (or 1). rint rounds halves to even.
 *   W      device bf16 [d_out, d] (pass the residual R = W - B A when r > 0)
 *   s      device fp32 [d]
 *   codes  device uint32 [ttq_codes_words(d_out, d, q)] output
 *   scale  device fp16 [d_out, d/g] output (sigma)
 *   zero   device fp16 [d_out, d/g] output (z, an integer held in fp16)
 * Needs no workspace. Bit-exact and deterministic for given (W, s). */
TTQ_API ttq_status ttq_requant(const void* W_bf16, int64_t d_out, int64_t d, const float* s, int32_t q,
                       int32_t g, uint32_t* codes, void* scale_f16, void* zero_f16,
                       cudaStream_t stream);

/* Re-quantization of one weight for P prompts at once (P = 1 .. 8), each against its own
 * statistic, from a single read of W: the multi-prompt case that [DR] section 5 leaves
 * open (every request of a serving batch carries its own D). Prompt p's results equal
 * ttq_requant(W, s + p * d, ...) bit for bit.
 *   W      device bf16 [d_out, d]
 *   s      device fp32 [P, d], prompt-major
 *   codes  device uint32 [P, ttq_codes_words(d_out, d, q)] output
 *   scale  device fp16 [P, d_out, d/g] output;  zero  device fp16 [P, d_out, d/g] output
 * P outside 1 .. 8 returns TTQ_ERR_UNSUPPORTED. Needs no workspace. */
TTQ_API ttq_status ttq_requant_batched(const void* W_bf16, int64_t d_out, int64_t d, const float* s,
                                       int32_t prompts, int32_t q, int32_t g, uint32_t* codes, void* scale_f16,
                                       void* zero_f16, cudaStream_t stream);

/* One prompt through a TTQ linear layer ([DR] section 2 and section 6: statistics and
 * scale-quantize-rescale at prefill): s = stats(X); (codes, scale, zero) = requant(W, s);
 * Y = (X diag(1/s)) deq(codes)^T + (X A^T) B^T, where deq(c) = (c - z) * sigma is the
 * quantized weight in the scaled domain. diag(1/s) is folded into X (bf16) instead of
 * into the weight, so the tensor cores multiply bf16 X diag(1/s) by bf16 deq(codes)
 * with fp32 accumulation.
 *   X      device bf16 [T, d], contiguous
 *   W      device bf16 [d_out, d] (the residual R = W - B A when r > 0)
 *   A, B   device bf16 [r, d] and [d_out, r] when cfg->r > 0, else NULL
 *   s, codes, scale, zero   outputs as in ttq_act_stats / ttq_requant, kept by the
 *          caller for the decode steps that follow
 *   Y      device bf16 [T, d_out] output
 *   ws     device scratch of at least ttq_workspace_size(T, d, d_out, cfg) bytes
 * With r > 0 and T > 8 the statistic comes out of the same pass over X as X A^T: per
 * 64-token block and channel the sum of |x|^p, then the blocks added in order. It is
 * deterministic, and it equals ttq_act_stats's s up to the fp32 rounding of a different
 * summation order (a few units in the last place). */
TTQ_API ttq_status ttq_linear_prefill(const void* X_bf16, int64_t T, int64_t d, const void* W_bf16,
                              int64_t d_out, const void* A_bf16, const void* B_bf16,
                              const ttq_config* cfg, float* s, uint32_t* codes, void* scale_f16,
                              void* zero_f16, void* Y_bf16, void* ws, size_t ws_bytes,
                              cudaStream_t stream);

/* Decode steps reuse the prefill's quantized weight ([DR] section 6: parameters computed
 * at prefill are reused at decode): Y = (X diag(1/s)) deq(codes)^T + (X A^T) B^T for b
 * new token rows, with s, codes, scale and zero from ttq_linear_prefill (or from
 * ttq_act_stats + ttq_requant). Any b >= 1 is accepted.
 *   X      device bf16 [b, d], contiguous;  Y  device bf16 [b, d_out] output
 *   ws     device scratch of at least ttq_workspace_size(b, d, d_out, cfg) bytes */
TTQ_API ttq_status ttq_linear_decode(const void* X_bf16, int64_t b, int64_t d, int64_t d_out,
                             const float* s, const uint32_t* codes, const void* scale_f16,
                             const void* zero_f16, const void* A_bf16, const void* B_bf16,
                             const ttq_config* cfg, void* Y_bf16, void* ws, size_t ws_bytes,
                             cudaStream_t stream);

/* Prefill of P prompts (P = 1 .. 8) through one TTQ linear layer, each prompt with its own
 * statistic and hence its own quantized weight (the multi-prompt case [DR] section 5
 * leaves open): per prompt s_p = stats(X_p) and X_p diag(1/s_p); one read of W
 * re-quantized for every prompt (as ttq_requant_batched); then, when the prompts' tokens
 * fill 256-token tiles (more than 128 tokens in all, codes rows of 16-byte multiples,
 * d_out > 128), one grouped tensor-core launch over every prompt's output tiles, else one
 * projection per prompt. Prompt p's results equal ttq_linear_prefill on its own operands
 * (same s, codes, scale, zero; Y to the same rounding).
 *   X      device bf16 [T_0 + ... + T_{P-1}, d], the prompts' tokens one after another
 *   T      HOST int64 [P] tokens per prompt (each >= 1)
 *   s      device fp32 [P, d];  codes  device uint32 [P, ttq_codes_words(d_out, d, q)]
 *   scale, zero   device fp16 [P, d_out, d/g];  Y  device bf16 [sum T, d_out]
 *   ws     device scratch of at least ttq_prefill_batched_workspace_size(T, P, ...) bytes
 * d_out must be a multiple of 8 and every prompt's code words and scale/zero elements a
 * multiple of 16 bytes (TTQ_ERR_MISALIGNED otherwise). */
TTQ_API ttq_status ttq_prefill_batched_workspace_size(const int64_t* T, int32_t prompts, int64_t d, int64_t d_out,
                                                      const ttq_config* cfg, size_t* bytes);
TTQ_API ttq_status ttq_linear_prefill_batched(const void* X_bf16, const int64_t* T, int32_t prompts, int64_t d,
                                              const void* W_bf16, int64_t d_out, const void* A_bf16,
                                              const void* B_bf16, const ttq_config* cfg, float* s,
                                              uint32_t* codes, void* scale_f16, void* zero_f16, void* Y_bf16,
                                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* Decode steps of several requests at once, each with its own prefill's parameters: the
 * multi-request decode that [DR] section 5 leaves open (every request of a serving batch
 * carries its own D, hence its own codes). Request p computes
 * Y_p = (X_p diag(1/s_p)) deq(codes_p)^T + (X_p A^T) B^T with the shared static A, B; its
 * result equals ttq_linear_decode on request p's operands. With b <= 2 tokens per request
 * every request runs in the same two launches (statistic fold and CUDA-core GEMV over all
 * requests' codes); with more tokens the requests run one after another.
 *   X      device bf16 [P, b, d];  Y  device bf16 [P, b, d_out] output
 *   s      device fp32 [P, d];  codes  device uint32 [P, ttq_codes_words(d_out, d, q)]
 *   scale, zero   device fp16 [P, d_out, d/g]
 *   ws     device scratch of at least ttq_decode_batched_workspace_size(P, b, ...) bytes
 * P = requests, 1 .. 4096 (TTQ_ERR_UNSUPPORTED otherwise). */
TTQ_API ttq_status ttq_decode_batched_workspace_size(int32_t requests, int64_t b, int64_t d, int64_t d_out,
                                                     const ttq_config* cfg, size_t* bytes);
TTQ_API ttq_status ttq_linear_decode_batched(const void* X_bf16, int32_t requests, int64_t b, int64_t d,
                                             int64_t d_out, const float* s, const uint32_t* codes,
                                             const void* scale_f16, const void* zero_f16, const void* A_bf16,
                                             const void* B_bf16, const ttq_config* cfg, void* Y_bf16, void* ws,
                                             size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * Decoder layer around the TTQ linears. The layers whose linears TTQ re-quantizes are
 * the Qwen3 dense decoders of the architecture table on the thelatestinai.com listing of
 * the TTQ paper (Table 15: layers, heads, KV heads, hidden size, head dim, MLP dim); the
 * parts between the linears are the published Qwen3 layer: pre-norm RMSNorm (Zhang &
 * Sennrich 2019), per-head RMSNorm of q and k, rotary position embedding with the
 * half-split pairing (Su et al. 2021), grouped-query attention, SwiGLU MLP (Shazeer 2020).
 * Arithmetic is fp32 with one bf16 rounding per stored value. The library has the
 * prompt's causal attention (tensor cores) and the decode step's attention (one token
 * over the cache).
 * --------------------------------------------------------------------------------- */

/* RMSNorm over `rows` rows of n channels, with the residual add of a pre-norm layer:
 *   when residual != NULL:  r <- bf16(r + y)  (the residual row is replaced), h = r
 *   else:                   h = y
 *   out = bf16(h * w / sqrt(mean(h^2) + eps))
 *   y, residual, out   device bf16 [rows, n]; residual may be NULL; the three must be
 *                      distinct buffers (equal pointers: TTQ_ERR_INVALID_ARG) that do not
 *                      overlap
 *   w                  device bf16 [n]
 * n % 8 == 0, 8 <= n <= 8192; eps > 0 (an all-zero row then gives zeros). */
TTQ_API ttq_status ttq_rmsnorm(const void* y_bf16, void* residual_bf16, const void* w_bf16, int64_t rows,
                               int64_t n, float eps, void* out_bf16, cudaStream_t stream);

/* Rotary table: table[pos][i] = (cos, sin)(pos * base^(-2i/head_dim)) for pos < positions,
 * i < head_dim/2, computed in fp64 and stored as fp32 pairs.
 *   table   device fp32 [positions, head_dim/2, 2] output
 * head_dim in {64, 128, 256} (TTQ_ERR_UNSUPPORTED otherwise); base > 1. */
TTQ_API ttq_status ttq_rope_table(int64_t positions, int64_t head_dim, double base, float* table,
                                  cudaStream_t stream);

/* The attention inputs of T tokens at positions pos0 .. pos0+T-1 from the stacked q|k|v
 * projection: per head, q and k are RMS-normalised over head_dim (weights q_norm,
 * k_norm) and rotated (pair (i, i + head_dim/2) by the table's angle for the position);
 *   q   written back in place into qkv;
 *   k   written to k_cache[pos0 + t][kv head];  v  copied to v_cache[pos0 + t][kv head].
 *   qkv        device bf16 [T, (heads + 2 kv_heads) * head_dim]: q heads, k heads, v heads
 *   q_norm, k_norm   device bf16 [head_dim]
 *   rope_table device fp32 from ttq_rope_table (table_positions rows)
 *   k_cache, v_cache device bf16 [cache_len, kv_heads, head_dim]; positions outside
 *              pos0 .. pos0+T-1 are left untouched
 *   pos0_dev   NULL, or a device int64 holding pos0 (then the host pos0 is ignored): the
 *              form a captured CUDA graph replays at a new position every step. The
 *              kernel checks pos0 + T <= min(cache_len, table_positions) itself; out of
 *              range it writes nothing and ttq_device_status() reports TTQ_ERR_INVALID_ARG.
 * With a host pos0, pos0 + T must fit the cache and the table (TTQ_ERR_INVALID_ARG).
 * head_dim in {64, 128, 256}; eps > 0. */
TTQ_API ttq_status ttq_qk_norm_rope(void* qkv_bf16, int64_t T, int64_t heads, int64_t kv_heads,
                                    int64_t head_dim, const void* q_norm_bf16, const void* k_norm_bf16, float eps,
                                    const float* rope_table, int64_t table_positions, int64_t pos0,
                                    const int64_t* pos0_dev, void* k_cache_bf16, void* v_cache_bf16,
                                    int64_t cache_len, cudaStream_t stream);

/* Attention of one new token over the first L cache positions (grouped-query, causal by
 * construction: the cache holds only earlier positions and the token's own):
 *   out[h] = sum_p softmax_p(q_h . k_p / sqrt(head_dim)) v_p,  k, v of kv head h / (heads/kv_heads)
 *   q        device bf16 [heads * head_dim] (the token's q heads, e.g. the first row of the
 *            stacked projection after ttq_qk_norm_rope)
 *   k_cache, v_cache  device bf16 [cache_len, kv_heads, head_dim]
 *   L        = length, or *pos_dev + 1 when pos_dev (device int64, the token's position) is
 *            given; a device-side L outside 1 .. cache_len gives zeros and
 *            ttq_device_status() reports TTQ_ERR_INVALID_ARG
 *   out      device bf16 [heads * head_dim]
 *   ws       device scratch of ttq_decode_attention_workspace_size() bytes
 * Split over positions, each split an fp32 online softmax, merged in a fixed order (the
 * result is reproducible). head_dim in {64, 128}; heads / kv_heads in {1, 2, 4, 8}. */
TTQ_API ttq_status ttq_decode_attention_workspace_size(int64_t heads, int64_t kv_heads, int64_t head_dim,
                                                       int64_t cache_len, size_t* bytes);
TTQ_API ttq_status ttq_decode_attention(const void* q_bf16, int64_t heads, int64_t kv_heads, int64_t head_dim,
                                        const void* k_cache_bf16, const void* v_cache_bf16, int64_t cache_len,
                                        int64_t length, const int64_t* pos_dev, void* out_bf16, void* ws,
                                        size_t ws_bytes, cudaStream_t stream);

/* Causal grouped-query attention of a prompt at positions 0 .. T-1 on the tensor cores:
 *   out[t, h] = sum_{p <= t} softmax_p(q_t,h . k_p / sqrt(head_dim)) v_p   (k, v of kv head
 *   h / (heads / kv_heads)), with q from the stacked projection and k, v from the caches
 *   qkv        device bf16 [T, (heads + 2 kv_heads) * head_dim], the q heads first (as left by
 *              ttq_qk_norm_rope, which also wrote positions 0 .. T-1 of the caches)
 *   k_cache, v_cache  device bf16 [cache_len, kv_heads, head_dim], cache_len >= T
 *   out        device bf16 [T, heads * head_dim], distinct from qkv
 * One CTA per (tile of 128 queries, head) walks the key tiles up to its diagonal: S = Q K^T
 * and O += P V on tcgen05 with fp32 accumulators in tensor memory, an fp32 online softmax
 * (running row maximum and sum), P rounded to bf16 for the second product.
 * head_dim 64 or 128 (TTQ_ERR_UNSUPPORTED otherwise); heads % kv_heads == 0; T <= 2^24. */
TTQ_API ttq_status ttq_prompt_attention(const void* qkv_bf16, int64_t T, int64_t heads, int64_t kv_heads,
                                        int64_t head_dim, const void* k_cache_bf16, const void* v_cache_bf16,
                                        int64_t cache_len, void* out_bf16, cudaStream_t stream);

/* *pos_dev += n on the device, in stream order (moves a captured decode step to the next
 * position). */
TTQ_API ttq_status ttq_position_advance(int64_t* pos_dev, int64_t n, cudaStream_t stream);

/* SwiGLU gate: out[t, c] = bf16(silu(gu[t, c]) * gu[t, inter + c]), silu(u) = u/(1+e^-u).
 *   gate_up  device bf16 [rows, 2 inter]: the gate half, then the up half (the stacked
 *            [W_gate; W_up] projection's output);  out  device bf16 [rows, inter]
 * inter % 8 == 0; out must not overlap gate_up. */
TTQ_API ttq_status ttq_silu_mul(const void* gate_up_bf16, int64_t rows, int64_t inter, void* out_bf16,
                                cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the device error word: TTQ_OK, or
 * TTQ_ERR_TIMEOUT when a kernel gave up on a bounded wait since the last call,
 * TTQ_ERR_INVALID_ARG when a position read from device memory was out of range or a
 * kernel found its shared-memory allocation too small for its layout (it then did no
 * work), or TTQ_ERR_CUDA when the synchronisation itself failed. */
TTQ_API ttq_status ttq_device_status(cudaStream_t stream);

/* Sets the limit, in nanoseconds, after which a kernel waiting on an mbarrier gives up
 * and records TTQ_ERR_TIMEOUT (default 2e9, i.e. two seconds). Applies to launches made
 * after the call. A limit of 0 restores the default. */
TTQ_API ttq_status ttq_set_wait_limit_ns(uint64_t ns);

/* Test hook for failure detection: while enabled, every later launch of the tensor-core
 * kernel first waits on a barrier that nothing ever arrives at, so that wait runs out
 * after the limit set by ttq_set_wait_limit_ns; the kernel then records TTQ_ERR_TIMEOUT,
 * drains its own copies, frees its tensor memory and returns without writing Y. Used to
 * test the bounded waits; never enable it in production. */
TTQ_API ttq_status ttq_debug_inject_stall(int32_t enable);

/* Stage tracing for measurement. With n >= 6 event handles (cudaEvent_t created by the
 * caller with timing enabled), every later ttq_linear_prefill call records, on its
 * stream: events[0] before the statistics, [1] after them, [2] after the fold (and the
 * low-rank projection X A^T), [3] after the re-quantization, [4] after the tensor-core
 * projection and [5] after the split-K reduction (when there is none, [5] directly
 * follows [4]). n = 0 (or events = NULL) turns tracing off. The library keeps the
 * handles, not copies: they must stay valid while tracing is on. Not thread-safe. */
TTQ_API ttq_status ttq_set_trace_events(void* const* events, int32_t n);

/* The CUDA runtime error code behind the most recent TTQ_ERR_CUDA returned to this host
 * thread (0 when there was none), and a static description of such a code. */
TTQ_API int32_t ttq_last_cuda_error(void);
TTQ_API const char* ttq_cuda_error_string(int32_t code);

/* A static string naming a status code. */
TTQ_API const char* ttq_status_string(ttq_status status);

#ifdef __cplusplus
}
#endif

#endif /* TTQ_H_ */
