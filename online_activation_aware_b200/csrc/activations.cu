// Kernels over the activations X [T, d] (bf16, row-major):
//   act_stats   per-channel statistic s_j = (mean_t |x_tj|^p + lambda)^(alpha/p), the
//               online diagonal D^(1/2) of the prompt (paper-daily.com deep reading of
//               TTQ, section 2; gist.science German summary, section 2);
//   fold        X diag(1/s) in bf16, the operand the projection multiplies (the
//               D^(-1/2) of W_hat = Q[W D^(1/2)] D^(-1/2) moved onto the activations);
// Both are HBM-bound streaming passes: a warp reads 512 contiguous bytes of a row
// per step (32 lanes x 16 B), so every DRAM sector fetched is used in full.
#include <algorithm>
#include <climits>

#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kColsPerBlock = 256;  // 32 lanes x 8 bf16
constexpr int kRowWarps = 8;        // warps of a block walk rows 8 apart

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int P>
__device__ __forceinline__ void accum8(float (&acc)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float a = bf16lo_to_f32(w[j]);
    const float b = bf16hi_to_f32(w[j]);
    if (P == 2) {
      acc[2 * j] = __fmaf_rn(a, a, acc[2 * j]);      // bf16^2 is exact in fp32
      acc[2 * j + 1] = __fmaf_rn(b, b, acc[2 * j + 1]);
    } else {
      acc[2 * j] = __fadd_rn(acc[2 * j], fabsf(a));
      acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], fabsf(b));
    }
  }
}

__device__ __forceinline__ float finalize_scale(float colsum, float T, float alpha_over_p,
                                                float lambda) {
  const float m = __fdiv_rn(colsum, T);  // mean over the prompt's tokens
  return powf(__fadd_rn(m, lambda), alpha_over_p);
}

// grid: (col_blocks, nsplit); block: 256 threads. Each block reduces its rows for 256
// columns into partial[split, col]; the last block of a column strip (in arrival order,
// counted in `counters`) sums the strip's partials in split order and writes s. The
// summation order is fixed, so the result does not depend on scheduling.
template <int P>
__global__ void __launch_bounds__(256) act_stats_kernel(const __nv_bfloat16* __restrict__ X,
                                                        int64_t T, int d, int64_t ld_x,
                                                        int64_t rows_per_split, int nsplit,
                                                        float alpha_over_p, float lambda,
                                                        float* __restrict__ partial,
                                                        unsigned* __restrict__ counters,
                                                        float* __restrict__ s) {
  __shared__ float red[kRowWarps][kColsPerBlock];
  __shared__ int is_last;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int col0 = blockIdx.x * kColsPerBlock + lane * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(T, r0 + rows_per_split);

  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  if (col0 < d) {
    const __nv_bfloat16* base = X + col0;
    int64_t r = r0 + warp;
    for (; r + 3 * kRowWarps < r1; r += 4 * kRowWarps) {
      const uint4 v0 = ld_stream(base + r * ld_x);
      const uint4 v1 = ld_stream(base + (r + kRowWarps) * ld_x);
      const uint4 v2 = ld_stream(base + (r + 2 * kRowWarps) * ld_x);
      const uint4 v3 = ld_stream(base + (r + 3 * kRowWarps) * ld_x);
      accum8<P>(acc, v0);
      accum8<P>(acc, v1);
      accum8<P>(acc, v2);
      accum8<P>(acc, v3);
    }
    for (; r < r1; r += kRowWarps) accum8<P>(acc, ld_stream(base + r * ld_x));
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = acc[j];
  __syncthreads();

  const int col = blockIdx.x * kColsPerBlock + threadIdx.x;
  float sum = 0.f;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) sum = __fadd_rn(sum, red[w][threadIdx.x]);

  if (nsplit == 1) {
    if (col < d) s[col] = finalize_scale(sum, static_cast<float>(T), alpha_over_p, lambda);
    return;
  }
  if (col < d) partial[static_cast<int64_t>(blockIdx.y) * d + col] = sum;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&counters[blockIdx.x], 1u);
    is_last = (prev == static_cast<unsigned>(nsplit - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (col < d) {
    float tot = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) tot = __fadd_rn(tot, __ldcg(&partial[static_cast<int64_t>(sp) * d + col]));
    s[col] = finalize_scale(tot, static_cast<float>(T), alpha_over_p, lambda);
  }
  if (threadIdx.x == 0) counters[blockIdx.x] = 0u;  // leave the strip counter ready
}

// The statistic as two launches that need no grid-wide synchronisation:
//   stats_partial_kernel  block (strip c, split k) sums |x|^p over its rows of a 256-column
//                         strip into partial[k, strip columns] (fp32, fixed order);
//   stats_finish_kernel   launched as the programmatic dependent of the first (its blocks
//                         are resident and waiting when the partial sums land); block c
//                         reduces strip c's partials in a fixed order (warp w takes splits
//                         w, w + 8, ...; the eight warp sums are then added in warp order)
//                         and writes s for the strip.
// The partial grid is sized to balance the rows each SM reads.
template <int P>
__global__ void __launch_bounds__(256, 5) stats_partial_kernel(const __nv_bfloat16* __restrict__ X, int64_t T,
                                                            int d, int64_t ld_x, int64_t rows_per_split,
                                                            float* __restrict__ partial) {
  __shared__ float red[kRowWarps][kColsPerBlock];
  grid_dep_launch();  // the fold kernel's blocks may take their places now
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int col0 = blockIdx.x * kColsPerBlock + lane * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(T, r0 + rows_per_split);
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  if (col0 < d) {
    const __nv_bfloat16* base = X + col0;
    // batches of 8 rows with all 8 loads in flight per lane, then the rest in predicated
    // batches of 4 (a row past the end reads as zero, which adds nothing)
    int64_t r = r0 + warp;
    for (; r + 7 * kRowWarps < r1; r += 8 * kRowWarps) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = ld_stream(base + (r + i * kRowWarps) * ld_x);
#pragma unroll
      for (int i = 0; i < 8; ++i) accum8<P>(acc, v[i]);
    }
    for (; r < r1; r += 4 * kRowWarps) {
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t rr = r + i * kRowWarps;
        v[i] = rr < r1 ? ld_stream(base + rr * ld_x) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) accum8<P>(acc, v[i]);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = acc[j];
  __syncthreads();
  const int col = blockIdx.x * kColsPerBlock + threadIdx.x;
  float sum = 0.f;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) sum = __fadd_rn(sum, red[w][threadIdx.x]);
  if (col < d) partial[static_cast<int64_t>(blockIdx.y) * d + col] = sum;
}

// s for the 256 columns of strip blockIdx.x from partial[nsplit, d], into s_out (shared
// memory, 256 floats; columns past d get 1). Needs all 256 threads; `red` is 8 x 256
// floats of shared scratch.
__device__ __forceinline__ void strip_scale(const float* __restrict__ partial, int d, int nsplit, float T,
                                            float alpha_over_p, float lambda, float (*red)[kColsPerBlock],
                                            float* s_out) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int col0 = blockIdx.x * kColsPerBlock + lane * 8;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  if (col0 < d) {
    constexpr int U = 2;  // splits in flight per warp
    for (int k0 = warp; k0 < nsplit; k0 += U * kRowWarps) {
      float4 va[U], vb[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + u * kRowWarps;
        if (k < nsplit) {
          const float* p = partial + static_cast<int64_t>(k) * d + col0;
          va[u] = __ldcg(reinterpret_cast<const float4*>(p));
          vb[u] = __ldcg(reinterpret_cast<const float4*>(p + 4));
        } else {
          va[u] = vb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        acc[0] = __fadd_rn(acc[0], va[u].x);
        acc[1] = __fadd_rn(acc[1], va[u].y);
        acc[2] = __fadd_rn(acc[2], va[u].z);
        acc[3] = __fadd_rn(acc[3], va[u].w);
        acc[4] = __fadd_rn(acc[4], vb[u].x);
        acc[5] = __fadd_rn(acc[5], vb[u].y);
        acc[6] = __fadd_rn(acc[6], vb[u].z);
        acc[7] = __fadd_rn(acc[7], vb[u].w);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = acc[j];
  __syncthreads();
  const int col = blockIdx.x * kColsPerBlock + threadIdx.x;
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) tot = __fadd_rn(tot, red[w][threadIdx.x]);
  s_out[threadIdx.x] = col < d ? finalize_scale(tot, T, alpha_over_p, lambda) : 1.f;
  __syncthreads();
}

// s alone from the partial sums: one block per strip (the finishing step of ttq_act_stats).
__global__ void __launch_bounds__(256) stats_finish_kernel(const float* __restrict__ partial, int d, int nsplit,
                                                           float T, float alpha_over_p, float lambda,
                                                           float* __restrict__ s) {
  __shared__ float red[kRowWarps][kColsPerBlock];
  __shared__ float s_sm[kColsPerBlock];
  grid_dep_wait();
  grid_dep_launch();
  strip_scale(partial, d, nsplit, T, alpha_over_p, lambda, red, s_sm);
  const int col = blockIdx.x * kColsPerBlock + threadIdx.x;
  if (col < d) s[col] = s_sm[threadIdx.x];
}

// grid: (col_blocks, row_splits); each thread owns 8 consecutive columns for all rows
// of its split, so the 8 reciprocals 1/s are formed once per thread.
__global__ void __launch_bounds__(256) fold_kernel(const __nv_bfloat16* __restrict__ X, int64_t T,
                                                   int d, int64_t ld_x,
                                                   const float* __restrict__ s,
                                                   int64_t rows_per_split,
                                                   __nv_bfloat16* __restrict__ Xf) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int col0 = blockIdx.x * kColsPerBlock + lane * 8;
  if (col0 >= d) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(T, r0 + rows_per_split);
  const float4 sa = *reinterpret_cast<const float4*>(s + col0);
  const float4 sb = *reinterpret_cast<const float4*>(s + col0 + 4);
  const float rs[8] = {__frcp_rn(sa.x), __frcp_rn(sa.y), __frcp_rn(sa.z), __frcp_rn(sa.w),
                       __frcp_rn(sb.x), __frcp_rn(sb.y), __frcp_rn(sb.z), __frcp_rn(sb.w)};
  for (int64_t r = r0 + warp; r < r1; r += kRowWarps) {
    const uint4 v = ld_stream(X + r * ld_x + col0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      o[j] = pack_bf16x2(__fmul_rn(bf16lo_to_f32(w[j]), rs[2 * j]),
                         __fmul_rn(bf16hi_to_f32(w[j]), rs[2 * j + 1]));
    *reinterpret_cast<uint4*>(Xf + r * d + col0) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

StatsPlan stats_plan(int64_t T, int64_t d) {
  StatsPlan p;
  p.col_blocks = static_cast<int>((d + kColsPerBlock - 1) / kColsPerBlock);
  // aim for about 4 blocks of 256 threads per SM on a 148-SM part, with at least 64
  // rows per split so each warp streams a few rows
  const int64_t target_blocks = 148 * 4;
  int64_t ns = (target_blocks + p.col_blocks - 1) / p.col_blocks;
  const int64_t max_ns = (T + 63) / 64;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  if (ns > 1024) ns = 1024;
  p.rows_per_split = (T + ns - 1) / ns;
  p.nsplit = static_cast<int>((T + p.rows_per_split - 1) / p.rows_per_split);
  return p;
}

StatsPlan split_plan(int64_t T, int64_t d, int num_sms) {
  StatsPlan p;
  p.col_blocks = static_cast<int>((d + kColsPerBlock - 1) / kColsPerBlock);
  if (num_sms < 1) num_sms = 1;
  // the row split that best balances the rows each SM reduces (blocks per SM rounded up,
  // times rows per block), with at least 32 rows per split; fewer splits win ties
  const int64_t max_ns = std::max<int64_t>(1, std::min<int64_t>(1024, (T + 31) / 32));
  int64_t best_ns = 1, best_cost = INT64_MAX;
  for (int64_t ns = 1; ns <= max_ns; ++ns) {
    const int64_t per_sm = (static_cast<int64_t>(p.col_blocks) * ns + num_sms - 1) / num_sms;
    const int64_t cost = per_sm * ((T + ns - 1) / ns);
    if (cost < best_cost) {
      best_cost = cost;
      best_ns = ns;
    }
  }
  p.rows_per_split = (T + best_ns - 1) / best_ns;
  p.nsplit = static_cast<int>((T + p.rows_per_split - 1) / p.rows_per_split);
  return p;
}

size_t split_partial_bytes(int64_t T, int64_t d, int num_sms) {
  return static_cast<size_t>(split_plan(T, d, num_sms).nsplit) * static_cast<size_t>(d) * sizeof(float);
}

namespace {

template <typename K, typename... Args>
cudaError_t launch_dependent(K kernel, dim3 grid, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int P>
cudaError_t launch_partials(const __nv_bfloat16* X, int64_t T, int d, int64_t ld_x, const StatsPlan& pl,
                            float* partial, cudaStream_t stream) {
  stats_partial_kernel<P><<<dim3(pl.col_blocks, pl.nsplit), 256, 0, stream>>>(X, T, d, ld_x, pl.rows_per_split,
                                                                               partial);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_act_stats(const void* X, int64_t T, int64_t d, int64_t ld_x, float alpha, float lambda, int p,
                             float* s, float* partial, int num_sms, cudaStream_t stream) {
  const StatsPlan pl = split_plan(T, d, num_sms);
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const int di = static_cast<int>(d);
  cudaError_t e = p == 2 ? launch_partials<2>(Xb, T, di, ld_x, pl, partial, stream)
                         : launch_partials<1>(Xb, T, di, ld_x, pl, partial, stream);
  if (e != cudaSuccess) return e;
  const float ap = alpha / static_cast<float>(p);
  return launch_dependent(stats_finish_kernel, dim3(pl.col_blocks), stream, static_cast<const float*>(partial), di,
                          pl.nsplit, static_cast<float>(T), ap, lambda, s);
}

cudaError_t launch_act_stats_capped(const void* X, int64_t T, int64_t d, int64_t ld_x, float alpha,
                                    float lambda, int p, float* s, float* partial,
                                    int64_t max_partial_floats, unsigned* counters,
                                    cudaStream_t stream) {
  StatsPlan pl = stats_plan(T, d);
  // stats_plan launches at most about 592 + col_blocks blocks (nsplit <= ceil(592 /
  // col_blocks)), so nsplit * d <= (592 + col_blocks) * 256 floats: 217,088 for d = 65,536,
  // below the 262,144 of the allocation-free entry point's array. The branch below only
  // guards callers with a smaller array.
  if (static_cast<int64_t>(pl.nsplit) * d > max_partial_floats) {
    int64_t ns = max_partial_floats / d;
    if (ns < 1) ns = 1;
    pl.rows_per_split = (T + ns - 1) / ns;
    pl.nsplit = static_cast<int>((T + pl.rows_per_split - 1) / pl.rows_per_split);
  }
  if (pl.nsplit > 1) {
    cudaError_t e = cudaMemsetAsync(counters, 0, pl.col_blocks * sizeof(unsigned), stream);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(pl.col_blocks, pl.nsplit);
  const float ap = alpha / static_cast<float>(p);
  if (p == 2)
    act_stats_kernel<2><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(X), T,
                                                  static_cast<int>(d), ld_x, pl.rows_per_split,
                                                  pl.nsplit, ap, lambda, partial, counters, s);
  else
    act_stats_kernel<1><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(X), T,
                                                  static_cast<int>(d), ld_x, pl.rows_per_split,
                                                  pl.nsplit, ap, lambda, partial, counters, s);
  return cudaGetLastError();
}

cudaError_t launch_fold(const void* X, int64_t T, int64_t d, int64_t ld_x, const float* s,
                        void* Xf, cudaStream_t stream) {
  const int col_blocks = static_cast<int>((d + kColsPerBlock - 1) / kColsPerBlock);
  const int64_t target_blocks = 148 * 8;
  int64_t ns = (target_blocks + col_blocks - 1) / col_blocks;
  const int64_t max_ns = (T + 31) / 32;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  if (ns > 65535) ns = 65535;
  const int64_t rps = (T + ns - 1) / ns;
  ns = (T + rps - 1) / rps;
  dim3 grid(col_blocks, static_cast<unsigned>(ns));
  fold_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(X), T,
                                        static_cast<int>(d), ld_x, s, rps,
                                        static_cast<__nv_bfloat16*>(Xf));
  return cudaGetLastError();
}

}  // namespace ttq
