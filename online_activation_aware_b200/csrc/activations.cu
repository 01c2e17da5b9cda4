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
constexpr int kStatsLoads = 16;     // 16-byte loads in flight per lane in the statistic

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The same load without `volatile`: X is read-only for the whole kernel, so the compiler
// may hoist a batch of these ahead of the arithmetic that consumes them (every load of
// the batch in flight at once).
__device__ __forceinline__ uint4 ld_stream_batch(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
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

// The statistic in one launch, with no global scratch: block (strip c, split k) sums
// |x|^p over its rows of a 256-column strip; the `nsplit` blocks of a strip form one
// thread-block cluster, and its first block adds the others' column sums straight out of
// their shared memory (distributed shared memory), in split order, and writes s.
//   - each lane keeps NLD 16-byte loads of its own rows in flight (a warp reads 512
//     contiguous bytes of a row per load), the tail in predicated batches of NLD/2;
//   - the order of every sum is fixed (lanes' rows in row order, warps in warp order,
//     splits in cluster rank order), so s is deterministic;
//   - the kernel is launched as a programmatic dependent (its launch overlaps the tail
//     of the kernel ahead, which it waits for before it reads X), and once that wait is
//     over lets the next kernel of the stream launch: that kernel's set-up and first loads
//     overlap this pass over X.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// fp32 at the same shared-memory offset in cluster block `rank`.
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Waits for a copy to land, bounded by a fixed two seconds whatever the caller's wait
// limit (used only to drain copies in flight before a block that gave up exits).
__device__ __forceinline__ void mbar_drain_stats(uint32_t bar, uint32_t parity, const DevErr& err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 2000000000ull) {
      atomicOr(err.word, kErrTimeout);
      return;
    }
  }
}

template <int P, int NLD>
__global__ void __launch_bounds__(256) stats_cluster_kernel(const __nv_bfloat16* __restrict__ X, int64_t T, int d,
                                                            int64_t ld_x, int64_t rows_per_split, int nsplit,
                                                            float alpha_over_p, float lambda,
                                                            float* __restrict__ s) {
  __shared__ float red[kRowWarps][kColsPerBlock];
  __shared__ float colsum[kColsPerBlock];
  pdl_enter();  // X (and s) may be written by the kernel ahead in the stream
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
    for (; r + (NLD - 1) * kRowWarps < r1; r += NLD * kRowWarps) {
      uint4 v[NLD];
#pragma unroll
      for (int i = 0; i < NLD; ++i) v[i] = ld_stream_batch(base + (r + i * kRowWarps) * ld_x);
#pragma unroll
      for (int i = 0; i < NLD; ++i) accum8<P>(acc, v[i]);
    }
    constexpr int H = NLD / 2;
    for (; r < r1; r += H * kRowWarps) {
      uint4 v[H];
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const int64_t rr = r + i * kRowWarps;
        v[i] = rr < r1 ? ld_stream_batch(base + rr * ld_x) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < H; ++i) accum8<P>(acc, v[i]);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = acc[j];
  __syncthreads();
  float sum = 0.f;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) sum = __fadd_rn(sum, red[w][threadIdx.x]);
  colsum[threadIdx.x] = sum;
  // every block of the cluster reaches both barriers (no early exit above): the first
  // makes all column sums visible, the second keeps each block's shared memory alive
  // until the first block has read it
  cluster_sync_all();
  if (cluster_rank() == 0) {
    float tot = 0.f;
    for (int k = 0; k < nsplit; ++k) tot = __fadd_rn(tot, ld_dsmem_f32(&colsum[threadIdx.x], k));
    const int col = blockIdx.x * kColsPerBlock + threadIdx.x;
    if (col < d) s[col] = finalize_scale(tot, static_cast<float>(T), alpha_over_p, lambda);
  }
  cluster_sync_all();
}

// The same statistic with X streamed by TMA: a producer warp loads tiles of 32 rows x
// 256 columns (16 KB) of the block's strip into a 4-stage shared-memory ring (no
// multicast; rows and columns outside X read as zeros), and eight consumer warps reduce
// them (warp w takes rows w, w + 8, w + 16, w + 24 of a tile; a lane reads 16 bytes of
// each, a warp the row's 512 contiguous bytes, so shared-memory reads are conflict-free).
// The bytes in flight per SM are set by the ring (64 KB per block), not by registers.
// Rows of the last tile that belong to the next split are skipped by the consumers.
// Every mbarrier wait is bounded; a block that gives up drains its copies and still
// meets its cluster at both barriers (its s is then wrong, and the device error word
// says so).
constexpr int kStatsTileRows = 32;
constexpr int kStatsStages = 4;
constexpr uint32_t kStatsTileBytes = kStatsTileRows * kColsPerBlock * 2;

struct StatsSmem {
  uint8_t tile[kStatsStages][kStatsTileBytes];
  uint64_t full[kStatsStages];
  uint64_t empty[kStatsStages];
  float red[kRowWarps][kColsPerBlock];
  float colsum[kColsPerBlock];
  int abort_flag;
};
constexpr size_t kStatsSmemBytes = sizeof(StatsSmem) + 128;  // + room to align the base to 128 B

template <int P>
__global__ void __launch_bounds__(288) stats_tma_kernel(const __grid_constant__ CUtensorMap tm_x, int64_t T, int d,
                                                        int64_t rows_per_split, int nsplit, float alpha_over_p,
                                                        float lambda, float* __restrict__ s, DevErr err) {
  extern __shared__ uint8_t smem_raw[];
  StatsSmem* sm = reinterpret_cast<StatsSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  pdl_enter();  // X (and s) may be written by the kernel ahead in the stream
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(T, r0 + rows_per_split);
  const int ntiles = r1 > r0 ? static_cast<int>((r1 - r0 + kStatsTileRows - 1) / kStatsTileRows) : 0;
  volatile int* abort_flag = &sm->abort_flag;
  const uint32_t full0 = smem_addr(&sm->full[0]);
  const uint32_t empty0 = smem_addr(&sm->empty[0]);
  if (tid == 0) {
    for (int i = 0; i < kStatsStages; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kRowWarps);
    }
    sm->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  if (warp == kRowWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      const int x0 = blockIdx.x * kColsPerBlock;
      int i = 0;
      for (; i < ntiles; ++i) {
        const int st = i % kStatsStages;
        if (i >= kStatsStages && !mbar_wait(empty0 + 8 * st, ((i / kStatsStages) - 1) & 1, err, abort_flag)) break;
        mbar_arrive_expect_tx(full0 + 8 * st, kStatsTileBytes);
        tma_load_2d(smem_addr(sm->tile[st]), &tm_x, full0 + 8 * st, x0,
                    static_cast<int>(r0 + static_cast<int64_t>(i) * kStatsTileRows));
      }
      if (*abort_flag) {
        // let every copy this block started land before its shared memory is released
        for (int k = i > kStatsStages ? i - kStatsStages : 0; k < i; ++k)
          mbar_drain_stats(full0 + 8 * (k % kStatsStages), (k / kStatsStages) & 1, err);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kStatsStages;
      // warp-uniform: either every lane of the warp consumes the tile or none does
      if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8 * st, (i / kStatsStages) & 1, err, abort_flag) ? 1 : 0))
        break;
      const uint8_t* t = sm->tile[st];
      const int64_t row0 = r0 + static_cast<int64_t>(i) * kStatsTileRows;
#pragma unroll
      for (int j = 0; j < kStatsTileRows / kRowWarps; ++j) {
        const int row = warp + kRowWarps * j;
        if (row0 + row < r1) accum8<P>(acc, *reinterpret_cast<const uint4*>(t + row * 512 + lane * 16));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
  }
  if (warp < kRowWarps) {
#pragma unroll
    for (int j = 0; j < 8; ++j) sm->red[warp][lane * 8 + j] = acc[j];
  }
  __syncthreads();
  if (tid < kColsPerBlock) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kRowWarps; ++w) sum = __fadd_rn(sum, sm->red[w][tid]);
    sm->colsum[tid] = sum;
  }
  cluster_sync_all();
  if (cluster_rank() == 0 && tid < kColsPerBlock) {
    float tot = 0.f;
    for (int k = 0; k < nsplit; ++k) tot = __fadd_rn(tot, ld_dsmem_f32(&sm->colsum[tid], k));
    const int col = blockIdx.x * kColsPerBlock + tid;
    if (col < d) s[col] = finalize_scale(tot, static_cast<float>(T), alpha_over_p, lambda);
  }
  cluster_sync_all();
}

// grid: (col_blocks, row_splits); each thread owns 8 consecutive columns for all rows
// of its split, so the 8 reciprocals 1/s are formed once per thread.
__global__ void __launch_bounds__(256) fold_kernel(const __nv_bfloat16* __restrict__ X, int64_t T,
                                                   int d, int64_t ld_x,
                                                   const float* __restrict__ s,
                                                   int64_t rows_per_split,
                                                   __nv_bfloat16* __restrict__ Xf) {
  pdl_enter();
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

StatsPlan cluster_plan(int64_t T, int64_t d, int num_sms) {
  StatsPlan p;
  p.col_blocks = static_cast<int>((d + kColsPerBlock - 1) / kColsPerBlock);
  if (num_sms < 1) num_sms = 1;
  // about two blocks per SM: the row split is the smallest power of two (a cluster size)
  // that reaches 2 * num_sms blocks, at most kStatsMaxSplit, and at most ceil(T / 32), so
  // a split has at least 32 rows. Then ceil(T / ns) >= 32 > ns, which makes the number of
  // non-empty splits exactly ns.
  const int64_t want = (2 * static_cast<int64_t>(num_sms) + p.col_blocks - 1) / p.col_blocks;
  const int64_t cap = std::min<int64_t>(kStatsMaxSplit, (T + 31) / 32);
  int64_t ns = 1;
  while (ns < want && 2 * ns <= cap) ns *= 2;
  p.rows_per_split = (T + ns - 1) / ns;
  p.nsplit = static_cast<int>((T + p.rows_per_split - 1) / p.rows_per_split);
  return p;
}

namespace {

template <int P, int NLD>
cudaError_t launch_cluster_stats(const __nv_bfloat16* X, int64_t T, int d, int64_t ld_x, const StatsPlan& pl,
                                 float ap, float lambda, float* s, cudaStream_t stream) {
  auto kernel = stats_cluster_kernel<P, NLD>;
  if (pl.nsplit > 8) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.col_blocks, pl.nsplit);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(pl.nsplit);
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, X, T, d, ld_x, pl.rows_per_split, pl.nsplit, ap, lambda, s);
}

template <int P>
cudaError_t launch_tma_stats(const CUtensorMap& map, int64_t T, int d, const StatsPlan& pl, float ap, float lambda,
                             float* s, const DevErr& err, cudaStream_t stream) {
  auto kernel = stats_tma_kernel<P>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kStatsSmemBytes));
  if (e == cudaSuccess && pl.nsplit > 8) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.col_blocks, pl.nsplit);
  cfg.blockDim = dim3((kRowWarps + 1) * 32);
  cfg.dynamicSmemBytes = kStatsSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(pl.nsplit);
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, map, T, d, pl.rows_per_split, pl.nsplit, ap, lambda, s, err);
}

}  // namespace

cudaError_t launch_act_stats(const void* X, int64_t T, int64_t d, int64_t ld_x, float alpha, float lambda, int p,
                             float* s, int num_sms, const DevErr& err, cudaStream_t stream) {
  const StatsPlan pl = cluster_plan(T, d, num_sms);
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const int di = static_cast<int>(d);
  const float ap = alpha / static_cast<float>(p);
  // X as a 2-D tensor [T, d] with row pitch ld_x (16-byte multiple, base 16-byte aligned),
  // boxes of 32 rows x 256 columns; where the driver declines the map, the same reduction
  // runs from plain loads
  CUtensorMap map;
  if (T < (int64_t(1) << 30) && encode_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, static_cast<uint64_t>(T), static_cast<uint64_t>(d),
                     static_cast<uint64_t>(ld_x), kColsPerBlock, kStatsTileRows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return p == 2 ? launch_tma_stats<2>(map, T, di, pl, ap, lambda, s, err, stream)
                  : launch_tma_stats<1>(map, T, di, pl, ap, lambda, s, err, stream);
  return p == 2 ? launch_cluster_stats<2, kStatsLoads>(Xb, T, di, ld_x, pl, ap, lambda, s, stream)
                : launch_cluster_stats<1, kStatsLoads>(Xb, T, di, ld_x, pl, ap, lambda, s, stream);
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
  return launch_pdl(fold_kernel, grid, dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(X), T,
                    static_cast<int>(d), ld_x, s, rps, static_cast<__nv_bfloat16*>(Xf));
}

}  // namespace ttq
