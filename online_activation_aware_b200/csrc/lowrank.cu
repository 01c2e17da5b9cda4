// The static low-rank side path of TTQ: U = X A^T, the [T, r] projection that the
// tensor-core GEMM multiplies by B in its extra K block (gist.science French summary,
// section 2B: W_hat = W_q + B A with B, A fixed from the SVD; paper-daily.com deep
// reading, section 2: low-rank compensation of the quantization residual).
//
// A skinny product (r <= 64 outputs per token) bound by the single read of X. Block
// (token block of 64, K split ks) streams its [64 x Kc] slice of X and the matching
// [r x Kc] slice of A by TMA through a 4-stage ring in shared memory (128-byte swizzle, so
// that ldmatrix is conflict-free; a producer warp issues the copies and the consumer
// warps hand stages back on mbarriers), and each of its first 4 warps multiplies 16
// tokens by A^T with mma.sync m16n8k16 (bf16 in, fp32 accumulate). The K splits write
// fp32 partial sums; a small dependent kernel adds them in split order (deterministic)
// and stores U in bf16 with its row padded to 64 (columns r..63 zero). For a few tokens (a
// decode step) one block computes each output over all of d instead.
//
// A prefill also needs the statistic s of the same X (paper-daily.com deep reading, section
// 2: s from the prompt's per-channel |x|^p means). With P = 1 or 2 the partial kernel sums
// |x|^p over its 64 tokens for every channel of each stage while the stage sits in shared
// memory (for r >= 32 in 4 more warps of its own), and the dependent kernel adds those
// rows in token-block order and finishes s: one read of X serves both, where a separate
// statistic kernel would read it once more.
#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kLrTok = 64;      // tokens per block (4 warps x 16)
constexpr int kLrK = 64;        // K per stage
constexpr int kLrStages = 4;
constexpr int kLrSmallTokens = 8;  // up to here one block per output (no partial sums in memory)

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of 16-byte chunk c (0..7) of row `row` in a [rows x 64] bf16 tile as the
// 128-byte TMA swizzle lays it out (tile base 1024-byte aligned)
__device__ __forceinline__ uint32_t swz(int row, int c) { return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4)); }

// Consumer warps of a block: with the statistic and r >= 32 four more warps take the
// statistic (the multiplying warps are busier there); otherwise the 4 warps do both.
template <int NT, int P>
constexpr int lr_consumer_warps() { return (P != 0 && NT >= 4) ? 8 : 4; }
template <int NT, int P>
constexpr int lr_threads() { return 32 * (lr_consumer_warps<NT, P>() + 1); }  // + the TMA producer warp

// Shared memory of a block: kLrStages x (X tile [64 x 64], A tile [R x 64]), 1024-byte
// aligned tiles, then the stage barriers and an abort flag.
template <int NT>
constexpr uint32_t lr_stage_bytes() { return kLrTok * kLrK * 2 + NT * 8 * kLrK * 2; }
template <int NT>
constexpr size_t lr_smem_bytes() { return 1024 + kLrStages * lr_stage_bytes<NT>() + 2 * kLrStages * 8 + 16; }

// Waits (bounded by a fixed two seconds) for the copies of a stage to land before the
// block's shared memory is released after an abort.
__device__ __forceinline__ void lr_drain(uint32_t bar, uint32_t parity, const DevErr& err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 2000000000ull) {
      atomicOr(err.word, kErrTimeout);
      return;
    }
  }
}

// grid: (token blocks, K splits); NT = r / 8 output tiles of 8 ranks; P = 0 (U only) or the
// statistic's exponent, whose per-block column sums go to spart[token block][channel].
// The last warp streams the block's X tiles [64 tokens x 64 channels] and A tiles
// [r x 64] by TMA (128-byte swizzle; rows past T and channels past d read as zero) into a
// ring of kLrStages stages (`full` barriers count the bytes); each consumer warp hands a
// stage back on its `empty` barrier when it is done with it, so the warps never meet at a
// block barrier.
template <int NT, int P>
__global__ void __launch_bounds__(lr_threads<NT, P>(), 2) lowrank_partial_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a, int T, int d, int kc,
    float* __restrict__ part, float* __restrict__ spart, const DevErr err) {
  constexpr int R = NT * 8;
  constexpr uint32_t kXBytes = kLrTok * kLrK * 2;  // 8 KB
  constexpr uint32_t kStage = lr_stage_bytes<NT>();
  constexpr int kCons = lr_consumer_warps<NT, P>();
  constexpr bool kSplit = kCons > 4;  // warps 4..7 take the statistic
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);  // the same stages through a generic pointer
  const uint32_t bar_full = sbase + kLrStages * kStage;
  const uint32_t bar_empty = bar_full + 8 * kLrStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kLrStages * kStage + 16 * kLrStages);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int t0 = blockIdx.x * kLrTok;
  const int k0 = blockIdx.y * kc;
  const int k1 = min(d, k0 + kc);
  const int nst = (k1 - k0 + kLrK - 1) / kLrK;

  if (tid == 0) {
    for (int s = 0; s < kLrStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kCons);  // one arrival per consumer warp
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_a);
  }
  __syncthreads();
  pdl_enter();  // X (and A) are read only after the kernel ahead has finished

  if (warp == kCons) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int st = 0; st < nst; ++st) {
        const int s = st % kLrStages;
        if (st >= kLrStages && !mbar_wait(bar_empty + 8 * s, ((st / kLrStages) - 1) & 1, err, abort_flag)) break;
        const uint32_t xs = sbase + s * kStage;
        mbar_arrive_expect_tx(bar_full + 8 * s, kStage);
        tma_load_2d(xs, &tm_x, bar_full + 8 * s, k0 + st * kLrK, t0);
        tma_load_2d(xs + kXBytes, &tm_a, bar_full + 8 * s, k0 + st * kLrK, 0);
        ++issued;
      }
      if (*abort_flag) {
        // every copy this block started lands before its shared memory is released
        for (int st = issued > kLrStages ? issued - kLrStages : 0; st < issued; ++st)
          lr_drain(bar_full + 8 * (st % kLrStages), (st / kLrStages) & 1, err);
      }
    }
    return;
  }

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[n][j] = 0.f;

  for (int st = 0; st < nst; ++st) {
    const int s = st % kLrStages;
    if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, (st / kLrStages) & 1, err, abort_flag) ? 1 : 0)) break;
    const uint32_t xs = sbase + s * kStage;
    const uint32_t as = xs + kXBytes;
#pragma unroll
    for (int kk = 0; kk < kLrK / 16 && (!kSplit || warp < 4); ++kk) {
      // A fragment: this warp's 16 tokens x 16 k (matrices: rows 0-7 / 8-15, k 0-7 / 8-15)
      uint32_t af[4];
      {
        const int mi = lane >> 3;
        const int row = warp * 16 + (lane & 7) + ((mi & 1) << 3);
        const int c = kk * 2 + (mi >> 1);
        ldmatrix_x4(xs + swz(row, c), af);
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        // B fragment: ranks 8n..8n+7 x 16 k (A is stored rank-major, k contiguous)
        uint32_t bf[2];
        const int mi = (lane >> 3) & 1;
        const int row = n * 8 + (lane & 7);
        ldmatrix_x2(as + swz(row, kk * 2 + mi), bf);
        mma_bf16_16816(acc[n], af, bf[0], bf[1]);
      }
    }
    if (P != 0 && (!kSplit || warp >= 4)) {
      // sum of |x|^p over the block's tokens for the stage's 64 channels: lane (pair cp,
      // quarter qr) takes channels 2cp, 2cp + 1 of rows 8 (i / 2) + 2 qr + i % 2, i = 0..15
      // (under the row swizzle a warp's four quarters then read 32 different banks; rows
      // past T are zero), and the quarters meet by two shuffles
      const int cp = (warp & 3) * 8 + (lane & 7), qr = lane >> 3;
      const uint8_t* xt = sgen + s * kStage + (cp & 3) * 4;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int row = 8 * (i >> 1) + 2 * qr + (i & 1);
        const uint32_t w = *reinterpret_cast<const uint32_t*>(xt + swz(row, cp >> 2));
        const float a = bf16lo_to_f32(w), b = bf16hi_to_f32(w);
        if constexpr (P == 2) {
          s0 = __fmaf_rn(a, a, s0);
          s1 = __fmaf_rn(b, b, s1);
        } else {
          s0 = __fadd_rn(s0, fabsf(a));
          s1 = __fadd_rn(s1, fabsf(b));
        }
      }
      s0 = __fadd_rn(s0, __shfl_xor_sync(0xffffffffu, s0, 8));
      s1 = __fadd_rn(s1, __shfl_xor_sync(0xffffffffu, s1, 8));
      s0 = __fadd_rn(s0, __shfl_xor_sync(0xffffffffu, s0, 16));
      s1 = __fadd_rn(s1, __shfl_xor_sync(0xffffffffu, s1, 16));
      const int k = k0 + st * kLrK + 2 * cp;
      if (qr == 0 && k < d)
        *reinterpret_cast<float2*>(spart + static_cast<int64_t>(blockIdx.x) * d + k) = make_float2(s0, s1);
    }
    __syncwarp();  // the warp's reads of the stage are done before its one arrival
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
  }

  // partial[ks][t][rank]: rows groupID and groupID + 8 of the warp's 16 tokens
  if (kSplit && warp >= 4) return;
  if (*abort_flag) return;
  const int g = lane >> 2, tig = lane & 3;
  float* pbase = part + static_cast<int64_t>(blockIdx.y) * T * R;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int t = t0 + warp * 16 + g + 8 * h;
    if (t < T) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(pbase + static_cast<int64_t>(t) * R + n * 8 + tig * 2) =
            make_float2(acc[n][2 * h], acc[n][2 * h + 1]);
    }
  }
}

// U[t][j] = bf16(sum over splits of part[ks][t][j]) for j < r, 0 for r <= j < 64, in the
// first ceil(T / 4) blocks. With P != 0 the blocks after them finish the statistic: block
// c takes channels 32c .. 32c + 31, its warp w sums the token-block rows w, w + 8, ... of
// spart in order, and warp 0 adds the 8 warp sums in order and writes s.
template <int P>
__global__ void __launch_bounds__(256) lowrank_reduce_kernel(const float* __restrict__ part, int T, int r, int ks,
                                                             __nv_bfloat16* __restrict__ U,
                                                             const float* __restrict__ spart, int d,
                                                             float alpha_over_p, float lambda, float* __restrict__ s) {
  grid_dep_wait();
  grid_dep_launch();
  const int nu = (T + 3) >> 2;  // blocks of U (256 outputs each)
  if constexpr (P != 0) {
    if (static_cast<int>(blockIdx.x) >= nu) {
      __shared__ float ws[8][32];
      const int col = (static_cast<int>(blockIdx.x) - nu) * 32 + (threadIdx.x & 31);
      const int w = threadIdx.x >> 5;
      const int ntb = (T + kLrTok - 1) / kLrTok;
      float v = 0.f;
      if (col < d)
        for (int tb = w; tb < ntb; tb += 8) v = __fadd_rn(v, spart[static_cast<int64_t>(tb) * d + col]);
      ws[w][threadIdx.x & 31] = v;
      __syncthreads();
      if (w == 0 && col < d) {
        float tot = ws[0][threadIdx.x];
#pragma unroll
        for (int i = 1; i < 8; ++i) tot = __fadd_rn(tot, ws[i][threadIdx.x]);
        s[col] = finalize_scale(tot, static_cast<float>(T), alpha_over_p, lambda);
      }
      return;
    }
  }
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;  // t * 64 + j
  if (e >= static_cast<int64_t>(T) * 64) return;
  const int t = static_cast<int>(e >> 6), j = static_cast<int>(e & 63);
  float v = 0.f;
  if (j < r)
    for (int sp = 0; sp < ks; ++sp) v = __fadd_rn(v, part[(static_cast<int64_t>(sp) * T + t) * r + j]);
  U[e] = __float2bfloat16_rn(v);
}

// Few tokens (a decode step): one block per (token t, column j) of U, its 256 threads
// striding over d in 8-channel chunks, fp32 sums reduced in a fixed order (warps, then
// the 8 warp sums); U[t][j] = bf16(sum_k X[t][k] A[j][k]) for j < r and 0 for r <= j < 64.
__global__ void __launch_bounds__(256) lowrank_small_kernel(const __nv_bfloat16* __restrict__ X, int d,
                                                            const __nv_bfloat16* __restrict__ A, int r,
                                                            __nv_bfloat16* __restrict__ U) {
  pdl_enter();
  __shared__ float red[8];
  const int t = blockIdx.x >> 6, j = blockIdx.x & 63;
  if (j >= r) {
    if (threadIdx.x == 0) U[blockIdx.x] = __float2bfloat16_rn(0.f);
    return;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(t) * d);
  const uint4* ar = reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * d);
  const int chunks = d >> 3;
  float acc = 0.f;
#pragma unroll 4
  for (int c = threadIdx.x; c < chunks; c += 256) {
    const uint4 xv = __ldg(xr + c), av = __ldg(ar + c);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc = __fmaf_rn(__uint_as_float(xw[q] << 16), __uint_as_float(aw[q] << 16), acc);
      acc = __fmaf_rn(__uint_as_float(xw[q] & 0xFFFF0000u), __uint_as_float(aw[q] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w];
    U[blockIdx.x] = __float2bfloat16_rn(v);
  }
}

}  // namespace

int lowrank_splits(int64_t T, int64_t d, int num_sms) {
  const int64_t tb = (T + kLrTok - 1) / kLrTok;
  const int64_t kst = (d + kLrK - 1) / kLrK;  // stages of K in all
  // at most two blocks per SM, so that the grid is one wave (a partial second wave of a
  // few blocks would double the pass)
  int64_t ks = (2 * static_cast<int64_t>(num_sms)) / tb;
  if (ks > kst) ks = kst;
  if (ks < 1) ks = 1;
  return static_cast<int>(ks);
}

size_t lowrank_partial_bytes(int64_t T, int64_t d, int r, int num_sms) {
  if (r <= 0) return 0;
  return static_cast<size_t>(lowrank_splits(T, d, num_sms)) * static_cast<size_t>(T) * static_cast<size_t>(r) *
         sizeof(float);
}

int lowrank_small_tokens() { return kLrSmallTokens; }

size_t lowrank_stats_bytes(int64_t T, int64_t d) {
  return static_cast<size_t>((T + kLrTok - 1) / kLrTok) * static_cast<size_t>(d) * sizeof(float);
}

namespace {

template <int NT, int P>
cudaError_t launch_partial_nt(dim3 grid, const CUtensorMap& mx, const CUtensorMap& ma, int T, int d, int kc,
                              float* partial, float* spart, const DevErr& err, cudaStream_t stream) {
  constexpr size_t smem = lr_smem_bytes<NT>();
  cudaError_t e =
      cudaFuncSetAttribute(lowrank_partial_kernel<NT, P>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  // all of the SM's unified memory as shared memory, so that two or three blocks fit
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(lowrank_partial_kernel<NT, P>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  return launch_pdl(lowrank_partial_kernel<NT, P>, grid, dim3(lr_threads<NT, P>()), smem, stream, mx, ma, T, d, kc,
                    partial, spart, err);
}

template <int P>
cudaError_t launch_partial(int nt, dim3 grid, const CUtensorMap& mx, const CUtensorMap& ma, int T, int d, int kc,
                           float* partial, float* spart, const DevErr& err, cudaStream_t stream) {
  switch (nt) {
    case 1: return launch_partial_nt<1, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    case 2: return launch_partial_nt<2, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    case 3: return launch_partial_nt<3, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    case 4: return launch_partial_nt<4, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    case 5: return launch_partial_nt<5, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    case 6: return launch_partial_nt<6, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    case 7: return launch_partial_nt<7, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
    default: return launch_partial_nt<8, P>(grid, mx, ma, T, d, kc, partial, spart, err, stream);
  }
}

// The partial kernel and its reduce; P = 0 for U alone, else also the statistic with
// exponent P into s.
template <int P>
cudaError_t launch_tiled(const void* X, int64_t T, int64_t d, const void* A, int r, void* U, float* partial,
                         float* spart, float alpha_over_p, float lambda, float* s, int num_sms, const DevErr& err,
                         cudaStream_t stream) {
  // X [T, d] and A [r, d] as tensor maps with 64-channel boxes (128 bytes, 128-byte swizzle):
  // 64 token rows of X, all r rows of A
  CUtensorMap mx, ma;
  if (!encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, static_cast<uint64_t>(T), static_cast<uint64_t>(d),
                      static_cast<uint64_t>(d), kLrK, kLrTok, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, static_cast<uint64_t>(r), static_cast<uint64_t>(d),
                      static_cast<uint64_t>(d), kLrK, static_cast<uint32_t>(r), CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int ks = lowrank_splits(T, d, num_sms);
  const int64_t kst = (d + kLrK - 1) / kLrK;
  const int kc = static_cast<int>((kst + ks - 1) / ks) * kLrK;
  const int ksr = static_cast<int>((d + kc - 1) / kc);  // splits that hold any K
  const dim3 grid(static_cast<unsigned>((T + kLrTok - 1) / kLrTok), static_cast<unsigned>(ksr));
  const int Ti = static_cast<int>(T), di = static_cast<int>(d);
  cudaError_t e = launch_partial<P>(r / 8, grid, mx, ma, Ti, di, kc, partial, spart, err, stream);
  if (e != cudaSuccess) return e;
  const int64_t nblk = (T + 3) / 4 + (P != 0 ? (d + 31) / 32 : 0);
  return launch_pdl(lowrank_reduce_kernel<P>, dim3(static_cast<unsigned>(nblk)), dim3(256), 0, stream,
                    static_cast<const float*>(partial), Ti, r, ksr, static_cast<__nv_bfloat16*>(U),
                    static_cast<const float*>(spart), di, alpha_over_p, lambda, s);
}

}  // namespace

cudaError_t launch_lowrank_u(const void* X, int64_t T, int64_t d, const void* A, int r, void* U, float* partial,
                             int num_sms, const DevErr& err, cudaStream_t stream) {
  if (T <= kLrSmallTokens) {
    return launch_pdl(lowrank_small_kernel, dim3(static_cast<unsigned>(T * 64)), dim3(256), 0, stream,
                      static_cast<const __nv_bfloat16*>(X), static_cast<int>(d), static_cast<const __nv_bfloat16*>(A),
                      r, static_cast<__nv_bfloat16*>(U));
  }
  return launch_tiled<0>(X, T, d, A, r, U, partial, nullptr, 0.f, 0.f, nullptr, num_sms, err, stream);
}

cudaError_t launch_lowrank_u_stats(const void* X, int64_t T, int64_t d, const void* A, int r, void* U,
                                   float* partial, float* stats_part, float alpha, float lambda, int p, float* s,
                                   int num_sms, const DevErr& err, cudaStream_t stream) {
  if (T <= kLrSmallTokens || (p != 1 && p != 2)) return cudaErrorInvalidValue;
  const float ap = alpha / static_cast<float>(p);
  return p == 2 ? launch_tiled<2>(X, T, d, A, r, U, partial, stats_part, ap, lambda, s, num_sms, err, stream)
                : launch_tiled<1>(X, T, d, A, r, U, partial, stats_part, ap, lambda, s, num_sms, err, stream);
}

}  // namespace ttq
