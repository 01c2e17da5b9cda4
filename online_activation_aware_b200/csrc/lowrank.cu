// The static low-rank side path of TTQ: U = X A^T, the [T, r] projection that the
// tensor-core GEMM multiplies by B in its extra K block (gist.science French summary,
// section 2B: W_hat = W_q + B A with B, A fixed from the SVD; paper-daily.com deep
// reading, section 2: low-rank compensation of the quantization residual).
//
// A skinny product (r <= 64 outputs per token) bound by the single read of X. Block
// (token block of 64, K split ks) streams its [64 x Kc] slice of X and the matching
// [r x Kc] slice of A through a 3-stage cp.async ring in shared memory (16-byte chunks,
// XOR-swizzled rows so that ldmatrix is conflict-free), and each of its 4 warps multiplies
// 16 tokens by A^T with mma.sync m16n8k16 (bf16 in, fp32 accumulate). The K splits write
// fp32 partial sums; a small dependent kernel adds them in split order (deterministic)
// and stores U in bf16 with its row padded to 64 (columns r..63 zero). For a few tokens (a
// decode step) one block computes each output over all of d instead.
#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kLrTok = 64;      // tokens per block (4 warps x 16)
constexpr int kLrK = 64;        // K per stage
constexpr int kLrStages = 3;
constexpr int kLrThreads = 128;
constexpr int kLrSmallTokens = 8;  // up to here one block per output (no partial sums in memory)

__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

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

// byte offset of 16-byte chunk c (0..7) of row `row` in a [rows x 64] bf16 tile
__device__ __forceinline__ uint32_t swz(int row, int c) { return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4)); }

// grid: (token blocks, K splits); NT = r / 8 output tiles of 8 ranks.
template <int NT>
__global__ void __launch_bounds__(kLrThreads) lowrank_partial_kernel(const __nv_bfloat16* __restrict__ X, int T,
                                                                     int d, const __nv_bfloat16* __restrict__ A,
                                                                     int kc, float* __restrict__ part) {
  pdl_enter();
  constexpr int R = NT * 8;
  constexpr uint32_t kXBytes = kLrTok * kLrK * 2;  // 8 KB
  constexpr uint32_t kABytes = R * kLrK * 2;
  __shared__ __align__(128) uint8_t sm[kLrStages * (kXBytes + kABytes)];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int t0 = blockIdx.x * kLrTok;
  const int k0 = blockIdx.y * kc;
  const int k1 = min(d, k0 + kc);
  const int nst = (k1 - k0 + kLrK - 1) / kLrK;
  const uint32_t sbase = smem_addr(sm);

  auto issue = [&](int st, int slot) {
    if (st < nst) {
      const int kb = k0 + st * kLrK;
      const uint32_t xs = sbase + slot * (kXBytes + kABytes);
      const uint32_t as = xs + kXBytes;
#pragma unroll
      for (int i = 0; i < (kLrTok * 8) / kLrThreads; ++i) {  // X: 64 rows x 8 chunks
        const int e = tid + i * kLrThreads;
        const int row = e >> 3, c = e & 7;
        const int t = min(t0 + row, T - 1);
        const int k = kb + c * 8;
        cp_async_16_zfill(xs + swz(row, c), X + static_cast<int64_t>(t) * d + (k < d ? k : 0), k < d);
      }
      for (int e = tid; e < R * 8; e += kLrThreads) {  // A: R rows x 8 chunks
        const int row = e >> 3, c = e & 7;
        const int k = kb + c * 8;
        cp_async_16_zfill(as + swz(row, c), A + static_cast<int64_t>(row) * d + (k < d ? k : 0), k < d);
      }
    }
    cp_async_commit();
  };

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[n][j] = 0.f;

#pragma unroll
  for (int i = 0; i < kLrStages - 1; ++i) issue(i, i);
  for (int st = 0; st < nst; ++st) {
    cp_async_wait<kLrStages - 2>();
    __syncthreads();  // stage st is in place for every thread; the slot refilled next is free
    issue(st + kLrStages - 1, (st + kLrStages - 1) % kLrStages);
    const int slot = st % kLrStages;
    const uint32_t xs = sbase + slot * (kXBytes + kABytes);
    const uint32_t as = xs + kXBytes;
#pragma unroll
    for (int kk = 0; kk < kLrK / 16; ++kk) {
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
  }
  cp_async_wait<0>();

  // partial[ks][t][rank]: rows groupID and groupID + 8 of the warp's 16 tokens
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

// U[t][j] = bf16(sum over splits of part[ks][t][j]) for j < r, 0 for r <= j < 64.
__global__ void __launch_bounds__(256) lowrank_reduce_kernel(const float* __restrict__ part, int T, int r, int ks,
                                                             __nv_bfloat16* __restrict__ U) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;  // t * 64 + j
  if (e >= static_cast<int64_t>(T) * 64) return;
  const int t = static_cast<int>(e >> 6), j = static_cast<int>(e & 63);
  float v = 0.f;
  if (j < r)
    for (int s = 0; s < ks; ++s) v = __fadd_rn(v, part[(static_cast<int64_t>(s) * T + t) * r + j]);
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
  int64_t ks = (2 * static_cast<int64_t>(num_sms) + tb - 1) / tb;  // about two blocks per SM
  if (ks > kst) ks = kst;
  if (ks < 1) ks = 1;
  return static_cast<int>(ks);
}

size_t lowrank_partial_bytes(int64_t T, int64_t d, int r, int num_sms) {
  if (r <= 0) return 0;
  return static_cast<size_t>(lowrank_splits(T, d, num_sms)) * static_cast<size_t>(T) * static_cast<size_t>(r) *
         sizeof(float);
}

cudaError_t launch_lowrank_u(const void* X, int64_t T, int64_t d, const void* A, int r, void* U, float* partial,
                             int num_sms, cudaStream_t stream) {
  if (T <= kLrSmallTokens) {
    return launch_pdl(lowrank_small_kernel, dim3(static_cast<unsigned>(T * 64)), dim3(256), 0, stream,
                      static_cast<const __nv_bfloat16*>(X), static_cast<int>(d), static_cast<const __nv_bfloat16*>(A),
                      r, static_cast<__nv_bfloat16*>(U));
  }
  const int ks = lowrank_splits(T, d, num_sms);
  const int64_t kst = (d + kLrK - 1) / kLrK;
  const int kc = static_cast<int>((kst + ks - 1) / ks) * kLrK;
  const int ksr = static_cast<int>((d + kc - 1) / kc);  // splits that hold any K
  const dim3 grid(static_cast<unsigned>((T + kLrTok - 1) / kLrTok), static_cast<unsigned>(ksr));
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const auto* Ab = static_cast<const __nv_bfloat16*>(A);
  const int Ti = static_cast<int>(T), di = static_cast<int>(d);
  cudaError_t e;
  const dim3 blk(kLrThreads);
  switch (r / 8) {
    case 1: e = launch_pdl(lowrank_partial_kernel<1>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    case 2: e = launch_pdl(lowrank_partial_kernel<2>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    case 3: e = launch_pdl(lowrank_partial_kernel<3>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    case 4: e = launch_pdl(lowrank_partial_kernel<4>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    case 5: e = launch_pdl(lowrank_partial_kernel<5>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    case 6: e = launch_pdl(lowrank_partial_kernel<6>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    case 7: e = launch_pdl(lowrank_partial_kernel<7>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
    default: e = launch_pdl(lowrank_partial_kernel<8>, grid, blk, 0, stream, Xb, Ti, di, Ab, kc, partial); break;
  }
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((T * 64 + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lowrank_reduce_kernel, static_cast<const float*>(partial), Ti, r, ksr,
                            static_cast<__nv_bfloat16*>(U));
}

}  // namespace ttq
