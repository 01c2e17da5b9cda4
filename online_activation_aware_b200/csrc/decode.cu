// Decode steps with few tokens (b <= 8): the projection as a CUDA-core GEMV that streams
// the prefill's packed codes once (paper-daily.com deep reading of TTQ, section 6:
// quantisation parameters are computed at prefill and reused at decode).
//
// For a weight row i and a unit of 32 consecutive inputs (all in one group g >= 32):
//   sum_k x'_tk (c_ik - z) sigma = sigma * ( sum_k (128 + c_ik) x'_tk - (128 + z) sum_k x'_tk )
// so each weight costs one byte permute (128 + c as a float) and one FMA per token; the
// per-unit sums of x' are formed once per CTA. x' = bf16(x * (1/s)) is formed in the
// prologue (the same rounding as the tensor-core path's fold), kept as fp32 in shared
// memory with each unit's 8 chunks of 4 floats rotated by (unit & 7), so the lanes of a
// warp, which read 8 different units at the same chunk, hit different banks.
// One warp per output row: lanes stride over the row's units with 16-byte code loads
// (512 contiguous bytes per warp step, q = 4), then reduce by shuffles.
#include "ttq_internal.h"

namespace ttq {

namespace {

__device__ __forceinline__ float code_plus_128f(uint32_t x, int b) {
  return __uint_as_float(__byte_perm(x, 0x43000000u, 0x7044u + (static_cast<unsigned>(b) << 8)));
}

// The packed codes of one 32-input unit (Q words) and their expansion to 32 floats
// 128 + c.
template <int Q>
__device__ __forceinline__ uint4 load_unit(const uint32_t* __restrict__ src) {
  if (Q == 4) return __ldg(reinterpret_cast<const uint4*>(src));
  if (Q == 2) return make_uint4(__ldg(src), __ldg(src + 1), 0u, 0u);
  return make_uint4(__ldg(src), __ldg(src + 1), __ldg(src + 2), 0u);
}

template <int Q>
__device__ __forceinline__ void unit_codes(const uint4& v, float (&f)[32]) {
  if (Q == 4) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = w[j] & 0x0F0F0F0Fu, hi = (w[j] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        f[8 * j + 2 * b] = code_plus_128f(lo, b);
        f[8 * j + 2 * b + 1] = code_plus_128f(hi, b);
      }
    }
  } else if (Q == 2) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      f[e] = __uint_as_float(0x43000000u | (((v.x >> (2 * e)) & 3u) << 16));
      f[16 + e] = __uint_as_float(0x43000000u | (((v.y >> (2 * e)) & 3u) << 16));
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      f[e] = __uint_as_float(0x43000000u |
                             ((((v.x >> e) & 1u) | (((v.y >> e) & 1u) << 1) | (((v.z >> e) & 1u) << 2)) << 16));
  }
}

template <int Q, int B>
__global__ void __launch_bounds__(256) decode_gemv_kernel(
    const __nv_bfloat16* __restrict__ X, const float* __restrict__ s, const uint32_t* __restrict__ codes,
    const __half* __restrict__ scale, const __half* __restrict__ zero, int d, int d_out, int log2g,
    const __nv_bfloat16* __restrict__ U, const __nv_bfloat16* __restrict__ Blr, int r,
    __nv_bfloat16* __restrict__ Y, int nb) {
  // nb <= B real token rows; rows nb..B-1 are zero and never written
  extern __shared__ float sm[];
  const int upr = d >> 5;          // units per row
  float* xs = sm;                  // [B][d], unit chunks rotated
  float* xsum = sm + B * d;        // [B][upr]
  // prologue: x' = bf16(x / s) as fp32, rotated layout; 8 inputs per step (16-byte loads)
  for (int c = threadIdx.x; c < (B * d) >> 3; c += blockDim.x) {
    const int t = c / (d >> 3);
    const int k0 = (c - t * (d >> 3)) << 3;
    const uint4 xv = t < nb ? __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(t) * d + k0))
                            : make_uint4(0u, 0u, 0u, 0u);
    const float4 sa = __ldg(reinterpret_cast<const float4*>(s + k0));
    const float4 sb = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
    const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
    const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    float xp[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      xp[2 * j] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lo, __frcp_rn(sv[2 * j]))));
      xp[2 * j + 1] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(hi, __frcp_rn(sv[2 * j + 1]))));
    }
    const int u = k0 >> 5, q0 = (k0 & 31) >> 2;  // unit and first 4-float chunk
    float4* dst = reinterpret_cast<float4*>(xs + t * d + u * 32);
    dst[q0 ^ (u & 7)] = make_float4(xp[0], xp[1], xp[2], xp[3]);
    dst[(q0 + 1) ^ (u & 7)] = make_float4(xp[4], xp[5], xp[6], xp[7]);
  }
  __syncthreads();
  {
    // per-unit sums: one warp per unit, one element per lane, shuffle reduction
    const int ln = threadIdx.x & 31;
    for (int e = threadIdx.x >> 5; e < B * upr; e += blockDim.x >> 5) {
      float a = xs[(e / upr) * d + (e % upr) * 32 + ln];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (ln == 0) xsum[e] = a;
    }
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int gpr = d >> log2g;
  const int64_t wpr = static_cast<int64_t>(upr) * Q;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < d_out; i += warps_total) {
    float part[B];
#pragma unroll
    for (int t = 0; t < B; ++t) part[t] = 0.f;
    const uint32_t* crow = codes + static_cast<int64_t>(i) * wpr;
    constexpr int kBatch = 8;  // units of a row whose loads are in flight together
    for (int u0 = lane; u0 < upr; u0 += 32 * kBatch) {
      uint4 cv[kBatch];
      float sg[kBatch], zp[kBatch];
#pragma unroll
      for (int kq = 0; kq < kBatch; ++kq) {
        const int u = u0 + 32 * kq;
        if (u < upr) {
          cv[kq] = load_unit<Q>(crow + static_cast<int64_t>(u) * Q);
          const int64_t gi = static_cast<int64_t>(i) * gpr + ((u << 5) >> log2g);
          sg[kq] = __half2float(scale[gi]);
          zp[kq] = 128.0f + __half2float(zero[gi]);
        }
      }
#pragma unroll
      for (int kq = 0; kq < kBatch; ++kq) {
        const int u = u0 + 32 * kq;
        if (u < upr) {
          float f[32];
          unit_codes<Q>(cv[kq], f);
#pragma unroll
          for (int t = 0; t < B; ++t) {
            const float4* xu = reinterpret_cast<const float4*>(xs + t * d + u * 32);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 x4 = xu[j ^ (u & 7)];
              a0 = __fmaf_rn(f[4 * j], x4.x, a0);
              a1 = __fmaf_rn(f[4 * j + 1], x4.y, a1);
              a2 = __fmaf_rn(f[4 * j + 2], x4.z, a2);
              a3 = __fmaf_rn(f[4 * j + 3], x4.w, a3);
            }
            const float acc = (a0 + a1) + (a2 + a3);
            part[t] = __fmaf_rn(sg[kq], __fmaf_rn(-zp[kq], xsum[t * upr + u], acc), part[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < B; ++t) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part[t] += __shfl_xor_sync(0xffffffffu, part[t], off);
    }
    if (lane < nb) {
      float y = 0.f;
#pragma unroll
      for (int t = 0; t < B; ++t)
        if (t == lane) y = part[t];
      if (r > 0) {
        for (int q = 0; q < r; ++q)
          y = __fmaf_rn(__bfloat162float(U[static_cast<int64_t>(lane) * 64 + q]),
                        __bfloat162float(Blr[static_cast<int64_t>(i) * r + q]), y);
      }
      Y[static_cast<int64_t>(lane) * d_out + i] = __float2bfloat16_rn(y);
    }
  }
}

template <int Q, int B>
cudaError_t launch_b(const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = (static_cast<size_t>(B) * a.d + static_cast<size_t>(B) * (a.d / 32)) * sizeof(float);
  auto kern = decode_gemv_kernel<Q, B>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  int64_t blocks = (a.d_out + 7) / 8;
  if (blocks > static_cast<int64_t>(sms) * per_sm) blocks = static_cast<int64_t>(sms) * per_sm;
  int lg = 0;
  while ((1 << lg) < a.g) ++lg;
  kern<<<static_cast<unsigned>(blocks), 256, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(a.X), a.s, a.codes, static_cast<const __half*>(a.scale),
      static_cast<const __half*>(a.zero), static_cast<int>(a.d), static_cast<int>(a.d_out), lg,
      static_cast<const __nv_bfloat16*>(a.U), static_cast<const __nv_bfloat16*>(a.Blr), a.r,
      static_cast<__nv_bfloat16*>(a.Y), static_cast<int>(a.b));
  return cudaGetLastError();
}

template <int Q>
cudaError_t launch_q(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.b) {
    case 1: return launch_b<Q, 1>(a, stream);
    case 2: return launch_b<Q, 2>(a, stream);
    case 3: case 4: return launch_b<Q, 4>(a, stream);
    default: return launch_b<Q, 8>(a, stream);
  }
}

}  // namespace

bool decode_gemv_ok(int64_t b, int64_t d) {
  if (b < 1 || b > kGemvMaxTokens) return false;
  const int64_t B = b <= 2 ? b : (b <= 4 ? 4 : 8);  // the kernel instance that serves b
  return (static_cast<size_t>(B) * d + static_cast<size_t>(B) * (d / 32)) * sizeof(float) <= 200 * 1024;
}

cudaError_t launch_decode_gemv(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.q) {
    case 2: return launch_q<2>(a, stream);
    case 3: return launch_q<3>(a, stream);
    default: return launch_q<4>(a, stream);
  }
}

}  // namespace ttq
