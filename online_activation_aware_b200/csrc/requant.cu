// Re-quantization of the weight for one prompt: Q[W diag(s)] with group-wise
// round-to-nearest, q bits, group size g along the input channels, per-group min/max
// scale and integer zero point (paper-daily.com deep reading of TTQ, section 2:
// W_hat = Q[W D^(1/2)] D^(-1/2); nubint.ai review, "proposed method": group-wise RTN
// quantize-dequantize). Rules, for each output row and group of g values v = fl32(w*s):
//   sigma = smallest fp16 >= fl32((max v - min v) / (2^q - 1)), within [2^-24, 65504]
//           (a zero range is replaced by |min v|, or by 1 when min v is 0),
//   z     = rint(fl32(-min v / sigma)) clamped to [-2048, 2048],
//   c     = clamp(rint(fl32(v / sigma)) + z, 0, 2^q - 1), halves to even.
//
// Memory-bound: each thread owns 32 consecutive weights of a row (64 B of bf16, 4 x 16-B
// loads) and writes their q*4 bytes of packed codes, so a warp streams 2 KB of W per
// step. A group spans g/32 adjacent lanes, which exchange min/max by warp shuffles.
//
// The per-element division v / sigma is the hot spot. It is computed as v * (1/sigma)
// and rounded with the 1.5 * 2^23 add (round half to even on the integer), which equals
// rint(fl32(v / sigma)) except when the quotient lies within a few ulps of a half
// integer; a unit whose closest quotient falls inside that window (|q| * 2^-21, far
// wider than the 2^-22.9 relative error of v * RN(1/sigma)) is recomputed with the
// IEEE-rounded division, so every code equals the one the rules above define.
#include "ttq_internal.h"

namespace ttq {

namespace {

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Smallest fp16 >= x (x > 0), kept within the finite positive range [2^-24, 65504].
__device__ __forceinline__ __half fp16_up_sat(float x) {
  if (x > 65504.f) return __ushort_as_half(static_cast<unsigned short>(0x7BFFu));
  __half h = __float2half_ru(x);
  if (__half_as_ushort(h) == 0u) h = __ushort_as_half(static_cast<unsigned short>(0x0001u));
  return h;
}

template <int Q>
__device__ __forceinline__ void store_codes(uint32_t* dst, const int (&c)[32]) {
  if (Q == 4) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t a = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) a |= static_cast<uint32_t>(c[8 * j + k]) << (4 * k);
      w[j] = a;
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (Q == 2) {
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t a = 0;
#pragma unroll
      for (int k = 0; k < 16; ++k) a |= static_cast<uint32_t>(c[16 * j + k]) << (2 * k);
      w[j] = a;
    }
    dst[0] = w[0];
    dst[1] = w[1];
  } else {  // Q == 3: three bit planes
#pragma unroll
    for (int b = 0; b < 3; ++b) {
      uint32_t a = 0;
#pragma unroll
      for (int k = 0; k < 32; ++k) a |= ((static_cast<uint32_t>(c[k]) >> b) & 1u) << k;
      dst[b] = a;
    }
  }
}

// One thread per unit of 32 weights; units are numbered row-major, so a row's units are
// contiguous and a group of g weights is g/32 consecutive units (and lanes).
template <int Q, int G>
__global__ void __launch_bounds__(256) requant_kernel(const __nv_bfloat16* __restrict__ W,
                                                      const float* __restrict__ s, int64_t nunits,
                                                      int units_per_row,
                                                      uint32_t* __restrict__ codes,
                                                      __half* __restrict__ scale,
                                                      __half* __restrict__ zero) {
  constexpr int LPG = G / 32;  // lanes per group
  constexpr float NQ = static_cast<float>((1 << Q) - 1);
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const int lane = threadIdx.x & 31;
  const int64_t warp_base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) & ~int64_t(31);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t wb = warp_base; wb < nunits; wb += stride) {
    const int64_t u = wb + lane;
    const bool valid = u < nunits;   // same for every lane of a group
    const int64_t uu = valid ? u : (nunits - 1);
    const int64_t row = uu / units_per_row;
    const int kc = static_cast<int>(uu - row * units_per_row) * 32;
    const int d = units_per_row * 32;

    // v = fl32(w * s) for the unit's 32 weights
    float v[32];
    const __nv_bfloat16* wp = W + row * d + kc;
    const float* sp = s + kc;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 wv = ld_stream(wp + 8 * j);
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(sp + 8 * j));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(sp + 8 * j + 4));
      v[8 * j + 0] = __fmul_rn(bf16lo_to_f32(wv.x), s0.x);
      v[8 * j + 1] = __fmul_rn(bf16hi_to_f32(wv.x), s0.y);
      v[8 * j + 2] = __fmul_rn(bf16lo_to_f32(wv.y), s0.z);
      v[8 * j + 3] = __fmul_rn(bf16hi_to_f32(wv.y), s0.w);
      v[8 * j + 4] = __fmul_rn(bf16lo_to_f32(wv.z), s1.x);
      v[8 * j + 5] = __fmul_rn(bf16hi_to_f32(wv.z), s1.y);
      v[8 * j + 6] = __fmul_rn(bf16lo_to_f32(wv.w), s1.z);
      v[8 * j + 7] = __fmul_rn(bf16hi_to_f32(wv.w), s1.w);
    }
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int k = 1; k < 32; ++k) {
      mn = fminf(mn, v[k]);
      mx = fmaxf(mx, v[k]);
    }
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }

    // group scale and zero point
    float rng = __fsub_rn(mx, mn);
    if (rng == 0.f) rng = (mn != 0.f) ? fabsf(mn) : 1.0f;
    const __half sig16 = fp16_up_sat(__fdiv_rn(rng, NQ));
    const float sig = __half2float(sig16);
    float zf = rintf(__fdiv_rn(-mn, sig));
    zf = fminf(fmaxf(zf, -2048.f), 2048.f);
    const int zi = static_cast<int>(zf);

    // fast path: q = v * RN(1/sigma), clamped to [-z, N - z], rounded half to even
    const float rcp = __frcp_rn(sig);
    const float lo = -zf;
    const float hi = __fsub_rn(NQ, zf);
    const float margin = fmaxf(fabsf(lo), fabsf(hi)) * 4.76837158203125e-7f;  // * 2^-21
    int c[32];
    float slack = 1.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float qv = fminf(fmaxf(__fmul_rn(v[k], rcp), lo), hi);
      const float t = __fadd_rn(qv, kMagic);
      const float n = __fsub_rn(t, kMagic);
      slack = fminf(slack, __fsub_rn(0.5f, fabsf(__fsub_rn(qv, n))));
      c[k] = (__float_as_int(t) - 0x4B400000) + zi;
    }
    if (slack <= margin) {
      // a quotient is near a rounding tie: recompute the unit with IEEE division
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float qe = __fadd_rn(rintf(__fdiv_rn(v[k], sig)), zf);
        c[k] = static_cast<int>(fminf(fmaxf(qe, 0.f), NQ));
      }
    }
    if (valid) {
      store_codes<Q>(codes + uu * Q, c);
      if ((lane % LPG) == 0) {
        const int64_t gi = row * (d / G) + kc / G;
        scale[gi] = sig16;
        zero[gi] = __float2half_rn(zf);
      }
    }
  }
}

template <int Q>
cudaError_t launch_q(int g, const __nv_bfloat16* W, const float* s, int64_t nunits,
                     int units_per_row, uint32_t* codes, __half* scale, __half* zero,
                     cudaStream_t stream) {
  const int64_t blocks64 = (nunits + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(blocks64 > 148 * 64 ? 148 * 64 : blocks64);
  switch (g) {
    case 32:
      requant_kernel<Q, 32><<<blocks, 256, 0, stream>>>(W, s, nunits, units_per_row, codes, scale, zero);
      break;
    case 64:
      requant_kernel<Q, 64><<<blocks, 256, 0, stream>>>(W, s, nunits, units_per_row, codes, scale, zero);
      break;
    default:
      requant_kernel<Q, 128><<<blocks, 256, 0, stream>>>(W, s, nunits, units_per_row, codes, scale, zero);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_requant(const void* W, int64_t d_out, int64_t d, const float* s, int q, int g,
                           uint32_t* codes, void* scale, void* zero, cudaStream_t stream) {
  const int units_per_row = static_cast<int>(d / 32);
  const int64_t nunits = d_out * units_per_row;
  const auto* Wb = static_cast<const __nv_bfloat16*>(W);
  auto* sc = static_cast<__half*>(scale);
  auto* zr = static_cast<__half*>(zero);
  switch (q) {
    case 2: return launch_q<2>(g, Wb, s, nunits, units_per_row, codes, sc, zr, stream);
    case 3: return launch_q<3>(g, Wb, s, nunits, units_per_row, codes, sc, zr, stream);
    default: return launch_q<4>(g, Wb, s, nunits, units_per_row, codes, sc, zr, stream);
  }
}

}  // namespace ttq
