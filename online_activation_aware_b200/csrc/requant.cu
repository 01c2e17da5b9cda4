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
// Memory-bound: a CTA owns a strip of 1024 columns (32 lanes x 32 weights) of a range
// of rows; every thread keeps the same 32 columns for all of its rows, so the strip's
// s values are staged once in shared memory, and it software-prefetches the next two
// rows' 64 B of bf16 weights (two register buffers) while it quantizes the current one,
// which keeps about 64 KB of loads in flight per SM. A warp streams 2 KB of a row per
// step and writes the row's packed codes as 512 contiguous bytes (q = 4). A group spans
// g/32 adjacent lanes, which exchange min/max by warp shuffles.
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

// v = fl32(w * s) for one unit: its 32 bf16 weights in `wv` (4 x 8), the strip's s in
// shared memory, chunk jj of lane l stored at l * 8 + (jj ^ (l & 7)) (conflict-free).
__device__ __forceinline__ void scale_unit(const uint4 (&wv)[4], const uint4* s_sm, int lane,
                                           float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 sa = s_sm[lane * 8 + ((2 * j) ^ (lane & 7))];
    const uint4 sb = s_sm[lane * 8 + ((2 * j + 1) ^ (lane & 7))];
    v[8 * j + 0] = __fmul_rn(bf16lo_to_f32(wv[j].x), __uint_as_float(sa.x));
    v[8 * j + 1] = __fmul_rn(bf16hi_to_f32(wv[j].x), __uint_as_float(sa.y));
    v[8 * j + 2] = __fmul_rn(bf16lo_to_f32(wv[j].y), __uint_as_float(sa.z));
    v[8 * j + 3] = __fmul_rn(bf16hi_to_f32(wv[j].y), __uint_as_float(sa.w));
    v[8 * j + 4] = __fmul_rn(bf16lo_to_f32(wv[j].z), __uint_as_float(sb.x));
    v[8 * j + 5] = __fmul_rn(bf16hi_to_f32(wv[j].z), __uint_as_float(sb.y));
    v[8 * j + 6] = __fmul_rn(bf16lo_to_f32(wv[j].w), __uint_as_float(sb.z));
    v[8 * j + 7] = __fmul_rn(bf16hi_to_f32(wv[j].w), __uint_as_float(sb.w));
  }
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Packs 32 codes held in the low bytes of `cb` (float bits 1.5 * 2^23 + code: the low
// byte of such a float is the code) into Q words at `dst`.
template <int Q>
__device__ __forceinline__ void store_code_bytes(uint32_t* dst, const uint32_t (&cb)[32]) {
  if (Q == 4) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t p[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) p[k] = cb[8 * j + 2 * k] + 16u * cb[8 * j + 2 * k + 1];  // low byte
      const uint32_t u = __byte_perm(p[0], p[1], 0x5140u);
      const uint32_t v = __byte_perm(p[2], p[3], 0x5140u);
      w[j] = __byte_perm(u, v, 0x5410u);
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (Q == 2) {
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t p[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = 16 * j + 4 * k;
        p[k] = (cb[e] + 4u * cb[e + 1]) + 16u * (cb[e + 2] + 4u * cb[e + 3]);  // low byte
      }
      const uint32_t u = __byte_perm(p[0], p[1], 0x5140u);
      const uint32_t v = __byte_perm(p[2], p[3], 0x5140u);
      w[j] = __byte_perm(u, v, 0x5410u);
    }
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else {  // Q == 3: three bit planes
#pragma unroll
    for (int b = 0; b < 3; ++b) {
      uint32_t a = 0;
#pragma unroll
      for (int k = 0; k < 32; ++k) a |= ((cb[k] >> b) & 1u) << k;
      dst[b] = a;
    }
  }
}

// Group parameters, codes and stores for one unit of 32 scaled weights. Every lane of
// the warp calls this together (the group's lanes exchange min/max by shuffles).
//
// Fast path (no clamp): when z is not clamped, every exact quotient v / sigma lies in
// [min v / sigma, max v / sigma] and rint of that interval is within [-z, N - z] except
// at exact half-integer ties, so the code needs no clamping unless some quotient is
// near a tie; units with a quotient within |q| * 2^-21 of a half integer, or whose
// group's z was clamped, take the exact path with IEEE division and the clamp.
template <int Q, int G>
__device__ __forceinline__ void quantize_unit(const float (&v)[32], int lane, bool store_ok,
                                              uint32_t* codes_dst, __half* scale_dst,
                                              __half* zero_dst) {
  constexpr int LPG = G / 32;  // lanes per group
  constexpr float NQ = static_cast<float>((1 << Q) - 1);
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float mn = v[0], mx = v[0];
#pragma unroll
  for (int k = 1; k < 31; k += 2) {
    mn = min3f(mn, v[k], v[k + 1]);
    mx = max3f(mx, v[k], v[k + 1]);
  }
  mn = fminf(mn, v[31]);
  mx = fmaxf(mx, v[31]);
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  float rng = __fsub_rn(mx, mn);
  if (rng == 0.f) rng = (mn != 0.f) ? fabsf(mn) : 1.0f;
  const __half sig16 = fp16_up_sat(__fdiv_rn(rng, NQ));
  const float sig = __half2float(sig16);
  const float zr = rintf(__fdiv_rn(-mn, sig));
  const float zf = fminf(fmaxf(zr, -2048.f), 2048.f);

  const float rcp = __frcp_rn(sig);
  const float margin = (fabsf(zf) + NQ) * 4.76837158203125e-7f;  // >= max(|lo|, |hi|) * 2^-21
  const uint64_t rcp2 = f2(rcp, rcp);
  const uint64_t magic2 = f2(kMagic, kMagic);
  const uint64_t z2 = f2(zf, zf);
  uint32_t cb[32];
  float fmax_ = 0.f;
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    const uint64_t q = f2mul(f2(v[k], v[k + 1]), rcp2);
    const uint64_t t = f2add(q, magic2);      // rounds q to an integer, half to even
    const uint64_t fr = f2sub(q, f2sub(t, magic2));  // q - rint(q), exact
    const uint64_t tz = f2add(t, z2);         // 1.5 * 2^23 + rint(q) + z, exact
    float f0, f1, c0, c1;
    unf2(fr, f0, f1);
    unf2(tz, c0, c1);
    fmax_ = max3f(fmax_, fabsf(f0), fabsf(f1));
    cb[k] = __float_as_uint(c0);
    cb[k + 1] = __float_as_uint(c1);
  }
  if (fmax_ >= 0.5f - margin || fabsf(zf) >= 2048.f) {
    // a quotient is near a rounding tie, or z was clamped: the exact definition
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float qe = __fadd_rn(rintf(__fdiv_rn(v[k], sig)), zf);
      cb[k] = static_cast<uint32_t>(fminf(fmaxf(qe, 0.f), NQ));
    }
  }
  if (store_ok) {
    store_code_bytes<Q>(codes_dst, cb);
    if ((lane % LPG) == 0) {
      *scale_dst = sig16;
      *zero_dst = __float2half_rn(zf);
    }
  }
}

// grid: (column strips of 32 units, row blocks); block: 8 warps. Warp w handles rows
// r0 + w, r0 + w + 8, ... of the block's range, two rows in flight ahead of the one it
// quantizes. Lanes past the end of a row compute on clamped data and store nothing.
template <int Q, int G>
__global__ void __launch_bounds__(256, 2) requant_kernel(const __nv_bfloat16* __restrict__ W,
                                                         const float* __restrict__ s, int d_out,
                                                         int units_per_row, int rows_per_cta,
                                                         uint32_t* __restrict__ codes,
                                                         __half* __restrict__ scale,
                                                         __half* __restrict__ zero) {
  __shared__ uint4 s_sm[32 * 8];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int unit = blockIdx.x * 32 + lane;
  const bool col_ok = unit < units_per_row;
  const int ucl = col_ok ? unit : units_per_row - 1;
  const int d = units_per_row * 32;
  const int gpr = d / G;
  {
    const int l = threadIdx.x >> 3;
    const int jj = threadIdx.x & 7;
    const int u = blockIdx.x * 32 + l;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (u < units_per_row) val = __ldg(reinterpret_cast<const uint4*>(s + static_cast<int64_t>(u) * 32 + jj * 4));
    s_sm[l * 8 + (jj ^ (l & 7))] = val;
  }
  __syncthreads();

  const int r0 = blockIdx.y * rows_per_cta;
  const int r1 = min(d_out, r0 + rows_per_cta);
  const __nv_bfloat16* wcol = W + static_cast<int64_t>(ucl) * 32;
  uint4 A[4], B[4];
  auto load = [&](uint4(&buf)[4], int row) {
    if (row < r1) {
      const __nv_bfloat16* p = wcol + static_cast<int64_t>(row) * d;
#pragma unroll
      for (int j = 0; j < 4; ++j) buf[j] = ld_stream(p + 8 * j);
    }
  };
  auto finish = [&](const float(&v)[32], int row) {
    const int64_t u = static_cast<int64_t>(row) * units_per_row + ucl;
    const int64_t gi = static_cast<int64_t>(row) * gpr + (ucl * 32) / G;
    quantize_unit<Q, G>(v, lane, col_ok, codes + u * Q, scale + gi, zero + gi);
  };
  int r = r0 + warp;
  load(A, r);
  load(B, r + 8);
  for (; r < r1; r += 16) {
    {
      float v[32];
      scale_unit(A, s_sm, lane, v);
      load(A, r + 16);
      finish(v, r);
    }
    if (r + 8 < r1) {
      float v[32];
      scale_unit(B, s_sm, lane, v);
      load(B, r + 24);
      finish(v, r + 8);
    }
  }
}

template <int Q>
cudaError_t launch_q(int g, const __nv_bfloat16* W, const float* s, int64_t d_out, int units_per_row,
                     uint32_t* codes, __half* scale, __half* zero, cudaStream_t stream) {
  const int strips = (units_per_row + 31) / 32;
  // about one wave of 2 CTAs per SM on a 148-SM part, at least 8 rows per CTA
  int64_t row_blocks = 296 / strips;
  const int64_t max_blocks = (d_out + 7) / 8;
  if (row_blocks > max_blocks) row_blocks = max_blocks;
  if (row_blocks < 1) row_blocks = 1;
  const int rows_per_cta = static_cast<int>((d_out + row_blocks - 1) / row_blocks);
  row_blocks = (d_out + rows_per_cta - 1) / rows_per_cta;
  dim3 grid(strips, static_cast<unsigned>(row_blocks));
  const int dout = static_cast<int>(d_out);
  switch (g) {
    case 32:
      requant_kernel<Q, 32><<<grid, 256, 0, stream>>>(W, s, dout, units_per_row, rows_per_cta, codes, scale, zero);
      break;
    case 64:
      requant_kernel<Q, 64><<<grid, 256, 0, stream>>>(W, s, dout, units_per_row, rows_per_cta, codes, scale, zero);
      break;
    default:
      requant_kernel<Q, 128><<<grid, 256, 0, stream>>>(W, s, dout, units_per_row, rows_per_cta, codes, scale, zero);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_requant(const void* W, int64_t d_out, int64_t d, const float* s, int q, int g,
                           uint32_t* codes, void* scale, void* zero, cudaStream_t stream) {
  const int units_per_row = static_cast<int>(d / 32);
  const auto* Wb = static_cast<const __nv_bfloat16*>(W);
  auto* sc = static_cast<__half*>(scale);
  auto* zr = static_cast<__half*>(zero);
  switch (q) {
    case 2: return launch_q<2>(g, Wb, s, d_out, units_per_row, codes, sc, zr, stream);
    case 3: return launch_q<3>(g, Wb, s, d_out, units_per_row, codes, sc, zr, stream);
    default: return launch_q<4>(g, Wb, s, d_out, units_per_row, codes, sc, zr, stream);
  }
}

}  // namespace ttq
