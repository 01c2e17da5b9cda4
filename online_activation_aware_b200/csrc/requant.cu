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
// The per-element division v / sigma is the hot spot. It is computed as v * RN(1/sigma)
// fused with the 1.5 * 2^23 + z add that rounds it to an integer (half to even), which
// equals rint(fl32(v / sigma)) + z except when the quotient lies within a few ulps of a
// half integer; a unit whose closest quotient falls inside a window of (|z| + N) * 2^-21
// around one (far wider than the 2^-24 relative error of v * RN(1/sigma)) is recomputed
// with the IEEE-rounded division, so every code equals the one the rules above define.
// W is read once with an evict-first L2 policy.
#include "ttq_internal.h"

namespace ttq {

namespace {

// Smallest fp16 >= x (x > 0), kept within the finite positive range [2^-24, 65504].
__device__ __forceinline__ __half fp16_up_sat(float x) {
  if (x > 65504.f) return __ushort_as_half(static_cast<unsigned short>(0x7BFFu));
  __half h = __float2half_ru(x);
  if (__half_as_ushort(h) == 0u) h = __ushort_as_half(static_cast<unsigned short>(0x0001u));
  return h;
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
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// A lane's 64 B of weights (one unit) sit in its warp's ring slot as four 16-byte chunks,
// chunk j of lane l at l * 4 + ((j + (l >> 1)) & 3): a quarter warp reading chunk j then
// touches eight different 16-byte bank groups (conflict-free).
__device__ __forceinline__ int wchunk(int lane, int j) { return lane * 4 + ((j + (lane >> 1)) & 3); }

// v[0..8) = fl32(w * s) for chunk j (8 weights) of the lane's unit; the strip's s in
// shared memory, chunk jj of lane l stored at l * 8 + (jj ^ (l & 7)) (conflict-free).
// Two products per packed f32x2 multiply (each lane of it rounds like __fmul_rn).
__device__ __forceinline__ void scale_chunk(const uint4* slot, const uint4* s_sm, int lane, int j,
                                            float* v) {
  const uint4 wq = slot[wchunk(lane, j)];
  const uint4 sa = s_sm[lane * 8 + ((2 * j) ^ (lane & 7))];
  const uint4 sb = s_sm[lane * 8 + ((2 * j + 1) ^ (lane & 7))];
  const uint32_t w[4] = {wq.x, wq.y, wq.z, wq.w};
  const float sv[8] = {__uint_as_float(sa.x), __uint_as_float(sa.y), __uint_as_float(sa.z),
                       __uint_as_float(sa.w), __uint_as_float(sb.x), __uint_as_float(sb.y),
                       __uint_as_float(sb.z), __uint_as_float(sb.w)};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint64_t p = f2mul(f2(bf16lo_to_f32(w[k]), bf16hi_to_f32(w[k])), f2(sv[2 * k], sv[2 * k + 1]));
    unf2(p, v[2 * k], v[2 * k + 1]);
  }
}

// Packing of a unit's 32 codes, 8 at a time (chunk j = codes 8j .. 8j + 7). A code is the
// low byte of c[k]: either the bits of the float 1.5 * 2^23 + code (whose low byte is the
// code) or the plain integer.
//   q = 4: acc[j] is the finished word (LSB-first nibbles);
//   q = 2: acc[j] holds 16 bits (LSB-first 2-bit fields) in its low half;
//   q = 3: acc[b] collects bit plane b of all 32 codes.
template <int Q>
__device__ __forceinline__ void put_chunk(uint32_t (&acc)[4], int j, const uint32_t (&c)[8]) {
  if (Q == 4) {
    uint32_t p[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) p[k] = c[2 * k] + 16u * c[2 * k + 1];  // low byte: two nibbles
    acc[j] = __byte_perm(__byte_perm(p[0], p[1], 0x5140u), __byte_perm(p[2], p[3], 0x5140u), 0x5410u);
  } else if (Q == 2) {
    const uint32_t lo = (c[0] + 4u * c[1]) + 16u * (c[2] + 4u * c[3]);  // low byte: four fields
    const uint32_t hi = (c[4] + 4u * c[5]) + 16u * (c[6] + 4u * c[7]);
    acc[j] = __byte_perm(lo, hi, 0x0040u);
  } else {
#pragma unroll
    for (int b = 0; b < 3; ++b) {
      uint32_t a = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) a |= ((c[k] >> b) & 1u) << k;
      acc[b] |= a << (8 * j);
    }
  }
}

template <int Q>
__device__ __forceinline__ void store_codes(uint32_t* dst, const uint32_t (&acc)[4]) {
  if (Q == 4) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(acc[0], acc[1], acc[2], acc[3]);
  } else if (Q == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(__byte_perm(acc[0], acc[1], 0x5410u), __byte_perm(acc[2], acc[3], 0x5410u));
  } else {
    dst[0] = acc[0];
    dst[1] = acc[1];
    dst[2] = acc[2];
  }
}

// Group parameters, codes and stores for one unit of 32 scaled weights. Every lane of
// the warp calls this together (the group's lanes exchange min/max by shuffles).
//
// Fast path: t = fl32(v * rcp + (1.5 * 2^23 + z)) with one rounding (packed FMA) holds
// 1.5 * 2^23 + rint(v * rcp + z) whenever that integer is in range, and its low byte is
// the code; fr = fl32((t - 1.5 * 2^23 - z) - v * rcp) is the distance of v * rcp from
// that integer. rcp = RN(1 / sigma) is within 2^-24 relative of 1 / sigma, so v * rcp is
// within |v / sigma| * 2^-24 of the exact quotient: rounding it gives rint(v / sigma)
// except within that distance of a half integer. When z is not clamped and sigma is not
// saturated, every exact quotient lies in [-z - 1/2, N - z + 1/2] up to the rounding of
// the range (sigma is rounded up to fp16), so the code needs no clamp either except at
// a half integer. A unit with some |fr| >= 1/2 - (|z| + N) * 2^-21 (a window far wider
// than those errors), or whose group has a clamped z or a saturated sigma, is recomputed
// with the IEEE-rounded division and the clamp, so every code equals the rule's.
template <int Q, int G>
__device__ __forceinline__ void quantize_unit(const float (&v)[32], const uint4* slot, const uint4* s_sm,
                                              int lane, bool store_ok, uint32_t* codes_dst,
                                              __half* scale_dst, __half* zero_dst) {
  constexpr int LPG = G / 32;  // lanes per group
  constexpr float NQ = static_cast<float>((1 << Q) - 1);
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  // min / max as four short chains (depth 6 instead of 16)
  float m4[4], x4[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float* u = &v[8 * c];
    float mn_ = min3f(u[0], u[1], u[2]);
    float mx_ = max3f(u[0], u[1], u[2]);
    mn_ = min3f(mn_, u[3], u[4]);
    mx_ = max3f(mx_, u[3], u[4]);
    mn_ = min3f(mn_, u[5], u[6]);
    mx_ = max3f(mx_, u[5], u[6]);
    m4[c] = fminf(mn_, u[7]);
    x4[c] = fmaxf(mx_, u[7]);
  }
  float mn = fminf(min3f(m4[0], m4[1], m4[2]), m4[3]);
  float mx = fmaxf(max3f(x4[0], x4[1], x4[2]), x4[3]);
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  float rng = __fsub_rn(mx, mn);
  if (rng == 0.f) rng = (mn != 0.f) ? fabsf(mn) : 1.0f;
  const float sig32 = __fdiv_rn(rng, NQ);
  const __half sig16 = fp16_up_sat(sig32);
  const float sig = __half2float(sig16);
  const float zr = rintf(__fdiv_rn(-mn, sig));
  const float zf = fminf(fmaxf(zr, -2048.f), 2048.f);

  const float rcp = __frcp_rn(sig);
  const float margin = (fabsf(zf) + NQ) * 4.76837158203125e-7f;  // >= max |v / sigma| * 2^-21
  const float mz = __fadd_rn(kMagic, zf);                         // exact
  const uint64_t rcp2 = f2(rcp, rcp);
  const uint64_t nrcp2 = f2(-rcp, -rcp);
  const uint64_t mz2 = f2(mz, mz);
  uint32_t acc[4] = {0u, 0u, 0u, 0u};
  float fmax_ = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t c8[8];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const uint64_t vv = f2(v[8 * j + k], v[8 * j + k + 1]);
      const uint64_t t = f2fma(vv, rcp2, mz2);        // 1.5 * 2^23 + rint(v * rcp + z)
      const uint64_t kk = f2sub(t, mz2);              // rint(v * rcp + z) - z, exact
      const uint64_t fr = f2fma(vv, nrcp2, kk);       // that - v * rcp, one rounding
      float f0, f1, c0, c1;
      unf2(fr, f0, f1);
      unf2(t, c0, c1);
      fmax_ = max3f(fmax_, fabsf(f0), fabsf(f1));
      c8[k] = __float_as_uint(c0);
      c8[k + 1] = __float_as_uint(c1);
    }
    put_chunk<Q>(acc, j, c8);
  }
  if (fmax_ >= 0.5f - margin || fabsf(zf) >= 2048.f || sig32 > 65504.f) {
    // a quotient is near a rounding tie, z was clamped or sigma saturated: the exact rule
    // (v is formed again from the weights still in the ring slot, 8 at a time)
    acc[0] = acc[1] = acc[2] = acc[3] = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v8[8];
      scale_chunk(slot, s_sm, lane, j, v8);
      uint32_t c8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float qe = __fadd_rn(rintf(__fdiv_rn(v8[k], sig)), zf);
        c8[k] = static_cast<uint32_t>(fminf(fmaxf(qe, 0.f), NQ));
      }
      put_chunk<Q>(acc, j, c8);
    }
  }
  if (store_ok) {
    store_codes<Q>(codes_dst, acc);
    if ((lane % LPG) == 0) {
      *scale_dst = sig16;
      *zero_dst = __float2half_rn(zf);
    }
  }
}

constexpr int kRqWarps = 8;    // re-quantization warps per CTA
constexpr int kFoldWarps = 2;  // activation-folding warps per CTA (fused form)
constexpr int kRqStages = 3;   // ring slots per warp (rows in flight: kRqStages - 1 ahead)

// Forms of the kernel: one prompt; one prompt with the fold of its activations; P prompts
// sharing one read of W.
enum RqMode { kRqSingle = 0, kRqFold = 1, kRqBatch = 2 };

__host__ __device__ constexpr size_t rq_smem_bytes(int mode, int prompts) {
  // s of every prompt (and, fused, 1/s) for the strip, then one ring per warp
  return ((mode == kRqFold ? 2 : prompts) * 32 * 8 + (kRqWarps + (mode == kRqFold ? kFoldWarps : 0)) * kRqStages * 32 * 4) *
         sizeof(uint4);
}

__host__ __device__ constexpr int rq_ctas_per_sm(int mode, int q) {
  return mode == kRqFold ? (q == 3 ? 2 : 3) : mode == kRqBatch ? 2 : (q == 3 ? 3 : 4);
}

__device__ __forceinline__ void cp_async_16_hint(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(pol)
               : "memory");
}

// X' = bf16(x * (1/s)) for one lane's 32 activations of a row (4 chunks of 8, read from the
// lane's ring slot), with the strip's reciprocals rs_sm laid out like s_sm.
__device__ __forceinline__ void fold_unit(const uint4* slot, const uint4* rs_sm, int lane, __nv_bfloat16* dst) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 xq = slot[wchunk(lane, j)];
    const uint4 ra = rs_sm[lane * 8 + ((2 * j) ^ (lane & 7))];
    const uint4 rb = rs_sm[lane * 8 + ((2 * j + 1) ^ (lane & 7))];
    const float r[8] = {__uint_as_float(ra.x), __uint_as_float(ra.y), __uint_as_float(ra.z), __uint_as_float(ra.w),
                        __uint_as_float(rb.x), __uint_as_float(rb.y), __uint_as_float(rb.z), __uint_as_float(rb.w)};
    const uint32_t w[4] = {xq.x, xq.y, xq.z, xq.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      o[k] = pack_bf16x2(__fmul_rn(bf16lo_to_f32(w[k]), r[2 * k]), __fmul_rn(bf16hi_to_f32(w[k]), r[2 * k + 1]));
    *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// grid: (column strips of 32 units, row blocks). Every warp streams rows through its own
// ring of kRqStages shared-memory slots: each lane copies its own 64 B of a row (cp.async,
// L2 evict-first: the data is read once) two rows ahead of the one it works on, and reads
// back only what it copied, so no barrier is needed. Warps 0..7 re-quantize rows r0 + w,
// r0 + w + 8, ... of the block's range of W. In the fused form (kRqFold), warps 8..9 at the
// same time fold the block's share of the activation rows over the same 1024 columns,
// X' = bf16(x * RN(1/s)), so the W stream and the X stream share the DRAM pipe instead of
// following one another. In the batched form (kRqBatch) each row of W, once in shared
// memory, is re-quantized against the statistic of each of P prompts in turn (prompt p
// writes codes + p * cstride, scale / zero + p * mstride). Lanes past the end of a row
// work on clamped addresses and store nothing.
template <int Q, int G, int MODE>
__global__ void __launch_bounds__((kRqWarps + (MODE == kRqFold ? kFoldWarps : 0)) * 32, rq_ctas_per_sm(MODE, Q))
    requant_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ s, int d_out, int units_per_row,
                   int rows_per_cta, uint32_t* __restrict__ codes, __half* __restrict__ scale,
                   __half* __restrict__ zero, const __nv_bfloat16* __restrict__ X, __nv_bfloat16* __restrict__ Xf,
                   int T, int x_rows_per_cta, int prompts, int64_t cstride, int64_t mstride) {
  constexpr bool FOLD = MODE == kRqFold;
  const int P = MODE == kRqBatch ? prompts : 1;
  extern __shared__ uint4 rq_smem[];
  uint4* s_sm = rq_smem;                            // [prompt][32 lanes x 8 chunks]
  uint4* rs_sm = rq_smem + 32 * 8;                  // fused: 1/s, same layout
  uint4* ring = rq_smem + (FOLD ? 2 : P) * 32 * 8;  // [warp][stage][32 lanes x 4 chunks]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const bool folder = FOLD && warp >= kRqWarps;
  const int unit = blockIdx.x * 32 + lane;
  const bool col_ok = unit < units_per_row;
  const int ucl = col_ok ? unit : units_per_row - 1;
  const int d = units_per_row * 32;
  // rows this warp streams: W rows r0 + w (step 8), or X rows t0 + (w - 8) (step kFoldWarps)
  int r, r1, step;
  const __nv_bfloat16* src;
  if (folder) {
    const int t0 = blockIdx.y * x_rows_per_cta;
    r = t0 + warp - kRqWarps;
    r1 = min(T, t0 + x_rows_per_cta);
    step = kFoldWarps;
    src = X;
  } else {
    const int w0 = blockIdx.y * rows_per_cta;
    r = w0 + warp;
    r1 = min(d_out, w0 + rows_per_cta);
    step = kRqWarps;
    src = W;
  }
  const __nv_bfloat16* next = src + static_cast<int64_t>(r) * d + static_cast<int64_t>(ucl) * 32;
  const uint32_t ring0 = smem_addr(ring + warp * (kRqStages * 32 * 4));
  int ahead = r;  // next row to copy
  auto issue = [&](int stage) {
    if (ahead < r1) {
      const uint64_t pol = l2_evict_first_policy();
      const uint32_t base = ring0 + static_cast<uint32_t>(stage) * (32 * 4 * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) cp_async_16_hint(base + 16u * wchunk(lane, j), next + 8 * j, pol);
    }
    cp_async_commit();  // one group per row, empty past the end, so the counting stays uniform
    ahead += step;
    next += static_cast<int64_t>(step) * d;
  };
#pragma unroll
  for (int i = 0; i < kRqStages - 1; ++i) issue(i);
  // W and X do not depend on the kernel ahead in the stream; s does. When launched as a
  // programmatic dependent, the first rows are in flight before this wait.
  grid_dep_wait();
  grid_dep_launch();
  if (threadIdx.x < 256) {
    const int l = threadIdx.x >> 3;
    const int jj = threadIdx.x & 7;
    const int u = blockIdx.x * 32 + l;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (u < units_per_row) val = __ldcg(reinterpret_cast<const uint4*>(s + static_cast<int64_t>(u) * 32 + jj * 4));
    s_sm[l * 8 + (jj ^ (l & 7))] = val;
    for (int p = 1; p < P; ++p) {  // batched: the other prompts' statistics
      uint4 vp = make_uint4(0u, 0u, 0u, 0u);
      if (u < units_per_row)
        vp = __ldcg(reinterpret_cast<const uint4*>(s + static_cast<int64_t>(p) * d + static_cast<int64_t>(u) * 32 +
                                                   jj * 4));
      s_sm[p * 256 + l * 8 + (jj ^ (l & 7))] = vp;
    }
    if (FOLD) {
      const uint4 rv = make_uint4(__float_as_uint(__frcp_rn(__uint_as_float(val.x))),
                                  __float_as_uint(__frcp_rn(__uint_as_float(val.y))),
                                  __float_as_uint(__frcp_rn(__uint_as_float(val.z))),
                                  __float_as_uint(__frcp_rn(__uint_as_float(val.w))));
      rs_sm[l * 8 + (jj ^ (l & 7))] = rv;
    }
  }
  __syncthreads();
  const uint4* wring = ring + warp * (kRqStages * 32 * 4);
  if (folder) {
    __nv_bfloat16* dst = Xf + static_cast<int64_t>(r) * d + static_cast<int64_t>(ucl) * 32;
    for (int stage = 0; r < r1; r += step) {
      issue(stage == 0 ? kRqStages - 1 : stage - 1);
      cp_async_wait<kRqStages - 1>();  // this lane's copy of row r has landed
      if (col_ok) fold_unit(wring + stage * (32 * 4), rs_sm, lane, dst);
      dst += static_cast<int64_t>(step) * d;
      stage = stage + 1 == kRqStages ? 0 : stage + 1;
    }
    cp_async_wait<0>();
    return;
  }
  const int gpr = d / G;
  uint32_t* cdst = codes + (static_cast<int64_t>(r) * units_per_row + ucl) * Q;
  const int64_t g0 = static_cast<int64_t>(r) * gpr + (ucl * 32) / G;
  __half* sdst = scale + g0;
  __half* zdst = zero + g0;
  for (int stage = 0; r < r1; r += step) {
    issue(stage == 0 ? kRqStages - 1 : stage - 1);
    cp_async_wait<kRqStages - 1>();  // this lane's copy of row r has landed
    const uint4* slot = wring + stage * (32 * 4);
    if (MODE == kRqBatch) {
#pragma unroll 1
      for (int p = 0; p < P; ++p) {
        const uint4* sp = s_sm + p * 256;
        float v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) scale_chunk(slot, sp, lane, j, &v[8 * j]);
        quantize_unit<Q, G>(v, slot, sp, lane, col_ok, cdst + p * cstride, sdst + p * mstride, zdst + p * mstride);
      }
    } else {
      float v[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) scale_chunk(slot, s_sm, lane, j, &v[8 * j]);
      quantize_unit<Q, G>(v, slot, s_sm, lane, col_ok, cdst, sdst, zdst);
    }
    cdst += static_cast<int64_t>(kRqWarps) * units_per_row * Q;
    sdst += static_cast<int64_t>(kRqWarps) * gpr;
    zdst += static_cast<int64_t>(kRqWarps) * gpr;
    stage = stage + 1 == kRqStages ? 0 : stage + 1;
  }
  cp_async_wait<0>();
}

struct RqArgs {
  const __nv_bfloat16* W;
  const float* s;
  int d_out, units_per_row, rows_per_cta;
  uint32_t* codes;
  __half* scale;
  __half* zero;
  const __nv_bfloat16* X;
  __nv_bfloat16* Xf;
  int T, x_rows_per_cta;
  int prompts;
  int64_t cstride, mstride;
};

template <int Q, int G, int MODE>
cudaError_t launch_qg(dim3 grid, const RqArgs& args, bool pdl, cudaStream_t stream) {
  // set on every launch (it belongs to the current context; for the largest batch)
  cudaError_t e = cudaFuncSetAttribute(requant_kernel<Q, G, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(rq_smem_bytes(MODE, MODE == kRqBatch ? kRequantMaxPrompts : 1)));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3((kRqWarps + (MODE == kRqFold ? kFoldWarps : 0)) * 32);
  cfg.dynamicSmemBytes = rq_smem_bytes(MODE, args.prompts);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, requant_kernel<Q, G, MODE>, args.W, args.s, args.d_out, args.units_per_row,
                            args.rows_per_cta, args.codes, args.scale, args.zero, args.X, args.Xf, args.T,
                            args.x_rows_per_cta, args.prompts, args.cstride, args.mstride);
}

template <int Q, int MODE>
cudaError_t launch_q(int g, RqArgs args, bool pdl, cudaStream_t stream) {
  const int strips = (args.units_per_row + 31) / 32;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // about one wave of resident CTAs (launch bounds), at least 8 rows of W per CTA
  const int per_sm = rq_ctas_per_sm(MODE, Q);
  const int64_t d_out = args.d_out;
  int64_t row_blocks = (per_sm * static_cast<int64_t>(sms)) / strips;
  const int64_t max_blocks = (d_out + 7) / 8;
  if (row_blocks > max_blocks) row_blocks = max_blocks;
  if (row_blocks < 1) row_blocks = 1;
  args.rows_per_cta = static_cast<int>((d_out + row_blocks - 1) / row_blocks);
  row_blocks = (d_out + args.rows_per_cta - 1) / args.rows_per_cta;
  args.x_rows_per_cta = MODE == kRqFold ? static_cast<int>((args.T + row_blocks - 1) / row_blocks) : 0;
  const dim3 grid(strips, static_cast<unsigned>(row_blocks));
  switch (g) {
    case 32: return launch_qg<Q, 32, MODE>(grid, args, pdl, stream);
    case 64: return launch_qg<Q, 64, MODE>(grid, args, pdl, stream);
    default: return launch_qg<Q, 128, MODE>(grid, args, pdl, stream);
  }
}

template <int MODE>
cudaError_t launch_any(int q, int g, const RqArgs& args, bool pdl, cudaStream_t stream) {
  switch (q) {
    case 2: return launch_q<2, MODE>(g, args, pdl, stream);
    case 3: return launch_q<3, MODE>(g, args, pdl, stream);
    default: return launch_q<4, MODE>(g, args, pdl, stream);
  }
}

}  // namespace

cudaError_t launch_requant(const void* W, int64_t d_out, int64_t d, const float* s, int q, int g,
                           uint32_t* codes, void* scale, void* zero, bool pdl, cudaStream_t stream) {
  RqArgs args{static_cast<const __nv_bfloat16*>(W), s, static_cast<int>(d_out), static_cast<int>(d / 32), 0, codes,
              static_cast<__half*>(scale), static_cast<__half*>(zero), nullptr, nullptr, 0, 0, 1, 0, 0};
  return launch_any<kRqSingle>(q, g, args, pdl, stream);
}

cudaError_t launch_requant_batched(const void* W, int64_t d_out, int64_t d, const float* s, int prompts, int q,
                                   int g, uint32_t* codes, void* scale, void* zero, cudaStream_t stream) {
  RqArgs args{static_cast<const __nv_bfloat16*>(W), s, static_cast<int>(d_out), static_cast<int>(d / 32), 0, codes,
              static_cast<__half*>(scale), static_cast<__half*>(zero), nullptr, nullptr, 0, 0, prompts,
              d_out * (d / 32) * q, d_out * (d / g)};
  return launch_any<kRqBatch>(q, g, args, false, stream);
}

cudaError_t launch_fold_requant(const void* X, int64_t T, void* Xf, const void* W, int64_t d_out, int64_t d,
                                const float* s, int q, int g, uint32_t* codes, void* scale, void* zero,
                                cudaStream_t stream) {
  RqArgs args{static_cast<const __nv_bfloat16*>(W), s, static_cast<int>(d_out), static_cast<int>(d / 32), 0, codes,
              static_cast<__half*>(scale), static_cast<__half*>(zero), static_cast<const __nv_bfloat16*>(X),
              static_cast<__nv_bfloat16*>(Xf), static_cast<int>(T), 0, 1, 0, 0};
  return launch_any<kRqFold>(q, g, args, true, stream);
}

}  // namespace ttq
