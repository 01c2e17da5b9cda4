// Kernels of the decoder layer around the TTQ linears (Qwen3-shaped stack: the shapes of
// Table 15 in the thelatestinai.com listing of "TTQ: Activation-Aware Test-Time
// Quantization ..."): RMSNorm with the residual add, per-head q/k RMSNorm with the rotary
// embedding and the key/value cache write, and the SwiGLU gate. All are HBM-bound
// elementwise or row-reduction passes: 16-byte (or per-lane 8-byte) coalesced loads and
// stores, fp32 arithmetic, one bf16 rounding per stored value.
//
//   rmsnorm_kernel      one block per row: r <- bf16(r + y) (optional), out = bf16(r w / rms)
//   rope_table_kernel   cos and sin of pos * base^(-2i/D) in fp64, stored as fp32 pairs
//   qk_norm_rope_kernel one warp per (token, head) of the stacked q|k|v projection
//   silu_mul_kernel     out = bf16(silu(gate) * up), grid-stride over 8-channel chunks
//   decode_attn_*       one new token's grouped-query attention over the cache, split over
//                       positions and merged (flash-decoding form), fp32 softmax
#include <algorithm>
#include <cmath>

#include "ttq_internal.h"

namespace ttq {
namespace {

constexpr int kNormThreads = 256;

// Launch as a programmatic dependent of the previous kernel in the stream (256 threads).
template <typename K, typename... Args>
cudaError_t launch_dependent(K kernel, dim3 grid, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float f[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = bf16lo_to_f32(w[j]);
    f[2 * j + 1] = bf16hi_to_f32(w[j]);
  }
}

__device__ __forceinline__ uint4 pack8(const float f[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// r_j <- bf16(r_j + y_j) when `residual` is given (the row of r is replaced), then
// out_j = bf16(h_j * w_j / sqrt(mean_j h_j^2 + eps)) with h the (updated) row.
// CPT = 8-channel chunks per thread (n <= 8 * 256 * CPT).
template <int CPT>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const __nv_bfloat16* __restrict__ y,
                                                              __nv_bfloat16* __restrict__ residual,
                                                              const __nv_bfloat16* __restrict__ w,
                                                              __nv_bfloat16* __restrict__ out, int n, float eps) {
  pdl_enter();
  __shared__ float red[kNormThreads / 32];
  const int64_t row = blockIdx.x;
  const int nchunks = n >> 3;
  const uint4* yr = reinterpret_cast<const uint4*>(y + row * n);
  uint4* rr = residual ? reinterpret_cast<uint4*>(residual + row * n) : nullptr;
  float h[CPT][8];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int k = threadIdx.x + c * kNormThreads;
    if (k < nchunks) {
      unpack8(__ldcs(yr + k), h[c]);
      if (rr) {
        float r[8];
        unpack8(rr[k], r);
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __fadd_rn(r[e], h[c][e]);
        const uint4 hv = pack8(r);
        rr[k] = hv;
        unpack8(hv, h[c]);  // the stored (rounded) sum is what the norm reads
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = __fmaf_rn(h[c][e], h[c][e], ss);
    }
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kNormThreads / 32; ++i) tot += red[i];
  const float inv = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(tot, static_cast<float>(n)), eps)));
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* orow = reinterpret_cast<uint4*>(out + row * n);
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int k = threadIdx.x + c * kNormThreads;
    if (k < nchunks) {
      float wf[8], o[8];
      unpack8(__ldg(wr + k), wf);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__fmul_rn(h[c][e], inv), wf[e]);
      orow[k] = pack8(o);
    }
  }
}

// table[pos][i] = (cos, sin)(pos * base^(-2i/D)), i < D/2; fp64 arguments and functions,
// rounded to fp32 once.
__global__ void rope_table_kernel(int64_t positions, int half, double base, float2* __restrict__ table) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= positions * half) return;
  const int64_t pos = idx / half;
  const int i = static_cast<int>(idx - pos * half);
  const double inv_freq = pow(base, -static_cast<double>(2 * i) / static_cast<double>(2 * half));
  double sn, cs;
  sincos(static_cast<double>(pos) * inv_freq, &sn, &cs);
  table[idx] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
}

// One warp per (token t, head slot hs) of the stacked projection row
// [q heads | k heads | v heads], each head D = 32 E channels; lane l holds channels
// [E l, E l + E), so lane l ^ 16 holds the rotary partners (+-D/2).
//   q heads: per-head RMSNorm (weight wq), rotation at position pos0 + t, in place;
//   k heads: the same with wk, written to k_cache[pos0 + t][head];
//   v heads: copied to v_cache[pos0 + t][head].
template <int E>
struct LaneVec;
template <>
struct LaneVec<2> { using T = uint32_t; };
template <>
struct LaneVec<4> { using T = uint2; };
template <>
struct LaneVec<8> { using T = uint4; };

template <int E>
__device__ __forceinline__ void lane_unpack(const typename LaneVec<E>::T& v, float f[E]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
  for (int j = 0; j < E / 2; ++j) {
    f[2 * j] = bf16lo_to_f32(w[j]);
    f[2 * j + 1] = bf16hi_to_f32(w[j]);
  }
}

template <int E>
__device__ __forceinline__ typename LaneVec<E>::T lane_pack(const float f[E]) {
  typename LaneVec<E>::T v;
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int j = 0; j < E / 2; ++j) w[j] = pack_bf16x2(f[2 * j], f[2 * j + 1]);
  return v;
}

template <int E>
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(__nv_bfloat16* __restrict__ qkv, int64_t T, int heads,
                                                          int kv_heads, const __nv_bfloat16* __restrict__ wq,
                                                          const __nv_bfloat16* __restrict__ wk, float eps,
                                                          const float2* __restrict__ table, int64_t pos0,
                                                          const int64_t* __restrict__ pos_dev, int64_t limit,
                                                          __nv_bfloat16* __restrict__ k_cache,
                                                          __nv_bfloat16* __restrict__ v_cache,
                                                          unsigned* __restrict__ err) {
  pdl_enter();
  using V = typename LaneVec<E>::T;
  constexpr int D = 32 * E;
  const int lane = threadIdx.x & 31;
  const int slots = heads + 2 * kv_heads;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (item >= T * slots) return;
  if (pos_dev) {
    // the position lives on the device (a captured decode step): check it here
    pos0 = *pos_dev;
    if (pos0 < 0 || pos0 + T > limit) {
      if (item == 0 && lane == 0) atomicOr(err, kErrRange);
      return;
    }
  }
  const int64_t t = item / slots;
  const int hs = static_cast<int>(item - t * slots);
  const int64_t pos = pos0 + t;
  __nv_bfloat16* src = qkv + t * static_cast<int64_t>(slots) * D + static_cast<int64_t>(hs) * D + lane * E;
  const V raw = *reinterpret_cast<const V*>(src);
  if (hs >= heads + kv_heads) {  // v head: straight copy into the cache
    const int64_t kvh = hs - heads - kv_heads;
    *reinterpret_cast<V*>(v_cache + (pos * kv_heads + kvh) * D + lane * E) = raw;
    return;
  }
  float x[E];
  lane_unpack<E>(raw, x);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = __fmaf_rn(x[e], x[e], ss);
  ss = warp_sum(ss);
  const float inv = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(ss, static_cast<float>(D)), eps)));
  const bool is_q = hs < heads;
  const V wraw = *reinterpret_cast<const V*>((is_q ? wq : wk) + lane * E);
  float wf[E];
  lane_unpack<E>(wraw, wf);
  float y[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) y[e] = __fmul_rn(__fmul_rn(x[e], inv), wf[e]);
  const bool first_half = lane < 16;
  const float2* trow = table + pos * (D / 2) + (lane & 15) * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float partner = __shfl_xor_sync(0xffffffffu, y[e], 16);
    const float2 cs = trow[e];
    // first half a: a cos - b sin; second half b: b cos + a sin (partner = the other one)
    o[e] = first_half ? __fsub_rn(__fmul_rn(y[e], cs.x), __fmul_rn(partner, cs.y))
                      : __fadd_rn(__fmul_rn(y[e], cs.x), __fmul_rn(partner, cs.y));
  }
  const V packed = lane_pack<E>(o);
  if (is_q) {
    *reinterpret_cast<V*>(src) = packed;
  } else {
    const int64_t kh = hs - heads;
    *reinterpret_cast<V*>(k_cache + (pos * kv_heads + kh) * D + lane * E) = packed;
  }
}

// out[t, c] = bf16(silu(gu[t, c]) * gu[t, I + c]), silu(u) = u / (1 + e^-u).
__global__ void __launch_bounds__(256) silu_mul_kernel(const __nv_bfloat16* __restrict__ gu, int64_t rows,
                                                      int64_t inter, __nv_bfloat16* __restrict__ out) {
  pdl_enter();
  const int64_t per_row = inter >> 3;
  const int64_t total = rows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_row;
    const int64_t c = i - t * per_row;
    const uint4* row = reinterpret_cast<const uint4*>(gu + t * 2 * inter);
    float g[8], u[8], o[8];
    unpack8(__ldcs(row + c), g);
    unpack8(__ldcs(row + per_row + c), u);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__fdiv_rn(g[e], __fadd_rn(1.f, expf(-g[e]))), u[e]);
    reinterpret_cast<uint4*>(out + t * inter)[c] = pack8(o);
  }
}


// ---------------------------------------------------------------- decode attention
//
// One new token's attention over the key/value cache (split over positions, then
// combined). Block (kv head kh, split sp) of 256 threads takes positions
// [sp * per, (sp + 1) * per) of the L valid ones, per = ceil(L / splits), in chunks of 256:
//   scores   thread i: s_g = q_g . k_p for position p = chunk start + i and the G query heads
//            h = kh G + g that read kv head kh (q pre-scaled by 1/sqrt(D), broadcast from
//            shared memory; k read as 16-byte chunks of its row);
//   softmax  per head the chunk's maximum and sum (one warp per head, fixed order), the
//            running maximum m, the rescale e^(m_old - m), weights e^(s - m) in place;
//   values   lane l holds channels [E l, E l + E) (coalesced v rows), warp w the positions
//            i = w (mod 8) of the chunk: acc_g += w_g,p v_p.
// The 8 warps' accumulators are added in a fixed order and written with (m, l) to `part`
// [kv_heads][splits][G][D + 2]; decode_attn_combine_kernel merges the splits per query head.
constexpr int kDecThreads = 256;
constexpr int kDecChunk = 256;

template <int E, int G>
__global__ void __launch_bounds__(kDecThreads) decode_attn_partial_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_cache,
    const __nv_bfloat16* __restrict__ v_cache, int kv_heads, int64_t cache_len, int64_t length,
    const int64_t* __restrict__ pos_dev, int splits, float scale, float* __restrict__ part,
    unsigned* __restrict__ err) {
  pdl_enter();
  using V = typename LaneVec<E>::T;
  constexpr int D = 32 * E;
  constexpr int kWarps = kDecThreads / 32;
  __shared__ __align__(16) float qs[G][D];
  __shared__ float sc[G][kDecChunk];
  __shared__ float sm_acc[kWarps][G][D];
  __shared__ float m_sh[G], l_sh[G], c_sh[G];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int kh = blockIdx.x;
  const int sp = blockIdx.y;
  int64_t L = pos_dev ? *pos_dev + 1 : length;
  if (L < 1 || L > cache_len) {
    if (kh == 0 && sp == 0 && tid == 0) atomicOr(err, kErrRange);
    L = 0;
  }
  const int64_t per = (L + splits - 1) / splits;
  const int64_t p0 = static_cast<int64_t>(sp) * per;
  const int64_t p1 = min(L, p0 + per);
  for (int i = tid; i < G * D; i += kDecThreads)
    qs[i / D][i % D] = __fmul_rn(__bfloat162float(q[static_cast<int64_t>(kh * G) * D + i]), scale);
  if (tid < G) {
    m_sh[tid] = -INFINITY;
    l_sh[tid] = 0.f;
  }
  float acc[G][E];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < E; ++e) acc[g][e] = 0.f;
  const int64_t row = static_cast<int64_t>(kv_heads) * D;
  __syncthreads();
  for (int64_t c0 = p0; c0 < p1; c0 += kDecChunk) {
    const int n = static_cast<int>(min(static_cast<int64_t>(kDecChunk), p1 - c0));
    // scores of position c0 + tid
    if (tid < n) {
      const uint4* kr = reinterpret_cast<const uint4*>(k_cache + (c0 + tid) * row + kh * D);
      float s[G];
#pragma unroll
      for (int g = 0; g < G; ++g) s[g] = 0.f;
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        float kf[8];
        unpack8(__ldg(kr + c), kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 qa = *reinterpret_cast<const float4*>(&qs[g][8 * c]);
          const float4 qb = *reinterpret_cast<const float4*>(&qs[g][8 * c + 4]);
          s[g] = __fmaf_rn(qa.x, kf[0], s[g]);
          s[g] = __fmaf_rn(qa.y, kf[1], s[g]);
          s[g] = __fmaf_rn(qa.z, kf[2], s[g]);
          s[g] = __fmaf_rn(qa.w, kf[3], s[g]);
          s[g] = __fmaf_rn(qb.x, kf[4], s[g]);
          s[g] = __fmaf_rn(qb.y, kf[5], s[g]);
          s[g] = __fmaf_rn(qb.z, kf[6], s[g]);
          s[g] = __fmaf_rn(qb.w, kf[7], s[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) sc[g][tid] = s[g];
    }
    __syncthreads();
    // per head (warp g): the chunk's maximum, the new running maximum, weights in place
    if (warp < G) {
      const int g = warp;
      float mx = -INFINITY;
      for (int i = lane; i < n; i += 32) mx = fmaxf(mx, sc[g][i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_sh[g];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int i = lane; i < n; i += 32) {
        const float w = expf(sc[g][i] - m_new);
        sc[g][i] = w;
        sum += w;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        const float c = expf(m_old - m_new);  // m_old = -inf on the first chunk: c = 0
        c_sh[g] = c;
        l_sh[g] = __fmaf_rn(l_sh[g], c, sum);
        m_sh[g] = m_new;
      }
    }
    __syncthreads();
    // values: lane's channels, warp's positions
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float c = c_sh[g];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[g][e] = __fmul_rn(acc[g][e], c);
    }
    const __nv_bfloat16* vb = v_cache + kh * D + lane * E;
#pragma unroll 4
    for (int i = warp; i < n; i += kWarps) {
      float vf[E];
      lane_unpack<E>(*reinterpret_cast<const V*>(vb + (c0 + i) * row), vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float w = sc[g][i];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] = __fmaf_rn(w, vf[e], acc[g][e]);
      }
    }
    __syncthreads();  // sc is rewritten by the next chunk
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < E; ++e) sm_acc[warp][g][lane * E + e] = acc[g][e];
  __syncthreads();
  float* out = part + (static_cast<int64_t>(kh) * splits + sp) * G * (D + 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, j = i % D;
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) a += sm_acc[w][g][j];
    out[g * (D + 2) + j] = a;
    if (j == 0) {
      out[g * (D + 2) + D] = m_sh[g];     // -inf and 0 when the split holds no position
      out[g * (D + 2) + D + 1] = l_sh[g];
    }
  }
}

// One block per query head h = kh G + g: merges the splits' (acc, m, l) and writes
// bf16(acc / l) to out[h * D ..]. The splits' weights e^(m_s - M) are formed once in
// shared memory; every sum runs in a fixed order.
constexpr int kDecMaxSplits = 256;
constexpr int kDecMaxBlocks = 256;

__global__ void __launch_bounds__(256) decode_attn_combine_kernel(const float* __restrict__ part, int G, int D,
                                                                 int splits, __nv_bfloat16* __restrict__ out) {
  __shared__ float wsm[kDecMaxSplits];
  __shared__ float red[8];
  __shared__ float Msh, Lsh;
  grid_dep_wait();
  grid_dep_launch();
  const int h = blockIdx.x;
  const int kh = h / G;
  const int g = h - kh * G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* base = part + static_cast<int64_t>(kh) * splits * G * (D + 2) + static_cast<int64_t>(g) * (D + 2);
  const int64_t stride = static_cast<int64_t>(G) * (D + 2);
  float mx = -INFINITY;
  for (int sp = threadIdx.x; sp < splits; sp += blockDim.x) mx = fmaxf(mx, base[sp * stride + D]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = red[0];
    for (int w = 1; w < 8; ++w) M = fmaxf(M, red[w]);
    Msh = M;
  }
  __syncthreads();
  const float M = Msh;
  float ls = 0.f;
  for (int sp = threadIdx.x; sp < splits; sp += blockDim.x) {
    const float f = M == -INFINITY ? 0.f : expf(base[sp * stride + D] - M);  // empty split: m = -inf, f = 0
    wsm[sp] = f;
    ls = __fmaf_rn(base[sp * stride + D + 1], f, ls);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
  __syncthreads();  // red[] is reused
  if (lane == 0) red[warp] = ls;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    Lsh = t;
  }
  __syncthreads();
  const float Ls = Lsh;
  // thread (half, j): half of the splits for channel j; the two halves added in order
  __shared__ float half_sum[256];
  const int halves = blockDim.x / D;  // 2 for D = 128, 4 for D = 64
  const int j = threadIdx.x % D, hf = threadIdx.x / D;
  const int per = (splits + halves - 1) / halves;
  const int s0 = hf * per, s1 = min(splits, s0 + per);
  float a = 0.f;
#pragma unroll 8
  for (int sp = s0; sp < s1; ++sp) a = __fmaf_rn(base[sp * stride + j], wsm[sp], a);
  half_sum[threadIdx.x] = a;
  __syncthreads();
  if (hf == 0) {
    float t = half_sum[j];
    for (int q = 1; q < halves; ++q) t += half_sum[q * D + j];
    out[static_cast<int64_t>(h) * D + j] = __float2bfloat16_rn(Ls > 0.f ? __fdiv_rn(t, Ls) : 0.f);
  }
}

__global__ void position_advance_kernel(int64_t* pos, int64_t n) {
  pdl_enter();
  *pos += n;
}

}  // namespace

int decode_attn_splits(int64_t cache_len, int kv_heads) {
  // at least 64 positions a block, at most 256 blocks (one wave at two blocks an SM)
  const int64_t by_len = (cache_len + 63) / 64;
  const int64_t cap = std::max<int64_t>(1, kDecMaxBlocks / kv_heads);
  return static_cast<int>(std::max<int64_t>(1, std::min(by_len, cap)));
}

size_t decode_attn_partial_bytes(int heads, int head_dim, int splits) {
  return static_cast<size_t>(heads) * splits * (head_dim + 2) * sizeof(float);
}

template <int E, int G>
static cudaError_t decode_attn_partial(dim3 grid, cudaStream_t stream, const __nv_bfloat16* q,
                                       const __nv_bfloat16* kc, const __nv_bfloat16* vc, int kv_heads,
                                       int64_t cache_len, int64_t length, const int64_t* pos_dev, int splits,
                                       float scale, float* part, unsigned* err) {
  return launch_pdl(decode_attn_partial_kernel<E, G>, grid, dim3(kDecThreads), 0, stream, q, kc, vc, kv_heads,
                    cache_len, length, pos_dev, splits, scale, part, err);
}

cudaError_t launch_decode_attention(const void* q, int heads, int kv_heads, int head_dim, const void* k_cache,
                                    const void* v_cache, int64_t cache_len, int64_t length, const int64_t* pos_dev,
                                    void* out, float* part, int splits, unsigned* err, cudaStream_t stream) {
  const int G = heads / kv_heads;
  const dim3 grid(static_cast<unsigned>(kv_heads), static_cast<unsigned>(splits));
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(head_dim)));
  auto qq = static_cast<const __nv_bfloat16*>(q);
  auto kc = static_cast<const __nv_bfloat16*>(k_cache);
  auto vc = static_cast<const __nv_bfloat16*>(v_cache);
  cudaError_t e = cudaErrorInvalidValue;
#define TTQ_DEC_ATTN(EE, GG)                                                                                         \
  if (head_dim == 32 * EE && G == GG)                                                                                \
    e = decode_attn_partial<EE, GG>(grid, stream, qq, kc, vc, kv_heads, cache_len, length, pos_dev, splits, scale, \
                                    part, err);
  TTQ_DEC_ATTN(2, 1) TTQ_DEC_ATTN(2, 2) TTQ_DEC_ATTN(2, 4) TTQ_DEC_ATTN(2, 8)
  TTQ_DEC_ATTN(4, 1) TTQ_DEC_ATTN(4, 2) TTQ_DEC_ATTN(4, 4) TTQ_DEC_ATTN(4, 8)
#undef TTQ_DEC_ATTN
  if (e != cudaSuccess) return e;
  return launch_dependent(decode_attn_combine_kernel, dim3(heads), stream, static_cast<const float*>(part), G,
                          head_dim, splits, static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_position_advance(int64_t* pos, int64_t n, cudaStream_t stream) {
  return launch_pdl(position_advance_kernel, dim3(1), dim3(1), 0, stream, pos, n);
}

namespace {
}  // namespace

cudaError_t launch_rmsnorm(const void* y, void* residual, const void* w, int64_t rows, int n, float eps, void* out,
                           cudaStream_t stream) {
  const int cpt = (n / 8 + kNormThreads - 1) / kNormThreads;
  auto yy = static_cast<const __nv_bfloat16*>(y);
  auto rr = static_cast<__nv_bfloat16*>(residual);
  auto ww = static_cast<const __nv_bfloat16*>(w);
  auto oo = static_cast<__nv_bfloat16*>(out);
  const dim3 grid(static_cast<unsigned>(rows));
  if (cpt <= 1) return launch_pdl(rmsnorm_kernel<1>, grid, dim3(kNormThreads), 0, stream, yy, rr, ww, oo, n, eps);
  if (cpt <= 2) return launch_pdl(rmsnorm_kernel<2>, grid, dim3(kNormThreads), 0, stream, yy, rr, ww, oo, n, eps);
  return launch_pdl(rmsnorm_kernel<4>, grid, dim3(kNormThreads), 0, stream, yy, rr, ww, oo, n, eps);
}

cudaError_t launch_rope_table(int64_t positions, int head_dim, double base, float* table, cudaStream_t stream) {
  const int half = head_dim / 2;
  const int64_t total = positions * half;
  rope_table_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
      positions, half, base, reinterpret_cast<float2*>(table));
  return cudaGetLastError();
}

cudaError_t launch_qk_norm_rope(void* qkv, int64_t T, int heads, int kv_heads, int head_dim, const void* wq,
                                const void* wk, float eps, const float* table, int64_t pos0, const int64_t* pos_dev,
                                int64_t limit, void* k_cache, void* v_cache, unsigned* err, cudaStream_t stream) {
  const int64_t items = T * (heads + 2 * kv_heads);
  const dim3 grid(static_cast<unsigned>((items + 7) / 8));
  auto q = static_cast<__nv_bfloat16*>(qkv);
  auto a = static_cast<const __nv_bfloat16*>(wq);
  auto b = static_cast<const __nv_bfloat16*>(wk);
  auto tb = reinterpret_cast<const float2*>(table);
  auto kc = static_cast<__nv_bfloat16*>(k_cache);
  auto vc = static_cast<__nv_bfloat16*>(v_cache);
  switch (head_dim) {
    case 64:
      return launch_pdl(qk_norm_rope_kernel<2>, grid, dim3(256), 0, stream, q, T, heads, kv_heads, a, b, eps, tb, pos0,
                        pos_dev, limit, kc, vc, err);
    case 128:
      return launch_pdl(qk_norm_rope_kernel<4>, grid, dim3(256), 0, stream, q, T, heads, kv_heads, a, b, eps, tb, pos0,
                        pos_dev, limit, kc, vc, err);
    case 256:
      return launch_pdl(qk_norm_rope_kernel<8>, grid, dim3(256), 0, stream, q, T, heads, kv_heads, a, b, eps, tb, pos0,
                        pos_dev, limit, kc, vc, err);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_silu_mul(const void* gu, int64_t rows, int64_t inter, void* out, int num_sms, cudaStream_t stream) {
  const int64_t total = rows * (inter / 8);
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(num_sms) * 8);
  return launch_pdl(silu_mul_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                    static_cast<const __nv_bfloat16*>(gu), rows, inter, static_cast<__nv_bfloat16*>(out));
}

}  // namespace ttq
