// Decode steps with few tokens (b <= 2): the projection as a CUDA-core GEMV that streams
// the prefill's packed codes once (paper-daily.com deep reading of TTQ, section 6:
// quantisation parameters are computed at prefill and reused at decode).
//
// For a weight row i and a group G of g inputs, cut into 32-input units V:
//   sum_{k in G} x'_tk (c_ik - z) sigma
//     = sigma * sum_{V in G} ( sum_{k in V} (128 + c_ik) x'_tk - (128 + z) sum_{k in V} x'_tk )
// so each weight costs one byte permute (128 + c as an fp32, exact) and half of a two-wide
// FMA (fma.rn.f32x2: pairs of inputs for one token, the token pair for two);
// each unit is finished on its own (scale and zero of its group), so a lane may take any
// set of units; the unit sums of x' come with x' from a small prep kernel.
//
// Layout of the work: one warp per 4 weight rows, the 32 lanes spanning the inputs (lane j
// takes the rows' 32-input units j, j + 32, ...), so that each row's lanes read contiguous
// codes per step (16-byte loads that bypass L1) and every x' value a lane loads (16-byte
// loads through L1, contiguous across the warp) serves 4 weights: a load's cost is its
// per-lane register writeback, so the reuse in registers is what keeps x' traffic below
// the code traffic (2 rows a warp measured slower at every shape of a Qwen3-8B layer).
// The codes of the next kDepth units are in flight while one is consumed; the 32 lanes are
// summed by shuffles in a fixed order. CTAs of 8 rows (up to 8 on an SM at 128 registers a
// thread) stage the rows' scale and zero in shared memory. x' (fp32, chunk-major, see xoff)
// and the unit sums come from a prep kernel chained to the GEMV by programmatic dependent
// launch: the GEMV issues its first code loads before waiting for x'. For two tokens the
// CTA's codes come instead by bulk copies into shared memory (fewer registers a thread).
#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kDepth = 4;  // 32-input units of codes in flight per lane (for each of its rows)
constexpr int kGemvThreads = 64;                                  // 2 warps
constexpr int kRowsPerCta = kRowsPerWarp * kGemvThreads / 32;     // 8

__device__ __forceinline__ float code_plus_128f(uint32_t x, int b) {
  return __uint_as_float(__byte_perm(x, 0x43000000u, 0x7044u + (static_cast<unsigned>(b) << 8)));
}

// Packed fp32 pairs (sm_100's two-wide FMA: each lane of the pair rounds like an fp32 FMA).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(a), "f"(b));
  return v;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return make_float2(a, b);
}

// The Q words holding one row's codes for one 32-input unit.
template <int Q>
struct UnitWords {
  uint32_t w[Q];
};

// Codes are read once: they bypass L1 (no_allocate) so that x', which every warp reads
// again and again, stays there.
template <int Q>
__device__ __forceinline__ UnitWords<Q> load_unit(const uint32_t* __restrict__ src) {
  UnitWords<Q> u;
  if (Q == 4) {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(u.w[0]), "=r"(u.w[1]), "=r"(u.w[2]), "=r"(u.w[3])
                 : "l"(src));
  } else if (Q == 2) {
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(u.w[0]), "=r"(u.w[1]) : "l"(src));
  } else {
#pragma unroll
    for (int i = 0; i < Q; ++i)
      asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(u.w[i]) : "l"(src + i));
  }
  return u;
}

// 128 + c (as fp32) of the unit's inputs 4*c4 .. 4*c4 + 3.
template <int Q>
__device__ __forceinline__ void codes4(const UnitWords<Q>& u, int c4, float (&f)[4]) {
  if (Q == 4) {
    // word c4 / 2 holds inputs 8j .. 8j + 7 as nibbles (input 8j + e at bits 4e)
    const uint32_t w = u.w[c4 >> 1];
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;  // even, odd inputs
    const int b0 = (c4 & 1) * 2;
    f[0] = code_plus_128f(lo, b0);
    f[1] = code_plus_128f(hi, b0);
    f[2] = code_plus_128f(lo, b0 + 1);
    f[3] = code_plus_128f(hi, b0 + 1);
  } else if (Q == 2) {
    // word c4 / 4 holds inputs 16j .. 16j + 15 (input 16j + e at bits 2e): masked by
    // 0x03030303 after a shift of 2e, byte b holds input 16j + 4b + e, one byte permute
    // per code (the masks are shared by the four c4 of a word once unrolled)
    const uint32_t w = u.w[c4 >> 2];
    const int b = c4 & 3;
#pragma unroll
    for (int e = 0; e < 4; ++e) f[e] = code_plus_128f((w >> (2 * e)) & 0x03030303u, b);
  } else {
    // three bit planes: bit b of input k at bit k of word b
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 4 * c4 + e;
      const uint32_t c = ((u.w[0] >> k) & 1u) | (((u.w[1] >> k) & 1u) << 1) | (((u.w[2] >> k) & 1u) << 2);
      f[e] = __uint_as_float(0x43000000u | (c << 16));
    }
  }
}

// One row's codes of one unit from shared memory (BULK form).
template <int Q>
__device__ __forceinline__ UnitWords<Q> lds_unit(const uint32_t* p) {
  UnitWords<Q> u;
  if (Q == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    u.w[0] = v.x; u.w[1] = v.y; u.w[2] = v.z; u.w[3] = v.w;
  } else if (Q == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    u.w[0] = v.x; u.w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < Q; ++i) u.w[i] = p[i];
  }
  return u;
}

// Bulk copy (no multicast) of `bytes` from global memory into this CTA's shared memory,
// counted in bytes on the barrier at `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// B floats of x' (or of the unit sums) for one input, token-minor.
template <int B>
struct TokVec {
  float v[B];
};
template <int B>
__device__ __forceinline__ TokVec<B> load_tok(const float* p) {
  TokVec<B> r;
  if (B == 1) {
    r.v[0] = p[0];
  } else if (B == 2) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    r.v[0] = a.x; r.v[1] = a.y;
  } else {
#pragma unroll
    for (int i = 0; i < B; i += 4) {
      const float4 a = *reinterpret_cast<const float4*>(p + i);
      r.v[i] = a.x; r.v[i + 1] = a.y; r.v[i + 2] = a.z; r.v[i + 3] = a.w;
    }
  }
  return r;
}

// x' layout, chunk-major: input k = 32 u + 4 c + e of token t sits at
// ((c * units + u) * 4 + e) * B + t, so that 32 lanes reading chunk c of 32 consecutive
// units read one contiguous block.
__host__ __device__ __forceinline__ int64_t xoff(int c, int u, int units, int B) {
  return (static_cast<int64_t>(c) * units + u) * 4 * B;
}

// One warp per kRowsPerWarp weight rows; lane j takes the rows' 32-input units j, j + 32,
// j + 64, ... so that each row's 32 lanes read 512 contiguous bytes of codes per step, and
// every x' value a lane loads serves all kRowsPerWarp rows (a load's cost is its per-lane
// register writeback, so reuse in registers is what cuts it). The codes of the next
// kDepth units are in flight while one is consumed (at d = 5120 a lane's five units are
// nearly all requested at once).
// BULK: instead, one thread copies the CTA's rows of codes (contiguous in memory) into
// shared memory with bulk copies, in np pieces along the inputs, each counted on a barrier
// of its own, before x' is ready; the lanes read their units from there as the pieces land.
template <int Q, int B, bool BULK>
__global__ void __launch_bounds__(kGemvThreads) decode_gemv_kernel(
    const uint32_t* __restrict__ codes, const __half* __restrict__ scale, const __half* __restrict__ zero,
    const float* xp, const float* usum, int d, int d_out, int log2g, const __nv_bfloat16* __restrict__ U,
    const __nv_bfloat16* __restrict__ Blr, int r, __nv_bfloat16* __restrict__ Y, int nb, int64_t cstride,
    int64_t mstride, int64_t wsf, int np, DevErr err) {
  // [kRowsPerCta][gpr] (sigma, 128 + z); BULK: then the codes [kRowsPerCta][d q / 32] words,
  // np barriers and an abort flag
  extern __shared__ __align__(16) float2 meta_sm[];
  {
    // request blockIdx.y of a batched decode: its own codes, scale, zero, x', U and Y
    const int64_t rq = blockIdx.y;
    codes += rq * cstride;
    scale += rq * mstride;
    zero += rq * mstride;
    xp += rq * wsf;
    usum += rq * wsf;
    if (U != nullptr) U += rq * nb * 64;
    Y += rq * nb * d_out;
  }
  constexpr int R = kRowsPerWarp;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int upr = d >> 5;                            // 32-input units per row
  const int lgu = log2g - 5;                         // log2 of units per group
  const int gpr = d >> log2g;
  const int row0 = blockIdx.x * kRowsPerCta + R * warp;  // the warp's first row
  const uint32_t* crow[R];
#pragma unroll
  for (int i = 0; i < R; ++i) crow[i] = codes + static_cast<int64_t>(row0 + i < d_out ? row0 + i : 0) * upr * Q;
  const int nsteps = (upr - lane + 31) >> 5;         // units of this lane: lane, lane + 32, ...
  uint32_t* code_sm = reinterpret_cast<uint32_t*>(meta_sm + kRowsPerCta * gpr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(code_sm + kRowsPerCta * upr * Q);
  volatile int* abort_sm = reinterpret_cast<volatile int*>(bars + np);
  const int pu = upr / (np > 0 ? np : 1);  // units per piece (BULK)

  // the first kDepth units' codes (BULK: all of the CTA's codes), and the CTA's scale/zero
  // into shared memory, before x' is ready
  UnitWords<Q> cb[BULK ? 1 : kDepth][R];
  if (BULK) {
    if (threadIdx.x == 0) {
      for (int pc = 0; pc < np; ++pc) mbar_init(smem_addr(bars + pc), 1);
      *abort_sm = 0;
      fence_mbar_init();
      const int nrows = min(kRowsPerCta, d_out - static_cast<int>(blockIdx.x) * kRowsPerCta);
      const uint32_t pbytes = static_cast<uint32_t>(pu * Q * 4);
      const uint32_t* src0 = codes + static_cast<int64_t>(blockIdx.x) * kRowsPerCta * upr * Q;
      for (int pc = 0; pc < np; ++pc) {
        mbar_arrive_expect_tx(smem_addr(bars + pc), static_cast<uint32_t>(nrows) * pbytes);
        for (int i = 0; i < nrows; ++i)
          bulk_load(smem_addr(code_sm + (i * upr + pc * pu) * Q), src0 + (static_cast<int64_t>(i) * upr + pc * pu) * Q,
                    pbytes, smem_addr(bars + pc));
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < kDepth; ++k) {
      if (k < nsteps) {
#pragma unroll
        for (int i = 0; i < R; ++i) cb[k][i] = load_unit<Q>(crow[i] + static_cast<int64_t>(lane + 32 * k) * Q);
      }
    }
  }
  {
    // the CTA's rows of scale and zero are contiguous: 16-byte loads when aligned and whole
    // (at g = 32 a row has d / 32 groups, too many for 2-byte loads one after another)
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta * gpr;
    const __half* sc = scale + m0;
    const __half* zc = zero + m0;
    const bool whole = (blockIdx.x + 1) * kRowsPerCta <= d_out;
    if (whole && ((reinterpret_cast<uintptr_t>(sc) | reinterpret_cast<uintptr_t>(zc)) & 15u) == 0) {
      const int n8 = kRowsPerCta * gpr / 8;
#pragma unroll 4
      for (int c = threadIdx.x; c < n8; c += blockDim.x) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(sc) + c);
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(zc) + c);
        const __half* ah = reinterpret_cast<const __half*>(&a);
        const __half* bh = reinterpret_cast<const __half*>(&b);
#pragma unroll
        for (int j = 0; j < 8; ++j) meta_sm[8 * c + j] = make_float2(__half2float(ah[j]), 128.0f + __half2float(bh[j]));
      }
    } else {
      for (int e = threadIdx.x; e < kRowsPerCta * gpr; e += blockDim.x) {
        const int rr = e / gpr, gi = e - rr * gpr;
        const int mrow = blockIdx.x * kRowsPerCta + rr;
        float2 v = make_float2(0.f, 128.f);
        if (mrow < d_out) {
          const int64_t o = static_cast<int64_t>(mrow) * gpr + gi;
          v = make_float2(__half2float(scale[o]), 128.0f + __half2float(zero[o]));
        }
        meta_sm[e] = v;
      }
    }
  }
  grid_dep_wait();    // x' and its unit sums are written by the prep kernel
  grid_dep_launch();  // the next kernel of the stream may begin launching
  __syncthreads();  // meta is in place

  float pacc[R][B];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int t = 0; t < B; ++t) pacc[i][t] = 0.f;
  int landed = 0;  // BULK: pieces known to have landed
  bool ok = true;
  const int wsteps = (upr + 31) >> 5;  // steps of the warp (of lane 0): the loop is warp-uniform
  for (int s0 = 0; ok && s0 < wsteps; s0 += kDepth) {
#pragma unroll
    for (int hb = 0; hb < kDepth; ++hb) {
      const int st = s0 + hb;
      if (BULK) {
        // the pieces holding this step's units of every lane of the warp (warp-uniform)
        const int need = min(np - 1, (32 * st + 31) / pu);
        while (ok && landed <= need) {
          ok = __all_sync(0xffffffffu, mbar_wait(smem_addr(bars + landed), 0, err, abort_sm) ? 1 : 0);
          ++landed;
        }
        if (!ok) break;
      }
      if (st < nsteps) {
        const int u = lane + 32 * st;
        // two-wide accumulators: one token, pairs of inputs (even, odd); two tokens, the
        // token pair of each input
        uint64_t acc2[R];
#pragma unroll
        for (int i = 0; i < R; ++i) acc2[i] = 0ull;
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          // x' of inputs 4 c4 .. 4 c4 + 3 of unit u for all B tokens
          float x[4 * B];
          const float* xb = xp + xoff(c4, u, upr, B);
#pragma unroll
          for (int i2 = 0; i2 < B; ++i2) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(xb + 4 * i2));
            x[4 * i2] = v.x; x[4 * i2 + 1] = v.y; x[4 * i2 + 2] = v.z; x[4 * i2 + 3] = v.w;
          }
          uint64_t xv[4];
          if (B == 1) {
            xv[0] = f2(x[0], x[1]);
            xv[1] = f2(x[2], x[3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) xv[e] = f2(x[e * B], x[e * B + 1]);
          }
#pragma unroll
          for (int i = 0; i < R; ++i) {
            float f[4];
            if (BULK)
              codes4<Q>(lds_unit<Q>(code_sm + ((R * warp + i) * upr + u) * Q), c4, f);
            else
              codes4<Q>(cb[hb][i], c4, f);
            if (B == 1) {
              acc2[i] = ffma2(f2(f[0], f[1]), xv[0], acc2[i]);
              acc2[i] = ffma2(f2(f[2], f[3]), xv[1], acc2[i]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) acc2[i] = ffma2(f2(f[e], f[e]), xv[e], acc2[i]);
            }
          }
        }
        float acc[R][B];
#pragma unroll
        for (int i = 0; i < R; ++i) {
          const float2 a = f2_unpack(acc2[i]);
          if (B == 1) {
            acc[i][0] = __fadd_rn(a.x, a.y);
          } else {
            acc[i][0] = a.x;
            acc[i][B - 1] = a.y;
          }
        }
        if (!BULK && st + kDepth < nsteps) {  // refill the slot just consumed, kDepth units ahead
#pragma unroll
          for (int i = 0; i < R; ++i)
            cb[hb][i] = load_unit<Q>(crow[i] + static_cast<int64_t>(u + 32 * kDepth) * Q);
        }
        // sigma * (sum (128 + c) x' - (128 + z) sum x') for this unit's group, per row
        const TokVec<B> xs = load_tok<B>(usum + static_cast<int64_t>(u) * B);
        const int grp = u >> lgu;
#pragma unroll
        for (int i = 0; i < R; ++i) {
          const float2 sz = meta_sm[(R * warp + i) * gpr + grp];
#pragma unroll
          for (int t = 0; t < B; ++t) pacc[i][t] = __fmaf_rn(sz.x, __fmaf_rn(-sz.y, xs.v[t], acc[i][t]), pacc[i][t]);
        }
      }
    }
  }
  if (BULK) {
    // after a failed wait, let every copy land before the shared memory is released
    __syncthreads();
    if (threadIdx.x == 0 && *abort_sm) {
      for (int pc = 0; pc < np; ++pc) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(smem_addr(bars + pc), 0) && globaltimer_ns() - t0 < 2000000000ull) {
        }
      }
    }
    if (*abort_sm) return;
  }
  // the warp's 32 lanes in a fixed order (butterfly: every lane ends with the same sums)
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int t = 0; t < B; ++t)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) pacc[i][t] += __shfl_xor_sync(0xffffffffu, pacc[i][t], off);
  // lane i * B + t stores token t of row i
  const int oi = lane / B, ot = lane - oi * B;
  const int orow = row0 + oi;
  if (oi < R && ot < nb && orow < d_out) {
    float y = 0.f;
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int t = 0; t < B; ++t)
        if (i == oi && t == ot) y = pacc[i][t];
    // the rank-r term: r % 8 == 0, the row of B and of U read as 16-byte chunks, all
    // requested before the first FMA
    const uint4* ur = reinterpret_cast<const uint4*>(U + static_cast<int64_t>(ot) * 64);
    const uint4* br = reinterpret_cast<const uint4*>(Blr + static_cast<int64_t>(orow) * r);
    for (int c0 = 0; c0 < r / 8; c0 += 4) {
      uint4 uv[4], bv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c0 + c < r / 8) {
          uv[c] = __ldg(ur + c0 + c);
          bv[c] = __ldg(br + c0 + c);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c0 + c < r / 8) {
          const uint32_t uw[4] = {uv[c].x, uv[c].y, uv[c].z, uv[c].w};
          const uint32_t bw[4] = {bv[c].x, bv[c].y, bv[c].z, bv[c].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            y = __fmaf_rn(__uint_as_float(uw[k] << 16), __uint_as_float(bw[k] << 16), y);
            y = __fmaf_rn(__uint_as_float(uw[k] & 0xFFFF0000u), __uint_as_float(bw[k] & 0xFFFF0000u), y);
          }
        }
      }
    }
    Y[static_cast<int64_t>(ot) * d_out + orow] = __float2bfloat16_rn(y);
  }
}

// x'[k][t] = bf16(x[t][k] * (1 / s_k)) as fp32 (rows t >= nb zero), the same rounding as
// the prefill's fold, in the chunk-major layout of xoff, and usum[v][t] = sum of x' over
// the 32-input unit v. One warp per (unit, token), in the first `prep_blocks` blocks.
// With a low-rank side path (A non-null) nb * 64 more blocks form U = X A^T (row stride
// 64): block (t, j) strides its 256 threads over d in 8-input chunks, fp32 sums reduced in
// a fixed order (warps, then the 8 warp sums); U[t][j] = 0 for r <= j < 64.
template <int B>
__global__ void __launch_bounds__(256) decode_prep_kernel(const __nv_bfloat16* __restrict__ X, int nb, int d,
                                                          const float* __restrict__ s, float* __restrict__ xp,
                                                          float* __restrict__ usum, int64_t wsf, int prep_blocks,
                                                          const __nv_bfloat16* __restrict__ A, int r,
                                                          __nv_bfloat16* __restrict__ U) {
  pdl_enter();  // X is written by the kernel ahead; then the GEMV may start loading codes
  {
    // request blockIdx.y of a batched decode: its own tokens, statistic, x' and U
    const int64_t rq = blockIdx.y;
    X += rq * nb * d;
    s += rq * d;
    xp += rq * wsf;
    usum += rq * wsf;
    if (U != nullptr) U += rq * nb * 64;
  }
  if (static_cast<int>(blockIdx.x) >= prep_blocks) {
    __shared__ float red[8];
    const int o = static_cast<int>(blockIdx.x) - prep_blocks;  // t * 64 + j
    const int t = o >> 6, j = o & 63;
    if (j >= r) {
      if (threadIdx.x == 0) U[o] = __float2bfloat16_rn(0.f);
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
      U[o] = __float2bfloat16_rn(v);
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int units = d >> 5;
  if (pair >= units * B) return;
  const int v = pair / B;
  const int t = pair - v * B;
  const int k = 32 * v + lane;
  float x = 0.f;
  if (t < nb)
    x = __bfloat162float(__float2bfloat16_rn(
        __fmul_rn(__bfloat162float(X[static_cast<int64_t>(t) * d + k]), __frcp_rn(s[k]))));
  xp[xoff(lane >> 2, v, units, B) + (lane & 3) * B + t] = x;
  float sum = x;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) usum[static_cast<int64_t>(v) * B + t] = sum;
}

int gemv_tokens(int64_t b) { return b <= 1 ? 1 : 2; }

size_t round16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }

// Workspace of the decode: x' [d][B] (chunks rotated per unit) and the unit sums [d / 32][B].
size_t gemv_ws_bytes(int64_t b, int64_t d) {
  const int B = gemv_tokens(b);
  return round16(static_cast<size_t>(d) * B * 4) + round16(static_cast<size_t>(d / 32) * B * 4);
}

template <int Q, int B>
cudaError_t launch_qb(const DecodeArgs& a, uint8_t* ws, cudaStream_t stream) {
  int lg = 0;
  while ((1 << lg) < a.g) ++lg;
  float* xp = reinterpret_cast<float*>(ws);
  float* usum = reinterpret_cast<float*>(ws + round16(static_cast<size_t>(a.d) * B * 4));
  const int units = static_cast<int>(a.d / 32);
  const int64_t wsf = static_cast<int64_t>(gemv_ws_bytes(a.b, a.d) / 4);  // one request's workspace, floats
  // the prep blocks, then (low-rank side path) one block per output of U
  const int prep_blocks = (units * B + 7) / 8;
  const bool lr = a.A != nullptr && a.r > 0;
  const int u_blocks = lr ? static_cast<int>(a.b) * 64 : 0;
  cudaError_t e = launch_pdl(decode_prep_kernel<B>, dim3(prep_blocks + u_blocks, a.requests), dim3(256), 0, stream,
                             static_cast<const __nv_bfloat16*>(a.X), static_cast<int>(a.b), static_cast<int>(a.d), a.s,
                             xp, usum, wsf, prep_blocks, static_cast<const __nv_bfloat16*>(lr ? a.A : nullptr),
                             lr ? a.r : 0, static_cast<__nv_bfloat16*>(lr ? const_cast<void*>(a.U) : nullptr));
  if (e != cudaSuccess) return e;
  // two tokens: codes by bulk copies when every row and every piece of a row is a whole
  // number of 16-byte blocks and the CTA's codes fit in shared memory beside its
  // scale/zero (at 5120 -> 8192, q = 4: 18.5 us a step against 19.9 us with the codes in
  // registers; for one token the register form is faster, 12.2 against 14.9 us)
  const size_t meta_bytes = static_cast<size_t>(kRowsPerCta) * (a.d / a.g) * sizeof(float2);
  const int64_t upr = a.d / 32;
  int np = 0;
  if (B == 2 && (a.d * Q) % 128 == 0 && (reinterpret_cast<uintptr_t>(a.codes) & 15u) == 0) {
    for (int n : {4, 2, 1}) {
      if (upr % n == 0 && ((upr / n) * Q) % 4 == 0 && (n == 1 || upr / n >= 32)) {
        np = n;
        break;
      }
    }
  }
  const size_t bulk_smem = meta_bytes + static_cast<size_t>(kRowsPerCta) * upr * Q * 4 + 8 * 4 + 16;
  if (bulk_smem > 200 * 1024) np = 0;
  const size_t smem = np > 0 ? bulk_smem : meta_bytes;
  auto kern = np > 0 ? decode_gemv_kernel<Q, B, true> : decode_gemv_kernel<Q, B, false>;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.d_out + kRowsPerCta - 1) / kRowsPerCta), static_cast<unsigned>(a.requests));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const uint32_t*>(a.codes),
                         static_cast<const __half*>(a.scale), static_cast<const __half*>(a.zero),
                         static_cast<const float*>(xp), static_cast<const float*>(usum), static_cast<int>(a.d),
                         static_cast<int>(a.d_out), lg, static_cast<const __nv_bfloat16*>(a.U),
                         static_cast<const __nv_bfloat16*>(a.Blr), a.r, static_cast<__nv_bfloat16*>(a.Y),
                         static_cast<int>(a.b), a.d_out * (a.d / 32) * Q, a.d_out * (a.d / a.g), wsf, np, a.err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int Q>
cudaError_t launch_q(const DecodeArgs& a, uint8_t* ws, cudaStream_t stream) {
  if (gemv_tokens(a.b) == 1) return launch_qb<Q, 1>(a, ws, stream);
  return launch_qb<Q, 2>(a, ws, stream);
}

}  // namespace

bool decode_gemv_ok(int64_t b, int64_t d) { return b >= 1 && b <= kGemvMaxTokens && d % 32 == 0; }

size_t decode_gemv_ws_bytes(int64_t b, int64_t d) { return gemv_ws_bytes(b, d); }

cudaError_t launch_decode_gemv(const DecodeArgs& a, void* ws, cudaStream_t stream) {
  auto* w = static_cast<uint8_t*>(ws);
  switch (a.q) {
    case 2: return launch_q<2>(a, w, stream);
    case 3: return launch_q<3>(a, w, stream);
    default: return launch_q<4>(a, w, stream);
  }
}

}  // namespace ttq
