// The projection of a TTQ linear layer on the 5th-generation tensor cores:
//   Y[t, i] = sum_k X'[t, k] * (c_ik - z_ig) * sigma_ig  (+ sum_r U[t, r] B[i, r])
// with X' = X diag(1/s) in bf16, the packed q-bit codes dequantised to bf16 inside the
// main loop, and the static low-rank term B (X A^T) added as one more K block
// (paper-daily.com deep reading of TTQ, section 2: W_hat = Q[W D^(1/2)] D^(-1/2) and
// W_hat = W_q + BA; section 5 notes a kernel that fuses the pre-scaling).
//
// Persistent kernel, one CTA per SM, walking 128 (weight rows) x BN (tokens) output
// tiles: D = A * B^T per K block of 64, A = dequantised weight tile [128 x 64], B = X'
// tile [BN x 64], fp32 accumulators in tensor memory, two of them so that the epilogue
// of one tile overlaps the main loop of the next. Warp roles (14 warps):
//   warp 0      TMA producer: X' tiles (and the low-rank U / B tiles) into a ring of
//               shared-memory stages, completion counted in bytes on `full` barriers;
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma (M = 128,
//               N = BN, K = 16, bf16 in, fp32 accumulate), commits each stage back to
//               `empty` and each finished tile to `tfull`;
//   warps 2-9   dequantisers: 256 threads, one per (tile row, half K block): each streams
//               its 32 codes and the group's scale/zero per K block through a private
//               cp.async ring, expands them to bf16 ((c - z) * sigma, exact in fp32, one
//               rounding) in the 128-byte-swizzled K-major layout the MMA reads, and
//               arrives on `afull`;
//   warps 10-13 epilogue: tcgen05.ld of the finished accumulator, bf16 conversion,
//               64-byte coalesced stores of Y (or fp32 split-K partials), then `tempty`.
// No TMA multicast is used anywhere. Every mbarrier wait is bounded in time.
#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kNumDqWarps = 8;
constexpr int kNumEpiWarps = 4;
constexpr int kDqWarp0 = 2;
constexpr int kEpiWarp0 = kDqWarp0 + kNumDqWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + kNumEpiWarps);  // 448
constexpr int kDqThreads = 32 * kNumDqWarps;                // 256
constexpr int kSlotBytes = 32;  // per dequant thread per K block: 16 B codes, 4 B scale, 4 B zero
constexpr uint32_t kATileBytes = kBM * kBK * 2;  // 16 KB
// TMA-fed codes: per stage a [128 rows x 32 B] codes tile (32-byte swizzle) and two
// [128 rows x 8 groups] fp16 tiles of scale and zero.
constexpr uint32_t kCodeTileBytes = kBM * 32;
constexpr uint32_t kMetaTileBytes = kBM * 16;
constexpr uint32_t kCStageBytes = kCodeTileBytes + 2 * kMetaTileBytes;  // 8 KB
constexpr int kMaxStages = 8;

struct __align__(16) Tail {
  uint64_t full[kMaxStages];
  uint64_t afull[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t stall;
  uint32_t tmem_base;
  int abort_flag;
};

// Waits (bounded by a fixed two seconds, whatever the caller's wait limit) for a phase
// without giving up on the abort flag; used to drain asynchronous work (TMA copies,
// MMAs) the CTA has started before it releases shared and tensor memory.
constexpr uint64_t kDrainNs = 2000000000ull;
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, const DevErr& err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainNs) {
      atomicOr(err.word, kErrTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

struct KernelArgs {
  const uint32_t* codes;
  const __half* scale;
  const __half* zero;
  __nv_bfloat16* Y;
  float* partial;
  int T, d, d_out, log2g, BN, nkb, kb_per_split, ksplit, has_lr;
  int m_tiles, n_tiles, num_tiles;
  int inject_stall;
  DevErr err;
};

// Output tile t: tokens fastest (neighbouring CTAs share weight rows), then weight
// rows, then the K split.
struct TileCoord {
  int m0, n0, split, kb0, nk, items;
  bool lr;
};

__device__ __forceinline__ TileCoord tile_coord(const KernelArgs& a, int t) {
  TileCoord c;
  const int n = t % a.n_tiles;
  const int rest = t / a.n_tiles;
  const int m = rest % a.m_tiles;
  c.split = rest / a.m_tiles;
  c.m0 = m * kBM;
  c.n0 = n * a.BN;
  c.kb0 = c.split * a.kb_per_split;
  const int kb1 = min(a.nkb, c.kb0 + a.kb_per_split);
  c.nk = kb1 - c.kb0;
  c.lr = a.has_lr && c.split == a.ksplit - 1;
  c.items = c.nk + (c.lr ? 1 : 0);
  return c;
}

// Walks this CTA's sequence of K-block items (tile by tile), as every role does.
struct ItemIter {
  int t;
  int j;
  TileCoord c;
  __device__ __forceinline__ void begin(const KernelArgs& a) {
    t = blockIdx.x;
    j = 0;
    if (t < a.num_tiles) c = tile_coord(a, t);
  }
  __device__ __forceinline__ bool valid(const KernelArgs& a) const { return t < a.num_tiles; }
  __device__ __forceinline__ void next(const KernelArgs& a) {
    if (++j == c.items) {
      j = 0;
      t += gridDim.x;
      if (t < a.num_tiles) c = tile_coord(a, t);
    }
  }
  __device__ __forceinline__ bool is_lr() const { return c.lr && j == c.nk; }
};

// Float 128 + c for a code c (< 128) held in byte `b` of `x`: byte permute of the code
// into mantissa bits 16-22 under the exponent of 128 (0x43000000).
__device__ __forceinline__ float code_plus_128(uint32_t x, int b) {
  return __uint_as_float(__byte_perm(x, 0x43000000u, 0x7044u + (static_cast<unsigned>(b) << 8)));
}

// Expands the 32 codes of one half K block (4 chunks of 8 weights) to bf16 and stores
// them in the swizzled A tile row `a_row`: chunk c of the row goes to 16-byte slot
// c ^ (row & 7), the 128-byte swizzle TMA would apply.
// Each weight is fma(128 + c, sigma, -(128 + z) * sigma): both products are exact in
// fp32 (at most 12 + 11 significant bits), so the result is (c - z) * sigma exactly,
// then rounded once to bf16.
template <int Q>
__device__ __forceinline__ void dequant_half(const uint32_t (&cw)[4], float sig, float negk,
                                             uint32_t a_row, int half, int m) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    float f[8];
    if (Q == 4) {
      const uint32_t w = cw[cc];
      const uint32_t lo = w & 0x0F0F0F0Fu;         // codes 0, 2, 4, 6 in bytes 0..3
      const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // codes 1, 3, 5, 7
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        f[2 * b] = code_plus_128(lo, b);
        f[2 * b + 1] = code_plus_128(hi, b);
      }
    } else if (Q == 2) {
      const uint32_t x = cw[cc >> 1] >> ((cc & 1) * 16);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(0x43000000u | (((x >> (2 * e)) & 3u) << 16));
    } else {  // Q == 3: bit planes, this chunk's 8 codes at bits [8cc, 8cc + 8)
      const uint32_t p0 = cw[0] >> (8 * cc), p1 = cw[1] >> (8 * cc), p2 = cw[2] >> (8 * cc);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        f[e] = __uint_as_float(0x43000000u | ((((p0 >> e) & 1u) | (((p1 >> e) & 1u) << 1) |
                                              (((p2 >> e) & 1u) << 2)) << 16));
    }
    uint32_t o[4];
    dequant_pack8(f, sig, negk, o);
    const int c = half * 4 + cc;
    sts128(a_row + ((c ^ (m & 7)) << 4), o[0], o[1], o[2], o[3]);
  }
}

// TQ: codes, scale and zero arrive by TMA in each stage (rows of 16-byte multiples);
// otherwise each dequantiser streams its own row through a private cp.async ring.
template <int Q, int S, int RING, bool TQ, int MINB>
__global__ void __launch_bounds__(kThreads, MINB)
    ttq_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_u,
                    const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                    const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_z,
                    const KernelArgs args) {
  static_assert(S == 2 || S == 4 || S == 8, "stages");
  static_assert(RING == 4 || RING == 8, "ring");
  constexpr int LOG2S = S == 8 ? 3 : (S == 4 ? 2 : 1);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int BN = args.BN;
  const uint32_t b_bytes = static_cast<uint32_t>(BN) * kBK * 2;
  const uint32_t sA = base;
  const uint32_t sB = sA + S * kATileBytes;
  const uint32_t sRing = sB + S * b_bytes;  // cp.async ring, or (TQ) the codes stages
  const uint32_t sTail = sRing + (TQ ? S * kCStageBytes : RING * kDqThreads * kSlotBytes);
  Tail* tail = reinterpret_cast<Tail*>(smem_raw + (sTail - raw));
  volatile int* abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t tmem_cols = (2 * BN < 32) ? 32u : static_cast<uint32_t>(2 * BN);
  const DevErr err = args.err;

  const uint32_t bar_full = smem_addr(&tail->full[0]);
  const uint32_t bar_afull = smem_addr(&tail->afull[0]);
  const uint32_t bar_empty = smem_addr(&tail->empty[0]);
  const uint32_t bar_tfull = smem_addr(&tail->tfull[0]);
  const uint32_t bar_tempty = smem_addr(&tail->tempty[0]);
  const uint32_t bar_drain = smem_addr(&tail->drain);
  const uint32_t bar_stall = smem_addr(&tail->stall);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_afull + 8 * s, kNumDqWarps);  // one arrival per dequant warp
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      mbar_init(bar_tempty + 8 * b, kNumEpiWarps);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);  // nothing ever arrives here (test hook, see inject_stall)
    tail->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_x);
    if (TQ) {
      prefetch_tensormap(&tm_c);
      prefetch_tensormap(&tm_sc);
      prefetch_tensormap(&tm_z);
    }
    if (args.has_lr) {
      prefetch_tensormap(&tm_u);
      prefetch_tensormap(&tm_b);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&tail->tmem_base), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched as a programmatic dependent: the set-up above overlaps the end of the kernel
  // that writes X' (and the codes); no global memory is touched before this wait
  grid_dep_wait();
  grid_dep_launch();  // the split-K reduction (or the next kernel) may begin launching
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kc = 0;
      ItemIter it;
      for (it.begin(args); it.valid(args); it.next(args), ++kc) {
        const uint32_t s = kc & (S - 1);
        if (kc >= S && !mbar_wait(bar_empty + 8 * s, ((kc >> LOG2S) - 1) & 1, err, abort_flag)) break;
        if (it.is_lr()) {
          mbar_arrive_expect_tx(bar_full + 8 * s, kATileBytes + b_bytes);
          tma_load_2d(sA + s * kATileBytes, &tm_b, bar_full + 8 * s, 0, it.c.m0);
          tma_load_2d(sB + s * b_bytes, &tm_u, bar_full + 8 * s, 0, it.c.n0);
        } else {
          const int kb = it.c.kb0 + it.j;
          mbar_arrive_expect_tx(bar_full + 8 * s, b_bytes + (TQ ? kCStageBytes : 0u));
          tma_load_2d(sB + s * b_bytes, &tm_x, bar_full + 8 * s, kb * kBK, it.c.n0);
          if (TQ) {
            const uint32_t cst = sRing + s * kCStageBytes;
            tma_load_2d(cst, &tm_c, bar_full + 8 * s, (2 * Q * kb) & ~3, it.c.m0);
            const int gx = ((kb * kBK) >> args.log2g) & ~7;
            tma_load_2d(cst + kCodeTileBytes, &tm_sc, bar_full + 8 * s, gx, it.c.m0);
            tma_load_2d(cst + kCodeTileBytes + kMetaTileBytes, &tm_z, bar_full + 8 * s, gx, it.c.m0);
          }
        }
      }
      if (*abort_flag) {
        // let every copy this CTA started land before shared memory is released
        for (uint32_t k = kc > S ? kc - S : 0; k < kc; ++k)
          mbar_drain(bar_full + 8 * (k & (S - 1)), (k >> LOG2S) & 1, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp walks the tiles (waits and loop values warp-uniform); one elected
    // lane issues the MMAs and commits
    {
      bool ok = true;
      if (args.inject_stall) ok = __all_sync(0xffffffffu, mbar_wait(bar_stall, 0, err, abort_flag) ? 1 : 0);
      uint32_t kc = 0;
      uint32_t tc = 0;
      const uint32_t idesc = idesc_bf16_f32(kBM, BN);
      for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x, ++tc) {
        const TileCoord c = tile_coord(args, t);
        const uint32_t b = tc & 1;
        if (tc >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_tempty + 8 * b, ((tc >> 1) - 1) & 1, err, abort_flag) ? 1 : 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + b * static_cast<uint32_t>(BN);
        for (int j = 0; j < c.items; ++j, ++kc) {
          const uint32_t s = kc & (S - 1);
          const uint32_t ph = (kc >> LOG2S) & 1;
          const bool ready = mbar_wait(bar_full + 8 * s, ph, err, abort_flag) &&
                             mbar_wait(bar_afull + 8 * s, ph, err, abort_flag);
          if (!__all_sync(0xffffffffu, ready ? 1 : 0)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(sA + s * kATileBytes);
          const uint64_t bd = sw128_kmajor_desc(sB + s * b_bytes);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_bf16(dacc, ad + 2 * k, bd + 2 * k, idesc, (j > 0 || k > 0) ? 1u : 0u);
            umma_commit(bar_empty + 8 * s);
          }
          __syncwarp();
        }
        if (ok && elect_one()) umma_commit(bar_tfull + 8 * b);
        __syncwarp();
      }
      if (elect_one()) {
        umma_commit(bar_drain);  // arrives once every MMA issued above has completed
        mbar_drain(bar_drain, 0, err);
      }
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ dequantisers
    const int dt = threadIdx.x - 32 * kDqWarp0;  // 0..255
    const int m = dt & (kBM - 1);                // tile row
    const int half = dt >> 7;                    // which 32 of the K block's 64 weights
    const int d = args.d;
    const int log2g = args.log2g;
    const int gpr = d >> log2g;  // groups per row
    const int64_t meta_total = static_cast<int64_t>(args.d_out) * gpr;
    const int64_t wpr = static_cast<int64_t>(d) * Q / 32;
    const uint32_t my_slot0 = sRing + dt * kSlotBytes;
    constexpr uint32_t kRingStride = kDqThreads * kSlotBytes;

    if constexpr (TQ) {
      // codes, scale and zero of each item arrive with the stage's TMA copies
      uint32_t kc = 0;
      ItemIter it;
      const uint32_t swz = static_cast<uint32_t>((m >> 2) & 1);  // 32-byte swizzle of row m
      for (it.begin(args); it.valid(args); it.next(args), ++kc) {
        const uint32_t s = kc & (S - 1);
        if (!__all_sync(0xffffffffu, (mbar_wait(bar_full + 8 * s, (kc >> LOG2S) & 1, err, abort_flag)) ? 1 : 0))
          break;  // warp-uniform: the warp arrives below as one
        if (!it.is_lr()) {
          const int i = it.c.m0 + m;
          const int kb = it.c.kb0 + it.j;
          const int k0 = kb * kBK + half * 32;
          const uint32_t a_row = sA + s * kATileBytes + m * 128;
          if (i < args.d_out && k0 < d) {
            const uint32_t cst = sRing + s * kCStageBytes;
            const uint32_t crow = cst + m * 32;
            uint32_t cw[4];
            if (Q == 4) {
              const uint4 v = lds128(crow + ((static_cast<uint32_t>(half) ^ swz) << 4));
              cw[0] = v.x; cw[1] = v.y; cw[2] = v.z; cw[3] = v.w;
            } else {
              const uint4 v0 = lds128(crow + ((0u ^ swz) << 4));
              const uint4 v1 = lds128(crow + ((1u ^ swz) << 4));
              const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
              const int woff = (2 * Q * kb) - ((2 * Q * kb) & ~3) + half * Q;  // first word of this half
              if (Q == 2) {
                cw[0] = woff == 0 ? w[0] : (woff == 2 ? w[2] : (woff == 4 ? w[4] : w[6]));
                cw[1] = woff == 0 ? w[1] : (woff == 2 ? w[3] : (woff == 4 ? w[5] : w[7]));
                cw[2] = cw[3] = 0u;
              } else {  // Q == 3: woff in {0, 2, 3, 5}
                cw[0] = woff == 0 ? w[0] : (woff == 2 ? w[2] : (woff == 3 ? w[3] : w[5]));
                cw[1] = woff == 0 ? w[1] : (woff == 2 ? w[3] : (woff == 3 ? w[4] : w[6]));
                cw[2] = woff == 0 ? w[2] : (woff == 2 ? w[4] : (woff == 3 ? w[5] : w[7]));
                cw[3] = 0u;
              }
            }
            const int goff = (k0 >> log2g) - (((kb * kBK) >> log2g) & ~7);  // 0..7
            const uint32_t sbits = lds16(cst + kCodeTileBytes + m * 16 + 2 * goff);
            const uint32_t zbits = lds16(cst + kCodeTileBytes + kMetaTileBytes + m * 16 + 2 * goff);
            const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(sbits)));
            const float z = __half2float(__ushort_as_half(static_cast<unsigned short>(zbits)));
            const float negk = -__fmul_rn(128.0f + z, sig);  // exact: |128 + z| < 2^12
            dequant_half<Q>(cw, sig, negk, a_row, half, m);
          } else {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int c = half * 4 + cc;
              sts128(a_row + ((c ^ (m & 7)) << 4), 0u, 0u, 0u, 0u);
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();  // the warp's shared-memory writes are ordered before its one arrival
        if (lane == 0) mbar_arrive(bar_afull + 8 * s);
      }
    } else {
      // prefetch side: issues the cp.async copies of one item into ring slot (item % RING)
      ItemIter pf;
      pf.begin(args);
      uint32_t pf_k = 0;
      auto issue = [&]() {
        if (pf.valid(args) && !pf.is_lr()) {
          const int i = pf.c.m0 + m;
          const int kb = pf.c.kb0 + pf.j;
          const int k0 = kb * kBK + half * 32;
          if (i < args.d_out && k0 < d) {
            const uint32_t dst = my_slot0 + (pf_k & (RING - 1)) * kRingStride;
            const uint32_t* src = args.codes + static_cast<int64_t>(i) * wpr + (k0 >> 5) * Q;
            if (Q == 4) {
              cp_async_16(dst, src);
            } else if (Q == 2) {
              cp_async_8(dst, src);
            } else {
              cp_async_4(dst, src);
              cp_async_4(dst + 4, src + 1);
              cp_async_4(dst + 8, src + 2);
            }
            const int64_t ge = static_cast<int64_t>(i) * gpr + (k0 >> log2g);
            const int64_t e0 = ge & ~int64_t(1);
            if (e0 + 1 < meta_total) {
              cp_async_4(dst + 16, args.scale + e0);
              cp_async_4(dst + 20, args.zero + e0);
            }
          }
        }
        cp_async_commit();
        if (pf.valid(args)) pf.next(args);
        ++pf_k;
      };
  #pragma unroll
      for (int p = 0; p < RING - 1; ++p) issue();

      uint32_t kc = 0;
      ItemIter it;
      for (it.begin(args); it.valid(args); it.next(args), ++kc) {
        issue();
        cp_async_wait<RING - 1>();
        const uint32_t s = kc & (S - 1);
        if (!__all_sync(0xffffffffu, (kc < S || mbar_wait(bar_empty + 8 * s, ((kc >> LOG2S) - 1) & 1, err, abort_flag)) ? 1 : 0))
          break;  // warp-uniform: the warp arrives below as one
        if (!it.is_lr()) {
          const int i = it.c.m0 + m;
          const int k0 = (it.c.kb0 + it.j) * kBK + half * 32;
          const uint32_t a_row = sA + s * kATileBytes + m * 128;
          if (i < args.d_out && k0 < d) {
            const uint32_t slot = my_slot0 + (kc & (RING - 1)) * kRingStride;
            const uint4 cv = lds128(slot);
            const uint4 mv = lds128(slot + 16);
            const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
            const int64_t ge = static_cast<int64_t>(i) * gpr + (k0 >> log2g);
            uint32_t sbits, zbits;
            if (((ge & ~int64_t(1)) + 1) < meta_total) {
              const int sh = static_cast<int>(ge & 1) * 16;
              sbits = (mv.x >> sh) & 0xFFFFu;
              zbits = (mv.y >> sh) & 0xFFFFu;
            } else {  // last element of an odd-length scale/zero array
              sbits = __half_as_ushort(args.scale[ge]);
              zbits = __half_as_ushort(args.zero[ge]);
            }
            const float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(sbits)));
            const float z = __half2float(__ushort_as_half(static_cast<unsigned short>(zbits)));
            const float negk = -__fmul_rn(128.0f + z, sig);  // exact: |128 + z| < 2^12
            dequant_half<Q>(cw, sig, negk, a_row, half, m);
          } else {
  #pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int c = half * 4 + cc;
              sts128(a_row + ((c ^ (m & 7)) << 4), 0u, 0u, 0u, 0u);
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();  // the warp's shared-memory writes are ordered before its one arrival
        if (lane == 0) mbar_arrive(bar_afull + 8 * s);
      }
  cp_async_wait<0>();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x, ++tc) {
      const TileCoord c = tile_coord(args, t);
      const uint32_t b = tc & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_tfull + 8 * b, (tc >> 1) & 1, err, abort_flag) ? 1 : 0);
      if (!ok) break;
      tc_fence_after();
      const int row = c.m0 + quarter * 32 + lane;
      const bool rok = row < args.d_out;
      const uint32_t taddr = lane_base + b * static_cast<uint32_t>(BN);
      for (int cc0 = 0; cc0 < BN; cc0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + cc0, r);
        tmem_ld_wait();
        if (rok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = c.n0 + cc0 + j;
            if (tok < args.T) {
              const float v = __uint_as_float(r[j]);
              if (args.ksplit == 1)
                args.Y[static_cast<int64_t>(tok) * args.d_out + row] = __float2bfloat16_rn(v);
              else
                args.partial[(static_cast<int64_t>(c.split) * args.T + tok) * args.d_out + row] = v;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_tempty + 8 * b);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Y[t, i] = bf16(sum over splits of partial[split, t, i]), summed in split order.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partial,
                                                            int ksplit, int64_t n,
                                                            __nv_bfloat16* __restrict__ Y) {
  pdl_enter();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += stride) {
    float acc = partial[e];
    for (int sp = 1; sp < ksplit; ++sp) acc = __fadd_rn(acc, partial[static_cast<int64_t>(sp) * n + e]);
    Y[e] = __float2bfloat16_rn(acc);
  }
}

// The driver's tensor-map encoder, looked up once (a function-local static is initialised
// exactly once even when several host threads make their first call together).
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

}  // namespace

namespace {
bool g_inject_stall = false;

// Small N tiles (decode, short prompts) are bound by the latency of their loads, so they
// get deeper pipelines; the stage counts keep shared memory within 227 KB.
int plan_stages(int BN, bool tq) {
  if (tq) return BN <= 32 ? 8 : 4;
  return BN <= 64 ? 8 : 4;
}
int plan_ring(int BN) { return (BN >= 256 || BN == 64) ? 4 : 8; }
int ilog2(int v) {
  int r = 0;
  while ((1 << r) < v) ++r;
  return r;
}

size_t smem_bytes_for(int BN, int stages, int ring, bool tq) {
  const size_t per_stage = kATileBytes + static_cast<size_t>(BN) * kBK * 2 + (tq ? kCStageBytes : 0);
  return 1024 + static_cast<size_t>(stages) * per_stage +
         (tq ? 0 : static_cast<size_t>(ring) * kDqThreads * kSlotBytes) + sizeof(Tail);
}


struct Maps {
  CUtensorMap x, u, b, c, sc, z;
};

template <int Q, int S, int RING, bool TQ, int MINB = 1>
cudaError_t launch_q(const Maps& mp, const KernelArgs& ka, int grid, size_t smem, cudaStream_t stream) {
  auto kern = ttq_gemm_kernel<Q, S, RING, TQ, MINB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mp.x, mp.u, mp.b, mp.c, mp.sc, mp.z, ka);
}
}  // namespace

void set_inject_stall(bool on) { g_inject_stall = on; }

// Codes and group scale/zero rows can be TMA-loaded when their row pitches are 16-byte
// multiples (every hidden size divisible by 128, with d / g divisible by 8).
bool tma_codes_ok(int64_t d, int q, int g) {
  return ((d * q / 8) % 16 == 0) && (((d / g) * 2) % 16 == 0);
}


bool encode_bf16_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint64_t row_stride_elems, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D row-major tensor map of `elem_bytes`-sized elements with a {box_cols, box_rows} box.
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, uint32_t elem_bytes, const void* base,
                 uint64_t rows, uint64_t cols, uint64_t row_stride_elems, uint32_t box_cols,
                 uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {row_stride_elems * elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D tensor map (innermost first): dims {n0, n1, n2} with byte strides {s1, s2} of dims 1
// and 2, a {b0, b1, b2} box, bf16 elements, 128-byte swizzle, zero fill outside.
bool encode_bf16_tmap_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[3] = {n0, n1, n2};
  cuuint64_t gstride[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

GemmPlan gemm_plan(int64_t T, int64_t d, int64_t d_out, int q, int g, int num_sms) {
  GemmPlan p{};
  int BN = 16;
  while (BN < 256 && BN < T) BN *= 2;
  p.BN = BN;
  // CTA pairs (2-SM MMA, half of X' per SM) for full 256-token tiles whenever the codes
  // can be TMA-loaded and there are at least two 128-row blocks of weights; short prompts
  // and decode steps (N <= 128) run faster on single CTAs
  p.pair = BN == 256 && tma_codes_ok(d, q, g) && d_out > kBM;
  const int rows_per_tile = p.pair ? 2 * kBM : kBM;
  p.m_tiles = static_cast<int>((d_out + rows_per_tile - 1) / rows_per_tile);
  p.n_tiles = static_cast<int>((T + BN - 1) / BN);
  p.nkb = static_cast<int>((d + kBK - 1) / kBK);
  p.smem_bytes = 0;
  // 16-token tiles (decode of a few tokens, very short prompts) run two CTAs per SM when
  // the codes come by TMA (4 stages of 26 KB each fit twice in shared memory)
  p.ctas_per_sm = (!p.pair && BN == 16 && tma_codes_ok(d, q, g)) ? 2 : 1;
  // One persistent CTA (or CTA pair) per SM slot (pair of SMs). Split K only when the
  // tiles cannot fill one wave, and then just enough to fill it: every split adds an fp32
  // partial write and read of Y.
  const int64_t slots = p.pair ? num_sms / 2 : static_cast<int64_t>(num_sms) * p.ctas_per_sm;
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  int best = 1;
  if (tiles < slots) {
    int64_t ns = slots / tiles;
    if (ns > p.nkb / 4) ns = p.nkb / 4;
    if (ns > 16) ns = 16;
    if (ns < 1) ns = 1;
    best = static_cast<int>(ns);
  }
  p.kb_per_split = (p.nkb + best - 1) / best;
  p.ksplit = (p.nkb + p.kb_per_split - 1) / p.kb_per_split;  // no empty split
  return p;
}

size_t gemm_partial_bytes(const GemmPlan& p, int64_t T, int64_t d_out) {
  if (p.ksplit <= 1) return 0;
  return static_cast<size_t>(p.ksplit) * static_cast<size_t>(T) * static_cast<size_t>(d_out) * sizeof(float);
}

cudaError_t launch_gemm_mainloop(const GemmArgs& a, const GemmPlan& plan, const DevErr& err,
                                 cudaStream_t stream) {
  if (plan.pair) return launch_gemm2sm(a, plan, err, g_inject_stall ? 1 : 0, stream);
  Maps mp;
  if (!encode_bf16_tmap(&mp.x, a.Xf, static_cast<uint64_t>(a.T), static_cast<uint64_t>(a.d),
                        static_cast<uint64_t>(a.d), static_cast<uint32_t>(plan.BN)))
    return cudaErrorInvalidValue;
  if (a.r > 0) {
    if (!encode_bf16_tmap(&mp.u, a.U, static_cast<uint64_t>(a.T), 64, 64, static_cast<uint32_t>(plan.BN)))
      return cudaErrorInvalidValue;
    if (!encode_bf16_tmap(&mp.b, a.Blr, static_cast<uint64_t>(a.d_out), static_cast<uint64_t>(a.r),
                          static_cast<uint64_t>(a.r), kBM))
      return cudaErrorInvalidValue;
  } else {
    mp.u = mp.x;
    mp.b = mp.x;
  }
  const bool tq = tma_codes_ok(a.d, a.q, a.g);
  if (tq) {
    const uint64_t wpr = static_cast<uint64_t>(a.d) * a.q / 32;
    const uint64_t gpr = static_cast<uint64_t>(a.d / a.g);
    if (!encode_tmap_2d(&mp.c, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.codes, a.d_out, wpr, wpr, 8, kBM,
                     CU_TENSOR_MAP_SWIZZLE_32B) ||
        !encode_tmap_2d(&mp.sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.scale, a.d_out, gpr, gpr, 8, kBM,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&mp.z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.zero, a.d_out, gpr, gpr, 8, kBM,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    mp.c = mp.sc = mp.z = mp.x;
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  KernelArgs ka;
  ka.codes = a.codes;
  ka.scale = static_cast<const __half*>(a.scale);
  ka.zero = static_cast<const __half*>(a.zero);
  ka.Y = static_cast<__nv_bfloat16*>(a.Y);
  ka.partial = a.partial;
  ka.T = static_cast<int>(a.T);
  ka.d = static_cast<int>(a.d);
  ka.d_out = static_cast<int>(a.d_out);
  ka.log2g = ilog2(a.g);
  ka.BN = plan.BN;
  ka.nkb = plan.nkb;
  ka.kb_per_split = plan.kb_per_split;
  ka.ksplit = plan.ksplit;
  ka.has_lr = a.r > 0 ? 1 : 0;
  ka.m_tiles = plan.m_tiles;
  ka.n_tiles = plan.n_tiles;
  ka.num_tiles = plan.m_tiles * plan.n_tiles * plan.ksplit;
  ka.inject_stall = g_inject_stall ? 1 : 0;
  ka.err = err;
  const int slots = sms * plan.ctas_per_sm;
  const int grid = ka.num_tiles < slots ? ka.num_tiles : slots;
  if (plan.ctas_per_sm == 2) {
    // 16-token tiles, two CTAs per SM (4 stages each, at most 72 registers a thread): two
    // independent pipelines per SM for the latency-bound hand-off of short K loops
    const size_t smem2 = smem_bytes_for(plan.BN, 4, 4, true);
    switch (a.q) {
      case 2: return launch_q<2, 4, 4, true, 2>(mp, ka, grid, smem2, stream);
      case 3: return launch_q<3, 4, 4, true, 2>(mp, ka, grid, smem2, stream);
      default: return launch_q<4, 4, 4, true, 2>(mp, ka, grid, smem2, stream);
    }
  }
  const int S = plan_stages(plan.BN, tq);
  const int R = plan_ring(plan.BN);
  const size_t smem = smem_bytes_for(plan.BN, S, R, tq);
#define TTQ_LAUNCH(SS, RR, TT)                                              \
  switch (a.q) {                                                            \
    case 2: return launch_q<2, SS, RR, TT>(mp, ka, grid, smem, stream);     \
    case 3: return launch_q<3, SS, RR, TT>(mp, ka, grid, smem, stream);     \
    default: return launch_q<4, SS, RR, TT>(mp, ka, grid, smem, stream);    \
  }
  if (tq) {
    if (S == 4) { TTQ_LAUNCH(4, 4, true) }
    TTQ_LAUNCH(8, 4, true)
  }
  if (S == 4 && R == 4) { TTQ_LAUNCH(4, 4, false) }
  if (S == 4 && R == 8) { TTQ_LAUNCH(4, 8, false) }
  if (S == 8 && R == 4) { TTQ_LAUNCH(8, 4, false) }
  TTQ_LAUNCH(8, 8, false)
#undef TTQ_LAUNCH
}

cudaError_t launch_gemm_reduce(const GemmArgs& a, const GemmPlan& plan, cudaStream_t stream) {
  if (plan.ksplit <= 1) return cudaSuccess;
  const int64_t n = a.T * a.d_out;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_pdl(splitk_reduce_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                    static_cast<const float*>(a.partial), plan.ksplit, n, static_cast<__nv_bfloat16*>(a.Y));
}

cudaError_t launch_gemm(const GemmArgs& a, const GemmPlan& plan, const DevErr& err,
                        cudaStream_t stream) {
  cudaError_t e = launch_gemm_mainloop(a, plan, err, stream);
  if (e == cudaSuccess) e = launch_gemm_reduce(a, plan, stream);
  return e;
}

}  // namespace ttq
