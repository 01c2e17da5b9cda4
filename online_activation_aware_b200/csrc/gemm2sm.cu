// The TTQ projection on pairs of SMs (2-SM UMMA, tcgen05 cta_group::2):
//   Y[t, i] = sum_k X'[t, k] * (c_ik - z_ig) * sigma_ig  (+ sum_r U[t, r] B[i, r])
// (paper-daily.com deep reading of TTQ, section 2: W_hat = Q[W D^(1/2)] D^(-1/2) and
// W_hat = W_q + BA).
//
// A cluster of two CTAs on two SMs computes a 256 (weight rows) x BN (tokens) tile with
// one tcgen05.mma.cta_group::2 per 16-wide K step, issued by the even CTA: each CTA
// dequantises its own 128 weight rows into its shared memory (the A operand) and loads
// half of the X' tile (BN/2 token rows, the B operand); the tensor cores of the pair read
// both halves of B, so every SM streams only half of X' from L2. Each CTA's tensor
// memory holds its 128 rows of the fp32 accumulator (two buffers, so the epilogue of one
// tile overlaps the main loop of the next). Per stage each CTA also TMA-loads the packed
// codes of its 128 rows and their group scale/zero.
//
// Warps per CTA: 0 TMA producer, 1 MMA issuer (even CTA), 2..17 dequantisers in two
// groups that take alternate K blocks, 18..21 epilogue.
//
// Barriers: `full` (X' halves of both CTAs, on the even CTA), `cfull` (own codes tile),
// `afull` (dequantised A tiles of both CTAs, on the even CTA), `empty` (stage consumed,
// multicast to both CTAs by the MMA commit), `tfull` / `tempty` (accumulator buffers).
// No TMA multicast is used; every mbarrier wait is bounded in time, and both CTAs meet
// at a cluster barrier after initialisation and before exit.
#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kBM = 128;  // rows per CTA (256 per pair)
constexpr int kBK = 64;
constexpr int kNumDqWarps = 16;
constexpr int kDqGroupWarps = 8;  // dequant warps per stage (two groups take alternate stages)
constexpr int kNumEpiWarps = 4;
constexpr int kDqWarp0 = 2;
constexpr int kEpiWarp0 = kDqWarp0 + kNumDqWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + kNumEpiWarps);  // 704
constexpr uint32_t kATileBytes = kBM * kBK * 2;              // 16 KB
constexpr uint32_t kCodeTileBytes = kBM * 32;                // [128 rows x 32 B], 32 B swizzle
constexpr uint32_t kMetaTileBytes = kBM * 16;                // [128 rows x 8 fp16 groups]
constexpr uint32_t kCStageBytes = kCodeTileBytes + 2 * kMetaTileBytes;
constexpr int kMaxStages = 8;
constexpr int kMaxGroups = kGemmMaxGroups;
constexpr uint64_t kDrainNs = 2000000000ull;

struct __align__(16) Tail {
  uint64_t full[kMaxStages];
  uint64_t cfull[kMaxStages];
  uint64_t afull[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t stall;
  uint32_t tmem_base;
  int abort_flag;
};

// ------------------------------------------------------------------ cluster helpers

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address, in the cluster's shared window, of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrivals on a barrier of either CTA of the pair (default release semantics at CTA
// scope: the data they announce is read by this CTA's own SM).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_addr), "r"(bytes)
               : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on a barrier
// that may live in the other CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma2_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on the barrier at `bar` (shared::cta offset) in both CTAs of the pair
// when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma2_commit_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, const DevErr& err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainNs) {
      atomicOr(err.word, kErrTimeout);
      return;
    }
  }
}

// A bounded wait for the single-thread roles (TMA producer, MMA issuer) that lets the
// hardware suspend the thread until the phase completes (suspend-time hint) instead of
// polling: their polls would take issue slots from the dequantising warps that share
// their schedulers (the projection at 5120 -> 8192, T = 4096 ran 287 -> 271 us).
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_suspend(uint32_t bar, uint32_t parity, const DevErr& err,
                                                  volatile int* abort_flag) {
  constexpr uint32_t kHintNs = 2000;
  if (mbar_try_wait_hint(bar, parity, kHintNs)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait_hint(bar, parity, kHintNs)) return true;
    if ((it & 7u) == 7u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > err.wait_ns) {
        atomicOr(err.word, kErrTimeout);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// Float 128 + c for a code c (< 128) in byte `b` of `x` (code in mantissa bits 16-22).
__device__ __forceinline__ float code_plus_128(uint32_t x, int b) {
  return __uint_as_float(__byte_perm(x, 0x43000000u, 0x7044u + (static_cast<unsigned>(b) << 8)));
}

// 32 codes of one half K block -> bf16 in the 128-byte-swizzled A tile row. Each weight
// is fma(128 + c, sigma, -(128 + z) sigma) = (c - z) sigma exactly (both products fit in
// 24 bits), rounded once to bf16.
template <int Q>
__device__ __forceinline__ void dequant_half(const uint32_t (&cw)[4], float sig, float negk, uint32_t a_row,
                                             int half, int m) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    float f[8];
    if (Q == 4) {
      const uint32_t w = cw[cc];
      const uint32_t lo = w & 0x0F0F0F0Fu;
      const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        f[2 * b] = code_plus_128(lo, b);
        f[2 * b + 1] = code_plus_128(hi, b);
      }
    } else if (Q == 2) {
      const uint32_t x = cw[cc >> 1] >> ((cc & 1) * 16);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(0x43000000u | (((x >> (2 * e)) & 3u) << 16));
    } else {
      const uint32_t p0 = cw[0] >> (8 * cc), p1 = cw[1] >> (8 * cc), p2 = cw[2] >> (8 * cc);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        f[e] = __uint_as_float(
            0x43000000u | ((((p0 >> e) & 1u) | (((p1 >> e) & 1u) << 1) | (((p2 >> e) & 1u) << 2)) << 16));
    }
    uint32_t o[4];
    dequant_pack8(f, sig, negk, o);
    const int c = half * 4 + cc;
    sts128(a_row + ((c ^ (m & 7)) << 4), o[0], o[1], o[2], o[3]);
  }
}

struct KernelArgs2 {
  __nv_bfloat16* Y;
  float* partial;
  int T, d, d_out, log2g, BN, nkb, kb_per_split, ksplit, has_lr;
  int m_tiles, n_tiles, num_tiles;  // m_tiles counts 256-row pair tiles
  int inject_stall;
  DevErr err;
  // Prompts stacked along the token axis (grouped form; 1 for a single prompt): prompt p
  // owns token rows seg_tok[p] .. seg_tok[p + 1] - 1 of X', U and Y, token tiles
  // seg_tiles[p] .. seg_tiles[p + 1] - 1, and rows p * d_out .. of the codes, scale, zero.
  int groups;
  int seg_tiles[kMaxGroups + 1];
  int seg_tok[kMaxGroups + 1];
};

struct TileCoord2 {
  int m0, n0, split, kb0, nk, items;  // m0: first row of the pair tile (within its prompt)
  int tend;                           // end of the tile's prompt along the token axis
  int coff;                           // first row of the prompt's codes / scale / zero
  bool lr;
};

__device__ __forceinline__ TileCoord2 tile_coord2(const KernelArgs2& a, int t) {
  TileCoord2 c;
  const int n = t % a.n_tiles;
  const int rest = t / a.n_tiles;
  const int m = rest % a.m_tiles;
  c.split = rest / a.m_tiles;
  c.m0 = m * 2 * kBM;
  int p = 0;
  while (p + 1 < a.groups && n >= a.seg_tiles[p + 1]) ++p;
  c.n0 = a.seg_tok[p] + (n - a.seg_tiles[p]) * a.BN;
  c.tend = a.seg_tok[p + 1];
  c.coff = p * a.d_out;
  c.kb0 = c.split * a.kb_per_split;
  const int kb1 = min(a.nkb, c.kb0 + a.kb_per_split);
  c.nk = kb1 - c.kb0;
  c.lr = a.has_lr && c.split == a.ksplit - 1;
  c.items = c.nk + (c.lr ? 1 : 0);
  return c;
}

// Walks the pair's item sequence (every role of both CTAs walks the same one).
struct ItemIter2 {
  int t, j;
  TileCoord2 c;
  __device__ __forceinline__ void begin(const KernelArgs2& a) {
    t = blockIdx.x >> 1;
    j = 0;
    if (t < a.num_tiles) c = tile_coord2(a, t);
  }
  __device__ __forceinline__ bool valid(const KernelArgs2& a) const { return t < a.num_tiles; }
  __device__ __forceinline__ void next(const KernelArgs2& a) {
    if (++j == c.items) {
      j = 0;
      t += gridDim.x >> 1;
      if (t < a.num_tiles) c = tile_coord2(a, t);
    }
  }
  __device__ __forceinline__ bool is_lr() const { return c.lr && j == c.nk; }
};

// Stage index and phase bit of a ring of S stages (S need not be a power of two).
struct Pipe {
  uint32_t stage = 0, phase = 0, count = 0;
  __device__ __forceinline__ void advance(int S) {
    ++count;
    if (++stage == static_cast<uint32_t>(S)) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

template <int Q, int S>
// 22 warps: a scheduler (SM sub-partition) holds up to 6 of them in its 16 K registers, so
// at most 80 registers per thread
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(80)
    ttq_gemm2sm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_u,
                       const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                       const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_z,
                       const KernelArgs2 args) {
  static_assert(S >= 2 && S <= kMaxStages, "stages");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int BN = args.BN;
  const int HB = BN >> 1;  // token rows of X' this CTA loads
  const uint32_t b_bytes = static_cast<uint32_t>(HB) * kBK * 2;
  const uint32_t sA = base;
  const uint32_t sB = sA + S * kATileBytes;
  const uint32_t sC = sB + S * b_bytes;
  const uint32_t sTail = sC + S * kCStageBytes;
  Tail* tail = reinterpret_cast<Tail*>(smem_raw + (sTail - raw));
  volatile int* abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t tmem_cols = (2 * BN < 32) ? 32u : static_cast<uint32_t>(2 * BN);
  const DevErr err = args.err;

  const uint32_t bar_full = smem_addr(&tail->full[0]);
  const uint32_t bar_cfull = smem_addr(&tail->cfull[0]);
  const uint32_t bar_afull = smem_addr(&tail->afull[0]);
  const uint32_t bar_empty = smem_addr(&tail->empty[0]);
  const uint32_t bar_tfull = smem_addr(&tail->tfull[0]);
  const uint32_t bar_tempty = smem_addr(&tail->tempty[0]);
  const uint32_t bar_drain = smem_addr(&tail->drain);
  const uint32_t bar_stall = smem_addr(&tail->stall);
  // barriers of the even CTA, as seen from this CTA
  const uint32_t lead_full = mapa_shared(bar_full, 0);
  const uint32_t lead_afull = mapa_shared(bar_afull, 0);
  const uint32_t lead_tempty = mapa_shared(bar_tempty, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full + 8 * s, 2);                 // both CTAs' expect_tx arrivals
      mbar_init(bar_cfull + 8 * s, 1);
      mbar_init(bar_afull + 8 * s, 2 * kDqGroupWarps);  // one arrival per dequant warp of the pair
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      mbar_init(bar_tempty + 8 * b, 2 * kNumEpiWarps);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);  // nothing ever arrives here (test hook, see inject_stall)
    tail->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_c);
    prefetch_tensormap(&tm_sc);
    prefetch_tensormap(&tm_z);
    if (args.has_lr) {
      prefetch_tensormap(&tm_u);
      prefetch_tensormap(&tm_b);
    }
  }
  if (warp == 1) {
    tmem_alloc2(smem_addr(&tail->tmem_base), tmem_cols);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  // launched as a programmatic dependent: the set-up above overlaps the end of the kernel
  // that writes X' and the codes; no global memory is touched before this wait
  grid_dep_wait();
  grid_dep_launch();  // the next kernel of the stream may begin launching
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      Pipe p;
      ItemIter2 it;
      bool aborted = false;
      for (it.begin(args); it.valid(args); it.next(args), p.advance(S)) {
        const uint32_t s = p.stage;
        if (p.count >= static_cast<uint32_t>(S) &&
            !mbar_wait_suspend(bar_empty + 8 * s, p.phase ^ 1u, err, abort_flag)) {
          aborted = true;
          break;
        }
        const int row0 = it.c.m0 + static_cast<int>(rank) * kBM;
        const int tok0 = it.c.n0 + static_cast<int>(rank) * HB;
        if (it.is_lr()) {
          mbar_arrive_expect_tx_cluster(lead_full + 8 * s, kATileBytes + b_bytes);
          tma_load_2d_pair(sA + s * kATileBytes, &tm_b, lead_full + 8 * s, 0, row0);
          tma_load_2d_pair(sB + s * b_bytes, &tm_u, lead_full + 8 * s, 0, tok0);
          mbar_arrive(bar_cfull + 8 * s);
        } else {
          const int kb = it.c.kb0 + it.j;
          mbar_arrive_expect_tx_cluster(lead_full + 8 * s, b_bytes);
          tma_load_2d_pair(sB + s * b_bytes, &tm_x, lead_full + 8 * s, kb * kBK, tok0);
          const uint32_t cst = sC + s * kCStageBytes;
          mbar_arrive_expect_tx(bar_cfull + 8 * s, kCStageBytes);
          const int crow0 = row0 + it.c.coff;  // the prompt's codes / scale / zero rows
          tma_load_2d(cst, &tm_c, bar_cfull + 8 * s, (2 * Q * kb) & ~3, crow0);
          const int gx = ((kb * kBK) >> args.log2g) & ~7;
          tma_load_2d(cst + kCodeTileBytes, &tm_sc, bar_cfull + 8 * s, gx, crow0);
          tma_load_2d(cst + kCodeTileBytes + kMetaTileBytes, &tm_z, bar_cfull + 8 * s, gx, crow0);
        }
      }
      if (aborted || *abort_flag) {
        // let this CTA's copies land before its shared memory is released: the codes
        // copies count on local barriers; the X' copies count on the even CTA's barrier,
        // so give them a fixed settling time (they complete within microseconds)
        for (uint32_t k = p.count > static_cast<uint32_t>(S) ? p.count - S : 0; k < p.count; ++k) {
          const uint32_t st = k % S;
          const uint32_t ph = (k / S) & 1u;
          mbar_drain(bar_cfull + 8 * st, ph, err);
        }
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    // the whole warp walks the tiles (waits and loop values warp-uniform); one elected
    // lane issues the MMAs and commits
    if (rank == 0) {
      bool ok = true;
      if (args.inject_stall) ok = __all_sync(0xffffffffu, mbar_wait(bar_stall, 0, err, abort_flag) ? 1 : 0);
      Pipe p;
      uint32_t tc = 0;
      const uint32_t idesc = idesc_bf16_f32(2 * kBM, BN);
      for (int t = blockIdx.x >> 1; ok && t < args.num_tiles; t += gridDim.x >> 1, ++tc) {
        const TileCoord2 c = tile_coord2(args, t);
        const uint32_t b = tc & 1;
        if (tc >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_tempty + 8 * b, ((tc >> 1) - 1) & 1, err, abort_flag) ? 1 : 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + b * static_cast<uint32_t>(BN);
        for (int j = 0; j < c.items; ++j, p.advance(S)) {
          const uint32_t s = p.stage;
          const bool ready = mbar_wait_suspend(bar_full + 8 * s, p.phase, err, abort_flag) &&
                             mbar_wait_suspend(bar_afull + 8 * s, p.phase, err, abort_flag);
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
              umma2_bf16(dacc, ad + 2 * k, bd + 2 * k, idesc, (j > 0 || k > 0) ? 1u : 0u);
            umma2_commit_both(bar_empty + 8 * s);
          }
          __syncwarp();
        }
        if (ok && elect_one()) umma2_commit_both(bar_tfull + 8 * b);
        __syncwarp();
      }
      if (elect_one()) {
        umma2_commit_both(bar_drain);  // arrives once every MMA issued above has completed
        mbar_drain(bar_drain, 0, err);
      }
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ dequantisers
    // two groups of 8 warps take alternate items (stages), so two A tiles are being
    // built at once: each group's 256 threads cover the 128 rows x 2 halves of an item
    const int dtx = threadIdx.x - 32 * kDqWarp0;  // 0..511
    const int dgroup = dtx >> 8;                   // this thread's group takes items of this parity
    const int dt = dtx & 255;
    const int m = dt & (kBM - 1);
    const int half = dt >> 7;
    const int d = args.d;
    const int log2g = args.log2g;
    const uint32_t swz = static_cast<uint32_t>((m >> 2) & 1);  // 32-byte swizzle of row m
    Pipe p;
    ItemIter2 it;
    uint32_t item = 0;
    for (it.begin(args); it.valid(args); it.next(args), p.advance(S), ++item) {
      if ((item & 1u) != static_cast<uint32_t>(dgroup)) continue;
      const uint32_t s = p.stage;
      // codes landed; the producer issued them only after this stage's previous MMA
      // completed, so the A tile of the stage is free as well
      if (!__all_sync(0xffffffffu, mbar_wait(bar_cfull + 8 * s, p.phase, err, abort_flag) ? 1 : 0))
        break;  // warp-uniform: the warp arrives below as one
      if (!it.is_lr()) {
        const int i = it.c.m0 + static_cast<int>(rank) * kBM + m;
        const int kb = it.c.kb0 + it.j;
        const int k0 = kb * kBK + half * 32;
        const uint32_t a_row = sA + s * kATileBytes + m * 128;
        if (i < args.d_out && k0 < d) {
          const uint32_t cst = sC + s * kCStageBytes;
          const uint32_t crow = cst + m * 32;
          uint32_t cw[4];
          if (Q == 4) {
            const uint4 v = lds128(crow + ((static_cast<uint32_t>(half) ^ swz) << 4));
            cw[0] = v.x; cw[1] = v.y; cw[2] = v.z; cw[3] = v.w;
          } else {
            const uint4 v0 = lds128(crow + ((0u ^ swz) << 4));
            const uint4 v1 = lds128(crow + ((1u ^ swz) << 4));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const int woff = (2 * Q * kb) - ((2 * Q * kb) & ~3) + half * Q;
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
      if (lane == 0) mbar_arrive_cluster(lead_afull + 8 * s);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t tc = 0;
    for (int t = blockIdx.x >> 1; t < args.num_tiles; t += gridDim.x >> 1, ++tc) {
      const TileCoord2 c = tile_coord2(args, t);
      const uint32_t b = tc & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_tfull + 8 * b, (tc >> 1) & 1, err, abort_flag) ? 1 : 0);
      if (!ok) break;
      tc_fence_after();
      const int row = c.m0 + static_cast<int>(rank) * kBM + quarter * 32 + lane;
      const bool rok = row < args.d_out;
      // rows in pairs (an even d_out keeps every pair inside Y and 4-byte aligned)
      const bool pair_rows = (args.d_out & 1) == 0;
      const uint32_t taddr = lane_base + b * static_cast<uint32_t>(BN);
      for (int cc0 = 0; cc0 < BN; cc0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + cc0, r);
        tmem_ld_wait();
        if (args.ksplit == 1 && pair_rows) {
          // lanes 2i and 2i + 1 hold rows `row` and `row + 1`: the even lane stores both rows
          // of the even tokens, the odd lane those of the odd tokens (one 4-byte bf16 pair
          // each, 128 contiguous bytes per warp store), after one exchange per token pair
          const bool odd = (lane & 1) != 0;
          const int row0 = row & ~1;
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float keep = __uint_as_float(odd ? r[j + 1] : r[j]);
            const float give = __uint_as_float(odd ? r[j] : r[j + 1]);
            const float got = __shfl_xor_sync(0xffffffffu, give, 1);
            const int tok = c.n0 + cc0 + j + (odd ? 1 : 0);
            if (tok < c.tend && row0 < args.d_out)
              *reinterpret_cast<uint32_t*>(args.Y + static_cast<int64_t>(tok) * args.d_out + row0) =
                  odd ? pack_bf16x2(got, keep) : pack_bf16x2(keep, got);
          }
        } else if (rok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = c.n0 + cc0 + j;
            if (tok < c.tend) {
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
      if (lane == 0) mbar_arrive_cluster(lead_tempty + 8 * b);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, tmem_cols);
  }
}

}  // namespace

namespace {

int stages_2sm(int BN) {
  // per CTA and stage: A 16 KB + half of the X' tile + 8 KB of codes / scale / zero,
  // as many stages as fit in 227 KB (at most 8)
  const int per = static_cast<int>(kATileBytes + (BN / 2) * kBK * 2 + kCStageBytes);
  int s = (232448 - 1024 - static_cast<int>(sizeof(Tail))) / per;
  if (s > 8) s = 8;
  return s;
}

size_t smem_2sm(int BN, int S) {
  return 1024 + static_cast<size_t>(S) * (kATileBytes + static_cast<size_t>(BN / 2) * kBK * 2 + kCStageBytes) +
         sizeof(Tail);
}

int ilog2i(int v) {
  int r = 0;
  while ((1 << r) < v) ++r;
  return r;
}

template <int Q, int S>
cudaError_t launch_2sm_q(const CUtensorMap* m, const KernelArgs2& ka, int grid, size_t smem, cudaStream_t stream) {
  auto kern = ttq_gemm2sm_kernel<Q, S>;
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
  return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], m[5], ka);
}

template <int S>
cudaError_t launch_2sm_s(int q, const CUtensorMap* m, const KernelArgs2& ka, int grid, size_t smem,
                         cudaStream_t stream) {
  switch (q) {
    case 2: return launch_2sm_q<2, S>(m, ka, grid, smem, stream);
    case 3: return launch_2sm_q<3, S>(m, ka, grid, smem, stream);
    default: return launch_2sm_q<4, S>(m, ka, grid, smem, stream);
  }
}

}  // namespace

cudaError_t launch_gemm2sm(const GemmArgs& a, const GemmPlan& plan, const DevErr& err, int inject_stall,
                           cudaStream_t stream, int groups, const int64_t* group_T) {
  const int BN = plan.BN;
  if (groups < 1 || groups > kMaxGroups || (groups > 1 && plan.ksplit != 1)) return cudaErrorInvalidValue;
  const int HB = BN / 2;
  CUtensorMap m[6];  // x, u, b, codes, scale, zero
  if (!encode_tmap_2d(&m[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.Xf, a.T, a.d, a.d, 64, HB,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (a.r > 0) {
    if (!encode_tmap_2d(&m[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.U, a.T, 64, 64, 64, HB,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(&m[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.Blr, a.d_out, a.r, a.r, 64, kBM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    m[1] = m[0];
    m[2] = m[0];
  }
  const uint64_t wpr = static_cast<uint64_t>(a.d) * a.q / 32;
  const uint64_t gpr = static_cast<uint64_t>(a.d / a.g);
  const uint64_t crows = static_cast<uint64_t>(groups) * a.d_out;  // the prompts' codes, stacked
  if (!encode_tmap_2d(&m[3], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.codes, crows, wpr, wpr, 8, kBM,
                      CU_TENSOR_MAP_SWIZZLE_32B) ||
      !encode_tmap_2d(&m[4], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.scale, crows, gpr, gpr, 8, kBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&m[5], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.zero, crows, gpr, gpr, 8, kBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  KernelArgs2 ka;
  ka.Y = static_cast<__nv_bfloat16*>(a.Y);
  ka.partial = a.partial;
  ka.T = static_cast<int>(a.T);
  ka.d = static_cast<int>(a.d);
  ka.d_out = static_cast<int>(a.d_out);
  ka.log2g = ilog2i(a.g);
  ka.BN = BN;
  ka.nkb = plan.nkb;
  ka.kb_per_split = plan.kb_per_split;
  ka.ksplit = plan.ksplit;
  ka.has_lr = a.r > 0 ? 1 : 0;
  ka.m_tiles = plan.m_tiles;
  ka.groups = groups;
  ka.seg_tiles[0] = 0;
  ka.seg_tok[0] = 0;
  for (int p = 0; p < groups; ++p) {
    const int64_t Tp = groups == 1 ? a.T : group_T[p];
    ka.seg_tiles[p + 1] = ka.seg_tiles[p] + static_cast<int>((Tp + BN - 1) / BN);
    ka.seg_tok[p + 1] = ka.seg_tok[p] + static_cast<int>(Tp);
  }
  if (ka.seg_tok[groups] != a.T) return cudaErrorInvalidValue;
  ka.n_tiles = ka.seg_tiles[groups];
  ka.num_tiles = plan.m_tiles * ka.n_tiles * plan.ksplit;
  ka.inject_stall = inject_stall;
  ka.err = err;
  const int pairs = sms / 2;
  const int grid = 2 * (ka.num_tiles < pairs ? ka.num_tiles : pairs);
  const int S = stages_2sm(BN);
  const size_t smem = smem_2sm(BN, S);
  switch (S) {
    case 5: return launch_2sm_s<5>(a.q, m, ka, grid, smem, stream);
    case 6: return launch_2sm_s<6>(a.q, m, ka, grid, smem, stream);
    case 7: return launch_2sm_s<7>(a.q, m, ka, grid, smem, stream);
    default: return launch_2sm_s<8>(a.q, m, ka, grid, smem, stream);
  }
}

}  // namespace ttq
