// Causal grouped-query attention of a prompt on the tensor cores (sm_100a), the attention of
// the Qwen3-shaped decoder layers whose linears run under TTQ (architecture table of the
// thelatestinai.com listing of the TTQ paper, Table 15: 32 query heads, 8 key/value heads of
// head dim 128 for Qwen3-8B). For query row t and head h (key/value head h / (H / Hkv)):
//   out[t, h] = sum_{p <= t} softmax_p(q_t . k_p / sqrt(D)) v_p,
// computed flash-style: one CTA per (tile of 128 queries, head) walks the key tiles of BK
// positions (64: two CTAs then share an SM) up to its diagonal, keeping a running row
// maximum m and sum l in fp32.
//
// Roles (6 warps):
//   warp 0    TMA: the Q tile once, then K and V tiles of the head's key/value head into a
//             two-stage ring (128-byte swizzled boxes of BK positions x 64 channels);
//   warp 1    owns the tensor memory and issues tcgen05.mma: S_j = Q K_j^T into one of two
//             BK-column fp32 accumulators (issued one tile ahead, so S_{j+1} runs while the
//             softmax works on S_j), and O += P_j V_j into a third; V is read as an MN-major
//             operand straight from its [position, channel] tile;
//   warps 2-5 softmax, one query row per thread (tensor-memory lane quadrant w % 4): scale,
//             causal mask on the diagonal tile, new row maximum, P = exp2(s - m) rounded to
//             bf16 into shared memory as the A operand of the second product, the running sum
//             from the same rounded values, and the rescaling of O in tensor memory by
//             exp2(m_old - m_new) before the next product lands, only when some row's
//             maximum has risen by more than 2^8; at the end O / l in bf16.
// The probabilities are rounded to bf16 for the tensor cores (the sum uses the rounded
// values, so the normalisation matches them); scores, maxima, sums and O stay fp32.
// Every mbarrier wait is bounded: a CTA that gives up records TTQ_ERR_TIMEOUT, drains the
// copies and products it started, frees its tensor memory and returns.
#include <cfloat>
#include <cmath>

#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kAttnTile = 128;        // queries per CTA
constexpr int kAttnThreads = 192;     // 6 warps
constexpr float kRescaleSlack = 8.0f;  // log2 units a row maximum may rise before O is rescaled
constexpr uint32_t kRowBox = 128 * 128;                  // 128 rows x 128 B (64 bf16): a Q or P box

struct AttnBars {
  uint64_t q_full;
  uint64_t k_full[2];
  uint64_t v_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// D channels, key tiles of BK positions. smem: Q | K0 | K1 | V0 | V1 | P (1024-byte
// aligned; Q as D / 64 boxes of 128 rows x 64 channels, K and V as D / 64 boxes of BK rows,
// P as BK / 64 boxes of 128 rows x 64 positions), then the barriers. Tensor memory: S0, S1
// (BK columns each), O (D columns). Two CTAs share an SM when both fit twice.
template <int D, int BK>
struct AttnLayout {
  static constexpr uint32_t kKVBox = BK * 128;
  static constexpr uint32_t kQBytes = (D / 64) * kRowBox;
  static constexpr uint32_t kKVBytes = (D / 64) * kKVBox;
  static constexpr uint32_t kPBytes = (BK / 64) * kRowBox;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffV = kOffK + 2 * kKVBytes;
  static constexpr uint32_t kOffP = kOffV + 2 * kKVBytes;
  static constexpr uint32_t kOffBars = kOffP + kPBytes;
  // + up to 896 bytes to align the base to 1024 (the dynamic base is 128-byte aligned; the
  // kernel checks its layout fits before it touches shared memory)
  static constexpr size_t kSmem = kOffBars + sizeof(AttnBars) + 896;
  static constexpr uint32_t kColS0 = 0, kColS1 = BK, kColO = 2 * BK;
  static constexpr uint32_t kTmemCols = (2 * BK + D) <= 256 ? 256u : 512u;
  // two CTAs per SM when their shared memory (plus the 1 KB each reserves) fits the SM's
  // 228 KB and their tensor memory its 512 columns
  static constexpr int kMinBlocks = (2 * (kSmem + 1024) <= 228 * 1024 && 2 * kTmemCols <= 512) ? 2 : 1;
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzled layout: rows of
// 64 bf16 (128 B) along MN, 8-row groups along K 1024 B apart (stride byte offset), and the
// next 64 MN elements one box further on (leading byte offset). Version 1, layout 2.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// 2^x (the hardware approximation; inputs are <= 0 here, -inf gives 0).
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Waits bounded by a fixed two seconds, ignoring the abort flag: drains copies and products
// a CTA started before it frees shared and tensor memory.
__device__ __forceinline__ void attn_drain(uint32_t bar, uint32_t parity, const DevErr& err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 2000000000ull) {
      atomicOr(err.word, kErrTimeout);
      return;
    }
  }
}

struct AttnArgs {
  int T;            // tokens of the prompt (positions 0 .. T-1)
  int G;            // query heads per key/value head
  int n_q;          // query tiles
  int ld_out;       // heads * head_dim
  float scale_log2; // log2(e) / sqrt(head_dim)
  __nv_bfloat16* out;
  DevErr err;
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v ? 1 : 0) != 0; }

template <int D, int BK>
__global__ void __launch_bounds__(kAttnThreads, AttnLayout<D, BK>::kMinBlocks)
    prompt_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using L = AttnLayout<D, BK>;
  constexpr uint32_t kOffQ = L::kOffQ, kOffK = L::kOffK, kOffV = L::kOffV, kOffP = L::kOffP;
  constexpr uint32_t kKVBox = L::kKVBox, kKVBytes = L::kKVBytes;
  constexpr uint32_t kColS0 = L::kColS0, kColS1 = L::kColS1, kColO = L::kColO;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if ((base - raw) + L::kOffBars + sizeof(AttnBars) > L::kSmem) {
    // the allocation cannot hold the aligned layout: report and leave before any barrier,
    // copy or tensor-memory allocation
    if (threadIdx.x == 0) atomicOr(a.err.word, kErrLayout);
    return;
  }
  AttnBars* bars = reinterpret_cast<AttnBars*>(smem_raw + (base - raw) + L::kOffBars);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int qt = a.n_q - 1 - static_cast<int>(blockIdx.y);  // the longest rows first
  const int hk = h / a.G;
  const int q0 = qt * kAttnTile;
  // key tiles up to the diagonal (and not past the prompt)
  const int nkv = min((q0 + kAttnTile + BK - 1) / BK, (a.T + BK - 1) / BK);
  volatile int* abort_flag = &bars->abort_flag;
  const DevErr err = a.err;
  const uint32_t b_q = smem_addr(&bars->q_full);
  const uint32_t b_kf = smem_addr(&bars->k_full[0]);
  const uint32_t b_vf = smem_addr(&bars->v_full[0]);
  const uint32_t b_ke = smem_addr(&bars->kv_empty[0]);
  const uint32_t b_sf = smem_addr(&bars->s_full[0]);
  const uint32_t b_sfree = smem_addr(&bars->s_free[0]);
  const uint32_t b_p = smem_addr(&bars->p_full);
  const uint32_t b_o = smem_addr(&bars->o_done);
  const uint32_t b_drain = smem_addr(&bars->drain);
  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_kf + 8 * i, 1);
      mbar_init(b_vf + 8 * i, 1);
      mbar_init(b_ke + 8 * i, 1);
      mbar_init(b_sf + 8 * i, 1);
      mbar_init(b_sfree + 8 * i, 4);  // one arrival per softmax warp
    }
    mbar_init(b_p, 4);
    mbar_init(b_o, 1);
    mbar_init(b_drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&bars->tmem_base), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_enter();  // q, k and v are written by the kernel ahead in the stream
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(b_q, L::kQBytes);
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) tma_load_2d(base + kOffQ + bx * kRowBox, &tm_q, b_q, h * D + 64 * bx, q0);
      int j = 0;
      for (; j < nkv; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(b_ke + 8 * st, ((j >> 1) - 1) & 1, err, abort_flag)) break;
        const int p0 = j * BK;
        const uint32_t ks = base + kOffK + st * kKVBytes;
        const uint32_t vs = base + kOffV + st * kKVBytes;
        mbar_arrive_expect_tx(b_kf + 8 * st, kKVBytes);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) tma_load_3d(ks + bx * kKVBox, &tm_k, b_kf + 8 * st, 64 * bx, hk, p0);
        mbar_arrive_expect_tx(b_vf + 8 * st, kKVBytes);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) tma_load_3d(vs + bx * kKVBox, &tm_v, b_vf + 8 * st, 64 * bx, hk, p0);
      }
      if (*abort_flag) {
        // every copy this CTA started lands before its shared memory is released
        attn_drain(b_q, 0, err);
        for (int k = j > 2 ? j - 2 : 0; k < j; ++k) {
          attn_drain(b_kf + 8 * (k & 1), (k >> 1) & 1, err);
          attn_drain(b_vf + 8 * (k & 1), (k >> 1) & 1, err);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_s = idesc_bf16_f32(kAttnTile, BK);
    const uint32_t idesc_pv = idesc_bf16_f32(kAttnTile, D) | (1u << 16);  // B (V) MN-major
    bool ok = warp_all(mbar_wait(b_q, 0, err, abort_flag));
    // S_j = Q K_j^T into accumulator j & 1 (K = head_dim in steps of 16: 4 per 64-channel box)
    auto issue_s = [&](int j) -> bool {
      const int st = j & 1;
      if (!warp_all(mbar_wait(b_kf + 8 * st, (j >> 1) & 1, err, abort_flag))) return false;
      if (j >= 2 && !warp_all(mbar_wait(b_sfree + 8 * st, ((j >> 1) - 1) & 1, err, abort_flag))) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t d = tmem + (st ? kColS1 : kColS0);
        const uint32_t ks = base + kOffK + st * kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * kRowBox + (kk & 3) * 32;
          const uint32_t ko = (kk >> 2) * kKVBox + (kk & 3) * 32;
          umma_bf16(d, sw128_kmajor_desc(base + kOffQ + qo), sw128_kmajor_desc(ks + ko), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(b_sf + 8 * st);
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; ok && j < nkv; ++j) {
      if (j + 1 < nkv && !(ok = issue_s(j + 1))) break;
      const int st = j & 1;
      if (!warp_all(mbar_wait(b_p, j & 1, err, abort_flag)) ||
          !warp_all(mbar_wait(b_vf + 8 * st, (j >> 1) & 1, err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        // O += P_j V_j: K = the tile's BK positions in steps of 16 (P: 4 per 64-position box;
        // V: 16 positions = two 8-row groups of 1024 B, the next 64 channels one box on)
        const uint32_t vs = base + kOffV + st * kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint32_t pa = base + kOffP + (kk >> 2) * kRowBox + (kk & 3) * 32;
          umma_bf16(tmem + kColO, sw128_kmajor_desc(pa), sw128_mnmajor_desc(vs + kk * 2048, kKVBox), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(b_ke + 8 * st);  // K_j and V_j may be overwritten once these are done
        umma_commit(b_o);            // O now holds P_0 V_0 + ... + P_j V_j
      }
      __syncwarp();
    }
    // every product issued above completes before tensor memory is released
    if (elect_one()) umma_commit(b_drain);
    __syncwarp();
    attn_drain(b_drain, 0, err);
  } else {
    // ------------------------------------------------------------ softmax (warps 2-5)
    const int quad = warp & 3;                       // tensor-memory lanes 32 quad .. 32 quad + 31
    const int r = quad * 32 + lane;                  // this thread's query row in the tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = a.scale_log2;
    float m = -FLT_MAX, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int st = j & 1;
      if (!warp_all(mbar_wait(b_sf + 8 * st, (j >> 1) & 1, err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[BK];
      {
        const uint32_t sc = tl + (st ? kColS1 : kColS0);
#pragma unroll
        for (int c32 = 0; c32 < BK / 32; ++c32)
          tmem_ld_32x32b_x32(sc + 32 * c32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c32]));
        tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_sfree + 8 * st);  // the accumulator may take S_{j+2}
      // scaled scores (log2 units); keys after the query (the diagonal tiles) are masked:
      // key j * BK + k is visible to row q0 + r when k <= q0 + r - j * BK
      const int lim = min(BK - 1, q0 + r - j * BK);
      // the row maximum as four interleaved chains (a 64-deep chain would set the latency)
      float mx4[4] = {m, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
      for (int k = 0; k < BK; ++k) {
        const float sv = k <= lim ? __fmul_rn(__uint_as_float(sr[k]), c) : -FLT_MAX;
        sr[k] = __float_as_uint(sv);
        mx4[k & 3] = fmaxf(mx4[k & 3], sv);
      }
      float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      // the row keeps its reference maximum until the tile's maximum exceeds it by more
      // than kRescaleSlack (log2 units): P = exp2(s - m) then stays below 2^kRescaleSlack
      // (exact in range for bf16, and l sums the same values), and O is rescaled in tensor
      // memory only when some row of the warp moves its reference
      if (mx <= m + kRescaleSlack) mx = m;
      const float corr = exp2_approx(__fsub_rn(m, mx));
      if (j > 0) {
        // P_{j-1} V_{j-1} has landed: O may be rescaled and the P buffer rewritten
        if (!warp_all(mbar_wait(b_o, (j - 1) & 1, err, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f ? 1 : 0)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tl + kColO + 32 * cc, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__fmul_rn(__uint_as_float(o[e]), corr));
            tmem_st_32x32b_x32(tl + kColO + 32 * cc, o);
          }
          tmem_st_wait();
        }
      }
      // P = exp2(s - m) rounded to bf16 into the swizzled K-major A tile (row r, positions in
      // 16-byte chunks of 8: chunk k8 of box k8 / 8 at slot (k8 % 8) ^ (r % 8)); the row sum
      // adds the rounded values
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};  // the row sum as four chains, added in a fixed order
      const uint32_t prow = base + kOffP + r * 128;
#pragma unroll
      for (int k8 = 0; k8 < BK / 8; ++k8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = exp2_approx(__fsub_rn(__uint_as_float(sr[8 * k8 + 2 * e]), mx));
          const float p1 = exp2_approx(__fsub_rn(__uint_as_float(sr[8 * k8 + 2 * e + 1]), mx));
          w[e] = pack_bf16x2(p0, p1);
          rs4[e] = __fadd_rn(rs4[e], __fadd_rn(bf16lo_to_f32(w[e]), bf16hi_to_f32(w[e])));
        }
        const uint32_t addr = prow + (k8 >> 3) * kRowBox + (((k8 & 7) ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                     "r"(w[3])
                     : "memory");
      }
      const float rs = __fadd_rn(__fadd_rn(rs4[0], rs4[1]), __fadd_rn(rs4[2], rs4[3]));
      l = __fmaf_rn(l, corr, rs);
      m = mx;
      fence_proxy_async_smem();  // the tensor cores read P through the async proxy
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_p);
    }
    if (ok && warp_all(mbar_wait(b_o, (nkv - 1) & 1, err, abort_flag))) {
      tc_fence_after();
      const float inv = __fdiv_rn(1.f, l);
      const int t = q0 + r;
      __nv_bfloat16* orow = a.out + static_cast<int64_t>(t) * a.ld_out + h * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tl + kColO + 32 * cc, o);
        tmem_ld_wait();
        if (t < a.T) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16x2(__fmul_rn(__uint_as_float(o[8 * q4]), inv), __fmul_rn(__uint_as_float(o[8 * q4 + 1]), inv));
            v.y = pack_bf16x2(__fmul_rn(__uint_as_float(o[8 * q4 + 2]), inv), __fmul_rn(__uint_as_float(o[8 * q4 + 3]), inv));
            v.z = pack_bf16x2(__fmul_rn(__uint_as_float(o[8 * q4 + 4]), inv), __fmul_rn(__uint_as_float(o[8 * q4 + 5]), inv));
            v.w = pack_bf16x2(__fmul_rn(__uint_as_float(o[8 * q4 + 6]), inv), __fmul_rn(__uint_as_float(o[8 * q4 + 7]), inv));
            *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * q4) = v;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace

namespace {

template <int D, int BK>
cudaError_t launch_attention_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                               int heads, cudaStream_t stream) {
  constexpr size_t smem = AttnLayout<D, BK>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(prompt_attention_kernel<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e == cudaSuccess)  // all of the SM's unified memory as shared memory, for two CTAs
    e = cudaFuncSetAttribute(prompt_attention_kernel<D, BK>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(heads), static_cast<unsigned>(a.n_q));
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prompt_attention_kernel<D, BK>, tq, tk, tv, a);
}

// Key tiles of 64 positions: with the two-stage K/V ring and the P tile, a CTA takes 112 KB of
// shared memory (D = 128) and 256 tensor-memory columns, so two CTAs share each SM and one's
// products run while the other's softmax works.
constexpr int kKeyTile = 64;
static_assert(AttnLayout<128, kKeyTile>::kMinBlocks == 2 && AttnLayout<64, kKeyTile>::kMinBlocks == 2,
              "two CTAs per SM");

}  // namespace

cudaError_t launch_prompt_attention(const void* qkv, int64_t T, int heads, int kv_heads, int head_dim,
                                    const void* k_cache, const void* v_cache, void* out, const DevErr& err,
                                    cudaStream_t stream) {
  if ((head_dim != 64 && head_dim != 128) || heads % kv_heads != 0 || T < 1) return cudaErrorInvalidValue;
  const uint64_t ncols = static_cast<uint64_t>(heads + 2 * kv_heads) * head_dim;
  CUtensorMap tq, tk, tv;
  // q: the first heads * head_dim channels of each row of the stacked projection
  if (!encode_bf16_tmap(&tq, qkv, static_cast<uint64_t>(T), ncols, ncols, kAttnTile)) return cudaErrorInvalidValue;
  // caches [position, kv head, channel], of which positions 0 .. T-1 (later ones read as zero)
  const uint64_t s1 = static_cast<uint64_t>(head_dim) * 2, s2 = static_cast<uint64_t>(kv_heads) * head_dim * 2;
  if (!encode_bf16_tmap_3d(&tk, k_cache, head_dim, kv_heads, static_cast<uint64_t>(T), s1, s2, 64, 1, kKeyTile) ||
      !encode_bf16_tmap_3d(&tv, v_cache, head_dim, kv_heads, static_cast<uint64_t>(T), s1, s2, 64, 1, kKeyTile))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.T = static_cast<int>(T);
  a.G = heads / kv_heads;
  a.n_q = static_cast<int>((T + kAttnTile - 1) / kAttnTile);
  a.ld_out = heads * head_dim;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  a.out = static_cast<__nv_bfloat16*>(out);
  a.err = err;
  return head_dim == 64 ? launch_attention_d<64, kKeyTile>(tq, tk, tv, a, heads, stream)
                        : launch_attention_d<128, kKeyTile>(tq, tk, tv, a, heads, stream);
}

}  // namespace ttq
