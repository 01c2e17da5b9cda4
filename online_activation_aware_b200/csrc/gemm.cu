// The projection of a TTQ linear layer on the 5th-generation tensor cores:
//   Y[t, i] = sum_k X'[t, k] * (c_ik - z_ig) * sigma_ig  (+ sum_r U[t, r] B[i, r])
// with X' = X diag(1/s) in bf16, the packed q-bit codes dequantised to bf16 inside the
// main loop, and the static low-rank term B (X A^T) added as one more K block
// (paper-daily.com deep reading of TTQ, section 2: W_hat = Q[W D^(1/2)] D^(-1/2) and
// W_hat = W_q + BA; section 5 notes a kernel that fuses the pre-scaling).
//
// One CTA computes a 128 (weight rows) x BN (tokens) tile: D = A * B^T with
// A = dequantised weight tile [128 x 64] and B = X' tile [BN x 64] per K block, the fp32
// accumulator in tensor memory (128 lanes x BN columns). Warp roles:
//   warp 0      TMA producer: X' tiles (and the low-rank U / B tiles) into a ring of
//               shared-memory stages, completion counted in bytes on `full` barriers;
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma (M=128, N=BN,
//               K=16, bf16 in, fp32 accumulate) and commits each stage back to `empty`;
//   warps 2-5   dequantisers: each thread owns one weight row of the tile, streams its
//               codes and group scale/zero through a private cp.async ring, writes 64
//               bf16 per K block in the 128-byte-swizzled K-major layout the MMA reads,
//               and arrives on `afull`; afterwards they are the epilogue (TMEM -> Y).
// No TMA multicast is used anywhere. Every mbarrier wait is bounded in time.
#include "ttq_internal.h"

namespace ttq {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxStages = 4;
constexpr int kThreads = 192;
constexpr int kDqThreads = 128;
constexpr int kSlotBytes = 48;  // per thread per K block: 32 B codes + 8 B scale + 8 B zero
constexpr uint32_t kATileBytes = kBM * kBK * 2;  // 16 KB

struct __align__(16) Tail {
  uint64_t full[kMaxStages];
  uint64_t afull[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t accum;
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
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

// exact float value of a small non-negative integer code: 2^23 + c, as bits
__device__ __forceinline__ float magic_code(uint32_t c) { return __uint_as_float(0x4B000000u | c); }

struct KernelArgs {
  const uint32_t* codes;
  const __half* scale;
  const __half* zero;
  __nv_bfloat16* Y;
  float* partial;
  int T, d, d_out, g, BN, stages, nkb, kb_per_split, ksplit, has_lr;
  DevErr err;
};

template <int Q, int RING>
__global__ void __launch_bounds__(kThreads, 2)
    ttq_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_u,
                    const __grid_constant__ CUtensorMap tm_b, const KernelArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int BN = args.BN;
  const int S = args.stages;
  const uint32_t b_bytes = static_cast<uint32_t>(BN) * kBK * 2;
  const uint32_t sA = base;
  const uint32_t sB = sA + S * kATileBytes;
  const uint32_t sRing = sB + S * b_bytes;
  const uint32_t sTail = sRing + RING * kDqThreads * kSlotBytes;
  Tail* tail = reinterpret_cast<Tail*>(smem_raw + (sTail - raw));
  volatile int* abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kBM;
  const int n0 = blockIdx.x * BN;
  const int split = blockIdx.z;
  const int kb0 = split * args.kb_per_split;
  const int kb1 = min(args.nkb, kb0 + args.kb_per_split);
  const int nk = kb1 - kb0;  // weight K blocks of this CTA
  const bool lr_here = args.has_lr && split == args.ksplit - 1;
  const int nblocks = nk + (lr_here ? 1 : 0);
  const uint32_t tmem_cols = BN < 32 ? 32u : static_cast<uint32_t>(BN);
  const DevErr err = args.err;

  const uint32_t bar_full = smem_addr(&tail->full[0]);
  const uint32_t bar_afull = smem_addr(&tail->afull[0]);
  const uint32_t bar_empty = smem_addr(&tail->empty[0]);
  const uint32_t bar_accum = smem_addr(&tail->accum);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_afull + 8 * s, kDqThreads);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_accum, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_x);
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
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nblocks; ++it) {
        const int s = it % S;
        if (it >= S && !mbar_wait(bar_empty + 8 * s, ((it / S) - 1) & 1, err, abort_flag)) break;
        if (lr_here && it == nblocks - 1) {
          mbar_arrive_expect_tx(bar_full + 8 * s, kATileBytes + b_bytes);
          tma_load_2d(sA + s * kATileBytes, &tm_b, bar_full + 8 * s, 0, m0);
          tma_load_2d(sB + s * b_bytes, &tm_u, bar_full + 8 * s, 0, n0);
        } else {
          mbar_arrive_expect_tx(bar_full + 8 * s, b_bytes);
          tma_load_2d(sB + s * b_bytes, &tm_x, bar_full + 8 * s, (kb0 + it) * kBK, n0);
        }
        issued = it + 1;
      }
      if (*abort_flag) {
        // let every copy this CTA started land before shared memory is released
        for (int it = issued > S ? issued - S : 0; it < issued; ++it)
          mbar_drain(bar_full + 8 * (it % S), (it / S) & 1, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, BN);
      for (int it = 0; it < nblocks; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const bool is_lr = lr_here && it == nblocks - 1;
        if (!mbar_wait(bar_full + 8 * s, ph, err, abort_flag)) break;
        if (!is_lr && !mbar_wait(bar_afull + 8 * s, ph, err, abort_flag)) break;
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(sA + s * kATileBytes);
        const uint64_t bd = sw128_kmajor_desc(sB + s * b_bytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16(tmem, ad + 2 * k, bd + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
        umma_commit(bar_empty + 8 * s);
      }
      umma_commit(bar_accum);  // arrives once every MMA issued above has completed
      mbar_drain(bar_accum, 0, err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequantisers
    const int dt = threadIdx.x - 64;  // 0..127: tile row
    const int i = m0 + dt;
    const bool row_ok = i < args.d_out;
    const int d = args.d;
    const int g = args.g;
    const int gpr = d / g;  // groups per row
    const int64_t meta_total = static_cast<int64_t>(args.d_out) * gpr;
    const int64_t wpr = static_cast<int64_t>(d) * Q / 32;
    const uint32_t* crow = args.codes + static_cast<int64_t>(row_ok ? i : 0) * wpr;
    const int64_t meta_row = static_cast<int64_t>(row_ok ? i : 0) * gpr;
    const uint32_t my_slot0 = sRing + dt * kSlotBytes;

    auto issue = [&](int j) {
      if (j < nk && row_ok) {
        const int kb = kb0 + j;
        const uint32_t dst = my_slot0 + (j % RING) * (kDqThreads * kSlotBytes);
        const int kvalid = min(kBK, d - kb * kBK);  // 64, or 32 on a ragged last block
        const int nwords = kvalid * Q / 32;
        const uint32_t* src = crow + static_cast<int64_t>(kb) * 2 * Q;
        if (Q == 4) {
          cp_async_16(dst, src);
          if (nwords == 8) cp_async_16(dst + 16, src + 4);
        } else {
          for (int w = 0; w < nwords; ++w) cp_async_4(dst + 4 * w, src + w);
        }
        // group scale/zero: the 4-byte-aligned fp16 pairs covering this block's groups
        const int64_t e = meta_row + (static_cast<int64_t>(kb) * kBK) / g;
        const int64_t e0 = e & ~int64_t(1);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (e0 + 2 * w + 1 < meta_total) {
            cp_async_4(dst + 32 + 4 * w, args.scale + e0 + 2 * w);
            cp_async_4(dst + 40 + 4 * w, args.zero + e0 + 2 * w);
          }
        }
      }
      cp_async_commit();
    };

#pragma unroll
    for (int j = 0; j < RING - 1; ++j) issue(j);

    for (int j = 0; j < nk; ++j) {
      issue(j + RING - 1);
      cp_async_wait<RING - 1>();
      const int s = j % S;
      if (j >= S && !mbar_wait(bar_empty + 8 * s, ((j / S) - 1) & 1, err, abort_flag)) break;
      const uint32_t slot = my_slot0 + (j % RING) * (kDqThreads * kSlotBytes);
      const uint32_t a_row = sA + s * kATileBytes + dt * 128;
      const int kb = kb0 + j;
      if (row_ok) {
        const uint4 c0 = lds128(slot);
        const uint4 c1 = lds128(slot + 16);
        const uint4 mt = lds128(slot + 32);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const uint32_t sw[2] = {mt.x, mt.y};
        const uint32_t zw[2] = {mt.z, mt.w};
        const int64_t e = meta_row + (static_cast<int64_t>(kb) * kBK) / g;
        const int64_t e0 = e & ~int64_t(1);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int kk = kb * kBK + c * 8;
          uint32_t o0 = 0, o1 = 0, o2 = 0, o3 = 0;
          if (kk < d) {
            const int64_t ge = meta_row + kk / g;
            const int off = static_cast<int>(ge - e0);  // 0..2
            const uint32_t sbits = (sw[off >> 1] >> ((off & 1) * 16)) & 0xFFFFu;
            const uint32_t zbits = (zw[off >> 1] >> ((off & 1) * 16)) & 0xFFFFu;
            float sig = __half2float(__ushort_as_half(static_cast<unsigned short>(sbits)));
            float zf = __half2float(__ushort_as_half(static_cast<unsigned short>(zbits)));
            if (ge == meta_total - 1 && (meta_total & 1)) {  // last element of an odd-length array
              sig = __half2float(args.scale[ge]);
              zf = __half2float(args.zero[ge]);
            }
            const float zm = 8388608.0f + zf;  // exact: |z| <= 2048
            uint32_t cc[8];
            if (Q == 4) {
              const uint32_t w = cw[c];
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2) cc[e2] = (w >> (4 * e2)) & 0xFu;
            } else if (Q == 2) {
              const uint32_t w = cw[c >> 1] >> ((c & 1) * 16);
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2) cc[e2] = (w >> (2 * e2)) & 0x3u;
            } else {
              const int u = c >> 2;
              const int sh = (c & 3) * 8;
              const uint32_t p0 = cw[3 * u] >> sh, p1 = cw[3 * u + 1] >> sh, p2 = cw[3 * u + 2] >> sh;
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2)
                cc[e2] = ((p0 >> e2) & 1u) | (((p1 >> e2) & 1u) << 1) | (((p2 >> e2) & 1u) << 2);
            }
            float f[8];
#pragma unroll
            for (int e2 = 0; e2 < 8; ++e2) f[e2] = __fmul_rn(__fsub_rn(magic_code(cc[e2]), zm), sig);
            o0 = pack_bf16x2(f[0], f[1]);
            o1 = pack_bf16x2(f[2], f[3]);
            o2 = pack_bf16x2(f[4], f[5]);
            o3 = pack_bf16x2(f[6], f[7]);
          }
          sts128(a_row + ((c ^ (dt & 7)) << 4), o0, o1, o2, o3);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) sts128(a_row + ((c ^ (dt & 7)) << 4), 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_afull + 8 * s);
    }
    cp_async_wait<0>();

    // ------------------------------------------------------------ epilogue
    // tcgen05.ld is warp-collective: take the TMEM path only when every lane saw the
    // accumulator complete
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(bar_accum, 0, err, abort_flag) ? 1 : 0);
    if (acc_ok) {
      tc_fence_after();
      const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
      const int row = m0 + quarter * 32 + lane;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      const bool rok = row < args.d_out;
      if (BN >= 32) {
        for (int cc0 = 0; cc0 < BN; cc0 += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + cc0, r);
          tmem_ld_wait();
          if (rok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = n0 + cc0 + j;
              if (t < args.T) {
                const float v = __uint_as_float(r[j]);
                if (args.ksplit == 1)
                  args.Y[static_cast<int64_t>(t) * args.d_out + row] = __float2bfloat16_rn(v);
                else
                  args.partial[(static_cast<int64_t>(split) * args.T + t) * args.d_out + row] = v;
              }
            }
          }
        }
      } else {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr, r);
        tmem_ld_wait();
        if (rok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = n0 + j;
            if (t < args.T) {
              const float v = __uint_as_float(r[j]);
              if (args.ksplit == 1)
                args.Y[static_cast<int64_t>(t) * args.d_out + row] = __float2bfloat16_rn(v);
              else
                args.partial[(static_cast<int64_t>(split) * args.T + t) * args.d_out + row] = v;
            }
          }
        }
      }
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
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += stride) {
    float acc = partial[e];
    for (int sp = 1; sp < ksplit; ++sp) acc = __fadd_rn(acc, partial[static_cast<int64_t>(sp) * n + e]);
    Y[e] = __float2bfloat16_rn(acc);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

size_t smem_bytes_for(int BN, int stages, int ring) {
  return 1024 + static_cast<size_t>(stages) * kATileBytes + static_cast<size_t>(stages) * BN * kBK * 2 +
         static_cast<size_t>(ring) * kDqThreads * kSlotBytes + sizeof(Tail);
}

}  // namespace

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

static int plan_ring(int BN) { return BN >= 256 ? 4 : 8; }
static int plan_stages(int BN) { return BN >= 128 ? 4 : 2; }

GemmPlan gemm_plan(int64_t T, int64_t d, int64_t d_out, int num_sms) {
  GemmPlan p{};
  int BN = 16;
  while (BN < 256 && BN < T) BN *= 2;
  p.BN = BN;
  p.m_tiles = static_cast<int>((d_out + kBM - 1) / kBM);
  p.n_tiles = static_cast<int>((T + BN - 1) / BN);
  p.nkb = static_cast<int>((d + kBK - 1) / kBK);
  p.smem_bytes = smem_bytes_for(BN, plan_stages(BN), plan_ring(BN));
  const size_t per_sm = 233472;  // 228 KB of shared memory per SM
  int per = static_cast<int>(per_sm / (p.smem_bytes + 1024));
  if (per < 1) per = 1;
  if (per > 2) per = 2;
  const int64_t slots = static_cast<int64_t>(num_sms) * per;
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  // Split K only when the tiles cannot fill one wave of the machine, and then just
  // enough to fill that one wave: every split adds an fp32 partial write and read of Y.
  int best = 1;
  if (tiles < slots) {
    int64_t ns = slots / tiles;
    if (ns > p.nkb / 4) ns = p.nkb / 4;
    if (ns > 16) ns = 16;
    if (ns < 1) ns = 1;
    best = static_cast<int>(ns);
  }
  p.ksplit = best;
  p.kb_per_split = (p.nkb + best - 1) / best;
  p.ksplit = (p.nkb + p.kb_per_split - 1) / p.kb_per_split;  // no empty split
  return p;
}

size_t gemm_partial_bytes(const GemmPlan& p, int64_t T, int64_t d_out) {
  if (p.ksplit <= 1) return 0;
  return static_cast<size_t>(p.ksplit) * static_cast<size_t>(T) * static_cast<size_t>(d_out) * sizeof(float);
}

template <int Q, int RING>
static cudaError_t launch_q(const CUtensorMap& tx, const CUtensorMap& tu, const CUtensorMap& tb,
                            const KernelArgs& ka, dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = ttq_gemm_kernel<Q, RING>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tx, tu, tb, ka);
  return cudaGetLastError();
}

cudaError_t launch_gemm_mainloop(const GemmArgs& a, const GemmPlan& plan, const DevErr& err,
                                 cudaStream_t stream) {
  CUtensorMap tx, tu, tb;
  if (!encode_bf16_tmap(&tx, a.Xf, static_cast<uint64_t>(a.T), static_cast<uint64_t>(a.d),
                        static_cast<uint64_t>(a.d), static_cast<uint32_t>(plan.BN)))
    return cudaErrorInvalidValue;
  if (a.r > 0) {
    if (!encode_bf16_tmap(&tu, a.U, static_cast<uint64_t>(a.T), 64, 64, static_cast<uint32_t>(plan.BN)))
      return cudaErrorInvalidValue;
    if (!encode_bf16_tmap(&tb, a.Blr, static_cast<uint64_t>(a.d_out), static_cast<uint64_t>(a.r),
                          static_cast<uint64_t>(a.r), kBM))
      return cudaErrorInvalidValue;
  } else {
    tu = tx;
    tb = tx;
  }
  KernelArgs ka;
  ka.codes = a.codes;
  ka.scale = static_cast<const __half*>(a.scale);
  ka.zero = static_cast<const __half*>(a.zero);
  ka.Y = static_cast<__nv_bfloat16*>(a.Y);
  ka.partial = a.partial;
  ka.T = static_cast<int>(a.T);
  ka.d = static_cast<int>(a.d);
  ka.d_out = static_cast<int>(a.d_out);
  ka.g = a.g;
  ka.BN = plan.BN;
  ka.stages = plan_stages(plan.BN);
  ka.nkb = plan.nkb;
  ka.kb_per_split = plan.kb_per_split;
  ka.ksplit = plan.ksplit;
  ka.has_lr = a.r > 0 ? 1 : 0;
  ka.err = err;
  dim3 grid(plan.n_tiles, plan.m_tiles, plan.ksplit);
  const int ring = plan_ring(plan.BN);
  cudaError_t e;
  if (ring == 4) {
    switch (a.q) {
      case 2: e = launch_q<2, 4>(tx, tu, tb, ka, grid, plan.smem_bytes, stream); break;
      case 3: e = launch_q<3, 4>(tx, tu, tb, ka, grid, plan.smem_bytes, stream); break;
      default: e = launch_q<4, 4>(tx, tu, tb, ka, grid, plan.smem_bytes, stream); break;
    }
  } else {
    switch (a.q) {
      case 2: e = launch_q<2, 8>(tx, tu, tb, ka, grid, plan.smem_bytes, stream); break;
      case 3: e = launch_q<3, 8>(tx, tu, tb, ka, grid, plan.smem_bytes, stream); break;
      default: e = launch_q<4, 8>(tx, tu, tb, ka, grid, plan.smem_bytes, stream); break;
    }
  }
  return e;
}

cudaError_t launch_gemm_reduce(const GemmArgs& a, const GemmPlan& plan, cudaStream_t stream) {
  if (plan.ksplit <= 1) return cudaSuccess;
  const int64_t n = a.T * a.d_out;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  splitk_reduce_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      a.partial, plan.ksplit, n, static_cast<__nv_bfloat16*>(a.Y));
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& a, const GemmPlan& plan, const DevErr& err,
                        cudaStream_t stream) {
  cudaError_t e = launch_gemm_mainloop(a, plan, err, stream);
  if (e == cudaSuccess) e = launch_gemm_reduce(a, plan, stream);
  return e;
}

}  // namespace ttq
