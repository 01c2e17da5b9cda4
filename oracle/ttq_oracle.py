"""Plain CPU oracle for TTQ, the activation-aware test-time quantization of a linear layer.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path (the CUDA library and its Python binding) never imports it, and this
module imports nothing from the product: the two share no code.

Every function restates one step of the method in the order and notation of the
pages, with numpy as the only library (``matmul`` and ``svd`` serve as steps). Floating
point work is fp64 where the method is mathematics (statistics, dequantised weights,
products) and pinned IEEE fp32 (numpy float32 ops, each rounded to nearest even) where
the product must match bit for bit (the quantizer).

Sources, cited below by the short tag in brackets:
  [DR]  "深度解读：TTQ: Activation-Aware Test-Time Quantization to Accelerate LLM
        Inference On The Fly" (paper-daily.com deep reading); §2 方法详解 (method),
        §5 局限 (limits), §6 工业实践 (deployment).
  [NR]  "[論文レビュー] TTQ: Activation-Aware Test-Time Quantization ..." (nubint.ai
        review); section 提案手法 (proposed method).
  [GDE] "TTQ: Activation-Aware Test-Time Quantization ..." (gist.science, German
        technical summary); §2 Methodik.
  [GFR] gist.science French technical summary of the same paper; §2A "Quantisation
        Consciente des Activations en Ligne", §2B "Décomposition en Rang Faible".
  [TL]  "TTQ: Activation-Aware Test-Time Quantization ..." (thelatestinai.com listing);
        abstract and Tables 1-18.

Readings taken where the pages are silent or disagree (each is a decision, listed
with its reason in the design notes):
  R1  the statistic is the per-channel MEAN of squares over the prompt's T tokens,
      s_j = (mean_t x_tj^2 + lambda)^(alpha/2) = D_jj^(1/2)  ([DR §2] writes
      diag[XX^T + lambda I]^alpha without 1/T; [GDE §2]/[GFR §2A] write an unsquared
      p-norm).  General p: s_j = (mean_t |x_tj|^p + lambda)^(alpha/p).
  R2  groups are g consecutive INPUT channels of one output row.
  R3  the quantizer is asymmetric min/max with an integer zero point:
        sigma = smallest fp16 >= fl32(range / (2^q - 1))   (round toward +inf),
        z     = rint(fl32(-min / sigma)), clamped to [-2048, 2048] (exact in fp16),
        c     = clamp(rint(fl32(v / sigma)) + z, 0, 2^q - 1),
      rint halves to even; range == 0 is replaced by |min| (or 1 when min == 0).
      sigma is kept within [2^-24, 65504] (the finite positive fp16 range).
  R4  low rank: B = U_r Sigma_r^(1/2), A = Sigma_r^(1/2) V_r^T from the fp64 SVD of W,
      both rounded to bf16; the quantised residual is R = bf16(W - B A).
  R5  decode tokens are folded by the prefill's s and reuse its codes.

Parity of this oracle with the authors' own (unpublished) implementation is
unpinned: their packing, quantizer tie rules and kernels are not on the pages.
"""

from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------------------
# Number formats used by the path (plain definitions, written from the IEEE formats)
# --------------------------------------------------------------------------------------


def round_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 value (8 significant bits), ties to even.

    Written from the format's definition: x = m * 2^e with m in [0.5, 1) (frexp), the
    bf16 value is rint(m * 2^8) * 2^(e-8). Returns float64 values that are exactly
    representable in bf16. Normal range only (the path never produces bf16 subnormals
    from its inputs).
    """
    a = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(a)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


FP16_MAX = 65504.0
FP16_MIN_SUBNORMAL = 2.0 ** -24


def round_fp16_up(x) -> np.ndarray:
    """Smallest IEEE binary16 value >= x, for x > 0, saturated to [2^-24, 65504] (R3).

    binary16 has 11 significant bits for |x| >= 2^-14 and a fixed quantum of 2^-24
    below that. Computed exactly in fp64 (inputs are fp32 values).
    """
    a = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(a)
    normal = np.ldexp(np.ceil(np.ldexp(m, 11)), e - 11)
    sub = np.ceil(a * 2.0 ** 24) * 2.0 ** -24
    out = np.where(a >= 2.0 ** -14, normal, sub)
    return np.clip(out, FP16_MIN_SUBNORMAL, FP16_MAX)


# --------------------------------------------------------------------------------------
# Step 1: online activation statistics  ([DR §2] D = diag[XX^T + lambda I]^alpha,
#         [GDE §2] / [GFR §2A] D_ii = (||X_i,:||_p + lambda)^alpha, reading R1)
# --------------------------------------------------------------------------------------


def act_stats(X, alpha: float, lam: float, p: int = 2):
    """Per-input-channel scale of one prompt.

    X is [T, d] (tokens by channels). Returns (s64, s32): s_j = (mean_t |x_tj|^p +
    lambda)^(alpha/p) in fp64, and the same value rounded to fp32 (the scale vector the
    quantizer and the fold use). At p = 2 this is D_jj^(1/2) with the mean reading R1.
    """
    X = np.asarray(X, dtype=np.float64)
    T = X.shape[0]
    m = np.sum(np.abs(X) ** p, axis=0) / T
    s64 = (m + lam) ** (alpha / p)
    return s64, s64.astype(np.float32)


# --------------------------------------------------------------------------------------
# Step 2: low-rank split, host set-up ([DR §2] W_hat = W_q + BA, SVD-initialised, r=16;
#         [GDE §2] B, A static, W_q the dynamically quantised residual; reading R4)
# --------------------------------------------------------------------------------------


def lowrank_split(W, r: int):
    """Returns (B [d',r], A [r,d], R [d',d]) as bf16-exact float64 arrays."""
    W = np.asarray(W, dtype=np.float64)
    U, S, Vt = np.linalg.svd(W, full_matrices=False)
    root = np.sqrt(S[:r])
    B = round_bf16(U[:, :r] * root[None, :])
    A = round_bf16(root[:, None] * Vt[:r, :])
    R = round_bf16(W - B @ A)
    return B, A, R


# --------------------------------------------------------------------------------------
# Step 3: scale - quantize of W diag(s)  ([DR §2] W_hat = Q[W D^(1/2)] D^(-1/2);
#         [NR 提案手法] group-wise RTN quantize-dequantize; reading R3)
# --------------------------------------------------------------------------------------


def requant(W, s32, q: int, g: int):
    """Quantize W diag(s) group by group.

    W: [d', d] bf16-exact values; s32: fp32 [d]. Returns (codes int64 [d', d],
    scale float16 [d', d/g], zero float16 [d', d/g]). v = fl32(w * s) is formed first,
    then each group of g consecutive input channels of a row is quantized on its own
    (reading R3). Every fp32 operation below is one numpy float32 operation, so each
    result is the IEEE round-to-nearest-even value; the work is written array-wise
    over all groups at once, with the same steps as for a single group.
    """
    f32 = np.float32
    W = np.asarray(W, dtype=f32)
    s32 = np.asarray(s32, dtype=f32)
    d_out, d = W.shape
    assert d % g == 0
    Nq = f32(2 ** q - 1)
    V = (W * s32[None, :]).reshape(d_out, d // g, g)        # v = fl32(w * s)
    mn = V.min(axis=2)
    mx = V.max(axis=2)
    rng = (mx - mn).astype(f32)                              # fl32(max - min)
    rng = np.where(rng == 0, np.where(mn != 0, np.abs(mn), f32(1.0)), rng).astype(f32)
    sigma32 = (rng / Nq).astype(f32)                         # fl32(range / N_q)
    sigma = round_fp16_up(sigma32).astype(f32)               # fp16, toward +inf
    z = np.rint((-mn) / sigma).astype(f32)                   # rint(fl32(-min / sigma))
    z = np.clip(z, f32(-2048.0), f32(2048.0)).astype(f32)
    c = np.rint(V / sigma[:, :, None]).astype(f32) + z[:, :, None]
    c = np.clip(c, f32(0.0), Nq)
    codes = c.astype(np.int64).reshape(d_out, d)
    return codes, sigma.astype(np.float16), z.astype(np.float16)


def quantize_group(v, q: int):
    """Quantize one group of fp32 values (already scaled by s): (codes, sigma, z)."""
    v = np.asarray(v, dtype=np.float32).reshape(1, -1)
    c, sg, z = requant(v, np.ones(v.shape[1], dtype=np.float32), q, v.shape[1])
    return c[0], float(sg[0, 0]), float(z[0, 0])


# --------------------------------------------------------------------------------------
# Packed code layout (this library's storage format, defined here from the format
# description: exactly q/8 bytes per weight, grouped along the input channels)
# --------------------------------------------------------------------------------------


def pack_codes(codes, q: int) -> np.ndarray:
    """Pack int codes [d', d] into uint32 words [d', d*q/32].

    q in {2, 4}: 32/q codes per word, code k of the word at bits [q*k, q*k + q).
    q = 3: every 32 consecutive codes take 3 words; word b holds bit b of each code,
    code k at bit k.
    """
    c = np.asarray(codes, dtype=np.uint64)
    d_out, d = c.shape
    assert d % 32 == 0
    if q in (2, 4):
        per = 32 // q
        c = c.reshape(d_out, d // per, per)
        words = np.zeros((d_out, d // per), dtype=np.uint64)
        for k in range(per):
            words |= c[:, :, k] << np.uint64(q * k)
        return words.astype(np.uint32)
    if q == 3:
        c = c.reshape(d_out, d // 32, 32)
        words = np.zeros((d_out, d // 32, 3), dtype=np.uint64)
        for b in range(3):
            for k in range(32):
                words[:, :, b] |= ((c[:, :, k] >> np.uint64(b)) & np.uint64(1)) << np.uint64(k)
        return words.reshape(d_out, d // 32 * 3).astype(np.uint32)
    raise ValueError("q must be 2, 3 or 4")


def unpack_codes(words, q: int, d: int) -> np.ndarray:
    """Inverse of pack_codes."""
    w = np.asarray(words, dtype=np.uint64)
    d_out = w.shape[0]
    if q in (2, 4):
        per = 32 // q
        out = np.zeros((d_out, d // per, per), dtype=np.int64)
        for k in range(per):
            out[:, :, k] = ((w >> np.uint64(q * k)) & np.uint64(2 ** q - 1)).astype(np.int64)
        return out.reshape(d_out, d)
    if q == 3:
        w = w.reshape(d_out, d // 32, 3)
        out = np.zeros((d_out, d // 32, 32), dtype=np.int64)
        for b in range(3):
            for k in range(32):
                out[:, :, k] |= (((w[:, :, b] >> np.uint64(k)) & np.uint64(1)) << np.uint64(b)).astype(np.int64)
        return out.reshape(d_out, d)
    raise ValueError("q must be 2, 3 or 4")


# --------------------------------------------------------------------------------------
# Step 4: dequantised weight ([DR §2] the D^(-1/2) on the right of Q[W D^(1/2)])
# --------------------------------------------------------------------------------------


def dequant_scaled(codes, scale, zero, g: int) -> np.ndarray:
    """w'_ik = (c_ik - z_ig) * sigma_ig in fp64: the quantised weight in the scaled
    domain (W diag(s))."""
    c = np.asarray(codes, dtype=np.float64)
    sg = np.repeat(np.asarray(scale, dtype=np.float64), g, axis=1)
    zz = np.repeat(np.asarray(zero, dtype=np.float64), g, axis=1)
    return (c - zz) * sg


def dequant_original(codes, scale, zero, g: int, s) -> np.ndarray:
    """W_hat = Q[W D^(1/2)] D^(-1/2): the scaled-domain weight divided by s per input
    channel."""
    return dequant_scaled(codes, scale, zero, g) / np.asarray(s, dtype=np.float64)[None, :]


# --------------------------------------------------------------------------------------
# Step 5: the projection ([DR §2]; fold of D^(-1/2) into X; low-rank term [GFR §2B])
# --------------------------------------------------------------------------------------


def fold(X, s) -> np.ndarray:
    """The folded activations X' = RN_bf16(x_tj / s_j) the projection multiplies: the
    D^(-1/2) of W_hat = Q[W D^(1/2)] D^(-1/2) applied to the activations instead of the
    weight ([DR §2]; [DR §5] names a kernel that fuses this pre-scaling), stored in bf16.

    X [T, d] holds bf16 values, s fp32 values. The quotient is formed in fp64 and rounded
    once to bf16. That equals rounding the exact quotient: for a bf16 midpoint m, x - m s
    is zero or at least 2^-33 |m s| (x has 8 significant bits, m 9 and s 24), far above
    the 2^-53 relative error of the fp64 division, so that division never moves a
    quotient onto or across a midpoint.
    """
    X = np.asarray(X, dtype=np.float64)
    return round_bf16(X / np.asarray(s, dtype=np.float64)[None, :])



def linear(X, s, codes, scale, zero, g: int, A=None, B=None) -> np.ndarray:
    """Y = (X diag(1/s)) w'^T  (+ (X A^T) B^T when low-rank factors are given), fp64.

    X [T, d] tokens by channels; returns Y [T, d']. The same formula serves the decode
    steps, with the prefill's s and codes (reading R5).
    """
    X = np.asarray(X, dtype=np.float64)
    Xf = X / np.asarray(s, dtype=np.float64)[None, :]
    Y = Xf @ dequant_scaled(codes, scale, zero, g).T
    if A is not None:
        Y = Y + (X @ np.asarray(A, dtype=np.float64).T) @ np.asarray(B, dtype=np.float64).T
    return Y


def prefill(X, W, q: int, g: int, alpha: float, lam: float, p: int = 2, A=None, B=None):
    """One prompt through a TTQ linear layer: statistics, requant of W (or of the
    residual R when A, B are given), projection. Returns a dict of every result."""
    s64, s32 = act_stats(X, alpha, lam, p)
    codes, scale, zero = requant(W, s32, q, g)
    Y = linear(X, s32, codes, scale, zero, g, A, B)
    return {"s64": s64, "s32": s32, "codes": codes, "scale": scale, "zero": zero, "Y": Y}


# --------------------------------------------------------------------------------------
# Step 6: overhead model ([GFR §2A] extra cost O(dT + 3d'd) against O(d'dT))
# --------------------------------------------------------------------------------------


def overhead_counts(T: int, d: int, d_out: int):
    """Operation counts of the statistics, the requant and the projection, and their
    ratio rho = (dT + 3d'd) / (d'dT) = 1/d' + 3/T."""
    ops_stats = d * T
    ops_requant = 3 * d_out * d
    ops_gemm = d_out * d * T
    return {"stats": ops_stats, "requant": ops_requant, "gemm": ops_gemm,
            "rho": (ops_stats + ops_requant) / ops_gemm}


def activation_loss(W, W_hat, X) -> float:
    """L = ||(W - W_hat) X^T||_F^2 for W, W_hat [d', d] and X [T, d] ([DR §2] the
    activation-weighted loss that AWQ-style scaling targets; the pages write it with X as
    [d, T], channels by tokens, which is the transpose of the layout here). The sum runs
    over every output channel and token (no mean over T)."""
    E = np.asarray(W, dtype=np.float64) - np.asarray(W_hat, dtype=np.float64)
    return float(np.sum((np.asarray(X, dtype=np.float64) @ E.T) ** 2))
