"""Plain CPU oracle for a stack of decoder layers whose linears run under TTQ.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path never imports it, and this module imports nothing from the product.

The layer shapes are those of the Qwen3 dense models in Table 15 of the
thelatestinai.com listing of "TTQ: Activation-Aware Test-Time Quantization ..." (layers,
heads, KV heads, hidden size, head dim, MLP dim). The pages describe the models only by
that table; the layer's structure is the published Qwen3 decoder (Yang et al. 2025), and
every step below is the textbook definition of its part, cited to the paper that defines it:

  RMSNorm        y = x / sqrt(mean(x^2) + eps) * w                (Zhang & Sennrich 2019)
  rotary PE      pairs (i, i + D/2) of each head rotated by the angle
                 pos * base^(-2i/D), i < D/2                      (Su et al. 2021, RoFormer;
                                                                   the half-split pairing)
  attention      softmax(q k^T / sqrt(D)) v, causal, query head h reading key/value
                 head h // (H / H_kv)                             (Vaswani et al. 2017;
                                                                   Ainslie et al. 2023, GQA)
  SwiGLU MLP     down( silu(gate x) * (up x) ), silu(u) = u / (1 + e^-u)   (Shazeer 2020)

The layer (pre-norm residual form):
  h  = RMSNorm_in(r)
  q, k, v = split(TTQ-linear(h; [Wq; Wk; Wv]))
  q, k = RoPE(RMSNorm_q(q)), RoPE(RMSNorm_k(k))      per head
  r  = r + TTQ-linear(attention(q, K, V); Wo)
  r  = r + TTQ-linear(SwiGLU(TTQ-linear(RMSNorm_post(r); [Wgate; Wup])); Wdown)
and the stack ends with a final RMSNorm.

Readings (decisions where the pages are silent; listed with reasons in the design notes):
  D1  each stored intermediate is computed in fp64 and rounded to bf16 once, where the
      GPU stores it (the GPU computes it in fp32 and rounds once);
  D2  RMSNorm eps = 1e-6, rotary base = 1e6 (the published Qwen3 configuration);
  D3  the residual stream is kept in bf16: r <- bf16(r + y);
  D4  q, k and v share one statistic (they read the same h), so they are one TTQ linear
      over the stacked weight [Wq; Wk; Wv]; gate and up likewise. This is exact: the
      statistic depends only on the layer input and the re-quantization is per output row.
      With static low-rank factors, the stacked linear takes A = [A_q; A_k; A_v] and the
      block-diagonal B = diag(B_q, B_k, B_v), whose term (X A^T) B^T gives every part its
      own rank-r term.
"""

from __future__ import annotations

import numpy as np

from oracle import ttq_oracle as O

EPS = 1e-6
ROPE_BASE = 1.0e6


def rmsnorm(x, w, eps: float = EPS) -> np.ndarray:
    """y = x / sqrt(mean_j x_j^2 + eps) * w over the last axis, fp64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def rope_angles(positions, D: int, base: float = ROPE_BASE) -> np.ndarray:
    """theta[p, i] = p * base^(-2i/D) for i < D/2 (RoFormer's frequencies), fp64."""
    i = np.arange(D // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * i / D)
    return np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x, positions, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate each pair (x_i, x_{i+D/2}) of every head by theta[pos, i]:
    (a, b) -> (a cos - b sin, b cos + a sin).  x [T, H, D], positions [T]."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    th = rope_angles(positions, D, base)[:, None, :]
    c, s = np.cos(th), np.sin(th)
    a, b = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def qk_norm_rope(qkv, heads: int, kv_heads: int, D: int, wq, wk, pos0: int,
                 eps: float = EPS, base: float = ROPE_BASE):
    """Split the stacked projection [T, (H + 2 H_kv) D] into q, k, v; per-head RMSNorm of
    q and k, then rotary embedding at positions pos0 .. pos0 + T - 1.
    Returns (q [T, H, D], k [T, H_kv, D], v [T, H_kv, D]) rounded to bf16 (D1)."""
    qkv = np.asarray(qkv, dtype=np.float64)
    T = qkv.shape[0]
    q = qkv[:, : heads * D].reshape(T, heads, D)
    k = qkv[:, heads * D: (heads + kv_heads) * D].reshape(T, kv_heads, D)
    v = qkv[:, (heads + kv_heads) * D:].reshape(T, kv_heads, D)
    pos = pos0 + np.arange(T)
    q = rope(rmsnorm(q, wq, eps), pos, base)
    k = rope(rmsnorm(k, wk, eps), pos, base)
    return O.round_bf16(q), O.round_bf16(k), O.round_bf16(v)


def attention(q, K, V, pos0: int) -> np.ndarray:
    """Causal grouped-query attention. q [T, H, D] at positions pos0 .. pos0 + T - 1,
    K, V [L, H_kv, D] for positions 0 .. L - 1 (L >= pos0 + T). Query t sees keys
    0 .. pos0 + t. Returns [T, H * D] in fp64."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, H, D = q.shape
    Hkv = K.shape[1]
    group = H // Hkv
    out = np.zeros((T, H, D))
    for h in range(H):
        kh = h // group
        S = q[:, h, :] @ K[:, kh, :].T / np.sqrt(D)          # [T, L]
        for t in range(T):
            n = pos0 + t + 1
            e = np.exp(S[t, :n] - S[t, :n].max())
            out[t, h] = (e / e.sum()) @ V[:n, kh, :]
    return out.reshape(T, H * D)


def silu_mul(gu, inter: int) -> np.ndarray:
    """SwiGLU's gate: silu(g) * u with g = gu[:, :I] and u = gu[:, I:], fp64."""
    gu = np.asarray(gu, dtype=np.float64)
    g, u = gu[:, :inter], gu[:, inter:]
    return g / (1.0 + np.exp(-g)) * u


def add_residual(r, y) -> np.ndarray:
    """r <- bf16(r + y) (D3)."""
    return O.round_bf16(np.asarray(r, dtype=np.float64) + np.asarray(y, dtype=np.float64))


class LayerState:
    """One layer's per-prompt TTQ results (statistic and codes of its four linears) and
    its key/value cache."""

    def __init__(self):
        self.ttq = {}
        self.K = None
        self.V = None


def ttq_linear(name, X, Wl, st: LayerState, q: int, g: int, alpha: float, lam: float, prefill: bool):
    """A TTQ linear: at prefill, statistic + requant of W (the residual R when the static
    low-rank factors a_<name>, b_<name> are present) from this X; at decode, the stored
    statistic and codes (the prefill's)."""
    A, B = Wl.get("a_" + name), Wl.get("b_" + name)
    if prefill:
        res = O.prefill(X, Wl["w_" + name], q, g, alpha, lam, A=A, B=B)
        st.ttq[name] = res
        return res["Y"]
    res = st.ttq[name]
    return O.linear(X, res["s32"], res["codes"], res["scale"], res["zero"], g, A, B)


def decoder_layer(r, y_prev, Wl, st: LayerState, shape, pos0: int, q: int, g: int, alpha: float,
                  lam: float, prefill: bool):
    """One layer over T tokens at positions pos0 .. pos0 + T - 1.

    r is the bf16 residual stream entering the layer, y_prev the previous layer's MLP
    output still to be added (None for the first layer). Wl holds the bf16 weights
    (w_qkv, w_o, w_gate_up, w_down, n_in, n_post, n_q, n_k, and a_*, b_* when the linears
    carry low-rank factors). Returns a dict of every
    intermediate, rounded to bf16 where the GPU stores it; ``r`` and ``down`` are what
    the next layer takes."""
    H, Hkv, D, I = shape["heads"], shape["kv_heads"], shape["head_dim"], shape["inter"]
    out = {}
    if y_prev is not None:
        r = add_residual(r, y_prev)
    out["r_in"] = r
    out["h"] = O.round_bf16(rmsnorm(r, Wl["n_in"]))
    out["qkv"] = O.round_bf16(ttq_linear("qkv", out["h"], Wl, st, q, g, alpha, lam, prefill))
    qh, kh, vh = qk_norm_rope(out["qkv"], H, Hkv, D, Wl["n_q"], Wl["n_k"], pos0)
    st.K = kh if st.K is None else np.concatenate([st.K[:pos0], kh])
    st.V = vh if st.V is None else np.concatenate([st.V[:pos0], vh])
    out["q"], out["k"], out["v"] = qh, kh, vh
    out["attn"] = O.round_bf16(attention(qh, st.K, st.V, pos0))
    out["o"] = O.round_bf16(ttq_linear("o", out["attn"], Wl, st, q, g, alpha, lam, prefill))
    r = add_residual(r, out["o"])
    out["r_mid"] = r
    out["h2"] = O.round_bf16(rmsnorm(r, Wl["n_post"]))
    out["gu"] = O.round_bf16(ttq_linear("gate_up", out["h2"], Wl, st, q, g, alpha, lam, prefill))
    out["m"] = O.round_bf16(silu_mul(out["gu"], I))
    out["down"] = O.round_bf16(ttq_linear("down", out["m"], Wl, st, q, g, alpha, lam, prefill))
    out["r"] = r
    return out


def final_norm(r, y_last, w) -> np.ndarray:
    """The stack's output: RMSNorm of the residual after the last layer's MLP output."""
    return O.round_bf16(rmsnorm(add_residual(r, y_last), w))
