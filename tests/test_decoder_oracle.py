"""Pins for the decoder-stack oracle: each test checks it against a closed form or an
invariant of the definition it restates, never against a retyped copy of its formula."""

import math

import numpy as np
import pytest

from oracle import decoder_oracle as DO
from oracle import ttq_oracle as O


# ------------------------------------------------------------------ RMSNorm


def test_rmsnorm_closed_forms():
    # mean square 4: every entry divided by 2
    np.testing.assert_allclose(DO.rmsnorm([2.0, -2.0, 2.0, -2.0], np.ones(4), eps=0.0), [1, -1, 1, -1], rtol=1e-15)
    # the weight multiplies per channel
    np.testing.assert_allclose(DO.rmsnorm([2.0, -2.0, 2.0, -2.0], [1, 2, 3, 4], eps=0.0), [1, -2, 3, -4],
                               rtol=1e-15)
    # eps enters under the root: mean square 1, eps 3 -> divide by 2
    np.testing.assert_allclose(DO.rmsnorm(np.ones(8), np.ones(8), eps=3.0), np.full(8, 0.5), rtol=1e-15)
    # (3, 4): mean square 12.5
    np.testing.assert_allclose(DO.rmsnorm([3.0, 4.0], [1.0, 1.0], eps=0.0), [3 / 12.5 ** 0.5, 4 / 12.5 ** 0.5],
                               rtol=1e-15)


def test_rmsnorm_invariants():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 96)) * rng.lognormal(size=(5, 1))
    y = DO.rmsnorm(x, np.ones(96), eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, rtol=1e-13)   # unit RMS rows
    np.testing.assert_allclose(DO.rmsnorm(7.5 * x, np.ones(96), eps=0.0), y, rtol=1e-13)  # scale invariant
    np.testing.assert_allclose(DO.rmsnorm(x[2:3], np.ones(96), eps=0.0), y[2:3], rtol=1e-15)  # per row


# ------------------------------------------------------------------ rotary embedding


def test_rope_rotation_sign_and_pairing():
    # D = 2: one pair at frequency 1, rotated counter-clockwise by the position
    np.testing.assert_allclose(DO.rope(np.array([[[1.0, 0.0]]]), [1])[0, 0], [math.cos(1), math.sin(1)], rtol=1e-15)
    np.testing.assert_allclose(DO.rope(np.array([[[0.0, 1.0]]]), [1])[0, 0], [-math.sin(1), math.cos(1)],
                               rtol=1e-15)
    # D = 4, base 100: channel 1 pairs with channel 3 at frequency 100^(-1/2) = 0.1
    e1 = np.array([[[0.0, 1.0, 0.0, 0.0]]])
    np.testing.assert_allclose(DO.rope(e1, [3], base=100.0)[0, 0], [0, math.cos(0.3), 0, math.sin(0.3)],
                               atol=1e-15)
    e0 = np.array([[[1.0, 0.0, 0.0, 0.0]]])
    np.testing.assert_allclose(DO.rope(e0, [3], base=100.0)[0, 0], [math.cos(3), 0, math.sin(3), 0], atol=1e-15)


def test_rope_invariants():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(6, 3, 64))
    np.testing.assert_array_equal(DO.rope(x, np.zeros(6)), x)                       # position 0: identity
    y = DO.rope(x, np.arange(6) * 1000 + 17)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # scores depend only on the position difference
    q, k = rng.normal(size=(1, 1, 64)), rng.normal(size=(1, 1, 64))
    s1 = np.sum(DO.rope(q, [40]) * DO.rope(k, [11]))
    s2 = np.sum(DO.rope(q, [1029]) * DO.rope(k, [1000]))
    np.testing.assert_allclose(s1, s2, rtol=1e-10)


def test_qk_norm_rope_split_order():
    # q section 1s, k section 2s, v section 3s: norms map q, k to 1s; position 0 leaves
    # them unrotated; v passes through
    H, Hkv, D = 4, 2, 8
    qkv = np.concatenate([np.ones((3, H * D)), np.full((3, Hkv * D), 2.0), np.full((3, Hkv * D), 3.0)], axis=1)
    q, k, v = DO.qk_norm_rope(qkv[:1], H, Hkv, D, np.ones(D), np.full(D, 0.5), 0, eps=0.0)
    np.testing.assert_array_equal(q, np.ones((1, H, D)))
    np.testing.assert_array_equal(k, np.full((1, Hkv, D), 0.5))
    np.testing.assert_array_equal(v, np.full((1, Hkv, D), 3.0))


# ------------------------------------------------------------------ SwiGLU


def test_silu_mul_pins():
    # sigmoid(ln 3) = 3/4, so silu(ln 3) * 2 = 1.5 ln 3; the up half multiplies
    np.testing.assert_allclose(DO.silu_mul([[math.log(3.0), 2.0]], 1), [[1.5 * math.log(3.0)]], rtol=1e-15)
    # swapping gate and up would give silu(2) ln 3 instead
    assert abs(DO.silu_mul([[2.0, math.log(3.0)]], 1)[0, 0] - 1.5 * math.log(3.0)) > 0.1
    # silu(x) - silu(-x) = x, and silu(0) = 0
    x = np.linspace(-30, 30, 61)
    gu = np.stack([x, np.ones_like(x)], axis=1)
    gun = np.stack([-x, np.ones_like(x)], axis=1)
    np.testing.assert_allclose(DO.silu_mul(gu, 1)[:, 0] - DO.silu_mul(gun, 1)[:, 0], x, atol=1e-13)
    assert DO.silu_mul([[0.0, 5.0]], 1)[0, 0] == 0.0


# ------------------------------------------------------------------ attention


def test_attention_single_key_and_uniform_keys():
    rng = np.random.default_rng(2)
    T, H, Hkv, D = 5, 4, 2, 8
    V = rng.normal(size=(T, Hkv, D))
    K = np.ones((T, Hkv, D))
    q = rng.normal(size=(T, H, D))
    # equal keys: query t averages v over positions 0..t (causal)
    out = DO.attention(q, K, V, 0).reshape(T, H, D)
    for t in range(T):
        for h in range(H):
            np.testing.assert_allclose(out[t, h], V[: t + 1, h // 2].mean(axis=0), rtol=1e-12, atol=1e-14)
    # one key: the output is its value
    out1 = DO.attention(q[:1], K[:1], V[:1], 0).reshape(1, H, D)
    np.testing.assert_allclose(out1[0, 3], V[0, 1], rtol=1e-15)


def test_attention_gqa_head_map_and_scale():
    H, Hkv, D = 4, 2, 4
    V = np.zeros((2, Hkv, D))
    V[:, 0] = 1.0            # key/value head 0 holds 1s, head 1 holds 2s
    V[:, 1] = 2.0
    K = np.zeros((2, Hkv, D))
    q = np.zeros((1, H, D))
    out = DO.attention(q, K, V, 1).reshape(1, H, D)
    np.testing.assert_allclose(out[0, :, 0], [1, 1, 2, 2], rtol=1e-15)   # heads 0,1 -> kv 0; 2,3 -> kv 1
    # score ln 3 after the 1/sqrt(D) scale: weights 3/4 and 1/4
    K[0, 0] = [1.0, 0, 0, 0]
    q[0, 0] = [2.0 * math.log(3.0), 0, 0, 0]
    V[0, 0], V[1, 0] = [4.0, 0, 0, 0], [8.0, 0, 0, 0]
    out = DO.attention(q, K, V, 1).reshape(1, H, D)
    np.testing.assert_allclose(out[0, 0, 0], 0.75 * 4 + 0.25 * 8, rtol=1e-14)


def test_attention_is_causal_and_decode_consistent():
    rng = np.random.default_rng(3)
    T, H, Hkv, D = 6, 2, 1, 16
    q, K, V = rng.normal(size=(T, H, D)), rng.normal(size=(T, Hkv, D)), rng.normal(size=(T, Hkv, D))
    a = DO.attention(q, K, V, 0)
    V2 = V.copy()
    V2[4:] += 10.0
    b = DO.attention(q, K, V2, 0)
    np.testing.assert_array_equal(a[:4], b[:4])          # later values do not reach earlier queries
    # a single query at position 5 over the 6 keys is the prefill's last row
    np.testing.assert_allclose(DO.attention(q[5:], K, V, 5), a[5:], rtol=1e-13)


# ------------------------------------------------------------------ stacked TTQ linears (reading D4)


def test_stacked_ttq_linear_equals_separate_linears():
    rng = np.random.default_rng(4)
    X = O.round_bf16(rng.standard_t(3, (40, 128)))
    Ws = [O.round_bf16(rng.normal(0, 0.02, (n, 128))) for n in (64, 32, 32)]
    st = O.prefill(X, np.concatenate(Ws), 4, 32, 0.5, 0.4)
    row = 0
    for W in Ws:
        one = O.prefill(X, W, 4, 32, 0.5, 0.4)
        n = W.shape[0]
        np.testing.assert_array_equal(st["codes"][row: row + n], one["codes"])
        np.testing.assert_array_equal(st["scale"][row: row + n], one["scale"])
        np.testing.assert_array_equal(st["Y"][:, row: row + n], one["Y"])
        row += n


def test_stacked_lowrank_term_equals_separate_terms():
    # stacked A = [A_1; A_2; A_3] and block-diagonal B give each part its own rank-r term
    rng = np.random.default_rng(7)
    r, d = 8, 128
    X = O.round_bf16(rng.standard_t(3, (24, d)))
    Ws = [O.round_bf16(rng.normal(0, 0.02, (n, d))) for n in (64, 32, 32)]
    As = [O.round_bf16(rng.normal(0, 0.02, (r, d))) for _ in Ws]
    Bs = [O.round_bf16(rng.normal(0, 0.02, (W.shape[0], r))) for W in Ws]
    Bst = np.zeros((128, 3 * r))
    row = 0
    for i, B in enumerate(Bs):
        Bst[row: row + B.shape[0], i * r: (i + 1) * r] = B
        row += B.shape[0]
    st = O.prefill(X, np.concatenate(Ws), 4, 32, 0.5, 0.4, A=np.concatenate(As), B=Bst)
    row = 0
    for W, A, B in zip(Ws, As, Bs):
        one = O.prefill(X, W, 4, 32, 0.5, 0.4, A=A, B=B)
        n = W.shape[0]
        np.testing.assert_array_equal(st["codes"][row: row + n], one["codes"])
        np.testing.assert_allclose(st["Y"][:, row: row + n], one["Y"], rtol=1e-12, atol=1e-12)
        row += n


# ------------------------------------------------------------------ the layer


def small_layer(rng, shape, hidden):
    H, Hkv, D, I = shape["heads"], shape["kv_heads"], shape["head_dim"], shape["inter"]
    def w(n, m):
        return O.round_bf16(rng.normal(0, m ** -0.5, (n, m)))
    return {"w_qkv": w((H + 2 * Hkv) * D, hidden), "w_o": w(hidden, H * D), "w_gate_up": w(2 * I, hidden),
            "w_down": w(hidden, I), "n_in": O.round_bf16(1 + 0.1 * rng.normal(size=hidden)),
            "n_post": O.round_bf16(1 + 0.1 * rng.normal(size=hidden)),
            "n_q": O.round_bf16(1 + 0.1 * rng.normal(size=D)), "n_k": O.round_bf16(1 + 0.1 * rng.normal(size=D))}


def test_layer_residual_wiring():
    # with the output projections zero, the residual stream passes through unchanged,
    # and the previous layer's output is added first
    rng = np.random.default_rng(5)
    shape = {"heads": 2, "kv_heads": 1, "head_dim": 32, "inter": 64}
    Wl = small_layer(rng, shape, 64)
    Wl["w_o"] = np.zeros_like(Wl["w_o"])
    Wl["w_down"] = np.zeros_like(Wl["w_down"])
    r = O.round_bf16(rng.normal(size=(7, 64)))
    y = O.round_bf16(rng.normal(size=(7, 64)))
    out = DO.decoder_layer(r, y, Wl, DO.LayerState(), shape, 0, 4, 32, 0.5, 0.4, True)
    np.testing.assert_array_equal(out["r"], O.round_bf16(r + y))
    np.testing.assert_array_equal(out["down"], np.zeros((7, 64)))


def test_layer_decode_reuses_prefill_codes_and_cache():
    rng = np.random.default_rng(6)
    shape = {"heads": 2, "kv_heads": 1, "head_dim": 32, "inter": 64}
    Wl = small_layer(rng, shape, 64)
    r = O.round_bf16(rng.normal(size=(9, 64)))
    st = DO.LayerState()
    DO.decoder_layer(r[:8], None, Wl, st, shape, 0, 4, 32, 0.5, 0.4, True)
    codes = st.ttq["qkv"]["codes"].copy()
    out = DO.decoder_layer(r[8:], None, Wl, st, shape, 8, 4, 32, 0.5, 0.4, False)
    np.testing.assert_array_equal(st.ttq["qkv"]["codes"], codes)
    assert st.K.shape[0] == 9 and st.V.shape[0] == 9
    # the decode token's q/k/v are those of the same token pushed through the stored
    # statistic and codes at position 8
    qkv = O.round_bf16(O.linear(out["h"], st.ttq["qkv"]["s32"], codes, st.ttq["qkv"]["scale"],
                                st.ttq["qkv"]["zero"], 32))
    np.testing.assert_array_equal(out["qkv"], qkv)
    _, kh, _ = DO.qk_norm_rope(qkv, 2, 1, 32, Wl["n_q"], Wl["n_k"], 8)
    np.testing.assert_array_equal(st.K[8:], kh)


# ------------------------------------------------------------------ the synthetic stack (host logic)


def test_decoder_weights_layout_follows_the_architecture_table():
    from online_activation_aware_b200 import synthetic

    sh = synthetic.QWEN3_SHAPES["8B"]          # Table 15: 36 layers, 32 / 8 heads, 4096, 128, 12288
    assert (sh["layers"], sh["heads"], sh["kv_heads"], sh["hidden"], sh["head_dim"], sh["inter"]) == \
        (36, 32, 8, 4096, 128, 12288)
    assert synthetic.decoder_linear_parts(sh, "qkv") == ([4096, 1024, 1024], 4096)
    assert synthetic.decoder_linear_parts(sh, "o") == ([4096], 4096)
    assert synthetic.decoder_linear_parts(sh, "gate_up") == ([12288, 12288], 4096)
    assert synthetic.decoder_linear_parts(sh, "down") == ([4096], 12288)
    small = dict(layers=1, heads=4, kv_heads=2, hidden=128, head_dim=32, inter=96)
    L = synthetic.draw_decoder_weights(small, 8, seed=3)[0]
    assert L["w_qkv"].shape == (4 * 32 + 2 * 2 * 32, 128) and L["a_qkv"].shape == (24, 128)
    b = L["b_qkv"]
    assert b.shape == (256, 24)
    # block diagonal: part i's rows use only columns i r .. (i + 1) r
    for i, (r0, r1) in enumerate(((0, 128), (128, 192), (192, 256))):
        blk = np.zeros_like(b[r0:r1], dtype=bool)
        blk[:, i * 8:(i + 1) * 8] = True
        assert np.all(b[r0:r1][~blk] == 0) and np.all(b[r0:r1][blk] != 0)
    assert L["b_gate_up"].shape == (192, 16) and L["a_down"].shape == (8, 96)
    # the same seed draws the same numbers
    L2 = synthetic.draw_decoder_weights(small, 8, seed=3)[0]
    assert all(np.array_equal(L[k], L2[k]) for k in L)
