"""Parity of the decoder-layer kernels and of the chained TTQ decoder stack (CUDA path,
through the C ABI) with the CPU oracle, on the same seeded inputs.

Bars:
  rmsnorm, qk_norm_rope, silu_mul   within one bf16 ulp of the oracle's fp64 value
      rounded to bf16 (the GPU computes in fp32 and rounds once, so it can land on the
      neighbouring bf16 value only when the exact result sits within fp32 error of a
      rounding boundary), plus an absolute floor of 2^-20 times the row's RMS for results
      that cancel to near zero in the rotation;
  v cache, untouched cache rows, the k/v part of the projection   bit-exact;
  TTQ linears in the stack   as in the single-layer tests: s within 1e-5, codes bit-exact
      given the GPU's s, Y within 5e-3 relative Frobenius of the oracle's fp64 product,
      and every output row within 3e-2 of the RMS row norm;
  prompt attention (the library's tensor-core kernel: bf16 probabilities, fp32 scores,
      softmax and accumulation)   8e-3 relative Frobenius against the oracle's fp64 softmax.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import online_activation_aware_b200 as ttq
from online_activation_aware_b200 import synthetic
from oracle import decoder_oracle as DO
from oracle import ttq_oracle as O

pytestmark = pytest.mark.gpu

S_RTOL = 1e-5
Y_RTOL = 5e-3
ATTN_RTOL = 8e-3
ROW_RTOL = 3e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ttq.load_library()
    yield
    assert ttq.device_status() == 0


def bf16(a):
    return synthetic.as_bf16(a).cuda()


def vals(t):
    return synthetic.bf16_values(t)


def ordinal(t):
    """bf16 bit patterns mapped to integers that step by one per representable value."""
    b = t.contiguous().view(torch.int16).cpu().numpy().astype(np.int64)
    return np.where(b < 0, -(b & 0x7FFF), b)


def assert_ulp(got, want64, floor=0.0):
    """got (bf16 tensor) within one bf16 ulp of RN_bf16(want64), or within `floor`."""
    want = synthetic.as_bf16(want64)
    du = np.abs(ordinal(got.cpu()) - ordinal(want))
    absd = np.abs(vals(got) - np.asarray(want64, dtype=np.float64))
    bad = (du > 1) & (absd > floor)
    assert not bad.any(), (int(bad.sum()), float(du.max()))
    assert np.mean(du != 0) < 0.02


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ------------------------------------------------------------------ kernels


@pytest.mark.parametrize("rows,n,res", [(77, 4096, True), (1, 256, False), (300, 1024, True), (5, 8192, True),
                                        (3, 8, False), (64, 2560, False), (9, 5120, True)])
def test_rmsnorm_parity(rows, n, res):
    rng = np.random.default_rng(rows * 7 + n)
    y = rng.normal(size=(rows, n)) * rng.lognormal(size=(rows, 1))
    w = 1 + 0.1 * rng.normal(size=n)
    r = rng.normal(size=(rows, n)) * 3 if res else None
    yb, wb = bf16(y), bf16(w)
    rb = bf16(r) if res else None
    r0 = vals(rb) if res else None
    out = ttq.rmsnorm(yb, wb, 1e-6, residual=rb)
    if res:
        assert_ulp(rb, r0 + vals(yb))      # the residual row now holds bf16(r + y)
    h = vals(rb) if res else vals(yb)
    assert_ulp(out, DO.rmsnorm(h, vals(wb)))


def test_rmsnorm_zero_row_and_constant_row():
    y = torch.zeros(2, 64, dtype=torch.bfloat16, device="cuda")
    y[1] = 2.0
    w = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    out = ttq.rmsnorm(y, w, 1e-6)
    assert torch.all(out[0] == 0)                 # 0 / sqrt(eps)
    assert torch.all(out[1] == 1.0)               # 2 / sqrt(4 + 1e-6) rounds to 1 in bf16


def test_rope_table_parity():
    for D, P in ((64, 33), (128, 4224), (256, 7)):
        tb = ttq.rope_table(P, D, 1.0e6).cpu().numpy().astype(np.float64)
        th = DO.rope_angles(np.arange(P), D, 1.0e6)
        np.testing.assert_allclose(tb[..., 0], np.cos(th), atol=2e-7)
        np.testing.assert_allclose(tb[..., 1], np.sin(th), atol=2e-7)


@pytest.mark.parametrize("T,H,Hkv,D,pos0", [(37, 8, 2, 128, 0), (1, 32, 8, 128, 4100), (20, 4, 4, 64, 3),
                                            (5, 6, 2, 256, 900), (64, 40, 8, 128, 0)])
def test_qk_norm_rope_parity(T, H, Hkv, D, pos0):
    rng = np.random.default_rng(T + H + D + pos0)
    qkv = rng.normal(size=(T, (H + 2 * Hkv) * D)) * rng.lognormal(size=(1, (H + 2 * Hkv) * D))
    wq, wk = 1 + 0.1 * rng.normal(size=D), 1 + 0.1 * rng.normal(size=D)
    qb, wqb, wkb = bf16(qkv), bf16(wq), bf16(wk)
    q_in = vals(qb)
    L = pos0 + T + 3
    table = ttq.rope_table(L, D, 1.0e6)
    kc = torch.full((L, Hkv, D), 7.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((L, Hkv, D), -5.0, dtype=torch.bfloat16, device="cuda")
    ttq.qk_norm_rope(qb, H, Hkv, D, wqb, wkb, 1e-6, table, pos0, kc, vc)
    # the oracle from the same bf16 inputs, before rounding (D1)
    x = q_in
    pos = pos0 + np.arange(T)
    q64 = DO.rope(DO.rmsnorm(x[:, : H * D].reshape(T, H, D), vals(wqb)), pos)
    k64 = DO.rope(DO.rmsnorm(x[:, H * D: (H + Hkv) * D].reshape(T, Hkv, D), vals(wkb)), pos)
    floor = 2.0 ** -20 * 2.0   # rows are RMS-normalised with weights near 1
    assert_ulp(qb[:, : H * D].reshape(T, H, D), q64, floor)
    assert_ulp(kc[pos0: pos0 + T], k64, floor)
    np.testing.assert_array_equal(vals(vc[pos0: pos0 + T]), q_in[:, (H + Hkv) * D:].reshape(T, Hkv, D))
    np.testing.assert_array_equal(vals(qb[:, H * D:]), q_in[:, H * D:])           # k|v part untouched
    for c, fill in ((kc, 7.0), (vc, -5.0)):
        assert torch.all(c[:pos0] == fill) and torch.all(c[pos0 + T:] == fill)
    # the same call with the position held on the device gives the same bits
    qb2 = bf16(qkv)
    kc2 = torch.full((L, Hkv, D), 7.0, dtype=torch.bfloat16, device="cuda")
    vc2 = torch.full((L, Hkv, D), -5.0, dtype=torch.bfloat16, device="cuda")
    pos_dev = torch.tensor([pos0], dtype=torch.int64, device="cuda")
    ttq.qk_norm_rope(qb2, H, Hkv, D, wqb, wkb, 1e-6, table, 0, kc2, vc2, pos0_dev=pos_dev)
    assert torch.equal(qb2, qb) and torch.equal(kc2, kc) and torch.equal(vc2, vc)


@pytest.mark.parametrize("rows,inter", [(50, 8), (33, 1024), (4, 12288), (1, 3072)])
def test_silu_mul_parity(rows, inter):
    rng = np.random.default_rng(rows + inter)
    gu = rng.normal(size=(rows, 2 * inter)) * 4
    gu[0, :8] = [0.0, -30.0, 30.0, -90.0, 90.0, 1e-3, -1e-3, 2.5]
    gb = bf16(gu)
    out = ttq.silu_mul(gb)
    assert_ulp(out, DO.silu_mul(vals(gb), inter), 1e-30)


# ------------------------------------------------------------------ the chained stack

SMALL = dict(layers=2, heads=8, kv_heads=2, hidden=512, head_dim=64, inter=1024)


def build_stack(shape, r, q, g, seed, max_len):
    from online_activation_aware_b200.decoder import TTQDecoder

    Wnp = synthetic.draw_decoder_weights(shape, r, seed)
    Wb = [{k: synthetic.as_bf16(v) for k, v in L.items()} for L in Wnp]
    Wv = [{k: vals(v) for k, v in L.items()} for L in Wb]
    fn = synthetic.as_bf16(1 + 0.1 * np.random.default_rng(seed + 1).normal(size=shape["hidden"]))
    dec = TTQDecoder(shape, [{k: v.cuda() for k, v in L.items()} for L in Wb], fn.cuda(), q, g, 0.5, 0.4, r=r,
                     max_len=max_len)
    return dec, Wv, vals(fn)


def check_ttq(lin, Xg, Yg, Wl, name, g, q, prefill, sample=None):
    """Y of one stacked TTQ linear against the oracle from the GPU's own input; with
    ``sample``, on that many seeded output rows (both ends included) instead of all."""
    X = vals(Xg)
    s_gpu = lin.s.cpu().numpy()
    if prefill:
        s64, _ = O.act_stats(X, 0.5, 0.4)
        assert np.max(np.abs(s_gpu - s64) / s64) <= S_RTOL
    W = Wl["w_" + name]
    rows = np.arange(W.shape[0])
    if sample is not None:
        rng = np.random.default_rng(W.shape[0] + len(name))
        rows = np.unique(np.concatenate([[0, W.shape[0] - 1], rng.choice(W.shape[0], sample, replace=False)]))
    oc, osc, oz = O.requant(W[rows], s_gpu, q, g)
    words = lin.codes.cpu().numpy().view(np.uint32).reshape(lin.d_out, -1)[rows]
    np.testing.assert_array_equal(words, O.pack_codes(oc, q))
    B = Wl.get("b_" + name)
    Yo = O.linear(X, s_gpu, oc, osc, oz, g, Wl.get("a_" + name), None if B is None else B[rows])
    Yg_ = vals(Yg)[:, rows]
    err = rel_fro(Yg_, Yo)
    assert err <= Y_RTOL, (name, err)
    # one wrong output row would hide under the Frobenius norm of thousands: bound each
    # row's error by a few times the bar, relative to the RMS row norm
    rms = np.linalg.norm(Yo) / np.sqrt(Yo.shape[1])
    row_err = np.linalg.norm(Yg_ - Yo, axis=0) / max(rms, 1e-300)
    assert row_err.max() <= ROW_RTOL, (name, float(row_err.max()))


def teacher_forced(shape, dec, Wv, fnv, x, T, steps, q, g, sample=None):
    """Runs the prefill and `steps` decode steps with every intermediate traced, and
    checks each step of each layer against the oracle fed the GPU's own input to it."""
    H, Hkv, D, I = shape["heads"], shape["kv_heads"], shape["head_dim"], shape["inter"]
    for step in range(steps + 1):
        rec = {}

        def trace(li, name, t):
            rec[(li, name)] = t.clone()

        prefill = step == 0
        if prefill:
            out = dec.prefill(x[:T].cuda(), trace=trace)
            pos0, n = 0, T
        else:
            out = dec.decode(x[T + step - 1: T + step].cuda(), trace=trace)
            pos0, n = T + step - 1, 1
        torch.cuda.synchronize()
        for li in range(shape["layers"]):
            Wl = Wv[li]
            lins = dec.layers[li]["lin"]
            g_ = lambda k: rec[(li, k)]
            assert_ulp(g_("h"), DO.rmsnorm(vals(g_("r_in")), Wl["n_in"]))
            check_ttq(lins["qkv"], g_("h"), g_("qkv"), Wl, "qkv", g, q, prefill, sample)
            qkv = vals(g_("qkv"))
            pos = pos0 + np.arange(n)
            q64 = DO.rope(DO.rmsnorm(qkv[:, : H * D].reshape(n, H, D), Wl["n_q"]), pos)
            k64 = DO.rope(DO.rmsnorm(qkv[:, H * D: (H + Hkv) * D].reshape(n, Hkv, D), Wl["n_k"]), pos)
            assert_ulp(g_("q").reshape(n, H, D), q64, 2.0 ** -19)
            assert_ulp(dec.k_cache[li, pos0: pos0 + n], k64, 2.0 ** -19)
            np.testing.assert_array_equal(vals(dec.v_cache[li, pos0: pos0 + n]),
                                          qkv[:, (H + Hkv) * D:].reshape(n, Hkv, D))
            K = vals(dec.k_cache[li, : pos0 + n])
            V = vals(dec.v_cache[li, : pos0 + n])
            a64 = DO.attention(vals(g_("q")).reshape(n, H, D), K, V, pos0)
            if prefill:
                assert rel_fro(vals(g_("attn")), a64) <= ATTN_RTOL
            else:   # the library's own decode attention: fp32 throughout
                assert_ulp(g_("attn"), a64, 2.0 ** -19)
            check_ttq(lins["o"], g_("attn"), g_("o"), Wl, "o", g, q, prefill, sample)
            assert_ulp(g_("r_mid"), vals(g_("r_in")) + vals(g_("o")))
            assert_ulp(g_("h2"), DO.rmsnorm(vals(g_("r_mid")), Wl["n_post"]))
            check_ttq(lins["gate_up"], g_("h2"), g_("gu"), Wl, "gate_up", g, q, prefill, sample)
            assert_ulp(g_("m"), DO.silu_mul(vals(g_("gu")), I), 1e-30)
            check_ttq(lins["down"], g_("m"), g_("down"), Wl, "down", g, q, prefill, sample)
            if li + 1 < shape["layers"]:
                # the next layer's residual is this one's plus its MLP output
                assert_ulp(rec[(li + 1, "r_in")], vals(g_("r_mid")) + vals(g_("down")))
        last = shape["layers"] - 1
        rf = DO.add_residual(vals(rec[(last, "r_mid")]), vals(rec[(last, "down")]))
        assert_ulp(out, DO.rmsnorm(rf, fnv))
    assert dec.length == T + steps


@pytest.mark.parametrize("r,q,g", [(0, 4, 64), (16, 2, 32)])
def test_stack_teacher_forced_parity(r, q, g):
    shape = SMALL
    T, steps = 96, 3
    dec, Wv, fnv = build_stack(shape, r, q, g, seed=40 + r, max_len=T + steps)
    x = synthetic.as_bf16(synthetic.draw_hidden(T + steps, shape["hidden"], seed=41))
    teacher_forced(shape, dec, Wv, fnv, x, T, steps, q, g)


def test_full_width_qwen3_8b_layer_teacher_forced():
    # one layer at the full Qwen3-8B width of the architecture table (hidden 4096, 32 query
    # and 8 key/value heads of 128, MLP 12288) with the stack's settings (q = 2, g = 32,
    # r = 16): a 256-token prompt and two decode steps; the TTQ linears are checked on 64
    # sampled output rows each, everything else in full
    shape = dict(synthetic.QWEN3_SHAPES["8B"], layers=1)
    T, steps, q, g, r = 256, 2, 2, 32, 16
    dec, Wv, fnv = build_stack(shape, r, q, g, seed=80, max_len=T + steps)
    x = synthetic.as_bf16(synthetic.draw_hidden(T + steps, shape["hidden"], seed=81))
    teacher_forced(shape, dec, Wv, fnv, x, T, steps, q, g, sample=64)


def test_stack_end_to_end_against_oracle_stack():
    # the whole stack, not teacher-forced: the oracle runs every layer from its own
    # results. Differences come from bf16 roundings landing on the other neighbour and
    # the rare code that sits on a rounding boundary; they stay small after two layers.
    shape = SMALL
    T, q, g, r = 64, 4, 64, 0
    dec, Wv, fnv = build_stack(shape, r, q, g, seed=50, max_len=T + 1)
    x = synthetic.as_bf16(synthetic.draw_hidden(T + 1, shape["hidden"], seed=51))
    outs = [dec.prefill(x[:T].cuda()).float().cpu().numpy(), dec.decode(x[T:].cuda()).float().cpu().numpy()]
    st = [DO.LayerState() for _ in range(shape["layers"])]
    for step, (xs, pos0, pre) in enumerate(((vals(x[:T]), 0, True), (vals(x[T:]), T, False))):
        rr, y = xs, None
        for li in range(shape["layers"]):
            o = DO.decoder_layer(rr, y, Wv[li], st[li], shape, pos0, q, g, 0.5, 0.4, pre)
            rr, y = o["r"], o["down"]
        ref = DO.final_norm(rr, y, fnv)
        # each chained step stays within its own bar (4 TTQ linears at 5e-3 and attention at
        # 8e-3 a layer); without teacher forcing their errors add, at most linearly:
        # 2 layers x 28e-3
        assert rel_fro(outs[step], ref) <= 5.6e-2, (step, rel_fro(outs[step], ref))


def test_decode_attention_parity_and_device_position():
    rng = np.random.default_rng(60)
    for H, Hkv, D, Lc, L in ((32, 8, 128, 4224, 4100), (8, 8, 64, 100, 1), (16, 2, 128, 700, 699), (4, 4, 64, 65, 64),
                             (64, 8, 128, 300, 257)):
        q = bf16(rng.normal(size=H * D))
        kc = bf16(rng.normal(size=(Lc, Hkv, D)))
        vc = bf16(rng.normal(size=(Lc, Hkv, D)))
        out = ttq.decode_attention(q, H, Hkv, D, kc, vc, length=L)
        a64 = DO.attention(vals(q).reshape(1, H, D), vals(kc[:L]), vals(vc[:L]), L - 1)
        assert_ulp(out, a64.reshape(-1), 2.0 ** -19)
        pos = torch.tensor([L - 1], dtype=torch.int64, device="cuda")
        out2 = ttq.decode_attention(q, H, Hkv, D, kc, vc, pos_dev=pos)
        assert torch.equal(out, out2)


def test_device_position_out_of_range_is_reported_not_written():
    H, Hkv, D, Lc = 4, 2, 64, 16
    table = ttq.rope_table(Lc, D, 1.0e6)
    qkv = bf16(np.ones((1, (H + 2 * Hkv) * D)))
    kc = torch.full((Lc, Hkv, D), 3.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((Lc, Hkv, D), 3.0, dtype=torch.bfloat16, device="cuda")
    w = bf16(np.ones(D))
    pos = torch.tensor([Lc], dtype=torch.int64, device="cuda")      # one past the cache
    ttq.qk_norm_rope(qkv, H, Hkv, D, w, w, 1e-6, table, 0, kc, vc, pos0_dev=pos)
    assert ttq.device_status() == -1
    assert torch.all(kc == 3.0) and torch.all(vc == 3.0)
    out = ttq.decode_attention(qkv, H, Hkv, D, kc, vc, pos_dev=pos)
    assert ttq.device_status() == -1
    assert torch.all(out == 0)
    pos.fill_(Lc - 1)                                                # the last row: in range
    ttq.qk_norm_rope(qkv, H, Hkv, D, w, w, 1e-6, table, 0, kc, vc, pos0_dev=pos)
    assert ttq.device_status() == 0
    assert torch.all(vc[Lc - 1] == 1.0) and torch.all(vc[: Lc - 1] == 3.0)


def test_captured_decode_step_equals_eager_steps():
    shape = SMALL
    T, steps = 40, 3
    x = synthetic.as_bf16(synthetic.draw_hidden(T + steps, shape["hidden"], seed=61)).cuda()
    dec, _, _ = build_stack(shape, 16, 2, 32, seed=62, max_len=T + steps)
    dec.prefill(x[:T])
    eager = [dec.decode(x[T + i: T + i + 1]).clone() for i in range(steps)]
    dec.prefill(x[:T])
    dec.capture_decode()
    graphed = [dec.decode(x[T + i: T + i + 1]).clone() for i in range(steps)]
    for a, b in zip(eager, graphed):
        assert torch.equal(a, b)
    assert int(dec.pos.item()) == T + steps


# ------------------------------------------------------------------ prompt attention (tensor cores)


def _attn_inputs(T, H, Hkv, D, seed, extra=0):
    rng = np.random.default_rng(seed)
    qkv = bf16(rng.normal(size=(T, (H + 2 * Hkv) * D)))
    kc = bf16(rng.normal(size=(T + extra, Hkv, D)))
    vc = bf16(rng.normal(size=(T + extra, Hkv, D)))
    return qkv, kc, vc


@pytest.mark.parametrize("T,H,Hkv,D", [(128, 8, 2, 128), (1, 8, 8, 128), (200, 4, 4, 128), (257, 16, 2, 128),
                                       (700, 32, 8, 128), (1000, 2, 1, 128), (96, 8, 2, 64), (300, 4, 2, 64)])
def test_prompt_attention_parity(T, H, Hkv, D):
    # every query row against the oracle's fp64 causal softmax attention; the probabilities
    # enter the second product in bf16, hence the attention bar; each row within 4x of it
    qkv, kc, vc = _attn_inputs(T, H, Hkv, D, seed=T + H)
    out = ttq.prompt_attention(qkv, H, Hkv, D, kc, vc)
    torch.cuda.synchronize()
    q = vals(qkv)[:, : H * D].reshape(T, H, D)
    a64 = DO.attention(q, vals(kc[:T]), vals(vc[:T]), 0)
    got = vals(out)
    assert np.isfinite(got).all()
    assert rel_fro(got, a64) <= ATTN_RTOL, rel_fro(got, a64)
    row = np.linalg.norm(got - a64, axis=1) / np.linalg.norm(a64, axis=1)
    assert row.max() <= 4 * ATTN_RTOL, float(row.max())


def test_prompt_attention_full_size_sampled_rows_and_cache_padding():
    # the Qwen3-8B shape (32 query heads, 8 key/value heads of 128) at a 4096-token prompt,
    # caches longer than the prompt (their later rows hold values that must not be read):
    # 64 sampled query rows, all heads, against the oracle; the same call twice gives the
    # same bits
    T, H, Hkv, D = 4096, 32, 8, 128
    qkv, kc, vc = _attn_inputs(T, H, Hkv, D, seed=11, extra=64)
    kc[T:] = 30.0
    vc[T:] = -30.0
    out = ttq.prompt_attention(qkv, H, Hkv, D, kc, vc)
    out2 = ttq.prompt_attention(qkv, H, Hkv, D, kc, vc)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    q = vals(qkv)[:, : H * D].reshape(T, H, D)
    K, V = vals(kc), vals(vc)
    rows = np.unique(np.concatenate([[0, 127, 128, T - 1], np.random.default_rng(12).choice(T, 60, replace=False)]))
    got = vals(out)
    for t in rows:
        a64 = DO.attention(q[t: t + 1], K[: t + 1], V[: t + 1], t)
        err = np.linalg.norm(got[t] - a64[0]) / np.linalg.norm(a64[0])
        assert err <= 4 * ATTN_RTOL, (int(t), float(err))
