"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by element
on the same seeded inputs.

Bars (from the method's arithmetic):
  s                 relative error <= 1e-5 against the oracle's fp64 statistic;
  codes/scale/zero  bit-exact when both sides get the same fp32 s;
  Y                 relative Frobenius error <= 5e-3 against the oracle's fp64 product
                    with the oracle's own codes (bf16 X diag(1/s), bf16 dequantised
                    weight and bf16 Y each add about 2^-9 relative rounding).
"""

import json
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import online_activation_aware_b200 as ttq
from online_activation_aware_b200 import synthetic
from oracle import ttq_oracle as O

pytestmark = pytest.mark.gpu

S_RTOL = 1e-5
Y_RTOL = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ttq.load_library()
    yield
    assert ttq.device_status() == 0
    path = os.environ.get("TTQ_PARITY_REPORT")
    if path and _REPORT:
        with open(path, "w") as f:
            json.dump({"cases": len(_REPORT), "max_rel_fro": max(e for _, e, _ in _REPORT),
                       "max_row_err": max(r for _, _, r in _REPORT),
                       "rows": [[str(t), e, r] for t, e, r in _REPORT]}, f, indent=1)


def layer(T, d, d_out, seed):
    X, W = synthetic.draw_layer(T, d, d_out, seed)
    Xb, Wb = synthetic.as_bf16(X), synthetic.as_bf16(W)
    return Xb, Wb, synthetic.bf16_values(Xb), synthetic.bf16_values(Wb)


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


ROW_RTOL = 3e-2
_REPORT = []


def check_y(Yg, Yo, tag=None):
    """Y against the oracle: relative Frobenius error <= Y_RTOL over the whole output,
    and every output channel (column of Y over the tokens) within ROW_RTOL of the RMS
    channel norm, so that one wrong row cannot hide under the norm of thousands. Both
    figures are recorded (written to $TTQ_PARITY_REPORT at the end of the session)."""
    Yg = np.asarray(Yg, dtype=np.float64).reshape(-1, np.shape(Yo)[-1])
    Yo = np.asarray(Yo, dtype=np.float64).reshape(-1, np.shape(Yo)[-1])
    err = rel_fro(Yg, Yo)
    rms = np.linalg.norm(Yo) / np.sqrt(Yo.shape[1])
    row = float((np.linalg.norm(Yg - Yo, axis=0) / max(rms, 1e-300)).max())
    _REPORT.append((tag, err, row))
    assert err <= Y_RTOL, (tag, err)
    assert row <= ROW_RTOL, (tag, row)
    return err, row


def gpu(t):
    return t.cuda()


def packed_np(codes_t, q, d_out, d):
    return codes_t.cpu().numpy().view(np.uint32).reshape(d_out, d * q // 32)


# ------------------------------------------------------------------ statistics


@pytest.mark.parametrize("T,d,alpha,p", [
    (128, 512, 0.5, 2), (37, 264, 0.75, 2), (1, 64, 0.5, 2), (2048, 768, 0.5, 2),
    (4096, 2048, 0.75, 2), (500, 320, 0.5, 1), (16384, 5120, 0.5, 2), (33, 72, 0.0, 2),
])
def test_act_stats_parity(T, d, alpha, p):
    Xb, _, X, _ = layer(T, d, 8, seed=T + d)
    s = ttq.act_stats(gpu(Xb), alpha, 0.4, p).cpu().numpy().astype(np.float64)
    s64, _ = O.act_stats(X, alpha, 0.4, p)
    err = np.max(np.abs(s - s64) / s64)
    assert err <= S_RTOL, err


def test_act_stats_deterministic_and_strided():
    Xb, _, X, _ = layer(3000, 1024, 8, seed=9)
    Xg = gpu(Xb)
    a = ttq.act_stats(Xg, 0.5, 0.4)
    b = ttq.act_stats(Xg, 0.5, 0.4)
    assert torch.equal(a, b)
    # a strided view (ld_x > d): only the first d columns count
    wide = torch.zeros(3000, 1040, dtype=torch.bfloat16, device="cuda")
    wide[:, :1024] = Xg
    lib = ttq.load_library()
    import ctypes
    s2 = torch.empty(1024, dtype=torch.float32, device="cuda")
    ws = ttq.alloc_workspace(3000, 1024, 0)
    rc = lib.ttq_act_stats(ctypes.c_void_p(wide.data_ptr()), 3000, 1024, 1040, ctypes.c_float(0.5),
                           ctypes.c_float(0.4), 2, ctypes.c_void_p(s2.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                           ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    assert torch.equal(a, s2)


def test_act_stats_degenerate_inputs():
    X = torch.zeros(64, 128, dtype=torch.bfloat16, device="cuda")
    s = ttq.act_stats(X, 1.0, 4.0).cpu().numpy()
    np.testing.assert_array_equal(s, np.full(128, 2.0, np.float32))   # (0 + 4)^(1/2)
    s = ttq.act_stats(gpu(synthetic.as_bf16(np.ones((5, 64)) * 3)), 0.0, 0.4).cpu().numpy()
    np.testing.assert_array_equal(s, np.ones(64, np.float32))         # alpha = 0: RTN


# ------------------------------------------------------------------ requant


def requant_check(Wb, W, s32, q, g):
    d_out, d = W.shape
    codes, scale, zero = ttq.requant(gpu(Wb), gpu(torch.from_numpy(s32)), q, g)
    oc, osc, oz = O.requant(W, s32, q, g)
    np.testing.assert_array_equal(packed_np(codes, q, d_out, d), O.pack_codes(oc, q))
    np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint16), osc.view(np.uint16))
    np.testing.assert_array_equal(zero.cpu().numpy().view(np.uint16), oz.view(np.uint16))


@pytest.mark.parametrize("q", [2, 3, 4])
@pytest.mark.parametrize("g", [32, 64, 128])
def test_requant_bitexact(q, g):
    Xb, Wb, X, W = layer(64, 256, 48, seed=100 + q * 10 + g)
    _, s32 = O.act_stats(X, 0.5, 0.4)
    requant_check(Wb, W, s32, q, g)


@pytest.mark.parametrize("d_out,d,q,g", [(1, 96, 3, 32), (3, 128, 2, 64), (130, 512, 4, 128), (7, 32, 4, 32),
                                         (257, 1024, 2, 32)])
def test_requant_ragged_shapes(d_out, d, q, g):
    Xb, Wb, X, W = layer(16, d, d_out, seed=d_out * 7 + d)
    _, s32 = O.act_stats(X, 0.75, 0.4)
    requant_check(Wb, W, s32, q, g)


@pytest.mark.parametrize("q", [2, 3, 4])
def test_requant_exact_ties(q):
    # weights on a grid of half steps: many v / sigma land exactly on .5 and exercise the
    # tie rule (halves to even) and the exact-division path of the kernel
    rng = np.random.default_rng(q)
    N = 2 ** q - 1
    d_out, d, g = 64, 128, 32
    half = rng.integers(-2 * N, 2 * N + 1, (d_out, d)).astype(np.float64) * 0.125
    grp = half.reshape(d_out, d // g, g)
    grp[:, :, 0] = -N * 0.125
    grp[:, :, 1] = N * 0.125
    W = grp.reshape(d_out, d)
    Wb = synthetic.as_bf16(W)
    requant_check(Wb, synthetic.bf16_values(Wb), np.ones(d, np.float32), q, g)


def test_requant_degenerate_groups():
    d_out, d = 8, 128
    W = np.zeros((d_out, d))
    W[1] = 0.5          # constant groups: zero range, |min| rule
    W[2] = -3.0
    W[3, :64] = 1e-3
    W[4] = np.tile([1.0, -1.0], d // 2)
    W[5] = 1e-30        # tiny values: sigma floors at the smallest fp16
    W[6, ::7] = 7.0
    Wb = synthetic.as_bf16(W)
    requant_check(Wb, synthetic.bf16_values(Wb), np.ones(d, np.float32), 3, 32)
    requant_check(Wb, synthetic.bf16_values(Wb), np.full(d, 0.3, np.float32), 4, 64)


@pytest.mark.parametrize("q", [2, 3, 4])
def test_requant_saturated_scale_and_clamped_zero(q):
    # groups whose range is so large that sigma saturates at the largest fp16 (every
    # quotient then needs the clamp), and groups whose spread is tiny next to their
    # offset (s varies by a few ulps across the group), so z is clamped to +-2048
    d_out, d, g = 6, 128, 32
    W = np.ones((d_out, d))
    W[0] = np.tile([3.0e6, -3.0e6, 1.0e5, -2.5e4], d // 4)
    W[1, ::3] = 2.0e7
    W[2] = -1.0
    W[3] = np.linspace(-4.0e6, 1.0e4, d)
    W[4, 64:] = 7.0e6
    Wb = synthetic.as_bf16(W)
    s = (1.0 + np.arange(d) * 2.0 ** -20).astype(np.float32)
    requant_check(Wb, synthetic.bf16_values(Wb), s, q, g)


@pytest.mark.parametrize("P,d_out,d,q,g", [(1, 130, 512, 4, 128), (3, 64, 96, 3, 32), (8, 257, 1024, 2, 64),
                                           (5, 200, 768, 4, 32)])
def test_requant_batched_matches_oracle_per_prompt(P, d_out, d, q, g):
    # one read of W, P statistics (each prompt's own activations): every prompt's codes,
    # scales and zeros equal the single-prompt oracle's bit for bit
    _, Wb, _, W = layer(8, d, d_out, seed=700 + P)
    S = []
    for p in range(P):
        Xp = synthetic.bf16_values(synthetic.as_bf16(synthetic.draw_layer(32, d, 1, seed=7000 + 13 * p)[0]))
        S.append(O.act_stats(Xp, 0.5 + 0.05 * p, 0.4)[1])
    S = np.stack(S).astype(np.float32)
    codes, scale, zero = ttq.requant_batched(gpu(Wb), gpu(torch.from_numpy(S)), q, g)
    for p in range(P):
        oc, osc, oz = O.requant(W, S[p], q, g)
        np.testing.assert_array_equal(packed_np(codes[p], q, d_out, d), O.pack_codes(oc, q))
        np.testing.assert_array_equal(scale[p].cpu().numpy().view(np.uint16), osc.view(np.uint16))
        np.testing.assert_array_equal(zero[p].cpu().numpy().view(np.uint16), oz.view(np.uint16))


def test_requant_fullsize_qwen3_32b_qproj_sampled_rows():
    # the 5120 -> 8192 projection at its full size; the oracle checks 64 sampled rows
    T, d, d_out, q, g = 4096, 5120, 8192, 4, 128
    Xb, Wb, X, W = layer(T, d, d_out, seed=3)
    _, s32 = O.act_stats(X, 0.5, 0.4)
    codes, scale, zero = ttq.requant(gpu(Wb), gpu(torch.from_numpy(s32)), q, g)
    rows = np.unique(np.concatenate([[0, d_out - 1], np.random.default_rng(0).choice(d_out, 62, replace=False)]))
    oc, osc, oz = O.requant(W[rows], s32, q, g)
    np.testing.assert_array_equal(packed_np(codes, q, d_out, d)[rows], O.pack_codes(oc, q))
    np.testing.assert_array_equal(scale.cpu().numpy()[rows].view(np.uint16), osc.view(np.uint16))
    np.testing.assert_array_equal(zero.cpu().numpy()[rows].view(np.uint16), oz.view(np.uint16))


# ------------------------------------------------------------------ projection (GEMM)


def oracle_inputs(T, d, d_out, q, g, r, seed, alpha=0.5):
    Xb, Wb, X, W = layer(T, d, d_out, seed)
    A = B = None
    if r > 0:
        B, A, W = O.lowrank_split(W, r)
    _, s32 = O.act_stats(X, alpha, 0.4)
    oc, osc, oz = O.requant(W, s32, q, g)
    return Xb, X, s32, oc, osc, oz, A, B


def gpu_linear_with_oracle_codes(Xb, s32, oc, osc, oz, A, B, q, g, r, d_out):
    d = Xb.shape[1]
    codes = gpu(torch.from_numpy(O.pack_codes(oc, q).view(np.int32).reshape(-1)))
    cfg = ttq.make_config(q, g, 0.5, 0.4, 2, r)
    At = gpu(synthetic.as_bf16(A)) if A is not None else None
    Bt = gpu(synthetic.as_bf16(B)) if B is not None else None
    Y = ttq.linear_decode(gpu(Xb), gpu(torch.from_numpy(s32)), codes, gpu(torch.from_numpy(osc)),
                          gpu(torch.from_numpy(oz)), cfg, d_out, At, Bt)
    return Y.float().cpu().numpy()


@pytest.mark.parametrize("T,d,d_out,q,g,r", [
    (1, 256, 128, 4, 32, 0), (7, 96, 48, 3, 32, 0), (16, 512, 512, 3, 32, 0), (100, 256, 300, 2, 64, 0),
    (128, 512, 256, 4, 128, 0), (300, 320, 200, 4, 64, 0), (1024, 768, 768, 4, 32, 0),
    (64, 256, 128, 4, 32, 16), (300, 512, 384, 3, 32, 16), (2048, 768, 3072, 4, 32, 0),
    (513, 1024, 640, 2, 32, 8), (4096, 512, 256, 4, 128, 0),
    # low rank: odd number of 8-rank tiles, the largest rank, K not a multiple of the
    # low-rank kernel's 64-wide stages, ragged token blocks
    (70, 96, 64, 3, 32, 24), (200, 1088, 256, 4, 64, 64), (1, 160, 96, 4, 32, 40),
])
def test_gemm_parity_with_oracle_codes(T, d, d_out, q, g, r):
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(T, d, d_out, q, g, r, seed=T * 3 + d)
    Yg = gpu_linear_with_oracle_codes(Xb, s32, oc, osc, oz, A, B, q, g, r, d_out)
    Yo = O.linear(X, s32, oc, osc, oz, g, A, B)
    assert np.isfinite(Yg).all()
    check_y(Yg, Yo)


# ------------------------------------------------------------------ full prefill


def prefill_check(T, d, d_out, q, g, alpha, r, seed, rows=None, p=2):
    Xb, Wb, X, W = layer(T, d, d_out, seed)
    A = B = None
    At = Bt = None
    Wq = W
    Wqb = Wb
    if r > 0:
        B, A, Wq = O.lowrank_split(W, r)
        At, Bt = gpu(synthetic.as_bf16(A)), gpu(synthetic.as_bf16(B))
        Wqb = synthetic.as_bf16(Wq)
    cfg = ttq.make_config(q, g, alpha, 0.4, p, r)
    out = ttq.linear_prefill(gpu(Xb), gpu(Wqb), cfg, At, Bt)
    s64, s32 = O.act_stats(X, alpha, 0.4, p)
    s_gpu = out["s"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(s_gpu - s64) / s64) <= S_RTOL
    if rows is None:
        rows = np.arange(d_out)
    oc, osc, oz = O.requant(Wq[rows], s32, q, g)
    gc = O.unpack_codes(packed_np(out["codes"], q, d_out, d)[rows], q, d)
    # codes come from the GPU's own s (within 1e-5 of the oracle's): only weights sitting
    # on a rounding boundary may move, and by one step
    diff = np.abs(gc - oc)
    assert diff.max() <= 1
    assert np.mean(diff != 0) <= 1e-3
    Ao = A
    Yo = O.linear(X, s32, oc, osc, oz, g, Ao, B[rows] if B is not None else None)
    Yg = out["Y"].float().cpu().numpy()[:, rows]
    check_y(Yg, Yo)
    return out


@pytest.mark.parametrize("Ts,d,d_out,q,g,r", [
    ((300, 517, 256), 1024, 640, 4, 64, 0),    # grouped launch, ragged last tiles
    ((1, 700), 768, 384, 3, 32, 16),           # grouped, a one-token prompt, low rank
    ((16, 40), 512, 256, 2, 32, 0),            # 56 tokens: one projection per prompt
    ((400, 200), 512, 128, 4, 128, 8),         # d_out = 128: one projection per prompt
])
def test_prefill_batched_matches_single_prompts(Ts, d, d_out, q, g, r):
    # several prompts, each with its own statistic and codes, in one call; prompt p must
    # match the oracle on its own tokens exactly as a single-prompt prefill does
    P = len(Ts)
    Xs, Xvs = [], []
    for p, Tp in enumerate(Ts):
        X = synthetic.draw_layer(Tp, d, 1, seed=5000 + 11 * p + Tp)[0]
        Xs.append(synthetic.as_bf16(X))
        Xvs.append(synthetic.bf16_values(Xs[-1]))
    _, Wb, _, W = layer(8, d, d_out, seed=5100 + d)
    A = B = At = Bt = None
    Wq, Wqb = W, Wb
    if r > 0:
        B, A, Wq = O.lowrank_split(W, r)
        At, Bt = gpu(synthetic.as_bf16(A)), gpu(synthetic.as_bf16(B))
        Wqb = synthetic.as_bf16(Wq)
    cfg = ttq.make_config(q, g, 0.5, 0.4, 2, r)
    out = ttq.linear_prefill_batched(gpu(torch.cat(Xs)), Ts, gpu(Wqb), cfg, At, Bt)
    off = 0
    for p, Tp in enumerate(Ts):
        s64, s32 = O.act_stats(Xvs[p], 0.5, 0.4)
        s_gpu = out["s"][p].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(s_gpu - s64) / s64) <= S_RTOL
        oc, osc, oz = O.requant(Wq, s32, q, g)
        gc = O.unpack_codes(packed_np(out["codes"][p], q, d_out, d), q, d)
        diff = np.abs(gc - oc)
        assert diff.max() <= 1 and np.mean(diff != 0) <= 1e-3
        Yo = O.linear(Xvs[p], s32, oc, osc, oz, g, A, B)
        Yg = out["Y"][off:off + Tp].float().cpu().numpy()
        assert np.isfinite(Yg).all()
        check_y(Yg, Yo, p)
        off += Tp


@pytest.mark.parametrize("T,d,d_out,q,g,r", [(300, 1024, 640, 4, 64, 0), (128, 512, 512, 3, 32, 16),
                                             (4096, 5120, 8192, 4, 128, 0)])
def test_prefill_p1_statistic(T, d, d_out, q, g, r):
    # the mean-|x| statistic (p = 1, the classic activation-aware reading) through the
    # whole prefill: s against the oracle's p = 1 statistic, codes within one step, Y
    rows = None if d_out <= 1024 else np.unique(np.concatenate([[0, d_out - 1],
                                                                np.random.default_rng(T).choice(d_out, 62, replace=False)]))
    prefill_check(T, d, d_out, q, g, 0.5, r, seed=T + d + 1, rows=rows, p=1)


@pytest.mark.parametrize("T,d,d_out,r,p", [
    (8, 256, 128, 8, 2),        # the last token count with the separate statistic kernel
    (9, 256, 128, 8, 2),        # the first with the statistic in the low-rank pass; 9 of 64 rows
    (65, 1088, 256, 24, 1),     # one token in the second block; K not a multiple of 64
    (300, 512, 384, 16, 2), (2048, 768, 512, 16, 1),
    (4100, 5120, 8192, 64, 2),  # the 32B query projection's width, ragged last token block
])
def test_statistic_from_lowrank_pass(T, d, d_out, r, p):
    # with a rank-r side path the prefill takes s from the same pass over X as X A^T: s
    # against the oracle, and against the separate statistic kernel (two fp32 sums in
    # different orders), then codes and Y as for every prefill
    rows = None if d_out <= 1024 else np.unique(np.concatenate([[0, d_out - 1],
                                                                np.random.default_rng(T).choice(d_out, 62, replace=False)]))
    prefill_check(T, d, d_out, 4, 128 if d % 128 == 0 else 32, 0.5, r, seed=T + 7 * d + r, rows=rows, p=p)
    Xb, Wb = layer(T, d, d_out, T + 7 * d + r)[:2]
    s_sep = ttq.act_stats(gpu(Xb), 0.5, 0.4, p).cpu().numpy().astype(np.float64)
    At = gpu(synthetic.as_bf16(np.zeros((r, d))))
    Bt = gpu(synthetic.as_bf16(np.zeros((d_out, r))))
    s_fused = ttq.linear_prefill(gpu(Xb), gpu(Wb), ttq.make_config(4, 32, 0.5, 0.4, p, r), At, Bt)["s"]
    s_fused = s_fused.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(s_fused - s_sep) / s_sep) <= 2e-6
    assert ttq.device_status() == 0


def test_decode_after_p1_prefill_matches_oracle():
    # decode steps reuse the p = 1 prefill's s and codes (the decode does not see p)
    T, d, d_out, q, g = 256, 1024, 384, 4, 64
    Xb, Wb, X, W = layer(T, d, d_out, seed=303)
    lin = ttq.TTQLinear(gpu(Wb), q, g, 0.5, 0.4, p=1)
    lin.prefill(gpu(Xb))
    s64, s32 = O.act_stats(X, 0.5, 0.4, 1)
    s_gpu = lin.s.cpu().numpy()
    assert np.max(np.abs(s_gpu.astype(np.float64) - s64) / s64) <= S_RTOL
    oc, osc, oz = O.requant(W, s_gpu, q, g)
    np.testing.assert_array_equal(packed_np(lin.codes, q, d_out, d), O.pack_codes(oc, q))
    for b in (1, 2, 5):
        xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=304 + b))
        Yg = lin.decode(gpu(xt)).float().cpu().numpy()
        check_y(Yg, O.linear(synthetic.bf16_values(xt), s_gpu, oc, osc, oz, g), ("p1 decode", b))


def test_prefill_batched_p1():
    Ts, d, d_out, q, g = (300, 200), 512, 256, 4, 32
    Xs = [synthetic.as_bf16(synthetic.draw_layer(Tp, d, 1, seed=310 + Tp)[0]) for Tp in Ts]
    _, Wb, _, W = layer(8, d, d_out, seed=311)
    cfg = ttq.make_config(q, g, 0.5, 0.4, 1, 0)
    out = ttq.linear_prefill_batched(gpu(torch.cat(Xs)), Ts, gpu(Wb), cfg)
    off = 0
    for p_, Tp in enumerate(Ts):
        Xv = synthetic.bf16_values(Xs[p_])
        s64, _ = O.act_stats(Xv, 0.5, 0.4, 1)
        s_gpu = out["s"][p_].cpu().numpy()
        assert np.max(np.abs(s_gpu.astype(np.float64) - s64) / s64) <= S_RTOL
        oc, osc, oz = O.requant(W, s_gpu, q, g)
        np.testing.assert_array_equal(packed_np(out["codes"][p_], q, d_out, d), O.pack_codes(oc, q))
        check_y(out["Y"][off:off + Tp].float().cpu().numpy(), O.linear(Xv, s_gpu, oc, osc, oz, g), ("p1 batched", p_))
        off += Tp


def test_prefill_single_512():
    prefill_check(128, 512, 512, 3, 32, 0.5, 0, seed=0)


def test_prefill_opt125m_fc1():
    prefill_check(2048, 768, 3072, 4, 32, 0.5, 0, seed=1004)


@pytest.mark.parametrize("g", [32, 64, 128])
def test_prefill_qwen3_1p7b_q_proj_lowrank(g):
    prefill_check(4096, 2048, 2048, 3, g, 0.75, 16, seed=2000)


def test_prefill_qwen3_8b_down_proj_q2_rows():
    rows = np.sort(np.random.default_rng(1).choice(4096, 48, replace=False))
    prefill_check(512, 12288, 4096, 2, 32, 0.5, 16, seed=4006, rows=rows)


@pytest.mark.parametrize("T", [16, 4096])
def test_prefill_fullsize_qwen3_32b_qproj(T):
    # the benchmark's launch configuration (5120 -> 8192, q = 4, g = 128); the oracle
    # checks s on every channel and Y on 64 sampled output rows
    rows = np.unique(np.concatenate([[0, 8191], np.random.default_rng(T).choice(8192, 62, replace=False)]))
    prefill_check(T, 5120, 8192, 4, 128, 0.5, 0, seed=3, rows=rows)


@pytest.mark.parametrize("b", [1, 8, 64])
def test_decode_qwen3_32b_qproj(b):
    d, d_out, q, g = 5120, 8192, 4, 128
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(1024, d, d_out, q, g, 0, seed=3)
    xt = synthetic.draw_tokens(b, d, seed=77 + b)
    xtb = synthetic.as_bf16(xt)
    Yg = gpu_linear_with_oracle_codes(xtb, s32, oc, osc, oz, None, None, q, g, 0, d_out)
    Yo = O.linear(synthetic.bf16_values(xtb), s32, oc, osc, oz, g)
    check_y(Yg, Yo)


def test_prefill_then_decode_reuses_codes():
    Xb, Wb, X, W = layer(256, 512, 384, seed=55)
    lin = ttq.TTQLinear(gpu(Wb), 4, 64, 0.5, 0.4)
    Y = lin.prefill(gpu(Xb))
    # decoding the prompt's own rows with the stored codes reproduces the prefill output
    Yd = lin.decode(gpu(Xb[:37].contiguous()))
    assert torch.equal(Y[:37], Yd) or rel_fro(Yd.float().cpu().numpy(), Y[:37].float().cpu().numpy()) < 1e-2


def test_zero_weight_and_zero_activation():
    T, d, d_out = 32, 128, 64
    X = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(d_out, d, dtype=torch.bfloat16, device="cuda")
    out = ttq.linear_prefill(X, W, ttq.make_config(4, 32, 0.5, 0.4))
    assert torch.count_nonzero(out["Y"]) == 0
    np.testing.assert_array_equal(out["s"].cpu().numpy(), np.full(d, np.float32(0.4) ** np.float32(0.25), np.float32))


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("q,g,r,d_out", [(4, 128, 0, 384), (3, 32, 0, 300), (2, 32, 16, 256), (4, 64, 8, 130),
                                         (4, 32, 64, 192)])
def test_decode_few_tokens_parity(b, q, g, r, d_out):
    # few decode tokens run on the CUDA-core GEMV (codes streamed once); same bar as the GEMM
    d = 1024
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(256, d, d_out, q, g, r, seed=900 + b * 10 + q)
    xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=31 + b))
    Yg = gpu_linear_with_oracle_codes(xt, s32, oc, osc, oz, A, B, q, g, r, d_out)
    Yo = O.linear(synthetic.bf16_values(xt), s32, oc, osc, oz, g, A, B)
    assert np.isfinite(Yg).all()
    check_y(Yg, Yo)


@pytest.mark.parametrize("b,d,d_out,q,g,r", [
    (1, 1024, 384, 4, 128, 0),
    (16, 1024, 300, 3, 32, 0),    # ragged last row block, g = 32
    (17, 512, 640, 2, 64, 16),    # low rank
    (33, 2048, 256, 4, 32, 8),
    (64, 768, 520, 4, 128, 0),
    (5, 256, 128 * 300, 4, 128, 0),  # many row blocks
    (2, 5120, 1024, 4, 128, 16),  # the Qwen3-32B hidden size with low rank
    (3, 5120, 520, 3, 64, 0),     # 3-bit bit planes, 10 slices of 10 units per row
    (1, 4096, 512, 2, 32, 24),    # one token: U formed in the GEMV's prep launch, odd 8-rank tiles
])
def test_decode_parity_shapes(b, d, d_out, q, g, r):
    # b <= 8 runs on the CUDA-core GEMV (one lane per weight row), larger b on the tensor cores
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(128, d, d_out, q, g, r, seed=700 + b + d_out)
    xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=5 + b))
    Yg = gpu_linear_with_oracle_codes(xt, s32, oc, osc, oz, A, B, q, g, r, d_out)
    Yo = O.linear(synthetic.bf16_values(xt), s32, oc, osc, oz, g, A, B)
    assert np.isfinite(Yg).all()
    check_y(Yg, Yo)


@pytest.mark.parametrize("P,b,d,d_out,q,g,r", [
    (1, 1, 1024, 384, 4, 128, 0), (3, 1, 512, 300, 3, 32, 0), (8, 2, 1024, 256, 4, 64, 16),
    (5, 2, 768, 130, 2, 32, 8), (4, 3, 512, 200, 4, 32, 16),   # b = 3: the requests one after another
])
def test_decode_batched_requests_match_oracle(P, b, d, d_out, q, g, r):
    # every request carries its own prefill (own statistic, codes, scale, zero); the shared
    # static low-rank factors come from the one weight
    _, Wb, _, W = layer(8, d, d_out, seed=4000 + P * 7 + b)
    A = B = None
    Wq = W
    if r > 0:
        B, A, Wq = O.lowrank_split(W, r)
    S, C, SC, Z, Xs, Ys = [], [], [], [], [], []
    for p in range(P):
        Xp = synthetic.bf16_values(synthetic.as_bf16(synthetic.draw_layer(64, d, 1, seed=4100 + 31 * p + b)[0]))
        s32 = O.act_stats(Xp, 0.5, 0.4)[1]
        oc, osc, oz = O.requant(Wq, s32, q, g)
        xt = synthetic.bf16_values(synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=4200 + 17 * p + b)))
        S.append(s32)
        C.append(O.pack_codes(oc, q).view(np.int32).reshape(-1))
        SC.append(osc)
        Z.append(oz)
        Xs.append(xt)
        Ys.append(O.linear(xt, s32, oc, osc, oz, g, A, B))
    cfg = ttq.make_config(q, g, 0.5, 0.4, 2, r)
    At = gpu(synthetic.as_bf16(A)) if A is not None else None
    Bt = gpu(synthetic.as_bf16(B)) if B is not None else None
    Xg = gpu(synthetic.as_bf16(np.stack(Xs)))
    Yg = ttq.linear_decode_batched(Xg, gpu(torch.from_numpy(np.stack(S))), gpu(torch.from_numpy(np.stack(C))),
                                   gpu(torch.from_numpy(np.stack(SC))), gpu(torch.from_numpy(np.stack(Z))), cfg,
                                   d_out, At, Bt)
    Yg = Yg.float().cpu().numpy()
    assert np.isfinite(Yg).all()
    for p in range(P):
        check_y(Yg[p], Ys[p], p)


@pytest.mark.parametrize("b,d", [(1, 992), (2, 160), (2, 96), (3, 992), (8, 160), (7, 96)])
def test_decode_small_hidden_parity(b, d):
    # hidden sizes with fewer 32-input units than lanes in a warp, and ragged unit counts
    d_out, q, g = 200, 4, 32
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(64, d, d_out, q, g, 0, seed=b * 11 + d)
    xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=9 + b))
    Yg = gpu_linear_with_oracle_codes(xt, s32, oc, osc, oz, None, None, q, g, 0, d_out)
    Yo = O.linear(synthetic.bf16_values(xt), s32, oc, osc, oz, g)
    check_y(Yg, Yo)


@pytest.mark.parametrize("b", [1, 8])
def test_decode_is_deterministic(b):
    # every reduction (GEMV lanes, split-K partials) runs in a fixed order: repeated steps
    # agree bit for bit
    d, d_out, q, g = 1024, 384, 4, 128
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(64, d, d_out, q, g, 0, seed=42)
    xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=43))
    Y1 = gpu_linear_with_oracle_codes(xt, s32, oc, osc, oz, None, None, q, g, 0, d_out)
    Y2 = gpu_linear_with_oracle_codes(xt, s32, oc, osc, oz, None, None, q, g, 0, d_out)
    np.testing.assert_array_equal(Y1, Y2)


@pytest.mark.parametrize("b", [2, 6])
@pytest.mark.parametrize("g", [32, 128])
def test_decode_far_zero_points(g, b):
    # groups whose scaled weights all share one sign get zero points far outside [0, 2^q - 1]
    # (up to the +-2048 clamp): (128 + z) sum x' must stay exact
    d, d_out, q = 1024, 256, 4
    Xb, Wb, X, W = layer(128, d, d_out, seed=77)
    _, s32 = O.act_stats(X, 0.5, 0.4)
    W = W.copy()
    rng = np.random.default_rng(5)
    for i in range(0, 40):
        k = slice((i % (d // g)) * g, (i % (d // g) + 1) * g)
        # scaled weights w * s of one sign in a narrow band
        W[i, k] = (0.05 + 1e-4 * rng.standard_normal(g)) / s32[k]
        W[i + 40, k] = (-0.03 + 2e-5 * rng.standard_normal(g)) / s32[k]
    W = synthetic.bf16_values(synthetic.as_bf16(W))
    oc, osc, oz = O.requant(W, s32, q, g)
    assert np.abs(oz).max() > 128
    xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=12))
    Yg = gpu_linear_with_oracle_codes(xt, s32, oc, osc, oz, None, None, q, g, 0, d_out)
    Yo = O.linear(synthetic.bf16_values(xt), s32, oc, osc, oz, g)
    check_y(Yg, Yo)


# ------------------------------------------------------------------ fold (X diag(1/s) in bf16)


def bf16_ulp(x):
    _, e = np.frexp(np.abs(np.asarray(x, dtype=np.float64)))
    return np.ldexp(1.0, e - 8)


def fold_check(Xf_gpu, X, s32):
    # the kernels form bf16(x * RN_fp32(1/s)); the oracle rounds the exact quotient x / s
    # once. The two differ only where x * RN(1/s) and x / s straddle a bf16 rounding
    # boundary: at most one bf16 step, and rarely
    want = O.fold(X, s32)
    diff = np.abs(Xf_gpu - want)
    assert np.all(diff <= bf16_ulp(np.maximum(np.abs(Xf_gpu), np.abs(want))) * (1 + 1e-12))
    assert np.mean(diff != 0) <= 1e-3, np.mean(diff != 0)


def read_folded(ws, T, d, d_out, cfg):
    off = ttq.workspace_folded_offset(T, d, d_out, cfg)
    return ws[off: off + 2 * T * d].view(torch.bfloat16).reshape(T, d).float().cpu().numpy()


@pytest.mark.parametrize("T,d,d_out,q,g,r", [
    (128, 512, 512, 3, 32, 0), (300, 1088, 256, 4, 64, 16), (4096, 5120, 8192, 4, 128, 0), (1, 96, 64, 2, 32, 0),
    (777, 800, 136, 4, 32, 0),
])
def test_prefill_fold_matches_oracle(T, d, d_out, q, g, r):
    # the fold fused into the prefill's re-quantization launch, read back from the workspace
    # and compared element by element with the oracle's fold by the GPU's own s
    Xb, Wb, X, W = layer(T, d, d_out, seed=T + 3 * d)
    cfg = ttq.make_config(q, g, 0.5, 0.4, 2, r)
    At = Bt = None
    if r > 0:
        B, A, Wq = O.lowrank_split(W, r)
        At, Bt, Wb = gpu(synthetic.as_bf16(A)), gpu(synthetic.as_bf16(B)), synthetic.as_bf16(Wq)
    ws = ttq.alloc_workspace(T, d, d_out, cfg)
    out = ttq.linear_prefill(gpu(Xb), gpu(Wb), cfg, At, Bt, ws=ws)
    torch.cuda.synchronize()
    fold_check(read_folded(ws, T, d, d_out, cfg), X, out["s"].cpu().numpy())


@pytest.mark.parametrize("b,d", [(3, 512), (64, 5120), (17, 800)])
def test_decode_fold_matches_oracle(b, d):
    # decode batches above two rows fold in their own kernel ahead of the tensor-core GEMM
    d_out, q, g = 256, 4, 32
    Xb, X, s32, oc, osc, oz, A, B = oracle_inputs(64, d, d_out, q, g, 0, seed=b + d)
    xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=b))
    cfg = ttq.make_config(q, g, 0.5, 0.4)
    ws = ttq.alloc_workspace(b, d, d_out, cfg)
    codes = gpu(torch.from_numpy(O.pack_codes(oc, q).view(np.int32).reshape(-1)))
    ttq.linear_decode(gpu(xt), gpu(torch.from_numpy(s32)), codes, gpu(torch.from_numpy(osc)),
                      gpu(torch.from_numpy(oz)), cfg, d_out, ws=ws)
    torch.cuda.synchronize()
    fold_check(read_folded(ws, b, d, d_out, cfg), synthetic.bf16_values(xt), s32)
