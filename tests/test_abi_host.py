"""The C-ABI library on the host, without a GPU: it loads, it exports every entry point
include/ttq.h declares, and argument errors come back synchronously with the
documented status before anything touches the device."""

import ctypes
import os
import re

import pytest

import online_activation_aware_b200 as ttq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE = 0, -1, -2, -3, -4


@pytest.fixture(scope="module")
def lib():
    from online_activation_aware_b200 import build

    build.build()
    return ttq.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "ttq.h")) as f:
        text = f.read()
    return re.findall(r"TTQ_API\s+[\w\s\*]+?\b(ttq_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ("ttq_act_stats", "ttq_requant", "ttq_linear_prefill", "ttq_linear_decode",
              "ttq_workspace_size", "ttq_codes_words", "ttq_device_status", "ttq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_codes_words(lib):
    assert ttq.codes_words(8192, 5120, 4) == 8192 * 5120 * 4 // 32
    assert ttq.codes_words(3, 96, 3) == 3 * 3 * 3
    assert lib.ttq_codes_words(4, 100, 4) == 0  # d not a multiple of 32
    assert lib.ttq_codes_words(4, 64, 5) == 0


def test_status_strings(lib):
    for code, name in ttq.STATUS.items():
        assert lib.ttq_status_string(code).decode() == name


def test_workspace_size_components(lib):
    cfg = ttq.make_config(4, 128, 0.5, 0.4)
    ws_stats = ttq.workspace_size(4096, 5120, 0)
    ws_full = ttq.workspace_size(4096, 5120, 8192, cfg)
    # the statistic alone reduces on chip and needs no workspace
    assert ws_stats == 0
    # the prefill's fused statistic + fold reduces on chip; the folded activations alone
    # are T * d bf16
    assert ws_full >= 4096 * 5120 * 2
    cfg_r = ttq.make_config(4, 128, 0.5, 0.4, r=16)
    # with a low-rank side path: U (bf16 [T, 64]) and the statistic's per-64-token-block
    # column sums of the fused pass (fp32 [T / 64, d])
    assert ttq.workspace_size(4096, 5120, 8192, cfg_r) >= ws_full + 4096 * 64 * 2 + (4096 // 64) * 5120 * 4
    # a decode of one or two tokens forms U in its prep launch: no block sums there
    assert ttq.workspace_size(2, 5120, 8192, cfg_r) < (4096 // 64) * 5120 * 4


def test_folded_offset_inside_workspace(lib):
    # the folded activations (bf16 [T, d]) fit inside the workspace at a 16-byte aligned offset
    for T, d, d_out, r in ((4096, 5120, 8192, 0), (17, 256, 96, 16), (3, 1024, 300, 8)):
        cfg = ttq.make_config(4, 32, 0.5, 0.4, r=r)
        off = ttq.workspace_folded_offset(T, d, d_out, cfg)
        assert off % 16 == 0
        assert off + 2 * T * d <= ttq.workspace_size(T, d, d_out, cfg)
    n = ctypes.c_size_t(0)
    cfg = ttq.make_config(4, 32, 0.5, 0.4)
    assert lib.ttq_workspace_folded_offset(16, 64, 8, None, ctypes.byref(n)) == INVALID
    assert lib.ttq_workspace_folded_offset(16, 64, 8, ctypes.byref(cfg), None) == INVALID
    assert lib.ttq_workspace_folded_offset(16, 64, 0, ctypes.byref(cfg), ctypes.byref(n)) == INVALID
    assert lib.ttq_workspace_folded_offset(16, 64, 8, ctypes.byref(ttq.make_config(5, 32, 0.5, 0.4)),
                                           ctypes.byref(n)) == UNSUPPORTED


def _p(v):
    return ctypes.c_void_p(v)


def test_requant_argument_errors(lib):
    a = 1 << 20  # a 16-byte-aligned fake address: never dereferenced on these paths
    assert lib.ttq_requant(_p(a), 16, 64, _p(a), 5, 32, _p(a), _p(a), _p(a), None) == UNSUPPORTED
    assert lib.ttq_requant(_p(a), 16, 64, _p(a), 4, 48, _p(a), _p(a), _p(a), None) == UNSUPPORTED
    assert lib.ttq_requant(_p(a), 16, 96, _p(a), 4, 64, _p(a), _p(a), _p(a), None) == INVALID
    assert lib.ttq_requant(None, 16, 64, _p(a), 4, 32, _p(a), _p(a), _p(a), None) == INVALID
    assert lib.ttq_requant(_p(a + 8), 16, 64, _p(a), 4, 32, _p(a), _p(a), _p(a), None) == MISALIGNED
    assert lib.ttq_requant(_p(a), 0, 64, _p(a), 4, 32, _p(a), _p(a), _p(a), None) == INVALID


def test_requant_batched_argument_errors(lib):
    a = 1 << 20
    assert lib.ttq_requant_batched(_p(a), 16, 64, _p(a), 0, 4, 32, _p(a), _p(a), _p(a), None) == UNSUPPORTED
    assert lib.ttq_requant_batched(_p(a), 16, 64, _p(a), 9, 4, 32, _p(a), _p(a), _p(a), None) == UNSUPPORTED
    assert lib.ttq_requant_batched(_p(a), 16, 64, _p(a), 2, 5, 32, _p(a), _p(a), _p(a), None) == UNSUPPORTED
    assert lib.ttq_requant_batched(_p(a), 16, 64, _p(a + 4), 2, 4, 32, _p(a), _p(a), _p(a), None) == MISALIGNED
    assert lib.ttq_requant_batched(_p(a), 16, 64, None, 2, 4, 32, _p(a), _p(a), _p(a), None) == INVALID


def test_act_stats_argument_errors(lib):
    a = 1 << 20
    f = ctypes.c_float
    assert lib.ttq_act_stats(_p(a), 8, 64, 64, f(0.5), f(0.4), 3, _p(a), _p(a), 1 << 20, None) == UNSUPPORTED
    assert lib.ttq_act_stats(_p(a), 8, 64, 64, f(-0.5), f(0.4), 2, _p(a), _p(a), 1 << 20, None) == INVALID
    assert lib.ttq_act_stats(_p(a), 8, 64, 64, f(0.5), f(0.0), 2, _p(a), _p(a), 1 << 20, None) == INVALID
    assert lib.ttq_act_stats(_p(a), 8, 64, 32, f(0.5), f(0.4), 2, _p(a), _p(a), 1 << 20, None) == INVALID
    assert lib.ttq_act_stats(_p(a), 8, 60, 64, f(0.5), f(0.4), 2, _p(a), _p(a), 1 << 20, None) == INVALID
    assert lib.ttq_act_stats(_p(a + 4), 8, 64, 64, f(0.5), f(0.4), 2, _p(a), _p(a), 1 << 20, None) == MISALIGNED
    assert lib.ttq_act_stats(_p(a), 8, 64, 64, f(0.5), f(0.4), 2, _p(a), _p(a + 4), 16, None) == MISALIGNED
    assert lib.ttq_act_stats(_p(a), 0, 64, 64, f(0.5), f(0.4), 2, _p(a), _p(a), 1 << 20, None) == INVALID


@pytest.mark.parametrize("cfg,status", [
    (dict(q=4, g=32, alpha=0.5, lam=0.4, p=2, r=12), UNSUPPORTED),   # r not a multiple of 8
    (dict(q=4, g=32, alpha=0.5, lam=0.4, p=2, r=72), UNSUPPORTED),   # r > 64
    (dict(q=4, g=32, alpha=0.5, lam=0.4, p=4, r=0), UNSUPPORTED),
    (dict(q=1, g=32, alpha=0.5, lam=0.4, p=2, r=0), UNSUPPORTED),
    (dict(q=4, g=32, alpha=0.5, lam=0.0, p=2, r=0), INVALID),        # lambda must be > 0
    (dict(q=4, g=32, alpha=float("nan"), lam=0.4, p=2, r=0), INVALID),
])
def test_prefill_config_errors(lib, cfg, status):
    a = 1 << 20
    c = ttq.make_config(cfg["q"], cfg["g"], cfg["alpha"], cfg["lam"], cfg["p"], cfg["r"])
    A = _p(a) if cfg["r"] > 0 else None
    rc = lib.ttq_linear_prefill(_p(a), 16, 128, _p(a), 64, A, A, ctypes.byref(c), _p(a), _p(a), _p(a),
                                _p(a), _p(a), _p(a), 1 << 30, None)
    assert rc == status


def test_prefill_lowrank_pointer_rules(lib):
    a = 1 << 20
    c0 = ttq.make_config(4, 32, 0.5, 0.4, 2, 0)
    c16 = ttq.make_config(4, 32, 0.5, 0.4, 2, 16)
    args = (_p(a), _p(a), _p(a), _p(a), _p(a), _p(a), 1 << 30, None)
    # factors given with r = 0, or missing with r > 0
    assert lib.ttq_linear_prefill(_p(a), 16, 128, _p(a), 64, _p(a), _p(a), ctypes.byref(c0), *args) == INVALID
    assert lib.ttq_linear_prefill(_p(a), 16, 128, _p(a), 64, None, None, ctypes.byref(c16), *args) == INVALID
    assert lib.ttq_linear_prefill(_p(a), 16, 128, _p(a), 64, _p(a + 2), _p(a), ctypes.byref(c16), *args) == MISALIGNED


def test_decode_argument_errors(lib):
    a = 1 << 20
    c = ttq.make_config(3, 128, 0.5, 0.4)
    assert lib.ttq_linear_decode(_p(a), 1, 96, 64, _p(a), _p(a), _p(a), _p(a), None, None, ctypes.byref(c),
                                 _p(a), _p(a), 1 << 30, None) == INVALID  # d % g != 0
    c = ttq.make_config(3, 32, 0.5, 0.4)
    assert lib.ttq_linear_decode(_p(a), 1, 96, 64, _p(a), _p(a), _p(a), _p(a), None, None, ctypes.byref(c),
                                 _p(a), None, 1 << 30, None) == WORKSPACE


def test_decode_batched_argument_errors(lib):
    a = 1 << 20
    c = ttq.make_config(4, 32, 0.5, 0.4)
    args = (_p(a), _p(a), _p(a), _p(a), None, None, ctypes.byref(c), _p(a), _p(a), 1 << 30, None)
    assert lib.ttq_linear_decode_batched(_p(a), 0, 1, 128, 64, *args) == UNSUPPORTED
    assert lib.ttq_linear_decode_batched(_p(a), 4097, 1, 128, 64, *args) == UNSUPPORTED
    assert lib.ttq_linear_decode_batched(_p(a + 8), 2, 1, 128, 64, *args) == MISALIGNED
    n = ctypes.c_size_t(0)
    assert lib.ttq_decode_batched_workspace_size(4, 1, 128, 64, ctypes.byref(c), ctypes.byref(n)) == OK
    assert n.value >= 4 * 128 * 4  # one x' slice per request


def test_prefill_batched_argument_errors(lib):
    a = 1 << 20
    c = ttq.make_config(4, 32, 0.5, 0.4)
    i64p = ctypes.c_int64 * 3
    T = i64p(16, 32, 8)
    tail = (_p(a), 64, None, None, ctypes.byref(c), _p(a), _p(a), _p(a), _p(a), _p(a), _p(a), 1 << 30, None)
    assert lib.ttq_linear_prefill_batched(_p(a), T, 0, 128, *tail) == UNSUPPORTED
    assert lib.ttq_linear_prefill_batched(_p(a), T, 9, 128, *tail) == UNSUPPORTED
    assert lib.ttq_linear_prefill_batched(_p(a), None, 2, 128, *tail) == INVALID
    assert lib.ttq_linear_prefill_batched(_p(a), i64p(16, 0, 8), 3, 128, *tail) == INVALID
    assert lib.ttq_linear_prefill_batched(_p(a + 8), T, 3, 128, *tail) == MISALIGNED
    n = ctypes.c_size_t(0)
    assert lib.ttq_prefill_batched_workspace_size(T, 3, 128, 64, ctypes.byref(c), ctypes.byref(n)) == OK
    assert n.value >= (16 + 32 + 8) * 128 * 2  # the folded activations of every prompt


def test_decoder_kernel_argument_errors(lib):
    a, b, c = 1 << 20, 1 << 21, 1 << 22
    f = ctypes.c_float
    # rmsnorm: sizes, eps, aliasing, alignment
    assert lib.ttq_rmsnorm(_p(a), None, _p(b), 4, 60, f(1e-6), _p(c), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a), None, _p(b), 4, 16384, f(1e-6), _p(c), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a), None, _p(b), 0, 64, f(1e-6), _p(c), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a), None, _p(b), 4, 64, f(0.0), _p(c), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a), _p(a), _p(b), 4, 64, f(1e-6), _p(c), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a), _p(c), _p(b), 4, 64, f(1e-6), _p(c), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a), None, _p(b), 4, 64, f(1e-6), _p(a), None) == INVALID
    assert lib.ttq_rmsnorm(_p(a + 2), None, _p(b), 4, 64, f(1e-6), _p(c), None) == MISALIGNED
    assert lib.ttq_rmsnorm(None, None, _p(b), 4, 64, f(1e-6), _p(c), None) == INVALID
    # rotary table
    assert lib.ttq_rope_table(16, 96, ctypes.c_double(1e6), _p(a), None) == UNSUPPORTED
    assert lib.ttq_rope_table(0, 128, ctypes.c_double(1e6), _p(a), None) == INVALID
    assert lib.ttq_rope_table(16, 128, ctypes.c_double(1.0), _p(a), None) == INVALID
    assert lib.ttq_rope_table(16, 128, ctypes.c_double(1e6), _p(a + 4), None) == MISALIGNED
    # q/k norm + rotation: head_dim, positions against the cache and the table, aliasing
    d = 1 << 23
    args = lambda T, D, pos0, tpos, clen, kc=b, vc=c: (_p(a), T, 8, 2, D, _p(d), _p(d), f(1e-6), _p(d), tpos, pos0,
                                                     None, _p(kc), _p(vc), clen, None)
    assert lib.ttq_qk_norm_rope(*args(4, 96, 0, 64, 64)) == UNSUPPORTED
    assert lib.ttq_qk_norm_rope(*args(4, 128, 61, 64, 128)) == INVALID      # past the table
    assert lib.ttq_qk_norm_rope(*args(4, 128, 61, 128, 64)) == INVALID      # past the cache
    assert lib.ttq_qk_norm_rope(*args(0, 128, 0, 64, 64)) == INVALID
    assert lib.ttq_qk_norm_rope(*args(4, 128, -1, 64, 64)) == INVALID
    assert lib.ttq_qk_norm_rope(*args(4, 128, 0, 64, 64, kc=b, vc=b)) == INVALID
    assert lib.ttq_qk_norm_rope(*args(4, 128, 0, 64, 64, kc=b + 8)) == MISALIGNED
    # a device-held position is checked on the device, but its pointer alignment here
    dev_pos = (_p(a), 4, 8, 2, 128, _p(d), _p(d), f(1e-6), _p(d), 64, 0, _p(d + 4), _p(b), _p(c), 64, None)
    assert lib.ttq_qk_norm_rope(*dev_pos) == MISALIGNED
    # decode attention
    sz = ctypes.c_size_t(0)
    assert lib.ttq_decode_attention_workspace_size(32, 8, 128, 4224, ctypes.byref(sz)) == OK
    assert sz.value >= 32 * 32 * 130 * 4        # 32 splits (256 blocks at most), (acc, m, l) per head
    assert lib.ttq_decode_attention_workspace_size(32, 8, 256, 4224, ctypes.byref(sz)) == UNSUPPORTED
    assert lib.ttq_decode_attention_workspace_size(48, 8, 128, 4224, ctypes.byref(sz)) == UNSUPPORTED  # 6 per kv
    assert lib.ttq_decode_attention_workspace_size(30, 8, 128, 4224, ctypes.byref(sz)) == INVALID
    att = lambda L, clen, pos=None, ws=d, wsb=1 << 20: (_p(a), 32, 8, 128, _p(b), _p(c), clen, L, pos, _p(d + 256),
                                                       _p(ws) if ws else None, wsb, None)
    assert lib.ttq_decode_attention(*att(0, 64)) == INVALID
    assert lib.ttq_decode_attention(*att(65, 64)) == INVALID
    assert lib.ttq_decode_attention(*att(10, 64, ws=None)) == WORKSPACE
    assert lib.ttq_decode_attention(*att(10, 64, wsb=16)) == WORKSPACE
    assert lib.ttq_decode_attention(*att(10, 64, pos=_p(d + 4))) == MISALIGNED
    assert lib.ttq_position_advance(None, 1, None) == INVALID
    assert lib.ttq_position_advance(_p(a + 4), 1, None) == MISALIGNED
    # SwiGLU gate
    assert lib.ttq_silu_mul(_p(a), 4, 12, _p(b), None) == INVALID
    assert lib.ttq_silu_mul(_p(a), 0, 16, _p(b), None) == INVALID
    assert lib.ttq_silu_mul(_p(a), 4, 16, _p(a), None) == INVALID
    assert lib.ttq_silu_mul(_p(a), 4, 16, _p(b + 2), None) == MISALIGNED


def test_binding_refuses_cpu_tensors(lib):
    torch = pytest.importorskip("torch")
    X = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ttq.act_stats(X, 0.5, 0.4, s=torch.zeros(64), ws=torch.zeros(1024, dtype=torch.uint8))
