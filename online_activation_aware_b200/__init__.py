"""TTQ (activation-aware test-time quantization) on NVIDIA B200: Python binding.

A thin ctypes layer over ``libttq.so`` (C ABI in ``include/ttq.h``). Every function
here only checks and marshals its arguments (torch CUDA tensors -> device pointers,
the current CUDA stream) and calls the library; all arithmetic of the hot path runs
in the library's CUDA kernels. There is no CPU fallback: when the library is missing
or a call fails, a ``TTQError`` is raised.

Functions keep the C names without the ``ttq_`` prefix:
``act_stats``, ``requant``, ``requant_batched``, ``linear_prefill``, ``linear_prefill_batched``,
``linear_decode``, ``linear_decode_batched``, ``workspace_size``,
``codes_words``, ``device_status``, ``set_wait_limit_ns``, and the decoder-layer kernels
``rmsnorm``, ``rope_table``, ``qk_norm_rope``, ``silu_mul``, ``prompt_attention``,
``decode_attention``, ``position_advance``. ``TTQLinear`` bundles one
layer's weight and the per-prompt buffers (prefill, then decode reusing the codes);
``online_activation_aware_b200.decoder`` chains them into a decoder stack.
"""

from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libttq.so")

STATUS = {0: "TTQ_OK", -1: "TTQ_ERR_INVALID_ARG", -2: "TTQ_ERR_UNSUPPORTED", -3: "TTQ_ERR_MISALIGNED",
          -4: "TTQ_ERR_WORKSPACE", -5: "TTQ_ERR_CUDA", -6: "TTQ_ERR_TIMEOUT", -7: "TTQ_ERR_TOO_LARGE"}


class TTQError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}{detail}")


class Config(ctypes.Structure):
    """Mirror of ``ttq_config``."""
    _fields_ = [("q", ctypes.c_int32), ("g", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("lambda_", ctypes.c_float), ("p", ctypes.c_int32), ("r", ctypes.c_int32)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libttq.so (once). Raises TTQError-compatible RuntimeError when it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m online_activation_aware_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    cfgp = ctypes.POINTER(Config)
    lib.ttq_codes_words.argtypes = [i64, i64, i32]
    lib.ttq_codes_words.restype = sz
    lib.ttq_workspace_size.argtypes = [i64, i64, i64, cfgp, ctypes.POINTER(sz)]
    lib.ttq_workspace_size.restype = i32
    lib.ttq_workspace_folded_offset.argtypes = [i64, i64, i64, cfgp, ctypes.POINTER(sz)]
    lib.ttq_workspace_folded_offset.restype = i32
    lib.ttq_act_stats.argtypes = [vp, i64, i64, i64, f32, f32, i32, vp, vp, sz, vp]
    lib.ttq_act_stats.restype = i32
    lib.ttq_act_stats_noalloc.argtypes = [vp, i64, i64, i64, f32, f32, i32, vp, vp]
    lib.ttq_act_stats_noalloc.restype = i32
    lib.ttq_requant.argtypes = [vp, i64, i64, vp, i32, i32, vp, vp, vp, vp]
    lib.ttq_requant.restype = i32
    lib.ttq_requant_batched.argtypes = [vp, i64, i64, vp, i32, i32, i32, vp, vp, vp, vp]
    lib.ttq_requant_batched.restype = i32
    lib.ttq_linear_prefill.argtypes = [vp, i64, i64, vp, i64, vp, vp, cfgp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.ttq_linear_prefill.restype = i32
    lib.ttq_linear_decode.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, cfgp, vp, vp, sz, vp]
    lib.ttq_linear_decode.restype = i32
    i64p = ctypes.POINTER(i64)
    lib.ttq_prefill_batched_workspace_size.argtypes = [i64p, i32, i64, i64, cfgp, ctypes.POINTER(sz)]
    lib.ttq_prefill_batched_workspace_size.restype = i32
    lib.ttq_linear_prefill_batched.argtypes = [vp, i64p, i32, i64, vp, i64, vp, vp, cfgp, vp, vp, vp, vp, vp, vp, sz,
                                               vp]
    lib.ttq_linear_prefill_batched.restype = i32
    lib.ttq_decode_batched_workspace_size.argtypes = [i32, i64, i64, i64, cfgp, ctypes.POINTER(sz)]
    lib.ttq_decode_batched_workspace_size.restype = i32
    lib.ttq_linear_decode_batched.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, vp, vp, cfgp, vp, vp, sz, vp]
    lib.ttq_linear_decode_batched.restype = i32
    lib.ttq_rmsnorm.argtypes = [vp, vp, vp, i64, i64, f32, vp, vp]
    lib.ttq_rmsnorm.restype = i32
    lib.ttq_rope_table.argtypes = [i64, i64, ctypes.c_double, vp, vp]
    lib.ttq_rope_table.restype = i32
    lib.ttq_qk_norm_rope.argtypes = [vp, i64, i64, i64, i64, vp, vp, f32, vp, i64, i64, vp, vp, vp, i64, vp]
    lib.ttq_qk_norm_rope.restype = i32
    lib.ttq_decode_attention_workspace_size.argtypes = [i64, i64, i64, i64, ctypes.POINTER(sz)]
    lib.ttq_decode_attention_workspace_size.restype = i32
    lib.ttq_decode_attention.argtypes = [vp, i64, i64, i64, vp, vp, i64, i64, vp, vp, vp, sz, vp]
    lib.ttq_decode_attention.restype = i32
    lib.ttq_prompt_attention.argtypes = [vp, i64, i64, i64, i64, vp, vp, i64, vp, vp]
    lib.ttq_prompt_attention.restype = i32
    lib.ttq_position_advance.argtypes = [vp, i64, vp]
    lib.ttq_position_advance.restype = i32
    lib.ttq_silu_mul.argtypes = [vp, i64, i64, vp, vp]
    lib.ttq_silu_mul.restype = i32
    lib.ttq_device_status.argtypes = [vp]
    lib.ttq_device_status.restype = i32
    lib.ttq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.ttq_set_wait_limit_ns.restype = i32
    lib.ttq_last_cuda_error.argtypes = []
    lib.ttq_last_cuda_error.restype = i32
    lib.ttq_cuda_error_string.argtypes = [i32]
    lib.ttq_cuda_error_string.restype = ctypes.c_char_p
    lib.ttq_debug_inject_stall.argtypes = [i32]
    lib.ttq_debug_inject_stall.restype = i32
    lib.ttq_set_trace_events.argtypes = [ctypes.POINTER(vp), i32]
    lib.ttq_set_trace_events.restype = i32
    lib.ttq_status_string.argtypes = [i32]
    lib.ttq_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != 0:
        detail = ""
        if status == -5 and _lib is not None:
            code = int(_lib.ttq_last_cuda_error())
            detail = f" (cuda error {code}: {_lib.ttq_cuda_error_string(code).decode()})"
        raise TTQError(fn, status, detail)


def _ptr(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_config(q: int, g: int, alpha: float, lam: float, p: int = 2, r: int = 0) -> Config:
    return Config(int(q), int(g), float(alpha), float(lam), int(p), int(r))


def codes_words(d_out: int, d: int, q: int) -> int:
    return int(load_library().ttq_codes_words(d_out, d, q))


def workspace_size(T: int, d: int, d_out: int, cfg: Config | None = None) -> int:
    n = ctypes.c_size_t(0)
    _check("ttq_workspace_size",
           load_library().ttq_workspace_size(T, d, d_out, ctypes.byref(cfg) if cfg is not None else None,
                                             ctypes.byref(n)))
    return int(n.value)


def workspace_folded_offset(T: int, d: int, d_out: int, cfg: Config) -> int:
    """Byte offset of the folded activations X diag(1/s) (bf16 [T, d]) in the workspace of
    a prefill (or of a decode of more than 2 rows) with these sizes."""
    n = ctypes.c_size_t(0)
    _check("ttq_workspace_folded_offset",
           load_library().ttq_workspace_folded_offset(T, d, d_out, ctypes.byref(cfg), ctypes.byref(n)))
    return int(n.value)


def alloc_workspace(T: int, d: int, d_out: int, cfg: Config | None = None, device="cuda"):
    import torch

    return torch.empty(max(workspace_size(T, d, d_out, cfg), 256), dtype=torch.uint8, device=device)


def act_stats(X, alpha: float, lam: float, p: int = 2, s=None, ws=None, stream=None):
    """s = (mean over tokens of |X|^p + lambda)^(alpha/p) per input channel; X [T, d] bf16."""
    import torch

    T, d = X.shape
    if s is None:
        s = torch.empty(d, dtype=torch.float32, device=X.device)
    if ws is None and workspace_size(T, d, 0) > 0:
        ws = alloc_workspace(T, d, 0, None, X.device)
    _check("ttq_act_stats", load_library().ttq_act_stats(
        _ptr(X, torch.bfloat16, "X"), T, d, X.stride(0), alpha, lam, p, _ptr(s, torch.float32, "s"),
        _ptr(ws, None, "ws"), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))
    return s


def requant(W, s, q: int, g: int, codes=None, scale=None, zero=None, stream=None):
    """Packed codes, fp16 scale and fp16 zero of Q[W diag(s)]; W [d_out, d] bf16."""
    import torch

    d_out, d = W.shape
    dev = W.device
    if codes is None:
        codes = torch.empty(codes_words(d_out, d, q), dtype=torch.int32, device=dev)
    if scale is None:
        scale = torch.empty(d_out, d // g, dtype=torch.float16, device=dev)
    if zero is None:
        zero = torch.empty(d_out, d // g, dtype=torch.float16, device=dev)
    _check("ttq_requant", load_library().ttq_requant(
        _ptr(W, torch.bfloat16, "W"), d_out, d, _ptr(s, torch.float32, "s"), q, g,
        _ptr(codes, torch.int32, "codes"), _ptr(scale, torch.float16, "scale"),
        _ptr(zero, torch.float16, "zero"), _stream(stream)))
    return codes, scale, zero


def requant_batched(W, S, q: int, g: int, codes=None, scale=None, zero=None, stream=None):
    """Codes, scale and zero of Q[W diag(s_p)] for P prompts from one read of W.

    W [d_out, d] bf16; S [P, d] fp32 (P = 1 .. 8). Returns (codes [P, words] int32,
    scale [P, d_out, d/g] fp16, zero [P, d_out, d/g] fp16)."""
    import torch

    d_out, d = W.shape
    P = S.shape[0]
    dev = W.device
    if codes is None:
        codes = torch.empty(P, codes_words(d_out, d, q), dtype=torch.int32, device=dev)
    if scale is None:
        scale = torch.empty(P, d_out, d // g, dtype=torch.float16, device=dev)
    if zero is None:
        zero = torch.empty(P, d_out, d // g, dtype=torch.float16, device=dev)
    _check("ttq_requant_batched", load_library().ttq_requant_batched(
        _ptr(W, torch.bfloat16, "W"), d_out, d, _ptr(S, torch.float32, "S"), P, q, g,
        _ptr(codes, torch.int32, "codes"), _ptr(scale, torch.float16, "scale"),
        _ptr(zero, torch.float16, "zero"), _stream(stream)))
    return codes, scale, zero


def linear_prefill(X, W, cfg: Config, A=None, B=None, out=None, ws=None, stream=None):
    """One prompt through a TTQ linear layer. Returns dict(s, codes, scale, zero, Y)."""
    import torch

    T, d = X.shape
    d_out = W.shape[0]
    dev = X.device
    o = out or {}
    s = o.get("s") if o.get("s") is not None else torch.empty(d, dtype=torch.float32, device=dev)
    codes = o.get("codes") if o.get("codes") is not None else torch.empty(
        codes_words(d_out, d, cfg.q), dtype=torch.int32, device=dev)
    scale = o.get("scale") if o.get("scale") is not None else torch.empty(
        d_out, d // cfg.g, dtype=torch.float16, device=dev)
    zero = o.get("zero") if o.get("zero") is not None else torch.empty(
        d_out, d // cfg.g, dtype=torch.float16, device=dev)
    Y = o.get("Y") if o.get("Y") is not None else torch.empty(T, d_out, dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = alloc_workspace(T, d, d_out, cfg, dev)
    _check("ttq_linear_prefill", load_library().ttq_linear_prefill(
        _ptr(X, torch.bfloat16, "X"), T, d, _ptr(W, torch.bfloat16, "W"), d_out,
        _ptr(A, torch.bfloat16, "A"), _ptr(B, torch.bfloat16, "B"), ctypes.byref(cfg),
        _ptr(s, torch.float32, "s"), _ptr(codes, torch.int32, "codes"), _ptr(scale, torch.float16, "scale"),
        _ptr(zero, torch.float16, "zero"), _ptr(Y, torch.bfloat16, "Y"), _ptr(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))
    return {"s": s, "codes": codes, "scale": scale, "zero": zero, "Y": Y}


def linear_decode(X, s, codes, scale, zero, cfg: Config, d_out: int, A=None, B=None, Y=None, ws=None,
                  stream=None):
    """Y = (X diag(1/s)) deq(codes)^T (+ (X A^T) B^T) for b token rows, reusing a prefill's codes."""
    import torch

    b, d = X.shape
    dev = X.device
    if Y is None:
        Y = torch.empty(b, d_out, dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = alloc_workspace(b, d, d_out, cfg, dev)
    _check("ttq_linear_decode", load_library().ttq_linear_decode(
        _ptr(X, torch.bfloat16, "X"), b, d, d_out, _ptr(s, torch.float32, "s"),
        _ptr(codes, torch.int32, "codes"), _ptr(scale, torch.float16, "scale"),
        _ptr(zero, torch.float16, "zero"), _ptr(A, torch.bfloat16, "A"), _ptr(B, torch.bfloat16, "B"),
        ctypes.byref(cfg), _ptr(Y, torch.bfloat16, "Y"), _ptr(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))
    return Y


def linear_prefill_batched(X, T, W, cfg: Config, A=None, B=None, ws=None, stream=None):
    """P prompts (token counts T, their tokens stacked in X [sum T, d]) through one layer,
    each with its own statistic and codes. Returns dict(s [P, d], codes [P, words],
    scale / zero [P, d_out, d/g], Y [sum T, d_out])."""
    import torch

    Tl = [int(t) for t in T]
    P = len(Tl)
    d = X.shape[1]
    d_out = W.shape[0]
    dev = X.device
    Ta = (ctypes.c_int64 * P)(*Tl)
    s = torch.empty(P, d, dtype=torch.float32, device=dev)
    codes = torch.empty(P, codes_words(d_out, d, cfg.q), dtype=torch.int32, device=dev)
    scale = torch.empty(P, d_out, d // cfg.g, dtype=torch.float16, device=dev)
    zero = torch.empty(P, d_out, d // cfg.g, dtype=torch.float16, device=dev)
    Y = torch.empty(sum(Tl), d_out, dtype=torch.bfloat16, device=dev)
    if ws is None:
        n = ctypes.c_size_t(0)
        _check("ttq_prefill_batched_workspace_size", load_library().ttq_prefill_batched_workspace_size(
            Ta, P, d, d_out, ctypes.byref(cfg), ctypes.byref(n)))
        ws = torch.empty(max(int(n.value), 256), dtype=torch.uint8, device=dev)
    _check("ttq_linear_prefill_batched", load_library().ttq_linear_prefill_batched(
        _ptr(X, torch.bfloat16, "X"), Ta, P, d, _ptr(W, torch.bfloat16, "W"), d_out,
        _ptr(A, torch.bfloat16, "A"), _ptr(B, torch.bfloat16, "B"), ctypes.byref(cfg),
        _ptr(s, torch.float32, "s"), _ptr(codes, torch.int32, "codes"), _ptr(scale, torch.float16, "scale"),
        _ptr(zero, torch.float16, "zero"), _ptr(Y, torch.bfloat16, "Y"), _ptr(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))
    return {"s": s, "codes": codes, "scale": scale, "zero": zero, "Y": Y}


def linear_decode_batched(X, s, codes, scale, zero, cfg: Config, d_out: int, A=None, B=None, Y=None, ws=None,
                          stream=None):
    """Decode steps of P requests at once, each with its own prefill's s, codes, scale
    and zero: X [P, b, d], s [P, d], codes [P, words], scale / zero [P, d_out, d/g];
    returns Y [P, b, d_out]."""
    import torch

    P, b, d = X.shape
    dev = X.device
    if Y is None:
        Y = torch.empty(P, b, d_out, dtype=torch.bfloat16, device=dev)
    if ws is None:
        n = ctypes.c_size_t(0)
        _check("ttq_decode_batched_workspace_size", load_library().ttq_decode_batched_workspace_size(
            P, b, d, d_out, ctypes.byref(cfg), ctypes.byref(n)))
        ws = torch.empty(max(int(n.value), 256), dtype=torch.uint8, device=dev)
    _check("ttq_linear_decode_batched", load_library().ttq_linear_decode_batched(
        _ptr(X, torch.bfloat16, "X"), P, b, d, d_out, _ptr(s, torch.float32, "s"),
        _ptr(codes, torch.int32, "codes"), _ptr(scale, torch.float16, "scale"),
        _ptr(zero, torch.float16, "zero"), _ptr(A, torch.bfloat16, "A"), _ptr(B, torch.bfloat16, "B"),
        ctypes.byref(cfg), _ptr(Y, torch.bfloat16, "Y"), _ptr(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))
    return Y


def device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the library's device error status."""
    return int(load_library().ttq_device_status(_stream(stream)))


def debug_inject_stall(enable: bool):
    """Test hook: makes the tensor-core kernel wait on a barrier nothing arrives at."""
    _check("ttq_debug_inject_stall", load_library().ttq_debug_inject_stall(1 if enable else 0))


def set_wait_limit_ns(ns: int):
    _check("ttq_set_wait_limit_ns", load_library().ttq_set_wait_limit_ns(int(ns)))


def set_trace_events(events):
    """Records stage boundaries of every later linear_prefill on these CUDA events
    (a list of 6 ``torch.cuda.Event(enable_timing=True)``), or stops when None."""
    lib = load_library()
    if not events:
        _check("ttq_set_trace_events", lib.ttq_set_trace_events(None, 0))
        return
    handles = []
    for ev in events:
        if ev.cuda_event == 0:  # torch creates the event lazily
            ev.record()
        handles.append(ev.cuda_event)
    arr = (ctypes.c_void_p * len(handles))(*handles)
    set_trace_events._keep = (arr, events)
    _check("ttq_set_trace_events", lib.ttq_set_trace_events(arr, len(handles)))


class TTQLinear:
    """One linear layer under TTQ: holds the bf16 weight (or residual R and the static
    factors A, B when r > 0) and, after ``prefill``, the prompt's s and packed codes that
    ``decode`` reuses."""

    def __init__(self, W, q: int, g: int, alpha: float, lam: float, p: int = 2, r: int = 0,
                 A=None, B=None):
        import torch

        self.cfg = make_config(q, g, alpha, lam, p, r)
        self.W = W
        self.A = A
        self.B = B
        self.d_out, self.d = W.shape
        dev = W.device
        self.s = torch.empty(self.d, dtype=torch.float32, device=dev)
        self.codes = torch.empty(codes_words(self.d_out, self.d, q), dtype=torch.int32, device=dev)
        self.scale = torch.empty(self.d_out, self.d // g, dtype=torch.float16, device=dev)
        self.zero = torch.empty(self.d_out, self.d // g, dtype=torch.float16, device=dev)
        self._ws = {}

    def workspace(self, T: int):
        if T not in self._ws:
            self._ws[T] = alloc_workspace(T, self.d, self.d_out, self.cfg, self.W.device)
        return self._ws[T]

    def prefill(self, X, Y=None, ws=None, stream=None):
        """Statistic, re-quantization and projection of one prompt X [T, d]; keeps s and the
        codes for ``decode``. ``ws`` (optional) is a scratch buffer of at least
        workspace_size(T, d, d_out, cfg) bytes shared with other layers."""
        out = {"s": self.s, "codes": self.codes, "scale": self.scale, "zero": self.zero, "Y": Y}
        ws = ws if ws is not None else self.workspace(X.shape[0])
        return linear_prefill(X, self.W, self.cfg, self.A, self.B, out=out, ws=ws, stream=stream)["Y"]

    def decode(self, X, Y=None, ws=None, stream=None):
        """Y for new tokens X [b, d] with the last prefill's s and codes."""
        ws = ws if ws is not None else self.workspace(X.shape[0])
        return linear_decode(X, self.s, self.codes, self.scale, self.zero, self.cfg, self.d_out, self.A,
                             self.B, Y=Y, ws=ws, stream=stream)


# ------------------------------------------------------------------ decoder-layer kernels


def rmsnorm(y, w, eps: float, residual=None, out=None, stream=None):
    """out = bf16(h w / rms(h)) per row, h = y, or h = r <- bf16(r + y) when ``residual``
    (updated in place) is given."""
    import torch

    rows, n = y.shape
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=y.device)
    _check("ttq_rmsnorm", load_library().ttq_rmsnorm(
        _ptr(y, torch.bfloat16, "y"), _ptr(residual, torch.bfloat16, "residual"), _ptr(w, torch.bfloat16, "w"),
        rows, n, ctypes.c_float(eps), _ptr(out, torch.bfloat16, "out"), _stream(stream)))
    return out


def rope_table(positions: int, head_dim: int, base: float, device="cuda", stream=None):
    """fp32 [positions, head_dim/2, 2] (cos, sin) of pos * base^(-2i/head_dim)."""
    import torch

    table = torch.empty(positions, head_dim // 2, 2, dtype=torch.float32, device=device)
    _check("ttq_rope_table", load_library().ttq_rope_table(positions, head_dim, ctypes.c_double(base),
                                                           _ptr(table, torch.float32, "table"), _stream(stream)))
    return table


def qk_norm_rope(qkv, heads: int, kv_heads: int, head_dim: int, q_norm, k_norm, eps: float, table, pos0: int,
                 k_cache, v_cache, pos0_dev=None, stream=None):
    """q heads of the stacked projection normalised and rotated in place; k (normalised,
    rotated) and v written to the caches at positions pos0 .. pos0 + T - 1 (pos0 read from
    the device int64 tensor ``pos0_dev`` when given)."""
    import torch

    T = qkv.shape[0]
    _check("ttq_qk_norm_rope", load_library().ttq_qk_norm_rope(
        _ptr(qkv, torch.bfloat16, "qkv"), T, heads, kv_heads, head_dim, _ptr(q_norm, torch.bfloat16, "q_norm"),
        _ptr(k_norm, torch.bfloat16, "k_norm"), ctypes.c_float(eps), _ptr(table, torch.float32, "table"),
        table.shape[0], pos0, _ptr(pos0_dev, torch.int64, "pos0_dev"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0], _stream(stream)))
    return qkv


def decode_attention_workspace_size(heads: int, kv_heads: int, head_dim: int, cache_len: int) -> int:
    n = ctypes.c_size_t(0)
    _check("ttq_decode_attention_workspace_size", load_library().ttq_decode_attention_workspace_size(
        heads, kv_heads, head_dim, cache_len, ctypes.byref(n)))
    return int(n.value)


def decode_attention(q, heads: int, kv_heads: int, head_dim: int, k_cache, v_cache, length: int = 0, pos_dev=None,
                     out=None, ws=None, stream=None):
    """One token's attention over the first L cache rows (L = length, or pos_dev + 1 read
    on the device). q [heads * head_dim] bf16 (any tensor whose first heads * head_dim
    elements are the token's q heads); returns out [heads * head_dim] bf16."""
    import torch

    L = k_cache.shape[0]
    if out is None:
        out = torch.empty(heads * head_dim, dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = torch.empty(decode_attention_workspace_size(heads, kv_heads, head_dim, L), dtype=torch.uint8,
                         device=q.device)
    _check("ttq_decode_attention", load_library().ttq_decode_attention(
        _ptr(q, torch.bfloat16, "q"), heads, kv_heads, head_dim, _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), L, length, _ptr(pos_dev, torch.int64, "pos_dev"),
        _ptr(out, torch.bfloat16, "out"), _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)))
    return out


def prompt_attention(qkv, heads: int, kv_heads: int, head_dim: int, k_cache, v_cache, out=None, stream=None):
    """Causal grouped-query attention of a prompt at positions 0 .. T-1 (q from the stacked
    projection qkv [T, ...], k and v from the caches' first T positions); returns
    out [T, heads * head_dim] bf16."""
    import torch

    T = qkv.shape[0]
    if out is None:
        out = torch.empty(T, heads * head_dim, dtype=torch.bfloat16, device=qkv.device)
    _check("ttq_prompt_attention", load_library().ttq_prompt_attention(
        _ptr(qkv, torch.bfloat16, "qkv"), T, heads, kv_heads, head_dim, _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0], _ptr(out, torch.bfloat16, "out"),
        _stream(stream)))
    return out


def position_advance(pos_dev, n: int = 1, stream=None):
    """pos_dev += n on the device, in stream order."""
    import torch

    _check("ttq_position_advance", load_library().ttq_position_advance(_ptr(pos_dev, torch.int64, "pos_dev"), n,
                                                                       _stream(stream)))


def silu_mul(gate_up, out=None, stream=None):
    """out = bf16(silu(gate) * up) with gate_up = [gate | up] along the channels."""
    import torch

    rows, two_i = gate_up.shape
    inter = two_i // 2
    if out is None:
        out = torch.empty(rows, inter, dtype=torch.bfloat16, device=gate_up.device)
    _check("ttq_silu_mul", load_library().ttq_silu_mul(
        _ptr(gate_up, torch.bfloat16, "gate_up"), rows, inter, _ptr(out, torch.bfloat16, "out"), _stream(stream)))
    return out
