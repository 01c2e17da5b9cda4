"""A stack of decoder layers whose linears run under TTQ: one prompt's prefill chained
through every layer (each layer's linears re-quantized from that layer's own
activations), then decode steps that reuse every layer's codes.

Shapes: the Qwen3 dense models of Table 15 in the thelatestinai.com listing of "TTQ:
Activation-Aware Test-Time Quantization ..." (``synthetic.QWEN3_SHAPES``). Each layer
has four TTQ linears: the stacked [Wq; Wk; Wv] (q, k and v read the same input, so one
statistic serves all three and stacking the rows changes no result), Wo, the stacked
[Wgate; Wup], and Wdown. With static low-rank factors a stacked linear carries
A = [A_1; A_2; ...] and the block-diagonal B, which gives every part its own term.

Between the linears run the library's kernels (``rmsnorm`` with the residual add,
``qk_norm_rope`` with the key/value cache write, ``silu_mul``, the prompt's causal
``prompt_attention`` on the tensor cores, and at decode ``decode_attention``). A decode step reads
its position from device memory and advances it on the device, so one captured CUDA graph
replays every step (``capture_decode``). There is no CPU path: every call raises when the
library is missing.
"""

from __future__ import annotations

import torch

import online_activation_aware_b200 as ttq

LINEARS = ("qkv", "o", "gate_up", "down")


class TTQDecoder:
    """Decoder stack over bf16 weights (one dict per layer: w_<lin>, optional a_<lin> and
    b_<lin>, n_in, n_post, n_q, n_k) with a key/value cache of ``max_len`` positions.

    ``prefill(x)`` takes the prompt's embeddings [T, hidden] (positions 0 .. T-1) and
    returns the final-normed hidden states; ``decode(x)`` takes the next token's
    embedding [1, hidden] and appends it at the following position. ``trace``, when
    given, is called as trace(layer, name, tensor) with every intermediate."""

    def __init__(self, shape: dict, weights: list, final_norm, q: int, g: int, alpha: float, lam: float,
                 r: int = 0, max_len: int = 4096 + 128, eps: float = 1e-6, rope_base: float = 1.0e6,
                 device="cuda"):
        self.shape = dict(shape)
        self.H, self.Hkv, self.D = shape["heads"], shape["kv_heads"], shape["head_dim"]
        self.hidden, self.inter = shape["hidden"], shape["inter"]
        if self.H % self.Hkv != 0:
            raise ValueError("heads must be a multiple of kv_heads")
        self.q, self.g, self.alpha, self.lam, self.r = q, g, alpha, lam, r
        self.eps, self.max_len, self.device = eps, max_len, device
        self.final_norm = final_norm
        self.layers = []
        for W in weights:
            L = {"norms": {k: W[k] for k in ("n_in", "n_post", "n_q", "n_k")}, "lin": {}}
            for name in LINEARS:
                A, B = W.get("a_" + name), W.get("b_" + name)
                rr = 0 if A is None else A.shape[0]
                L["lin"][name] = ttq.TTQLinear(W["w_" + name], q, g, alpha, lam, 2, rr, A, B)
            self.layers.append(L)
        n = len(self.layers)
        self.k_cache = torch.empty(n, max_len, self.Hkv, self.D, dtype=torch.bfloat16, device=device)
        self.v_cache = torch.empty_like(self.k_cache)
        self.table = ttq.rope_table(max_len, self.D, rope_base, device=device)
        self.length = 0
        self.pos = torch.zeros(1, dtype=torch.int64, device=device)   # next token's position
        self.attn_ws = torch.empty(ttq.decode_attention_workspace_size(self.H, self.Hkv, self.D, max_len),
                                   dtype=torch.uint8, device=device)
        self._ws = {}
        self._graph = None

    # -------------------------------------------------------------- buffers

    def workspace(self, T: int):
        """One scratch buffer shared by every linear of the stack (the largest need)."""
        if T not in self._ws:
            need = max(ttq.workspace_size(T, lin.d, lin.d_out, lin.cfg)
                       for L in self.layers for lin in L["lin"].values())
            self._ws[T] = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        return self._ws[T]

    # -------------------------------------------------------------- the stack

    def _attention(self, li: int, qkv, T: int, prefill: bool):
        H, D = self.H, self.D
        if not prefill:
            # one token at the device-held position, over the cache up to and including it
            return ttq.decode_attention(qkv, H, self.Hkv, D, self.k_cache[li], self.v_cache[li], pos_dev=self.pos,
                                        ws=self.attn_ws).view(1, H * D)
        return ttq.prompt_attention(qkv, H, self.Hkv, D, self.k_cache[li], self.v_cache[li])

    def _run(self, x, prefill: bool, trace=None):
        T = x.shape[0]
        if not prefill and T != 1:
            raise NotImplementedError("decode appends one token per call")
        if prefill and T > self.max_len:
            raise ValueError(f"{T} tokens exceed the cache of {self.max_len}")
        ws = self.workspace(T)
        r = x.clone()
        y = None
        for li, L in enumerate(self.layers):
            lin, nm = L["lin"], L["norms"]
            step = (lambda X, name: lin[name].prefill(X, ws=ws)) if prefill else \
                (lambda X, name: lin[name].decode(X, ws=ws))
            if y is None:
                h = ttq.rmsnorm(r, nm["n_in"], self.eps)
            else:
                h = ttq.rmsnorm(y, nm["n_in"], self.eps, residual=r)
            qkv = step(h, "qkv")
            if trace:
                trace(li, "r_in", r)
                trace(li, "h", h)
                trace(li, "qkv", qkv)
            ttq.qk_norm_rope(qkv, self.H, self.Hkv, self.D, nm["n_q"], nm["n_k"], self.eps, self.table, 0,
                             self.k_cache[li], self.v_cache[li], pos0_dev=None if prefill else self.pos)
            attn = self._attention(li, qkv, T, prefill)
            o = step(attn, "o")
            h2 = ttq.rmsnorm(o, nm["n_post"], self.eps, residual=r)
            gu = step(h2, "gate_up")
            m = ttq.silu_mul(gu)
            y = step(m, "down")
            if trace:
                trace(li, "q", qkv[:, : self.H * self.D])
                trace(li, "attn", attn)
                trace(li, "o", o)
                trace(li, "r_mid", r)
                trace(li, "h2", h2)
                trace(li, "gu", gu)
                trace(li, "m", m)
                trace(li, "down", y)
        out = ttq.rmsnorm(y, self.final_norm, self.eps, residual=r)
        if prefill:
            self.pos.fill_(T)
        else:
            ttq.position_advance(self.pos, 1)
        return out

    def prefill(self, x, trace=None):
        """Embeddings [T, hidden] bf16 of a new prompt -> final-normed hidden [T, hidden]."""
        out = self._run(x, True, trace)
        self.length = x.shape[0]
        return out

    def decode(self, x, trace=None):
        """Embedding [1, hidden] of the next token -> its final-normed hidden [1, hidden].
        Replays the captured step when ``capture_decode`` was called."""
        if self.length == 0:
            raise RuntimeError("decode needs a prefill first")
        if self.length + 1 > self.max_len:
            raise ValueError(f"position {self.length} is past the cache of {self.max_len}")
        if self._graph is not None and trace is None:
            self._x_static.copy_(x)
            self._graph.replay()
            out = self._out_static
        else:
            out = self._run(x, False, trace)
        self.length += 1
        return out

    def capture_decode(self):
        """Captures one decode step (all layers, the position advance included) in a CUDA
        graph; later ``decode`` calls replay it. Needs a prefill first (the capture runs the
        step once eagerly to set up its buffers, then restores the position)."""
        if self.length == 0:
            raise RuntimeError("capture_decode needs a prefill first")
        self._x_static = torch.zeros(1, self.hidden, dtype=torch.bfloat16, device=self.device)
        self.workspace(1)
        saved = self.pos.clone()
        self._run(self._x_static, False)            # eager warm-up: buffers, function attributes
        self.pos.copy_(saved)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._out_static = self._run(self._x_static, False)
        self.pos.copy_(saved)
        torch.cuda.synchronize()
        self._graph = g
        return g
