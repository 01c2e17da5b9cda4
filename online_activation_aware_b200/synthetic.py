"""Seeded synthetic inputs for TTQ linear layers (shared by tests, bench and smoke).

This module only draws random numbers and rounds them to the bf16 storage format; it
holds none of the method's arithmetic. The distributions follow the workloads the
pages measure on (Qwen3/OPT projections with outlier-heavy activations):

  mag_j  ~ lognormal(0, 1) per input channel, 8 channels (drawn without replacement)
           scaled by 20 (activation outliers),
  X_tj   = Student-t(nu=3) * mag_j,
  W_ij   ~ Normal(0, 0.02^2),

drawn in exactly that order from ``numpy.random.default_rng(seed)``.
The layer shapes come from the architecture tables of the thelatestinai.com listing of
"TTQ: Activation-Aware Test-Time Quantization ..." (Tables 14 and 15).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def draw_layer(T: int, d: int, d_out: int, seed: int, n_outliers: int = 8,
               outlier_gain: float = 20.0):
    """Returns (X [T, d], W [d_out, d]) as float64 arrays (not yet rounded)."""
    rng = np.random.default_rng(seed)
    mag = rng.lognormal(0.0, 1.0, d)
    idx = rng.choice(d, min(n_outliers, d), replace=False)
    mag[idx] *= outlier_gain
    X = rng.standard_t(3, (T, d)) * mag[None, :]
    W = rng.normal(0.0, 0.02, (d_out, d))
    return X, W


def draw_tokens(b: int, d: int, seed: int, n_outliers: int = 8, outlier_gain: float = 20.0):
    """Decode-step activations [b, d] with the same per-channel magnitude recipe."""
    rng = np.random.default_rng(seed)
    mag = rng.lognormal(0.0, 1.0, d)
    idx = rng.choice(d, min(n_outliers, d), replace=False)
    mag[idx] *= outlier_gain
    return rng.standard_t(3, (b, d)) * mag[None, :]


def as_bf16(a):
    """Round an array to bf16 storage (round to nearest even, via torch's conversion).

    Returns a CPU ``torch.bfloat16`` tensor.
    """
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_values(t) -> np.ndarray:
    """The exact values of a bf16 tensor, as a float64 numpy array."""
    import torch

    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


@dataclass
class Linear:
    name: str
    d: int
    d_out: int


@dataclass
class Workload:
    """One measured configuration: a set of linear layers and the TTQ settings."""
    name: str
    layers: list
    T: int
    q: int
    g: int
    alpha: float
    lam: float
    r: int = 0
    p: int = 2
    seed: int = 0
    decode_batches: tuple = ()
    decode_steps: int = 0
    g_sweep: tuple = ()
    T_sweep: tuple = ()
    extra: dict = field(default_factory=dict)

    def layer_seed(self, idx: int) -> int:
        return 1000 * self.seed + idx if len(self.layers) > 1 else self.seed


def _qwen3_8b_layer():
    return [Linear("q_proj", 4096, 4096), Linear("k_proj", 4096, 1024),
            Linear("v_proj", 4096, 1024), Linear("o_proj", 4096, 4096),
            Linear("gate_proj", 4096, 12288), Linear("up_proj", 4096, 12288),
            Linear("down_proj", 12288, 4096)]


WORKLOADS = {
    # single 512 -> 512 layer, small enough for the oracle to finish in seconds
    "single_512": Workload("single_512", [Linear("linear", 512, 512)], T=128, q=3, g=32,
                           alpha=0.5, lam=0.4, seed=0),
    # OPT-125M-shaped layer set (hidden 768, MLP 3072)
    "opt125m_set": Workload("opt125m_set",
                            [Linear("q_proj", 768, 768), Linear("k_proj", 768, 768),
                             Linear("v_proj", 768, 768), Linear("out_proj", 768, 768),
                             Linear("fc1", 768, 3072), Linear("fc2", 3072, 768)],
                            T=2048, q=4, g=32, alpha=0.5, lam=0.4, seed=1),
    # Qwen3-1.7B-shaped layers (hidden 2048, 8 KV heads of 128, MLP 6144)
    "qwen3_1p7b_set": Workload("qwen3_1p7b_set",
                               [Linear("q_proj", 2048, 2048), Linear("k_proj", 2048, 1024),
                                Linear("v_proj", 2048, 1024), Linear("gate_proj", 2048, 6144),
                                Linear("up_proj", 2048, 6144), Linear("down_proj", 6144, 2048)],
                               T=4096, q=3, g=32, alpha=0.75, lam=0.4, r=16, seed=2,
                               g_sweep=(32, 64, 128)),
    # Qwen3-32B query projection 5120 -> 8192 (64 heads of 128)
    "qwen3_32b_qproj": Workload("qwen3_32b_qproj", [Linear("q_proj", 5120, 8192)], T=4096,
                                q=4, g=128, alpha=0.5, lam=0.4, r=0, seed=3,
                                decode_batches=(1, 8, 64), decode_steps=256,
                                T_sweep=(16, 128, 1024, 4096, 16384)),
    # Qwen3-8B-shaped stack: 36 layers x 7 linears, every one through TTQ
    "qwen3_8b_stack": Workload("qwen3_8b_stack", _qwen3_8b_layer(), T=4096, q=2, g=32,
                               alpha=0.5, lam=0.4, r=16, seed=4, decode_batches=(1,),
                               decode_steps=128, extra={"layers": 36}),
}


# ------------------------------------------------------------------ decoder stacks

# Qwen3 dense models (Table 15 of the thelatestinai.com listing): layers, heads, KV heads,
# hidden size, head dim, MLP dim.
QWEN3_SHAPES = {
    "0.6B": dict(layers=28, heads=16, kv_heads=8, hidden=1024, head_dim=128, inter=3072),
    "1.7B": dict(layers=28, heads=16, kv_heads=8, hidden=2048, head_dim=128, inter=6144),
    "4B": dict(layers=36, heads=32, kv_heads=8, hidden=2560, head_dim=128, inter=9728),
    "8B": dict(layers=36, heads=32, kv_heads=8, hidden=4096, head_dim=128, inter=12288),
    "14B": dict(layers=40, heads=40, kv_heads=8, hidden=5120, head_dim=128, inter=17408),
    "32B": dict(layers=64, heads=64, kv_heads=8, hidden=5120, head_dim=128, inter=25600),
}

# the four TTQ linears of a decoder layer (q|k|v and gate|up each stacked into one)
DECODER_LINEARS = ("qkv", "o", "gate_up", "down")


def decoder_linear_parts(shape: dict, name: str):
    """Output rows of the parts stacked in one decoder linear, and its input width."""
    H, Hkv, D, h, I = shape["heads"], shape["kv_heads"], shape["head_dim"], shape["hidden"], shape["inter"]
    return {"qkv": ([H * D, Hkv * D, Hkv * D], h), "o": ([h], H * D), "gate_up": ([I, I], h),
            "down": ([h], I)}[name]


def draw_decoder_weights(shape: dict, r: int, seed: int, layers: int | None = None):
    """Random-init weights of a decoder stack, float64 numpy (not yet rounded), one dict
    per layer: w_<lin> [rows, in] ~ N(0, 1/in) with the parts of a stacked linear one
    after another; norm weights 1 + N(0, 0.1^2); with r > 0 the static low-rank factors of
    every part, a ~ N(0, 0.02^2) [r, in] and b ~ N(0, 0.02^2) [rows, r], stacked as
    a_<lin> [parts r, in] and the block-diagonal b_<lin> [rows, parts r] (zeros off the
    blocks), and w_<lin> standing for the residual R."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(layers if layers is not None else shape["layers"]):
        L = {}
        for name in DECODER_LINEARS:
            parts, d_in = decoder_linear_parts(shape, name)
            L["w_" + name] = rng.normal(0.0, d_in ** -0.5, (sum(parts), d_in))
            if r > 0:
                L["a_" + name] = rng.normal(0.0, 0.02, (len(parts) * r, d_in))
                b = np.zeros((sum(parts), len(parts) * r))
                row = 0
                for i, n in enumerate(parts):
                    b[row: row + n, i * r: (i + 1) * r] = rng.normal(0.0, 0.02, (n, r))
                    row += n
                L["b_" + name] = b
        for name, n in (("n_in", shape["hidden"]), ("n_post", shape["hidden"]), ("n_q", shape["head_dim"]),
                        ("n_k", shape["head_dim"])):
            L[name] = 1.0 + 0.1 * rng.normal(size=n)
        out.append(L)
    return out


def draw_hidden(T: int, hidden: int, seed: int):
    """Token embeddings entering the stack [T, hidden] ~ N(0, 1) (float64)."""
    return np.random.default_rng(seed).normal(size=(T, hidden))


def device_decoder_weights(shape: dict, r: int, seed: int, device="cuda", layers: int | None = None):
    """The same recipe drawn on the device (torch's seeded CUDA generator; different numbers
    from the numpy draw), bf16 tensors: for stacks too large to draw on the host."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def normal(rows, cols, std):
        t = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
        t.normal_(0.0, std, generator=gen)
        return t

    out = []
    for _ in range(layers if layers is not None else shape["layers"]):
        L = {}
        for name in DECODER_LINEARS:
            parts, d_in = decoder_linear_parts(shape, name)
            L["w_" + name] = normal(sum(parts), d_in, d_in ** -0.5)
            if r > 0:
                L["a_" + name] = normal(len(parts) * r, d_in, 0.02)
                b = torch.zeros(sum(parts), len(parts) * r, dtype=torch.bfloat16, device=device)
                row = 0
                for i, n in enumerate(parts):
                    b[row: row + n, i * r: (i + 1) * r] = normal(n, r, 0.02)
                    row += n
                L["b_" + name] = b
        for name, n in (("n_in", shape["hidden"]), ("n_post", shape["hidden"]), ("n_q", shape["head_dim"]),
                        ("n_k", shape["head_dim"])):
            L[name] = (1.0 + 0.1 * normal(1, n, 1.0).float()).to(torch.bfloat16).reshape(n)
        out.append(L)
    return out
