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
