"""Seeded synthetic inputs for DBF layers.

This module only draws numbers: sign matrices, fp16 scale vectors and fp16
activations with the shapes and value distributions of the workloads below.
It holds none of the method's arithmetic, so both the fp64 oracle (``oracle/``)
and the CUDA path (``binary_factorized_weight_b200``) may consume it without
sharing any computation.

Workloads (shapes of Llama-2-7B / Llama-3-8B projections, the models the
"Addition is almost all you need" pages evaluate DBF on, section 4 of the
gist.science technical summary; no weights are available, so signs and scales
are random):

* ``tiny``      n = m_in = 256, k = 128 (1 bit/weight); a, mid, b = |N(0,1)| + 0.1
* ``tiny_int``  same shape; a = mid = b = 1, x uniform integers in [-8, 8]
* ``attn_1b``   4096 x 4096, k = 2048 (1.0 bit/weight); lognormal(-3, 0.5) scales
* ``attn_2b``   4096 x 4096, k = 4096 (2.0 bits/weight)
* ``mlp_up``    m_in = 4096 -> n = 14336, k = 4736 (~1.49 bits/weight)
* ``layer_set`` the seven projections of one decoder layer, at 1 and 2 bits/weight

Seeds: ``default_rng(1000 * config_index + rotation)``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "LayerShape",
    "CONFIGS",
    "LAYER_SET",
    "rng_for",
    "sign_matrix",
    "abs_normal_scales",
    "lognormal_scales",
    "unit_scales",
    "normal_activations",
    "integer_activations",
    "sylvester_hadamard",
    "projection_signs",
    "make_layer",
]


@dataclass(frozen=True)
class LayerShape:
    """Shape and value recipe of one synthetic DBF layer."""

    name: str
    index: int  # config index used in the seed
    n: int  # outputs (rows of A)
    k: int  # middle dimension (cols of A, rows of B)
    m_in: int  # inputs (cols of B)
    scales: str  # "absnormal" | "lognormal" | "unit"
    x: str  # "normal" | "int"
    batches: tuple = field(default=(1,))


CONFIGS = {
    "tiny": LayerShape("tiny", 0, 256, 128, 256, "absnormal", "normal", (1, 4)),
    "tiny_int": LayerShape("tiny_int", 0, 256, 128, 256, "unit", "int", (1, 4, 128, 2048)),
    "attn_1b": LayerShape("attn_1b", 1, 4096, 2048, 4096, "lognormal", "normal", (1,)),
    "attn_2b": LayerShape("attn_2b", 2, 4096, 4096, 4096, "lognormal", "normal", (1, 4, 16)),
    "mlp_up": LayerShape("mlp_up", 3, 14336, 4736, 4096, "lognormal", "normal", (1, 2048)),
}

# One Llama-3-8B-shaped decoder layer (GQA: k/v project 4096 -> 1024).  The
# middle dimension k is the 1 and 2 bits/weight value of k(n+m_in)/(n*m_in)
# rounded to the nearest multiple of 64 (ties up).
LAYER_SET = {
    1: [
        LayerShape("q_1b", 4, 4096, 2048, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("k_1b", 4, 1024, 832, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("v_1b", 4, 1024, 832, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("o_1b", 4, 4096, 2048, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("gate_1b", 4, 14336, 3200, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("up_1b", 4, 14336, 3200, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("down_1b", 4, 4096, 3200, 14336, "lognormal", "normal", (1, 16, 128, 2048)),
    ],
    2: [
        LayerShape("q_2b", 4, 4096, 4096, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("k_2b", 4, 1024, 1664, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("v_2b", 4, 1024, 1664, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("o_2b", 4, 4096, 4096, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("gate_2b", 4, 14336, 6400, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("up_2b", 4, 14336, 6400, 4096, "lognormal", "normal", (1, 16, 128, 2048)),
        LayerShape("down_2b", 4, 4096, 6400, 14336, "lognormal", "normal", (1, 16, 128, 2048)),
    ],
}


def rng_for(config_index: int, rotation: int = 0) -> np.random.Generator:
    """The generator every workload draws from: seed = 1000*config_index + rotation."""
    return np.random.default_rng(1000 * int(config_index) + int(rotation))


def sign_matrix(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """i.i.d. uniform +-1 entries as int8, shape (rows, cols)."""
    bits = rng.integers(0, 2, size=(rows, cols), dtype=np.int8)
    return (1 - 2 * bits).astype(np.int8)


def abs_normal_scales(rng: np.random.Generator, size: int, shift: float = 0.1) -> np.ndarray:
    """|N(0,1)| + shift, rounded to fp16 (round to nearest even)."""
    return (np.abs(rng.standard_normal(size)) + shift).astype(np.float16)


def lognormal_scales(rng: np.random.Generator, size: int, mu: float = -3.0, sigma: float = 0.5) -> np.ndarray:
    """lognormal(mu, sigma), rounded to fp16."""
    return rng.lognormal(mu, sigma, size).astype(np.float16)


def unit_scales(size: int) -> np.ndarray:
    return np.ones(size, dtype=np.float16)


def normal_activations(rng: np.random.Generator, batch: int, m_in: int) -> np.ndarray:
    """N(0,1) activations rounded to fp16, shape (batch, m_in)."""
    return rng.standard_normal((batch, m_in)).astype(np.float16)


def integer_activations(rng: np.random.Generator, batch: int, m_in: int, lo: int = -8, hi: int = 8) -> np.ndarray:
    """Uniform integers in [lo, hi] stored as fp16 (exact), shape (batch, m_in)."""
    return rng.integers(lo, hi + 1, size=(batch, m_in)).astype(np.float16)


def projection_signs(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """A rows x cols random sign matrix scaled by 1/sqrt(rows), as fp32 (the
    random projection that starts a factorisation)."""
    return (sign_matrix(rng, rows, cols).astype(np.float64) / np.sqrt(rows)).astype(np.float32)


def sylvester_hadamard(p: int) -> np.ndarray:
    """The 2^p x 2^p Sylvester sign pattern H[i, j] = (-1)^popcount(i & j), int8."""
    size = 1 << p
    idx = np.arange(size, dtype=np.int64)
    anded = idx[:, None] & idx[None, :]
    parity = np.zeros_like(anded)
    while np.any(anded):
        parity ^= anded & 1
        anded >>= 1
    return (1 - 2 * parity).astype(np.int8)


def make_layer(shape: LayerShape, batch: int, rotation: int = 0) -> dict:
    """Draw one layer: signs A (n x k), B (k x m_in); fp16 a (n), mid (k), b (m_in); x (batch x m_in).

    The draw order is fixed (A, B, a, mid, b, x) so a given seed always gives the
    same tensors whatever the caller does with them.
    """
    rng = rng_for(shape.index, rotation)
    A = sign_matrix(rng, shape.n, shape.k)
    B = sign_matrix(rng, shape.k, shape.m_in)
    if shape.scales == "absnormal":
        a = abs_normal_scales(rng, shape.n)
        mid = abs_normal_scales(rng, shape.k)
        b = abs_normal_scales(rng, shape.m_in)
    elif shape.scales == "lognormal":
        a = lognormal_scales(rng, shape.n)
        mid = lognormal_scales(rng, shape.k)
        b = lognormal_scales(rng, shape.m_in)
    elif shape.scales == "unit":
        a, mid, b = unit_scales(shape.n), unit_scales(shape.k), unit_scales(shape.m_in)
    else:
        raise ValueError(f"unknown scale recipe {shape.scales!r}")
    if shape.x == "normal":
        x = normal_activations(rng, batch, shape.m_in)
    elif shape.x == "int":
        x = integer_activations(rng, batch, shape.m_in)
    else:
        raise ValueError(f"unknown activation recipe {shape.x!r}")
    return {"A": A, "B": B, "a": a, "mid": mid, "b": b, "x": x}
