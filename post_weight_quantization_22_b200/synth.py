"""Seeded synthetic layer inputs shared by the GPU path's tests, the oracle's tests and the bench.

This module draws random numbers and nothing else: it holds none of the quantization
arithmetic (no Hessian, no factorisation, no grid, no rounding to codes).  Both sides of every
parity check receive the same arrays from here.

Workload shapes follow the layer shapes of 7-8B LLMs that the GPTQ-as-Babai page evaluates on
("The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm", section 4):
q/k/v/o 4096-wide, MLP 14336-wide.  The pages calibrate on WikiText-2 / C4 activations, which are
not available here; a decaying-spectrum generator with a few outlier channels stands in for them.

Recipes (all numpy ``default_rng`` streams, fp64 draws, then rounded to the storage dtype):

* ``calib_activations(T, n, seed)``: X = Z diag(k^-0.8) V^T with Z ~ N(0,1) of shape T x n and V
  Haar-orthogonal (QR of an n x n Gaussian with the sign of diag(R) folded in); then 4 seeded
  input channels are multiplied by 20 (outlier channels).
* ``post_silu_like(G)``: sign(G) |G|^1.5, the down-projection input.
* ``layer_weights(m, n, seed)``: N(0, 0.02^2) entries; 1 % of rows (seeded) are replaced by
  0.02 * Student-t(4) draws (heavy-tailed outlier rows).
* ``tiny_weights(m, n, seed)``: N(0, 0.02^2) with round(0.02 n) seeded columns multiplied by 10.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "calib_activations",
    "post_silu_like",
    "layer_weights",
    "tiny_weights",
    "to_bf16",
    "WORKLOADS",
    "workload",
]


def to_bf16(a: np.ndarray):
    """Round to bfloat16 (round-to-nearest-even) and return a torch CPU bf16 tensor."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _haar_orthogonal(n: int, rng: np.random.Generator) -> np.ndarray:
    g = rng.standard_normal((n, n))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def calib_activations(T: int, n: int, seed: int, decay: float = 0.8,
                      n_outlier: int = 4, outlier_gain: float = 20.0) -> np.ndarray:
    """T tokens x n features, fp64, decaying singular spectrum 1/k^decay plus outlier channels."""
    rng = np.random.default_rng(seed)
    v = _haar_orthogonal(n, rng)
    z = rng.standard_normal((T, n))
    z *= np.arange(1, n + 1, dtype=np.float64) ** (-decay)
    x = z @ v.T
    idx = rng.choice(n, size=min(n_outlier, n), replace=False)
    x[:, idx] *= outlier_gain
    return x


def post_silu_like(g: np.ndarray) -> np.ndarray:
    return np.sign(g) * np.abs(g) ** 1.5


def layer_weights(m: int, n: int, seed: int, std: float = 0.02,
                  outlier_row_frac: float = 0.01, t_dof: float = 4.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = std * rng.standard_normal((m, n))
    k = int(round(outlier_row_frac * m))
    if k > 0:
        rows = rng.choice(m, size=k, replace=False)
        w[rows] = std * rng.standard_t(t_dof, size=(k, n))
    return w


def tiny_weights(m: int, n: int, seed: int, std: float = 0.02,
                 col_frac: float = 0.02, gain: float = 10.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = std * rng.standard_normal((m, n))
    k = int(round(col_frac * n))
    if k > 0:
        cols = rng.choice(n, size=k, replace=False)
        w[:, cols] *= gain
    return w


# name -> recipe.  "dtype" is the storage dtype of both W and X; quantization settings follow the
# workloads' own descriptions (bits, group size, column order, clipping).
WORKLOADS = {
    "tiny_256x512": dict(m=256, n=512, T=2048, dtype="fp32", bits=4, group=0, reverse=0, clip=1,
                         w_seed=0, x_seed=101, w_kind="tiny", x_kind="calib"),
    "q_proj_4096x4096": dict(m=4096, n=4096, T=4096, dtype="bf16", bits=4, group=128, reverse=0,
                             clip=1, w_seed=1, x_seed=102, w_kind="layer", x_kind="calib"),
    "mlp_up_14336x4096": dict(m=14336, n=4096, T=8192, dtype="bf16", bits=3, group=128, reverse=0,
                              clip=1, w_seed=2, x_seed=103, w_kind="layer", x_kind="calib"),
    "mlp_down_4096x14336": dict(m=4096, n=14336, T=8192, dtype="bf16", bits=3, group=128,
                                reverse=0, clip=1, w_seed=12, x_seed=113, w_kind="layer",
                                x_kind="post_silu"),
    "clipfree_babai_4096x4096": dict(m=4096, n=4096, T=4096, dtype="bf16", bits=3, group=0,
                                     reverse=1, clip=0, w_seed=3, x_seed=104, w_kind="layer",
                                     x_kind="calib"),
}

# The 8B-shaped block sweep: per block, four distinct inputs (attention input shared by q/k/v,
# the o_proj input, the MLP input shared by gate/up, the down_proj input); 2-bit, group 64.
SWEEP_LAYERS = (
    ("q", 4096, 4096, "attn"), ("k", 1024, 4096, "attn"), ("v", 1024, 4096, "attn"),
    ("o", 4096, 4096, "o"), ("gate", 14336, 4096, "mlp"), ("up", 14336, 4096, "mlp"),
    ("down", 4096, 14336, "down"),
)
SWEEP_INPUT_INDEX = {"attn": 0, "o": 1, "mlp": 2, "down": 3}
SWEEP_T = 8192
SWEEP_BLOCKS = 32


def sweep_seeds(block: int, layer_index: int, input_kind: str):
    """(weight seed, activation seed) of layer ``layer_index`` in block ``block`` of the sweep."""
    return 1000 + 10 * block + layer_index, 5000 + 10 * block + SWEEP_INPUT_INDEX[input_kind]


def sweep_block(block: int, T: int = SWEEP_T, scale: int = 1):
    """Inputs of one block of the sweep: ({layer name: W}, {input key: X}), bf16 torch CPU
    tensors.  The attention, o_proj and MLP inputs use the decaying-spectrum generator, the
    down_proj input its post-SiLU-like transform.  ``scale`` divides every dimension (reduced
    cases for tests)."""
    Ws, Xs = {}, {}
    for li, (name, m, n, kind) in enumerate(SWEEP_LAYERS):
        w_seed, x_seed = sweep_seeds(block, li, kind)
        Ws[name] = to_bf16(make_w("layer", m // scale, n // scale, w_seed))
        if kind not in Xs:
            x_kind = "post_silu" if kind == "down" else "calib"
            Xs[kind] = to_bf16(make_x(x_kind, T // scale, n // scale, x_seed))
    return Ws, Xs


def make_x(x_kind: str, T: int, n: int, seed: int) -> np.ndarray:
    if x_kind == "calib":
        return calib_activations(T, n, seed)
    if x_kind == "post_silu":
        return post_silu_like(calib_activations(T, n, seed))
    raise ValueError(x_kind)


def make_w(w_kind: str, m: int, n: int, seed: int) -> np.ndarray:
    if w_kind == "tiny":
        return tiny_weights(m, n, seed)
    if w_kind == "layer":
        return layer_weights(m, n, seed)
    raise ValueError(w_kind)


def workload(name: str, m: int | None = None, n: int | None = None, T: int | None = None):
    """Return (W, X, spec) for a named workload.

    W and X are torch CPU tensors in the workload's storage dtype (bf16 or fp32); the values
    after that rounding are the ground truth for both sides.  ``m``, ``n`` and ``T`` override the
    shape (same recipe and seeds), which the tests use for reduced cases.
    """
    import torch

    spec = dict(WORKLOADS[name])
    if m is not None:
        spec["m"] = m
    if n is not None:
        spec["n"] = n
    if T is not None:
        spec["T"] = T
    w = make_w(spec["w_kind"], spec["m"], spec["n"], spec["w_seed"])
    x = make_x(spec["x_kind"], spec["T"], spec["n"], spec["x_seed"])
    if spec["dtype"] == "bf16":
        return to_bf16(w), to_bf16(x), spec
    return (torch.from_numpy(w.astype(np.float32)), torch.from_numpy(x.astype(np.float32)), spec)
