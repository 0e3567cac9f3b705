"""Seeded synthetic inputs for the activation-sparse linear layer.

This module is shared by the CPU oracle (``oracle/``), the GPU parity tests and
``bench.py``.  It draws random numbers and rounds them to IEEE binary16; it holds
none of the method's arithmetic (no mask, no product, no score).

Recipe (every draw uses ``numpy.random.default_rng`` (PCG64), values are drawn in
float64 and rounded once to fp16, round-to-nearest-even):

* Weights are drawn directly in the transposed layout ``WT`` of shape
  ``(d_in, d_out)``, row-major, so row ``i`` of ``WT`` holds every weight that
  multiplies input ``i``.  Entries are i.i.d., so the orientation of the draw
  does not change the distribution.
* For one projection, the weight is drawn first, then the activation, from one
  generator seeded with ``seed``.
* The threshold that sets a target sparsity ``s`` is the order statistic
  ``sort(|x|)[floor(s * d)]`` (0-based, ascending).  It stands in for the
  histogram calibration that TEAL performs on real activations (TEAL README,
  "Accuracy Usage"), which needs model weights and data.  ``s = 0`` gives the
  smallest magnitude, which keeps every finite entry.

Distributions follow the workloads the pages measure on: Laplace activations and
N(0, 0.02^2) weights for the TEAL-style threshold layer, Student-t(4)
activations with N(0, 0.01^2) weights for Q-Sparse top-k at 70B shapes, N(0, 1)
activations for the RaNA gated MLP, Laplace tokens for Block Q-Sparse N:M.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "LLAMA2_7B_PROJECTIONS", "QSPARSE_70B_PROJECTIONS", "NM_PATTERNS",
    "LLAMA2_SPARSITIES", "QSPARSE_KEEP_FRACTIONS",
    "draw_weight", "draw_vector", "quantile_threshold", "topk_count",
    "Projection", "projection", "rana_mlp", "nm_tokens", "tiny_gemv", "llama2_7b_layer",
    "rank_adapter", "batch_tokens", "q8_projection",
]

# Llama-2-7B decode projections at batch 1: (name, d_in, d_out).
LLAMA2_7B_PROJECTIONS = (
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096),
)
LLAMA2_SPARSITIES = (0.0, 0.25, 0.40, 0.50, 0.65)

# Q-Sparse at Llama-70B MLP shapes: (name, d_in, d_out).
QSPARSE_70B_PROJECTIONS = (("up", 8192, 28672), ("down", 28672, 8192))
QSPARSE_KEEP_FRACTIONS = (0.60, 0.50, 0.40)

# Block Q-Sparse N:M patterns as (N kept, M block).
NM_PATTERNS = ((2, 4), (8, 16), (16, 32), (1, 4))

_CHUNK = 1 << 22  # elements per draw; chunked draws equal one large draw


def _fill(rng: np.random.Generator, shape, draw) -> np.ndarray:
    """Draw ``prod(shape)`` float64 samples in chunks, rounding each chunk to fp16."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = draw(rng, hi - lo).astype(np.float16)
    return out.reshape(shape)


def draw_weight(rng, d_in: int, d_out: int, sigma: float) -> np.ndarray:
    """Transposed weight WT (d_in, d_out) with i.i.d. N(0, sigma^2) entries, fp16."""
    return _fill(rng, (d_in, d_out), lambda r, n: r.normal(0.0, sigma, n))


def draw_vector(rng, shape, dist: str) -> np.ndarray:
    """Activations of the given shape, fp16. ``dist`` in laplace / normal / student_t4."""
    if dist == "laplace":
        f = lambda r, n: r.laplace(0.0, 1.0, n)
    elif dist == "normal":
        f = lambda r, n: r.normal(0.0, 1.0, n)
    elif dist == "student_t4":
        f = lambda r, n: r.standard_t(4.0, n)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return _fill(rng, shape if isinstance(shape, tuple) else (shape,), f)


def quantile_threshold(x: np.ndarray, sparsity: float) -> float:
    """``sort(|x|)[floor(s*d)]`` as a Python float (exactly an fp16 value)."""
    mags = np.sort(np.abs(x.astype(np.float64)).ravel())
    d = mags.size
    pos = min(d - 1, int(math.floor(sparsity * d)))
    return float(mags[pos])


def topk_count(keep_fraction: float, d: int) -> int:
    """Number of entries kept for a top-k fraction: ``floor(f*d + 0.5)``."""
    return int(math.floor(keep_fraction * d + 0.5))


@dataclass
class Projection:
    name: str
    WT: np.ndarray          # (d_in, d_out) fp16, row-major
    x: np.ndarray           # (d_in,) fp16
    thresholds: dict = field(default_factory=dict)  # sparsity -> t

    @property
    def d_in(self) -> int:
        return self.WT.shape[0]

    @property
    def d_out(self) -> int:
        return self.WT.shape[1]


def projection(name: str, d_in: int, d_out: int, *, sigma: float, dist: str,
               seed: int, sparsities=()) -> Projection:
    """One linear layer: weight first, then activation, from ``default_rng(seed)``."""
    rng = np.random.default_rng(seed)
    WT = draw_weight(rng, d_in, d_out, sigma)
    x = draw_vector(rng, d_in, dist)
    return Projection(name, WT, x, {s: quantile_threshold(x, s) for s in sparsities})


def tiny_gemv(seed: int = 0) -> Projection:
    """1024 x 1024 weight ~ N(0, 0.02^2), Laplace x, t = sort|x|[512] (50 %)."""
    return projection("tiny", 1024, 1024, sigma=0.02, dist="laplace", seed=seed,
                      sparsities=(0.5,))


def llama2_7b(seed: int = 0, names=None):
    """The seven Llama-2-7B decode projections; projection ``j`` uses seed ``1000*seed + j``."""
    out = []
    for j, (name, d_in, d_out) in enumerate(LLAMA2_7B_PROJECTIONS):
        if names is not None and name not in names:
            continue
        out.append(projection(name, d_in, d_out, sigma=0.02, dist="laplace",
                              seed=1000 * seed + j, sparsities=LLAMA2_SPARSITIES))
    return out


def llama2_7b_layer(seed: int = 0):
    """One decoder layer as the model wires it: k and v read the same hidden
    state as q, and up the same as gate, so they share its threshold mask.
    Returns the seven projections in order q, k, v, o, gate, up, down."""
    projs = {p.name: p for p in llama2_7b(seed)}
    for shared, src in (("k", "q"), ("v", "q"), ("up", "gate")):
        p = projs[shared]
        projs[shared] = Projection(p.name, p.WT, projs[src].x, dict(projs[src].thresholds))
    return [projs[n] for n, _, _ in LLAMA2_7B_PROJECTIONS]


def qsparse_70b(seed: int = 0, names=None):
    """Q-Sparse top-k projections at 70B MLP shapes (Student-t(4) activations)."""
    out = []
    for j, (name, d_in, d_out) in enumerate(QSPARSE_70B_PROJECTIONS):
        if names is not None and name not in names:
            continue
        out.append(projection(name, d_in, d_out, sigma=0.01, dist="student_t4",
                              seed=1000 * seed + 100 + j))
    return out


@dataclass
class RanaMLP:
    WgT: np.ndarray   # (d_model, d_ff) fp16
    WuT: np.ndarray   # (d_model, d_ff) fp16
    WdT: np.ndarray   # (d_ff, d_model) fp16
    x: np.ndarray     # (d_model,) fp16


def rana_mlp(seed: int = 0, d_model: int = 4096, d_ff: int = 11008,
             sigma: float = 0.02) -> RanaMLP:
    """Gated MLP weights (gate, up, down drawn in that order) then x ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    WgT = draw_weight(rng, d_model, d_ff, sigma)
    WuT = draw_weight(rng, d_model, d_ff, sigma)
    WdT = draw_weight(rng, d_ff, d_model, sigma)
    x = draw_vector(rng, d_model, "normal")
    return RanaMLP(WgT, WuT, WdT, x)


def batch_tokens(seed: int = 0, B: int = 4, d_in: int = 4096, d_out: int = 11008,
                 sigma: float = 0.02, sparsity: float = 0.5):
    """A weight WT (d_in, d_out) then B Laplace tokens X (B, d_in), and one
    threshold shared by the tokens: the ``sparsity`` quantile of the pooled
    |X| (a per-layer calibrated threshold, as TEAL uses for every token)."""
    rng = np.random.default_rng(seed)
    WT = draw_weight(rng, d_in, d_out, sigma)
    X = draw_vector(rng, (B, d_in), "laplace")
    return WT, X, quantile_threshold(X, sparsity)


def q8_projection(seed: int = 0, d_in: int = 4096, d_out: int = 11008, q_sigma: float = 40.0,
                  w_sigma: float = 0.02, sparsities=(0.5,)):
    """An int8 weight as a quantised checkpoint holds it, then x ~ Laplace(0, 1).

    QT (d_in, d_out) int8: N(0, q_sigma^2) rounded to the nearest integer and
    clipped to [-127, 127]; scale (d_out,) float32: w_sigma / q_sigma times
    U(0.9, 1.1), so that s_j * q has the spread of the fp16 weights.  Returns
    (QT, scale, x, {sparsity: t}).
    """
    rng = np.random.default_rng(seed)
    QT = np.empty((d_in, d_out), dtype=np.int8)
    flat = QT.reshape(-1)
    for lo in range(0, flat.size, _CHUNK):
        hi = min(flat.size, lo + _CHUNK)
        flat[lo:hi] = np.clip(np.rint(rng.normal(0.0, q_sigma, hi - lo)), -127, 127).astype(np.int8)
    scale = (w_sigma / q_sigma * rng.uniform(0.9, 1.1, d_out)).astype(np.float32)
    x = draw_vector(rng, d_in, "laplace")
    return QT, scale, x, {s: quantile_threshold(x, s) for s in sparsities}


def q4_projection(seed: int = 0, d_in: int = 4096, d_out: int = 11008, q_sigma: float = 2.5,
                  w_sigma: float = 0.02, sparsities=(0.5,)):
    """An int4 weight as a quantised checkpoint holds it, then x ~ Laplace(0, 1).

    q (d_in, d_out): N(0, q_sigma^2) rounded to the nearest integer and clipped
    to [-8, 7], packed two to a byte (even column in bits 0..3, odd column in
    bits 4..7, two's complement) into QT4 (d_in, d_out / 2) uint8; scale
    (d_out,) float32: w_sigma / q_sigma times U(0.9, 1.1).  Returns
    (QT4, scale, x, {sparsity: t}).
    """
    rng = np.random.default_rng(seed)
    QT4 = np.empty((d_in, d_out // 2), dtype=np.uint8)
    rows = max(1, _CHUNK // max(1, d_out))
    for lo in range(0, d_in, rows):
        hi = min(d_in, lo + rows)
        q = np.clip(np.rint(rng.normal(0.0, q_sigma, (hi - lo, d_out))), -8, 7).astype(np.int64)
        nib = q & 0xF
        QT4[lo:hi] = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scale = (w_sigma / q_sigma * rng.uniform(0.9, 1.1, d_out)).astype(np.float32)
    x = draw_vector(rng, d_in, "laplace")
    return QT4, scale, x, {s: quantile_threshold(x, s) for s in sparsities}


def f8_projection(seed: int = 0, d_in: int = 4096, d_out: int = 11008, q_sigma: float = 64.0,
                  w_sigma: float = 0.02, sparsities=(0.5,)):
    """An fp8 (e4m3) weight as a quantised checkpoint holds it, then x ~ Laplace(0, 1).

    QT (d_in, d_out) uint8 e4m3 codes: N(0, q_sigma^2) clipped to the format's
    range [-448, 448] and rounded to the nearest e4m3 value (torch's float8_e4m3fn
    conversion); scale (d_out,) float32: w_sigma / q_sigma times U(0.9, 1.1).
    Returns (QT, scale, x, {sparsity: t}).
    """
    import torch
    rng = np.random.default_rng(seed)
    QT = np.empty((d_in, d_out), dtype=np.uint8)
    flat = QT.reshape(-1)
    for lo in range(0, flat.size, _CHUNK):
        hi = min(flat.size, lo + _CHUNK)
        v = np.clip(rng.normal(0.0, q_sigma, hi - lo), -448.0, 448.0).astype(np.float32)
        flat[lo:hi] = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    scale = (w_sigma / q_sigma * rng.uniform(0.9, 1.1, d_out)).astype(np.float32)
    x = draw_vector(rng, d_in, "laplace")
    return QT, scale, x, {s: quantile_threshold(x, s) for s in sparsities}


@dataclass
class RankAdapter:
    BT: np.ndarray    # (d_in, r) fp16: B transposed
    AT: np.ndarray    # (r, d_out) fp16: A transposed
    x: np.ndarray     # (d_in,) fp16


def rank_adapter(seed: int = 0, d_in: int = 4096, r: int = 2048, d_out: int = 4096,
                 sigma_a: float = 0.02) -> RankAdapter:
    """Rank adapter factors (B then A) and x ~ Laplace(0, 1).

    B ~ N(0, 1/d_in), so that v = Bx has entries of order one; A ~ N(0, sigma_a^2).
    """
    rng = np.random.default_rng(seed)
    BT = draw_weight(rng, d_in, r, 1.0 / math.sqrt(d_in))
    AT = draw_weight(rng, r, d_out, sigma_a)
    x = draw_vector(rng, d_in, "laplace")
    return RankAdapter(BT, AT, x)


def nm_tokens(seed: int = 0, rows: int = 4096, d: int = 1024, d_out: int = 1024,
              sigma: float = 0.02):
    """Block Q-Sparse batch: WT (d, d_out) then X (rows, d) ~ Laplace, both fp16."""
    rng = np.random.default_rng(seed)
    WT = draw_weight(rng, d, d_out, sigma)
    X = draw_vector(rng, (rows, d), "laplace")
    return WT, X
