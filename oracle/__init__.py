"""CPU oracle for the activation-sparse linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``sparse_input_gemv_threshold_b200``) never imports
it, and it never imports the product: the two share no code.  The only module
both sides use is ``workloads`` (seeded random inputs, no method arithmetic).

It is a plain, slow, obviously correct restatement in numpy float64 of what the
pages define.  Library primitives (a stable sort, a float64 matrix product,
``exp``, the fp64 -> fp16 cast) serve as single steps; nothing is blocked, fused
or reordered.

Sources, cited by page title and section:

* [QS]   "Q-Sparse: All Large Language Models can be Fully Sparsely-Activated"
         (OpenReview rebuttal).  A1 to the second reviewer defines activation
         sparsity as the share of zero entries of X in WX; A3 (FLOPs) counts
         2 d^2 for a d x d by d x 1 product; A1 on MoE says Q-Sparse keeps, per
         token, the entries of largest magnitude; A2 (batched inference) brings
         in Block Q-Sparse with N:M activation sparsity.
* [TEAL] "Training-Free Activation Sparsity in Large Language Models" (TEAL
         README), Abstract: magnitude-based activation sparsity of the hidden
         states that feed each matrix multiplication.
* [RaNA] "Adaptive Rank Allocation: Speeding Up Modern Transformers with RaNA
         Adapters" (OpenReview rebuttal): Q3, Eqn. 12 (RaNA neuron masker) and
         the CATS masker beside it; Q5.1, the linear-layer rank adapter
         Linear(x) ~ A(m(x) . Bx), whose masked product skips the columns of A
         whose mask entry is 0; Q4, its masker squares Bx element-wise and
         compares with a threshold (eqn. 9); Q2 to the fourth reviewer, one
         plain GEMV for v = Bx and one masked GEMV for A(m(x) . v).
* [RaNA] Q6 (batched inference with inconsistent masks) leaves a masked GEMV
         for batch sizes above one, where every token has its own mask, to
         future work; the batched product below is that operation.
* [TEAL] Limitations: quantised sparse kernels are missing; [QS] A1 on
         batched inference: quantisation, which shrinks the weight bytes
         moved per decoding step, is orthogonal to activation sparsity.  The
         weight-quantised product below is that combination.
* [NM]   "Motivating Next-Gen Accelerators with Flexible (N:M) Activation
         Sparsity ..." (summary), Methodology: in blocks of size M, N non-zero
         elements are kept; selection criterion ACT = absolute activation size.

Readings where the pages are silent or disagree (each one is a choice):

* Threshold comparison is ``|x_i| >= t`` ([RaNA] Eqn. 12 writes ``>= t``; TEAL
  gives no operator), with t a float32 value.  A NaN is never kept by a
  threshold.
* Ranking by magnitude (top-k, N:M): larger |x| first, equal |x| by lower index
  first; +v and -v tie, +0 and -0 tie; a NaN ranks below every number.
* N:M keeps the N largest of each M consecutive elements ([NM] Methodology;
  [QS] A2 words it as "N ... to be zero", which the 50 % patterns do not tell
  apart; 1:4 read as keep one of four, 75 % sparsity).
* ||W^down_i||_F in Eqn. 12 is the l2 norm of the weights that multiply neuron
  i, i.e. row i of the transposed down weight, computed in float64 and rounded
  once to float32.
* Eqn. 12 precision: g and u in float64 from the fp16 inputs, h rounded once to
  fp16, ``s_i = float32(|h_i|) * norm_i`` as one float32 multiply, ``s_i >= t``.
* Rank adapter precision: v = Bx in float64 from the fp16 inputs, rounded once
  to fp16 (the intermediate activation of an fp16 model); the score is
  ``float32(v_i) * float32(v_i)`` as one float32 multiply; ``score >= t``.
* Weight-quantised product (the pages fix no format): int8 weights q with one
  float32 scale per output column, ``W_ij = s_j * q_ij``; the activation and
  its mask stay fp16, and ``y_j = s_j * sum_i q_ij (m_i x_i)``.  The same with
  fp8 e4m3 weights (OCP E4M3, decoded exactly) in place of int8.
* N:M mitigation variants ([NM] Methodology: selection criteria ACT and WT,
  error mitigation D-/S-/L-PTS and VAR): a per-token shift mu gives
  ``x' = fp16(float32(x) - mu)`` (the product adds back ``mu * r_j`` with
  ``r_j = sum_i WT[i, j]``); the WT criterion scores ``float32(|x'_i|) *
  norm_i`` (one float32 multiply, ``norm_i`` the l2 norm of the weights that
  multiply input i) in place of ``|x'_i|``; VAR scales a token's kept values
  by ``gamma = sqrt(sum x'^2 / sum (m x')^2)`` so that the masked activation
  keeps the token's l2 norm (gamma = 1 when either sum is 0).
* Outputs: y in float64 (used for the error bound) and rounded once to fp16.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, hand-derived fixtures under ``tests/golden/``, brute force on
tiny inputs, reductions to the dense product).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "fp16", "magnitude_order", "threshold_mask", "topk_mask", "nm_mask",
    "compact", "pack_bits", "unpack_bits", "sparsity", "flops",
    "masked_matvec", "sparse_linear", "silu", "row_norms", "rana_hidden",
    "rana_scores", "rana_mask", "gated_mlp", "nm_gemm",
    "rank_adapter_hidden", "rank_adapter_scores", "rank_adapter",
    "union_mask", "batched_sparse_linear", "q8_sparse_linear", "teal_mlp",
    "pts_shift", "wt_scores", "nm_mask_by_score", "var_gamma", "nm_variant", "nm_variant_gemm",
    "nm_pack_2of4", "e4m3_value", "f8_sparse_linear", "int4_values", "q4_sparse_linear",
]


# ---------------------------------------------------------------------------
# Rounding
# ---------------------------------------------------------------------------

def fp16(v) -> np.ndarray:
    """Round float64 values once to IEEE binary16, round-to-nearest-even.

    numpy's float64 -> float16 cast rounds directly from the 52-bit mantissa
    (no detour through float32); the pins check this against exact rational
    arithmetic, including values just off a halfway point.
    """
    with np.errstate(over="ignore"):
        return np.asarray(v, dtype=np.float64).astype(np.float16)


# ---------------------------------------------------------------------------
# Masks
# ---------------------------------------------------------------------------

def _magnitude_key(x) -> np.ndarray:
    """|x| in float64 with NaN mapped below every magnitude (to -1)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    return np.where(np.isnan(a), -1.0, a)


def magnitude_order(x) -> np.ndarray:
    """Indices of a 1-D ``x`` by |x| descending, ties by lower index ([QS] A1 on MoE)."""
    key = _magnitude_key(x)
    return np.argsort(-key, kind="stable")


def threshold_mask(x, t: float) -> np.ndarray:
    """[TEAL] Abstract: keep x_i when |x_i| >= t (a NaN is never kept).

    The threshold is a float32 value (the layer takes it as one), so ``t`` is
    rounded to float32 first; |x_i| of an fp16 input is exact in float64."""
    return np.abs(np.asarray(x, dtype=np.float64)) >= np.float64(np.float32(t))


def topk_mask(x, k: int) -> np.ndarray:
    """[QS] A1 on MoE: per token keep the k entries of largest magnitude."""
    x = np.asarray(x).ravel()
    if not 0 <= k <= x.size:
        raise ValueError("k out of range")
    m = np.zeros(x.size, dtype=bool)
    m[magnitude_order(x)[:k]] = True
    return m


def nm_mask(X, n: int, m: int) -> np.ndarray:
    """[NM] Methodology / [QS] A2: per row, in each block of M consecutive
    elements keep the N of largest magnitude (ties by lower index)."""
    X = np.asarray(X)
    squeeze = X.ndim == 1
    X2 = X.reshape(1, -1) if squeeze else X
    rows, d = X2.shape
    if not (1 <= n <= m) or d % m:
        raise ValueError("need 1 <= n <= m and m | d")
    key = _magnitude_key(X2).reshape(rows, d // m, m)
    order = np.argsort(-key, axis=-1, kind="stable")
    keep = np.zeros((rows, d // m, m), dtype=bool)
    np.put_along_axis(keep, order[..., :n], True, axis=-1)
    keep = keep.reshape(rows, d)
    return keep[0] if squeeze else keep


def compact(mask) -> np.ndarray:
    """Ascending int32 indices of the kept entries ([RaNA] Q5.1: the product
    skips the columns whose mask entry is 0, so only these are visited)."""
    return np.flatnonzero(np.asarray(mask).ravel()).astype(np.int32)


def pack_bits(mask) -> np.ndarray:
    """Bit i%32 of uint32 word i//32 is mask[i] (little-endian within a word).

    A 2-D mask packs each row separately, rows padded to whole words.
    """
    mask = np.asarray(mask, dtype=bool)
    if mask.ndim == 2:
        return np.stack([pack_bits(r) for r in mask]) if len(mask) else \
            np.zeros((0, (mask.shape[1] + 31) // 32), np.uint32)
    d = mask.size
    words = (d + 31) // 32
    padded = np.zeros(words * 32, dtype=np.uint64)
    padded[:d] = mask
    weights = np.left_shift(np.uint64(1), np.arange(32, dtype=np.uint64))
    return (padded.reshape(words, 32) * weights).sum(axis=1).astype(np.uint32)


def unpack_bits(words, d: int) -> np.ndarray:
    """Inverse of :func:`pack_bits` for one row of ``d`` entries."""
    words = np.asarray(words, dtype=np.uint32)
    bits = (words[:, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return bits.ravel()[:d].astype(bool)


def sparsity(mask) -> float:
    """[QS] A1 to the second reviewer: share of zero entries of the masked input."""
    mask = np.asarray(mask)
    return float(1.0 - mask.sum() / mask.size) if mask.size else 0.0


def flops(d_out: int, nnz: int) -> int:
    """[QS] A3: a d_out x d_in by d_in x 1 product costs 2 d_out d_in; with
    only nnz inputs kept it costs 2 d_out nnz (mask cost left out)."""
    return 2 * int(d_out) * int(nnz)


def nm_pack_2of4(X, n: int) -> dict:
    """The 2:4 operand of an N:M mask with M = 4 ([NM] Hardware implications:
    2:4 is the pattern the hardware supports; [NM] Methodology / [QS] A2 for
    the mask).  Per row and block of four entries: the kept entries of
    :func:`nm_mask` (n = 2), or the kept entry plus a padding slot at the
    block's smallest position that is not kept, holding +0 (n = 1, 1:4
    padded to 2:4), both slots in ascending position order.  Returns fp16
    ``values`` and uint8 ``positions`` (0..3 within the block), each of shape
    (rows, d/2), and the ``mask``."""
    X = np.asarray(X, dtype=np.float16)
    X2 = X.reshape(1, -1) if X.ndim == 1 else X
    if n not in (1, 2):
        raise ValueError("the 2:4 operand packs 2:4 or 1:4")
    rows, d = X2.shape
    mask = nm_mask(X2, n, 4)
    values = np.zeros((rows, d // 2), dtype=np.float16)
    positions = np.zeros((rows, d // 2), dtype=np.uint8)
    for r in range(rows):
        for b in range(d // 4):
            kept = [j for j in range(4) if mask[r, 4 * b + j]]
            slots = kept if n == 2 else sorted(kept + [min(j for j in range(4) if j not in kept)])
            for s, j in enumerate(slots):
                positions[r, 2 * b + s] = j
                values[r, 2 * b + s] = X2[r, 4 * b + j] if j in kept else np.float16(0.0)
    return {"values": values, "positions": positions, "mask": mask}


# ---------------------------------------------------------------------------
# The sparse-input product y = W (m . x)
# ---------------------------------------------------------------------------

def masked_matvec(WT, x, mask, cols=None):
    """y_j = sum_i WT[i, j] * (m_i ? x_i : 0) in float64 ([RaNA] Q5.1).

    ``WT`` is the transposed weight (d_in, d_out): row i multiplies input i.
    Returns ``(y64, bound)`` with ``bound_j = sum_i |WT[i, j] * m_i x_i|``,
    the scale of the per-element error tolerance.  ``cols`` restricts the
    output to a subset of output columns.
    """
    WT = np.asarray(WT)
    if cols is not None:
        WT = WT[:, np.asarray(cols)]
    xm = np.where(np.asarray(mask, dtype=bool), np.asarray(x, dtype=np.float64), 0.0)
    W64 = WT.astype(np.float64)
    y64 = xm @ W64
    bound = np.abs(xm) @ np.abs(W64)
    return y64, bound


def sparse_linear(WT, x, mask, cols=None) -> dict:
    """Mask applied, product taken, result rounded once to fp16."""
    y64, bound = masked_matvec(WT, x, mask, cols)
    idx = compact(mask)
    return {"mask": np.asarray(mask, dtype=bool), "idx": idx, "nnz": int(idx.size),
            "y64": y64, "y16": fp16(y64), "bound": bound}


# ---------------------------------------------------------------------------
# RaNA gated-MLP neuron masker (Eqn. 12)
# ---------------------------------------------------------------------------

def silu(z):
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)), float64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def row_norms(WT) -> np.ndarray:
    """l2 norm of each row of a transposed weight, float64, rounded to float32.

    For the down projection, row i of WdT holds the weights that multiply
    neuron i: the ||W^down_i||_F of [RaNA] Eqn. 12.
    """
    W64 = np.asarray(WT).astype(np.float64)
    return np.sqrt((W64 * W64).sum(axis=1)).astype(np.float32)


def rana_hidden(x, WgT, WuT):
    """g = GateProj(x), u = UpProj(x) in float64; h = fp16(SiLU(g) * u).

    h is the input of the down projection ([RaNA] Q3, the sentence after
    Eqn. 12).
    """
    x64 = np.asarray(x, dtype=np.float64)
    g = x64 @ np.asarray(WgT).astype(np.float64)
    u = x64 @ np.asarray(WuT).astype(np.float64)
    return g, u, fp16(silu(g) * u)


def rana_scores(h16, norms32) -> np.ndarray:
    """s_i = |h_i| * ||W^down_i|| as one float32 multiply ([RaNA] Eqn. 12)."""
    h32 = np.abs(np.asarray(h16, dtype=np.float16)).astype(np.float32)
    return (h32 * np.asarray(norms32, dtype=np.float32)).astype(np.float32)


def rana_mask(s32, t: float) -> np.ndarray:
    """m_i = s_i >= t, compared in float32 ([RaNA] Eqn. 12)."""
    return np.asarray(s32, dtype=np.float32) >= np.float32(t)


def gated_mlp(x, WgT, WuT, WdT, norms32, t: float, cols=None) -> dict:
    """Eqn. 12 masker then the masked down projection y = W_down (m . h)."""
    g, u, h16 = rana_hidden(x, WgT, WuT)
    s32 = rana_scores(h16, norms32)
    m = rana_mask(s32, t)
    out = sparse_linear(WdT, h16, m, cols)
    out.update({"g": g, "u": u, "h16": h16, "s32": s32})
    return out


# ---------------------------------------------------------------------------
# RaNA linear-layer rank adapter A (m(x) . Bx)
# ---------------------------------------------------------------------------

def rank_adapter_hidden(x, BT):
    """v = Bx in float64 from the fp16 inputs, and v rounded once to fp16.

    ``BT`` is B transposed, (d_in, r): row i multiplies input i.  This is the
    plain GEMV of [RaNA] Q2 (fourth reviewer).
    """
    v64 = np.asarray(x, dtype=np.float64) @ np.asarray(BT).astype(np.float64)
    return v64, fp16(v64)


def rank_adapter_scores(v16) -> np.ndarray:
    """s_i = v_i^2 as one float32 multiply ([RaNA] Q4: the masker squares Bx
    element-wise, eqn. 9)."""
    v32 = np.asarray(v16, dtype=np.float16).astype(np.float32)
    return (v32 * v32).astype(np.float32)


def rank_adapter(x, BT, AT, t: float, cols=None) -> dict:
    """[RaNA] Q5.1: Linear(x) ~ A (m(x) . Bx) with m_i = (Bx)_i^2 >= t.

    ``AT`` is A transposed, (r, d_out): row i multiplies v_i, so the masked
    product skips the rows of AT (columns of A) whose mask entry is 0.
    """
    v64, v16 = rank_adapter_hidden(x, BT)
    s32 = rank_adapter_scores(v16)
    m = rana_mask(s32, t)
    out = sparse_linear(AT, v16, m, cols)
    out.update({"v64": v64, "v16": v16, "s32": s32})
    return out


# ---------------------------------------------------------------------------
# A few tokens, each with its own mask ([RaNA] Q6)
# ---------------------------------------------------------------------------

def union_mask(masks) -> np.ndarray:
    """Rows any token keeps: the weight rows a batched product must read."""
    return np.asarray(masks, dtype=bool).any(axis=0)


def batched_sparse_linear(WT, X, masks, cols=None) -> dict:
    """y_b = W (m_b . x_b) for every token b: the single-token product of
    [RaNA] Q5.1 with token b's own mask ([RaNA] Q6).  Returns stacked
    ``y64``, ``bound`` (tokens x outputs) and the union of the masks."""
    X = np.asarray(X)
    masks = np.asarray(masks, dtype=bool)
    outs = [masked_matvec(WT, X[b], masks[b], cols) for b in range(X.shape[0])]
    y64 = np.stack([o[0] for o in outs]) if outs else np.zeros((0, 0))
    bound = np.stack([o[1] for o in outs]) if outs else np.zeros((0, 0))
    return {"y64": y64, "y16": fp16(y64), "bound": bound, "union": union_mask(masks)}


# ---------------------------------------------------------------------------
# N:M selection and error-mitigation variants ([NM] Methodology)
# ---------------------------------------------------------------------------

def pts_shift(X, shift) -> np.ndarray:
    """Per-token shift (PTS): x' = fp16(float32(x) - mu_row), one rounding."""
    X32 = np.asarray(X, dtype=np.float16).astype(np.float32)
    mu = np.asarray(shift, dtype=np.float32).reshape(-1, 1)
    return (X32 - mu).astype(np.float16)


def wt_scores(Xs, norms) -> np.ndarray:
    """WT criterion: float32(|x'_i|) * norm_i as one float32 multiply."""
    a = np.abs(np.asarray(Xs, dtype=np.float16)).astype(np.float32)
    return (a * np.asarray(norms, dtype=np.float32).reshape(1, -1)).astype(np.float32)


def nm_mask_by_score(S, n: int, m: int) -> np.ndarray:
    """Per row, in each block of m consecutive entries keep the n of largest
    score; equal scores by lower index, a NaN score below every number."""
    S = np.asarray(S, dtype=np.float64)
    rows, d = S.shape
    out = np.zeros((rows, d), dtype=bool)
    for r in range(rows):
        for b0 in range(0, d, m):
            blk = S[r, b0:b0 + m]
            key = np.where(np.isnan(blk), -np.inf, blk)
            nan = np.isnan(blk)
            # sort by (score desc, NaN last, index asc)
            order = sorted(range(blk.size), key=lambda j: (nan[j], -key[j], j))
            out[r, b0 + np.array(order[:n])] = True
    return out


def var_gamma(Xs, mask) -> np.ndarray:
    """VAR: per row gamma = sqrt(sum x'^2 / sum (m x')^2) in float64 (1 when
    either sum is 0), the scale that gives the masked row the l2 norm of x'."""
    X64 = np.asarray(Xs, dtype=np.float16).astype(np.float64)
    full = (X64 * X64).sum(axis=1)
    kept = np.where(mask, X64 * X64, 0.0).sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        g = np.sqrt(full / kept)
    return np.where((full > 0) & (kept > 0), g, 1.0)


def nm_variant(X, n: int, m: int, shift=None, norms=None, var: bool = False) -> dict:
    """The masked activation block of one N:M variant: shift (PTS), score
    (|x'| for ACT, WT with norms), select n of m, then scale (VAR)."""
    X = np.asarray(X, dtype=np.float16)
    Xs = pts_shift(X, shift) if shift is not None else X
    if norms is None:
        mask = nm_mask(Xs, n, m)
    else:
        mask = nm_mask_by_score(wt_scores(Xs, norms), n, m)
    gamma = var_gamma(Xs, mask) if var else np.ones(X.shape[0])
    Xm64 = np.where(mask, Xs.astype(np.float64), 0.0) * gamma.reshape(-1, 1)
    return {"xs": Xs, "mask": mask, "gamma": gamma, "xm64": Xm64, "xm16": fp16(Xm64)}


def nm_variant_gemm(Xm, WT, shift=None, rows=None):
    """Y = Xm WT + mu r^T (r_j = sum_i WT[i, j], the shift added back), float64.
    ``Xm`` is the masked (and scaled) activation block.  Returns (Y64, bound)
    with bound = |Xm| |WT| + |mu| sum_i |WT[i, j]|."""
    Xm = np.asarray(Xm, dtype=np.float64)
    W64 = np.asarray(WT).astype(np.float64)
    mu = np.zeros(Xm.shape[0]) if shift is None else np.asarray(shift, dtype=np.float32).astype(np.float64)
    if rows is not None:
        Xm, mu = Xm[np.asarray(rows)], mu[np.asarray(rows)]
    Y = Xm @ W64 + np.outer(mu, W64.sum(axis=0))
    bound = np.abs(Xm) @ np.abs(W64) + np.outer(np.abs(mu), np.abs(W64).sum(axis=0))
    return Y, bound


# ---------------------------------------------------------------------------
# Weight-quantised sparse product ([TEAL] Limitations, [QS] A1)
# ---------------------------------------------------------------------------

def q8_sparse_linear(QT, scale, x, mask, cols=None) -> dict:
    """y_j = s_j * sum_i QT[i, j] * (m_i ? x_i : 0) in float64.

    ``QT`` is the int8 weight transposed, (d_in, d_out); ``scale`` the float32
    scale of each output column, so that W[j, i] = s_j * QT[i, j].  Returns
    the same fields as :func:`sparse_linear`, with
    ``bound_j = |s_j| * sum_i |QT[i, j] * m_i x_i|``.
    """
    QT = np.asarray(QT, dtype=np.int8)
    s64 = np.asarray(scale, dtype=np.float32).astype(np.float64)
    if cols is not None:
        QT, s64 = QT[:, np.asarray(cols)], s64[np.asarray(cols)]
    xm = np.where(np.asarray(mask, dtype=bool), np.asarray(x, dtype=np.float64), 0.0)
    Q64 = QT.astype(np.float64)
    y64 = (xm @ Q64) * s64
    bound = (np.abs(xm) @ np.abs(Q64)) * np.abs(s64)
    idx = compact(mask)
    return {"mask": np.asarray(mask, dtype=bool), "idx": idx, "nnz": int(idx.size),
            "y64": y64, "y16": fp16(y64), "bound": bound}


def e4m3_value(codes) -> np.ndarray:
    """The value of each fp8 e4m3 code (the OCP 8-bit floating-point format
    E4M3: sign bit 7, four exponent bits 6..3 with bias 7, three mantissa bits
    2..0; exponent 0 is subnormal, 2^-6 * m/8; S.1111.111 is NaN; no
    infinities), exactly, in float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def f8_sparse_linear(QT, scale, x, mask, cols=None) -> dict:
    """y_j = s_j * sum_i e4m3(QT[i, j]) * (m_i ? x_i : 0) in float64: the
    weight-quantised product of :func:`q8_sparse_linear` with fp8 e4m3 weights
    (one float32 scale per output column) in place of int8 ones."""
    QT = np.asarray(QT, dtype=np.uint8)
    s64 = np.asarray(scale, dtype=np.float32).astype(np.float64)
    if cols is not None:
        QT, s64 = QT[:, np.asarray(cols)], s64[np.asarray(cols)]
    Q64 = e4m3_value(QT)
    xm = np.where(np.asarray(mask, dtype=bool), np.asarray(x, dtype=np.float64), 0.0)
    y64 = (xm @ Q64) * s64
    bound = (np.abs(xm) @ np.abs(Q64)) * np.abs(s64)
    idx = compact(mask)
    return {"mask": np.asarray(mask, dtype=bool), "idx": idx, "nnz": int(idx.size),
            "y64": y64, "y16": fp16(y64), "bound": bound}


def int4_values(packed) -> np.ndarray:
    """The int4 weights held two to a byte: byte b of a row carries weight 2b
    in bits 0..3 and weight 2b + 1 in bits 4..7, each a 4-bit two's-complement
    integer in [-8, 7].  (d_in, d_out / 2) uint8 in, (d_in, d_out) int8 out."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = p & 0xF, p >> 4
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out.astype(np.int8)


def q4_sparse_linear(QT4, scale, x, mask, cols=None) -> dict:
    """y_j = s_j * sum_i q[i, j] * (m_i ? x_i : 0) in float64 with int4 weights
    q (packed two to a byte, :func:`int4_values`) and one float32 scale per
    output column: the weight-quantised product of :func:`q8_sparse_linear`
    with 4-bit weights in place of 8-bit ones."""
    Q = int4_values(QT4)
    s64 = np.asarray(scale, dtype=np.float32).astype(np.float64)
    if cols is not None:
        Q, s64 = Q[:, np.asarray(cols)], s64[np.asarray(cols)]
    Q64 = Q.astype(np.float64)
    xm = np.where(np.asarray(mask, dtype=bool), np.asarray(x, dtype=np.float64), 0.0)
    y64 = (xm @ Q64) * s64
    bound = (np.abs(xm) @ np.abs(Q64)) * np.abs(s64)
    idx = compact(mask)
    return {"mask": np.asarray(mask, dtype=bool), "idx": idx, "nnz": int(idx.size),
            "y64": y64, "y16": fp16(y64), "bound": bound}


def teal_mlp(x, WgT, WuT, WdT, t_x: float, t_h: float, cols=None) -> dict:
    """A gated MLP with TEAL's magnitude threshold on the input of every
    product ([TEAL] Abstract: the hidden states that feed each matrix
    multiplication): g and u from the kept entries of x (|x_i| >= t_x), float64;
    h = fp16(SiLU(g) * u); y = W_down (m . h) with m_i = |h_i| >= t_h."""
    m_x = threshold_mask(x, t_x)
    g, _ = masked_matvec(WgT, x, m_x)
    u, _ = masked_matvec(WuT, x, m_x)
    h16 = fp16(silu(g) * u)
    m_h = threshold_mask(h16, t_h)
    out = sparse_linear(WdT, h16, m_h, cols)
    out.update({"mask_x": m_x, "g": g, "u": u, "h16": h16})
    return out


# ---------------------------------------------------------------------------
# Block Q-Sparse batched product Y = (M . X) WT
# ---------------------------------------------------------------------------

def nm_gemm(X, WT, mask, rows=None):
    """Y[r, j] = sum_i (M . X)[r, i] WT[i, j] in float64 ([QS] A2, Block Q-Sparse).

    Returns ``(Y64, bound)`` with ``bound[r, j] = sum_i |(M . X)[r, i] WT[i, j]|``.
    ``rows`` restricts the output to a subset of tokens.
    """
    X = np.asarray(X)
    mask = np.asarray(mask, dtype=bool)
    if rows is not None:
        X, mask = X[np.asarray(rows)], mask[np.asarray(rows)]
    Xm = np.where(mask, X.astype(np.float64), 0.0)
    W64 = np.asarray(WT).astype(np.float64)
    return Xm @ W64, np.abs(Xm) @ np.abs(W64)
