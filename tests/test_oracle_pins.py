"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

None of these re-types the oracle's formula or re-calls its library routine.
They use hand-derived fixtures (tests/golden/), exact rational arithmetic,
closed forms, brute force over all subsets on tiny inputs, pure-Python loops,
and reductions to the plain dense product.
"""
import itertools
import math
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import golden_path


# ---------------------------------------------------------------------------
# fixtures readers
# ---------------------------------------------------------------------------

def _floats(s):
    return [float(v) for v in s.split()]


def _read_lines(name):
    with open(golden_path(name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------
# fp16 round-to-nearest-even
# ---------------------------------------------------------------------------

def _fp16_exact(v: Fraction) -> Fraction:
    """Binary16 RNE by exact rational arithmetic (finite results only)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = math.floor(math.log2(a))
    # adjust for log2 rounding
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -14)                      # subnormals share the 2^-14 binade spacing
    ulp = Fraction(2) ** (e - 10)
    q, r = divmod(a, ulp)
    if r * 2 > ulp or (r * 2 == ulp and q % 2 == 1):
        q += 1
    return sign * q * ulp


def test_fp16_roundtrips_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16)
    back = oracle.fp16(h.astype(np.float64))
    nan = np.isnan(h)
    assert np.array_equal(back.view(np.uint16)[~nan], bits[~nan])
    assert np.isnan(back[nan]).all()


def test_fp16_halfway_and_off_halfway_against_exact_rationals():
    rng = np.random.default_rng(1)
    pos = np.arange(1, 0x7BFF, dtype=np.uint16)   # finite positives, a < b pairs
    pick = rng.choice(pos, 400, replace=False)
    picks = np.concatenate([pick, [1, 2, 0x3FF, 0x400, 0x401, 0x3BFF, 0x3C00, 0x7BFE]]).astype(np.uint16)
    for b in picks:
        a = np.array([b], dtype=np.uint16).view(np.float16)[0]
        c = np.array([b + 1], dtype=np.uint16).view(np.float16)[0]
        mid = (float(a) + float(c)) / 2.0           # exact in float64
        for v in (mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf)):
            want = _fp16_exact(Fraction(float(v)))
            got = Fraction(float(oracle.fp16(v)))
            assert got == want, (float(a), float(c), float(v))
            # and for the negative side
            assert Fraction(float(oracle.fp16(-v))) == -want


def test_fp16_overflow_and_underflow_edges():
    assert float(oracle.fp16(65504.0)) == 65504.0
    assert float(oracle.fp16(65519.99)) == 65504.0
    assert math.isinf(float(oracle.fp16(65520.0)))      # tie goes to even = 2^16 = inf
    assert float(oracle.fp16(2.0 ** -25)) == 0.0         # tie to even (0)
    assert float(oracle.fp16(np.nextafter(2.0 ** -25, 1.0))) == 2.0 ** -24


# ---------------------------------------------------------------------------
# masks
# ---------------------------------------------------------------------------

def test_threshold_golden():
    lines = _read_lines("threshold_small.txt")
    x = np.array(_floats(lines[0].split(":", 1)[1]), dtype=np.float16)
    n = 0
    for ln in lines[1:]:
        t, m = ln.split(":", 1)[1].split("|")
        want = np.array([int(v) for v in m.split()], dtype=bool)
        assert np.array_equal(oracle.threshold_mask(x, float(t)), want), ln
        n += 1
    assert n == 5


def test_threshold_matches_brute_force_loop_and_sorted_count():
    rng = np.random.default_rng(2)
    x = workloads.draw_vector(rng, 3001, "laplace")
    for s in (0.0, 0.25, 0.5, 0.65, 0.99):
        t = workloads.quantile_threshold(x, s)
        m = oracle.threshold_mask(x, t)
        loop = [abs(float(v)) >= t for v in x]
        assert m.tolist() == loop
        mags = sorted(abs(float(v)) for v in x)
        first = next(i for i, v in enumerate(mags) if v >= t)
        assert int(m.sum()) == len(mags) - first
        assert int(m.sum()) >= x.size - math.floor(s * x.size)


def test_threshold_is_a_float32_value():
    """The threshold is compared as the float32 value the layer receives: a t
    within half a float32 ulp above 0.5 is 0.5 (so |x| = 0.5 is kept), while
    0.5002 stays above 0.5 and below the next fp16 value 0.50048828125."""
    x = np.array([0.5, -0.5, 0.49975586, 0.50048828125], dtype=np.float16)
    assert list(oracle.threshold_mask(x, 0.5 + 1e-12)) == [True, True, False, True]
    assert list(oracle.threshold_mask(x, 0.5002)) == [False, False, False, True]
    assert np.float32(0.5 + 1e-12) == np.float32(0.5) and 0.5 + 1e-12 > 0.5


def test_threshold_never_keeps_nan_and_keeps_inf():
    x = np.array([np.nan, np.inf, -np.inf, 1.0], dtype=np.float16)
    assert oracle.threshold_mask(x, 0.0).tolist() == [False, True, True, True]


def test_topk_golden():
    lines = _read_lines("topk_small.txt")
    x = np.array(_floats(lines[0].split(":", 1)[1]), dtype=np.float16)
    for ln in lines[1:]:
        k, idx = ln.split(":", 1)[1].split("|")
        want = [int(v) for v in idx.split()]
        assert oracle.compact(oracle.topk_mask(x, int(k))).tolist() == want, ln


def _lexmin_maxsum_subset(vals, k):
    """All k-subsets; the max sum of |v| (exact in float64 for fp16 data),
    the lexicographically smallest sorted index tuple among the maxima."""
    best, best_set = None, None
    for sub in itertools.combinations(range(len(vals)), k):  # lexicographic order
        s = sum(abs(float(vals[i])) for i in sub)
        if best is None or s > best:
            best, best_set = s, sub
    return list(best_set) if best_set is not None else []


def test_topk_brute_force_tiny():
    rng = np.random.default_rng(3)
    for trial in range(60):
        d = int(rng.integers(1, 10))
        # few distinct magnitudes to force ties, random signs and signed zeros
        vals = rng.choice([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 2.0, 3.0, -3.0], size=d)
        x = np.array(vals, dtype=np.float16)
        for k in range(d + 1):
            got = oracle.compact(oracle.topk_mask(x, k)).tolist()
            assert got == _lexmin_maxsum_subset(x, k), (x, k)


def test_topk_invariants_large():
    rng = np.random.default_rng(4)
    x = workloads.draw_vector(rng, 28672, "student_t4")
    mags = np.abs(x.astype(np.float64))
    for f in workloads.QSPARSE_KEEP_FRACTIONS:
        k = workloads.topk_count(f, x.size)
        m = oracle.topk_mask(x, k)
        assert int(m.sum()) == k
        assert mags[m].min() >= mags[~m].max()
        kstar = mags[m].min()
        tie_kept = np.flatnonzero(m & (mags == kstar))
        tie_drop = np.flatnonzero(~m & (mags == kstar))
        if tie_drop.size:
            assert tie_kept.max() < tie_drop.min()
    assert workloads.topk_count(0.6, 8192) == 4915
    assert workloads.topk_count(0.4, 28672) == 11469


def test_topk_nan_ranks_last():
    x = np.array([np.nan, 0.0, np.inf, -1.0, np.nan], dtype=np.float16)
    assert oracle.compact(oracle.topk_mask(x, 3)).tolist() == [1, 2, 3]
    assert oracle.compact(oracle.topk_mask(x, 4)).tolist() == [0, 1, 2, 3]


def test_nm_golden():
    lines = _read_lines("nm_small.txt")
    row, checked = None, 0
    for ln in lines:
        if ln.startswith("row:"):
            row = np.array(_floats(ln[4:]), dtype=np.float16)
            continue
        nm, m = ln.split("|")
        n, mm = (int(v) for v in nm.split())
        want = np.array([int(v) for v in m.split()], dtype=bool)
        assert np.array_equal(oracle.nm_mask(row, n, mm), want), ln
        checked += 1
    assert checked == 8


def test_nm_pack_golden():
    lines = _read_lines("nm_packed_small.txt")
    row, checked = None, 0
    for ln in lines:
        if ln.startswith("row:"):
            row = np.array(_floats(ln[4:]), dtype=np.float16)
            continue
        head, vals, pos = ln.split("|")
        p = oracle.nm_pack_2of4(row, int(head))
        want_v = np.array(_floats(vals), dtype=np.float16)
        assert np.array_equal(p["values"][0].view(np.uint16), want_v.view(np.uint16)), ln
        assert p["positions"][0].tolist() == [int(v) for v in pos.split()], ln
        checked += 1
    assert checked == 4


@pytest.mark.parametrize("n", [2, 1])
def test_nm_pack_decodes_to_the_masked_block(n):
    """Scattering the slots back to their positions gives the masked X (bit
    for bit, +0 where dropped); positions ascend inside every block; a 1:4
    block pads at its smallest unkept position, with +0."""
    rng = np.random.default_rng(40 + n)
    X = rng.choice([0.0, -0.0, 0.5, -0.5, 1.0, 2.0, -2.0], size=(6, 64)).astype(np.float16)
    X[0, :5] = np.nan
    X = np.concatenate([X, rng.laplace(0, 1, (4, 64)).astype(np.float16)])
    p = oracle.nm_pack_2of4(X, n)
    rows, d = X.shape
    back = np.zeros_like(X)
    pos = p["positions"].reshape(rows, d // 4, 2).astype(int)
    vals = p["values"].reshape(rows, d // 4, 2)
    assert (pos[..., 0] < pos[..., 1]).all()
    for r in range(rows):
        for b in range(d // 4):
            for s in range(2):
                back[r, 4 * b + pos[r, b, s]] = vals[r, b, s]
    want = np.where(oracle.nm_mask(X, n, 4), X, np.float16(0))
    assert np.array_equal(back.view(np.uint16), want.view(np.uint16))
    if n == 1:
        kept = oracle.nm_mask(X, 1, 4).reshape(rows, d // 4, 4)
        first_free = np.argmax(~kept, axis=-1)
        pad_slot = np.where(np.take_along_axis(kept, pos, axis=-1), -1, pos).max(axis=-1)
        assert np.array_equal(pad_slot, first_free)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (3, 4), (4, 8), (8, 16)])
def test_nm_brute_force_blocks(n, m):
    rng = np.random.default_rng(5 + n + m)
    rows = []
    for _ in range(3):
        rows.append(rng.choice([0.0, -0.0, 0.25, -0.25, 1.0, -1.0, 2.0], size=m))
    rows.append(rng.laplace(0, 1, m))
    X = np.array(rows, dtype=np.float16)
    M = oracle.nm_mask(X, n, m)
    for r in range(X.shape[0]):
        assert int(M[r].sum()) == n
        assert oracle.compact(M[r]).tolist() == _lexmin_maxsum_subset(X[r], n)


def test_nm_exact_count_per_block_large():
    WT, X = workloads.nm_tokens(seed=0, rows=64, d=1024, d_out=8)
    for n, m in workloads.NM_PATTERNS:
        M = oracle.nm_mask(X, n, m)
        assert (M.reshape(64, -1, m).sum(-1) == n).all()
        assert abs(oracle.sparsity(M) - (1 - n / m)) < 1e-12


def test_nm_equals_topk_per_block():
    """An N:M mask is top-N applied to each block on its own."""
    rng = np.random.default_rng(6)
    X = rng.laplace(0, 1, (5, 64)).astype(np.float16)
    M = oracle.nm_mask(X, 8, 16)
    for r in range(5):
        for b in range(4):
            blk = X[r, 16 * b:16 * (b + 1)]
            assert np.array_equal(M[r, 16 * b:16 * (b + 1)], oracle.topk_mask(blk, 8))


def test_pack_bits_known_words():
    m = np.zeros(70, dtype=bool)
    m[[0, 31, 32, 69]] = True
    w = oracle.pack_bits(m)
    assert w.tolist() == [0x80000001, 0x1, 0x20]
    assert np.array_equal(oracle.unpack_bits(w, 70), m)


def test_compact_is_ascending_and_complete():
    m = np.array([0, 1, 1, 0, 0, 1], dtype=bool)
    assert oracle.compact(m).tolist() == [1, 2, 5]
    assert oracle.compact(np.zeros(4, bool)).tolist() == []


# ---------------------------------------------------------------------------
# product
# ---------------------------------------------------------------------------

def _triple_loop(W_rows, x, mask):
    """y_j = sum_i W[j][i] * m_i x_i with W in its natural (d_out, d_in)
    orientation, as the pages write W X ("Q-Sparse ...", A3)."""
    d_out, d_in = len(W_rows), len(x)
    y = []
    for j in range(d_out):
        acc = Fraction(0)
        for i in range(d_in):
            if mask[i]:
                acc += Fraction(float(W_rows[j][i])) * Fraction(float(x[i]))
        y.append(acc)
    return y


def test_product_matches_exact_triple_loop_nonsquare():
    rng = np.random.default_rng(7)
    d_in, d_out = 37, 23
    W = rng.normal(0, 0.02, (d_out, d_in)).astype(np.float16)      # natural orientation
    x = rng.laplace(0, 1, d_in).astype(np.float16)
    mask = oracle.threshold_mask(x, workloads.quantile_threshold(x, 0.4))
    y64, bound = oracle.masked_matvec(W.T.copy(), x, mask)
    exact = _triple_loop(W, x, mask)
    for j in range(d_out):
        assert abs(Fraction(float(y64[j])) - exact[j]) <= Fraction(1, 10 ** 12) * (1 + abs(exact[j]))
        b = sum(abs(Fraction(float(W[j, i])) * Fraction(float(x[i]))) for i in range(d_in) if mask[i])
        assert abs(Fraction(float(bound[j])) - b) <= Fraction(1, 10 ** 12) * (1 + b)


def test_product_identity_and_permutation():
    rng = np.random.default_rng(8)
    d = 64
    x = rng.laplace(0, 1, d).astype(np.float16)
    mask = oracle.topk_mask(x, 20)
    out = oracle.sparse_linear(np.eye(d, dtype=np.float16), x, mask)
    assert np.array_equal(out["y16"], np.where(mask, x, np.float16(0)))
    perm = rng.permutation(d)
    P = np.zeros((d, d), dtype=np.float16)          # y_j = x_{perm[j]}, so WT[perm[j], j] = 1
    P[perm, np.arange(d)] = 1
    out = oracle.sparse_linear(P, x, mask)
    assert np.array_equal(out["y16"], np.where(mask[perm], x[perm], np.float16(0)))


def test_zero_sparsity_reduces_to_dense_product():
    rng = np.random.default_rng(9)
    p = workloads.projection("t", 48, 40, sigma=0.02, dist="laplace", seed=9, sparsities=(0.0,))
    for mask in (oracle.threshold_mask(p.x, p.thresholds[0.0]),
                 oracle.topk_mask(p.x, p.d_in),
                 oracle.nm_mask(p.x, 4, 4)):
        assert mask.all()
        y64, _ = oracle.masked_matvec(p.WT, p.x, mask)
        exact = _triple_loop(p.WT.T, p.x, np.ones(p.d_in, bool))
        assert all(abs(Fraction(float(a)) - b) <= Fraction(1, 10 ** 12) for a, b in zip(y64, exact))


def test_empty_mask_gives_zero_output():
    p = workloads.projection("t", 16, 8, sigma=0.02, dist="laplace", seed=1)
    out = oracle.sparse_linear(p.WT, p.x, np.zeros(16, bool))
    assert out["nnz"] == 0 and not out["y64"].any() and not out["bound"].any()


def test_cols_subset_equals_full_columns():
    p = workloads.projection("t", 32, 24, sigma=0.02, dist="laplace", seed=2)
    m = oracle.topk_mask(p.x, 10)
    full, _ = oracle.masked_matvec(p.WT, p.x, m)
    cols = [3, 0, 23, 7]
    sub, _ = oracle.masked_matvec(p.WT, p.x, m, cols=cols)
    assert np.array_equal(sub, full[cols])


def test_flops_and_sparsity_definitions():
    # "Q-Sparse ...", A3: 2 d^2 for a d x d weight and a d x 1 input.
    assert oracle.flops(4096, 4096) == 2 * 4096 ** 2
    x = workloads.draw_vector(np.random.default_rng(3), 4096, "laplace")
    for s in workloads.LLAMA2_SPARSITIES:
        m = oracle.threshold_mask(x, workloads.quantile_threshold(x, s))
        # the Laplace draw has ties in fp16, so sparsity is at most the target
        assert oracle.sparsity(m) <= s + 1e-12
        assert oracle.flops(4096, int(m.sum())) == 2 * 4096 * int(m.sum())


# ---------------------------------------------------------------------------
# RaNA Eqn. 12
# ---------------------------------------------------------------------------

def _silu_decimal(z: float) -> Decimal:
    getcontext().prec = 40
    z = Decimal(z)
    return z / (1 + (-z).exp())


def test_silu_closed_forms():
    assert float(oracle.silu(0.0)) == 0.0
    ln3 = math.log(3.0)
    # sigmoid(ln 3) = 3/4 and sigmoid(-ln 3) = 1/4
    assert abs(float(oracle.silu(ln3)) - 0.75 * ln3) < 1e-15
    assert abs(float(oracle.silu(-ln3)) + 0.25 * ln3) < 1e-15
    zs = np.linspace(-30, 30, 241)
    # SiLU(z) - SiLU(-z) = z
    assert np.allclose(oracle.silu(zs) - oracle.silu(-zs), zs, atol=1e-13, rtol=0)
    for z in (-20.0, -3.5, -0.1, 0.7, 5.0, 30.0):
        assert abs(Decimal(float(oracle.silu(z))) - _silu_decimal(z)) <= Decimal(1e-15) * (1 + abs(_silu_decimal(z)))
    assert float(oracle.silu(-1000.0)) == 0.0


def _rana_fixture():
    lines = dict(ln.split(":", 1) for ln in _read_lines("rana_eqn12.txt"))
    return ({k: np.array(_floats(v)) for k, v in lines.items() if k in ("g", "u", "norm")},
            float(lines["t"]), [int(v) for v in lines["rana"].split()],
            [int(v) for v in lines["cats"].split()])


def test_rana_eqn12_golden_and_cats():
    vals, t, want_rana, want_cats = _rana_fixture()
    d_ff = vals["g"].size
    x = np.array([1.0], dtype=np.float16)
    WgT = vals["g"].astype(np.float16).reshape(1, d_ff)
    WuT = vals["u"].astype(np.float16).reshape(1, d_ff)
    norms = vals["norm"].astype(np.float32)
    g, u, h16 = oracle.rana_hidden(x, WgT, WuT)
    assert np.array_equal(g, vals["g"]) and np.array_equal(u, vals["u"])
    s = oracle.rana_scores(h16, norms)
    for i in range(d_ff):
        exact = abs(_silu_decimal(vals["g"][i]) * Decimal(vals["u"][i])) * Decimal(float(norms[i]))
        # h is rounded once to fp16 (rel. 2^-11) and s once more to fp32
        assert abs(Decimal(float(s[i])) - exact) <= exact * Decimal(2.0 ** -11 + 2.0 ** -23)
    assert oracle.rana_mask(s, t).astype(int).tolist() == want_rana
    # CATS ("RaNA ...", Q3) is Eqn. 12 with u = 1 and unit norms
    ones = np.ones((1, d_ff), np.float16)
    _, _, h_c = oracle.rana_hidden(x, WgT, ones)
    s_c = oracle.rana_scores(h_c, np.ones(d_ff, np.float32))
    assert oracle.rana_mask(s_c, t).astype(int).tolist() == want_cats
    for i in range(d_ff):
        assert abs(float(s_c[i]) - abs(float(_silu_decimal(vals["g"][i])))) <= 2.0 ** -11 * abs(float(s_c[i])) + 1e-30


def test_rana_cats_special_case_random():
    """u = 1 and norm = 1: the RaNA mask is |fp16(SiLU(g))| >= t, computed here
    with scalar math.exp, independent of numpy."""
    rng = np.random.default_rng(10)
    d_model, d_ff = 8, 300
    x = rng.normal(0, 1, d_model).astype(np.float16)
    WgT = rng.normal(0, 0.5, (d_model, d_ff)).astype(np.float16)
    WuT_ones = np.zeros((d_model, d_ff), np.float16)
    # u = 1: put 1/x_0 ... simpler: x_0 = 1 and the u weights only on row 0
    x[0] = 1.0
    WuT_ones[0, :] = 1.0
    g, u, h16 = oracle.rana_hidden(x, WgT, WuT_ones)
    assert (u == 1.0).all()
    s = oracle.rana_scores(h16, np.ones(d_ff, np.float32))
    t = 0.3
    m = oracle.rana_mask(s, t)
    for i in range(d_ff):
        gi = sum(float(x[k]) * float(WgT[k, i]) for k in range(d_model))
        silu = gi / (1.0 + math.exp(-gi))
        h = float(np.float16(silu))   # fp16 rounding; decision compared away from ties
        if abs(abs(silu) - t) > 1e-3:
            assert m[i] == (abs(h) >= t) == (abs(silu) >= t)


def test_rana_scale_invariance():
    """Doubling every norm and t leaves the mask unchanged (exact in fp32)."""
    rng = np.random.default_rng(11)
    h = rng.normal(0, 1, 500).astype(np.float16)
    norms = np.abs(rng.normal(1, 0.2, 500)).astype(np.float32)
    s1 = oracle.rana_scores(h, norms)
    s2 = oracle.rana_scores(h, norms * np.float32(2))
    assert np.array_equal(oracle.rana_mask(s1, 0.7), oracle.rana_mask(s2, 1.4))


def test_row_norms_pythagorean():
    WT = np.array([[3, 4, 0], [5, 12, 0], [1, 1, 1], [0, 0, 0]], dtype=np.float16)
    assert oracle.row_norms(WT).tolist() == [5.0, 13.0, float(np.float32(math.sqrt(3))), 0.0]


def test_gated_mlp_down_product_uses_h_and_mask():
    vals, t, want_rana, _ = _rana_fixture()
    d_ff = vals["g"].size
    x = np.array([1.0], dtype=np.float16)
    WgT = vals["g"].astype(np.float16).reshape(1, d_ff)
    WuT = vals["u"].astype(np.float16).reshape(1, d_ff)
    WdT = np.eye(d_ff, dtype=np.float16)         # y = m . h exactly
    out = oracle.gated_mlp(x, WgT, WuT, WdT, vals["norm"].astype(np.float32), t)
    want = np.where(np.array(want_rana, bool), out["h16"], np.float16(0))
    assert np.array_equal(out["y16"], want)


# ---------------------------------------------------------------------------
# batched N:M product
# ---------------------------------------------------------------------------

def test_nm_gemm_rows_equal_masked_matvec_and_triple_loop():
    WT, X = workloads.nm_tokens(seed=1, rows=6, d=32, d_out=5)
    M = oracle.nm_mask(X, 2, 4)
    Y, B = oracle.nm_gemm(X, WT, M)
    for r in range(6):
        exact = _triple_loop(WT.T, X[r], M[r])
        assert all(abs(Fraction(float(a)) - b) <= Fraction(1, 10 ** 12) for a, b in zip(Y[r], exact))
    Yn, _ = oracle.nm_gemm(X, WT, np.ones_like(M))
    exact = _triple_loop(WT.T, X[0], np.ones(32, bool))
    assert all(abs(Fraction(float(a)) - b) <= Fraction(1, 10 ** 12) for a, b in zip(Yn[0], exact))
    Ysub, _ = oracle.nm_gemm(X, WT, M, rows=[4, 1])
    assert np.array_equal(Ysub, Y[[4, 1]])


# ---------------------------------------------------------------------------
# input recipe
# ---------------------------------------------------------------------------

def test_quantile_threshold_hits_target_on_distinct_values():
    x = np.arange(1, 1001, dtype=np.float16)         # distinct magnitudes
    for s in (0.0, 0.25, 0.5, 0.65):
        t = workloads.quantile_threshold(x, s)
        assert int(oracle.threshold_mask(x, t).sum()) == 1000 - math.floor(s * 1000)


def test_workloads_are_seeded_and_chunking_invariant():
    a = workloads.tiny_gemv(0)
    b = workloads.tiny_gemv(0)
    assert np.array_equal(a.WT, b.WT) and np.array_equal(a.x, b.x)
    rng = np.random.default_rng(0)
    direct = rng.normal(0.0, 0.02, 1024 * 1024).astype(np.float16).reshape(1024, 1024)
    assert np.array_equal(direct, a.WT)
    assert a.thresholds[0.5] == workloads.quantile_threshold(a.x, 0.5)


# ---------------------------------------------------------------------------
# RaNA linear-layer rank adapter
# ---------------------------------------------------------------------------

def _rank_adapter_fixture():
    x, B, A, v, cases = None, [], [], None, []
    for ln in _read_lines("rank_adapter_tiny.txt"):
        if ln.startswith("x:"):
            x = _floats(ln[2:])
        elif ln.startswith("B:"):
            B.append(_floats(ln[2:]))
        elif ln.startswith("A:"):
            A.append(_floats(ln[2:]))
        elif ln.startswith("v:"):
            v = _floats(ln[2:])
        else:
            t, m, y = ln.split("|")
            cases.append((float(t), [int(c) for c in m.split()], _floats(y)))
    return (np.array(x, np.float16), np.array(B, np.float16), np.array(A, np.float16),
            np.array(v), cases)


def test_rank_adapter_golden():
    x, B, A, v, cases = _rank_adapter_fixture()
    v64, v16 = oracle.rank_adapter_hidden(x, B.T)
    assert v64.tolist() == v.tolist() and v16.astype(np.float64).tolist() == v.tolist()
    assert oracle.rank_adapter_scores(v16).tolist() == (v * v).tolist()
    for t, m, y in cases:
        out = oracle.rank_adapter(x, B.T, A.T, t)
        assert out["mask"].astype(int).tolist() == m, t
        assert out["y64"].tolist() == y, t


def test_rank_adapter_identity_b_is_the_threshold_layer():
    """B = I makes v = x exactly; the square of an fp16 value is exact in fp32,
    so v_i^2 >= c^2 is |x_i| >= c and the adapter is the threshold layer on A."""
    rng = np.random.default_rng(21)
    d, d_out = 300, 40
    x = rng.laplace(0, 1, d).astype(np.float16)
    AT = rng.normal(0, 0.02, (d, d_out)).astype(np.float16)
    eye = np.eye(d, dtype=np.float16)
    for c in (0.0, 0.25, float(np.sort(np.abs(x))[150]), 3.0):
        out = oracle.rank_adapter(x, eye, AT, c * c)
        ref = oracle.sparse_linear(AT, x, oracle.threshold_mask(x, c))
        assert np.array_equal(out["mask"], ref["mask"])
        assert np.array_equal(out["y64"], ref["y64"])


def test_rank_adapter_masked_rows_do_not_matter():
    """Rows of A^T whose mask entry is 0 never reach y ([RaNA] Q5.1)."""
    rng = np.random.default_rng(22)
    d_in, r, d_out = 64, 48, 24
    x = rng.normal(0, 1, d_in).astype(np.float16)
    BT = rng.normal(0, 0.2, (d_in, r)).astype(np.float16)
    AT = rng.normal(0, 0.2, (r, d_out)).astype(np.float16)
    out = oracle.rank_adapter(x, BT, AT, 1.0)
    assert 0 < out["nnz"] < r
    AT2 = AT.copy()
    AT2[~out["mask"]] = np.float16(1000.0)
    assert np.array_equal(oracle.rank_adapter(x, BT, AT2, 1.0)["y64"], out["y64"])
    # t = 0 keeps every finite v: the unmasked two-GEMV product
    dense = oracle.rank_adapter(x, BT, AT, 0.0)
    assert dense["nnz"] == r
    v16 = dense["v16"].astype(np.float64)
    want = [sum(v16[i] * float(AT[i, j]) for i in range(r)) for j in range(d_out)]
    assert np.allclose(dense["y64"], want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# A few tokens with their own masks
# ---------------------------------------------------------------------------

def test_batched_tokens_golden():
    WT, xs, ms, ys, t, union = [], [], [], [], None, None
    for ln in _read_lines("batched_tokens_tiny.txt"):
        if ln.startswith("WT:"):
            WT.append(_floats(ln[3:]))
        elif ln.startswith("t:"):
            t = float(ln[2:])
        elif ln.startswith("union:"):
            union = [int(v) for v in ln[6:].split()]
        elif ln.startswith("x:"):
            x, m, y = ln[2:].split("|")
            xs.append(_floats(x)); ms.append([int(v) for v in m.split()]); ys.append(_floats(y))
    WT = np.array(WT, np.float16)
    X = np.array(xs, np.float16)
    masks = np.stack([oracle.threshold_mask(x, t) for x in X])
    assert masks.astype(int).tolist() == ms
    out = oracle.batched_sparse_linear(WT, X, masks)
    assert out["y64"].tolist() == ys
    assert out["union"].astype(int).tolist() == union


def test_batched_tokens_properties():
    """One token is the single-token product; permuting tokens permutes the
    outputs; rows outside the union never matter; identical tokens agree."""
    rng = np.random.default_rng(31)
    d_in, d_out, B = 96, 40, 5
    WT = rng.normal(0, 0.05, (d_in, d_out)).astype(np.float16)
    X = rng.laplace(0, 1, (B, d_in)).astype(np.float16)
    t = 1.2
    masks = np.stack([oracle.threshold_mask(x, t) for x in X])
    out = oracle.batched_sparse_linear(WT, X, masks)
    one = oracle.sparse_linear(WT, X[2], masks[2])
    assert np.array_equal(out["y64"][2], one["y64"])
    perm = np.array([3, 0, 4, 1, 2])
    outp = oracle.batched_sparse_linear(WT, X[perm], masks[perm])
    assert np.array_equal(outp["y64"], out["y64"][perm])
    assert 0 < out["union"].sum() < d_in
    WT2 = WT.copy()
    WT2[~out["union"]] = np.float16(500.0)
    assert np.array_equal(oracle.batched_sparse_linear(WT2, X, masks)["y64"], out["y64"])
    Xs = np.repeat(X[:1], 3, axis=0)
    ms = np.repeat(masks[:1], 3, axis=0)
    same = oracle.batched_sparse_linear(WT, Xs, ms)["y64"]
    assert np.array_equal(same[0], same[1]) and np.array_equal(same[1], same[2])
    assert np.array_equal(oracle.union_mask(ms), masks[0])


# ---------------------------------------------------------------------------
# Weight-quantised sparse product
# ---------------------------------------------------------------------------

def test_q8_golden():
    Q, vals = [], {}
    for ln in _read_lines("q8_tiny.txt"):
        key, v = ln.split(":", 1)
        if key == "Q":
            Q.append([int(c) for c in v.split()])
        else:
            vals[key] = v
    QT = np.array(Q, np.int8)
    x = np.array(_floats(vals["x"]), np.float16)
    m = oracle.threshold_mask(x, float(vals["t"]))
    assert m.astype(int).tolist() == [int(c) for c in vals["mask"].split()]
    out = oracle.q8_sparse_linear(QT, np.array(_floats(vals["scale"]), np.float32), x, m)
    assert out["y64"].tolist() == _floats(vals["y"])


def test_q8_is_the_fp16_product_on_exact_dequantised_weights():
    """With power-of-two scales, s_j * q_ij is exact in fp16, and the
    quantised product equals the fp16 product on those weights exactly."""
    rng = np.random.default_rng(41)
    d_in, d_out = 200, 48
    QT = rng.integers(-127, 128, (d_in, d_out)).astype(np.int8)
    scale = (2.0 ** -rng.integers(6, 10, d_out)).astype(np.float32)
    WT = (QT.astype(np.float64) * scale.astype(np.float64)).astype(np.float16)
    assert np.array_equal(WT.astype(np.float64), QT.astype(np.float64) * scale.astype(np.float64))
    x = rng.laplace(0, 1, d_in).astype(np.float16)
    m = oracle.threshold_mask(x, 0.8)
    a = oracle.q8_sparse_linear(QT, scale, x, m)
    b = oracle.sparse_linear(WT, x, m)
    assert np.array_equal(a["y64"], b["y64"]) and np.array_equal(a["bound"], b["bound"])
    cols = np.array([0, 7, 47])
    c = oracle.q8_sparse_linear(QT, scale, x, m, cols=cols)
    assert np.array_equal(c["y64"], a["y64"][cols])


# ---------------------------------------------------------------------------
# N:M selection and mitigation variants
# ---------------------------------------------------------------------------

def _nmv_fixture():
    f = {}
    for ln in _read_lines("nm_variants_tiny.txt"):
        k, v = ln.split(":", 1)
        f[k] = [part.strip() for part in v.split("|")]
    return f


def test_nm_variants_golden():
    f = _nmv_fixture()
    x = np.array([_floats(f["act"][0])], np.float16)
    assert oracle.nm_variant(x, 2, 4)["mask"].astype(int)[0].tolist() == [int(v) for v in f["act"][1].split()]
    norms = np.array(_floats(f["wt"][1]), np.float32)
    out = oracle.nm_variant(x, 2, 4, norms=norms)
    assert out["mask"].astype(int)[0].tolist() == [int(v) for v in f["wt"][2].split()]
    xp = np.array([_floats(f["pts"][0])], np.float16)
    mu = np.array([float(f["pts"][1])], np.float32)
    out = oracle.nm_variant(xp, 2, 4, shift=mu, var=True)
    assert out["xs"].astype(np.float64)[0].tolist() == _floats(f["pts"][2])
    assert out["mask"].astype(int)[0].tolist() == [int(v) for v in f["pts"][3].split()]
    full, kept = _floats(f["var"][0])
    assert out["gamma"][0] == pytest.approx(math.sqrt(full / kept), rel=1e-15)
    WT = np.array([[1, 0], [0, 1], [1, 1], [2, -1]], np.float16)
    all_kept = oracle.nm_variant(xp, 4, 4, shift=mu)
    Y, _ = oracle.nm_variant_gemm(all_kept["xm64"], WT, shift=mu)
    assert Y[0].tolist() == _floats(f["gemm"][0])
    assert Y[0].tolist() == (xp.astype(np.float64) @ WT.astype(np.float64))[0].tolist()


def test_nm_variants_reduce_to_plain_nm():
    rng = np.random.default_rng(51)
    X = rng.choice([0.0, 0.5, -0.5, 1.0, -2.0, 3.0], size=(6, 64)).astype(np.float16)
    X[0, :5] = np.nan
    for n, m in ((2, 4), (1, 4), (3, 8), (8, 16), (16, 32)):
        plain = oracle.nm_mask(X, n, m)
        out = oracle.nm_variant(X, n, m)
        assert np.array_equal(out["mask"], plain)
        assert np.array_equal(out["xm16"].view(np.uint16), np.where(plain, X, np.float16(0)).view(np.uint16))
        # scoring by |x| itself, or WT with equal power-of-two norms, is ACT
        by_score = oracle.nm_mask_by_score(np.abs(X.astype(np.float32)), n, m)
        assert np.array_equal(by_score, plain)
        wt = oracle.nm_variant(X, n, m, norms=np.full(64, 2.0, np.float32))
        assert np.array_equal(wt["mask"], plain)
        # a zero shift changes nothing
        z = oracle.nm_variant(X, n, m, shift=np.zeros(6, np.float32))
        assert np.array_equal(z["mask"], plain)


def test_var_restores_the_row_norm():
    rng = np.random.default_rng(52)
    X = rng.laplace(0, 1, (5, 128)).astype(np.float16)
    out = oracle.nm_variant(X, 2, 4, shift=rng.normal(0, 0.1, 5).astype(np.float32), var=True)
    xs = out["xs"].astype(np.float64)
    assert np.allclose(np.linalg.norm(out["xm64"], axis=1), np.linalg.norm(xs, axis=1), rtol=1e-13)
    zero = oracle.var_gamma(np.zeros((1, 8), np.float16), np.ones((1, 8), bool))
    assert zero.tolist() == [1.0]


# ---------------------------------------------------------------------------
# Gated MLP with TEAL thresholds on both inputs
# ---------------------------------------------------------------------------

def test_teal_mlp_reductions():
    """t_x = 0 keeps every input: g, u and h are those of the dense gated MLP;
    t_h = 0 then makes y the dense down product of h; an empty input mask
    gives g = u = 0, h = 0 and y = 0."""
    rng = np.random.default_rng(61)
    d_model, d_ff = 24, 40
    x = rng.normal(0, 1, d_model).astype(np.float16)
    WgT = rng.normal(0, 0.3, (d_model, d_ff)).astype(np.float16)
    WuT = rng.normal(0, 0.3, (d_model, d_ff)).astype(np.float16)
    WdT = rng.normal(0, 0.3, (d_ff, d_model)).astype(np.float16)
    g, u, h = oracle.rana_hidden(x, WgT, WuT)
    out = oracle.teal_mlp(x, WgT, WuT, WdT, 0.0, 0.0)
    assert np.array_equal(out["g"], g) and np.array_equal(out["u"], u)
    assert np.array_equal(out["h16"].view(np.uint16), h.view(np.uint16))
    dense = oracle.sparse_linear(WdT, h, np.ones(d_ff, bool))
    assert np.array_equal(out["y64"], dense["y64"])
    none = oracle.teal_mlp(x, WgT, WuT, WdT, float("inf"), 0.0)
    assert not none["mask_x"].any() and not np.any(none["h16"].astype(np.float64))
    assert not np.any(none["y64"])
    # the input mask acts on the rows of W_gate and W_up: dropping x_i equals zeroing it
    t = float(np.sort(np.abs(x.astype(np.float64)))[12])
    part = oracle.teal_mlp(x, WgT, WuT, WdT, t, 0.3)
    x0 = np.where(oracle.threshold_mask(x, t), x, np.float16(0))
    g0, u0, h0 = oracle.rana_hidden(x0, WgT, WuT)
    assert np.array_equal(part["h16"].view(np.uint16), h0.view(np.uint16))
    assert np.array_equal(part["mask"], oracle.threshold_mask(h0, 0.3))


def test_int4_decode_by_hand_and_by_arithmetic_shifts():
    """Nibble decoding of the packed int4 weights: bytes worked out by hand
    (low nibble first), then all 256 bytes against sign extension by an
    arithmetic right shift of the nibble moved to the top of an int8."""
    v = oracle.int4_values(np.array([[0x00, 0x7F, 0x80, 0x8F, 0x21, 0xF7]], np.uint8))
    assert v.tolist() == [[0, 0, -1, 7, 0, -8, -1, -8, 1, 2, 7, -1]]
    codes = np.arange(256, dtype=np.uint8)
    lo = (codes << 4).astype(np.uint8).view(np.int8) >> 4
    hi = codes.view(np.int8) >> 4
    dec = oracle.int4_values(codes.reshape(1, 256))[0]
    assert np.array_equal(dec[0::2], lo) and np.array_equal(dec[1::2], hi)
    assert dec.min() == -8 and dec.max() == 7


def test_q4_product_is_the_int8_product_on_the_decoded_weights():
    """The int4 product equals the (golden-pinned) int8 product on the decoded
    weights exactly, and a brute-force double loop."""
    rng = np.random.default_rng(14)
    QT4 = rng.integers(0, 256, (36, 12), dtype=np.uint8)
    scale = rng.uniform(0.5, 2.0, 24).astype(np.float32)
    x = rng.laplace(0, 1, 36).astype(np.float16)
    m = oracle.threshold_mask(x, 0.6)
    a = oracle.q4_sparse_linear(QT4, scale, x, m)
    Q = oracle.int4_values(QT4)
    b = oracle.q8_sparse_linear(Q, scale, x, m)
    assert np.array_equal(a["y64"], b["y64"]) and np.array_equal(a["bound"], b["bound"])
    brute = [float(scale[j]) * sum(int(Q[i, j]) * float(x[i]) for i in range(36) if m[i])
             for j in range(24)]
    assert np.allclose(a["y64"], brute, rtol=1e-12, atol=1e-12)
    cols = np.array([1, 10, 23])
    c = oracle.q4_sparse_linear(QT4, scale, x, m, cols=cols)
    assert np.array_equal(c["y64"], a["y64"][cols])


def test_e4m3_decode_matches_the_library_format_and_closed_forms():
    """Every one of the 256 e4m3 codes against torch's float8_e4m3fn (an
    independent implementation of the same published format), plus values
    worked out by hand from the definition."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], lib[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(lib[ok]))
    v = oracle.e4m3_value
    assert v(0x38) == 1.0 and v(0xB8) == -1.0          # exponent 7 = bias, mantissa 0
    assert v(0x7E) == 448.0                             # largest finite: 2^8 * 1.75
    assert v(0x01) == 2.0 ** -9 and v(0x08) == 2.0 ** -6   # smallest subnormal, smallest normal
    assert v(0x07) == 7 * 2.0 ** -9                     # largest subnormal
    assert np.isnan(v(0x7F)) and np.isnan(v(0xFF)) and np.signbit(v(0x80))
    pos = ours[:0x7F]
    assert (np.diff(pos) > 0).all()                    # codes 0 .. 0x7E increase


def test_f8_product_is_the_fp16_product_on_exact_decoded_weights():
    """With every scale 1 the fp8 product equals the plain masked product on
    the decoded weights, and the per-column scale multiplies column j."""
    rng = np.random.default_rng(12)
    QT = rng.integers(0, 256, (40, 24), dtype=np.uint8)
    QT[(QT & 0x7F) == 0x7F] = 0x38                      # no NaN codes
    x = rng.laplace(0, 1, 40).astype(np.float16)
    m = oracle.threshold_mask(x, 0.7)
    W = oracle.e4m3_value(QT)
    ref = oracle.masked_matvec(W, x, m)
    out = oracle.f8_sparse_linear(QT, np.ones(24, np.float32), x, m)
    assert np.allclose(out["y64"], ref[0], rtol=0, atol=0)
    sc = rng.uniform(0.5, 2.0, 24).astype(np.float32)
    out2 = oracle.f8_sparse_linear(QT, sc, x, m)
    assert np.array_equal(out2["y64"], ref[0] * sc.astype(np.float64))
    brute = np.array([sum(float(W[i, j]) * float(x[i]) for i in range(40) if m[i]) for j in range(24)])
    assert np.allclose(out["y64"], brute, rtol=1e-12, atol=1e-12)

