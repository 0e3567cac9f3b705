"""GPU parity of the threshold / top-k masks and the split-K sparse GEMV.

Every call goes through the C ABI (the ctypes binding); every expected value
comes from the CPU oracle on the same seeded inputs.  Masks and index lists
are compared bit for bit; outputs element by element within
|y - y64| <= 2e-3 * sum_i |W_ij x_i|.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, mask_words, to_dev, to_host

pytestmark = pytest.mark.gpu


def _check_threshold(sig, WT, x, t, what):
    ref = oracle.sparse_linear(WT, x, oracle.threshold_mask(x, t))
    dW, dx = to_dev(WT), to_dev(x)
    y = to_host(sig.sparse_gemv(dW, dx, t=t))
    assert_within(y, ref["y64"], ref["bound"], what)
    mb, idx, nnz = sig.sparsify_threshold(dx, t)
    n = int(to_host(nnz)[0])
    assert n == ref["nnz"], what
    assert np.array_equal(mask_words(mb), oracle.pack_bits(ref["mask"])), what
    assert np.array_equal(to_host(idx)[:n], ref["idx"]), what
    return y, ref


def test_tiny_config(sig):
    p = workloads.tiny_gemv(0)
    _check_threshold(sig, p.WT, p.x, p.thresholds[0.5], "tiny 1024x1024 @ 50%")


@pytest.mark.parametrize("d_in,d_out", [(1, 8), (7, 16), (33, 24), (100, 264), (257, 1000),
                                        (1000, 2056), (2049, 520), (5000, 4104), (31, 4096)])
def test_ragged_shapes(sig, d_in, d_out):
    p = workloads.projection("r", d_in, d_out, sigma=0.02, dist="laplace", seed=d_in * 7 + d_out,
                             sparsities=(0.0, 0.3, 0.5, 0.9))
    for s, t in p.thresholds.items():
        _check_threshold(sig, p.WT, p.x, t, f"{d_in}x{d_out} s={s}")


def test_threshold_between_fp16_values_and_not_a_float32(sig):
    """t reaches the library as a float32: 0.5 + 1e-12 arrives as 0.5 (|x| =
    0.5 kept), 0.5002 as a float32 between two fp16 values (0.5 dropped,
    0.50048828125 kept).  The oracle rounds t to float32 the same way."""
    rng = np.random.default_rng(21)
    WT = workloads.draw_weight(rng, 1000, 264, 0.02)
    x = rng.choice([0.5, -0.5, 0.49975586, 0.50048828125, -0.50048828125, 1.0, 0.0],
                   size=1000).astype(np.float16)
    for t in (0.5 + 1e-12, 0.5002, 0.50048828125 - 1e-9):
        _check_threshold(sig, WT, x, t, f"t={t!r}")


def test_empty_and_full_masks(sig):
    p = workloads.projection("e", 300, 136, sigma=0.02, dist="laplace", seed=5)
    y, ref = _check_threshold(sig, p.WT, p.x, float("inf"), "empty mask")
    assert ref["nnz"] == 0 and not np.any(y.astype(np.float64))
    assert np.all(y.view(np.uint16) == 0)      # +0, not -0 or NaN
    _check_threshold(sig, p.WT, p.x, 0.0, "full mask")
    # the explicit index path with nnz = 0
    import torch
    dW, dx = to_dev(p.WT), to_dev(p.x)
    idx = torch.zeros(300, dtype=torch.int32, device="cuda")
    nnz = torch.zeros(1, dtype=torch.int32, device="cuda")
    y2 = to_host(sig.sparse_gemv(dW, dx, idx=idx, nnz=nnz))
    assert np.all(y2.view(np.uint16) == 0)


def test_wide_slice_path(sig):
    """d_out above 296 column tiles: one slice per tile, so a slice owns all
    257 input groups and the prologue takes the chunked path of mask words
    and per-chunk placement (the one-group-per-thread path stops at 256)."""
    p = workloads.projection("w", 2056, 76032, sigma=0.02, dist="laplace", seed=19,
                             sparsities=(0.5,))
    t = p.thresholds[0.5]
    cols = np.concatenate([np.arange(16), np.random.default_rng(3).choice(76032, 240, replace=False),
                           np.arange(76032 - 16, 76032)])
    y = to_host(sig.sparse_gemv(to_dev(p.WT), to_dev(p.x), t=t))
    ref = oracle.sparse_linear(p.WT, p.x, oracle.threshold_mask(p.x, t), cols=cols)
    assert_within(y[cols], ref["y64"], ref["bound"], "wide slices")


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.99])
def test_largest_input_width(sig, sparsity):
    """d_in = SIG_MAX_D_IN (131072): one column tile, 64 slices of 256 input
    groups each (the widest slice of the one-group-per-thread prologue); also
    the index path over the same rows."""
    p = workloads.projection("m", 131072, 64, sigma=0.02, dist="laplace", seed=23,
                             sparsities=(sparsity,))
    t = p.thresholds[sparsity]
    dW, dx = to_dev(p.WT), to_dev(p.x)
    ref = oracle.sparse_linear(p.WT, p.x, oracle.threshold_mask(p.x, t))
    y = to_host(sig.sparse_gemv(dW, dx, t=t))
    assert_within(y, ref["y64"], ref["bound"], f"d_in 131072 s={sparsity}")
    mb, idx, nnz = sig.sparsify_threshold(dx, t)
    assert int(to_host(nnz)[0]) == ref["nnz"]
    y2 = to_host(sig.sparse_gemv(dW, dx, idx=idx, nnz=nnz))
    assert_within(y2, ref["y64"], ref["bound"], f"d_in 131072 s={sparsity} index list")


def test_slice_rows_in_several_chunks(sig):
    """One slice per tile (d_out above 296 tiles) over 4200 kept inputs: the
    chunked prologue places the slice's rows in two chunks (at most 4096 rows
    of a slice are staged in shared memory at once)."""
    p = workloads.projection("c", 4200, 76032, sigma=0.02, dist="laplace", seed=31,
                             sparsities=(0.0,))
    t = p.thresholds[0.0]
    cols = np.concatenate([np.arange(16), np.random.default_rng(7).choice(76032, 240, replace=False),
                           np.arange(76032 - 16, 76032)])
    y = to_host(sig.sparse_gemv(to_dev(p.WT), to_dev(p.x), t=t))
    ref = oracle.sparse_linear(p.WT, p.x, oracle.threshold_mask(p.x, t), cols=cols)
    assert ref["nnz"] == 4200
    assert_within(y[cols], ref["y64"], ref["bound"], "two chunks")


def test_widest_output(sig):
    """d_out = 2^20 (4096 column tiles, one slice each, no workspace)."""
    p = workloads.projection("n", 8, 1 << 20, sigma=0.02, dist="laplace", seed=29,
                             sparsities=(0.5,))
    t = p.thresholds[0.5]
    assert sig.workspace_bytes(sig.OP_SPARSE_GEMV, 8, 1 << 20) == 0
    y = to_host(sig.sparse_gemv(to_dev(p.WT), to_dev(p.x), t=t))
    cols = np.concatenate([np.arange(64), np.random.default_rng(5).choice(1 << 20, 448, replace=False),
                           np.arange((1 << 20) - 64, 1 << 20)])
    ref = oracle.sparse_linear(p.WT, p.x, oracle.threshold_mask(p.x, t), cols=cols)
    assert_within(y[cols], ref["y64"], ref["bound"], "d_out 2^20")


def test_index_path_and_fused_path_agree(sig):
    # the two paths split the kept rows differently (interleaved 8-input groups
    # under a threshold, equal runs of an index list), so they agree within the
    # bound, each one bit for bit with itself
    p = workloads.projection("i", 4096, 4096, sigma=0.02, dist="laplace", seed=11,
                             sparsities=(0.5,))
    dW, dx = to_dev(p.WT), to_dev(p.x)
    t = p.thresholds[0.5]
    ref = oracle.sparse_linear(p.WT, p.x, oracle.threshold_mask(p.x, t))
    y_fused = to_host(sig.sparse_gemv(dW, dx, t=t))
    _, idx, nnz = sig.sparsify_threshold(dx, t)
    y_idx = to_host(sig.sparse_gemv(dW, dx, idx=idx, nnz=nnz))
    assert_within(y_fused, ref["y64"], ref["bound"], "fused")
    assert_within(y_idx, ref["y64"], ref["bound"], "index list")
    assert np.array_equal(y_idx.view(np.uint16),
                          to_host(sig.sparse_gemv(dW, dx, idx=idx, nnz=nnz)).view(np.uint16))


def test_out_of_range_indices_are_skipped(sig):
    import torch
    p = workloads.projection("o", 64, 64, sigma=0.02, dist="laplace", seed=3)
    good = np.array([1, 5, 9, 40], dtype=np.int32)
    idx = np.array([1, 5, -3, 9, 64, 40, 1 << 30], dtype=np.int32)
    dW, dx = to_dev(p.WT), to_dev(p.x)
    y = to_host(sig.sparse_gemv(dW, dx, idx=to_dev(idx),
                                nnz=torch.tensor([idx.size], dtype=torch.int32, device="cuda")))
    m = np.zeros(64, bool)
    m[good] = True
    ref = oracle.sparse_linear(p.WT, p.x, m)
    assert_within(y, ref["y64"], ref["bound"], "skip invalid")
    # nnz larger than d_in is clamped
    idx2 = np.arange(64, dtype=np.int32)
    y2 = to_host(sig.sparse_gemv(dW, dx, idx=to_dev(idx2),
                                 nnz=torch.tensor([1000], dtype=torch.int32, device="cuda")))
    ref2 = oracle.sparse_linear(p.WT, p.x, np.ones(64, bool))
    assert_within(y2, ref2["y64"], ref2["bound"], "clamped nnz")


def test_bitwise_determinism(sig):
    p = workloads.projection("d", 11008, 4096, sigma=0.02, dist="laplace", seed=4,
                             sparsities=(0.4,))
    dW, dx = to_dev(p.WT), to_dev(p.x)
    t = p.thresholds[0.4]
    first = to_host(sig.sparse_gemv(dW, dx, t=t)).view(np.uint16).copy()
    for _ in range(5):
        again = to_host(sig.sparse_gemv(dW, dx, t=t)).view(np.uint16)
        assert np.array_equal(first, again)


@pytest.mark.parametrize("name", ["q", "gate", "down"])
def test_llama2_7b_projection_all_sparsities(sig, name):
    (p,) = workloads.llama2_7b(0, names=(name,))
    dW, dx = to_dev(p.WT), to_dev(p.x)
    W64 = None
    for s, t in p.thresholds.items():
        m = oracle.threshold_mask(p.x, t)
        ref = oracle.sparse_linear(p.WT, p.x, m)
        y = to_host(sig.sparse_gemv(dW, dx, t=t))
        assert_within(y, ref["y64"], ref["bound"], f"llama2-7b {name} s={s}")
        mb, idx, nnz = sig.sparsify_threshold(dx, t)
        assert int(to_host(nnz)[0]) == ref["nnz"]
        assert np.array_equal(mask_words(mb), oracle.pack_bits(m))
    del W64


# ---------------------------------------------------------------------------
# several weights sharing one input (q, k, v; gate, up)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d_in,d_outs", [(4096, (4096, 4096, 4096)), (4096, (11008, 11008)),
                                         (1000, (4096, 1024, 1024)), (257, (264, 8, 1000, 4104))])
def test_multi_weight_threshold(sig, d_in, d_outs):
    rng = np.random.default_rng(d_in + sum(d_outs))
    x = workloads.draw_vector(rng, d_in, "laplace")
    Ws = [workloads.draw_weight(rng, d_in, d, 0.02) for d in d_outs]
    t = workloads.quantile_threshold(x, 0.5)
    m = oracle.threshold_mask(x, t)
    ys = sig.sparse_gemv_multi([to_dev(W) for W in Ws], to_dev(x), t=t)
    for p, (W, y) in enumerate(zip(Ws, ys)):
        ref = oracle.sparse_linear(W, x, m)
        assert_within(to_host(y), ref["y64"], ref["bound"], f"multi weight {p} of {d_outs}")


def test_multi_weight_index_path_and_single_weight_equivalence(sig):
    layer = workloads.llama2_7b_layer(0)
    q, k, v = layer[0], layer[1], layer[2]
    assert q.x is k.x and q.x is v.x
    dx = to_dev(q.x)
    kk = workloads.topk_count(0.5, q.d_in)
    mb, idx, nnz = sig.sparsify_topk(dx, kk)
    m = oracle.topk_mask(q.x, kk)
    ys = sig.sparse_gemv_multi([to_dev(p.WT) for p in (q, k, v)], dx, idx=idx, nnz=nnz)
    for p, y in zip((q, k, v), ys):
        ref = oracle.sparse_linear(p.WT, p.x, m)
        assert_within(to_host(y), ref["y64"], ref["bound"], f"multi idx {p.name}")
    # one weight through the multi entry point is the single-weight call
    dW = to_dev(q.WT)
    t = q.thresholds[0.5]
    (y1,) = sig.sparse_gemv_multi([dW], dx, t=t)
    y2 = sig.sparse_gemv(dW, dx, t=t)
    assert np.array_equal(to_host(y1).view(np.uint16), to_host(y2).view(np.uint16))


# ---------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------

def _check_topk(sig, x, k, what):
    mb, idx, nnz = sig.sparsify_topk(to_dev(x), k)
    m = oracle.topk_mask(x, k)
    assert int(to_host(nnz)[0]) == k, what
    assert np.array_equal(mask_words(mb), oracle.pack_bits(m)), what
    assert np.array_equal(to_host(idx)[:k], oracle.compact(m)), what
    return mb, idx, nnz


@pytest.mark.parametrize("d", [1, 2, 31, 33, 1000, 8192, 12288, 12289, 28672, 32767, 65537, 131072])
def test_topk_masks_random(sig, d):
    x = workloads.draw_vector(np.random.default_rng(d), d, "student_t4")
    for k in sorted({0, 1, d // 3, d // 2, workloads.topk_count(0.6, d), d - 1, d}):
        if 0 <= k <= d:
            _check_topk(sig, x, k, f"d={d} k={k}")


def test_topk_heavy_ties_and_specials(sig):
    rng = np.random.default_rng(9)
    x = rng.choice([0.0, -0.0, 1.0, -1.0, 0.5, -0.5, 2.0], size=5000).astype(np.float16)
    for k in (0, 1, 17, 700, 2500, 4999, 5000):
        _check_topk(sig, x, k, f"ties k={k}")
    x = np.full(777, 3.0, dtype=np.float16)
    x[::2] = -3.0
    for k in (1, 100, 776):
        _check_topk(sig, x, k, f"all equal k={k}")
    x = rng.standard_normal(600).astype(np.float16)
    x[[3, 77, 300]] = np.nan
    x[[5, 500]] = np.inf
    x[[6]] = -np.inf
    x[[10, 11]] = 65504.0
    x[[12]] = np.float16(6e-8)     # subnormal
    for k in (1, 3, 4, 100, 597, 598, 600):
        _check_topk(sig, x, k, f"specials k={k}")
    # ties that span the CTAs of the cluster path
    x = rng.choice([0.5, -1.0, 1.0, 2.0, -0.0], size=40000).astype(np.float16)
    for k in (1, 7999, 8000, 13333, 20000, 31999, 39999, 40000):
        _check_topk(sig, x, k, f"cluster ties k={k}")
    x = np.full(70001, -7.0, dtype=np.float16)
    for k in (1, 35000, 70000):
        _check_topk(sig, x, k, f"cluster all equal k={k}")


@pytest.mark.parametrize("name", ["up", "down"])
def test_qsparse_70b_topk_then_gemv(sig, name):
    (p,) = workloads.qsparse_70b(0, names=(name,))
    dW, dx = to_dev(p.WT), to_dev(p.x)
    cols = np.unique(np.concatenate([np.random.default_rng(1).choice(p.d_out, 384, replace=False),
                                     [0, 1, p.d_out - 1]]))
    for f in workloads.QSPARSE_KEEP_FRACTIONS:
        k = workloads.topk_count(f, p.d_in)
        mb, idx, nnz = _check_topk(sig, p.x, k, f"70b {name} f={f}")
        y = to_host(sig.sparse_gemv(dW, dx, idx=idx, nnz=nnz))
        ref = oracle.sparse_linear(p.WT, p.x, oracle.topk_mask(p.x, k), cols=cols)
        assert_within(y[cols], ref["y64"], ref["bound"], f"70b {name} f={f}")
        assert np.isfinite(y.astype(np.float32)).all()
