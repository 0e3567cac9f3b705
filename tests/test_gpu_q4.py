"""GPU parity of the sparse GEMV with int4 weights, two to a byte, and one
float32 scale per output column (TEAL README, Limitations; Q-Sparse rebuttal,
A1: quantisation is orthogonal to activation sparsity).  Every output is
compared with the oracle within |y - y64| <= 2e-3 * |s_j| * sum_i |q_ij m_i x_i|."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu


def _check(sig, QT4, scale, x, t, what, cols=None):
    y = to_host(sig.sparse_gemv_q4(to_dev(QT4), to_dev(scale), to_dev(x), t))
    ref = oracle.q4_sparse_linear(QT4, scale, x, oracle.threshold_mask(x, t), cols=cols)
    assert_within(y if cols is None else y[cols], ref["y64"], ref["bound"], what)
    return y, ref


@pytest.mark.parametrize("d_in,d_out", [(4096, 11008), (4096, 4096), (11008, 4096),
                                        (1000, 528), (33, 16), (4096, 16)])
def test_q4_shapes_and_sparsities(sig, d_in, d_out):
    QT4, scale, x, ts = workloads.q4_projection(seed=d_in + d_out, d_in=d_in, d_out=d_out,
                                                 sparsities=(0.0, 0.5, 0.65))
    for s_, t in ts.items():
        _check(sig, QT4, scale, x, t, f"{d_in}x{d_out} s={s_}")


def test_q4_every_code_extremes_and_degenerate_masks(sig):
    """Every byte value appears (all 16 x 16 nibble pairs), the two saturated
    columns hold 7 and -8 everywhere, then the empty and the full mask."""
    QT4, scale, x, ts = workloads.q4_projection(seed=3, d_in=512, d_out=256)
    QT4[:256, 0] = np.arange(256, dtype=np.uint8)
    QT4[:, 1] = 0x77          # columns 2, 3: +7
    QT4[:, 2] = 0x88          # columns 4, 5: -8
    _check(sig, QT4, scale, x, ts[0.5], "every byte, saturated columns")
    y, _ = _check(sig, QT4, scale, x, float("inf"), "empty mask")
    assert np.all(y.view(np.uint16) == 0)
    _check(sig, QT4, scale, x, 0.0, "full mask")


def test_q4_wide_slice_path(sig):
    """596 column tiles, more than the grid's 592 CTA slots: one slice per
    tile, 257 input groups per slice, so the prologue takes the chunked path
    of mask words."""
    QT4, scale, x, ts = workloads.q4_projection(seed=19, d_in=2056, d_out=152576)
    cols = np.concatenate([np.arange(16), np.random.default_rng(4).choice(152576, 240, replace=False),
                           np.arange(152576 - 16, 152576)])
    _check(sig, QT4, scale, x, ts[0.5], "wide slices", cols=cols)


def test_q4_agrees_with_int8_on_the_same_weights(sig):
    """The int4 kernel and the int8 kernel on the decoded weights split the
    rows the same way and add in the same order: bit-identical y."""
    QT4, scale, x, ts = workloads.q4_projection(seed=8, d_in=4096, d_out=4096)
    Q8 = oracle.int4_values(QT4)
    a = to_host(sig.sparse_gemv_q4(to_dev(QT4), to_dev(scale), to_dev(x), ts[0.5]))
    b = to_host(sig.sparse_gemv_q8(to_dev(Q8), to_dev(scale), to_dev(x), ts[0.5]))
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_q4_deterministic(sig):
    QT4, scale, x, ts = workloads.q4_projection(seed=4)
    dQ, ds, dx = to_dev(QT4), to_dev(scale), to_dev(x)
    first = to_host(sig.sparse_gemv_q4(dQ, ds, dx, ts[0.5])).view(np.uint16).copy()
    for _ in range(3):
        assert np.array_equal(first, to_host(sig.sparse_gemv_q4(dQ, ds, dx, ts[0.5])).view(np.uint16))
