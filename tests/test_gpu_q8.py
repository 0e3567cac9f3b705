"""GPU parity of the weight-quantised sparse GEMV: int8 weights with one
float32 scale per output column (TEAL README, Limitations; Q-Sparse rebuttal,
A1: quantisation is orthogonal to activation sparsity).  Every output is
compared with the oracle within |y - y64| <= 2e-3 * |s_j| * sum_i |q_ij m_i x_i|."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu


def _check(sig, QT, scale, x, t, what):
    y = to_host(sig.sparse_gemv_q8(to_dev(QT), to_dev(scale), to_dev(x), t))
    ref = oracle.q8_sparse_linear(QT, scale, x, oracle.threshold_mask(x, t))
    assert_within(y, ref["y64"], ref["bound"], what)
    return y, ref


@pytest.mark.parametrize("d_in,d_out", [(4096, 11008), (4096, 4096), (11008, 4096),
                                        (1000, 528), (33, 16), (4096, 16)])
def test_q8_shapes_and_sparsities(sig, d_in, d_out):
    QT, scale, x, ts = workloads.q8_projection(seed=d_in + d_out, d_in=d_in, d_out=d_out,
                                                sparsities=(0.0, 0.5, 0.65))
    for s_, t in ts.items():
        _check(sig, QT, scale, x, t, f"{d_in}x{d_out} s={s_}")


def test_q8_extremes_and_degenerate_masks(sig):
    QT, scale, x, ts = workloads.q8_projection(seed=3, d_in=512, d_out=256)
    QT[:, :8] = 127
    QT[:, 8:16] = -127
    y, ref = _check(sig, QT, scale, x, ts[0.5], "saturated columns")
    y, ref = _check(sig, QT, scale, x, float("inf"), "empty mask")
    assert np.all(y.view(np.uint16) == 0)
    _check(sig, QT, scale, x, 0.0, "full mask")


def test_q8_wide_slice_path(sig):
    """More than 296 column tiles of 512: one slice per tile, 257 input groups
    per slice, so the prologue takes the chunked path of mask words."""
    QT, scale, x, ts = workloads.q8_projection(seed=18, d_in=2056, d_out=152576)
    cols = np.concatenate([np.arange(16), np.random.default_rng(2).choice(152576, 240, replace=False),
                           np.arange(152576 - 16, 152576)])
    y = to_host(sig.sparse_gemv_q8(to_dev(QT), to_dev(scale), to_dev(x), ts[0.5]))
    ref = oracle.q8_sparse_linear(QT, scale, x, oracle.threshold_mask(x, ts[0.5]), cols=cols)
    assert_within(y[cols], ref["y64"], ref["bound"], "wide slices")


def test_q8_deterministic(sig):
    QT, scale, x, ts = workloads.q8_projection(seed=4)
    dQ, ds, dx = to_dev(QT), to_dev(scale), to_dev(x)
    first = to_host(sig.sparse_gemv_q8(dQ, ds, dx, ts[0.5])).view(np.uint16).copy()
    for _ in range(3):
        assert np.array_equal(first, to_host(sig.sparse_gemv_q8(dQ, ds, dx, ts[0.5])).view(np.uint16))
