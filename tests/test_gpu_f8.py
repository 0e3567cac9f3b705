"""GPU parity of the weight-quantised sparse GEMV with fp8 e4m3 weights and
one float32 scale per output column (TEAL README, Limitations; Q-Sparse
rebuttal, A1: quantisation is orthogonal to activation sparsity).  Every
output is compared with the oracle, which decodes the e4m3 codes exactly from
the format's definition, within |y - y64| <= 2e-3 * |s_j| * sum_i |q_ij m_i x_i|."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu


def _check(sig, QT, scale, x, t, what, cols=None):
    y = to_host(sig.sparse_gemv_f8(to_dev(QT), to_dev(scale), to_dev(x), t))
    ref = oracle.f8_sparse_linear(QT, scale, x, oracle.threshold_mask(x, t), cols=cols)
    assert_within(y if cols is None else y[cols], ref["y64"], ref["bound"], what)
    return y, ref


@pytest.mark.parametrize("d_in,d_out", [(4096, 11008), (4096, 4096), (11008, 4096),
                                        (1000, 528), (33, 16), (4096, 16)])
def test_f8_shapes_and_sparsities(sig, d_in, d_out):
    QT, scale, x, ts = workloads.f8_projection(seed=d_in + d_out, d_in=d_in, d_out=d_out,
                                                sparsities=(0.0, 0.5, 0.65))
    for s_, t in ts.items():
        _check(sig, QT, scale, x, t, f"{d_in}x{d_out} s={s_}")


def test_f8_every_code_and_degenerate_masks(sig):
    """Each of the 254 finite codes (subnormals, both signs, +-448) appears in
    its own column; the hardware conversion must match the definition."""
    rng = np.random.default_rng(9)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    QT = np.zeros((64, 256), dtype=np.uint8)
    QT[:, :codes.size] = codes[None, :]
    QT[::3] = rng.permutation(QT[::3].T).T
    scale = rng.uniform(0.5, 2.0, 256).astype(np.float32)
    x = workloads.draw_vector(rng, 64, "laplace")
    _check(sig, QT, scale, x, workloads.quantile_threshold(x, 0.5), "every code")
    y, _ = _check(sig, QT, scale, x, float("inf"), "empty mask")
    assert np.all(y.view(np.uint16) == 0)
    _check(sig, QT, scale, x, 0.0, "full mask")


def test_f8_wide_slice_path(sig):
    """d_out above 296 column tiles of 512: one slice per tile, 257 input
    groups per slice, so the prologue takes the chunked path of mask words."""
    QT, scale, x, ts = workloads.f8_projection(seed=17, d_in=2056, d_out=152576)
    cols = np.concatenate([np.arange(16), np.random.default_rng(1).choice(152576, 240, replace=False),
                           np.arange(152576 - 16, 152576)])
    _check(sig, QT, scale, x, ts[0.5], "wide slices", cols=cols)


def test_f8_deterministic(sig):
    QT, scale, x, ts = workloads.f8_projection(seed=4)
    dQ, ds, dx = to_dev(QT), to_dev(scale), to_dev(x)
    first = to_host(sig.sparse_gemv_f8(dQ, ds, dx, ts[0.5])).view(np.uint16).copy()
    for _ in range(3):
        assert np.array_equal(first, to_host(sig.sparse_gemv_f8(dQ, ds, dx, ts[0.5])).view(np.uint16))
