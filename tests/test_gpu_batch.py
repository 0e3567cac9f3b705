"""GPU parity of the batched product with per-token masks, y_b = W (m_b . x_b)
("Adaptive Rank Allocation ... RaNA Adapters", rebuttal Q5.1 for the product,
Q6 for batches whose masks disagree), up to 16 tokens.  Every token is compared element by
element with the oracle within |y - y64| <= 2e-3 * sum_i |W_ij m_b,i x_b,i|."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu


def _check(sig, WT, X, t, what):
    Y = to_host(sig.sparse_gemv_batch(to_dev(WT), to_dev(X), t))
    masks = np.stack([oracle.threshold_mask(x, t) for x in X])
    ref = oracle.batched_sparse_linear(WT, X, masks)
    for b in range(X.shape[0]):
        assert_within(Y[b], ref["y64"][b], ref["bound"][b], f"{what} token {b}")
    return Y, ref


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 9, 12, 16])
def test_batch_llama_gate_shape(sig, B):
    WT, X, t = workloads.batch_tokens(seed=B, B=B)
    _, ref = _check(sig, WT, X, t, f"4096->11008 B={B}")
    if B > 1:
        assert ref["union"].sum() > np.max([oracle.threshold_mask(x, t).sum() for x in X])


@pytest.mark.parametrize("d_in,d_out,B", [(4096, 4096, 4), (11008, 4096, 8), (1000, 264, 3),
                                          (8, 8, 2), (2048, 131072 // 16, 6), (11008, 4096, 16),
                                          (1000, 264, 13)])
def test_batch_shapes(sig, d_in, d_out, B):
    WT, X, t = workloads.batch_tokens(seed=d_in + d_out + B, B=B, d_in=d_in, d_out=d_out)
    _check(sig, WT, X, t, f"{d_in}x{d_out} B={B}")


def test_batch_degenerate_masks_and_identical_tokens(sig):
    WT, X, t = workloads.batch_tokens(seed=9, B=4, d_in=512, d_out=256)
    Y, _ = _check(sig, WT, X, float("inf"), "t = inf")
    assert np.all(Y.view(np.uint16) == 0)
    _check(sig, WT, X, 0.0, "t = 0")
    # one token masks everything, the others keep their rows
    X2 = X.copy()
    X2[1] = np.float16(0.001)
    Y2, _ = _check(sig, WT, X2, t, "one empty token")
    assert np.all(Y2[1].view(np.uint16) == 0)
    # identical tokens give identical outputs, bit for bit
    X3 = np.repeat(X[:1], 11, axis=0)
    Y3 = to_host(sig.sparse_gemv_batch(to_dev(WT), to_dev(X3), t))
    for b in range(1, 11):
        assert np.array_equal(Y3[0].view(np.uint16), Y3[b].view(np.uint16))


def test_batch_deterministic(sig):
    WT, X, t = workloads.batch_tokens(seed=12, B=16, d_in=4096, d_out=4096)
    dW, dX = to_dev(WT), to_dev(X)
    first = to_host(sig.sparse_gemv_batch(dW, dX, t)).view(np.uint16).copy()
    for _ in range(3):
        assert np.array_equal(first, to_host(sig.sparse_gemv_batch(dW, dX, t)).view(np.uint16))
