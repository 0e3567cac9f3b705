"""GPU parity of the RaNA linear-layer rank adapter y = A (m . v), v = fp16(Bx),
m_i = v_i^2 >= t ("Adaptive Rank Allocation ... RaNA Adapters", rebuttal Q5.1,
Q4 on eqn. 9, Q2 on the two GEMVs).

Checked at two levels, as for the Eqn. 12 masker:
  strict      v within the plain GEMV bound of the oracle's float64 Bx; the
              mask equals the oracle's rule applied to the GPU's v, bit for
              bit; y within |y - y64| <= 2e-3 * sum |A_ij m_i v_i| of the
              oracle product on (GPU v, GPU mask);
  end to end  the oracle's own mask differs from the GPU's only where its
              score is within 2^-7 (relative) of t, the reach of the few-ulp
              difference between float32 and float64 accumulation of v.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, mask_words, to_dev, to_host

pytestmark = pytest.mark.gpu


def _run(sig, ra, t):
    import torch
    r = ra.BT.shape[1]
    v = torch.empty(r, dtype=torch.float16, device="cuda")
    mask = torch.empty((r + 31) // 32, dtype=torch.int32, device="cuda")
    y = sig.rank_adapter_sparse(to_dev(ra.x), to_dev(ra.BT), to_dev(ra.AT), t, v_out=v,
                                mask_out=mask)
    return to_host(y), to_host(v), oracle.unpack_bits(mask_words(mask), r)


def _median_score_threshold(ra):
    _, v16 = oracle.rank_adapter_hidden(ra.x, ra.BT)
    s = np.sort(oracle.rank_adapter_scores(v16))
    return float(s[s.size // 2])


def _check(sig, ra, t, what):
    y, v, m = _run(sig, ra, t)
    v64, _ = oracle.rank_adapter_hidden(ra.x, ra.BT)
    bound_v = np.abs(ra.x.astype(np.float64)) @ np.abs(ra.BT.astype(np.float64))
    assert_within(v, v64, bound_v, what + ": v")
    m_rule = oracle.rana_mask(oracle.rank_adapter_scores(v), t)
    assert np.array_equal(m, m_rule), what + ": mask"
    ref = oracle.sparse_linear(ra.AT, v, m_rule)
    assert_within(y, ref["y64"], ref["bound"], what + ": y")
    full = oracle.rank_adapter(ra.x, ra.BT, ra.AT, t)
    diff = full["mask"] != m
    s = full["s32"].astype(np.float64)
    assert np.all(np.abs(s[diff] - t) <= 2.0 ** -7 * abs(t)), what + ": end to end mask"
    return y, m


# (64, 64, 76800): 300 output tiles, one slice each (no split-K partials)
@pytest.mark.parametrize("d_in,r,d_out", [(64, 48, 24), (1000, 264, 520), (33, 8, 8),
                                          (4096, 2048, 4096), (4096, 1024, 11008),
                                          (64, 64, 76800)])
def test_rank_adapter_shapes(sig, d_in, r, d_out):
    ra = workloads.rank_adapter(seed=d_in + r + d_out, d_in=d_in, r=r, d_out=d_out)
    t = _median_score_threshold(ra)
    y, m = _check(sig, ra, t, f"{d_in}->{r}->{d_out}")
    assert 0.3 * r <= m.sum() <= 0.7 * r


def test_rank_adapter_all_and_none_kept(sig):
    ra = workloads.rank_adapter(seed=5, d_in=512, r=256, d_out=128)
    y, m = _check(sig, ra, 0.0, "t = 0")
    assert m.all()
    y, m = _check(sig, ra, float("inf"), "t = inf")
    assert not m.any() and np.all(y.view(np.uint16) == 0)


def test_rank_adapter_deterministic(sig):
    import torch
    ra = workloads.rank_adapter(seed=6)
    t = _median_score_threshold(ra)
    dx, dB, dA = to_dev(ra.x), to_dev(ra.BT), to_dev(ra.AT)
    first = to_host(sig.rank_adapter_sparse(dx, dB, dA, t)).view(np.uint16).copy()
    for _ in range(3):
        again = to_host(sig.rank_adapter_sparse(dx, dB, dA, t)).view(np.uint16)
        assert np.array_equal(first, again)
    # without v_out / mask_out the product is the same
    y, _, _ = _run(sig, ra, t)
    assert np.array_equal(first, y.view(np.uint16))
    del torch


# (64, 48, 24) and (33, 8, 8): the output tile's second 128-column half is
# empty, and the slice finishing it must not advance the tile's epoch before
# every slice has read it
@pytest.mark.parametrize("d_in,r,d_out", [(4096, 2048, 4096), (64, 48, 24), (33, 8, 8),
                                          (1000, 264, 520)])
def test_rank_adapter_repeated_calls_on_one_workspace(sig, d_in, r, d_out):
    """One workspace through many calls: the split-K partial sums carry the
    tile's epoch, which every call advances once; results equal those of a
    fresh workspace bit for bit, and no bounded wait gives up."""
    import torch
    ra = workloads.rank_adapter(seed=7, d_in=d_in, r=r, d_out=d_out)
    d_in, r = ra.BT.shape
    d_out = ra.AT.shape[1]
    t_mid = _median_score_threshold(ra)
    ts = [t_mid, 0.5 * t_mid, 2.0 * t_mid]
    dx, dB, dA = to_dev(ra.x), to_dev(ra.BT), to_dev(ra.AT)
    n_ws = sig.workspace_bytes(sig.OP_RANK_ADAPTER, d_in, d_out, r)

    def new_ws():
        return torch.zeros(n_ws, dtype=torch.uint8, device="cuda")

    fresh = {t: to_host(sig.rank_adapter_sparse(dx, dB, dA, t, ws=new_ws())).view(np.uint16).copy()
             for t in ts}
    ws = new_ws()
    for k in range(12):
        t = ts[k % 3]
        y = to_host(sig.rank_adapter_sparse(dx, dB, dA, t, ws=ws)).view(np.uint16)
        assert np.array_equal(y, fresh[t]), (k, t)
    # a changed activation between calls on the same workspace
    x2 = (ra.x.astype(np.float32) * -1.5).astype(np.float16)
    y2 = to_host(sig.rank_adapter_sparse(to_dev(x2), dB, dA, t_mid, ws=ws)).view(np.uint16)
    ref2 = to_host(sig.rank_adapter_sparse(to_dev(x2), dB, dA, t_mid, ws=new_ws())).view(np.uint16)
    assert np.array_equal(y2, ref2)
    assert sig.take_device_error() == 0
