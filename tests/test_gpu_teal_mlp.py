"""GPU parity of the gated MLP with TEAL's magnitude threshold on the input of
every product (TEAL README, Abstract): |x_i| >= t_x for gate and up (one fused
launch with the SiLU(g) u epilogue), |h_i| >= t_h for down.

Checked like the RaNA masker: strictly (the h mask follows bit for bit from
the GPU's own h, and y is within tolerance of the product on that mask) and
end to end against the oracle's own h (g and u carry the float32 summation
bound through h = SiLU(g) u; masks may differ only where |h| is that close to t_h)."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import (assert_within, fp32_sum_bound, mask_words, silu_mul_tolerance,
                            to_dev, to_host)

pytestmark = pytest.mark.gpu


def _case(sig, mlp, x, t_x, t_h, what):
    import torch
    d_model, d_ff = mlp.WgT.shape
    dx, dg, du, dd = (to_dev(a) for a in (x, mlp.WgT, mlp.WuT, mlp.WdT))
    h_out = torch.empty(d_ff, dtype=torch.float16, device="cuda")
    mask_out = torch.empty((d_ff + 31) // 32, dtype=torch.int32, device="cuda")
    y = to_host(sig.teal_mlp_sparse(dx, dg, du, dd, t_x, t_h, h_out=h_out, mask_out=mask_out))
    h = to_host(h_out)
    m_gpu = oracle.unpack_bits(mask_words(mask_out), d_ff)
    m_strict = oracle.threshold_mask(h, t_h)
    assert np.array_equal(m_gpu, m_strict), what
    ref = oracle.sparse_linear(mlp.WdT, h, m_strict)
    assert_within(y, ref["y64"], ref["bound"], what + " strict")

    full = oracle.teal_mlp(x, mlp.WgT, mlp.WuT, mlp.WdT, t_x, t_h)
    h_ref, g, u = full["h16"], full["g"], full["u"]
    # g and u: float32 sums of the kept products (conftest.fp32_sum_bound)
    xm = np.where(full["mask_x"], np.abs(x.astype(np.float64)), 0.0)
    n_terms = int(np.count_nonzero(xm))
    eg = fp32_sum_bound(n_terms, xm @ np.abs(mlp.WgT.astype(np.float64)))
    eu = fp32_sum_bound(n_terms, xm @ np.abs(mlp.WuT.astype(np.float64)))
    tol_h = silu_mul_tolerance(g, u, eg, eu, h_ref)
    dh = np.abs(h.astype(np.float64) - h_ref.astype(np.float64))
    assert (dh <= tol_h).all(), (what + " h", int((dh > tol_h).sum()))
    diff = np.flatnonzero(m_gpu != full["mask"])
    assert (np.abs(np.abs(h_ref[diff].astype(np.float64)) - t_h) <= tol_h[diff]).all(), what + " mask"
    extra = np.abs(mlp.WdT[diff].astype(np.float64) *
                   np.maximum(np.abs(h[diff]), np.abs(h_ref[diff])).astype(np.float64)[:, None]).sum(0)
    err = np.abs(y.astype(np.float64) - full["y64"])
    assert (err <= 2e-3 * (full["bound"] + extra) + extra + 2.0 ** -24).all(), what + " y end to end"
    return full


def _thresholds(mlp, x, s_x=0.5, s_h=0.5):
    t_x = workloads.quantile_threshold(x, s_x)
    _, _, h = oracle.rana_hidden(np.where(oracle.threshold_mask(x, t_x), x, np.float16(0)),
                                 mlp.WgT, mlp.WuT)
    return t_x, workloads.quantile_threshold(h, s_h)


def test_teal_mlp_llama2_7b_shapes(sig):
    mlp = workloads.rana_mlp(5)
    x = workloads.draw_vector(np.random.default_rng(5), mlp.WgT.shape[0], "laplace")
    t_x, t_h = _thresholds(mlp, x)
    full = _case(sig, mlp, x, t_x, t_h, "4096/11008 at 50 %/50 %")
    assert abs(oracle.sparsity(full["mask_x"]) - 0.5) < 0.01


def test_teal_mlp_small_and_degenerate(sig):
    mlp = workloads.rana_mlp(6, d_model=256, d_ff=520, sigma=0.05)
    x = workloads.draw_vector(np.random.default_rng(6), 256, "laplace")
    _case(sig, mlp, x, 0.0, 0.0, "keeps all")
    _case(sig, mlp, x, float("inf"), 0.0, "empty input mask")
    t_x, t_h = _thresholds(mlp, x, 0.4, 0.65)
    _case(sig, mlp, x, t_x, t_h, "40 %/65 %")
