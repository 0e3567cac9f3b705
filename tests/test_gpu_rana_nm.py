"""GPU parity of the RaNA gated-MLP masker, the N:M mask and the N:M GEMM."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import (assert_within, fp32_sum_bound, mask_words, silu_mul_tolerance,
                            to_dev, to_host)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# RaNA Eqn. 12
# ---------------------------------------------------------------------------

def test_row_norms_bit_exact(sig):
    rng = np.random.default_rng(2)
    for rows, cols in ((11008, 4096), (37, 8), (5, 4104)):
        W = workloads.draw_weight(rng, rows, cols, 0.02)
        got = to_host(sig.row_norms(to_dev(W)))
        assert np.array_equal(got, oracle.row_norms(W)), (rows, cols)


def _rana_case(sig, mlp, t, what):
    import torch
    d_model, d_ff = mlp.WgT.shape
    dx, dg, du, dd = (to_dev(a) for a in (mlp.x, mlp.WgT, mlp.WuT, mlp.WdT))
    norms_gpu = sig.row_norms(dd)
    norms = oracle.row_norms(mlp.WdT)
    assert np.array_equal(to_host(norms_gpu), norms)
    h_out = torch.empty(d_ff, dtype=torch.float16, device="cuda")
    mask_out = torch.empty((d_ff + 31) // 32, dtype=torch.int32, device="cuda")
    y = to_host(sig.gated_mlp_sparse(dx, dg, du, dd, norms_gpu, t, h_out=h_out, mask_out=mask_out))
    h = to_host(h_out)
    m_gpu = oracle.unpack_bits(mask_words(mask_out), d_ff)

    # strict: the mask and y follow from the GPU's own h by the oracle's rule
    s = oracle.rana_scores(h, norms)
    m_strict = oracle.rana_mask(s, t)
    assert np.array_equal(m_gpu, m_strict), what
    ref = oracle.sparse_linear(mlp.WdT, h, m_strict)
    assert_within(y, ref["y64"], ref["bound"], what + " strict")

    # end to end against the oracle's own h.  g and u are float32 sums of
    # d_model exact products on the GPU: each carries at most the float32
    # summation bound gamma_d * sum|W x|, which h = SiLU(g) u carries on
    # (conftest.silu_mul_tolerance).
    full = oracle.gated_mlp(mlp.x, mlp.WgT, mlp.WuT, mlp.WdT, norms, t)
    h_ref, g, u = full["h16"], full["g"], full["u"]
    x64 = np.abs(mlp.x.astype(np.float64))
    n_terms = int(np.count_nonzero(mlp.x))
    eg = fp32_sum_bound(n_terms, x64 @ np.abs(mlp.WgT.astype(np.float64)))
    eu = fp32_sum_bound(n_terms, x64 @ np.abs(mlp.WuT.astype(np.float64)))
    tol_h = silu_mul_tolerance(g, u, eg, eu, h_ref)
    dh = np.abs(h.astype(np.float64) - h_ref.astype(np.float64))
    assert (dh <= tol_h).all(), (what + " h", int((dh > tol_h).sum()))
    assert (dh <= np.spacing(np.abs(h_ref))).mean() > 0.999, what + " h mostly within 1 ulp"
    diff = np.flatnonzero(m_gpu != full["mask"])
    s_ref = full["s32"].astype(np.float64)
    slack = tol_h[diff] * norms[diff].astype(np.float64) + 2.0 ** -10 * t
    assert (np.abs(s_ref[diff] - t) <= slack).all(), what + " mask"
    extra = np.abs(mlp.WdT[diff].astype(np.float64) *
                   np.maximum(np.abs(h[diff]), np.abs(h_ref[diff])).astype(np.float64)[:, None]).sum(0)
    err = np.abs(y.astype(np.float64) - full["y64"])
    slack = 2e-3 * (full["bound"] + extra) + extra + 2.0 ** -24
    assert (err <= slack).all(), what + " y end to end"
    return full


def test_rana_config_full(sig):
    mlp = workloads.rana_mlp(0)
    norms = oracle.row_norms(mlp.WdT)
    _, _, h = oracle.rana_hidden(mlp.x, mlp.WgT, mlp.WuT)
    s = oracle.rana_scores(h, norms)
    t = float(np.sort(s)[len(s) // 2])          # 50 % quantile of the oracle's scores
    full = _rana_case(sig, mlp, t, "rana 4096/11008")
    assert abs(oracle.sparsity(full["mask"]) - 0.5) < 0.01


def test_rana_small_and_degenerate(sig):
    mlp = workloads.rana_mlp(3, d_model=256, d_ff=520, sigma=0.05)
    _rana_case(sig, mlp, 0.0, "t = 0 keeps all")
    _rana_case(sig, mlp, float("inf"), "t = inf keeps none")
    _rana_case(sig, mlp, 0.05, "t = 0.05")


# ---------------------------------------------------------------------------
# N:M mask
# ---------------------------------------------------------------------------

def _check_nm(sig, X, n, m, what):
    Xm, mb = sig.sparsify_nm(to_dev(X), n, m)
    M = oracle.nm_mask(X, n, m)
    assert np.array_equal(mask_words(mb), oracle.pack_bits(M)), what
    want = np.where(M, X, np.float16(0))
    assert np.array_equal(to_host(Xm).view(np.uint16), want.view(np.uint16)), what


@pytest.mark.parametrize("n,m", workloads.NM_PATTERNS)
def test_nm_mask_config(sig, n, m):
    _, X = workloads.nm_tokens(0)
    _check_nm(sig, X, n, m, f"{n}:{m}")


def test_nm_mask_ragged_and_ties(sig):
    rng = np.random.default_rng(12)
    for d, ms in ((40, (1, 2, 4, 8)), (48, (16,)), (96, (32,)), (8, (1, 2, 4, 8))):
        X = rng.choice([0.0, -0.0, 1.0, -1.0, 0.25, 2.0, -2.0], size=(5, d)).astype(np.float16)
        X[0, :3] = np.nan
        X[1, 1] = np.inf
        for m in ms:
            for n in sorted({1, min(3, m), max(1, m // 2), max(1, m - 1), m}):
                _check_nm(sig, X, n, m, f"d={d} {n}:{m}")
    _check_nm(sig, np.zeros((0, 64), np.float16), 2, 4, "zero rows")
    # several vectors per thread, rows whose last word is partial
    X = workloads.draw_vector(rng, (37, 1000), "laplace")
    for n, m in ((1, 1), (1, 2), (2, 4), (1, 4), (3, 8), (8, 8)):
        _check_nm(sig, X, n, m, f"37x1000 {n}:{m}")
    # 16- and 32-entry blocks on rows of 1024 and 992 entries (31 words, the
    # grid's last warp partly past the end), several n
    for d in (1024, 992):
        X = workloads.draw_vector(rng, (37, d), "laplace")
        for n, m in ((5, 16), (8, 16), (15, 16), (1, 32), (11, 32), (16, 32), (32, 32)):
            _check_nm(sig, X, n, m, f"37x{d} {n}:{m}")


# ---------------------------------------------------------------------------
# N:M activation GEMM on the tensor cores
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n,m", workloads.NM_PATTERNS)
def test_nm_gemm_config(sig, n, m):
    WT, X = workloads.nm_tokens(0)
    Y = to_host(sig.nm_act_gemm(to_dev(X), to_dev(WT), n, m))
    M = oracle.nm_mask(X, n, m)
    Y64, B = oracle.nm_gemm(X, WT, M)
    assert_within(Y, Y64, B, f"nm gemm {n}:{m}")
    assert sig.take_device_error() == 0


@pytest.mark.parametrize("rows,K,N", [(128, 64, 128), (256, 192, 384), (384, 1024, 256),
                                      (128, 4096, 512), (256, 64, 256), (512, 1024, 768),
                                      (768, 2048, 512), (256, 2048, 2048), (512, 4096, 2304)])
def test_nm_gemm_shapes(sig, rows, K, N):
    WT, X = workloads.nm_tokens(rows + K + N, rows=rows, d=K, d_out=N)
    for n, m in ((2, 4), (4, 4)):
        Y = to_host(sig.nm_act_gemm(to_dev(X), to_dev(WT), n, m))
        Y64, B = oracle.nm_gemm(X, WT, oracle.nm_mask(X, n, m))
        assert_within(Y, Y64, B, f"nm gemm {rows}x{K}x{N} {n}:{m}")
    assert sig.take_device_error() == 0
