"""GPU parity of the N:M selection and mitigation variants ("Motivating
Next-Gen Accelerators with Flexible (N:M) Activation Sparsity ...", summary,
Methodology: criteria ACT and WT, mitigation PTS and VAR).

Masks are compared bit for bit with the oracle; the masked block bit for bit
without VAR and within one fp16 ulp with it (gamma is a float32 sum on the
GPU, float64 in the oracle); the GEMM within |Y - Y64| <= 2e-3 * bound of
the oracle product on the GPU's masked block, the shift added back."""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, mask_words, to_dev, to_host

pytestmark = pytest.mark.gpu


def _ulp_close(a16, b16):
    a = a16.astype(np.float64)
    b = b16.astype(np.float64)
    ulp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float16)).astype(np.float64)
    return np.all(np.abs(a - b) <= ulp)


def _inputs(rows=64, d=1024, seed=3):
    WT, X = workloads.nm_tokens(seed, rows=128, d=d, d_out=1024)
    X = X[:rows].copy()
    shift = X.astype(np.float32).mean(axis=1).astype(np.float32)    # a dynamic per-token shift
    return WT, X, shift


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (8, 16), (16, 32), (4, 8)])
@pytest.mark.parametrize("use_shift,use_wt,var", [(False, False, False), (True, False, False),
                                                  (False, True, False), (False, False, True),
                                                  (True, True, True)])
def test_nm_variant_masks(sig, n, m, use_shift, use_wt, var):
    WT, X, shift = _inputs()
    norms_gpu = sig.row_norms(to_dev(WT))
    norms = oracle.row_norms(WT)
    assert np.array_equal(to_host(norms_gpu), norms)
    Xm, bits, gamma = sig.sparsify_nm_ex(to_dev(X), n, m, shift=to_dev(shift) if use_shift else None,
                                         norms=norms_gpu if use_wt else None, var=var,
                                         want_gamma=True)
    ref = oracle.nm_variant(X, n, m, shift=shift if use_shift else None,
                            norms=norms if use_wt else None, var=var)
    what = f"{n}:{m} shift={use_shift} wt={use_wt} var={var}"
    assert np.array_equal(mask_words(bits), oracle.pack_bits(ref["mask"])), what
    got = to_host(Xm)
    if var:
        assert _ulp_close(got, ref["xm16"]), what
        assert np.allclose(to_host(gamma), ref["gamma"], rtol=1e-5, atol=0), what
    else:
        assert np.array_equal(got.view(np.uint16), ref["xm16"].view(np.uint16)), what


def test_nm_variant_ties_nan_and_ragged(sig):
    rng = np.random.default_rng(14)
    for d in (40, 96):
        X = rng.choice([0.0, -0.0, 1.0, -1.0, 0.25, 2.0, -2.0], size=(7, d)).astype(np.float16)
        X[0, :3] = np.nan
        X[1, 1] = np.inf
        shift = rng.choice([0.0, 0.25, -1.0], size=7).astype(np.float32)
        norms = rng.choice([0.5, 1.0, 2.0], size=d).astype(np.float32)
        for m in ((1, 2, 4, 8) if d == 40 else (16, 32)):
            for n in sorted({1, max(1, m // 2), m}):
                for sh, nr in ((None, None), (shift, None), (None, norms), (shift, norms)):
                    Xm, bits, _ = sig.sparsify_nm_ex(to_dev(X), n, m,
                                                     shift=None if sh is None else to_dev(sh),
                                                     norms=None if nr is None else to_dev(nr))
                    ref = oracle.nm_variant(X, n, m, shift=sh, norms=nr)
                    what = f"d={d} {n}:{m} shift={sh is not None} wt={nr is not None}"
                    assert np.array_equal(mask_words(bits), oracle.pack_bits(ref["mask"])), what
                    got, want = to_host(Xm), ref["xm16"]
                    if sh is None:   # no shift: the input's bits, NaN payloads included
                        assert np.array_equal(got.view(np.uint16), want.view(np.uint16)), what
                    else:            # float32 arithmetic may change a NaN's payload
                        both_nan = np.isnan(got) & np.isnan(want)
                        assert np.array_equal(np.where(both_nan, 0, got.view(np.uint16)),
                                              np.where(both_nan, 0, want.view(np.uint16))), what


def test_col_sums(sig):
    WT, _, _ = _inputs()
    got = to_host(sig.col_sums_of(to_dev(WT)))
    want = WT.astype(np.float64).sum(axis=0).astype(np.float32)
    assert np.all(np.abs(got.astype(np.float64) - want) <= np.spacing(np.abs(want)).astype(np.float64))


@pytest.mark.parametrize("n,m,use_shift,use_wt,var", [(2, 4, True, True, True), (8, 16, True, False, False), (4, 4, True, False, False),
                                                      (2, 4, False, True, False), (16, 32, False, False, True)])
def test_nm_variant_gemm(sig, n, m, use_shift, use_wt, var):
    WT, X, shift = _inputs(rows=128)
    dW, dX = to_dev(WT), to_dev(X)
    norms = sig.row_norms(dW) if use_wt else None
    dshift = to_dev(shift) if use_shift else None
    Y = to_host(sig.nm_act_gemm_ex(dX, dW, n, m, shift=dshift, norms=norms, var=var))
    Xm, _, _ = sig.sparsify_nm_ex(dX, n, m, shift=dshift, norms=norms, var=var, want_bits=False)
    Y64, bound = oracle.nm_variant_gemm(to_host(Xm), WT, shift=shift if use_shift else None)
    assert_within(Y, Y64, bound, f"{n}:{m} shift={use_shift} wt={use_wt} var={var}")
    # with the shift, the product stays close to the plain x W on the kept rows' scale
    if use_shift and n == m:
        assert_within(Y, X.astype(np.float64) @ WT.astype(np.float64), bound, "shift added back")
