"""Failure detection of the tensor-core GEMMs' bounded waits, without a GPU
fault: the wait limit is shortened to a few cycles (sig_set_wait_limit), so
the MMA thread's wait for its first stage of data gives up long before the
copy lands.  The kernel must then record the give-up in the device error word
(sig_take_device_error returns SIG_ERR_TIMEOUT with a non-zero code), let its
issued copies land, free its tensor memory and return; with the default limit
restored, the next GEMM on the same context is correct and the word stays 0."""
import ctypes

import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu

SIG_OK, SIG_ERR_TIMEOUT = 0, 6


def _give_up_then_recover(sig, run, check):
    import torch
    assert sig.take_device_error() == 0
    try:
        sig.set_wait_limit(64)
        run()
        torch.cuda.synchronize()
        code = ctypes.c_uint(0)
        st = sig._lib.sig_take_device_error(ctypes.byref(code), None)
    finally:
        sig.set_wait_limit(0)
    assert st == SIG_ERR_TIMEOUT and code.value != 0, (st, code.value)
    assert sig.take_device_error() == 0           # read-and-clear
    check(run())
    torch.cuda.synchronize()
    code = ctypes.c_uint(0)
    assert sig._lib.sig_take_device_error(ctypes.byref(code), None) == SIG_OK and code.value == 0


def test_dense_gemm_wait_gives_up(sig):
    WT, X = workloads.nm_tokens(3, rows=128, d=64, d_out=128)
    dX, dW = to_dev(X), to_dev(WT)

    def run():
        return sig.nm_act_gemm(dX, dW, 4, 4)       # n == m: the dense GEMM on X, one K stage

    def check(Y):
        Y64, B = oracle.nm_gemm(X, WT, np.ones_like(X, dtype=bool))
        assert_within(to_host(Y), Y64, B, "dense gemm after recovery")
    _give_up_then_recover(sig, run, check)


def test_sparse_gemm_wait_gives_up(sig):
    WT, X = workloads.nm_tokens(4, rows=128, d=512, d_out=256)
    dX, dW = to_dev(X), to_dev(WT)
    packed = sig.sparsify_nm_packed(dX, 2)

    def run():
        return sig.nm_act_gemm_packed(packed, 128, 512, dW)   # four K stages, two in flight

    def check(Y):
        Y64, B = oracle.nm_gemm(X, WT, oracle.nm_mask(X, 2, 4))
        assert_within(to_host(Y), Y64, B, "sparse gemm after recovery")
    _give_up_then_recover(sig, run, check)


def test_deep_pipeline_gives_up_mid_ring(sig):
    """Sixteen K stages through the four-stage ring of the one-CTA kernel: the
    producer has issued a full ring when the MMA thread gives up, and every
    issued copy must land before the CTAs exit."""
    WT, X = workloads.nm_tokens(5, rows=128, d=1024, d_out=256)
    dX, dW = to_dev(X), to_dev(WT)

    def run():
        return sig.nm_act_gemm(dX, dW, 8, 8)

    def check(Y):
        Y64, B = oracle.nm_gemm(X, WT, np.ones_like(X, dtype=bool))
        assert_within(to_host(Y), Y64, B, "deep ring after recovery")
    _give_up_then_recover(sig, run, check)
