"""At zero sparsity the sparse product is the dense GEMV.

The float64 oracle product, cuBLAS through torch.matmul (fp16 operands,
float32 accumulation, fp16 result) and the library's sparse path with t = 0
must each meet the parity bound |y - y64| <= 2e-3 * sum_i |W_ij x_i| on the
three Llama-2-7B projection shapes: the oracle's dense product is checked
against an independent library here, not only against itself.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu


def cublas_gemv(WT, x):
    import torch
    flag = torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    try:
        return torch.matmul(x.view(1, -1), WT).view(-1)
    finally:
        torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = flag


@pytest.mark.parametrize("name", ["q", "gate", "down"])
def test_zero_sparsity_oracle_cublas_and_sparse_path_agree(sig, name):
    (p,) = workloads.llama2_7b(0, names=(name,))
    ref = oracle.sparse_linear(p.WT, p.x, np.ones(p.d_in, bool))
    dW, dx = to_dev(p.WT), to_dev(p.x)
    assert_within(to_host(cublas_gemv(dW, dx)), ref["y64"], ref["bound"], f"cuBLAS {name}")
    assert_within(to_host(sig.sparse_gemv(dW, dx, t=0.0)), ref["y64"], ref["bound"],
                  f"sparse path at t = 0, {name}")
