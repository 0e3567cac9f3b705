"""gated_mlp_sparse_noalloc, the gated-MLP entry point that allocates nothing.

It serves callers that cannot allocate device memory where they run the layer
(a plugin whose host program owns all device memory, a serving loop with a
memory budget fixed at start-up, C code without an allocator).  This file is
named so that pytest collects it last.

The test calls it through the C ABI twice in a row and checks each output
against the existing gated_mlp_sparse on the same inputs.  The two entry
points run the same kernels with the same launch plan and split-K order, so y
must be bit-identical (which implies the tolerance the other parity tests
use).  Both calls run on the same stream, so the second call finds the first
call's contents in the shared scratch array.
"""
import numpy as np
import pytest

import workloads
from tests.conftest import assert_within, mask_words, to_dev, to_host

pytestmark = pytest.mark.gpu


def _bound(WdT, h, mask_words_, d_ff):
    """sum over kept i of |WdT[i, j] * h_i| per output j."""
    bits = (mask_words_[:, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    m = bits.ravel()[:d_ff].astype(bool)
    hm = np.where(m, h.astype(np.float64), 0.0)
    return np.abs(hm) @ np.abs(WdT.astype(np.float64))


def test_noalloc_matches_gated_mlp_twice_in_a_row(sig):
    import torch
    mlp = workloads.rana_mlp(5, d_model=1024, d_ff=2816)
    d_model, d_ff = mlp.WgT.shape
    dx, dg, du, dd = (to_dev(a) for a in (mlp.x, mlp.WgT, mlp.WuT, mlp.WdT))
    norms = sig.row_norms(dd)
    words = (d_ff + 31) // 32

    # the existing entry point, with its own workspace; threshold = median score
    h_ref = torch.empty(d_ff, dtype=torch.float16, device="cuda")
    m_ref = torch.empty(words, dtype=torch.int32, device="cuda")
    sig.gated_mlp_sparse(dx, dg, du, dd, norms, 0.0, h_out=h_ref)
    s = (h_ref.float().abs() * norms).cpu().numpy()
    t = float(np.sort(s)[d_ff // 2])
    y_ref = to_host(sig.gated_mlp_sparse(dx, dg, du, dd, norms, t, h_out=h_ref, mask_out=m_ref))
    h_host, mw = to_host(h_ref), mask_words(m_ref)
    bound = _bound(mlp.WdT, h_host, mw, d_ff)

    for call in range(2):
        h = torch.empty(d_ff, dtype=torch.float16, device="cuda")
        m = torch.empty(words, dtype=torch.int32, device="cuda")
        y = to_host(sig.gated_mlp_sparse_noalloc(dx, dg, du, dd, norms, t, h_out=h, mask_out=m))
        assert np.array_equal(to_host(h).view(np.uint16), h_host.view(np.uint16)), call
        assert np.array_equal(mask_words(m), mw), call
        assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16)), call
        assert_within(y, y_ref.astype(np.float64), bound, f"no-alloc call {call}")

    # without h_out / mask_out the hidden vector stays in the library's array
    y3 = to_host(sig.gated_mlp_sparse_noalloc(dx, dg, du, dd, norms, t))
    assert np.array_equal(y3.view(np.uint16), y_ref.view(np.uint16))
    assert_within(y3, y_ref.astype(np.float64), bound, "no-alloc without h_out")
    torch.cuda.synchronize()


def test_noalloc_rejects_sizes_beyond_its_maximum(sig):
    """The largest accepted d_ff fits the 4 MiB array; one step beyond is
    rejected with SIG_ERR_SHAPE.  Real (small) device buffers back every
    pointer, so nothing could fault even if the size checks did not stop it."""
    import torch
    d_model, d_ff = 8, 131072 + 8
    assert sig.workspace_bytes(sig.OP_GATED_MLP, d_model, 131072) <= 4 << 20
    x = torch.zeros(d_model, dtype=torch.float16, device="cuda")
    Wg = torch.zeros((d_model, d_ff), dtype=torch.float16, device="cuda")
    Wu = torch.zeros_like(Wg)
    Wd = torch.zeros((d_ff, d_model), dtype=torch.float16, device="cuda")
    norms = torch.ones(d_ff, dtype=torch.float32, device="cuda")
    with pytest.raises(sig.SigError) as e:
        sig.gated_mlp_sparse_noalloc(x, Wg, Wu, Wd, norms, 0.1)
    assert e.value.status == 2   # SIG_ERR_SHAPE
    # the largest d_ff that is accepted runs (zero weights: y = 0)
    Wg, Wu = Wg[:, :131072].contiguous(), Wu[:, :131072].contiguous()
    Wd, norms = Wd[:131072].contiguous(), norms[:131072].contiguous()
    y = sig.gated_mlp_sparse_noalloc(x, Wg, Wu, Wd, norms, 0.1)
    assert not y.float().abs().sum().item()
