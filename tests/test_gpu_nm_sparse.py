"""GPU parity of the packed 2:4 operand (sparsify_nm's packed output) and of
the N:M GEMM on the sparse tensor cores (tcgen05.mma.sp), for 2:4 and for 1:4
padded to 2:4 (Block Q-Sparse, "Q-Sparse ..." rebuttal, A2; 2:4 as the
hardware pattern, "Motivating Next-Gen Accelerators with Flexible (N:M)
Activation Sparsity ...", Hardware implications).

The packed bytes are decoded here from the layout include/sig.h documents and
compared bit for bit with the oracle's slot values and positions; the GEMM is
compared element by element with the oracle's float64 product on the mask.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.conftest import assert_within, to_dev, to_host

pytestmark = pytest.mark.gpu


def decode_packed(buf, rows, d):
    """(values [rows, d/2] fp16, positions [rows, d/2] uint8) from the packed
    bytes, following the layout documented for sparsify_nm in include/sig.h."""
    buf = np.asarray(buf, dtype=np.uint8)
    assert buf.size == rows * d * 9 // 8
    values = buf[:rows * d].view(np.float16).reshape(rows, d // 2)
    meta = buf[rows * d:].reshape(rows // 128, d // 128, 128, 16)
    positions = np.zeros((rows, d // 2), dtype=np.uint8)
    L = np.arange(128)
    for j in range(4):
        for s in range(2):
            for i in range(2):
                byte = meta[:, :, :, 4 * j + 2 * s + i]               # (R, C, L)
                r = (L % 8) + 8 * s + 16 * (L // 16)                    # row inside the block
                e0 = 32 * j + 16 * ((L // 8) % 2) + 8 * i               # first entry of the byte
                for k in range(2):
                    nib = (byte >> (4 * k)) & 0xF
                    blk = (e0 + 4 * k) // 4                             # block inside the 128 entries
                    for R in range(rows // 128):
                        for C in range(d // 128):
                            rr = 128 * R + r
                            cc = 2 * (32 * C + blk)
                            positions[rr, cc] = nib[R, C] & 3
                            positions[rr, cc + 1] = nib[R, C] >> 2
    return values, positions


def _check_pack(sig, X, n, what):
    rows, d = X.shape
    buf = to_host(sig.sparsify_nm_packed(to_dev(X), n))
    vals, pos = decode_packed(buf, rows, d)
    ref = oracle.nm_pack_2of4(X, n)
    assert np.array_equal(vals.view(np.uint16), ref["values"].view(np.uint16)), what + " values"
    assert np.array_equal(pos, ref["positions"]), what + " positions"
    return buf


def test_packed_layout_spot_byte(sig):
    """One byte worked out by hand from the header: row 9 (lane 1 + 8 = 9 for
    entries 16 .. 31, second half of the row pair 1 / 9), entries 16 .. 19
    keep positions 1 and 3, entries 20 .. 23 keep 0 and 2: byte
    16 * 9 + 4 * 0 + 2 * 1 + 0 = 146 holds 0xD | 0x8 << 4 = 0x8D."""
    X = np.zeros((128, 128), dtype=np.float16)
    X[9, 16:24] = [0.0, 3.0, 1.0, -2.0, 5.0, 0.5, -4.0, 0.0]
    buf = to_host(sig.sparsify_nm_packed(to_dev(X), 2))
    assert buf[128 * 128 + 146] == 0x8D
    assert buf[128 * 128 + 146 - 2] == 0x44          # row 1 (all zeros): positions 0, 1


@pytest.mark.parametrize("n", [2, 1])
def test_packed_operand_config(sig, n):
    _, X = workloads.nm_tokens(0)
    _check_pack(sig, X, n, f"4096x1024 {n}:4")


def test_packed_operand_ties_and_specials(sig):
    rng = np.random.default_rng(31)
    X = rng.choice([0.0, -0.0, 1.0, -1.0, 0.25, 2.0, -2.0], size=(256, 384)).astype(np.float16)
    X[0, :7] = np.nan
    X[1, 3] = np.inf
    X[2, 10] = -np.inf
    X[3, :] = -0.0
    for n in (2, 1):
        _check_pack(sig, X, n, f"ties {n}:4")


@pytest.mark.parametrize("n", [2, 1])
def test_sparse_gemm_config(sig, n):
    """Block Q-Sparse at 4096 tokens x 1024 -> 1024 on the sparse tensor cores."""
    WT, X = workloads.nm_tokens(0)
    Y = to_host(sig.nm_act_gemm(to_dev(X), to_dev(WT), n, 4))
    Y64, B = oracle.nm_gemm(X, WT, oracle.nm_mask(X, n, 4))
    assert_within(Y, Y64, B, f"sparse gemm {n}:4")
    assert sig.take_device_error() == 0


@pytest.mark.parametrize("rows,K,N", [(128, 128, 128), (256, 256, 384), (384, 1024, 256),
                                      (128, 4096, 512), (512, 640, 1280), (256, 128, 256),
                                      (768, 2048, 512), (1280, 384, 256), (256, 2048, 2048),
                                      (512, 4096, 2304)])
def test_sparse_gemm_shapes(sig, rows, K, N):
    """One-CTA tiles, and CTA-pair tiles (rows and N multiples of 256, N and K
    at least 2048)."""
    WT, X = workloads.nm_tokens(rows + K + N, rows=rows, d=K, d_out=N)
    for n in (2, 1):
        Y = to_host(sig.nm_act_gemm(to_dev(X), to_dev(WT), n, 4))
        Y64, B = oracle.nm_gemm(X, WT, oracle.nm_mask(X, n, 4))
        assert_within(Y, Y64, B, f"sparse gemm {rows}x{K}x{N} {n}:4")
    assert sig.take_device_error() == 0


def test_gemm_paths_of_large_token_blocks(sig):
    """9472 tokens x 1024 -> 1024: 296 one-CTA tiles of 128 x 256, so the 2:4
    GEMM takes 128-column tiles, and 74 pair tiles of 256 x 512, so the dense
    GEMM (8:16 on the masked block) takes the wide CTA-pair kernel at K = 1024.
    Every output of 512 sampled token rows is checked."""
    rows, K, N = 9472, 1024, 1024
    WT, X = workloads.nm_tokens(7, rows=rows, d=K, d_out=N)
    sample = np.sort(np.random.default_rng(5).choice(rows, 512, replace=False))
    dX, dW = to_dev(X), to_dev(WT)
    for n, m in ((2, 4), (8, 16)):
        Y = to_host(sig.nm_act_gemm(dX, dW, n, m))
        Y64, B = oracle.nm_gemm(X, WT, oracle.nm_mask(X, n, m), rows=sample)
        assert_within(Y[sample], Y64, B, f"{rows}x{K}x{N} {n}:{m}")
    assert sig.take_device_error() == 0


def test_packed_entry_point_matches_the_fused_call(sig):
    """nm_act_gemm_packed on sparsify_nm's packed output is the product
    nm_act_gemm computes for 2:4 (bit for bit: same operand, same kernel)."""
    WT, X = workloads.nm_tokens(7, rows=512, d=1024, d_out=768)
    dX, dW = to_dev(X), to_dev(WT)
    for n in (2, 1):
        packed = sig.sparsify_nm_packed(dX, n)
        Yp = to_host(sig.nm_act_gemm_packed(packed, 512, 1024, dW))
        Yf = to_host(sig.nm_act_gemm(dX, dW, n, 4))
        assert np.array_equal(Yp.view(np.uint16), Yf.view(np.uint16)), n
        Y64, B = oracle.nm_gemm(X, WT, oracle.nm_mask(X, n, 4))
        assert_within(Yp, Y64, B, f"packed entry {n}:4")
    assert sig.take_device_error() == 0


def test_sparse_gemm_reveals_the_decoded_operand(sig):
    """With WT the identity, Y is the activation block the sparse MMA decoded
    from the packed values and metadata: it must be the masked X exactly
    (every product is x * 1 and every sum has one non-zero term)."""
    rng = np.random.default_rng(8)
    X = rng.laplace(0, 1, (256, 256)).astype(np.float16)
    WT = np.eye(256, dtype=np.float16)
    for n in (2, 1):
        Y = to_host(sig.nm_act_gemm(to_dev(X), to_dev(WT), n, 4))
        want = np.where(oracle.nm_mask(X, n, 4), X, np.float16(0))
        bad = np.argwhere(Y.view(np.uint16) != want.view(np.uint16))
        assert bad.size == 0, (n, bad[:8].tolist())
