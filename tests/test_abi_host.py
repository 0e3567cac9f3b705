"""Host-side tests of the C ABI: no GPU needed, no kernel is launched.

Every call here fails argument validation, which runs on the host before any
CUDA call, so the returned status is the whole behaviour under test.
"""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT, load_builder

HEADER = os.path.join(ROOT, "include", "sig.h")

OK, NULL, SHAPE, ALIGN, WORKSPACE, CUDA, TIMEOUT, ARG = range(8)
FAKE = 1 << 40            # an aligned, never dereferenced "device" address
FAKE_ODD = FAKE + 2       # 2-byte aligned only


@pytest.fixture(scope="module")
def lib():
    path = load_builder().build()
    lib = ctypes.CDLL(path)
    import sparse_input_gemv_threshold_b200 as sig  # noqa: F401  (sets argtypes on its own handle)
    for name, (res, args) in sig._SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decl = re.findall(r"^SIG_API\s+(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)
    return sorted(set(decl))


def test_header_declares_the_six_entry_points():
    names = declared_functions()
    for fn in ("sparsify_threshold", "sparsify_topk", "sparsify_nm", "sparse_gemv",
               "gated_mlp_sparse", "nm_act_gemm"):
        assert fn in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    # nothing else leaks out with default visibility except the ABI
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", os.path.join(ROOT, "sparse_input_gemv_threshold_b200", "libsig.so")],
                         capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported


def test_binding_covers_every_declared_symbol():
    import sparse_input_gemv_threshold_b200 as sig
    assert set(declared_functions()) <= set(sig._SIGNATURES)


def test_status_strings_and_version(lib):
    assert lib.sig_abi_version() == 2
    for s in range(8):
        assert lib.sig_status_string(s)
    assert lib.sig_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    ws = lib.sig_workspace_bytes
    assert ws(1, 4096, 4096, 0) > 0           # split-K partials and per-tile counters
    assert ws(1, 4096, 4096, 0) % 256 == 0
    assert ws(1, 64, 131072, 0) == 0          # > 296 column tiles: one slice, no partials
    assert ws(1, 4096, 296 * 256, 0) > 0      # 296 tiles of 256 columns still split K
    assert ws(1, 4096, 296 * 256 + 8, 0) == 0
    assert ws(1, 0, 4096, 0) == 0            # invalid shape
    assert ws(1, 4096, 12, 0) == 0           # d_out % 8
    assert ws(2, 8192, 0, 0) == 0            # top-k needs none
    assert ws(3, 4096, 11008, 0) > ws(1, 11008, 4096, 0)
    assert ws(4, 1024, 1024, 4096) == 4096 * 1024 * 2   # the masked activation block
    assert ws(77, 1, 1, 1) == 0


def test_sparse_gemv_validation(lib):
    f = lib.sparse_gemv
    big = 1 << 30
    assert f(None, 64, 64, FAKE, 0.0, None, None, FAKE, FAKE, big, None) == NULL
    assert f(FAKE, 64, 64, FAKE, 0.0, FAKE, None, FAKE, FAKE, big, None) == NULL   # idx w/o nnz
    assert f(FAKE, 0, 64, FAKE, 0.0, None, None, FAKE, FAKE, big, None) == SHAPE
    assert f(FAKE, 131073, 64, FAKE, 0.0, None, None, FAKE, FAKE, big, None) == SHAPE
    assert f(FAKE, 64, 60, FAKE, 0.0, None, None, FAKE, FAKE, big, None) == SHAPE
    assert f(FAKE, 64, 0, FAKE, 0.0, None, None, FAKE, FAKE, big, None) == SHAPE
    assert f(FAKE_ODD, 64, 64, FAKE, 0.0, None, None, FAKE, FAKE, big, None) == ALIGN
    assert f(FAKE, 64, 64, FAKE_ODD, 0.0, None, None, FAKE, FAKE, big, None) == ALIGN
    assert f(FAKE, 64, 64, FAKE, 0.0, None, None, FAKE_ODD, FAKE, big, None) == ALIGN
    assert f(FAKE, 64, 64, FAKE, 0.0, None, None, FAKE, None, big, None) == WORKSPACE
    need = lib.sig_workspace_bytes(1, 64, 64, 0)
    assert need > 0
    assert f(FAKE, 64, 64, FAKE, 0.0, None, None, FAKE, FAKE, need - 1, None) == WORKSPACE
    assert f(FAKE, 64, 64, FAKE, 0.0, None, None, FAKE, FAKE + 16, need, None) == ALIGN


def test_mask_validation(lib):
    assert lib.sparsify_threshold(None, 8, 0.0, FAKE, None, None, None) == NULL
    assert lib.sparsify_threshold(FAKE, 8, 0.0, None, None, None, None) == NULL
    assert lib.sparsify_threshold(FAKE, 0, 0.0, FAKE, None, None, None) == SHAPE
    assert lib.sparsify_threshold(FAKE_ODD, 8, 0.0, FAKE, None, None, None) == ALIGN
    t = lib.sparsify_topk
    assert t(FAKE, 8, 9, FAKE, FAKE, FAKE, None, 0, None) == ARG
    assert t(FAKE, 8, -1, FAKE, FAKE, FAKE, None, 0, None) == ARG
    assert t(FAKE, 8, 2, FAKE, None, FAKE, None, 0, None) == NULL
    assert t(FAKE, 0, 0, FAKE, FAKE, FAKE, None, 0, None) == SHAPE
    assert t(FAKE, 131073, 5, FAKE, FAKE, FAKE, None, 0, None) == SHAPE
    n = lib.sparsify_nm
    assert n(FAKE, 4, 64, 3, 2, FAKE, FAKE, None, None) == ARG      # n > m
    assert n(FAKE, 4, 64, 0, 4, FAKE, FAKE, None, None) == ARG      # n < 1
    assert n(FAKE, 4, 60, 2, 3, FAKE, FAKE, None, None) == ARG      # m not a power of two
    assert n(FAKE, 4, 36, 2, 8, FAKE, FAKE, None, None) == SHAPE    # m does not divide d
    assert n(FAKE, 4, 64, 2, 4, None, None, None, None) == NULL     # no output requested
    assert n(FAKE, -1, 64, 2, 4, FAKE, FAKE, None, None) == SHAPE
    assert n(None, 0, 64, 2, 4, None, None, None, None) == OK          # empty batch
    # the packed 2:4 operand: 2:4 and 1:4 only, rows and d multiples of 128
    assert n(FAKE, 128, 128, 4, 8, None, None, FAKE, None) == ARG
    assert n(FAKE, 128, 128, 2, 2, None, None, FAKE, None) == ARG
    assert n(FAKE, 128, 128, 3, 4, None, None, FAKE, None) == ARG
    assert n(FAKE, 100, 128, 2, 4, None, None, FAKE, None) == SHAPE
    assert n(FAKE, 128, 192, 2, 4, None, None, FAKE, None) == SHAPE
    assert n(FAKE, 128, 128, 1, 4, None, None, FAKE + 8, None) == ALIGN
    pb = lib.sig_nm_packed_bytes
    assert pb(128, 128) == 128 * 128 * 9 // 8
    assert pb(4096, 1024) == 4096 * 1024 * 9 // 8
    assert pb(100, 128) == 0 and pb(128, 64) == 0 and pb(0, 128) == 0
    g = lib.nm_act_gemm_packed
    assert g(None, 128, 128, FAKE, 128, FAKE, None) == NULL
    assert g(FAKE, 128, 128, FAKE, 96, FAKE, None) == SHAPE
    assert g(FAKE, 128, 64, FAKE, 128, FAKE, None) == SHAPE
    assert g(FAKE, 96, 128, FAKE, 128, FAKE, None) == SHAPE
    assert g(FAKE + 8, 128, 128, FAKE, 128, FAKE, None) == ALIGN


def test_multi_validation(lib):
    f = lib.sparse_gemv_multi
    P = ctypes.c_void_p * 2
    I = ctypes.c_int64 * 2
    W, Y, D = P(FAKE, FAKE), P(FAKE, FAKE), I(64, 64)
    big = 1 << 30
    assert f(0, W, D, 64, FAKE, 0.0, None, None, Y, FAKE, big, None) == ARG
    assert f(5, W, D, 64, FAKE, 0.0, None, None, Y, FAKE, big, None) == ARG
    assert f(2, None, D, 64, FAKE, 0.0, None, None, Y, FAKE, big, None) == NULL
    assert f(2, P(FAKE, None), D, 64, FAKE, 0.0, None, None, Y, FAKE, big, None) == NULL
    assert f(2, W, I(64, 60), 64, FAKE, 0.0, None, None, Y, FAKE, big, None) == SHAPE
    assert f(2, P(FAKE, FAKE_ODD), D, 64, FAKE, 0.0, None, None, Y, FAKE, big, None) == ALIGN
    assert f(2, W, D, 64, FAKE, 0.0, None, None, Y, None, big, None) == WORKSPACE
    need = lib.sig_workspace_bytes_multi(2, D, 64)
    assert need > 0
    assert f(2, W, D, 64, FAKE, 0.0, None, None, Y, FAKE, need - 1, None) == WORKSPACE
    assert lib.sig_workspace_bytes_multi(0, D, 64) == 0


def test_q8_validation(lib):
    f = lib.sparse_gemv_q8
    big = 1 << 30
    assert f(None, FAKE, 64, 64, FAKE, 0.0, FAKE, FAKE, big, None) == NULL
    assert f(FAKE, None, 64, 64, FAKE, 0.0, FAKE, FAKE, big, None) == NULL
    assert f(FAKE, FAKE, 64, 20, FAKE, 0.0, FAKE, FAKE, big, None) == SHAPE    # d_out % 8
    assert f(FAKE, FAKE, 0, 64, FAKE, 0.0, FAKE, FAKE, big, None) == SHAPE
    assert f(FAKE_ODD, FAKE, 64, 64, FAKE, 0.0, FAKE, FAKE, big, None) == ALIGN
    assert f(FAKE, FAKE + 1, 64, 64, FAKE, 0.0, FAKE, FAKE, big, None) == ALIGN   # scale alignment
    need = lib.sig_workspace_bytes(7, 64, 64, 0)
    assert need > 0
    assert f(FAKE, FAKE, 64, 64, FAKE, 0.0, FAKE, FAKE, need - 1, None) == WORKSPACE
    assert lib.sig_workspace_bytes(7, 64, 20, 0) == 0
    assert lib.sig_workspace_bytes(8, 64, 64, 0) == need      # fp8: the same plan
    assert lib.sig_workspace_bytes(9, 64, 64, 0) == need      # int4: the same plan
    q4 = lib.sparse_gemv_q4
    assert q4(None, FAKE, 64, 64, FAKE, 0.0, FAKE, FAKE, big, None) == NULL
    assert q4(FAKE, FAKE, 64, 64, None, 0.0, FAKE, FAKE, big, None) == NULL
    assert q4(FAKE, FAKE, 64, 20, FAKE, 0.0, FAKE, FAKE, big, None) == SHAPE    # d_out % 8
    assert q4(FAKE_ODD, FAKE, 64, 64, FAKE, 0.0, FAKE, FAKE, big, None) == ALIGN
    assert q4(FAKE, FAKE, 64, 64, FAKE, 0.0, FAKE, FAKE, need - 1, None) == WORKSPACE


def test_batch_validation(lib):
    f = lib.sparse_gemv_batch
    big = 1 << 30
    assert f(None, 64, 64, FAKE, 2, 0.0, FAKE, FAKE, big, None) == NULL
    assert f(FAKE, 64, 64, FAKE, 0, 0.0, FAKE, FAKE, big, None) == ARG
    assert f(FAKE, 64, 64, FAKE, 17, 0.0, FAKE, FAKE, big, None) == ARG
    assert f(FAKE, 60, 64, FAKE, 2, 0.0, FAKE, FAKE, big, None) == SHAPE     # d_in % 8
    assert f(FAKE, 64, 60, FAKE, 2, 0.0, FAKE, FAKE, big, None) == SHAPE     # d_out % 8
    assert f(FAKE, 64, 64, FAKE_ODD, 2, 0.0, FAKE, FAKE, big, None) == ALIGN
    need = lib.sig_workspace_bytes(6, 64, 64, 2)
    assert need > 0
    assert f(FAKE, 64, 64, FAKE, 2, 0.0, FAKE, FAKE, need - 1, None) == WORKSPACE
    assert f(FAKE, 64, 64, FAKE, 2, 0.0, FAKE, None, need, None) == WORKSPACE
    assert lib.sig_workspace_bytes(6, 64, 64, 17) == 0
    assert lib.sig_workspace_bytes(6, 64, 64, 16) > 0
    assert lib.sig_workspace_bytes(6, 60, 64, 2) == 0


def test_teal_mlp_validation(lib):
    f = lib.teal_mlp_sparse
    big = 1 << 30
    assert f(None, FAKE, FAKE, FAKE, 64, 128, 0.0, 0.0, FAKE, None, None, FAKE, big, None) == NULL
    assert f(FAKE, FAKE, FAKE, FAKE, 64, 120 + 4, 0.0, 0.0, FAKE, None, None, FAKE, big, None) == SHAPE
    assert f(FAKE, FAKE_ODD, FAKE, FAKE, 64, 128, 0.0, 0.0, FAKE, None, None, FAKE, big, None) == ALIGN
    need = lib.sig_workspace_bytes(3, 64, 128, 0)
    assert f(FAKE, FAKE, FAKE, FAKE, 64, 128, 0.0, 0.0, FAKE, None, None, FAKE, need - 1, None) == WORKSPACE


def test_rank_adapter_validation(lib):
    f = lib.rank_adapter_sparse
    big = 1 << 30
    assert f(None, FAKE, FAKE, 64, 32, 16, 0.0, FAKE, None, None, FAKE, big, None) == NULL
    assert f(FAKE, FAKE, FAKE, 64, 30, 16, 0.0, FAKE, None, None, FAKE, big, None) == SHAPE
    assert f(FAKE, FAKE, FAKE, 64, 32, 12, 0.0, FAKE, None, None, FAKE, big, None) == SHAPE
    assert f(FAKE, FAKE_ODD, FAKE, 64, 32, 16, 0.0, FAKE, None, None, FAKE, big, None) == ALIGN
    need = lib.sig_workspace_bytes(5, 64, 16, 32)
    assert need > 0
    assert f(FAKE, FAKE, FAKE, 64, 32, 16, 0.0, FAKE, None, None, FAKE, need - 1, None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, 64, 32, 16, 0.0, FAKE, None, None, None, need, None) == WORKSPACE
    assert lib.sig_workspace_bytes(5, 64, 16, 30) == 0


def test_gated_and_gemm_validation(lib):
    g = lib.gated_mlp_sparse
    big = 1 << 30
    assert g(FAKE, FAKE, FAKE, FAKE, None, 64, 128, 0.1, FAKE, None, None, FAKE, big, None) == NULL
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 124, 0.1, FAKE, None, None, FAKE, big, None) == SHAPE
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 128, 0.1, FAKE, None, None, FAKE, 16, None) == WORKSPACE
    assert g(FAKE, FAKE, FAKE_ODD, FAKE, FAKE, 64, 128, 0.1, FAKE, None, None, FAKE, big, None) == ALIGN
    m = lib.nm_act_gemm
    assert m(FAKE, 100, 1024, FAKE, 1024, 2, 4, FAKE, FAKE, big, None) == SHAPE    # rows % 128
    assert m(FAKE, 256, 1000, FAKE, 1024, 2, 4, FAKE, FAKE, big, None) == SHAPE    # K % 64
    assert m(FAKE, 256, 1024, FAKE, 1000, 2, 4, FAKE, FAKE, big, None) == SHAPE    # N % 128
    assert m(FAKE, 256, 1024, FAKE, 1024, 5, 4, FAKE, FAKE, big, None) == ARG
    assert m(FAKE, 256, 1024, FAKE, 1024, 2, 4, FAKE, FAKE, 10, None) == WORKSPACE
    assert m(None, 256, 1024, FAKE, 1024, 2, 4, FAKE, FAKE, big, None) == NULL
    r = lib.sig_row_norms
    assert r(FAKE, 4, 12, FAKE, None) == SHAPE
    assert r(FAKE, 4, 16, None, None) == NULL
    assert lib.sig_take_device_error(None, None) == NULL
    assert lib.sig_workspace_init(None, 16, None) == NULL
    assert lib.sig_workspace_init(FAKE + 16, 16, None) == ALIGN
    assert lib.sig_workspace_init(None, 0, None) == OK


def test_binding_fails_loudly_without_the_library(tmp_path):
    """The product path has no fallback: with libsig.so absent, importing the
    binding raises instead of computing anything elsewhere."""
    import types
    src = open(os.path.join(ROOT, "sparse_input_gemv_threshold_b200", "__init__.py")).read()
    key = 'LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsig.so")'
    assert key in src
    missing = str(tmp_path / "libsig.so")
    mod = types.ModuleType("sig_without_library")
    with pytest.raises(ImportError):
        exec(compile(src.replace(key, f"LIB_PATH = {missing!r}"), "sig_without_library", "exec"),
             mod.__dict__)


def test_product_never_touches_the_oracle():
    """Neither the binding, the build script nor the CUDA sources name the
    oracle package; only tests, the smoke check and the bench's CPU legs may."""
    pkg = os.path.join(ROOT, "sparse_input_gemv_threshold_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "oracle/" not in text, f


def test_nm_variant_and_helper_validation(lib):
    e = lib.sparsify_nm_ex
    assert e(FAKE, 4, 64, 3, 2, None, None, 0, FAKE, None, None, None) == ARG       # n > m
    assert e(FAKE, 4, 36, 2, 8, None, None, 0, FAKE, None, None, None) == SHAPE     # m does not divide d
    assert e(FAKE, 4, 64, 2, 4, None, None, 0, None, None, None, None) == NULL      # X_masked required
    assert e(None, 4, 64, 2, 4, None, None, 0, FAKE, None, None, None) == NULL
    assert e(None, 0, 64, 2, 4, None, None, 1, None, None, None, None) == OK        # empty batch
    assert e(FAKE, 4, 64, 2, 4, None, FAKE + 4, 0, FAKE, None, None, None) == ALIGN   # norms: 16 B
    assert e(FAKE, 4, 64, 2, 4, FAKE + 2, None, 0, FAKE, None, None, None) == ALIGN   # shift: 4 B
    assert e(FAKE, 4, 64, 2, 4, None, None, 1, FAKE, None, FAKE + 2, None) == ALIGN   # gamma: 4 B
    assert e(FAKE, 4, 64, 2, 4, None, None, 0, FAKE, FAKE + 1, None, None) == ALIGN   # mask: 4 B
    g = lib.nm_act_gemm_ex
    big = 1 << 30
    args = dict(shift=None, norms=None, var=0, cs=None, ws=FAKE, nbytes=big)

    def call(rows=256, K=1024, N=1024, n=2, m=4, **kw):
        a = {**args, **kw}
        return g(FAKE, rows, K, FAKE, N, n, m, a["shift"], a["norms"], a["var"], a["cs"], FAKE,
                 a["ws"], a["nbytes"], None)
    assert call(shift=FAKE) == NULL                      # a shift needs the weight's column sums
    assert call(rows=100) == SHAPE
    assert call(K=1000) == SHAPE
    assert call(n=5) == ARG
    assert call(shift=FAKE + 2, cs=FAKE) == ALIGN
    assert call(shift=FAKE, cs=FAKE + 2) == ALIGN
    assert call(norms=FAKE + 4) == ALIGN
    assert call(nbytes=16) == WORKSPACE
    assert call(ws=None) == WORKSPACE
    c = lib.sig_col_sums
    assert c(None, 4, 16, FAKE, None) == NULL
    assert c(FAKE, 4, 16, None, None) == NULL
    assert c(FAKE, 0, 16, FAKE, None) == SHAPE
    assert c(FAKE + 1, 4, 16, FAKE, None) == ALIGN       # fp16: 2 B
    assert c(FAKE, 4, 16, FAKE + 2, None) == ALIGN       # float32: 4 B
    assert lib.sig_row_norms(FAKE, 4, 16, FAKE + 2, None) == ALIGN


def test_noalloc_validation(lib):
    f = lib.gated_mlp_sparse_noalloc
    assert f(FAKE, FAKE, FAKE, FAKE, None, 64, 128, 0.1, FAKE, None, None, None) == NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 60, 128, 0.1, FAKE, None, None, None) == SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 131072 + 8, 0.1, FAKE, None, None, None) == SHAPE
    assert f(FAKE, FAKE_ODD, FAKE, FAKE, FAKE, 64, 128, 0.1, FAKE, None, None, None) == ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 64, 128, 0.1, FAKE, None, None, None) == ALIGN
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 128, 0.1, FAKE, None, FAKE + 1, None) == ALIGN


def test_noalloc_scratch_covers_every_accepted_shape(lib):
    """Every (d_model, d_ff) that gated_mlp_sparse accepts (multiples of 8 up
    to SIG_MAX_D_IN) fits the allocation-free entry point's 4 MiB scratch.

    The gated MLP's workspace is the sum of a term that depends only on d_ff
    (the gate/up product's counters and partials, and the hidden vector) and
    one that depends only on d_model (the down product's): the maximum of the
    sum is the sum of the two one-dimensional maxima.  The decomposition is
    checked on a spread of pairs first, so that a change that couples the two
    terms fails here instead of hiding an oversize shape."""
    ws = lib.sig_workspace_bytes
    OP_GATED_MLP, LIMIT, MAX_D = 3, 4 << 20, 131072
    sizes = range(8, MAX_D + 1, 8)
    base = ws(OP_GATED_MLP, 8, 8, 0)
    f = {d: ws(OP_GATED_MLP, 8, d, 0) - base for d in sizes}      # d_ff term
    g = {d: ws(OP_GATED_MLP, d, 8, 0) - base for d in sizes}      # d_model term
    for dm in (8, 1024, 4096, 8192, 11008, 28672, 75776, MAX_D):
        for dff in (8, 4096, 11008, 28672, 75776, 75784, MAX_D):
            assert ws(OP_GATED_MLP, dm, dff, 0) == base + f[dff] + g[dm], (dm, dff)
    worst = base + max(f.values()) + max(g.values())
    assert worst <= LIMIT, worst


def test_32bit_buffers_must_be_4_byte_aligned(lib):
    """Masks, index lists, counts and float vectors are checked on the host,
    like the 16-byte rules, before anything is enqueued."""
    big = 1 << 30
    odd = FAKE + 2
    st = lib.sparsify_threshold
    assert st(FAKE, 64, 0.0, odd, None, None, None) == ALIGN
    assert st(FAKE, 64, 0.0, FAKE, odd, None, None) == ALIGN
    assert st(FAKE, 64, 0.0, FAKE, FAKE, odd, None) == ALIGN
    tk = lib.sparsify_topk
    assert tk(FAKE, 64, 3, odd, FAKE, FAKE, None, 0, None) == ALIGN
    assert tk(FAKE, 64, 3, FAKE, odd, FAKE, None, 0, None) == ALIGN
    assert tk(FAKE, 64, 3, FAKE, FAKE, odd, None, 0, None) == ALIGN
    assert lib.sparsify_nm(FAKE, 4, 64, 2, 4, None, odd, None, None) == ALIGN
    sg = lib.sparse_gemv
    assert sg(FAKE, 64, 64, FAKE, 0.0, odd, FAKE, FAKE, FAKE, big, None) == ALIGN
    assert sg(FAKE, 64, 64, FAKE, 0.0, FAKE, odd, FAKE, FAKE, big, None) == ALIGN
    P = ctypes.c_void_p * 2
    I = ctypes.c_int64 * 2
    mm = lib.sparse_gemv_multi
    assert mm(2, P(FAKE, FAKE), I(64, 64), 64, FAKE, 0.0, odd, FAKE, P(FAKE, FAKE), FAKE, big,
              None) == ALIGN
    ga = lib.gated_mlp_sparse
    assert ga(FAKE, FAKE, FAKE, FAKE, odd, 64, 128, 0.1, FAKE, None, None, FAKE, big, None) == ALIGN
    assert ga(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 128, 0.1, FAKE, None, odd, FAKE, big, None) == ALIGN
    te = lib.teal_mlp_sparse
    assert te(FAKE, FAKE, FAKE, FAKE, 64, 128, 0.0, 0.0, FAKE, None, odd, FAKE, big, None) == ALIGN
    ra = lib.rank_adapter_sparse
    assert ra(FAKE, FAKE, FAKE, 64, 32, 16, 0.0, FAKE, None, odd, FAKE, big, None) == ALIGN
