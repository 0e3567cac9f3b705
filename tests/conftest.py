import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: large shapes; several seconds of CPU work")


def load_builder():
    """The build script as a module, loaded by path (the package import would
    load the library it builds)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "sig_build", os.path.join(ROOT, "sparse_input_gemv_threshold_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def golden_path(name: str) -> str:
    return os.path.join(GOLDEN, name)


# ---------------------------------------------------------------------------
# GPU helpers (used only by tests marked gpu)
# ---------------------------------------------------------------------------

@pytest.fixture(scope="session")
def sig():
    """The product binding, built in-tree if needed.  Fails (never skips) when
    the library or the GPU is missing: a gpu test must run the CUDA path."""
    import torch
    load_builder().build()
    import sparse_input_gemv_threshold_b200 as mod
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    return mod


@pytest.fixture(autouse=True)
def _no_bounded_wait_gave_up(request):
    """After every gpu test: no kernel may have given up a bounded wait (the
    library's device error words are read and cleared).  A test that makes a
    wait run out on purpose reads and clears the words itself."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    mod = sys.modules.get("sparse_input_gemv_threshold_b200")
    if mod is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    code = mod.take_device_error()
    assert code == 0, f"a kernel gave up a bounded wait (device error bits {code:#x})"


def to_dev(a):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(t):
    return t.detach().cpu().numpy()


def mask_words(t):
    """Device int32 mask words -> numpy uint32."""
    return to_host(t).view("uint32")


def assert_within(y16, y64, bound, what=""):
    """The parity tolerance per output: |y - y64| <= 2e-3 * sum|W x| (plus one
    fp16 subnormal step, the finest spacing an fp16 result can have)."""
    import numpy as np
    y = np.asarray(y16, dtype=np.float16).astype(np.float64).ravel()
    y64 = np.asarray(y64, dtype=np.float64).ravel()
    bound = np.asarray(bound, dtype=np.float64).ravel()
    err = np.abs(y - y64)
    tol = 2e-3 * bound + 2.0 ** -24
    bad = np.flatnonzero(err > tol)
    if bad.size:
        j = bad[np.argmax((err - tol)[bad])]
        raise AssertionError(f"{what}: {bad.size}/{y.size} outputs out of tolerance; "
                             f"worst j={j} y={y[j]} ref={y64[j]} bound={bound[j]}")
    assert np.isfinite(y).all()


def fp32_sum_bound(n_terms, abs_sum):
    """Worst-case error of a float32 sum of ``n_terms`` exactly representable
    products, in any order: gamma_n * sum|terms| with gamma_n = n u / (1 - n u),
    u = 2^-24 (every fp16 x fp16 product is exact in float32; only the n - 1
    additions round)."""
    import numpy as np
    u = 2.0 ** -24
    n = np.asarray(n_terms, dtype=np.float64)
    return n * u / (1.0 - n * u) * np.asarray(abs_sum, dtype=np.float64)


def silu_mul_tolerance(g, u, eg, eu, h_ref):
    """How far the GPU's h = fp16(SiLU(g) u), computed in float32 from g and u
    that carry errors of at most eg and eu, may sit from the oracle's h (float64
    g, u, one fp16 rounding): the errors carried through h = SiLU(g) u by its
    derivatives (dSiLU/dg = sigma(g) (1 + g (1 - sigma(g)))), eight float32
    roundings of the SiLU and product evaluation, and one fp16 ulp for the
    final rounding."""
    import numpy as np
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-g))
    dsilu = sg * (1.0 + g * (1.0 - sg))
    h64 = g * sg * u
    return (np.spacing(np.abs(h_ref)).astype(np.float64) + np.abs(dsilu * u) * eg
            + np.abs(g * sg) * eu + 8 * 2.0 ** -24 * np.abs(h64))
