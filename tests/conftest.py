import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if gpu_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionstart(session):
    """Build libfa.so and the oracle in-tree before any test imports them
    (a no-op when both are up to date)."""
    import shutil
    if shutil.which("nvcc") or os.path.exists("/usr/local/cuda/bin/nvcc"):
        from flashattention_attention_b200 import build as fa_build
        fa_build.build()
    import oracle
    oracle.build()


def bf16_half_spacing(r):
    """Half the distance between neighbouring bf16 numbers at |r| (8
    significant bits: 2^(e-8) for |r| in [2^e, 2^(e+1))); the most a correct
    round-to-nearest cast to bf16 can move a value."""
    import numpy as np
    a = np.maximum(np.abs(np.asarray(r, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(np.int64) - 8)


def assert_close_bf16(got, ref, atol=2e-2, rel_l2=5e-3, what=""):
    """The bf16 output gate against the fp64 oracle run on the same bf16
    inputs: relative L2 <= 5e-3, and every element within 2e-2 of the oracle
    once the output's own cast to bf16 is allowed for, i.e.
    |got - ref| <= 2e-2 + half the bf16 spacing at ref.  The allowance is at
    most 2^-9 |ref|: it matters only for |ref| >= 2, and above 8 no bf16
    number lies within 2e-2 of most reals, so a flat 2e-2 would fail even a
    correctly rounded result.  The flat max abs is reported beside it."""
    import numpy as np
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    diff = np.abs(g - r)
    err = diff.max() if g.size else 0.0
    excess = (diff - bf16_half_spacing(r)).max() if g.size else 0.0
    denom = np.linalg.norm(r)
    rl2 = np.linalg.norm(g - r) / denom if denom > 0 else np.linalg.norm(g - r)
    assert excess <= atol and rl2 <= rel_l2, (
        f"{what}: max abs {err:.3e} (beyond the bf16 cast {excess:.3e}), rel L2 {rl2:.3e}")
    return err, rl2


def assert_close_bf16_planes(got, ref, what="", chunk=8):
    """assert_close_bf16 over a large [planes, rows, d] result, a few planes
    at a time (bounded host memory); the same gate on the whole array."""
    import numpy as np
    n = ref.shape[0]
    assert tuple(got.shape) == tuple(ref.shape), (tuple(got.shape), ref.shape)
    err = excess = 0.0
    sq_diff = sq_ref = 0.0
    for p0 in range(0, n, chunk):
        g = got[p0:p0 + chunk].float().numpy().astype(np.float64) if hasattr(got, "float") else \
            np.asarray(got[p0:p0 + chunk], dtype=np.float64)
        r = np.asarray(ref[p0:p0 + chunk], dtype=np.float64)
        assert np.isfinite(g).all(), f"{what}: non-finite output in planes {p0}..{p0 + chunk - 1}"
        diff = np.abs(g - r)
        err = max(err, float(diff.max()))
        excess = max(excess, float((diff - bf16_half_spacing(r)).max()))
        sq_diff += float((diff * diff).sum())
        sq_ref += float((r * r).sum())
    rl2 = (sq_diff / sq_ref) ** 0.5 if sq_ref > 0 else sq_diff ** 0.5
    assert excess <= 2e-2 and rl2 <= 5e-3, (
        f"{what}: max abs {err:.3e} (beyond the bf16 cast {excess:.3e}), rel L2 {rl2:.3e}")
    return err, rl2


@pytest.fixture(scope="session")
def decode_workload():
    """The full-size int8-KV decode workload (CPU tensors), built once."""
    from flashattention_attention_b200 import inputs
    return inputs.int8kv_decode()
