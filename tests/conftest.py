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


def assert_close_bf16(got, ref, atol=2e-2, rel_l2=5e-3, what=""):
    """The bf16 output gate: max abs <= 2e-2 and relative
    L2 <= 5e-3 against the fp64 oracle run on the same bf16 inputs."""
    import numpy as np
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - r).max() if g.size else 0.0
    denom = np.linalg.norm(r)
    rl2 = np.linalg.norm(g - r) / denom if denom > 0 else np.linalg.norm(g - r)
    assert err <= atol and rl2 <= rel_l2, f"{what}: max abs {err:.3e}, rel L2 {rl2:.3e}"
    return err, rl2


@pytest.fixture(scope="session")
def decode_workload():
    """The full-size int8-KV decode workload (CPU tensors), built once."""
    from flashattention_attention_b200 import inputs
    return inputs.int8kv_decode()
