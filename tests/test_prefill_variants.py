"""The opt-in prefill variants against the fp64 oracle, each in a child
process with its switch set (the library reads the switches once, at load):

* FA_PREFILL_PAIR=1: clusters of two CTAs run M = 256 tensor-core tiles, so
  one K/V fetch serves four query heads of a GQA group (d = 128, group size a
  multiple of 4);
* FA_PREFILL_QUAD=1: one CTA takes four query heads of a group with 64-key
  tiles (d = 64, bf16, group size a multiple of 4).

SKaiNET-transformers PR #419, Summary: one task per GQA group.  The bf16 and
int8-KV prefill parity files (full-size workloads included), the ring steps
and the paged prefill run again under each switch; cases the variant does not
cover run the default kernels there as well."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_parity_files(env_var):
    env = dict(os.environ, **{env_var: "1"})
    files = ["test_fwd_bf16.py", "test_fwd_int8.py", "test_ring.py", "test_decode_paged.py"]
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu"] + [
        os.path.join(ROOT, "tests", f) for f in files]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def test_prefill_parity_with_cta_pairs():
    _run_parity_files("FA_PREFILL_PAIR")


def test_prefill_parity_with_four_heads_per_cta():
    _run_parity_files("FA_PREFILL_QUAD")
