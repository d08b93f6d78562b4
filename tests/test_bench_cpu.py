"""The bench's own bookkeeping, on the CPU: the FLOP count of a prefill (128 x
128 tiles of a fixed grid that the visible band touches, and the exact
visible pairs) against a brute-force mask, the headline workload's figures,
and the rule that a committed DRAM-traffic figure is reported only while the
kernel's sources hash the same as when it was captured."""
import os
import shutil
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def brute_band(s_q, s_k, causal, window, tile=128):
    """Tiles of the fixed grid holding a visible (query, key) pair, and the
    pairs, straight from the mask (bottom-right causal alignment; a window
    W keeps the W keys up to the query's own position)."""
    i = np.arange(s_q)[:, None]
    j = np.arange(s_k)[None, :]
    p = i + s_k - s_q
    vis = np.ones((s_q, s_k), dtype=bool)
    if causal:
        vis &= j <= p
    if window > 0:
        vis &= j > p - window
    tiles = 0
    for qb in range(0, s_q, tile):
        for kb in range(0, s_k, tile):
            tiles += bool(vis[qb:qb + tile, kb:kb + tile].any())
    return tiles, int(vis.sum())


@pytest.mark.parametrize("s_q,s_k", [(128, 128), (300, 300), (33, 127), (127, 33), (1, 700), (700, 1), (256, 640),
                                     (513, 257)])
@pytest.mark.parametrize("causal,window", [(True, 0), (False, 0), (True, 100), (False, 100), (True, 1),
                                           (True, 300)])
def test_band_tiles_equals_the_brute_force_mask(s_q, s_k, causal, window):
    import bench
    assert bench.band_tiles(s_q, s_k, causal, window) == brute_band(s_q, s_k, causal, window)


def test_headline_flops():
    """B = 4, Hq = 32, S = 4096, d = 128, causal: 32 q-blocks give 32 * 33 / 2
    tiles per head plane (0.5669 TFLOP) and S (S + 1) / 2 pairs (0.5499)."""
    import bench
    from flashattention_attention_b200 import inputs
    w = inputs.gqa_causal_prefill()
    tiles_flops, exact_flops = bench.prefill_flops(w)
    per_pair = 4 * 32 * 4 * 128
    assert tiles_flops == per_pair * (32 * 33 // 2) * 128 * 128
    assert exact_flops == per_pair * 4096 * 4097 // 2
    assert round(tiles_flops / 1e12, 4) == 0.5669 and round(exact_flops / 1e12, 4) == 0.5499


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    import bench
    csrc = tmp_path / "flashattention_attention_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.KERNEL_SOURCES["decode_sk_kernel<128>"]:
        shutil.copy(os.path.join(ROOT, "flashattention_attention_b200", "csrc", f), csrc / f)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    import hashlib
    h = hashlib.sha256()
    for f in bench.KERNEL_SOURCES["decode_sk_kernel<128>"]:
        h.update((csrc / f).read_bytes())
    sha = h.hexdigest()[:16]
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# kernel source_sha bytes_per_launch\n"
        f"decode_sk_kernel<128> {sha} 123456 1 2 capture.md\n"
        "decode_sk_kernel<128,bf16> 0000000000000000 999 1 2 capture.md\n")
    assert bench.measured_traffic("decode_sk_kernel<128>") == 123456
    assert bench.measured_traffic("decode_sk_kernel<128,bf16>") is None   # another source hash
    assert bench.measured_traffic("no_such_kernel") is None
    with open(csrc / "decode.cu", "a") as fh:                            # the source changes
        fh.write("\n")
    assert bench.measured_traffic("decode_sk_kernel<128>") is None


def test_committed_traffic_file_is_consistent():
    """Every line of profiles/traffic.txt names a kernel the bench knows, a
    16-hex-digit source hash, and bytes per launch = read + write."""
    import bench
    lines = [l.split() for l in open(os.path.join(ROOT, "profiles", "traffic.txt")) if not l.startswith("#")]
    assert lines
    for f in lines:
        assert f[0] in bench.KERNEL_SOURCES, f[0]
        assert len(f[1]) == 16 and int(f[1], 16) >= 0
        assert int(f[2]) == int(f[3]) + int(f[4]) > 0
