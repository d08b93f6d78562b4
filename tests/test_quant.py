"""GPU parity of fa_compress_kv against the fp32 oracle quantiser: codes and
scales must match bit for bit (fkl_python PR #6, Summary: per-token int8 with
one fp32 scale; bit-exact gate)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def gpu_compress(x):
    from flashattention_attention_b200 import fa
    codes, scales = fa.compress_kv(x.cuda().contiguous())
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    return codes.cpu().numpy(), scales.cpu().numpy()


def assert_bit_exact(x):
    c, s = gpu_compress(x)
    rc, rs = oracle.compress_kv(x)
    assert np.array_equal(s.view(np.uint32), rs.view(np.uint32)), "scales differ"
    bad = np.argwhere(c != rc)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,d", [(1, 16), (7, 64), (33, 128), (130, 128), (5, 256), (3, 1024),
                                    (9, 48), (1001, 128), (17, 640)])
def test_bit_exact_random(dtype, rows, d):
    rng = np.random.default_rng(rows * 1000 + d)
    mag = 10.0 ** rng.uniform(-6, 6, size=(rows, 1))
    x = torch.from_numpy(rng.standard_normal((rows, d)) * mag).float().to(dtype)
    assert_bit_exact(x)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_special_rows(dtype):
    d = 64
    rows = []
    rows.append(np.zeros(d))                                            # all zero: s = 0, codes 0
    halves = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 126.5, -126.5, 127.0])
    rows.append(np.resize(halves, d))                                   # ties at s = 1
    one_hot = np.zeros(d); one_hot[5] = -3.0
    rows.append(one_hot)                                                 # single nonzero
    rows.append(np.full(d, 7.25))                                       # constant row
    rows.append(np.linspace(-1, 1, d) * 1e-30)                          # tiny values
    rows.append(np.linspace(-1, 1, d) * 3e38)                           # near fp32 max
    x = torch.tensor(np.stack(rows), dtype=torch.float32).to(dtype)
    assert_bit_exact(x)


def test_subnormal_fp32():
    rng = np.random.default_rng(5)
    x = torch.from_numpy((rng.standard_normal((8, 32)) * 1e-39).astype(np.float32))
    assert_bit_exact(x)


def test_compression_ratio_from_buffers():
    """fkl_python PR #6, Verification: the compression ratio (3.76 against
    a gate of 3.5) at head_dim 64, measured from the GPU's own output buffers."""
    x = torch.randn(4096, 64)
    c, s = gpu_compress(x)
    ratio = x.numel() * 4 / (c.nbytes + s.nbytes)
    assert f"{ratio:.2f}" == "3.76" and ratio > 3.5


def test_full_decode_cache_rows(decode_workload):
    """Every valid (token, kv-head) row of the int8-KV decode workload's K and
    V caches (4,361,088 rows of d = 128), bit for bit."""
    w = decode_workload
    for t in (w.k, w.v):
        rows = torch.cat([t[b * w.hkv:(b + 1) * w.hkv, :w.lengths[b]].reshape(-1, w.d)
                          for b in range(w.batch)])
        assert_bit_exact(rows)


def test_near_ties_fp32():
    """Rows built so that most quotients x / s fall within a few ulps of a
    half-integer (k + 0.5), where a quotient that is not the correctly
    rounded one would flip the code; s takes random significands over many
    binades (both the reciprocal-and-correction path and, for |s| beyond
    2^60 or below 2^-60, the IEEE-division path)."""
    rng = np.random.default_rng(11)
    rows, d = 1 << 15, 128
    expo = rng.integers(-70, 70, rows).astype(np.float64)
    s_target = (1.0 + rng.random(rows)) * np.exp2(expo)
    amax = (s_target * 127.0).astype(np.float32)
    s = amax / np.float32(127.0)                               # what the quantiser computes
    k = rng.integers(0, 127, (rows, d - 1)).astype(np.float32)
    x = ((k + np.float32(0.5)) * s[:, None]).astype(np.float32)
    step = rng.integers(-3, 4, (rows, d - 1))
    for _ in range(3):
        up, dn = step > 0, step < 0
        x = np.where(up, np.nextafter(x, np.float32(np.inf)), np.where(dn, np.nextafter(x, np.float32(-np.inf)), x))
        step = step - np.sign(step)
    x = np.minimum(x, amax[:, None])
    x *= np.where(rng.random((rows, d - 1)) < 0.5, np.float32(-1), np.float32(1))
    full = np.concatenate([amax[:, None], x], axis=1).astype(np.float32)
    assert_bit_exact(torch.from_numpy(full))
