"""GPU parity of fa_attention_decode over a bf16 KV cache against the fp64
oracle on the same bf16 values (the one-query decode step that fkl_python
PR #6, Verification, checks against 256 cached keys, here with an
uncompressed cache;
bf16 output gate: max abs <= 2e-2 and relative L2 <= 5e-3).
Cache rows outside the attended band may hold any bytes, NaN and Inf
included; they must not reach the result."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def gpu_decode_bf16(w, k=None, v=None, **kw):
    from flashattention_attention_b200 import fa
    k = w.k if k is None else k
    v = w.v if v is None else v
    lens = torch.tensor(w.lengths, dtype=torch.int32, device="cuda")
    out = fa.attention_decode(w.q.reshape(-1, w.d).cuda(), k.cuda(), v.cuda(), lens, hq=w.hq, hkv=w.hkv,
                              scale=w.scale, **kw)
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    return out.cpu()


def oracle_decode_bf16(w, window=0, epilogue=(), rows=None):
    return oracle.decode(w.q, w.k, w.v, w.lengths, hq=w.hq, hkv=w.hkv, scale=w.scale, window=window,
                         epilogue=epilogue, rows=rows)


CASES = [
    # B, hq, hkv, d, cap, lengths
    (3, 8, 2, 128, 1024, [1, 256, 1000]),
    (4, 32, 8, 128, 2048, [31, 32, 33, 2048]),
    (2, 8, 8, 128, 512, [257, 511]),          # G = 1
    (2, 16, 2, 128, 768, [700, 100]),         # G = 8
    (2, 4, 2, 64, 1024, [999, 64]),           # d = 64
    (1, 2, 1, 128, 256, [256]),               # the page's s_k = 256 decode step
    (2, 32, 2, 128, 1024, [1000, 77]),        # G = 16: two passes of 8 heads
    (1, 12, 1, 64, 512, [333]),               # G = 12: two passes of 6
    (3, 8, 2, 32, 1024, [1000, 33, 512]),     # d = 32: one 32-dim chunk (64-byte swizzle)
    (2, 8, 2, 96, 1024, [999, 100]),          # d = 96: a 64-dim chunk and a 32-dim tail
    (2, 8, 2, 256, 1024, [1000, 33]),         # d = 256: four 64-dim chunks, one ring stage per worker
    (1, 16, 1, 256, 512, [512]),              # d = 256, G = 16
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-hq{c[1]}-hkv{c[2]}-d{c[3]}")
def test_decode_bf16_cases(case):
    B, hq, hkv, d, cap, lengths = case
    w = inputs.decode_cache("t", lengths=lengths, hq=hq, hkv=hkv, d=d, capacity=cap, seed=27, kv_int8=False)
    got = gpu_decode_bf16(w)
    ref = oracle_decode_bf16(w)
    assert_close_bf16(got.float().numpy().reshape(ref.shape), ref, what=str(case))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_decode_bf16_window_epilogue_and_poisoned_rows(d):
    """Rows past L_b and, with a window, rows before L_b - W are NaN / Inf in
    both caches; the result must equal the oracle on the clean cache."""
    lengths = [2000, 300, 1025, 45]
    w = inputs.decode_cache("t", lengths=lengths, hq=8, hkv=2, d=d, capacity=2048, seed=28, kv_int8=False)
    window = 700
    k, v = w.k.clone(), w.v.clone()
    for b, L in enumerate(lengths):
        lo = max(0, L - window)
        for t, bad in ((k, float("nan")), (v, float("inf"))):
            t[b * 2:(b + 1) * 2, L:] = bad
            t[b * 2:(b + 1) * 2, :lo] = -bad if bad == float("inf") else bad
    epi = [("mul", 2.0), ("add", 0.5)]
    got = gpu_decode_bf16(w, k=k, v=v, window=window, epilogue=epi)
    ref = oracle_decode_bf16(w, window=window, epilogue=epi)
    g = got.float().numpy().reshape(ref.shape)
    assert np.isfinite(g).all()
    assert_close_bf16(g, ref)


def test_decode_bf16_empty_cache_and_split_invariance():
    from flashattention_attention_b200 import fa  # noqa: F401  (extension must load)
    w = inputs.decode_cache("t", lengths=[0, 4096, 3000], hq=8, hkv=2, d=128, capacity=4096, seed=29,
                            kv_int8=False)
    a = gpu_decode_bf16(w, epilogue=[("add", 0.5)], split_keys=256)
    b = gpu_decode_bf16(w, epilogue=[("add", 0.5)], split_keys=4096)
    ref = oracle_decode_bf16(w, epilogue=[("add", 0.5)])
    ga = a.float().numpy().reshape(ref.shape)
    assert np.all(ga[:8] == 0.5)
    assert_close_bf16(ga, ref)
    assert_close_bf16(b.float().numpy().reshape(ref.shape), ref)


def test_full_size_bf16_decode():
    """The decode workload's shape with an uncompressed cache: B=16, Hq=32,
    Hkv=8, d=128, capacity 32768, lengths U[1024, 32768] from seed 0; every
    output row checked."""
    w = inputs.int8kv_decode()
    got = gpu_decode_bf16(w, max_seqlen=max(w.lengths))
    ref = oracle_decode_bf16(w)
    assert_close_bf16(got.float().numpy().reshape(ref.shape), ref, what="full bf16 decode")
