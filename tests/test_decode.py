"""GPU parity of fa_attention_decode (int8 KV cache) against the fp64 oracle
on the dequantised cache (fkl_python PR #6, Verification: a one-query
decode step over 256 int8-cached keys; bf16 output gate: max abs <= 2e-2
and relative L2 <= 5e-3)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def build_case(seed, B, hq, hkv, d, cap, lengths):
    return inputs.decode_cache("t", lengths=lengths, hq=hq, hkv=hkv, d=d, capacity=cap, seed=seed)


def gpu_decode(w, **kw):
    from flashattention_attention_b200 import fa
    kc, ks = fa.compress_kv(w.k.cuda())
    vc, vs = fa.compress_kv(w.v.cuda())
    lens = torch.tensor(w.lengths, dtype=torch.int32, device="cuda")
    out = fa.attention_decode(w.q.reshape(-1, w.d).cuda(), kc, vc, lens, hq=w.hq, hkv=w.hkv,
                              k_scales=ks, v_scales=vs, scale=w.scale, **kw)
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    return out.cpu(), (kc.cpu().numpy(), ks.cpu().numpy(), vc.cpu().numpy(), vs.cpu().numpy())


def oracle_decode(w, gpu_codes=None, window=0, epilogue=(), rows=None):
    rk, rks = oracle.compress_kv(w.k)
    rv, rvs = oracle.compress_kv(w.v)
    if gpu_codes is not None:  # the quantiser gate: bit-exact
        kc, ks, vc, vs = gpu_codes
        assert np.array_equal(kc, rk) and np.array_equal(ks.view(np.uint32), rks.view(np.uint32))
        assert np.array_equal(vc, rv) and np.array_equal(vs.view(np.uint32), rvs.view(np.uint32))
    return oracle.decode(w.q, oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs), w.lengths,
                         hq=w.hq, hkv=w.hkv, scale=w.scale, window=window, epilogue=epilogue, rows=rows)


CASES = [
    # B, hq, hkv, d, cap, lengths
    (3, 8, 2, 128, 1024, [1, 256, 1000]),
    (4, 32, 8, 128, 2048, [31, 32, 33, 2048]),
    (2, 8, 8, 128, 512, [257, 511]),          # G = 1
    (2, 16, 2, 128, 768, [700, 100]),         # G = 8
    (2, 4, 2, 64, 1024, [999, 64]),           # d = 64
    (1, 2, 1, 128, 256, [256]),               # the page's s_k = 256 decode step
    (2, 32, 2, 128, 1024, [1000, 77]),        # G = 16: two passes of 8 heads
    (2, 24, 2, 64, 512, [300, 512]),          # G = 12: two passes of 6
    (1, 9, 1, 128, 512, [400]),               # G = 9: three passes of 3
    (3, 8, 2, 32, 1024, [1000, 33, 512]),     # d = 32
    (2, 8, 2, 96, 1024, [999, 100]),          # d = 96
    (2, 8, 2, 256, 1024, [700, 1024]),        # d = 256
    (1, 32, 2, 256, 512, [300]),              # d = 256 with a group of 16
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-hq{c[1]}-hkv{c[2]}-d{c[3]}")
def test_decode_cases(case):
    B, hq, hkv, d, cap, lengths = case
    w = build_case(7, B, hq, hkv, d, cap, lengths)
    got, codes = gpu_decode(w)
    ref = oracle_decode(w, codes)
    assert_close_bf16(got.float().numpy().reshape(ref.shape), ref, what=str(case))


def test_decode_window_and_epilogue():
    w = build_case(8, 3, 8, 2, 128, 2048, [2000, 300, 1025])
    epi = [("mul", 2.0), ("add", 0.5)]
    got, codes = gpu_decode(w, window=700, epilogue=epi)
    ref = oracle_decode(w, codes, window=700, epilogue=epi)
    assert_close_bf16(got.float().numpy().reshape(ref.shape), ref)


def test_decode_empty_cache_gives_epilogue_of_zero():
    w = build_case(9, 2, 4, 2, 128, 256, [0, 100])
    got, codes = gpu_decode(w, epilogue=[("add", 0.5)])
    ref = oracle_decode(w, codes, epilogue=[("add", 0.5)])
    g = got.float().numpy().reshape(ref.shape)
    assert np.all(g[:4] == 0.5)
    assert_close_bf16(g, ref)


def test_split_count_does_not_change_the_result():
    w = build_case(10, 2, 8, 2, 128, 4096, [4096, 3000])
    a, _ = gpu_decode(w, split_keys=256)
    b, _ = gpu_decode(w, split_keys=4096)
    ref = oracle_decode(w)
    assert_close_bf16(a.float().numpy().reshape(ref.shape), ref)
    assert_close_bf16(b.float().numpy().reshape(ref.shape), ref)
    assert (a.float() - b.float()).abs().max() <= 2e-2


def test_full_size_int8_decode(decode_workload):
    """The full workload: B=16, Hq=32, Hkv=8, d=128, capacity 32768, cache
    lengths U[1024, 32768] from seed 0 -- every output row checked."""
    w = decode_workload
    got, codes = gpu_decode(w, max_seqlen=max(w.lengths))
    ref = oracle_decode(w, codes)
    assert_close_bf16(got.float().numpy().reshape(ref.shape), ref, what="full decode")
