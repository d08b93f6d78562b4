"""A seeded sweep over the configuration space of the tensor-core prefill
and the decode, each case against the fp64 oracle at a small size (the same
gates as the hand-picked cases: bf16 output within max abs 2e-2 of the
oracle plus half a bf16 unit, relative L2 <= 5e-3; int8 codes and scales
bit-exact; fkl_python PR #6, Verification).  The draws cover what the
hand-picked cases cover one axis at a time, in combination: layout (dense or
varlen), head size (32 .. 256), GQA group, causal and window masks
(SKaiNET-transformers PR #419, Summary: GQA groups and sliding windows),
s_q against s_k, bf16 or int8 K/V, and the epilogue chain."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu

HEAD_SIZES = [32, 64, 96, 128, 160, 192, 224, 256]
N_PREFILL = 24
N_DECODE = 12


def prefill_case(i):
    """Case i of the sweep: every choice drawn from default_rng(1000 + i)."""
    rng = np.random.default_rng(1000 + i)
    d = int(rng.choice(HEAD_SIZES))
    hkv = int(rng.choice([1, 2, 4]))
    group = int(rng.choice([1, 2, 3, 4, 8]))
    varlen = bool(rng.integers(2))
    causal = bool(rng.integers(2))
    window = int(rng.choice([0, 0, 37, 128, 300]))
    int8 = bool(rng.integers(2))
    n_epi = int(rng.integers(0, 4))
    epilogue = [(("mul", "add")[int(rng.integers(2))], float(rng.choice([-1.5, 0.25, 0.5, 2.0, 3.0])))
                for _ in range(n_epi)]
    if varlen:
        lengths = [int(x) for x in rng.integers(1, 300, int(rng.integers(1, 5)))]
        shape = dict(lengths=lengths)
    else:
        s_k = int(rng.integers(1, 400))
        s_q = int(rng.choice([s_k, int(rng.integers(1, 400))]))
        shape = dict(batch=int(rng.integers(1, 3)), s_q=s_q, s_k=s_k)
    return dict(d=d, hkv=hkv, hq=hkv * group, varlen=varlen, causal=causal, window=window, int8=int8,
                epilogue=epilogue, **shape)


def _ids(n, prefix):
    return [f"{prefix}{i}" for i in range(n)]


@pytest.mark.parametrize("i", range(N_PREFILL), ids=_ids(N_PREFILL, "prefill"))
def test_prefill_sweep(i):
    from flashattention_attention_b200 import fa
    c = prefill_case(i)
    kw = dict(hq=c["hq"], hkv=c["hkv"], causal=c["causal"], window=c["window"], epilogue=c["epilogue"])
    if c["varlen"]:
        w = inputs.varlen_prefill("sweep", lengths=c["lengths"], hq=c["hq"], hkv=c["hkv"], d=c["d"],
                                  dtype=torch.bfloat16, causal=c["causal"], window=c["window"], seed=i)
        cu = inputs.cu_from_lengths(c["lengths"])
        gpu_kw = dict(cu_seqlens_q=cu.cuda(), max_seqlen_q=max(c["lengths"]))
        ref_kw = dict(cu_seqlens_q=cu.numpy())
    else:
        w = inputs.dense_prefill("sweep", batch=c["batch"], hq=c["hq"], hkv=c["hkv"], s_q=c["s_q"], s_k=c["s_k"],
                                 d=c["d"], dtype=torch.bfloat16, causal=c["causal"], window=c["window"], seed=i)
        gpu_kw, ref_kw = {}, {}
    k, v = w.k, w.v
    if c["int8"]:
        kc, ks = fa.compress_kv(k.cuda())
        vc, vs = fa.compress_kv(v.cuda())
        rk, rks = oracle.compress_kv(k)
        rv, rvs = oracle.compress_kv(v)
        assert np.array_equal(kc.cpu().numpy(), rk) and np.array_equal(vc.cpu().numpy(), rv)
        assert np.array_equal(ks.cpu().numpy().view(np.uint32), rks.view(np.uint32))
        assert np.array_equal(vs.cpu().numpy().view(np.uint32), rvs.view(np.uint32))
        got = fa.attention_fwd(w.q.cuda(), kc, vc, k_scales=ks, v_scales=vs, **kw, **gpu_kw)
        k_ref, v_ref = oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs)
    else:
        got = fa.attention_fwd(w.q.cuda(), k.cuda(), v.cuda(), **kw, **gpu_kw)
        k_ref, v_ref = k, v
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    ref = oracle.attention(w.q, k_ref, v_ref, **kw, **ref_kw)
    assert_close_bf16(got.float().cpu().numpy(), ref, what=str(c))


def decode_case(i):
    rng = np.random.default_rng(2000 + i)
    d = int(rng.choice([32, 64, 96, 128, 256]))
    hkv = int(rng.choice([1, 2, 4]))
    group = int(rng.choice([1, 2, 4, 8, 12, 16]))
    cap = 32 * int(rng.integers(1, 24))
    lengths = [int(x) for x in rng.integers(0, cap + 1, int(rng.integers(1, 6)))]
    window = int(rng.choice([0, 0, 50, 300]))
    int8 = bool(rng.integers(2))
    epilogue = [("mul", 2.0), ("add", -0.25)] if rng.integers(2) else []
    return dict(d=d, hkv=hkv, hq=hkv * group, cap=cap, lengths=lengths, window=window, int8=int8,
                epilogue=epilogue)


@pytest.mark.parametrize("i", range(N_DECODE), ids=_ids(N_DECODE, "decode"))
def test_decode_sweep(i):
    from flashattention_attention_b200 import fa
    c = decode_case(i)
    w = inputs.decode_cache("sweep", lengths=c["lengths"], hq=c["hq"], hkv=c["hkv"], d=c["d"], capacity=c["cap"],
                            seed=i, kv_int8=c["int8"])
    lens = torch.tensor(c["lengths"], dtype=torch.int32, device="cuda")
    q = w.q.reshape(-1, c["d"]).cuda()
    kw = dict(hq=c["hq"], hkv=c["hkv"], window=c["window"], epilogue=c["epilogue"])
    if c["int8"]:
        kc, ks = fa.compress_kv(w.k.cuda())
        vc, vs = fa.compress_kv(w.v.cuda())
        got = fa.attention_decode(q, kc, vc, lens, k_scales=ks, v_scales=vs, **kw)
        rk, rks = oracle.compress_kv(w.k)
        rv, rvs = oracle.compress_kv(w.v)
        k_ref, v_ref = oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs)
    else:
        got = fa.attention_decode(q, w.k.cuda(), w.v.cuda(), lens, **kw)
        k_ref, v_ref = w.k, w.v
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    ref = oracle.decode(w.q, k_ref, v_ref, np.array(c["lengths"]), **kw)
    assert_close_bf16(got.float().cpu().numpy().reshape(ref.shape), ref, what=str(c))
