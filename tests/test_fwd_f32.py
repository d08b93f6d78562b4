"""GPU parity of the fp32 CUDA-core path of fa_attention_fwd against the fp64
oracle: max abs error <= 1e-5 (fkl_python PR #6, Verification: the dense
causal check at head size 64, the ragged 33/127 check at head size 32, and
the fused epilogue checked against the same ops applied on the host).
"""
import numpy as np
import pytest
import torch

import oracle
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu
TOL = 1e-5


def run_dense(q, k, v, hq, hkv, **kw):
    from flashattention_attention_b200 import fa
    out = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), hq=hq, hkv=hkv, **kw)
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    return out.cpu()


def check(got, ref, tol=TOL):
    err = np.abs(got.double().numpy() - ref).max()
    assert err <= tol, f"max abs {err:.3e}"
    return err


def test_tiny_fp32_causal_workload():
    w = inputs.tiny_fp32_causal()
    got = run_dense(w.q, w.k, w.v, w.hq, w.hkv, causal=True, scale=w.scale)
    ref = oracle.attention(w.q, w.k, w.v, hq=w.hq, hkv=w.hkv, causal=True, scale=w.scale)
    check(got, ref)


CASES = [
    # B, hq, hkv, s_q, s_k, d, causal, window
    (1, 2, 2, 64, 64, 64, True, 0),
    (2, 4, 2, 33, 127, 32, False, 0),     # ragged 33/127, non-causal
    (2, 4, 2, 33, 127, 32, True, 0),      # ragged 33/127, causal bottom-right
    (1, 8, 2, 100, 100, 128, True, 17),   # GQA + window
    (1, 3, 1, 50, 70, 96, False, 9),      # window without causal
    (2, 2, 2, 90, 40, 64, True, 0),       # s_q > s_k: 50 empty rows per head
    (1, 2, 1, 37, 37, 256, True, 0),
    (1, 1, 1, 1, 1, 64, True, 0),
    (1, 2, 2, 5, 300, 160, True, 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_dense_cases(case):
    B, hq, hkv, s_q, s_k, d, causal, window = case
    rng = np.random.default_rng(sum(case))
    q = inputs.normal(rng, (B * hq, s_q, d), torch.float32)
    k = inputs.normal(rng, (B * hkv, s_k, d), torch.float32)
    v = inputs.normal(rng, (B * hkv, s_k, d), torch.float32)
    got = run_dense(q, k, v, hq, hkv, causal=causal, window=window, scale=0.3)
    ref = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=causal, window=window, scale=0.3)
    check(got, ref)


def test_varlen_ragged_33_127():
    """The other reading of 'ragged 33/127': two packed sequences of lengths
    33 and 127 at d = 32, plus more lengths that straddle the 32-row tiles."""
    from flashattention_attention_b200 import fa
    lengths = [33, 127, 1, 64, 65]
    cu = inputs.cu_from_lengths(lengths)
    rng = np.random.default_rng(3)
    hq, hkv, d = 4, 2, 32
    tot = sum(lengths)
    q = inputs.normal(rng, (hq, tot, d), torch.float32)
    k = inputs.normal(rng, (hkv, tot, d), torch.float32)
    v = inputs.normal(rng, (hkv, tot, d), torch.float32)
    for causal, window in [(True, 0), (False, 0), (True, 20)]:
        out = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), hq=hq, hkv=hkv, causal=causal,
                               window=window, cu_seqlens_q=cu.cuda(), max_seqlen_q=max(lengths))
        ref = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=causal, window=window,
                               cu_seqlens_q=cu.numpy())
        check(out.cpu(), ref)


def test_epilogue_fused_equals_host_applied():
    """fkl_python PR #6, Verification: the fused epilogue equals the host-
    applied one with zero error.  In fp32 the fused Mul(2.0), Add(0.5) must equal the same ops
    applied on the host in fp32, bit for bit; changing the values or the
    list's length instantiates no new kernel."""
    from flashattention_attention_b200 import fa
    w = inputs.tiny_fp32_causal()
    base = run_dense(w.q, w.k, w.v, w.hq, w.hkv, causal=True, scale=w.scale).numpy()
    variants = fa.kernel_variants_used()
    longest = [("mul", 2.0), ("add", 0.5), ("mul", 0.25), ("add", -1.0), ("mul", 3.0), ("add", 0.125),
               ("mul", -0.5), ("add", 2.0)]  # the most ops a call takes (FA_MAX_EPILOGUE)
    for epi in ([("mul", 2.0), ("add", 0.5)], [("mul", -3.0), ("add", 1.25)], [("add", 0.5)],
                [("mul", 2.0), ("add", 0.5), ("mul", 0.25)], longest):
        fused = run_dense(w.q, w.k, w.v, w.hq, w.hkv, causal=True, scale=w.scale, epilogue=epi).numpy()
        host = base.copy()
        for op, val in epi:
            host = (host * np.float32(val)) if op == "mul" else (host + np.float32(val))
            host = host.astype(np.float32)
        assert np.array_equal(fused.view(np.uint32), host.view(np.uint32))
    assert fa.kernel_variants_used() == variants


def test_empty_band_rows_are_mean_of_v():
    """SKaiNET-transformers PR #419, Summary: empty band -> uniform softmax."""
    rng = np.random.default_rng(11)
    q = inputs.normal(rng, (2, 40, 64), torch.float32)
    k = inputs.normal(rng, (2, 10, 64), torch.float32)
    v = inputs.normal(rng, (2, 10, 64), torch.float32)
    got = run_dense(q, k, v, 2, 2, causal=True, epilogue=[("mul", 2.0)]).double().numpy()
    for h in range(2):
        np.testing.assert_allclose(got[h, :30], np.broadcast_to(2 * v[h].double().numpy().mean(0), (30, 64)),
                                   atol=1e-6)


I8_CASES = [
    # B, hq, hkv, s_q, s_k, d, causal, window
    (1, 2, 2, 64, 64, 64, True, 0),
    (1, 8, 2, 100, 100, 128, True, 17),   # GQA + window
    (2, 4, 2, 33, 127, 32, False, 0),     # ragged 33/127
    (2, 2, 1, 90, 40, 64, True, 0),       # s_q > s_k: empty rows get the mean of dequantised V
]


@pytest.mark.parametrize("case", I8_CASES, ids=lambda c: "-".join(map(str, c)))
def test_int8_kv_exact_vs_dequantised_oracle(case):
    """fkl_python PR #6, Verification: attention over the int8 cache agrees
    with an oracle run on the dequantised cache.  fp32 queries over an int8 cache made by fa_compress_kv from fp32
    K/V (codes and scales bit-exact with the oracle's quantiser) match the fp64
    oracle run on the dequantised cache within the fp32 gate."""
    from flashattention_attention_b200 import fa
    B, hq, hkv, s_q, s_k, d, causal, window = case
    rng = np.random.default_rng(50 + sum(case))
    q = inputs.normal(rng, (B * hq, s_q, d), torch.float32)
    k = inputs.normal(rng, (B * hkv, s_k, d), torch.float32)
    v = inputs.normal(rng, (B * hkv, s_k, d), torch.float32)
    kc, ks = fa.compress_kv(k.cuda())
    vc, vs = fa.compress_kv(v.cuda())
    rk, rks = oracle.compress_kv(k)
    rv, rvs = oracle.compress_kv(v)
    assert np.array_equal(kc.cpu().numpy(), rk) and np.array_equal(vc.cpu().numpy(), rv)
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), rks.view(np.uint32))
    assert np.array_equal(vs.cpu().numpy().view(np.uint32), rvs.view(np.uint32))
    out = fa.attention_fwd(q.cuda(), kc, vc, k_scales=ks, v_scales=vs, hq=hq, hkv=hkv, causal=causal,
                           window=window, scale=0.3, epilogue=[("mul", 2.0), ("add", -1.0)])
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    ref = oracle.attention(q, oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs), hq=hq, hkv=hkv,
                           causal=causal, window=window, scale=0.3, epilogue=[("mul", 2.0), ("add", -1.0)])
    # |Mul(2)| doubles the absolute error of the normalised output
    check(out.cpu(), ref, tol=2 * TOL)
