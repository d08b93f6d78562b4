"""fa_attention_decode_noalloc: the decode entry point for callers that
cannot allocate device memory when they call (a plug-in inside a serving
runtime that owns every device byte through its own arena, or code that must
not trigger the implicit synchronisation of a cudaMalloc).  Its partials live
in a scratch array built into the library instead of a caller workspace.

Called through the C ABI and compared with fa_attention_decode on the same
inputs and with the fp64 oracle on the dequantised cache, within the bf16
tolerance the decode tests use, on two calls in a row with different
problems (the shared scratch keeps the previous call's contents, which must
not leak into the next result).  A cache length past the capacity is clamped
and reported through fa_check_device_error, which reads this entry point's
own status word.  This file is collected last so that a failure here never
hides another test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _prepare(seed, lengths, hq, hkv, cap):
    from flashattention_attention_b200 import fa
    w = inputs.decode_cache("t", lengths=lengths, hq=hq, hkv=hkv, d=128, capacity=cap, seed=seed)
    kc, ks = fa.compress_kv(w.k.cuda())
    vc, vs = fa.compress_kv(w.v.cuda())
    lens = torch.tensor(w.lengths, dtype=torch.int32, device="cuda")
    q = w.q.reshape(-1, 128).cuda()
    return w, q, kc, ks, vc, vs, lens


def _noalloc(q, kc, ks, vc, vs, lens, hq, hkv, split_keys=0, epilogue=()):
    from flashattention_attention_b200 import fa
    out = torch.full_like(q, float("nan"))
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = fa.decode_params(q, kc, vc, lens, out, dummy, hq=hq, hkv=hkv, k_scales=ks, v_scales=vs,
                         split_keys=split_keys, epilogue=epilogue)
    p.workspace = None          # this entry point takes no workspace
    p.workspace_bytes = 0
    st = fa.lib.fa_attention_decode_noalloc(ctypes.byref(p), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == fa.FA_OK, fa.lib.fa_status_string(st)
    torch.cuda.synchronize()
    return out


def _existing(q, kc, ks, vc, vs, lens, hq, hkv, split_keys=0, epilogue=()):
    from flashattention_attention_b200 import fa
    out = fa.attention_decode(q, kc, vc, lens, hq=hq, hkv=hkv, k_scales=ks, v_scales=vs,
                              split_keys=split_keys, epilogue=epilogue)
    torch.cuda.synchronize()
    return out


def _oracle(w, hq, hkv, epilogue=()):
    rk, rks = oracle.compress_kv(w.k)
    rv, rvs = oracle.compress_kv(w.v)
    return oracle.decode(w.q, oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs), w.lengths, hq=hq, hkv=hkv,
                         epilogue=epilogue)


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    from flashattention_attention_b200 import fa
    # first call: a larger problem that fills more of the scratch
    w1, *a1 = _prepare(21, [4000, 1500, 3000, 64], 32, 8, 4096)
    first = _noalloc(*a1, 32, 8)
    # second call: a smaller problem with an epilogue; stale records from the
    # first call sit in the scratch where this call's splits do not write
    w2, *a2 = _prepare(22, [700, 2049], 16, 2, 4096)
    epi = [("mul", 2.0), ("add", 0.5)]
    second = _noalloc(*a2, 16, 2, split_keys=256, epilogue=epi)
    assert fa.check_device_error() == fa.FA_OK

    ref1 = _existing(*a1, 32, 8)
    ref2 = _existing(*a2, 16, 2, split_keys=256, epilogue=epi)
    assert_close_bf16(first.float().cpu().numpy(), ref1.float().cpu().numpy(), what="first call")
    assert_close_bf16(second.float().cpu().numpy(), ref2.float().cpu().numpy(), what="second call")
    # the same split choice runs the same kernels: identical bits
    assert torch.equal(second, ref2)
    # and both agree with the oracle on the dequantised cache
    o1 = _oracle(w1, 32, 8)
    o2 = _oracle(w2, 16, 2, epilogue=epi)
    assert_close_bf16(first.float().cpu().numpy().reshape(o1.shape), o1, what="first call vs oracle")
    assert_close_bf16(second.float().cpu().numpy().reshape(o2.shape), o2, what="second call vs oracle")


def test_noalloc_reports_a_cache_length_past_the_capacity():
    """L_b > capacity is clamped to the capacity and reported: the result is
    attention over the whole cache, and fa_check_device_error (which reads
    this entry point's own status word) returns FA_ERR_INVALID once, then
    FA_OK again."""
    from flashattention_attention_b200 import fa
    cap = 1024
    w, q, kc, ks, vc, vs, lens = _prepare(23, [cap, 300], 8, 2, cap)
    assert fa.check_device_error() == fa.FA_OK
    over = torch.tensor([cap + 77, 300], dtype=torch.int32, device="cuda")
    got = _noalloc(q, kc, ks, vc, vs, over, 8, 2)
    assert fa.check_device_error() == fa.FA_ERR_INVALID
    assert fa.check_device_error() == fa.FA_OK  # read and cleared
    ref = _oracle(w, 8, 2)  # w.lengths = [cap, 300]: the clamped problem
    assert_close_bf16(got.float().cpu().numpy().reshape(ref.shape), ref, what="clamped length vs oracle")


def test_noalloc_rejects_problems_beyond_the_scratch():
    from flashattention_attention_b200 import fa
    # one record per (sequence, q-head) needs batch * hq * (128 + 2) * 4 bytes:
    # 2048 * 8 * 520 > 8 MiB leaves no room for the workers' records
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    p = fa.DecodeParams()
    p.q = p.k_cache = p.v_cache = p.out = q.data_ptr()
    p.k_scales = p.v_scales = p.cache_seqlens = q.data_ptr()
    p.kv_dtype, p.batch, p.hq, p.hkv, p.head_dim, p.capacity = fa.FA_I8, 2048, 8, 8, 128, 256
    p.softmax_scale = 0.088
    assert fa.lib.fa_attention_decode_noalloc(ctypes.byref(p), None) == fa.FA_ERR_WORKSPACE
    # the same with grouped heads: 256 sequences x 64 q-heads
    p.batch, p.hq, p.hkv, p.capacity = 256, 64, 8, 1024
    assert fa.lib.fa_attention_decode_noalloc(ctypes.byref(p), None) == fa.FA_ERR_WORKSPACE
