"""GPU parity of fa_kv_append: a one-token cache write at a device-side slot
(FlashRT QKV Cache RoPE, Kernels: the slot is read from a device-side int32
position, so a captured decode graph can reuse it), quantised on the way in with the
int8 scheme of fkl_python PR #6, Summary.  The caches after the call must
equal the oracle's plain definition bit for bit, and a captured CUDA graph
of append + decode steps must match the oracle step by step."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16

pytestmark = pytest.mark.gpu


def _fa():
    from flashattention_attention_b200 import fa
    return fa


def _caches(rng, B, hkv, cap, d, int8):
    if int8:
        kc = torch.from_numpy(rng.integers(-127, 128, (B * hkv, cap, d)).astype(np.int8))
        vc = torch.from_numpy(rng.integers(-127, 128, (B * hkv, cap, d)).astype(np.int8))
        ks = torch.from_numpy(rng.random((B * hkv, cap)).astype(np.float32))
        vs = torch.from_numpy(rng.random((B * hkv, cap)).astype(np.float32))
        return kc, vc, ks, vs
    kc = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    vc = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    return kc, vc, None, None


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [64, 128, 48, 256])
def test_append_int8_bit_exact(x_dtype, d):
    fa = _fa()
    rng = np.random.default_rng(d * 10 + (x_dtype == torch.float32))
    B, hkv, cap = 5, 3, 40
    kc, vc, ks, vs = _caches(rng, B, hkv, cap, d, True)
    kn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32) * 3).to(x_dtype)
    vn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).to(x_dtype)
    pos = torch.tensor([0, cap - 1, 17, 3, 17], dtype=torch.int32)
    lens = torch.zeros(B, dtype=torch.int32)
    g = [t.cuda() for t in (kc, vc, ks, vs, kn, vn, pos, lens)]
    fa.kv_append(g[4], g[5], g[0], g[1], g[6], hkv=hkv, k_scales=g[2], v_scales=g[3], cache_seqlens=g[7])
    assert fa.check_device_error() == fa.FA_OK
    rk, rks, rl = oracle.kv_append(kc, ks, kn, pos, hkv, seqlens=lens)
    rv, rvs, _ = oracle.kv_append(vc, vs, vn, pos, hkv)
    assert np.array_equal(g[0].cpu().numpy(), rk) and np.array_equal(g[1].cpu().numpy(), rv)
    assert np.array_equal(g[2].cpu().numpy().view(np.uint32), rks.view(np.uint32))
    assert np.array_equal(g[3].cpu().numpy().view(np.uint32), rvs.view(np.uint32))
    assert np.array_equal(g[7].cpu().numpy(), rl)
    # the appended rows are exactly what fa_compress_kv makes of the new rows
    codes, scales = fa.compress_kv(g[4])
    ip = pos.long()
    rows = torch.arange(B * hkv) // hkv
    assert torch.equal(g[0][torch.arange(B * hkv), ip[rows].cuda()], codes)
    assert torch.equal(g[2][torch.arange(B * hkv), ip[rows].cuda()], scales)


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float32])
def test_append_bf16_cache(x_dtype):
    fa = _fa()
    rng = np.random.default_rng(7)
    B, hkv, cap, d = 3, 2, 33 * 2, 128
    kc, vc, _, _ = _caches(rng, B, hkv, cap, d, False)
    kn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).to(x_dtype)
    vn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).to(x_dtype)
    pos = torch.tensor([5, 0, cap - 1], dtype=torch.int32)
    g = [t.cuda() for t in (kc, vc, kn, vn, pos)]
    fa.kv_append(g[2], g[3], g[0], g[1], g[4], hkv=hkv)
    assert fa.check_device_error() == fa.FA_OK
    # bf16 storage of the new row: exact for bf16, round to nearest even for fp32
    rk, _, _ = oracle.kv_append(kc.float(), None, kn.bfloat16().float(), pos, hkv)
    rv, _, _ = oracle.kv_append(vc.float(), None, vn.bfloat16().float(), pos, hkv)
    assert np.array_equal(g[0].float().cpu().numpy(), rk) and np.array_equal(g[1].float().cpu().numpy(), rv)


def test_out_of_range_slot_is_skipped_and_reported():
    fa = _fa()
    rng = np.random.default_rng(9)
    B, hkv, cap, d = 3, 2, 16, 64
    kc, vc, ks, vs = _caches(rng, B, hkv, cap, d, True)
    kn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).bfloat16()
    pos = torch.tensor([-1, cap, 4], dtype=torch.int32)
    lens = torch.full((B,), 9, dtype=torch.int32)
    g = [t.cuda() for t in (kc, vc, ks, vs, kn, pos, lens)]
    fa.kv_append(g[4], g[4], g[0], g[1], g[5], hkv=hkv, k_scales=g[2], v_scales=g[3], cache_seqlens=g[6])
    assert fa.check_device_error() == fa.FA_ERR_INVALID
    assert fa.check_device_error() == fa.FA_OK  # the status word was cleared
    rk, rks, rl = oracle.kv_append(kc, ks, kn, pos, hkv, seqlens=lens)
    assert np.array_equal(g[0].cpu().numpy(), rk)
    assert np.array_equal(g[2].cpu().numpy().view(np.uint32), rks.view(np.uint32))
    assert list(g[6].cpu().numpy()) == [9, 9, 5] == list(rl)


def test_graph_of_append_and_decode_steps():
    """One captured CUDA graph: append the step's K/V at cur_pos, decode over
    cache_seqlens = cur_pos + 1, advance cur_pos.  Replayed for several steps
    with new rows and queries copied in between, every step's output matches
    the oracle (appended cache, then decode) within the bf16 gate."""
    fa = _fa()
    rng = np.random.default_rng(31)
    B, hq, hkv, d, cap, steps = 4, 8, 2, 128, 1024, 5
    lens0 = rng.integers(100, 900, B).astype(np.int32)
    k_full = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    v_full = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    kc, ks = fa.compress_kv(k_full.cuda())
    vc, vs = fa.compress_kv(v_full.cuda())
    cur = torch.from_numpy(lens0).cuda()
    lens = torch.from_numpy(lens0).cuda()
    kn = torch.empty((B * hkv, d), dtype=torch.bfloat16, device="cuda")
    vn = torch.empty_like(kn)
    q = torch.empty((B * hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(fa.decode_workspace_size(B, hq, cap, d), dtype=torch.uint8, device="cuda")

    def step():
        fa.kv_append(kn, vn, kc, vc, cur, hkv=hkv, k_scales=ks, v_scales=vs, cache_seqlens=lens)
        fa.attention_decode(q, kc, vc, lens, hq=hq, hkv=hkv, k_scales=ks, v_scales=vs, workspace=ws, out=out)
        cur.add_(1)

    # warm up on a side stream (status word, kernel attributes), then restore the state
    snap = [t.clone() for t in (kc, vc, ks, vs, cur, lens)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        kn.zero_(), vn.zero_(), q.zero_()
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for t, s in zip((kc, vc, ks, vs, cur, lens), snap):
        t.copy_(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    assert fa.check_device_error() == fa.FA_OK

    rk, rks = kc.cpu().numpy(), ks.cpu().numpy()
    rv, rvs = vc.cpu().numpy(), vs.cpu().numpy()
    pos = lens0.copy()
    for s in range(steps):
        kn_h = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).bfloat16()
        vn_h = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).bfloat16()
        q_h = torch.from_numpy(rng.standard_normal((B * hq, d)).astype(np.float32)).bfloat16()
        kn.copy_(kn_h), vn.copy_(vn_h), q.copy_(q_h)
        graph.replay()
        torch.cuda.synchronize()
        rk, rks, _ = oracle.kv_append(rk, rks, kn_h, pos, hkv)
        rv, rvs, _ = oracle.kv_append(rv, rvs, vn_h, pos, hkv)
        pos = pos + 1
        ref = oracle.decode(q_h.reshape(B * hq, 1, d), oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs),
                            list(pos), hq=hq, hkv=hkv)
        assert_close_bf16(out.float().cpu().numpy().reshape(ref.shape), ref, what=f"step {s}")
    assert np.array_equal(kc.cpu().numpy(), rk) and np.array_equal(ks.cpu().numpy().view(np.uint32),
                                                                      rks.view(np.uint32))
    assert list(cur.cpu().numpy()) == list(lens0 + steps) == list(lens.cpu().numpy() + 0)
    assert fa.check_device_error() == fa.FA_OK
    del graph
