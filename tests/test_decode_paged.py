"""GPU parity of fa_attention_decode_paged: decode over a page pool through a
block table (SKaiNET-transformers PR #419, Summary: the kernel reads the
cached prefix where it lies rather than a per-token copy of it).  The pages
of a dense cache scattered over a pool in random order must give the dense
decode's output bit for bit (the page's tests compare the in-place view with
the copied one), and the oracle's within the bf16 gate."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16

pytestmark = pytest.mark.gpu


def _fa():
    from flashattention_attention_b200 import fa
    return fa


def paginate(dense, scales, lengths, hkv, page_size, extra, rng):
    """Scatter the pages of a dense [B*hkv, cap, d] cache over a shuffled pool
    [num_pages, hkv, page_size, d]; table entries of pages past a sequence's
    length stay -1 (never read)."""
    B = len(lengths)
    cap, d = dense.shape[1], dense.shape[2]
    max_pages = cap // page_size
    need = [max(1, -(-int(L) // page_size)) for L in lengths]
    num_pages = sum(need) + extra
    order = rng.permutation(num_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    pool = torch.zeros((num_pages, hkv, page_size, d), dtype=dense.dtype)
    spool = None if scales is None else torch.zeros((num_pages, hkv, page_size), dtype=torch.float32)
    k = 0
    for b in range(B):
        for lp in range(need[b]):
            pg = int(order[k])
            k += 1
            table[b, lp] = pg
            for g in range(hkv):
                pool[pg, g] = dense[b * hkv + g, lp * page_size:(lp + 1) * page_size]
                if scales is not None:
                    spool[pg, g] = scales[b * hkv + g, lp * page_size:(lp + 1) * page_size]
    return pool, spool, torch.from_numpy(table)


@pytest.mark.parametrize("int8", [True, False])
@pytest.mark.parametrize("d,page_size,window,hq,hkv", [(128, 64, 0, 16, 4), (128, 256, 0, 16, 4), (64, 32, 0, 16, 4),
                                                       (128, 64, 300, 16, 4), (128, 64, 0, 32, 2), (96, 64, 0, 16, 4),
                                                       (256, 128, 0, 8, 2)])
def test_paged_equals_dense(int8, d, page_size, window, hq, hkv):
    fa = _fa()
    rng = np.random.default_rng(d + page_size + window + int8 + hq)
    B, cap = 6, 1024
    lengths = [1000, 1, 0, 512, 1024, 333]
    k = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    q = torch.from_numpy(rng.standard_normal((B * hq, d)).astype(np.float32)).bfloat16().cuda()
    lens = torch.tensor(lengths, dtype=torch.int32).cuda()
    if int8:
        kc, ks = fa.compress_kv(k.cuda())
        vc, vs = fa.compress_kv(v.cuda())
        kc, ks, vc, vs = kc.cpu(), ks.cpu(), vc.cpu(), vs.cpu()
    else:
        kc, ks, vc, vs = k, None, v, None
    kp, ksp, table = paginate(kc, ks, lengths, hkv, page_size, 7, rng)
    # V in the same pages as K
    vp = torch.zeros_like(kp)
    vsp = None if vs is None else torch.zeros_like(ksp)
    for b in range(B):
        for lp in range(cap // page_size):
            pg = int(table[b, lp])
            if pg < 0:
                continue
            for g in range(hkv):
                vp[pg, g] = vc[b * hkv + g, lp * page_size:(lp + 1) * page_size]
                if vs is not None:
                    vsp[pg, g] = vs[b * hkv + g, lp * page_size:(lp + 1) * page_size]
    cuda = lambda t: None if t is None else t.cuda()
    dense = fa.attention_decode(q, cuda(kc), cuda(vc), lens, hq=hq, hkv=hkv, k_scales=cuda(ks),
                                v_scales=cuda(vs), window=window)
    paged = fa.attention_decode_paged(q, cuda(kp), cuda(vp), lens, cuda(table), hq=hq, hkv=hkv,
                                      k_scales=cuda(ksp), v_scales=cuda(vsp), window=window)
    assert fa.check_device_error() == fa.FA_OK
    assert torch.equal(dense, paged)
    kref = oracle.dequantize(kc, ks) if int8 else kc.float().numpy()
    vref = oracle.dequantize(vc, vs) if int8 else vc.float().numpy()
    ref = oracle.decode(q.cpu().reshape(B * hq, 1, d), kref, vref, lengths, hq=hq, hkv=hkv, window=window)
    assert_close_bf16(paged.float().cpu().numpy().reshape(ref.shape), ref)


def test_bad_page_id_is_reported_and_stays_in_the_pool():
    fa = _fa()
    rng = np.random.default_rng(3)
    B, hq, hkv, d, page_size, max_pages = 2, 8, 2, 128, 64, 4
    num_pages = 8
    kp = torch.from_numpy(rng.integers(-127, 128, (num_pages, hkv, page_size, d)).astype(np.int8)).cuda()
    ks = torch.from_numpy(rng.random((num_pages, hkv, page_size)).astype(np.float32)).cuda()
    table = torch.tensor([[0, 1, 2, 3], [4, 5, 99, -1]], dtype=torch.int32).cuda()  # 99: outside the pool
    lens = torch.tensor([256, 150], dtype=torch.int32).cuda()
    q = torch.from_numpy(rng.standard_normal((B * hq, d)).astype(np.float32)).bfloat16().cuda()
    out = fa.attention_decode_paged(q, kp, kp, lens, table, hq=hq, hkv=hkv, k_scales=ks, v_scales=ks)
    assert fa.check_device_error() == fa.FA_ERR_INVALID
    assert fa.check_device_error() == fa.FA_OK
    # sequence 0 only used valid pages: its output is the dense one
    dense_k = kp[:4].permute(1, 0, 2, 3).reshape(hkv, 4 * page_size, d).contiguous()
    dense_s = ks[:4].permute(1, 0, 2).reshape(hkv, 4 * page_size).contiguous()
    ref = fa.attention_decode(q[:hq].contiguous(), dense_k, dense_k, lens[:1].contiguous(), hq=hq, hkv=hkv,
                              k_scales=dense_s, v_scales=dense_s)
    assert torch.isfinite(out[:hq].float()).all()
    assert_close_bf16(out[:hq].float().cpu().numpy(), ref.float().cpu().numpy())


@pytest.mark.parametrize("int8", [True, False])
def test_paged_append_then_decode_equals_dense(int8):
    """A decode step on pages: append the new token into its page (through the
    table), then decode; the dense cache given the same append must agree bit
    for bit, and the pool rows outside the written slots stay as they were."""
    fa = _fa()
    rng = np.random.default_rng(40 + int8)
    B, hq, hkv, d, cap, page_size = 4, 16, 4, 128, 512, 64
    lengths = [300, 63, 64, 511]       # the new token lands at these slots
    k = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16()
    if int8:
        kc, ks = (t.cpu() for t in fa.compress_kv(k.cuda()))
        vc, vs = (t.cpu() for t in fa.compress_kv(v.cuda()))
    else:
        kc, ks, vc, vs = k, None, v, None
    kp, ksp, table = paginate(kc, ks, [L + 1 for L in lengths], hkv, page_size, 3, rng)
    vp = torch.zeros_like(kp)
    vsp = None if vs is None else torch.zeros_like(ksp)
    for b in range(B):
        for lp in range(cap // page_size):
            pg = int(table[b, lp])
            if pg >= 0:
                for g in range(hkv):
                    vp[pg, g] = vc[b * hkv + g, lp * page_size:(lp + 1) * page_size]
                    if vs is not None:
                        vsp[pg, g] = vs[b * hkv + g, lp * page_size:(lp + 1) * page_size]
    cuda = lambda t: None if t is None else t.cuda()
    kc, vc, ks, vs, kp, vp, ksp, vsp, table = map(cuda, (kc, vc, ks, vs, kp, vp, ksp, vsp, table))
    kp0 = kp.clone()
    kn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).bfloat16().cuda()
    vn = torch.from_numpy(rng.standard_normal((B * hkv, d)).astype(np.float32)).bfloat16().cuda()
    pos = torch.tensor(lengths, dtype=torch.int32).cuda()
    lens_d = torch.zeros(B, dtype=torch.int32).cuda()
    lens_p = torch.zeros(B, dtype=torch.int32).cuda()
    fa.kv_append(kn, vn, kc, vc, pos, hkv=hkv, k_scales=ks, v_scales=vs, cache_seqlens=lens_d)
    fa.kv_append_paged(kn, vn, kp, vp, pos, table, hkv=hkv, k_scales=ksp, v_scales=vsp, cache_seqlens=lens_p)
    assert torch.equal(lens_d, lens_p) and list(lens_p.cpu().numpy()) == [L + 1 for L in lengths]
    q = torch.from_numpy(rng.standard_normal((B * hq, d)).astype(np.float32)).bfloat16().cuda()
    dense = fa.attention_decode(q, kc, vc, lens_d, hq=hq, hkv=hkv, k_scales=ks, v_scales=vs)
    paged = fa.attention_decode_paged(q, kp, vp, lens_p, table, hq=hq, hkv=hkv, k_scales=ksp, v_scales=vsp)
    assert fa.check_device_error() == fa.FA_OK
    assert torch.equal(dense, paged)
    # exactly one row per (sequence, kv head) of the K pool changed
    changed = (kp != kp0).any(dim=-1).nonzero().cpu().numpy()
    tab = table.cpu().numpy()
    expect = {(int(tab[b, L // page_size]), g, L % page_size) for b, L in enumerate(lengths) for g in range(hkv)}
    assert {tuple(x) for x in changed} <= expect


def paginate_varlen(x, scales, lens, hkv, page_size, rng, extra=3):
    """Pages of a varlen [hkv, total, d] tensor (sequence b owns rows
    cu[b]..cu[b+1]-1 of every head plane) over a shuffled pool; returns the
    pool, its scale pool and the block table."""
    B = len(lens)
    need = [max(1, -(-int(L) // page_size)) for L in lens]
    max_pages = max(need) + 1
    num_pages = sum(need) + extra
    order = rng.permutation(num_pages)
    d = x.shape[-1]
    pool = torch.zeros((num_pages, hkv, page_size, d), dtype=x.dtype)
    spool = None if scales is None else torch.zeros((num_pages, hkv, page_size), dtype=torch.float32)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    cu = np.concatenate([[0], np.cumsum(lens)])
    k = 0
    for b in range(B):
        for lp in range(need[b]):
            pg = int(order[k])
            k += 1
            table[b, lp] = pg
            a, e = cu[b] + lp * page_size, min(cu[b] + (lp + 1) * page_size, cu[b + 1])
            if e > a:
                pool[pg, :, :e - a] = x[:, a:e]
                if scales is not None:
                    spool[pg, :, :e - a] = scales[:, a:e]
    return pool, spool, torch.from_numpy(table)


@pytest.mark.parametrize("int8", [False, True])
@pytest.mark.parametrize("d,page_size,window", [(128, 128, 0), (128, 256, 0), (64, 128, 200), (96, 128, 0),
                                                (32, 256, 100), (256, 128, 0), (160, 256, 300)])
def test_paged_prefill_equals_varlen(int8, d, page_size, window):
    """Chunked prefill over a paged cache: each sequence's new queries (fewer
    than its keys, bottom-right causal) attend to its whole prefix read from
    shuffled pages; bit-identical to the contiguous varlen prefill, and the
    oracle's within the bf16 gate."""
    fa = _fa()
    rng = np.random.default_rng(50 + d + page_size + window + int8)
    hq, hkv = 8, 2
    k_lens = [700, 129, 1024, 40]
    q_lens = [64, 129, 300, 40]
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(k_lens)]), dtype=torch.int32)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(q_lens)]), dtype=torch.int32)
    tk, tq = int(cu_k[-1]), int(cu_q[-1])
    k = torch.from_numpy(rng.standard_normal((hkv, tk, d)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((hkv, tk, d)).astype(np.float32)).bfloat16()
    q = torch.from_numpy(rng.standard_normal((hq, tq, d)).astype(np.float32)).bfloat16().cuda()
    if int8:
        kc, ks = (t.cpu() for t in fa.compress_kv(k.cuda()))
        vc, vs = (t.cpu() for t in fa.compress_kv(v.cuda()))
    else:
        kc, ks, vc, vs = k, None, v, None
    kp, ksp, table = paginate_varlen(kc, ks, k_lens, hkv, page_size, rng)
    vp, vsp, _ = paginate_varlen(vc, vs, k_lens, hkv, page_size, np.random.default_rng(0))
    # V in K's pages
    vp = torch.zeros_like(kp)
    vsp = None if vs is None else torch.zeros_like(ksp)
    cu = np.concatenate([[0], np.cumsum(k_lens)])
    for b in range(len(k_lens)):
        for lp in range(table.shape[1]):
            pg = int(table[b, lp])
            if pg < 0:
                continue
            a, e = cu[b] + lp * page_size, min(cu[b] + (lp + 1) * page_size, cu[b + 1])
            if e > a:
                vp[pg, :, :e - a] = vc[:, a:e]
                if vs is not None:
                    vsp[pg, :, :e - a] = vs[:, a:e]
    cuda = lambda t: None if t is None else t.cuda()
    epi = [("mul", 2.0), ("add", 0.5)]
    ref_gpu = fa.attention_fwd(q, cuda(kc), cuda(vc), hq=hq, hkv=hkv, causal=True, window=window, epilogue=epi,
                               k_scales=cuda(ks), v_scales=cuda(vs), cu_seqlens_q=cu_q.cuda(),
                               cu_seqlens_k=cu_k.cuda(), max_seqlen_q=max(q_lens), max_seqlen_k=max(k_lens))
    paged = fa.attention_fwd_paged(q, cuda(kp), cuda(vp), cu_k.cuda(), cuda(table), hq=hq, hkv=hkv, causal=True,
                                   window=window, epilogue=epi, k_scales=cuda(ksp), v_scales=cuda(vsp),
                                   cu_seqlens_q=cu_q.cuda(), max_seqlen_q=max(q_lens))
    assert fa.check_device_error() == fa.FA_OK
    assert torch.equal(ref_gpu, paged)
    kref = oracle.dequantize(kc, ks) if int8 else kc.float().numpy()
    vref = oracle.dequantize(vc, vs) if int8 else vc.float().numpy()
    ref = oracle.attention(q.cpu(), kref, vref, hq=hq, hkv=hkv, causal=True, window=window, epilogue=epi,
                           cu_seqlens_q=cu_q.numpy(), cu_seqlens_k=cu_k.numpy())
    assert_close_bf16(paged.float().cpu().numpy(), ref)


def test_paged_prefill_dense_queries_and_empty_band():
    """Dense queries [B*hq, s_q, d] over paged keys, with one sequence holding
    fewer keys than queries: its first s_q - s_k rows see no key and get the
    mean of V (the empty-band rule), read through the pages."""
    fa = _fa()
    rng = np.random.default_rng(61)
    B, hq, hkv, d, s_q, page_size = 3, 4, 2, 128, 200, 128
    k_lens = [300, 150, 130]  # sequences 1, 2: the first 50 and 70 query rows see no key
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(k_lens)]), dtype=torch.int32)
    tk = int(cu_k[-1])
    k = torch.from_numpy(rng.standard_normal((hkv, tk, d)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((hkv, tk, d)).astype(np.float32)).bfloat16()
    q = torch.from_numpy(rng.standard_normal((B * hq, s_q, d)).astype(np.float32)).bfloat16().cuda()
    kp, _, table = paginate_varlen(k, None, k_lens, hkv, page_size, rng)
    vp = torch.zeros_like(kp)
    cu = cu_k.numpy()
    for b in range(B):
        for lp in range(table.shape[1]):
            pg = int(table[b, lp])
            if pg < 0:
                continue
            a, e = cu[b] + lp * page_size, min(cu[b] + (lp + 1) * page_size, cu[b + 1])
            if e > a:
                vp[pg, :, :e - a] = v[:, a:e]
    out = fa.attention_fwd_paged(q, kp.cuda(), vp.cuda(), cu_k.cuda(), table.cuda(), hq=hq, hkv=hkv, causal=True)
    assert fa.check_device_error() == fa.FA_OK
    # oracle: per sequence, dense q against that sequence's keys
    qh = q.cpu().reshape(B, hq, s_q, d)
    for b in range(B):
        kb = k[:, cu[b]:cu[b + 1]].float().numpy()
        vb = v[:, cu[b]:cu[b + 1]].float().numpy()
        ref = oracle.attention(qh[b].float().numpy(), kb, vb, hq=hq, hkv=hkv, causal=True)
        got = out.cpu().reshape(B, hq, s_q, d)[b].float().numpy()
        assert_close_bf16(got, ref, what=f"sequence {b}")
