"""GPU parity of the partial-result prefill (fa_attention_fwd_lse), the merge
(fa_attention_merge), the prefill that merges into an accumulator in its
epilogue (fa_attention_fwd_acc) and the ring step sequence they make (kernbench2 commit
message, ADR-0060 (long context): K/V rotated around the ring, an
online-softmax merge at every ring step).  The
multi-rank schedule itself is covered on CPU by test_multiprocess_cpu.py."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16, assert_close_bf16_planes

pytestmark = pytest.mark.gpu


def _fa():
    from flashattention_attention_b200 import fa
    return fa


def _bf(rng, *shape):
    return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).bfloat16()


@pytest.mark.parametrize("d,causal,s_q,s_k", [(128, True, 300, 300), (128, False, 130, 517), (64, True, 200, 90),
                                              (128, True, 64, 700)])
def test_fwd_lse_matches_oracle(d, causal, s_q, s_k):
    fa = _fa()
    rng = np.random.default_rng(d + s_q + s_k)
    hq, hkv, B = 4, 2, 2
    q, k, v = _bf(rng, B * hq, s_q, d), _bf(rng, B * hkv, s_k, d), _bf(rng, B * hkv, s_k, d)
    out, lse = fa.attention_fwd_lse(q.cuda(), k.cuda(), v.cuda(), hq=hq, hkv=hkv, causal=causal)
    assert fa.check_device_error() == fa.FA_OK
    ro, rl = oracle.attention_lse(q, k, v, hq=hq, hkv=hkv, causal=causal)
    got_l = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(got_l), np.isneginf(rl))   # rows without keys (s_q > s_k, causal)
    fin = np.isfinite(rl)
    assert np.abs(got_l[fin] - rl[fin]).max() < 2e-3
    assert_close_bf16(out.float().cpu().numpy(), ro)
    assert not out.float()[torch.from_numpy(~fin)].any()


@pytest.mark.parametrize("d,part_dtype", [(128, torch.bfloat16), (96, torch.float32), (256, torch.bfloat16),
                                          (32, torch.float32)])
def test_merge_matches_oracle_and_writes_the_final_output(d, part_dtype):
    fa = _fa()
    rng = np.random.default_rng(80 + d)
    rows = 1001
    acc = torch.from_numpy(rng.standard_normal((rows, d)).astype(np.float32))
    lacc = torch.from_numpy(rng.standard_normal(rows).astype(np.float32))
    part = torch.from_numpy(rng.standard_normal((rows, d)).astype(np.float32)).to(part_dtype)
    lpart = torch.from_numpy(rng.standard_normal(rows).astype(np.float32))
    lacc[:10] = float("-inf")   # empty accumulator rows take the partial
    lpart[5:15] = float("-inf")  # empty partial rows leave the accumulator (rows 5-9: both empty)
    acc[:10] = 0
    g_acc, g_lacc = acc.cuda(), lacc.cuda()
    out = torch.empty((rows, d), dtype=part_dtype, device="cuda")
    fa.attention_merge(g_acc, g_lacc, part.cuda(), lpart.cuda(), out=out, epilogue=[("mul", 2.0)])
    assert fa.check_device_error() == fa.FA_OK
    ro, rl = oracle.merge(acc.double().numpy(), lacc.double().numpy(), part.double().numpy(), lpart.double().numpy())
    assert np.allclose(g_acc.cpu().numpy(), ro, rtol=1e-5, atol=1e-5)
    gl = g_lacc.cpu().numpy()
    assert np.array_equal(np.isneginf(gl), np.isneginf(rl)) and np.allclose(gl[np.isfinite(rl)], rl[np.isfinite(rl)],
                                                                            rtol=1e-5, atol=1e-5)
    # out is the merged fp32 row (the one stored in the accumulator) after the
    # epilogue, rounded once to the output type
    assert torch.equal(out, (2.0 * g_acc).to(part_dtype))
    # finalise only (no partial): out = epilogue(accumulator), accumulator untouched
    before = g_acc.clone()
    fa.attention_merge(g_acc, g_lacc, out=out, epilogue=[("add", 1.0)])
    assert torch.equal(g_acc, before)
    assert torch.equal(out, (before + 1.0).to(part_dtype))


def _epi(y, epilogue):
    for op, val in epilogue:
        y = y * val if op == "mul" else y + val
    return y


@pytest.mark.parametrize("int8", [False, True])
def test_fwd_acc_over_ragged_key_chunks_matches_oracle(int8):
    """Keys split into ragged chunks (lengths not multiples of the 128-key
    tile), merged chunk by chunk in the prefill's epilogue: the final output
    equals the oracle over all keys, and the intermediate accumulator equals
    the oracle's merge of the chunks' partial results.  The accumulator is
    NaN before the first step, which must not read it."""
    fa = _fa()
    rng = np.random.default_rng(11 + int8)
    B, hq, hkv, d, s_q = 2, 4, 2, 128, 333
    chunks = [300, 77, 517]
    q = _bf(rng, B * hq, s_q, d)
    k, v = _bf(rng, B * hkv, sum(chunks), d), _bf(rng, B * hkv, sum(chunks), d)
    gq = q.cuda()
    if int8:
        kc, ks = fa.compress_kv(k.cuda())
        vc, vs = fa.compress_kv(v.cuda())
        k_ref, v_ref = oracle.dequantize(kc.cpu(), ks.cpu()), oracle.dequantize(vc.cpu(), vs.cpu())
    else:
        kc, vc, ks, vs = k.cuda(), v.cuda(), None, None
        k_ref, v_ref = k, v
    acc_o = torch.full((B * hq, s_q, d), float("nan"), device="cuda")
    acc_l = torch.full((B * hq, s_q), float("nan"), device="cuda")
    epi = [("mul", 2.0), ("add", -0.25)]
    pos = np.cumsum([0] + chunks)
    ro = rl = None
    for c in range(len(chunks)):
        sl = slice(int(pos[c]), int(pos[c + 1]))
        part = lambda t: t[:, sl].contiguous()
        last = c == len(chunks) - 1
        out = fa.attention_fwd_acc(gq, part(kc), part(vc), acc_o, acc_l, hq=hq, hkv=hkv, first=c == 0, last=last,
                                   epilogue=epi, k_scales=None if ks is None else part(ks),
                                   v_scales=None if vs is None else part(vs))
        assert fa.check_device_error() == fa.FA_OK
        po, pl = oracle.attention_lse(q, k_ref[:, sl], v_ref[:, sl], hq=hq, hkv=hkv)
        ro, rl = (po, pl) if ro is None else oracle.merge(ro, rl, po, pl)
        if not last:
            assert out is None
            assert_close_bf16(acc_o.cpu().numpy(), ro, what=f"accumulator after chunk {c}")
            # int8: K enters the tensor core as c*s rounded to bf16, ~2^-9 per score
            assert np.abs(acc_l.cpu().numpy() - rl).max() < (1e-2 if int8 else 2e-3)
    ref = oracle.attention(q, k_ref, v_ref, hq=hq, hkv=hkv, epilogue=epi)
    assert_close_bf16(out.float().cpu().numpy(), ref)
    assert np.allclose(_epi(ro, epi), ref, atol=1e-9)  # the oracle's merge itself


def test_fwd_acc_rows_without_keys_merge_nothing():
    """Causal with s_q > s_k leaves rows i < s_q - s_k without keys: a middle
    step leaves their accumulator rows bit for bit, a first step makes them
    empty (o = 0, lse = -inf), the last step writes the epilogue of the
    accumulator (of 0 when it is also the first)."""
    fa = _fa()
    rng = np.random.default_rng(12)
    B, hq, hkv, d, s_q, s_k = 1, 4, 2, 128, 300, 90
    q, k, v = _bf(rng, B * hq, s_q, d).cuda(), _bf(rng, B * hkv, s_k, d).cuda(), _bf(rng, B * hkv, s_k, d).cuda()
    n_empty = s_q - s_k
    acc_o0 = torch.from_numpy(rng.standard_normal((B * hq, s_q, d)).astype(np.float32)).cuda()
    acc_l0 = torch.from_numpy(rng.standard_normal((B * hq, s_q)).astype(np.float32)).cuda()
    epi = [("add", 1.5)]
    # middle step
    a_o, a_l = acc_o0.clone(), acc_l0.clone()
    fa.attention_fwd_acc(q, k, v, a_o, a_l, hq=hq, hkv=hkv, causal=True)
    assert torch.equal(a_o[:, :n_empty], acc_o0[:, :n_empty]) and torch.equal(a_l[:, :n_empty], acc_l0[:, :n_empty])
    po, pl = oracle.attention_lse(q.cpu(), k.cpu(), v.cpu(), hq=hq, hkv=hkv, causal=True)
    ro, rl = oracle.merge(acc_o0.cpu().double().numpy(), acc_l0.cpu().double().numpy(), po, pl)
    assert_close_bf16(a_o.cpu().numpy(), ro)
    # first step
    a_o, a_l = acc_o0.clone(), acc_l0.clone()
    fa.attention_fwd_acc(q, k, v, a_o, a_l, hq=hq, hkv=hkv, causal=True, first=True)
    assert not a_o[:, :n_empty].any() and bool(torch.isneginf(a_l[:, :n_empty]).all())
    assert_close_bf16(a_o[:, n_empty:].cpu().numpy(), po[:, n_empty:])
    # last step, then first-and-last
    a_o, a_l = acc_o0.clone(), acc_l0.clone()
    out = fa.attention_fwd_acc(q, k, v, a_o, a_l, hq=hq, hkv=hkv, causal=True, last=True, epilogue=epi)
    assert torch.equal(a_o, acc_o0) and torch.equal(a_l, acc_l0)  # the last step leaves the accumulator
    assert torch.equal(out[:, :n_empty], (acc_o0[:, :n_empty] + 1.5).bfloat16())
    assert_close_bf16(out.float().cpu().numpy(), _epi(ro, epi))
    out = fa.attention_fwd_acc(q, k, v, a_o, a_l, hq=hq, hkv=hkv, causal=True, first=True, last=True, epilogue=epi)
    assert bool((out[:, :n_empty] == 1.5).all())
    assert_close_bf16(out[:, n_empty:].float().cpu().numpy(), _epi(po[:, n_empty:], epi))
    assert fa.check_device_error() == fa.FA_OK


def test_rows_with_no_keys_at_all_are_written():
    """s_k = 0 without the causal mask: every row has no key; the plain
    prefill writes zeros (then the epilogue), on both the tensor-core and the
    fp32 path, and the partial result is empty."""
    fa = _fa()
    rng = np.random.default_rng(13)
    hq, hkv, d = 4, 2, 128
    for dt in (torch.bfloat16, torch.float32):
        q = torch.from_numpy(rng.standard_normal((2 * hq, 70, d)).astype(np.float32)).to(dt).cuda()
        kv = torch.zeros((2 * hkv, 8, d), dtype=dt, device="cuda")
        k0 = kv[:, :0]
        out = torch.full_like(q, float("nan"))
        fa.attention_fwd(q, k0, k0, hq=hq, hkv=hkv, epilogue=[("add", 0.75)], out=out)
        assert bool((out == 0.75).all()), dt
    q = q.bfloat16()
    o, lse = fa.attention_fwd_lse(q, k0.bfloat16(), k0.bfloat16(), hq=hq, hkv=hkv)
    assert not o.any() and bool(torch.isneginf(lse).all())
    assert fa.check_device_error() == fa.FA_OK


@pytest.mark.parametrize("n_blocks", [1, 3, 4])
def test_ring_steps_on_one_gpu_equal_full_attention(n_blocks):
    """The sequence of kernel calls a ring of n ranks makes, run in one
    process: query block r attends to the K/V blocks 0..r (the diagonal one
    causal, earlier ones unmasked).  Both the partial-result form
    (fa_attention_fwd_lse, then fa_attention_merge) and the fused one
    (ring.attend_blocks, fa_attention_fwd_acc) equal the full causal prefill
    within the bf16 gate."""
    from flashattention_attention_b200 import ring
    fa = _fa()
    rng = np.random.default_rng(90 + n_blocks)
    B, hq, hkv, d, blk = 2, 8, 2, 128, 256
    S = blk * n_blocks
    q, k, v = _bf(rng, B * hq, S, d).cuda(), _bf(rng, B * hkv, S, d).cuda(), _bf(rng, B * hkv, S, d).cuda()
    epi = [("mul", 0.5), ("add", 1.0)]
    full = fa.attention_fwd(q, k, v, hq=hq, hkv=hkv, causal=True, epilogue=epi)
    ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), hq=hq, hkv=hkv, causal=True, epilogue=epi)
    sl = lambda t, b: t[:, b * blk:(b + 1) * blk].contiguous()
    outs, fused = [], []
    for r in range(n_blocks):
        acc_o = torch.zeros((B * hq, blk, d), dtype=torch.float32, device="cuda")
        acc_l = torch.full((B * hq, blk), float("-inf"), dtype=torch.float32, device="cuda")
        for b in range(r, -1, -1):  # the order a ring delivers the blocks in
            o, l = fa.attention_fwd_lse(sl(q, r), sl(k, b), sl(v, b), hq=hq, hkv=hkv, causal=(b == r))
            fa.attention_merge(acc_o, acc_l, o, l)
        out = torch.empty((B * hq, blk, d), dtype=torch.bfloat16, device="cuda")
        fa.attention_merge(acc_o, acc_l, out=out, epilogue=epi)
        outs.append(out)
        # the fused form, every block offered (later ones skipped), in ring order
        blocks = [((r - s) % n_blocks, sl(k, (r - s) % n_blocks), sl(v, (r - s) % n_blocks)) for s in range(n_blocks)]
        fused.append(ring.attend_blocks(sl(q, r), blocks, rank=r, n_blocks=n_blocks, hq=hq, hkv=hkv, causal=True,
                                        epilogue=epi))
    assert fa.check_device_error() == fa.FA_OK
    for got in (torch.cat(outs, dim=1), torch.cat(fused, dim=1)):
        assert_close_bf16(got.float().cpu().numpy(), ref)
        assert_close_bf16(got.float().cpu().numpy(), full.float().cpu().numpy())
    # the driver itself with a one-process ring
    one = ring.ring_attention_fwd(q, k, v, hq=hq, hkv=hkv, causal=True, epilogue=epi)
    assert torch.equal(one, full)  # one block, first and last: the plain kernel's arithmetic


def test_full_size_ring_last_rank():
    """The bench's ring line at full size: the last rank of a 4-way causal
    ring (B=4, Hq=32, Hkv=8, block 4096, d=128: queries at positions
    12288..16383 over 16384 keys), run through ring.attend_blocks exactly as
    timed; every row of two whole KV groups (the first of sequence 0 and the
    last of sequence 3, 8 query heads) checked against the oracle."""
    from flashattention_attention_b200 import inputs, ring
    fa = _fa()
    w = inputs.ring_cp_last_rank()
    R, blk = w.seqlen_k // w.seqlen_q, w.seqlen_q
    q = w.q.cuda()
    kb = [w.k[:, b * blk:(b + 1) * blk].contiguous().cuda() for b in range(R)]
    vb = [w.v[:, b * blk:(b + 1) * blk].contiguous().cuda() for b in range(R)]
    blocks = [((R - 1 - s) % R, kb[(R - 1 - s) % R], vb[(R - 1 - s) % R]) for s in range(R)]
    got = ring.attend_blocks(q, blocks, rank=R - 1, n_blocks=R, hq=w.hq, hkv=w.hkv, causal=True).cpu()
    assert fa.check_device_error() == fa.FA_OK
    assert torch.isfinite(got.float()).all()
    G = w.hq // w.hkv
    for b, g in ((0, 0), (w.batch - 1, w.hkv - 1)):
        planes = [b * w.hq + g * G + j for j in range(G)]
        ref = oracle.attention(w.q[planes], w.k[[b * w.hkv + g]], w.v[[b * w.hkv + g]], hq=G, hkv=1, causal=True)
        assert_close_bf16_planes(got[planes], ref, what=f"full-size ring, sequence {b} KV group {g}")


def test_fwd_acc_varlen_keys_in_two_sets():
    """Varlen queries whose keys arrive as two packed sets with their own
    per-sequence counts (cu_seqlens_k), merged in the epilogue, equal the
    oracle's attention over each sequence's keys of both sets.  One sequence
    has no keys in the first set."""
    fa = _fa()
    rng = np.random.default_rng(21)
    hq, hkv, d = 4, 2, 128
    q_lens, ka, kb = [100, 300, 1], [50, 0, 7], [130, 260, 200]
    cu = lambda L: torch.tensor(np.concatenate([[0], np.cumsum(L)]), dtype=torch.int32)
    q = _bf(rng, hq, sum(q_lens), d)
    k1, v1 = _bf(rng, hkv, sum(ka), d), _bf(rng, hkv, sum(ka), d)
    k2, v2 = _bf(rng, hkv, sum(kb), d), _bf(rng, hkv, sum(kb), d)
    acc_o = torch.empty((hq, sum(q_lens), d), dtype=torch.float32, device="cuda")
    acc_l = torch.empty((hq, sum(q_lens)), dtype=torch.float32, device="cuda")
    epi = [("add", 0.25)]
    common = dict(hq=hq, hkv=hkv, cu_seqlens_q=cu(q_lens).cuda(), max_seqlen_q=max(q_lens))
    fa.attention_fwd_acc(q.cuda(), k1.cuda(), v1.cuda(), acc_o, acc_l, first=True, cu_seqlens_k=cu(ka).cuda(),
                         max_seqlen_k=max(ka), **common)
    out = fa.attention_fwd_acc(q.cuda(), k2.cuda(), v2.cuda(), acc_o, acc_l, last=True, epilogue=epi,
                               cu_seqlens_k=cu(kb).cuda(), max_seqlen_k=max(kb), **common)
    assert fa.check_device_error() == fa.FA_OK
    # the oracle over each sequence's keys of both sets, concatenated per sequence
    cq, ca_, cb_ = cu(q_lens).numpy(), cu(ka).numpy(), cu(kb).numpy()
    ks, vs, ck = [], [], [0]
    for b in range(len(q_lens)):
        ks += [k1[:, ca_[b]:ca_[b + 1]], k2[:, cb_[b]:cb_[b + 1]]]
        vs += [v1[:, ca_[b]:ca_[b + 1]], v2[:, cb_[b]:cb_[b + 1]]]
        ck.append(ck[-1] + ka[b] + kb[b])
    kc, vc = torch.cat(ks, dim=1), torch.cat(vs, dim=1)
    ref = oracle.attention(q, kc, vc, hq=hq, hkv=hkv, epilogue=epi, cu_seqlens_q=cq,
                           cu_seqlens_k=np.array(ck, dtype=np.int32))
    assert_close_bf16(out.float().cpu().numpy(), ref)
