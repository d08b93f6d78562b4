"""GPU parity of the TurboQuant KV cache (the C attention library's README,
"TurboQuant KV Cache Compression"): fa_tq_compress against the oracle's codes
and norms (a code may differ only where the oracle's coordinate sits within
fp32 rounding of a cell edge), and fa_tq_attention_decode against the oracle's
decode over the oracle's dequantisation of the same cache."""
import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16
from oracle import turboquant as tq

pytestmark = pytest.mark.gpu


def _fa():
    from flashattention_attention_b200 import fa
    return fa


def _signs(d, seed):
    from flashattention_attention_b200 import inputs
    return inputs.rotation_signs(d, seed)


def _check_codes(got_packed, got_norms, x, signs, bits, what=""):
    d = x.shape[-1]
    lv = tq.codebook(d, bits)
    codes, norms = tq.quantize(x, signs, lv)
    got = tq.unpack(got_packed, bits, d)
    u = tq.unit_coords(x, signs)
    near = np.min(np.abs(u[..., None] - tq.edges_of(lv)), axis=-1) < 2e-6
    bad = (got != codes) & ~near
    assert not bad.any(), f"{what}: {int(bad.sum())} codes differ away from a cell edge"
    assert np.mean(got != codes) < 1e-3, what
    assert np.allclose(got_norms, norms, rtol=2e-6, atol=0), what


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_compress_matches_oracle(d, bits, dtype):
    fa = _fa()
    rng = np.random.default_rng(d + 10 * bits + (dtype == torch.float32))
    rows = 1003
    x = torch.from_numpy((rng.standard_normal((rows, d)) * rng.uniform(0.1, 10, (rows, 1))).astype(np.float32))
    x[7] = 0  # a zero row: u = 0, the lower of the two middle levels
    x = x.to(dtype)
    s = _signs(d, bits)
    lv = fa.tq_codebook(d, bits)
    codes, norms = fa.tq_compress(x.cuda(), s.cuda(), lv.cuda(), bits)
    assert fa.check_device_error() == fa.FA_OK
    _check_codes(codes.cpu().numpy(), norms.cpu().numpy(), x.double().numpy(), s.numpy(), bits, f"d{d} b{bits}")
    zero = tq.unpack(codes[7].cpu().numpy(), bits, d)
    assert np.all(zero == (1 << bits) // 2 - 1) and norms[7].item() == 0


def _cache(rng, B, hkv, cap, d, kb, vb, seed):
    fa = _fa()
    k = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16().cuda()
    v = torch.from_numpy(rng.standard_normal((B * hkv, cap, d)).astype(np.float32)).bfloat16().cuda()
    s = _signs(d, seed).cuda()
    lk, lv = fa.tq_codebook(d, kb).cuda(), fa.tq_codebook(d, vb).cuda()
    kc, kn = fa.tq_compress(k, s, lk, kb)
    vc, vn = fa.tq_compress(v, s, lv, vb)
    return dict(kc=kc, kn=kn, vc=vc, vn=vn, s=s, lk=lk, lv=lv)


def _dequant(c, d, kb, vb):
    s = c["s"].cpu().numpy()
    kh = tq.dequantize(c["kc"].cpu().numpy(), c["kn"].cpu().numpy(), s, kb, tq.codebook(d, kb), d)
    vh = tq.dequantize(c["vc"].cpu().numpy(), c["vn"].cpu().numpy(), s, vb, tq.codebook(d, vb), d)
    return kh, vh


@pytest.mark.parametrize("d,kb,vb,group", [(128, 4, 2, 4), (128, 3, 3, 8), (128, 2, 4, 1), (64, 4, 4, 2),
                                           (64, 3, 2, 4), (128, 4, 4, 2)])
def test_decode_matches_oracle_on_the_same_cache(d, kb, vb, group):
    fa = _fa()
    rng = np.random.default_rng(d + kb * 10 + vb + group)
    hkv = 2
    hq = hkv * group
    lengths = [4097, 1, 2048, 33, 0]  # several 2048-key splits, ragged tails, an empty cache
    B, cap = len(lengths), 4200
    c = _cache(rng, B, hkv, cap, d, kb, vb, seed=kb)
    q = torch.from_numpy(rng.standard_normal((B * hq, d)).astype(np.float32)).bfloat16()
    lens = torch.tensor(lengths, dtype=torch.int32).cuda()
    epi = [("mul", 2.0), ("add", 0.5)]
    out = fa.tq_attention_decode(q.cuda(), c["kc"], c["kn"], c["vc"], c["vn"], lens, hq=hq, hkv=hkv, k_bits=kb,
                                 v_bits=vb, k_levels=c["lk"], v_levels=c["lv"], signs=c["s"], epilogue=epi)
    assert fa.check_device_error() == fa.FA_OK
    kh, vh = _dequant(c, d, kb, vb)
    got = out.float().cpu().numpy()
    live = [b for b, L in enumerate(lengths) if L > 0]
    for b in live:
        ref = oracle.decode(q.reshape(B * hq, 1, d)[b * hq:(b + 1) * hq], kh[b * hkv:(b + 1) * hkv],
                            vh[b * hkv:(b + 1) * hkv], [lengths[b]], hq=hq, hkv=hkv, epilogue=epi)
        assert_close_bf16(got[b * hq:(b + 1) * hq], ref.reshape(hq, d), what=f"sequence {b}")
    assert np.all(got[(B - 1) * hq:] == 0.5)  # the empty cache: the epilogue of 0


def test_length_beyond_the_capacity_is_clamped_and_reported():
    fa = _fa()
    rng = np.random.default_rng(5)
    d, hkv, hq, cap = 128, 1, 4, 300
    c = _cache(rng, 1, hkv, cap, d, 4, 2, seed=1)
    q = torch.from_numpy(rng.standard_normal((hq, d)).astype(np.float32)).bfloat16().cuda()
    args = dict(hq=hq, hkv=hkv, k_bits=4, v_bits=2, k_levels=c["lk"], v_levels=c["lv"], signs=c["s"])
    a = fa.tq_attention_decode(q, c["kc"], c["kn"], c["vc"], c["vn"], torch.tensor([cap + 5], dtype=torch.int32).cuda(),
                               **args)
    assert fa.check_device_error() == fa.FA_ERR_INVALID
    b = fa.tq_attention_decode(q, c["kc"], c["kn"], c["vc"], c["vn"], torch.tensor([cap], dtype=torch.int32).cuda(),
                               **args)
    assert fa.check_device_error() == fa.FA_OK
    assert torch.equal(a, b)


def test_quality_against_the_uncompressed_cache():
    """K4/V2 and K4/V4 against exact attention on the bf16 cache: the
    attention-output cosine the page reports (about 0.94 and 0.99)."""
    fa = _fa()
    rng = np.random.default_rng(6)
    d, hkv, hq, L = 128, 2, 8, 512
    k = torch.from_numpy(rng.standard_normal((hkv, L, d)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((hkv, L, d)).astype(np.float32)).bfloat16()
    q = torch.from_numpy(rng.standard_normal((hq, d)).astype(np.float32)).bfloat16()
    ref = oracle.decode(q.reshape(hq, 1, d), k, v, [L], hq=hq, hkv=hkv).reshape(hq, d)
    s = _signs(d, 3).cuda()
    cos = {}
    for vb in (2, 4):
        lk, lv = fa.tq_codebook(d, 4).cuda(), fa.tq_codebook(d, vb).cuda()
        kc, kn = fa.tq_compress(k.cuda(), s, lk, 4)
        vc, vn = fa.tq_compress(v.cuda(), s, lv, vb)
        o = fa.tq_attention_decode(q.cuda(), kc, kn, vc, vn, torch.tensor([L], dtype=torch.int32).cuda(), hq=hq,
                                   hkv=hkv, k_bits=4, v_bits=vb, k_levels=lk, v_levels=lv, signs=s)
        o = o.float().cpu().numpy()
        cos[vb] = float(np.mean(np.sum(o * ref, -1) / (np.linalg.norm(o, axis=-1) * np.linalg.norm(ref, axis=-1))))
    assert 0.92 <= cos[2] <= 0.96 and 0.985 <= cos[4] <= 0.995, cos


def test_full_size_decode_workload_sampled(decode_workload):
    """The bench's TurboQuant line: the decode workload's cache (B=16, Hq=32,
    Hkv=8, d=128, lengths U[1024, 32768], capacity 32768) compressed K4/V2,
    one decode step; four sequences checked against the oracle."""
    fa = _fa()
    w = decode_workload
    s = _signs(128, 0).cuda()
    lk, lv = fa.tq_codebook(128, 4).cuda(), fa.tq_codebook(128, 2).cuda()
    kc, kn = fa.tq_compress(w.k.cuda(), s, lk, 4)
    vc, vn = fa.tq_compress(w.v.cuda(), s, lv, 2)
    lens = torch.tensor(w.lengths, dtype=torch.int32).cuda()
    out = fa.tq_attention_decode(w.q.reshape(-1, 128).cuda(), kc, kn, vc, vn, lens, hq=32, hkv=8, k_bits=4,
                                 v_bits=2, k_levels=lk, v_levels=lv, signs=s)
    assert fa.check_device_error() == fa.FA_OK
    got = out.float().cpu().numpy()
    sn = s.cpu().numpy()
    for b in (0, 5, 11, 15):
        L = int(w.lengths[b])
        sl = slice(b * 8, (b + 1) * 8)
        kh = tq.dequantize(kc[sl, :L].cpu().numpy(), kn[sl, :L].cpu().numpy(), sn, 4, tq.codebook(128, 4), 128)
        vh = tq.dequantize(vc[sl, :L].cpu().numpy(), vn[sl, :L].cpu().numpy(), sn, 2, tq.codebook(128, 2), 128)
        ref = oracle.decode(w.q[b * 32:(b + 1) * 32], kh, vh, [L], hq=32, hkv=8).reshape(32, 128)
        assert_close_bf16(got[b * 32:(b + 1) * 32], ref, what=f"sequence {b} (L={L})")
