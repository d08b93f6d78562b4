"""GPU parity of the tensor-core prefill (bf16 Q/K/V) against the fp64
oracle on the same bf16 inputs: max abs <= 2e-2 and relative L2 <= 5e-3
(fkl_python PR #6, Verification: dense causal, ragged 33/127, fused
epilogue == host-applied; SKaiNET-transformers PR #419, Summary: GQA groups,
sliding windows, empty bands)."""
import pytest
import torch

import oracle
from conftest import assert_close_bf16, assert_close_bf16_planes
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def gpu_fwd(q, k, v, **kw):
    from flashattention_attention_b200 import fa
    out = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), **kw)
    torch.cuda.synchronize()
    assert fa.check_device_error() == fa.FA_OK
    return out.cpu()


DENSE = [
    # B, hq, hkv, s_q, s_k, d, causal, window
    (1, 2, 1, 128, 128, 128, False, 0),
    (2, 8, 2, 300, 300, 128, True, 0),
    (1, 4, 4, 200, 333, 64, True, 0),      # G = 1: one Q tile per CTA
    (1, 4, 2, 257, 1000, 128, False, 0),
    (1, 4, 2, 513, 513, 64, True, 100),    # causal + window
    (1, 6, 2, 130, 50, 128, True, 0),      # s_q > s_k: empty-band rows
    (2, 4, 2, 33, 127, 64, True, 0),       # ragged 33/127
    (2, 4, 2, 33, 127, 128, False, 0),
    (1, 8, 1, 64, 700, 128, False, 200),   # window without causal
    (1, 2, 2, 1, 1, 64, True, 0),
    (1, 6, 3, 384, 384, 64, True, 0),      # G = 2
    (2, 4, 2, 33, 127, 32, True, 0),       # ragged 33/127 at d = 32 (fkl_python PR #6, Verification)
    (2, 4, 2, 33, 127, 32, False, 0),
    (1, 6, 2, 130, 50, 32, True, 0),       # d = 32 with empty-band rows
    (1, 8, 2, 300, 300, 96, True, 0),      # d = 96: a 64-dim chunk and a 32-dim tail
    (1, 4, 1, 257, 700, 96, False, 200),
    (1, 4, 4, 200, 333, 96, True, 0),
    (1, 4, 2, 300, 300, 256, True, 0),     # d = 256: one Q tile per CTA, 64-key tiles
    (2, 2, 1, 33, 127, 256, False, 0),
    (1, 4, 2, 257, 700, 192, True, 150),   # d = 192 with a window
    (1, 2, 2, 130, 50, 160, True, 0),      # d = 160 (a 32-dim tail) with empty-band rows
    (1, 8, 2, 200, 200, 224, False, 0),    # d = 224
]


@pytest.mark.parametrize("case", DENSE, ids=lambda c: "-".join(map(str, c)))
def test_dense(case):
    B, hq, hkv, s_q, s_k, d, causal, window = case
    w = inputs.dense_prefill("t", batch=B, hq=hq, hkv=hkv, s_q=s_q, s_k=s_k, d=d,
                             dtype=torch.bfloat16, causal=causal, window=window, seed=sum(case))
    got = gpu_fwd(w.q, w.k, w.v, hq=hq, hkv=hkv, causal=causal, window=window)
    ref = oracle.attention(w.q, w.k, w.v, hq=hq, hkv=hkv, causal=causal, window=window)
    assert_close_bf16(got.float().numpy(), ref, what=str(case))


@pytest.mark.parametrize("d", [32, 64, 96, 128, 256])
@pytest.mark.parametrize("causal,window", [(True, 0), (True, 100), (False, 0)])
def test_varlen(d, causal, window):
    lengths = [33, 127, 1, 300, 129, 256]
    w = inputs.varlen_prefill("t", lengths=lengths, hq=8, hkv=2, d=d, dtype=torch.bfloat16,
                              causal=causal, window=window, seed=d + window)
    cu = inputs.cu_from_lengths(lengths)
    got = gpu_fwd(w.q, w.k, w.v, hq=8, hkv=2, causal=causal, window=window,
                  cu_seqlens_q=cu.cuda(), max_seqlen_q=max(lengths))
    ref = oracle.attention(w.q, w.k, w.v, hq=8, hkv=2, causal=causal, window=window,
                           cu_seqlens_q=cu.numpy())
    assert_close_bf16(got.float().numpy(), ref)


def test_varlen_rows_past_a_sequence_end_are_untouched():
    """Rows of the next sequence inside a Q tile must not be written by the
    previous sequence's tile (canary: out pre-filled, compare every row)."""
    from flashattention_attention_b200 import fa
    lengths = [5, 200, 7]
    w = inputs.varlen_prefill("t", lengths=lengths, hq=4, hkv=2, d=128, dtype=torch.bfloat16,
                              causal=True, seed=3)
    cu = inputs.cu_from_lengths(lengths)
    out = torch.full_like(w.q, 1234.0).cuda()
    fa.attention_fwd(w.q.cuda(), w.k.cuda(), w.v.cuda(), hq=4, hkv=2, causal=True,
                     cu_seqlens_q=cu.cuda(), max_seqlen_q=200, out=out)
    ref = oracle.attention(w.q, w.k, w.v, hq=4, hkv=2, causal=True, cu_seqlens_q=cu.numpy())
    assert_close_bf16(out.cpu().float().numpy(), ref)


def test_epilogue_and_determinism():
    from flashattention_attention_b200 import fa
    w = inputs.dense_prefill("t", batch=1, hq=4, hkv=2, s_q=260, s_k=260, d=128,
                             dtype=torch.bfloat16, causal=True, seed=5)
    epi = [("mul", 2.0), ("add", 0.5)]
    variants = None
    outs = []
    for vals in ([("mul", 2.0), ("add", 0.5)], [("mul", -1.5), ("add", 3.0)], [("mul", 2.0), ("add", 0.5)]):
        outs.append(gpu_fwd(w.q, w.k, w.v, hq=4, hkv=2, causal=True, epilogue=vals))
        if variants is None:
            variants = fa.kernel_variants_used()
    assert fa.kernel_variants_used() == variants  # values never instantiate a new kernel
    assert torch.equal(outs[0], outs[2])          # bitwise run-to-run determinism
    ref = oracle.attention(w.q, w.k, w.v, hq=4, hkv=2, causal=True, epilogue=epi)
    assert_close_bf16(outs[0].float().numpy(), ref)
    ref2 = oracle.attention(w.q, w.k, w.v, hq=4, hkv=2, causal=True, epilogue=[("mul", -1.5), ("add", 3.0)])
    assert_close_bf16(outs[1].float().numpy(), ref2)
    # the most ops a call takes (FA_MAX_EPILOGUE = 8), still no new kernel
    longest = [("mul", 2.0), ("add", 0.5), ("mul", 0.25), ("add", -1.0), ("mul", 3.0), ("add", 0.125),
               ("mul", -0.5), ("add", 2.0)]
    got = gpu_fwd(w.q, w.k, w.v, hq=4, hkv=2, causal=True, epilogue=longest)
    assert fa.kernel_variants_used() == variants
    ref3 = oracle.attention(w.q, w.k, w.v, hq=4, hkv=2, causal=True, epilogue=longest)
    assert_close_bf16(got.float().numpy(), ref3)


def test_gqa_equals_repeated_kv():
    w = inputs.dense_prefill("t", batch=1, hq=8, hkv=2, s_q=200, s_k=200, d=64,
                             dtype=torch.bfloat16, causal=True, seed=6)
    a = gpu_fwd(w.q, w.k, w.v, hq=8, hkv=2, causal=True)
    b = gpu_fwd(w.q, w.k.repeat_interleave(4, 0), w.v.repeat_interleave(4, 0), hq=8, hkv=8, causal=True)
    assert (a.float() - b.float()).abs().max() <= 2e-2


def test_full_size_gqa_causal_prefill():
    """B=4, Hq=32, Hkv=8, S=4096, d=128, causal: the bench's launch, every
    output row checked against the oracle."""
    w = inputs.gqa_causal_prefill()
    got = gpu_fwd(w.q, w.k, w.v, hq=32, hkv=8, causal=True)
    ref = oracle.attention(w.q, w.k, w.v, hq=32, hkv=8, causal=True)
    assert_close_bf16_planes(got, ref, what="full-size prefill, every row")


def test_full_size_varlen_window_epilogue():
    """8 packed sequences U[33, 8192], Hq=32, Hkv=8, d=64, causal, window
    1024, epilogue [Mul(2.0), Add(0.5)]: the bench's launch, every output row
    checked against the oracle."""
    w = inputs.varlen_window_prefill()
    cu = inputs.cu_from_lengths(w.lengths)
    got = gpu_fwd(w.q, w.k, w.v, hq=32, hkv=8, causal=True, window=1024, epilogue=w.epilogue,
                  cu_seqlens_q=cu.cuda(), max_seqlen_q=max(w.lengths))
    ref = oracle.attention(w.q, w.k, w.v, hq=32, hkv=8, causal=True, window=1024, epilogue=w.epilogue,
                           cu_seqlens_q=cu.numpy())
    assert_close_bf16_planes(got, ref, what="full-size varlen, every row")
