"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/fa.h declares, and rejects bad arguments on the host before any
CUDA call (fa.h: "Argument checks run on the host before any launch")."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def test_header_declares_the_three_calls():
    names = header_functions()
    for n in ("fa_compress_kv", "fa_attention_fwd", "fa_attention_decode"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from flashattention_attention_b200 import fa
    for name in header_functions():
        assert hasattr(fa.lib, name), name


@pytest.fixture(scope="module")
def fa():
    from flashattention_attention_b200 import fa as mod
    return mod


class FakeTensor:
    """Carries a (never dereferenced) address through the fa.py marshalling."""
    def __init__(self, addr, shape, dtype):
        self._a, self.shape, self.dtype = addr, shape, dtype

    def data_ptr(self):
        return self._a

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        return 1


def fwd(fa, **kw):
    import torch
    base = dict(hq=4, hkv=2, causal=True)
    q = FakeTensor(0x10000, (4, 64, 128), torch.bfloat16)
    k = FakeTensor(0x20000, (2, 64, 128), torch.bfloat16)
    v = FakeTensor(0x30000, (2, 64, 128), torch.bfloat16)
    o = FakeTensor(0x40000, (4, 64, 128), torch.bfloat16)
    tensors = dict(q=q, k=k, v=v, out=o)
    for name in ("q", "k", "v", "out"):
        if name in kw:
            tensors[name] = kw.pop(name)
    base.update(kw)
    p = fa.fwd_params(tensors["q"], tensors["k"], tensors["v"], tensors["out"], **base)
    return p


def call_fwd(fa, p):
    return fa.lib.fa_attention_fwd(ctypes.byref(p), None)


def test_fwd_rejects_bad_arguments(fa):
    import torch
    assert fa.lib.fa_attention_fwd(None, None) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.hq = 3  # hq % hkv != 0
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.head_dim = 48  # not a multiple of 32
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.head_dim = 288  # multiple of 32 but no tensor-core kernel (32 .. 256)
    assert call_fwd(fa, p) == fa.FA_ERR_UNSUPPORTED
    p = fwd(fa)
    p.head_dim, p.kv_dtype = 288, fa.FA_I8  # int8 K/V: the same head sizes
    p.k_scales, p.v_scales = 0x50000, 0x58000
    assert call_fwd(fa, p) == fa.FA_ERR_UNSUPPORTED
    p = fwd(fa)
    p.n_epilogue = 9
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.n_epilogue = 1
    p.epilogue[0].op = 7  # unknown op
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.q = 0x10008  # misaligned
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.out = None
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID
    p = fwd(fa, k=FakeTensor(0x20000, (2, 64, 128), torch.int8),
            v=FakeTensor(0x30000, (2, 64, 128), torch.int8))
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID  # int8 without scales
    p = fwd(fa, q=FakeTensor(0x10000, (4, 64, 128), torch.float32))
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID  # fp32 q with bf16 kv
    p = fwd(fa)
    p.softmax_scale = float("nan")
    assert call_fwd(fa, p) == fa.FA_ERR_INVALID


def test_fwd_empty_problem_is_a_noop(fa):
    p = fwd(fa)
    p.seqlen_q = 0
    p.q = p.k = p.v = p.out = None
    assert call_fwd(fa, p) == fa.FA_OK


def test_compress_rejects_bad_arguments(fa):
    lib = fa.lib
    assert lib.fa_compress_kv(0x1000, fa.FA_BF16, 4, 15, 0x2000, 0x3000, None) == fa.FA_ERR_INVALID
    assert lib.fa_compress_kv(0x1000, fa.FA_I8, 4, 64, 0x2000, 0x3000, None) == fa.FA_ERR_INVALID
    assert lib.fa_compress_kv(0x1008, fa.FA_BF16, 4, 64, 0x2000, 0x3000, None) == fa.FA_ERR_INVALID
    assert lib.fa_compress_kv(None, fa.FA_BF16, 4, 64, 0x2000, 0x3000, None) == fa.FA_ERR_INVALID
    assert lib.fa_compress_kv(None, fa.FA_BF16, 0, 64, None, None, None) == fa.FA_OK
    assert lib.fa_compress_kv(0x1000, fa.FA_BF16, -1, 64, 0x2000, 0x3000, None) == fa.FA_ERR_INVALID


def decode_p(fa, **over):
    import torch
    q = FakeTensor(0x10000, (16, 128), torch.bfloat16)
    kc = FakeTensor(0x20000, (4, 1024, 128), torch.int8)
    vc = FakeTensor(0x30000, (4, 1024, 128), torch.int8)
    sl = FakeTensor(0x40000, (2,), torch.int32)
    o = FakeTensor(0x50000, (16, 128), torch.bfloat16)
    need = fa.decode_workspace_size(2, 16, 1024, 128)
    ws = FakeTensor(0x100000, (need,), torch.uint8)
    p = fa.decode_params(q, kc, vc, sl, o, ws, hq=8, hkv=2, k_scales=FakeTensor(0x60000, (4, 1024), None),
                         v_scales=FakeTensor(0x70000, (4, 1024), None))
    for k, v in over.items():
        setattr(p, k, v)
    return p


def test_decode_rejects_bad_arguments(fa):
    lib = fa.lib
    call = lambda p: lib.fa_attention_decode(ctypes.byref(p), None)
    assert lib.fa_attention_decode(None, None) == fa.FA_ERR_INVALID
    assert call(decode_p(fa, hq=9)) == fa.FA_ERR_INVALID
    assert call(decode_p(fa, capacity=1000)) == fa.FA_ERR_INVALID       # not a multiple of 32
    assert call(decode_p(fa, max_seqlen=2048)) == fa.FA_ERR_INVALID     # above capacity
    assert call(decode_p(fa, split_keys=100)) == fa.FA_ERR_INVALID
    assert call(decode_p(fa, head_dim=160)) == fa.FA_ERR_UNSUPPORTED   # int8 cache: 32, 64, 96, 128, 256
    assert call(decode_p(fa, hq=32, hkv=2)) != fa.FA_ERR_UNSUPPORTED    # a group of 16 runs in two passes
    assert call(decode_p(fa, k_scales=None)) == fa.FA_ERR_INVALID
    assert call(decode_p(fa, workspace_bytes=16)) == fa.FA_ERR_WORKSPACE
    assert call(decode_p(fa, workspace=None)) == fa.FA_ERR_WORKSPACE
    assert call(decode_p(fa, q=0x10004)) == fa.FA_ERR_INVALID


def test_workspace_size_formula(fa):
    # tile plan (int32 prefix [B+1] and per-segment counters [B*hq], 256-byte
    # padded), then one (d + 2)-float record per (sequence, q-head) and per
    # (worker warp, head of a group of at most 8); without a GPU the library
    # assumes 148 SMs: 148 * 2 CTAs * 4 warps
    workers = 148 * 2 * 4
    plan = lambda b, hq: ((b + 1 + b * hq) * 4 + 255) // 256 * 256
    assert fa.decode_workspace_size(16, 32, 32768, 128) == plan(16, 32) + (16 * 32 + workers * 8) * 130 * 4
    assert fa.decode_workspace_size(1, 2, 256, 64) == plan(1, 2) + (1 * 2 + workers * 2) * 66 * 4
    assert fa.decode_workspace_size(0, 1, 1, 64) == 0


def test_status_strings(fa):
    for s in range(6):
        assert fa.lib.fa_status_string(s)
    assert fa.lib.fa_status_string(99) == b"unknown status"


def append_call(fa, **kw):
    """fa_kv_append through the C ABI with fake (never dereferenced) pointers;
    every case here must be rejected on the host before any CUDA call."""
    p = fa.KvAppendParams()
    p.k_new, p.v_new, p.x_dtype = 0x10000, 0x20000, fa.FA_BF16
    p.k_cache, p.v_cache, p.cache_dtype = 0x30000, 0x40000, fa.FA_I8
    p.k_scales, p.v_scales = 0x50000, 0x60000
    p.cur_pos, p.cache_seqlens = 0x70000, 0x80000
    p.batch, p.hkv, p.head_dim, p.capacity = 4, 2, 128, 64
    for k, v in kw.items():
        setattr(p, k, v)
    return fa.lib.fa_kv_append(ctypes.byref(p), None)


def test_kv_append_rejects_bad_arguments(fa):
    assert fa.lib.fa_kv_append(None, None) == fa.FA_ERR_INVALID
    assert append_call(fa, head_dim=8) == fa.FA_ERR_INVALID            # below 16
    assert append_call(fa, head_dim=136) == fa.FA_ERR_INVALID          # not a multiple of 16
    assert append_call(fa, head_dim=2048) == fa.FA_ERR_INVALID
    assert append_call(fa, x_dtype=fa.FA_I8) == fa.FA_ERR_INVALID      # new rows must be float
    assert append_call(fa, cache_dtype=fa.FA_F32) == fa.FA_ERR_INVALID
    assert append_call(fa, k_scales=None) == fa.FA_ERR_INVALID         # int8 cache needs scales
    assert append_call(fa, cur_pos=None) == fa.FA_ERR_INVALID
    assert append_call(fa, k_new=0x10004) == fa.FA_ERR_INVALID         # 16-byte alignment
    assert append_call(fa, capacity=0) == fa.FA_ERR_INVALID
    assert append_call(fa, hkv=0) == fa.FA_ERR_INVALID
    assert append_call(fa, batch=-1) == fa.FA_ERR_INVALID
    # cache_seqlens overlapping cur_pos (one warp writes what others read)
    assert append_call(fa, cache_seqlens=0x70000) == fa.FA_ERR_INVALID
    assert append_call(fa, cache_seqlens=0x70000 + 16, batch=8) == fa.FA_ERR_INVALID


def test_kv_append_empty_batch_is_a_noop(fa):
    assert append_call(fa, batch=0) == fa.FA_OK


def test_decode_paged_rejects_bad_arguments(fa):
    import torch
    q = FakeTensor(0x10000, (8, 128), torch.bfloat16)
    kp = FakeTensor(0x20000, (16, 2, 64, 128), torch.int8)
    lens = FakeTensor(0x30000, (2,), torch.int32)
    o = FakeTensor(0x40000, (8, 128), torch.bfloat16)
    ws = FakeTensor(0x50000, (1 << 24,), torch.uint8)
    sc = FakeTensor(0x60000, (16, 2, 64), torch.float32)
    p = fa.decode_params(q, kp, kp, lens, o, ws, hq=4, hkv=2, k_scales=sc, v_scales=sc)

    def call(**kw):
        pg = fa.KvPages(0x70000, 4, 64, 16)
        p.capacity = 256
        for k, v in kw.items():
            if hasattr(pg, k):
                setattr(pg, k, v)
            else:
                setattr(p, k, v)
        return fa.lib.fa_attention_decode_paged(ctypes.byref(p), ctypes.byref(pg), None)

    assert fa.lib.fa_attention_decode_paged(ctypes.byref(p), None, None) == fa.FA_ERR_INVALID
    assert call(page_size=48) == fa.FA_ERR_INVALID           # not a multiple of 32
    assert call(capacity=512) == fa.FA_ERR_INVALID           # capacity != max_pages * page_size
    assert call(block_table=None) == fa.FA_ERR_INVALID
    assert call(block_table=0x70004) == fa.FA_ERR_INVALID    # alignment
    assert call(num_pages=0) == fa.FA_ERR_INVALID
    assert call(num_pages=1 << 24) == fa.FA_ERR_UNSUPPORTED  # pool rows past 2^31
    assert call(workspace_bytes=16) == fa.FA_ERR_WORKSPACE


def test_kv_append_paged_rejects_bad_arguments(fa):
    def call(**kw):
        p = fa.KvAppendParams()
        p.k_new, p.v_new, p.x_dtype = 0x10000, 0x20000, fa.FA_BF16
        p.k_cache, p.v_cache, p.cache_dtype = 0x30000, 0x40000, fa.FA_I8
        p.k_scales, p.v_scales = 0x50000, 0x60000
        p.cur_pos, p.cache_seqlens = 0x70000, 0x80000
        p.batch, p.hkv, p.head_dim, p.capacity = 4, 2, 128, 256
        pg = fa.KvPages(0x90000, 4, 64, 16)
        for k, v in kw.items():
            setattr(pg if hasattr(pg, k) else p, k, v)
        return fa.lib.fa_kv_append_paged(ctypes.byref(p), ctypes.byref(pg), None)
    assert call(capacity=512) == fa.FA_ERR_INVALID        # capacity != max_pages * page_size
    assert call(block_table=None) == fa.FA_ERR_INVALID
    assert call(num_pages=0) == fa.FA_ERR_INVALID
    assert call(head_dim=8) == fa.FA_ERR_INVALID
    assert call(batch=0) == fa.FA_OK


def test_fwd_paged_rejects_bad_arguments(fa):
    def call(**kw):
        p = fa.FwdParams()
        p.q, p.k, p.v, p.out = 0x10000, 0x20000, 0x30000, 0x40000
        p.q_dtype, p.kv_dtype = fa.FA_BF16, fa.FA_BF16
        p.batch, p.hq, p.hkv, p.head_dim, p.seqlen_q = 2, 4, 2, 128, 64
        p.cu_seqlens_k = 0x50000
        p.causal, p.softmax_scale = 1, 0.125
        pg = fa.KvPages(0x60000, 4, 128, 8)
        for k, v in kw.items():
            setattr(pg if hasattr(pg, k) else p, k, v)
        return fa.lib.fa_attention_fwd_paged(ctypes.byref(p), ctypes.byref(pg), None)
    assert call(page_size=64) == fa.FA_ERR_INVALID          # not a multiple of 128
    assert call(cu_seqlens_k=None) == fa.FA_ERR_INVALID      # per-sequence key counts required
    assert call(block_table=None) == fa.FA_ERR_INVALID
    assert call(q_dtype=fa.FA_F32, kv_dtype=fa.FA_F32) == fa.FA_ERR_INVALID   # tensor-core path only
    assert call(head_dim=288) == fa.FA_ERR_UNSUPPORTED
    assert call(kv_dtype=fa.FA_I8) == fa.FA_ERR_INVALID       # int8 needs scales
    assert call(seqlen_q=0) == fa.FA_OK                       # nothing to do


def test_fwd_lse_rejects_bad_arguments(fa):
    import torch
    lse = 0x50000
    assert fa.lib.fa_attention_fwd_lse(None, lse, None) == fa.FA_ERR_INVALID
    p = fwd(fa)
    assert fa.lib.fa_attention_fwd_lse(ctypes.byref(p), None, None) == fa.FA_ERR_INVALID  # no lse buffer
    assert fa.lib.fa_attention_fwd_lse(ctypes.byref(p), 0x50004, None) == fa.FA_ERR_INVALID  # misaligned lse
    p = fwd(fa, q=FakeTensor(0x10000, (4, 64, 128), torch.float32), k=FakeTensor(0x20000, (2, 64, 128), torch.float32),
            v=FakeTensor(0x30000, (2, 64, 128), torch.float32), out=FakeTensor(0x40000, (4, 64, 128), torch.float32))
    assert fa.lib.fa_attention_fwd_lse(ctypes.byref(p), lse, None) == fa.FA_ERR_UNSUPPORTED  # fp32: no lse output
    p = fwd(fa)
    p.hq = 3
    assert fa.lib.fa_attention_fwd_lse(ctypes.byref(p), lse, None) == fa.FA_ERR_INVALID
    p = fwd(fa)
    p.seqlen_q = 0
    p.q = p.k = p.v = p.out = None
    assert fa.lib.fa_attention_fwd_lse(ctypes.byref(p), None, None) == fa.FA_OK  # empty problem


def test_merge_rejects_bad_arguments(fa):
    assert fa.lib.fa_attention_merge(None, None) == fa.FA_ERR_INVALID

    def params(**kw):
        p = fa.MergeParams()
        p.o_acc, p.lse_acc, p.o_part, p.lse_part = 0x10000, 0x20000, 0x30000, 0x40000
        p.part_dtype, p.rows, p.head_dim = fa.FA_BF16, 10, 128
        for key, val in kw.items():
            setattr(p, key, val)
        return fa.lib.fa_attention_merge(ctypes.byref(p), None)

    assert params(head_dim=48) == fa.FA_ERR_INVALID
    assert params(head_dim=288) == fa.FA_ERR_INVALID
    assert params(rows=-1) == fa.FA_ERR_INVALID
    assert params(part_dtype=fa.FA_I8) == fa.FA_ERR_INVALID
    assert params(out=0x50000, out_dtype=fa.FA_I8) == fa.FA_ERR_INVALID
    assert params(lse_part=None) == fa.FA_ERR_INVALID
    assert params(o_acc=None) == fa.FA_ERR_INVALID
    assert params(o_acc=0x10008) == fa.FA_ERR_INVALID
    assert params(n_epilogue=9) == fa.FA_ERR_INVALID
    assert params(rows=0, o_acc=None, lse_acc=None) == fa.FA_OK


def test_fwd_acc_rejects_bad_arguments(fa):
    import torch
    acc, lse = 0x60000, 0x70000
    call = lambda p, a=acc, l=lse, f=0: fa.lib.fa_attention_fwd_acc(ctypes.byref(p) if p is not None else None,
                                                                    a, l, f, None)
    assert call(None) == fa.FA_ERR_INVALID
    p = fwd(fa)
    assert call(p, f=4) == fa.FA_ERR_INVALID                  # unknown flag
    assert call(p, a=None) == fa.FA_ERR_INVALID               # no accumulator
    assert call(p, l=0x70008) == fa.FA_ERR_INVALID            # misaligned lse_acc
    p.out = None
    assert call(p, f=fa.FA_ACC_LAST) == fa.FA_ERR_INVALID     # the last step writes out
    p = fwd(fa, q=FakeTensor(0x10000, (4, 64, 128), torch.float32), k=FakeTensor(0x20000, (2, 64, 128), torch.float32),
            v=FakeTensor(0x30000, (2, 64, 128), torch.float32), out=FakeTensor(0x40000, (4, 64, 128), torch.float32))
    assert call(p) == fa.FA_ERR_UNSUPPORTED                   # fp32 path
    p = fwd(fa)
    p.head_dim = 288
    assert call(p) == fa.FA_ERR_UNSUPPORTED
    p = fwd(fa)
    p.seqlen_q = 0
    p.q = p.k = p.v = p.out = None
    assert call(p, a=None, l=None, f=3) == fa.FA_OK           # empty problem


@pytest.mark.parametrize("d,bits", [(64, 2), (64, 4), (128, 2), (128, 3), (128, 4)])
def test_tq_codebook_host_function_matches_the_oracle(fa, d, bits):
    """fa_tq_codebook runs on the host: its levels (own quadrature and Lloyd
    iteration in the library) against the oracle's (incomplete-beta path)."""
    import numpy as np
    from oracle import turboquant as tq
    lv = fa.tq_codebook(d, bits).numpy()
    assert np.array_equal(lv, -lv[::-1])  # exactly antisymmetric
    assert np.abs(lv - tq.codebook(d, bits)).max() < 1e-7


def test_tq_rejects_bad_arguments(fa):
    buf = (ctypes.c_float * 16)()
    assert fa.lib.fa_tq_codebook(128, 4, None) == fa.FA_ERR_INVALID
    assert fa.lib.fa_tq_codebook(127, 4, ctypes.cast(buf, ctypes.c_void_p)) == fa.FA_ERR_INVALID
    assert fa.lib.fa_tq_codebook(128, 9, ctypes.cast(buf, ctypes.c_void_p)) == fa.FA_ERR_INVALID
    assert fa.lib.fa_tq_compress(None, None) == fa.FA_ERR_INVALID

    def comp(**kw):
        p = fa.TqCompressParams()
        p.x, p.x_dtype, p.rows, p.head_dim, p.bits = 0x1000, fa.FA_BF16, 10, 128, 4
        p.signs, p.levels, p.codes, p.norms = 0x2000, 0x3000, 0x4000, 0x5000
        for k, v in kw.items():
            setattr(p, k, v)
        return fa.lib.fa_tq_compress(ctypes.byref(p), None)

    assert comp(head_dim=96) == fa.FA_ERR_UNSUPPORTED
    assert comp(bits=5) == fa.FA_ERR_UNSUPPORTED
    assert comp(x_dtype=fa.FA_I8) == fa.FA_ERR_INVALID
    assert comp(codes=None) == fa.FA_ERR_INVALID
    assert comp(x=0x1008) == fa.FA_ERR_INVALID
    assert comp(rows=-1) == fa.FA_ERR_INVALID
    assert comp(rows=0, x=None) == fa.FA_OK

    def dec(**kw):
        p = fa.TqDecodeParams()
        p.q, p.k_codes, p.k_norms, p.v_codes, p.v_norms = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000
        p.k_levels, p.v_levels, p.signs, p.cache_seqlens, p.out = 0x6000, 0x7000, 0x8000, 0x9000, 0xa000
        p.batch, p.hq, p.hkv, p.head_dim, p.capacity, p.k_bits, p.v_bits = 2, 8, 2, 128, 4096, 4, 2
        p.softmax_scale = 0.1
        p.workspace = 0xb000
        p.workspace_bytes = fa.tq_decode_workspace_size(2, 8, 128, 4096)
        for k, v in kw.items():
            setattr(p, k, v)
        return fa.lib.fa_tq_attention_decode(ctypes.byref(p), None)

    assert fa.tq_decode_workspace_size(2, 8, 128, 4096) == 2 * 8 * 2 * 130 * 4  # two 2048-key splits
    assert dec(hq=6) == fa.FA_ERR_UNSUPPORTED          # group of 3
    assert dec(hq=7) == fa.FA_ERR_INVALID              # hq % hkv != 0
    assert dec(head_dim=96) == fa.FA_ERR_UNSUPPORTED
    assert dec(v_bits=1) == fa.FA_ERR_UNSUPPORTED
    assert dec(capacity=0) == fa.FA_ERR_INVALID
    assert dec(softmax_scale=float("inf")) == fa.FA_ERR_INVALID
    assert dec(signs=None) == fa.FA_ERR_INVALID
    assert dec(workspace_bytes=16) == fa.FA_ERR_WORKSPACE
    assert dec(n_epilogue=9) == fa.FA_ERR_INVALID
    assert dec(batch=0) == fa.FA_OK


def test_binding_rejects_tensors_smaller_than_their_sizes_say(fa):
    """The C ABI sees pointers and sizes only: the binding checks that every
    tensor has the shape the sizes imply (and int32 index tensors), so a
    kernel is never pointed past a tensor's end."""
    import torch
    F = FakeTensor
    bf, i32, f32 = torch.bfloat16, torch.int32, torch.float32
    q, k, o = F(0x1000, (4, 64, 128), bf), F(0x2000, (2, 64, 128), bf), F(0x3000, (4, 64, 128), bf)
    fa.fwd_params(q, k, k, o, hq=4, hkv=2)  # consistent: accepted
    with pytest.raises(ValueError):
        fa.fwd_params(q, F(0x2000, (1, 64, 128), bf), k, o, hq=4, hkv=2)  # fewer K planes than batch*hkv
    with pytest.raises(ValueError):
        fa.fwd_params(q, k, F(0x2000, (2, 63, 128), bf), o, hq=4, hkv=2)  # V shorter than K
    with pytest.raises(ValueError):
        fa.fwd_params(q, k, k, F(0x3000, (4, 64, 64), bf), hq=4, hkv=2)   # out narrower than q
    with pytest.raises(ValueError):
        fa.fwd_params(q, k, k, o, hq=3, hkv=1)                             # batch*hq does not divide
    with pytest.raises(ValueError):
        fa.fwd_params(q, F(0x2000, (2, 64, 128), torch.int8), k, o, hq=4, hkv=2,
                      k_scales=F(0x4000, (2, 32), f32))                     # scales of the wrong length
    cu = F(0x5000, (3,), i32)
    with pytest.raises(ValueError):
        fa.fwd_params(F(0x1000, (4, 100, 128), bf), F(0x2000, (2, 90, 128), bf), F(0x2000, (2, 90, 128), bf),
                      F(0x3000, (4, 100, 128), bf), hq=4, hkv=2, cu_seqlens_q=cu,
                      cu_seqlens_k=F(0x6000, (4,), i32), max_seqlen_q=60)  # B + 1 entries differ
    with pytest.raises(ValueError):
        fa.fwd_params(F(0x1000, (4, 100, 128), bf), F(0x2000, (2, 90, 128), bf), F(0x2000, (2, 90, 128), bf),
                      F(0x3000, (4, 100, 128), bf), hq=4, hkv=2, cu_seqlens_q=F(0x5000, (3,), torch.int64),
                      max_seqlen_q=60)                                      # int64 offsets
    lens = F(0x7000, (2,), i32)
    fa._cache_shapes(F(0x1000, (8, 128), bf), F(0x2000, (4, 256, 128), bf), F(0x2000, (4, 256, 128), bf),
                     None, None, lens, None, 4, 2)
    with pytest.raises(ValueError):  # cache planes for one sequence only
        fa._cache_shapes(F(0x1000, (8, 128), bf), F(0x2000, (2, 256, 128), bf), F(0x2000, (2, 256, 128), bf),
                         None, None, lens, None, 4, 2)
    with pytest.raises(ValueError):  # q rows for one sequence only
        fa._cache_shapes(F(0x1000, (4, 128), bf), None, None, None, None, lens, None, 4, 2)
    with pytest.raises(ValueError):  # float lengths
        fa._cache_shapes(F(0x1000, (8, 128), bf), None, None, None, None, F(0x7000, (2,), f32), None, 4, 2)
    with pytest.raises(ValueError):  # pools with the wrong KV head count
        fa._pool_shapes(F(0x2000, (16, 3, 64, 128), bf), F(0x2000, (16, 3, 64, 128), bf), None, None, 2, 128)
    with pytest.raises(ValueError):  # new rows for fewer sequences than cur_pos has
        fa._append_shapes(F(0x1000, (2, 128), bf), F(0x1000, (2, 128), bf), F(0x7000, (2,), i32), None, 2)
