"""Thin ctypes binding of libfa.so (include/fa.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  torch supplies device memory and the current
stream.  Importing this module loads ``lib/libfa.so`` and raises ImportError
when it is missing -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence, Tuple

import torch

# FA_LIBRARY may name another build of the same library (e.g. one compiled
# with different tuning constants); by default the in-tree build is loaded.
_LIB_PATH = os.environ.get("FA_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                                                          "libfa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libfa.so not built ({_LIB_PATH}); run __graft_entry__.build() "
                      "or python flashattention_attention_b200/build.py")
lib = ctypes.CDLL(_LIB_PATH)

# --- fa.h mirrors -------------------------------------------------------------
FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(6)
FA_F32, FA_BF16, FA_I8 = 0, 1, 2
FA_EPI_MUL, FA_EPI_ADD = 1, 2
FA_MAX_EPILOGUE = 8
FA_ACC_FIRST, FA_ACC_LAST = 1, 2


class EpiOp(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int32), ("value", ctypes.c_float)]


class FwdParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("q_dtype", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("seqlen_q", ctypes.c_int32), ("seqlen_k", ctypes.c_int32),
                ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
                ("total_q", ctypes.c_int32), ("total_k", ctypes.c_int32),
                ("max_seqlen_q", ctypes.c_int32), ("max_seqlen_k", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("window", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("n_epilogue", ctypes.c_int32),
                ("epilogue", EpiOp * FA_MAX_EPILOGUE)]


class DecodeParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("cache_seqlens", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("kv_dtype", ctypes.c_int32), ("batch", ctypes.c_int32), ("hq", ctypes.c_int32),
                ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32), ("window", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("split_keys", ctypes.c_int32),
                ("n_epilogue", ctypes.c_int32), ("epilogue", EpiOp * FA_MAX_EPILOGUE),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


class MergeParams(ctypes.Structure):
    _fields_ = [("o_acc", ctypes.c_void_p), ("lse_acc", ctypes.c_void_p), ("o_part", ctypes.c_void_p),
                ("part_dtype", ctypes.c_int32), ("lse_part", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("head_dim", ctypes.c_int32), ("out", ctypes.c_void_p), ("out_dtype", ctypes.c_int32),
                ("n_epilogue", ctypes.c_int32), ("epilogue", EpiOp * FA_MAX_EPILOGUE)]


class TqCompressParams(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_dtype", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("head_dim", ctypes.c_int32), ("bits", ctypes.c_int32), ("signs", ctypes.c_void_p),
                ("levels", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("norms", ctypes.c_void_p)]


class TqDecodeParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k_codes", ctypes.c_void_p), ("k_norms", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_norms", ctypes.c_void_p), ("k_levels", ctypes.c_void_p),
                ("v_levels", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("cache_seqlens", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("capacity", ctypes.c_int32), ("k_bits", ctypes.c_int32),
                ("v_bits", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("out", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("n_epilogue", ctypes.c_int32), ("epilogue", EpiOp * FA_MAX_EPILOGUE)]


class KvPages(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("max_pages", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class KvAppendParams(ctypes.Structure):
    _fields_ = [("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p), ("x_dtype", ctypes.c_int32),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("cache_dtype", ctypes.c_int32), ("cur_pos", ctypes.c_void_p),
                ("cache_seqlens", ctypes.c_void_p), ("batch", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("capacity", ctypes.c_int32)]


lib.fa_compress_kv.restype = ctypes.c_int
lib.fa_compress_kv.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int32,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
lib.fa_attention_fwd.restype = ctypes.c_int
lib.fa_attention_fwd.argtypes = [ctypes.POINTER(FwdParams), ctypes.c_void_p]
lib.fa_decode_workspace_size.restype = ctypes.c_size_t
lib.fa_decode_workspace_size.argtypes = [ctypes.c_int32] * 4
lib.fa_attention_decode.restype = ctypes.c_int
lib.fa_attention_decode.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_void_p]
lib.fa_attention_fwd_lse.restype = ctypes.c_int
lib.fa_attention_fwd_lse.argtypes = [ctypes.POINTER(FwdParams), ctypes.c_void_p, ctypes.c_void_p]
lib.fa_attention_fwd_acc.restype = ctypes.c_int
lib.fa_attention_fwd_acc.argtypes = [ctypes.POINTER(FwdParams), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                     ctypes.c_void_p]
lib.fa_attention_merge.restype = ctypes.c_int
lib.fa_attention_merge.argtypes = [ctypes.POINTER(MergeParams), ctypes.c_void_p]
lib.fa_attention_fwd_paged.restype = ctypes.c_int
lib.fa_attention_fwd_paged.argtypes = [ctypes.POINTER(FwdParams), ctypes.POINTER(KvPages), ctypes.c_void_p]
lib.fa_attention_decode_paged.restype = ctypes.c_int
lib.fa_attention_decode_paged.argtypes = [ctypes.POINTER(DecodeParams), ctypes.POINTER(KvPages), ctypes.c_void_p]
lib.fa_kv_append.restype = ctypes.c_int
lib.fa_kv_append.argtypes = [ctypes.POINTER(KvAppendParams), ctypes.c_void_p]
lib.fa_kv_append_paged.restype = ctypes.c_int
lib.fa_kv_append_paged.argtypes = [ctypes.POINTER(KvAppendParams), ctypes.POINTER(KvPages), ctypes.c_void_p]
lib.fa_tq_codebook.restype = ctypes.c_int
lib.fa_tq_codebook.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
lib.fa_tq_compress.restype = ctypes.c_int
lib.fa_tq_compress.argtypes = [ctypes.POINTER(TqCompressParams), ctypes.c_void_p]
lib.fa_tq_decode_workspace_size.restype = ctypes.c_size_t
lib.fa_tq_decode_workspace_size.argtypes = [ctypes.c_int32] * 4
lib.fa_tq_attention_decode.restype = ctypes.c_int
lib.fa_tq_attention_decode.argtypes = [ctypes.POINTER(TqDecodeParams), ctypes.c_void_p]
lib.fa_status_string.restype = ctypes.c_char_p
lib.fa_status_string.argtypes = [ctypes.c_int]
lib.fa_check_device_error.restype = ctypes.c_int
lib.fa_check_device_error.argtypes = [ctypes.c_void_p]
lib.fa_selftest_watchdog.restype = ctypes.c_int
lib.fa_selftest_watchdog.argtypes = [ctypes.c_uint64, ctypes.c_void_p]
lib.fa_kernel_variants_used.restype = ctypes.c_int32
lib.fa_kernel_variants_used.argtypes = []
lib.fa_kernel_launches.restype = ctypes.c_int64
lib.fa_kernel_launches.argtypes = []


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {lib.fa_status_string(status).decode()} (status {status})")
        self.status = status


def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


_DT = {torch.float32: FA_F32, torch.bfloat16: FA_BF16, torch.int8: FA_I8}


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _fill_epilogue(arr, epilogue: Sequence[Tuple[str, float]]) -> int:
    if len(epilogue) > FA_MAX_EPILOGUE:
        raise ValueError(f"at most {FA_MAX_EPILOGUE} epilogue ops")
    for i, (op, val) in enumerate(epilogue):
        name = op.lower() if isinstance(op, str) else op
        arr[i].op = {"mul": FA_EPI_MUL, "add": FA_EPI_ADD}.get(name, name)
        arr[i].value = float(val)
    return len(epilogue)


def _shape(t, want, name: str):
    """ValueError unless t has the shape `want` (None: any extent).  The C
    ABI sees only pointers and sizes, so a tensor smaller than its sizes say
    must be caught here, before a kernel reads past it."""
    got = tuple(t.shape)
    if len(got) != len(want) or any(w is not None and g != w for g, w in zip(got, want)):
        shown = tuple("*" if w is None else w for w in want)
        raise ValueError(f"{name} has shape {got}, expected {shown}")


def _int32(t, name: str):
    if t is not None and t.dtype != torch.int32:
        raise ValueError(f"{name} must be int32")


def _contig_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


# --- API ----------------------------------------------------------------------

def compress_kv(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                scales: Optional[torch.Tensor] = None, stream=None):
    """Per-row int8 codes + fp32 scales of x [..., d] (bf16 or fp32)."""
    _contig_cuda(x, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(lib.fa_compress_kv(_ptr(x), _DT[x.dtype], rows, d, _ptr(codes), _ptr(scales), _stream(stream)),
           "fa_compress_kv")
    return codes, scales


def fwd_params(q, k, v, out, *, hq, hkv, causal=False, window=0, scale=None, epilogue=(),
               k_scales=None, v_scales=None, cu_seqlens_q=None, cu_seqlens_k=None,
               max_seqlen_q=None, max_seqlen_k=None) -> FwdParams:
    d = q.shape[-1]
    if hq <= 0 or hkv <= 0:
        raise ValueError("hq and hkv must be positive")
    if cu_seqlens_q is None:
        if len(q.shape) != 3 or q.shape[0] % hq:
            raise ValueError(f"dense q must be [batch*hq, s_q, d]; got {tuple(q.shape)} with hq={hq}")
        _shape(k, (q.shape[0] // hq * hkv, None, d), "k")
    else:
        _int32(cu_seqlens_q, "cu_seqlens_q")
        _int32(cu_seqlens_k, "cu_seqlens_k")
        _shape(q, (hq, None, d), "q")
        _shape(k, (hkv, None, d), "k")
        if cu_seqlens_k is not None:
            _shape(cu_seqlens_k, (cu_seqlens_q.numel(),), "cu_seqlens_k")
    _shape(v, tuple(k.shape), "v")
    _shape(out, tuple(q.shape), "out")
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        if t is not None:
            _shape(t, tuple(k.shape[:2]), name)
    p = FwdParams()
    p.q, p.k, p.v, p.out = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    p.k_scales = None if k_scales is None else k_scales.data_ptr()
    p.v_scales = None if v_scales is None else v_scales.data_ptr()
    p.q_dtype, p.kv_dtype = _DT[q.dtype], _DT[k.dtype]
    p.hq, p.hkv, p.head_dim = hq, hkv, q.shape[-1]
    if cu_seqlens_q is None:
        p.batch = q.shape[0] // hq
        p.seqlen_q, p.seqlen_k = q.shape[1], k.shape[1]
    else:
        p.batch = cu_seqlens_q.numel() - 1
        p.cu_seqlens_q = cu_seqlens_q.data_ptr()
        p.cu_seqlens_k = None if cu_seqlens_k is None else cu_seqlens_k.data_ptr()
        p.total_q, p.total_k = q.shape[1], k.shape[1]
        p.max_seqlen_q = int(max_seqlen_q)
        p.max_seqlen_k = int(max_seqlen_k if max_seqlen_k is not None else max_seqlen_q)
    p.causal, p.window = int(bool(causal)), int(window)
    p.softmax_scale = float(scale if scale is not None else 1.0 / math.sqrt(q.shape[-1]))
    p.n_epilogue = _fill_epilogue(p.epilogue, epilogue)
    return p


def attention_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, hq: int, hkv: int,
                  causal: bool = False, window: int = 0, scale: Optional[float] = None,
                  epilogue: Sequence[Tuple[str, float]] = (), k_scales=None, v_scales=None,
                  cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None, max_seqlen_k=None,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Fused attention forward; layouts and semantics as fa_attention_fwd in fa.h."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _contig_cuda(t, name)
    if out is None:
        out = torch.empty_like(q)
    p = fwd_params(q, k, v, out, hq=hq, hkv=hkv, causal=causal, window=window, scale=scale,
                   epilogue=epilogue, k_scales=k_scales, v_scales=v_scales, cu_seqlens_q=cu_seqlens_q,
                   cu_seqlens_k=cu_seqlens_k, max_seqlen_q=max_seqlen_q, max_seqlen_k=max_seqlen_k)
    _check(lib.fa_attention_fwd(ctypes.byref(p), _stream(stream)), "fa_attention_fwd")
    return out


def attention_fwd_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, hq: int, hkv: int,
                      causal: bool = False, window: int = 0, scale: Optional[float] = None,
                      k_scales=None, v_scales=None, cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None,
                      max_seqlen_k=None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      stream=None):
    """Partial attention result (bf16 path): (out, lse) with lse the natural
    log-sum-exp of each row's scaled scores (-inf and out = 0 for a row
    without keys).  As fa_attention_fwd_lse in fa.h; no epilogue."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _contig_cuda(t, name)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    p = fwd_params(q, k, v, out, hq=hq, hkv=hkv, causal=causal, window=window, scale=scale, epilogue=(),
                   k_scales=k_scales, v_scales=v_scales, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                   max_seqlen_q=max_seqlen_q, max_seqlen_k=max_seqlen_k)
    _check(lib.fa_attention_fwd_lse(ctypes.byref(p), _ptr(lse), _stream(stream)), "fa_attention_fwd_lse")
    return out, lse


def attention_fwd_acc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o_acc: torch.Tensor,
                      lse_acc: torch.Tensor, *, hq: int, hkv: int, causal: bool = False, window: int = 0,
                      scale: Optional[float] = None, first: bool = False, last: bool = False,
                      out: Optional[torch.Tensor] = None, epilogue: Sequence[Tuple[str, float]] = (),
                      k_scales=None, v_scales=None, cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None,
                      max_seqlen_k=None, stream=None) -> Optional[torch.Tensor]:
    """Attention of q over these keys merged into the fp32 accumulator
    (o_acc [..., d] like q, lse_acc [...]) in the kernel's epilogue.  first:
    the accumulator is empty and not read; last: the merged rows go to `out`
    (allocated in q's dtype if None) after the epilogue and are returned,
    the accumulator is left as it was.  As fa_attention_fwd_acc in fa.h."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o_acc", o_acc), ("lse_acc", lse_acc)):
        _contig_cuda(t, name)
    if o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32:
        raise ValueError("the accumulator is fp32")
    if o_acc.shape != q.shape or lse_acc.shape != q.shape[:-1]:
        raise ValueError("o_acc must have q's shape and lse_acc q's shape without the last dim")
    if last and out is None:
        out = torch.empty_like(q)
    p = fwd_params(q, k, v, out if last else q, hq=hq, hkv=hkv, causal=causal, window=window, scale=scale,
                   epilogue=epilogue, k_scales=k_scales, v_scales=v_scales, cu_seqlens_q=cu_seqlens_q,
                   cu_seqlens_k=cu_seqlens_k, max_seqlen_q=max_seqlen_q, max_seqlen_k=max_seqlen_k)
    if not last:
        p.out = None
    flags = (FA_ACC_FIRST if first else 0) | (FA_ACC_LAST if last else 0)
    _check(lib.fa_attention_fwd_acc(ctypes.byref(p), _ptr(o_acc), _ptr(lse_acc), flags, _stream(stream)),
           "fa_attention_fwd_acc")
    return out if last else None


def attention_merge(o_acc: torch.Tensor, lse_acc: torch.Tensor, o_part: Optional[torch.Tensor] = None,
                    lse_part: Optional[torch.Tensor] = None, *, out: Optional[torch.Tensor] = None,
                    epilogue: Sequence[Tuple[str, float]] = (), stream=None) -> Optional[torch.Tensor]:
    """Fold the partial result (o_part, lse_part) into the fp32 accumulator
    (o_acc [..., d], lse_acc [...]) in place; with `out`, also write the
    merged rows after the epilogue.  As fa_attention_merge in fa.h."""
    _contig_cuda(o_acc, "o_acc")
    _contig_cuda(lse_acc, "lse_acc")
    _shape(lse_acc, tuple(o_acc.shape[:-1]), "lse_acc")
    if o_part is not None:
        _shape(o_part, tuple(o_acc.shape), "o_part")
        if lse_part is None:
            raise ValueError("lse_part is required with o_part")
        _shape(lse_part, tuple(lse_acc.shape), "lse_part")
    if out is not None:
        _shape(out, tuple(o_acc.shape), "out")
    p = MergeParams()
    p.o_acc, p.lse_acc = o_acc.data_ptr(), lse_acc.data_ptr()
    if o_part is not None:
        _contig_cuda(o_part, "o_part")
        _contig_cuda(lse_part, "lse_part")
        p.o_part, p.part_dtype, p.lse_part = o_part.data_ptr(), _DT[o_part.dtype], lse_part.data_ptr()
    p.head_dim = o_acc.shape[-1]
    p.rows = o_acc.numel() // p.head_dim
    if out is not None:
        _contig_cuda(out, "out")
        p.out, p.out_dtype = out.data_ptr(), _DT[out.dtype]
    p.n_epilogue = _fill_epilogue(p.epilogue, epilogue)
    _check(lib.fa_attention_merge(ctypes.byref(p), _stream(stream)), "fa_attention_merge")
    return out


def _pool_shapes(k_pages, v_pages, k_scales, v_scales, hkv: int, d: int):
    """Page pools [num_pages, hkv, page_size, d] and their scales
    [num_pages, hkv, page_size]."""
    _shape(k_pages, (None, hkv, None, d), "k_pages")
    _shape(v_pages, tuple(k_pages.shape), "v_pages")
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        if t is not None:
            _shape(t, tuple(k_pages.shape[:3]), name)


def _cache_shapes(q, k_cache, v_cache, k_scales, v_scales, cache_seqlens, out, hq: int, hkv: int):
    """Decode operands: q [batch*hq, d] or [batch*hq, 1, d], dense caches
    [batch*hkv, capacity, d] and scales [batch*hkv, capacity]."""
    _int32(cache_seqlens, "cache_seqlens")
    batch, d = cache_seqlens.numel(), q.shape[-1]
    if q.numel() != batch * hq * d:
        raise ValueError(f"q has shape {tuple(q.shape)}, expected batch*hq = {batch * hq} rows of {d}")
    if k_cache is not None:
        _shape(k_cache, (batch * hkv, None, d), "k_cache")
        _shape(v_cache, tuple(k_cache.shape), "v_cache")
        for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
            if t is not None:
                _shape(t, tuple(k_cache.shape[:2]), name)
    if out is not None:
        _shape(out, tuple(q.shape), "out")


def attention_fwd_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                        cu_seqlens_k: torch.Tensor, block_table: torch.Tensor, *, hq: int, hkv: int,
                        causal: bool = False, window: int = 0, scale: Optional[float] = None,
                        epilogue: Sequence[Tuple[str, float]] = (), k_scales=None, v_scales=None,
                        cu_seqlens_q=None, max_seqlen_q=None, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """Prefill over page pools k_pages/v_pages [num_pages, hkv, page_size, d]
    (int8 with scales [num_pages, hkv, page_size], or bf16) through a device
    int32 block_table [B, max_pages]; q dense [B*hq, s_q, d] or varlen
    [hq, total_q, d] with cu_seqlens_q.  As fa_attention_fwd_paged in fa.h."""
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages), ("cu_seqlens_k", cu_seqlens_k),
                    ("block_table", block_table)):
        _contig_cuda(t, name)
    d = q.shape[-1]
    _pool_shapes(k_pages, v_pages, k_scales, v_scales, hkv, d)
    for name, t in (("cu_seqlens_k", cu_seqlens_k), ("block_table", block_table), ("cu_seqlens_q", cu_seqlens_q)):
        _int32(t, name)
    batch = cu_seqlens_k.numel() - 1
    _shape(block_table, (batch, None), "block_table")
    if cu_seqlens_q is None:
        _shape(q, (batch * hq, None, d), "q")
    else:
        _shape(q, (hq, None, d), "q")
        _shape(cu_seqlens_q, (batch + 1,), "cu_seqlens_q")
    if out is not None:
        _shape(out, tuple(q.shape), "out")
    if out is None:
        out = torch.empty_like(q)
    p = FwdParams()
    p.q, p.k, p.v, p.out = q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), out.data_ptr()
    p.k_scales = None if k_scales is None else k_scales.data_ptr()
    p.v_scales = None if v_scales is None else v_scales.data_ptr()
    p.q_dtype, p.kv_dtype = _DT[q.dtype], _DT[k_pages.dtype]
    p.hq, p.hkv, p.head_dim = hq, hkv, q.shape[-1]
    p.batch = cu_seqlens_k.numel() - 1
    p.cu_seqlens_k = cu_seqlens_k.data_ptr()
    if cu_seqlens_q is None:
        p.seqlen_q = q.shape[1]
    else:
        p.cu_seqlens_q = cu_seqlens_q.data_ptr()
        p.total_q = q.shape[1]
        p.max_seqlen_q = int(max_seqlen_q)
    p.causal, p.window = int(bool(causal)), int(window)
    p.softmax_scale = float(scale if scale is not None else 1.0 / math.sqrt(q.shape[-1]))
    p.n_epilogue = _fill_epilogue(p.epilogue, epilogue)
    num_pages, _, page_size, _ = k_pages.shape
    pg = KvPages(block_table.data_ptr(), block_table.shape[1], page_size, num_pages)
    _check(lib.fa_attention_fwd_paged(ctypes.byref(p), ctypes.byref(pg), _stream(stream)), "fa_attention_fwd_paged")
    return out


def decode_workspace_size(batch: int, hq: int, capacity: int, head_dim: int) -> int:
    return int(lib.fa_decode_workspace_size(batch, hq, capacity, head_dim))


def decode_params(q, k_cache, v_cache, cache_seqlens, out, workspace, *, hq, hkv, k_scales=None,
                  v_scales=None, window=0, scale=None, epilogue=(), max_seqlen=0,
                  split_keys=0) -> DecodeParams:
    p = DecodeParams()
    p.q, p.k_cache, p.v_cache = q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr()
    p.k_scales = None if k_scales is None else k_scales.data_ptr()
    p.v_scales = None if v_scales is None else v_scales.data_ptr()
    p.cache_seqlens, p.out = cache_seqlens.data_ptr(), out.data_ptr()
    p.kv_dtype = _DT[k_cache.dtype]
    p.batch = cache_seqlens.numel()
    p.hq, p.hkv, p.head_dim, p.capacity = hq, hkv, q.shape[-1], k_cache.shape[1]
    p.max_seqlen, p.window = int(max_seqlen), int(window)
    p.softmax_scale = float(scale if scale is not None else 1.0 / math.sqrt(q.shape[-1]))
    p.split_keys = int(split_keys)
    p.n_epilogue = _fill_epilogue(p.epilogue, epilogue)
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = workspace.numel() * workspace.element_size()
    return p


def attention_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     cache_seqlens: torch.Tensor, *, hq: int, hkv: int, k_scales=None, v_scales=None,
                     window: int = 0, scale: Optional[float] = None,
                     epilogue: Sequence[Tuple[str, float]] = (), max_seqlen: int = 0,
                     split_keys: int = 0, workspace: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """s_q = 1 decode; q [B*hq, d] (or [B*hq, 1, d]) bf16, caches [B*hkv, cap, d]."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("cache_seqlens", cache_seqlens)):
        _contig_cuda(t, name)
    _cache_shapes(q, k_cache, v_cache, k_scales, v_scales, cache_seqlens, out, hq, hkv)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        nbytes = decode_workspace_size(cache_seqlens.numel(), hq, k_cache.shape[1], q.shape[-1])
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    p = decode_params(q, k_cache, v_cache, cache_seqlens, out, workspace, hq=hq, hkv=hkv,
                      k_scales=k_scales, v_scales=v_scales, window=window, scale=scale,
                      epilogue=epilogue, max_seqlen=max_seqlen, split_keys=split_keys)
    _check(lib.fa_attention_decode(ctypes.byref(p), _stream(stream)), "fa_attention_decode")
    return out


def attention_decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                           cache_seqlens: torch.Tensor, block_table: torch.Tensor, *, hq: int, hkv: int,
                           k_scales=None, v_scales=None, window: int = 0, scale: Optional[float] = None,
                           epilogue: Sequence[Tuple[str, float]] = (), max_seqlen: int = 0,
                           split_keys: int = 0, workspace: Optional[torch.Tensor] = None,
                           out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """s_q = 1 decode over page pools k_pages/v_pages [num_pages, hkv, page_size, d]
    (int8 with scales [num_pages, hkv, page_size], or bf16) through a device
    int32 block_table [B, max_pages]; as fa_attention_decode_paged in fa.h."""
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages), ("cache_seqlens", cache_seqlens),
                    ("block_table", block_table)):
        _contig_cuda(t, name)
    _pool_shapes(k_pages, v_pages, k_scales, v_scales, hkv, q.shape[-1])
    _cache_shapes(q, None, None, None, None, cache_seqlens, out, hq, hkv)
    _int32(block_table, "block_table")
    _shape(block_table, (cache_seqlens.numel(), None), "block_table")
    num_pages, _, page_size, d = k_pages.shape
    max_pages = block_table.shape[1]
    capacity = max_pages * page_size
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        nbytes = decode_workspace_size(cache_seqlens.numel(), hq, capacity, d)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    p = decode_params(q, k_pages, v_pages, cache_seqlens, out, workspace, hq=hq, hkv=hkv,
                      k_scales=k_scales, v_scales=v_scales, window=window, scale=scale,
                      epilogue=epilogue, max_seqlen=max_seqlen, split_keys=split_keys)
    p.capacity = capacity
    pg = KvPages(block_table.data_ptr(), max_pages, page_size, num_pages)
    _check(lib.fa_attention_decode_paged(ctypes.byref(p), ctypes.byref(pg), _stream(stream)),
           "fa_attention_decode_paged")
    return out


def kv_append(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              cur_pos: torch.Tensor, *, hkv: int, k_scales=None, v_scales=None, cache_seqlens=None,
              stream=None) -> None:
    """Write one new token per sequence (k_new, v_new [B*hkv, d]) into the
    caches [B*hkv, cap, d] at slot cur_pos[b] (device int32 [B]); an int8
    cache is quantised on the way in (scales required), a bf16 one stored
    as bf16.  cache_seqlens (device int32 [B]), if given, becomes cur_pos + 1.
    Layouts and semantics as fa_kv_append in fa.h."""
    _append_shapes(k_new, v_new, cur_pos, cache_seqlens, hkv)
    _shape(k_cache, (cur_pos.numel() * hkv, None, k_new.shape[-1]), "k_cache")
    _shape(v_cache, tuple(k_cache.shape), "v_cache")
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        if t is not None:
            _shape(t, tuple(k_cache.shape[:2]), name)
    p = _append_params(k_new, v_new, k_cache, v_cache, cur_pos, hkv, k_scales, v_scales, cache_seqlens)
    _check(lib.fa_kv_append(ctypes.byref(p), _stream(stream)), "fa_kv_append")


def kv_append_paged(k_new: torch.Tensor, v_new: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                    cur_pos: torch.Tensor, block_table: torch.Tensor, *, hkv: int, k_scales=None,
                    v_scales=None, cache_seqlens=None, stream=None) -> None:
    """kv_append into page pools [num_pages, hkv, page_size, d] through a
    device int32 block_table [B, max_pages]; as fa_kv_append_paged in fa.h."""
    _contig_cuda(block_table, "block_table")
    _append_shapes(k_new, v_new, cur_pos, cache_seqlens, hkv)
    _pool_shapes(k_pages, v_pages, k_scales, v_scales, hkv, k_new.shape[-1])
    _int32(block_table, "block_table")
    _shape(block_table, (cur_pos.numel(), None), "block_table")
    p = _append_params(k_new, v_new, k_pages, v_pages, cur_pos, hkv, k_scales, v_scales, cache_seqlens)
    num_pages, _, page_size, d = k_pages.shape
    p.head_dim, p.capacity = d, block_table.shape[1] * page_size
    pg = KvPages(block_table.data_ptr(), block_table.shape[1], page_size, num_pages)
    _check(lib.fa_kv_append_paged(ctypes.byref(p), ctypes.byref(pg), _stream(stream)), "fa_kv_append_paged")


def _append_shapes(k_new, v_new, cur_pos, cache_seqlens, hkv: int):
    _int32(cur_pos, "cur_pos")
    _int32(cache_seqlens, "cache_seqlens")
    _shape(k_new, (cur_pos.numel() * hkv, None), "k_new")
    _shape(v_new, tuple(k_new.shape), "v_new")
    if cache_seqlens is not None:
        _shape(cache_seqlens, (cur_pos.numel(),), "cache_seqlens")


def _append_params(k_new, v_new, k_cache, v_cache, cur_pos, hkv, k_scales, v_scales, cache_seqlens):
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("cur_pos", cur_pos)):
        _contig_cuda(t, name)
    p = KvAppendParams()
    p.k_new, p.v_new, p.x_dtype = k_new.data_ptr(), v_new.data_ptr(), _DT[k_new.dtype]
    p.k_cache, p.v_cache, p.cache_dtype = k_cache.data_ptr(), v_cache.data_ptr(), _DT[k_cache.dtype]
    p.k_scales = None if k_scales is None else k_scales.data_ptr()
    p.v_scales = None if v_scales is None else v_scales.data_ptr()
    p.cur_pos = cur_pos.data_ptr()
    p.cache_seqlens = None if cache_seqlens is None else cache_seqlens.data_ptr()
    p.batch, p.hkv = cur_pos.numel(), hkv
    p.head_dim, p.capacity = k_cache.shape[-1], k_cache.shape[1]
    return p


def check_device_error(stream=None) -> int:
    """Synchronise and return (then clear) the device status: FA_OK,
    FA_ERR_TIMEOUT, or FA_ERR_INVALID (a device-side argument was out of range)."""
    return int(lib.fa_check_device_error(_stream(stream)))


def selftest_watchdog(budget_cycles: int, stream=None) -> int:
    return int(lib.fa_selftest_watchdog(budget_cycles, _stream(stream)))


def kernel_variants_used() -> int:
    return int(lib.fa_kernel_variants_used())


def kernel_launches() -> int:
    return int(lib.fa_kernel_launches())


# --- TurboQuant KV cache -------------------------------------------------------

def tq_codebook(head_dim: int, bits: int) -> torch.Tensor:
    """The 2^bits Lloyd-Max levels (fp32, CPU) of the Beta(head_dim/2,
    head_dim/2) law in u-space.  As fa_tq_codebook in fa.h."""
    out = (ctypes.c_float * (1 << bits))()
    _check(lib.fa_tq_codebook(head_dim, bits, ctypes.cast(out, ctypes.c_void_p)), "fa_tq_codebook")
    return torch.tensor(list(out), dtype=torch.float32)


def tq_compress(x: torch.Tensor, signs: torch.Tensor, levels: torch.Tensor, bits: int,
                codes: Optional[torch.Tensor] = None, norms: Optional[torch.Tensor] = None, stream=None):
    """(codes uint8 [..., d*bits/8], norms fp32 [...]) of rows x [..., d]
    (bf16 or fp32).  signs / levels: fp32 CUDA tensors.  As fa_tq_compress."""
    for name, t in (("x", x), ("signs", signs), ("levels", levels)):
        _contig_cuda(t, name)
    d = x.shape[-1]
    _shape(signs, (d,), "signs")
    _shape(levels, (1 << bits,), "levels")
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (d * bits // 8,), dtype=torch.uint8, device=x.device)
    if norms is None:
        norms = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _shape(codes, tuple(x.shape[:-1]) + (d * bits // 8,), "codes")
    _shape(norms, tuple(x.shape[:-1]), "norms")
    p = TqCompressParams()
    p.x, p.x_dtype, p.rows, p.head_dim, p.bits = x.data_ptr(), _DT[x.dtype], x.numel() // d if d else 0, d, bits
    p.signs, p.levels, p.codes, p.norms = signs.data_ptr(), levels.data_ptr(), codes.data_ptr(), norms.data_ptr()
    _check(lib.fa_tq_compress(ctypes.byref(p), _stream(stream)), "fa_tq_compress")
    return codes, norms


def tq_decode_workspace_size(batch: int, hq: int, head_dim: int, capacity: int) -> int:
    return int(lib.fa_tq_decode_workspace_size(batch, hq, head_dim, capacity))


def tq_attention_decode(q: torch.Tensor, k_codes: torch.Tensor, k_norms: torch.Tensor, v_codes: torch.Tensor,
                        v_norms: torch.Tensor, cache_seqlens: torch.Tensor, *, hq: int, hkv: int, k_bits: int,
                        v_bits: int, k_levels: torch.Tensor, v_levels: torch.Tensor, signs: torch.Tensor,
                        scale: Optional[float] = None, epilogue: Sequence[Tuple[str, float]] = (),
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """One decode step over a TurboQuant cache: q [B*hq, d] (or [B*hq, 1, d])
    bf16, codes [B*hkv, capacity, d*bits/8], norms [B*hkv, capacity].  As
    fa_tq_attention_decode in fa.h."""
    for name, t in (("q", q), ("k_codes", k_codes), ("k_norms", k_norms), ("v_codes", v_codes),
                    ("v_norms", v_norms), ("cache_seqlens", cache_seqlens), ("k_levels", k_levels),
                    ("v_levels", v_levels), ("signs", signs)):
        _contig_cuda(t, name)
    d = q.shape[-1]
    batch = cache_seqlens.numel()
    _cache_shapes(q, None, None, None, None, cache_seqlens, out, hq, hkv)
    _shape(k_codes, (batch * hkv, None, d * k_bits // 8), "k_codes")
    cap = k_codes.shape[1]
    _shape(v_codes, (batch * hkv, cap, d * v_bits // 8), "v_codes")
    _shape(k_norms, (batch * hkv, cap), "k_norms")
    _shape(v_norms, (batch * hkv, cap), "v_norms")
    _shape(k_levels, (1 << k_bits,), "k_levels")
    _shape(v_levels, (1 << v_bits,), "v_levels")
    _shape(signs, (d,), "signs")
    if out is None:
        out = torch.empty_like(q)
    need = tq_decode_workspace_size(batch, hq, d, cap)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    p = TqDecodeParams()
    p.q, p.k_codes, p.k_norms, p.v_codes, p.v_norms = (q.data_ptr(), k_codes.data_ptr(), k_norms.data_ptr(),
                                                       v_codes.data_ptr(), v_norms.data_ptr())
    p.k_levels, p.v_levels, p.signs, p.cache_seqlens = (k_levels.data_ptr(), v_levels.data_ptr(), signs.data_ptr(),
                                                        cache_seqlens.data_ptr())
    p.batch, p.hq, p.hkv, p.head_dim, p.capacity, p.k_bits, p.v_bits = batch, hq, hkv, d, cap, k_bits, v_bits
    p.softmax_scale = float(scale if scale is not None else 1.0 / math.sqrt(d))
    p.out, p.workspace, p.workspace_bytes = out.data_ptr(), workspace.data_ptr(), workspace.numel()
    p.n_epilogue = _fill_epilogue(p.epilogue, epilogue)
    _check(lib.fa_tq_attention_decode(ctypes.byref(p), _stream(stream)), "fa_tq_attention_decode")
    return out

