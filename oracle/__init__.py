"""fp64 CPU oracle for the fused attention library -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU
baseline and reference arm) may import this package.  The product path never
does, and this package never imports the product package: the two share no
code.  The arithmetic lives in ``oracle.c`` (plain C, fp64, one materialised
score row at a time, two-pass softmax); this module only lays out arrays and
calls it.

Definitions followed:
  * attention: fkl_python PR #6 ("fkl.flash_attention: FA-2 forward with fused
    epilogue + compressed int8 KV cache"), Summary -- softmax(q k^T * scale) v
    with causal masking, layout (batch*heads, seq, head_dim), fused epilogue
    ops applied to the attention output; Foundry attention/README.md, "What it
    is (and is not)" -- the standard way, materialising the scores;
  * empty sliding-window band -> uniform softmax: SKaiNET-transformers PR #419,
    Summary;
  * GQA: SKaiNET-transformers PR #419, Summary (one task per GQA group);
    query head h reads KV head h // (hq // hkv);
  * int8 KV: fkl_python PR #6, Summary ("compress_kv(): per-token int8
    quantization (one fp32 scale/token)"); the oracle attends over the
    dequantised cache c * s;
  * cache append at a device-side slot: FlashRT QKV Cache RoPE, Kernels
    (the write slot comes from a device-side int32 position tensor): row
    b*hkv + g of the new token goes to slot cur_pos[b] of its cache row,
    compressed as compress_kv does; nothing else changes;
  * partial results over disjoint key sets and their merge: kernbench2
    commit message, ADR-0060 (long context: an online-softmax merge of the
    per-step (m, l, O) state at every ring step), written with the
    log-sum-exp lse = m + log l;
  * TurboQuant KV compression (rotation, Beta(d/2, d/2) Lloyd-Max codebook,
    bit-packing): the C attention library's README, "TurboQuant KV Cache
    Compression" -- in ``oracle/turboquant.py`` (numpy, fp64), pinned by
    ``tests/test_turboquant_oracle.py``.

Every function is pinned by ``tests/test_oracle.py`` against closed forms,
invariants, torch's fp64 scaled_dot_product_attention, pure-Python brute force
and the compression ratio the fkl page prints.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Iterable, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

EPI_MUL = 1
EPI_ADD = 2

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, IEEE arithmetic, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-std=c99", "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, dp, ip = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [dp, dp, dp, dp, i64, i64, i64, i64,
                                         i64, i64, dp, dp, i64, i64, dp, dp,
                                         ctypes.c_double, ctypes.c_int, i64,
                                         ctypes.c_int, ip, dp, i64, dp]
        lib.oracle_compress_kv.restype = None
        lib.oracle_compress_kv.argtypes = [dp, i64, i64, dp, dp]
        lib.oracle_dequantize.restype = None
        lib.oracle_dequantize.argtypes = [dp, dp, i64, i64, dp]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Any CPU array or torch tensor -> C-contiguous float64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _epilogue_arrays(epilogue: Sequence):
    ops, vals = [], []
    for op, val in epilogue:
        name = op.lower()
        if name == "mul":
            ops.append(EPI_MUL)
        elif name == "add":
            ops.append(EPI_ADD)
        else:
            raise ValueError(f"unknown epilogue op {op!r}")
        vals.append(float(val))
    return (np.asarray(ops if ops else [0], dtype=np.int32),
            np.asarray(vals if vals else [0.0], dtype=np.float64), len(ops))


def _run(q, k, v, out, batch, hq, hkv, d, qb, qh, q_start, q_len, kb, kh,
         k_start, k_len, scale, causal, window, epilogue, rows):
    ops, vals, n_epi = _epilogue_arrays(epilogue)
    q_start = np.ascontiguousarray(q_start, dtype=np.int64)
    q_len = np.ascontiguousarray(q_len, dtype=np.int64)
    k_start = np.ascontiguousarray(k_start, dtype=np.int64)
    k_len = np.ascontiguousarray(k_len, dtype=np.int64)
    if rows is not None:
        sel = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n_sel = sel.shape[0]
        if n_sel == 0:
            return
    else:
        sel = np.zeros((1, 3), dtype=np.int64)
        n_sel = 0
    rc = _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), batch, hq,
                                  hkv, d, qb, qh, _ptr(q_start), _ptr(q_len), kb, kh,
                                  _ptr(k_start), _ptr(k_len), float(scale), int(bool(causal)),
                                  int(window), n_epi, _ptr(ops), _ptr(vals), n_sel, _ptr(sel))
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments")


def attention(q, k, v, *, hq: int, hkv: int, causal: bool = False, window: int = 0,
              scale: Optional[float] = None, epilogue: Sequence = (),
              cu_seqlens_q=None, cu_seqlens_k=None,
              rows: Optional[Iterable] = None) -> np.ndarray:
    """fp64 attention forward.

    Dense layout: q [B*hq, s_q, d], k/v [B*hkv, s_k, d].
    Varlen layout (cu_seqlens_q/k given, int [B+1]): q [hq, total_q, d],
    k/v [hkv, total_k, d]; sequence b owns rows cu[b]:cu[b+1].
    ``rows``: optional (b, h, i) triples; only those output rows are computed
    (the rest of the returned array is zero).
    Returns float64 of q's shape.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros_like(q)
    if cu_seqlens_q is None:
        batch = q.shape[0] // hq
        s_q, s_k = q.shape[1], k.shape[1]
        if k.shape[0] != batch * hkv or v.shape != k.shape:
            raise ValueError("dense layout: k/v must be [B*hkv, s_k, d]")
        _run(q, k, v, out, batch, hq, hkv, d, hq * s_q, s_q, np.zeros(batch),
             np.full(batch, s_q), hkv * s_k, s_k, np.zeros(batch), np.full(batch, s_k),
             scale, causal, window, epilogue, rows)
    else:
        cq = np.asarray(cu_seqlens_q, dtype=np.int64)
        ck = np.asarray(cu_seqlens_k if cu_seqlens_k is not None else cu_seqlens_q, dtype=np.int64)
        batch = cq.shape[0] - 1
        tq, tk = q.shape[1], k.shape[1]
        _run(q, k, v, out, batch, hq, hkv, d, 0, tq, cq[:-1], np.diff(cq), 0, tk,
             ck[:-1], np.diff(ck), scale, causal, window, epilogue, rows)
    return out


def attention_lse(q, k, v, *, hq: int, hkv: int, causal: bool = False, window: int = 0,
                  scale: Optional[float] = None, cu_seqlens_q=None, cu_seqlens_k=None):
    """Partial attention result: (o, lse) in fp64, numpy, one (sequence,
    head) score matrix at a time.  lse[row] = log of the sum of exp(scale *
    q.k) over the row's visible keys, o[row] the softmax-weighted mean of
    their values; a row with no visible key has lse = -inf and o = 0 (it
    weighs nothing when partial results over disjoint key sets are merged).
    Layouts, masks and the GQA map as attention(); no epilogue.
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    d = qf.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    group = hq // hkv
    o = np.zeros_like(qf)
    lse = np.full(qf.shape[:-1], -np.inf)
    if cu_seqlens_q is None:
        batch = qf.shape[0] // hq
        spans = [((b * hq, 0, qf.shape[1]), (b * hkv, 0, kf.shape[1])) for b in range(batch)]
    else:
        cq, ck = np.asarray(cu_seqlens_q), np.asarray(cu_seqlens_k)
        spans = [((0, int(cq[b]), int(cq[b + 1] - cq[b])), (0, int(ck[b]), int(ck[b + 1] - ck[b])))
                 for b in range(len(cq) - 1)]
    for (qp, q0, s_q), (kp, k0, s_k) in spans:
        i = np.arange(s_q)[:, None]
        j = np.arange(s_k)[None, :]
        pos = i + s_k - s_q
        vis = np.ones((s_q, s_k), dtype=bool)
        if causal:
            vis &= j <= pos
        if window > 0:
            vis &= j > pos - window
        for h in range(hq):
            g = h // group
            qs = qf[qp + h, q0:q0 + s_q] if cu_seqlens_q is None else qf[h, q0:q0 + s_q]
            ks = kf[kp + g, k0:k0 + s_k] if cu_seqlens_q is None else kf[g, k0:k0 + s_k]
            vs = vf[kp + g, k0:k0 + s_k] if cu_seqlens_q is None else vf[g, k0:k0 + s_k]
            x = np.where(vis, scale * (qs @ ks.T), -np.inf)
            m = x.max(axis=1, initial=-np.inf)
            has = np.isfinite(m)
            w = np.exp(x - np.where(has, m, 0.0)[:, None])
            l = w.sum(axis=1)
            rows = np.where(has)[0]
            out = np.zeros((s_q, d))
            out[rows] = (w[rows] @ vs) / l[rows, None]
            ls = np.full(s_q, -np.inf)
            ls[rows] = m[rows] + np.log(l[rows])
            if cu_seqlens_q is None:
                o[qp + h, q0:q0 + s_q] = out
                lse[qp + h, q0:q0 + s_q] = ls
            else:
                o[h, q0:q0 + s_q] = out
                lse[h, q0:q0 + s_q] = ls
    return o, lse


def merge(o_a, lse_a, o_b, lse_b):
    """The partial result over the union of two disjoint key sets:
    lse = log(e^lse_a + e^lse_b), o = o_a e^(lse_a - lse) + o_b e^(lse_b - lse)
    (fp64; rows empty in both stay o = 0, lse = -inf)."""
    oa, ob = _f64(o_a), _f64(o_b)
    la, lb = np.asarray(lse_a, dtype=np.float64), np.asarray(lse_b, dtype=np.float64)
    lse = np.logaddexp(la, lb)
    fin = np.isfinite(lse)
    safe = np.where(fin, lse, 0.0)  # rows empty on both sides get weight 0
    wa = np.where(fin, np.exp(la - safe), 0.0)
    wb = np.where(fin, np.exp(lb - safe), 0.0)
    return oa * wa[..., None] + ob * wb[..., None], lse


def decode(q, k_cache, v_cache, cache_seqlens, *, hq: int, hkv: int, window: int = 0,
           scale: Optional[float] = None, epilogue: Sequence = (),
           rows: Optional[Iterable] = None) -> np.ndarray:
    """fp64 single-query decode against a per-sequence KV cache.

    q [B*hq, 1, d]; k_cache/v_cache [B*hkv, cap, d] (already dequantised for
    an int8 cache); cache_seqlens [B]: keys 0..L_b-1 of sequence b are
    attended (the current token is already in the cache).  With s_q = 1 the
    bottom-right causal position is L_b - 1, so every cached key is visible
    (a window W keeps the last W).
    """
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    lens = np.asarray(cache_seqlens, dtype=np.int64)
    batch = lens.shape[0]
    cap = kc.shape[1]
    out = np.zeros_like(q)
    _run(q, kc, vc, out, batch, hq, hkv, d, hq, 1, np.zeros(batch), np.ones(batch),
         hkv * cap, cap, np.zeros(batch), lens, scale, True, window, epilogue, rows)
    return out


def compress_kv(x):
    """Per-row int8 codes + fp32 scales, in IEEE fp32 (bit-exact reference).

    x: [..., d] (fp32 or bf16; bf16 widens to fp32 exactly).  Returns
    (codes int8 of x's shape, scales float32 of x.shape[:-1]).
    """
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    d = x32.shape[-1]
    rows = x32.size // d if d else 0
    codes = np.zeros(x32.shape, dtype=np.int8)
    scales = np.zeros(x32.shape[:-1], dtype=np.float32)
    if rows:
        _load().oracle_compress_kv(_ptr(x32), rows, d, _ptr(codes), _ptr(scales))
    return codes, scales


def kv_append(cache, scales, new, cur_pos, hkv: int, seqlens=None):
    """The cache after appending one token per sequence (plain definition).

    cache: [B*hkv, cap, d] int8 codes (with scales [B*hkv, cap] fp32) or a
    float cache (scales None, the row stored as given); new: [B*hkv, d];
    cur_pos: [B] slots.  Returns (cache, scales, seqlens) as new arrays: row
    u = b*hkv + g of `new` written at [u, cur_pos[b]] (compressed by
    compress_kv for an int8 cache), seqlens[b] = cur_pos[b] + 1.  A slot
    outside [0, cap) leaves sequence b untouched (and its seqlens entry).
    """
    def host(a):
        return a.detach().cpu().numpy() if hasattr(a, "detach") else np.asarray(a)
    c = host(cache).copy()
    sc = None if scales is None else host(scales).copy()
    x = host(new) if not hasattr(new, "detach") else new.detach().cpu().float().numpy()
    pos = np.asarray(host(cur_pos), dtype=np.int64)
    sl = None if seqlens is None else np.asarray(host(seqlens), dtype=np.int32).copy()
    cap = c.shape[1]
    for u in range(c.shape[0]):
        b = u // hkv
        p = int(pos[b])
        if p < 0 or p >= cap:
            continue
        if sc is not None:
            codes, s = compress_kv(np.asarray(x[u], dtype=np.float32)[None, :])
            c[u, p] = codes[0]
            sc[u, p] = s[0]
        else:
            c[u, p] = x[u]
        if sl is not None:
            sl[b] = p + 1
    return c, sc, sl


def dequantize(codes, scales) -> np.ndarray:
    """c * s in fp64 (exact)."""
    if hasattr(codes, "detach"):
        codes = codes.detach().cpu().numpy()
    if hasattr(scales, "detach"):
        scales = scales.detach().cpu().numpy()
    c = np.ascontiguousarray(codes, dtype=np.int8)
    s = np.ascontiguousarray(scales, dtype=np.float32)
    d = c.shape[-1]
    out = np.zeros(c.shape, dtype=np.float64)
    rows = c.size // d if d else 0
    if rows:
        _load().oracle_dequantize(_ptr(c), _ptr(s), rows, d, _ptr(out))
    return out
