"""Pins for the fp64 oracle, checked against things other than itself.

Each pin cites the passage it follows.  The attention oracle is pinned by:
torch's fp64 scaled_dot_product_attention with an explicit boolean mask built
from tril/triu diagonals (a library routine); pure-Python brute force on tiny
inputs that normalises without a max shift; closed forms (Q = 0, a single
key, causal row 0, empty band); invariants (key permutation, key shift,
linearity in V); and special-case reductions (GQA, varlen, window, decode).
The quantiser is pinned by exact half-way rounding against numpy.rint, by its
invariants, and by the compression ratio printed on the fkl page.
``test_mutants_are_caught`` plants plausible mistakes in a copy of the C
oracle and checks that the pins reject every one of them.
"""
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from flashattention_attention_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers (test side)

def band_mask(s_q, s_k, causal, window):
    """Boolean [s_q, s_k] visibility mask from tril/triu diagonals.
    Bottom-right alignment: query i sits at key position i + s_k - s_q."""
    m = torch.ones(s_q, s_k, dtype=torch.bool)
    off = s_k - s_q
    if causal:
        m = torch.tril(m, diagonal=off)
    if window > 0:
        m = m & torch.triu(torch.ones(s_q, s_k, dtype=torch.bool), diagonal=off - window + 1)
    return m


def sdpa_reference(q, k, v, hq, hkv, causal, window, scale):
    """torch fp64 SDPA over dense [B*h, s, d] inputs, GQA via repeat_interleave."""
    B = q.shape[0] // hq
    s_q, s_k, d = q.shape[1], k.shape[1], q.shape[2]
    qt = torch.as_tensor(q, dtype=torch.float64).reshape(B, hq, s_q, d)
    kt = torch.as_tensor(k, dtype=torch.float64).reshape(B, hkv, s_k, d)
    vt = torch.as_tensor(v, dtype=torch.float64).reshape(B, hkv, s_k, d)
    kt = kt.repeat_interleave(hq // hkv, dim=1)
    vt = vt.repeat_interleave(hq // hkv, dim=1)
    mask = band_mask(s_q, s_k, causal, window)
    out = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return out.reshape(B * hq, s_q, d).numpy(), mask.numpy()


def rand(rng, *shape):
    return rng.standard_normal(shape)


# ----------------------------------------------------------------------------
# pins, written as plain functions so the mutation test can rerun them

SDPA_CASES = [
    # B, hq, hkv, s_q, s_k, d, causal, window
    (1, 1, 1, 7, 7, 8, False, 0),
    (2, 4, 2, 9, 9, 16, True, 0),
    (1, 8, 2, 5, 13, 8, True, 0),       # s_q < s_k: bottom-right causal
    (2, 2, 1, 11, 11, 4, True, 3),      # causal + window
    (1, 3, 3, 6, 10, 8, False, 4),      # window without causal (left bound only)
    (1, 4, 1, 16, 16, 32, True, 16),    # window == s: same as causal
    (1, 2, 2, 12, 5, 8, True, 0),       # s_q > s_k: leading rows empty (excluded here)
]


def pin_sdpa():
    """fkl_python PR #6, Summary: softmax(q k^T) v, causal flag, (batch*heads,
    seq, head_dim) layout; GQA per SKaiNET-transformers PR #419, Summary."""
    rng = np.random.default_rng(1)
    for (B, hq, hkv, s_q, s_k, d, causal, window) in SDPA_CASES:
        q, k, v = rand(rng, B * hq, s_q, d), rand(rng, B * hkv, s_k, d), rand(rng, B * hkv, s_k, d)
        scale = 0.37 + 0.1 * d ** -0.5
        got = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=causal, window=window, scale=scale)
        ref, mask = sdpa_reference(q, k, v, hq, hkv, causal, window, scale)
        rows = mask.any(axis=1)
        assert rows.any()
        np.testing.assert_allclose(got[:, rows], ref[:, rows], rtol=0, atol=1e-12)


def brute_force(q, k, v, hq, hkv, causal, window, scale):
    """Pure-Python loops; weights exp(x_j) / sum exp(x_l) with no max shift."""
    B = len(q) // hq
    G = hq // hkv
    out = []
    for b in range(B):
        for h in range(hq):
            qq = q[b * hq + h]
            kk = k[b * hkv + h // G]
            vv = v[b * hkv + h // G]
            s_q, s_k, d = len(qq), len(kk), len(qq[0])
            rows = []
            for i in range(s_q):
                vis = []
                for j in range(s_k):
                    p = i + s_k - s_q
                    ok = (not causal or j <= p) and (window <= 0 or j > p - window)
                    if ok:
                        vis.append(j)
                if vis:
                    e = {j: math.exp(scale * sum(qq[i][c] * kk[j][c] for c in range(d))) for j in vis}
                    z = sum(e.values())
                    rows.append([sum(e[j] * vv[j][c] for j in vis) / z for c in range(d)])
                else:
                    rows.append([sum(vv[j][c] for j in range(s_k)) / s_k if s_k else 0.0
                                 for c in range(d)])
            out.append(rows)
    return np.array(out)


def pin_brute_force():
    rng = np.random.default_rng(2)
    for (B, hq, hkv, s_q, s_k, d, causal, window) in [(1, 2, 1, 3, 4, 3, True, 0),
                                                       (2, 2, 2, 4, 4, 2, False, 0),
                                                       (1, 4, 2, 4, 3, 4, True, 2),
                                                       (1, 1, 1, 4, 2, 3, True, 0)]:
        q, k, v = rand(rng, B * hq, s_q, d), rand(rng, B * hkv, s_k, d), rand(rng, B * hkv, s_k, d)
        got = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=causal, window=window, scale=0.7)
        ref = brute_force(q.tolist(), k.tolist(), v.tolist(), hq, hkv, causal, window, 0.7)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)


def pin_zero_query():
    """Q = 0 makes every visible score equal: the output is the mean of V over
    the band (closed form)."""
    rng = np.random.default_rng(3)
    s_q, s_k, d, W = 9, 12, 8, 4
    v = rand(rng, 1, s_k, d)
    k = rand(rng, 1, s_k, d)
    q = np.zeros((1, s_q, d))
    got = oracle.attention(q, k, v, hq=1, hkv=1, causal=True, window=W)
    mask = band_mask(s_q, s_k, True, W).numpy()
    for i in range(s_q):
        np.testing.assert_allclose(got[0, i], v[0, mask[i]].mean(axis=0), rtol=0, atol=1e-14)


def pin_single_key_and_row0():
    """One key: o = v_0 exactly.  Causal row 0 of a square problem: o = v_0."""
    rng = np.random.default_rng(4)
    q, k, v = rand(rng, 3, 5, 16), rand(rng, 3, 1, 16), rand(rng, 3, 1, 16)
    got = oracle.attention(q, k, v, hq=3, hkv=3, causal=False)
    assert np.array_equal(got, np.broadcast_to(v, got.shape))
    q, k, v = rand(rng, 2, 6, 16), rand(rng, 2, 6, 16), rand(rng, 2, 6, 16)
    got = oracle.attention(q, k, v, hq=2, hkv=2, causal=True)
    assert np.array_equal(got[:, 0], v[:, 0])


def pin_empty_band():
    """SKaiNET-transformers PR #419, Summary: a row whose sliding-window band
    holds no key falls back to the uniform softmax, i.e. the mean of all V rows.  Here s_q > s_k
    under causal masking leaves the first s_q - s_k rows with no visible key."""
    rng = np.random.default_rng(5)
    s_q, s_k, d = 10, 4, 8
    q, k, v = rand(rng, 2, s_q, d), rand(rng, 2, s_k, d), rand(rng, 2, s_k, d)
    got = oracle.attention(q, k, v, hq=2, hkv=2, causal=True)
    for h in range(2):
        for i in range(s_q - s_k):
            np.testing.assert_allclose(got[h, i], v[h].mean(axis=0), rtol=0, atol=1e-15)
    # decode against an empty cache gives zeros
    out = oracle.decode(rand(rng, 2, 1, d), np.zeros((1, 8, d)), np.ones((1, 8, d)), [0],
                        hq=2, hkv=1)
    assert not out.any()


def pin_invariants():
    """Non-causal attention is invariant under a joint permutation of the
    (k, v) rows; adding one vector to every key shifts each row's scores by a
    constant and leaves the output unchanged; the output is linear in V."""
    rng = np.random.default_rng(6)
    q, k, v = rand(rng, 2, 7, 8), rand(rng, 2, 11, 8), rand(rng, 2, 11, 8)
    base = oracle.attention(q, k, v, hq=2, hkv=2)
    perm = rng.permutation(11)
    np.testing.assert_allclose(oracle.attention(q, k[:, perm], v[:, perm], hq=2, hkv=2), base,
                               rtol=0, atol=1e-13)
    shifted = oracle.attention(q, k + rand(rng, 1, 1, 8), v, hq=2, hkv=2)
    np.testing.assert_allclose(shifted, base, rtol=0, atol=1e-12)
    v2 = rand(rng, 2, 11, 8)
    lin = oracle.attention(q, k, 2.0 * v - 3.0 * v2, hq=2, hkv=2, causal=True, window=5)
    ref = (2.0 * oracle.attention(q, k, v, hq=2, hkv=2, causal=True, window=5)
           - 3.0 * oracle.attention(q, k, v2, hq=2, hkv=2, causal=True, window=5))
    np.testing.assert_allclose(lin, ref, rtol=0, atol=1e-12)


def pin_reductions():
    """GQA == MHA with KV heads repeated; varlen == per-sequence dense calls;
    a window >= s_k == plain causal; decode == the last row of a prefill."""
    rng = np.random.default_rng(7)
    hq, hkv, s, d = 8, 2, 10, 8
    q, k, v = rand(rng, hq, s, d), rand(rng, hkv, s, d), rand(rng, hkv, s, d)
    gqa = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=True)
    mha = oracle.attention(q, np.repeat(k, hq // hkv, axis=0), np.repeat(v, hq // hkv, axis=0),
                           hq=hq, hkv=hq, causal=True)
    assert np.array_equal(gqa, mha)

    lengths = [5, 1, 9, 3]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    tot = cu[-1]
    qv, kv, vv = rand(rng, hq, tot, d), rand(rng, hkv, tot, d), rand(rng, hkv, tot, d)
    var = oracle.attention(qv, kv, vv, hq=hq, hkv=hkv, causal=True, window=3, cu_seqlens_q=cu)
    for b in range(len(lengths)):
        sl = slice(cu[b], cu[b + 1])
        dense = oracle.attention(qv[:, sl], kv[:, sl], vv[:, sl], hq=hq, hkv=hkv, causal=True,
                                 window=3)
        assert np.array_equal(var[:, sl], dense)

    wide = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=True, window=s)
    assert np.array_equal(wide, gqa)

    L = [10, 6]
    cap = 12
    kc, vc = np.zeros((2 * hkv, cap, d)), np.zeros((2 * hkv, cap, d))
    qd = rand(rng, 2 * hq, 1, d)
    for b in range(2):
        kc[b * hkv:(b + 1) * hkv, :L[b]] = rand(rng, hkv, L[b], d)
        vc[b * hkv:(b + 1) * hkv, :L[b]] = rand(rng, hkv, L[b], d)
    dec = oracle.decode(qd, kc, vc, L, hq=hq, hkv=hkv)
    for b in range(2):
        qp = np.concatenate([rand(rng, hq, L[b] - 1, d), qd[b * hq:(b + 1) * hq]], axis=1)
        pre = oracle.attention(qp, kc[b * hkv:(b + 1) * hkv, :L[b]], vc[b * hkv:(b + 1) * hkv, :L[b]],
                               hq=hq, hkv=hkv, causal=True)
        np.testing.assert_allclose(dec[b * hq:(b + 1) * hq, 0], pre[:, -1], rtol=0, atol=1e-15)


def pin_epilogue():
    """fkl_python PR #6, Summary: epilogue=[Mul(2.0), Add(0.5)] runs on the
    attention output, in order (Mul first, then Add)."""
    rng = np.random.default_rng(8)
    q, k, v = rand(rng, 2, 6, 8), rand(rng, 2, 6, 8), rand(rng, 2, 6, 8)
    o = oracle.attention(q, k, v, hq=2, hkv=2, causal=True)
    ma = oracle.attention(q, k, v, hq=2, hkv=2, causal=True, epilogue=[("mul", 2.0), ("add", 0.5)])
    am = oracle.attention(q, k, v, hq=2, hkv=2, causal=True, epilogue=[("add", 0.5), ("mul", 2.0)])
    np.testing.assert_allclose(ma, 2.0 * o + 0.5, rtol=0, atol=1e-15)
    np.testing.assert_allclose(am, 2.0 * (o + 0.5), rtol=0, atol=1e-15)


def pin_row_selection():
    """Computing a subset of rows gives those rows of the full result."""
    rng = np.random.default_rng(9)
    q, k, v = rand(rng, 4, 9, 8), rand(rng, 2, 9, 8), rand(rng, 2, 9, 8)
    full = oracle.attention(q, k, v, hq=2, hkv=1, causal=True, window=4)
    sel = [(0, 1, 3), (1, 0, 8), (1, 1, 0)]
    part = oracle.attention(q, k, v, hq=2, hkv=1, causal=True, window=4, rows=sel)
    for (b, h, i) in sel:
        assert np.array_equal(part[b * 2 + h, i], full[b * 2 + h, i])


def pin_quantiser_rounding():
    """fkl_python PR #6, Summary: per-token int8 with one fp32 scale.  A row
    whose max |x| is 127 has scale exactly 1, so its codes are x rounded half
    to even, which numpy.rint computes."""
    halves = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 126.5, -126.5, 0.49999997, 2.5000002],
                      dtype=np.float32)
    row = np.concatenate([halves, np.array([127.0, -3.25, 64.75], dtype=np.float32)])
    codes, scales = oracle.compress_kv(row[None, :])
    assert scales[0] == np.float32(1.0)
    assert np.array_equal(codes[0].astype(np.int64), np.rint(row).astype(np.int64))


def pin_quantiser_invariants():
    """|c| <= 127; each row's max-|x| element maps to +-127; |x - c s| <= s/2
    (to rounding); an all-zero row has scale 0 and zero codes."""
    rng = np.random.default_rng(10)
    x = rng.standard_normal((64, 128)).astype(np.float32) * rng.uniform(1e-3, 1e3, (64, 1)).astype(np.float32)
    x[5] = 0.0
    codes, scales = oracle.compress_kv(x)
    assert np.abs(codes.astype(np.int32)).max() <= 127
    assert scales[5] == 0 and not codes[5].any()
    for r in range(64):
        if r == 5:
            continue
        a = np.argmax(np.abs(x[r]))
        assert abs(int(codes[r, a])) == 127 and np.sign(codes[r, a]) == np.sign(x[r, a])
        err = np.abs(x[r].astype(np.float64) - codes[r].astype(np.float64) * float(scales[r]))
        assert err.max() <= 0.5 * float(scales[r]) * (1 + 1e-5)
        np.testing.assert_allclose(float(scales[r]), np.abs(x[r]).max() / 127.0, rtol=1e-7)


def pin_compression_ratio():
    """fkl_python PR #6, Verification: the compressed cache is 3.76 times
    smaller than fp32, against a gate of 3.5.
    Measured from the oracle's output buffers at head_dim 64 against fp32."""
    with open(os.path.join(GOLDEN, "compression_ratio.txt")) as f:
        fields = dict(line.split("=", 1) for line in f.read().split("\n")
                      if "=" in line and not line.startswith("#"))
    d = int(fields["head_dim"])
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1000, d)).astype(np.float32)
    codes, scales = oracle.compress_kv(x)
    ratio = x.nbytes / (codes.nbytes + scales.nbytes)
    assert f"{ratio:.2f}" == fields["ratio"].strip()
    assert ratio > float(fields["gate"])
    assert abs(ratio - d / (d / 4 + 1)) < 1e-12


def pin_int8_end_to_end():
    """fkl_python PR #6, Summary and Verification: attention over the int8
    cache stays within ~1e-3-order error of the unquantised result (the page
    measured 3.9e-3).  A loose bound: the error is nonzero and below 2e-2."""
    rng = np.random.default_rng(12)
    q, k, v = rand(rng, 4, 64, 64), rand(rng, 4, 64, 64), rand(rng, 4, 64, 64)
    exact = oracle.attention(q, k, v, hq=4, hkv=4, causal=True)
    kq = oracle.dequantize(*oracle.compress_kv(k.astype(np.float32)))
    vq = oracle.dequantize(*oracle.compress_kv(v.astype(np.float32)))
    approx = oracle.attention(q, kq, vq, hq=4, hkv=4, causal=True)
    err = np.abs(approx - exact).max()
    assert 1e-5 < err < 2e-2


ALL_PINS = [pin_sdpa, pin_brute_force, pin_zero_query, pin_single_key_and_row0, pin_empty_band,
            pin_invariants, pin_reductions, pin_epilogue, pin_row_selection,
            pin_quantiser_rounding, pin_quantiser_invariants, pin_compression_ratio,
            pin_int8_end_to_end]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# ----------------------------------------------------------------------------
# mutation test: plausible mistakes planted in a copy of the C oracle

MUTANTS = {
    "dropped_scale": ("score[j] = scale * dot;", "score[j] = dot;"),
    "causal_top_left": ("int64_t p = i + s_k - s_q;", "int64_t p = i;"),
    "causal_strict": ("if (causal && j > p) return 0;", "if (causal && j >= p) return 0;"),
    "window_off_by_one": ("if (window > 0 && j <= p - window) return 0;",
                          "if (window > 0 && j < p - window) return 0;"),
    "gqa_modulo": ("int64_t g = h / group;", "int64_t g = h % hkv;"),
    "empty_band_zero": ("for (c = 0; c < d; ++c) out_row[c] /= (double)s_k;",
                        "for (c = 0; c < d; ++c) out_row[c] = 0.0;"),
    "no_max_shift_sign": ("score[j] = exp(score[j] - m);", "score[j] = exp(m - score[j]);"),
    "transposed_kv": ("out_row[c] += w * v_rows[j * kv_row_stride + c];",
                      "out_row[c] += w * k_rows[j * kv_row_stride + c];"),
    "epilogue_reversed": ("for (int e = 0; e < n_epi; ++e) {", "for (int e = n_epi - 1; e >= 0; --e) {"),
    "quant_truncate": ("float t = nearbyintf(xr[c] / s);", "float t = truncf(xr[c] / s);"),
    "quant_scale_128": ("float s = amax / 127.0f;", "float s = amax / 128.0f;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name, monkeypatch):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    tmp = tempfile.mkdtemp()
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = os.path.join(tmp, "libmutant.so")
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                               "-std=c99", "-shared", "-fPIC", "-o", lib, path, "-lm"])
        monkeypatch.setattr(oracle, "_LIB", lib)
        monkeypatch.setattr(oracle, "_SRC", path)
        monkeypatch.setattr(oracle, "_lib", None)
        caught = []
        for pin in ALL_PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"mutant {name} passed every pin"
    finally:
        monkeypatch.setattr(oracle, "_lib", None)
        shutil.rmtree(tmp)


def test_workload_lengths():
    """The seeded lengths of the benchmarked workloads are reproducible."""
    w = inputs.varlen_lengths(0, 8, 33, 8192)
    assert w == [6974, 5230, 4203, 2234, 2544, 367, 646, 167]
    lens = np.random.default_rng(0).integers(1024, 32769, 16)
    assert int(lens.sum()) == 272568


# ---------------------------------------------------------------- cache append
def test_kv_append_writes_exactly_the_slots():
    """FlashRT QKV Cache RoPE, Kernels (a single-slot cache write at a
    device-side cur_pos): only rows (b*hkv + g, cur_pos[b]) change, each
    within half a quantisation step of the new row, and the lengths become
    cur_pos + 1; an out-of-range slot leaves its sequence untouched."""
    rng = np.random.default_rng(21)
    B, hkv, cap, d = 4, 3, 16, 32
    cache = rng.integers(-127, 128, (B * hkv, cap, d)).astype(np.int8)
    scales = rng.random((B * hkv, cap)).astype(np.float32)
    new = rng.standard_normal((B * hkv, d)).astype(np.float32)
    pos = np.array([0, cap - 1, 7, cap])  # the last one is out of range
    lens = np.array([5, 5, 5, 5], dtype=np.int32)
    c2, s2, l2 = oracle.kv_append(cache, scales, new, pos, hkv, seqlens=lens)
    changed = np.argwhere((c2 != cache).any(axis=2) | (s2 != scales))
    expect = {(b * hkv + g, int(pos[b])) for b in range(B - 1) for g in range(hkv)}
    assert {tuple(x) for x in changed} <= expect
    for u, p_ in expect:
        s_ = float(s2[u, p_])
        assert s_ == pytest.approx(np.abs(new[u]).max() / 127.0, rel=1e-6)
        err = np.abs(new[u].astype(np.float64) - c2[u, p_].astype(np.float64) * s_)
        assert err.max() <= s_ / 2 * (1 + 1e-6)
    assert list(l2) == [1, cap, 8, 5]
    assert np.array_equal(c2[(B - 1) * hkv:], cache[(B - 1) * hkv:])


def test_kv_append_float_cache_stores_the_row():
    rng = np.random.default_rng(22)
    cache = np.zeros((2, 4, 16), dtype=np.float32)
    new = rng.standard_normal((2, 16)).astype(np.float32)
    c2, s2, l2 = oracle.kv_append(cache, None, new, np.array([2]), 2)
    assert s2 is None and l2 is None
    assert np.array_equal(c2[:, 2], new) and not c2[:, [0, 1, 3]].any()


# ---------------------------------------------------------------- partial results and merge
def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_attention_lse_matches_attention_and_logsumexp():
    """The numpy partial-result oracle against the C oracle (outputs of rows
    with keys) and torch.logsumexp of the masked fp64 scores (lse)."""
    import torch
    rng = np.random.default_rng(70)
    hq, hkv, s_q, s_k, d = 4, 2, 37, 53, 32
    q, k, v = _rand(rng, hq, s_q, d), _rand(rng, hkv, s_k, d), _rand(rng, hkv, s_k, d)
    for causal, window in ((False, 0), (True, 0), (True, 9), (False, 7)):
        o, lse = oracle.attention_lse(q, k, v, hq=hq, hkv=hkv, causal=causal, window=window)
        ref = oracle.attention(q, k, v, hq=hq, hkv=hkv, causal=causal, window=window)
        fin = np.isfinite(lse)
        assert np.allclose(o[fin], ref[fin], rtol=1e-12, atol=1e-12)
        for h in range(hq):
            x = torch.tensor(q[h] @ k[h // 2].T / np.sqrt(d))
            i = torch.arange(s_q)[:, None] + s_k - s_q
            j = torch.arange(s_k)[None, :]
            vis = torch.ones(s_q, s_k, dtype=torch.bool)
            if causal:
                vis &= j <= i
            if window > 0:
                vis &= j > i - window
            want = torch.logsumexp(x.masked_fill(~vis, float("-inf")), dim=1).numpy()
            assert np.allclose(lse[h], want, rtol=1e-12, atol=1e-12)


def test_attention_lse_empty_rows():
    rng = np.random.default_rng(71)
    q, k, v = _rand(rng, 2, 10, 16), _rand(rng, 2, 4, 16), _rand(rng, 2, 4, 16)
    o, lse = oracle.attention_lse(q, k, v, hq=2, hkv=2, causal=True)
    assert np.all(np.isneginf(lse[:, :6])) and not o[:, :6].any()  # rows i < s_q - s_k see no key
    assert np.all(np.isfinite(lse[:, 6:]))


def test_merge_of_disjoint_key_sets_is_attention_over_their_union():
    """Splitting the keys into blocks, attending to each and merging gives
    attention over all keys (the identity the ring and split schedules rely
    on), for any split and order, with empty blocks weighing nothing."""
    rng = np.random.default_rng(72)
    hq, hkv, s, d = 4, 2, 48, 16
    q, k, v = _rand(rng, hq, s, d), _rand(rng, hkv, s, d), _rand(rng, hkv, s, d)
    full_o, full_lse = oracle.attention_lse(q, k, v, hq=hq, hkv=hkv)
    cuts = [0, 5, 20, 20, 48]  # includes an empty block
    acc_o, acc_lse = np.zeros_like(full_o), np.full(full_lse.shape, -np.inf)
    for a, b in zip(cuts[:-1], cuts[1:]):
        po, pl = oracle.attention_lse(q, k[:, a:b], v[:, a:b], hq=hq, hkv=hkv)
        acc_o, acc_lse = oracle.merge(acc_o, acc_lse, po, pl)
    assert np.allclose(acc_o, full_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(acc_lse, full_lse, rtol=1e-12, atol=1e-12)


_REAL_LSE, _REAL_MERGE = oracle.attention_lse, oracle.merge


def _lse_log2_units(*a, **k):
    o, lse = _REAL_LSE(*a, **k)
    return o, lse * np.log2(np.e)


def _merge_swapped(o_a, lse_a, o_b, lse_b):
    # each side weighted by the other's share
    o, lse = _REAL_MERGE(o_a, lse_a, o_b, lse_b)
    la, lb = np.asarray(lse_a, np.float64), np.asarray(lse_b, np.float64)
    fin = np.isfinite(lse)
    safe = np.where(fin, lse, 0.0)
    wa = np.where(fin, np.exp(lb - safe), 0.0)
    wb = np.where(fin, np.exp(la - safe), 0.0)
    return np.asarray(o_a, np.float64) * wa[..., None] + np.asarray(o_b, np.float64) * wb[..., None], lse


def _merge_max_lse(o_a, lse_a, o_b, lse_b):
    o, _ = _REAL_MERGE(o_a, lse_a, o_b, lse_b)
    return o, np.maximum(np.asarray(lse_a, np.float64), np.asarray(lse_b, np.float64))


@pytest.mark.parametrize("name,attr,wrong,pin", [
    ("lse in log2 units", "attention_lse", _lse_log2_units, "test_attention_lse_matches_attention_and_logsumexp"),
    ("merge weights swapped", "merge", _merge_swapped, "test_merge_of_disjoint_key_sets_is_attention_over_their_union"),
    ("merged lse = max", "merge", _merge_max_lse, "test_merge_of_disjoint_key_sets_is_attention_over_their_union"),
])
def test_a_planted_partial_result_mistake_fails_a_pin(monkeypatch, name, attr, wrong, pin):
    """Mistakes planted in the partial-result oracle fail its pins."""
    monkeypatch.setattr(oracle, attr, wrong)
    with pytest.raises(AssertionError):
        globals()[pin]()
