"""Pins of the TurboQuant oracle (oracle/turboquant.py) against what the
C attention library's README, "TurboQuant KV Cache Compression", and the
mathematics fix: the Hadamard matrix of scipy, orthonormality, the Lloyd-Max
optimality conditions by independent quadrature, Max's Gaussian quantiser
table in the large-d limit, the page's 9.14x ratio and its quality figures."""
import numpy as np
import pytest

from oracle import turboquant as tq


@pytest.mark.parametrize("n", [1, 2, 8, 64, 128])
def test_fwht_is_the_sylvester_hadamard_matrix(n):
    from scipy.linalg import hadamard
    rng = np.random.default_rng(n)
    x = rng.standard_normal((3, n))
    assert np.allclose(tq.fwht(x), x @ hadamard(n).T, rtol=0, atol=1e-12)


def test_rotation_is_orthonormal_with_the_signs_first():
    from scipy.linalg import hadamard
    rng = np.random.default_rng(1)
    d = 128
    s = rng.choice([-1.0, 1.0], d)
    x = rng.standard_normal((5, d))
    y = tq.rotate(x, s)
    assert np.allclose(y, (x * s) @ hadamard(d).T / np.sqrt(d), atol=1e-12)  # signs before H
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    assert np.allclose(tq.unrotate(y, s), x, atol=1e-12)


@pytest.mark.parametrize("d,bits", [(64, 2), (64, 4), (128, 2), (128, 3), (128, 4)])
def test_codebook_meets_the_lloyd_max_conditions(d, bits):
    """Each level is the centroid of its cell under the density of u,
    proportional to (1 - u^2)^(d/2 - 1), computed here by adaptive
    quadrature (independent of the incomplete-beta path); the edges are the
    midpoints; the levels are symmetric and ascending."""
    from scipy.integrate import quad
    lv = tq.codebook(d, bits)
    assert lv.shape == (1 << bits,) and np.all(np.diff(lv) > 0)
    assert np.allclose(lv, -lv[::-1], atol=1e-12)
    e = np.concatenate(([-1.0], tq.edges_of(lv), [1.0]))
    f = lambda u: (1.0 - u * u) ** (d / 2 - 1)
    for i in range(len(lv)):
        m0 = quad(f, e[i], e[i + 1], epsabs=0, epsrel=1e-13, limit=200)[0]
        m1 = quad(lambda u: u * f(u), e[i], e[i + 1], epsabs=0, epsrel=1e-13, limit=200)[0]
        assert abs(m1 / m0 - lv[i]) < 1e-9 * max(1.0, abs(lv[i])), (i, m1 / m0, lv[i])


# Max (1960), "Quantizing for minimum distortion", Table I: the optimum
# quantiser outputs of the unit Gaussian (positive half) and its mean squared error
GAUSS_LEVELS = {1: [0.7979], 2: [0.4528, 1.510], 3: [0.2451, 0.7560, 1.344, 2.152],
                4: [0.1284, 0.3881, 0.6568, 0.9424, 1.256, 1.618, 2.069, 2.733]}
GAUSS_MSE = {1: 0.3634, 2: 0.1175, 3: 0.03454, 4: 0.009497}


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_large_d_codebook_is_the_gaussian_lloyd_max_quantiser(bits):
    """u has variance 1/(d+1) and tends to a Gaussian as d grows, so
    sqrt(d+1) times the levels tends to Max's table."""
    from scipy.special import betainc
    d = 1 << 16
    lv = tq.codebook(d, bits) * np.sqrt(d + 1)
    half = lv[len(lv) // 2:]
    assert np.allclose(half, GAUSS_LEVELS[bits], rtol=0, atol=2e-3), half
    # distortion of the scaled quantiser, by the incomplete-beta identities
    a = d / 2.0
    e_t = (np.concatenate(([-1.0], tq.edges_of(lv / np.sqrt(d + 1)), [1.0])) + 1) / 2
    lv_t = (lv / np.sqrt(d + 1) + 1) / 2
    m0 = np.diff(betainc(a, a, e_t))
    m1 = 0.5 * np.diff(betainc(a + 1, a, e_t))
    m2 = (a * (a + 1) / ((2 * a) * (2 * a + 1))) * np.diff(betainc(a + 2, a, e_t))
    mse_t = np.sum(m2 - 2 * lv_t * m1 + lv_t ** 2 * m0)
    assert abs(4 * mse_t * (d + 1) - GAUSS_MSE[bits]) < 2e-3 * GAUSS_MSE[bits] + 1e-5


def test_codes_are_the_nearest_level():
    rng = np.random.default_rng(2)
    d = 64
    lv = tq.codebook(d, 3)
    s = rng.choice([-1.0, 1.0], d)
    x = rng.standard_normal((50, d))
    codes, norms = tq.quantize(x, s, lv)
    u = tq.unit_coords(x, s)
    dist = np.abs(u[..., None] - lv)
    assert np.all(dist[np.arange(50)[:, None], np.arange(d), codes] <= dist.min(axis=-1) + 1e-15)
    assert np.allclose(norms, np.linalg.norm(x, axis=-1))
    z, zn = tq.quantize(np.zeros((1, d)), s, lv)  # a zero row: u = 0, the level just above 0
    assert zn[0] == 0 and np.all(z == 4)


def test_bit_packing_is_lsb_first():
    # codes 1, 2, 3, 0 at 2 bits: stream bits 1,0 | 0,1 | 1,1 | 0,0 -> 0b00111001
    assert tq.pack(np.array([1, 2, 3, 0], np.uint8), 2).tolist() == [0x39]
    # eight 3-bit codes: the expected bytes cut from the LSB-first bit string
    c = np.array([5, 3, 7, 0, 1, 2, 4, 6], np.uint8)
    p = tq.pack(c, 3)
    stream = "".join(format(int(v), "03b")[::-1] for v in c)  # LSB first per code
    want = [int(stream[8 * i: 8 * i + 8][::-1], 2) for i in range(3)]
    assert p.tolist() == want
    rng = np.random.default_rng(3)
    for bits in (2, 3, 4):
        for d in (64, 128):
            codes = rng.integers(0, 1 << bits, (7, d)).astype(np.uint8)
            packed = tq.pack(codes, bits)
            assert packed.shape == (7, d * bits // 8)
            assert np.array_equal(tq.unpack(packed, bits, d), codes)


def test_k4_v2_is_9_14_times_smaller_than_fp32():
    """The page puts the default K4/V2 at 9.14 times less memory than fp32
    (d = 64: 512 bytes of fp32 K and V per token and head against 56)."""
    d = 64
    ratio = (2 * 4 * d) / (tq.bytes_per_row(d, 4) + tq.bytes_per_row(d, 2))
    assert round(ratio, 2) == 9.14


def _attention(q, k, v):
    s = q @ k.T / np.sqrt(q.shape[-1])
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    return (p / p.sum(axis=-1, keepdims=True)) @ v


def test_quality_in_the_range_the_page_reports():
    """The page: attention-output cosine about 0.94 for K4/V2 on synthetic
    data and about 0.99 for K4/V4 (value bits drive the error).  On N(0,1)
    queries, keys and values (d = 128, 512 keys) the oracle gives 0.937 and
    0.991, and the error falls as the value bits grow."""
    rng = np.random.default_rng(4)
    d, n = 128, 512
    s = rng.choice([-1.0, 1.0], d)
    q, k, v = rng.standard_normal((64, d)), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    ref = _attention(q, k, v)

    def cos(kb, vb):
        lk, lv = tq.codebook(d, kb), tq.codebook(d, vb)
        kh = tq.dequantize(*tq.compress(k, s, kb, lk), s, kb, lk, d)
        vh = tq.dequantize(*tq.compress(v, s, vb, lv), s, vb, lv, d)
        o = _attention(q, kh, vh)
        return float(np.mean(np.sum(o * ref, -1) / (np.linalg.norm(o, axis=-1) * np.linalg.norm(ref, axis=-1))))

    c42, c43, c44 = cos(4, 2), cos(4, 3), cos(4, 4)
    assert 0.92 <= c42 <= 0.955, c42   # the page: about 0.94
    assert 0.985 <= c44 <= 0.995, c44  # the page: about 0.99
    assert c42 < c43 < c44


def _plant(monkeypatch, name, fn):
    monkeypatch.setattr(tq, name, fn)
    tq._codebook_cached.cache_clear()


_REAL = {n: getattr(tq, n) for n in ("fwht", "rotate", "_codebook", "pack", "dequantize", "edges_of")}

PLANTS = {
    # butterfly outputs swapped: H with its rows reordered
    "fwht_swapped": ("fwht", lambda x: _REAL["fwht"](x)[..., ::-1].copy(),
                     lambda mp: test_fwht_is_the_sylvester_hadamard_matrix(8)),
    # signs applied after the transform instead of before it
    "signs_after_H": ("rotate", lambda x, s: _REAL["fwht"](np.asarray(x, np.float64)) * np.asarray(s, np.float64)
                      / np.sqrt(np.asarray(x).shape[-1]),
                      lambda mp: test_rotation_is_orthonormal_with_the_signs_first()),
    # the quantiles the iteration starts from, not the Lloyd-Max fixed point
    "no_lloyd_iteration": ("_codebook", lambda d, b: _REAL["_codebook"](d, b, iters=1),
                           lambda mp: test_codebook_meets_the_lloyd_max_conditions(64, 4)),
    # a uniform codebook of the right range
    "uniform_levels": ("_codebook", lambda d, b: np.linspace(-3, 3, 1 << b) / np.sqrt(d + 1),
                       lambda mp: test_large_d_codebook_is_the_gaussian_lloyd_max_quantiser(2)),
    # cell edges at the levels themselves instead of the midpoints
    "edges_at_levels": ("edges_of", lambda lv: np.asarray(lv, np.float64)[1:],
                        lambda mp: test_codes_are_the_nearest_level()),
    # most significant bit first within each code
    "msb_first": ("pack", lambda c, b: _REAL["pack"](np.sum(((np.asarray(c, np.uint8)[..., None] >> np.arange(b))
                                                            & 1) << np.arange(b)[::-1], -1).astype(np.uint8), b),
                  lambda mp: test_bit_packing_is_lsb_first()),
    # the inverse rotation without the signs
    "unrotate_without_signs": ("dequantize", lambda p, n, s, b, lv, d: _REAL["dequantize"](p, n, np.ones(d), b, lv, d),
                               lambda mp: test_quality_in_the_range_the_page_reports()),
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_a_planted_mistake_fails_a_pin(monkeypatch, plant):
    """Each plausible mistake, planted in the oracle, makes its pin fail."""
    name, wrong, pin = PLANTS[plant]
    _plant(monkeypatch, name, wrong)
    try:
        with pytest.raises(AssertionError):
            pin(monkeypatch)
    finally:
        tq._codebook_cached.cache_clear()
