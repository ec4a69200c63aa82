"""Pins of the oracle's E8 nearest-point decoder against brute force and
textbook facts about E8 = D8 u (D8 + 1/2):

* membership of every output (all-integer or all-half-integer, even sum);
* optimality against exhaustive enumeration of lattice points near y (fp64);
* the covering radius of E8 is 1;
* the 240 minimal vectors (norm^2 2) are found from 0.9 v;
* worked examples in tests/golden/e8_examples.txt.
"""
import itertools
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e8_examples.txt")


_OFFS = np.array(list(itertools.product((-1, 0, 1), repeat=8)), np.float64)  # 6561 x 8


def brute_force_e8(y: np.ndarray, batch: int = 128) -> tuple[np.ndarray, np.ndarray]:
    """Exhaustive nearest E8 point (fp64) of each row of y [n][8].

    A nearest point lies within the covering radius (1) of y, so each of its
    coordinates is within 1 of y_i: on the grid Z + shift that leaves the
    nearest grid value and its two neighbours, 3^8 candidates per coset, each
    kept only if its coordinates (minus the shift) have an even sum.
    Returns (best 2q [n][8] int, best squared distance [n])."""
    y = np.asarray(y, np.float64)
    n = y.shape[0]
    best_d = np.full(n, np.inf)
    best_t = np.zeros((n, 8), np.int64)
    for lo in range(0, n, batch):
        yb = y[lo:lo + batch]
        for shift in (0.0, 0.5):
            base = np.rint(yb - shift)
            g = base[:, None, :] + _OFFS[None]  # [b][6561][8] integer part
            even = (g.sum(-1) % 2) == 0
            pts = g + shift
            d = ((pts - yb[:, None, :]) ** 2).sum(-1)
            d = np.where(even, d, np.inf)
            j = d.argmin(1)
            dj = d[np.arange(len(yb)), j]
            sl = slice(lo, lo + len(yb))
            better = dj < best_d[sl]
            best_d[sl] = np.where(better, dj, best_d[sl])
            tt = np.rint(2 * pts[np.arange(len(yb)), j]).astype(np.int64)
            best_t[sl][better] = tt[better]
    return best_t, best_d


def check_membership(t: np.ndarray):
    par = t & 1
    assert np.all((par == par[:, :1])), "coordinates mix integer and half-integer"
    half = par[:, 0] == 1
    g = np.where(half[:, None], (t - 1) // 2, t // 2)
    assert np.all(g.sum(1) % 2 == 0), "E8 point with odd coordinate sum"


def sqdist(t, y):
    return ((t.astype(np.float64) / 2 - y.astype(np.float64)) ** 2).sum(1)


def test_membership_and_covering_radius(oq):
    rng = np.random.default_rng(11)
    y = np.concatenate([
        rng.uniform(-4, 4, (20000, 8)),
        rng.normal(0, 2, (20000, 8)),
        rng.uniform(-1e5, 1e5, (2000, 8)),
    ]).astype(np.float32)
    t, coset, d = oq.e8_nearest(y)
    check_membership(t)
    assert np.all(coset == (t[:, 0] & 1))
    exact = sqdist(t, y)
    assert exact.max() <= 1.0 + 1e-5, "beyond the E8 covering radius"
    # the returned fp32 distance is the squared distance up to fp32 rounding
    assert np.allclose(d, exact, rtol=1e-5, atol=1e-6)


def test_optimal_vs_brute_force(oq):
    rng = np.random.default_rng(12)
    parts = [
        rng.uniform(-3.6, 3.6, (1500, 8)),
        rng.normal(0, 1.5, (1000, 8)),
        # adversarial: exact half-integers, integers, quarter points and ties
        rng.integers(-8, 9, (400, 8)) / 2.0,
        rng.integers(-16, 17, (400, 8)) / 4.0,
        rng.integers(-4, 5, (300, 8)) + rng.choice([0.5, -0.5], (300, 8)) * (rng.random((300, 8)) < 0.3),
    ]
    y = np.concatenate(parts).astype(np.float32)
    t, _, _ = oq.e8_nearest(y)
    check_membership(t)
    bt, bd = brute_force_e8(y)
    got = sqdist(t, y)
    # the oracle decides in fp32; it may only lose against the exact minimum by rounding
    assert np.all(got <= bd + 1e-5), np.max(got - bd)
    # and it must hit the unique minimiser whenever the runner-up is clearly farther
    mism = np.any(t != bt, 1)
    assert np.all(np.abs(got[mism] - bd[mism]) <= 1e-5)


def e8_roots() -> np.ndarray:
    roots = []
    for i, j in itertools.combinations(range(8), 2):
        for si in (-1, 1):
            for sj in (-1, 1):
                v = np.zeros(8)
                v[i], v[j] = si, sj
                roots.append(v)
    for signs in itertools.product((-0.5, 0.5), repeat=8):
        if sum(1 for s in signs if s < 0) % 2 == 0:
            roots.append(np.array(signs))
    return np.array(roots)


def test_240_roots(oq):
    r = e8_roots()
    assert r.shape == (240, 8)
    assert np.allclose((r ** 2).sum(1), 2.0)
    t, _, _ = oq.e8_nearest((0.9 * r).astype(np.float32))
    assert np.array_equal(t, np.rint(2 * r).astype(np.int32))


def test_lattice_points_are_fixed(oq):
    rng = np.random.default_rng(13)
    g = rng.integers(-3, 4, (5000, 8))
    g[:, 0] += g.sum(1) % 2  # even sum
    half = rng.random(5000) < 0.5
    pts = g + np.where(half[:, None], 0.5, 0.0)
    t, cs, d = oq.e8_nearest(pts.astype(np.float32))
    assert np.array_equal(t, np.rint(2 * pts).astype(np.int32))
    assert np.array_equal(cs, half.astype(np.int32))
    assert np.all(d == 0)


def load_golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            ys, qs, ds = line.split("|")
            rows.append((np.array(ys.split(), np.float32), np.array(qs.split(), np.float64),
                         float(ds)))
    return rows


def test_golden_examples(oq):
    rows = load_golden()
    assert len(rows) >= 5
    for y, q, dist in rows:
        t, _, d = oq.e8_nearest(y[None])
        assert np.array_equal(t[0], np.rint(2 * q).astype(np.int32)), (y, t[0] / 2, q)
        assert abs(float(d[0]) - dist) < 1e-6
        # the worked example must also be a true nearest point
        _, bd = brute_force_e8(y[None])
        assert abs(bd[0] - dist) < 1e-6


@pytest.mark.parametrize("bits", [2, 3])
def test_clamp_ranges(oq, bits):
    """Codes stay in the b-bit range: lattice coordinates beyond it are clamped."""
    rng = np.random.default_rng(14)
    x = rng.normal(0, 1, (3000, 128)).astype(np.float32)
    x[:, :4] *= 30  # strong outliers: large |y| after the rotation on some groups
    xb = oq.f32_to_bf16_bits(x).reshape(3000, 128)
    words, meta, clamps = oq.encode_vectors(xb, bits)
    assert words.shape == (3000, 4 * bits)
    # all codes representable by construction of the layout; the unused integer
    # code (2^b - 1) must never appear in an integer-coset group
    codes = unpack_codes(words, bits)
    coset = (meta[:, None] >> np.arange(16)[None, :]) & 1
    full = np.repeat(coset, 8, axis=1)
    assert np.all(codes[full == 0] <= (1 << bits) - 2)
    assert np.all(codes < (1 << bits))


def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    """Independent unpacker: code of coordinate c at bits [b*c, b*c+b) of the
    vector's little-endian word stream."""
    n = words.shape[0]
    stream = np.zeros((n, 32 * words.shape[1]), np.uint8)
    for w in range(words.shape[1]):
        for b in range(32):
            stream[:, 32 * w + b] = (words[:, w] >> np.uint32(b)) & 1
    codes = np.zeros((n, 128), np.int64)
    for c in range(128):
        for k in range(bits):
            codes[:, c] |= stream[:, bits * c + k].astype(np.int64) << k
    return codes


@pytest.mark.parametrize("bits", [2, 3])
def test_e8_codes_are_clamped_nearest_points(oq, bits):
    """The batched E8 step with codes: each code decodes (t = 2j - lim) to the
    nearest point's 2q clipped to the b-bit range of its coset."""
    rng = np.random.default_rng(15)
    y = np.concatenate([
        rng.uniform(-4.5, 4.5, (20000, 8)),
        rng.integers(-8, 9, (2000, 8)) / 2.0,
        rng.normal(0, 1, (2000, 8)) * 1e-6,
    ]).astype(np.float32)
    codes, coset = oq.e8_codes(y, bits)
    t, cs, _ = oq.e8_nearest(y)
    assert np.array_equal(coset, cs)
    j = (codes[:, None].astype(np.int64) >> (bits * np.arange(8))[None, :]) & ((1 << bits) - 1)
    lim = np.where(coset == 1, (1 << bits) - 1, (1 << bits) - 2)[:, None]
    assert np.array_equal(2 * j - lim, np.clip(t, -lim, lim))
    assert np.all(codes < (1 << (8 * bits)))
