"""Pins of the oracle's box-constrained E8 step and of the exact packing.

The exact 24/16-bit packing folds each group's coset bit into the low bit of
its last code, which the even sum of E8 points makes redundant.  That needs
every coded point to lie in E8, while the encoder's clamp (nearest E8 point,
then each 2q clamped) can leave E8.  The reading taken: code the nearest
point of E8 inside the b-bit code box.  Pins from the mathematics:

* every output is a point of E8 inside the box;
* it is the nearest such point: brute force over all of E8 in the box for
  b = 2 (3^8 + 4^8 points), and for b = 3 over every point within one step
  of each coordinate's clamped rounding (each coordinate of the optimum is its
  clamped rounding or the nearest in-range value of the other parity);
* when the unconstrained decoder's point lies inside the box, both agree;
* the exact packing is a bijection on these points (pack then unpack is the
  identity), and it would lose information for points off E8 (the encoder's
  clamp), which is why the box rule is needed;
* at the vector level the box encoder equals the codec wherever the codec
  clamps nothing, and the exact layout (coset bit folded, sigma alone in the
  meta) converts to the regular one and back without loss.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle as oq
from e8_lattice_vector_nq_b200 import synth


def unpack_codes(c, bits):
    return np.array([(int(c) >> (bits * i)) & ((1 << bits) - 1) for i in range(8)], np.int64)


def codes_to_q(c, half, bits):
    j = unpack_codes(c, bits)
    lim = (1 << bits) - (1 if half else 2)
    return (2 * j - lim) / 2.0


def groups(seed, n):
    rng = np.random.default_rng(seed)
    parts = [rng.normal(0, s, (n, 8)) for s in (0.5, 1.0, 2.0, 4.0)]
    parts.append(rng.uniform(-6, 6, (n, 8)))
    base = rng.integers(-4, 4, (n, 8))
    parts.append(base + 0.5 * rng.choice([-1.0, 1.0], (n, 8)))  # rounding ties
    parts.append(base + 0.25 * rng.choice([-1.0, 1.0], (n, 8)))  # coset ties
    return np.concatenate(parts).astype(np.float32)


@pytest.mark.parametrize("bits", [2, 3])
def test_points_are_in_e8_and_in_the_box(bits):
    y = groups(bits, 2000)
    c, h, _ = oq.e8_box_codes(y, bits)
    top = 2 ** (bits - 1)
    for g in range(len(y)):
        q = codes_to_q(c[g], h[g], bits)
        f = q - 0.5 * h[g]
        assert np.all(f == np.round(f))                    # all in Z or all in Z + 1/2
        assert int(np.sum(f)) % 2 == 0                     # even sum (D8 or D8 + 1/2)
        lim_q = top - 0.5 if h[g] else top - 1
        assert np.all(np.abs(q) <= lim_q)


def box_points_b2():
    pts = []
    for vals, half in (((-1, 0, 1), 0), ((-1.5, -0.5, 0.5, 1.5), 1)):
        for p in itertools.product(vals, repeat=8):
            a = np.array(p)
            if int(np.sum(a - 0.5 * half)) % 2 == 0:
                pts.append(a)
    return np.array(pts)


def test_nearest_in_box_by_full_enumeration_b2():
    P = box_points_b2()  # all of E8 inside the 2-bit box
    # even-sum points: (3^8 + 1) / 2 of the integer grid, 4^8 / 2 of the half grid
    assert len(P) == (3 ** 8 + 1) // 2 + 4 ** 8 // 2
    y = groups(11, 60)
    c, h, _ = oq.e8_box_codes(y, 2)
    for g in range(len(y)):
        d = np.sum((P - y[g].astype(np.float64)) ** 2, axis=1)
        q = codes_to_q(c[g], h[g], 2)
        mine = np.sum((q - y[g]) ** 2)
        assert mine <= d.min() + 1e-9


def test_nearest_in_box_by_neighbourhood_enumeration_b3():
    y = groups(12, 80)
    c, h, _ = oq.e8_box_codes(y, 3)
    steps = np.array(list(itertools.product((-1, 0, 1), repeat=8)))
    for g in range(len(y)):
        best = np.inf
        for half, lo, hi in ((0, -3, 3), (1, -4, 3)):
            u = y[g].astype(np.float64) - 0.5 * half
            f0 = np.clip(np.rint(u), lo, hi)
            F = f0 + steps
            ok = np.all((F >= lo) & (F <= hi), axis=1) & (np.sum(F, axis=1) % 2 == 0)
            d = np.sum((F[ok] - u) ** 2, axis=1)
            best = min(best, d.min())
        q = codes_to_q(c[g], h[g], 3)
        assert np.sum((q - y[g]) ** 2) <= best + 1e-9


@pytest.mark.parametrize("bits", [2, 3])
def test_agrees_with_the_decoder_inside_the_box(bits):
    y = groups(20 + bits, 3000)
    t, hs, dist = oq.e8_nearest(y)
    c, h, d = oq.e8_box_codes(y, bits)
    top = 2 ** (bits - 1)
    inside = 0
    for g in range(len(y)):
        q = t[g] / 2.0
        lim_q = top - 0.5 if hs[g] else top - 1
        if np.all(np.abs(q) <= lim_q):
            inside += 1
            mine = codes_to_q(c[g], h[g], bits)
            # the same point, or (fp32 distances computed in a different
            # order) an exact tie between two points
            assert np.array_equal(mine, q) or abs(float(d[g]) - float(dist[g])) < 1e-5
    assert inside > 1000


@pytest.mark.parametrize("bits", [2, 3])
def test_exact_packing_round_trip(bits):
    y = groups(30 + bits, 1000)
    c, h, _ = oq.e8_box_codes(y, bits)
    for g in range(len(y)):
        j = unpack_codes(c[g], bits).astype(np.uint32)
        w = oq.exact_pack(j, int(h[g]), bits)
        assert w < (1 << (8 * bits))
        jj, hh = oq.exact_unpack(w, bits)
        assert np.array_equal(jj, j) and hh == h[g]


def test_the_encoder_clamp_can_leave_e8():
    """Large groups: the nearest-then-clamp codes of the encoder break the
    even sum for some groups, so the exact packing could not carry them."""
    rng = np.random.default_rng(5)
    y = rng.uniform(-7, 7, (4000, 8)).astype(np.float32)
    c, h = oq.e8_codes(y, 3)
    broken = 0
    for g in range(len(y)):
        j = unpack_codes(c[g], 3)
        broken += int(np.sum(j)) % 2
    assert broken > 0
    cb, hb, _ = oq.e8_box_codes(y, 3)
    assert all(int(np.sum(unpack_codes(cb[g], 3))) % 2 == 0 for g in range(len(y)))


def synthetic_vectors(seed, n):
    """n synthetic key vectors (bf16 bits, [n][128]) of the tiny workload."""
    wl = synth.WORKLOADS["tiny"]
    k, _ = synth.gen_layer(wl, seed % 4, "cpu", tokens=n // 8)
    return k.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1, 128)


@pytest.mark.parametrize("bits", [2, 3])
def test_vector_encoder_matches_the_codec_where_nothing_clamps(bits):
    """Vectors whose regular encode clamps no coordinate: the box encoder gives
    the same words and meta (the box then contains the decoder's points)."""
    x = synthetic_vectors(bits, 2048)
    same = 0
    for i in range(0, x.shape[0], 64):
        blk = x[i:i + 64]
        w0, m0, _ = oq.encode_vectors(blk, bits)
        w1, m1 = oq.encode_vectors_box(blk, bits)
        for r in range(blk.shape[0]):
            _, _, cl = oq.encode_vectors(blk[r:r + 1], bits)
            if cl == 0:
                assert np.array_equal(w0[r], w1[r]) and m0[r] == m1[r]
                same += 1
    assert same > 100


@pytest.mark.parametrize("bits", [2, 3])
def test_exact_layout_round_trip_and_decode(bits):
    """fold then unfold restores the box encoder's words and meta; the exact
    layout differs from the regular one in at most one bit per group; and
    decoding the unfolded vectors gives the box encoder's reconstruction."""
    x = synthetic_vectors(10 + bits, 2048)
    w, m = oq.encode_vectors_box(x, bits)
    ew, sig = oq.fold_exact(w, m, bits)
    assert np.array_equal(sig, (m >> 16).astype(np.uint16))
    diff = np.unpackbits((ew ^ w).view(np.uint8), axis=1).sum(axis=1)
    assert np.all(diff <= 16)
    w2, m2 = oq.unfold_exact(ew, sig, bits)
    assert np.array_equal(w2, w) and np.array_equal(m2, m)
    assert np.array_equal(oq.decode_vectors(w2, m2, bits), oq.decode_vectors(w, m, bits))


@pytest.mark.parametrize("name,bits", [("k", 3), ("v", 2)])
def test_box_rule_costs_little_reconstruction_error(name, bits):
    """The price of the parity-preserving clamp: on 2048 tokens of layer 0 of the
    Mistral-shaped cache the box-constrained points differ from the codec's on
    about a fifth of the vectors, and the mean relative reconstruction error
    rises by under 1 % (0.1977 -> 0.1981 for 3-bit keys, 0.5037 -> 0.5051 for
    2-bit values): the clamped codec point is not bound to E8 and can sit a
    little closer."""
    wl = synth.WORKLOADS["mistral7b_32k"]
    k, v = synth.gen_layer(wl, 0, "cpu", tokens=2048)
    X = k if name == "k" else v
    x = X.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1, 128)
    w0, m0, _ = oq.encode_vectors(x, bits)
    w1, m1 = oq.encode_vectors_box(x, bits)
    xx = oq.bf16_bits_to_f32(x).astype(np.float64)

    def err(w, m):
        r = oq.reconstruct_vectors(w, m, bits).astype(np.float64)
        return np.mean(np.linalg.norm(xx - r, axis=1) / np.linalg.norm(xx, axis=1))

    e_clamp, e_box = err(w0, m0), err(w1, m1)
    assert e_clamp <= e_box < 1.01 * e_clamp
