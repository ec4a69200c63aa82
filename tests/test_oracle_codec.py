"""Pins of the oracle's vector codec (encode: RoPE undo, FWHT, scale, E8,
clamp, pack; decode: unpack, inverse FWHT, RoPE redo, bf16) against an
independent fp64 numpy restatement that uses the Hadamard matrix, direct
cos/sin, numpy's fp16 conversion and brute-force E8 search.
"""
import numpy as np
import pytest

from tests.test_oracle_e8 import brute_force_e8, unpack_codes
from tests.test_oracle_transforms import hadamard

H128 = hadamard(128).astype(np.float64)
C64 = 1.0 / np.sqrt(128.0)


def f32(bits):
    return np.array([bits], np.uint32).view(np.float32)[0]


C32 = f32(0x3DB504F3)
G32 = {3: f32(0x3CCEE116), 2: f32(0x3D715BEF)}


def rope_fp64(v, pos, theta, direction):
    w = theta ** (-np.arange(64) / 64.0)
    ang = direction * pos[:, None].astype(np.float64) * w[None]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[:, :64], v[:, 64:]
    return np.concatenate([a * c - b * s, b * c + a * s], 1)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Independent packer: code of coordinate c at bits [b*c, b*c+b)."""
    n = codes.shape[0]
    words = np.zeros((n, 4 * bits), np.uint64)
    for c in range(128):
        for k in range(bits):
            p = bits * c + k
            words[:, p // 32] |= ((codes[:, c].astype(np.uint64) >> np.uint64(k)) & np.uint64(1)) << np.uint64(p % 32)
    return words.astype(np.uint32)


def reference_reconstruct(words, meta, bits, pos=None, theta=None):
    codes = unpack_codes(words, bits)
    coset = np.repeat(((meta[:, None] >> np.arange(16)[None]) & 1).astype(np.int64), 8, 1)
    t = 2 * codes - (1 << bits) + 2 - coset
    sig = (meta >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    x = (t.astype(np.float64) @ H128.T) * (sig[:, None] * 0.5 * C64)
    if pos is not None:
        x = rope_fp64(x, pos, theta, +1)
    return x, t


def make_inputs(oq, n, seed, outliers=True):
    rng = np.random.default_rng(seed)
    lam = np.exp(0.5 * rng.normal(0, 1, (1, 128)))
    if outliers:
        lam[0, rng.choice(128, 4, replace=False)] *= 8
    x = rng.normal(0, 1, (n, 128)) * lam
    return oq.f32_to_bf16_bits(x.astype(np.float32)).reshape(n, 128)


@pytest.mark.parametrize("bits,rope", [(3, True), (2, False), (2, True), (3, False)])
def test_encode_matches_fp64_restatement(oq, bits, rope):
    n, theta = 400, 1e6
    xb = make_inputs(oq, n, 20 + bits + 2 * rope)
    rng = np.random.default_rng(30)
    pos = rng.integers(0, 1 << 17, n)
    c, s = oq.rope_cs(theta, pos)
    words, meta, _ = oq.encode_vectors(xb, bits, rope=rope, c=c, s=s)

    x = oq.bf16_bits_to_f32(xb).astype(np.float64).reshape(n, 128)
    u = rope_fp64(x, pos, theta, -1) if rope else x
    v = u @ H128.T
    M = np.abs(v).max(1)
    sig = np.minimum((M.astype(np.float32) * G32[bits]), np.float32(65504)).astype(np.float16)
    sig_bits = sig.view(np.uint16)
    got_sig = (meta >> 16).astype(np.uint16)
    # the fp16 scale may differ only where fp32 vs fp64 sums land on a rounding edge
    assert np.mean(got_sig != sig_bits) < 2e-3
    same = got_sig == sig_bits
    y = v * (float(C32) / sig.astype(np.float64))[:, None]
    bt, bd = brute_force_e8(y[same].reshape(-1, 8))
    lim_half, lim_int = (1 << bits) - 1, (1 << bits) - 2
    half = (bt[:, 0] & 1) == 1
    lim = np.where(half, lim_half, lim_int)[:, None]
    tc = np.clip(bt, -lim, lim)
    codes_ref = ((tc + lim) // 2).reshape(-1, 128)
    coset_ref = half.reshape(-1, 16)
    codes = unpack_codes(words[same], bits)
    coset = ((meta[same][:, None] >> np.arange(16)[None]) & 1).astype(bool)
    grp_mis = np.any((codes != codes_ref).reshape(-1, 16, 8), -1) | (coset != coset_ref)
    # fp32 (oracle) vs fp64 (restatement) decisions only split on near-ties
    assert grp_mis.mean() < 2e-3, grp_mis.mean()
    if grp_mis.any():
        yg = y[same].reshape(-1, 8)[grp_mis.ravel()]
        _, got_t = reference_reconstruct(words[same], meta[same], bits)
        gt = got_t.reshape(-1, 8)[grp_mis.ravel()]
        dg = ((gt / 2 - yg) ** 2).sum(1)
        assert np.all(np.abs(dg - bd[grp_mis.ravel()]) < 1e-3)


@pytest.mark.parametrize("bits", [2, 3])
def test_decode_every_code_at_every_coordinate(oq, bits):
    rng = np.random.default_rng(40 + bits)
    n = 4096
    codes = rng.integers(0, 1 << bits, (n, 128))
    coset = rng.integers(0, 2, (n, 16))
    full = np.repeat(coset, 8, 1)
    codes = np.where(full == 0, np.minimum(codes, (1 << bits) - 2), codes)  # integer coset range
    sig = np.abs(rng.normal(0, 1, n)).astype(np.float16)
    meta = (coset << np.arange(16)).sum(1).astype(np.uint32) | (sig.view(np.uint16).astype(np.uint32) << 16)
    words = pack_codes(codes, bits)
    pos = rng.integers(0, 1 << 16, n)
    for rope in (False, True):
        c, s = oq.rope_cs(5e5, pos)
        out = oq.decode_vectors(words, meta, bits, rope=rope, c=c, s=s)
        got = oq.bf16_bits_to_f32(out).astype(np.float64).reshape(n, 128)
        ref, t = reference_reconstruct(words, meta, bits, pos if rope else None, 5e5)
        assert np.array_equal(unpack_codes(words, bits), codes)
        scale = np.abs(ref).max(1, keepdims=True)
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * scale)


@pytest.mark.parametrize("bits", [2, 3])
def test_round_trip_error_bound(oq, bits):
    """Unclamped vectors: ||x - x_hat|| <= 1 * sigma * sqrt(128) * ... per group radius 1,
    i.e. ||y - q|| <= 4 over 16 groups, mapped back by the orthonormal H/sqrt(128)."""
    n = 2000
    xb = make_inputs(oq, n, 50 + bits)
    words, meta, _ = oq.encode_vectors(xb, bits)
    out = oq.decode_vectors(words, meta, bits)
    x = oq.bf16_bits_to_f32(xb).astype(np.float64).reshape(n, 128)
    xh = oq.bf16_bits_to_f32(out).astype(np.float64).reshape(n, 128)
    sig = (meta >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    err = np.linalg.norm(x - xh, axis=1)
    bound = 4.0 * sig * np.sqrt(128.0) * C64 * 1.0001 + 2.0 ** -8 * np.linalg.norm(xh, axis=1)
    # clamped vectors may exceed the lattice bound; they are rare at these scales
    _, t = reference_reconstruct(words, meta, bits)
    assert np.mean(err <= bound) > 0.97
    cos = (x * xh).sum(1) / (np.linalg.norm(x, axis=1) * np.linalg.norm(xh, axis=1))
    assert np.median(cos) > (0.97 if bits == 3 else 0.90)


def test_degenerate_vectors(oq):
    z = np.zeros((1, 128), np.uint16)
    for bits in (2, 3):
        w, m, _ = oq.encode_vectors(z, bits)
        assert m[0] == 0  # sigma 0, integer coset everywhere
        codes = unpack_codes(w, bits)
        assert np.all(codes == (1 << (bits - 1)) - 1)  # q = 0
        out = oq.decode_vectors(w, m, bits)
        assert np.all(out == 0)
    # huge input saturates the fp16 scale at 65504 and clamps codes
    big = oq.f32_to_bf16_bits(np.full(128, 1e9, np.float32)).reshape(1, 128)
    w, m, cl = oq.encode_vectors(big, 3)
    assert (m[0] >> 16) == 0x7BFF and cl > 0
    # tiny input: fp16 subnormal scale still reconstructs proportionally
    tiny = oq.f32_to_bf16_bits(np.linspace(-1, 1, 128).astype(np.float32) * 1e-6).reshape(1, 128)
    w, m, _ = oq.encode_vectors(tiny, 3)
    assert 0 < (m[0] >> 16) < 0x0400
