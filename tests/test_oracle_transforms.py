"""Pins of the oracle's number formats, Hadamard transform and rotary tables.

* fp32 -> fp16 and fp32 -> bf16 rounding against numpy / torch conversions;
* FWHT against the Sylvester Hadamard matrix built by Kronecker products,
  H H^T = 128 I, and the normalised transform being its own inverse;
* RoPE tables against direct fp64 cos/sin, the identity at position 0, the
  undo/redo round trip, and undoing the synthetic cache's fp64 rotation
  (the complex-rotation form of split-half RoPE).
"""
from decimal import Decimal, getcontext

import numpy as np
import torch

from e8_lattice_vector_nq_b200 import synth


def hadamard(n: int) -> np.ndarray:
    h = np.array([[1]], np.int64)
    while h.shape[0] < n:
        h = np.kron(np.array([[1, 1], [1, -1]], np.int64), h)
    return h


# ------------------------------------------------------------ number formats
def test_fp16_rounding_matches_numpy(oq):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.normal(0, 1, 100000),
        rng.uniform(-65519, 65519, 100000),
        np.exp(rng.uniform(-20, 0, 100000)) * rng.choice([-1, 1], 100000),  # subnormal range
        # exact ties at several binades: odd multiples of half an fp16 ulp
        (2 * rng.integers(0, 1024, 20000) + 1) * 2.0 ** -11 + 1.0,
        (2 * rng.integers(0, 1024, 20000) + 1) * 2.0 ** -25,
        [0.0, -0.0, 65504.0, 65519.0, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 1e-30],
    ]).astype(np.float32)
    ours = oq.f32_to_f16_bits(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_matches_torch(oq):
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.normal(0, 1, 100000) * np.exp(rng.uniform(-30, 30, 100000)),
        (np.arange(1, 20000, dtype=np.float64) * 2.0 ** -16 + 1.0),  # includes exact ties
    ]).astype(np.float32)
    ours = oq.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_scale_constants_are_nearest_fp32():
    """C = fp32(1/sqrt 128), G_b = fp32(1/(A_b sqrt 128)), A_3 = 3.5, A_2 = 1.5."""
    getcontext().prec = 60
    r = Decimal(1) / Decimal(128).sqrt()
    src = open(__import__("oracle").__file__.replace("__init__.py", "nq_oracle.c")).read()
    for name, val in (("OQ_C_BITS", r), ("OQ_G3_BITS", r / Decimal("3.5")),
                      ("OQ_G2_BITS", r / Decimal("1.5"))):
        line = [l for l in src.splitlines() if l.startswith(f"#define {name}")][0]
        bits = int(line.split()[2].rstrip("u"), 16)
        f = np.array([bits], np.uint32).view(np.float32)[0]
        lo = np.nextafter(f, np.float32(-1))
        hi = np.nextafter(f, np.float32(1))
        err = abs(Decimal(float(f)) - val)
        assert err <= abs(Decimal(float(lo)) - val) and err <= abs(Decimal(float(hi)) - val), name


# ------------------------------------------------------------------- FWHT
def test_hadamard_orthogonal():
    H = hadamard(128)
    assert np.array_equal(H @ H.T, 128 * np.eye(128, dtype=np.int64))


def test_fwht_equals_hadamard_matrix(oq):
    rng = np.random.default_rng(3)
    x = rng.integers(-1000, 1000, (500, 128))
    got = oq.fwht(x.astype(np.float32))
    want = x @ hadamard(128).T
    assert np.array_equal(got.astype(np.int64), want)
    # basis vectors give the columns (natural / Sylvester order)
    eye = np.eye(128, dtype=np.float32)
    assert np.array_equal(oq.fwht(eye).astype(np.int64), hadamard(128).T)


def test_fwht_float_close_to_exact(oq):
    rng = np.random.default_rng(4)
    x = rng.normal(0, 1, (500, 128)).astype(np.float32)
    got = oq.fwht(x).astype(np.float64)
    want = x.astype(np.float64) @ hadamard(128).T
    assert np.max(np.abs(got - want)) < 128 * 7 * 2 ** -23 * np.max(np.abs(x)) * 4
    back = oq.fwht(oq.fwht(x)).astype(np.float64) / 128
    assert np.max(np.abs(back - x)) < 1e-5


# ------------------------------------------------------------------- RoPE
def test_rope_tables_vs_fp64(oq):
    rng = np.random.default_rng(5)
    for theta in (1e4, 5e5, 1e6):
        pos = np.concatenate([np.arange(0, 600), rng.integers(0, 1 << 17, 2000)])
        c, s = oq.rope_cs(theta, pos)
        w = theta ** (-np.arange(64) / 64.0)
        ang = pos[:, None].astype(np.float64) * w[None]
        assert np.max(np.abs(c - np.cos(ang))) < 3e-7
        assert np.max(np.abs(s - np.sin(ang))) < 3e-7


def test_rope_position_zero_is_identity(oq):
    c, s = oq.rope_cs(1e4, [0])
    assert np.all(c == 1.0) and np.all(s == 0.0)
    rng = np.random.default_rng(6)
    v = rng.normal(0, 1, (1, 128)).astype(np.float32)
    assert np.array_equal(oq.rope_apply(v, c, s, -1), v)
    assert np.array_equal(oq.rope_apply(v, c, s, +1), v)


def test_rope_round_trip(oq):
    rng = np.random.default_rng(7)
    pos = rng.integers(0, 1 << 17, 1000)
    c, s = oq.rope_cs(1e6, pos)
    v = rng.normal(0, 1, (1000, 128)).astype(np.float32)
    back = oq.rope_apply(oq.rope_apply(v, c, s, -1), c, s, +1)
    assert np.max(np.abs(back - v)) < 4e-6 * np.max(np.abs(v))


def test_generator_rope_is_complex_rotation():
    rng = np.random.default_rng(8)
    x = torch.from_numpy(rng.normal(0, 1, (3, 50, 128)))
    pos = torch.arange(100, 150)
    got = synth.rope_forward_fp64(x, pos, 1e4).numpy()
    z = x[..., :64].numpy() + 1j * x[..., 64:].numpy()
    w = 1e4 ** (-np.arange(64) / 64.0)
    rot = z * np.exp(1j * pos.numpy()[:, None] * w[None])
    assert np.allclose(got[..., :64], rot.real) and np.allclose(got[..., 64:], rot.imag)


def test_rope_undo_recovers_prerope_keys(oq):
    wl = synth.WORKLOADS["tiny"]
    K, _ = synth.gen_layer(wl, 0, "cpu", tokens=300)
    pre = synth.gen_prerope_keys(wl, 0, "cpu", tokens=300).numpy()  # [H][T][128] fp64
    kb = K.view(torch.int16).numpy().view(np.uint16)
    H, T, _ = kb.shape
    c, s = oq.rope_cs(wl.theta, np.arange(T))
    for h in range(H):
        v = oq.bf16_bits_to_f32(kb[h]).reshape(T, 128)
        u = oq.rope_apply(v, c, s, -1).astype(np.float64)
        # bf16 rounding of the stored key (2^-9 relative per coordinate, rotated)
        # plus fp32 table error
        tol = 2.0 ** -8 * np.abs(pre[h]).max(-1, keepdims=True) + 1e-5
        assert np.all(np.abs(u - pre[h]) <= tol)


def test_hadamard_spreads_outlier_channels(oq):
    """The rotation spreads outliers ([NQ-pt] step 4: an outlier would otherwise
    dominate the scale): on keys with 4 of 128 channels scaled x8 (the
    synthetic generator's outlier channels), the absmax-to-RMS ratio of each
    vector drops after the normalised Walsh-Hadamard transform.  The transform
    is orthogonal up to its 1/sqrt(128), so the RMS is unchanged and only the
    peak falls."""
    wl = synth.WORKLOADS["tiny"]
    pre = synth.gen_prerope_keys(wl, 0, "cpu", tokens=256).numpy().reshape(-1, 128)
    x = pre.astype(np.float32)
    y = oq.fwht(x) / np.float32(np.sqrt(128.0))

    def peak_to_rms(a):
        return np.abs(a).max(-1) / np.sqrt((a.astype(np.float64) ** 2).mean(-1))

    before, after = peak_to_rms(x), peak_to_rms(y)
    assert np.allclose(np.sqrt((y.astype(np.float64) ** 2).mean(-1)),
                       np.sqrt((x.astype(np.float64) ** 2).mean(-1)), rtol=1e-5)
    assert np.median(before) > 1.5 * np.median(after)
    assert np.mean(after < before) > 0.95
