"""Pins of the oracle's decode-phase attention over a packed unit.

* its fp32 reconstructions round (bf16, RNE) to exactly the pinned decode output;
* the attention itself equals scipy's softmax / logsumexp applied to the
  reconstructed keys and values (library routines, fp64);
* closed forms: one token gives that token's value and score; a zero scale gives
  uniform weights (the mean of the values);
* query head j attends with KV head j // G.
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

D = 128


def packed_unit(oq, seed, H, T, n=None, kept=None, bits_k=3, bits_v=2, theta=1e4):
    rng = np.random.default_rng(seed)
    K = oq.f32_to_bf16_bits(rng.normal(0, 1, (H, T, D)).astype(np.float32)).reshape(H, T, D)
    V = oq.f32_to_bf16_bits(rng.normal(0, 1, (H, T, D)).astype(np.float32)).reshape(H, T, D)
    n = T if n is None else n
    return oq.encode_unit(K, V, n, kept=kept, theta=theta, bits_k=bits_k, bits_v=bits_v)


def reconstruct_unit(oq, r, positions, theta, bits_k, bits_v):
    H, n = r["k_meta"].shape
    c, s = oq.rope_cs(theta, positions)
    k = np.stack([oq.reconstruct_vectors(r["k_codes"][h], r["k_meta"][h], bits_k, rope=True,
                                         c=c, s=s) for h in range(H)])
    v = np.stack([oq.reconstruct_vectors(r["v_codes"][h], r["v_meta"][h], bits_v)
                  for h in range(H)])
    return k, v


def test_reconstruction_rounds_to_the_decode_output(oq):
    theta = 1e6
    r = packed_unit(oq, 1, 2, 300, theta=theta)
    pos = np.arange(300)
    k, v = reconstruct_unit(oq, r, pos, theta, 3, 2)
    Kd, Vd = oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], theta=theta)
    assert np.array_equal(oq.f32_to_bf16_bits(k).reshape(Kd.shape), Kd)
    assert np.array_equal(oq.f32_to_bf16_bits(v).reshape(Vd.shape), Vd)


@pytest.mark.parametrize("H,G,bits_k", [(1, 1, 3), (2, 4, 3), (4, 2, 2)])
def test_attention_equals_library_softmax(oq, H, G, bits_k):
    theta, T = 5e5, 700
    rng = np.random.default_rng(H * 10 + G)
    kept = np.sort(rng.choice(T, 333, replace=False)).astype(np.int32)
    r = packed_unit(oq, 2, H, T, n=333, kept=kept, bits_k=bits_k, theta=theta)
    q = rng.normal(0, 1, (H * G, D)).astype(np.float32)
    scale = 1 / np.sqrt(D)
    out, lse = oq.attend_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], q, G, scale,
                              positions=kept, theta=theta, bits_k=bits_k)
    k, v = reconstruct_unit(oq, r, kept, theta, bits_k, 2)
    for j in range(H * G):
        h = j // G
        s = scale * (k[h].astype(np.float64) @ q[j].astype(np.float64))
        p = softmax(s)
        np.testing.assert_allclose(out[j], p @ v[h].astype(np.float64), rtol=1e-12, atol=1e-12)
        assert abs(lse[j] - logsumexp(s)) <= 1e-12 * max(1.0, abs(lse[j]))


def test_one_token_and_uniform_weights(oq):
    theta = 1e4
    r = packed_unit(oq, 3, 2, 50, theta=theta)
    rng = np.random.default_rng(4)
    q = rng.normal(0, 1, (2, D)).astype(np.float32)
    k, v = reconstruct_unit(oq, r, np.arange(50), theta, 3, 2)
    # a single token: its value, its score
    one = {key: (val[:, :1].copy() if key != "clamps" else val) for key, val in r.items()}
    out, lse = oq.attend_unit(one["k_codes"], one["k_meta"], one["v_codes"], one["v_meta"], q, 1,
                              0.5, theta=theta)
    for h in range(2):
        assert np.array_equal(out[h], v[h, 0].astype(np.float64))
        s0 = 0.5 * float(k[h, 0].astype(np.float64) @ q[h].astype(np.float64))
        assert abs(lse[h] - s0) <= 1e-14 * abs(s0)  # fp64 summation order only
    # zero scale: every token weighs 1/n
    out, lse = oq.attend_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], q, 1, 0.0,
                              theta=theta)
    for h in range(2):
        np.testing.assert_allclose(out[h], v[h].astype(np.float64).mean(0), rtol=0, atol=1e-12)
        assert abs(lse[h] - np.log(50)) <= 1e-12


def test_query_head_uses_kv_head_j_over_g(oq):
    theta, H, G = 1e4, 3, 2
    r = packed_unit(oq, 5, H, 80, theta=theta)
    rng = np.random.default_rng(6)
    q = rng.normal(0, 1, (H * G, D)).astype(np.float32)
    out, lse = oq.attend_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], q, G, 0.1,
                              theta=theta)
    for j in range(H * G):
        h = j // G
        o1, l1 = oq.attend_unit(r["k_codes"][h:h + 1], r["k_meta"][h:h + 1], r["v_codes"][h:h + 1],
                                r["v_meta"][h:h + 1], q[j:j + 1], 1, 0.1, theta=theta)
        assert np.array_equal(out[j], o1[0]) and lse[j] == l1[0]
