"""GPU decode attention over the packed cache (nq_attend) against the oracle.

The kernel reconstructs keys and values in fp32 exactly as the decode path
does before its bf16 rounding, but scores, exponentials and sums run in fp32
in the kernel's own order (online softmax over tiles of 16 tokens within
chunks of at least 64, values accumulated in the Hadamard code domain and
transformed once per query head).  Bound used here,
per output vector (the per-vector relative form of the reconstruction bound
on K/V, ten times tighter): ||out - out_ref||_2 <= 1e-4 ||out_ref||_2, and
|lse - lse_ref| <= 1e-4 (1 + |lse_ref|).  Sources of error: a 128-term fp32
dot product per score (relative error of order sqrt(128) 2^-24 of
sum |q_i k_i|), the fp32 exponential (2^-21 relative), fp32 running sums of
weighted codes over each chunk, and the fp32 Hadamard transform of the
merged sums (128 terms per output); together of order 1e-6 of ||out||, so
the bound leaves two orders of magnitude of margin for cancellation in
averaged outputs.
"""
import numpy as np
import pytest
import torch

from e8_lattice_vector_nq_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from e8_lattice_vector_nq_b200 import build, nq as nqmod

    build.build()
    return nqmod


def u32(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def check(nq, oq, K, V, kept, n, G, bits_k, bits_v, theta, pos_base=0, seed=0, scale=None,
          q_scale=1.0):
    units, H = K.shape[0], K.shape[1]
    max_pos = int(K.shape[2]) + pos_base
    rope = nq.rope_tables(theta, max_pos)
    ks = nq.PackedStore.empty(units, H, n, bits_k)
    vs = nq.PackedStore.empty(units, H, n, bits_v)
    nq.nq_encode(K, V, ks, vs, n, rope, max_pos, kept=kept, pos_base=pos_base)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn(units, H * G, 128, device="cuda", generator=g) * q_scale
    sc = scale if scale is not None else 128 ** -0.5
    out, lse = nq.nq_attend(q, ks, vs, n, G, rope, max_pos, scale=sc, positions=kept,
                            pos_base=pos_base)
    torch.cuda.synchronize()
    worst = 0.0
    for u in range(units):
        ref, ref_lse = oq.attend_unit(u32(ks.codes[u]), u32(ks.meta[u]), u32(vs.codes[u]),
                                      u32(vs.meta[u]), q[u].cpu().numpy(), G, sc,
                                      positions=None if kept is None else kept[u].cpu().numpy(),
                                      pos_base=pos_base, theta=theta, bits_k=bits_k, bits_v=bits_v)
        got = out[u].double().cpu().numpy()
        rel = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
        assert np.all(rel <= 1e-4), (u, rel.max())
        gl = lse[u].double().cpu().numpy()
        assert np.all(np.abs(gl - ref_lse) <= 1e-4 * (1 + np.abs(ref_lse))), np.abs(gl - ref_lse).max()
        worst = max(worst, float(rel.max()))
    return worst


def test_attend_evicted_cache_gqa(nq, oq):
    wl = synth.WORKLOADS["mistral7b_32k"]
    T = 2000
    K = torch.stack([synth.gen_layer(wl, l, "cuda", tokens=T)[0][:2] for l in range(2)])
    V = torch.stack([synth.gen_layer(wl, l, "cuda", tokens=T)[1][:2] for l in range(2)])
    scores = nq.nq_score(K, 64)
    kept = nq.nq_select(scores, 64, 60)
    n = kept.shape[1]
    check(nq, oq, K, V, kept, n, 4, 3, 2, wl.theta)


@pytest.mark.parametrize("n,G,bits_k,bits_v", [(1, 1, 3, 2), (255, 8, 2, 2), (256, 2, 3, 3),
                                               (257, 3, 2, 3), (1000, 1, 3, 2)])
def test_attend_ragged_lengths_and_formats(nq, oq, n, G, bits_k, bits_v):
    wl = synth.WORKLOADS["qwen25_7b_64k"]
    k, v = synth.gen_layer(wl, 5, "cuda", tokens=n)
    check(nq, oq, k[None], v[None], None, n, G, bits_k, bits_v, wl.theta, pos_base=300, seed=n)


def test_attend_two_head_groups_several_units(nq, oq):
    """12 KV heads (two CTAs of 6 warps per chunk), 3 units, 700 tokens."""
    wl = synth.WORKLOADS["tiny"]
    K, V = [], []
    for u in range(3):
        k0, v0 = synth.gen_layer(wl, 2 * u, "cuda", tokens=700)
        k1, v1 = synth.gen_layer(wl, 2 * u + 1, "cuda", tokens=700)
        K.append(torch.cat([k0, k1[:4]]))
        V.append(torch.cat([v0, v1[:4]]))
    check(nq, oq, torch.stack(K), torch.stack(V), None, 700, 2, 3, 2, wl.theta, seed=5)


def test_attend_sharp_and_flat_softmax(nq, oq):
    wl = synth.WORKLOADS["tiny"]
    k, v = synth.gen_layer(wl, 0, "cuda", tokens=600)
    # large queries: a few tokens dominate; zero scale: uniform weights
    check(nq, oq, k[None], v[None], None, 600, 2, 3, 2, wl.theta, seed=1, q_scale=8.0)
    check(nq, oq, k[None], v[None], None, 600, 2, 3, 2, wl.theta, seed=2, scale=0.0)


def test_attend_full_mistral_layer_sampled(nq, oq):
    """One Mistral-shaped layer at full size (8 KV heads, 13 147 kept of 32 768
    tokens, 32 query heads), all heads checked against the oracle."""
    wl = synth.WORKLOADS["mistral7b_32k"]
    k, v = synth.gen_layer(wl, 7, "cuda")
    K, V = k[None], v[None]
    kept = nq.nq_select(nq.nq_score(K, wl.window), wl.window, wl.evict_pct)
    check(nq, oq, K, V, kept, kept.shape[1], 4, 3, 2, wl.theta, seed=3)
    assert nq.device_error() == 0


def test_attend_rejects_bad_arguments(nq):
    L = nq.lib()
    pk = nq.Packed(0x20000, 0x30000, 64, 64, 3)
    fake = nq.ctypes.c_void_p(0x10000)
    assert L.nq_attend(fake, 1, 8, 9, nq.ctypes.byref(pk), nq.ctypes.byref(pk), 64, 0, None, 0, 0,
                       fake, 64, 0.1, fake, None, fake, 1 << 20, None) == nq.NQ_ERR_INVALID
    assert L.nq_attend(fake, 1, 8, 4, nq.ctypes.byref(pk), nq.ctypes.byref(pk), 0, 0, None, 0, 0,
                       fake, 64, 0.1, fake, None, fake, 1 << 20, None) == nq.NQ_ERR_INVALID
    assert L.nq_attend(fake, 1, 8, 4, nq.ctypes.byref(pk), nq.ctypes.byref(pk), 64, 0, None, 0, 0,
                       fake, 64, 0.1, fake, None, fake, 16, None) == nq.NQ_ERR_WORKSPACE
