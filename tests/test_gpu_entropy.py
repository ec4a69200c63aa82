"""GPU delta + entropy stage (nq_entropy_encode / nq_entropy_decode) against
the oracle: tables, stream offsets and every coded word bit for bit, and the
decode restoring the code words exactly."""
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


def pack_codes(j, bits):
    """uint32 code words [..., 4*bits] of codes j [..., 128] (code c at bits [b c, b c + b))."""
    words = np.zeros(j.shape[:-1] + (4 * bits,), np.uint32)
    for c in range(128):
        for k in range(bits):
            p = bits * c + k
            words[..., p >> 5] |= ((j[..., c] >> k) & 1).astype(np.uint32) << np.uint32(p & 31)
    return words


def store_from_words(nq, words, bits, cap=None, slot0=0):
    units, heads, n = words.shape[:3]
    cap = n + slot0 if cap is None else cap
    st = nq.PackedStore.empty(units, heads, cap, bits)
    st.codes.zero_()
    st.meta.zero_()
    st.codes[:, :, slot0:slot0 + n] = torch.from_numpy(words.view(np.int32)).cuda()
    return st


def check(nq, oq, st, n, delta, slot0=0):
    bits = st.bits
    units, heads = st.meta.shape[:2]
    coded = nq.nq_entropy_encode(st, n, delta=delta, slot0=slot0)
    torch.cuda.synchronize()
    ref_codes = u32(st.codes[:, :, slot0:slot0 + n])
    freq, offsets, words = oq.entropy_encode_store(ref_codes, bits, delta)
    assert np.array_equal(coded.freq.cpu().numpy().view(np.uint16), freq)
    got_off = coded.offsets.cpu().numpy().view(np.uint32)
    assert np.array_equal(got_off, offsets)
    total = coded.total_words()
    assert total == words.size
    assert np.array_equal(coded.words[:total].cpu().numpy().view(np.uint16), words)
    # decode into a fresh store at the same slots: the code words come back exactly
    out = nq.PackedStore.empty(units, heads, st.codes.shape[2], bits)
    out.codes.fill_(-1)
    nq.nq_entropy_decode(coded, out, slot0=slot0)
    torch.cuda.synchronize()
    assert np.array_equal(u32(out.codes[:, :, slot0:slot0 + n]), ref_codes)
    return total


@pytest.mark.parametrize("bits,delta", [(3, True), (3, False), (2, True), (2, False)])
def test_encoded_cache(nq, oq, bits, delta):
    """Codes of a real encode (tiny workload, 2 units x 8 heads x 2100 tokens)."""
    wl = synth.WORKLOADS["tiny"]
    T = 2100
    K = torch.stack([synth.gen_layer(wl, l, "cuda", tokens=T)[0] for l in range(2)])
    V = torch.stack([synth.gen_layer(wl, l, "cuda", tokens=T)[1] for l in range(2)])
    rope = nq.rope_tables(wl.theta, T)
    ks = nq.PackedStore.empty(2, 8, T, bits)
    vs = nq.PackedStore.empty(2, 8, T, bits)
    nq.nq_encode(K, V, ks, vs, T, rope, T)
    check(nq, oq, ks, T, delta)
    check(nq, oq, vs, T, delta)


@pytest.mark.parametrize("n", [1, 2, 2047, 2048, 2049, 5000])
@pytest.mark.parametrize("bits", [2, 3])
def test_random_codes_ragged_lengths(nq, oq, n, bits):
    rng = np.random.default_rng(n * 10 + bits)
    j = rng.integers(0, 1 << bits, (1, 3, n, 128))
    st = store_from_words(nq, pack_codes(j, bits), bits)
    check(nq, oq, st, n, delta=bool(n % 2))


def test_correlated_codes_with_slot_offset(nq, oq):
    """A slow random walk of the codes (differences mostly 0): the delta
    streams are much shorter; slots 37 .. 37+3000 of a 4096-slot store."""
    rng = np.random.default_rng(11)
    n, bits, slot0 = 3000, 3, 37
    steps = rng.integers(-1, 2, (2, 4, n, 128)) * (rng.random((2, 4, n, 128)) < 0.1)
    j = np.cumsum(steps, axis=2) % 8
    st = store_from_words(nq, pack_codes(j, bits), bits, cap=4096, slot0=slot0)
    t_delta = check(nq, oq, st, n, delta=True, slot0=slot0)
    t_plain = check(nq, oq, st, n, delta=False, slot0=slot0)
    assert t_delta < 0.6 * t_plain


def test_single_symbol_streams(nq, oq):
    """All codes equal: one symbol with F = 4096, every stream is the bare
    initial state (2 words)."""
    n = 3000
    j = np.full((1, 2, n, 128), 5)
    st = store_from_words(nq, pack_codes(j, 3), 3)
    total = check(nq, oq, st, n, delta=True)
    assert total == 2 * nq.lib().nq_entropy_streams(1, 2, n)


def test_full_mistral_layer(nq, oq):
    """One Mistral-shaped layer at full size: 8 heads x 13 147 kept tokens,
    keys K3 and values V2, all streams against the oracle."""
    wl = synth.WORKLOADS["mistral7b_32k"]
    k, v = synth.gen_layer(wl, 3, "cuda")
    K, V = k[None], v[None]
    kept = nq.nq_select(nq.nq_score(K, wl.window), wl.window, wl.evict_pct)
    n = kept.shape[1]
    rope = nq.rope_tables(wl.theta, wl.tokens)
    ks = nq.PackedStore.empty(1, 8, n, 3)
    vs = nq.PackedStore.empty(1, 8, n, 2)
    nq.nq_encode(K, V, ks, vs, n, rope, wl.tokens, kept=kept)
    check(nq, oq, ks, n, delta=True)
    check(nq, oq, vs, n, delta=False)
