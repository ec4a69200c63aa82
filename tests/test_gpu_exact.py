"""GPU exact (24/16-bit) packing against the oracle, bit for bit.

nq_encode_exact must equal the oracle's box-constrained encoder folded into the
exact layout (oq_encode_vector_box then oq_fold_exact): codes with the coset
bit in the low bit of each group's code 7, and the fp16 scale; nq_decode_exact
must equal the oracle's decode of the unfolded store (oq_unfold_exact then
oq_decode_vector).  The lattice step alone (nq_e8_box_quantise) is driven with
groups aimed at its decision boundaries (exact and near coset ties, rounding
ties, tied move costs, values outside the box).  The entropy stage codes an
exact store's codes as they are.
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


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u32(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def box_groups(seed: int, n: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    sign = lambda: rng.choice([-1.0, 1.0], (n, 8))
    base = rng.integers(-4, 4, (n, 8)).astype(np.float64)
    sets = [
        rng.normal(0, 1, (n, 8)),
        rng.normal(0, 2.5, (n, 8)),
        rng.uniform(-6, 6, (n, 8)),                             # outside the box too
        base + 0.25 * sign(),                                   # coset ties
        base + (0.25 + rng.normal(0, 1e-6, (n, 8))) * sign(),
        base + 0.5 * sign(),                                    # rounding ties
        base + rng.normal(0, 1e-6, (n, 8)),
        base,                                                   # integers (odd sums: tied costs)
        np.where(rng.random((n, 8)) < 0.5, base, base + 0.5),
        rng.choice([-4.5, -3.5, 3.5, 4.5, 3.75, -3.75], (n, 8)),  # at and past the box edges
        rng.normal(0, 1, (n, 8)) * 1e-30,
    ]
    y = np.concatenate(sets).astype(np.float32)
    y[rng.random(y.shape) < 0.01] = -0.0
    return y


def folded(codes, coset, bits):
    c = codes.astype(np.uint32)
    bit = np.uint32(1 << (7 * bits))
    return (c & ~bit) | (coset.astype(np.uint32) << np.uint32(7 * bits))


@pytest.mark.parametrize("bits", [2, 3])
def test_box_step_matches_oracle(nq, oq, bits):
    y = box_groups(11 + bits, 20000)
    y = y[np.random.default_rng(4).permutation(len(y))]
    rc, rh, _ = oq.e8_box_codes(y, bits)
    codes, coset = nq.nq_e8_box_quantise(torch.from_numpy(y).cuda(), bits)
    torch.cuda.synchronize()
    got = codes.cpu().numpy().view(np.uint32)
    want = folded(rc, rh, bits)
    bad = np.nonzero((got != want) | (coset.cpu().numpy().astype(np.int32) != rh))[0]
    assert bad.size == 0, (bad.size, y[bad[:3]], got[bad[:3]], want[bad[:3]])


def oracle_exact(oq, x, bits, rope=False, c=None, s=None):
    w, m = oq.encode_vectors_box(x, bits, rope=rope, c=c, s=s)
    return oq.fold_exact(w, m, bits)


def run_case(nq, oq, wl, units, T, bk, bv, evict_pct=0, W=16, strided=False, slot0=0,
             pos_base=0):
    Ks, Vs = [], []
    for u in range(units):
        K, V = synth.gen_layer(wl, u, "cuda", tokens=T)
        Ks.append(K)
        Vs.append(V)
    K, V = torch.stack(Ks), torch.stack(Vs)
    if strided:  # a view with padding between heads and units
        big = torch.zeros(units, wl.heads + 1, T + 8, 128, dtype=torch.bfloat16, device="cuda")
        big[:, :wl.heads, :T] = K
        K = big[:, :wl.heads, :T]
    kept = None
    n = T
    if evict_pct:
        scores = nq.nq_score(K, W)
        kept = nq.nq_select(scores, W, evict_pct)
        n = kept.shape[1]
    max_pos = pos_base + T
    rope = nq.rope_tables(wl.theta, max_pos)
    ks = nq.ExactStore.empty(units, wl.heads, slot0 + n, bk)
    vs = nq.ExactStore.empty(units, wl.heads, slot0 + n, bv)
    nq.nq_encode_exact(K, V, ks, vs, n, rope, max_pos, kept=kept, pos_base=pos_base, slot0=slot0)
    Kd = torch.empty(units, wl.heads, n, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    nq.nq_decode_exact(ks, vs, n, Kd, Vd, rope, max_pos, positions=kept, pos_base=pos_base,
                       slot0=slot0)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    kp = None if kept is None else kept.cpu().numpy()
    for u in range(units):
        src = np.arange(n) if kp is None else kp[u].astype(np.int64)
        c, s = oq.rope_cs(wl.theta, pos_base + src)
        H = wl.heads
        Kx = u16(K[u])[:, src].reshape(-1, 128)
        Vx = u16(V[u])[:, src].reshape(-1, 128)
        cc, ss = np.tile(c, (H, 1)), np.tile(s, (H, 1))
        kw, ksig = oracle_exact(oq, Kx, bk, rope=True, c=cc, s=ss)
        vw, vsig = oracle_exact(oq, Vx, bv)
        assert np.array_equal(u32(ks.codes[u, :, slot0:slot0 + n]).reshape(-1, 4 * bk), kw)
        assert np.array_equal(u16(ks.sigma[u, :, slot0:slot0 + n]).reshape(-1), ksig)
        assert np.array_equal(u32(vs.codes[u, :, slot0:slot0 + n]).reshape(-1, 4 * bv), vw)
        assert np.array_equal(u16(vs.sigma[u, :, slot0:slot0 + n]).reshape(-1), vsig)
        kr, km = oq.unfold_exact(kw, ksig, bk)
        vr, vm = oq.unfold_exact(vw, vsig, bv)
        Ko = oq.decode_vectors(kr, km, bk, rope=True, c=cc, s=ss)
        Vo = oq.decode_vectors(vr, vm, bv)
        assert np.array_equal(u16(Kd[u]).reshape(-1, 128), Ko)
        assert np.array_equal(u16(Vd[u]).reshape(-1, 128), Vo)
    return ks, vs, n


@pytest.mark.parametrize("name,units,T,bk,bv,pct", [
    ("tiny", 1, 2048, 3, 2, 0),
    ("mistral7b_32k", 2, 1000, 3, 2, 60),
    ("qwen25_7b_64k", 3, 777, 3, 2, 35),
    ("decode_append", 2, 300, 2, 2, 0),
    ("mistral7b_32k", 1, 513, 3, 3, 0),
])
def test_exact_encode_decode_match_oracle(nq, oq, name, units, T, bk, bv, pct):
    run_case(nq, oq, synth.WORKLOADS[name], units, T, bk, bv, evict_pct=pct)


def test_exact_strided_offsets(nq, oq):
    run_case(nq, oq, synth.WORKLOADS["mistral7b_32k"], 2, 257, 3, 2, strided=True, slot0=5,
             pos_base=100)


def test_exact_degenerate_vectors(nq, oq):
    """Zero rows (sigma 0), a saturated scale (coordinates far outside the
    box), tiny values, exact lattice-like inputs; inputs within the library's
    contract (|x| <= 2^30)."""
    H, T = 2, 40
    x = torch.randn(1, H, T, 128, device="cuda")
    x[0, 0, 0] = 0
    x[0, 0, 1] = 1e9
    x[0, 0, 5] = -1e9 * (torch.arange(128, device="cuda") % 2)
    x[0, 1, 2] = -1e-30
    x[0, 1, 3] = torch.arange(128, device="cuda") % 3 - 1.0
    x[0, 1, 4] = 0.5
    K = x.to(torch.bfloat16)
    V = (x * 3).to(torch.bfloat16)
    rope = nq.rope_tables(1e4, T)
    ks = nq.ExactStore.empty(1, H, T, 3)
    vs = nq.ExactStore.empty(1, H, T, 2)
    nq.nq_encode_exact(K, V, ks, vs, T, rope, T)
    torch.cuda.synchronize()
    c, s = oq.rope_cs(1e4, np.arange(T))
    kw, ksig = oracle_exact(oq, u16(K[0]).reshape(-1, 128), 3, rope=True, c=np.tile(c, (H, 1)),
                            s=np.tile(s, (H, 1)))
    vw, vsig = oracle_exact(oq, u16(V[0]).reshape(-1, 128), 2)
    assert np.array_equal(u32(ks.codes[0]).reshape(-1, 12), kw)
    assert np.array_equal(u16(ks.sigma[0]).reshape(-1), ksig)
    assert np.array_equal(u32(vs.codes[0]).reshape(-1, 8), vw)
    assert np.array_equal(u16(vs.sigma[0]).reshape(-1), vsig)
    assert u16(ks.sigma[0])[0, 1] == 0x7BFF  # the saturated scale, 65504


def test_exact_store_size(nq):
    L = nq.lib()
    assert L.nq_packed_exact_bytes_per_vector(3) == 50
    assert L.nq_packed_exact_bytes_per_vector(2) == 34
    assert L.nq_packed_exact_bytes_per_vector(4) == -1


def test_exact_codes_through_the_entropy_stage(nq, oq):
    ks, vs, n = run_case(nq, oq, synth.WORKLOADS["mistral7b_32k"], 2, 600, 3, 2)
    for st in (ks, vs):
        coded = nq.nq_entropy_encode(st.codes_store(), n, delta=True)
        freq, offsets, words = oq.entropy_encode_store(u32(st.codes), st.bits, True)
        assert np.array_equal(coded.offsets.cpu().numpy().view(np.uint32), offsets)
        assert np.array_equal(coded.words[:words.size].cpu().numpy().view(np.uint16), words)
        back = nq.ExactStore.empty(2, st.codes.shape[1], n, st.bits)
        nq.nq_entropy_decode(coded, back.codes_store())
        torch.cuda.synchronize()
        assert torch.equal(back.codes, st.codes)


def test_exact_rejects_bad_stores(nq):
    L = nq.lib()
    K = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16, device="cuda")
    st = nq.ExactStore.empty(1, 1, 16, 3)
    d = st.desc()
    d.bits = 4
    rope = nq.rope_tables(1e4, 16)
    import ctypes

    rc = L.nq_encode_exact(nq._ptr(K), nq.kv_strides(K), None, nq.KVStrides(0, 0, 0), 1, 1, 16, 16,
                           None, 0, 0, nq._ptr(rope), 16, ctypes.byref(d), None, 0, None)
    assert rc == nq.NQ_ERR_INVALID
    d = st.desc()
    d.sigma = st.sigma.data_ptr() + 1  # misaligned scale array
    rc = L.nq_encode_exact(nq._ptr(K), nq.kv_strides(K), None, nq.KVStrides(0, 0, 0), 1, 1, 16, 16,
                           None, 0, 0, nq._ptr(rope), 16, ctypes.byref(d), None, 0, None)
    assert rc == nq.NQ_ERR_INVALID and "2-byte" in L.nq_last_error().decode()
