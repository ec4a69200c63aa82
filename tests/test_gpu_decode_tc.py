"""GPU decode on the tensor cores against the oracle, bit for bit.

nq_decode runs its 128-point transform as an f16 matrix product on the tensor
cores, in tiles of 128 vectors: 8 / hg slot tiles of a group of hg heads
(hg = the largest divisor of the head count up to 8; keys need hg >= 3).  By
default it does so only for calls large enough to pay for its per-CTA setup,
so this file selects that engine for every size (nq_set_decode_engine) and
checks it against the CUDA-core engine as well.  The cases here drive the
tensor-core path with stores that span the whole code space (random code
words, every coset mask, scales from zero and subnormal to the largest fp16),
ragged slot counts on both sides of the 16-slot tile, every head-group size
1..8 (with idle rows for 3, 5, 6 and 7), several head groups (16 and 24
heads), kept-list positions with one and two RoPE tables per tile, output
views with padding and token-major output views, slot and position offsets,
and the exact layout.  Every
decoded bf16 element must equal the oracle's decode of the same store.
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
    nqmod.set_decode_engine(nqmod.DECODE_TENSOR_CORES)
    yield nqmod
    nqmod.set_decode_engine(nqmod.DECODE_AUTO)


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u32(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def random_store(nq, units, heads, cap, bits, seed):
    """Packed store with uniformly random code words and coset masks, and
    scales drawn from every fp16 range (0, subnormal, normal, the largest)."""
    g = np.random.default_rng(seed)
    st = nq.PackedStore.empty(units, heads, cap, bits)
    words = g.integers(0, 2**32, size=(units, heads, cap, 4 * bits), dtype=np.uint64).astype(np.uint32)
    mask = g.integers(0, 2**16, size=(units, heads, cap), dtype=np.uint32)
    kind = g.integers(0, 4, size=(units, heads, cap))
    sig = np.where(kind == 0, g.integers(0x3000, 0x4C00, size=kind.shape),       # typical
          np.where(kind == 1, g.integers(0, 0x0400, size=kind.shape),             # 0 and subnormal
          np.where(kind == 2, g.integers(0x0400, 0x7C00, size=kind.shape),        # any normal
                   0x7BFF))).astype(np.uint32)                                      # 65504
    meta = mask | (sig << 16)
    st.codes.copy_(torch.from_numpy(words.view(np.int32)))
    st.meta.copy_(torch.from_numpy(meta.view(np.int32)))
    return st


def oracle_decode(oq, store, u, slot0, n, bits, rope, theta, positions):
    c = s = None
    H = store.meta.shape[1]
    if rope:
        c, s = oq.rope_cs(theta, positions)
        c, s = np.tile(c, (H, 1)), np.tile(s, (H, 1))
    words = u32(store.codes[u, :, slot0:slot0 + n]).reshape(-1, 4 * bits)
    meta = u32(store.meta[u, :, slot0:slot0 + n]).reshape(-1)
    return oq.decode_vectors(words, meta, bits, rope=rope, c=c, s=s).reshape(H, n, 128)


@pytest.mark.parametrize("heads,n,bk,bv", [
    (8, 1, 3, 2), (8, 15, 2, 3), (8, 16, 3, 3), (8, 17, 2, 2), (8, 255, 3, 2),
    (16, 1000, 3, 2), (24, 333, 2, 3), (8, 4100, 3, 2),
    (4, 1000, 3, 2), (4, 17, 2, 3), (12, 333, 3, 2), (3, 257, 2, 3), (5, 100, 3, 2),
    (7, 77, 3, 3), (6, 48, 2, 2), (2, 300, 3, 2), (1, 500, 3, 3), (1, 15, 2, 2),
])
def test_random_stores_match_oracle(nq, oq, heads, n, bk, bv):
    units, theta = 3, 5e5
    ks = random_store(nq, units, heads, n, bk, 11 + n)
    vs = random_store(nq, units, heads, n, bv, 12 + n)
    rope = nq.rope_tables(theta, n)
    Kd = torch.empty(units, heads, n, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    nq.nq_decode(ks, vs, n, Kd, Vd, rope, n)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    pos = np.arange(n)
    for u in range(units):
        assert np.array_equal(u16(Kd[u]), oracle_decode(oq, ks, u, 0, n, bk, True, theta, pos))
        assert np.array_equal(u16(Vd[u]), oracle_decode(oq, vs, u, 0, n, bv, False, theta, pos))


@pytest.mark.parametrize("heads", [8, 4, 3])
def test_kept_positions_views_and_offsets(nq, oq, heads):
    """Evicted-cache positions, padded output views, slot0 > 0, pos_base > 0
    (one RoPE table per tile for 8 heads, two for 4 and 3)."""
    units, n, slot0, pos_base, theta = 2, 300, 37, 1000, 1e6
    ks = random_store(nq, units, heads, 400, 3, 5)
    vs = random_store(nq, units, heads, 400, 2, 6)
    g = np.random.default_rng(3)
    kept = np.stack([np.sort(g.choice(5000, n, replace=False)) for _ in range(units)]).astype(np.int32)
    positions = torch.from_numpy(kept).cuda()
    max_pos = pos_base + 5000
    rope = nq.rope_tables(theta, max_pos)
    out_k = torch.zeros(units, heads + 1, 320, 144, dtype=torch.bfloat16, device="cuda")
    out_v = torch.zeros_like(out_k)
    Ko, Vo = out_k[:, :heads, 10:310, 16:], out_v[:, :heads, 10:310, :128]
    nq.nq_decode(ks, vs, n, Ko, Vo, rope, max_pos, positions=positions, pos_base=pos_base,
                 slot0=slot0)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    for u in range(units):
        Kr = oracle_decode(oq, ks, u, slot0, n, 3, True, theta, pos_base + kept[u].astype(np.int64))
        Vr = oracle_decode(oq, vs, u, slot0, n, 2, False, theta, None)
        assert np.array_equal(u16(Ko[u]), Kr) and np.array_equal(u16(Vo[u]), Vr)
    # nothing outside the views was written
    for o in (out_k, out_v):
        assert torch.count_nonzero(o[:, heads]) == 0
        assert torch.count_nonzero(o[:, :, :10]) == 0 and torch.count_nonzero(o[:, :, 310:]) == 0
    assert torch.count_nonzero(out_k[..., :16]) == 0 and torch.count_nonzero(out_v[..., 128:]) == 0


@pytest.mark.parametrize("engine", ["tensor", "cuda"])
@pytest.mark.parametrize("heads", [8, 4, 3])
def test_token_major_output_views(nq, oq, heads, engine):
    """Outputs held token-major ([units][tokens][heads][128], passed as a permuted
    view, so the head stride is below the token stride): the paired key rows
    (8 and 4 heads) store boxes of 2 heads x 16 tokens through a map that lists
    heads before tokens, which must land on the same elements."""
    units, n, theta = 2, 277, 1e6
    ks = random_store(nq, units, heads, 300, 3, 21)
    vs = random_store(nq, units, heads, 300, 2, 22)
    max_pos = 4096
    rope = nq.rope_tables(theta, max_pos)
    out_k = torch.zeros(units, n + 9, heads, 128, dtype=torch.bfloat16, device="cuda")
    out_v = torch.zeros_like(out_k)
    Ko, Vo = out_k[:, 4:4 + n].permute(0, 2, 1, 3), out_v[:, 4:4 + n].permute(0, 2, 1, 3)
    if engine == "cuda":
        nq.set_decode_engine(nq.DECODE_CUDA_CORES)
    try:
        nq.nq_decode(ks, vs, n, Ko, Vo, rope, max_pos)
        torch.cuda.synchronize()
    finally:
        nq.set_decode_engine(nq.DECODE_TENSOR_CORES)
    assert nq.device_error() == 0
    for u in range(units):
        Kr = oracle_decode(oq, ks, u, 0, n, 3, True, theta, np.arange(n, dtype=np.int64))
        Vr = oracle_decode(oq, vs, u, 0, n, 2, False, theta, None)
        assert np.array_equal(u16(Ko[u]), Kr) and np.array_equal(u16(Vo[u]), Vr)
    for o in (out_k, out_v):  # nothing outside the views was written
        assert torch.count_nonzero(o[:, :4]) == 0 and torch.count_nonzero(o[:, 4 + n:]) == 0


@pytest.mark.parametrize("name", ["tiny", "decode_append", "qwen25_7b_64k", "mistral7b_32k"])
def test_encoded_caches_match_oracle(nq, oq, name):
    """Real encodes (the codes the method produces) through the tensor-core decode."""
    wl = synth.WORKLOADS[name]
    units, T = 2, 1500
    K = torch.stack([synth.gen_layer(wl, u, "cuda", tokens=T)[0] for u in range(units)])
    V = torch.stack([synth.gen_layer(wl, u, "cuda", tokens=T)[1] for u in range(units)])
    codec = nq.Codec(units, wl.heads, T, wl.theta, wl.bits_k, wl.bits_v, window=wl.window,
                     evict_pct=wl.evict_pct)
    codec.encode(K, V)
    Kd = torch.empty(units, wl.heads, codec.n, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    codec.decode(Kd, Vd)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    for u in range(units):
        pos = (codec.kept[u].cpu().numpy().astype(np.int64) if codec.evict
               else np.arange(codec.n))
        assert np.array_equal(u16(Kd[u]), oracle_decode(oq, codec.k_store, u, 0, codec.n, wl.bits_k,
                                                        True, wl.theta, pos))
        assert np.array_equal(u16(Vd[u]), oracle_decode(oq, codec.v_store, u, 0, codec.n,
                                                        wl.bits_v, False, wl.theta, pos))


def test_exact_layout_random_stores(nq, oq):
    """Exact-layout stores with random codes and scales (8 heads: tensor-core path)."""
    units, heads, n, theta = 2, 8, 700, 1e4
    g = np.random.default_rng(21)
    stores, refs = [], []
    for bits in (3, 2):
        st = nq.ExactStore.empty(units, heads, n, bits)
        words = g.integers(0, 2**32, size=(units, heads, n, 4 * bits), dtype=np.uint64).astype(np.uint32)
        sig = g.integers(0, 0x7C00, size=(units, heads, n)).astype(np.uint16)
        st.codes.copy_(torch.from_numpy(words.view(np.int32)))
        st.sigma.copy_(torch.from_numpy(sig.view(np.int16)))
        stores.append(st)
        refs.append((words, sig))
    rope = nq.rope_tables(theta, n)
    Kd = torch.empty(units, heads, n, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    nq.nq_decode_exact(stores[0], stores[1], n, Kd, Vd, rope, n)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    c, s = oq.rope_cs(theta, np.arange(n))
    c, s = np.tile(c, (heads, 1)), np.tile(s, (heads, 1))
    for u in range(units):
        for out, (words, sig), bits, rope_on in ((Kd, refs[0], 3, True), (Vd, refs[1], 2, False)):
            w, m = oq.unfold_exact(words[u].reshape(-1, 4 * bits), sig[u].reshape(-1), bits)
            ref = oq.decode_vectors(w, m, bits, rope=rope_on, c=c if rope_on else None,
                                    s=s if rope_on else None).reshape(heads, n, 128)
            assert np.array_equal(u16(out[u]), ref)


@pytest.mark.parametrize("heads,n,exact", [(8, 37, False), (16, 700, False), (8, 129, True),
                                            (4, 500, False), (3, 33, True), (1, 100, False)])
def test_engines_give_the_same_bits(nq, heads, n, exact):
    """The tensor-core and CUDA-core engines decode the same store to the same bits."""
    units, theta = 2, 1e6
    if exact:
        ks, vs = nq.ExactStore.empty(units, heads, n, 3), nq.ExactStore.empty(units, heads, n, 2)
        for st, seed in ((ks, 1), (vs, 2)):
            g = np.random.default_rng(seed)
            st.codes.copy_(torch.from_numpy(g.integers(0, 2**32, size=st.codes.shape,
                                                       dtype=np.uint64).astype(np.uint32).view(np.int32)))
            st.sigma.copy_(torch.from_numpy(g.integers(0, 0x7C00, size=st.sigma.shape)
                                            .astype(np.uint16).view(np.int16)))
        dec = nq.nq_decode_exact
    else:
        ks, vs = random_store(nq, units, heads, n, 3, 31), random_store(nq, units, heads, n, 2, 32)
        dec = nq.nq_decode
    rope = nq.rope_tables(theta, n)
    outs = []
    try:
        for engine in (nq.DECODE_TENSOR_CORES, nq.DECODE_CUDA_CORES):
            nq.set_decode_engine(engine)
            Kd = torch.empty(units, heads, n, 128, dtype=torch.bfloat16, device="cuda")
            Vd = torch.empty_like(Kd)
            dec(ks, vs, n, Kd, Vd, rope, n)
            torch.cuda.synchronize()
            outs.append((u16(Kd), u16(Vd)))
    finally:
        nq.set_decode_engine(nq.DECODE_TENSOR_CORES)
    assert nq.device_error() == 0
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])

