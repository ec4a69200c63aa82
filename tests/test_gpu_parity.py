"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Codes, coset masks, fp16 scales and reconstructed bf16 values must match bit
for bit: both sides run the same fp32 operation sequence.  Kept-token sets
must match exactly except where the fp64 scores of the two sides (different
summation orders) straddle the selection threshold within 1e-12 relative;
such positions are counted and must stay below 1e-6 of the tokens.
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


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def make_cache(wl, units, T, device="cuda", seed_offset=0):
    Ks, Vs = [], []
    for u in range(units):
        K, V = synth.gen_layer(wl, u, device, tokens=T, seed_offset=seed_offset)
        Ks.append(K)
        Vs.append(V)
    return torch.stack(Ks), torch.stack(Vs)


def oracle_encode(oq, K, V, n, kept, theta, bk, bv, pos_base=0):
    out = []
    for u in range(K.shape[0]):
        kp = None if kept is None else kept[u]
        out.append(oq.encode_unit(u16(K[u]), u16(V[u]), n, kept=kp, pos_base=pos_base, theta=theta,
                                  bits_k=bk, bits_v=bv))
    return out


def assert_packed_equal(store, ref, key, slot0=0):
    codes = u32(store.codes)
    meta = u32(store.meta)
    n = ref[0][f"{key}_meta"].shape[1]
    for u, r in enumerate(ref):
        got_c = codes[u, :, slot0:slot0 + n]
        got_m = meta[u, :, slot0:slot0 + n]
        bad = np.any(got_c != r[f"{key}_codes"], -1) | (got_m != r[f"{key}_meta"])
        assert not bad.any(), f"{key}: {int(bad.sum())} vectors differ in unit {u} (first {np.argwhere(bad)[:3].tolist()})"


def run_codec_case(nq, oq, wl, units, T, W, pct, bk=3, bv=2, device="cuda"):
    K, V = make_cache(wl, units, T, device)
    codec = nq.Codec(units, wl.heads, T, wl.theta, bk, bv, window=W, evict_pct=pct)
    codec.encode(K, V)
    Kd = torch.empty(units, wl.heads, codec.n, 128, dtype=torch.bfloat16, device=device)
    Vd = torch.empty_like(Kd)
    codec.decode(Kd, Vd)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    kept = None
    if codec.evict:
        kept_gpu = codec.kept.cpu().numpy()
        kept = []
        for u in range(units):
            s_or = oq.score_unit(u16(K[u]), W)
            s_gpu = codec.scores[u].cpu().numpy()
            assert np.max(np.abs(s_gpu - s_or)) <= 1e-12 * np.max(np.abs(s_or))
            k_or = oq.select(s_or, W, pct)
            if not np.array_equal(k_or, kept_gpu[u]):
                # only positions whose score ties the threshold within 1e-12 may differ
                diff = np.setxor1d(k_or, kept_gpu[u])
                thr = np.sort(s_or[1:T - W])[::-1][codec.n - 1 - W - 1]
                assert np.all(np.abs(s_or[diff] - thr) <= 1e-12 * np.abs(thr)), diff
                assert diff.size <= max(2, 1e-6 * T)
            kept.append(kept_gpu[u])  # encode parity on the GPU's (valid) set
        kept = np.stack(kept)
    ref = oracle_encode(oq, K, V, codec.n, kept, wl.theta, bk, bv)
    assert_packed_equal(codec.k_store, ref, "k")
    assert_packed_equal(codec.v_store, ref, "v")
    for u, r in enumerate(ref):
        Ko, Vo = oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"],
                                positions=None if kept is None else kept[u], theta=wl.theta,
                                bits_k=bk, bits_v=bv)
        assert np.array_equal(u16(Kd[u]), Ko), "decoded K differs"
        assert np.array_equal(u16(Vd[u]), Vo), "decoded V differs"
    return codec


def test_tiny_workload_exact(nq, oq):
    """1 layer x 8 heads x 2048 tokens, theta 1e4, K3V2, no eviction."""
    wl = synth.WORKLOADS["tiny"]
    run_codec_case(nq, oq, wl, units=1, T=2048, W=64, pct=0)


def test_mistral_shape_eviction(nq, oq):
    """Mistral-shaped heads/theta with 60% eviction, window 64, ragged T."""
    wl = synth.WORKLOADS["mistral7b_32k"]
    run_codec_case(nq, oq, wl, units=2, T=3001, W=64, pct=60)


def test_qwen_shape_eviction(nq, oq):
    """4 KV heads, theta 1e6, 5 (head, channel) pairs x20, 35% eviction, window 128."""
    wl = synth.WORKLOADS["qwen25_7b_64k"]
    run_codec_case(nq, oq, wl, units=2, T=2600, W=128, pct=35)


@pytest.mark.parametrize("heads", [1, 3, 12])
def test_head_counts_and_k2v2(nq, oq, heads):
    wl = synth.Workload("h", 1, heads, 700, 5e5, 7, bits_k=2, bits_v=2)
    run_codec_case(nq, oq, wl, units=1, T=700, W=16, pct=50, bk=2, bv=2)


def test_k3v3_and_full_eviction(nq, oq):
    wl = synth.Workload("x", 1, 8, 513, 1e4, 8)
    run_codec_case(nq, oq, wl, units=1, T=513, W=32, pct=100, bk=3, bv=3)


def test_strided_inputs_slot_offsets_positions(nq, oq):
    """Non-contiguous K/V views, slot0 > 0, pos_base > 0, explicit positions."""
    wl = synth.Workload("s", 1, 4, 300, 1e6, 9)
    big_k = torch.zeros(2, 6, 400, 136, dtype=torch.bfloat16, device="cuda")
    big_v = torch.zeros_like(big_k)
    K, V = make_cache(wl, 2, 300)
    big_k[:, 1:5, 50:350, 8:] = K
    big_v[:, 1:5, 50:350, :128] = V
    Kv, Vv = big_k[:, 1:5, 50:350, 8:], big_v[:, 1:5, 50:350, :128]
    n, slot0, pos_base = 300, 37, 1000
    rope = nq.rope_tables(wl.theta, 4096)
    ks = nq.PackedStore.empty(2, 4, 400, 3)
    vs = nq.PackedStore.empty(2, 4, 400, 2)
    nq.nq_encode(Kv, Vv, ks, vs, n, rope, 4096, pos_base=pos_base, slot0=slot0)
    # positions for decode: pos_base + i for slot i, given explicitly
    pos = torch.arange(n, dtype=torch.int32, device="cuda").repeat(2, 1).contiguous()
    out_k = torch.zeros(2, 4, 320, 144, dtype=torch.bfloat16, device="cuda")
    out_v = torch.zeros_like(out_k)
    Ko, Vo = out_k[:, :, 10:310, 16:], out_v[:, :, 10:310, :128]
    nq.nq_decode(ks, vs, n, Ko, Vo, rope, 4096, positions=pos, pos_base=pos_base, slot0=slot0)
    torch.cuda.synchronize()
    ref = oracle_encode(oq, K, V, n, None, wl.theta, 3, 2, pos_base=pos_base)
    assert_packed_equal(ks, ref, "k", slot0=slot0)
    assert_packed_equal(vs, ref, "v", slot0=slot0)
    for u, r in enumerate(ref):
        Kr, Vr = oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"],
                                pos_base=pos_base, theta=wl.theta, bits_k=3, bits_v=2)
        assert np.array_equal(u16(Ko[u]), Kr) and np.array_equal(u16(Vo[u]), Vr)
    # nothing outside the views was written
    assert torch.count_nonzero(out_k[:, :, :10]) == 0 and torch.count_nonzero(out_k[:, :, 310:]) == 0
    assert torch.count_nonzero(out_k[..., :16]) == 0


def test_append_one_token_per_unit(nq, oq):
    """Decode-append regime: each unit appends one token at position P into slot P."""
    wl = synth.WORKLOADS["decode_append"]
    units, P = 6, 16384 + 5
    K, V = make_cache(wl, units, 1)
    rope = nq.rope_tables(wl.theta, 16640)
    ks = nq.PackedStore.empty(units, wl.heads, 16640, 2)
    vs = nq.PackedStore.empty(units, wl.heads, 16640, 2)
    nq.nq_encode(K, V, ks, vs, 1, rope, 16640, pos_base=P, slot0=P)
    Ko = torch.empty(units, wl.heads, 1, 128, dtype=torch.bfloat16, device="cuda")
    Vo = torch.empty_like(Ko)
    nq.nq_decode(ks, vs, 1, Ko, Vo, rope, 16640, pos_base=P, slot0=P)
    torch.cuda.synchronize()
    ref = oracle_encode(oq, K, V, 1, None, wl.theta, 2, 2, pos_base=P)
    assert_packed_equal(ks, ref, "k", slot0=P)
    assert_packed_equal(vs, ref, "v", slot0=P)
    for u, r in enumerate(ref):
        Kr, Vr = oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], pos_base=P,
                                theta=wl.theta, bits_k=2, bits_v=2)
        assert np.array_equal(u16(Ko[u]), Kr) and np.array_equal(u16(Vo[u]), Vr)


def test_degenerate_vectors(nq, oq):
    """Zero rows (sigma 0), saturated scales, exact lattice-like inputs, a single slot."""
    H, T = 2, 40
    x = torch.randn(1, H, T, 128, device="cuda")
    x[0, 0, 0] = 0
    x[0, 0, 1] = 1e9
    x[0, 1, 2] = -1e-30
    x[0, 1, 3] = torch.arange(128, device="cuda") % 3 - 1.0
    x[0, 1, 4] = 0.5
    K = x.to(torch.bfloat16)
    V = (x * 3).to(torch.bfloat16)
    rope = nq.rope_tables(1e4, T)
    ks = nq.PackedStore.empty(1, H, T, 3)
    vs = nq.PackedStore.empty(1, H, T, 2)
    nq.nq_encode(K, V, ks, vs, T, rope, T)
    torch.cuda.synchronize()
    ref = oracle_encode(oq, K, V, T, None, 1e4, 3, 2)
    assert_packed_equal(ks, ref, "k")
    assert_packed_equal(vs, ref, "v")
    assert u32(ks.meta)[0, 0, 0] == 0


def test_score_select_edge_cases(nq, oq):
    """Ties in scores, keep-all, only BOS + window, window = T - 1."""
    T = 4100
    s = torch.tensor(np.repeat(np.arange(41, dtype=np.float64), 100), device="cuda").reshape(1, T)
    s[0, 17] = -0.0
    for W, pct in [(64, 60), (64, 100), (64, 0), (T - 1, 50), (1, 99)]:
        kept = nq.nq_select(s.contiguous(), W, pct)
        ref = oq.select(s[0].cpu().numpy(), W, pct)
        assert np.array_equal(kept[0].cpu().numpy(), ref), (W, pct)


def test_units_zero_and_n_zero_launch_nothing(nq):
    K = torch.zeros(1, 8, 16, 128, dtype=torch.bfloat16, device="cuda")
    rope = nq.rope_tables(1e4, 16)
    ks = nq.PackedStore.empty(1, 8, 16, 3)
    nq.nq_encode(K, None, ks, None, 0, rope, 16)
    torch.cuda.synchronize()
