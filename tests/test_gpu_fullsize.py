"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (every layer of the cache in one call per stage), checked on
sampled layers / slots that the CPU oracle recomputes one by one, plus
properties that hold at any size (kept counts, BOS + window kept, ascending
positions, protected layers bit-identical).

Workloads (seeded synthetic caches, e8_lattice_vector_nq_b200/synth.py):
  mistral7b_32k   32 L x 8 H x 32768 T, theta 1e6, K3V2, 60 % eviction, W 64
  llama3_8b_128k  32 L x 8 H x 131072 T, theta 5e5, K3V2, no eviction
  qwen25_7b_64k   28 L x 4 H x 65536 T, theta 1e6, layers 0,1,26,27 bf16,
                  others K3V2 with 35 % eviction, W 128
  decode_append   64 sequences x 32 L x 8 H, 16384-token caches, K2V2, one
                  token appended per (sequence, layer) for 256 steps, layer
                  s mod 32 of every sequence decoded at sampled steps
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


def gen_cache(wl, device="cuda"):
    K = torch.empty(wl.layers, wl.heads, wl.tokens, 128, dtype=torch.bfloat16, device=device)
    V = torch.empty_like(K)
    for l in range(wl.layers):
        k, v = synth.gen_layer(wl, l, device)
        K[l].copy_(k)
        V[l].copy_(v)
    return K, V


def check_unit(oq, wl, Ku, Vu, codec_unit, kept_gpu, slots, K_dec, V_dec):
    """Oracle encode/decode of the given slots of one unit vs the GPU results."""
    src = slots if kept_gpu is None else kept_gpu[slots]  # source token = RoPE position
    Kh = u16(Ku)[:, src]  # [H][len][128]
    Vh = u16(Vu)[:, src]
    H = Ku.shape[0]
    # vectors in (slot, head) order, each with its slot's (cos, sin) row
    c, s = oq.rope_cs(wl.theta, src)
    kc, km, _ = oq.encode_vectors(Kh.transpose(1, 0, 2).reshape(-1, 128), wl.bits_k, rope=True,
                                  c=np.repeat(c, H, 0), s=np.repeat(s, H, 0))
    vc, vm, _ = oq.encode_vectors(Vh.transpose(1, 0, 2).reshape(-1, 128), wl.bits_v)
    gk_c, gk_m, gv_c, gv_m = codec_unit
    gkc = u32(gk_c)[:, slots].transpose(1, 0, 2).reshape(-1, 4 * wl.bits_k)
    gkm = u32(gk_m)[:, slots].T.reshape(-1)
    gvc = u32(gv_c)[:, slots].transpose(1, 0, 2).reshape(-1, 4 * wl.bits_v)
    gvm = u32(gv_m)[:, slots].T.reshape(-1)
    assert np.array_equal(gkc, kc) and np.array_equal(gkm, km), "K codes differ"
    assert np.array_equal(gvc, vc) and np.array_equal(gvm, vm), "V codes differ"
    if K_dec is not None:
        Ko = oq.decode_vectors(kc, km, wl.bits_k, rope=True, c=np.repeat(c, H, 0),
                               s=np.repeat(s, H, 0))
        Vo = oq.decode_vectors(vc, vm, wl.bits_v)
        gK = u16(K_dec)[:, slots].transpose(1, 0, 2).reshape(-1, 128)
        gV = u16(V_dec)[:, slots].transpose(1, 0, 2).reshape(-1, 128)
        assert np.array_equal(gK, Ko) and np.array_equal(gV, Vo), "decoded rows differ"


def kept_properties(kept, T, W, n):
    k = kept.cpu().numpy()
    assert k.shape[1] == n
    assert np.all(k[:, 0] == 0)
    assert np.all(k[:, -W:] == np.arange(T - W, T)[None])
    assert np.all(np.diff(k, axis=1) > 0)


def run_evicting_workload(nq, oq, wl, sample_layers, protected=()):
    torch.manual_seed(0)
    K, V = gen_cache(wl)
    cache = nq.LayeredCache(wl.layers, wl.heads, wl.tokens, wl.theta, wl.bits_k, wl.bits_v,
                            wl.window, wl.evict_pct, protected)
    cache.encode(K, V)
    codec = cache.codec
    Kd = torch.empty(codec.units, wl.heads, codec.n, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    cache.decode_quantised(Kd, Vd)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    if codec.evict:
        kept_properties(codec.kept, wl.tokens, wl.window, codec.n)
    for l in protected:
        assert torch.equal(cache.kept_bf16_K[l], K[l]) and torch.equal(cache.kept_bf16_V[l], V[l])
    rng = np.random.default_rng(123)
    for l in sample_layers:
        u = l - cache.q0
        kept = None
        if codec.evict:
            s_or = oq.score_unit(u16(K[l]), wl.window)
            s_gpu = codec.scores[u].cpu().numpy()
            assert np.max(np.abs(s_gpu - s_or)) <= 1e-12 * np.max(np.abs(s_or))
            k_or = oq.select(s_or, wl.window, wl.evict_pct)
            kept = codec.kept[u].cpu().numpy()
            diff = np.setxor1d(k_or, kept)
            assert diff.size <= max(2, 1e-6 * wl.tokens), diff
        slots = np.sort(rng.choice(codec.n, size=min(codec.n, 3000), replace=False))
        unit = (codec.k_store.codes[u], codec.k_store.meta[u], codec.v_store.codes[u],
                codec.v_store.meta[u])
        check_unit(oq, wl, K[l], V[l], unit, kept, slots, Kd[u], Vd[u])


def test_mistral7b_32k_full(nq, oq):
    wl = synth.WORKLOADS["mistral7b_32k"]
    run_evicting_workload(nq, oq, wl, sample_layers=[0, 13, 31])


def test_llama3_8b_128k_full(nq, oq):
    wl = synth.WORKLOADS["llama3_8b_128k"]
    run_evicting_workload(nq, oq, wl, sample_layers=[0, 31])


def test_qwen25_7b_64k_full(nq, oq):
    wl = synth.WORKLOADS["qwen25_7b_64k"]
    run_evicting_workload(nq, oq, wl, sample_layers=[2, 25], protected=wl.protected_layers)


def test_decode_append_full(nq, oq):
    wl = synth.WORKLOADS["decode_append"]
    S, L, H, T0 = wl.sequences, wl.layers, wl.heads, wl.tokens
    cap = T0 + wl.append_steps
    store = nq.AppendStore(S, L, H, cap, wl.theta, wl.bits_k, wl.bits_v)
    check_seqs = (0, 21, 63)
    kept_inputs = {}
    for s in range(S):
        Ks = torch.empty(L, H, T0, 128, dtype=torch.bfloat16, device="cuda")
        Vs = torch.empty_like(Ks)
        for l in range(L):
            k, v = synth.gen_layer(wl, l, "cuda", seed_offset=1000 * s)
            Ks[l].copy_(k)
            Vs[l].copy_(v)
        store.fill(s, Ks, Vs)
        if s in check_seqs:
            kept_inputs[s] = (Ks, Vs)
    appended = {}
    checks = {0, 1, 31, 255}
    for step in range(wl.append_steps):
        pos = T0 + step
        g = torch.Generator(device="cuda")
        g.manual_seed(wl.seed * 1000003 + step)
        Kn = (torch.randn(S * L, H, 1, 128, generator=g, device="cuda") * 2).to(torch.bfloat16)
        Vn = torch.randn(S * L, H, 1, 128, generator=g, device="cuda").to(torch.bfloat16)
        store.append(Kn, Vn, pos)
        for s in check_seqs:
            appended[(s, step)] = (Kn.view(S, L, H, 1, 128)[s].clone(),
                                   Vn.view(S, L, H, 1, 128)[s].clone())
        if step in checks:
            layer = step % L
            n = pos + 1
            Ko = torch.empty(S, H, n, 128, dtype=torch.bfloat16, device="cuda")
            Vo = torch.empty_like(Ko)
            store.decode_layer(layer, n, Ko, Vo)
            torch.cuda.synchronize()
            for s in check_seqs:
                Kfull = torch.cat([kept_inputs[s][0][layer]] +
                                  [appended[(s, t)][0][layer] for t in range(step + 1)], dim=1)
                Vfull = torch.cat([kept_inputs[s][1][layer]] +
                                  [appended[(s, t)][1][layer] for t in range(step + 1)], dim=1)
                slots = np.concatenate([np.sort(np.random.default_rng(step + s).choice(
                    T0, 500, replace=False)), np.arange(T0, n)])
                unit = (store.k.codes.view(S, L, H, cap, -1)[s, layer],
                        store.k.meta.view(S, L, H, cap)[s, layer],
                        store.v.codes.view(S, L, H, cap, -1)[s, layer],
                        store.v.meta.view(S, L, H, cap)[s, layer])
                check_unit(oq, wl, Kfull, Vfull, unit, None, slots, Ko[s], Vo[s])
    assert nq.device_error() == 0
