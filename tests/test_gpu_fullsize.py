"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (every layer of the cache in one call per stage), checked in
full against the CPU oracle on all host cores (oracle/parity.py):

  tiny            1 L x 8 H x 2048 T, theta 1e4, K3V2, no eviction: every vector
  mistral7b_32k   32 L x 8 H x 32768 T, theta 1e6, K3V2, 60 % eviction, W 64:
                  every layer's scores and kept set, every kept vector's codes
                  and decoded rows
  llama3_8b_128k  32 L x 8 H x 131072 T, theta 5e5, K3V2, no eviction: every
                  layer, streamed to the oracle layer by layer
  qwen25_7b_64k   28 L x 4 H x 65536 T, theta 1e6, layers 0,1,26,27 bf16, the
                  others K3V2 with 35 % eviction, W 128: every quantised layer,
                  protected layers bit-identical
  decode_append   64 sequences x 32 L x 8 H, 16384-token caches, K2V2, one
                  token appended per (sequence, layer) for 256 steps: every
                  appended token of every unit; the initial caches of
                  sequences 0, 21 and 63 (all layers); the full reconstruction
                  of layer s mod 32 at steps 0, 1, 31 and 255 for those
                  sequences (a sample, stated as such)

The exact (24/16-bit) layout is checked the same way on every layer of the
Mistral- and Llama-shaped caches (no mismatch is excused there).

Parity rule: kept sets and codes bit-exact except where the
oracle's value lies within 1e-5 relative of a decision boundary; those are
counted, reported and must stay below 1e-6 of the elements; decoded bf16
identical.  Counts are printed (pytest -s) and appended as JSON lines to the
file named by NQ_PARITY_REPORT when set.
"""
import json
import os

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


@pytest.fixture(scope="module")
def pool(oq):
    from oracle import parity

    p = parity.make_pool()
    yield p
    p.shutdown()


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


def report(name, tot):
    from oracle import parity

    line = dict(workload=name, **tot, failures=parity.verdict(tot))
    print(json.dumps(line))
    path = os.environ.get("NQ_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(line) + "\n")
    return line


def assert_parity(name, results):
    from oracle import parity

    tot = parity.merge(results)
    line = report(name, tot)
    assert not line["failures"], line


def kept_properties(kept, T, W, n):
    k = kept.cpu().numpy()
    assert k.shape[1] == n
    assert np.all(k[:, 0] == 0)
    assert np.all(k[:, -W:] == np.arange(T - W, T)[None])
    assert np.all(np.diff(k, axis=1) > 0)


def run_layered(nq, wl, pool, protected=()):
    """Encode + decode the whole cache as the benchmark does, then check every
    quantised layer against the oracle (one worker job per layer)."""
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
    from oracle import parity

    def jobs():
        for u in range(codec.units):
            l = cache.q0 + u
            yield {"K": u16(K[l]), "V": u16(V[l]), "theta": wl.theta, "bits_k": wl.bits_k,
                   "bits_v": wl.bits_v, "window": wl.window,
                   "pct": wl.evict_pct if codec.evict else 0,
                   "gpu_scores": codec.scores[u].cpu().numpy() if codec.evict else None,
                   "gpu_kept": codec.kept[u].cpu().numpy() if codec.evict else None,
                   "gk_codes": u32(codec.k_store.codes[u]), "gk_meta": u32(codec.k_store.meta[u]),
                   "gv_codes": u32(codec.v_store.codes[u]), "gv_meta": u32(codec.v_store.meta[u]),
                   "gK": u16(Kd[u]), "gV": u16(Vd[u])}

    return parity.run_jobs(pool, jobs())


def test_tiny_full(nq, pool):
    wl = synth.WORKLOADS["tiny"]
    assert_parity(wl.name, run_layered(nq, wl, pool))


def test_mistral7b_32k_full(nq, pool):
    wl = synth.WORKLOADS["mistral7b_32k"]
    assert_parity(wl.name, run_layered(nq, wl, pool))


def test_llama3_8b_128k_full(nq, pool):
    wl = synth.WORKLOADS["llama3_8b_128k"]
    assert_parity(wl.name, run_layered(nq, wl, pool))


def test_qwen25_7b_64k_full(nq, pool):
    wl = synth.WORKLOADS["qwen25_7b_64k"]
    assert_parity(wl.name, run_layered(nq, wl, pool, protected=wl.protected_layers))


def test_decode_append_full(nq, pool):
    from oracle import parity

    wl = synth.WORKLOADS["decode_append"]
    S, L, H, T0 = wl.sequences, wl.layers, wl.heads, wl.tokens
    steps = wl.append_steps
    cap = T0 + steps
    store = nq.AppendStore(S, L, H, cap, wl.theta, wl.bits_k, wl.bits_v)
    check_seqs = (0, 21, 63)
    inputs = {}
    for s in range(S):
        Ks = torch.empty(L, H, T0, 128, dtype=torch.bfloat16, device="cuda")
        Vs = torch.empty_like(Ks)
        for l in range(L):
            k, v = synth.gen_layer(wl, l, "cuda", seed_offset=1000 * s)
            Ks[l].copy_(k)
            Vs[l].copy_(v)
        store.fill(s, Ks, Vs)
        if s in check_seqs:
            inputs[s] = (Ks, Vs)
    K_app = torch.empty(steps, S * L, H, 128, dtype=torch.bfloat16, device="cuda")
    V_app = torch.empty_like(K_app)
    checks = {0: None, 1: None, 31: None, 255: None}
    decoded = {}
    for step in range(steps):
        pos = T0 + step
        g = torch.Generator(device="cuda")
        g.manual_seed(wl.seed * 1000003 + step)
        Kn = (torch.randn(S * L, H, 1, 128, generator=g, device="cuda") * 2).to(torch.bfloat16)
        Vn = torch.randn(S * L, H, 1, 128, generator=g, device="cuda").to(torch.bfloat16)
        store.append(Kn, Vn, pos)
        K_app[step].copy_(Kn[:, :, 0])
        V_app[step].copy_(Vn[:, :, 0])
        if step in checks:
            n = pos + 1
            Ko = torch.empty(S, H, n, 128, dtype=torch.bfloat16, device="cuda")
            Vo = torch.empty_like(Ko)
            store.decode_layer(step % L, n, Ko, Vo)
            decoded[step] = {s: (u16(Ko[s]), u16(Vo[s])) for s in check_seqs}
            del Ko, Vo
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    kc = store.k.codes.view(S, L, H, cap, -1)
    km = store.k.meta.view(S, L, H, cap)
    vc = store.v.codes.view(S, L, H, cap, -1)
    vm = store.v.meta.view(S, L, H, cap)
    base = {"theta": wl.theta, "bits_k": wl.bits_k, "bits_v": wl.bits_v, "window": 0, "pct": 0}

    def jobs():
        # every appended token of every unit: slots T0 .. T0+steps-1 at those positions
        Ka = u16(K_app).reshape(steps, S, L, H, 128)
        Va = u16(V_app).reshape(steps, S, L, H, 128)
        for s in range(S):
            kcs, kms = u32(kc[s, :, :, T0:]), u32(km[s, :, :, T0:])
            vcs, vms = u32(vc[s, :, :, T0:]), u32(vm[s, :, :, T0:])
            for l in range(L):
                yield dict(base, K=np.ascontiguousarray(Ka[:, s, l].transpose(1, 0, 2)),
                           V=np.ascontiguousarray(Va[:, s, l].transpose(1, 0, 2)), pos_base=T0,
                           gk_codes=kcs[l], gk_meta=kms[l], gv_codes=vcs[l], gv_meta=vms[l])
        # the initial caches of the checked sequences, all layers
        for s in check_seqs:
            Ks, Vs = inputs[s]
            for l in range(L):
                yield dict(base, K=u16(Ks[l]), V=u16(Vs[l]), gk_codes=u32(kc[s, l, :, :T0]),
                           gk_meta=u32(km[s, l, :, :T0]), gv_codes=u32(vc[s, l, :, :T0]),
                           gv_meta=u32(vm[s, l, :, :T0]))
        # full reconstructions at the checked steps (encode of all slots compared too)
        for step, per_seq in decoded.items():
            l, n = step % L, T0 + step + 1
            for s in check_seqs:
                Ks, Vs = inputs[s]
                Kin = np.concatenate([u16(Ks[l]), Ka[:step + 1, s, l].transpose(1, 0, 2)], axis=1)
                Vin = np.concatenate([u16(Vs[l]), Va[:step + 1, s, l].transpose(1, 0, 2)], axis=1)
                yield dict(base, K=Kin, V=Vin, gk_codes=u32(kc[s, l, :, :n]),
                           gk_meta=u32(km[s, l, :, :n]), gv_codes=u32(vc[s, l, :, :n]),
                           gv_meta=u32(vm[s, l, :, :n]), gK=per_seq[s][0], gV=per_seq[s][1])

    assert_parity(wl.name, parity.run_jobs(pool, jobs()))


def run_exact(nq, wl, pool):
    """The exact (24/16-bit) layout over the whole cache in one call per stage
    (scores, selection, nq_encode_exact, nq_decode_exact), every layer checked
    against the oracle's box-constrained encoder folded into that layout."""
    from oracle import parity

    K, V = gen_cache(wl)
    L, H, T = wl.layers, wl.heads, wl.tokens
    evict = wl.evict_pct > 0 and T > 1 + wl.window
    kept, scores, n = None, None, T
    if evict:
        scores = nq.nq_score(K, wl.window)
        kept = nq.nq_select(scores, wl.window, wl.evict_pct)
        n = kept.shape[1]
    rope = nq.rope_tables(wl.theta, T)
    ks = nq.ExactStore.empty(L, H, n, wl.bits_k)
    vs = nq.ExactStore.empty(L, H, n, wl.bits_v)
    nq.nq_encode_exact(K, V, ks, vs, n, rope, T, kept=kept)
    Kd = torch.empty(L, H, n, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    nq.nq_decode_exact(ks, vs, n, Kd, Vd, rope, T, positions=kept)
    torch.cuda.synchronize()
    assert nq.device_error() == 0

    def jobs():
        for l in range(L):
            yield {"K": u16(K[l]), "V": u16(V[l]), "theta": wl.theta, "bits_k": wl.bits_k,
                   "bits_v": wl.bits_v, "window": wl.window, "pct": wl.evict_pct if evict else 0,
                   "exact": True,
                   "gpu_scores": scores[l].cpu().numpy() if evict else None,
                   "gpu_kept": kept[l].cpu().numpy() if evict else None,
                   "gk_codes": u32(ks.codes[l]),
                   "gk_meta": ks.sigma[l].cpu().numpy().view(np.uint16),
                   "gv_codes": u32(vs.codes[l]),
                   "gv_meta": vs.sigma[l].cpu().numpy().view(np.uint16),
                   "gK": u16(Kd[l]), "gV": u16(Vd[l])}

    return parity.run_jobs(pool, jobs())


def test_mistral7b_32k_exact_layout_full(nq, pool):
    wl = synth.WORKLOADS["mistral7b_32k"]
    assert_parity(wl.name + ":exact", run_exact(nq, wl, pool))


def test_llama3_8b_128k_exact_layout_full(nq, pool):
    wl = synth.WORKLOADS["llama3_8b_128k"]
    assert_parity(wl.name + ":exact", run_exact(nq, wl, pool))
