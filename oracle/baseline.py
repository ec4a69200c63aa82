"""The oracle timed as the CPU baseline.

TEST INFRASTRUCTURE: only the CPU-baseline leg and the reference arm of
``bench.py`` call this module.  It times the C oracle as it stands (one
single-threaded pass per call; many calls in parallel worker processes give
the all-cores figure) on seeded synthetic inputs drawn on the CPU by the
shared input generator.  It adds none of the method's arithmetic.
"""
from __future__ import annotations

import time
from dataclasses import asdict, replace

import numpy as np


def _u16(t):
    import torch

    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_pass(oq, K, V, theta, bits_k, bits_v, window, pct, pos_base=0):
    """One unit through the oracle: score, select (when evicting), encode,
    decode.  K, V [H][T][128] bf16 bits."""
    T = K.shape[1]
    evict = pct > 0 and T > 1 + window
    kept = None
    n = T
    if evict:
        s = oq.score_unit(K, window)
        kept = oq.select(s, window, pct)
        n = kept.size
    r = oq.encode_unit(K, V, n, kept=kept, pos_base=pos_base, theta=theta, bits_k=bits_k,
                       bits_v=bits_v)
    oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], positions=kept,
                   pos_base=pos_base, theta=theta, bits_k=bits_k, bits_v=bits_v)


def workload_fields(wl) -> dict:
    return asdict(wl)


def timed_unit(job: dict) -> dict:
    """Draw one layer (or its first ``tokens`` tokens) of a workload on the CPU
    and time one oracle pass over it.  Returns the bf16 bytes of the sample,
    the wall-clock interval of the oracle pass and its seconds."""
    import oracle as oq
    from e8_lattice_vector_nq_b200 import synth

    oq.build()
    wl = synth.Workload(**job["workload"])
    if job.get("tokens"):
        wl = replace(wl, tokens=int(job["tokens"]))
    K, V = synth.gen_layer(wl, job.get("layer", 0), "cpu")
    K, V = _u16(K), _u16(V)
    t0 = time.time()
    c0 = time.perf_counter()
    oracle_pass(oq, K, V, wl.theta, wl.bits_k, wl.bits_v, wl.window, wl.evict_pct)
    sec = time.perf_counter() - c0
    return {"bytes": K.nbytes + V.nbytes, "t0": t0, "t1": time.time(), "seconds": sec}


def timed_append_step(job: dict) -> dict:
    """A bounded sample of one decode-append step through the oracle: the
    encode of one appended token for ``units`` (sequence, layer) units at
    position T0, and the full decode of one unit's T0 tokens.  Bytes are the
    bf16 appended in plus the bf16 decoded out; the unit's initial encode is
    set-up and not timed."""
    import torch

    import oracle as oq
    from e8_lattice_vector_nq_b200 import synth

    oq.build()
    wl = synth.Workload(**job["workload"])
    H, T0, units = wl.heads, wl.tokens, int(job["units"])
    g = torch.Generator()
    g.manual_seed(int(job.get("seed", 0)))
    Ka = _u16((torch.randn(units, H, 1, 128, generator=g) * 2).to(torch.bfloat16))
    Va = _u16(torch.randn(units, H, 1, 128, generator=g).to(torch.bfloat16))
    K0, V0 = synth.gen_layer(wl, 0, "cpu")
    K0, V0 = _u16(K0), _u16(V0)
    t0 = time.time()
    c0 = time.perf_counter()
    for u in range(units):
        oq.encode_unit(Ka[u], Va[u], 1, pos_base=T0, theta=wl.theta, bits_k=wl.bits_k,
                       bits_v=wl.bits_v)
    c1 = time.perf_counter()
    r = oq.encode_unit(K0, V0, T0, theta=wl.theta, bits_k=wl.bits_k, bits_v=wl.bits_v)
    c2 = time.perf_counter()
    oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], theta=wl.theta,
                   bits_k=wl.bits_k, bits_v=wl.bits_v)
    c3 = time.perf_counter()
    return {"bytes": Ka.nbytes + Va.nbytes + K0.nbytes + V0.nbytes, "t0": t0, "t1": time.time(),
            "seconds": (c1 - c0) + (c3 - c2)}
