"""Parity accounting between the GPU path and the oracle.

TEST INFRASTRUCTURE: used by ``tests/`` and by the CPU-baseline leg of
``bench.py`` only.  It holds none of the method's arithmetic: every value it
compares with comes from the C oracle (``oracle/nq_oracle.c``).

The parity rule: kept sets and lattice codes must match the oracle bit for bit,
except where the oracle's own value lies within ``EXCUSE_REL`` (1e-5) relative
of the boundary of the decision that differs -- the k-th score for a kept set,
the scale's fp16 rounding, a coordinate's rounding, the parity move or the
coset choice for a code (``oracle.encode_margins``).  Excused mismatches are
counted and must stay below 1e-6 of the elements; unexcused ones must be zero.
Decoded bf16 rows of vectors whose codes match must be identical.

``check_layer`` compares one unit (one layer of one sequence) and returns the
counts; it runs in worker processes started with the ``spawn`` method (safe
after CUDA was initialised in the parent), so a whole cache is checked on all
host cores.
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

EXCUSE_REL = 1e-5
MAX_EXCUSED_FRACTION = 1e-6

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def make_pool(workers: int | None = None):
    """A process pool with spawn workers (never fork after CUDA init); by
    default one per host core, at most 16 (each holds a few GB at the largest
    layer sizes)."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor

    n = max(1, min(workers or min(host_cores(), 16), host_cores()))
    pool = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"),
                               initializer=_worker_init)
    # start every worker now (each imports torch and loads the oracle), so
    # that timed work never waits for a worker to come up
    list(pool.map(_warm, range(n)))
    return pool


def _worker_init():
    if _ROOT not in sys.path:
        sys.path.insert(0, _ROOT)
    import torch  # noqa: F401  (the input generator needs it)

    import oracle

    oracle._load()


def _warm(_):
    time.sleep(0.5)  # held long enough that the pool starts a process per task
    return os.getpid()


def code_fields(words: np.ndarray, bits: int) -> np.ndarray:
    """[..., 4*bits] uint32 words -> [..., 128] codes (code c at bits [b c, b c + b))."""
    w = np.asarray(words, dtype=np.uint64)
    out = np.empty(w.shape[:-1] + (128,), np.uint32)
    mask = (1 << bits) - 1
    for c in range(128):
        p = bits * c
        lo = w[..., p >> 5] >> np.uint64(p & 31)
        if (p & 31) + bits > 32:
            lo = lo | (w[..., (p >> 5) + 1] << np.uint64(32 - (p & 31)))
        out[..., c] = (lo & np.uint64(mask)).astype(np.uint32)
    return out


def kept_set_parity(s_or: np.ndarray, kept_or: np.ndarray, kept_gpu: np.ndarray, W: int,
                    pct: int) -> dict:
    """Kept-set comparison of one unit: positions in one set only, and how
    many of them score within EXCUSE_REL of the selection threshold (the
    smallest kept middle score of the oracle)."""
    diff = np.setxor1d(kept_or, kept_gpu)
    T = s_or.size
    if diff.size == 0:
        return {"tokens": T, "kept_diff": 0, "kept_excused": 0, "kept_unexcused": 0}
    mid = kept_or[(kept_or > 0) & (kept_or < T - W)]
    thr = s_or[mid].min() if mid.size else 0.0
    near = np.abs(s_or[diff] - thr) <= EXCUSE_REL * max(abs(thr), 1e-300)
    return {"tokens": T, "kept_diff": int(diff.size), "kept_excused": int(near.sum()),
            "kept_unexcused": int((~near).sum())}


def _codes_parity(oq, x_rows, gw, gm, ow, om, bits, rope, c, s, exact=False):
    """One store (keys or values): compare [N][4b] words and [N] meta words
    (exact layout: [N] fp16 scales, and no mismatch is excused: the margins
    describe the regular step's decisions, not the box step's)."""
    bad = np.nonzero(np.any(gw != ow, axis=1) | (gm != om))[0]
    res = {"vectors": int(gm.size), "mismatch_vectors": int(bad.size), "mismatch_codes": 0,
           "excused_codes": 0, "unexcused_codes": 0}
    if bad.size:
        gc, oc = code_fields(gw[bad], bits), code_fields(ow[bad], bits)
        hi = 0xFFFF if exact else 0xFFFF0000
        per_vec = (gc != oc).sum(axis=1) + 128 * ((gm[bad] & hi) != (om[bad] & hi))
        per_vec = np.maximum(per_vec, (gm[bad] != om[bad]).astype(np.int64))
        if exact:
            near = np.zeros(bad.size, bool)
        else:
            mg = oq.encode_margins(x_rows[bad], bits, rope=rope,
                                   c=None if c is None else c[bad],
                                   s=None if s is None else s[bad])
            near = mg <= EXCUSE_REL
        res["mismatch_codes"] = int(per_vec.sum())
        res["excused_codes"] = int(per_vec[near].sum())
        res["unexcused_codes"] = int(per_vec[~near].sum())
    return res, bad


def check_layer(job: dict) -> dict:
    """Oracle vs GPU for one unit.  ``job`` holds numpy arrays:

    K, V       [H][T_in][128] uint16 bf16 inputs of the unit
    theta, bits_k, bits_v, window, pct (pct 0: no eviction)
    pos_base   RoPE position of input token 0 (appended tokens)
    gpu_scores [T] fp64 (evicting units), gpu_kept [n] int32 (or None: slots
               are tokens 0..n-1)
    gk_codes [H][n][4 bk], gk_meta [H][n], gv_codes, gv_meta  (GPU store)
    exact      True for an exact-layout store (gk_meta / gv_meta then hold
               the fp16 scales; the oracle side is its box-constrained
               encoder folded into that layout)
    gK, gV     [H][n][128] uint16 GPU decode output (optional)
    Returns counts (see module doc) and the oracle's seconds."""
    import oracle as oq

    t0 = time.perf_counter()
    K, V = job["K"], job["V"]
    H, T_in = V.shape[0], V.shape[1]
    bk, bv = job["bits_k"], job["bits_v"]
    theta, pos_base = job["theta"], job.get("pos_base", 0)
    out = {"units": 1}
    kept = job.get("gpu_kept")
    if job.get("pct", 0) > 0 and T_in > 1 + job["window"]:
        s_or = oq.score_unit(K, job["window"])
        sg = job["gpu_scores"]
        out["score_max_rel"] = float(np.max(np.abs(sg - s_or)) / max(np.max(np.abs(s_or)), 1e-300))
        k_or = oq.select(s_or, job["window"], job["pct"])
        out.update(kept_set_parity(s_or, k_or, kept, job["window"], job["pct"]))
        if out["kept_diff"] == 0:
            kept = k_or  # identical lists: encode on the oracle's own
    n = job["gk_meta"].shape[1]
    src = np.arange(n, dtype=np.int64) if kept is None else np.asarray(kept, np.int64)
    # vectors in (head, slot) order, matching the [H][n] stores
    Kx = K[:, src].reshape(-1, 128)
    Vx = V[:, src].reshape(-1, 128)
    c, s = oq.rope_cs(theta, pos_base + src)
    c, s = np.tile(c, (H, 1)), np.tile(s, (H, 1))
    exact = bool(job.get("exact", False))
    if exact:  # box-constrained step, folded into the exact layout
        kw, km = oq.fold_exact(*oq.encode_vectors_box(Kx, bk, rope=True, c=c, s=s), bk)
        vw, vm = oq.fold_exact(*oq.encode_vectors_box(Vx, bv), bv)
    else:
        kw, km, _ = oq.encode_vectors(Kx, bk, rope=True, c=c, s=s)
        vw, vm, _ = oq.encode_vectors(Vx, bv)
    t_oracle = time.perf_counter() - t0
    rk, bad_k = _codes_parity(oq, Kx, job["gk_codes"].reshape(-1, 4 * bk),
                              job["gk_meta"].reshape(-1), kw, km, bk, True, c, s, exact)
    rv, bad_v = _codes_parity(oq, Vx, job["gv_codes"].reshape(-1, 4 * bv),
                              job["gv_meta"].reshape(-1), vw, vm, bv, False, None, None, exact)
    out["vectors"] = rk["vectors"] + rv["vectors"]
    out["elements"] = 128 * out["vectors"]
    for key in ("mismatch_vectors", "mismatch_codes", "excused_codes", "unexcused_codes"):
        out[key] = rk[key] + rv[key]
    if job.get("gK") is not None:
        t1 = time.perf_counter()
        if exact:
            kw, km = oq.unfold_exact(kw, km, bk)
            vw, vm = oq.unfold_exact(vw, vm, bv)
        Ko = oq.decode_vectors(kw, km, bk, rope=True, c=c, s=s)
        Vo = oq.decode_vectors(vw, vm, bv)
        t_oracle += time.perf_counter() - t1
        gK, gV = job["gK"].reshape(-1, 128), job["gV"].reshape(-1, 128)
        okk = np.ones(Ko.shape[0], bool)
        okk[bad_k] = False
        okv = np.ones(Vo.shape[0], bool)
        okv[bad_v] = False
        out["bf16_diff"] = int((gK[okk] != Ko[okk]).sum() + (gV[okv] != Vo[okv]).sum())
        rel = 0.0
        for g, o, ok in ((gK, Ko, okk), (gV, Vo, okv)):
            gf = (g[ok].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            of = (o[ok].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            num = np.linalg.norm(gf - of, axis=1)
            den = np.maximum(np.linalg.norm(of, axis=1), 1e-300)
            if num.size:
                rel = max(rel, float(np.max(num / den)))
        out["recon_max_rel"] = rel
    out["oracle_s"] = t_oracle
    return out


def run_jobs(pool, jobs, fn=None, inflight: int | None = None) -> list:
    """Run fn (check_layer) over an iterable of jobs on the pool, with at most
    `inflight` jobs held at once (the jobs are built lazily, so a large cache
    is never copied to host memory whole)."""
    from concurrent.futures import FIRST_COMPLETED, wait

    fn = fn or check_layer
    limit = inflight or 2 * pool._max_workers
    pending, results = set(), []
    for job in jobs:
        pending.add(pool.submit(fn, job))
        if len(pending) >= limit:
            done, pending = wait(pending, return_when=FIRST_COMPLETED)
            results.extend(f.result() for f in done)
    results.extend(f.result() for f in pending)
    return results


def merge(results) -> dict:
    """Sum the counts of many units (max for the relative errors)."""
    tot: dict = {}
    for r in results:
        for k, v in r.items():
            if k in ("score_max_rel", "recon_max_rel"):
                tot[k] = max(tot.get(k, 0.0), v)
            else:
                tot[k] = tot.get(k, 0) + v
    return tot


def verdict(tot: dict) -> list[str]:
    """The parity rule applied to merged counts: a list of failures (empty if
    the rule holds)."""
    bad = []
    if tot.get("unexcused_codes", 0):
        bad.append(f"{tot['unexcused_codes']} code mismatches away from any decision boundary")
    if tot.get("kept_unexcused", 0):
        bad.append(f"{tot['kept_unexcused']} kept-set differences away from the threshold")
    el = tot.get("elements", 0)
    if el and tot.get("excused_codes", 0) >= MAX_EXCUSED_FRACTION * el:
        bad.append(f"{tot['excused_codes']} excused code mismatches >= 1e-6 of {el} elements")
    tk = tot.get("tokens", 0)
    if tk and tot.get("kept_excused", 0) >= max(MAX_EXCUSED_FRACTION * tk, 1):
        bad.append(f"{tot['kept_excused']} excused kept-set differences among {tk} tokens")
    if tot.get("bf16_diff", 0):
        bad.append(f"{tot['bf16_diff']} decoded bf16 elements differ")
    if tot.get("recon_max_rel", 0.0) > 1e-3:
        bad.append(f"reconstruction error {tot['recon_max_rel']:.2e} > 1e-3 per vector")
    if tot.get("score_max_rel", 0.0) > 1e-12:
        bad.append(f"score error {tot['score_max_rel']:.2e} > 1e-12 of the largest score")
    return bad
