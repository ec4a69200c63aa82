#!/usr/bin/env python
"""Benchmark of the KV-cache eviction + E8 lattice codec hot path on B200.

One step = one pass of the whole path over one synthetic KV cache held in
HBM: key-key scores -> token selection -> E8 encode (K3V2) -> decode back to
bf16, all layers batched into one call per stage.  Default workload: the
Mistral-7B-shaped cache (32 layers x 8 KV heads x 32768 tokens x 128, bf16,
theta 1e6, 60% eviction with BOS + 64-token window), inputs 4.3 GB > L2.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU runs are replicas (weak scaling):
every rank compresses its own cache; there is no data-path collective.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from e8_lattice_vector_nq_b200 import synth  # noqa: E402

METRIC = "KV encode+decode GB/s (bf16 in)"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mistral7b_32k")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--e2e-chunk", type=int, default=1, help="layers per pipelined chunk (e2e)")
    ap.add_argument("--cpu-layers", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-attend", action="store_true", help="skip the decode-attention timing")
    ap.add_argument("--no-entropy", action="store_true",
                    help="skip the delta + entropy stage timing")
    ap.add_argument("--layerwise", action="store_true",
                    help="also time score -> select -> encode layer by layer (keys stay in L2 "
                         "between score and encode) against the all-layer calls")
    ap.add_argument("--layers", type=int, default=0, help="override layer count (small runs)")
    ap.add_argument("--tokens", type=int, default=0, help="override token count (small runs)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# The translation unit the encode kernel is compiled from (its source and every
# header it includes, the public header among them).
ENCODE_SOURCES = ("e8_lattice_vector_nq_b200/csrc/nq_codec.cu",
                  "e8_lattice_vector_nq_b200/csrc/nq_codec_math.cuh",
                  "e8_lattice_vector_nq_b200/csrc/nq_device.cuh",
                  "e8_lattice_vector_nq_b200/csrc/nq_internal.h",
                  "include/nq.h")


def kernel_source_hash() -> str:
    """Hash of the encode kernel's sources with comments and whitespace
    removed, so that only a change of code (not of its documentation) retires
    a recorded traffic figure."""
    import re

    h = hashlib.sha256()
    for f in ENCODE_SOURCES:
        with open(os.path.join(ROOT, f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:12]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from profiles/traffic.txt, if taken on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_source_hash()
    with open(p) as f:
        for line in f:
            parts = line.split("#", 1)[0].split()
            if len(parts) == 4 and parts[0] == kernel and parts[1] == workload and parts[3] == cur:
                return float(parts[2])
    return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed
    region: NVML polled every ~2 ms on a background thread (a timed region of
    a few milliseconds still gets samples), else nvidia-smi every 200 ms.  The
    GPU is found by its UUID, so CUDA_VISIBLE_DEVICES does not matter."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.samples = []  # (sm_mhz, reasons bitmask)
        self.max_mhz = None
        self.source = None
        self.proc = None
        self.path = None
        self.thread = None

    def _uuid(self):
        try:
            u = str(torch.cuda.get_device_properties(self.device_index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return None

    def __enter__(self):
        uuid = self._uuid()
        try:
            import threading

            import pynvml

            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid
                 else pynvml.nvmlDeviceGetHandleByIndex(self.device_index))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self._stop = threading.Event()
            # one sample now, so that even a sub-millisecond region has one
            self.samples.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                 int(reasons_fn(h))))

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                             int(reasons_fn(h))))
                    except Exception:
                        pass
                    time.sleep(0.002)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            self.source = "nvml"
            return self
        except Exception:
            self.thread = None
        try:
            import tempfile

            self.path = tempfile.mktemp(suffix=".csv")
            q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap")
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid or str(self.device_index), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()
            self._read_smi()

    def _read_smi(self):
        if not self.path or not os.path.exists(self.path):
            return
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 7:
                    continue
                try:
                    sm, mx = float(p[0]), float(p[1])
                except ValueError:
                    continue
                self.max_mhz = max(self.max_mhz or 0.0, mx)
                bits = 0
                for (name, bit), v in zip(self.REASONS, p[3:7]):
                    if v.lower().startswith("active"):
                        bits |= bit
                self.samples.append((sm, bits))
        os.unlink(self.path)

    def summary(self):
        if not self.samples:
            return None
        bits = 0
        for _, b in self.samples:
            bits |= b
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz,
                "reasons": [name for name, bit in self.REASONS if bits & bit],
                "samples": len(self.samples), "source": self.source}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                             timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank's device-timed duration, max-reduced."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def build_workload(args):
    wl = synth.WORKLOADS[args.workload]
    kw = {}
    if args.layers:
        kw["layers"] = args.layers
    if args.tokens:
        kw["tokens"] = args.tokens
    if kw:
        from dataclasses import replace

        wl = replace(wl, **kw)
    return wl


def gen_cache(wl, device, layers=None):
    L = wl.layers if layers is None else layers
    K = torch.empty(L, wl.heads, wl.tokens, 128, dtype=torch.bfloat16, device=device)
    V = torch.empty_like(K)
    for l in range(L):
        k, v = synth.gen_layer(wl, l, device)
        K[l].copy_(k)
        V[l].copy_(v)
        del k, v
    return K, V


def algorithmic_bytes(wl, n_kept, units):
    H, T = wl.heads, wl.tokens
    bk = 4 * 4 * wl.bits_k + 4
    bv = 4 * 4 * wl.bits_v + 4
    evict = wl.evict_pct > 0 and T > 1 + wl.window
    out = {
        "encode": units * (n_kept * H * (256 + 256 + bk + bv) + (n_kept * 4 if evict else 0)),
        "decode": units * (n_kept * H * (bk + bv + 256 + 256) + (n_kept * 4 if evict else 0)),
    }
    if evict:
        out["score"] = units * (T * H * 256 + T * 8)
        out["select"] = units * (T * 8 + n_kept * 4)
    return out


# --------------------------------------------------------------- oracle arm
def oracle_pass(oq, Kl, Vl, wl):
    """One layer through the CPU oracle: score, select, encode, decode."""
    T = Kl.shape[1]
    evict = wl.evict_pct > 0 and T > 1 + wl.window
    kept = None
    n = T
    if evict:
        s = oq.score_unit(Kl, wl.window)
        kept = oq.select(s, wl.window, wl.evict_pct)
        n = kept.size
    r = oq.encode_unit(Kl, Vl, n, kept=kept, theta=wl.theta, bits_k=wl.bits_k, bits_v=wl.bits_v)
    oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"], positions=kept,
                   theta=wl.theta, bits_k=wl.bits_k, bits_v=wl.bits_v)


def host_layer(wl, layer, device):
    k, v = synth.gen_layer(wl, layer, device)
    u16 = lambda t: t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return u16(k), u16(v)


def cpu_baseline(wl, layers, device, hl=None):
    import oracle as oq

    oq.build()
    t = 0.0
    nbytes = 0
    for l in range(layers):
        Kl, Vl = hl if hl is not None else host_layer(wl, l, device)
        t0 = time.perf_counter()
        oracle_pass(oq, Kl, Vl, wl)
        t += time.perf_counter() - t0
        nbytes += Kl.nbytes + Vl.nbytes
    return {"value": nbytes / t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{layers} of {wl.layers} layers ({wl.heads} heads x {wl.tokens} tokens), "
                      f"score+select+encode+decode, single-threaded C oracle"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    wl = build_workload(args)
    device = "cuda" if torch.cuda.is_available() else "cpu"
    import oracle as oq

    oq.build()
    Kl, Vl = host_layer(wl, 0, device)
    per = Kl.nbytes + Vl.nbytes
    for _ in range(args.warmup):
        oracle_pass(oq, Kl, Vl, wl)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(oq, Kl, Vl, wl)
    dt = time.perf_counter() - t0
    val = per * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.layers, "heads": wl.heads, "tokens": wl.tokens,
                   "bits": f"K{wl.bits_k}V{wl.bits_v}", "evict_pct": wl.evict_pct,
                   "window": wl.window, "theta": wl.theta,
                   "step": "one layer of the cache per step (bounded sample)"},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"1 of {wl.layers} layers per step"},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    from e8_lattice_vector_nq_b200 import nq

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    wl = build_workload(args)
    units = wl.layers
    K, V = gen_cache(wl, device)
    codec = nq.Codec(units, wl.heads, wl.tokens, wl.theta, wl.bits_k, wl.bits_v, window=wl.window,
                     evict_pct=wl.evict_pct, device=device)
    n = codec.n
    Kd = torch.empty(units, wl.heads, n, 128, dtype=torch.bfloat16, device=device)
    Vd = torch.empty_like(Kd)
    stream = torch.cuda.current_stream(device)
    stages = ["score", "select", "encode", "decode"] if codec.evict else ["encode", "decode"]

    def step(ev=None):
        if codec.evict:
            if ev: ev[0].record(stream)
            nq.nq_score(K, codec.W, codec.scores, codec.ws)
            if ev: ev[1].record(stream)
            nq.nq_select(codec.scores, codec.W, codec.pct, codec.kept)
            if ev: ev[2].record(stream)
        elif ev:
            ev[2].record(stream)
        nq.nq_encode(K, V, codec.k_store, codec.v_store, n, codec.rope, codec.max_pos, kept=codec.kept)
        if ev: ev[3].record(stream)
        nq.nq_decode(codec.k_store, codec.v_store, n, Kd, Vd, codec.rope, codec.max_pos,
                     positions=codec.kept)
        if ev: ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    def timed():
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(device.index if device.index is not None else local) as clk:
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            start.record(stream)
            for i in range(args.steps):
                step(evs[i])
            end.record(stream)
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
        per = {}
        if codec.evict:
            per["score"] = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
            per["select"] = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
        per["encode"] = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
        per["decode"] = sum(e[3].elapsed_time(e[4]) for e in evs) / args.steps
        return start.elapsed_time(end), per, clk.summary()

    ms, per_stage, clocks = timed()
    # a slowdown other than the power cap during the timed region: measure once more
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    redo = int(bool(clocks and bad & set(clocks["reasons"])))
    if world > 1:
        t = torch.tensor([redo], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        redo = int(t.item())
    if redo:
        ms, per_stage, clocks = timed()
        if clocks is not None:
            clocks["remeasured"] = True
    ms = max_over_ranks(ms, world, device)
    assert nq.device_error() == 0, "a kernel reported an in-kernel failure"

    in_bytes = K.numel() * 2 + V.numel() * 2
    ms_step = ms / args.steps
    value = world * in_bytes / (ms_step * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(wl, n, units)
    dom = max(per_stage, key=per_stage.get)
    achieved = alg[dom] / (per_stage[dom] * 1e-3) / 1e9
    kernel_name = {"score": "score_kernel", "select": "select_kernel", "encode": "encode_kernel",
                   "decode": "decode_kernel"}[dom]
    # the recorded figure belongs to the named workload at its full size only
    full_size = wl == synth.WORKLOADS[args.workload]
    traffic = recorded_traffic(kernel_name, wl.name) if full_size else None

    enc_ms = sum(per_stage[s] for s in stages if s != "decode")
    out_bytes = Kd.numel() * 2 + Vd.numel() * 2
    packed_bits = codec.packed_bytes * 8
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.layers, "heads": wl.heads, "tokens": wl.tokens,
                   "head_dim": 128, "bits": f"K{wl.bits_k}V{wl.bits_v}",
                   "evict_pct": wl.evict_pct, "window": wl.window, "theta": wl.theta,
                   "kept_per_layer": n, "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"replicas x{world}"},
        "stages_ms": {k: round(v, 4) for k, v in per_stage.items()},
        "encode_gbs": in_bytes / (enc_ms * 1e-3) / 1e9,
        "decode_gbs": out_bytes / (per_stage["decode"] * 1e-3) / 1e9,
        "tokens_layers_per_s": world * wl.tokens * wl.layers / (ms_step * 1e-3),
        "bits_per_elem": packed_bits / (K.numel() + V.numel()),
        "hbm_frac_of_step": (sum(alg.values()) / (ms_step * 1e-3) / 1e9) / peak,
        "roofline": {"kernel": kernel_name, "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes": alg[dom]},
        "gpu_launches": args.steps * ((3 if codec.evict else 0) + 4),
    }
    if clocks:
        line["clocks"] = clocks

    if not args.no_attend:
        line["decode_attention"] = attend_timing(args, codec, Kd, Vd, stream, world)
    line["reconstruction"] = reconstruction_quality(K, V, Kd, Vd, codec)
    if args.layerwise:
        line["layerwise_encode"] = layerwise_timing(codec, K, V, stream, world)
    if not args.no_entropy:
        line["entropy_stage"] = entropy_timing(args, codec, stream, world,
                                               K.numel() + V.numel())
    if not args.no_e2e:
        line["e2e"] = e2e(args, K, V, Kd, Vd, codec, stream, world, in_bytes)
    if not args.no_cpu_baseline and rank == 0:
        del Kd, Vd
        hl = (K[0].cpu().view(torch.int16).numpy().view(np.uint16),
              V[0].cpu().view(torch.int16).numpy().view(np.uint16))
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_layers, device, hl=hl)
    if rank == 0:
        print(json.dumps(line), flush=True)


def attend_timing(args, codec, Kd, Vd, stream, world, G: int = 4):
    """One decode step of attention (one query per query head, G query heads
    per KV head) over the whole packed cache: nq_attend (reconstruction inside
    the attention) against nq_decode to bf16 followed by torch's
    scaled_dot_product_attention on the bf16 cache.  CUDA events, max over ranks."""
    import torch.nn.functional as F

    from e8_lattice_vector_nq_b200 import nq

    units, heads, n = codec.units, codec.heads, codec.n
    scale = 128 ** -0.5
    g = torch.Generator(device=Kd.device)
    g.manual_seed(7)
    q = torch.randn(units, heads * G, 128, device=Kd.device, generator=g)
    qb = q.to(torch.bfloat16).view(units, heads * G, 1, 128)
    ws = torch.empty(max(nq.lib().nq_attend_workspace_bytes(units, heads, G, n), 16) // 4,
                     dtype=torch.float32, device=Kd.device)

    def fused():
        nq.nq_attend(q, codec.k_store, codec.v_store, n, G, codec.rope, codec.max_pos, scale=scale,
                     positions=codec.kept, ws=ws)

    def sdpa():
        F.scaled_dot_product_attention(qb, Kd, Vd, scale=scale, enable_gqa=True)

    def unfused():
        codec.decode(Kd, Vd)
        sdpa()

    def t(fn, reps=max(args.steps, 10)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            fn()
        e.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(s.elapsed_time(e) / reps, world, Kd.device)

    f_ms, u_ms, s_ms = t(fused), t(unfused), t(sdpa)
    packed = codec.k_store.nbytes + codec.v_store.nbytes
    return {"query_heads_per_kv_head": G, "tokens": n, "units": units, "kv_heads": heads,
            "fused_ms": f_ms, "decode_then_sdpa_ms": u_ms, "sdpa_on_bf16_ms": s_ms,
            "speedup_vs_decode_then_sdpa": u_ms / f_ms,
            "fused_packed_read_gbs": packed / (f_ms * 1e-3) / 1e9}


def reconstruction_quality(K, V, Kd, Vd, codec, layers=(0, 15, 31)):
    """Diagnostic (outside the timed region): the decoded cache against its
    input rows (the kept ones), per vector: mean cosine similarity and mean
    relative L2 error, on a few layers.  Keys are compared with RoPE applied on
    both sides (the decoder re-applies it)."""
    import torch.nn.functional as F

    sample = [l for l in layers if l < codec.units]
    res = {"layers_sampled": sample}
    for name, X, Xd in (("k", K, Kd), ("v", V, Vd)):
        cos, rel = [], []
        for l in sample:
            x = X[l] if codec.kept is None else X[l][:, codec.kept[l].long()]
            x, xd = x.float(), Xd[l].float()
            cos.append(F.cosine_similarity(x, xd, dim=-1).mean().item())
            rel.append(((x - xd).norm(dim=-1) / x.norm(dim=-1).clamp_min(1e-30)).mean().item())
        res[name] = {"cosine_mean": sum(cos) / len(cos), "rel_l2_mean": sum(rel) / len(rel)}
    return res


def layerwise_timing(codec, K, V, stream, world, reps: int = 10):
    """score -> select -> encode over all layers in one call each, against the
    same calls one layer at a time (the order in which a layer's keys are still
    in L2 when encode re-reads the kept rows).  CUDA events, max over ranks."""

    def batched():
        codec.encode(K, V, stream)

    def per_layer():
        for l in range(codec.units):
            codec.encode(K, V, stream, units=slice(l, l + 1))

    def t(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b) / reps, world, K.device)

    return {"all_layers_ms": t(batched), "layer_by_layer_ms": t(per_layer)}


def entropy_timing(args, codec, stream, world, total_elems):
    """The delta + rANS stage over the lattice indices of the whole packed
    cache (keys and values, every layer in one call each): coded size and
    encode / decode time, with and without the token difference.  Code bits
    are per kept element; the cache figure (coded codes + raw meta) is per
    element of the bf16 input cache, like bits_per_elem.  CUDA events, max
    over ranks."""
    from e8_lattice_vector_nq_b200 import nq

    res = {}
    elems = 0
    for name, st in (("k", codec.k_store), ("v", codec.v_store)):
        elems += st.meta.numel() * 128
    dev = codec.k_store.codes.device
    out = {"k": nq.PackedStore.empty(codec.units, codec.heads, codec.n, codec.k_store.bits, dev),
           "v": nq.PackedStore.empty(codec.units, codec.heads, codec.n, codec.v_store.bits, dev)}
    ws = nq.entropy_workspace(codec.units, codec.heads, codec.n, dev)
    coded = {}
    for delta in (True, False):

        def enc():
            for name, st in (("k", codec.k_store), ("v", codec.v_store)):
                coded[name] = nq.nq_entropy_encode(st, codec.n, delta=delta, ws=ws,
                                                   coded=coded.get(name))

        def dec():
            for name in ("k", "v"):
                nq.nq_entropy_decode(coded[name], out[name])

        def t(fn, reps=5):
            fn()
            torch.cuda.synchronize()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            for _ in range(reps):
                fn()
            e.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(s.elapsed_time(e) / reps, world, dev)

        enc_ms = t(enc)
        dec_ms = t(dec)
        exact = all(torch.equal(out[nm].codes, st.codes)
                    for nm, st in (("k", codec.k_store), ("v", codec.v_store)))
        coded_bytes = sum(c.coded_bytes() for c in coded.values())
        code_bytes = codec.k_store.codes.numel() * 4 + codec.v_store.codes.numel() * 4
        meta_bytes = codec.k_store.meta.numel() * 4 + codec.v_store.meta.numel() * 4
        res["delta" if delta else "plain"] = {
            "encode_ms": enc_ms, "decode_ms": dec_ms,
            "codes_bits_per_elem_raw": code_bytes * 8 / elems,
            "codes_bits_per_elem_coded": coded_bytes * 8 / elems,
            "codes_ratio": code_bytes / coded_bytes,
            "cache_bits_per_elem_with_meta": (coded_bytes + meta_bytes) * 8 / total_elems,
            "encode_gbs_codes_in": code_bytes / (enc_ms * 1e-3) / 1e9,
            "decode_gbs_codes_out": code_bytes / (dec_ms * 1e-3) / 1e9,
            "round_trip_exact": bool(exact)}
    return res


def e2e(args, K, V, Kd, Vd, codec, stream, world, in_bytes):
    """Same metric through the public API with HOST buffers: pinned H2D of the
    inputs, the four calls, D2H of the reconstructed cache, every step, as
    nq.HostRoundTrip pipelines them (chunks of layers on three streams)."""
    from e8_lattice_vector_nq_b200 import nq

    Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
    Vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    Kh.copy_(K)
    Vh.copy_(V)
    Koh = torch.empty(Kd.shape, dtype=Kd.dtype, pin_memory=True)
    Voh = torch.empty(Vd.shape, dtype=Vd.dtype, pin_memory=True)
    rt = nq.HostRoundTrip(codec, K, V, Kd, Vd, chunk_units=args.e2e_chunk)

    def step():
        rt.run(Kh, Vh, Koh, Voh)

    step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.e2e_steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / args.e2e_steps, world, K.device)
    link = link_rates(Kh, K, Kd, Koh)
    h2d = rt.h2d_bytes(Kh, Vh)
    bound = in_bytes / (h2d / (link["h2d_gbs"] * 1e9)) / 1e9  # GB/s of KV in, H2D-bound
    value = world * in_bytes / (ms * 1e-3) / 1e9
    return {"value": value, "unit": "GB/s",
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": Kd.numel() * 2 + Vd.numel() * 2,
            "ms_per_step": ms, "steps": args.e2e_steps, "chunk_layers": args.e2e_chunk,
            "values_read_in_place": rt.values_in_place, "link": link,
            "h2d_bound_gbs": world * bound, "frac_of_h2d_bound": value / (world * bound)}


def link_rates(Kh, K, Kd, Koh, reps: int = 3):
    """Pinned copy rates of this GPU's host link with the run's own buffers:
    host-to-device (Kh -> K), device-to-host (Kd -> Koh) and both at once on
    two streams with equal byte counts (aggregate).  CUDA events on the
    current stream, which joins the two copy streams before the stop event."""
    dev = K.device
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)

    def h2d():
        s1.wait_stream(cur)
        with torch.cuda.stream(s1):
            K.copy_(Kh, non_blocking=True)

    def d2h():
        s2.wait_stream(cur)
        with torch.cuda.stream(s2):
            Koh.copy_(Kd, non_blocking=True)

    m = Kd.numel()  # equal byte counts both ways for the duplex figure
    Kh_m, K_m = Kh.view(-1)[:m], K.view(-1)[:m]

    def both():
        s1.wait_stream(cur)
        with torch.cuda.stream(s1):
            K_m.copy_(Kh_m, non_blocking=True)
        d2h()

    def t(fn):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(cur)
        for _ in range(reps):
            fn()
        cur.wait_stream(s1)
        cur.wait_stream(s2)
        b.record(cur)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e-3

    nh, nd = Kh.numel() * Kh.element_size(), Kd.numel() * Kd.element_size()
    return {"h2d_gbs": nh / t(h2d) / 1e9, "d2h_gbs": nd / t(d2h) / 1e9,
            "both_ways_gbs": 2 * nd / t(both) / 1e9}


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
