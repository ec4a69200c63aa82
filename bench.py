#!/usr/bin/env python
"""Benchmark of the KV-cache eviction + E8 lattice codec hot path on B200.

One step = one pass of the whole path over one synthetic KV cache held in
HBM: key-key scores -> token selection (when the workload evicts) -> E8
encode -> decode back to bf16, all layers batched into one call per stage.
Default (headline) workload: the Llama-3-8B-shaped long-context cache (32
layers x 8 KV heads x 131072 tokens x 128, bf16, theta 5e5, K3V2, no
eviction: 17.2 GB in, larger than L2), the largest single-GPU workload.  The
other four workloads (tiny, Mistral-7B-shaped with 60 % eviction, Qwen2.5-7B-
shaped with protected layers, decode-append) are timed after it and reported
under "configs", each with the oracle timed beside it.

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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b_128k")
    ap.add_argument("--configs", default="all",
                    help="other workloads timed after the headline and reported under 'configs' "
                         "(comma list, 'all' or 'none')")
    ap.add_argument("--config-steps", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--e2e-chunk", type=int, default=1, help="layers per pipelined chunk (e2e)")
    ap.add_argument("--cpu-tokens", type=int, default=65536,
                    help="tokens per layer in the timed oracle sample (at most the layer)")
    ap.add_argument("--cpu-workers", type=int, default=0,
                    help="worker processes of the all-cores oracle figure (0: every core)")
    ap.add_argument("--parity-layers", default="0,-1",
                    help="layers of the headline cache checked against the oracle in the "
                         "CPU-baseline leg (comma list, negative from the end)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-attend", action="store_true", help="skip the decode-attention timing")
    ap.add_argument("--no-exact", action="store_true",
                    help="skip the exact (24/16-bit) layout timing")
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
                  "e8_lattice_vector_nq_b200/csrc/nq_tc_slots.cuh",
                  "e8_lattice_vector_nq_b200/csrc/nq_tcgen05.cuh",
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


def build_workload(args, name=None):
    wl = synth.WORKLOADS[name or args.workload]
    kw = {}
    if args.layers and name is None:
        kw["layers"] = args.layers
    if args.tokens and name is None:
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


def vector_bytes(bits):
    return 4 * 4 * bits + 4  # packed codes + the meta word


def algorithmic_bytes(wl, n_kept, units):
    """DRAM bytes each stage must move per call over `units` layers: the
    kernels' algorithmic bytes (the bf16 rows read or written, the packed
    vectors, the kept lists and scores)."""
    H, T = wl.heads, wl.tokens
    bk, bv = vector_bytes(wl.bits_k), vector_bytes(wl.bits_v)
    evict = wl.evict_pct > 0 and T > 1 + wl.window
    out = {
        "encode": units * (n_kept * H * (256 + 256 + bk + bv) + (n_kept * 4 if evict else 0)),
        "decode": units * (n_kept * H * (bk + bv + 256 + 256) + (n_kept * 4 if evict else 0)),
    }
    if evict:
        out["score"] = units * (T * H * 256 + T * 8)
        out["select"] = units * (T * 8 + n_kept * 4)
    return out


KERNEL_OF = {"score": "score_kernel", "select": "select_kernel", "encode": "encode_kernel",
             "decode": "decode_kernel"}


def kernel_of(stage: str, heads: int, units: int = 0, n: int = 0) -> str:
    """The kernel a stage launches.  Decode (the default engine) runs on the
    tensor cores when the head group hg (largest divisor of heads up to 8) is
    at least 3 and the call has two 128-vector tiles per warpgroup of the SMs
    (tiles = units * groups * ceil(slot tiles / (8 // hg)), 4 warpgroups per
    SM, 3 for keys with two RoPE tables); the key launch decides the name."""
    if stage != "decode":
        return KERNEL_OF[stage]
    hg = max(g for g in range(1, 9) if heads % g == 0)
    m = 8 // hg
    if m > 2:
        return KERNEL_OF[stage]
    slot_tiles = (n + 15) // 16
    tiles = units * (heads // hg) * ((slot_tiles + m - 1) // m)
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    nwg = 3 if m == 2 else 4
    return "decode_tc_kernel" if tiles >= 2 * nwg * sms else KERNEL_OF[stage]


def timed_region(fn, steps, stream, device, world, n_events):
    """Run fn(events_of_step) for `steps` steps between a barrier and a
    synchronize on both sides, clocks sampled meanwhile; returns total ms,
    the per-step event lists and the clock summary."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(steps):
            fn(evs[i])
        end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    return start.elapsed_time(end), evs, clk.summary()


def with_remeasure(measure, world, device):
    """measure() once more if its clock record shows a hardware or thermal
    slowdown (every rank takes the same decision)."""
    res = measure()
    clocks = res[-1]
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    redo = int(bool(clocks and bad & set(clocks["reasons"])))
    if world > 1:
        t = torch.tensor([redo], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        redo = int(t.item())
    if redo:
        res = measure()
        if res[-1] is not None:
            res[-1]["remeasured"] = True
    return res


def time_cache(nq, wl, device, steps, warmup, world):
    """The whole cache through score -> select -> encode -> decode, every
    layer in one call per stage, timed with CUDA events on the launching
    stream.  Protected layers (kept in bf16) are not part of the step."""
    q_layers = wl.quantised_layers
    units = len(q_layers)
    K, V = gen_cache(wl, device)
    Kq, Vq = (K, V) if units == wl.layers else (K[q_layers[0]:q_layers[-1] + 1],
                                                   V[q_layers[0]:q_layers[-1] + 1])
    codec = nq.Codec(units, wl.heads, wl.tokens, wl.theta, wl.bits_k, wl.bits_v,
                     window=wl.window, evict_pct=wl.evict_pct, device=device)
    n = codec.n
    Kd = torch.empty(units, wl.heads, n, 128, dtype=torch.bfloat16, device=device)
    Vd = torch.empty_like(Kd)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        if codec.evict:
            if ev: ev[0].record(stream)
            nq.nq_score(Kq, codec.W, codec.scores, codec.ws)
            if ev: ev[1].record(stream)
            nq.nq_select(codec.scores, codec.W, codec.pct, codec.kept)
            if ev: ev[2].record(stream)
        elif ev:
            ev[2].record(stream)
        nq.nq_encode(Kq, Vq, codec.k_store, codec.v_store, n, codec.rope, codec.max_pos,
                     kept=codec.kept)
        if ev: ev[3].record(stream)
        nq.nq_decode(codec.k_store, codec.v_store, n, Kd, Vd, codec.rope, codec.max_pos,
                     positions=codec.kept)
        if ev: ev[4].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    def measure():
        ms, evs, clocks = timed_region(step, steps, stream, device, world, 5)
        per = {}
        if codec.evict:
            per["score"] = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
            per["select"] = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
        per["encode"] = sum(e[2].elapsed_time(e[3]) for e in evs) / steps
        per["decode"] = sum(e[3].elapsed_time(e[4]) for e in evs) / steps
        return ms, per, clocks

    ms, per, clocks = with_remeasure(measure, world, device)
    ms = max_over_ranks(ms, world, device)
    per = {k: max_over_ranks(v, world, device) for k, v in per.items()}
    assert nq.device_error() == 0, "a kernel reported an in-kernel failure"
    return {"K": K, "V": V, "Kq": Kq, "Vq": Vq, "Kd": Kd, "Vd": Vd, "codec": codec,
            "ms_step": ms / steps, "per_stage": per, "clocks": clocks, "stream": stream,
            "launches_per_step": (3 if codec.evict else 0) + 4}


def figures(wl, t, world, peak, peak_kind, traffic_for=None):
    """Throughput, stage bandwidths and rooflines of a timed cache."""
    codec, per, ms_step = t["codec"], t["per_stage"], t["ms_step"]
    n, units = codec.n, codec.units
    in_bytes = t["K"].numel() * 2 + t["V"].numel() * 2  # the whole bf16 cache
    q_in = t["Kq"].numel() * 2 + t["Vq"].numel() * 2
    alg = algorithmic_bytes(wl, n, units)
    roof = {}
    for stage, ms in per.items():
        ach = alg[stage] / (ms * 1e-3) / 1e9
        r = {"kernel": kernel_of(stage, wl.heads, units, n), "bound": "hbm", "achieved": ach, "peak": peak,
             "peak_kind": peak_kind, "unit": "GB/s", "frac": ach / peak,
             "frac_of_8tbs_spec": ach / 8000.0, "algorithmic_bytes": alg[stage], "ms": ms}
        if stage == "select":
            r["bound"] = "latency"  # a few MB per call: radix passes on cluster barriers
        roof[stage] = r
    enc_ms = sum(v for k, v in per.items() if k != "decode")
    out_bytes = t["Kd"].numel() * 2 + t["Vd"].numel() * 2
    bits = codec.packed_bytes * 8
    if units != wl.layers:  # protected layers stay bf16
        bits += 16 * (in_bytes - q_in) // 2
    return {
        "value": world * in_bytes / (ms_step * 1e-3) / 1e9,
        "ms_per_step": ms_step,
        "stages_ms": {k: round(v, 4) for k, v in per.items()},
        "encode_gbs": q_in / (enc_ms * 1e-3) / 1e9,
        "decode_gbs": out_bytes / (per["decode"] * 1e-3) / 1e9,
        "tokens_layers_per_s": world * wl.tokens * wl.layers / (ms_step * 1e-3),
        "bits_per_elem": bits / (in_bytes / 2),
        "hbm_frac_of_step": (sum(alg.values()) / (ms_step * 1e-3) / 1e9) / peak,
        "rooflines": roof,
    }


def time_append(nq, wl, device, world, warmup=3):
    """The decode-append regime: a store of `sequences` x `layers` units of
    `tokens` encoded tokens (set-up, not timed), then `append_steps` steps,
    each appending one bf16 token per unit (encode) and reconstructing every
    token of layer step mod layers for every sequence (decode)."""
    S, L, H, T0, steps = wl.sequences, wl.layers, wl.heads, wl.tokens, wl.append_steps
    cap = T0 + steps
    store = nq.AppendStore(S, L, H, cap, wl.theta, wl.bits_k, wl.bits_v, device=device)
    for s in range(S):
        Ks = torch.empty(L, H, T0, 128, dtype=torch.bfloat16, device=device)
        Vs = torch.empty_like(Ks)
        for l in range(L):
            k, v = synth.gen_layer(wl, l, device, seed_offset=1000 * s)
            Ks[l].copy_(k)
            Vs[l].copy_(v)
        store.fill(s, Ks, Vs)
        del Ks, Vs
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 1000003)
    Kn = (torch.randn(steps, S * L, H, 1, 128, generator=g, device=device) * 2).to(torch.bfloat16)
    Vn = torch.randn(steps, S * L, H, 1, 128, generator=g, device=device).to(torch.bfloat16)
    Ko = torch.empty(S, H, cap, 128, dtype=torch.bfloat16, device=device)
    Vo = torch.empty_like(Ko)
    stream = torch.cuda.current_stream(device)

    def step_at(i, ev=None):
        pos = T0 + i
        if ev: ev[0].record(stream)
        store.append(Kn[i], Vn[i], pos)
        if ev: ev[1].record(stream)
        store.decode_layer(i % L, pos + 1, Ko[:, :, :pos + 1], Vo[:, :, :pos + 1])
        if ev: ev[2].record(stream)

    for _ in range(warmup):  # rewritten by the timed steps
        step_at(0)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    counter = {"i": 0}

    def one(ev):
        step_at(counter["i"], ev)
        counter["i"] += 1

    def measure():
        counter["i"] = 0
        ms, evs, clocks = timed_region(one, steps, stream, device, world, 3)
        enc = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
        dec = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
        return ms, enc, dec, clocks

    ms, enc, dec, clocks = with_remeasure(measure, world, device)
    ms, enc, dec = (max_over_ranks(x, world, device) for x in (ms, enc, dec))
    assert nq.device_error() == 0, "a kernel reported an in-kernel failure"
    ms_step = ms / steps
    bk, bv = vector_bytes(wl.bits_k), vector_bytes(wl.bits_v)
    app_units = S * L * H  # vectors appended per step (keys and values each)
    in_b = app_units * 256 * 2
    # decoded per step: every token of one layer for every sequence (mean n over the steps)
    n_mean = T0 + (steps + 1) / 2
    out_b = S * H * n_mean * 256 * 2
    enc_alg = app_units * (512 + bk + bv)
    dec_alg = S * H * n_mean * (bk + bv + 512)
    peak, peak_kind = measured_peaks()
    roof = {}
    for stage, alg, sms in (("encode", enc_alg, enc), ("decode", dec_alg, dec)):
        ach = alg / (sms * 1e-3) / 1e9
        roof[stage] = {"kernel": kernel_of(stage, H, S, int(n_mean)), "bound": "hbm", "achieved": ach, "peak": peak,
                       "peak_kind": peak_kind, "unit": "GB/s", "frac": ach / peak,
                       "frac_of_8tbs_spec": ach / 8000.0, "algorithmic_bytes": alg, "ms": sms}
    roof["encode"]["bound"] = "latency"  # 16 384 vectors per append: one short launch pair
    packed = store.k.nbytes + store.v.nbytes
    return {"value": world * (in_b + out_b) / (ms_step * 1e-3) / 1e9, "ms_per_step": ms_step,
            "steps": steps, "total_ms": ms,
            "stages_ms": {"append_encode": round(enc, 4), "layer_decode": round(dec, 4)},
            "tokens_layers_per_s": world * (S * L + S * n_mean) / (ms_step * 1e-3),
            "bits_per_elem": packed * 8 / (S * L * H * cap * 128 * 2),
            "rooflines": roof, "clocks": clocks,
            "metric_note": "bf16 bytes appended (in) + decoded (out) per step"}


# --------------------------------------------------------------- oracle legs
def oracle_workers(args) -> int:
    """Worker processes of the all-cores oracle figure: every host core, at
    most 32 (each holds about a GB at the largest sample)."""
    from oracle import parity

    return args.cpu_workers or min(parity.host_cores(), 32)


def cpu_baseline(args, wl, pool, workers):
    """The oracle as it stands, timed on the host cores: single-threaded on one
    layer sample, and `workers` such samples (distinct layers) in parallel
    processes (wall clock from the first pass's start to the last one's end).
    The sample is one layer cut to at most --cpu-tokens tokens."""
    from oracle import baseline, parity

    fields = baseline.workload_fields(wl)
    tokens = min(wl.tokens, args.cpu_tokens)
    job = lambda l: {"workload": fields, "layer": l % wl.layers, "tokens": tokens}  # noqa: E731
    if wl.name == "decode_append":
        job = lambda l: {"workload": fields, "units": 64, "seed": l}  # noqa: E731
        fn = baseline.timed_append_step
    else:
        fn = baseline.timed_unit
    single = pool.submit(fn, job(0)).result()
    if workers > 1:
        res = list(pool.map(fn, [job(l) for l in range(workers)]))
        wall = max(r["t1"] for r in res) - min(r["t0"] for r in res)
        tot = sum(r["bytes"] for r in res)
    else:
        wall, tot = single["seconds"], single["bytes"]
    what = ("one append of 64 units + one unit's decode" if wl.name == "decode_append" else
            f"one layer ({wl.heads} heads x {tokens} of {wl.tokens} tokens)")
    return {"value": tot / wall / 1e9, "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": f"{workers} worker process(es), each {what} through the single-threaded "
                      f"C oracle (score/select/encode/decode), wall clock of the parallel run",
            "host_cores": parity.host_cores(),
            "single_thread": {"value": single["bytes"] / single["seconds"] / 1e9,
                              "unit": "GB/s", "cores": 1, "sample": what}}


def headline_parity(args, wl, t, pool):
    """The headline cache's GPU outputs on a few layers against the oracle
    (oracle/parity.py: excused and unexcused mismatches, decoded bf16)."""
    from oracle import parity

    codec, units = t["codec"], t["codec"].units
    layers = sorted({(int(x) % units) for x in args.parity_layers.split(",") if x.strip()})
    u16 = lambda x: x.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    u32 = lambda x: x.cpu().contiguous().numpy().view(np.uint32)  # noqa: E731
    futs = []
    for u in layers:
        job = {"K": u16(t["Kq"][u]), "V": u16(t["Vq"][u]), "theta": wl.theta,
               "bits_k": wl.bits_k, "bits_v": wl.bits_v, "window": wl.window,
               "pct": wl.evict_pct if codec.evict else 0,
               "gpu_scores": codec.scores[u].cpu().numpy() if codec.evict else None,
               "gpu_kept": codec.kept[u].cpu().numpy() if codec.evict else None,
               "gk_codes": u32(codec.k_store.codes[u]), "gk_meta": u32(codec.k_store.meta[u]),
               "gv_codes": u32(codec.v_store.codes[u]), "gv_meta": u32(codec.v_store.meta[u]),
               "gK": u16(t["Kd"][u]), "gV": u16(t["Vd"][u])}
        futs.append(pool.submit(parity.check_layer, job))
    tot = parity.merge(f.result() for f in futs)
    return {"layers_checked": layers, "elements": tot.get("elements", 0),
            "excused": tot.get("excused_codes", 0) + tot.get("kept_excused", 0),
            "unexcused": tot.get("unexcused_codes", 0) + tot.get("kept_unexcused", 0),
            "kept_set_differences": tot.get("kept_diff", 0),
            "bf16_elements_differing": tot.get("bf16_diff", 0),
            "recon_max_rel": tot.get("recon_max_rel", 0.0),
            "failures": parity.verdict(tot),
            "rule": "bit-exact codes and kept sets; a mismatch is excused only within 1e-5 "
                    "relative of a decision boundary (must stay below 1e-6 of elements)"}


def run_reference(args, world, rank):
    """The reference arm: the oracle (the CPU restatement of the method) as it
    stands, on the host cores, each step a bounded sample of the workload: one
    layer sample per worker process, all workers in parallel."""
    if rank != 0:
        return
    wl = build_workload(args)
    from oracle import baseline, parity

    workers = oracle_workers(args)
    fields = baseline.workload_fields(wl)
    tokens = min(wl.tokens, args.cpu_tokens // 8 if args.cpu_tokens >= 8 else 1)
    if wl.name == "decode_append":
        fn, job = baseline.timed_append_step, lambda l: {"workload": fields, "units": 16, "seed": l}
    else:
        fn, job = baseline.timed_unit, lambda l: {"workload": fields, "layer": l % wl.layers,
                                                  "tokens": tokens}
    pool = parity.make_pool(workers)
    try:
        for _ in range(args.warmup):
            list(pool.map(fn, [job(l) for l in range(workers)]))
        nbytes, dt = 0, 0.0
        for _ in range(args.steps):
            res = list(pool.map(fn, [job(l) for l in range(workers)]))
            nbytes += sum(r["bytes"] for r in res)
            # the step's oracle work: first pass start to last pass end
            dt += max(r["t1"] for r in res) - min(r["t0"] for r in res)
    finally:
        pool.shutdown()
    val = nbytes / dt / 1e9
    what = ("one append of 16 units + one unit's decode" if wl.name == "decode_append" else
            f"one layer ({wl.heads} heads x {tokens} tokens)")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.layers, "heads": wl.heads, "tokens": wl.tokens,
                   "bits": f"K{wl.bits_k}V{wl.bits_v}", "evict_pct": wl.evict_pct,
                   "window": wl.window, "theta": wl.theta,
                   "step": f"{workers} worker processes x {what} (bounded sample)"},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": workers, "kind": "oracle",
                         "sample": f"{workers} workers x {what} per step"},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def config_names(args):
    if args.configs == "none":
        return []
    names = [n for n in synth.WORKLOADS if n != args.workload] if args.configs == "all" else \
        [n.strip() for n in args.configs.split(",") if n.strip() and n.strip() != args.workload]
    return names


def run_ours(args, world, rank, local):
    from e8_lattice_vector_nq_b200 import nq

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    wl = build_workload(args)
    peak, peak_kind = measured_peaks()
    # oracle worker processes (spawn) for the CPU legs, rank 0 only
    pool, workers = None, 0
    if not args.no_cpu_baseline and rank == 0:
        from oracle import parity

        workers = oracle_workers(args)
        pool = parity.make_pool(workers)
    try:
        line = _run_ours(args, world, rank, device, wl, peak, peak_kind, pool, workers, nq)
    finally:
        if pool is not None:
            pool.shutdown()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _run_ours(args, world, rank, device, wl, peak, peak_kind, pool, workers, nq):
    if wl.name == "decode_append":
        f = time_append(nq, wl, device, world, args.warmup)
        line = {"metric": METRIC, "value": f["value"], "unit": "GB/s", "n_gpus": world,
                "steps": f["steps"], "warmup": args.warmup, "ms_per_step": f["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic",
                "config": {"workload": wl.name, "sequences": wl.sequences, "layers": wl.layers,
                           "heads": wl.heads, "tokens": wl.tokens, "append_steps": wl.append_steps,
                           "bits": f"K{wl.bits_k}V{wl.bits_v}", "theta": wl.theta,
                           "parallelism": f"replicas x{world}"},
                **{k: v for k, v in f.items() if k not in ("value", "ms_per_step", "steps")}}
        line["roofline"] = f["rooflines"]["decode"]
        line["gpu_launches"] = f["steps"] * 4
        if pool is not None:
            line["cpu_baseline"] = cpu_baseline(args, wl, pool, workers)
        return line

    t = time_cache(nq, wl, device, args.steps, args.warmup, world)
    f = figures(wl, t, world, peak, peak_kind)
    dom = max(t["per_stage"], key=t["per_stage"].get)
    roof = dict(f["rooflines"][dom])
    full_size = wl == synth.WORKLOADS[args.workload]
    roof["traffic"] = recorded_traffic(roof["kernel"], wl.name) if full_size else None
    for stage, r in f["rooflines"].items():
        r["traffic"] = recorded_traffic(r["kernel"], wl.name) if full_size else None
    codec = t["codec"]
    line = {
        "metric": METRIC, "value": f["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": f["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.layers, "heads": wl.heads, "tokens": wl.tokens,
                   "head_dim": 128, "bits": f"K{wl.bits_k}V{wl.bits_v}",
                   "evict_pct": wl.evict_pct, "window": wl.window, "theta": wl.theta,
                   "kept_per_layer": codec.n, "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"replicas x{world}"},
        **{k: v for k, v in f.items() if k not in ("value", "ms_per_step")},
        "roofline": roof,
        "gpu_launches": args.steps * t["launches_per_step"],
    }
    if t["clocks"]:
        line["clocks"] = t["clocks"]
    K, V, Kd, Vd, stream = t["K"], t["V"], t["Kd"], t["Vd"], t["stream"]
    if pool is not None:  # the timed step's outputs, before any other leg reuses the buffers
        line["parity"] = headline_parity(args, wl, t, pool)
    if not args.no_attend:
        line["decode_attention"] = attend_timing(args, codec, Kd, Vd, stream, world)
    line["reconstruction"] = reconstruction_quality(t["Kq"], t["Vq"], Kd, Vd, codec)
    if not args.no_exact:
        line["exact_layout"] = exact_timing(args, wl, t, world, peak, peak_kind)
    if args.layerwise:
        line["layerwise_encode"] = layerwise_timing(codec, t["Kq"], t["Vq"], stream, world)
    if not args.no_entropy:
        line["entropy_stage"] = entropy_timing(args, codec, stream, world, K.numel() + V.numel())
    if not args.no_e2e:
        in_bytes = K.numel() * 2 + V.numel() * 2
        line["e2e"] = e2e(args, t["Kq"], t["Vq"], Kd, Vd, codec, stream, world, in_bytes)
    if pool is not None:
        line["cpu_baseline"] = cpu_baseline(args, wl, pool, workers)
    del t, K, V, Kd, Vd, codec
    torch.cuda.empty_cache()

    configs = {}
    for name in config_names(args):
        cw = synth.WORKLOADS[name]
        if cw.name == "decode_append":
            cf = time_append(nq, cw, device, world, args.warmup)
        else:
            ct = time_cache(nq, cw, device, args.config_steps, args.warmup, world)
            cf = figures(cw, ct, world, peak, peak_kind)
            cf["clocks"] = ct["clocks"]
            del ct
        cf.pop("metric_note", None)
        if pool is not None:
            cf["cpu_baseline"] = cpu_baseline(args, cw, pool, 1)
        configs[name] = cf
        torch.cuda.empty_cache()
    if configs:
        line["configs"] = configs
    if not args.no_entropy:
        line["entropy_correlated"] = entropy_correlated(args, device, world)
    return line


def exact_timing(args, wl, t, world, peak, peak_kind):
    """The exact (24/16-bit) layout on the same cache: nq_encode_exact and
    nq_decode_exact over every layer in one call each (the box-constrained E8
    step, the coset bit folded into the codes, a uint16 scale per vector),
    timed like the main stages; bits per element of the stored cache."""
    from e8_lattice_vector_nq_b200 import nq

    codec, stream, dev = t["codec"], t["stream"], t["Kd"].device
    units, heads, n = codec.units, codec.heads, codec.n
    ks = nq.ExactStore.empty(units, heads, n, wl.bits_k, dev)
    vs = nq.ExactStore.empty(units, heads, n, wl.bits_v, dev)
    Kq, Vq, Kd, Vd = t["Kq"], t["Vq"], t["Kd"], t["Vd"]

    def enc():
        nq.nq_encode_exact(Kq, Vq, ks, vs, n, codec.rope, codec.max_pos, kept=codec.kept)

    def dec():
        nq.nq_decode_exact(ks, vs, n, Kd, Vd, codec.rope, codec.max_pos, positions=codec.kept)

    def tm(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b) / reps, world, dev)

    reps = max(3, min(args.steps, 10))
    enc_ms, dec_ms = tm(enc, reps), tm(dec, reps)
    # the outputs hold the exact layout's reconstruction now: put the regular one back
    nq.nq_decode(codec.k_store, codec.v_store, n, Kd, Vd, codec.rope, codec.max_pos,
                 positions=codec.kept)
    torch.cuda.synchronize()
    assert nq.device_error() == 0
    per_vec_bytes = 16 * wl.bits_k + 2 + 16 * wl.bits_v + 2
    kept_bytes = (n * 4 * units) if codec.kept is not None else 0
    alg = units * n * heads * (512 + per_vec_bytes) + kept_bytes
    elems = (t["K"].numel() + t["V"].numel())
    stored = ks.nbytes + vs.nbytes + kept_bytes
    roof = {}
    for stage, ms in (("encode", enc_ms), ("decode", dec_ms)):
        ach = alg / (ms * 1e-3) / 1e9
        roof[stage] = {"kernel": kernel_of(stage, heads, units, n) + " (exact layout)", "bound": "hbm",
                       "achieved": ach, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                       "frac": ach / peak, "algorithmic_bytes": alg, "ms": ms}
    return {"encode_ms": enc_ms, "decode_ms": dec_ms,
            "bits_per_coordinate": {"k": (16 * wl.bits_k + 2) * 8 / 128,
                                    "v": (16 * wl.bits_v + 2) * 8 / 128},
            "bits_per_elem": stored * 8 / elems, "rooflines": roof,
            "encode_vs_regular": enc_ms / t["per_stage"]["encode"],
            "decode_vs_regular": dec_ms / t["per_stage"]["decode"]}


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
    # eight query heads per KV head (the variant that runs one CTA per SM)
    q8 = torch.randn(units, heads * 8, 128, device=Kd.device, generator=g)
    ws8 = torch.empty(max(nq.lib().nq_attend_workspace_bytes(units, heads, 8, n), 16) // 4,
                      dtype=torch.float32, device=Kd.device)
    f8_ms = t(lambda: nq.nq_attend(q8, codec.k_store, codec.v_store, n, 8, codec.rope,
                                   codec.max_pos, scale=scale, positions=codec.kept, ws=ws8))
    return {"query_heads_per_kv_head": G, "tokens": n, "units": units, "kv_heads": heads,
            "fused_ms": f_ms, "decode_then_sdpa_ms": u_ms, "sdpa_on_bf16_ms": s_ms,
            "speedup_vs_decode_then_sdpa": u_ms / f_ms,
            "fused_packed_read_gbs": packed / (f_ms * 1e-3) / 1e9,
            "fused_ms_8_query_heads_per_kv_head": f8_ms,
            "fused_packed_read_gbs_8_query_heads": packed / (f8_ms * 1e-3) / 1e9}


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
    cache (keys and values): coded size and encode / decode time, with and
    without the token difference.  One call per store covers as many layers
    as its 32-bit stream offsets allow (all of them up to 32K tokens; chunks of
    layers beyond).  Code bits are per kept element; the cache figure (coded
    codes + raw meta) is per element of the bf16 input cache, like
    bits_per_elem.  CUDA events, max over ranks."""
    from e8_lattice_vector_nq_b200 import nq

    L = nq.lib()
    units, heads, n = codec.units, codec.heads, codec.n
    per = units
    while per > 1 and L.nq_entropy_max_words(per, heads, n) > 0xFFFFFFFF:
        per = (per + 1) // 2
    chunks = [slice(u, min(u + per, units)) for u in range(0, units, per)]
    res = {"layers_per_call": per, "calls_per_store": len(chunks)}
    elems = 0
    for name, st in (("k", codec.k_store), ("v", codec.v_store)):
        elems += st.meta.numel() * 128
    dev = codec.k_store.codes.device
    out = {"k": nq.PackedStore.empty(units, heads, n, codec.k_store.bits, dev),
           "v": nq.PackedStore.empty(units, heads, n, codec.v_store.bits, dev)}
    ws = nq.entropy_workspace(per, heads, n, dev)
    stores = {"k": codec.k_store, "v": codec.v_store}
    coded = {}
    for delta in (True, False):

        def enc():
            for name, st in stores.items():
                for c, sl in enumerate(chunks):
                    coded[(name, c)] = nq.nq_entropy_encode(st.select_units(sl), n, delta=delta,
                                                            ws=ws, coded=coded.get((name, c)))

        def dec():
            for name in stores:
                for c, sl in enumerate(chunks):
                    nq.nq_entropy_decode(coded[(name, c)], out[name].select_units(sl))

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
        exact = all(torch.equal(out[nm].codes, st.codes) for nm, st in stores.items())
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


def pinned_buffers(K, V, Kd, Vd):
    """Pinned host copies for the leading units of the cache: all of them if
    the host lets the process pin that much, else the largest power-of-two
    share that it does (page-locking can fail on hosts with a low lock limit)."""
    units = K.shape[0]
    use = units
    while use >= 1:
        bufs = []
        try:
            for t in (K, V, Kd, Vd):
                bufs.append(torch.empty((use,) + tuple(t.shape[1:]), dtype=t.dtype,
                                        pin_memory=True))
            return use, bufs
        except RuntimeError:
            del bufs
            torch.cuda.synchronize()
            use //= 2
    return 0, None


def entropy_correlated(args, device, world, rho: float = 0.95, layers: int = 4):
    """The delta + rANS stage on a cache whose tokens are correlated (an AR(1)
    process along the tokens, rho between neighbours; synth.gen_layer_correlated),
    the situation the pages' "consecutive tokens give similar lattice indices"
    describes: Mistral-shaped layers, no eviction (consecutive tokens stay
    neighbours), K3V2.  Coded size with and without the token difference, and
    the lossless round trip."""
    from e8_lattice_vector_nq_b200 import nq

    wl = synth.WORKLOADS["mistral7b_32k"]
    K = torch.empty(layers, wl.heads, wl.tokens, 128, dtype=torch.bfloat16, device=device)
    V = torch.empty_like(K)
    for l in range(layers):
        k, v = synth.gen_layer_correlated(wl, l, device, rho=rho)
        K[l].copy_(k)
        V[l].copy_(v)
    codec = nq.Codec(layers, wl.heads, wl.tokens, wl.theta, wl.bits_k, wl.bits_v, device=device)
    codec.encode(K, V)
    elems = (codec.k_store.meta.numel() + codec.v_store.meta.numel()) * 128
    code_bytes = codec.k_store.codes.numel() * 4 + codec.v_store.codes.numel() * 4
    meta_bytes = codec.k_store.meta.numel() * 4 + codec.v_store.meta.numel() * 4
    res = {"rho": rho, "layers": layers, "tokens": wl.tokens, "heads": wl.heads, "bits": "K3V2",
           "codes_bits_per_elem_raw": code_bytes * 8 / elems}
    for delta in (True, False):
        coded = {nm: nq.nq_entropy_encode(st, codec.n, delta=delta)
                 for nm, st in (("k", codec.k_store), ("v", codec.v_store))}
        exact = True
        for nm, st in (("k", codec.k_store), ("v", codec.v_store)):
            back = nq.PackedStore.empty(layers, wl.heads, codec.n, st.bits, device)
            nq.nq_entropy_decode(coded[nm], back)
            exact = exact and torch.equal(back.codes, st.codes)
        cb = sum(c.coded_bytes() for c in coded.values())
        res["delta" if delta else "plain"] = {
            "codes_bits_per_elem_coded": cb * 8 / elems, "codes_ratio": code_bytes / cb,
            "cache_bits_per_elem_with_meta": (cb + meta_bytes) * 8 / elems,
            "round_trip_exact": bool(exact)}
    del K, V, codec
    torch.cuda.empty_cache()
    return res


def e2e(args, K, V, Kd, Vd, codec, stream, world, in_bytes):
    """Same metric through the public API with HOST buffers: pinned H2D of the
    inputs, the four calls, D2H of the reconstructed cache, every step, as
    nq.HostRoundTrip pipelines them (chunks of layers on three streams).  When
    the host cannot pin the whole cache, the layers it can pin serve as a ring
    that every layer of the cache passes through (values copied); with values
    read in place (eviction) the leading layers it can pin are timed instead.
    The line says which."""
    from e8_lattice_vector_nq_b200 import nq

    units = K.shape[0]
    use, bufs = pinned_buffers(K, V, Kd, Vd)
    if not use:
        return {"unavailable": "the host refused to pin even one layer of the cache"}
    Kh, Vh, Koh, Voh = bufs
    Kh.copy_(K[:use])
    Vh.copy_(V[:use])
    ring = use < units and not codec.evict and use % args.e2e_chunk == 0
    rt = nq.HostRoundTrip(codec, K, V, Kd, Vd, chunk_units=args.e2e_chunk,
                          units=None if ring else use)
    timed = units if ring else use
    sub_in = in_bytes * timed // units

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
    link = link_rates(Kh, K[:use], Kd[:use], Koh)
    h2d = rt.h2d_bytes(Kh, Vh)
    bound = sub_in / (h2d / (link["h2d_gbs"] * 1e9)) / 1e9  # GB/s of KV in, H2D-bound
    value = world * sub_in / (ms * 1e-3) / 1e9
    out = {"value": value, "unit": "GB/s",
           "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": rt.d2h_bytes(Koh, Voh),
           "ms_per_step": ms, "steps": args.e2e_steps, "chunk_layers": args.e2e_chunk,
           "values_read_in_place": rt.values_in_place, "link": link,
           "h2d_bound_gbs": world * bound, "frac_of_h2d_bound": value / (world * bound)}
    if ring:
        out["host_ring_layers"] = use
        out["note"] = (f"the host pinned only {use} of {units} layers: they serve as a ring that "
                       f"all {units} layers pass through, both ways, every step")
    elif use < units:
        out["layers_timed"] = use
        out["note"] = (f"the host pinned only {use} of {units} layers; the step is those layers "
                       f"(the rate is per byte of bf16 KV in)")
    del Kh, Vh, Koh, Voh, bufs
    return out


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
