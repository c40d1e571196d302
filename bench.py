#!/usr/bin/env python
"""Benchmark of the fused SDPA forward on B200.

Headline workload (one step = one decode call through the C ABI):
  decode ("vector" path of MLX issue #3885): bf16, B=1, qL=1, kL=4096,
  Hq=32, Hkv=8 (GQA 4), D=256, additive mask [1,1,1,kL] U(-1,0) with the last
  10% of keys -inf; Q/K/V ~ N(0,1) seeded.
Metric: decode KV GB/s = algorithmic bytes (K+V+Q+O footprint) / time.  Reported
alongside:
  "prefill": TFLOP/s of the head-dim-72 and head-dim-512 bf16 prefill workloads
             and of one fp32 prefill row (FFMA roofline);
  "mla_decode": microseconds per absorbed-MLA decode call on the small latent
             fixture (fp32 and bf16);
  "e2e": the headline metric through the C ABI from pinned host buffers;
  "cpu_baseline": the float64 oracle on the host's cores.

Timing: W warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, CUDA events on the launching stream,
max over ranks.  The K/V cache rotates over enough copies to exceed the
126 MB L2, so every step reads K and V from HBM.  The steps are replayed from
a CUDA graph (the decode call is a few microseconds; eager launches would time
the host).  Multi-GPU: every rank runs the same per-GPU problem on its own
copy (the (batch, KV-head) units are independent: no data-path collective),
so scaling is weak and the value is the sum over ranks.

``--impl reference`` times the float64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SDPA prefill TFLOP/s & decode KV GB/s on 1 B200, as fraction of roofline"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- workloads
def decode_workload(kL=4096):
    return dict(name=f"decode bf16 B=1 qL=1 kL={kL} Hq=32 Hkv=8 D=256 additive mask [1,1,1,kL] (last 10% -inf)",
                seed=1001, B=1, Hq=32, Hkv=8, Lq=1, Lk=kL, Dqk=256, Dv=256, dtype="bf16", mask="decode_additive",
                layout="bhld")


PREFILL_WORKLOADS = [
    dict(name="prefill bf16 B=1 H=16 L=8192 D=72 no mask [B,L,H,D]", seed=1003, B=1, Hq=16, Hkv=16, Lq=8192,
         Lk=8192, Dqk=72, Dv=72, dtype="bf16", mask="none", layout="blhd"),
    dict(name="prefill fp16 B=1 H=16 L=8192 D=72 no mask [B,L,H,D]", seed=1003, B=1, Hq=16, Hkv=16, Lq=8192,
         Lk=8192, Dqk=72, Dv=72, dtype="f16", mask="none", layout="blhd"),
    dict(name="prefill bf16 B=1 H=16 L=8192 D=72 bool mask [1,1,L,L] p_keep=0.9 [B,L,H,D]", seed=1003, B=1,
         Hq=16, Hkv=16, Lq=8192, Lk=8192, Dqk=72, Dv=72, dtype="bf16", mask="bool", layout="blhd"),
    dict(name="prefill bf16 B=1 Hq=32 Hkv=4 L=4096 D=512 causal", seed=1002, B=1, Hq=32, Hkv=4, Lq=4096, Lk=4096,
         Dqk=512, Dv=512, dtype="bf16", mask="causal", layout="bhld"),
    dict(name="prefill fp32 B=2 Hq=32 Hkv=8 L=2048 D=64 no mask (sweep row, three-term TF32 on tcgen05)",
         seed=1004, B=2, Hq=32, Hkv=8, Lq=2048, Lk=2048, Dqk=64, Dv=64, dtype="f32", mask="none", layout="bhld"),
    dict(name="prefill fp32 B=2 Hq=32 Hkv=8 L=2048 D=128 no mask (sweep row, FFMA path)", seed=1004, B=2, Hq=32,
         Hkv=8, Lq=2048, Lk=2048, Dqk=128, Dv=128, dtype="f32", mask="none", layout="bhld"),
    dict(name="prefill bf16 B=1 Hq=32 Hkv=16 L=8192 D=256 sliding window 1024 (Gemma-4 sliding-layer shape)",
         seed=1010, B=1, Hq=32, Hkv=16, Lq=8192, Lk=8192, Dqk=256, Dv=256, dtype="bf16", mask="sliding",
         window=1024, layout="bhld"),
]

# fp32 on the CUDA cores (FFMA): peak = SMs x 128 FMA lanes x 2 FLOP x max SM clock
FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# fp32 on the tensor cores (kind::tf32): the measured bf16 peak x the nominal dense
# tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s); the three-term split issues 3 MMAs per product
TF32_OVER_BF16 = 1.1 / 2.25


def decode_bytes(w):
    """Algorithmic bytes of one decode call: K+V read once (for a sliding window,
    only the keys some query's window holds), Q read, O written."""
    e = 2 if w["dtype"] in ("bf16", "f16") else 4
    keys = w["Lk"] if w["mask"] != "sliding" else min(w["Lk"], w["window"] + w["Lq"] - 1)
    kv = w["B"] * w["Hkv"] * keys * (w["Dqk"] + w["Dv"])
    qo = w["B"] * w["Hq"] * w["Lq"] * (w["Dqk"] + w["Dv"])
    return e * (kv + qo)


def visible_keys(w):
    """Keys summed over the query rows of one (batch, head) that the mask leaves visible
    (every key; half for causal at Lq = Lk; the window's keys for a sliding window)."""
    Lq, Lk = w["Lq"], w["Lk"]
    if w["mask"] == "sliding":
        own = np.arange(Lq, dtype=np.int64) + (Lk - Lq)
        return int(np.clip(np.minimum(own + 1, w["window"]), 0, None).sum())
    return Lq * Lk / 2 if w["mask"] == "causal" else Lq * Lk


def prefill_flops(w):
    """Algorithmic FLOPs: 2 (Dqk + Dv) per visible (query, key) pair."""
    return 2.0 * w["B"] * w["Hq"] * visible_keys(w) * (w["Dqk"] + w["Dv"])


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "scaled_dot_product_14_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(key, files):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(key)
    if not d or d.get("source_sha") != kernel_source_hash(files):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(busy), "power_w_max": max(r["power"] for r in rows)}


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU, ranks from the launcher's RANK / LOCAL_RANK / WORLD_SIZE.
    NCCL between GPUs; gloo runs the same plumbing on host memory only."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n_gpus != world:
        print(f"note: --gpus {n_gpus} but WORLD_SIZE={world}; using {world} rank(s)", file=sys.stderr)
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world, bytes_per_step, steps, ms):
    """Whole-job throughput: every rank moves bytes_per_step per step (weak scaling),
    over the slowest rank's time."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------- our arm
def device_case(w, rank):
    import torch
    from scaled_dot_product_14_b200 import inputs as I
    c = I.make_case(w["seed"] + 17 * rank, w["B"], w["Hq"], w["Hkv"], w["Lq"], w["Lk"], w["Dqk"], w["Dv"],
                    dtype=I.DTYPE_BY_NAME[w["dtype"]], mask=w["mask"], layout=w["layout"],
                    window=w.get("window", 0))

    def dev(a, is_mask=False):
        if is_mask and c.mask_kind == I.MASK_BOOL:
            return torch.from_numpy(a).cuda()
        if c.dtype == I.F32:
            return torch.from_numpy(a).cuda()
        tdt = torch.bfloat16 if c.dtype == I.BF16 else torch.float16
        return torch.from_numpy(a.view(np.int16)).view(tdt).cuda()

    t = dict(q=dev(c.q), k=dev(c.k), v=dev(c.v), mask=None if c.mask is None else dev(c.mask, True))
    return c, t


def call(S, c, t, k, v, out, stream):
    if c.window:
        st = S.sdpa_forward_window(t["q"].data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), c.B, c.Hq, c.Hkv,
                                   c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, c.scale, c.window, c.dtype, stream)
        if st != 0:
            raise S.SdpaError(st, "sdpa_forward_window")
        return
    st = S.sdpa_forward(t["q"].data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), c.B, c.Hq, c.Hkv, c.Lq, c.Lk,
                        c.Dqk, c.Dv, c.all_strides16, c.scale, c.mask_kind,
                        None if t["mask"] is None else t["mask"].data_ptr(),
                        None if t["mask"] is None else c.mask_strides, c.dtype, stream)
    if st != 0:
        raise S.SdpaError(st)


def decode_graph(S, c, t, copies, steps, stream):
    """A CUDA graph of exactly `steps` C-ABI decode calls, call i on K/V copy i % copies."""
    import torch
    ks = [t["k"]] + [t["k"].clone() for _ in range(copies - 1)]
    vs = [t["v"]] + [t["v"].clone() for _ in range(copies - 1)]
    out = torch.empty(c.B * c.Hq * c.Lq * c.Dv, dtype=t["q"].dtype, device="cuda")
    sp = stream.cuda_stream
    with torch.cuda.stream(stream):
        call(S, c, t, ks[0], vs[0], out, sp)          # allocates the split-K workspace before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(steps):
            call(S, c, t, ks[i % copies], vs[i % copies], out, sp)
    torch.cuda.synchronize()
    return graph, ks, vs, out


def time_decode(S, w, rank, world, stream, steps, warmup, soak, clocks=None):
    """W eager warm-up calls, an untimed soak of graph replays, then one replay
    of a graph of exactly `steps` calls between events on the launching stream
    (barrier and synchronize on both sides; max over ranks)."""
    import torch
    c, t = device_case(w, rank)
    kv_bytes = t["k"].numel() * t["k"].element_size() + t["v"].numel() * t["v"].element_size()
    copies = max(2, math.ceil(2 * L2_BYTES / kv_bytes))
    graph, ks, vs, out = decode_graph(S, c, t, copies, steps, stream)
    sp = stream.cuda_stream
    launches = S.sdpa_last_launch_count()
    with torch.cuda.stream(stream):
        for i in range(warmup):
            call(S, c, t, ks[i % copies], vs[i % copies], out, sp)
    if clocks:
        clocks.start()
    soak_end = time.time() + soak
    while time.time() < soak_end:
        with torch.cuda.stream(stream):
            graph.replay()
        stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):            # replay() launches on the current stream
        ev0.record(stream)
        graph.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)

    # each launch alone: the library brackets each kernel with events on the
    # launching stream; a GPU-side sleep queued first lets the profiled launches
    # queue up behind it, so they run back to back with no host gaps
    S.sdpa_profile_enable(True)
    S.sdpa_profile_collect()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(20_000_000)          # ~10 ms of GPU time while the host enqueues
        for r in range(2 * copies):
            call(S, c, t, ks[r % copies], vs[r % copies], out, sp)
    torch.cuda.synchronize()
    prof = S.sdpa_profile_collect()
    S.sdpa_profile_enable(False)
    fam = "decode_mma" if c.dtype != 0 else "decode_ffma"
    n_dec, ms_dec = prof[fam]
    del graph, ks, vs, out, t
    return dict(c=c, ms=ms, copies=copies, kv_bytes=kv_bytes, launches=launches, clocks=clk,
                us_isolated=1e3 * ms_dec / max(n_dec, 1))


def run_ours(args, peaks):
    import torch
    import scaled_dot_product_14_b200 as S
    from scaled_dot_product_14_b200 import build
    world, rank, local = dist_setup(args.gpus)
    if rank == 0 and not os.path.exists(S.LIB_PATH):
        build.build()
    barrier(world)
    stream = torch.cuda.Stream()
    steps, warmup = args.steps, max(args.warmup, 3)

    w = decode_workload(args.kl)
    bytes_per_step = decode_bytes(w)
    r = time_decode(S, w, rank, world, stream, steps, warmup, args.soak, ClockSampler(local))
    ms_per_step = r["ms"] / steps
    value = aggregate_gbs(world, bytes_per_step, steps, r["ms"])
    launches_per_step = r["launches"]
    # The decode kernel is the only kernel of a step (one launch per call on this
    # path): its average launch duration over the timed region is the timed
    # region's duration divided by the launches in it.
    dec_us = 1e3 * ms_per_step / max(launches_per_step, 1)
    achieved = bytes_per_step / (dec_us * 1e-6) / 1e9
    traffic = ncu_traffic(f"decode_mma kL={args.kl}", ["decode_mma.cu", "common.cuh", "kernels.h"])
    roof = {"bound": "hbm", "kernel": "decode_mma_kernel", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "algorithmic_bytes_per_launch": bytes_per_step,
            "kernel_us": round(dec_us, 3), "launches_per_step": launches_per_step,
            "kernel_us_isolated": round(r["us_isolated"], 3),
            "frac_isolated": round(bytes_per_step / (r["us_isolated"] * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
            "timing": "kernel_us = timed region / launches in it (CUDA events on the launching stream, "
                      "graph replay, consecutive launches overlap their prologues); kernel_us_isolated = "
                      "event pair around each launch, launches queued back to back",
            "peak_source": f"{peaks['source']} hbm_gbs (copy, burst)"}

    result = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": steps,
              "warmup": warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
              "config": {"workload": w["name"], "kv_copies_rotated": r["copies"],
                         "l2": f"inputs larger than L2: {r['copies']} rotating K/V copies "
                               f"({r['copies'] * r['kv_bytes'] / 2**20:.0f} MiB > 126 MB L2)",
                         "launch": "CUDA graph of the C-ABI calls, one replay", "soak_s": args.soak,
                         "parallelism": f"replicas x{world} (no collective)"},
              "roofline": roof, "clocks": r["clocks"], "gpu_launches": launches_per_step * steps}

    if not args.no_e2e:
        c, t = device_case(w, rank)
        out = torch.empty(c.B * c.Hq * c.Lq * c.Dv, dtype=t["q"].dtype, device="cuda")
        result["e2e"] = e2e(S, c, t, out, stream, args, world)
        del c, t, out
    if not args.no_extra:
        result["decode"] = decode_leg(S, stream, peaks, rank, world, args)
    if not args.no_prefill:
        result["prefill"] = prefill_leg(S, stream, peaks, rank, args, local)
        result["mla_decode"] = mla_leg(S, stream, peaks, rank, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        if not args.no_extra:
            result["cpu_baseline_configs"] = cpu_baseline_configs(args.cpu_seconds / 4)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


DECODE_EXTRA = [
    decode_workload(1024),
    dict(name="decode bf16 B=1 qL=1 kL=4096 Hq=32 Hkv=16 D=256 sliding window 1024 (Gemma-4 sliding-layer shape)",
         seed=1011, B=1, Hq=32, Hkv=16, Lq=1, Lk=4096, Dqk=256, Dv=256, dtype="bf16", mask="sliding", window=1024,
         layout="bhld"),
    dict(name="decode bf16 B=1 qL=1 kL=1024 Hq=32 Hkv=4 D=512 no mask", seed=1002, B=1, Hq=32, Hkv=4, Lq=1,
         Lk=1024, Dqk=512, Dv=512, dtype="bf16", mask="none", layout="bhld"),
    dict(name="decode bf16 B=1 qL=1 kL=4096 Hq=32 Hkv=4 D=512 no mask", seed=1002, B=1, Hq=32, Hkv=4, Lq=1,
         Lk=4096, Dqk=512, Dv=512, dtype="bf16", mask="none", layout="bhld"),
]


def decode_leg(S, stream, peaks, rank, world, args):
    """The other decode configurations, timed like the headline (graph replay of
    exactly --steps calls over rotating K/V copies larger than L2)."""
    res = []
    for w in DECODE_EXTRA:
        r = time_decode(S, w, rank, world, stream, args.steps, max(args.warmup, 3), 0.2)
        nb = decode_bytes(w)
        us = 1e3 * r["ms"] / args.steps / max(r["launches"], 1)
        gbs = nb / (us * 1e-6) / 1e9
        res.append({"workload": w["name"], "us_per_call": round(us, 3),
                    "us_isolated": round(r["us_isolated"], 3), "algorithmic_bytes": nb,
                    "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm_gbs"],
                    "frac": round(gbs / peaks["hbm_gbs"], 4), "bound": "hbm", "launches_per_call": r["launches"],
                    "steps": args.steps, "kv_copies_rotated": r["copies"]})
    return res


def run_prefill_only(args, peaks):
    import torch
    import scaled_dot_product_14_b200 as S
    from scaled_dot_product_14_b200 import build
    if not os.path.exists(S.LIB_PATH):
        build.build()
    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    for entry in prefill_leg(S, stream, peaks, 0, args, 0):
        print(json.dumps(entry), flush=True)


def usable_cpus():
    """CPUs this process may run on (its affinity set), which is what the oracle's
    thread pool can actually use."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def parse_cpulist(text):
    """A sysfs CPU list ("0-3,8,10-11") as a set of CPU numbers."""
    cpus = set()
    for part in text.strip().split(","):
        part = part.strip()
        if not part:
            continue
        if "-" in part:
            a, b = part.split("-")
            cpus.update(range(int(a), int(b) + 1))
        else:
            cpus.add(int(part))
    return cpus


def gpu_local_cpus(device):
    """The CPUs of the GPU's NUMA node (sysfs local_cpulist of its PCI function)
    that this process may run on, or None when that cannot be read."""
    import torch
    try:
        pr = torch.cuda.get_device_properties(device)
        path = (f"/sys/bus/pci/devices/{pr.pci_domain_id:04x}:{pr.pci_bus_id:02x}:"
                f"{pr.pci_device_id:02x}.0/local_cpulist")
        with open(path) as f:
            cpus = parse_cpulist(f.read()) & os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


def e2e(S, c, t, out, stream, args, world):
    """Same metric through the C ABI from pinned host buffers: H2D of the step's
    inputs, the call, D2H of the output, all inside the timed region.  The host
    buffers are allocated and driven from the CPUs next to the GPU (the process's
    CPU affinity is restored afterwards)."""
    import torch
    saved = os.sched_getaffinity(0)
    local_cpus = gpu_local_cpus(torch.cuda.current_device())
    pinned = False
    if local_cpus:
        try:
            os.sched_setaffinity(0, local_cpus)
            pinned = True
        except OSError:
            pass
    try:
        res = _e2e_timed(S, c, t, out, stream, args, world)
    finally:
        if pinned:
            try:
                os.sched_setaffinity(0, saved)
            except OSError:
                pass
    res["host_cpus"] = (f"{len(local_cpus)} CPUs of the GPU's NUMA node" if pinned
                        else "process default (GPU NUMA node not found)")
    return res


def _e2e_timed(S, c, t, out, stream, args, world):
    import torch
    host = {k: v.cpu().pin_memory() for k, v in t.items() if v is not None}
    dev = {k: torch.empty_like(v) for k, v in t.items() if v is not None}
    host_out = torch.empty(out.numel(), dtype=out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out.numel() * out.element_size()
    n = max(3, min(args.steps, 50))

    def step():
        for k in host:
            dev[k].copy_(host[k], non_blocking=True)
        td = dict(dev)
        td.setdefault("mask", None)
        call(S, c, td, dev["k"], dev["v"], out, stream.cuda_stream)
        host_out.copy_(out, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            step()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    val = aggregate_gbs(world, decode_bytes(decode_workload(args.kl)), n, ms)
    return {"value": round(val, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "ms_per_step": round(ms / n, 4)}


def prefill_leg(S, stream, peaks, rank, args, local=0):
    """Each prefill workload: an untimed soak (clocks sampled meanwhile), then
    `iters` launches each timed alone with events on the launching stream, the
    L2 flushed (a 256 MiB write) between them."""
    import torch
    res = []
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")
    for w in PREFILL_WORKLOADS:
        S.sdpa_reset_counters()   # the kernel family of this workload is read back below
        c, t = device_case(w, rank)
        out = torch.empty(c.B * c.Hq * c.Lq * c.Dv, dtype=t["q"].dtype, device="cuda")
        sp = stream.cuda_stream
        clocks = ClockSampler(local) if args.prefill_soak > 0 else None
        with torch.cuda.stream(stream):
            for _ in range(10):                 # warm-up launches
                call(S, c, t, t["k"], t["v"], out, sp)
            torch.cuda.synchronize()
            if clocks:
                clocks.start()
                soak_end = time.time() + args.prefill_soak
                while time.time() < soak_end:
                    for _ in range(8):
                        call(S, c, t, t["k"], t["v"], out, sp)
                    stream.synchronize()
            n = args.prefill_iters
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            for e0, e1 in evs:
                flush.fill_(1)
                e0.record(stream)
                call(S, c, t, t["k"], t["v"], out, sp)
                e1.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop() if clocks else None
        times = [e0.elapsed_time(e1) for e0, e1 in evs]
        ms = statistics.median(times)
        fl = prefill_flops(w)
        tf = fl / (ms * 1e-3) / 1e12
        cnt = S.sdpa_get_counters()
        kernel = ("prefill_tcgen05" if cnt["prefill_tcgen05_launches"] else
                  "prefill_tf32x3" if cnt["prefill_tf32_launches"] else "prefill_ffma")
        if kernel == "prefill_ffma":
            peak, src, bound = FFMA_TFLOPS, "FFMA: 148 SMs x 128 lanes x 2 x 1.965 GHz (nominal)", "alu"
        elif kernel == "prefill_tf32x3":
            peak = peaks["bf16_tflops"] * TF32_OVER_BF16
            src = (f"{peaks['source']} bf16_tflops x 1.1/2.25 (nominal dense tf32/bf16); "
                   "3 tf32 MMAs per product, so frac <= 1/3 and tensor_pipe_frac = 3 x frac")
            bound = "tensor"
        else:
            peak, src, bound = peaks["bf16_tflops"], f"{peaks['source']} bf16_tflops (cuBLAS, burst)", "tensor"
        entry = {"workload": w["name"], "ms": round(ms, 4), "ms_min": round(min(times), 4),
                 "ms_max": round(max(times), 4), "tflops": round(tf, 2),
                 "algorithmic_flops": fl, "peak_tflops": round(peak, 1), "peak_source": src,
                 "frac": round(tf / peak, 4), "bound": bound, "kernel": kernel,
                 **({"tensor_pipe_frac": round(3 * tf / peak, 4)} if kernel == "prefill_tf32x3" else {}),
                 "iters": n, "warmup": 10, "timing": "median of the timed launches",
                 "l2": "flushed between timed launches"}
        if clk:
            entry["clocks"] = clk
        res.append(entry)
        del t, out
        torch.cuda.empty_cache()
    del flush
    return res


MLA_WORKLOAD = dict(name="mla absorbed decode (keys = 32 latent + 8 rope, values = the latent columns of the "
                         "same rows) B=1 Hq=4 Hkv=1 qL=1 kL=4096, additive mask [1,1,1,kL]",
                    seed=1008, B=1, Hq=4, Hkv=1, Lq=1, Lk=4096, Dqk=40, Dv=32, mask="decode_additive",
                    layout="bhld")


def mla_leg(S, stream, peaks, rank, args):
    """Absorbed-MLA decode on the small latent fixture: V is passed as the first
    32 columns of K (same buffer, K's strides), so each latent row is read once.
    Launches timed alone with events, the L2 flushed between them."""
    import dataclasses
    import torch
    res = []
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")
    for dt in ("f32", "bf16"):
        w = dict(MLA_WORKLOAD, dtype=dt)
        c, t = device_case(w, rank)
        st = list(c.strides)
        st[8:12] = st[4:8]                         # V strides = K strides
        c = dataclasses.replace(c, strides=tuple(st))
        t["v"] = t["k"]
        out = torch.empty(c.B * c.Hq * c.Lq * c.Dv, dtype=t["q"].dtype, device="cuda")
        sp = stream.cuda_stream
        with torch.cuda.stream(stream):
            for _ in range(3):
                call(S, c, t, t["k"], t["v"], out, sp)
            n = args.prefill_iters
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            for e0, e1 in evs:
                flush.fill_(1)
                e0.record(stream)
                call(S, c, t, t["k"], t["v"], out, sp)
                e1.record(stream)
        torch.cuda.synchronize()
        us = 1e3 * statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
        e = 4 if dt == "f32" else 2
        nbytes = e * (c.B * c.Hkv * c.Lk * c.Dqk + c.B * c.Hq * c.Lq * (c.Dqk + c.Dv))
        gbs = nbytes / (us * 1e-6) / 1e9
        res.append({"workload": w["name"], "dtype": dt, "us_per_call": round(us, 3),
                    "algorithmic_bytes": nbytes, "mask_bytes": e * c.Lk, "achieved_gbs": round(gbs, 1),
                    "peak_gbs": peaks["hbm_gbs"], "frac": round(gbs / peaks["hbm_gbs"], 4),
                    "bound": "latency (0.3-0.7 MB per call: memory round trips, not bandwidth)",
                    "launches_per_call": S.sdpa_last_launch_count(),
                    "iters": n, "timing": "median", "l2": "flushed between timed launches"})
        del t, out
    del flush
    return res


def cpu_baseline(w, seconds):
    """The float64 oracle as it stands on this host's cores, on full decode steps."""
    import oracle
    from scaled_dot_product_14_b200 import inputs as I
    oracle.build()
    c = I.make_case(w["seed"], w["B"], w["Hq"], w["Hkv"], w["Lq"], w["Lk"], w["Dqk"], w["Dv"],
                    dtype=I.DTYPE_BY_NAME[w["dtype"]], mask=w["mask"], layout=w["layout"])
    threads = usable_cpus()
    n, t0 = 0, time.time()
    while True:
        oracle.sdpa_rows(c.q, c.k, c.v, B=c.B, Hq=c.Hq, Hkv=c.Hkv, Lq=c.Lq, Lk=c.Lk, Dqk=c.Dqk, Dv=c.Dv,
                         strides=c.strides, scale=c.scale, dtype=c.dtype, mask_kind=c.mask_kind, mask=c.mask,
                         mask_strides=c.mask_strides, threads=threads)
        n += 1
        if time.time() - t0 >= seconds or n >= 1000:
            break
    el = time.time() - t0
    return {"value": round(decode_bytes(w) * n / el / 1e9, 4), "unit": "GB/s", "cores": min(threads, c.B * c.Hq),
            "kind": "oracle", "sample": f"{n} full decode steps ({c.B * c.Hq} query rows x {c.Lk} keys each) "
                                        f"in {el:.1f} s; rows split over host threads"}


ORACLE_CONFIGS = [
    dict(name="config 1: fp32 B=2 L=82 H=8 D=64 no mask [B,L,H,D] (N(0,1) copy)", seed=1000, B=2, Hq=8, Hkv=8,
         Lq=82, Lk=82, Dqk=64, Dv=64, dtype="f32", mask="none", layout="blhd", kind="prefill"),
    dict(decode_workload(1024), kind="decode"),
    dict(DECODE_EXTRA[2], kind="decode"),
    dict(DECODE_EXTRA[3], kind="decode"),
    dict(PREFILL_WORKLOADS[3], kind="prefill"),
    dict(PREFILL_WORKLOADS[0], kind="prefill"),
    dict(PREFILL_WORKLOADS[1], kind="prefill"),
    dict(PREFILL_WORKLOADS[2], kind="prefill"),
]


def cpu_baseline_configs(seconds):
    """The float64 oracle, as it stands, on configs 1-4 (host cores, rows split
    over threads).  Decode configs and config 1 run whole calls; the large
    prefill configs run seeded samples of query rows for about `seconds` each,
    and their throughput is extrapolated from the time per row."""
    import oracle
    from scaled_dot_product_14_b200 import inputs as I
    oracle.build()
    threads = usable_cpus()
    res = []
    for w in ORACLE_CONFIGS:
        c = I.make_case(w["seed"], w["B"], w["Hq"], w["Hkv"], w["Lq"], w["Lk"], w["Dqk"], w["Dv"],
                        dtype=I.DTYPE_BY_NAME[w["dtype"]], mask=w["mask"], layout=w["layout"])
        total_rows = c.B * c.Hq * c.Lq
        args = dict(B=c.B, Hq=c.Hq, Hkv=c.Hkv, Lq=c.Lq, Lk=c.Lk, Dqk=c.Dqk, Dv=c.Dv, strides=c.strides,
                    scale=c.scale, dtype=c.dtype, mask_kind=c.mask_kind, mask=c.mask, mask_strides=c.mask_strides,
                    threads=threads)
        whole = total_rows * c.Lk <= 2 ** 22
        n_rows, t0, calls = 0, time.time(), 0
        while True:
            if whole:
                oracle.sdpa_rows(c.q, c.k, c.v, **args)
                n_rows += total_rows
            else:
                rows = I.sample_rows(w["seed"] + calls, c.B, c.Hq, c.Lq, 4 * threads, include_edges=False)
                oracle.sdpa_rows(c.q, c.k, c.v, rows=rows, **args)
                n_rows += len(rows)
            calls += 1
            if time.time() - t0 >= seconds:
                break
        el = time.time() - t0
        est_s = el / n_rows * total_rows          # one whole call
        if w["kind"] == "decode":
            val, unit = decode_bytes(w) / est_s / 1e9, "GB/s"
        else:
            val, unit = prefill_flops(w) / est_s / 1e12, "TFLOP/s"
        res.append({"workload": w["name"], "value": round(val, 6), "unit": unit, "cores": threads,
                    "kind": "oracle", "seconds_per_call": round(est_s, 4),
                    "sample": (f"{calls} whole calls in {el:.1f} s" if whole else
                               f"{n_rows} seeded query rows of {total_rows} in {el:.1f} s; "
                               f"extrapolated per row x rows")})
    return res


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from scaled_dot_product_14_b200 import inputs as I
    oracle.build()
    w = decode_workload(args.kl)
    c = I.make_case(w["seed"], w["B"], w["Hq"], w["Hkv"], w["Lq"], w["Lk"], w["Dqk"], w["Dv"],
                    dtype=I.DTYPE_BY_NAME[w["dtype"]], mask=w["mask"], layout=w["layout"])
    threads = usable_cpus()

    def step():
        oracle.sdpa_rows(c.q, c.k, c.v, B=c.B, Hq=c.Hq, Hkv=c.Hkv, Lq=c.Lq, Lk=c.Lk, Dqk=c.Dqk, Dv=c.Dv,
                         strides=c.strides, scale=c.scale, dtype=c.dtype, mask_kind=c.mask_kind, mask=c.mask,
                         mask_strides=c.mask_strides, threads=threads)

    for _ in range(max(args.warmup, 1)):
        step()
    t0 = time.time()
    for _ in range(args.steps):
        step()
    el = time.time() - t0
    val = decode_bytes(w) * args.steps / el / 1e9
    cores = min(threads, c.B * c.Hq)
    print(json.dumps({"metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": world,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * el / args.steps, 3),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic", "impl": "reference",
                      "config": {"workload": w["name"], "parallelism": "host threads (oracle)"},
                      "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                       "sample": f"each step = one full decode call ({c.B * c.Hq} rows x {c.Lk} keys)"},
                      "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--kl", type=int, default=4096, help="decode key length (1024 or 4096 on the pages)")
    ap.add_argument("--soak", type=float, default=1.0, help="untimed seconds under load before timing")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill workloads and print their lines (profiling)")
    ap.add_argument("--prefill-iters", type=int, default=50)
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other decode configurations and the oracle timing on configs 1-4")
    ap.add_argument("--prefill-soak", type=float, default=1.0,
                    help="untimed seconds per prefill workload while clocks are sampled (0: no sampling)")
    args = ap.parse_args()
    if args.prefill_only:
        run_prefill_only(args, load_peaks())
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args, load_peaks())


if __name__ == "__main__":
    main()
