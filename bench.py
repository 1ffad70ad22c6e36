"""Benchmark of the fused compressed-state AdamW step (libfo, sm_100a).

Default workload: the Llama-3.1-8B parameter list (291 tensors, 8,030,261,248
parameters), bf16 + 8-bit ECC masters, 8-bit companded m / v, bf16 Student-t
gradients; one step = one multi-tensor fo_adamw_step launch over all 291
tensors.  Inputs are resident in HBM before timing; one step moves ~98 GB,
far above the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun);
by default the list is sharded over the ranks as in data-parallel training
(--mode dp: NCCL reduce-scatter of the gradients, the fused step on each
rank's groups, all-gather of x'; strong scaling), or every rank steps its own
copy (--mode replicas: weak scaling, no data-path collective); time = max
over ranks of the device-event time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused AdamW step Gparams/s and achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e specification (context beside the measured or fallback peak)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fo", choices=["fo", "reference"])
    ap.add_argument("--config", default="llama3.1-8b")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-piece", type=int, default=1 << 26,
                    help="parameters per host<->device piece of the end-to-end leg (whole groups; 2^26 measured "
                         "best of 2^23..2^26)")
    ap.add_argument("--e2e-ring", type=int, default=3, help="device stage buffers of the end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-params", type=int, default=1 << 24)
    ap.add_argument("--launch-mode", default="multi", choices=["multi", "release"])
    ap.add_argument("--mode", default=None, choices=["fused", "dp", "replicas"],
                    help="fused: one GPU steps the whole list (default for one GPU); dp: the list is sharded "
                         "over the ranks, one step = NCCL reduce-scatter of the 16-bit gradients, the fused "
                         "step on each rank's groups, all-gather of x' (default for several GPUs); replicas: "
                         "every rank steps its own copy of the list, no collective")
    ap.add_argument("--bucket-groups", type=int, default=1 << 22,
                    help="groups of 32 elements per data-parallel bucket (2^22: 128M parameters, 256 MB of "
                         "16-bit gradients)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 512 MB buffer before every timed step and time each step's kernels alone "
                         "(for workloads that fit in the 126 MB L2)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move)

def algorithmic_bytes(wl) -> int:
    """Bytes one step must read + write: downcast weights (r+w), ECC (r+w),
    gradient (r), momentum codes (r+w) and scales (r+w), variance codes and
    scales (r+w, AdamW only)."""
    wb = 2
    eb = wl.ecc_bits // 8
    total = 0
    for t in wl.tensors:
        n = t.numel
        ng = (n + 31) // 32
        rd = n * (wb + eb + 2 + 1) + 2 * ng
        wr = n * (wb + eb + 1) + 2 * ng
        if wl.optimizer == "adamw":
            rd += n + 2 * ng
            wr += n + 2 * ng
        total += rd + wr
    return total


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha() -> str:
    """Hash of the kernel sources' code (comments and whitespace removed), so
    that a profile stays attached to the code it measured."""
    import re

    h = hashlib.sha256()
    for f in ("fo_codec.cuh", "fo_kernels.cuh", "fo_api.cu"):
        with open(os.path.join(ROOT, "bit_states_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def traffic_from_profile(config: str):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(config)
    if not e or e.get("kernel_source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        # samples under load: power above the idle level
        load = [s for s, p in zip(sm, pw) if p > 200.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower().startswith("active")})
        pload = [p for p in pw if p > 200.0] or pw
        # nvidia-smi's power reading trails the load (it averages over a window),
        # so the steady figure is the median of the second half of the samples
        steady = pload[len(pload) // 2:]
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(pw) if pw else None,
                "power_w_median": statistics.median(pload) if pload else None,
                "power_w_steady": statistics.median(steady) if steady else None}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline; also the reference arm)

def cpu_sample(wl, n_params: int, rank_seed: int = 0):
    """A bounded sample of the workload for the oracle: whole groups drawn
    uniformly from every tensor in proportion to its size."""
    import oracle

    rng = np.random.default_rng(1234 + rank_seed)
    total = wl.numel
    parts = []
    for ti, t in enumerate(wl.tensors):
        ng = (t.numel + 31) // 32
        k = max(1, int(round(n_params / 32 * t.numel / total)))
        k = min(k, ng)
        g = np.sort(rng.choice(ng, size=k, replace=False)) if k < ng else np.arange(ng)
        g = g[32 * g + 32 <= t.numel] if (32 * g + 32 > t.numel).any() and g.size > 1 else g
        idx = (32 * g[:, None] + np.arange(32)[None, :]).ravel()
        idx = idx[idx < t.numel]
        x = wl.master_values(ti, idx)
        gb = wl.grad_bits(ti, 1, idx)
        parts.append((x, gb))
    x = np.concatenate([p[0] for p in parts])
    gb = np.concatenate([p[1] for p in parts])
    w, e = oracle.encode_master(x, 0 if wl.w_dtype == "bf16" else 1, wl.ecc_bits, threads=os.cpu_count() or 1)
    return w, e, gb


def time_oracle(wl, n_params: int, steps: int, warmup: int, threads: int, min_seconds: float = 0.0):
    """Oracle throughput on a bounded sample: `warmup` untimed steps, then
    `steps` timed steps, continued until at least `min_seconds` have passed.
    Returns (Gparams/s, seconds, params per step, timed steps)."""
    import oracle

    w, e, gb = cpu_sample(wl, n_params)
    st = oracle.State.zeros_like_master(w, e, adam=(wl.optimizer == "adamw"))
    wdt = 0 if wl.w_dtype == "bf16" else 1
    gdt = 0 if wl.grad_dtype == "bf16" else 1

    def one(t):
        if wl.optimizer == "adamw":
            oracle.adamw_step(st, gb, **wl.hparams, step=t, wdt=wdt, gdt=gdt, ecc_bits=wl.ecc_bits,
                              threads=threads)
        else:
            h = wl.hparams
            oracle.sgdm_step(st, gb, lr=h["lr"], momentum=h["momentum"], dampening=h["dampening"],
                             weight_decay=h["weight_decay"], nesterov=bool(h["nesterov"]), step=t, wdt=wdt,
                             gdt=gdt, ecc_bits=wl.ecc_bits, threads=threads)

    for t in range(1, warmup + 1):
        one(t)
    t0 = time.perf_counter()
    k = 0
    while k < steps or time.perf_counter() - t0 < min_seconds:
        one(warmup + 1 + k)
        k += 1
    dt = time.perf_counter() - t0
    n = w.size
    return n * k / dt / 1e9, dt, n, k


def arm_config(wl, args, world):
    """The workload description both arms print."""
    abytes = algorithmic_bytes(wl)
    return {"workload": f"{wl.name}: {len(wl.tensors)} tensors, {wl.numel} params per GPU, "
                        f"{wl.optimizer} {wl.w_dtype}+ecc{wl.ecc_bits}, int8/uint8 companded states",
            "launch": "one multi-tensor launch per step" if args.launch_mode == "multi" else
                      f"{len(wl.tensors)} per-tensor launches per step (gradient release order)",
            "l2": ("L2 flushed (512 MB write) before every step; steps timed alone" if args.flush_l2 else
                   "inputs larger than L2 (%.2f GB per step vs 126 MB)" % (abytes / 1e9)),
            "parallelism": f"weak-scaling shards x{world}, no data-path collective"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from workloads import workload

    wl = workload(args.config)
    threads = os.cpu_count() or 1
    # each step is a bounded sample of the workload sized to keep the whole
    # run within a few minutes of host time
    n_params = min(args.cpu_sample_params, 1 << 24)
    value, dt, n, steps = time_oracle(wl, n_params, args.steps if args.steps <= 20 else 20, min(args.warmup, 3),
                                      threads)
    sample = f"{n} params per step (whole 32-groups drawn from all {len(wl.tensors)} tensors of {wl.name}), " \
             f"AdamW step 1.., {threads} host threads"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "Gparams/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": min(args.warmup, 3),
            "ms_per_step": round(dt / steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": arm_config(wl, args, world),
            "cpu_baseline": {"value": round(value, 6), "unit": "Gparams/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "Gparams/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm

def main():
    args = parse()
    if args.config.endswith("-release"):
        args.launch_mode = "release"  # the gradient-release workload is one call per tensor
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.mode is None:
        args.mode = "dp" if world > 1 else "fused"
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.mode == "dp":
        return run_dp(args, rank, world, local)

    import torch

    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    from bit_states_b200 import build as fobuild
    from bit_states_b200 import fo
    from bit_states_b200.state import CompressedParams
    from workloads import device as wdev
    from workloads import workload

    fobuild.build()
    wdev.build()
    fo.load()

    wl = workload(args.config)
    wl.seed = rank  # each rank steps its own shard (same shapes, its own values)
    adam = wl.optimizer == "adamw"
    dev = torch.device("cuda", local)
    P = CompressedParams([t.numel for t in wl.tensors], dev, adam=adam, ecc_bits=wl.ecc_bits,
                         w_dtype=wl.w_dtype)
    buf = torch.empty(max(t.numel for t in wl.tensors), dtype=torch.float32, device=dev)
    for ti, t in enumerate(wl.tensors):
        x = buf[:t.numel]
        wdev.master_f32(wl, ti, x)
        P.encode_from(ti, x)
    del buf
    garena = torch.empty(P.total, dtype=torch.int16, device=dev)
    gviews = [garena[o:o + n] for o, n in zip(P.offsets, P.numels)]
    for ti, v in enumerate(gviews):
        wdev.grad_16(wl, ti, 1, v)
    torch.cuda.synchronize()

    fmt = fo.make_format(wl.w_dtype, wl.grad_dtype, wl.ecc_bits)
    h = wl.hparams
    stream = torch.cuda.current_stream()
    descs = fo.descriptors(P.states, gviews)
    order = list(range(len(wl.tensors)))[::-1]
    single = [fo.descriptors([P.states[i]], [gviews[i]]) for i in order]
    launches_per_step = 1 if args.launch_mode == "multi" else len(order)
    if args.launch_mode == "multi" and len(wl.tensors) > 384:
        launches_per_step = (len(wl.tensors) + 383) // 384

    def do_step(t):
        if adam:
            hp = fo.fo_adamw_hparams(h["lr"], h["beta1"], h["beta2"], h["eps"], h["weight_decay"], t)
            if args.launch_mode == "multi":
                fo.fo_adamw_step(descs, len(P.states), fmt, hp, stream)
            else:
                for d in single:
                    fo.fo_adamw_step(d, 1, fmt, hp, stream)
        else:
            hp = fo.fo_sgdm_hparams(h["lr"], h["momentum"], h["dampening"], h["weight_decay"],
                                    int(h["nesterov"]), t)
            if args.launch_mode == "multi":
                fo.fo_sgdm_step(descs, len(P.states), fmt, hp, stream)
            else:
                for d in single:
                    fo.fo_sgdm_step(d, 1, fmt, hp, stream)

    t = 0
    for _ in range(args.warmup):
        t += 1
        do_step(t)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()

    gpu_id = "0"
    try:
        props = torch.cuda.get_device_properties(local)
        gpu_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except Exception:
        gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[local] if "CUDA_VISIBLE_DEVICES" in os.environ else str(local)
    sampler = ClockSampler(gpu_id)
    sampler.start()

    K = args.steps
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None
    # one event pair around the K steps; with an L2 flush between steps, one
    # pair per step, so that only the steps themselves are timed (events
    # between steps would add host work per step, which shows on lists whose
    # step takes tens of microseconds)
    nev = K if flush is not None else 1
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    if flush is None:
        ev_s[0].record(stream)
    for k in range(K):
        t += 1
        if flush is not None:
            flush.fill_(k & 0xFF)
            ev_s[k].record(stream)
        do_step(t)
        if flush is not None:
            ev_e[k].record(stream)
    if flush is None:
        ev_e[0].record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    fo.fo_check_errors()  # raises if a step kernel gave up a bounded wait (chunks left unstepped)
    if flush is not None:
        per_launch_ms = statistics.mean(ev_s[k].elapsed_time(ev_e[k]) for k in range(K))
        total_ms = per_launch_ms * K
    else:
        total_ms = ev_s[0].elapsed_time(ev_e[0])
        per_launch_ms = total_ms / K
    if dist:
        tt = torch.tensor([total_ms, per_launch_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        total_ms, per_launch_ms = float(tt[0]), float(tt[1])

    # ---- the practical ceiling: the same byte mix without the arithmetic ----
    ceiling_ms, ceiling_clocks = None, {}
    if args.launch_mode == "multi":
        def do_copy():
            fo.fo_stream_copy(descs, len(P.states), fmt, adam, stream)

        for _ in range(3):
            do_copy()
        Kc = K  # as many launches as the timed steps, so that clocks and power settle alike
        cs = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
        ce = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
        csampler = ClockSampler(gpu_id)
        csampler.start()
        torch.cuda.synchronize()
        for k in range(Kc):
            if flush is not None:
                flush.fill_(k & 0xFF)
            cs[k].record(stream)
            do_copy()
            ce[k].record(stream)
        torch.cuda.synchronize()
        ceiling_clocks = csampler.stop()
        ceiling_ms = statistics.mean(cs[k].elapsed_time(ce[k]) for k in range(Kc))
        if dist:
            tc = torch.tensor([ceiling_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(tc, op=dist.ReduceOp.MAX)
            ceiling_ms = float(tc[0])

    # ---- a plain two-stream device copy (torch) for the same time: the HBM
    # reference point for the power the byte mix itself draws ----
    plain = None
    if args.launch_mode == "multi" and ceiling_ms is not None:
        nb = 4 << 30
        src = torch.empty(nb, dtype=torch.uint8, device=dev)
        dst = torch.empty(nb, dtype=torch.uint8, device=dev)
        src.fill_(1)
        for _ in range(3):
            dst.copy_(src)
        torch.cuda.synchronize()
        one = torch.cuda.Event(enable_timing=True)
        two = torch.cuda.Event(enable_timing=True)
        one.record(stream)
        dst.copy_(src)
        two.record(stream)
        torch.cuda.synchronize()
        Kp = max(10, int(ceiling_ms * Kc / max(one.elapsed_time(two), 1e-3)))
        psampler = ClockSampler(gpu_id)
        psampler.start()
        torch.cuda.synchronize()
        one.record(stream)
        for _ in range(Kp):
            dst.copy_(src)
        two.record(stream)
        torch.cuda.synchronize()
        pclocks = psampler.stop()
        pms = one.elapsed_time(two) / Kp
        plain = {"kernel": "torch copy_ of a 4 GiB buffer (one read and one write stream)",
                 "achieved": round(2 * nb / (pms / 1e3) / 1e9, 1), "unit": "GB/s", "launches": Kp,
                 "clocks": {k: pclocks.get(k) for k in ("sm_mhz", "power_w_median", "power_w_steady")}}
        del src, dst

    n_params = wl.numel
    value = world * n_params * K / (total_ms / 1e3) / 1e9
    abytes = algorithmic_bytes(wl)
    peak, peak_kind = measured_peaks()
    achieved = abytes / (per_launch_ms / 1e3) / 1e9 if launches_per_step == 1 else abytes / (per_launch_ms / 1e3) / 1e9
    traffic = traffic_from_profile(args.config) if launches_per_step == 1 else None

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, P, fmt, dev, dist, world, torch, fo)

    # ---- CPU oracle baseline (rank 0, N = 1) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        v, dt, n, k = time_oracle(wl, args.cpu_sample_params, 1, 1, threads, min_seconds=10.0)
        cpu = {"value": round(v, 6), "unit": "Gparams/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} params (whole 32-groups drawn from all {len(wl.tensors)} tensors), "
                         f"{k} {wl.optimizer} steps after one warm step, {threads} host threads, "
                         f"{dt:.2f} s timed"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "Gparams/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": arm_config(wl, args, world),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_kind": peak_kind, "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes_per_launch": abytes, "kernel": "fo::step_kernel"},
            "ceiling": None if ceiling_ms is None else {
                "kernel": "fo_stream_copy: the step's byte mix with the same staging, work split and "
                          "stores, no arithmetic (after the timed region)",
                "achieved": round(abytes / (ceiling_ms / 1e3) / 1e9, 1), "unit": "GB/s",
                "frac_of_peak": round(abytes / (ceiling_ms / 1e3) / 1e9 / peak, 4),
                "step_frac_of_ceiling": round(ceiling_ms / per_launch_ms, 4),
                "clocks": {k: ceiling_clocks.get(k) for k in ("sm_mhz", "power_w_median", "power_w_steady",
                                                              "power_w_max")},
                "plain_copy": plain},
            "clocks": clocks,
            "gpu_launches": K * launches_per_step,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _free_port() -> int:
    import socket

    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    port = so.getsockname()[1]
    so.close()
    return port


def run_dp(args, rank, world, local):
    """Data-parallel step of one model over `world` GPUs (strong scaling: the
    list is the same for every N).  The flat layout of the parameter list is
    cut into buckets; rank r owns the r-th slice of every bucket (its ECC,
    momentum and variance codes and scales) and holds the whole x'.  One step:
    NCCL reduce-scatter of the 16-bit gradients, the fused step of the owned
    slices, all-gather of x' in place, bucket by bucket on a communication
    stream (bit_states_b200.dp).  Rank 0 holds the synthetic gradient and the
    other ranks zeros, so the reduced gradient is rank 0's exactly, in any
    summation order.  Also timed: the steps alone and the exchange alone."""
    import datetime

    import torch
    import torch.distributed as dist

    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    else:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=300), device_id=dev)

    from bit_states_b200 import build as fobuild
    from bit_states_b200 import fo
    from bit_states_b200.dp import DataParallelStep, FlatLayout, ShardedState
    from workloads import device as wdev
    from workloads import workload

    fobuild.build()
    wdev.build()
    fo.load()
    wl = workload(args.config)
    adam = wl.optimizer == "adamw"
    layout = FlatLayout([t.numel for t in wl.tensors], world, bucket_groups=args.bucket_groups)
    st = ShardedState(layout, rank, dev, adam=adam, ecc_bits=wl.ecc_bits)
    fmt = fo.make_format(wl.w_dtype, wl.grad_dtype, wl.ecc_bits)
    # masters: the same synthetic values on every rank, encoded by the owner
    # of each group and all-gathered
    x32 = torch.zeros(layout.numel, dtype=torch.float32, device=dev)
    for ti, t in enumerate(wl.tensors):
        wdev.master_f32(wl, ti, layout.tensor_view(x32, ti))
    st.encode_from(x32, fmt, w_dtype=wl.w_dtype)
    del x32
    grads = torch.zeros(layout.numel, dtype=torch.int16, device=dev)
    if rank == 0:
        for ti in range(len(wl.tensors)):
            wdev.grad_16(wl, ti, 1, layout.tensor_view(grads, ti))
    h = wl.hparams
    dp = DataParallelStep(st, fmt=fmt, hparams=h, reduce_op="sum", grad_dtype=wl.grad_dtype,
                          w_dtype=wl.w_dtype, optimizer=wl.optimizer)
    torch.cuda.synchronize()
    dist.barrier()
    stream = torch.cuda.current_stream()

    def timed(fn, k):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        dist.barrier()
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        tt = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        return float(tt[0]) / k

    t = [0]

    def one_step():
        t[0] += 1
        dp.step(grads, t[0])

    def step_only():
        t[0] += 1
        dp.step_only(t[0], stream)

    for _ in range(args.warmup):
        one_step()
    gpu_id = "0"
    try:
        props = torch.cuda.get_device_properties(local)
        gpu_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    K = args.steps
    total_ms = timed(one_step, K)
    clocks = sampler.stop()
    fo.fo_check_errors()
    step_ms = timed(step_only, max(3, K // 2))
    comm_ms = timed(lambda: dp.exchange(grads), max(3, K // 2))
    fo.fo_check_errors()

    n_params = wl.numel
    value = n_params / (total_ms / 1e3) / 1e9
    owned = st.m_q.numel()
    per_param = algorithmic_bytes(wl) / n_params
    step_bytes = per_param * owned
    peak, peak_kind = measured_peaks()
    achieved = step_bytes / (step_ms / 1e3) / 1e9
    overlap = (step_ms + comm_ms - total_ms) / min(step_ms, comm_ms) if min(step_ms, comm_ms) > 0 else None

    # end to end through the public API: every step copies this rank's
    # gradient from pinned host memory (in pieces) and reads x' back
    PIECE = 1 << 24
    host_g = torch.empty(PIECE, dtype=torch.int16, pin_memory=True)
    host_g.copy_(grads[:PIECE].cpu() if layout.numel >= PIECE else torch.zeros(PIECE, dtype=torch.int16))
    host_w = torch.empty(PIECE, dtype=torch.int16, pin_memory=True)

    def e2e_step():
        for a in range(0, layout.numel, PIECE):
            b = min(layout.numel, a + PIECE)
            grads[a:b].copy_(host_g[:b - a], non_blocking=True)
        one_step()
        for a in range(0, layout.numel, PIECE):
            b = min(layout.numel, a + PIECE)
            host_w[:b - a].copy_(st.w[a:b], non_blocking=True)

    e2e_steps = max(1, min(args.e2e_steps, 3))
    e2e = None
    if not args.no_e2e:
        e2e_ms = timed(e2e_step, e2e_steps)
        e2e = {"value": round(n_params / (e2e_ms / 1e3) / 1e9, 3), "unit": "Gparams/s",
               "h2d_bytes_per_step": 2 * layout.numel, "d2h_bytes_per_step": 2 * layout.numel,
               "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
               "how": f"per step and rank: the rank's 16-bit gradient from a pinned host buffer to the device in "
                      f"pieces of {PIECE} elements, the data-parallel step, x' back to pinned host memory"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        v, dt, n, k = time_oracle(wl, args.cpu_sample_params, 1, 1, threads, min_seconds=10.0)
        cpu = {"value": round(v, 6), "unit": "Gparams/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} params (whole 32-groups drawn from all {len(wl.tensors)} tensors), "
                         f"{k} {wl.optimizer} steps after one warm step, {threads} host threads, {dt:.2f} s timed"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "Gparams/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(total_ms, 4), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{wl.name}: {len(wl.tensors)} tensors, {n_params} params in total, "
                                   f"{wl.optimizer} {wl.w_dtype}+ecc{wl.ecc_bits}, int8/uint8 companded states",
                       "launch": f"{len(layout.buckets)} buckets of <= {args.bucket_groups} groups; per bucket a "
                                 "fused step on this rank's slice",
                       "l2": "inputs larger than L2 (%.2f GB per step per GPU vs 126 MB)" % (step_bytes / 1e9),
                       "parallelism": f"data parallel x{world}: NCCL reduce-scatter of 16-bit gradients, fused step "
                                      f"on owned groups, in-place all-gather of x'"},
            "exchange": {"total_ms": round(total_ms, 3), "steps_only_ms": round(step_ms, 3),
                         "exchange_only_ms": round(comm_ms, 3),
                         "overlap": None if overlap is None else round(overlap, 3),
                         "bytes_per_rank": {"reduce_scatter_in": 2 * layout.numel * (world - 1) // world,
                                            "all_gather_in": 2 * layout.numel * (world - 1) // world}},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": None, "peak_kind": peak_kind,
                         "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes_per_launch": int(step_bytes / max(1, len(layout.buckets))),
                         "kernel": "fo::step_kernel (the owned slices' steps, timed without the exchange)"},
            "clocks": clocks,
            "gpu_launches": K * len(layout.buckets),
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def run_e2e(args, wl, P, fmt, dev, dist, world, torch, fo):
    """Same metric through the public API with host buffers: every step
    copies each tensor's bf16 gradient from pinned host memory and reads the
    updated downcast weights back to pinned host memory, in gradient-release
    order.  Tensors are cut at group boundaries into pieces of at most
    PIECE elements, so that the host-to-device copies, the step launches and
    the device-to-host copies of consecutive pieces overlap (a ring of stage
    buffers on the device, one stream per copy direction)."""
    from bit_states_b200.fo import TensorState

    if wl.optimizer != "adamw":
        return None
    from workloads import device as wdev

    PIECE, RING = max(32, args.e2e_piece // 32 * 32), max(2, args.e2e_ring)
    pieces = []                            # (tensor, first element, elements), release order
    for ti in list(range(len(P.numels)))[::-1]:
        n = P.numels[ti]
        for e0 in range(0, n, PIECE):
            pieces.append((ti, e0, min(PIECE, n - e0)))
    stage = [torch.empty(PIECE, dtype=torch.int16, device=dev) for _ in range(RING)]
    # host gradient: a synthetic gradient piece, the source of every piece's
    # copy (the bytes moved are the full list's)
    big = int(np.argmax(P.numels))
    tmp = torch.empty(P.numels[big], dtype=torch.int16, device=dev)
    wdev.grad_16(wl, big, 1, tmp)
    host_g = torch.empty(PIECE, dtype=torch.int16, pin_memory=True)
    host_g.copy_(tmp[:PIECE])
    del tmp
    host_w = torch.empty(PIECE, dtype=torch.int16, pin_memory=True)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    comp = torch.cuda.current_stream(dev)
    h2d = sum(P.numels) * 2
    d2h = sum(P.numels) * 2
    h = wl.hparams
    descs = []
    for ti, e0, n in pieces:
        st = P.states[ti]
        g0, g1 = e0 // 32, (e0 + n + 31) // 32
        sub = TensorState(st.w[e0:e0 + n], st.ecc[e0:e0 + n], st.m_q[e0:e0 + n], st.m_scale[g0:g1],
                          st.v_q[e0:e0 + n], st.v_scale[g0:g1])
        descs.append((sub, n))

    def one_step(t):
        hp = fo.fo_adamw_hparams(h["lr"], h["beta1"], h["beta2"], h["eps"], h["weight_decay"], t)
        done = [None] * RING
        for j, (sub, n) in enumerate(descs):
            b = j % RING
            with torch.cuda.stream(s_in):
                if done[b] is not None:
                    s_in.wait_event(done[b])
                stage[b][:n].copy_(host_g[:n], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            comp.wait_event(ev_in)
            fo.fo_adamw_step(fo.descriptors([sub], [stage[b][:n]]), 1, fmt, hp, comp)
            ev_done = torch.cuda.Event()
            ev_done.record(comp)
            done[b] = ev_done
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done)
                host_w[:n].copy_(sub.w, non_blocking=True)
        comp.wait_stream(s_out)
        comp.wait_stream(s_in)

    t0 = 10_000
    one_step(t0)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    K = args.e2e_steps
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for k in range(K):
        one_step(t0 + 1 + k)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist:
        tt = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt[0])
    value = world * sum(P.numels) * K / (ms / 1e3) / 1e9
    return {"value": round(value, 3), "unit": "Gparams/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / K, 3), "steps": K,
            "how": f"tensors cut into group-aligned pieces of <= {PIECE} params in gradient-release order; per "
                   "piece: pinned-host bf16 grad -> device (copy stream), fo_adamw_step, updated bf16 weights -> "
                   f"pinned host (copy stream); {RING} device stage buffers, copies overlapped with the steps",
            "launches_per_step": len(descs)}


if __name__ == "__main__":
    sys.exit(main())
