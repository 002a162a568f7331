#!/usr/bin/env python
"""MLA decode benchmark on B200: TFLOP/s, HBM GB/s and the roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload metric] [--impl ours|reference]

A step is one full MLA decode (main kernel + split-KV combine) of the
workload with inputs already resident in HBM.  The default workload is the
headline line: B=64 sequences, Sq=1, H=128 heads, every L=8192, d_qk=576,
d_v=512, bf16 N(0,1) seeded synthetic data; its kv (604 MB) is larger than
the 126 MB L2, so no flush is needed between steps.  Prints ONE JSON line on
rank 0.  Under torchrun (N > 1) every rank runs an independent replica (the
path has no cross-GPU exchange); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only other implementation of
this path) on a bounded sample of the same workload, on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from mla_decode_attention_11_b200 import workloads as W  # noqa: E402

METRIC = "MLA decode TFLOP/s + HBM GB/s at B=64,H=128,L=8192; fraction of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (a multi-GPU job takes as long as its
    slowest rank); x itself when dist is None (one process)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Units per second of the whole job: every rank processes units_per_rank
    (independent replicas, weak scaling) in ms milliseconds, the max over ranks."""
    return world * units_per_rank / (ms * 1e-3)


L2_BYTES = 126e6  # B200 L2 (the device's own size is read at run time where it matters)
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}  # HBM3e and dense bf16, nominal
MAX_PLAUSIBLE_FRAC = 1.2  # a roofline fraction above this means the timed kernel skipped work


def l2_note(cache_bytes: float) -> str:
    """How the timed steps relate to L2: no flush is done between steps, which
    is sound only when the cache streamed per step is larger than L2."""
    if cache_bytes > L2_BYTES:
        return "inputs larger than L2 (kv %.0f MB > 126 MB), no flush" % (cache_bytes / 1e6)
    return "kv %.0f MB fits in L2 (126 MB), no flush: steps after the first may hit L2" % (cache_bytes / 1e6)


def needs_flush(cache_bytes: float, l2_bytes: float) -> bool:
    """Flush L2 between timed decodes unless the cache streamed per decode is
    at least twice the L2 size (then a decode evicts its own inputs)."""
    return cache_bytes < 2 * l2_bytes


def flush_note(cache_bytes: float, l2_bytes: float) -> str:
    return ("kv %.0f MB < 2 x L2 (%.0f MB): L2 flushed (a %.0f MB write) before every timed decode, each decode "
            "timed by its own events" % (cache_bytes / 1e6, l2_bytes / 1e6, 2 * l2_bytes / 1e6))


def compare_rows(out_rows, lse_rows, ref_out, ref_lse) -> dict:
    """Parity of the timed run's own outputs against the oracle on the rows the
    CPU baseline computed (the tolerances of the parity tests)."""
    import numpy as np
    o = np.asarray(out_rows, dtype=np.float64).reshape(ref_out.shape)
    d = o - ref_out
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref_out), 1e-300))
    lg = np.asarray(lse_rows, dtype=np.float64).reshape(-1)
    lr = ref_lse.reshape(-1)
    fin = np.isfinite(lr)
    lse_err = float(np.abs(lg[fin] - lr[fin]).max()) if fin.any() else 0.0
    ok = bool(np.all(np.isfinite(o)) and max_abs <= 2e-2 and rel <= 5e-3 and lse_err <= 1e-3
              and np.array_equal(np.isfinite(lg), fin))
    return {"rows": int(ref_out.shape[0]), "max_abs": max_abs, "rel_l2": rel, "lse_max_abs": lse_err,
            "tolerance": "max-abs 2e-2, rel-L2 5e-3, lse 1e-3", "ok": ok}


def mma_tensor_peak(peaks: dict, e4m3_mma: bool) -> float:
    """Dense tensor peak (TFLOP/s) of a kernel's own MMA type: bf16 and f16
    MMAs run at the measured bf16 rate, E4M3 MMAs (kind::f8f6f4) at twice it
    (the nominal 4.5 / 2.25 PFLOP/s ratio).  The algorithmic flops stay the
    definition's: the E4M3 kernels' extra MMAs for their q and P terms are
    their own cost, not work of the decode."""
    return peaks["bf16_tflops"] * (2.0 if e4m3_mma else 1.0)


def roofline_point(flops: float, nbytes: float, kernel_ms: float, hbm_gbs: float, tensor_tflops: float):
    """(bound, achieved, peak, unit) of one kernel launch: HBM-bound when the
    arithmetic intensity is below the ridge of the two peaks, else tensor-bound."""
    ridge = tensor_tflops * 1e12 / (hbm_gbs * 1e9)
    if flops / nbytes < ridge:
        return "hbm", nbytes / (kernel_ms * 1e-3) / 1e9, hbm_gbs, "GB/s"
    return "tensor", flops / (kernel_ms * 1e-3) / 1e12, tensor_tflops, "TFLOP/s"


def refuse(line: dict, why: str) -> None:
    """A number that cannot be right is not printed as a result."""
    sys.stderr.write("bench.py: refusing to report this measurement: %s\n%s\n" % (why, json.dumps(line)))
    sys.exit(1)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    from mla_decode_attention_11_b200 import build as B
    h = hashlib.sha256()
    for s in B.sources():
        with open(s, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """DRAM bytes per main-kernel launch from a committed ncu summary, used only
    if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(workload)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash():
        return None, None
    return float(ent["dram_bytes_per_launch"]), ent.get("note")


def workload_desc(w: W.Workload) -> str:
    L = f"U[{w.L_lo},{w.L}]" if w.L_lo is not None else f"{w.L} (all)"
    return (f"{w.name}: B={w.B} Sq={w.Sq} H={w.H} L={L}, d_qk=576 (512 latent + 64 rope), d_v=512, "
            f"bf16 N(0,{w.sigma:g}) seed {w.seed}, scale 576^-0.5")


class ClockSampler:
    """Polls SM clock / throttle reasons through NVML during the timed region."""

    REASONS = {0x0000000000000004: "sw_power_cap", 0x0000000000000008: "hw_slowdown",
               0x0000000000000020: "sw_thermal_slowdown", 0x0000000000000040: "hw_thermal_slowdown",
               0x0000000000000080: "hw_power_brake_slowdown", 0x0000000000000001: "gpu_idle",
               0x0000000000000002: "applications_clocks_setting", 0x0000000000000100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = torch.cuda.get_device_properties(device_index).uuid
            u = str(uuid)
            if not u.startswith("GPU-"):
                u = "GPU-" + u
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(u)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.0005)

    def start(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr:
            self._stop.set()
            self._thr.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def cpu_oracle_sample(w: W.Workload, q, kv, sl, seqs, num_threads: int = 0, keep: bool = False):
    """Time the oracle, as it stands, on whole sequences `seqs` (all heads);
    with keep, also return its rows (out [n, 512], lse [n]) and their ids."""
    import numpy as np
    import oracle
    R = w.Sq * w.H
    rows = np.concatenate([np.arange(b * R, (b + 1) * R) for b in seqs]).astype(np.int64)
    t0 = time.perf_counter()
    ro, rl = oracle.mla_decode_rows(q, kv, sl, w.scale, rows, num_threads=num_threads)
    dt = time.perf_counter() - t0
    flops = sum(int(sl[b]) for b in seqs) * R * 2 * (W.D_QK + W.D_V)
    threads = num_threads if num_threads > 0 else oracle.max_threads()
    if keep:
        return flops, dt, threads, (rows, ro, rl)
    return flops, dt, threads


def run_reference(args, w: W.Workload):
    """--impl reference: the fp64 CPU oracle on a bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    q, kv, sl = W.generate(w, tail_fill=0.0)
    seqs_per_step = 1
    for i in range(args.warmup):
        cpu_oracle_sample(w, q, kv, sl, [i % w.B])
    tot_flops, tot_t, cores = 0, 0.0, 1
    for i in range(args.steps):
        f, dt, cores = cpu_oracle_sample(w, q, kv, sl, [(args.warmup + i) % w.B])
        tot_flops += f
        tot_t += dt
    value = tot_flops / tot_t / 1e12
    sample = (f"{seqs_per_step} whole sequence per step ({w.Sq * w.H} query rows x L={w.L}) of the "
              f"{w.B}-sequence workload, {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "parallelism": "host cores (OpenMP)", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w: W.Workload):
    from mla_decode_attention_11_b200 import binding as M

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    q, kv, sl = W.generate(w, tail_fill=0.0)
    qd, kvd, sld = q.to(dev), kv.to(dev), sl.to(dev)
    if args.batch_invariant is not None:
        plan = M.mla_decode_plan_batch_invariant(w.B, w.Sq, w.H, w.L, device=local, split_tiles=args.batch_invariant)
    else:
        plan = M.mla_decode_plan(w.B, w.Sq, w.H, w.L, device=local)
    ws = M.alloc_workspace(plan, device=dev)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.empty((w.B, w.Sq, w.H, W.D_V), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Sq, w.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    # --sinks: the same decode with per-head attention-sink logits (seeded)
    sinks_d = None
    if args.sinks:
        gs = torch.Generator().manual_seed(w.seed + 17)
        sinks_d = (torch.randn(w.H, generator=gs) * 2.0).to(dev)

    def step():
        if sinks_d is None:
            M.mla_decode_run(plan, qd, kvd, sld, w.scale, out, lse, ws, stream=stream)
        else:
            M.mla_decode_run_sinks(plan, qd, kvd, sld, w.scale, sinks_d, out, lse, ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    M.mla_decode_check(plan, ws, stream=stream)

    # Inputs larger than twice L2 are streamed as they are; a smaller cache gets
    # an L2 flush (a write of twice the L2 size) before every timed decode, and
    # each decode is then timed by its own pair of events.
    l2_bytes = float(torch.cuda.get_device_properties(dev).L2_cache_size)
    cache_bytes = kv.numel() * 2
    flush_buf = torch.empty(int(2 * l2_bytes), dtype=torch.uint8, device=dev) \
        if needs_flush(cache_bytes, l2_bytes) else None

    # Without a flush the K timed decodes are launched as one CUDA graph
    # (captured, not run, here), so that the host-side cost of a call (~25 us
    # through Python) does not leave the GPU idle between the launches of small
    # workloads.
    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(n):
                    fn()
        return g

    def flushed_ms(fn, n):
        """Mean device time of fn over n calls, L2 flushed before each; a GPU
        sleep in front lets the host enqueue all of it before it starts."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        with torch.cuda.stream(stream):
            torch.cuda._sleep(int(20e6 + 2e6 * n))
            for i in range(n):
                flush_buf.fill_(i & 0xFF)
                evs[i][0].record(stream)
                fn()
                evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in evs) / n

    g_steps = capture(step, args.steps) if flush_buf is None else None
    torch.cuda.synchronize(dev)

    # ---- timed region: K full steps
    clocks = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    if flush_buf is None:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):  # a graph replays on the current stream
            e0.record(stream)
            g_steps.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        t_ms = e0.elapsed_time(e1) / args.steps
    else:
        t_ms = flushed_ms(step, args.steps)
    clk = clocks.stop()
    if dist:
        dist.barrier()
    M.mla_decode_check(plan, ws, stream=stream)
    out_timed, lse_timed = out.cpu(), lse.cpu()  # the timed run's own result, checked below
    t_ms = max_over_ranks(t_ms, dist, dev)

    # ---- per-kernel breakdown: the same launches, each kernel alone (phase 1 =
    # main kernel, phase 2 = split-KV combine), back to back in a graph, or one
    # by one after a flush as above
    n_brk = max(3, min(args.steps, 50))

    def phase_ms(phase):
        fn = lambda: M.mla_decode_run_phase(plan, qd, kvd, sld, w.scale, out, lse, ws, phase, stream=stream)
        if flush_buf is not None:
            return flushed_ms(fn, n_brk)
        g = capture(fn, n_brk)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / n_brk

    main_avg = phase_ms(1)
    comb_avg = phase_ms(2)
    del g_steps
    M.mla_decode_check(plan, ws, stream=stream)

    # ---- end to end through the public API with host buffers
    e2e_steps = max(1, min(args.steps, 5))
    qh, kvh, slh = q.pin_memory(), kv.pin_memory(), sl.pin_memory()
    outh = torch.empty((w.B, w.Sq, w.H, W.D_V), dtype=torch.bfloat16).pin_memory()
    lseh = torch.empty((w.B, w.Sq, w.H), dtype=torch.float32).pin_memory()
    bufs = {}
    with torch.cuda.stream(stream):  # copies and launches on the bench stream
        M.mla_decode_host(qh, kvh, slh, w.scale, plan, ws, dev_bufs=bufs, out_host=outh, lse_host=lseh)
        torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            M.mla_decode_host(qh, kvh, slh, w.scale, plan, ws, dev_bufs=bufs, out_host=outh, lse_host=lseh)
        f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = f0.elapsed_time(f1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    h2d = q.numel() * 2 + kv.numel() * 2 + sl.numel() * 4
    d2h = outh.numel() * 2 + lseh.numel() * 4
    M.mla_decode_check(plan, ws, stream=stream)

    flops = w.algorithmic_flops(sl)
    nbytes = w.algorithmic_bytes(sl)
    peaks, peak_src = load_peaks()
    value = whole_job_rate(world, flops, t_ms) / 1e12
    hbm_gbs = whole_job_rate(world, nbytes, t_ms) / 1e9
    bound, achieved, peak, unit = roofline_point(flops, nbytes, main_avg, peaks["hbm_gbs"],
                                                 mma_tensor_peak(peaks, e4m3_mma=False))
    spec = SPEC_PEAKS["hbm_gbs"] if bound == "hbm" else SPEC_PEAKS["bf16_tflops"]
    roof_time_ms = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12)) * 1e3
    # the record was taken with the default plan; a batch-invariant plan moves other bytes
    traffic, traffic_note = load_traffic(w.name) if not plan.split_tiles else (None, None)

    cpu_base = None
    check = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on the whole workload once (~4 s on 16 host cores for the
        # headline line, or a bounded number of sequences of larger ones); its
        # rows double as the check of the timed run's own outputs
        R = w.Sq * w.H
        per_seq = float(sl.to(torch.float64).mean()) * R * 2 * (W.D_QK + W.D_V)
        n_seq = max(1, min(w.B, int(4e11 / per_seq)))  # 0.4 TFLOP of fp64 work at most (~10 s)
        seqs = list(range(n_seq))
        f_cpu, dt_cpu, cores, (rows, ro, rl) = cpu_oracle_sample(w, q, kv, sl, seqs, keep=True)
        cpu_base = {"value": f_cpu / dt_cpu / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                    "sample": f"{len(seqs)} of {w.B} sequences, all {R} query rows, "
                              f"{dt_cpu:.1f} s of fp64 CPU work"}
        if w.name in ("tiny", "dsv3"):
            # per-core context: the same oracle on one host thread, one sequence
            f1, dt1, _ = cpu_oracle_sample(w, q, kv, sl, [0], num_threads=1)
            cpu_base["single_core"] = {"value": f1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                                       "sample": f"1 sequence, all {R} query rows, {dt1:.2f} s"}
        check = compare_rows(out_timed.reshape(-1, W.D_V)[rows].to(torch.float64).numpy(),
                             lse_timed.reshape(-1)[rows].to(torch.float64).numpy(), ro, rl)
        if args.sinks:  # the oracle rows above have no sinks; the sink path is checked by the tests
            check = {"skipped": "sink decode: the CPU-baseline rows have no sinks"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_desc(w) + (" + per-head attention sinks" if args.sinks else "")
                       + (f" + batch-invariant plan ({plan.split_tiles}-tile chunks)" if plan.split_tiles else ""),
                       "global_batch": w.B * world, "seq_len": w.L,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "kernel": {1: "transposed", 2: "pair"}.get(plan.kernel, str(plan.kernel)),
                       "group_rows": plan.group_rows, "partitions": plan.num_partitions,
                       "l2": flush_note(cache_bytes, l2_bytes) if flush_buf is not None else l2_note(cache_bytes)},
            "hbm_gbs": hbm_gbs,
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else peak_src,
                         "spec_peak": spec, "frac_of_spec": achieved / spec,
                         "kernel": "mla_decode_transposed_kernel" if plan.kernel == 1 else "mla_decode_pair_kernel",
                         "kernel_ms": main_avg, "combine_ms": comb_avg,
                         "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                         "tensor_tflops": flops / (main_avg * 1e-3) / 1e12,
                         "tensor_frac": flops / (main_avg * 1e-3) / 1e12 / peaks["bf16_tflops"],
                         "step_roofline_frac": roof_time_ms / t_ms, "traffic_note": traffic_note},
            "e2e": {"value": whole_job_rate(world, flops, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": 2 * args.steps,
            "clocks": clk,
            "cpu_baseline": cpu_base,
            "output_check": check,
        }
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        frac = achieved / peak
        if not (0.0 < frac <= MAX_PLAUSIBLE_FRAC):
            refuse(line, f"roofline fraction {frac:.3f} is outside (0, {MAX_PLAUSIBLE_FRAC}]")
        if check is not None and check.get("ok") is False:
            refuse(line, "the timed run's outputs do not match the oracle")
        print(json.dumps(line), flush=True)


def run_mha(args, w: W.MhaWorkload):
    """MHA decode (the second workload on the same skeleton): same timing
    rules as run_ours, one GPU, no reference arm."""
    from mla_decode_attention_11_b200 import binding as M
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    q, k, v, sl = W.generate_mha(w, tail_fill=0.0)
    qd, kd, vd, sld = q.to(dev), k.to(dev), v.to(dev), sl.to(dev)
    plan = M.mha_decode_plan(w.B, w.Sq, w.H, w.Hkv, w.L, device=0)
    ws = M.alloc_workspace(plan, device=dev)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.empty((w.B, w.Sq, w.H, W.MHA_D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Sq, w.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    def step():
        M.mha_decode_run(plan, qd, kd, vd, sld, w.scale, out, lse, ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    M.mla_decode_check(plan, ws, stream=stream)

    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(n):
                    fn()
        return g

    def replay_ms(g, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / n

    g_steps = capture(step, args.steps)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(0)
    clocks.start()
    t_ms = replay_ms(g_steps, args.steps)
    clk = clocks.stop()
    del g_steps
    n_brk = max(3, min(args.steps, 50))
    main_ms = replay_ms(capture(lambda: M.mha_decode_run_phase(plan, qd, kd, vd, sld, w.scale, out, lse, ws, 1,
                                                               stream=stream), n_brk), n_brk)
    comb_ms = replay_ms(capture(lambda: M.mha_decode_run_phase(plan, qd, kd, vd, sld, w.scale, out, lse, ws, 2,
                                                               stream=stream), n_brk), n_brk)
    M.mla_decode_check(plan, ws, stream=stream)
    # end to end: host buffers in, host buffers out, copies inside the timed region
    qh, kh, vh, slh = q.pin_memory(), k.pin_memory(), v.pin_memory(), sl.pin_memory()
    outh = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    lseh = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            sld.copy_(slh, non_blocking=True)
            step()
            outh.copy_(out, non_blocking=True)
            lseh.copy_(lse, non_blocking=True)
        f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = f0.elapsed_time(f1) / e2e_steps
    flops, nbytes = w.algorithmic_flops(sl), w.algorithmic_bytes(sl)
    peaks, peak_src = load_peaks()
    cpu_base = None
    if not args.no_cpu_baseline:
        import oracle
        nb = min(w.B, 8)
        t0 = time.perf_counter()
        oracle.mha_decode(q[:nb], k[:nb], v[:nb], sl[:nb], w.scale)
        dt = time.perf_counter() - t0
        f_cpu = int(sl[:nb].to(torch.int64).sum()) * w.Sq * w.H * 2 * (2 * W.MHA_D)
        cpu_base = {"value": f_cpu / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
                    "sample": f"{nb} of {w.B} sequences, all query rows, {dt:.1f} s of fp64 CPU work"}
    achieved = nbytes / (main_ms * 1e-3) / 1e9
    traffic, traffic_note = load_traffic(w.name)
    line = {
        "metric": f"MHA decode TFLOP/s + HBM GB/s at B={w.B},H={w.H},Hkv={w.Hkv},d=128,L={w.L}; fraction of roofline",
        "value": flops / (t_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} Sq={w.Sq} H={w.H} Hkv={w.Hkv} L={w.L}, d=128, bf16 "
                               f"N(0,{w.sigma:g}) seed {w.seed}, scale 128^-0.5",
                   "global_batch": w.B, "seq_len": w.L, "parallelism": "single GPU", "kernel": "transposed (MHA)",
                   "group_rows": plan.group_rows, "partitions": plan.num_partitions,
                   "l2": l2_note(k.numel() * 2 + v.numel() * 2)},
        "hbm_gbs": nbytes / (t_ms * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                     "traffic_note": traffic_note,
                     "kernel": "mla_decode_transposed_kernel<G, MhaShape>", "kernel_ms": main_ms,
                     "combine_ms": comb_ms, "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                     "step_roofline_frac": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3 / t_ms},
        "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": q.numel() * 2 + k.numel() * 2 + v.numel() * 2 + sl.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 2 + lse.numel() * 4, "ms_per_step": e2e_ms},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu_base,
    }
    print(json.dumps(line), flush=True)


def run_fp8(args, w: W.Workload):
    """MLA decode over an FP8 (E4M3) latent cache: same timing rules as
    run_ours (graph replay, per-kernel graphs, host-buffer e2e), one GPU."""
    from mla_decode_attention_11_b200 import binding as M
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    q, codes, ks, sl = W.generate_fp8(w)
    qd, cd, sld = q.to(dev), codes.to(dev), sl.to(dev)
    kernel = {"default": 0, "widen": M.MLA_KERNEL_FP8, "operands": M.MLA_KERNEL_FP8_MMA,
              "pair": M.MLA_KERNEL_FP8_PAIR}[args.fp8_kernel]
    plan = M.mla_decode_plan_fp8(w.B, w.Sq, w.H, w.L, device=0, kernel=kernel)
    ws = M.alloc_workspace(plan, device=dev)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.empty((w.B, w.Sq, w.H, W.D_V), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Sq, w.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    def step():
        M.mla_decode_run_fp8(plan, qd, cd, ks, sld, w.scale, out, lse, ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    M.mla_decode_check(plan, ws, stream=stream)

    # As for the bf16 cache: a cache smaller than twice L2 gets an L2 flush
    # before every timed decode, each decode timed by its own events; a larger
    # one streams as it is, the decodes replayed as one CUDA graph.
    l2_bytes = float(torch.cuda.get_device_properties(dev).L2_cache_size)
    cache_bytes = float(codes.numel())
    flush_buf = torch.empty(int(2 * l2_bytes), dtype=torch.uint8, device=dev) \
        if needs_flush(cache_bytes, l2_bytes) else None

    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(n):
                    fn()
        return g

    def timed_ms(fn, n):
        if flush_buf is not None:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            with torch.cuda.stream(stream):
                torch.cuda._sleep(int(20e6 + 2e6 * n))
                for i in range(n):
                    flush_buf.fill_(i & 0xFF)
                    evs[i][0].record(stream)
                    fn()
                    evs[i][1].record(stream)
            torch.cuda.synchronize(dev)
            return sum(a.elapsed_time(b) for a, b in evs) / n
        g = capture(fn, n)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        del g
        return a.elapsed_time(b) / n

    if flush_buf is None:
        g_steps = capture(step, args.steps)
        torch.cuda.synchronize(dev)
    clocks = ClockSampler(0)
    clocks.start()
    if flush_buf is None:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g_steps.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        t_ms = a.elapsed_time(b) / args.steps
        del g_steps
    else:
        t_ms = timed_ms(step, args.steps)
    clk = clocks.stop()
    n_brk = max(3, min(args.steps, 50))
    main_ms = timed_ms(lambda: M.mla_decode_run_fp8_phase(plan, qd, cd, ks, sld, w.scale, out, lse, ws, 1,
                                                          stream=stream), n_brk)
    comb_ms = timed_ms(lambda: M.mla_decode_run_fp8_phase(plan, qd, cd, ks, sld, w.scale, out, lse, ws, 2,
                                                          stream=stream), n_brk)
    M.mla_decode_check(plan, ws, stream=stream)
    # end to end: host buffers in, host buffers out, copies inside the timed region
    qh, ch, slh = q.pin_memory(), codes.pin_memory(), sl.pin_memory()
    outh = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    lseh = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            qd.copy_(qh, non_blocking=True)
            cd.copy_(ch, non_blocking=True)
            sld.copy_(slh, non_blocking=True)
            step()
            outh.copy_(out, non_blocking=True)
            lseh.copy_(lse, non_blocking=True)
        f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = f0.elapsed_time(f1) / e2e_steps
    M.mla_decode_check(plan, ws, stream=stream)
    flops, nbytes = w.algorithmic_flops(sl), w.algorithmic_bytes_fp8(sl)
    peaks, peak_src = load_peaks()
    cpu_base = None
    check = None
    if not args.no_cpu_baseline:
        import numpy as np
        import oracle
        R = w.Sq * w.H
        b0 = 0
        rows = np.arange(b0 * R, (b0 + 1) * R, dtype=np.int64)
        t0 = time.perf_counter()
        ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale, row_ids=rows)
        dt = time.perf_counter() - t0
        check = compare_rows(out.reshape(-1, W.D_V)[torch.from_numpy(rows)].cpu().to(torch.float64).numpy(),
                             lse.reshape(-1)[torch.from_numpy(rows)].cpu().to(torch.float64).numpy(),
                             np.asarray(ro, dtype=np.float64).reshape(len(rows), W.D_V),
                             np.asarray(rl, dtype=np.float64).reshape(-1))
        f_cpu = int(sl[b0]) * R * 2 * (W.D_QK + W.D_V)
        cpu_base = {"value": f_cpu / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
                    "sample": f"1 of {w.B} sequences, all {R} query rows, {dt:.1f} s of fp64 CPU work"}
    e4m3_mma = plan.kernel in (M.MLA_KERNEL_FP8_PAIR, M.MLA_KERNEL_FP8_MMA)
    tensor_peak = mma_tensor_peak(peaks, e4m3_mma)
    bound, achieved, peak, unit = roofline_point(flops, nbytes, main_ms, peaks["hbm_gbs"], tensor_peak)
    fp8_kernel_label, fp8_kernel_name, traffic_key = {
        M.MLA_KERNEL_FP8_PAIR: ("FP8 operands on a CTA pair (kind::f8f6f4)", "mla_decode_pair_fp8_kernel",
                                w.name + "_fp8"),
        M.MLA_KERNEL_FP8_MMA: ("FP8 operands (kind::f8f6f4)", "mla_decode_fp8mma_kernel<G>", w.name + "_fp8mma"),
        M.MLA_KERNEL_FP8: ("transposed (FP8)", "mla_decode_transposed_kernel<G, MlaFp8Shape>", w.name + "_fp8widen"),
    }[plan.kernel]
    if plan.kernel == M.MLA_KERNEL_FP8_MMA and plan.kernel == M.mla_decode_plan_fp8(w.B, w.Sq, w.H, w.L, device=-1).kernel:
        traffic_key = w.name + "_fp8"  # the plan's default kernel for this shape
    traffic, traffic_note = load_traffic(traffic_key)
    line = {
        "metric": METRIC + " (FP8 latent cache)",
        "value": flops / (t_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 cache, f16 MMA" if plan.kernel == M.MLA_KERNEL_FP8 else "e4m3 cache, e4m3 MMA",
        "data": "synthetic",
        "config": {"workload": workload_desc(w) + f"; cache quantised to E4M3, kv_scale = amax/448 = {ks:.6g}",
                   "global_batch": w.B, "seq_len": w.L, "parallelism": "single GPU",
                   "kernel": fp8_kernel_label,
                   "group_rows": plan.group_rows, "partitions": plan.num_partitions,
                   "l2": flush_note(cache_bytes, l2_bytes) if flush_buf is not None else l2_note(cache_bytes)},
        "hbm_gbs": nbytes / (t_ms * 1e-3) / 1e9,
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                     "traffic_note": traffic_note,
                     "kernel": fp8_kernel_name, "kernel_ms": main_ms,
                     "combine_ms": comb_ms, "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                     "hbm_frac": nbytes / (main_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "tensor_frac": flops / (main_ms * 1e-3) / 1e12 / tensor_peak,
                     "tensor_peak_tflops": tensor_peak,
                     "tensor_peak_note": ("E4M3 MMAs: twice the bf16 figure (nominal 4.5 / 2.25 PFLOP/s)"
                                          if e4m3_mma else "f16 MMAs: the bf16 figure"),
                     "step_roofline_frac": max(nbytes / (peaks["hbm_gbs"] * 1e9),
                                               flops / (tensor_peak * 1e12)) * 1e3 / t_ms},
        "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": q.numel() * 2 + codes.numel() + sl.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 2 + lse.numel() * 4, "ms_per_step": e2e_ms},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu_base,
        "output_check": check,
    }
    frac = achieved / peak
    if not (0.0 < frac <= MAX_PLAUSIBLE_FRAC):
        refuse(line, f"roofline fraction {frac:.3f} is outside (0, {MAX_PLAUSIBLE_FRAC}]")
    if check is not None and check.get("ok") is False:
        refuse(line, "the timed run's outputs do not match the oracle")
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="metric", choices=sorted(W.WORKLOADS) + sorted(W.MHA_WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch-invariant", type=int, default=None, metavar="SPLIT_TILES",
                    help="use the batch-invariant plan, sequences cut every SPLIT_TILES KV tiles (0 = default)")
    ap.add_argument("--sinks", action="store_true",
                    help="time the attention-sink entry point (per-head sink logits) on the same workload")
    ap.add_argument("--fp8", action="store_true",
                    help="the same MLA workload over an FP8 (E4M3) latent cache (mla_decode_run_fp8)")
    ap.add_argument("--fp8-kernel", choices=["default", "pair", "operands", "widen"], default="default",
                    help="FP8 cache kernel: the plan's default, the CTA-pair operand kernel (Sq*H % 128 == 0), "
                         "the transposed operand kernel, or the widening kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.workload in W.MHA_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the MLA workloads"}))
            return
        run_mha(args, W.MHA_WORKLOADS[args.workload])
        return
    w = W.WORKLOADS[args.workload]
    if args.fp8:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the bf16 cache"}))
            return
        run_fp8(args, w)
        return
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
