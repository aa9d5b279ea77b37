"""Benchmark of one DSpark round (draft -> schedule -> verify) on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen3] [--impl reference]

A step is one round over the qwen3-shaped workload (B=64 requests, K=8 draft
positions, V=151,936, rank-256 bf16 Markov factors), inputs resident in HBM.
L2 is flushed (512 MB write, untimed) before every timed round, as a target
forward pass would between rounds; each round is timed with CUDA events on
its stream and the per-kernel stages with events around each library call.
Under torchrun every rank runs an independent replica (the path has no
exchange step; weak scaling) and the time is the max over ranks.

--impl reference times the CPU oracle (oracle/, fp64 numpy) on the host on a
bounded sample of the same workload (a few requests per round, scaled to the
full batch); it is the baseline arm, not a GPU implementation.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the measured copy peak is the roofline's denominator)
sys.path.insert(0, ROOT)

import synth  # noqa: E402

HBM_FALLBACK_GBS = 6650.0


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": HBM_FALLBACK_GBS, "source": "fallback"}


def l2_read_gbs(stream, mb: int = 32, passes: int = 64, reps: int = 5):
    """Read bandwidth from L2 in GB/s: the probe library (libdspark_probe.so)
    reads an L2-resident buffer of `mb` MB `passes` times with L2-only 16-byte
    loads; the median of `reps` timed launches on `stream`, after two untimed
    ones that also make the buffer resident. None when the probe is missing or
    fails (the bench line then carries no L2 fraction)."""
    try:
        import ctypes
        import torch
        lib = ctypes.CDLL(os.path.join(ROOT, "speculative_decoding_semi_b200", "libdspark_probe.so"))
        lib.dspark_probe_sink_words.restype = ctypes.c_size_t
        lib.dspark_probe_l2_read.restype = ctypes.c_int
        lib.dspark_probe_l2_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p,
                                             ctypes.c_size_t, ctypes.c_void_p]
        words = int(lib.dspark_probe_sink_words())
        nbytes = mb * 1024 * 1024
        buf = torch.ones(nbytes // 4, dtype=torch.float32, device="cuda")
        sink = torch.empty(max(words, 1), dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        times = []
        for k in range(reps + 2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            st = lib.dspark_probe_l2_read(ctypes.c_void_p(buf.data_ptr()), nbytes, passes,
                                          ctypes.c_void_p(sink.data_ptr()), words,
                                          ctypes.c_void_p(stream.cuda_stream))
            e1.record(stream)
            if st != 0:
                return None
            e1.synchronize()
            if k >= 2:
                times.append(e0.elapsed_time(e1))
        return nbytes * passes / (statistics.median(times) * 1e-3) / 1e9
    except Exception:
        return None


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of x over all ranks of the process group (x itself when
    there is one rank): every multi-GPU time is the slowest rank's."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, slowest_ms: float) -> float:
    """Units all ranks processed per second over the slowest rank's time
    (replicas: every rank runs the same number of units)."""
    return units_per_rank * world / (slowest_ms / 1000.0)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    # 0.5 ms: a short timed region (20 rounds at qwen3 are ~10 ms on the GPU)
    # still gets ten or more samples; the sampler is a host thread, and the
    # rounds are timed by CUDA events, so it does not enter the measurement
    def __init__(self, index: int, period: float = 0.0005):
        self.samples, self.reasons, self.period = [], set(), period
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                mask = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_rate(inp: dict, seconds: float, n_req: int = 4):
    """Rounds/s of the oracle from rounds on n_req requests, scaled to the batch."""
    import oracle
    B = inp["base"].shape[0]
    rounds, spent = 0, 0.0
    t_start = time.perf_counter()
    while spent < seconds and rounds < 64:
        reqs = (np.arange(n_req) + rounds * n_req) % B
        t0 = time.perf_counter()
        oracle.run_round(inp, requests=reqs)
        spent += time.perf_counter() - t0
        rounds += 1
        if time.perf_counter() - t_start > 2 * seconds:
            break
    return 1.0 / (spent / rounds * (B / n_req)), rounds, spent


def cpu_baseline(inp: dict, seconds: float = 15.0, single_thread_seconds: float = 0.0) -> dict:
    """The oracle as it stands, on host cores, on a bounded sample of requests
    (numpy's own thread pool over the host cores; with single_thread_seconds,
    also one thread)."""
    try:
        import threadpoolctl
        cores = max((i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()), default=1)
    except Exception:
        threadpoolctl = None
        cores = os.cpu_count() or 1
    B = inp["base"].shape[0]
    n_req = 4
    value, rounds, spent = _oracle_rate(inp, seconds, n_req)
    out = {"value": value, "unit": "rounds/s", "cores": int(cores), "kind": "oracle",
           "extrapolated": True, "host_cpus": os.cpu_count(), "cpu_model": cpu_model(),
           "sample": f"{rounds} oracle rounds of {n_req} of {B} requests each (draft+verify per request, "
                     f"schedule on the full batch), scaled by {B}/{n_req}; {spent:.1f} s of CPU work"}
    if single_thread_seconds > 0 and threadpoolctl is not None:
        with threadpoolctl.threadpool_limits(limits=1):
            v1, r1, s1 = _oracle_rate(inp, single_thread_seconds, n_req)
        out["single_thread"] = {"value": v1, "unit": "rounds/s", "cores": 1,
                                "sample": f"{r1} rounds of {n_req} requests, scaled; {s1:.1f} s"}
    return out


def source_digest() -> str:
    """sha256 over the library's CUDA sources: a recorded DRAM traffic figure is
    only reported while the kernels are the ones it was measured on."""
    h = hashlib.sha256()
    src = os.path.join(ROOT, "speculative_decoding_semi_b200", "csrc")
    for name in sorted(os.listdir(src)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(src, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def measured_traffic(workload: str) -> dict:
    """DRAM bytes (read + write) per launch of each kernel, from the ncu capture
    recorded in profiles/traffic.json, or {} when the sources have changed."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        tj = json.load(f)
    if tj.get("workload") != workload or tj.get("source_sha256") != source_digest():
        return {}
    return {k: v for k, v in tj.get("dram_bytes_per_launch", {}).items()}


def draft_bytes(B, K, V, r, factor_bytes, variant="a"):
    """Algorithmic HBM bytes of one draft launch: base read + z write (variant
    A) or the operand rows (variant B) + Bf once + gathered A rows +
    per-position outputs."""
    out = B * K * V * 4 if variant == "a" else B * K * r * 2
    return B * K * V * 4 + out + r * V * factor_bytes + B * K * r * factor_bytes + B * K * (4 + 4 + 8 + 4)


def verify_bytes(V, K, verify_len, accepted, r=256, factor_bytes=2, variant="a"):
    """Algorithmic HBM bytes of one verify call: every target row 0..L_b once,
    plus, for each rejected request, the z row (variant A) or the base row,
    with Bf once and the operand rows, to recompute it (variant B)."""
    rows = int((verify_len + 1).sum())
    rejected = int((accepted < verify_len).sum())
    extra = 0 if variant == "a" or rejected == 0 else r * V * factor_bytes + rejected * r * 2
    return rows * V * 4 + rejected * V * 4 + extra


def round_variant(choice: str, B: int) -> str:
    """Variant A stores z; variant B recomputes the rejected rows in verify.
    B measured faster from B = 128 on (the z write grows with B; the
    recompute's pass over Bf does not), A below that."""
    if choice != "auto":
        return choice
    return "b" if B >= 128 else "a"


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = synth.workload(args.workload)
    inp = synth.make_round(w)
    for _ in range(args.warmup):
        cpu_baseline(inp, seconds=0.5)
    t0 = time.perf_counter()
    cb = None
    vals = []
    for _ in range(args.steps):
        cb = cpu_baseline(inp, seconds=max(2.0, 20.0 / max(1, args.steps)))
        vals.append(cb["value"])
    value = statistics.median(vals)
    cb["value"] = value
    line = {"impl": "reference", "metric": "draft+schedule+verify rounds/sec", "value": value,
            "unit": "rounds/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 / value,
            "ms_per_step_extrapolated": "oracle time on a sample of 4 requests per round, scaled to the batch; "
                                        "not a measured time of a whole round",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": config_of(w), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "rounds/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": time.perf_counter() - t0}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": f"{w.name}: B={w.B} K={w.K} V={w.V} r={w.r} {w.factor_dtype} factors, fp32 logits",
            "B": w.B, "K": w.K, "V": w.V, "r": w.r, "seed": w.seed,
            "l2": "flushed by a 512 MB write before every timed round (untimed)",
            "parallelism": "replicas (one independent round per GPU)"}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from speculative_decoding_semi_b200 import dspark_read_device_error
    from speculative_decoding_semi_b200 import round as rnd

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = synth.workload(args.workload)
    inp = synth.make_round(w, seed=w.seed + rank)
    B, K, V, r = w.B, w.K, w.V, w.r
    d = rnd.to_device(inp)
    variant = round_variant(args.variant, B)
    bufs = rnd.RoundBuffers(B, K, V, r, variant=variant)
    stream = torch.cuda.Stream()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    # draft, schedule, verify (plan, main), and variant B's residual kernel
    launches_per_round = 1 + 1 + 2 + (1 if variant == "b" else 0)

    def one_round(ev=None):
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
            if ev:
                ev[0].record(stream)
            rnd.draft(d, bufs, stream)
            if ev:
                ev[1].record(stream)
            rnd.schedule(d, bufs, stream)
            if ev:
                ev[2].record(stream)
            rnd.verify(d, bufs, stream=stream)
            if ev:
                ev[3].record(stream)

    for _ in range(max(3, args.warmup)):
        one_round()
    torch.cuda.synchronize()
    st, detail = dspark_read_device_error(bufs.workspace, stream)
    if st != 0:
        raise RuntimeError(f"device error {st} detail {detail:#x} during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for k in range(args.steps):
            one_round(evs[k])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st, detail = dspark_read_device_error(bufs.workspace, stream)
    if st != 0:
        raise RuntimeError(f"device error {st} detail {detail:#x} in the timed region")
    t_draft = [e[0].elapsed_time(e[1]) for e in evs]
    t_sched = [e[1].elapsed_time(e[2]) for e in evs]
    t_ver = [e[2].elapsed_time(e[3]) for e in evs]
    t_round = [a + b + c for a, b, c in zip(t_draft, t_sched, t_ver)]
    total_ms = max_over_ranks(sum(t_round), world, device="cuda")
    value = whole_job_rate(args.steps, world, total_ms)

    L = bufs.verify_len.cpu().numpy()
    acc = bufs.accepted.cpu().numpy()
    n_out = bufs.n_out.cpu().numpy()
    peaks = measured_peaks()
    fb = 2 if w.factor_dtype == "bf16" else 4
    dbytes = draft_bytes(B, K, V, r, fb, variant)
    vbytes = verify_bytes(V, K, L, acc, r, fb, variant)
    med = statistics.median
    draft_gbs = dbytes / (med(t_draft) * 1e-3) / 1e9
    verify_gbs = vbytes / (med(t_ver) * 1e-3) / 1e9
    round_gbs = (dbytes + vbytes) / (med(t_round) * 1e-3) / 1e9
    # the draft's floor if verify recomputed the rejected z rows instead of
    # reading them back (z never written): base read + Bf once + the rest
    dbytes_b = draft_bytes(B, K, V, r, fb, "b")

    # end to end through the public API with host buffers: copy this round's
    # inputs from pinned host memory, run the round, read the result back
    e2e = None
    if not args.no_e2e:
        host = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).pin_memory()
                for k in ("base", "target", "anchor", "u_draft", "u_accept", "u_resample", "conf")}
        out_host = torch.empty(B * (K + 1) + B, dtype=torch.int32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = out_host.numel() * 4
        e2e_steps = max(2, min(args.steps, 10))
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(e2e_steps):
                for k2, t in host.items():
                    dst = d[k2].view(-1) if k2 != "target" else d[k2].view(-1)
                    dst.copy_(t.view(-1), non_blocking=True)
                rnd.run_round(d, bufs, stream)
                out_host[: B * (K + 1)].copy_(bufs.out_tokens.view(-1), non_blocking=True)
                out_host[B * (K + 1):].copy_(bufs.n_out.view(-1), non_blocking=True)
            ev1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world, device="cuda")
        e2e = {"value": whole_job_rate(e2e_steps, world, e2e_ms), "unit": "rounds/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "note": "Markov factors are model weights kept resident; per-round logits, confidences "
                       "and uniforms are copied in, emitted tokens copied out"}

    # the draft reads Bf once per position; with few requests per position
    # those reads come from L2, so their rate is also set against L2's
    l2_gbs = l2_read_gbs(stream)
    bf_reads = K * r * V * fb
    bf_gbs = bf_reads / (med(t_draft) * 1e-3) / 1e9
    roofline_l2 = None
    if l2_gbs:
        roofline_l2 = {"bound": "l2", "kernel": "dspark_markov_draft" + ("_b" if variant == "b" else ""),
                       "achieved": bf_gbs, "peak": l2_gbs, "unit": "GB/s", "frac": bf_gbs / l2_gbs,
                       "bytes": bf_reads,
                       "note": "Bf [r,V] read at each of the K positions, against the L2 read bandwidth "
                               "measured in this run (32 MB resident buffer, L2-only 16-byte loads)"}

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(inp, seconds=args.cpu_seconds, single_thread_seconds=min(5.0, args.cpu_seconds / 3))

    traffic = measured_traffic(w.name)
    line = {
        "metric": "draft+schedule+verify rounds/sec", "value": value, "unit": "rounds/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "dtype_detail": "fp32 logits, bf16 Markov factors with fp32 accumulation, fp64 vocabulary sums",
        "data": "synthetic", "config": dict(config_of(w), variant=variant),
        "tokens_per_s": value * float(n_out.sum()),
        "stages_ms_median": {"draft": med(t_draft), "schedule": med(t_sched), "verify": med(t_ver)},
        "draft_us_per_position": 1000.0 * med(t_draft) / K,
        "round_ms": {"median": med(t_round), "p10": float(np.percentile(t_round, 10)),
                     "p90": float(np.percentile(t_round, 90))},
        "roofline": {"bound": "hbm", "kernel": "dspark_markov_draft" + ("_b" if variant == "b" else ""),
                     "achieved": draft_gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": draft_gbs / peaks["hbm_gbs"],
                     "traffic": traffic.get("draft_tc_kernel") if variant == "a" else None,
                     "algorithmic_bytes": dbytes,
                     "peak_source": peaks["source"], "frac_nominal": draft_gbs / NOMINAL_HBM_GBS,
                     "frac_design_b_floor": dbytes_b / (med(t_draft) * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "roofline_verify": {"bound": "hbm", "achieved": verify_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": verify_gbs / peaks["hbm_gbs"],
                            "traffic": traffic.get("verify_kernel") if variant == "a" else None,
                            "algorithmic_bytes": vbytes, "frac_nominal": verify_gbs / NOMINAL_HBM_GBS},
        "roofline_round": {"bound": "hbm", "achieved": round_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": round_gbs / peaks["hbm_gbs"], "frac_nominal": round_gbs / NOMINAL_HBM_GBS,
                           "algorithmic_bytes": dbytes + vbytes},
        "roofline_l2": roofline_l2,
        "round_stats": {"verify_tokens": int((L + 1).sum()), "accepted_mean": float(acc.mean()),
                        "emitted_per_round": int(n_out.sum())},
        "gpu_launches": launches_per_round * args.steps,
        "clocks": clocks.summary(),
        "e2e": e2e,
        "cpu_baseline": cb,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen3")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--variant", default="auto", choices=["auto", "a", "b"],
                    help="a: the draft stores z; b: verify recomputes the rejected rows; auto: b from B = 128 on")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
