"""Measured round-time profiles T(n) for the scheduler.

QbitAI article "DSpark: ten concepts are enough", section "variable-length
drafts and hardware-aware scheduling": the GPU's throughput is measured ahead
of time at each batch size and turned into a reference curve, from which each
request's verify length is chosen. dspark_schedule reads that curve as a table
T(n), the round time in ms at n verify-batch tokens (each request's last token
plus its verified drafts).

build_profile measures this library's own share of a round on the device it
runs on: the draft of B requests (a fixed cost per round) plus the schedule
and the verification of n packed target rows, timed with CUDA events after an
L2-flushing write, at a grid of n from B to B(K+1); the table interpolates
linearly between grid points, extends the last segment beyond them, and is
made non-decreasing (a longer verify batch never takes less time). A serving
engine would add its target forward pass at each n, timed the same way.
"""
from __future__ import annotations

import numpy as np
import torch

from . import round as rnd
from .binding import dspark_verify


def split_lengths(n: int, B: int, K: int) -> np.ndarray:
    """Verify lengths L_b in [0, K] with sum(L_b + 1) = n, as equal as possible
    (the first requests take the remainder). Needs B <= n <= B (K + 1)."""
    if not B <= n <= B * (K + 1):
        raise ValueError(f"n={n} outside [{B}, {B * (K + 1)}]")
    extra = n - B
    L = np.full(B, extra // B, np.int64)
    L[: extra % B] += 1
    return L


def interpolate(grid: np.ndarray, ms: np.ndarray, n_prof: int) -> np.ndarray:
    """T(n) for n = 1..n_prof from measurements at increasing grid points:
    linear between points, the first value below the grid, the last segment's
    slope beyond it, then a running maximum so that T never decreases."""
    grid = np.asarray(grid, np.float64)
    ms = np.asarray(ms, np.float64)
    if grid.ndim != 1 or grid.size < 1 or np.any(np.diff(grid) <= 0):
        raise ValueError("grid must be strictly increasing")
    n = np.arange(1, n_prof + 1, dtype=np.float64)
    t = np.interp(n, grid, ms)
    if grid.size >= 2:
        slope = (ms[-1] - ms[-2]) / (grid[-1] - grid[-2])
        beyond = n > grid[-1]
        t[beyond] = ms[-1] + max(slope, 0.0) * (n[beyond] - grid[-1])
    return np.maximum.accumulate(t).astype(np.float32)


def grid_points(B: int, K: int, points: int) -> np.ndarray:
    """`points` verify-batch sizes from B to B (K + 1), spaced evenly."""
    return np.unique(np.linspace(B, B * (K + 1), max(2, points)).round().astype(np.int64))


def build_profile(inp: dict, n_prof: int, points: int = 8, reps: int = 5, stream=None) -> dict:
    """Measure T(n) for the round shape of `inp` (host inputs as synth makes
    them: base, factors, anchors, uniforms, confidences, target rows).
    Returns {"grid", "ms", "table"}: the measured sizes, their median times
    (ms) and the interpolated table for n = 1..n_prof."""
    B, K, V = inp["base"].shape
    r = inp["A"].shape[1]
    d = rnd.to_device(inp)
    bufs = rnd.RoundBuffers(B, K, V, r)
    s = torch.cuda.current_stream() if stream is None else stream
    flush = torch.empty(128 * 1024 * 1024, dtype=torch.float32, device=d["base"].device)
    grid = grid_points(B, K, points)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    out = []
    for n in grid:
        L = torch.as_tensor(split_lengths(int(n), B, K), dtype=torch.int32, device=d["base"].device)
        row_start = torch.zeros(B, dtype=torch.int64, device=L.device)
        row_start[1:] = torch.cumsum(L.long() + 1, 0)[:-1]
        target = d["target"][: int(n)]   # n packed rows: their values only pace the stream
        times = []
        for _ in range(reps + 1):
            with torch.cuda.stream(s):
                flush.fill_(1.0)
                ev[0].record(s)
                rnd.draft(d, bufs, s)
                rnd.schedule(d, bufs, s)
                ev[1].record(s)
                dspark_verify(target, row_start, bufs.z, bufs.lse_q, bufs.q_tok, bufs.draft_tokens, L, d["u_accept"],
                              d["u_resample"], bufs.accepted, bufs.out_tokens, bufs.n_out, bufs.workspace, s)
                ev[2].record(s)
            ev[2].synchronize()
            times.append(ev[0].elapsed_time(ev[2]))
        out.append(float(np.median(times[1:])))
    ms = np.asarray(out)
    return {"grid": grid, "ms": ms, "table": interpolate(grid, ms, n_prof)}
