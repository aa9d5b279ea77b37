"""DSpark rounds on the GPU through the C ABI: draft -> schedule -> verify.

`RoundBuffers` owns the device outputs and the workspace of one round shape;
`run_round` enqueues the three library calls on one stream without any host
synchronisation (the scheduler's verify lengths and row offsets stay on the
device and feed the verification directly). `run_rounds` chains rounds on the
device (online temperature calibration and the next anchors included), as a
plain stream of launches or one captured CUDA graph.
"""
from __future__ import annotations

import numpy as np
import torch

from .binding import (dspark_advance_anchor, dspark_calibrate, dspark_markov_draft, dspark_markov_draft_b,
                      dspark_rnn_draft, dspark_rnn_draft_b, dspark_schedule, dspark_verify, dspark_verify_b,
                      dspark_workspace_bytes, dspark_workspace_init)


def to_device(inputs: dict, device="cuda") -> dict:
    """Host numpy round inputs (bf16 factors as uint16 bits) -> device tensors."""
    out = {}
    for k, v in inputs.items():
        if not isinstance(v, np.ndarray):
            continue
        if k in ("A", "Bf", "W") and v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).to(device).view(torch.bfloat16)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device)
    B, K = inputs["u_draft"].shape
    if "target" in out:
        out["target"] = out["target"].reshape(B * (K + 1), -1)
        out["row_start_dense"] = torch.arange(B, dtype=torch.int64, device=device) * (K + 1)
    return out


class RoundBuffers:
    """Variant "a" stores the draft logits z [B,K,V]; variant "b" stores the
    operand rows op_rows [B,K,r] (bf16) instead and verification recomputes
    the rejected row of z."""

    def __init__(self, B: int, K: int, V: int, r: int, device="cuda", variant: str = "a"):
        if variant not in ("a", "b"):
            raise ValueError("variant must be 'a' or 'b'")
        self.B, self.K, self.V, self.r, self.variant = B, K, V, r, variant
        i32, f32, f64 = torch.int32, torch.float32, torch.float64
        self.draft_tokens = torch.empty(B, K, dtype=i32, device=device)
        self.q_tok = torch.empty(B, K, dtype=f32, device=device)
        self.lse_q = torch.empty(B, K, dtype=f64, device=device)
        self.z = torch.empty(B, K, V, dtype=f32, device=device) if variant == "a" else None
        self.op_rows = torch.empty(B, K, r, dtype=torch.bfloat16, device=device) if variant == "b" else None
        self.verify_len = torch.empty(B, dtype=i32, device=device)
        self.survival = torch.empty(B, K, dtype=f32, device=device)
        self.row_start = torch.empty(B, dtype=torch.int64, device=device)
        self.n_tokens = torch.empty(1, dtype=i32, device=device)
        self.accepted = torch.empty(B, dtype=i32, device=device)
        self.out_tokens = torch.empty(B, K + 1, dtype=i32, device=device)
        self.n_out = torch.empty(B, dtype=i32, device=device)
        self.workspace = torch.empty(dspark_workspace_bytes(B, K, V, r), dtype=torch.uint8, device=device)
        dspark_workspace_init(self.workspace)


def draft(d: dict, bufs: RoundBuffers, stream=None, anchor=None):
    """The Markov head, or the RNN head when d holds its recurrent weight "W";
    `anchor` overrides d["anchor"]."""
    anchor = d["anchor"] if anchor is None else anchor
    out = (bufs.draft_tokens, bufs.q_tok, bufs.lse_q)
    if bufs.variant == "b":
        if d.get("W") is not None:
            dspark_rnn_draft_b(d["base"], d["A"], d["W"], d["Bf"], anchor, d["u_draft"], *out, bufs.op_rows,
                               bufs.workspace, stream)
        else:
            dspark_markov_draft_b(d["base"], d["A"], d["Bf"], anchor, d["u_draft"], *out, bufs.op_rows,
                                  bufs.workspace, stream)
    elif d.get("W") is not None:
        dspark_rnn_draft(d["base"], d["A"], d["W"], d["Bf"], anchor, d["u_draft"], *out, bufs.z, bufs.workspace,
                         stream)
    else:
        dspark_markov_draft(d["base"], d["A"], d["Bf"], anchor, d["u_draft"], *out, bufs.z, bufs.workspace, stream)


def schedule(d: dict, bufs: RoundBuffers, stream=None, temps=None):
    dspark_schedule(d["conf"], d["temps"] if temps is None else temps, d["profile"], bufs.verify_len, bufs.survival,
                    bufs.row_start, bufs.n_tokens, bufs.workspace, stream)


def verify(d: dict, bufs: RoundBuffers, target=None, row_start=None, verify_len=None, stream=None):
    """Verify against `target` rows addressed by `row_start` (default: the dense
    [B,K+1,V] target of `d`, row_start[b] = b*(K+1))."""
    target = d["target"] if target is None else target
    row_start = d["row_start_dense"] if row_start is None else row_start
    verify_len = bufs.verify_len if verify_len is None else verify_len
    tail = (bufs.lse_q, bufs.q_tok, bufs.draft_tokens, verify_len, d["u_accept"], d["u_resample"], bufs.accepted,
            bufs.out_tokens, bufs.n_out, bufs.workspace, stream)
    if bufs.variant == "b":
        dspark_verify_b(target, row_start, d["base"], bufs.op_rows, d["Bf"], *tail)
    else:
        dspark_verify(target, row_start, bufs.z, *tail)


def run_round(d: dict, bufs: RoundBuffers, stream=None):
    draft(d, bufs, stream)
    schedule(d, bufs, stream)
    verify(d, bufs, stream=stream)


class RoundState:
    """What carries from one round to the next on the device: the anchors
    (the last token each request emitted) and the calibrated temperatures."""

    def __init__(self, anchor: torch.Tensor, temps: torch.Tensor):
        self.anchor = anchor.clone()
        self.temps = temps.clone()


HISTORY = {"anchor": ("B",), "temps": ("K",), "draft_tokens": ("B", "K"), "q_tok": ("B", "K"),
           "lse_q": ("B", "K"), "verify_len": ("B",), "survival": ("B", "K"), "row_start": ("B",),
           "n_tokens": (1,), "accepted": ("B",), "out_tokens": ("B", "K+1"), "n_out": ("B",)}


def run_rounds(inputs: list, bufs: RoundBuffers, state: RoundState, rounds: int, calibrate=None,
               record: bool = True, graph: bool = False, stream=None) -> dict:
    """`rounds` rounds back to back on one stream, with no host synchronisation:
    draft -> schedule -> verify -> (calibrate) -> next anchors. Round r reads
    inputs[r % len(inputs)] (device dicts from to_device; in a serving system
    the backbone and target forward passes would refill these between rounds)
    and the anchors and temperatures in `state`, which the round updates.
    calibrate = (eta, t_min, t_max) turns on the online temperature step.
    With record=True each round's state and outputs are copied into history
    tensors [rounds, ...] (device-to-device). With graph=True the rounds are
    captured once as a CUDA graph and replayed; the graph is returned in the
    result under "graph" so that it can be replayed again.
    """
    B, K = bufs.B, bufs.K
    dims = {"B": B, "K": K, "K+1": K + 1}
    hist = {}
    if record:
        for name, shape in HISTORY.items():
            ref = state.anchor if name == "anchor" else state.temps if name == "temps" else getattr(bufs, name)
            hist[name] = torch.empty((rounds,) + tuple(dims.get(s, s) for s in shape), dtype=ref.dtype,
                                     device=ref.device)

    def body(s):
        for r in range(rounds):
            d = inputs[r % len(inputs)]
            if record:
                hist["anchor"][r].copy_(state.anchor, non_blocking=True)
                hist["temps"][r].copy_(state.temps, non_blocking=True)
            draft(d, bufs, s, anchor=state.anchor)
            schedule(d, bufs, s, temps=state.temps)
            verify(d, bufs, stream=s)
            if record:
                for name in HISTORY:
                    if name not in ("anchor", "temps"):
                        hist[name][r].copy_(getattr(bufs, name), non_blocking=True)
            if calibrate is not None:
                eta, t_min, t_max = calibrate
                dspark_calibrate(d["conf"], bufs.verify_len, bufs.accepted, state.temps, bufs.workspace, eta, t_min,
                                 t_max, s)
            dspark_advance_anchor(bufs.out_tokens, bufs.n_out, state.anchor, bufs.workspace, s)

    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body(torch.cuda.current_stream())
        g.replay()
        hist["graph"] = g
    else:
        body(stream)
    return hist
