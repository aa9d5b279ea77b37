"""One DSpark round on the GPU through the C ABI: draft -> schedule -> verify.

`RoundBuffers` owns the device outputs and the workspace of one round shape;
`run_round` enqueues the three library calls on one stream without any host
synchronisation (the scheduler's verify lengths and row offsets stay on the
device and feed the verification directly).
"""
from __future__ import annotations

import numpy as np
import torch

from .binding import (dspark_markov_draft, dspark_schedule, dspark_verify, dspark_workspace_bytes,
                      dspark_workspace_init)


def to_device(inputs: dict, device="cuda") -> dict:
    """Host numpy round inputs (bf16 factors as uint16 bits) -> device tensors."""
    out = {}
    for k, v in inputs.items():
        if not isinstance(v, np.ndarray):
            continue
        if k in ("A", "Bf") and v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).to(device).view(torch.bfloat16)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device)
    B, K = inputs["u_draft"].shape
    if "target" in out:
        out["target"] = out["target"].reshape(B * (K + 1), -1)
        out["row_start_dense"] = torch.arange(B, dtype=torch.int64, device=device) * (K + 1)
    return out


class RoundBuffers:
    def __init__(self, B: int, K: int, V: int, r: int, device="cuda"):
        self.B, self.K, self.V, self.r = B, K, V, r
        i32, f32, f64 = torch.int32, torch.float32, torch.float64
        self.draft_tokens = torch.empty(B, K, dtype=i32, device=device)
        self.q_tok = torch.empty(B, K, dtype=f32, device=device)
        self.lse_q = torch.empty(B, K, dtype=f64, device=device)
        self.z = torch.empty(B, K, V, dtype=f32, device=device)
        self.verify_len = torch.empty(B, dtype=i32, device=device)
        self.survival = torch.empty(B, K, dtype=f32, device=device)
        self.row_start = torch.empty(B, dtype=torch.int64, device=device)
        self.n_tokens = torch.empty(1, dtype=i32, device=device)
        self.accepted = torch.empty(B, dtype=i32, device=device)
        self.out_tokens = torch.empty(B, K + 1, dtype=i32, device=device)
        self.n_out = torch.empty(B, dtype=i32, device=device)
        self.workspace = torch.empty(dspark_workspace_bytes(B, K, V, r), dtype=torch.uint8, device=device)
        dspark_workspace_init(self.workspace)


def draft(d: dict, bufs: RoundBuffers, stream=None):
    dspark_markov_draft(d["base"], d["A"], d["Bf"], d["anchor"], d["u_draft"], bufs.draft_tokens, bufs.q_tok,
                        bufs.lse_q, bufs.z, bufs.workspace, stream)


def schedule(d: dict, bufs: RoundBuffers, stream=None):
    dspark_schedule(d["conf"], d["temps"], d["profile"], bufs.verify_len, bufs.survival, bufs.row_start,
                    bufs.n_tokens, bufs.workspace, stream)


def verify(d: dict, bufs: RoundBuffers, target=None, row_start=None, verify_len=None, stream=None):
    """Verify against `target` rows addressed by `row_start` (default: the dense
    [B,K+1,V] target of `d`, row_start[b] = b*(K+1))."""
    dspark_verify(d["target"] if target is None else target,
                  d["row_start_dense"] if row_start is None else row_start,
                  bufs.z, bufs.lse_q, bufs.q_tok, bufs.draft_tokens,
                  bufs.verify_len if verify_len is None else verify_len,
                  d["u_accept"], d["u_resample"], bufs.accepted, bufs.out_tokens, bufs.n_out,
                  bufs.workspace, stream)


def run_round(d: dict, bufs: RoundBuffers, stream=None):
    draft(d, bufs, stream)
    schedule(d, bufs, stream)
    verify(d, bufs, stream=stream)
