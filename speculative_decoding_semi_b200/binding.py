"""Thin ctypes binding of libdspark (argument marshalling only).

The functions carry the C names of include/dspark.h and take torch CUDA
tensors (for device memory) plus an optional torch.cuda.Stream; every step of
the computation runs in the library's kernels. If the library is missing the
import fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdspark.so")

DSPARK_F32, DSPARK_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error",
          4: "device-wide wait timed out", 5: "device-side check failed"}


class DSparkError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: int | None = None):
        self.status = status
        self.detail = detail
        msg = f"{fn}: {STATUS.get(status, status)} (status {status})"
        if detail is not None:
            msg += f", detail 0x{detail:08x}"
        super().__init__(msg)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python speculative_decoding_semi_b200/build.py` "
            "(nvcc, sm_100a). There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    lib.dspark_workspace_bytes.argtypes = [I, I, I, I]
    lib.dspark_workspace_bytes.restype = Z
    lib.dspark_workspace_init.argtypes = [P, Z, S]
    lib.dspark_workspace_init.restype = I
    lib.dspark_markov_draft.argtypes = [P, P, P, I, I, P, P, I, I, I, P, P, P, P, P, Z, S]
    lib.dspark_markov_draft.restype = I
    lib.dspark_rnn_draft.argtypes = [P, P, P, P, I, I, P, P, I, I, I, P, P, P, P, P, Z, S]
    lib.dspark_rnn_draft.restype = I
    lib.dspark_schedule.argtypes = [P, P, P, I, I, I, P, P, P, P, P, Z, S]
    lib.dspark_schedule.restype = I
    lib.dspark_verify.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, P, P, P, P, Z, S]
    lib.dspark_verify.restype = I
    lib.dspark_markov_draft_b.argtypes = [P, P, P, I, I, P, P, I, I, I, P, P, P, P, P, Z, S]
    lib.dspark_markov_draft_b.restype = I
    lib.dspark_rnn_draft_b.argtypes = [P, P, P, P, I, I, P, P, I, I, I, P, P, P, P, P, Z, S]
    lib.dspark_rnn_draft_b.restype = I
    lib.dspark_verify_b.argtypes = [P, P, P, P, P, I, P, P, P, P, P, P, I, I, I, P, P, P, P, Z, S]
    lib.dspark_verify_b.restype = I
    lib.dspark_read_device_error.argtypes = [P, S, ctypes.POINTER(ctypes.c_uint32)]
    lib.dspark_read_device_error.restype = I
    lib.dspark_schedule_static.argtypes = [P, P, P, I, I, I, P, P, P, P, S]
    lib.dspark_schedule_static.restype = I
    F = ctypes.c_float
    lib.dspark_calibrate.argtypes = [P, P, P, I, I, F, F, F, P, P, Z, S]
    lib.dspark_calibrate.restype = I
    lib.dspark_advance_anchor.argtypes = [P, P, I, I, P, P, Z, S]
    lib.dspark_advance_anchor.restype = I
    lib.dspark_set_wait_budget.argtypes = [P, ctypes.c_uint32, S]
    lib.dspark_set_wait_budget.restype = I
    lib.dspark_inject_stall.argtypes = [P, I, ctypes.c_uint32, S]
    lib.dspark_inject_stall.restype = I
    lib.dspark_status_string.argtypes = [I]
    lib.dspark_status_string.restype = ctypes.c_char_p
    return lib


lib = _load()


def _ptr(t: torch.Tensor | None, name: str, dtype=None, numel=None) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor (the library computes on the GPU only)")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements, got {t.numel()}")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != 0:
        raise DSparkError(fn, status)


def dspark_workspace_bytes(B: int, K: int, V: int, r: int) -> int:
    n = lib.dspark_workspace_bytes(B, K, V, r)
    if n == 0:
        raise DSparkError("dspark_workspace_bytes", 1)
    return int(n)


def dspark_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check("dspark_workspace_init",
           lib.dspark_workspace_init(_ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)))


def dspark_markov_draft(base_logits, A, Bf, anchor, u_draft, draft_tokens, q_tok, lse_q, z, workspace,
                        stream=None) -> None:
    B, K, V = base_logits.shape
    r = A.shape[1]
    if A.dtype == torch.bfloat16 and Bf.dtype == torch.bfloat16:
        dt = DSPARK_BF16
    elif A.dtype == torch.float32 and Bf.dtype == torch.float32:
        dt = DSPARK_F32
    else:
        raise TypeError("A and Bf must both be float32 or both bfloat16")
    st = lib.dspark_markov_draft(
        _ptr(base_logits, "base_logits", torch.float32), _ptr(A, "A", numel=V * r), _ptr(Bf, "Bf", numel=r * V),
        dt, r, _ptr(anchor, "anchor", torch.int32, B), _ptr(u_draft, "u_draft", torch.float32, B * K),
        B, K, V, _ptr(draft_tokens, "draft_tokens", torch.int32, B * K), _ptr(q_tok, "q_tok", torch.float32, B * K),
        _ptr(lse_q, "lse_q", torch.float64, B * K), _ptr(z, "z", torch.float32, B * K * V),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("dspark_markov_draft", st)


def dspark_rnn_draft(base_logits, A, W, Bf, anchor, u_draft, draft_tokens, q_tok, lse_q, z, workspace,
                     stream=None) -> None:
    """Draft with the RNN sequential head (W [r,r] bf16); bf16 factors only."""
    B, K, V = base_logits.shape
    r = A.shape[1]
    if not (A.dtype == Bf.dtype == W.dtype == torch.bfloat16):
        raise TypeError("the RNN head takes bf16 A, W and Bf")
    st = lib.dspark_rnn_draft(
        _ptr(base_logits, "base_logits", torch.float32), _ptr(A, "A", numel=V * r), _ptr(W, "W", numel=r * r),
        _ptr(Bf, "Bf", numel=r * V), DSPARK_BF16, r, _ptr(anchor, "anchor", torch.int32, B),
        _ptr(u_draft, "u_draft", torch.float32, B * K), B, K, V,
        _ptr(draft_tokens, "draft_tokens", torch.int32, B * K), _ptr(q_tok, "q_tok", torch.float32, B * K),
        _ptr(lse_q, "lse_q", torch.float64, B * K), _ptr(z, "z", torch.float32, B * K * V),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("dspark_rnn_draft", st)


def dspark_markov_draft_b(base_logits, A, Bf, anchor, u_draft, draft_tokens, q_tok, lse_q, op_rows, workspace,
                          stream=None) -> None:
    """Variant B of dspark_markov_draft: no z; op_rows [B,K,r] (bfloat16)
    receives the operand row of every position. bf16 factors only."""
    B, K, V = base_logits.shape
    r = A.shape[1]
    if not (A.dtype == Bf.dtype == torch.bfloat16):
        raise TypeError("variant B takes bf16 A and Bf")
    st = lib.dspark_markov_draft_b(
        _ptr(base_logits, "base_logits", torch.float32), _ptr(A, "A", numel=V * r), _ptr(Bf, "Bf", numel=r * V),
        DSPARK_BF16, r, _ptr(anchor, "anchor", torch.int32, B), _ptr(u_draft, "u_draft", torch.float32, B * K),
        B, K, V, _ptr(draft_tokens, "draft_tokens", torch.int32, B * K), _ptr(q_tok, "q_tok", torch.float32, B * K),
        _ptr(lse_q, "lse_q", torch.float64, B * K), _ptr(op_rows, "op_rows", torch.bfloat16, B * K * r),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("dspark_markov_draft_b", st)


def dspark_rnn_draft_b(base_logits, A, W, Bf, anchor, u_draft, draft_tokens, q_tok, lse_q, op_rows, workspace,
                       stream=None) -> None:
    """Variant B of dspark_rnn_draft (op_rows in place of z)."""
    B, K, V = base_logits.shape
    r = A.shape[1]
    if not (A.dtype == Bf.dtype == W.dtype == torch.bfloat16):
        raise TypeError("the RNN head takes bf16 A, W and Bf")
    st = lib.dspark_rnn_draft_b(
        _ptr(base_logits, "base_logits", torch.float32), _ptr(A, "A", numel=V * r), _ptr(W, "W", numel=r * r),
        _ptr(Bf, "Bf", numel=r * V), DSPARK_BF16, r, _ptr(anchor, "anchor", torch.int32, B),
        _ptr(u_draft, "u_draft", torch.float32, B * K), B, K, V,
        _ptr(draft_tokens, "draft_tokens", torch.int32, B * K), _ptr(q_tok, "q_tok", torch.float32, B * K),
        _ptr(lse_q, "lse_q", torch.float64, B * K), _ptr(op_rows, "op_rows", torch.bfloat16, B * K * r),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("dspark_rnn_draft_b", st)


def dspark_schedule(conf_logits, temps, profile_ms, verify_len, survival, row_start, n_tokens, workspace,
                    stream=None) -> None:
    B, K = conf_logits.shape
    st = lib.dspark_schedule(
        _ptr(conf_logits, "conf_logits", torch.float32), _ptr(temps, "temps", torch.float32, K),
        _ptr(profile_ms, "profile_ms", torch.float32), profile_ms.numel(), B, K,
        _ptr(verify_len, "verify_len", torch.int32, B), _ptr(survival, "survival", torch.float32, B * K),
        _ptr(row_start, "row_start", torch.int64, B), _ptr(n_tokens, "n_tokens", torch.int32, 1),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("dspark_schedule", st)


def dspark_schedule_static(conf_logits, temps, profile_ms, verify_len, survival, row_start, n_tokens,
                           stream=None) -> None:
    """dspark_schedule without a workspace (scratch in a static device array
    inside the library), for callers that cannot allocate device memory. Same
    outputs; B*K is limited to 16384; calls must not overlap on the GPU."""
    B, K = conf_logits.shape
    st = lib.dspark_schedule_static(
        _ptr(conf_logits, "conf_logits", torch.float32), _ptr(temps, "temps", torch.float32, K),
        _ptr(profile_ms, "profile_ms", torch.float32), profile_ms.numel(), B, K,
        _ptr(verify_len, "verify_len", torch.int32, B), _ptr(survival, "survival", torch.float32, B * K),
        _ptr(row_start, "row_start", torch.int64, B), _ptr(n_tokens, "n_tokens", torch.int32, 1),
        _stream(stream))
    _check("dspark_schedule_static", st)


def dspark_verify(target_logits, row_start, z, lse_q, q_tok, draft_tokens, verify_len, u_accept, u_resample,
                  accepted, out_tokens, n_out, workspace, stream=None) -> None:
    B, K, V = z.shape
    if target_logits.shape[-1] != V:
        raise ValueError("target_logits must have V columns")
    st = lib.dspark_verify(
        _ptr(target_logits, "target_logits", torch.float32), _ptr(row_start, "row_start", torch.int64, B),
        _ptr(z, "z", torch.float32), _ptr(lse_q, "lse_q", torch.float64, B * K),
        _ptr(q_tok, "q_tok", torch.float32, B * K), _ptr(draft_tokens, "draft_tokens", torch.int32, B * K),
        _ptr(verify_len, "verify_len", torch.int32, B), _ptr(u_accept, "u_accept", torch.float32, B * K),
        _ptr(u_resample, "u_resample", torch.float32, B), B, K, V,
        _ptr(accepted, "accepted", torch.int32, B), _ptr(out_tokens, "out_tokens", torch.int32, B * (K + 1)),
        _ptr(n_out, "n_out", torch.int32, B), _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _stream(stream))
    _check("dspark_verify", st)


def dspark_verify_b(target_logits, row_start, base_logits, op_rows, Bf, lse_q, q_tok, draft_tokens, verify_len,
                    u_accept, u_resample, accepted, out_tokens, n_out, workspace, stream=None) -> None:
    """Variant B of dspark_verify: the rejected row's z is recomputed from
    base_logits, op_rows [B,K,r] (bfloat16) and Bf [r,V] (bfloat16)."""
    B, K, V = base_logits.shape
    r = Bf.shape[0]
    if target_logits.shape[-1] != V:
        raise ValueError("target_logits must have V columns")
    st = lib.dspark_verify_b(
        _ptr(target_logits, "target_logits", torch.float32), _ptr(row_start, "row_start", torch.int64, B),
        _ptr(base_logits, "base_logits", torch.float32), _ptr(op_rows, "op_rows", torch.bfloat16, B * K * r),
        _ptr(Bf, "Bf", torch.bfloat16, r * V), r, _ptr(lse_q, "lse_q", torch.float64, B * K),
        _ptr(q_tok, "q_tok", torch.float32, B * K), _ptr(draft_tokens, "draft_tokens", torch.int32, B * K),
        _ptr(verify_len, "verify_len", torch.int32, B), _ptr(u_accept, "u_accept", torch.float32, B * K),
        _ptr(u_resample, "u_resample", torch.float32, B), B, K, V,
        _ptr(accepted, "accepted", torch.int32, B), _ptr(out_tokens, "out_tokens", torch.int32, B * (K + 1)),
        _ptr(n_out, "n_out", torch.int32, B), _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _stream(stream))
    _check("dspark_verify_b", st)


def dspark_calibrate(conf_logits, verify_len, accepted, temps, workspace, eta: float, t_min: float, t_max: float,
                     stream=None) -> None:
    """One online step of the sequential temperatures (temps updated in place)."""
    B, K = conf_logits.shape
    st = lib.dspark_calibrate(
        _ptr(conf_logits, "conf_logits", torch.float32), _ptr(verify_len, "verify_len", torch.int32, B),
        _ptr(accepted, "accepted", torch.int32, B), B, K, float(eta), float(t_min), float(t_max),
        _ptr(temps, "temps", torch.float32, K), _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _stream(stream))
    _check("dspark_calibrate", st)


def dspark_advance_anchor(out_tokens, n_out, anchor, workspace, stream=None) -> None:
    """anchor[b] = out_tokens[b, n_out[b]-1], for the next round."""
    B, K1 = out_tokens.shape
    st = lib.dspark_advance_anchor(
        _ptr(out_tokens, "out_tokens", torch.int32), _ptr(n_out, "n_out", torch.int32, B), B, K1 - 1,
        _ptr(anchor, "anchor", torch.int32, B), _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _stream(stream))
    _check("dspark_advance_anchor", st)


DSPARK_INJECT_NONE, DSPARK_INJECT_DRAFT_SLICE_SUMS, DSPARK_INJECT_VERIFY_BARRIER = 0, 1, 2
DSPARK_INJECT_RESIDUAL_SLICE_SUMS = 3


def dspark_set_wait_budget(workspace, microseconds: int, stream=None) -> None:
    _check("dspark_set_wait_budget", lib.dspark_set_wait_budget(_ptr(workspace, "workspace", torch.uint8),
                                                                int(microseconds), _stream(stream)))


def dspark_inject_stall(workspace, where: int, cta: int = 0, stream=None) -> None:
    _check("dspark_inject_stall", lib.dspark_inject_stall(_ptr(workspace, "workspace", torch.uint8), int(where),
                                                          int(cta), _stream(stream)))


def dspark_read_device_error(workspace, stream=None) -> tuple[int, int]:
    detail = ctypes.c_uint32(0)
    st = lib.dspark_read_device_error(_ptr(workspace, "workspace", torch.uint8), _stream(stream),
                                      ctypes.byref(detail))
    if st in (1, 3):
        raise DSparkError("dspark_read_device_error", st)
    return int(st), int(detail.value)


def dspark_status_string(status: int) -> str:
    return lib.dspark_status_string(status).decode()
