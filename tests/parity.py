"""GPU-vs-oracle comparison of one round (test infrastructure).

Integer outputs must match exactly, except where the oracle's own decision
margin is below MARGIN (1e-5): inverse-CDF margin d < 1e-5, accept margin
|u - p/q| < 1e-5, or a scheduler near-tie (|P_(m*) - P_(m*+1)| < 1e-5 P_(m*)
or a runner-up objective within 1e-5). Such mismatches are counted as
excused and their pooled count must stay at or under 0.1% of the decisions
(a point rate, no allowance for sampling noise); any other mismatch fails. After an excused mismatch the oracle continues from the GPU's
choice (teacher forcing), so one near-tie counts once.
Float outputs: q_tok and survival within 2e-3 relative, lse_q within 2e-3
absolute; z within 1e-4 absolute + 1e-5 relative (fp32 rounding of base +
bias, with the bias accumulated in fp32).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
import synth

MARGIN = 1e-5
RATE = 1e-3

# Pooled tallies of this process, by test, for the end-of-run summary.
SUMMARY: dict = {}


@dataclasses.dataclass
class Tally:
    decisions: int = 0
    excused: int = 0
    flagged: int = 0
    failures: list = dataclasses.field(default_factory=list)
    by_kind: dict = dataclasses.field(default_factory=dict)

    def add(self, other: "Tally"):
        self.decisions += other.decisions
        self.excused += other.excused
        self.flagged += other.flagged
        self.failures += other.failures
        for k, v in other.by_kind.items():
            a = self.by_kind.setdefault(k, [0, 0])
            a[0] += v[0]
            a[1] += v[1]

    def count(self, kind: str, decisions: int, excused: int):
        self.decisions += decisions
        self.excused += excused
        a = self.by_kind.setdefault(kind, [0, 0])
        a[0] += decisions
        a[1] += excused

    def check(self, name: str | None = None):
        if name is not None:
            SUMMARY[name] = {"decisions": self.decisions, "excused": self.excused, "flagged": self.flagged,
                             "by_kind": {k: list(v) for k, v in self.by_kind.items()}}
        assert not self.failures, self.failures[:10]
        assert within_rate(self.excused, self.decisions), (self.excused, self.decisions, self.flagged)


def within_rate(excused: int, decisions: int) -> bool:
    """Excused mismatches must stay under RATE (0.1%) of the decisions, as a
    point rate: excused <= 0.001 * decisions (so none at all below 1,000)."""
    return excused <= RATE * decisions


def compare_draft(inp, gpu, requests, tally: Tally, check_z=True):
    """gpu: dict of numpy outputs for the sampled `requests` (tokens, q_tok, lse_q, z).
    With inp["W"] (the RNN head's recurrent weight) the oracle is rnn_draft."""
    base = inp["base"][requests]
    if inp.get("W") is not None:
        d = oracle.rnn_draft(base, inp["A"], inp["W"], inp["Bf"], inp["anchor"][requests], inp["u_draft"][requests],
                             teacher=gpu["tokens"].astype(np.int64), keep_z=True)
    else:
        d = oracle.draft(base, inp["A"], inp["Bf"], inp["anchor"][requests], inp["u_draft"][requests],
                         teacher=gpu["tokens"].astype(np.int64), keep_z=True)
    mism = d["t"] != gpu["tokens"]
    small = d["margin"] < MARGIN
    tally.flagged += int(small.sum())
    tally.count("draft", mism.size, int((mism & small).sum()))
    bad = np.argwhere(mism & ~small)
    for b, i in bad[:5]:
        tally.failures.append(("draft token", int(requests[b]), int(i), int(d["t"][b, i]), int(gpu["tokens"][b, i]),
                               float(d["margin"][b, i])))
    rel = np.abs(gpu["q_tok"] - d["q_tok"]) / np.maximum(d["q_tok"], 1e-300)
    if rel.max() > 2e-3:
        tally.failures.append(("q_tok rel", float(rel.max())))
    err = np.abs(gpu["lse_q"] - d["lse"]).max()
    if err > 2e-3:
        tally.failures.append(("lse_q abs", float(err)))
    if check_z:
        zerr = np.abs(gpu["z"].astype(np.float64) - d["z"]) - 1e-5 * np.abs(d["z"])
        if zerr.max() > 1e-4:
            idx = np.unravel_index(np.argmax(zerr), zerr.shape)
            tally.failures.append(("z", float(zerr.max()), idx))
    return d


def compare_schedule(inp, gpu, tally: Tally):
    P = oracle.survival(inp["conf"], inp["temps"])
    s = oracle.schedule(P, inp["profile"])
    rel = np.abs(gpu["survival"] - P) / P
    if rel.max() > 2e-3:
        tally.failures.append(("survival rel", float(rel.max())))
    B = P.shape[0]
    L = gpu["verify_len"]
    exc = 0
    if not np.array_equal(L, s["verify_len"]):
        if s["gap_item"] < MARGIN or s["gap_obj"] < MARGIN:
            exc = int((L != s["verify_len"]).sum())
        else:
            tally.failures.append(("verify_len", np.argwhere(L != s["verify_len"]).ravel()[:5].tolist(),
                                   float(s["gap_item"]), float(s["gap_obj"])))
    tally.count("schedule", B, exc)
    # the GPU's own offsets must be the exclusive scan of its own lengths
    exp_rs = np.concatenate([[0], np.cumsum(L.astype(np.int64) + 1)[:-1]])
    if not np.array_equal(gpu["row_start"], exp_rs):
        tally.failures.append(("row_start", gpu["row_start"][:5].tolist(), exp_rs[:5].tolist()))
    if int(gpu["n_tokens"]) != int((L + 1).sum()):
        tally.failures.append(("n_tokens", int(gpu["n_tokens"]), int((L + 1).sum())))
    return s


def compare_verify(inp, draft_oracle, gpu_draft, gpu, verify_len, requests, tally: Tally):
    """Teacher-forced: the oracle verifies the GPU's tokens with the GPU's lengths."""
    B, K, V = inp["base"].shape
    rows = inp["target"].reshape(B * (K + 1), V)
    rs = np.arange(B, dtype=np.int64) * (K + 1)
    vo = oracle.verify(rows, rs, draft_oracle["z"], draft_oracle["lse"], draft_oracle["q_tok"],
                       gpu_draft["tokens"], verify_len, inp["u_accept"], inp["u_resample"],
                       requests=requests)
    acc_g = gpu["accepted"]
    vo2 = None
    for idx, b in enumerate(requests):
        Lb = int(verify_len[b])
        margins = vo["accept_margin"][idx]
        tally.flagged += int(sum(m < MARGIN for m in margins))
        ao, ag = int(vo["accepted"][idx]), int(acc_g[idx])
        exc = 0
        if ao != ag:
            j = min(ao, ag)  # first position where the decisions differ (0-based)
            if j < len(margins) and margins[j] < MARGIN:
                exc = 1
            else:
                tally.failures.append(("accepted", int(b), ao, ag, margins[j] if j < len(margins) else None))
        tally.count("accept", len(margins), exc)
        if not (1 <= gpu["n_out"][idx] <= Lb + 1) or gpu["n_out"][idx] != ag + 1:
            tally.failures.append(("n_out", int(b), int(gpu["n_out"][idx]), ag))
        if not np.array_equal(gpu["out_tokens"][idx, :ag], gpu_draft["tokens"][idx, :ag]):
            tally.failures.append(("prefix", int(b)))
        if np.any(gpu["out_tokens"][idx, ag + 1:] != -1):
            tally.failures.append(("padding", int(b)))
    # final token, teacher-forced on the GPU's acceptance count
    vo2 = oracle.verify(rows, rs, draft_oracle["z"], draft_oracle["lse"], draft_oracle["q_tok"],
                        gpu_draft["tokens"], verify_len, inp["u_accept"], inp["u_resample"],
                        forced_accepted=_full(acc_g, requests, B), requests=requests)
    for idx, b in enumerate(requests):
        m = vo2["final_margin"][idx]
        tally.flagged += int(m < MARGIN)
        fg = int(gpu["out_tokens"][idx, acc_g[idx]])
        exc = 0
        if fg != int(vo2["final"][idx]):
            if m < MARGIN:
                exc = 1
            else:
                tally.failures.append(("final", int(b), int(vo2["final"][idx]), fg, float(m), vo2["final_mode"][idx]))
        tally.count("final", 1, exc)
    return vo2


def _full(vals, requests, B):
    out = np.zeros(B, np.int64)
    out[np.asarray(requests)] = vals
    return out


def gpu_round(inp, requests=None, packed=False, bufs=None, variant="a"):
    """Run draft -> schedule -> verify through the library; numpy outputs.
    `bufs` (optional) reuses the outputs and workspace of an earlier round;
    variant "b" stores no z (the draft returns the operand rows instead)."""
    from speculative_decoding_semi_b200 import round as rnd

    B, K, V = inp["base"].shape
    r = inp["A"].shape[1]
    d = rnd.to_device(inp)
    if bufs is None:
        bufs = rnd.RoundBuffers(B, K, V, r, variant=variant)
    rnd.draft(d, bufs)
    rnd.schedule(d, bufs)
    if packed:
        L = bufs.verify_len.cpu().numpy()
        rs = bufs.row_start.cpu().numpy()
        tgt = torch.from_numpy(synth.pack_rows(inp["target"], L, rs)).cuda()
        rnd.verify(d, bufs, target=tgt, row_start=bufs.row_start)
    else:
        rnd.verify(d, bufs)
    torch.cuda.synchronize()
    from speculative_decoding_semi_b200 import dspark_read_device_error
    st, detail = dspark_read_device_error(bufs.workspace)
    assert st == 0, (st, hex(detail))
    reqs = np.arange(B) if requests is None else np.asarray(requests)
    ridx = torch.as_tensor(reqs, device=bufs.draft_tokens.device)
    take = lambda t: t.index_select(0, ridx).cpu().numpy()
    keep_z = bufs.z is not None and len(reqs) * K * V <= 64 * 16 * 151936
    out = {
        "draft": {"tokens": take(bufs.draft_tokens), "q_tok": take(bufs.q_tok), "lse_q": take(bufs.lse_q),
                  "z": take(bufs.z) if keep_z else None,
                  "op_rows": (take(bufs.op_rows.view(torch.int16)).view(np.uint16)
                              if bufs.op_rows is not None else None)},
        "schedule": {"verify_len": bufs.verify_len.cpu().numpy(), "survival": bufs.survival.cpu().numpy(),
                     "row_start": bufs.row_start.cpu().numpy(), "n_tokens": bufs.n_tokens.cpu().numpy()[0]},
        "verify": {"accepted": take(bufs.accepted), "out_tokens": take(bufs.out_tokens), "n_out": take(bufs.n_out)},
    }
    return out


def compare_round(inp, g, reqs, tally: Tally, check_z=True):
    """Compare one round's GPU outputs `g` (as gpu_round returns them) with
    the oracle on the same inputs."""
    d = compare_draft(inp, g["draft"], reqs, tally, check_z=check_z and g["draft"].get("z") is not None)
    compare_schedule(inp, g["schedule"], tally)
    compare_verify(inp, d, g["draft"], g["verify"], g["schedule"]["verify_len"], reqs, tally)


def check_op_rows(inp, gpu_draft, requests, tally: Tally):
    """Variant B: the operand row of position i must be A[t_{i-1}] bit for bit
    (t_{-1} the anchor) for the Markov head; for the RNN head the oracle's
    state h_i (teacher-forced on the GPU's tokens) rounded to bf16, within one
    bf16 step (the two fp64 states differ by rounding)."""
    rows = gpu_draft["op_rows"]
    toks = gpu_draft["tokens"].astype(np.int64)
    anchor = np.asarray(inp["anchor"])[requests].astype(np.int64)
    prev = np.concatenate([anchor[:, None], toks[:, :-1]], axis=1)
    if inp.get("W") is None:
        want = np.asarray(inp["A"])[prev]
        bad = np.argwhere(np.any(rows != want, axis=-1))
        if len(bad):
            tally.failures.append(("op_rows", [tuple(int(x) for x in b) for b in bad[:5]]))
        return
    d = oracle.rnn_draft(inp["base"][requests], inp["A"], inp["W"], inp["Bf"], anchor, inp["u_draft"][requests],
                         teacher=toks, keep_z=False)
    want = oracle.round_to_bf16(d["h"])
    got = synth.bf16_bits_to_f32(rows).astype(np.float64)
    step = np.abs(want) * 2.0 ** -7 + 1e-40
    err = np.abs(got - want) / step
    if err.max() > 1.0 + 1e-9:
        tally.failures.append(("op_rows rnn", float(err.max())))


def check_round(inp, requests=None, packed=False, tally: Tally | None = None, check_z=True, bufs=None,
                variant="a"):
    B = inp["base"].shape[0]
    reqs = np.arange(B) if requests is None else np.asarray(requests)
    g = gpu_round(inp, reqs, packed=packed, bufs=bufs, variant=variant)
    t = Tally() if tally is None else tally
    compare_round(inp, g, reqs, t, check_z=check_z)
    if g["draft"]["op_rows"] is not None:
        check_op_rows(inp, g["draft"], reqs, t)
    return t, g
