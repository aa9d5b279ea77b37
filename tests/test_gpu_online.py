"""The steps between rounds on the device, against the oracle.

- dspark_calibrate (online sequential temperature scaling) against
  oracle.calibrate, step by step, on outcomes of every kind;
- dspark_advance_anchor (the next round's anchors) exactly;
- rounds chained on the device with no host synchronisation (draft ->
  schedule -> verify -> calibrate -> next anchors), as launches and as one
  captured CUDA graph: every round matches the oracle given that round's
  anchors and temperatures, and the anchors and temperatures handed to the
  next round are the ones the oracle's rules give.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

CAL = (0.05, 0.05, 20.0)   # eta, t_min, t_max


def _ws():
    from speculative_decoding_semi_b200 import binding
    ws = torch.empty(binding.dspark_workspace_bytes(8, 8, 64, 8), dtype=torch.uint8, device="cuda")
    binding.dspark_workspace_init(ws)
    return ws


@pytest.mark.parametrize("B,K", [(1, 1), (7, 4), (64, 8), (300, 16), (2, 32)])
def test_calibrate_matches_oracle(B, K):
    from speculative_decoding_semi_b200 import binding
    rng = np.random.default_rng(B * 100 + K)
    ws = _ws()
    temps = torch.tensor(1 + 0.1 * np.arange(1, K + 1), dtype=torch.float32, device="cuda")
    for step in range(5):
        conf = rng.normal(1.0, 2.0, size=(B, K)).astype(np.float32)
        L = rng.integers(0, K + 1, size=B).astype(np.int32)
        acc = np.minimum(rng.integers(0, K + 1, size=B), L).astype(np.int32)
        before = temps.cpu().numpy().astype(np.float64)
        binding.dspark_calibrate(torch.from_numpy(conf).cuda(), torch.from_numpy(L).cuda(),
                                 torch.from_numpy(acc).cuda(), temps, ws, *CAL)
        got = temps.cpu().numpy().astype(np.float64)
        want = oracle.calibrate(conf, before, L, acc, *CAL)
        assert np.all(np.abs(got - want) <= 1e-6 * np.abs(want)), (step, got, want)
    assert binding.dspark_read_device_error(ws)[0] == 0


def test_calibrate_reports_bad_counts():
    from speculative_decoding_semi_b200 import binding
    ws = _ws()
    conf = torch.zeros(3, 4, device="cuda")
    L = torch.tensor([1, 9, 2], dtype=torch.int32, device="cuda")     # 9 > K
    acc = torch.tensor([1, 0, 2], dtype=torch.int32, device="cuda")
    temps = torch.ones(4, device="cuda")
    binding.dspark_calibrate(conf, L, acc, temps, ws, *CAL)
    st, detail = binding.dspark_read_device_error(ws)
    assert st == 5 and detail == (0x50000000 | 1)


def test_advance_anchor():
    from speculative_decoding_semi_b200 import binding
    rng = np.random.default_rng(3)
    B, K = 37, 6
    out = rng.integers(0, 1000, size=(B, K + 1)).astype(np.int32)
    n = rng.integers(1, K + 2, size=B).astype(np.int32)
    anchor = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    ws = _ws()
    binding.dspark_advance_anchor(torch.from_numpy(out).cuda(), torch.from_numpy(n).cuda(), anchor, ws)
    assert np.array_equal(anchor.cpu().numpy(), out[np.arange(B), n - 1])
    assert binding.dspark_read_device_error(ws)[0] == 0


@pytest.mark.parametrize("graph", [False, True])
def test_rounds_chained_on_the_device(graph):
    from speculative_decoding_semi_b200 import round as rnd
    w = synth.custom(1, B=16, K=6, V=16384, r=64, n_prof=128)
    factors = synth.make_factors(w)
    host = [synth.make_round(w, seed=400 + k, factors=factors) for k in range(3)]
    dev = [rnd.to_device(h) for h in host]
    bufs = rnd.RoundBuffers(w.B, w.K, w.V, w.r)
    state = rnd.RoundState(dev[0]["anchor"], dev[0]["temps"])
    R = 7
    if graph:   # one eager round first: the library's first launches set kernel attributes
        rnd.run_rounds(dev, bufs, rnd.RoundState(dev[0]["anchor"], dev[0]["temps"]), 1, calibrate=CAL, record=False)
    hist = rnd.run_rounds(dev, bufs, state, R, calibrate=CAL, graph=graph)
    torch.cuda.synchronize()
    from speculative_decoding_semi_b200 import dspark_read_device_error
    assert dspark_read_device_error(bufs.workspace)[0] == 0
    H = {k: v.cpu().numpy() for k, v in hist.items() if k != "graph"}
    t = parity.Tally()
    reqs = np.arange(w.B)
    for r in range(R):
        inp = dict(host[r % len(host)])
        inp["anchor"], inp["temps"] = H["anchor"][r], H["temps"][r]
        g = {"draft": {"tokens": H["draft_tokens"][r], "q_tok": H["q_tok"][r], "lse_q": H["lse_q"][r]},
             "schedule": {"verify_len": H["verify_len"][r], "survival": H["survival"][r],
                          "row_start": H["row_start"][r], "n_tokens": H["n_tokens"][r][0]},
             "verify": {"accepted": H["accepted"][r], "out_tokens": H["out_tokens"][r], "n_out": H["n_out"][r]}}
        parity.compare_round(inp, g, reqs, t, check_z=False)
        # what this round hands to the next one
        nxt_anchor = H["out_tokens"][r][reqs, H["n_out"][r] - 1]
        nxt_temps = oracle.calibrate(inp["conf"], H["temps"][r].astype(np.float64), H["verify_len"][r],
                                     H["accepted"][r], *CAL)
        after_anchor = H["anchor"][r + 1] if r + 1 < R else state.anchor.cpu().numpy()
        after_temps = H["temps"][r + 1] if r + 1 < R else state.temps.cpu().numpy()
        assert np.array_equal(after_anchor, nxt_anchor), r
        assert np.all(np.abs(after_temps - nxt_temps) <= 1e-6 * nxt_temps), (r, after_temps, nxt_temps)
    t.check(f"rounds chained on the device (graph={graph})")
    # the loop did move the state
    assert not np.array_equal(H["anchor"][0], H["anchor"][-1])
    assert not np.allclose(H["temps"][0], H["temps"][-1])


def test_profile_builder_feeds_the_scheduler():
    """A T(n) table measured on this device (the library's draft, schedule and
    verify of n packed rows) is positive, non-decreasing and drives
    dspark_schedule, which then agrees with the oracle on it."""
    from speculative_decoding_semi_b200.profile import build_profile
    w = synth.custom(1, B=16, K=6, V=16384, r=64, n_prof=128)
    inp = synth.make_round(w, seed=5)
    prof = build_profile(inp, n_prof=128, points=5, reps=3)
    tab = prof["table"]
    assert tab.shape == (128,) and np.all(np.isfinite(tab)) and np.all(tab > 0)
    assert np.all(np.diff(tab) >= 0)
    assert prof["grid"][0] == 16 and prof["grid"][-1] == 16 * 7
    inp["profile"] = tab
    t, _ = parity.check_round(inp)
    t.check()
