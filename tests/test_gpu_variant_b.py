"""Variant B of the round on the GPU (no stored z; the rejected row of z
recomputed on the tensor cores) against the CPU oracle.

The oracle is the same as for variant A: the method's definition does not
change, only where z lives. Cases: shapes with ragged last tiles and
vocabulary slices of one quadrant; batches whose rejected requests fill one,
two and four residual groups (N = 128 per group); no rejected request at all;
one request with one position; the RNN head; packed ragged
target rows; full-size workloads on sampled requests; extreme logits (p
weighed with the row's own shift; the slow redraw of a draft row beyond the
fixed-shift range without stored z); and variant A and B on the same inputs.
"""
import numpy as np
import pytest
import torch

import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("like,sizes", [
    (1, dict(B=12, K=5, V=37024, r=64, n_prof=256)),
    (1, dict(B=3, K=2, V=96, r=256, n_prof=16)),
    (1, dict(B=17, K=4, V=4096, r=192, n_prof=80)),
    (1, dict(B=3, K=16, V=4128, r=256, n_prof=64)),
    # residual groups: up to 128 rejected requests per MMA, so these batches
    # use two groups
    (3, dict(B=256, K=4, V=8192, r=64, n_prof=1280)),
    (4, dict(B=512, K=2, V=4096, r=64, n_prof=1600)),
    (1, dict(B=130, K=3, V=8192, r=128, n_prof=600)),
    (1, dict(B=3, K=32, V=2048, r=64, n_prof=128)),
])
def test_variant_b_matches_oracle(like, sizes):
    t = parity.Tally()
    w = synth.custom(like, **sizes)
    for seed in range(3):
        parity.check_round(synth.make_round(w, seed=310 + seed), tally=t, variant="b")
    t.check(f"variant b {sizes}")


def test_variant_b_four_residual_groups():
    """More than 384 rejected requests (four residual groups of up to 128):
    a flat profile verifies every position and u_accept near 1 rejects a draft
    whenever p(t) < q(t), about half of them at each position."""
    w = synth.custom(2, B=512, K=4, V=4096, r=64, n_prof=2600)
    t = parity.Tally()
    inp = synth.make_round(w, seed=320)
    inp["u_accept"] = np.full_like(inp["u_accept"], 0.9999)
    _, g = parity.check_round(inp, tally=t, variant="b")
    L = g["schedule"]["verify_len"]
    rejected = int(np.sum(g["verify"]["accepted"] < L))
    assert rejected > 384, rejected
    t.check("variant b four groups")


@pytest.mark.parametrize("sizes,wstd", [
    (dict(B=6, K=5, V=8192, r=64, n_prof=64), 0.05),
    (dict(B=40, K=4, V=16384, r=128, n_prof=256), 0.02),
])
def test_variant_b_rnn_head(sizes, wstd):
    t = parity.Tally()
    w = synth.custom(1, **sizes)
    for seed in range(2):
        inp = synth.make_round(w, seed=330 + seed)
        rng = np.random.default_rng(330 + seed)
        inp["W"] = synth.f32_to_bf16_bits(rng.standard_normal((w.r, w.r), dtype=np.float32) * np.float32(wstd))
        parity.check_round(inp, tally=t, variant="b")
    t.check(f"variant b rnn {sizes}")


def test_variant_b_packed_target_rows():
    w = synth.custom(1, B=16, K=6, V=12352, r=64, n_prof=80)
    t = parity.Tally()
    for seed in range(2):
        parity.check_round(synth.make_round(w, seed=340 + seed), packed=True, tally=t, variant="b")
    t.check("variant b packed")


@pytest.mark.parametrize("key,sample", [("qwen3", 8), ("highconc", 6), ("mixed", 6), ("latency", 1)])
def test_variant_b_full_size(key, sample):
    t = parity.Tally()
    inp = synth.make_round(key)
    B = inp["base"].shape[0]
    reqs = np.unique(np.linspace(0, B - 1, sample).astype(int))
    parity.check_round(inp, requests=reqs, tally=t, variant="b")
    t.check(f"variant b {key}")


@pytest.mark.parametrize("key,seeds,sample", [("qwen3", 6, 8), ("latency", 40, None), ("highconc", 2, 16),
                                             ("mixed", 2, 16)])
def test_variant_b_seed_volume(key, seeds, sample):
    """More seeds of every full-size workload in variant B, the excused
    near-ties pooled; the Markov factors drawn once per workload."""
    t = parity.Tally()
    factors = synth.make_factors(key)
    for k in range(seeds):
        inp = synth.make_round(key, seed=7500 + k, factors=factors)
        B = inp["base"].shape[0]
        reqs = None if sample is None else np.unique(np.linspace(k % 3, B - 1, sample).astype(int))
        parity.check_round(inp, requests=reqs, tally=t, variant="b")
    t.check(f"variant b {key} x{seeds}")


def test_variant_b_agrees_with_variant_a():
    """Same inputs, both variants: the drafts are the same computation (z from
    the same tensor-core GEMM) and the verify outputs follow the definition, so
    every token agrees except where the oracle's margin is a near-tie."""
    w = synth.custom(1, B=64, K=8, V=32768, r=256, n_prof=2048)
    differ = total = 0
    for seed in range(3):
        inp = synth.make_round(w, seed=350 + seed)
        ga = parity.gpu_round(inp, variant="a")
        gb = parity.gpu_round(inp, variant="b")
        np.testing.assert_array_equal(ga["schedule"]["verify_len"], gb["schedule"]["verify_len"])
        same = np.all(ga["draft"]["tokens"] == gb["draft"]["tokens"], axis=1)
        same &= np.all(ga["verify"]["out_tokens"] == gb["verify"]["out_tokens"], axis=1)
        same &= ga["verify"]["n_out"] == gb["verify"]["n_out"]
        differ += int(np.sum(~same))
        total += same.size
    assert differ <= 1, (differ, total)


def test_variant_b_extreme_logits():
    """Draft rows whose exp(z) leaves fp32's range and target rows far above
    and below the fixed shift: variant B weighs p with the row's own base-2
    log-sum as the shift."""
    w = synth.custom(1, B=6, K=4, V=8192, r=64, n_prof=64)
    t = parity.Tally()
    for seed in range(2):
        inp = synth.make_round(w, seed=900 + seed)
        base = inp["base"].copy()
        tgt = inp["target"].copy()
        base[0] += 90.0
        base[1, 1] -= 150.0
        tgt[2] += 90.0
        tgt[3, 0] -= 150.0
        inp["base"], inp["target"] = base, tgt
        parity.check_round(inp, tally=t, variant="b")
    t.check("variant b extreme logits")


def test_variant_b_rows_beyond_fp64_range():
    """As test_rows_beyond_fp64_range_are_redrawn for variant A: without stored
    z the draft redraws such a row from z recomputed one unit at a time. Valid
    tokens and no mismatch at a margin of 1e-5 or more."""
    w = synth.custom(1, B=6, K=4, V=8192, r=64, n_prof=64)
    t = parity.Tally()
    for seed in range(2):
        inp = synth.make_round(w, seed=950 + seed)
        base = inp["base"].copy()
        base[4, 2] += 720.0
        base[5, 3] -= 800.0
        inp["base"] = base
        _, g = parity.check_round(inp, tally=t, variant="b")
        toks = g["draft"]["tokens"]
        assert np.all((toks >= 0) & (toks < w.V))
    assert not t.failures, t.failures[:10]


def test_variant_b_no_residual():
    """Nothing to resample: every verify length 0 (a profile that makes any
    verified token too expensive), and every draft accepted (u_accept = 0);
    the residual kernel then has no group and only the bonus draws remain."""
    w = synth.custom(1, B=10, K=4, V=4096, r=64, n_prof=40)
    inp = synth.make_round(w, seed=3)
    inp["profile"] = (1.0 + 1000.0 * np.maximum(np.arange(1, 41) - 10, 0)).astype(np.float32)
    t, g = parity.check_round(inp, variant="b")
    t.check()
    assert np.all(g["schedule"]["verify_len"] == 0)
    assert np.all(g["verify"]["n_out"] == 1)
    inp = synth.make_round(w, seed=4)
    inp["u_accept"] = np.zeros_like(inp["u_accept"])
    t, g = parity.check_round(inp, variant="b")
    t.check()
    assert np.all(g["verify"]["accepted"] == g["schedule"]["verify_len"])


def test_variant_b_single_request():
    for V in (64, 151936):
        w = synth.custom(1, B=1, K=1, V=V, r=64, n_prof=4)
        t = parity.Tally()
        for seed in range(3):
            parity.check_round(synth.make_round(w, seed=seed), tally=t, variant="b")
        t.check()


def test_variant_b_unsupported_shapes():
    from speculative_decoding_semi_b200 import DSparkError, round as rnd
    w = synth.custom(1, B=4, K=2, V=1024, r=32, n_prof=32)  # r not a multiple of 64
    inp = synth.make_round(w, seed=1)
    d = rnd.to_device(inp)
    bufs = rnd.RoundBuffers(4, 2, 1024, 32, variant="b")
    with pytest.raises(DSparkError) as e:
        rnd.draft(d, bufs)
    assert e.value.status == 2
    torch.cuda.synchronize()
