"""Invariants of the CPU oracle's bookkeeping, which the GPU parity tests lean on.

- Verifying a sample of requests (the per-request draft arrays given for the
  sample only, the batch-wide arrays indexed by request) gives, for each
  sampled request, what verifying the whole batch gives.
- Target rows packed by the scheduler's row offsets (a ragged verify batch)
  give the same outputs as the dense [B, K+1, V] layout.
- When the adjusted distribution max(0, p - q) vanishes (target row equal to
  the draft row) the final token comes from p, as the reading of the
  wangjunjian.com "Speculative Decoding" article, step 4, takes it: checked
  against a scipy softmax and numpy searchsorted.
- A round over a sample of requests equals the full round at those requests.
"""
import numpy as np
import scipy.special

import oracle
import synth


def _small(seed, B=7, K=4, V=64, r=8):
    w = synth.custom(0, B=B, K=K, V=V, r=r, n_prof=B * (K + 1) + 3)
    inp = synth.make_round(w, seed=seed)
    # a flat profile verifies every position, so that rejections occur
    inp["profile"] = np.ones(w.n_prof, np.float32)
    return inp


def _verify_full(inp):
    B, K, V = inp["base"].shape
    d = oracle.draft(inp["base"], inp["A"], inp["Bf"], inp["anchor"], inp["u_draft"])
    s = oracle.schedule(oracle.survival(inp["conf"], inp["temps"]), inp["profile"])
    rows = inp["target"].reshape(B * (K + 1), V)
    rs = synth.dense_row_start(B, K)
    v = oracle.verify(rows, rs, d["z"], d["lse"], d["q_tok"], d["t"], s["verify_len"],
                      inp["u_accept"], inp["u_resample"])
    return d, s, v


def test_verify_on_a_request_sample_matches_the_full_batch():
    for seed in range(4):
        inp = _small(seed)
        B, K, V = inp["base"].shape
        d, s, v = _verify_full(inp)
        assert np.any(v["accepted"] < s["verify_len"])      # some rejections
        reqs = np.array([6, 1, 4])
        rows = inp["target"].reshape(B * (K + 1), V)
        vs = oracle.verify(rows, synth.dense_row_start(B, K), d["z"][reqs], d["lse"][reqs], d["q_tok"][reqs],
                           d["t"][reqs], s["verify_len"], inp["u_accept"], inp["u_resample"], requests=reqs)
        for key in ("accepted", "final", "n_out"):
            np.testing.assert_array_equal(vs[key], v[key][reqs], err_msg=key)
        np.testing.assert_array_equal(vs["out_tokens"], v["out_tokens"][reqs])


def test_packed_rows_match_the_dense_layout():
    for seed in range(4):
        inp = _small(10 + seed)
        B, K, V = inp["base"].shape
        d, s, v = _verify_full(inp)
        packed = synth.pack_rows(inp["target"], s["verify_len"], s["row_start"])
        assert packed.shape[0] == s["n_tokens"]
        vp = oracle.verify(packed, s["row_start"], d["z"], d["lse"], d["q_tok"], d["t"], s["verify_len"],
                           inp["u_accept"], inp["u_resample"])
        for key in ("accepted", "final", "n_out"):
            np.testing.assert_array_equal(vp[key], v[key], err_msg=key)
        np.testing.assert_array_equal(vp["out_tokens"], v["out_tokens"])


def test_vanished_residual_falls_back_to_the_target():
    rng = np.random.default_rng(31)
    B, K, V = 5, 3, 40
    z = rng.normal(0, 2, size=(B, K, V))
    tokens = rng.integers(0, V, size=(B, K))
    lse = scipy.special.logsumexp(z, axis=-1)
    q_tok = np.exp(np.take_along_axis(z, tokens[..., None], -1)[..., 0] - lse)
    # target rows 0..K-1 equal the draft rows: p = q, so max(0, p - q) is zero
    rows = np.concatenate([z, rng.normal(0, 2, size=(B, 1, V))], axis=1).reshape(B * (K + 1), V)
    rs = np.arange(B) * (K + 1)
    L = np.full(B, K)
    ur = rng.random(size=B, dtype=np.float32)
    forced = np.array([0, 1, 2, 1, 0])
    v = oracle.verify(rows, rs, z, lse, q_tok, tokens, L, np.zeros((B, K), np.float32), ur,
                      forced_accepted=forced)
    for b in range(B):
        f = forced[b]
        assert v["final_mode"][b] == "residual_fallback"
        p = scipy.special.softmax(z[b, f])
        cdf = np.cumsum(p)
        assert v["final"][b] == np.searchsorted(cdf, float(ur[b]) * cdf[-1], side="right")
        assert v["n_out"][b] == f + 1
        np.testing.assert_array_equal(v["out_tokens"][b, :f], tokens[b, :f])


def test_round_on_a_request_sample_matches_the_full_round():
    inp = _small(40, B=9)
    full = oracle.run_round(inp)
    reqs = np.array([0, 5, 8])
    part = oracle.run_round(inp, requests=reqs)
    np.testing.assert_array_equal(part["schedule"]["verify_len"], full["schedule"]["verify_len"])
    np.testing.assert_array_equal(part["draft"]["t"], full["draft"]["t"][reqs])
    np.testing.assert_array_equal(part["draft"]["q_tok"], full["draft"]["q_tok"][reqs])
    np.testing.assert_array_equal(part["verify"]["out_tokens"], full["verify"]["out_tokens"][reqs])
    np.testing.assert_array_equal(part["verify"]["n_out"], full["verify"]["n_out"][reqs])
