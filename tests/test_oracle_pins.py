"""Pins of the CPU oracle to facts that do not come from the oracle itself.

- losslessness: exhaustive enumeration at V=8 (the pages' claim that
  verification keeps the target distribution exactly);
- zero Markov factors reduce the draft to independent per-position sampling
  (numpy searchsorted on a scipy softmax);
- the bias equals a brute-force fp64 triple loop;
- the scheduler equals brute force over every length assignment;
- survival closed forms and a scipy cross-check;
- inverse-CDF boundary cases.
"""
import itertools

import numpy as np
import pytest
import scipy.special

import oracle
import synth
from tests import enumeration as en


@pytest.fixture(scope="module")
def prob():
    return en.make_problem()


@pytest.mark.parametrize("L", [0, 1, 2, 3])
def test_lossless_exhaustive_v8(prob, L):
    batch = en.build_batch(prob, L)
    n = len(batch["weight"])
    rows = batch["target"].reshape(n * (en.K + 1), en.V)
    rs = np.arange(n, dtype=np.int64) * (en.K + 1)
    d = oracle.draft(batch["base"], prob["A"], prob["Bf"], batch["anchor"], batch["u_draft"])
    # every draft uniform is the midpoint of its path's interval
    assert np.array_equal(d["t"], batch["path"])
    v = oracle.verify(rows, rs, d["z"], d["lse"], d["q_tok"], d["t"], batch["verify_len"],
                      batch["u_accept"], batch["u_resample"])
    assert np.all((v["n_out"] >= 1) & (v["n_out"] <= L + 1))
    assert np.all(v["n_out"] == v["accepted"] + 1)
    for i in range(n):
        a = v["accepted"][i]
        assert np.array_equal(v["out_tokens"][i, :a], batch["path"][i, :a])
    joint = en.tally(batch, v["out_tokens"], v["n_out"])
    en.check_lossless(prob, batch, joint)
    en.check_accept_rate(prob, batch, v["accepted"])


def test_lossless_detects_wrong_residual(prob, monkeypatch):
    """A plausible mistake (resampling from p instead of max(0,p-q)) must fail the pin."""
    batch = en.build_batch(prob, 2)
    n = len(batch["weight"])
    rows = batch["target"].reshape(n * (en.K + 1), en.V)
    rs = np.arange(n, dtype=np.int64) * (en.K + 1)
    d = oracle.draft(batch["base"], prob["A"], prob["Bf"], batch["anchor"], batch["u_draft"])
    real_softmax = oracle.softmax
    # planted mistake: the residual subtracts q of the wrong position (zero vector)
    monkeypatch.setattr(oracle, "softmax", lambda z: real_softmax(z) if np.ndim(z) > 1 else np.zeros_like(z))
    v = oracle.verify(rows, rs, d["z"], d["lse"], d["q_tok"], d["t"], batch["verify_len"],
                      batch["u_accept"], batch["u_resample"])
    joint = en.tally(batch, v["out_tokens"], v["n_out"])
    with pytest.raises(AssertionError):
        en.check_lossless(prob, batch, joint)


def test_zero_factors_is_independent_sampling():
    rng = np.random.default_rng(3)
    B, K, V, r = 6, 5, 257, 4
    base = rng.normal(0, 2, size=(B, K, V)).astype(np.float32)
    u = rng.random(size=(B, K), dtype=np.float32)
    anchor = rng.integers(0, V, size=B).astype(np.int32)
    for A, Bf in ((np.zeros((V, r), np.float32), rng.normal(size=(r, V)).astype(np.float32)),
                  (rng.normal(size=(V, r)).astype(np.float32), np.zeros((r, V), np.float32))):
        d = oracle.draft(base, A, Bf, anchor, u)
        for b in range(B):
            for i in range(K):
                q = scipy.special.softmax(base[b, i].astype(np.float64))
                cdf = np.cumsum(q)
                expect = int(np.searchsorted(cdf, float(u[b, i]) * cdf[-1], side="right"))
                assert d["t"][b, i] == expect
                assert abs(d["q_tok"][b, i] - q[expect]) < 1e-12
                lse = scipy.special.logsumexp(base[b, i].astype(np.float64))
                assert abs(d["lse"][b, i] - lse) < 1e-12


def test_bias_brute_force():
    rng = np.random.default_rng(4)
    B, V, r = 3, 7, 5
    A = rng.normal(size=(V, r)).astype(np.float32)
    Bf = rng.normal(size=(r, V)).astype(np.float32)
    t = np.array([6, 0, 3])
    got = oracle.markov_bias(A.astype(np.float64), Bf.astype(np.float64), t)
    for b in range(B):
        for v in range(V):
            acc = 0.0
            for k in range(r):
                acc += float(A[t[b], k]) * float(Bf[k, v])
            assert abs(got[b, v] - acc) < 1e-12


def test_bias_changes_tokens_under_stress_factors():
    """With factors ~N(0,0.3) dropping the bias must change most draws."""
    rng = np.random.default_rng(5)
    B, K, V, r = 16, 4, 512, 16
    base = rng.normal(0, 2, size=(B, K, V)).astype(np.float32)
    A = rng.normal(0, 0.3, size=(V, r)).astype(np.float32)
    Bf = rng.normal(0, 0.3, size=(r, V)).astype(np.float32)
    u = rng.random(size=(B, K), dtype=np.float32)
    anchor = rng.integers(0, V, size=B).astype(np.int32)
    with_bias = oracle.draft(base, A, Bf, anchor, u)["t"]
    without = oracle.draft(base, np.zeros_like(A), Bf, anchor, u)["t"]
    assert np.mean(with_bias != without) > 0.5


def test_bf16_widening_exact():
    x = np.array([1.0, -2.5, 3.140625, 1e-3], np.float32)
    bits = synth.f32_to_bf16_bits(x)
    back = oracle.bf16_to_f64(bits)
    assert back[0] == 1.0 and back[1] == -2.5 and back[2] == 3.140625
    assert abs(back[3] - 1e-3) / 1e-3 < 2 ** -8


def _brute_schedule(P, T):
    B, K = P.shape
    best, best_L = -np.inf, None
    for L in itertools.product(range(K + 1), repeat=B):
        n = B + sum(L)
        if n > len(T):
            continue
        S = sum(P[b, :L[b]].sum() for b in range(B))
        obj = (B + S) / T[n - 1]
        if obj > best:
            best, best_L = obj, L
    return best, best_L


@pytest.mark.parametrize("seed", range(12))
def test_schedule_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 5))
    K = int(rng.integers(1, 5))
    conf = rng.normal(1, 1.5, size=(B, K))
    temps = 1 + 0.1 * np.arange(1, K + 1)
    P = oracle.survival(conf, temps)
    n_prof = B * (K + 1) + int(rng.integers(0, 3))
    kind = seed % 3
    n = np.arange(1, n_prof + 1)
    if kind == 0:
        T = 1 + rng.uniform(0, 0.3) * np.maximum(n - rng.integers(1, n_prof), 0)
    elif kind == 1:
        T = 1 + 0.05 * n + 0.2 * rng.random(n_prof)   # non-monotone
    else:
        T = rng.uniform(0.5, 2.0, size=n_prof)        # arbitrary
    s = oracle.schedule(P, T)
    best, _ = _brute_schedule(P, T)
    got = s["objective"][s["m_star"]]
    assert abs(got - best) <= 1e-12 * best
    L = s["verify_len"]
    assert L.sum() == s["m_star"]
    assert abs((B + sum(P[b, :L[b]].sum() for b in range(B))) / T[B + L.sum() - 1] - best) <= 1e-12 * best
    assert np.array_equal(s["row_start"], np.concatenate([[0], np.cumsum(L + 1)[:-1]]))
    assert s["n_tokens"] == int((L + 1).sum())


def test_schedule_flat_profile_takes_everything():
    rng = np.random.default_rng(1)
    B, K = 5, 16
    P = oracle.survival(rng.normal(1, 1, size=(B, K)), 1 + 0.1 * np.arange(1, K + 1))
    s = oracle.schedule(P, np.ones(2048))
    assert np.all(s["verify_len"] == K)


def test_schedule_single_request_is_argmax():
    P = np.array([[0.9, 0.5, 0.1]])
    T = np.array([1.0, 1.2, 1.5, 2.5])   # T(1..4)
    s = oracle.schedule(P, T)
    objs = [(1 + P[0, :L].sum()) / T[L] for L in range(4)]
    assert s["verify_len"][0] == int(np.argmax(objs))


@pytest.mark.parametrize("seed", range(6))
def test_schedule_steeper_profile_never_lengthens(seed):
    rng = np.random.default_rng(200 + seed)
    B, K = 8, 6
    P = oracle.survival(rng.normal(1, 1, size=(B, K)), 1 + 0.1 * np.arange(1, K + 1))
    n = np.arange(1, 200)
    T = 1 + 0.01 * np.maximum(n - 20, 0)
    g = np.maximum.accumulate(1 + rng.random(n.size) * 0.05 * (n / n.size))
    a = oracle.schedule(P, T)["verify_len"].sum()
    b = oracle.schedule(P, T * g)["verify_len"].sum()
    assert b <= a


def test_survival_closed_forms_and_scipy():
    K = 6
    temps = 1 + 0.1 * np.arange(1, K + 1)
    P0 = oracle.survival(np.zeros((1, K)), temps)
    assert np.array_equal(P0[0], 0.5 ** np.arange(1, K + 1))
    Pbig = oracle.survival(np.full((1, K), 1e4), temps)
    assert np.all(Pbig == 1.0)
    rng = np.random.default_rng(9)
    conf = rng.normal(1, 2, size=(7, K))
    P = oracle.survival(conf, temps)
    ref = np.cumprod(scipy.special.expit(conf / temps[None, :]), axis=1)
    assert np.max(np.abs(P - ref) / ref) < 1e-14
    assert np.all(np.diff(P, axis=1) <= 0)


def test_icdf_boundaries():
    w = np.array([0.0, 1.0, 0.0, 1.0])
    k, m = oracle.icdf(w, np.float32(0.0))
    assert k[0] == 1 and m[0] == 0.0
    k, m = oracle.icdf(w, np.float32(0.5))
    assert k[0] == 3 and m[0] == 0.0          # exactly on a boundary: margin 0, strict '>'
    k, m = oracle.icdf(w, np.float32(0.25))
    assert k[0] == 1 and abs(m[0] - 0.25) < 1e-15
    k, _ = oracle.icdf(np.array([0.0, 0.0, 3.0, 0.0]), np.float32(0.9999999))
    assert k[0] == 2
    rng = np.random.default_rng(2)
    for _ in range(50):
        w = rng.random(33) * (rng.random(33) > 0.3)
        u = rng.random(dtype=np.float32)
        C = np.cumsum(w)
        k, _ = oracle.icdf(w, u)
        assert k[0] == np.searchsorted(C, float(u) * C[-1], side="right")
        assert w[k[0]] > 0


def test_verify_special_cases():
    rng = np.random.default_rng(11)
    B, K, V = 6, 4, 50
    z = rng.normal(0, 2, size=(B, K, V))
    tokens = rng.integers(0, V, size=(B, K))
    lse = scipy.special.logsumexp(z, axis=-1)
    q_tok = np.exp(np.take_along_axis(z, tokens[..., None], -1)[..., 0] - lse)
    # target rows equal to the draft rows: everything is accepted, bonus from row L_b
    rows = np.concatenate([z, rng.normal(size=(B, 1, V))], axis=1).reshape(B * (K + 1), V)
    rs = np.arange(B) * (K + 1)
    L = np.array([0, 1, 2, 3, 4, 4])
    ua = rng.random(size=(B, K), dtype=np.float32)
    ur = rng.random(size=B, dtype=np.float32)
    v = oracle.verify(rows, rs, z, lse, q_tok, tokens, L, ua, ur)
    assert np.array_equal(v["accepted"], L)
    for b in range(B):
        p = scipy.special.softmax(rows[rs[b] + L[b]])
        cdf = np.cumsum(p)
        assert v["final"][b] == np.searchsorted(cdf, float(ur[b]) * cdf[-1], side="right")
        assert np.array_equal(v["out_tokens"][b, :L[b]], tokens[b, :L[b]])
