"""Pins of the CPU oracle to facts that do not come from the oracle itself.

- losslessness: exhaustive enumeration at V=8 (the pages' claim that
  verification keeps the target distribution exactly), with the draft
  intervals built independently of the oracle so that its chain is checked;
- the draft's chain across positions: factors that force t_i = f(t_{i-1})
  (the bias comes from the previous token, the anchor at position 1), with
  and without teacher forcing, and planted mistakes that must fail;
- verification with forced acceptance counts: the final token comes from the
  row after the accepted prefix, through max(0, p - q) or the bonus row;
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


# ---------------------------------------------------------------------------
# The draft's chain across positions. QbitAI article, section "a cheaper
# sequential module: the Markov head": the correction at a position depends on
# the token drawn just before it. Factors at the tiny workload's sizes (V=1024,
# r=32) are built so that A[t] . Bf adds +60 at exactly one token f(t) and 0
# everywhere else; with base logits ~N(0,2) that token then holds all but
# ~1e-20 of the mass, so any uniform in (0.001, 0.999) draws it and the chain
# is forced: t_1 = f(anchor), t_i = f(t_{i-1}).
CV, CR, CK, CB = 1024, 32, 6, 5


def _chain_target(k):
    """f's value for rank slot k: a token whose slot is k + 1 (mod r), so f
    iterated from any anchor walks through distinct tokens."""
    return CR * ((7 * k + 3) % CR) + (k + 1) % CR


def _chain_factors():
    A = np.zeros((CV, CR), np.float32)
    A[np.arange(CV), np.arange(CV) % CR] = 60.0          # A[t] = 60 e_{t mod r}
    Bf = np.zeros((CR, CV), np.float32)
    Bf[np.arange(CR), [_chain_target(k) for k in range(CR)]] = 1.0
    return A, Bf


def _f(t):
    return _chain_target(int(t) % CR)


def _chain_inputs(seed):
    rng = np.random.default_rng(seed)
    base = rng.normal(0, 2, size=(CB, CK, CV)).astype(np.float32)
    u = rng.uniform(0.001, 0.999, size=(CB, CK)).astype(np.float32)
    anchor = rng.integers(0, CV, size=CB).astype(np.int32)
    return base, u, anchor


def _expected_chain(anchor):
    out = np.empty((len(anchor), CK), np.int64)
    for b, a in enumerate(anchor):
        t = int(a)
        for i in range(CK):
            t = _f(t)
            out[b, i] = t
    return out


def _check_chain(d, base, anchor):
    exp = _expected_chain(anchor)
    assert np.array_equal(d["t"], exp)
    assert np.all(np.abs(d["q_tok"] - 1.0) < 1e-12)
    for b in range(CB):
        for i in range(CK):
            assert abs(d["lse"][b, i] - (60.0 + float(base[b, i, exp[b, i]]))) < 1e-12


@pytest.mark.parametrize("seed", range(3))
def test_draft_chain_follows_previous_token(seed):
    A, Bf = _chain_factors()
    base, u, anchor = _chain_inputs(seed)
    d = oracle.draft(base, A, Bf, anchor, u)
    _check_chain(d, base, anchor)
    # the chain's tokens are distinct from the first one: biasing every
    # position by the anchor would be visible
    assert np.all(d["t"][:, 1:] != d["t"][:, :1])


def test_draft_teacher_forcing_follows_the_teacher():
    """With a teacher path the bias at position i comes from teacher[i-1]
    (the anchor at i = 1): the oracle's own draw is f(teacher[i-1]) and q_tok
    is q at the teacher's token."""
    A, Bf = _chain_factors()
    base, u, anchor = _chain_inputs(11)
    rng = np.random.default_rng(12)
    teacher = rng.integers(0, CV, size=(CB, CK))
    chain = _expected_chain(anchor)
    teacher[teacher == chain] = (teacher[teacher == chain] + 1) % CV   # differs from the free chain
    d = oracle.draft(base, A, Bf, anchor, u, teacher=teacher)
    prev = np.concatenate([anchor[:, None].astype(np.int64), teacher[:, :-1]], axis=1)
    want = np.vectorize(_f)(prev)
    assert np.array_equal(d["t"], want)
    assert np.array_equal(d["chain"], teacher)
    for b in range(CB):
        for i in range(CK):
            top = want[b, i]
            if teacher[b, i] == top:
                continue
            q_expected = np.exp(float(base[b, i, teacher[b, i]]) - 60.0 - float(base[b, i, top]))
            assert abs(d["q_tok"][b, i] - q_expected) <= 1e-9 * q_expected


def _planted_draft_step(monkeypatch, mistake):
    real = oracle.draft_step
    first = {}

    def wrapped(base_i, A64, Bf64, t_prev, u):
        if mistake == "anchor":
            first.setdefault("t", np.array(t_prev))
            t_prev = first["t"]          # never moves past the anchor
        elif mistake == "no_bias":
            A64 = np.zeros_like(A64)
        return real(base_i, A64, Bf64, t_prev, u)

    monkeypatch.setattr(oracle, "draft_step", wrapped)


@pytest.mark.parametrize("mistake", ["anchor", "no_bias"])
def test_chain_pin_detects_planted_mistakes(monkeypatch, mistake):
    """Plausible mistakes in the chain (every position biased by the anchor;
    the bias dropped) must fail the chain pin."""
    A, Bf = _chain_factors()
    base, u, anchor = _chain_inputs(0)
    _planted_draft_step(monkeypatch, mistake)
    d = oracle.draft(base, A, Bf, anchor, u)
    with pytest.raises(AssertionError):
        _check_chain(d, base, anchor)


# ---------------------------------------------------------------------------
# Verification with a forced number of acceptances (teacher forcing of the
# final token). [Tags] "Speculative Decoding", steps 4-5: after the accepted
# prefix the next token comes from the target row after it (all accepted) or
# from the adjusted distribution max(0, p - q) at the first rejection. Target
# row rho holds two tokens d_rho < e_rho with +60 each (p = 1/2 on each); the
# draft row of the same position puts all its mass on e_rho. Then the
# residual max(0, p - q) is 1/2 on d_rho alone (final = d_f for a forced
# count f < L and any uniform), while the bonus (f = L) draws from both halves
# (u = 0.75 picks e_L).
FV, FK = 64, 4


def _forced_case():
    rng = np.random.default_rng(21)
    B = 1
    d_tok = np.array([3, 10, 17, 24, 31])
    e_tok = np.array([40, 45, 50, 55, 60])
    target = rng.normal(0, 2, size=(FK + 1, FV))
    target[np.arange(FK + 1), d_tok] = 60.0
    target[np.arange(FK + 1), e_tok] = 60.0
    z = rng.normal(0, 2, size=(B, FK, FV))
    z[0, np.arange(FK), e_tok[:FK]] = 60.0
    lse = scipy.special.logsumexp(z, axis=-1)
    tokens = np.array([[7, 8, 9, 11]])
    q_tok = np.exp(np.take_along_axis(z, tokens[..., None], -1)[..., 0] - lse)
    return target, z, lse, q_tok, tokens, d_tok, e_tok


def _check_forced(target, z, lse, q_tok, tokens, d_tok, e_tok):
    L = np.array([FK])
    for f in range(FK + 1):
        v = oracle.verify(target, np.array([0]), z, lse, q_tok, tokens, L,
                          np.full((1, FK), 0.5, np.float32), np.array([0.75], np.float32),
                          forced_accepted=np.array([f]))
        want = e_tok[FK] if f == FK else d_tok[f]
        assert v["final"][0] == want, (f, v["final"][0], want)
        assert v["n_out"][0] == f + 1
        assert np.array_equal(v["out_tokens"][0, :f], tokens[0, :f])
        assert v["out_tokens"][0, f] == want


def test_verify_forced_acceptances_draw_from_the_right_row():
    _check_forced(*_forced_case())


@pytest.mark.parametrize("mistake", ["q_dropped", "q_added", "row_off_by_one"])
def test_forced_pin_detects_planted_mistakes(monkeypatch, mistake):
    """Dropping q from the residual, adding it instead of subtracting it, or
    reading the row after the rejection must fail the forced-acceptance pin."""
    real = oracle.softmax
    if mistake == "q_dropped":
        monkeypatch.setattr(oracle, "softmax", lambda z: real(z) if np.ndim(z) > 1 else np.zeros_like(z))
    elif mistake == "q_added":
        # a sign error: the residual weights become max(0, p + q)
        monkeypatch.setattr(oracle, "softmax", lambda z: real(z) if np.ndim(z) > 1 else -real(z))
    else:
        monkeypatch.setattr(oracle, "softmax",
                            lambda z: real(np.roll(z, -1, axis=0)) if np.ndim(z) > 1 else real(z))
    with pytest.raises(AssertionError):
        _check_forced(*_forced_case())
