"""Pins of the oracle's RNN sequential head (host only).

- bf16 rounding from fp64 against a bit-level rounding of the fp64 value;
- W = 0 reduces the RNN head to the (pinned) Markov head with factors
  bf16(tanh(A));
- a tiny case against a brute-force recurrence written out here with scalar
  loops (math.tanh, term-by-term sums);
- the state carries the whole prefix: changing the anchor changes the bias
  at every later position, which the Markov head would not do beyond the first.
"""
import math
import struct

import numpy as np
import pytest

import oracle


def _bf16_bits_rne(x: float) -> float:
    """Round an fp64 value to bf16 by its bits: keep 1 + 7 mantissa bits (of
    52), round half to even on the dropped 45 bits, carry into the exponent."""
    (u,) = struct.unpack("<Q", struct.pack("<d", x))
    drop = 45
    low = u & ((1 << drop) - 1)
    u &= ~((1 << drop) - 1)
    half = 1 << (drop - 1)
    if low > half or (low == half and (u >> drop) & 1):
        u += 1 << drop
    return struct.unpack("<d", struct.pack("<Q", u))[0]


def test_round_to_bf16_matches_bit_rounding():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-3, 2000),
                         [0.0, 1.0, -1.0, 1.00390625, 1.005859375, 2.0 ** -20, 1 - 2 ** -30]])
    # exact ties: 1 + 2^-8 (between 1 and 1 + 2^-7) goes to even (1.0); 1 + 3 * 2^-8 goes up
    xs = np.concatenate([xs, [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)]])
    got = oracle.round_to_bf16(xs)
    for x, g in zip(xs, got):
        assert g == _bf16_bits_rne(float(x)), (x, g)
    assert oracle.round_to_bf16(np.array([1 + 2 ** -8]))[0] == 1.0


def test_zero_recurrence_is_the_markov_head():
    rng = np.random.default_rng(1)
    B, K, V, r = 5, 6, 300, 8
    base = rng.normal(0, 2, size=(B, K, V)).astype(np.float32)
    A = rng.normal(0, 0.5, size=(V, r)).astype(np.float32)
    Bf = rng.normal(0, 0.5, size=(r, V)).astype(np.float32)
    u = rng.random(size=(B, K), dtype=np.float32)
    anchor = rng.integers(0, V, size=B)
    d = oracle.rnn_draft(base, A, np.zeros((r, r)), Bf, anchor, u)
    m = oracle.draft(base, oracle.round_to_bf16(np.tanh(A.astype(np.float64))), Bf, anchor, u)
    assert np.array_equal(d["t"], m["t"])
    assert np.max(np.abs(d["z"] - m["z"])) < 1e-12
    assert np.max(np.abs(d["lse"] - m["lse"])) < 1e-12


def test_brute_force_recurrence():
    rng = np.random.default_rng(2)
    B, K, V, r = 2, 4, 11, 3
    base = rng.normal(0, 1, size=(B, K, V)).astype(np.float32)
    A = rng.normal(0, 0.8, size=(V, r)).astype(np.float32)
    W = rng.normal(0, 0.8, size=(r, r)).astype(np.float32)
    Bf = rng.normal(0, 0.8, size=(r, V)).astype(np.float32)
    u = rng.random(size=(B, K), dtype=np.float32)
    anchor = np.array([3, 7])
    d = oracle.rnn_draft(base, A, W, Bf, anchor, u)
    for b in range(B):
        h = [0.0] * r
        prev = int(anchor[b])
        for i in range(K):
            h = [math.tanh(float(A[prev, k]) + sum(float(W[k, m]) * h[m] for m in range(r))) for k in range(r)]
            hb = [_bf16_bits_rne(x) for x in h]
            z = [float(base[b, i, v]) + sum(hb[k] * float(Bf[k, v]) for k in range(r)) for v in range(V)]
            mx = max(z)
            w = [math.exp(x - mx) for x in z]
            tot = sum(w)
            thr = float(u[b, i]) * tot
            acc, t = 0.0, None
            for v in range(V):
                acc += w[v]
                if acc > thr:
                    t = v
                    break
            assert np.allclose(d["h"][b, i], h, rtol=0, atol=1e-14)
            assert d["t"][b, i] == t
            assert abs(d["lse"][b, i] - (mx + math.log(tot))) < 1e-12
            prev = t


def test_state_carries_the_prefix():
    """With the RNN head the anchor reaches every later position's bias; a
    planted mistake that resets the state each position (a Markov head) must
    not pass this."""
    rng = np.random.default_rng(3)
    B, K, V, r = 1, 5, 64, 6
    base = np.zeros((B, K, V), np.float32)
    A = rng.normal(0, 1, size=(V, r)).astype(np.float32)
    W = rng.normal(0, 1, size=(r, r)).astype(np.float32)
    Bf = rng.normal(0, 1, size=(r, V)).astype(np.float32)
    u = np.full((B, K), 0.5, np.float32)
    teacher = np.array([[10, 20, 30, 40, 50]])
    a = oracle.rnn_draft(base, A, W, Bf, np.array([1]), u, teacher=teacher)
    b = oracle.rnn_draft(base, A, W, Bf, np.array([2]), u, teacher=teacher)
    # same drafted tokens after the anchor, different anchors: every position differs
    assert np.all(np.abs(a["z"] - b["z"]).max(axis=-1) > 1e-6)
    # a Markov head (no recurrence) would differ at position 1 only
    m1 = oracle.rnn_draft(base, A, np.zeros((r, r)), Bf, np.array([1]), u, teacher=teacher)
    m2 = oracle.rnn_draft(base, A, np.zeros((r, r)), Bf, np.array([2]), u, teacher=teacher)
    assert np.abs(m1["z"][:, 1:] - m2["z"][:, 1:]).max() == 0.0
