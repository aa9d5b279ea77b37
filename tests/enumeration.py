"""Exhaustive enumeration of one round at V=8 (test infrastructure).

Every uniform of a round acts through a piecewise-constant map, so the
output distribution is an exact finite sum: enumerate every draft path
(t_1..t_K), every accept/reject outcome per position and every resample
interval, evaluate the pipeline once at the midpoint of each piece, and
weight the result by the piece's length. The target distribution of each row
depends on the drafted prefix through a random table p_rho(.|y_<rho), as a
real target model's would.

The batch is built here; `tally` turns any implementation's outputs on it into
joint probabilities that the losslessness identity can be checked against.
"""
from __future__ import annotations

import itertools

import numpy as np

V, K, R = 8, 3, 2


def _softmax(x):
    e = np.exp(x - x.max(-1, keepdims=True))
    return e / e.sum(-1, keepdims=True)


def _mid_f32(lo, hi):
    """fp32 point strictly inside [lo, hi) (asserted)."""
    m = np.float32((lo + hi) / 2.0)
    assert lo <= float(m) < hi, (lo, hi, m)
    return m


def _draft_q(prob, paths):
    """Draft distributions along every path, built here without the oracle:
    position i (0-based) is corrected by the token before it (the anchor at
    i = 0) with the bias summed term by term in fp64, then softmaxed. The
    uniforms placed at the midpoints of these intervals are what makes the
    oracle's own chain (oracle.draft without teacher forcing) checkable
    against the paths."""
    A = prob["A"].astype(np.float64)
    Bf = prob["Bf"].astype(np.float64)
    n = len(paths)
    q = np.empty((n, K, V))
    for pi in range(n):
        prev = int(prob["anchor"])
        for i in range(K):
            z = prob["base"][i].astype(np.float64).copy()
            for v in range(V):
                for k in range(R):
                    z[v] += A[prev, k] * Bf[k, v]
            q[pi, i] = _softmax(z)
            prev = int(paths[pi, i])
    return q


def make_problem(seed=7, factor_std=0.7):
    rng = np.random.default_rng(seed)
    prob = {
        "base": rng.normal(0, 2, size=(K, V)).astype(np.float32),
        "A": rng.normal(0, factor_std, size=(V, R)).astype(np.float32),
        "Bf": rng.normal(0, factor_std, size=(R, V)).astype(np.float32),
        "anchor": np.int32(5),
        # target logits per prefix: table[rho][prefix tuple] -> [V]
        "table": [{} for _ in range(K + 1)],
    }
    for rho in range(K + 1):
        for prefix in itertools.product(range(V), repeat=rho):
            prob["table"][rho][prefix] = rng.normal(0, 2, size=V).astype(np.float32)
    return prob


def build_batch(prob, L):
    """All pieces for verify length L (0 <= L <= K).

    Returns a dict of batch arrays (one row per piece) plus `weight` [N] and
    `q` [N,K,V] (the draft distributions along each path, built without the oracle).
    """
    paths = np.array(list(itertools.product(range(V), repeat=K)), np.int64)  # [512,K]
    n = len(paths)
    base = np.broadcast_to(prob["base"], (n, K, V)).copy()
    anchor = np.full(n, prob["anchor"], np.int32)
    q = _draft_q(prob, paths)  # [n,K,V], q[:, i] = q_{i+1}(. | t_i)
    rows = {k: [] for k in ("path", "u_draft", "u_accept", "u_resample", "weight", "target", "q")}
    for pi in range(n):
        path = paths[pi]
        # draft uniforms: midpoint of each drafted token's interval
        ud, wd = [], 1.0
        for i in range(K):
            C = np.concatenate([[0.0], np.cumsum(q[pi, i])])
            t = path[i]
            ud.append(_mid_f32(C[t], C[t + 1]))
            wd *= C[t + 1] - C[t]
        # target rows along this path
        tgt = np.stack([prob["table"][rho][tuple(path[:rho])] for rho in range(K)]
                       + [prob["table"][K][tuple(path[:K])]])
        p = _softmax(tgt.astype(np.float64))
        for pattern in itertools.product((True, False), repeat=L):
            ua, wa, jstar = [], 1.0, None
            for j in range(1, L + 1):
                a = min(1.0, p[j - 1, path[j - 1]] / q[pi, j - 1, path[j - 1]])
                if pattern[j - 1]:
                    if a <= 0:
                        wa = 0.0
                        break
                    ua.append(_mid_f32(0.0, a))
                    wa *= a
                else:
                    if a >= 1.0:
                        wa = 0.0
                        break
                    ua.append(_mid_f32(a, 1.0))
                    wa *= 1.0 - a
                    if jstar is None:
                        jstar = j
            if wa == 0.0:
                continue
            ua += [np.float32(0.5)] * (K - len(ua))
            # resample distribution implied by the pieces (residual or bonus)
            if jstar is not None:
                w = np.maximum(0.0, p[jstar - 1] - q[pi, jstar - 1])
            else:
                w = p[L]
            Cr = np.concatenate([[0.0], np.cumsum(w)]) / w.sum()
            for v in range(V):
                if Cr[v + 1] - Cr[v] <= 0:
                    continue
                rows["path"].append(path)
                rows["u_draft"].append(np.array(ud, np.float32))
                rows["u_accept"].append(np.array(ua, np.float32))
                rows["u_resample"].append(_mid_f32(Cr[v], Cr[v + 1]))
                rows["weight"].append(wd * wa * (Cr[v + 1] - Cr[v]))
                rows["target"].append(tgt)
                rows["q"].append(q[pi])
    out = {k: np.stack(v) if k != "u_resample" else np.array(v, np.float32) for k, v in rows.items()}
    N = len(out["weight"])
    out["base"] = np.broadcast_to(prob["base"], (N, K, V)).copy()
    out["anchor"] = np.full(N, prob["anchor"], np.int32)
    out["verify_len"] = np.full(N, L, np.int64)
    out["L"] = L
    return out


def tally(batch, out_tokens, n_out):
    """Joint probabilities P(y_1..y_j, N >= j) from an implementation's outputs."""
    joint = [dict() for _ in range(K + 2)]
    for w, toks, n in zip(batch["weight"], out_tokens, n_out):
        for j in range(1, int(n) + 1):
            key = tuple(int(x) for x in toks[:j])
            joint[j][key] = joint[j].get(key, 0.0) + w
    return joint


def check_lossless(prob, batch, joint, tol=1e-12):
    """P(y_j = v, N >= j, y_<j) == p_j(v | y_<j) * P(N >= j, y_<j) for all j, prefixes."""
    L = batch["L"]
    total = float(np.sum(batch["weight"]))
    assert abs(total - 1.0) < 1e-12, total
    worst = 0.0
    for j in range(1, L + 2):
        prefixes = {}
        for key, pr in joint[j].items():
            prefixes.setdefault(key[:-1], {})[key[-1]] = pr
        for prefix, dist in prefixes.items():
            reach = sum(dist.values())
            rho = j - 1
            tgt = prob["table"][rho][prefix] if rho < K else prob["table"][K][prefix]
            p = _softmax(tgt.astype(np.float64))
            for v in range(V):
                worst = max(worst, abs(dist.get(v, 0.0) - p[v] * reach))
    assert worst < tol, worst
    return worst


def check_accept_rate(prob, batch, accepted, tol=1e-12):
    """P(accept draft j | drafts < j accepted, prefix) == sum_v min(p_j, q_j)."""
    L = batch["L"]
    worst = 0.0
    for j in range(1, L + 1):
        reach, acc, qrow = {}, {}, {}
        for w, path, a, q in zip(batch["weight"], batch["path"], accepted, batch["q"]):
            if a < j - 1:
                continue
            prefix = tuple(int(x) for x in path[: j - 1])
            reach[prefix] = reach.get(prefix, 0.0) + w
            if a >= j:
                acc[prefix] = acc.get(prefix, 0.0) + w
            qrow.setdefault(prefix, q[j - 1])
        for prefix, rw in reach.items():
            p = _softmax(prob["table"][j - 1][prefix].astype(np.float64))
            expected = float(np.minimum(p, qrow[prefix]).sum())
            worst = max(worst, abs(acc.get(prefix, 0.0) / rw - expected))
    assert worst < tol, worst
    return worst
