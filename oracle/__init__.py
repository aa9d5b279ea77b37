"""CPU oracle for one round of DSpark-style speculative decoding (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg (and
bench.py --impl reference) may import or call it. It shares no code with the
CUDA path; the only module both sides use is `synth` (seeded inputs).

Every function is the plain definition of one step, written in float64 with
numpy primitives (matmul, exp, cumsum, sort) and no blocking or reordering.
Sources (four web pages on DeepSeek's DSpark; titles abbreviated):
  [Thread]  sina.cn, "Fireworks AI CTO Dzhulgakov explains DSpark", items 1-10
  [QbitAI]  hzrcw.cc, "DSpark: ten concepts are enough", headed sections
  [Essay]   10100.com, "speculative decoding is not making the model think less"
  [Tags]    wangjunjian.com, tag page "speculative-decoding" (DSpark abstract,
            summary, and the generic speculative-decoding recipe)
The pages state each step in words only; where they leave a detail open the
reading taken is named in the function's docstring.

Pins (tests/test_oracle_*.py): exhaustive enumeration at V=8 that the verified
output is distributed exactly as the target; factors that force each draft
token to be a fixed function of the previous one (the chain, with and without
teacher forcing); forced acceptance counts that fix which row the final token
comes from; zero Markov factors reduce the draft to independent per-position
inverse-CDF sampling; the bias equals a brute-force fp64 triple loop; the
scheduler equals brute force over every length assignment; survival has
closed forms at c=0 and c -> +-inf; a request sample, packed target rows and
a vanished residual (fallback to p) agree with the full batch, the dense
layout and a scipy draw from p.
"""
from __future__ import annotations

import numpy as np

__all__ = ["bf16_to_f64", "softmax", "icdf", "markov_bias", "draft_step", "draft",
           "survival", "schedule", "verify", "run_round", "calibrate", "round_to_bf16", "rnn_draft"]


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def factors_f64(A, Bf) -> tuple[np.ndarray, np.ndarray]:
    if A.dtype == np.uint16:
        return bf16_to_f64(A), bf16_to_f64(Bf)
    return A.astype(np.float64), Bf.astype(np.float64)


def softmax(z: np.ndarray) -> np.ndarray:
    """q = exp(z - max z) / sum exp(z - max z) along the last axis, fp64."""
    z = np.asarray(z, np.float64)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def icdf(w: np.ndarray, u) -> tuple[np.ndarray, np.ndarray]:
    """Inverse-CDF sample of each row of weights w with its uniform u.

    Returns (k, margin): k = smallest index with C_k > u*W where C is the
    running sum of w and W = C[-1] (strict '>' so a zero-weight entry is never
    returned); if rounding leaves no such index, the largest k with w_k > 0.
    margin = min(u*W - C_{k-1}, C_k - u*W) / W with C_{-1} = 0: the distance of
    the threshold to the nearest boundary of the chosen interval.
    Sampling by a supplied uniform follows the recipe on [Tags], article
    "Speculative Decoding", steps 3-4 (compare with a random number; resample).
    """
    w = np.atleast_2d(np.asarray(w, np.float64))
    u = np.atleast_1d(np.asarray(u, np.float32)).astype(np.float64)
    C = np.cumsum(w, axis=-1)
    W = C[:, -1]
    thr = u * W
    above = C > thr[:, None]
    has = above.any(axis=-1)
    k = np.where(has, above.argmax(axis=-1), 0)
    if not has.all():
        last_pos = w.shape[1] - 1 - (w[:, ::-1] > 0).argmax(axis=-1)
        k = np.where(has, k, last_pos)
    rows = np.arange(w.shape[0])
    Ck = C[rows, k]
    Cprev = np.where(k > 0, C[rows, np.maximum(k - 1, 0)], 0.0)
    with np.errstate(invalid="ignore", divide="ignore"):
        margin = np.minimum(thr - Cprev, Ck - thr) / W
    return k.astype(np.int64), margin


def markov_bias(A64: np.ndarray, Bf64: np.ndarray, t_prev: np.ndarray) -> np.ndarray:
    """Low-rank Markov head: bias[b, :] = A[t_prev[b], :] @ Bf.

    [QbitAI] section "a cheaper sequential module: the Markov head" and [Essay]
    section "parallel drafts are fast ...": the head looks only at the previous
    token and is factorised at rank 256. Reading: the correction is exactly the
    product of the two factors, added to the backbone logits, unscaled.
    """
    return A64[np.asarray(t_prev, np.int64)] @ Bf64


def draft_step(base_i: np.ndarray, A64, Bf64, t_prev, u) -> dict:
    """One position of the semi-autoregressive draft, for all requests.

    [QbitAI] section "DSpark = Eagle + DFlash": the parallel backbone gives base
    logits for every position at once; a sequential head then adds a
    prefix-dependent bias left to right. z = base + A[t_prev] Bf, q = softmax(z),
    t = ICDF(q, u), q_tok = q(t), lse = log sum exp z.
    """
    z = np.asarray(base_i, np.float64) + markov_bias(A64, Bf64, t_prev)
    zmax = z.max(axis=-1)
    e = np.exp(z - zmax[:, None])
    W = e.sum(axis=-1)
    q = e / W[:, None]
    t, margin = icdf(q, u)
    rows = np.arange(z.shape[0])
    return {"z": z, "t": t, "q_tok": q[rows, t], "lse": zmax + np.log(W), "margin": margin}


def draft(base, A, Bf, anchor, u_draft, teacher=None, keep_z=True) -> dict:
    """K-step Markov draft over all requests of the batch.

    Position 1 is corrected by the anchor token (the last token before the
    block); position i > 1 by the token drawn at i-1. With `teacher` [B,K] the
    chain continues from the teacher's token at each step (teacher forcing)
    while t/margin still report the oracle's own draw; q_tok is then q at the
    teacher's token, as verification would see it.
    """
    base = np.asarray(base)
    B, K, V = base.shape
    A64, Bf64 = factors_f64(A, Bf)
    t_prev = np.asarray(anchor, np.int64)
    out = {k: [] for k in ("t", "q_tok", "lse", "margin", "z")}
    for i in range(K):
        s = draft_step(base[:, i], A64, Bf64, t_prev, u_draft[:, i])
        chain = s["t"] if teacher is None else np.asarray(teacher[:, i], np.int64)
        q_tok = np.exp(s["z"][np.arange(B), chain] - s["lse"])
        out["t"].append(s["t"])
        out["q_tok"].append(q_tok)
        out["lse"].append(s["lse"])
        out["margin"].append(s["margin"])
        if keep_z:
            out["z"].append(s["z"])
        t_prev = chain
    res = {k: np.stack(v, axis=1) for k, v in out.items() if v}
    res["chain"] = res["t"] if teacher is None else np.asarray(teacher, np.int64)
    return res


def survival(conf, temps) -> np.ndarray:
    """Cumulative prefix-survival P[b,j] = prod_{k<=j} sigmoid(conf[b,k] / T_k).

    [QbitAI] section "variable-length drafts and hardware-aware scheduling": a
    confidence head scores each draft position's chance to survive
    verification; [Essay] section "the hard step ...": that chance is
    conditional on all earlier drafts passing, and it is calibrated by
    sequential temperature scaling. Reading: per-position logistic with
    temperature T_j; the cumulative survival is the product.
    """
    c = np.asarray(conf, np.float64)
    T = np.asarray(temps, np.float64)[None, :]
    s = 1.0 / (1.0 + np.exp(-c / T))
    return np.cumprod(s, axis=1)


def schedule(P: np.ndarray, profile) -> dict:
    """Per-request verify lengths maximising expected emitted tokens per time.

    [Thread] item 4 and [QbitAI] section "speculation is not free": time per
    token = (draft time + verify time) / accepted tokens. [QbitAI] section
    "variable-length drafts ...": a pre-measured throughput-vs-batch curve
    and the survival estimates choose each request's verify length.
    Reading: items (b,j) with value P[b,j] are ranked by P descending, then j
    ascending, then b ascending; taking the first m gives S_m expected accepted
    drafts; the round emits B + S_m tokens in expected value (each request also
    emits its resampled or bonus token) and takes T(B + m) ms, where
    T(n) = profile[n-1] and n counts verify-batch tokens (each request's last
    token plus its L_b drafts). m* is the smallest maximiser of
    (B + S_m) / T(B + m) over 0 <= m <= min(B*K, n_prof - B); L_b counts request
    b's items among the first m*.
    """
    P = np.asarray(P, np.float64)
    B, K = P.shape
    T = np.asarray(profile, np.float64)
    M = min(B * K, T.shape[0] - B)
    if M < 0:
        raise ValueError("profile shorter than the batch")
    jj, bb = np.meshgrid(np.arange(K), np.arange(B))
    vals, js, bs = P.ravel(), jj.ravel(), bb.ravel()
    order = np.lexsort((bs, js, -vals))
    S = np.concatenate([[0.0], np.cumsum(vals[order])])[: M + 1]
    m = np.arange(M + 1)
    obj = (B + S) / T[B + m - 1]
    m_star = int(np.argmax(obj))
    L = np.bincount(bs[order[:m_star]], minlength=B).astype(np.int64)
    counts = L + 1
    row_start = np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(np.int64)
    # margins used to excuse GPU/oracle disagreements at near-ties
    sorted_vals = vals[order]
    gap_item = np.inf
    if 0 < m_star < vals.size:
        gap_item = abs(sorted_vals[m_star - 1] - sorted_vals[m_star]) / max(sorted_vals[m_star - 1], 1e-300)
    rest = np.delete(obj, m_star)
    gap_obj = np.inf if rest.size == 0 else (obj[m_star] - rest.max()) / obj[m_star]
    return {"verify_len": L, "row_start": row_start, "n_tokens": int(counts.sum()),
            "m_star": m_star, "objective": obj, "gap_item": gap_item, "gap_obj": gap_obj,
            "order": order}


def verify(target_rows, row_start, z, lse_q, q_tok, tokens, verify_len, u_accept, u_resample,
           forced_accepted=None, requests=None) -> dict:
    """Lossless rejection-sampling verification, one request at a time.

    [QbitAI] section "speculative decoding": candidates are checked one by one
    by rejection sampling, the longest correct prefix is kept and one token is
    resampled at the first divergence; this keeps the target's distribution
    exactly ([Essay] section "speculative decoding is not ...", citing
    Leviathan et al.). [Tags] "Speculative Decoding", steps 3-5: compare the
    two models' probabilities with a random number; if all are accepted sample
    the next token from the target, else resample from an adjusted
    distribution. Readings (the pages print no formula): accept draft j iff
    u_a * q_j(t_j) < p_j(t_j), i.e. u_a < min(1, p/q); the adjusted
    distribution is max(0, p - q) renormalised (falling back to p if it sums
    to 0); p_j = softmax(target row j-1) and the bonus uses row L_b.

    z [B,K,V], lse_q, q_tok, tokens [B,K] are the draft's (z may be fp64).
    forced_accepted [B] (optional) makes the final token follow that many
    acceptances (teacher forcing) while `accepted` reports the oracle's own.
    """
    B = len(verify_len) if requests is None else len(requests)
    reqs = range(len(verify_len)) if requests is None else requests
    K = tokens.shape[1]
    res = {"accepted": [], "accepted_used": [], "final": [], "n_out": [], "out_tokens": [],
           "accept_margin": [], "final_margin": [], "final_mode": []}
    for idx, b in enumerate(reqs):
        Lb = int(verify_len[b])
        rows = np.asarray(target_rows[row_start[b]: row_start[b] + Lb + 1], np.float64)
        p = softmax(rows)
        acc = Lb
        margins = []
        for j in range(1, Lb + 1):
            t = int(tokens[idx, j - 1])
            pj, qj = p[j - 1, t], float(q_tok[idx, j - 1])
            ua = float(np.float32(u_accept[b, j - 1]))
            margins.append(abs(ua - pj / qj))
            if not (ua * qj < pj):
                acc = j - 1
                break
        used = acc if forced_accepted is None else int(forced_accepted[b])
        if used < Lb:
            q = softmax(np.asarray(z[idx, used], np.float64))
            w = np.maximum(0.0, p[used] - q)
            mode = "residual"
            if w.sum() == 0.0:
                w, mode = p[used], "residual_fallback"
        else:
            w, mode = p[Lb], "bonus"
        k, m = icdf(w, u_resample[b])
        out = np.full(K + 1, -1, np.int64)
        out[:used] = tokens[idx, :used]
        out[used] = k[0]
        res["accepted"].append(acc)
        res["accepted_used"].append(used)
        res["final"].append(int(k[0]))
        res["n_out"].append(used + 1)
        res["out_tokens"].append(out)
        res["accept_margin"].append(margins)
        res["final_margin"].append(float(m[0]))
        res["final_mode"].append(mode)
    for key in ("accepted", "accepted_used", "final", "n_out", "final_margin"):
        res[key] = np.asarray(res[key])
    res["out_tokens"] = np.stack(res["out_tokens"]) if res["out_tokens"] else np.zeros((0, K + 1), np.int64)
    return res


def run_round(inp: dict, requests=None) -> dict:
    """Draft -> survival -> schedule -> verify for one round of inputs from synth.

    The scheduler couples all requests (it is cheap and always runs on the full
    batch); draft and verify are per request, so `requests` may restrict them to
    a sample. Verification reads the dense target layout.
    """
    B, K, V = inp["base"].shape
    reqs = np.arange(B) if requests is None else np.asarray(requests)
    d = draft(inp["base"][reqs], inp["A"], inp["Bf"], inp["anchor"][reqs], inp["u_draft"][reqs])
    P = survival(inp["conf"], inp["temps"])
    s = schedule(P, inp["profile"])
    rows = inp["target"].reshape(B * (K + 1), V)
    rs = np.arange(B, dtype=np.int64) * (K + 1)
    v = verify(rows, rs, d["z"], d["lse"], d["q_tok"], d["t"], s["verify_len"],
               inp["u_accept"], inp["u_resample"], requests=reqs)
    return {"draft": d, "survival": P, "schedule": s, "verify": v, "requests": reqs}


def calibrate(conf, temps, verify_len, accepted, eta: float, t_min: float, t_max: float) -> np.ndarray:
    """One online step of sequential temperature scaling from a round's outcome.

    [QbitAI] section "online drafter calibration": the confidence head is
    over-confident, so its scores are post-processed by sequential temperature
    scaling, and the calibration runs online, correcting itself from the
    acceptance actually observed on the current workload; [Thread] item 10
    (observe the drafter at run time and adjust the thresholds dynamically);
    [Essay] section "the hard step ...": the confidence is the chance that a
    position survives given that every earlier draft passed.
    Reading: position j's temperature T_j is the scale of a logistic model
    s = sigmoid(c / T_j) of that conditional survival, and temperature scaling
    fits it by the negative log-likelihood of observed outcomes. The
    observations of position j in a round are the requests that reached it
    (drafts 1..j-1 accepted) and verified it (j <= L_b), with outcome
    y = 1 if draft j was accepted. Online, each round takes one gradient step
    on theta_j = 1 / T_j with the mean gradient over those observations:
        g_j = (1/n_j) sum_b (sigmoid(c_bj theta_j) - y_bj) c_bj
        theta_j <- theta_j - eta g_j,  T_j = clamp(1 / theta_j, t_min, t_max).
    A position with no observation keeps its temperature. Returns the new
    temperatures (fp64).
    """
    c = np.asarray(conf, np.float64)
    T = np.asarray(temps, np.float64).copy()
    L = np.asarray(verify_len, np.int64)
    acc = np.asarray(accepted, np.int64)
    B, K = c.shape
    for j in range(1, K + 1):
        reached = (acc >= j - 1) & (L >= j)
        n = int(reached.sum())
        if n == 0:
            continue
        theta = 1.0 / T[j - 1]
        cj = c[reached, j - 1]
        y = (acc[reached] >= j).astype(np.float64)
        s = 1.0 / (1.0 + np.exp(-cj * theta))
        g = float(np.sum((s - y) * cj)) / n
        theta = theta - eta * g
        T[j - 1] = np.clip(1.0 / theta, t_min, t_max) if theta > 0 else t_max
    return T


def round_to_bf16(x) -> np.ndarray:
    """fp64 values rounded to the nearest bfloat16 (8 significant bits, ties to
    even), returned as fp64. Direct from fp64 (no intermediate fp32 rounding):
    for a normal x with 2^e <= |x| < 2^(e+1) the bf16 spacing is 2^(e-7), and
    x / 2^(e-7) is exact in fp64, so rounding that quotient half-to-even and
    scaling back is the correctly rounded value."""
    x = np.asarray(x, np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    e = np.floor(np.log2(np.abs(x[nz])))
    # guard against log2 landing one below an exact power of two
    e = np.where(np.abs(x[nz]) >= 2.0 ** (e + 1), e + 1, e)
    q = 2.0 ** (e - 7)
    out[nz] = np.round(x[nz] / q) * q
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def rnn_draft(base, A, W, Bf, anchor, u_draft, teacher=None, keep_z=True) -> dict:
    """K-step draft with the RNN sequential head.

    [QbitAI] section "a cheaper sequential module: the Markov head", last
    paragraph, and [Essay] section "parallel drafts are fast ...": besides the
    default Markov head (previous token only) the paper offers an RNN head that
    tracks the prefix of the whole draft block; both are light sequential
    modules that correct the parallel backbone's base logits left to right.
    Reading (the pages give no equations): an Elman recurrence over the
    drafted tokens with the Markov head's factors as input embedding and
    output projection,
        h_0 = 0,  h_i = tanh(A[t_{i-1}] + W h_{i-1}),  z_i = base_i + bf16(h_i) Bf,
    t_0 the anchor, W [r,r] the recurrent weight; the state is rounded to
    bfloat16 where it meets the bf16 projection, as the factors are. With
    W = 0 this is the Markov head with factors bf16(tanh(A)).
    Same outputs as draft() (teacher forcing included), plus "h" [B,K,r], the
    fp64 states before rounding.
    """
    base = np.asarray(base)
    B, K, V = base.shape
    A64, Bf64 = factors_f64(A, Bf)
    W64 = bf16_to_f64(W) if np.asarray(W).dtype == np.uint16 else np.asarray(W, np.float64)
    r = A64.shape[1]
    t_prev = np.asarray(anchor, np.int64)
    h = np.zeros((B, r))
    out = {k: [] for k in ("t", "q_tok", "lse", "margin", "z", "h")}
    for i in range(K):
        h = np.tanh(A64[t_prev] + h @ W64.T)
        hb = round_to_bf16(h)
        z = np.asarray(base[:, i], np.float64) + hb @ Bf64
        zmax = z.max(axis=-1)
        e = np.exp(z - zmax[:, None])
        Wsum = e.sum(axis=-1)
        q = e / Wsum[:, None]
        t, margin = icdf(q, u_draft[:, i])
        lse = zmax + np.log(Wsum)
        chain = t if teacher is None else np.asarray(teacher[:, i], np.int64)
        out["t"].append(t)
        out["q_tok"].append(np.exp(z[np.arange(B), chain] - lse))
        out["lse"].append(lse)
        out["margin"].append(margin)
        out["h"].append(h)
        if keep_z:
            out["z"].append(z)
        t_prev = chain
    res = {k: np.stack(v, axis=1) for k, v in out.items() if v}
    res["chain"] = res["t"] if teacher is None else np.asarray(teacher, np.int64)
    return res
