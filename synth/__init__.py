"""Seeded synthetic inputs for one round of DSpark-style speculative decoding.

This module is the only code shared by the CPU oracle and the CUDA path. It
draws random numbers and lays them out; it holds none of the method's
arithmetic (no softmax, no sampling, no scheduling).

Workloads (rank-256 Markov head as in the QbitAI article "DSpark, 10 points",
section "a cheaper sequential module: the Markov head"; vocabulary sizes of
Qwen3 and DeepSeek-V3):

  tiny     B=4   K=4  V=1024    r=32  fp32 factors N(0,0.1)
  qwen3    B=64  K=8  V=151936  r=256 bf16 factors N(0,0.02)  (the timed workload)
  latency  B=1   K=16 V=151936  r=256 bf16
  highconc B=256 K=16 V=151936  r=256 bf16
  mixed    B=512 K=16 V=129280  r=256 bf16

Every workload: base draft logits ~N(0,2) fp32; target logits for row
rho < K are base[:, rho] + N(0, sigma_b); the bonus row (rho = K) is an
independent N(0,2); T_j = 1 + 0.1 j; anchor uniform in [0,V); uniforms
U[0,1) in fp32.  Seeds: 1000 + workload index, split by
numpy SeedSequence(seed).spawn(12) in the fixed order of STREAMS.
"""
from __future__ import annotations

import dataclasses
import numpy as np

STREAMS = ("base", "A", "Bf", "target_noise", "bonus", "conf", "u_draft",
           "u_accept", "u_resample", "anchor", "sigma", "profile_jitter")


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    K: int
    V: int
    r: int
    factor_dtype: str          # "f32" or "bf16"
    factor_std: float
    n_prof: int

    @property
    def seed(self) -> int:
        return 1000 + self.index


WORKLOADS = (
    Workload(0, "tiny", 4, 4, 1024, 32, "f32", 0.1, 2048),
    Workload(1, "qwen3", 64, 8, 151936, 256, "bf16", 0.02, 2048),
    Workload(2, "latency", 1, 16, 151936, 256, "bf16", 0.02, 2048),
    Workload(3, "highconc", 256, 16, 151936, 256, "bf16", 0.02, 4352),
    Workload(4, "mixed", 512, 16, 129280, 256, "bf16", 0.02, 4096),
)


def workload(key) -> Workload:
    if isinstance(key, Workload):
        return key
    if isinstance(key, int):
        return WORKLOADS[key]
    for w in WORKLOADS:
        if w.name == key:
            return w
    raise KeyError(key)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bits.
    Finite inputs only (the uint32 sum cannot carry out of 32 bits for them)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng, shape, std):
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _sigma(w: Workload, rng) -> np.ndarray:
    B = w.B
    if w.index == 0:
        return np.ones(B, np.float32)
    if w.index == 1:
        return np.where(np.arange(B) < B // 2, 1.0, 3.0).astype(np.float32)
    if w.index == 2:
        return np.full(B, 0.5, np.float32)
    if w.index == 3:
        return rng.choice(np.array([0.5, 1.0, 2.0, 4.0], np.float32), size=B)
    if w.index == 4:
        return np.exp(rng.uniform(np.log(0.3), np.log(5.0), size=B)).astype(np.float32)
    raise ValueError(w)


def _profile(w: Workload, rng) -> np.ndarray:
    """Round time T(n) in ms for n = 1..n_prof verify-batch tokens."""
    n = np.arange(1, w.n_prof + 1, dtype=np.float64)
    if w.index == 0:
        t = 1.0 + 0.01 * n
    elif w.index == 1:
        t = 1.0 + 0.004 * np.maximum(n - 256, 0)
    elif w.index == 2:
        t = np.ones_like(n)
    elif w.index == 3:
        t = 1.0 + 0.01 * np.maximum(n - 512, 0)
    elif w.index == 4:
        t = np.where(n <= 1024, 1.0 + 0.0002 * n, 1.0 + 0.0002 * 1024 + 0.004 * (n - 1024))
        t = t * (1.0 + 0.01 * rng.standard_normal(size=n.shape))
    else:
        raise ValueError(w)
    return t.astype(np.float32)


def _conf(w: Workload, rng, sigma) -> np.ndarray:
    if w.index in (3, 4):
        mean = (3.0 - sigma)[:, None]
    else:
        mean = np.ones((w.B, 1), np.float32)
    return (mean + rng.standard_normal(size=(w.B, w.K), dtype=np.float32)).astype(np.float32)


def custom(like, **sizes) -> Workload:
    """A workload with another workload's recipe (sigma, confidence, profile
    shape, factor dtype) and the given sizes, e.g. custom(1, B=8, V=37000)."""
    return dataclasses.replace(workload(like), **sizes)


def make_factors(key, seed: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """The Markov factors (A [V,r], Bf [r,V]) that make_round draws for this seed."""
    w = workload(key)
    ss = np.random.SeedSequence(w.seed if seed is None else seed)
    rngs = dict(zip(STREAMS, (np.random.default_rng(s) for s in ss.spawn(len(STREAMS)))))
    A = _normal(rngs["A"], (w.V, w.r), w.factor_std)
    Bf = _normal(rngs["Bf"], (w.r, w.V), w.factor_std)
    if w.factor_dtype == "bf16":
        A, Bf = f32_to_bf16_bits(A), f32_to_bf16_bits(Bf)
    return A, Bf


def make_round(key, seed: int | None = None, with_target: bool = True, factors=None) -> dict:
    """All inputs of one round of the given workload, as host numpy arrays.

    Keys: base [B,K,V] f32; A [V,r], Bf [r,V] (f32, or uint16 bf16 bits);
    anchor [B] i32; u_draft [B,K], u_accept [B,K], u_resample [B] f32;
    conf [B,K] f32; temps [K] f32; profile [n_prof] f32; sigma [B] f32;
    target [B,K+1,V] f32 (dense: row rho of request b at b*(K+1)+rho).
    `factors` (A, Bf) replaces the seed's own factors: the Markov head's
    weights, which stay fixed while the per-round inputs change; every other
    stream is the seed's.
    """
    w = workload(key)
    ss = np.random.SeedSequence(w.seed if seed is None else seed)
    rngs = dict(zip(STREAMS, (np.random.default_rng(s) for s in ss.spawn(len(STREAMS)))))
    B, K, V, r = w.B, w.K, w.V, w.r
    out = {"workload": w}
    out["base"] = _normal(rngs["base"], (B, K, V), 2.0)
    if factors is None:
        A = _normal(rngs["A"], (V, r), w.factor_std)
        Bf = _normal(rngs["Bf"], (r, V), w.factor_std)
        if w.factor_dtype == "bf16":
            A, Bf = f32_to_bf16_bits(A), f32_to_bf16_bits(Bf)
    else:
        A, Bf = factors
        assert A.shape == (V, r) and Bf.shape == (r, V)
    out["A"], out["Bf"] = A, Bf
    sigma = _sigma(w, rngs["sigma"])
    out["sigma"] = sigma
    if with_target:
        tgt = np.empty((B, K + 1, V), np.float32)
        noise_rng = rngs["target_noise"]
        for b in range(B):
            tgt[b, :K] = out["base"][b]
            tgt[b, :K] += _normal(noise_rng, (K, V), float(sigma[b]))
        tgt[:, K] = _normal(rngs["bonus"], (B, V), 2.0)
        out["target"] = tgt
    out["conf"] = _conf(w, rngs["conf"], sigma)
    out["temps"] = (1.0 + 0.1 * np.arange(1, K + 1)).astype(np.float32)
    out["u_draft"] = rngs["u_draft"].random(size=(B, K), dtype=np.float32)
    out["u_accept"] = rngs["u_accept"].random(size=(B, K), dtype=np.float32)
    out["u_resample"] = rngs["u_resample"].random(size=B, dtype=np.float32)
    out["anchor"] = rngs["anchor"].integers(0, V, size=B, dtype=np.int32)
    out["profile"] = _profile(w, rngs["profile_jitter"])
    return out


def dense_row_start(B: int, K: int) -> np.ndarray:
    """Row offsets of the dense [B,K+1,V] target layout."""
    return (np.arange(B, dtype=np.int64) * (K + 1)).astype(np.int64)


def pack_rows(target_dense: np.ndarray, verify_len: np.ndarray, row_start: np.ndarray) -> np.ndarray:
    """Gather rows 0..L_b of each request to rows row_start[b].. of a packed array.

    Data movement only: it stands in for a target forward pass run on the
    ragged verify batch. row_start is given (it is a scheduler output).
    """
    B, _, V = target_dense.shape
    counts = np.asarray(verify_len, np.int64) + 1
    n_rows = int(np.max(np.asarray(row_start, np.int64) + counts)) if B else 0
    packed = np.zeros((n_rows, V), np.float32)
    for b in range(B):
        packed[row_start[b]: row_start[b] + counts[b]] = target_dense[b, : counts[b]]
    return packed
