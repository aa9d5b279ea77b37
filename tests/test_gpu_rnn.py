"""The RNN sequential head on the GPU against oracle.rnn_draft, and a whole
round (schedule and verify on the RNN draft's outputs) against the oracle."""
import numpy as np
import pytest

import synth
from tests import parity

pytestmark = pytest.mark.gpu


def _with_w(inp, std, seed):
    r = inp["A"].shape[1]
    rng = np.random.default_rng(seed)
    inp = dict(inp)
    inp["W"] = synth.f32_to_bf16_bits(rng.normal(0, std, size=(r, r)).astype(np.float32))
    return inp


@pytest.mark.parametrize("like,sizes,wstd", [
    (1, dict(B=12, K=5, V=37024, r=64, n_prof=256), 0.1),
    (1, dict(B=3, K=16, V=4096, r=256, n_prof=64), 0.05),
    (1, dict(B=130, K=3, V=8192, r=128, n_prof=600), 0.08),
    (1, dict(B=17, K=4, V=4096, r=192, n_prof=80), 0.08),
])
def test_rnn_round_matches_oracle(like, sizes, wstd):
    w = synth.custom(like, **sizes)
    t = parity.Tally()
    for seed in range(2):
        inp = _with_w(synth.make_round(w, seed=600 + seed), wstd, 700 + seed)
        parity.check_round(inp, tally=t)
    t.check(f"rnn {sizes}")


def test_rnn_full_size_qwen3():
    inp = _with_w(synth.make_round("qwen3"), 0.05, 11)
    t, _ = parity.check_round(inp)
    t.check("rnn qwen3")


def test_rnn_head_needs_the_tensor_core_shapes():
    from speculative_decoding_semi_b200 import binding
    from speculative_decoding_semi_b200 import round as rnd
    w = synth.custom(1, B=4, K=2, V=1000, r=64, n_prof=16)   # V % 32 != 0
    inp = _with_w(synth.make_round(w, seed=1), 0.1, 2)
    d = rnd.to_device(inp)
    bufs = rnd.RoundBuffers(4, 2, 1000, 64)
    with pytest.raises(binding.DSparkError) as e:
        rnd.draft(d, bufs)
    assert e.value.status == 2
