"""dspark_schedule_static, the scheduler entry point that allocates nothing.

It exists for callers that cannot allocate device memory (a framework that
owns the allocator, code running under stream capture, a hot path that
forbids cudaMalloc): its scratch is a static device array inside the
library. Its outputs must equal those of dspark_schedule (same kernels), on
two calls in a row with different inputs, since every call shares and
rewrites the one array. Kept in its own file, collected last, so that a
stop-at-first-failure run has run every other test first; it also passes
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _inputs(key, seed):
    inp = synth.make_round(key, seed=seed, with_target=False)
    return {k: torch.from_numpy(np.ascontiguousarray(inp[k])).cuda() for k in ("conf", "temps", "profile")}


def _outputs(B, K):
    return (torch.full((B,), -7, dtype=torch.int32, device="cuda"),
            torch.full((B, K), -7.0, dtype=torch.float32, device="cuda"),
            torch.full((B,), -7, dtype=torch.int64, device="cuda"),
            torch.full((1,), -7, dtype=torch.int32, device="cuda"))


def test_static_schedule_matches_workspace_schedule_twice():
    from speculative_decoding_semi_b200 import binding

    # the last case has B*K = 16384, the limit, where the scratch layout fills
    # the static array exactly
    for key, seed in (("qwen3", 11), (synth.custom(4, B=512, K=16, V=8, n_prof=4096), 12),
                      (synth.custom(4, B=512, K=32, V=8, n_prof=512 * 33), 13)):
        d = _inputs(key, seed)
        B, K = d["conf"].shape
        ws = torch.zeros(binding.dspark_workspace_bytes(B, K, 8, 1), dtype=torch.uint8, device="cuda")
        ref = _outputs(B, K)
        binding.dspark_schedule(d["conf"], d["temps"], d["profile"], *ref, ws)
        got = _outputs(B, K)
        binding.dspark_schedule_static(d["conf"], d["temps"], d["profile"], *got)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        assert int(got[3].item()) == int((got[0].long() + 1).sum().item())


def test_static_schedule_rejects_too_many_items():
    from speculative_decoding_semi_b200 import binding

    B, K = 1024, 32  # 32768 items > 16384
    conf = torch.zeros(B, K, device="cuda")
    temps = torch.ones(K, device="cuda")
    prof = torch.ones(B * (K + 1), device="cuda")
    with pytest.raises(binding.DSparkError) as e:
        binding.dspark_schedule_static(conf, temps, prof, *_outputs(B, K))
    assert e.value.status == 1
