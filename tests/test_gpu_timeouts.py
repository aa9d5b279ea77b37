"""Failure detection without a GPU fault: a bounded device-wide wait that runs
out reports DSPARK_ERR_TIMEOUT and leaves the context and the workspace usable.

A test hook in the workspace makes one CTA skip one publish (the draft's
slice sums at position 1, verify's arrival at its first device-wide barrier,
or the variant-B residual kernel's slice sums); with a 2 ms wait budget the other CTAs' waits run out, the kernel
lets its copies land, frees its tensor memory and returns. Nothing traps,
faults or waits without a bound. The same workspace then runs a normal round,
which must match the oracle.
"""
import numpy as np
import pytest

import synth
from tests import parity

pytestmark = pytest.mark.gpu

TIMEOUT = 4


def _setup(seed, variant="a"):
    from speculative_decoding_semi_b200 import round as rnd
    # bf16 factors, r % 64 == 0, V % 32 == 0: the tensor-core draft kernel
    w = synth.custom(1, B=8, K=3, V=8192, r=64, n_prof=64)
    inp = synth.make_round(w, seed=seed)
    return inp, rnd.to_device(inp), rnd.RoundBuffers(8, 3, 8192, 64, variant=variant)


def _normal_round_after(inp, bufs):
    from speculative_decoding_semi_b200 import binding as bn
    bn.dspark_inject_stall(bufs.workspace, bn.DSPARK_INJECT_NONE)
    bn.dspark_set_wait_budget(bufs.workspace, 0)
    t, _ = parity.check_round(inp, bufs=bufs)
    t.check()


@pytest.mark.parametrize("cta", [0, 1, 100])
def test_draft_wait_runs_out_and_reports_timeout(cta):
    from speculative_decoding_semi_b200 import binding as bn
    from speculative_decoding_semi_b200 import round as rnd
    inp, d, bufs = _setup(31 + cta)
    bn.dspark_set_wait_budget(bufs.workspace, 2000)
    bn.dspark_inject_stall(bufs.workspace, bn.DSPARK_INJECT_DRAFT_SLICE_SUMS, cta)
    rnd.draft(d, bufs)
    st, detail = bn.dspark_read_device_error(bufs.workspace)
    assert st == TIMEOUT, (st, hex(detail))
    assert bn.dspark_read_device_error(bufs.workspace)[0] == 0   # read once, then cleared
    _normal_round_after(inp, bufs)


def test_verify_barrier_runs_out_and_reports_timeout():
    from speculative_decoding_semi_b200 import binding as bn
    from speculative_decoding_semi_b200 import round as rnd
    inp, d, bufs = _setup(41)
    rnd.draft(d, bufs)
    rnd.schedule(d, bufs)
    assert bn.dspark_read_device_error(bufs.workspace)[0] == 0
    bn.dspark_set_wait_budget(bufs.workspace, 2000)
    bn.dspark_inject_stall(bufs.workspace, bn.DSPARK_INJECT_VERIFY_BARRIER, 1)
    rnd.verify(d, bufs)
    st, detail = bn.dspark_read_device_error(bufs.workspace)
    assert st == TIMEOUT, (st, hex(detail))
    _normal_round_after(inp, bufs)


def test_residual_wait_runs_out_and_reports_timeout():
    """Variant B: one CTA of the residual kernel skips its slice-sum publish;
    the CTAs that draw the resampled tokens wait for it and run out."""
    from speculative_decoding_semi_b200 import binding as bn
    from speculative_decoding_semi_b200 import round as rnd
    inp, d, bufs = _setup(43, variant="b")
    d["u_accept"].fill_(0.999)  # rejections at almost every verified position
    rnd.draft(d, bufs)
    rnd.schedule(d, bufs)
    assert bn.dspark_read_device_error(bufs.workspace)[0] == 0
    assert int(bufs.verify_len.sum()) > 0
    bn.dspark_set_wait_budget(bufs.workspace, 2000)
    bn.dspark_inject_stall(bufs.workspace, bn.DSPARK_INJECT_RESIDUAL_SLICE_SUMS, 1)
    rnd.verify(d, bufs)
    st, detail = bn.dspark_read_device_error(bufs.workspace)
    assert st == TIMEOUT, (st, hex(detail))
    _normal_round_after(inp, bufs)


def test_budget_and_hook_arguments_checked_on_the_host():
    import torch

    from speculative_decoding_semi_b200 import binding as bn
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(bn.DSparkError):
        bn.dspark_inject_stall(ws, 7, 0)
    with pytest.raises(bn.DSparkError):
        bn.dspark_inject_stall(ws, bn.DSPARK_INJECT_DRAFT_SLICE_SUMS, 1 << 24)
    bn.dspark_set_wait_budget(ws, 123)
    bn.dspark_inject_stall(ws, bn.DSPARK_INJECT_VERIFY_BARRIER, 5)
    words = ws[:16].view(torch.int32).cpu().numpy()
    assert words[2] == 123 and words[3] == (2 << 24 | 5)
