"""Failure detection without a GPU fault: a bounded device wait runs out, the kernel records
NLD_DEVERR_TIMEOUT in the device error word and leaves in order, nld_sync reports
NLD_ERR_TIMEOUT, and the context keeps working.

The wait that runs out is the projection chain's grid-wide phase counter: the test hook launches
layer 0's four-phase chain with a 2 ms limit and CTA 0 withholding its first arrival (an arrival
that never comes).  No copy or remote store is in flight at that wait.  Afterwards a draft
forward must still match the oracle (logit bar of the small bf16 shape, 2e-2)."""
import pytest

import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, make_pair

pytestmark = pytest.mark.gpu

CFG = synth.SMALL_BF16


def test_phase_counter_wait_runs_out_and_context_recovers():
    import self_speculation_b200 as nb
    ctx, om, _ = make_pair(CFG)
    p = synth.prompt_tokens(1, 90, CFG.vocab, seed=12)
    ctx.nld_prefill(p.cuda())
    ctx.nld_sync()
    ctx.nld_debug_timeout_chain(2_000_000)
    with pytest.raises(nb.NldError) as ei:
        ctx.nld_sync()
    assert ei.value.status == 6, ei.value
    ctx.nld_sync()                       # the error word was cleared
    st = odec.prefill(om, p, CFG.max_seq + 64)
    gl = gpu_logits(ctx, 1, 1, CFG.block_k)
    ol = odec.draft_forward(om, st, CFG.block_k)
    assert (gl.double() - ol.double()).abs().max().item() < 2e-2
