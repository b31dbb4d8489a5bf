"""The decode round at the 8B layer shape, in the launch configuration the bench times.

Shape: d 4096, 32 q / 8 kv heads x 128, FFN 12288, vocab 151936 (1187 LM-head tiles), k = 32,
batch 1 — every per-layer launch of the 36-layer benchmark model (the four-phase layer chain
with its split-K factors and ring depth, the cluster attention, the LM-head chain, finalize) with
2 layers, so that the oracle can run the whole forward on the host.  Prompt 100: the cached
prefix ends off a page boundary.

Bars.  With N(0, 0.02^2) weights over d = 4096 the logits spread with std ~1.28 (vs ~0.46 at
the small bf16 shape, where the absolute 2e-2 bar holds with margin), and the bf16 rounding of
the stored activations alone moves them by up to ~0.05: the rounding-matched oracle and the
fp32 oracle differ by that much (measured 0.052; the library is 0.040 from the
rounding-matched oracle).  So at this shape the logit bar is that floor, measured in the test:
    max |gpu - oracle_bf16io| <= 1.25 * max |oracle_bf16io - oracle_f32|,
argmax equal wherever the top-2 margin exceeds 5e-2 plus twice that floor (an error of the
floor's size on each of the two top logits cannot reorder them), and the round's commit is
bit-exact given the GPU's own argmaxes.
"""
import pytest
import torch

import oracle
import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, gpu_state, make_pair, top2_margin

pytestmark = pytest.mark.gpu

CFG = synth.LLAMA8B.replace(n_layers=2, max_seq=512)
MARGIN = 5e-2


@pytest.fixture(scope="module")
def pair():
    ctx, om, W = make_pair(CFG, device_weights=True)
    om32 = oracle.OracleModel(CFG, W, "f32")
    p = synth.prompt_tokens(1, 100, CFG.vocab, seed=11)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, CFG.max_seq + 64)
    st32 = odec.prefill(om32, p, CFG.max_seq + 64)
    yield ctx, om, om32, st, st32
    ctx.close()


def _check(gl, ol, of):
    floor = (ol.double() - of.double()).abs().max().item()
    err = (gl.double() - ol.double()).abs().max().item()
    assert err <= 1.25 * floor, (err, floor)
    sure = top2_margin(ol) > MARGIN + 2 * floor
    # top-2 gaps of 151936 logits of std 1.28 average ~0.26, so about half the rows qualify
    assert sure.float().mean().item() >= 0.25
    assert torch.equal(gl.argmax(-1)[sure], odec.argmax_lowest(ol.double())[sure])


def test_draft_and_verify_logits(pair):
    ctx, om, om32, st, st32 = pair
    k = CFG.block_k
    lens, pend, _, _ = gpu_state(ctx, 1)
    assert lens == st.lens and pend == st.pending
    gl = gpu_logits(ctx, 1, 1, k)
    _check(gl, odec.draft_forward(om, st, k), odec.draft_forward(om32, st32, k))
    _, _, draft, _ = gpu_state(ctx, 1)
    assert draft == gl.argmax(-1).tolist()
    gv = gpu_logits(ctx, 2, 1, k + 1)
    _check(gv, odec.verify_forward(om, st, draft), odec.verify_forward(om32, st32, draft))


def test_round_commit_bit_exact(pair):
    ctx, om, om32, st, st32 = pair
    k = CFG.block_k
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    ctx.nld_selfspec_round(toks, nc, None)
    ctx.nld_sync()
    lens, pend, draft, ver = gpu_state(ctx, 1)
    want = odec.commit_after_verify(draft[0], ver[0])
    assert int(nc.item()) == len(want)
    assert toks[0, :len(want)].cpu().tolist() == want
    assert lens[0] == st.lens[0] + len(want) and pend[0] == want[-1]
