"""bf16 path (tcgen05 GEMMs, tensor-core attention) against the rounding-matched oracle.

Shape: 2 layers, d 512, 8 q / 2 kv heads x 128 (GQA group 4), FFN 1536, vocab 5000 (a ragged
last LM-head tile), k = 32, batch up to 4: every projection spans several row tiles, batch 1
runs the cluster split-K path (M = 32/33 tokens) and batch 3 the wide-tile path (M = 96/99);
prompt lengths put the KV prefix off page boundaries.

Bars (stated for the decode round): logits max-abs error <= 2e-2; argmax equal wherever the
oracle's top-2 margin exceeds 5e-2; acceptance lengths, committed ids and lengths bit-exact given
the GPU's own draft and verify argmaxes.
"""
import pytest
import torch

import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, gpu_state, make_pair, top2_margin

pytestmark = pytest.mark.gpu

CFG = synth.SMALL_BF16
TOL = 2e-2
MARGIN = 5e-2


def _check_logits(gl, ol):
    err = (gl.double() - ol.double()).abs().max().item()
    assert err < TOL, err
    marg = top2_margin(ol)
    am_g = gl.argmax(-1)
    am_o = odec.argmax_lowest(ol.double())
    sure = marg > MARGIN
    assert torch.equal(am_g[sure], am_o[sure])
    return err


@pytest.mark.parametrize("B,P", [(1, 100), (3, 77)])
def test_forward_logits_all_modes(B, P):
    ctx, om, _ = make_pair(CFG)
    p = synth.prompt_tokens(B, P, CFG.vocab, seed=4)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, CFG.max_seq + 64)
    k = CFG.block_k
    lens, pend, _, _ = gpu_state(ctx, B)
    assert lens == st.lens and pend == st.pending
    gl = gpu_logits(ctx, 1, B, k)
    ol = odec.draft_forward(om, st, k)
    _check_logits(gl, ol)
    _, _, draft, _ = gpu_state(ctx, B)
    assert draft == gl.argmax(-1).tolist()
    gv = gpu_logits(ctx, 2, B, k + 1)
    ov = odec.verify_forward(om, st, draft)
    _check_logits(gv, ov)
    gd = gpu_logits(ctx, 3, B, k)
    _check_logits(gd, ol)
    ga = gpu_logits(ctx, 0, B, 1)
    st2 = odec.prefill(om, p, CFG.max_seq + 64)
    _check_logits(ga, odec.ar_forward(om, st2))


@pytest.mark.parametrize("kernel,tile", [(3, 64), (3, 128), (4, 64), (4, 128)])
@pytest.mark.parametrize("B,P", [(1, 100), (3, 77)])
def test_draft_verify_logits_each_tcgen05_attention_form(kernel, tile, B, P):
    """The model's own attention launches (fp32 q and P as (hi, lo) operands) on the tcgen05
    kernel with 2 / 4 softmax threads per row and 64- / 128-key KV tiles, whatever the planner
    would pick: draft and verify logits within the bar."""
    import self_speculation_b200 as nb
    lib = nb.load_library()
    assert lib.nld_debug_attention_kernel(kernel) == 0
    assert lib.nld_debug_attention_tile(tile) == 0
    try:
        ctx, om, _ = make_pair(CFG)
        p = synth.prompt_tokens(B, P, CFG.vocab, seed=4)
        ctx.nld_prefill(p.cuda())
        st = odec.prefill(om, p, CFG.max_seq + 64)
        k = CFG.block_k
        gl = gpu_logits(ctx, 1, B, k)
        _check_logits(gl, odec.draft_forward(om, st, k))
        _, _, draft, _ = gpu_state(ctx, B)
        gv = gpu_logits(ctx, 2, B, k + 1)
        _check_logits(gv, odec.verify_forward(om, st, draft))
        del ctx
    finally:
        assert lib.nld_debug_attention_kernel(0) == 0
        assert lib.nld_debug_attention_tile(0) == 0


def test_rounds_commit_bit_exact_given_argmaxes():
    """Teacher-forced over several rounds: the oracle replays each round's commit on the GPU's
    draft and verify argmaxes; tokens, counts, lengths and pending tokens must match exactly,
    and the oracle's own logits for that round must agree with the GPU's argmaxes."""
    B = 2
    ctx, om, _ = make_pair(CFG)
    p = synth.prompt_tokens(B, 130, CFG.vocab, seed=5)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, CFG.max_seq + 64)
    k = CFG.block_k
    toks = torch.empty(B, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(B, dtype=torch.int32, device="cuda")
    for _ in range(4):
        ctx.nld_selfspec_round(toks, nc, None)
        ctx.nld_sync()
        lens, pend, draft, ver = gpu_state(ctx, B)
        # oracle logits of this round's forwards, on the GPU's drafts
        ol = odec.draft_forward(om, st, k)
        marg = top2_margin(ol)
        am = odec.argmax_lowest(ol)
        sure = marg > MARGIN
        assert torch.equal(torch.tensor(draft)[sure], am[sure])
        ov = odec.verify_forward(om, st, draft)
        vm = top2_margin(ov)
        assert torch.equal(torch.tensor(ver)[vm > MARGIN], odec.argmax_lowest(ov)[vm > MARGIN])
        committed = [odec.commit_after_verify(draft[b], ver[b]) for b in range(B)]
        for b in range(B):
            c = int(nc[b])
            assert c == len(committed[b])
            assert toks[b, :c].cpu().tolist() == committed[b]
        odec.apply_commit(st, committed)
        assert lens == st.lens and pend == st.pending


def test_forced_commit_sweep_bit_exact():
    ctx, om, _ = make_pair(CFG)
    p = synth.prompt_tokens(1, 64, CFG.vocab, seed=6)
    ctx.nld_prefill(p.cuda())
    k = CFG.block_k
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    expect_len = 63
    for c in [1, 2, 17, 32, 33]:
        force = torch.tensor([c], dtype=torch.int32, device="cuda")
        ctx.nld_selfspec_round(toks, nc, force)
        ctx.nld_sync()
        lens, pend, draft, ver = gpu_state(ctx, 1)
        want = odec.commit_after_verify(draft[0], ver[0], forced=c)
        assert toks[0, :c].cpu().tolist() == want and int(nc.item()) == c
        expect_len += c
        assert lens[0] == expect_len and pend[0] == want[-1]


def test_split_commit_path_matches_round():
    """nld_selfspec_draft_verify + nld_kv_commit == nld_selfspec_round (deterministic kernels)."""
    p = synth.prompt_tokens(1, 90, CFG.vocab, seed=7)
    k = CFG.block_k
    res = []
    for split in (False, True):
        ctx, _, _ = make_pair(CFG)
        ctx.nld_prefill(p.cuda())
        toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
        nc = torch.empty(1, dtype=torch.int32, device="cuda")
        seq = []
        for _ in range(3):
            if split:
                ctx.nld_selfspec_draft_verify()
                ctx.nld_kv_commit(None, toks, nc)
            else:
                ctx.nld_selfspec_round(toks, nc, None)
            ctx.nld_sync()
            seq.append(toks[0, :int(nc.item())].cpu().tolist())
        res.append(seq)
    assert res[0] == res[1]


def test_diffusion_step_commit_rule_given_gpu_confidences():
    """Peaky logits (LM head x40) so several slots pass tau: the committed slots must be exactly
    those the rule picks from the GPU's own confidences; the block then fills and the lengths
    and pending tokens match the oracle's KV-fill bookkeeping."""
    B = 2
    W = synth.model_weights(CFG, 0, lm_head_scale=40.0)
    ctx, om, _ = make_pair(CFG, weights=W)
    p = synth.prompt_tokens(B, 70, CFG.vocab, seed=8)
    ctx.nld_prefill(p.cuda())
    k = CFG.block_k
    blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(B, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(B, dtype=torch.int32, device="cuda")
    prev = [[CFG.vocab] * k for _ in range(B)]
    filled = False
    multi = 0
    for step in range(k + 1):
        filled = ctx.nld_diffuse_block_step(0.9, blk, conf, nc)
        g_conf = conf.cpu()
        g_blk = blk.cpu().tolist()
        for b in range(B):
            masked = [t == CFG.vocab for t in prev[b]]
            if not any(masked):
                assert int(nc[b]) == 0
                continue
            pick = odec.diffusion_commit(masked, g_conf[b].tolist(), 0.9)
            assert int(nc[b]) == sum(pick)
            multi = max(multi, sum(pick))
            for s in range(k):
                if pick[s]:
                    assert g_blk[b][s] != CFG.vocab
                else:
                    assert g_blk[b][s] == prev[b][s]
        prev = [list(r) for r in g_blk]
        if filled:
            break
    assert filled and multi > 1
    assert all(CFG.vocab not in r for r in prev)
    lens, pend, _, _ = gpu_state(ctx, B)
    assert lens == [69 + k] * B
    assert pend == [prev[b][k - 1] for b in range(B)]


def test_diffusion_confidence_matches_oracle():
    """conf = 1/sum_v exp(l_v - l_max): logits within eps give conf within a factor exp(2 eps),
    so the 2e-2 logit bar bounds the relative confidence error by ~4e-2."""
    ctx, om, _ = make_pair(CFG)
    p = synth.prompt_tokens(1, 66, CFG.vocab, seed=11)
    ctx.nld_prefill(p.cuda())
    k = CFG.block_k
    blk = torch.empty(1, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(1, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    st = odec.prefill(om, p, CFG.max_seq + 64)
    st.block = [[CFG.vocab] * k]
    ol = odec.diffusion_forward(om, st, k)
    ctx.nld_diffuse_block_step(0.9, blk, conf, nc)
    oc = odec.confidence(ol.double())[0]
    rel = ((conf.cpu()[0].double() - oc) / oc).abs().max().item()
    assert rel < 4e-2, rel


def test_ar_steps_track_oracle_teacher_forced():
    B = 2
    ctx, om, _ = make_pair(CFG)
    p = synth.prompt_tokens(B, 65, CFG.vocab, seed=9)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, CFG.max_seq + 64)
    t = torch.empty(B, dtype=torch.int32, device="cuda")
    for _ in range(5):
        ol = odec.ar_forward(om, st)
        ctx.nld_ar_step(t)
        ctx.nld_sync()
        got = t.cpu().tolist()
        marg = top2_margin(ol[:, 0])
        want = odec.argmax_lowest(ol[:, 0]).tolist()
        for b in range(B):
            if marg[b] > MARGIN:
                assert got[b] == want[b]
            st.lens[b] += 1
            st.pending[b] = got[b]


def test_batch_rows_independent():
    """A sequence's logits do not depend on the other sequences of the batch beyond rounding:
    a different batch changes the GEMM tiling (summation order, then bf16 activation rounding),
    so the bar is the logit bar itself, plus argmax agreement where the margin is clear."""
    p = synth.prompt_tokens(3, 80, CFG.vocab, seed=10)
    ctx, _, _ = make_pair(CFG)
    ctx.nld_prefill(p.cuda())
    all3 = gpu_logits(ctx, 1, 3, CFG.block_k)
    ctx1, _, _ = make_pair(CFG)
    ctx1.nld_prefill(p[1:2].cuda())
    one = gpu_logits(ctx1, 1, 1, CFG.block_k)
    assert (all3[1] - one[0]).abs().max().item() < TOL
    sure = top2_margin(one[0]) > MARGIN
    assert torch.equal(all3[1].argmax(-1)[sure], one[0].argmax(-1)[sure])
