"""fp32 tiny model (2 layers, d 256, 4x64 heads, FFN 1024, vocab 4096+MASK, k=8): the CUDA
library against the fp64 oracle — logits within 1e-4, token-exact generation in all three
modes (AR, self-speculation, diffusion)."""
import pytest
import torch

import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, gpu_state, make_pair

pytestmark = pytest.mark.gpu

CFG = synth.TINY_F32
TOL = 1e-4


def _prompt(B=1, P=64, seed=1):
    return synth.prompt_tokens(B, P, CFG.vocab, seed=seed)


def test_logits_draft_verify_ar_match_oracle():
    ctx, om, _ = make_pair(CFG)
    p = _prompt()
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, 256)
    k = CFG.block_k
    lens, pend, _, _ = gpu_state(ctx, 1)
    assert lens == st.lens and pend == st.pending
    gl = gpu_logits(ctx, 1, 1, k)                       # draft
    ol = odec.draft_forward(om, st, k)
    assert (gl.double() - ol).abs().max().item() < TOL
    _, _, draft, _ = gpu_state(ctx, 1)
    assert draft == odec.argmax_lowest(ol).tolist()
    gv = gpu_logits(ctx, 2, 1, k + 1)                   # verify on the GPU's drafts
    ov = odec.verify_forward(om, st, draft)
    assert (gv.double() - ov).abs().max().item() < TOL
    ga = gpu_logits(ctx, 0, 1, 1)                       # AR
    st2 = odec.prefill(om, p, 256)
    oa = odec.ar_forward(om, st2)
    assert (ga.double() - oa).abs().max().item() < TOL
    gd = gpu_logits(ctx, 3, 1, k)                       # diffusion (all open == draft)
    assert (gd.double() - ol).abs().max().item() < TOL


def _gpu_selfspec(ctx, n, k, force=None):
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    out, per = [], []
    while len(out) < n:
        ctx.nld_selfspec_round(toks, nc, force)
        ctx.nld_sync()
        c = int(nc.item())
        per.append(c)
        out += toks[0, :c].cpu().tolist()
    return out[:n], per


def test_selfspec_and_ar_generation_token_exact():
    ctx, om, _ = make_pair(CFG)
    p = _prompt()
    ctx.nld_prefill(p.cuda())
    got, per = _gpu_selfspec(ctx, 64, CFG.block_k)
    want, wper = odec.selfspec_generate(om, p, 64, CFG.block_k, 256)
    ar = odec.ar_generate(om, p, 64, 256)
    assert got == want[0] == ar[0]
    assert all(1 <= c <= CFG.block_k + 1 for c in per)
    # AR steps through the library
    ctx2, _, _ = make_pair(CFG)
    ctx2.nld_prefill(p.cuda())
    t = torch.empty(1, dtype=torch.int32, device="cuda")
    seq = []
    for _ in range(64):
        ctx2.nld_ar_step(t)
        ctx2.nld_sync()
        seq.append(int(t.item()))
    assert seq == ar[0]


def test_selfspec_multi_accept_token_exact():
    """Peaky LM head tied to the embedding makes drafts match: exercises a > 0 commits."""
    W = synth.model_weights(CFG, 5)
    W[-1] = (W[0][:CFG.vocab].clone() * 50.0)
    ctx, om, _ = make_pair(CFG, weights=W)
    p = _prompt(seed=9)
    ctx.nld_prefill(p.cuda())
    got, per = _gpu_selfspec(ctx, 48, CFG.block_k)
    want, _ = odec.selfspec_generate(om, p, 48, CFG.block_k, 256)
    assert got == want[0]
    assert max(per) > 1


def _gpu_diffuse(ctx, n, k, tau):
    blk = torch.empty(1, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(1, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    out, steps = [], 0
    while len(out) < n:
        filled = ctx.nld_diffuse_block_step(tau, blk, conf, nc)
        steps += 1
        assert int(nc.item()) >= 1
        if filled:
            out += blk[0].cpu().tolist()
    return out[:n], steps


@pytest.mark.parametrize("scale,tau", [(1.0, 0.9), (60.0, 0.9), (1.0, 1.5), (1.0, 0.0)])
def test_diffusion_generation_token_exact(scale, tau):
    W = synth.model_weights(CFG, 0, lm_head_scale=scale)
    ctx, om, _ = make_pair(CFG, weights=W)
    p = _prompt()
    ctx.nld_prefill(p.cuda())
    got, steps = _gpu_diffuse(ctx, 32, CFG.block_k, tau)
    want, wsteps = odec.diffuse_generate(om, p, 32, CFG.block_k, tau, 256)
    assert got == want[0]
    assert steps == wsteps


def test_forced_commit_counts():
    ctx, om, _ = make_pair(CFG)
    p = _prompt()
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, 256)
    k = CFG.block_k
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    for c in [k + 1, 1, 4, k]:
        force = torch.tensor([c], dtype=torch.int32, device="cuda")
        ctx.nld_selfspec_round(toks, nc, force)
        ctx.nld_sync()
        committed, drafts, ver, _, _ = odec.selfspec_round(om, st, k, forced=[c])
        assert int(nc.item()) == c
        assert toks[0, :c].cpu().tolist() == committed[0]
        assert toks[0, c:].cpu().tolist() == [-1] * (k + 1 - c)
        lens, pend, _, _ = gpu_state(ctx, 1)
        assert lens == st.lens and pend == st.pending


def test_prompt_of_one_token_and_block_of_one():
    cfg = CFG.replace(block_k=1)
    ctx, om, _ = make_pair(cfg)
    p = _prompt(P=1)
    ctx.nld_prefill(p.cuda())
    toks = torch.empty(1, 2, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    out = []
    while len(out) < 10:
        ctx.nld_selfspec_round(toks, nc, None)
        ctx.nld_sync()
        out += toks[0, :int(nc.item())].cpu().tolist()
    want = odec.ar_generate(om, p, 10, 64)
    assert out[:10] == want[0]


def test_kv_full_is_reported_before_launch():
    cfg = CFG.replace(max_seq=80)
    ctx, om, _ = make_pair(cfg)
    ctx.nld_prefill(_prompt(P=64).cuda())
    toks = torch.empty(1, cfg.block_k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    import self_speculation_b200 as nb
    with pytest.raises(nb.NldError) as ei:
        for _ in range(40):
            ctx.nld_selfspec_round(toks, nc, None)
    assert ei.value.status == 4
    ctx.nld_sync()                        # no device error: nothing was written past capacity
    lens, _, _, _ = gpu_state(ctx, 1)
    assert lens[0] <= 80


def test_diffusion_confidence_matches_oracle_f32():
    ctx, om, _ = make_pair(CFG)
    p = _prompt()
    ctx.nld_prefill(p.cuda())
    k = CFG.block_k
    blk = torch.empty(1, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(1, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    st = odec.prefill(om, p, 256)
    r = odec.diffusion_step(om, st, k, 0.9)
    ctx.nld_diffuse_block_step(0.9, blk, conf, nc)
    rel = ((conf.cpu()[0].double() - r["conf"][0]) / r["conf"][0]).abs().max().item()
    assert rel < 1e-3
    assert blk.cpu()[0].tolist() == st.block[0] or r["filled"]
