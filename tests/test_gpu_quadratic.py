"""Quadratic self-speculation on the GPU (nld_quadratic_round), against the oracle's reading of
the mode (ranhao.site notes section 8.1; shilu.ai blog, performance highlights: the mode is named
and credited with more tokens per forward, not defined): one forward per round of (k+1)^2 rows,
the causal verify rows of the current drafts plus a pre-draft block for every acceptance
outcome; the round commits like the linear round and the block of the outcome that happened
gives the next drafts.

fp32 tiny model (k = 8, 81 rows per forward): generation token-exact against
oracle.decode.quadratic_generate, equal to AR greedy (lossless), one forward per round; with a
peaky LM head tied to the embedding, rounds accept several drafts, so the block choice matters.
bf16 small shape (k = 32, 1089 rows per forward: wide tiles, two-interval attention masks,
RoPE positions apart from KV slots): the quadratic forward's logits within 2e-2 of the oracle
with argmax agreement where the top-2 margin exceeds 5e-2, and rounds whose commits and next
drafts are bit-exact given the GPU's own argmaxes.
"""
import pytest
import torch

import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, gpu_state, make_pair, top2_margin

pytestmark = pytest.mark.gpu


def _gpu_quadratic(ctx, n, k):
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    out, per = [], []
    while len(out) < n:
        ctx.nld_quadratic_round(toks, nc)
        ctx.nld_sync()
        c = int(nc.item())
        per.append(c)
        out += toks[0, :c].cpu().tolist()
    return out[:n], per


@pytest.mark.parametrize("peaky", [False, True])
def test_quadratic_generation_token_exact_f32(peaky):
    cfg = synth.TINY_F32.replace(max_seq=320)
    W = synth.model_weights(cfg, 5)
    if peaky:
        W[-1] = W[0][:cfg.vocab].clone() * 50.0
    ctx, om, _ = make_pair(cfg, weights=W)
    p = synth.prompt_tokens(1, 64, cfg.vocab, seed=9)
    ctx.nld_prefill(p.cuda())
    got, per = _gpu_quadratic(ctx, 48, cfg.block_k)
    want, forwards, wper = odec.quadratic_generate(om, p, 48, cfg.block_k, 400)
    assert got == want[0]
    assert per == wper[0] and forwards == len(per) + 1
    assert got == odec.ar_generate(om, p, 48, 400)[0]
    if peaky:
        assert max(per) > 1


def test_quadratic_forward_logits_bf16():
    cfg = synth.SMALL_BF16.replace(max_seq=1600)
    k = cfg.block_k
    ctx, om, _ = make_pair(cfg)
    p = synth.prompt_tokens(1, 100, cfg.vocab, seed=17)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, cfg.max_seq + 64)
    gpu_logits(ctx, 1, 1, k)                      # draft forward: stores the drafts
    _, _, draft, _ = gpu_state(ctx, 1)
    gq = gpu_logits(ctx, 4, 1, (k + 1) * (k + 1))
    ov, op = odec.quadratic_forward(om, st, draft)
    ol = torch.cat([ov, op.reshape(1, (k + 1) * k, -1)], dim=1)
    err = (gq.double() - ol.double()).abs().max().item()
    assert err < 2e-2, err
    sure = top2_margin(ol) > 5e-2
    assert torch.equal(gq.argmax(-1)[sure], odec.argmax_lowest(ol.double())[sure])


def test_quadratic_rounds_bf16_bit_exact_given_argmaxes():
    cfg = synth.SMALL_BF16.replace(max_seq=1600)
    k = cfg.block_k
    W = synth.model_weights(cfg, 0)
    W[-1] = (W[0][:cfg.vocab].float() * 30.0).to(W[-1].dtype)   # peaky, tied: drafts get accepted
    ctx, om, _ = make_pair(cfg, weights=W)
    p = synth.prompt_tokens(1, 90, cfg.vocab, seed=18)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, cfg.max_seq + 64)
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    # the first round begins with a linear draft forward (deterministic): the debug draft
    # forward gives the same drafts, which the round then verifies
    gpu_logits(ctx, 1, 1, k)
    _, _, drafts, _ = gpu_state(ctx, 1)
    for _ in range(4):
        ctx.nld_quadratic_round(toks, nc)
        ctx.nld_sync()
        lens, pend, nxt, ver = gpu_state(ctx, 1)
        vl, pl = odec.quadratic_forward(om, st, drafts)
        sure = top2_margin(vl[0]) > 5e-2
        assert torch.equal(torch.tensor(ver[0])[sure], odec.argmax_lowest(vl[0])[sure])
        # commit from the GPU's verify argmaxes, against the drafts it verified
        want = odec.commit_after_verify(drafts[0], ver[0])
        c = int(nc.item())
        assert c == len(want) and toks[0, :c].cpu().tolist() == want
        # the next drafts are the argmaxes of pre-draft block c-1 of the oracle's forward
        blk = pl[0, c - 1]
        sure = top2_margin(blk) > 5e-2
        assert torch.equal(torch.tensor(nxt[0])[sure], odec.argmax_lowest(blk)[sure])
        odec.apply_commit(st, [want])
        assert lens == st.lens and pend == st.pending
        drafts = nxt
