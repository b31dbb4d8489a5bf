"""nld_diffuse_block_step_fused: the diffusion KV fill deferred into the next block's first
denoising step (one forward of 2k rows: k causal rows that write the complete block's KV, then
the new block).

fp32 tiny model: token-exact against the oracle's fused driver (itself pinned equal to the
unfused driver, tests/test_oracle_pins.py), with one call per denoising step and no separate
fill forwards.  bf16 small model (k = 32, 2k = 64 rows per sequence, batch 2): the fused call's
bookkeeping (len += k, pending = b_k) and commit rule given the GPU's own confidences, and its
confidences against the oracle's fused forward (bar: conf within a factor exp(2 * 2e-2)).
"""
import pytest
import torch

import synth
from oracle import decode as odec
from tests._helpers import gpu_state, make_pair

pytestmark = pytest.mark.gpu


def _gpu_diffuse_fused(ctx, cfg, n, tau, B=1):
    k = cfg.block_k
    blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(B, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(B, dtype=torch.int32, device="cuda")
    out, calls, fills = [], 0, 0
    pending = False
    while len(out) < n:
        filled = ctx.nld_diffuse_block_step_fused(tau, blk, conf, nc)
        calls += 1
        assert filled == pending            # a deferred fill runs in the next call
        b0 = blk[0].cpu().tolist()
        pending = cfg.vocab not in b0
        fills += int(filled)
        if pending:
            out += b0
    return out[:n], calls, fills, pending


@pytest.mark.parametrize("scale,tau", [(1.0, 0.9), (60.0, 0.9), (1.0, 1.5), (1.0, 0.0)])
def test_fused_generation_token_exact_f32(scale, tau):
    cfg = synth.TINY_F32
    W = synth.model_weights(cfg, 0, lm_head_scale=scale)
    ctx, om, _ = make_pair(cfg, weights=W)
    p = synth.prompt_tokens(1, 64, cfg.vocab, seed=1)
    ctx.nld_prefill(p.cuda())
    got, calls, fills, pending = _gpu_diffuse_fused(ctx, cfg, 32, tau)
    want, forwards, steps = odec.diffuse_generate_fused(om, p, 32, cfg.block_k, tau, 256)
    assert got == want[0]
    assert calls == steps == forwards
    # the fill still deferred after the last block runs alone before the next decode call
    lens, _, _, _ = gpu_state(ctx, 1)
    assert pending and lens[0] == 63 + fills * cfg.block_k
    tok = torch.empty(1, dtype=torch.int32, device="cuda")
    ctx.nld_ar_step(tok)
    lens, _, _, _ = gpu_state(ctx, 1)
    assert lens[0] == 63 + (fills + 1) * cfg.block_k + 1


def test_fused_step_bookkeeping_and_commit_rule_bf16():
    cfg = synth.SMALL_BF16
    B, k = 2, synth.SMALL_BF16.block_k
    W = synth.model_weights(cfg, 0, lm_head_scale=40.0)
    ctx, om, _ = make_pair(cfg, weights=W)
    p = synth.prompt_tokens(B, 70, cfg.vocab, seed=8)
    ctx.nld_prefill(p.cuda())
    blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(B, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(B, dtype=torch.int32, device="cuda")
    # tau 0 completes every block in one step: each later call is a fused fill + first step
    first = ctx.nld_diffuse_block_step_fused(0.0, blk, conf, nc)
    assert not first and cfg.vocab not in blk.cpu().flatten().tolist()
    prev = blk.cpu().tolist()
    lens0, _, _, _ = gpu_state(ctx, B)
    filled = ctx.nld_diffuse_block_step_fused(0.9, blk, conf, nc)
    assert filled
    lens, pend, _, _ = gpu_state(ctx, B)
    assert lens == [l + k for l in lens0]
    assert pend == [prev[b][k - 1] for b in range(B)]
    g_conf, g_blk = conf.cpu(), blk.cpu().tolist()
    for b in range(B):
        pick = odec.diffusion_commit([True] * k, g_conf[b].tolist(), 0.9)
        assert int(nc[b]) == sum(pick) >= 1
        for s in range(k):
            assert (g_blk[b][s] != cfg.vocab) == pick[s]


def test_fused_confidence_matches_oracle_bf16():
    cfg = synth.SMALL_BF16
    k = cfg.block_k
    ctx, om, _ = make_pair(cfg)
    p = synth.prompt_tokens(1, 66, cfg.vocab, seed=11)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, cfg.max_seq + 64)
    blk = torch.empty(1, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(1, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    ctx.nld_diffuse_block_step_fused(0.0, blk, conf, nc)   # one step completes the block
    st.block = [blk[0].cpu().tolist()]
    ctx.nld_diffuse_block_step_fused(0.9, blk, conf, nc)   # fused fill + first step
    ol = odec.fill_diffusion_forward(om, st, k)
    oc = odec.confidence(ol.double())[0]
    rel = ((conf.cpu()[0].double() - oc) / oc).abs().max().item()
    assert rel < 4e-2, rel
