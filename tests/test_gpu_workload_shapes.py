"""Parity at the shapes of the benchmarked workloads beyond the 8B self-speculation round.

* 14B layer shape (40 q / 8 kv heads: GQA group 5; d 5120: 40 row tiles; FFN 17408; vocab
  151936), 2 layers: batch 1 on the decode path, and batch 64 (M = 64 x 33 = 2112 token rows,
  the wide-tile path with 17 token tiles) compared on sampled sequences.
* 8B layer shape, 2 layers: a diffusion step at batch 16 (M = 512) and the fused diffusion fill
  at batch 4 (one forward of 4 x 2k = 256 rows, two token tiles).

Bars (the decode round's, against the oracle as specified: bf16 weights and KV cache, fp32
accumulation and activations): logits max-abs error <= 2e-2, argmax equal wherever the oracle's
top-2 margin exceeds 5e-2; confidences within a factor exp(2 * 2e-2) (a logit error e moves the
largest softmax probability by at most a factor exp(2e)); commit decisions exact given the
GPU's own confidences.  Sequences never see one another, so a sampled sequence's oracle runs on
that sequence alone.
"""
import pytest
import torch

import oracle
import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, gpu_state, make_pair, top2_margin

pytestmark = pytest.mark.gpu

TOL = 2e-2
MARGIN = 5e-2


def _check(gl, ol):
    err = (gl.double() - ol.double()).abs().max().item()
    assert err <= TOL, err
    sure = top2_margin(ol) > MARGIN
    assert sure.float().mean().item() >= 0.5
    assert torch.equal(gl.argmax(-1)[sure], odec.argmax_lowest(ol.double())[sure])


@pytest.fixture(scope="module")
def w14():
    cfg = synth.LLAMA14B.replace(n_layers=2, max_batch=64, max_seq=192)
    return cfg, synth.model_weights(cfg, 0, device="cuda")


def test_14b_layer_shape_batch1(w14):
    cfg, W = w14
    ctx, om, _ = make_pair(cfg.replace(max_batch=1), weights=W, device_weights=True)
    p = synth.prompt_tokens(1, 100, cfg.vocab, seed=13)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, cfg.max_seq + 64)
    k = cfg.block_k
    gl = gpu_logits(ctx, 1, 1, k)
    _check(gl, odec.draft_forward(om, st, k))
    _, _, draft, _ = gpu_state(ctx, 1)
    gv = gpu_logits(ctx, 2, 1, k + 1)
    _check(gv, odec.verify_forward(om, st, draft))
    ctx.close()


def test_14b_batch64_wide_tiles_sampled(w14):
    cfg, W = w14
    B, P, k = 64, 40, cfg.block_k
    ctx, om, _ = make_pair(cfg, weights=W, device_weights=True)
    p = synth.prompt_tokens(B, P, cfg.vocab, seed=14)
    ctx.nld_prefill(p.cuda())
    dl = torch.empty(B, k, cfg.vocab, dtype=torch.float32, device="cuda")
    ctx.nld_debug_logits(1, dl)
    ctx.nld_sync()
    _, _, draft, _ = gpu_state(ctx, B)
    vl = torch.empty(B, k + 1, cfg.vocab, dtype=torch.float32, device="cuda")
    ctx.nld_debug_logits(2, vl)
    ctx.nld_sync()
    for b in (0, 29, 63):
        st = odec.prefill(om, p[b:b + 1], cfg.max_seq + 64)
        _check(dl[b:b + 1].cpu(), odec.draft_forward(om, st, k))
        _check(vl[b:b + 1].cpu(), odec.verify_forward(om, st, [draft[b]]))
    ctx.close()


@pytest.fixture(scope="module")
def w8():
    cfg = synth.LLAMA8B.replace(n_layers=2, max_batch=16, max_seq=256)
    return cfg, synth.model_weights(cfg, 0, device="cuda")


def test_8b_diffusion_step_batch16(w8):
    cfg, W = w8
    B, k = 16, cfg.block_k
    ctx, om, _ = make_pair(cfg, weights=W, device_weights=True)
    p = synth.prompt_tokens(B, 64, cfg.vocab, seed=15)
    ctx.nld_prefill(p.cuda())
    gl = torch.empty(B, k, cfg.vocab, dtype=torch.float32, device="cuda")
    ctx.nld_debug_logits(3, gl)
    ctx.nld_sync()
    blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(B, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(B, dtype=torch.int32, device="cuda")
    ctx.nld_diffuse_block_step(0.9, blk, conf, nc)
    g_conf, g_blk = conf.cpu(), blk.cpu().tolist()
    for b in range(B):
        pick = odec.diffusion_commit([True] * k, g_conf[b].tolist(), 0.9)
        assert int(nc[b]) == sum(pick) >= 1
        assert all((g_blk[b][s] != cfg.vocab) == pick[s] for s in range(k))
    for b in (0, 15):
        st = odec.prefill(om, p[b:b + 1], cfg.max_seq + 64)
        st.block = [[cfg.vocab] * k]
        ol = odec.diffusion_forward(om, st, k)
        _check(gl[b:b + 1].cpu(), ol)
        oc = odec.confidence(ol.double())[0]
        assert ((g_conf[b].double() - oc) / oc).abs().max().item() < 4e-2
    ctx.close()


def test_8b_fused_fill_batch4(w8):
    cfg, W = w8
    B, k = 4, cfg.block_k
    ctx, om, _ = make_pair(cfg.replace(max_batch=4), weights=W, device_weights=True)
    p = synth.prompt_tokens(B, 70, cfg.vocab, seed=16)
    ctx.nld_prefill(p.cuda())
    blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(B, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(B, dtype=torch.int32, device="cuda")
    assert not ctx.nld_diffuse_block_step_fused(0.0, blk, conf, nc)   # tau 0 completes every block
    prev = blk.cpu().tolist()
    assert all(cfg.vocab not in r for r in prev)
    lens0, _, _, _ = gpu_state(ctx, B)
    assert ctx.nld_diffuse_block_step_fused(0.9, blk, conf, nc)       # fused fill + first step
    lens, pend, _, _ = gpu_state(ctx, B)
    assert lens == [l + k for l in lens0]
    assert pend == [prev[b][k - 1] for b in range(B)]
    g_conf, g_blk = conf.cpu(), blk.cpu().tolist()
    for b in range(B):
        pick = odec.diffusion_commit([True] * k, g_conf[b].tolist(), 0.9)
        assert int(nc[b]) == sum(pick) >= 1
        assert all((g_blk[b][s] != cfg.vocab) == pick[s] for s in range(k))
    for b in (0, 3):
        st = odec.prefill(om, p[b:b + 1], cfg.max_seq + 64)
        st.block = [prev[b]]
        oc = odec.confidence(odec.fill_diffusion_forward(om, st, k).double())[0]
        assert ((g_conf[b].double() - oc) / oc).abs().max().item() < 4e-2
    ctx.close()
