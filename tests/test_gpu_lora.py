"""LoRA drafter (nld_init_lora): a low-rank delta scale * B (A att) on o_proj in the
block-bidirectional forwards only (Nemotron-Labs-Diffusion notes, ranhao.site, section 6).

fp32 tiny model (rank 8): draft logits within 1e-4 of the fp64 oracle with the same adapter,
verify and AR logits equal to the adapter-free oracle's, token-exact self-speculation (with
the oracle's per-round acceptance counts, which depend on the drafts) and diffusion (unfused
and fused fill).  bf16 (the adapter folded into the layer chain: z = scale * A att beside the
attention output, B as more K columns of the O projection): draft and diffusion logits of the
small model (rank 128, the pages' rank; rank 16, zero-padded to a whole k tile) and draft
logits at the 8B layer shape within 2e-2 of the oracle.  Host logic: rank changes are refused,
rank 0 switches the adapter off and the forwards return to the adapter-free results bit for bit.
"""
import pytest
import torch

import self_speculation_b200 as nb
import synth
from oracle import decode as odec
from tests._helpers import gpu_logits, gpu_state, make_pair

pytestmark = pytest.mark.gpu


def _adapter(cfg, r, seed, std):
    """A [r, Hq*hd], B [d, r] per layer, in the config dtype."""
    flat = synth.lora_weights(cfg, r, seed, std)
    return flat[0::2], flat[1::2]


def _load(ctx, om, A, B, scale):
    flat = [t for pair in zip(A, B) for t in pair]
    ctx.nld_init_lora(len(A[0]), scale, flat)
    om.set_lora([a.double() for a in A], [b.double() for b in B], scale)


def test_draft_logits_and_frozen_paths_f32():
    cfg = synth.TINY_F32
    ctx, om, W = make_pair(cfg)
    _, plain, _ = make_pair(cfg, weights=W)
    A, B = _adapter(cfg, 8, seed=7, std=0.05)
    _load(ctx, om, A, B, 5.0)
    p = synth.prompt_tokens(1, 64, cfg.vocab, seed=1)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, 256)
    k = cfg.block_k
    gl = gpu_logits(ctx, 1, 1, k)
    ol = odec.draft_forward(om, st, k)
    assert (gl.double() - ol).abs().max().item() < 1e-4
    # not vacuous: the adapter moves the drafter's logits well beyond the bar
    assert (ol - odec.draft_forward(plain, st, k)).abs().max().item() > 0.1
    _, _, draft, _ = gpu_state(ctx, 1)
    gv = gpu_logits(ctx, 2, 1, k + 1)
    assert (gv.double() - odec.verify_forward(plain, st, draft)).abs().max().item() < 1e-4
    ga = gpu_logits(ctx, 0, 1, 1)
    assert (ga.double() - odec.ar_forward(plain, st)).abs().max().item() < 1e-4


def _gpu_selfspec(ctx, n, k):
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    out, per = [], []
    while len(out) < n:
        ctx.nld_selfspec_round(toks, nc, None)
        ctx.nld_sync()
        c = int(nc.item())
        per.append(c)
        out += toks[0, :c].cpu().tolist()
    return out[:n], per


def test_selfspec_token_exact_with_oracle_acceptance_f32():
    cfg = synth.TINY_F32
    W = synth.model_weights(cfg, 5)
    W[-1] = W[0][:cfg.vocab].clone() * 50.0        # peaky head tied to the embedding: drafts hit
    ctx, om, _ = make_pair(cfg, weights=W)
    A, B = _adapter(cfg, 8, seed=3, std=0.02)
    _load(ctx, om, A, B, 5.0)
    p = synth.prompt_tokens(1, 64, cfg.vocab, seed=9)
    ctx.nld_prefill(p.cuda())
    got, per = _gpu_selfspec(ctx, 48, cfg.block_k)
    want, wper = odec.selfspec_generate(om, p, 48, cfg.block_k, 256)
    assert got == want[0]
    # lossless: the adapter changes the drafts, never the committed tokens
    assert got == odec.ar_generate(om, p, 48, 256)[0]
    assert per == wper[0][:len(per)]


def _gpu_diffuse(ctx, n, k, tau, fused):
    """Generate n tokens by diffusion steps; with the fused call a block is complete when no
    mask is left in it (its fill runs inside the next call)."""
    blk = torch.empty(1, k, dtype=torch.int32, device="cuda")
    conf = torch.empty(1, k, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    out, steps = [], 0
    while len(out) < n:
        if fused:
            ctx.nld_diffuse_block_step_fused(tau, blk, conf, nc)
            done = ctx.cfg.mask_id not in blk[0].cpu().tolist()
        else:
            done = ctx.nld_diffuse_block_step(tau, blk, conf, nc)
        steps += 1
        if done:
            out += blk[0].cpu().tolist()
    return out[:n], steps


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("scale,tau", [(5.0, 0.9), (20.0, 0.9)])
def test_diffusion_token_exact_f32(fused, scale, tau):
    cfg = synth.TINY_F32
    W = synth.model_weights(cfg, 0, lm_head_scale=60.0)
    ctx, om, _ = make_pair(cfg, weights=W)
    _, plain, _ = make_pair(cfg, weights=W)
    A, B = _adapter(cfg, 8, seed=7, std=0.05)
    _load(ctx, om, A, B, scale)
    p = synth.prompt_tokens(1, 64, cfg.vocab, seed=1)
    ctx.nld_prefill(p.cuda())
    got, steps = _gpu_diffuse(ctx, 32, cfg.block_k, tau, fused)
    if fused:
        want, forwards, wsteps = odec.diffuse_generate_fused(om, p, 32, cfg.block_k, tau, 256)
    else:
        want, wsteps = odec.diffuse_generate(om, p, 32, cfg.block_k, tau, 256)
    assert got == want[0]
    assert steps == wsteps
    assert want[0] != odec.diffuse_generate(plain, p, 32, cfg.block_k, tau, 256)[0][0]


def test_draft_logits_bf16_rank128():
    cfg = synth.SMALL_BF16
    ctx, om, W = make_pair(cfg)
    _, plain, _ = make_pair(cfg, weights=W)
    A, B = _adapter(cfg, 128, seed=11, std=0.02)
    _load(ctx, om, A, B, 4.0)
    p = synth.prompt_tokens(2, 70, cfg.vocab, seed=4)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, cfg.max_seq + 64)
    k = cfg.block_k
    gl = gpu_logits(ctx, 1, 2, k)
    ol = odec.draft_forward(om, st, k)
    assert (gl.double() - ol.double()).abs().max().item() < 2e-2
    assert (ol.double() - odec.draft_forward(plain, st, k).double()).abs().max().item() > 0.1
    gd = gpu_logits(ctx, 3, 2, k)               # a diffusion step's forward over a mask block
    st.block = [[cfg.mask_id] * k for _ in range(2)]
    assert (gd.double() - odec.diffusion_forward(om, st, k).double()).abs().max().item() < 2e-2


def test_rank_rules_and_switch_off_bit_exact():
    cfg = synth.SMALL_BF16
    ctx, _, _ = make_pair(cfg)
    p = synth.prompt_tokens(1, 70, cfg.vocab, seed=4)
    ctx.nld_prefill(p.cuda())
    k = cfg.block_k
    base = gpu_logits(ctx, 1, 1, k)
    A, B = _adapter(cfg, 16, seed=2, std=0.02)
    flat = [t for pair in zip(A, B) for t in pair]
    ctx.nld_init_lora(16, 4.0, flat)
    on = gpu_logits(ctx, 1, 1, k)
    assert not torch.equal(on, base)
    A2, B2 = _adapter(cfg, 8, seed=2, std=0.02)
    with pytest.raises(nb.NldError):
        ctx.nld_init_lora(8, 4.0, [t for pair in zip(A2, B2) for t in pair])
    with pytest.raises(nb.NldError):
        ctx.nld_init_lora(16, 4.0, flat[:-1])
    ctx.nld_init_lora(0, 0.0)
    assert torch.equal(gpu_logits(ctx, 1, 1, k), base)
    # the same rank loads again: back to the adapter's logits
    ctx.nld_init_lora(16, 4.0, flat)
    assert torch.equal(gpu_logits(ctx, 1, 1, k), on)


def test_draft_logits_bf16_rank128_8b_layer_shape():
    # the bench's adapter shape: K = 4096 + 128 over split 4 (17 / 17 / 17 / 15 k tiles)
    cfg = synth.LLAMA8B.replace(n_layers=2, max_seq=512)
    ctx, om, W = make_pair(cfg, device_weights=True)
    A, B = _adapter(cfg, 128, seed=5, std=0.02)
    _load(ctx, om, A, B, 1.0)
    p = synth.prompt_tokens(1, 100, cfg.vocab, seed=11)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, cfg.max_seq + 64)
    k = cfg.block_k
    gl = gpu_logits(ctx, 1, 1, k)
    ol = odec.draft_forward(om, st, k)
    assert (gl.double() - ol.double()).abs().max().item() < 2e-2
    ctx.close()
