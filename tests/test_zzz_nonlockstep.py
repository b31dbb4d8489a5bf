"""Per-sequence (non-lockstep) diffusion, nld_diffuse_step_nonlockstep: one forward of k rows
per sequence where a sequence whose block completed runs its causal KV fill while the others
keep denoising.

fp32 tiny model, batch 3 with sequences that progress at different rates: token-exact against
the oracle's per-sequence driver (itself pinned to every sequence's stand-alone generation,
tests/test_oracle_pins.py), with the same per-step state of every sequence (open, completed,
filled); a fill left due when AR decoding resumes runs first and the AR tokens match the
oracle's.  bf16 small model, batch 4: a fill moves len by k and makes b_k pending, the others
follow the commit rule on the GPU's own confidences.  This file is collected after the other
GPU tests so that a failure here does not hide theirs.
"""
import pytest
import torch

import synth
from oracle import decode as odec
from tests._helpers import gpu_state, make_pair

pytestmark = pytest.mark.gpu


def _bufs(B, k):
    return (torch.empty(B, k, dtype=torch.int32, device="cuda"),
            torch.empty(B, k, dtype=torch.float32, device="cuda"),
            torch.empty(B, dtype=torch.int32, device="cuda"),
            torch.empty(B, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("scale,tau", [(30.0, 0.7), (30.0, 0.9), (60.0, 0.5)])
def test_generation_and_states_token_exact_f32(scale, tau):
    cfg = synth.TINY_F32.replace(max_batch=3)
    B, k, n = 3, cfg.block_k, 16
    W = synth.model_weights(cfg, 0, lm_head_scale=scale)
    ctx, om, _ = make_pair(cfg, weights=W)
    p = synth.prompt_tokens(B, 40, cfg.vocab, seed=3)
    ctx.nld_prefill(p.cuda())
    want, wforwards, wstates = odec.diffuse_generate_nonlockstep(om, p, n, k, tau, 256)
    blk, conf, nc, state = _bufs(B, k)
    out = [[] for _ in range(B)]
    states = []
    while min(len(o) for o in out) < n:
        ctx.nld_diffuse_step_nonlockstep(tau, blk, conf, nc, state)
        ctx.nld_sync()          # the call does not synchronise; outputs are read next
        s = state.cpu().tolist()
        states.append(s)
        g = blk.cpu().tolist()
        for b in range(B):
            if s[b] == 1:
                assert cfg.mask_id not in g[b]
                out[b] += g[b]
            if s[b] == 2:
                assert g[b] == [cfg.mask_id] * k and int(nc[b]) == 0
    assert [o[:n] for o in out] == want
    assert states == wstates and len(states) == wforwards


def test_due_fill_runs_before_ar_f32():
    cfg = synth.TINY_F32.replace(max_batch=3)
    B, k, tau = 3, cfg.block_k, 0.7
    W = synth.model_weights(cfg, 0, lm_head_scale=30.0)
    ctx, om, _ = make_pair(cfg, weights=W)
    p = synth.prompt_tokens(B, 40, cfg.vocab, seed=3)
    ctx.nld_prefill(p.cuda())
    st = odec.prefill(om, p, 256)
    fill_next = [False] * B
    blk, conf, nc, state = _bufs(B, k)
    # step until some sequence has a completed block whose fill is due and another has not
    for _ in range(20):
        ctx.nld_diffuse_step_nonlockstep(tau, blk, conf, nc, state)
        ctx.nld_sync()          # the call does not synchronise; outputs are read next
        _, wstate, _, fill_next = odec.diffusion_step_nonlockstep(om, st, k, tau, fill_next)
        assert state.cpu().tolist() == wstate
        if any(fill_next) and not all(fill_next):
            break
    assert any(fill_next) and not all(fill_next)
    odec.flush_fills(om, st, k, fill_next)
    toks = torch.empty(B, dtype=torch.int32, device="cuda")
    ctx.nld_ar_step(toks)
    lens, pend, _, _ = gpu_state(ctx, B)
    nxt = odec.ar_step(om, st)
    assert toks.cpu().tolist() == nxt
    assert lens == st.lens and pend == st.pending


def test_bookkeeping_and_commit_rule_bf16():
    cfg = synth.SMALL_BF16
    B, k = 4, cfg.block_k
    W = synth.model_weights(cfg, 0, lm_head_scale=40.0)
    ctx, _, _ = make_pair(cfg, weights=W)
    ctx.nld_prefill(synth.prompt_tokens(B, 70, cfg.vocab, seed=8).cuda())
    blk, conf, nc, state = _bufs(B, k)
    prev_blk = [[cfg.mask_id] * k for _ in range(B)]
    lens0, _, _, _ = gpu_state(ctx, B)
    seen = set()
    # threshold 0 commits every open slot: blocks complete at steps 2 and 5, fill at 3 and 6
    for tau in [0.9, 0.9, 0.0, 0.9, 0.9, 0.0, 0.9]:
        ctx.nld_diffuse_step_nonlockstep(tau, blk, conf, nc, state)
        ctx.nld_sync()          # the call does not synchronise; outputs are read next
        s = state.cpu().tolist()
        lens, pend, _, _ = gpu_state(ctx, B)
        g_blk, g_conf = blk.cpu().tolist(), conf.cpu()
        for b in range(B):
            seen.add(s[b])
            if s[b] == 2:
                assert lens[b] == lens0[b] + k and pend[b] == prev_blk[b][k - 1]
                assert g_blk[b] == [cfg.mask_id] * k
            else:
                assert lens[b] == lens0[b]
                masked = [t == cfg.mask_id for t in prev_blk[b]]
                pick = odec.diffusion_commit(masked, g_conf[b].tolist(), tau)
                assert int(nc[b]) == sum(pick) >= 1
                for slot in range(k):
                    if pick[slot]:
                        assert g_blk[b][slot] != cfg.mask_id
                    else:
                        assert g_blk[b][slot] == prev_blk[b][slot]
                assert (s[b] == 1) == (cfg.mask_id not in g_blk[b])
        prev_blk, lens0 = g_blk, lens
    assert {0, 1, 2} <= seen
