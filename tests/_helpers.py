"""Shared helpers of the GPU tests: build a library context and an oracle from the same seeded
synthetic inputs (module `synth`)."""
from __future__ import annotations

import torch

import oracle
import synth
from oracle import decode as odec


def make_pair(cfg, seed=0, precision=None, weights=None, device_weights=False):
    """(library Context, OracleModel, weights) on identical weights."""
    import self_speculation_b200 as nb
    W = weights if weights is not None else synth.model_weights(cfg, seed)
    ctx = nb.Context(cfg)
    if device_weights:
        ctx.nld_init_weights([w.cuda() for w in W], on_device=True)
    else:
        ctx.nld_init_weights(W, on_device=False)
    if precision is None:
        precision = "f64" if cfg.dtype == synth.F32 else "f32kv"
    om = oracle.OracleModel(cfg, W, precision)
    return ctx, om, W


def gpu_state(ctx, B):
    k = ctx.cfg.block_k
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    pend = torch.zeros(B, dtype=torch.int32, device="cuda")
    draft = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    ver = torch.zeros(B, k + 1, dtype=torch.int32, device="cuda")
    ctx.nld_debug_state(lens, pend, draft, ver)
    ctx.nld_sync()
    return lens.cpu().tolist(), pend.cpu().tolist(), draft.cpu().tolist(), ver.cpu().tolist()


def gpu_logits(ctx, mode, B, m):
    out = torch.empty(B, m, ctx.cfg.vocab, dtype=torch.float32, device="cuda")
    ctx.nld_debug_logits(mode, out)
    ctx.nld_sync()
    return out.cpu()


def top2_margin(logits):
    t = torch.topk(logits.double(), 2, dim=-1).values
    return t[..., 0] - t[..., 1]


def oracle_state_from(om, prompt, capacity):
    return odec.prefill(om, prompt, capacity)
