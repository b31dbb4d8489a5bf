"""Prefill of a batch of prompts of different lengths (nld_prefill with per-sequence lengths).

Sequences never see one another, so each sequence of a ragged batch must decode exactly as it
would alone: the oracle prefills every prompt on its own and the caches are merged into one
batch state.  fp32 tiny model: self-speculation rounds token-exact against the fp64 oracle
(ranhao.site notes section 5.3, r9-hu digest "Method": lossless rounds of 1..k+1 tokens).
bf16 small shape: per-round commits bit-exact given the GPU's own draft and verify argmaxes, and
the argmaxes equal to the oracle's where its top-2 margin exceeds 5e-2.
"""
import pytest
import torch

import synth
from oracle import decode as odec
from tests._helpers import gpu_state, make_pair, top2_margin

pytestmark = pytest.mark.gpu

LENS = [37, 200, 64]


def _ragged(cfg, seed):
    B, S = len(LENS), max(LENS)
    p = synth.prompt_tokens(B, S, cfg.vocab, seed=seed)
    for b, n in enumerate(LENS):
        p[b, n:] = -5            # padding the library must ignore
    return p


def _oracle_state(om, p, capacity):
    parts = [odec.prefill(om, p[b:b + 1, :n], capacity) for b, n in enumerate(LENS)]
    return odec.SeqState(cache=[c for s in parts for c in s.cache],
                         lens=[s.lens[0] for s in parts], pending=[s.pending[0] for s in parts])


def test_ragged_prefill_selfspec_token_exact_f32():
    cfg = synth.TINY_F32.replace(max_batch=3, max_seq=320)
    ctx, om, _ = make_pair(cfg)
    p = _ragged(cfg, seed=21)
    lens = torch.tensor(LENS, dtype=torch.int32, device="cuda")
    pend = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    ctx.nld_prefill(p.cuda(), lens, pend)
    st = _oracle_state(om, p, 400)
    g_lens, g_pend, _, _ = gpu_state(ctx, 3)
    assert g_lens == [n - 1 for n in LENS] == st.lens
    assert g_pend == pend.cpu().tolist() == st.pending
    k = cfg.block_k
    toks = torch.empty(3, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(3, dtype=torch.int32, device="cuda")
    for _ in range(6):
        ctx.nld_selfspec_round(toks, nc, None)
        ctx.nld_sync()
        committed, *_ = odec.selfspec_round(om, st, k)
        for b in range(3):
            c = int(nc[b])
            assert toks[b, :c].cpu().tolist() == committed[b]
        g_lens, g_pend, _, _ = gpu_state(ctx, 3)
        assert g_lens == st.lens and g_pend == st.pending


def test_ragged_prefill_bf16_commits_given_argmaxes():
    cfg = synth.SMALL_BF16.replace(max_batch=3)
    ctx, om, _ = make_pair(cfg)
    p = _ragged(cfg, seed=22)
    ctx.nld_prefill(p.cuda(), torch.tensor(LENS, dtype=torch.int32, device="cuda"))
    st = _oracle_state(om, p, cfg.max_seq + 64)
    k = cfg.block_k
    toks = torch.empty(3, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(3, dtype=torch.int32, device="cuda")
    for _ in range(3):
        ctx.nld_selfspec_round(toks, nc, None)
        ctx.nld_sync()
        g_lens, g_pend, draft, ver = gpu_state(ctx, 3)
        ol = odec.draft_forward(om, st, k)
        sure = top2_margin(ol) > 5e-2
        assert torch.equal(torch.tensor(draft)[sure], odec.argmax_lowest(ol)[sure])
        ov = odec.verify_forward(om, st, draft)
        vs = top2_margin(ov) > 5e-2
        assert torch.equal(torch.tensor(ver)[vs], odec.argmax_lowest(ov)[vs])
        committed = [odec.commit_after_verify(draft[b], ver[b]) for b in range(3)]
        for b in range(3):
            assert int(nc[b]) == len(committed[b])
            assert toks[b, :len(committed[b])].cpu().tolist() == committed[b]
        odec.apply_commit(st, committed)
        assert g_lens == st.lens and g_pend == st.pending


def test_prompt_length_out_of_range_flags_device_error():
    import self_speculation_b200 as nb
    cfg = synth.TINY_F32.replace(max_batch=2)
    ctx, _, _ = make_pair(cfg)
    p = synth.prompt_tokens(2, 16, cfg.vocab, seed=3)
    ctx.nld_prefill(p.cuda(), torch.tensor([16, 17], dtype=torch.int32, device="cuda"))
    with pytest.raises(nb.NldError) as ei:
        ctx.nld_sync()
    assert ei.value.status == 7
    lens, _, _, _ = gpu_state(ctx, 2)
    assert lens == [15, 15]
