"""Pins of the CPU oracle against facts the pages and mathematics fix (no GPU).

Each test checks the oracle against something other than itself: hand-written fixtures,
closed forms, textbook special cases, brute force on tiny inputs and invariants stated by
the pages (Nemotron-Labs-Diffusion: ranhao.site notes sections 3.2, 4.3, 5.1-5.3; r9-hu
digest "Method"; shilu.ai "Deploy and infer with SGLang").
"""
import itertools
import math
import os

import pytest
import torch

import oracle
import synth
from oracle import decode as odec
from oracle import model as omod

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _tiny(**kw):
    return synth.TINY_F32.replace(**kw)


# ---------------------------------------------------------------- hand-written fixtures --

def _read_cases(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append([part.split() for part in line.split("|")])
    return rows


def test_accept_golden_cases():
    for d, v, c in _read_cases("accept_cases.txt"):
        d, v, c = [int(x) for x in d], [int(x) for x in v], [int(x) for x in c]
        assert odec.commit_after_verify(d, v) == c
        assert odec.accept_length(d, v) + 1 == len(c)


def test_diffusion_golden_cases():
    for mk, cf, tau, want in _read_cases("diffusion_cases.txt"):
        got = odec.diffusion_commit([x == "1" for x in mk], [float(x) for x in cf], float(tau[0]))
        assert got == [x == "1" for x in want]


def test_mask_golden():
    lines = [l.split() for l in open(os.path.join(GOLD, "mask_n2_m4.txt"))
             if l.strip() and not l.startswith("#")]
    i = 0
    while i < len(lines):
        assert lines[i][0] == "block_size"
        bs = int(lines[i][1])
        want = torch.tensor([[int(x) for x in lines[i + r]] for r in range(1, 5)], dtype=torch.bool)
        assert torch.equal(omod.block_mask(4, 2, bs), want)
        i += 5


# ------------------------------------------------------------------------ acceptance --

@pytest.mark.parametrize("k", [1, 2, 5, 12])
def test_accept_exhaustive_patterns(k):
    """All 2^k match patterns: committed length == 1 + index of first mismatch (or k+1),
    always within [1, k+1]."""
    for pat in itertools.product([True, False], repeat=k):
        draft = list(range(100, 100 + k))
        verify = [d if ok else d + 7 for d, ok in zip(draft, pat)] + [999]
        first_bad = next((i for i, ok in enumerate(pat) if not ok), k)
        got = odec.commit_after_verify(draft, verify)
        assert len(got) == first_bad + 1
        assert 1 <= len(got) <= k + 1
        assert got == verify[:first_bad + 1]


def test_accept_random_k32():
    g = torch.Generator().manual_seed(5)
    for _ in range(2000):
        pat = (torch.rand(32, generator=g) < 0.9).tolist()
        draft = list(range(32))
        verify = [d if ok else -1 for d, ok in zip(draft, pat)] + [77]
        first_bad = pat.index(False) if False in pat else 32
        assert len(odec.commit_after_verify(draft, verify)) == first_bad + 1


def test_forced_commit():
    d = [1, 2, 3]
    v = [1, 9, 9, 9]
    assert odec.commit_after_verify(d, v, forced=1) == [1]
    assert odec.commit_after_verify(d, v, forced=3) == [1, 2, 9]
    assert odec.commit_after_verify(d, v, forced=4) == [1, 2, 3, 9]


# ------------------------------------------------------------------------------ masks --

@pytest.mark.parametrize("n,m", [(0, 1), (0, 7), (5, 1), (5, 8), (33, 32)])
def test_block_size_one_is_causal(n, m):
    assert torch.equal(omod.block_mask(m, n, 1), omod.causal_mask(m, n))


def test_single_block_sees_whole_block_and_prefix():
    msk = omod.block_mask(8, 3, 8)
    assert bool(msk.all())


def _attention_bruteforce(q, k, v, mask):
    """Per query, per head: gather the visible keys and do the two-pass softmax by hand."""
    Hq, m, hd = q.shape
    Hkv = k.shape[0]
    out = torch.zeros_like(q)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for r in range(m):
            vis = [j for j in range(k.shape[1]) if bool(mask[r, j])]
            s = [float((q[h, r] * k[g, j]).sum()) / math.sqrt(hd) for j in vis]
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            z = sum(w)
            acc = torch.zeros(hd, dtype=q.dtype)
            for wj, j in zip(w, vis):
                acc += (wj / z) * v[g, j]
            out[h, r] = acc
    return out


@pytest.mark.parametrize("bs", [1, 2, 4])
def test_attention_matches_bruteforce(bs):
    g = torch.Generator().manual_seed(3)
    Hq, Hkv, hd, n, m = 4, 2, 8, 3, 4
    q = torch.randn(Hq, m, hd, generator=g, dtype=torch.float64)
    k = torch.randn(Hkv, n + m, hd, generator=g, dtype=torch.float64)
    v = torch.randn(Hkv, n + m, hd, generator=g, dtype=torch.float64)
    mask = omod.block_mask(m, n, bs)
    got = omod.attention_explicit(q, k, v, mask)
    want = _attention_bruteforce(q, k, v, mask)
    assert torch.allclose(got, want, atol=1e-12, rtol=0)


def test_gqa_equals_mha_with_repeated_kv():
    g = torch.Generator().manual_seed(4)
    Hq, Hkv, hd, L, m = 8, 2, 16, 10, 3
    q = torch.randn(Hq, m, hd, generator=g, dtype=torch.float64)
    k = torch.randn(Hkv, L, hd, generator=g, dtype=torch.float64)
    v = torch.randn(Hkv, L, hd, generator=g, dtype=torch.float64)
    mask = omod.causal_mask(m, L - m)
    a = omod.attention_explicit(q, k, v, mask)
    b = omod.attention_explicit(q, k.repeat_interleave(Hq // Hkv, 0),
                                v.repeat_interleave(Hq // Hkv, 0), mask)
    assert torch.allclose(a, b, atol=1e-14, rtol=0)
    # a wrong grouping (kv head = j % Hkv) must differ
    c = omod.attention_explicit(q, k.repeat(Hq // Hkv, 1, 1), v.repeat(Hq // Hkv, 1, 1), mask)
    assert not torch.allclose(a, c)


# ------------------------------------------------------------------------ norm / rope --

def test_rmsnorm_closed_form():
    for c in [0.5, -3.0, 1e-2]:
        x = torch.full((1, 64), c, dtype=torch.float64)
        eps = 1e-6
        want = math.copysign(1.0, c) / math.sqrt(1.0 + eps / (c * c))
        assert torch.allclose(omod.rmsnorm(x, eps), torch.full_like(x, want), atol=1e-14)


def test_rope_position_zero_is_identity():
    x = torch.randn(5, 64, dtype=torch.float64)
    assert torch.allclose(omod.rope_rotate(x, torch.zeros(5), 10000.0), x, atol=0)


def test_rope_matches_complex_rotation():
    """Rotate-half RoPE == multiplying z_i = x_i + i*x_{i+hd/2} by exp(i*pos*theta^(-2i/hd))."""
    g = torch.Generator().manual_seed(6)
    hd, theta = 64, 10000.0
    x = torch.randn(7, hd, generator=g, dtype=torch.float64)
    pos = torch.tensor([0, 1, 2, 17, 100, 511, 4000], dtype=torch.float64)
    got = omod.rope_rotate(x, pos, theta)
    for r in range(7):
        for i in range(hd // 2):
            ang = float(pos[r]) * theta ** (-2.0 * i / hd)
            z = complex(float(x[r, i]), float(x[r, i + hd // 2])) * complex(math.cos(ang), math.sin(ang))
            assert abs(float(got[r, i]) - z.real) < 1e-12
            assert abs(float(got[r, i + hd // 2]) - z.imag) < 1e-12


def test_rope_relative_position_invariance():
    g = torch.Generator().manual_seed(7)
    q = torch.randn(64, generator=g, dtype=torch.float64)
    k = torch.randn(64, generator=g, dtype=torch.float64)
    def dot(pq, pk):
        return float((omod.rope_rotate(q[None], torch.tensor([pq]), 1e4)
                      * omod.rope_rotate(k[None], torch.tensor([pk]), 1e4)).sum())
    assert abs(dot(10, 3) - dot(107, 100)) < 1e-10
    assert abs(dot(10, 3) - dot(10, 4)) > 1e-6


# ------------------------------------------------------------------------ model forward --

def test_forward_closed_form_without_residual_updates():
    """With Wo = 0 and Wd = 0 the layers leave h = E[t], so logits = rmsnorm(E[t]) Wlm^T."""
    cfg = _tiny(n_layers=1)
    W = synth.model_weights(cfg, 0)
    W[5] = torch.zeros_like(W[5])    # wo
    W[9] = torch.zeros_like(W[9])    # wd
    mdl = oracle.OracleModel(cfg, W, "f64")
    toks = torch.tensor([[3, 9, 4000, cfg.mask_id]])
    cache = mdl.new_cache(1, 16)
    logits = mdl.forward(toks, [0], cache, block_size=4, write_kv=False)
    E = W[0].double()
    h = E[toks[0].long()]
    want = (h / torch.sqrt((h * h).mean(-1, keepdim=True) + cfg.rms_eps)) @ W[-1].double().t()
    assert torch.allclose(logits[0], want, atol=1e-12)


def test_single_key_attention_returns_value():
    """A one-token forward with an empty cache attends to its own key only: the attention
    output is exactly v, so h1 = h0 + v Wo^T (checked by hand on layer 0)."""
    cfg = _tiny(n_layers=1)
    W = synth.model_weights(cfg, 1)
    W[9] = torch.zeros_like(W[9])    # wd = 0: only the attention branch updates h
    mdl = oracle.OracleModel(cfg, W, "f64")
    t = torch.tensor([[11]])
    logits = mdl.forward(t, [0], mdl.new_cache(1, 4), block_size=1, write_kv=False)
    h0 = W[0].double()[11]
    a = h0 / torch.sqrt((h0 * h0).mean() + cfg.rms_eps)
    v = a @ W[4].double().t()
    h1 = h0 + v @ W[5].double().t()
    want = (h1 / torch.sqrt((h1 * h1).mean() + cfg.rms_eps)) @ W[-1].double().t()
    assert torch.allclose(logits[0, 0], want, atol=1e-12)


def test_causal_forward_ignores_future_tokens():
    cfg = _tiny()
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    a = torch.tensor([[1, 2, 3, 4, 5, 6]])
    b = torch.tensor([[1, 2, 3, 99, 98, 97]])
    la = mdl.forward(a, [0], mdl.new_cache(1, 8), 1, False)
    lb = mdl.forward(b, [0], mdl.new_cache(1, 8), 1, False)
    assert torch.allclose(la[0, :3], lb[0, :3], atol=0)
    assert not torch.allclose(la[0, 3], lb[0, 3])


def test_block_forward_is_bidirectional_inside_block():
    cfg = _tiny()
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    a = torch.tensor([[1, 2, 3, 4]])
    b = torch.tensor([[1, 2, 3, 99]])
    la = mdl.forward(a, [0], mdl.new_cache(1, 8), 4, False)
    lb = mdl.forward(b, [0], mdl.new_cache(1, 8), 4, False)
    assert not torch.allclose(la[0, 0], lb[0, 0])


def test_kv_cache_reuse_equals_full_causal_forward():
    """Prefill rows 0..n-1 then a causal forward over n..n+m-1 == one causal forward."""
    cfg = _tiny()
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    toks = synth.prompt_tokens(1, 12, cfg.vocab, seed=3).long()
    full = mdl.forward(toks, [0], mdl.new_cache(1, 16), 1, False)
    cache = mdl.new_cache(1, 16)
    mdl.forward(toks[:, :7], [0], cache, 1, True, with_logits=False)
    part = mdl.forward(toks[:, 7:], [7], cache, 1, True)
    assert torch.allclose(full[0, 7:], part[0], atol=1e-12)


def test_draft_with_block_one_is_ar_step():
    cfg = _tiny()
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    p = synth.prompt_tokens(1, 20, cfg.vocab, seed=4)
    st1 = odec.prefill(mdl, p, 64)
    st2 = odec.prefill(mdl, p, 64)
    d = odec.draft_forward(mdl, st1, 1)
    a = odec.ar_forward(mdl, st2)
    assert torch.allclose(d, a, atol=0)


# ------------------------------------------------------------- self-speculation semantics --

@pytest.mark.parametrize("seed,k", [(0, 8), (1, 8), (2, 3), (3, 1)])
def test_selfspec_is_lossless_against_ar(seed, k):
    """At temperature 0 self-speculation reproduces AR greedy decoding token for token
    (shilu.ai, LinearSpec).  Holds for any weights, so it pins the round logic."""
    cfg = _tiny(n_layers=1, max_seq=200)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, seed), "f64")
    p = synth.prompt_tokens(1, 24, cfg.vocab, seed=seed + 10)
    ar = odec.ar_generate(mdl, p, 24, 128)
    ss, per_round = odec.selfspec_generate(mdl, p, 24, k, 128)
    assert ss == ar
    assert all(1 <= c <= k + 1 for c in per_round[0])


def test_selfspec_lossless_with_peaky_logits_multi_accept():
    """A scaled LM head makes drafts agree with the verifier often, exercising a > 0."""
    cfg = _tiny(n_layers=1, max_seq=200)
    W = synth.model_weights(cfg, 5)
    # a structured model: the LM head reads the embedding of the input token strongly, so
    # the argmax chain becomes predictable and drafts match.
    W[-1] = W[0][:cfg.vocab].clone() * 50.0
    mdl = oracle.OracleModel(cfg, W, "f64")
    p = synth.prompt_tokens(1, 16, cfg.vocab, seed=9)
    ar = odec.ar_generate(mdl, p, 40, 128)
    ss, per_round = odec.selfspec_generate(mdl, p, 40, 8, 128)
    assert ss == ar
    assert max(per_round[0]) > 1


def test_selfspec_kv_equals_ar_kv():
    cfg = _tiny(n_layers=2, max_seq=200)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 2), "f64")
    p = synth.prompt_tokens(1, 16, cfg.vocab, seed=2)
    st_a = odec.prefill(mdl, p, 128)
    for _ in range(12):
        odec.ar_step(mdl, st_a)
    st_s = odec.prefill(mdl, p, 128)
    while st_s.lens[0] < st_a.lens[0]:
        odec.selfspec_round(mdl, st_s, 4)
    n = st_a.lens[0]
    for l in range(cfg.n_layers):
        assert torch.allclose(st_a.cache[0][l][0][:, :n], st_s.cache[0][l][0][:, :n], atol=1e-12)
        assert torch.allclose(st_a.cache[0][l][1][:, :n], st_s.cache[0][l][1][:, :n], atol=1e-12)


def test_selfspec_batched_matches_single():
    cfg = _tiny(n_layers=1, max_seq=200)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    p = synth.prompt_tokens(2, 12, cfg.vocab, seed=8)
    both, _ = odec.selfspec_generate(mdl, p, 10, 4, 64)
    one, _ = odec.selfspec_generate(mdl, p[1:], 10, 4, 64)
    assert both[1] == one[0]


# ------------------------------------------------------------------------ diffusion --

def test_diffusion_threshold_above_one_commits_one_per_step():
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    p = synth.prompt_tokens(1, 10, cfg.vocab)
    st = odec.prefill(mdl, p, 64)
    k = 4
    for step in range(k):
        r = odec.diffusion_step(mdl, st, k, tau=1.5)
        assert len(r["newly"][0]) == 1
        assert r["filled"] == (step == k - 1)


def test_diffusion_threshold_zero_commits_whole_block():
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    st = odec.prefill(mdl, synth.prompt_tokens(1, 10, cfg.vocab), 64)
    r = odec.diffusion_step(mdl, st, 4, tau=0.0)
    assert len(r["newly"][0]) == 4 and r["filled"]
    assert st.lens[0] == 9 + 4


def test_diffusion_block_one_equals_ar():
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    p = synth.prompt_tokens(1, 10, cfg.vocab)
    ar = odec.ar_generate(mdl, p, 6, 64)
    df, steps = odec.diffuse_generate(mdl, p, 6, 1, 0.9, 64)
    assert df == ar and steps == 6


def test_diffusion_peaky_logits_multi_commit():
    cfg = _tiny(n_layers=1)
    W = synth.model_weights(cfg, 0, lm_head_scale=60.0)
    mdl = oracle.OracleModel(cfg, W, "f64")
    st = odec.prefill(mdl, synth.prompt_tokens(1, 10, cfg.vocab), 64)
    r = odec.diffusion_step(mdl, st, 8, tau=0.9)
    assert len(r["newly"][0]) >= 2


def test_confidence_and_argmax_closed_forms():
    l = torch.tensor([[0.0, math.log(3.0), math.log(3.0), 0.0]], dtype=torch.float64)
    assert int(odec.argmax_lowest(l)[0]) == 1
    assert abs(float(odec.confidence(l)[0]) - 3.0 / 8.0) < 1e-15


def test_f32kv_mode_is_fp32_over_a_bf16_cache():
    """"f32kv" is the fp32 forward whose KV cache holds bf16 numbers: the rows it caches are
    bf16 values within one bf16 spacing of the exact (f64) rows, and its logits differ from the
    exact forward by the effect of that rounding (nonzero, well under the 2e-2 bar), while the
    plain fp32 forward differs only by fp32 rounding."""
    cfg = synth.SMALL_BF16.replace(n_layers=1)
    W = synth.model_weights(cfg, 0)
    toks = synth.prompt_tokens(1, 9, cfg.vocab, seed=3).long()
    models = {p: oracle.OracleModel(cfg, W, p) for p in ("f64", "f32", "f32kv")}
    caches = {p: m.new_cache(1, 16) for p, m in models.items()}
    logits = {p: m.forward(toks, [0], caches[p], 1, True).double() for p, m in models.items()}
    for kv in (0, 1):
        exact = caches["f64"][0][0][kv][:, :9]
        held = caches["f32kv"][0][0][kv][:, :9]
        assert held.dtype == torch.bfloat16
        # bf16 has 8 significand bits: neighbouring values are at most 2^-7 |x| apart
        assert ((held.double() - exact).abs() <= 2.0 ** -7 * exact.abs() + 1e-30).all()
        assert not torch.equal(held.double(), exact)
    e32 = (logits["f32"] - logits["f64"]).abs().max().item()
    ekv = (logits["f32kv"] - logits["f64"]).abs().max().item()
    assert e32 < 1e-4
    assert 1e-4 < ekv < 1e-2


def test_mlp_branch_closed_form():
    """With Wo = 0 only the SwiGLU branch updates h: h1 = h0 + (silu(a Wg^T) * a Wu^T) Wd^T,
    a = rmsnorm(h0); silu taken from torch.nn.functional (independent of the oracle)."""
    cfg = _tiny(n_layers=1)
    W = synth.model_weights(cfg, 3)
    W[5] = torch.zeros_like(W[5])    # wo
    mdl = oracle.OracleModel(cfg, W, "f64")
    t = torch.tensor([[7, 8]])
    logits = mdl.forward(t, [0], mdl.new_cache(1, 4), block_size=1, write_kv=False)
    h0 = W[0].double()[t[0].long()]
    a = h0 / torch.sqrt((h0 * h0).mean(-1, keepdim=True) + cfg.rms_eps)
    u = torch.nn.functional.silu(a @ W[7].double().t()) * (a @ W[8].double().t())
    h1 = h0 + u @ W[9].double().t()
    want = (h1 / torch.sqrt((h1 * h1).mean(-1, keepdim=True) + cfg.rms_eps)) @ W[-1].double().t()
    assert torch.allclose(logits[0], want, atol=1e-12)


# ---------------------------------------------- fused KV fill (deferred fill, next row f1) --

def test_fused_fill_mask_reduces_to_causal_and_block_masks():
    n, c, bs = 5, 4, 4
    m = c + bs
    full = omod.block_mask(m, n, bs, causal_rows=c)
    # the first c rows are the causal mask's rows
    assert torch.equal(full[:c, :n + c], omod.causal_mask(c, n))
    assert not full[:c, n + c:].any()
    # the block rows see the prefix, every fill row and their whole block
    assert full[c:].all()
    # no causal rows: unchanged
    assert torch.equal(omod.block_mask(m, n, bs, 0), omod.block_mask(m, n, bs))


def _state_with_complete_block(mdl, k, seed):
    st = odec.prefill(mdl, synth.prompt_tokens(2, 11, mdl.cfg.vocab, seed=seed), 96)
    st.block = [[mdl.cfg.mask_id] * k for _ in range(2)]
    st.block = [list(odec.argmax_lowest(odec.diffusion_forward(mdl, st, k))[b].tolist())
                for b in range(2)]
    return st


@pytest.mark.parametrize("with_lora", [False, True])
def test_fused_fill_equals_fill_then_denoise(with_lora):
    """The fused forward's KV rows and last k logit rows equal the causal fill forward
    followed by the plain denoising forward of the next block (fp64, exact up to rounding).
    With a LoRA drafter the fill rows stay on the frozen path and the block rows take it."""
    import copy
    cfg = _tiny(n_layers=2)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    if with_lora:
        A, B = _lora(cfg, 8, seed=3)
        mdl.set_lora(A, B, 5.0)
    k = 4
    st = _state_with_complete_block(mdl, k, seed=3)
    a, b = copy.deepcopy(st), copy.deepcopy(st)
    # separate: fill (causal, writes KV) then the new block's first denoising forward
    toks = torch.tensor([[a.pending[i]] + a.block[i][:k - 1] for i in range(2)], dtype=torch.int64)
    mdl.forward(toks, a.lens, a.cache, block_size=1, write_kv=True, with_logits=False)
    for i in range(2):
        a.lens[i] += k
        a.pending[i] = a.block[i][k - 1]
    a.block = [[cfg.mask_id] * k for _ in range(2)]
    la = odec.diffusion_forward(mdl, a, k)
    # fused
    lb = odec.fill_diffusion_forward(mdl, b, k)
    assert (la - lb).abs().max().item() < 1e-10
    assert a.lens == b.lens and a.pending == b.pending and a.block == b.block
    for i in range(2):
        for layer in range(cfg.n_layers):
            for t in range(2):
                x, y = a.cache[i][layer][t][:, :a.lens[i]], b.cache[i][layer][t][:, :b.lens[i]]
                assert (x - y).abs().max().item() < 1e-12


@pytest.mark.parametrize("tau", [0.9, 0.0, 1.5])
def test_fused_fill_generation_equals_unfused(tau):
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0, lm_head_scale=30.0), "f64")
    p = synth.prompt_tokens(2, 10, cfg.vocab, seed=5)
    k = 4
    ref, steps = odec.diffuse_generate(mdl, p, 12, k, tau, 96)
    got, forwards, fsteps = odec.diffuse_generate_fused(mdl, p, 12, k, tau, 96)
    assert got == ref
    assert fsteps == steps and forwards == steps   # no separate fill forwards


# ------------------------------------------------------------ LoRA drafter (next row f3) --

def _lora(cfg, r, seed, std=0.02):
    g = torch.Generator().manual_seed(seed)
    qd = cfg.n_q_heads * cfg.head_dim
    A = [torch.randn(r, qd, generator=g, dtype=torch.float64) * std for _ in range(cfg.n_layers)]
    B = [torch.randn(cfg.d_model, r, generator=g, dtype=torch.float64) * std for _ in range(cfg.n_layers)]
    return A, B


def test_lora_equals_merged_o_proj_in_draft():
    """The LoRA forward equals the plain forward with W_o + scale * B A (the merge identity of a
    low-rank adapter), in fp64."""
    cfg = _tiny(n_layers=2)
    W = synth.model_weights(cfg, 0)
    A, B = _lora(cfg, 8, seed=3)
    sc = 5.0
    lo = oracle.OracleModel(cfg, W, "f64")
    lo.set_lora(A, B, sc)
    Wm = list(W)
    for l in range(cfg.n_layers):
        Wm[1 + 9 * l + 4] = W[1 + 9 * l + 4].double() + sc * (B[l] @ A[l])
    merged = oracle.OracleModel(cfg, Wm, "f64")
    plain = oracle.OracleModel(cfg, W, "f64")
    p = synth.prompt_tokens(2, 20, cfg.vocab, seed=4)
    # the clean prefix is written by the frozen (plain) weights; only the draft differs
    st = odec.prefill(plain, p, 96)
    a, b = odec.draft_forward(lo, st, 8), odec.draft_forward(merged, st, 8)
    assert (a - b).abs().max().item() < 1e-10
    # and the delta is not negligible at this scale
    assert (a - odec.draft_forward(plain, st, 8)).abs().max().item() > 1e-3


def test_lora_only_in_drafter_forwards():
    cfg = _tiny(n_layers=2)
    W = synth.model_weights(cfg, 0)
    A, B = _lora(cfg, 8, seed=3)
    lo, pl = oracle.OracleModel(cfg, W, "f64"), oracle.OracleModel(cfg, W, "f64")
    lo.set_lora(A, B, 5.0)
    p = synth.prompt_tokens(1, 20, cfg.vocab, seed=4)
    s1, s2 = odec.prefill(lo, p, 96), odec.prefill(pl, p, 96)
    drafts = [[3, 7, 11, 2, 5, 9, 1, 4]]
    assert torch.equal(odec.verify_forward(lo, s1, drafts), odec.verify_forward(pl, s2, drafts))
    assert torch.equal(odec.ar_forward(lo, s1), odec.ar_forward(pl, s2))
    zero = [torch.zeros_like(b) for b in B]
    lo.set_lora(A, zero, 5.0)
    assert torch.equal(odec.draft_forward(lo, s1, 8), odec.draft_forward(pl, s2, 8))


# ---------------------------------------------- per-sequence diffusion (next row f4) --

def _varied_prompts(cfg, B, P, seed):
    return synth.prompt_tokens(B, P, cfg.vocab, seed=seed)


@pytest.mark.parametrize("tau", [0.9, 0.6, 0.3])
def test_nonlockstep_tokens_equal_each_sequence_alone(tau):
    """Sequences are independent: per-sequence diffusion of a batch gives every sequence the
    tokens the lockstep driver gives it alone (fp64)."""
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0, lm_head_scale=30.0), "f64")
    p = _varied_prompts(cfg, 3, 10, seed=6)
    k = 4
    got, forwards, states = odec.diffuse_generate_nonlockstep(mdl, p, 12, k, tau, 96)
    for b in range(3):
        alone, _ = odec.diffuse_generate(mdl, p[b:b + 1], 12, k, tau, 96)
        assert got[b] == alone[0]
    # every step is one forward; a fill always follows the step that completed the block
    assert forwards == len(states)
    for b in range(3):
        seq = [st[b] for st in states]
        for i, v in enumerate(seq[:-1]):
            assert (seq[i + 1] == 2) == (v == 1)


def test_nonlockstep_saves_forwards_when_progress_differs():
    """With sequences that finish their blocks at different steps, lockstep runs every block
    as long as the slowest sequence; per-sequence scheduling does not wait (forwards counted
    for the same number of generated tokens)."""
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0, lm_head_scale=30.0), "f64")
    p = _varied_prompts(cfg, 3, 10, seed=6)
    k, tau, n = 4, 0.6, 12
    _, nl_forwards, states = odec.diffuse_generate_nonlockstep(mdl, p, n, k, tau, 96)
    # lockstep: each step is one forward, plus one fill forward per completed set of blocks
    _, ls_steps = odec.diffuse_generate(mdl, p, n, k, tau, 96)
    ls_forwards = ls_steps + n // k
    # per sequence, the steps it needs alone (denoising + one fill per block)
    alone = []
    for b in range(3):
        _, s1 = odec.diffuse_generate(mdl, p[b:b + 1], n, k, tau, 96)
        alone.append(s1 + n // k)
    assert len(set(alone)) > 1                        # the sequences progress differently
    assert nl_forwards < ls_forwards
    # the batch runs until its slowest sequence is done, give or take its last fill
    assert max(alone) - 1 <= nl_forwards <= max(alone) + 1


# ------------------------------------------ quadratic self-speculation (next row f2) --

def test_quadratic_layout_small_case_by_hand():
    """n = 2 cached rows, k = 1: rows V0 (x_n at 2), V1 (d_1 at 3), P0 (mask at 3), P1 (mask
    at 4); keys are the 2 cached rows then the 4 rows of the forward."""
    m, pos, mask = odec.quadratic_layout(2, 1)
    assert m == 4 and pos.tolist() == [2, 3, 3, 4]
    T, F = True, False
    want = [[T, T, T, F, F, F],     # V0: prefix, itself
             [T, T, T, T, F, F],    # V1: prefix, V0, itself
             [T, T, T, F, T, F],    # P0: prefix, V0 (outcome a = 0 keeps x_n), itself
             [T, T, T, T, F, T]]    # P1: prefix, V0, V1, itself
    assert mask.tolist() == want


@pytest.mark.parametrize("k", [2, 4])
def test_quadratic_layout_invariants(k):
    n = 5
    m, pos, mask = odec.quadratic_layout(n, k)
    assert m == (k + 1) ** 2                    # quadratic in k
    assert mask[:, :n].all()
    assert torch.equal(mask[:k + 1, :n + k + 1], omod.causal_mask(k + 1, n))
    assert not mask[:k + 1, n + k + 1:].any()   # verify rows never see a pre-draft row
    for a in range(k + 1):
        r0 = k + 1 + a * k
        rows = mask[r0:r0 + k]
        assert rows[:, n:n + a + 1].all() and not rows[:, n + a + 1:n + k + 1].any()
        assert rows[:, n + r0:n + r0 + k].all()
        assert rows[:, n + k + 1:].sum().item() == k * k     # no other block's rows
        assert pos[r0:r0 + k].tolist() == list(range(n + a + 1, n + a + 1 + k))


def test_quadratic_forward_equals_verify_and_separate_predrafts():
    """The verify rows equal the linear verify forward (logits and KV rows), and pre-draft
    block a equals a block forward of k masks at n+a+1 over the prefix extended by the causal
    rows of x_n, d_1..d_a: the two constructions agree in fp64."""
    import copy
    cfg = _tiny(n_layers=2)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    A, B = _lora(cfg, 8, seed=3)
    mdl.set_lora(A, B, 5.0)                     # the pre-draft rows are drafter rows
    k = 3
    st = odec.prefill(mdl, synth.prompt_tokens(2, 9, cfg.vocab, seed=2), 96)
    drafts = [[5, 17, 3], [8, 8, 2]]
    s_lin, s_quad = copy.deepcopy(st), copy.deepcopy(st)
    vl = odec.verify_forward(mdl, s_lin, drafts)
    ql, pl = odec.quadratic_forward(mdl, s_quad, drafts)
    assert (ql - vl).abs().max().item() < 1e-10
    for b in range(2):
        n = st.lens[b]
        for layer in range(cfg.n_layers):
            for t in range(2):
                x = s_lin.cache[b][layer][t][:, n:n + k + 1]
                y = s_quad.cache[b][layer][t][:, n:n + k + 1]
                assert (x - y).abs().max().item() < 1e-12
    for a in range(k + 1):
        sep = copy.deepcopy(st)
        toks = torch.tensor([[sep.pending[b]] + drafts[b][:a] for b in range(2)], dtype=torch.int64)
        mdl.forward(toks, sep.lens, sep.cache, block_size=1, write_kv=True, with_logits=False)
        starts = [sep.lens[b] + a + 1 for b in range(2)]
        masks = torch.full((2, k), cfg.mask_id, dtype=torch.int64)
        want = mdl.forward(masks, starts, sep.cache, block_size=k, write_kv=False, lora=True)
        assert (pl[:, a] - want).abs().max().item() < 1e-10


@pytest.mark.parametrize("seed", [9, 4])
def test_quadratic_generation_is_lossless_and_one_forward_per_round(seed):
    cfg = _tiny(n_layers=1)
    W = synth.model_weights(cfg, 5)
    W[-1] = W[0][:cfg.vocab].clone() * 50.0      # peaky head tied to the embedding: drafts hit
    mdl = oracle.OracleModel(cfg, W, "f64")
    p = synth.prompt_tokens(2, 12, cfg.vocab, seed=seed)
    k, n = 4, 24
    got, forwards, per = odec.quadratic_generate(mdl, p, n, k, 128)
    assert got == odec.ar_generate(mdl, p, n, 128)
    rounds = len(per[0])
    assert forwards == 1 + rounds
    assert all(1 <= c <= k + 1 for row in per for c in row)
    assert max(c for row in per for c in row) > 1        # multi-token commits happen


def test_quadratic_round_picks_the_block_of_the_outcome():
    """Drafts equal to the AR continuation are all accepted (k+1 commits) and the next drafts
    come from block P_k; drafts that miss at once commit 1 token and use block P_0."""
    import copy
    cfg = _tiny(n_layers=1)
    mdl = oracle.OracleModel(cfg, synth.model_weights(cfg, 0), "f64")
    k = 3
    p = synth.prompt_tokens(1, 10, cfg.vocab, seed=7)
    cont = odec.ar_generate(mdl, p, k + 1, 64)[0]
    st = odec.prefill(mdl, p, 64)
    for drafts, a in (([cont[:k]], k), ([[(cont[0] + 1) % cfg.vocab] * k], 0)):
        s1, s2 = copy.deepcopy(st), copy.deepcopy(st)
        _, pl = odec.quadratic_forward(mdl, s1, drafts)
        committed, nxt = odec.quadratic_round(mdl, s2, drafts)
        assert committed[0] == cont[:a + 1]
        assert nxt[0] == odec.argmax_lowest(pl[0, a]).tolist()
        assert s2.lens[0] == st.lens[0] + a + 1 and s2.pending[0] == cont[a]


def _golden_rows(name):
    return [l.split() for l in open(os.path.join(GOLD, name))
            if l.strip() and not l.startswith("#")]


def test_fused_fill_mask_golden():
    want = torch.tensor([[int(x) for x in r] for r in _golden_rows("mask_fill_n2_c2_bs2_m6.txt")],
                        dtype=torch.bool)
    assert torch.equal(omod.block_mask(6, 2, 2, causal_rows=2), want)


def test_quadratic_layout_golden():
    rows = _golden_rows("quadratic_n1_k2.txt")
    assert rows[0][0] == "positions"
    m, pos, mask = odec.quadratic_layout(1, 2)
    assert pos.tolist() == [int(x) for x in rows[0][1:]]
    want = torch.tensor([[int(x) for x in r] for r in rows[1:]], dtype=torch.bool)
    assert m == 9 and torch.equal(mask, want)
