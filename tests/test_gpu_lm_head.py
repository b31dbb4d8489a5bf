"""Stand-alone fused LM head + greedy token + confidence (nld_lm_head_argmax) against a float64
evaluation of its definition: logits = (h / rms(h)) W^T over bf16 inputs, argmax with the lowest
id on ties, confidence = largest softmax probability.  Logits are accumulated in fp32 on the
GPU (errors ~1e-5 here), so argmaxes must agree wherever the top-2 margin exceeds 1e-3 and
confidences within 1e-3 relative."""
import pytest
import torch

from oracle import decode as odec

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _reference(h, w):
    hd = h.double()
    inv = 1.0 / torch.sqrt((hd * hd).mean(-1, keepdim=True) + EPS)
    logits = (hd @ w.double().t()) * inv
    return logits, odec.argmax_lowest(logits), odec.confidence(logits)


def _run(h, w):
    import self_speculation_b200 as nb
    M, d = h.shape
    V = w.shape[0]
    ws = torch.zeros(nb.nld_lm_head_workspace_size(M, d, V), dtype=torch.uint8, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    cf = torch.empty(M, dtype=torch.float32, device="cuda")
    nb.nld_lm_head_argmax(h.cuda(), w.cuda(), EPS, am, cf, ws)
    torch.cuda.synchronize()
    return am.cpu(), cf.cpu()


@pytest.mark.parametrize("M,d,V,scale", [(33, 512, 5000, 1.0), (77, 1024, 4096, 30.0),
                                         (1, 4096, 151936, 1.0), (300, 512, 1000, 5.0)])
def test_lm_head_matches_definition(M, d, V, scale):
    g = torch.Generator().manual_seed(M + d + V)
    h = torch.randn(M, d, generator=g).to(torch.bfloat16)
    w = (torch.randn(V, d, generator=g) * 0.02 * scale).to(torch.bfloat16)
    logits, am_ref, cf_ref = _reference(h, w)
    am, cf = _run(h, w)
    top = torch.topk(logits, 2, dim=-1).values
    sure = (top[:, 0] - top[:, 1]) > 1e-3
    assert torch.equal(am[sure].long(), am_ref[sure])
    assert ((cf.double() - cf_ref) / cf_ref).abs().max().item() < 1e-3


def test_lm_head_ties_pick_lowest_id():
    g = torch.Generator().manual_seed(3)
    M, d, V = 8, 256, 700
    h = torch.randn(M, d, generator=g).to(torch.bfloat16)
    w = (torch.randn(V, d, generator=g) * 0.02).to(torch.bfloat16)
    w[650] = h[0] * 0.5      # dominant row for token 0, duplicated at ids 129 and 650
    w[129] = w[650]
    am, _ = _run(h, w)
    assert int(am[0]) == 129
