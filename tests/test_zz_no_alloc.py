"""nld_lm_head_argmax_static: the allocation-free variant of the stand-alone LM head, for callers
that cannot allocate device memory (code inside a framework that owns every device allocation
through its own pool; latency-critical paths where cudaMalloc would synchronise the device).

It must give what nld_lm_head_argmax gives with a caller workspace, on two calls in a row (the
built-in scratch keeps the previous call's contents), and refuse shapes whose scratch exceeds
the built-in size.  This file is collected last so that a failure here does not hide others."""
import pytest
import torch

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _inputs(M, d, V, seed):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(M, d, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(V, d, generator=g) * 0.02).to(torch.bfloat16).cuda()
    return h, w


def test_static_scratch_matches_workspace_entry_two_calls():
    import self_speculation_b200 as nb
    for call, (M, d, V) in enumerate([(33, 4096, 151936), (65, 512, 5000)]):
        h, w = _inputs(M, d, V, seed=10 + call)
        ws = torch.zeros(nb.nld_lm_head_workspace_size(M, d, V), dtype=torch.uint8, device="cuda")
        am_ref = torch.empty(M, dtype=torch.int32, device="cuda")
        cf_ref = torch.empty(M, dtype=torch.float32, device="cuda")
        nb.nld_lm_head_argmax(h, w, EPS, am_ref, cf_ref, ws)
        am = torch.full((M,), -7, dtype=torch.int32, device="cuda")
        cf = torch.full((M,), -7.0, dtype=torch.float32, device="cuda")
        nb.nld_lm_head_argmax_static(h, w, EPS, am, cf)
        torch.cuda.synchronize()
        # same kernels, same tiling: the argmax must agree and the confidence within the
        # 1e-3 relative bar of the LM-head tests
        assert torch.equal(am.cpu(), am_ref.cpu())
        assert ((cf - cf_ref).abs() / cf_ref).max().item() < 1e-3


def test_static_scratch_rejects_oversize():
    import self_speculation_b200 as nb
    lib = nb.load_library()
    limit = lib.nld_lm_head_static_max_bytes()
    assert limit == 8 << 20
    M, d, V = 1024, 4096, 151936          # needs ~19.6 MB of scratch
    assert nb.nld_lm_head_workspace_size(M, d, V) > limit
    h = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(V, d, dtype=torch.bfloat16, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    cf = torch.empty(M, dtype=torch.float32, device="cuda")
    with pytest.raises(nb.NldError) as ei:
        nb.nld_lm_head_argmax_static(h, w, EPS, am, cf)
    assert ei.value.status == 1 and "exceeds the built-in" in str(ei.value)
