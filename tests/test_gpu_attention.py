"""Stand-alone block-causal GQA attention over the paged bf16 KV cache (nld_attention) against
the oracle's explicit-mask attention.

Inputs: Q, K, V i.i.d. N(0,1) rounded to bf16; 32 q heads / 8 kv heads x 128; a block of m
queries per sequence after a cached prefix; per-sequence prefixes off page boundaries; pages of
each sequence scattered over the pool (page table).  Bar: max-abs error 2e-2 on outputs that
are convex combinations of N(0,1) values (|o| < ~4): bf16 output rounding contributes <= 8e-3,
the bf16 rounding of the probabilities in the P.V product a few 1e-3 more.
"""
import pytest
import torch

import synth
from oracle import model as omod

pytestmark = pytest.mark.gpu

HQ, HKV, HD = 32, 8, 128
TOL = 2e-2


KERNELS = {"mma_sync": (2, 0), "tcgen05_2_k64": (3, 64), "tcgen05_2_k128": (3, 128),
           "tcgen05_4_k64": (4, 64), "tcgen05_4_k128": (4, 128)}


@pytest.fixture(autouse=True, params=list(KERNELS))
def attention_kernel(request):
    """Every case runs on each tensor-core attention kernel: mma.sync, and tcgen05 with 2 or 4
    softmax threads per row and KV tiles of 64 keys (P in TMEM columns of its own) or 128 (P
    over S), whatever the split lengths (the process-wide switches are put back afterwards)."""
    import self_speculation_b200 as nb
    lib = nb.load_library()
    kernel, tile = KERNELS[request.param]
    assert lib.nld_debug_attention_kernel(kernel) == 0
    assert lib.nld_debug_attention_tile(tile) == 0
    yield request.param
    assert lib.nld_debug_attention_kernel(0) == 0
    assert lib.nld_debug_attention_tile(0) == 0


def _setup(lens, m, seed=2, shuffle_seed=0):
    import self_speculation_b200 as nb
    B = len(lens)
    L = max(lens)
    q, k, v = synth.attention_operands(B, m, HQ, HKV, HD, L, seed=seed)
    pps = (L + m + 63) // 64
    n_pages = B * pps + 3
    g = torch.Generator().manual_seed(shuffle_seed)
    perm = torch.randperm(n_pages, generator=g)[:B * pps].view(B, pps).to(torch.int32)
    pool = torch.zeros(n_pages, 2, HKV, 64, HD, dtype=torch.bfloat16)
    for b in range(B):
        n = lens[b] + m
        for j in range(n):
            pg, sl = int(perm[b, j // 64]), j % 64
            # sequence b uses rows 0..lens[b]-1 as prefix and the next m rows for its queries
            src = j if j < lens[b] else (L + (j - lens[b]))
            pool[pg, 0, :, sl] = k[b, :, src]
            pool[pg, 1, :, sl] = v[b, :, src]
    return q, k, v, pool, perm, pps


def _oracle(q, k, v, lens, m, bs):
    B = q.shape[0]
    L = k.shape[2] - m
    out = torch.empty(B, m, HQ, HD, dtype=torch.float64)
    for b in range(B):
        n = lens[b]
        keys = torch.cat([k[b, :, :n], k[b, :, L:L + m]], dim=1).double()
        vals = torch.cat([v[b, :, :n], v[b, :, L:L + m]], dim=1).double()
        mask = omod.block_mask(m, n, bs)
        o = omod.attention_explicit(q[b].transpose(0, 1).double(), keys, vals, mask)
        out[b] = o.transpose(0, 1)
    return out


def _run(q, pool, perm, lens, m, bs, max_len):
    import self_speculation_b200 as nb
    B = q.shape[0]
    out = torch.empty(B, m, HQ, HD, dtype=torch.bfloat16, device="cuda")
    nb.nld_attention(q.cuda(), pool.cuda(), perm.cuda(), torch.tensor(lens, dtype=torch.int32).cuda(),
                     bs, max_len, out)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("bs", [32, 1, 8])
@pytest.mark.parametrize("lens", [[0], [37, 200, 64], [1000]])
def test_attention_block_modes(bs, lens):
    m = 32
    q, k, v, pool, perm, pps = _setup(lens, m)
    got = _run(q, pool, perm, lens, m, bs, max(lens) + m)
    want = _oracle(q, k, v, lens, m, bs)
    err = (got.double() - want).abs().max().item()
    assert err < TOL, err


def test_attention_33_rows_causal():
    lens = [129, 5]
    m = 33
    q, k, v, pool, perm, pps = _setup(lens, m)
    got = _run(q, pool, perm, lens, m, 1, max(lens) + m)
    want = _oracle(q, k, v, lens, m, 1)
    assert (got.double() - want).abs().max().item() < TOL


def test_block_size_one_equals_causal_and_differs_from_block():
    lens = [300]
    m = 32
    q, k, v, pool, perm, pps = _setup(lens, m)
    a = _run(q, pool, perm, lens, m, 1, 332)
    b = _run(q, pool, perm, lens, m, 32, 332)
    # row 0 of a block sees the whole block in block mode, only itself in causal mode
    assert (a[0, 0].float() - b[0, 0].float()).abs().max().item() > 1e-2
    # the last row sees the same keys in both modes
    assert (a[0, -1].float() - b[0, -1].float()).abs().max().item() < 1e-2


def test_attention_long_prefix_sampled():
    """Batch 8, 4k prefix: full oracle over the sampled sequences 0 and 7."""
    lens = [4096] * 8
    m = 32
    q, k, v, pool, perm, pps = _setup(lens, m, shuffle_seed=3)
    got = _run(q, pool, perm, lens, m, 32, 4096 + m)
    for b in (0, 7):
        want = _oracle(q[b:b + 1], k[b:b + 1], v[b:b + 1], [4096], m, 32)
        assert (got[b:b + 1].double() - want).abs().max().item() < TOL


def test_repeated_calls_identical():
    """Deterministic merge order: repeated calls give bit-identical outputs."""
    lens = [500]
    m = 32
    q, k, v, pool, perm, pps = _setup(lens, m)
    a = _run(q, pool, perm, lens, m, 32, 532)
    b = _run(q, pool, perm, lens, m, 32, 532)
    assert torch.equal(a, b)


@pytest.mark.parametrize("L,bs", [(16384, 32), (16384, 1), (16384, 8), (32768, 32), (32768, 1)])
def test_attention_microbench_prefix_batch32_sampled(L, bs):
    """The attention micro-workload's largest points: batch 32, prefixes 16k and 32k, block
    (32), causal (1) and block size 8 masks; operands built on the GPU, pages scattered by a
    random page table; the oracle runs on sequences 0 and 31."""
    B, m = 32, 32
    q, k, v = synth.attention_operands(B, m, HQ, HKV, HD, L, seed=5, device="cuda")
    pps = (L + m + 63) // 64
    n_pages = B * pps
    g = torch.Generator(device="cuda").manual_seed(7)
    perm = torch.randperm(n_pages, generator=g, device="cuda").view(B, pps).to(torch.int32)
    pool = torch.zeros(n_pages, 2, HKV, 64, HD, dtype=torch.bfloat16, device="cuda")
    j = torch.arange(L + m, device="cuda")
    pg = perm[:, j // 64].long()                       # [B, L+m] page of key row j
    sl = (j % 64)[None, :].expand(B, -1)               # its slot in the page
    pool_k, pool_v = pool[:, 0], pool[:, 1]
    pool_k[pg, :, sl, :] = k.permute(0, 2, 1, 3)
    pool_v[pg, :, sl, :] = v.permute(0, 2, 1, 3)
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    import self_speculation_b200 as nb
    out = torch.empty(B, m, HQ, HD, dtype=torch.bfloat16, device="cuda")
    nb.nld_attention(q, pool, perm, lens, bs, L + m, out)
    torch.cuda.synchronize()
    for b in (0, B - 1):
        want = _oracle(q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu(), [L], m, bs)
        assert (out[b:b + 1].cpu().double() - want).abs().max().item() < TOL
