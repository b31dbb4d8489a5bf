"""Host logic of the launch planners, on CPU through the pure-host hooks nld_plan_chain and
nld_plan_attention: every plan the library can make for the benchmark and test shapes keeps
the kernels' limits (227 KB of shared memory, TMEM columns a power of two covering the
double-buffered accumulator, split-K factors that give every rank work, <= 9 attention warps,
<= 8 KV splits, no KV split left without a tile), and the plans at the benchmarked decode shape
are the ones the committed launch list records (layer chain 132 CTAs in clusters of 4, layer-0
QKV 96 CTAs in clusters of 2, attention in query tiles of <= 64 rows and single-tile KV
splits)."""
import ctypes
import itertools

import pytest

import self_speculation_b200 as nb
import synth

SMEM_BUDGET = 227 * 1024
MAX_STAGES = 8
# clusters of each size resident at once with one ~200 KB CTA per SM on 148 SMs (the device
# reports these through an occupancy query; 33 clusters of 4 is the measured figure)
B200_CLUSTERS = [0, 148, 74, 0, 33, 0, 0, 0, 16]


def plan_chain(M, phases, clusters=B200_CLUSTERS, hilo=1):
    lib = nb.load_library()
    n = len(phases)
    rows = (ctypes.c_int * n)(*[r for r, _ in phases])
    K = (ctypes.c_int * n)(*[k for _, k in phases])
    mc = (ctypes.c_int * 9)(*clusters)
    out = (ctypes.c_int * 20)()
    st = lib.nld_plan_chain(M, n, rows, K, mc, hilo, out)
    assert st == 0, lib.nld_last_error(None)
    o = list(out)
    return dict(CS=o[0], NT=o[1], xr=o[2], kps=o[3], stages=o[4], slots=o[5], tmem=o[6],
                grid=o[7], smem=o[8], tok_tiles=o[9],
                split=[(o[10 + 2 * p], o[11 + 2 * p]) for p in range(n)])


def plan_attention(batch, m, Hq, Hkv, max_len, sms=148, kernel=0, tile=0):
    """kernel: 0 the planner's choice, 1 tcgen05, 2 mma.sync; tile: keys per tcgen05 KV tile, 0
    the planner's choice (the process-wide settings are put back)."""
    lib = nb.load_library()
    out = (ctypes.c_int * 8)()
    assert lib.nld_debug_attention_kernel(kernel) == 0
    assert lib.nld_debug_attention_tile(tile) == 0
    try:
        assert lib.nld_plan_attention(batch, m, Hq, Hkv, max_len, sms, out) == 0
    finally:
        assert lib.nld_debug_attention_kernel(0) == 0
        assert lib.nld_debug_attention_tile(0) == 0
    return dict(zip(["G", "QT", "q_tiles", "rows", "NW", "S", "tc", "tile"], list(out)))


def chains(cfg):
    """The projection chains of a forward: layer-0 QKV, a decode layer, the last layer with the
    LM head, and the stand-alone LM head."""
    qd, kvd, d, F, V = cfg.q_dim, cfg.kv_dim, cfg.d_model, cfg.ffn_dim, cfg.vocab
    o, gu, dn, qkv, lm = (d, qd), (2 * F, d), (d, F), (qd + 2 * kvd, d), (V, d)
    return {"qkv0": [qkv], "layer": [o, gu, dn, qkv], "last": [o, gu, dn, lm], "lm": [lm]}


def decode_Ms(cfg):
    k = cfg.block_k
    Ms = {1, 2048}
    for B in {1, 2, 4, cfg.max_batch}:
        Ms |= {B, B * k, B * (k + 1), B * 2 * k}
    return sorted(m for m in Ms if m <= max(2048, cfg.max_batch * (k + 1)))


SHAPES = [("8b", synth.LLAMA8B.replace(max_batch=64)), ("14b", synth.LLAMA14B.replace(max_batch=64)),
          ("small", synth.SMALL_BF16)]


@pytest.mark.parametrize("name,cfg", SHAPES, ids=[s[0] for s in SHAPES])
def test_chain_plans_keep_kernel_limits(name, cfg):
    for M in decode_Ms(cfg):
        for kind, phases in chains(cfg).items():
            # the context's chains take (hi, lo) activation row pairs; the stand-alone LM head
            # takes the caller's plain bf16 rows
            hilo = 0 if kind == "lm" else 1
            for clusters in (B200_CLUSTERS, [0, 100, 50, 0, 20, 0, 0, 0, 8]):
                P = plan_chain(M, phases, clusters, hilo)
                where = (name, kind, M, clusters[4])
                assert P["smem"] <= SMEM_BUDGET, where
                assert 2 <= P["stages"] <= MAX_STAGES and P["kps"] in (1, 2), where
                assert P["stages"] >= 3 or P["kps"] == 1, where
                assert P["CS"] in (1, 2, 4, 8) and clusters[P["CS"]] >= 1, where
                NT = P["NT"]
                NN = NT << hilo            # MMA N: activation rows of a token tile
                assert NT % 16 == 0 and 16 <= NT and NN <= 256 and NT * P["tok_tiles"] >= M, where
                assert P["xr"] % 8 == 0 and P["xr"] <= NN, where
                if P["tok_tiles"] == 1:
                    assert P["xr"] >= M << hilo, where
                t = P["tmem"]
                assert t & (t - 1) == 0 and 2 * NN <= t <= 512, where
                # the MMA reads NN activation rows from each xr-row box: the last box of the
                # ring is read (NN - xr) rows past its end, which must stay in the allocation
                ring = P["stages"] * P["kps"] * (16384 + P["xr"] * 128)
                assert P["smem"] >= ring + (NN - P["xr"]) * 128, where
                assert P["grid"] % P["CS"] == 0 and P["grid"] <= P["CS"] * clusters[P["CS"]], where
                if len(phases) > 1 and NT <= 64:
                    assert P["CS"] == 4, where
                for (rows, K), (s, ks) in zip(phases, P["split"]):
                    KT = K // 64
                    assert P["CS"] % s == 0 and s * ks >= KT and (s - 1) * ks < KT, where
                # split-K receive slots: (s - 1) senders x the 16-token chunks a rank owns
                for s, _ in P["split"]:
                    if s > 1:
                        assert P["slots"] >= (s - 1) * -(-(NT // 16) // s), where


def test_decode_plans_match_the_recorded_launch_list():
    cfg = synth.LLAMA8B
    ch = chains(cfg)
    # (hi, lo) activation rows: 66 / 64 rows per k-tile box, MMA N = 96 / 64
    for M, NT, xr in ((33, 48, 72), (32, 32, 64)):
        P = plan_chain(M, ch["layer"])
        assert (P["CS"], P["NT"], P["xr"], P["stages"], P["grid"]) == (4, NT, xr, 4, 132)
        L = plan_chain(M, ch["last"])
        assert (L["CS"], L["grid"]) == (4, 132)
    Q = plan_chain(33, ch["qkv0"])
    assert (Q["CS"], Q["grid"]) == (2, 96)


@pytest.mark.parametrize("name,cfg", SHAPES, ids=[s[0] for s in SHAPES])
def test_attention_plans_keep_kernel_limits(name, cfg):
    for M in decode_Ms(cfg):
        for B in {1, 4, cfg.max_batch}:
            if M % B:
                continue
            m = M // B
            if m > 2 * cfg.block_k + 1:
                continue
            for max_len, kernel in itertools.product((m, 64, 900, 4096 + m, 32768), (0, 1, 2)):
                A = plan_attention(B, m, cfg.n_q_heads, cfg.n_kv_heads, max_len, kernel=kernel)
                where = (name, B, m, max_len, kernel)
                assert A["G"] * cfg.n_kv_heads == cfg.n_q_heads, where
                assert 1 <= A["QT"] <= m and A["QT"] * A["q_tiles"] >= m, where
                assert A["rows"] == A["QT"] * A["G"] and A["rows"] <= 16 * A["NW"], where
                assert 1 <= A["NW"] <= 9 and A["rows"] <= 144, where
                assert A["tc"] == {1: 1, 2: 0}.get(kernel, A["tc"]), where
                if A["tc"]:
                    assert A["rows"] <= 128, where   # one tcgen05 MMA tile
                assert 1 <= A["S"] <= 8, where
                assert A["tile"] in ((64, 128) if A["tc"] else (64,)), where
                assert A["S"] <= -(-max_len // A["tile"]), where   # every split has a KV tile
                if B * A["q_tiles"] * cfg.n_kv_heads >= 2 * 148:
                    assert A["S"] == 1, where


def test_attention_plan_of_the_benchmarked_round():
    # tcgen05 (the planner's choice; KV tiles of 64 keys at batch 1): verify forward (m = 33: 2
    # query tiles of 17 positions x 4 heads) and draft forward (m = 32: one 128-row tile); 545
    # keys = 9 tiles in 5 splits of <= 2, 865 keys = 14 tiles in 7 splits, 1400 keys = 22 tiles
    # in 8 splits of <= 3
    for keys, S in ((545, 5), (865, 7), (1400, 8)):
        v = plan_attention(1, 33, 32, 8, keys)
        d = plan_attention(1, 32, 32, 8, keys)
        assert (v["G"], v["QT"], v["q_tiles"], v["rows"], v["S"], v["tc"], v["tile"]) == (4, 17, 2, 68, S, 1, 64)
        assert (d["QT"], d["q_tiles"], d["rows"], d["S"], d["tc"], d["tile"]) == (32, 1, 128, S, 1, 64)
    # mma.sync: 3 query tiles of 11 positions (3 warps) and 2 tiles of 16 positions (4 warps)
    for keys, S in ((545, 5), (865, 7)):
        v = plan_attention(1, 33, 32, 8, keys, kernel=2)
        d = plan_attention(1, 32, 32, 8, keys, kernel=2)
        assert (v["G"], v["QT"], v["q_tiles"], v["NW"], v["S"], v["tc"]) == (4, 11, 3, 3, S, 0)
        assert (d["QT"], d["q_tiles"], d["NW"], d["S"], d["tc"]) == (16, 2, 4, S, 0)
    # many sequences: the 33-position verify block of 4 heads in two tcgen05 tiles of 17 and 16
    # positions (2 x 56 < 132 rows of one 9-warp mma.sync CTA), a 32-position block in one
    b = plan_attention(64, 33, 32, 8, 4096 + 33)
    assert (b["QT"], b["q_tiles"], b["rows"], b["S"], b["tc"]) == (17, 2, 68, 1, 1)
    b = plan_attention(64, 33, 32, 8, 4096 + 33, kernel=2)
    assert (b["QT"], b["q_tiles"], b["NW"], b["S"], b["tc"]) == (33, 1, 9, 1, 0)
    b = plan_attention(64, 32, 32, 8, 4096 + 32)
    assert (b["QT"], b["q_tiles"], b["rows"], b["S"], b["tc"], b["tile"]) == (32, 1, 128, 1, 1, 128)
    # the tcgen05 KV tile: 64 keys while a split holds <= 3 pages, else 128 (1056 keys = 17
    # pages: 6 splits of 3 at batch 1; 4128 keys = 65 pages = 33 tiles of 128 keys: 7 splits of
    # 5 at batch 1, 2 splits of 17 at batch 8; 16416 keys at batch 1: 8 splits of 17 tiles)
    b = plan_attention(1, 32, 32, 8, 1056)
    assert (b["S"], b["tc"], b["tile"]) == (6, 1, 64)
    b = plan_attention(8, 32, 32, 8, 1056)
    assert (b["tc"], b["tile"]) == (1, 128)
    b = plan_attention(1, 32, 32, 8, 4128)
    assert (b["S"], b["tc"], b["tile"]) == (7, 1, 128)
    b = plan_attention(8, 32, 32, 8, 4128)
    assert (b["S"], b["tc"], b["tile"]) == (2, 1, 128)
    b = plan_attention(1, 32, 32, 8, 16416)
    assert (b["S"], b["tc"], b["tile"]) == (8, 1, 128)
    # a forced tile plans the splits in its own tiles: 545 keys = 9 pages = 5 tiles of 128 keys
    # (5 splits of one); 4128 keys at batch 8 in 64-key tiles: 2 splits of 33
    b = plan_attention(1, 32, 32, 8, 545, tile=128)
    assert (b["S"], b["tc"], b["tile"]) == (5, 1, 128)
    b = plan_attention(8, 32, 32, 8, 4128, tile=64)
    assert (b["S"], b["tc"], b["tile"]) == (2, 1, 64)
    # the tile is the tcgen05 kernel's: mma.sync plans keep 64-key pages
    assert plan_attention(1, 1, 32, 8, 4096, tile=128)["tile"] == 64
    # small query tiles (a 4-row single-token decode, 32-row blocks of many sequences) cost the
    # tcgen05 kernel a whole 128-row tile per KV tile: they stay on mma.sync; 64-row blocks go to
    # tcgen05
    assert plan_attention(1, 1, 32, 8, 4096)["tc"] == 0
    assert plan_attention(64, 1, 32, 8, 4096)["tc"] == 0
    assert plan_attention(16, 8, 32, 8, 2048)["tc"] == 0
    assert plan_attention(16, 16, 32, 8, 2048)["tc"] == 1
    assert plan_attention(1, 16, 32, 8, 2048)["tc"] == 1


def test_plan_hooks_reject_bad_sizes():
    lib = nb.load_library()
    out = (ctypes.c_int * 20)()
    rows = (ctypes.c_int * 1)(4096)
    bad_k = (ctypes.c_int * 1)(100)
    mc = (ctypes.c_int * 9)(*B200_CLUSTERS)
    assert lib.nld_plan_chain(33, 1, rows, bad_k, mc, 1, out) == 1
    assert lib.nld_plan_chain(0, 1, rows, (ctypes.c_int * 1)(4096), mc, 1, out) == 1
    none = (ctypes.c_int * 9)(*([0] * 9))
    assert lib.nld_plan_chain(33, 1, rows, (ctypes.c_int * 1)(4096), none, 1, out) == 8   # unsupported
    assert lib.nld_plan_attention(1, 33, 32, 7, 100, 148, (ctypes.c_int * 8)()) == 1
