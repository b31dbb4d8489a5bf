#!/usr/bin/env python
"""Benchmark of the self-speculation decode round (8B-shaped decoder, batch 1 per GPU).

A step is one linear self-speculation round through the C ABI: draft forward (one
bidirectional block of k=32 positions over the cached prefix), causal verify forward (k+1
positions), greedy acceptance and KV commit.  Weights are random-init bf16 of the 8B shape
(36 layers, d 4096, 32/8 heads x 128, FFN 12288, vocab 151936); the prompt is 512 uniform
random ids (synthetic stand-in for the benchmark prompts).  Every forward streams 15.1 GB of
weights, far above the 126 MB L2, so no L2 flush is needed between steps.

Multi-GPU: replicas only (every rank decodes its own sequence; there is no exchange step in
the round).  Timing: CUDA events on the library's stream, max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "committed tokens/s & self-spec rounds/s at batch 1 (8B shape); % HBM roofline"
PROMPT = 512
K_BLOCK = 32
GEN_TOKENS = 1024      # the generation length of the 8B self-speculation workload
HBM_FALLBACK_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return HBM_FALLBACK_GBS, "fallback"


def kernel_source_sha() -> str:
    """Hash of the layer-chain kernel's own sources (the kernel, its epilogues and the device
    helpers it includes)."""
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "epilogue.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "self_speculation_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha") != kernel_source_sha():
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class Clocks:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce(vals, op, world):
    """Replica timing reduction: max (time) or sum (tokens) over ranks.  The only collective of
    a multi-GPU run; the decode round itself exchanges nothing between replicas."""
    import torch
    if world == 1:
        return vals
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(vals, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return t.tolist()


# ------------------------------------------------------------------------- CPU oracle leg --

class OracleRounds:
    """The CPU oracle as it stands running whole linear self-speculation rounds of the 8B shape:
    all 36 layers and the LM head, fp32 arithmetic with a bf16 KV cache, weights held as bf16
    and widened per matmul.  The cache holds 511 zero-valued rows (the work of a round does not
    depend on the cached values), so no 511-token prefill is run on the host.  Each call of
    round() is one draft forward (k rows), one verify forward (k+1 rows) and the commit, timed
    with the host clock."""

    def __init__(self, threads: int, n_layers: int = 36):
        import torch

        import oracle
        import synth
        torch.set_num_threads(threads)
        self.cfg = synth.LLAMA8B.replace(n_layers=n_layers)
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        W = [w.cpu() for w in synth.model_weights(self.cfg, 0, device=dev)]
        self.om = oracle.OracleModel(self.cfg, W, "f32kv")
        self.cap = PROMPT + 8 * (K_BLOCK + 1)

    def round(self):
        """Seconds of one measured round and the tokens it committed."""
        t_d, drafts = self.draft()
        t_v, committed = self.verify_commit(drafts)
        return t_d + t_v, committed

    def _state(self):
        from oracle import decode as odec
        return odec.SeqState(cache=self.om.new_cache(1, self.cap), lens=[PROMPT - 1], pending=[7])

    def draft(self):
        """Seconds of one draft forward (k rows, block-bidirectional) and its drafts."""
        import torch

        from oracle import decode as odec
        om, cfg, k = self.om, self.cfg, K_BLOCK
        self.st = self._state()
        t0 = time.perf_counter()
        draft_toks = torch.full((1, k), cfg.mask_id, dtype=torch.int64)
        draft_toks[0, 0] = self.st.pending[0]
        dl = om.forward(draft_toks, self.st.lens, self.st.cache, block_size=k, write_kv=False)
        drafts = odec.argmax_lowest(dl).tolist()[0]
        return time.perf_counter() - t0, drafts

    def verify_commit(self, drafts):
        """Seconds of the verify forward (k+1 causal rows) and commit after draft(); tokens
        committed."""
        import torch

        from oracle import decode as odec
        om, st = self.om, self.st
        t0 = time.perf_counter()
        ver_toks = torch.tensor([[st.pending[0]] + drafts], dtype=torch.int64)
        vl = om.forward(ver_toks, st.lens, st.cache, block_size=1, write_kv=True)
        committed = odec.commit_after_verify(drafts, odec.argmax_lowest(vl).tolist()[0])
        return time.perf_counter() - t0, len(committed)


# ------------------------------------------------------------------------------ our arm --

def run_ours(args, world, rank, local):
    import torch

    import self_speculation_b200 as nb
    import synth
    from self_speculation_b200 import build as nbuild

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    nbuild.build()
    K, W = args.steps, args.warmup
    max_seq = (PROMPT + (K_BLOCK + 1) * (W + K + 2) + 63) // 64 * 64 + 64
    max_seq = max(max_seq, PROMPT + GEN_TOKENS + 4 * (K_BLOCK + 1))
    cfg = synth.LLAMA8B.replace(max_seq=max_seq)
    torch_stream = torch.cuda.Stream()          # owned by torch; the library orders on it
    ctx = nb.Context(cfg, stream=torch_stream.cuda_stream)
    weights = synth.model_weights(cfg, 0, device="cuda")
    ctx.nld_init_weights(weights, on_device=True)
    del weights
    if args.lora:
        # optional drafter adapter on o_proj (seeded random, scale 1): draft forwards only
        ctx.nld_init_lora(args.lora, 1.0, synth.lora_weights(cfg, args.lora, 0, device="cuda"))
    torch.cuda.empty_cache()
    prompt = synth.prompt_tokens(1, PROMPT, cfg.vocab, seed=1 + rank)
    ctx.nld_prefill(prompt.cuda())
    toks = torch.empty(1, K_BLOCK + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    lens = torch.empty(1, dtype=torch.int32, device="cuda")
    for _ in range(W):
        ctx.nld_selfspec_round(toks, nc, None)
    ctx.nld_sync()
    ctx.nld_debug_state(lens)
    ctx.nld_sync()
    len0 = int(lens.item())
    stream = torch_stream
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = Clocks(local)
    clk.start()
    time.sleep(0.3)
    e0.record(stream)
    for _ in range(K):
        ctx.nld_selfspec_round(toks, nc, None)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = clk.stop()
    ms = e0.elapsed_time(e1)
    ctx.nld_sync()
    ctx.nld_debug_state(lens)
    ctx.nld_sync()
    len1 = int(lens.item())
    committed = len1 - len0
    max_ms, = reduce([ms], "max", world)
    tot_committed, = reduce([float(committed)], "sum", world)
    value = tot_committed / (max_ms / 1e3)
    rounds_per_s = world * K / (max_ms / 1e3)

    # round roofline: weight bytes of two forwards + KV rows read + KV rows written
    hbm, peak_src = peaks()
    wbytes = cfg.weight_bytes_per_forward()
    kvb = cfg.kv_bytes_per_token()
    L_avg = (len0 + len1) / 2.0
    round_bytes = 2 * wbytes + (2 * L_avg + K_BLOCK + (K_BLOCK + 1)) * kvb \
        + (2 * K_BLOCK + 1) * kvb + 2 * cfg.n_layers * args.lora * (cfg.q_dim + cfg.d_model)
    round_s = ms / 1e3 / K
    round_gbs = round_bytes / round_s / 1e9

    # dominant kernel: the fused gate/up GEMM of a verify forward (201 MB of weights / launch)
    M = K_BLOCK + 1
    kern = {}
    names = ["qkv", "o", "gate_up", "down", "lm_head"]
    n_rows = [cfg.q_dim + 2 * cfg.kv_dim, cfg.d_model, 2 * cfg.ffn_dim, cfg.d_model, cfg.vocab]
    k_dim = [cfg.d_model, cfg.q_dim, cfg.d_model, cfg.ffn_dim, cfg.d_model]
    for w, (nm, nr, kd) in enumerate(zip(names, n_rows, k_dim)):
        reps = 10 if nm == "lm_head" else 40
        t = ctx.nld_time_gemm(w, 0, M, reps)
        byts = 2 * nr * kd + 2 * M * kd + (2 * M * nr // (2 if nm == "gate_up" else 1))
        kern[nm] = {"ms": round(t, 5), "GB/s": round(byts / (t / 1e3) / 1e9, 1),
                    "bytes": byts}
    # dominant kernel: the decode chain of a layer (O, gate/up, down, next layer's QKV in one
    # persistent launch), timed alone over the verify forward's M = k+1 rows
    ch_ms = ctx.nld_time_chain(0, M, 20)
    ch_bytes = sum(kern[n]["bytes"] for n in ("o", "gate_up", "down", "qkv"))
    ch_gbs = ch_bytes / (ch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(ch_gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ch_gbs / hbm, 4),
                "traffic": ncu_traffic("gemm_chain_layer_8b_m32.txt"),
                "kernel": "gemm_chain_kernel: one decode layer (O, gate/up, down, next QKV), "
                          "8B shape, M=33 tokens, timed alone with CUDA events",
                "bytes_per_launch": ch_bytes, "ms_per_launch": round(ch_ms, 5),
                "peak_kind": f"{peak_src} HBM copy (burst)"}

    # end to end through the public API: prompt H2D from pinned memory, prefill, K rounds, each
    # followed by a D2H read of the committed tokens and counts
    ctx2_tokens = 0
    host_prompt = prompt.pin_memory()
    h_toks = torch.empty(1, K_BLOCK + 1, dtype=torch.int32).pin_memory()
    h_nc = torch.empty(1, dtype=torch.int32).pin_memory()
    dev_prompt = torch.empty_like(prompt, device="cuda")
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        dev_prompt.copy_(host_prompt, non_blocking=True)
    stream.synchronize()
    ctx.nld_prefill(dev_prompt)
    for _ in range(K):
        ctx.nld_selfspec_round(toks, nc, None)
        with torch.cuda.stream(stream):
            h_toks.copy_(toks, non_blocking=True)
            h_nc.copy_(nc, non_blocking=True)
        stream.synchronize()
        ctx2_tokens += int(h_nc[0])
    e2e_s = time.perf_counter() - t0
    max_e2e, = reduce([e2e_s], "max", world)
    tot_e2e, = reduce([float(ctx2_tokens)], "sum", world)
    e2e = {"value": round(tot_e2e / max_e2e, 3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(PROMPT * 4 / K), "d2h_bytes_per_step": (K_BLOCK + 2) * 4,
           "includes": "prompt upload + prefill of 512 tokens + K rounds with a D2H read each"}

    # generation of config 3's length: a fresh 512-token prompt, rounds until 1024 tokens are
    # committed (the cached prefix grows 512 -> 1536), timed with CUDA events on the stream
    gen = None
    if not args.no_generation:
        ctx.nld_prefill(prompt.cuda())
        ctx.nld_sync()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        rounds, done = 0, 0
        while done < GEN_TOKENS:
            burst = max(1, min(64, (GEN_TOKENS - done + K_BLOCK) // (K_BLOCK + 1)))
            for _ in range(burst):
                ctx.nld_selfspec_round(toks, nc, None)
            rounds += burst
            ctx.nld_debug_state(lens)
            ctx.nld_sync()
            done = int(lens.item()) - (PROMPT - 1)
        g1.record(stream)
        g1.synchronize()
        gms = g0.elapsed_time(g1)
        gen = {"tokens": done, "rounds": rounds, "ms": round(gms, 2),
               "tokens_per_s": round(done / (gms / 1e3), 3),
               "ms_per_round": round(gms / rounds, 4),
               "prefix": f"{PROMPT} -> {PROMPT + done}",
               "note": "host reads the length every up to 64 rounds to stop at 1024 tokens"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        ref = OracleRounds(threads)
        secs, ncommit = [], 0
        for _ in range(2):
            s_round, c = ref.round()
            secs.append(s_round)
            ncommit += c
        cpu = {"value": round(ncommit / sum(secs), 5), "unit": "tokens/s", "cores": threads,
               "kind": "oracle",
               "sample": (f"2 whole self-speculation rounds of the 8B shape (36 layers + LM head, "
                          f"fp32 with a bf16 KV cache, 511 cached rows), measured: "
                          f"{', '.join(f'{x:.2f}' for x in secs)} s; {ncommit} committed tokens"),
               "round_s": round(sum(secs) / len(secs), 3)}

    # two forwards (draft, verify), each: embed, QKV chain of layer 0, per layer one attention
    # and one chain (O, gate/up, down, then the next QKV or, last, the LM head); then finalize
    # for draft, verify and commit; with an adapter the draft forward has one more launch per
    # layer (z = scale A att; B is folded into the chain's O projection)
    per_round = 2 * (1 + 1 + 2 * cfg.n_layers) + 3 + (cfg.n_layers if args.lora else 0)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(max_ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "8B-shaped linear self-speculation round, batch 1 per GPU, k=32, "
                               "prompt 512 random ids, random-init bf16 weights",
                   "layers": cfg.n_layers, "d_model": cfg.d_model, "heads": "32q/8kv x 128",
                   "ffn": cfg.ffn_dim, "vocab": cfg.vocab, "batch_per_gpu": 1, "block_k": K_BLOCK,
                   "prompt": PROMPT, "parallelism": f"replicas x{world}",
                   "lora_rank": args.lora,
                   "l2": "no flush: 15.1 GB of weights per forward exceed the 126 MB L2"},
        "rounds_per_s": round(rounds_per_s, 3),
        "tokens_per_forward": round(tot_committed / (2 * world * K), 4),
        "round_roofline": {"bound": "hbm", "achieved": round(round_gbs, 1), "peak": hbm,
                           "unit": "GB/s", "frac": round(round_gbs / hbm, 4),
                           "bytes_per_round": int(round_bytes)},
        "roofline": roofline,
        "kernels": kern,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "generation_1024": gen,
        "gpu_launches": K * per_round,
        "clocks": clocks,
    }
    ctx.close()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank, local):
    """The oracle as it stands on the host cores (rank 0 only), on the 8B round: the steps
    alternate between a round's draft forward and its verify forward + commit (all 36 layers and
    the LM head each), timed with the host clock, so that a step is half a round (~2.5 s) and the
    committed tokens are counted at the verify steps."""
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    ref = OracleRounds(threads, args.ref_layers)
    secs, committed = [], 0
    # the last step is a verify step: with an odd step count one more (untimed) draft leads
    lead = (args.warmup + args.steps) % 2
    drafts = None
    for i in range(-lead, args.warmup + args.steps):
        if (i + lead) % 2 == 0:
            s_step, drafts = ref.draft()
            c = 0
        else:
            s_step, c = ref.verify_commit(drafts)
        if i >= args.warmup:
            secs.append(s_step)
            committed += c
    value = committed / sum(secs)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(secs) / len(secs), 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "8B-shaped linear self-speculation round, batch 1, k=32, "
                               "prompt 512 random ids (CPU oracle)",
                   "layers": args.ref_layers, "parallelism": "host cores of rank 0"},
        "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle",
                         "sample": (f"per step: half a round, alternating the draft forward and the verify "
                                    f"forward + commit (each over {args.ref_layers} layers plus the LM head, "
                                    f"fp32 with a bf16 KV cache) at 511 cached rows, measured; tokens counted "
                                    f"at the verify steps")},
        "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _events_ms(fn, stream, reps, warm=3):
    import torch
    for _ in range(warm):
        fn()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def run_attention(args):
    """Attention micro-workload: 32 q / 8 kv heads x 128, a block of m = 32 queries per sequence
    (--attn-m) after a cached prefix of 1k/4k/16k/32k, batch 1/8/32, modes block-bidirectional
    (block 32), strict causal and block size 1.  Q/K/V ~ N(0,1) bf16 (seed 2) in a paged pool.
    HBM bytes per call: B*(L+m)*8*128*2*2 (K and V) + 2*B*m*32*128*2 (Q and O)."""
    import torch

    import self_speculation_b200 as nb
    from self_speculation_b200 import build as nbuild
    nbuild.build()
    hbm, peak_src = peaks()
    Hq, Hkv, hd, m = 32, 8, 128, args.attn_m
    stream = torch.cuda.current_stream()
    lib = nb.load_library()
    if lib.nld_debug_attention_tile(args.attn_tile) != 0:
        raise SystemExit("nld_debug_attention_tile refused the tile")
    points = []
    grid = [(L, B) for L in (1024, 4096, 16384, 32768) for B in (1, 8, 32)]
    if args.attn_point:
        L, B = (int(v) for v in args.attn_point.split(","))
        grid = [(L, B)]
    for L, B in grid:
        pps = (L + m + 63) // 64
        n_pages = B * pps
        g = torch.Generator(device="cuda").manual_seed(2)
        pool = torch.randn((n_pages, 2, Hkv, 64, hd), generator=g, device="cuda").to(torch.bfloat16)
        q = torch.randn((B, m, Hq, hd), generator=g, device="cuda").to(torch.bfloat16)
        perm = torch.randperm(n_pages, generator=g, device="cuda").to(torch.int32).view(B, pps)
        lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
        out = torch.empty_like(q)
        byts = B * (L + m) * Hkv * hd * 2 * 2 + 2 * B * m * Hq * hd * 2
        for mode, bs in (("block", 32), ("causal", 1), ("block_size_1", 1)):
            ms = _events_ms(lambda: nb.nld_attention(q, pool, perm, lens, bs, L + m, out,
                                                     stream.cuda_stream), stream, reps=20)
            gbs = byts / (ms / 1e3) / 1e9
            points.append({"prefix": L, "batch": B, "mode": mode, "us": round(ms * 1e3, 2),
                           "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4),
                           "l2_resident": byts < 126e6})
        del pool, q, perm, out
        torch.cuda.empty_cache()
    big = [p for p in points if not p["l2_resident"]] or points
    best = max(big, key=lambda p: p["GB/s"])
    print(json.dumps({
        "metric": "attention HBM throughput (block-causal GQA over paged bf16 KV)",
        "value": best["GB/s"], "unit": "GB/s", "n_gpus": 1, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"attention micro-workload: 32q/8kv x 128, {m} queries per sequence",
                   "tcgen05_kv_tile": args.attn_tile or "planner",
                   "l2": "not flushed: points under 126 MB are marked l2_resident"},
        "roofline": {"bound": "hbm", "achieved": best["GB/s"], "peak": hbm, "unit": "GB/s",
                     "frac": best["frac"], "traffic": None, "peak_kind": f"{peak_src} HBM copy"},
        "points": points}), flush=True)


def _model_ctx(cfg, seed=0):
    import torch

    import self_speculation_b200 as nb
    import synth
    st = torch.cuda.Stream()
    ctx = nb.Context(cfg, stream=st.cuda_stream)
    w = synth.model_weights(cfg, seed, device="cuda")
    ctx.nld_init_weights(w, on_device=True)
    del w
    torch.cuda.empty_cache()
    return ctx, st


def run_diffusion(args):
    """8B-shaped block diffusion: block 32 of [MASK], confidence threshold 0.9 (at least one commit
    per step), batch 1/4/16, prompt 2048 random ids; steps until 512 tokens per sequence are
    committed: lockstep with the causal KV fill when every block is complete, lockstep with the
    fill fused into the next step, and per-sequence (non-lockstep) steps without host syncs."""
    import torch

    import synth
    from self_speculation_b200 import build as nbuild
    nbuild.build()
    hbm, peak_src = peaks()
    P, N = 2048, 512
    pts = []
    for B in (1, 4, 16):
        cfg = synth.LLAMA8B.replace(max_batch=B, max_seq=P + 3 * N + 256)
        ctx, st = _model_ctx(cfg)
        prompt = synth.prompt_tokens(B, P, cfg.vocab, seed=1).cuda()
        k = cfg.block_k
        blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
        conf = torch.empty(B, k, dtype=torch.float32, device="cuda")
        nc = torch.empty(B, dtype=torch.int32, device="cuda")
        lens = torch.empty(B, dtype=torch.int32, device="cuda")
        step_bytes = cfg.weight_bytes_per_forward() + B * (P + N / 2) * cfg.kv_bytes_per_token()
        point = {"batch": B}
        for fused in (False, True):
            step_fn = ctx.nld_diffuse_block_step_fused if fused else ctx.nld_diffuse_block_step
            # each variant from the same prompt (same prefix lengths), after 3 warm-up steps
            ctx.nld_prefill(prompt)
            for _ in range(3):
                step_fn(0.9, blk, conf, nc)
            ctx.nld_sync()
            torch.cuda.synchronize()
            steps, fills, t0 = 0, 0, time.perf_counter()
            committed = 0
            while committed < N and steps < 4 * N:
                fills += int(step_fn(0.9, blk, conf, nc))
                committed += int(nc.min())
                steps += 1
            ctx.nld_sync()
            dt = time.perf_counter() - t0
            # unfused: a fill forward per block besides the steps; fused: one forward per step up
            # to 256 token rows (batch x 2k), past which the library runs the fill alone
            fwd = steps if (fused and B * 2 * k <= 256) else steps + fills
            point["fused" if fused else "unfused"] = {
                "steps": steps, "forwards": fwd, "s": round(dt, 3),
                "committed_tokens": committed * B, "tokens_per_s": round(committed * B / dt, 2),
                "steps_per_s": round(steps / dt, 2),
                "hbm_frac": round(step_bytes * fwd / dt / 1e9 / hbm, 4)}
        # per-sequence steps, as many forwards as the unfused variant took, no host sync between
        # them; committed tokens = KV rows filled (completed blocks whose fill ran)
        S = point["unfused"]["forwards"]
        state = torch.empty(B, dtype=torch.int32, device="cuda")
        ctx.nld_prefill(prompt)
        for _ in range(3):
            ctx.nld_diffuse_step_nonlockstep(0.9, blk, conf, nc, state)
        ctx.nld_debug_state(lens)
        ctx.nld_sync()
        l1 = lens.clone()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(S):
            ctx.nld_diffuse_step_nonlockstep(0.9, blk, conf, nc, state)
        ctx.nld_sync()
        dt = time.perf_counter() - t0
        ctx.nld_debug_state(lens)
        ctx.nld_sync()
        filled = int((lens - l1).sum().item())
        point["nonlockstep"] = {"steps": S, "forwards": S, "s": round(dt, 3),
                                "filled_tokens": filled, "tokens_per_s": round(filled / dt, 2),
                                "steps_per_s": round(S / dt, 2),
                                "hbm_frac": round(step_bytes * S / dt / 1e9 / hbm, 4)}
        pts.append(point)
        ctx.close()
        del ctx
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    print(json.dumps({
        "metric": "committed tokens/s, 8B-shaped block diffusion (tau 0.9)",
        "value": pts[-1]["fused"]["tokens_per_s"],
        "unit": "tokens/s", "n_gpus": 1, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "8B-shaped diffusion mode, block 32, prompt 2048, 512 tokens per "
                               "variant (unfused KV fill, fused fill, per-sequence steps; each from the same prompt after 3 warm-up steps)",
                   "timing": "host wall clock; lockstep steps synchronise once each by design, "
                             "per-sequence steps do not"},
        "points": pts}), flush=True)


def run_commit_sweep(args):
    """8B-shaped commit-path sweep: after a draft+verify pair, nld_kv_commit with a forced count
    c = 1..k+1 (random weights accept nothing on their own), timed alone with CUDA events on the
    library stream.  The commit moves no KV row (the verify forward wrote rows n..n+k at their
    final slots), so its time should not depend on c."""
    import torch

    import synth
    from self_speculation_b200 import build as nbuild
    nbuild.build()
    reps = 5
    cs = [1, 2, 4, 8, 16, 24, 32, 33]
    cfg = synth.LLAMA8B.replace(max_seq=PROMPT + reps * (sum(cs) + 3 * 33) + 256)
    ctx, stream = _model_ctx(cfg)
    ctx.nld_prefill(synth.prompt_tokens(1, PROMPT, cfg.vocab, seed=1).cuda())
    k = cfg.block_k
    toks = torch.empty(1, k + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    force = torch.empty(1, dtype=torch.int32, device="cuda")
    for _ in range(3):                                   # warm-up: graphs captured
        ctx.nld_selfspec_draft_verify()
        force.fill_(1)
        torch.cuda.synchronize()
        ctx.nld_kv_commit(force, toks, nc)
    ctx.nld_sync()
    points = []
    for c in cs:
        force.fill_(c)
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            ctx.nld_selfspec_draft_verify()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ctx.nld_kv_commit(force, toks, nc)
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
            assert int(nc.item()) == c
        points.append({"c": c, "us_median": round(sorted(ts)[len(ts) // 2], 2),
                       "us_min": round(min(ts), 2)})
    ctx.close()
    print(json.dumps({
        "metric": "commit-path time vs forced commit count, 8B shape, batch 1, k=32",
        "unit": "us", "higher_is_better": False, "n_gpus": 1, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "8B-shaped nld_kv_commit after a draft+verify pair, forced c",
                   "timing": "CUDA events on the library stream around the commit call only"},
        "points": points}), flush=True)


def run_sweep14b(args):
    """14B-shaped concurrency sweep: 40 layers, d 5120, 40/8 heads x 128, FFN 17408, vocab 151936;
    4k-token random prefixes; batch 1/4/16/64; AR step vs self-spec round (k=32) vs diffusion
    step; tokens/s per user and aggregate."""
    import torch

    import synth
    from self_speculation_b200 import build as nbuild
    nbuild.build()
    hbm, peak_src = peaks()
    P = 4096
    reps = max(3, args.steps // 10)
    pts = []
    for B in (1, 4, 16, 64):
        cfg = synth.LLAMA14B.replace(max_batch=B, max_seq=P + 33 * (3 * reps + 12) + 64)
        ctx, st = _model_ctx(cfg)
        ctx.nld_prefill(synth.prompt_tokens(B, P, cfg.vocab, seed=1).cuda())
        k = cfg.block_k
        t1 = torch.empty(B, dtype=torch.int32, device="cuda")
        tk = torch.empty(B, k + 1, dtype=torch.int32, device="cuda")
        nc = torch.empty(B, dtype=torch.int32, device="cuda")
        lens = torch.empty(B, dtype=torch.int32, device="cuda")
        ar_ms = _events_ms(lambda: ctx.nld_ar_step(t1), st, reps)
        ctx.nld_debug_state(lens)
        ctx.nld_sync()
        l0 = int(lens.sum())
        ss_ms = _events_ms(lambda: ctx.nld_selfspec_round(tk, nc, None), st, reps, warm=2)
        ctx.nld_debug_state(lens)
        ctx.nld_sync()
        ss_tok = (int(lens.sum()) - l0) / (reps + 2)
        blk = torch.empty(B, k, dtype=torch.int32, device="cuda")
        cf = torch.empty(B, k, dtype=torch.float32, device="cuda")
        t0 = time.perf_counter()
        dsteps, dtok = 0, 0
        for _ in range(reps):
            ctx.nld_diffuse_block_step(0.9, blk, cf, nc)
            dtok += int(nc.sum())
            dsteps += 1
        d_s = (time.perf_counter() - t0) / dsteps
        wb = cfg.weight_bytes_per_forward()
        kvb = B * P * cfg.kv_bytes_per_token()
        pts.append({
            "batch": B,
            "ar": {"ms": round(ar_ms, 3), "tokens_per_s": round(B / (ar_ms / 1e3), 1),
                   "per_user": round(1 / (ar_ms / 1e3), 1),
                   "hbm_frac": round((wb + kvb) / (ar_ms / 1e3) / 1e9 / hbm, 4)},
            "selfspec": {"ms": round(ss_ms, 3), "tokens_per_s": round(ss_tok / (ss_ms / 1e3), 1),
                         "per_user": round(ss_tok / B / (ss_ms / 1e3), 1),
                         "hbm_frac": round(2 * (wb + kvb) / (ss_ms / 1e3) / 1e9 / hbm, 4)},
            "diffusion": {"ms": round(d_s * 1e3, 3), "tokens_per_s": round(dtok / dsteps / d_s, 1),
                          "per_user": round(dtok / dsteps / B / d_s, 1)}})
        ctx.close()
        del ctx
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    print(json.dumps({
        "metric": "tokens/s per user and aggregate, 14B shape (AR / self-spec / diffusion)",
        "value": pts[-1]["ar"]["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "14B-shaped concurrency sweep, 4k prefixes, batch 1/4/16/64"},
        "points": pts}), flush=True)


def run_probe(args):
    """Small case for ncu captures: a 2-layer model of the 8B layer shape (full vocab), prompt
    512, then each projection GEMM launched alone at M=33 tokens (nld_time_gemm, reps=2) and one
    self-speculation round."""
    import torch

    import self_speculation_b200 as nb
    import synth
    from self_speculation_b200 import build as nbuild
    nbuild.build()
    cfg = synth.LLAMA8B.replace(n_layers=2, max_seq=1024)
    st = torch.cuda.Stream()
    ctx = nb.Context(cfg, stream=st.cuda_stream)
    ctx.nld_init_weights(synth.model_weights(cfg, 0, device="cuda"), on_device=True)
    if args.lora:
        ctx.nld_init_lora(args.lora, 1.0, synth.lora_weights(cfg, args.lora, 0, device="cuda"))
    ctx.nld_prefill(synth.prompt_tokens(1, PROMPT, cfg.vocab, seed=1).cuda())
    toks = torch.empty(1, K_BLOCK + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    ctx.nld_selfspec_round(toks, nc, None)
    ctx.nld_sync()
    out = {}
    plans = {}
    for w, nm in enumerate(["qkv", "o", "gate_up", "down", "lm_head"]):
        out[nm] = ctx.nld_time_gemm(w, 0, K_BLOCK + 1, 2)
        plans[nm] = ctx.nld_debug_gemm_plan(w, K_BLOCK + 1)
    ctx.nld_selfspec_round(toks, nc, None)
    ctx.nld_sync()
    # full decode chain of layer 0 (O, gate/up, down, QKV of layer 1)
    names = ["start", "setup"] + [f"{k}{p}" for p in range(4) for k in ("w0_", "epi_go_", "epi_done_")] \
        + ["mma_last", "exit"]
    tr = torch.zeros(148 * 16 + 256, dtype=torch.int64, device="cuda")
    G = ctx.nld_trace_chain(0, K_BLOCK + 1, tr)
    t = tr[:148 * 16].view(148, 16)[:G].cpu().double()
    t0 = t[:, 0].min()
    traces = {"ctas": G}
    for i, ph in enumerate(names):
        col = t[:, i]
        col = col[col > 0] - t0
        if len(col):
            traces[ph] = [round(float(col.min()) / 1e3, 2), round(float(col.median()) / 1e3, 2),
                          round(float(col.max()) / 1e3, 2)]
    ctx.close()
    torch.cuda.synchronize()
    print(json.dumps({"probe_ms": out}))
    print(json.dumps({"plans": plans}))
    print(json.dumps({"chain_trace_us_min_med_max": traces}))
    # CTA 0's pipeline: per stage iteration issue / MMA start / slot freed, per tile epilogue
    it = tr[148 * 16:148 * 16 + 256].view(4, 64).cpu().double()
    rel = lambda v: [round((float(x) - float(t0)) / 1e3, 2) if x > 0 else None for x in v]
    print(json.dumps({"cta0_pipeline_us": {"issue": rel(it[0]), "mma": rel(it[1]), "freed": rel(it[2]),
                                           "epi_tiles": [rel(it[3][8 * i:8 * i + 8]) for i in range(8)]}}))


def run_layer_trace(args):
    """Timeline of one layer inside a live self-speculation round (8B shape, batch 1, prompt 512,
    the graphs the bench replays): the global timer at each stamp of nld_debug_layer_trace, per
    CTA of that layer's last attention launch in the round (the verify forward's) and of the
    chain launch after it, as min / median / max over CTAs in microseconds after the attention's
    dependency on the previous chain is met (no JSON bench line)."""
    import torch

    import self_speculation_b200 as nb
    import synth
    from self_speculation_b200 import build as nbuild
    nbuild.build()
    cfg = synth.LLAMA8B.replace(max_seq=2048)
    st = torch.cuda.Stream()
    ctx = nb.Context(cfg, stream=st.cuda_stream)
    ctx.nld_init_weights(synth.model_weights(cfg, 0, device="cuda"), on_device=True)
    torch.cuda.empty_cache()
    ctx.nld_prefill(synth.prompt_tokens(1, PROMPT, cfg.vocab, seed=1).cuda())
    toks = torch.empty(1, K_BLOCK + 1, dtype=torch.int32, device="cuda")
    nc = torch.empty(1, dtype=torch.int32, device="cuda")
    for _ in range(args.warmup):
        ctx.nld_selfspec_round(toks, nc, None)
    ctx.nld_sync()
    at = torch.zeros(4096 * 16, dtype=torch.int64, device="cuda")
    ch = torch.zeros(148 * 16 + 256, dtype=torch.int64, device="cuda")
    ctx.nld_debug_layer_trace(args.layer_trace, at, ch)
    ctx.nld_selfspec_round(toks, nc, None)
    ctx.nld_sync()
    ctx.nld_debug_layer_trace(-1)
    a = at.view(-1, 16).cpu().double()
    # the draft forward's launch of the layer wrote first: keep the CTAs that entered with the
    # round's last launch, and per stamp the values it wrote
    a = a[a[:, 0] > a[:, 0].max() - 100e3]
    t0 = a[:, 1][a[:, 1] > 0].min()

    def stats(col):
        col = col[col > t0 - 100e3]
        if len(col) == 0:
            return None
        v = (col - t0) / 1e3
        return [round(float(v.min()), 2), round(float(v.median()), 2), round(float(v.max()), 2)]
    attn_names = {0: "entry", 1: "dependency_met", 2: "query_staged", 3: "kv_tile0", 4: "kv_tile1",
                  12: "last_pv_done", 13: "partial_written", 10: "cluster_published",
                  14: "first_row_merged", 11: "output_written"}
    c = ch[:148 * 16].view(148, 16).cpu().double()
    c = c[c[:, 0] > 0]
    chain_names = ["start", "setup"] + [f"{k}{p}" for p in ("O", "GU", "D", "QKV")
                                        for k in ("w0_", "epi_go_", "epi_done_")] + ["mma_last", "exit"]
    print(json.dumps({
        "layer": args.layer_trace, "attention_ctas": int(a.shape[0]), "chain_ctas": int(c.shape[0]),
        "attention_us_min_med_max": {nm: stats(a[:, i]) for i, nm in attn_names.items()},
        "chain_us_min_med_max": {nm: stats(c[:, i]) for i, nm in enumerate(chain_names)}}), flush=True)
    ctx.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-layers", type=int, default=36,
                    help="layers of the reference arm's model (36 = the 8B shape; fewer only to "
                         "exercise the arm's output quickly)")
    ap.add_argument("--no-generation", action="store_true",
                    help="skip the 1024-token generation measured after the timed rounds")
    ap.add_argument("--lora", type=int, default=0,
                    help="rank of a seeded random o_proj adapter in the draft forwards (0: none)")
    ap.add_argument("--workload", choices=["selfspec8b", "attention", "diffusion8b", "sweep14b",
                                           "commit8b"],
                    default="selfspec8b")
    ap.add_argument("--attn-m", type=int, default=32,
                    help="queries per sequence of the attention workload (32; 1 = single-token decode)")
    ap.add_argument("--attn-point", default="",
                    help="attention workload: one point 'prefix,batch' instead of the whole grid")
    ap.add_argument("--attn-tile", type=int, default=0, choices=[0, 64, 128],
                    help="attention workload: keys per tcgen05 KV tile (0 = the planner's choice, 64, 128)")
    ap.add_argument("--probe", action="store_true",
                    help="small kernel-probe case for profiler captures (no JSON bench line)")
    ap.add_argument("--layer-trace", type=int, default=-1,
                    help="timeline of this layer's verify attention and the chain after it in a "
                         "live round (no JSON bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.probe:
        run_probe(args)
    elif args.layer_trace >= 0:
        run_layer_trace(args)
    elif args.workload == "attention":
        run_attention(args)
    elif args.workload == "diffusion8b":
        run_diffusion(args)
    elif args.workload == "sweep14b":
        run_sweep14b(args)
    elif args.workload == "commit8b":
        run_commit_sweep(args)
    elif args.impl == "reference":
        run_reference(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
