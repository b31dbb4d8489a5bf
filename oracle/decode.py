"""Oracle decoding procedures: AR steps, self-speculation rounds, block-diffusion steps.

Test infrastructure only (see the package docstring).  Written from:
* ranhao.site notes section 5.1 (AR: left-to-right p(x_i | x_<i)), 5.2 (a block starts as
  [MASK] tokens and is denoised over several forwards, committing high-confidence positions),
  5.3 (the diffusion pathway drafts k tokens in parallel, the AR pathway verifies, the
  longest correct prefix is accepted and acceptance stops at the first mismatch);
* r9-hu digest "Method", tri-mode inference (k drafts from one forward, a causal second
  forward verifies them, 1 to k+1 tokens per round);
* shilu.ai "Deploy and infer with SGLang" (32-token blocks; a confidence threshold decides
  which tokens are committed each step; self-speculation is lossless against AR at
  temperature 0).

Readings where the pages are silent (each is listed with its reason in the design notes):
* State between rounds: KV rows 0..n-1 are cached; the last committed token x_n is
  "pending" (committed, no KV row yet) and sits at position n.
* Shifted prediction in every mode: the output row at position i scores the token at i+1.
  A draft block is [x_n, MASK x (k-1)] at positions n..n+k-1 and its k rows give the k
  drafts d_1..d_k; with k == 1 the draft forward is exactly the AR step.
* Verify input is [x_n, d_1..d_k] (k+1 rows, causal) giving v_1..v_{k+1}; a = the number of
  leading i with d_i == v_i; the round commits v_1..v_{a+1}, KV rows n..n+a come from the
  verify forward, pending becomes v_{a+1}.
* Argmax ties resolve to the lowest token id; confidence is the largest softmax probability
  over the V real tokens; a diffusion step commits every still-masked slot whose confidence
  is >= tau, or else the single most confident one (lowest slot on ties).  A complete
  block gets one causal forward over [x_n, b_1..b_{k-1}] that writes its KV rows; b_k
  becomes the pending token.  With several sequences, a sequence whose block is complete
  waits (its rows are computed and ignored) until every block is complete.
* LoRA drafter (optional, OracleModel.set_lora): the low-rank o_proj delta applies to the
  block-bidirectional forwards (draft, diffusion denoising) only; causal forwards (verify, AR,
  prefill, KV fill) use the frozen weights, so committed KV rows never contain it.
* Fused fill (the deferred form of the KV fill): the causal forward over the complete block
  and the first denoising forward of the next block run as one forward of 2k rows,
  [x_n, b_1..b_{k-1}, b_k, MASK x (k-1)] at positions n..n+2k-1, whose first k rows are
  causal and whose last k rows are one bidirectional block that sees the first k.  In exact
  arithmetic its KV rows n..n+k-1 and its last k logit rows equal those of the fill followed
  by the plain denoising forward.
* Quadratic self-speculation (named by the pages, not defined there): one forward per round
  holds the causal verify rows of the current drafts and, for each possible acceptance
  length a = 0..k, a pre-draft block of the next round (k mask rows at n+a+1..n+a+k that see
  the prefix, the verify rows of x_n, d_1..d_a and each other).  The round commits as the
  linear round does; the next drafts come from the block of the outcome that happened.
  (k+1)^2 rows per forward: quadratic in k.  See quadratic_layout.
* Per-sequence (non-lockstep) diffusion: a sequence whose block completed runs its causal KV
  fill in its next step while the other sequences of the batch keep denoising; each step is
  one forward of k rows per sequence.  Sequences never see one another, so every sequence's
  tokens equal those it would generate alone.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import torch


def argmax_lowest(logits: torch.Tensor) -> torch.Tensor:
    """Index of the largest logit along the last axis, the lowest index among equal maxima."""
    mx = logits.max(dim=-1, keepdim=True).values
    idx = torch.arange(logits.shape[-1]).expand_as(logits)
    big = torch.full_like(idx, logits.shape[-1])
    return torch.where(logits == mx, idx, big).min(dim=-1).values


def confidence(logits: torch.Tensor) -> torch.Tensor:
    """Largest softmax probability along the last axis: 1 / sum_v exp(l_v - max l)."""
    mx = logits.max(dim=-1, keepdim=True).values
    return 1.0 / torch.exp(logits - mx).sum(dim=-1)


def accept_length(draft: List[int], verify: List[int]) -> int:
    """Greedy longest matching prefix: the number of leading positions i (0-based, i < k)
    with draft[i] == verify[i]; stops at the first mismatch."""
    a = 0
    for d, v in zip(draft, verify):
        if d != v:
            break
        a += 1
    return a


def commit_after_verify(draft: List[int], verify: List[int],
                        forced: Optional[int] = None) -> List[int]:
    """Tokens a round commits: v_1..v_{a+1} (== d_1..d_a, v_{a+1}).  With a forced count c
    (1..k+1) the round commits d_1..d_{c-1}, v_c instead: the tokens the verify forward's
    first c KV rows belong to, closed by that forward's prediction."""
    k = len(draft)
    assert len(verify) == k + 1
    if forced is None:
        a = accept_length(draft, verify)
        return list(verify[:a + 1])
    assert 1 <= forced <= k + 1
    return list(draft[:forced - 1]) + [verify[forced - 1]]


def diffusion_commit(masked: List[bool], conf: List[float], tau: float) -> List[bool]:
    """Slots committed by one confidence-threshold step: every masked slot with conf >= tau;
    if none qualifies, the masked slot of highest confidence (lowest slot on ties)."""
    pick = [mk and (cf >= tau) for mk, cf in zip(masked, conf)]
    if any(pick) or not any(masked):
        return pick
    best = None
    for i, (mk, cf) in enumerate(zip(masked, conf)):
        if mk and (best is None or cf > conf[best]):
            best = i
    pick[best] = True
    return pick


@dataclasses.dataclass
class SeqState:
    cache: list               # OracleModel cache
    lens: List[int]           # cached KV rows per sequence
    pending: List[int]        # committed token without a KV row, at position lens[b]
    block: Optional[List[List[int]]] = None   # diffusion block b_1..b_k (mask id = open)


def prefill(model, prompt: torch.Tensor, capacity: int) -> SeqState:
    """Causal forward over prompt[:, :P-1] writing KV rows 0..P-2; pending = prompt[:, P-1]."""
    B, P = prompt.shape
    cache = model.new_cache(B, capacity)
    if P > 1:
        model.forward(prompt[:, :P - 1], [0] * B, cache, block_size=1, write_kv=True,
                      with_logits=False)
    return SeqState(cache=cache, lens=[P - 1] * B, pending=[int(t) for t in prompt[:, P - 1]])


def ar_forward(model, st: SeqState) -> torch.Tensor:
    """Logits [B, 1, V] of the causal one-token forward over the pending tokens (writes KV)."""
    toks = torch.tensor(st.pending, dtype=torch.int64)[:, None]
    return model.forward(toks, st.lens, st.cache, block_size=1, write_kv=True)


def ar_step(model, st: SeqState) -> List[int]:
    logits = ar_forward(model, st)
    nxt = argmax_lowest(logits[:, 0]).tolist()
    for b in range(len(st.lens)):
        st.lens[b] += 1
        st.pending[b] = nxt[b]
    return nxt


def draft_forward(model, st: SeqState, k: int) -> torch.Tensor:
    """Logits [B, k, V] of the diffusion draft forward over [x_n, MASK x (k-1)], one
    bidirectional block over the cached prefix.  Draft KV rows are not kept."""
    B = len(st.lens)
    toks = torch.full((B, k), model.cfg.mask_id, dtype=torch.int64)
    toks[:, 0] = torch.tensor(st.pending)
    return model.forward(toks, st.lens, st.cache, block_size=k, write_kv=False, lora=True)


def verify_forward(model, st: SeqState, drafts: List[List[int]]) -> torch.Tensor:
    """Logits [B, k+1, V] of the causal forward over [x_n, d_1..d_k]; writes KV rows
    n..n+k (only the accepted ones become part of the cache, by the length update)."""
    toks = torch.tensor([[st.pending[b]] + list(drafts[b]) for b in range(len(st.lens))],
                        dtype=torch.int64)
    return model.forward(toks, st.lens, st.cache, block_size=1, write_kv=True)


def apply_commit(st: SeqState, committed: List[List[int]]) -> None:
    for b, toks in enumerate(committed):
        st.lens[b] += len(toks)
        st.pending[b] = toks[-1]


def selfspec_round(model, st: SeqState, k: int, forced: Optional[List[int]] = None):
    """One linear self-speculation round.  Returns (committed token lists, drafts, verify
    argmaxes, draft logits, verify logits)."""
    dl = draft_forward(model, st, k)
    drafts = argmax_lowest(dl).tolist()
    vl = verify_forward(model, st, drafts)
    ver = argmax_lowest(vl).tolist()
    committed = [commit_after_verify(drafts[b], ver[b], None if forced is None else forced[b])
                 for b in range(len(st.lens))]
    apply_commit(st, committed)
    return committed, drafts, ver, dl, vl


def quadratic_layout(n: int, k: int):
    """Rows, positions and mask of the quadratic self-speculation forward at cached length n.

    Rows 0..k are the verify rows V_i (inputs x_n, d_1..d_k at positions n..n+k, causal).
    Then, for every acceptance outcome a = 0..k, a pre-draft block P_a of k rows: the mask id
    at positions n+a+1 .. n+a+k.  P_a stands for the next round's draft block
    [v_{a+1}, MASK x (k-1)] with v_{a+1} not yet known (it is being computed by V_a in the
    same forward), so its first slot is a mask too.  P_a sees the cached prefix, the verify
    rows V_0..V_a (the tokens x_n, d_1..d_a that outcome a keeps) and all of its own rows;
    nothing else.  Returns (m, positions [m], mask [m, n+m])."""
    m = (k + 1) + (k + 1) * k
    pos = torch.empty(m, dtype=torch.int64)
    mask = torch.zeros(m, n + m, dtype=torch.bool)
    mask[:, :n] = True
    for i in range(k + 1):
        pos[i] = n + i
        mask[i, n:n + i + 1] = True
    for a in range(k + 1):
        r0 = (k + 1) + a * k
        pos[r0:r0 + k] = torch.arange(n + a + 1, n + a + 1 + k)
        mask[r0:r0 + k, n:n + a + 1] = True
        mask[r0:r0 + k, n + r0:n + r0 + k] = True
    return m, pos, mask


def quadratic_forward(model, st: SeqState, drafts: List[List[int]]):
    """One forward of quadratic self-speculation: the verify rows of the current drafts and
    the k+1 pre-draft blocks of the next round.  Writes the verify rows' KV at n..n+k (the
    pre-draft rows' K/V are not kept); the LoRA drafter, if any, applies to the pre-draft
    rows only.  Returns (verify logits [B, k+1, V], pre-draft logits [B, k+1, k, V])."""
    B = len(st.lens)
    k = len(drafts[0])
    mask_id = model.cfg.mask_id
    m = (k + 1) * (k + 1)
    toks = torch.tensor([[st.pending[b]] + list(drafts[b]) + [mask_id] * ((k + 1) * k)
                         for b in range(B)], dtype=torch.int64)
    positions, masks = [], []
    for b in range(B):
        _, pos, mask = quadratic_layout(st.lens[b], k)
        positions.append(pos)
        masks.append(mask)
    lora_rows = torch.zeros(B, m, dtype=torch.bool)
    lora_rows[:, k + 1:] = True
    logits = model.forward_rows(toks, torch.stack(positions), st.lens, st.cache, masks,
                                write_kv_rows=k + 1, lora_rows=lora_rows)
    V = logits.shape[-1]
    return logits[:, :k + 1], logits[:, k + 1:].reshape(B, k + 1, k, V)


def quadratic_round(model, st: SeqState, drafts: List[List[int]]):
    """One quadratic round: verify the drafts and commit as in the linear round (greedy
    longest matching prefix, 1..k+1 tokens); the next round's drafts are the argmaxes of the
    pre-draft block of the outcome that happened.  Returns (committed, next drafts)."""
    vl, pl = quadratic_forward(model, st, drafts)
    ver = argmax_lowest(vl).tolist()
    committed, nxt = [], []
    for b in range(len(st.lens)):
        c = commit_after_verify(drafts[b], ver[b])
        committed.append(c)
        nxt.append(argmax_lowest(pl[b, len(c) - 1]).tolist())
    apply_commit(st, committed)
    return committed, nxt


def diffusion_forward(model, st: SeqState, k: int) -> torch.Tensor:
    """Logits [B, k, V] of one denoising forward over [x_n, b_1..b_{k-1}] (open slots hold
    the mask id), one bidirectional block; row i scores slot b_{i+1}."""
    toks = torch.tensor([[st.pending[b]] + st.block[b][:k - 1] for b in range(len(st.lens))],
                        dtype=torch.int64)
    return model.forward(toks, st.lens, st.cache, block_size=k, write_kv=False, lora=True)


def diffusion_step(model, st: SeqState, k: int, tau: float):
    """One denoising step for every sequence (lockstep).  Returns a dict with
    newly: per sequence the (slot, token) pairs committed this step,
    conf [B,k], argmax [B,k] (row i scores slot i, i.e. b_{i+1}),
    filled: whether the blocks completed and got their causal KV-fill forward,
    blocks: the completed blocks (b_1..b_k per sequence) when filled, else None."""
    mask_id = model.cfg.mask_id
    B = len(st.lens)
    if st.block is None:
        st.block = [[mask_id] * k for _ in range(B)]
    logits = diffusion_forward(model, st, k)
    conf = confidence(logits)
    am = argmax_lowest(logits)
    newly = []
    for b in range(B):
        masked = [t == mask_id for t in st.block[b]]
        pick = diffusion_commit(masked, conf[b].tolist(), tau)
        got = []
        for s in range(k):
            if pick[s]:
                st.block[b][s] = int(am[b, s])
                got.append((s, int(am[b, s])))
        newly.append(got)
    filled = all(mask_id not in st.block[b] for b in range(B))
    blocks = None
    if filled:
        blocks = [list(st.block[b]) for b in range(B)]
        toks = torch.tensor([[st.pending[b]] + st.block[b][:k - 1] for b in range(B)],
                            dtype=torch.int64)
        model.forward(toks, st.lens, st.cache, block_size=1, write_kv=True, with_logits=False)
        for b in range(B):
            st.lens[b] += k
            st.pending[b] = st.block[b][k - 1]
        st.block = [[mask_id] * k for _ in range(B)]
    return dict(newly=newly, conf=conf, argmax=am, filled=filled, blocks=blocks,
                logits=logits)


def fill_diffusion_forward(model, st: SeqState, k: int) -> torch.Tensor:
    """The fused fill: st.block is complete.  One forward over
    [x_n, b_1..b_{k-1}, b_k, MASK x (k-1)] (first k rows causal, last k rows one block) writes
    the complete block's KV rows; then lens += k, pending = b_k, a fresh block of masks.
    A LoRA drafter applies to the last k (block) rows only.  Returns the logits [B, k, V] of the last k rows (the new block's first denoising step)."""
    mask_id = model.cfg.mask_id
    B = len(st.lens)
    toks = torch.tensor([[st.pending[b]] + st.block[b] + [mask_id] * (k - 1) for b in range(B)],
                        dtype=torch.int64)
    logits = model.forward(toks, st.lens, st.cache, block_size=k, write_kv=True,
                           causal_rows=k, lora=True)
    for b in range(B):
        st.lens[b] += k
        st.pending[b] = st.block[b][k - 1]
    st.block = [[mask_id] * k for _ in range(B)]
    return logits[:, k:]


def diffusion_step_fused(model, st: SeqState, k: int, tau: float, fill_pending: bool):
    """One denoising step with the deferred fill: when fill_pending (the previous step
    completed the block), the fill and this step are the one fused forward; a block completed
    by this step is not filled now (returned fill_pending = True).  Same commit rule as
    diffusion_step.  Returns (dict as diffusion_step without the fill, fill_pending)."""
    mask_id = model.cfg.mask_id
    B = len(st.lens)
    if st.block is None:
        st.block = [[mask_id] * k for _ in range(B)]
    logits = fill_diffusion_forward(model, st, k) if fill_pending else diffusion_forward(model, st, k)
    conf = confidence(logits)
    am = argmax_lowest(logits)
    newly = []
    for b in range(B):
        masked = [t == mask_id for t in st.block[b]]
        pick = diffusion_commit(masked, conf[b].tolist(), tau)
        got = []
        for s in range(k):
            if pick[s]:
                st.block[b][s] = int(am[b, s])
                got.append((s, int(am[b, s])))
        newly.append(got)
    complete = all(mask_id not in st.block[b] for b in range(B))
    blocks = [list(st.block[b]) for b in range(B)] if complete else None
    return dict(newly=newly, conf=conf, argmax=am, complete=complete, blocks=blocks,
                logits=logits), complete


def _one(st: SeqState, b: int) -> SeqState:
    """Sequence b of st as a batch of one: its cache and block lists are shared with st, its
    length and pending token copied."""
    return SeqState(cache=[st.cache[b]], lens=[st.lens[b]], pending=[st.pending[b]],
                    block=None if st.block is None else [st.block[b]])


def _fill_one(model, st: SeqState, b: int, k: int) -> None:
    """Causal KV fill of sequence b's complete block: len += k, pending = b_k, fresh masks."""
    one = _one(st, b)
    toks = torch.tensor([[one.pending[0]] + one.block[0][:k - 1]], dtype=torch.int64)
    model.forward(toks, one.lens, one.cache, block_size=1, write_kv=True, with_logits=False)
    st.lens[b] += k
    st.pending[b] = st.block[b][k - 1]
    st.block[b] = [model.cfg.mask_id] * k


def flush_fills(model, st: SeqState, k: int, fill_next: List[bool]) -> None:
    """Run the fills that per-sequence diffusion left due (before another decode mode)."""
    for b in range(len(st.lens)):
        if fill_next[b]:
            _fill_one(model, st, b, k)


def diffusion_step_nonlockstep(model, st: SeqState, k: int, tau: float, fill_next: List[bool]):
    """One step of per-sequence (non-lockstep) diffusion: every sequence takes k rows of one
    forward.  A sequence whose block completed in an earlier step (fill_next[b]) runs its
    causal KV fill over [x_n, b_1..b_{k-1}] (then len += k, pending = b_k, a fresh block of
    masks); every other sequence takes one denoising step with the commit rule of
    diffusion_step.  No sequence waits for the others.  Sequences are independent, so each is
    computed as a batch of one.  Returns (newly [B] (slot, token) lists, state [B]: 0 block
    still open, 1 block completed by this step, 2 filled in this step; blocks [B]: the
    completed block where state is 1, else None; the new fill_next)."""
    mask_id = model.cfg.mask_id
    B = len(st.lens)
    if st.block is None:
        st.block = [[mask_id] * k for _ in range(B)]
    newly, state, blocks, nxt = [], [], [], []
    for b in range(B):
        one = _one(st, b)
        if fill_next[b]:
            _fill_one(model, st, b, k)
            newly.append([])
            state.append(2)
            blocks.append(None)
            nxt.append(False)
            continue
        logits = diffusion_forward(model, one, k)
        conf = confidence(logits)[0]
        am = argmax_lowest(logits)[0]
        masked = [t == mask_id for t in st.block[b]]
        pick = diffusion_commit(masked, conf.tolist(), tau)
        got = []
        for slot in range(k):
            if pick[slot]:
                st.block[b][slot] = int(am[slot])
                got.append((slot, int(am[slot])))
        newly.append(got)
        done = mask_id not in st.block[b]
        state.append(1 if done else 0)
        blocks.append(list(st.block[b]) if done else None)
        nxt.append(done)
    return newly, state, blocks, nxt


def diffuse_generate_nonlockstep(model, prompt: torch.Tensor, n_tokens: int, k: int, tau: float,
                                 capacity: int) -> Tuple[List[List[int]], int, List[List[int]]]:
    """Per-sequence diffusion until every sequence has n_tokens.  Returns (tokens per sequence
    in position order, number of forwards (= steps: one batched forward each), the per-step
    state lists)."""
    st = prefill(model, prompt, capacity)
    B = prompt.shape[0]
    out = [[] for _ in range(B)]
    fill_next = [False] * B
    states = []
    while min(len(o) for o in out) < n_tokens:
        _, state, blocks, fill_next = diffusion_step_nonlockstep(model, st, k, tau, fill_next)
        states.append(state)
        for b in range(B):
            if state[b] == 1:
                out[b].extend(blocks[b])
    return [o[:n_tokens] for o in out], len(states), states


# ---- generation drivers (exactly N generated tokens; the last round is truncated) ----------

def ar_generate(model, prompt: torch.Tensor, n_tokens: int, capacity: int) -> List[List[int]]:
    st = prefill(model, prompt, capacity)
    out = [[] for _ in range(prompt.shape[0])]
    while len(out[0]) < n_tokens:
        nxt = ar_step(model, st)
        for b, t in enumerate(nxt):
            out[b].append(t)
    return out


def selfspec_generate(model, prompt: torch.Tensor, n_tokens: int, k: int, capacity: int
                      ) -> Tuple[List[List[int]], List[List[int]]]:
    """Returns (tokens per sequence, commits per round per sequence)."""
    st = prefill(model, prompt, capacity)
    B = prompt.shape[0]
    out = [[] for _ in range(B)]
    per_round = [[] for _ in range(B)]
    while min(len(o) for o in out) < n_tokens:
        committed, *_ = selfspec_round(model, st, k)
        for b in range(B):
            out[b].extend(committed[b])
            per_round[b].append(len(committed[b]))
    return [o[:n_tokens] for o in out], per_round


def quadratic_generate(model, prompt: torch.Tensor, n_tokens: int, k: int, capacity: int
                       ) -> Tuple[List[List[int]], int, List[List[int]]]:
    """Quadratic self-speculation: one diffusion draft forward to start, then one forward per
    round.  Returns (tokens per sequence, forwards, commits per round per sequence)."""
    st = prefill(model, prompt, capacity)
    B = prompt.shape[0]
    drafts = argmax_lowest(draft_forward(model, st, k)).tolist()
    forwards = 1
    out = [[] for _ in range(B)]
    per_round = [[] for _ in range(B)]
    while min(len(o) for o in out) < n_tokens:
        committed, drafts = quadratic_round(model, st, drafts)
        forwards += 1
        for b in range(B):
            out[b].extend(committed[b])
            per_round[b].append(len(committed[b]))
    return [o[:n_tokens] for o in out], forwards, per_round


def diffuse_generate_fused(model, prompt: torch.Tensor, n_tokens: int, k: int, tau: float,
                           capacity: int) -> Tuple[List[List[int]], int, int]:
    """diffuse_generate with the deferred, fused fill.  Returns (tokens per sequence in
    position order, number of forwards, number of denoising steps); a fill still pending at
    the end is not run (its tokens are committed)."""
    st = prefill(model, prompt, capacity)
    B = prompt.shape[0]
    out = [[] for _ in range(B)]
    steps = forwards = 0
    pending = False
    while min(len(o) for o in out) < n_tokens:
        r, pending = diffusion_step_fused(model, st, k, tau, pending)
        steps += 1
        forwards += 1
        if r["complete"]:
            for b in range(B):
                out[b].extend(r["blocks"][b])
    return [o[:n_tokens] for o in out], forwards, steps


def diffuse_generate(model, prompt: torch.Tensor, n_tokens: int, k: int, tau: float,
                     capacity: int) -> Tuple[List[List[int]], int]:
    """Returns (tokens per sequence in position order, number of denoising steps)."""
    st = prefill(model, prompt, capacity)
    B = prompt.shape[0]
    out = [[] for _ in range(B)]
    steps = 0
    while min(len(o) for o in out) < n_tokens:
        r = diffusion_step(model, st, k, tau)
        steps += 1
        if r["filled"]:
            for b in range(B):
                out[b].extend(r["blocks"][b])
    return [o[:n_tokens] for o in out], steps
