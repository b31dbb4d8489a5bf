"""Oracle decoder forward: a plain Llama-style transformer with explicit attention masks.

Test infrastructure only (see the package docstring).  Everything here is the textbook
definition written out with whole-tensor torch CPU ops (a matmul is the only library
primitive used as a step); nothing is blocked, fused or reordered.

Model (Llama-style decoder named for the workloads; weights from `synth`):
  h0 = E[t]
  per layer:  a = rmsnorm(h) * g1
              q, k, v = a Wq^T, a Wk^T, a Wv^T ; RoPE on q and k at the absolute position
              query head j reads kv head floor(j / (Hq/Hkv))
              o = softmax(q k^T / sqrt(hd) + mask) v ;  h += o Wo^T
              m = rmsnorm(h) * g2 ;  h += (silu(m Wg^T) * (m Wu^T)) Wd^T
  logits = (rmsnorm(h) * gf) Wlm^T                          over the V real tokens
  rmsnorm(x) = x / sqrt(mean(x^2) + eps)

Attention mask (ranhao.site notes section 3.2 and r9-hu digest "Method": bidirectional
inside a block, causal across blocks, the clean prefix reused as KV; section 4.3: the clean
stream is strictly causal).  A forward covers positions n..n+m-1 of one sequence, cut into
blocks of `block_size` starting at n.  A query sees every cached prefix key (j < n) and
every key of the forward whose block index is not above its own.  block_size == 1 is the
strictly causal mask.

Precision modes
  "f64"    float64 everywhere (the reference semantics).
  "f32"    float32 everywhere.
  "f32kv"  float32 everywhere, with a bf16 KV cache: the key and value rows are stored in a
           bfloat16 cache and every attention reads them back from it (a forward's own rows
           included).  Together with weights given as bf16 values this is the bf16
           configuration as specified (bf16 weights and KV cache, fp32 accumulation and fp32
           activations); the bf16 parity tests state their tolerances against it.
"""
from __future__ import annotations

import math
from typing import List, Optional

import torch

F32 = 0
BF16 = 1


def rmsnorm(x: torch.Tensor, eps: float) -> torch.Tensor:
    """x / sqrt(mean(x^2) + eps) over the last axis (no gain)."""
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps)


def rope_rotate(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotary embedding, rotate-half pairing: element i is paired with i + hd/2 and the pair
    is rotated by angle pos * theta^(-2i/hd).  x: [..., hd]; pos broadcasts against x[..., 0]."""
    hd = x.shape[-1]
    half = hd // 2
    i = torch.arange(half, dtype=torch.float64)
    inv_freq = theta ** (-2.0 * i / hd)                      # [half]
    ang = pos.to(torch.float64)[..., None] * inv_freq        # [..., half]
    c = torch.cos(ang).to(x.dtype)
    s = torch.sin(ang).to(x.dtype)
    x1 = x[..., :half]
    x2 = x[..., half:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def causal_mask(m: int, n: int) -> torch.Tensor:
    """[m, n+m] bool: query r (position n+r) sees key j iff j <= n+r."""
    j = torch.arange(n + m)[None, :]
    r = torch.arange(m)[:, None]
    return j <= n + r


def block_mask(m: int, n: int, block_size: int, causal_rows: int = 0) -> torch.Tensor:
    """[m, n+m] bool: prefix keys (j < n) always visible; keys of the forward are visible
    when their block index (j-n)//block_size is not above the query's r//block_size.

    causal_rows = c > 0 (the fused diffusion KV fill): the first c rows of the forward are
    strictly causal (a complete block being written into the clean prefix), and the blocks
    of block_size start after them: row r >= c sees the prefix, all c causal rows, and the
    keys of its own and earlier blocks counted from c."""
    j = torch.arange(n + m)[None, :]
    r = torch.arange(m)[:, None]
    in_prefix = j < n
    if causal_rows == 0:
        key_blk = torch.div(j - n, block_size, rounding_mode="floor")
        q_blk = torch.div(r, block_size, rounding_mode="floor")
        return in_prefix | ((j >= n) & (key_blk <= q_blk))
    c = causal_rows
    causal_part = (r < c) & (j <= n + r)
    in_fill = (j >= n) & (j < n + c)
    key_blk = torch.div(j - n - c, block_size, rounding_mode="floor")
    q_blk = torch.div(r - c, block_size, rounding_mode="floor")
    block_part = (r >= c) & (in_fill | ((j >= n + c) & (key_blk <= q_blk)))
    return (in_prefix & (r >= 0)) | causal_part | block_part


def attention_explicit(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       mask: torch.Tensor) -> torch.Tensor:
    """Masked softmax attention written out: q [Hq, m, hd], k/v [Hkv, L, hd], mask [m, L].
    Query head j uses kv head j // (Hq/Hkv).  Masked scores are -inf."""
    Hq, m, hd = q.shape
    Hkv = k.shape[0]
    group = Hq // Hkv
    kv_idx = torch.arange(Hq) // group
    kk = k[kv_idx]                                            # [Hq, L, hd]
    vv = v[kv_idx]
    s = torch.matmul(q, kk.transpose(1, 2)) / math.sqrt(hd)  # [Hq, m, L]
    s = s.masked_fill(~mask[None, :, :], float("-inf"))
    p = torch.softmax(s, dim=-1)
    return torch.matmul(p, vv)


class OracleModel:
    """Holds the weights (as given, bf16 or fp32 CPU tensors in the boundary's order) and
    runs forwards with an explicit KV cache [B][layer] -> (K [Hkv, cap, hd], V ...)."""

    def __init__(self, cfg, weights: List[Optional[torch.Tensor]], precision: str = "f64"):
        assert precision in ("f64", "f32", "f32kv")
        self.cfg = cfg
        self.precision = precision
        self.cdt = torch.float64 if precision == "f64" else torch.float32
        w = [None if t is None else t.detach().cpu() for t in weights]
        self.embed = w[0]
        self.layers = []
        for l in range(cfg.n_layers):
            b = 1 + 9 * l
            self.layers.append(dict(g1=w[b], wq=w[b + 1], wk=w[b + 2], wv=w[b + 3], wo=w[b + 4],
                                    g2=w[b + 5], wg=w[b + 6], wu=w[b + 7], wd=w[b + 8]))
        self.gf = w[1 + 9 * cfg.n_layers]
        self.lm = w[2 + 9 * cfg.n_layers]
        self.lora = None

    def set_lora(self, A: List[torch.Tensor], B: List[torch.Tensor], scale: float) -> None:
        """Low-rank delta on o_proj for the diffusion drafter (ranhao.site notes section 6:
        LoRA of rank 128 on o_proj, trained for the diffusion pathway while the AR verifier
        stays frozen): per layer A [r, Hq*hd], B [d, r]; a block-bidirectional forward adds
        scale * B (A att) to the residual next to o_proj's output."""
        self.lora = (list(A), list(B), float(scale))

    # -- helpers ------------------------------------------------------------------------
    def _w(self, t: torch.Tensor) -> torch.Tensor:
        return t.to(self.cdt)

    def _mm(self, x: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
        return torch.matmul(x, self._w(w).t())

    def _normed_mm(self, h: torch.Tensor, g: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
        """(rmsnorm(h) * g) W^T."""
        return self._mm(rmsnorm(h, self.cfg.rms_eps) * self._w(g), w)

    @property
    def kv_dtype(self):
        """Element type of the KV cache: bfloat16 in "f32kv", else the compute type."""
        return torch.bfloat16 if self.precision == "f32kv" else self.cdt

    def _kv(self, x: torch.Tensor) -> torch.Tensor:
        """A key or value row as the cache holds it (stored in kv_dtype, read back)."""
        return x.to(self.kv_dtype).to(self.cdt)

    def new_cache(self, batch: int, capacity: int):
        c = self.cfg
        return [[(torch.zeros(c.n_kv_heads, capacity, c.head_dim, dtype=self.kv_dtype),
                  torch.zeros(c.n_kv_heads, capacity, c.head_dim, dtype=self.kv_dtype))
                 for _ in range(c.n_layers)] for _ in range(batch)]

    # -- forward ------------------------------------------------------------------------
    def forward(self, tokens: torch.Tensor, starts: List[int], cache, block_size: int,
                write_kv: bool, layers: Optional[List[int]] = None,
                with_logits: bool = True, causal_rows: int = 0,
                lora: bool = False) -> Optional[torch.Tensor]:
        """tokens [B, m] at positions starts[b]..starts[b]+m-1 over cached rows
        [0, starts[b]).  block_size 1 = causal; block_size m = one bidirectional block.
        write_kv stores this forward's K/V rows into the cache at their positions.
        lora: the adapter (if set) applies to the rows that attend block-bidirectionally,
        i.e. all rows but the leading causal_rows.
        Returns logits [B, m, V] (compute dtype) or None."""
        B, m = tokens.shape
        positions = torch.stack([torch.arange(int(starts[b]), int(starts[b]) + m) for b in range(B)])
        masks = [block_mask(m, int(starts[b]), block_size, causal_rows) for b in range(B)]
        lora_rows = None
        if lora:
            lora_rows = torch.zeros(B, m, dtype=torch.bool)
            lora_rows[:, causal_rows:] = True
        return self.forward_rows(tokens, positions, starts, cache, masks,
                                 write_kv_rows=m if write_kv else 0, lora_rows=lora_rows,
                                 layers=layers, with_logits=with_logits)

    def forward_rows(self, tokens: torch.Tensor, positions: torch.Tensor, starts: List[int],
                     cache, masks: List[torch.Tensor], write_kv_rows: int = 0,
                     lora_rows: Optional[torch.Tensor] = None,
                     layers: Optional[List[int]] = None,
                     with_logits: bool = True) -> Optional[torch.Tensor]:
        """The general forward: row r of sequence b has token tokens[b, r] at absolute
        position positions[b, r] (RoPE); its keys are the cached rows [0, starts[b]) followed
        by this forward's m rows, and masks[b] [m, starts[b]+m] says which it sees.  The
        first write_kv_rows rows store their K/V into the cache at their positions (which
        must be starts[b]+r).  lora_rows [B, m] (bool) picks the rows that take the adapter's
        delta when one is set.  Returns logits [B, m, V] (compute dtype) or None."""
        c = self.cfg
        B, m = tokens.shape
        hd, Hq, Hkv = c.head_dim, c.n_q_heads, c.n_kv_heads
        for b in range(B):
            n = int(starts[b])
            assert masks[b].shape == (m, n + m)
            assert all(int(positions[b, r]) == n + r for r in range(write_kv_rows))
        h = self._w(self.embed[tokens.long()])                # [B, m, d]
        for li in (range(c.n_layers) if layers is None else layers):
            L = self.layers[li]
            q = self._normed_mm(h, L["g1"], L["wq"]).view(B, m, Hq, hd)
            k = self._normed_mm(h, L["g1"], L["wk"]).view(B, m, Hkv, hd)
            v = self._normed_mm(h, L["g1"], L["wv"]).view(B, m, Hkv, hd)
            att = torch.empty(B, m, Hq, hd, dtype=self.cdt)
            for b in range(B):
                n = int(starts[b])
                pos = positions[b]
                qb = rope_rotate(q[b], pos[:, None], c.rope_theta)                # [m, Hq, hd]
                kb = self._kv(rope_rotate(k[b], pos[:, None], c.rope_theta))      # [m, Hkv, hd]
                vb = self._kv(v[b])
                Kc, Vc = cache[b][li]
                keys = torch.cat([Kc[:, :n].to(self.cdt), kb.transpose(0, 1)], dim=1)   # [Hkv, n+m, hd]
                vals = torch.cat([Vc[:, :n].to(self.cdt), vb.transpose(0, 1)], dim=1)
                o = attention_explicit(qb.transpose(0, 1), keys, vals, masks[b])  # [Hq, m, hd]
                att[b] = o.transpose(0, 1)
                w = write_kv_rows
                if w:
                    Kc[:, n:n + w] = kb[:w].transpose(0, 1).to(self.kv_dtype)
                    Vc[:, n:n + w] = vb[:w].transpose(0, 1).to(self.kv_dtype)
            a2 = att.reshape(B, m, Hq * hd)
            if lora_rows is not None and self.lora is not None:
                # the delta joins the residual first, on the drafter rows only
                LA, LB, sc = self.lora[0][li], self.lora[1][li], self.lora[2]
                delta = sc * self._mm(self._mm(a2, LA), LB)
                h = h + torch.where(lora_rows[..., None], delta, torch.zeros_like(delta))
            h = h + self._mm(a2, L["wo"])
            g = self._normed_mm(h, L["g2"], L["wg"])
            u = self._normed_mm(h, L["g2"], L["wu"])
            act = g / (1.0 + torch.exp(-g)) * u                     # silu(g) * u
            h = h + self._mm(act, L["wd"])
        if not with_logits:
            return None
        return self._normed_mm(h, self.gf, self.lm)
