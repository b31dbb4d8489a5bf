"""Seeded synthetic inputs shared by the oracle, the CUDA library's tests and the bench.

This module holds no arithmetic of the decoding method. It only describes model shapes
and draws the random weights, prompts and attention operands that both sides consume, so
that the oracle and the library see the very same arrays.

Shapes follow the Llama-style decoder the self-speculation workloads are quoted on
(Nemotron-Labs-Diffusion technical report digest, ranhao.site notes, sections 2 and 5;
HuggingFace blog translation, shilu.ai, "Deploy and infer with SGLang": 32-token block).

Weight recipe (reading of the pages, which publish no weights): every matrix and the
embedding are i.i.d. N(0, 0.02^2); RMSNorm gains are 1; there are no biases; the LM head
is not tied to the embedding.  The embedding has vocab+1 rows, the extra row being the
[MASK] token (id == vocab).  bf16 configurations round the drawn fp32 values to bf16
(round-to-nearest-even) once, and both sides receive the rounded arrays.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    dtype: int = BF16          # F32 or BF16: storage type of weights, activations and KV
    max_batch: int = 1
    max_seq: int = 2048
    page_size: int = 64
    block_k: int = 32
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0

    @property
    def mask_id(self) -> int:
        return self.vocab

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def replace(self, **kw) -> "ModelConfig":
        return dataclasses.replace(self, **kw)

    def weight_bytes_per_forward(self) -> int:
        """Bytes of weights a forward streams (embedding rows excluded)."""
        el = 4 if self.dtype == F32 else 2
        per_layer = (self.q_dim + 2 * self.kv_dim) * self.d_model + self.d_model * self.q_dim \
            + 3 * self.ffn_dim * self.d_model
        return el * (self.n_layers * per_layer + self.vocab * self.d_model)

    def kv_bytes_per_token(self) -> int:
        el = 4 if self.dtype == F32 else 2
        return el * 2 * self.n_layers * self.kv_dim


# Workload shapes (sizes as stated for each workload).
TINY_F32 = ModelConfig(n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=4, head_dim=64,
                       ffn_dim=1024, vocab=4096, dtype=F32, max_batch=1, max_seq=256,
                       block_k=8)
# Small bf16 shape for kernel parity: spans several tiles per GEMM, GQA group 4, a ragged
# vocabulary tail (5000 = 39*128 + 8) and the hd=128 tensor-core attention path.
SMALL_BF16 = ModelConfig(n_layers=2, d_model=512, n_q_heads=8, n_kv_heads=2, head_dim=128,
                         ffn_dim=1536, vocab=5000, dtype=BF16, max_batch=4, max_seq=640,
                         block_k=32)
LLAMA8B = ModelConfig(n_layers=36, d_model=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                      ffn_dim=12288, vocab=151936, dtype=BF16, max_batch=1, max_seq=2048,
                      block_k=32)
LLAMA14B = ModelConfig(n_layers=40, d_model=5120, n_q_heads=40, n_kv_heads=8, head_dim=128,
                       ffn_dim=17408, vocab=151936, dtype=BF16, max_batch=64, max_seq=4352,
                       block_k=32)


def weight_names(cfg: ModelConfig) -> List[str]:
    names = ["embed"]
    for l in range(cfg.n_layers):
        names += [f"l{l}.attn_norm", f"l{l}.wq", f"l{l}.wk", f"l{l}.wv", f"l{l}.wo",
                  f"l{l}.mlp_norm", f"l{l}.wg", f"l{l}.wu", f"l{l}.wd"]
    names += ["final_norm", "lm_head"]
    return names


def weight_shapes(cfg: ModelConfig) -> List[tuple]:
    d, F = cfg.d_model, cfg.ffn_dim
    shapes = [(cfg.vocab + 1, d)]
    for _ in range(cfg.n_layers):
        shapes += [(d,), (cfg.q_dim, d), (cfg.kv_dim, d), (cfg.kv_dim, d), (d, cfg.q_dim),
                   (d,), (F, d), (F, d), (d, F)]
    shapes += [(d,), (cfg.vocab, d)]
    return shapes


def _storage_dtype(cfg: ModelConfig):
    return torch.float32 if cfg.dtype == F32 else torch.bfloat16


def model_weights(cfg: ModelConfig, seed: int = 0, device: str = "cpu",
                  std: float = 0.02, layers: Optional[List[int]] = None,
                  lm_head_scale: float = 1.0) -> List[Optional[torch.Tensor]]:
    """Weights in the boundary's tensor order: embed, then per layer
    (attn_norm, wq, wk, wv, wo, mlp_norm, wg, wu, wd), then final_norm, lm_head.
    Matrices are row-major [out, in].

    Drawn tensor by tensor from one torch generator seeded with `seed` on `device`, so a
    given (cfg, seed, device) always gives the same arrays.  `layers` restricts which
    layers are materialised (others are None) for bounded CPU samples of large shapes;
    skipped layers still advance nothing, so a layer's values depend on its index only.
    `lm_head_scale` multiplies the LM head (peaky logits for multi-commit tests).
    """
    dt = _storage_dtype(cfg)
    out: List[Optional[torch.Tensor]] = []
    names = weight_names(cfg)
    shapes = weight_shapes(cfg)
    for idx, (name, shape) in enumerate(zip(names, shapes)):
        lid = int(name[1:].split(".")[0]) if (name.startswith("l") and name[1].isdigit()) else None
        if layers is not None and lid is not None and lid not in layers:
            out.append(None)
            continue
        if len(shape) == 1:
            out.append(torch.ones(shape, dtype=dt, device=device))
            continue
        g = torch.Generator(device=device)
        g.manual_seed(seed * 1000003 + idx)
        w = torch.empty(shape, dtype=torch.float32, device=device)
        w.normal_(0.0, std, generator=g)
        if name == "lm_head" and lm_head_scale != 1.0:
            w.mul_(lm_head_scale)
        out.append(w.to(dt))
        del w
    return out


def lora_weights(cfg: ModelConfig, rank: int, seed: int, std: float = 0.02,
                 device: str = "cpu") -> List[torch.Tensor]:
    """An o_proj adapter in the boundary's order: per layer A [rank, Hq*hd] then B [d, rank],
    N(0, std^2) drawn in fp32 from one CPU generator seeded with `seed` (A_0, B_0, A_1, ...),
    stored in the config dtype and moved to `device`."""
    g = torch.Generator().manual_seed(seed)
    dt = _storage_dtype(cfg)
    out: List[torch.Tensor] = []
    for _ in range(cfg.n_layers):
        out.append((torch.randn(rank, cfg.q_dim, generator=g) * std).to(dt).to(device))
        out.append((torch.randn(cfg.d_model, rank, generator=g) * std).to(dt).to(device))
    return out


def prompt_tokens(batch: int, length: int, vocab: int, seed: int = 1) -> torch.Tensor:
    """Uniform-random real token ids in [0, vocab), int32 [batch, length] (stand-in for the
    benchmark prompts, which are not available)."""
    g = torch.Generator()
    g.manual_seed(seed)
    return torch.randint(0, vocab, (batch, length), generator=g, dtype=torch.int64).to(torch.int32)


def attention_operands(batch: int, m: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                       prefix: int, seed: int = 2, device: str = "cpu"):
    """Q [batch, m, Hq, hd] and per-sequence K, V [batch, Hkv, prefix+m, hd], all i.i.d.
    N(0,1) rounded to bf16 (attention micro-workload)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = torch.randn((batch, m, n_q_heads, head_dim), generator=g, device=device)
    k = torch.randn((batch, n_kv_heads, prefix + m, head_dim), generator=g, device=device)
    v = torch.randn((batch, n_kv_heads, prefix + m, head_dim), generator=g, device=device)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
