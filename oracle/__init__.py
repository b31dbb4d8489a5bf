"""CPU oracle for the tri-mode decode round (test infrastructure only).

A plain, slow, obviously correct restatement of what the decode round computes, written
from the pages on Nemotron-Labs-Diffusion:

* ranhao.site technical-report notes (zh), sections 3.2 (block-wise attention:
  bidirectional inside a block, causal across blocks, prefix KV reused), 4.3 (the clean
  stream is strictly causal), 5.1 (AR decoding), 5.2 (block-wise diffusion decoding with
  confidence-based commits) and 5.3 (self-speculation: the diffusion pathway drafts k
  tokens, the AR pathway verifies, the longest correct prefix is accepted, stopping at the
  first mismatch);
* r9-hu paper digest, "Method" (diffusion loss with a clean prefix, block attention mask;
  tri-mode inference: k drafts in one forward, causal verification, 1..k+1 tokens a round);
* shilu.ai translation of the HuggingFace blog, "Deploy and infer with SGLang" (32-token
  blocks, a confidence threshold decides commits, self-speculation is lossless against AR
  at temperature 0).

Only `tests/`, the package entry point's `smoke()` and the bench's CPU-baseline leg may
import this package.  The product path never calls it, and it shares no code with the
CUDA library: the two meet only in the seeded inputs of `synth`.

Parity unpinned: whether the shifted-prediction reading (block row i predicts position
i+1, see `decode.py`) matches the released checkpoints; any accuracy, acceptance-rate or
tokens-per-forward figure of a trained model.  Neither can be pinned without trained
weights.
"""
from .model import OracleModel, rmsnorm, rope_rotate, attention_explicit, block_mask, causal_mask
from .decode import (accept_length, commit_after_verify, diffusion_commit, SeqState,
                     prefill, ar_step, selfspec_round, diffusion_step, ar_generate,
                     selfspec_generate, diffuse_generate, argmax_lowest, confidence)

__all__ = ["OracleModel", "rmsnorm", "rope_rotate", "attention_explicit", "block_mask",
           "causal_mask", "accept_length", "commit_after_verify", "diffusion_commit",
           "SeqState", "prefill", "ar_step", "selfspec_round", "diffusion_step",
           "ar_generate", "selfspec_generate", "diffuse_generate", "argmax_lowest",
           "confidence"]
