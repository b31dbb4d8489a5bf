"""Python binding of the nld C ABI (include/nld.h): argument marshalling only.

Every step of the decode path runs in the CUDA library `libnld.so` built from `csrc/`.  The
binding passes raw device pointers of torch tensors; there is no fallback: if the library is
missing or no GPU is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libnld.so")
HEADER = os.path.join(os.path.dirname(PKG_DIR), "include", "nld.h")

NLD_F32, NLD_BF16 = 0, 1
NLD_MODE_AR, NLD_MODE_DRAFT, NLD_MODE_VERIFY, NLD_MODE_DIFFUSE, NLD_MODE_QUAD = 0, 1, 2, 3, 4
STATUS = {0: "NLD_OK", 1: "NLD_ERR_ARG", 2: "NLD_ERR_OOM", 3: "NLD_ERR_CUDA", 4: "NLD_ERR_KV_FULL",
          5: "NLD_ERR_STATE", 6: "NLD_ERR_TIMEOUT", 7: "NLD_ERR_DEVICE", 8: "NLD_ERR_UNSUPPORTED"}


class nld_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn_dim", ctypes.c_int),
                ("vocab", ctypes.c_int), ("dtype", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_seq", ctypes.c_int), ("page_size", ctypes.c_int), ("block_k", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


class NldError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libnld.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} not found: build it with `python -m self_speculation_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "nld_create": ([ctypes.POINTER(nld_config), P, ctypes.POINTER(P)], I),
        "nld_destroy": ([P], I),
        "nld_init_weights": ([P, ctypes.POINTER(P), I, I], I),
        "nld_init_lora": ([P, I, F, ctypes.POINTER(P), I, I], I),
        "nld_prefill": ([P, P, I, P, I, P], I),
        "nld_ar_step": ([P, P], I),
        "nld_selfspec_draft_verify": ([P], I),
        "nld_kv_commit": ([P, P, P, P], I),
        "nld_selfspec_round": ([P, P, P, P], I),
        "nld_quadratic_round": ([P, P, P], I),
        "nld_diffuse_block_step": ([P, F, P, P, P, P], I),
        "nld_diffuse_block_step_fused": ([P, F, P, P, P, P], I),
        "nld_diffuse_step_nonlockstep": ([P, F, P, P, P, P], I),
        "nld_debug_logits": ([P, I, P], I),
        "nld_debug_state": ([P, P, P, P, P], I),
        "nld_sync": ([P], I),
        "nld_time_gemm": ([P, I, I, I, I, ctypes.POINTER(F)], I),
        "nld_trace_gemm": ([P, I, I, I, P, ctypes.POINTER(I)], I),
        "nld_debug_gemm_plan": ([P, I, I, ctypes.POINTER(I)], I),
        "nld_plan_chain": ([I, I, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I), I,
                            ctypes.POINTER(I)], I),
        "nld_plan_attention": ([I, I, I, I, I, I, ctypes.POINTER(I)], I),
        "nld_trace_chain": ([P, I, I, P, ctypes.POINTER(I)], I),
        "nld_time_chain": ([P, I, I, I, ctypes.POINTER(F)], I),
        "nld_debug_chain_tuning": ([P, I, I, I, I, I, I], I),
        "nld_debug_timeout_chain": ([P, ctypes.c_ulonglong], I),
        "nld_debug_attention_tuning": ([P, I, I], I),
        "nld_debug_attention_kernel": ([I], I),
        "nld_debug_attention_tile": ([I], I),
        "nld_debug_layer_trace": ([P, I, P, S, P, S], I),
        "nld_stream": ([P], P),
        "nld_last_error": ([P], ctypes.c_char_p),
        "nld_attention": ([P, P, P, I, I, P, I, I, I, I, I, I, I, P, P], I),
        "nld_lm_head_workspace_size": ([I, I, I], S),
        "nld_lm_head_argmax": ([P, P, I, I, I, F, P, P, P, S, P], I),
        "nld_lm_head_static_max_bytes": ([], S),
        "nld_lm_head_argmax_static": ([P, P, I, I, I, F, P, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def header_functions() -> list:
    """Names of the functions include/nld.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(nld_\w+)\s*\(", txt, re.M)))


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _cfg_struct(cfg) -> nld_config:
    return nld_config(cfg.n_layers, cfg.d_model, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim,
                      cfg.ffn_dim, cfg.vocab, cfg.dtype, cfg.max_batch, cfg.max_seq,
                      cfg.page_size, cfg.block_k, cfg.rms_eps, cfg.rope_theta)


class Context:
    """One nld_ctx.  `cfg` is any object with the nld_config fields."""

    def __init__(self, cfg, stream: Optional[int] = None):
        self.lib = load_library()
        self.cfg = cfg
        self._c = _cfg_struct(cfg)
        h = ctypes.c_void_p()
        self._check(self.lib.nld_create(ctypes.byref(self._c), stream, ctypes.byref(h)), None)
        self.h = h

    def _check(self, status: int, h) -> None:
        if status != 0:
            msg = self.lib.nld_last_error(h).decode()
            raise NldError(status, msg)

    def close(self) -> None:
        if getattr(self, "h", None):
            self.lib.nld_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- entry points (same names as the C ABI) -------------------------------------------
    def nld_stream(self) -> int:
        return self.lib.nld_stream(self.h)

    def nld_init_weights(self, tensors: Sequence, on_device: Optional[bool] = None) -> None:
        tensors = [t.contiguous() for t in tensors]
        if on_device is None:
            on_device = tensors[0].is_cuda
        arr = (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])
        self._check(self.lib.nld_init_weights(self.h, arr, len(tensors), int(on_device)), self.h)

    def nld_init_lora(self, rank: int, scale: float, tensors: Optional[Sequence] = None,
                      on_device: Optional[bool] = None) -> None:
        tensors = [t.contiguous() for t in (tensors or [])]
        if on_device is None:
            on_device = bool(tensors) and tensors[0].is_cuda
        arr = (ctypes.c_void_p * max(1, len(tensors)))(*[t.data_ptr() for t in tensors])
        self._check(self.lib.nld_init_lora(self.h, rank, scale, arr if tensors else None,
                                           len(tensors), int(on_device)), self.h)

    def nld_prefill(self, tokens, lens=None, pending_out=None) -> None:
        """tokens [B, stride] int32 (device); lens [B] int32 prompt lengths (None: all stride);
        pending_out [B] int32 receives the pending tokens."""
        B, P = tokens.shape
        self._check(self.lib.nld_prefill(self.h, _ptr(tokens), P, _ptr(lens), B, _ptr(pending_out)),
                    self.h)

    def nld_ar_step(self, tokens_out) -> None:
        self._check(self.lib.nld_ar_step(self.h, _ptr(tokens_out)), self.h)

    def nld_selfspec_draft_verify(self) -> None:
        self._check(self.lib.nld_selfspec_draft_verify(self.h), self.h)

    def nld_kv_commit(self, nrows, tokens_out, ncommit_out) -> None:
        self._check(self.lib.nld_kv_commit(self.h, _ptr(nrows), _ptr(tokens_out), _ptr(ncommit_out)),
                    self.h)

    def nld_selfspec_round(self, tokens_out, ncommit_out, force=None) -> None:
        self._check(self.lib.nld_selfspec_round(self.h, _ptr(tokens_out), _ptr(ncommit_out),
                                                _ptr(force)), self.h)

    def nld_quadratic_round(self, tokens_out, ncommit_out) -> None:
        self._check(self.lib.nld_quadratic_round(self.h, _ptr(tokens_out), _ptr(ncommit_out)), self.h)

    def nld_diffuse_block_step(self, threshold: float, block_out, conf_out, ncommit_out) -> bool:
        filled = ctypes.c_int32(0)
        self._check(self.lib.nld_diffuse_block_step(self.h, float(threshold), _ptr(block_out),
                                                    _ptr(conf_out), _ptr(ncommit_out),
                                                    ctypes.byref(filled)), self.h)
        return bool(filled.value)

    def nld_diffuse_block_step_fused(self, threshold: float, block_out, conf_out, ncommit_out) -> bool:
        filled = ctypes.c_int32(0)
        self._check(self.lib.nld_diffuse_block_step_fused(self.h, float(threshold), _ptr(block_out),
                                                          _ptr(conf_out), _ptr(ncommit_out),
                                                          ctypes.byref(filled)), self.h)
        return bool(filled.value)

    def nld_diffuse_step_nonlockstep(self, threshold: float, block_out=None, conf_out=None,
                                     ncommit_out=None, state_out=None) -> None:
        self._check(self.lib.nld_diffuse_step_nonlockstep(self.h, float(threshold), _ptr(block_out),
                                                          _ptr(conf_out), _ptr(ncommit_out),
                                                          _ptr(state_out)), self.h)

    def nld_debug_logits(self, mode: int, logits_out) -> None:
        self._check(self.lib.nld_debug_logits(self.h, int(mode), _ptr(logits_out)), self.h)

    def nld_debug_state(self, lens=None, pending=None, draft=None, verify=None) -> None:
        self._check(self.lib.nld_debug_state(self.h, _ptr(lens), _ptr(pending), _ptr(draft),
                                             _ptr(verify)), self.h)

    def nld_time_gemm(self, which: int, layer: int, M: int, reps: int) -> float:
        ms = ctypes.c_float(0.0)
        self._check(self.lib.nld_time_gemm(self.h, which, layer, M, reps, ctypes.byref(ms)), self.h)
        return ms.value

    def nld_trace_gemm(self, which: int, layer: int, M: int, trace) -> int:
        g = ctypes.c_int(0)
        self._check(self.lib.nld_trace_gemm(self.h, which, layer, M, _ptr(trace), ctypes.byref(g)),
                    self.h)
        return g.value

    def nld_time_chain(self, layer: int, M: int, reps: int) -> float:
        ms = ctypes.c_float(0.0)
        self._check(self.lib.nld_time_chain(self.h, layer, M, reps, ctypes.byref(ms)), self.h)
        return ms.value

    def nld_trace_chain(self, layer: int, M: int, trace) -> int:
        g = ctypes.c_int(0)
        self._check(self.lib.nld_trace_chain(self.h, layer, M, _ptr(trace), ctypes.byref(g)), self.h)
        return g.value

    def nld_debug_chain_tuning(self, stage_cap: int = 0, k_tiles_per_stage: int = 0,
                               boundary_prefetch: int = 16, act_3d: int = 1,
                               runahead_stages: int = 0, warm_next: int = 0) -> None:
        self._check(self.lib.nld_debug_chain_tuning(self.h, int(stage_cap), int(k_tiles_per_stage),
                                                    int(boundary_prefetch), int(act_3d),
                                                    int(runahead_stages), int(warm_next)), self.h)

    def nld_debug_layer_trace(self, layer: int = -1, attn_trace=None, chain_trace=None) -> None:
        """Timestamp one layer's attention and chain launches (int64 device tensors, zeroed by
        the caller); layer -1 turns the hook off."""
        self._check(self.lib.nld_debug_layer_trace(
            self.h, int(layer), _ptr(attn_trace), 0 if attn_trace is None else attn_trace.numel(),
            _ptr(chain_trace), 0 if chain_trace is None else chain_trace.numel()), self.h)

    def nld_debug_attention_tuning(self, rows_per_cta: int = 0, min_tiles_per_split: int = 0) -> None:
        self._check(self.lib.nld_debug_attention_tuning(self.h, int(rows_per_cta), int(min_tiles_per_split)),
                    self.h)

    def nld_debug_timeout_chain(self, timeout_ns: int) -> None:
        self._check(self.lib.nld_debug_timeout_chain(self.h, int(timeout_ns)), self.h)

    def nld_debug_gemm_plan(self, which: int, M: int) -> dict:
        v = (ctypes.c_int * 8)()
        self._check(self.lib.nld_debug_gemm_plan(self.h, which, M, v), self.h)
        keys = ["NT", "tok_tiles", "row_tiles", "KT", "split", "ks", "ctas", "stages"]
        return dict(zip(keys, list(v)))

    def nld_sync(self) -> None:
        self._check(self.lib.nld_sync(self.h), self.h)


def nld_attention(q, kv_pool, page_table, lens, block_size: int, max_len: int, out,
                  stream: Optional[int] = None) -> None:
    """q [B, m, Hq, hd] bf16, kv_pool [n_pages, 2, Hkv, 64, hd] bf16, page_table [B, pps] int32,
    lens [B] int32, out like q."""
    lib = load_library()
    B, m, Hq, hd = q.shape
    n_pages, _, Hkv, _, _ = kv_pool.shape
    st = lib.nld_attention(_ptr(q), _ptr(kv_pool), _ptr(page_table), page_table.shape[1], n_pages,
                           _ptr(lens), B, m, Hq, Hkv, hd, int(block_size), int(max_len), _ptr(out),
                           stream)
    if st != 0:
        raise NldError(st, lib.nld_last_error(None).decode())


def nld_lm_head_workspace_size(M: int, d: int, vocab: int) -> int:
    return load_library().nld_lm_head_workspace_size(M, d, vocab)


def _current_stream(stream: Optional[int]) -> int:
    """The caller's stream, else torch's current stream on the current device (not the legacy
    default stream, so inputs produced on a side stream are ordered before the launches)."""
    if stream is not None:
        return stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _lm_head_args(hidden, lm_weight, argmax_out, conf_out):
    import torch
    for name, t, dt in (("hidden", hidden, torch.bfloat16), ("lm_weight", lm_weight, torch.bfloat16),
                        ("argmax_out", argmax_out, torch.int32), ("conf_out", conf_out, torch.float32)):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == dt):
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    if hidden.dim() != 2 or lm_weight.dim() != 2 or lm_weight.shape[1] != hidden.shape[1]:
        raise ValueError("hidden [M, d] and lm_weight [vocab, d] expected")
    M = hidden.shape[0]
    if argmax_out.numel() < M or conf_out.numel() < M:
        raise ValueError(f"argmax_out and conf_out must hold at least M = {M} elements")
    return M, hidden.shape[1], lm_weight.shape[0]


def nld_lm_head_argmax(hidden, lm_weight, rms_eps: float, argmax_out, conf_out, workspace,
                       stream: Optional[int] = None) -> None:
    """hidden [M, d] bf16, lm_weight [vocab, d] bf16, argmax_out [M] int32, conf_out [M] fp32,
    workspace uint8 of nld_lm_head_workspace_size bytes."""
    lib = load_library()
    M, d, vocab = _lm_head_args(hidden, lm_weight, argmax_out, conf_out)
    stream = _current_stream(stream)
    st = lib.nld_lm_head_argmax(_ptr(hidden), _ptr(lm_weight), M, d, vocab, float(rms_eps),
                                _ptr(argmax_out), _ptr(conf_out), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), stream)
    if st != 0:
        raise NldError(st, lib.nld_last_error(None).decode())


def nld_lm_head_argmax_static(hidden, lm_weight, rms_eps: float, argmax_out, conf_out,
                              stream: Optional[int] = None) -> None:
    """nld_lm_head_argmax with the library's built-in scratch (allocates nothing)."""
    lib = load_library()
    M, d, vocab = _lm_head_args(hidden, lm_weight, argmax_out, conf_out)
    stream = _current_stream(stream)
    st = lib.nld_lm_head_argmax_static(_ptr(hidden), _ptr(lm_weight), M, d, vocab, float(rms_eps),
                                       _ptr(argmax_out), _ptr(conf_out), stream)
    if st != 0:
        raise NldError(st, lib.nld_last_error(None).decode())
