"""The C-ABI library builds, loads and exports every entry point include/nld.h declares (no GPU;
no compute calls)."""
import ctypes
import os
import subprocess

import pytest

import self_speculation_b200 as nb
from self_speculation_b200 import build as nbuild


def test_library_builds_and_loads():
    path = nbuild.build()
    assert os.path.exists(path)
    lib = nb.load_library()
    assert lib is not None


def test_every_header_function_is_exported():
    nbuild.build()
    names = nb.header_functions()
    assert "nld_selfspec_round" in names and "nld_kv_commit" in names
    out = subprocess.run(["nm", "-D", "--defined-only", nb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = nb.load_library()
    for n in names:
        assert hasattr(lib, n)


def _cfg(**kw):
    import synth
    return synth.TINY_F32.replace(**kw)


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(d_model=200), dict(page_size=32),
                                 dict(block_k=0), dict(block_k=33), dict(n_kv_heads=3),
                                 dict(dtype=7), dict(ffn_dim=1000), dict(max_seq=9000)])
def test_invalid_config_rejected_before_any_cuda_call(bad):
    lib = nb.load_library()
    c = nb._cfg_struct(_cfg(**bad))
    h = ctypes.c_void_p()
    st = lib.nld_create(ctypes.byref(c), None, ctypes.byref(h))
    assert st == 1, nb.STATUS.get(st)
    assert b"invalid config" in lib.nld_last_error(None)
    assert not h.value


def test_null_arguments_rejected():
    lib = nb.load_library()
    assert lib.nld_create(None, None, None) == 1
    assert lib.nld_destroy(None) == 0
    assert lib.nld_prefill(None, None, 1, None, 1, None) == 1
    assert lib.nld_debug_chain_tuning(None, 0, 0, 16, 1, 0, 0) == 1
    assert lib.nld_debug_timeout_chain(None, 1000000) == 1
    assert lib.nld_debug_layer_trace(None, -1, None, 0, None, 0) == 1
    assert lib.nld_selfspec_round(None, None, None, None) == 1
    assert lib.nld_sync(None) == 1
    assert lib.nld_attention(None, None, None, 1, 1, None, 1, 32, 32, 8, 128, 1, 32, None, None) == 1
    assert lib.nld_init_lora(None, 8, 1.0, None, 0, 0) == 1
    assert lib.nld_diffuse_block_step_fused(None, 0.9, None, None, None, None) == 1
    assert lib.nld_diffuse_step_nonlockstep(None, 0.9, None, None, None, None) == 1
    assert lib.nld_plan_chain(1, 1, None, None, None, 1, None) == 1
    assert lib.nld_plan_attention(1, 1, 8, 8, 1, 148, None) == 1
    assert lib.nld_debug_attention_kernel(5) == 1
    assert lib.nld_debug_attention_kernel(-1) == 1
    assert lib.nld_debug_attention_kernel(0) == 0
    assert lib.nld_debug_attention_tile(32) == 1
    assert lib.nld_debug_attention_tile(256) == 1
    assert lib.nld_debug_attention_tile(0) == 0
