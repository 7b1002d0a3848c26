"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/llama_block.h declares, computes the KV-cache ledger of
the mechanics page (chapter 04), and rejects bad arguments on the host before
anything reaches a device."""

import ctypes
import re
from pathlib import Path

import numpy as np
import pytest

import llama_pre_norm_b200 as lb
from oracle import block as ob

HEADER = Path(__file__).resolve().parent.parent / "include" / "llama_block.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([A-Za-z_][A-Za-z0-9_]*)\s*\(", text)
    skip = {"if", "defined", "sizeof"}
    return sorted({n for n in names if n not in skip and not n.isupper()})


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "llama_block_create" in names and "causal_attn" in names and len(names) == 34
    for n in names:
        assert hasattr(lb.lib, n), f"{n} declared in llama_block.h but not exported"


def test_kv_cache_bytes_matches_ledger():
    for B, hkv, dh, t, dt, nb in [(1, 8, 128, 4096, lb.LB_BF16, 2), (32, 32, 128, 4224, lb.LB_BF16, 2),
                                  (3, 4, 64, 100, lb.LB_F32, 4)]:
        assert lb.llama_block_kv_cache_bytes(B, hkv, dh, t, dt) == ob.kv_cache_bytes(1, B, t, hkv, dh, nb)
    assert lb.llama_block_kv_cache_bytes(0, 8, 128, 10, lb.LB_BF16) == 0
    assert lb.llama_block_kv_cache_bytes(1, 8, 128, 10, 7) == 0


def _create(*args):
    out = ctypes.c_void_p()
    st = lb.lib.llama_block_create(*args, ctypes.byref(out))
    return st, out.value


@pytest.mark.parametrize("args,want", [
    ((0, 4, 4, 64, 688, 1e-6, 1e4, lb.LB_F32, 64), 1),        # d = 0
    ((256, 4, 4, 64, 688, 0.0, 1e4, lb.LB_F32, 64), 1),       # eps = 0
    ((256, 4, 4, 64, 688, 1e-6, 1e4, 5, 64), 1),              # bad dtype
    ((256, 4, 4, 96, 688, 1e-6, 1e4, lb.LB_F32, 64), 2),      # head_dim 96
    ((256, 6, 4, 64, 688, 1e-6, 1e4, lb.LB_F32, 64), 2),      # 6 % 4 != 0
    ((4096, 32, 32, 128, 11008, 1e-6, 1e4, lb.LB_BF16, -1), 1),  # max_pos
    ((4100, 32, 32, 128, 11008, 1e-6, 1e4, lb.LB_BF16, 64), 2),  # d % 64 for bf16
])
def test_create_rejects_bad_arguments_on_host(args, want):
    st, h = _create(*args)
    assert st == want and h is None
    assert lb.llama_block_last_error() != ""


def test_create_null_out_and_null_handles():
    assert lb.lib.llama_block_create(256, 4, 4, 64, 688, 1e-6, 1e4, 0, 64, None) == 1
    assert lb.lib.llama_block_set_weights(None, *([None] * 10)) == 1
    assert lb.lib.llama_block_prefill(None, None, None, 1, 1, None, None, 1, None, None) == 1
    assert lb.lib.llama_block_decode(None, None, None, 1, None, None, 1, None, None) == 1
    assert lb.lib.llama_block_reserve(None, 1, 1) == 1
    assert lb.lib.llama_block_quantize_decode_weights(None, 1, None) == 1
    assert lb.lib.llama_block_set_rope_dynamic_ntk(None, 2.0, 2048, None) == 1
    assert lb.lib.llama_block_tp_mlp(None, None, None, None, None, 1, None) == 1
    assert lb.lib.llama_block_tp_add(None, None, None, 4, 8, 1, None) == 1
    assert lb.lib.llama_block_tp_add(None, None, None, 4, 7, 1, None) == 1
    assert lb.lib.llama_block_set_lengths(None, None, 1) == 1
    assert lb.lib.llama_block_enable_timing(None, 1) == 1
    assert lb.lib.llama_block_stage_times(None, None, 0, None) == 1
    assert lb.lib.llama_block_stage_name(None, 0) == b""
    assert lb.lib.llama_block_launch_count(None) == 0
    assert lb.lib.llama_block_extend(None, None, None, 1, 1, None, None, 1, None, None) == 1
    assert lb.lib.llama_stack_create(0, 256, 4, 4, 64, 688, 1e-6, 1e4, 0, 64, ctypes.byref(ctypes.c_void_p())) == 1
    assert lb.lib.llama_stack_create(1, 256, 4, 4, 64, 688, 1e-6, 1e4, 0, 64, None) == 1
    assert lb.lib.llama_stack_layer(None, 0) is None
    assert lb.lib.llama_stack_prefill(None, None, None, 1, 1, None, None, 1, None, None) == 1
    assert lb.lib.llama_stack_decode(None, None, None, 1, None, None, 1, None, None) == 1
    assert lb.lib.llama_stack_set_lengths(None, None, 1) == 1
    lb.lib.llama_stack_destroy(None)
    lb.lib.llama_block_destroy(None)  # no-op


def test_standalone_entry_points_reject_bad_arguments():
    assert lb.lib.rmsnorm(None, None, None, 1, 8, 1e-6, 0, None) == 1
    assert lb.lib.rmsnorm(1, 1, 1, 1, 12, 1e-6, 0, None) == 2          # d % 8
    assert lb.lib.rmsnorm(1, 1, 1, 1, 8, 1e-6, 9, None) == 1           # dtype
    assert lb.lib.rope_apply(None, None, 1, 1, 1, 64, 1e4, 0, None) == 1
    assert lb.lib.rope_apply(1, 1, 1, 1, 1, 63, 1e4, 0, None) == 1     # odd head_dim
    assert lb.lib.causal_attn(1, 1, 1, 1, 1, 5, 4, 2, 2, 64, 4, 1, None) == 1   # Tq > Tk
    assert lb.lib.causal_attn(1, 1, 1, 1, 1, 4, 4, 2, 2, 64, 3, 1, None) == 1   # stride < Tk
    assert lb.lib.causal_attn(1, 1, 1, 1, 1, 4, 4, 2, 2, 80, 4, 1, None) == 2   # head_dim
    assert lb.lib.causal_attn(1, 1, 1, 1, 1, 4, 4, 3, 2, 64, 4, 1, None) == 2   # grouping
    assert lb.lib.swiglu_mlp(None, 1, 1, 1, 1, 1, 64, 64, 1, None) == 1
    assert lb.lib.swiglu_mlp(1, 1, 1, 1, 1, 1, 96, 64, 1, None) == 2   # bf16 d % 64
    assert lb.lib.llama_block_selftest_timeout(0, None) == 1


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(2, 8)
    with pytest.raises(ValueError):
        lb.rmsnorm(x, torch.ones(8), torch.zeros(2, 8), 1e-6)
