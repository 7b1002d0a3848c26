"""The decode attention entry point that allocates nothing.

Some callers cannot allocate device memory while they run (a fixed device
memory budget, memory owned by the host application's own pool, or a launch
path that must not synchronise the way an allocation can). For them the
library offers `decode_attn_static_scratch`, which keeps its split-KV partials
in a fixed array inside the library instead of a workspace.

These tests call it through the C ABI twice in a row and check each output
against the fp64 oracle's causal attention (one query per sequence at position
kv_len[b], keys 0..kv_len[b], GQA grouping by repeat_kv) within the bf16
tolerance the other tests use; they check that the second call leaves the
device's free memory unchanged and that the error word reads clean after each
call; that lengths outside the cache set the entry point's error word, which
llama_block_sync_status(NULL) reads and clears; and that calls whose partials
would not fit, or whose K/V are misaligned, are refused on the host. This file
is named so that pytest collects it last."""

import gc

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import make_tensor
from tests.helpers import BF16_TOL, as_np, row_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb


def _oracle(q, k, v, lens, seqs):
    """Oracle attention of query q[b, h] at position lens[b] over keys 0..lens[b]."""
    out = []
    for b in seqs:
        L = int(lens[b])
        qb = as_np(q[b:b + 1]).reshape(1, q.shape[1], 1, q.shape[2])
        out.append(ob.causal_attention(qb, as_np(k[b:b + 1, :, :L + 1]), as_np(v[b:b + 1, :, :L + 1])))
    return np.concatenate(out, axis=0)[:, :, 0, :]  # [len(seqs), H, dh]


@pytest.mark.parametrize("B,H,Hkv,dh,L,ks", [(4, 8, 2, 128, 517, 640), (32, 32, 32, 128, 4096, 4224),
                                              (3, 4, 4, 64, 40, 64), (2, 6, 2, 128, 700, 768)])
def test_static_scratch_decode_attention_matches_oracle(B, H, Hkv, dh, L, ks):
    q = make_tensor((B, H, dh), 900, torch.bfloat16)
    k = make_tensor((B, Hkv, ks, dh), 901, torch.bfloat16)
    v = make_tensor((B, Hkv, ks, dh), 902, torch.bfloat16)
    lens = [L - (13 * b) % min(L, 200) for b in range(B)]  # ragged lengths, the longest L
    seqs = list(range(B)) if B <= 4 else [0, 9, 22, B - 1]
    want = _oracle(q, k, v, lens, seqs)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kv_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = torch.empty(B, H * dh, dtype=torch.bfloat16, device="cuda")
    free_after_first = None
    for call in range(2):
        o.fill_(float("nan"))
        torch.cuda.synchronize()
        if call == 1:
            gc.collect()  # tensors of earlier tests in reference cycles are freed now, not mid-call
            free_after_first = torch.cuda.mem_get_info()[0]
            alloc_after_first = torch.cuda.memory_allocated()
        lb.decode_attn_static_scratch(qd, kd, vd, o, kv_len)
        lb.llama_block_sync_status()  # raises unless the error words read clean
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_after_first
            assert torch.cuda.memory_allocated() == alloc_after_first
        assert row_err(o.view(B, H, dh)[seqs], want) <= BF16_TOL


@pytest.mark.parametrize("bad_len", ["k_stride", "negative"])
def test_static_scratch_out_of_range_length_is_reported(bad_len):
    """A length whose key count does not fit the cache (or is negative) makes the
    kernel skip every K/V read and set the entry point's error word; sync_status
    with a NULL handle returns LB_ERR_CACHE_FULL and clears it."""
    B, H, dh, ks = 2, 4, 128, 128
    q = torch.zeros(B, H, dh, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(B, H, ks, dh, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(B, H * dh, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([5, ks if bad_len == "k_stride" else -1], dtype=torch.int32, device="cuda")
    lb.decode_attn_static_scratch(q, k, k, o, lens)
    with pytest.raises(lb.LlamaBlockError) as ei:
        lb.llama_block_sync_status()
    assert ei.value.status == 5  # LB_ERR_CACHE_FULL
    lb.llama_block_sync_status()  # cleared


def test_static_scratch_rejects_calls_that_do_not_fit():
    B, H, dh, ks = 64, 64, 128, 8192  # 64*64*64*130 floats > the 6 Mi-float array
    q = torch.zeros(B, H, dh, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 8, dh, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(B, H * dh, dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = lb.lib.decode_attn_static_scratch(q.data_ptr(), k.data_ptr(), k.data_ptr(), o.data_ptr(),
                                           lens.data_ptr(), B, H, H, dh, ks, None)
    assert st == 1
    assert "exceeds the fixed scratch" in lb.llama_block_last_error()


def test_static_scratch_rejects_misaligned_kv():
    B, H, dh, ks = 1, 2, 64, 64
    q = torch.zeros(B, H, dh, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(B * H * ks * dh + 8, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(B, H * dh, dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = lb.lib.decode_attn_static_scratch(q.data_ptr(), k.data_ptr() + 2, k.data_ptr(), o.data_ptr(),
                                           lens.data_ptr(), B, H, H, dh, ks, None)
    assert st == 1
    assert "16-byte aligned" in lb.llama_block_last_error()
