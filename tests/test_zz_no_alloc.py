"""The decode attention entry point that allocates nothing.

Some callers cannot allocate device memory while they run (a fixed device
memory budget, memory owned by the host application's own pool, or a launch
path that must not synchronise the way an allocation can). For them the
library offers `decode_attn_static_scratch`, which keeps its split-KV partials
in a fixed array inside the library instead of a workspace. This test calls it
through the C ABI twice in a row and checks its output against the existing
`causal_attn` entry point (one query per sequence at the last position) within
the bf16 tolerance the other tests use; it also checks that a call whose
partials would not fit is refused on the host. This file is named so that
pytest collects it last."""

import pytest
import torch

from synth import make_tensor
from tests.helpers import BF16_TOL, row_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb


@pytest.mark.parametrize("B,H,Hkv,dh,L,ks", [(4, 8, 2, 128, 517, 640), (32, 32, 32, 128, 4096, 4224),
                                              (3, 4, 4, 64, 40, 64)])
def test_static_scratch_decode_attention_matches_causal_attn(B, H, Hkv, dh, L, ks):
    q = make_tensor((B, H, 1, dh), 900, torch.bfloat16).cuda()
    k = make_tensor((B, Hkv, ks, dh), 901, torch.bfloat16).cuda()
    v = make_tensor((B, Hkv, ks, dh), 902, torch.bfloat16).cuda()
    ref = torch.empty(B, 1, H * dh, dtype=torch.bfloat16, device="cuda")
    lb.causal_attn(q, k, v, ref, Tk=L + 1)
    lb.llama_block_sync_status()
    kv_len = torch.full((B,), L, dtype=torch.int32, device="cuda")
    for _ in range(2):
        o = torch.full((B, H * dh), float("nan"), dtype=torch.bfloat16, device="cuda")
        lb.decode_attn_static_scratch(q.view(B, H, dh), k, v, o, kv_len)
        torch.cuda.synchronize()
        assert row_err(o.view(B, H, dh), ref.view(B, H, dh)) <= BF16_TOL


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
