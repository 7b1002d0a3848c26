"""GPU parity of chunked prefill (llama_block_extend) and of a multi-layer stack
(llama_stack_*) against the fp64 oracle: prefill -> extend -> decode, the
prefill -> decode handoff of the mechanics page's chapter 04, with the cache
offset landing inside a tile (not a multiple of 128) so the offset causal mask
and the RoPE positions L + t are exercised."""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import BlockConfig, make_decode_x, make_weights, make_x
from tests.helpers import BF16_TOL, F32_TOL, cuda, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb

CFGS = [
    BlockConfig("ext-f32", d=256, n_heads=4, n_kv_heads=2, head_dim=64, f=512, B=2, T=1, dtype="f32",
                gain="1+N(0,0.1)"),
    BlockConfig("ext-bf16-gqa", d=512, n_heads=4, n_kv_heads=2, head_dim=128, f=1024, B=2, T=1,
                dtype="bf16", gain="1+N(0,0.1)"),
    BlockConfig("ext-bf16-dh64", d=256, n_heads=8, n_kv_heads=8, head_dim=64, f=640, B=1, T=1,
                dtype="bf16"),
]
CHUNKS = [77, 150, 33]  # prefill 77 tokens, then extend by 150 and by 33


def _tol(cfg):
    return F32_TOL if cfg.dtype == "f32" else BF16_TOL


def _oracle_args(cfg):
    return cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_block_prefill_extend_decode(cfg):
    W = make_weights(cfg)
    T_all = sum(CHUNKS)
    X = make_x(cfg, T=T_all)
    t_max = T_all + 4
    dt = cfg.torch_dtype
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base,
                        dt, max_pos=t_max)
    blk.set_weights(weights_to_cuda(W))
    kc = torch.zeros(cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=dt, device="cuda")
    vc = torch.zeros_like(kc)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    kr = np.zeros((cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim))
    vr = np.zeros_like(kr)
    L = 0
    for i, T in enumerate(CHUNKS):
        x = X[:, L:L + T].contiguous()
        y = torch.empty(cfg.B, T, cfg.d, dtype=dt, device="cuda")
        (blk.prefill if i == 0 else blk.extend)(cuda(x), y, kc, vc, lens)
        blk.sync_status()
        want = ob.block_extend(x, W, *_oracle_args(cfg), kr, vr, L)
        assert row_err(y, want["y"]) <= _tol(cfg), (i, L, T)
        assert row_err(kc[:, :, L:L + T], want["k_new"]) <= _tol(cfg)
        kr[:, :, L:L + T], vr[:, :, L:L + T] = want["k_new"], want["v_new"]
        L += T
        assert lens.tolist() == [L] * cfg.B
    # the chunked result equals the last rows of one prefill over everything
    full = ob.block_prefill(X, W, *_oracle_args(cfg), rows=list(range(L - 5, L)))
    assert row_err(y[:, -5:], full["y"]) <= _tol(cfg)
    for s in range(2):
        x = make_decode_x(cfg, s)
        yd = torch.empty(cfg.B, 1, cfg.d, dtype=dt, device="cuda")
        blk.decode(cuda(x), yd, kc, vc, lens)
        blk.sync_status()
        want = ob.block_decode(x, W, *_oracle_args(cfg), kr, vr, [L] * cfg.B)
        assert row_err(yd, want["y"]) <= _tol(cfg)
        kr[:, :, L:L + 1], vr[:, :, L:L + 1] = want["k_new"], want["v_new"]
        L += 1
    blk.close()


def test_extend_rejects_ragged_and_overflowing_lengths():
    cfg = CFGS[0]
    W = make_weights(cfg)
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, dtype=torch.float32,
                        max_pos=64)
    blk.set_weights(weights_to_cuda(W))
    kc = torch.zeros(2, cfg.n_kv_heads, 64, cfg.head_dim, device="cuda")
    vc = torch.zeros_like(kc)
    lens = torch.tensor([3, 5], dtype=torch.int32, device="cuda")
    x = torch.zeros(2, 4, cfg.d, device="cuda")
    y = torch.empty_like(x)
    blk.set_lengths([3, 5])
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.extend(x, y, kc, vc, lens)
    assert ei.value.name == "LB_ERR_UNSUPPORTED"
    blk.set_lengths([62, 62])
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.extend(x, y, kc, vc, lens)
    assert ei.value.name == "LB_ERR_CACHE_FULL"
    blk.close()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_stack_prefill_extend_decode(dtype):
    n_layers = 3
    cfg = BlockConfig("stack", d=256, n_heads=4, n_kv_heads=2, head_dim=128 if dtype == "bf16" else 64,
                      f=512, B=2, T=1, dtype=dtype, gain="1+N(0,0.1)")
    Ws = [make_weights(cfg, seed=10 + l) for l in range(n_layers)]
    T1, T2 = 130, 45
    X = make_x(cfg, T=T1 + T2)
    t_max = T1 + T2 + 4
    dt = cfg.torch_dtype
    st = lb.LlamaStack(n_layers, cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps,
                       cfg.rope_base, dt, max_pos=t_max)
    for l in range(n_layers):
        st.set_layer_weights(l, weights_to_cuda(Ws[l]))
    kcs = [torch.zeros(cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=dt, device="cuda")
           for _ in range(n_layers)]
    vcs = [torch.zeros_like(k) for k in kcs]
    lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    y1 = torch.empty(cfg.B, T1, cfg.d, dtype=dt, device="cuda")
    st.prefill(cuda(X[:, :T1]), y1, kcs, vcs, lens)
    y2 = torch.empty(cfg.B, T2, cfg.d, dtype=dt, device="cuda")
    st.extend(cuda(X[:, T1:]), y2, kcs, vcs, lens)
    lb.llama_block_sync_status()
    torch.cuda.synchronize()
    ref = ob.stack_prefill(X, Ws, *_oracle_args(cfg))
    assert row_err(y1, ref["y"][:, :T1]) <= _tol(cfg)
    assert row_err(y2, ref["y"][:, T1:]) <= _tol(cfg)
    for l in range(n_layers):
        assert row_err(kcs[l][:, :, :T1 + T2], ref["k"][l]) <= _tol(cfg)
    assert lens.tolist() == [T1 + T2] * cfg.B
    # two decode steps through all layers, each layer on its own cache
    kr = [np.concatenate([ref["k"][l], np.zeros((cfg.B, cfg.n_kv_heads, 4, cfg.head_dim))], axis=2)
          for l in range(n_layers)]
    vr = [np.concatenate([ref["v"][l], np.zeros((cfg.B, cfg.n_kv_heads, 4, cfg.head_dim))], axis=2)
          for l in range(n_layers)]
    L = T1 + T2
    for s in range(2):
        x = make_decode_x(cfg, s)
        yd = torch.empty(cfg.B, 1, cfg.d, dtype=dt, device="cuda")
        st.decode(cuda(x), yd, kcs, vcs, lens)
        torch.cuda.synchronize()
        h = x
        for l in range(n_layers):
            out = ob.block_decode(h, Ws[l], *_oracle_args(cfg), kr[l], vr[l], [L] * cfg.B)
            kr[l][:, :, L:L + 1], vr[l][:, :, L:L + 1] = out["k_new"], out["v_new"]
            h = out["y"]
        assert row_err(yd, h) <= _tol(cfg)
        L += 1
        assert lens.tolist() == [L] * cfg.B
    st.close()


def test_stack_decode_with_int8_weights():
    """INT8 weight-only decode through a 3-layer stack: every layer against the oracle
    run on its dequantized INT8 weights."""
    n_layers = 3
    cfg = BlockConfig("stack-int8", d=256, n_heads=4, n_kv_heads=2, head_dim=128, f=512, B=2, T=1,
                      dtype="bf16")
    Ws = [make_weights(cfg, seed=20 + l) for l in range(n_layers)]
    T1 = 70
    X = make_x(cfg, T=T1)
    t_max = T1 + 4
    st = lb.LlamaStack(n_layers, cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps,
                       cfg.rope_base, torch.bfloat16, max_pos=t_max)
    for l in range(n_layers):
        st.set_layer_weights(l, weights_to_cuda(Ws[l]))
    kcs = [torch.zeros(cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
           for _ in range(n_layers)]
    vcs = [torch.zeros_like(k) for k in kcs]
    lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    y1 = torch.empty(cfg.B, T1, cfg.d, dtype=torch.bfloat16, device="cuda")
    st.prefill(cuda(X), y1, kcs, vcs, lens)  # prefill keeps the bf16 weights
    st.quantize_decode_weights()
    torch.cuda.synchronize()
    ref = ob.stack_prefill(X, Ws, *_oracle_args(cfg))
    W8s = [ob.int8_decode_weights(W) for W in Ws]
    kr = [np.concatenate([ref["k"][l], np.zeros((cfg.B, cfg.n_kv_heads, 4, cfg.head_dim))], axis=2)
          for l in range(n_layers)]
    vr = [np.concatenate([ref["v"][l], np.zeros((cfg.B, cfg.n_kv_heads, 4, cfg.head_dim))], axis=2)
          for l in range(n_layers)]
    L = T1
    for s in range(2):
        x = make_decode_x(cfg, s)
        yd = torch.empty(cfg.B, 1, cfg.d, dtype=torch.bfloat16, device="cuda")
        st.decode(cuda(x), yd, kcs, vcs, lens)
        lb.llama_block_sync_status()
        torch.cuda.synchronize()
        h = x
        for l in range(n_layers):
            out = ob.block_decode(h, W8s[l], *_oracle_args(cfg), kr[l], vr[l], [L] * cfg.B)
            kr[l][:, :, L:L + 1], vr[l][:, :, L:L + 1] = out["k_new"], out["v_new"]
            h = out["y"]
        assert row_err(yd, h) <= BF16_TOL
        L += 1
    st.close()
