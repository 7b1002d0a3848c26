"""GPU parity of the whole block (prefill and KV-cache decode) against the fp64
oracle, at sizes the oracle evaluates in seconds: several tiles with ragged
tails, MHA and GQA, head_dim 64 and 128, fp32 and bf16.

Besides the block output X'' (the stated tolerance: fp32 1e-4 relative, bf16
2e-2 per-row max-norm), the tests compare the KV cache the prefill writes
(post-RoPE K and V) and the residual-free branch sum X'' - X, so that an error
in a branch cannot hide behind the residual stream."""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import BlockConfig, TINY_F32, make_cache, make_decode_x, make_weights, make_x
from tests.helpers import BF16_TOL, F32_TOL, as_np, branch_err, cuda, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb


SMALL_BF16 = [
    BlockConfig("bf16-gqa", d=512, n_heads=4, n_kv_heads=2, head_dim=128, f=1408, B=2, T=200,
                dtype="bf16", gain="1+N(0,0.1)"),
    BlockConfig("bf16-dh64", d=256, n_heads=4, n_kv_heads=4, head_dim=64, f=704, B=1, T=129,
                dtype="bf16"),
    BlockConfig("bf16-rep8", d=1024, n_heads=8, n_kv_heads=1, head_dim=128, f=2816, B=1, T=384,
                dtype="bf16", gain="1+N(0,0.1)"),
]

# GQA groupings outside {1, 2, 4, 8} (repeat_kv allows any n_rep = H / H_kv): the decode
# attention then serves one (n_rep = 3) or two (n_rep = 6) query heads per CTA, or all
# 16 with eight per CTA
GQA_ANY = [
    BlockConfig("bf16-rep3", d=512, n_heads=6, n_kv_heads=2, head_dim=64, f=1024, B=2, T=150,
                dtype="bf16", gain="1+N(0,0.1)"),
    BlockConfig("bf16-rep6", d=768, n_heads=12, n_kv_heads=2, head_dim=64, f=1024, B=1, T=300,
                dtype="bf16"),
    BlockConfig("bf16-rep16", d=1024, n_heads=16, n_kv_heads=1, head_dim=64, f=1536, B=1, T=200,
                dtype="bf16"),
    BlockConfig("f32-rep3", d=384, n_heads=6, n_kv_heads=2, head_dim=64, f=512, B=1, T=70,
                dtype="f32", gain="1+N(0,0.1)"),
]


def _oracle_prefill(cfg, X, W):
    return ob.block_prefill(X, W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base)


def _run_prefill(cfg, X, W, t_max):
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps,
                        cfg.rope_base, cfg.torch_dtype, max_pos=t_max + 8)
    blk.set_weights(weights_to_cuda(W))
    dt = cfg.torch_dtype
    kc = torch.zeros(cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=dt, device="cuda")
    vc = torch.zeros_like(kc)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    y = torch.empty(cfg.B, cfg.T, cfg.d, dtype=dt, device="cuda")
    blk.prefill(cuda(X), y, kc, vc, lens)
    blk.sync_status()
    return blk, y, kc, vc, lens


def _tol(cfg):
    return F32_TOL if cfg.dtype == "f32" else BF16_TOL


def _check(cfg, got, want):
    assert row_err(got, want) <= _tol(cfg)


@pytest.mark.parametrize("cfg", [TINY_F32] + SMALL_BF16 + GQA_ANY, ids=lambda c: c.name)
def test_block_prefill(cfg):
    W = make_weights(cfg)
    X = make_x(cfg)
    t_max = cfg.T + 16
    blk, y, kc, vc, lens = _run_prefill(cfg, X, W, t_max)
    ref = _oracle_prefill(cfg, X, W)
    _check(cfg, y, ref["y"])
    _check(cfg, kc[:, :, :cfg.T], ref["k"])
    _check(cfg, vc[:, :, :cfg.T], ref["v"])
    u = 2.0 ** -24 if cfg.dtype == "f32" else 2.0 ** -8
    assert branch_err(y, ref["y"], ref["x1"], ref["attn"] + ref["mlp"], u) <= _tol(cfg)
    assert lens.tolist() == [cfg.T] * cfg.B
    blk.close()


@pytest.mark.parametrize("cfg", [TINY_F32.with_(B=2, T=40)] + SMALL_BF16[:2] + GQA_ANY,
                         ids=lambda c: c.name)
def test_block_decode_after_prefill(cfg):
    """Prefill T tokens, then decode 3 tokens; each decode output equals the
    oracle's decode (and hence the last row of a full recompute)."""
    W = make_weights(cfg)
    X = make_x(cfg, T=cfg.T + 3)
    t_max = cfg.T + 8
    pre = cfg.with_(T=cfg.T)
    blk, y, kc, vc, lens = _run_prefill(pre, X[:, :cfg.T].contiguous(), W, t_max)
    ref = _oracle_prefill(pre, X[:, :cfg.T], W)
    kr = np.zeros((cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim))
    vr = np.zeros_like(kr)
    kr[:, :, :cfg.T], vr[:, :, :cfg.T] = ref["k"], ref["v"]
    for s in range(3):
        L = cfg.T + s
        x = X[:, L:L + 1].contiguous()
        yd = torch.empty(cfg.B, 1, cfg.d, dtype=cfg.torch_dtype, device="cuda")
        blk.decode(cuda(x), yd, kc, vc, lens)
        blk.sync_status()
        want = ob.block_decode(x, W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps,
                               cfg.rope_base, kr, vr, [L] * cfg.B)
        _check(cfg, yd, want["y"])
        _check(cfg, kc[:, :, L:L + 1], want["k_new"])
        kr[:, :, L:L + 1], vr[:, :, L:L + 1] = want["k_new"], want["v_new"]
        assert lens.tolist() == [L + 1] * cfg.B
    # and the last decode equals the last row of a full prefill over T+3 tokens
    full = _oracle_prefill(cfg.with_(T=cfg.T + 3), X, W)
    _check(cfg, yd, full["y"][:, -1:])
    blk.close()


@pytest.mark.parametrize("lens0", [[5, 130, 257], [0, 1, 300]], ids=["ragged", "from-empty"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_decode_ragged_lengths(dtype, lens0):
    """Caller-filled caches of different lengths per sequence (set_lengths); a sequence
    of length 0 decodes its first token, which attends to itself alone."""
    cfg = BlockConfig("ragged", d=256, n_heads=4, n_kv_heads=2, head_dim=64, f=512, B=3, T=1,
                      dtype=dtype, cache_len=300, gain="1+N(0,0.1)")
    t_max = 320
    W = make_weights(cfg)
    k0, v0 = make_cache(cfg, t_max)
    for b, L in enumerate(lens0):  # zero beyond each sequence's length
        k0[b, :, L:] = 0
        v0[b, :, L:] = 0
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps,
                        cfg.rope_base, cfg.torch_dtype, max_pos=t_max)
    blk.set_weights(weights_to_cuda(W))
    kc, vc = cuda(k0), cuda(v0)
    lens = torch.tensor(lens0, dtype=torch.int32, device="cuda")
    blk.set_lengths(lens0)
    kr, vr = as_np(k0), as_np(v0)
    cur = list(lens0)
    for s in range(2):
        x = make_decode_x(cfg, s)
        y = torch.empty(cfg.B, 1, cfg.d, dtype=cfg.torch_dtype, device="cuda")
        blk.decode(cuda(x), y, kc, vc, lens)
        blk.sync_status()
        want = ob.block_decode(x, W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps,
                               cfg.rope_base, kr, vr, cur)
        _check(cfg, y, want["y"])
        for b in range(cfg.B):
            kr[b, :, cur[b]], vr[b, :, cur[b]] = want["k_new"][b, :, 0], want["v_new"][b, :, 0]
            cur[b] += 1
        assert lens.tolist() == cur
    blk.close()


def test_cache_full_and_missing_lengths_are_rejected_on_host():
    cfg = TINY_F32.with_(B=1, T=8)
    W = make_weights(cfg)
    blk, y, kc, vc, lens = _run_prefill(cfg, make_x(cfg), W, t_max=8)  # cache exactly full
    x = torch.zeros(1, 1, cfg.d, device="cuda")
    yd = torch.empty_like(x)
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.decode(x, yd, kc, vc, lens)
    assert ei.value.name == "LB_ERR_CACHE_FULL"
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.decode(torch.zeros(2, 1, cfg.d, device="cuda"), torch.empty(2, 1, cfg.d, device="cuda"),
                   kc, vc, lens)
    assert ei.value.name == "LB_ERR_INVALID_ARG"
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.prefill(cuda(make_x(cfg, T=9)), torch.empty(1, 9, cfg.d, device="cuda"), kc, vc, lens)
    assert ei.value.name == "LB_ERR_CACHE_FULL"
    blk.close()
    fresh = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, dtype=torch.float32,
                          max_pos=16)
    with pytest.raises(lb.LlamaBlockError) as ei:
        fresh.prefill(cuda(make_x(cfg)), torch.empty(1, 8, cfg.d, device="cuda"), kc, vc, lens)
    assert ei.value.name == "LB_ERR_NO_WEIGHTS"
    fresh.close()


def test_calls_leave_the_current_device_unchanged():
    """Handle calls select the handle's device for their duration and restore the
    caller's (with one GPU both are device 0; the call must not disturb it)."""
    cfg = TINY_F32.with_(B=1, T=8)
    before = torch.cuda.current_device()
    blk, y, kc, vc, lens = _run_prefill(cfg, make_x(cfg), make_weights(cfg), t_max=16)
    blk.sync_status()
    assert torch.cuda.current_device() == before
    blk.close()
    assert torch.cuda.current_device() == before
