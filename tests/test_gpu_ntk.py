"""Dynamic NTK RoPE scaling on the GPU ("LMDrive 大语言模型（LLM）核心推理单元" §2.2 names the
feature, "supports dynamic NTK scaling", without a formula: parity unpinned).

The kernels are compared with the fp64 oracle run at the base the reading gives for each
call (``oracle.block.dynamic_ntk_rope_base``, pinned by its invariants in
test_oracle.py): a prefill, an extend and decode steps that go beyond the trained
context L0, decode steps that cross it, a later short prefill on the same handle (whose
table rows the long calls had rewritten) and the switch back to plain RoPE. Besides the
block output, the post-RoPE keys the calls write are compared directly, and the test
checks that the plain base would have failed them."""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import BlockConfig, make_decode_x, make_weights, make_x
from tests.helpers import BF16_TOL, F32_TOL, cuda, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb

L0, FACTOR = 96, 2.0
CFGS = [
    BlockConfig("ntk-f32", d=256, n_heads=4, n_kv_heads=2, head_dim=64, f=512, B=2, T=150,
                dtype="f32"),
    BlockConfig("ntk-bf16", d=512, n_heads=4, n_kv_heads=2, head_dim=128, f=1408, B=2, T=200,
                dtype="bf16", gain="1+N(0,0.1)"),
]


def _tol(cfg):
    return F32_TOL if cfg.dtype == "f32" else BF16_TOL


def _base(cfg, L):
    return ob.dynamic_ntk_rope_base(cfg.rope_base, cfg.head_dim, L, L0, FACTOR)


def _new_block(cfg, W, t_max):
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps,
                        cfg.rope_base, cfg.torch_dtype, max_pos=t_max)
    blk.set_weights(weights_to_cuda(W))
    return blk


def _caches(cfg, t_max):
    kc = torch.zeros(cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=cfg.torch_dtype, device="cuda")
    return kc, torch.zeros_like(kc), torch.zeros(cfg.B, dtype=torch.int32, device="cuda")


def _prefill(cfg, blk, X, t_max):
    kc, vc, lens = _caches(cfg, t_max)
    y = torch.empty(X.shape[0], X.shape[1], cfg.d, dtype=cfg.torch_dtype, device="cuda")
    blk.prefill(cuda(X), y, kc, vc, lens)
    blk.sync_status()
    return y, kc, vc, lens


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_prefill_and_decode_beyond_the_trained_context(cfg):
    W, X = make_weights(cfg), make_x(cfg)
    T, tol = cfg.T, _tol(cfg)
    t_max = T + 8
    blk = _new_block(cfg, W, t_max)
    blk.set_rope_dynamic_ntk(FACTOR, L0)
    y, kc, vc, lens = _prefill(cfg, blk, X, t_max)
    args = (cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps)
    ref = ob.block_prefill(X, W, *args, _base(cfg, T))
    assert row_err(y, ref["y"]) <= tol
    assert row_err(kc[:, :, :T], ref["k"]) <= tol
    plain = ob.block_prefill(X, W, *args, cfg.rope_base)
    assert row_err(kc[:, :, :T], plain["k"]) > 10 * tol  # the two bases are told apart
    # decode: each step rotates its token with the base of the length it reaches
    kr = np.zeros((cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim))
    vr = np.zeros_like(kr)
    kr[:, :, :T], vr[:, :, :T] = ref["k"], ref["v"]
    L = T
    for s in range(2):
        x = make_decode_x(cfg, s)
        yd = torch.empty(cfg.B, 1, cfg.d, dtype=cfg.torch_dtype, device="cuda")
        blk.decode(cuda(x), yd, kc, vc, lens)
        blk.sync_status()
        want = ob.block_decode(x, W, *args, _base(cfg, L + 1), kr, vr, [L] * cfg.B)
        assert row_err(yd, want["y"]) <= tol
        assert row_err(kc[:, :, L:L + 1], want["k_new"]) <= tol
        kr[:, :, L:L + 1], vr[:, :, L:L + 1] = want["k_new"], want["v_new"]
        L += 1
    # a short prefill on the same handle reads table rows the long calls rewrote: plain base
    Xs = X[:, :64].contiguous()
    ys, kcs, _, _ = _prefill(cfg, blk, Xs, t_max)
    short = ob.block_prefill(Xs, W, *args, cfg.rope_base)
    assert row_err(ys, short["y"]) <= tol
    assert row_err(kcs[:, :, :64], short["k"]) <= tol
    # switched off: the long prefill is plain RoPE again
    blk.set_rope_dynamic_ntk(0.0, 0)
    y2, kc2, _, _ = _prefill(cfg, blk, X, t_max)
    assert row_err(y2, plain["y"]) <= tol
    assert row_err(kc2[:, :, :T], plain["k"]) <= tol
    blk.close()


def test_extend_and_decode_across_the_trained_context():
    """Chunked prefill up to L0 - 1 tokens is plain RoPE; the next chunk and the decode
    steps past L0 use the base of the length each call reaches."""
    cfg = CFGS[1].with_(name="ntk-cross", B=1)
    W = make_weights(cfg)
    T1, T2 = L0 - 1, 40
    X = make_x(cfg, T=T1 + T2)
    t_max = T1 + T2 + 8
    blk = _new_block(cfg, W, t_max)
    blk.set_rope_dynamic_ntk(FACTOR, L0)
    args = (cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps)
    y1, kc, vc, lens = _prefill(cfg, blk, X[:, :T1].contiguous(), t_max)
    ref1 = ob.block_prefill(X[:, :T1], W, *args, cfg.rope_base)  # T1 < L0: plain
    assert row_err(y1, ref1["y"]) <= BF16_TOL
    kr = np.zeros((cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim))
    vr = np.zeros_like(kr)
    kr[:, :, :T1], vr[:, :, :T1] = ref1["k"], ref1["v"]
    y2 = torch.empty(cfg.B, T2, cfg.d, dtype=cfg.torch_dtype, device="cuda")
    blk.extend(cuda(X[:, T1:].contiguous()), y2, kc, vc, lens)
    blk.sync_status()
    ref2 = ob.block_extend(X[:, T1:], W, *args, _base(cfg, T1 + T2), kr, vr, T1)
    assert row_err(y2, ref2["y"]) <= BF16_TOL
    assert row_err(kc[:, :, T1:T1 + T2], ref2["k_new"]) <= BF16_TOL
    # the cached prefix keeps its plain rotation
    assert row_err(kc[:, :, :T1], ref1["k"]) <= BF16_TOL
    kr[:, :, T1:T1 + T2], vr[:, :, T1:T1 + T2] = ref2["k_new"], ref2["v_new"]
    L = T1 + T2
    x = make_decode_x(cfg, 0)
    yd = torch.empty(cfg.B, 1, cfg.d, dtype=cfg.torch_dtype, device="cuda")
    blk.decode(cuda(x), yd, kc, vc, lens)
    blk.sync_status()
    want = ob.block_decode(x, W, *args, _base(cfg, L + 1), kr, vr, [L] * cfg.B)
    assert row_err(yd, want["y"]) <= BF16_TOL
    assert row_err(kc[:, :, L:L + 1], want["k_new"]) <= BF16_TOL
    blk.close()


def test_rejects_bad_scaling_arguments():
    cfg = CFGS[0]
    blk = _new_block(cfg, make_weights(cfg), 64)
    for factor, orig in ((0.5, 32), (float("nan"), 32), (2.0, -1)):
        with pytest.raises(lb.LlamaBlockError) as ei:
            blk.set_rope_dynamic_ntk(factor, orig)
        assert ei.value.name == "LB_ERR_INVALID_ARG"
    blk.close()
