"""Tensor-parallel block ("深入解析Llama MLP模块" page §6.3) on one GPU: two shard handles
(heads, KV heads and intermediate columns split in two, tp_shard_weights) stand for
two ranks; the all-reduce of each branch's partial sums is the library's tp_add of
the two partials (both shards run on one GPU), and the block output y = x + o + m must match
the fp64 oracle of the unsplit block, for a prefill and two decode steps, and every
shard's cache must hold its KV heads. The decode steps also run with INT8 weights."""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import BlockConfig, make_decode_x, make_weights, make_x
from tests.helpers import BF16_TOL, cuda, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb

CFG = BlockConfig("tp-bf16", d=512, n_heads=8, n_kv_heads=2, head_dim=64, f=1408, B=2, T=200,
                  dtype="bf16", gain="1+N(0,0.1)")
WORLD = 2


@pytest.mark.parametrize("int8", [False, True], ids=["bf16", "int8"])
def test_tp_block_matches_the_unsplit_block(int8):
    # INT8 codes quantize the weight the kernel multiplies the normalised row by (the gain
    # folded in); with unit gains that is the oracle's W
    cfg = CFG.with_(gain="ones") if int8 else CFG
    W = make_weights(cfg)
    X = make_x(cfg)
    hs, ks, fs = cfg.n_heads // WORLD, cfg.n_kv_heads // WORLD, cfg.f // WORLD
    t_max = cfg.T + 4
    dt = torch.bfloat16
    shards, caches, lens = [], [], []
    for r in range(WORLD):
        Ws = lb.tp_shard_weights(W, r, WORLD, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim)
        blk = lb.LlamaBlock(cfg.d, hs, ks, cfg.head_dim, fs, cfg.eps, cfg.rope_base, dt, max_pos=t_max)
        blk.set_weights(weights_to_cuda(Ws))
        shards.append(blk)
        kc = torch.zeros(cfg.B, ks, t_max, cfg.head_dim, dtype=dt, device="cuda")
        caches.append((kc, torch.zeros_like(kc)))
        lens.append(torch.zeros(cfg.B, dtype=torch.int32, device="cuda"))

    def layer(x, attn):
        """One TP layer over rows x: attention partials, 'all-reduce', MLP partials, 'all-reduce'."""
        o = [torch.empty_like(x) for _ in range(WORLD)]
        for r in range(WORLD):
            attn(r, o[r])
        o_sum = torch.empty_like(x)
        lb.llama_block_tp_add(o[0], o[1], o_sum)
        x1 = [torch.empty_like(x) for _ in range(WORLD)]
        m = [torch.empty_like(x) for _ in range(WORLD)]
        for r in range(WORLD):
            lb.llama_block_tp_mlp(shards[r].handle, x, o_sum, x1[r], m[r])
        assert torch.equal(x1[0], x1[1])  # every rank holds the same X'
        m_sum, y = torch.empty_like(x), torch.empty_like(x)
        lb.llama_block_tp_add(m[0], m[1], m_sum)
        lb.llama_block_tp_add(x1[0], m_sum, y)
        return y

    # prefill
    xg = cuda(X)
    y = layer(xg, lambda r, o: lb.llama_block_tp_attn_prefill(shards[r].handle, xg, o, *caches[r], lens[r]))
    lb.llama_block_sync_status()
    ref = ob.block_prefill(X, W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base)
    assert row_err(y, ref["y"]) <= BF16_TOL
    for r in range(WORLD):
        assert row_err(caches[r][0][:, :, :cfg.T], ref["k"][:, r * ks:(r + 1) * ks]) <= BF16_TOL
        assert row_err(caches[r][1][:, :, :cfg.T], ref["v"][:, r * ks:(r + 1) * ks]) <= BF16_TOL
        assert lens[r].tolist() == [cfg.T] * cfg.B
    # decode, optionally with INT8 weights in every shard
    if int8:
        for blk in shards:
            blk.quantize_decode_weights()
        W = ob.int8_decode_weights(W)
    # the oracle's own prefill K/V as the decode reference's cache
    kr = np.zeros((cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim))
    vr = np.zeros_like(kr)
    kr[:, :, :cfg.T], vr[:, :, :cfg.T] = ref["k"], ref["v"]
    L = cfg.T
    for s in range(2):
        x = make_decode_x(cfg, s)
        xg = cuda(x)
        yd = layer(xg, lambda r, o: lb.llama_block_tp_attn_decode(shards[r].handle, xg, o, *caches[r],
                                                                  lens[r]))
        lb.llama_block_sync_status()
        want = ob.block_decode(x, W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base,
                               kr, vr, [L] * cfg.B)
        assert row_err(yd, want["y"]) <= BF16_TOL
        kr[:, :, L:L + 1], vr[:, :, L:L + 1] = want["k_new"], want["v_new"]
        L += 1
        for r in range(WORLD):
            assert lens[r].tolist() == [L] * cfg.B
    for blk in shards:
        blk.close()


def test_tp_entry_points_reject_fp32_and_missing_weights():
    blk = lb.LlamaBlock(256, 2, 1, 64, 256, dtype=torch.float32, max_pos=16)
    x = torch.zeros(1, 4, 256, device="cuda")
    o = torch.empty_like(x)
    with pytest.raises(lb.LlamaBlockError) as ei:
        lb.llama_block_tp_mlp(blk.handle, x, x.clone(), torch.empty_like(x), o)
    assert ei.value.name in ("LB_ERR_UNSUPPORTED", "LB_ERR_NO_WEIGHTS")
    blk.close()
