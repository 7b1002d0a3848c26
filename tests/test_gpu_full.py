"""GPU parity at the full workload sizes, in the launch configuration bench.py
times (the handle's prefill / decode through the C ABI, bf16):

  * LLaMA-7B-shaped prefill (B=1, T=2048), 13B-shaped (B=4, T=1024) and the
    70B-shaped GQA block (64 query / 8 KV heads, T=4096),
  * two KV-cache decode steps of the 7B-, 13B- and 70B-shaped blocks with B=32 and
    4096 cached positions, and of the 7B-shaped block with INT8 weights.

The oracle evaluates sampled outputs: 64 token rows per sequence (first, last
and 62 seeded-random rows; K and V are projected for every token since
attention needs them) for prefill, and 4 of the 32 sequences for decode
(sequences are independent). The KV cache written by prefill is compared at
the sampled positions."""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import DECODE7B, LLAMA13B, LLAMA70B, LLAMA7B, make_cache, make_decode_x, make_weights, make_x, sample_rows
from tests.helpers import BF16_TOL, as_np, branch_err, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb


@pytest.mark.parametrize("cfg", [LLAMA7B, LLAMA13B, LLAMA70B], ids=lambda c: c.name)
def test_full_size_prefill_sampled_rows(cfg):
    W = make_weights(cfg)
    X = make_x(cfg)
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base,
                        torch.bfloat16, max_pos=cfg.T)
    blk.set_weights(weights_to_cuda(W))
    kc = torch.zeros(cfg.B, cfg.n_kv_heads, cfg.T, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    y = torch.empty(cfg.B, cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    blk.prefill(X.cuda(), y, kc, vc, lens)
    blk.sync_status()
    rows = sample_rows(cfg.T, 64, seed=11)
    ref = ob.block_prefill(X, W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base, rows=rows)
    got = y[:, rows]
    e_y = row_err(got, ref["y"])
    e_k = row_err(kc[:, :, rows], ref["k"][:, :, rows])
    e_v = row_err(vc[:, :, rows], ref["v"][:, :, rows])
    e_b = branch_err(got, ref["y"], ref["x1"], ref["attn"] + ref["mlp"])
    print(f"{cfg.name}: y {e_y:.2e}  k {e_k:.2e}  v {e_v:.2e}  branch {e_b:.2e}")
    assert e_y <= BF16_TOL and e_k <= BF16_TOL and e_v <= BF16_TOL and e_b <= BF16_TOL
    assert lens.tolist() == [cfg.T] * cfg.B
    blk.close()


DECODE_CFGS = [
    DECODE7B,
    # the 13B and the 70B GQA blocks in the same decode setting (B=32, 4096 cached
    # positions); the 70B one runs the n_rep = 8 decode attention at full size
    LLAMA13B.with_(name="llama13b-decode", B=32, T=1, cache_len=4096, decode_steps=2),
    LLAMA70B.with_(name="llama70b-gqa-decode", B=32, T=1, cache_len=4096, decode_steps=2),
]


@pytest.mark.parametrize("cfg,int8", [(c, False) for c in DECODE_CFGS] + [(DECODE7B, True)],
                         ids=lambda v: v.name if hasattr(v, "name") else ("int8" if v else "bf16"))
def test_full_size_decode_step(cfg, int8):
    """Two decode steps; with int8, the INT8 weight-only path against the oracle run on
    the dequantized weights."""
    t_max = cfg.cache_len + 2
    W = make_weights(cfg)
    k0, v0 = make_cache(cfg, t_max)
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base,
                        torch.bfloat16, max_pos=t_max)
    blk.set_weights(weights_to_cuda(W))
    if int8:
        blk.quantize_decode_weights()
        W = ob.int8_decode_weights(W)
    kc, vc = k0.cuda(), v0.cuda()
    seqs = [0, 9, 22, 31]
    L = cfg.cache_len
    kr = as_np(k0[seqs, :, :L + 2])  # the oracle's cache: the synthetic host data
    vr = as_np(v0[seqs, :, :L + 2])
    del k0, v0
    lens = torch.full((cfg.B,), cfg.cache_len, dtype=torch.int32, device="cuda")
    blk.set_lengths([cfg.cache_len] * cfg.B)
    for s in range(2):
        x = make_decode_x(cfg, s)
        y = torch.empty(cfg.B, 1, cfg.d, dtype=torch.bfloat16, device="cuda")
        blk.decode(x.cuda(), y, kc, vc, lens)
        blk.sync_status()
        want = ob.block_decode(x[seqs], W, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps,
                               cfg.rope_base, kr, vr, [L + s] * len(seqs))
        e_y = row_err(y[seqs], want["y"])
        e_k = row_err(kc[seqs, :, L + s:L + s + 1], want["k_new"])
        e_v = row_err(vc[seqs, :, L + s:L + s + 1], want["v_new"])
        e_b = branch_err(y[seqs], want["y"], want["x1"], want["attn"] + want["mlp"])
        print(f"{cfg.name} {'int8' if int8 else 'bf16'} step {s}: y {e_y:.2e}  k {e_k:.2e}  "
              f"v {e_v:.2e}  branch {e_b:.2e}")
        assert e_y <= BF16_TOL and e_k <= BF16_TOL and e_v <= BF16_TOL and e_b <= BF16_TOL
        kr[:, :, L + s:L + s + 1], vr[:, :, L + s:L + s + 1] = want["k_new"], want["v_new"]
        assert lens.tolist() == [L + s + 1] * cfg.B
    blk.close()
