"""GPU parity of the INT8 weight-only decode path (llama_block_quantize_decode_weights):
per-output-row symmetric INT8 codes of every projection (the Llama MLP page §6.4
INT8 weights), decode steps compared with the fp64 oracle run on the dequantized
weights (oracle.block.int8_decode_weights).

INT8 rounding noise alone moves a decode row by about 1e-2 of its max-norm, half
the bf16 tolerance, so agreement with the INT8 oracle does not show that the INT8
weights were used. The per-GEMM cases therefore plant one outlier per row in one
weight group (each row's outlier in a different column), which makes the INT8 and
the bf16 results of the oracle differ by two tolerances or more; the GPU must match
the INT8 one and miss the bf16 one. A further case makes both paths form the same
products exactly and asks for agreement to the rounding of the outputs.

The projections have std 0.15 so that the branches, not the residual, dominate y;
W_q and W_k keep std 0.02, since larger q and k make the softmax so sharp that bf16
storage of q and k alone moves y by more than a tolerance.
"""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import BlockConfig, make_cache, make_decode_x, make_weights
from tests.helpers import BF16_TOL, as_np, cuda, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb

# d = 1024 (12 full tiles of the fused QKV rows, 8 of o_proj), f = 2816 (44 tiles of
# the interleaved gate/up rows)
CFG = BlockConfig("w8", d=1024, n_heads=8, n_kv_heads=2, head_dim=128, f=2816, B=4, T=1,
                  dtype="bf16", cache_len=200, weight_std=0.15)
# ragged everywhere: 5 heads of 64 (QKV rows 960 = 7.5 tiles, d = 320 = 2.5 tiles),
# f = 704, the maximum INT8 batch of 32, no GQA
CFG_RAGGED = BlockConfig("w8-ragged", d=320, n_heads=5, n_kv_heads=5, head_dim=64, f=704, B=32,
                         T=1, dtype="bf16", cache_len=150)
GROUPS = {"qkv": ("wq", "wk", "wv"), "o": ("wo",), "gate_up": ("w_gate", "w_up"),
          "down": ("w_down",)}
QK_STD = 0.02


def _weights(cfg, seed=0):
    W = make_weights(cfg, seed=seed)
    for k in ("wq", "wk"):
        W[k] = (W[k].double() * (QK_STD / cfg.weight_std)).to(W[k].dtype)
    return W


def _std(cfg, key):
    return QK_STD if key in ("wq", "wk") else cfg.weight_std


def _outliers(w, std):
    """Row r gets +-sqrt(in) * std at column 7r mod in (sign alternating by row)."""
    w = w.clone()
    o, i = w.shape
    r = torch.arange(o)
    sign = torch.where(r % 2 == 0, 1.0, -1.0)
    w[r, (r * 7) % i] = (i ** 0.5 * std * sign).to(w.dtype)
    return w


def _lens(cfg):
    return [cfg.cache_len - (37 * b) % (cfg.cache_len // 2) for b in range(cfg.B)]


def _run(cfg, W, quantize, steps=2, W_after=None):
    """Decode `steps` tokens on caller-filled caches of ragged lengths; returns the
    per-step GPU outputs and the per-step oracle outputs for INT8 and bf16 weights
    (both oracles follow the GPU-independent cache recurrence of their own)."""
    lens0 = _lens(cfg)
    t_max = cfg.cache_len + steps + 4
    k0, v0 = make_cache(cfg, t_max)
    for b, L in enumerate(lens0):
        k0[b, :, L:] = 0
        v0[b, :, L:] = 0
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps,
                        cfg.rope_base, cfg.torch_dtype, max_pos=t_max)
    blk.set_weights(weights_to_cuda(W))
    if quantize:
        blk.quantize_decode_weights()
    if W_after is not None:  # set_weights after enabling re-quantizes
        blk.set_weights(weights_to_cuda(W_after))
        W = W_after
    kc, vc = cuda(k0), cuda(v0)
    lens = torch.tensor(lens0, dtype=torch.int32, device="cuda")
    blk.set_lengths(lens0)
    W8 = ob.int8_decode_weights(W)
    args = (cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base)
    caches = {"w8": (as_np(k0), as_np(v0)), "bf16": (as_np(k0), as_np(v0))}
    cur = list(lens0)
    out = []
    for s in range(steps):
        x = make_decode_x(cfg, s)
        y = torch.empty(cfg.B, 1, cfg.d, dtype=cfg.torch_dtype, device="cuda")
        blk.decode(cuda(x), y, kc, vc, lens)
        blk.sync_status()
        k_new = torch.stack([kc[b, :, cur[b]] for b in range(cfg.B)])[:, :, None]
        want = {}
        for name, Wx in (("w8", W8), ("bf16", W)):
            kr, vr = caches[name]
            want[name] = ob.block_decode(x, Wx, *args, kr, vr, cur)
            for b in range(cfg.B):
                kr[b, :, cur[b]] = want[name]["k_new"][b, :, 0]
                vr[b, :, cur[b]] = want[name]["v_new"][b, :, 0]
        out.append((y, k_new, want))
        cur = [c + 1 for c in cur]
        assert lens.tolist() == cur
    blk.close()
    return out


def _int8_exact(w, gen):
    """A weight matrix that INT8 represents exactly: w = 2^-9 q, q ~ N(0, 20) rounded
    and clipped to [-126, 126], one element per row at +-127 (so s = 2^-9 exactly)."""
    o, i = w.shape
    q = torch.clamp(torch.round(torch.randn(o, i, generator=gen, dtype=torch.float64) * 20), -126, 126)
    r = torch.arange(o)
    q[r, (r * 11) % i] = torch.where(r % 2 == 0, 127.0, -127.0).double()
    return (q * 2.0 ** -9).to(w.dtype)


def test_int8_path_matches_bf16_path_on_int8_exact_weights():
    """On weights with exact INT8 codes and power-of-two row scales the INT8 GEMMs form
    the same products as the bf16 GEMMs and the scale is exact; only the fp32 summation
    order may differ (the INT8 GEMM splits K in 128-deep blocks, the bf16 one in 64-deep
    blocks). So every stored K row agrees to one bf16 rounding, and y to a few."""
    cfg = CFG.with_(weight_std=0.02)
    W = make_weights(cfg)
    gen = torch.Generator().manual_seed(77)
    for k in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
        W[k] = _int8_exact(W[k], gen)
    q8, s8 = ob.quantize_int8_rows(W["w_down"])
    assert np.all(s8 == np.float32(2.0 ** -9))
    assert np.array_equal(ob.dequantize_int8_rows(q8, s8), as_np(W["w_down"]))
    (y16, k16, want), = _run(cfg, W, quantize=False, steps=1)
    (y8, k8, _), = _run(cfg, W, quantize=True, steps=1)
    ulp = 2.0 ** -7  # relative spacing bound of bf16 normals
    assert torch.all((k8.float() - k16.float()).abs() <= ulp * k16.float().abs() + 1e-30)
    assert row_err(y8, y16.double().cpu().numpy()) <= 4e-3
    assert (y8 == y16).double().mean().item() >= 0.5
    assert row_err(y8, want["w8"]["y"]) <= BF16_TOL


@pytest.mark.parametrize("cfg", [CFG, CFG_RAGGED], ids=lambda c: c.name)
def test_int8_decode_matches_oracle(cfg):
    for y, k_new, want in _run(cfg, _weights(cfg), quantize=True):
        assert row_err(y, want["w8"]["y"]) <= BF16_TOL
        assert row_err(k_new, want["w8"]["k_new"]) <= BF16_TOL


@pytest.mark.parametrize("group", list(GROUPS))
def test_int8_decode_uses_int8_weights_of_each_gemm(group):
    W = _weights(CFG)
    for k in GROUPS[group]:
        W[k] = _outliers(W[k], _std(CFG, k))
    for y, k_new, want in _run(CFG, W, quantize=True, steps=1):
        sep = row_err(want["w8"]["y"], want["bf16"]["y"])
        assert sep >= 2 * BF16_TOL  # the case separates INT8 from bf16 weights
        assert row_err(y, want["w8"]["y"]) <= BF16_TOL
        assert row_err(y, want["bf16"]["y"]) > BF16_TOL
        if group == "qkv":
            assert row_err(k_new, want["w8"]["k_new"]) <= BF16_TOL


def test_int8_requantizes_on_set_weights_and_can_be_disabled():
    W0 = _weights(CFG)
    W1 = _weights(CFG, seed=5)
    for k in GROUPS["down"] + GROUPS["qkv"]:
        W1[k] = _outliers(W1[k], _std(CFG, k))
    (y, _, want), = _run(CFG, W0, quantize=True, steps=1, W_after=W1)
    assert row_err(want["w8"]["y"], want["bf16"]["y"]) >= 2 * BF16_TOL
    assert row_err(y, want["w8"]["y"]) <= BF16_TOL
    assert row_err(y, want["bf16"]["y"]) > BF16_TOL
    # disabled again: the bf16 weights
    (y, _, want), = _run(CFG, W1, quantize=False, steps=1)
    assert row_err(y, want["bf16"]["y"]) <= BF16_TOL


def test_int8_batches_above_32_decode_with_bf16_weights():
    cfg = CFG.with_(B=33, cache_len=64)
    W = _weights(cfg)
    W["w_down"] = _outliers(W["w_down"], cfg.weight_std)
    (y, _, want), = _run(cfg, W, quantize=True, steps=1)
    assert row_err(want["w8"]["y"], want["bf16"]["y"]) >= 2 * BF16_TOL
    assert row_err(y, want["bf16"]["y"]) <= BF16_TOL


def test_int8_rejected_for_f32_and_without_weights():
    cfg = CFG.with_(dtype="f32")
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, dtype=torch.float32,
                        max_pos=16)
    blk.set_weights(weights_to_cuda(make_weights(cfg)))
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.quantize_decode_weights()
    assert ei.value.name == "LB_ERR_UNSUPPORTED"
    blk.close()
    blk = lb.LlamaBlock(CFG.d, CFG.n_heads, CFG.n_kv_heads, CFG.head_dim, CFG.f, dtype=torch.bfloat16,
                        max_pos=16)
    with pytest.raises(lb.LlamaBlockError) as ei:
        blk.quantize_decode_weights()
    assert ei.value.name == "LB_ERR_NO_WEIGHTS"
    blk.close()
