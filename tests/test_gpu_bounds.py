"""Out-of-bounds write checks (canaries) and GQA/MHA equivalence on the GPU.

Every buffer the library writes is carved from a larger, sentinel-filled allocation;
after prefill, extend and decode, everything outside the elements the call owns
(the output rows, and the cache positions of the new tokens) must be bit-for-bit
what it was: the sentinel past the end of a buffer, and the untouched cache rows.
Shapes are ragged (T not a multiple of the 128-row tiles, GQA, head_dim 64 and 128)
so that the tails of every kernel are exercised.

GQA (LMDrive page §2.3, repeat_kv): a block with n_kv_heads < n_heads must give the
result of the block whose K/V projections repeat each KV head n_rep times.
"""

import pytest
import torch

from synth import BlockConfig, make_decode_x, make_weights, make_x
from tests.helpers import BF16_TOL, F32_TOL, cuda, row_err, weights_to_cuda

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb

PAD = 4096  # sentinel elements after every buffer


def _guarded(shape, dtype, fill_bits):
    """A tensor of `shape` at the start of a larger allocation whose every element
    (the tensor's own too) holds the bit pattern `fill_bits`."""
    n = 1
    for s in shape:
        n *= s
    int_t = torch.int16 if dtype == torch.bfloat16 else torch.int32
    raw = torch.full((n + PAD,), fill_bits, dtype=int_t, device="cuda")
    return raw, raw.view(dtype)[:n].view(*shape)


def _tail_intact(raw, n, fill_bits):
    return bool(torch.all(raw[n:] == fill_bits).item())


CFGS = [
    BlockConfig("bounds-bf16-gqa", d=512, n_heads=8, n_kv_heads=2, head_dim=64, f=1408, B=2, T=200,
                dtype="bf16"),
    BlockConfig("bounds-bf16-dh128", d=256, n_heads=2, n_kv_heads=1, head_dim=128, f=704, B=3, T=77,
                dtype="bf16"),
    BlockConfig("bounds-f32", d=256, n_heads=4, n_kv_heads=2, head_dim=64, f=512, B=2, T=50,
                dtype="f32"),
]


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_calls_write_only_their_own_elements(cfg):
    dt = cfg.torch_dtype
    bits = 0x7BCD if dt == torch.bfloat16 else 0x7BCD1234  # finite, unlikely values
    W = make_weights(cfg)
    T1, T2 = cfg.T, 29
    t_max = T1 + T2 + 8
    X = make_x(cfg, T=T1 + T2)
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base,
                        dt, max_pos=t_max)
    blk.set_weights(weights_to_cuda(W))
    shape_c = (cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim)
    kraw, kc = _guarded(shape_c, dt, bits)
    vraw, vc = _guarded(shape_c, dt, bits)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    n_c = kc.numel()

    def check_cache(written_upto):
        # positions >= written_upto of every (sequence, head) still hold the sentinel
        for c in (kc, vc):
            rest = c[:, :, written_upto:].contiguous().view(torch.int16 if dt == torch.bfloat16 else torch.int32)
            assert bool(torch.all(rest == bits).item()), written_upto
        assert _tail_intact(kraw, n_c, bits) and _tail_intact(vraw, n_c, bits)

    # prefill of T1 tokens
    yraw, y = _guarded((cfg.B, T1, cfg.d), dt, bits)
    blk.prefill(cuda(X[:, :T1].contiguous()), y, kc, vc, lens)
    blk.sync_status()
    assert _tail_intact(yraw, y.numel(), bits)
    assert torch.isfinite(y.float()).all()
    check_cache(T1)
    # extend by T2 tokens: rows [0, T1) of the cache must not change
    before = (kc[:, :, :T1].clone(), vc[:, :, :T1].clone())
    y2raw, y2 = _guarded((cfg.B, T2, cfg.d), dt, bits)
    blk.extend(cuda(X[:, T1:].contiguous()), y2, kc, vc, lens)
    blk.sync_status()
    assert _tail_intact(y2raw, y2.numel(), bits)
    assert torch.equal(kc[:, :, :T1], before[0]) and torch.equal(vc[:, :, :T1], before[1])
    check_cache(T1 + T2)
    # two decode steps: each writes exactly position L of every sequence
    L = T1 + T2
    for s in range(2):
        before = (kc[:, :, :L].clone(), vc[:, :, :L].clone())
        ydraw, yd = _guarded((cfg.B, 1, cfg.d), dt, bits)
        blk.decode(cuda(make_decode_x(cfg, s)), yd, kc, vc, lens)
        blk.sync_status()
        assert _tail_intact(ydraw, yd.numel(), bits)
        assert torch.equal(kc[:, :, :L], before[0]) and torch.equal(vc[:, :, :L], before[1])
        L += 1
        check_cache(L)
        assert lens.tolist() == [L] * cfg.B
    blk.close()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gqa_block_equals_mha_block_with_repeated_kv_heads(dtype):
    cfg = BlockConfig("gqa", d=512, n_heads=8, n_kv_heads=2, head_dim=64, f=1024, B=2, T=150,
                      dtype=dtype, gain="1+N(0,0.1)")
    n_rep = cfg.n_heads // cfg.n_kv_heads
    W = make_weights(cfg)
    Wm = dict(W)
    for k in ("wk", "wv"):  # KV head j of the MHA block = KV head j // n_rep of the GQA one
        Wm[k] = W[k].view(cfg.n_kv_heads, cfg.head_dim, cfg.d).repeat_interleave(n_rep, dim=0).reshape(
            cfg.n_heads * cfg.head_dim, cfg.d).contiguous()
    X = cuda(make_x(cfg))
    dt = cfg.torch_dtype
    out = {}
    for name, w, hkv in (("gqa", W, cfg.n_kv_heads), ("mha", Wm, cfg.n_heads)):
        blk = lb.LlamaBlock(cfg.d, cfg.n_heads, hkv, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base, dt,
                            max_pos=cfg.T + 2)
        blk.set_weights(weights_to_cuda(w))
        kc = torch.zeros(cfg.B, hkv, cfg.T + 2, cfg.head_dim, dtype=dt, device="cuda")
        vc = torch.zeros_like(kc)
        lens = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
        y = torch.empty(cfg.B, cfg.T, cfg.d, dtype=dt, device="cuda")
        blk.prefill(X, y, kc, vc, lens)
        yd = torch.empty(cfg.B, 1, cfg.d, dtype=dt, device="cuda")
        blk.decode(cuda(make_decode_x(cfg, 0)), yd, kc, vc, lens)
        blk.sync_status()
        out[name] = (y, yd, kc)
        blk.close()
    tol = BF16_TOL / 4 if dtype == "bf16" else F32_TOL
    assert row_err(out["gqa"][0], out["mha"][0].double().cpu().numpy()) <= tol
    assert row_err(out["gqa"][1], out["mha"][1].double().cpu().numpy()) <= tol
    # the MHA cache holds each GQA KV head n_rep times
    rep = out["gqa"][2].repeat_interleave(n_rep, dim=1)
    assert row_err(rep, out["mha"][2].double().cpu().numpy()) <= tol
