"""GPU parity of the standalone entry points against the fp64 oracle.

Each test feeds the same seeded inputs (rounded to the compute dtype) to the
C ABI (through the ctypes binding) and to ``oracle/``, and compares element by
element: fp32 within 1e-4 relative, bf16 within 2e-2 per-row max-norm. Sizes
span several tiles with ragged tails."""

import numpy as np
import pytest
import torch

from oracle import block as ob
from synth import make_tensor
from tests.helpers import BF16_TOL, F32_TOL, as_np, cuda, row_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import llama_pre_norm_b200 as lb


def _tol(dt):
    return F32_TOL if dt == torch.float32 else BF16_TOL


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,d", [(1, 256), (7, 4096), (33, 5120), (5, 8192), (3, 8)])
def test_rmsnorm(dt, rows, d):
    x = make_tensor((rows, d), 100 + d, dt, std=2.0)
    g = make_tensor((d,), 200 + d, dt, std=0.1, mean=1.0)
    y = torch.empty_like(x, device="cuda")
    lb.rmsnorm(cuda(x), cuda(g), y, 1e-6)
    lb.llama_block_sync_status()
    want = ob.rmsnorm(x, g, 1e-6)
    assert row_err(y, want) <= _tol(dt)


def test_rmsnorm_zero_rows_is_noop():
    x = torch.zeros(0, 64, device="cuda")
    lb.rmsnorm(x, torch.ones(64, device="cuda"), torch.zeros(0, 64, device="cuda"), 1e-6)
    lb.llama_block_sync_status()


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dh", [64, 128])
def test_rope_apply(dt, dh):
    B, H, T = 2, 3, 37
    x = make_tensor((B, H, T, dh), 300 + dh, dt)
    pos = torch.randint(0, 5000, (B, T), generator=torch.Generator().manual_seed(7), dtype=torch.int32)
    xg = cuda(x)
    lb.rope_apply(xg, cuda(pos), 10000.0)
    lb.llama_block_sync_status()
    want = ob.apply_rope(x, pos.numpy().astype(np.float64)[:, None, :], 10000.0)
    assert row_err(xg, want) <= _tol(dt)


ATTN_CASES = [
    # B, H, Hkv, Tq, Tk, k_stride, dh
    (1, 4, 4, 64, 64, 64, 64),        # tiny, single partial tile
    (2, 4, 2, 300, 300, 320, 128),    # GQA, 3 query tiles, ragged tail
    (1, 16, 2, 256, 256, 256, 128),   # n_rep = 8
    (2, 2, 2, 130, 400, 512, 64),     # queries at an offset (chunked prefill)
    (3, 2, 1, 1, 513, 600, 128),      # a single decode-like query per sequence
    (1, 2, 2, 384, 384, 384, 128),    # exact tiles
    (2, 2, 2, 130, 400, 512, 128),    # offset; consecutive-row CTA pairs, one key block
                                      # after all rows of the first CTA
    (1, 6, 2, 200, 333, 352, 128),    # offset, n_rep = 3 (odd: consecutive-row pairs)
    (2, 4, 1, 129, 129, 160, 128),    # n_rep = 4 (head pairs), one row past a tile
    (1, 4, 4, 600, 600, 640, 128),    # five 128-key blocks: every buffer and ring stage reused
]


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("case", ATTN_CASES)
def test_causal_attn(dt, case):
    B, H, Hkv, Tq, Tk, ks, dh = case
    q = make_tensor((B, H, Tq, dh), 400, dt)
    k = make_tensor((B, Hkv, ks, dh), 401, dt)
    v = make_tensor((B, Hkv, ks, dh), 402, dt)
    kg, vg = cuda(k), cuda(v)
    if ks > Tk:  # rows beyond Tk must never be read into the result
        kg[:, :, Tk:] = float("nan")
        vg[:, :, Tk:] = float("nan")
    o = torch.empty(B, Tq, H * dh, dtype=dt, device="cuda")
    lb.causal_attn(cuda(q), kg, vg, o, Tk=Tk)
    lb.llama_block_sync_status()
    want = ob.causal_attention(q, k[:, :, :Tk], v[:, :, :Tk])  # [B,H,Tq,dh]
    want = want.transpose(0, 2, 1, 3).reshape(B, Tq, H * dh)
    got = as_np(o).reshape(B, Tq, H, dh)
    assert row_err(got, want.reshape(B, Tq, H, dh)) <= _tol(dt)


@pytest.mark.parametrize("slope", [0.05, 1.0, 20.0])
def test_causal_attn_scores_growing_along_keys(slope):
    """Online-softmax reference moves: component 0 of key t is slope * t and of every
    query +1 (even heads) or -1 (odd heads), so along the keys the scores grow (the
    running max moves between 128-key steps: by about 0.6, 11 and 226 natural-log
    units per step for the three slopes, the last far past the fp32 exponent range if
    a step's exponentials were taken against the previous reference) or shrink (the
    max stays at key 0). Compared with the fp64 oracle like every other attention case."""
    dt = torch.bfloat16
    B, H, Hkv, T, dh = 1, 4, 2, 600, 128
    q = make_tensor((B, H, T, dh), 410, torch.float32, std=0.5)
    k = make_tensor((B, Hkv, T, dh), 411, torch.float32, std=0.5)
    v = make_tensor((B, Hkv, T, dh), 412, torch.float32)
    q[:, 0::2, :, 0] = 1.0
    q[:, 1::2, :, 0] = -1.0
    k[:, :, :, 0] = slope * torch.arange(T, dtype=torch.float32)
    q, k, v = q.to(dt), k.to(dt), v.to(dt)
    o = torch.empty(B, T, H * dh, dtype=dt, device="cuda")
    lb.causal_attn(cuda(q), cuda(k), cuda(v), o)
    lb.llama_block_sync_status()
    want = ob.causal_attention(q, k, v).transpose(0, 2, 1, 3).reshape(B, T, H, dh)
    assert row_err(as_np(o).reshape(B, T, H, dh), want) <= BF16_TOL


@pytest.mark.parametrize("dt,M,d,f", [
    (torch.float32, 17, 256, 688),
    (torch.bfloat16, 300, 512, 1000),   # ragged M, f not a multiple of 128
    (torch.bfloat16, 256, 1024, 2816),  # exact tiles
    (torch.bfloat16, 5, 512, 384),
])
def test_swiglu_mlp(dt, M, d, f):
    h = make_tensor((M, d), 500, dt)
    wg = make_tensor((f, d), 501, dt, std=0.05)
    wu = make_tensor((f, d), 502, dt, std=0.05)
    wd = make_tensor((d, f), 503, dt, std=0.05)
    y = torch.empty(M, d, dtype=dt, device="cuda")
    lb.swiglu_mlp(cuda(h), cuda(wg), cuda(wu), cuda(wd), y)
    lb.llama_block_sync_status()
    want = ob.swiglu_mlp(h, wg, wu, wd)
    assert row_err(y, want) <= _tol(dt)


def test_bounded_wait_times_out_cleanly():
    """A wait on a barrier nothing completes gives up after its budget, latches
    the error word, and the context stays usable."""
    lb.llama_block_selftest_timeout(50_000_000)  # 50 ms
    with pytest.raises(lb.LlamaBlockError) as ei:
        lb.llama_block_sync_status()
    assert ei.value.name == "LB_ERR_TIMEOUT"
    lb.llama_block_sync_status()  # cleared
    x = torch.ones(2, 64, device="cuda")
    y = torch.empty_like(x)
    lb.rmsnorm(x, torch.ones(64, device="cuda"), y, 1e-6)
    lb.llama_block_sync_status()
    assert torch.allclose(y, torch.ones_like(y), atol=1e-5)
