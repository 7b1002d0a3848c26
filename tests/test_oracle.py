"""Pins for the fp64 oracle, checked against what the pages and mathematics fix.

Nothing here touches a GPU. Each test names the passage it follows. The pins
are chosen so that a plausible slip in the oracle (a dropped term, a wrong sign
or index, a transposed operand, a wrong head grouping) fails at least one:

* worked examples printed on the pages (tests/golden/*.json),
* closed forms and invariants the pages state,
* independent library routines (torch fp64 ``rms_norm``, ``linear``,
  ``scaled_dot_product_attention``, ``silu``) and an independent complex-number
  formulation of RoPE on tiny inputs.
"""

import json
import math
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import block as ob

GOLD = Path(__file__).parent / "golden"


def _gold(name):
    return json.loads((GOLD / name).read_text())


def _half_ulp(decimals):
    return 0.5 * 10.0 ** (-decimals) + 1e-12


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_worked_example():
    """LMDrive page §2.1: [1,2,3] -> mean square 4.67, rms 2.16, ≈[0.46,0.93,1.39]."""
    g = _gold("rmsnorm_worked_example.json")
    x = np.array(g["x"])
    y = ob.rmsnorm(x, np.array(g["g"]), g["eps"])
    assert abs(np.mean(x * x) - g["mean_sq_printed"]) <= _half_ulp(g["mean_sq_decimals"])
    assert abs(math.sqrt(np.mean(x * x)) - g["rms_printed"]) <= _half_ulp(g["rms_decimals"])
    np.testing.assert_allclose(y, g["y_printed"], rtol=0, atol=_half_ulp(g["y_decimals"]))
    # the exact value behind the printed digits
    np.testing.assert_allclose(y, x / math.sqrt(14.0 / 3.0 + 1e-6), rtol=1e-15)


def test_rmsnorm_matches_torch_rms_norm():
    """Runnable example 05 of the LLM-mechanics page: manual RMSNorm == F.rms_norm."""
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(7, 33, generator=gen, dtype=torch.float64) * 3.0
    g = 1.0 + 0.1 * torch.randn(33, generator=gen, dtype=torch.float64)
    ref = F.rms_norm(x, (33,), g, 1e-6).numpy()
    np.testing.assert_allclose(ob.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-14)


def test_rmsnorm_output_rms_is_one_and_constant_vector():
    """Example 05 expects output RMS ≈ 1 with unit gain; a constant vector c·1
    maps to g·c/sqrt(c²+eps) (closed form of §02.3's equation)."""
    x = np.random.default_rng(0).normal(size=(4, 4096)) * 5
    y = ob.rmsnorm(x, np.ones(4096), 1e-6)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-7)
    c, eps = -0.37, 1e-6
    g = np.linspace(0.5, 1.5, 16)
    np.testing.assert_allclose(ob.rmsnorm(np.full(16, c), g, eps), g * c / math.sqrt(c * c + eps),
                               rtol=1e-14)
    # no mean subtraction: a shifted vector does not normalise to the same output
    v = np.arange(1.0, 9.0)
    assert not np.allclose(ob.rmsnorm(v, np.ones(8), eps), ob.rmsnorm(v - v.mean(), np.ones(8), eps))


# ---------------------------------------------------------------- RoPE
def test_rope_worked_example():
    """LMDrive page §2.2: head_dim=4, pos=2 -> inv_freq=[1,0.01], freqs=[2,0.02],
    cos≈[-0.416,1.0], sin≈[0.909,0.02], q0'=q0cos2-q2sin2, q1'=q1cos.02-q3sin.02."""
    g = _gold("rope_worked_example.json")
    dh, pos, base = g["head_dim"], g["pos"], g["base"]
    inv = ob.rope_inv_freq(dh, base)
    for got, want, dec in zip(inv, g["inv_freq_printed"], g["inv_freq_decimals"]):
        assert abs(got - want) <= _half_ulp(dec)
    cos, sin = ob.rope_cos_sin(np.array([pos]), dh, base)
    half = dh // 2
    for i in range(half):
        assert abs(pos * inv[i] - g["freqs_printed"][i]) <= _half_ulp(g["freqs_decimals"][i])
        assert abs(cos[0, i] - g["cos_printed"][i]) <= _half_ulp(g["cos_decimals"][i])
        assert abs(sin[0, i] - g["sin_printed"][i]) <= _half_ulp(g["sin_decimals"][i])
        # emb = cat(freqs, freqs): the second half repeats the first
        assert cos[0, i + half] == cos[0, i] and sin[0, i + half] == sin[0, i]
    q = np.array([0.3, -1.1, 0.7, 2.0])
    r = ob.apply_rope(q, np.array(pos, dtype=float), base)
    q0, q1, q2, q3 = q
    assert r[0] == pytest.approx(q0 * math.cos(2.0) - q2 * math.sin(2.0), abs=1e-15)
    assert r[1] == pytest.approx(q1 * math.cos(0.02) - q3 * math.sin(0.02), abs=1e-15)
    # the other half, from rotate_half(x) = cat(-x2, x1)
    assert r[2] == pytest.approx(q2 * math.cos(2.0) + q0 * math.sin(2.0), abs=1e-15)
    assert r[3] == pytest.approx(q3 * math.cos(0.02) + q1 * math.sin(0.02), abs=1e-15)


def _rope_complex(x, pos, base):
    """Independent formulation: pair (x_i, x_{i+d/2}) as the complex number
    x_i + j x_{i+d/2}, multiplied by exp(j * pos * base^(-2i/d))."""
    x = torch.as_tensor(x, dtype=torch.float64)
    d = x.shape[-1]
    theta = torch.tensor([base ** (-2.0 * i / d) for i in range(d // 2)], dtype=torch.float64)
    ang = torch.as_tensor(pos, dtype=torch.float64)[..., None] * theta
    z = torch.complex(x[..., : d // 2], x[..., d // 2:]) * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([z.real, z.imag], dim=-1).numpy()


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(3, 5, 64))
    pos = np.arange(5, dtype=float)[None, :] + np.array([[0.0], [100.0], [4095.0]])
    np.testing.assert_allclose(ob.apply_rope(x, pos, 10000.0), _rope_complex(x, pos, 10000.0),
                               rtol=1e-12, atol=1e-12)


def test_rope_half_split_is_permuted_interleaved_form():
    """The LLM-mechanics page §02.2 rotates interleaved pairs x_{2i:2i+2} by
    R(mθ_i); the half-split (rotate_half) form is the same map after moving
    dimension pair (i, i+d/2) to (2i, 2i+1)."""
    d, base, m = 8, 10000.0, 7.0
    x = np.random.default_rng(2).normal(size=d)
    perm = np.empty(d, dtype=int)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    xi = x[perm]  # interleaved layout
    out_i = np.empty(d)
    for i in range(d // 2):
        th = m * base ** (-2.0 * i / d)
        R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        out_i[2 * i:2 * i + 2] = R @ xi[2 * i:2 * i + 2]
    np.testing.assert_allclose(ob.apply_rope(x, np.array(m), base)[perm], out_i, rtol=1e-14, atol=1e-15)


def test_rope_invariants():
    """Runnable example 04 and §02.2: position 0 is the identity, the norm is
    preserved, and <R(m)q, R(n)k> depends only on n - m."""
    rng = np.random.default_rng(3)
    q, k = rng.normal(size=128), rng.normal(size=128)
    np.testing.assert_array_equal(ob.apply_rope(q, np.array(0.0), 1e4), q)
    assert np.linalg.norm(ob.apply_rope(q, np.array(7.0), 1e4)) == pytest.approx(np.linalg.norm(q), rel=1e-14)
    r = lambda x, p: ob.apply_rope(x, np.array(float(p)), 1e4)  # noqa: E731
    assert r(q, 2) @ r(k, 5) == pytest.approx(r(q, 9) @ r(k, 12), rel=1e-12)
    assert r(q, 2) @ r(k, 5) == pytest.approx(q @ r(k, 3), rel=1e-12)
    assert not math.isclose(r(q, 2) @ r(k, 5), r(q, 2) @ r(k, 6), rel_tol=1e-6)


# ---------------------------------------------------------------- attention
def _rand(shape, seed):
    return np.random.default_rng(seed).normal(size=shape)


def test_causal_mask_zero_future_and_rows_sum_to_one():
    """Runnable example 03 / §02.1: attention[future] == 0 exactly, rows sum to 1;
    LAB 02: query 3 reads keys 0..3 only."""
    q, k, v = _rand((1, 2, 6, 8), 0), _rand((1, 2, 6, 8), 1), _rand((1, 2, 6, 8), 2)
    o, p = ob.causal_attention(q, k, v, return_probs=True)
    future = np.triu(np.ones((6, 6), dtype=bool), 1)
    assert np.all(p[..., future] == 0.0)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    assert np.all(p[0, :, 3, :4] > 0) and np.all(p[0, :, 3, 4:] == 0)
    # row 0 sees only key 0: output is v_0 exactly; a single token gives O = V
    np.testing.assert_array_equal(o[0, :, 0], v[0, :, 0])
    o1 = ob.causal_attention(q[:, :, :1], k[:, :, :1], v[:, :, :1])
    np.testing.assert_array_equal(o1, v[:, :, :1])


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (8, 1)])
def test_attention_matches_torch_sdpa(H, Hkv):
    """Scaled dot-product softmax attention with the causal mask and repeat_kv
    (LMDrive page §2.3) against torch's fp64 SDPA with enable_gqa."""
    B, T, dh = 2, 9, 16
    q, k, v = _rand((B, H, T, dh), 10), _rand((B, Hkv, T, dh), 11), _rand((B, Hkv, T, dh), 12)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                                         is_causal=True, enable_gqa=(H != Hkv)).numpy()
    np.testing.assert_allclose(ob.causal_attention(q, k, v), ref, rtol=1e-12, atol=1e-13)


def test_gqa_equals_mha_with_duplicated_kv_heads():
    """repeat_kv: GQA equals MHA after each KV head is duplicated n_rep times
    in place (head h reads KV head h // n_rep)."""
    H, Hkv, T, dh = 6, 2, 7, 8
    q, k, v = _rand((1, H, T, dh), 20), _rand((1, Hkv, T, dh), 21), _rand((1, Hkv, T, dh), 22)
    kd = torch.from_numpy(k).repeat_interleave(H // Hkv, dim=1).numpy()
    vd = torch.from_numpy(v).repeat_interleave(H // Hkv, dim=1).numpy()
    np.testing.assert_allclose(ob.causal_attention(q, k, v), ob.causal_attention(q, kd, vd), rtol=1e-15)
    # and not the other grouping (h % H_kv)
    kt = np.tile(k, (1, H // Hkv, 1, 1))
    vt = np.tile(v, (1, H // Hkv, 1, 1))
    assert not np.allclose(ob.causal_attention(q, k, v), ob.causal_attention(q, kt, vt))


def test_offset_queries_equal_last_rows_of_full_attention():
    """Runnable example 07: decode (one query over all keys) equals the last
    row of the full recompute; more generally Tq < Tk queries sit at the end."""
    H, T, dh = 3, 11, 8
    q, k, v = _rand((2, H, T, dh), 30), _rand((2, H, T, dh), 31), _rand((2, H, T, dh), 32)
    full = ob.causal_attention(q, k, v)
    np.testing.assert_allclose(ob.causal_attention(q[:, :, -1:], k, v), full[:, :, -1:], rtol=1e-13)
    np.testing.assert_allclose(ob.causal_attention(q[:, :, -4:], k, v), full[:, :, -4:], rtol=1e-13)
    np.testing.assert_allclose(ob.causal_attention(q, k, v, rows=[0, 5, 10]), full[:, :, [0, 5, 10]],
                               rtol=1e-14)


# ---------------------------------------------------------------- SwiGLU MLP
def test_mlp_param_count_table():
    """Llama-MLP page §3.2 table and §3.3: 3·d·f parameters, no bias."""
    g = _gold("mlp_param_table.json")
    for row in g["rows"]:
        d, f = row["d"], row["f"]
        n = ob.mlp_param_count(np.empty((f, d)), np.empty((f, d)), np.empty((d, f)))
        assert n == 3 * d * f
        assert abs(n / 1e8 - row["params_1e8"]) <= _half_ulp(g["decimals"]), row
        assert abs(f / d - row["f_over_d"]) <= _half_ulp(g["decimals"]), row
    seven = g["rows"][0]
    total = seven["layers"] * 3 * seven["d"] * seven["f"]
    assert round(total / 1e8) == g["total_7b_mlp_params_printed_1e8"]


def test_silu_closed_forms():
    """SiLU(z) = z·σ(z) (LMDrive page §2.4)."""
    z = np.array([0.0, 1.0, -1.0, 40.0, -800.0])
    s = ob.silu(z)
    assert s[0] == 0.0
    assert s[1] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert s[2] == pytest.approx(-1.0 / (1.0 + math.e), rel=1e-15)
    assert s[3] == pytest.approx(40.0, rel=1e-15)
    assert s[4] == 0.0


def test_swiglu_matches_torch_and_is_not_relu2():
    """Runnable example 06: same shape as the input, different from ReLU²;
    equals torch's linear/silu composition; a zero down_proj gives 0."""
    rng = np.random.default_rng(40)
    d, f = 16, 40
    h = rng.normal(size=(3, 5, d))
    wg, wu, wd = rng.normal(size=(f, d)) * .2, rng.normal(size=(f, d)) * .2, rng.normal(size=(d, f)) * .2
    y = ob.swiglu_mlp(h, wg, wu, wd)
    th = torch.from_numpy(h)
    ref = F.linear(F.silu(F.linear(th, torch.from_numpy(wg))) * F.linear(th, torch.from_numpy(wu)),
                   torch.from_numpy(wd)).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)
    assert y.shape == h.shape
    relu2 = (np.maximum(h @ wg.T, 0) ** 2) @ wd.T
    assert not np.allclose(y, relu2)
    assert np.all(ob.swiglu_mlp(h, wg, wu, np.zeros_like(wd)) == 0)
    # gate gets the activation, up does not (Llama-MLP page §4.2)
    assert not np.allclose(y, ob.swiglu_mlp(h, wu, wg, wd))


# ---------------------------------------------------------------- block
def _tiny_weights(d=8, H=2, Hkv=1, dh=4, f=12, seed=50, gains=True):
    rng = np.random.default_rng(seed)
    W = {
        "wq": rng.normal(size=(H * dh, d)) * .3, "wk": rng.normal(size=(Hkv * dh, d)) * .3,
        "wv": rng.normal(size=(Hkv * dh, d)) * .3, "wo": rng.normal(size=(d, H * dh)) * .3,
        "w_gate": rng.normal(size=(f, d)) * .3, "w_up": rng.normal(size=(f, d)) * .3,
        "w_down": rng.normal(size=(d, f)) * .3,
        "g_attn": 1 + .1 * rng.normal(size=d) if gains else np.ones(d),
        "g_mlp": 1 + .1 * rng.normal(size=d) if gains else np.ones(d),
    }
    return W


def _torch_block(X, W, H, Hkv, dh, eps, base):
    """The block composed from torch fp64 library routines (rms_norm, linear,
    complex-number RoPE, SDPA with enable_gqa, silu) — independent of the
    oracle's own arithmetic."""
    t = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in W.items()}
    X = torch.from_numpy(X)
    B, T, d = X.shape
    h = F.rms_norm(X, (d,), t["g_attn"], eps)
    q = F.linear(h, t["wq"]).view(B, T, H, dh).transpose(1, 2)
    k = F.linear(h, t["wk"]).view(B, T, Hkv, dh).transpose(1, 2)
    v = F.linear(h, t["wv"]).view(B, T, Hkv, dh).transpose(1, 2)
    pos = np.arange(T, dtype=float)
    q = torch.from_numpy(_rope_complex(q.numpy(), pos, base))
    k = torch.from_numpy(_rope_complex(k.numpy(), pos, base))
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=(H != Hkv))
    x1 = X + F.linear(o.transpose(1, 2).reshape(B, T, H * dh), t["wo"])
    h2 = F.rms_norm(x1, (d,), t["g_mlp"], eps)
    y = x1 + F.linear(F.silu(F.linear(h2, t["w_gate"])) * F.linear(h2, t["w_up"]), t["w_down"])
    return y.numpy(), k.numpy(), v.numpy()


@pytest.mark.parametrize("H,Hkv", [(2, 1), (2, 2), (4, 2)])
def test_block_matches_torch_composition(H, Hkv):
    """Pre-norm block (LMDrive page §2.5; LLM-mechanics chapter-02 equation),
    d=8, d_h=4, f=12, T=5 as brute force against torch fp64 routines."""
    d, dh, f, T = 8, 4, 12, 5
    W = _tiny_weights(d, H, Hkv, dh, f)
    X = np.random.default_rng(51).normal(size=(2, T, d))
    out = ob.block_prefill(X, W, H, Hkv, dh, 1e-6, 10000.0)
    y, k, v = _torch_block(X, W, H, Hkv, dh, 1e-6, 10000.0)
    np.testing.assert_allclose(out["y"], y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["k"], k, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["v"], v, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["y"], out["x1"] + out["mlp"], rtol=1e-15)
    np.testing.assert_allclose(out["x1"], X + out["attn"], rtol=1e-15)


def test_block_shape_and_zero_weight_identity():
    """Example 02: the block keeps [batch, length, width]; with zero o_proj and
    down_proj both residual branches vanish and X'' = X."""
    W = _tiny_weights()
    X = np.random.default_rng(52).normal(size=(3, 6, 8))
    assert ob.block_prefill(X, W, 2, 1, 4, 1e-6, 1e4)["y"].shape == X.shape
    W0 = dict(W, wo=np.zeros_like(W["wo"]), w_down=np.zeros_like(W["w_down"]))
    np.testing.assert_array_equal(ob.block_prefill(X, W0, 2, 1, 4, 1e-6, 1e4)["y"], X)


def test_block_row_sampling_is_consistent():
    """The row-sampled mode (used at full workload sizes) returns exactly the
    selected rows of the full evaluation."""
    W = _tiny_weights(d=16, H=4, Hkv=2, dh=4, f=20)
    X = np.random.default_rng(53).normal(size=(2, 13, 16))
    full = ob.block_prefill(X, W, 4, 2, 4, 1e-6, 1e4)
    rows = [0, 4, 12]
    part = ob.block_prefill(X, W, 4, 2, 4, 1e-6, 1e4, rows=rows)
    for key in ("y", "x1", "attn", "mlp", "o"):
        np.testing.assert_allclose(part[key], full[key][:, rows], rtol=1e-13, atol=1e-14)


def test_decode_equals_prefill_last_row():
    """Runnable examples 07/08 at block level: after a prefill of T tokens the
    cache holds T keys; decoding token T at position T (the cache length, as
    chapter 04 requires) gives the last row of a full prefill of T+1 tokens."""
    H, Hkv, dh, d, f, T = 4, 2, 8, 16, 24, 6
    W = _tiny_weights(d, H, Hkv, dh, f, seed=60)
    X = np.random.default_rng(61).normal(size=(2, T + 1, d))
    full = ob.block_prefill(X, W, H, Hkv, dh, 1e-6, 1e4)
    pre = ob.block_prefill(X[:, :T], W, H, Hkv, dh, 1e-6, 1e4)
    t_max = T + 3
    kc = np.zeros((2, Hkv, t_max, dh))
    vc = np.zeros((2, Hkv, t_max, dh))
    kc[:, :, :T], vc[:, :, :T] = pre["k"], pre["v"]
    dec = ob.block_decode(X[:, T:], W, H, Hkv, dh, 1e-6, 1e4, kc, vc, [T, T])
    np.testing.assert_allclose(dec["y"], full["y"][:, T:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dec["k_new"], full["k"][:, :, T:], rtol=1e-12, atol=1e-13)
    # decoding from the wrong position (0 instead of the cache length) differs
    bad = ob.block_decode(X[:, T:], W, H, Hkv, dh, 1e-6, 1e4, kc, vc, [0, 0])
    assert not np.allclose(bad["y"], dec["y"])


def test_decode_ragged_cache_lengths():
    """Sequences with different cache lengths each attend to their own prefix."""
    H, Hkv, dh, d, f = 2, 2, 4, 8, 12
    W = _tiny_weights(d, H, Hkv, dh, f, seed=70)
    X = np.random.default_rng(71).normal(size=(2, 9, d))
    lens = [3, 7]
    kc = np.zeros((2, Hkv, 10, dh))
    vc = np.zeros((2, Hkv, 10, dh))
    want = []
    for b, L in enumerate(lens):
        pre = ob.block_prefill(X[b:b + 1, :L], W, H, Hkv, dh, 1e-6, 1e4)
        kc[b, :, :L], vc[b, :, :L] = pre["k"][0], pre["v"][0]
        want.append(ob.block_prefill(X[b:b + 1, :L + 1], W, H, Hkv, dh, 1e-6, 1e4)["y"][0, L])
    xs = np.stack([X[0, 3:4], X[1, 7:8]])
    dec = ob.block_decode(xs, W, H, Hkv, dh, 1e-6, 1e4, kc, vc, lens)
    np.testing.assert_allclose(dec["y"][:, 0], np.stack(want), rtol=1e-12, atol=1e-12)


def test_decode_from_an_empty_cache_attends_to_itself():
    """A first token decoded into an empty cache has one key: the softmax is 1 and each
    query head's attention output is the new value vector of its KV head (GQA group)."""
    H, Hkv, dh, d, f = 4, 2, 4, 8, 12
    W = _tiny_weights(d, H, Hkv, dh, f, seed=72)
    x = np.random.default_rng(73).normal(size=(2, 1, d))
    kc = np.zeros((2, Hkv, 3, dh))
    dec = ob.block_decode(x, W, H, Hkv, dh, 1e-6, 1e4, kc, kc.copy(), [0, 0])
    rep = H // Hkv
    for h in range(H):
        np.testing.assert_allclose(dec["o"][:, 0, h * dh:(h + 1) * dh], dec["v_new"][:, h // rep, 0],
                                   rtol=1e-12, atol=1e-12)
    # and it is the one-token prefill
    for b in range(2):
        pre = ob.block_prefill(x[b:b + 1], W, H, Hkv, dh, 1e-6, 1e4)
        np.testing.assert_allclose(dec["y"][b], pre["y"][0], rtol=1e-12, atol=1e-12)


def test_dynamic_ntk_base_invariants():
    """Dynamic NTK scaling (named, without a formula, by [LMDrive] §2.2; parity unpinned):
    the invariants that define the reading taken. Up to the trained context the base is
    unchanged and it is continuous there; beyond it the highest rotary frequency stays 1
    and the lowest one slows down by exactly s = factor * L / L0 - (factor - 1); the base
    grows with L and with the factor."""
    base, L0 = 10000.0, 2048
    for dh in (64, 128):
        for factor in (1.0, 2.0, 4.0):
            assert ob.dynamic_ntk_rope_base(base, dh, 1, L0, factor) == base
            assert ob.dynamic_ntk_rope_base(base, dh, L0, L0, factor) == base
            assert math.isclose(ob.dynamic_ntk_rope_base(base, dh, L0 + 1, L0, factor), base, rel_tol=5e-3)
            prev = base
            for L in (L0 + 1, 3000, 4096, 8192, 32768):
                b2 = ob.dynamic_ntk_rope_base(base, dh, L, L0, factor)
                s = factor * L / L0 - (factor - 1.0)
                f0, f1 = ob.rope_inv_freq(dh, base), ob.rope_inv_freq(dh, b2)
                assert f1[0] == 1.0
                assert math.isclose(f1[-1], f0[-1] / s, rel_tol=1e-12)
                assert np.all(np.diff(f1) < 0) and np.all(f1 <= f0)
                assert b2 > prev
                prev = b2
        assert ob.dynamic_ntk_rope_base(base, dh, 4096, L0, 4.0) > ob.dynamic_ntk_rope_base(base, dh, 4096, L0, 2.0)
    assert ob.dynamic_ntk_rope_base(base, 128, 4096, 0, 2.0) == base  # off


def test_kv_cache_bytes_ledger():
    """Chapter 04 memory accounting: L·2·B·T·H_kv·d_h·bytes equals the size of
    an allocated [layers,B,T,H_kv,D] K and V buffer pair (source-map layout)
    and example 08's product for fp32."""
    g = _gold("kv_cache_ledger.json")
    s = g["lab05_shape_per_layer"]
    for layers, dt in ((1, np.float16), (32, np.float16), (3, np.float32)):
        bytes_ = ob.kv_cache_bytes(layers, s["B"], s["T"], s["H_kv"], s["d_h"], np.dtype(dt).itemsize)
        buf = np.empty((2, layers, s["B"], s["T"], s["H_kv"], s["d_h"]), dtype=dt)
        assert bytes_ == buf.nbytes
    T, layers, batch, heads, hd = 4096, 2, 3, 8, 128
    assert ob.kv_cache_bytes(layers, batch, T, heads, hd, g["example08_dtype_bytes"]) == \
        T * layers * batch * heads * hd * 2 * 4


# ---------------------------------------------------------------- chunked prefill / stack
def test_extend_reduces_to_prefill_and_decode():
    """Chunked prefill: appending T2 tokens after a prefill of T1 gives the last
    T2 rows of a prefill of T1+T2 (causal attention only looks back); at L=0 it
    is the prefill itself; with T=1 it is the decode step."""
    H, Hkv, dh, d, f = 4, 2, 8, 16, 24
    W = _tiny_weights(d, H, Hkv, dh, f, seed=80)
    X = np.random.default_rng(81).normal(size=(2, 9, d))
    full = ob.block_prefill(X, W, H, Hkv, dh, 1e-6, 1e4)
    pre = ob.block_prefill(X[:, :5], W, H, Hkv, dh, 1e-6, 1e4)
    ext = ob.block_extend(X[:, 5:], W, H, Hkv, dh, 1e-6, 1e4, pre["k"], pre["v"], 5)
    np.testing.assert_allclose(ext["y"], full["y"][:, 5:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ext["k_new"], full["k"][:, :, 5:], rtol=1e-12, atol=1e-13)
    z = np.zeros((2, Hkv, 0, dh))
    np.testing.assert_allclose(ob.block_extend(X, W, H, Hkv, dh, 1e-6, 1e4, z, z, 0)["y"], full["y"],
                               rtol=1e-13, atol=1e-13)
    one = ob.block_extend(X[:, 5:6], W, H, Hkv, dh, 1e-6, 1e4, pre["k"], pre["v"], 5)
    dec = ob.block_decode(X[:, 5:6], W, H, Hkv, dh, 1e-6, 1e4, pre["k"], pre["v"], [5, 5])
    np.testing.assert_allclose(one["y"], dec["y"], rtol=1e-13, atol=1e-13)


def test_stack_one_layer_is_the_block_and_zero_layers_pass_through():
    """A one-layer stack is the block; layers whose o_proj and down_proj are zero
    leave the residual stream unchanged, whatever their attention and MLP do."""
    H, Hkv, dh, d, f = 2, 1, 4, 8, 12
    W = _tiny_weights(d, H, Hkv, dh, f, seed=90)
    X = np.random.default_rng(91).normal(size=(1, 6, d))
    one = ob.stack_prefill(X, [W], H, Hkv, dh, 1e-6, 1e4)
    ref = ob.block_prefill(X, W, H, Hkv, dh, 1e-6, 1e4)
    np.testing.assert_array_equal(one["y"], ref["y"])
    Z = dict(W, wo=np.zeros_like(W["wo"]), w_down=np.zeros_like(W["w_down"]))
    three = ob.stack_prefill(X, [Z, W, Z], H, Hkv, dh, 1e-6, 1e4)
    np.testing.assert_allclose(three["y"], ref["y"], rtol=1e-14, atol=1e-14)
    # and the stack extend continues every layer's cache
    pre = ob.stack_prefill(X[:, :4], [W, W], H, Hkv, dh, 1e-6, 1e4)
    ext = ob.stack_extend(X[:, 4:], [W, W], H, Hkv, dh, 1e-6, 1e4, pre["k"], pre["v"], 4)
    full = ob.stack_prefill(X, [W, W], H, Hkv, dh, 1e-6, 1e4)
    np.testing.assert_allclose(ext["y"], full["y"][:, 4:], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- INT8 decode weights
def test_int8_row_quantization_properties():
    """Per-row symmetric INT8: codes in [-127, 127], each non-zero row reaches
    |q| = 127 at its absmax, the reconstruction error is at most half a step,
    weights that are exact multiples of the step are reproduced exactly, and a
    zero row stays zero."""
    rng = np.random.default_rng(100)
    w = rng.normal(size=(16, 64)).astype(np.float32) * 0.02
    w[3] = 0.0
    step = np.float32(0.125)
    w[5] = step * rng.integers(-127, 128, size=64).astype(np.float32)
    w[5, 0] = 127 * step
    q, s = ob.quantize_int8_rows(w)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert q.min() >= -127 and q.max() <= 127
    for r in range(16):
        if r == 3:
            assert s[r] == 0 and np.all(q[r] == 0)
            continue
        assert np.max(np.abs(q[r].astype(int))) == 127
        err = np.abs(ob.dequantize_int8_rows(q[r:r + 1], s[r:r + 1])[0] - w[r].astype(np.float64))
        assert np.all(err <= 0.5 * float(s[r]) * (1 + 1e-6))
    np.testing.assert_array_equal(ob.dequantize_int8_rows(q[5:6], s[5:6])[0], w[5].astype(np.float64))
    # the decode block on INT8 weights is the block on the dequantized weights
    W = _tiny_weights(d=8, H=2, Hkv=1, dh=4, f=12, seed=101)
    Wq = ob.int8_decode_weights(W)
    assert set(Wq) == set(W) and np.array_equal(Wq["g_attn"], W["g_attn"])
    assert not np.array_equal(Wq["wq"], W["wq"])

