"""fp64 CPU oracle of the LLaMA pre-norm decoder block (test infrastructure).

This module is test infrastructure. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it. The CUDA library never calls it and shares no code with it.

It is the plain mathematical definition of the block written out in float64,
step by step in the order the pages give, with numpy's matmul as the only
library primitive. Inputs arrive already rounded to the compute dtype and are
widened exactly to float64; nothing here mimics the GPU's roundings.

Sources (page title, then section):
  [LMDrive]  "LMDrive 大语言模型（LLM）核心推理单元": §2.1 LlamaRMSNorm,
             §2.2 LlamaRotaryEmbedding (rotate_half), §2.3 LlamaAttention
             (q/k/v projections, RoPE, past_key_value concat, repeat_kv,
             scaled scores, mask, softmax), §2.4 LlamaMLP, §2.5 LlamaDecoderLayer.
  [Mechanics] "LLM 核心机制交互讲义": chapter 02 (block equation, §02.1 causal
             mask, §02.2 RoPE, §02.3 RMSNorm, §02.4 SwiGLU), chapter 04 (KV cache
             equation, memory accounting).
  [LlamaMLP] "深入解析Llama MLP模块：SwiGLU激活函数与参数配置详解": §3.3 (3df,
             no bias), §4.2 (gate gets SiLU, up does not, then down).

Readings where the pages are silent or disagree:
  * RoPE pairs dimension i with i + d_h/2 (rotate_half, [LMDrive] §2.2), not the
    interleaved (2i, 2i+1) pairs of [Mechanics] §02.2; the two differ by a fixed
    permutation of the head dimensions.
  * No bias on any projection.
  * GQA groups consecutive query heads: query head h reads KV head h // n_rep.
  * The KV cache holds keys after RoPE; decode positions start at the cache
    length ([Mechanics] chapter 04, "position offset must follow the cache").

Every function here is pinned by ``tests/test_oracle.py`` (worked examples from
the pages, closed forms, invariants, and library routines on tiny inputs), except
``dynamic_ntk_rope_base``: parity unpinned. [LMDrive] §2.2 names dynamic NTK
scaling without a formula; that function is the reading taken, checked only
against the invariants that define it.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    """Widen a numpy array or CPU torch tensor exactly to float64."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # local import: torch only used for the exact dtype widening

        a = a.to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# RMSNorm — [LMDrive] §2.1 and [Mechanics] §02.3:
#   RMSNorm(x) = g ⊙ x / sqrt(mean_i(x_i^2) + eps), no mean subtraction.
# --------------------------------------------------------------------------
def rmsnorm(x, g, eps: float) -> np.ndarray:
    x = _f64(x)
    g = _f64(g)
    mean_sq = np.mean(x * x, axis=-1, keepdims=True)
    return g * (x / np.sqrt(mean_sq + eps))


# --------------------------------------------------------------------------
# RoPE — [LMDrive] §2.2: inv_freq = 1 / base^(2i/d) for i = 0..d/2-1,
# freqs = positions ⊗ inv_freq, emb = cat(freqs, freqs), cos = cos(emb),
# sin = sin(emb), x' = x * cos + rotate_half(x) * sin,
# rotate_half(x) = cat(-x[d/2:], x[:d/2]).
# --------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, base: float) -> np.ndarray:
    exps = np.arange(0, head_dim, 2, dtype=np.float64) / head_dim
    return 1.0 / (float(base) ** exps)


def dynamic_ntk_rope_base(base: float, head_dim: int, L: int, L0: int, factor: float) -> float:
    """Rotary base for a call whose longest sequence reaches L tokens, under dynamic NTK
    scaling with trained context L0 and scale factor `factor`.

    PARITY UNPINNED: [LMDrive] §2.2 says the rotary module supports dynamic NTK scaling
    to extend the maximum sequence length, and gives no formula. Reading taken (the
    NTK-aware rule): up to L0 the base is unchanged; beyond it, with
    s = factor * L / L0 - (factor - 1) (1 at L = L0), the base grows so that the
    highest rotary frequency (base^0 = 1) stays put and the lowest one,
    base^(-(d_h - 2) / d_h), slows down by exactly s. Solving
    base'^(-(d_h - 2) / d_h) = base^(-(d_h - 2) / d_h) / s for base' gives the return value.
    """
    if L0 <= 0 or L <= L0:
        return float(base)
    s = factor * L / L0 - (factor - 1.0)
    return float(base) * s ** (head_dim / (head_dim - 2.0))


def rope_cos_sin(positions, head_dim: int, base: float):
    """cos, sin tables of shape positions.shape + (head_dim,)."""
    pos = _f64(positions)
    freqs = pos[..., None] * rope_inv_freq(head_dim, base)
    emb = np.concatenate([freqs, freqs], axis=-1)
    return np.cos(emb), np.sin(emb)


def rotate_half(x: np.ndarray) -> np.ndarray:
    half = x.shape[-1] // 2
    return np.concatenate([-x[..., half:], x[..., :half]], axis=-1)


def apply_rope(x, positions, base: float) -> np.ndarray:
    """Rotate the last axis of ``x`` (length head_dim) at ``positions``.

    ``positions`` broadcasts against ``x.shape[:-1]``.
    """
    x = _f64(x)
    cos, sin = rope_cos_sin(positions, x.shape[-1], base)
    return x * cos + rotate_half(x) * sin


# --------------------------------------------------------------------------
# Attention — [LMDrive] §2.3 and [Mechanics] §02.1:
#   A = softmax(Q K^T / sqrt(d_h) + M),  M_ij = 0 for j <= i, -inf for j > i,
#   O = A V, with K/V heads expanded by repeat_kv.
# --------------------------------------------------------------------------
def repeat_kv(kv: np.ndarray, n_rep: int) -> np.ndarray:
    """[B, H_kv, T, d_h] -> [B, H_kv * n_rep, T, d_h], each KV head repeated
    n_rep times in place (KV head j serves query heads j*n_rep .. j*n_rep+n_rep-1)."""
    return np.repeat(kv, n_rep, axis=1)


def softmax(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def causal_attention(q, k, v, rows=None, return_probs: bool = False):
    """Causal softmax attention with GQA.

    q: [B, H, Tq, d_h]; k, v: [B, H_kv, Tk, d_h] with Tk >= Tq. Query row i
    sits at absolute position Tk - Tq + i and sees keys 0 .. Tk - Tq + i
    (for Tq == Tk this is the plain lower-triangular mask).
    ``rows``: optional list of query rows to compute (others are skipped).
    Returns O [B, H, len(rows) or Tq, d_h] (and the probabilities if asked).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Tq, dh = q.shape
    Hkv, Tk = k.shape[1], k.shape[2]
    assert H % Hkv == 0 and Tk >= Tq
    n_rep = H // Hkv
    rows = list(range(Tq)) if rows is None else list(rows)
    qr = q[:, :, rows, :]
    offs = Tk - Tq
    qpos = np.asarray(rows)[:, None] + offs
    kpos = np.arange(Tk)[None, :]
    M = np.where(kpos <= qpos, 0.0, -np.inf)  # [R, Tk]
    out = np.empty((B, H, len(rows), dh))
    probs = np.empty((B, H, len(rows), Tk)) if return_probs else None
    scale = 1.0 / np.sqrt(dh)
    for b in range(B):
        for h in range(H):
            kh = k[b, h // n_rep]  # the head repeat_kv places at index h
            vh = v[b, h // n_rep]
            s = (qr[b, h] @ kh.T) * scale + M
            p = softmax(s)
            out[b, h] = p @ vh
            if return_probs:
                probs[b, h] = p
    return (out, probs) if return_probs else out


# --------------------------------------------------------------------------
# SwiGLU MLP — [LMDrive] §2.4, [LlamaMLP] §4.2:
#   down_proj( SiLU(gate_proj(x)) * up_proj(x) ),  SiLU(z) = z * sigmoid(z),
#   three bias-free linears ([LlamaMLP] §3.3: 3*d*f parameters).
# --------------------------------------------------------------------------
def sigmoid(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z) -> np.ndarray:
    z = _f64(z)
    return z * sigmoid(z)


def linear(x, w) -> np.ndarray:
    """nn.Linear without bias: y = x W^T, W stored [out, in]."""
    return _f64(x) @ _f64(w).T


def swiglu_mlp(h, w_gate, w_up, w_down) -> np.ndarray:
    gate = linear(h, w_gate)
    up = linear(h, w_up)
    return linear(silu(gate) * up, w_down)


def mlp_param_count(w_gate, w_up, w_down) -> int:
    """Number of MLP parameters actually used (no bias tensors exist)."""
    return int(np.size(w_gate) + np.size(w_up) + np.size(w_down))


# --------------------------------------------------------------------------
# Decoder block — [LMDrive] §2.5 and the chapter-02 equation of [Mechanics]:
#   X' = X + Attn(RMSNorm_1(X)),  X'' = X' + SwiGLU(RMSNorm_2(X')).
# --------------------------------------------------------------------------
def _split_heads(y: np.ndarray, n: int, dh: int) -> np.ndarray:
    """[B, T, n*dh] -> [B, n, T, dh] (view(B,T,n,dh).transpose(1,2))."""
    B, T, _ = y.shape
    return y.reshape(B, T, n, dh).transpose(0, 2, 1, 3)


def _merge_heads(o: np.ndarray) -> np.ndarray:
    """[B, n, T, dh] -> [B, T, n*dh] (transpose(1,2).reshape)."""
    B, n, T, dh = o.shape
    return o.transpose(0, 2, 1, 3).reshape(B, T, n * dh)


def block_prefill(X, W: dict, n_heads: int, n_kv_heads: int, head_dim: int,
                  eps: float, rope_base: float, rows=None) -> dict:
    """Prefill forward of one block over X [B, T, d], positions 0..T-1.

    W holds wq, wk, wv, wo, w_gate, w_up, w_down ([out, in]) and g_attn, g_mlp.
    ``rows``: optional token rows (shared by every batch row) at which the
    query side, o_proj and the MLP are evaluated; K and V are always computed
    for every token since attention needs them.

    Returns a dict: y (X''), x1 (X'), attn (o_proj output, the attention
    branch), mlp (the MLP branch), o (attention output before o_proj,
    [B, rows, H*d_h]), k, v (post-RoPE keys and values, [B, H_kv, T, d_h]:
    what the KV cache holds), rows.
    """
    X = _f64(X)
    B, T, d = X.shape
    rows = list(range(T)) if rows is None else list(rows)
    H, Hkv, dh = n_heads, n_kv_heads, head_dim

    h = rmsnorm(X, W["g_attn"], eps)
    k = _split_heads(linear(h, W["wk"]), Hkv, dh)
    v = _split_heads(linear(h, W["wv"]), Hkv, dh)
    q = _split_heads(linear(h[:, rows, :], W["wq"]), H, dh)
    pos_all = np.arange(T, dtype=np.float64)
    k = apply_rope(k, pos_all[None, None, :], rope_base)
    q = apply_rope(q, np.asarray(rows, dtype=np.float64)[None, None, :], rope_base)

    # Attention over the full K/V for the selected query rows. The mask uses
    # the absolute row index, so embed the selected queries at their rows.
    o = _attend_rows(q, k, v, rows, T)
    o_flat = _merge_heads(o)
    attn = linear(o_flat, W["wo"])
    x1 = X[:, rows, :] + attn

    h2 = rmsnorm(x1, W["g_mlp"], eps)
    mlp = swiglu_mlp(h2, W["w_gate"], W["w_up"], W["w_down"])
    y = x1 + mlp
    return {"y": y, "x1": x1, "attn": attn, "mlp": mlp, "o": o_flat,
            "k": k, "v": v, "rows": rows}


def _attend_rows(q_sel, k, v, rows, T):
    """Causal attention for queries that sit at absolute rows ``rows`` of a
    length-T sequence; q_sel is [B, H, len(rows), dh]."""
    B, H, R, dh = q_sel.shape
    q_full = np.zeros((B, H, T, dh))
    q_full[:, :, rows, :] = q_sel
    return causal_attention(q_full, k, v, rows=rows)


def block_decode(x, W: dict, n_heads: int, n_kv_heads: int, head_dim: int,
                 eps: float, rope_base: float, k_cache, v_cache, cache_len) -> dict:
    """One decode step: x [B, 1, d]; sequence b has ``cache_len[b]`` cached
    (post-RoPE) keys/values in k_cache/v_cache [B, H_kv, >=len, d_h].

    Following chapter 04 of [Mechanics]: only the new token's q, k, v are
    computed, at position cache_len[b]; k, v are appended; q attends to all
    cache_len[b] + 1 keys. Returns y [B,1,d], the new k/v [B,H_kv,1,d_h], and
    the branch outputs.
    """
    x = _f64(x)
    kc, vc = _f64(k_cache), _f64(v_cache)
    B, one, d = x.shape
    assert one == 1
    H, Hkv, dh = n_heads, n_kv_heads, head_dim
    lens = [int(t) for t in np.asarray(cache_len).reshape(-1)]

    h = rmsnorm(x, W["g_attn"], eps)
    q = _split_heads(linear(h, W["wq"]), H, dh)
    k = _split_heads(linear(h, W["wk"]), Hkv, dh)
    v = _split_heads(linear(h, W["wv"]), Hkv, dh)
    o = np.empty((B, H, 1, dh))
    k_new = np.empty_like(k)
    v_new = np.empty_like(v)
    for b in range(B):
        L = lens[b]
        pos = np.full((1, 1, 1), float(L))
        qb = apply_rope(q[b:b + 1], pos, rope_base)
        kb = apply_rope(k[b:b + 1], pos, rope_base)
        k_new[b], v_new[b] = kb[0], v[b]
        K_all = np.concatenate([kc[b:b + 1, :, :L], kb], axis=2)
        V_all = np.concatenate([vc[b:b + 1, :, :L], v[b:b + 1]], axis=2)
        o[b:b + 1] = causal_attention(qb, K_all, V_all)
    o_flat = _merge_heads(o)
    attn = linear(o_flat, W["wo"])
    x1 = x + attn
    h2 = rmsnorm(x1, W["g_mlp"], eps)
    mlp = swiglu_mlp(h2, W["w_gate"], W["w_up"], W["w_down"])
    return {"y": x1 + mlp, "x1": x1, "attn": attn, "mlp": mlp, "o": o_flat,
            "k_new": k_new, "v_new": v_new}


def block_extend(x, W: dict, n_heads: int, n_kv_heads: int, head_dim: int, eps: float,
                 rope_base: float, k_cache, v_cache, L: int) -> dict:
    """Append T new tokens x [B, T, d] to sequences that already hold L cached
    (post-RoPE) keys/values each (chunked prefill). The new tokens sit at
    positions L .. L+T-1 (mechanics page chapter 04: positions follow the cache
    length); token i attends to the L cached keys and to new tokens 0..i.
    Returns y [B, T, d], the new keys/values k_new, v_new [B, H_kv, T, d_h] and
    the branch outputs."""
    x = _f64(x)
    kc, vc = _f64(k_cache), _f64(v_cache)
    B, T, d = x.shape
    H, Hkv, dh = n_heads, n_kv_heads, head_dim
    h = rmsnorm(x, W["g_attn"], eps)
    q = _split_heads(linear(h, W["wq"]), H, dh)
    k = _split_heads(linear(h, W["wk"]), Hkv, dh)
    v = _split_heads(linear(h, W["wv"]), Hkv, dh)
    pos = (L + np.arange(T, dtype=np.float64))[None, None, :]
    q = apply_rope(q, pos, rope_base)
    k = apply_rope(k, pos, rope_base)
    K_all = np.concatenate([kc[:, :, :L], k], axis=2)
    V_all = np.concatenate([vc[:, :, :L], v], axis=2)
    o = causal_attention(q, K_all, V_all)  # queries sit at the last T positions
    o_flat = _merge_heads(o)
    attn = linear(o_flat, W["wo"])
    x1 = x + attn
    h2 = rmsnorm(x1, W["g_mlp"], eps)
    mlp = swiglu_mlp(h2, W["w_gate"], W["w_up"], W["w_down"])
    return {"y": x1 + mlp, "x1": x1, "attn": attn, "mlp": mlp, "o": o_flat,
            "k_new": k, "v_new": v}


# --------------------------------------------------------------------------
# Tensor parallelism — [Llama-MLP] §6.3: with Q/K/V and gate/up split by output rows
# and o_proj and down by input columns, every rank's branch output is a partial sum;
# an all-reduce over ranks completes the branch. A rank's slice is itself a block
# with n_heads / W query heads, n_kv_heads / W KV heads and f / W intermediate columns.
# --------------------------------------------------------------------------
def tp_attention_partial(X, Ws: dict, n_heads: int, n_kv_heads: int, head_dim: int, eps: float,
                         rope_base: float) -> dict:
    """One rank's attention-branch partial of a prefill (its heads' attention times its
    o_proj columns, no residual) and the K/V of its heads."""
    out = block_prefill(X, Ws, n_heads, n_kv_heads, head_dim, eps, rope_base)
    return {"o": out["attn"], "k": out["k"], "v": out["v"]}


def tp_attention_partial_decode(x, Ws: dict, n_heads: int, n_kv_heads: int, head_dim: int,
                                eps: float, rope_base: float, k_cache, v_cache, cache_len) -> dict:
    """One rank's attention-branch partial of a decode step over its heads' cache."""
    out = block_decode(x, Ws, n_heads, n_kv_heads, head_dim, eps, rope_base, k_cache, v_cache,
                       cache_len)
    return {"o": out["attn"], "k_new": out["k_new"], "v_new": out["v_new"]}


def tp_mlp_partial(X1, Ws: dict, eps: float) -> np.ndarray:
    """One rank's MLP-branch partial: SwiGLU over its intermediate columns of the full
    RMSNorm(X'), times its down columns."""
    return swiglu_mlp(rmsnorm(X1, Ws["g_mlp"], eps), Ws["w_gate"], Ws["w_up"], Ws["w_down"])


# --------------------------------------------------------------------------
# A stack of blocks — the "x L blocks" of the chapter-02 diagram of [Mechanics]
# and the 32 decoder layers of [LMDrive] §1/§5: layer l's output is layer l+1's
# input; each layer has its own KV cache.
# --------------------------------------------------------------------------
def stack_prefill(X, Ws: list, n_heads: int, n_kv_heads: int, head_dim: int, eps: float,
                  rope_base: float) -> dict:
    """Prefill through len(Ws) layers. Returns y and the per-layer caches."""
    h = _f64(X)
    ks, vs = [], []
    for W in Ws:
        out = block_prefill(h, W, n_heads, n_kv_heads, head_dim, eps, rope_base)
        h = out["y"]
        ks.append(out["k"])
        vs.append(out["v"])
    return {"y": h, "k": ks, "v": vs}


def stack_extend(x, Ws: list, n_heads: int, n_kv_heads: int, head_dim: int, eps: float,
                 rope_base: float, k_caches: list, v_caches: list, L: int) -> dict:
    """Append T tokens through every layer (each layer reads its own cache)."""
    h = _f64(x)
    ks, vs = [], []
    for W, kc, vc in zip(Ws, k_caches, v_caches):
        out = block_extend(h, W, n_heads, n_kv_heads, head_dim, eps, rope_base, kc, vc, L)
        h = out["y"]
        ks.append(out["k_new"])
        vs.append(out["v_new"])
    return {"y": h, "k_new": ks, "v_new": vs}


# --------------------------------------------------------------------------
# Weight-only INT8 for decode ("深入解析Llama MLP模块" §6.4 recommends INT8 weights to
# cut inference memory; the page gives no scheme). Reading taken: symmetric,
# per output row (per nn.Linear output feature): s = max|w| / 127, q = rint(w / s)
# in [-127, 127], w ~ s * q. The scale and the rounding decide integers, so they
# are taken in fp32 exactly as the GPU takes them (IEEE division, round half to
# even); everything after that is fp64.
# --------------------------------------------------------------------------
def quantize_int8_rows(w):
    """Per-row symmetric INT8 codes and fp32 scales of a weight matrix [out, in]."""
    w32 = np.asarray(_f64(w), dtype=np.float32)
    amax = np.max(np.abs(w32), axis=1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint(w32 / safe[:, None]).astype(np.float32)
    q = np.clip(q, -127, 127)
    q = np.where(s[:, None] > 0, q, 0).astype(np.int8)
    return q, s


def dequantize_int8_rows(q, s) -> np.ndarray:
    return np.asarray(s, dtype=np.float64)[:, None] * np.asarray(q, dtype=np.float64)


def int8_decode_weights(W: dict) -> dict:
    """The block weights as the INT8 decode path sees them: every projection
    replaced by its dequantized INT8 form (RMSNorm gains unchanged)."""
    out = dict(W)
    for k in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
        out[k] = dequantize_int8_rows(*quantize_int8_rows(W[k]))
    return out


# --------------------------------------------------------------------------
# KV-cache memory accounting — [Mechanics] chapter 04, "MEMORY ACCOUNTING":
#   bytes = L x 2 x B x T x H_kv x d_h x bytes(dtype)
# --------------------------------------------------------------------------
def kv_cache_bytes(layers: int, B: int, T: int, n_kv_heads: int, head_dim: int,
                   dtype_bytes: int) -> int:
    return layers * 2 * B * T * n_kv_heads * head_dim * dtype_bytes
