"""Python binding of the B200 LLaMA pre-norm decoder block library.

A thin ctypes layer over ``libllama_block.so`` (the C ABI declared in
``include/llama_block.h``): every function here has the C name, checks and
marshals its arguments (torch tensors -> device pointers, the current CUDA
stream -> ``cudaStream_t``) and raises :class:`LlamaBlockError` on a non-OK
status. All computation runs in the library's CUDA kernels; there is no CPU
path, and importing this package fails loudly when the library is not built.
"""

from __future__ import annotations

import ctypes
import os
from pathlib import Path

import torch

__all__ = [
    "LB_F32", "LB_BF16", "LlamaBlockError", "lib", "lib_path", "dtype_code",
    "llama_block_create", "llama_block_set_weights", "llama_block_reserve",
    "llama_block_quantize_decode_weights", "llama_block_set_rope_dynamic_ntk",
    "llama_block_prefill", "llama_block_extend", "llama_block_decode", "llama_block_set_lengths",
    "llama_block_kv_cache_bytes", "llama_block_sync_status", "llama_block_destroy",
    "llama_block_last_error", "llama_block_selftest_timeout", "llama_block_enable_timing",
    "llama_block_stage_times", "llama_block_stage_name", "llama_block_launch_count",
    "rmsnorm", "rope_apply", "causal_attn", "swiglu_mlp", "decode_attn_static_scratch", "LlamaBlock",
    "llama_stack_create", "llama_stack_layer", "llama_stack_prefill", "llama_stack_extend",
    "llama_stack_decode", "llama_stack_set_lengths", "llama_stack_destroy", "LlamaStack",
    "llama_block_tp_attn_prefill", "llama_block_tp_attn_decode", "llama_block_tp_mlp",
    "llama_block_tp_add", "tp_shard_weights",
]

LB_F32, LB_BF16 = 0, 1
STATUS = {0: "LB_OK", 1: "LB_ERR_INVALID_ARG", 2: "LB_ERR_UNSUPPORTED", 3: "LB_ERR_CUDA",
          4: "LB_ERR_OOM", 5: "LB_ERR_CACHE_FULL", 6: "LB_ERR_TIMEOUT", 7: "LB_ERR_NO_WEIGHTS"}

lib_path = Path(os.environ.get("LLAMA_BLOCK_LIB", Path(__file__).resolve().parent / "libllama_block.so"))
if not lib_path.exists():
    raise ImportError(
        f"llama_pre_norm_b200: CUDA library {lib_path} is not built "
        "(run `python llama_pre_norm_b200/build.py`); there is no fallback path")
lib = ctypes.CDLL(str(lib_path))

_p, _i, _f, _sz, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_longlong
_pp = ctypes.POINTER(ctypes.c_void_p)
_SIGS = {
    "llama_block_create": (_i, [_i, _i, _i, _i, _i, _f, _f, _i, _i, _pp]),
    "llama_block_set_weights": (_i, [_p] * 11),
    "llama_block_reserve": (_i, [_p, _i, _i]),
    "llama_block_quantize_decode_weights": (_i, [_p, _i, _p]),
    "llama_block_set_rope_dynamic_ntk": (_i, [_p, _f, _i, _p]),
    "llama_block_tp_attn_prefill": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p]),
    "llama_block_tp_attn_decode": (_i, [_p, _p, _p, _i, _p, _p, _i, _p, _p]),
    "llama_block_tp_mlp": (_i, [_p, _p, _p, _p, _p, _i, _p]),
    "llama_block_tp_add": (_i, [_p, _p, _p, _i, _i, _i, _p]),
    "llama_block_prefill": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p]),
    "llama_block_extend": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p]),
    "llama_block_decode": (_i, [_p, _p, _p, _i, _p, _p, _i, _p, _p]),
    "llama_stack_create": (_i, [_i, _i, _i, _i, _i, _i, _f, _f, _i, _i, _pp]),
    "llama_stack_layer": (_p, [_p, _i]),
    "llama_stack_prefill": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p]),
    "llama_stack_extend": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p]),
    "llama_stack_decode": (_i, [_p, _p, _p, _i, _p, _p, _i, _p, _p]),
    "llama_stack_set_lengths": (_i, [_p, _p, _i]),
    "llama_stack_destroy": (None, [_p]),
    "llama_block_set_lengths": (_i, [_p, _p, _i]),
    "llama_block_kv_cache_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "llama_block_sync_status": (_i, [_p, _p]),
    "llama_block_destroy": (None, [_p]),
    "llama_block_last_error": (ctypes.c_char_p, []),
    "llama_block_selftest_timeout": (_i, [_ll, _p]),
    "llama_block_enable_timing": (_i, [_p, _i]),
    "llama_block_stage_times": (_i, [_p, _p, _i, ctypes.POINTER(ctypes.c_int)]),
    "llama_block_stage_name": (ctypes.c_char_p, [_p, _i]),
    "llama_block_launch_count": (ctypes.c_ulonglong, [_p]),
    "rmsnorm": (_i, [_p, _p, _p, _i, _i, _f, _i, _p]),
    "rope_apply": (_i, [_p, _p, _i, _i, _i, _i, _f, _i, _p]),
    "causal_attn": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p]),
    "swiglu_mlp": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _p]),
    "decode_attn_static_scratch": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class LlamaBlockError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        msg = lib.llama_block_last_error().decode(errors="replace")
        super().__init__(f"{where}: {self.name}: {msg}")


def _check(st: int, where: str) -> None:
    if st != 0:
        raise LlamaBlockError(st, where)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return LB_F32
    if dt == torch.bfloat16:
        return LB_BF16
    raise TypeError(f"unsupported dtype {dt} (float32 or bfloat16)")


def _ptr(t: torch.Tensor | None, name: str, dtype=None) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ----------------------------------------------------------------- handle API
def llama_block_create(d, n_heads, n_kv_heads, head_dim, f, eps, rope_base, dtype, max_pos) -> int:
    out = ctypes.c_void_p()
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    _check(lib.llama_block_create(d, n_heads, n_kv_heads, head_dim, f, eps, rope_base, code, max_pos,
                                  ctypes.byref(out)), "llama_block_create")
    return out.value


def llama_block_set_weights(h, wq, wk, wv, wo, w_gate, w_up, w_down, g_attn, g_mlp, stream=None):
    dt = wq.dtype
    ptrs = [_ptr(t, n, dt) for t, n in ((wq, "wq"), (wk, "wk"), (wv, "wv"), (wo, "wo"),
                                         (w_gate, "w_gate"), (w_up, "w_up"), (w_down, "w_down"),
                                         (g_attn, "g_attn"), (g_mlp, "g_mlp"))]
    _check(lib.llama_block_set_weights(h, *ptrs, _stream(stream)), "llama_block_set_weights")


def llama_block_quantize_decode_weights(h, enable=True, stream=None):
    _check(lib.llama_block_quantize_decode_weights(h, 1 if enable else 0, _stream(stream)),
           "llama_block_quantize_decode_weights")


def llama_block_set_rope_dynamic_ntk(h, factor, original_max_pos, stream=None):
    """Dynamic NTK RoPE scaling (see the C header); original_max_pos = 0 turns it off."""
    _check(lib.llama_block_set_rope_dynamic_ntk(h, float(factor), int(original_max_pos), _stream(stream)),
           "llama_block_set_rope_dynamic_ntk")


def llama_block_reserve(h, max_tokens, max_batch):
    _check(lib.llama_block_reserve(h, max_tokens, max_batch), "llama_block_reserve")


def llama_block_prefill(h, x, y, k_cache, v_cache, cache_len, stream=None):
    B, T, _ = x.shape
    t_max = k_cache.shape[2]
    _check(lib.llama_block_prefill(h, _ptr(x, "x"), _ptr(y, "y", x.dtype), B, T,
                                   _ptr(k_cache, "k_cache", x.dtype), _ptr(v_cache, "v_cache", x.dtype),
                                   t_max, _ptr(cache_len, "cache_len", torch.int32), _stream(stream)),
           "llama_block_prefill")


def llama_block_extend(h, x, y, k_cache, v_cache, cache_len, stream=None):
    B, T, _ = x.shape
    t_max = k_cache.shape[2]
    _check(lib.llama_block_extend(h, _ptr(x, "x"), _ptr(y, "y", x.dtype), B, T,
                                  _ptr(k_cache, "k_cache", x.dtype), _ptr(v_cache, "v_cache", x.dtype),
                                  t_max, _ptr(cache_len, "cache_len", torch.int32), _stream(stream)),
           "llama_block_extend")


def llama_block_decode(h, x, y, k_cache, v_cache, cache_len, stream=None):
    B = x.shape[0]
    t_max = k_cache.shape[2]
    _check(lib.llama_block_decode(h, _ptr(x, "x"), _ptr(y, "y", x.dtype), B,
                                  _ptr(k_cache, "k_cache", x.dtype), _ptr(v_cache, "v_cache", x.dtype),
                                  t_max, _ptr(cache_len, "cache_len", torch.int32), _stream(stream)),
           "llama_block_decode")


# ----------------------------------------------------------------- tensor parallelism
def tp_shard_weights(W: dict, rank: int, world: int, n_heads: int, n_kv_heads: int,
                     head_dim: int) -> dict:
    """Rank `rank`'s slice of a block's nn.Linear weights ("深入解析Llama MLP模块" page
    §6.3, Megatron split): q/k/v rows of its heads and gate/up rows of its intermediate
    columns (column-parallel), o_proj and down columns of the same (row-parallel); the
    RMSNorm gains whole. Argument slicing only; the shard handle is created with
    (d, n_heads // world, n_kv_heads // world, head_dim, f // world)."""
    f = W["w_gate"].shape[0]
    if n_heads % world or n_kv_heads % world or f % world:
        raise ValueError("n_heads, n_kv_heads and f must divide by the number of ranks")
    hq, hk, fs = n_heads // world, n_kv_heads // world, f // world
    q0, k0, f0 = rank * hq * head_dim, rank * hk * head_dim, rank * fs
    return {
        "wq": W["wq"][q0:q0 + hq * head_dim].contiguous(),
        "wk": W["wk"][k0:k0 + hk * head_dim].contiguous(),
        "wv": W["wv"][k0:k0 + hk * head_dim].contiguous(),
        "wo": W["wo"][:, q0:q0 + hq * head_dim].contiguous(),
        "w_gate": W["w_gate"][f0:f0 + fs].contiguous(),
        "w_up": W["w_up"][f0:f0 + fs].contiguous(),
        "w_down": W["w_down"][:, f0:f0 + fs].contiguous(),
        "g_attn": W["g_attn"], "g_mlp": W["g_mlp"],
    }


def llama_block_tp_attn_prefill(h, x, o_part, k_cache, v_cache, cache_len, stream=None):
    B, T, _ = x.shape
    _check(lib.llama_block_tp_attn_prefill(h, _ptr(x, "x"), _ptr(o_part, "o_part", x.dtype), B, T,
                                           _ptr(k_cache, "k_cache", x.dtype),
                                           _ptr(v_cache, "v_cache", x.dtype), k_cache.shape[2],
                                           _ptr(cache_len, "cache_len", torch.int32), _stream(stream)),
           "llama_block_tp_attn_prefill")


def llama_block_tp_attn_decode(h, x, o_part, k_cache, v_cache, cache_len, stream=None):
    _check(lib.llama_block_tp_attn_decode(h, _ptr(x, "x"), _ptr(o_part, "o_part", x.dtype), x.shape[0],
                                          _ptr(k_cache, "k_cache", x.dtype),
                                          _ptr(v_cache, "v_cache", x.dtype), k_cache.shape[2],
                                          _ptr(cache_len, "cache_len", torch.int32), _stream(stream)),
           "llama_block_tp_attn_decode")


def llama_block_tp_mlp(h, x, o_sum, x1, m_part, stream=None):
    M = x.numel() // x.shape[-1]
    _check(lib.llama_block_tp_mlp(h, _ptr(x, "x"), _ptr(o_sum, "o_sum", x.dtype), _ptr(x1, "x1", x.dtype),
                                  _ptr(m_part, "m_part", x.dtype), M, _stream(stream)),
           "llama_block_tp_mlp")


def llama_block_tp_add(a, b, out, stream=None):
    d = a.shape[-1]
    _check(lib.llama_block_tp_add(_ptr(a, "a"), _ptr(b, "b", a.dtype), _ptr(out, "out", a.dtype),
                                  a.numel() // d, d, dtype_code(a.dtype), _stream(stream)),
           "llama_block_tp_add")


def llama_block_set_lengths(h, lens):
    arr = (ctypes.c_int32 * len(lens))(*[int(v) for v in lens])
    _check(lib.llama_block_set_lengths(h, arr, len(lens)), "llama_block_set_lengths")


def llama_block_kv_cache_bytes(B, n_kv_heads, head_dim, t_max, dtype) -> int:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return int(lib.llama_block_kv_cache_bytes(B, n_kv_heads, head_dim, t_max, code))


def llama_block_sync_status(h=None, stream=None):
    _check(lib.llama_block_sync_status(h, _stream(stream)), "llama_block_sync_status")


def llama_block_destroy(h):
    lib.llama_block_destroy(h)


def llama_block_last_error() -> str:
    return lib.llama_block_last_error().decode(errors="replace")


def llama_block_selftest_timeout(budget_ns: int, stream=None):
    _check(lib.llama_block_selftest_timeout(int(budget_ns), _stream(stream)), "llama_block_selftest_timeout")


def llama_block_enable_timing(h, enable=True):
    _check(lib.llama_block_enable_timing(h, 1 if enable else 0), "llama_block_enable_timing")


def llama_block_stage_times(h) -> list:
    """[(stage name, device ms)] of the last prefill/decode call (timing enabled)."""
    n = ctypes.c_int(0)
    buf = (ctypes.c_float * 16)()
    _check(lib.llama_block_stage_times(h, buf, 16, ctypes.byref(n)), "llama_block_stage_times")
    return [(llama_block_stage_name(h, i), float(buf[i])) for i in range(n.value)]


def llama_block_stage_name(h, i) -> str:
    return lib.llama_block_stage_name(h, i).decode()


def llama_block_launch_count(h) -> int:
    return int(lib.llama_block_launch_count(h))


# ----------------------------------------------------------------- standalone entry points
def rmsnorm(x, g, y, eps, stream=None):
    d = x.shape[-1]
    rows = x.numel() // d
    _check(lib.rmsnorm(_ptr(x, "x"), _ptr(g, "g", x.dtype), _ptr(y, "y", x.dtype), rows, d, eps,
                       dtype_code(x.dtype), _stream(stream)), "rmsnorm")


def rope_apply(x, pos, base, stream=None):
    B, H, T, dh = x.shape
    _check(lib.rope_apply(_ptr(x, "x"), _ptr(pos, "pos", torch.int32), B, T, H, dh, base,
                          dtype_code(x.dtype), _stream(stream)), "rope_apply")


def causal_attn(q, k, v, o, Tk=None, stream=None):
    B, H, Tq, dh = q.shape
    Hkv, k_stride = k.shape[1], k.shape[2]
    Tk = k_stride if Tk is None else Tk
    _check(lib.causal_attn(_ptr(q, "q"), _ptr(k, "k", q.dtype), _ptr(v, "v", q.dtype),
                           _ptr(o, "o", q.dtype), B, Tq, Tk, H, Hkv, dh, k_stride,
                           dtype_code(q.dtype), _stream(stream)), "causal_attn")


def swiglu_mlp(h, w_gate, w_up, w_down, y, stream=None):
    d = h.shape[-1]
    M = h.numel() // d
    f = w_gate.shape[0]
    _check(lib.swiglu_mlp(_ptr(h, "h"), _ptr(w_gate, "w_gate", h.dtype), _ptr(w_up, "w_up", h.dtype),
                          _ptr(w_down, "w_down", h.dtype), _ptr(y, "y", h.dtype), M, d, f,
                          dtype_code(h.dtype), _stream(stream)), "swiglu_mlp")


def decode_attn_static_scratch(q, k, v, o, kv_len, stream=None):
    """Decode attention that allocates no device memory (see the C header).
    q [B, H, head_dim]; k, v [B, H_kv, k_stride, head_dim]; o [B, H * head_dim];
    kv_len int32 [B] (query b sits at position kv_len[b] and sees keys 0..kv_len[b])."""
    B, H, dh = q.shape
    Hkv, ks = k.shape[1], k.shape[2]
    _check(lib.decode_attn_static_scratch(_ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                          _ptr(v, "v", torch.bfloat16), _ptr(o, "o", torch.bfloat16),
                                          _ptr(kv_len, "kv_len", torch.int32), B, H, Hkv, dh, ks,
                                          _stream(stream)), "decode_attn_static_scratch")


class LlamaBlock:
    """Owns a ``llama_block`` handle (create / set_weights / prefill / decode)."""

    def __init__(self, d, n_heads, n_kv_heads, head_dim, f, eps=1e-6, rope_base=10000.0,
                 dtype=torch.bfloat16, max_pos=4096):
        self.d, self.n_heads, self.n_kv_heads, self.head_dim, self.f = d, n_heads, n_kv_heads, head_dim, f
        self.dtype = dtype
        self.max_pos = max_pos
        self.handle = llama_block_create(d, n_heads, n_kv_heads, head_dim, f, eps, rope_base,
                                         dtype_code(dtype), max_pos)

    def set_weights(self, w: dict, stream=None):
        llama_block_set_weights(self.handle, w["wq"], w["wk"], w["wv"], w["wo"], w["w_gate"],
                                w["w_up"], w["w_down"], w["g_attn"], w["g_mlp"], stream)

    def reserve(self, max_tokens, max_batch):
        llama_block_reserve(self.handle, max_tokens, max_batch)

    def quantize_decode_weights(self, enable=True, stream=None):
        llama_block_quantize_decode_weights(self.handle, enable, stream)

    def set_rope_dynamic_ntk(self, factor, original_max_pos, stream=None):
        llama_block_set_rope_dynamic_ntk(self.handle, factor, original_max_pos, stream)

    def prefill(self, x, y, k_cache, v_cache, cache_len, stream=None):
        llama_block_prefill(self.handle, x, y, k_cache, v_cache, cache_len, stream)

    def extend(self, x, y, k_cache, v_cache, cache_len, stream=None):
        llama_block_extend(self.handle, x, y, k_cache, v_cache, cache_len, stream)

    def decode(self, x, y, k_cache, v_cache, cache_len, stream=None):
        llama_block_decode(self.handle, x, y, k_cache, v_cache, cache_len, stream)

    def set_lengths(self, lens):
        llama_block_set_lengths(self.handle, lens)

    def sync_status(self, stream=None):
        llama_block_sync_status(self.handle, stream)

    def enable_timing(self, enable=True):
        llama_block_enable_timing(self.handle, enable)

    def stage_times(self) -> list:
        return llama_block_stage_times(self.handle)

    @property
    def launch_count(self) -> int:
        return llama_block_launch_count(self.handle)

    def close(self):
        if self.handle:
            llama_block_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------- stack of blocks
def _ptr_array(ts, name, dtype):
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t, f"{name}[{i}]", dtype)
    return arr


def llama_stack_create(n_layers, d, n_heads, n_kv_heads, head_dim, f, eps, rope_base, dtype, max_pos) -> int:
    out = ctypes.c_void_p()
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    _check(lib.llama_stack_create(n_layers, d, n_heads, n_kv_heads, head_dim, f, eps, rope_base, code,
                                  max_pos, ctypes.byref(out)), "llama_stack_create")
    return out.value


def llama_stack_layer(st, layer) -> int:
    h = lib.llama_stack_layer(st, layer)
    if not h:
        raise IndexError(f"layer {layer} out of range")
    return h


def _stack_call(fn, name, st, x, y, k_caches, v_caches, cache_len, stream, with_T=True):
    B, T = x.shape[0], x.shape[1]
    t_max = k_caches[0].shape[2]
    args = [st, _ptr(x, "x"), _ptr(y, "y", x.dtype), B]
    if with_T:
        args.append(T)
    args += [_ptr_array(k_caches, "k_caches", x.dtype), _ptr_array(v_caches, "v_caches", x.dtype), t_max,
             _ptr(cache_len, "cache_len", torch.int32), _stream(stream)]
    _check(fn(*args), name)


def llama_stack_prefill(st, x, y, k_caches, v_caches, cache_len, stream=None):
    _stack_call(lib.llama_stack_prefill, "llama_stack_prefill", st, x, y, k_caches, v_caches, cache_len, stream)


def llama_stack_extend(st, x, y, k_caches, v_caches, cache_len, stream=None):
    _stack_call(lib.llama_stack_extend, "llama_stack_extend", st, x, y, k_caches, v_caches, cache_len, stream)


def llama_stack_decode(st, x, y, k_caches, v_caches, cache_len, stream=None):
    _stack_call(lib.llama_stack_decode, "llama_stack_decode", st, x, y, k_caches, v_caches, cache_len, stream,
                with_T=False)


def llama_stack_set_lengths(st, lens):
    arr = (ctypes.c_int32 * len(lens))(*[int(v) for v in lens])
    _check(lib.llama_stack_set_lengths(st, arr, len(lens)), "llama_stack_set_lengths")


def llama_stack_destroy(st):
    lib.llama_stack_destroy(st)


class LlamaStack:
    """Owns a ``llama_stack`` of n_layers blocks (per-layer weights and caches)."""

    def __init__(self, n_layers, d, n_heads, n_kv_heads, head_dim, f, eps=1e-6, rope_base=10000.0,
                 dtype=torch.bfloat16, max_pos=4096):
        self.n_layers = n_layers
        self.handle = llama_stack_create(n_layers, d, n_heads, n_kv_heads, head_dim, f, eps, rope_base,
                                         dtype_code(dtype), max_pos)

    def set_layer_weights(self, layer, w: dict, stream=None):
        h = llama_stack_layer(self.handle, layer)
        llama_block_set_weights(h, w["wq"], w["wk"], w["wv"], w["wo"], w["w_gate"], w["w_up"],
                                w["w_down"], w["g_attn"], w["g_mlp"], stream)

    def quantize_decode_weights(self, enable=True, stream=None):
        """INT8 weight-only decode projections for every layer (or back to bf16)."""
        for layer in range(self.n_layers):
            llama_block_quantize_decode_weights(llama_stack_layer(self.handle, layer), enable, stream)

    def set_rope_dynamic_ntk(self, factor, original_max_pos, stream=None):
        """Dynamic NTK RoPE scaling for every layer (original_max_pos = 0: off)."""
        for layer in range(self.n_layers):
            llama_block_set_rope_dynamic_ntk(llama_stack_layer(self.handle, layer), factor,
                                             original_max_pos, stream)

    def prefill(self, x, y, k_caches, v_caches, cache_len, stream=None):
        llama_stack_prefill(self.handle, x, y, k_caches, v_caches, cache_len, stream)

    def extend(self, x, y, k_caches, v_caches, cache_len, stream=None):
        llama_stack_extend(self.handle, x, y, k_caches, v_caches, cache_len, stream)

    def decode(self, x, y, k_caches, v_caches, cache_len, stream=None):
        llama_stack_decode(self.handle, x, y, k_caches, v_caches, cache_len, stream)

    def set_lengths(self, lens):
        llama_stack_set_lengths(self.handle, lens)

    def close(self):
        if self.handle:
            llama_stack_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
