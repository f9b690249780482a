"""Python binding of libi4rt: INT4 weight-only batch-1 decode on B200 (sm_100a).

Argument marshalling only. Every computation runs in the CUDA kernels of
``libi4rt.so`` (built by ``python -m int4_weight_only_02_b200.build``); there
is no CPU or PyTorch fallback, and a missing library raises at first use.
PyTorch provides device memory and streams: tensors are passed by
``data_ptr()``, and calls run on ``torch.cuda.current_stream()`` unless a
stream is given.

Layouts (see include/i4rt.h): INT4 weights [N][K/8] uint32 (8 consecutive k
per word, field i at bits 4i..4i+3, two's complement), fp16 group-128 scales
[N][K/128], KV pools [pages][kv heads][page_size][128] fp16.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libi4rt.so")
_lib = None

I4_OK, I4_EINVAL, I4_EALIGN, I4_EUNSUPPORTED, I4_ECUDA, I4_ENOMEM = 0, -1, -2, -3, -4, -5

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class I4Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"i4rt status {status}: {msg}")
        self.status = status


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", _i), ("hidden", _i), ("intermediate", _i), ("n_q_heads", _i), ("n_kv_heads", _i),
                ("head_dim", _i), ("vocab", _i), ("group", _i), ("page_size", _i), ("max_ctx", _i),
                ("rope_theta", _f), ("rms_eps", _f)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("w_qkv", "s_qkv", "b_qkv", "w_o", "s_o", "w_gate_up", "s_gate_up", "w_down",
                                   "s_down", "ln_in", "ln_post")]


class ModelWeights(ctypes.Structure):
    _fields_ = [("embed", _vp), ("layers", ctypes.POINTER(LayerWeights)), ("ln_final", _vp), ("w_lm", _vp),
                ("s_lm", _vp)]


class SeqState(ctypes.Structure):
    _fields_ = [("token", _vp), ("pos", _vp), ("ctx_len", _vp), ("page_table", _vp),
                ("k_pools", ctypes.POINTER(_vp)), ("v_pools", ctypes.POINTER(_vp)), ("num_pages", _i),
                ("logits", _vp), ("prompt", _vp), ("n_prompt", _i), ("history", _vp), ("status", _vp)]


class RmsnormRopeArgs(ctypes.Structure):
    _fields_ = [("x_in", _vp), ("resid", _vp), ("gamma", _vp), ("out", _vp), ("M", _i), ("H", _i), ("eps", _f),
                ("qkv", _vp), ("pos", _vp), ("B", _i), ("Hq", _i), ("Hkv", _i), ("D", _i), ("theta", _f),
                ("k_pool", _vp), ("v_pool", _vp), ("page_table", _vp), ("page_size", _i),
                ("max_pages_per_seq", _i)]


_SIGS = {
    "i4_last_error": (ctypes.c_char_p, []),
    "i4_version": (ctypes.c_char_p, []),
    "int4_gemv": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "int4_gemm": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "int4_gemm_ws_bytes": (_sz, [_i, _i, _i]),
    "i4_int4_gemv_variant": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "i4_int4_unpack": (_i, [_vp, _vp, _i, _i, _vp]),
    "paged_gqa_decode_ws_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "paged_gqa_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "paged_gqa_decode_static": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "i4_paged_gqa_decode_strided": (_i, [_vp, ctypes.c_longlong, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                         _f, _vp, _sz, _vp]),
    "i4_embed_gather": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "i4_argmax_rows": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "i4_paged_gather": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "rmsnorm_rope": (_i, [ctypes.POINTER(RmsnormRopeArgs), _vp]),
    "i4_rmsnorm": (_i, [_vp, _vp, _vp, _vp, _i, _i, _f, _vp]),
    "i4_rope_kv_append": (_i, [_vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp, _i, _i, _vp]),
    "silu_mul": (_i, [_vp, _vp, _i, _i, _vp]),
    "decode_step_graph_create": (_i, [ctypes.POINTER(ModelDesc), ctypes.POINTER(ModelWeights),
                                      ctypes.POINTER(SeqState), ctypes.POINTER(_vp)]),
    "decode_step_graph_replay": (_i, [_vp, _vp]),
    "decode_step_eager": (_i, [_vp, _vp]),
    "decode_step_kernel_count": (_i, [_vp]),
    "decode_step_phase_count": (_i, [_vp]),
    "decode_step_is_persistent": (_i, [_vp]),
    "decode_step_trace": (_i, [_vp, ctypes.POINTER(ctypes.c_ulonglong), _sz]),
    "decode_step_graph_destroy": (_i, [_vp]),
    "decode_step_launch_kernel": (_i, [_vp, _i, _vp]),
    "decode_step_buffer_copy": (_i, [_vp, _i, _vp, _sz, _i, _vp]),
    "i4_set_option": (_i, [ctypes.c_char_p, _i]),
    "i4_device_error": (_i, [_i]),
}


def lib() -> ctypes.CDLL:
    """Load libi4rt.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libi4rt.so not found at {LIB_PATH}; build it with "
                               "`python -m int4_weight_only_02_b200.build` (nvcc, sm_100a)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def exported_symbols():
    return sorted(_SIGS)


def _check(status: int, name: str):
    if status != I4_OK:
        raise I4Error(status, f"{name}: {lib().i4_last_error().decode()}")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def device_error(reset: bool = True) -> int:
    """0, or 1 when a bounded in-kernel wait gave up (synchronises the device)."""
    v = int(lib().i4_device_error(int(reset)))
    if v < 0:
        _check(v, "i4_device_error")
    return v


def set_option(name: str, value: int):
    _check(lib().i4_set_option(name.encode(), int(value)), "i4_set_option")


# ------------------------------------------------------------------ kernels

def int4_gemv(w, scales, x, bias=None, y=None, out_fp32: bool = False, group: int = 128, stream=None,
              unpack: int | None = None, max_ctas: int = 0):
    """y[M][N] = x[M][K] . dequant(w, scales)^T (+ bias), fp32 accumulation."""
    import torch
    x2 = x if x.dim() == 2 else x.view(1, -1)
    M, K = x2.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), device=x.device, dtype=torch.float32 if out_fp32 else torch.float16)
    if unpack is None and max_ctas == 0:
        st = lib().int4_gemv(_p(w), _p(scales), _p(x2), _p(bias), _p(y), int(out_fp32), M, N, K, group,
                             _stream(stream))
    else:
        st = lib().i4_int4_gemv_variant(_p(w), _p(scales), _p(x2), _p(bias), _p(y), int(out_fp32), M, N, K,
                                        0 if unpack is None else unpack, max_ctas, _stream(stream))
    _check(st, "int4_gemv")
    return y if x.dim() == 2 else y.view(-1)


def int4_gemm_ws_bytes(M: int, N: int, K: int) -> int:
    return int(lib().int4_gemm_ws_bytes(M, N, K))


def int4_gemm(w, scales, x, bias=None, y=None, out_fp32: bool = False, group: int = 128, ws=None, stream=None):
    """y[M][N] = x[M][K] . dequant(w, scales)^T (+ bias) on the tcgen05 tensor cores (any M). With `ws` (a
    zeroed uint8 device tensor of at least int4_gemm_ws_bytes(M, N, K) bytes) K may be split over CTAs."""
    import torch
    M, K = x.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), device=x.device, dtype=torch.float32 if out_fp32 else torch.float16)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().int4_gemm(_p(w), _p(scales), _p(x), _p(bias), _p(y), int(out_fp32), M, N, K, group, _p(ws), nb,
                           _stream(stream)), "int4_gemm")
    return y


def int4_unpack(w, K: int, stream=None):
    import torch
    q = torch.empty((w.shape[0], K), device=w.device, dtype=torch.int8)
    _check(lib().i4_int4_unpack(_p(w), _p(q), w.shape[0], K, _stream(stream)), "i4_int4_unpack")
    return q


def paged_gqa_decode_ws_bytes(B, Hq, Hkv, D, page_size, max_pages_per_seq) -> int:
    return int(lib().paged_gqa_decode_ws_bytes(B, Hq, Hkv, D, page_size, max_pages_per_seq))


def paged_gqa_decode(q, k_pool, v_pool, page_table, ctx_len, out=None, scale=None, ws=None, stream=None):
    """out [B][Hq][D] fp16; the workspace is allocated zeroed when not given."""
    import torch
    B, Hq, D = q.shape
    _, Hkv, P, _ = k_pool.shape
    max_pages = page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    nbytes = paged_gqa_decode_ws_bytes(B, Hq, Hkv, D, P, max_pages)
    if ws is None:
        ws = torch.zeros(nbytes, device=q.device, dtype=torch.uint8)
    scale = 1.0 / D ** 0.5 if scale is None else scale
    _check(lib().paged_gqa_decode(_p(q), _p(k_pool), _p(v_pool), _p(page_table), _p(ctx_len), _p(out), B, Hq, Hkv, D,
                                  P, max_pages, float(scale), _p(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "paged_gqa_decode")
    return out


def paged_gqa_decode_static(q, k_pool, v_pool, page_table, ctx_len, out=None, scale=None, stream=None):
    """paged_gqa_decode with the library's fixed device scratch instead of a workspace (allocates nothing
    besides `out` when it is not given)."""
    import torch
    B, Hq, D = q.shape
    _, Hkv, P, _ = k_pool.shape
    if out is None:
        out = torch.empty_like(q)
    scale = 1.0 / D ** 0.5 if scale is None else scale
    _check(lib().paged_gqa_decode_static(_p(q), _p(k_pool), _p(v_pool), _p(page_table), _p(ctx_len), _p(out), B, Hq,
                                         Hkv, D, P, page_table.shape[1], float(scale), _stream(stream)),
           "paged_gqa_decode_static")
    return out


def paged_gqa_decode_strided(q, q_stride: int, Hq: int, k_pool, v_pool, page_table, ctx_len, out, ws, scale=None,
                             stream=None):
    """paged_gqa_decode reading the q rows of sequence b at q[b * q_stride ...] (e.g. inside qkv rows)."""
    B = page_table.shape[0]
    _, Hkv, P, D = k_pool.shape
    scale = 1.0 / D ** 0.5 if scale is None else scale
    _check(lib().i4_paged_gqa_decode_strided(_p(q), int(q_stride), _p(k_pool), _p(v_pool), _p(page_table),
                                             _p(ctx_len), _p(out), B, Hq, Hkv, D, P, page_table.shape[1],
                                             float(scale), _p(ws), ws.numel() * ws.element_size(),
                                             _stream(stream)), "i4_paged_gqa_decode_strided")
    return out


def embed_gather(table, tokens, out, stream=None):
    """out[b] = table[tokens[b]] (token ids clamped to the table)."""
    V, H = table.shape
    _check(lib().i4_embed_gather(_p(table), _p(tokens), _p(out), tokens.numel(), H, V, _stream(stream)),
           "i4_embed_gather")
    return out


def argmax_rows(logits, tokens, pos=None, ctx_len=None, stream=None):
    """tokens[b] = argmax(logits[b]) (lowest index on ties); pos and ctx_len advance by one when given."""
    B, N = logits.shape
    _check(lib().i4_argmax_rows(_p(logits), _p(tokens), _p(pos), _p(ctx_len), B, N, _stream(stream)),
           "i4_argmax_rows")
    return tokens


def paged_gather(pool, page_table, ctx_len, max_ctx: int, out=None, stream=None):
    import torch
    _, Hkv, P, D = pool.shape
    B, max_pages = page_table.shape
    if out is None:
        out = torch.zeros((B, Hkv, max_ctx, D), device=pool.device, dtype=pool.dtype)
    _check(lib().i4_paged_gather(_p(pool), _p(page_table), _p(ctx_len), _p(out), B, Hkv, D, P, max_pages, max_ctx,
                                 _stream(stream)), "i4_paged_gather")
    return out


def rmsnorm(x, gamma, out=None, resid=None, eps: float = 1e-6, stream=None):
    import torch
    x2 = x if x.dim() == 2 else x.view(1, -1)
    if out is None:
        out = torch.empty_like(x2)
    _check(lib().i4_rmsnorm(_p(x2), _p(resid), _p(gamma), _p(out), x2.shape[0], x2.shape[1], float(eps),
                            _stream(stream)), "i4_rmsnorm")
    return out if x.dim() == 2 else out.view(-1)


def rope_kv_append(qkv, pos, Hq: int, Hkv: int, theta: float = 1e6, k_pool=None, v_pool=None, page_table=None,
                   stream=None):
    """Rotates the q and k heads of qkv [B][(Hq+2Hkv)*128] in place; appends k, v to the pools when given."""
    B = qkv.shape[0] if qkv.dim() == 2 else 1
    P = k_pool.shape[2] if k_pool is not None else 0
    max_pages = page_table.shape[-1] if page_table is not None else 0
    _check(lib().i4_rope_kv_append(_p(qkv), _p(pos), B, Hq, Hkv, 128, float(theta), _p(k_pool), _p(v_pool),
                                   _p(page_table), P, max_pages, _stream(stream)), "i4_rope_kv_append")
    return qkv


def rmsnorm_rope(args: RmsnormRopeArgs, stream=None):
    _check(lib().rmsnorm_rope(ctypes.byref(args), _stream(stream)), "rmsnorm_rope")


def silu_mul(gate_up, out=None, stream=None):
    import torch
    g2 = gate_up if gate_up.dim() == 2 else gate_up.view(1, -1)
    M, I2 = g2.shape
    if out is None:
        out = torch.empty((M, I2 // 2), device=gate_up.device, dtype=torch.float16)
    _check(lib().silu_mul(_p(g2), _p(out), M, I2 // 2, _stream(stream)), "silu_mul")
    return out if gate_up.dim() == 2 else out.view(-1)


from .runtime import BatchedDecode, DecodeGraph, DeviceModel, Prefill, Sequence  # noqa: E402,F401
