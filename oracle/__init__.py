"""CPU oracle for the batch-1 INT4 weight-only decode path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It never touches the CUDA library and
the CUDA library never touches it; the two share only the seeded input
generators of ``int4_weight_only_02_b200.synth``.

Everything is computed in float64 from the plain definitions and rounded to
fp16 exactly where the decode step stores a tensor (logits stay fp32). The
heavy loops (the INT4 linear layer and attention) live in ``i4_oracle.c``;
the glue (RMSNorm, RoPE, SiLU-mul, residual add, argmax, the layer order) is
numpy here.

Source pages: "How To Build Your Own LLM Runtime From Scratch". Its
"Technical Details" section lists the pieces (INT4 weight packing and
dequantisation, a paged KV cache, attention with a softmax that must be right
at page tails, a Qwen2.5-Coder-7B decoder of 28 layers, hidden 3584, MLP 18944,
vocabulary 152064, see the model-configuration item of its technical-analysis
section). Where the pages are silent this module takes the plainest reading:

* INT4: 8 consecutive k per uint32, field i in bits 4i..4i+3, two's complement;
  symmetric fp16 scale per row per 128 consecutive k.
* RMSNorm: y = x / sqrt(mean(x^2) + eps) * gamma, one rounding at the end.
* RoPE: rotate-half pairs (i, i + D/2), omega_i = theta^(-2i/D), angle = p*omega_i,
  0-based positions; applied to q and k after the qkv bias.
* Attention: scale 1/sqrt(D), causal including the current token, query head h
  reads kv head h // (n_q / n_kv).
* SiLU-mul: m = g / (1 + exp(-g)) * u.
* Residual: r = fp16(r + fp16(y)).
* Argmax: the lowest index among equal maxima.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against closed forms, invariants and brute force; the composed 28-layer model
is pinned only through its parts (no trained weights, no printed logits).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "i4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``i4_oracle.c`` with gcc (float64, no FP contraction or reassociation)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
    return _lib


def set_threads(n: int = 0) -> int:
    """OpenMP threads of the C loops (0 = leave as is); returns the count in effect (results do not depend
    on it)."""
    return int(lib().o_set_threads(int(n)))


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


_i64 = ctypes.c_int64
_f64 = ctypes.c_double


def f16(a) -> np.ndarray:
    """Round float64 values to fp16 (IEEE round-to-nearest-even)."""
    return np.asarray(a, dtype=np.float64).astype(np.float16)


def f16_c(a: np.ndarray) -> np.ndarray:
    """Round to fp16 through the C helper (pinned against numpy in the tests)."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().o_f64_to_f16(_p(a), _i64(a.size), _p(out))
    return out.view(np.float16)


def widen_c(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.float16)
    out = np.empty(h.shape, dtype=np.float64)
    lib().o_f16_to_f64(_p(h.view(np.uint16)), _i64(h.size), _p(out))
    return out


# ------------------------------------------------------------------ INT4

def unpack_int4(w: np.ndarray, k: int) -> np.ndarray:
    """int8 [N][K] from packed uint32 [N][K/8]."""
    w = np.ascontiguousarray(w, dtype=np.uint32)
    n = w.shape[0]
    assert w.shape[1] * 8 == k
    q = np.empty((n, k), dtype=np.int8)
    lib().o_unpack_int4(_p(w), _i64(n), _i64(k), _p(q))
    return q


def int4_linear(w: np.ndarray, s: np.ndarray, x: np.ndarray, bias=None, group: int = 128) -> np.ndarray:
    """float64 y[M][N] = sum_k q[n][k] s[n][k/group] x[m][k] (+ bias[n]); x is fp16 [M][K] or [K]."""
    w = np.ascontiguousarray(w, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float16)
    x2 = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float16)
    n, k = w.shape[0], w.shape[1] * 8
    assert s.shape == (n, k // group) and x2.shape[1] == k
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float16)
    y = np.empty((x2.shape[0], n), dtype=np.float64)
    lib().o_int4_linear(_p(w), _p(s.view(np.uint16)), _p(x2.view(np.uint16)),
                        _p(None if b is None else b.view(np.uint16)),
                        _i64(x2.shape[0]), _i64(n), _i64(k), _i64(group), _p(y))
    return y if np.ndim(x) == 2 else y[0]


def int4_gemv(w, s, x, bias=None, group: int = 128, out_dtype=np.float16) -> np.ndarray:
    """The INT4 linear layer with its output stored as fp16 (or fp32 for logits)."""
    y = int4_linear(w, s, x, bias, group)
    return y.astype(np.float32) if out_dtype == np.float32 else f16(y)


# ------------------------------------------------------------------ glue

def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """fp16 y = x / sqrt(mean(x^2) + eps) * gamma, rows of x normalised separately."""
    xd = np.asarray(x, dtype=np.float64)
    ms = np.mean(xd * xd, axis=-1, keepdims=True)
    return f16(xd / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64))


def rope_angles(pos: int, d: int, theta: float) -> np.ndarray:
    i = np.arange(d // 2, dtype=np.float64)
    return float(pos) * np.power(float(theta), -2.0 * i / d)


def rope(v: np.ndarray, pos: int, theta: float = 1e6) -> np.ndarray:
    """Rotate-half RoPE of head vectors v [..., D] at 0-based position pos; fp16 out."""
    vd = np.asarray(v, dtype=np.float64)
    d = vd.shape[-1]
    a = rope_angles(pos, d, theta)
    c, s = np.cos(a), np.sin(a)
    lo, hi = vd[..., : d // 2], vd[..., d // 2:]
    return f16(np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1))


def silu_mul(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    g = np.asarray(gate, dtype=np.float64)
    return f16(g / (1.0 + np.exp(-g)) * np.asarray(up, dtype=np.float64))


def residual_add(r: np.ndarray, y: np.ndarray) -> np.ndarray:
    return f16(np.asarray(r, dtype=np.float64) + np.asarray(y, dtype=np.float64))


def argmax(logits: np.ndarray) -> int:
    """Lowest index among equal maxima."""
    v = np.asarray(logits)
    return int(np.flatnonzero(v == v.max())[0])


# ------------------------------------------------------------------ attention

def paged_attention(q, k_pool, v_pool, page_table, ctx: int, scale=None, return_probs=False):
    """float64 o [n_q][D] of one sequence over ctx tokens of a paged pool."""
    q = np.ascontiguousarray(q, dtype=np.float16)
    k_pool = np.ascontiguousarray(k_pool, dtype=np.float16)
    v_pool = np.ascontiguousarray(v_pool, dtype=np.float16)
    table = np.ascontiguousarray(page_table, dtype=np.int32)
    n_q, d = q.shape
    _, n_kv, page_size, d2 = k_pool.shape
    assert d2 == d and v_pool.shape == k_pool.shape and n_q % n_kv == 0
    assert table.size * page_size >= ctx >= 1
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((n_q, d), dtype=np.float64)
    probs = np.empty((n_q, ctx), dtype=np.float64) if return_probs else None
    lib().o_paged_attention(_p(q.view(np.uint16)), _p(k_pool.view(np.uint16)), _p(v_pool.view(np.uint16)),
                            _p(table), _i64(ctx), _i64(n_q), _i64(n_kv), _i64(d), _i64(page_size),
                            _f64(scale), _p(out), _p(probs))
    return (out, probs) if return_probs else out


def contiguous_attention(q, k, v, scale=None, return_probs=False):
    """Same attention over contiguous K, V [n_kv][ctx][D]."""
    q = np.ascontiguousarray(q, dtype=np.float16)
    k = np.ascontiguousarray(k, dtype=np.float16)
    v = np.ascontiguousarray(v, dtype=np.float16)
    n_q, d = q.shape
    n_kv, ctx, _ = k.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((n_q, d), dtype=np.float64)
    probs = np.empty((n_q, ctx), dtype=np.float64) if return_probs else None
    lib().o_contiguous_attention(_p(q.view(np.uint16)), _p(k.view(np.uint16)), _p(v.view(np.uint16)),
                                 _i64(ctx), _i64(n_q), _i64(n_kv), _i64(d), _f64(scale), _p(out), _p(probs))
    return (out, probs) if return_probs else out


def paged_gather(pool, page_table, ctx: int) -> np.ndarray:
    """[n_kv][ctx][D] rows of one sequence, in token order."""
    pool = np.ascontiguousarray(pool, dtype=np.float16)
    table = np.ascontiguousarray(page_table, dtype=np.int32)
    _, n_kv, page_size, d = pool.shape
    out = np.empty((n_kv, ctx, d), dtype=np.float16)
    lib().o_paged_gather(_p(pool.view(np.uint16)), _p(table), _i64(ctx), _i64(n_kv), _i64(d),
                         _i64(page_size), _p(out.view(np.uint16)))
    return out


from .model import DecoderOracle  # noqa: E402,F401
