"""Seeded synthetic inputs for the batch-1 INT4 decode path.

This module is shared by the tests, ``bench.py`` and the callers of the CPU
oracle. It draws random numbers and fixes shapes; it holds none of the
method's arithmetic (no unpacking, no dequantisation, no norms, no attention).

Every tensor comes from its own keyed stream
``default_rng(SeedSequence([seed, *key]))``, so any tensor (one layer's gate/up
matrix, say) can be regenerated on its own, in any order, on any machine.

Value recipes (the pages print no weights; these follow the workload
description of the 7B-shape decode benchmark):

* packed INT4 weights: uniformly random uint32 words. Eight signed 4-bit
  fields per word, so every field is uniform over [-8, 7];
* group scales: uniform in [0.005, 0.02], drawn in float64, rounded to fp16.
  In the full decoder every group scale also gets a random sign: the codes
  uniform over [-8, 7] have mean -1/2, so all-positive scales give every weight
  matrix a common negative mean; through the MLP that mean feeds back from
  layer to layer and the fp16 residual overflows to inf in the second layer.
  Random signs make the mean zero and keep the 28-layer residual near 400 RMS;
* activations, K/V, queries, embedding rows: N(0, 1), rounded to fp16;
* qkv bias: N(0, 0.1), rounded to fp16;
* RMSNorm weights (gamma): N(1, 0.1), rounded to fp16;
* page tables: random permutations of the physical pages;
* prompt: token ids uniform in [0, vocab).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class ModelShape:
    """Qwen2.5-7B-shaped decoder (28 layers, hidden 3584, MLP 18944, vocab 152064)."""
    layers: int = 28
    hidden: int = 3584
    inter: int = 18944
    n_q: int = 28
    n_kv: int = 4
    head_dim: int = 128
    vocab: int = 152064
    group: int = 128
    page_size: int = 16
    max_ctx: int = 4096
    theta: float = 1.0e6
    eps: float = 1.0e-6

    @property
    def qkv_rows(self) -> int:
        return (self.n_q + 2 * self.n_kv) * self.head_dim

    @property
    def max_pages(self) -> int:
        return (self.max_ctx + self.page_size - 1) // self.page_size


QWEN7B = ModelShape()

# tensor keys inside one layer
W_QKV, S_QKV, B_QKV, W_O, S_O, W_GU, S_GU, W_D, S_D, LN_IN, LN_POST = range(11)
GLOBAL = 100000  # layer key for tensors outside the layers
EMBED, LN_FINAL, W_LM, S_LM, PROMPT, PAGE_TABLE = range(6)


def rng_for(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), *map(int, key)]))


def packed_int4(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """[n][k/8] uint32 words; each 4-bit field uniform over its 16 codes."""
    assert k % 8 == 0
    return rng.integers(0, 2**32, size=(n, k // 8), dtype=np.uint32)


def group_scales(rng: np.random.Generator, n: int, k: int, group: int = 128, signed: bool = False) -> np.ndarray:
    """[n][k/group] fp16 with magnitudes uniform in [0.005, 0.02]; a random sign per group when `signed`."""
    assert k % group == 0
    mag = rng.uniform(0.005, 0.02, size=(n, k // group))
    if signed:
        mag = mag * (2.0 * rng.integers(0, 2, size=mag.shape) - 1.0)
    return mag.astype(np.float16)


def normal_f16(rng: np.random.Generator, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float16)
    flat = out.reshape(-1)
    step = 1 << 24
    for i in range(0, flat.size, step):
        m = min(step, flat.size - i)
        flat[i:i + m] = (rng.standard_normal(m) * std + mean).astype(np.float16)
    return out


# ---------------------------------------------------------------- unit cases

def gemv_case(n: int, k: int, m: int = 1, group: int = 128, seed: int = 0, bias: bool = False):
    """One INT4 linear layer: (w [n][k/8] u32, s [n][k/g] f16, x [m][k] f16, b [n] f16 or None)."""
    w = packed_int4(rng_for(seed, 1, n, k, 0), n, k)
    s = group_scales(rng_for(seed, 1, n, k, 1), n, k, group)
    x = normal_f16(rng_for(seed, 1, n, k, 2 + m), (m, k))
    b = normal_f16(rng_for(seed, 1, n, k, 99), (n,), 0.0, 0.1) if bias else None
    return w, s, x, b


def attention_case(ctx_lens, n_q: int = 28, n_kv: int = 4, d: int = 128, page_size: int = 16,
                   seed: int = 0, spare_pages: int = 0):
    """Paged decode attention inputs for len(ctx_lens) sequences.

    Pages are drawn without replacement from one shuffled pool shared by all
    sequences; the last page of each sequence is partially filled when its
    length is not a multiple of the page size. Returns
    (q [B][n_q][d], k_pool, v_pool [num_pages][n_kv][page_size][d], page_table
    [B][max_pages], ctx_len [B] int32).
    """
    ctx_lens = np.asarray(ctx_lens, dtype=np.int64)
    bsz = len(ctx_lens)
    need = [(int(c) + page_size - 1) // page_size for c in ctx_lens]
    max_pages = max(max(need), 1)
    num_pages = sum(need) + spare_pages
    rng = rng_for(seed, 2, bsz, page_size, int(ctx_lens.sum()))
    perm = rng.permutation(num_pages).astype(np.int32)
    table = np.zeros((bsz, max_pages), dtype=np.int32)
    off = 0
    for b, p in enumerate(need):
        table[b, :p] = perm[off:off + p]
        off += p
    q = normal_f16(rng, (bsz, n_q, d))
    k_pool = normal_f16(rng, (num_pages, n_kv, page_size, d))
    v_pool = normal_f16(rng, (num_pages, n_kv, page_size, d))
    return q, k_pool, v_pool, table, ctx_lens.astype(np.int32)


def ragged_lengths(length: int, batch: int, seed: int = 0) -> np.ndarray:
    """Per-sequence lengths uniform over the integers in [length/2, length]."""
    rng = rng_for(seed, 3, length, batch)
    return rng.integers(length // 2, length + 1, size=batch).astype(np.int32)


# ---------------------------------------------------------------- full model

def layer_weights(shape: ModelShape, layer: int, seed: int = 0) -> dict:
    h, i, g, nqkv = shape.hidden, shape.inter, shape.group, shape.qkv_rows
    r = lambda code: rng_for(seed, layer, code)
    return {
        "w_qkv": packed_int4(r(W_QKV), nqkv, h),
        "s_qkv": group_scales(r(S_QKV), nqkv, h, g, signed=True),
        "b_qkv": normal_f16(r(B_QKV), (nqkv,), 0.0, 0.1),
        "w_o": packed_int4(r(W_O), h, shape.n_q * shape.head_dim),
        "s_o": group_scales(r(S_O), h, shape.n_q * shape.head_dim, g, signed=True),
        "w_gu": packed_int4(r(W_GU), 2 * i, h),
        "s_gu": group_scales(r(S_GU), 2 * i, h, g, signed=True),
        "w_d": packed_int4(r(W_D), h, i),
        "s_d": group_scales(r(S_D), h, i, g, signed=True),
        "ln_in": normal_f16(r(LN_IN), (h,), 1.0, 0.1),
        "ln_post": normal_f16(r(LN_POST), (h,), 1.0, 0.1),
    }


def global_weights(shape: ModelShape, seed: int = 0) -> dict:
    r = lambda code: rng_for(seed, GLOBAL, code)
    return {
        "embed": normal_f16(r(EMBED), (shape.vocab, shape.hidden)),
        "ln_final": normal_f16(r(LN_FINAL), (shape.hidden,), 1.0, 0.1),
        "w_lm": packed_int4(r(W_LM), shape.vocab, shape.hidden),
        "s_lm": group_scales(r(S_LM), shape.vocab, shape.hidden, shape.group, signed=True),
    }


def prompt_tokens(shape: ModelShape, n: int = 512, seed: int = 0) -> np.ndarray:
    return rng_for(seed, GLOBAL, PROMPT, n).integers(0, shape.vocab, size=n).astype(np.int32)


def page_table(shape: ModelShape, seed: int = 0) -> np.ndarray:
    """One sequence's table: a random permutation of all max_ctx/page_size pages."""
    return rng_for(seed, GLOBAL, PAGE_TABLE).permutation(shape.max_pages).astype(np.int32)
