"""The 28-layer decoder step of the oracle -- TEST INFRASTRUCTURE.

Composes the functions of this package in the order of one decode token of a
Qwen2.5-7B-shaped decoder ("How To Build Your Own LLM Runtime From Scratch",
model configuration in its technical-analysis section: 28 layers, hidden 3584,
MLP 18944, vocabulary 152064):

  r = E[token]
  per layer:  x = RMSNorm(r); [q|k|v] = fp16(W_qkv x + b); q, k = RoPE(q, k, pos);
              K/V of the layer's pool at (page_table[pos / P], pos % P) = k, v;
              o = attention(q, K/V[0..pos]); r = fp16(r + fp16(W_o o));
              x = RMSNorm(r); [g|u] = fp16(W_gu x); m = fp16(silu(g) u);
              r = fp16(r + fp16(W_d m))
  logits = fp32(W_lm RMSNorm(r)); next = argmax(logits)

A prompt may be fed a whole block of tokens at once: every row of the block
goes through exactly the elementwise operations of a one-token step, and
token i only reads K/V up to its own position, so the result is the same as
feeding the tokens one by one (``tests/test_oracle_model.py`` checks this).

Pins: the parts are pinned in ``tests/test_oracle_primitives.py``; the
composition is pinned by the block-prompt identity, the K/V page placement and
two closed-form special cases (zero o/down projections; zero queries) in
``tests/test_oracle_model.py``. The general composition with every branch active
has no independent reference: parity unpinned beyond those cases.
"""
from __future__ import annotations

import numpy as np

from . import argmax, f16, int4_gemv, int4_linear, paged_attention, residual_add, rmsnorm, rope, silu_mul


class DecoderOracle:
    def __init__(self, shape, layers, glob, page_table, num_pages=None):
        self.shape = shape
        self.layers = layers
        self.glob = glob
        self.page_table = np.asarray(page_table, dtype=np.int32)
        num_pages = int(self.page_table.max()) + 1 if num_pages is None else num_pages
        kv = (num_pages, shape.n_kv, shape.page_size, shape.head_dim)
        self.k_pools = [np.zeros(kv, dtype=np.float16) for _ in layers]
        self.v_pools = [np.zeros(kv, dtype=np.float16) for _ in layers]

    # one layer over a block of consecutive positions; returns the new residual rows
    def layer(self, li: int, r: np.ndarray, positions, trace: dict | None = None) -> np.ndarray:
        sh, w = self.shape, self.layers[li]
        d, nq, nkv, ps = sh.head_dim, sh.n_q, sh.n_kv, sh.page_size
        x = rmsnorm(r, w["ln_in"], sh.eps)
        qkv = f16(int4_linear(w["w_qkv"], w["s_qkv"], x, w["b_qkv"], sh.group))
        o = np.empty((len(positions), nq * d), dtype=np.float16)
        qs, ks = [], []
        for i, p in enumerate(positions):
            q = rope(qkv[i, : nq * d].reshape(nq, d), p, sh.theta)
            k = rope(qkv[i, nq * d:(nq + nkv) * d].reshape(nkv, d), p, sh.theta)
            v = qkv[i, (nq + nkv) * d:].reshape(nkv, d)
            page, slot = self.page_table[p // ps], p % ps
            self.k_pools[li][page, :, slot, :] = k
            self.v_pools[li][page, :, slot, :] = v
            qs.append(q)
            ks.append(k)
        for i, p in enumerate(positions):
            o[i] = f16(paged_attention(qs[i], self.k_pools[li], self.v_pools[li], self.page_table, p + 1)).reshape(-1)
        r = residual_add(r, f16(int4_linear(w["w_o"], w["s_o"], o, None, sh.group)))
        r_mid = r
        x2 = rmsnorm(r, w["ln_post"], sh.eps)
        gu = f16(int4_linear(w["w_gu"], w["s_gu"], x2, None, sh.group))
        m = silu_mul(gu[:, : sh.inter], gu[:, sh.inter:])
        r = residual_add(r, f16(int4_linear(w["w_d"], w["s_d"], m, None, sh.group)))
        if trace is not None:
            trace.update(x=x, qkv=qkv, q=np.stack(qs), k=np.stack(ks), o=o, r_mid=r_mid, x2=x2, gu=gu, m=m, r=r)
        return r

    def forward(self, tokens, start_pos: int, traces: list | None = None):
        """Feed tokens at positions start_pos.. ; returns (fp32 logits of the last token, final residual rows)."""
        tokens = np.atleast_1d(np.asarray(tokens, dtype=np.int64))
        positions = list(range(start_pos, start_pos + len(tokens)))
        r = self.glob["embed"][tokens].astype(np.float16)
        for li in range(len(self.layers)):
            tr = {} if traces is not None else None
            r = self.layer(li, r, positions, tr)
            if traces is not None:
                traces.append(tr)
        x = rmsnorm(r[-1], self.glob["ln_final"], self.shape.eps)
        logits = int4_gemv(self.glob["w_lm"], self.glob["s_lm"], x, None, self.shape.group, np.float32)
        return logits, r

    def generate(self, prompt, n_new: int, block_prompt: bool = True):
        """Greedy decode: returns (generated token ids [n_new], fp32 logits of each generating step)."""
        prompt = np.asarray(prompt, dtype=np.int64)
        if block_prompt:
            logits, _ = self.forward(prompt, 0)
        else:
            for p, t in enumerate(prompt):
                logits, _ = self.forward([t], p)
        out, all_logits = [], []
        pos = len(prompt)
        for _ in range(n_new):
            tok = argmax(logits)
            out.append(tok)
            all_logits.append(logits)
            if len(out) == n_new:
                break
            logits, _ = self.forward([tok], pos)
            pos += 1
        return np.asarray(out, dtype=np.int32), np.stack(all_logits)
