"""Pins for the oracle's composed decoder (no GPU).

The composed model has no printed reference (no trained weights, no logits on
the pages), so it is pinned through its parts (test_oracle_primitives.py),
through these structural facts: feeding a prompt as one block equals feeding
it token by token; a repeated run is deterministic; the residual stream of the
7B-shaped random model stays finite in fp16; and through two special cases with
closed forms computed here from the definitions: zero o/down projections reduce
every step to lm_head(RMSNorm(embedding)), and zero queries make attention the
running mean of the cached V rows (which also pins the GQA head mapping, the K/V
append and read, the o projection and the residual adds).
"""
import numpy as np

import oracle
from int4_weight_only_02_b200 import synth

TINY = synth.ModelShape(layers=2, hidden=256, inter=384, n_q=4, n_kv=2, head_dim=64, vocab=500,
                        group=128, page_size=16, max_ctx=64)


def tiny_oracle(seed=0):
    layers = [synth.layer_weights(TINY, i, seed) for i in range(TINY.layers)]
    glob = synth.global_weights(TINY, seed)
    return oracle.DecoderOracle(TINY, layers, glob, synth.page_table(TINY, seed))


def test_block_prompt_equals_token_by_token():
    prompt = synth.prompt_tokens(TINY, 21, seed=1)
    a = tiny_oracle()
    b = tiny_oracle()
    ta, la = a.generate(prompt, 6, block_prompt=True)
    tb, lb = b.generate(prompt, 6, block_prompt=False)
    assert np.array_equal(ta, tb)
    assert np.array_equal(la, lb)
    for li in range(TINY.layers):
        assert np.array_equal(a.k_pools[li], b.k_pools[li])
        assert np.array_equal(a.v_pools[li], b.v_pools[li])


def test_kv_lands_in_permuted_pages():
    o = tiny_oracle()
    prompt = synth.prompt_tokens(TINY, 20, seed=2)
    o.forward(prompt, 0)
    table = o.page_table
    for li in range(TINY.layers):
        used = set(int(table[t // 16]) for t in range(20))
        for page in range(o.k_pools[li].shape[0]):
            nonzero = np.any(o.k_pools[li][page] != 0)
            assert nonzero == (page in used)
        # page of tokens 16..19 holds exactly 4 filled slots
        last = table[1]
        filled = np.any(o.k_pools[li][last] != 0, axis=(0, 2))
        assert list(filled) == [True] * 4 + [False] * 12


def test_trace_shapes_and_finiteness():
    o = tiny_oracle()
    traces = []
    logits, r = o.forward([5, 7, 9], 0, traces)
    assert logits.dtype == np.float32 and logits.shape == (TINY.vocab,)
    assert len(traces) == TINY.layers
    for tr in traces:
        for name, v in tr.items():
            assert np.all(np.isfinite(v.astype(np.float64))), name
    assert traces[0]["gu"].shape == (3, 2 * TINY.inter)


# ---- closed forms of the composition (expected values computed here, from the definitions, without the oracle)

def _dequant(words, scales):
    """Test-side dequantisation: field i of word j is k = 8j + i, two's complement; one scale per 128 k."""
    words = np.asarray(words).astype(np.uint64)
    n, w = words.shape
    nib = (words[:, :, None] >> (np.arange(8, dtype=np.uint64) * 4)) & 0xF
    q = np.where(nib >= 8, nib.astype(np.int64) - 16, nib.astype(np.int64)).reshape(n, w * 8)
    return q * np.repeat(np.asarray(scales, dtype=np.float64), 128, axis=1)


def _norm16(r, gamma, eps):
    r = np.asarray(r, dtype=np.float64)
    return (r / np.sqrt(np.mean(r * r, axis=-1, keepdims=True) + eps) * np.asarray(gamma, np.float64)).astype(np.float16)


def _zeroed(layers, keys):
    out = []
    for lw in layers:
        lw = dict(lw)
        for k in keys:
            lw[k] = np.zeros_like(lw[k])
        out.append(lw)
    return out


def test_zero_o_and_down_reduce_to_lm_head_of_the_embedding():
    """With W_o = W_down = 0 every residual add adds an exact zero, so each token's logits are
    W_lm RMSNorm(E[token]) whatever the layers compute, and greedy decode iterates that map."""
    layers = _zeroed([synth.layer_weights(TINY, i, 0) for i in range(TINY.layers)], ("w_o", "w_d"))
    glob = synth.global_weights(TINY, 0)
    dec = oracle.DecoderOracle(TINY, layers, glob, synth.page_table(TINY, 0))
    prompt = synth.prompt_tokens(TINY, 6, 0)
    toks, logits = dec.generate(prompt, 5)
    w_lm = _dequant(glob["w_lm"], glob["s_lm"])

    def step_logits(tok):
        return (w_lm @ _norm16(glob["embed"][tok], glob["ln_final"], TINY.eps).astype(np.float64)).astype(np.float32)

    want_tok, t = [], int(prompt[-1])
    for i in range(5):
        lg = step_logits(t)
        np.testing.assert_allclose(logits[i], lg, rtol=1e-6, atol=1e-6)
        t = int(np.flatnonzero(lg == lg.max())[0])
        want_tok.append(t)
    assert list(toks) == want_tok


def test_zero_query_attention_is_the_running_mean_of_v():
    """With the q rows of W_qkv and their bias zero, every score is 0, so each query head's output is the
    plain mean of its kv head's cached V rows over positions 0..p (GQA: head h reads kv head h // G);
    with W_down = 0 the residual after the layer is E[tok] + fp16(W_o o) and the logits follow."""
    shape = synth.ModelShape(layers=1, hidden=256, inter=384, n_q=4, n_kv=2, head_dim=64, vocab=500,
                             group=128, page_size=16, max_ctx=64)
    lw = synth.layer_weights(shape, 0, 3)
    nq, nkv, d = shape.n_q, shape.n_kv, shape.head_dim
    lw["w_qkv"] = lw["w_qkv"].copy()
    lw["w_qkv"][: nq * d] = 0
    lw["b_qkv"] = lw["b_qkv"].copy()
    lw["b_qkv"][: nq * d] = 0
    lw["w_d"] = np.zeros_like(lw["w_d"])
    glob = synth.global_weights(shape, 3)
    tokens = synth.prompt_tokens(shape, 7, 3)
    dec = oracle.DecoderOracle(shape, [lw], glob, synth.page_table(shape, 3))
    logits, r = dec.forward(tokens, 0)

    w_qkv = _dequant(lw["w_qkv"], lw["s_qkv"])
    w_o = _dequant(lw["w_o"], lw["s_o"])
    w_lm = _dequant(glob["w_lm"], glob["s_lm"])
    e = glob["embed"][tokens].astype(np.float16)
    x = _norm16(e, lw["ln_in"], shape.eps).astype(np.float64)
    v = ((x @ w_qkv[(nq + nkv) * d:].T) + lw["b_qkv"][(nq + nkv) * d:].astype(np.float64)).astype(np.float16)
    v = v.astype(np.float64).reshape(len(tokens), nkv, d)
    G = nq // nkv
    for p in range(len(tokens)):
        o = np.concatenate([v[: p + 1, h // G].mean(axis=0) for h in range(nq)]).astype(np.float16)
        y = (w_o @ o.astype(np.float64)).astype(np.float16)
        r_want = (e[p].astype(np.float64) + y.astype(np.float64)).astype(np.float16)
        # the oracle sums in a different order: allow one fp16 ulp of the residual
        assert np.max(np.abs(r[p].astype(np.float64) - r_want.astype(np.float64))
                      / np.maximum(np.abs(r_want.astype(np.float64)), 1.0)) <= 2 ** -10
    lg = (w_lm @ _norm16(r[-1], glob["ln_final"], shape.eps).astype(np.float64)).astype(np.float32)
    np.testing.assert_allclose(logits, lg, rtol=1e-6, atol=1e-6)
