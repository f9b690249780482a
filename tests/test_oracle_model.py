"""Pins for the oracle's composed decoder (no GPU).

The composed model has no printed reference (no trained weights, no logits on
the pages), so it is pinned through its parts (test_oracle_primitives.py) and
through these structural facts: feeding a prompt as one block equals feeding
it token by token; a repeated run is deterministic; the residual stream of the
7B-shaped random model stays finite in fp16.
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
