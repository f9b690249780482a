"""The captured decode step through the C ABI vs the CPU oracle (needs a B200).

* a 2-layer decoder with the same kernels (head_dim 128, GQA, paged KV):
  greedy tokens identical to the oracle, logits within tolerance;
* graph replay and eager launches give bit-identical results;
* the 28-layer 7B-shape decoder: 512-token prompt then 128 greedy tokens,
  identical to the oracle's stream stored in tests/golden (written by
  tests/golden/make_decode_golden.py, which calls only the oracle).
"""
import json
import os

import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import normwise_err

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SMALL = synth.ModelShape(layers=2, hidden=256, inter=384, n_q=2, n_kv=1, head_dim=128, vocab=1000, group=128,
                         page_size=16, max_ctx=256)


def small_setup(i4, cuda, seed=0, n_prompt=20):
    layers = [synth.layer_weights(SMALL, i, seed) for i in range(SMALL.layers)]
    glob = synth.global_weights(SMALL, seed)
    table = synth.page_table(SMALL, seed)
    prompt = synth.prompt_tokens(SMALL, n_prompt, seed)
    model = i4.DeviceModel(SMALL, layers, glob, device=cuda)
    return layers, glob, table, prompt, model


def run_steps(graph, n, eager=False):
    for _ in range(n):
        graph.eager() if eager else graph.replay()


def test_small_decoder_matches_oracle(i4lib, cuda):
    import torch
    layers, glob, table, prompt, model = small_setup(i4lib, cuda)
    n_new = 12
    ref_tokens, ref_logits = oracle.DecoderOracle(SMALL, layers, glob, table).generate(prompt, n_new)
    seq = i4lib.Sequence(model, table, prompt)
    g = i4lib.DecodeGraph(model, seq)
    assert g.kernel_count == 5 * SMALL.layers + 1
    logits = []
    for step in range(len(prompt) + n_new - 1):
        g.replay()
        if step >= len(prompt) - 1:
            torch.cuda.synchronize()
            logits.append(seq.logits.cpu().numpy().copy())
    torch.cuda.synchronize()
    hist = seq.history.cpu().numpy()
    assert np.array_equal(hist[: len(prompt)], prompt)
    assert np.array_equal(hist[len(prompt): len(prompt) + n_new], ref_tokens)
    assert int(seq.pos.item()) == len(prompt) + n_new - 1
    assert int(seq.ctx_len.item()) == len(prompt) + n_new
    assert int(seq.status.item()) == 0
    for i in range(n_new):
        assert normwise_err(logits[i], ref_logits[i]) <= 2e-3, i
    g.close()


def test_graph_equals_eager_bit_exact(i4lib, cuda):
    import torch
    _, _, table, prompt, model = small_setup(i4lib, cuda, seed=1, n_prompt=9)
    seqs = [i4lib.Sequence(model, table, prompt) for _ in range(2)]
    gs = [i4lib.DecodeGraph(model, s) for s in seqs]
    run_steps(gs[0], 40, eager=False)
    run_steps(gs[1], 40, eager=True)
    torch.cuda.synchronize()
    a, b = seqs
    assert torch.equal(a.history, b.history)
    assert torch.equal(a.logits, b.logits)
    for l in range(SMALL.layers):
        assert torch.equal(a.k_pools[l], b.k_pools[l])
        assert torch.equal(a.v_pools[l], b.v_pools[l])
    for g in gs:
        g.close()


def test_context_limit_sets_status(i4lib, cuda):
    import torch
    _, _, table, prompt, model = small_setup(i4lib, cuda, seed=2, n_prompt=4)
    seq = i4lib.Sequence(model, table, prompt)
    g = i4lib.DecodeGraph(model, seq)
    run_steps(g, SMALL.max_ctx + 3)
    torch.cuda.synchronize()
    assert int(seq.status.item()) == 1
    assert int(seq.pos.item()) == SMALL.max_ctx - 1
    g.close()


GOLDEN = os.path.join(HERE, "golden", "decode_qwen7b_int4_seed0.json")


@pytest.mark.skipif(not os.path.exists(GOLDEN), reason="golden token stream not generated")
def test_qwen7b_shape_greedy_stream_matches_oracle(i4lib, cuda):
    import torch
    gold = json.load(open(GOLDEN))
    shape = synth.QWEN7B
    prompt = synth.prompt_tokens(shape, gold["n_prompt"], gold["seed"])
    assert [int(t) for t in prompt[:8]] == gold["prompt_head"]
    model = i4lib.DeviceModel.synthetic(shape, gold["seed"], device=cuda)
    seq = i4lib.Sequence(model, synth.page_table(shape, gold["seed"]), prompt)
    g = i4lib.DecodeGraph(model, seq)
    n_prompt, n_new = gold["n_prompt"], gold["n_new"]
    run_steps(g, n_prompt - 1)
    g.replay()  # the step at the last prompt position produces the first new token
    torch.cuda.synchronize()
    first_logits = seq.logits.cpu().numpy()
    np.testing.assert_allclose(first_logits[:8], gold["first_logits_head"], rtol=0, atol=2e-2)
    run_steps(g, n_new - 1)
    torch.cuda.synchronize()
    got = seq.history.cpu().numpy()[n_prompt: n_prompt + n_new]
    want = np.asarray(gold["tokens"])
    mism = np.flatnonzero(got != want)
    detail = ""
    if mism.size:
        i = int(mism[0])
        detail = f"first mismatch at step {i}: oracle top-2 gap {gold['top2_gap'][i]:.4g} " \
                 f"(top-1 logit {gold['top1_logit'][i]:.4g})"
    assert mism.size == 0, detail
    assert int(seq.status.item()) == 0
    g.close()
