"""Write the oracle's greedy token stream for the 7B-shape INT4 decoder.

Workload: 28-layer Qwen2.5-7B-shaped decoder, random INT4 group-128 weights
(seed 0, see int4_weight_only_02_b200.synth), a 512-token prompt of uniform
random ids, then 128 greedy tokens; page size 16 and a permuted page table of
256 pages. Calls only the CPU oracle; nothing here touches the CUDA library.

Run:  python tests/golden/make_decode_golden.py  [--prompt 512] [--new 128]
Output: tests/golden/decode_qwen7b_int4_seed0.json
"""
import argparse
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from int4_weight_only_02_b200 import synth  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--prompt", type=int, default=512)
    ap.add_argument("--new", type=int, default=128)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--out", default=os.path.join(HERE, "decode_qwen7b_int4_seed0.json"))
    a = ap.parse_args()
    shape = synth.QWEN7B
    t0 = time.time()
    layers = [synth.layer_weights(shape, i, a.seed) for i in range(shape.layers)]
    glob = synth.global_weights(shape, a.seed)
    prompt = synth.prompt_tokens(shape, a.prompt, a.seed)
    table = synth.page_table(shape, a.seed)
    print(f"weights generated in {time.time() - t0:.1f} s", flush=True)
    dec = oracle.DecoderOracle(shape, layers, glob, table, num_pages=shape.max_pages)
    t0 = time.time()
    tokens, logits = dec.generate(prompt, a.new, block_prompt=True)
    el = time.time() - t0
    top2 = np.sort(logits, axis=1)[:, -2:]
    top5 = np.argsort(-logits, axis=1, kind="stable")[:, :5]
    sample_idx = np.random.default_rng(2024).choice(shape.vocab, size=2048, replace=False)
    rec = {
        "workload": "qwen2.5-7b-shape int4-g128 decoder, seed %d, prompt %d, %d greedy steps, page 16"
                    % (a.seed, a.prompt, a.new),
        "seed": a.seed,
        "n_prompt": a.prompt,
        "n_new": a.new,
        "prompt_head": [int(t) for t in prompt[:8]],
        "tokens": [int(t) for t in tokens],
        "top1_logit": [float(v) for v in top2[:, 1]],
        "top2_gap": [float(v) for v in (top2[:, 1] - top2[:, 0])],
        "first_logits_head": [float(v) for v in logits[0, :8]],
        "top5": [[[int(i), float(logits[j, i])] for i in top5[j]] for j in range(len(tokens))],
        "first_logits_sample": {"index": [int(i) for i in sample_idx],
                                "value": [float(logits[0, i]) for i in sample_idx]},
        "oracle_seconds": round(el, 1),
        "oracle_threads": os.cpu_count(),
    }
    with open(a.out, "w") as f:
        json.dump(rec, f, indent=1)
    print(f"done in {el:.1f} s -> {a.out}")


if __name__ == "__main__":
    main()
