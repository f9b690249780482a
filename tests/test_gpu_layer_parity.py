"""Per-kernel, teacher-forced parity of the production decode step at the 7B shape (needs a B200).

The CPU oracle runs the full 28-layer Qwen2.5-7B-shaped decoder (random INT4
weights, seed 0) over a block of 9 tokens at positions 504..512, with the KV
cache of positions 0..503 of every layer filled with seeded N(0, 4^2) fp16
values (the spread of this model's own K/V). Its trace at position 512 gives
every intermediate tensor of layers 0, 13 and 27 and the final residual.

The GPU model holds those three layers (and the embedding, final norm and
lm_head) and runs its real decode-step kernels one at a time through
decode_step_launch_kernel. Every kernel gets the oracle's inputs (the residual,
q, the attention output, SiLU(gate)*up and the K/V cache are written into the
step's buffers and pools first), so each comparison isolates one kernel:

  qkv    : RMSNorm (layer 0: embedding row) -> INT4 GEMV + bias -> RoPE -> K/V append
  attn   : paged GQA attention over 513 positions (the last page partly filled)
  o      : INT4 GEMV -> residual add
  gate/up: RMSNorm -> INT4 GEMV -> SiLU(gate) * up
  down   : INT4 GEMV -> residual add
  lm_head: final RMSNorm -> INT4 GEMV (fp32 logits) -> argmax -> state advance

fp16 outputs must be within the normwise 2e-3 of the workload; the fraction of
fp16 elements whose bits differ from the oracle's is recorded (fp32 sums on the
GPU against fp64 sums in the oracle round some stores to the other neighbour).
The five kernels of each layer are then also run back to back from the
layer's input residual (the composition inside one layer).
"""
import dataclasses
import json
import os

import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import FLIP_RATE, normwise_err

pytestmark = pytest.mark.gpu

TOL = 2e-3
LAYERS = (0, 13, 27)
FIRST_POS, POS = 504, 512
SHAPE = synth.QWEN7B
# the fp32 logits of lm_head: the fused RMSNorm rounds x to fp16, and where that rounding differs from the
# oracle's by one ulp (a fraction of a percent of the 3584 elements) a logit moves by ~|w| * 2^-11; the
# bound is 10x the normwise error of such a spread of flips (~2e-6 of max |logit|)
LOGIT_TOL = 2e-5


def kv_prefix(layer: int, which: int, shape):
    """Seeded N(0, 4^2) fp16 rows for the cache positions below FIRST_POS (input recipe of this test)."""
    rng = synth.rng_for(0, 7000 + layer, which)
    return synth.normal_f16(rng, (FIRST_POS, shape.n_kv, shape.head_dim), 0.0, 4.0)


def fill_prefix(k_pool, v_pool, table, layer, shape):
    for which, pool in ((0, k_pool), (1, v_pool)):
        rows = kv_prefix(layer, which, shape)
        for p in range(FIRST_POS):
            pool[table[p // shape.page_size], :, p % shape.page_size, :] = rows[p]


@pytest.fixture(scope="module")
def oracle_run():
    layers = [synth.layer_weights(SHAPE, i, 0) for i in range(SHAPE.layers)]
    glob = synth.global_weights(SHAPE, 0)
    table = synth.page_table(SHAPE, 0)
    tokens = synth.prompt_tokens(SHAPE, POS - FIRST_POS + 1, seed=3)
    dec = oracle.DecoderOracle(SHAPE, layers, glob, table, num_pages=SHAPE.max_pages)
    for li in range(SHAPE.layers):
        fill_prefix(dec.k_pools[li], dec.v_pools[li], table, li, SHAPE)
    traces = []
    logits, r = dec.forward(tokens, FIRST_POS, traces)
    final_r = r[-1]
    kv = {li: (dec.k_pools[li].copy(), dec.v_pools[li].copy()) for li in LAYERS}
    picked = {li: layers[li] for li in LAYERS}
    return dict(layers=picked, glob=glob, table=table, tokens=tokens, traces=traces, logits=logits,
                final_r=final_r, kv=kv)


def bits_differ(got, ref):
    g = np.asarray(got, dtype=np.float16).view(np.uint16)
    r = np.asarray(ref, dtype=np.float16).view(np.uint16)
    return float(np.mean(g != r))


class Report:
    def __init__(self):
        self.rows = []

    def add(self, layer, tensor, got, ref):
        err = normwise_err(got, ref)
        rate = bits_differ(got, ref)
        self.rows.append({"layer": layer, "tensor": tensor, "normwise": err, "fp16_mismatch": rate})
        return err


@pytest.fixture(scope="module")
def gpu_model(i4lib, cuda, oracle_run):
    o = oracle_run
    shape3 = dataclasses.replace(SHAPE, layers=len(LAYERS))
    return i4lib.DeviceModel(shape3, [o["layers"][li] for li in LAYERS], o["glob"], device=cuda)


@pytest.fixture(scope="module", params=["persistent", "per-kernel"])
def gpu_step(request, i4lib, cuda, oracle_run, gpu_model):
    """The step as one persistent kernel (each phase launched alone) and as one kernel per phase."""
    persistent = request.param == "persistent"
    seq = i4lib.Sequence(gpu_model, oracle_run["table"], None)
    i4lib.set_option("persistent", int(persistent))
    try:
        graph = i4lib.DecodeGraph(gpu_model, seq)
    finally:
        i4lib.set_option("persistent", 1)
    assert graph.persistent == persistent
    yield gpu_model, seq, graph
    graph.close()


def set_state(seq, token, pos):
    seq.token.fill_(int(token))
    seq.pos.fill_(pos)
    seq.ctx_len.fill_(pos + 1)
    seq.status.zero_()


def upload_layer_cache(seq, j, kv, table, torch, cuda, clear_current=True):
    k, v = kv
    k = k.copy()
    v = v.copy()
    if clear_current:  # the kernel under test writes position POS itself
        k[table[POS // SHAPE.page_size], :, POS % SHAPE.page_size, :] = 0
        v[table[POS // SHAPE.page_size], :, POS % SHAPE.page_size, :] = 0
    seq.k_pools[j].copy_(torch.from_numpy(k).to(cuda))
    seq.v_pools[j].copy_(torch.from_numpy(v).to(cuda))


def current_row(pool, table):
    return pool[table[POS // SHAPE.page_size], :, POS % SHAPE.page_size, :]


def t16(a, torch, cuda):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float16))).to(cuda)


def test_each_kernel_teacher_forced(i4lib, cuda, oracle_run, gpu_step):
    import torch
    o = oracle_run
    model, seq, graph = gpu_step
    nq, nkv, d = SHAPE.n_q, SHAPE.n_kv, SHAPE.head_dim
    table = o["table"]
    rep = Report()
    for j, li in enumerate(LAYERS):
        tr = o["traces"][li]
        row = -1  # position POS
        r_in = o["glob"]["embed"][o["tokens"][row]] if li == 0 else o["traces"][li - 1]["r"][row]
        q_ref, k_ref = tr["q"][row], tr["k"][row]
        v_ref = tr["qkv"][row, (nq + nkv) * d:].reshape(nkv, d)
        base = 5 * j

        # qkv: RMSNorm (embedding for layer 0) + GEMV + bias + RoPE + K/V append
        upload_layer_cache(seq, j, o["kv"][li], table, torch, cuda)
        set_state(seq, o["tokens"][row], POS)
        if li > 0:
            graph.write_buffer("resid", t16(r_in, torch, cuda))
        graph.launch_kernel(base + 0)
        torch.cuda.synchronize()
        q_got = graph.read_buffer("q").cpu().numpy().reshape(nq, d)
        k_got = current_row(seq.k_pools[j].cpu().numpy(), table)
        v_got = current_row(seq.v_pools[j].cpu().numpy(), table)
        assert rep.add(li, "q (qkv+RoPE)", q_got, q_ref) <= TOL
        assert rep.add(li, "k row (RoPE, appended)", k_got, k_ref) <= TOL
        assert rep.add(li, "v row (appended)", v_got, v_ref) <= TOL
        if li == 0:  # the embedding row becomes the residual
            r_got = graph.read_buffer("resid").cpu().numpy()
            assert np.array_equal(r_got.view(np.uint16), np.asarray(r_in, np.float16).view(np.uint16))

        # attention over the oracle's q and cache (current row included)
        upload_layer_cache(seq, j, o["kv"][li], table, torch, cuda, clear_current=False)
        graph.write_buffer("q", t16(q_ref.reshape(-1), torch, cuda))
        set_state(seq, o["tokens"][row], POS)
        graph.launch_kernel(base + 1)
        torch.cuda.synchronize()
        attn_got = graph.read_buffer("attn").cpu().numpy()
        assert rep.add(li, "attention out", attn_got, tr["o"][row]) <= TOL

        # o projection + residual add
        graph.write_buffer("attn", t16(tr["o"][row], torch, cuda))
        graph.write_buffer("resid", t16(r_in, torch, cuda))
        graph.launch_kernel(base + 2)
        torch.cuda.synchronize()
        assert rep.add(li, "resid after o", graph.read_buffer("resid").cpu().numpy(), tr["r_mid"][row]) <= TOL

        # RMSNorm + gate/up + SiLU-mul
        graph.write_buffer("resid", t16(tr["r_mid"][row], torch, cuda))
        graph.launch_kernel(base + 3)
        torch.cuda.synchronize()
        assert rep.add(li, "silu(gate)*up", graph.read_buffer("mlp").cpu().numpy(), tr["m"][row]) <= TOL

        # down projection + residual add
        graph.write_buffer("mlp", t16(tr["m"][row], torch, cuda))
        graph.write_buffer("resid", t16(tr["r_mid"][row], torch, cuda))
        graph.launch_kernel(base + 4)
        torch.cuda.synchronize()
        assert rep.add(li, "resid after down", graph.read_buffer("resid").cpu().numpy(), tr["r"][row]) <= TOL

    # final RMSNorm + lm_head (fp32 logits) + argmax + state advance
    graph.write_buffer("resid", t16(o["final_r"], torch, cuda))
    set_state(seq, o["tokens"][-1], POS)
    graph.launch_kernel(graph.phase_count - 1)
    torch.cuda.synchronize()
    lg = seq.logits.cpu().numpy()
    err = normwise_err(lg, o["logits"])
    rep.rows.append({"layer": "final", "tensor": "logits (fp32)", "normwise": err,
                     "fp16_mismatch": None})
    assert err <= LOGIT_TOL, err
    got_tok = int(seq.token.item())
    assert got_tok == int(np.flatnonzero(lg == lg.max())[0])
    ref_sorted = np.sort(o["logits"].astype(np.float64))
    if ref_sorted[-1] - ref_sorted[-2] > 1e-3:
        assert got_tok == oracle.argmax(o["logits"])
    assert int(seq.pos.item()) == POS + 1 and int(seq.ctx_len.item()) == POS + 2
    assert int(seq.status.item()) == 0 and i4lib.device_error() == 0

    worst = max(r["fp16_mismatch"] for r in rep.rows if r["fp16_mismatch"] is not None)
    for r in rep.rows:
        print(f"layer {r['layer']:>5} {r['tensor']:<24} normwise {r['normwise']:.2e} "
              + (f"fp16 mismatch {r['fp16_mismatch']:.4f}" if r["fp16_mismatch"] is not None else ""))
    print(f"worst fp16 mismatch rate {worst:.4f}")
    # The tie bound assumes independent one-ulp flips at FLIP_RATE at most. Every tensor whose fp16
    # elements round independently stays there; silu(gate)*up may read higher because one RMSNorm
    # output element that rounds to the other neighbour moves all gate/up products together (layer 13:
    # 21 % of the stores, normwise 4.6e-4; the same bits come out of the stand-alone kernels chained).
    for r in rep.rows:
        if r["fp16_mismatch"] is not None and r["tensor"] != "silu(gate)*up":
            assert r["fp16_mismatch"] <= FLIP_RATE, r
    path = os.environ.get("I4_PARITY_REPORT")
    if path:
        path = path.replace(".json", "_persistent.json" if graph.persistent else "_per_kernel.json")
        with open(path, "w") as f:
            json.dump({"rows": rep.rows, "worst_fp16_mismatch": worst}, f, indent=1)


def test_each_layer_composed(i4lib, cuda, oracle_run, gpu_step):
    """The five kernels of each layer back to back from the oracle's input residual and cache."""
    import torch
    o = oracle_run
    model, seq, graph = gpu_step
    for j, li in enumerate(LAYERS):
        tr = o["traces"][li]
        r_in = o["glob"]["embed"][o["tokens"][-1]] if li == 0 else o["traces"][li - 1]["r"][-1]
        upload_layer_cache(seq, j, o["kv"][li], o["table"], torch, cuda)
        set_state(seq, o["tokens"][-1], POS)
        if li > 0:
            graph.write_buffer("resid", t16(r_in, torch, cuda))
        for k in range(5):
            graph.launch_kernel(5 * j + k)
        torch.cuda.synchronize()
        err = normwise_err(graph.read_buffer("resid").cpu().numpy(), tr["r"][-1])
        print(f"layer {li}: composed residual normwise {err:.2e}")
        assert err <= TOL, (li, err)
    assert i4lib.device_error() == 0
