"""Batch-1 decode benchmark of the 7B-shape INT4 weight-only decoder on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl i4|reference]

A step is one decode token: one replay of the captured CUDA graph (28 layers x
{qkv+RoPE+KV append, paged attention, o, RMSNorm+gate/up+SiLU, down} + final
norm, lm_head and argmax: 141 kernels). Setup (untimed): random-init INT4
weights (seed 0), a 512-token prompt of uniform random ids fed through the
same graph, then W warm-up tokens; then K timed tokens, each at a context one
longer than the last. Every token streams 3.65 GB of INT4 weights and scales
(more than the 126 MB L2), so no L2 flush is needed between steps.

Printed (rank 0, one JSON line): tok/s over all ranks (replicas: one sequence
per GPU, no exchange), ms/token (max over ranks, CUDA events), the end-to-end
rate through the public API with the token copied host->device and the next
token device->host every step, the roofline of the dominant kernel (the
RMSNorm+gate/up+SiLU GEMV) against the measured HBM copy bandwidth, the whole
step against 8 TB/s and the measured bandwidth, SM clocks sampled during the
timed region, and the CPU oracle timed on a bounded sample.

--impl reference times the CPU oracle instead (rank 0 only), each step one
decoder layer of one token at context 513, scaled to tok/s.

Other modes (one JSON line per case, not the benchmark line):
  --profile-kernel NAME  one kernel of a one-layer model, for ncu captures;
  --attention-sweep      paged attention over contexts 512-32768, page sizes 16/64,
                         batches 1/8/32 with ragged lengths (KV GB/s, L2-cold);
  --gemv-batch           the gate/up GEMV for 1, 2, 4 and 8 vectors (weight GB/s);
  --batched-decode B     B sequences decoded together (tok/s over the batch);
  --prefill B            time to first token with B prompt positions per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tok/s at batch 1 (7B-shape INT4); INT4 GEMV HBM GB/s vs B200 peak"
WORKLOAD = ("qwen2.5-7b-shape decoder (28 layers, hidden 3584, mlp 18944, 28q/4kv heads, head_dim 128, "
            "vocab 152064), int4 group-128 fp16-scale weights (codes uniform in [-8, 7], |scale| uniform in "
            "[0.005, 0.02] with a random sign per group: all-positive scales overflow the fp16 residual in "
            "layer 1), batch 1, 512-token prompt then greedy decode, paged KV page 16, one CUDA graph per token")
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.lines = gpu_id, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", self.gpu_id], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except Exception:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


GEMV_SOURCES = ["gemv_stream.cu", "gemv_parts.cuh", "gemv.cuh", "common.cuh", "async.cuh", "mma.cuh"]
PERSIST_SOURCES = ["persist.cu", "persist.cuh", "gemv_parts.cuh", "gemv.cuh", "common.cuh", "async.cuh", "mma.cuh"]


def sources_hash(names) -> str:
    """First 16 hex digits of the sha256 over the named kernel sources, in order."""
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "int4_weight_only_02_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def traffic_from_profile(profile: str, names):
    """DRAM bytes (read + write) per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256_16") != sources_hash(names):
        return None
    try:
        return float(vals["dram_bytes_per_full_launch"])
    except Exception:
        return None


def primed_oracle(shape, layers_np, glob_np, first_pos: int, n_tokens: int):
    """The CPU oracle decoder with the KV cache below `first_pos` filled with seeded random fp16 values
    (N(0, 4^2), the spread of the model's own K/V), ready to decode tokens at first_pos, first_pos + 1, ..."""
    import numpy as np

    import oracle
    from int4_weight_only_02_b200 import synth
    dec = oracle.DecoderOracle(shape, layers_np, glob_np, synth.page_table(shape, 0), num_pages=shape.max_pages)
    rng = np.random.default_rng(123)
    used = (first_pos + n_tokens + shape.page_size - 1) // shape.page_size
    for li in range(shape.layers):
        for pool in (dec.k_pools[li], dec.v_pools[li]):
            for p in dec.page_table[:used]:
                pool[p] = (rng.standard_normal(pool[p].shape) * 4).astype(np.float16)
    return dec


def oracle_cpu_sample(shape, layers_np, glob_np, n_tokens: int = 8):
    """The CPU oracle as it stands: n_tokens full decode steps at positions 512.. (bounded sample)."""
    import oracle
    dec = primed_oracle(shape, layers_np, glob_np, 512, n_tokens)
    threads = oracle.set_threads(0)
    t0 = time.perf_counter()
    tok = 1
    for i in range(n_tokens):
        logits, _ = dec.forward([tok], 512 + i)
        tok = oracle.argmax(logits)
    el = time.perf_counter() - t0
    return {"value": round(n_tokens / el, 4), "unit": "tok/s", "cores": threads, "host_cpus": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{n_tokens} full decode tokens (28 layers + lm_head) at positions 512..{511 + n_tokens}, "
                      f"KV below filled with random fp16, fp64 C/numpy oracle, {threads} OpenMP threads "
                      f"({el:.1f} s)"}


def oracle_unit_configs():
    """The unit workloads timed on the CPU oracle, one thread (pinned to one core) and all threads:
    qkv INT4 GEMV (K 3584, N 4608), paged attention (28/4 heads, ctx 512, page 16), MLP block
    (RMSNorm, gate/up GEMV, SiLU-mul, down GEMV); ms and algorithmic GB/s of each."""
    import numpy as np

    import oracle
    from int4_weight_only_02_b200 import synth
    w, s, x, b = synth.gemv_case(4608, 3584, seed=0, bias=True)
    q, kp, vp, table, ctx = synth.attention_case([512], page_size=16, seed=0)
    mw_gu, ms_gu, mx, _ = synth.gemv_case(37888, 3584, seed=0)
    mw_d, ms_d, _, _ = synth.gemv_case(3584, 18944, seed=0)
    gamma = synth.normal_f16(synth.rng_for(0, 77), (3584,), 1.0, 0.1)
    units = {
        "C0a_qkv_gemv": (lambda: oracle.int4_gemv(w, s, x[0], b), 4608 * 1792 + 4608 * 28 * 2),
        "C0b_attention_ctx512": (lambda: oracle.paged_attention(q[0], kp, vp, table[0], 512), 512 * 4 * 128 * 2 * 2),
        "C1_mlp_block": (lambda: oracle.int4_gemv(mw_d, ms_d, oracle.silu_mul(
            *np.split(oracle.int4_gemv(mw_gu, ms_gu, oracle.rmsnorm(mx[0], gamma, 1e-6)), 2))),
            37888 * 1792 + 37888 * 28 * 2 + 3584 * 9472 + 3584 * 148 * 2),
    }
    all_threads = oracle.set_threads(0)
    out = {"nproc": os.cpu_count(), "threads_all": all_threads}
    try:
        aff = os.sched_getaffinity(0)
    except AttributeError:
        aff = None
    for name, (fn, nbytes) in units.items():
        rec = {"bytes": nbytes}
        for label, threads in (("one_thread", 1), ("all_threads", all_threads)):
            oracle.set_threads(threads)
            if threads == 1 and aff:
                os.sched_setaffinity(0, {min(aff)})
            try:
                fn()
                reps, t0 = 0, time.perf_counter()
                while reps < 3 or time.perf_counter() - t0 < 0.5:
                    fn()
                    reps += 1
                ms = (time.perf_counter() - t0) / reps * 1e3
            finally:
                if aff:
                    os.sched_setaffinity(0, aff)
            rec[label] = {"ms": round(ms, 3), "GBs": round(nbytes / (ms * 1e-3) / 1e9, 3)}
        out[name] = rec
    oracle.set_threads(all_threads)
    return out


def run_reference(args):
    """CPU oracle arm: each step is one full decode token of the same workload (28 layers, final norm,
    lm_head, argmax) at positions 512, 513, ... after a KV cache of seeded random values; tok/s =
    steps / the timed steps' total time."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    from int4_weight_only_02_b200 import synth
    shape = synth.QWEN7B
    layers = [synth.layer_weights(shape, i, 0) for i in range(shape.layers)]
    glob = synth.global_weights(shape, 0)
    dec = primed_oracle(shape, layers, glob, 512, args.warmup + args.steps)
    threads = oracle.set_threads(0)
    tok, pos = int(synth.prompt_tokens(shape, 512, 0)[-1]), 512
    for _ in range(args.warmup):
        logits, _ = dec.forward([tok], pos)
        tok, pos = oracle.argmax(logits), pos + 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        logits, _ = dec.forward([tok], pos)
        tok, pos = oracle.argmax(logits), pos + 1
    el = time.perf_counter() - t0
    ms_tok = el / args.steps * 1e3
    value = args.steps / el
    sample = (f"{args.steps} timed full decode tokens (28 layers + lm_head + argmax) at positions "
              f"{512 + args.warmup}..{pos - 1} after {args.warmup} warm-up tokens; KV cache below position 512 "
              f"seeded random fp16; fp64 C/numpy oracle, {threads} OpenMP threads on {os.cpu_count()} host cpus "
              f"({el:.1f} s timed)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_tok, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "prompt": 512},
            "cpu_baseline": {"value": round(value, 5), "unit": "tok/s", "cores": threads,
                             "host_cpus": os.cpu_count(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(value_ms: float, world: int, device) -> float:
    """The slowest rank's time (all ranks take part in the same collective)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(steps: int, world: int, ms_max: float) -> float:
    """Replicas: every rank decodes `steps` tokens of its own sequence; the job rate uses the slowest rank."""
    return world * steps / (ms_max / 1e3)


def teacher_forced(i4, model, shape, gold, torch):
    """The oracle's 128 greedy tokens forced as the input stream after the 512-token prompt: at every step
    the GPU's argmax against the oracle's token, with the oracle's top-2 gap where they differ, and the
    first generated step's logits against the oracle's sampled logits."""
    import numpy as np

    from int4_weight_only_02_b200 import synth
    prompt = synth.prompt_tokens(shape, gold["n_prompt"], gold["seed"])
    want = np.asarray(gold["tokens"])
    gaps = np.asarray(gold["top2_gap"])
    forced = np.concatenate([prompt, want[:-1]]).astype(np.int32)
    seq = i4.Sequence(model, synth.page_table(shape, gold["seed"]), forced)
    g = i4.DecodeGraph(model, seq)
    for _ in range(len(prompt) - 1):
        g.replay()
    picks, first_err = [], None
    idx = np.asarray(gold["first_logits_sample"]["index"])
    ref = np.asarray(gold["first_logits_sample"]["value"])
    for i in range(len(want)):
        g.replay()
        lg = seq.logits.cpu().numpy()
        if i == 0:
            first_err = float(np.max(np.abs(lg[idx].astype(np.float64) - ref)))
        picks.append(int(np.flatnonzero(lg == lg.max())[0]))
    g.close()
    picks = np.asarray(picks)
    diff = np.flatnonzero(picks != want)
    return {"teacher_forced_agree": int(len(want) - diff.size), "teacher_forced_steps": int(len(want)),
            "teacher_forced_disagree_at": [[int(i), round(float(gaps[i]), 4)] for i in diff],
            "first_step_max_abs_logit_err": round(first_err, 5),
            "oracle_gaps_below_0.1": int(np.sum(gaps < 0.1))}


PROFILE_KERNELS = {"qkv": 0, "attention": 1, "o": 2, "gate_up": 3, "down": 4, "lm_head": 5, "token": -1,
                   "gemm_gate_up_m512": -2}


def run_profile_kernel(args):
    """One-layer decoder with the 7B layer shapes (1.5 GB on the device); launches one kernel of the
    decode step `--launches` times. Not a benchmark: a small, fixed case for ncu."""
    import torch

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    if args.pdl is not None:
        i4.set_option("pdl", args.pdl)
    if args.unpack is not None:
        i4.set_option("unpack", args.unpack)
    if args.gemv_ctas is not None:
        i4.set_option("gemv_ctas_per_sm", args.gemv_ctas)
    if args.gemv_prex is not None:
        i4.set_option("gemv_prex", args.gemv_prex)

    if args.l2_prefetch is not None:
        i4.set_option("l2_prefetch", args.l2_prefetch)
    if args.persistent is not None:
        i4.set_option("persistent", args.persistent)
    dev = torch.device("cuda", 0)
    if PROFILE_KERNELS[args.profile_kernel] == -2:  # prompt-prefill gate/up GEMM (tcgen05): M = 512 rows
        shape = synth.QWEN7B
        lw = synth.layer_weights(shape, 0, 0)
        w, sc = (i4.runtime.to_device(lw[k], dev) for k in ("w_gu", "s_gu"))
        x = (torch.randn(512, shape.hidden, device=dev) * 0.5).half()
        n_out = 2 * shape.inter
        y = torch.empty(512, n_out, device=dev, dtype=torch.float16)
        ws = torch.zeros(max(i4.int4_gemm_ws_bytes(512, n_out, shape.hidden), 256), dtype=torch.uint8, device=dev)
        for _ in range(args.launches):
            i4.int4_gemm(w, sc, x, y=y, ws=ws)
        torch.cuda.synchronize()
        print(json.dumps({"profile_kernel": args.profile_kernel, "launches": args.launches,
                          "M": 512, "N": n_out, "K": shape.hidden, "device_error": i4.device_error()}))
        return 0
    shape = synth.ModelShape(layers=1)
    layers = [synth.layer_weights(synth.QWEN7B, 0, 0)]
    glob = synth.global_weights(shape, 0)
    model = i4.DeviceModel(shape, layers, glob, device=dev)
    seq = i4.Sequence(model, synth.page_table(shape, 0), synth.prompt_tokens(shape, 512, 0))
    graph = i4.DecodeGraph(model, seq)
    for _ in range(args.prime_steps):
        graph.replay()
    k = PROFILE_KERNELS[args.profile_kernel]
    index = k if k < 5 else graph.phase_count - 1
    for _ in range(args.launches):
        if k < 0:
            graph.replay()  # the whole one-layer token step
        else:
            graph.launch_kernel(index)
    torch.cuda.synchronize()
    print(json.dumps({"profile_kernel": args.profile_kernel, "index": index, "launches": args.launches,
                      "persistent": graph.persistent, "device_error": i4.device_error()}))
    graph.close()
    return 0


def run_trace_step(args):
    """Phase timestamps of one persistent decode step of the 7B-shape model after a --prompt token prompt:
    per phase kind, the median over CTAs of the time from the phase start (grid barrier passed) to its input
    staged, from staged to done, and the barrier wait (the next phase's start after this CTA's done), in us;
    the raw [phase][cta][4] array goes to the .npz path given."""
    import numpy as np
    import torch

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    dev = torch.device("cuda", 0)
    i4.set_option("trace", 1)
    if args.l2_ahead is not None:
        i4.set_option("l2_ahead", args.l2_ahead)
    shape = synth.QWEN7B
    model = i4.DeviceModel.synthetic(shape, device=dev)
    seq = i4.Sequence(model, synth.page_table(shape, 0), synth.prompt_tokens(shape, args.prompt, 0))
    graph = i4.DecodeGraph(model, seq)
    if not graph.persistent:
        raise SystemExit("the trace needs the persistent step")
    for _ in range(args.prompt + 2):
        graph.replay()
    torch.cuda.synchronize()
    grid = torch.cuda.get_device_properties(dev).multi_processor_count
    tr = graph.trace(grid).astype(np.int64)
    np.savez(args.trace_step, trace=tr)
    kinds = ["qkv", "attention", "o", "gate_up", "down"]
    t0 = tr[0, :, 0].min()
    out = {}
    for pi in range(tr.shape[0]):
        kind = "lm_head" if pi == tr.shape[0] - 1 else kinds[pi % 5]
        start, staged, done = tr[pi, :, 0], tr[pi, :, 1], tr[pi, :, 2]
        nxt = tr[pi + 1, :, 0] if pi + 1 < tr.shape[0] else None
        has = done > 0
        rec = out.setdefault(kind, {"stage_us": [], "work_us": [], "wait_us": [], "span_us": []})
        if kind != "attention":
            m = has & (staged > 0)
            rec["stage_us"].append(float(np.median(staged[m] - start[m])) / 1e3 if m.any() else 0.0)
            rec["work_us"].append(float(np.median(done[m] - staged[m])) / 1e3 if m.any() else 0.0)
        else:
            rec["work_us"].append(float(np.median(done - start)) / 1e3)
        if nxt is not None:
            m = has
            rec["wait_us"].append(float(np.median(nxt[m] - done[m])) / 1e3 if m.any() else 0.0)
            rec["span_us"].append(float(nxt.min() - start.min()) / 1e3)
    summary = {k: {kk: round(float(np.mean(v)), 3) for kk, v in r.items() if v} for k, r in out.items()}
    print(json.dumps({"trace_step": args.trace_step, "ctx": int(seq.ctx_len.item()),
                      "token_us": round(float(tr[-1, :, 2].max() - t0) / 1e3, 1), "per_phase_mean": summary,
                      "device_error": i4.device_error()}), flush=True)
    graph.close()
    return 0


def run_attention_sweep(args):
    """Paged decode attention sweep (contexts 512-32768, page sizes 16 and 64, batches 1/8/32,
    ragged lengths uniform in [L/2, L], pages drawn from one shuffled shared pool): KV bytes read
    per second against the measured HBM peak, one JSON line per case. Each case is timed as a
    CUDA graph of (L2 flush, attention) pairs minus a graph of the flushes alone, so every launch
    starts L2-cold. K/V values come from a seeded device generator (timing only; parity is the
    tests' job)."""
    import numpy as np
    import torch

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    dev = torch.device("cuda", 0)
    peak, peak_kind = measured_peaks()
    gen = torch.Generator(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = 10

    def graph_ms(body):
        side = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.stream(side):
            body(side)  # warm-up outside the capture
            with torch.cuda.graph(g, stream=side):
                for _ in range(reps):
                    body(side)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        best = None
        for _ in range(3):
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / reps
            best = t if best is None else min(best, t)
        return best

    contexts = [int(c) for c in args.sweep_contexts.split(",")]
    for L in contexts:
        for P in (16, 64):
            for B in (1, 8, 32):
                lens = synth.ragged_lengths(L, B, seed=L + B) if B > 1 else np.array([L], np.int32)
                need = [(int(n) + P - 1) // P for n in lens]
                max_pages = max(need)
                n_pool = sum(need)
                perm = synth.rng_for(0, 7, L, P, B).permutation(n_pool).astype(np.int32)
                table = np.zeros((B, max_pages), np.int32)
                off = 0
                for b, n in enumerate(need):
                    table[b, :n] = perm[off:off + n]
                    off += n
                gen.manual_seed(L * 1000 + P * 10 + B)
                kp = torch.randn((n_pool, 4, P, 128), generator=gen, device=dev).half()
                vp = torch.randn((n_pool, 4, P, 128), generator=gen, device=dev).half()
                q = torch.randn((B, 28, 128), generator=gen, device=dev).half()
                tab = torch.from_numpy(table).to(dev)
                ctx = torch.from_numpy(lens.astype(np.int32)).to(dev)
                out = torch.empty_like(q)
                ws = torch.zeros(i4.paged_gqa_decode_ws_bytes(B, 28, 4, 128, P, max_pages), dtype=torch.uint8,
                                 device=dev)

                def flush_only(st):
                    flush.add_(1)

                def both(st):
                    flush.add_(1)
                    i4.paged_gqa_decode(q, kp, vp, tab, ctx, out=out, ws=ws, stream=st)

                ms = graph_ms(both) - graph_ms(flush_only)
                kv = int(lens.astype(np.int64).sum()) * 4 * 128 * 2 * 2
                gbs = kv / (ms * 1e-3) / 1e9
                print(json.dumps({"sweep": "paged_gqa_decode", "ctx_max": L, "page_size": P, "batch": B,
                                  "kv_bytes": kv, "us": round(ms * 1e3, 2), "GBs": round(gbs, 1),
                                  "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": peak_kind,
                                  "device_error": i4.device_error()}), flush=True)
                del kp, vp, q, out, ws
    return 0


def run_gemv_batch(args):
    """INT4 GEMV at the gate/up shape (K = 3584, N = 37888, plain fp16 output) for M = 1, 2, 4, 8 vectors:
    the first step of batched decode. Each launch is L2-cold (a graph of (flush, GEMV) pairs minus the
    flushes); one JSON line per M with weight GB/s against the measured HBM peak."""
    import numpy as np
    import torch

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    dev = torch.device("cuda", 0)
    peak, peak_kind = measured_peaks()
    n, k = 37888, 3584
    w, s, _, _ = synth.gemv_case(n, k, seed=0)
    wd, sd = torch.from_numpy(w).to(dev), torch.from_numpy(s).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = 10
    for m in (1, 2, 4, 8):
        x = torch.randn((m, k), generator=torch.Generator(device=dev).manual_seed(m), device=dev).half()
        y = torch.empty((m, n), dtype=torch.float16, device=dev)

        def graph_ms(with_gemv):
            side = torch.cuda.Stream()
            g = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            with torch.cuda.stream(side):
                i4.int4_gemv(wd, sd, x, y=y, stream=side)
                with torch.cuda.graph(g, stream=side):
                    for _ in range(reps):
                        flush.add_(1)
                        if with_gemv:
                            i4.int4_gemv(wd, sd, x, y=y, stream=side)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            best = None
            for _ in range(3):
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                t = e0.elapsed_time(e1) / reps
                best = t if best is None else min(best, t)
            return best

        ms = graph_ms(True) - graph_ms(False)
        wbytes = n * (k // 2) + n * (k // 128) * 2
        gbs = wbytes / (ms * 1e-3) / 1e9
        print(json.dumps({"gemv_batch": m, "N": n, "K": k, "us": round(ms * 1e3, 2), "weight_GBs": round(gbs, 1),
                          "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                          "vector_GEMVs_per_s": round(m / (ms * 1e-3), 1), "device_error": i4.device_error()}),
              flush=True)
    return 0


def run_int8_ab(args):
    """The INT8-activation A/B at the gate/up (K 3584, N 37888) and down (K 18944, N 3584) shapes, one vector:
    the production tensor-core path (unpack 3), the exact CUDA-core fp16 unpack (0) and the int8-activation
    dp4a variant (5), each L2-cold (a graph of (flush, GEMV) pairs minus the flushes), weight GB/s against the
    measured HBM peak, and each one's normwise error against the oracle on 256 sampled rows."""
    import numpy as np
    import torch

    import int4_weight_only_02_b200 as i4
    import oracle
    from int4_weight_only_02_b200 import synth
    dev = torch.device("cuda", 0)
    peak, peak_kind = measured_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = 10
    names = {3: "fp16 x, mma.sync (production)", 0: "fp16 x, exact CUDA-core unpack", 5: "int8 x, dp4a"}
    for n, k in ((37888, 3584), (3584, 18944)):
        w, s, x, _ = synth.gemv_case(n, k, seed=0)
        wd, sd, xd = (torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(dev) for a in (w, s, x))
        y = torch.empty((1, n), dtype=torch.float16, device=dev)
        rows = np.sort(np.random.default_rng(1).choice(n, size=256, replace=False))
        ref = oracle.f16(oracle.int4_linear(w[rows], s[rows], x))
        for unp in (3, 0, 5):
            def graph_ms(with_gemv):
                side = torch.cuda.Stream()
                g = torch.cuda.CUDAGraph()
                torch.cuda.synchronize()
                with torch.cuda.stream(side):
                    i4.int4_gemv(wd, sd, xd, y=y, unpack=unp, stream=side)
                    with torch.cuda.graph(g, stream=side):
                        for _ in range(reps):
                            flush.add_(1)
                            if with_gemv:
                                i4.int4_gemv(wd, sd, xd, y=y, unpack=unp, stream=side)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                best = None
                for _ in range(3):
                    e0.record()
                    g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    t = e0.elapsed_time(e1) / reps
                    best = t if best is None else min(best, t)
                return best

            ms = graph_ms(True) - graph_ms(False)
            err = float(np.max(np.abs(y.cpu().numpy()[0, rows].astype(np.float64) - ref[0])) /
                        np.max(np.abs(ref[0].astype(np.float64))))
            wbytes = n * (k // 2) + n * (k // 128) * 2
            gbs = wbytes / (ms * 1e-3) / 1e9
            print(json.dumps({"int8_ab": names[unp], "unpack": unp, "N": n, "K": k, "us": round(ms * 1e3, 2),
                              "weight_GBs": round(gbs, 1), "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                              "normwise_err_vs_oracle": err, "device_error": i4.device_error()}), flush=True)
    return 0


def run_batched_decode(args):
    """B sequences of the 7B-shape decoder decoded together (one CUDA graph of library calls per step),
    each with its own 512-token prompt (teacher-forced, untimed) and page-table row; then K timed steps.
    One JSON line: tokens/s over all sequences."""
    import numpy as np
    import torch

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    dev = torch.device("cuda", 0)
    B = args.batched_decode
    shape = synth.QWEN7B
    model = i4.DeviceModel.synthetic(shape, device=dev)
    tables = synth.rng_for(0, 9, B).permutation(B * shape.max_pages).astype(np.int32).reshape(B, shape.max_pages)
    bd = i4.BatchedDecode(model, tables, num_pages=B * shape.max_pages)
    prompts = np.stack([synth.prompt_tokens(shape, args.prompt, seed=b) for b in range(B)])
    bd.reset(prompts[:, 0])
    stream = torch.cuda.current_stream()
    for t in range(args.prompt):
        bd.step(stream=stream)
        if t + 1 < args.prompt:
            bd.tokens.copy_(torch.from_numpy(prompts[:, t + 1]).to(dev, non_blocking=False))
    torch.cuda.synchronize()
    bd.capture()
    for _ in range(args.warmup):
        bd.replay()
    torch.cuda.synchronize()
    ctx0 = int(bd.ctx_len[0].item())
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        bd.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"batched_decode": B, "metric": "decode tok/s, batch of sequences (7B-shape INT4)",
                      "value": round(B / (ms * 1e-3), 1), "unit": "tok/s", "ms_per_step": round(ms, 4),
                      "steps": args.steps, "warmup": args.warmup, "ctx_first": ctx0,
                      "ctx_last": int(bd.ctx_len[0].item()) - 1, "launches_per_step": (8 + -(-B // bd.down_rows)) * shape.layers + 4,
                      "device_error": i4.device_error()}), flush=True)
    return 0


def run_prefill(args):
    """Time to first token of the 7B-shape decoder for a --prompt token prompt, every prompt position at once:
    the linear layers on the tcgen05 INT4 GEMM (M = prompt rows), causal paged attention, lm_head for the last
    position (Prefill.run, one stream, CUDA events around it after one warm-up run). Beside it: the same prompt
    fed one token per step through the decode graph (the first tokens must agree), and one layer's parts at the
    full prompt (each timed alone over 10 launches): the four GEMMs with their tensor throughput, attention and
    the glue kernels. One JSON line; exit status 1 when the first tokens differ or a device error is set."""
    import numpy as np
    import torch

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    dev = torch.device("cuda", 0)
    shape = synth.QWEN7B
    n = args.prompt
    model = i4.DeviceModel.synthetic(shape, device=dev)
    table = synth.page_table(shape, 0)
    prompt = synth.prompt_tokens(shape, n, seed=0)
    seq = i4.Sequence(model, table, None)
    pre = i4.Prefill(model, seq, max_tokens=n)
    pre.run(prompt)  # warm-up: tensor maps, shared-memory attributes
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    pre.run(prompt)
    e1.record()
    torch.cuda.synchronize()
    ttft_ms = e0.elapsed_time(e1)
    tok = int(seq.token.item())

    def timed(fn, reps=10):
        fn()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    lw = model.layers[0]
    h, inter, nqkv = shape.hidden, shape.inter, shape.qkv_rows
    ws = pre.gemm_ws  # the split-K workspace the prefill itself uses
    parts = {
        "qkv_gemm": (lambda: i4.int4_gemm(lw["w_qkv"], lw["s_qkv"], pre.xn, lw["b_qkv"], y=pre.qkv, ws=ws), nqkv, h),
        "o_gemm": (lambda: i4.int4_gemm(lw["w_o"], lw["s_o"], pre.attn, y=pre.y, ws=ws), h, h),
        "gate_up_gemm": (lambda: i4.int4_gemm(lw["w_gu"], lw["s_gu"], pre.xn, y=pre.gu, ws=ws), 2 * inter, h),
        "down_gemm": (lambda: i4.int4_gemm(lw["w_d"], lw["s_d"], pre.mlp, y=pre.y, ws=ws), h, inter),
    }
    peak_tf, peak_kind = measured_tensor_peak()
    layer = {}
    gemm_ms = 0.0
    for name, (fn, N, K) in parts.items():
        ms = timed(fn)
        gemm_ms += ms
        tf = 2.0 * n * N * K / (ms * 1e-3) / 1e12
        layer[name] = {"us": round(ms * 1e3, 1), "TFLOPs": round(tf, 1), "frac_of_peak": round(tf / peak_tf, 4)}
    layer["attention_causal"] = {"us": round(1e3 * timed(lambda: i4.paged_gqa_decode_strided(
        pre.qkv, nqkv, shape.n_q, seq.k_pools[0], seq.v_pools[0], pre.tables, pre.ctx, pre.attn, pre.attn_ws)), 1)}
    layer["glue"] = {"us": round(1e3 * timed(lambda: (
        i4.rmsnorm(pre.y, lw["ln_post"], out=pre.xn, resid=pre.r), i4.silu_mul(pre.gu, out=pre.mlp),
        i4.rope_kv_append(pre.qkv, pre.pos, shape.n_q, shape.n_kv, shape.theta))), 1)}
    # the same prompt one token per step through the decode graph
    seq2 = i4.Sequence(model, table, prompt)
    graph = i4.DecodeGraph(model, seq2)
    for _ in range(n):
        graph.replay()
    torch.cuda.synchronize()
    seq2.reset()
    e0.record()
    for _ in range(n):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    token_ms = e0.elapsed_time(e1)
    first = int(seq2.history[n].item())
    graph.close()
    err = i4.device_error()
    layer_flops = 2.0 * n * (nqkv * h + h * h + 2 * inter * h + h * inter)
    print(json.dumps({"prefill": "tcgen05", "prompt": n, "ttft_ms": round(ttft_ms, 2),
                      "prompt_tok_s": round(n / (ttft_ms * 1e-3), 1),
                      "gemm_flops_per_token_step": layer_flops * shape.layers,
                      "gemm_TFLOPs_whole_prefill": round(layer_flops * shape.layers / (ttft_ms * 1e-3) / 1e12, 1),
                      "tensor_peak_TFLOPs": peak_tf, "tensor_peak_kind": peak_kind,
                      "layer0_parts": layer, "ttft_ms_token_by_token": round(token_ms, 2),
                      "first_token_prefill": tok, "first_token_graph": first, "device_error": err}), flush=True)
    if tok != first or err:
        print(f"prefill: first tokens differ ({tok} vs {first}) or device error {err}", file=sys.stderr)
        return 1
    return 0


def measured_tensor_peak():
    """Dense fp16/bf16 tensor peak (TFLOP/s): the measured cuBLAS bf16 burst figure, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst; fp16 runs at the same rate)"
    except Exception:
        return 1590.0, "fallback"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="i4", choices=["i4", "reference"])
    ap.add_argument("--prompt", type=int, default=512)
    ap.add_argument("--eager-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pdl", type=int, default=None, help="override programmatic dependent launch (0/1)")
    ap.add_argument("--unpack", type=int, default=None, help="override the GEMV unpack variant (0..4, 4 = per shape)")
    ap.add_argument("--gemv-ctas", type=int, default=None, help="override the GEMV CTAs per SM (1 or 2)")
    ap.add_argument("--gemv-prex", type=int, default=None,
                    help="override the weight stages a GEMV copies before its loads of x are issued (0..8)")
    ap.add_argument("--l2-prefetch", type=int, default=None, help="override the next-GEMV L2 prefetch (0/1)")
    ap.add_argument("--l2-ahead", type=int, default=None,
                    help="override the tiles each CTA of the persistent step prefetches into L2 ahead (0..64)")
    ap.add_argument("--persistent", type=int, default=None,
                    help="override the persistent one-kernel step (1) against one kernel per phase (0)")
    ap.add_argument("--profile-kernel", default=None, choices=sorted(PROFILE_KERNELS),
                    help="profiling mode: a one-layer model of the same shapes, then only this kernel of the "
                         "decode step, --launches times (for ncu captures)")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--prime-steps", type=int, default=0, help="profiling mode: decode steps run first")
    ap.add_argument("--trace-step", default=None,
                    help="phase timestamps of one persistent decode step, raw array saved to this .npz path")
    ap.add_argument("--attention-sweep", action="store_true",
                    help="paged attention sweep over contexts, page sizes 16/64 and batches 1/8/32 (KV GB/s)")
    ap.add_argument("--sweep-contexts", default="512,2048,8192,32768")
    ap.add_argument("--prefill", action="store_true",
                    help="time to first token of a --prompt token prompt prefilled on the tcgen05 GEMM")
    ap.add_argument("--batched-decode", type=int, default=0,
                    help="decode this many sequences together (1..8) through the batched library calls")
    ap.add_argument("--int8-ab", action="store_true",
                    help="INT8-activation (dp4a) GEMV against the fp16 paths at the gate/up and down shapes")
    ap.add_argument("--gemv-batch", action="store_true",
                    help="INT4 GEMV at the gate/up shape for 1, 2, 4 and 8 vectors (weight GB/s)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_kernel:
        return run_profile_kernel(args)
    if args.trace_step:
        return run_trace_step(args)
    if args.attention_sweep:
        return run_attention_sweep(args)
    if args.gemv_batch:
        return run_gemv_batch(args)
    if args.int8_ab:
        return run_int8_ab(args)
    if args.batched_decode:
        return run_batched_decode(args)
    if args.prefill:
        return run_prefill(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import numpy as np
    import torch
    import torch.distributed as dist

    import int4_weight_only_02_b200 as i4
    from int4_weight_only_02_b200 import synth
    from int4_weight_only_02_b200.runtime import to_device

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    i4.lib()
    if args.pdl is not None:
        i4.set_option("pdl", args.pdl)
    if args.unpack is not None:
        i4.set_option("unpack", args.unpack)
    if args.gemv_ctas is not None:
        i4.set_option("gemv_ctas_per_sm", args.gemv_ctas)
    if args.gemv_prex is not None:
        i4.set_option("gemv_prex", args.gemv_prex)

    if args.l2_prefetch is not None:
        i4.set_option("l2_prefetch", args.l2_prefetch)
    if args.persistent is not None:
        i4.set_option("persistent", args.persistent)
    if args.l2_ahead is not None:
        i4.set_option("l2_ahead", args.l2_ahead)

    shape = synth.QWEN7B
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    layers_np = []
    model = i4.DeviceModel.__new__(i4.DeviceModel)
    model.shape, model.device, model.layers = shape, dev, []
    for li in range(shape.layers):
        lw = synth.layer_weights(shape, li, 0)
        model.layers.append({k: to_device(v, dev) for k, v in lw.items()})
        if want_cpu:
            layers_np.append(lw)
    glob_np = synth.global_weights(shape, 0)
    model.glob = {k: to_device(v, dev) for k, v in glob_np.items()}
    if not want_cpu:
        glob_np = None

    prompt = synth.prompt_tokens(shape, args.prompt, seed=rank)
    seq = i4.Sequence(model, synth.page_table(shape, 0), prompt)
    graph = i4.DecodeGraph(model, seq)
    n_k = graph.kernel_count
    stream = torch.cuda.current_stream()

    # prompt ingestion and warm-up (untimed)
    for _ in range(args.prompt + args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    ctx0 = int(seq.ctx_len.item())

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    ms_tok = ms_max / args.steps
    status = int(seq.status.item())
    ctx1 = int(seq.ctx_len.item())

    # end to end through the public API: token host->device, step, next token device->host, every step
    tok_h = torch.empty(1, dtype=torch.int32, pin_memory=True)
    out_h = torch.empty(1, dtype=torch.int32, pin_memory=True)
    tok_h.copy_(seq.token.cpu())
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        seq.token.copy_(tok_h, non_blocking=True)
        graph.replay()
        out_h.copy_(seq.token, non_blocking=True)
        stream.synchronize()
        tok_h[0] = out_h[0]
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_tok_s = job_tokens_per_s(args.steps, world, max_over_ranks(e0.elapsed_time(e1), world, dev))

    # spread over a longer decode: 8 more chunks of 16 tokens, ms/token of each chunk
    chunk_ms = []
    for _ in range(8):
        e0.record(stream)
        for _ in range(16):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        chunk_ms.append(e0.elapsed_time(e1) / 16)
    ctx_spread = int(seq.ctx_len.item()) - 1

    # eager launches of the same kernels (the pages' eager-vs-graph comparison)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.eager_steps):
        graph.eager()
    e1.record(stream)
    torch.cuda.synchronize()
    eager_ms = e0.elapsed_time(e1) / max(args.eager_steps, 1)

    # dominant kernel alone: RMSNorm + gate/up GEMV + SiLU of each layer (70 MB each, L2-cold)
    spreads = {}

    def time_kernel(index_fn, reps=10, name=None):
        """Mean device time of one launch: the kernel of every layer captured back to back in one
        CUDA graph, each of `reps` replays timed between two events on the launching stream; the
        per-launch minimum and maximum over the replays go to spreads[name]."""
        side = torch.cuda.Stream()
        cg = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.stream(side):
            with torch.cuda.graph(cg, stream=side):
                for li in range(shape.layers):
                    graph.launch_kernel(index_fn(li))
        torch.cuda.synchronize()
        cg.replay()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        ev[0].record(stream)
        for r in range(reps):
            cg.replay()
            ev[r + 1].record(stream)
        torch.cuda.synchronize()
        per = [ev[r].elapsed_time(ev[r + 1]) / shape.layers for r in range(reps)]
        if name:
            spreads[name] = (min(per), max(per))
        return ev[0].elapsed_time(ev[reps]) / (reps * shape.layers)

    h, inter = shape.hidden, shape.inter
    gu_bytes = 2 * inter * (h // 2) + 2 * inter * (h // 128) * 2 + 2 * h * 2 + inter * 2
    gu_ms = time_kernel(lambda li: 5 * li + 3, name="gate_up")
    down_bytes = h * (inter // 2) + h * (inter // 128) * 2 + inter * 2 + 2 * h * 2
    down_ms = time_kernel(lambda li: 5 * li + 4, name="down")
    qkv_rows = shape.qkv_rows
    qkv_bytes = qkv_rows * (h // 2) + qkv_rows * (h // 128) * 2 + 2 * qkv_rows * 2 + 2 * h * 2
    qkv_ms = time_kernel(lambda li: 5 * li + 0, name="qkv")
    o_bytes = h * (h // 2) + h * (h // 128) * 2 + h * 2 + 2 * h * 2
    o_ms = time_kernel(lambda li: 5 * li + 2, name="o")
    attn_ms = time_kernel(lambda li: 5 * li + 1, name="attention")
    # lm_head: the last kernel of the step, launched 28 times (it also advances the sequence state,
    # which nothing reads afterwards)
    lm_bytes = shape.vocab * (h // 2) + shape.vocab * (h // 128) * 2 + shape.vocab * 4 + 2 * h * 2
    lm_ms = time_kernel(lambda li: graph.phase_count - 1, name="lm_head")
    torch.cuda.synchronize()
    # restore a consistent residual/KV state is not needed afterwards: nothing else runs

    peak, peak_kind = measured_peaks()
    gu_gbs = gu_bytes / (gu_ms * 1e-3) / 1e9

    weight_bytes = model.weight_bytes()
    ctx_mean = (ctx0 + ctx1 - 1) / 2.0
    kv_bytes = 2 * shape.layers * shape.n_kv * shape.head_dim * 2 * ctx_mean
    step_bytes = weight_bytes + kv_bytes
    step_gbs = step_bytes / (ms_tok * 1e-3) / 1e9
    if graph.persistent:
        # the dominant (and only) kernel: one launch per token streams every weight byte and the context's K/V
        roofline = {"kernel": "decode_persistent_kernel: the whole token (28 x {qkv, attention, o, gate/up, "
                              "down} + lm_head) in one launch, one CTA per SM",
                    "bound": "hbm", "achieved": round(step_gbs, 1), "peak": peak,
                    "peak_kind": f"{peak_kind} copy bandwidth", "unit": "GB/s", "frac": round(step_gbs / peak, 4),
                    "traffic": traffic_from_profile("decode_persistent_qwen7b.md", PERSIST_SOURCES),
                    "bytes_per_launch": int(step_bytes), "us_per_launch": round(ms_tok * 1e3, 2),
                    "timing": "CUDA events over the timed graph replays (one kernel per replay)"}
    else:
        roofline = {"kernel": "rmsnorm+gate/up int4 gemv+silu (K=3584, N=37888)", "bound": "hbm",
                    "achieved": round(gu_gbs, 1), "peak": peak, "peak_kind": f"{peak_kind} copy bandwidth",
                    "unit": "GB/s", "frac": round(gu_gbs / peak, 4),
                    "traffic": traffic_from_profile("gemv_gate_up_qwen7b.md", GEMV_SOURCES),
                    "bytes_per_launch": gu_bytes, "us_per_launch": round(gu_ms * 1e3, 2)}

    line = {
        "metric": METRIC, "value": round(job_tokens_per_s(args.steps, world, ms_max), 2), "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_tok, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "prompt": args.prompt, "ctx_first": ctx0, "ctx_last": ctx1 - 1,
                   "arith": "int4 weights x fp16 activations, fp32 accumulate", "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2: 3.65 GB of weights streamed per step, no flush",
                   "kernels_per_step": n_k, "status": status},
        "roofline": roofline,
        "persistent_step": graph.persistent,
        # each phase launched alone (its own launch, stream start-up and drain): diagnostics only; mean
        # over 10 graph replays of the 28 launches, with the per-launch min/max over the replays
        "phase_launches_spread_us": {k: [round(a * 1e3, 2), round(b * 1e3, 2)] for k, (a, b) in spreads.items()},
        "phase_launches": {
            "qkv": {"us": round(qkv_ms * 1e3, 2), "GBs": round(qkv_bytes / (qkv_ms * 1e-3) / 1e9, 1)},
            "o": {"us": round(o_ms * 1e3, 2), "GBs": round(o_bytes / (o_ms * 1e-3) / 1e9, 1)},
            "gate_up": {"us": round(gu_ms * 1e3, 2), "GBs": round(gu_gbs, 1)},
            "down": {"us": round(down_ms * 1e3, 2), "GBs": round(down_bytes / (down_ms * 1e-3) / 1e9, 1)},
            "attention": {"us": round(attn_ms * 1e3, 2),
                          "GBs": round(2 * shape.n_kv * shape.head_dim * 2 * (ctx1 - 1) / (attn_ms * 1e-3) / 1e9, 1)},
            "lm_head": {"us": round(lm_ms * 1e3, 2), "GBs": round(lm_bytes / (lm_ms * 1e-3) / 1e9, 1)}},
        "step_roofline": {"bytes_per_step": int(step_bytes), "achieved_GBs": round(step_gbs, 1),
                          "frac_of_8TBs": round(step_gbs / NOMINAL_HBM_GBS, 4),
                          "frac_of_measured": round(step_gbs / peak, 4)},
        "eager_ms_per_step": round(eager_ms, 3),
        "token_spread": {"tokens": 128, "chunks": 8, "ctx_last": ctx_spread,
                         "ms_per_token_min": round(min(chunk_ms), 4),
                         "ms_per_token_median": round(statistics.median(chunk_ms), 4),
                         "ms_per_token_max": round(max(chunk_ms), 4)},
        "e2e": {"value": round(e2e_tok_s, 2), "unit": "tok/s", "h2d_bytes_per_step": 4, "d2h_bytes_per_step": 4},
        "gpu_launches": args.steps * n_k,
        "clocks": clocks.summary(),
    }
    golden = os.path.join(ROOT, "tests", "golden", "decode_qwen7b_int4_seed0.json")
    if rank == 0 and args.prompt == 512 and os.path.exists(golden):
        gold = json.load(open(golden))
        hist = seq.history.cpu().numpy()[512: 512 + len(gold["tokens"])]
        n = min(len(hist), int(seq.pos.item()) + 1 - 512)
        same = 0
        while same < n and int(hist[same]) == int(gold["tokens"][same]):
            same += 1
        line["greedy_vs_oracle"] = {"compared": n, "identical_prefix": same,
                                    "note": "free-running; first difference expected at an oracle top-2 near-tie"}
        line["greedy_vs_oracle"].update(teacher_forced(i4, model, shape, gold, torch))
    graph.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if want_cpu:
            del model, seq
            line["cpu_baseline"] = oracle_cpu_sample(shape, layers_np, glob_np)
            del layers_np, glob_np
            line["cpu_baseline_units"] = oracle_unit_configs()
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
