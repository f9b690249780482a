"""Device-side model, sequence state and the captured decode step (argument marshalling only).

``DeviceModel`` holds the INT4 weights of a Qwen2.5-7B-shaped decoder in HBM,
``Sequence`` one sequence's paged KV pools and on-device decode state, and
``DecodeGraph`` the decode step of ``libi4rt`` (one CUDA graph per token,
``decode_step_graph_*``). PyTorch only allocates the memory.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import (LayerWeights, ModelDesc, ModelWeights, SeqState, _check, _p, _stream, lib, synth)

_LAYER_KEYS = ("w_qkv", "s_qkv", "b_qkv", "w_o", "s_o", "w_gu", "s_gu", "w_d", "s_d", "ln_in", "ln_post")
_LAYER_FIELDS = ("w_qkv", "s_qkv", "b_qkv", "w_o", "s_o", "w_gate_up", "s_gate_up", "w_down", "s_down", "ln_in",
                 "ln_post")


def to_device(a: np.ndarray, device="cuda"):
    """Upload a numpy array; uint32 words travel as int32 (same bits)."""
    import torch
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def _gemm_workspace(s, rows: int, dev):
    """A zeroed split-K workspace for every linear layer of the model at `rows` activation rows."""
    import torch
    from . import int4_gemm_ws_bytes
    nqkv = (s.n_q + 2 * s.n_kv) * s.head_dim
    shapes = [(nqkv, s.hidden), (s.hidden, s.n_q * s.head_dim), (2 * s.inter, s.hidden), (s.hidden, s.inter),
              (s.vocab, s.hidden)]
    nbytes = max(int4_gemm_ws_bytes(rows, n, k) for n, k in shapes)
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)


class DeviceModel:
    def __init__(self, shape: synth.ModelShape, layers, glob, device="cuda"):
        self.shape = shape
        self.device = device
        self.layers = [{k: to_device(v, device) for k, v in lw.items()} for lw in layers]
        self.glob = {k: to_device(v, device) for k, v in glob.items()}

    @classmethod
    def synthetic(cls, shape: synth.ModelShape = synth.QWEN7B, seed: int = 0, device="cuda"):
        """Random-init weights of the given shape, generated and uploaded one layer at a time."""
        self = cls.__new__(cls)
        self.shape, self.device = shape, device
        self.layers = []
        for i in range(shape.layers):
            self.layers.append({k: to_device(v, device) for k, v in synth.layer_weights(shape, i, seed).items()})
        self.glob = {k: to_device(v, device) for k, v in synth.global_weights(shape, seed).items()}
        return self

    def weight_bytes(self) -> int:
        """INT4 words + fp16 scales streamed per token (28 layers and lm_head)."""
        n = 0
        for lw in self.layers:
            for k in ("w_qkv", "s_qkv", "w_o", "s_o", "w_gu", "s_gu", "w_d", "s_d"):
                n += lw[k].numel() * lw[k].element_size()
        for k in ("w_lm", "s_lm"):
            n += self.glob[k].numel() * self.glob[k].element_size()
        return n

    def desc(self) -> ModelDesc:
        s = self.shape
        return ModelDesc(s.layers, s.hidden, s.inter, s.n_q, s.n_kv, s.head_dim, s.vocab, s.group, s.page_size,
                         s.max_ctx, s.theta, s.eps)


class Sequence:
    """One sequence: K/V pools per layer, a page table, and the on-device decode state."""

    def __init__(self, model: DeviceModel, page_table: np.ndarray, prompt: np.ndarray | None = None,
                 num_pages: int | None = None):
        import torch
        s, dev = model.shape, model.device
        self.model = model
        self.num_pages = int(num_pages if num_pages is not None else s.max_pages)
        kv = (self.num_pages, s.n_kv, s.page_size, s.head_dim)
        self.k_pools = [torch.zeros(kv, dtype=torch.float16, device=dev) for _ in range(s.layers)]
        self.v_pools = [torch.zeros(kv, dtype=torch.float16, device=dev) for _ in range(s.layers)]
        self.page_table = to_device(np.asarray(page_table, dtype=np.int32), dev)
        self.token = torch.zeros(1, dtype=torch.int32, device=dev)
        self.pos = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ctx_len = torch.ones(1, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.logits = torch.zeros(s.vocab, dtype=torch.float32, device=dev)
        self.history = torch.zeros(s.max_ctx, dtype=torch.int32, device=dev)
        self.prompt = None
        if prompt is not None:
            self.prompt = to_device(np.asarray(prompt, dtype=np.int32), dev)
        self.reset()

    def reset(self, first_token: int | None = None):
        """Position 0 with the first prompt token (or `first_token`)."""
        tok = first_token
        if tok is None:
            tok = int(self.prompt[0].item()) if self.prompt is not None else 0
        self.token.fill_(tok)
        self.pos.zero_()
        self.ctx_len.fill_(1)
        self.status.zero_()
        self.history.zero_()
        self.history[0] = tok

    def state(self) -> SeqState:
        self._kp = (ctypes.c_void_p * len(self.k_pools))(*[t.data_ptr() for t in self.k_pools])
        self._vp = (ctypes.c_void_p * len(self.v_pools))(*[t.data_ptr() for t in self.v_pools])
        return SeqState(self.token.data_ptr(), self.pos.data_ptr(), self.ctx_len.data_ptr(),
                        self.page_table.data_ptr(), self._kp, self._vp, self.num_pages, self.logits.data_ptr(),
                        self.prompt.data_ptr() if self.prompt is not None else None,
                        int(self.prompt.numel()) if self.prompt is not None else 0,
                        self.history.data_ptr(), self.status.data_ptr())


class DecodeGraph:
    """The decode step of libi4rt: ``replay()`` runs one token as one cudaGraphLaunch."""

    def __init__(self, model: DeviceModel, seq: Sequence):
        self.model, self.seq = model, seq
        layers = (LayerWeights * len(model.layers))()
        for i, lw in enumerate(model.layers):
            for key, field in zip(_LAYER_KEYS, _LAYER_FIELDS):
                setattr(layers[i], field, lw[key].data_ptr())
        g = model.glob
        weights = ModelWeights(g["embed"].data_ptr(), layers, g["ln_final"].data_ptr(), g["w_lm"].data_ptr(),
                               g["s_lm"].data_ptr())
        desc = model.desc()
        state = seq.state()
        handle = ctypes.c_void_p()
        _check(lib().decode_step_graph_create(ctypes.byref(desc), ctypes.byref(weights), ctypes.byref(state),
                                              ctypes.byref(handle)), "decode_step_graph_create")
        self._h = handle

    @property
    def kernel_count(self) -> int:
        """Kernel launches per step (1 for the persistent step)."""
        return int(lib().decode_step_kernel_count(self._h))

    @property
    def phase_count(self) -> int:
        """Phases per step: 5 per layer (qkv, attention, o, gate/up, down) and lm_head."""
        return int(lib().decode_step_phase_count(self._h))

    @property
    def persistent(self) -> bool:
        return bool(lib().decode_step_is_persistent(self._h))

    def trace(self, grid: int):
        """Phase timestamps of the last launch [phase][cta][4] (ns; graphs created with the "trace" option)."""
        n = self.phase_count * grid * 4
        buf = (ctypes.c_ulonglong * n)()
        _check(lib().decode_step_trace(self._h, buf, n), "decode_step_trace")
        return np.frombuffer(buf, dtype=np.uint64).reshape(self.phase_count, grid, 4).copy()

    def replay(self, stream=None):
        _check(lib().decode_step_graph_replay(self._h, _stream(stream)), "decode_step_graph_replay")

    def eager(self, stream=None):
        _check(lib().decode_step_eager(self._h, _stream(stream)), "decode_step_eager")

    def launch_kernel(self, index: int, stream=None):
        """Run only phase `index` of the step as one launch (tests, benchmarking; see decode_step_launch_kernel)."""
        _check(lib().decode_step_launch_kernel(self._h, index, _stream(stream)), "decode_step_launch_kernel")

    BUFFERS = {"resid": 0, "q": 1, "attn": 2, "mlp": 3}

    def _buffer_len(self, name: str) -> int:
        s = self.model.shape
        return {"resid": s.hidden, "q": s.n_q * s.head_dim, "attn": s.n_q * s.head_dim, "mlp": s.inter}[name]

    def read_buffer(self, name: str, stream=None):
        """Copy of one of the step's activation buffers ('resid', 'q', 'attn', 'mlp') as an fp16 tensor."""
        import torch
        out = torch.empty(self._buffer_len(name), dtype=torch.float16, device=self.model.device)
        _check(lib().decode_step_buffer_copy(self._h, self.BUFFERS[name], _p(out), out.numel() * 2, 0,
                                             _stream(stream)), "decode_step_buffer_copy")
        return out

    def write_buffer(self, name: str, values, stream=None):
        """Overwrite one of the step's activation buffers with fp16 `values` (a device tensor)."""
        import torch
        v = values.to(device=self.model.device, dtype=torch.float16).contiguous()
        assert v.numel() == self._buffer_len(name)
        _check(lib().decode_step_buffer_copy(self._h, self.BUFFERS[name], _p(v), v.numel() * 2, 1,
                                             _stream(stream)), "decode_step_buffer_copy")
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()

    def close(self):
        if getattr(self, "_h", None):
            _check(lib().decode_step_graph_destroy(self._h), "decode_step_graph_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class BatchedDecode:
    """B sequences decoded together: one step is a CUDA graph of library calls -- embedding gather,
    batched INT4 linear layers (B <= 8: the B vectors as mma.sync columns where the shape allows; B > 8:
    the tcgen05 GEMM), batched
    RMSNorm (+ residual), RoPE + K/V append, B-sequence paged attention reading q inside the qkv
    rows, SiLU-mul, lm_head and a per-row argmax that advances each sequence's position.
    Every sequence has its own page-table row over per-layer pools shared by the batch.
    """

    def __init__(self, model: DeviceModel, page_tables: np.ndarray, num_pages: int):
        import torch
        from . import paged_gqa_decode_ws_bytes
        s, dev = model.shape, model.device
        self.model, self.shape = model, s
        self.B = B = int(page_tables.shape[0])
        self._tables_np = np.asarray(page_tables, dtype=np.int32).copy()
        self.page_tables = to_device(self._tables_np, dev)
        kv = (int(num_pages), s.n_kv, s.page_size, s.head_dim)
        self.k_pools = [torch.zeros(kv, dtype=torch.float16, device=dev) for _ in range(s.layers)]
        self.v_pools = [torch.zeros(kv, dtype=torch.float16, device=dev) for _ in range(s.layers)]
        i32 = dict(dtype=torch.int32, device=dev)
        f16 = dict(dtype=torch.float16, device=dev)
        self.tokens = torch.zeros(B, **i32)
        self.pos = torch.zeros(B, **i32)
        self.ctx_len = torch.ones(B, **i32)
        nqkv = (s.n_q + 2 * s.n_kv) * s.head_dim
        self.r = torch.zeros((B, s.hidden), **f16)
        self.xn = torch.zeros((B, s.hidden), **f16)
        self.qkv = torch.zeros((B, nqkv), **f16)
        self.attn = torch.zeros((B, s.n_q * s.head_dim), **f16)
        self.y = torch.zeros((B, s.hidden), **f16)
        self.gu = torch.zeros((B, 2 * s.inter), **f16)
        self.mlp = torch.zeros((B, s.inter), **f16)
        self.logits = torch.zeros((B, s.vocab), dtype=torch.float32, device=dev)
        nbytes = paged_gqa_decode_ws_bytes(B, s.n_q, s.n_kv, s.head_dim, s.page_size, page_tables.shape[1])
        self.attn_ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.gemm_ws = _gemm_workspace(s, B, dev) if B > 8 else None
        self.graph = None
        # vectors per down-projection call: the batched tensor-core GEMV takes rows of up to 4096 weights;
        # longer rows go through the register kernel, whose x stage holds a power-of-two number of vectors
        # at 68 bytes per 32 weights each, within 200 KB
        self.down_rows = B
        if s.inter > 4096 and B <= 8:  # more than 8 rows run on the tcgen05 GEMM, which takes any row length
            mr = 1
            while mr * 2 <= B and mr * 2 * (s.inter // 32) * 68 <= 200 * 1024:
                mr *= 2
            self.down_rows = mr

    def reset(self, first_tokens):
        """Position 0 of every sequence, with the given first tokens."""
        import torch
        self.tokens.copy_(torch.as_tensor(np.asarray(first_tokens, dtype=np.int32)))
        self.pos.zero_()
        self.ctx_len.fill_(1)

    def _linear(self, w, sc, x, bias=None, y=None, out_fp32=False, stream=None):
        from . import int4_gemm, int4_gemv
        if self.B > 8:  # the tcgen05 GEMM, K split over CTAs where the tiles leave SMs idle
            return int4_gemm(w, sc, x, bias, y=y, out_fp32=out_fp32, ws=self.gemm_ws, stream=stream)
        return int4_gemv(w, sc, x, bias, y=y, out_fp32=out_fp32, stream=stream)

    def step(self, stream=None):
        """Enqueue one decode step of all B sequences on `stream` (no allocation, capturable)."""
        from . import argmax_rows, embed_gather, paged_gqa_decode_strided, rmsnorm, rope_kv_append, silu_mul
        int4_gemv = self._linear
        m, s = self.model, self.shape
        g, L = m.glob, m.layers
        nqkv = (s.n_q + 2 * s.n_kv) * s.head_dim
        embed_gather(g["embed"], self.tokens, self.r, stream=stream)
        rmsnorm(self.r, L[0]["ln_in"], out=self.xn, eps=s.eps, stream=stream)
        for li, lw in enumerate(L):
            int4_gemv(lw["w_qkv"], lw["s_qkv"], self.xn, lw["b_qkv"], y=self.qkv, stream=stream)
            rope_kv_append(self.qkv, self.pos, s.n_q, s.n_kv, s.theta, self.k_pools[li], self.v_pools[li],
                           self.page_tables, stream=stream)
            paged_gqa_decode_strided(self.qkv, nqkv, s.n_q, self.k_pools[li], self.v_pools[li], self.page_tables,
                                     self.ctx_len, self.attn, self.attn_ws, stream=stream)
            int4_gemv(lw["w_o"], lw["s_o"], self.attn, y=self.y, stream=stream)
            rmsnorm(self.y, lw["ln_post"], out=self.xn, resid=self.r, eps=s.eps, stream=stream)
            int4_gemv(lw["w_gu"], lw["s_gu"], self.xn, y=self.gu, stream=stream)
            silu_mul(self.gu, out=self.mlp, stream=stream)
            for m0 in range(0, self.B, self.down_rows):  # rows beyond 4096 weights: the x stage holds <= 4 vectors
                int4_gemv(lw["w_d"], lw["s_d"], self.mlp[m0:m0 + self.down_rows], y=self.y[m0:m0 + self.down_rows],
                          stream=stream)
            gamma = L[li + 1]["ln_in"] if li + 1 < len(L) else g["ln_final"]
            rmsnorm(self.y, gamma, out=self.xn, resid=self.r, eps=s.eps, stream=stream)
        int4_gemv(g["w_lm"], g["s_lm"], self.xn, y=self.logits, out_fp32=True, stream=stream)
        argmax_rows(self.logits, self.tokens, self.pos, self.ctx_len, stream=stream)

    def capture(self):
        """Capture one step as a CUDA graph (after one eager step has configured every kernel)."""
        import torch
        side = torch.cuda.Stream()
        self.graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.stream(side):
            with torch.cuda.graph(self.graph, stream=side):
                self.step(stream=side)
        torch.cuda.synchronize()

    def replay(self):
        self.graph.replay()

    def prefill(self, prompt, graph: bool = True) -> int:
        """Causal prefill of ONE sequence, B prompt tokens per step: every row of the batch is one prompt
        position of the same sequence (all page-table rows must be equal), row b at position c + b with
        context c + b + 1, so attention over the shared pages is causal and the K/V of the whole chunk land
        before any row reads them. len(prompt) must be a multiple of B and fit the page-table row. Returns
        the first generated token (the argmax at the last prompt position).

        Afterwards the K/V of positions 0..n-1 sit in this object's pools and row b of the batch is at
        position n - B + b + 1; decoding of the sequence continues from position n with
        ``continue_state(n, first_token)`` (every row then computes the same next token)."""
        import torch
        prompt = np.asarray(prompt, dtype=np.int32)
        B, n = self.B, len(prompt)
        if n % B:
            raise ValueError(f"prompt length {n} is not a multiple of the batch {B}")
        if not np.all(self._tables_np == self._tables_np[:1]):
            raise ValueError("prefill needs every page-table row to be the same sequence's row")
        cap = self._tables_np.shape[1] * self.shape.page_size
        if n > cap:
            raise ValueError(f"prompt length {n} exceeds the page-table row ({cap} positions)")
        if graph and self.graph is None:
            self._prefill_chunk(prompt[:B], 0)
            self.step()
            torch.cuda.synchronize()
            self.capture()
            start = B
        else:
            start = 0
        for c in range(start, n, B):
            self._prefill_chunk(prompt[c:c + B], c)
            self.replay() if graph else self.step()
        torch.cuda.synchronize()
        return int(self.tokens[B - 1].item())

    def continue_state(self, n: int, first_token: int):
        """After ``prefill`` of n tokens: every row set to decode the same sequence at position n (token
        first_token, context n + 1) over the K/V the prefill left in this object's pools."""
        import torch
        self.tokens.fill_(int(first_token))
        self.pos.fill_(int(n))
        self.ctx_len.fill_(int(n) + 1)

    def _prefill_chunk(self, tokens, c: int):
        import torch
        self.tokens.copy_(torch.from_numpy(np.ascontiguousarray(tokens)))
        self.pos.copy_(torch.arange(c, c + self.B, dtype=torch.int32))
        self.ctx_len.copy_(torch.arange(c + 1, c + self.B + 1, dtype=torch.int32))


class Prefill:
    """Prompt prefill of one sequence with every prompt position at once.

    Per layer the n prompt positions are n activation rows: batched RMSNorm, the qkv / o / gate-up / down
    linear layers on the tcgen05 INT4 GEMM (``int4_gemm``), RoPE and the K/V append of all n positions into
    the Sequence's own pages, causal paged attention (query row p over positions 0..p of the same pages, read
    inside the qkv rows), SiLU-mul and the residual adds. The final norm and lm_head run for the last position
    only; the argmax becomes the sequence's next token, so a DecodeGraph over the same Sequence continues at
    position n. All launches go to one stream (no host synchronisation inside ``run``).
    """

    def __init__(self, model: DeviceModel, seq: Sequence, max_tokens: int = 512):
        import torch
        from . import paged_gqa_decode_ws_bytes
        s, dev = model.shape, model.device
        self.model, self.seq, self.shape = model, seq, s
        self.n_max = n = int(max_tokens)
        if n > s.max_ctx - 1:
            raise ValueError(f"max_tokens {n} leaves no room for decoding within max_ctx {s.max_ctx}")
        i32 = dict(dtype=torch.int32, device=dev)
        f16 = dict(dtype=torch.float16, device=dev)
        nqkv = (s.n_q + 2 * s.n_kv) * s.head_dim
        self.tokens = torch.zeros(n, **i32)
        self.pos = torch.arange(n, **i32)
        self.ctx = torch.arange(1, n + 1, **i32)
        # every row reads the sequence's own page-table row
        self.tables = seq.page_table.view(1, -1).expand(n, -1).contiguous()
        self.r = torch.zeros((n, s.hidden), **f16)
        self.xn = torch.zeros((n, s.hidden), **f16)
        self.qkv = torch.zeros((n, nqkv), **f16)
        self.attn = torch.zeros((n, s.n_q * s.head_dim), **f16)
        self.y = torch.zeros((n, s.hidden), **f16)
        self.gu = torch.zeros((n, 2 * s.inter), **f16)
        self.mlp = torch.zeros((n, s.inter), **f16)
        self.logits = torch.zeros((1, s.vocab), dtype=torch.float32, device=dev)
        # the attention workspace for any prompt length up to n (its split layout depends on the row count)
        nbytes = max(paged_gqa_decode_ws_bytes(b, s.n_q, s.n_kv, s.head_dim, s.page_size, self.tables.shape[1])
                     for b in range(1, n + 1))
        self.attn_ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.gemm_ws = _gemm_workspace(s, n, dev)

    def run(self, prompt, stream=None):
        """Enqueue the prefill of `prompt` (host ids or a device int32 tensor, 1 <= n <= max_tokens) on `stream`;
        afterwards the Sequence holds the prompt's K/V, token = the first generated token, pos = n,
        ctx_len = n + 1 and history[0..n] = prompt + that token."""
        import torch
        from . import (argmax_rows, embed_gather, int4_gemm, int4_gemv, paged_gqa_decode_strided, rmsnorm,
                       rope_kv_append, silu_mul)
        m, s, seq = self.model, self.shape, self.seq
        g, L = m.glob, m.layers
        if isinstance(prompt, torch.Tensor):
            n = int(prompt.numel())
            toks = prompt.to(device=m.device, dtype=torch.int32)
        else:
            prompt = np.asarray(prompt, dtype=np.int32)
            n = len(prompt)
            toks = torch.from_numpy(prompt).to(m.device)
        if not 1 <= n <= self.n_max:
            raise ValueError(f"prompt length {n} outside [1, {self.n_max}]")
        nqkv = (s.n_q + 2 * s.n_kv) * s.head_dim
        st = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(st):
            self.tokens[:n].copy_(toks, non_blocking=True)
            r, xn, qkv, attn, y, gu, mlp = (t[:n] for t in (self.r, self.xn, self.qkv, self.attn, self.y, self.gu,
                                                            self.mlp))
            embed_gather(g["embed"], self.tokens[:n], r, stream=st)
            rmsnorm(r, L[0]["ln_in"], out=xn, eps=s.eps, stream=st)
            for li, lw in enumerate(L):
                int4_gemm(lw["w_qkv"], lw["s_qkv"], xn, lw["b_qkv"], y=qkv, ws=self.gemm_ws, stream=st)
                rope_kv_append(qkv, self.pos[:n], s.n_q, s.n_kv, s.theta, seq.k_pools[li], seq.v_pools[li],
                               self.tables[:n], stream=st)
                paged_gqa_decode_strided(qkv, nqkv, s.n_q, seq.k_pools[li], seq.v_pools[li], self.tables[:n],
                                         self.ctx[:n], attn, self.attn_ws, stream=st)
                int4_gemm(lw["w_o"], lw["s_o"], attn, y=y, ws=self.gemm_ws, stream=st)
                rmsnorm(y, lw["ln_post"], out=xn, resid=r, eps=s.eps, stream=st)
                int4_gemm(lw["w_gu"], lw["s_gu"], xn, y=gu, ws=self.gemm_ws, stream=st)
                silu_mul(gu, out=mlp, stream=st)
                int4_gemm(lw["w_d"], lw["s_d"], mlp, y=y, ws=self.gemm_ws, stream=st)
                gamma = L[li + 1]["ln_in"] if li + 1 < len(L) else g["ln_final"]
                rmsnorm(y, gamma, out=xn, resid=r, eps=s.eps, stream=st)
            # the last position's logits and the first generated token; the sequence continues at position n
            int4_gemv(g["w_lm"], g["s_lm"], xn[n - 1:n], y=self.logits, out_fp32=True, stream=st)
            seq.pos.fill_(n - 1)
            seq.ctx_len.fill_(n)
            argmax_rows(self.logits, seq.token, seq.pos, seq.ctx_len, stream=st)
            seq.history[:n].copy_(self.tokens[:n], non_blocking=True)
            seq.history[n:n + 1].copy_(seq.token, non_blocking=True)
            seq.status.zero_()
        return seq.token
