// The decode step of the 28-layer decoder as one captured CUDA graph.
//
// "How To Build Your Own LLM Runtime From Scratch" ("Technical Details", CUDA
// graph item; second lesson): per-launch driver overhead dominated their eager
// decode (~119 ms/token) and graph replay removed it (~17 ms/token on H100)
// without changing a kernel. Here one token is 5 kernels per layer plus one:
//
//   qkv   : RMSNorm(r) (layer 0: embedding gather) -> INT4 GEMV -> +bias, RoPE, K/V append
//   attn  : paged GQA decode attention (split-K + LSE merge)
//   o     : INT4 GEMV -> r += fp16(y)
//   gu    : RMSNorm(r) -> INT4 GEMV [gate | up] -> SiLU(gate) * up
//   down  : INT4 GEMV -> r += fp16(y)
//   lm    : RMSNorm(r) -> INT4 GEMV (fp32 logits) -> argmax -> token, pos, ctx_len advance
//
// All per-token state (token, position, context length) lives in device
// memory and is advanced by the last kernel, so the same graph is replayed for
// every token with no host work in between. Kernels may be launched with
// programmatic dependent launch; each one waits (griddepcontrol.wait) before
// reading what its predecessors wrote.
#include <cmath>
#include <string>
#include <vector>

#include "attention.cuh"
#include "common.cuh"
#include "gemv.cuh"
#include "persist.cuh"

namespace i4 {
int launch_rope_table(float2 *cs, int max_ctx, int d, double theta, cudaStream_t stream);
extern bool g_l2_prefetch;
bool g_dry_run = false;
bool g_pdl = true;
bool g_l2_prefetch = false;

bool g_persistent = false;
bool g_trace = false;
int g_l2_ahead = 8;
}  // namespace i4

using namespace i4;

struct i4_graph {
    i4_model_desc d;
    i4_model_weights w;
    std::vector<i4_layer_weights> layers;
    i4_seq_state seq;
    std::vector<uint16_t *> kp, vp;
    char *ws = nullptr;
    uint16_t *resid = nullptr, *q = nullptr, *attn = nullptr, *mlp = nullptr;
    float2 *rope_cs = nullptr;
    unsigned long long *best = nullptr;
    unsigned *arrive = nullptr;
    unsigned *sched = nullptr;  // per kernel of the step: the counter pair of a GEMV's dynamic tile schedule
    char *attn_ws = nullptr;
    AttnWs attn_layout = {};
    cudaStream_t cap = nullptr;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    bool pdl = false;
    bool l2pf = false;  // each GEMV prefetches the next GEMV's weights into L2
    int unpack = UNPACK_EXACT;
    int n_kernels = 0;
    // persistent step: one kernel per token over all phases (persist.cu)
    bool persistent = false;
    bool coop = true;
    PersistPlan plan = {};
    PersistArgs pargs = {};
    int n_phases = 0;
    unsigned long long *trace = nullptr;  // [phase][cta][4] timestamps when created with the "trace" option
};

// Phases [begin, end) of the persistent step as one launch.
static int launch_phases(i4_graph *g, cudaStream_t st, int begin, int end) {
    if (g_dry_run) return persist_configure(g->plan);
    PersistArgs a = g->pargs;
    a.phase_begin = begin;
    a.phase_end = end;
    return persist_launch(a, g->plan, st, g->coop);
}

static int enqueue_step(i4_graph *g, cudaStream_t st, int *count, int only = -1) {
    if (g->persistent) {
        if (count) *count = 1;
        return only >= 0 ? launch_phases(g, st, only, only + 1) : launch_phases(g, st, 0, g->n_phases);
    }
    const i4_model_desc &d = g->d;
    const int H = d.hidden, I = d.intermediate, D = d.head_dim;
    const int nqkv = (d.n_q_heads + 2 * d.n_kv_heads) * D;
    const int max_pages = d.max_ctx / d.page_size;
    int n = 0, st_ = 0;
    auto pdl = [&]() { return g->pdl && n > 0 && only < 0; };
    auto skip = [&]() { return only >= 0 && only != n; };
    // L2 prefetch target of a GEMV: the weights and scales of the GEMV that follows it
    auto prefetch = [&](GemvArgs &a, const uint32_t *w, const uint16_t *sc, int rows, int k) {
        if (!g->l2pf || only >= 0) return;
        const size_t cap = 48u << 20;  // a share of L2 the streaming kernels leave alone
        a.pf_a = w;
        a.pf_a_bytes = (size_t)rows * (k / 2) < cap ? (size_t)rows * (k / 2) : cap;
        a.pf_b = sc;
        a.pf_b_bytes = (size_t)rows * (k / 64);
    };
    for (int l = 0; l < d.n_layers; ++l) {
        const i4_layer_weights &L = g->layers[l];
        {  // qkv + RoPE + KV append
            GemvArgs a = {};
            a.w = L.w_qkv;
            a.s = L.s_qkv;
            a.N = nqkv;
            a.K = H;
            a.M = 1;
            a.x = l == 0 ? g->w.embed : g->resid;
            a.gamma = L.ln_in;
            a.eps = d.rms_eps;
            a.token = g->seq.token;
            a.vocab = d.vocab;
            a.resid_out = g->resid;
            a.bias = L.b_qkv;
            a.pos = g->seq.pos;
            a.page_table = g->seq.page_table;
            a.k_pool = g->kp[l];
            a.v_pool = g->vp[l];
            a.q_out = g->q;
            a.rope_cs = g->rope_cs;
            a.n_q = d.n_q_heads;
            a.n_kv = d.n_kv_heads;
            a.page_size = d.page_size;
            a.max_ctx = d.max_ctx;
            a.status = g->seq.status;
            prefetch(a, L.w_o, L.s_o, H, d.n_q_heads * D);
            a.sched = nullptr;  // fixed ranges: measured faster here
            if (!skip() && (st_ = launch_gemv(l == 0 ? PRO_EMBED : PRO_RMSNORM, EPI_ROPE_KV, a, st, pdl(), g->unpack, 0))) return st_;
            ++n;
        }
        {  // attention
            AttnParams p = {};
            p.q = g->q;
            p.k_pool = g->kp[l];
            p.v_pool = g->vp[l];
            p.page_table = g->seq.page_table;
            p.ctx_len = g->seq.ctx_len;
            p.out = g->attn;
            p.B = 1;
            p.Hq = d.n_q_heads;
            p.q_stride = (long long)d.n_q_heads * D;
            p.Hkv = d.n_kv_heads;
            p.page_size = d.page_size;
            p.max_pages = max_pages;
            p.splits = g->attn_layout.splits;
            p.cluster = g->attn_layout.cluster;
            p.scale = (float)(1.0 / std::sqrt((double)D));
            p.ws = g->attn_ws;
            p.counters_off = g->attn_layout.counters_off;
            p.ml_off = g->attn_layout.ml_off;
            p.acc_off = g->attn_layout.acc_off;
            if (!skip() && (st_ = launch_paged_gqa_decode(p, st, pdl()))) return st_;
            ++n;
        }
        {  // o projection + residual
            GemvArgs a = {};
            a.w = L.w_o;
            a.s = L.s_o;
            a.N = H;
            a.K = d.n_q_heads * D;
            a.M = 1;
            a.x = g->attn;
            a.y = g->resid;
            prefetch(a, L.w_gate_up, L.s_gate_up, 2 * I, H);
            a.sched = nullptr;  // fixed ranges: measured faster here
            if (!skip() && (st_ = launch_gemv(PRO_PLAIN, EPI_RESID, a, st, pdl(), g->unpack, 0))) return st_;
            ++n;
        }
        {  // RMSNorm + gate/up + SiLU-mul
            GemvArgs a = {};
            a.w = L.w_gate_up;
            a.s = L.s_gate_up;
            a.N = 2 * I;
            a.K = H;
            a.M = 1;
            a.x = g->resid;
            a.gamma = L.ln_post;
            a.eps = d.rms_eps;
            a.y = g->mlp;
            a.inter = I;
            prefetch(a, L.w_down, L.s_down, H, I);
            a.sched = nullptr;  // fixed ranges: measured faster here
            if (!skip() && (st_ = launch_gemv(PRO_RMSNORM, EPI_SILU, a, st, pdl(), g->unpack, 0))) return st_;
            ++n;
        }
        {  // down projection + residual
            GemvArgs a = {};
            a.w = L.w_down;
            a.s = L.s_down;
            a.N = H;
            a.K = I;
            a.M = 1;
            a.x = g->mlp;
            a.y = g->resid;
            if (l + 1 < d.n_layers)
                prefetch(a, g->layers[l + 1].w_qkv, g->layers[l + 1].s_qkv, nqkv, H);
            else
                prefetch(a, g->w.w_lm, g->w.s_lm, d.vocab, H);
            a.sched = g->sched ? g->sched + 2 * n : nullptr;  // dynamic tiles: measured faster here
            if (!skip() && (st_ = launch_gemv(PRO_PLAIN, EPI_RESID, a, st, pdl(), g->unpack, 0))) return st_;
            ++n;
        }
    }
    {  // final norm + lm_head + argmax + state advance
        GemvArgs a = {};
        a.w = g->w.w_lm;
        a.s = g->w.s_lm;
        a.N = d.vocab;
        a.K = H;
        a.M = 1;
        a.x = g->resid;
        a.gamma = g->w.ln_final;
        a.eps = d.rms_eps;
        a.y = g->seq.logits;
        a.best = g->best;
        a.arrive = g->arrive;
        a.token_io = g->seq.token;
        a.pos_io = g->seq.pos;
        a.ctx_io = g->seq.ctx_len;
        a.prompt = g->seq.prompt;
        a.n_prompt = g->seq.prompt ? g->seq.n_prompt : 0;
        a.history = g->seq.history;
        a.max_ctx = d.max_ctx;
        a.status = g->seq.status;
        a.sched = g->sched ? g->sched + 2 * n : nullptr;  // dynamic tiles: measured faster here
            if (!skip() && (st_ = launch_gemv(PRO_RMSNORM, EPI_ARGMAX, a, st, pdl(), g->unpack, 0))) return st_;
        ++n;
    }
    if (count) *count = n;
    return I4_OK;
}

static int validate(const i4_model_desc *d, const i4_model_weights *w, const i4_seq_state *s) {
    if (!d || !w || !s) return fail(I4_EINVAL, "decode_step_graph_create: null descriptor");
    if (d->n_layers < 1 || d->hidden < 128 || d->intermediate < 128 || d->vocab < 1 || d->n_q_heads < 1 ||
        d->n_kv_heads < 1 || d->max_ctx < 1 || d->page_size < 1)
        return fail(I4_EINVAL, "model: non-positive size");
    if (d->group != 128) return fail(I4_EUNSUPPORTED, "model: group %d (only 128)", d->group);
    if (d->head_dim != 128) return fail(I4_EUNSUPPORTED, "model: head_dim %d (only 128)", d->head_dim);
    if (d->hidden % 128 || d->intermediate % 128 || d->hidden > 32768 || d->intermediate > 32768)
        return fail(I4_EUNSUPPORTED, "model: hidden and intermediate must be multiples of 128 up to 32768");
    if (d->n_q_heads % d->n_kv_heads || d->n_q_heads / d->n_kv_heads > 8)
        return fail(I4_EUNSUPPORTED, "model: n_q_heads / n_kv_heads must be an integer <= 8");
    if ((d->n_q_heads * d->head_dim) % 128 || d->n_q_heads * d->head_dim > 32768)
        return fail(I4_EUNSUPPORTED, "model: n_q_heads * head_dim");
    if (d->page_size < 8 || d->page_size > 128 || (d->page_size & (d->page_size - 1)))
        return fail(I4_EUNSUPPORTED, "model: page_size %d must be a power of two in [8, 128]", d->page_size);
    if (d->max_ctx > 32768) return fail(I4_EUNSUPPORTED, "model: max_ctx above 32768");
    if (d->max_ctx % d->page_size) return fail(I4_EINVAL, "model: max_ctx must be a multiple of page_size");
    if (!(d->rms_eps >= 0.f) || !(d->rope_theta > 0.f)) return fail(I4_EINVAL, "model: eps/theta");
    if (!w->embed || !w->layers || !w->ln_final || !w->w_lm || !w->s_lm) return fail(I4_EINVAL, "weights: null");
    if (!aligned(w->embed, 16) || !aligned(w->ln_final, 16) || !aligned(w->w_lm, 16))
        return fail(I4_EALIGN, "weights: 16-byte alignment");
    for (int l = 0; l < d->n_layers; ++l) {
        const i4_layer_weights &L = w->layers[l];
        if (!L.w_qkv || !L.s_qkv || !L.b_qkv || !L.w_o || !L.s_o || !L.w_gate_up || !L.s_gate_up || !L.w_down ||
            !L.s_down || !L.ln_in || !L.ln_post)
            return fail(I4_EINVAL, "weights: null pointer in layer %d", l);
        if (!aligned(L.w_qkv, 16) || !aligned(L.w_o, 16) || !aligned(L.w_gate_up, 16) || !aligned(L.w_down, 16) ||
            !aligned(L.ln_in, 16) || !aligned(L.ln_post, 16))
            return fail(I4_EALIGN, "weights: 16-byte alignment in layer %d", l);
    }
    if (!s->token || !s->pos || !s->ctx_len || !s->page_table || !s->k_pools || !s->v_pools || !s->logits ||
        !s->status)
        return fail(I4_EINVAL, "seq: null pointer");
    if (s->num_pages < d->max_ctx / d->page_size) return fail(I4_EINVAL, "seq: pools hold fewer pages than max_ctx needs");
    if (s->prompt && (s->n_prompt < 1 || s->n_prompt > d->max_ctx)) return fail(I4_EINVAL, "seq: n_prompt");
    for (int l = 0; l < d->n_layers; ++l)
        if (!s->k_pools[l] || !s->v_pools[l] || !aligned(s->k_pools[l], 16) || !aligned(s->v_pools[l], 16))
            return fail(I4_EINVAL, "seq: pool of layer %d null or misaligned", l);
    return I4_OK;
}

static void release(i4_graph *g) {
    if (!g) return;
    if (g->exec) cudaGraphExecDestroy(g->exec);
    if (g->graph) cudaGraphDestroy(g->graph);
    if (g->cap) cudaStreamDestroy(g->cap);
    if (g->ws) cudaFree(g->ws);
    delete g;
}

static size_t a256(size_t v) { return (v + 255) & ~(size_t)255; }

extern "C" int decode_step_graph_create(const i4_model_desc *desc, const i4_model_weights *weights,
                                        const i4_seq_state *seq, i4_graph **out) {
    if (!out) return fail(I4_EINVAL, "decode_step_graph_create: out is null");
    *out = nullptr;
    int st = validate(desc, weights, seq);
    if (st) return st;
    const int pages = desc->max_ctx / desc->page_size;
    {  // every page id of the table must index the pools
        std::vector<int32_t> tab(pages);
        cudaError_t e = cudaMemcpy(tab.data(), seq->page_table, sizeof(int32_t) * pages, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_check(e, "decode_step_graph_create: reading the page table");
        for (int i = 0; i < pages; ++i)
            if (tab[i] < 0 || tab[i] >= seq->num_pages)
                return fail(I4_EINVAL, "seq: page_table[%d] = %d outside [0, %d)", i, tab[i], seq->num_pages);
    }
    i4_graph *g = new i4_graph();
    g->d = *desc;
    g->w = *weights;
    g->layers.assign(weights->layers, weights->layers + desc->n_layers);
    g->w.layers = g->layers.data();
    g->seq = *seq;
    g->kp.assign(seq->k_pools, seq->k_pools + desc->n_layers);
    g->vp.assign(seq->v_pools, seq->v_pools + desc->n_layers);
    g->seq.k_pools = g->kp.data();
    g->seq.v_pools = g->vp.data();
    g->pdl = g_pdl;
    g->l2pf = g_l2_prefetch;
    g->unpack = g_default_unpack;

    const int H = desc->hidden, D = desc->head_dim;
    g->attn_layout = attn_ws_layout(1, desc->n_q_heads, desc->n_kv_heads, desc->page_size, pages);
    size_t off = 0;
    const size_t o_resid = off; off += a256((size_t)H * 2);
    const size_t o_q = off; off += a256((size_t)desc->n_q_heads * D * 2);
    const size_t o_attn = off; off += a256((size_t)desc->n_q_heads * D * 2);
    const size_t o_mlp = off; off += a256((size_t)desc->intermediate * 2);
    const size_t o_rope = off; off += a256((size_t)desc->max_ctx * (D / 2) * sizeof(float2));
    const size_t o_best = off; off += 256;
    const size_t o_sched = off; off += a256((size_t)(5 * desc->n_layers + 1) * 2 * sizeof(unsigned));
    const size_t o_attn_ws = off; off += a256(g->attn_layout.bytes);
    g->n_phases = 5 * desc->n_layers + 1;
    if (g_persistent) g->plan = persist_plan(*desc);
    g->persistent = g_persistent && g->plan.ok;
    const size_t o_phases = off; off += g->persistent ? a256(sizeof(PPhase) * g->n_phases) : 0;
    const size_t o_pws = off; off += g->persistent ? a256(g->plan.ws_bytes) : 0;
    const size_t trace_bytes = (size_t)g->n_phases * g->plan.grid * 4 * sizeof(unsigned long long);
    const size_t o_trace = off; off += (g->persistent && g_trace) ? a256(trace_bytes) : 0;
    if (cudaMalloc(&g->ws, off) != cudaSuccess) {
        cudaGetLastError();
        release(g);
        return fail(I4_ENOMEM, "decode_step_graph_create: cudaMalloc(%zu) failed", off);
    }
    g->resid = reinterpret_cast<uint16_t *>(g->ws + o_resid);
    g->q = reinterpret_cast<uint16_t *>(g->ws + o_q);
    g->attn = reinterpret_cast<uint16_t *>(g->ws + o_attn);
    g->mlp = reinterpret_cast<uint16_t *>(g->ws + o_mlp);
    g->rope_cs = reinterpret_cast<float2 *>(g->ws + o_rope);
    g->best = reinterpret_cast<unsigned long long *>(g->ws + o_best);
    g->arrive = reinterpret_cast<unsigned *>(g->ws + o_best + 8);
    g->sched = reinterpret_cast<unsigned *>(g->ws + o_sched);
    g->attn_ws = g->ws + o_attn_ws;

    std::vector<PPhase> phases;
    if (g->persistent) {
        phases.resize(g->n_phases);
        persist_fill_phases(*desc, g->plan, phases.data());
        for (int i = 0; i < g->n_phases; ++i) {
            PPhase &p = phases[i];
            const i4_layer_weights *L = p.layer < desc->n_layers ? &g->layers[p.layer] : nullptr;
            switch (p.kind) {
                case PH_QKV: p.w = L->w_qkv; p.s = L->s_qkv; p.gamma = L->ln_in; p.bias = L->b_qkv;
                             p.k_pool = g->kp[p.layer]; p.v_pool = g->vp[p.layer]; break;
                case PH_ATTN: p.k_pool = g->kp[p.layer]; p.v_pool = g->vp[p.layer]; break;
                case PH_O: p.w = L->w_o; p.s = L->s_o; break;
                case PH_GU: p.w = L->w_gate_up; p.s = L->s_gate_up; p.gamma = L->ln_post; break;
                case PH_DOWN: p.w = L->w_down; p.s = L->s_down; break;
                case PH_LM: p.w = g->w.w_lm; p.s = g->w.s_lm; p.gamma = g->w.ln_final; break;
            }
        }
        PersistArgs &a = g->pargs;
        a.phases = reinterpret_cast<const PPhase *>(g->ws + o_phases);
        a.slot_bytes = g->plan.slot_bytes;
        a.stages = g->plan.stages;
        a.l2_ahead = g_l2_ahead;
        a.resid = g->resid;
        a.q = g->q;
        a.attn = g->attn;
        a.mlp = g->mlp;
        a.logits = seq->logits;
        a.embed = weights->embed;
        a.rope_cs = g->rope_cs;
        a.vocab = desc->vocab;
        a.hidden = H;
        a.inter = desc->intermediate;
        a.n_q = desc->n_q_heads;
        a.n_kv = desc->n_kv_heads;
        a.page_size = desc->page_size;
        a.max_pages = pages;
        a.max_ctx = desc->max_ctx;
        a.eps = desc->rms_eps;
        a.attn_scale = (float)(1.0 / std::sqrt((double)D));
        a.token = seq->token;
        a.pos = seq->pos;
        a.ctx_len = seq->ctx_len;
        a.status = seq->status;
        a.history = seq->history;
        a.prompt = seq->prompt;
        a.n_prompt = seq->prompt ? seq->n_prompt : 0;
        a.page_table = seq->page_table;
        char *pw = g->ws + o_pws;
        a.bar_count = reinterpret_cast<unsigned long long *>(pw);
        a.best = reinterpret_cast<unsigned long long *>(pw + 8);
        a.arrive = reinterpret_cast<unsigned *>(pw + 16);
        a.attn_count = reinterpret_cast<unsigned *>(pw + 256);
        a.attn_max_splits = g->plan.attn_max_splits;
        const size_t cells = (size_t)desc->n_kv_heads * g->plan.attn_max_splits * 8;
        a.attn_ml = reinterpret_cast<float2 *>(pw + 512);
        a.attn_acc = reinterpret_cast<float *>(pw + 512 + a256(cells * sizeof(float2)));
        if (g_trace) g->trace = a.trace = reinterpret_cast<unsigned long long *>(g->ws + o_trace);
    }
    if ((st = cuda_check(cudaStreamCreateWithFlags(&g->cap, cudaStreamNonBlocking), "stream create")) ||
        (st = cuda_check(cudaMemsetAsync(g->ws, 0, off, g->cap), "workspace clear")) ||
        (st = launch_rope_table(g->rope_cs, desc->max_ctx, D, (double)desc->rope_theta, g->cap)) ||
        (g->persistent &&
         (st = cuda_check(cudaMemcpyAsync(g->ws + o_phases, phases.data(), sizeof(PPhase) * g->n_phases,
                                          cudaMemcpyHostToDevice, g->cap), "phase table upload"))) ||
        (st = cuda_check(cudaStreamSynchronize(g->cap), "workspace init"))) {
        release(g);
        return st;
    }
    // configure every kernel variant (shared-memory limits, occupancy) outside the capture; a persistent
    // step the device cannot hold (one CTA per SM) falls back to one kernel per phase
    g_dry_run = true;
    st = enqueue_step(g, g->cap, &g->n_kernels);
    if (st && g->persistent) {
        g->persistent = false;
        st = enqueue_step(g, g->cap, &g->n_kernels);
    }
    g_dry_run = false;
    if (st) {
        release(g);
        return st;
    }
    if ((st = cuda_check(cudaStreamBeginCapture(g->cap, cudaStreamCaptureModeThreadLocal), "begin capture"))) {
        release(g);
        return st;
    }
    st = enqueue_step(g, g->cap, nullptr);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(g->cap, &graph);
    g->graph = graph;
    if (st || (st = cuda_check(e, "end capture")) ||
        (st = cuda_check(cudaGraphInstantiate(&g->exec, g->graph, 0), "graph instantiate"))) {
        release(g);
        return st;
    }
    *out = g;
    return I4_OK;
}

extern "C" int decode_step_graph_replay(i4_graph *g, void *stream) {
    if (!g || !g->exec) return fail(I4_EINVAL, "decode_step_graph_replay: no graph");
    return cuda_check(cudaGraphLaunch(g->exec, (cudaStream_t)stream), "graph launch");
}

extern "C" int decode_step_eager(i4_graph *g, void *stream) {
    if (!g) return fail(I4_EINVAL, "decode_step_eager: no graph");
    return enqueue_step(g, (cudaStream_t)stream, nullptr);
}

extern "C" int decode_step_kernel_count(const i4_graph *g) { return g ? g->n_kernels : 0; }

extern "C" int decode_step_phase_count(const i4_graph *g) { return g ? g->n_phases : 0; }

extern "C" int decode_step_launch_kernel(i4_graph *g, int index, void *stream) {
    if (!g) return fail(I4_EINVAL, "decode_step_launch_kernel: no graph");
    if (index < 0 || index >= g->n_phases)
        return fail(I4_EINVAL, "decode_step_launch_kernel: index %d outside [0, %d)", index, g->n_phases);
    return enqueue_step(g, (cudaStream_t)stream, nullptr, index);
}

extern "C" int decode_step_is_persistent(const i4_graph *g) { return g && g->persistent ? 1 : 0; }

extern "C" int decode_step_trace(i4_graph *g, unsigned long long *host_out, size_t n) {
    if (!g || !host_out) return fail(I4_EINVAL, "decode_step_trace: null argument");
    if (!g->trace) return fail(I4_EINVAL, "decode_step_trace: graph was not created with the \"trace\" option");
    const size_t need = (size_t)g->n_phases * g->plan.grid * 4;
    if (n < need) return fail(I4_EINVAL, "decode_step_trace: %zu entries needed", need);
    return cuda_check(cudaMemcpy(host_out, g->trace, need * sizeof(unsigned long long), cudaMemcpyDeviceToHost),
                      "decode_step_trace");
}

extern "C" int decode_step_buffer_copy(i4_graph *g, int which, void *dev, size_t bytes, int dir, void *stream) {
    if (!g || !dev) return fail(I4_EINVAL, "decode_step_buffer_copy: null argument");
    if (dir != 0 && dir != 1) return fail(I4_EINVAL, "decode_step_buffer_copy: dir must be 0 (out) or 1 (in)");
    uint16_t *buf = nullptr;
    size_t n = 0;
    switch (which) {
        case I4_BUF_RESID: buf = g->resid; n = (size_t)g->d.hidden * 2; break;
        case I4_BUF_Q: buf = g->q; n = (size_t)g->d.n_q_heads * g->d.head_dim * 2; break;
        case I4_BUF_ATTN: buf = g->attn; n = (size_t)g->d.n_q_heads * g->d.head_dim * 2; break;
        case I4_BUF_MLP: buf = g->mlp; n = (size_t)g->d.intermediate * 2; break;
        default: return fail(I4_EINVAL, "decode_step_buffer_copy: unknown buffer %d", which);
    }
    if (bytes != n) return fail(I4_EINVAL, "decode_step_buffer_copy: buffer %d holds %zu bytes, got %zu", which, n, bytes);
    void *dst = dir == 0 ? dev : (void *)buf;
    const void *src = dir == 0 ? (const void *)buf : dev;
    return cuda_check(cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToDevice, (cudaStream_t)stream),
                      "decode_step_buffer_copy");
}

extern "C" int decode_step_graph_destroy(i4_graph *g) {
    if (!g) return fail(I4_EINVAL, "decode_step_graph_destroy: null");
    release(g);
    return I4_OK;
}

// Library options: "pdl" (programmatic dependent launch inside the decode step,
// 0/1) and "unpack" (GEMV unpack variant, 0 exact / 1 subnormal). They apply to
// graphs created afterwards and to int4_gemv calls.
extern "C" int i4_set_option(const char *name, int value) {
    if (!name) return fail(I4_EINVAL, "i4_set_option: null name");
    const std::string n(name);
    if (n == "pdl") {
        g_pdl = value != 0;
        return I4_OK;
    }
    if (n == "unpack") {
        if (value < UNPACK_EXACT || value > UNPACK_AUTO) return fail(I4_EINVAL, "unpack must be 0, 1, 2, 3 or 4");
        g_default_unpack = value;
        return I4_OK;
    }
    if (n == "stream") {
        set_stream_options(value, 0);
        return I4_OK;
    }
    if (n == "l2_ahead") {
        if (value < 0 || value > 64) return fail(I4_EINVAL, "l2_ahead must be in [0, 64]");
        g_l2_ahead = value;
        return I4_OK;
    }
    if (n == "trace") {
        g_trace = value != 0;
        return I4_OK;
    }
    if (n == "persistent") {
        g_persistent = value != 0;
        return I4_OK;
    }
    if (n == "l2_prefetch") {
        g_l2_prefetch = value != 0;
        return I4_OK;
    }
    if (n == "test_stall") {
        set_test_stall(value != 0);
        return I4_OK;
    }
    if (n == "gemv_prex") {
        if (value < 0 || value > 8) return fail(I4_EINVAL, "gemv_prex must be in [0, 8]");
        set_stream_prex(value);
        return I4_OK;
    }
    if (n == "gemv_ctas_per_sm") {
        if (value < 1 || value > 2) return fail(I4_EINVAL, "gemv_ctas_per_sm must be 1 or 2");
        set_stream_ctas_per_sm(value);
        return I4_OK;
    }
    if (n == "stream_smem_kb") {
        if (value < 32 || value > 227) return fail(I4_EINVAL, "stream_smem_kb must be in [32, 227]");
        set_stream_options(-1, value);
        return I4_OK;
    }
    return fail(I4_EINVAL, "i4_set_option: unknown option '%s'", name);
}
