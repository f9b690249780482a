// Internal interface of the persistent decode step (persist.cu): one launch
// runs a range of the token's phases (5 per layer + lm_head) on one CTA per SM.
#pragma once

#include "common.cuh"

namespace i4 {

enum PhaseKind : int { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_GU = 3, PH_DOWN = 4, PH_LM = 5 };

// One phase of the token. GEMV phases stream `tiles` tiles of R rows (N rows
// of K weights in all); tile t goes to CTA (first + t) % grid, so consecutive
// phases continue the round robin and every SM streams the same bytes.
struct PPhase {
    int kind, layer;
    int N, K, R, tiles, first;
    const uint32_t *w;
    const uint16_t *s;
    const uint16_t *gamma;  // RMSNorm weight of the prologue (QKV, GU, LM)
    const uint16_t *bias;   // qkv bias (QKV)
    uint16_t *k_pool, *v_pool;  // the layer's pools (QKV appends, ATTN reads)
};

struct PersistArgs {
    const PPhase *phases;
    int phase_begin, phase_end;
    int slot_bytes, stages;
    int l2_ahead;  // tiles of its own stream each CTA prefetches into L2 ahead of the ring
    // activations (written and read inside the launch)
    uint16_t *resid, *q, *attn, *mlp;
    float *logits;
    // model constants
    const uint16_t *embed;
    const float2 *rope_cs;  // [max_ctx][64] (cos, sin)
    int vocab, hidden, inter, n_q, n_kv, page_size, max_pages, max_ctx;
    float eps, attn_scale;
    // sequence state
    int32_t *token, *pos, *ctx_len, *status, *history;
    const int32_t *prompt;
    int n_prompt;
    const int32_t *page_table;
    // synchronisation and scratch (zeroed once at creation; every launch leaves them reusable)
    unsigned long long *bar_count;  // grid barrier arrivals (only grows)
    unsigned long long *best;
    unsigned *arrive;
    unsigned *attn_count;   // [n_kv] arrivals of the attention splits
    float2 *attn_ml;        // [n_kv][max_splits][8] (max, sum) per split and head
    float *attn_acc;        // [n_kv][max_splits][8][128] unnormalised outputs
    int attn_max_splits;
    // optional timestamps (globaltimer ns), [phase - phase_begin][cta][4]: consumers start the phase (after
    // the grid barrier), x staged, phase work done; the producer issues the phase's first tile
    unsigned long long *trace;
};

struct PersistPlan {
    bool ok;
    int grid, slot_bytes, stages, smem, xarea_bytes, attn_max_splits;
    size_t ws_bytes;  // sync words + attention scratch
};

// Geometry of the persistent step for a model (ok = false when a shape is outside it).
PersistPlan persist_plan(const i4_model_desc &d);
// Tiles, rows per tile and round-robin offsets of every phase; `phases` has 5 * n_layers + 1 entries.
void persist_fill_phases(const i4_model_desc &d, const PersistPlan &plan, PPhase *phases);
int persist_configure(const PersistPlan &plan);
int persist_launch(const PersistArgs &a, const PersistPlan &plan, cudaStream_t stream, bool cooperative);
int read_persist_error(int reset);

}  // namespace i4
