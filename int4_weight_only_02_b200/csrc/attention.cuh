// Internal interface of the paged decode attention kernel (see attention.cu).
#pragma once

#include "common.cuh"

namespace i4 {

struct AttnParams {
    const uint16_t *q, *k_pool, *v_pool;
    const int32_t *page_table, *ctx_len;
    uint16_t *out;
    int B, Hq, Hkv, page_size, max_pages;
    long long q_stride;   // elements between the q rows of consecutive sequences (Hq * 128 when packed)
    int splits, cluster;  // grid x (a multiple of cluster) and CTAs per cluster along x
    float scale;
    char *ws;
    size_t counters_off, ml_off, acc_off;
};

struct AttnWs {
    int splits, cluster;
    size_t counters_off, ml_off, acc_off, bytes;
};

AttnWs attn_ws_layout(int B, int Hq, int Hkv, int page_size, int max_pages);
int launch_paged_gqa_decode(const AttnParams &p, cudaStream_t stream, bool pdl);

}  // namespace i4
