// Paged grouped-query decode attention: split-K over the context with a
// log-sum-exp merge, on tensor cores.
//
// "How To Build Your Own LLM Runtime From Scratch" ("Technical Details": paged
// KV cache and attention; lessons: a __syncthreads() inside a
// warp-specialised branch corrupted the softmax at KV-page tails). The H100
// design there was warp-specialised with TMA. At batch 1 one kv head of one
// layer holds well under 1 MB of K/V at the contexts decode runs at, so this
// kernel is bound by latency, not bandwidth, and its design keeps the chain
// from launch to output short:
//
//  * Work. Grid (S, Hkv, B) in clusters of CL CTAs along x. The context of
//    sequence b is cut into tiles of 64 tokens and CTA s takes tiles
//    [s*tpc, (s+1)*tpc). tpc comes from ctx_len[b] on the device, so a captured
//    graph stays valid as the context grows; contexts of up to 8*CL tiles stay
//    inside one cluster.
//  * Data. Every warp stages its own 16 tokens of each tile: 16-byte cp.async
//    copies from the pool pages into a per-warp two-stage shared-memory ring,
//    each 64-dim half of a row at 128 bytes with its 16-byte chunks XOR-swizzled
//    by row, so the ldmatrix reads below are free of bank conflicts. Page-table
//    entries are read 32 tiles ahead. A page below the one holding position
//    ctx-1 was written by an earlier step, so its copies are issued before the
//    programmatic dependency wait; the current page's after it.
//  * Math. Each of the 4 warps takes 16 tokens of a tile.
//    S = Q K^T on mma.m16n8k16 with the G <= 8 query heads that share the kv
//    head as the M rows (rows G..15 are zero), so each K row is read once for
//    all G heads. P = 2^(S - m) rounded to fp16 then feeds O^T = V^T P^T
//    (M = 16 dims, N = 8 heads, K = 16 tokens) directly from the S
//    accumulators. Online softmax per warp, fp32 accumulation throughout.
//  * Merge. The 4 warps merge in shared memory; the CTAs of a cluster push
//    their (m, l, o) into the rank-0 CTA's shared memory (distributed shared
//    memory), which merges them. With one active cluster that CTA writes the
//    output; otherwise cluster leaders write partials to the workspace and the
//    last to arrive merges them:
//      M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
#include <mutex>

#include "async.cuh"
#include "attention.cuh"
#include "common.cuh"
#include "mma.cuh"

namespace i4 {

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;                        // query heads per kv head (MMA rows used)
constexpr int kWarpTokens = 16;                     // tokens of a tile per warp
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTileTokens = kWarps * kWarpTokens;   // 64
constexpr int kStages = 2;                          // ring depth of every warp
constexpr int kMaxCluster = 8;
constexpr int kOneClusterTiles = 8;  // contexts up to kMaxCluster * this many tiles stay in one cluster
constexpr int kMaxSplits = 256;
constexpr int kMaxCtx = 32768;
constexpr int kMaxPageSize = 128;
constexpr float kLog2e = 1.4426950408889634f;

// Dynamic shared memory (128-byte aligned base):
//   ring  [warp][stage] {K dims 0-63, K dims 64-127, V dims 0-63, V dims 64-127}, each [16 tokens][128 B]
//   recv  [kMaxCluster][kHeadDim][kMaxGroup] fp32 o and [kMaxCluster][kMaxGroup] (m, l) pushed by the cluster
// The warp partials reuse the ring once every tile is consumed; the cross-cluster merge reuses recv.
constexpr unsigned kRegionBytes = kWarpTokens * 128;
constexpr unsigned kWarpStageBytes = 4 * kRegionBytes;
constexpr unsigned kRingBytes = kWarps * kStages * kWarpStageBytes;
constexpr unsigned kRecvOff = kRingBytes;
constexpr unsigned kRecvBytes = kMaxCluster * kHeadDim * kMaxGroup * 4;
constexpr unsigned kRecvMlOff = kRecvOff + kRecvBytes;
constexpr unsigned kDynSmem = 128 + kRecvMlOff + kMaxCluster * kMaxGroup * 8;
constexpr int kCtasPerSm = (228 * 1024) / (kDynSmem + 2048);  // with the static part and the per-CTA reserve
static_assert(kWarps * kHeadDim * kMaxGroup * 4 <= kRingBytes, "warp partials must fit in the ring");
static_assert(2 * kMaxGroup * kMaxSplits * 4 <= kRecvBytes, "merge weights must fit in the receive buffer");

__device__ int g_attn_error = 0;

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// How the n_tiles tiles of one sequence are spread over the `splits` CTAs of a (b, g) row.
struct Split {
    int tpc, active, clusters;  // tiles per CTA, CTAs with tiles, clusters with such CTAs
};
__host__ __device__ inline Split split_work(int n_tiles, int splits, int cl) {
    Split w;
    w.tpc = n_tiles <= cl * kOneClusterTiles ? (n_tiles + cl - 1) / cl : (n_tiles + splits - 1) / splits;
    if (w.tpc < 1) w.tpc = 1;
    w.active = (n_tiles + w.tpc - 1) / w.tpc;
    w.clusters = (w.active + cl - 1) / cl;
    return w;
}

AttnWs attn_ws_layout(int B, int Hq, int Hkv, int page_size, int max_pages) {
    // one wave of CTAs over the SMs, whole clusters, no more CTAs than tiles
    const int max_tiles = (int)(((long long)max_pages * page_size + kTileTokens - 1) / kTileTokens);
    const int rows = B * Hkv;
    int s = (kCtasPerSm * kNumSMs + rows - 1) / rows;
    s = s < max_tiles ? s : max_tiles;
    s = s < kMaxSplits ? s : kMaxSplits;
    s = s < 1 ? 1 : s;
    const int cl = s < kMaxCluster ? s : kMaxCluster;
    AttnWs L;
    L.splits = s / cl * cl;
    L.cluster = cl;
    const size_t G = (size_t)(Hq / Hkv);
    const size_t cells = (size_t)rows * (L.splits / cl) * G;  // one partial per cluster and head
    L.counters_off = 0;
    L.ml_off = align256((size_t)rows * sizeof(unsigned));
    L.acc_off = L.ml_off + align256(cells * sizeof(float2));
    L.bytes = L.acc_off + align256(cells * kHeadDim * sizeof(float));
    return L;
}

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive_release() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_f4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_f2(uint32_t addr, float a, float b) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
// oh[h] = sum_k cw[k][h] * part[k][d][h] over n <= N partials laid out [k][dim][head]
template <int N>
__device__ __forceinline__ void combine(float (&oh)[kMaxGroup], const float *part, const float (*cw)[kMaxGroup],
                                        int d, int n = N) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) oh[h] = 0.f;
#pragma unroll
    for (int k = 0; k < N; ++k) {
        if (k < n) {
            const float4 lo = *reinterpret_cast<const float4 *>(part + ((size_t)k * kHeadDim + d) * kMaxGroup);
            const float4 hi = *reinterpret_cast<const float4 *>(part + ((size_t)k * kHeadDim + d) * kMaxGroup + 4);
            const float4 wl = *reinterpret_cast<const float4 *>(&cw[k][0]);
            const float4 wh = *reinterpret_cast<const float4 *>(&cw[k][4]);
            oh[0] = fmaf(wl.x, lo.x, oh[0]);
            oh[1] = fmaf(wl.y, lo.y, oh[1]);
            oh[2] = fmaf(wl.z, lo.z, oh[2]);
            oh[3] = fmaf(wl.w, lo.w, oh[3]);
            oh[4] = fmaf(wh.x, hi.x, oh[4]);
            oh[5] = fmaf(wh.y, hi.y, oh[5]);
            oh[6] = fmaf(wh.z, hi.z, oh[6]);
            oh[7] = fmaf(wh.w, hi.w, oh[7]);
        }
    }
}

// ------------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kThreads, kCtasPerSm) paged_gqa_decode_kernel(const AttnParams p) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ float2 wml[kMaxCluster][kMaxGroup];  // (m, l) of the 4 warps, later of the cluster's CTAs
    __shared__ __align__(16) float cw[kMaxCluster][kMaxGroup];  // merge weights
    __shared__ float cM[kMaxGroup], cL[kMaxGroup];
    __shared__ int is_last;

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.Hq / p.Hkv, P = p.page_size, CL = p.cluster;
    const int pshift = __ffs(P) - 1;  // page_size is a power of two: t / P == t >> pshift
    const int max_ctx = p.max_pages * P;
    int ctx = p.ctx_len[b];  // advanced by an earlier step's last kernel, never by this kernel's predecessor
    ctx = ctx < 1 ? 1 : (ctx > max_ctx ? max_ctx : ctx);
    const int n_tiles = (ctx + kTileTokens - 1) / kTileTokens;
    const Split w = split_work(n_tiles, p.splits, CL);
    if (s / CL >= w.clusters) return;  // the whole cluster leaves before any barrier
    cluster_arrive_relaxed();          // "started": awaited before the first store into the leader
    const uint32_t rank = cluster_rank();
    const int tile0 = s * w.tpc;
    int n_my = n_tiles - tile0;
    n_my = n_my < 0 ? 0 : (n_my > w.tpc ? w.tpc : n_my);

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 127u) & ~127u;
    unsigned char *gbase = smem_raw + (base - raw);
    const uint32_t ring = base + warp * kStages * kWarpStageBytes;  // this warp's stages

    // ---------------- staging: lane copies 16-byte chunk (lane & 15) of rows (lane >> 4) + 2j, j < 8
    const int last_page = (ctx - 1) >> pshift;
    const int32_t *table = p.page_table + (size_t)b * p.max_pages;
    const size_t head_rows = (size_t)g * P;  // row offset of kv head g inside a page
    auto slab = [&](int i) { return (tile0 + i) * kTileTokens + warp * kWarpTokens; };  // first token of tile i
    // page-table entries of the pages holding the first and the last token of the warp's 16, 32 tiles per batch
    auto fetch = [&](int batch, int &ea, int &eb) {
        const int i = batch * 32 + lane;
        const int t = slab(i);
        ea = eb = 0;
        if (i < n_my && t < ctx) {
            const int tl = t + kWarpTokens - 1 < ctx ? t + kWarpTokens - 1 : ctx - 1;
            ea = table[t >> pshift];
            eb = table[tl >> pshift];
        }
    };
    int cur_batch = 0, ca, cb, na, nb;
    fetch(0, ca, cb);
    fetch(1, na, nb);
    const int chunk = lane & 15, row_lo = lane >> 4;
    const uint32_t chunk_off = (chunk >> 3) * kRegionBytes;  // K: dims 0-63 or 64-127
    bool waited = false;
    auto issue = [&](int i) {  // tile i into stage i % kStages (warp-uniform control flow)
        const int batch = i >> 5;
        while (cur_batch < batch) {
            ca = na;
            cb = nb;
            fetch(++cur_batch + 1, na, nb);
        }
        const int ea = __shfl_sync(0xffffffffu, ca, i & 31), eb = __shfl_sync(0xffffffffu, cb, i & 31);
        const int t = slab(i);
        if (!waited && t < ctx) {
            const int tl = t + kWarpTokens - 1 < ctx ? t + kWarpTokens - 1 : ctx - 1;
            if ((tl >> pshift) == last_page) {
                grid_dep_wait();  // the current page's new row comes from the preceding kernel
                waited = true;
            }
        }
        const uint32_t st = ring + (i % kStages) * kWarpStageBytes + chunk_off;
        const int pa = t >> pshift;
        // element offsets of this kv head's rows in the two pages the warp's 16 tokens can touch
        const size_t base_a = (((size_t)ea * p.Hkv) * P + head_rows) * kHeadDim + chunk * 8;
        const size_t base_b = (((size_t)eb * p.Hkv) * P + head_rows) * kHeadDim + chunk * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = row_lo + 2 * j, tok = t + r;
            if (tok < ctx) {
                const size_t off = ((tok >> pshift) == pa ? base_a : base_b) + (size_t)(tok & (P - 1)) * kHeadDim;
                const uint32_t dst = st + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
                cp_async16(dst, p.k_pool + off);
                cp_async16(dst + 2 * kRegionBytes, p.v_pool + off);
            }
        }
    };
#pragma unroll 1
    for (int i = 0; i < kStages; ++i) {
        if (i < n_my) issue(i);
        cp_async_commit();
    }
    if (!waited) grid_dep_wait();  // q comes from the preceding kernel
    grid_dep_launch();

    const int gq = lane >> 2, tig = lane & 3;  // MMA group (row) and thread-in-group
    uint32_t qa[8][2];
    {
        const uint32_t *qrow =
            reinterpret_cast<const uint32_t *>(p.q + (size_t)b * p.q_stride + (size_t)(g * G + gq) * kHeadDim);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qa[kk][0] = gq < G ? qrow[8 * kk + tig] : 0u;
            qa[kk][1] = gq < G ? qrow[8 * kk + 4 + tig] : 0u;
        }
    }
    const float qscale = p.scale * kLog2e;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const int r8 = lane & 7, mi = lane >> 3;  // ldmatrix: row within an 8x8 matrix, matrix index
#pragma unroll 1
    for (int i = 0; i < n_my; ++i) {
        cp_async_wait<kStages - 1>();  // this lane's copies of tile i have landed
        __syncwarp();                  // and every other lane's
        const int valid = ctx - slab(i);  // tokens of this warp's 16 that exist
        if (valid > 0) {
            const uint32_t kb = ring + (i % kStages) * kWarpStageBytes, vb = kb + 2 * kRegionBytes;
            // S[h][t] = q_h . k_t over 8 k-steps of 16 dims; s0: tokens 0-7, s1: tokens 8-15
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
                const int c = 4 * k2 + mi;  // 16-byte chunk of the 256-byte row
                const uint32_t off = (c >> 3) * kRegionBytes + (((c & 7) ^ r8) << 4);
                uint32_t b0, b1, b2, b3, e0, e1, e2, e3;
                ldsm_x4(kb + off + r8 * 128, b0, b1, b2, b3);
                ldsm_x4(kb + off + (r8 + 8) * 128, e0, e1, e2, e3);
                mma16816(s0, qa[2 * k2][0], 0u, qa[2 * k2][1], 0u, b0, b1);
                mma16816(s1, qa[2 * k2][0], 0u, qa[2 * k2][1], 0u, e0, e1);
                mma16816(s0, qa[2 * k2 + 1][0], 0u, qa[2 * k2 + 1][1], 0u, b2, b3);
                mma16816(s1, qa[2 * k2 + 1][0], 0u, qa[2 * k2 + 1][1], 0u, e2, e3);
            }
            // this lane: head gq, tokens j, j+1, j+8, j+9 of the warp's 16
            const int j = 2 * tig;
            float sv[4] = {s0[0] * qscale, s0[1] * qscale, s1[0] * qscale, s1[1] * qscale};
            uint32_t mk01 = 0xffffffffu, mk89 = 0xffffffffu;
            if (valid < kWarpTokens) {
                sv[0] = j < valid ? sv[0] : -INFINITY;
                sv[1] = j + 1 < valid ? sv[1] : -INFINITY;
                sv[2] = j + 8 < valid ? sv[2] : -INFINITY;
                sv[3] = j + 9 < valid ? sv[3] : -INFINITY;
                mk01 = (j < valid ? 0x0000ffffu : 0u) | (j + 1 < valid ? 0xffff0000u : 0u);
                mk89 = (j + 8 < valid ? 0x0000ffffu : 0u) | (j + 9 < valid ? 0xffff0000u : 0u);
            }
            float mc = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, 1));
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, 2));
            const float m_new = fmaxf(m_run, mc);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = exp2f(m_run - m_use);
            const __half2 p01 = __floats2half2_rn(exp2f(sv[0] - m_use), exp2f(sv[1] - m_use));
            const __half2 p89 = __floats2half2_rn(exp2f(sv[2] - m_use), exp2f(sv[3] - m_use));
            const float2 f01 = __half22float2(p01), f89 = __half22float2(p89);
            l_run = fmaf(l_run, alpha, (f01.x + f01.y) + (f89.x + f89.y));
            m_run = m_new;
            // O^T columns of this lane are heads 2*tig and 2*tig+1, whose rescale factors live in lanes 8*tig and 8*tig+4
            const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * tig);
            const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
            const uint32_t pb0 = h2_bits(p01), pb1 = h2_bits(p89);
#pragma unroll
            for (int im = 0; im < 8; ++im) {
                // V^T tile: dims 16*im.., the warp's 16 tokens; matrices (t0-7, d lo), (t0-7, d hi), (t8-15, d lo), (t8-15, d hi)
                const int c = 2 * im + (mi & 1);
                const int row = (mi >> 1) * 8 + r8;
                uint32_t a0, a1, a2, a3;
                ldsm_x4_trans(vb + (c >> 3) * kRegionBytes + row * 128 + (((c & 7) ^ r8) << 4), a0, a1, a2, a3);
                o[im][0] *= a_lo;
                o[im][1] *= a_hi;
                o[im][2] *= a_lo;
                o[im][3] *= a_hi;
                mma16816(o[im], a0 & mk01, a1 & mk01, a2 & mk89, a3 & mk89, pb0, pb1);
            }
        }
        __syncwarp();  // every lane is done with this stage before it is refilled
        if (i + kStages < n_my) issue(i + kStages);
        cp_async_commit();
    }
    cp_async_wait<0>();
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

    // ---------------- merge the 4 warps (the ring becomes the partial buffer)
    const int d = tid;  // the output dim this thread merges
    float *wo = reinterpret_cast<float *>(gbase);  // [warp][dim][head]
    __syncthreads();
    if (tig == 0) wml[warp][gq] = make_float2(m_run, l_run);
#pragma unroll
    for (int im = 0; im < 8; ++im) {
        float *r = wo + ((size_t)warp * kHeadDim + 16 * im + gq) * kMaxGroup + 2 * tig;
        *reinterpret_cast<float2 *>(r) = make_float2(o[im][0], o[im][1]);
        *reinterpret_cast<float2 *>(r + 8 * kMaxGroup) = make_float2(o[im][2], o[im][3]);
    }
    __syncthreads();
    if (tid < 32) {  // lane 4 h + k: weight of warp k's partial of head h
        const int h = tid >> 2, k = tid & 3;
        const float2 v = wml[k][h];
        float M = fmaxf(v.x, __shfl_xor_sync(0xffffffffu, v.x, 1));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
        const float wt = merge_weight(v.x, M);
        float L = wt * v.y;
        L += __shfl_xor_sync(0xffffffffu, L, 1);
        L += __shfl_xor_sync(0xffffffffu, L, 2);
        cw[k][h] = wt;
        if (k == 0) {
            cM[h] = M;
            cL[h] = L;
        }
    }
    __syncthreads();
    float oh[kMaxGroup];
    combine<kWarps>(oh, wo, cw, d);

    // ---------------- push this CTA's partial into the cluster leader (rank 0)
    cluster_wait();  // every CTA of the cluster has started
    {
        const uint32_t dst = map_to_rank(base + kRecvOff + ((rank * kHeadDim + d) * kMaxGroup) * 4, 0);
        st_cluster_f4(dst, oh[0], oh[1], oh[2], oh[3]);
        st_cluster_f4(dst + 16, oh[4], oh[5], oh[6], oh[7]);
        if (d < kMaxGroup) st_cluster_f2(map_to_rank(base + kRecvMlOff + (rank * kMaxGroup + d) * 8, 0), cM[d], cL[d]);
    }
    cluster_arrive_release();
    cluster_wait();
    if (rank != 0) return;

    // ---------------- leader: merge the cluster's CTAs
    const float *co = reinterpret_cast<const float *>(gbase + kRecvOff);
    const float2 *cml = reinterpret_cast<const float2 *>(gbase + kRecvMlOff);
    if (tid < 64) {  // lane 8 h + k: normalised weight of rank k's partial of head h
        const int h = tid >> 3, k = tid & 7;
        const float2 v = k < CL ? cml[k * kMaxGroup + h] : make_float2(-INFINITY, 0.f);
        float M = fmaxf(v.x, __shfl_xor_sync(0xffffffffu, v.x, 1));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 4));
        const float wt = merge_weight(v.x, M);
        float L = wt * v.y;
        L += __shfl_xor_sync(0xffffffffu, L, 1);
        L += __shfl_xor_sync(0xffffffffu, L, 2);
        L += __shfl_xor_sync(0xffffffffu, L, 4);
        cw[k][h] = wt * (1.0f / L);
        if (k == 0) {
            cM[h] = M;
            cL[h] = L;
        }
    }
    __syncthreads();
    combine<kMaxCluster>(oh, co, cw, d, CL);  // the cluster's output, normalised
    uint16_t *out = p.out + ((size_t)b * p.Hq + g * G) * kHeadDim + d;
    if (w.clusters == 1) {
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
            if (h < G) out[(size_t)h * kHeadDim] = float_to_half_bits(oh[h]);
        return;
    }

    // ---------------- several clusters: partials through the workspace, the last leader merges
    const int cid = s / CL, n_cl = w.clusters;
    const int max_cl = p.splits / CL;
    const size_t cell0 = ((size_t)b * p.Hkv + g) * max_cl * G;  // (b, g, cluster 0, head 0)
    float2 *ml = reinterpret_cast<float2 *>(p.ws + p.ml_off);
    float *pacc = reinterpret_cast<float *>(p.ws + p.acc_off);
    unsigned *counter = reinterpret_cast<unsigned *>(p.ws + p.counters_off) + (size_t)b * p.Hkv + g;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
        if (h < G) pacc[(cell0 + (size_t)cid * G + h) * kHeadDim + d] = oh[h];
    if (d < G) ml[cell0 + (size_t)cid * G + d] = make_float2(cM[d], cL[d]);
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(counter, 1u) == (unsigned)n_cl - 1u;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    float *coef = reinterpret_cast<float *>(gbase + kRecvOff);  // [kMaxGroup][kMaxSplits]
    float *lsum = coef + kMaxGroup * kMaxSplits;
    for (int i = tid; i < n_cl * G; i += kThreads) {
        const float2 v = __ldcg(&ml[cell0 + i]);
        coef[(i % G) * kMaxSplits + i / G] = v.x;
        lsum[(i % G) * kMaxSplits + i / G] = v.y;
    }
    __syncthreads();
    for (int h = warp; h < G; h += kWarps) {  // warp w: heads w, w+4
        float *ch = coef + h * kMaxSplits;
        const float *lh = lsum + h * kMaxSplits;
        float M = -INFINITY;
        for (int k = lane; k < n_cl; k += 32) M = fmaxf(M, ch[k]);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
        float L = 0.f;
        for (int k = lane; k < n_cl; k += 32) {  // the partials are normalised: weight 2^(m_k - M) l_k
            const float wt = merge_weight(ch[k], M) * lh[k];
            ch[k] = wt;
            L += wt;
        }
        L = warp_sum(L);
        const float inv = 1.0f / L;
        __syncwarp();
        for (int k = lane; k < n_cl; k += 32) ch[k] *= inv;
    }
    __syncthreads();
    // four clusters' partials of every head per pass, all loads issued before the first use
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) oh[h] = 0.f;
    for (int k0 = 0; k0 < n_cl; k0 += 4) {
        float v[kMaxGroup][4];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[h][u] = (h < G && k0 + u < n_cl) ? __ldcg(&pacc[(cell0 + (size_t)(k0 + u) * G + h) * kHeadDim + d])
                                                   : 0.f;
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (h < G && k0 + u < n_cl) oh[h] = fmaf(coef[h * kMaxSplits + k0 + u], v[h][u], oh[h]);
    }
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
        if (h < G) out[(size_t)h * kHeadDim] = float_to_half_bits(oh[h]);
    if (tid == 0) *counter = 0u;  // ready for the next call
}

// ------------------------------------------------------------------ host side

int launch_paged_gqa_decode(const AttnParams &p, cudaStream_t stream, bool pdl) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(paged_gqa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
    });
    if (attr_err != cudaSuccess) return cuda_check(attr_err, "paged_gqa_decode smem attribute");
    if (g_dry_run) return I4_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.splits, p.Hkv, p.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kDynSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cuda_check(cudaLaunchKernelEx(&cfg, paged_gqa_decode_kernel, p), "paged_gqa_decode launch");
}

int read_attn_error(int reset) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_attn_error, sizeof v);
    if (e != cudaSuccess) return cuda_check(e, "reading the attention error flag");
    if (reset && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_attn_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_check(e, "clearing the attention error flag");
    }
    return v;
}

// out[b][g][t][:] = pool row of token t, t < ctx_len[b]
__global__ void paged_gather_kernel(const uint16_t *pool, const int32_t *table, const int32_t *ctx_len, uint16_t *out,
                                    int Hkv, int D, int P, int max_pages, int max_ctx) {
    const int b = blockIdx.z, g = blockIdx.y;
    int ctx = ctx_len[b];
    ctx = ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx);
    ctx = ctx > max_pages * P ? max_pages * P : ctx;
    const int vec = D / 8;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ctx * vec; i += gridDim.x * blockDim.x) {
        const int t = i / vec, c = i % vec;
        const size_t src = (((size_t)table[(size_t)b * max_pages + t / P] * Hkv + g) * P + t % P) * D + 8 * c;
        const size_t dst = (((size_t)b * Hkv + g) * max_ctx + t) * D + 8 * c;
        *reinterpret_cast<uint4 *>(out + dst) = *reinterpret_cast<const uint4 *>(pool + src);
    }
}

}  // namespace i4

using namespace i4;

static int attn_check(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool, const int32_t *page_table,
                      const int32_t *ctx_len, const uint16_t *out, int B, int Hq, int Hkv, int D, int page_size,
                      int max_pages) {
    if (!q || !k_pool || !v_pool || !page_table || !ctx_len || !out)
        return fail(I4_EINVAL, "paged_gqa_decode: null pointer");
    if (B < 1 || Hq < 1 || Hkv < 1 || max_pages < 1) return fail(I4_EINVAL, "paged_gqa_decode: bad sizes");
    if (D != 128) return fail(I4_EUNSUPPORTED, "paged_gqa_decode: head_dim %d (only 128)", D);
    if (Hq % Hkv != 0 || Hq / Hkv > 8) return fail(I4_EUNSUPPORTED, "paged_gqa_decode: Hq/Hkv must be an integer <= 8");
    if (page_size < 8 || page_size > kMaxPageSize || (page_size & (page_size - 1)))
        return fail(I4_EUNSUPPORTED, "paged_gqa_decode: page_size %d must be a power of two in [8, %d]", page_size,
                    kMaxPageSize);
    if (B > 65535 || Hkv > 65535) return fail(I4_EUNSUPPORTED, "paged_gqa_decode: grid too large");
    if ((long long)max_pages * page_size > kMaxCtx)
        return fail(I4_EUNSUPPORTED, "paged_gqa_decode: max_pages_per_seq * page_size above %d tokens", kMaxCtx);
    if (!aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(out, 16) ||
        !aligned(page_table, 4) || !aligned(ctx_len, 4))
        return fail(I4_EALIGN, "paged_gqa_decode: q/pools/out must be 16-byte aligned");
    return I4_OK;
}

extern "C" size_t paged_gqa_decode_ws_bytes(int B, int Hq, int Hkv, int D, int page_size, int max_pages_per_seq) {
    if (B < 1 || Hkv < 1 || Hq < Hkv || D != 128 || page_size < 1 || max_pages_per_seq < 1) return 0;
    return attn_ws_layout(B, Hq, Hkv, page_size, max_pages_per_seq).bytes;
}

static int decode_attention(const uint16_t *q, long long q_stride, const uint16_t *k_pool, const uint16_t *v_pool,
                            const int32_t *page_table, const int32_t *ctx_len, uint16_t *out, int B, int Hq, int Hkv,
                            int D, int page_size, int max_pages_per_seq, float scale, void *ws, size_t ws_bytes,
                            void *stream) {
    int st = attn_check(q, k_pool, v_pool, page_table, ctx_len, out, B, Hq, Hkv, D, page_size, max_pages_per_seq);
    if (st) return st;
    const AttnWs L = attn_ws_layout(B, Hq, Hkv, page_size, max_pages_per_seq);
    if (!ws || ws_bytes < L.bytes)
        return fail(I4_EINVAL, "paged_gqa_decode: workspace of %zu bytes needed (got %zu)", L.bytes, ws_bytes);
    if (!aligned(ws, 256)) return fail(I4_EALIGN, "paged_gqa_decode: workspace must be 256-byte aligned");
    AttnParams p = {};
    p.q = q;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.page_table = page_table;
    p.ctx_len = ctx_len;
    p.out = out;
    p.B = B;
    p.Hq = Hq;
    p.q_stride = q_stride;
    p.Hkv = Hkv;
    p.page_size = page_size;
    p.max_pages = max_pages_per_seq;
    p.scale = scale;
    p.splits = L.splits;
    p.cluster = L.cluster;
    p.ws = reinterpret_cast<char *>(ws);
    p.counters_off = L.counters_off;
    p.ml_off = L.ml_off;
    p.acc_off = L.acc_off;
    return launch_paged_gqa_decode(p, (cudaStream_t)stream, false);
}

extern "C" int paged_gqa_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                                const int32_t *page_table, const int32_t *ctx_len, uint16_t *out, int B, int Hq,
                                int Hkv, int D, int page_size, int max_pages_per_seq, float scale, void *ws,
                                size_t ws_bytes, void *stream) {
    return decode_attention(q, (long long)Hq * D, k_pool, v_pool, page_table, ctx_len, out, B, Hq, Hkv, D, page_size,
                            max_pages_per_seq, scale, ws, ws_bytes, stream);
}

extern "C" int i4_paged_gqa_decode_strided(const uint16_t *q, long long q_stride, const uint16_t *k_pool,
                                           const uint16_t *v_pool, const int32_t *page_table, const int32_t *ctx_len,
                                           uint16_t *out, int B, int Hq, int Hkv, int D, int page_size,
                                           int max_pages_per_seq, float scale, void *ws, size_t ws_bytes,
                                           void *stream) {
    if (q_stride < (long long)Hq * D || q_stride % 8)
        return fail(I4_EINVAL, "i4_paged_gqa_decode_strided: q_stride %lld must be >= Hq*D and a multiple of 8",
                    q_stride);
    return decode_attention(q, q_stride, k_pool, v_pool, page_table, ctx_len, out, B, Hq, Hkv, D, page_size,
                            max_pages_per_seq, scale, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------- no-allocation variant

// Split-K scratch of paged_gqa_decode_static: a fixed array in the module's
// device memory, so the call itself never allocates. Every GPU that loads the
// library keeps these bytes until the process exits. All calls share it.
static constexpr size_t kStaticScratchBytes = 8u << 20;
static __device__ __align__(256) unsigned char g_attn_static_scratch[kStaticScratchBytes];

static constexpr int kMaxDevices = 64;
static std::mutex g_static_scratch_mu;
static char *g_static_scratch_dev[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device. The array's name in host code is only a host-side handle, never a
// device address, so kernels get this pointer instead.
static int static_scratch_ptr(char **out) {
    int dev = 0;
    int st = cuda_check(cudaGetDevice(&dev), "paged_gqa_decode_static: cudaGetDevice");
    if (st) return st;
    if (dev < 0 || dev >= kMaxDevices) return fail(I4_EUNSUPPORTED, "paged_gqa_decode_static: device %d", dev);
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    if (!g_static_scratch_dev[dev]) {
        void *ptr = nullptr;
        st = cuda_check(cudaGetSymbolAddress(&ptr, g_attn_static_scratch), "paged_gqa_decode_static: scratch address");
        if (st) return st;
        g_static_scratch_dev[dev] = reinterpret_cast<char *>(ptr);
    }
    *out = g_static_scratch_dev[dev];
    return I4_OK;
}

extern "C" int paged_gqa_decode_static(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                                       const int32_t *page_table, const int32_t *ctx_len, uint16_t *out, int B,
                                       int Hq, int Hkv, int D, int page_size, int max_pages_per_seq, float scale,
                                       void *stream) {
    int st = attn_check(q, k_pool, v_pool, page_table, ctx_len, out, B, Hq, Hkv, D, page_size, max_pages_per_seq);
    if (st) return st;
    const AttnWs L = attn_ws_layout(B, Hq, Hkv, page_size, max_pages_per_seq);
    if (L.bytes > kStaticScratchBytes)
        return fail(I4_EUNSUPPORTED,
                    "paged_gqa_decode_static: this shape needs %zu bytes of split-K scratch, the static scratch "
                    "holds %zu; use paged_gqa_decode with a caller workspace",
                    L.bytes, kStaticScratchBytes);
    char *ws = nullptr;
    if ((st = static_scratch_ptr(&ws))) return st;
    // the merge counters must start at zero; the rest of the scratch is written before it is read
    st = cuda_check(cudaMemsetAsync(ws + L.counters_off, 0, (size_t)B * Hkv * sizeof(unsigned), (cudaStream_t)stream),
                    "paged_gqa_decode_static: clearing the counters");
    if (st) return st;
    AttnParams p = {};
    p.q = q;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.page_table = page_table;
    p.ctx_len = ctx_len;
    p.out = out;
    p.B = B;
    p.Hq = Hq;
    p.q_stride = (long long)Hq * 128;
    p.Hkv = Hkv;
    p.page_size = page_size;
    p.max_pages = max_pages_per_seq;
    p.scale = scale;
    p.splits = L.splits;
    p.cluster = L.cluster;
    p.ws = ws;
    p.counters_off = L.counters_off;
    p.ml_off = L.ml_off;
    p.acc_off = L.acc_off;
    return launch_paged_gqa_decode(p, (cudaStream_t)stream, false);
}

extern "C" int i4_paged_gather(const uint16_t *pool, const int32_t *page_table, const int32_t *ctx_len, uint16_t *out,
                               int B, int Hkv, int D, int page_size, int max_pages_per_seq, int max_ctx, void *stream) {
    if (!pool || !page_table || !ctx_len || !out) return fail(I4_EINVAL, "i4_paged_gather: null pointer");
    if (B < 1 || Hkv < 1 || D < 8 || D % 8 || page_size < 1 || max_pages_per_seq < 1 || max_ctx < 1)
        return fail(I4_EINVAL, "i4_paged_gather: bad sizes");
    if (!aligned(pool, 16) || !aligned(out, 16)) return fail(I4_EALIGN, "i4_paged_gather: 16-byte alignment");
    paged_gather_kernel<<<dim3(64, Hkv, B), 256, 0, (cudaStream_t)stream>>>(pool, page_table, ctx_len, out, Hkv, D,
                                                                           page_size, max_pages_per_seq, max_ctx);
    return launch_check("i4_paged_gather");
}
