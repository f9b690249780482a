// The whole decode step of one token as ONE persistent kernel.
//
// "How To Build Your Own LLM Runtime From Scratch" ("Technical Details": the
// decode GEMVs with fused INT4 dequantisation are where the time goes, and the
// step is replayed as one captured CUDA graph). At batch 1 a token is a stream
// of 3.65 GB of INT4 weights; launching 141 kernels per token stops that stream
// at every kernel boundary (each GEMV pays the start-up of its own stream and
// the drain of its tail). Here one CTA per SM runs every phase of the token:
//
//   per layer:  QKV  x = RMSNorm(r) (layer 0: embedding row) -> INT4 GEMV + bias -> RoPE, K/V append
//               ATTN paged GQA attention over the context (split over CTAs, log-sum-exp merge)
//               O    INT4 GEMV of the attention output -> r += fp16(y)
//               GU   x = RMSNorm(r) -> INT4 GEMV [gate | up] -> SiLU(gate) * up
//               DOWN INT4 GEMV -> r += fp16(y)
//   then        LM   x = RMSNorm(r) -> INT4 GEMV (fp32 logits) -> argmax -> state advance
//
// Warp 0 of every CTA is the producer: one thread streams the CTA's weight
// tiles of ALL phases, in order, into a ring of shared-memory slots with bulk
// asynchronous copies (cp.async.bulk, no tensor map, no multicast). Weights do
// not depend on activations, so the stream never waits for a phase to finish;
// it only waits for free slots. The 16 consumer warps wait at a grid-wide
// barrier between phases (every phase reads what all CTAs wrote in the one
// before), stage the phase's input vector in shared memory and consume the
// tiles already waiting in the ring.
//
// Tiles of a phase are dealt round robin over the CTAs, continuing where the
// previous phase stopped, so every SM streams the same number of bytes per
// token within one tile. Every wait is bounded (kWaitCycles); on a timeout the
// kernel records device error 1, stops issuing work, waits (bounded) for its
// own copies in flight and returns. The grid must be co-resident: one CTA per
// SM, checked with the occupancy query and launched cooperatively.
//
// Data written by one phase and read by a later one (residual, q, attention
// output, SiLU output, K/V rows, attention partials) is read with L2-coherent
// loads (ld.global.cg / cp.async.cg) after the grid barrier's acquire.
#include <cstring>

#include "async.cuh"
#include "common.cuh"
#include "gemv.cuh"
#include "gemv_parts.cuh"
#include "mma.cuh"
#include "persist.cuh"

namespace i4 {

constexpr int kPW = 16;               // consumer warps
constexpr int kPC = kPW * 32;         // consumer threads
constexpr int kPT = kPC + 32;         // + producer warp
constexpr int kPMaxStages = 8;
constexpr int kAW = 4;                // attention warps per CTA
constexpr int kATile = 16;            // keys per attention warp tile
constexpr unsigned kARegion = kATile * 128;       // one 64-dim half of 16 rows
constexpr unsigned kAWarpBytes = 4 * kARegion;    // K lo, K hi, V lo, V hi
constexpr int kAMaxG = 8;                          // query heads per kv head
constexpr int kAMaxSplitsSmem = 256;               // splits of one kv head the final merge holds in shared memory
constexpr float kLog2eP = 1.4426950408889634f;
constexpr int kMaxXWords = 8;         // x words per consumer thread: K <= 8 * 512 * 8 = 32768

__device__ int g_persist_error = 0;

__host__ __device__ constexpr int p_blocks(int K) { return (K + 1023) >> 10; }
__host__ __device__ constexpr int p_x_bytes(int K) { return p_blocks(K) * 2048 + (K >> 7) * 4; }

// ------------------------------------------------------------------ tiles

__device__ __forceinline__ int rr_pos(const PPhase &ph, int cta, int G) {
    const int r = cta - ph.first;
    return r < 0 ? r + G : r;
}

__device__ __forceinline__ int my_tile_count(const PPhase &ph, int cta, int G) {
    const int r = rr_pos(ph, cta, G);
    return r >= ph.tiles ? 0 : (ph.tiles - 1 - r) / G + 1;
}

struct TileRows {
    int ra0, rb0, pairs;  // pair p of the tile: global rows (ra0 + p, rb0 + p), slot rows (p, pairs + p)
};

__device__ __forceinline__ TileRows tile_rows(const PPhase &ph, int t, int inter) {
    TileRows r;
    const int half = ph.R >> 1;
    if (ph.kind == PH_QKV) {  // rotate-half partners (i, i + 64) of one 128-row head
        const int tph = 64 / half, head = t / tph;
        r.ra0 = head * 128 + (t - head * tph) * half;
        r.rb0 = r.ra0 + 64;
        r.pairs = half;
    } else if (ph.kind == PH_GU) {  // gate row n with up row n
        r.ra0 = t * half;
        r.rb0 = inter + r.ra0;
        r.pairs = half;
    } else {  // consecutive rows; a short last tile
        const int r0 = t * ph.R, na = (ph.N - r0) < ph.R ? (ph.N - r0) : ph.R;
        r.pairs = na >> 1;
        r.ra0 = r0;
        r.rb0 = r0 + r.pairs;
    }
    return r;
}

__device__ __forceinline__ void issue_tile_p(const PPhase &ph, const TileRows &tr, unsigned char *st, uint64_t *bar,
                                             uint64_t pol) {
    const unsigned wrow = (unsigned)ph.K >> 1, srow = (unsigned)ph.K >> 6, np = (unsigned)tr.pairs;
    mbar_expect_tx(bar, 2u * np * (wrow + srow));
    const unsigned char *w = reinterpret_cast<const unsigned char *>(ph.w);
    const unsigned char *s = reinterpret_cast<const unsigned char *>(ph.s);
    unsigned char *sc = st + (size_t)ph.R * wrow;
    if (tr.rb0 == tr.ra0 + tr.pairs) {
        bulk_load(st, w + (size_t)tr.ra0 * wrow, 2u * np * wrow, bar, pol);
        bulk_load(sc, s + (size_t)tr.ra0 * srow, 2u * np * srow, bar, pol);
    } else {
        bulk_load(st, w + (size_t)tr.ra0 * wrow, np * wrow, bar, pol);
        bulk_load(st + (size_t)np * wrow, w + (size_t)tr.rb0 * wrow, np * wrow, bar, pol);
        bulk_load(sc, s + (size_t)tr.ra0 * srow, np * srow, bar, pol);
        bulk_load(sc + (size_t)np * srow, s + (size_t)tr.rb0 * srow, np * srow, bar, pol);
    }
}

__device__ __forceinline__ void prefetch_l2(const void *p, unsigned bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// L2 prefetch of a tile's weights and scales (same ranges as issue_tile_p).
__device__ __forceinline__ void prefetch_tile_p(const PPhase &ph, const TileRows &tr) {
    const unsigned wrow = (unsigned)ph.K >> 1, srow = (unsigned)ph.K >> 6, np = (unsigned)tr.pairs;
    const unsigned char *w = reinterpret_cast<const unsigned char *>(ph.w);
    const unsigned char *s = reinterpret_cast<const unsigned char *>(ph.s);
    if (tr.rb0 == tr.ra0 + tr.pairs) {
        prefetch_l2(w + (size_t)tr.ra0 * wrow, 2u * np * wrow);
        prefetch_l2(s + (size_t)tr.ra0 * srow, 2u * np * srow);
    } else {
        prefetch_l2(w + (size_t)tr.ra0 * wrow, np * wrow);
        prefetch_l2(w + (size_t)tr.rb0 * wrow, np * wrow);
        prefetch_l2(s + (size_t)tr.ra0 * srow, np * srow);
        prefetch_l2(s + (size_t)tr.rb0 * srow, np * srow);
    }
}

// Walks one CTA's tiles over the phases of a launch in stream order.
struct TileIter {
    int p, k, n, r;
    PPhase ph;
    bool done;
};

__device__ __forceinline__ void tile_iter_seek(TileIter &it, const PersistArgs &a, int G) {
    while (it.k >= it.n) {
        if (++it.p >= a.phase_end) {
            it.done = true;
            return;
        }
        it.ph = a.phases[it.p];
        it.k = 0;
        it.n = it.ph.kind == PH_ATTN ? 0 : my_tile_count(it.ph, blockIdx.x, G);
        it.r = rr_pos(it.ph, blockIdx.x, G);
    }
}

__device__ __forceinline__ TileIter tile_iter_begin(const PersistArgs &a, int G) {
    TileIter it;
    it.p = a.phase_begin - 1;
    it.k = it.n = it.r = 0;
    it.done = false;
    tile_iter_seek(it, a, G);
    return it;
}

// This CTA's share of the K/V pages of the context (positions < ctx) of one layer, prefetched into L2
// while the layer's qkv phase runs: (page, kv head, K or V) items dealt round robin over the CTAs.
__device__ __forceinline__ void prefetch_kv(const PersistArgs &a, const PPhase &ph, int ctx) {
    const int pages = (ctx + a.page_size - 1) / a.page_size;
    const unsigned bytes = (unsigned)a.page_size * 256u;
    const int items = pages * a.n_kv * 2;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const int pg = it / (a.n_kv * 2), rest = it - pg * a.n_kv * 2, g = rest >> 1;
        const size_t off = ((size_t)a.page_table[pg] * a.n_kv + g) * a.page_size * 128;
        prefetch_l2((rest & 1) ? ph.v_pool + off : ph.k_pool + off, bytes);
    }
}

// ------------------------------------------------------------------ consumer helpers

using Consumers = NamedGroup<32, kPC>;

__device__ __forceinline__ uint4 ldcg_u4(const uint16_t *p) { return __ldcg(reinterpret_cast<const uint4 *>(p)); }
__device__ __forceinline__ float ldcg_h(const uint16_t *p) { return half_bits_to_float(__ldcg(p)); }

__device__ __forceinline__ bool aborted() { return *reinterpret_cast<volatile int *>(&g_persist_error) != 0; }

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void stamp(const PersistArgs &a, int p, int k) {
    if (a.trace) a.trace[((size_t)(p - a.phase_begin) * gridDim.x + blockIdx.x) * 4 + k] = global_ns();
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier of the consumer warps (the producer never waits on one).
// One 64-bit counter that only grows: barrier k of a launch waits until it
// reaches (base + k) * grid, where base = counter / grid read at the start of
// the launch (a CTA reads it before its first arrival, so no barrier of this
// launch can have completed yet). Each CTA adds 1 with release semantics and
// polls with acquire loads (bounded).
__device__ bool grid_barrier(const PersistArgs &a, unsigned long long target, const Consumers &grp, int *s_ok) {
    grp.sync();
    if (grp.tid() == 0) {
        int ok = 1;
        if (aborted()) {  // some wait of the launch gave up: leave together (the others see the flag too)
            ok = 0;
        } else {
            unsigned long long old;
            asm volatile("atom.add.release.gpu.global.u64 %0, [%1], 1;" : "=l"(old) : "l"(a.bar_count) : "memory");
            if (old + 1 < target) {
                const long long t0 = clock64();
                while (ld_acquire_u64(a.bar_count) < target) {
                    if (aborted()) {
                        ok = 0;
                        break;
                    }
                    if (clock64() - t0 > kWaitCycles) {
                        record_error(&g_persist_error, 1);
                        ok = 0;
                        break;
                    }
                }
            }
        }
        *s_ok = ok;
    }
    grp.sync();
    return *s_ok != 0;
}

// Stage the phase's input vector in the tensor-core lane order of the GEMV
// (per 1024-weight block, word and lane one 16-byte entry) and 8 * sum(x) per
// 128-weight group. PRO_PLAIN copies x; PRO_RMSNORM and PRO_EMBED compute
// x = fp16(r / sqrt(mean(r^2) + eps) * gamma) in fp32 (PRO_EMBED: r is the
// embedding row of the token, written to the residual when write_resid).
// Thread t handles words t, t + 512, ...; the 16 words of a 128-weight group
// sit on 16 consecutive lanes, whose sums meet by shuffles. gpre holds the
// thread's first two gamma words, loaded before the phase's grid barrier.
template <int PRO>
__device__ __noinline__ void stage_x_p(const PersistArgs &a, int K, const uint16_t *src, const uint16_t *gamma,
                                       const uint4 *gpre, uint4 *xt, float *sx8, float *red, const Consumers &grp,
                                       bool write_resid) {
    const int nwords = K >> 3, nb = p_blocks(K), tid = grp.tid();
    for (int i = nwords + tid; i < nb * 128; i += kPC) {  // padding of a partial last block
        const int b = i >> 7, l = (i & 127) >> 2, w = i & 3;
        xt[(b * 4 + w) * 32 + l] = make_uint4(0u, 0u, 0u, 0u);
    }
    // the first kKeepWords words of each thread stay in registers between the two passes of RMSNorm; rows
    // longer than kKeepWords * kPC * 8 values read the rest again
    constexpr int kKeepWords = 2;
    auto load = [&](int wd) {
        return PRO == PRO_EMBED ? *reinterpret_cast<const uint4 *>(src + 8 * wd) : ldcg_u4(src + 8 * wd);
    };
    uint4 rv[kKeepWords];
    float inv = 0.f;
    if constexpr (PRO != PRO_PLAIN) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxXWords; ++i) {
            const int wd = tid + i * kPC;
            if (wd < nwords) {
                const uint4 v = load(wd);
                if (i < kKeepWords) rv[i] = v;
                const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
                    ss = fmaf(f.x, f.x, ss);
                    ss = fmaf(f.y, f.y, ss);
                }
            }
        }
        ss = group_sum(ss, red, grp);
        inv = 1.0f / sqrtf(ss / (float)K + a.eps);
    }
    // rounds of 512 words; every lane takes part in each round's shuffles (nwords is a multiple of 16, so the
    // 16 lanes of a group are all inside or all outside the row)
    const int rounds = (nwords + kPC - 1) / kPC;
    for (int i = 0; i < rounds; ++i) {
        const int wd = tid + i * kPC;
        const bool in = wd < nwords;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (in) {
            if constexpr (PRO == PRO_PLAIN) {
                x = ldcg_u4(src + 8 * wd);
            } else {
                const uint4 gv = i < kKeepWords ? gpre[i < kKeepWords ? i : 0]
                                                : *reinterpret_cast<const uint4 *>(gamma + 8 * wd);
                const uint4 v = i < kKeepWords ? rv[i < kKeepWords ? i : 0] : load(wd);
                if constexpr (PRO == PRO_EMBED) {
                    if (write_resid) *reinterpret_cast<uint4 *>(a.resid + 8 * wd) = v;
                }
                const uint32_t r[4] = {v.x, v.y, v.z, v.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
                uint32_t o[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 fr = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
                    const float2 fg = __half22float2(*reinterpret_cast<const __half2 *>(&g[t]));
                    const __half2 h = __floats2half2_rn(fr.x * inv * fg.x, fr.y * inv * fg.y);
                    o[t] = *reinterpret_cast<const uint32_t *>(&h);
                }
                x = make_uint4(o[0], o[1], o[2], o[3]);
            }
            const int b = wd >> 7, l = (wd & 127) >> 2, w = wd & 3;
            const uint4 pp = permute_pairs(x);  // (x0,x4) (x1,x5) (x2,x6) (x3,x7)
            xt[(b * 4 + w) * 32 + l] = make_uint4(pp.x, pp.z, pp.y, pp.w);
        }
        const uint32_t e[4] = {x.x, x.y, x.z, x.w};
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&e[q]));
            t += f.x + f.y;
        }
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        t += __shfl_xor_sync(0xffffffffu, t, 4);
        t += __shfl_xor_sync(0xffffffffu, t, 8);
        if (in && (tid & 15) == 0) sx8[wd >> 4] = 8.0f * t;
    }
    grp.sync();
}

// Epilogue inputs in global memory, loaded before the tile's arithmetic.
struct EpiVals {
    float a, b;
    float2 cs;
    int page;
};

template <int KIND>
__device__ __forceinline__ EpiVals epi_load_p(const PersistArgs &a, const PPhase &ph, int ra, int rb, int pos) {
    EpiVals e = {0.f, 0.f, make_float2(0.f, 0.f), 0};
    if constexpr (KIND == PH_QKV) {
        e.a = half_bits_to_float(ph.bias[ra]);
        e.b = half_bits_to_float(ph.bias[rb]);
        const int head = ra >> 7;
        if (pos >= 0 && pos < a.max_ctx) {
            if (head < a.n_q + a.n_kv) e.cs = a.rope_cs[(size_t)pos * 64 + (ra & 63)];
            if (head >= a.n_q) e.page = a.page_table[pos / a.page_size];
        }
    } else if constexpr (KIND == PH_O || KIND == PH_DOWN) {
        e.a = ldcg_h(a.resid + ra);
        e.b = ldcg_h(a.resid + rb);
    }
    return e;
}

template <int KIND>
__device__ __forceinline__ void epi_store_p(const PersistArgs &a, const PPhase &ph, int ra, int rb, float va,
                                            float vb, const EpiVals &e, int pos, unsigned long long &best) {
    if constexpr (KIND == PH_QKV) {
        const int head = ra >> 7, i = ra & 63;
        const float xa = rnd16(va + e.a), xb = rnd16(vb + e.b);
        if (pos < 0 || pos >= a.max_ctx) {
            if (a.status) *a.status = 2;
            return;
        }
        if (head < a.n_q + a.n_kv) {
            uint16_t oa, ob;
            rope_pair(xa, xb, e.cs, oa, ob);
            if (head < a.n_q) {
                a.q[head * 128 + i] = oa;
                a.q[head * 128 + i + 64] = ob;
            } else {
                const size_t off = (((size_t)e.page * a.n_kv + (head - a.n_q)) * a.page_size + pos % a.page_size) * 128;
                ph.k_pool[off + i] = oa;
                ph.k_pool[off + i + 64] = ob;
            }
        } else {
            const size_t off =
                (((size_t)e.page * a.n_kv + (head - a.n_q - a.n_kv)) * a.page_size + pos % a.page_size) * 128;
            ph.v_pool[off + i] = float_to_half_bits(xa);
            ph.v_pool[off + i + 64] = float_to_half_bits(xb);
        }
    } else if constexpr (KIND == PH_O || KIND == PH_DOWN) {
        a.resid[ra] = float_to_half_bits(e.a + rnd16(va));
        a.resid[rb] = float_to_half_bits(e.b + rnd16(vb));
    } else if constexpr (KIND == PH_GU) {
        a.mlp[ra] = silu_mul_bits(rnd16(va), rnd16(vb));
    } else if constexpr (KIND == PH_LM) {
        a.logits[ra] = va;
        a.logits[rb] = vb;
        unsigned long long k = argmax_key(va, ra);
        best = k > best ? k : best;
        k = argmax_key(vb, rb);
        best = k > best ? k : best;
    }
}

// All of this CTA's tiles of one GEMV phase (tiles r, r + grid, ... of the
// phase; i0 = the tile sequence number of the first one). Tiles of 16 row pairs
// give each consumer warp one pair; other tiles deal their pair-blocks evenly
// over the warps and meet in shared memory. A wait that gives up records the
// device error and turns the rest of the phase into no-ops for this warp; the
// control flow (and every shared barrier) stays the same for all warps.
template <int KIND, int KC>
__device__ __noinline__ unsigned long long gemv_tiles(const PersistArgs &a, const PPhase &ph, int n, int r, int i0,
                                                      unsigned char *ring, uint64_t *full, uint64_t *empty,
                                                      const uint4 *xt, const float *sx8, float2 *part, int pos) {
    const int K = KC ? KC : ph.K, wrow = K >> 1, groups = K >> 7, nb = p_blocks(K);
    const int tid = threadIdx.x - 32, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, S = a.stages;
    const Consumers grp;
    unsigned long long best = 0ull;
    for (int k = 0; k < n; ++k) {
        const int i = i0 + k, s = i % S, use = i / S;
        const TileRows tr = tile_rows(ph, r + k * G, a.inter);
        const unsigned char *st = ring + (size_t)s * a.slot_bytes;
        const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + (size_t)ph.R * wrow);
        if (tr.pairs == kPW) {
            EpiVals ev = {0.f, 0.f, make_float2(0.f, 0.f), 0};
            if (lane == 0) ev = epi_load_p<KIND>(a, ph, tr.ra0 + warp, tr.rb0 + warp, pos);
            bool ok = mbar_wait(&full[s], (unsigned)(use & 1));
            if (!ok) record_error(&g_persist_error, 1);
            ok = __all_sync(0xffffffffu, ok);
            float2 v = make_float2(0.f, 0.f);
            if (ok)
                v = pair_dot<KC>(st, K, warp, kPW + warp, sc + (size_t)warp * groups, sc + (size_t)(kPW + warp) * groups,
                                 xt, sx8, 0, nb, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            v = warp_sum2(v);
            if (lane == 0 && ok) epi_store_p<KIND>(a, ph, tr.ra0 + warp, tr.rb0 + warp, v.x, v.y, ev, pos, best);
        } else {
            float2 *pp = part + (size_t)(i & 1) * 16 * kPW;  // [pair][warp] of this tile's parity
            const int U = tr.pairs * nb, u0 = warp * U / kPW, u1 = (warp + 1) * U / kPW;
            EpiVals ev = {0.f, 0.f, make_float2(0.f, 0.f), 0};
            if (tid < tr.pairs) ev = epi_load_p<KIND>(a, ph, tr.ra0 + tid, tr.rb0 + tid, pos);
            bool ok = mbar_wait(&full[s], (unsigned)(use & 1));
            if (!ok) record_error(&g_persist_error, 1);
            ok = __all_sync(0xffffffffu, ok);
            for (int u = u0; u < u1 && ok;) {
                const int pr = u / nb, bs = u - pr * nb, be = (bs + (u1 - u)) < nb ? (bs + (u1 - u)) : nb;
                float2 v = pair_dot<KC>(st, K, pr, tr.pairs + pr, sc + (size_t)pr * groups,
                                        sc + (size_t)(tr.pairs + pr) * groups, xt, sx8, bs, be, lane);
                v = warp_sum2(v);
                if (lane == 0) pp[pr * kPW + warp] = v;
                u += be - bs;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            grp.sync();
            if (tid < tr.pairs) {
                float2 v = make_float2(0.f, 0.f);
                for (int w = 0; w < kPW; ++w) {
                    const float2 q = pp[tid * kPW + w];
                    v.x += q.x;
                    v.y += q.y;
                    pp[tid * kPW + w] = make_float2(0.f, 0.f);
                }
                if (ok) epi_store_p<KIND>(a, ph, tr.ra0 + tid, tr.rb0 + tid, v.x, v.y, ev, pos, best);
            }
        }
    }
    return best;
}

// ------------------------------------------------------------------ attention phase

// Split of the context over the CTAs of one kv head: S CTAs per head, each a
// contiguous run of 16-key tiles, dealt over its kAW warps.
__device__ __forceinline__ int attn_splits(int n_tiles, int G, int n_kv, int max_splits) {
    int s = (n_tiles + kAW - 1) / kAW;
    const int cap = G / n_kv < max_splits ? G / n_kv : max_splits;
    s = s < cap ? s : cap;
    return s < 1 ? 1 : s;
}

// One CTA's share of paged GQA decode attention for kv head g: its warps stage
// 16-key tiles (K and V rows, 16-byte cp.async, 64-dim halves XOR-swizzled by
// row) and run S = Q K^T and O^T = V^T P^T on mma.m16n8k16 with the group's
// query heads as MMA rows, online softmax in the log2 domain; the warps merge
// in shared memory, the CTA writes its (max, sum, unnormalised output) partial,
// and the last CTA of the head to arrive merges all partials into the output.
__device__ __noinline__ void attention_phase(const PersistArgs &a, const PPhase &ph, int ph_index, unsigned char *area,
                                             int ctx, int *s_flag) {
    const int tid = threadIdx.x - 32, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, Gq = a.n_q / a.n_kv;
    const int n_tiles = (ctx + kATile - 1) / kATile;
    const int S = attn_splits(n_tiles, G, a.n_kv, a.attn_max_splits);
    if ((int)blockIdx.x >= a.n_kv * S) return;
    const int g = blockIdx.x / S, s = blockIdx.x % S;
    const int tpc = (n_tiles + S - 1) / S;
    const int t_begin = s * tpc, t_end = (t_begin + tpc) < n_tiles ? (t_begin + tpc) : n_tiles;
    const int P = a.page_size, pshift = __ffs(P) - 1;
    const int32_t *table = a.page_table;
    const uint32_t base = smem_u32(area);
    const uint32_t ring = base + warp * kAWarpBytes;

    const int gq = lane >> 2, tig = lane & 3;
    uint32_t qa[8][2];
    {
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(a.q + (size_t)(g * Gq + gq) * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qa[kk][0] = gq < Gq ? __ldcg(qrow + 8 * kk + tig) : 0u;
            qa[kk][1] = gq < Gq ? __ldcg(qrow + 8 * kk + 4 + tig) : 0u;
        }
    }
    const float qscale = a.attn_scale * kLog2eP;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const int r8 = lane & 7, mi = lane >> 3;
    const int chunk = lane & 15, row_lo = lane >> 4;
    const uint32_t chunk_off = (chunk >> 3) * kARegion;
    const size_t head_rows = (size_t)g * P;
    if (warp < kAW) {
        for (int tt = t_begin + warp; tt < t_end; tt += kAW) {
            const int t0 = tt * kATile;
            const int tl = (t0 + kATile - 1) < ctx ? (t0 + kATile - 1) : ctx - 1;
            const int pa = t0 >> pshift;
            const int ea = table[pa], eb = table[tl >> pshift];
            const size_t base_a = (((size_t)ea * a.n_kv) * P + head_rows) * 128 + chunk * 8;
            const size_t base_b = (((size_t)eb * a.n_kv) * P + head_rows) * 128 + chunk * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = row_lo + 2 * j, tok = t0 + r;
                if (tok < ctx) {
                    const size_t off = ((tok >> pshift) == pa ? base_a : base_b) + (size_t)(tok & (P - 1)) * 128;
                    const uint32_t dst = ring + chunk_off + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
                    cp_async16(dst, ph.k_pool + off);
                    cp_async16(dst + 2 * kARegion, ph.v_pool + off);
                }
            }
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            const int valid = ctx - t0;
            const uint32_t kb = ring, vb = ring + 2 * kARegion;
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
                const int c = 4 * k2 + mi;
                const uint32_t off = (c >> 3) * kARegion + (((c & 7) ^ r8) << 4);
                uint32_t b0, b1, b2, b3, e0, e1, e2, e3;
                ldsm_x4(kb + off + r8 * 128, b0, b1, b2, b3);
                ldsm_x4(kb + off + (r8 + 8) * 128, e0, e1, e2, e3);
                mma16816(s0, qa[2 * k2][0], 0u, qa[2 * k2][1], 0u, b0, b1);
                mma16816(s1, qa[2 * k2][0], 0u, qa[2 * k2][1], 0u, e0, e1);
                mma16816(s0, qa[2 * k2 + 1][0], 0u, qa[2 * k2 + 1][1], 0u, b2, b3);
                mma16816(s1, qa[2 * k2 + 1][0], 0u, qa[2 * k2 + 1][1], 0u, e2, e3);
            }
            const int j = 2 * tig;
            float sv[4] = {s0[0] * qscale, s0[1] * qscale, s1[0] * qscale, s1[1] * qscale};
            uint32_t mk01 = 0xffffffffu, mk89 = 0xffffffffu;
            if (valid < kATile) {
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
            const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * tig);
            const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
            const uint32_t pb0 = h2_bits(p01), pb1 = h2_bits(p89);
#pragma unroll
            for (int im = 0; im < 8; ++im) {
                const int c = 2 * im + (mi & 1);
                const int row = (mi >> 1) * 8 + r8;
                uint32_t a0, a1, a2, a3;
                ldsm_x4_trans(vb + (c >> 3) * kARegion + row * 128 + (((c & 7) ^ r8) << 4), a0, a1, a2, a3);
                o[im][0] *= a_lo;
                o[im][1] *= a_hi;
                o[im][2] *= a_lo;
                o[im][3] *= a_hi;
                mma16816(o[im], a0 & mk01, a1 & mk01, a2 & mk89, a3 & mk89, pb0, pb1);
            }
            __syncwarp();  // every lane is done with the stage before it is refilled
        }
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if (tid == 0) stamp(a, ph_index, 1);  // warp 0's tiles done

    // merge the kAW warps (the staging area becomes the partial buffer) -- all 16 warps take part in
    // the barriers; warps >= kAW hold empty partials and are not read
    float *wo = reinterpret_cast<float *>(area);                                       // [warp][dim][head]
    float2 *wml = reinterpret_cast<float2 *>(area + kAW * 128 * kAMaxG * 4);          // [warp][head]
    float *cw = reinterpret_cast<float *>(wml + kAW * kAMaxG);                         // [warp][head]
    float *cML = cw + kAW * kAMaxG;                                                    // M[head], L[head]
    const Consumers grp;
    grp.sync();
    if (warp < kAW) {
        if (tig == 0) wml[warp * kAMaxG + gq] = make_float2(m_run, l_run);
#pragma unroll
        for (int im = 0; im < 8; ++im) {
            float *r = wo + ((size_t)warp * 128 + 16 * im + gq) * kAMaxG + 2 * tig;
            *reinterpret_cast<float2 *>(r) = make_float2(o[im][0], o[im][1]);
            *reinterpret_cast<float2 *>(r + 8 * kAMaxG) = make_float2(o[im][2], o[im][3]);
        }
    }
    grp.sync();
    if (tid < 32) {  // lane 4 h + k: weight of warp k's partial of head h
        const int h = tid >> 2, k = tid & 3;
        const float2 v = wml[k * kAMaxG + h];
        float M = fmaxf(v.x, __shfl_xor_sync(0xffffffffu, v.x, 1));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
        const float wt = merge_weight(v.x, M);
        float L = wt * v.y;
        L += __shfl_xor_sync(0xffffffffu, L, 1);
        L += __shfl_xor_sync(0xffffffffu, L, 2);
        cw[k * kAMaxG + h] = wt;
        if (k == 0) {
            cML[h] = M;
            cML[kAMaxG + h] = L;
        }
    }
    grp.sync();
    const size_t cell = ((size_t)g * a.attn_max_splits + s) * kAMaxG;
    if (tid < 128) {  // thread = output dim
        const int d = tid;
        for (int h = 0; h < Gq; ++h) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < kAW; ++k) acc = fmaf(cw[k * kAMaxG + h], wo[((size_t)k * 128 + d) * kAMaxG + h], acc);
            a.attn_acc[(cell + h) * 128 + d] = acc;
        }
        if (d < Gq) a.attn_ml[cell + d] = make_float2(cML[d], cML[kAMaxG + d]);
    }
    __threadfence();
    grp.sync();
    if (tid == 0) *s_flag = atomicAdd(a.attn_count + g, 1u) == (unsigned)S - 1u;
    grp.sync();
    if (tid == 0) stamp(a, ph_index, 3);  // partial published
    if (!*s_flag) return;
    __threadfence();
    // last CTA of this kv head: out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s. The (m, l) of all
    // splits are loaded at once into shared memory, each head's normalised weights computed there, and
    // every thread then sums its outputs' partials with independent loads.
    float *coef = reinterpret_cast<float *>(area);             // [head][split] weight, then normalised
    float *lsum = coef + kAMaxG * kAMaxSplitsSmem;             // [head][split] l
    const float2 *mlg = a.attn_ml + (size_t)g * a.attn_max_splits * kAMaxG;
    for (int i = tid; i < S * kAMaxG; i += kPC) {
        const float2 v = __ldcg(&mlg[i]);
        coef[(i % kAMaxG) * kAMaxSplitsSmem + i / kAMaxG] = v.x;
        lsum[(i % kAMaxG) * kAMaxSplitsSmem + i / kAMaxG] = v.y;
    }
    grp.sync();
    if (warp < Gq) {  // warp h: weights of head h
        float *ch = coef + warp * kAMaxSplitsSmem;
        const float *lh = lsum + warp * kAMaxSplitsSmem;
        float M = -INFINITY;
        for (int k = lane; k < S; k += 32) M = fmaxf(M, ch[k]);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
        float L = 0.f;
        for (int k = lane; k < S; k += 32) {
            const float wt = merge_weight(ch[k], M);
            ch[k] = wt;
            L = fmaf(wt, lh[k], L);
        }
        L = warp_sum(L);
        const float inv = 1.0f / L;
        __syncwarp();
        for (int k = lane; k < S; k += 32) ch[k] *= inv;
    }
    grp.sync();
    const float *accg = a.attn_acc + (size_t)g * a.attn_max_splits * kAMaxG * 128;
    for (int o = tid; o < Gq * 128; o += kPC) {
        const int h = o >> 7, d = o & 127;
        const float *ch = coef + h * kAMaxSplitsSmem;
        float acc = 0.f;
        for (int k0 = 0; k0 < S; k0 += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = k0 + u < S ? __ldcg(&accg[((size_t)(k0 + u) * kAMaxG + h) * 128 + d]) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (k0 + u < S) acc = fmaf(ch[k0 + u], v[u], acc);
        }
        a.attn[(size_t)(g * Gq + h) * 128 + d] = float_to_half_bits(acc);
    }
    if (tid == 0) a.attn_count[g] = 0u;  // ready for the next layer
}

// ------------------------------------------------------------------ the kernel

__global__ void __maxnreg__(96) decode_persistent_kernel(const PersistArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kPMaxStages];
    __shared__ __align__(8) uint64_t empty[kPMaxStages];
    __shared__ float red[32];
    __shared__ float2 part[2][16][kPW];  // per-warp partial sums of a tile's pairs [tile parity][pair][warp]
    __shared__ unsigned long long wbest[kPW];
    __shared__ int s_ok, s_flag;

    const int S = a.stages, G = gridDim.x, cta = blockIdx.x;
    unsigned char *ring = smem;
    unsigned char *xarea = smem + (size_t)S * a.slot_bytes;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kPW);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = threadIdx.x; i < 2 * 16 * kPW; i += blockDim.x) (&part[0][0][0])[i] = make_float2(0.f, 0.f);
    __syncthreads();

    if (threadIdx.x < 32) {
        // ---------------- producer: the CTA's tiles of every phase in order into the ring; a second walk
        // a.l2_ahead tiles further on prefetches into L2, so HBM keeps streaming while the consumers wait at
        // barriers or attention (the ring itself holds only a few microseconds of the stream)
        if (threadIdx.x != 0) return;
        const uint64_t pol = evict_first_policy();
        int ctx = *a.ctx_len;
        ctx = ctx < 1 ? 1 : (ctx > a.max_ctx ? a.max_ctx : ctx);
        TileIter it = tile_iter_begin(a, G), ahead = it;
        int kv_layer = -1;  // last layer whose K/V pages were prefetched
        for (int j = 0; j < a.l2_ahead && !ahead.done; ++j) {
            prefetch_tile_p(ahead.ph, tile_rows(ahead.ph, ahead.r + ahead.k * G, a.inter));
            ++ahead.k;
            tile_iter_seek(ahead, a, G);
        }
        int i = 0;
        bool ok = true;
        for (; !it.done; ++i) {
            if (it.k == 0) stamp(a, it.p, 3);
            if (it.ph.kind == PH_QKV && it.ph.layer != kv_layer && it.p + 1 < a.phase_end) {
                kv_layer = it.ph.layer;
                prefetch_kv(a, a.phases[it.p + 1], ctx);
            }
            const int s = i % S, use = i / S;
            if (use > 0 && !mbar_wait(&empty[s], (unsigned)((use - 1) & 1))) {
                record_error(&g_persist_error, 1);
                ok = false;
                break;
            }
            if (aborted()) {
                ok = false;
                break;
            }
            issue_tile_p(it.ph, tile_rows(it.ph, it.r + it.k * G, a.inter), ring + (size_t)s * a.slot_bytes, &full[s],
                         pol);
            if (!ahead.done) {
                prefetch_tile_p(ahead.ph, tile_rows(ahead.ph, ahead.r + ahead.k * G, a.inter));
                ++ahead.k;
                tile_iter_seek(ahead, a, G);
            }
            ++it.k;
            tile_iter_seek(it, a, G);
        }
        if (!ok) {  // the consumers stopped: wait for the copies still in flight into this CTA's ring
            for (int j = i - S > 0 ? i - S : 0; j < i; ++j) mbar_wait(&full[j % S], (unsigned)((j / S) & 1));
        }
        return;
    }

    // ---------------- consumers
    const Consumers grp;
    const int tid = grp.tid(), warp = tid >> 5, lane = tid & 31;
    unsigned long long bar_base = 0;
    if (tid == 0) bar_base = ld_acquire_u64(a.bar_count) / (unsigned long long)G;
    int ctx = *a.ctx_len;
    ctx = ctx < 1 ? 1 : (ctx > a.max_ctx ? a.max_ctx : ctx);
    const int pos = *a.pos;
    unsigned long long best = 0ull;
    int nbar = 0, i = 0;
    bool lm = false;
    PPhase ph = a.phases[a.phase_begin];
    uint4 gpre[2];  // this thread's first gamma words of the phase's RMSNorm, loaded ahead of its barrier
    auto prefetch_gamma = [&](const PPhase &q) {
        if (q.gamma) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int wd = tid + k * kPC;
                gpre[k] = wd < (q.K >> 3) ? *reinterpret_cast<const uint4 *>(q.gamma + 8 * wd) : make_uint4(0, 0, 0, 0);
            }
        }
    };
    prefetch_gamma(ph);
    for (int p = a.phase_begin; p < a.phase_end; ++p) {
        if (p > a.phase_begin && !grid_barrier(a, (bar_base + (unsigned long long)(++nbar)) * G, grp, &s_ok)) break;
        if (tid == 0) stamp(a, p, 0);
        if (ph.kind == PH_ATTN) {
            attention_phase(a, ph, p, xarea, ctx, &s_flag);
            if (tid == 0) stamp(a, p, 2);
        } else {
            lm = lm || ph.kind == PH_LM;
            const int n = my_tile_count(ph, cta, G), r = rr_pos(ph, cta, G);
            if (n > 0) {
                const int K = ph.K, nb = p_blocks(K);
                uint4 *xt = reinterpret_cast<uint4 *>(xarea);
                float *sx8 = reinterpret_cast<float *>(xarea + (size_t)nb * 2048);
                if (ph.kind == PH_QKV && ph.layer == 0) {
                    int tok = *a.token;
                    tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);
                    // the CTA holding the phase's first tile also writes the embedding row to the residual
                    stage_x_p<PRO_EMBED>(a, K, a.embed + (size_t)tok * K, ph.gamma, gpre, xt, sx8, red, grp, r == 0);
                } else if (ph.kind == PH_QKV || ph.kind == PH_GU || ph.kind == PH_LM) {
                    stage_x_p<PRO_RMSNORM>(a, K, a.resid, ph.gamma, gpre, xt, sx8, red, grp, false);
                } else {
                    stage_x_p<PRO_PLAIN>(a, K, ph.kind == PH_O ? a.attn : a.mlp, nullptr, gpre, xt, sx8, red, grp,
                                         false);
                }
                if (tid == 0) stamp(a, p, 1);
                float2 *pp = &part[0][0][0];
                unsigned long long b = 0ull;
                switch (ph.kind) {
                    case PH_QKV:
                        b = K == 3584 ? gemv_tiles<PH_QKV, 3584>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos)
                                      : gemv_tiles<PH_QKV, 0>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos);
                        break;
                    case PH_O:
                        b = K == 3584 ? gemv_tiles<PH_O, 3584>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos)
                                      : gemv_tiles<PH_O, 0>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos);
                        break;
                    case PH_GU:
                        b = K == 3584 ? gemv_tiles<PH_GU, 3584>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos)
                                      : gemv_tiles<PH_GU, 0>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos);
                        break;
                    case PH_DOWN:
                        b = K == 18944 ? gemv_tiles<PH_DOWN, 18944>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos)
                                       : gemv_tiles<PH_DOWN, 0>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos);
                        break;
                    default:
                        b = K == 3584 ? gemv_tiles<PH_LM, 3584>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos)
                                      : gemv_tiles<PH_LM, 0>(a, ph, n, r, i, ring, full, empty, xt, sx8, pp, pos);
                        break;
                }
                best = b > best ? b : best;
                i += n;
                if (tid == 0) stamp(a, p, 2);
            }
        }
        if (p + 1 < a.phase_end) {  // the next phase's descriptor and gamma, in flight during the barrier
            ph = a.phases[p + 1];
            prefetch_gamma(ph);
        }
    }
    // every consumer thread reaches this point through the same barriers: a failed wait only skips
    // arithmetic, and leaving early happens at a grid barrier, uniformly for the CTA
    if (lm) {
        // lm_head: pick the token over all CTAs; the last CTA to arrive advances the sequence state
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        if (lane == 0) wbest[warp] = best;
        grp.sync();
        if (tid == 0 && !aborted()) {
            unsigned long long b = 0ull;
            for (int w = 0; w < kPW; ++w) b = wbest[w] > b ? wbest[w] : b;
            atomicMax(a.best, b);
            __threadfence();
            const bool last = atomicAdd(a.arrive, 1u) == (unsigned)G - 1u;
            if (last) {
                __threadfence();
                const unsigned long long bb = atomicAdd(a.best, 0ull);
                const int idx = (int)(0xFFFFFFFFu - (uint32_t)(bb & 0xFFFFFFFFull));
                const int np = pos + 1;
                if (np >= a.max_ctx || pos < 0) {
                    if (a.status) *a.status = 1;
                } else {
                    const int tok = (a.prompt && np < a.n_prompt) ? a.prompt[np] : idx;
                    *a.token = tok;
                    *a.pos = np;
                    *a.ctx_len = np + 1;
                    if (a.history) a.history[np] = tok;
                }
                *a.best = 0ull;
                *a.arrive = 0u;
                __threadfence();
            }
        }
    }
}

// ------------------------------------------------------------------ host side

static int g_persist_max_dyn = -1;

PersistPlan persist_plan(const i4_model_desc &d) {
    PersistPlan pl = {};
    pl.ok = false;
    const int H = d.hidden, I = d.intermediate, QD = d.n_q_heads * d.head_dim;
    if (d.head_dim != 128 || H % 512 || I % 512 || QD % 512 || d.n_q_heads % d.n_kv_heads ||
        d.n_q_heads / d.n_kv_heads > kAMaxG || d.n_kv_heads > 64 || d.vocab % 2 || d.page_size < 8)
        return pl;
    auto rowb = [](int K) { return (K >> 1) + (K >> 6); };
    int slot = 32 * rowb(H);                       // QKV, GU and the K = hidden GEMVs: 32-row tiles
    if (2 * rowb(I) > slot) slot = 2 * rowb(I);    // down: at least one row pair
    if (2 * rowb(QD) > slot) slot = 2 * rowb(QD);
    slot = (slot + 127) / 128 * 128;
    int xa = p_x_bytes(H);
    if (p_x_bytes(I) > xa) xa = p_x_bytes(I);
    if (p_x_bytes(QD) > xa) xa = p_x_bytes(QD);
    const int attn_bytes = kAW * (int)kAWarpBytes;
    if (attn_bytes > xa) xa = attn_bytes;
    xa = (xa + 127) / 128 * 128;
    int dev = 0, sms = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return pl;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaFuncAttributes fa = {};
    if (cudaFuncGetAttributes(&fa, decode_persistent_kernel) != cudaSuccess) return pl;
    const int budget = optin - (int)fa.sharedSizeBytes - 1024;
    int stages = (budget - xa) / slot;
    if (stages > kPMaxStages) stages = kPMaxStages;
    if (stages < 2 || sms < 1) return pl;
    pl.grid = sms;
    pl.slot_bytes = slot;
    pl.stages = stages;
    pl.xarea_bytes = xa;
    pl.smem = stages * slot + xa;
    pl.attn_max_splits = sms / d.n_kv_heads < kAMaxSplitsSmem ? sms / d.n_kv_heads : kAMaxSplitsSmem;
    const size_t cells = (size_t)d.n_kv_heads * pl.attn_max_splits * kAMaxG;
    pl.ws_bytes = 256 /* sync words */ + 256 /* attention counters */ + ((cells * sizeof(float2) + 255) & ~(size_t)255) +
                  cells * 128 * sizeof(float);
    pl.ok = true;
    return pl;
}

void persist_fill_phases(const i4_model_desc &d, const PersistPlan &pl, PPhase *ph) {
    const int H = d.hidden, I = d.intermediate, QD = d.n_q_heads * d.head_dim;
    const int nqkv = (d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim;
    auto rowb = [](int K) { return (K >> 1) + (K >> 6); };
    auto rows_fit = [&](int K) {
        int R = pl.slot_bytes / rowb(K);
        R = R > 32 ? 32 : R;
        return R & ~1;
    };
    long long dealt = 0;
    int n = 0;
    auto push = [&](int kind, int layer, int N, int K, int R, int tiles) {
        PPhase p = {};
        p.kind = kind;
        p.layer = layer;
        p.N = N;
        p.K = K;
        p.R = R;
        p.tiles = tiles;
        p.first = (int)(dealt % pl.grid);
        dealt += tiles;
        ph[n++] = p;
    };
    for (int l = 0; l < d.n_layers; ++l) {
        push(PH_QKV, l, nqkv, H, 32, nqkv / 32);
        push(PH_ATTN, l, 0, 0, 0, 0);
        const int Ro = rows_fit(QD);
        push(PH_O, l, H, QD, Ro, (H + Ro - 1) / Ro);
        push(PH_GU, l, 2 * I, H, 32, I / 16);
        const int Rd = rows_fit(I);
        push(PH_DOWN, l, H, I, Rd, (H + Rd - 1) / Rd);
    }
    const int Rl = rows_fit(H);
    push(PH_LM, d.n_layers, d.vocab, H, Rl, (d.vocab + Rl - 1) / Rl);
}

int persist_configure(const PersistPlan &pl) {
    if (pl.smem > g_persist_max_dyn) {
        cudaError_t e =
            cudaFuncSetAttribute(decode_persistent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
        if (e != cudaSuccess) return cuda_check(e, "persistent step: shared-memory attribute");
        g_persist_max_dyn = pl.smem;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_persistent_kernel, kPT, pl.smem);
    if (e != cudaSuccess) return cuda_check(e, "persistent step: occupancy");
    if (per_sm < 1) {
        cudaFuncAttributes fa = {};
        cudaFuncGetAttributes(&fa, decode_persistent_kernel);
        return fail(I4_EUNSUPPORTED,
                    "persistent step: a CTA does not fit on an SM (%d threads, %d registers, %zu + %d bytes of "
                    "shared memory, max %d threads)",
                    kPT, fa.numRegs, fa.sharedSizeBytes, pl.smem, fa.maxThreadsPerBlock);
    }
    return I4_OK;
}

int persist_launch(const PersistArgs &a, const PersistPlan &pl, cudaStream_t stream, bool cooperative) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(kPT);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cooperative ? 1 : 0;
    return cuda_check(cudaLaunchKernelEx(&cfg, decode_persistent_kernel, a), "persistent decode step launch");
}

int read_persist_error(int reset) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_persist_error, sizeof v);
    if (e != cudaSuccess) return cuda_check(e, "reading the persistent-step error flag");
    if (reset && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_persist_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_check(e, "clearing the persistent-step error flag");
    }
    return v;
}

}  // namespace i4
