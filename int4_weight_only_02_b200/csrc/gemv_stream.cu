// Streaming INT4 GEMV: whole weight rows move HBM -> shared memory with bulk
// asynchronous copies (cp.async.bulk, no tensor map, no multicast) into a ring
// of stages guarded by mbarriers; one producer thread keeps the ring full while
// eight consumer warps unpack and accumulate out of shared memory.
//
// Why: at batch 1 a GEMV is a pure weight stream ("Technical Details" of "How
// To Build Your Own LLM Runtime From Scratch": INT4 dequantisation fused into
// the decode GEMVs). Issuing loads from the consumer registers serialises
// load and compute inside each warp; here the bytes in flight per SM are the
// two CTAs' rings (~90-100 KB each), independent of the compute. The producer
// issues its first copies before the kernel waits on its predecessor
// (programmatic dependent launch), so the weight stream of kernel N+1 can start
// while kernel N drains. Two CTAs per SM, tiles of whole rows assigned in
// balanced contiguous ranges.
//
// Tiles: R = 16 rows (K <= 4096) or R = 2 rows (larger K). Row-pair epilogues
// keep both rows of a pair in one tile: consecutive rows (plain / residual /
// logits), gate row n with up row n (SiLU), and rotate-half partners i, i+64 of
// one head (RoPE). Two consumers share the producer and the tiles: the CUDA-core
// one (gemv_stream_kernel: a warp per row pair with x in registers for R = 16,
// all consumer threads splitting K with x in shared memory for R = 2) and the
// tensor-core one (gemv_tc_kernel, below). Every wait is bounded: on a timeout
// the kernel records I4 device error 1 and stops issuing work.
#include <type_traits>

#include "common.cuh"
#include "gemv.cuh"
#include "async.cuh"
#include "gemv_parts.cuh"

namespace i4 {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kStreamThreads = kConsumers + 32;  // warp 0 produces
constexpr int kMaxStages = 8;
constexpr int kWin = 8;  // tiles per epilogue window of the tensor-core consumer
constexpr int kStaticTiles = 2;  // tiles per CTA assigned before the shared counter takes over

__device__ int g_device_error = 0;

template <int EPI>
constexpr bool kPaired = (EPI == EPI_SILU || EPI == EPI_ROPE_KV);

// Global rows of tile t: stream A rows [ra0, ra0 + na), stream B rows [rb0, rb0 + nb).
template <int EPI, int R>
__device__ __forceinline__ void tile_rows(const GemvArgs &a, int t, int &ra0, int &na, int &rb0, int &nb) {
    if constexpr (EPI == EPI_SILU) {
        ra0 = t * (R / 2);
        rb0 = a.inter + ra0;
        na = nb = R / 2;
    } else if constexpr (EPI == EPI_ROPE_KV) {
        const int p0 = t * (R / 2), head = p0 >> 6, i0 = p0 & 63;
        ra0 = head * 128 + i0;
        rb0 = ra0 + 64;
        na = nb = R / 2;
    } else {
        ra0 = t * R;
        na = (a.N - ra0) < R ? (a.N - ra0) : R;
        rb0 = 0;
        nb = 0;
    }
}

template <int EPI, int R>
__device__ __forceinline__ void issue_tile(const GemvArgs &a, int t, unsigned char *stage, uint64_t *bar,
                                           uint64_t pol) {
    const int wrow = a.K >> 1, srow = a.K >> 6;
    int ra0, na, rb0, nb;
    tile_rows<EPI, R>(a, t, ra0, na, rb0, nb);
    const unsigned bytes = (unsigned)((na + nb) * (wrow + srow));
    mbar_expect_tx(bar, bytes);
    const unsigned char *w = reinterpret_cast<const unsigned char *>(a.w);
    const unsigned char *s = reinterpret_cast<const unsigned char *>(a.s);
    unsigned char *sc = stage + R * wrow;
    bulk_load(stage, w + (size_t)ra0 * wrow, na * wrow, bar, pol);
    bulk_load(sc, s + (size_t)ra0 * srow, na * srow, bar, pol);
    if (nb) {
        bulk_load(stage + na * wrow, w + (size_t)rb0 * wrow, nb * wrow, bar, pol);
        bulk_load(sc + na * srow, s + (size_t)rb0 * srow, nb * srow, bar, pol);
    }
}

constexpr int kMaxHalvesPerLane = 8;  // register-resident x: K <= 32 lanes * 8 half-chunks * 16 = 4096

template <int PRO, int EPI, int UNP, int R>
__global__ void __launch_bounds__(kStreamThreads, 2) gemv_stream_kernel(const GemvArgs a, const StreamGeom geo) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages];
    __shared__ __align__(8) uint64_t empty[kMaxStages];
    __shared__ float red[32];
    __shared__ float rowpart[2][kConsumerWarps][2];

    const int K = a.K, nhr = K >> 4, wrow = K >> 1, srow = K >> 6;
    const int S = geo.stages;
    unsigned char *ring = smem;
    uint4 *xe = reinterpret_cast<uint4 *>(smem + (size_t)S * geo.stage_bytes);
    uint4 *xo = xe + nhr;
    float *sxh = reinterpret_cast<float *>(xo + nhr);
    const float4 *xf = reinterpret_cast<const float4 *>(xe);  // fp32 unpack: K floats in place of xe/xo/sxh
    // INT8 activations: xq [K/16] uint4, sq [K/16] int, scx [K/128] float, then K fp16 of staging space
    uint4 *xq = xe;
    int *sq = reinterpret_cast<int *>(xq + nhr);
    float *scx = reinterpret_cast<float *>(sq + nhr);
    uint16_t *xtmp = reinterpret_cast<uint16_t *>(scx + (K >> 7));
    // balanced contiguous ranges: tile counts of any two CTAs differ by at most one
    const int t_begin = (int)(((long long)blockIdx.x * geo.tiles) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * geo.tiles) / gridDim.x);
    const int n_tiles = t_end - t_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    unsigned long long best = 0ull;
    if (threadIdx.x < 32) {
        // ---------------- producer: weights do not depend on earlier kernels, so no dependency wait
        if (threadIdx.x == 0) {
            const uint64_t pol = evict_first_policy();
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % S, n = i / S;
                if (n > 0 && !mbar_wait(&empty[s], (unsigned)((n - 1) & 1))) {
                    record_error(&g_device_error, 1);
                    break;
                }
                issue_tile<EPI, R>(a, t_begin + i, ring + (size_t)s * geo.stage_bytes, &full[s], pol);
            }
        }
    } else {
        // ---------------- consumers
        const NamedGroup<32, kConsumers> grp;
        grid_dep_wait();
        if constexpr (UNP == UNPACK_MAGIC32)
            stage_x_f32<PRO>(a, reinterpret_cast<float4 *>(xe), red, grp);
        else if constexpr (UNP == UNPACK_DP4A)
            stage_x_int8<PRO>(a, xq, sq, scx, xtmp, red, grp);
        else
            stage_x_halves<PRO, UNP>(a, xe, xo, sxh, red, grp);
        grp.sync();
        grid_dep_launch();
        const int c = grp.tid(), warp = c >> 5, lane = c & 31;
        bool ok = true;
        if constexpr (R == 16) {
            // one warp per row pair; lane l takes half-chunks l, l+32, ... of both rows, x kept in registers
            const int nh = nhr >> 5;
            uint4 x0[kMaxHalvesPerLane], x1[kMaxHalvesPerLane];
            float sx[kMaxHalvesPerLane];
#pragma unroll
            for (int i = 0; i < kMaxHalvesPerLane; ++i) {
                if (UNP != UNPACK_MAGIC32 && i < nh) {
                    const int h = lane + 32 * i;
                    if constexpr (UNP == UNPACK_DP4A) {  // x0: int8 x, sx: its group scale, x1.x: its integer sum
                        x0[i] = xq[h];
                        sx[i] = scx[h >> 3];
                        x1[i] = make_uint4((uint32_t)sq[h], 0u, 0u, 0u);
                    } else {
                        x0[i] = xe[h];
                        x1[i] = xo[h];
                        sx[i] = (UNP == UNPACK_SUBNORMAL) ? sxh[h] : 0.f;
                    }
                }
            }
            const int tra = kPaired<EPI> ? warp : 2 * warp, trb = kPaired<EPI> ? warp + 8 : 2 * warp + 1;
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % S, n = i / S, t = t_begin + i;
                if (ok && !mbar_wait(&full[s], (unsigned)(n & 1))) {
                    record_error(&g_device_error, 1);
                    ok = false;
                }
                int ra0, na, rb0, nb;
                tile_rows<EPI, R>(a, t, ra0, na, rb0, nb);
                const bool live = ok && trb < na + nb;
                RowAcc ra = {0.f, 0.f, 0.f}, rb = {0.f, 0.f, 0.f};
                if (live) {
                    const unsigned char *st = ring + (size_t)s * geo.stage_bytes;
                    const uint2 *wa = reinterpret_cast<const uint2 *>(st + (size_t)tra * wrow);
                    const uint2 *wb = reinterpret_cast<const uint2 *>(st + (size_t)trb * wrow);
                    const uint16_t *sa = reinterpret_cast<const uint16_t *>(st + (size_t)R * wrow + (size_t)tra * srow);
                    const uint16_t *sb = reinterpret_cast<const uint16_t *>(st + (size_t)R * wrow + (size_t)trb * srow);
#pragma unroll
                    for (int k = 0; k < kMaxHalvesPerLane; ++k) {
                        if (k < nh) {
                            const int h = lane + 32 * k;
                            if constexpr (UNP == UNPACK_MAGIC32) {
                                float4 x4[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) x4[e] = xf[4 * h + e];
                                half_acc_f32(wa[h], x4, half_bits_to_float(sa[h >> 3]), ra);
                                half_acc_f32(wb[h], x4, half_bits_to_float(sb[h >> 3]), rb);
                            } else if constexpr (UNP == UNPACK_DP4A) {
                                half_acc_dp4a(wa[h], x0[k], (int)x1[k].x, half_bits_to_float(sa[h >> 3]) * sx[k], ra);
                                half_acc_dp4a(wb[h], x0[k], (int)x1[k].x, half_bits_to_float(sb[h >> 3]) * sx[k], rb);
                            } else {
                                half_acc<UNP>(wa[h], x0[k], x1[k], half_bits_to_float(sa[h >> 3]), sx[k], ra);
                                half_acc<UNP>(wb[h], x0[k], x1[k], half_bits_to_float(sb[h >> 3]), sx[k], rb);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with the stage
                float acc_a = warp_sum(row_value<UNP>(ra));
                float acc_b = warp_sum(row_value<UNP>(rb));
                if (lane == 0 && live) {
                    const int p = t * 8 + warp;
                    int pa, pb;
                    pair_rows<EPI>(a, p, pa, pb);
                    epilogue<EPI, 1>(a, p, pa, pb, &acc_a, &acc_b, best);
                }
            }
        } else {
            // two rows per tile; all consumer threads split K, x read from shared memory once for both rows
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % S, n = i / S, t = t_begin + i;
                if (ok && !mbar_wait(&full[s], (unsigned)(n & 1))) {
                    record_error(&g_device_error, 1);
                    ok = false;
                }
                RowAcc r0 = {0.f, 0.f, 0.f}, r1 = {0.f, 0.f, 0.f};
                if (ok) {
                    const unsigned char *st = ring + (size_t)s * geo.stage_bytes;
                    const uint2 *w0 = reinterpret_cast<const uint2 *>(st);
                    const uint2 *w1 = reinterpret_cast<const uint2 *>(st + wrow);
                    const uint16_t *s0 = reinterpret_cast<const uint16_t *>(st + (size_t)R * wrow);
                    const uint16_t *s1 = reinterpret_cast<const uint16_t *>(st + (size_t)R * wrow + srow);
#pragma unroll 2
                    for (int h = c; h < nhr; h += kConsumers) {
                        if constexpr (UNP == UNPACK_MAGIC32) {
                            float4 x4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) x4[e] = xf[4 * h + e];
                            half_acc_f32(w0[h], x4, half_bits_to_float(s0[h >> 3]), r0);
                            half_acc_f32(w1[h], x4, half_bits_to_float(s1[h >> 3]), r1);
                        } else if constexpr (UNP == UNPACK_DP4A) {
                            const uint4 q4 = xq[h];
                            const float g = scx[h >> 3];
                            half_acc_dp4a(w0[h], q4, sq[h], half_bits_to_float(s0[h >> 3]) * g, r0);
                            half_acc_dp4a(w1[h], q4, sq[h], half_bits_to_float(s1[h >> 3]) * g, r1);
                        } else {
                            const uint4 e = xe[h], o = xo[h];
                            const float sxv = (UNP == UNPACK_SUBNORMAL) ? sxh[h] : 0.f;
                            half_acc<UNP>(w0[h], e, o, half_bits_to_float(s0[h >> 3]), sxv, r0);
                            half_acc<UNP>(w1[h], e, o, half_bits_to_float(s1[h >> 3]), sxv, r1);
                        }
                    }
                }
                float acc0 = row_value<UNP>(r0), acc1 = row_value<UNP>(r1);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                acc0 = warp_sum(acc0);
                acc1 = warp_sum(acc1);
                if (lane == 0) {
                    rowpart[i & 1][warp][0] = acc0;
                    rowpart[i & 1][warp][1] = acc1;
                }
                grp.sync();
                if (c == 0 && ok) {
                    float v0 = 0.f, v1 = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        v0 += rowpart[i & 1][w][0];
                        v1 += rowpart[i & 1][w][1];
                    }
                    int pa, pb;
                    pair_rows<EPI>(a, t, pa, pb);
                    epilogue<EPI, 1>(a, t, pa, pb, &v0, &v1, best);
                }
            }
        }
    }
    if constexpr (EPI == EPI_ARGMAX) finish_step(a, best);
}

// ---------------------------------------------------------------- tensor-core consumer (UNPACK_MMA)
//
// Same producer, ring and tiles as above (whole rows, one bulk copy per tile
// stream), but the multiply-accumulate runs on mma.sync.m16n8k16 (fp16 in,
// fp32 accumulate) and one MMA consumes 256 weights:
//   * a warp works on a row pair (r, r'): A rows 0-7 hold row r, rows 8-15 row r';
//   * lane (g, c) = (lane / 4, lane % 4) reads 16 contiguous bytes of each row
//     (32 weights), so one 16-byte load instruction covers 512 contiguous bytes
//     of one row and never conflicts on shared-memory banks; a block is the
//     1024 weights one such load covers, and lane (g, c) of block b holds
//     k = 1024 b + 32 (4 g + c) .. + 31, all inside group 8 b + g;
//   * the lane's A fragment is its own weights (subnormal LOP3 unpack: low
//     fields u * 2^-24 into the "lo" MMA, high fields 16 u * 2^-24 into the
//     "hi" MMA) and its B fragment the x values at the same k, so B column g is
//     fed only by lanes (g, *): D[g][g] is row r's dot product over group 8b+g
//     and D[g+8][g] row r''s. Lane (g, g / 2) holds both; the other D entries
//     mix groups and are never read;
//   * per block and row: y += s * ((lo + hi / 16) * 2^24 - 8 * sum_group(x)).
// x is staged once per CTA in lane order (per block, word and lane one 16-byte
// entry: x pairs (0,4) (2,6) for the lo MMA, (1,5) (3,7) for the hi MMA), so a lane's four B loads per block are
// 16-byte loads of consecutive lanes. Long rows (K > 4096) use 2-row tiles
// whose blocks are split over the 8 consumer warps and summed in shared memory.
constexpr int kTcBlockK = 1024;

__host__ __device__ constexpr int tc_blocks(int K) { return (K + kTcBlockK - 1) / kTcBlockK; }
// staged x: [block][word 0..3][lane] uint4, then 8 * sum(x) per group (fp32)
__host__ __device__ constexpr long long tc_x_bytes(int K) { return (long long)tc_blocks(K) * 2048 + (K / 128) * 4; }

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A * B (accumulator starts at zero)
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// This CTA's share of an L2 prefetch of [base, base + bytes): 16-byte granules split
// evenly over the grid.
__device__ __forceinline__ void prefetch_share(const void *base, size_t bytes) {
    if (!base || !bytes) return;
    const size_t granules = bytes >> 4, per = (granules + gridDim.x - 1) / gridDim.x;
    const size_t g0 = (size_t)blockIdx.x * per;
    if (g0 >= granules) return;
    const size_t n = (granules - g0) < per ? (granules - g0) : per;
    const char *p = reinterpret_cast<const char *>(base) + (g0 << 4);
    for (size_t done = 0; done < n; done += (1u << 20) >> 4) {  // at most 1 MiB per instruction
        const size_t m = (n - done) < ((1u << 20) >> 4) ? (n - done) : ((1u << 20) >> 4);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p + (done << 4)), "r"((unsigned)(m << 4))
                     : "memory");
    }
}

// RMSNorm prologues: gamma words held in registers from before the dependency wait (gamma does not
// depend on the previous kernel), for rows of up to kXRegWords * 8 * 256 = 4096 weights.
constexpr int kXRegWords = 2;

// Word c of x into the lane-order layout, and the sum of its 128-weight group into sx8 (times 8):
// the 16 words of a group sit on 16 consecutive lanes of one warp (c = thread + 256 k, K % 128 == 0),
// so four xor-shuffles give the group sum. Every lane of the warp calls it (v = 0 and no store past K).
__device__ __forceinline__ void stage_word_tc(uint4 *xt, float *sx8, int c, int nwords, uint4 v) {
    float t = 0.f;
    if (c < nwords) {
        const int b = c >> 7, l = (c & 127) >> 2, w = c & 3;
        const uint4 pp = permute_pairs(v);  // (x0,x4) (x1,x5) (x2,x6) (x3,x7)
        xt[(b * 4 + w) * 32 + l] = make_uint4(pp.x, pp.z, pp.y, pp.w);
        const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[q]));
            t += f.x + f.y;
        }
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if ((threadIdx.x & 15) == 0 && c < nwords) sx8[c >> 4] = 8.0f * t;
}

// fp16(r / sqrt(mean(r^2) + eps) * gamma) of one word (fp32 math, the formula of every RMSNorm here)
__device__ __forceinline__ uint4 rmsnorm_word(uint4 rv, uint4 gv, float inv) {
    const uint32_t r[4] = {rv.x, rv.y, rv.z, rv.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t o[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 fr = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
        const float2 fg = __half22float2(*reinterpret_cast<const __half2 *>(&g[t]));
        const __half2 h = __floats2half2_rn(fr.x * inv * fg.x, fr.y * inv * fg.y);
        o[t] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ float sumsq_word(uint4 rv, float ss) {
    const uint32_t r[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
        ss = fmaf(f.x, f.x, ss);
        ss = fmaf(f.y, f.y, ss);
    }
    return ss;
}

// Stage x (plain, RMSNorm of the residual row, or RMSNorm of the embedding row) in lane order with
// its group sums. Thread t owns words t, t + 256, ...; loads are issued together before any use, so
// one memory latency covers the row (the weight copies of this kernel are already queued ahead of it).
template <int PRO, int LB, class Group>
__device__ __forceinline__ void stage_x_tc(const GemvArgs &a, uint4 *xt, float *sx8, float *red, const Group &grp,
                                           const uint4 (&gpre)[kXRegWords], uint64_t *xbar) {
    // tells the producer that this warp's loads of x are issued (the weight copies it holds back go after them)
    auto issued = [&]() {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(xbar);
    };
    const int K = a.K, nwords = K >> 3, nb = tc_blocks(K), T = grp.size(), tid = grp.tid();
    const int rounds = (nwords + T - 1) / T;
    // zero the padding past K (lanes of a partial last block read it)
    for (int i = nwords + tid; i < nb * 128; i += T) {
        const int b = i >> 7, l = (i & 127) >> 2, w = i & 3;
        xt[(b * 4 + w) * 32 + l] = make_uint4(0u, 0u, 0u, 0u);
    }
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (PRO == PRO_PLAIN) {
        for (int k0 = 0; k0 < rounds; k0 += LB) {  // LB loads in flight per thread
            uint4 v[LB];
#pragma unroll
            for (int u = 0; u < LB; ++u) {
                const int c = tid + T * (k0 + u);
                v[u] = c < nwords ? *reinterpret_cast<const uint4 *>(a.x + 8 * c) : zero;
            }
            if (k0 == 0) issued();
#pragma unroll
            for (int u = 0; u < LB; ++u)
                if (k0 + u < rounds) stage_word_tc(xt, sx8, tid + T * (k0 + u), nwords, v[u]);
        }
    } else {
        const uint16_t *src = a.x;
        if constexpr (PRO == PRO_EMBED) {
            int tok = *a.token;
            tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);
            src = a.x + (size_t)tok * K;
        }
        if (rounds <= kXRegWords) {
            uint4 r[kXRegWords];
            float ss = 0.f;
#pragma unroll
            for (int u = 0; u < kXRegWords; ++u) {
                const int c = tid + T * u;
                r[u] = c < nwords ? *reinterpret_cast<const uint4 *>(src + 8 * c) : zero;
            }
            issued();
#pragma unroll
            for (int u = 0; u < kXRegWords; ++u)
                if (tid + T * u < nwords) ss = sumsq_word(r[u], ss);
            ss = group_sum(ss, red, grp);
            const float inv = 1.0f / sqrtf(ss / (float)K + a.eps);
#pragma unroll
            for (int u = 0; u < kXRegWords; ++u) {
                const int c = tid + T * u;
                if constexpr (PRO == PRO_EMBED) {
                    if (blockIdx.x == 0 && c < nwords) *reinterpret_cast<uint4 *>(a.resid_out + 8 * c) = r[u];
                }
                if (u < rounds) stage_word_tc(xt, sx8, c, nwords, c < nwords ? rmsnorm_word(r[u], gpre[u], inv) : zero);
            }
        } else {
            float ss = 0.f;
            for (int c = tid; c < nwords; c += T) ss = sumsq_word(*reinterpret_cast<const uint4 *>(src + 8 * c), ss);
            issued();
            ss = group_sum(ss, red, grp);
            const float inv = 1.0f / sqrtf(ss / (float)K + a.eps);
            for (int k = 0; k < rounds; ++k) {
                const int c = tid + T * k;
                uint4 x = zero;
                if (c < nwords) {
                    const uint4 rv = *reinterpret_cast<const uint4 *>(src + 8 * c);
                    if constexpr (PRO == PRO_EMBED) {
                        if (blockIdx.x == 0) *reinterpret_cast<uint4 *>(a.resid_out + 8 * c) = rv;
                    }
                    x = rmsnorm_word(rv, *reinterpret_cast<const uint4 *>(a.gamma + 8 * c), inv);
                }
                stage_word_tc(xt, sx8, c, nwords, x);
            }
        }
    }
}

template <int PRO, int EPI, int R, int KC, bool DYN>
__global__ void __launch_bounds__(kStreamThreads, 2) gemv_tc_kernel(const GemvArgs a, const StreamGeom geo) {
    constexpr int PP = R / 2;               // row pairs per tile
    constexpr int WP = kConsumerWarps / PP;  // warps per row pair
    static_assert(kWin == 8 && kConsumerWarps == 8 && (WP == 1 || WP == kConsumerWarps),
                  "window flush: 8 tiles over 4-lane groups (one pair per warp) or over the 8 warps (one pair per tile)");
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages];
    __shared__ __align__(8) uint64_t empty[kMaxStages];
    __shared__ __align__(8) uint64_t xbar;  // the consumer warps have issued their loads of x
    __shared__ float red[32];
    __shared__ float2 stash[kConsumerWarps][kWin][8];  // diagonal partial sums of a window

    const int K = a.K, wrow = K >> 1, groups = K >> 7, nb = tc_blocks(K);
    const int S = geo.stages;
    unsigned char *ring = smem;
    uint4 *xt = reinterpret_cast<uint4 *>(smem + (size_t)S * geo.stage_bytes);
    float *sx8 = reinterpret_cast<float *>(xt + (size_t)nb * 128);
    __shared__ int stage_tile[kMaxStages];  // tile held by each stage; -1: no more tiles

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init(&xbar, kConsumerWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // Tile order of this CTA. Static: a contiguous balanced range. Dynamic (a.sched given): the first
    // kStaticTiles tiles c, c + G, ... then tiles claimed from a.sched[0] (offset by kStaticTiles * G)
    // until they run out, so CTAs whose memory is served faster take more of the tail; the last CTA
    // to run out resets both counters for the next launch.
    const int G = gridDim.x, c = blockIdx.x;
    const int t_begin = (int)(((long long)c * geo.tiles) / G);
    const int t_end = (int)(((long long)(c + 1) * geo.tiles) / G);
    const int n_tiles = t_end - t_begin;
    constexpr bool dyn = DYN;  // the counter pair a.sched is given
    auto static_tile = [&](int i) -> int {  // tile i of this CTA when known without the counter, else -2
        if constexpr (!DYN) return t_begin + i < t_end ? t_begin + i : -1;
        if (i < kStaticTiles) return c + i * G < geo.tiles ? c + i * G : -2;
        return -2;
    };

    unsigned long long best = 0ull;
    if (threadIdx.x < 32) {
        // ---------------- producer: weights do not depend on earlier kernels, so no dependency wait
        if (threadIdx.x == 0) {
            const uint64_t pol = evict_first_policy();
            // geo.prex stages go out at once; the rest wait until x is requested, so the loads of x
            // do not queue behind a whole ring of weight copies
            const int prex = geo.prex < S ? geo.prex : S;
            int claimed = -1;  // next counter value, requested one tile ahead so its latency overlaps a wait
            if (dyn && kStaticTiles * G >= geo.tiles) claimed = geo.tiles;  // nothing left for the counter
            // fixed ranges: exactly n_tiles stages, no end marker (the consumers know the count)
            for (int i = 0; DYN || i < n_tiles; ++i) {
                const int s = i % S, n = i / S;
                int t = static_tile(i);
                if (t == -2) {  // from the counter
                    if (claimed < 0) claimed = kStaticTiles * G + (int)atomicAdd(&a.sched[0], 1u);
                    t = claimed < geo.tiles ? claimed : -1;
                    claimed = -1;
                }
                if (i == prex && !mbar_wait(&xbar, 0u)) {
                    record_error(&g_device_error, 1);
                    break;
                }
                if (n > 0 && !mbar_wait(&empty[s], (unsigned)((n - 1) & 1))) {
                    record_error(&g_device_error, 1);
                    break;
                }
                if constexpr (DYN) {
                    stage_tile[s] = t;
                    if (t < 0) {
                        mbar_arrive(&full[s]);  // the end marker: completes the phase without bytes
                        break;
                    }
                }
                if (geo.test_stall && i == 0) continue;  // the bounded-wait test: stage 0 never fills
                issue_tile<EPI, R>(a, t, ring + (size_t)s * geo.stage_bytes, &full[s], pol);
                if constexpr (DYN) {
                    if (static_tile(i + 1) == -2 && claimed < 0)
                        claimed = kStaticTiles * G + (int)atomicAdd(&a.sched[0], 1u);
                }
                if (i == S - 1) {  // ring filled: spare DRAM time goes to the next kernel
                    prefetch_share(a.pf_a, a.pf_a_bytes);
                    prefetch_share(a.pf_b, a.pf_b_bytes);
                }
            }
            if constexpr (DYN) {
                __threadfence();
                if (atomicAdd(&a.sched[1], 1u) == (unsigned)G - 1) {  // every CTA has stopped claiming
                    a.sched[0] = 0u;
                    a.sched[1] = 0u;
                    __threadfence();
                }
            }
        }
    } else {
        // ---------------- consumers
        const NamedGroup<32, kConsumers> grp;
        uint4 gpre[kXRegWords];
#pragma unroll
        for (int u = 0; u < kXRegWords; ++u) {
            const int cw = grp.tid() + kConsumers * u;
            gpre[u] = (PRO != PRO_PLAIN && cw < (K >> 3)) ? *reinterpret_cast<const uint4 *>(a.gamma + 8 * cw)
                                                            : make_uint4(0u, 0u, 0u, 0u);
        }
        grid_dep_wait();
        const EpiCta ecta = epi_cta<EPI>(a);  // issued before the staging so its latency overlaps it
        // all of x in one round of loads when K is fixed (10 words per thread at K = 18944)
        constexpr int LB = KC > 0 ? (KC / 8 + kConsumers - 1) / kConsumers : 4;
        stage_x_tc<PRO, LB>(a, xt, sx8, red, grp, gpre, &xbar);
        grp.sync();
        grid_dep_launch();
        const int c_id = grp.tid(), warp = c_id >> 5, lane = c_id & 31;
        const int pr = warp / WP, wp = warp % WP;
        const int b0 = (wp * nb) / WP, b1 = ((wp + 1) * nb) / WP;
        const int tra = kPaired<EPI> ? pr : 2 * pr, trb = kPaired<EPI> ? pr + PP : 2 * pr + 1;
        const int g8 = lane >> 2;
        const bool diag = (lane & 3) == (g8 >> 1);  // the lane holding group g8's diagonal of the MMA
        // the lane that finishes window tile fk: lane 4 fk of each warp (one pair per warp), or lane 0 of
        // warp fk (one pair per tile, split over all warps)
        const int fk = WP == 1 ? (lane >> 2) : warp;
        const bool fin = WP == 1 ? (lane & 3) == 0 : lane == 0;
        const int fpr = WP == 1 ? pr : 0;
        const int ftrb = kPaired<EPI> ? fpr + PP : 2 * fpr + 1;
        bool ok = true, more = true;
        // Tiles go in windows of kWin: per tile only the dot products (the diagonal lanes park their
        // partial sums in shared memory); the row sums and the epilogues of a whole window follow at
        // its end, spread over lanes, so no reduction or epilogue latency sits between two tiles.
        for (int i0 = 0; (DYN ? more : i0 < n_tiles) && ok; i0 += kWin) {
            const int kn = DYN ? kWin : ((n_tiles - i0) < kWin ? (n_tiles - i0) : kWin);
            // epilogue inputs: loaded now for tiles known in advance, else as the tile arrives
            int ft = static_tile(i0 + fk), fp = 0, fpa = 0, fpb = 0;
            bool flive = false;
            EpiIn ein = {0.f, 0.f, make_float2(0.f, 0.f), 0};
            auto fin_setup = [&](int t) {
                int ra0, na, rb0, nbr;
                tile_rows<EPI, R>(a, t, ra0, na, rb0, nbr);
                fp = t * PP + fpr;
                pair_rows<EPI>(a, fp, fpa, fpb);
                flive = fin && ftrb < na + nbr;
                if (flive) ein = epi_load<EPI>(a, fp, fpa, fpb, ecta);
            };
            if (ft >= 0) fin_setup(ft);
            int nw = 0;
            for (int k = 0; k < kn; ++k) {
                const int i = i0 + k, s = i % S, n = i / S;
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (unsigned)(n & 1)));
                if (!ok) {
                    if (lane == 0) record_error(&g_device_error, 1);
                    break;
                }
                int t = t_begin + i;  // fixed ranges: known without reading the stage
                if constexpr (DYN) {
                    t = *reinterpret_cast<volatile int *>(&stage_tile[s]);
                    if (t < 0) {
                        more = false;
                        break;
                    }
                }
                if (k == fk && ft < 0) {
                    ft = t;
                    fin_setup(t);
                }
                int ra0, na, rb0, nb_rows;
                tile_rows<EPI, R>(a, t, ra0, na, rb0, nb_rows);
                float2 tot = make_float2(0.f, 0.f);
                if (trb < na + nb_rows) {
                    const unsigned char *st = ring + (size_t)s * geo.stage_bytes;
                    const uint16_t *sa = reinterpret_cast<const uint16_t *>(st + (size_t)R * wrow) + tra * groups;
                    const uint16_t *sb = reinterpret_cast<const uint16_t *>(st + (size_t)R * wrow) + trb * groups;
                    // K is a compile-time constant for the 7B shapes (KC > 0): offsets become immediates
                    tot = pair_dot<KC>(st, K, tra, trb, sa, sb, xt, sx8, b0, b1, lane);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with the stage
                if (diag) stash[warp][k][g8] = tot;
                nw = k + 1;
            }
            const bool mine = flive && ok && fk < nw;
            if constexpr (WP == 1) {
                __syncwarp();
                const int q = lane & 3;
                float2 v = make_float2(0.f, 0.f);
                if (fk < nw) {
                    const float2 u0 = stash[warp][fk][2 * q], u1 = stash[warp][fk][2 * q + 1];
                    v = make_float2(u0.x + u1.x, u0.y + u1.y);
                }
                v.x += __shfl_xor_sync(0xffffffffu, v.x, 1);
                v.y += __shfl_xor_sync(0xffffffffu, v.y, 1);
                v.x += __shfl_xor_sync(0xffffffffu, v.x, 2);
                v.y += __shfl_xor_sync(0xffffffffu, v.y, 2);
                if (mine) epilogue_in<EPI>(a, fp, fpa, fpb, v.x, v.y, ein, ecta, best);
                __syncwarp();  // the stash is rewritten by the next window
            } else {
                // every warp saw the same tiles (one pair per tile); a failed wait in one warp ends all
                const bool all_ok = bar1_and(ok), all_more = bar1_and(more);
                ok = all_ok;
                more = all_more;
                float2 v = make_float2(0.f, 0.f);
                if (fk < nw) {  // 8 warps x 8 groups of partial sums for this tile's pair
                    const float2 u0 = stash[lane >> 3][fk][lane & 7], u1 = stash[(lane >> 3) + 4][fk][lane & 7];
                    v = make_float2(u0.x + u1.x, u0.y + u1.y);
                }
                v = warp_sum2(v);
                if (mine) epilogue_in<EPI>(a, fp, fpa, fpb, v.x, v.y, ein, ecta, best);
                grp.sync();
            }
        }
        if constexpr (EPI == EPI_ARGMAX) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
                best = other > best ? other : best;
            }
        }
    }
    if constexpr (EPI == EPI_ARGMAX) finish_step(a, best);
}

// ---------------------------------------------------------------- batched tensor-core consumer (M = 2..8)
//
// y[m][n] = x[m] . w[n] for up to 8 vectors (a batch of decode steps): the 8 B
// columns of mma.m16n8k16 are the 8 vectors, the 16 A rows are 16 weight rows
// of a tile, so every D entry is useful and each unpacked weight serves the whole
// batch. Lane (g, c) reads 16 bytes (32 weights) of rows g and g + 8 per group of
// 128 weights; its B fragment is vector g's x at the same k (staged once per CTA
// in lane order; vectors past M are zero). The 8 consumer warps split the tile's
// groups and their partial sums meet in shared memory. Rows only up to 4096
// weights (the 8 staged vectors take 2 bytes x 8 x K of shared memory), one CTA
// per SM.
constexpr int kTcbBudget = 212 * 1024;  // + 8 KB of static partial sums within the 227 KB per CTA

__host__ __device__ constexpr long long tcb_x_bytes(int K) { return (long long)(K / 128) * 2048 + 8LL * (K / 128) * 4; }

template <class Group>
__device__ __forceinline__ void stage_x_tcb(const GemvArgs &a, uint4 *xb, float *sx8, const Group &grp) {
    const int groups = a.K >> 7, nwords = a.K >> 3;
    for (int i = grp.tid(); i < 8 * nwords; i += grp.size()) {  // i = vector * nwords + word
        const int n = i / nwords, wd = i % nwords;
        const int j = wd >> 4, c = (wd >> 2) & 3, w = wd & 3;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (n < a.M) {
            const uint4 pp = permute_pairs(*reinterpret_cast<const uint4 *>(a.x + (size_t)n * a.K + 8 * wd));
            v = make_uint4(pp.x, pp.z, pp.y, pp.w);  // (x0,x4) (x2,x6) | (x1,x5) (x3,x7)
        }
        xb[(j * 4 + w) * 32 + 4 * n + c] = v;
    }
    grp.sync();
    for (int i = grp.tid(); i < 8 * groups; i += grp.size()) {  // i = vector * groups + group
        const int n = i / groups, j = i % groups;
        float t = 0.f;
        for (int w = 0; w < 4; ++w)
            for (int c = 0; c < 4; ++c) {
                const uint4 e = xb[(j * 4 + w) * 32 + 4 * n + c];
                const uint32_t v[4] = {e.x, e.y, e.z, e.w};
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v[q]));
                    t += f.x + f.y;
                }
            }
        sx8[n * groups + j] = 8.0f * t;
    }
}

template <int EPI>
__global__ void __launch_bounds__(kStreamThreads, 1) gemv_tcb_kernel(const GemvArgs a, const StreamGeom geo) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages];
    __shared__ __align__(8) uint64_t empty[kMaxStages];
    __shared__ float red[2][kConsumerWarps][16][8];  // per-warp partial sums [row][vector], tile parity

    const int K = a.K, wrow = K >> 1, groups = K >> 7;
    const int S = geo.stages;
    unsigned char *ring = smem;
    uint4 *xb = reinterpret_cast<uint4 *>(smem + (size_t)S * geo.stage_bytes);
    float *sx8 = reinterpret_cast<float *>(xb + (size_t)groups * 128);
    const int t_begin = (int)(((long long)blockIdx.x * geo.tiles) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * geo.tiles) / gridDim.x);
    const int n_tiles = t_end - t_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (threadIdx.x < 32) {
        if (threadIdx.x == 0) {
            const uint64_t pol = evict_first_policy();
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % S, n = i / S;
                if (n > 0 && !mbar_wait(&empty[s], (unsigned)((n - 1) & 1))) {
                    record_error(&g_device_error, 1);
                    break;
                }
                issue_tile<EPI, 16>(a, t_begin + i, ring + (size_t)s * geo.stage_bytes, &full[s], pol);
            }
        }
        return;
    }
    const NamedGroup<32, kConsumers> grp;
    grid_dep_wait();
    stage_x_tcb(a, xb, sx8, grp);
    grp.sync();
    grid_dep_launch();
    const int c_id = grp.tid(), warp = c_id >> 5, lane = c_id & 31;
    const int g = lane >> 2, c = lane & 3;
    const int j0 = (warp * groups) / kConsumerWarps, j1 = ((warp + 1) * groups) / kConsumerWarps;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
        const int s = i % S, n = i / S, t = t_begin + i;
        if (ok && !mbar_wait(&full[s], (unsigned)(n & 1))) {
            record_error(&g_device_error, 1);
            ok = false;
        }
        const int r0 = t * 16, rows = (a.N - r0) < 16 ? (a.N - r0) : 16;
        float tot[4] = {0.f, 0.f, 0.f, 0.f};  // (row g, vec 2c) (row g, vec 2c+1) (row g+8, vec 2c) (row g+8, vec 2c+1)
        if (ok) {
            const unsigned char *st = ring + (size_t)s * geo.stage_bytes;
            // rows past the tile's end hold stale bytes: their results are never stored
            const unsigned char *wg = st + (size_t)g * wrow + 16 * c;
            const unsigned char *wg8 = st + (size_t)(g + 8) * wrow + 16 * c;
            const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + (size_t)16 * wrow);
            for (int j = j0; j < j1; ++j) {
                const uint4 qa = *reinterpret_cast<const uint4 *>(wg + 64 * j);
                const uint4 qb = *reinterpret_cast<const uint4 *>(wg8 + 64 * j);
                const uint32_t wra[4] = {qa.x, qa.y, qa.z, qa.w}, wrb[4] = {qb.x, qb.y, qb.z, qb.w};
                float lo[4], hi[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint4 xc = xb[(j * 4 + w) * 32 + lane];
                    uint32_t ua[4], ub[4];
                    unpack_word_subnormal(wra[w], ua);
                    unpack_word_subnormal(wrb[w], ub);
                    if (w == 0) {
                        mma_16816_z(lo, ua[0], ub[0], ua[2], ub[2], xc.x, xc.y);
                        mma_16816_z(hi, ua[1], ub[1], ua[3], ub[3], xc.z, xc.w);
                    } else {
                        mma_16816(lo, ua[0], ub[0], ua[2], ub[2], xc.x, xc.y);
                        mma_16816(hi, ua[1], ub[1], ua[3], ub[3], xc.z, xc.w);
                    }
                }
                const float sg = half_bits_to_float(sc[g * groups + j]), sg8 = half_bits_to_float(sc[(g + 8) * groups + j]);
                const float sxa = sx8[(2 * c) * groups + j], sxb = sx8[(2 * c + 1) * groups + j];
                tot[0] = fmaf(fmaf(hi[0], 0.0625f, lo[0]) * 16777216.0f - sxa, sg, tot[0]);
                tot[1] = fmaf(fmaf(hi[1], 0.0625f, lo[1]) * 16777216.0f - sxb, sg, tot[1]);
                tot[2] = fmaf(fmaf(hi[2], 0.0625f, lo[2]) * 16777216.0f - sxa, sg8, tot[2]);
                tot[3] = fmaf(fmaf(hi[3], 0.0625f, lo[3]) * 16777216.0f - sxb, sg8, tot[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        red[i & 1][warp][g][2 * c] = tot[0];
        red[i & 1][warp][g][2 * c + 1] = tot[1];
        red[i & 1][warp][g + 8][2 * c] = tot[2];
        red[i & 1][warp][g + 8][2 * c + 1] = tot[3];
        grp.sync();
        if (c_id < 128 && ok) {
            const int row = c_id >> 3, m = c_id & 7;
            if (row < rows && m < a.M) {
                float v = 0.f;
                for (int w = 0; w < kConsumerWarps; ++w) v += red[i & 1][w][row][m];
                if (a.bias) v += half_bits_to_float(a.bias[r0 + row]);
                if constexpr (EPI == EPI_F32)
                    reinterpret_cast<float *>(a.y)[(size_t)m * a.N + r0 + row] = v;
                else
                    reinterpret_cast<uint16_t *>(a.y)[(size_t)m * a.N + r0 + row] = float_to_half_bits(v);
            }
        }
    }
}

// ---------------------------------------------------------------- host side

static bool g_stream_enabled = true;
static int g_stream_smem_budget = 110 * 1024;  // two CTAs per SM
static int g_stream_ctas_per_sm = 2;
static int g_stream_prex = 1;
static int g_test_stall = 0;

void set_stream_options(int enabled, int smem_kb) {
    if (enabled >= 0) g_stream_enabled = enabled != 0;
    if (smem_kb > 0) g_stream_smem_budget = smem_kb * 1024;
}

void set_stream_ctas_per_sm(int n) { g_stream_ctas_per_sm = n; }
void set_stream_prex(int n) { g_stream_prex = n; }
void set_test_stall(int on) { g_test_stall = on; }

bool stream_geometry(int epi, const GemvArgs &a, StreamGeom &g, int unp) {
    g.prex = g_stream_prex;
    g.test_stall = g_test_stall;
    if (!g_stream_enabled || a.K % 512 != 0 || a.K > 32768 || a.N < 2) return false;
    if (unp == UNPACK_MMA && a.M > 1) {
        // batched tensor-core kernel: plain x, fp16/fp32 output, rows of up to 4096 weights
        if (a.M > 8 || !(epi == EPI_F16 || epi == EPI_F32) || a.K > 4096) return false;
        if (!aligned(a.w, 16) || !aligned(a.s, 16) || !aligned(a.x, 16)) return false;
        const long long wrow = a.K / 2, srow = a.K / 64;
        g.R = 16;
        g.stage_bytes = (int)(((16 * (wrow + srow)) + 127) / 128 * 128);
        const long long xs_bytes = (tcb_x_bytes(a.K) + 127) / 128 * 128;
        int stages = (int)((kTcbBudget - xs_bytes) / g.stage_bytes);
        if (stages > kMaxStages) stages = kMaxStages;
        if (stages < 2) return false;
        g.stages = stages;
        g.tiles = (a.N + 15) / 16;
        g.grid = g.tiles < kNumSMs ? g.tiles : kNumSMs;
        g.tiles_per_cta = (g.tiles + g.grid - 1) / g.grid;
        g.smem = (int)(stages * (long long)g.stage_bytes + xs_bytes);
        return true;
    }
    if (a.M != 1) return false;
    if (unp == UNPACK_MMA) {
        const bool paired = (epi == EPI_SILU || epi == EPI_ROPE_KV);
        const int R = a.K <= 32 * kMaxHalvesPerLane * 16 ? 16 : 2;
        if (paired && R != 16) return false;
        if (!paired && a.N % 2 != 0) return false;
        if (epi == EPI_SILU && a.inter % (R / 2) != 0) return false;
        if (!aligned(a.w, 16) || !aligned(a.s, 16)) return false;
        const long long wrow = a.K / 2, srow = a.K / 64;
        g.R = R;
        g.stage_bytes = (int)(((R * (wrow + srow)) + 127) / 128 * 128);
        const long long xs_bytes = (tc_x_bytes(a.K) + 127) / 128 * 128;
        int stages = (int)((g_stream_smem_budget - xs_bytes) / g.stage_bytes);
        if (stages > kMaxStages) stages = kMaxStages;
        if (stages < 2) return false;
        g.stages = stages;
        const long long pairs = (epi == EPI_SILU) ? a.inter : (long long)(a.N / 2);
        g.tiles = paired ? (int)(pairs / (R / 2)) : (a.N + R - 1) / R;
        g.grid = g.tiles < g_stream_ctas_per_sm * kNumSMs ? g.tiles : g_stream_ctas_per_sm * kNumSMs;
        g.tiles_per_cta = (g.tiles + g.grid - 1) / g.grid;
        g.smem = (int)(stages * (long long)g.stage_bytes + xs_bytes);
        return true;
    }
    const bool paired = (epi == EPI_SILU || epi == EPI_ROPE_KV);
    const int R = a.K <= 32 * kMaxHalvesPerLane * 16 ? 16 : 2;
    if (paired && R != 16) return false;
    if (!paired && a.N % 2 != 0) return false;
    if (epi == EPI_SILU && a.inter % (R / 2) != 0) return false;
    const long long wrow = a.K / 2, srow = a.K / 64;
    if (!aligned(a.w, 16) || !aligned(a.s, 16)) return false;
    g.R = R;
    g.stage_bytes = (int)(((R * (wrow + srow)) + 127) / 128 * 128);
    const long long xs_bytes =
        unp == UNPACK_MAGIC32 ? (long long)a.K * 4
        : unp == UNPACK_DP4A  ? (long long)a.K + (long long)(a.K / 16) * 4 + (long long)(a.K / 128) * 4 + (long long)a.K * 2
                              : (long long)a.K * 2 + (long long)(a.K / 16) * 4;
    long long room = g_stream_smem_budget - xs_bytes;
    int stages = (int)(room / g.stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    g.stages = stages;
    const long long pairs = (epi == EPI_SILU) ? a.inter : (long long)(a.N / 2);
    g.tiles = paired ? (int)(pairs / (R / 2)) : (a.N + R - 1) / R;
    g.grid = g.tiles < g_stream_ctas_per_sm * kNumSMs ? g.tiles : g_stream_ctas_per_sm * kNumSMs;
    g.tiles_per_cta = (g.tiles + g.grid - 1) / g.grid;
    g.smem = (int)(stages * (long long)g.stage_bytes + xs_bytes);
    return true;
}

template <int PRO, int EPI, int UNP, int R>
static int launch_stream_t(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    auto kern = gemv_stream_kernel<PRO, EPI, UNP, R>;
    static int configured = -1;
    if (geo.smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
        if (e != cudaSuccess) return cuda_check(e, "stream gemv smem attribute");
        configured = geo.smem;
    }
    if (g_dry_run) return I4_OK;
    return cuda_check(launch(kern, dim3(geo.grid), dim3(kStreamThreads), (size_t)geo.smem, stream, pdl, a, geo),
                      "stream gemv launch");
}

template <int PRO, int EPI, int UNP>
static int launch_stream_r(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    if (geo.R == 16) return launch_stream_t<PRO, EPI, UNP, 16>(a, geo, stream, pdl);
    if constexpr (EPI == EPI_SILU || EPI == EPI_ROPE_KV) {
        return fail(I4_EUNSUPPORTED, "stream gemv: paired epilogue needs 16-row tiles");
    } else {
        return launch_stream_t<PRO, EPI, UNP, 2>(a, geo, stream, pdl);
    }
}

template <int PRO, int EPI, int R, int KC, bool DYN>
static int launch_tc_kd(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    auto kern = gemv_tc_kernel<PRO, EPI, R, KC, DYN>;
    static int configured = -1;
    if (geo.smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
        if (e != cudaSuccess) return cuda_check(e, "tensor-core gemv smem attribute");
        configured = geo.smem;
    }
    if (g_dry_run) return I4_OK;
    return cuda_check(launch(kern, dim3(geo.grid), dim3(kStreamThreads), (size_t)geo.smem, stream, pdl, a, geo),
                      "tensor-core gemv launch");
}

// The shared-counter tile schedule (a.sched) is built for the residual and argmax epilogues (the down
// projection and lm_head of the decode step, where it measured faster); other launches take fixed ranges.
template <int PRO, int EPI, int R, int KC>
static int launch_tc_k(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    if constexpr (EPI == EPI_RESID || EPI == EPI_ARGMAX) {
        if (a.sched) return launch_tc_kd<PRO, EPI, R, KC, true>(a, geo, stream, pdl);
    }
    return launch_tc_kd<PRO, EPI, R, KC, false>(a, geo, stream, pdl);
}

// rows of 3584 weights (16-row tiles) and 18944 weights (2-row tiles), the decoder's two row lengths, get
// kernels with K fixed at compile time; other shapes the generic one
template <int PRO, int EPI, int R>
static int launch_tc_t(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    if constexpr (R == 16) {
        if (a.K == 3584) return launch_tc_k<PRO, EPI, R, 3584>(a, geo, stream, pdl);
    } else {
        if (a.K == 18944) return launch_tc_k<PRO, EPI, R, 18944>(a, geo, stream, pdl);
    }
    return launch_tc_k<PRO, EPI, R, 0>(a, geo, stream, pdl);
}

template <int EPI>
static int launch_tcb_t(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    auto kern = gemv_tcb_kernel<EPI>;
    static int configured = -1;
    if (geo.smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
        if (e != cudaSuccess) return cuda_check(e, "batched tensor-core gemv smem attribute");
        configured = geo.smem;
    }
    if (g_dry_run) return I4_OK;
    return cuda_check(launch(kern, dim3(geo.grid), dim3(kStreamThreads), (size_t)geo.smem, stream, pdl, a, geo),
                      "batched tensor-core gemv launch");
}

template <int PRO, int EPI>
static int launch_mma_t(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    if (a.M > 1) {
        if constexpr (PRO == PRO_PLAIN && (EPI == EPI_F16 || EPI == EPI_F32)) {
            return launch_tcb_t<EPI>(a, geo, stream, pdl);
        } else {
            return fail(I4_EUNSUPPORTED, "batched tensor-core gemv: plain prologue and fp16/fp32 output only");
        }
    }
    if (geo.R == 16) return launch_tc_t<PRO, EPI, 16>(a, geo, stream, pdl);
    if constexpr (EPI == EPI_SILU || EPI == EPI_ROPE_KV) {
        return fail(I4_EUNSUPPORTED, "tensor-core gemv: paired epilogue needs 16-row tiles");
    } else {
        return launch_tc_t<PRO, EPI, 2>(a, geo, stream, pdl);
    }
}

template <int PRO, int EPI>
static int launch_stream_u(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl, int unp) {
    if (unp == UNPACK_MMA) return launch_mma_t<PRO, EPI>(a, geo, stream, pdl);
    if (unp == UNPACK_MAGIC32) return launch_stream_r<PRO, EPI, UNPACK_MAGIC32>(a, geo, stream, pdl);
    if (unp == UNPACK_DP4A) {
        if constexpr (PRO == PRO_PLAIN && (EPI == EPI_F16 || EPI == EPI_F32))
            return launch_stream_r<PRO, EPI, UNPACK_DP4A>(a, geo, stream, pdl);
        else
            return fail(I4_EUNSUPPORTED, "int8-activation gemv: plain x and fp16/fp32 output only");
    }
    if (unp == UNPACK_SUBNORMAL) return launch_stream_r<PRO, EPI, UNPACK_SUBNORMAL>(a, geo, stream, pdl);
    return launch_stream_r<PRO, EPI, UNPACK_EXACT>(a, geo, stream, pdl);
}

int launch_gemv_stream(int pro, int epi, const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl,
                       int unp) {
    switch (pro * 16 + epi) {
        case PRO_PLAIN * 16 + EPI_F16: return launch_stream_u<PRO_PLAIN, EPI_F16>(a, geo, stream, pdl, unp);
        case PRO_PLAIN * 16 + EPI_F32: return launch_stream_u<PRO_PLAIN, EPI_F32>(a, geo, stream, pdl, unp);
        case PRO_PLAIN * 16 + EPI_RESID: return launch_stream_u<PRO_PLAIN, EPI_RESID>(a, geo, stream, pdl, unp);
        case PRO_RMSNORM * 16 + EPI_ROPE_KV:
            return launch_stream_u<PRO_RMSNORM, EPI_ROPE_KV>(a, geo, stream, pdl, unp);
        case PRO_EMBED * 16 + EPI_ROPE_KV: return launch_stream_u<PRO_EMBED, EPI_ROPE_KV>(a, geo, stream, pdl, unp);
        case PRO_RMSNORM * 16 + EPI_SILU: return launch_stream_u<PRO_RMSNORM, EPI_SILU>(a, geo, stream, pdl, unp);
        case PRO_RMSNORM * 16 + EPI_ARGMAX:
            return launch_stream_u<PRO_RMSNORM, EPI_ARGMAX>(a, geo, stream, pdl, unp);
        default: return fail(I4_EUNSUPPORTED, "stream gemv: no variant pro=%d epi=%d", pro, epi);
    }
}

int read_gemv_error(int reset) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
    if (e != cudaSuccess) return cuda_check(e, "reading the device error flag");
    if (reset && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_check(e, "clearing the device error flag");
    }
    return v;
}

int read_attn_error(int reset);
int read_persist_error(int reset);
int read_gemm_error(int reset);

}  // namespace i4

// Device-side error flag (1 = a bounded wait inside a kernel timed out). Synchronous.
extern "C" int i4_device_error(int reset) {
    const int a = i4::read_gemv_error(reset);
    const int b = i4::read_attn_error(reset);
    const int c = i4::read_persist_error(reset);
    const int d = i4::read_gemm_error(reset);
    if (a < 0) return a;
    if (b < 0) return b;
    if (c < 0) return c;
    if (d < 0) return d;
    return a ? a : (b ? b : (c ? c : d));
}
