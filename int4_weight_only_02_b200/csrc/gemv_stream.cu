// Streaming INT4 GEMV: whole weight rows move HBM -> shared memory with bulk
// asynchronous copies (cp.async.bulk, no tensor map, no multicast) into a ring
// of stages guarded by mbarriers; one producer thread keeps the ring full while
// eight consumer warps unpack and accumulate out of shared memory.
//
// Why: at batch 1 a GEMV is a pure weight stream ("Technical Details" of "How
// To Build Your Own LLM Runtime From Scratch": INT4 dequantisation fused into
// the decode GEMVs). Issuing loads from the consumer registers serialises
// load and compute inside each warp; here the bytes in flight per SM are the
// ring (up to ~190 KB), independent of the compute. The producer issues its
// first copies before the kernel waits on its predecessor (programmatic
// dependent launch), so the weight stream of kernel N+1 starts while kernel N
// drains. One CTA per SM, tiles of whole rows assigned in contiguous ranges.
//
// Tiles: R = 16 rows (K <= 4096; a warp per row pair, x in registers) or R =
// 2 rows (larger K; all consumer threads split K, x from shared memory). Row-pair epilogues keep both rows of a pair
// in one tile: consecutive rows (plain / residual / logits), gate row n with
// up row n (SiLU), and rotate-half partners i, i+64 of one head (RoPE).
// Every wait is bounded: on a timeout the kernel records I4 device error 1
// and stops issuing work.
#include "common.cuh"
#include "gemv.cuh"
#include "async.cuh"
#include "gemv_parts.cuh"

namespace i4 {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kStreamThreads = kConsumers + 32;  // warp 0 produces
constexpr int kMaxStages = 8;

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
                    x0[i] = xe[h];
                    x1[i] = xo[h];
                    sx[i] = (UNP == UNPACK_SUBNORMAL) ? sxh[h] : 0.f;
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
// Same ring, same tiles of 16 rows (K <= 4096), but the multiply-accumulate runs
// on mma.sync.m16n8k16 (fp16 in, fp32 accumulate): the 16 weight rows of a
// tile are the A operand, x (the same vector in all 8 columns of B) the B
// operand. The unpack is the LOP3 subnormal one (u = q + 8 as u * 2^-24, or
// 16u * 2^-24 for the high field of each byte), so low and high fields feed two
// accumulators; per group of 128 k a warp folds them with the row's scale:
//   y += s * ((lo + hi/16) * 2^24 - 8 * sum_group(x)).
// Seven consumer warps split the tile's groups evenly; their row sums meet in
// shared memory and eight threads run the pair epilogues. Rows are placed
// kMmaRowPad bytes apart in shared memory (one bulk copy per row) so the
// 16-byte fragment loads of two rows never hit the same banks.
constexpr int kMmaWarps = 7;
constexpr int kMmaConsumers = kMmaWarps * 32;
constexpr int kMmaThreads = kMmaConsumers + 32;
constexpr int kMmaRowPad = 64;

// Shared-memory distance between the rows of a tile: the row bytes rounded up so
// that consecutive rows start 64 bytes apart modulo 128 (two rows of one
// 16-byte fragment load then cover all 32 banks once).
__host__ __device__ constexpr int mma_row_stride(int seg) { return seg + ((64 - (seg & 127) + 128) & 127); }

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int EPI>
__device__ __forceinline__ void issue_tile_rows(const GemvArgs &a, int t, unsigned char *stage, int row_stride,
                                                uint64_t *bar, uint64_t pol) {
    const int wrow = a.K >> 1, srow = a.K >> 6;
    int ra0, na, rb0, nb;
    tile_rows<EPI, 16>(a, t, ra0, na, rb0, nb);
    mbar_expect_tx(bar, (unsigned)((na + nb) * (wrow + srow)));
    const unsigned char *w = reinterpret_cast<const unsigned char *>(a.w);
    const unsigned char *s = reinterpret_cast<const unsigned char *>(a.s);
    unsigned char *sc = stage + 16 * row_stride;
    for (int r = 0; r < na; ++r)
        bulk_load(stage + (size_t)r * row_stride, w + (size_t)(ra0 + r) * wrow, wrow, bar, pol);
    for (int r = 0; r < nb; ++r)
        bulk_load(stage + (size_t)(na + r) * row_stride, w + (size_t)(rb0 + r) * wrow, wrow, bar, pol);
    bulk_load(sc, s + (size_t)ra0 * srow, na * srow, bar, pol);
    if (nb) bulk_load(sc + na * srow, s + (size_t)rb0 * srow, nb * srow, bar, pol);
}

// x for the tensor-core consumer: for group j, slot p (0..3) and lane class c
// (0..3), xm[16j + 4p + c] = pair-permuted word 16j + 4c + p, so the four lane
// classes read 64 contiguous bytes; sxg[j] = sum of the group's 128 x values.
template <int PRO, class Group>
__device__ __forceinline__ void stage_x_mma(const GemvArgs &a, uint4 *xm, float *sxg, float *red, const Group &grp) {
    for_each_x_word<PRO>(a, red, grp, [&](int wd, uint4 v) {
        const int j = wd >> 4, c = (wd >> 2) & 3, p = wd & 3;
        xm[16 * j + 4 * p + c] = permute_pairs(v);
    });
    grp.sync();
    for (int j = grp.tid(); j < (a.K >> 7); j += grp.size()) {
        float t = 0.f;
        for (int i = 0; i < 16; ++i) {
            const uint4 e = xm[16 * j + i];
            const uint32_t v[4] = {e.x, e.y, e.z, e.w};
            for (int q = 0; q < 4; ++q) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v[q]));
                t += f.x + f.y;
            }
        }
        sxg[j] = t;
    }
}

template <int PRO, int EPI>
__global__ void __launch_bounds__(kMmaThreads, 2) gemv_mma_kernel(const GemvArgs a, const StreamGeom geo) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages];
    __shared__ __align__(8) uint64_t empty[kMaxStages];
    __shared__ float red[32];
    __shared__ float part[2][kMmaWarps][16];

    const int K = a.K, groups = K >> 7, srow = K >> 6;
    const int row_stride = mma_row_stride(K >> 1);
    const int S = geo.stages;
    unsigned char *ring = smem;
    uint4 *xm = reinterpret_cast<uint4 *>(smem + (size_t)S * geo.stage_bytes);
    float *sxg = reinterpret_cast<float *>(xm + (K >> 3));
    const int t_begin = (int)(((long long)blockIdx.x * geo.tiles) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * geo.tiles) / gridDim.x);
    const int n_tiles = t_end - t_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kMmaWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    unsigned long long best = 0ull;
    if (threadIdx.x < 32) {
        if (threadIdx.x == 0) {
            const uint64_t pol = evict_first_policy();
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % S, n = i / S;
                if (n > 0 && !mbar_wait(&empty[s], (unsigned)((n - 1) & 1))) {
                    record_error(&g_device_error, 1);
                    break;
                }
                issue_tile_rows<EPI>(a, t_begin + i, ring + (size_t)s * geo.stage_bytes, row_stride, &full[s], pol);
            }
        }
    } else {
        const NamedGroup<32, kMmaConsumers> grp;
        grid_dep_wait();
        stage_x_mma<PRO>(a, xm, sxg, red, grp);
        grp.sync();
        grid_dep_launch();
        const int c_id = grp.tid(), warp = c_id >> 5, lane = c_id & 31;
        const int g = lane >> 2, cl = lane & 3;
        const int j0 = (warp * groups) / kMmaWarps, j1 = ((warp + 1) * groups) / kMmaWarps;
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            const int s = i % S, n = i / S, t = t_begin + i;
            if (ok && !mbar_wait(&full[s], (unsigned)(n & 1))) {
                record_error(&g_device_error, 1);
                ok = false;
            }
            int ra0, na, rb0, nb;
            tile_rows<EPI, 16>(a, t, ra0, na, rb0, nb);
            const int rows = na + nb;
            const unsigned char *st = ring + (size_t)s * geo.stage_bytes;
            const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + 16 * row_stride);
            // rows past the tile's end hold stale bytes: their results are never used
            const unsigned char *wg = st + (size_t)g * row_stride;
            const unsigned char *wg8 = st + (size_t)(g + 8) * row_stride;
            float tot_g = 0.f, tot_g8 = 0.f;
            if (ok) {
                for (int j = j0; j < j1; ++j) {
                    const uint4 qa = *reinterpret_cast<const uint4 *>(wg + (size_t)(16 * j + 4 * cl) * 4);
                    const uint4 qb = *reinterpret_cast<const uint4 *>(wg8 + (size_t)(16 * j + 4 * cl) * 4);
                    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
                    float lo[4] = {0.f, 0.f, 0.f, 0.f}, hi[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint4 xc = xm[16 * j + 4 * p + cl];
                        uint32_t ua[4], ub[4];
                        unpack_word_subnormal(wa[p], ua);   // (k0,k4) (k1,k5) (k2,k6) (k3,k7)
                        unpack_word_subnormal(wb[p], ub);
                        const uint32_t alo[4] = {ua[0], ub[0], ua[2], ub[2]};  // low fields
                        const uint32_t ahi[4] = {ua[1], ub[1], ua[3], ub[3]};  // high fields (16u)
                        mma_16816(lo, alo, xc.x, xc.z);
                        mma_16816(hi, ahi, xc.y, xc.w);
                    }
                    const float sx8 = 8.0f * sxg[j];
                    const float vg = fmaf(hi[0], 0.0625f, lo[0]) * 16777216.0f - sx8;
                    const float vg8 = fmaf(hi[2], 0.0625f, lo[2]) * 16777216.0f - sx8;
                    tot_g = fmaf(vg, half_bits_to_float(sc[g * groups + j]), tot_g);
                    tot_g8 = fmaf(vg8, half_bits_to_float(sc[(g + 8) * groups + j]), tot_g8);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (cl == 0) {
                part[i & 1][warp][g] = tot_g;
                part[i & 1][warp][g + 8] = tot_g8;
            }
            grp.sync();
            if (c_id < 8 && ok) {
                const int tra = kPaired<EPI> ? c_id : 2 * c_id, trb = kPaired<EPI> ? c_id + 8 : 2 * c_id + 1;
                if (trb < rows) {
                    float va = 0.f, vb = 0.f;
                    for (int w = 0; w < kMmaWarps; ++w) {
                        va += part[i & 1][w][tra];
                        vb += part[i & 1][w][trb];
                    }
                    const int p = t * 8 + c_id;
                    int pa, pb;
                    pair_rows<EPI>(a, p, pa, pb);
                    epilogue<EPI, 1>(a, p, pa, pb, &va, &vb, best);
                }
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

// ---------------------------------------------------------------- K-split tensor-core consumer
//
// For rows too long for whole-row tiles (the MLP down projection, K = 18944):
// a work unit is one 16-row tile times one of Q slices of K (the smallest Q
// that divides the groups and keeps a stage near 40 KB; Q = 4 for K = 18944,
// 37 groups per slice). The producer copies the 16 row segments of the slice
// plus the tile's whole scale block (its rows are contiguous, so one copy; the
// per-slice part of a scale row would not be 16-byte aligned). Seven consumer
// warps run the same mma.sync loop over the slice's groups; the unit's 16 row
// sums go to a global fp32 workspace and the unit that completes a tile's Q
// slices (an arrival counter, no waiting) adds them in slice order and runs the
// epilogue, so results do not depend on timing. One CTA per SM, contiguous
// unit ranges, four-deep ring.
constexpr int kKsplitMaxStage = 48 * 1024;

static int ksplit_slices(int K) {
    const int groups = K / 128, wrow = K / 2;
    for (int q = 2; q <= 16; ++q) {
        if (groups % q) continue;
        const long long stage = 16LL * mma_row_stride(wrow / q) + 16LL * (K / 64);
        if (stage <= kKsplitMaxStage) return q;
    }
    return 0;
}

size_t ksplit_ws_bytes(int N, int K) {
    const int q = ksplit_slices(K);
    if (!q || K <= 32 * kMaxHalvesPerLane * 16) return 0;
    const size_t tiles = (size_t)(N + 15) / 16;
    const size_t cnt = (tiles * sizeof(unsigned) + 255) & ~(size_t)255;
    return cnt + tiles * q * 16 * sizeof(float);
}

template <int PRO, int EPI>
__global__ void __launch_bounds__(kMmaThreads, 1) gemv_mma_ksplit_kernel(const GemvArgs a, const StreamGeom geo,
                                                                         int Q) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages];
    __shared__ __align__(8) uint64_t empty[kMaxStages];
    __shared__ float red[32];
    __shared__ float part[2][kMmaWarps][16];

    const int K = a.K, groups = K >> 7, srow = K >> 6, wrow = K >> 1;
    const int GQ = groups / Q, seg = wrow / Q;
    const int row_stride = mma_row_stride(seg);
    const int S = geo.stages;
    unsigned char *ring = smem;
    uint4 *xm = reinterpret_cast<uint4 *>(smem + (size_t)S * geo.stage_bytes);
    float *sxg = reinterpret_cast<float *>(xm + (K >> 3));
    const int u_begin = (int)(((long long)blockIdx.x * geo.tiles) / gridDim.x);
    const int u_end = (int)(((long long)(blockIdx.x + 1) * geo.tiles) / gridDim.x);
    const int n_units = u_end - u_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kMmaWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (threadIdx.x < 32) {
        if (threadIdx.x == 0) {
            const uint64_t pol = evict_first_policy();
            const unsigned char *w = reinterpret_cast<const unsigned char *>(a.w);
            const unsigned char *sg = reinterpret_cast<const unsigned char *>(a.s);
            for (int i = 0; i < n_units; ++i) {
                const int s = i % S, n = i / S, u = u_begin + i, t = u / Q, q = u % Q;
                if (n > 0 && !mbar_wait(&empty[s], (unsigned)((n - 1) & 1))) {
                    record_error(&g_device_error, 1);
                    break;
                }
                const int r0 = t * 16, rows = (a.N - r0) < 16 ? (a.N - r0) : 16;
                unsigned char *st = ring + (size_t)s * geo.stage_bytes;
                mbar_expect_tx(&full[s], (unsigned)(rows * (seg + srow)));
                for (int r = 0; r < rows; ++r)
                    bulk_load(st + (size_t)r * row_stride, w + (size_t)(r0 + r) * wrow + (size_t)q * seg, seg, &full[s],
                              pol);
                bulk_load(st + 16 * row_stride, sg + (size_t)r0 * srow, rows * srow, &full[s], pol);
            }
        }
    } else {
        const NamedGroup<32, kMmaConsumers> grp;
        grid_dep_wait();
        stage_x_mma<PRO>(a, xm, sxg, red, grp);
        grp.sync();
        grid_dep_launch();
        const int c_id = grp.tid(), warp = c_id >> 5, lane = c_id & 31;
        const int g = lane >> 2, cl = lane & 3;
        const int jl0 = (warp * GQ) / kMmaWarps, jl1 = ((warp + 1) * GQ) / kMmaWarps;
        bool ok = true;
        unsigned long long best = 0ull;
        for (int i = 0; i < n_units; ++i) {
            const int s = i % S, n = i / S, u = u_begin + i, t = u / Q, q = u % Q;
            if (ok && !mbar_wait(&full[s], (unsigned)(n & 1))) {
                record_error(&g_device_error, 1);
                ok = false;
            }
            const int r0 = t * 16, rows = (a.N - r0) < 16 ? (a.N - r0) : 16;
            const unsigned char *st = ring + (size_t)s * geo.stage_bytes;
            const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + 16 * row_stride);
            const unsigned char *wg = st + (size_t)g * row_stride;
            const unsigned char *wg8 = st + (size_t)(g + 8) * row_stride;
            float tot_g = 0.f, tot_g8 = 0.f;
            if (ok) {
                for (int jl = jl0; jl < jl1; ++jl) {
                    const int j = q * GQ + jl;  // group index along K
                    const uint4 qa = *reinterpret_cast<const uint4 *>(wg + (size_t)(16 * jl + 4 * cl) * 4);
                    const uint4 qb = *reinterpret_cast<const uint4 *>(wg8 + (size_t)(16 * jl + 4 * cl) * 4);
                    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
                    float lo[4] = {0.f, 0.f, 0.f, 0.f}, hi[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint4 xc = xm[16 * j + 4 * p + cl];
                        uint32_t ua[4], ub[4];
                        unpack_word_subnormal(wa[p], ua);
                        unpack_word_subnormal(wb[p], ub);
                        const uint32_t alo[4] = {ua[0], ub[0], ua[2], ub[2]};
                        const uint32_t ahi[4] = {ua[1], ub[1], ua[3], ub[3]};
                        mma_16816(lo, alo, xc.x, xc.z);
                        mma_16816(hi, ahi, xc.y, xc.w);
                    }
                    const float sx8 = 8.0f * sxg[j];
                    const float vg = fmaf(hi[0], 0.0625f, lo[0]) * 16777216.0f - sx8;
                    const float vg8 = fmaf(hi[2], 0.0625f, lo[2]) * 16777216.0f - sx8;
                    tot_g = fmaf(vg, half_bits_to_float(sc[g * groups + j]), tot_g);
                    tot_g8 = fmaf(vg8, half_bits_to_float(sc[(g + 8) * groups + j]), tot_g8);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (cl == 0) {
                part[i & 1][warp][g] = tot_g;
                part[i & 1][warp][g + 8] = tot_g8;
            }
            grp.sync();
            if (warp == 0) {
                // this slice's 16 row sums to the workspace, then count the tile's slices
                float *pw = a.part_ws + ((size_t)t * Q + q) * 16;
                if (lane < 16) {
                    float v = 0.f;
                    for (int w = 0; w < kMmaWarps; ++w) v += part[i & 1][w][lane];
                    pw[lane] = v;
                    __threadfence();
                }
                __syncwarp();
                unsigned prev = 0;
                if (lane == 0) prev = atomicAdd(a.tile_cnt + t, 1u);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == (unsigned)Q - 1u && ok) {
                    __threadfence();
                    if (lane < 8 && 2 * lane + 1 < rows) {
                        float va = 0.f, vb = 0.f;
                        for (int qq = 0; qq < Q; ++qq) {
                            va += __ldcg(a.part_ws + ((size_t)t * Q + qq) * 16 + 2 * lane);
                            vb += __ldcg(a.part_ws + ((size_t)t * Q + qq) * 16 + 2 * lane + 1);
                        }
                        const int p = t * 8 + lane;
                        int pa, pb;
                        pair_rows<EPI>(a, p, pa, pb);
                        epilogue<EPI, 1>(a, p, pa, pb, &va, &vb, best);
                    }
                    if (lane == 0) a.tile_cnt[t] = 0u;  // ready for the next launch
                }
            }
        }
    }
}

// ---------------------------------------------------------------- host side

static bool g_stream_enabled = true;
static int g_stream_smem_budget = 110 * 1024;  // two CTAs per SM

void set_stream_options(int enabled, int smem_kb) {
    if (enabled >= 0) g_stream_enabled = enabled != 0;
    if (smem_kb > 0) g_stream_smem_budget = smem_kb * 1024;
}

bool stream_geometry(int epi, const GemvArgs &a, StreamGeom &g, int unp) {
    if (!g_stream_enabled || a.M != 1 || a.K % 512 != 0 || a.K > 32768 || a.N < 2) return false;
    if (unp == UNPACK_MMA && a.K > 32 * kMaxHalvesPerLane * 16) {
        // long rows: K-split tensor-core kernel (plain / fp32 / residual epilogues, needs a workspace)
        const int Q = ksplit_slices(a.K);
        if (!Q || !a.part_ws || !a.tile_cnt || a.N % 2 != 0) return false;
        if (!(epi == EPI_F16 || epi == EPI_F32 || epi == EPI_RESID)) return false;
        if (!aligned(a.w, 16) || !aligned(a.s, 16)) return false;
        g.R = -Q;  // marks the K-split kernel; |R| = slices
        const long long seg = a.K / 2 / Q;
        g.stage_bytes = (int)((16LL * mma_row_stride((int)seg) + 16 * (a.K / 64) + 127) / 128 * 128);
        const long long xs_bytes = (long long)a.K * 2 + (long long)(a.K / 128) * 4;
        int stages = (int)((220 * 1024 - xs_bytes) / g.stage_bytes);
        if (stages > kMaxStages) stages = kMaxStages;
        if (stages < 2) return false;
        g.stages = stages;
        g.tiles = ((a.N + 15) / 16) * Q;  // work units
        g.grid = g.tiles < kNumSMs ? g.tiles : kNumSMs;
        g.tiles_per_cta = (g.tiles + g.grid - 1) / g.grid;
        g.smem = (int)(stages * (long long)g.stage_bytes + xs_bytes);
        return true;
    }
    if (unp == UNPACK_MMA) {
        if (a.K > 32 * kMaxHalvesPerLane * 16) return false;  // full-row tiles only
        const bool paired = (epi == EPI_SILU || epi == EPI_ROPE_KV);
        if (!paired && a.N % 2 != 0) return false;
        if (epi == EPI_SILU && a.inter % 8 != 0) return false;
        if (!aligned(a.w, 16) || !aligned(a.s, 16)) return false;
        g.R = 16;
        const long long row_stride = mma_row_stride(a.K / 2);
        g.stage_bytes = (int)((16 * row_stride + 16 * (a.K / 64) + 127) / 128 * 128);
        const long long xs_bytes = (long long)a.K * 2 + (long long)(a.K / 128) * 4;
        int stages = (int)((g_stream_smem_budget - xs_bytes) / g.stage_bytes);
        if (stages > kMaxStages) stages = kMaxStages;
        if (stages < 2) return false;
        g.stages = stages;
        const long long pairs = (epi == EPI_SILU) ? a.inter : (long long)(a.N / 2);
        g.tiles = paired ? (int)(pairs / 8) : (a.N + 15) / 16;
        g.grid = g.tiles < 2 * kNumSMs ? g.tiles : 2 * kNumSMs;
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
        unp == UNPACK_MAGIC32 ? (long long)a.K * 4 : (long long)a.K * 2 + (long long)(a.K / 16) * 4;
    long long room = g_stream_smem_budget - xs_bytes;
    int stages = (int)(room / g.stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    g.stages = stages;
    const long long pairs = (epi == EPI_SILU) ? a.inter : (long long)(a.N / 2);
    g.tiles = paired ? (int)(pairs / (R / 2)) : (a.N + R - 1) / R;
    g.grid = g.tiles < 2 * kNumSMs ? g.tiles : 2 * kNumSMs;
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

template <int PRO, int EPI>
static int launch_ksplit_t(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    if constexpr (EPI == EPI_F16 || EPI == EPI_F32 || EPI == EPI_RESID) {
        auto kern = gemv_mma_ksplit_kernel<PRO, EPI>;
        static int configured = -1;
        if (geo.smem > configured) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
            if (e != cudaSuccess) return cuda_check(e, "k-split gemv smem attribute");
            configured = geo.smem;
        }
        if (g_dry_run) return I4_OK;
        return cuda_check(
            launch(kern, dim3(geo.grid), dim3(kMmaThreads), (size_t)geo.smem, stream, pdl, a, geo, -geo.R),
            "k-split gemv launch");
    } else {
        return fail(I4_EUNSUPPORTED, "k-split gemv: epilogue not supported");
    }
}

template <int PRO, int EPI>
static int launch_mma_t(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl) {
    if (geo.R < 0) return launch_ksplit_t<PRO, EPI>(a, geo, stream, pdl);
    auto kern = gemv_mma_kernel<PRO, EPI>;
    static int configured = -1;
    if (geo.smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
        if (e != cudaSuccess) return cuda_check(e, "mma gemv smem attribute");
        configured = geo.smem;
    }
    if (g_dry_run) return I4_OK;
    return cuda_check(launch(kern, dim3(geo.grid), dim3(kMmaThreads), (size_t)geo.smem, stream, pdl, a, geo),
                      "mma gemv launch");
}

template <int PRO, int EPI>
static int launch_stream_u(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl, int unp) {
    if (unp == UNPACK_MMA) return launch_mma_t<PRO, EPI>(a, geo, stream, pdl);
    if (unp == UNPACK_MAGIC32) return launch_stream_r<PRO, EPI, UNPACK_MAGIC32>(a, geo, stream, pdl);
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

}  // namespace i4

// Device-side error flag (1 = a bounded wait inside a kernel timed out). Synchronous.
extern "C" int i4_device_error(int reset) {
    const int a = i4::read_gemv_error(reset);
    const int b = i4::read_attn_error(reset);
    if (a < 0) return a;
    if (b < 0) return b;
    return a ? a : b;
}
