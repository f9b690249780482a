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

// ---------------------------------------------------------------- host side

static bool g_stream_enabled = true;
static int g_stream_smem_budget = 110 * 1024;  // two CTAs per SM

void set_stream_options(int enabled, int smem_kb) {
    if (enabled >= 0) g_stream_enabled = enabled != 0;
    if (smem_kb > 0) g_stream_smem_budget = smem_kb * 1024;
}

bool stream_geometry(int epi, const GemvArgs &a, StreamGeom &g, int unp) {
    if (!g_stream_enabled || a.M != 1 || a.K % 512 != 0 || a.K > 32768 || a.N < 2) return false;
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
static int launch_stream_u(const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl, int unp) {
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
