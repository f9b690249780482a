// INT4 weight-only GEMM on the 5th-generation tensor cores (tcgen05, TMEM):
//   y[m][n] = sum_k W[n][k] x[m][k] (+ bias[n]),   W[n][k] = q[n][k] * s[n][k / 128]
// for many activation rows at once: batched decode (M = 8 .. 64 sequences) and
// the prompt's prefill (M = 512 tokens). "How To Build Your Own LLM Runtime
// From Scratch" ("Technical Details": INT4 dequantisation fused into the
// linear layers; the prefill of a 512-token prompt gives the time to first
// token). With M rows the weight stream is shared by M dot products, so from
// M ~ 32 on the work is a dense contraction and belongs on the tensor cores.
//
// The weights are the MMA's A operand (M = 128 weight rows per CTA) and the
// activations its B operand (N = the tokens), so one CTA computes a 128 x BN
// tile of y^T with the fp32 accumulator in tensor memory:
//   warp 0     one thread issues TMA copies per 64-wide K chunk: the raw INT4
//              rows (128 x 32 bytes) and the fp16 activation rows (BN x 128
//              bytes, 128-byte swizzle), completing on an mbarrier;
//   warps 2-9  threads t and t + 128 dequantise the two halves of weight row t
//              of the chunk into two fp16 tiles in the same 128-byte-swizzled
//              K-major layout:
//              hi = fp16(q * s) and lo = fma(q, s, -hi), the exact remainder
//              (q * s has at most 14 significant bits), so hi + lo = q * s;
//   warp 1     allocates the TMEM columns, and one thread issues
//              tcgen05.mma (kind::f16, M = 128, N = min(BN, 256), K = 16) on
//              shared-memory descriptors for both tiles into one accumulator,
//              committing each stage back to an mbarrier so its buffers can be
//              refilled;
//   warps 2-5  finally read their 32 TMEM lanes each (tcgen05.ld) and store y.
// Every product q * s * x is exact in the fp32 accumulation. When the tiles of
// a layer are too few to fill the GPU, K is split over gridDim.z CTAs: each
// writes its fp32 partial of y to the caller's workspace and a second, fully
// parallel kernel adds the partials in split order with the bias and stores y.
// No multicast; one GPU.
#include <cuda.h>

#include <mutex>

#include "async.cuh"
#include "common.cuh"
#include "gemv.cuh"
#include "gemv_parts.cuh"

namespace i4 {

constexpr int kGBM = 128;           // weight rows per CTA (MMA M)
constexpr int kGBK = 64;            // K per stage: one 128-byte row of fp16
constexpr int kGDeqWarps = 8;       // dequantisation warps: two per weight row, four words each
constexpr int kGThreads = 64 + 32 * kGDeqWarps;
constexpr int kGMaxStages = 6;
constexpr unsigned kGATile = kGBM * kGBK * 2;  // one dequantised weight tile (hi or lo), 16 KB
constexpr unsigned kGRaw = kGBM * kGBK / 2;    // raw INT4 rows, 4 KB

__device__ int g_gemm_error = 0;

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), the
// two 16-byte halves of one K = 16 step adjacent (leading byte offset 16),
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;               // leading byte offset: 16 B
    d |= (uint64_t)(1024 >> 4) << 32;     // stride byte offset: 1024 B
    d |= (uint64_t)1 << 46;               // version
    d |= (uint64_t)2 << 61;               // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, fp16 A and B, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// generic-proxy shared-memory writes become visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ bool gemm_aborted() { return *reinterpret_cast<volatile int *>(&g_gemm_error) != 0; }

// ------------------------------------------------------------------ the kernel

struct GemmArgs {
    const uint16_t *scales, *bias;
    void *y;
    int y_fp32, M, N, K, stages;
    int chunks_per_split;  // K chunks of one split (gridDim.z splits)
    float *part;           // split partials [split][M][N] fp32 (splits > 1)
};

// Dynamic shared memory per stage (1024-byte aligned): A hi 16 KB | A lo 16 KB | B tile BN x 128 B | raw INT4 4 KB.
template <int BN>
__host__ __device__ constexpr unsigned gemm_stage_bytes() {
    return 2 * kGATile + (unsigned)BN * 128u + kGRaw;
}

template <int BN>
__global__ void __launch_bounds__(kGThreads, 1)
    i4_gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                      const GemmArgs a) {
    constexpr int NMMA = BN < 256 ? BN : 256;          // N of one MMA instruction
    constexpr int NHALF = BN / NMMA;                   // instructions per K step
    constexpr unsigned TCOLS = BN < 32 ? 32 : BN;      // TMEM columns (power of two)
    constexpr unsigned XBOX = BN < 256 ? BN : 256;     // activation rows per TMA copy
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    __shared__ __align__(8) uint64_t raw_full[kGMaxStages], a_full[kGMaxStages], empty[kGMaxStages], acc_full;
    __shared__ uint32_t tmem_base;

    const int S = a.stages, K = a.K;
    const int c_begin = blockIdx.z * a.chunks_per_split;
    const int c_end = (c_begin + a.chunks_per_split) < K / kGBK ? (c_begin + a.chunks_per_split) : K / kGBK;
    const int n_chunks = c_end > c_begin ? c_end - c_begin : 0;
    const int n0 = blockIdx.x * kGBM, m0 = blockIdx.y * BN;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    auto stage_a = [&](int s) { return smem + (size_t)s * gemm_stage_bytes<BN>(); };
    auto stage_lo = [&](int s) { return stage_a(s) + kGATile; };
    auto stage_b = [&](int s) { return stage_a(s) + 2 * kGATile; };
    auto stage_raw = [&](int s) { return stage_b(s) + (size_t)BN * 128; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&raw_full[s], 1);
            mbar_init(&a_full[s], kGDeqWarps);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // the accumulator: TCOLS fp32 columns x 128 lanes
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(TCOLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            for (int c = 0; c < n_chunks; ++c) {
                const int s = c % S, use = c / S;
                if (use > 0 && !mbar_wait(&empty[s], (unsigned)((use - 1) & 1))) {
                    record_error(&g_gemm_error, 1);
                    break;
                }
                if ((c & 15) == 15 && gemm_aborted()) break;  // a global read: not on every chunk's path
                const int kc = c_begin + c;
                mbar_expect_tx(&raw_full[s], kGRaw + (unsigned)BN * 128u);
                tma_load_2d(stage_raw(s), &tm_w, kc * (kGBK / 2), n0, &raw_full[s]);
#pragma unroll
                for (int h = 0; h < BN / (int)XBOX; ++h)
                    tma_load_2d(stage_b(s) + (size_t)h * XBOX * 128, &tm_x, kc * kGBK, m0 + h * (int)XBOX, &raw_full[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(kGBM, NMMA);
            for (int c = 0; c < n_chunks; ++c) {
                const int s = c % S, use = c / S;
                if (!mbar_wait(&a_full[s], (unsigned)(use & 1)) || !mbar_wait(&raw_full[s], (unsigned)(use & 1))) {
                    record_error(&g_gemm_error, 1);
                    break;
                }
                fence_after_sync();
                const uint32_t sa = smem_u32(stage_a(s)), sl = smem_u32(stage_lo(s)), sb = smem_u32(stage_b(s));
#pragma unroll
                for (int kk = 0; kk < kGBK / 16; ++kk) {
                    const uint64_t ad = desc_sw128(sa + 32 * kk), ld = desc_sw128(sl + 32 * kk);
#pragma unroll
                    for (int h = 0; h < NHALF; ++h) {
                        const uint64_t bd = desc_sw128(sb + (uint32_t)(h * NMMA * 128) + 32 * kk);
                        umma_f16(tmem + (uint32_t)(h * NMMA), ad, bd, idesc, (c > 0 || kk > 0) ? 1 : 0);
                        umma_f16(tmem + (uint32_t)(h * NMMA), ld, bd, idesc, 1);
                    }
                }
                umma_commit(&empty[s]);  // the stage's buffers are free once these MMAs have read them
            }
            umma_commit(&acc_full);  // every MMA issued above has completed
        }
    } else {
        // ---------------- dequantisation (threads t, t + 128: the two halves of weight row t), then the
        // epilogue (warps 2-5)
        const int td = threadIdx.x - 64, t = td & 127, half = td >> 7;
        const int n = n0 + t, groups = K >> 7;
        const bool row_ok = n < a.N;
        const uint16_t *srow = a.scales + (size_t)(row_ok ? n : 0) * groups;
        uint16_t s_next = (row_ok && n_chunks > 0) ? ldg_u16(srow + (c_begin * kGBK >> 7)) : 0;
        bool ok = true;
        for (int c = 0; c < n_chunks; ++c) {
            const int s = c % S, use = c / S;
            const uint16_t sc = s_next;
            if (c + 1 < n_chunks) s_next = row_ok ? ldg_u16(srow + ((c_begin + c + 1) * kGBK >> 7)) : 0;
            if (ok && !mbar_wait(&raw_full[s], (unsigned)(use & 1))) {
                record_error(&g_gemm_error, 1);
                ok = false;
            }
            if (ok) {
                const uint4 r0 = *reinterpret_cast<const uint4 *>(stage_raw(s) + (size_t)t * 32 + 16 * half);
                const uint32_t words[4] = {r0.x, r0.y, r0.z, r0.w};
                const uint32_t s2 = (uint32_t)sc | ((uint32_t)sc << 16);
                const size_t roff = (size_t)(t >> 3) * 1024 + (size_t)(t & 7) * 128;
                unsigned char *arow = stage_a(s) + roff, *lrow = stage_lo(s) + roff;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {  // word j: k = 8j .. 8j + 7 of the chunk -> 16-byte chunk j
                    const int j = 4 * half + jj;
                    uint32_t q[4];
                    unpack_word_exact(words[jj], q);  // (k0,k4) (k1,k5) (k2,k6) (k3,k7), exact integers
                    uint32_t w[4], r[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __half2 qh = *reinterpret_cast<const __half2 *>(&q[e]);
                        const __half2 sh = *reinterpret_cast<const __half2 *>(&s2);
                        const __half2 hi = __hmul2(qh, sh);
                        const __half2 lo = __hfma2(qh, sh, __hneg2(hi));  // q * s - hi, exact
                        w[e] = *reinterpret_cast<const uint32_t *>(&hi);
                        r[e] = *reinterpret_cast<const uint32_t *>(&lo);
                    }
                    const int pos16 = (j ^ (t & 7)) << 4;
                    *reinterpret_cast<uint4 *>(arow + pos16) =
                        make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                                   __byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632));
                    *reinterpret_cast<uint4 *>(lrow + pos16) =
                        make_uint4(__byte_perm(r[0], r[1], 0x5410), __byte_perm(r[2], r[3], 0x5410),
                                   __byte_perm(r[0], r[1], 0x7632), __byte_perm(r[2], r[3], 0x7632));
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[s]);
        }
        // epilogue (warps 2-5): TMEM lane 32 * (warp % 4) + lane holds row n0 + that lane, columns = tokens m0 ..
        if (warp < 6) {
        if (!mbar_wait(&acc_full, 0u)) record_error(&g_gemm_error, 1);
        fence_after_sync();
        const int row = 32 * (warp & 3) + lane, nn = n0 + row;
        const float bias = (a.bias && nn < a.N) ? half_bits_to_float(a.bias[nn]) : 0.f;
        const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        auto store = [&](int m, float v) {
            if (a.y_fp32)
                reinterpret_cast<float *>(a.y)[(size_t)m * a.N + nn] = v + bias;
            else
                reinterpret_cast<uint16_t *>(a.y)[(size_t)m * a.N + nn] = float_to_half_bits(v + bias);
        };
        if (gridDim.z == 1) {
            if (!__any_sync(0xffffffffu, gemm_aborted())) {  // warp-uniform around the warp-wide tcgen05.ld
#pragma unroll 1
                for (int j0 = 0; j0 < BN; j0 += 16) {
                    float v[16];
                    tmem_ld16(taddr + (uint32_t)j0, v);
                    if (nn < a.N) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (m0 + j0 + i < a.M) store(m0 + j0 + i, v[i]);
                    }
                }
            }
        } else {
            // split K: this split's partial tile to the workspace, [split][m][n] fp32 (coalesced over the
            // rows n); gemm_reduce_kernel sums the splits in order afterwards
            float *mine = a.part + (size_t)blockIdx.z * a.M * a.N;
#pragma unroll 1
            for (int j0 = 0; j0 < BN; j0 += 16) {
                float v[16];
                tmem_ld16(taddr + (uint32_t)j0, v);  // warp-wide: every lane takes part
                if (nn < a.N) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (m0 + j0 + i < a.M) mine[(size_t)(m0 + j0 + i) * a.N + nn] = v[i];
                }
            }
        }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS) : "memory");
    }
}

// y[m][n] = sum_z part[z][m][n] (+ bias[n]), the splits added in order; 8 outputs per thread.
__global__ void gemm_reduce_kernel(const float *part, const uint16_t *bias, void *y, int y_fp32, int M, int N,
                                   int splits) {
    const size_t total = (size_t)M * N;
    for (size_t i = (size_t)(blockIdx.x * blockDim.x + threadIdx.x) * 8; i < total;
         i += (size_t)gridDim.x * blockDim.x * 8) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        const int n0 = (int)(i % N);
        for (int z = 0; z < splits; ++z) {
            const float *pz = part + (size_t)z * total + i;
            if (i + 8 <= total && ((reinterpret_cast<uintptr_t>(pz) & 15) == 0)) {
                const float4 u = __ldcs(reinterpret_cast<const float4 *>(pz));
                const float4 w = __ldcs(reinterpret_cast<const float4 *>(pz + 4));
                acc[0] += u.x; acc[1] += u.y; acc[2] += u.z; acc[3] += u.w;
                acc[4] += w.x; acc[5] += w.y; acc[6] += w.z; acc[7] += w.w;
            } else {
                for (int e = 0; e < 8 && i + e < total; ++e) acc[e] += __ldcs(pz + e);
            }
        }
        for (int e = 0; e < 8 && i + e < total; ++e) {
            int n = n0 + e;
            if (n >= N) n -= N;
            const float v = acc[e] + (bias ? half_bits_to_float(bias[n]) : 0.f);
            if (y_fp32)
                reinterpret_cast<float *>(y)[i + e] = v;
            else
                reinterpret_cast<uint16_t *>(y)[i + e] = float_to_half_bits(v);
        }
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 2-D tiled tensor map over a row-major [rows][cols] matrix of elem-byte elements.
static int make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(I4_ECUDA, "int4_gemm: cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (uint64_t)elem};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(I4_ECUDA, "int4_gemm: tensor map encode failed (%d)", (int)r);
    return I4_OK;
}

// Splits of K for a grid of `tiles` output tiles: enough CTAs to cover the SMs, each split at least 8 chunks.
static int gemm_splits(int tiles, int chunks, int sms) {
    int ks = (sms + tiles - 1) / tiles;
    const int cap = chunks / 8 > 1 ? chunks / 8 : 1;
    ks = ks < cap ? ks : cap;
    return ks < 1 ? 1 : ks;
}

static int gemm_bn(int M) {
    return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : M <= 256 ? 256 : 512;
}

static int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms < 1) sms = kNumSMs;
    }
    return sms;
}

size_t gemm_ws_bytes(int M, int N, int K) {
    const int BN = gemm_bn(M);
    const int tiles = ((N + kGBM - 1) / kGBM) * ((M + BN - 1) / BN);
    const int ks = gemm_splits(tiles, K / kGBK, num_sms());
    if (ks == 1) return 0;
    return (size_t)ks * M * N * sizeof(float);
}

template <int BN>
static int launch_gemm_bn(const uint32_t *w, const uint16_t *s, const uint16_t *x, const uint16_t *bias, void *y,
                          int y_fp32, int M, int N, int K, void *ws, size_t ws_bytes, cudaStream_t stream) {
    CUtensorMap tw, tx;
    int st = make_map(&tw, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)N, kGBK / 2, kGBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st) return st;
    st = make_map(&tx, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M, kGBK, BN < 256 ? BN : 256,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (st) return st;
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const unsigned per = gemm_stage_bytes<BN>();
    int stages = (int)((optin - 4096 - 1024) / per);  // 1 KB for the alignment of the dynamic base
    stages = stages > kGMaxStages ? kGMaxStages : stages;
    const int chunks = K / kGBK;
    stages = stages > chunks ? chunks : stages;
    if (stages < 1) return fail(I4_EUNSUPPORTED, "int4_gemm: tile does not fit in shared memory");
    const size_t smem = (size_t)stages * per + 1024;
    static int configured = -1;
    if ((int)smem > configured) {
        cudaError_t e =
            cudaFuncSetAttribute(i4_gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_check(e, "int4_gemm smem attribute");
        configured = (int)smem;
    }
    const int tiles_n = (N + kGBM - 1) / kGBM, tiles_m = (M + BN - 1) / BN;
    int ks = 1;
    GemmArgs a = {s, bias, y, y_fp32, M, N, K, stages, chunks, nullptr};
    if (ws) {  // split K over the caller's workspace when the tiles alone leave SMs idle
        ks = gemm_splits(tiles_n * tiles_m, chunks, num_sms());
        if (ks > 1) {
            const size_t need = gemm_ws_bytes(M, N, K);
            if (ws_bytes < need) return fail(I4_EINVAL, "int4_gemm: workspace of %zu bytes needed (got %zu)", need, ws_bytes);
            a.part = reinterpret_cast<float *>(ws);
            a.chunks_per_split = (chunks + ks - 1) / ks;
            ks = (chunks + a.chunks_per_split - 1) / a.chunks_per_split;
        }
    }
    const dim3 grid(tiles_n, tiles_m, ks);
    i4_gemm_tc_kernel<BN><<<grid, kGThreads, smem, stream>>>(tw, tx, a);
    int st2 = launch_check("int4_gemm");
    if (st2 || ks == 1) return st2;
    const size_t outs = (size_t)M * N;
    const int blocks = (int)((outs / 8 + 255) / 256) < 4 * num_sms() ? (int)((outs / 8 + 255) / 256) : 4 * num_sms();
    gemm_reduce_kernel<<<blocks > 0 ? blocks : 1, 256, 0, stream>>>(a.part, bias, y, y_fp32, M, N, ks);
    return launch_check("int4_gemm split-K reduction");
}

int launch_int4_gemm(const uint32_t *w, const uint16_t *s, const uint16_t *x, const uint16_t *bias, void *y,
                     int y_fp32, int M, int N, int K, void *ws, size_t ws_bytes, cudaStream_t stream) {
    switch (gemm_bn(M)) {
        case 16: return launch_gemm_bn<16>(w, s, x, bias, y, y_fp32, M, N, K, ws, ws_bytes, stream);
        case 32: return launch_gemm_bn<32>(w, s, x, bias, y, y_fp32, M, N, K, ws, ws_bytes, stream);
        case 64: return launch_gemm_bn<64>(w, s, x, bias, y, y_fp32, M, N, K, ws, ws_bytes, stream);
        case 128: return launch_gemm_bn<128>(w, s, x, bias, y, y_fp32, M, N, K, ws, ws_bytes, stream);
        case 256: return launch_gemm_bn<256>(w, s, x, bias, y, y_fp32, M, N, K, ws, ws_bytes, stream);
        default: return launch_gemm_bn<512>(w, s, x, bias, y, y_fp32, M, N, K, ws, ws_bytes, stream);
    }
}

int read_gemm_error(int reset) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof v);
    if (e != cudaSuccess) return cuda_check(e, "reading the GEMM error flag");
    if (reset && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_check(e, "clearing the GEMM error flag");
    }
    return v;
}

}  // namespace i4

using namespace i4;

extern "C" size_t int4_gemm_ws_bytes(int M, int N, int K) {
    if (M < 1 || N < 1 || K < 128 || K % 128) return 0;
    return gemm_ws_bytes(M, N, K);
}

extern "C" int int4_gemm(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
                         int y_is_fp32, int M, int N, int K, int group, void *ws, size_t ws_bytes, void *stream) {
    if (!w || !scales || !x || !y) return fail(I4_EINVAL, "int4_gemm: null pointer");
    if (M < 1 || N < 1 || K < 1) return fail(I4_EINVAL, "int4_gemm: M, N, K must be positive");
    if (group != 128) return fail(I4_EUNSUPPORTED, "int4_gemm: group %d (only 128)", group);
    if (K % 128) return fail(I4_EINVAL, "int4_gemm: K %% 128 != 0");
    if (K > 65536 || N > (1 << 24) || M > (1 << 20)) return fail(I4_EUNSUPPORTED, "int4_gemm: shape too large");
    if (!aligned(w, 16) || !aligned(x, 16) || !aligned(scales, 2) || !aligned(y, y_is_fp32 ? 4 : 2))
        return fail(I4_EALIGN, "int4_gemm: w and x must be 16-byte aligned");
    if (ws && !aligned(ws, 256)) return fail(I4_EALIGN, "int4_gemm: workspace must be 256-byte aligned");
    if (g_dry_run) return I4_OK;
    return launch_int4_gemm(w, scales, x, bias, y, y_is_fp32, M, N, K, ws, ws_bytes, (cudaStream_t)stream);
}
