// INT4 weight-only GEMV with fused dequantisation, for the batch-1 decode step.
//
// "How To Build Your Own LLM Runtime From Scratch" ("Technical Details"):
// weight packing, INT4 dequantisation and the GEMV shapes of the decoder
// (qkv, o, gate/up, down, lm_head). Its third lesson: a byte-permute unpack
// beat __dp4a on Hopper, and the INT8-activation path was removed. Here the
// activations stay fp16 and the unpack is register-level LOP3 / byte-permute.
//
// Work split: one warp per row pair, one half-warp per row. Lane l of a half
// reads 16-byte chunks l, l+16, l+32, ... of its row (32 weights each), so a
// half-warp streams 256 contiguous bytes per step and the whole matrix is
// read exactly once with 128-bit coalesced loads. Chunk j lies in group j/4,
// so each chunk's fp32 partial is multiplied by one fp16 scale. The two
// halves are reduced with four shuffles each and lane 0 runs the epilogue.
//
// x is staged once per CTA in shared memory in the pairing the unpack
// produces: for each 8-k word, the half2 pairs (k0,k4) (k1,k5) (k2,k6) (k3,k7).
//
// Fused prologues: plain x, RMSNorm of the residual, embedding gather +
// RMSNorm. Fused epilogues: fp16 / fp32 store (+bias), residual add, qkv bias +
// RoPE + KV-page append, SiLU(gate)*up, and lm_head argmax with the on-device
// advance of the decode state.
#include <cstdarg>
#include <cstdio>

#include "common.cuh"
#include "gemv.cuh"
#include "gemv_parts.cuh"

namespace i4 {

// ---------------------------------------------------------------- kernel

template <int PRO, int EPI, int UNP, int MR>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvArgs a) {
    extern __shared__ uint4 smem[];
    __shared__ float red[32];
    const int K = a.K, nu4 = K >> 5, groups = K >> 7;
    uint4 *xs = smem;
    float *sxs = reinterpret_cast<float *>(xs + MR * 4 * nu4);

    grid_dep_wait();
    stage_x<PRO, UNP, MR>(a, xs, sxs, red, CtaGroup());
    __syncthreads();
    grid_dep_launch();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, half = lane >> 4, l16 = lane & 15;
    const int n_pairs = num_pairs<EPI>(a);
    const uint64_t pol = evict_first_policy();
    unsigned long long best = 0ull;
    constexpr int UNR = 8;

    for (int p = blockIdx.x * kGemvWarps + warp; p < n_pairs; p += gridDim.x * kGemvWarps) {
        int ra, rb;
        pair_rows<EPI>(a, p, ra, rb);
        const int row = half ? rb : ra;
        float acc[MR];
#pragma unroll
        for (int m = 0; m < MR; ++m) acc[m] = 0.f;
        if (row >= 0) {
            const uint4 *wrow = reinterpret_cast<const uint4 *>(a.w) + (size_t)row * nu4;
            const uint16_t *srow = a.s + (size_t)row * groups;
            for (int j0 = l16; j0 < nu4; j0 += 16 * UNR) {
                uint4 wv[UNR];
                float sc[UNR];
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int j = j0 + 16 * u;
                    if (j < nu4) {
                        wv[u] = ldg_stream(wrow + j, pol);
                        sc[u] = half_bits_to_float(ldg_u16(srow + (j >> 2)));
                    }
                }
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int j = j0 + 16 * u;
                    if (j < nu4) {
#pragma unroll
                        for (int m = 0; m < MR; ++m) {
                            const float d = chunk_dot<UNP>(wv[u], xs + (m * 4) * nu4 + j, nu4);
                            if constexpr (UNP == UNPACK_EXACT) {
                                acc[m] = fmaf(d, sc[u], acc[m]);
                            } else {
                                acc[m] = fmaf(d - 8.0f * sxs[m * nu4 + j], sc[u], acc[m]);
                            }
                        }
                    }
                }
            }
        }
        float vb[MR];
#pragma unroll
        for (int m = 0; m < MR; ++m) {
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
            vb[m] = __shfl_sync(0xffffffffu, acc[m], 16);
        }
        if (lane == 0) epilogue<EPI, MR>(a, p, ra, rb, acc, vb, best);
    }
    if constexpr (EPI == EPI_ARGMAX) {
        best = __shfl_sync(0xffffffffu, best, 0);
        finish_step(a, best);
    }
}

// Test export kernel: the exact unpack of the GEMV, written out as int8.
__global__ void unpack_kernel(const uint32_t *w, int8_t *q, long long n_words) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_words;
         i += (long long)gridDim.x * blockDim.x) {
        uint32_t v[4];
        unpack_word_exact(w[i], v);
        int8_t out[8];
        for (int t = 0; t < 4; ++t) {
            const __half2 h = *reinterpret_cast<const __half2 *>(&v[t]);
            out[t] = (int8_t)__half2float(__low2half(h));       // k0..k3 are the low halves
            out[t + 4] = (int8_t)__half2float(__high2half(h));  // k4..k7 the high halves
        }
        for (int t = 0; t < 8; ++t) q[i * 8 + t] = out[t];
    }
}

// ---------------------------------------------------------------- host launchers

size_t gemv_smem_bytes(int K, int mr, int unp) {
    const size_t nu4 = (size_t)K >> 5;
    return (size_t)mr * 4 * nu4 * sizeof(uint4) + (unp == UNPACK_SUBNORMAL ? (size_t)mr * nu4 * sizeof(float) : 0);
}

template <int PRO, int EPI, int UNP, int MR>
static int launch_gemv_t(const GemvArgs &a, cudaStream_t stream, bool pdl, int max_ctas) {
    auto kern = gemv_kernel<PRO, EPI, UNP, MR>;
    const size_t smem = gemv_smem_bytes(a.K, MR, UNP);
    static int configured_smem = -1;
    static int occ = 0;
    if ((int)smem > configured_smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_check(e, "gemv smem attribute");
        configured_smem = (int)smem;
        occ = 0;
    }
    if (occ == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvThreads, smem);
        if (e != cudaSuccess) return cuda_check(e, "gemv occupancy");
        if (occ < 1) return fail(I4_EUNSUPPORTED, "gemv: K=%d does not fit on an SM", a.K);
    }
    if (g_dry_run) return I4_OK;
    const int pairs = (EPI == EPI_SILU) ? a.inter : (a.N + 1) / 2;
    int grid = (pairs + kGemvWarps - 1) / kGemvWarps;
    int cap = kNumSMs * occ;
    if (max_ctas > 0 && max_ctas < cap) cap = max_ctas;
    if (grid > cap) grid = cap;
    if (EPI == EPI_ARGMAX && grid > kNumSMs * occ) grid = kNumSMs * occ;
    return cuda_check(launch(kern, dim3(grid), dim3(kGemvThreads), smem, stream, pdl, a), "gemv launch");
}

template <int PRO, int EPI, int UNP>
static int launch_gemv_mr(const GemvArgs &a, cudaStream_t stream, bool pdl, int max_ctas) {
    if (a.M <= 1) return launch_gemv_t<PRO, EPI, UNP, 1>(a, stream, pdl, max_ctas);
    if constexpr (PRO == PRO_PLAIN && (EPI == EPI_F16 || EPI == EPI_F32)) {
        if (a.M <= 2) return launch_gemv_t<PRO, EPI, UNP, 2>(a, stream, pdl, max_ctas);
        if (a.M <= 4) return launch_gemv_t<PRO, EPI, UNP, 4>(a, stream, pdl, max_ctas);
        return launch_gemv_t<PRO, EPI, UNP, 8>(a, stream, pdl, max_ctas);
    }
    return fail(I4_EUNSUPPORTED, "gemv: fused variants take one row");
}

template <int PRO, int EPI>
static int launch_gemv_u(const GemvArgs &a, cudaStream_t stream, bool pdl, int unp, int max_ctas) {
    if (unp == UNPACK_SUBNORMAL) return launch_gemv_mr<PRO, EPI, UNPACK_SUBNORMAL>(a, stream, pdl, max_ctas);
    return launch_gemv_mr<PRO, EPI, UNPACK_EXACT>(a, stream, pdl, max_ctas);
}

int g_default_unpack = UNPACK_AUTO;

int launch_gemv(int pro, int epi, const GemvArgs &a, cudaStream_t stream, bool pdl, int unp, int max_ctas) {
    if (unp < 0) unp = g_default_unpack;
    if (unp == UNPACK_AUTO) unp = a.M <= 8 ? UNPACK_MMA : UNPACK_EXACT;
    StreamGeom geo;
    if (max_ctas == 0 && stream_geometry(epi, a, geo, unp)) return launch_gemv_stream(pro, epi, a, geo, stream, pdl, unp);
    if (unp == UNPACK_DP4A) return fail(I4_EUNSUPPORTED, "int8-activation gemv: shape outside the streaming kernel");
    if (max_ctas == 0 && unp == UNPACK_MMA && stream_geometry(epi, a, geo, UNPACK_SUBNORMAL))
        return launch_gemv_stream(pro, epi, a, geo, stream, pdl, UNPACK_SUBNORMAL);  // rows too long for 16-row tiles
    if (unp == UNPACK_MAGIC32 || unp == UNPACK_MMA) unp = UNPACK_SUBNORMAL;  // register kernel: fp16 unpacks only
    switch (pro * 16 + epi) {
        case PRO_PLAIN * 16 + EPI_F16: return launch_gemv_u<PRO_PLAIN, EPI_F16>(a, stream, pdl, unp, max_ctas);
        case PRO_PLAIN * 16 + EPI_F32: return launch_gemv_u<PRO_PLAIN, EPI_F32>(a, stream, pdl, unp, max_ctas);
        case PRO_PLAIN * 16 + EPI_RESID: return launch_gemv_u<PRO_PLAIN, EPI_RESID>(a, stream, pdl, unp, max_ctas);
        case PRO_RMSNORM * 16 + EPI_ROPE_KV:
            return launch_gemv_u<PRO_RMSNORM, EPI_ROPE_KV>(a, stream, pdl, unp, max_ctas);
        case PRO_EMBED * 16 + EPI_ROPE_KV: return launch_gemv_u<PRO_EMBED, EPI_ROPE_KV>(a, stream, pdl, unp, max_ctas);
        case PRO_RMSNORM * 16 + EPI_SILU: return launch_gemv_u<PRO_RMSNORM, EPI_SILU>(a, stream, pdl, unp, max_ctas);
        case PRO_RMSNORM * 16 + EPI_ARGMAX:
            return launch_gemv_u<PRO_RMSNORM, EPI_ARGMAX>(a, stream, pdl, unp, max_ctas);
        default: return fail(I4_EUNSUPPORTED, "gemv: no variant pro=%d epi=%d", pro, epi);
    }
}

}  // namespace i4

using namespace i4;

static int gemv_entry(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
                      int y_is_fp32, int M, int N, int K, int group, int unp, int max_ctas, cudaStream_t stream) {
    if (!w || !scales || !x || !y) return fail(I4_EINVAL, "int4_gemv: null pointer");
    if (group != 128) return fail(I4_EUNSUPPORTED, "int4_gemv: group must be 128 (got %d)", group);
    if (K <= 0 || K % 128 != 0 || K > 32768)
        return fail(I4_EINVAL, "int4_gemv: K=%d must be a positive multiple of 128 <= 32768", K);
    if (N <= 0) return fail(I4_EINVAL, "int4_gemv: N=%d", N);
    if (M < 1 || M > 8) return fail(I4_EUNSUPPORTED, "int4_gemv: M=%d outside [1, 8]", M);
    if (!aligned(w, 16) || !aligned(x, 16)) return fail(I4_EALIGN, "int4_gemv: w and x must be 16-byte aligned");
    if (!aligned(scales, 2) || (bias && !aligned(bias, 2)) || !aligned(y, y_is_fp32 ? 4 : 2))
        return fail(I4_EALIGN, "int4_gemv: scales/bias/y misaligned");
    const int mr = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
    if (gemv_smem_bytes(K, mr, UNPACK_SUBNORMAL) > 200 * 1024)
        return fail(I4_EUNSUPPORTED, "int4_gemv: M*K too large for the shared-memory x stage");
    GemvArgs a = {};
    a.w = w;
    a.s = scales;
    a.N = N;
    a.K = K;
    a.x = x;
    a.M = M;
    a.bias = bias;
    a.y = y;
    return launch_gemv(PRO_PLAIN, y_is_fp32 ? EPI_F32 : EPI_F16, a, stream, false, unp, max_ctas);
}

extern "C" int int4_gemm(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
                         int y_is_fp32, int M, int N, int K, int group, void *ws, size_t ws_bytes, void *stream);

extern "C" int int4_gemv(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
                         int y_is_fp32, int M, int N, int K, int group, void *stream) {
    // more than 8 activation rows: a dense contraction, on the tcgen05 GEMM
    if (M > 8) return int4_gemm(w, scales, x, bias, y, y_is_fp32, M, N, K, group, nullptr, 0, stream);
    return gemv_entry(w, scales, x, bias, y, y_is_fp32, M, N, K, group, -1, 0, (cudaStream_t)stream);
}

// int4_gemv with an explicit unpack variant (0 exact, 1 subnormal) and a CTA cap
// (0 = none); used by the tests and the benchmark to compare variants.
extern "C" int i4_int4_gemv_variant(const uint32_t *w, const uint16_t *scales, const uint16_t *x,
                                    const uint16_t *bias, void *y, int y_is_fp32, int M, int N, int K, int unpack,
                                    int max_ctas, void *stream) {
    if (unpack < UNPACK_EXACT || unpack > UNPACK_DP4A) return fail(I4_EINVAL, "unknown unpack variant");
    if (unpack == UNPACK_DP4A && (M != 1 || max_ctas != 0 || K % 512 != 0))
        return fail(I4_EUNSUPPORTED, "int8-activation gemv: one vector, K %% 512 == 0, the streaming kernel");
    return gemv_entry(w, scales, x, bias, y, y_is_fp32, M, N, K, 128, unpack, max_ctas, (cudaStream_t)stream);
}

extern "C" int i4_int4_unpack(const uint32_t *w, int8_t *q, int N, int K, void *stream) {
    if (!w || !q) return fail(I4_EINVAL, "i4_int4_unpack: null pointer");
    if (N <= 0 || K <= 0 || K % 8 != 0) return fail(I4_EINVAL, "i4_int4_unpack: bad shape N=%d K=%d", N, K);
    const long long words = (long long)N * (K / 8);
    const int grid = (int)((words + 255) / 256 < 4096 ? (words + 255) / 256 : 4096);
    unpack_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(w, q, words);
    return launch_check("i4_int4_unpack");
}
