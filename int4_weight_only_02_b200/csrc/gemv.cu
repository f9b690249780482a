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

namespace i4 {

// ---------------------------------------------------------------- unpack

// Signed 4-bit fields of one word, exactly, as fp16 pairs matching the x
// staging order: out[0] = (k0, k4), out[1] = (k1, k5), out[2] = (k2, k6), out[3] = (k3, k7).
// A single LOP3 places the field, flipped to offset-binary u = q + 8, under the
// exponent of 1024 (low fields) or as 16u under it (high fields); one f16x2
// subtract or fma then yields q exactly.
__device__ __forceinline__ void unpack_word_exact(uint32_t q, uint32_t out[4]) {
    const uint32_t q2 = q >> 8;
    const uint32_t lo = lop3_select(q, 0x000F000Fu, 0x64086408u);   // 1024 + u   (k0, k4)
    const uint32_t hi = lop3_select(q, 0x00F000F0u, 0x64806480u);   // 1024 + 16u (k1, k5)
    const uint32_t lo2 = lop3_select(q2, 0x000F000Fu, 0x64086408u); // (k2, k6)
    const uint32_t hi2 = lop3_select(q2, 0x00F000F0u, 0x64806480u); // (k3, k7)
    out[0] = hsub2_bits(lo, 0x64086408u);                 // - 1032
    out[1] = hfma2_bits(hi, 0x2C002C00u, 0xD480D480u);    // / 16 - 72
    out[2] = hsub2_bits(lo2, 0x64086408u);
    out[3] = hfma2_bits(hi2, 0x2C002C00u, 0xD480D480u);
}

// Offset-binary fields u = q + 8 as fp16 subnormals u * 2^-24 (low fields) and
// 16u * 2^-24 (high fields): one LOP3 per pair, no float op.
__device__ __forceinline__ void unpack_word_subnormal(uint32_t q, uint32_t out[4]) {
    const uint32_t q2 = q >> 8;
    out[0] = lop3_and_xor(q, 0x000F000Fu, 0x00080008u);
    out[1] = lop3_and_xor(q, 0x00F000F0u, 0x00800080u);
    out[2] = lop3_and_xor(q2, 0x000F000Fu, 0x00080008u);
    out[3] = lop3_and_xor(q2, 0x00F000F0u, 0x00800080u);
}

// sum over the 32 weights of one chunk of q * x (exact unpack) or of u * x
// (subnormal unpack; the caller subtracts 8 * sum(x)).
template <int UNP>
__device__ __forceinline__ float chunk_dot(const uint4 &wv, const uint4 *xw, int stride) {
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
    if constexpr (UNP == UNPACK_EXACT) {
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint32_t v[4];
            unpack_word_exact(words[t], v);
            const uint4 xc = xw[t * stride];
            acc = fma2_f16_f32(v[0], xc.x, acc);
            acc = fma2_f16_f32(v[1], xc.y, acc);
            acc = fma2_f16_f32(v[2], xc.z, acc);
            acc = fma2_f16_f32(v[3], xc.w, acc);
        }
        return acc;
    } else {
        float alo = 0.f, ahi = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint32_t v[4];
            unpack_word_subnormal(words[t], v);
            const uint4 xc = xw[t * stride];
            alo = fma2_f16_f32(v[0], xc.x, alo);
            ahi = fma2_f16_f32(v[1], xc.y, ahi);
            alo = fma2_f16_f32(v[2], xc.z, alo);
            ahi = fma2_f16_f32(v[3], xc.w, ahi);
        }
        return fmaf(ahi, 0.0625f, alo) * 16777216.0f;
    }
}

// ---------------------------------------------------------------- prologue

__device__ __forceinline__ uint4 permute_pairs(uint4 xv) {
    // (x0..x7) -> (x0,x4) (x1,x5) (x2,x6) (x3,x7)
    uint4 o;
    o.x = __byte_perm(xv.x, xv.z, 0x5410);
    o.y = __byte_perm(xv.x, xv.z, 0x7632);
    o.z = __byte_perm(xv.y, xv.w, 0x5410);
    o.w = __byte_perm(xv.y, xv.w, 0x7632);
    return o;
}

__device__ __forceinline__ float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    const int nw = blockDim.x >> 5;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
}

// Stage x (MR vectors of K fp16) into shared memory, pair-permuted:
// xs[m][w][j] holds word w (0..3) of chunk j (0..K/32-1); sxs[m][j] = sum of the
// chunk's 32 x values (subnormal unpack only).
template <int PRO, int UNP, int MR>
__device__ void stage_x(const GemvArgs &a, uint4 *xs, float *sxs, float *red) {
    const int K = a.K, nu4 = K >> 5, nwords = K >> 3;
    const uint16_t *src = a.x;
    if constexpr (PRO == PRO_EMBED) {
        int tok = *a.token;
        tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);
        src = a.x + (size_t)tok * K;
    }
    if constexpr (PRO == PRO_PLAIN) {
        for (int m = 0; m < MR; ++m)
            for (int c = threadIdx.x; c < nwords; c += blockDim.x) {
                uint4 xv = make_uint4(0, 0, 0, 0);
                if (m < a.M) xv = *reinterpret_cast<const uint4 *>(a.x + (size_t)m * K + 8 * c);
                xs[(m * 4 + (c & 3)) * nu4 + (c >> 2)] = permute_pairs(xv);
            }
    } else {
        // RMSNorm of the residual row: x = fp16(r / sqrt(mean(r^2) + eps) * gamma)
        float ss = 0.f;
        for (int c = threadIdx.x; c < nwords; c += blockDim.x) {
            const uint4 rv = *reinterpret_cast<const uint4 *>(src + 8 * c);
            const uint32_t r[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
        ss = block_sum(ss, red);
        const float inv = 1.0f / sqrtf(ss / (float)K + a.eps);
        for (int c = threadIdx.x; c < nwords; c += blockDim.x) {
            const uint4 rv = *reinterpret_cast<const uint4 *>(src + 8 * c);
            const uint4 gv = *reinterpret_cast<const uint4 *>(a.gamma + 8 * c);
            if constexpr (PRO == PRO_EMBED) {
                if (blockIdx.x == 0) *reinterpret_cast<uint4 *>(a.resid_out + 8 * c) = rv;
            }
            const uint32_t r[4] = {rv.x, rv.y, rv.z, rv.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t o[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 fr = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
                const float2 fg = __half22float2(*reinterpret_cast<const __half2 *>(&g[t]));
                const __half2 h = __floats2half2_rn(fr.x * inv * fg.x, fr.y * inv * fg.y);
                o[t] = *reinterpret_cast<const uint32_t *>(&h);
            }
            xs[(c & 3) * nu4 + (c >> 2)] = permute_pairs(make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
    if constexpr (UNP == UNPACK_SUBNORMAL) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < MR * nu4; idx += blockDim.x) {
            const int m = idx / nu4, j = idx - m * nu4;
            float t = 0.f;
            for (int w = 0; w < 4; ++w) {
                const uint4 xc = xs[(m * 4 + w) * nu4 + j];
                const uint32_t v[4] = {xc.x, xc.y, xc.z, xc.w};
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v[e]));
                    t += f.x + f.y;
                }
            }
            sxs[idx] = t;
        }
    }
}

// ---------------------------------------------------------------- pair mapping

template <int EPI>
__device__ __forceinline__ int num_pairs(const GemvArgs &a) {
    if constexpr (EPI == EPI_SILU) return a.inter;
    return (a.N + 1) >> 1;
}

template <int EPI>
__device__ __forceinline__ void pair_rows(const GemvArgs &a, int p, int &ra, int &rb) {
    if constexpr (EPI == EPI_ROPE_KV) {          // (i, i + 64) inside a 128-row head
        const int head = p >> 6, i = p & 63;
        ra = head * 128 + i;
        rb = ra + 64;
    } else if constexpr (EPI == EPI_SILU) {      // (gate n, up n)
        ra = p;
        rb = p + a.inter;
    } else {
        ra = 2 * p;
        rb = (2 * p + 1 < a.N) ? 2 * p + 1 : -1;
    }
}

// ---------------------------------------------------------------- epilogues

__device__ __forceinline__ float rnd16(float v) { return __half2float(__float2half_rn(v)); }

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    if (v == 0.f) v = 0.f;  // -0 ranks with +0
    uint32_t b = __float_as_uint(v);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)b << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}

template <int EPI, int MR>
__device__ __forceinline__ void epilogue(const GemvArgs &a, int p, int ra, int rb, const float *va, const float *vb,
                                         unsigned long long &best) {
    if constexpr (EPI == EPI_F16 || EPI == EPI_F32) {
        for (int m = 0; m < MR; ++m) {
            if (m >= a.M) break;
            float ya = va[m], yb = vb[m];
            if (a.bias) {
                ya += half_bits_to_float(a.bias[ra]);
                if (rb >= 0) yb += half_bits_to_float(a.bias[rb]);
            }
            if constexpr (EPI == EPI_F16) {
                uint16_t *y = reinterpret_cast<uint16_t *>(a.y) + (size_t)m * a.N;
                y[ra] = float_to_half_bits(ya);
                if (rb >= 0) y[rb] = float_to_half_bits(yb);
            } else {
                float *y = reinterpret_cast<float *>(a.y) + (size_t)m * a.N;
                y[ra] = ya;
                if (rb >= 0) y[rb] = yb;
            }
        }
    } else if constexpr (EPI == EPI_RESID) {
        uint16_t *r = reinterpret_cast<uint16_t *>(a.y);
        r[ra] = float_to_half_bits(half_bits_to_float(r[ra]) + rnd16(va[0]));
        if (rb >= 0) r[rb] = float_to_half_bits(half_bits_to_float(r[rb]) + rnd16(vb[0]));
    } else if constexpr (EPI == EPI_SILU) {
        reinterpret_cast<uint16_t *>(a.y)[p] = silu_mul_bits(rnd16(va[0]), rnd16(vb[0]));
    } else if constexpr (EPI == EPI_ROPE_KV) {
        const int head = p >> 6, i = p & 63;
        const float xa = rnd16(va[0] + half_bits_to_float(a.bias[ra]));
        const float xb = rnd16(vb[0] + half_bits_to_float(a.bias[rb]));
        int pos = *a.pos;
        if (pos < 0 || pos >= a.max_ctx) {
            if (a.status) *a.status = 2;
            return;
        }
        if (head < a.n_q + a.n_kv) {
            uint16_t oa, ob;
            rope_pair(xa, xb, a.rope_cs[(size_t)pos * 64 + i], oa, ob);
            if (head < a.n_q) {
                a.q_out[head * 128 + i] = oa;
                a.q_out[head * 128 + i + 64] = ob;
            } else {
                const int g = head - a.n_q;
                const size_t off =
                    (((size_t)a.page_table[pos / a.page_size] * a.n_kv + g) * a.page_size + pos % a.page_size) * 128;
                a.k_pool[off + i] = oa;
                a.k_pool[off + i + 64] = ob;
            }
        } else {
            const int g = head - a.n_q - a.n_kv;
            const size_t off =
                (((size_t)a.page_table[pos / a.page_size] * a.n_kv + g) * a.page_size + pos % a.page_size) * 128;
            a.v_pool[off + i] = float_to_half_bits(xa);
            a.v_pool[off + i + 64] = float_to_half_bits(xb);
        }
    } else if constexpr (EPI == EPI_ARGMAX) {
        float *lg = reinterpret_cast<float *>(a.y);
        lg[ra] = va[0];
        unsigned long long k = argmax_key(va[0], ra);
        best = k > best ? k : best;
        if (rb >= 0) {
            lg[rb] = vb[0];
            k = argmax_key(vb[0], rb);
            best = k > best ? k : best;
        }
    }
}

// Last CTA of the lm_head GEMV: pick the token and advance the sequence state.
__device__ void finish_step(const GemvArgs &a, unsigned long long cta_best) {
    __shared__ unsigned long long sbest[8];
    __shared__ int is_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sbest[warp] = cta_best;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long b = 0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) b = sbest[i] > b ? sbest[i] : b;
        atomicMax(a.best, b);
        __threadfence();
        const unsigned prev = atomicAdd(a.arrive, 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last || threadIdx.x != 0) return;
    __threadfence();
    const unsigned long long b = atomicAdd(a.best, 0ull);
    const int idx = (int)(0xFFFFFFFFu - (uint32_t)(b & 0xFFFFFFFFull));
    const int pos = *a.pos_io;
    const int np = pos + 1;
    if (np >= a.max_ctx || pos < 0) {
        if (a.status) *a.status = 1;
    } else {
        const int tok = (a.prompt && np < a.n_prompt) ? a.prompt[np] : idx;
        *a.token_io = tok;
        *a.pos_io = np;
        *a.ctx_io = np + 1;
        if (a.history) a.history[np] = tok;
    }
    *a.best = 0ull;
    *a.arrive = 0u;
    __threadfence();
}

// ---------------------------------------------------------------- kernel

template <int PRO, int EPI, int UNP, int MR>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvArgs a) {
    extern __shared__ uint4 smem[];
    __shared__ float red[32];
    const int K = a.K, nu4 = K >> 5, groups = K >> 7;
    uint4 *xs = smem;
    float *sxs = reinterpret_cast<float *>(xs + MR * 4 * nu4);

    grid_dep_wait();
    stage_x<PRO, UNP, MR>(a, xs, sxs, red);
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

int g_default_unpack = UNPACK_EXACT;

int launch_gemv(int pro, int epi, const GemvArgs &a, cudaStream_t stream, bool pdl, int unp, int max_ctas) {
    if (unp < 0) unp = g_default_unpack;
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

extern "C" int int4_gemv(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
                         int y_is_fp32, int M, int N, int K, int group, void *stream) {
    return gemv_entry(w, scales, x, bias, y, y_is_fp32, M, N, K, group, -1, 0, (cudaStream_t)stream);
}

// int4_gemv with an explicit unpack variant (0 exact, 1 subnormal) and a CTA cap
// (0 = none); used by the tests and the benchmark to compare variants.
extern "C" int i4_int4_gemv_variant(const uint32_t *w, const uint16_t *scales, const uint16_t *x,
                                    const uint16_t *bias, void *y, int y_is_fp32, int M, int N, int K, int unpack,
                                    int max_ctas, void *stream) {
    if (unpack != UNPACK_EXACT && unpack != UNPACK_SUBNORMAL) return fail(I4_EINVAL, "unknown unpack variant");
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
