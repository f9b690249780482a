// Glue kernels of a decoder layer: RMSNorm (+ residual add), RoPE + KV-page
// append, SiLU-mul, and the RoPE (cos, sin) table of the decode step.
//
// The pages of "How To Build Your Own LLM Runtime From Scratch" list these only
// by implication (a Qwen2.5 decoder, "Technical Details"); the decode step
// fuses them into its GEMVs (gemv.cu). These stand-alone forms are the public
// calls rmsnorm_rope / i4_rmsnorm / i4_rope_kv_append / silu_mul and use the
// same per-element arithmetic as the fused forms.
#include "common.cuh"
#include "gemv.cuh"
#include "gemv_parts.cuh"  // argmax_key

namespace i4 {

constexpr int kNormThreads = 256;

// One CTA per row: optional resid += x, then out = fp16(v * inv_rms * gamma).
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const uint16_t *x_in, uint16_t *resid,
                                                             const uint16_t *gamma, uint16_t *out, int H, float eps) {
    grid_dep_wait();
    __shared__ float red[32];
    const int row = blockIdx.x;
    const uint16_t *xr = x_in + (size_t)row * H;
    uint16_t *rr = resid ? resid + (size_t)row * H : nullptr;
    const int nvec = H / 8;
    float ss = 0.f;
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
        uint4 v = *reinterpret_cast<const uint4 *>(xr + 8 * c);
        if (rr) {
            const uint4 r = *reinterpret_cast<const uint4 *>(rr + 8 * c);
            const uint32_t a[4] = {r.x, r.y, r.z, r.w}, b[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
            for (int t = 0; t < 4; ++t) {
                const float2 fa = __half22float2(*reinterpret_cast<const __half2 *>(&a[t]));
                const float2 fb = __half22float2(*reinterpret_cast<const __half2 *>(&b[t]));
                const __half2 h = __floats2half2_rn(fa.x + fb.x, fa.y + fb.y);
                o[t] = *reinterpret_cast<const uint32_t *>(&h);
            }
            v = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4 *>(rr + 8 * c) = v;
        }
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        for (int t = 0; t < 4; ++t) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[t]));
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
        }
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    const float inv = 1.0f / sqrtf(tot / (float)H + eps);
    const uint16_t *src = rr ? rr : xr;  // each thread re-reads only the vectors it wrote itself
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
        const uint4 v = *reinterpret_cast<const uint4 *>(src + 8 * c);
        const uint4 gv = *reinterpret_cast<const uint4 *>(gamma + 8 * c);
        const uint32_t r[4] = {v.x, v.y, v.z, v.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
        uint32_t o[4];
        for (int t = 0; t < 4; ++t) {
            const float2 fr = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
            const float2 fg = __half22float2(*reinterpret_cast<const __half2 *>(&g[t]));
            const __half2 h = __floats2half2_rn(fr.x * inv * fg.x, fr.y * inv * fg.y);
            o[t] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(out + (size_t)row * H + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// One thread per (sequence, head, pair i): rotate q/k heads in place, append k and v.
__global__ void rope_kv_kernel(uint16_t *qkv, const int32_t *pos, int Hq, int Hkv, float theta, uint16_t *k_pool,
                               uint16_t *v_pool, const int32_t *table, int P, int max_pages) {
    grid_dep_wait();
    const int b = blockIdx.y;
    const int heads = Hq + 2 * Hkv;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= heads * 64) return;
    const int head = idx >> 6, i = idx & 63;
    int p = pos[b];
    const int max_ctx = max_pages * P;
    if (p < 0 || p >= max_ctx) return;
    uint16_t *v = qkv + ((size_t)b * heads + head) * 128;
    const float a = half_bits_to_float(v[i]), c = half_bits_to_float(v[i + 64]);
    uint16_t oa = v[i], ob = v[i + 64];
    if (head < Hq + Hkv) {
        rope_pair(a, c, rope_cos_sin(p, i, 128, (double)theta), oa, ob);
        v[i] = oa;
        v[i + 64] = ob;
    }
    if (head >= Hq && k_pool) {
        const int g = head < Hq + Hkv ? head - Hq : head - Hq - Hkv;
        uint16_t *pool = head < Hq + Hkv ? k_pool : v_pool;
        const size_t off = (((size_t)table[(size_t)b * max_pages + p / P] * Hkv + g) * P + p % P) * 128;
        pool[off + i] = oa;
        pool[off + i + 64] = ob;
    }
}

__global__ void silu_mul_kernel(const uint16_t *gu, uint16_t *out, int M, int I) {
    grid_dep_wait();
    const long long n = (long long)M * I;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long m = idx / I, i = idx - m * I;
        const float g = half_bits_to_float(gu[m * 2 * I + i]);
        const float u = half_bits_to_float(gu[m * 2 * I + I + i]);
        out[idx] = silu_mul_bits(g, u);
    }
}

__global__ void rope_table_kernel(float2 *cs, int max_ctx, int d, double theta) {
    const int half = d / 2;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < max_ctx * half; idx += gridDim.x * blockDim.x)
        cs[idx] = rope_cos_sin(idx / half, idx % half, d, theta);
}

// out[b][:] = table[clamp(tokens[b])][:], one CTA per row, 16-byte copies
__global__ void embed_gather_kernel(const uint16_t *table, const int32_t *tokens, uint16_t *out, int H, int vocab) {
    grid_dep_wait();
    const int b = blockIdx.x;
    int t = tokens[b];
    t = t < 0 ? 0 : (t >= vocab ? vocab - 1 : t);
    const uint4 *src = reinterpret_cast<const uint4 *>(table + (size_t)t * H);
    uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)b * H);
    for (int c = threadIdx.x; c < H / 8; c += blockDim.x) dst[c] = src[c];
}

// tokens[b] = argmax of logits[b][:] (lowest index among equal maxima, -0 ranks with +0); then, when
// given, pos[b] += 1 and ctx_len[b] += 1. One CTA per row.
__global__ void __launch_bounds__(256) argmax_rows_kernel(const float *logits, int32_t *tokens, int32_t *pos,
                                                          int32_t *ctx_len, int N) {
    grid_dep_wait();
    __shared__ unsigned long long best[8];
    const int b = blockIdx.x;
    const float *row = logits + (size_t)b * N;
    unsigned long long k = 0ull;
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const unsigned long long c = argmax_key(row[i], i);
        k = c > k ? c : k;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, k, o);
        k = other > k ? other : k;
    }
    if ((threadIdx.x & 31) == 0) best[threadIdx.x >> 5] = k;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) k = best[w] > k ? best[w] : k;
        tokens[b] = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
        if (pos) pos[b] += 1;
        if (ctx_len) ctx_len[b] += 1;
    }
}

int launch_rope_table(float2 *cs, int max_ctx, int d, double theta, cudaStream_t stream) {
    rope_table_kernel<<<256, 256, 0, stream>>>(cs, max_ctx, d, theta);
    return launch_check("rope table");
}

}  // namespace i4

using namespace i4;

extern "C" int i4_rmsnorm(const uint16_t *x_in, uint16_t *resid, const uint16_t *gamma, uint16_t *out, int M, int H,
                          float eps, void *stream) {
    if (!x_in || !gamma || !out) return fail(I4_EINVAL, "i4_rmsnorm: null pointer");
    if (M < 1 || H < 8 || H % 8 || H > 32768) return fail(I4_EINVAL, "i4_rmsnorm: bad sizes M=%d H=%d", M, H);
    if (!aligned(x_in, 16) || !aligned(gamma, 16) || !aligned(out, 16) || (resid && !aligned(resid, 16)))
        return fail(I4_EALIGN, "i4_rmsnorm: 16-byte alignment required");
    rmsnorm_kernel<<<M, kNormThreads, 0, (cudaStream_t)stream>>>(x_in, resid, gamma, out, H, eps);
    return launch_check("i4_rmsnorm");
}

extern "C" int i4_rope_kv_append(uint16_t *qkv, const int32_t *pos, int B, int Hq, int Hkv, int D, float theta,
                                 uint16_t *k_pool, uint16_t *v_pool, const int32_t *page_table, int page_size,
                                 int max_pages_per_seq, void *stream) {
    if (!qkv || !pos) return fail(I4_EINVAL, "i4_rope_kv_append: null pointer");
    if (D != 128) return fail(I4_EUNSUPPORTED, "i4_rope_kv_append: head_dim %d (only 128)", D);
    if (B < 1 || Hq < 1 || Hkv < 1 || B > 65535) return fail(I4_EINVAL, "i4_rope_kv_append: bad sizes");
    if (k_pool && (!v_pool || !page_table || page_size < 1 || max_pages_per_seq < 1))
        return fail(I4_EINVAL, "i4_rope_kv_append: pools need v_pool, page_table and sizes");
    const int pairs = (Hq + 2 * Hkv) * 64;
    rope_kv_kernel<<<dim3((pairs + 127) / 128, B), 128, 0, (cudaStream_t)stream>>>(
        qkv, pos, Hq, Hkv, theta, k_pool, v_pool, page_table, page_size, max_pages_per_seq);
    return launch_check("i4_rope_kv_append");
}

extern "C" int rmsnorm_rope(const i4_rmsnorm_rope_args *a, void *stream) {
    if (!a) return fail(I4_EINVAL, "rmsnorm_rope: null args");
    if (!a->x_in && !a->qkv) return fail(I4_EINVAL, "rmsnorm_rope: both parts empty");
    if (a->x_in) {
        int st = i4_rmsnorm(a->x_in, a->resid, a->gamma, a->out, a->M, a->H, a->eps, stream);
        if (st) return st;
    }
    if (a->qkv)
        return i4_rope_kv_append(a->qkv, a->pos, a->B, a->Hq, a->Hkv, a->D, a->theta, a->k_pool, a->v_pool,
                                 a->page_table, a->page_size, a->max_pages_per_seq, stream);
    return I4_OK;
}

extern "C" int silu_mul(const uint16_t *gate_up, uint16_t *out, int M, int I, void *stream) {
    if (!gate_up || !out) return fail(I4_EINVAL, "silu_mul: null pointer");
    if (M < 1 || I < 1) return fail(I4_EINVAL, "silu_mul: bad sizes M=%d I=%d", M, I);
    const long long n = (long long)M * I;
    const int grid = (int)((n + 255) / 256 < 4 * kNumSMs ? (n + 255) / 256 : 4 * kNumSMs);
    silu_mul_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(gate_up, out, M, I);
    return launch_check("silu_mul");
}

extern "C" int i4_embed_gather(const uint16_t *table, const int32_t *tokens, uint16_t *out, int B, int H, int vocab,
                               void *stream) {
    if (!table || !tokens || !out) return fail(I4_EINVAL, "i4_embed_gather: null pointer");
    if (B < 1 || B > 65535 || H < 8 || H % 8 || vocab < 1) return fail(I4_EINVAL, "i4_embed_gather: bad sizes");
    if (!aligned(table, 16) || !aligned(out, 16)) return fail(I4_EALIGN, "i4_embed_gather: 16-byte alignment required");
    embed_gather_kernel<<<B, 256, 0, (cudaStream_t)stream>>>(table, tokens, out, H, vocab);
    return launch_check("i4_embed_gather");
}

extern "C" int i4_argmax_rows(const float *logits, int32_t *tokens, int32_t *pos, int32_t *ctx_len, int B, int N,
                              void *stream) {
    if (!logits || !tokens) return fail(I4_EINVAL, "i4_argmax_rows: null pointer");
    if (B < 1 || B > 65535 || N < 1) return fail(I4_EINVAL, "i4_argmax_rows: bad sizes");
    argmax_rows_kernel<<<B, 256, 0, (cudaStream_t)stream>>>(logits, tokens, pos, ctx_len, N);
    return launch_check("i4_argmax_rows");
}
