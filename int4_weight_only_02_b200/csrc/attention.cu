// Paged grouped-query decode attention: split-K over KV pages with a
// log-sum-exp merge.
//
// "How To Build Your Own LLM Runtime From Scratch" ("Technical Details":
// paged KV cache and attention; lessons: a __syncthreads() inside a
// warp-specialised branch corrupted the softmax at KV-page tails). The H100
// design there was warp-specialised with TMA; at batch 1 a decode head reads
// well under 1 MB, so this kernel has no producer/consumer roles: thread 0
// issues one bulk copy (cp.async.bulk, no multicast) per K page and per V page
// of the CTA's range into shared memory, every thread then runs the same
// three phases, and every barrier is reached by the whole CTA (CTAs without
// work leave before the first barrier, as a whole).
//
// Grid (S, Hkv, B). CTA (s, g, b) takes pages [s*pps, (s+1)*pps) of sequence b
// for kv head g and all G = Hq/Hkv query heads that share it, so each K/V row
// is read once for G heads. pps is derived on the device from ctx_len[b], so a
// captured graph stays valid as the context grows. One page of one kv head is
// page_size contiguous rows of 256 bytes, so a page is one copy.
//   phase A: 16 threads per token (8 dims each), 8 tokens per pass;
//            scores = q.k * scale * log2(e) into shared memory.
//   phase B: per head, max and sum of exp2 over the CTA's tokens.
//   phase C: o[h][:] += p[h][t] * V[t][:], same thread layout as phase A.
// With one active split the CTA writes the normalised output; otherwise it
// writes (m, l, o) partials and the last CTA to arrive for (b, g) merges them:
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// Pages below the current token's page were written by earlier decode steps,
// so their copies start before the dependency wait (programmatic launch); the
// page holding position ctx-1 is copied after it.
#include <mutex>

#include "async.cuh"
#include "attention.cuh"
#include "common.cuh"

namespace i4 {

constexpr int kAttnThreads = 128;
constexpr int kMaxGroup = 8;
constexpr int kHeadDim = 128;
constexpr int kMaxTokensPerSplit = 128;
constexpr int kMinTokensPerSplit = 64;
constexpr int kMaxSplits = 256;
constexpr int kMaxCtx = kMaxSplits * kMaxTokensPerSplit;
constexpr float kLog2e = 1.4426950408889634f;

__device__ int g_attn_error = 0;

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

int attn_splits(int B, int Hkv, int page_size, int max_pages) {
    // enough CTAs to cover the SMs twice, no split above kMaxTokensPerSplit tokens
    const int max_pps = kMaxTokensPerSplit / page_size > 0 ? kMaxTokensPerSplit / page_size : 1;
    int s_min = (max_pages + max_pps - 1) / max_pps;
    int s_par = (2 * kNumSMs + B * Hkv - 1) / (B * Hkv);
    int s = s_par > s_min ? s_par : s_min;
    if (s > max_pages) s = max_pages;
    if (s > kMaxSplits) s = kMaxSplits;
    return s < 1 ? 1 : s;
}

AttnWs attn_ws_layout(int B, int Hq, int Hkv, int page_size, int max_pages) {
    AttnWs L;
    L.splits = attn_splits(B, Hkv, page_size, max_pages);
    const size_t G = (size_t)(Hq / Hkv);
    const size_t cells = (size_t)B * Hkv * L.splits * G;
    L.counters_off = 0;
    L.ml_off = align256((size_t)B * Hkv * sizeof(unsigned));
    L.acc_off = L.ml_off + align256(cells * sizeof(float2));
    L.bytes = L.acc_off + align256(cells * kHeadDim * sizeof(float));
    return L;
}

// Largest token range one CTA can be given: the shared-memory K and V tiles are this long.
static int attn_tile_tokens(const AttnParams &p) {
    const int min_pps = (kMinTokensPerSplit + p.page_size - 1) / p.page_size;
    int pps = (p.max_pages + p.splits - 1) / p.splits;
    pps = pps < min_pps ? min_pps : pps;
    return pps * p.page_size;
}

__global__ void __launch_bounds__(kAttnThreads) paged_gqa_decode_kernel(AttnParams p) {
    extern __shared__ __align__(128) unsigned char kv_smem[];
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int G = p.Hq / p.Hkv;
    const int P = p.page_size;
    const int max_ctx = p.max_pages * P;
    int ctx = p.ctx_len[b];  // written by an earlier step, never by this kernel's predecessor
    ctx = ctx < 1 ? 1 : (ctx > max_ctx ? max_ctx : ctx);
    const int n_pages = (ctx + P - 1) / P;
    const int min_pps = (kMinTokensPerSplit + P - 1) / P;
    int pps = (n_pages + p.splits - 1) / p.splits;
    pps = pps < min_pps ? min_pps : pps;
    const int active = (n_pages + pps - 1) / pps;
    if (s >= active) return;  // the whole CTA leaves; no barrier has been reached

    __shared__ float qs[kMaxGroup][kHeadDim];
    __shared__ float sc[kMaxGroup][kMaxTokensPerSplit];
    __shared__ float red[4][kMaxGroup][kHeadDim];
    __shared__ float coef[kMaxGroup][kMaxSplits];
    __shared__ float lsum[kMaxGroup][kMaxSplits];
    __shared__ float mh[kMaxGroup], lh[kMaxGroup];
    __shared__ __align__(8) uint64_t kbar, vbar;
    __shared__ int is_last;

    const int tid = threadIdx.x;
    const int p0 = s * pps;
    const int p1 = (p0 + pps) < n_pages ? (p0 + pps) : n_pages;
    const int t0 = p0 * P;
    const int t1 = (p1 * P) < ctx ? (p1 * P) : ctx;
    const int T = t1 - t0;
    const int32_t *table = p.page_table + (size_t)b * p.max_pages;
    const float qscale = p.scale * kLog2e;
    const unsigned page_bytes = (unsigned)P * kHeadDim * 2;
    unsigned char *ks = kv_smem;                                   // [tile tokens][128] fp16
    unsigned char *vs = kv_smem + (size_t)p.tile_tokens * kHeadDim * 2;
    const int last_page = n_pages - 1;                            // holds position ctx-1

    if (tid == 0) {
        mbar_init(&kbar, 1);
        mbar_init(&vbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const uint64_t pol = evict_first_policy();
    if (tid == 0) {
        mbar_expect_tx(&kbar, (unsigned)(p1 - p0) * page_bytes);
        mbar_expect_tx(&vbar, (unsigned)(p1 - p0) * page_bytes);
        for (int pg = p0; pg < p1; ++pg) {
            if (pg == last_page) continue;
            const size_t off = ((size_t)table[pg] * p.Hkv + g) * P * kHeadDim;
            bulk_load(ks + (size_t)(pg - p0) * page_bytes, p.k_pool + off, page_bytes, &kbar, pol);
            bulk_load(vs + (size_t)(pg - p0) * page_bytes, p.v_pool + off, page_bytes, &vbar, pol);
        }
    }
    grid_dep_wait();  // q and the current token's K/V row come from the preceding kernel
    if (tid == 0 && last_page >= p0 && last_page < p1) {
        const size_t off = ((size_t)table[last_page] * p.Hkv + g) * P * kHeadDim;
        bulk_load(ks + (size_t)(last_page - p0) * page_bytes, p.k_pool + off, page_bytes, &kbar, pol);
        bulk_load(vs + (size_t)(last_page - p0) * page_bytes, p.v_pool + off, page_bytes, &vbar, pol);
    }

    // q of the G heads, fp32, pre-scaled
    for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
        const int h = i / kHeadDim, d = i % kHeadDim;
        qs[h][d] = half_bits_to_float(p.q[((size_t)b * p.Hq + g * G + h) * kHeadDim + d]) * qscale;
    }
    __syncthreads();
    bool ok = mbar_wait(&kbar, 0);
    if (!ok) record_error(&g_attn_error, 1);

    const int tk = tid >> 4;         // token lane 0..7
    const int dl = tid & 15;         // 8 dims [8dl, 8dl+8)
    // ---- phase A: scores
    {
        float qr[kMaxGroup][8];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) qr[h][e] = h < G ? qs[h][8 * dl + e] : 0.f;
        // every lane runs the same passes (the shuffles below need the full warp)
        for (int tb = 0; tb < T; tb += 8) {
            const int t = tb + tk;
            const bool live = t < T;
            uint4 kv = make_uint4(0, 0, 0, 0);
            if (live && ok) kv = *reinterpret_cast<const uint4 *>(ks + ((size_t)t * kHeadDim + 8 * dl) * 2);
            const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
            float kf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&kw[e]));
                kf[2 * e] = f.x;
                kf[2 * e + 1] = f.y;
            }
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) {
                float d = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) d = fmaf(qr[h][e], kf[e], d);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                if (live && dl == 0 && h < G) sc[h][t] = d;
            }
        }
    }
    __syncthreads();

    // ---- phase B: per-head max and sum of exp2 (warp w takes heads w, w+4)
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int h = warp; h < G; h += 4) {
            float m = -INFINITY;
            for (int t = lane; t < T; t += 32) m = fmaxf(m, sc[h][t]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float l = 0.f;
            for (int t = lane; t < T; t += 32) {
                const float e = exp2f(sc[h][t] - m);
                sc[h][t] = e;
                l += e;
            }
            l = warp_sum(l);
            if (lane == 0) {
                mh[h] = m;
                lh[h] = l;
            }
        }
    }
    __syncthreads();
    if (!mbar_wait(&vbar, 0)) {
        record_error(&g_attn_error, 1);
        ok = false;
    }

    // ---- phase C: o = sum_t p_t v_t
    float acc[kMaxGroup][8];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
    for (int t = tk; t < T && ok; t += 8) {
        const uint4 vv = *reinterpret_cast<const uint4 *>(vs + ((size_t)t * kHeadDim + 8 * dl) * 2);
        const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
        float vf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&vw[e]));
            vf[2 * e] = f.x;
            vf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < G) {
                const float pt = sc[h][t];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(pt, vf[e], acc[h][e]);
            }
        }
    }
    // reduce the 8 token lanes: lanes l and l^16 share dims, then across the 4 warps
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], 16);
    const int warp = tid >> 5;
    if ((tid & 31) < 16) {
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
            if (h < G)
#pragma unroll
                for (int e = 0; e < 8; ++e) red[warp][h][8 * dl + e] = acc[h][e];
    }
    __syncthreads();

    if (active == 1) {
        for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
            const int h = i / kHeadDim, d = i % kHeadDim;
            const float o = (red[0][h][d] + red[1][h][d]) + (red[2][h][d] + red[3][h][d]);
            p.out[((size_t)b * p.Hq + g * G + h) * kHeadDim + d] = float_to_half_bits(o / lh[h]);
        }
        return;
    }

    // ---- split partials and the last-arriving merge
    const size_t cell0 = (((size_t)b * p.Hkv + g) * p.splits) * G;  // (b, g, split 0, head 0)
    float2 *ml = reinterpret_cast<float2 *>(p.ws + p.ml_off);
    float *pacc = reinterpret_cast<float *>(p.ws + p.acc_off);
    unsigned *counter = reinterpret_cast<unsigned *>(p.ws + p.counters_off) + (size_t)b * p.Hkv + g;
    for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
        const int h = i / kHeadDim, d = i % kHeadDim;
        const float o = (red[0][h][d] + red[1][h][d]) + (red[2][h][d] + red[3][h][d]);
        pacc[(cell0 + (size_t)s * G + h) * kHeadDim + d] = o;
    }
    if (tid < G) ml[cell0 + (size_t)s * G + tid] = make_float2(mh[tid], lh[tid]);
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(counter, 1u);
        is_last = (prev == (unsigned)active - 1u);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // every split's (m, l) into shared memory at once (one coalesced pass), then per head
    // (warp w takes heads w, w + 4) the maximum and the normalised weights 2^(m_j - M) / L
    for (int i = tid; i < active * G; i += kAttnThreads) {
        const float2 v = __ldcg(&ml[cell0 + i]);
        coef[i % G][i / G] = v.x;
        lsum[i % G][i / G] = v.y;
    }
    __syncthreads();
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int h = warp; h < G; h += 4) {
            float M = -INFINITY;
            for (int j = lane; j < active; j += 32) M = fmaxf(M, coef[h][j]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            float L = 0.f;
            for (int j = lane; j < active; j += 32) {
                const float w = exp2f(coef[h][j] - M);
                coef[h][j] = w;
                L = fmaf(w, lsum[h][j], L);
            }
            L = warp_sum(L);
            const float invL = 1.0f / L;
            __syncwarp();
            for (int j = lane; j < active; j += 32) coef[h][j] *= invL;
        }
    }
    __syncthreads();
    for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
        const int h = i / kHeadDim, d = i % kHeadDim;
        float o = 0.f;
#pragma unroll 16
        for (int j = 0; j < active; ++j) o = fmaf(coef[h][j], __ldcg(&pacc[(cell0 + (size_t)j * G + h) * kHeadDim + d]), o);
        p.out[((size_t)b * p.Hq + g * G + h) * kHeadDim + d] = float_to_half_bits(o);
    }
    if (tid == 0) *counter = 0u;  // ready for the next call
}

int launch_paged_gqa_decode(const AttnParams &p_in, cudaStream_t stream, bool pdl) {
    AttnParams p = p_in;
    p.tile_tokens = attn_tile_tokens(p);
    const int smem = 2 * p.tile_tokens * kHeadDim * 2;
    static int configured = -1;
    if (smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(paged_gqa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_check(e, "paged_gqa_decode smem attribute");
        configured = smem;
    }
    if (g_dry_run) return I4_OK;
    return cuda_check(launch(paged_gqa_decode_kernel, dim3(p.splits, p.Hkv, p.B), dim3(kAttnThreads), (size_t)smem,
                             stream, pdl, p),
                      "paged_gqa_decode launch");
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
    if (page_size < 8 || page_size > kMaxTokensPerSplit || (page_size & (page_size - 1)))
        return fail(I4_EUNSUPPORTED, "paged_gqa_decode: page_size %d must be a power of two in [8, %d]", page_size,
                    kMaxTokensPerSplit);
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

extern "C" int paged_gqa_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                                const int32_t *page_table, const int32_t *ctx_len, uint16_t *out, int B, int Hq,
                                int Hkv, int D, int page_size, int max_pages_per_seq, float scale, void *ws,
                                size_t ws_bytes, void *stream) {
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
    p.Hkv = Hkv;
    p.page_size = page_size;
    p.max_pages = max_pages_per_seq;
    p.scale = scale;
    p.splits = L.splits;
    p.ws = reinterpret_cast<char *>(ws);
    p.counters_off = L.counters_off;
    p.ml_off = L.ml_off;
    p.acc_off = L.acc_off;
    return launch_paged_gqa_decode(p, (cudaStream_t)stream, false);
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
    p.Hkv = Hkv;
    p.page_size = page_size;
    p.max_pages = max_pages_per_seq;
    p.scale = scale;
    p.splits = L.splits;
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
