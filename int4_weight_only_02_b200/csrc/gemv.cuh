// Internal interface of the fused INT4 GEMV kernels (see gemv.cu).
#pragma once

#include "common.cuh"

namespace i4 {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

enum GemvPrologue : int { PRO_PLAIN = 0, PRO_RMSNORM = 1, PRO_EMBED = 2 };
enum GemvEpilogue : int { EPI_F16 = 0, EPI_F32 = 1, EPI_RESID = 2, EPI_ROPE_KV = 3, EPI_SILU = 4, EPI_ARGMAX = 5 };
// UNPACK_AUTO picks per launch: the tensor-core kernels (single-vector, or batched for M <= 8 with rows of
// up to 4096 weights; the fastest measured), else the exact CUDA-core unpack.
// UNPACK_DP4A is the INT8-activation variant (x quantised to int8 per 128-group, dp4a products); it changes
// the arithmetic, so it is selected only explicitly (i4_int4_gemv_variant), for comparison.
enum GemvUnpack : int {
    UNPACK_EXACT = 0, UNPACK_SUBNORMAL = 1, UNPACK_MAGIC32 = 2, UNPACK_MMA = 3, UNPACK_AUTO = 4, UNPACK_DP4A = 5
};

struct GemvArgs {
    const uint32_t *w;
    const uint16_t *s;
    int N, K, M;
    // prologue: x [M][K] (plain), residual [K] (rmsnorm) or embedding table [vocab][K] (embed)
    const uint16_t *x;
    const uint16_t *gamma;
    float eps;
    const int32_t *token;
    int vocab;
    uint16_t *resid_out;
    // epilogue
    const uint16_t *bias;
    void *y;  // fp16/fp32 out, residual (in/out), SiLU output or fp32 logits
    // qkv: RoPE + KV append (head_dim 128)
    const int32_t *pos;
    const int32_t *page_table;
    uint16_t *k_pool, *v_pool, *q_out;
    const float2 *rope_cs;  // [max_ctx][64] (cos, sin)
    int n_q, n_kv, page_size, max_ctx;
    // gate/up: intermediate size
    int inter;
    // lm_head: argmax and state advance
    unsigned long long *best;
    unsigned *arrive;
    int32_t *token_io, *pos_io, *ctx_io, *history, *status;
    const int32_t *prompt;
    int n_prompt;
    // L2 prefetch of the next kernel's weights and scales (bulk prefetch split over
    // the CTAs, issued once the ring is first filled); null pointers = none
    const void *pf_a, *pf_b;
    size_t pf_a_bytes, pf_b_bytes;
    // tensor-core GEMV: two zeroed counters of a dynamic tile schedule, owned by this launch until it
    // completes (left zeroed again); null = each CTA takes a fixed contiguous range of tiles
    unsigned *sched;
};

size_t gemv_smem_bytes(int K, int mr, int unp);

// Geometry of the streaming (bulk-copy pipelined) GEMV for one launch.
struct StreamGeom {
    int R;              // rows per tile (16 or 2)
    int stage_bytes;    // weights + scales of one tile, padded to 128 B
    int stages;         // ring depth
    int tiles, tiles_per_cta, grid;
    int smem;           // dynamic shared memory bytes
    int prex;           // tensor-core consumer: stages copied before the loads of x are issued
    int test_stall;     // tests of the bounded waits: the producer skips its first copy (see set_test_stall)
};
// False when the shape or alignment does not fit the streaming kernel.
bool stream_geometry(int epi, const GemvArgs &a, StreamGeom &g, int unp);
int launch_gemv_stream(int pro, int epi, const GemvArgs &a, const StreamGeom &geo, cudaStream_t stream, bool pdl,
                       int unp);
void set_stream_options(int enabled, int smem_kb);
void set_stream_ctas_per_sm(int n);
void set_stream_prex(int n);
// Test of the bounded waits: while set, the tensor-core GEMV's producer never copies its first tile, so the
// consumers' wait for it and then the producer's wait for a free stage run out (~2 s each) and the kernel
// records device error 1 and returns; no fault, the context stays usable.
void set_test_stall(int on);
// unp < 0 selects the library default; max_ctas <= 0 means no cap.
int launch_gemv(int pro, int epi, const GemvArgs &a, cudaStream_t stream, bool pdl, int unp, int max_ctas);

extern int g_default_unpack;

// RoPE rotation of one (i, i + D/2) pair, fp32 with explicit roundings so the
// fused and the stand-alone paths give identical bits.
__device__ __forceinline__ void rope_pair(float a, float b, float2 cs, uint16_t &oa, uint16_t &ob) {
    oa = float_to_half_bits(__fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y)));
    ob = float_to_half_bits(__fadd_rn(__fmul_rn(b, cs.x), __fmul_rn(a, cs.y)));
}

// (cos, sin) of pos * theta^(-2i/D), evaluated in fp64 and rounded to fp32.
__device__ __forceinline__ float2 rope_cos_sin(int pos, int i, int d, double theta) {
    const double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
    double s, c;
    sincos(ang, &s, &c);
    return make_float2((float)c, (float)s);
}

__device__ __forceinline__ uint16_t silu_mul_bits(float g, float u) {
    const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
    return float_to_half_bits(__fmul_rn(silu, u));
}

}  // namespace i4
