/*
 * i4rt -- batch-1 INT4 weight-only decode of a Qwen2.5-7B-shaped decoder on
 * NVIDIA B200 (sm_100a). C ABI of libi4rt.so.
 *
 * The operations follow "How To Build Your Own LLM Runtime From Scratch"
 * ("Technical Details": INT4 weight packing and dequantisation, a paged KV
 * cache, attention over it, and a decode step captured as one CUDA graph; the
 * CUDA-graph item of the same section gives eager ~119 ms/token versus graph
 * replay ~17 ms/token on H100). The pages fix no formats; this library uses:
 *
 *   INT4 weights  w[N][K/8] uint32. Word j of row n holds k = 8j .. 8j+7;
 *                 field i (bits 4i..4i+3) is k = 8j+i as a two's-complement
 *                 integer in [-8, 7].
 *   scales        s[N][K/group] fp16, symmetric: W[n][k] = q[n][k] * s[n][k/group].
 *   fp16          IEEE binary16, passed as uint16_t bit patterns.
 *   KV pools      [num_pages][n_kv][page_size][head_dim] fp16, one K and one V
 *                 pool per layer; token t of sequence b is in page
 *                 page_table[b][t / page_size], slot t % page_size.
 *
 * Conventions shared by every call:
 *   - Return value: I4_OK (0) or a negative I4_E* status. i4_last_error()
 *     returns a text for the last failure on the calling thread.
 *   - Tensor pointers are device memory owned by the caller unless a comment
 *     says "host". The library never frees caller memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it; arguments are validated on the host before any
 *     launch, and an invalid call launches nothing.
 *   - No call allocates device memory, synchronises the device or reads
 *     device memory on the host, except decode_step_graph_create/destroy.
 */
#ifndef I4RT_H
#define I4RT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define I4_API __attribute__((visibility("default")))
#else
#define I4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define I4_OK 0
#define I4_EINVAL (-1)       /* null pointer, bad shape or size */
#define I4_EALIGN (-2)       /* pointer alignment below the stated requirement */
#define I4_EUNSUPPORTED (-3) /* valid but not implemented (e.g. head_dim != 128) */
#define I4_ECUDA (-4)        /* a CUDA runtime call or launch failed */
#define I4_ENOMEM (-5)       /* device allocation failed (graph create only) */

/* Text of the last failure on this thread ("" if none). Never NULL. */
I4_API const char *i4_last_error(void);

/* Library version string. */
I4_API const char *i4_version(void);

/*
 * INT4 weight-only linear layer ("INT4 dequantization" fused into the product):
 *   y[m][n] = sum_k q[n][k] * s[n][k/group] * x[m][k]  (+ bias[n])
 * accumulated in fp32, stored as fp16 (y_is_fp32 = 0) or fp32 (y_is_fp32 = 1).
 *   w      [N][K/8] uint32, 16-byte aligned;
 *   scales [N][K/group] fp16, 2-byte aligned;
 *   x      [M][K] fp16, 16-byte aligned;  bias [N] fp16 or NULL;
 *   y      [M][N], 4-byte aligned for fp32.
 * Requires group == 128, K % 128 == 0, K <= 32768, M >= 1, N >= 1. M > 8 runs
 * int4_gemm below. For M <= 8, shapes off the tensor-core paths stage the M
 * vectors in shared memory, which allows M <= 8 up to K = 12032 and M <= 4 up
 * to K = 24064 (larger M * K is refused with I4_EUNSUPPORTED). The kernel is
 * chosen by the "unpack" option below.
 */
I4_API int int4_gemv(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
              int y_is_fp32, int M, int N, int K, int group, void *stream);

/*
 * The same INT4 linear layer for many activation rows (batched decode, prompt
 * prefill) on the tcgen05 tensor cores: each 64-wide K chunk of 128 weight rows
 * is dequantised to fp16 (q * s, rounded once) in shared memory and multiplied
 * with the fp16 activations by tcgen05.mma into fp32 accumulators in tensor
 * memory; y = accumulator (+ bias), stored as fp16 or fp32.
 *   w [N][K/8] uint32 and x [M][K] fp16, 16-byte aligned; scales [N][K/128];
 *   bias [N] or NULL; y [M][N]. group == 128, K % 128 == 0, K <= 65536.
 * The weights enter the product exactly: each dequantised weight q * s is
 * held as two fp16 terms, hi = fp16(q * s) and lo = q * s - hi (exact), both
 * multiplied into the same fp32 accumulator.
 * Any M >= 1 (tiles of 16 .. 512 activation rows per CTA); the tensor maps of
 * w and x are encoded on the host at each call.
 *   ws, ws_bytes: optional workspace (256-byte aligned) of
 *   int4_gemm_ws_bytes(M, N, K) bytes (0 when the shape is not split). With
 *   it, shapes whose 128-row tiles leave SMs idle split K over several CTAs,
 *   and a second kernel adds their fp32 partials in split order; without it
 *   (NULL) K is not split. Calls sharing one workspace must not overlap on
 *   the GPU.
 */
I4_API size_t int4_gemm_ws_bytes(int M, int N, int K);
I4_API int int4_gemm(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias, void *y,
                     int y_is_fp32, int M, int N, int K, int group, void *ws, size_t ws_bytes, void *stream);

/*
 * Test export: q[n][k] = signed field of w (bit-exact unpack check).
 *   w [N][K/8] uint32; q [N][K] int8. K % 8 == 0.
 */
I4_API int i4_int4_unpack(const uint32_t *w, int8_t *q, int N, int K, void *stream);

/*
 * Paged grouped-query decode attention ("paged KV cache, and attention"; the
 * softmax must be exact at partially filled last pages). For each sequence b
 * and query head h, with kv head g = h / (Hq / Hkv) and n = ctx_len[b]:
 *   s_t = scale * q[b][h] . K[g][t],  p = softmax(s over t < n),
 *   out[b][h] = sum_t p_t V[g][t]        (fp32 math, fp16 out)
 * computed as split-K over pages with a log-sum-exp merge.
 *   q, out      [B][Hq][D] fp16, 16-byte aligned;
 *   k_pool, v_pool [num_pages][Hkv][page_size][D] fp16, 16-byte aligned;
 *   page_table  [B][max_pages_per_seq] int32 physical page ids;
 *   ctx_len     [B] int32 device array, tokens per sequence INCLUDING the
 *               current one, 1 <= ctx_len[b] <= max_pages_per_seq * page_size;
 *   ws          workspace of paged_gqa_decode_ws_bytes(...) bytes, 256-byte
 *               aligned, ZEROED by the caller before its first use; every call
 *               leaves its counters zero again. Calls sharing one ws must not
 *               overlap on the GPU.
 * Requires D == 128, 1 <= Hq / Hkv <= 8 (Hq % Hkv == 0), page_size a power of
 * two in [8, 128], max_pages_per_seq * page_size <= 32768, B >= 1.
 */
I4_API size_t paged_gqa_decode_ws_bytes(int B, int Hq, int Hkv, int D, int page_size, int max_pages_per_seq);
I4_API int paged_gqa_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool, const int32_t *page_table,
                     const int32_t *ctx_len, uint16_t *out, int B, int Hq, int Hkv, int D, int page_size,
                     int max_pages_per_seq, float scale, void *ws, size_t ws_bytes, void *stream);

/*
 * paged_gqa_decode without a workspace argument and without any allocation.
 * The pages have no counterpart of this call; it exists for callers that
 * cannot hand out device memory: code that runs where cudaMalloc is not
 * allowed or not wanted (inside a stream capture, on a real-time decode loop
 * that must not block in the allocator, or as a plugin of a host framework
 * that owns every device buffer).
 *   Same arguments, layouts and results as paged_gqa_decode, minus ws and
 *   ws_bytes. The split-K scratch is an 8 MiB array in the library's device
 *   memory, which every GPU that loads the library keeps until the process
 *   exits. A shape whose scratch (paged_gqa_decode_ws_bytes) exceeds 8 MiB is
 *   rejected with I4_EUNSUPPORTED.
 *   The first call on a device looks the array's address up (once per
 *   device); make that first call before any stream capture.
 *   Each call clears the merge counters with an asynchronous memset on
 *   `stream`, then launches the kernel. All calls share the one array and it
 *   keeps the last call's contents: calls that overlap on the GPU (for example
 *   on two streams) race with each other. No cudaMalloc, cudaFree or other
 *   allocating routine is called.
 */
I4_API int paged_gqa_decode_static(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                                   const int32_t *page_table, const int32_t *ctx_len, uint16_t *out, int B, int Hq,
                                   int Hkv, int D, int page_size, int max_pages_per_seq, float scale, void *stream);

/*
 * paged_gqa_decode with the q rows of consecutive sequences q_stride elements
 * apart (q_stride >= Hq * D, a multiple of 8), so q can be read where a fused
 * qkv projection left it: q of sequence b is q[b * q_stride .. + Hq * D).
 * Same workspace, layouts, results and errors as paged_gqa_decode otherwise.
 */
I4_API int i4_paged_gqa_decode_strided(const uint16_t *q, long long q_stride, const uint16_t *k_pool,
                                       const uint16_t *v_pool, const int32_t *page_table, const int32_t *ctx_len,
                                       uint16_t *out, int B, int Hq, int Hkv, int D, int page_size,
                                       int max_pages_per_seq, float scale, void *ws, size_t ws_bytes, void *stream);

/*
 * Test export: out[b][g][t][:] = pool row of token t (t < ctx_len[b]) for kv
 * head g, in token order (bit-exact page-indexing check). Rows t >= ctx_len[b]
 * are left untouched.  out [B][Hkv][max_ctx][D] fp16.
 */
I4_API int i4_paged_gather(const uint16_t *pool, const int32_t *page_table, const int32_t *ctx_len, uint16_t *out, int B,
                    int Hkv, int D, int page_size, int max_pages_per_seq, int max_ctx, void *stream);

/*
 * RMSNorm and RoPE + KV append, the glue of a decoder layer. Either part may
 * be skipped by leaving its first pointer NULL; when both are given the norm
 * runs first.
 *
 * Norm part (x_in != NULL), for each of M rows of H values:
 *   if resid != NULL:  resid = fp16(resid + x_in), v = resid  else v = x_in
 *   out = fp16(v / sqrt(mean(v^2) + eps) * gamma)          (fp32 math)
 *   x_in, resid, out [M][H] fp16; gamma [H] fp16; H % 8 == 0, H <= 32768.
 *
 * RoPE part (qkv != NULL), for each of B sequences at position pos[b]:
 *   qkv [B][(Hq + 2 Hkv) * D] fp16 laid out [q heads | k heads | v heads];
 *   q and k heads are rotated in place (rotate-half pairs (i, i + D/2),
 *   angle pos * theta^(-2i/D), fp32 math), then k and v of each kv head are
 *   written to page_table[b][pos / page_size], slot pos % page_size of the
 *   pools (skipped when k_pool is NULL). D == 128.
 */
typedef struct i4_rmsnorm_rope_args {
    /* norm part */
    const uint16_t *x_in;
    uint16_t *resid;
    const uint16_t *gamma;
    uint16_t *out;
    int M, H;
    float eps;
    /* rope + append part */
    uint16_t *qkv;
    const int32_t *pos;
    int B, Hq, Hkv, D;
    float theta;
    uint16_t *k_pool, *v_pool;
    const int32_t *page_table;
    int page_size, max_pages_per_seq;
} i4_rmsnorm_rope_args;

I4_API int rmsnorm_rope(const i4_rmsnorm_rope_args *args, void *stream);
I4_API int i4_rmsnorm(const uint16_t *x_in, uint16_t *resid, const uint16_t *gamma, uint16_t *out, int M, int H, float eps,
               void *stream);
I4_API int i4_rope_kv_append(uint16_t *qkv, const int32_t *pos, int B, int Hq, int Hkv, int D, float theta,
                      uint16_t *k_pool, uint16_t *v_pool, const int32_t *page_table, int page_size,
                      int max_pages_per_seq, void *stream);

/*
 * SwiGLU gate: out[m][i] = fp16(silu(g) * u), g = gate_up[m][i], u = gate_up[m][I + i],
 * silu(g) = g / (1 + exp(-g)) in fp32.  gate_up [M][2I] fp16; out [M][I] fp16.
 */
I4_API int silu_mul(const uint16_t *gate_up, uint16_t *out, int M, int I, void *stream);

/*
 * Embedding rows of a batch of tokens: out[b][:] = table[t][:] with
 * t = tokens[b] clamped to [0, vocab). table [vocab][H] fp16, tokens [B] int32
 * device array, out [B][H] fp16; H % 8 == 0, table and out 16-byte aligned.
 */
I4_API int i4_embed_gather(const uint16_t *table, const int32_t *tokens, uint16_t *out, int B, int H, int vocab,
                           void *stream);

/*
 * Greedy choice per row: tokens[b] = the index of the largest logits[b][:]
 * (the lowest such index; -0 ranks with +0); then, when pos / ctx_len are not
 * NULL, pos[b] += 1 and ctx_len[b] += 1 (the step's state advance).
 * logits [B][N] fp32; tokens, pos, ctx_len [B] int32 device arrays.
 */
I4_API int i4_argmax_rows(const float *logits, int32_t *tokens, int32_t *pos, int32_t *ctx_len, int B, int N,
                          void *stream);

/* ---------------------------------------------------------------- decode step */

typedef struct i4_model_desc {
    int n_layers, hidden, intermediate, n_q_heads, n_kv_heads, head_dim, vocab;
    int group;      /* INT4 group size along K, must be 128 */
    int page_size;  /* tokens per KV page */
    int max_ctx;    /* page table length * page_size */
    float rope_theta, rms_eps;
} i4_model_desc;

typedef struct i4_layer_weights {
    const uint32_t *w_qkv;     /* [(Hq + 2 Hkv) D][hidden/8], rows [q | k | v] */
    const uint16_t *s_qkv;     /* [(Hq + 2 Hkv) D][hidden/128] */
    const uint16_t *b_qkv;     /* [(Hq + 2 Hkv) D] */
    const uint32_t *w_o;       /* [hidden][Hq D/8] */
    const uint16_t *s_o;
    const uint32_t *w_gate_up; /* [2 intermediate][hidden/8], rows [gate | up] */
    const uint16_t *s_gate_up;
    const uint32_t *w_down;    /* [hidden][intermediate/8] */
    const uint16_t *s_down;
    const uint16_t *ln_in;     /* input_layernorm gamma [hidden] */
    const uint16_t *ln_post;   /* post_attention_layernorm gamma [hidden] */
} i4_layer_weights;

typedef struct i4_model_weights {
    const uint16_t *embed;             /* [vocab][hidden] fp16 */
    const i4_layer_weights *layers;    /* HOST array of n_layers (copied at create) */
    const uint16_t *ln_final;          /* [hidden] */
    const uint32_t *w_lm;              /* [vocab][hidden/8] */
    const uint16_t *s_lm;              /* [vocab][hidden/128] */
} i4_model_weights;

/*
 * One sequence's decode state, all device memory owned by the caller.
 * A step reads token[0] at position pos[0] (ctx_len[0] must equal pos[0] + 1),
 * appends its K/V, writes fp32 logits [vocab], and then advances the state on
 * the device: pos += 1, ctx_len += 1, token = prompt[pos] while pos < n_prompt,
 * else the argmax of the logits (lowest index on ties); history[pos] = token.
 * Steps whose position would reach max_ctx set *status to 1 and do nothing.
 */
typedef struct i4_seq_state {
    int32_t *token, *pos, *ctx_len;   /* [1] each */
    const int32_t *page_table;        /* [max_ctx / page_size] */
    uint16_t *const *k_pools;         /* HOST array of n_layers device pointers */
    uint16_t *const *v_pools;         /* HOST array of n_layers device pointers */
    int num_pages;                    /* pages in each pool */
    float *logits;                    /* [vocab] */
    const int32_t *prompt;            /* [n_prompt] or NULL */
    int n_prompt;
    int32_t *history;                 /* [max_ctx] or NULL */
    int32_t *status;                  /* [1], 0 = ok */
} i4_seq_state;

typedef struct i4_graph i4_graph;

/*
 * Build the decode step: allocates its private workspace, validates shapes and
 * captures every kernel of one token into a CUDA graph on an internal stream.
 * The descriptors are copied; the device buffers they point at must outlive
 * the graph. Returns I4_ENOMEM, I4_EINVAL, I4_EUNSUPPORTED or I4_ECUDA on failure.
 */
I4_API int decode_step_graph_create(const i4_model_desc *desc, const i4_model_weights *weights, const i4_seq_state *seq,
                             i4_graph **out);
/* Launch the captured token step on `stream` (one cudaGraphLaunch). */
I4_API int decode_step_graph_replay(i4_graph *g, void *stream);
/* The same step as individual kernel launches on `stream` (no graph). */
I4_API int decode_step_eager(i4_graph *g, void *stream);
/* Kernel launches in one step (eager or inside the graph): 1 for the persistent
 * step, 5 * n_layers + 1 for the per-kernel step. */
I4_API int decode_step_kernel_count(const i4_graph *g);
/* Phases of one step: 5 * n_layers + 1 (per layer qkv, attention, o, gate/up,
 * down; then lm_head). */
I4_API int decode_step_phase_count(const i4_graph *g);
/* 1 when the step runs as one persistent kernel, 0 for one kernel per phase. */
I4_API int decode_step_is_persistent(const i4_graph *g);
/*
 * Diagnostics of a persistent step created with the "trace" option: copies the
 * timestamps (GPU global timer, ns) of the last launch to HOST memory
 * `host_out` of n >= phase_count * grid * 4 entries, laid out [phase][cta][4]:
 * consumers begin the phase, its input vector is staged, its work is done, and
 * the producer issues the phase's first tile (0 where the CTA had no such
 * event); for attention phases entries 1 and 3 are the CTA's key tiles done
 * and its partial result published. Synchronous.
 */
I4_API int decode_step_trace(i4_graph *g, unsigned long long *host_out, size_t n);
I4_API int decode_step_graph_destroy(i4_graph *g);
/*
 * Test and benchmark export: run only phase `index` (0 <= index < phase count)
 * of the step on `stream`, with the step's arguments, as one launch. Per layer
 * l the phases are 5l+0 qkv, 5l+1 attention, 5l+2 o, 5l+3 gate/up, 5l+4 down;
 * the last is lm_head + argmax, which advances the sequence state. Phases that
 * add into the residual or write K/V leave values that the next full step
 * rewrites.
 */
I4_API int decode_step_launch_kernel(i4_graph *g, int index, void *stream);

/*
 * Test export: copy one of the step's own activation buffers to (dir = 0) or
 * from (dir = 1) the caller's device buffer `dev`, asynchronously on `stream`.
 * `bytes` must equal the buffer's size:
 *   I4_BUF_RESID  the fp16 residual stream [hidden];
 *   I4_BUF_Q      q after RoPE, fp16 [n_q_heads * head_dim];
 *   I4_BUF_ATTN   the attention output, fp16 [n_q_heads * head_dim];
 *   I4_BUF_MLP    SiLU(gate) * up, fp16 [intermediate].
 * With decode_step_launch_kernel this lets a test give one kernel of the step
 * chosen inputs and read back its outputs.
 */
#define I4_BUF_RESID 0
#define I4_BUF_Q 1
#define I4_BUF_ATTN 2
#define I4_BUF_MLP 3
I4_API int decode_step_buffer_copy(i4_graph *g, int which, void *dev, size_t bytes, int dir, void *stream);

/*
 * Library options, applied to graphs created afterwards and to later calls:
 *   "pdl"    0/1 (default 1): launch the kernels of a decode step with programmatic
 *            dependent launch (each kernel still waits for its predecessor's
 *            results before reading them);
 *   "unpack" 0..4: INT4 unpack / multiply variant of the GEMV: 0 exact fp16
 *            values, 1 offset-binary fp16 subnormals with a sum(x) correction
 *            (both fp16 x fp16 -> fp32 FMAs), 2 fp32 values from an exponent
 *            trick (packed fp32 FMAs), 3 the subnormal fields as the A operand of
 *            mma.sync (tensor cores, fp32 accumulate; for M = 2..8 the vectors are
 *            the MMA's N columns, rows of up to 4096 weights), 4 (default): 3
 *            where it applies, else 0;
 *   "stream" 0/1: use the bulk-copy pipelined GEMV where the shape allows it
 *            (M == 1, K % 512 == 0, 16-byte aligned w and scales), default 1;
 *   "stream_smem_kb" 32..227: shared memory budget of that kernel's ring;
 *   "gemv_ctas_per_sm" 1/2 (default 2): CTAs per SM of the pipelined GEMV grids;
 *   "test_stall" 0/1 (default 0): for tests of the bounded waits only: the
 *            tensor-core GEMV's producer skips its first copy, its consumers'
 *            wait and then its own run out (~2 s each), the launch records
 *            device error 1 (i4_device_error) and returns; never set it in use;
 *   "gemv_prex" 0..8 (default 1): weight stages the tensor-core GEMV copies
 *            before its loads of x are issued (the rest follow them, so x does
 *            not queue behind a full ring of weight copies);
 *   "l2_ahead" 0..64 (default 8): tiles of its own weight stream each CTA of a
 *            persistent step prefetches into L2 ahead of its shared-memory ring;
 *   "trace"  0/1 (default 0): persistent steps created afterwards record phase
 *            timestamps (see decode_step_trace);
 *   "persistent" 0/1 (default 1): build decode steps as one persistent kernel
 *            per token (one CTA per SM running every phase, the weight stream
 *            never stopping at phase boundaries; shapes it does not cover fall
 *            back to one kernel per phase);
 *   "l2_prefetch" 0/1 (default 0): in a decode step, each GEMV prefetches the
 *            next GEMV's weights into L2 (up to 48 MB) once its own ring is full.
 * Not thread-safe; set options before creating graphs.
 */
I4_API int i4_set_option(const char *name, int value);

/*
 * Device-side error flag: 0, or 1 when a bounded wait inside a kernel gave up
 * (the kernel then stopped early and its outputs are invalid). Synchronises
 * with the device; reset != 0 clears the flag. Negative on a CUDA error.
 */
I4_API int i4_device_error(int reset);

/*
 * int4_gemv with an explicit unpack variant (as for "unpack") and a cap on the
 * number of CTAs (0 = none; any cap selects the register-streaming kernel
 * instead of the bulk-copy pipelined one); for tests and benchmarks.
 * unpack 5 is the INT8-activation variant, the alternative the pages' lesson on
 * byte permutes against __dp4a describes: x is quantised to int8 per 128-group
 * (scale max|x| / 127, round to nearest), the nibbles become offset-binary
 * bytes, dp4a sums the products with an exact -8 * sum(x) correction, and the
 * group's integer sum is scaled by s_w * s_x in fp32. Its result carries the
 * int8 rounding of x (it is not the INT4 weight-only product); M == 1 and
 * K % 512 == 0 only (the bulk-copy streaming kernel, plain fp16/fp32 output).
 */
I4_API int i4_int4_gemv_variant(const uint32_t *w, const uint16_t *scales, const uint16_t *x, const uint16_t *bias,
                                void *y, int y_is_fp32, int M, int N, int K, int unpack, int max_ctas, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* I4RT_H */
