// Device building blocks of the INT4 GEMV kernels (gemv.cu, gemv_stream.cu):
// register-level unpack, the per-chunk dot product, the x stage with its
// fused prologues, row-pair mapping and the fused epilogues.
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "mma.cuh"

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

// fp32 unpack: a field kept in place under an fp32 exponent is 2^(23-4i) + u
// (u = q + 8, the LOP3 flips bit 3 of the field); one packed add of
// -(2^(23-4i) + 8) per two fields gives q exactly, one packed FMA per two
// weights accumulates q * x in fp32. Fields 4-7 use the word shifted by 16.
__device__ __forceinline__ float2 magic_pair(uint32_t q, uint32_t m0, uint32_t c0, uint32_t m1, uint32_t c1,
                                             float2 off) {
    return fadd2(make_float2(__uint_as_float(lop3_select(q, m0, c0)), __uint_as_float(lop3_select(q, m1, c1))), off);
}

// acc += q . x over one word (8 weights); x8 = the word's 8 x values in order.
__device__ __forceinline__ float2 word_dot_f32(uint32_t q, const float4 &xa, const float4 &xb, float2 acc) {
    const float2 off01 = make_float2(-8388616.0f, -524296.0f), off23 = make_float2(-32776.0f, -2056.0f);
    const uint32_t qh = q >> 16;
    const float2 v01 = magic_pair(q, 0x0000000Fu, 0x4B000008u, 0x000000F0u, 0x49000080u, off01);
    const float2 v23 = magic_pair(q, 0x00000F00u, 0x47000800u, 0x0000F000u, 0x45008000u, off23);
    const float2 v45 = magic_pair(qh, 0x0000000Fu, 0x4B000008u, 0x000000F0u, 0x49000080u, off01);
    const float2 v67 = magic_pair(qh, 0x00000F00u, 0x47000800u, 0x0000F000u, 0x45008000u, off23);
    acc = ffma2(v01, make_float2(xa.x, xa.y), acc);
    acc = ffma2(v23, make_float2(xa.z, xa.w), acc);
    acc = ffma2(v45, make_float2(xb.x, xb.y), acc);
    acc = ffma2(v67, make_float2(xb.z, xb.w), acc);
    return acc;
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

// The threads that stage x: the whole CTA, or the consumer warps of a
// warp-specialised CTA, which synchronise on named barrier 1 only (a CTA-wide
// barrier inside a role branch would also wait for the producer warp).
struct CtaGroup {
    __device__ __forceinline__ int tid() const { return threadIdx.x; }
    __device__ __forceinline__ int size() const { return blockDim.x; }
    __device__ __forceinline__ void sync() const { __syncthreads(); }
};

template <int FIRST, int COUNT>
struct NamedGroup {
    static_assert(FIRST % 32 == 0 && COUNT % 32 == 0, "whole warps");
    __device__ __forceinline__ int tid() const { return (int)threadIdx.x - FIRST; }
    __device__ __forceinline__ int size() const { return COUNT; }
    __device__ __forceinline__ void sync() const { asm volatile("bar.sync 1, %0;" ::"n"(COUNT) : "memory"); }
};

// Named barrier 1 over the 256 consumer threads that also ANDs a predicate across them.
__device__ __forceinline__ bool bar1_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

template <class Group>
__device__ __forceinline__ float group_sum(float v, float *red, const Group &g) {
    v = warp_sum(v);
    const int warp = g.tid() >> 5, lane = g.tid() & 31;
    g.sync();
    if (lane == 0) red[warp] = v;
    g.sync();
    float t = 0.f;
    const int nw = g.size() >> 5;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
}

// Produce the K/8 words (8 fp16 each) of the GEMV input x and hand each to
// store(word_index, uint4): the plain vector, or RMSNorm of the residual row
// (embedding row for PRO_EMBED, which CTA 0 also copies to the residual):
//   x = fp16(r / sqrt(mean(r^2) + eps) * gamma), fp32 math.
template <int PRO, class Group, class Store>
__device__ __forceinline__ void for_each_x_word(const GemvArgs &a, float *red, const Group &grp, Store store) {
    const int K = a.K, nwords = K >> 3;
    const uint16_t *src = a.x;
    if constexpr (PRO == PRO_EMBED) {
        int tok = *a.token;
        tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);
        src = a.x + (size_t)tok * K;
    }
    if constexpr (PRO == PRO_PLAIN) {
        for (int c = grp.tid(); c < nwords; c += grp.size()) store(c, *reinterpret_cast<const uint4 *>(src + 8 * c));
    } else {
        float ss = 0.f;
        for (int c = grp.tid(); c < nwords; c += grp.size()) {
            const uint4 rv = *reinterpret_cast<const uint4 *>(src + 8 * c);
            const uint32_t r[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
        ss = group_sum(ss, red, grp);
        const float inv = 1.0f / sqrtf(ss / (float)K + a.eps);
        for (int c = grp.tid(); c < nwords; c += grp.size()) {
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
            store(c, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

// Stage x for the streaming kernel in half-chunks of 16 k (two words):
// xe[h] / xo[h] = pair-permuted even / odd word of half-chunk h; sxh[h] = sum of
// its 16 values (subnormal unpack only).
// Stage x as plain fp32 (fp32 unpack).
template <int PRO, class Group>
__device__ __forceinline__ void stage_x_f32(const GemvArgs &a, float4 *xf, float *red, const Group &grp) {
    for_each_x_word<PRO>(a, red, grp, [&](int c, uint4 v) {
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
        const float2 f2 = __half22float2(*reinterpret_cast<const __half2 *>(&v.z));
        const float2 f3 = __half22float2(*reinterpret_cast<const __half2 *>(&v.w));
        xf[2 * c] = make_float4(f0.x, f0.y, f1.x, f1.y);
        xf[2 * c + 1] = make_float4(f2.x, f2.y, f3.x, f3.y);
    });
}

template <int PRO, int UNP, class Group>
__device__ __forceinline__ void stage_x_halves(const GemvArgs &a, uint4 *xe, uint4 *xo, float *sxh, float *red,
                                               const Group &grp) {
    for_each_x_word<PRO>(a, red, grp, [&](int c, uint4 v) { ((c & 1) ? xo : xe)[c >> 1] = permute_pairs(v); });
    if constexpr (UNP == UNPACK_SUBNORMAL) {
        grp.sync();
        for (int h = grp.tid(); h < (a.K >> 4); h += grp.size()) {
            const uint4 e = xe[h], o = xo[h];
            const uint32_t v[8] = {e.x, e.y, e.z, e.w, o.x, o.y, o.z, o.w};
            float t = 0.f;
            for (int i = 0; i < 8; ++i) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v[i]));
                t += f.x + f.y;
            }
            sxh[h] = t;
        }
    }
}

// Dot product of one half-chunk (words w.x, w.y = 16 weights of a row) with its
// staged x: sum q*x (exact unpack) or sum u*x with u = q + 8 (subnormal unpack).
template <int UNP>
__device__ __forceinline__ float half_dot(uint2 w, const uint4 &x0, const uint4 &x1) {
    uint32_t va[4], vb[4];
    if constexpr (UNP == UNPACK_EXACT) {
        unpack_word_exact(w.x, va);
        unpack_word_exact(w.y, vb);
        float a0 = fma2_f16_f32(va[0], x0.x, 0.f), a1 = fma2_f16_f32(va[1], x0.y, 0.f);
        float b0 = fma2_f16_f32(vb[0], x1.x, 0.f), b1 = fma2_f16_f32(vb[1], x1.y, 0.f);
        a0 = fma2_f16_f32(va[2], x0.z, a0);
        a1 = fma2_f16_f32(va[3], x0.w, a1);
        b0 = fma2_f16_f32(vb[2], x1.z, b0);
        b1 = fma2_f16_f32(vb[3], x1.w, b1);
        return (a0 + a1) + (b0 + b1);
    } else {
        unpack_word_subnormal(w.x, va);
        unpack_word_subnormal(w.y, vb);
        float alo = fma2_f16_f32(va[0], x0.x, 0.f), ahi = fma2_f16_f32(va[1], x0.y, 0.f);
        float blo = fma2_f16_f32(vb[0], x1.x, 0.f), bhi = fma2_f16_f32(vb[1], x1.y, 0.f);
        alo = fma2_f16_f32(va[2], x0.z, alo);
        ahi = fma2_f16_f32(va[3], x0.w, ahi);
        blo = fma2_f16_f32(vb[2], x1.z, blo);
        bhi = fma2_f16_f32(vb[3], x1.w, bhi);
        return fmaf(ahi + bhi, 0.0625f, alo + blo) * 16777216.0f;
    }
}

// Row accumulator of the streaming kernel. Exact unpack: v = sum s*q*x.
// Subnormal unpack: lo = sum s*u*x*2^-24 over low fields, hi the same over high
// fields (which carry 16u), cx = sum s*x; the row value is
// (lo + hi/16) * 2^24 - 8 * cx (u = q + 8), computed once per row.
struct RowAcc {
    float lo, hi, cx;
};

template <int UNP>
__device__ __forceinline__ void half_acc(uint2 w, const uint4 &x0, const uint4 &x1, float s, float sx, RowAcc &r) {
    uint32_t va[4], vb[4];
    if constexpr (UNP == UNPACK_EXACT) {
        unpack_word_exact(w.x, va);
        unpack_word_exact(w.y, vb);
        float a0 = fma2_f16_f32(va[0], x0.x, 0.f), a1 = fma2_f16_f32(va[1], x0.y, 0.f);
        a0 = fma2_f16_f32(va[2], x0.z, a0);
        a1 = fma2_f16_f32(va[3], x0.w, a1);
        a0 = fma2_f16_f32(vb[0], x1.x, a0);
        a1 = fma2_f16_f32(vb[1], x1.y, a1);
        a0 = fma2_f16_f32(vb[2], x1.z, a0);
        a1 = fma2_f16_f32(vb[3], x1.w, a1);
        r.lo = fmaf(s, a0 + a1, r.lo);
    } else {
        unpack_word_subnormal(w.x, va);
        unpack_word_subnormal(w.y, vb);
        float lo = fma2_f16_f32(va[0], x0.x, 0.f), hi = fma2_f16_f32(va[1], x0.y, 0.f);
        lo = fma2_f16_f32(va[2], x0.z, lo);
        hi = fma2_f16_f32(va[3], x0.w, hi);
        lo = fma2_f16_f32(vb[0], x1.x, lo);
        hi = fma2_f16_f32(vb[1], x1.y, hi);
        lo = fma2_f16_f32(vb[2], x1.z, lo);
        hi = fma2_f16_f32(vb[3], x1.w, hi);
        r.lo = fmaf(s, lo, r.lo);
        r.hi = fmaf(s, hi, r.hi);
        r.cx = fmaf(s, sx, r.cx);
    }
}

// fp32 unpack: 16 weights (words w.x, w.y) against x4[0..3] = their 16 x values.
__device__ __forceinline__ void half_acc_f32(uint2 w, const float4 *x4, float s, RowAcc &r) {
    float2 p = word_dot_f32(w.x, x4[0], x4[1], make_float2(0.f, 0.f));
    p = word_dot_f32(w.y, x4[2], x4[3], p);
    const float2 acc = ffma2(make_float2(s, s), p, make_float2(r.lo, r.hi));
    r.lo = acc.x;
    r.hi = acc.y;
}

// INT8-activation variant: x quantised to int8 per 128-group (scale sx_g = max|x_g| / 127, round to
// nearest), the weight nibbles turned into offset-binary bytes u = q + 8 with one LOP3 (low nibbles) or a
// shift and a LOP3 (high nibbles), four dp4a per 16 weights against the int8 x bytes in the same order, and
// the exact integer correction - 8 * sum(x_q); the integer sum of the half-chunk is then scaled by
// s_w * sx_g in fp32. xq = (x0,x2,x4,x6) (x1,x3,x5,x7) (x8,x10,x12,x14) (x9,x11,x13,x15) of the half-chunk.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void half_acc_dp4a(uint2 w, const uint4 &xq, int sq, float s_w_sx, RowAcc &r) {
    const uint32_t la = lop3_and_xor(w.x, 0x0F0F0F0Fu, 0x08080808u);
    const uint32_t ha = lop3_and_xor(w.x >> 4, 0x0F0F0F0Fu, 0x08080808u);
    const uint32_t lb = lop3_and_xor(w.y, 0x0F0F0F0Fu, 0x08080808u);
    const uint32_t hb = lop3_and_xor(w.y >> 4, 0x0F0F0F0Fu, 0x08080808u);
    int acc = dp4a_us(la, xq.x, -8 * sq);
    acc = dp4a_us(ha, xq.y, acc);
    acc = dp4a_us(lb, xq.z, acc);
    acc = dp4a_us(hb, xq.w, acc);
    r.lo = fmaf((float)acc, s_w_sx, r.lo);
}

template <int UNP>
__device__ __forceinline__ float row_value(const RowAcc &r) {
    if constexpr (UNP == UNPACK_MAGIC32) return r.lo + r.hi;
    if constexpr (UNP == UNPACK_EXACT || UNP == UNPACK_DP4A) return r.lo;
    return fmaf(r.hi, 0.0625f, r.lo) * 16777216.0f - 8.0f * r.cx;
}

// INT8 stage: x (after the prologue) quantised per 128-group. xq[h] holds half-chunk h's 16 values as int8 in
// the dp4a order above, sq[h] their integer sum, scx[g] the group's scale; tmp holds K fp16 values.
template <int PRO, class Group>
__device__ __forceinline__ void stage_x_int8(const GemvArgs &a, uint4 *xq, int *sq, float *scx, uint16_t *tmp,
                                             float *red, const Group &grp) {
    const int K = a.K, groups = K >> 7, nhr = K >> 4;
    for_each_x_word<PRO>(a, red, grp, [&](int c, uint4 v) { reinterpret_cast<uint4 *>(tmp)[c] = v; });
    grp.sync();
    // group scales: a warp per group
    const int warp = grp.tid() >> 5, lane = grp.tid() & 31, nw = grp.size() >> 5;
    for (int g = warp; g < groups; g += nw) {
        float m = 0.f;
        for (int i = lane; i < 128; i += 32) m = fmaxf(m, fabsf(half_bits_to_float(tmp[g * 128 + i])));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        if (lane == 0) scx[g] = m > 0.f ? m / 127.0f : 1.0f;
    }
    grp.sync();
    for (int h = grp.tid(); h < nhr; h += grp.size()) {
        const float inv = 1.0f / scx[h >> 3];
        int q[16], sum = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            int v = __float2int_rn(half_bits_to_float(tmp[16 * h + i]) * inv);
            v = v > 127 ? 127 : (v < -127 ? -127 : v);
            q[i] = v;
            sum += v;
        }
        auto pack = [&](int o) {  // bytes x_o, x_{o+2}, x_{o+4}, x_{o+6}
            return (uint32_t)(q[o] & 0xFF) | ((uint32_t)(q[o + 2] & 0xFF) << 8) | ((uint32_t)(q[o + 4] & 0xFF) << 16) |
                   ((uint32_t)(q[o + 6] & 0xFF) << 24);
        };
        xq[h] = make_uint4(pack(0), pack(1), pack(8), pack(9));
        sq[h] = sum;
    }
}

// Stage x (MR vectors of K fp16) into shared memory, pair-permuted:
// xs[m][w][j] holds word w (0..3) of chunk j (0..K/32-1); sxs[m][j] = sum of the
// chunk's 32 x values (subnormal unpack only).
template <int PRO, int UNP, int MR, class Group>
__device__ __forceinline__ void stage_x(const GemvArgs &a, uint4 *xs, float *sxs, float *red, const Group &grp) {
    const int K = a.K, nu4 = K >> 5, nwords = K >> 3;
    const uint16_t *src = a.x;
    if constexpr (PRO == PRO_EMBED) {
        int tok = *a.token;
        tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);
        src = a.x + (size_t)tok * K;
    }
    if constexpr (PRO == PRO_PLAIN) {
        for (int m = 0; m < MR; ++m)
            for (int c = grp.tid(); c < nwords; c += grp.size()) {
                uint4 xv = make_uint4(0, 0, 0, 0);
                if (m < a.M) xv = *reinterpret_cast<const uint4 *>(a.x + (size_t)m * K + 8 * c);
                xs[(m * 4 + (c & 3)) * nu4 + (c >> 2)] = permute_pairs(xv);
            }
    } else {
        // RMSNorm of the residual row: x = fp16(r / sqrt(mean(r^2) + eps) * gamma)
        float ss = 0.f;
        for (int c = grp.tid(); c < nwords; c += grp.size()) {
            const uint4 rv = *reinterpret_cast<const uint4 *>(src + 8 * c);
            const uint32_t r[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[t]));
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
        ss = group_sum(ss, red, grp);
        const float inv = 1.0f / sqrtf(ss / (float)K + a.eps);
        for (int c = grp.tid(); c < nwords; c += grp.size()) {
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
        grp.sync();
        for (int idx = grp.tid(); idx < MR * nu4; idx += grp.size()) {
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

// Epilogue inputs read from global memory, loaded at the start of a tile so their
// latency hides under the tile's arithmetic (the residual of EPI_RESID, the bias
// and cos/sin of EPI_ROPE_KV, the bias of EPI_F16/EPI_F32).
struct EpiIn {
    float a, b;
    float2 cs;
    int page;
};

// Per-CTA constant of EPI_ROPE_KV: the position (read once, after the dependency wait; the page-table
// entry of its page is read with each tile's other epilogue inputs).
struct EpiCta {
    int pos;
};

template <int EPI>
__device__ __forceinline__ EpiCta epi_cta(const GemvArgs &a) {
    EpiCta c = {0};
    if constexpr (EPI == EPI_ROPE_KV) c.pos = *a.pos;
    return c;
}

template <int EPI>
__device__ __forceinline__ EpiIn epi_load(const GemvArgs &a, int p, int ra, int rb, const EpiCta &c) {
    EpiIn e = {0.f, 0.f, make_float2(0.f, 0.f), 0};
    if constexpr (EPI == EPI_RESID) {
        const uint16_t *r = reinterpret_cast<const uint16_t *>(a.y);
        e.a = half_bits_to_float(r[ra]);
        if (rb >= 0) e.b = half_bits_to_float(r[rb]);
    } else if constexpr (EPI == EPI_ROPE_KV) {
        e.a = half_bits_to_float(a.bias[ra]);
        e.b = half_bits_to_float(a.bias[rb]);
        if (c.pos >= 0 && c.pos < a.max_ctx) {
            if ((p >> 6) < a.n_q + a.n_kv) e.cs = a.rope_cs[(size_t)c.pos * 64 + (p & 63)];
            if ((p >> 6) >= a.n_q) e.page = a.page_table[c.pos / a.page_size];
        }
    } else if constexpr (EPI == EPI_F16 || EPI == EPI_F32) {
        if (a.bias) {
            e.a = half_bits_to_float(a.bias[ra]);
            if (rb >= 0) e.b = half_bits_to_float(a.bias[rb]);
        }
    }
    return e;
}

// epilogue<EPI, 1> with the inputs already loaded (same arithmetic, same stores)
template <int EPI>
__device__ __forceinline__ void epilogue_in(const GemvArgs &a, int p, int ra, int rb, float va, float vb,
                                            const EpiIn &e, const EpiCta &c, unsigned long long &best) {
    if constexpr (EPI == EPI_F16 || EPI == EPI_F32) {
        if (a.bias) {
            va += e.a;
            vb += e.b;
        }
        if constexpr (EPI == EPI_F16) {
            uint16_t *y = reinterpret_cast<uint16_t *>(a.y);
            y[ra] = float_to_half_bits(va);
            if (rb >= 0) y[rb] = float_to_half_bits(vb);
        } else {
            float *y = reinterpret_cast<float *>(a.y);
            y[ra] = va;
            if (rb >= 0) y[rb] = vb;
        }
    } else if constexpr (EPI == EPI_RESID) {
        uint16_t *r = reinterpret_cast<uint16_t *>(a.y);
        r[ra] = float_to_half_bits(e.a + rnd16(va));
        if (rb >= 0) r[rb] = float_to_half_bits(e.b + rnd16(vb));
    } else if constexpr (EPI == EPI_SILU) {
        reinterpret_cast<uint16_t *>(a.y)[p] = silu_mul_bits(rnd16(va), rnd16(vb));
    } else if constexpr (EPI == EPI_ROPE_KV) {
        const int head = p >> 6, i = p & 63;
        const float xa = rnd16(va + e.a);
        const float xb = rnd16(vb + e.b);
        if (c.pos < 0 || c.pos >= a.max_ctx) {
            if (a.status) *a.status = 2;
            return;
        }
        if (head < a.n_q + a.n_kv) {
            uint16_t oa, ob;
            rope_pair(xa, xb, e.cs, oa, ob);
            if (head < a.n_q) {
                a.q_out[head * 128 + i] = oa;
                a.q_out[head * 128 + i + 64] = ob;
            } else {
                const int g = head - a.n_q;
                const size_t off = (((size_t)e.page * a.n_kv + g) * a.page_size + c.pos % a.page_size) * 128;
                a.k_pool[off + i] = oa;
                a.k_pool[off + i + 64] = ob;
            }
        } else {
            const int g = head - a.n_q - a.n_kv;
            const size_t off = (((size_t)e.page * a.n_kv + g) * a.page_size + c.pos % a.page_size) * 128;
            a.v_pool[off + i] = float_to_half_bits(xa);
            a.v_pool[off + i + 64] = float_to_half_bits(xb);
        }
    } else if constexpr (EPI == EPI_ARGMAX) {
        float *lg = reinterpret_cast<float *>(a.y);
        lg[ra] = va;
        unsigned long long k = argmax_key(va, ra);
        best = k > best ? k : best;
        if (rb >= 0) {
            lg[rb] = vb;
            k = argmax_key(vb, rb);
            best = k > best ? k : best;
        }
    }
}

// Last CTA of the lm_head GEMV: pick the token and advance the sequence state.
__device__ __forceinline__ void finish_step(const GemvArgs &a, unsigned long long cta_best) {
    __shared__ unsigned long long sbest[32];
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

// ---------------------------------------------------------------- tensor-core row-pair dot product

// One 1024-weight block of the row pair (a, b) on tensor cores: lane (g, c)
// holds 16 contiguous bytes of each row (32 weights, all in group 8b + g),
// unpacked with one shift and four LOP3s per word into offset-binary fp16
// subnormals (u * 2^-24 for low fields, 16u * 2^-24 for high fields) as the A
// operand of mma.m16n8k16; its B fragment is x at the same k. B column g is fed
// only by lanes (g, *), so D[g][g] is row a's dot product over the lane group's
// 128-weight group and D[g + 8][g] row b's; lane (g, g / 2) holds both and adds
// s * ((lo + hi / 16) * 2^24 - 8 * sum(x)) to tot. Other lanes add garbage that
// the caller never reads (it masks them before the warp sum).
__device__ __forceinline__ void block_dot(uint4 qa, uint4 qb, const uint4 *xb, float sxj, float sa, float sb,
                                          bool odd, float2 &tot) {
    const uint32_t wra[4] = {qa.x, qa.y, qa.z, qa.w}, wrb[4] = {qb.x, qb.y, qb.z, qb.w};
    float lo[4], hi[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint4 xc = xb[w * 32];  // (x0,x4) (x2,x6) (x1,x5) (x3,x7)
        uint32_t ua[4], ub[4];
        unpack_word_subnormal(wra[w], ua);  // (k0,k4) 16(k1,k5) (k2,k6) 16(k3,k7)
        unpack_word_subnormal(wrb[w], ub);
        if (w == 0) {
            mma16816_z(lo, ua[0], ub[0], ua[2], ub[2], xc.x, xc.y);
            mma16816_z(hi, ua[1], ub[1], ua[3], ub[3], xc.z, xc.w);
        } else {
            mma16816(lo, ua[0], ub[0], ua[2], ub[2], xc.x, xc.y);
            mma16816(hi, ua[1], ub[1], ua[3], ub[3], xc.z, xc.w);
        }
    }
    const float2 l2 = odd ? make_float2(lo[1], lo[3]) : make_float2(lo[0], lo[2]);
    const float2 h2 = odd ? make_float2(hi[1], hi[3]) : make_float2(hi[0], hi[2]);
    const float2 v = ffma2(ffma2(h2, make_float2(0.0625f, 0.0625f), l2), make_float2(16777216.0f, 16777216.0f),
                           make_float2(-sxj, -sxj));
    tot = ffma2(v, make_float2(sa, sb), tot);
}

// Row pair (slot rows row_a, row_b) against x over blocks [b0, b1); K is a
// compile-time constant when KC > 0 (all offsets then become immediates).
template <int KC>
__device__ __forceinline__ float2 pair_dot(const unsigned char *st, int K, int row_a, int row_b, const uint16_t *sa,
                                           const uint16_t *sb, const uint4 *xt, const float *sx8, int b0, int b1,
                                           int lane) {
    const int Kk = KC ? KC : K, wrow = Kk >> 1, groups = Kk >> 7, kfull = Kk >> 10;
    const int g = lane >> 2, c = lane & 3;
    const bool diag = c == (g >> 1), odd = g & 1;
    const unsigned char *wa = st + (size_t)row_a * wrow + 16 * lane;
    const unsigned char *wb = st + (size_t)row_b * wrow + 16 * lane;
    const uint4 *xl = xt + lane;
    float2 tot = make_float2(0.f, 0.f);
    auto full_block = [&](int b) {
        const uint4 qa = *reinterpret_cast<const uint4 *>(wa + 512 * b);
        const uint4 qb = *reinterpret_cast<const uint4 *>(wb + 512 * b);
        const int j = 8 * b + g;
        block_dot(qa, qb, xl + b * 128, sx8[j], half_bits_to_float(sa[j]), half_bits_to_float(sb[j]), odd, tot);
    };
    auto part_block = [&](int b) {  // past K: all-zero codes (u = 0); groups past K are never read
        uint4 qa = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u), qb = qa;
        if (1024 * b + 32 * lane < Kk) {
            qa = *reinterpret_cast<const uint4 *>(wa + 512 * b);
            qb = *reinterpret_cast<const uint4 *>(wb + 512 * b);
        }
        // lanes of groups past K hold zero codes; their scales and sums are zero too, so they add nothing
        const int j = 8 * b + g;
        const bool in = j < groups;
        block_dot(qa, qb, xl + b * 128, in ? sx8[j] : 0.f, in ? half_bits_to_float(sa[j]) : 0.f,
                  in ? half_bits_to_float(sb[j]) : 0.f, odd, tot);
    };
    if constexpr (KC > 0) {
        if (b0 == 0 && b1 == (KC + 1023) / 1024) {  // the whole row, unrolled
#pragma unroll
            for (int b = 0; b < KC / 1024; ++b) full_block(b);
            if constexpr (KC % 1024) part_block(KC / 1024);
            return diag ? tot : make_float2(0.f, 0.f);
        }
    }
    const int bf = b1 < kfull ? b1 : kfull;
#pragma unroll 2
    for (int b = b0; b < bf; ++b) full_block(b);
    for (int b = bf > b0 ? bf : b0; b < b1; ++b) part_block(b);
    return diag ? tot : make_float2(0.f, 0.f);
}

__device__ __forceinline__ float2 warp_sum2(float2 v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
        v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    }
    return v;
}

}  // namespace i4
