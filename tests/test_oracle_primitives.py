"""Pins for the CPU oracle's primitives (no GPU).

Each expected value here comes from a closed form, an exact-integer
construction, a library routine, an invariant or a brute-force count -- never
from re-running the oracle's own formula. The cases are chosen so that a
plausible slip (a shifted or swapped nibble, a lost sign, a scale indexed by
the wrong group, a transposed operand, a wrong RoPE pairing or frequency, a
softmax without the max shift or the 1/sqrt(D) scale, a wrong GQA mapping, a
page-table off-by-one) breaks at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth


def pack_fields(q: np.ndarray) -> np.ndarray:
    """Test-side packing: q int [N][K] in [-8, 7] -> uint32 [N][K/8], field i at bits 4i."""
    n, k = q.shape
    u = (q.astype(np.int64) & 0xF).reshape(n, k // 8, 8)
    words = np.zeros((n, k // 8), dtype=np.int64)
    for i in range(8):
        words |= u[:, :, i] << (4 * i)
    return words.astype(np.uint32)


# ------------------------------------------------------------------ fp16 conversion

def test_f16_widen_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16)
    got = oracle.widen_c(h)
    want = h.astype(np.float64)
    finite = np.isfinite(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[np.isinf(want)], want[np.isinf(want)])


def test_f16_round_matches_numpy_including_ties():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 5, 100000),
                           [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-8, 6e-8, 3e-8, -3e-8]])
    # exact midpoints between neighbouring fp16 values: ties must go to even
    h = np.arange(1, 31744, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    h_next = (np.arange(1, 31744, 7, dtype=np.uint16) + 1).view(np.float16).astype(np.float64)
    vals = np.concatenate([vals, (h + h_next) / 2.0, -(h + h_next) / 2.0])
    got = oracle.f16_c(vals).view(np.uint16)
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


# ------------------------------------------------------------------ INT4 unpack

def test_unpack_every_value_in_every_position():
    rng = np.random.default_rng(2)
    rows = []
    expect = []
    for pos in range(8):
        for v in range(-8, 8):
            q = rng.integers(-8, 8, size=8)
            q[pos] = v
            rows.append(q)
            expect.append((pos, v))
    q = np.array(rows)
    w = pack_fields(q)
    got = oracle.unpack_int4(w, 8)
    assert np.array_equal(got, q)
    for r, (pos, v) in enumerate(expect):
        assert got[r, pos] == v


def test_unpack_known_words():
    w = np.array([[0x76543210, 0x89ABCDEF, 0x00000008, 0xF0000000]], dtype=np.uint32)
    got = oracle.unpack_int4(w, 32)[0]
    assert list(got[0:8]) == [0, 1, 2, 3, 4, 5, 6, 7]
    assert list(got[8:16]) == [-1, -2, -3, -4, -5, -6, -7, -8]
    assert list(got[16:24]) == [-8, 0, 0, 0, 0, 0, 0, 0]
    assert list(got[24:32]) == [0, 0, 0, 0, 0, 0, 0, -1]


# ------------------------------------------------------------------ INT4 linear

def test_linear_exact_integer_case():
    """Power-of-two scales and small integer x: every partial sum is exact, so the
    result must equal the integer product computed in int64."""
    rng = np.random.default_rng(3)
    n, k, g = 40, 512, 128
    q = rng.integers(-8, 8, size=(n, k))
    e = rng.integers(-6, 0, size=(n, k // g))           # scales 2^e
    s = np.ldexp(1.0, e).astype(np.float16)
    xi = rng.integers(-4, 5, size=(3, k))
    x = xi.astype(np.float16)
    got = oracle.int4_linear(pack_fields(q), s, x, None, g)
    # exact: sum_g 2^e[n][g] * sum_{k in g} q x  (integer sums scaled by powers of two)
    part = np.einsum("ngk,mgk->mng", q.reshape(n, k // g, g), xi.reshape(3, k // g, g))
    want = (part * np.ldexp(1.0, e)[None]).sum(-1)
    assert np.array_equal(got, want)


def test_linear_one_hot_selects_a_scaled_column():
    rng = np.random.default_rng(4)
    n, k, g = 24, 384, 128
    q = rng.integers(-8, 8, size=(n, k))
    s = rng.uniform(0.005, 0.02, size=(n, k // g)).astype(np.float16)
    w = pack_fields(q)
    for col in [0, 1, 7, 8, 127, 128, 129, 255, 383]:
        x = np.zeros(k, dtype=np.float16)
        x[col] = 1.0
        got = oracle.int4_linear(w, s, x, None, g)
        want = q[:, col] * s[:, col // g].astype(np.float64)
        assert np.array_equal(got, want), col


def test_linear_bias_and_zero_input():
    n, k = 16, 256
    w = synth.packed_int4(np.random.default_rng(5), n, k)
    s = synth.group_scales(np.random.default_rng(6), n, k)
    b = synth.normal_f16(np.random.default_rng(7), (n,), 0.0, 0.1)
    got = oracle.int4_linear(w, s, np.zeros(k, np.float16), b)
    assert np.array_equal(got, b.astype(np.float64))


def test_linear_matches_float64_matmul_of_test_side_dequant():
    rng = np.random.default_rng(8)
    n, k, g = 33, 640, 128
    q = rng.integers(-8, 8, size=(n, k))
    s = rng.uniform(0.005, 0.02, size=(n, k // g)).astype(np.float16)
    x = rng.standard_normal((5, k)).astype(np.float16)
    b = rng.standard_normal(n).astype(np.float16)
    wd = q * np.repeat(s.astype(np.float64), g, axis=1)
    want = x.astype(np.float64) @ wd.T + b.astype(np.float64)
    got = oracle.int4_linear(pack_fields(q), s, x, b, g)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_linear_rows_independent_of_batch():
    w, s, x, b = synth.gemv_case(48, 512, m=6, seed=1, bias=True)
    y_all = oracle.int4_linear(w, s, x, b)
    for m in range(6):
        assert np.array_equal(oracle.int4_linear(w, s, x[m], b), y_all[m])


def test_linear_is_linear():
    w, s, x, _ = synth.gemv_case(64, 1024, m=2, seed=2)
    xa, xb = x[0].astype(np.float64), x[1].astype(np.float64)
    ya, yb = oracle.int4_linear(w, s, x[0]), oracle.int4_linear(w, s, x[1])
    xs = (xa + xb).astype(np.float16)          # exact when no rounding happens: check only where exact
    exact = xs.astype(np.float64) == xa + xb
    xs[~exact] = 0
    xa2 = np.where(exact, xa, 0).astype(np.float16)
    xb2 = np.where(exact, xb, 0).astype(np.float16)
    y_sum = oracle.int4_linear(w, s, xs)
    np.testing.assert_allclose(y_sum, oracle.int4_linear(w, s, xa2) + oracle.int4_linear(w, s, xb2),
                               rtol=1e-12, atol=1e-12)
    assert np.abs(ya).max() > 0 and np.abs(yb).max() > 0


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_unit_gamma_gives_unit_rms():
    x = synth.normal_f16(np.random.default_rng(9), (3584,), 0.0, 30.0)
    y = oracle.rmsnorm(x, np.ones(3584, np.float16)).astype(np.float64)
    assert abs(math.sqrt(np.mean(y * y)) - 1.0) < 1e-3


def test_rmsnorm_constant_vector_closed_form():
    for c in [0.5, 3.0, -7.25]:
        x = np.full(256, c, dtype=np.float16)
        gamma = np.linspace(0.5, 1.5, 256).astype(np.float16)
        y = oracle.rmsnorm(x, gamma, eps=1e-6)
        want = (np.sign(c) / math.sqrt(1.0 + 1e-6 / (c * c))) * gamma.astype(np.float64)
        assert np.array_equal(y, want.astype(np.float16))


def test_rmsnorm_scale_invariance():
    x = synth.normal_f16(np.random.default_rng(10), (3584,))
    g = synth.normal_f16(np.random.default_rng(11), (3584,), 1.0, 0.1)
    y1 = oracle.rmsnorm(x, g, eps=0.0)
    y2 = oracle.rmsnorm((x.astype(np.float64) * 4.0).astype(np.float16), g, eps=0.0)
    assert np.array_equal(y1, y2)


# ------------------------------------------------------------------ RoPE

def test_rope_position_zero_is_identity():
    v = synth.normal_f16(np.random.default_rng(12), (4, 128))
    assert np.array_equal(oracle.rope(v, 0, 1e6), v)


def test_rope_two_dims_is_a_plain_rotation():
    for p in [1, 2, 7, 100]:
        got = oracle.rope(np.array([1.0, 0.0], np.float16), p, 1e6).astype(np.float64)
        np.testing.assert_allclose(got, [math.cos(p), math.sin(p)], atol=1e-3)
        got = oracle.rope(np.array([0.0, 1.0], np.float16), p, 1e6).astype(np.float64)
        np.testing.assert_allclose(got, [-math.sin(p), math.cos(p)], atol=1e-3)


def test_rope_frequency_and_pairing():
    # D = 4, theta = 100: pair (0, 2) turns at 1 rad/position, pair (1, 3) at 100^(-1/2) = 0.1.
    v = np.array([1.0, 1.0, 0.0, 0.0], np.float16)
    got = oracle.rope(v, 3, 100.0).astype(np.float64)
    want = [math.cos(3.0), math.cos(0.3), math.sin(3.0), math.sin(0.3)]
    np.testing.assert_allclose(got, want, atol=1e-3)


def test_rope_preserves_pair_norms():
    v = synth.normal_f16(np.random.default_rng(13), (28, 128))
    r = oracle.rope(v, 1234, 1e6).astype(np.float64)
    vd = v.astype(np.float64)
    n0 = vd[:, :64] ** 2 + vd[:, 64:] ** 2
    n1 = r[:, :64] ** 2 + r[:, 64:] ** 2
    np.testing.assert_allclose(n1, n0, rtol=4e-3, atol=1e-3)


def test_rope_relative_position():
    rng = np.random.default_rng(14)
    q = synth.normal_f16(rng, (128,))
    k = synth.normal_f16(rng, (128,))
    ref = oracle.rope(q, 7, 1e6).astype(np.float64) @ oracle.rope(k, 3, 1e6).astype(np.float64)
    for m in [4, 50, 900, 4000]:
        d = oracle.rope(q, m + 4, 1e6).astype(np.float64) @ oracle.rope(k, m, 1e6).astype(np.float64)
        assert abs(d - ref) < 0.05, (m, d, ref)
    far = oracle.rope(q, 11, 1e6).astype(np.float64) @ oracle.rope(k, 3, 1e6).astype(np.float64)
    assert abs(far - ref) > 0.05   # a different offset gives a different score


# ------------------------------------------------------------------ SiLU-mul, residual, argmax

def test_silu_mul_closed_forms():
    g = np.array([0.0, 1.0, -1.0, 20.0, -20.0, 2.0], np.float16)
    u = np.array([5.0, 1.0, 1.0, 1.0, 1.0, -3.0], np.float16)
    got = oracle.silu_mul(g, u).astype(np.float64)
    sig1 = 0.7310585786300049
    want = [0.0, sig1, -(1 - sig1), 20.0, -20.0 * 2.061153622438558e-09, -3.0 * 2.0 * 0.8807970779778823]
    np.testing.assert_allclose(got, np.array(want).astype(np.float16).astype(np.float64), rtol=0, atol=0)


def test_residual_add_rounds_once():
    r = np.array([2048.0, 1.0], np.float16)
    y = np.array([1.0, 2.0 ** -11], np.float16)
    got = oracle.residual_add(r, y)
    assert got[0] == 2048.0     # 2049 is a tie between 2048 and 2050 -> even
    assert got[1] == 1.0        # 1 + 2^-11 is a tie -> even


def test_argmax_lowest_index_on_ties():
    v = np.array([1.0, 3.0, -2.0, 3.0, 3.0], np.float32)
    assert oracle.argmax(v) == 1
    assert oracle.argmax(np.array([-1.0, -1.0], np.float32)) == 0


# ------------------------------------------------------------------ attention

def _contig(pool, table, ctx):
    return oracle.paged_gather(pool, table, ctx)


@pytest.mark.parametrize("ctx", [1, 15, 16, 17, 511, 513])
def test_paged_equals_contiguous_at_page_tails(ctx):
    q, kp, vp, table, _ = synth.attention_case([ctx], seed=ctx)
    o_paged = oracle.paged_attention(q[0], kp, vp, table[0], ctx)
    o_cont = oracle.contiguous_attention(q[0], _contig(kp, table[0], ctx), _contig(vp, table[0], ctx))
    assert np.array_equal(o_paged, o_cont)


def test_paged_attention_invariant_under_page_permutation():
    rng = np.random.default_rng(15)
    ctx, ps = 100, 16
    n_pages = 7
    q = synth.normal_f16(rng, (8, 64))
    k = synth.normal_f16(rng, (2, ctx, 64))
    v = synth.normal_f16(rng, (2, ctx, 64))
    ref = oracle.contiguous_attention(q, k, v)
    for trial in range(20):
        perm = rng.permutation(n_pages + 3)[:n_pages].astype(np.int32)
        kp = np.zeros((n_pages + 3, 2, ps, 64), np.float16)
        vp = np.zeros_like(kp)
        for t in range(ctx):
            kp[perm[t // ps], :, t % ps] = k[:, t]
            vp[perm[t // ps], :, t % ps] = v[:, t]
        # rows past ctx in the last page hold garbage that must never be read
        kp[perm[-1], :, ctx % ps:] = 1000.0
        vp[perm[-1], :, ctx % ps:] = -1000.0
        assert np.array_equal(oracle.paged_attention(q, kp, vp, perm, ctx), ref), trial


def test_paged_gather_brute_force():
    q, kp, vp, table, ctx = synth.attention_case([37], page_size=16, seed=3, spare_pages=2)
    g = oracle.paged_gather(kp, table[0], 37)
    for t in range(37):
        assert np.array_equal(g[:, t], kp[table[0, t // 16], :, t % 16])


def test_softmax_rows_sum_to_one():
    q, kp, vp, table, _ = synth.attention_case([513], seed=4)
    _, p = oracle.paged_attention(q[0], kp, vp, table[0], 513, return_probs=True)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_attention_single_token_returns_its_value():
    q, kp, vp, table, _ = synth.attention_case([1], seed=5)
    o = oracle.paged_attention(q[0], kp, vp, table[0], 1)
    for h in range(28):
        assert np.array_equal(o[h], vp[table[0, 0], h // 7, 0].astype(np.float64))


def test_attention_equal_keys_give_mean_value():
    rng = np.random.default_rng(16)
    ctx = 40
    q = synth.normal_f16(rng, (4, 32))
    k = np.repeat(synth.normal_f16(rng, (2, 1, 32)), ctx, axis=1)
    v = synth.normal_f16(rng, (2, ctx, 32))
    o = oracle.contiguous_attention(q, k, v)
    for h in range(4):
        np.testing.assert_allclose(o[h], v[h // 2].astype(np.float64).mean(0), rtol=0, atol=1e-12)


def test_attention_dominant_key_and_gqa_mapping():
    d, ctx = 16, 9
    q = np.zeros((6, d), np.float16)
    q[:, 0] = 8.0
    k = np.zeros((3, ctx, d), np.float16)
    v = np.zeros((3, ctx, d), np.float16)
    for g in range(3):
        k[g, 2 + g, 0] = 100.0       # score gap 8*100/4 = 200 -> all weight on token 2+g
        v[g, :, :] = -1.0
        v[g, 2 + g, :] = g + 1
    o = oracle.contiguous_attention(q, k, v)
    for h in range(6):                # heads 0,1 -> kv 0; 2,3 -> kv 1; 4,5 -> kv 2
        np.testing.assert_allclose(o[h], np.full(d, h // 2 + 1.0), rtol=0, atol=1e-12)


def test_attention_two_keys_closed_form_with_scale():
    d = 64
    q = np.zeros((1, d), np.float16)
    q[0, 0] = 2.0
    k = np.zeros((1, 2, d), np.float16)
    k[0, 0, 0] = 1.0                  # raw score 2
    k[0, 1, 0] = 3.0                  # raw score 6
    v = np.zeros((1, 2, d), np.float16)
    v[0, 0, :] = 1.0
    v[0, 1, :] = 0.0
    o = oracle.contiguous_attention(q, k, v)
    w0 = 1.0 / (1.0 + math.exp((6.0 - 2.0) / math.sqrt(d)))
    np.testing.assert_allclose(o[0], np.full(d, w0), rtol=1e-14, atol=0)


def test_attention_is_shift_safe_for_large_scores():
    d = 8
    q = np.zeros((1, d), np.float16)
    q[0, 0] = 60000.0
    k = np.zeros((1, 3, d), np.float16)
    k[0, :, 0] = [60000.0, 60000.0, 0.0]
    v = np.zeros((1, 3, d), np.float16)
    v[0, 0, :] = 2.0
    v[0, 1, :] = 4.0
    o = oracle.contiguous_attention(q, k, v)
    np.testing.assert_allclose(o[0], np.full(d, 3.0), rtol=0, atol=1e-12)
