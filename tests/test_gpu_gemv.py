"""INT4 GEMV and unpack through the C ABI vs the CPU oracle (needs a B200).

Tolerance: the workload names a max relative error of 2e-3 for fp16 outputs
with fp32 accumulation, read here as normwise max|g - r| / max|r| (the oracle
sums in fp64). Both unpack variants are checked. Exact-arithmetic inputs
(power-of-two scales, small integer x) must come out bit-exact.
"""
import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import dev, normwise_err

pytestmark = pytest.mark.gpu

TOL = 2e-3


def run_gemv(i4, cuda, w, s, x, b=None, out_fp32=False, unpack=None, max_ctas=0):
    y = i4.int4_gemv(dev(w, cuda), dev(s, cuda), dev(np.atleast_2d(x), cuda),
                     None if b is None else dev(b, cuda), out_fp32=out_fp32, unpack=unpack, max_ctas=max_ctas)
    import torch
    torch.cuda.synchronize()
    return y.cpu().numpy()


def pack_fields(q):
    n, k = q.shape
    u = (q.astype(np.int64) & 0xF).reshape(n, k // 8, 8)
    words = np.zeros((n, k // 8), dtype=np.int64)
    for i in range(8):
        words |= u[:, :, i] << (4 * i)
    return words.astype(np.uint32)


def test_unpack_bit_exact(i4lib, cuda):
    rng = np.random.default_rng(0)
    w = rng.integers(0, 2**32, size=(37, 64), dtype=np.uint32)
    w[0, :16] = np.arange(16, dtype=np.uint32) * 0x11111111  # every code in every field
    got = i4lib.int4_unpack(dev(w, cuda), 512).cpu().numpy()
    assert np.array_equal(got, oracle.unpack_int4(w, 512))


@pytest.mark.parametrize("unpack", [0, 1, 2, 3])
@pytest.mark.parametrize("kernel", ["stream", "register"])
def test_qkv_shape_against_oracle(i4lib, cuda, unpack, kernel):
    w, s, x, b = synth.gemv_case(4608, 3584, seed=0, bias=True)
    ref = oracle.int4_gemv(w, s, x[0], b)
    got = run_gemv(i4lib, cuda, w, s, x, b, unpack=unpack, max_ctas=0 if kernel == "stream" else 1 << 20)[0]
    assert normwise_err(got, ref) <= TOL
    assert np.mean(got == ref) >= 0.98  # fp32 vs fp64 sums round to the same fp16 almost always


@pytest.mark.parametrize("unpack", [0, 1, 2, 3])
def test_exact_arithmetic_is_bit_exact(i4lib, cuda, unpack):
    rng = np.random.default_rng(1)
    n, k = 96, 1024
    q = rng.integers(-8, 8, size=(n, k))
    s = np.ldexp(1.0, rng.integers(-8, -4, size=(n, k // 128))).astype(np.float16)
    x = rng.integers(-3, 4, size=(1, k)).astype(np.float16)
    w = pack_fields(q)
    ref = oracle.int4_gemv(w, s, x[0], None)
    got = run_gemv(i4lib, cuda, w, s, x, unpack=unpack)[0]
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))
    got32 = run_gemv(i4lib, cuda, w, s, x, out_fp32=True, unpack=unpack)[0]
    assert np.array_equal(got32, oracle.int4_linear(w, s, x[0]).astype(np.float32))


@pytest.mark.parametrize("n,k,m", [(1, 128, 1), (37, 640, 1), (129, 384, 2), (64, 3584, 3), (50, 1152, 5),
                                   (33, 256, 8)])
def test_ragged_shapes_and_batches(i4lib, cuda, n, k, m):
    w, s, x, b = synth.gemv_case(n, k, m=m, seed=3, bias=True)
    ref = oracle.int4_gemv(w, s, x, b)
    for unpack in (0, 1):
        got = run_gemv(i4lib, cuda, w, s, x, b, unpack=unpack)
        assert got.shape == (m, n)
        assert normwise_err(got, ref) <= TOL


@pytest.mark.parametrize("kernel,unpack", [("stream", 0), ("stream", 1), ("stream", 2), ("stream", 3), ("register", 0)])
def test_mlp_shapes_against_oracle(i4lib, cuda, kernel, unpack):
    # gate/up K=3584 N=37888 and down K=18944 N=3584 (the MLP block of the 7B shape)
    for n, k in [(37888, 3584), (3584, 18944)]:
        w, s, x, _ = synth.gemv_case(n, k, seed=5)
        ref = oracle.int4_gemv(w, s, x[0])
        got = run_gemv(i4lib, cuda, w, s, x, unpack=unpack, max_ctas=0 if kernel == "stream" else 1 << 20)[0]
        assert normwise_err(got, ref) <= TOL, (n, k)
        assert np.mean(got == ref) >= 0.98


@pytest.mark.parametrize("n", [2, 16, 18, 30, 4096 + 14])
def test_stream_kernel_partial_tiles(i4lib, cuda, n):
    # rows not a multiple of the 16-row tile: the last tile copies and computes only its rows
    w, s, x, b = synth.gemv_case(n, 512, seed=8, bias=True)
    ref = oracle.int4_gemv(w, s, x[0], b)
    for unpack in (0, 1, 2, 3):
        got = run_gemv(i4lib, cuda, w, s, x, b, unpack=unpack)[0]
        assert normwise_err(got, ref) <= TOL
    assert i4lib.device_error() == 0


def test_lm_head_fp32_logits(i4lib, cuda):
    w, s, x, _ = synth.gemv_case(152064, 3584, seed=6)
    ref = oracle.int4_linear(w, s, x[0])
    got = run_gemv(i4lib, cuda, w, s, x, out_fp32=True)[0]
    assert got.dtype == np.float32
    assert normwise_err(got, ref) <= 1e-5
    assert int(np.argmax(got)) == oracle.argmax(ref.astype(np.float32))


def test_bad_arguments_raise(i4lib, cuda):
    import torch
    w, s, x, _ = synth.gemv_case(8, 256, seed=7)
    wd, sd = dev(w, cuda), dev(s, cuda)
    xd = dev(x, cuda)
    with pytest.raises(i4lib.I4Error):
        i4lib.int4_gemv(wd, sd, xd, group=64)
    with pytest.raises(i4lib.I4Error):  # K not a multiple of the group
        i4lib.int4_gemv(wd[:, :12], sd, torch.zeros((2, 96), dtype=torch.float16, device=cuda))
    with pytest.raises(i4lib.I4Error):  # the int8-activation variant takes one vector only
        i4lib.int4_gemv(wd, sd, torch.zeros((2, 256), dtype=torch.float16, device=cuda), unpack=5)


@pytest.mark.parametrize("n,k", [(3584, 18944), (64, 4608), (30, 8192), (6, 2560), (14, 1536)])
def test_tensor_core_kernel_block_edges(i4lib, cuda, n, k):
    """The tensor-core kernel on long rows (2-row tiles, blocks split over warps) and on K that
    ends inside a 1024-weight block (18944, 2560 and 1536 leave half or a quarter of a block)."""
    import torch
    w, s, x, b = synth.gemv_case(n, k, seed=9, bias=True)
    ref = oracle.int4_gemv(w, s, x[0], b)
    args = [dev(a, cuda) for a in (w, s, x)]
    got = i4lib.int4_gemv(*args, bias=dev(b, cuda), unpack=3)
    torch.cuda.synchronize()
    assert normwise_err(got.cpu().numpy()[0], ref) <= TOL
    assert i4lib.device_error() == 0


@pytest.mark.parametrize("n,k,m", [(4608, 3584, 2), (1000, 3584, 4), (3584, 2048, 8), (18, 512, 7)])
def test_batched_tensor_core_kernel(i4lib, cuda, n, k, m):
    """M = 2..8 vectors as the MMA's N columns (default path and explicit variant 3): qkv-sized and
    ragged row counts, fp16 and fp32 outputs, bias."""
    w, s, x, b = synth.gemv_case(n, k, m=m, seed=10, bias=True)
    ref = oracle.int4_gemv(w, s, x, b)
    for unpack in (3, None):
        got = run_gemv(i4lib, cuda, w, s, x, b, unpack=unpack)
        assert got.shape == (m, n)
        assert normwise_err(got, ref) <= TOL, unpack
    ref32 = oracle.int4_linear(w, s, x, b)
    got32 = run_gemv(i4lib, cuda, w, s, x, b, out_fp32=True, unpack=3)
    assert normwise_err(got32, ref32) <= 1e-5
    assert i4lib.device_error() == 0


def test_batched_tensor_core_exact_arithmetic(i4lib, cuda):
    """Power-of-two scales and small integer x: every vector of the batch comes out bit-exact."""
    rng = np.random.default_rng(5)
    n, k, m = 80, 1024, 6
    q = rng.integers(-8, 8, size=(n, k))
    s = np.ldexp(1.0, rng.integers(-8, -4, size=(n, k // 128))).astype(np.float16)
    x = rng.integers(-3, 4, size=(m, k)).astype(np.float16)
    w = pack_fields(q)
    got = run_gemv(i4lib, cuda, w, s, x, unpack=3)
    for i in range(m):
        ref = oracle.int4_gemv(w, s, x[i], None)
        assert np.array_equal(got[i].view(np.uint16), ref.view(np.uint16)), i


@pytest.mark.parametrize("n,k", [(37888, 3584), (3584, 18944)])
def test_weight_stage_holdback_keeps_bits(i4lib, cuda, n, k):
    """The number of weight stages copied before x is requested (option gemv_prex) changes only when
    copies start: the outputs are bit-identical for 0, 1 (default) and 3 stages."""
    import torch
    w, s, x, _ = synth.gemv_case(n, k, seed=11)
    args = [dev(a, cuda) for a in (w, s, x)]
    outs = []
    try:
        for prex in (0, 1, 3):
            i4lib.set_option("gemv_prex", prex)
            outs.append(i4lib.int4_gemv(*args).cpu().numpy())
    finally:
        i4lib.set_option("gemv_prex", 1)
    torch.cuda.synchronize()
    assert np.array_equal(outs[0].view(np.uint16), outs[1].view(np.uint16))
    assert np.array_equal(outs[2].view(np.uint16), outs[1].view(np.uint16))
    assert normwise_err(outs[1][0], oracle.int4_gemv(w, s, x[0])) <= TOL
    assert i4lib.device_error() == 0


def test_bounded_wait_reports_and_the_context_recovers(i4lib, cuda):
    """Failure detection without a fault: with the test-only stall the producer never copies its first
    tile, so the consumers' wait for it and the producer's wait for a free stage run out (~2 s each).
    The launch returns, the host reads device error 1, and the next call on the same context is
    correct."""
    import torch
    w, s, x, b = synth.gemv_case(4608, 3584, seed=12, bias=True)
    args = [dev(a, cuda) for a in (w, s, x)]
    bias = dev(b, cuda)
    assert i4lib.device_error() == 0
    i4lib.set_option("test_stall", 1)
    try:
        i4lib.int4_gemv(*args, bias=bias)
        torch.cuda.synchronize()
    finally:
        i4lib.set_option("test_stall", 0)
    assert i4lib.device_error() == 1  # read and cleared
    got = i4lib.int4_gemv(*args, bias=bias).cpu().numpy()[0]
    assert normwise_err(got, oracle.int4_gemv(w, s, x[0], b)) <= TOL
    assert i4lib.device_error() == 0
