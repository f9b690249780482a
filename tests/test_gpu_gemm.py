"""The tcgen05 INT4 GEMM (many activation rows: batched decode and prefill) vs the CPU oracle (needs a B200).

y[m][n] = sum_k q[n][k] s[n][k/128] x[m][k] (+ bias) with the weights dequantised to fp16 in shared
memory and multiplied on tcgen05.mma into fp32 TMEM accumulators. Covered: every activation tile
width (16, 32, 64, 128, 256, 512 rows per CTA), ragged M and N (partial tiles read zero-filled TMA
rows), the 7B shapes (qkv, o, gate/up, down) at batch 32 and 64 and at the 512-token prefill,
fp16 and fp32 outputs, bias; an exact-arithmetic case must match bit for bit (any misplaced
element of the swizzled tiles, descriptors or TMEM read-back shows there).
"""
import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import dev, normwise_err

pytestmark = pytest.mark.gpu

TOL = 2e-3


def run_gemm(i4, cuda, w, s, x, b=None, out_fp32=False, split=True):
    """The GEMM with a split-K workspace (split=True: the launch configuration of batched decode and
    prefill) or without one."""
    import torch
    M, K = x.shape
    ws = None
    if split:
        ws = torch.zeros(max(i4.int4_gemm_ws_bytes(M, w.shape[0], K), 256), dtype=torch.uint8, device=cuda)
    y = i4.int4_gemm(dev(w, cuda), dev(s, cuda), dev(x, cuda), None if b is None else dev(b, cuda), out_fp32=out_fp32,
                     ws=ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("M,N,K", [(16, 256, 512), (20, 1000, 1024), (32, 4608, 3584), (64, 3584, 3584),
                                   (100, 384, 2048), (128, 640, 1024), (200, 512, 512), (300, 256, 2048),
                                   (512, 512, 3584)])
def test_gemm_shapes_against_oracle(i4lib, cuda, M, N, K, split):
    w, s, x, b = synth.gemv_case(N, K, m=M, seed=M + N, bias=True)
    got = run_gemm(i4lib, cuda, w, s, x, b, split=split)
    ref = oracle.f16(oracle.int4_linear(w, s, x, b))
    assert got.shape == (M, N)
    assert normwise_err(got, ref) <= TOL
    assert i4lib.device_error() == 0


def test_gemm_weights_enter_exactly(i4lib, cuda):
    """Scales whose products with the codes need more than fp16's 11 significant bits (so fp16(q * s) alone
    would be off) and one-hot activations: y[m][n] = q[n][k_m] * s[n][k_m / 128] exactly, so the fp32 output
    must equal the oracle's value bit for bit -- the two-term dequantisation holds every weight exactly."""
    rng = np.random.default_rng(8)
    M, N, K = 64, 256, 1024
    w = rng.integers(0, 2**32, size=(N, K // 8), dtype=np.uint32)
    s = rng.uniform(0.005, 0.02, size=(N, K // 128)).astype(np.float16)
    ks = rng.choice(K, size=M, replace=False)
    x = np.zeros((M, K), dtype=np.float16)
    x[np.arange(M), ks] = 1.0
    got = run_gemm(i4lib, cuda, w, s, x, out_fp32=True)
    ref = oracle.int4_linear(w, s, x).astype(np.float32)
    assert np.array_equal(got, ref)


def test_gemm_fp32_output(i4lib, cuda):
    w, s, x, _ = synth.gemv_case(2048, 3584, m=48, seed=5)
    got = run_gemm(i4lib, cuda, w, s, x, out_fp32=True)
    ref = oracle.int4_linear(w, s, x)
    assert got.dtype == np.float32
    assert normwise_err(got, ref) <= TOL


def test_gemm_exact_arithmetic_bit_exact(i4lib, cuda):
    """Power-of-two scales and small-integer activations: every dequantised weight is exact in fp16, every
    product and partial sum exact in fp32, so the result must equal the oracle's bit for bit."""
    rng = np.random.default_rng(3)
    M, N, K = 70, 300, 1024
    w = rng.integers(0, 2**32, size=(N, K // 8), dtype=np.uint32)
    s = (2.0 ** rng.integers(-6, -2, size=(N, K // 128))).astype(np.float16)
    x = rng.integers(-3, 4, size=(M, K)).astype(np.float16)
    b = (rng.integers(-8, 8, size=N) * 0.25).astype(np.float16)
    got = run_gemm(i4lib, cuda, w, s, x, b)
    ref = oracle.f16(oracle.int4_linear(w, s, x, b))
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("name,N,K", [("qkv", 4608, 3584), ("o", 3584, 3584), ("gate_up", 37888, 3584),
                                      ("down", 3584, 18944)])
@pytest.mark.parametrize("M", [32, 64, 512])
def test_gemm_7b_shapes_sampled(i4lib, cuda, name, N, K, M):
    """The decoder's layer shapes at batch 32 / 64 and the 512-token prefill, in the launch configuration the
    batched decode and prefill use; the oracle checks 96 sampled output rows (all M columns of each)."""
    w, s, x, _ = synth.gemv_case(N, K, m=M, seed=N + M)
    got = run_gemm(i4lib, cuda, w, s, x)
    rows = np.sort(np.random.default_rng(N + M).choice(N, size=96, replace=False))
    rows[-1] = N - 1  # the last tile's last row
    ref = oracle.f16(oracle.int4_linear(w[rows], s[rows], x))
    assert normwise_err(got[:, rows], ref) <= TOL
    assert i4lib.device_error() == 0


def test_gemv_routes_many_rows_to_gemm(i4lib, cuda):
    import torch
    w, s, x, b = synth.gemv_case(1024, 2048, m=24, seed=9, bias=True)
    y = i4lib.int4_gemv(dev(w, cuda), dev(s, cuda), dev(x, cuda), dev(b, cuda))
    torch.cuda.synchronize()
    ref = oracle.f16(oracle.int4_linear(w, s, x, b))
    assert normwise_err(y.cpu().numpy(), ref) <= TOL
