"""The INT8-activation A/B variant of the INT4 GEMV (dp4a) vs the oracle (needs a B200).

The pages tell of an INT8-activation path that lost to byte-permute unpacking on H100 and was removed;
this variant re-measures that alternative on B200 beside the production path. It is a different
function: x is rounded to int8 per 128-group (scale max|x| / 127), so against the oracle's INT4 product
it carries that rounding. Checked here:
* exact case: when every group's x are integers with max |x| = 127 the int8 rounding is the identity,
  every integer partial sum is exact and the fp32 scaling of power-of-two scales is exact, so the
  result equals the oracle's bit for bit (pins the nibble-to-byte order, dp4a operand order and the
  -8 * sum(x) correction);
* general inputs at the gate/up and down shapes: the normwise error against the oracle stays within
  INT8_TOL. With x ~ N(0, 1) a group's max is ~3, so the rounding step is ~0.024 and a dot product of
  K terms moves by ~ sqrt(K) * 0.024 / sqrt(12) * rms(w), about 1e-3 of the largest output; INT8_TOL
  allows 10x that.
"""
import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import dev, normwise_err

pytestmark = pytest.mark.gpu

INT8_TOL = 1e-2
DP4A = 5


def run(i4, cuda, w, s, x, unpack):
    import torch
    y = i4.int4_gemv(dev(w, cuda), dev(s, cuda), dev(x, cuda), unpack=unpack)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_int8_exact_case_bit_exact(i4lib, cuda):
    rng = np.random.default_rng(12)
    N, K = 512, 3584
    w = rng.integers(0, 2**32, size=(N, K // 8), dtype=np.uint32)
    s = (2.0 ** rng.integers(-10, -6, size=(N, K // 128))).astype(np.float16)
    x = rng.integers(-127, 128, size=(1, K)).astype(np.float64)
    x.reshape(-1, 128)[:, 0] = 127.0  # every group's max |x| is 127: the int8 scale is 1
    x = x.astype(np.float16)
    got = run(i4lib, cuda, w, s, x, DP4A)
    ref = oracle.f16(oracle.int4_linear(w, s, x))
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("N,K", [(37888, 3584), (3584, 18944), (4608, 3584)])
def test_int8_variant_error_against_oracle(i4lib, cuda, N, K):
    w, s, x, _ = synth.gemv_case(N, K, seed=N)
    got = run(i4lib, cuda, w, s, x, DP4A)
    rows = np.sort(np.random.default_rng(N).choice(N, size=512, replace=False))
    ref = oracle.f16(oracle.int4_linear(w[rows], s[rows], x))
    err = normwise_err(got[:, rows], ref)
    print(f"int8-activation normwise error at N={N} K={K}: {err:.2e}")
    assert err <= INT8_TOL
    assert i4lib.device_error() == 0
