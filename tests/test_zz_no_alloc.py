"""paged_gqa_decode_static: the attention call that allocates nothing.

Some callers cannot hand the library device memory: code running where
cudaMalloc is not allowed or not wanted (inside a stream capture, on a decode
loop that must never block in the allocator, or as a plugin of a framework that
owns every device buffer). For them the library keeps a fixed split-K scratch
array in its own device memory. These tests check, through the C ABI, that on
two calls in a row with different shapes this variant returns exactly the bits
paged_gqa_decode (caller workspace) returns -- the same kernel, splits and
scratch layout, so any scratch-offset or counter error would show -- that both
match the CPU oracle within the attention tolerance, and that a shape too large
for the fixed scratch is refused with a clear status.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import dev, normwise_err

TOL = 2e-3  # the attention tolerance used throughout the GPU tests


@pytest.mark.gpu
def test_static_scratch_matches_workspace_variant_on_consecutive_calls(i4lib, cuda):
    import torch
    cases = [
        synth.attention_case([512], page_size=16, seed=0),                     # the 7B decode shape, ctx 512
        synth.attention_case([700, 33, 1200], page_size=64, seed=1, spare_pages=2),  # a ragged batch after it
    ]
    for q, kp, vp, table, ctx in cases:
        args = [dev(a, cuda) for a in (q, kp, vp, table, ctx)]
        want = i4lib.paged_gqa_decode(*args)
        got = i4lib.paged_gqa_decode_static(*args)
        torch.cuda.synchronize()
        w, g = want.cpu().numpy(), got.cpu().numpy()
        # same kernel, same splits, same scratch layout: identical bits
        assert np.array_equal(g.view(np.uint16), w.view(np.uint16))
        for b, n in enumerate(ctx):
            ref = oracle.f16(oracle.paged_attention(q[b], kp, vp, table[b], int(n)))
            assert normwise_err(g[b], ref) <= TOL, (b, int(n))
    assert i4lib.device_error() == 0


def test_static_scratch_refuses_oversized_shapes(i4lib):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    # 4096 sequences x 8 kv heads need 4 KB of fp32 partials per head, far more than the fixed scratch
    st = i4lib.lib().paged_gqa_decode_static(fake, fake, fake, fake, fake, fake, 4096, 64, 8, 128, 64, 512, 1.0, None)
    assert st == i4lib.I4_EUNSUPPORTED
    assert b"static scratch" in i4lib.lib().i4_last_error()
