"""Paged GQA decode attention through the C ABI vs the CPU oracle (needs a B200).

Covers the page-tail lengths (1, P-1, P, P+1, 511, 513), ragged batches over a
shared permuted page pool (page sizes 16 and 64), long contexts, the sweep's
largest shapes (sampled), bit-exact page indexing, and bit-identical results
under any page permutation.
"""
import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import dev, normwise_err

pytestmark = pytest.mark.gpu

TOL = 2e-3


def run_attention(i4, cuda, q, kp, vp, table, ctx):
    import torch
    out = i4.paged_gqa_decode(dev(q, cuda), dev(kp, cuda), dev(vp, cuda), dev(table, cuda), dev(ctx, cuda))
    torch.cuda.synchronize()
    return out.cpu().numpy()


def check_case(i4, cuda, ctx_lens, page_size, seed, n_q=28, n_kv=4):
    q, kp, vp, table, ctx = synth.attention_case(ctx_lens, n_q=n_q, n_kv=n_kv, page_size=page_size, seed=seed)
    got = run_attention(i4, cuda, q, kp, vp, table, ctx)
    for b, n in enumerate(ctx):
        ref = oracle.f16(oracle.paged_attention(q[b], kp, vp, table[b], int(n)))
        err = normwise_err(got[b], ref)
        assert err <= TOL, (b, int(n), err)


def test_config0_ctx512_page16(i4lib, cuda):
    check_case(i4lib, cuda, [512], 16, seed=0)


@pytest.mark.parametrize("ctx", [1, 7, 15, 16, 17, 31, 33, 511, 513, 1000])
def test_page_tails(i4lib, cuda, ctx):
    check_case(i4lib, cuda, [ctx], 16, seed=ctx)


@pytest.mark.parametrize("page_size", [16, 64])
@pytest.mark.parametrize("length,batch", [(512, 8), (2048, 8), (512, 32)])
def test_ragged_batches(i4lib, cuda, page_size, length, batch):
    lens = synth.ragged_lengths(length, batch, seed=length + batch)
    check_case(i4lib, cuda, lens, page_size, seed=page_size + batch)


@pytest.mark.parametrize("ctx,page_size", [(8192, 16), (32768, 64)])
def test_long_context(i4lib, cuda, ctx, page_size):
    check_case(i4lib, cuda, [ctx], page_size, seed=11)


@pytest.mark.parametrize("length,batch,page_size", [(32768, 8, 16), (8192, 32, 64)])
def test_sweep_full_size_sampled(i4lib, cuda, length, batch, page_size):
    """The attention sweep's largest shapes (ragged lengths in [L/2, L], one shared permuted pool) in the
    launch configuration the sweep times; the oracle checks the longest, the shortest and one more
    sequence in full."""
    lens = synth.ragged_lengths(length, batch, seed=length + batch)
    q, kp, vp, table, ctx = synth.attention_case(lens, page_size=page_size, seed=page_size + batch + 1)
    got = run_attention(i4lib, cuda, q, kp, vp, table, ctx)
    for b in sorted({int(np.argmax(ctx)), int(np.argmin(ctx)), batch // 2}):
        ref = oracle.f16(oracle.paged_attention(q[b], kp, vp, table[b], int(ctx[b])))
        err = normwise_err(got[b], ref)
        assert err <= TOL, (b, int(ctx[b]), err)
    assert np.all(np.isfinite(got.astype(np.float32)))


def test_group_sizes(i4lib, cuda):
    check_case(i4lib, cuda, [300, 77], 16, seed=12, n_q=8, n_kv=8)     # G = 1
    check_case(i4lib, cuda, [300, 77], 16, seed=13, n_q=16, n_kv=2)    # G = 8


def test_permutation_invariance_bit_exact(i4lib, cuda):
    q, kp, vp, table, ctx = synth.attention_case([200], page_size=16, seed=21, spare_pages=5)
    ref = run_attention(i4lib, cuda, q, kp, vp, table, ctx)
    rng = np.random.default_rng(0)
    n_pages = kp.shape[0]
    used = (200 + 15) // 16
    for _ in range(5):
        perm = rng.permutation(n_pages).astype(np.int32)
        kp2 = np.zeros_like(kp)
        vp2 = np.zeros_like(vp)
        t2 = np.zeros_like(table)
        for i in range(used):
            kp2[perm[i]] = kp[table[0, i]]
            vp2[perm[i]] = vp[table[0, i]]
            t2[0, i] = perm[i]
        got = run_attention(i4lib, cuda, q, kp2, vp2, t2, ctx)
        assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


def test_paged_gather_bit_exact(i4lib, cuda):
    q, kp, vp, table, ctx = synth.attention_case([37, 100, 16], page_size=16, seed=31, spare_pages=3)
    got = i4lib.paged_gather(dev(kp, cuda), dev(table, cuda), dev(ctx, cuda), 112).cpu().numpy()
    for b, n in enumerate(ctx):
        assert np.array_equal(got[b, :, :n], oracle.paged_gather(kp, table[b], int(n)))


def test_workspace_counters_return_to_zero(i4lib, cuda):
    import torch
    q, kp, vp, table, ctx = synth.attention_case([900], page_size=16, seed=41)
    B, Hq, D = q.shape
    nbytes = i4lib.paged_gqa_decode_ws_bytes(B, Hq, 4, D, 16, table.shape[1])
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=cuda)
    args = [dev(a, cuda) for a in (q, kp, vp, table, ctx)]
    a = i4lib.paged_gqa_decode(*args, ws=ws).clone()
    b = i4lib.paged_gqa_decode(*args, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert int(ws[:256].view(torch.int32).abs().sum().item()) == 0
