"""RMSNorm, RoPE + KV append and SiLU-mul through the C ABI vs the CPU oracle (needs a B200)."""
import numpy as np
import pytest

import oracle
from int4_weight_only_02_b200 import synth
from helpers import dev, normwise_err

pytestmark = pytest.mark.gpu


def sync():
    import torch
    torch.cuda.synchronize()


def test_rmsnorm_rows(i4lib, cuda):
    rng = synth.rng_for(0, 9)
    x = synth.normal_f16(rng, (3, 3584), 0.0, 20.0)
    g = synth.normal_f16(rng, (3584,), 1.0, 0.1)
    got = i4lib.rmsnorm(dev(x, cuda), dev(g, cuda), eps=1e-6).cpu().numpy()
    ref = oracle.rmsnorm(x, g, 1e-6)
    assert normwise_err(got, ref) <= 2e-3
    assert np.mean(got == ref) >= 0.95


def test_rmsnorm_with_residual(i4lib, cuda):
    import torch
    rng = synth.rng_for(0, 10)
    x = synth.normal_f16(rng, (2, 3584))
    r = synth.normal_f16(rng, (2, 3584), 0.0, 30.0)
    g = synth.normal_f16(rng, (3584,), 1.0, 0.1)
    rd = dev(r, cuda)
    out = torch.empty_like(rd)
    i4lib.rmsnorm(dev(x, cuda), dev(g, cuda), out=out, resid=rd)
    sync()
    r_ref = oracle.residual_add(r, x)
    assert np.array_equal(rd.cpu().numpy(), r_ref)
    assert normwise_err(out.cpu().numpy(), oracle.rmsnorm(r_ref, g)) <= 2e-3


@pytest.mark.parametrize("pos", [0, 1, 17, 511, 4095])
def test_rope_and_kv_append(i4lib, cuda, pos):
    import torch
    nq, nkv, d, ps, pages = 28, 4, 128, 16, 256
    rng = synth.rng_for(0, 11, pos)
    qkv = synth.normal_f16(rng, (1, (nq + 2 * nkv) * d))
    table = rng.permutation(pages).astype(np.int32)[None]
    kp = torch.zeros((pages, nkv, ps, d), dtype=torch.float16, device=cuda)
    vp = torch.zeros_like(kp)
    qd = dev(qkv, cuda)
    i4lib.rope_kv_append(qd, dev(np.array([pos], np.int32), cuda), nq, nkv, 1e6, kp, vp, dev(table, cuda))
    sync()
    got = qd.cpu().numpy()[0]
    q_ref = oracle.rope(qkv[0, : nq * d].reshape(nq, d), pos, 1e6)
    k_ref = oracle.rope(qkv[0, nq * d:(nq + nkv) * d].reshape(nkv, d), pos, 1e6)
    v_ref = qkv[0, (nq + nkv) * d:].reshape(nkv, d)
    assert normwise_err(got[: nq * d].reshape(nq, d), q_ref) <= 2e-3
    assert np.mean(got[: nq * d].reshape(nq, d) == q_ref) >= 0.97
    page, slot = table[0, pos // ps], pos % ps
    kpn, vpn = kp.cpu().numpy(), vp.cpu().numpy()
    assert normwise_err(kpn[page, :, slot], k_ref) <= 2e-3
    assert np.array_equal(vpn[page, :, slot], v_ref)
    kpn[page, :, slot] = 0
    vpn[page, :, slot] = 0
    assert not kpn.any() and not vpn.any()  # nothing else written


def test_silu_mul(i4lib, cuda):
    rng = synth.rng_for(0, 12)
    gu = synth.normal_f16(rng, (2, 2 * 18944), 0.0, 4.0)
    got = i4lib.silu_mul(dev(gu, cuda)).cpu().numpy()
    ref = oracle.silu_mul(gu[:, :18944], gu[:, 18944:])
    assert normwise_err(got, ref) <= 2e-3
    assert np.mean(got == ref) >= 0.99
