"""GPU parity of attn_bwd (dQ, dK, dV) against the fp64 backward oracle, on the
same bf16 inputs.  The GPU forward provides O and LSE, as a caller would.

Tolerance, per gradient tensor G: |G - G_ref| <= 1e-2 * max|G_ref| beyond the
half-ulp of the bf16 output grid at G_ref.  P and dS enter the tensor cores as
bf16 (relative rounding 2^-9 per term, independent across the ~N terms of each
sum), D is formed from the bf16 forward output, accumulation is fp32, and the
result is stored in bf16; 1e-2 of the tensor's largest entry bounds these with
a margin of about 3 in the runs below.  Where the reference vanishes identically
(a single key: P = 1, so dS = P (dP - D) = 0 exactly, while the kernel forms D
from the bf16 output and dP on the tensor cores), max|G_ref| is floored at 1e-2,
an absolute bound of 1e-4 for gradients of unit-variance inputs.  Structure is exact: keys beyond a
sample's key length get dK = dV = 0, query rows with no visible key get dQ = 0.
"""
import numpy as np
import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from workloads import make_qkv

from tolerances import bf16_half_ulp

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
G_TOL = 1e-2


def run_bwd(q, k, v, do, **kw):
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    args = {n: (t.to(DEV) if torch.is_tensor(t) else t) for n, t in kw.items()}
    out, lse = ea.attention(qd, kd, vd, **args)
    dq, dk, dv = ea.attention_backward(qd, kd, vd, out, lse, dod, **args)
    ea.check_device_status()
    return dq, dk, dv


def assert_grad_close(name, g, ref):
    g = g.double().cpu().numpy()
    assert np.isfinite(g).all(), f"{name}: non-finite"
    scale = max(np.abs(ref).max(), 1e-2)
    err = np.abs(g - ref) - bf16_half_ulp(ref)
    worst = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= G_TOL * scale, (f"{name}: |d| - half_ulp = {err.max():.3e} > {G_TOL} * {scale:.3e} "
                                        f"at {worst}: {g[worst]} vs {ref[worst]}")


def check(B, Hq, Hkv, Nq, Nk, d, seed, causal=False, key_lens=None):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    do, _, _ = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed + 1)
    kw = dict(is_causal=causal)
    if key_lens is not None:
        kw["key_lens"] = torch.tensor(key_lens, dtype=torch.int32)
    dq, dk, dv = run_bwd(q, k, v, do, **kw)
    rq, rk, rv = oracle.attention_bwd(q, k, v, do, is_causal=causal, key_lens=key_lens)
    assert_grad_close("dq", dq, rq)
    assert_grad_close("dk", dk, rk)
    assert_grad_close("dv", dv, rv)
    return dq, dk, dv


@pytest.mark.parametrize("Nq,Nk", [(128, 128), (200, 260), (257, 300), (1, 130), (300, 1), (640, 512)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_shapes(Nq, Nk, d, causal):
    check(2, 2, 2, Nq, Nk, d, seed=Nq + 3 * Nk + d + causal, causal=causal)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_grouped_heads(d):
    check(2, 8, 2, 300, 300, d, seed=11 + d, causal=True)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_key_lens_structure(d):
    lens = [300, 0, 129, 1]
    dq, dk, dv = check(4, 2, 2, 200, 300, d, seed=21 + d, key_lens=lens)
    for b, n in enumerate(lens):
        assert torch.all(dk[b, :, n:] == 0) and torch.all(dv[b, :, n:] == 0)
    assert torch.all(dq[1] == 0)


def test_bwd_deterministic():
    q, k, v = make_qkv(1, 4, 2, 384, 384, 128, seed=31)
    do, _, _ = make_qkv(1, 4, 2, 384, 384, 128, seed=32)
    a = run_bwd(q, k, v, do, is_causal=True)
    b = run_bwd(q, k, v, do, is_causal=True)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


# ----------------------------------------------- score and mask variants
def check_variant(B, Hq, Hkv, Nq, Nk, d, seed, causal=False, mask=None, softcap=0.0, mask2d=None):
    """attn_bwd_ex against the backward oracle with the same variant; the GPU
    forward (attn_fwd with the mask, or attn_fwd_mod) provides O and LSE."""
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    do, _, _ = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed + 1)
    kw = dict(is_causal=causal, softcap=softcap, mask2d=mask2d)
    if mask is not None:
        kw["attn_mask"] = mask
    dq, dk, dv = run_bwd(q, k, v, do, **kw)
    rq, rk, rv = oracle.attention_bwd(q, k, v, do, is_causal=causal, softcap=softcap, mask2d=mask2d,
                                      mask=None if mask is None else mask.double().numpy())
    assert_grad_close("dq", dq, rq)
    assert_grad_close("dk", dk, rk)
    assert_grad_close("dv", dv, rv)
    return dq, dk, dv


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_softcap(d, causal):
    """A cap of 1 on scores of standard deviation 1: tanh bends most of them."""
    check_variant(2, 4, 2, 300, 260, d, seed=41 + d + causal, causal=causal, softcap=1.0)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_additive_mask(d):
    g = torch.Generator().manual_seed(7)
    mask = torch.randn(2, 2, 200, 260, generator=g) * 2.0
    mask[0, 1, :, 100:] = -float("inf")   # padding-like stripe
    mask[1, 0, 7, :] = -float("inf")      # a query row with no key
    dq, dk, dv = check_variant(2, 2, 2, 200, 260, d, seed=51 + d, mask=mask)
    assert torch.all(dq[1, 0, 7] == 0)


def test_bwd_additive_mask_broadcast_causal():
    g = torch.Generator().manual_seed(8)
    mask = torch.randn(1, 1, 257, 257, generator=g)
    check_variant(2, 4, 4, 257, 257, 128, seed=61, causal=True, mask=mask)


@pytest.mark.parametrize("mask2d", [("neighborhood", 20, 3), ("window", 16, 4), ("window", 16, 4, 2)])
@pytest.mark.parametrize("d", [64, 128])
def test_bwd_mask2d(mask2d, d):
    check_variant(2, 2, 1, 400, 400, d, seed=71 + d, mask2d=mask2d)


def test_bwd_neighbourhood_softcap_causal():
    """The 56-wide grid of the ViT workload, radius 5, with the cap of 30."""
    check_variant(1, 2, 2, 56 * 6, 56 * 6, 64, seed=81, causal=True, softcap=30.0, mask2d=("neighborhood", 56, 5))


def test_bwd_variants_off_equal_plain():
    """attn_bwd_ex with every variant off and attn_bwd give the same bits."""
    q, k, v = make_qkv(1, 2, 2, 300, 300, 64, seed=91)
    do, _, _ = make_qkv(1, 2, 2, 300, 300, 64, seed=92)
    a = run_bwd(q, k, v, do)
    b = run_bwd(q, k, v, do, softcap=0.0, mask2d=None)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


@pytest.mark.parametrize("N,causal", [(4096, False), (2048, True)])
def test_bwd_long_head_against_the_oracle(N, causal):
    """One head of the long workload's shape (d = 128, N = 4096: each dK/dV CTA
    loops over 32 query blocks, each dQ CTA over 32 key blocks, 64 half blocks
    through the two TMEM buffers, as in the benchmark's launch; the causal case at
    N = 2048), every element of dQ, dK and dV against the oracle."""
    check(1, 1, 1, N, N, 128, seed=1100 + N + causal, causal=causal)
