"""Pins of the backward oracle's score and mask variants (additive mask,
soft-capping, 2-D neighbourhood and window masks), each against something
other than its own formulas:

- central finite differences of the forward oracle's loss sum(dO * O), in fp64,
  entry by entry (the forward oracle is pinned on its own in
  test_oracle_variants.py);
- torch autograd in float64 through a restatement of the forward in torch
  operations (scores, cap * tanh(x / cap), mask added, -inf outside the
  visible keys, softmax, P V): another code base reaching the same definition.

Planted mistakes in a copy of the backward oracle must fail one of them.
"""
import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).numpy()


def visible(Nq, Nk, is_causal=False, mask2d=None):
    """Boolean [Nq, Nk]: which keys each query row may see (2-D rule written
    from the grid coordinates, independently of the oracles)."""
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    ok = np.ones((Nq, Nk), dtype=bool)
    if is_causal:
        ok &= j <= i
    if mask2d is not None:
        W, size = mask2d[1], mask2d[2]
        ri, ci, rj, cj = i // W, i % W, j // W, j % W
        if mask2d[0] == "neighborhood":
            ok &= (np.abs(ri - rj) < size) & (np.abs(ci - cj) < size)
        else:
            sh = mask2d[3] if len(mask2d) > 3 else 0
            ok &= ((ri + sh) // size == (rj + sh) // size) & ((ci + sh) // size == (cj + sh) // size)
    return ok


def torch_grads(q, k, v, do, *, scale, mask=None, softcap=0.0, is_causal=False, mask2d=None):
    q, k, v, do = (torch.tensor(t, dtype=torch.float64, requires_grad=i < 3) for i, t in enumerate((q, k, v, do)))
    group = q.shape[1] // k.shape[1]
    kk, vv = k.repeat_interleave(group, dim=1), v.repeat_interleave(group, dim=1)
    x = scale * q @ kk.transpose(-1, -2)
    if softcap:
        x = softcap * torch.tanh(x / softcap)
    if mask is not None:
        x = x + torch.tensor(mask, dtype=torch.float64)
    ok = torch.tensor(visible(q.shape[2], k.shape[2], is_causal, mask2d))
    x = x.masked_fill(~ok, float("-inf"))
    # rows with no visible key give P = 0 (and no gradient): softmax of a
    # finite stand-in row, multiplied by 0
    has_key = torch.isfinite(x).any(dim=-1, keepdim=True)
    p = torch.softmax(torch.where(has_key, x, torch.zeros_like(x)), dim=-1) * has_key
    o = p @ vv
    (o * do).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


CASES = [
    dict(name="softcap", B=1, Hq=2, Hkv=1, Nq=6, Nk=7, d=3, kw=dict(scale=1.3, softcap=1.5)),
    dict(name="softcap_causal", B=1, Hq=2, Hkv=2, Nq=6, Nk=6, d=4, kw=dict(scale=2.0, softcap=0.8, is_causal=True)),
    dict(name="additive", B=2, Hq=2, Hkv=1, Nq=5, Nk=6, d=3, kw=dict(scale=0.7), mask=True),
    dict(name="neighborhood", B=1, Hq=2, Hkv=1, Nq=12, Nk=12, d=3,
         kw=dict(scale=0.9, mask2d=("neighborhood", 4, 2))),
    dict(name="window_shift", B=1, Hq=1, Hkv=1, Nq=16, Nk=16, d=3,
         kw=dict(scale=0.9, mask2d=("window", 4, 2, 1), softcap=2.0)),
]


def case_inputs(c):
    B, Hq, Hkv, Nq, Nk, d = (c[x] for x in ("B", "Hq", "Hkv", "Nq", "Nk", "d"))
    q, k, v, do = rnd((B, Hq, Nq, d), 1), rnd((B, Hkv, Nk, d), 2), rnd((B, Hkv, Nk, d), 3), rnd((B, Hq, Nq, d), 4)
    kw = dict(c["kw"])
    if c.get("mask"):
        m = rnd((B, Hq, Nq, Nk), 5, 2.0)
        m[0, 1, 2, :] = -np.inf          # a row with no key
        m[1, 0, :, 4] = -np.inf          # a key no row sees
        kw["mask"] = m
    return q, k, v, do, kw


def fd_errors(q, k, v, do, kw, grads):
    """Max |analytic - central difference| over every entry of dQ, dK, dV."""
    eps = 1e-6
    fwd_kw = {x: kw[x] for x in kw}

    def loss(qq, kk, vv):
        o, _ = oracle.attention(qq, kk, vv, **fwd_kw)
        return float((np.nan_to_num(o) * do).sum())

    worst = 0.0
    for idx, (t, g) in enumerate(zip((q, k, v), grads)):
        for pos in np.ndindex(*t.shape):
            tp, tm = t.copy(), t.copy()
            tp[pos] += eps
            tm[pos] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = tp, tm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            worst = max(worst, abs(fd - g[pos]))
    return worst


@pytest.mark.parametrize("c", CASES, ids=[c["name"] for c in CASES])
def test_against_finite_differences(c):
    q, k, v, do, kw = case_inputs(c)
    grads = oracle.attention_bwd(q, k, v, do, **kw)
    assert fd_errors(q, k, v, do, kw, grads) < 1e-7


@pytest.mark.parametrize("c", CASES, ids=[c["name"] for c in CASES])
def test_against_torch_autograd(c):
    q, k, v, do, kw = case_inputs(c)
    ours = oracle.attention_bwd(q, k, v, do, **kw)
    ref = torch_grads(q, k, v, do, **kw)
    for a, b in zip(ours, ref):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


MUTANTS = {
    "softcap_derivative_dropped": ("for (int j = 0; j < Nk; ++j) dp[j] *= c[j];", ""),
    "softcap_derivative_sign": ("c[j] = 1.0 - th * th;", "c[j] = 1.0 + th * th;"),
    "mask_before_cap": ("if (mrow) p[j] += mrow[j];", "if (mrow) p[j] += 2.0 * mrow[j];"),
    "window_without_shift": ("return (ri + sh) / w == (rj + sh) / w && (ci + sh) / w == (cj + sh) / w;",
                             "return ri / w == rj / w && ci / w == cj / w;"),
    "neighbourhood_inclusive": ("return dr < a->m2_size && dc < a->m2_size;",
                                "return dr <= a->m2_size && dc <= a->m2_size;"),
    "mask2d_ignored": ("|| !bwd_allowed_2d(a, i, j)", ""),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    before, after = MUTANTS[name]
    src = oracle.source_text_bwd()
    assert src.count(before) == 1, f"mutation anchor of {name} not found"
    lib = oracle.compile_variant_bwd(src.replace(before, after), str(tmp_path / f"mut_{name}.so"))
    caught = False
    for c in CASES:
        q, k, v, do, kw = case_inputs(c)
        got = oracle.attention_bwd(q, k, v, do, lib=lib, **kw)
        ref = torch_grads(q, k, v, do, **kw)
        if any(not np.allclose(a, b, rtol=1e-8, atol=1e-10) for a, b in zip(got, ref)):
            caught = True
            break
    assert caught, f"pins miss the mutant {name}"
