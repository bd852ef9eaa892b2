"""Pins of the backward oracle (dQ, dK, dV for an upstream dO), each against
something other than its own formulas:

- central finite differences of the forward oracle's loss sum(dO * O), in fp64,
  entry by entry on small grouped / causal / padded problems;
- torch autograd through scaled_dot_product_attention in float64 on the CPU
  (a library special case: no padding, grouped heads expanded);
- closed forms: when every V row is the same vector, O does not depend on Q or
  K, so dQ = dK = 0 exactly, and dV = P^T dO sums to sum_i dO_i over keys;
  a query row with no visible key gets dQ = 0 and gives its keys nothing.

Planted mistakes in a copy of the backward oracle must fail one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).numpy()


def loss(q, k, v, do, **kw):
    o, _ = oracle.attention(q, k, v, **kw)
    return float((np.nan_to_num(o) * do).sum())


def finite_difference_failures(lib=None):
    failed = []
    cases = [
        dict(B=1, Hq=2, Hkv=1, Nq=5, Nk=6, d=3, kw=dict(scale=0.7)),
        dict(B=2, Hq=2, Hkv=2, Nq=6, Nk=6, d=4, kw=dict(scale=0.5, is_causal=True)),
        dict(B=2, Hq=4, Hkv=2, Nq=4, Nk=7, d=3, kw=dict(scale=0.9, key_lens=[7, 3])),
    ]
    eps = 1e-6
    for ci, c in enumerate(cases):
        B, Hq, Hkv, Nq, Nk, d = c["B"], c["Hq"], c["Hkv"], c["Nq"], c["Nk"], c["d"]
        q, k, v = rnd((B, Hq, Nq, d), 10 + ci, 1.5), rnd((B, Hkv, Nk, d), 20 + ci), rnd((B, Hkv, Nk, d), 30 + ci)
        do = rnd((B, Hq, Nq, d), 40 + ci)
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, lib=lib, **c["kw"])
        rng = np.random.default_rng(ci)
        for name, x, g in [("dq", q, dq), ("dk", k, dk), ("dv", v, dv)]:
            for _ in range(6):
                idx = tuple(rng.integers(0, n) for n in x.shape)
                xp, xm = x.copy(), x.copy()
                xp[idx] += eps
                xm[idx] -= eps
                args = {"q": q, "k": k, "v": v}
                key = name[1]
                num = (loss(**{**args, key: xp}, do=do, **c["kw"]) - loss(**{**args, key: xm}, do=do, **c["kw"])) / (2 * eps)
                if not abs(num - g[idx]) < 1e-6 * max(1.0, abs(num)):
                    failed.append(f"fd case {ci} {name}{idx}: {num} vs {g[idx]}")
                    break
    return failed


def sdpa_failures(lib=None):
    failed = []
    B, Hq, Hkv, Nq, Nk, d = 2, 4, 2, 9, 11, 5
    q, k, v = rnd((B, Hq, Nq, d), 1, 1.5), rnd((B, Hkv, Nk, d), 2), rnd((B, Hkv, Nk, d), 3)
    do = rnd((B, Hq, Nq, d), 4)
    for causal in (False, True):
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(
            tq, tk.repeat_interleave(Hq // Hkv, 1), tv.repeat_interleave(Hq // Hkv, 1), is_causal=causal, scale=0.6)
        o.backward(torch.tensor(do))
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=0.6, is_causal=causal, lib=lib)
        for name, a, b in [("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)]:
            if not np.allclose(a, b.numpy(), atol=1e-12, rtol=0):
                failed.append(f"sdpa causal={causal} {name}")
    return failed


def closed_form_failures(lib=None):
    failed = []
    B, Hq, Hkv, Nq, Nk, d = 1, 2, 1, 6, 8, 4
    q, k = rnd((B, Hq, Nq, d), 5, 2.0), rnd((B, Hkv, Nk, d), 6)
    v = np.broadcast_to(rnd((1, 1, 1, d), 7), (B, Hkv, Nk, d)).copy()
    do = rnd((B, Hq, Nq, d), 8)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=0.8, lib=lib)
    if not (np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13):
        failed.append("constant V gives zero dQ, dK")
    if not np.allclose(dv.sum(axis=2), do.sum(axis=(1, 2))[:, None], atol=1e-12):
        failed.append("dV columns sum to sum of dO")
    # a query row with no visible key (key length 0)
    q2, k2, v2 = rnd((2, 1, 3, d), 9), rnd((2, 1, 5, d), 10), rnd((2, 1, 5, d), 11)
    do2 = rnd((2, 1, 3, d), 12)
    dq2, dk2, dv2 = oracle.attention_bwd(q2, k2, v2, do2, key_lens=[0, 5], lib=lib)
    if not (np.all(dq2[0] == 0) and np.all(dk2[0] == 0) and np.all(dv2[0] == 0)):
        failed.append("empty key set")
    return failed


def test_backward_finite_differences():
    assert finite_difference_failures() == []


def test_backward_matches_torch_autograd_fp64():
    assert sdpa_failures() == []


def test_backward_closed_forms():
    assert closed_form_failures() == []


BWD_MUTANTS = {
    "no_delta": ("dp[j] = p[j] * (dp[j] - D);", "dp[j] = p[j] * dp[j];"),
    "dq_without_scale": ("dQ[(int64_t)i * d + t] = a->scale * s;", "dQ[(int64_t)i * d + t] = s;"),
    "dk_uses_dO": ("sk += dP[(int64_t)i * Nk + j] * Q[(int64_t)i * d + t];",
                   "sk += dP[(int64_t)i * Nk + j] * dO[(int64_t)i * d + t];"),
    "dv_uses_dS": ("sv += P[(int64_t)i * Nk + j] * dO[(int64_t)i * d + t];",
                   "sv += dP[(int64_t)i * Nk + j] * dO[(int64_t)i * d + t];"),
    "group_not_summed": ("dK[(int64_t)j * d + t] += a->scale * sk;", "dK[(int64_t)j * d + t] = a->scale * sk;"),
    "causal_off_by_one": ("(a->is_causal && j > i)", "(a->is_causal && j >= i)"),
    "dp_transposed_v": ("s += dO[(int64_t)i * d + t] * V[(int64_t)j * d + t];",
                        "s += dO[(int64_t)i * d + t] * V[(int64_t)t * d % (Nk * d) + j % d];"),
}


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_pins_catch_planted_mistake(name, tmp_path):
    before, after = BWD_MUTANTS[name]
    src = oracle.source_text_bwd()
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    lib = oracle.compile_variant_bwd(src.replace(before, after), str(tmp_path / f"mut_{name}.so"))
    failed = sdpa_failures(lib) + closed_form_failures(lib)
    if not failed:
        failed = finite_difference_failures(lib)
    assert failed, f"planted mistake '{name}' passed every pin"
