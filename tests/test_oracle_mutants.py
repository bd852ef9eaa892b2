"""Plant a mistake in a copy of the oracle (on the CPU) and check that the pins
catch it.  Each mutant is a plausible slip: a dropped scale, a sign flip in the
max shift, an off-by-one mask, the wrong K/V head, a log in the wrong base, a
transposed operand, a missing normalisation.
"""
import math

import numpy as np
import pytest
import torch

import oracle

MUTANTS = {
    "dropped_scale": ("s[j] = a->scale * dot;", "s[j] = dot;"),
    "sign_of_shift": ("s[j] = exp(s[j] - M);", "s[j] = exp(M - s[j]);"),
    "causal_off_by_one": ("(a->is_causal && j > i)", "(a->is_causal && j >= i)"),
    "padding_off_by_one": ("if (j >= len ||", "if (j > len ||"),
    "wrong_kv_head": ("const int hk = h / group;", "const int hk = h % a->Hkv;"),
    "lse_log2": ("M + log(L)", "M + log2(L)"),
    "v_transposed": ("oi[t] += s[j] * vj[t];", "oi[t] += s[j] * vh[(int64_t)t * a->Nk + j % a->Nk];"),
    "no_normalisation": ("oi[t] /= L;", "oi[t] /= 1.0;"),
    "mask_before_scale": ("s[j] = a->scale * dot;\n        if (a->softcap > 0.0) s[j] = a->softcap * tanh(s[j] / a->softcap);\n        if (mrow) s[j] += mrow[j];",
                          "s[j] = dot;\n        if (mrow) s[j] += mrow[j];\n        s[j] *= a->scale;"),
}


def rnd(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).numpy()


def pin_battery(lib):
    """Runs a compact subset of the pins against ``lib``; returns the names of the
    pins that fail."""
    failed = []

    def check(name, ok):
        if not ok:
            failed.append(name)

    # brute force (pure Python loops) on a small grouped, causal, padded case with a mask
    B, Hq, Hkv, Nq, Nk, d = 2, 4, 2, 5, 7, 3
    q, k, v = rnd((B, Hq, Nq, d), 1, 2.0), rnd((B, Hkv, Nk, d), 2), rnd((B, Hkv, Nk, d), 3)
    mask = rnd((1, 1, Nq, Nk), 4)
    for causal, lens, mk in [(True, [7, 3], None), (False, None, mask)]:
        o, lse = oracle.attention(q, k, v, is_causal=causal, key_lens=lens, mask=mk, scale=0.6, lib=lib)
        o2, lse2 = oracle.attention_loops(q, k, v, is_causal=causal, key_lens=lens, mask=mk, scale=0.6)
        check("brute_force_O", np.allclose(o, o2, rtol=0, atol=1e-12))
        check("brute_force_LSE", np.allclose(lse, lse2, rtol=0, atol=1e-12))
    # K = 0 closed form
    kz = np.zeros((1, 1, 6, 3))
    vz = rnd((1, 1, 6, 3), 5)
    o, lse = oracle.attention(rnd((1, 1, 4, 3), 6), kz, vz, scale=2.0, lib=lib)
    check("zero_keys_mean", np.allclose(o[0, 0], vz[0, 0].mean(axis=0), atol=1e-14))
    check("zero_keys_lse", np.allclose(lse, math.log(6), atol=1e-14))
    # single dominant score closed form
    qd = np.zeros((1, 1, 1, 2)); qd[0, 0, 0, 0] = 2.0
    kd = np.zeros((1, 1, 5, 2)); kd[0, 0, 3, 0] = 2.0
    vd = rnd((1, 1, 5, 2), 7)
    o, lse = oracle.attention(qd, kd, vd, scale=0.5, lib=lib)
    s = 2.0
    exp_o = (math.exp(s) * vd[0, 0, 3] + vd[0, 0].sum(0) - vd[0, 0, 3]) / (math.exp(s) + 4)
    check("dominant_O", np.allclose(o[0, 0, 0], exp_o, atol=1e-13))
    check("dominant_LSE", abs(lse[0, 0, 0] - math.log(math.exp(s) + 4)) < 1e-13)
    # library special case: torch SDPA (float64, CPU)
    o, _ = oracle.attention(q, k, v, is_causal=True, scale=0.6, lib=lib)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k).repeat_interleave(2, 1),
        torch.from_numpy(v).repeat_interleave(2, 1), is_causal=True, scale=0.6)
    check("sdpa", np.allclose(o, ref.numpy(), atol=1e-12))
    return failed


def test_unmutated_oracle_passes_battery():
    assert pin_battery(None) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    before, after = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    lib = oracle.compile_variant(src.replace(before, after), str(tmp_path / f"mut_{name}.so"))
    failed = pin_battery(lib)
    assert failed, f"planted mistake '{name}' passed every pin"
