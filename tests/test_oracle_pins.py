"""Pins for the fp64 oracle: closed forms, invariants, brute force and a library
special case.  None of these compares the oracle with itself.  CPU only.

Each pin is chosen so that a plausible slip in the oracle (a dropped scale, a
wrong sign in the max shift, a transposed operand, an off-by-one in a mask, the
wrong K/V head for a grouped query head, a log in the wrong base) fails at least
one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_qkv

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rnd(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).numpy()


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,lens", [
    (1, 1, 1, 1, 1, 1, False, None),
    (1, 2, 1, 3, 5, 4, False, None),
    (2, 2, 2, 5, 5, 3, True, None),
    (2, 4, 2, 4, 7, 8, False, [3, 7]),
    (2, 2, 1, 6, 6, 2, True, [0, 4]),
    (1, 3, 3, 7, 3, 5, True, None),   # causal with Nq > Nk (top-left)
    (1, 1, 1, 2, 9, 4, True, None),   # causal with Nq < Nk
])
def test_brute_force_loops(B, Hq, Hkv, Nq, Nk, d, causal, lens):
    q = rnd((B, Hq, Nq, d), 1)
    k = rnd((B, Hkv, Nk, d), 2)
    v = rnd((B, Hkv, Nk, d), 3)
    o, lse = oracle.attention(q, k, v, is_causal=causal, key_lens=lens, scale=0.37)
    o2, lse2 = oracle.attention_loops(q, k, v, is_causal=causal, key_lens=lens, scale=0.37)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse2)
    np.testing.assert_allclose(lse[fin], lse2[fin], rtol=0, atol=1e-12)


def test_brute_force_additive_mask():
    B, H, Nq, Nk, d = 1, 2, 4, 6, 3
    q, k, v = rnd((B, H, Nq, d), 4), rnd((B, H, Nk, d), 5), rnd((B, H, Nk, d), 6)
    mask = rnd((1, H, Nq, Nk), 7, 2.0)
    mask[0, 1, 2, :3] = -np.inf
    o, lse = oracle.attention(q, k, v, mask=mask)
    o2, lse2 = oracle.attention_loops(q, k, v, mask=mask)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


# ------------------------------------------------- online == two-pass (pages)
@pytest.mark.parametrize("block", [1, 7, 16, 128])
@pytest.mark.parametrize("causal,lens", [(False, None), (True, None), (False, [5, 40])])
def test_online_matches_two_pass(block, causal, lens):
    """Tiled online softmax reaches the two-pass result (jsqmd.com/news/722897 s2.2)."""
    B, Hq, Hkv, N, d = 2, 4, 2, 40, 16
    q, k, v = rnd((B, Hq, N, d), 10, 3.0), rnd((B, Hkv, N, d), 11), rnd((B, Hkv, N, d), 12)
    o, lse = oracle.attention(q, k, v, is_causal=causal, key_lens=lens)
    o2, lse2 = oracle.attention_online(q, k, v, block=block, is_causal=causal, key_lens=lens)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


# ----------------------------------------------------------- closed forms
def test_probability_rows_sum_to_one_and_o_is_pv():
    B, Hq, Hkv, N, d = 2, 2, 1, 33, 8
    q, k, v = rnd((B, Hq, N, d), 20, 2.0), rnd((B, Hkv, N, d), 21), rnd((B, Hkv, N, d), 22)
    lens = [33, 9]
    p = oracle.probabilities(q, k, is_causal=True, key_lens=lens)
    assert np.all(np.abs(p.sum(-1) - 1.0) < 1e-14)
    assert np.all(p >= 0)
    o, _ = oracle.attention(q, k, v, is_causal=True, key_lens=lens)
    np.testing.assert_allclose(o, np.einsum("bhij,bhjd->bhid", p, np.repeat(v, 2, axis=1)),
                               rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_keys_give_mean_of_valid_values(causal):
    """K = 0: every score is 0, so O_i is the mean of V over the valid keys and
    LSE_i = ln(n_valid) for any scale."""
    B, H, Nq, Nk, d = 2, 3, 9, 11, 5
    q = rnd((B, H, Nq, d), 30)
    k = np.zeros((B, H, Nk, d))
    v = rnd((B, H, Nk, d), 31)
    lens = [11, 4]
    o, lse = oracle.attention(q, k, v, is_causal=causal, key_lens=lens, scale=1.7)
    for b in range(B):
        for i in range(Nq):
            n = min(lens[b], i + 1) if causal else lens[b]
            np.testing.assert_allclose(o[b, :, i], v[b, :, :n].mean(axis=1), rtol=0, atol=1e-14)
            np.testing.assert_allclose(lse[b, :, i], math.log(n), rtol=0, atol=1e-14)


def test_identical_keys_give_mean_and_shifted_lse():
    B, H, Nq, Nk, d = 1, 2, 5, 13, 6
    q = rnd((B, H, Nq, d), 40)
    k0 = rnd((d,), 41)
    k = np.broadcast_to(k0, (B, H, Nk, d)).copy()
    v = rnd((B, H, Nk, d), 42)
    scale = 0.25
    o, lse = oracle.attention(q, k, v, scale=scale)
    for h in range(H):
        for i in range(Nq):
            s = scale * float(q[0, h, i] @ k0)
            np.testing.assert_allclose(o[0, h, i], v[0, h].mean(axis=0), rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[0, h, i], s + math.log(Nk), rtol=0, atol=1e-12)


@pytest.mark.parametrize("alpha", [1.0, 2.0, 3.0, 8.0])
def test_single_dominant_score(alpha):
    """Q row = alpha*e1, K row j* = alpha*e1, other K rows 0: s = scale*alpha^2 at
    j*, 0 elsewhere, so O = (e^s v_j* + sum_{j!=j*} v_j) / (e^s + n - 1) and
    LSE = ln(e^s + n - 1); as s grows O -> v_j*."""
    Nk, d, jstar, scale = 10, 4, 6, 0.5
    q = np.zeros((1, 1, 1, d)); q[0, 0, 0, 0] = alpha
    k = np.zeros((1, 1, Nk, d)); k[0, 0, jstar, 0] = alpha
    v = rnd((1, 1, Nk, d), 50)
    o, lse = oracle.attention(q, k, v, scale=scale)
    s = scale * alpha * alpha
    others = v[0, 0].sum(axis=0) - v[0, 0, jstar]
    expect = (math.exp(s) * v[0, 0, jstar] + others) / (math.exp(s) + Nk - 1)
    np.testing.assert_allclose(o[0, 0, 0], expect, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0, 0], math.log(math.exp(s) + Nk - 1), rtol=0, atol=1e-13)


def test_single_dominant_score_limit():
    Nk, d, jstar = 8, 2, 3
    q = np.zeros((1, 1, 1, d)); q[0, 0, 0, 1] = 30.0
    k = np.zeros((1, 1, Nk, d)); k[0, 0, jstar, 1] = 30.0
    v = rnd((1, 1, Nk, d), 51)
    o, lse = oracle.attention(q, k, v, scale=1.0)  # s = 900: e^-900 underflows
    np.testing.assert_array_equal(o[0, 0, 0], v[0, 0, jstar])
    assert lse[0, 0, 0] == 900.0


def test_unit_values_give_unit_output():
    B, H, N, d = 2, 2, 17, 3
    q, k = rnd((B, H, N, d), 60, 4.0), rnd((B, H, N, d), 61)
    v = np.ones((B, H, N, d))
    o, _ = oracle.attention(q, k, v, is_causal=True, key_lens=[17, 5])
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def test_causal_first_row_and_single_key():
    B, H, N, d = 1, 2, 6, 4
    q, k, v = rnd((B, H, N, d), 70), rnd((B, H, N, d), 71), rnd((B, H, N, d), 72)
    o, lse = oracle.attention(q, k, v, is_causal=True, scale=0.3)
    np.testing.assert_array_equal(o[0, :, 0], v[0, :, 0])
    np.testing.assert_allclose(lse[0, :, 0], 0.3 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0]),
                               rtol=0, atol=1e-14)
    o1, _ = oracle.attention(q, k, v, key_lens=[1])
    np.testing.assert_array_equal(o1[0], np.broadcast_to(v[0, :, :1], o1[0].shape))


def test_causal_last_row_equals_full_row():
    B, H, N, d = 1, 1, 9, 4
    q, k, v = rnd((B, H, N, d), 73), rnd((B, H, N, d), 74), rnd((B, H, N, d), 75)
    oc, lc = oracle.attention(q, k, v, is_causal=True)
    of, lf = oracle.attention(q, k, v, is_causal=False)
    np.testing.assert_array_equal(oc[0, 0, -1], of[0, 0, -1])
    assert lc[0, 0, -1] == lf[0, 0, -1]
    assert not np.allclose(oc[0, 0, 0], of[0, 0, 0])


def test_empty_key_set_gives_zero_and_neg_inf():
    q, k, v = rnd((2, 1, 3, 4), 80), rnd((2, 1, 5, 4), 81), rnd((2, 1, 5, 4), 82)
    o, lse = oracle.attention(q, k, v, key_lens=[0, 5])
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def test_masked_keys_contribute_nothing():
    """Changing K/V at masked positions (padding or above the diagonal) leaves O
    and LSE bitwise unchanged."""
    B, H, N, d = 2, 2, 24, 8
    q, k, v = rnd((B, H, N, d), 90), rnd((B, H, N, d), 91), rnd((B, H, N, d), 92)
    lens = [24, 10]
    o, lse = oracle.attention(q, k, v, is_causal=True, key_lens=lens)
    k2, v2 = k.copy(), v.copy()
    k2[1, :, 10:] = 1e4 * rnd((H, N - 10, d), 93)
    v2[1, :, 10:] = -1e4
    o2, lse2 = oracle.attention(q, k2, v2, is_causal=True, key_lens=lens)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    # causal: the last key only reaches the last row
    k3, v3 = k.copy(), v.copy()
    k3[0, :, -1] = 7e3
    v3[0, :, -1] = 5e3
    o3, lse3 = oracle.attention(q, k3, v3, is_causal=True, key_lens=lens)
    np.testing.assert_array_equal(o3[0, :, :-1], o[0, :, :-1])
    assert not np.array_equal(o3[0, :, -1], o[0, :, -1])


def test_constant_mask_shifts_lse_only():
    B, H, N, d = 1, 2, 12, 4
    q, k, v = rnd((B, H, N, d), 100), rnd((B, H, N, d), 101), rnd((B, H, N, d), 102)
    o, lse = oracle.attention(q, k, v)
    o2, lse2 = oracle.attention(q, k, v, mask=np.full((1, 1, 1, 1), 2.5))
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse2, lse + 2.5, rtol=0, atol=1e-13)


def test_key_permutation_invariance():
    B, H, N, d = 1, 2, 15, 6
    q, k, v = rnd((B, H, N, d), 110), rnd((B, H, N, d), 111), rnd((B, H, N, d), 112)
    perm = np.random.default_rng(3).permutation(N)
    o, lse = oracle.attention(q, k, v)
    o2, lse2 = oracle.attention(q, k[:, :, perm], v[:, :, perm])
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)


def test_grouped_heads_equal_repeated_heads():
    B, Hq, Hkv, N, d = 2, 6, 2, 10, 4
    q, k, v = rnd((B, Hq, N, d), 120), rnd((B, Hkv, N, d), 121), rnd((B, Hkv, N, d), 122)
    o, lse = oracle.attention(q, k, v, is_causal=True)
    o2, lse2 = oracle.attention(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), is_causal=True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    # and query head 3 must read K/V head 1 (contiguous groups), not head 0
    o3, _ = oracle.attention(q[:, 3:4], k[:, 1:2], v[:, 1:2], is_causal=True)
    np.testing.assert_array_equal(o3[:, 0], o[:, 3])


def test_row_subset_matches_full():
    B, H, N, d = 1, 2, 30, 8
    q, k, v = rnd((B, H, N, d), 130), rnd((B, H, N, d), 131), rnd((B, H, N, d), 132)
    o, lse = oracle.attention(q, k, v, is_causal=True)
    rows = [0, 7, 29]
    o2, lse2 = oracle.attention(q, k, v, is_causal=True, rows=rows)
    np.testing.assert_array_equal(o2[:, :, rows], o[:, :, rows])
    np.testing.assert_array_equal(lse2[:, :, rows], lse[:, :, rows])
    assert np.isnan(o2[0, 0, 1]).all()


def test_threads_do_not_change_results():
    B, H, N, d = 2, 3, 20, 8
    q, k, v = rnd((B, H, N, d), 140), rnd((B, H, N, d), 141), rnd((B, H, N, d), 142)
    o1, l1 = oracle.attention(q, k, v, n_threads=1)
    o4, l4 = oracle.attention(q, k, v, n_threads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(l1, l4)


def test_rejects_bad_arguments():
    q, k, v = rnd((1, 3, 4, 2), 150), rnd((1, 2, 4, 2), 151), rnd((1, 2, 4, 2), 152)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v)  # Hq % Hkv != 0
    q = rnd((1, 2, 4, 2), 153)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, key_lens=[5])  # key_len > Nk


# -------------------------------------------------- library special case
@pytest.mark.parametrize("causal,lens,gqa", [(False, None, False), (True, None, False),
                                            (False, [13, 31], False), (True, None, True)])
def test_matches_torch_sdpa_math_fp64(causal, lens, gqa):
    """torch's CPU scaled_dot_product_attention in float64 is an independent code
    base that reaches the same textbook definition."""
    B, Hq, N, d = 2, 4, 31, 16
    Hkv = 2 if gqa else Hq
    q, k, v = rnd((B, Hq, N, d), 160, 2.0), rnd((B, Hkv, N, d), 161), rnd((B, Hkv, N, d), 162)
    o, _ = oracle.attention(q, k, v, is_causal=causal, key_lens=lens, scale=0.2)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    mask = None
    if lens is not None:
        j = torch.arange(N)
        mask = torch.zeros(B, 1, 1, N, dtype=torch.float64)
        mask[(j[None, :] >= torch.tensor(lens)[:, None])[:, None, None, :]] = -math.inf
    if gqa:
        tk, tv = tk.repeat_interleave(Hq // Hkv, dim=1), tv.repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask, is_causal=causal, scale=0.2)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------ golden values
def test_flop_count_matches_page_figure():
    """jsqmd.com/news/722897 section 3.1 prints ~4N^2 d = 8.6 GFLOP for one head at
    N=4096, d=128; the benchmark's FLOP count must agree."""
    path = os.path.join(GOLDEN, "flash_flops_one_head.txt")
    vals = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            key, val = line.split("=")
            vals[key.strip()] = float(val)
    from workloads import Workload
    w = Workload("one_head", 1, 1, 1, int(vals["N"]), int(vals["N"]), int(vals["d"]))
    assert abs(w.flops() / 1e9 - vals["gflop"]) < 0.05
    assert WORKLOADS["long_causal"].flops() * 2 == WORKLOADS["long"].flops()


def test_tiny_workload_full_oracle_is_fast_and_finite():
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.seed)
    o, lse = oracle.attention(q, k, v)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    # softmax weights are convex: every output lies inside the range of V
    vv = v.double().numpy()
    assert (o <= vv.max(axis=2, keepdims=True) + 1e-12).all()
    assert (o >= vv.min(axis=2, keepdims=True) - 1e-12).all()
