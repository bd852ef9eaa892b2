"""Pins of the oracle's score and mask variants, each against something other
than the oracle's own formula:

soft-capping (the score_mod example of the PyTorch attention article,
atyun.com/61003.html): the limit cap -> infinity is plain attention; the
deviation from it shrinks as 1/cap^2 (cap * tanh(x / cap) = x - x^3 / (3 cap^2)
+ ...); saturated scores give closed-form weights e^(+-cap); an additive mask
is added after the cap.

2-D masks (the neighbourhood mask_mod of the same article, the window attention
of xxmr.cn/news/81028 section 3.2): radius or window large enough is no mask;
radius 1 or window 1 leaves each token alone (O = V, LSE = own score); windows
equal plain attention on the gathered tokens of each window (the reshape and
gather route of the same section); a neighbourhood equals plain attention of
each query over the keys of its grid slice.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).numpy()


def qkv(B, H, N, d, seed):
    return rnd((B, H, N, d), seed, 1.5), rnd((B, H, N, d), seed + 1), rnd((B, H, N, d), seed + 2)


# ------------------------------------------------------------------ soft-capping
def softcap_failures(lib=None):
    failed = []
    q, k, v = qkv(2, 2, 9, 4, 10)
    o0, l0 = oracle.attention(q, k, v, scale=0.7, lib=lib)
    o, l = oracle.attention(q, k, v, scale=0.7, softcap=1e7, lib=lib)
    if not (np.abs(o - o0).max() < 1e-9 and np.abs(l - l0).max() < 1e-9):
        failed.append("limit")
    # deviation ~ 1/cap^2: halving 1/cap quarters it
    _, la = oracle.attention(q, k, v, scale=0.7, softcap=40.0, lib=lib)
    _, lb = oracle.attention(q, k, v, scale=0.7, softcap=80.0, lib=lib)
    ratio = np.abs(la - l0).max() / np.abs(lb - l0).max()
    if not 3.7 < ratio < 4.3:
        failed.append(f"asymptotic ratio {ratio}")
    # saturation: scores +-250 -> logits +-cap; keys 0..2 positive, 3..7 negative
    d = 4
    qs = np.zeros((1, 1, 1, d)); qs[..., 0] = 50.0
    ks = np.zeros((1, 1, 8, d)); ks[0, 0, :3, 0] = 10.0; ks[0, 0, 3:, 0] = -10.0
    vs = rnd((1, 1, 8, d), 20)
    cap = 2.0
    o, l = oracle.attention(qs, ks, vs, scale=0.5, softcap=cap, lib=lib)
    w = np.array([math.exp(cap)] * 3 + [math.exp(-cap)] * 5)
    if not (abs(l[0, 0, 0] - math.log(w.sum())) < 1e-12 and
            np.allclose(o[0, 0, 0], (w[:, None] * vs[0, 0]).sum(0) / w.sum(), atol=1e-12)):
        failed.append("saturation")
    # an additive mask comes after the cap: saturated logit +-cap, then + mask
    mask = np.zeros((1, 1, 1, 8)); mask[..., 4] = 3.0; mask[..., 1] = -np.inf
    o, l = oracle.attention(qs, ks, vs, scale=0.5, softcap=cap, mask=mask, lib=lib)
    w2 = np.array([math.exp(cap), 0.0, math.exp(cap), math.exp(-cap), math.exp(3.0 - cap)] + [math.exp(-cap)] * 3)
    if not (abs(l[0, 0, 0] - math.log(w2.sum())) < 1e-12 and
            np.allclose(o[0, 0, 0], (w2[:, None] * vs[0, 0]).sum(0) / w2.sum(), atol=1e-12)):
        failed.append("mask_after_cap")
    return failed


def test_softcap_pins():
    assert softcap_failures() == []


# -------------------------------------------------------------------- 2-D masks
def gather_windows(Hg, Wg, w, shift):
    """Token indices of each window: rows [a*w - shift, (a+1)*w - shift) and the
    same for columns, clipped to the grid (index slicing of a 2-D array)."""
    grid = np.arange(Hg * Wg).reshape(Hg, Wg)
    out = []
    for a in range(-1, Hg // w + 2):
        for b in range(-1, Wg // w + 2):
            r0, c0 = max(a * w - shift, 0), max(b * w - shift, 0)
            r1, c1 = max(min((a + 1) * w - shift, Hg), 0), max(min((b + 1) * w - shift, Wg), 0)
            idx = grid[r0:r1, c0:c1].ravel()
            if idx.size:
                out.append(idx)
    return out


def mask2d_failures(lib=None):
    failed = []
    Hg, Wg = 5, 6
    N = Hg * Wg
    q, k, v = qkv(1, 2, N, 4, 30)
    o0, l0 = oracle.attention(q, k, v, scale=0.8, lib=lib)
    # no-op sizes
    for m in [("neighborhood", Wg, max(Hg, Wg)), ("window", Wg, N, 0)]:
        o, l = oracle.attention(q, k, v, scale=0.8, mask2d=m, lib=lib)
        if not (np.abs(o - o0).max() < 1e-12 and np.abs(l - l0).max() < 1e-12):
            failed.append(f"noop {m[0]}")
    # alone: O = V, LSE = own score
    own = 0.8 * np.einsum("bhnd,bhnd->bhn", q, k)
    for m in [("neighborhood", Wg, 1), ("window", Wg, 1, 0)]:
        o, l = oracle.attention(q, k, v, scale=0.8, mask2d=m, lib=lib)
        if not (np.abs(o - v).max() < 1e-12 and np.abs(l - own).max() < 1e-12):
            failed.append(f"alone {m[0]}")
    # windows == plain attention per gathered window
    for w, shift in [(2, 0), (3, 0), (2, 1), (4, 2)]:
        o, l = oracle.attention(q, k, v, scale=0.8, mask2d=("window", Wg, w, shift), lib=lib)
        for idx in gather_windows(Hg, Wg, w, shift):
            og, lg = oracle.attention(q[:, :, idx], k[:, :, idx], v[:, :, idx], scale=0.8)
            if not (np.abs(o[:, :, idx] - og).max() < 1e-12 and np.abs(l[:, :, idx] - lg).max() < 1e-12):
                failed.append(f"window w={w} shift={shift}")
                break
    # neighbourhood == plain attention of each query over its grid slice
    grid = np.arange(N).reshape(Hg, Wg)
    for R in [2, 3]:
        o, l = oracle.attention(q, k, v, scale=0.8, mask2d=("neighborhood", Wg, R), lib=lib)
        bad = False
        for i in range(N):
            r, c = divmod(i, Wg)
            idx = grid[max(r - R + 1, 0):r + R, max(c - R + 1, 0):c + R].ravel()
            og, lg = oracle.attention(q[:, :, i:i + 1], k[:, :, idx], v[:, :, idx], scale=0.8)
            if not (np.abs(o[:, :, i:i + 1] - og).max() < 1e-12 and np.abs(l[:, :, i:i + 1] - lg).max() < 1e-12):
                bad = True
        if bad:
            failed.append(f"neighborhood R={R}")
    return failed


def test_mask2d_pins():
    assert mask2d_failures() == []


def test_mask2d_with_causal_and_padding_is_the_intersection():
    """Masks combine by intersection: the 2-D mask under causal and key lengths
    equals the 2-D mask written as an additive -inf mask with causal and lengths."""
    Hg, Wg = 4, 5
    N = Hg * Wg
    q, k, v = qkv(2, 2, N, 4, 40)
    for m in [("neighborhood", Wg, 2), ("window", Wg, 2, 1)]:
        o, l = oracle.attention(q, k, v, is_causal=True, key_lens=[N, 13], mask2d=m)
        allowed = np.zeros((N, N), dtype=bool)
        for idx in (gather_windows(Hg, Wg, 2, 1) if m[0] == "window" else []):
            allowed[np.ix_(idx, idx)] = True
        if m[0] == "neighborhood":
            grid = np.arange(N).reshape(Hg, Wg)
            for i in range(N):
                r, c = divmod(i, Wg)
                allowed[i, grid[max(r - 1, 0):r + 2, max(c - 1, 0):c + 2].ravel()] = True
        add = np.where(allowed, 0.0, -np.inf)[None, None]
        o2, l2 = oracle.attention(q, k, v, is_causal=True, key_lens=[N, 13], mask=add)
        np.testing.assert_allclose(o, o2, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(l), np.isneginf(l2))
        fin = np.isfinite(l2)
        np.testing.assert_allclose(l[fin], l2[fin], atol=1e-12)


VARIANT_MUTANTS = {
    "cap_before_scale": ("s[j] = a->scale * dot;\n        if (a->softcap > 0.0) s[j] = a->softcap * tanh(s[j] / a->softcap);",
                         "s[j] = dot;\n        if (a->softcap > 0.0) s[j] = a->softcap * tanh(s[j] / a->softcap);\n        s[j] *= a->scale;"),
    "cap_inside_out": ("s[j] = a->softcap * tanh(s[j] / a->softcap);", "s[j] = tanh(s[j]);"),
    "mask_before_cap": ("if (a->softcap > 0.0) s[j] = a->softcap * tanh(s[j] / a->softcap);\n        if (mrow) s[j] += mrow[j];",
                        "if (mrow) s[j] += mrow[j];\n        if (a->softcap > 0.0) s[j] = a->softcap * tanh(s[j] / a->softcap);"),
    "radius_inclusive": ("return dr < a->m2_size && dc < a->m2_size;", "return dr <= a->m2_size && dc <= a->m2_size;"),
    "window_rows_only": ("return (ri + sh) / w == (rj + sh) / w && (ci + sh) / w == (cj + sh) / w;",
                         "return (ri + sh) / w == (rj + sh) / w;"),
    "shift_one_side": ("return (ri + sh) / w == (rj + sh) / w && (ci + sh) / w == (cj + sh) / w;",
                       "return (ri + sh) / w == rj / w && (ci + sh) / w == cj / w;"),
    "key_column_typo": ("const int ri = i / W, ci = i % W, rj = j / W, cj = j % W;",
                        "const int ri = i / W, ci = i % W, rj = j / W, cj = j / W;"),
}


@pytest.mark.parametrize("name", sorted(VARIANT_MUTANTS))
def test_variant_pins_catch_planted_mistake(name, tmp_path):
    before, after = VARIANT_MUTANTS[name]
    src = oracle.source_text()
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    lib = oracle.compile_variant(src.replace(before, after), str(tmp_path / f"mut_{name}.so"))
    assert softcap_failures(lib) + mask2d_failures(lib), f"planted mistake '{name}' passed every pin"
