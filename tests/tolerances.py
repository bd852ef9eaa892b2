"""Tolerances of the forward-pass parity tests (bf16 inputs, fp32
accumulation, bf16 output) and the checks that apply them.  Host code only:
the GPU tests call these on kernel results, and the CPU tests pin their power
on planted errors.

  * per element, |O - O_ref| <= max(1e-2, half_ulp(O_ref)
    + 2^-8 sum_j P_ij |V_jc| + 2^-12 |O_ref|), where sum_j P_ij |V_jc| is the
    oracle's output with |V| (``reference``).  The stated 1e-2 holds wherever
    the two roundings of the bf16 path fit in it.  They do not always: the
    output is rounded to bf16 (half an ulp is 2^-7 = 0.0078 for |O| in [2, 4),
    2^-6 = 0.0156 from 4 up, so from |O| = 4 no bf16 value need lie within 1e-2
    of the exact result: 4.0156 is 0.0156 from both neighbours 4.0 and
    4.03125), and every probability is rounded to bf16 before the P V product
    (relative error at most 2^-8 per weight), which moves O by up to
    2^-8 sum_j P_ij |V_jc|.  On a row with few visible keys that is not
    averaged away: a causal row with two keys gave O = 2.34375 against
    O_ref = 2.35394 (|dO| = 0.0102), its pre-rounding value 0.0023 low from
    the rounded weight of one key, then rounded down on a grid of spacing 2^-6.
    2^-12 |O_ref| covers the fp32 arithmetic;
  * root-mean-square, RMS(O - O_ref) <= 2 * 2^-8 * RMS(O_ref) (RMS_C below);
  * max |LSE - LSE_ref| <= 1e-3 (LSE is fp32);
  * rows with no key: O = 0 exactly and LSE = -inf.
"""
import numpy as np

O_TOL = 1e-2
LSE_TOL = 1e-3


def bf16_half_ulp(x):
    """Half the spacing of the bf16 grid at |x| (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 8), 0.0)


# RMS bound.  Two roundings reach O, each of relative size at most 2^-8 and
# spread over its interval: the bf16 output rounding (RMS <= 2^-8 / sqrt(3) of
# |O|), and the rounding of every probability to bf16 before P V.  The latter
# moves O_i by sum_j p_ij d_ij v_j / l_i; with values v_j of zero mean,
# independent of the weights, its mean square is E[d^2] sum_j p_ij^2 v_j^2 /
# l_i^2, and E[O_i^2] = sum_j p_ij^2 E[v^2] / l_i^2, so again RMS <= 2^-8 /
# sqrt(3) of RMS(O).  Together sqrt(2/3) 2^-8 = 0.82 * 2^-8; the factor 2 keeps
# a margin of 2.4.  A key block skipped at N = 4096 (32 blocks) moves O by
# about RMS(O) / sqrt(32) = 0.18 RMS(O), 23 times the bound.
RMS_C = 2.0


def o_bound(ro, rabs=None):
    """Per-element bound on |O - O_ref| (module docstring); rabs = sum_j P_ij
    |V_jc| from ``reference`` (without it, only the output rounding and the fp32
    term are allowed beyond 1e-2)."""
    extra = 0.0 if rabs is None else 2.0 ** -8 * np.asarray(rabs)
    return np.maximum(O_TOL, bf16_half_ulp(ro) + extra + 2.0 ** -12 * np.abs(ro))


def reference(q, k, v, **kw):
    """The fp64 oracle's O and LSE, and its O with |V| (sum_j P_ij |V_jc|, the
    scale of the probability rounding's error) for the same inputs and options."""
    import oracle
    ro, rl = oracle.attention(q, k, v, **kw)
    va = v.abs() if hasattr(v, "abs") else np.abs(v)
    ra, _ = oracle.attention(q, k, va, **kw)
    return ro, rl, ra


def error_stats(o, lse, ro, rl):
    """Raw errors of a result against the oracle: max |dO|, max |dLSE| over
    rows with a key, and RMS(dO) / RMS(O_ref)."""
    fin = np.isfinite(rl)
    d_lse = float(np.abs(lse[fin] - rl[fin]).max()) if fin.any() else 0.0
    rms_ref = float(np.sqrt(np.mean(ro * ro)))
    rms_err = float(np.sqrt(np.mean((o - ro) ** 2)))
    return {"max_dO": float(np.abs(o - ro).max()), "max_dLSE": d_lse,
            "rms_ratio": rms_err / rms_ref if rms_ref > 0 else 0.0, "rms_err": rms_err, "rms_ref": rms_ref}


def rms_ok(stats):
    return stats["rms_err"] <= RMS_C * 2.0 ** -8 * stats["rms_ref"]


def assert_close(o, lse, ro, rl, rows=None, rms=True, label=None, rabs=None):
    """Checks a kernel result against the oracle with the tolerances of the
    module docstring; returns the raw error figures (error_stats) and prints
    them when a label is given."""
    o, lse = _host(o), _host(lse)
    if rows is not None:
        o, lse, ro, rl = o[..., rows, :], lse[..., rows], ro[..., rows, :], rl[..., rows]
        rabs = None if rabs is None else rabs[..., rows, :]
    assert np.isfinite(o).all(), "non-finite output"
    excess = np.abs(o - ro) - o_bound(ro, rabs)
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 0, (f"|dO| over the bound by {excess.max()} at {worst}: "
                               f"O={o[worst]} O_ref={ro[worst]}")
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(rl))
    stats = error_stats(o, lse, ro, rl)
    stats["over_1e-2"] = int((np.abs(o - ro) > O_TOL).sum())
    if label is not None:
        print(f"PARITY {label}: max|dO| {stats['max_dO']:.3e}  max|dLSE| {stats['max_dLSE']:.3e}  "
              f"RMS(dO)/RMS(O_ref) {stats['rms_ratio']:.3e}  elements |dO|>1e-2: {stats['over_1e-2']}")
    assert stats["max_dLSE"] <= LSE_TOL, f"max|dLSE| = {stats['max_dLSE']}"
    if rms:
        assert rms_ok(stats), f"RMS(dO)/RMS(O_ref) = {stats['rms_ratio']:.3e} > {RMS_C} * 2^-8"
    # rows with no key: exact zeros
    assert (o[np.isneginf(rl)] == 0).all()
    return stats




def _host(x):
    """fp64 numpy copy of a torch tensor (any device) or an array."""
    if hasattr(x, "detach"):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)
