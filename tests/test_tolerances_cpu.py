"""The parity tolerances (tests/tolerances.py) on planted results, on the CPU.

A result that carries only the roundings the kernel is allowed (each
probability rounded to bf16 before P V, the output rounded to bf16) must pass;
results with a plausible kernel slip must fail, at the size of the long
workload (N = 4096 keys, 32 key blocks of 128), where one block is 1/32 of a
row: a key block left out of P V, a key block counted twice, and a block whose
contribution missed its rescale factor.  The planted slips act on the oracle's
own probability matrix, so only the checks are under test.
"""
import numpy as np
import pytest
import torch

import oracle
from tolerances import assert_close, reference
from workloads import make_qkv

NK = 4096
ROWS = list(range(0, 4096, 97)) + [127, 128, 4095]


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


@pytest.fixture(scope="module")
def head():
    """One (batch, head) of the long workload's shape: sampled query rows
    against all 4096 keys, with the oracle's O, LSE and probabilities."""
    q, k, v = make_qkv(1, 1, 1, NK, NK, 128, seed=2024)
    q = q[:, :, ROWS]
    ro, rl, ra = reference(q, k, v)
    p = oracle.probabilities(q, k)  # normalised rows, [1, 1, rows, NK]
    return ro, rl, ra, p, v.double().numpy()


def with_weights(p, v):
    """O = P V for a given (possibly altered) probability matrix, rounded to bf16."""
    return bf16(np.einsum("bhij,bhjc->bhic", p, v))


def rounded_like_the_kernel(p, v):
    """O with each weight exp(s - M) rounded to bf16 and divided by the unrounded
    row sum, then the output rounded to bf16."""
    pm = p / np.where(p.max(axis=-1, keepdims=True) > 0, p.max(axis=-1, keepdims=True), 1.0)
    l = pm.sum(axis=-1, keepdims=True)
    return with_weights(bf16(pm) / np.where(l > 0, l, 1.0), v)


def test_allowed_roundings_pass(head):
    ro, rl, ra, p, v = head
    stats = assert_close(rounded_like_the_kernel(p, v), rl, ro, rl, rabs=ra)
    assert stats["rms_ratio"] < 2.0 ** -8  # well inside the bound (2 * 2^-8)


def test_allowed_roundings_pass_on_short_causal_rows():
    """Rows with one to a few visible keys: there the probability rounding is not
    averaged away and may take |dO| past 1e-2 at |O| in [2, 4); the bound's
    2^-8 sum_j P_ij |V_jc| term admits it."""
    q, k, v = make_qkv(2, 4, 4, 200, 260, 64, seed=3)
    ro, rl, ra = reference(q, k, v, is_causal=True)
    p = oracle.probabilities(q, k, is_causal=True)
    o = rounded_like_the_kernel(p, v.double().numpy())
    assert_close(o, rl, ro, rl, rabs=ra)


@pytest.mark.parametrize("slip", ["block_dropped", "block_twice", "block_unscaled"])
def test_a_slip_in_one_key_block_fails(head, slip):
    ro, rl, ra, p, v = head
    j0, j1 = 17 * 128, 18 * 128  # one block in the middle of the ring
    pw = p.copy()
    if slip == "block_dropped":
        pw[..., j0:j1] = 0.0
    elif slip == "block_twice":
        pw[..., j0:j1] *= 2.0
    else:  # the block's terms kept a stale reference max: off by 2^-8 (tau = 8)
        pw[..., j0:j1] *= 2.0 ** -8
    with pytest.raises(AssertionError):
        assert_close(with_weights(pw, v), rl, ro, rl, rabs=ra)


def test_wrong_lse_fails(head):
    ro, rl, ra, p, v = head
    with pytest.raises(AssertionError):
        assert_close(bf16(ro), rl + 2e-3, ro, rl)


def test_half_ulp_allowance_only_above_four():
    """Without the probability term: |O| < 4 gets exactly the stated 1e-2; at
    4.0156 the nearest bf16 values are 0.0156 away, and the bound admits them."""
    from tolerances import o_bound
    b = o_bound(np.array([0.0, 1e-3, 2.0, 3.99, 4.0156, 64.3]))
    assert np.allclose(b[:4], 1e-2)
    assert b[4] >= 4.0156 - 4.0 and b[4] < 0.02
    assert b[5] < 0.3
