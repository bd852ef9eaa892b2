"""GPU parity of attn_fwd_mod (soft-capped scores, 2-D neighbourhood and window
masks) against the fp64 oracle, with the tolerances of the plain path:
|O - O_ref| <= 1e-2 beyond the bf16 half-ulp, |LSE - LSE_ref| <= 1e-3, masked
keys and rows without keys exact."""
import math

import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from workloads import make_qkv

from test_parity_gpu import run_gpu
from tolerances import assert_close, reference

pytestmark = pytest.mark.gpu


def check(B, Hq, Hkv, Nq, Nk, d, seed, softcap=0.0, mask2d=None, causal=False, key_lens=None):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    kw = dict(is_causal=causal, softcap=softcap, mask2d=mask2d)
    if key_lens is not None:
        kw["key_lens"] = torch.tensor(key_lens, dtype=torch.int32)
    out, lse = run_gpu(q, k, v, **kw)
    ro, rl, ra = reference(q, k, v, is_causal=causal, softcap=softcap, mask2d=mask2d, key_lens=key_lens)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("cap", [30.0, 5.0, 1.0])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap(cap, d, causal):
    check(2, 4, 2, 300, 300, d, seed=int(cap) + d + causal, softcap=cap, causal=causal)


@pytest.mark.parametrize("d", [64, 128])
def test_softcap_ragged_and_padded(d):
    check(3, 2, 2, 200, 260, d, seed=5 + d, softcap=30.0, key_lens=[260, 0, 131])


@pytest.mark.parametrize("R", [1, 3, 5])
@pytest.mark.parametrize("d", [64, 128])
def test_neighborhood_ragged_grid(R, d):
    # 20 tokens per row, 17 rows: 340 tokens, the last key block ragged
    check(2, 2, 2, 340, 340, d, seed=R + d, mask2d=("neighborhood", 20, R))


def test_neighborhood_56x56_radius5():
    """The mask_mod example's grid (224 / 4 = 56 patches per row, N = 3136)."""
    check(1, 2, 2, 3136, 3136, 64, seed=77, mask2d=("neighborhood", 56, 5))


@pytest.mark.parametrize("w,shift", [(4, 0), (8, 0), (8, 4), (5, 2)])
@pytest.mark.parametrize("d", [64, 128])
def test_windows(w, shift, d):
    check(2, 2, 1, 16 * 12, 16 * 12, d, seed=w * 10 + shift + d, mask2d=("window", 16, w, shift))


def test_windows_56_grid_shifted():
    check(1, 2, 2, 3136, 3136, 64, seed=78, mask2d=("window", 56, 7, 3))


def test_one_token_per_row_is_a_sliding_window():
    """grid_w = 1 turns the neighbourhood into the band |i - j| < R."""
    check(1, 2, 2, 1000, 1000, 128, seed=79, mask2d=("neighborhood", 1, 100))


@pytest.mark.parametrize("d", [64, 128])
def test_softcap_with_mask2d_causal_and_padding(d):
    check(3, 2, 2, 340, 340, d, seed=80 + d, softcap=20.0, mask2d=("neighborhood", 20, 3), causal=True,
          key_lens=[340, 100, 0])


def test_mod_without_variants_equals_attn_fwd():
    q, k, v = make_qkv(2, 4, 2, 257, 300, 128, seed=81)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, l1 = ea.attention(qd, kd, vd, is_causal=True)
    o2 = torch.empty_like(qd)
    l2 = torch.empty_like(l1)
    st = ea.attn_fwd_mod(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o2.data_ptr(), l2.data_ptr(),
                         2, 4, 2, 257, 300, 128, 0.0, True, mod=ea.score_mod(), stream=ea._stream_handle(None))
    assert st == ea.ATTN_OK
    ea.check_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_masked_keys_bit_exact_under_mask2d():
    """Keys outside every query's grid rectangle can hold anything finite."""
    W, R, N, d = 20, 2, 340, 64
    q, k, v = make_qkv(1, 2, 2, N, N, d, seed=82)
    o1, l1 = run_gpu(q, k, v, mask2d=("neighborhood", W, R))
    # rows 0..2 of the grid see key rows 0..3 at most: scramble keys from row 8 on for queries of rows 0..2
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 8 * W:] = 50 * torch.randn(1, 2, N - 8 * W, d).to(torch.bfloat16)
    v2[:, :, 8 * W:] = 50 * torch.randn(1, 2, N - 8 * W, d).to(torch.bfloat16)
    o2, l2 = run_gpu(q, k2, v2, mask2d=("neighborhood", W, R))
    rows = slice(0, 3 * W)
    assert torch.equal(o1[:, :, rows], o2[:, :, rows]) and torch.equal(l1[:, :, rows], l2[:, :, rows])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap_polynomial_and_special_function_blocks(d, causal):
    """Query rows scaled from 0.3 to 30 under cap 30: the warps of the first rows
    keep every raw score of their key blocks within the polynomial's range
    (|scale * s / cap| <= 0.75) and take the FMA-pipe tanh, the last ones do not
    and take 1 - 2 / (1 + e^(2u)); both in one call, against the oracle."""
    B, H, N, cap = 1, 2, 700, 30.0
    q, k, v = make_qkv(B, H, H, N, N, d, seed=90 + d + causal)
    ramp = torch.logspace(math.log10(0.3), math.log10(30.0), N).view(1, 1, N, 1)
    q = (q.float() * ramp).to(torch.bfloat16)
    # the premise, per warp of 32 rows: the largest |scale * s / cap| over its keys
    u = (q.double() @ k.double().transpose(-1, -2)).abs() / math.sqrt(d) / cap
    if causal:
        u = u * torch.ones(N, N, dtype=torch.bool).tril()
    per_warp = torch.stack([u[..., r:r + 32, :].amax(dim=(-1, -2)) for r in range(0, N, 32)], dim=-1)
    assert (per_warp <= 0.7).any() and (per_warp > 0.8).any()
    out, lse = run_gpu(q, k, v, is_causal=causal, softcap=cap)
    ro, rl, ra = reference(q, k, v, is_causal=causal, softcap=cap)
    assert_close(out, lse, ro, rl, rabs=ra)
