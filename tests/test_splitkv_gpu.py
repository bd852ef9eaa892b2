"""GPU parity of the split-KV entry point (keys cut into ranges, partial results
merged by their log-sum-exp) against the fp64 oracle, which computes the
unsplit attention: the merge is exact, so the same tolerances apply as for
attn_fwd (tests/tolerances.py; masked structure exact)."""
import math

import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from workloads import make_qkv

from tolerances import O_TOL, assert_close, bf16_half_ulp, o_bound, reference

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def run_split(q, k, v, n_splits, **kw):
    args = {n: (t.to(DEV) if torch.is_tensor(t) else t) for n, t in kw.items()}
    out, lse = ea.attention(q.to(DEV), k.to(DEV), v.to(DEV), split_kv=n_splits, **args)
    ea.check_device_status()
    return out, lse


@pytest.mark.parametrize("Nq,Nk,n_splits", [
    (1, 4096, 0), (1, 4096, 4), (1, 5000, 7), (3, 1000, 3), (1, 129, 2), (16, 2048, 16),
    (300, 1500, 5), (1, 100, 4), (257, 640, 0), (2, 128 * 37, 0),
])
@pytest.mark.parametrize("d", [64, 128])
def test_splitkv_shapes(Nq, Nk, n_splits, d):
    B, Hq, Hkv = 2, 8, 2
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=Nq * 3 + Nk + d + n_splits)
    out, lse = run_split(q, k, v, n_splits)
    ro, rl, ra = reference(q, k, v)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("d", [64, 128])
def test_splitkv_causal(d):
    """Top-left causal mask with key ranges: early rows have no key in later ranges."""
    B, H, N = 1, 4, 1000
    q, k, v = make_qkv(B, H, H, N, N, d, seed=71 + d)
    out, lse = run_split(q, k, v, 4, is_causal=True)
    ro, rl, ra = reference(q, k, v, is_causal=True)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("d", [64, 128])
def test_splitkv_key_lens(d):
    """Ragged key lengths: whole ranges past a sample's length, and a sample with none."""
    B, Hq, Hkv, Nq, Nk = 5, 4, 4, 2, 3000
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=81 + d)
    lens = torch.tensor([3000, 0, 1, 1025, 2999], dtype=torch.int32)
    out, lse = run_split(q, k, v, 6, key_lens=lens)
    ro, rl, ra = reference(q, k, v, key_lens=lens.tolist())
    assert_close(out, lse, ro, rl, rabs=ra)


def test_splitkv_additive_mask():
    B, H, Nq, Nk, d = 2, 2, 5, 1300, 128
    q, k, v = make_qkv(B, H, H, Nq, Nk, d, seed=91)
    g = torch.Generator().manual_seed(9)
    mask = torch.randn(B, H, Nq, Nk, generator=g) * 2.0
    mask[0, 0, 1, :] = -math.inf           # a row with no key
    mask[1, 1, :, 300:] = -math.inf        # every range but the first empty for this head
    out, lse = run_split(q, k, v, 5, attn_mask=mask)
    ro, rl, ra = reference(q, k, v, mask=mask.double().numpy())
    assert_close(out, lse, ro, rl, rabs=ra)


def test_splitkv_matches_unsplit_call_and_is_deterministic():
    B, Hq, Hkv, Nq, Nk, d = 4, 16, 4, 1, 8192, 128
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=97)
    a_out, a_lse = run_split(q, k, v, 8)
    b_out, b_lse = run_split(q, k, v, 8)
    assert torch.equal(a_out, b_out) and torch.equal(a_lse, b_lse)
    u_out, u_lse = ea.attention(q.to(DEV), k.to(DEV), v.to(DEV))
    ea.check_device_status()
    assert (a_out.float() - u_out.float()).abs().max().item() <= 2e-2
    assert (a_lse - u_lse).abs().max().item() <= 2e-3


def test_splitkv_no_lse_and_short_workspace():
    B, H, Nq, Nk, d = 1, 2, 1, 2048, 64
    q, k, v = make_qkv(B, H, H, Nq, Nk, d, seed=99)
    out, lse = run_split(q, k, v, 4, return_lse=False)
    assert lse is None
    ro, _, ra = reference(q, k, v)
    assert (abs(out.double().cpu().numpy() - ro) - o_bound(ro, ra)).max() <= 0
    st, n, nbytes = ea.attn_splitkv_plan(B, H, Nq, Nk, d, 4, 0)
    assert st == ea.ATTN_OK and n == 4 and nbytes > 0
    small = torch.empty(nbytes - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        ea.attention(q.to(DEV), k.to(DEV), v.to(DEV), split_kv=4, workspace=small)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.empty_like(qd)
    st = ea.attn_fwd_splitkv(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), None,
                             B, H, H, Nq, Nk, d, 0.0, 0, n_splits=4, workspace=small.data_ptr(),
                             workspace_bytes=small.numel(), stream=ea._stream_handle(None))
    assert st == ea.ATTN_ERR_INVALID_ARG
