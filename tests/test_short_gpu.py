"""GPU parity of the short-key path (d = 64, at most 256 keys: one tensor-memory
accumulator per score row, exact softmax without rescaling) against the fp64
oracle.  The cases cover what is particular to it: every key count class
(1, < 16, multiples of 16 and not, 256), runs of tiles that share one K/V head
across both K/V buffers and both tensor-memory slots, grouped heads, causal
rows with Nq above and below Nk, key lengths of 0 between non-empty batches
(empty tiles between runs), and rows past Nq inside the last tile."""
import numpy as np
import pytest
import torch

import exact_attention_157_b200 as ea
from tolerances import assert_close, reference
from workloads import make_qkv

from test_parity_gpu import run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Nk", [1, 7, 16, 33, 77, 128, 129, 196, 240, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_key_counts(Nk, causal):
    B, Hq, Hkv, Nq = 3, 4, 2, 300
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, 64, seed=Nk * 11 + causal)
    out, lse = run_gpu(q, k, v, is_causal=causal)
    ro, rl, ra = reference(q, k, v, is_causal=causal)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk", [
    (64, 16, 16, 196, 196),   # the ViT shape, fewer batches: several heads per CTA
    (2, 8, 8, 4096, 77),      # the cross-attention shape: 32 tiles per head, runs across CTAs
    (40, 8, 2, 130, 100),     # grouped heads: 4 query heads per K/V run, a 2-row last tile
    (300, 3, 1, 64, 256),     # one tile per head, more tiles than SMs, full 256 keys
])
def test_many_tiles_and_runs(B, Hq, Hkv, Nq, Nk):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, 64, seed=B + Hq + Nq + Nk)
    out, lse = run_gpu(q, k, v)
    ro, rl, ra = reference(q, k, v)
    assert_close(out, lse, ro, rl, rabs=ra, label=f"short B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk}")


@pytest.mark.parametrize("causal", [False, True])
def test_key_lens_with_empty_batches(causal):
    """Key lengths of 0 between non-empty batches: their tiles carry no run and
    write O = 0, LSE = -inf; the K/V buffers and slots of the others stay in step."""
    B, Hq, Hkv, Nq, Nk = 9, 4, 4, 260, 77
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, 64, seed=5 + causal)
    lens = torch.tensor([77, 0, 8, 0, 0, 40, 77, 1, 0], dtype=torch.int32)
    out, lse = run_gpu(q, k, v, is_causal=causal, key_lens=lens)
    ro, rl, ra = reference(q, k, v, is_causal=causal, key_lens=lens.tolist())
    assert_close(out, lse, ro, rl, rabs=ra)
    assert torch.all(out[1].cpu() == 0) and torch.all(torch.isneginf(lse[1].cpu()))


def test_masked_keys_are_bit_exact():
    B, H, Nq, Nk = 4, 3, 200, 150
    q, k, v = make_qkv(B, H, H, Nq, Nk, 64, seed=7)
    lens = torch.tensor([150, 77, 16, 1], dtype=torch.int32)
    out1, lse1 = run_gpu(q, k, v, key_lens=lens)
    k2, v2 = k.clone(), v.clone()
    for b, n in enumerate(lens.tolist()):
        k2[b, :, n:] = 1e4 * torch.randn(H, Nk - n, 64).to(torch.bfloat16)
        v2[b, :, n:] = -1e4
    out2, lse2 = run_gpu(q, k2, v2, key_lens=lens)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_deterministic_and_no_lse():
    q, k, v = make_qkv(16, 8, 8, 196, 196, 64, seed=9)
    a = run_gpu(q, k, v)
    b = run_gpu(q, k, v)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    dev = torch.device("cuda:0")
    out, lse = ea.attention(q.to(dev), k.to(dev), v.to(dev), return_lse=False)
    ea.check_device_status()
    assert lse is None and torch.equal(out, a[0])


def test_large_scores():
    """Scores of a few hundred: the exact maximum is taken before any exponential."""
    q, k, v = make_qkv(2, 2, 2, 256, 200, 64, seed=13)
    q = (q.float() * 25.0).to(torch.bfloat16)  # scores of std 25
    out, lse = run_gpu(q, k, v)
    ro, rl, ra = reference(q, k, v)
    assert_close(out, lse, ro, rl, rabs=ra)
    assert np.abs(rl).max() > 100


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("q_gain", [4.0, 10.0])
def test_later_keys_dominate(causal, q_gain):
    """Later 64-key steps exceed the first step's maximum by far more than the
    rescale threshold (2^8): the stored probabilities and the row sum are
    rescaled by powers of two, several times per row.  Rescales over the 960
    rows, counted on these inputs in fp64: gain 4, 2376 with 930 rows rescaling
    at least twice (causal 951, 296); gain 10, 2537 (causal 1058, 346)."""
    B, H, N = 2, 2, 240
    q, k, v = make_qkv(B, H, H, N, N, 64, seed=17 + causal)
    ramp = torch.linspace(0.05, 8.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float() * q_gain).to(torch.bfloat16)
    out, lse = run_gpu(q, k, v, is_causal=causal)
    ro, rl, ra = reference(q, k, v, is_causal=causal)
    assert_close(out, lse, ro, rl, rabs=ra)
