"""GPU parity: the sm_100a kernels (through the C ABI) against the fp64 oracle
on the same seeded bf16 inputs.

Tolerances: tests/tolerances.py (max(1e-2, half an ulp of bf16 + 2^-12 |O|) per
element, an RMS bound, 1e-3 on LSE); mask structure bit-exact (a masked key
changes nothing, a row with no key gives O = 0 and LSE = -inf).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from tolerances import LSE_TOL, O_TOL, assert_close, bf16_half_ulp, o_bound, reference  # noqa: F401
from workloads import WORKLOADS, make_inputs, make_qkv

pytestmark = pytest.mark.gpu


def run_gpu(q, k, v, **kw):
    dev = torch.device("cuda:0")
    args = {}
    for name, val in kw.items():
        args[name] = val.to(dev) if torch.is_tensor(val) else val
    out, lse = ea.attention(q.to(dev), k.to(dev), v.to(dev), **args)
    ea.check_device_status()
    return out, lse


SHAPES = [(1, 1), (2, 2), (127, 127), (128, 128), (129, 129), (200, 260), (255, 300), (300, 255), (1, 513),
          (513, 1), (77, 640)]


@pytest.mark.parametrize("Nq,Nk", SHAPES)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_vs_oracle(Nq, Nk, d, causal):
    B, Hq, Hkv = 2, 4, 2
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=Nq * 7 + Nk * 13 + d + causal)
    out, lse = run_gpu(q, k, v, is_causal=causal)
    ro, rl, ra = reference(q, k, v, is_causal=causal)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("Nq,Nk", [(100, 300), (1, 256), (300, 200)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_many_units_per_cta_with_idle_tile(Nq, Nk, d, causal):
    """More work units than SMs, where the second 128-row tile of some or all
    units has no rows (Nq <= 128, or the last unit of each head at Nq = 300):
    the persistent CTAs run several such units back to back."""
    B, Hq, Hkv = 48, 8, 4
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=Nq + Nk + d + causal)
    out, lse = run_gpu(q, k, v, is_causal=causal)
    ro, rl, ra = reference(q, k, v, is_causal=causal)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("masked", [False, True])
def test_single_tile_last_round(d, masked):
    """154 two-tile units on 148 SMs: the last round's 6 units run as 12
    single-tile units (both halves of each; the second half of a head's last unit
    holds rows 2688..2799 of 2800), with key lengths, or with an additive mask
    broadcast over batch and heads; 400 keys keep the oracle quick."""
    B, H, N, Nk = 2, 7, 2800, 400
    q, k, v = make_qkv(B, H, H, N, Nk, d, seed=41 + d + masked)
    if masked:
        g = torch.Generator().manual_seed(43)
        mask = torch.randn(1, 1, N, Nk, generator=g)
        out, lse = run_gpu(q, k, v, attn_mask=mask)
        ro, rl, ra = reference(q, k, v, mask=mask.double().numpy())
    else:
        lens = torch.tensor([400, 150], dtype=torch.int32)
        out, lse = run_gpu(q, k, v, key_lens=lens)
        ro, rl, ra = reference(q, k, v, key_lens=lens.tolist())
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_key_lens_vs_oracle(d, causal):
    B, H, N = 5, 2, 300
    q, k, v = make_qkv(B, H, H, N, N, d, seed=31 + d)
    lens = torch.tensor([0, 1, 128, 129, 300], dtype=torch.int32)
    out, lse = run_gpu(q, k, v, is_causal=causal, key_lens=lens)
    ro, rl, ra = reference(q, k, v, is_causal=causal, key_lens=lens.tolist())
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("d", [64, 128])
def test_additive_mask_dense(d):
    B, H, Nq, Nk = 2, 2, 200, 260
    q, k, v = make_qkv(B, H, H, Nq, Nk, d, seed=41 + d)
    g = torch.Generator().manual_seed(5)
    mask = torch.randn(B, H, Nq, Nk, generator=g) * 3.0
    mask[0, 1, :, 100:] = -math.inf          # padding-like stripe
    mask[1, 0, 7, :] = -math.inf             # a row with no key
    out, lse = run_gpu(q, k, v, attn_mask=mask)
    ro, rl, ra = reference(q, k, v, mask=mask.double().numpy())
    assert_close(out, lse, ro, rl, rabs=ra)


def test_additive_mask_broadcast_and_causal():
    B, H, N, d = 2, 4, 257, 128
    q, k, v = make_qkv(B, H, H, N, N, d, seed=43)
    g = torch.Generator().manual_seed(6)
    mask = torch.randn(1, 1, N, N, generator=g)  # broadcast over batch and heads (stride 0)
    out, lse = run_gpu(q, k, v, attn_mask=mask, is_causal=True)
    ro, rl, ra = reference(q, k, v, mask=mask.double().numpy(), is_causal=True)
    assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_masked_keys_are_bit_exact(causal, d):
    """Finite garbage at masked key positions changes no output bit (d = 64 runs the
    decoupled form of the kernel, d = 128 the aliased one)."""
    B, H, N = 3, 2, 384
    q, k, v = make_qkv(B, H, H, N, N, d, seed=51)
    lens = torch.tensor([384, 200, 129], dtype=torch.int32)
    out1, lse1 = run_gpu(q, k, v, is_causal=causal, key_lens=lens)
    k2, v2 = k.clone(), v.clone()
    for b, n in enumerate(lens.tolist()):
        k2[b, :, n:] = 1e4 * torch.randn(H, N - n, d).to(torch.bfloat16)
        v2[b, :, n:] = -1e4
    out2, lse2 = run_gpu(q, k2, v2, is_causal=causal, key_lens=lens)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    if causal:
        k3, v3 = k.clone(), v.clone()
        k3[0, :, -1] = 3e3
        v3[0, :, -1] = 2e3
        out3, _ = run_gpu(q, k3, v3, is_causal=True, key_lens=lens)
        assert torch.equal(out3[0, :, :-1], out1[0, :, :-1])
        assert not torch.equal(out3[0, :, -1], out1[0, :, -1])


@pytest.mark.parametrize("d", [64, 128])
def test_deterministic(d):
    q, k, v = make_qkv(2, 4, 4, 1000, 1000, d, seed=61)
    a = run_gpu(q, k, v, is_causal=True)
    b = run_gpu(q, k, v, is_causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_large_scores_stay_exact():
    """Scores of a few hundred (large Q) exercise the lazy rescale: the running
    max grows by far more than the threshold between blocks."""
    B, H, N, d = 1, 2, 1024, 64
    q, k, v = make_qkv(B, H, H, N, N, d, seed=71)
    ramp = torch.linspace(0.1, 6.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.bfloat16)  # later keys dominate
    q = (q.float() * 4.0).to(torch.bfloat16)
    out, lse = run_gpu(q, k, v)
    ro, rl, ra = reference(q, k, v)
    assert_close(out, lse, ro, rl, rabs=ra)


def test_explicit_scale():
    q, k, v = make_qkv(1, 2, 2, 200, 200, 64, seed=81)
    out, lse = run_gpu(q, k, v, scale=0.05)
    ro, rl, ra = reference(q, k, v, scale=0.05)
    assert_close(out, lse, ro, rl, rabs=ra)


def test_no_lse_requested():
    q, k, v = make_qkv(1, 2, 2, 130, 130, 64, seed=91)
    dev = torch.device("cuda:0")
    out, lse = ea.attention(q.to(dev), k.to(dev), v.to(dev), return_lse=False)
    ea.check_device_status()
    assert lse is None
    ro, rl, ra = reference(q, k, v)
    assert (np.abs(out.double().cpu().numpy() - ro) - o_bound(ro, ra)).max() <= 0


# ---------------------------------------------------------- full workloads
def sample_rows(Nq, n_random, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(Nq, size=min(n_random, Nq), replace=False).tolist())
    for t in range(0, Nq, 128):
        rows.update({t, min(t + 127, Nq - 1)})
    rows.add(Nq - 1)
    return sorted(rows)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_vs_oracle(name):
    """Each workload at its full size, in the launch configuration the benchmark
    times; small ones are checked in full, large ones on sampled rows of the
    first and last (batch, head) (both K/V groups for grouped heads)."""
    w = WORKLOADS[name]
    dev = torch.device("cuda:0")
    q, k, v, kl = make_inputs(w, device=dev)
    out, lse = ea.attention(q, k, v, is_causal=w.is_causal, key_lens=kl, split_kv=0 if w.split_kv else None,
                            softcap=w.softcap, mask2d=w.mask2d)
    ea.check_device_status()
    full = w.B * w.Hq * w.Nq * w.Nk * w.d <= 2e10
    kl_list = None if kl is None else kl.cpu().tolist()
    var = dict(softcap=w.softcap, mask2d=w.mask2d)
    if full:
        ro, rl, ra = reference(q.cpu(), k.cpu(), v.cpu(), is_causal=w.is_causal, key_lens=kl_list, **var)
        assert_close(out.cpu(), lse.cpu(), ro, rl, rabs=ra, label=f"{name} (all rows)")
        return
    group = w.Hq // w.Hkv
    for (b, h) in [(0, 0), (w.B - 1, w.Hq - 1)]:
        hk = h // group
        rows = sample_rows(w.Nq, 512, seed=b * 1000 + h)
        ro, rl, ra = reference(q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, hk:hk + 1].cpu(),
                                  v[b:b + 1, hk:hk + 1].cpu(), is_causal=w.is_causal,
                                  key_lens=None if kl_list is None else [kl_list[b]], rows=rows, **var)
        assert_close(out[b:b + 1, h:h + 1].cpu(), lse[b:b + 1, h:h + 1].cpu(), ro, rl, rabs=ra, rows=rows,
                     label=f"{name} (b={b}, h={h}, {len(rows)} rows)")
    assert torch.isfinite(out).all()


# -------------------------------------------------------------- error paths
def test_bounded_wait_reports_timeout_and_context_survives():
    ea.attn_set_wait_timeout_ns(20_000_000)  # 20 ms
    try:
        assert ea.attn_selftest_timeout(ea._stream_handle(None)) == ea.ATTN_OK
        st, info = ea.attn_check_device_status(ea._stream_handle(None))
        assert st == ea.ATTN_ERR_TIMEOUT, (st, hex(info))
        assert (info >> 8) & 0xff == 9  # the self-test role
        # the error word was cleared and the context still works
        assert ea.attn_check_device_status(ea._stream_handle(None))[0] == ea.ATTN_OK
    finally:
        ea.attn_set_wait_timeout_ns(0)
    q, k, v = make_qkv(1, 2, 2, 128, 128, 64, seed=3)
    out, lse = run_gpu(q, k, v)
    ro, rl, ra = reference(q, k, v)
    assert_close(out, lse, ro, rl, rabs=ra)


def test_invalid_arguments_raise():
    dev = torch.device("cuda:0")
    q = torch.zeros(1, 3, 8, 64, dtype=torch.bfloat16, device=dev)
    kv = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(ea.AttnError) as e:
        ea.attention(q, kv, kv)
    assert e.value.status == ea.ATTN_ERR_INVALID_ARG
    q = torch.zeros(1, 2, 8, 96, dtype=torch.bfloat16, device=dev)
    with pytest.raises(ea.AttnError) as e:
        ea.attention(q, q, q)
    assert e.value.status == ea.ATTN_ERR_UNSUPPORTED
    q = torch.zeros(1, 2, 8, 64, dtype=torch.float16, device=dev)
    with pytest.raises(TypeError):
        ea.attention(q, q, q)


def test_out_of_range_key_lens_are_reported():
    q, k, v = make_qkv(2, 1, 1, 64, 64, 64, seed=4)
    dev = torch.device("cuda:0")
    lens = torch.tensor([64, 99], dtype=torch.int32, device=dev)
    out, _ = ea.attention(q.to(dev), k.to(dev), v.to(dev), key_lens=lens)
    st, info = ea.attn_check_device_status(ea._stream_handle(None))
    assert st == ea.ATTN_ERR_DEVICE, hex(info)
    assert torch.isfinite(out).all()  # clamped to Nk, memory-safe


# ------------------------------------------------------- short key sequences
@pytest.mark.parametrize("Nq,Nk", [(196, 196), (4096, 77), (17, 256), (300, 33), (1, 1)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_short_keys_vs_oracle(Nq, Nk, d, causal):
    """Short key sequences (the ViT and text cross-attention shapes), with key lengths."""
    B, Hq, Hkv = 2, 4, 2
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=Nq + 5 * Nk + d + causal)
    lens = torch.tensor([Nk, max(Nk // 3, 0)], dtype=torch.int32)
    out, lse = run_gpu(q, k, v, is_causal=causal, key_lens=lens)
    ro, rl, ra = reference(q, k, v, is_causal=causal, key_lens=lens.tolist())
    assert_close(out, lse, ro, rl, rabs=ra)


def test_short_keys_masked_keys_bit_exact():
    B, H, Nq, Nk, d = 3, 2, 200, 200, 64
    q, k, v = make_qkv(B, H, H, Nq, Nk, d, seed=61)
    lens = torch.tensor([200, 77, 0], dtype=torch.int32)
    out1, lse1 = run_gpu(q, k, v, key_lens=lens)
    k2, v2 = k.clone(), v.clone()
    for b, n in enumerate(lens.tolist()):
        k2[b, :, n:] = 1e4 * torch.randn(H, Nk - n, d).to(torch.bfloat16)
        v2[b, :, n:] = 1e4 * torch.randn(H, Nk - n, d).to(torch.bfloat16)
    out2, lse2 = run_gpu(q, k2, v2, key_lens=lens)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    assert torch.all(out1[2] == 0) and torch.all(torch.isneginf(lse1[2]))
