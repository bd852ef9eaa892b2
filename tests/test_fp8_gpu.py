"""GPU parity of attn_fwd_fp8 against the fp64 oracle on the dequantized FP8
inputs ("FlashAttention technical analysis", jsqmd.com/news/722897, sections
4.2 and 6.3: FP8 operands, block scales, higher-precision softmax).

Tolerance, derived from the arithmetic.  The scores are exact products of
E4M3 values summed in fp32, and the row sums use the fp32 exponentials, so the
one coarse rounding is that of the probabilities to E4M3 before the second
product.  The kernel stores P' = 2^6 * 2^(s - m) * sv_j / sv_max, m within 2^2
of the row max and sv_j the key block's V scale: a relative error of at most
2^-4 (3 mantissa bits, round to nearest) for normal values, at most 2^-10
absolute (2^-16 of the row max in P units, times sv_max / sv_j) below 2^-6.
Hence, per element,

    |O - O_ref| <= 2^-4 * sum_j P_ij |V_jc|  +  2^-8 |O_ref|  +  1e-2

where sum_j P_ij |V_jc| is the oracle's output with |V| (the codes with the
sign bit cleared), 2^-8 |O_ref| is the bf16 output rounding, and 1e-2 (the
bf16 path's tolerance) covers the subnormal and fp32 terms.  Because the
first term is loose for long rows, a second check bounds the root-mean-square
error by twice its expectation for independent roundings (variance at most
2^-8 / 3 * sum_j P_ij^2 V_jc^2), plus the output rounding.  LSE: the bf16
path's 1e-3 (it uses no rounded probability).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from workloads import make_fp8_inputs, quantize_e4m3_blocks

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3


def run_fp8(q8, k8, v8, qs, ks, vs, **kw):
    dev = torch.device("cuda:0")
    args = {n: (x.to(dev) if torch.is_tensor(x) else x) for n, x in kw.items()}
    out, lse = ea.attention_fp8(q8.to(dev), k8.to(dev), v8.to(dev), qs.to(dev), ks.to(dev), vs.to(dev), **args)
    ea.check_device_status()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def check(q8, k8, v8, qs, ks, vs, *, is_causal=False, key_lens=None, rms=True):
    kl = None if key_lens is None else torch.tensor(key_lens, dtype=torch.int32)
    o, lse = run_fp8(q8, k8, v8, qs, ks, vs, is_causal=is_causal, key_lens=kl)
    kw = dict(is_causal=is_causal, key_lens=key_lens)
    ro, rl = oracle.attention_fp8(q8, k8, v8, qs, ks, vs, **kw)
    r_abs, _ = oracle.attention_fp8(q8, k8, v8 & 0x7F, qs, ks, vs, **kw)
    assert np.isfinite(o).all()
    bound = 2.0 ** -4 * r_abs + 2.0 ** -8 * np.abs(ro) + 1e-2
    excess = np.abs(o - ro) - bound
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 0, f"|dO| over bound by {excess.max()} at {worst}: O={o[worst]} O_ref={ro[worst]}"
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(rl))
    fin = np.isfinite(rl)
    if fin.any():
        assert np.abs(lse[fin] - rl[fin]).max() <= LSE_TOL
    assert (o[np.isneginf(rl)] == 0).all()
    if rms:
        qd, kd, vd = (oracle.dequantize_blocks(c, s) for c, s in ((q8, qs), (k8, ks), (v8, vs)))
        p = oracle.probabilities(qd, kd, **kw)
        group = q8.shape[1] // k8.shape[1]
        expect = rms_expected(p, np.repeat(vd, group, axis=1), np.repeat(np.asarray(vs, np.float64), group, axis=1),
                              ro)
        got = math.sqrt(((o - ro) ** 2).mean())
        assert got <= 2.0 * expect + 1e-6, f"rms error {got} vs expected {expect}"
        print(f"fp8 rms error {got:.3e}, expected scale {expect:.3e}, max excess {excess.max():.3e}")
    return o, ro


def rms_expected(p, vr, vs, ro):
    """Expected root-mean-square error of O for independent roundings: each
    probability rounded to E4M3 (relative error uniform within 2^-4 for normal
    values; for subnormal ones an absolute step of 2^-16 (sv_max / sv_j) / l_i,
    with 1 / l_i <= max_j P_ij), plus the bf16 output rounding (2^-9 |O|).
    p: oracle probabilities [B, H, rows, Nk]; vr: dequantized V per query head
    [B, H, Nk, d]; vs: V block scales per query head [B, H, ceil(Nk / 128)]."""
    nk = p.shape[-1]
    ratio = np.repeat(vs.max(axis=-1, keepdims=True) / vs, 128, axis=-1)[..., :nk]
    a = np.maximum(2.0 ** -4 * p, 2.0 ** -16 * ratio[:, :, None, :] * p.max(axis=-1, keepdims=True))
    var = np.einsum("bhij,bhjc->bhic", a * a, vr * vr) / 3.0
    return math.sqrt(var.mean() + (2.0 ** -9) ** 2 * (ro * ro).mean())


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (127, 129), (128, 128), (300, 300), (77, 640), (513, 200)])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_vs_oracle(Nq, Nk, causal):
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(2, 4, 2, Nq, Nk, 128, seed=Nq * 3 + Nk * 5 + causal)
    check(q8, k8, v8, qs, ks, vs, is_causal=causal)


def test_long_keys_lazy_rescale():
    """32 key blocks per row: the running max, the stale-max correction and the
    V-scale fold accumulate over many blocks."""
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 2, 1, 256, 4096, 128, seed=11)
    check(q8, k8, v8, qs, ks, vs)


def gained_inputs(B, Hq, Hkv, Nq, Nk, seed):
    """N(0, 1) draws with every 128-row block multiplied by its own gain
    2^u, u uniform in [-3, 3], so that the block scales differ by up to 64x."""
    g = torch.Generator().manual_seed(seed)

    def draw(h, n):
        x = torch.randn((B, h, n, 128), generator=g)
        nb = (n + 127) // 128
        gain = torch.exp2(torch.rand((B, h, nb), generator=g) * 6 - 3)
        return x * gain.repeat_interleave(128, dim=-1)[..., :n, None]

    (q8, qs), (k8, ks), (v8, vs) = (quantize_e4m3_blocks(t) for t in (draw(Hq, Nq), draw(Hkv, Nk), draw(Hkv, Nk)))
    return q8, k8, v8, qs, ks, vs


@pytest.mark.parametrize("causal", [False, True])
def test_block_scales_that_differ(causal):
    q8, k8, v8, qs, ks, vs = gained_inputs(2, 4, 2, 384, 1000, seed=12 + causal)
    check(q8, k8, v8, qs, ks, vs, is_causal=causal)


def test_key_lengths_ragged_and_zero():
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(3, 2, 2, 200, 700, 128, seed=13)
    check(q8, k8, v8, qs, ks, vs, key_lens=[700, 0, 131])


def test_grouped_heads():
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 8, 1, 300, 512, 128, seed=14)
    check(q8, k8, v8, qs, ks, vs, is_causal=True)


def test_single_key_returns_its_value_row():
    """One key: P = 1 exactly (the block's V scale is the head's largest), so O
    is the dequantized V row up to the bf16 output rounding, and LSE is the
    scaled score."""
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 2, 2, 130, 1, 128, seed=15)
    o, lse = run_fp8(q8, k8, v8, qs, ks, vs)
    vd = oracle.dequantize_blocks(v8, vs)
    ref = np.broadcast_to(vd[:, :, :1, :], o.shape)
    # the kernel divides by an fp32 row sum within an ulp of 1: allow the bf16 rounding
    assert (np.abs(o - ref) <= 2.0 ** -8 * np.abs(ref) * (1 + 1e-5)).all()
    qd, kd = oracle.dequantize_blocks(q8, qs), oracle.dequantize_blocks(k8, ks)
    s = np.einsum("bhid,bhd->bhi", qd, kd[:, :, 0, :]) / math.sqrt(128)
    assert np.abs(lse - s).max() <= LSE_TOL


def test_float8_dtype_accepted_and_same_result():
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 2, 2, 130, 130, 128, seed=16)
    o1, l1 = run_fp8(q8, k8, v8, qs, ks, vs)
    f8 = torch.float8_e4m3fn
    o2, l2 = run_fp8(q8.view(f8), k8.view(f8), v8.view(f8), qs, ks, vs)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_full_size_sampled_rows():
    """B8 H32 N4096 d128 (the long-sequence workload) in FP8, inputs drawn on the
    device: sampled rows of three heads against the oracle, per element and in
    root-mean-square (a key block left out of P V moves O by about 1/sqrt(32)
    of its size, far above the RMS bound)."""
    B, H, N = 8, 32, 4096
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(B, H, H, N, N, 128, seed=17, device="cuda:0")
    o, lse = run_fp8(q8, k8, v8, qs, ks, vs)
    rng = np.random.default_rng(17)
    rows = np.unique(np.concatenate([rng.choice(N, 192, replace=False), [0, 1, 127, 128, 2047, 4094, 4095]]))
    for b, h in [(0, 0), (3, 17), (7, 31)]:
        cut = lambda t: t[b:b + 1, h:h + 1].cpu()  # noqa: E731
        qd = _deq_rows(cut(q8)[:, :, rows], cut(qs)[:, :, rows // 128])
        kd = oracle.dequantize_blocks(cut(k8), cut(ks))
        vd = oracle.dequantize_blocks(cut(v8), cut(vs))
        ro, rl = oracle.attention(qd, kd, vd)
        r_abs, _ = oracle.attention(qd, kd, oracle.dequantize_blocks(cut(v8) & 0x7F, cut(vs)))
        bound = 2.0 ** -4 * r_abs[0, 0] + 2.0 ** -8 * np.abs(ro[0, 0]) + 1e-2
        got = o[b, h][rows]
        assert (np.abs(got - ro[0, 0]) <= bound).all()
        assert np.abs(lse[b, h][rows] - rl[0, 0]).max() <= LSE_TOL
        expect = rms_expected(oracle.probabilities(qd, kd), vd, cut(vs).double().numpy(), ro)
        err = math.sqrt(((got - ro[0, 0]) ** 2).mean())
        print(f"PARITY long_fp8 (b={b}, h={h}, {len(rows)} rows): max|dO| {np.abs(got - ro[0, 0]).max():.3e}  "
              f"max|dLSE| {np.abs(lse[b, h][rows] - rl[0, 0]).max():.3e}  RMS(dO) {err:.3e} "
              f"(expected {expect:.3e}, RMS(O_ref) {math.sqrt((ro ** 2).mean()):.3e})")
        assert err <= 2.0 * expect + 1e-6, f"rms error {err} vs expected {expect}"


def _deq_rows(codes, scales):
    """Dequantize selected rows whose block scales are given one per row."""
    return oracle.e4m3_decode(codes.numpy()) * np.asarray(scales, dtype=np.float64)[..., None]


def test_deterministic():
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(2, 4, 2, 600, 900, 128, seed=18)
    o1, l1 = run_fp8(q8, k8, v8, qs, ks, vs, is_causal=True)
    o2, l2 = run_fp8(q8, k8, v8, qs, ks, vs, is_causal=True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_masked_keys_are_bit_exact():
    """Other codes at masked key positions (past each key length) change no
    output bit; the block scales are kept, so P's V-scale fold is unchanged."""
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(3, 2, 2, 300, 384, 128, seed=19)
    lens = [384, 200, 129]
    kl = torch.tensor(lens, dtype=torch.int32)
    o1, l1 = run_fp8(q8, k8, v8, qs, ks, vs, key_lens=kl)
    g = torch.Generator().manual_seed(20)
    k2, v2 = k8.clone(), v8.clone()
    for b, n in enumerate(lens):
        # random finite E4M3 codes (0x7F and 0xFF, the NaN codes, excluded)
        for t in (k2, v2):
            c = torch.randint(0, 0x7F, (2, 384 - n, 128), generator=g, dtype=torch.int64)
            sign = torch.randint(0, 2, c.shape, generator=g, dtype=torch.int64) << 7
            t[b, :, n:] = (c | sign).to(torch.uint8)
    o2, l2 = run_fp8(q8, k2, v2, qs, ks, vs, key_lens=kl)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
