"""Pins of the oracle's FP8 input handling: the E4M3 decode against torch's
float8_e4m3fn conversion for all 256 codes and against values fixed by the
format; the per-block scales against a closed form; quantize -> dequantize of
the input generator within the format's rounding bound."""
import numpy as np
import pytest
import torch

import oracle
from workloads import make_fp8_inputs, quantize_e4m3_blocks


def test_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[fin], ref[fin])


def test_decode_values_fixed_by_the_format():
    table = {0x00: 0.0, 0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0x07: 7 * 2.0 ** -9,
             0xB8: -1.0, 0x40: 2.0, 0x3C: 1.5, 0xFE: -448.0}
    for code, val in table.items():
        assert oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0] == val, hex(code)
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_block_scales_apply_per_128_rows():
    codes = np.full((1, 1, 300, 2), 0x38, dtype=np.uint8)  # all 1.0
    scales = np.array([[[2.0, 3.0, 5.0]]])
    x = oracle.dequantize_blocks(codes, scales)
    assert (x[0, 0, :128] == 2.0).all() and (x[0, 0, 128:256] == 3.0).all() and (x[0, 0, 256:] == 5.0).all()


def test_generator_roundtrip_within_e4m3_rounding():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(2, 3, 260, 16, generator=g)
    codes, scales = quantize_e4m3_blocks(x)
    assert codes.dtype == torch.uint8 and scales.shape == (2, 3, 3)
    back = oracle.dequantize_blocks(codes.numpy(), scales.numpy())
    s = scales.numpy()[..., np.arange(260) // 128][..., None]
    # normal range: relative error <= 2^-4; subnormal range: absolute <= 2^-10 * scale
    err = np.abs(back - x.double().numpy())
    assert (err <= np.maximum(2.0 ** -4 * np.abs(x.double().numpy()), 2.0 ** -10 * s) + 1e-12).all()
    # every block uses the full range: its largest magnitude decodes to 448 * scale
    for blk in range(3):
        rows = slice(128 * blk, min(128 * (blk + 1), 260))
        assert np.allclose(np.abs(back[..., rows, :]).max(axis=(-1, -2)), 448.0 * scales.numpy()[..., blk])


def test_attention_fp8_is_the_definition_on_dequantized_inputs():
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 2, 1, 130, 140, 32, seed=5)
    o, lse = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), qs.numpy(), ks.numpy(), vs.numpy(),
                                  scale=0.2, is_causal=True)
    qd, kd, vd = (oracle.dequantize_blocks(c.numpy(), s.numpy()) for c, s in ((q8, qs), (k8, ks), (v8, vs)))
    o2, lse2 = oracle.attention_loops(qd, kd, vd, scale=0.2, is_causal=True)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, atol=1e-12)
