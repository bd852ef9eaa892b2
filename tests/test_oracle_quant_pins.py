"""Pins of the oracle's E4M3 encoder and block quantiser (CPU), and planted
mistakes in a copy of them that the pins must catch.

The encoder is pinned by the format itself (every finite code round-trips
through its value; a midpoint between neighbouring codes goes to the even
code), by a table of values fixed by the format, and, as a library special
case, by torch's float8_e4m3fn conversion.  The quantiser is pinned by what
its definition fixes: the block's largest magnitude maps to +-448, every value
comes back within half a grid step times the scale, a zero block has scale 1
and zero codes, and the block boundaries fall every 128 rows."""
import inspect

import numpy as np
import pytest
import torch

import oracle

FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def torch_e4m3(y):
    return torch.from_numpy(np.asarray(y, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_every_finite_code_round_trips():
    vals = oracle.e4m3_decode(FINITE).astype(np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals), FINITE)


def test_midpoints_go_to_the_even_code():
    pos = np.arange(0x00, 0x7E, dtype=np.uint8)  # neighbours c, c + 1 up to 448
    lo, hi = oracle.e4m3_decode(pos), oracle.e4m3_decode(pos + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # exact in fp32
    even = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint8)
    np.testing.assert_array_equal(oracle.e4m3_encode(mid), even)
    np.testing.assert_array_equal(oracle.e4m3_encode(-mid), even | 0x80)
    # just off the midpoint: the nearer neighbour
    up = np.nextafter(mid, np.float32(1e9))
    np.testing.assert_array_equal(oracle.e4m3_encode(up), pos + 1)


def test_table_of_values():
    table = [(0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -9, 0x01),
             (2.0 ** -6, 0x08), (1.125, 0x39), (240.0, 0x77), (0.75 * 2.0 ** -6, 0x06), (3.5 * 2.0 ** -9, 0x04)]
    for v, c in table:
        assert oracle.e4m3_encode(np.array([v], dtype=np.float32))[0] == c, (v, hex(c))


def test_agrees_with_torch_conversion():
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.uniform(-448, 448, 100000), rng.normal(0, 2.0 ** -7, 100000),
                        rng.normal(0, 1, 100000)]).astype(np.float32)
    y = np.clip(y, -448, 448)
    np.testing.assert_array_equal(oracle.e4m3_encode(y), torch_e4m3(y))


def test_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.e4m3_encode(np.array([449.0], dtype=np.float32))


def test_block_quantiser_properties():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 3, (2, 3, 300, 64)).astype(np.float32)
    x[1, 2, 128:256] = 0.0  # an all-zero block
    codes, scales = oracle.quantize_e4m3_blocks(x)
    assert codes.shape == x.shape and scales.shape == (2, 3, 3) and scales.dtype == np.float32
    for j in range(3):
        blk = x[..., 128 * j:128 * (j + 1), :]
        amax = np.abs(blk).max(axis=(-1, -2))
        expect = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), 1.0)
        np.testing.assert_array_equal(scales[..., j], expect)
    assert scales[1, 2, 1] == 1.0 and (codes[1, 2, 128:256] == 0).all()
    # the largest magnitude of each non-zero block is +-448 in codes
    for b in range(2):
        for h in range(3):
            for j in range(3):
                blk = x[b, h, 128 * j:128 * (j + 1)]
                if np.abs(blk).max() == 0:
                    continue
                i = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
                assert codes[b, h, 128 * j + i[0], i[1]] in (0x7E, 0xFE)
    # every value back within half a grid step of its binade, times the scale
    deq = oracle.dequantize_blocks(codes, scales)
    ys = x.astype(np.float64) / np.repeat(scales, 128, axis=-1)[..., :300, None]
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(ys), 2.0 ** -6))) - 3)
    err = np.abs(deq - x.astype(np.float64)) / np.repeat(scales, 128, axis=-1)[..., :300, None]
    assert (err <= step / 2 * (1 + 1e-6)).all()


SOURCE = inspect.getsource(oracle.e4m3_encode) + "\n" + inspect.getsource(oracle.quantize_e4m3_blocks)

MUTANTS = {
    "ties_away_from_zero": ("np.rint(a / np.exp2(e - 3.0))", "np.floor(a / np.exp2(e - 3.0) + 0.5)"),
    "exponent_bias_8": ("((e + 7) << 3)", "((e + 8) << 3)"),
    "no_carry_to_next_binade": ("carry = units == 16", "carry = units == 17"),
    "subnormal_grid": ("e = np.maximum(e, -6)", "e = np.maximum(e, -7)"),
    "scale_over_240": ("(amax / np.float32(448.0))", "(amax / np.float32(240.0))"),
    "sign_dropped": ("sign = np.signbit(y).astype(np.int64) << 7", "sign = np.signbit(y).astype(np.int64) << 8"),
    "block_of_127_rows": ("xb = x[..., j * block:(j + 1) * block, :]", "xb = x[..., j * block:(j + 1) * block - 1, :]"),
}


def build(src):
    ns = {"np": np}
    exec(src, ns)  # noqa: S102 - a copy of the oracle's own source, mutated in the test
    return ns["e4m3_encode"], ns["quantize_e4m3_blocks"]


def battery(encode, quantize) -> bool:
    """The pins above as one predicate (True when all hold)."""
    try:
        vals = oracle.e4m3_decode(FINITE).astype(np.float32)
        if not np.array_equal(encode(vals), FINITE):
            return False
        pos = np.arange(0x00, 0x7E, dtype=np.uint8)
        mid = ((oracle.e4m3_decode(pos) + oracle.e4m3_decode(pos + 1)) / 2).astype(np.float32)
        if not np.array_equal(encode(mid), np.where(pos % 2 == 0, pos, pos + 1)):
            return False
        rng = np.random.default_rng(7)
        y = np.clip(rng.normal(0, 20, 20000), -448, 448).astype(np.float32)
        if not np.array_equal(encode(y), torch_e4m3(y)):
            return False
        x = rng.normal(0, 3, (1, 2, 260, 16)).astype(np.float32)
        codes, scales = quantize(x)
        amax = np.abs(x[..., 128:256, :]).max(axis=(-1, -2))
        if not np.array_equal(scales[..., 1], (amax / np.float32(448.0)).astype(np.float32)):
            return False
        return bool(np.array_equal(codes, torch_e4m3(np.clip(x / np.repeat(scales, 128, axis=-1)[..., :260, None],
                                                             -448, 448))))
    except (IndexError, ValueError):
        return False


def test_unmutated_copy_passes_battery():
    assert battery(*build(SOURCE))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    assert SOURCE.count(old) == 1, f"mutation anchor of {name} not found in the oracle"
    assert not battery(*build(SOURCE.replace(old, new))), f"pins miss the mutant {name}"
