"""Plant a mistake in a copy of the oracle's FP8 input handling (on the CPU) and
check that the pins of test_oracle_fp8_pins catch it.  Each mutant is a
plausible slip in reading the E4M3 format or the block scales: the exponent
bias, the subnormal scale, the subnormal branch, the NaN codes, the sign bit,
the block size."""
import inspect

import numpy as np
import pytest
import torch

import oracle

SOURCE = inspect.getsource(oracle.e4m3_decode) + "\n" + inspect.getsource(oracle.dequantize_blocks)

MUTANTS = {
    "exponent_bias_8": ("np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)"),
    "subnormal_scale": ("(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7"),
    "subnormal_as_normal": ("np.where(e == 0,", "np.where(e < 0,"),
    "nan_only_positive": ("(c & 0x7F) == 0x7F", "c == 0x7F"),
    "sign_ignored": ("np.where(c & 0x80, -1.0, 1.0)", "np.where(c & 0x100, -1.0, 1.0)"),
    "block_of_127_rows": ("np.arange(n) // block", "np.arange(n) // (block - 1)"),
}


def build(src):
    ns = {"np": np}
    exec(src, ns)  # noqa: S102 - a copy of the oracle's own source, mutated in the test
    return ns["e4m3_decode"], ns["dequantize_blocks"]


def battery(decode, dequantize) -> bool:
    """The FP8 pins as one predicate: True when all of them hold."""
    try:
        codes = np.arange(256, dtype=np.uint8)
        ours = decode(codes)
        ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        if not np.array_equal(np.isnan(ours), np.isnan(ref)):
            return False
        fin = ~np.isnan(ref)
        if not np.array_equal(ours[fin], ref[fin]):
            return False
        table = {0x00: 0.0, 0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0xB8: -1.0}
        if any(decode(np.array([c], dtype=np.uint8))[0] != v for c, v in table.items()):
            return False
        x = dequantize(np.full((1, 1, 300, 2), 0x38, dtype=np.uint8), np.array([[[2.0, 3.0, 5.0]]]))
        return bool((x[0, 0, :128] == 2.0).all() and (x[0, 0, 128:256] == 3.0).all() and (x[0, 0, 256:] == 5.0).all())
    except (IndexError, ValueError):
        return False


def test_unmutated_copy_passes_battery():
    assert battery(*build(SOURCE))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    assert SOURCE.count(old) == 1, f"mutation anchor of {name} not found in the oracle"
    assert not battery(*build(SOURCE.replace(old, new))), f"pins miss the mutant {name}"
