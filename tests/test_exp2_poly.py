"""The FMA-pipe exp2 used for part of the softmax exponentials: its constants
in the kernel source match the fit, and a float32 emulation of the kernel's
exact sequence of operations stays within the fitted error bound.  CPU only."""
import os
import re
import runpy

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "exact_attention_157_b200", "csrc", "fwd_kernel_pp.cuh")
FIT = os.path.join(ROOT, "exact_attention_157_b200", "csrc", "fit_exp2_poly.py")


def kernel_constants():
    src = open(KERNEL).read()
    body = src[src.index("void exp2_poly_pair"):]
    vals = dict(re.findall(r"constexpr uint64_t (k\w+) = splat2\(0x([0-9A-Fa-f]{8})u\)", body))
    return {k: np.uint32(int(v, 16)).view(np.float32) for k, v in vals.items()}


def emulate(x, k):
    f32 = np.float32
    xx = np.maximum(x.astype(f32), f32(-120.0))
    t = (xx + k["kMagic"]).astype(f32)
    f = ((t + k["kNegMagic"]).astype(f32) * k["kNegOne"] + xx).astype(f32)
    p = (f * k["kC3"] + k["kC2"]).astype(f32)
    p = (p * f + k["kC1"]).astype(f32)
    p = (p * f + k["kC0"]).astype(f32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_constants_match_fit():
    k = kernel_constants()
    assert k["kMagic"] == np.float32(1.5 * 2 ** 23) and k["kNegMagic"] == -k["kMagic"] and k["kNegOne"] == -1
    fit = runpy.run_path(FIT)
    c, err = fit["remez_relative"]()
    assert err < 8e-5
    for i, name in enumerate(["kC0", "kC1", "kC2", "kC3"]):
        assert k[name] == np.float32(c[i]), (name, k[name], c[i])


def test_relative_error_bound():
    k = kernel_constants()
    x = np.linspace(-60.0, 9.0, 2_000_001, dtype=np.float32)
    e = emulate(x, k)
    rel = np.abs(e.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 7.6e-5
    # exact powers of two within the bound, and monotone non-decreasing
    assert np.all(np.diff(e.astype(np.float64)) >= -1e-12 * np.abs(e[1:]))


def test_clamp_gives_tiny_positive():
    k = kernel_constants()
    e = emulate(np.array([-121.0, -500.0, -1e30], dtype=np.float32), k)
    assert np.all(e > 0) and np.all(e < 1e-35)
