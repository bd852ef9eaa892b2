"""CPU-only checks of the C ABI: the library loads, exports every symbol that
include/attn.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

import exact_attention_157_b200 as ea

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from exact_attention_157_b200 import build
    build.build()


def test_header_declares_expected_entry_points():
    assert set(declared_functions()) == set(ea.EXPORTED)


@pytest.mark.parametrize("name", declared_functions())
def test_library_exports_symbol(name):
    lib = ctypes.CDLL(ea.LIB_PATH)
    assert hasattr(lib, name), name


def test_version_and_strings():
    assert ea.version() >= 100
    for st in range(7):
        assert isinstance(ea.status_string(st), str) and ea.status_string(st)
    assert ea.status_string(99) == "unknown status"


A = 4096  # a 16-byte-aligned fake address; never dereferenced (validation fails first)


@pytest.mark.parametrize("args,status", [
    (dict(q=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(out=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(B=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(Nq=-1), ea.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_INVALID_ARG),
    (dict(scale=-1.0), ea.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), ea.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), ea.ATTN_ERR_INVALID_ARG),
    (dict(key_lens=A, additive_mask=A), ea.ATTN_ERR_INVALID_ARG),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), ea.ATTN_ERR_UNSUPPORTED),
    (dict(q=A + 8), ea.ATTN_ERR_ALIGNMENT),
    (dict(v=A + 2), ea.ATTN_ERR_ALIGNMENT),
    (dict(lse=A + 2), ea.ATTN_ERR_ALIGNMENT),
    (dict(additive_mask=A, mask_strides=(-1, 0, 0)), ea.ATTN_ERR_INVALID_ARG),
])
def test_argument_validation_is_host_side(args, status):
    kw = dict(q=A, k=A, v=A, out=A, lse=None, B=1, Hq=2, Hkv=2, Nq=8, Nk=8, d=64,
              scale=0.0, is_causal=0, key_lens=None, additive_mask=None, mask_strides=None)
    kw.update(args)
    assert ea.attn_fwd(**kw) == status


def test_timeout_setting_accepts_values():
    assert ea.attn_set_wait_timeout_ns(123456789) == ea.ATTN_OK
    assert ea.attn_set_wait_timeout_ns(0) == ea.ATTN_OK  # restores the default


def test_torch_wrapper_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        ea.attention(q, q, q)


def test_package_does_not_import_oracle():
    src = open(os.path.join(ROOT, "exact_attention_157_b200", "__init__.py")).read()
    assert "oracle" not in src
    for f in os.listdir(os.path.join(ROOT, "exact_attention_157_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "exact_attention_157_b200", "csrc", f)).read()
