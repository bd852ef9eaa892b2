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


# ------------------------------------------------------------------ split-KV plan
def _ws_bytes(rows, d, s):
    r = lambda x: (x + 255) // 256 * 256
    return r(s * rows * d * 4) + r(s * rows * 4)


@pytest.mark.parametrize("B,Hq,Nq,Nk,d,req,used", [
    (8, 32, 1, 16384, 128, 1, 1),
    (8, 32, 1, 16384, 128, 4, 4),
    (2, 4, 7, 300, 64, 3, 3),     # 3 key blocks, 3 ranges of one block
    (2, 4, 7, 300, 64, 5, 3),     # capped at the number of key blocks
    (2, 4, 7, 512, 64, 3, 2),     # 4 blocks in ranges of ceil(4/3) = 2 blocks -> 2 ranges
    (1, 1, 1, 100, 128, 8, 1),    # a single key block never splits
])
def test_splitkv_plan_requested(B, Hq, Nq, Nk, d, req, used):
    """Tile-kernel plans (causal shapes never take the decode kernel)."""
    st, n, nbytes = ea.attn_splitkv_plan(B, Hq, Nq, Nk, d, req, 148, is_causal=True)
    assert st == ea.ATTN_OK
    assert n == used
    assert nbytes == (_ws_bytes(B * Hq * Nq, d, n) if n > 1 else 0)


@pytest.mark.parametrize("B,Hq,Nq,Nk", [(8, 32, 1, 16384), (1, 8, 4, 32768), (8, 32, 4096, 4096),
                                         (4, 8, 77, 2000), (1, 1, 1, 1 << 20)])
def test_splitkv_plan_auto_minimises_stated_cost(B, Hq, Nq, Nk):
    """The automatic range count is the first minimiser of
    ceil(units * s / SMs) * (key blocks per range + 2) over range counts s
    that the equal-length cut realises exactly (the header's model)."""
    sms = 148
    nb = -(-Nk // 128)
    units = B * Hq * (-(-Nq // 256))
    best, best_cost = 1, None
    for s in range(1, min(128, nb) + 1):
        per = -(-nb // s)
        if -(-nb // per) != s:
            continue
        cost = -(-(units * s) // sms) * (per + 2)
        if best_cost is None or cost < best_cost:
            best, best_cost = s, cost
    st, n, _ = ea.attn_splitkv_plan(B, Hq, Nq, Nk, 128, 0, sms, is_causal=True)
    assert st == ea.ATTN_OK and n == best


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,req,used", [
    (4, 16, 4, 1, 5000, 128, 6, 6),
    (1, 1, 1, 1, 100, 128, 8, 4),       # 4 chunks of 32 keys: at most 4 ranges
])
def test_splitkv_plan_decode_requested(B, Hq, Hkv, Nq, Nk, d, req, used):
    st, n, nbytes = ea.attn_splitkv_plan(B, Hq, Nq, Nk, d, req, 148, Hkv=Hkv)
    assert st == ea.ATTN_OK
    assert n == used
    assert nbytes == _ws_bytes(B * Hq * Nq, d, n)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d", [
    (8, 32, 8, 1, 16384, 128), (1, 32, 8, 1, 131072, 128), (2, 8, 2, 3, 3000, 64), (64, 16, 16, 1, 4096, 64),
    (3, 24, 3, 2, 77777, 128)])
def test_splitkv_plan_decode_auto_minimises_stated_cost(B, Hq, Hkv, Nq, Nk, d):
    """Decode-kernel plans: the first minimiser of
    ceil(B * Hkv * n / SMs) * (chunks per range + 15) over the counts the equal
    cut realises, at least 6 chunks per range (the header's model); always a
    workspace."""
    sms = 148
    chunks = -(-Nk // 32)
    most = max(chunks // 6, 1)
    best, best_cost = 1, None
    for t in range(1, min(most, 128) + 1):
        per = -(-chunks // t)
        if -(-chunks // per) != t:
            continue
        cost = -(-(B * Hkv * t) // sms) * (per + 15)
        if best_cost is None or cost < best_cost:
            best, best_cost = t, cost
    st, n, nbytes = ea.attn_splitkv_plan(B, Hq, Nq, Nk, d, 0, sms, Hkv=Hkv)
    assert st == ea.ATTN_OK and n == best
    assert nbytes == _ws_bytes(B * Hq * Nq, d, n)


def test_splitkv_plan_decode_rows_limit():
    """More than 16 query rows per K/V head, or causal, falls back to the tile plan."""
    tile = ea.attn_splitkv_plan(1, 32, 17, 4096, 128, 0, 148, Hkv=32, is_causal=True)
    assert ea.attn_splitkv_plan(1, 32, 17, 4096, 128, 0, 148, Hkv=32) == tile
    assert ea.attn_splitkv_plan(1, 32, 1, 4096, 128, 0, 148, Hkv=1) == \
        ea.attn_splitkv_plan(1, 32, 1, 4096, 128, 0, 148, Hkv=1, is_causal=True)


def test_splitkv_plan_rejects_bad_sizes():
    assert ea.attn_splitkv_plan(0, 1, 1, 1, 64, 0, 148)[0] == ea.ATTN_ERR_INVALID_ARG
    assert ea.attn_splitkv_plan(1, 1, 1, 1, 64, -1, 148)[0] == ea.ATTN_ERR_INVALID_ARG
    assert ea.attn_splitkv_plan(1, 1, 1, 1, 64, 0, -5)[0] == ea.ATTN_ERR_INVALID_ARG
    assert ea.attn_splitkv_plan(1, 1, 1, 1, 96, 0, 148)[0] == ea.ATTN_ERR_UNSUPPORTED
    assert ea.attn_splitkv_plan(1, 3, 1, 1, 64, 0, 148, Hkv=2)[0] == ea.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    (dict(n_splits=-1), ea.ATTN_ERR_INVALID_ARG),
    (dict(workspace=A + 16), ea.ATTN_ERR_ALIGNMENT),
    (dict(q=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
])
def test_splitkv_validation_is_host_side(args, status):
    kw = dict(q=A, k=A, v=A, out=A, lse=None, B=1, Hq=2, Hkv=2, Nq=1, Nk=4096, d=128,
              scale=0.0, is_causal=0, n_splits=4, workspace=A, workspace_bytes=1 << 20)
    kw.update(args)
    assert ea.attn_fwd_splitkv(**kw) == status


# ------------------------------------------------------------ score / mask variants
@pytest.mark.parametrize("mod,status", [
    (None, ea.ATTN_ERR_INVALID_ARG),
    (ea.score_mod(softcap=-1.0), ea.ATTN_ERR_INVALID_ARG),
    (ea.score_mod(softcap=float("inf")), ea.ATTN_ERR_INVALID_ARG),
    (ea.AttnScoreMod(0.0, 3, 8, 2, 0), ea.ATTN_ERR_INVALID_ARG),
    (ea.score_mod(mask2d=("neighborhood", 0, 2)), ea.ATTN_ERR_INVALID_ARG),
    (ea.score_mod(mask2d=("window", 8, 0)), ea.ATTN_ERR_INVALID_ARG),
    (ea.score_mod(mask2d=("window", 8, 4, -1)), ea.ATTN_ERR_INVALID_ARG),
])
def test_score_mod_validation_is_host_side(mod, status):
    assert ea.attn_fwd_mod(A, A, A, A, None, 1, 2, 2, 64, 64, 64, 0.0, 0, mod=mod) == status


def test_score_mod_struct_layout_matches_header():
    import re
    text = open(HEADER).read()
    body = re.search(r"typedef struct attn_score_mod_t \{(.*?)\} attn_score_mod_t;", text, re.S).group(1)
    names = re.findall(r"\b(?:float|int)\s+(\w+);", body)
    assert names == [f[0] for f in ea.AttnScoreMod._fields_]
    assert ctypes.sizeof(ea.AttnScoreMod) == 20


# ------------------------------------------------------------------- backward
def test_bwd_plan_bytes():
    st, nb = ea.attn_bwd_plan(2, 4, 300)
    assert st == ea.ATTN_OK
    rows = 2 * 4 * 384  # rows padded to a multiple of 128 per head
    assert nb == 2 * ((rows * 4 + 255) // 256 * 256)
    assert ea.attn_bwd_plan(0, 4, 300)[0] == ea.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    (dict(dq=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(workspace=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(workspace_bytes=16), ea.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_INVALID_ARG),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(dk=A + 8), ea.ATTN_ERR_ALIGNMENT),
    (dict(workspace=A + 16), ea.ATTN_ERR_ALIGNMENT),
    (dict(scale=-2.0), ea.ATTN_ERR_INVALID_ARG),
])
def test_bwd_validation_is_host_side(args, status):
    kw = dict(q=A, k=A, v=A, out=A, lse=A, dout=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=2, Nq=64, Nk=64, d=64,
              scale=0.0, is_causal=0, key_lens=None, workspace=A, workspace_bytes=1 << 20)
    kw.update(args)
    assert ea.attn_bwd(**kw) == status


# ------------------------------------------------------------------- FP8
@pytest.mark.parametrize("args,status", [
    (dict(q8=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(v_scale=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(out=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_INVALID_ARG),
    (dict(Nk=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), ea.ATTN_ERR_INVALID_ARG),
    (dict(d=64), ea.ATTN_ERR_UNSUPPORTED),
    (dict(k8=A + 8), ea.ATTN_ERR_ALIGNMENT),
    (dict(q_scale=A + 2), ea.ATTN_ERR_ALIGNMENT),
    (dict(lse=A + 1), ea.ATTN_ERR_ALIGNMENT),
])
def test_fp8_validation_is_host_side(args, status):
    kw = dict(q8=A, k8=A, v8=A, q_scale=A, k_scale=A, v_scale=A, out=A, lse=None, B=1, Hq=2, Hkv=2,
              Nq=64, Nk=64, d=128, scale=0.0, is_causal=0)
    kw.update(args)
    assert ea.attn_fwd_fp8(**kw) == status


@pytest.mark.parametrize("args,status", [
    (dict(q=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(Hkv=0), ea.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_INVALID_ARG),
    (dict(scale=-1.0), ea.ATTN_ERR_INVALID_ARG),
    (dict(n_splits=-1), ea.ATTN_ERR_INVALID_ARG),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(k=A + 4), ea.ATTN_ERR_ALIGNMENT),
])
def test_noalloc_argument_errors_come_before_device_setup(args, status):
    """attn_fwd_splitkv_noalloc checks every argument before its one-time
    device set-up: on this GPU-less host any CUDA call would fail with
    ATTN_ERR_CUDA or ATTN_ERR_UNSUPPORTED instead of the argument error."""
    kw = dict(q=A, k=A, v=A, out=A, lse=None, B=1, Hq=2, Hkv=2, Nq=8, Nk=8, d=64,
              scale=0.0, is_causal=0, key_lens=None, additive_mask=None, mask_strides=None, n_splits=0)
    kw.update(args)
    assert ea.attn_fwd_splitkv_noalloc(**kw) == status


def test_exp2_selftest_argument_errors():
    lib = ea.lib()
    assert lib.attn_selftest_exp2_poly(None, None, -1, None) == ea.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_exp2_poly(None, None, 4, None) == ea.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_exp2_poly(A + 2, A, 4, None) == ea.ATTN_ERR_ALIGNMENT
    assert lib.attn_selftest_exp2_poly(None, None, 0, None) == ea.ATTN_OK  # nothing to do
