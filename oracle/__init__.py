"""fp64 CPU oracle for the exact attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it.

Contents
--------
``attention``            the definition (three steps, two-pass softmax) in plain C,
                         fp64, threaded over rows (``attn_oracle.c``); optional
                         soft-capped scores and 2-D neighbourhood / window masks.
``attention_online``     a numpy fp64 re-statement of the tiled algorithm with a
                         running max ``m`` and running sum ``l`` rescaled per key
                         block, used only to cross-check ``attention``.
``probabilities``        the materialised probability matrix P (numpy fp64), for
                         the row-sum invariant.
``attention_loops``      pure-Python loops for tiny inputs (brute force).
``attention_bwd``        the gradients dQ, dK, dV of the definition for a given dO, in
                         plain C, fp64 (``attn_oracle_bwd.c``).
``e4m3_decode``,         FP8 inputs: the E4M3 code -> value map written from the format
``dequantize_blocks``,   (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals,
``attention_fp8``        no infinities, S.1111.111 = NaN) and per-128-row block scales;
                         the result is the definition on the dequantized values.
``e4m3_encode``,         the value -> code map (round to nearest even) and the block
``quantize_e4m3_blocks`` quantiser (scale = block amax / 448), in fp32 arithmetic.

Sources: "FlashAttention technical analysis" (jsqmd.com/news/722897) section 2.1
(the three steps), section 2.2 (tiling plus online softmax with running max and
sum), section 3.3 (only the O(N) statistics are kept) and section 6.2 (two-pass
safe softmax); "Flash Attention in a production Stable-Diffusion service"
(xxmr.cn/news/81028) section 2.3 (order: QK^T, scale, add mask, softmax, PV).

Readings where the pages are silent: see the header of ``attn_oracle.c``; the
numpy variants below follow the same readings.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_SRC_BWD = os.path.join(_HERE, "attn_oracle_bwd.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_LIB_BWD = os.path.join(_LIB_DIR, "liboracle_bwd.so")
_lock = threading.Lock()
_lib = None
_lib_bwd = None


def _gcc(src: str, out: str, force: bool):
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, src, "-lm", "-lpthread"])
        os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` and ``attn_oracle_bwd.c`` into ``_build/`` with gcc
    (no fast-math, no contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    _gcc(_SRC, _LIB, force)
    _gcc(_SRC_BWD, _LIB_BWD, force)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    lib.oracle_attention_fwd.restype = ctypes.c_int
    lib.oracle_attention_fwd.argtypes = [
        dp, dp, dp, dp, dp,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int,
        ip, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ip, ctypes.c_int, ctypes.c_int]
    lib.oracle_attention_fwd_mod.restype = ctypes.c_int
    lib.oracle_attention_fwd_mod.argtypes = [
        dp, dp, dp, dp, dp,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int,
        ip, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ip, ctypes.c_int, ctypes.c_int]
    lib.oracle_default_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def _bind_bwd(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    lib.oracle_attention_bwd.restype = ctypes.c_int
    lib.oracle_attention_bwd.argtypes = [
        dp, dp, dp, dp, dp, dp, dp,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int, ip, ip, ctypes.c_int, ctypes.c_int]
    lib.oracle_attention_bwd_mod.restype = ctypes.c_int
    lib.oracle_attention_bwd_mod.argtypes = [
        dp, dp, dp, dp, dp, dp, dp,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int, ip,
        dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ip, ctypes.c_int, ctypes.c_int]
    return lib


def _load_bwd():
    global _lib_bwd
    with _lock:
        if _lib_bwd is None:
            build()
            _lib_bwd = _bind_bwd(_LIB_BWD)
    return _lib_bwd


def source_text_bwd() -> str:
    with open(_SRC_BWD) as f:
        return f.read()


def compile_variant_bwd(src_text: str, out_path: str):
    """Compile a modified copy of the backward oracle (mutant tests only)."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-o", out_path, c_path, "-lm", "-lpthread"])
    return _bind_bwd(out_path)


def attention_bwd(q, k, v, dout, *, scale: float | None = None, is_causal: bool = False, key_lens=None,
                  units=None, n_threads: int = 0, lib=None, mask=None, softcap: float = 0.0, mask2d=None):
    """Gradients of the definition for the upstream gradient ``dout`` (fp64).

    q, dout: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; key_lens: [B] or None;
    units: optional list of b * Hkv + hkv pairs to compute (others are NaN).
    mask: additive mask broadcastable to [B, Hq, Nq, Nk]; softcap: cap of the
    soft-capped score (0: off); mask2d: None, ("neighborhood", W, R) or
    ("window", W, w[, shift]), as in ``attention``.
    Returns (dQ [B, Hq, Nq, d], dK [B, Hkv, Nk, d], dV [B, Hkv, Nk, d]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    kl = None if key_lens is None else np.ascontiguousarray(np.asarray(key_lens, dtype=np.int32))
    un = None if units is None else np.ascontiguousarray(np.asarray(units, dtype=np.int32))
    mk, sb, sh, sq = None, 0, 0, 0
    if mask is not None:
        mk, sb, sh, sq = _mask_view(mask, B, Hq, Nq, Nk)
    kind, W, size, shift = 0, 1, 1, 0
    if mask2d is not None:
        kind = {"neighborhood": 1, "window": 2}[mask2d[0]]
        W, size = int(mask2d[1]), int(mask2d[2])
        shift = int(mask2d[3]) if len(mask2d) > 3 else 0
    rc = (lib or _load_bwd()).oracle_attention_bwd_mod(
        _ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
        B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(is_causal)),
        _ptr(kl, ctypes.c_int32), _ptr(mk), sb, sh, sq, float(softcap or 0.0), kind, W, size, shift,
        _ptr(un, ctypes.c_int32), 0 if un is None else len(un), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_attention_bwd rejected its arguments (status {rc})")
    return dq, dk, dv


def compile_variant(src_text: str, out_path: str):
    """Compile a modified copy of the oracle source to ``out_path`` and return a
    loaded handle for ``attention(..., lib=handle)``.  Used only by the tests that
    plant a mistake in the oracle to show that the pins catch it."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-o", out_path, c_path, "-lm", "-lpthread"])
    return _bind(out_path)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _f64(x) -> np.ndarray:
    """Exact conversion of a CPU tensor / array to a contiguous fp64 numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype)) if a is not None else None


def _mask_view(mask, B, Hq, Nq, Nk):
    """Return (fp64 array, sb, sh, sq) for a mask broadcastable to [B, Hq, Nq, Nk]."""
    m = np.asarray(mask, dtype=np.float64)
    while m.ndim < 4:
        m = m[None]
    m = np.broadcast_to(m, (B, Hq, Nq, Nk))
    base = np.ascontiguousarray(m[:, :, :, :])  # materialise (tests only; sizes are small)
    return base, Hq * Nq * Nk, Nq * Nk, Nk


MASK2D_KINDS = {"neighborhood": 1, "window": 2}


def attention(q, k, v, *, scale: float | None = None, is_causal: bool = False,
              key_lens=None, mask=None, rows=None, n_threads: int = 0, lib=None,
              softcap: float = 0.0, mask2d=None):
    """The definition, in fp64.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; key_lens: [B] ints or None;
    mask: additive mask broadcastable to [B, Hq, Nq, Nk] or None;
    rows: optional list of query indices computed in every head (others are NaN);
    softcap: > 0 replaces the scaled score x by softcap * tanh(x / softcap);
    mask2d: None, ("neighborhood", W, R) or ("window", W, w, shift) -- token n
    of a row-major grid with W tokens per row sits at (n // W, n % W); see
    ``attn_oracle.c`` for the two rules.
    Returns (O [B, Hq, Nq, d] fp64, LSE [B, Hq, Nq] fp64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.full((B, Hq, Nq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    kl = None if key_lens is None else np.ascontiguousarray(np.asarray(key_lens, dtype=np.int32))
    rw = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    mk, sb, sh, sq = (None, 0, 0, 0) if mask is None else _mask_view(_f64(mask), B, Hq, Nq, Nk)
    if softcap == 0.0 and mask2d is None:
        rc = (lib or _load()).oracle_attention_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
            B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(is_causal)),
            _ptr(kl, ctypes.c_int32), _ptr(mk), sb, sh, sq,
            _ptr(rw, ctypes.c_int32), 0 if rw is None else len(rw), int(n_threads))
    else:
        kind, W, size, shift = 0, 0, 0, 0
        if mask2d is not None:
            kind = MASK2D_KINDS[mask2d[0]]
            W, size = int(mask2d[1]), int(mask2d[2])
            shift = int(mask2d[3]) if len(mask2d) > 3 else 0
        rc = (lib or _load()).oracle_attention_fwd_mod(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
            B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(is_causal)),
            _ptr(kl, ctypes.c_int32), _ptr(mk), sb, sh, sq,
            float(softcap), kind, W, size, shift,
            _ptr(rw, ctypes.c_int32), 0 if rw is None else len(rw), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_attention_fwd rejected its arguments (status {rc})")
    return out, lse


def e4m3_decode(codes) -> np.ndarray:
    """Value of each FP8 E4M3 code (uint8): sign bit 7, exponent bits 6..3 with
    bias 7, mantissa bits 2..0; exponent 0 is subnormal (m / 8 * 2^-6); the
    all-ones exponent and mantissa (0x7F, 0xFF) is NaN; there are no infinities.
    The format behind the FP8 tensor-core inputs of "FlashAttention technical
    analysis" (jsqmd.com/news/722897) sections 4.2 and 6.3."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = sign * val
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def dequantize_blocks(codes, scales, block: int = 128) -> np.ndarray:
    """codes [..., N, d] (E4M3), scales [..., ceil(N / block)]: row i of every
    head is multiplied by its block's scale, scales[..., i // block] ("each
    block keeps its own scale factor", jsqmd.com/news/722897 section 6.3)."""
    x = e4m3_decode(codes)
    s = np.asarray(scales, dtype=np.float64)
    n = x.shape[-2]
    idx = np.arange(n) // block
    return x * s[..., idx][..., None]


def e4m3_encode(y) -> np.ndarray:
    """E4M3 code (uint8) of each fp32 value y, |y| <= 448, rounded to the nearest
    representable value with ties to the even code: written from the format
    (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
    holds the subnormals m / 8 * 2^-6; the largest finite value is 1.75 * 2^8 =
    448).  The sign bit is taken from y's sign bit (-0.0 gives 0x80)."""
    y = np.asarray(y, dtype=np.float32)
    if (np.abs(y) > 448.0).any() or np.isnan(y).any():
        raise ValueError("e4m3_encode: values must be finite and within [-448, 448]")
    a = np.abs(y).astype(np.float64)  # exact
    sign = np.signbit(y).astype(np.int64) << 7
    # binade of each value (normals: exponent e in [-6, 8]); subnormals use e = -6
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    e = np.maximum(e, -6)
    # the value in units of the grid spacing 2^(e - 3) of its binade, rounded half to even
    units = np.rint(a / np.exp2(e - 3.0)).astype(np.int64)  # 8..16 for normals, 0..8 below 2^-6
    normal = a >= 2.0 ** -6
    carry = units == 16  # rounded up to the next binade
    e = np.where(carry, e + 1, e)
    units = np.where(carry, 8, units)
    code_normal = ((e + 7) << 3) | (units - 8)
    code_sub = units  # units of 2^-9; 8 means exactly 2^-6, code 0x08, the first normal
    code = np.where(normal, code_normal, code_sub)
    return (sign | code).astype(np.uint8)


def quantize_e4m3_blocks(x, block: int = 128):
    """FP8 block quantisation of x [..., N, d] ("each block keeps its own scale
    factor", "FlashAttention technical analysis", jsqmd.com/news/722897,
    section 6.3): per block of `block` rows of each head, in fp32 arithmetic,
      amax = max |x| over the block,  scale = amax / 448 (1 when amax = 0),
      code = e4m3(min(max(x / scale, -448), 448))
    with the division and e4m3 both rounding to nearest even.  Returns (codes
    uint8 [..., N, d], scales fp32 [..., ceil(N / block)])."""
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[-2]
    nb = (n + block - 1) // block
    scales = np.empty(x.shape[:-2] + (nb,), dtype=np.float32)
    codes = np.empty(x.shape, dtype=np.uint8)
    for j in range(nb):
        xb = x[..., j * block:(j + 1) * block, :]
        amax = np.abs(xb).max(axis=(-1, -2))
        sc = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)
        scales[..., j] = sc
        y = (xb / sc[..., None, None]).astype(np.float32)  # fp32, correctly rounded
        codes[..., j * block:(j + 1) * block, :] = e4m3_encode(np.clip(y, np.float32(-448.0), np.float32(448.0)))
    return codes, scales


def attention_fp8(q8, k8, v8, q_scale, k_scale, v_scale, **kw):
    """The definition on the dequantized FP8 inputs (fp64): (O, LSE)."""
    return attention(dequantize_blocks(q8, q_scale), dequantize_blocks(k8, k_scale),
                     dequantize_blocks(v8, v_scale), **kw)


def _masked_scores(q, k, scale, is_causal, key_lens, mask):
    """Scaled scores with masked positions at -inf, [B, Hq, Nq, Nk] fp64 (numpy)."""
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    group = Hq // Hkv
    kk = np.repeat(k, group, axis=1)  # query head h reads K/V head h // group
    s = scale * np.einsum("bhid,bhjd->bhij", q, kk)
    if mask is not None:
        s = s + np.broadcast_to(np.asarray(mask, dtype=np.float64), s.shape)
    j = np.arange(Nk)
    if key_lens is not None:
        kl = np.asarray(key_lens).reshape(B, 1, 1, 1)
        s = np.where(j[None, None, None, :] >= kl, -np.inf, s)
    if is_causal:
        i = np.arange(Nq)
        s = np.where(j[None, :] > i[:, None], -np.inf, s)
    return s


def probabilities(q, k, *, scale=None, is_causal=False, key_lens=None, mask=None):
    """Materialised softmax matrix P [B, Hq, Nq, Nk] (fp64); fully masked rows are 0."""
    q, k = _f64(q), _f64(k)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    s = _masked_scores(q, k, scale, is_causal, key_lens, mask)
    m = s.max(axis=-1, keepdims=True)
    safe_m = np.where(np.isneginf(m), 0.0, m)
    p = np.exp(s - safe_m)
    l = p.sum(axis=-1, keepdims=True)
    return np.where(l > 0, p / np.where(l > 0, l, 1.0), 0.0)


def attention_online(q, k, v, *, block: int, scale=None, is_causal=False, key_lens=None, mask=None):
    """Tiled re-statement: loop over key blocks of size ``block`` keeping, per row,
    a running max m, a running sum l and an unnormalised accumulator acc; when a
    block raises the max, rescale l and acc by exp(m_old - m_new); divide once at
    the end (jsqmd.com/news/722897 section 2.2 and the deferred rescaling of
    section 4.1).  fp64, numpy, tiny inputs only.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    group = Hq // Hkv
    vv = np.repeat(v, group, axis=1)
    s_all = _masked_scores(q, k, scale, is_causal, key_lens, mask)
    m = np.full((B, Hq, Nq), -np.inf)
    l = np.zeros((B, Hq, Nq))
    acc = np.zeros((B, Hq, Nq, d))
    for j0 in range(0, Nk, block):
        s = s_all[..., j0:j0 + block]
        m_new = np.maximum(m, s.max(axis=-1))
        # rows that have seen no unmasked key keep m = -inf; use 0 as the shift there
        shift = np.where(np.isneginf(m_new), 0.0, m_new)
        alpha = np.where(np.isneginf(m), 0.0, np.exp(m - shift))
        p = np.exp(s - shift[..., None])
        l = alpha * l + p.sum(axis=-1)
        acc = alpha[..., None] * acc + np.einsum("bhij,bhjd->bhid", p, vv[:, :, j0:j0 + block])
        m = m_new
    out = np.where(l[..., None] > 0, acc / np.where(l > 0, l, 1.0)[..., None], 0.0)
    lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return out, lse


def attention_loops(q, k, v, *, scale=None, is_causal=False, key_lens=None, mask=None):
    """Brute force with pure-Python loops and the math module; tiny inputs only."""
    q, k, v = _f64(q).tolist(), _f64(k).tolist(), _f64(v).tolist()
    B, Hq, Nq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, Nk = len(k[0]), len(k[0][0])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mk = None if mask is None else np.broadcast_to(_f64(mask), (B, Hq, Nq, Nk)).tolist()
    out = [[[[0.0] * d for _ in range(Nq)] for _ in range(Hq)] for _ in range(B)]
    lse = [[[0.0] * Nq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        n_valid = Nk if key_lens is None else int(key_lens[b])
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(Nq):
                keys = [j for j in range(Nk) if j < n_valid and not (is_causal and j > i)]
                scores = {}
                for j in keys:
                    dot = 0.0
                    for t in range(d):
                        dot += q[b][h][i][t] * k[b][hk][j][t]
                    sc = scale * dot + (mk[b][h][i][j] if mk is not None else 0.0)
                    if sc != -math.inf:
                        scores[j] = sc
                if not scores:
                    lse[b][h][i] = -math.inf
                    continue
                top = max(scores.values())
                w = {j: math.exp(sc - top) for j, sc in scores.items()}
                total = sum(w.values())
                for t in range(d):
                    out[b][h][i][t] = sum(w[j] * v[b][hk][j][t] for j in w) / total
                lse[b][h][i] = top + math.log(total)
    return np.array(out, dtype=np.float64), np.array(lse, dtype=np.float64)
