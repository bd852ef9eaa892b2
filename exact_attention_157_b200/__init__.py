"""Python binding of the sm_100a exact attention library (include/attn.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of ``libattn_sm100.so``.  There is no fallback: if the library or a
B200 is missing, calls raise.

    from exact_attention_157_b200 import attention
    out, lse = attention(q, k, v, is_causal=True)        # torch bf16 CUDA tensors

Split-KV (decode-shaped inputs: few queries, many keys):

    out, lse = attention(q, k, v, split_kv=0)            # 0 = automatic range count

Lower level, with the C names and raw pointers:

    attn_fwd(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, B, Hq, Hkv, Nq, Nk, d,
             scale, is_causal, key_lens_ptr, mask_ptr, mask_strides, stream)
    attn_splitkv_plan(B, Hq, Nq, Nk, d, n_splits, sm_count) -> (status, n_used, bytes)
    attn_fwd_splitkv(..., n_splits, workspace_ptr, workspace_bytes, stream)
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_sm100.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_ALIGNMENT = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
ATTN_ERR_DEVICE = 6
ATTN_ERR_SCRATCH = 7
NOALLOC_SCRATCH_BYTES = 16 << 20  # ATTN_NOALLOC_SCRATCH_BYTES

# Every symbol include/attn.h declares.
EXPORTED = ("attn_fwd", "attn_fwd_mod", "attn_fwd_fp8", "attn_bwd_plan", "attn_bwd", "attn_splitkv_plan", "attn_fwd_splitkv", "attn_fwd_splitkv_noalloc",
            "attn_check_device_status", "attn_set_wait_timeout_ns", "attn_selftest_timeout",
            "attn_selftest_exp2_poly", "attn_quantize_e4m3_blocks", "attn_bwd_ex", "attn_status_string", "attn_last_cuda_error", "attn_version")

MASK2D_KINDS = {None: 0, "neighborhood": 1, "window": 2}


class AttnScoreMod(ctypes.Structure):
    """attn_score_mod_t of include/attn.h."""
    _fields_ = [("softcap", ctypes.c_float), ("mask2d_kind", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("size", ctypes.c_int), ("shift", ctypes.c_int)]


def score_mod(softcap=0.0, mask2d=None) -> AttnScoreMod:
    """Build an attn_score_mod_t: mask2d is None, ("neighborhood", W, R) or
    ("window", W, w[, shift])."""
    m = AttnScoreMod(float(softcap or 0.0), 0, 0, 0, 0)
    if mask2d is not None:
        m.mask2d_kind = MASK2D_KINDS[mask2d[0]]
        m.grid_w, m.size = int(mask2d[1]), int(mask2d[2])
        m.shift = int(mask2d[3]) if len(mask2d) > 3 else 0
    return m


_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = status_string(status)
        if status == ATTN_ERR_CUDA:
            msg += f" (cudaError {last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def lib() -> ctypes.CDLL:
    """Load ``libattn_sm100.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing; build it with "
                                  "`python -m exact_attention_157_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            L.attn_fwd.restype = i
            L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp, vp]
            L.attn_fwd_mod.restype = i
            L.attn_fwd_mod.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, ctypes.POINTER(AttnScoreMod), vp]
            L.attn_fwd_fp8.restype = i
            L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp]
            L.attn_bwd_plan.restype = i
            L.attn_bwd_plan.argtypes = [i, i, i, ctypes.POINTER(ctypes.c_size_t)]
            L.attn_bwd.restype = i
            L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp,
                                   ctypes.c_size_t, vp]
            L.attn_splitkv_plan.restype = i
            L.attn_splitkv_plan.argtypes = [i, i, i, i, i, i, i, i, i, ctypes.POINTER(i),
                                            ctypes.POINTER(ctypes.c_size_t)]
            L.attn_fwd_splitkv.restype = i
            L.attn_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp,
                                           i, vp, ctypes.c_size_t, vp]
            L.attn_fwd_splitkv_noalloc.restype = i
            L.attn_fwd_splitkv_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp, i, vp]
            L.attn_check_device_status.restype = i
            L.attn_check_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
            L.attn_set_wait_timeout_ns.restype = i
            L.attn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
            L.attn_selftest_timeout.restype = i
            L.attn_selftest_timeout.argtypes = [vp]
            L.attn_selftest_exp2_poly.restype = i
            L.attn_selftest_exp2_poly.argtypes = [vp, vp, i, vp]
            L.attn_quantize_e4m3_blocks.restype = i
            L.attn_quantize_e4m3_blocks.argtypes = [vp, vp, vp, i, i, i, vp]
            L.attn_bwd_ex.restype = i
            L.attn_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp,
                                      ctypes.POINTER(AttnScoreMod), vp, ctypes.c_size_t, vp]
            L.attn_status_string.restype = ctypes.c_char_p
            L.attn_status_string.argtypes = [i]
            L.attn_last_cuda_error.restype = i
            L.attn_last_cuda_error.argtypes = []
            L.attn_version.restype = i
            L.attn_version.argtypes = []
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def last_cuda_error() -> int:
    return int(lib().attn_last_cuda_error())


def version() -> int:
    return int(lib().attn_version())


# ------------------------------------------------------------- C-named calls
def attn_fwd(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal,
             key_lens=None, additive_mask=None, mask_strides=None, stream=None) -> int:
    """The C entry point with raw device pointers (ints); returns the status code."""
    ms = None
    if mask_strides is not None:
        arr = (ctypes.c_int64 * 3)(*[int(x) for x in mask_strides])
        ms = ctypes.cast(arr, ctypes.c_void_p)
    return int(lib().attn_fwd(q, k, v, out, lse, int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                              float(scale), int(bool(is_causal)), key_lens, additive_mask, ms, stream))


def attn_fwd_mod(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens=None, mod=None,
                 stream=None) -> int:
    """The C variant entry point with raw device pointers (ints) and an
    AttnScoreMod (or None, passed as NULL); returns the status code."""
    return int(lib().attn_fwd_mod(q, k, v, out, lse, int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                  float(scale), int(bool(is_causal)), key_lens,
                                  None if mod is None else ctypes.byref(mod), stream))


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal,
                 key_lens=None, stream=None) -> int:
    """The C FP8 entry point with raw device pointers (ints); returns the status code."""
    return int(lib().attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, out, lse, int(B), int(Hq), int(Hkv),
                                  int(Nq), int(Nk), int(d), float(scale), int(bool(is_causal)), key_lens, stream))


def attn_bwd_plan(B, Hq, Nq):
    """The C planner of the backward pass: returns (status, workspace bytes)."""
    nb = ctypes.c_size_t(0)
    st = int(lib().attn_bwd_plan(int(B), int(Hq), int(Nq), ctypes.byref(nb)))
    return st, int(nb.value)


def attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, is_causal,
             key_lens=None, workspace=None, workspace_bytes=0, stream=None) -> int:
    """The C backward entry point with raw device pointers (ints); returns the status code."""
    return int(lib().attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, int(B), int(Hq), int(Hkv), int(Nq), int(Nk),
                              int(d), float(scale), int(bool(is_causal)), key_lens, workspace,
                              int(workspace_bytes), stream))


def attn_splitkv_plan(B, Hq, Nq, Nk, d, n_splits=0, sm_count=0, *, Hkv=None, is_causal=False):
    """The C planner: returns (status, key ranges planned, workspace bytes).
    Hkv defaults to Hq (no grouped heads)."""
    n = ctypes.c_int(0)
    nb = ctypes.c_size_t(0)
    st = int(lib().attn_splitkv_plan(int(B), int(Hq), int(Hq if Hkv is None else Hkv), int(Nq), int(Nk), int(d),
                                     int(bool(is_causal)), int(n_splits), int(sm_count),
                                     ctypes.byref(n), ctypes.byref(nb)))
    return st, int(n.value), int(nb.value)


def attn_fwd_splitkv(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal,
                     key_lens=None, additive_mask=None, mask_strides=None, n_splits=0,
                     workspace=None, workspace_bytes=0, stream=None) -> int:
    """The C split-KV entry point with raw device pointers (ints); returns the status code."""
    ms = None
    if mask_strides is not None:
        arr = (ctypes.c_int64 * 3)(*[int(x) for x in mask_strides])
        ms = ctypes.cast(arr, ctypes.c_void_p)
    return int(lib().attn_fwd_splitkv(q, k, v, out, lse, int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                      float(scale), int(bool(is_causal)), key_lens, additive_mask, ms,
                                      int(n_splits), workspace, int(workspace_bytes), stream))


def attn_fwd_splitkv_noalloc(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal,
                             key_lens=None, additive_mask=None, mask_strides=None, n_splits=0,
                             stream=None) -> int:
    """The C split-KV entry point that uses the library's fixed scratch buffer
    (raw device pointers as ints); returns the status code."""
    ms = None
    if mask_strides is not None:
        arr = (ctypes.c_int64 * 3)(*[int(x) for x in mask_strides])
        ms = ctypes.cast(arr, ctypes.c_void_p)
    return int(lib().attn_fwd_splitkv_noalloc(q, k, v, out, lse, int(B), int(Hq), int(Hkv), int(Nq), int(Nk),
                                              int(d), float(scale), int(bool(is_causal)), key_lens, additive_mask,
                                              ms, int(n_splits), stream))


def attn_check_device_status(stream=None):
    """Synchronises ``stream``; returns (status, raw error word)."""
    info = ctypes.c_uint32(0)
    st = int(lib().attn_check_device_status(stream, ctypes.byref(info)))
    return st, int(info.value)


def attn_set_wait_timeout_ns(ns: int) -> int:
    return int(lib().attn_set_wait_timeout_ns(int(ns)))


def attn_selftest_timeout(stream=None) -> int:
    return int(lib().attn_selftest_timeout(stream))


def quantize_e4m3_blocks(x, stream=None):
    """FP8 E4M3 block quantisation of a contiguous bf16 CUDA tensor [..., N, d]
    on the device (attn_quantize_e4m3_blocks): returns (codes uint8 [..., N, d],
    scales fp32 [..., ceil(N / 128)]), the inputs of attention_fp8."""
    import torch
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() >= 2):
        raise TypeError("x must be a contiguous bfloat16 CUDA tensor [..., N, d]")
    N, d = x.shape[-2], x.shape[-1]
    heads = x.numel() // (N * d) if N * d > 0 else 0
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty(tuple(x.shape[:-2]) + ((N + 127) // 128,), dtype=torch.float32, device=x.device)
    st = int(lib().attn_quantize_e4m3_blocks(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), int(heads), int(N),
                                             int(d), _stream_handle(stream)))
    if st != ATTN_OK:
        raise AttnError(st, "attn_quantize_e4m3_blocks")
    return codes, scales


def exp2_poly(x, stream=None):
    """2^x by the FP8 path's FMA-pipe polynomial (attn_selftest_exp2_poly) for a
    contiguous fp32 CUDA tensor; returns a new tensor."""
    import torch
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise TypeError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    st = int(lib().attn_selftest_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(), _stream_handle(stream)))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_exp2_poly")
    return y


# ------------------------------------------------------- torch marshalling
def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_bf16_cuda(name, t, ndim):
    import torch
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


def attention(q, k, v, *, scale: float | None = None, is_causal: bool = False, key_lens=None,
              attn_mask=None, out=None, lse=None, return_lse: bool = True, stream=None,
              split_kv: int | None = None, workspace=None, softcap: float = 0.0, mask2d=None):
    """O = softmax(scale * Q K^T + mask) V on bf16 CUDA tensors.

    q [B, Hq, Nq, d], k/v [B, Hkv, Nk, d] (contiguous bf16); key_lens int32 [B]
    (CUDA) or None; attn_mask fp32 CUDA tensor broadcastable to [B, Hq, Nq, Nk]
    with a contiguous last dimension, or None.  split_kv=None runs attn_fwd;
    an int runs attn_fwd_splitkv with at most that many key ranges (0 =
    automatic), its workspace taken from ``workspace`` (a CUDA tensor of at
    least the planned bytes) or allocated here.  softcap > 0 or a mask2d
    (("neighborhood", W, R) or ("window", W, w[, shift])) runs attn_fwd_mod.
    Returns (out, lse or None).
    """
    import torch
    _check_bf16_cuda("q", q, 4)
    _check_bf16_cuda("k", k, 4)
    _check_bf16_cuda("v", v, 4)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if Bk != B or dk != d or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q, k, v shapes disagree")
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_bf16_cuda("out", out, 4)
        if tuple(out.shape) != tuple(q.shape):
            raise ValueError("out has the wrong shape")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()
                            or tuple(lse.shape) != (B, Hq, Nq)):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Nq] tensor")
    kl_ptr = None
    if key_lens is not None:
        if key_lens.dtype != torch.int32 or key_lens.device != q.device or key_lens.numel() != B:
            raise ValueError("key_lens must be an int32 CUDA tensor with B entries")
        key_lens = key_lens.contiguous()
        kl_ptr = key_lens.data_ptr()
    m_ptr, m_strides = None, None
    if attn_mask is not None:
        if attn_mask.dtype != torch.float32 or attn_mask.device != q.device:
            raise ValueError("attn_mask must be a float32 CUDA tensor")
        m = attn_mask
        while m.dim() < 4:
            m = m.unsqueeze(0)
        m = m.expand(B, Hq, Nq, Nk)
        if m.stride(3) != 1:
            m = m.contiguous()
        m_ptr, m_strides = m.data_ptr(), (m.stride(0), m.stride(1), m.stride(2))
    sc = 0.0 if scale is None else float(scale)
    lse_ptr = None if lse is None else lse.data_ptr()
    if softcap or mask2d is not None:
        if split_kv is not None or attn_mask is not None:
            raise ValueError("softcap / mask2d combine with neither split_kv nor attn_mask")
        st = attn_fwd_mod(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr, B, Hq, Hkv, Nq, Nk, d,
                          sc, is_causal, kl_ptr, score_mod(softcap, mask2d), _stream_handle(stream))
        if st != ATTN_OK:
            raise AttnError(st, "attn_fwd_mod")
        return out, lse
    if split_kv is None:
        st = attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr, B, Hq, Hkv, Nq, Nk, d,
                      sc, is_causal, kl_ptr, m_ptr, m_strides, _stream_handle(stream))
        if st != ATTN_OK:
            raise AttnError(st, "attn_fwd")
        return out, lse
    st, _, nbytes = attn_splitkv_plan(B, Hq, Nq, Nk, d, int(split_kv), 0, Hkv=Hkv, is_causal=is_causal)
    if st != ATTN_OK:
        raise AttnError(st, "attn_splitkv_plan")
    if workspace is None:
        workspace = torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=q.device)
    elif workspace.device != q.device or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA tensor of at least {nbytes} bytes")
    st = attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr, B, Hq, Hkv, Nq, Nk,
                          d, sc, is_causal, kl_ptr, m_ptr, m_strides, int(split_kv), workspace.data_ptr(),
                          workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_splitkv")
    return out, lse


def attention_fp8(q8, k8, v8, q_scale, k_scale, v_scale, *, scale: float | None = None, is_causal: bool = False,
                  key_lens=None, out=None, lse=None, return_lse: bool = True, stream=None):
    """attn_fwd_fp8 on CUDA tensors: q8 [B, Hq, Nq, 128], k8/v8 [B, Hkv, Nk, 128]
    (uint8 or float8_e4m3fn, contiguous), scales fp32 [B, H, ceil(N / 128)].
    Returns (out bf16 [B, Hq, Nq, 128], lse or None)."""
    import torch

    def codes(name, t):
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda" or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D CUDA tensor")
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8)
        if t.dtype != torch.uint8:
            raise TypeError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn)")
        return t

    q8, k8, v8 = codes("q8", q8), codes("k8", k8), codes("v8", v8)
    B, Hq, Nq, d = q8.shape
    Bk, Hkv, Nk, dk = k8.shape
    if Bk != B or dk != d or tuple(v8.shape) != tuple(k8.shape):
        raise ValueError("q8, k8, v8 shapes disagree")
    for name, t, h, n in (("q_scale", q_scale, Hq, Nq), ("k_scale", k_scale, Hkv, Nk), ("v_scale", v_scale, Hkv, Nk)):
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or t.device != q8.device
                or not t.is_contiguous() or tuple(t.shape) != (B, h, (n + 127) // 128)):
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor of shape {(B, h, (n + 127) // 128)}")
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=q8.device)
    else:
        _check_bf16_cuda("out", out, 4)
        if tuple(out.shape) != (B, Hq, Nq, d):
            raise ValueError("out has the wrong shape")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()
                            or tuple(lse.shape) != (B, Hq, Nq)):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Nq] tensor")
    kl_ptr = None
    if key_lens is not None:
        if key_lens.dtype != torch.int32 or key_lens.device != q8.device or key_lens.numel() != B:
            raise ValueError("key_lens must be an int32 CUDA tensor with B entries")
        key_lens = key_lens.contiguous()
        kl_ptr = key_lens.data_ptr()
    st = attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_scale.data_ptr(), k_scale.data_ptr(),
                      v_scale.data_ptr(), out.data_ptr(), None if lse is None else lse.data_ptr(), B, Hq, Hkv, Nq,
                      Nk, d, 0.0 if scale is None else float(scale), is_causal, kl_ptr, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")
    return out, lse


def attention_backward(q, k, v, out, lse, dout, *, scale: float | None = None, is_causal: bool = False,
                       key_lens=None, workspace=None, stream=None, dq=None, dk=None, dv=None,
                       attn_mask=None, softcap: float = 0.0, mask2d=None):
    """dQ, dK, dV of ``attention`` for the upstream gradient ``dout`` (bf16 CUDA
    tensors shaped like q / k / v); ``out`` and ``lse`` are the forward results
    for the same inputs and options (attn_mask, softcap, mask2d as in
    ``attention``).  Returns (dq, dk, dv)."""
    import torch
    for name, t, nd in (("q", q, 4), ("k", k, 4), ("v", v, 4), ("out", out, 4), ("dout", dout, 4)):
        _check_bf16_cuda(name, t, nd)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q / out / dout or k / v shapes disagree")
    if lse is None or lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Nq) or not lse.is_contiguous():
        raise ValueError("lse must be the contiguous fp32 [B, Hq, Nq] LSE of the forward pass")
    st, nbytes = attn_bwd_plan(B, Hq, Nq)
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_plan")
    if workspace is None:
        workspace = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        _check_bf16_cuda(name, t, 4)
        if tuple(t.shape) != tuple(ref.shape):
            raise ValueError(f"{name} has the wrong shape")
    kl_ptr = None
    if key_lens is not None:
        key_lens = key_lens.contiguous()
        kl_ptr = key_lens.data_ptr()
    sc = 0.0 if scale is None else float(scale)
    if attn_mask is None and not softcap and mask2d is None:
        st = attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d, sc, is_causal, kl_ptr,
                      workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream))
        if st != ATTN_OK:
            raise AttnError(st, "attn_bwd")
        return dq, dk, dv
    m_ptr, ms = None, None
    if attn_mask is not None:
        if attn_mask.dtype != torch.float32 or attn_mask.device != q.device:
            raise ValueError("attn_mask must be a float32 CUDA tensor")
        m = attn_mask
        while m.dim() < 4:
            m = m.unsqueeze(0)
        m = m.expand(B, Hq, Nq, Nk)
        if m.stride(3) != 1:
            m = m.contiguous()
        m_ptr = m.data_ptr()
        ms = ctypes.cast((ctypes.c_int64 * 3)(m.stride(0), m.stride(1), m.stride(2)), ctypes.c_void_p)
    mod = score_mod(softcap, mask2d) if (softcap or mask2d is not None) else None
    st = int(lib().attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                               dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                               sc, int(bool(is_causal)), kl_ptr, m_ptr, ms,
                               None if mod is None else ctypes.byref(mod), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream_handle(stream)))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_ex")
    return dq, dk, dv


def check_device_status(stream=None):
    """Raises AttnError if a kernel recorded a device-side failure."""
    st, info = attn_check_device_status(_stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, f"device status (word 0x{info:08x})")


class HostAttention:
    """End-to-end call for inputs that live in (pinned) host memory.

    The batch is cut into ``chunks`` parts that flow through three streams:
    chunk c+1 is copied host -> device while the kernel runs on chunk c and
    chunk c-1's O and LSE are copied back, so the two copy directions and the
    kernels overlap (each copy direction has its own engine).  The call is
    ordered on ``stream``: it starts after the work already queued there and
    everything it does, the last copy back included, precedes the work queued
    there after it.  The device staging buffers (and a split-KV workspace when
    ``split_kv`` is not None, planned for ``is_causal``), the two copy streams
    and their events are made once, here, and reused.  With ``split_kv=0``
    (automatic) each chunk's key ranges are planned for the chunk's batch size.
    """

    def __init__(self, B, Hq, Hkv, Nq, Nk, d, device="cuda:0", with_lse=True, with_key_lens=False,
                 split_kv=None, is_causal=False, chunks=None):
        import torch
        dev = torch.device(device)
        bf = torch.bfloat16
        self.shape = (B, Hq, Hkv, Nq, Nk, d)
        self.q = torch.empty((B, Hq, Nq, d), dtype=bf, device=dev)
        self.k = torch.empty((B, Hkv, Nk, d), dtype=bf, device=dev)
        self.v = torch.empty((B, Hkv, Nk, d), dtype=bf, device=dev)
        self.out = torch.empty((B, Hq, Nq, d), dtype=bf, device=dev)
        self.lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev) if with_lse else None
        self.key_lens = torch.empty((B,), dtype=torch.int32, device=dev) if with_key_lens else None
        self.split_kv = split_kv
        self.workspace = None
        n = min(B, 8) if chunks is None else max(1, min(int(chunks), B))
        self.bounds = [(B * i // n, B * (i + 1) // n) for i in range(n)]
        if split_kv is not None:
            # each chunk is planned for its own batch size (a smaller batch may take
            # more key ranges): the workspace holds the largest of those plans
            nbytes = 0
            for cb in sorted({b1 - b0 for b0, b1 in self.bounds}):
                st, _, nb = attn_splitkv_plan(cb, Hq, Nq, Nk, d, int(split_kv), 0, Hkv=Hkv, is_causal=is_causal)
                if st != ATTN_OK:
                    raise AttnError(st, "attn_splitkv_plan")
                nbytes = max(nbytes, nb)
            self.workspace = torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=dev)
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.ev_in = [torch.cuda.Event() for _ in self.bounds]
        self.ev_out = [torch.cuda.Event() for _ in self.bounds]

    def __call__(self, q_h, k_h, v_h, out_h, lse_h=None, key_lens_h=None, *, scale=None,
                 is_causal=False, stream=None, softcap=0.0, mask2d=None):
        import torch
        s = torch.cuda.current_stream() if stream is None else stream
        # the staging buffers are free once the work queued on s (earlier calls included) is done
        self.h2d.wait_stream(s)
        for (b0, b1), ev_in, ev_out in zip(self.bounds, self.ev_in, self.ev_out):
            with torch.cuda.stream(self.h2d):
                self.q[b0:b1].copy_(q_h[b0:b1], non_blocking=True)
                self.k[b0:b1].copy_(k_h[b0:b1], non_blocking=True)
                self.v[b0:b1].copy_(v_h[b0:b1], non_blocking=True)
                if key_lens_h is not None:
                    self.key_lens[b0:b1].copy_(key_lens_h[b0:b1], non_blocking=True)
                ev_in.record(self.h2d)
            s.wait_event(ev_in)
            kl = None if key_lens_h is None else self.key_lens[b0:b1]
            lse = None if self.lse is None else self.lse[b0:b1]
            attention(self.q[b0:b1], self.k[b0:b1], self.v[b0:b1], scale=scale, is_causal=is_causal, key_lens=kl,
                      out=self.out[b0:b1], lse=lse, return_lse=lse is not None, stream=s,
                      split_kv=self.split_kv, workspace=self.workspace, softcap=softcap, mask2d=mask2d)
            ev_out.record(s)
            self.d2h.wait_event(ev_out)
            with torch.cuda.stream(self.d2h):
                out_h[b0:b1].copy_(self.out[b0:b1], non_blocking=True)
                if lse_h is not None and lse is not None:
                    lse_h[b0:b1].copy_(lse, non_blocking=True)
        s.wait_stream(self.d2h)  # the copies back complete before later work on s
        return out_h, lse_h
