"""attn_fwd_splitkv_noalloc: split-KV with the library's fixed scratch buffer,
called through the C ABI with raw device pointers and compared with the
caller-workspace entry point attn_fwd_splitkv (and the fp64 oracle) within the
parity tolerances, on two calls in a row.  Collected last so that it also runs
after every other GPU test; it must pass on its own in a fresh process too."""
import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from workloads import make_qkv

from tolerances import assert_close, reference

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    return q, k, v, q.to(DEV), k.to(DEV), v.to(DEV)


def _noalloc(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, n_splits, key_lens=None, causal=False, mask=None, out=None,
             lse=None, check=True):
    out = torch.empty_like(qd) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=DEV) if lse is None else lse
    st = ea.attn_fwd_splitkv_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                     B, Hq, Hkv, Nq, Nk, d, 0.0, causal,
                                     key_lens=None if key_lens is None else key_lens.data_ptr(),
                                     additive_mask=None if mask is None else mask.data_ptr(),
                                     n_splits=n_splits, stream=ea._stream_handle(None))
    assert st == ea.ATTN_OK, ea.status_string(st)
    if check:
        ea.check_device_status()
    return out, lse


def _with_workspace(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, n_splits, key_lens=None, causal=False, mask=None):
    st, _, nbytes = ea.attn_splitkv_plan(B, Hq, Nq, Nk, d, n_splits, 0, Hkv=Hkv, is_causal=causal)
    assert st == ea.ATTN_OK
    ws = torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(qd)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=DEV)
    st = ea.attn_fwd_splitkv(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, Hq, Hkv, Nq, Nk, d, 0.0, causal,
                             key_lens=None if key_lens is None else key_lens.data_ptr(),
                             additive_mask=None if mask is None else mask.data_ptr(),
                             n_splits=n_splits, workspace=ws.data_ptr(), workspace_bytes=nbytes,
                             stream=ea._stream_handle(None))
    assert st == ea.ATTN_OK, ea.status_string(st)
    ea.check_device_status()
    return out, lse


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,n_splits", [
    (4, 16, 4, 1, 5000, 128, 0),
    (2, 8, 2, 3, 3000, 64, 6),
    (1, 4, 4, 200, 1100, 128, 3),
])
def test_noalloc_matches_workspace_entry_point_twice(B, Hq, Hkv, Nq, Nk, d, n_splits):
    q, k, v, qd, kd, vd = _inputs(B, Hq, Hkv, Nq, Nk, d, seed=B * 100 + Nq + Nk + d)
    ref_o, ref_l = _with_workspace(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, n_splits)
    ro, rl, ra = reference(q, k, v)
    for _ in range(2):  # two calls in a row reuse the same scratch
        out, lse = _noalloc(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, n_splits)
        assert (out.float() - ref_o.float()).abs().max().item() <= 1e-2
        assert (lse - ref_l).abs().max().item() <= 1e-3
        assert_close(out, lse, ro, rl, rabs=ra)


@pytest.mark.parametrize("case", ["causal", "decode_shape_with_mask"])
def test_noalloc_causal_and_masked_decode_shape_twice(case):
    """The two other plan branches: a causal call (tile kernel, key ranges that
    end at the diagonal), and a decoding shape given an additive mask, which runs
    the tile kernel with the range count of the decode plan."""
    if case == "causal":
        B, Hq, Hkv, Nq, Nk, d, n_splits = 2, 4, 2, 700, 700, 64, 3
    else:
        B, Hq, Hkv, Nq, Nk, d, n_splits = 2, 8, 2, 2, 2500, 128, 0
    q, k, v, qd, kd, vd = _inputs(B, Hq, Hkv, Nq, Nk, d, seed=29 + Nk)
    mask = None
    if case != "causal":
        g = torch.Generator().manual_seed(30)
        mask = torch.randn(B, Hq, Nq, Nk, generator=g) * 2.0
        mask[0, 1, 0, 600:] = -float("inf")
    causal = case == "causal"
    md = None if mask is None else mask.to(DEV)
    ref_o, ref_l = _with_workspace(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, n_splits, causal=causal, mask=md)
    ro, rl, ra = reference(q, k, v, is_causal=causal, mask=None if mask is None else mask.double().numpy())
    for _ in range(2):
        out, lse = _noalloc(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, n_splits, causal=causal, mask=md)
        assert (out.float() - ref_o.float()).abs().max().item() <= 1e-2
        assert (lse - ref_l).abs().max().item() <= 1e-3
        assert_close(out, lse, ro, rl, rabs=ra)
        assert_close(ref_o, ref_l, ro, rl, rabs=ra)


def test_noalloc_key_lens_twice_and_no_new_device_memory():
    B, Hq, Hkv, Nq, Nk, d = 3, 8, 8, 2, 4000, 128
    q, k, v, qd, kd, vd = _inputs(B, Hq, Hkv, Nq, Nk, d, seed=17)
    lens = torch.tensor([4000, 0, 1500], dtype=torch.int32, device=DEV)
    ref_o, ref_l = _with_workspace(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, 5, key_lens=lens)
    _noalloc(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, 5, key_lens=lens)  # set-up done by now
    outs = [torch.empty_like(qd) for _ in range(2)]
    lses = [torch.empty((B, Hq, Nq), dtype=torch.float32, device=DEV) for _ in range(2)]
    torch.cuda.synchronize()
    # only the library calls run between the two readings of free device memory
    free0 = torch.cuda.mem_get_info(DEV)[0]
    for i in range(2):
        _noalloc(qd, kd, vd, B, Hq, Hkv, Nq, Nk, d, 5, key_lens=lens, out=outs[i], lse=lses[i], check=False)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info(DEV)[0]
    ea.check_device_status()
    assert free1 == free0
    for out, lse in zip(outs, lses):
        assert (out.float() - ref_o.float()).abs().max().item() <= 1e-2
        fin = torch.isfinite(ref_l)
        assert torch.equal(torch.isneginf(lse), torch.isneginf(ref_l))
        assert (lse[fin] - ref_l[fin]).abs().max().item() <= 1e-3


def test_noalloc_rejects_plans_beyond_the_fixed_buffer():
    # 4096 rows x 8 ranges x (128 + 1) fp32 values = 16.9 MB > 16 MiB; real buffers
    B, Hq, Hkv, Nq, Nk, d = 1, 8, 8, 512, 8192, 128
    st, used, nbytes = ea.attn_splitkv_plan(B, Hq, Nq, Nk, d, 8, 0, Hkv=Hkv)
    assert st == ea.ATTN_OK and used == 8 and nbytes > ea.NOALLOC_SCRATCH_BYTES
    _, _, _, qd, kd, vd = _inputs(B, Hq, Hkv, Nq, Nk, d, seed=23)
    out = torch.zeros_like(qd)
    st = ea.attn_fwd_splitkv_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), out.data_ptr(), None,
                                     B, Hq, Hkv, Nq, Nk, d, 0.0, False, n_splits=8,
                                     stream=ea._stream_handle(None))
    assert st == ea.ATTN_ERR_SCRATCH
    assert "scratch" in ea.status_string(st)
    torch.cuda.synchronize()
    assert int(out.abs().sum().item()) == 0  # nothing was launched
