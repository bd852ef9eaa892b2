"""The end-to-end call with host buffers (HostAttention): the batch is cut into
chunks whose copies and kernels overlap on three streams; the result must be
bit-identical to the call on device-resident inputs, over repeated calls
(later calls reuse the staging buffers) and for every chunk count."""
import pytest
import torch

import exact_attention_157_b200 as ea
from workloads import make_qkv

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.mark.parametrize("chunks", [1, 3, 5])
def test_matches_device_call_bitwise(chunks):
    B, Hq, Hkv, N, d = 5, 4, 2, 300, 128
    lens = torch.tensor([300, 0, 17, 256, 129], dtype=torch.int32)
    runner = ea.HostAttention(B, Hq, Hkv, N, N, d, device=DEV, with_key_lens=True, chunks=chunks)
    for seed in (1, 2):  # two calls: the second reuses the staging buffers
        q, k, v = make_qkv(B, Hq, Hkv, N, N, d, seed=seed)
        ref_o, ref_l = ea.attention(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=True, key_lens=lens.to(DEV))
        qh, kh, vh, lh = (t.pin_memory() for t in (q, k, v, lens))
        oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        lseh = torch.empty((B, Hq, N), dtype=torch.float32).pin_memory()
        runner(qh, kh, vh, oh, lseh, lh, is_causal=True)
        torch.cuda.current_stream().synchronize()
        ea.check_device_status()
        assert torch.equal(oh, ref_o.cpu()) and torch.equal(lseh, ref_l.cpu())


def test_short_keys_and_split_kv():
    """The short-key kernel and the split-KV path behind the same host call.  A
    fixed range count keeps the key ranges of every chunk those of the whole
    batch (an automatic count is planned per chunk: equal within the parity
    tolerances, not bit for bit)."""
    for (B, Hq, Hkv, Nq, Nk, d, split) in [(8, 4, 4, 196, 196, 64, None), (6, 8, 2, 1, 3000, 128, 4)]:
        q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=B + Nk)
        ref_o, ref_l = ea.attention(q.to(DEV), k.to(DEV), v.to(DEV), split_kv=split)
        runner = ea.HostAttention(B, Hq, Hkv, Nq, Nk, d, device=DEV, split_kv=split, chunks=4)
        oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        lseh = torch.empty((B, Hq, Nq), dtype=torch.float32).pin_memory()
        runner(q.pin_memory(), k.pin_memory(), v.pin_memory(), oh, lseh)
        torch.cuda.current_stream().synchronize()
        ea.check_device_status()
        assert torch.equal(oh, ref_o.cpu()) and torch.equal(lseh, ref_l.cpu())


def test_automatic_split_kv_chunks_plan_their_own_ranges():
    """split_kv=0 (automatic) on a decoding shape: a chunk of one batch entry
    takes more key ranges than the whole batch, so the workspace must hold the
    largest chunk plan; the result equals the device call within the parity
    tolerances (the ranges, and so the merge order, differ)."""
    B, Hq, Hkv, Nq, Nk, d = 8, 32, 8, 1, 16384, 128
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=5)
    ref_o, ref_l = ea.attention(q.to(DEV), k.to(DEV), v.to(DEV), split_kv=0)
    runner = ea.HostAttention(B, Hq, Hkv, Nq, Nk, d, device=DEV, split_kv=0)
    oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    lseh = torch.empty((B, Hq, Nq), dtype=torch.float32).pin_memory()
    runner(q.pin_memory(), k.pin_memory(), v.pin_memory(), oh, lseh)
    torch.cuda.current_stream().synchronize()
    ea.check_device_status()
    assert (oh.float() - ref_o.cpu().float()).abs().max().item() <= 1e-2
    assert (lseh - ref_l.cpu()).abs().max().item() <= 1e-3
