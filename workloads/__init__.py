"""Seeded synthetic attention workloads shared by the tests, the smoke check and
the benchmark.

This module holds no attention arithmetic: it only names the shapes and draws
the random inputs, so that the CUDA path and the fp64 oracle see the same bf16
bits.  Q, K and V are drawn i.i.d. N(0, 1) in fp32 from a seeded torch
generator and rounded to bf16 (round to nearest even); per-sample key lengths
are drawn uniformly from [8, 77].

The shapes stand in for the pages' workloads (no model weights or datasets are
used):
  tiny         B1  H2  N128          d64   -- small enough for full brute force
  vit          B128 H16 N196         d64   -- 14x14-patch ViT self-attention
                                               (atyun.com/61003.html, toy ViT)
  long         B8  H32 N4096         d128  -- the B8 H32 N4096 d128 benchmark shape
  long_causal  same, is_causal             (aiknowledge.cn FlashAttention benchmark page)
  unet_self    B4  H8  N4096         d64   -- 64x64-latent UNet self-attention
  unet_cross   B4  H8  Nq4096 Nk77   d64   -- UNet text cross-attention, padded keys
                                               (xxmr.cn/news/81028, sections 2.1-2.2)
  prefill_gqa  B1  Hq32 Hkv2 N16384  d128, causal -- grouped-head LLM prefill
                                               (jsqmd.com/news/348824, causal=True)
  decode_gqa   B8  Hq32 Hkv8 Nq1 Nk16384 d128 -- one decoding step over a 16K-key
                                               cache, grouped heads (the decoding
                                               phase of jsqmd.com/news/722897,
                                               section 5.2); run with split-KV
  long_bwd, long_causal_bwd, prefill_gqa_bwd -- the backward pass (dQ, dK, dV) of the
                        same shapes (section 3.3 of jsqmd.com/news/722897: training
                        recomputes P from the saved statistics)
  vit3136_softcap       B8 H12 N3136 d64, soft-cap 30 -- the 56 x 56-patch ViT of
  vit3136_neighborhood  B8 H12 N3136 d64, radius-5      the PyTorch attention article
                        neighbourhood on the 56-wide    (atyun.com/61003.html: its
                        token grid                      score_mod and mask_mod examples)
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    is_causal: bool = False
    key_lens: tuple | None = None  # (low, high) inclusive range of per-sample key lengths
    seed: int = 0
    split_kv: bool = False  # run through the split-KV entry point (automatic range count)
    softcap: float = 0.0    # > 0: soft-capped scores (attn_fwd_mod)
    mask2d: tuple | None = None  # ("neighborhood", W, R) or ("window", W, w, shift) (attn_fwd_mod)
    backward: bool = False  # the step is the backward pass (attn_bwd) of this shape
    fp8: bool = False       # FP8 E4M3 inputs with per-128-row block scales (attn_fwd_fp8)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """FLOPs as the metric counts them: forward 4*B*Hq*Nq*Nk*d, halved when causal.

        The count 4*N^2*d for one head is the one "FlashAttention technical analysis"
        (jsqmd.com/news/722897) section 3.1 uses (8.6 GFLOP at N=4096, d=128).  The
        backward pass counts its five N x N x d products (S recomputed, dP, dV, dQ,
        dK): 2.5 times the forward count.
        """
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d
        if self.backward:
            f *= 2.5
        return f / 2.0 if self.is_causal else f

    def qkvo_bytes(self) -> int:
        """Compulsory HBM bytes: read Q, K, V once, write O once (bf16)."""
        return 2 * self.d * (2 * self.B * self.Hq * self.Nq + 2 * self.B * self.Hkv * self.Nk)

    def lse_bytes(self) -> int:
        return 4 * self.B * self.Hq * self.Nq


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", 1, 2, 2, 128, 128, 64, seed=1000),
        Workload("vit", 128, 16, 16, 196, 196, 64, seed=1001),
        Workload("long", 8, 32, 32, 4096, 4096, 128, seed=1002),
        Workload("long_causal", 8, 32, 32, 4096, 4096, 128, is_causal=True, seed=1012),
        Workload("unet_self", 4, 8, 8, 4096, 4096, 64, seed=1003),
        Workload("unet_cross", 4, 8, 8, 4096, 77, 64, key_lens=(8, 77), seed=1013),
        Workload("prefill_gqa", 1, 32, 2, 16384, 16384, 128, is_causal=True, seed=1004),
        Workload("decode_gqa", 8, 32, 8, 1, 16384, 128, seed=1005, split_kv=True),
        Workload("long_bwd", 8, 32, 32, 4096, 4096, 128, seed=1008, backward=True),
        Workload("long_causal_bwd", 8, 32, 32, 4096, 4096, 128, is_causal=True, seed=1009, backward=True),
        Workload("prefill_gqa_bwd", 1, 32, 2, 16384, 16384, 128, is_causal=True, seed=1010, backward=True),
        Workload("long_fp8", 8, 32, 32, 4096, 4096, 128, seed=1014, fp8=True),
        Workload("long_causal_fp8", 8, 32, 32, 4096, 4096, 128, is_causal=True, seed=1015, fp8=True),
        # quarters of long_fp8, long, long_bwd and decode_gqa (inputs still larger than
        # L2, under 1 GB on the device), for full ncu captures
        Workload("long_fp8_small", 2, 32, 32, 4096, 4096, 128, seed=1016, fp8=True),
        Workload("long_small", 2, 32, 32, 4096, 4096, 128, seed=1017),
        Workload("long_bwd_small", 2, 32, 32, 4096, 4096, 128, seed=1018, backward=True),
        Workload("decode_gqa_small", 2, 32, 8, 1, 16384, 128, seed=1019, split_kv=True),
        Workload("long_causal_small", 2, 32, 32, 4096, 4096, 128, is_causal=True, seed=1020),
        Workload("long_causal_fp8_small", 2, 32, 32, 4096, 4096, 128, is_causal=True, seed=1022, fp8=True),
        # half of prefill_gqa (one K/V head and its 16 query heads)
        Workload("prefill_gqa_small", 1, 16, 1, 16384, 16384, 128, is_causal=True, seed=1021),
        Workload("vit3136_softcap", 8, 12, 12, 3136, 3136, 64, seed=1006, softcap=30.0),
        Workload("vit3136_neighborhood", 8, 12, 12, 3136, 3136, 64, seed=1007, mask2d=("neighborhood", 56, 5)),
    ]
}


def quantize_e4m3_blocks(x: torch.Tensor, block: int = 128):
    """Per-128-row-block FP8 E4M3 codes of x [..., N, d] (fp32): scale = amax of
    the block / 448 (the largest finite E4M3 value), codes = round-to-nearest of
    x / scale by torch's float8_e4m3fn conversion.  Returns (codes uint8, scales
    fp32 [..., ceil(N / block)])."""
    n = x.shape[-2]
    nb = (n + block - 1) // block
    pad = nb * block - n
    xp = torch.nn.functional.pad(x, (0, 0, 0, pad))
    xb = xp.reshape(*x.shape[:-2], nb, block, x.shape[-1])
    amax = xb.abs().amax(dim=(-1, -2))
    scales = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).to(torch.float32)
    y = (xb / scales[..., None, None]).clamp(-448.0, 448.0).reshape(*xp.shape)[..., :n, :]
    return y.to(torch.float8_e4m3fn).view(torch.uint8).contiguous(), scales.contiguous()


def make_fp8_inputs(B, Hq, Hkv, Nq, Nk, d, seed, device="cpu"):
    """FP8 Q, K, V (codes and per-128-row scales) from N(0, 1) fp32 draws of a
    generator on ``device`` seeded with ``seed``."""
    g = torch.Generator(device=device).manual_seed(int(seed))
    q = torch.randn((B, Hq, Nq, d), generator=g, device=device)
    k = torch.randn((B, Hkv, Nk, d), generator=g, device=device)
    v = torch.randn((B, Hkv, Nk, d), generator=g, device=device)
    (q8, qs), (k8, ks), (v8, vs) = (quantize_e4m3_blocks(t) for t in (q, k, v))
    return q8, k8, v8, qs, ks, vs


def make_qkv(B, Hq, Hkv, Nq, Nk, d, seed, device="cpu"):
    """bf16 Q [B,Hq,Nq,d], K/V [B,Hkv,Nk,d], i.i.d. N(0,1) rounded to bf16."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))

    def draw(shape):
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)

    q = draw((B, Hq, Nq, d))
    k = draw((B, Hkv, Nk, d))
    v = draw((B, Hkv, Nk, d))
    return q, k, v


def make_key_lens(B, low, high, seed):
    """int32 [B] drawn uniformly from [low, high] inclusive (CPU generator)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7919)
    return torch.randint(int(low), int(high) + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def make_inputs(w: Workload, device="cpu", seed=None):
    """Returns (q, k, v, key_lens or None) for a workload."""
    s = w.seed if seed is None else seed
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, s, device)
    kl = None
    if w.key_lens is not None:
        kl = make_key_lens(w.B, w.key_lens[0], w.key_lens[1], s).to(device)
    return q, k, v, kl
