"""The device FP8 block quantiser (attn_quantize_e4m3_blocks) against the
oracle's quantiser: codes and scales bit-exact (both take every rounding
decision in fp32, to nearest even), then the quantised tensors through the FP8
forward pass against the oracle on the same codes."""
import numpy as np
import pytest
import torch

import exact_attention_157_b200 as ea
import oracle
from workloads import make_qkv

from test_fp8_gpu import check

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def quantize_both(x_bf16):
    codes, scales = ea.quantize_e4m3_blocks(x_bf16.to(DEV))
    ea.check_device_status()
    ref_c, ref_s = oracle.quantize_e4m3_blocks(x_bf16.float().numpy())
    return codes.cpu().numpy(), scales.cpu().numpy(), ref_c, ref_s


@pytest.mark.parametrize("shape", [(2, 3, 300, 128), (1, 1, 1, 64), (4, 2, 128, 128), (3, 5, 129, 64),
                                   (1, 2, 4096, 128)])
def test_bit_exact_against_the_oracle(shape):
    g = torch.Generator().manual_seed(sum(shape))
    x = (torch.randn(shape, generator=g) * torch.exp2(torch.randint(-20, 20, shape[:-1] + (1,), generator=g)))
    x = x.to(torch.bfloat16)
    codes, scales, ref_c, ref_s = quantize_both(x)
    np.testing.assert_array_equal(scales, ref_s)
    np.testing.assert_array_equal(codes, ref_c)


def test_special_blocks():
    """A zero block (scale 1, codes 0), negative zeros (code 0x80), a block whose
    magnitudes span the subnormal range, and the largest bf16 values."""
    x = torch.zeros(1, 4, 260, 128)
    x[0, 1] = -0.0
    x[0, 2] = torch.randn(260, 128) * 1e-6
    x[0, 2, 5, 7] = 1.0  # amax 1: the rest falls into E4M3's subnormals
    x[0, 3] = torch.randn(260, 128) * 1e37
    x = x.to(torch.bfloat16)
    codes, scales, ref_c, ref_s = quantize_both(x)
    np.testing.assert_array_equal(scales, ref_s)
    np.testing.assert_array_equal(codes, ref_c)
    assert (scales[0, 0] == 1.0).all() and (codes[0, 0] == 0).all() and (codes[0, 1] == 0x80).all()


def test_quantised_inputs_through_the_fp8_forward():
    """bf16 Q, K, V -> device quantiser -> attn_fwd_fp8, against the oracle on the
    same codes and scales (the FP8 tolerances of test_fp8_gpu)."""
    q, k, v = make_qkv(2, 4, 2, 300, 700, 128, seed=21)
    qc, qs = ea.quantize_e4m3_blocks(q.to(DEV))
    kc, ks = ea.quantize_e4m3_blocks(k.to(DEV))
    vc, vs = ea.quantize_e4m3_blocks(v.to(DEV))
    ea.check_device_status()
    cpu = [t.cpu() for t in (qc, kc, vc, qs, ks, vs)]
    check(*cpu, is_causal=True)


def test_argument_errors():
    x = torch.zeros(1, 2, 8, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ea.AttnError) as e:
        ea.quantize_e4m3_blocks(x)
    assert e.value.status == ea.ATTN_ERR_UNSUPPORTED
    with pytest.raises(TypeError):
        ea.quantize_e4m3_blocks(torch.zeros(1, 8, 64, device=DEV))
