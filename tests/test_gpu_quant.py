"""GPU parity of the weight quantisers (MXFP8, NVFP4) against the oracle.

Codes, block scales and matrix scales are integer decisions: bit-exact.
The kernels' per-block arithmetic is also checked on the CPU (host build,
test_quant_codec_host.py); here the launch, indexing and packing on the
device are what is new.  Sizes span several grid strides and ragged grids.
"""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.load_library()


def _weights(shape, seed, kind):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if kind == "normal":
        w = torch.randn(shape, generator=g) * 0.02
    else:  # magnitudes from bf16 subnormals to 1e30, zero blocks
        w = torch.randn(shape, generator=g) * torch.exp2(torch.randint(-135, 100, shape[:-1] + (1,), generator=g).float())
        w.view(-1, shape[-1])[0, :48] = 0.0
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("shape,kind", [((3, 64, 256), "normal"), ((2, 40, 96), "wide"), ((1, 7, 32), "normal")])
def test_mxfp8_matches_oracle(shape, kind):
    w = _weights(shape, 0, kind).cuda()
    codes = torch.empty(shape, dtype=torch.uint8, device="cuda")
    scales = torch.empty(shape[:-1] + (shape[-1] // 32,), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8(w, codes, scales)
    torch.cuda.synchronize()
    oc, os_ = oracle.mxfp8_quantize(W.bf16_bits(w.cpu()).reshape(-1, shape[-1]))
    np.testing.assert_array_equal(scales.cpu().numpy().reshape(os_.shape), os_)
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(oc.shape), oc)


@pytest.mark.parametrize("shape,kind", [((3, 32, 128), "normal"), ((2, 24, 80), "wide"), ((5, 3, 16), "normal")])
def test_nvfp4_matches_oracle(shape, kind):
    w = _weights(shape, 1, kind).cuda()
    nmat, rows, K = shape
    codes = torch.empty((nmat, rows, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((nmat, rows, K // 16), dtype=torch.uint8, device="cuda")
    st = torch.empty(nmat, dtype=torch.float32, device="cuda")
    moe.moe_quantize_nvfp4(w, codes, scales, st)
    torch.cuda.synchronize()
    bits = W.bf16_bits(w.cpu())
    for m in range(nmat):
        oc, os_, ost = oracle.nvfp4_quantize(bits[m])
        assert st[m].item() == np.float32(ost)
        np.testing.assert_array_equal(scales[m].cpu().numpy(), os_)
        np.testing.assert_array_equal(codes[m].cpu().numpy(), oc)


def test_full_size_drafter_down_projection():
    """The 16-expert drafter's W_down (16 x 5120 x 1024): several grid strides.
    Experts 0 and 15 in full against the oracle, the matrix scales of all."""
    E, H, I = 16, 5120, 1024
    w = (torch.randn((E, H, I), device="cuda", generator=torch.Generator(device="cuda").manual_seed(3)) * 0.02
         ).to(torch.bfloat16)
    c8 = torch.empty((E, H, I), dtype=torch.uint8, device="cuda")
    s8 = torch.empty((E, H, I // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8(w, c8, s8)
    c4 = torch.empty((E, H, I // 2), dtype=torch.uint8, device="cuda")
    s4 = torch.empty((E, H, I // 16), dtype=torch.uint8, device="cuda")
    st = torch.empty(E, dtype=torch.float32, device="cuda")
    moe.moe_quantize_nvfp4(w, c4, s4, st)
    torch.cuda.synchronize()
    amax = w.float().abs().amax(dim=(1, 2)).cpu().numpy()
    np.testing.assert_array_equal(st.cpu().numpy(), (amax / np.float32(2688.0)).astype(np.float32))
    for e in (0, 15):
        bits = W.bf16_bits(w[e].cpu())
        oc, os_ = oracle.mxfp8_quantize(bits)
        np.testing.assert_array_equal(c8[e].cpu().numpy(), oc)
        np.testing.assert_array_equal(s8[e].cpu().numpy(), os_)
        oc, os_, ost = oracle.nvfp4_quantize(bits)
        assert st[e].item() == np.float32(ost)
        np.testing.assert_array_equal(c4[e].cpu().numpy(), oc)
        np.testing.assert_array_equal(s4[e].cpu().numpy(), os_)
