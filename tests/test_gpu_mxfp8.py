"""GPU parity of the layer with MXFP8 expert weights (moe_forward_mxfp8).

The oracle's MXFP8 layer (oracle.forward_mxfp8) quantises every expert
matrix to MXFP8 along its reduction axis -- E4M3 codes, one power-of-two
scale per 32 weights -- dequantises it exactly and runs the bf16 layer
definition; the GPU gets the codes from its own quantiser
(moe_quantize_mxfp8, then moe_mxfp8_pack_scales) and turns each weight tile
back into bf16 in shared memory.  Checked here:
  * the scale repacking, bit for bit (an index permutation);
  * small layers against the oracle's MXFP8 layer on every row (routing and
    dispatch bit-exact, rel-L2 <= 5e-3, every row <= 1e-2), through the
    fused one-launch and the two-launch FFN, shared expert, budget, top-p;
  * the conversion is exact: moe_forward_mxfp8 writes the same output bits
    as moe_forward on the dequantised bf16 weights (the same MMAs on the
    same values), on weights whose blocks span E4M3 subnormals and scales
    above 2^7, and on the full-size drafter and 256-expert layers;
  * the full-size 16 x 1024 drafter and the 256-expert T = 64 layer against
    the oracle's MXFP8 layer on sampled rows.
"""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

import oracle
from parity_util import check_layer, gpu_forward, lib_config, sample_rows, weights_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability()[0] == 10, "needs an sm_100 (B200) device"
    moe.load_library()


def _quantise(w):
    """GPU quantiser: codes, unpacked scales, packed scales of one weight tensor."""
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.shape[:-1] + (w.shape[-1] // 32,), dtype=torch.uint8, device=w.device)
    moe.moe_quantize_mxfp8(w, codes, scales)
    packed = torch.empty_like(scales)
    moe.moe_mxfp8_pack_scales(scales, packed)
    return codes, scales, packed


def _mxfp8_weights(inp):
    """MoEWeightsMXFP8 from the GPU quantiser, and the torch dequantisation of
    the same codes (code value x 2^(scale - 127), exact in bf16) as MoEWeights."""
    q, deq = {}, {}
    for name in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        w = getattr(inp, name)
        if w is None:
            continue
        codes, scales, packed = _quantise(w)
        q[name], q[name + "_scale"] = codes, packed
        v = codes.view(torch.float8_e4m3fn).float() * torch.exp2(
            scales.float() - 127.0).repeat_interleave(32, dim=-1)
        deq[name] = v.to(torch.bfloat16)
        assert torch.equal(deq[name].float(), v), "dequantised weight not exact in bf16"
    wq = moe.MoEWeightsMXFP8(**q, ws_gate_vec=inp.ws_gvec, w_router=inp.w_router)
    wd = moe.MoEWeights(deq["w_gate"], deq["w_up"], deq["w_down"], deq.get("ws_gate"), deq.get("ws_up"),
                        deq.get("ws_down"), inp.ws_gvec, inp.w_router)
    return wq, wd


def test_pack_scales_layout():
    """[rows, K / 32] -> [rows / 64][K / 128][64][4], bit for bit."""
    g = torch.Generator(device="cpu").manual_seed(3)
    for rows, K in ((64, 128), (192, 640), (2048, 7168)):
        s = torch.randint(0, 255, (rows, K // 32), generator=g, dtype=torch.uint8)
        packed = torch.empty_like(s).cuda()
        moe.moe_mxfp8_pack_scales(s.cuda(), packed)
        want = s.numpy().reshape(rows // 64, 64, K // 128, 4).transpose(0, 2, 1, 3).reshape(-1)
        assert (packed.cpu().numpy().reshape(-1) == want).all()


SMALL = [
    W.MoEConfig("q_tiny", T=16, H=256, E=8, I=128, k=2),
    W.MoEConfig("q_shared", T=100, H=384, E=8, I=256, k=2, Is=128, zipf_alpha=1.0),
    W.MoEConfig("q_ragged", T=37, H=256, E=16, I=128, k=3, Is=256, zipf_alpha=1.0),
    W.MoEConfig("q_budget", T=32, H=256, E=32, I=128, k=4, budget=5, Is=128),
    W.MoEConfig("q_topp", T=64, H=256, E=48, I=128, k=6, topp=0.7),
    W.MoEConfig("q_no_norm", T=50, H=256, E=8, I=128, k=2, norm_topk=False, Is=128),
    W.MoEConfig("q_two_launch", T=600, H=256, E=4, I=128, k=2, Is=128, zipf_alpha=0.5),  # mean group >= 128
    W.MoEConfig("q_many_experts", T=64, H=128, E=256, I=128, k=8),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_mxfp8_small_layers(cfg):
    inp = W.make_inputs(cfg, device="cuda")
    wq, _ = _mxfp8_weights(inp)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_mxfp8)
    diag = check_layer(cfg, inp, g, wmap=oracle.mxfp8_weights)
    print(cfg.label, diag)


def test_mxfp8_layer_equals_oracle_forward_mxfp8():
    """The oracle's own MXFP8 layer function, all rows, routing included."""
    cfg = SMALL[1]
    inp = W.make_inputs(cfg, device="cuda")
    wq, _ = _mxfp8_weights(inp)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_mxfp8)
    b = W.bf16_bits
    ref = oracle.forward_mxfp8(b(inp.x), inp.logits.cpu().numpy(), b(inp.w_gate), b(inp.w_up), b(inp.w_down),
                               ws_gate=b(inp.ws_gate), ws_up=b(inp.ws_up), ws_down=b(inp.ws_down),
                               ws_gvec=b(inp.ws_gvec), k=cfg.k, nthreads=oracle.max_threads())
    assert (g.idx == ref.idx).all() and (g.perm == ref.perm).all()
    err = np.linalg.norm(g.out - ref.out) / np.linalg.norm(ref.out)
    assert err <= 5e-3, err


def _wide_range(inp, seed):
    """Weights whose 32-blocks hold values 2^-20 below their largest (E4M3
    subnormal codes and zeros) and one expert scaled by 2^20 (block scales
    above 2^7: the two-multiply conversion)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    for name in ("w_gate", "w_up", "w_down"):
        w = getattr(inp, name)
        f = torch.exp2(-torch.randint(0, 21, w.shape, generator=g, device="cuda").float())
        v = w.float() * f
        v[1] *= 2.0 ** 20
        w.copy_(v.to(torch.bfloat16))


@pytest.mark.parametrize("cfg,wide", [
    (W.MoEConfig("qb_small", T=100, H=384, E=8, I=256, k=2, Is=128), False),
    (W.MoEConfig("qb_wide", T=64, H=256, E=4, I=128, k=2, Is=128), True),
    (W.MoEConfig("qb_two_launch", T=600, H=256, E=4, I=128, k=2, Is=128), True),
], ids=["small", "wide_range", "two_launch_wide_range"])
def test_mxfp8_bits_equal_bf16_on_dequantised_weights(cfg, wide):
    inp = W.make_inputs(cfg, device="cuda")
    if wide:
        _wide_range(inp, 7)
    wq, wd = _mxfp8_weights(inp)
    if wide:  # the blocks do reach subnormal codes and the large scales
        codes, scales, _ = _quantise(inp.w_gate)
        assert ((codes & 0x78) == 0).logical_and((codes & 0x07) != 0).any()
        assert (scales > 134).any()
    a = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_mxfp8)
    b = gpu_forward(cfg, inp, weights=wd)
    assert a.status == 0 and b.status == 0
    assert (a.out_bits == b.out_bits).all()


@pytest.fixture(scope="module")
def large_q():
    """The 256-expert layer (T up to 512), its MXFP8 weights and their dequantisation."""
    cfg = W.LARGE_256E.with_(T=512)
    inp = W.make_inputs(cfg, device="cuda")
    wq, wd = _mxfp8_weights(inp)
    yield cfg, inp, wq, wd
    del inp, wq, wd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,alpha", [(64, 0.0), (512, 1.0)])
def test_mxfp8_large_bits_equal_bf16_on_dequantised_weights(large_q, T, alpha):
    base_cfg, base, wq, wd = large_q
    cfg = base_cfg.with_(T=T, zipf_alpha=alpha)
    logits = base.logits[:T] + W.zipf_bias(cfg.E, alpha, "cuda")
    inp = W.MoEInputs(base.x[:T].contiguous(), logits.contiguous(), base.w_gate, base.w_up, base.w_down)
    a = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_mxfp8)
    b = gpu_forward(cfg, inp, weights=wd)
    assert a.status == 0 and b.status == 0
    assert (a.out_bits == b.out_bits).all()


def test_mxfp8_large_T64_against_oracle(large_q):
    """256 experts, T = 64: the oracle's MXFP8 layer on one sampled token (8 experts)."""
    base_cfg, base, wq, _ = large_q
    cfg = base_cfg.with_(T=64)
    inp = W.MoEInputs(base.x[:64].contiguous(), base.logits[:64].contiguous(), base.w_gate, base.w_up, base.w_down)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_mxfp8)
    diag = check_layer(cfg, inp, g, rows=np.array([63], np.int32), wmap=oracle.mxfp8_weights)
    print(cfg.label, diag)


@pytest.mark.parametrize("cfg,nrows", [(W.DRAFTER_16x1024, 3), (W.DRAFTER_512x512, 2)],
                         ids=["drafter_16x1024", "drafter_512x512"])
def test_mxfp8_drafter_layers(cfg, nrows):
    """Full-size drafter layers: every output bit equal to the bf16 path on the
    dequantised weights, and sampled rows against the oracle's MXFP8 layer."""
    inp = W.make_inputs(cfg, device="cuda")
    wq, wd = _mxfp8_weights(inp)
    a = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_mxfp8)
    b = gpu_forward(cfg, inp, weights=wd)
    assert a.status == 0 and (a.out_bits == b.out_bits).all()
    diag = check_layer(cfg, inp, a, rows=sample_rows(cfg.T, nrows), wmap=oracle.mxfp8_weights)
    print(cfg.label, diag)
