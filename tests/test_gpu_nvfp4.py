"""GPU parity of the layer with NVFP4 expert weights (moe_forward_nvfp4).

The oracle's NVFP4 layer (oracle.forward_nvfp4) quantises every expert
matrix to NVFP4 along its reduction axis -- E2M1 codes, an E4M3 scale per 16
weights, an fp32 scale per matrix -- takes code x block scale (exact in
bf16) as the weights and multiplies each projection's output by the matrix
scale; the GPU gets the codes from its own quantiser (moe_quantize_nvfp4,
then moe_nvfp4_pack_scales), turns each weight tile back into bf16 in tensor
memory and applies the matrix scales in the epilogues.  Checked here:
  * the scale repacking, bit for bit (an index permutation);
  * small layers against the oracle's NVFP4 layer on every row (routing and
    dispatch bit-exact, rel-L2 <= 5e-3, every row <= 1e-2), through the
    fused one-launch and the two-launch FFN, shared expert, budget, top-p;
  * the conversion is exact: with every matrix scale set to 1 the layer
    writes the same output bits as moe_forward on the bf16 weights code x
    block scale (the same MMAs on the same values), also on weights whose
    block scales are E4M3 subnormals, and on the full-size layers;
  * the full-size 16 x 1024 drafter and the 256-expert T = 64 layer against
    the oracle's NVFP4 layer on sampled rows.
"""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

import oracle
from parity_util import check_layer, gpu_forward, sample_rows

pytestmark = pytest.mark.gpu

NAMES = ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")
E2M1 = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability()[0] == 10, "needs an sm_100 (B200) device"
    moe.load_library()


def _quantise(w):
    """GPU quantiser, one matrix scale per leading index: codes, unpacked and
    packed block scales, matrix scales."""
    w3 = w.reshape((-1,) + tuple(w.shape[-2:]))
    codes = torch.empty(w.shape[:-1] + (w.shape[-1] // 2,), dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.shape[:-1] + (w.shape[-1] // 16,), dtype=torch.uint8, device=w.device)
    ts = torch.empty(w3.shape[0], dtype=torch.float32, device=w.device)
    moe.moe_quantize_nvfp4(w3, codes, scales, ts)
    packed = torch.empty_like(scales)
    moe.moe_nvfp4_pack_scales(scales, packed)
    return codes, scales, packed, ts


def _dequantise(codes, scales):
    """code x block scale in torch (the E2M1 table, the E4M3 scale as
    float8_e4m3fn), exact in bf16."""
    lut = torch.tensor(E2M1, dtype=torch.float32, device=codes.device)
    nib = torch.stack([codes & 15, codes >> 4], dim=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,)).long()
    c = lut[nib & 7] * torch.where((nib & 8) != 0, -1.0, 1.0)
    v = c * scales.view(torch.float8_e4m3fn).float().repeat_interleave(16, dim=-1)
    b = v.to(torch.bfloat16)
    assert torch.equal(b.float(), v), "code x block scale not exact in bf16"
    return b


def _nvfp4_weights(inp, unit_scales=False):
    """MoEWeightsNVFP4 from the GPU quantiser, and code x block scale as
    MoEWeights (bf16).  unit_scales: every matrix scale replaced by 1, so that
    both describe the same layer."""
    q, deq = {}, {}
    for name in NAMES:
        w = getattr(inp, name)
        if w is None:
            continue
        codes, scales, packed, ts = _quantise(w)
        q[name], q[name + "_scale"] = codes, packed
        q[name + "_tscale"] = torch.ones_like(ts) if unit_scales else ts
        deq[name] = _dequantise(codes, scales)
    shared = {}
    if "ws_gate" in q:
        shared = dict(ws_gate=q["ws_gate"], ws_up=q["ws_up"], ws_down=q["ws_down"], ws_gate_scale=q["ws_gate_scale"],
                      ws_up_scale=q["ws_up_scale"], ws_down_scale=q["ws_down_scale"],
                      ws_tscale=torch.cat([q["ws_gate_tscale"], q["ws_up_tscale"], q["ws_down_tscale"]]))
    wq = moe.MoEWeightsNVFP4(q["w_gate"], q["w_up"], q["w_down"], q["w_gate_scale"], q["w_up_scale"],
                             q["w_down_scale"], q["w_gate_tscale"], q["w_up_tscale"], q["w_down_tscale"], **shared,
                             ws_gate_vec=inp.ws_gvec, w_router=inp.w_router)
    wd = moe.MoEWeights(deq["w_gate"], deq["w_up"], deq["w_down"], deq.get("ws_gate"), deq.get("ws_up"),
                        deq.get("ws_down"), inp.ws_gvec, inp.w_router)
    return wq, wd


def test_pack_scales_layout():
    """[rows, K / 16] -> [rows / 64][K / 128][64][8], bit for bit."""
    g = torch.Generator(device="cpu").manual_seed(5)
    for rows, K in ((64, 128), (192, 640), (2048, 7168)):
        s = torch.randint(0, 255, (rows, K // 16), generator=g, dtype=torch.uint8)
        packed = torch.empty_like(s).cuda()
        moe.moe_nvfp4_pack_scales(s.cuda(), packed)
        want = s.numpy().reshape(rows // 64, 64, K // 128, 8).transpose(0, 2, 1, 3).reshape(-1)
        assert (packed.cpu().numpy().reshape(-1) == want).all()


def test_quantiser_matches_oracle():
    """The GPU quantiser's codes, block scales and matrix scale equal the
    oracle's on the matrices these tests use (so both sides hold one layer)."""
    cfg = W.MoEConfig("q", T=16, H=256, E=2, I=128, k=2)
    inp = W.make_inputs(cfg, device="cuda")
    codes, scales, _, ts = _quantise(inp.w_gate)
    for e in range(cfg.E):
        c, s, t = oracle.nvfp4_quantize(W.bf16_bits(inp.w_gate[e]))
        assert (codes[e].cpu().numpy() == c).all() and (scales[e].cpu().numpy() == s).all()
        assert np.float32(t) == ts[e].cpu().numpy()


SMALL = [
    W.MoEConfig("n_tiny", T=16, H=256, E=8, I=128, k=2),
    W.MoEConfig("n_shared", T=100, H=384, E=8, I=256, k=2, Is=128, zipf_alpha=1.0),
    W.MoEConfig("n_ragged", T=37, H=256, E=16, I=128, k=3, Is=256, zipf_alpha=1.0),
    W.MoEConfig("n_budget", T=32, H=256, E=32, I=128, k=4, budget=5, Is=128),
    W.MoEConfig("n_topp", T=64, H=256, E=48, I=128, k=6, topp=0.7),
    W.MoEConfig("n_no_norm", T=50, H=256, E=8, I=128, k=2, norm_topk=False, Is=128),
    W.MoEConfig("n_two_launch", T=600, H=256, E=4, I=128, k=2, Is=128, zipf_alpha=0.5),  # mean group >= 128
    W.MoEConfig("n_many_experts", T=64, H=128, E=256, I=128, k=8),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_nvfp4_small_layers(cfg):
    inp = W.make_inputs(cfg, device="cuda")
    wq, _ = _nvfp4_weights(inp)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_nvfp4)
    diag = check_layer(cfg, inp, g, wmap=oracle.nvfp4_weights)
    print(cfg.label, diag)


def test_nvfp4_layer_equals_oracle_forward_nvfp4():
    """The oracle's own NVFP4 layer function, all rows, routing included."""
    cfg = SMALL[1]
    inp = W.make_inputs(cfg, device="cuda")
    wq, _ = _nvfp4_weights(inp)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_nvfp4)
    b = W.bf16_bits
    ref = oracle.forward_nvfp4(b(inp.x), inp.logits.cpu().numpy(), b(inp.w_gate), b(inp.w_up), b(inp.w_down),
                               ws_gate=b(inp.ws_gate), ws_up=b(inp.ws_up), ws_down=b(inp.ws_down),
                               ws_gvec=b(inp.ws_gvec), k=cfg.k, nthreads=oracle.max_threads())
    assert (g.idx == ref.idx).all() and (g.perm == ref.perm).all()
    err = np.linalg.norm(g.out - ref.out) / np.linalg.norm(ref.out)
    assert err <= 5e-3, err


def _wide_range(inp, seed):
    """Weights whose 16-blocks are scaled by 2^-0 .. 2^-24 (block scales down
    to E4M3 subnormals and zero blocks) and one expert scaled by 2^20 (a large
    matrix scale)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    for name in ("w_gate", "w_up", "w_down"):
        w = getattr(inp, name)
        blocks = w.shape[:-1] + (w.shape[-1] // 16,)
        f = torch.exp2(-torch.randint(0, 25, blocks, generator=g, device="cuda").float()).repeat_interleave(16, -1)
        v = w.float() * f
        v[1] *= 2.0 ** 20
        w.copy_(v.to(torch.bfloat16))


@pytest.mark.parametrize("cfg,wide", [
    (W.MoEConfig("nb_small", T=100, H=384, E=8, I=256, k=2, Is=128), False),
    (W.MoEConfig("nb_wide", T=64, H=256, E=4, I=128, k=2, Is=128), True),
    (W.MoEConfig("nb_two_launch", T=600, H=256, E=4, I=128, k=2, Is=128), True),
], ids=["small", "wide_range", "two_launch_wide_range"])
def test_nvfp4_bits_equal_bf16_on_dequantised_weights(cfg, wide):
    inp = W.make_inputs(cfg, device="cuda")
    if wide:
        _wide_range(inp, 9)
    wq, wd = _nvfp4_weights(inp, unit_scales=True)
    if wide:  # the blocks do reach subnormal scales
        _, scales, _, _ = _quantise(inp.w_gate)
        assert ((scales & 0x78) == 0).logical_and((scales & 0x07) != 0).any()
    a = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_nvfp4)
    b = gpu_forward(cfg, inp, weights=wd)
    assert a.status == 0 and b.status == 0
    assert (a.out_bits == b.out_bits).all()


def test_nvfp4_wide_range_against_oracle():
    cfg = W.MoEConfig("n_wide", T=64, H=256, E=4, I=128, k=2, Is=128)
    inp = W.make_inputs(cfg, device="cuda")
    _wide_range(inp, 11)
    wq, _ = _nvfp4_weights(inp)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_nvfp4)
    diag = check_layer(cfg, inp, g, wmap=oracle.nvfp4_weights)
    print(cfg.label, diag)


@pytest.fixture(scope="module")
def large_q():
    """The 256-expert layer (T up to 512), its NVFP4 weights (real and unit
    matrix scales) and code x block scale as bf16 weights."""
    cfg = W.LARGE_256E.with_(T=512)
    inp = W.make_inputs(cfg, device="cuda")
    wq, wd = _nvfp4_weights(inp)
    wq1 = moe.MoEWeightsNVFP4(**{**wq.__dict__, "w_gate_tscale": torch.ones_like(wq.w_gate_tscale),
                                 "w_up_tscale": torch.ones_like(wq.w_up_tscale),
                                 "w_down_tscale": torch.ones_like(wq.w_down_tscale)})
    yield cfg, inp, wq, wq1, wd
    del inp, wq, wq1, wd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,alpha", [(64, 0.0), (512, 1.0)])
def test_nvfp4_large_bits_equal_bf16_on_dequantised_weights(large_q, T, alpha):
    base_cfg, base, _, wq1, wd = large_q
    cfg = base_cfg.with_(T=T, zipf_alpha=alpha)
    logits = base.logits[:T] + W.zipf_bias(cfg.E, alpha, "cuda")
    inp = W.MoEInputs(base.x[:T].contiguous(), logits.contiguous(), base.w_gate, base.w_up, base.w_down)
    a = gpu_forward(cfg, inp, weights=wq1, fwd=moe.moe_forward_nvfp4)
    b = gpu_forward(cfg, inp, weights=wd)
    assert a.status == 0 and b.status == 0
    assert (a.out_bits == b.out_bits).all()


def test_nvfp4_large_T64_against_oracle(large_q):
    """256 experts, T = 64: the oracle's NVFP4 layer on one sampled token (8 experts)."""
    base_cfg, base, wq, _, _ = large_q
    cfg = base_cfg.with_(T=64)
    inp = W.MoEInputs(base.x[:64].contiguous(), base.logits[:64].contiguous(), base.w_gate, base.w_up, base.w_down)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_nvfp4)
    diag = check_layer(cfg, inp, g, rows=np.array([63], np.int32), wmap=oracle.nvfp4_weights)
    print(cfg.label, diag)


@pytest.mark.parametrize("cfg,nrows", [(W.DRAFTER_16x1024, 3), (W.DRAFTER_512x512, 2)],
                         ids=["drafter_16x1024", "drafter_512x512"])
def test_nvfp4_drafter_layers(cfg, nrows):
    """Full-size drafter layers: with unit matrix scales every output bit equal
    to the bf16 path on code x block scale; with the real ones, sampled rows
    against the oracle's NVFP4 layer."""
    inp = W.make_inputs(cfg, device="cuda")
    wq1, wd = _nvfp4_weights(inp, unit_scales=True)
    a = gpu_forward(cfg, inp, weights=wq1, fwd=moe.moe_forward_nvfp4)
    b = gpu_forward(cfg, inp, weights=wd)
    assert a.status == 0 and (a.out_bits == b.out_bits).all()
    del wq1, wd
    wq, _ = _nvfp4_weights(inp)
    g = gpu_forward(cfg, inp, weights=wq, fwd=moe.moe_forward_nvfp4)
    diag = check_layer(cfg, inp, g, rows=sample_rows(cfg.T, nrows), wmap=oracle.nvfp4_weights)
    print(cfg.label, diag)
