"""Expert-parallel host logic without a GPU: sharding every weight type by
expert, and EPLayer's argument checks.

The packed block-scale layout (include/moe.h, moe_mxfp8_pack_scales /
moe_nvfp4_pack_scales) is restated here from its definition --
[rows / 64][K / 128][64][b], b = 4 (MXFP8) or 8 (NVFP4) scales of a row per
128-wide K block -- and the test checks what shard_weights relies on:
packing a whole layer and slicing out one rank's experts gives the bytes of
packing that rank's experts alone."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200.ep import EPLayer, shard_weights


def pack_rows(scales: np.ndarray, per_block: int) -> np.ndarray:
    """[rows, K / block] scales -> the packed layout, flat."""
    rows, nb = scales.shape
    ks = nb // per_block  # 128-wide K blocks
    return scales.reshape(rows // 64, 64, ks, per_block).transpose(0, 2, 1, 3).reshape(-1)


@pytest.mark.parametrize("per_block", [4, 8])
@pytest.mark.parametrize("E,I,K,world", [(8, 128, 256, 2), (16, 192, 384, 4), (6, 64, 128, 3)])
def test_packing_then_slicing_by_expert_is_packing_the_slice(per_block, E, I, K, world):
    rng = np.random.default_rng(E * I + K + per_block)
    s = rng.integers(0, 255, size=(E * I, K // 128 * per_block), dtype=np.uint8)
    whole = pack_rows(s, per_block).reshape(E, I, -1)  # the [E, I, K / block] tensor the binding allocates
    epr = E // world
    for r in range(world):
        mine = s[r * epr * I:(r + 1) * epr * I]
        assert np.array_equal(whole[r * epr:(r + 1) * epr].reshape(-1), pack_rows(mine, per_block))


def _mxfp8(E, I, H, Is):
    u8 = lambda *shape: torch.zeros(shape, dtype=torch.uint8)
    return moe.MoEWeightsMXFP8(u8(E, I, H), u8(E, I, H), u8(E, H, I), u8(E, I, H // 32), u8(E, I, H // 32),
                               u8(E, H, I // 32), ws_gate=u8(Is, H), ws_up=u8(Is, H), ws_down=u8(H, Is),
                               ws_gate_scale=u8(Is, H // 32), ws_up_scale=u8(Is, H // 32),
                               ws_down_scale=u8(H, Is // 32), ws_gate_vec=torch.zeros(H, dtype=torch.bfloat16))


def _nvfp4(E, I, H, Is):
    u8 = lambda *shape: torch.zeros(shape, dtype=torch.uint8)
    ts = torch.arange(3 * E, dtype=torch.float32).reshape(3, E)
    return moe.MoEWeightsNVFP4(u8(E, I, H // 2), u8(E, I, H // 2), u8(E, H, I // 2), u8(E, I, H // 16),
                               u8(E, I, H // 16), u8(E, H, I // 16), ts[0], ts[1], ts[2], ws_gate=u8(Is, H // 2),
                               ws_up=u8(Is, H // 2), ws_down=u8(H, Is // 2), ws_gate_scale=u8(Is, H // 16),
                               ws_up_scale=u8(Is, H // 16), ws_down_scale=u8(H, Is // 16), ws_tscale=torch.ones(3),
                               ws_gate_vec=torch.zeros(H, dtype=torch.bfloat16))


@pytest.mark.parametrize("make", [_mxfp8, _nvfp4], ids=["mxfp8", "nvfp4"])
def test_shard_weights_block_scaled(make):
    E, I, H, Is, world = 8, 128, 256, 128, 4
    w = make(E, I, H, Is)
    for r in range(world):
        sh = shard_weights(w, world, r)
        assert type(sh) is type(w)
        for name in ("w_gate", "w_up", "w_down", "w_gate_scale", "w_up_scale", "w_down_scale"):
            whole, part = getattr(w, name), getattr(sh, name)
            assert part.shape[0] == E // world and part.is_contiguous()
            # a view at the rank's first expert, no copy
            assert part.data_ptr() == whole.data_ptr() + r * (E // world) * whole[0].numel() * whole.element_size()
        for name in ("ws_gate", "ws_up", "ws_down", "ws_gate_scale", "ws_up_scale", "ws_down_scale", "ws_gate_vec"):
            assert getattr(sh, name) is getattr(w, name)
        if isinstance(w, moe.MoEWeightsNVFP4):
            assert sh.w_up_tscale.tolist() == w.w_up_tscale[r * 2:(r + 1) * 2].tolist()
            assert sh.ws_tscale is w.ws_tscale


def test_ep_layer_argument_checks():
    cfg = moe.MoEConfig(256, 8, 128, 2, 128, True, 0, 0.0)
    w = _mxfp8(8, 128, 256, 128)
    EPLayer(cfg, 4, 0, shard_weights(w, 4, 0))  # 2 experts a rank, k = 2: accepted
    with pytest.raises(ValueError):
        EPLayer(moe.MoEConfig(256, 8, 128, 2, 128, True, 3, 0.0), 4, 0, shard_weights(w, 4, 0))  # a budget
    with pytest.raises(ValueError):
        EPLayer(cfg, 3, 0, shard_weights(w, 4, 0))  # 8 experts over 3 ranks
    with pytest.raises(ValueError):
        EPLayer(cfg, 2, 0, shard_weights(w, 4, 0))  # holds 2 experts, 4 expected
    with pytest.raises(ValueError):
        EPLayer(cfg, 8, 0, shard_weights(w, 8, 0))  # 1 expert a rank < k with a shared expert
    with pytest.raises(TypeError):
        EPLayer(cfg, 4, 0, object())
