"""Expert parallelism (routed_expert_ffn_renorm_b200.ep) on one GPU: W ranks
emulated in one process, each with its share of the experts and of the
tokens, the two all-to-alls done as in-process copies (the ranks' kernels
run one after another; none waits on another rank).  Every output row must
equal moe_forward's on the whole layer, bit for bit: each row is computed
by the same kernels on the same operands in the same order."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W
from routed_expert_ffn_renorm_b200.ep import EPLayer, shard_weights

from parity_util import check_layer, gpu_forward, lib_config, weights_of

pytestmark = pytest.mark.gpu


def _blocks(counts):
    off = np.concatenate([[0], np.cumsum(counts)])
    return [slice(int(off[i]), int(off[i + 1])) for i in range(len(counts))]


def ep_emulated(cfg, inp, world, full=None):
    """The layer through EPLayer on `world` emulated ranks (weights `full`,
    default the bf16 ones); returns out [T, H]."""
    c = lib_config(cfg)
    full = weights_of(inp) if full is None else full
    layers = [EPLayer(c, world, r, shard_weights(full, world, r)) for r in range(world)]
    tok = np.array_split(np.arange(cfg.T), world)
    xs = [inp.x[t[0]:t[-1] + 1].contiguous() if len(t) else inp.x[:0] for t in tok]
    ls = [inp.logits[t[0]:t[-1] + 1].contiguous() if len(t) else inp.logits[:0] for t in tok]
    states, sends = zip(*[layers[r].dispatch(xs[r], ls[r]) for r in range(world)])
    # rank d receives block d of every source's send, sources in rank order
    recv = []
    for d in range(world):
        parts = [(sends[s].rows[_blocks(sends[s].counts)[d]], sends[s].local_idx[_blocks(sends[s].counts)[d]],
                  sends[s].local_w[_blocks(sends[s].counts)[d]]) for s in range(world)]
        recv.append(tuple(torch.cat([p[i] for p in parts]) for i in range(3)))
    done = [layers[d].experts(*recv[d]) for d in range(world)]
    outs = []
    for s in range(world):
        # in rank d's received order the rows of source s are block s of [counts of each source to d]
        back = torch.cat([done[d][_blocks([sends[q].counts[d] for q in range(world)])[s]] for d in range(world)])
        outs.append(layers[s].combine(states[s], back))
    torch.cuda.synchronize()
    return torch.cat(outs)


CASES = [
    (W.MoEConfig("ep_shared", T=64, H=256, E=8, I=128, k=2, Is=128), 2),
    (W.MoEConfig("ep_k_gt_w", T=100, H=256, E=16, I=64, k=4, Is=64, zipf_alpha=1.0), 2),
    (W.MoEConfig("ep_four", T=150, H=384, E=32, I=128, k=6, topp=0.7), 4),
    (W.MoEConfig("ep_eight", T=333, H=256, E=64, I=64, k=8, Is=128, zipf_alpha=1.5), 8),
    (W.MoEConfig("ep_no_norm", T=40, H=256, E=8, I=128, k=2, norm_topk=False), 4),
]


@pytest.mark.parametrize("cfg,world", CASES, ids=[c.name for c, _ in CASES])
def test_ep_equals_single_gpu_layer(cfg, world):
    inp = W.make_inputs(cfg, device="cuda")
    ref = gpu_forward(cfg, inp)
    out = ep_emulated(cfg, inp, world)
    assert (W.bf16_bits(out) == ref.out_bits).all(), "expert-parallel output differs from moe_forward"
    print(cfg.label, "world", world, check_layer(cfg, inp, ref))


CASES_Q = [
    (W.MoEConfig("ep_q_shared", T=64, H=256, E=8, I=128, k=2, Is=128, zipf_alpha=1.0), 2),
    (W.MoEConfig("ep_q_four", T=100, H=384, E=16, I=256, k=4), 4),
]


@pytest.mark.parametrize("fmt", ["mxfp8", "nvfp4"])
@pytest.mark.parametrize("cfg,world", CASES_Q, ids=[c.name for c, _ in CASES_Q])
def test_ep_block_scaled_equals_single_gpu_layer(cfg, world, fmt):
    """Block-scaled expert weights, sharded by expert (codes, packed scales,
    matrix scales): bit for bit the single-GPU block-scaled layer."""
    inp = W.make_inputs(cfg, device="cuda")
    pack = moe.pack_mxfp8 if fmt == "mxfp8" else moe.pack_nvfp4
    fwd = moe.moe_forward_mxfp8 if fmt == "mxfp8" else moe.moe_forward_nvfp4
    wq = pack(weights_of(inp))
    ref = gpu_forward(cfg, inp, weights=wq, fwd=fwd)
    out = ep_emulated(cfg, inp, world, full=wq)
    assert ref.status == 0
    assert (W.bf16_bits(out) == ref.out_bits).all(), "expert-parallel output differs from the single-GPU layer"


def test_ep_rejects_budget():
    cfg = W.MoEConfig("ep_budget", T=16, H=256, E=8, I=128, k=2, budget=3)
    inp = W.make_inputs(cfg, device="cuda")
    with pytest.raises(ValueError):
        EPLayer(lib_config(cfg), 2, 0, shard_weights(weights_of(inp), 2, 0))
