"""moe_expert_ffn_noalloc: the expert FFN for callers that cannot allocate
device memory (a plugin that only receives its input and output buffers, a
serving loop that must not allocate once running).  Its scratch lives in a
fixed device array inside the library instead of a caller workspace.

Checked here through the C ABI against moe_expert_ffn (the workspace
version) on the same dispatched batch, bit for bit (the same kernel on the
same inputs), for two calls in a row -- the second with a different batch,
so it runs on the scratch the first one left behind -- through the fused
one-launch FFN, the two-launch FFN and the two-launch FFN of CTA pairs.
This file is collected last so that a failure here leaves every other test
already run; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

from parity_util import lib_config, rel_l2, weights_of

pytestmark = pytest.mark.gpu


def _dispatched(cfg, seed):
    """Route and dispatch one seeded batch; returns what the FFN needs."""
    dev = "cuda"
    c = lib_config(cfg)
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    inp = W.make_inputs(cfg, device=dev, seed=seed)
    ws = torch.zeros(moe.workspace_bytes(c, T), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    sgate = torch.empty(T, dtype=torch.float32, device=dev) if cfg.Is else None
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    moe.moe_route(c, inp.logits, idx, w, x=inp.x if cfg.Is else None, ws_gate_vec=inp.ws_gvec, sgate=sgate)
    moe.moe_dispatch(c, idx, counts, offsets, perm, slot_pos, ws, x=inp.x, x_perm=x_perm)
    return c, inp, ws, w, sgate, offsets, perm, x_perm


def _kept_rows(cfg, perm):
    """ybuf rows the FFN writes: slot rows t*(k+1)+j of kept slots, plus the shared rows."""
    k = cfg.k
    slots = perm.cpu().numpy().astype(np.int64)
    rows = slots + slots // k
    if cfg.Is:
        rows = np.concatenate([rows, np.arange(cfg.T) * (k + 1) + k])
    return torch.from_numpy(np.sort(rows))


# The fused one-launch FFN (mean group < 128 tokens), the two-launch FFN
# (gate/up, then down, on the array's separate counters), and the two-launch
# FFN of CTA pairs (every weight-tile count even) -- all within the 8 MiB of
# activations the array holds.
NOALLOC_CASES = [
    W.DRAFTER_16x1024,
    W.MoEConfig("ragged", T=37, H=256, E=16, I=64, k=3, Is=64),
    W.MoEConfig("two_launch", T=512, H=256, E=8, I=128, k=2, Is=64),
    W.MoEConfig("two_launch_pair", T=512, H=256, E=8, I=128, k=2, Is=128),
]


@pytest.mark.parametrize("cfg", NOALLOC_CASES, ids=lambda c: c.name)
def test_noalloc_matches_workspace_version_twice(cfg):
    """Same kernel, same inputs: the no-alloc call writes the same ybuf bits as
    moe_expert_ffn, on two calls in a row with different batches."""
    assert torch.cuda.is_available()
    for call, seed in enumerate((11, 12)):  # two calls in a row, different batches
        c, inp, ws, w, sgate, offsets, perm, x_perm = _dispatched(cfg, seed)
        wts = weights_of(inp)
        shape = (cfg.T, cfg.k + 1, cfg.H)
        y_ws = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        y_na = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        moe.moe_expert_ffn(c, inp.x, x_perm, offsets, perm, w, wts, y_ws, ws, sgate=sgate)
        moe.moe_expert_ffn_noalloc(c, inp.x, x_perm, offsets, perm, w, wts, y_na, sgate=sgate,
                                   device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "device status of the no-alloc call"
        assert moe.status_read(ws) == 0
        rows = _kept_rows(cfg, perm[: int(offsets[cfg.E].item())]).cuda()
        a = y_na.view(-1, cfg.H)[rows]
        b = y_ws.view(-1, cfg.H)[rows]
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), \
            f"call {call}: rel-L2 {rel_l2(a.float().cpu().numpy(), b.float().cpu().numpy()):.3e}"
        assert torch.isfinite(a.float()).all() and a.float().abs().sum() > 0


def test_noalloc_rejects_batches_beyond_its_scratch():
    # 2 * T*k*I bytes of h rows must fit in 8 MiB: T=4096, k=8, I=2048 needs 128 MiB
    cfg = W.MoEConfig("big", T=4096, H=256, E=16, I=2048, k=8)
    c = lib_config(cfg)
    dev = "cuda"
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    dummy = torch.zeros(16, dtype=torch.bfloat16, device=dev)
    wts = moe.MoEWeights(dummy, dummy, dummy)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_expert_ffn_noalloc(c, torch.zeros((T, H), dtype=torch.bfloat16, device=dev),
                                   torch.zeros((T * k, 8), dtype=torch.bfloat16, device=dev),
                                   torch.zeros(E + 1, dtype=torch.int32, device=dev),
                                   torch.zeros(T * k, dtype=torch.int32, device=dev),
                                   torch.zeros((T, k), dtype=torch.float32, device=dev), wts,
                                   torch.zeros(8, dtype=torch.bfloat16, device=dev))
    assert ei.value.code == -3
