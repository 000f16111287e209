"""The bounds-checked library (libmoe_checked.so, built with MOE_DEBUG_BOUNDS).

Its kernels range-check the index inputs a caller hands the stage entry
points -- expert ids given to moe_dispatch, the dispatch offsets and perm
entries given to moe_expert_ffn -- and report a bad one as
MOE_STATUS_BOUNDS in the status word, skipping the access (no trap).
Checked here: the small parity layers run through it with status 0 and the
release library's output bits; and each kind of bad index is reported while
every access stays in range (the checks run before the index is used).  The
bad-perm case runs on the checked library only: the release library trusts
perm, as its header says.
"""
import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

from parity_util import check_layer, gpu_forward, lib_config, weights_of

pytestmark = pytest.mark.gpu


@pytest.fixture
def checked(monkeypatch):
    """Route every binding call through the checked library for one test."""
    assert torch.cuda.is_available()
    lib = moe.load_library(variant="checked")
    release = moe.load_library()
    monkeypatch.setattr(moe, "_lib", lib)
    yield lib
    monkeypatch.setattr(moe, "_lib", release)


CASES = [
    W.MoEConfig("tiny", T=16, H=256, E=8, I=128, k=2),
    W.MoEConfig("ragged", T=37, H=256, E=16, I=64, k=3, Is=64, zipf_alpha=1.0),
    W.MoEConfig("budget", T=32, H=256, E=32, I=64, k=4, budget=3, zipf_alpha=1.2),
    W.MoEConfig("topp", T=64, H=256, E=48, I=64, k=6, Is=64, topp=0.7),
    W.MoEConfig("two_launch", T=600, H=512, E=8, I=256, k=2, Is=256),
    W.MoEConfig("separate_stages", T=1500, H=128, E=64, I=64, k=6, budget=9, topp=0.6, zipf_alpha=0.5),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_checked_library_same_bits_status_clean(cfg, checked):
    inp = W.make_inputs(cfg, device="cuda")
    g = gpu_forward(cfg, inp)
    assert g.status == 0
    check_layer(cfg, inp, g)
    torch.cuda.synchronize()
    moe._lib = moe.load_library()  # the release library on the same inputs
    r = gpu_forward(cfg, inp)
    assert (r.out_bits == g.out_bits).all()


def _dispatched(cfg, inp, ws):
    T, k, E = cfg.T, cfg.k, cfg.E
    c = lib_config(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    sgate = torch.empty(T, dtype=torch.float32, device="cuda") if cfg.Is else None
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    slot_pos = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((T * k, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_route(c, inp.logits, idx, w, x=inp.x if cfg.Is else None, ws_gate_vec=inp.ws_gvec, sgate=sgate)
    return c, idx, w, sgate, counts, offsets, perm, slot_pos, x_perm


@pytest.mark.parametrize("T", [40, 5000])  # the one-block sort (T*k <= 8192), and histogram + scan + scatter
def test_bad_expert_id_reported(T, checked):
    cfg = W.MoEConfig("bad_id", T=T, H=128, E=16, I=64, k=2)
    inp = W.make_inputs(cfg, device="cuda")
    ws = torch.zeros(moe.workspace_bytes(lib_config(cfg), T), dtype=torch.uint8, device="cuda")
    c, idx, w, sgate, counts, offsets, perm, slot_pos, x_perm = _dispatched(cfg, inp, ws)
    idx[3, 1] = cfg.E + 7  # out of range in a kept slot
    moe.moe_dispatch(c, idx, counts, offsets, perm, slot_pos, ws, x=inp.x, x_perm=x_perm)
    torch.cuda.synchronize()
    assert moe.status_read(ws) & moe.MOE_STATUS_BOUNDS
    assert int(counts.sum()) == T * cfg.k - 1 and int(slot_pos[3 * cfg.k + 1]) == -1


def test_bad_offsets_reported(checked):
    cfg = W.MoEConfig("bad_offsets", T=64, H=256, E=8, I=128, k=2, Is=64)
    inp = W.make_inputs(cfg, device="cuda")
    ws = torch.zeros(moe.workspace_bytes(lib_config(cfg), cfg.T), dtype=torch.uint8, device="cuda")
    c, idx, w, sgate, counts, offsets, perm, slot_pos, x_perm = _dispatched(cfg, inp, ws)
    moe.moe_dispatch(c, idx, counts, offsets, perm, slot_pos, ws, x=inp.x, x_perm=x_perm)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0
    bad = offsets.clone()
    bad[3], bad[4] = offsets[4] + 1000, offsets[3]  # not monotone, past T*k
    ybuf = torch.zeros((cfg.T, cfg.k + 1, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(c, inp.x, x_perm, bad, perm, w, weights_of(inp), ybuf, ws, sgate=sgate)
    torch.cuda.synchronize()
    assert moe.status_read(ws) & moe.MOE_STATUS_BOUNDS
    moe.status_clear(ws)
    moe.moe_expert_ffn(c, inp.x, x_perm, offsets, perm, w, weights_of(inp), ybuf, ws, sgate=sgate)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0


@pytest.mark.parametrize("launches", ["fused", "two"])
def test_bad_perm_reported(launches, checked):
    cfg = (W.MoEConfig("bad_perm", T=64, H=256, E=8, I=128, k=2, Is=64) if launches == "fused"
           else W.MoEConfig("bad_perm2", T=600, H=256, E=4, I=128, k=2, Is=64))
    inp = W.make_inputs(cfg, device="cuda")
    ws = torch.zeros(moe.workspace_bytes(lib_config(cfg), cfg.T), dtype=torch.uint8, device="cuda")
    c, idx, w, sgate, counts, offsets, perm, slot_pos, x_perm = _dispatched(cfg, inp, ws)
    moe.moe_dispatch(c, idx, counts, offsets, perm, slot_pos, ws, x=inp.x, x_perm=x_perm)
    bad = perm.clone()
    bad[5] = cfg.T * cfg.k + 123
    bad[9] = -4
    ybuf = torch.zeros((cfg.T, cfg.k + 1, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(c, inp.x, x_perm, offsets, bad, w, weights_of(inp), ybuf, ws, sgate=sgate)
    torch.cuda.synchronize()
    assert moe.status_read(ws) & moe.MOE_STATUS_BOUNDS
    # every other slot row was written as in a clean call
    ref = torch.zeros_like(ybuf)
    moe.status_clear(ws)
    moe.moe_expert_ffn(c, inp.x, x_perm, offsets, perm, w, weights_of(inp), ref, ws, sgate=sgate)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0
    p = perm.cpu().numpy().astype(np.int64)
    rows = np.delete(p, [5, 9])
    rows = torch.from_numpy(rows + rows // cfg.k).cuda()
    assert torch.equal(ybuf.view(-1, cfg.H)[rows].view(torch.int16), ref.view(-1, cfg.H)[rows].view(torch.int16))


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_nonfinite_logits_reported(bad, checked):
    """The checked library's moe_forward reports a NaN or infinite router logit
    (MOE_STATUS_NONFINITE) before routing; a clean call leaves the bit clear."""
    cfg = W.MoEConfig("bad_logit", T=24, H=256, E=8, I=128, k=2, Is=64)
    inp = W.make_inputs(cfg, device="cuda")
    g = gpu_forward(cfg, inp)
    assert g.status == 0
    logits = inp.logits.clone()
    logits[5, 3] = bad
    g = gpu_forward(cfg, W.MoEInputs(inp.x, logits, inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up,
                                     inp.ws_down, inp.ws_gvec))
    assert g.status & moe.MOE_STATUS_NONFINITE


def test_combine_clamps_keff():
    """moe_combine reads a token's own rows only: keff outside [0, k] counts as
    its nearest end (every build)."""
    cfg = W.MoEConfig("keff", T=8, H=256, E=8, I=128, k=3)
    c = lib_config(cfg)
    y = torch.randn((cfg.T, cfg.k + 1, cfg.H), device="cuda").to(torch.bfloat16)
    keff = torch.tensor([3, 9, -2, 0, 1, 2, 3, 100], dtype=torch.int32, device="cuda")
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(c, y, out, keff=keff)
    ref = torch.empty_like(out)
    moe.moe_combine(c, y, ref, keff=keff.clamp(0, cfg.k))
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
