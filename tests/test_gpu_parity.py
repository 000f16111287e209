"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Bit-exact for routing indices, budget drops, counts, offsets, perm and
slot_pos; fp32-ulp close for routing weights and the shared gate; relative
L2 <= 5e-3 on the bf16 layer output (and <= 1e-2 on every compared row).
Small shapes compare every output row and span several weight tiles, several
token tiles and ragged tails; the full-size workloads compare a stratified
set of rows -- one from every (expert group, 256-row token tile), the first
and last row of every group, one from every shared-expert tile, and seeded
extra tokens -- so every work item of both GEMM phases is reached (routing
and dispatch always in full).
"""
import os

import numpy as np
import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

import oracle
from parity_util import check_layer, gpu_forward, lib_config, logits_bound, sample_rows, stratified_rows, weights_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability()[0] == 10, "needs an sm_100 (B200) device"
    moe.load_library()


def _run(cfg, device="cuda", gen_device="cpu", rows=None, **mk):
    inp = W.make_inputs(cfg, device=gen_device, **mk)
    if gen_device != device:
        inp = W.MoEInputs(*(t.to(device) if t is not None else None for t in (
            inp.x, inp.logits, inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up, inp.ws_down,
            inp.ws_gvec)))
    g = gpu_forward(cfg, inp)
    return check_layer(cfg, inp, g, rows=rows), g, inp


SMALL = [
    W.TINY,
    W.MoEConfig("multi_tile", T=1000, H=384, E=4, I=192, k=2, Is=128),
    W.MoEConfig("ragged", T=37, H=256, E=16, I=64, k=3, Is=64, zipf_alpha=1.0),
    W.MoEConfig("k_eq_E", T=20, H=128, E=4, I=64, k=4),
    W.MoEConfig("one_expert", T=33, H=128, E=1, I=64, k=1),
    W.MoEConfig("single_token", T=1, H=256, E=8, I=128, k=2, Is=64),
    W.MoEConfig("no_norm", T=50, H=256, E=8, I=128, k=2, norm_topk=False, Is=64),
    W.MoEConfig("budget_small", T=32, H=256, E=32, I=64, k=4, budget=3, zipf_alpha=1.2),
    W.MoEConfig("budget_one", T=32, H=256, E=32, I=64, k=4, budget=1),
    W.MoEConfig("budget_no_norm", T=40, H=256, E=32, I=64, k=4, budget=5, norm_topk=False, Is=64),
    W.MoEConfig("budget_chunks", T=700, H=128, E=64, I=64, k=6, budget=9, zipf_alpha=0.5),
    W.MoEConfig("max_experts", T=64, H=128, E=1024, I=64, k=8),
    W.MoEConfig("max_topk", T=16, H=128, E=64, I=64, k=32),
    # per-token top-p trim: lane router (32 < E <= 64), warp router, 16-byte lane loads (E > 128), no norm,
    # with the budget (fused front end, one-block and chunked budgets)
    W.MoEConfig("topp_lane", T=64, H=256, E=48, I=64, k=6, Is=64, topp=0.7),
    W.MoEConfig("topp_warp", T=50, H=256, E=128, I=64, k=8, topp=0.5, zipf_alpha=0.5),
    W.MoEConfig("topp_vec", T=40, H=128, E=256, I=64, k=8, topp=0.85),
    W.MoEConfig("topp_no_norm", T=48, H=256, E=16, I=64, k=4, norm_topk=False, topp=0.3),
    W.MoEConfig("topp_budget", T=32, H=256, E=128, I=64, k=8, budget=12, topp=0.8, zipf_alpha=1.2),
    W.MoEConfig("topp_budget_block", T=700, H=128, E=64, I=64, k=6, budget=9, topp=0.6, zipf_alpha=0.5),
    W.MoEConfig("topp_budget_chunks", T=1500, H=128, E=64, I=64, k=6, budget=9, topp=0.6, zipf_alpha=0.5),
    W.MoEConfig("topp_tiny_p", T=33, H=128, E=16, I=64, k=4, Is=64, topp=1e-6),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_layers(cfg):
    diag, g, _ = _run(cfg)
    print(cfg.label, diag)


# Enough down items (>= 8 per SM) that small groups take two weight tiles per
# down item; H = 1920 gives an odd number of 128-row output tiles (a last
# item with one tile), and T = 96 lets the shared expert's down items pair up.
MERGED = [
    W.MoEConfig("merged_odd_tiles", T=256, H=1920, E=128, I=128, k=4, Is=128, zipf_alpha=0.5),
    W.MoEConfig("merged_shared", T=96, H=1920, E=128, I=128, k=4, Is=128),
]


@pytest.mark.parametrize("cfg", MERGED, ids=lambda c: c.name)
def test_merged_down_items(cfg):
    diag, g, _ = _run(cfg)
    print(cfg.label, diag)


@pytest.mark.parametrize("bn", [32, 64])
def test_merged_down_items_bits(bn, monkeypatch):
    """Narrower token tiles pair fewer groups (only those of <= BN/2 tokens); the
    output bits do not move."""
    cfg = MERGED[0]
    inp = W.make_inputs(cfg, device="cuda")
    ref = gpu_forward(cfg, inp)
    monkeypatch.setenv("MOE_FORCE_BN", str(bn))
    got = gpu_forward(cfg, inp)
    assert (got.out_bits == ref.out_bits).all()


# CTA pairs (cta_group::2): layers whose mean group has >= 128 tokens run the
# FFN as two launches of CTA pairs; every weight-tile count here is even.
PAIRED = [
    W.MoEConfig("pair_shared", T=600, H=512, E=8, I=256, k=2, Is=256),
    W.MoEConfig("pair_ragged", T=333, H=256, E=4, I=128, k=3, Is=128, zipf_alpha=1.0),
]


@pytest.mark.parametrize("cfg", PAIRED, ids=lambda c: c.name)
def test_cta_pair_layers(cfg):
    diag, g, _ = _run(cfg)
    print(cfg.label, diag)


@pytest.mark.parametrize("cfg", PAIRED, ids=lambda c: c.name)
def test_cta_pair_bits_equal_single_cta(cfg, monkeypatch):
    """The pair's M = 256 MMAs accumulate every output element in the same K
    order as the single-CTA path: identical bits."""
    inp = W.make_inputs(cfg, device="cuda")
    monkeypatch.setenv("MOE_FORCE_PAIR", "1")
    a = gpu_forward(cfg, inp)
    monkeypatch.setenv("MOE_FORCE_PAIR", "0")
    b = gpu_forward(cfg, inp)
    assert a.status == 0 and b.status == 0
    assert (a.out_bits == b.out_bits).all()


def test_force_pair_rejects_bad_values(monkeypatch):
    cfg = PAIRED[0]
    inp = W.make_inputs(cfg, device="cuda")
    monkeypatch.setenv("MOE_FORCE_PAIR", "2")
    with pytest.raises(moe.MoEError):
        gpu_forward(cfg, inp)


def test_hot_expert_multi_tile():
    """Every token routes to expert 3 first: one group of T rows, several token tiles."""
    cfg = W.MoEConfig("hot", T=600, H=256, E=8, I=128, k=2, Is=64)
    inp = W.make_inputs(cfg)
    inp.logits[:, 3] += 50.0
    inp = W.MoEInputs(*(t.cuda() if t is not None else None for t in (
        inp.x, inp.logits, inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up, inp.ws_down, inp.ws_gvec)))
    g = gpu_forward(cfg, inp)
    assert g.counts[3] == cfg.T
    print(check_layer(cfg, inp, g))


def test_sgate_varies():
    """A gate vector of scale 1 makes sigmoid(g.x) spread over (0, 1)."""
    cfg = W.MoEConfig("gate", T=64, H=512, E=8, I=64, k=2, Is=128)
    diag, g, _ = _run(cfg, std=0.5, gate_std=1.0)
    assert g.sgate.min() < 0.2 and g.sgate.max() > 0.8


def test_empty_tokens_after_budget_are_zero():
    cfg = W.MoEConfig("empty", T=32, H=256, E=128, I=64, k=8, budget=4)
    diag, g, _ = _run(cfg)
    assert (g.keff == 0).any()


def test_deterministic_bits():
    cfg = W.MoEConfig("det", T=500, H=256, E=16, I=128, k=4, Is=64, budget=10, zipf_alpha=1.0)
    inp = W.make_inputs(cfg, device="cuda")
    a = gpu_forward(cfg, inp)
    b = gpu_forward(cfg, inp)
    assert (a.out_bits == b.out_bits).all() and (a.perm == b.perm).all() and (a.w == b.w).all()


@pytest.mark.parametrize("bn,bns", [(32, None), (64, None), (128, None), (256, None), (256, 32), (256, 128),
                                    (128, 64)])
def test_tile_config_invariance(bn, bns, monkeypatch):
    """Forced token-tile sizes (routed / shared) give bit-identical outputs
    (tiling never changes a K-reduction)."""
    cfg = W.MoEConfig("inv", T=700, H=256, E=8, I=128, k=2, Is=64, zipf_alpha=1.5)
    inp = W.make_inputs(cfg, device="cuda")
    ref = gpu_forward(cfg, inp)
    monkeypatch.setenv("MOE_FORCE_BN", str(bn))
    if bns is not None:
        monkeypatch.setenv("MOE_FORCE_BNS", str(bns))
    got = gpu_forward(cfg, inp)
    assert (got.out_bits == ref.out_bits).all()


@pytest.mark.parametrize("pages", [24, 25, 33, 57])
def test_ring_size_invariance(pages, monkeypatch):
    """Small shared-memory rings (24 pages hold one 256-token K step) force
    wrap-around skips and retire waits at every step; the output bits stay put."""
    cfg = W.MoEConfig("ring", T=300, H=512, E=8, I=128, k=2, Is=128, zipf_alpha=1.2)
    inp = W.make_inputs(cfg, device="cuda")
    ref = gpu_forward(cfg, inp)
    monkeypatch.setenv("MOE_FORCE_PAGES", str(pages))
    got = gpu_forward(cfg, inp)
    assert (got.out_bits == ref.out_bits).all()


@pytest.mark.parametrize("env", [{"MOE_FORCE_BN": "48"}, {"MOE_FORCE_BNS": "512"}, {"MOE_FORCE_PAGES": "23"},
                                 {"MOE_FORCE_PAGES": "x"}, {"MOE_FORCE_BN": "64", "MOE_FORCE_BNS": "128"}])
def test_force_overrides_reject_bad_values(env, monkeypatch):
    cfg = W.TINY
    inp = W.make_inputs(cfg, device="cuda")
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    with pytest.raises(moe.MoEError):
        gpu_forward(cfg, inp)


# moe_forward takes the fused front-end launch when a budget is set, T*k <= 8192
# and T*E <= 16384, the separate route / budget / dispatch launches otherwise;
# both must match the stage entry points bit for bit.
STAGEWISE = [
    W.MoEConfig("stages", T=96, H=256, E=16, I=128, k=4, Is=64, budget=6, zipf_alpha=1.0),  # front
    W.MoEConfig("stages_nobudget", T=200, H=256, E=32, I=64, k=3, Is=64),  # separate
    W.MoEConfig("stages_budget_idle", T=40, H=128, E=16, I=64, k=2, budget=16),  # front, union <= N
    W.MoEConfig("stages_no_norm", T=64, H=128, E=64, I=64, k=6, budget=5, norm_topk=False, zipf_alpha=0.8),  # front
    W.MoEConfig("stages_e1024", T=16, H=128, E=1024, I=64, k=8, budget=20),  # front, largest E
    W.MoEConfig("stages_slots_max", T=1024, H=128, E=16, I=64, k=8, Is=64, budget=9),  # front, T*k = 8192
    W.MoEConfig("stages_big_logits", T=700, H=128, E=64, I=64, k=6, budget=9, zipf_alpha=0.5),  # separate
    W.MoEConfig("stages_topp", T=96, H=256, E=16, I=128, k=4, Is=64, budget=6, topp=0.6, zipf_alpha=1.0),  # front
    W.MoEConfig("stages_topp_warp", T=64, H=128, E=128, I=64, k=8, budget=12, topp=0.8),  # front, warp router
    W.MoEConfig("stages_topp_nobudget", T=200, H=256, E=32, I=64, k=3, Is=64, topp=0.5),  # separate
    W.MoEConfig("stages_topp_chunks", T=1500, H=128, E=64, I=64, k=6, budget=9, topp=0.7),  # separate, chunked
]


@pytest.mark.parametrize("cfg", STAGEWISE, ids=lambda c: c.name)
def test_stagewise_entry_points(cfg):
    """route -> budget -> dispatch -> expert_ffn -> combine called one by one
    equals moe_forward bit for bit, every auxiliary output included."""
    inp = W.make_inputs(cfg, device="cuda")
    ref = gpu_forward(cfg, inp)
    c = lib_config(cfg)
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    dev = "cuda"
    ws = torch.zeros(moe.workspace_bytes(c, T), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    sgate = torch.empty(T, dtype=torch.float32, device=dev) if cfg.Is else None
    keff = torch.empty(T, dtype=torch.int32, device=dev)
    kept = torch.zeros(E, dtype=torch.uint8, device=dev)
    nd = torch.zeros(1, dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    ybuf = torch.empty((T, k + 1, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    moe.moe_route(c, inp.logits, idx, w, x=inp.x if cfg.Is else None, ws_gate_vec=inp.ws_gvec if cfg.Is else None,
                  sgate=sgate, keff=keff)
    if cfg.budget:
        moe.moe_budget(c, idx, w, keff, kept, nd, ws)
    moe.moe_dispatch(c, idx, counts, offsets, perm, slot_pos, ws, keff=keff, x=inp.x, x_perm=x_perm)
    moe.moe_expert_ffn(c, inp.x, x_perm, offsets, perm, w, weights_of(inp), ybuf, ws, sgate=sgate)
    moe.moe_combine(c, ybuf, out, keff=keff)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0
    assert (idx.cpu().numpy() == ref.idx).all()
    assert (w.cpu().numpy().view(np.uint32) == ref.w.view(np.uint32)).all()
    assert (keff.cpu().numpy() == ref.keff).all()
    if cfg.budget:
        assert (kept.cpu().numpy() == ref.kept).all() and int(nd.item()) == ref.n_dropped
    if cfg.Is:
        assert (sgate.cpu().numpy().view(np.uint32) == ref.sgate.view(np.uint32)).all()
    assert (counts.cpu().numpy() == ref.counts).all() and (offsets.cpu().numpy() == ref.offsets).all()
    total = int(offsets[E])
    assert (perm[:total].cpu().numpy() == ref.perm).all()
    assert (slot_pos.cpu().numpy() == ref.slot_pos).all()
    assert (W.bf16_bits(out) == ref.out_bits).all()
    # x_perm rows are exact copies of the routed tokens
    xp = x_perm[:total].cpu()
    src = inp.x.cpu()[perm[:total].cpu().long() // k]
    assert torch.equal(xp, src)


# ------------------------------------------------------ router projection --
PROJ = [
    W.MoEConfig("proj_tiny", T=16, H=256, E=8, I=128, k=2),                 # one split, one tile
    W.MoEConfig("proj_split", T=40, H=1024, E=24, I=64, k=4, Is=64),        # K split over CTAs
    W.MoEConfig("proj_wide", T=300, H=512, E=200, I=64, k=6, topp=0.8),     # 3 x 2 tiles, ragged E, split
    W.MoEConfig("proj_many_tiles", T=2000, H=256, E=64, I=64, k=2),         # 16 tiles, no split
    W.MoEConfig("proj_e1000", T=7, H=384, E=1000, I=64, k=8, budget=30),    # 8 expert tiles, budget front end
    W.MoEConfig("proj_drafter", T=224, H=5120, E=16, I=1024, k=2, Is=2048),  # the drafter layer's shape
]


@pytest.mark.parametrize("cfg", PROJ, ids=lambda c: c.name)
def test_router_projection(cfg):
    """moe_router_logits against the oracle's fp64 projection (fp32 error
    bound per logit), the same bits twice, and moe_forward without logits
    equal, bit for bit, to moe_forward on those logits; the layer then
    matches the oracle run on the GPU's logits."""
    inp = W.make_inputs(cfg, device="cuda", router=True)
    c = lib_config(cfg)
    ws = torch.zeros(moe.workspace_bytes(c, cfg.T), dtype=torch.uint8, device="cuda")
    lg = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device="cuda")
    moe.moe_router_logits(c, inp.x, inp.w_router, lg, ws)
    lg2 = torch.full_like(lg, float("nan"))
    moe.moe_router_logits(c, inp.x, inp.w_router, lg2, ws)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0
    g = lg.cpu().numpy()
    assert (g.view(np.uint32) == lg2.cpu().numpy().view(np.uint32)).all(), "projection not deterministic"
    xb, wb = W.bf16_bits(inp.x), W.bf16_bits(inp.w_router)
    ref = oracle.router_logits(xb, wb)
    assert (np.abs(g.astype(np.float64) - ref) <= logits_bound(xb, wb)).all(), \
        f"max logit error {np.abs(g - ref).max():.3e}"
    # the layer with the projection inside moe_forward
    inp_l = W.MoEInputs(inp.x, lg, inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up, inp.ws_down,
                        inp.ws_gvec)
    ref_run = gpu_forward(cfg, inp_l)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    aux_lg = torch.full_like(lg, float("nan"))
    ws2 = torch.zeros(moe.workspace_bytes(c, cfg.T), dtype=torch.uint8, device="cuda")
    moe.moe_forward(c, inp.x, None, weights_of(inp), out, ws2, aux={"logits": aux_lg})
    torch.cuda.synchronize()
    assert moe.status_read(ws2) == 0
    assert (aux_lg.cpu().numpy().view(np.uint32) == g.view(np.uint32)).all()
    assert (W.bf16_bits(out) == ref_run.out_bits).all()
    check_layer(cfg, inp_l, ref_run, rows=sample_rows(cfg.T, 48))


def test_forward_without_logits_needs_router_weights():
    cfg = W.MoEConfig("noproj", T=8, H=256, E=8, I=128, k=2)
    inp = W.make_inputs(cfg, device="cuda")
    c = lib_config(cfg)
    ws = torch.zeros(moe.workspace_bytes(c, cfg.T), dtype=torch.uint8, device="cuda")
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError):
        moe.moe_forward(c, inp.x, None, weights_of(inp), out, ws)


def test_budget_is_exact_sequential_sum():
    """Up to 8192 slots the budget sums each expert's weights in exactly token-then-slot
    order, so the kept set equals the oracle's with no near-tie allowance."""
    import oracle
    for cfg in (W.MoEConfig("bex", T=700, H=128, E=64, I=64, k=6, budget=9, zipf_alpha=0.5),
                W.MoEConfig("bex2", T=1000, H=128, E=128, I=64, k=8, budget=40, zipf_alpha=0.3)):
        inp = W.make_inputs(cfg, device="cuda")
        g = gpu_forward(cfg, inp)
        idx_o, w_o = oracle.route(inp.logits.cpu().numpy(), cfg.k, cfg.norm_topk)
        idx_b, w_b, keff_b, kept_b, nd_b = oracle.budget(idx_o, w_o, cfg.E, cfg.budget, cfg.norm_topk)
        assert (g.kept == kept_b).all() and g.n_dropped == nd_b
        assert (g.idx == idx_b).all() and (g.keff == keff_b).all()


def test_zero_tokens_is_noop():
    c = lib_config(W.TINY)
    dev = "cuda"
    ws = torch.zeros(moe.workspace_bytes(c, 1), dtype=torch.uint8, device=dev)
    x = torch.empty((0, W.TINY.H), dtype=torch.bfloat16, device=dev)
    inp = W.make_inputs(W.TINY, device=dev)
    moe.moe_forward(c, x, torch.empty((0, W.TINY.E), device=dev), weights_of(inp),
                    torch.empty((0, W.TINY.H), dtype=torch.bfloat16, device=dev), ws)
    torch.cuda.synchronize()


# ------------------------------------------------------------ full sizes --

def _strat(cfg, n_random):
    """Row chooser for check_layer: every (group, token tile), group ends, shared tiles."""
    return lambda offsets, perm: stratified_rows(cfg.T, cfg.k, offsets, perm, tile=256, n_random=n_random,
                                                 shared_tile=128 if cfg.Is else 0)


DRAFTERS = [W.DRAFTER_16x1024, W.DRAFTER_512x512, W.DRAFTER_512x512.with_(zipf_alpha=0.0),
            W.DRAFTER_512x512.with_(topp=0.8)]


@pytest.mark.parametrize("cfg", DRAFTERS, ids=["drafter_16x1024", "drafter_512x512_a1", "drafter_512x512_a0",
                                               "drafter_512x512_a1_topp0.8"])
def test_drafter_layers(cfg):
    diag, g, _ = _run(cfg, gen_device="cuda", rows=_strat(cfg, 32))
    print(cfg.label, diag)


def test_drafter_layer_router_projection():
    """The 512 x 512 drafter layer with its logits from the router projection
    inside moe_forward: the projection's logits within the fp32 bound of the
    oracle's, then the whole layer on those logits."""
    cfg = W.DRAFTER_512x512.with_(router_proj=True)
    inp = W.make_inputs(cfg, device="cuda")
    c = lib_config(cfg)
    ws = torch.zeros(moe.workspace_bytes(c, cfg.T), dtype=torch.uint8, device="cuda")
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    lg = torch.full((cfg.T, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_forward(c, inp.x, None, weights_of(inp), out, ws, aux={"logits": lg})
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0
    xb, wb = W.bf16_bits(inp.x), W.bf16_bits(inp.w_router)
    g_lg = lg.cpu().numpy()
    assert (np.abs(g_lg.astype(np.float64) - oracle.router_logits(xb, wb)) <= logits_bound(xb, wb)).all()
    inp_l = W.MoEInputs(inp.x, lg, inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up, inp.ws_down,
                        inp.ws_gvec)
    g = gpu_forward(cfg.with_(router_proj=False), inp_l)
    assert (g.out_bits == W.bf16_bits(out)).all(), "moe_forward with the projection differs from given logits"
    diag = check_layer(cfg, inp_l, g, rows=_strat(cfg, 32))
    print(cfg.label, diag, "touched", int((g.counts > 0).sum()))


@pytest.mark.parametrize("N", W.BUDGETS)
def test_budget_layer(N):
    cfg = W.BUDGET_S32.with_(budget=N)
    diag, g, _ = _run(cfg, gen_device="cuda")
    assert g.n_dropped > 0 and int(g.kept.sum()) == N
    print(cfg.label, diag, "n_dropped", g.n_dropped)


@pytest.fixture(scope="module")
def large_inputs():
    """256 experts x 2048 x 7168 (22.5 GB bf16) drawn once; logits N(0,1) for the
    largest T; host copies of expert weights shared by the tests."""
    cfg = W.LARGE_256E.with_(T=max(W.LARGE_T_SWEEP))
    inp = W.make_inputs(cfg, device="cuda")
    yield cfg, inp, {}
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", W.LARGE_T_SWEEP)
@pytest.mark.parametrize("alpha", W.LARGE_ALPHAS)
def test_large_layer(large_inputs, T, alpha):
    """Every (T, alpha) point of the 256-expert sweep, rows stratified over every
    (expert group, token tile) plus >= 256 seeded tokens at T >= 4096."""
    base_cfg, base, cache = large_inputs
    cfg = base_cfg.with_(T=T, zipf_alpha=alpha)
    logits = base.logits[:T] + W.zipf_bias(cfg.E, alpha, "cuda")
    inp = W.MoEInputs(base.x[:T].contiguous(), logits.contiguous(), base.w_gate, base.w_up, base.w_down)
    g = gpu_forward(cfg, inp)
    diag = check_layer(cfg, inp, g, rows=_strat(cfg, 256 if T >= 4096 else 64), weight_cache=cache)
    print(cfg.label, diag, "max group", int(g.counts.max()), "touched", int((g.counts > 0).sum()))


@pytest.mark.parametrize("cfg", [W.MoEConfig("phases", T=300, H=256, E=8, I=192, k=2, Is=128, zipf_alpha=1.0),
                                 W.MoEConfig("phases_noshared", T=77, H=384, E=16, I=64, k=4)],
                         ids=lambda c: c.name)
def test_split_phases_match_fused(cfg):
    """moe_expert_gate_up then moe_expert_down (two launches) writes the same
    ybuf bits as the fused one-launch moe_expert_ffn."""
    c = lib_config(cfg)
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    dev = "cuda"
    inp = W.make_inputs(cfg, device=dev)
    ws = torch.zeros(moe.workspace_bytes(c, T), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    sgate = torch.empty(T, dtype=torch.float32, device=dev) if cfg.Is else None
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    y1 = torch.zeros((T, k + 1, H), dtype=torch.bfloat16, device=dev)
    y2 = torch.zeros((T, k + 1, H), dtype=torch.bfloat16, device=dev)
    moe.moe_route(c, inp.logits, idx, w, x=inp.x if cfg.Is else None, ws_gate_vec=inp.ws_gvec, sgate=sgate)
    moe.moe_dispatch(c, idx, counts, offsets, perm, slot_pos, ws, x=inp.x, x_perm=x_perm)
    wts = weights_of(inp)
    moe.moe_expert_ffn(c, inp.x, x_perm, offsets, perm, w, wts, y1, ws, sgate=sgate)
    moe.moe_expert_gate_up(c, inp.x, x_perm, offsets, wts, ws)
    moe.moe_expert_down(c, T, offsets, perm, w, wts, y2, ws, sgate=sgate)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == 0
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
