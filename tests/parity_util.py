"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare them.

Comparison rules (the tolerance is the one stated for the layer output):
  * routing indices, budget drops, counts, offsets, perm, slot_pos: bit-exact;
  * routing weights: fp32 within 2e-6 relative (GPU and CPU exp differ by ulps);
  * the layer output: relative L2 error <= 5e-3 over the compared rows
    (bf16 inputs/outputs, fp32 accumulation on the GPU, fp64 in the oracle),
    and no single row above 1e-2 (a row's error is the same rounding of h,
    ybuf and out, about 2e-3 RMS, so a row twice the layer bound points at a
    wrong tile rather than rounding);
  * budget near-ties: when the GPU keeps a different expert set, the
    oracle's aggregate gap between the last kept and first dropped expert
    must be <= 1e-5 of the largest aggregate; the oracle's step 4
    (compaction and renormalisation) is then run with the GPU's kept set and
    must give the GPU's post-budget routing (indices and keff bit-exact,
    weights within 2e-6), and the downstream comparison uses it.
  * top-p near-ties: when the GPU keeps a different number of slots of a
    token, the oracle's prefix mass at some slot of that token must be
    within 1e-5 of topp (the trim decided on ulp-different weights), and
    the kept slots must still be a prefix of the oracle's top-k; the
    downstream comparison then uses the GPU's routing.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

import oracle
import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

REL_L2_TOL = 5e-3
ROW_REL_L2_TOL = 1e-2
W_RTOL = 2e-6
NEAR_TIE = 1e-5


def lib_config(cfg: W.MoEConfig) -> moe.MoEConfig:
    return moe.MoEConfig(cfg.H, cfg.E, cfg.I, cfg.k, cfg.Is, cfg.norm_topk, cfg.budget, cfg.topp)


def topp_margin(w: np.ndarray, p: float, t: int) -> float:
    """Smallest |prefix mass - p| over the decisions of token t (fp32, slot order)."""
    mass = np.float32(0.0)
    m = np.inf
    for j in range(w.shape[1]):
        if j > 0:
            m = min(m, abs(float(mass) - p))
        mass = np.float32(mass + w[t, j])
    return m


def weights_of(inp: W.MoEInputs) -> moe.MoEWeights:
    return moe.MoEWeights(inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up, inp.ws_down, inp.ws_gvec,
                          inp.w_router)


def logits_bound(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    """Per-logit error bound of an fp32 accumulation: 1e-5 * sum_h |x_h w_h| (+ 1e-6)."""
    x = x_bits.view(np.uint16).astype(np.uint32) << 16
    w = wr_bits.view(np.uint16).astype(np.uint32) << 16
    xf = np.abs(x.view(np.float32).astype(np.float64))
    wf = np.abs(w.view(np.float32).astype(np.float64))
    return 1e-5 * (xf @ wf.T) + 1e-6


@dataclass
class GpuResult:
    out: np.ndarray       # [T, H] float32 (bf16 values)
    idx: np.ndarray
    w: np.ndarray
    keff: np.ndarray
    kept: np.ndarray
    n_dropped: int
    counts: np.ndarray
    offsets: np.ndarray
    perm: np.ndarray      # [sum keff]
    slot_pos: np.ndarray
    sgate: Optional[np.ndarray]
    status: int
    out_bits: np.ndarray  # raw bf16 bits, for bit-identity checks


def gpu_forward(cfg: W.MoEConfig, inp: W.MoEInputs, ws: Optional[torch.Tensor] = None, weights=None,
                fwd=None) -> GpuResult:
    """moe_forward (or `fwd`, e.g. moe_forward_mxfp8, with `weights`) on the inputs."""
    dev = inp.x.device
    T, k, E = cfg.T, cfg.k, cfg.E
    c = lib_config(cfg)
    if ws is None:
        ws = torch.empty(moe.workspace_bytes(c, T), dtype=torch.uint8, device=dev)
        moe.status_clear(ws)
    aux = dict(
        topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
        topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
        keff=torch.empty(T, dtype=torch.int32, device=dev),
        expert_kept=torch.zeros(E, dtype=torch.uint8, device=dev),
        n_dropped=torch.zeros(1, dtype=torch.int32, device=dev),
        counts=torch.empty(E, dtype=torch.int32, device=dev),
        offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
        perm=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev),
        slot_pos=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev),
    )
    if cfg.Is:
        aux["sgate"] = torch.empty(T, dtype=torch.float32, device=dev)
    out = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)
    (fwd or moe.moe_forward)(c, inp.x, inp.logits, weights if weights is not None else weights_of(inp), out, ws,
                             aux=aux)
    status = moe.status_read(ws)
    torch.cuda.synchronize()
    h = {n: t.cpu().numpy() for n, t in aux.items()}
    total = int(h["offsets"][E])
    return GpuResult(out.float().cpu().numpy(), h["topk_idx"], h["topk_w"], h["keff"], h["expert_kept"],
                     int(h["n_dropped"][0]), h["counts"], h["offsets"], h["perm"][:total], h["slot_pos"][: T * k],
                     h.get("sgate"), status, W.bf16_bits(out))


def rel_l2(a: np.ndarray, ref: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / den) if den > 0 else float(np.linalg.norm(a))


def row_rel_l2(a: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Relative L2 error of every row; a zero reference row counts the
    row's own norm (it must be exactly zero too)."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.linalg.norm(a - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def stratified_rows(T: int, k: int, offsets: np.ndarray, perm: np.ndarray, tile: int = 256, n_random: int = 0,
                    shared_tile: int = 0, seed: int = 1) -> np.ndarray:
    """Tokens whose outputs cover every work item of the expert FFN: for each
    expert group, one seeded dispatched row of every token tile of `tile`
    rows, plus the group's first and last row (the ragged tail); for the
    shared expert (shared_tile > 0), one seeded token of every tile of its
    rows; plus token 0, token T-1 and n_random seeded tokens.  A row's output
    depends on every weight tile of its group, so one row per (group, token
    tile) reaches every (weight tile, token tile) item of both phases."""
    rng = np.random.default_rng(seed)
    toks = {0, T - 1}
    E = len(offsets) - 1
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi <= lo:
            continue
        picks = [lo, hi - 1]
        for t0 in range(lo, hi, tile):
            picks.append(t0 + int(rng.integers(0, min(tile, hi - t0))))
        toks.update(int(perm[p]) // k for p in picks)
    if shared_tile:
        for t0 in range(0, T, shared_tile):
            toks.add(t0 + int(rng.integers(0, min(shared_tile, T - t0))))
    if n_random:
        toks.update(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    return np.array(sorted(toks), dtype=np.int32)


def sample_rows(T: int, n: int, seed: int = 1) -> np.ndarray:
    """First, last and n-2 seeded tokens in between (all tokens if n >= T)."""
    if n >= T:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), size=max(n - 2, 0), replace=False)
    return np.unique(np.concatenate([[0, T - 1], mid])).astype(np.int32)


def _expert_dicts(inp: W.MoEInputs, experts, cache: Optional[dict] = None, wmap=None):
    """Host copies of the listed experts' weights (through `wmap`, e.g. the
    oracle's MXFP8 weights, when given); `cache` (keyed by expert) keeps them
    across calls on the same weight tensors."""
    bits = W.bf16_bits if wmap is None else (lambda t: wmap(W.bf16_bits(t)))
    cache = {} if cache is None else cache
    for e in experts:
        if e not in cache:
            cache[e] = (bits(inp.w_gate[e]), bits(inp.w_up[e]), bits(inp.w_down[e]))
    return ({e: cache[e][0] for e in experts}, {e: cache[e][1] for e in experts},
            {e: cache[e][2] for e in experts})


def check_layer(cfg: W.MoEConfig, inp: W.MoEInputs, g: GpuResult, rows=None,
                nthreads: Optional[int] = None, weight_cache: Optional[dict] = None, wmap=None) -> dict:
    """Compare a GPU forward with the oracle; returns diagnostics, asserts.
    `wmap` maps each expert matrix's bf16 bits to the weights the oracle
    uses (e.g. oracle.mxfp8_weights for the MXFP8 layer), or to (weights,
    matrix scale) pairs (oracle.nvfp4_weights for the NVFP4 layer); default:
    as is."""
    assert g.status == 0, f"device status {g.status}"
    T, k, E = cfg.T, cfg.k, cfg.E
    nthreads = nthreads or oracle.max_threads()
    logits = inp.logits.cpu().numpy()
    # route (bit-exact indices, fp32 weights within ulps)
    idx_o, w_o = oracle.route(logits, k, cfg.norm_topk)
    diag = {}
    # the top-p trim on the oracle's routing
    if cfg.topp:
        idx_p, w_p, keff_p = oracle.topp(idx_o, w_o, cfg.topp, cfg.norm_topk)
    else:
        idx_p, w_p, keff_p = idx_o, w_o, np.full(T, k, np.int32)
    if cfg.budget == 0:
        if (g.idx == idx_p).all() and (g.keff == keff_p).all():
            np.testing.assert_allclose(g.w, w_p, rtol=W_RTOL, atol=1e-7)
            idx_b, w_b, keff_b = idx_p, w_p, keff_p
        else:
            assert cfg.topp, "routing indices differ"
            bad = np.nonzero((g.keff != keff_p) | (g.idx != idx_p).any(1))[0]
            for t in bad:
                c = int(g.keff[t])
                assert (g.idx[t, :c] == idx_o[t, :c]).all() and (g.idx[t, c:] == -1).all(), "not a top-k prefix"
                m = topp_margin(w_o, cfg.topp, int(t))
                assert m <= NEAR_TIE, f"top-p kept count differs with margin {m}"
            diag["topp_near"] = int(len(bad))
            idx_b, w_b, keff_b = g.idx, g.w, g.keff
    else:
        # the budget on the oracle's own (trimmed) routing
        idx_b, w_b, keff_b, kept_b, nd_b = oracle.budget(idx_p, w_p, E, cfg.budget, cfg.norm_topk)
        if (kept_b == g.kept).all() and (g.idx == idx_b).all() and (g.keff == keff_b).all():
            assert g.n_dropped == nd_b
            np.testing.assert_allclose(g.w, w_b, rtol=W_RTOL, atol=1e-7)
        else:
            valid = idx_p >= 0
            agg = np.zeros(E)
            np.add.at(agg, idx_p[valid], w_p[valid].astype(np.float64))
            union = np.unique(idx_p[valid])
            order = union[np.lexsort((union, -agg[union]))]
            gap = agg[order[cfg.budget - 1]] - agg[order[cfg.budget]] if len(union) > cfg.budget else np.inf
            near_budget = gap <= NEAR_TIE * agg.max()
            near_topp = bool(cfg.topp) and min(topp_margin(w_o, cfg.topp, t) for t in range(T)) <= NEAR_TIE
            assert near_budget or near_topp, f"budget keep-set differs with gap {gap}"
            diag["near_tie"] = float(gap)
            assert int(g.kept.sum()) == min(cfg.budget, len(union)), "GPU kept-set size"
            assert set(np.nonzero(g.kept)[0].tolist()) <= set(union.tolist()), "GPU kept an expert outside the union"
            if not near_topp:  # same routing before the budget: step 4 with the GPU's kept set
                idx_b, w_b, keff_b = oracle.budget_apply(idx_p, w_p, g.kept, cfg.norm_topk)
                assert (g.idx == idx_b).all() and (g.keff == keff_b).all(), "compaction with the GPU's kept set"
                np.testing.assert_allclose(g.w, w_b, rtol=W_RTOL, atol=1e-7)
                assert g.n_dropped == len(union) - cfg.budget
            idx_b, w_b, keff_b = g.idx, g.w, g.keff
    # dispatch on the same routing: bit-exact
    counts, offsets, perm, slot_pos = oracle.dispatch(idx_b, keff_b, E)
    assert (g.counts == counts).all() and (g.offsets == offsets).all(), "counts/offsets differ"
    assert (g.perm == perm).all() and (g.slot_pos == slot_pos).all(), "perm/slot_pos differ"
    # shared gate
    if cfg.Is:
        sg = oracle.shared_gate(W.bf16_bits(inp.ws_gvec), W.bf16_bits(inp.x))
        np.testing.assert_allclose(g.sgate, sg, rtol=1e-5, atol=1e-6)
    # layer output on the chosen rows
    if rows is None:
        rows = np.arange(T, dtype=np.int32)
    elif callable(rows):  # rows chosen from the (now verified) dispatch
        rows = rows(offsets, perm)
    need = sorted({int(idx_b[t, j]) for t in rows for j in range(int(keff_b[t]))})
    wg, wu, wd = _expert_dicts(inp, need, weight_cache, wmap)
    kw = {}
    if need and isinstance(wg[need[0]], tuple):  # (weights, matrix scale) per expert matrix
        sc = np.ones((max(max(need), int(idx_b.max(initial=0))) + 1, 3))
        for e in need:
            sc[e] = [float(wg[e][1]), float(wu[e][1]), float(wd[e][1])]
        wg, wu, wd = ({e: m[e][0] for e in need} for m in (wg, wu, wd))
        kw["scales"] = sc
    if cfg.Is:
        sb = W.bf16_bits if wmap is None else (lambda t: wmap(W.bf16_bits(t)))
        sgw, suw, sdw = sb(inp.ws_gate), sb(inp.ws_up), sb(inp.ws_down)
        if isinstance(sgw, tuple):
            kw["shared_scales"] = np.array([float(sgw[1]), float(suw[1]), float(sdw[1])])
            sgw, suw, sdw = sgw[0], suw[0], sdw[0]
        kw.update(ws_gate=sgw, ws_up=suw, ws_down=sdw, ws_gvec=W.bf16_bits(inp.ws_gvec))
    ref = oracle.combine_rows(W.bf16_bits(inp.x), idx_b, w_b, keff_b, wg, wu, wd, I=cfg.I, rows=rows,
                              nthreads=nthreads, **kw)
    err = rel_l2(g.out[rows], ref)
    diag["rel_l2"] = err
    diag["rows"] = int(len(rows))
    row_err = row_rel_l2(g.out[rows], ref)
    worst = int(np.argmax(row_err)) if len(rows) else 0
    diag["row_rel_l2_max"] = float(row_err[worst]) if len(rows) else 0.0
    diag["row_rel_l2_worst_token"] = int(rows[worst]) if len(rows) else -1
    assert err <= REL_L2_TOL, f"rel-L2 {err:.3e} > {REL_L2_TOL}"
    assert diag["row_rel_l2_max"] <= ROW_REL_L2_TOL, \
        f"token {diag['row_rel_l2_worst_token']}: row rel-L2 {diag['row_rel_l2_max']:.3e} > {ROW_REL_L2_TOL}"
    # rows with no kept slot and no shared expert must be exactly zero
    if not cfg.Is:
        empty = np.nonzero(keff_b == 0)[0]
        assert (g.out[empty] == 0).all()
    return diag
