"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Every check here compares the oracle against something other than itself:
values printed on the pages (tests/golden), hand-worked examples, closed
forms, exhaustive search on tiny inputs, library routines (torch softmax,
silu, linear, stable sorts) and invariants.  No GPU is used.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from routed_expert_ffn_renorm_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def bits(t):
    return W.bf16_bits(t)


# ---------------------------------------------------------------- shapes --

def test_param_counts_match_drafter_table(oracle_mod):
    g = _gold("drafter_ffn_params.json")
    H, Is = g["hidden"], g["shared_intermediate"]
    for row in g["rows"]:
        shared = oracle_mod.ffn_params(H, row["Is"]) if row["Is"] else 0
        total = row["E"] * oracle_mod.ffn_params(H, row["I"]) + shared
        active = row["k"] * oracle_mod.ffn_params(H, row["I"]) + shared
        if "params_M" in row:
            assert round(total / 1e6) == row["params_M"], row["what"]
        else:
            assert round(total / 1e9, 2) == row["params_B"], row["what"]
        assert round(active / 1e6) == row["active_M"], row["what"]
    moe = 16 * oracle_mod.ffn_params(H, 1024) + oracle_mod.ffn_params(H, Is)
    assert round(moe / oracle_mod.ffn_params(H, 17408), 2) == g["size_ratio"]["ratio"]
    for b in g["expert_bytes"]:
        nbytes = b["experts"] * oracle_mod.ffn_params(H, b["I"]) * 2
        assert abs(nbytes / 1e9 - b["approx_GB"]) <= b["rel_tol"] * b["approx_GB"], b["what"]
    ub = g["union_bound"]
    # the union of a block's routed experts can never exceed tokens * k
    rng = np.random.default_rng(3)
    for _ in range(200):
        logits = rng.standard_normal((ub["tokens"], ub["E"])).astype(np.float32)
        idx, _ = oracle_mod.route(logits, ub["k"])
        assert len(set(idx.ravel().tolist())) <= ub["max_union"]


# ----------------------------------------------------------------- route --

def test_router_logits_unit_vectors_and_torch(oracle_mod):
    """x = unit vector e_h picks column h of W_r exactly; random inputs match
    torch's fp64 linear map rounded to fp32."""
    H, E = 48, 7
    wr = _bf(np.random.default_rng(2).standard_normal((E, H)))
    eye = _bf(np.eye(H))
    lg = oracle_mod.router_logits(bits(eye), bits(wr))
    assert (lg == wr.float().numpy().T).all()
    x = _bf(np.random.default_rng(3).standard_normal((9, H)))
    ref = F.linear(x.double(), wr.double()).float().numpy()
    np.testing.assert_allclose(oracle_mod.router_logits(bits(x), bits(wr)), ref, rtol=1e-6, atol=1e-7)
    # the bias-free map is linear: doubling x (exact in bf16) doubles the logits exactly
    assert (oracle_mod.router_logits(bits(x * 2), bits(wr)) == 2 * oracle_mod.router_logits(bits(x), bits(wr))).all()


def test_route_closed_form_worked_example(oracle_mod):
    # logits ln(1..4): softmax = (1,2,3,4)/10; top-2 = experts 3, 2;
    # renormalised weights 4/7, 3/7.
    logits = np.log(np.array([[1.0, 2.0, 3.0, 4.0]], np.float32))
    idx, w = oracle_mod.route(logits, 2, norm_topk=True)
    assert idx.tolist() == [[3, 2]]
    np.testing.assert_allclose(w[0], [4 / 7, 3 / 7], rtol=1e-6)
    idx, w = oracle_mod.route(logits, 2, norm_topk=False)
    np.testing.assert_allclose(w[0], [0.4, 0.3], rtol=1e-6)


def test_route_ties_take_lower_id(oracle_mod):
    logits = np.array([[1.0, 2.0, 2.0, 0.0, 2.0]], np.float32)
    idx, w = oracle_mod.route(logits, 3)
    assert idx.tolist() == [[1, 2, 4]]
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-6)


@pytest.mark.parametrize("E,k", [(8, 1), (8, 2), (8, 3), (6, 6), (10, 4)])
def test_route_brute_force_topk(oracle_mod, E, k):
    rng = np.random.default_rng(E * 100 + k)
    logits = rng.standard_normal((64, E)).astype(np.float32)
    idx, w = oracle_mod.route(logits, k)
    for t in range(logits.shape[0]):
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(float(logits[t, e]) for e in s))
        assert sorted(idx[t].tolist()) == sorted(best)
        assert all(logits[t, idx[t, j]] >= logits[t, idx[t, j + 1]] for j in range(k - 1))


def test_route_weights_against_torch_softmax(oracle_mod):
    rng = np.random.default_rng(7)
    E, k = 32, 6
    logits = (rng.standard_normal((50, E)) * 3).astype(np.float32)
    p = torch.softmax(torch.from_numpy(logits).double(), dim=-1).numpy()
    idx, w = oracle_mod.route(logits, k, norm_topk=False)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=2e-6, atol=1e-9)
    idx2, wn = oracle_mod.route(logits, k, norm_topk=True)
    assert (idx2 == idx).all()
    ref = np.take_along_axis(p, idx, 1)
    np.testing.assert_allclose(wn, ref / ref.sum(1, keepdims=True), rtol=2e-6)
    np.testing.assert_allclose(wn.sum(1), 1.0, rtol=1e-6)
    # ratios fixed by the logit gaps: w_a / w_b = exp(l_a - l_b)
    r = wn[:, 0] / wn[:, 1]
    gap = np.take_along_axis(logits, idx[:, :1], 1)[:, 0].astype(np.float64) - \
        np.take_along_axis(logits, idx[:, 1:2], 1)[:, 0]
    np.testing.assert_allclose(r, np.exp(gap), rtol=1e-5)
    # torch.topk gives the same expert sets
    tk = torch.topk(torch.from_numpy(logits), k, dim=-1).indices.numpy()
    assert (np.sort(tk, 1) == np.sort(idx, 1)).all()


def test_route_k_equals_E_is_full_softmax(oracle_mod):
    rng = np.random.default_rng(11)
    logits = rng.standard_normal((20, 7)).astype(np.float32)
    for norm in (True, False):
        idx, w = oracle_mod.route(logits, 7, norm_topk=norm)
        full = np.zeros_like(w)
        np.put_along_axis(full, idx, w, 1)
        np.testing.assert_allclose(full, torch.softmax(torch.from_numpy(logits).double(), -1).numpy(),
                                   rtol=2e-6)


# ---------------------------------------------------------------- budget --

def test_budget_worked_example(oracle_mod):
    g = _gold("budget_worked_example.json")
    idx = np.array(g["idx"], np.int32)
    w = np.array(g["w"], np.float32)
    for norm, key in ((True, "expect_norm"), (False, "expect_no_norm")):
        ex = g[key]
        i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, g["E"], g["N"], norm_topk=norm)
        assert i2.tolist() == ex["idx"]
        assert w2.tolist() == ex["w"]
        assert keff.tolist() == ex["keff"]
        assert kept.tolist() == ex["kept"]
        assert nd == ex["n_dropped"]
    i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, g["E"], g["N"], norm_topk=True)
    counts, offsets, perm, slot_pos = oracle_mod.dispatch(i2, keff, g["E"])
    d = g["dispatch"]
    assert counts.tolist() == d["counts"] and offsets.tolist() == d["offsets"]
    assert perm.tolist() == d["perm"] and slot_pos.tolist() == d["slot_pos"]


def test_budget_apply_worked_example(oracle_mod):
    """Step 4 for a given kept set: the hand-worked other side of the example's tie."""
    g = _gold("budget_worked_example.json")
    idx = np.array(g["idx"], np.int32)
    w = np.array(g["w"], np.float32)
    alt = g["alternative_kept"]
    for norm, key in ((True, "expect_norm"), (False, "expect_no_norm")):
        i2, w2, keff = oracle_mod.budget_apply(idx, w, np.array(alt["kept"], np.uint8), norm_topk=norm)
        assert i2.tolist() == alt[key]["idx"] and w2.tolist() == alt[key]["w"] and keff.tolist() == alt[key]["keff"]


@pytest.mark.parametrize("norm", [True, False])
def test_budget_apply_with_own_kept_set_is_budget(oracle_mod, norm):
    """budget() = choose the kept set, then step 4: applying step 4 to the
    router output with budget()'s kept set gives its outputs bit for bit."""
    for seed, N in ((3, 4), (4, 12), (5, 20)):
        idx, w = _route_for_budget(oracle_mod, 32, 128, 8, seed)
        i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, 128, N, norm_topk=norm)
        i3, w3, keff3 = oracle_mod.budget_apply(idx, w, kept, norm_topk=norm)
        assert (i3 == i2).all() and (w3.view(np.uint32) == w2.view(np.uint32)).all() and (keff3 == keff).all()


# ----------------------------------------------------------------- top-p --

def test_topp_worked_example(oracle_mod):
    g = _gold("topp_worked_example.json")
    idx = np.array(g["idx"], np.int32)
    w = np.array(g["w"], np.float32)
    for case in g["cases"]:
        for norm, key in ((True, "expect_norm"), (False, "expect_no_norm")):
            if key not in case:
                continue
            ex = case[key]
            i2, w2, keff = oracle_mod.topp(idx, w, case["topp"], norm_topk=norm)
            assert i2.tolist() == ex["idx"], (case["topp"], norm)
            assert w2.tolist() == ex["w"], (case["topp"], norm)
            assert keff.tolist() == ex["keff"], (case["topp"], norm)
    b = g["with_budget"]
    i2, w2, keff = oracle_mod.topp(idx, w, b["topp"], norm_topk=True)
    i3, w3, keff3, kept, nd = oracle_mod.budget(i2, w2, g["E"], b["N"], norm_topk=True)
    ex = b["expect"]
    assert i3.tolist() == ex["idx"] and w3.tolist() == ex["w"] and keff3.tolist() == ex["keff"]
    assert kept.tolist() == ex["kept"] and nd == ex["n_dropped"]


@pytest.mark.parametrize("norm", [True, False])
def test_topp_invariants(oracle_mod, norm):
    T, E, k = 64, 64, 8
    rng = np.random.default_rng(11)
    idx, w = oracle_mod.route((rng.standard_normal((T, E)) * 1.5).astype(np.float32), k, norm_topk=norm)
    for p in (0.0, 1.0, 1.5, -0.25):  # off: unchanged, bit for bit
        i2, w2, keff = oracle_mod.topp(idx, w, p, norm_topk=norm)
        assert (i2 == idx).all() and (w2.view(np.uint32) == w.view(np.uint32)).all() and (keff == k).all()
    for p in (1e-6, 0.3, 0.5, 0.8, 0.95):
        i2, w2, keff = oracle_mod.topp(idx, w, p, norm_topk=norm)
        for t in range(T):
            c = int(keff[t])
            assert 1 <= c <= k
            # the mass before the last kept slot is below p, the kept mass reaches p (fp32, slot order)
            mass = [np.float32(0.0)]
            for j in range(k):
                mass.append(np.float32(mass[-1] + w[t, j]))
            assert c == 1 or mass[c - 1] < np.float32(p)
            assert c == k or mass[c] >= np.float32(p)
            assert i2[t, :c].tolist() == idx[t, :c].tolist()
            assert (i2[t, c:] == -1).all() and (w2[t, c:] == 0).all()
            if c == k or not norm:
                assert (w2[t, :c].view(np.uint32) == w[t, :c].view(np.uint32)).all()
            else:
                s = np.float32(0.0)
                for j in range(c):
                    s = np.float32(s + w[t, j])
                assert (w2[t, :c] == (w[t, :c] / s).astype(np.float32)).all()
        if p == 1e-6:
            assert (keff == 1).all()
            if norm:
                assert (w2[:, 0] == 1.0).all()


def test_topp_then_budget_composition(oracle_mod):
    """The budget after a top-p trim: trimmed slots take no part, and a token
    the budget leaves whole keeps its post-trim weights bit for bit."""
    T, E, k = 40, 48, 6
    rng = np.random.default_rng(17)
    idx, w = oracle_mod.route((rng.standard_normal((T, E)) - 0.8 * np.log1p(np.arange(E))).astype(np.float32), k)
    i1, w1, keff1 = oracle_mod.topp(idx, w, 0.7)
    union = sorted(set(i1[i1 >= 0].tolist()))
    i_off, w_off, keff_off, kept_off, nd_off = oracle_mod.budget(i1, w1, E, 0)
    assert (i_off == i1).all() and (w_off.view(np.uint32) == w1.view(np.uint32)).all()
    assert keff_off.tolist() == keff1.tolist() and nd_off == 0
    assert sorted(np.nonzero(kept_off)[0].tolist()) == union
    N = len(union) // 2
    i2, w2, keff2, kept, nd = oracle_mod.budget(i1, w1, E, N)
    assert nd == len(union) - N and int(kept.sum()) == N
    whole = 0
    for t in range(T):
        surv = [j for j in range(keff1[t]) if kept[i1[t, j]]]
        assert keff2[t] == len(surv) and i2[t, :len(surv)].tolist() == [int(i1[t, j]) for j in surv]
        if len(surv) == keff1[t]:
            whole += 1
            assert (w2[t, :keff1[t]].view(np.uint32) == w1[t, :keff1[t]].view(np.uint32)).all()
    assert whole > 0


def _route_for_budget(oracle_mod, T, E, k, seed, alpha=0.0):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits += (-alpha * np.log1p(np.arange(E))).astype(np.float32)
    return oracle_mod.route(logits, k)


@pytest.mark.parametrize("seed", range(6))
def test_budget_brute_force_keeps_heaviest_subset(oracle_mod, seed):
    T, E, k = 5, 10, 3
    idx, w = _route_for_budget(oracle_mod, T, E, k, seed)
    union = sorted(set(idx.ravel().tolist()))
    agg = {e: float(w[idx == e].astype(np.float64).sum()) for e in union}
    for N in range(1, len(union)):
        i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, E, N)
        best = max(itertools.combinations(union, N), key=lambda s: sum(agg[e] for e in s))
        assert sorted(np.nonzero(kept)[0].tolist()) == sorted(best)
        assert nd == len(union) - N
        assert set(i2[i2 >= 0].tolist()) <= set(best)


@pytest.mark.parametrize("norm", [True, False])
def test_budget_invariants(oracle_mod, norm):
    T, E, k = 32, 128, 8
    idx, w = oracle_mod.route(
        (np.random.default_rng(5).standard_normal((T, E)) - 1.2 * np.log1p(np.arange(E))).astype(np.float32),
        k, norm_topk=norm)
    nu = len(set(idx.ravel().tolist()))
    for N in (0, nu, nu + 5):  # off, or a budget no smaller than the union: unchanged
        i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, E, N, norm_topk=norm)
        assert (i2 == idx).all() and (w2.view(np.uint32) == w.view(np.uint32)).all()
        assert (keff == k).all() and nd == 0
        assert sorted(np.nonzero(kept)[0].tolist()) == sorted(set(idx.ravel().tolist()))
    for N in (1, 4, 12, 24):
        if N >= nu:
            continue
        i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, E, N, norm_topk=norm)
        assert nd == nu - N and int(kept.sum()) == N
        assert set(i2[i2 >= 0].tolist()) == set(np.nonzero(kept)[0].tolist())
        for t in range(T):
            c = keff[t]
            surv = [j for j in range(k) if kept[idx[t, j]]]
            assert c == len(surv)
            assert i2[t, :c].tolist() == [int(idx[t, j]) for j in surv]   # order kept
            assert (i2[t, c:] == -1).all() and (w2[t, c:] == 0).all()
            if c == k or not norm:  # untouched tokens / no renormalisation: bit-identical
                assert (w2[t, :c].view(np.uint32) == w[t, surv].view(np.uint32)).all()
            elif c > 0:
                assert abs(float(w2[t, :c].astype(np.float64).sum()) - 1.0) < 1e-6
                np.testing.assert_allclose(w2[t, :c], w[t, surv] / w[t, surv].sum(), rtol=1e-6)


def test_budget_drops_can_empty_tokens(oracle_mod):
    idx, w = _route_for_budget(oracle_mod, 32, 128, 8, 9, alpha=0.0)
    i2, w2, keff, kept, nd = oracle_mod.budget(idx, w, 128, 4)
    assert (keff == 0).any()
    empty = np.nonzero(keff == 0)[0]
    assert (i2[empty] == -1).all() and (w2[empty] == 0).all()


# -------------------------------------------------------------- dispatch --

@pytest.mark.parametrize("T,E,k,N", [(16, 8, 2, 0), (33, 16, 4, 5), (64, 128, 8, 12), (1, 4, 4, 0)])
def test_dispatch_matches_stable_sort(oracle_mod, T, E, k, N):
    idx, w = _route_for_budget(oracle_mod, T, E, k, T + E, alpha=1.0)
    idx, w, keff, kept, nd = oracle_mod.budget(idx, w, E, N)
    counts, offsets, perm, slot_pos = oracle_mod.dispatch(idx, keff, E)
    slots = np.array([t * k + j for t in range(T) for j in range(keff[t])], np.int64)
    experts = idx.ravel()[slots]
    order = np.lexsort((slots, experts))  # expert first, slot id second
    assert perm.tolist() == slots[order].tolist()
    assert counts.tolist() == np.bincount(experts, minlength=E).tolist()
    assert offsets.tolist() == [0] + np.cumsum(np.bincount(experts, minlength=E)).tolist()
    assert int(counts.sum()) == int(keff.sum())
    if N == 0:
        assert int(counts.sum()) == T * k
    assert (slot_pos[perm] == np.arange(perm.size)).all()
    dropped = np.setdiff1d(np.arange(T * k), slots)
    assert (slot_pos[dropped] == -1).all()


def test_dispatch_empty_batch(oracle_mod):
    counts, offsets, perm, slot_pos = oracle_mod.dispatch(np.zeros((0, 2), np.int32), np.zeros(0, np.int32), 4)
    assert counts.tolist() == [0] * 4 and offsets.tolist() == [0] * 5 and perm.size == 0


# ------------------------------------------------------------ expert FFN --

def _bf(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def test_ffn_closed_form_unit_vectors(oracle_mod):
    # H=3, I=2.  x = e_0, gate row 0 picks a*x_0, up row 0 picks b*x_0, other
    # rows zero: h = (silu(a)*b, 0), y = silu(a)*b * W_down[:, 0].
    a, b = 1.1015625, 0.75           # exact in bf16
    H, I = 3, 2
    wg = np.zeros((I, H), np.float32); wg[0, 0] = a
    wu = np.zeros((I, H), np.float32); wu[0, 0] = b
    wd = np.array([[0.5, 3.0], [-2.0, 1.0], [0.25, 0.0]], np.float32)  # [H, I]
    x = np.array([[1.0, 0.0, 0.0], [-1.0, 0.0, 0.0]], np.float32)
    y = oracle_mod.expert_rows(bits(_bf(wg)), bits(_bf(wu)), bits(_bf(wd)), bits(_bf(x)))
    s_pos, s_neg = y[0, 0] / (0.5 * b), y[1, 0] / (0.5 * -b)   # silu(a), silu(-a)
    # silu(a) - silu(-a) = a  and  silu(a) + silu(-a) = a * tanh(a / 2)
    assert abs((s_pos - s_neg) - a) < 1e-12
    assert abs((s_pos + s_neg) - a * math.tanh(a / 2)) < 1e-12
    # sigmoid(ln 3) = 3/4: a is ln 3 rounded to bf16
    assert abs(s_pos / a - 0.75) < 1e-3
    np.testing.assert_allclose(y[0], s_pos * b * wd[:, 0], rtol=1e-12)


def test_ffn_single_expert_is_plain_swiglu_mlp(oracle_mod):
    cfg = W.MoEConfig("one", T=9, H=96, E=1, I=40, k=1)
    inp = W.make_inputs(cfg, std=0.2)
    r = oracle_mod.forward(bits(inp.x), inp.logits.numpy(), bits(inp.w_gate), bits(inp.w_up), bits(inp.w_down),
                           k=1)
    x = inp.x.double()
    ref = F.linear(F.silu(F.linear(x, inp.w_gate[0].double())) * F.linear(x, inp.w_up[0].double()),
                   inp.w_down[0].double())
    np.testing.assert_allclose(r.out, ref.numpy(), rtol=1e-10, atol=1e-14)
    assert (r.w == 1.0).all()


def test_combine_k_equals_E_is_softmax_mixture(oracle_mod):
    cfg = W.MoEConfig("mix", T=7, H=64, E=4, I=32, k=4)
    inp = W.make_inputs(cfg, std=0.2)
    r = oracle_mod.forward(bits(inp.x), inp.logits.numpy(), bits(inp.w_gate), bits(inp.w_up), bits(inp.w_down),
                           k=4)
    x = inp.x.double()
    ys = torch.stack([F.linear(F.silu(F.linear(x, inp.w_gate[e].double())) * F.linear(x, inp.w_up[e].double()),
                               inp.w_down[e].double()) for e in range(4)], 1)        # [T, E, H]
    p = torch.softmax(inp.logits.double(), -1)
    ref = torch.einsum("te,teh->th", p, ys).numpy()
    # routing weights are fp32 in the oracle: relative 1e-6 of the output scale
    np.testing.assert_allclose(r.out, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


@pytest.mark.parametrize("N,norm", [(0, True), (3, True), (3, False), (1, True)])
def test_forward_dense_masked_loop(oracle_mod, N, norm):
    """Dense loop over ALL experts per token, masked by routing (no dispatch)."""
    cfg = W.MoEConfig("dense", T=12, H=64, E=6, I=32, k=3, Is=64, norm_topk=norm, budget=N, zipf_alpha=0.5)
    inp = W.make_inputs(cfg, std=0.2, gate_std=1.0)
    r = oracle_mod.forward(bits(inp.x), inp.logits.numpy(), bits(inp.w_gate), bits(inp.w_up), bits(inp.w_down),
                           k=3, norm_topk=norm, budget=N, ws_gate=bits(inp.ws_gate), ws_up=bits(inp.ws_up),
                           ws_down=bits(inp.ws_down), ws_gvec=bits(inp.ws_gvec))
    x = inp.x.double()
    out = torch.zeros((cfg.T, cfg.H), dtype=torch.float64)
    for t in range(cfg.T):
        for e in range(cfg.E):
            hits = [j for j in range(r.keff[t]) if r.idx[t, j] == e]
            assert len(hits) <= 1
            if hits:
                y = F.linear(F.silu(F.linear(x[t], inp.w_gate[e].double())) * F.linear(x[t], inp.w_up[e].double()),
                             inp.w_down[e].double())
                out[t] += float(r.w[t, hits[0]]) * y
        s = torch.sigmoid(torch.dot(inp.ws_gvec.double(), x[t]))
        out[t] += s * F.linear(F.silu(F.linear(x[t], inp.ws_gate.double())) * F.linear(x[t], inp.ws_up.double()),
                               inp.ws_down.double())
    np.testing.assert_allclose(r.out, out.numpy(), rtol=1e-9, atol=1e-13)


@pytest.mark.parametrize("N,p", [(0, 0.6), (4, 0.8), (3, 0.0)])
def test_forward_routes_topp_then_budget(oracle_mod, N, p):
    """forward() applies the top-p trim before the budget, and its dense
    output follows the resulting routing."""
    cfg = W.MoEConfig("dense", T=12, H=64, E=6, I=32, k=3, norm_topk=True, budget=N, zipf_alpha=0.5)
    inp = W.make_inputs(cfg, std=0.2)
    r = oracle_mod.forward(bits(inp.x), inp.logits.numpy(), bits(inp.w_gate), bits(inp.w_up), bits(inp.w_down),
                           k=3, budget=N, topp=p)
    idx, w = oracle_mod.route(inp.logits.numpy(), 3)
    i1, w1, _ = oracle_mod.topp(idx, w, p)
    i2, w2, keff, kept, nd = oracle_mod.budget(i1, w1, cfg.E, N)
    assert (r.idx == i2).all() and (r.w.view(np.uint32) == w2.view(np.uint32)).all()
    assert (r.keff == keff).all() and r.n_dropped == nd
    x = inp.x.double()
    out = torch.zeros((cfg.T, cfg.H), dtype=torch.float64)
    for t in range(cfg.T):
        for j in range(int(keff[t])):
            e = int(i2[t, j])
            y = F.linear(F.silu(F.linear(x[t], inp.w_gate[e].double())) * F.linear(x[t], inp.w_up[e].double()),
                         inp.w_down[e].double())
            out[t] += float(w2[t, j]) * y
    np.testing.assert_allclose(r.out, out.numpy(), rtol=1e-9, atol=1e-13)


def test_shared_gate_closed_form(oracle_mod):
    # sigmoid(0) = 1/2 exactly; sigmoid(z) + sigmoid(-z) = 1
    g = bits(_bf([1.0, -2.0, 0.5]))
    x = bits(_bf([[0.0, 0.0, 0.0], [1.0, 0.25, 2.0], [-1.0, -0.25, -2.0]]))
    s = oracle_mod.shared_gate(g, x)
    assert s[0] == 0.5
    assert abs(s[1] + s[2] - 1.0) < 1e-15
    assert abs(s[1] - 1.0 / (1.0 + math.exp(-1.5))) < 1e-15 and s[1] > 0.5   # z = 1 - 0.5 + 1 = 1.5


def test_forward_rows_subset_matches_full(oracle_mod):
    cfg = W.MoEConfig("sub", T=20, H=64, E=8, I=32, k=2, Is=32)
    inp = W.make_inputs(cfg)
    args = (bits(inp.x), inp.logits.numpy(), bits(inp.w_gate), bits(inp.w_up), bits(inp.w_down))
    kw = dict(k=2, ws_gate=bits(inp.ws_gate), ws_up=bits(inp.ws_up), ws_down=bits(inp.ws_down),
              ws_gvec=bits(inp.ws_gvec))
    full = oracle_mod.forward(*args, **kw, nthreads=2)
    rows = np.array([19, 0, 7], np.int32)
    sub = oracle_mod.forward(*args, **kw, rows=rows)
    assert (sub.out == full.out[rows]).all()
