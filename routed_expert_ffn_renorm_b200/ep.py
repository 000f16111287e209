"""Expert parallelism: the routed experts of a layer split over W ranks.

One process per GPU.  Rank r holds the routed experts [r * epr, (r + 1) *
epr), epr = E / W, and the whole shared expert; each rank routes its own
tokens.  The multi-rank MegaMoE of DeepGEMM PR #381 ("B200 performance",
EP8) and DeepGEMM fork PR #5 is the design this follows: a dispatch that
sends every routed token row to the rank holding its expert, the expert
FFN there, and a combine that brings the weighted outputs back.  Here the
two exchanges are NCCL all-to-alls (torch.distributed) over NVLink; every
other step is one of the library's kernels, called through the C ABI:

  home rank:    moe_route -> moe_ep_rank_ids -> moe_dispatch over W "experts"
                (slots grouped by destination rank, rows gathered in that
                order) -> moe_ep_pack (local expert id, weight per row)
  exchange:     rows, local ids and weights to their ranks
  expert rank:  moe_dispatch (k = 1) -> moe_expert_ffn (weighted) ->
                moe_combine (the weighted rows made contiguous)
  exchange:     the weighted rows back, in the order they came
  home rank:    moe_ep_unpack (rows to token order) -> the shared expert
                (moe_expert_ffn with no routed rows) -> moe_combine

Every row is computed by the same kernels on the same operands in the same
order as in moe_forward, so the output is moe_forward's, bit for bit (the
GPU test runs two ranks on one GPU, exchanging in process).  The batch-union
expert budget couples every rank's tokens and is not supported here
(budget must be 0); the top-p trim is per token and is.

The weights may be bf16 (MoEWeights) or block-scaled (MoEWeightsMXFP8,
MoEWeightsNVFP4): the expert FFN calls are then the matching
moe_expert_ffn_mxfp8 / moe_expert_ffn_nvfp4, and the output is
moe_forward_mxfp8's / moe_forward_nvfp4's, bit for bit.

The stage methods (dispatch, experts, combine) do no communication; forward()
puts the exchanges between them.  `exchange` is the only function that talks
to other ranks.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import dataclasses

from . import (MoEConfig, MoEWeights, MoEWeightsMXFP8, MoEWeightsNVFP4, moe_combine, moe_dispatch, moe_ep_pack,
               moe_ep_rank_ids, moe_ep_unpack, moe_expert_ffn, moe_expert_ffn_mxfp8, moe_expert_ffn_nvfp4, moe_route,
               workspace_bytes)

# the expert FFN entry point of each weight type
_FFN = {MoEWeights: moe_expert_ffn, MoEWeightsMXFP8: moe_expert_ffn_mxfp8, MoEWeightsNVFP4: moe_expert_ffn_nvfp4}


def exchange(send_counts: Sequence[int], tensors: Sequence["torch.Tensor"], group=None):
    """All-to-all of variable-size row blocks.  tensors[i] holds
    sum(send_counts) rows, the first send_counts[0] for rank 0, the next for
    rank 1, ...; returns (recv_counts, received tensors), the rows from rank
    0 first.  Every rank must call it with the same number of tensors, in
    the same order (the collectives are matched by order)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    dev = tensors[0].device if tensors else torch.device("cpu")
    sc = torch.tensor(list(send_counts), dtype=torch.int64, device=dev)
    if sc.numel() != world:
        raise ValueError(f"send_counts has {sc.numel()} entries for {world} ranks")
    rc = torch.empty_like(sc)
    dist.all_to_all_single(rc, sc, group=group)
    recv_counts = [int(v) for v in rc.cpu().tolist()]
    out = []
    for t in tensors:
        r = torch.empty((sum(recv_counts),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_to_all_single(r, t.contiguous(), recv_counts, list(send_counts), group=group)
        out.append(r)
    return recv_counts, out


@dataclass
class EPState:
    """What the home rank keeps between dispatch and combine."""
    T: int
    send_counts: List[int]
    idx: "torch.Tensor"      # [T, k] global expert ids after routing
    w: "torch.Tensor"        # [T, k] routing weights
    keff: "torch.Tensor"     # [T] kept slots
    sgate: Optional["torch.Tensor"]
    offsets: "torch.Tensor"  # [W + 1] rows per destination rank, as a prefix sum
    perm: "torch.Tensor"     # [T*k] slot ids in send order
    x: "torch.Tensor"        # the home rank's tokens [T, H]


@dataclass
class EPSend:
    """The rows a home rank sends, grouped by destination rank."""
    counts: List[int]
    rows: "torch.Tensor"       # [n, H] bf16
    local_idx: "torch.Tensor"  # [n] expert id on the destination rank
    local_w: "torch.Tensor"    # [n] routing weight


class EPLayer:
    """One rank's share of an expert-parallel routed-MoE layer.

    cfg: the whole layer (E = all routed experts, budget 0).  weights: this
    rank's routed experts (w_gate, w_up [epr, I, H], w_down [epr, H, I], or
    their codes and scales) and the whole shared expert (and its gate
    vector): MoEWeights, MoEWeightsMXFP8 or MoEWeightsNVFP4 on the device
    (shard_weights cuts them from a whole layer's)."""

    def __init__(self, cfg: MoEConfig, world: int, rank: int, weights):
        import torch
        if cfg.budget:
            raise ValueError("the batch-union expert budget spans every rank's tokens; expert parallelism needs budget 0")
        if world < 1 or cfg.n_routed_experts % world:
            raise ValueError("n_routed_experts must be a multiple of the number of ranks")
        if type(weights) not in _FFN:
            raise TypeError(f"unsupported weight type {type(weights).__name__}")
        self.cfg, self.world, self.rank, self.weights = cfg, world, rank, weights
        self._ffn = _FFN[type(weights)]
        self.epr = cfg.n_routed_experts // world
        if weights.w_gate.shape[0] != self.epr:
            raise ValueError(f"this rank holds {self.epr} experts, got {weights.w_gate.shape[0]}")
        if cfg.shared_intermediate_size and self.epr < cfg.num_experts_per_tok:
            # the shared expert runs as an FFN call over this rank's experts with no routed rows,
            # which takes a config with k <= its expert count
            raise ValueError("with a shared expert each rank must hold at least k experts")
        self.dev = weights.w_gate.device
        # the experts on this rank: k = 1, no shared expert; the shared expert alone
        self.cfg_local = MoEConfig(cfg.hidden, self.epr, cfg.moe_intermediate_size, 1, 0, False, 0, 0.0)
        self.cfg_shared = MoEConfig(cfg.hidden, self.epr, cfg.moe_intermediate_size, cfg.num_experts_per_tok,
                                    cfg.shared_intermediate_size, cfg.norm_topk, 0, cfg.topp)
        self._torch = torch

    def _ws(self, cfg, T):
        ws = self._torch.zeros(workspace_bytes(cfg, max(T, 1)), dtype=self._torch.uint8, device=self.dev)
        return ws

    # -------------------------------------------------------------- stages --
    def dispatch(self, x, logits):
        """Route this rank's tokens and gather the rows to send (no communication)."""
        torch, cfg = self._torch, self.cfg
        T, k, H, W = x.shape[0], cfg.num_experts_per_tok, cfg.hidden, self.world
        dev = self.dev
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        keff = torch.empty(T, dtype=torch.int32, device=dev)
        sgate = torch.empty(T, dtype=torch.float32, device=dev) if cfg.shared_intermediate_size else None
        moe_route(cfg, logits, idx, w, x=x if sgate is not None else None,
                  ws_gate_vec=self.weights.ws_gate_vec if sgate is not None else None, sgate=sgate, keff=keff)
        ridx = torch.empty_like(idx)
        moe_ep_rank_ids(idx, ridx, self.epr)
        # slots grouped by destination rank: a dispatch over max(W, k) "experts" (a
        # dispatch needs k <= E; the ids past W - 1 receive nothing), rows gathered in
        # that order
        Wd = max(W, k)
        cfg_r = MoEConfig(cfg.hidden, Wd, cfg.moe_intermediate_size, k, 0, cfg.norm_topk, 0, 0.0)
        counts = torch.empty(Wd, dtype=torch.int32, device=dev)
        offsets = torch.empty(Wd + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
        slot_pos = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
        x_perm = torch.empty((max(T * k, 1), H), dtype=torch.bfloat16, device=dev)
        ws = self._ws(cfg_r, T)
        moe_dispatch(cfg_r, ridx, counts, offsets, perm, slot_pos, ws, keff=keff, x=x, x_perm=x_perm)
        local_idx = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
        local_w = torch.empty(max(T * k, 1), dtype=torch.float32, device=dev)
        n_dev = offsets[Wd:Wd + 1]
        moe_ep_pack(n_dev, perm, idx, w, local_idx, local_w, self.epr)
        send_counts = [int(v) for v in counts[:W].cpu().tolist()]  # the exchange needs its sizes on the host
        n = sum(send_counts)
        state = EPState(T, send_counts, idx, w, keff, sgate, offsets[:W + 1], perm, x)
        return state, EPSend(send_counts, x_perm[:n], local_idx[:n], local_w[:n])

    def experts(self, rows, local_idx, local_w):
        """The FFN of this rank's experts on received rows; returns the weighted
        output rows, contiguous, in the order received (no communication)."""
        torch, cfg = self._torch, self.cfg_local
        R, H, dev = rows.shape[0], cfg.hidden, self.dev
        out = torch.empty((R, H), dtype=torch.bfloat16, device=dev)
        if R == 0:
            return out
        idx = local_idx.reshape(R, 1).contiguous()
        w = local_w.reshape(R, 1).contiguous()
        E = self.epr
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(R, dtype=torch.int32, device=dev)
        slot_pos = torch.empty(R, dtype=torch.int32, device=dev)
        x_perm = torch.empty((R, H), dtype=torch.bfloat16, device=dev)
        ybuf = torch.empty((R, 2, H), dtype=torch.bfloat16, device=dev)
        ws = self._ws(cfg, R)
        moe_dispatch(cfg, idx, counts, offsets, perm, slot_pos, ws, x=rows, x_perm=x_perm)
        self._ffn(cfg, rows, x_perm, offsets, perm, w, self.weights, ybuf, ws)
        moe_combine(cfg, ybuf, out)  # k = 1, no shared expert: row r = ybuf[r, 0], exactly
        return out

    def combine(self, state: EPState, returned):
        """Returned weighted rows (send order) to token order, plus the shared
        expert, summed per token (no communication)."""
        torch, cfg = self._torch, self.cfg
        T, k, H, dev = state.T, cfg.num_experts_per_tok, cfg.hidden, self.dev
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        if T == 0:
            return out
        ybuf = torch.empty((T, k + 1, H), dtype=torch.bfloat16, device=dev)
        if returned.shape[0]:
            moe_ep_unpack(cfg, T, state.offsets[self.world:self.world + 1], state.perm, returned, ybuf)
        if cfg.shared_intermediate_size:
            # the shared expert alone: no routed rows (all dispatch offsets zero)
            cs = self.cfg_shared
            ws = self._ws(cs, T)
            zero_off = torch.zeros(self.epr + 1, dtype=torch.int32, device=dev)
            x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
            self._ffn(cs, state.x, x_perm, zero_off, state.perm, state.w, self.weights, ybuf, ws,
                      sgate=state.sgate)
        moe_combine(cfg, ybuf, out, keff=state.keff)
        return out

    # ------------------------------------------------------------- forward --
    def forward(self, x, logits, group=None):
        """The layer on this rank's tokens: dispatch, exchange, experts,
        exchange back, combine.  Every rank of the group calls it."""
        state, send = self.dispatch(x, logits)
        recv_counts, (rows, lidx, lw) = exchange(send.counts, [send.rows, send.local_idx, send.local_w], group)
        done = self.experts(rows, lidx, lw)
        _, (back,) = exchange(recv_counts, [done], group)
        return self.combine(state, back)


def shard_weights(weights, world: int, rank: int):
    """Rank `rank`'s share of a whole layer's weights: its routed experts
    (contiguous views, no copy) and the whole shared expert.  Works for every
    weight type: the routed arrays (w_gate, w_up, w_down and, block-scaled,
    their packed scales and matrix scales) all lead with the expert index --
    the packed scale layout keeps each expert's rows in a contiguous run of
    64-row groups, as many bytes as its [I, K / block] slice."""
    E = weights.w_gate.shape[0]
    epr = E // world
    sl = slice(rank * epr, (rank + 1) * epr)
    routed = {f.name: getattr(weights, f.name)[sl] for f in dataclasses.fields(weights)
              if f.name.startswith("w_") and f.name != "w_router" and getattr(weights, f.name) is not None}
    return dataclasses.replace(weights, **routed)
