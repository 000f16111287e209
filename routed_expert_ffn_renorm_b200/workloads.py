"""Seeded synthetic inputs for the routed-MoE FFN layer.

This module only draws random numbers and lays them out; it holds none of
the layer's arithmetic.  The CUDA path (through the binding) and the CPU
oracle (in the tests and the benchmark's CPU leg) are both fed from here.

Recipe (the same for every workload):
  * draw order: x, logits, W_gate, W_up, W_down, shared W_gate, W_up,
    W_down, shared gate vector -- all from one torch.Generator seeded with
    ``seed`` on the chosen device;
  * x and every weight ~ N(0, 0.02) drawn in fp32, rounded once to bf16;
  * with a router projection (``router=True``), W_r [E, H] ~ N(0, 1 / (std
    sqrt(H))) drawn last, so that x . W_r^T is about N(0, 1) like the
    given logits;
  * router logits ~ N(0, 1) in fp32, plus a per-expert popularity bias
    -alpha * ln(e + 1) (Zipf popularity 1/(e+1)^alpha; alpha = 0 is uniform
    routing).  The skew knob follows the "--skew-alpha" Zipf router bias of
    DeepGEMM PR #381 ("Validation"), whose exact form the page leaves open.

The workload shapes follow the pages' own workloads: the drafter layers of
SpecForge PR #943 (7-token DSpark blocks x 32 requests = 224 tokens,
16 x 1024 top-2 and 512 x 512 top-10 experts, shared expert 2048), the
256-expert top-8 layer of DeepGEMM PR #381 ("B200 performance"), and the
32-position batch union of colibri issue_budget.md.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int            # tokens in the batch
    H: int            # hidden
    E: int            # n_routed_experts
    I: int            # moe_intermediate_size
    k: int            # num_experts_per_tok
    Is: int = 0       # shared-expert intermediate size (0 = none)
    norm_topk: bool = True
    budget: int = 0   # EXPERT_BUDGET (0 = off)
    zipf_alpha: float = 0.0
    topp: float = 0.0  # per-token top-p trim (0 = off)
    router_proj: bool = False  # logits from the router projection x . W_r^T instead of given
    seed: int = 0

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    @property
    def label(self) -> str:
        s = f"{self.name}:T{self.T}_H{self.H}_E{self.E}_I{self.I}_k{self.k}"
        if self.Is:
            s += f"_Is{self.Is}"
        if self.budget:
            s += f"_N{self.budget}"
        if self.zipf_alpha:
            s += f"_a{self.zipf_alpha:g}"
        if self.topp:
            s += f"_p{self.topp:g}"
        if self.router_proj:
            s += "_proj"
        return s


# The named workloads.
TINY = MoEConfig("tiny", T=16, H=256, E=8, I=128, k=2)
DRAFTER_16x1024 = MoEConfig("drafter_16x1024", T=224, H=5120, E=16, I=1024, k=2, Is=2048)
DRAFTER_512x512 = MoEConfig("drafter_512x512", T=224, H=5120, E=512, I=512, k=10, Is=2048, zipf_alpha=1.0)
LARGE_256E = MoEConfig("large_256e", T=16384, H=7168, E=256, I=2048, k=8)  # T swept over LARGE_T_SWEEP
BUDGET_S32 = MoEConfig("budget_s32", T=32, H=4096, E=128, I=1536, k=8, budget=12, zipf_alpha=1.2)

WORKLOADS = {c.name: c for c in (TINY, DRAFTER_16x1024, DRAFTER_512x512, LARGE_256E, BUDGET_S32)}
LARGE_T_SWEEP = (64, 512, 4096, 16384)
LARGE_ALPHAS = (0.0, 1.0, 1.5)
BUDGETS = (4, 12, 24)


@dataclass
class MoEInputs:
    x: torch.Tensor          # [T, H] bf16
    logits: torch.Tensor     # [T, E] f32
    w_gate: torch.Tensor     # [E, I, H] bf16
    w_up: torch.Tensor       # [E, I, H] bf16
    w_down: torch.Tensor     # [E, H, I] bf16
    ws_gate: Optional[torch.Tensor] = None   # [Is, H] bf16
    ws_up: Optional[torch.Tensor] = None     # [Is, H] bf16
    ws_down: Optional[torch.Tensor] = None   # [H, Is] bf16
    ws_gvec: Optional[torch.Tensor] = None   # [H] bf16
    w_router: Optional[torch.Tensor] = None  # [E, H] bf16 (router projection)


def zipf_bias(E: int, alpha: float, device="cpu") -> torch.Tensor:
    """Log-popularity bias -alpha * ln(e + 1) for e = 0..E-1 (fp32)."""
    e = torch.arange(E, dtype=torch.float64, device=device)
    return (-alpha * torch.log1p(e)).to(torch.float32)


def _normal_bf16(shape, std, gen, device):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def make_inputs(cfg: MoEConfig, device="cpu", seed: Optional[int] = None, std: float = 0.02,
                gate_std: Optional[float] = None, router: bool = False) -> MoEInputs:
    """Draw one seeded input set for ``cfg`` on ``device``.

    Large expert tensors are drawn one expert at a time so that the fp32
    temporaries stay small."""
    seed = cfg.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, H, E, I = cfg.T, cfg.H, cfg.E, cfg.I
    x = _normal_bf16((T, H), std, gen, device)
    logits = torch.randn((T, E), generator=gen, device=device, dtype=torch.float32)
    if cfg.zipf_alpha:
        logits = logits + zipf_bias(E, cfg.zipf_alpha, device)
    w_gate = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    w_up = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    w_down = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
    for e in range(E):
        w_gate[e] = _normal_bf16((I, H), std, gen, device)
    for e in range(E):
        w_up[e] = _normal_bf16((I, H), std, gen, device)
    for e in range(E):
        w_down[e] = _normal_bf16((H, I), std, gen, device)
    inp = MoEInputs(x, logits, w_gate, w_up, w_down)
    if cfg.Is:
        inp.ws_gate = _normal_bf16((cfg.Is, H), std, gen, device)
        inp.ws_up = _normal_bf16((cfg.Is, H), std, gen, device)
        inp.ws_down = _normal_bf16((H, cfg.Is), std, gen, device)
        inp.ws_gvec = _normal_bf16((H,), std if gate_std is None else gate_std, gen, device)
    if router or cfg.router_proj:
        inp.w_router = _normal_bf16((E, H), 1.0 / (std * math.sqrt(H)), gen, device)
    return inp


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")

