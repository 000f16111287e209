"""B200 (sm_100a) routed Mixture-of-Experts FFN forward.

Thin Python binding over the C ABI of ``libmoe.so`` (declared in
``include/moe.h``): the functions below have the C entry points' names and
only marshal arguments -- torch tensors in, device pointers and the current
CUDA stream out.  Every step of the layer runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and a missing or unbuildable
library raises.

    cfg = MoEConfig(hidden=5120, n_routed_experts=16, moe_intermediate_size=1024,
                    num_experts_per_tok=2, shared_intermediate_size=2048)
    ws = torch.empty(workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    status_clear(ws)
    moe_forward(cfg, x, logits, weights, out, ws)
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

__all__ = [
    "MoEConfig", "MoEWeights", "MoEError", "load_library", "workspace_bytes", "moe_router_logits", "moe_route",
    "moe_budget",
    "moe_dispatch", "moe_expert_ffn", "moe_expert_gate_up", "moe_expert_down", "moe_expert_ffn_noalloc",
    "moe_combine", "moe_forward", "moe_quantize_mxfp8", "moe_quantize_nvfp4",
    "MoEWeightsMXFP8", "moe_mxfp8_pack_scales", "moe_expert_ffn_mxfp8", "moe_forward_mxfp8", "pack_mxfp8",
    "MoEWeightsNVFP4", "moe_nvfp4_pack_scales", "moe_expert_ffn_nvfp4", "moe_forward_nvfp4", "pack_nvfp4",
    "moe_ep_rank_ids", "moe_ep_pack", "moe_ep_unpack",
    "status_read", "status_clear",
    "EXPORTED_SYMBOLS", "MOE_STATUS_TIMEOUT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libmoe_checked.so")  # built with MOE_DEBUG_BOUNDS

EXPORTED_SYMBOLS = (
    "moe_workspace_bytes", "moe_route", "moe_budget", "moe_dispatch", "moe_expert_ffn", "moe_combine",
    "moe_forward", "moe_status_read", "moe_status_clear", "moe_error_string", "moe_expert_gate_up",
    "moe_expert_down", "moe_expert_ffn_noalloc", "moe_router_logits", "moe_quantize_mxfp8", "moe_quantize_nvfp4",
    "moe_mxfp8_pack_scales", "moe_expert_ffn_mxfp8", "moe_forward_mxfp8",
    "moe_nvfp4_pack_scales", "moe_expert_ffn_nvfp4", "moe_forward_nvfp4",
    "moe_ep_rank_ids", "moe_ep_pack", "moe_ep_unpack",
)
NOALLOC_SCRATCH_BYTES = 8 << 20  # MOE_NOALLOC_SCRATCH_BYTES
MOE_STATUS_TIMEOUT = 1
MOE_STATUS_BOUNDS = 2
MOE_STATUS_NONFINITE = 4


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (code {code})")
        self.code = code


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "hidden", "n_routed_experts", "moe_intermediate_size", "num_experts_per_tok",
        "shared_intermediate_size", "norm_topk", "budget")] + [("topp", ctypes.c_float)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down", "ws_gate_vec", "w_router")]


class _WeightsMXFP8(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "w_gate_scale", "w_up_scale", "w_down_scale", "ws_gate", "ws_up", "ws_down",
        "ws_gate_scale", "ws_up_scale", "ws_down_scale", "ws_gate_vec", "w_router")]


class _WeightsNVFP4(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "w_gate_scale", "w_up_scale", "w_down_scale", "w_gate_tscale", "w_up_tscale",
        "w_down_tscale", "ws_gate", "ws_up", "ws_down", "ws_gate_scale", "ws_up_scale", "ws_down_scale",
        "ws_tscale", "ws_gate_vec", "w_router")]


class _Aux(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "topk_w", "sgate", "keff", "expert_kept", "n_dropped", "counts", "offsets", "perm",
        "slot_pos", "logits")]


@dataclass(frozen=True)
class MoEConfig:
    """The layer's configuration keys (names as in the drafter config files)."""
    hidden: int
    n_routed_experts: int
    moe_intermediate_size: int
    num_experts_per_tok: int
    shared_intermediate_size: int = 0
    norm_topk: bool = True
    budget: int = 0
    topp: float = 0.0  # per-token top-p trim; 0 (or >= 1) = off

    def _c(self) -> _Config:
        return _Config(self.hidden, self.n_routed_experts, self.moe_intermediate_size, self.num_experts_per_tok,
                       self.shared_intermediate_size, int(bool(self.norm_topk)), self.budget, float(self.topp))


@dataclass
class MoEWeights:
    """Device bf16 weights: w_gate, w_up [E, I, H]; w_down [E, H, I];
    optional shared expert ws_gate, ws_up [Is, H], ws_down [H, Is], ws_gate_vec [H];
    optional router projection w_router [E, H] (used when moe_forward gets no logits)."""
    w_gate: "torch.Tensor"
    w_up: "torch.Tensor"
    w_down: "torch.Tensor"
    ws_gate: Optional["torch.Tensor"] = None
    ws_up: Optional["torch.Tensor"] = None
    ws_down: Optional["torch.Tensor"] = None
    ws_gate_vec: Optional["torch.Tensor"] = None
    w_router: Optional["torch.Tensor"] = None

    def _c(self) -> _Weights:
        return _Weights(*(_ptr(getattr(self, n), allow_none=True) for n in (
            "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down", "ws_gate_vec", "w_router")))


@dataclass
class MoEWeightsMXFP8:
    """Device MXFP8 expert weights: E4M3 codes (uint8) in the bf16 weights'
    shapes -- w_gate, w_up [E, I, H], w_down [E, H, I], optional shared
    ws_gate, ws_up [Is, H], ws_down [H, Is] -- and each matrix's UE8M0 scales
    in the FFN's packed layout (moe_mxfp8_pack_scales); ws_gate_vec [H] and
    w_router [E, H] stay bf16.  pack_mxfp8() builds one from MoEWeights."""
    w_gate: "torch.Tensor"
    w_up: "torch.Tensor"
    w_down: "torch.Tensor"
    w_gate_scale: "torch.Tensor"
    w_up_scale: "torch.Tensor"
    w_down_scale: "torch.Tensor"
    ws_gate: Optional["torch.Tensor"] = None
    ws_up: Optional["torch.Tensor"] = None
    ws_down: Optional["torch.Tensor"] = None
    ws_gate_scale: Optional["torch.Tensor"] = None
    ws_up_scale: Optional["torch.Tensor"] = None
    ws_down_scale: Optional["torch.Tensor"] = None
    ws_gate_vec: Optional["torch.Tensor"] = None
    w_router: Optional["torch.Tensor"] = None

    def _c(self) -> _WeightsMXFP8:
        return _WeightsMXFP8(*(_ptr(getattr(self, n), allow_none=True) for n, _ in _WeightsMXFP8._fields_))


@dataclass
class MoEWeightsNVFP4:
    """Device NVFP4 expert weights: E2M1 codes (uint8, two per byte, the
    lower K in the low nibble) -- w_gate, w_up [E, I, H // 2], w_down
    [E, H, I // 2], optional shared ws_gate, ws_up [Is, H // 2], ws_down
    [H, Is // 2] -- each matrix's E4M3 block scales in the FFN's packed
    layout (moe_nvfp4_pack_scales), and the fp32 matrix scales: w_*_tscale
    [E] and ws_tscale [3] (shared gate, up, down).  ws_gate_vec [H] and
    w_router [E, H] stay bf16.  pack_nvfp4() builds one from MoEWeights."""
    w_gate: "torch.Tensor"
    w_up: "torch.Tensor"
    w_down: "torch.Tensor"
    w_gate_scale: "torch.Tensor"
    w_up_scale: "torch.Tensor"
    w_down_scale: "torch.Tensor"
    w_gate_tscale: "torch.Tensor"
    w_up_tscale: "torch.Tensor"
    w_down_tscale: "torch.Tensor"
    ws_gate: Optional["torch.Tensor"] = None
    ws_up: Optional["torch.Tensor"] = None
    ws_down: Optional["torch.Tensor"] = None
    ws_gate_scale: Optional["torch.Tensor"] = None
    ws_up_scale: Optional["torch.Tensor"] = None
    ws_down_scale: Optional["torch.Tensor"] = None
    ws_tscale: Optional["torch.Tensor"] = None
    ws_gate_vec: Optional["torch.Tensor"] = None
    w_router: Optional["torch.Tensor"] = None

    def _c(self) -> _WeightsNVFP4:
        return _WeightsNVFP4(*(_ptr(getattr(self, n), allow_none=True) for n, _ in _WeightsNVFP4._fields_))


_lib = None
_checked = None
_lock = threading.Lock()


def load_library(build_if_stale: bool = True, variant: str = "release"):
    """Load libmoe.so (building it first when missing or older than its
    sources).  variant="checked" loads libmoe_checked.so instead, the same
    library built with MOE_DEBUG_BOUNDS (range checks on the caller's index
    inputs, reported as MOE_STATUS_BOUNDS); the functions below always call
    the release library unless a test swaps it in."""
    global _lib, _checked
    with _lock:
        if variant == "release" and _lib is not None:
            return _lib
        if variant == "checked" and _checked is not None:
            return _checked
        path = LIB_PATH if variant == "release" else CHECKED_LIB_PATH
        if build_if_stale:
            from . import _build
            if _build.stale(variant):
                _build.build(variant=variant)
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m routed_expert_ffn_renorm_b200._build`")
        lib = ctypes.CDLL(path)
        P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        cfg = ctypes.POINTER(_Config)
        lib.moe_workspace_bytes.restype = sz
        lib.moe_workspace_bytes.argtypes = [cfg, i32]
        lib.moe_route.argtypes = [cfg, i32, P, P, P, P, P, P, P, P]
        lib.moe_router_logits.argtypes = [cfg, i32, P, P, P, P, sz, P]
        lib.moe_budget.argtypes = [cfg, i32, P, P, P, P, P, P, sz, P]
        lib.moe_dispatch.argtypes = [cfg, i32, P, P, P, P, P, P, P, P, P, sz, P]
        lib.moe_expert_ffn.argtypes = [cfg, i32, P, P, P, P, P, P, ctypes.POINTER(_Weights), P, P, sz, P]
        lib.moe_combine.argtypes = [cfg, i32, P, P, P, P]
        lib.moe_expert_gate_up.argtypes = [cfg, i32, P, P, P, ctypes.POINTER(_Weights), P, sz, P]
        lib.moe_expert_down.argtypes = [cfg, i32, P, P, P, P, ctypes.POINTER(_Weights), P, P, sz, P]
        lib.moe_expert_ffn_noalloc.argtypes = [cfg, i32, P, P, P, P, P, P, ctypes.POINTER(_Weights), P, P, P]
        lib.moe_forward.argtypes = [cfg, i32, P, P, ctypes.POINTER(_Weights), P, ctypes.POINTER(_Aux), P, sz, P]
        lib.moe_status_read.argtypes = [P, ctypes.POINTER(i32), P]
        lib.moe_status_clear.argtypes = [P, P]
        i64 = ctypes.c_int64
        lib.moe_quantize_mxfp8.argtypes = [i64, i32, P, P, P, P]
        lib.moe_quantize_nvfp4.argtypes = [i32, i64, i32, P, P, P, P, P]
        lib.moe_mxfp8_pack_scales.argtypes = [i64, i32, P, P, P]
        lib.moe_ep_rank_ids.argtypes = [i32, i32, i32, P, P, P]
        lib.moe_ep_pack.argtypes = [i32, P, i32, P, P, P, P, P, P]
        lib.moe_ep_unpack.argtypes = [cfg, i32, i32, P, P, P, P, P]
        lib.moe_expert_ffn_mxfp8.argtypes = [cfg, i32, P, P, P, P, P, P, ctypes.POINTER(_WeightsMXFP8), P, P, sz, P]
        lib.moe_forward_mxfp8.argtypes = [cfg, i32, P, P, ctypes.POINTER(_WeightsMXFP8), P, ctypes.POINTER(_Aux), P,
                                          sz, P]
        lib.moe_nvfp4_pack_scales.argtypes = [i64, i32, P, P, P]
        lib.moe_expert_ffn_nvfp4.argtypes = [cfg, i32, P, P, P, P, P, P, ctypes.POINTER(_WeightsNVFP4), P, P, sz, P]
        lib.moe_forward_nvfp4.argtypes = [cfg, i32, P, P, ctypes.POINTER(_WeightsNVFP4), P, ctypes.POINTER(_Aux), P,
                                          sz, P]
        lib.moe_error_string.restype = ctypes.c_char_p
        lib.moe_error_string.argtypes = [ctypes.c_int]
        for name in EXPORTED_SYMBOLS:
            if name not in ("moe_workspace_bytes", "moe_error_string"):
                getattr(lib, name).restype = ctypes.c_int
        if variant == "release":
            _lib = lib
        else:
            _checked = lib
        return lib


def _ptr(t, allow_none: bool = False):
    if t is None:
        if allow_none:
            return None
        raise ValueError("tensor argument is None")
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"expected a torch.Tensor, got {type(t).__name__}")
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _expect(t, dtype, numel: int, name: str):
    """Host-side size check of a tensor the library writes or reads in full:
    a wrong dtype or a short buffer would otherwise become an out-of-bounds
    device access."""
    if t.dtype != dtype or t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements of {dtype}, got {t.numel()} of {t.dtype}")


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, rc: int):
    if rc != 0:
        msg = load_library().moe_error_string(rc).decode()
        raise MoEError(fn, rc, msg)


def workspace_bytes(cfg: MoEConfig, T: int) -> int:
    n = load_library().moe_workspace_bytes(ctypes.byref(cfg._c()), T)
    if n == 0:
        raise MoEError("moe_workspace_bytes", -1, "invalid configuration")
    return int(n)


def moe_router_logits(cfg: MoEConfig, x, w_router, logits, ws, stream=None):
    """logits [T, E] f32 = x [T, H] . w_router [E, H]^T on the tensor cores."""
    T = x.shape[0]
    _check("moe_router_logits", load_library().moe_router_logits(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(w_router), _ptr(logits), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_quantize_mxfp8(w, codes, scales, stream=None):
    """MXFP8 weights: w [..., K] bf16 -> codes [..., K] uint8 (E4M3) and
    scales [..., K // 32] uint8 (UE8M0), blocks along the last axis."""
    import torch
    K = w.shape[-1]
    _expect(w, torch.bfloat16, w.numel(), "w")
    _expect(codes, torch.uint8, w.numel(), "codes")
    _expect(scales, torch.uint8, w.numel() // 32, "scales")
    _check("moe_quantize_mxfp8", load_library().moe_quantize_mxfp8(
        w.numel() // K, K, _ptr(w), _ptr(codes), _ptr(scales), _stream(stream)))


def moe_quantize_nvfp4(w, codes, scales, tensor_scale, stream=None):
    """NVFP4 weights: w [nmat, rows, K] bf16 -> codes [nmat, rows, K // 2]
    uint8 (two E2M1 per byte, element 2i low), scales [nmat, rows, K // 16]
    uint8 (E4M3), tensor_scale [nmat] fp32 (one per matrix)."""
    import torch
    nmat, rows, K = w.shape
    _expect(w, torch.bfloat16, w.numel(), "w")
    _expect(codes, torch.uint8, w.numel() // 2, "codes")
    _expect(scales, torch.uint8, w.numel() // 16, "scales")
    _expect(tensor_scale, torch.float32, nmat, "tensor_scale")
    _check("moe_quantize_nvfp4", load_library().moe_quantize_nvfp4(
        nmat, rows, K, _ptr(w), _ptr(codes), _ptr(scales), _ptr(tensor_scale), _stream(stream)))


def moe_mxfp8_pack_scales(scales, packed, stream=None):
    """MXFP8 scales [rows, K // 32] uint8 -> the FFN's layout
    [rows / 64][K / 128][64][4] (rows % 64 == 0, K % 128 == 0)."""
    import torch
    kb = scales.shape[-1]
    _expect(scales, torch.uint8, scales.numel(), "scales")
    _expect(packed, torch.uint8, scales.numel(), "packed")
    _check("moe_mxfp8_pack_scales", load_library().moe_mxfp8_pack_scales(
        scales.numel() // kb, kb * 32, _ptr(scales), _ptr(packed), _stream(stream)))


def pack_mxfp8(weights: MoEWeights, stream=None) -> MoEWeightsMXFP8:
    """Quantise every expert matrix of `weights` to MXFP8 on the GPU
    (moe_quantize_mxfp8, then moe_mxfp8_pack_scales); the gate vector and
    the router projection are passed through.  Allocates the outputs."""
    import torch

    def one(w):
        codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
        scales = torch.empty(w.shape[:-1] + (w.shape[-1] // 32,), dtype=torch.uint8, device=w.device)
        moe_quantize_mxfp8(w, codes, scales, stream=stream)
        packed = torch.empty_like(scales)
        moe_mxfp8_pack_scales(scales, packed, stream=stream)
        return codes, packed

    (g, gs), (u, us), (d, ds) = one(weights.w_gate), one(weights.w_up), one(weights.w_down)
    out = MoEWeightsMXFP8(g, u, d, gs, us, ds, ws_gate_vec=weights.ws_gate_vec, w_router=weights.w_router)
    if weights.ws_gate is not None:
        (out.ws_gate, out.ws_gate_scale), (out.ws_up, out.ws_up_scale), (out.ws_down, out.ws_down_scale) = (
            one(weights.ws_gate), one(weights.ws_up), one(weights.ws_down))
    return out


def moe_expert_ffn_mxfp8(cfg: MoEConfig, x, x_perm, offsets, perm, topk_w, weights: MoEWeightsMXFP8, ybuf, ws, *,
                         sgate=None, stream=None):
    """moe_expert_ffn with MXFP8 expert weights."""
    T = x.shape[0]
    w = weights._c()
    _check("moe_expert_ffn_mxfp8", load_library().moe_expert_ffn_mxfp8(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(x_perm), _ptr(offsets), _ptr(perm), _ptr(topk_w),
        _ptr(sgate, True), ctypes.byref(w), _ptr(ybuf), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_forward_mxfp8(cfg: MoEConfig, x, logits, weights: MoEWeightsMXFP8, out, ws, *, aux: Optional[dict] = None,
                      stream=None):
    """moe_forward with MXFP8 expert weights (arguments as moe_forward)."""
    T = x.shape[0]
    w = weights._c()
    a = _Aux()
    if aux:
        for name, t in aux.items():
            setattr(a, name, _ptr(t))
    _check("moe_forward_mxfp8", load_library().moe_forward_mxfp8(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(logits, True), ctypes.byref(w), _ptr(out), ctypes.byref(a),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_nvfp4_pack_scales(scales, packed, stream=None):
    """NVFP4 block scales [rows, K // 16] uint8 -> the FFN's layout
    [rows / 64][K / 128][64][8] (rows % 64 == 0, K % 128 == 0)."""
    import torch
    kb = scales.shape[-1]
    _expect(scales, torch.uint8, scales.numel(), "scales")
    _expect(packed, torch.uint8, scales.numel(), "packed")
    _check("moe_nvfp4_pack_scales", load_library().moe_nvfp4_pack_scales(
        scales.numel() // kb, kb * 16, _ptr(scales), _ptr(packed), _stream(stream)))


def pack_nvfp4(weights: MoEWeights, stream=None) -> MoEWeightsNVFP4:
    """Quantise every expert matrix of `weights` to NVFP4 on the GPU
    (moe_quantize_nvfp4 with one matrix scale per expert matrix, then
    moe_nvfp4_pack_scales); the gate vector and the router projection are
    passed through.  Allocates the outputs."""
    import torch

    def one(w, tscale):
        w3 = w.reshape((-1,) + tuple(w.shape[-2:]))
        codes = torch.empty(w.shape[:-1] + (w.shape[-1] // 2,), dtype=torch.uint8, device=w.device)
        scales = torch.empty(w.shape[:-1] + (w.shape[-1] // 16,), dtype=torch.uint8, device=w.device)
        moe_quantize_nvfp4(w3, codes, scales, tscale, stream=stream)
        packed = torch.empty_like(scales)
        moe_nvfp4_pack_scales(scales, packed, stream=stream)
        return codes, packed

    E = weights.w_gate.shape[0]
    ts = torch.empty(3, E, dtype=torch.float32, device=weights.w_gate.device)
    (g, gs), (u, us), (d, ds) = (one(weights.w_gate, ts[0]), one(weights.w_up, ts[1]), one(weights.w_down, ts[2]))
    out = MoEWeightsNVFP4(g, u, d, gs, us, ds, ts[0], ts[1], ts[2], ws_gate_vec=weights.ws_gate_vec,
                          w_router=weights.w_router)
    if weights.ws_gate is not None:
        out.ws_tscale = torch.empty(3, dtype=torch.float32, device=weights.ws_gate.device)
        (out.ws_gate, out.ws_gate_scale), (out.ws_up, out.ws_up_scale), (out.ws_down, out.ws_down_scale) = (
            one(weights.ws_gate, out.ws_tscale[0:1]), one(weights.ws_up, out.ws_tscale[1:2]),
            one(weights.ws_down, out.ws_tscale[2:3]))
    return out


def moe_expert_ffn_nvfp4(cfg: MoEConfig, x, x_perm, offsets, perm, topk_w, weights: MoEWeightsNVFP4, ybuf, ws, *,
                         sgate=None, stream=None):
    """moe_expert_ffn with NVFP4 expert weights."""
    T = x.shape[0]
    w = weights._c()
    _check("moe_expert_ffn_nvfp4", load_library().moe_expert_ffn_nvfp4(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(x_perm), _ptr(offsets), _ptr(perm), _ptr(topk_w),
        _ptr(sgate, True), ctypes.byref(w), _ptr(ybuf), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_forward_nvfp4(cfg: MoEConfig, x, logits, weights: MoEWeightsNVFP4, out, ws, *, aux: Optional[dict] = None,
                      stream=None):
    """moe_forward with NVFP4 expert weights (arguments as moe_forward)."""
    T = x.shape[0]
    w = weights._c()
    a = _Aux()
    if aux:
        for name, t in aux.items():
            setattr(a, name, _ptr(t))
    _check("moe_forward_nvfp4", load_library().moe_forward_nvfp4(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(logits, True), ctypes.byref(w), _ptr(out), ctypes.byref(a),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_ep_rank_ids(topk_idx, rank_idx, experts_per_rank: int, stream=None):
    """rank_idx = topk_idx // experts_per_rank (-1 stays -1): the rank holding each slot's expert."""
    T, k = topk_idx.shape
    _check("moe_ep_rank_ids", load_library().moe_ep_rank_ids(T, k, experts_per_rank, _ptr(topk_idx), _ptr(rank_idx),
                                                             _stream(stream)))


def moe_ep_pack(n_sent, perm, topk_idx, topk_w, local_idx, local_w, experts_per_rank: int, stream=None):
    """For the first n_sent[0] (device) entries p of perm: local_idx[p] =
    topk_idx[perm[p]] % experts_per_rank, local_w[p] = topk_w[perm[p]]."""
    _check("moe_ep_pack", load_library().moe_ep_pack(
        local_idx.numel(), _ptr(n_sent), experts_per_rank, _ptr(perm), _ptr(topk_idx), _ptr(topk_w), _ptr(local_idx),
        _ptr(local_w), _stream(stream)))


def moe_ep_unpack(cfg: MoEConfig, T: int, n_returned, perm, rows, ybuf, stream=None):
    """ybuf[s + s // k] = rows[p] for p < n_returned[0] (device), s = perm[p]."""
    _check("moe_ep_unpack", load_library().moe_ep_unpack(
        ctypes.byref(cfg._c()), T, rows.shape[0], _ptr(n_returned), _ptr(perm), _ptr(rows), _ptr(ybuf),
        _stream(stream)))


def moe_route(cfg: MoEConfig, logits, topk_idx, topk_w, *, x=None, ws_gate_vec=None, sgate=None, keff=None,
              stream=None):
    T = logits.shape[0]
    _check("moe_route", load_library().moe_route(
        ctypes.byref(cfg._c()), T, _ptr(logits), _ptr(x, True), _ptr(ws_gate_vec, True), _ptr(topk_idx),
        _ptr(topk_w), _ptr(sgate, True), _ptr(keff, True), _stream(stream)))


def moe_budget(cfg: MoEConfig, topk_idx, topk_w, keff, expert_kept, n_dropped, ws, stream=None):
    T = topk_idx.shape[0]
    _check("moe_budget", load_library().moe_budget(
        ctypes.byref(cfg._c()), T, _ptr(topk_idx), _ptr(topk_w), _ptr(keff), _ptr(expert_kept), _ptr(n_dropped),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_dispatch(cfg: MoEConfig, topk_idx, counts, offsets, perm, slot_pos, ws, *, keff=None, x=None, x_perm=None,
                 stream=None):
    T = topk_idx.shape[0]
    _check("moe_dispatch", load_library().moe_dispatch(
        ctypes.byref(cfg._c()), T, _ptr(topk_idx), _ptr(keff, True), _ptr(x, True), _ptr(counts), _ptr(offsets),
        _ptr(perm), _ptr(slot_pos), _ptr(x_perm, True), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_expert_ffn(cfg: MoEConfig, x, x_perm, offsets, perm, topk_w, weights: MoEWeights, ybuf, ws, *, sgate=None,
                   stream=None):
    T = x.shape[0]
    w = weights._c()
    _check("moe_expert_ffn", load_library().moe_expert_ffn(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(x_perm), _ptr(offsets), _ptr(perm), _ptr(topk_w),
        _ptr(sgate, True), ctypes.byref(w), _ptr(ybuf), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_expert_gate_up(cfg: MoEConfig, x, x_perm, offsets, weights: MoEWeights, ws, stream=None):
    T = x.shape[0]
    w = weights._c()
    _check("moe_expert_gate_up", load_library().moe_expert_gate_up(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(x_perm), _ptr(offsets), ctypes.byref(w), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_expert_down(cfg: MoEConfig, T: int, offsets, perm, topk_w, weights: MoEWeights, ybuf, ws, *, sgate=None,
                    stream=None):
    w = weights._c()
    _check("moe_expert_down", load_library().moe_expert_down(
        ctypes.byref(cfg._c()), T, _ptr(offsets), _ptr(perm), _ptr(topk_w), _ptr(sgate, True), ctypes.byref(w),
        _ptr(ybuf), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_expert_ffn_noalloc(cfg: MoEConfig, x, x_perm, offsets, perm, topk_w, weights: MoEWeights, ybuf, *,
                           sgate=None, device_status=None, stream=None):
    """moe_expert_ffn without a workspace, for callers that cannot allocate
    device memory: the scratch lives in a fixed 8 MiB device array inside the
    library (batches needing more raise MoEError with code -3).  Calls whose
    work overlaps on the GPU share that array and must not run concurrently."""
    T = x.shape[0]
    w = weights._c()
    _check("moe_expert_ffn_noalloc", load_library().moe_expert_ffn_noalloc(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(x_perm), _ptr(offsets), _ptr(perm), _ptr(topk_w), _ptr(sgate, True),
        ctypes.byref(w), _ptr(ybuf), _ptr(device_status, True), _stream(stream)))


def moe_combine(cfg: MoEConfig, ybuf, out, *, keff=None, stream=None):
    T = out.shape[0]
    _check("moe_combine", load_library().moe_combine(
        ctypes.byref(cfg._c()), T, _ptr(ybuf), _ptr(keff, True), _ptr(out), _stream(stream)))


def moe_forward(cfg: MoEConfig, x, logits, weights: MoEWeights, out, ws, *, aux: Optional[dict] = None,
                stream=None):
    """The whole layer on the current stream.  ``logits`` may be None when
    ``weights.w_router`` is set: the router projection computes them.
    ``aux`` may map moe_aux_t member names (topk_idx, topk_w, sgate, keff,
    expert_kept, n_dropped, counts, offsets, perm, slot_pos, logits) to
    device tensors to receive them."""
    T = x.shape[0]
    w = weights._c()
    a = _Aux()
    if aux:
        for name, t in aux.items():
            setattr(a, name, _ptr(t))
    _check("moe_forward", load_library().moe_forward(
        ctypes.byref(cfg._c()), T, _ptr(x), _ptr(logits, True), ctypes.byref(w), _ptr(out), ctypes.byref(a),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def status_read(ws, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("moe_status_read", load_library().moe_status_read(_ptr(ws), ctypes.byref(v), _stream(stream)))
    return int(v.value)


def status_clear(ws, stream=None):
    _check("moe_status_clear", load_library().moe_status_clear(_ptr(ws), _stream(stream)))
