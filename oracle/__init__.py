"""The oracle -- TEST INFRASTRUCTURE, not product code.

A plain CPU definition of the routed-MoE FFN forward (route -> budget ->
dispatch -> SwiGLU expert FFN -> weighted combine + sigmoid-gated shared
expert), written in C (``moe_oracle.c``) and wrapped here with ctypes.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline/reference
legs of ``bench.py`` may import this package.  The CUDA library never calls
it, and the two share no source.

Each function follows a passage of the pages:
  * SpecForge PR #943 (Qwen3.8-27B DSpark MoE drafter), "Modifications":
    the router projection and softmax router with renormalised top-k,
    sigmoid-gated shared expert,
    grouped dispatch; its FFN parameter table fixes the gated FFN's shape.
  * colibri issue_budget.md (EXPERT_BUDGET), "How it works" steps 1-5 and
    "Safety": the batch-union expert budget; "Relationship to existing
    features": the per-position top-p trim (TOPP) that runs before it.
  * ``quant_oracle.c``: the block-scaled FP8 (MXFP8) and NVFP4 expert-weight
    formats that DeepGEMM fork PR #5 and DeepGEMM PR #381 name for expert
    weights, with their published definitions (E4M3, E2M1, UE8M0 codecs,
    block quantisers and dequantisers).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SRCS = (_SRC, os.path.join(_HERE, "quant_oracle.c"))
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(os.path.getmtime(f) for f in _SRCS):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", *_SRCS, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32 = ctypes.c_int32
    lib.oracle_ffn_params.restype = ctypes.c_int64
    lib.oracle_ffn_params.argtypes = [ctypes.c_int64, ctypes.c_int64]
    lib.oracle_route.argtypes = [i32, i32, i32, i32, P, P, P]
    lib.oracle_router_logits.argtypes = [i32, i32, i32, P, P, P]
    lib.oracle_budget.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P]
    lib.oracle_budget_apply.argtypes = [i32, i32, i32, P, P, P, P]
    lib.oracle_topp.argtypes = [i32, i32, i32, ctypes.c_float, P, P, P]
    lib.oracle_dispatch.argtypes = [i32, i32, i32, P, P, P, P, P, P]
    lib.oracle_expert_rows.argtypes = [i32, i32, P, P, P, i32, P, P, i32]
    lib.oracle_shared_gate_row.restype = ctypes.c_double
    lib.oracle_shared_gate_row.argtypes = [i32, P, P]
    lib.oracle_forward.argtypes = [i32] * 8 + [ctypes.c_float] + [P] * 11 + [i32, P, P] + [P] * 9 + [i32]
    lib.oracle_combine_rows.argtypes = [i32] * 5 + [P] * 4 + [P] * 3 + [P] * 6 + [i32, P, P, i32]
    lib.oracle_max_threads.restype = ctypes.c_int
    i64 = ctypes.c_int64
    for name in ("oracle_e4m3_decode", "oracle_e4m3_encode", "oracle_e2m1_decode", "oracle_e2m1_encode",
                 "oracle_ue8m0_decode"):
        getattr(lib, name).argtypes = [i64, P, P]
        getattr(lib, name).restype = None
    lib.oracle_mxfp8_quantize.argtypes = [i64, i64, P, P, P]
    lib.oracle_mxfp8_dequantize.argtypes = [i64, i64, P, P, P]
    lib.oracle_nvfp4_quantize.argtypes = [i64, i64, P, P, P, P]
    lib.oracle_nvfp4_dequantize.argtypes = [i64, i64, P, P, ctypes.c_float, P]
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def ffn_params(H: int, I: int) -> int:
    """Parameters of one gated expert FFN (gate, up, down projections)."""
    return int(_load().oracle_ffn_params(H, I))


def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """logits = x . W_r^T (fp64 accumulation, rounded once to fp32).
    x [T, H], w_router [E, H]: bf16 bit patterns.  Returns [T, E] float32."""
    x = _c(x, np.uint16)
    wr = _c(w_router, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((max(T, 1), E), np.float32)
    _check(_load().oracle_router_logits(T, H, E, _ptr(x), _ptr(wr), _ptr(out)), "router_logits")
    return out[:T]


def route(logits: np.ndarray, k: int, norm_topk: bool = True):
    """Softmax over all experts, top-k by logit, renormalised if norm_topk.

    Returns (idx [T,k] int32, w [T,k] float32)."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _check(_load().oracle_route(T, E, k, int(bool(norm_topk)), _ptr(logits), _ptr(idx), _ptr(w)), "route")
    return idx, w


def topp(idx: np.ndarray, w: np.ndarray, p: float, norm_topk: bool = True):
    """Per-token top-p trim of the router output (copies; inputs untouched):
    the shortest prefix of each token's slots whose weights reach p.

    Returns (idx, w, keff [T])."""
    idx = np.array(idx, np.int32, copy=True, order="C")
    w = np.array(w, np.float32, copy=True, order="C")
    T, k = idx.shape
    keff = np.empty(max(T, 1), np.int32)
    _check(_load().oracle_topp(T, k, int(bool(norm_topk)), float(p), _ptr(idx), _ptr(w), _ptr(keff)), "topp")
    return idx, w, keff[:T]


def budget(idx: np.ndarray, w: np.ndarray, E: int, N: int, norm_topk: bool = True):
    """EXPERT_BUDGET cap over the batch union (copies; inputs untouched).
    Slots with idx -1 (a top-p trim's tail) take no part.

    Returns (idx, w, keff [T], kept [E] uint8, n_dropped)."""
    idx = np.array(idx, np.int32, copy=True, order="C")
    w = np.array(w, np.float32, copy=True, order="C")
    T, k = idx.shape
    keff = np.empty(T, np.int32)
    kept = np.empty(E, np.uint8)
    nd = np.zeros(1, np.int32)
    _check(_load().oracle_budget(T, E, k, N, int(bool(norm_topk)), _ptr(idx), _ptr(w), _ptr(keff),
                                 _ptr(kept), _ptr(nd)), "budget")
    return idx, w, keff, kept, int(nd[0])


def budget_apply(idx: np.ndarray, w: np.ndarray, kept: np.ndarray, norm_topk: bool = True):
    """Step 4 of the budget for a GIVEN kept set (copies; inputs untouched):
    each token's slots of kept experts move to the front in order, the tail
    becomes (-1, 0), and a token that lost a valid slot is renormalised when
    norm_topk.  budget() is this step after choosing the kept set; a test
    uses it to check a near-tie that the GPU decided the other way.

    Returns (idx, w, keff [T])."""
    idx = np.array(idx, np.int32, copy=True, order="C")
    w = np.array(w, np.float32, copy=True, order="C")
    kept = _c(kept, np.uint8)
    T, k = idx.shape
    if idx.size and int(idx.max()) >= kept.shape[0]:
        raise ValueError("routing names an expert outside the kept mask")
    keff = np.ascontiguousarray((idx >= 0).sum(axis=1), dtype=np.int32)
    if T == 0:
        keff = np.zeros(1, np.int32)
    _check(_load().oracle_budget_apply(T, k, int(bool(norm_topk)), _ptr(kept), _ptr(idx), _ptr(w), _ptr(keff)),
           "budget_apply")
    return idx, w, keff[:T]


def dispatch(idx: np.ndarray, keff: np.ndarray, E: int):
    """Group kept slots by expert. Returns (counts, offsets, perm, slot_pos)."""
    idx = _c(idx, np.int32)
    keff = _c(keff, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.full(max(T * k, 1), -1, np.int32)
    slot_pos = np.empty(max(T * k, 1), np.int32)
    _check(_load().oracle_dispatch(T, E, k, _ptr(idx), _ptr(keff), _ptr(counts), _ptr(offsets),
                                   _ptr(perm), _ptr(slot_pos)), "dispatch")
    total = int(offsets[E])
    return counts, offsets, perm[:total].copy(), slot_pos[: T * k].copy()


def expert_rows(wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, x: np.ndarray, nthreads: int = 1):
    """SwiGLU FFN of one expert on rows of x (all bf16 as uint16 bit patterns).

    wg, wu: [I, H]; wd: [H, I]; x: [n, H].  Returns y [n, H] float64."""
    wg, wu, wd, x = (_c(a, np.uint16) for a in (wg, wu, wd, x))
    I, H = wg.shape
    n = x.shape[0]
    y = np.empty((n, H), np.float64)
    _check(_load().oracle_expert_rows(H, I, _ptr(wg), _ptr(wu), _ptr(wd), n, _ptr(x), _ptr(y), nthreads),
           "expert_rows")
    return y


def shared_gate(g: np.ndarray, x: np.ndarray) -> np.ndarray:
    """sigmoid(g . x_t) for every row of x (bf16 bit patterns)."""
    g = _c(g, np.uint16)
    x = _c(x, np.uint16)
    lib = _load()
    H = g.shape[0]
    return np.array([lib.oracle_shared_gate_row(H, _ptr(g), _ptr(x[t])) for t in range(x.shape[0])])


@dataclass
class ForwardResult:
    out: np.ndarray        # [n_rows, H] float64, rows in the order requested
    idx: np.ndarray        # [T, k] int32 (after the budget)
    w: np.ndarray          # [T, k] float32 (after the budget)
    keff: np.ndarray       # [T] int32
    kept: np.ndarray       # [E] uint8
    n_dropped: int
    counts: np.ndarray     # [E]
    offsets: np.ndarray    # [E+1]
    perm: np.ndarray       # [sum keff]
    slot_pos: np.ndarray   # [T*k]


def _expert_ptrs(w, E):
    """Per-expert pointer array from a full [E, ...] array or a dict {e: array}."""
    arr = (ctypes.c_void_p * E)()
    keep = []
    if isinstance(w, dict):
        for e, a in w.items():
            a = _c(a, np.uint16)
            keep.append(a)
            arr[e] = a.ctypes.data
    else:
        a = _c(w, np.uint16)
        keep.append(a)
        step = a[0].nbytes if E else 0
        for e in range(E):
            arr[e] = a.ctypes.data + e * step
    return arr, keep


def _scale_ptrs(scales, shared_scales, E):
    """Per-projection output factors: scales [E, 3] (gate, up, down) and
    shared_scales [3], float64; None passes NULL (no factor)."""
    keep = []
    ps = pss = None
    if scales is not None:
        a = _c(scales, np.float64).reshape(E, 3)
        keep.append(a)
        ps = _ptr(a)
    if shared_scales is not None:
        b = _c(shared_scales, np.float64).reshape(3)
        keep.append(b)
        pss = _ptr(b)
    return ps, pss, keep


def forward(x, logits, w_gate, w_up, w_down, *, k: int, norm_topk: bool = True, budget: int = 0,
            topp: float = 0.0, ws_gate=None, ws_up=None, ws_down=None, ws_gvec=None, rows=None,
            nthreads: int = 1, I: int = None, scales=None, shared_scales=None) -> ForwardResult:
    """The whole layer. x and all weights are bf16 bit patterns (uint16).

    x [T,H]; logits [T,E] f32; w_gate, w_up [E,I,H] and w_down [E,H,I] as full
    arrays, or as dicts {expert: [I,H] / [H,I] array} holding only the experts
    the requested rows route to (then pass I);
    shared (optional): ws_gate, ws_up [Is,H], ws_down [H,Is], ws_gvec [H].
    rows: token ids whose output to compute (default: all);
    scales [E, 3], shared_scales [3]: factors on each projection's output
    (gate, up, down), the fp32 matrix scales of block-scaled weights."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    T, H = x.shape
    E = logits.shape[1]
    if I is None:
        I = w_gate.shape[1]
    pg, kg = _expert_ptrs(w_gate, E)
    pu, ku = _expert_ptrs(w_up, E)
    pd, kd = _expert_ptrs(w_down, E)
    Is = 0
    if ws_gate is not None:
        ws_gate, ws_up, ws_down, ws_gvec = (_c(a, np.uint16) for a in (ws_gate, ws_up, ws_down, ws_gvec))
        Is = ws_gate.shape[0]
    else:
        ws_gate = ws_up = ws_down = ws_gvec = np.zeros(1, np.uint16)
    rows = np.arange(T, dtype=np.int32) if rows is None else _c(rows, np.int32)
    n_rows = rows.shape[0]
    out = np.empty((max(n_rows, 1), H), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    keff = np.empty(max(T, 1), np.int32)
    kept = np.empty(E, np.uint8)
    nd = np.zeros(1, np.int32)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.full(max(T * k, 1), -1, np.int32)
    slot_pos = np.empty(max(T * k, 1), np.int32)
    ps, pss, _keep = _scale_ptrs(scales, shared_scales, E)
    rc = _load().oracle_forward(
        T, H, E, I, k, Is, int(bool(norm_topk)), budget, float(topp),
        _ptr(x), _ptr(logits), pg, pu, pd,
        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(ws_gvec), ps, pss,
        n_rows, _ptr(rows), _ptr(out),
        _ptr(idx), _ptr(w), _ptr(keff), _ptr(kept), _ptr(nd),
        _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(slot_pos), nthreads)
    _check(rc, "forward")
    total = int(offsets[E])
    return ForwardResult(out[:n_rows], idx, w, keff[:T], kept, int(nd[0]), counts, offsets,
                         perm[:total].copy(), slot_pos[: T * k].copy())


def combine_rows(x, idx, w, keff, w_gate, w_up, w_down, *, I: int, ws_gate=None, ws_up=None, ws_down=None,
                 ws_gvec=None, rows=None, nthreads: int = 1, scales=None, shared_scales=None) -> np.ndarray:
    """Expert FFN + weighted combine (+ gated shared expert) for GIVEN routing
    (idx/w/keff, e.g. after a budget), for the listed token rows.  Weights as
    in forward().  Returns out [n_rows, H] float64."""
    x = _c(x, np.uint16)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    keff = _c(keff, np.int32)
    T, H = x.shape
    k = idx.shape[1]
    if isinstance(w_gate, dict):  # pointer table must cover every expert id idx can name
        E = max(max(w_gate, default=0), int(idx.max(initial=0))) + 1
    else:
        E = w_gate.shape[0]
        if idx.size and int(idx.max()) >= E:
            raise ValueError("routing names an expert outside the weight arrays")
    pg, kg = _expert_ptrs(w_gate, E)
    pu, ku = _expert_ptrs(w_up, E)
    pd, kd = _expert_ptrs(w_down, E)
    Is = 0
    if ws_gate is not None:
        ws_gate, ws_up, ws_down, ws_gvec = (_c(a, np.uint16) for a in (ws_gate, ws_up, ws_down, ws_gvec))
        Is = ws_gate.shape[0]
    else:
        ws_gate = ws_up = ws_down = ws_gvec = np.zeros(1, np.uint16)
    rows = np.arange(T, dtype=np.int32) if rows is None else _c(rows, np.int32)
    out = np.empty((max(rows.shape[0], 1), H), np.float64)
    ps, pss, _keep = _scale_ptrs(scales, shared_scales, E)
    _check(_load().oracle_combine_rows(T, H, I, k, Is, _ptr(x), _ptr(idx), _ptr(w), _ptr(keff), pg, pu, pd,
                                       _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(ws_gvec), ps, pss,
                                       rows.shape[0], _ptr(rows), _ptr(out), nthreads), "combine_rows")
    return out[: rows.shape[0]]



# ------------------------------------------------ block-scaled weights --
def _codec(name, a, in_dtype, out_dtype):
    a = _c(a, in_dtype)
    out = np.empty(a.shape, out_dtype)
    getattr(_load(), name)(a.size, _ptr(a), _ptr(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> their values (float64; NaN for 0x7F, 0xFF)."""
    return _codec("oracle_e4m3_decode", codes, np.uint8, np.float64)


def e4m3_encode(x) -> np.ndarray:
    """Values -> the nearest E4M3 codes (ties to even, saturating at 448)."""
    return _codec("oracle_e4m3_encode", x, np.float64, np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    """E2M1 codes (low nibble of each uint8) -> their values (float64)."""
    return _codec("oracle_e2m1_decode", codes, np.uint8, np.float64)


def e2m1_encode(x) -> np.ndarray:
    """Values -> the nearest E2M1 codes (ties to even, saturating at 6)."""
    return _codec("oracle_e2m1_encode", x, np.float64, np.uint8)


def ue8m0_decode(codes) -> np.ndarray:
    """UE8M0 scale codes -> 2^(c - 127) (NaN for 255)."""
    return _codec("oracle_ue8m0_decode", codes, np.uint8, np.float64)


def mxfp8_quantize(w):
    """bf16 bit patterns [rows, K] (K % 32 == 0) -> (E4M3 codes [rows, K],
    UE8M0 scales [rows, K / 32]); blocks run along the last axis."""
    w = _c(w, np.uint16)
    rows, K = w.reshape(-1, w.shape[-1]).shape
    codes = np.empty(w.shape, np.uint8)
    scales = np.empty(w.shape[:-1] + (K // 32,), np.uint8)
    _check(_load().oracle_mxfp8_quantize(rows, K, _ptr(w), _ptr(codes), _ptr(scales)), "mxfp8_quantize")
    return codes, scales


def mxfp8_dequantize(codes, scales) -> np.ndarray:
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    K = codes.shape[-1]
    out = np.empty(codes.shape, np.float64)
    _check(_load().oracle_mxfp8_dequantize(codes.size // K, K, _ptr(codes), _ptr(scales), _ptr(out)),
           "mxfp8_dequantize")
    return out


def nvfp4_quantize(w):
    """bf16 bit patterns [rows, K] (K % 16 == 0), one matrix -> (packed E2M1
    codes [rows, K / 2], E4M3 block scales [rows, K / 16], fp32 matrix scale)."""
    w = _c(w, np.uint16)
    rows, K = w.reshape(-1, w.shape[-1]).shape
    codes = np.empty(w.shape[:-1] + (K // 2,), np.uint8)
    scales = np.empty(w.shape[:-1] + (K // 16,), np.uint8)
    st = np.zeros(1, np.float32)
    _check(_load().oracle_nvfp4_quantize(rows, K, _ptr(w), _ptr(codes), _ptr(scales), _ptr(st)),
           "nvfp4_quantize")
    return codes, scales, float(st[0])


def nvfp4_dequantize(codes, scales, tensor_scale: float) -> np.ndarray:
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    K = codes.shape[-1] * 2
    out = np.empty(codes.shape[:-1] + (K,), np.float64)
    _check(_load().oracle_nvfp4_dequantize(codes.size * 2 // K, K, _ptr(codes), _ptr(scales),
                                           float(np.float32(tensor_scale)), _ptr(out)), "nvfp4_dequantize")
    return out


def f64_to_bf16_exact(v) -> np.ndarray:
    """float64 values that bf16 holds exactly -> bf16 bit patterns; raises
    when one is not exact (the dequantised MXFP8 weights always are in the
    exponent range of these layers)."""
    v = np.asarray(v, np.float64)
    f = v.astype(np.float32)
    bits = f.view(np.uint32)
    back = f.astype(np.float64)
    exact = np.array_equal(back, v) or np.array_equal(back, v, equal_nan=True)  # the NaN-aware pass only if needed
    if not exact or np.any(bits & 0xFFFF):
        raise ValueError("value not representable in bf16")
    return (bits >> 16).astype(np.uint16)


def mxfp8_weights(w):
    """An expert matrix (bf16 bits, reduction axis last) stored as MXFP8:
    the bf16 bit patterns of its dequantised values, which the MMA then
    consumes unchanged."""
    codes, scales = mxfp8_quantize(w)
    return f64_to_bf16_exact(mxfp8_dequantize(codes, scales))


def forward_mxfp8(x, logits, w_gate, w_up, w_down, *, ws_gate=None, ws_up=None, ws_down=None, **kw):
    """The layer with MXFP8 expert weights (routed and shared; the shared
    gate vector stays bf16): each matrix quantised along its reduction axis,
    dequantised exactly, then the bf16 layer definition."""
    shared = {}
    if ws_gate is not None:
        shared = dict(ws_gate=mxfp8_weights(ws_gate), ws_up=mxfp8_weights(ws_up), ws_down=mxfp8_weights(ws_down))
    return forward(x, logits, mxfp8_weights(w_gate), mxfp8_weights(w_up), mxfp8_weights(w_down),
                   **shared, **kw)


def nvfp4_weights(w):
    """Expert matrices [..., rows, K] (bf16 bits, reduction axis last) stored
    as NVFP4, one fp32 matrix scale per leading index: (the bf16 bit patterns
    of element x block scale, exact in bf16, and the matrix scales)."""
    w = _c(w, np.uint16)
    lead = w.shape[:-2]
    flat = w.reshape((-1,) + w.shape[-2:])
    vals, sts = [], []
    for m in flat:
        codes, scales, st = nvfp4_quantize(m)
        vals.append(f64_to_bf16_exact(nvfp4_dequantize(codes, scales, 1.0)))
        sts.append(st)
    return np.stack(vals).reshape(w.shape), np.array(sts, np.float64).reshape(lead)


def forward_nvfp4(x, logits, w_gate, w_up, w_down, *, ws_gate=None, ws_up=None, ws_down=None, **kw):
    """The layer with NVFP4 expert weights (routed and shared; the shared gate
    vector stays bf16): each expert matrix quantised along its reduction axis
    with its own fp32 scale; the projections take element x block scale as
    their weights and multiply their outputs by the matrix scale."""
    (wg, sg), (wu, su), (wd, sd) = (nvfp4_weights(a) for a in (w_gate, w_up, w_down))
    extra = {}
    if ws_gate is not None:
        (g2, s2g), (u2, s2u), (d2, s2d) = (nvfp4_weights(a) for a in (ws_gate, ws_up, ws_down))
        extra = dict(ws_gate=g2, ws_up=u2, ws_down=d2, shared_scales=np.array([s2g, s2u, s2d], np.float64))
    return forward(x, logits, wg, wu, wd, scales=np.stack([sg, su, sd], axis=-1), **extra, **kw)
