"""The C ABI on a host without a GPU: the library builds, loads and exports
every function include/moe.h declares; argument checks reject bad calls
before any CUDA work (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

import routed_expert_ffn_renorm_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(moe.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = moe.load_library()
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert set(_declared()) <= exported


def _cfg(**kw):
    base = dict(hidden=256, n_routed_experts=8, moe_intermediate_size=128, num_experts_per_tok=2,
                shared_intermediate_size=0, norm_topk=True, budget=0, topp=0.0)
    base.update(kw)
    return moe._Config(*[float(v) if n == "topp" else int(v) for n, v in base.items()])


FAKE = ctypes.c_void_p(1 << 20)      # never dereferenced: the checks fail first
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


@pytest.mark.parametrize("kw,code", [
    (dict(n_routed_experts=0), -1), (dict(num_experts_per_tok=0), -1), (dict(num_experts_per_tok=9), -1),
    (dict(budget=-1), -1), (dict(norm_topk=2), -1), (dict(hidden=200), -2), (dict(moe_intermediate_size=96), -2),
    (dict(shared_intermediate_size=32), -2), (dict(n_routed_experts=2048, num_experts_per_tok=2), -2),
    (dict(n_routed_experts=64, num_experts_per_tok=33), -2),
    (dict(topp=float("nan")), -1), (dict(topp=-0.5), -1), (dict(topp=float("inf")), -1),
])
def test_config_checks(kw, code):
    lib = moe.load_library()
    c = _cfg(**kw)
    assert lib.moe_workspace_bytes(ctypes.byref(c), 16) == 0
    rc = lib.moe_route(ctypes.byref(c), 16, FAKE, None, None, FAKE, FAKE, None, None, None)
    assert rc == code


def test_pointer_checks_and_noop():
    lib = moe.load_library()
    c = _cfg()
    # T = 0 is a no-op, whatever the pointers
    assert lib.moe_forward(ctypes.byref(c), 0, None, None, None, None, None, None, 0, None) == 0
    assert lib.moe_route(ctypes.byref(c), -1, FAKE, None, None, FAKE, FAKE, None, None, None) == -1
    assert lib.moe_route(ctypes.byref(c), 16, MISALIGNED, None, None, FAKE, FAKE, None, None, None) == -1
    assert lib.moe_route(ctypes.byref(c), 16, None, None, None, FAKE, FAKE, None, None, None) == -1
    # sgate requested without a shared expert
    assert lib.moe_route(ctypes.byref(c), 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == -1
    # a top-p trim needs somewhere to put the kept counts
    cp = _cfg(topp=0.5)
    assert lib.moe_route(ctypes.byref(cp), 16, FAKE, None, None, FAKE, FAKE, None, None, None) == -1
    # short workspace
    ws_need = lib.moe_workspace_bytes(ctypes.byref(c), 16)
    assert ws_need > 0
    assert lib.moe_budget(ctypes.byref(c), 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws_need - 1, None) == -3
    assert lib.moe_dispatch(ctypes.byref(c), 16, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                            ws_need - 256, None) == -3
    w = moe._Weights(FAKE.value, FAKE.value, FAKE.value, None, None, None, None)
    assert lib.moe_forward(ctypes.byref(c), 16, FAKE, FAKE, ctypes.byref(w), FAKE, None, FAKE, 16, None) == -3
    # shared expert configured but its weights missing
    cs = _cfg(shared_intermediate_size=64)
    assert lib.moe_forward(ctypes.byref(cs), 16, FAKE, FAKE, ctypes.byref(w), FAKE, None, FAKE,
                           1 << 30, None) == -1
    assert lib.moe_error_string(-3) == b"workspace too small"


def test_workspace_grows_with_tokens():
    lib = moe.load_library()
    c = _cfg(shared_intermediate_size=64)
    a = lib.moe_workspace_bytes(ctypes.byref(c), 16)
    b = lib.moe_workspace_bytes(ctypes.byref(c), 1024)
    assert 0 < a < b and b % 256 == 0


def test_quantiser_argument_checks():
    lib = moe.load_library()
    # sizes: K must be a positive multiple of the block (32 for MXFP8, 16 for NVFP4)
    for K in (0, 16, 33, -32):
        assert lib.moe_quantize_mxfp8(4, K, FAKE, FAKE, FAKE, None) == -1
    assert lib.moe_quantize_mxfp8(-1, 64, FAKE, FAKE, FAKE, None) == -1
    for nmat, K in ((0, 16), (65536, 16), (1, 8), (1, 24)):
        assert lib.moe_quantize_nvfp4(nmat, 4, K, FAKE, FAKE, FAKE, FAKE, None) == -1
    # pointers: unaligned or missing
    assert lib.moe_quantize_mxfp8(4, 64, MISALIGNED, FAKE, FAKE, None) == -1
    assert lib.moe_quantize_mxfp8(4, 64, FAKE, MISALIGNED, FAKE, None) == -1
    assert lib.moe_quantize_mxfp8(4, 64, FAKE, FAKE, None, None) == -1
    assert lib.moe_quantize_nvfp4(2, 4, 32, FAKE, FAKE, FAKE, ctypes.c_void_p(FAKE.value + 2), None) == -1
    assert lib.moe_quantize_nvfp4(2, 4, 32, FAKE, FAKE, None, FAKE, None) == -1
    assert lib.moe_quantize_nvfp4(2, 4, 32, FAKE, FAKE, FAKE, None, None) == -1
    # no rows: nothing to do, whatever the data pointers
    assert lib.moe_quantize_mxfp8(0, 64, None, None, None, None) == 0
    assert lib.moe_quantize_nvfp4(3, 0, 32, None, None, None, FAKE, None) == 0


def test_mxfp8_argument_checks():
    """The MXFP8 entry points reject bad shapes and pointers before any launch."""
    lib = moe.load_library()
    P = ctypes.c_void_p
    # scale repacking: rows a multiple of 64, K of 128, aligned pointers
    assert lib.moe_mxfp8_pack_scales(63, 256, FAKE, FAKE, None) == -1
    assert lib.moe_mxfp8_pack_scales(64, 192, FAKE, FAKE, None) == -1
    assert lib.moe_mxfp8_pack_scales(64, 256, MISALIGNED, FAKE, None) == -1
    assert lib.moe_mxfp8_pack_scales(0, 256, None, None, None) == 0
    full = moe._WeightsMXFP8(*([FAKE.value] * 12 + [FAKE.value, FAKE.value]))
    ws_bytes = lib.moe_workspace_bytes(ctypes.byref(_cfg()), 16)
    args = (16, FAKE, FAKE, FAKE, FAKE, FAKE, None)
    # I = 64 is a legal bf16 shape but not an MXFP8 one (128-wide K steps)
    c = _cfg(moe_intermediate_size=64)
    assert lib.moe_expert_ffn_mxfp8(ctypes.byref(c), *args, ctypes.byref(full), FAKE, FAKE, 1 << 40, None) == -2
    assert lib.moe_forward_mxfp8(ctypes.byref(c), 16, FAKE, FAKE, ctypes.byref(full), FAKE, None, FAKE, 1 << 40,
                                 None) == -2
    c = _cfg()
    assert lib.moe_expert_ffn_mxfp8(ctypes.byref(c), *args, None, FAKE, FAKE, ws_bytes, None) == -1
    bad = moe._WeightsMXFP8(*([FAKE.value] * 3 + [MISALIGNED.value] + [FAKE.value] * 10))
    assert lib.moe_expert_ffn_mxfp8(ctypes.byref(c), *args, ctypes.byref(bad), FAKE, FAKE, ws_bytes, None) == -1
    assert lib.moe_expert_ffn_mxfp8(ctypes.byref(c), *args, ctypes.byref(full), FAKE, FAKE, ws_bytes - 1,
                                    None) == -3
    # a shared expert needs its codes and scales
    cs = _cfg(shared_intermediate_size=128)
    noshared = moe._WeightsMXFP8(*([FAKE.value] * 6 + [None] * 6 + [FAKE.value, FAKE.value]))
    ws_s = lib.moe_workspace_bytes(ctypes.byref(cs), 16)
    assert lib.moe_expert_ffn_mxfp8(ctypes.byref(cs), *args[:-1], FAKE, ctypes.byref(noshared), FAKE, FAKE, ws_s,
                                    None) == -1
    assert lib.moe_forward_mxfp8(ctypes.byref(c), 0, None, None, ctypes.byref(full), None, None, None, 0, None) == 0


def test_nvfp4_argument_checks():
    """The NVFP4 entry points reject bad shapes and pointers before any launch."""
    lib = moe.load_library()
    # scale repacking: rows a multiple of 64, K of 128, aligned pointers
    assert lib.moe_nvfp4_pack_scales(63, 256, FAKE, FAKE, None) == -1
    assert lib.moe_nvfp4_pack_scales(64, 192, FAKE, FAKE, None) == -1
    assert lib.moe_nvfp4_pack_scales(64, 256, FAKE, MISALIGNED, None) == -1
    assert lib.moe_nvfp4_pack_scales(0, 256, None, None, None) == 0
    nf = len(moe._WeightsNVFP4._fields_)
    full = moe._WeightsNVFP4(*([FAKE.value] * nf))
    ws_bytes = lib.moe_workspace_bytes(ctypes.byref(_cfg()), 16)
    args = (16, FAKE, FAKE, FAKE, FAKE, FAKE, None)
    # I = 64 is a legal bf16 shape but not an NVFP4 one (128-wide K steps)
    c = _cfg(moe_intermediate_size=64)
    assert lib.moe_expert_ffn_nvfp4(ctypes.byref(c), *args, ctypes.byref(full), FAKE, FAKE, 1 << 40, None) == -2
    assert lib.moe_forward_nvfp4(ctypes.byref(c), 16, FAKE, FAKE, ctypes.byref(full), FAKE, None, FAKE, 1 << 40,
                                 None) == -2
    c = _cfg()
    assert lib.moe_expert_ffn_nvfp4(ctypes.byref(c), *args, None, FAKE, FAKE, ws_bytes, None) == -1
    names = [n for n, _ in moe._WeightsNVFP4._fields_]
    for field, value in (("w_down_scale", MISALIGNED.value), ("w_up_tscale", None),
                         ("w_gate_tscale", FAKE.value + 2)):  # a matrix-scale pointer must be 4-byte aligned
        vals = [FAKE.value] * nf
        vals[names.index(field)] = value
        bad = moe._WeightsNVFP4(*vals)
        assert lib.moe_expert_ffn_nvfp4(ctypes.byref(c), *args, ctypes.byref(bad), FAKE, FAKE, ws_bytes,
                                        None) == -1, field
    assert lib.moe_expert_ffn_nvfp4(ctypes.byref(c), *args, ctypes.byref(full), FAKE, FAKE, ws_bytes - 1,
                                    None) == -3
    # a shared expert needs its codes, block scales and matrix scales
    cs = _cfg(shared_intermediate_size=128)
    ws_s = lib.moe_workspace_bytes(ctypes.byref(cs), 16)
    vals = [FAKE.value] * nf
    vals[names.index("ws_tscale")] = None
    noscale = moe._WeightsNVFP4(*vals)
    assert lib.moe_expert_ffn_nvfp4(ctypes.byref(cs), *args[:-1], FAKE, ctypes.byref(noscale), FAKE, FAKE, ws_s,
                                    None) == -1
    assert lib.moe_forward_nvfp4(ctypes.byref(c), 0, None, None, ctypes.byref(full), None, None, None, 0, None) == 0
