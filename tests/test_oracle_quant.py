"""Pins of the oracle's block-scaled expert-weight formats (CPU only).

The formats (E4M3, E2M1 and UE8M0 codes; MXFP8 and NVFP4 block scaling) are
pinned to things outside the oracle: torch's own float8 dtypes where torch
has them, the constants that define each format, exact round trips of values
the format holds, the error bound of round-to-nearest, and the identity of
the quantised layer on weights that are already representable.  The second
half plants plausible mistakes in a copy of the oracle's source and checks
that a pin catches each one.
"""
import importlib.util
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
QSRC = os.path.join(ROOT, "oracle", "quant_oracle.c")
MSRC = os.path.join(ROOT, "oracle", "moe_oracle.c")


def _bf16_bits(a) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_value(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------- pins --
def pin_e4m3_constants(o):
    v = o.e4m3_decode(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x77, 0x7E, 0xB8, 0xFE, 0x80], np.uint8))
    assert v.tolist() == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 240.0, 448.0, -1.0, -448.0, 0.0]
    assert np.isnan(o.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def pin_e4m3_decode_matches_torch(o):
    c = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(o.e4m3_decode(c), ref)


def pin_e4m3_encode_nearest_even(o):
    c = np.array([i for i in range(256) if i not in (0x7F, 0xFF)], np.uint8)
    v = o.e4m3_decode(c)
    np.testing.assert_array_equal(o.e4m3_encode(v), c)  # every finite value is its own code
    pos = np.arange(0x7F, dtype=np.uint8)
    pv = o.e4m3_decode(pos)
    mid = (pv[:-1] + pv[1:]) / 2
    even = np.where(pos[:-1] % 2 == 0, pos[:-1], pos[1:])
    np.testing.assert_array_equal(o.e4m3_encode(mid), even)  # ties to the even code
    gap = pv[1:] - pv[:-1]
    np.testing.assert_array_equal(o.e4m3_encode(mid - gap / 8), pos[:-1])
    np.testing.assert_array_equal(o.e4m3_encode(mid + gap / 8), pos[1:])
    assert o.e4m3_encode([449.0, 464.0, 500.0, 1e9, -1e9, 1.2e18, 3e38, -3e38]).tolist() == \
        [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0x7E, 0xFE]
    assert o.e4m3_encode([-0.0, -1e-6, 1e-6]).tolist() == [0x80, 0x80, 0x00]
    x = np.random.default_rng(0).standard_normal(4096) * np.exp2(np.random.default_rng(1).integers(-12, 8, 4096))
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(o.e4m3_encode(x.astype(np.float64)), ref)


def pin_e2m1_table(o):
    v = o.e2m1_decode(np.arange(16, dtype=np.uint8))
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert v[:8].tolist() == mags and v[8:].tolist() == [-m for m in mags]
    assert o.e2m1_encode(np.array(mags)).tolist() == list(range(8))
    # ties between neighbours go to the even code; beyond 6 saturates
    assert o.e2m1_encode([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 100.0]).tolist() == [0, 2, 2, 4, 4, 6, 6, 7, 7]
    assert o.e2m1_encode([0.26, 0.74, 2.4, 5.1, -5.1, -0.0, 1e18, -3e38]).tolist() == [1, 1, 4, 7, 15, 8, 7, 15]


def pin_ue8m0_matches_torch(o):
    c = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(c).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal(o.ue8m0_decode(c), ref)
    assert o.ue8m0_decode(np.array([127], np.uint8))[0] == 1.0


def _weights(rows, K, seed, sigma=0.02):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((rows, K)) * sigma
    w[0, :32] = 0.0                            # an all-zero block
    w[1, 32:64] = 0.0
    w[1, 40] = 3.0                             # a block with one non-zero
    w[2] *= np.repeat(np.exp2(rng.integers(-20, 6, K // 32)), 32)  # block magnitudes far apart
    return _bf16_bits(w)


def pin_mxfp8_scale_rule(o):
    w = _weights(8, 256, seed=2)
    codes, scales = o.mxfp8_quantize(w)
    x = _bf16_value(w).reshape(8, -1, 32)
    amax = np.abs(x).max(axis=2)
    q = o.e4m3_decode(codes).reshape(8, -1, 32)
    sc = scales.astype(np.int64) - 127
    nz = amax > 0
    np.testing.assert_array_equal(sc[nz], np.floor(np.log2(amax[nz])).astype(np.int64) - 8)
    assert (sc[~nz] == -127).all() and (codes.reshape(8, -1, 32)[~nz] % 128 == 0).all()
    scaled = amax[nz] / np.exp2(sc[nz])
    assert ((scaled >= 256) & (scaled < 512)).all()
    qmax = np.abs(q).max(axis=2)[nz]
    assert ((qmax >= 256) & (qmax <= 448)).all()


def pin_mxfp8_error_bound(o):
    w = _weights(16, 512, seed=3)
    codes, scales = o.mxfp8_quantize(w)
    x = _bf16_value(w).reshape(16, 512)
    xh = o.mxfp8_dequantize(codes, scales)
    X = np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)
    v = np.abs(x) / X
    with np.errstate(divide="ignore"):
        half_ulp = np.where(v >= 2.0 ** -6, np.exp2(np.floor(np.log2(np.maximum(v, 2.0 ** -6))) - 4), 2.0 ** -10)
    err = np.abs(x - xh) / X
    clipped = v > 448
    assert (err[~clipped] <= half_ulp[~clipped] * (1 + 1e-12)).all()
    np.testing.assert_array_equal(np.abs(xh[clipped]) / X[clipped], 448.0)
    assert np.array_equal(np.sign(xh[xh != 0]), np.sign(x[xh != 0]))


def pin_mxfp8_exact_identity(o):
    rng = np.random.default_rng(4)
    c = rng.integers(0, 0x7F, (4, 128)).astype(np.uint8) | (rng.integers(0, 2, (4, 128)) << 7).astype(np.uint8)
    c[:, ::32] = 0x70 | rng.integers(0, 7, (4, 4)).astype(np.uint8)  # each block's max in [256, 448)
    c[:, 1::32] = 0x00
    vals = o.e4m3_decode(c) * np.exp2(rng.integers(-20, -8, (4, 4))).repeat(32, axis=1)
    w = _bf16_bits(vals)
    assert np.array_equal(_bf16_value(w), vals)
    codes, scales = o.mxfp8_quantize(w)
    np.testing.assert_array_equal(o.mxfp8_dequantize(codes, scales), vals)
    np.testing.assert_array_equal(o.f64_to_bf16_exact(o.mxfp8_dequantize(codes, scales)), w)


def pin_nvfp4_scale_rule(o):
    w = _weights(8, 256, seed=5)
    codes, scales, st = o.nvfp4_quantize(w)
    x = _bf16_value(w)
    amax = np.abs(x).max()
    assert st == float(np.float32(amax) / np.float32(2688.0))
    sb = o.e4m3_decode(scales)
    assert (sb <= 448).all() and (sb >= 0).all()
    amax_b = np.abs(x).reshape(8, -1, 16).max(axis=2)
    want = amax_b / (6 * st)
    nz = want >= 2.0 ** -6
    assert (np.abs(sb[nz] - want[nz]) <= want[nz] * 2.0 ** -4 * (1 + 1e-6)).all()  # E4M3 rounding
    r, b = np.unravel_index(np.argmax(amax_b), amax_b.shape)
    assert sb[r, b] == 448.0
    q = o.e2m1_decode(np.stack([codes & 15, codes >> 4], axis=-1).reshape(8, 256))
    assert np.abs(q).max() == 6.0 and np.abs(q[r, b * 16:(b + 1) * 16]).max() == 6.0


def pin_nvfp4_error_bound(o):
    w = _weights(16, 512, seed=6)
    codes, scales, st = o.nvfp4_quantize(w)
    x = _bf16_value(w)
    xh = o.nvfp4_dequantize(codes, scales, st)
    s = np.repeat(o.e4m3_decode(scales), 16, axis=1) * st
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s > 0, np.abs(x) / s, 0.0)
    half_step = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    inside = (v <= 6) & (s > 0)
    assert (np.abs(x - xh)[inside] <= half_step[inside] * s[inside] * (1 + 1e-6)).all()
    beyond = v > 6
    np.testing.assert_allclose(np.abs(xh[beyond]), 6 * s[beyond], rtol=0)
    assert (xh[s == 0] == 0).all()


def pin_nvfp4_exact_identity_and_packing(o):
    rng = np.random.default_rng(7)
    K = 64
    e2 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mag = e2[rng.integers(0, 8, (4, K))]
    mag[:, ::16] = 6.0                                 # every block reaches 6
    sign = np.where(rng.integers(0, 2, (4, K)) == 1, -1.0, 1.0)
    sbv = o.e4m3_decode(rng.integers(0x30, 0x7E, (4, K // 16)).astype(np.uint8))
    sbv[0, 0] = 448.0                                  # the matrix amax block: s_t = 2^-6 exactly
    vals = sign * mag * np.repeat(sbv, 16, axis=1) * 2.0 ** -6
    w = _bf16_bits(vals)
    assert np.array_equal(_bf16_value(w), vals)
    codes, scales, st = o.nvfp4_quantize(w)
    assert st == 2.0 ** -6
    np.testing.assert_array_equal(o.e4m3_decode(scales), sbv)
    np.testing.assert_array_equal(o.nvfp4_dequantize(codes, scales, st), vals)
    # element 2i in the low nibble, 2i + 1 in the high one
    lo = o.e2m1_decode(codes & 15) * np.repeat(sbv, 8, axis=1) * st
    hi = o.e2m1_decode(codes >> 4) * np.repeat(sbv, 8, axis=1) * st
    np.testing.assert_array_equal(lo, vals[:, 0::2])
    np.testing.assert_array_equal(hi, vals[:, 1::2])


def pin_forward_mxfp8(o):
    rng = np.random.default_rng(8)
    T, H, E, I, k, Is = 12, 64, 4, 32, 2, 32
    x = _bf16_bits(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    mk = lambda *s: _bf16_bits(rng.standard_normal(s) * 0.1)
    wg, wu, wd = mk(E, I, H), mk(E, I, H), mk(E, H, I)
    sg, su, sd, gv = mk(Is, H), mk(Is, H), mk(H, Is), mk(H)
    kw = dict(k=k, ws_gvec=gv)
    base = o.forward(x, logits, wg, wu, wd, ws_gate=sg, ws_up=su, ws_down=sd, **kw).out
    quant = o.forward_mxfp8(x, logits, wg, wu, wd, ws_gate=sg, ws_up=su, ws_down=sd, **kw).out
    rel = np.linalg.norm(quant - base) / np.linalg.norm(base)
    # E4M3 keeps 3 mantissa bits: each weight within 2^-4 (about 3.6 % RMS), and the
    # three projections of the layer add up to a few percent, never zero here
    assert 0 < rel < 0.12
    # weights that MXFP8 already holds: the quantised layer is the bf16 layer
    q = [o.mxfp8_weights(a) for a in (wg, wu, wd, sg, su, sd)]
    base_q = o.forward(x, logits, *q[:3], ws_gate=q[3], ws_up=q[4], ws_down=q[5], **kw).out
    again = o.forward_mxfp8(x, logits, *q[:3], ws_gate=q[3], ws_up=q[4], ws_down=q[5], **kw).out
    np.testing.assert_array_equal(again, base_q)
    # a plain dense check of one token through one expert, in fp64
    d = o.mxfp8_dequantize(*o.mxfp8_quantize(wg[0]))
    np.testing.assert_array_equal(_bf16_value(q[0][0]).reshape(I, H), d)


def _exact_nvfp4_matrix(o, rng, rows, K, st_exp):
    """Values NVFP4 holds exactly, whose quantisation gives back s_t = 2^st_exp:
    every block reaches 6 x its scale and one block has the largest scale."""
    e2 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mag = e2[rng.integers(0, 8, (rows, K))]
    mag[:, ::16] = 6.0
    sign = np.where(rng.integers(0, 2, (rows, K)) == 1, -1.0, 1.0)
    sbv = o.e4m3_decode(rng.integers(0x30, 0x7E, (rows, K // 16)).astype(np.uint8))
    sbv[0, 0] = 448.0
    return sign * mag * np.repeat(sbv, 16, axis=1) * 2.0 ** st_exp


def _small_layer(rng, T=12, H=64, E=4, I=32, k=2, Is=32, sigma=0.1):
    x = _bf16_bits(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    mk = lambda *s: _bf16_bits(rng.standard_normal(s) * sigma)
    return x, logits, [mk(E, I, H), mk(E, I, H), mk(E, H, I)], [mk(Is, H), mk(Is, H), mk(H, Is)], mk(H)


def pin_forward_output_scales(o):
    rng = np.random.default_rng(9)
    x, logits, (wg, wu, wd), (sg, su, sd), gv = _small_layer(rng)
    E = wg.shape[0]
    base = o.forward(x, logits, wg, wu, wd, ws_gate=sg, ws_up=su, ws_down=sd, ws_gvec=gv, k=2).out
    up = lambda a, p: _bf16_bits(_bf16_value(a).reshape(a.shape) * 2.0 ** p)
    # weights times 2, 4, 8 (gate, up, down), output factors 1/2, 1/4, 1/8: the same layer, bit for bit
    scaled = o.forward(x, logits, up(wg, 1), up(wu, 2), up(wd, 3), ws_gate=up(sg, 1), ws_up=up(su, 2),
                       ws_down=up(sd, 3), ws_gvec=gv, k=2, scales=np.tile([0.5, 0.25, 0.125], (E, 1)),
                       shared_scales=[0.5, 0.25, 0.125]).out
    np.testing.assert_array_equal(scaled, base)
    ones = o.forward(x, logits, wg, wu, wd, ws_gate=sg, ws_up=su, ws_down=sd, ws_gvec=gv, k=2,
                     scales=np.ones((E, 3)), shared_scales=np.ones(3)).out
    np.testing.assert_array_equal(ones, base)
    # per-expert factors: expert 1's down factor 2 doubles exactly its routed contribution
    w2 = np.ones((E, 3))
    w2[1, 2] = 2.0
    f = o.forward(x, logits, wg, wu, wd, k=2, scales=w2)
    plain = o.forward(x, logits, wg, wu, wd, k=2)
    only1 = o.combine_rows(x, plain.idx, plain.w, plain.keff, np.where(np.arange(E)[:, None, None] == 1, wg, 0),
                           wu, wd, I=wg.shape[1])
    np.testing.assert_allclose(f.out - plain.out, only1, rtol=1e-12, atol=1e-15)


def pin_forward_nvfp4(o):
    rng = np.random.default_rng(10)
    x, logits, (wg, wu, wd), (sg, su, sd), gv = _small_layer(rng)
    kw = dict(ws_gvec=gv, k=2)
    base = o.forward(x, logits, wg, wu, wd, ws_gate=sg, ws_up=su, ws_down=sd, **kw).out
    quant = o.forward_nvfp4(x, logits, wg, wu, wd, ws_gate=sg, ws_up=su, ws_down=sd, **kw).out
    rel = np.linalg.norm(quant - base) / np.linalg.norm(base)
    assert 0 < rel < 0.5  # one mantissa bit: tens of percent, never exact here
    # weights that NVFP4 holds with power-of-two matrix scales: the quantised layer is the bf16 layer
    E, I, H = wg.shape
    ex = lambda shape, p: _bf16_bits(np.stack([_exact_nvfp4_matrix(o, rng, *shape, p) for _ in range(E)]))
    eg, eu, ed = ex((I, H), -8), ex((I, H), -9), ex((H, I), -7)
    es = [_bf16_bits(_exact_nvfp4_matrix(o, rng, *s, p)) for s, p in (((32, H), -8), ((32, H), -6), ((H, 32), -9))]
    want = o.forward(x, logits, eg, eu, ed, ws_gate=es[0], ws_up=es[1], ws_down=es[2], **kw).out
    got = o.forward_nvfp4(x, logits, eg, eu, ed, ws_gate=es[0], ws_up=es[1], ws_down=es[2], **kw).out
    np.testing.assert_array_equal(got, want)


PINS = [pin_e4m3_constants, pin_e4m3_decode_matches_torch, pin_e4m3_encode_nearest_even, pin_e2m1_table,
        pin_ue8m0_matches_torch, pin_mxfp8_scale_rule, pin_mxfp8_error_bound, pin_mxfp8_exact_identity,
        pin_nvfp4_scale_rule, pin_nvfp4_error_bound, pin_nvfp4_exact_identity_and_packing, pin_forward_mxfp8,
        pin_forward_output_scales, pin_forward_nvfp4]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(oracle_mod, pin):
    pin(oracle_mod)


# -------------------------------------------------------------- mutants --
MUTANTS = {
    "e4m3_bias_8": ("quant", "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    "e4m3_subnormal_exp": ("quant", "ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    "ties_to_larger": ("quant", "(d == best_d && (c & 1) == 0 && (best & 1) != 0)", "(d == best_d)"),
    "ieee_style_top_exponent": ("quant", "if (e == 15 && m == 7) return NAN;", "if (e == 15) return NAN;"),
    "sign_dropped": ("quant", "return signbit(x) ? (uint8_t)(c | 0x80) : c;", "return c;"),
    "e2m1_bias_0": ("quant", "ldexp(1.0 + 0.5 * (double)m, e - 1)", "ldexp(1.0 + 0.5 * (double)m, e)"),
    "mx_scale_ceil": ("quant", "se = e2 - 1 - 8;", "se = e2 - 8;"),
    "mx_scale_emax_7": ("quant", "se = e2 - 1 - 8;", "se = e2 - 1 - 7;"),
    "nvfp4_global_448x4": ("quant", "amax / 2688.0f", "amax / 1792.0f"),
    "nvfp4_block_max_4": ("quant", "amax_b / (6.0f * st)", "amax_b / (4.0f * st)"),
    "nvfp4_nibbles_swapped": ("quant", "codes[at / 2] |= (uint8_t)(at % 2 == 0 ? q : q << 4);",
                              "codes[at / 2] |= (uint8_t)(at % 2 == 0 ? q << 4 : q);"),
    "mx_dequant_wrong_block": ("quant", "(int)scales[r * (K / 32) + i / 32] - 127", "(int)scales[r * (K / 32) + i / 16 % (K / 32)] - 127"),
    "scale_gate_up_swapped": ("moe", "g *= sg;\n        u *= su;", "g *= su;\n        u *= sg;"),
    "scale_down_dropped": ("moe", "y[o] = sd * a;", "y[o] = a;"),
    "shared_scales_ignored": ("moe", "swiglu_ffn(H, Is, ws_gate, ws_up, ws_down, shared_scales, xt, hbuf, y);",
                              "swiglu_ffn(H, Is, ws_gate, ws_up, ws_down, NULL, xt, hbuf, y);"),
    "scales_of_expert_0": ("moe", "scales ? scales + (size_t)e * 3 : NULL", "scales"),
}


def _load_mutant(name, tmp):
    which, old, new = MUTANTS[name]
    target, other = (QSRC, MSRC) if which == "quant" else (MSRC, QSRC)
    src = open(target).read()
    assert src.count(old) == 1, f"mutant {name}: anchor not found exactly once"
    path_c = os.path.join(tmp, f"{name}.c")
    path_so = os.path.join(tmp, f"lib{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", other, path_c, "-o", path_so, "-lm"],
                   check=True)
    spec = importlib.util.spec_from_file_location(f"oracle_qmutant_{name}", os.path.join(ROOT, "oracle", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    mod._LIB = path_so
    mod.build = lambda force=False: path_so
    return mod


@pytest.fixture(scope="module")
def tmpdir_mod():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_quant_mutant_is_caught(name, tmpdir_mod):
    mod = _load_mutant(name, tmpdir_mod)
    failed = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            failed.append(pin.__name__)
        except (ValueError, FloatingPointError):
            failed.append(pin.__name__ + " (error)")
    assert failed, f"no pin caught the mutant {name}"
    print(name, "caught by", failed)
