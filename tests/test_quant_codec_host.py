"""The CUDA library's block-scaled weight codes, built for the host, against
the oracle (CPU only).

quant_codec.cuh holds one function per block (MXFP8, NVFP4) that the
quantiser kernels call for every block index; it uses integer and IEEE fp32
arithmetic only, so a host build takes the kernels' decisions.  This test
compiles it with g++ (tests/native/quant_codec_host.cpp) and compares every
code, scale and matrix scale bit for bit with oracle/quant_oracle.c, which
rounds by searching its code tables instead; and the exact bf16 decoders
(code x block scale, built from the bits) with the oracle's dequantisers.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHIM = os.path.join(ROOT, "tests", "native", "quant_codec_host.cpp")


@pytest.fixture(scope="module")
def host():
    with tempfile.TemporaryDirectory() as d:
        so = os.path.join(d, "libquant_codec_host.so")
        subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", SHIM, "-o", so], check=True)
        lib = ctypes.CDLL(so)
        P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        for name in ("host_e4m3_encode", "host_e4m3_decode", "host_e2m1_encode"):
            getattr(lib, name).argtypes = [i64, P, P]
            getattr(lib, name).restype = None
        lib.host_mxfp8_quantize.argtypes = [i64, i32, P, P, P]
        lib.host_nvfp4_quantize.argtypes = [i32, i64, i32, P, P, P, P]
        lib.host_mxfp8_to_bf16.argtypes = [i64, i32, P, P, P]
        lib.host_nvfp4_to_bf16.argtypes = [i64, i32, P, P, P]
        yield lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _encode(lib, name, v):
    v = np.ascontiguousarray(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    getattr(lib, name)(v.size, _p(v), _p(out))
    return out


def _finite_bf16_patterns():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]  # no Inf / NaN


def _values(rng):
    """fp32 values: every finite bf16 value, scaled copies, full-mantissa
    randoms over E4M3's range, exact E4M3 midpoints and their neighbours."""
    bf = (_finite_bf16_patterns().astype(np.uint32) << 16).view(np.float32)
    scaled = np.concatenate([bf[np.abs(bf) < 1e30] * np.float32(2.0 ** k) for k in (-12, -5, 3, 9)])
    rnd = (rng.standard_normal(200000) * np.exp2(rng.uniform(-14, 10, 200000))).astype(np.float32)
    return np.concatenate([bf, scaled, rnd, np.array([0.0, -0.0, 448.0, 449.0, 463.99, 464.0, 465.0, 480.0,
                                                       1e30, -1e30, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11,
                                                       2.0 ** -130], np.float32)])


def test_e4m3_encode_matches_oracle(host, oracle_mod):
    rng = np.random.default_rng(0)
    v = _values(rng)
    v = v[np.isfinite(v)]
    np.testing.assert_array_equal(_encode(host, "host_e4m3_encode", v), oracle_mod.e4m3_encode(v.astype(np.float64)))
    # every midpoint between neighbouring codes, exactly and nudged either way
    pos = np.arange(0x7F, dtype=np.uint8)
    pv = oracle_mod.e4m3_decode(pos)
    mid = ((pv[:-1] + pv[1:]) / 2).astype(np.float32)
    for m in (mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)), -mid):
        np.testing.assert_array_equal(_encode(host, "host_e4m3_encode", m), oracle_mod.e4m3_encode(m.astype(np.float64)))


def test_e4m3_decode_matches_oracle(host, oracle_mod):
    c = np.array([i for i in range(256) if i not in (0x7F, 0xFF)], np.uint8)
    out = np.empty(c.shape, np.float32)
    host.host_e4m3_decode(c.size, _p(c), _p(out))
    np.testing.assert_array_equal(out.astype(np.float64), oracle_mod.e4m3_decode(c))


def test_e2m1_encode_matches_oracle(host, oracle_mod):
    rng = np.random.default_rng(1)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    v = np.concatenate([(rng.standard_normal(200000) * 3).astype(np.float32), mids, -mids,
                        np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(9)),
                        np.array([0.0, -0.0, 6.0, 6.5, 1e30, -1e30, 1e-40], np.float32)])
    np.testing.assert_array_equal(_encode(host, "host_e2m1_encode", v), oracle_mod.e2m1_encode(v.astype(np.float64)))


def _matrix(rng, rows, K, kind):
    if kind == "normal":
        w = rng.standard_normal((rows, K)) * 0.02
    elif kind == "wide":  # block magnitudes from bf16 subnormals to 1e30, zeros, lone values
        w = rng.standard_normal((rows, K)) * np.exp2(rng.integers(-135, 100, (rows, 1)))
        w[0, :48] = 0.0
        w[1, 16:32] = 0.0
        w[1, 20] = -3.0
    else:  # every finite bf16 pattern, in order
        pat = _finite_bf16_patterns()
        pat = pat[: (pat.size // K) * K][: rows * K]
        return pat.reshape(-1, K)
    import torch
    return torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("kind", ["normal", "wide", "patterns"])
def test_mxfp8_blocks_match_oracle(host, oracle_mod, kind):
    rng = np.random.default_rng(2)
    w = np.ascontiguousarray(_matrix(rng, 64, 256, kind))
    rows, K = w.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    host.host_mxfp8_quantize(rows, K, _p(w), _p(codes), _p(scales))
    oc, os_ = oracle_mod.mxfp8_quantize(w)
    np.testing.assert_array_equal(scales, os_)
    np.testing.assert_array_equal(codes, oc)


@pytest.mark.parametrize("kind", ["normal", "wide", "patterns"])
def test_nvfp4_blocks_match_oracle(host, oracle_mod, kind):
    rng = np.random.default_rng(3)
    mats = [np.ascontiguousarray(_matrix(rng, 32, 128, kind)) for _ in range(3)]
    rows, K = mats[0].shape
    w = np.ascontiguousarray(np.stack(mats))
    codes = np.empty((3, rows, K // 2), np.uint8)
    scales = np.empty((3, rows, K // 16), np.uint8)
    st = np.empty(3, np.float32)
    host.host_nvfp4_quantize(3, rows, K, _p(w), _p(codes), _p(scales), _p(st))
    for m in range(3):
        oc, os_, ost = oracle_mod.nvfp4_quantize(mats[m])
        assert st[m] == np.float32(ost)
        np.testing.assert_array_equal(scales[m], os_)
        np.testing.assert_array_equal(codes[m], oc)


def test_mxfp8_decode_to_bf16_is_exact(host, oracle_mod):
    """Every finite E4M3 code at every scale exponent in [-117, 119]: the
    bf16 built from the bits equals the oracle's fp64 dequantisation."""
    se = np.arange(-117, 120)
    codes = np.tile(np.arange(256, dtype=np.uint8), (se.size, 1))
    codes[:, [0x7F, 0xFF]] = 0  # the NaN codes are never produced
    scales = np.repeat((se + 127).astype(np.uint8)[:, None], 256 // 32, axis=1)
    out = np.empty(codes.shape, np.uint16)
    host.host_mxfp8_to_bf16(codes.shape[0], 256, _p(codes), _p(scales), _p(out))
    want = oracle_mod.f64_to_bf16_exact(oracle_mod.mxfp8_dequantize(codes, scales))
    np.testing.assert_array_equal(out, want)


def test_nvfp4_decode_to_bf16_is_exact(host, oracle_mod):
    """Every E2M1 code with every finite E4M3 block scale: element x block
    scale as bf16 equals the oracle's dequantisation (matrix scale 1)."""
    sc = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    q = np.arange(16, dtype=np.uint8)
    codes = np.tile((q[0::2] | (q[1::2] << 4)).astype(np.uint8), (sc.size, 1))  # 16 elements per row
    scales = sc[:, None]
    out = np.empty((sc.size, 16), np.uint16)
    host.host_nvfp4_to_bf16(sc.size, 16, _p(codes), _p(scales), _p(out))
    want = oracle_mod.f64_to_bf16_exact(oracle_mod.nvfp4_dequantize(codes, scales, 1.0))
    np.testing.assert_array_equal(out, want)
