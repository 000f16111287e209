"""bench.py's CPU legs with block-scaled weights (the cpu_baseline and the
reference arm): the oracle inputs bench builds for an MXFP8 or NVFP4 layer
-- only the experts the sample routes to, NVFP4 matrix scales as output
factors -- give the same rows as the oracle's own MXFP8 / NVFP4 layer
functions on all experts.  No GPU."""
import numpy as np
import pytest

import bench
import oracle
from routed_expert_ffn_renorm_b200 import workloads as W


@pytest.mark.parametrize("fmt", ["bf16", "mxfp8", "nvfp4"])
def test_host_inputs_match_the_oracle_layers(fmt):
    cfg = W.MoEConfig("bench_host", T=24, H=256, E=8, I=128, k=2, Is=128, zipf_alpha=1.0)
    inp = W.make_inputs(cfg)
    rows = bench.sample_order(cfg.T)[:4]
    x, logits, wg, wu, wd, extra = bench.host_inputs(cfg, inp, len(rows), fmt)
    got = oracle.forward(x, logits, wg, wu, wd, k=cfg.k, norm_topk=cfg.norm_topk, rows=rows, nthreads=2, I=cfg.I,
                         **extra).out
    b = W.bf16_bits
    shared = dict(ws_gate=b(inp.ws_gate), ws_up=b(inp.ws_up), ws_down=b(inp.ws_down), ws_gvec=b(inp.ws_gvec))
    f = {"bf16": oracle.forward, "mxfp8": oracle.forward_mxfp8, "nvfp4": oracle.forward_nvfp4}[fmt]
    want = f(b(inp.x), logits, b(inp.w_gate), b(inp.w_up), b(inp.w_down), k=cfg.k, norm_topk=cfg.norm_topk,
             rows=rows, nthreads=2, **shared).out
    assert np.array_equal(got, want)


def test_stage_work_weight_bytes():
    """Algorithmic weight bytes per format: 2, 1 + 1/32 and 1/2 + 1/16 a weight."""
    cfg = W.MoEConfig("bytes", T=8, H=256, E=4, I=128, k=1)
    counts = [2, 0, 3, 3]  # three touched experts
    per = {f: bench.stage_work(cfg, counts, f)["ffn"]["bytes"] for f in ("bf16", "mxfp8", "nvfp4")}
    weights = 3 * 3 * cfg.H * cfg.I
    other = per["bf16"] - weights * 2
    assert per["mxfp8"] - other == pytest.approx(weights * (1 + 1 / 32))
    assert per["nvfp4"] - other == pytest.approx(weights * (0.5 + 1 / 16))
