"""The failure path on the GPU, without a fault: a pipeline wait that runs out.

The fused expert FFN (one launch for both GEMM phases) makes each down item
wait, bounded, until its group's gate/up items have stored their h rows.
Two test hooks make that wait run out on purpose -- MOE_TEST_STALL_GROUP
gives one group a readiness target its gate/up items never reach, and
MOE_TEST_WAIT_LIMIT_US shortens the wait to 1 ms.  The launch must then end
by itself within milliseconds (no trap, no hang: every role sees the abort
flag, the producer waits for its copies, TMEM is freed), report
MOE_STATUS_TIMEOUT in the status word, and leave the context usable: the
next call on the same workspace, after moe_status_clear, is bit-identical
to a clean run and matches the oracle.
"""
import time

import pytest
import torch

import routed_expert_ffn_renorm_b200 as moe
from routed_expert_ffn_renorm_b200 import workloads as W

from parity_util import check_layer, gpu_forward, lib_config

pytestmark = pytest.mark.gpu

CASES = [
    # mean group 16 tokens: the fused one-launch FFN; stall the shared expert (group E) or routed expert 0
    (W.MoEConfig("stall_shared", T=64, H=256, E=8, I=128, k=2, Is=128), 8),
    (W.MoEConfig("stall_routed", T=200, H=512, E=16, I=128, k=2, Is=64, zipf_alpha=1.0), 0),
]


@pytest.mark.parametrize("cfg,group", CASES, ids=[c.name for c, _ in CASES])
def test_readiness_wait_times_out_and_context_stays_usable(cfg, group, monkeypatch):
    assert torch.cuda.is_available()
    inp = W.make_inputs(cfg, device="cuda")
    ref = gpu_forward(cfg, inp)
    assert ref.status == 0
    ws = torch.zeros(moe.workspace_bytes(lib_config(cfg), cfg.T), dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("MOE_TEST_WAIT_LIMIT_US", "1000")
    monkeypatch.setenv("MOE_TEST_STALL_GROUP", str(group))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    bad = gpu_forward(cfg, inp, ws=ws)
    dt = time.perf_counter() - t0
    assert bad.status & moe.MOE_STATUS_TIMEOUT, f"status {bad.status}"
    assert dt < 2.0, f"the aborted launch took {dt:.2f} s (the 4 s limits should not be reached)"
    monkeypatch.delenv("MOE_TEST_WAIT_LIMIT_US")
    monkeypatch.delenv("MOE_TEST_STALL_GROUP")
    moe.status_clear(ws)
    again = gpu_forward(cfg, inp, ws=ws)
    assert again.status == 0
    assert (again.out_bits == ref.out_bits).all()
    print(cfg.label, check_layer(cfg, inp, again))


@pytest.mark.parametrize("env", [{"MOE_TEST_WAIT_LIMIT_US": "0"}, {"MOE_TEST_WAIT_LIMIT_US": "x"},
                                 {"MOE_TEST_STALL_GROUP": "-1"}, {"MOE_TEST_STALL_GROUP": "9"}])
def test_hooks_reject_bad_values(env, monkeypatch):
    cfg = CASES[0][0]
    inp = W.make_inputs(cfg, device="cuda")
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    with pytest.raises(moe.MoEError):
        gpu_forward(cfg, inp)
