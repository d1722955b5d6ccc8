"""The give-up path of the bounded device waits, made to run without any GPU
fault, trap or hang.

Every mbarrier wait in the tensor-core prefill has a budget; when it runs out
the kernel records a timeout in the device status word, its roles stop issuing
work, the loads and MMAs already issued are awaited, and it returns.
gret_debug_inject_timeout makes the next call's TMA warp wait, before its first
load, on a barrier that nothing arrives at, with a budget of about 2^20
cycles.  The call must come back as GRET_ERR_TIMEOUT through
gret_last_device_status (once), and the next call on the same context must be
correct against the oracle.
"""
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_retention_sequence_b200 import build
    build.build()
    gret.load()


@pytest.mark.parametrize("dv,chunk,N", [(256, 64, 700), (128, 128, 900)])
def test_injected_timeout_is_reported_and_next_call_is_correct(dv, chunk, N):
    cfg = gi.C2.scaled(B=1, H=2, N=N, dv=dv, chunk=chunk, seed=900 + dv)
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC and segs > 1       # the state pass and combine run before the fused kernel
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    assert gret.gret_last_device_status(None) == gret.Status.OK

    gret.gret_debug_inject_timeout(1)
    try:
        gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    finally:
        gret.gret_debug_inject_timeout(0)
    assert gret.gret_last_device_status(None) == gret.Status.ERR_TIMEOUT
    assert gret.gret_last_device_status(None) == gret.Status.OK      # reported once, then cleared

    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    assert gret.gret_last_device_status(None) == gret.Status.OK
    O_ref, _, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps)
    assert_close(O, O_ref, "bf16", "O after the timed-out call")
    assert_close(Sf, S_ref, "bf16", "S_final after the timed-out call")
