"""GPU parity of the CUDA-core chunkwise prefill against the fp64 oracle.

Inputs come from ``gret_inputs``; the oracle runs the recurrent form in fp64 on
the same stored values; the GPU runs through the C ABI.  The fp32 workload is
the small 1 x 2 x 256 x 64 x 64 (chunk 64) case; the others cover ragged tails,
N = 1, odd head sizes, both io dtypes and extreme gates."""
import math

import numpy as np
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


def _dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def _run_and_check(cfg, expect_path=None, check_y=True):
    inp = gi.prefill_inputs(cfg)
    d = _dev(inp)
    if expect_path is not None:
        assert gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk,
                                 gret.Dtype.BF16 if cfg.io == "bf16" else gret.Dtype.F32)[0] == expect_path
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    Y = None
    if check_y:
        Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, eps=cfg.eps,
                            epilogue="none", want_state=False)
    gret.check_device_status()
    O_ref, Y_ref, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps)
    assert_close(O, O_ref, cfg.io, "O")
    assert_close(Sf, S_ref, cfg.io, "S_final")
    if check_y:
        assert_close(Y, Y_ref, cfg.io, "Y")


def test_fp32_workload():
    _run_and_check(gi.C1, expect_path=gret.Path.SIMT)


@pytest.mark.parametrize("B,H,N,dk,dv,chunk,io", [
    (2, 3, 200, 32, 48, 64, "f32"),     # ragged tail, odd dv
    (1, 2, 1, 16, 16, 16, "f32"),       # a single token
    (1, 1, 77, 64, 32, 32, "bf16"),     # bf16 io on the CUDA-core kernel
    (2, 2, 130, 128, 128, 16, "f32"),   # many short chunks, large heads
    (1, 2, 300, 64, 64, 128, "f32"),    # chunk larger than the remaining tail
    # chunk 256, the pages' block size: the chunk does not fit in shared memory
    # and is worked through in blocks of 64 or 16 rows and columns
    (1, 2, 600, 64, 64, 256, "f32"),    # two full chunks and a ragged one
    (1, 2, 700, 128, 128, 256, "bf16"), # the benchmark's head size, chunk 256
    (1, 1, 300, 128, 256, 256, "bf16"), # d_v 256: blocks of 16
    (1, 1, 200, 128, 256, 128, "bf16"), # chunk 128 with d_v 256 (no tensor-core variant)
])
def test_shapes(B, H, N, dk, dv, chunk, io):
    cfg = gi.C1.scaled(B=B, H=H, N=N, dk=dk, dv=dv, chunk=chunk, io=io, seed=100 + N,
                       qkv_var=1.0 / dk, z_dist=tuple((-4.0, 1.0) if h % 2 else (8.0, 0.5)
                                                      for h in range(H)))
    _run_and_check(cfg)


def test_extreme_gates():
    # z = +inf gives gamma = 1 exactly, z = -inf gives gamma = 0 exactly
    cfg = gi.C1.scaled(B=1, H=2, N=150, dk=32, dv=32, chunk=32, seed=7, qkv_var=1 / 32)
    inp = gi.prefill_inputs(cfg)
    z = inp["z"].clone()
    z[0, ::3, 0] = float("inf")
    z[0, 1::5, 0] = float("-inf")
    z[0, :, 1] = -60.0
    inp["z"] = z
    d = _dev(inp)
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk)
    gret.check_device_status()
    O_ref, _, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps)
    assert_close(O, O_ref, "f32", "O")
    assert_close(Sf, S_ref, "f32", "S_final")


def test_output_untouched_outside_tensor():
    # canary bands around O and S_final stay intact
    cfg = gi.C1.scaled(N=100)
    d = _dev(gi.prefill_inputs(cfg))
    pad = 4096
    Obuf = torch.full((pad * 2 + cfg.B * cfg.N * cfg.H * cfg.dv,), 7.25, device="cuda")
    Sbuf = torch.full((pad * 2 + cfg.B * cfg.H * cfg.dk * cfg.dv,), -3.5, device="cuda")
    O = Obuf[pad:pad + cfg.B * cfg.N * cfg.H * cfg.dv].view(cfg.B, cfg.N, cfg.H, cfg.dv)
    Sf = Sbuf[pad:pad + cfg.B * cfg.H * cfg.dk * cfg.dv].view(cfg.B, cfg.H, cfg.dk, cfg.dv)
    gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, O=O, S_final=Sf)
    torch.cuda.synchronize()
    assert torch.all(Obuf[:pad] == 7.25) and torch.all(Obuf[-pad:] == 7.25)
    assert torch.all(Sbuf[:pad] == -3.5) and torch.all(Sbuf[-pad:] == -3.5)
