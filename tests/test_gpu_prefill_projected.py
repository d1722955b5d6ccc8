"""GPU parity of the prefill whose gate logits come from the gate projection
(gret_prefill_projected) against the fp64 oracle's projection followed by its
prefill ("YOCO 深度技术分析", section 2.2: gamma = sigmoid(X W_gamma)^(1/tau)).

X carries a constant feature in channel 0, so that z = X W_gamma has the
workloads' gate-logit means (row 0 of W_gamma) around the random part of the
other channels.  Cases: the fused tensor-core prologue (d_v 256 chunk 64 and
d_v 128 chunk 128; head counts padded to the MMA's 16/32 columns; d_model not
a multiple of the 64-column load box; several token tiles and sequence
segments; a fast/slow head mix), a d_model the fused prologue does not take
(CUDA-core projection, then the tensor-core prefill), and the fp32 path.
O, the pre-norm Y and S_final are compared at the path's tolerance.
"""
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


def _projection_inputs(cfg, d_model, means, seed):
    """X [B,N,d_model] (channel 0 = 1) in cfg.io and W_gamma [d_model,H] fp32
    whose row 0 holds each head's mean gate logit."""
    X = gi.random_unit(seed, 31, (cfg.B, cfg.N, d_model), 0.0, 1.0 / d_model, "f32")
    X[..., 0] = 1.0
    X = gi.to_storage(X.double().numpy(), cfg.io)
    W = gi.random_unit(seed, 32, (d_model, cfg.H), 0.0, 1.5, "f32")
    W[0] = torch.tensor([means[h % len(means)] for h in range(cfg.H)], dtype=torch.float32)
    return X, W


def _check(cfg, d_model, means=(3.0,), seed=0, expect_path=gret.Path.TC):
    io = gret.Dtype.BF16 if cfg.io == "bf16" else gret.Dtype.F32
    path, _ = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io)
    assert path == expect_path
    inp = gi.prefill_inputs(cfg)
    X, W = _projection_inputs(cfg, d_model, means, seed)
    d = {k: v.cuda() for k, v in inp.items()}
    Xd, Wd = X.cuda(), W.cuda()
    O, Sf = gret.prefill_projected(d["Q"], d["K"], d["V"], Xd, Wd, d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    Y, _ = gret.prefill_projected(d["Q"], d["K"], d["V"], Xd, Wd, None, cfg.tau, cfg.chunk, eps=cfg.eps,
                                  epilogue="none", want_state=False)
    gret.check_device_status()
    O_ref, Y_ref, S_ref = oracle.prefill_projected(inp["Q"], inp["K"], inp["V"], X, W, inp["G"], cfg.tau, cfg.eps)
    for name, got, ref in (("Y", Y, Y_ref), ("S_final", Sf, S_ref), ("O", O, O_ref)):
        assert_close(got, ref, cfg.io, name)


def test_tc_dv256_chunk64_ragged_model_dim():
    cfg = gi.C2.scaled(B=2, H=4, N=300, dv=256, chunk=64, seed=801)
    _check(cfg, d_model=200, seed=801)


def test_tc_dv128_chunk128_padded_heads():
    cfg = gi.C2.scaled(B=1, H=20, N=700, dv=128, chunk=128, seed=802)
    _check(cfg, d_model=1024, means=(4.0,), seed=802)


def test_tc_gate_stress_head_mix():
    cfg = gi.C5.scaled(B=1, H=4, N=1000, seed=803)
    _check(cfg, d_model=512, means=(-4.0, 8.0), seed=803)


def test_unaligned_model_dim_takes_cuda_core_projection():
    # d_model = 100: rows of X are not 16-byte multiples apart, so no TMA
    cfg = gi.C2.scaled(B=1, H=2, N=200, dv=256, chunk=64, seed=804)
    _check(cfg, d_model=100, seed=804)


def test_fp32_path():
    cfg = gi.C1.scaled(B=1, H=3, N=150, seed=805)
    _check(cfg, d_model=96, means=(2.0,), seed=805, expect_path=gret.Path.SIMT)


def test_projected_equals_plain_prefill_on_the_same_logits():
    """The fused prologue and the plain gate scan see the same gate: feeding
    gret_prefill the oracle's z = X W_gamma (rounded to fp32) gives outputs
    within the bf16 bounds of the projected call's."""
    cfg = gi.C2.scaled(B=1, H=4, N=500, dv=256, chunk=64, seed=806)
    inp = gi.prefill_inputs(cfg)
    X, W = _projection_inputs(cfg, 256, (3.0,), 806)
    z = torch.from_numpy(oracle.gate_project(X, W).astype(np.float32))
    d = {k: v.cuda() for k, v in inp.items()}
    O1, S1 = gret.prefill_projected(d["Q"], d["K"], d["V"], X.cuda(), W.cuda(), d["G"], cfg.tau, cfg.chunk)
    O2, S2 = gret.prefill(d["Q"], d["K"], d["V"], z.cuda(), d["G"], cfg.tau, cfg.chunk)
    gret.check_device_status()
    assert_close(O1, O2.double().cpu().numpy(), "bf16", "O")
    assert_close(S1, S2.double().cpu().numpy(), "bf16", "S_final")
