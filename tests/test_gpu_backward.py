"""GPU parity of gret_prefill_backward against the fp64 backward oracle
(autograd of the recurrent definition, itself pinned by finite differences).

Cases: the fp32 path (1e-4 of max|ref|) with an initial state and a gradient
on the final state, both epilogues, ragged chunk tails; bf16 inputs and
gradients at the benchmark's head sizes on the tensor-core path (bf16
tolerance; d_v 256 runs on CTA pairs, d_v 128 on single CTAs) over one and
several chunks, and the benchmark's full length on sampled units; a
gate-stress mix of fast- and slow-decaying heads; bf16 with d_k 64 (the
CUDA-core chunk kernels); head sizes that are not multiples of 32 (the serial
path)."""
import numpy as np
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
from oracle import gret_oracle_grad as og
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_retention_sequence_b200 import build
    build.build()
    gret.load()


def _run(cfg, epilogue="gn_swish", with_s0=True, with_dsf=True):
    inp = gi.prefill_inputs(cfg)
    shape_o = (cfg.B, cfg.N, cfg.H, cfg.dv)
    shape_s = (cfg.B, cfg.H, cfg.dk, cfg.dv)
    dO = gi.random_unit(cfg.seed, 910, shape_o, io=cfg.io)
    S0 = gi.random_unit(cfg.seed, 911, shape_s, var=0.04) if with_s0 else None
    dSf = gi.random_unit(cfg.seed, 912, shape_s, var=0.01) if with_dsf else None
    d = {k: v.cuda() for k, v in inp.items()}
    got = gret.prefill_backward(d["Q"], d["K"], d["V"], d["z"], d["G"] if epilogue != "none" else None, dO.cuda(),
                                cfg.tau, eps=cfg.eps, epilogue=epilogue,
                                S0=S0.cuda() if with_s0 else None, dS_final=dSf.cuda() if with_dsf else None)
    gret.check_device_status()
    ref = og.prefill_backward(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps, dO, S0=S0,
                              dS_final=dSf, epilogue=epilogue)
    for name in ("dQ", "dK", "dV"):
        assert_close(got[name], ref[name], cfg.io, name)
    assert_close(got["dz"], ref["dz"], "f32" if cfg.io == "f32" else "bf16", "dz")
    if epilogue != "none":
        assert_close(got["dG"], ref["dG"], cfg.io, "dG")
    else:
        assert got["dG"] is None
    if with_s0:
        assert_close(got["dS0"], ref["dS0"], "f32" if cfg.io == "f32" else "bf16", "dS0")


@pytest.mark.parametrize("epilogue", ["gn_swish", "none"])
def test_fp32_with_states(epilogue):
    _run(gi.C1.scaled(N=200, seed=71), epilogue=epilogue)


def test_fp32_from_zero_one_block():
    _run(gi.C1.scaled(N=17, seed=72), with_s0=False, with_dsf=False)


def test_bf16_benchmark_heads():
    _run(gi.C2.scaled(B=1, H=2, N=100, seed=73))


def test_bf16_gate_stress():
    _run(gi.C2.scaled(B=1, H=2, N=160, dv=128, seed=74, z_dist=((-4.0, 1.0), (8.0, 0.5))))


def test_bf16_several_chunks_ragged():
    # the tensor-core path: three 128-token chunks, the last one 44 tokens long,
    # both states given
    cfg = gi.C2.scaled(B=2, H=1, N=300, seed=75)
    assert gret.gret_prefill_backward_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, gret.Dtype.BF16) == 6
    _run(cfg)


def test_fp32_prenorm_many_chunks():
    _run(gi.C1.scaled(N=130, dk=32, dv=96, seed=76), epilogue="none")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_serial_path_odd_head_sizes(io):
    base = gi.C1 if io == "f32" else gi.C2
    cfg = base.scaled(B=1, H=2, N=70, dk=48, dv=80, seed=77)
    dt = gret.Dtype.F32 if io == "f32" else gret.Dtype.BF16
    assert gret.gret_prefill_backward_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, dt) == 2
    _run(cfg)


def test_bf16_tensor_core_path_prenorm():
    # d_k 128 bf16 takes the tensor-core (tcgen05) kernels; the plain epilogue (dy = dO)
    _run(gi.C2.scaled(B=1, H=2, N=200, seed=78), epilogue="none")


def test_bf16_cuda_core_chunked_path():
    # bf16 with d_k 64: the CUDA-core chunk kernels (chunks of 64 tokens)
    cfg = gi.C2.scaled(B=1, H=2, N=150, dk=64, dv=128, seed=79)
    assert gret.gret_prefill_backward_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, gret.Dtype.BF16) == 5
    _run(cfg)


@pytest.mark.slow
def test_bf16_full_benchmark_length_sampled_units():
    """The benchmark's whole backward (B4 H16 N4096, d_k 128, d_v 256, both
    states given), as the bench launches it; sampled (batch, head) units -- each
    depends on its own inputs only -- against the oracle run on that unit alone
    over all 4096 tokens."""
    cfg = gi.C2
    inp = gi.prefill_inputs(cfg)
    shape_o = (cfg.B, cfg.N, cfg.H, cfg.dv)
    shape_s = (cfg.B, cfg.H, cfg.dk, cfg.dv)
    dO = gi.random_unit(cfg.seed, 910, shape_o, io=cfg.io)
    S0 = gi.random_unit(cfg.seed, 911, shape_s, var=0.04)
    dSf = gi.random_unit(cfg.seed, 912, shape_s, var=0.01)
    d = {k: v.cuda() for k, v in inp.items()}
    got = gret.prefill_backward(d["Q"], d["K"], d["V"], d["z"], d["G"], dO.cuda(), cfg.tau, eps=cfg.eps,
                                S0=S0.cuda(), dS_final=dSf.cuda())
    gret.check_device_status()
    for b, h in ((0, 0), (3, 15)):
        u = lambda x: x[b:b + 1, :, h:h + 1]  # noqa: E731
        ref = og.prefill_backward(u(inp["Q"]), u(inp["K"]), u(inp["V"]), u(inp["z"]), u(inp["G"]), cfg.tau,
                                  cfg.eps, u(dO), S0=S0[b:b + 1, h:h + 1], dS_final=dSf[b:b + 1, h:h + 1])
        for name in ("dQ", "dK", "dV", "dG"):
            assert_close(u(got[name]), ref[name], "bf16", f"{name} unit {(b, h)}")
        assert_close(got["dz"][b:b + 1, :, h:h + 1], ref["dz"], "bf16", f"dz unit {(b, h)}")
        assert_close(got["dS0"][b:b + 1, h:h + 1], ref["dS0"], "bf16", f"dS0 unit {(b, h)}")


def _sampled_units(cfg, units, seed_s0=911):
    """The whole backward of cfg on the GPU; the listed (batch, head) units
    against the oracle run on that unit alone."""
    inp = gi.prefill_inputs(cfg)
    shape_o = (cfg.B, cfg.N, cfg.H, cfg.dv)
    shape_s = (cfg.B, cfg.H, cfg.dk, cfg.dv)
    dO = gi.random_unit(cfg.seed, 910, shape_o, io=cfg.io)
    S0 = gi.random_unit(cfg.seed, seed_s0, shape_s, var=0.04)
    dSf = gi.random_unit(cfg.seed, 912, shape_s, var=0.01)
    d = {k: v.cuda() for k, v in inp.items()}
    got = gret.prefill_backward(d["Q"], d["K"], d["V"], d["z"], d["G"], dO.cuda(), cfg.tau, eps=cfg.eps,
                                S0=S0.cuda(), dS_final=dSf.cuda())
    gret.check_device_status()
    for b, h in units:
        u = lambda x: x[b:b + 1, :, h:h + 1]  # noqa: E731
        ref = og.prefill_backward(u(inp["Q"]), u(inp["K"]), u(inp["V"]), u(inp["z"]), u(inp["G"]), cfg.tau,
                                  cfg.eps, u(dO), S0=S0[b:b + 1, h:h + 1], dS_final=dSf[b:b + 1, h:h + 1])
        for name in ("dQ", "dK", "dV", "dG"):
            assert_close(u(got[name]), ref[name], "bf16", f"{name} unit {(b, h)}")
        assert_close(got["dz"][b:b + 1, :, h:h + 1], ref["dz"], "bf16", f"dz unit {(b, h)}")
        assert_close(got["dS0"][b:b + 1, h:h + 1], ref["dS0"], "bf16", f"dS0 unit {(b, h)}")


@pytest.mark.slow
def test_bf16_dv128_more_chunks_than_ctas():
    """d_v 128 (one CTA per chunk): 2 heads x 81 chunks of a ragged 10300-token
    sequence are more chunks than SMs, so the persistent gradient kernels take
    several chunks each; fast-decaying gates."""
    cfg = gi.C2.scaled(B=1, H=2, N=10300, dv=128, seed=81, z_dist=((-2.0, 1.0),))
    _sampled_units(cfg, [(0, 1)])


@pytest.mark.slow
def test_bf16_dv256_pairs_more_chunks_than_pairs():
    """d_v 256 (a CTA pair per chunk): 3 heads x 26 chunks of a 3288-token
    sequence (the last chunk 88 tokens) are more chunks than SM pairs."""
    cfg = gi.C2.scaled(B=1, H=3, N=3288, seed=82)
    _sampled_units(cfg, [(0, 0), (0, 2)])


@pytest.mark.parametrize("dv,N", [(256, 1), (256, 129), (128, 1), (128, 129)])
def test_bf16_tensor_core_edge_lengths(dv, N):
    """The tensor-core backward on a single token and on one chunk plus one token
    (the last chunk's one row), without states: nearly every launched CTA of the
    persistent kernels has no chunk to take."""
    _run(gi.C2.scaled(B=1, H=1, N=N, dv=dv, seed=90 + N + dv), with_s0=False, with_dsf=False)
