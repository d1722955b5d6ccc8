"""GPU parity of the sequence-parallel prefill's computing steps on one device.

The slices of one sequence are processed in turn on the same GPU: the
state-only pass of each slice (gret_prefill_state), the fold of the slices
before it (gret_state_fold), and the prefill of the slice from that state --
either from scratch (gret_prefill_from_state) or resumed from the state pass's
workspace (gret_prefill_resume), which shifts the pieces the state pass folded
from zero by the slice's initial state.
The concatenated outputs and the last state are compared with one oracle
prefill of the whole sequence; the state-only pass is also compared with the
oracle's state and decay of each slice alone.  (The all-gather between devices
is covered by the gloo test of the same code on the CPU.)"""
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


def _run(cfg, cuts, expect_path, with_s0, resume=False):
    io = gret.Dtype.BF16 if cfg.io == "bf16" else gret.Dtype.F32
    assert gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io)[0] == expect_path
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    S0 = gi.random_unit(cfg.seed, 904, (cfg.B, cfg.H, cfg.dk, cfg.dv), var=0.04) if with_s0 else None
    S0d = S0.cuda() if with_s0 else None
    sl = [{k: v[:, a:b].contiguous() for k, v in d.items()} for a, b in zip(cuts[:-1], cuts[1:])]
    # one workspace per slice, kept for the resumed prefill of that slice
    wss = []
    for s in sl:
        n = s["K"].shape[1]
        need = gret.gret_prefill_state_workspace_size(cfg.B, cfg.H, n, cfg.dk, cfg.dv, cfg.chunk, io)
        wss.append(torch.empty(max(need, 256), dtype=torch.uint8, device="cuda"))
    parts = [gret.prefill_state(s["K"], s["V"], s["z"], cfg.tau, cfg.chunk, workspace=w) for s, w in zip(sl, wss)]
    gret.check_device_status()
    # the state-only pass alone, against the oracle on each slice
    for (a, b), (dS, decay) in zip(zip(cuts[:-1], cuts[1:]), parts):
        lg = oracle.log_gamma(inp["z"][:, a:b], cfg.tau)
        _, S_ref = oracle.recurrent(inp["K"][:, a:b], inp["K"][:, a:b], inp["V"][:, a:b], lg)
        assert_close(dS, S_ref, cfg.io, f"dS of slice {a}:{b}")
        np.testing.assert_allclose(decay.cpu().double().numpy(), np.asarray(lg).sum(axis=1), rtol=1e-4, atol=1e-3)
    dS_all = torch.stack([p[0] for p in parts])
    decay_all = torch.stack([p[1] for p in parts])
    outs = []
    for r, s in enumerate(sl):
        S_in = gret.state_fold(dS_all, decay_all, r, S0=S0d)
        O, S = gret.prefill(s["Q"], s["K"], s["V"], s["z"], s["G"], cfg.tau, cfg.chunk, eps=cfg.eps, S0=S_in,
                            workspace=wss[r] if resume else None, resume=resume)
        outs.append((O, S))
    S_whole = gret.state_fold(dS_all, decay_all, len(sl), S0=S0d)
    gret.check_device_status()
    O_ref, _, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps, S0=S0)
    assert_close(torch.cat([o for o, _ in outs], dim=1), O_ref, cfg.io, "O of all slices")
    assert_close(outs[-1][1], S_ref, cfg.io, "state after the last slice")
    assert_close(S_whole, S_ref, cfg.io, "fold of every slice")


def test_tc_three_ragged_slices():
    cfg = gi.C2.scaled(B=1, H=4, N=3000, chunk=64, seed=61)
    _run(cfg, (0, 700, 1500, 3000), gret.Path.TC, with_s0=True)


def test_tc_dv128_chunk128():
    cfg = gi.C2.scaled(B=2, H=2, N=2000, dv=128, chunk=128, seed=62, z_dist=((4.0, 1.0),))
    _run(cfg, (0, 1000, 1130, 2000), gret.Path.TC, with_s0=False)


def test_tc_gate_stress():
    cfg = gi.C2.scaled(B=1, H=2, N=2048, chunk=64, seed=63, z_dist=((-4.0, 1.0), (8.0, 0.5)))
    _run(cfg, (0, 1024, 2048), gret.Path.TC, with_s0=True)


def test_simt_fp32():
    cfg = gi.C1.scaled(N=256, seed=64)
    _run(cfg, (0, 100, 256), gret.Path.SIMT, with_s0=True)


@pytest.mark.parametrize("dv,chunk,N,cuts", [(256, 64, 3000, (0, 700, 1500, 3000)),
                                             (128, 128, 2000, (0, 1000, 1130, 2000)),
                                             (128, 64, 5000, (0, 2500, 5000))])
def test_tc_resumed_from_the_state_pass(dv, chunk, N, cuts):
    cfg = gi.C2.scaled(B=1, H=4, N=N, dv=dv, chunk=chunk, seed=65 + dv + chunk,
                       z_dist=((-4.0, 1.0), (8.0, 0.5), (3.0, 1.5), (0.0, 2.0)))
    _run(cfg, cuts, gret.Path.TC, with_s0=True, resume=True)


def test_simt_resumed_is_from_state():
    cfg = gi.C1.scaled(N=256, seed=66)
    _run(cfg, (0, 100, 256), gret.Path.SIMT, with_s0=True, resume=True)


def test_fold_on_unaligned_buffers():
    """gret_state_fold with its increments, initial state and output one float
    past a 16-byte boundary (the fold's element-wise variant): folding the
    state-only passes of two slices from S0 gives the oracle's state after the
    whole sequence."""
    cfg = gi.C2.scaled(B=1, H=2, N=700, chunk=64, seed=67)
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    S0 = gi.random_unit(cfg.seed, 904, (cfg.B, cfg.H, cfg.dk, cfg.dv), var=0.04)
    parts = [gret.prefill_state(d["K"][:, a:b].contiguous(), d["V"][:, a:b].contiguous(),
                                d["z"][:, a:b].contiguous(), cfg.tau, cfg.chunk) for a, b in ((0, 300), (300, 700))]

    def off_by_one_float(x):
        buf = torch.empty(x.numel() + 1, dtype=torch.float32, device="cuda")
        v = buf[1:].view(x.shape)
        v.copy_(x)
        assert v.data_ptr() % 16 == 4
        return v

    dS_all = off_by_one_float(torch.stack([p[0] for p in parts]))
    decay_all = torch.stack([p[1] for p in parts])
    out = off_by_one_float(torch.zeros((cfg.B, cfg.H, cfg.dk, cfg.dv), device="cuda"))
    S = gret.state_fold(dS_all, decay_all, 2, S0=off_by_one_float(S0.cuda()), out=out)
    gret.check_device_status()
    lg = oracle.log_gamma(inp["z"], cfg.tau)
    _, S_ref = oracle.recurrent(inp["K"], inp["K"], inp["V"], lg, S0=S0)
    assert_close(S, S_ref, cfg.io, "fold of both slices from S0")
