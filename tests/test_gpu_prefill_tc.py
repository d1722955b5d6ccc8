"""GPU parity of the tensor-core (tcgen05/TMEM) chunkwise prefill against the
fp64 oracle, bf16 tolerance (max 2e-2 of max|ref|, relative L2 5e-3) on the
output O, the pre-norm output Y and the final state S.

Small cases cover each kernel variant (d_v 128/256, chunk 64/128), one chunk,
ragged tails and the sequence-segment split with its state carry; the full
workloads run in the benchmark's launch configuration and are compared on a
sample of (batch, head) units that the oracle recomputes on its own."""
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


def _cfg(B, H, N, dv, chunk, seed, z_dist=((3.0, 1.5),)):
    return gi.C2.scaled(B=B, H=H, N=N, dv=dv, chunk=chunk, seed=seed, z_dist=z_dist)


def _check_full(cfg):
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, epilogue="none",
                        want_state=False)
    gret.check_device_status()
    O_ref, Y_ref, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps)
    assert_close(Y, Y_ref, "bf16", "Y")
    assert_close(Sf, S_ref, "bf16", "S_final")
    assert_close(O, O_ref, "bf16", "O")
    return segs


@pytest.mark.parametrize("N", [64, 1, 200, 640])
def test_dv256_chunk64(N):
    _check_full(_cfg(1, 2, N, 256, 64, 200 + N))


@pytest.mark.parametrize("N", [1, 2, 128, 300, 1100])
def test_dv128_chunk128(N):
    _check_full(_cfg(1, 2, N, 128, 128, 300 + N, z_dist=((4.0, 1.0),)))


@pytest.mark.parametrize("N", [1, 130, 700])
def test_dv256_chunk128(N):
    """d_v 256 in 128-token chunks: the output-rows kernel as a CTA pair, each
    CTA owning half of the channels and of the state."""
    _check_full(_cfg(1, 2, N, 256, 128, 600 + N))


def test_dv256_pair_segment_carry():
    """Four units cut into 16 segments each: the pair kernel resumes every
    segment from the state pass's carried state (its own half of each)."""
    segs = _check_full(_cfg(1, 4, 6000, 256, 64, 611, z_dist=((3.0, 1.5), (-4.0, 1.0), (8.0, 0.5), (0.0, 2.0))))
    assert segs > 1


@pytest.mark.parametrize("N", [64, 500])
def test_dv128_chunk64(N):
    _check_full(_cfg(2, 1, N, 128, 64, 400 + N))


def test_segment_carry_many_segments():
    # two units over 40 chunks: split into many segments carried by the state pass
    cfg = _cfg(1, 2, 40 * 64 - 17, 256, 64, 77,
               z_dist=((-4.0, 1.0), (8.0, 0.5)))
    segs = _check_full(cfg)
    assert segs > 1


def test_gate_stress_mixed_heads():
    cfg = gi.C5.scaled(B=1, H=4, N=1500, z_dist=((-4.0, 1.0), (8.0, 0.5), (-4.0, 1.0), (8.0, 0.5)))
    _check_full(cfg)


def _full_workload_sampled(cfg, units):
    """The whole workload in the benchmark's launch configuration; O, the
    pre-norm Y (GroupNorm would hide a uniform scale error, and S_final an
    error confined to the intra-chunk part) and S_final of sampled units
    against the oracle run on each unit alone."""
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, epilogue="none",
                        want_state=False)
    gret.check_device_status()
    assert torch.isfinite(O.float()).all() and torch.isfinite(Sf).all() and torch.isfinite(Y.float()).all()
    for b, h in units:
        u = gi.prefill_unit_inputs(cfg, b, h)
        for name in ("Q", "V", "z"):
            assert torch.equal(u[name], inp[name][b, :, h])
        O_ref, Y_ref, S_ref = oracle.prefill(u["Q"][None, :, None], u["K"][None, :, None], u["V"][None, :, None],
                                             u["z"][None, :, None], u["G"][None, :, None], cfg.tau, cfg.eps)
        assert_close(O[b, :, h], O_ref[0, :, 0], "bf16", f"O unit {(b, h)}")
        assert_close(Y[b, :, h], Y_ref[0, :, 0], "bf16", f"Y unit {(b, h)}")
        assert_close(Sf[b, h], S_ref[0, 0], "bf16", f"S unit {(b, h)}")


@pytest.mark.slow
def test_full_workload_b4_h16_n4096_dv256():
    _full_workload_sampled(gi.C2, [(0, 0), (1, 7), (3, 15)])


@pytest.mark.slow
def test_full_workload_b1_h32_n65536_dv128():
    _full_workload_sampled(gi.C3, [(0, 0), (0, 31)])


@pytest.mark.slow
def test_full_workload_gate_stress_b2_h16_n32768():
    _full_workload_sampled(gi.C5, [(0, 0), (1, 8), (1, 15)])


@pytest.mark.parametrize("dv,chunk", [(256, 64), (128, 128), (128, 64)])
def test_lazy_and_eager_state_scaling(dv, chunk):
    """148 units (one segment each, 8-16 chunks): moderate gates (z ~ N(-2,1),
    log-decay about -8.5 per 64 tokens) run several lazy chunks between eager
    rescales; the other heads stay near gamma = 1 (lazy throughout)."""
    H = 148
    cfg = _cfg(1, H, 1024, dv, chunk, 91, z_dist=tuple((-2.0, 1.0) if h % 2 else (6.0, 1.0) for h in range(H)))
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC and segs == 1
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, epilogue="none",
                        want_state=False)
    gret.check_device_status()
    for h in (0, 1, 77, 146, 147):
        sl = lambda x: x[:, :, h:h + 1]
        O_ref, Y_ref, S_ref = oracle.prefill(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["z"]),
                                             sl(inp["G"]), cfg.tau, cfg.eps)
        assert_close(Y[:, :, h:h + 1], Y_ref, "bf16", f"Y head {h}")
        assert_close(O[:, :, h:h + 1], O_ref, "bf16", f"O head {h}")
        assert_close(Sf[:, h:h + 1], S_ref, "bf16", f"S head {h}")


def test_state_pass_pieces():
    """50 units split into 2 segments of 8 chunks: the state pass cuts the first
    segment into pieces (about one CTA per SM) folded back by the combine pass."""
    H = 50
    cfg = _cfg(1, H, 1024, 128, 64, 93, z_dist=tuple((0.0, 2.0) if h % 2 else (5.0, 1.0) for h in range(H)))
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC and segs == 2
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    gret.check_device_status()
    for h in (0, 1, 25, 49):
        sl = lambda x: x[:, :, h:h + 1]
        O_ref, _, S_ref = oracle.prefill(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["z"]),
                                         sl(inp["G"]), cfg.tau, cfg.eps)
        assert_close(O[:, :, h:h + 1], O_ref, "bf16", f"O head {h}")
        assert_close(Sf[:, h:h + 1], S_ref, "bf16", f"S head {h}")


@pytest.mark.parametrize("dv,chunk,N", [(128, 64, 14245), (128, 128, 28501)])
def test_state_pass_long_and_short_pieces(dv, chunk, N):
    """Eight units split into 18 segments: the 136 segments before the last of
    each unit are fewer than the SMs but more than half of them, so the state
    pass cuts each into a long and a short piece (more than 13 chunks per
    segment); the carried states must be those of the unsplit recurrence."""
    cfg = _cfg(1, 8, N, dv, chunk, 500 + chunk, z_dist=((4.0, 1.0),))
    segs = _check_full(cfg)
    assert segs == 18
