"""GPU parity of gret_prefill_from_state (prefill that starts from a given
state S0) against the fp64 oracle run from the same S0.

"YOCO 深度技术分析", sections 5.3.2 and 5.3.3: the state S is all that passes
between blocks and between the devices of Chunk Parallelism, so a prefill
from S0 must equal the tail of one longer prefill whose head left S0 behind.
The cases cover both paths (fp32 CUDA-core, bf16 tensor-core), the tensor-core
variants, a split into sequence segments with state-pass pieces (where S0 has
to enter the segment combine), and two chained calls against one long
oracle prefill."""
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu

TID_S0 = 901


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_retention_sequence_b200 import build
    build.build()
    gret.load()


def _s0(cfg, var=0.04):
    return gi.random_unit(cfg.seed, TID_S0, (cfg.B, cfg.H, cfg.dk, cfg.dv), var=var)


def _check(cfg, expect_path, min_segments=1):
    io = gret.Dtype.BF16 if cfg.io == "bf16" else gret.Dtype.F32
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io)
    assert path == expect_path and segs >= min_segments
    inp = gi.prefill_inputs(cfg)
    S0 = _s0(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    S0d = S0.cuda()
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps, S0=S0d)
    Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, eps=cfg.eps,
                        epilogue="none", want_state=False, S0=S0d)
    gret.check_device_status()
    assert torch.equal(S0d.cpu(), S0)          # S0 is read only
    O_ref, Y_ref, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps,
                                         S0=S0)
    assert_close(Y, Y_ref, cfg.io, "Y")
    assert_close(O, O_ref, cfg.io, "O")
    assert_close(Sf, S_ref, cfg.io, "S_final")


def test_simt_fp32():
    _check(gi.C1.scaled(N=200, seed=31), gret.Path.SIMT)


@pytest.mark.parametrize("N", [64, 200])
def test_tc_dv256_chunk64(N):
    _check(gi.C2.scaled(B=1, H=2, N=N, chunk=64, seed=32 + N), gret.Path.TC)


def test_tc_dv128_chunk128_segments():
    _check(gi.C2.scaled(B=1, H=2, N=1100, dv=128, chunk=128, seed=33, z_dist=((4.0, 1.0),)), gret.Path.TC,
           min_segments=2)


def test_tc_segments_with_pieces():
    # 50 units, 2 segments of 8 chunks, the first cut into state-pass pieces:
    # S0 has to reach segment 1 through the combine pass
    H = 50
    cfg = gi.C2.scaled(B=1, H=H, N=1024, dv=128, chunk=64, seed=34,
                       z_dist=tuple((0.0, 2.0) if h % 2 else (5.0, 1.0) for h in range(H)))
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC and segs == 2
    inp = gi.prefill_inputs(cfg)
    S0 = _s0(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps, S0=S0.cuda())
    gret.check_device_status()
    for h in (0, 1, 26, 49):
        sl = lambda x: x[:, :, h:h + 1]
        O_ref, _, S_ref = oracle.prefill(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["z"]), sl(inp["G"]),
                                         cfg.tau, cfg.eps, S0=S0[:, h:h + 1])
        assert_close(O[:, :, h:h + 1], O_ref, "bf16", f"O head {h}")
        assert_close(Sf[:, h:h + 1], S_ref, "bf16", f"S head {h}")


def test_two_calls_continue_one_sequence():
    # tokens [0, 700) from zero, then [700, 1500) from the state the first call
    # left: the second call must reproduce the tail of one 1500-token prefill
    cfg = gi.C2.scaled(B=1, H=4, N=1500, chunk=64, seed=35)
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    cut = 700
    head = {k: v[:, :cut].contiguous() for k, v in d.items()}
    tail = {k: v[:, cut:].contiguous() for k, v in d.items()}
    _, S_mid = gret.prefill(head["Q"], head["K"], head["V"], head["z"], head["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    O2, S2 = gret.prefill(tail["Q"], tail["K"], tail["V"], tail["z"], tail["G"], cfg.tau, cfg.chunk, eps=cfg.eps,
                          S0=S_mid)
    gret.check_device_status()
    O_ref, _, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps)
    assert_close(O2, O_ref[:, cut:], "bf16", "O of the second call")
    assert_close(S2, S_ref, "bf16", "S_final of the second call")


def test_null_s0_is_the_zero_state():
    cfg = gi.C2.scaled(B=1, H=2, N=300, chunk=64, seed=36)
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O_a, S_a = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    O_b, S_b = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps,
                            S0=torch.zeros_like(S_a))
    gret.check_device_status()
    assert torch.equal(O_a, O_b) and torch.equal(S_a, S_b)
