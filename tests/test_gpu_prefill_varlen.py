"""GPU parity of gret_prefill_varlen (packed batches of sequences of
different lengths) against the fp64 oracle run on each sequence alone.

Each case packs sequences of ragged lengths -- one token, one chunk minus or
plus one, empty, several chunks -- into one [total][H][d] batch: a sequence's
last chunk then runs into the next sequence's rows, which must neither enter
its state nor be overwritten by its output.  The rows after the batch are a
canary band that must stay untouched.  On the tensor-core path the work is
planned on the device: long sequences are cut into segments joined by a state
pass, and the cases below include batches where that happens."""
import numpy as np
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu

TID_S0 = 902


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_retention_sequence_b200 import build
    build.build()
    gret.load()


def _run(lengths, dv, chunk, io="bf16", dk=128, H=2, seed=0, with_s0=False, expect_path=gret.Path.TC,
         epilogue="gn_swish"):
    total = int(sum(lengths))
    base = gi.C2 if io == "bf16" else gi.C1
    cfg = base.scaled(B=1, H=H, N=total, dk=dk, dv=dv, chunk=chunk, seed=seed)
    dt = gret.Dtype.BF16 if io == "bf16" else gret.Dtype.F32
    assert gret.prefill_path(len(lengths), H, max(lengths), dk, dv, chunk, dt)[0] == expect_path
    inp = {k: v[0] for k, v in gi.prefill_inputs(cfg).items()}        # [total, H, d]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    d = {k: v.cuda() for k, v in inp.items()}
    cu_d = torch.from_numpy(cu).cuda()
    S0 = gi.random_unit(seed, TID_S0, (len(lengths), H, dk, dv), var=0.04) if with_s0 else None
    pad = 37
    O_buf = torch.full((total + pad, H, dv), float("nan"), dtype=d["V"].dtype, device="cuda")
    O, Sf = gret.prefill_varlen(d["Q"], d["K"], d["V"], d["z"], d["G"], cu_d, max(lengths), cfg.tau, chunk,
                                eps=cfg.eps, O=O_buf[:total], epilogue=epilogue,
                                S0=S0.cuda() if S0 is not None else None)
    gret.check_device_status()
    assert torch.isnan(O_buf[total:].float()).all(), "rows after the batch were written"
    for b, (a0, a1) in enumerate(zip(cu[:-1], cu[1:])):
        sl = lambda x: x[a0:a1][None]
        s0 = S0[b:b + 1] if S0 is not None else None
        if a1 == a0:
            want = s0[0].double().numpy() if s0 is not None else np.zeros((H, dk, dv))
            assert np.array_equal(Sf[b].double().cpu().numpy(), want), f"S_final of empty sequence {b}"
            continue
        O_ref, Y_ref, S_ref = oracle.prefill(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["z"]), sl(inp["G"]),
                                             cfg.tau, cfg.eps, S0=s0)
        ref = Y_ref if epilogue == "none" else O_ref
        assert_close(O[a0:a1][None], ref, io, f"O of sequence {b} ({a1 - a0} tokens)")
        assert_close(Sf[b:b + 1], S_ref, io, f"S_final of sequence {b}")
    return d, cu_d, O, Sf


def test_tc_dv256_chunk64_ragged():
    _run([1, 63, 64, 65, 200, 0, 700, 130], 256, 64, seed=41)


def test_tc_dv256_chunk64_prenorm_and_state():
    _run([129, 7, 300], 256, 64, seed=42, with_s0=True, epilogue="none")


def test_tc_dv128_chunk128_many_segments():
    # 8 units with 9 chunks in the longest sequence: nine segments, the later
    # ones empty for the short sequences
    _run([300, 5, 1100, 128], 128, 128, H=2, seed=43, with_s0=True)


def test_tc_dv128_chunk64():
    _run([500, 64, 1, 77], 128, 64, H=3, seed=44)


def test_simt_fp32():
    _run([10, 0, 100, 256], 64, 64, io="f32", dk=64, seed=45, expect_path=gret.Path.SIMT, with_s0=True)


@pytest.mark.parametrize("lengths,dv,chunk,H", [
    # one and a half work slots' share of these batches is a few chunks, so the
    # long sequences are cut on the device into several segments each (3; 5 and
    # 2; 6 and 2) that a state pass joins; the others stay whole
    ([3000, 50, 1, 64, 200, 0, 700], 256, 64, 16),
    ([2500, 130, 1, 0, 1000], 128, 128, 8),
    ([1900, 3, 640], 128, 64, 12),
])
def test_long_sequences_split_on_the_device(lengths, dv, chunk, H):
    _run(lengths, dv, chunk, H=H, seed=47 + dv + chunk, with_s0=True)


def test_equal_lengths_match_the_uniform_call():
    B, N, H = 3, 333, 2
    cfg = gi.C2.scaled(B=B, H=H, N=N, chunk=64, seed=46)
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    O_u, S_u = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    packed = {k: v.reshape(B * N, *v.shape[2:]) for k, v in d.items()}
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    O_v, S_v = gret.prefill_varlen(packed["Q"], packed["K"], packed["V"], packed["z"], packed["G"], cu, N, cfg.tau,
                                   cfg.chunk, eps=cfg.eps)
    gret.check_device_status()
    # the packed plan may cut the sequences differently from the uniform split:
    # the same values up to the bf16 rounding of the tensor-core path
    assert_close(O_v.reshape(B, N, H, -1), O_u.double().cpu().numpy(), "bf16", "O")
    assert_close(S_v, S_u.double().cpu().numpy(), "bf16", "S_final")


@pytest.mark.parametrize("dv,chunk", [(128, 128), (256, 64)])
def test_many_short_sequences(dv, chunk):
    """200 sequences of 0 to 299 tokens and 4 heads: 800 units, more than five
    times the SMs, in the plan's longest-first order; empty sequences keep
    S_final = S0."""
    lengths = [int(x) for x in np.random.default_rng(5).integers(0, 300, size=200)]
    lengths[3] = 0
    lengths[7] = 1
    _run(lengths, dv, chunk, H=4, seed=48 + dv, with_s0=True)
