"""The prefill entry point that allocates nothing (gret_prefill_noalloc).

Some callers -- plugins and custom-op hosts that only receive device pointers,
or code paths where cudaMalloc is not allowed -- cannot hand the library a
workspace.  gret_prefill_noalloc serves them from a fixed scratch array the
library reserves on each GPU.  These tests call it through the C ABI and check
that it gives the same results as gret_prefill with a caller workspace, on two
calls in a row (the shared scratch keeps the first call's contents).

The file is named so that pytest collects it last; it also passes when run
alone in a fresh process.
"""
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
from parity import assert_close


@pytest.fixture(scope="module")
def lib():
    from gated_retention_sequence_b200 import build
    build.build()
    return gret.load()


def test_noalloc_rejects_requests_beyond_its_scratch(lib):
    # 64 units x 200000 tokens needs more decay-sum scratch than the fixed
    # array holds; the call returns before any GPU work (the pointers are
    # never used, so this runs without a GPU too)
    B, H, N, dk, dv, chunk = 4, 16, 200000, 128, 256, 64
    need = gret.gret_prefill_workspace_size(B, H, N, dk, dv, chunk, gret.Dtype.BF16)
    assert need > (32 << 20)
    fake = 0x10000
    st = gret.gret_prefill_noalloc(fake, fake, fake, fake, fake, 16.0, chunk, fake, None, B, H, N, dk, dv,
                                   gret.Dtype.BF16, 1e-5, gret.Epilogue.GN_SWISH, None)
    assert st == gret.Status.ERR_UNSUPPORTED


def _call_noalloc(d, O, S, cfg):
    stream = torch.cuda.current_stream()
    return gret.gret_prefill_noalloc(d["Q"].data_ptr(), d["K"].data_ptr(), d["V"].data_ptr(), d["z"].data_ptr(),
                                     d["G"].data_ptr(), cfg.tau, cfg.chunk, O.data_ptr(), S.data_ptr(),
                                     cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, gret.Dtype.BF16, cfg.eps,
                                     gret.Epilogue.GN_SWISH, stream.cuda_stream)


@pytest.mark.gpu
@pytest.mark.parametrize("N,dv,chunk", [(700, 256, 64), (1100, 128, 128)])
def test_noalloc_matches_workspace_entry_twice(lib, N, dv, chunk):
    cfg = gi.C2.scaled(B=1, H=4, N=N, dv=dv, chunk=chunk, seed=123 + N)
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC and segs > 1     # the split path, which uses scratch
    d = {k: v.cuda() for k, v in gi.prefill_inputs(cfg).items()}
    O_ref, S_ref = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    torch.cuda.synchronize()
    for call in range(2):
        O = torch.full_like(O_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        assert _call_noalloc(d, O, S, cfg) == gret.Status.OK
        gret.check_device_status()
        assert_close(O, O_ref.double().cpu().numpy(), "bf16", f"O, call {call}")
        assert_close(S, S_ref.double().cpu().numpy(), "bf16", f"S_final, call {call}")
