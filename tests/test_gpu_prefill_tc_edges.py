"""The method's degenerate gates on the tensor-core (tcgen05/TMEM) prefill.

The gate is gamma = sigmoid(z)^(1/tau) ("YOCO 深度技术分析", section 2.2), so
z -> +inf gives gamma = 1 (no forgetting: causal linear attention) and
z -> -inf gives gamma = 0 (every token forgets all before it).  On the GPU the
per-token log-decay is clamped at -64; below that the state a token carries
is smaller than 1e-27 of its new term, far inside the bf16 tolerance.

Each kernel instantiation of the tensor-core path -- (d_v 256, chunk 64,
pipelined), (d_v 128, chunk 64) and (d_v 128, chunk 128, bf16 state copy) --
runs:

* ``mixed``: heads with z = +inf everywhere, heads with z = -inf on scattered
  tokens (the clamp), heads with z = -60 on scattered tokens, and an ordinary
  head, at tau = 16;
* ``fast``: tau = 1 and z ~ N(-4, 1), a log-decay of about -4 per token, so
  that every block of C/4 columns of P drops by more than 40 and takes the
  direct-exponential branch, and every chunk takes the eager state rescale.

O, the pre-norm Y and S_final are compared element by element with the fp64
oracle at the bf16 bounds (max 2e-2 of max|ref|, relative L2 5e-3).
"""
import numpy as np
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu

INSTANCES = [(256, 64, 330), (128, 64, 270), (128, 128, 390)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_retention_sequence_b200 import build
    build.build()
    gret.load()


def _mixed_gates(z, H):
    """Per head h % 4: 0 -> z = +inf; 1 -> z = -inf on every 7th token from 3;
    2 -> z = -60 on every 5th token from 1; 3 -> unchanged."""
    z = z.clone()
    N = z.shape[1]
    for h in range(H):
        kind = h % 4
        if kind == 0:
            z[:, :, h] = float("inf")
        elif kind == 1:
            z[:, 3:N:7, h] = float("-inf")
        elif kind == 2:
            z[:, 1:N:5, h] = -60.0
    return z


def _run(cfg, inp):
    path, _ = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, gret.Dtype.BF16)
    assert path == gret.Path.TC
    d = {k: v.cuda() for k, v in inp.items()}
    O, Sf = gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps)
    Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, epilogue="none",
                        want_state=False)
    gret.check_device_status()
    O_ref, Y_ref, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps)
    for name, got, ref in (("Y", Y, Y_ref), ("S_final", Sf, S_ref), ("O", O, O_ref)):
        assert_close(got, ref, "bf16", name)
    return Y, Y_ref


@pytest.mark.parametrize("dv,chunk,N", INSTANCES)
def test_mixed_extreme_gates(dv, chunk, N):
    cfg = gi.C2.scaled(B=1, H=4, N=N, dv=dv, chunk=chunk, seed=500 + dv + chunk)
    inp = gi.prefill_inputs(cfg)
    inp["z"] = _mixed_gates(inp["z"], cfg.H)
    Y, Y_ref = _run(cfg, inp)
    # head 0 is causal linear attention: its output keeps growing with the
    # context, unlike the forgetting heads; per head, too, the error stays in bounds
    for h in range(cfg.H):
        assert_close(Y[:, :, h], Y_ref[:, :, h], "bf16", f"Y head {h}")


@pytest.mark.parametrize("dv,chunk,N", INSTANCES)
def test_fast_decay_direct_exponentials(dv, chunk, N):
    cfg = gi.C2.scaled(B=2, H=2, N=N, dv=dv, chunk=chunk, seed=600 + dv + chunk, tau=1.0,
                       z_dist=((-4.0, 1.0),))
    inp = gi.prefill_inputs(cfg)
    # the kernel takes the direct branch where a block of C/4 columns drops by
    # more than 40 in log-decay: make sure this input has such blocks everywhere
    lg = oracle.log_gamma(inp["z"], cfg.tau)
    blk = chunk // 4
    drops = [-lg[0, s + 1:s + blk, 0].sum() for s in range(0, N - blk, blk)]
    assert min(drops) > 40.0
    _run(cfg, inp)


def test_all_gamma_zero_is_diagonal_only():
    """z = -inf everywhere: Y_n = (Q_n . K_n) V_n ("YOCO 深度技术分析" section 2.2
    with gamma = 0), on the pipelined d_v 256 kernel over several segments."""
    cfg = gi.C2.scaled(B=1, H=2, N=1000, dv=256, chunk=64, seed=701)
    inp = gi.prefill_inputs(cfg)
    inp["z"] = torch.full_like(inp["z"], float("-inf"))
    _run(cfg, inp)
    Q, K, V = (oracle.as_f64(inp[n]) for n in ("Q", "K", "V"))
    diag = np.einsum("bnhk,bnhk->bnh", Q, K)[..., None] * V
    d = {k: v.cuda() for k, v in inp.items()}
    Y, _ = gret.prefill(d["Q"], d["K"], d["V"], d["z"], None, cfg.tau, cfg.chunk, epilogue="none",
                        want_state=False)
    assert_close(Y, diag, "bf16", "Y vs (Q.K) V")
