"""Pins of the backward oracle (oracle/gret_oracle_grad.py) on the CPU.

The gradients are checked against central finite differences of the loss
<O, dO> + <S_N, dS_N> in fp64 -- a check that does not go through the
oracle's differentiation -- for every input, both epilogues and with an initial
state; and the forward being differentiated is checked against the C oracle's
prefill."""
import numpy as np
import pytest
import torch

import oracle
from oracle import gret_oracle_grad as og


def _case(seed, B=1, N=5, H=2, dk=3, dv=4, with_s0=True):
    rng = np.random.default_rng(seed)
    d = dict(Q=rng.normal(0, 0.5, (B, N, H, dk)), K=rng.normal(0, 0.5, (B, N, H, dk)),
             V=rng.normal(0, 0.5, (B, N, H, dv)), z=rng.normal(1.0, 1.5, (B, N, H)),
             G=rng.normal(0, 1.0, (B, N, H, dv)))
    S0 = rng.normal(0, 0.3, (B, H, dk, dv)) if with_s0 else None
    dO = rng.normal(0, 1.0, (B, N, H, dv))
    dSf = rng.normal(0, 1.0, (B, H, dk, dv))
    return d, S0, dO, dSf


def _loss(d, S0, dO, dSf, tau, eps, epilogue):
    t = {k: torch.from_numpy(v) for k, v in d.items()}
    O, S = og.forward(t["Q"], t["K"], t["V"], t["z"], t["G"], tau, eps,
                      torch.from_numpy(S0) if S0 is not None else None, epilogue)
    return float((O * torch.from_numpy(dO)).sum() + (S * torch.from_numpy(dSf)).sum())


@pytest.mark.parametrize("epilogue,with_s0", [("gn_swish", True), ("none", True), ("gn_swish", False)])
def test_gradients_match_finite_differences(epilogue, with_s0):
    tau, eps, h = 4.0, 1e-5, 1e-6
    d, S0, dO, dSf = _case(7, with_s0=with_s0)
    g = og.prefill_backward(d["Q"], d["K"], d["V"], d["z"], d["G"], tau, eps, dO, S0=S0, dS_final=dSf,
                            epilogue=epilogue)
    names = ["Q", "K", "V", "z"] + (["G"] if epilogue != "none" else []) + (["S0"] if with_s0 else [])
    rng = np.random.default_rng(3)
    for name in names:
        base = S0 if name == "S0" else d[name]
        grad = g["dS0"] if name == "S0" else g["d" + name]
        for _ in range(6):                       # six random coordinates of each input
            idx = tuple(rng.integers(0, s) for s in base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += h
            minus[idx] -= h
            if name == "S0":
                fp = _loss(d, plus, dO, dSf, tau, eps, epilogue)
                fm = _loss(d, minus, dO, dSf, tau, eps, epilogue)
            else:
                fp = _loss(dict(d, **{name: plus}), S0, dO, dSf, tau, eps, epilogue)
                fm = _loss(dict(d, **{name: minus}), S0, dO, dSf, tau, eps, epilogue)
            fd = (fp - fm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])
    if epilogue == "none":
        assert g["dG"] is None
    if not with_s0:
        assert g["dS0"] is None


def test_forward_equals_the_c_oracle():
    d, S0, _, _ = _case(11, B=2, N=37, H=2, dk=5, dv=6)
    t = {k: torch.from_numpy(v) for k, v in d.items()}
    O, S = og.forward(t["Q"], t["K"], t["V"], t["z"], t["G"], 16.0, 1e-5, torch.from_numpy(S0))
    O_ref, _, S_ref = oracle.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], 16.0, 1e-5, S0=S0)
    np.testing.assert_allclose(O.numpy(), O_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S.numpy(), S_ref, rtol=1e-10, atol=1e-12)
