"""fp64 gradients of the gated-retention prefill (backward oracle).

TEST INFRASTRUCTURE ONLY: imported by the tests; never by the GPU library.

What it computes.  The prefill of "YOCO 深度技术分析", section 2.2, written as
its recurrent definition in plain PyTorch fp64 CPU operations:
    log gamma_n = -softplus(-z_n) / tau            (gamma_n = sigmoid(z_n)^(1/tau))
    S_n         = gamma_n S_{n-1} + K_n^T V_n      (S_0 given or zero)
    Y_n         = Q_n S_n
    O_n         = GroupNorm(Y_n) (.) swish(G_n)    (biased variance, eps, no affine;
                                                    or O = Y for the pre-norm epilogue)
and, for an upstream gradient dO (and optionally dS_N on the final state), the
gradients of  L = <O, dO> + <S_N, dS_N>  with respect to Q, K, V, z, G and S_0,
by PyTorch's reverse-mode differentiation of that loop (a library primitive
used as one step).  The pages give the forward only; the backward is its exact
derivative.

Parity status: pinned by central finite differences in fp64 on small inputs
for every input (``tests/test_oracle_grad_pins.py``), and the forward it
differentiates equals the C oracle's prefill.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch


def _t(x) -> torch.Tensor:
    if isinstance(x, torch.Tensor):
        return x.detach().to(torch.float64).cpu()
    return torch.from_numpy(np.asarray(x, dtype=np.float64))


def forward(Q, K, V, z, G, tau: float, eps: float, S0=None, epilogue: str = "gn_swish"):
    """O [B,N,H,dv], S_N [B,H,dk,dv] as torch fp64 tensors (differentiable)."""
    B, N, H, dk = Q.shape
    dv = V.shape[-1]
    lg = -torch.nn.functional.softplus(-z) / tau
    S = S0 if S0 is not None else torch.zeros((B, H, dk, dv), dtype=torch.float64)
    ys = []
    for n in range(N):
        S = torch.exp(lg[:, n])[:, :, None, None] * S + K[:, n, :, :, None] * V[:, n, :, None, :]
        ys.append(torch.einsum("bhk,bhkv->bhv", Q[:, n], S))
    Y = torch.stack(ys, 1)
    if epilogue == "none":
        return Y, S
    mean = Y.mean(-1, keepdim=True)
    var = ((Y - mean) ** 2).mean(-1, keepdim=True)
    return (Y - mean) / torch.sqrt(var + eps) * (G * torch.sigmoid(G)), S


def prefill_backward(Q, K, V, z, G, tau: float, eps: float, dO, S0=None, dS_final=None,
                     epilogue: str = "gn_swish") -> Dict[str, np.ndarray]:
    """Gradients of <O, dO> + <S_N, dS_final>: dQ, dK, dV, dz, dG (None for the
    pre-norm epilogue) and dS0 (None when S0 is None), as fp64 numpy arrays."""
    Qt, Kt, Vt, zt = (_t(x).requires_grad_(True) for x in (Q, K, V, z))
    Gt = _t(G).requires_grad_(True) if epilogue != "none" else None
    S0t = _t(S0).requires_grad_(True) if S0 is not None else None
    O, S = forward(Qt, Kt, Vt, zt, Gt, tau, eps, S0t, epilogue)
    loss = (O * _t(dO)).sum()
    if dS_final is not None:
        loss = loss + (S * _t(dS_final)).sum()
    wrt = [Qt, Kt, Vt, zt] + ([Gt] if Gt is not None else []) + ([S0t] if S0t is not None else [])
    grads = torch.autograd.grad(loss, wrt, allow_unused=True)
    out = dict(zip(("dQ", "dK", "dV", "dz"), grads[:4]))
    i = 4
    out["dG"] = grads[i] if Gt is not None else None
    i += 1 if Gt is not None else 0
    out["dS0"] = grads[i] if S0t is not None else None
    return {k: (None if v is None else v.numpy()) for k, v in out.items()}
