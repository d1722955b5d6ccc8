"""The chunk-parallel decomposition of the backward, as the kernels compute it,
restated in numpy (fp64) and checked against the backward oracle (autograd of
the recurrent definition, itself pinned by finite differences).

Steps per (batch, head): the state increment and decay of every chunk, a scan
for the state before every chunk, per chunk y and the GroupNorm * swish backward
and G_c = sum_t e^{b_t} q_t^T dy_t, a reverse scan for the gradient at every
chunk's end, then per chunk dq, dk, dv and the gate gradient from four sums.
The forward is the chunkwise form of "YOCO 深度技术分析" (sections 2.2, 5.3.2).
A mistake in any of the formulas -- a sign, a missing decay factor, a wrong
prefix/suffix range in the gate sums -- shows as a gradient mismatch here,
independently of the GPU."""
import numpy as np
import pytest

from oracle import gret_oracle_grad as og


def _log_gamma(z, tau):
    return np.maximum(-np.logaddexp(0.0, -z) / tau, -64.0)


def _chunked_backward(Q, K, V, z, G, dO, tau, eps, S0, dSf, C, gn):
    B, N, H, dk = Q.shape
    dv = V.shape[-1]
    nc = -(-N // C)
    out = {name: np.zeros_like(x) for name, x in (("dQ", Q), ("dK", K), ("dV", V), ("dz", z), ("dG", V))}
    out["dS0"] = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            lg = _log_gamma(z[b, :, h], tau)
            chunks = []
            for c in range(nc):
                n0 = c * C
                L = min(C, N - n0)
                bc = np.cumsum(lg[n0:n0 + L])
                chunks.append((n0, L, bc, bc[-1]))
            # 1 + 2: state before every chunk
            S = np.zeros((nc, dk, dv))
            S[0] = S0[b, h] if S0 is not None else 0.0
            for c in range(1, nc):
                n0, L, bc, bL = chunks[c - 1]
                inc = (K[b, n0:n0 + L, h] * np.exp(bL - bc)[:, None]).T @ V[b, n0:n0 + L, h]
                S[c] = np.exp(bL) * S[c - 1] + inc
            # 3: dy and G_c per chunk
            dS = np.zeros((nc, dk, dv))
            dys = []
            for c in range(nc):
                n0, L, bc, bL = chunks[c]
                q, k, v = Q[b, n0:n0 + L, h], K[b, n0:n0 + L, h], V[b, n0:n0 + L, h]
                do = dO[b, n0:n0 + L, h]
                if gn:
                    A = (q @ k.T) * np.tril(np.exp(bc[:, None] - bc[None, :]))
                    y = A @ v + np.exp(bc)[:, None] * (q @ S[c])
                    mean = y.mean(1, keepdims=True)
                    rstd = 1.0 / np.sqrt(((y - mean) ** 2).mean(1, keepdims=True) + eps)
                    n = (y - mean) * rstd
                    g = G[b, n0:n0 + L, h]
                    sg = 1.0 / (1.0 + np.exp(-g))
                    out["dG"][b, n0:n0 + L, h] = do * n * sg * (1.0 + g * (1.0 - sg))
                    dn = do * g * sg
                    dy = rstd * (dn - dn.mean(1, keepdims=True) - n * (dn * n).mean(1, keepdims=True))
                else:
                    dy = do
                dys.append(dy)
                dS[c] = (q * np.exp(bc)[:, None]).T @ dy
            # 4: gradient at every chunk's end, and at the start of the sequence
            cur = dSf[b, h] if dSf is not None else np.zeros((dk, dv))
            for c in range(nc - 1, -1, -1):
                g_c = dS[c].copy()
                dS[c] = cur
                cur = np.exp(chunks[c][3]) * cur + g_c
            out["dS0"][b, h] = cur
            # 5: per chunk gradients
            for c in range(nc):
                n0, L, bc, bL = chunks[c]
                q, k, v = Q[b, n0:n0 + L, h], K[b, n0:n0 + L, h], V[b, n0:n0 + L, h]
                dy, Sc, dSp = dys[c], S[c], dS[c]
                mask = np.tril(np.ones((L, L)))
                E = np.exp(bc[:, None] - bc[None, :]) * mask
                A = (q @ k.T) * E
                D = (dy @ v.T) * mask
                eb, wl = np.exp(bc), np.exp(bL - bc)
                dyS, VdS = dy @ Sc.T, v @ dSp.T
                out["dQ"][b, n0:n0 + L, h] = (D * E) @ k + eb[:, None] * dyS
                out["dK"][b, n0:n0 + L, h] = (D * E).T @ q + wl[:, None] * VdS
                out["dV"][b, n0:n0 + L, h] = A.T @ dy + wl[:, None] * (k @ dSp)
                M = A * D
                prefix = np.cumsum(M, 1) - M                       # sum_{s < j} M_ts
                F = np.array([prefix[j:, j].sum() for j in range(L)])
                rr = eb * (q * dyS).sum(1)
                us = wl * (k * VdS).sum(1)
                dlg = F + np.cumsum(rr[::-1])[::-1] + np.exp(bL) * (dSp * Sc).sum() + (np.cumsum(us) - us)
                zz = z[b, n0:n0 + L, h]
                deriv = np.where(lg[n0:n0 + L] > -64.0, (1.0 - 1.0 / (1.0 + np.exp(-zz))) / tau, 0.0)
                out["dz"][b, n0:n0 + L, h] = dlg * deriv
    return out


@pytest.mark.parametrize("B,N,H,dk,dv,C,gn", [
    (1, 37, 2, 4, 6, 8, True),      # ragged last chunk
    (2, 16, 1, 3, 5, 4, False),     # plain epilogue, chunks that divide N
    (1, 70, 1, 8, 8, 64, True),     # one full chunk and a short one
    (1, 9, 1, 2, 3, 16, True),      # a single partial chunk
    (1, 300, 1, 8, 8, 128, True),   # the tensor-core kernels' chunk: two full chunks and a 44-token one
])
def test_chunk_decomposition_matches_the_oracle(B, N, H, dk, dv, C, gn):
    rng = np.random.default_rng(100 + N)
    Q, K = rng.normal(0, 0.5, (B, N, H, dk)), rng.normal(0, 0.5, (B, N, H, dk))
    V, G, dO = rng.normal(0, 0.5, (B, N, H, dv)), rng.normal(0, 1, (B, N, H, dv)), rng.normal(0, 1, (B, N, H, dv))
    z = rng.normal(1.0, 1.5, (B, N, H))
    S0, dSf = rng.normal(0, 0.3, (B, H, dk, dv)), rng.normal(0, 1, (B, H, dk, dv))
    epi = "gn_swish" if gn else "none"
    ref = og.prefill_backward(Q, K, V, z, G, 4.0, 1e-5, dO, S0=S0, dS_final=dSf, epilogue=epi)
    got = _chunked_backward(Q, K, V, z, G, dO, 4.0, 1e-5, S0, dSf, C, gn)
    for name in ["dQ", "dK", "dV", "dz", "dS0"] + (["dG"] if gn else []):
        r = np.asarray(ref[name])
        err = np.abs(got[name] - r).max() / np.abs(r).max()
        assert err < 1e-10, (name, err)
