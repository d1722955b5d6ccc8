"""Pins of the fp64 oracle to what the pages and the mathematics fix.

No test here re-types the oracle's formula: each compares the oracle with an
independent statement of the same result (another of the three equivalent
forms, a closed form, a worked value, a library routine, or an identity that
holds for the recurrence), chosen so that a dropped term, a wrong index or sign,
or a transposed operand fails at least one of them.  ``test_mutants_are_caught``
plants such mistakes in a copy of the oracle (on the CPU) and checks that the
pins notice.

Sources: "YOCO 深度技术分析", section 2.2 (gate, parallel and recurrent forms,
GroupNorm + swish), section 5.3.2 (chunkwise form; the three forms are exactly
equivalent), section 5.3.7 (prefill hands its last state to recurrent decode);
"YOCO" (zdszero.github.io), section "Self-Decoder" (S_t = gamma_t S_{t-1} +
K_t^T V_t, y_t = Q_t S_t).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from gret_inputs import random_unit

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, tid, shape, var=1.0):
    return random_unit(seed, tid, shape, 0.0, var, "f32").double().numpy()


def _problem(seed, B, N, H, dk, dv, z_mean=2.0, z_var=1.0, tau=4.0):
    Q = _rand(seed, 1, (B, N, H, dk), 1.0 / dk)
    K = _rand(seed, 2, (B, N, H, dk), 1.0 / dk)
    V = _rand(seed, 3, (B, N, H, dv), 1.0)
    z = z_mean + math.sqrt(z_var) * _rand(seed, 5, (B, N, H))
    lg = oracle.log_gamma(z, tau)
    return Q, K, V, lg


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- gate
def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return rows


def test_gate_worked_values():
    for z, tau, gamma in _read_golden("gate_values.txt"):
        lg = oracle.log_gamma(np.array([z]), tau)[0]
        assert math.exp(lg) == pytest.approx(gamma, rel=1e-14, abs=0)


def test_gate_limits_and_second_route():
    z = np.linspace(-30, 30, 241)
    for tau in (1.0, 3.0, 16.0):
        lg = oracle.log_gamma(z, tau)
        # second route: log of the sigmoid, computed with numpy's logaddexp
        ref = -np.logaddexp(0.0, -z) / tau
        assert np.max(np.abs(lg - ref)) < 1e-14
        assert np.all(lg <= 0)
        assert np.all(np.diff(lg) > 0)          # gamma increases with z
    # z -> +inf: gamma -> 1; z -> -inf: log gamma -> z / tau
    assert oracle.log_gamma(np.array([60.0]), 16.0)[0] == pytest.approx(-math.exp(-60) / 16, rel=1e-9)
    assert oracle.log_gamma(np.array([-60.0]), 16.0)[0] == pytest.approx(-60 / 16, rel=1e-12)
    # tau -> inf: gamma -> 1
    assert abs(oracle.log_gamma(np.array([-3.0]), 1e12)[0]) < 1e-10


# ---------------------------------------------------------------- three forms
@pytest.mark.parametrize("dk,dv", [(1, 1), (2, 8), (8, 2), (16, 16), (8, 1)])
def test_parallel_equals_recurrent(dk, dv):
    B, N, H = 2, 37, 3
    Q, K, V, lg = _problem(11 + dk * 7 + dv, B, N, H, dk, dv)
    Yr, _ = oracle.recurrent(Q, K, V, lg)
    Yp = oracle.parallel(Q, K, V, lg)
    assert _rel(Yp, Yr) < 1e-12


def test_parallel_equals_recurrent_with_initial_state():
    B, N, H, dk, dv = 1, 64, 2, 8, 16
    Q, K, V, lg = _problem(5, B, N, H, dk, dv, z_mean=0.0, z_var=4.0, tau=1.0)
    S0 = _rand(6, 9, (B, H, dk, dv))
    Yr, _ = oracle.recurrent(Q, K, V, lg, S0=S0)
    Yp = oracle.parallel(Q, K, V, lg, S0=S0)
    assert _rel(Yp, Yr) < 1e-12


@pytest.mark.parametrize("chunk", [1, 2, 3, 4, 7, 16, 48, 64, 100, 128])
def test_chunkwise_independent_of_chunk(chunk):
    B, N, H, dk, dv = 1, 100, 2, 16, 8
    Q, K, V, lg = _problem(21, B, N, H, dk, dv, z_mean=-1.0, z_var=9.0, tau=1.0)
    S0 = _rand(22, 9, (B, H, dk, dv))
    Yr, Sr = oracle.recurrent(Q, K, V, lg, S0=S0)
    Yc, Sc = oracle.chunkwise(Q, K, V, lg, chunk, S0=S0)
    assert _rel(Yc, Yr) < 1e-11
    assert _rel(Sc, Sr) < 1e-11


def test_gamma_one_is_causal_linear_attention():
    # lg = 0: Y_n = sum_{m<=n} (Q_n . K_m) V_m, as a prefix sum of outer products
    B, N, H, dk, dv = 2, 50, 2, 8, 4
    Q, K, V, _ = _problem(31, B, N, H, dk, dv)
    lg = np.zeros((B, N, H))
    Y, Sf = oracle.recurrent(Q, K, V, lg)
    outer = np.einsum("bnhi,bnhj->bnhij", K, V)
    S = np.cumsum(outer, axis=1)
    ref = np.einsum("bnhi,bnhij->bnhj", Q, S)
    assert _rel(Y, ref) < 1e-12
    assert _rel(Sf, S[:, -1]) < 1e-12
    Yc, _ = oracle.chunkwise(Q, K, V, lg, 7)
    assert _rel(Yc, ref) < 1e-12


def test_gamma_zero_keeps_only_the_current_token():
    # lg = -inf (gamma = 0): Y_n = (Q_n . K_n) V_n
    B, N, H, dk, dv = 1, 20, 2, 8, 6
    Q, K, V, _ = _problem(41, B, N, H, dk, dv)
    lg = np.full((B, N, H), -np.inf)
    ref = np.einsum("bnhi,bnhi->bnh", Q, K)[..., None] * V
    Y, Sf = oracle.recurrent(Q, K, V, lg)
    assert _rel(Y, ref) < 1e-14
    assert _rel(Sf, np.einsum("bhi,bhj->bhij", K[:, -1], V[:, -1])) < 1e-14
    Yp = oracle.parallel(Q, K, V, lg)
    assert _rel(Yp, ref) < 1e-14
    # epilogue closed form: GN(c V) = c (V - mu) / sqrt(c^2 var + eps)
    G = _rand(42, 4, (B, N, H, dv))
    eps = 1e-5
    O = oracle.groupnorm_swish(Y, G, eps)
    c = np.einsum("bnhi,bnhi->bnh", Q, K)[..., None]
    mu = V.mean(-1, keepdims=True)
    var = ((V - mu) ** 2).mean(-1, keepdims=True)
    swish = G / (1 + np.exp(-G))
    ref_o = c * (V - mu) / np.sqrt(c * c * var + eps) * swish
    assert _rel(O, ref_o) < 1e-12


def test_constant_gamma_geometric_series():
    rows = _read_golden("retnet_constant_gamma.txt")
    for gamma in sorted({r[0] for r in rows}):
        N = 5
        one = np.ones((1, N, 1, 1))
        lg = np.full((1, N, 1), math.log(gamma))
        Y, _ = oracle.recurrent(one, one, one, lg)
        Yp = oracle.parallel(one, one, one, lg)
        Yc, _ = oracle.chunkwise(one, one, one, lg, 2)
        for g, n, yn in rows:
            if g == gamma:
                for got in (Y, Yp, Yc):
                    assert got[0, int(n) - 1, 0, 0] == pytest.approx(yn, rel=1e-14)


def test_constant_gamma_retnet_mask():
    # RetNet retention: D[n][m] = gamma^(n-m) from powers, not products
    B, N, H, dk, dv = 1, 40, 1, 8, 8
    Q, K, V, _ = _problem(51, B, N, H, dk, dv)
    gamma = 0.93
    lg = np.full((B, N, H), math.log(gamma))
    n = np.arange(N)
    D = np.where(n[:, None] >= n[None, :], gamma ** (n[:, None] - n[None, :]).clip(0), 0.0)
    A = Q[0, :, 0] @ K[0, :, 0].T
    ref = (A * D) @ V[0, :, 0]
    Y, _ = oracle.recurrent(Q, K, V, lg)
    assert _rel(Y[0, :, 0], ref) < 1e-12


def test_state_decomposition():
    # S(x || y) = e^{sum lg(y)} S(x) + S(y from 0)
    B, N, H, dk, dv = 1, 60, 2, 8, 8
    Q, K, V, lg = _problem(61, B, N, H, dk, dv, z_mean=1.0, z_var=2.0, tau=2.0)
    cut = 23
    _, S_all = oracle.recurrent(Q, K, V, lg)
    _, S_x = oracle.recurrent(Q[:, :cut], K[:, :cut], V[:, :cut], lg[:, :cut])
    _, S_y = oracle.recurrent(Q[:, cut:], K[:, cut:], V[:, cut:], lg[:, cut:])
    decay = np.exp(lg[:, cut:].sum(axis=1))  # [B,H]
    assert _rel(S_all, decay[..., None, None] * S_x + S_y) < 1e-12
    # and the second segment's outputs equal a prefill started from S(x)
    Y_all, _ = oracle.recurrent(Q, K, V, lg)
    Y_y, _ = oracle.recurrent(Q[:, cut:], K[:, cut:], V[:, cut:], lg[:, cut:], S0=S_x)
    assert _rel(Y_y, Y_all[:, cut:]) < 1e-12


# ---------------------------------------------------------------- epilogue
def test_groupnorm_swish_matches_torch():
    rows, dv = 300, 64
    Y = _rand(71, 1, (rows, dv), 3.0) + 0.7
    G = _rand(71, 2, (rows, dv))
    for eps in (1e-5, 1e-2):
        O = oracle.groupnorm_swish(Y, G, eps)
        yt = torch.from_numpy(Y)
        ref = torch.nn.functional.group_norm(yt, 1, eps=eps) * torch.nn.functional.silu(torch.from_numpy(G))
        assert _rel(O, ref.numpy()) < 1e-13


def test_groupnorm_invariants():
    rows, dv, eps = 50, 32, 1e-3
    Y = _rand(72, 1, (rows, dv), 0.01)
    G = np.full((rows, dv), 60.0)             # swish(60) / 60 = 1 - 1e-26
    O = oracle.groupnorm_swish(Y, G, eps) / 60.0
    var = Y.var(-1)
    assert np.max(np.abs(O.mean(-1))) < 1e-13
    assert np.max(np.abs(O.var(-1) - var / (var + eps))) < 1e-12


# ---------------------------------------------------------------- decode chaining
def test_decode_chaining_equals_longer_prefill():
    B, N0, T, H, dk, dv = 2, 33, 9, 2, 8, 16
    Q, K, V, lg = _problem(81, B, N0 + T, H, dk, dv)
    G = _rand(81, 4, (B, N0 + T, H, dv))
    eps = 1e-5
    O_all, Y_all, S_all = oracle.prefill(Q, K, V, None, G, 16.0, eps, lg=lg)
    _, _, S = oracle.prefill(Q[:, :N0], K[:, :N0], V[:, :N0], None, G[:, :N0], 16.0, eps, lg=lg[:, :N0])
    for t in range(T):
        n = N0 + t
        o, y, S = oracle.decode_step(Q[:, n], K[:, n], V[:, n], None, G[:, n], S, 16.0, eps, lg=lg[:, n])
        assert _rel(y, Y_all[:, n]) < 1e-12
        assert _rel(o, O_all[:, n]) < 1e-12
    assert _rel(S, S_all) < 1e-12


def test_decode_step_gate_from_logits():
    # the step's own gate path: z -> gamma = sigmoid(z)^(1/tau)
    ns, H, dk, dv = 3, 2, 4, 8
    q, k = _rand(91, 1, (ns, H, dk)), _rand(91, 2, (ns, H, dk))
    v, g = _rand(91, 3, (ns, H, dv)), _rand(91, 4, (ns, H, dv))
    z = _rand(91, 5, (ns, H))
    S = _rand(91, 6, (ns, H, dk, dv))
    tau = 3.0
    _, y, Sn = oracle.decode_step(q, k, v, z, g, S, tau, 1e-5)
    gamma = (1.0 / (1.0 + np.exp(-z))) ** (1.0 / tau)
    S_ref = gamma[..., None, None] * S + np.einsum("shi,shj->shij", k, v)
    assert _rel(Sn, S_ref) < 1e-14
    assert _rel(y, np.einsum("shi,shij->shj", q, S_ref)) < 1e-13


# ---------------------------------------------------------------- planted mistakes
MUTANTS = {
    # D[n][m] starting the product at m (decays the current token)
    "mask_from_m": ("for (int i = m + 1; i <= n; ++i) p *= gam[i];",
                    "for (int i = m; i <= n; ++i) p *= gam[i];"),
    # recurrence: decay applied to the new outer product too
    "decay_new_term": ("S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + k[i] * v[j];",
                       "S[(size_t)i * dv + j] = g * (S[(size_t)i * dv + j] + k[i] * v[j]);"),
    # chunkwise: inter-chunk read not decayed
    "no_inter_decay": ("y[j] = et * acc;", "y[j] = acc;"),
    # chunkwise: decay exponent sign flipped in the intra-chunk term
    "intra_sign": ("a *= exp(bc[t] - bc[s]);", "a *= exp(bc[s] - bc[t]);"),
    # chunkwise: state carry missing the chunk-total decay
    "carry_decay": ("for (size_t e = 0; e < (size_t)dk * dv; ++e) Sn[e] = eL * S[e];",
                    "for (size_t e = 0; e < (size_t)dk * dv; ++e) Sn[e] = S[e];"),
    # epilogue: unbiased variance
    "unbiased_var": ("var /= dv;", "var /= (dv - 1);"),
    # epilogue: sigmoid gate instead of swish
    "gate_sigmoid": ("o[j] = (y[j] - mu) * rs * g[j] * sg;", "o[j] = (y[j] - mu) * rs * sg;"),
    # gate: missing temperature
    "no_tau": ("lg[i] = -sp / tau;", "lg[i] = -sp;"),
}


def _pins_pass(lib) -> bool:
    try:
        for dk, dv in [(2, 8), (8, 1)]:
            Q, K, V, lg = _problem(11 + dk * 7 + dv, 2, 37, 3, dk, dv)
            lg = oracle.log_gamma(2.0 + _rand(3, 5, (2, 37, 3)), 4.0, lib=lib)
            if _rel(oracle.parallel(Q, K, V, lg, lib=lib), oracle.recurrent(Q, K, V, lg, lib=lib)[0]) > 1e-12:
                return False
            for c in (3, 16):
                Yc, Sc = oracle.chunkwise(Q, K, V, lg, c, lib=lib)
                Yr, Sr = oracle.recurrent(Q, K, V, lg, lib=lib)
                if _rel(Yc, Yr) > 1e-11 or _rel(Sc, Sr) > 1e-11:
                    return False
        rows = _read_golden("retnet_constant_gamma.txt")
        one = np.ones((1, 5, 1, 1))
        for g, n, yn in rows:
            Y, _ = oracle.recurrent(one, one, one, np.full((1, 5, 1), math.log(g)), lib=lib)
            if abs(Y[0, int(n) - 1, 0, 0] - yn) > 1e-12 * yn:
                return False
        for z, tau, gamma in _read_golden("gate_values.txt"):
            if abs(math.exp(oracle.log_gamma(np.array([z]), tau, lib=lib)[0]) - gamma) > 1e-13:
                return False
        Y = _rand(71, 1, (30, 16), 3.0)
        G = _rand(71, 2, (30, 16))
        ref = (torch.nn.functional.group_norm(torch.from_numpy(Y), 1, eps=1e-5)
               * torch.nn.functional.silu(torch.from_numpy(G))).numpy()
        if _rel(oracle.groupnorm_swish(Y, G, 1e-5, lib=lib), ref) > 1e-13:
            return False
    except Exception:
        return False
    return True


def test_unmutated_oracle_passes_pins(tmp_path):
    lib = oracle.build_variant(oracle.source_text(), str(tmp_path))
    assert _pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    lib = oracle.build_variant(src.replace(old, new), str(tmp_path))
    assert not _pins_pass(lib), f"planted mistake {name} was not caught by the pins"
