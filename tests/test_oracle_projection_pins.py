"""Pins of the oracle's gate projection and rotation against what the pages and
the mathematics fix (CPU only).

* gate_project, z = X W_gamma ("YOCO 深度技术分析" section 2.2): a hand-checked
  worked value, numpy's matmul as a second route, and that a one-hot token
  picks out one row of W_gamma.
* rotate, the Theta of Q = (X W_Q) (.) Theta read as RoPE on consecutive pairs:
  closed-form worked values (tests/golden/rotation_values.txt), the pair norms
  it keeps, R(a) R(b) = R(a + b), and that the rotated scores q_m . k_n depend
  on the positions only through m - n.
* prefill_projected: the projection followed by the prefill equals the
  prefill fed with precomputed gate logits.
Planted mistakes in copies of the oracle source must each fail a pin.
"""
import math
import os

import numpy as np
import pytest

import gret_inputs as gi
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(seed, tid, shape, mean=0.0, var=1.0):
    return gi.random_unit(seed, tid, shape, mean, var, "f32").double().numpy()


def _rotation_rows():
    rows = []
    with open(os.path.join(GOLDEN, "rotation_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            left, right = line.split("|")
            a = left.split()
            d, base, pos = int(a[0]), float(a[1]), int(a[2])
            rows.append((d, base, pos, [float(x) for x in a[3:]], [float(x) for x in right.split()]))
    return rows


def _projection_pins_pass(lib=None) -> bool:
    try:
        # worked value: [1, 2] . [[3, -1], [4, 0.5]] = [1*3 + 2*4, 1*(-1) + 2*0.5] = [11, 0]
        z = oracle.gate_project(np.array([[1.0, 2.0]]), np.array([[3.0, -1.0], [4.0, 0.5]]), lib=lib)
        if not np.array_equal(z, np.array([[11.0, 0.0]])):
            return False
        # second route: numpy's matmul, on a non-square W
        X = _rand(31, 1, (2, 5, 48))
        W = _rand(31, 2, (48, 3))
        z = oracle.gate_project(X, W, lib=lib)
        if z.shape != (2, 5, 3) or np.max(np.abs(z - X @ W)) > 1e-12 * np.max(np.abs(X @ W)):
            return False
        # worked rotation values (closed forms)
        for d, base, pos, x, want in _rotation_rows():
            got = oracle.rotate(np.array(x).reshape(1, 1, 1, d), base, pos0=pos, lib=lib).ravel()
            if np.max(np.abs(got - np.array(want))) > 1e-14:
                return False
        # R(a) R(b) = R(a + b), per token position (N = 1 rows at offsets)
        Xr = _rand(32, 1, (1, 1, 2, 16))
        ab = oracle.rotate(oracle.rotate(Xr, 500.0, pos0=37, lib=lib), 500.0, pos0=1000, lib=lib)
        if np.max(np.abs(ab - oracle.rotate(Xr, 500.0, pos0=1037, lib=lib))) > 1e-12:
            return False
        # rotated scores depend on positions only through their difference
        q = _rand(33, 1, (1, 1, 1, 32))
        k = _rand(33, 2, (1, 1, 1, 32))
        s1 = np.sum(oracle.rotate(q, 10000.0, pos0=70, lib=lib) * oracle.rotate(k, 10000.0, pos0=15, lib=lib))
        s2 = np.sum(oracle.rotate(q, 10000.0, pos0=4055, lib=lib) * oracle.rotate(k, 10000.0, pos0=4000, lib=lib))
        if abs(s1 - s2) > 1e-11 * (1 + abs(s1)):
            return False
    except Exception:
        return False
    return True


def test_projection_pins():
    assert _projection_pins_pass()


def test_one_hot_token_picks_a_row_of_w():
    W = _rand(34, 1, (40, 4))
    X = np.zeros((1, 40))
    X[0, 17] = 1.0
    assert np.array_equal(oracle.gate_project(X, W)[0], W[17])


def test_rotation_keeps_pair_norms_and_position_zero():
    X = _rand(35, 1, (2, 9, 3, 64))
    R = oracle.rotate(X, 10000.0)
    pn = lambda a: a[..., 0::2] ** 2 + a[..., 1::2] ** 2  # noqa: E731
    assert np.max(np.abs(pn(R) - pn(X))) < 1e-12
    assert np.array_equal(R[:, 0], X[:, 0])        # position 0: the identity


def test_projected_prefill_equals_prefill_on_precomputed_logits():
    cfg = gi.C2.scaled(B=2, H=3, N=40, dk=16, dv=32, seed=36)
    inp = gi.prefill_inputs(cfg)
    d_model = 24
    X = _rand(36, 7, (cfg.B, cfg.N, d_model), 0.0, 1.0 / d_model)
    W = _rand(36, 8, (d_model, cfg.H), 3.0, 1.0)
    O1, Y1, S1 = oracle.prefill_projected(inp["Q"], inp["K"], inp["V"], X, W, inp["G"], cfg.tau, cfg.eps)
    O2, Y2, S2 = oracle.prefill(inp["Q"], inp["K"], inp["V"], X @ W, inp["G"], cfg.tau, cfg.eps)
    for a, b in ((O1, O2), (Y1, Y2), (S1, S2)):
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))
    # with the rotation: the same as the prefill of rotated Q and K
    O3, _, S3 = oracle.prefill_projected(inp["Q"], inp["K"], inp["V"], X, W, inp["G"], cfg.tau, cfg.eps,
                                         theta_base=10000.0)
    Qr, Kr = oracle.rotate(inp["Q"], 10000.0), oracle.rotate(inp["K"], 10000.0)
    O4, _, S4 = oracle.prefill(Qr, Kr, inp["V"], X @ W, inp["G"], cfg.tau, cfg.eps)
    assert np.max(np.abs(O3 - O4)) <= 1e-12 * np.max(np.abs(O4))
    assert np.max(np.abs(S3 - S4)) <= 1e-12 * np.max(np.abs(S4))


MUTANTS = {
    # rotation turning the wrong way
    "rot_sign": ("y[2 * j] = x[2 * j] * c - x[2 * j + 1] * s;", "y[2 * j] = x[2 * j] * c + x[2 * j + 1] * s;"),
    # frequencies base^(-j/d) instead of base^(-2j/d)
    "rot_exponent": ("double theta = pow(base, -2.0 * j / d);", "double theta = pow(base, -1.0 * j / d);"),
    # position offset ignored
    "rot_position": ("double ang = (double)(pos0 + n) * theta;", "double ang = (double)(n) * theta;"),
    # W read transposed
    "proj_transposed": ("acc += X[(size_t)r * d_model + i] * W[(size_t)i * H + h];",
                        "acc += X[(size_t)r * d_model + i] * W[(size_t)h * d_model + i];"),
}


def test_unmutated_oracle_passes_projection_pins(tmp_path):
    assert _projection_pins_pass(oracle.build_variant(oracle.source_text(), str(tmp_path)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_projection_mutants_are_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    lib = oracle.build_variant(src.replace(old, new), str(tmp_path))
    assert not _projection_pins_pass(lib), f"planted mistake {name} was not caught by the pins"
