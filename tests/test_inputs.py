"""The seeded input generator: determinism, slicing and distributions."""
import math

import numpy as np
import torch

import gret_inputs as gi


def test_unit_slice_matches_full_tensor():
    cfg = gi.C1.scaled(B=2, H=3, N=40, dk=16, dv=32, io="bf16",
                       z_dist=((-4.0, 1.0), (8.0, 0.5), (0.0, 2.0)))
    full = gi.prefill_inputs(cfg)
    for b in range(cfg.B):
        for h in range(cfg.H):
            unit = gi.prefill_unit_inputs(cfg, b, h)
            head = gi.prefill_unit_inputs(cfg, b, h, tokens=13)
            for name in ("Q", "K", "V", "G", "z"):
                assert torch.equal(full[name][b, :, h], unit[name]), name
                assert torch.equal(full[name][b, :13, h], head[name]), name


def test_decode_unit_slice_matches_full():
    cfg = gi.C4.__class__(**{**gi.C4.__dict__, "num_seqs": 3, "H": 2, "steps": 4, "dk": 16, "dv": 32})
    full = gi.decode_step_inputs(cfg)
    for s in range(3):
        for h in range(2):
            unit = gi.decode_unit_step_inputs(cfg, s, h)
            for name in ("q", "k", "v", "g", "z"):
                assert torch.equal(full[name][:, s, h], unit[name]), name


def test_deterministic_and_streams_differ():
    a = gi.random_unit(7, 1, (1000,))
    b = gi.random_unit(7, 1, (1000,))
    c = gi.random_unit(7, 2, (1000,))
    d = gi.random_unit(8, 1, (1000,))
    assert torch.equal(a, b)
    assert not torch.equal(a, c)
    assert not torch.equal(a, d)


def test_normal_moments():
    x = gi.standard_normal_at(3, 4, np.arange(400000))
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.01
    assert abs(((x ** 4).mean()) - 3.0) < 0.05   # Gaussian kurtosis


def test_config_distributions():
    cfg = gi.C5.scaled(B=1, N=2048)
    z = gi.prefill_inputs(cfg)["z"].double()
    assert abs(z[..., :8].mean() + 4.0) < 0.05 and abs(z[..., :8].var() - 1.0) < 0.05
    assert abs(z[..., 8:].mean() - 8.0) < 0.05 and abs(z[..., 8:].var() - 0.5) < 0.05
    q = gi.prefill_inputs(gi.C2.scaled(B=1, N=256))["Q"].double()
    assert abs(q.var() - 1.0 / 128) < 2e-4


def test_bf16_rounding_is_rne():
    v = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5 - 2 ** -9], dtype=np.float64)
    out = gi.to_storage(v, "bf16").float().numpy()
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(out, ref)
