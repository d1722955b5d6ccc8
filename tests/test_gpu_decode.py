"""GPU parity of the recurrent decode step against the fp64 oracle.

Prior states come from the oracle's own prefill of seeded prompts (rounded to
fp32, the state's storage type); the GPU then runs consecutive steps through
the C ABI, one launch per step, and each step's output and the final state are
compared with the oracle's decode steps on the same inputs."""
import numpy as np
import pytest
import torch

import gated_retention_sequence_b200 as gret
import gret_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_retention_sequence_b200 import build
    build.build()
    gret.load()


def _small_cfg(io="bf16", **kw):
    base = dict(num_seqs=6, H=3, dk=128, dv=256, steps=5, prior_len=64, io=io, seed=31)
    base.update(kw)
    return gi.DecodeConfig(name="decode-small", tau=16.0, qkv_var=1.0 / base["dk"],
                           z_dist=(3.0, 1.5), **base)


def _oracle_prior(cfg):
    p = cfg.prior_prefill()
    inp = gi.prefill_inputs(p)
    _, _, S = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], p.tau, p.eps)
    return S   # fp64 [S,H,dk,dv]


@pytest.mark.parametrize("io,dk,dv", [("bf16", 128, 256), ("f32", 64, 64), ("bf16", 16, 16),
                                      ("f32", 128, 48)])
def test_decode_steps(io, dk, dv):
    cfg = _small_cfg(io=io, dk=dk, dv=dv)
    S_ref = _oracle_prior(cfg)
    S_gpu = torch.from_numpy(S_ref.astype(np.float32)).cuda()
    S_ref = S_gpu.double().cpu().numpy()        # start both from the same fp32 state
    steps = gi.decode_step_inputs(cfg)
    for t in range(cfg.steps):
        d = {k: v[t].cuda() for k, v in steps.items()}
        o = gret.decode_step(d["q"], d["k"], d["v"], d["z"], d["g"], S_gpu, cfg.tau, cfg.eps)
        y = None
        o_ref, y_ref, S_ref = oracle.decode_step(steps["q"][t], steps["k"][t], steps["v"][t],
                                                 steps["z"][t], steps["g"][t], S_ref, cfg.tau, cfg.eps)
        assert_close(o, o_ref, io, f"o step {t}")
    gret.check_device_status()
    assert_close(S_gpu, S_ref, io, "S after steps")


def test_decode_pre_norm_output():
    cfg = _small_cfg(io="bf16", steps=1)
    S_ref = _oracle_prior(cfg)
    S_gpu = torch.from_numpy(S_ref.astype(np.float32)).cuda()
    S_ref = S_gpu.double().cpu().numpy()
    st = gi.decode_step_inputs(cfg)
    d = {k: v[0].cuda() for k, v in st.items()}
    y = gret.decode_step(d["q"], d["k"], d["v"], d["z"], None, S_gpu, cfg.tau, epilogue="none")
    _, y_ref, _ = oracle.decode_step(st["q"][0], st["k"][0], st["v"][0], st["z"][0], st["g"][0],
                                     S_ref, cfg.tau)
    assert_close(y, y_ref, "bf16", "y")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_prefill_then_decode_equals_longer_prefill(io):
    # prefill hands its last state to recurrent decode ("YOCO 深度技术分析", 5.3.7)
    N0, T = 150, 6
    cfg = gi.C1.scaled(B=2, H=2, N=N0 + T, dk=128 if io == "bf16" else 64,
                       dv=256 if io == "bf16" else 64, chunk=64, io=io, seed=55,
                       qkv_var=1.0 / (128 if io == "bf16" else 64))
    inp = gi.prefill_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    _, S = gret.prefill(d["Q"][:, :N0].contiguous(), d["K"][:, :N0].contiguous(),
                        d["V"][:, :N0].contiguous(), d["z"][:, :N0].contiguous(),
                        d["G"][:, :N0].contiguous(), cfg.tau, cfg.chunk)
    outs = []
    for t in range(T):
        n = N0 + t
        outs.append(gret.decode_step(d["Q"][:, n].contiguous(), d["K"][:, n].contiguous(),
                                     d["V"][:, n].contiguous(), d["z"][:, n].contiguous(),
                                     d["G"][:, n].contiguous(), S, cfg.tau))
    gret.check_device_status()
    O_ref, _, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau)
    assert_close(torch.stack(outs, 1), O_ref[:, N0:], io, "decoded outputs")
    assert_close(S, S_ref, io, "final state")


def test_full_decode_workload_sampled():
    """256 sequences x 16 heads, 128 x 256 fp32 states, 64 consecutive steps.

    The oracle recomputes a sample of units one by one: their prior states come
    from its own 512-token prefill; the remaining units hold seeded random
    states (they are streamed by the same launch but not compared)."""
    cfg = gi.C4
    rng_units = [(0, 0), (17, 5), (128, 9), (255, 15)]
    S_gpu = gi.random_unit(cfg.seed, 99, (cfg.num_seqs, cfg.H, cfg.dk, cfg.dv), 0.0, 0.05).cuda()
    p = cfg.prior_prefill()
    ref_state = {}
    for s, h in rng_units:
        u = gi.prefill_unit_inputs(p, s, h)
        _, _, S = oracle.prefill(u["Q"][None, :, None], u["K"][None, :, None], u["V"][None, :, None],
                                 u["z"][None, :, None], u["G"][None, :, None], p.tau, p.eps)
        S32 = torch.from_numpy(S[0, 0].astype(np.float32))
        S_gpu[s, h] = S32.cuda()
        ref_state[(s, h)] = S32.double().numpy()
    steps = gi.decode_step_inputs(cfg)
    dsteps = {k: v.cuda() for k, v in steps.items()}
    outs = []
    for t in range(cfg.steps):
        o = gret.decode_step(dsteps["q"][t], dsteps["k"][t], dsteps["v"][t], dsteps["z"][t],
                             dsteps["g"][t], S_gpu, cfg.tau, cfg.eps)
        outs.append(o[[s for s, _ in rng_units], [h for _, h in rng_units]].cpu())
    gret.check_device_status()
    got = torch.stack(outs, 0)   # [T, units, dv]
    for i, (s, h) in enumerate(rng_units):
        S = ref_state[(s, h)]
        refs = []
        for t in range(cfg.steps):
            o_ref, _, S4 = oracle.decode_step(steps["q"][t, s, h][None, None], steps["k"][t, s, h][None, None],
                                              steps["v"][t, s, h][None, None], steps["z"][t, s, h][None, None],
                                              steps["g"][t, s, h][None, None], S[None, None], cfg.tau, cfg.eps)
            S = S4[0, 0]
            refs.append(o_ref[0, 0])
        assert_close(got[:, i], np.stack(refs), "bf16", f"o unit {(s, h)}")
        assert_close(S_gpu[s, h], S, "bf16", f"S unit {(s, h)}")
