"""Host-side arithmetic of bench.py: the algorithmic byte and flop counts the
roofline objects divide by, the backward summary, and the ragged length mix of
the packed-batch measurement (no GPU needed)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
import gret_inputs as gi  # noqa: E402

PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "test"}


def test_prefill_bytes_of_the_benchmark():
    # per token and head: Q, K (128 bf16 each), V, G, O (256 bf16 each), one fp32
    # gate logit; plus one 128 x 256 fp32 final state per (batch, head)
    cfg = gi.C2
    per_token_head = 2 * (128 + 128 + 256 + 256 + 256) + 4
    want = 4 * 4096 * 16 * per_token_head + 4 * 16 * 128 * 256 * 4
    assert bench.prefill_alg(cfg)[0] == want == 546308096


def test_decode_bytes():
    cfg = gi.C4
    state = 128 * 256 * 4
    per_unit = 2 * state + 2 * (128 + 128 + 256 + 256 + 256) + 4
    assert bench.decode_alg(cfg) == 256 * 16 * per_unit


def test_backward_flops_count_each_product():
    cfg = gi.C2
    C, dk, dv = bench.BACKWARD_CHUNK, cfg.dk, cfg.dv
    # flops of one chunk of one head, product by product (2 per multiply-add)
    state = 2 * C * dk * dv                       # one C x dk x dv product
    causal = lambda m, n, k: 2 * m * n * k // 2   # noqa: E731  (half of a C x C side)
    per_chunk = 6 * state                         # increment, Q S, G_c, dy S^T, V dS'^T, K dS'
    per_chunk += 2 * causal(C, C, dk)             # Q K^T (dy step and gradient step)
    per_chunk += causal(C, dv, C)                 # A V
    per_chunk += causal(C, C, dv)                 # dy V^T
    per_chunk += causal(C, dv, C)                 # A^T dy
    per_chunk += causal(C, dk, C) * 2             # D K and D^T Q
    chunks = cfg.B * cfg.H * cfg.N // C
    assert bench.backward_alg_flops(cfg) == chunks * per_chunk


def test_backward_summary():
    cfg = gi.C2
    out = bench.backward_summary(cfg, steps=4, ms=20.0, world=1, peaks=PEAKS, launches_per_call=6)
    assert out["ms_per_step"] == pytest.approx(5.0)
    assert out["value"] == pytest.approx(4 * 4096 / 5e-3 / 1e6)
    rf = out["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert rf["achieved"] == pytest.approx(bench.backward_alg_flops(cfg) / 5e-3 / 1e12)
    # the tensor-core backward's products are kind::f16 (bf16 operands): the bf16 peak
    assert rf["peak"] == pytest.approx(1600.0)
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"])
    assert out["path_hbm"]["alg_bytes"] == bench.backward_alg(cfg)
    assert out["gpu_launches"] == 24


def test_varlen_mix():
    lengths = bench.varlen_lengths(16384, 4096, seed=17)
    assert sum(lengths) == 16384
    assert min(lengths) >= 1 and max(lengths) <= 4096
    assert 1 in lengths                                  # a one-token sequence
    assert any(n % 64 for n in lengths)                  # ragged chunk tails
    assert bench.varlen_lengths(16384, 4096, seed=17) == lengths


def test_projection_bytes():
    # X rows of d_model bf16, W_gamma fp32, and two fp32 words (decay sum and
    # P-block factor) per token and head of the padded sequence
    cfg = gi.C2
    d_model = 16 * 128
    want = 4 * 4096 * d_model * 2 + d_model * 16 * 4 + 2 * 64 * 4096 * 4
    assert bench.projection_alg(cfg, d_model) == (want, 2 * 4 * 4096 * 16 * d_model)
