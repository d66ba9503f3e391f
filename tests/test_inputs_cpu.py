"""The workload shapes and the seeded input recipe (CPU only).

The workloads' key counts are checked against the hand-enumerated N_vis of tests/golden/, and
the input generator against the recipe it states: one CPU generator per tensor seeded from
(seed, chunk, step, tensor id), N(0, 1) values rounded to bf16, sigma-4 outlier key rows with
probability 0.01 on the stress workload, and e4m3 inputs that are the same draws divided by a
power-of-two scale.
"""
from __future__ import annotations

import os

import pytest
import torch

from block_causal_attention_sliding_b200 import synth
from block_causal_attention_sliding_b200.configs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _golden_nvis():
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "visible_keys.txt"), encoding="utf-8") as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, T, n_cond, W, k, nvis = line.split()
                rows.append((name, int(T), int(n_cond), int(W), int(k), int(nvis)))
    return rows


@pytest.mark.parametrize("name,T,n_cond,W,k,nvis", _golden_nvis())
def test_workload_key_counts_match_golden(name, T, n_cond, W, k, nvis):
    wl = WORKLOADS[name]
    assert (wl.T, wl.n_cond, wl.W) == (T, n_cond, W)
    assert wl.n_vis(k) == nvis


def test_720p_forward_work():
    """4 * B * H * T * N_vis * d over the valid keys: 631.31 GFLOP per steady 720p forward."""
    wl = WORKLOADS["720p"]
    assert wl.steady_k() == 4
    assert wl.flops_forward(wl.steady_k()) == 4 * 24 * 3180 * 16156 * 128
    assert round(wl.flops_forward(wl.steady_k()) / 1e9, 2) == 631.31
    assert wl.flops_forward(wl.steady_k(), n_q=16) == 4 * 24 * 16 * 16156 * 128


def test_seeded_draws_reproduce_and_differ():
    wl = WORKLOADS["tiny"]
    a = synth.chunk_inputs(wl, 2, 1)
    b = synth.chunk_inputs(wl, 2, 1)
    for x, y in zip(a, b):
        assert torch.equal(x, y)                                   # same seed, same values
    others = [synth.chunk_inputs(wl, 2, 0), synth.chunk_inputs(wl, 3, 1), synth.chunk_inputs(wl, 2, 1, seed=1)]
    for o in others:
        for x, y in zip(a, o):
            assert not torch.equal(x, y)
    Q, K, V = a
    assert not torch.equal(Q, K) and not torch.equal(K, V)        # own stream per tensor
    # the seed formula and a direct draw from it
    assert synth.stream_seed(3, 7, 1, synth.TID_V) == 3_000_000 + 700 + 10 + 2
    g = torch.Generator().manual_seed(synth.stream_seed(0, 2, 1, synth.TID_V))
    ref = torch.randn((wl.B, wl.T, wl.H, wl.d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(V, ref)


def test_short_queries_are_the_first_rows_of_a_full_draw():
    wl = WORKLOADS["720p"]
    Qs, Ks, Vs = synth.chunk_inputs(wl, 4, 0, n_q=16)
    Qf, Kf, Vf = synth.chunk_inputs(wl, 4, 0)
    assert Qs.shape == (1, 16, 24, 128) and torch.equal(Qs, Qf[:, :16])
    assert torch.equal(Ks, Kf) and torch.equal(Vs, Vf)


def test_values_are_bf16_gaussians():
    wl = WORKLOADS["720p"]
    Q, K, V = synth.chunk_inputs(wl, 0, 0)
    for t in (Q, K, V):
        assert t.dtype == torch.bfloat16 and t.shape == (1, 3180, 24, 128) and t.is_contiguous()
        f = t.float()
        assert abs(f.mean().item()) < 0.01 and abs(f.std().item() - 1.0) < 0.01


def test_stress_outlier_rows():
    """About 1% of the stress workload's key rows (condition K here) carry sigma 4; values and
    queries carry none."""
    wl = WORKLOADS["stress"]
    Kc, Vc = synth.cond_inputs(wl)
    rms_k = Kc.float().pow(2).mean(-1).sqrt()          # per (b, token, h) row of d = 128
    rms_v = Vc.float().pow(2).mean(-1).sqrt()
    frac = (rms_k > 2.5).float().mean().item()
    assert 0.008 < frac < 0.012, frac                   # 65,536 rows: 1% +- 0.2% is > 5 sigma
    out = rms_k[rms_k > 2.5]
    assert abs(out.mean().item() - 4.0) < 0.1            # those rows have sigma 4
    assert (rms_v > 2.5).sum().item() == 0
    assert WORKLOADS["720p"].outlier_p == 0.0


def test_e4m3_inputs_are_scaled_draws():
    """e4m3 inputs: the bf16 draws divided by a power-of-two scale and rounded to e4m3; the
    dequantised values are exact in float32 and stay finite for sigma-4 outlier keys."""
    wl = WORKLOADS["stress"]
    s = synth.FP8_SCALE
    m, e = torch.frexp(torch.tensor(s))
    assert m.item() == 0.5                               # a power of two
    Q8, K8, V = synth.chunk_inputs_fp8(wl, 0, 0)
    Q, K, _ = synth.chunk_inputs(wl, 0, 0)
    assert Q8.dtype == K8.dtype == torch.float8_e4m3fn and V.dtype == torch.bfloat16
    Kd = synth.from_e4m3(K8)
    assert torch.isfinite(Kd).all()
    assert torch.equal(Kd, K8.float() * s)
    assert torch.equal(K8, (K.float() / s).to(torch.float8_e4m3fn))
    # e4m3 keeps 3 mantissa bits: each dequantised value is within 2^-4 of the bf16 draw, or
    # within half a subnormal step (2^-10, scaled) below e4m3's normal range
    err = (Kd - K.float()).abs()
    assert (err <= K.float().abs() * 2.0 ** -4 + 2.0 ** -10 * s).all()
    _, _, V8 = synth.chunk_inputs_fp8(WORKLOADS["tiny"], 0, 0, v8=True)
    assert V8.dtype == torch.float8_e4m3fn
