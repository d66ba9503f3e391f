"""Host-side checks of arithmetic the CUDA kernels use (no GPU needed).

exp2_poly (csrc/ptx.cuh) replaces a share of the MUFU exponentials with FMA-pipe arithmetic:
a Cody-Waite split x = j + f, |f| <= 1/2, a cubic for 2^f, and j added into the exponent bits.
Its bound is pinned here by replaying the same float32 steps (fused multiply-adds rounded once)
against numpy's exp2 in float64 over the whole input range the softmax can produce.

Also here: a float64 model of the rounding of P to e4m3 (the e4m3-P tolerance), and of the
kernels' online softmax with its lazy rescale thresholds and e4m3 weight offset (read from the
kernel source) together with the merge of split pieces, which must give exact softmax attention
for any split of the key tiles and keep every weight inside e4m3's range.
"""
from __future__ import annotations

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _poly_constants():
    src = open(os.path.join(ROOT, "block_causal_attention_sliding_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[: body.index("}")]
    lo = float(re.search(r"fmaxf\(x, (-?[0-9.]+)f\)", body).group(1))
    magic = float(re.search(r"magic = ([0-9.]+)f", body).group(1))
    coef = [float(v) for v in re.findall(r"fmaf\([a-z]*,?\s*([0-9.]+)f", body)]
    c3, c2 = [float(v) for v in re.search(r"fmaf\(([0-9.]+)f, f, ([0-9.]+)f\)", body).groups()]
    c1 = float(re.search(r"fmaf\(p, f, ([0-9.]+)f\);\s*p = fmaf\(p, f, ([0-9.]+)f\)", body).group(1))
    c0 = float(re.search(r"fmaf\(p, f, ([0-9.]+)f\);\s*return", body).group(1))
    assert coef  # the source still has the fused steps this test replays
    return lo, magic, (np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3))


def _fma32(a, b, c):
    # float32 fused multiply-add: exact product and sum in float64, one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_replay(x):
    lo, magic, (c0, c1, c2, c3) = _poly_constants()
    x = np.maximum(x.astype(np.float32), np.float32(lo))
    m = np.float32(magic)
    t = (x + m).astype(np.float32)
    f = (x - (t - m).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 1_000_000))])
    got = exp2_poly_replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    # well below bf16's half-ulp (2^-9 ~ 2e-3), the precision P is stored in
    assert rel.max() < 1.0e-4, rel.max()


def test_exp2_poly_masked_and_extremes():
    x = np.array([-np.inf, -1e30, -200.0, -125.0, 0.0, 1.0, 8.0], dtype=np.float32)
    got = exp2_poly_replay(x)
    assert np.all(np.isfinite(got)) and np.all(got >= 0)
    assert got[0] < 1e-37 and got[1] < 1e-37 and got[2] < 1e-37      # masked keys weigh ~0
    np.testing.assert_allclose(got[4:], [1.0, 2.0, 256.0], rtol=1e-4)


def _p_rounding_errors(seed: int = 0, n_q: int = 64, n_k: int = 4096, d: int = 128):
    """Mean-relative error of attention when P is rounded the two ways the kernels round it,
    against exact float64 attention, on inputs shaped like the synthetic workloads (N(0,1)
    queries, keys and values, scale 1/sqrt(d)):
      * bf16 P: p rounded to bf16 (round to nearest even), and the row sum adds those rounded
        weights, as the bf16 kernels do;
      * e4m3 P: p formed as 2^(x + 4) relative to the row's reference max and rounded to e4m3
        (round to nearest, saturating), the row sum adding the unrounded weights, as the e4m3-P
        kernels do.
    Returns (bf16 mean-rel, e4m3 mean-rel)."""
    import torch

    g = torch.Generator().manual_seed(seed)
    q = torch.randn(n_q, d, generator=g, dtype=torch.float64)
    k = torch.randn(n_k, d, generator=g, dtype=torch.float64)
    v = torch.randn(n_k, d, generator=g, dtype=torch.float64)
    s = (q @ k.T) / np.sqrt(d)
    x = (s - s.max(dim=1, keepdim=True).values) * np.log2(np.e)   # log2 weights, max 0
    p = torch.exp2(x)
    exact = (p @ v) / p.sum(dim=1, keepdim=True)

    def mean_rel(out):
        return float((out - exact).abs().sum() / exact.abs().sum())

    pb = p.float().to(torch.bfloat16).double()
    out_b = (pb @ v) / pb.sum(dim=1, keepdim=True)
    p8 = torch.exp2(x + 4.0)                                       # <= 16, e4m3 limit 448
    q8 = p8.float().to(torch.float8_e4m3fn).double()
    out_8 = (q8 @ v) / p8.sum(dim=1, keepdim=True)
    return mean_rel(out_b), mean_rel(out_8)


def test_e4m3_p_tolerance_model():
    """The e4m3-P tolerance (16 x the parity one: max-abs 1.6e-1, mean-rel 3.2e-2) rests on e4m3
    rounding each weight by up to 2^-4 of itself against bf16's 2^-8.  Modelled here in float64:
    the e4m3 error is about 16 x the bf16 one and stays inside 3.2e-2, and the bf16 error stays
    inside the parity bound of 2e-3."""
    eb, e8 = _p_rounding_errors()
    assert eb < 2e-3, eb
    assert e8 < 3.2e-2, e8
    assert 8.0 < e8 / eb < 24.0, (eb, e8, e8 / eb)


# ------------------------------------------------------------------ online softmax and merges

def _softmax_constants():
    """The kernels' lazy-rescale thresholds and e4m3 weight offset (log2 units), read from the
    source so that a change there is checked here."""
    src = open(os.path.join(ROOT, "block_causal_attention_sliding_b200", "csrc", "attn_common.cuh")).read()

    def get(name):
        return float(re.search(rf"constexpr float {name} = ([0-9.]+)f;", src).group(1))

    return get("kRescaleThreshold"), get("kP8Offset"), get("kP8Threshold")


def _online_piece(x, V, tiles, tau, off):
    """One piece of the kernels' online softmax over the key tiles `tiles` ((lo, hi) ranges, in
    order) for one query row, in float64: x holds the row's scores in log2 units (s * scale *
    log2 e).  The reference max moves only when a tile's max exceeds it by more than tau; the
    weights are 2^(x - m_ref + off).  Returns the partial (O, m_ref, l) and the largest weight."""
    m_ref, O, l, pmax = None, np.zeros(V.shape[1]), 0.0, 0.0
    for lo, hi in tiles:
        m_new = x[lo:hi].max()
        if m_ref is None:
            m_ref = m_new
        elif m_new > m_ref + tau:
            f = 2.0 ** (m_ref - m_new)
            O *= f
            l *= f
            m_ref = m_new
        p = 2.0 ** (x[lo:hi] - m_ref + off)
        pmax = max(pmax, float(p.max()))
        O += p @ V[lo:hi]
        l += p.sum()
    return O, m_ref, l, pmax


def _merge(parts):
    """The split-K / stream-K merge of partials (O_i, m_i, l_i): rescale each to the largest m."""
    M = max(m for _, m, _ in parts)
    O = sum(2.0 ** (m - M) * o for o, m, _ in parts)
    l = sum(2.0 ** (m - M) * li for _, m, li in parts)
    return O / l


def _score_rows(rng, n):
    """Score rows (log2 units) that exercise the lazy rescale: Gaussian rows at the workloads'
    logit spread, rows that climb by just under and just over the threshold per tile, a single
    huge outlier late in the row, and falling rows."""
    tile = 128
    steps = np.repeat(np.arange((n + tile - 1) // tile), tile)[:n]
    return [
        rng.standard_normal(n) * 1.5,
        rng.standard_normal(n) * 0.3 + steps * 7.9,          # climbs just under 2^8 per tile
        rng.standard_normal(n) * 0.3 + steps * 8.1,          # climbs just over it
        rng.standard_normal(n) * 0.3 + steps * 3.9,          # just under 2^4 per tile
        np.where(np.arange(n) == n - 77, 60.0, rng.standard_normal(n)),
        -steps * 5.0 + rng.standard_normal(n),
    ]


def test_online_softmax_and_merge_are_exact():
    """The kernels' online softmax -- lazy rescale at 2^kRescaleThreshold (bf16 P) or
    2^kP8Threshold with weights offset by 2^kP8Offset (e4m3 P) -- and the merge of split pieces
    give exact softmax attention whatever the split, and keep every weight at most
    2^(threshold + offset): 256 for both, below e4m3's largest finite value 448, with each row's
    largest weight at 2^offset or more (inside e4m3's normal range, which starts at 2^-6)."""
    tau16, off8, tau8 = _softmax_constants()
    assert (tau16, off8, tau8) == (8.0, 4.0, 4.0)
    rng = np.random.default_rng(11)
    n, d = 1000, 16                       # 8 key tiles, the last one ragged (104 keys)
    V = rng.standard_normal((n, d))
    tiles = [(lo, min(lo + 128, n)) for lo in range(0, n, 128)]
    for x in _score_rows(rng, n):
        w = np.exp2(x - x.max())
        exact = (w @ V) / w.sum()
        for tau, off in ((tau16, 0.0), (tau8, off8)):
            # whole row in one piece, then several random splits of the tile sequence
            cuts_list = [[]] + [sorted(rng.choice(np.arange(1, len(tiles)), size=k, replace=False).tolist())
                                for k in (1, 2, 4, 7) for _ in range(3)]
            for cuts in cuts_list:
                bounds = [0] + cuts + [len(tiles)]
                parts, pmax = [], 0.0
                for a, b in zip(bounds, bounds[1:]):
                    O, m, l, pm = _online_piece(x, V, tiles[a:b], tau, off)
                    parts.append((O, m, l))
                    pmax = max(pmax, pm)
                got = _merge(parts)
                np.testing.assert_allclose(got, exact, rtol=1e-12, atol=1e-12)
                assert pmax <= 2.0 ** (tau + off) * (1 + 1e-12)
                assert pmax >= 2.0 ** off
    assert 2.0 ** (tau8 + off8) < 448.0


def test_online_softmax_threshold_is_needed():
    """Guard for the test above: without the rescale (a reference max that never moves) the
    weights of a climbing row overflow any bound, so the threshold is what keeps them small."""
    rng = np.random.default_rng(3)
    n = 1000
    steps = np.repeat(np.arange(8), 128)[:n]
    x = rng.standard_normal(n) * 0.3 + steps * 8.1
    tiles = [(lo, min(lo + 128, n)) for lo in range(0, n, 128)]
    _, _, _, pmax = _online_piece(x, np.ones((n, 1)), tiles, tau=np.inf, off=0.0)
    assert pmax > 2.0 ** 50
