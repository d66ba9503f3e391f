"""GPU parity: the CUDA library, called through its C ABI, against the FP64 oracle.

Tables (segment list and chunk bitmap row) and cache contents are compared bit for bit;
attention outputs (fp32) within max-abs 1e-2 and mean-relative 2e-3, bf16 outputs within the
tolerance derived from those (parity_util.bf16_out_tol).  Full rows for the small workloads
(several 128-row tiles with ragged tails); on the 480p, 720p and stress workloads, sampled rows:
both ends, every tile edge, one random row in every 32-row quarter of every tile (every softmax
warp of every tile), plus random rows on top.  Every full-path schedule (persistent, grid,
three-buffer, CTA pair) is covered, as are the split-K path, the joint and committing forwards,
batched commits, and e4m3 handles (compared on their dequantised inputs; e4m3 P at its own
tolerance, parity_util.E4M3_P_TOL).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_sliding_b200 import synth
from block_causal_attention_sliding_b200.configs import WORKLOADS, Workload

from parity_util import (bf16_out_tol, check_table, compare, make_handle, sample_rows, stream_and_check,
                         stream_and_check_commit, stream_and_check_fp8, stream_and_check_joint)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_attention_sliding_b200 import build as B
    B.build()
    oracle.build()
    d = torch.device("cuda", 0)
    torch.cuda.set_device(d)
    return d


# a workload spanning several tiles with ragged tails everywhere: T = 300 = 128 + 128 + 44,
# n_cond = 40, two streams, three heads
RAGGED = Workload("ragged", B=2, H=3, d=128, T=300, n_cond=40, W=2, sink=True, chunks=6, steps=2)


# ------------------------------------------------------------------ K1 tables (bit-exact)

@pytest.mark.parametrize("name", ["tiny", "480p", "720p", "long720p", "stress"])
def test_tables_every_chunk(dev, name):
    wl = WORKLOADS[name]
    # the table depends only on W, sink, n_cond and T; a one-head, d=64 handle is enough
    small = dataclasses.replace(wl, B=1, H=1, d=64)
    h = make_handle(small, dev)
    z = torch.zeros((1, small.T, 1, 64), dtype=torch.bfloat16, device=dev)
    for k in range(wl.chunks):
        check_table(h.table().cpu().numpy(), k, wl.W, wl.sink, wl.n_cond, wl.T)
        h.append_chunk(z, z)
    assert h.status() == 0


@pytest.mark.parametrize("W,sink,n_cond", [(0, True, 8), (0, False, 0), (1, False, 3), (5, True, 0),
                                           (64, True, 2)])
def test_tables_other_windows(dev, W, sink, n_cond):
    wl = Workload("t", B=1, H=1, d=64, T=5, n_cond=n_cond, W=W, sink=sink, chunks=80, steps=1)
    h = make_handle(wl, dev)
    z = torch.zeros((1, 5, 1, 64), dtype=torch.bfloat16, device=dev)
    for k in range(wl.chunks):
        check_table(h.table().cpu().numpy(), k, W, sink, n_cond, 5)
        h.append_chunk(z, z)
    h.reset()
    check_table(h.table().cpu().numpy(), 0, W, sink, n_cond, 5)


# ------------------------------------------------------------------ K2 ring cache (bit-exact)

@pytest.mark.parametrize("W,sink", [(3, True), (2, False), (0, True), (1, True)])
def test_cache_contents_match_ring_model(dev, W, sink):
    B, H, d, T = 2, 3, 64, 40
    wl = Workload("c", B=B, H=H, d=d, T=T, n_cond=0, W=W, sink=sink, chunks=12, steps=1)
    h = make_handle(wl, dev)
    kc, vc = h.cache_views()
    kc.fill_(float("nan"))
    vc.fill_(float("nan"))
    ring = oracle.Ring(B=B, H=H, d=d, T=T, n_cond=0, W=W, sink=sink, Kc=None, Vc=None)
    chunks = {}
    for c in range(wl.chunks):
        K = synth.draw((B, T, H, d), 77 + 2 * c)
        V = synth.draw((B, T, H, d), 78 + 2 * c)
        chunks[c] = (K, V)
        h.append_chunk(K.to(dev), V.to(dev))
        ring.append(K, V)
        torch.cuda.synchronize()
        for s, held in enumerate(ring.slot_chunks()):
            gk = kc[:, :, s].cpu()          # [B, H, T, d]
            gv = vc[:, :, s].cpu()
            if held < 0:
                assert torch.isnan(gk.float()).all() and torch.isnan(gv.float()).all()
            else:
                ek, ev = chunks[held]
                assert torch.equal(gk.view(torch.int16), ek.permute(0, 2, 1, 3).contiguous().view(torch.int16))
                assert torch.equal(gv.view(torch.int16), ev.permute(0, 2, 1, 3).contiguous().view(torch.int16))
    assert h.status() == 0


@pytest.mark.parametrize("B,H,d,T", [(1, 24, 128, 300), (2, 3, 64, 17), (1, 32, 128, 130), (2, 50, 64, 9),
                                     (1, 24, 128, 3180)])
def test_commit_tma_matches_ring_model(dev, B, H, d, T):
    """Chunk commits by TMA bulk copies (forced where the automatic choice would take the copy
    kernel): every slot bit-exact against the oracle's ring model after every commit, empty slots
    untouched, tables advanced.  Shapes: one full head box and ragged row groups, fewer heads than
    a box, two head boxes (the second partly past H), d = 64 and the 720p chunk."""
    from parity_util import check_cache_against_ring
    W, chunks = 2, 6
    wl = Workload("ct", B=B, H=H, d=d, T=T, n_cond=0, W=W, sink=True, chunks=chunks, steps=1)
    h = make_handle(wl, dev, commit_path="tma")
    assert h.commit_kind() == "tma"
    kc, vc = h.cache_views()
    kc.fill_(float("nan"))
    vc.fill_(float("nan"))
    ring = oracle.Ring(B=B, H=H, d=d, T=T, n_cond=0, W=W, sink=True, Kc=None, Vc=None)
    held = {}
    for c in range(chunks):
        K = synth.draw((B, T, H, d), 900 + 2 * c)
        V = synth.draw((B, T, H, d), 901 + 2 * c)
        h.append_chunk(K.to(dev), V.to(dev))
        ring.append(K, V)
        held[c] = (K, V)
        torch.cuda.synchronize()
        check_cache_against_ring(h, ring, held)
        check_table(h.table().cpu().numpy(), c + 1, W, True, 0, T)
    assert h.status() == 0


def test_commit_path_choice(dev):
    """The automatic commit path: TMA where every SM gets a full ring of items (720p, stress),
    the copy kernel for smaller commits (480p, tiny); either can be forced."""
    kinds = {}
    for name in ("tiny", "480p", "720p", "stress"):
        wl = WORKLOADS[name]
        h = make_handle(wl, dev)
        kinds[name] = h.commit_kind()
        h.close()
    assert kinds == {"tiny": "copy", "480p": "copy", "720p": "tma", "stress": "tma"}, kinds
    wl = WORKLOADS["720p"]
    h = make_handle(wl, dev, commit_path="copy")
    assert h.commit_kind() == "copy"
    h.close()


# ------------------------------------------------------------------ K3 / K4 attention

@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("max_short_q", [-1, 0])
def test_tiny_full_stream(dev, out_dtype, max_short_q):
    """Every chunk and both denoise steps of the tiny workload, all rows; -1 forces the full
    path, 0 lets the 16 queries take the split-K path."""
    wl = WORKLOADS["tiny"]
    res = stream_and_check(wl, dev, chunks=wl.chunks, out_dtype=out_dtype, max_short_q=max_short_q)
    assert len(res) == wl.chunks * wl.steps


@pytest.mark.parametrize("schedule", ["persistent", "grid", "tri", "pair"])
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("max_short_q", [-1, 0])
def test_ragged_multi_tile(dev, d, max_short_q, schedule):
    """T = 300 gives one full pair and one single-tile pair per head; with the persistent
    schedule the few items per CTA force many-way splits of every pair's key tiles."""
    if schedule == "pair" and d != 128:
        pytest.skip("the CTA-pair schedule is d = 128 only (refused at create otherwise)")
    wl = dataclasses.replace(RAGGED, d=d)
    stream_and_check(wl, dev, chunks=wl.chunks, max_short_q=max_short_q, schedule=schedule)


@pytest.mark.parametrize("schedule", ["persistent", "grid", "tri", "pair"])
@pytest.mark.parametrize("W,sink,n_cond", [(0, False, 40), (0, True, 0), (4, False, 7), (1, True, 130)])
def test_ragged_other_windows(dev, W, sink, n_cond, schedule):
    wl = dataclasses.replace(RAGGED, W=W, sink=sink, n_cond=n_cond, chunks=6)
    stream_and_check(wl, dev, chunks=wl.chunks, max_short_q=-1, schedule=schedule)


@pytest.mark.parametrize("schedule", ["persistent", "tri", "pair"])
@pytest.mark.parametrize("H,T", [(1, 300), (1, 129), (5, 640), (2, 1400), (7, 3180)])
def test_persistent_split_shapes(dev, H, T, schedule):
    """Shapes whose cost line cuts units into 2, 3 or more pieces (one head: a handful of CTAs
    share every unit), and one with whole rounds before the stream-K leftover."""
    wl = Workload("split", B=1, H=H, d=128, T=T, n_cond=64, W=1, sink=True, chunks=4, steps=2)
    stream_and_check(wl, dev, chunks=wl.chunks, max_short_q=-1, schedule=schedule,
                     check_at=None if T < 3000 else {0, 3}, n_rows=None if T < 3000 else 48)


@pytest.mark.parametrize("schedule", ["persistent", "tri", "pair"])
def test_persistent_repeatable(dev, schedule):
    """The merge counters return to zero after every launch, and split pieces are merged in a
    fixed order whichever arrives last: repeated forwards give bit-identical output."""
    wl = RAGGED
    h = make_handle(wl, dev, max_short_q=-1, schedule=schedule)
    Kc, Vc = synth.cond_inputs(wl)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    Q, K, V = (t.to(dev) for t in synth.chunk_inputs(wl, 0, 0))
    first = h.forward(Q, K, V).clone()
    for _ in range(5):
        assert torch.equal(h.forward(Q, K, V), first)
    assert h.status() == 0


def test_stale_slots_poisoned_with_nan(dev):
    """Unused and not-yet-filled ring slots hold NaN: they are never read."""
    wl = dataclasses.replace(RAGGED, W=4, chunks=4)
    stream_and_check(wl, dev, chunks=wl.chunks, max_short_q=-1, poison=True)


def test_permutation_within_chunk(dev):
    """Permuting the current chunk's keys (with their values) leaves the output unchanged."""
    wl = RAGGED
    h = make_handle(wl, dev)
    Kc, Vc = synth.cond_inputs(wl)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    for k in range(3):
        _, K, V = synth.chunk_inputs(wl, k, 0)
        h.append_chunk(K.to(dev), V.to(dev))
    Q, K, V = synth.chunk_inputs(wl, 3, 0)
    perm = torch.randperm(wl.T, generator=torch.Generator().manual_seed(3))
    a = h.forward(Q.to(dev), K.to(dev), V.to(dev)).cpu().numpy()
    b = h.forward(Q.to(dev), K[:, perm].contiguous().to(dev), V[:, perm].contiguous().to(dev)).cpu().numpy()
    # the same keys fall into other tiles, so lazy-rescale points and bf16 rounding of P
    # differ: equal within the parity tolerance, not bit for bit
    compare(b, a.astype(np.float64))


def test_480p_sampled(dev):
    wl = WORKLOADS["480p"]
    res = stream_and_check(wl, dev, chunks=wl.chunks, check_at={0, 1, 2, 3, 4, 15}, n_rows=64,
                           keep_last=wl.W + 1, gen_on_device=True)
    assert len(res) == 12


def test_720p_sampled(dev):
    """The 720p workload on the benchmark's schedule with fp32 output: chunks 0, 1, W, W+1,
    W+2 and the last of 32, about 256 rows per check (every 32-row quarter of every tile)."""
    wl = WORKLOADS["720p"]
    res = stream_and_check(wl, dev, chunks=wl.chunks, check_at={0, 1, 3, 4, 5, 31}, n_rows=104,
                           keep_last=wl.W + 1, gen_on_device=True)
    assert len(res) == 12


def test_720p_bench_config(dev):
    """The 720p stream exactly as the benchmark runs it: automatic schedule (the persistent
    kernel), bf16 output.  At chunks 0, W + 1 and the last of 32: the bf16 output against the
    oracle within the tolerance derived for bf16 output, and bit for bit the round-to-nearest
    bf16 of the same kernel's fp32 output (a second handle fed the same inputs)."""
    wl = WORKLOADS["720p"]
    hb = make_handle(wl, dev, out_dtype=torch.bfloat16)
    hf = make_handle(wl, dev, out_dtype=torch.float32)
    assert hb.schedule_for() == "persistent" == hf.schedule_for()
    Kc, Vc = synth.cond_inputs(wl, device=dev)
    for h in (hb, hf):
        h.set_cond(Kc, Vc)
    Kc, Vc = Kc.cpu(), Vc.cpu()
    hist_K, hist_V, checked = [], [], 0
    for k in range(wl.chunks):
        for step in range(wl.steps):
            Q, K, V = synth.chunk_inputs(wl, k, step, device=dev)
            ob = hb.forward(Q, K, V)
            if k in (0, wl.W + 1, wl.chunks - 1):
                of = hf.forward(Q, K, V)
                assert torch.equal(ob, of.to(torch.bfloat16)), (k, step)
                r = sample_rows(wl.T, 104, seed=1000 * k + step)
                ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=k,
                                       Kc=Kc, Vc=Vc, hist_K=hist_K, hist_V=hist_V, Q=Q.cpu(), K_cur=K.cpu(),
                                       V_cur=V.cpu(), rows=r)
                compare(ob.float().cpu().numpy()[:, r], ref, *bf16_out_tol(ref))
                checked += 1
        for h in (hb, hf):
            h.append_chunk(K, V)
        hist_K.append(K.cpu())
        hist_V.append(V.cpu())
        for c in range(1, max(1, len(hist_K) - (wl.W + 1))):
            hist_K[c] = None
            hist_V[c] = None
    torch.cuda.synchronize()
    assert hb.status() == 0 and hf.status() == 0 and checked == 6


def test_720p_sampled_tri(dev):
    """The 720p workload on the three-buffer kernel: chunks 0, W+1 and the last of 12."""
    wl = WORKLOADS["720p"]
    res = stream_and_check(wl, dev, chunks=12, check_at={0, 4, 11}, n_rows=40, keep_last=wl.W + 1,
                           gen_on_device=True, schedule="tri")
    assert len(res) == 6


def test_720p_sampled_pair(dev):
    """The 720p workload on the CTA-pair kernel: chunks 0, W+1 and the last of 12, rows in every
    32-row quarter of every tile (25 Q tiles per head: the last pair has one tile)."""
    wl = WORKLOADS["720p"]
    res = stream_and_check(wl, dev, chunks=12, check_at={0, 4, 11}, n_rows=104, keep_last=wl.W + 1,
                           gen_on_device=True, schedule="pair")
    assert len(res) == 6


def test_480p_sampled_pair(dev):
    wl = WORKLOADS["480p"]
    res = stream_and_check(wl, dev, chunks=6, check_at={0, 1, 3, 5}, n_rows=64, keep_last=wl.W + 1,
                           gen_on_device=True, schedule="pair")
    assert len(res) == 8


def test_stress_sampled_pair(dev):
    """Four streams, 32 heads, W = 6, sigma-4 key outliers (O rescales) on the CTA-pair kernel."""
    wl = WORKLOADS["stress"]
    res = stream_and_check(wl, dev, chunks=8, check_at={0, 7}, n_rows=0, keep_last=wl.W + 1,
                           gen_on_device=True, schedule="pair")
    assert len(res) == 4


def test_stress_sampled_tri(dev):
    wl = WORKLOADS["stress"]
    res = stream_and_check(wl, dev, chunks=8, check_at={7}, n_rows=0, keep_last=wl.W + 1,
                           gen_on_device=True, schedule="tri")
    assert len(res) == 2


def test_stress_sampled(dev):
    """Four streams, 32 heads, W = 6, 512 condition tokens, 1% sigma-4 key outliers."""
    wl = WORKLOADS["stress"]
    res = stream_and_check(wl, dev, chunks=9, check_at={0, 7, 8}, n_rows=0, keep_last=wl.W + 1,
                           gen_on_device=True)
    assert len(res) == 6


@pytest.mark.parametrize("n_q", [1, 16, 64, 128])
def test_short_queries_720p(dev, n_q):
    """Split-K path: n_q queries against the steady-state 720p cache."""
    wl = WORKLOADS["720p"]
    stream_and_check(wl, dev, chunks=6, check_at={0, 5}, n_q=n_q, keep_last=wl.W + 1, gen_on_device=True)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("H", [3, 24])
@pytest.mark.parametrize("n_q", [1, 33, 100, 128])
def test_short_queries_ragged(dev, d, H, n_q):
    """Split-K path on ragged shapes, all rows of every chunk: query counts that fill one to four
    32-row quarters of the tile, partly; H = 3 leaves most slices empty or one tile long, H = 24
    gives slices of four and five tiles (both S buffers, odd and even counts)."""
    wl = dataclasses.replace(RAGGED, d=d, H=H)
    res = stream_and_check(wl, dev, chunks=wl.chunks, n_q=n_q, max_short_q=0)
    assert len(res) == wl.chunks * wl.steps


@pytest.mark.parametrize("d", [128, 64])
def test_short_queries_rescale(dev, d):
    """Split-K path with all key tiles of a head in one slice (B*H above the SM count) and the
    last chunk's keys scaled by 8, so that the row max jumps on the final tiles: the O rescale
    then runs while the next tile's scores are already in the other S buffer."""
    wl = Workload("rescale", B=1, H=150, d=d, T=300, n_cond=40, W=2, sink=True, chunks=4, steps=1)
    h = make_handle(wl, dev, max_short_q=0)
    Kc, Vc = synth.cond_inputs(wl)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    hist_K, hist_V = [], []
    for k in range(wl.chunks):
        Q, K, V = synth.chunk_inputs(wl, k, 0, n_q=40)
        if k == wl.chunks - 1:
            K = K * 8   # exact in bf16
        out = h.forward(Q.to(dev), K.to(dev), V.to(dev))
        ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=k, Kc=Kc, Vc=Vc,
                               hist_K=hist_K, hist_V=hist_V, Q=Q, K_cur=K, V_cur=V)
        compare(out.float().cpu().numpy(), ref)
        h.append_chunk(K.to(dev), V.to(dev))
        hist_K.append(K)
        hist_V.append(V)
    torch.cuda.synchronize()
    assert h.status() == 0


# ------------------------------------------------------------------ condition-stream queries

@pytest.mark.parametrize("schedule", ["auto", "persistent", "grid", "tri"])
def test_joint_tiny_stream(dev, schedule):
    """The tiny workload through the joint forward: the 16 chunk queries and the 8 condition
    queries share one launch; every chunk and step, all rows of both outputs."""
    wl = WORKLOADS["tiny"]
    res = stream_and_check_joint(wl, dev, chunks=wl.chunks, schedule=schedule)
    assert len(res) == 2 * wl.chunks * wl.steps


@pytest.mark.parametrize("schedule", ["persistent", "grid", "tri", "pair"])
@pytest.mark.parametrize("d,T,n_cond", [(128, 300, 40), (128, 256, 130), (64, 300, 200), (128, 129, 1)])
def test_joint_ragged(dev, d, T, n_cond, schedule):
    """Ragged tails in both query sets: the chunk's last Q tile and a condition tile share a
    pair (T = 300, n_cond = 40: 3 + 1 tiles), two condition tiles form a pair (n_cond = 130),
    an odd tile total (T = 300, n_cond = 200 at d = 64: 3 + 2 tiles), one condition query."""
    if schedule == "pair" and d != 128:
        pytest.skip("the CTA-pair schedule is d = 128 only (refused at create otherwise)")
    wl = dataclasses.replace(RAGGED, d=d, T=T, n_cond=n_cond, chunks=4)
    res = stream_and_check_joint(wl, dev, chunks=wl.chunks, schedule=schedule)
    assert len(res) == 2 * wl.chunks * wl.steps


@pytest.mark.parametrize("schedule", ["persistent", "tri"])
def test_prompt_change_mid_stream(dev, schedule):
    """Prompt edits while streaming: the condition K/V are replaced before chunks 2 and 4;
    both outputs follow the new condition from that chunk on, and the cached history (sink
    and window) is unaffected."""
    wl = dataclasses.replace(RAGGED, chunks=6)
    res = stream_and_check_joint(wl, dev, chunks=wl.chunks, prompts={2: 1, 4: 2}, schedule=schedule)
    assert len(res) == 2 * wl.chunks * wl.steps


def test_joint_720p_sampled(dev):
    """720p: 3180 chunk queries and 256 condition queries in one launch, sampled rows at
    chunks 0 and W + 1, with a prompt change before chunk W + 1."""
    wl = WORKLOADS["720p"]
    res = stream_and_check_joint(wl, dev, chunks=5, check_at={0, 4}, n_rows=40, prompts={4: 1},
                                 keep_last=wl.W + 1, gen_on_device=True)
    assert len(res) == 8


# ------------------------------------------------------------------ fused clean-KV commit

@pytest.mark.parametrize("schedule", ["persistent", "grid", "tri", "pair"])
@pytest.mark.parametrize("W,sink", [(2, True), (1, False), (3, True), (0, True)])
def test_commit_in_forward_stream(dev, W, sink, schedule):
    """The clean pass commits its own K/V: tables and cache contents bit-exact against the
    oracle's ring with a spare slot after every chunk, both outputs against the oracle."""
    wl = dataclasses.replace(RAGGED, W=W, sink=sink, chunks=7)
    res = stream_and_check_commit(wl, dev, chunks=wl.chunks, schedule=schedule)
    assert len(res) == wl.chunks * wl.steps


@pytest.mark.parametrize("schedule", ["persistent", "tri"])
@pytest.mark.parametrize("fp8", ["qk", "qkv"])
@pytest.mark.parametrize("W,sink", [(2, True), (1, False)])
def test_fp8_commit_in_forward_stream(dev, W, sink, fp8, schedule):
    """The committing forward on e4m3 handles (e4m3 K, and V with "qkv"): the cache holds the
    committed e4m3 tensors bit for bit after every chunk, tables exact, both outputs against the
    oracle on the dequantised inputs.  The persistent kernel stores the tiles itself (one box of
    128-byte rows per e4m3 tile); the three-buffer kernel's forward is followed by the copy."""
    wl = dataclasses.replace(RAGGED, W=W, sink=sink, chunks=6)
    res = stream_and_check_commit(wl, dev, chunks=wl.chunks, schedule=schedule, fp8=fp8)
    assert len(res) == wl.chunks * wl.steps


def test_fp8_commit_720p_sampled(dev):
    """720p, e4m3 Q/K/V, the clean pass committing on the persistent kernel: sampled rows at
    chunks 0, W + 1 and the last of 6; cache and table checked after every chunk."""
    wl = WORKLOADS["720p"]
    res = stream_and_check_commit(wl, dev, chunks=6, check_at={0, 4, 5}, n_rows=32, keep_last=wl.W + 2,
                                  gen_on_device=True, fp8="qkv")
    assert len(res) == 6


@pytest.mark.parametrize("schedule", ["persistent", "grid"])
def test_commit_mixed_with_append(dev, schedule):
    """Commits in the forward and plain appends interleaved on one handle: the same cache."""
    wl = dataclasses.replace(RAGGED, d=64, chunks=8)
    stream_and_check_commit(wl, dev, chunks=wl.chunks, schedule=schedule, append_at={1, 4, 5})


@pytest.mark.parametrize("schedule", ["persistent", "tri"])
@pytest.mark.parametrize("H,T", [(1, 129), (5, 640)])
def test_commit_split_shapes(dev, H, T, schedule):
    """Shapes whose first Q-tile pair is cut between several CTAs: every K/V tile of the chunk
    is stored exactly once."""
    wl = Workload("split", B=1, H=H, d=128, T=T, n_cond=64, W=2, sink=True, chunks=5, steps=2)
    stream_and_check_commit(wl, dev, chunks=wl.chunks, schedule=schedule)


def test_commit_720p_sampled(dev):
    """720p in the benchmark's launch configuration, clean pass committing: sampled rows at
    chunks 0, W + 1 and the last, cache bit-exact after every chunk."""
    wl = WORKLOADS["720p"]
    res = stream_and_check_commit(wl, dev, chunks=7, check_at={0, 4, 6}, n_rows=32, keep_last=wl.W + 1,
                                  gen_on_device=True)
    assert len(res) == 6


# ------------------------------------------------------------------ several layers per chunk step

LAYERS = [dict(W=2, sink=True, n_cond=40, commit_in_forward=False), dict(W=1, sink=False, n_cond=8, commit_in_forward=False),
          dict(W=3, sink=True, n_cond=0, commit_in_forward=True), dict(W=0, sink=True, n_cond=40, commit_in_forward=False),
          dict(W=2, sink=False, n_cond=130, commit_in_forward=True)]


@pytest.mark.parametrize("commit_path,d", [("copy", 64), ("tma", 64), ("tma", 128)])
def test_append_batched_matches_ring(dev, commit_path, d):
    """Five layers with different windows, sinks, condition counts and slot counts, committed
    together: every layer's table and cache equal its own oracle model, bit for bit, with the
    copy kernel and with the batched TMA bulk copies (every handle forcing them)."""
    from block_causal_attention_sliding_b200.api import append_chunk_batched
    from parity_util import check_cache_against_ring
    B, H, T, chunks = 2, 3, 40, 9
    hs, rings, held = [], [], []
    for cfg in LAYERS:
        wl = Workload("l", B=B, H=H, d=d, T=T, n_cond=cfg["n_cond"], W=cfg["W"], sink=cfg["sink"], chunks=chunks, steps=1)
        h = make_handle(wl, dev, commit_in_forward=cfg["commit_in_forward"], commit_path=commit_path)
        assert h.commit_kind() == commit_path
        kc, vc = h.cache_views()
        kc.fill_(float("nan"))
        vc.fill_(float("nan"))
        hs.append(h)
        rings.append(oracle.Ring(B=B, H=H, d=d, T=T, n_cond=0, W=cfg["W"], sink=cfg["sink"], Kc=None, Vc=None, R=h.R))
        held.append({})
    for c in range(chunks):
        Ks = [synth.draw((B, T, H, d), 500 + 10 * c + 2 * l) for l in range(len(hs))]
        Vs = [synth.draw((B, T, H, d), 501 + 10 * c + 2 * l) for l in range(len(hs))]
        append_chunk_batched(hs, [K.to(dev) for K in Ks], [V.to(dev) for V in Vs])
        torch.cuda.synchronize()
        for l, (h, cfg) in enumerate(zip(hs, LAYERS)):
            rings[l].append(Ks[l], Vs[l])
            held[l][c] = (Ks[l], Vs[l])
            check_cache_against_ring(h, rings[l], held[l])
            check_table(h.table().cpu().numpy(), c + 1, cfg["W"], cfg["sink"], cfg["n_cond"], T, R=h.R)
    for h in hs:
        assert h.status() == 0


def test_decode_step_graph_capture(dev):
    """Short-query forwards (the split-K kernel, then its combine as a programmatic dependent
    launch) and a single-handle commit (copy and table advance in one launch), captured once into
    a CUDA graph and replayed chunk after chunk, give the eager calls' outputs bit for bit."""
    wl = dataclasses.replace(RAGGED, H=24, chunks=6)
    n_q = 40

    def handle():
        h = make_handle(wl, dev, max_short_q=0)
        Kc, Vc = synth.cond_inputs(wl)
        h.set_cond(Kc.to(dev), Vc.to(dev))
        return h

    def inputs(k):
        return [[t.to(dev) for t in synth.chunk_inputs(wl, k, s, n_q=n_q)] for s in range(wl.steps)]

    eager = handle()
    eager_out = []
    for k in range(wl.chunks):
        x = inputs(k)
        eager_out.append([eager.forward(*x[s]).clone() for s in range(wl.steps)])
        eager.append_chunk(x[-1][1], x[-1][2])
    torch.cuda.synchronize()
    g = handle()
    static_in = inputs(0)
    static_out = [torch.empty((wl.B, n_q, wl.H, wl.d), dtype=torch.float32, device=dev) for _ in range(wl.steps)]

    def step():
        for s in range(wl.steps):
            g.forward(*static_in[s], out=static_out[s])
        g.append_chunk(static_in[-1][1], static_in[-1][2])

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.current_stream().wait_stream(side)
    for k in range(wl.chunks):
        for dst_s, src_s in zip(static_in, inputs(k)):
            for dst, src in zip(dst_s, src_s):
                dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        for s in range(wl.steps):
            assert torch.equal(static_out[s], eager_out[k][s]), (k, s)
    assert np.array_equal(g.table().cpu().numpy(), eager.table().cpu().numpy())
    assert eager.status() == 0 and g.status() == 0


def test_chunk_step_graph_capture(dev):
    """A three-layer chunk step -- each layer's two forwards, then one batched commit -- captured
    once into a CUDA graph and replayed chunk after chunk gives the same outputs, bit for bit,
    as the same calls run eagerly, and both match the oracle at the checked chunks."""
    from block_causal_attention_sliding_b200.api import append_chunk_batched
    wl = dataclasses.replace(RAGGED, chunks=6)
    L = 3
    def layer_handles():
        hs = []
        for l in range(L):
            h = make_handle(wl, dev, schedule="persistent" if l != 1 else "tri")
            Kc, Vc = synth.cond_inputs(wl, seed=l)
            h.set_cond(Kc.to(dev), Vc.to(dev))
            hs.append(h)
        return hs
    def inputs(k):
        return [[[t.to(dev) for t in synth.chunk_inputs(wl, k, s, seed=10 + l)] for s in range(wl.steps)] for l in range(L)]
    # eager
    eager_hs = layer_handles()
    eager_out = []
    for k in range(wl.chunks):
        x = inputs(k)
        outs = [[eager_hs[l].forward(*x[l][s]).clone() for s in range(wl.steps)] for l in range(L)]
        append_chunk_batched(eager_hs, [x[l][-1][1] for l in range(L)], [x[l][-1][2] for l in range(L)])
        eager_out.append(outs)
    torch.cuda.synchronize()
    # graph: static input and output buffers, one capture of a whole chunk step
    g_hs = layer_handles()
    static_in = inputs(0)
    static_out = [[torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.float32, device=dev) for _ in range(wl.steps)]
                  for _ in range(L)]

    def step():
        for l in range(L):
            for s in range(wl.steps):
                g_hs[l].forward(*static_in[l][s], out=static_out[l][s])
        append_chunk_batched(g_hs, [static_in[l][-1][1] for l in range(L)], [static_in[l][-1][2] for l in range(L)])

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.current_stream().wait_stream(side)
    for k in range(wl.chunks):
        x = inputs(k)
        for l in range(L):
            for s in range(wl.steps):
                for dst, src in zip(static_in[l][s], x[l][s]):
                    dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        for l in range(L):
            for s in range(wl.steps):
                assert torch.equal(static_out[l][s], eager_out[k][l][s]), (k, l, s)
    for h in eager_hs + g_hs:
        assert h.status() == 0
    # spot check against the oracle: layer 0, last chunk, last step
    k = wl.chunks - 1
    Kc, Vc = synth.cond_inputs(wl, seed=0)
    hist = [synth.chunk_inputs(wl, c, wl.steps - 1, seed=10) for c in range(k)]
    Q, K, V = synth.chunk_inputs(wl, k, wl.steps - 1, seed=10)
    ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=k, Kc=Kc, Vc=Vc,
                           hist_K=[t[1] for t in hist], hist_V=[t[2] for t in hist], Q=Q, K_cur=K, V_cur=V)
    compare(eager_out[k][0][-1].cpu().numpy(), ref)


# ------------------------------------------------------------------ e4m3 queries and keys

@pytest.mark.parametrize("schedule", ["tri", "persistent"])
@pytest.mark.parametrize("W,sink,n_cond", [(2, True, 40), (1, False, 130), (0, True, 0)])
def test_fp8_qk_ragged(dev, W, sink, n_cond, schedule):
    """e4m3 Q and K (S on kind::f8f6f4, e4m3 K cache), bf16 V: every chunk and step, all rows,
    against the oracle on the dequantised inputs, on both kernels with an e4m3 form."""
    wl = dataclasses.replace(RAGGED, W=W, sink=sink, n_cond=n_cond, chunks=6)
    res = stream_and_check_fp8(wl, dev, chunks=wl.chunks, schedule=schedule)
    assert len(res) == wl.chunks * wl.steps


@pytest.mark.parametrize("schedule", ["tri", "persistent"])
def test_fp8_qk_joint(dev, schedule):
    """e4m3 chunk and condition queries in one joint launch."""
    wl = dataclasses.replace(RAGGED, n_cond=130, chunks=4)
    res = stream_and_check_fp8(wl, dev, chunks=wl.chunks, joint=True, schedule=schedule)
    assert len(res) == 2 * wl.chunks * wl.steps


@pytest.mark.parametrize("commit_path", ["copy", "tma"])
def test_fp8_qk_cache_bytes(dev, commit_path):
    """The e4m3 K cache holds exactly the appended e4m3 keys (bit for bit) at half the bytes, with
    either commit path (the TMA one moves K in boxes of 128-byte rows, V in 256-byte rows)."""
    wl = dataclasses.replace(RAGGED, chunks=3)
    sc = synth.FP8_SCALE
    h = make_handle(wl, dev)
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    h8 = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                qk_fp8=True, q_scale=sc, k_scale=sc, commit_path=commit_path, device=dev)
    assert h8.commit_kind() == commit_path
    assert h8.workspace_bytes() < h.workspace_bytes()
    kc, vc = h8.cache_views()
    for c in range(wl.chunks):
        _, K8, V = synth.chunk_inputs_fp8(wl, c, 1)
        h8.append_chunk(K8.to(dev), V.to(dev))
        torch.cuda.synchronize()
        s_ = oracle.slot(c, wl.W, wl.sink)
        assert torch.equal(kc[:, :, s_].cpu().view(torch.uint8), K8.permute(0, 2, 1, 3).contiguous().view(torch.uint8))
        assert torch.equal(vc[:, :, s_].cpu().view(torch.int16), V.permute(0, 2, 1, 3).contiguous().view(torch.int16))
    assert h8.status() == 0


@pytest.mark.parametrize("schedule", ["tri", "persistent"])
@pytest.mark.parametrize("W,sink,n_cond", [(2, True, 40), (1, False, 130), (0, True, 0)])
def test_fp8_pv_ragged(dev, W, sink, n_cond, schedule):
    """e4m3 Q, K and V (P V on kind::f8f6f4 with e4m3 P, e4m3 K and V caches): every chunk and
    step, all rows, against the oracle on the dequantised inputs at the e4m3-P tolerance."""
    wl = dataclasses.replace(RAGGED, W=W, sink=sink, n_cond=n_cond, chunks=6)
    res = stream_and_check_fp8(wl, dev, chunks=wl.chunks, pv8=True, schedule=schedule)
    assert len(res) == wl.chunks * wl.steps


@pytest.mark.parametrize("schedule", ["tri", "persistent"])
def test_fp8_pv_joint(dev, schedule):
    """e4m3 chunk and condition queries with e4m3 V in one joint launch."""
    wl = dataclasses.replace(RAGGED, n_cond=130, chunks=4)
    res = stream_and_check_fp8(wl, dev, chunks=wl.chunks, joint=True, pv8=True, schedule=schedule)
    assert len(res) == 2 * wl.chunks * wl.steps


@pytest.mark.parametrize("commit_path", ["copy", "tma"])
def test_fp8_pv_cache_bytes(dev, commit_path):
    """With e4m3 V the V cache holds exactly the appended e4m3 values (bit for bit), and the whole
    K/V cache takes half the bytes of the bf16 one, with either commit path."""
    wl = dataclasses.replace(RAGGED, chunks=3)
    sc = synth.FP8_SCALE
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    h = make_handle(wl, dev)
    h8 = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                qk_fp8=True, q_scale=sc, k_scale=sc, pv_fp8=True, v_scale=sc,
                                commit_path=commit_path, device=dev)
    assert h8.commit_kind() == commit_path
    kc, vc = h8.cache_views()
    kb, vb = h.cache_views()
    assert kc.numel() * kc.element_size() * 2 == kb.numel() * kb.element_size()
    assert vc.numel() * vc.element_size() * 2 == vb.numel() * vb.element_size()
    for c in range(wl.chunks):
        _, K8, V8 = synth.chunk_inputs_fp8(wl, c, 1, v8=True)
        h8.append_chunk(K8.to(dev), V8.to(dev))
        torch.cuda.synchronize()
        s_ = oracle.slot(c, wl.W, wl.sink)
        assert torch.equal(kc[:, :, s_].cpu().view(torch.uint8), K8.permute(0, 2, 1, 3).contiguous().view(torch.uint8))
        assert torch.equal(vc[:, :, s_].cpu().view(torch.uint8), V8.permute(0, 2, 1, 3).contiguous().view(torch.uint8))
    assert h8.status() == 0


def test_fp8_pv_720p_sampled(dev):
    """720p with e4m3 Q, K and V: sampled rows at chunks 0, W + 1 and the last of 7."""
    wl = WORKLOADS["720p"]
    res = stream_and_check_fp8(wl, dev, chunks=7, check_at={0, 4, 6}, n_rows=32, keep_last=wl.W + 1,
                               gen_on_device=True, pv8=True)
    assert len(res) == 6


@pytest.mark.parametrize("pv8", [False, True])
@pytest.mark.parametrize("n_q", [1, 128])
def test_fp8_short_queries_720p(dev, n_q, pv8):
    """Split-K path with e4m3 Q and K (and V, P with pv8) against the steady-state 720p cache,
    all n_q rows at chunks 0 and 5."""
    wl = WORKLOADS["720p"]
    res = stream_and_check_fp8(wl, dev, chunks=6, check_at={0, 5}, keep_last=wl.W + 1, gen_on_device=True,
                               pv8=pv8, n_q=n_q)
    assert len(res) == 2 * wl.steps


@pytest.mark.parametrize("pv8", [False, True])
@pytest.mark.parametrize("H", [3, 24])
@pytest.mark.parametrize("n_q", [1, 33, 100])
def test_fp8_short_queries_ragged(dev, H, n_q, pv8):
    """Split-K path with e4m3 inputs on ragged shapes, every chunk and step: H = 3 leaves most
    slices empty or one tile long, H = 24 gives slices of several tiles."""
    wl = dataclasses.replace(RAGGED, H=H, chunks=5)
    res = stream_and_check_fp8(wl, dev, chunks=wl.chunks, pv8=pv8, n_q=n_q)
    assert len(res) == wl.chunks * wl.steps


@pytest.mark.parametrize("pv8", [False, True])
def test_fp8_480p_sampled(dev, pv8):
    """480p with e4m3 inputs on the automatic schedule (the three-buffer kernel: 96 Q-tile pairs
    on 148 SMs), sampled rows at chunks 0, W + 1 and the last of 6."""
    wl = WORKLOADS["480p"]
    res = stream_and_check_fp8(wl, dev, chunks=6, check_at={0, 3, 5}, n_rows=64, keep_last=wl.W + 1,
                               gen_on_device=True, pv8=pv8)
    assert len(res) == 6


def test_fp8_qk_720p_sampled(dev):
    """720p with e4m3 Q and K: sampled rows at chunks 0, W + 1 and the last of 7."""
    wl = WORKLOADS["720p"]
    res = stream_and_check_fp8(wl, dev, chunks=7, check_at={0, 4, 6}, n_rows=32, keep_last=wl.W + 1,
                               gen_on_device=True)
    assert len(res) == 6


def test_long_horizon_constant_memory(dev):
    """225 chunks: the device table stays exact, memory does not grow, the last chunk matches
    the oracle on sampled rows."""
    wl = WORKLOADS["long720p"]
    torch.cuda.synchronize()
    res = None
    before = None
    h = make_handle(wl, dev)
    ws = h.workspace_bytes()
    del h
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated(dev)
    res = stream_and_check(wl, dev, chunks=wl.chunks, check_at={wl.chunks - 1}, n_rows=24,
                           keep_last=wl.W + 1, gen_on_device=True)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated(dev) <= before + 4096
    assert len(res) == 2 and ws > 0
