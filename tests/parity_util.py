"""Shared helpers for the GPU parity tests: stream a workload through the CUDA library and the
FP64 oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from block_causal_attention_sliding_b200 import synth
from block_causal_attention_sliding_b200.api import SlidingWindowAttention

MAX_ABS = 1e-2      # tolerances on fp32 output, against the FP64 oracle
MEAN_REL = 2e-3     # mean-relative = sum |got - ref| / sum |ref|


BF16_U = 2.0 ** -8   # unit roundoff of bf16 (8 significant bits, round to nearest even)


def bf16_out_tol(ref: np.ndarray, max_abs: float = MAX_ABS, mean_rel: float = MEAN_REL):
    """Tolerance for bf16 output, derived from the fp32 one.  The kernel computes the output
    in fp32 and rounds it once to bf16, which moves each value by at most BF16_U of itself:
    |got - ref| <= |fp32 - ref| + BF16_U (|ref| + |fp32 - ref|).  So max-abs grows by
    BF16_U (max|ref| + max_abs) and mean-relative by BF16_U (1 + mean_rel)."""
    top = float(np.abs(ref).max()) if ref.size else 0.0
    return max_abs + BF16_U * (top + max_abs), mean_rel + BF16_U * (1.0 + mean_rel)


def _log_errors(ma: float, mr: float, n: int, tol) -> None:
    """Append the observed errors to the file named by SWATTN_PARITY_LOG (one JSON line per
    comparison, tagged with the running test), when that variable is set."""
    path = os.environ.get("SWATTN_PARITY_LOG")
    if not path:
        return
    rec = {"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], "max_abs": ma, "mean_rel": mr,
           "values": n, "tol": [float(tol[0]), float(tol[1])]}
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def compare(got: np.ndarray, ref: np.ndarray, max_abs: float = MAX_ABS, mean_rel: float = MEAN_REL):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite output"
    d = np.abs(got.astype(np.float64) - ref)
    ma = float(d.max())
    mr = float(d.sum() / max(np.abs(ref).sum(), 1e-300))
    _log_errors(ma, mr, int(d.size), (max_abs, mean_rel))
    assert ma <= max_abs and mr <= mean_rel, f"max-abs {ma:.3e} (<= {max_abs}), mean-rel {mr:.3e} (<= {mean_rel})"
    return ma, mr


VIS_SPAN = 64      # chunks covered by the window word of the device's bitmap row


def vis_offset(W: int) -> int:
    """Index of the bitmap row in the device table (after 3 + 4 (W + 3) segment ints)."""
    return 3 + 4 * (W + 3)


def expand_vis_row(words, k: int) -> np.ndarray:
    """The device's constant-size bitmap row [vis_sink, vis_lo, vis_hi] expanded to the full row
    vis[k][j], j < k (uint8).  Bit i of vis_hi:vis_lo is chunk k - 64 + i; vis_sink is chunk 0.
    Asserts that no bit names a chunk before 0 and that the two encodings of chunk 0 agree."""
    vis_sink, lo, hi = (int(x) & 0xffffffff for x in words)
    assert vis_sink in (0, 1), vis_sink
    word = lo | (hi << 32)
    row = np.zeros(k, dtype=np.uint8)
    for i in range(VIS_SPAN):
        j = k - VIS_SPAN + i
        bit = (word >> i) & 1
        if j < 0:
            assert bit == 0, (k, i)
        elif bit:
            row[j] = 1
    if k >= 1:
        if k <= VIS_SPAN:
            assert row[0] == vis_sink, (k, row[0], vis_sink)
        row[0] |= vis_sink
    else:
        assert vis_sink == 0
    return row


def check_table(got: np.ndarray, k: int, W: int, sink: bool, n_cond: int, T: int, R=None) -> None:
    """The device table for active chunk k, bit for bit against the oracle: the segment list
    (unused entries -1) and the chunk bitmap row."""
    off = vis_offset(W)
    assert got.shape[0] == off + 3, got.shape
    ref = oracle.table(k, W, sink, n_cond, T, R=R)
    np.testing.assert_array_equal(got[: len(ref)], ref)
    assert (got[len(ref):off] == -1).all()
    np.testing.assert_array_equal(expand_vis_row(got[off:off + 3], k), oracle.vis_row(k, W, sink))


def sample_rows(n_q: int, n: int, seed: int) -> np.ndarray:
    """Query rows checked on the large workloads:
      - both ends and both sides of every 128-row tile edge;
      - one random row in every 32-row quarter of every tile, so that every softmax warp (a
        warp owns one 32-lane quarter of a tile's rows) is compared in every tile;
      - n random rows on top of those (distinct from them)."""
    fixed = {0, 1, n_q - 1, n_q - 2}
    for e in range(128, n_q, 128):
        fixed.update({e - 1, e})
    rng = np.random.default_rng(seed)
    for q0 in range(0, n_q, 32):
        fixed.add(int(rng.integers(q0, min(q0 + 32, n_q))))
    fixed = {r for r in fixed if 0 <= r < n_q}
    rest = np.array(sorted(set(range(n_q)) - fixed), dtype=np.int64)
    extra = rng.choice(rest, size=min(len(rest), max(0, n)), replace=False) if len(rest) else []
    return np.array(sorted(fixed | set(int(x) for x in extra)), dtype=np.int32)


def make_handle(wl, dev, *, out_dtype=torch.float32, max_short_q=0, W=None, sink=None, n_cond=None,
                schedule="auto", commit_in_forward=False, commit_path="auto"):
    return SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W if W is None else W,
                                  n_cond=wl.n_cond if n_cond is None else n_cond,
                                  sink=wl.sink if sink is None else sink, out_dtype=out_dtype,
                                  max_short_q=max_short_q, schedule=schedule,
                                  commit_in_forward=commit_in_forward, commit_path=commit_path, device=dev)


def tol_for(out_dtype, ref, tol=None):
    """The tolerance of one comparison: the one given, else the parity tolerance for fp32 output
    and the derived one (bf16_out_tol) for bf16 output."""
    if tol is not None:
        return tol
    return bf16_out_tol(ref) if out_dtype == torch.bfloat16 else (MAX_ABS, MEAN_REL)


def stream_and_check(wl, dev, *, chunks, check_at=None, rows=None, n_rows=None, n_q=None,
                     out_dtype=torch.float32, max_short_q=0, poison=False, seed=0,
                     tol=None, keep_last=None, gen_on_device=False, schedule="auto"):
    """Stream `chunks` chunks (2 forwards then an append each).  At the chunks in `check_at`
    (all if None) compare the CUDA output with the oracle, on all rows or on sampled rows.
    With gen_on_device the seeded draws use the GPU generator (faster for big shapes); the
    oracle then reads host copies of exactly those bf16 values.
    Returns a list of (k, step, max_abs, mean_rel)."""
    h = make_handle(wl, dev, out_dtype=out_dtype, max_short_q=max_short_q, schedule=schedule)
    if poison:
        kc, vc = h.cache_views()
        kc.fill_(float("nan"))
        vc.fill_(float("nan"))
    gdev = dev if gen_on_device else "cpu"
    Kc, Vc = synth.cond_inputs(wl, seed=seed, device=gdev)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    Kc, Vc = Kc.cpu(), Vc.cpu()
    hist_K, hist_V = [], []
    results = []
    nq = wl.T if n_q is None else n_q
    for k in range(chunks):
        for step in range(wl.steps):
            Q, K, V = synth.chunk_inputs(wl, k, step, seed=seed, n_q=nq, device=gdev)
            out = h.forward(Q.to(dev), K.to(dev), V.to(dev))
            if check_at is None or k in check_at:
                Q = Q.cpu()
                r = rows
                if r is None and n_rows is not None:
                    r = sample_rows(nq, n_rows, seed=1000 * k + step)
                ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink,
                                       k=k, Kc=Kc, Vc=Vc, hist_K=hist_K, hist_V=hist_V, Q=Q,
                                       K_cur=K.cpu(), V_cur=V.cpu(), rows=r)
                got = out.float().cpu().numpy()
                if r is not None:
                    got = got[:, r]
                ma, mr = compare(got, ref, *tol_for(out_dtype, ref, tol))
                results.append((k, step, ma, mr))
        h.append_chunk(K.to(dev), V.to(dev))
        hist_K.append(K.cpu())
        hist_V.append(V.cpu())
        if keep_last is not None:
            # only the sink and the most recent chunks are ever visible; drop the rest from
            # host memory (the oracle raises if a dropped chunk turns out to be visible)
            for c in range(1, max(1, len(hist_K) - keep_last)):
                hist_K[c] = None
                hist_V[c] = None
    torch.cuda.synchronize()
    assert h.status() == 0, f"device status {h.status():#x}"
    return results


def stream_and_check_joint(wl, dev, *, chunks, check_at=None, n_rows=None, prompts=None,
                           out_dtype=torch.float32, seed=0, schedule="auto", gen_on_device=False,
                           keep_last=None, tol=(MAX_ABS, MEAN_REL)):
    """Stream `chunks` chunks through the joint forward (the chunk's queries and the condition
    queries in one launch; 2 steps, then an append each).  `prompts` maps a chunk index to a
    prompt version: before that chunk the condition K/V are replaced (set_cond), and the oracle
    uses the new ones from there on.  At the chunks in `check_at` (all if None) both outputs
    are compared with the oracle, on all rows or on `n_rows` sampled rows of each.
    Returns a list of (k, step, which, max_abs, mean_rel)."""
    h = make_handle(wl, dev, out_dtype=out_dtype, schedule=schedule)
    gdev = dev if gen_on_device else "cpu"
    prompts = dict(prompts or {})
    Kc, Vc = synth.cond_inputs(wl, seed=seed, device=gdev)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    Kc, Vc = Kc.cpu(), Vc.cpu()
    hist_K, hist_V = [], []
    results = []
    for k in range(chunks):
        if k in prompts:
            Kc, Vc = synth.cond_inputs(wl, seed=seed, version=prompts[k], device=gdev)
            h.set_cond(Kc.to(dev), Vc.to(dev))
            Kc, Vc = Kc.cpu(), Vc.cpu()
        for step in range(wl.steps):
            Q, K, V = synth.chunk_inputs(wl, k, step, seed=seed, device=gdev)
            Qc = synth.cond_queries(wl, k, step, seed=seed, device=gdev)
            out, out_c = h.forward_joint(Q.to(dev), Qc.to(dev), K.to(dev), V.to(dev))
            if check_at is None or k in check_at:
                for which, q, o, n in (("chunk", Q, out, wl.T), ("cond", Qc, out_c, wl.n_cond)):
                    r = None if n_rows is None else sample_rows(n, n_rows, seed=1000 * k + step)
                    ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink,
                                           k=k, Kc=Kc, Vc=Vc, hist_K=hist_K, hist_V=hist_V, Q=q.cpu(),
                                           K_cur=K.cpu(), V_cur=V.cpu(), rows=r)
                    got = o.float().cpu().numpy()
                    if r is not None:
                        got = got[:, r]
                    ma, mr = compare(got, ref, *tol)
                    results.append((k, step, which, ma, mr))
        h.append_chunk(K.to(dev), V.to(dev))
        hist_K.append(K.cpu())
        hist_V.append(V.cpu())
        if keep_last is not None:
            for c in range(1, max(1, len(hist_K) - keep_last)):
                hist_K[c] = None
                hist_V[c] = None
    torch.cuda.synchronize()
    assert h.status() == 0, f"device status {h.status():#x}"
    return results


def _bits(t):
    """The raw bits of a bf16 (int16 view) or e4m3 (uint8 view) tensor."""
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.uint8)


def poison_cache(h):
    """Fill the handle's K/V cache with NaN (bf16 or e4m3)."""
    for t in h.cache_views():
        if t.element_size() == 2:
            t.fill_(float("nan"))
        else:
            t.view(torch.uint8).fill_(0x7F)   # e4m3 NaN


def check_cache_against_ring(h, ring, chunks):
    """Every slot of the handle's cache holds, bit for bit, the chunk the oracle's ring model
    puts there (the tensors appended, bf16 or e4m3); slots the model leaves empty still hold the
    NaN poison."""
    kc, vc = h.cache_views()
    held = ring.slot_chunks()
    assert len(held) == kc.shape[2]
    for s, c in enumerate(held):
        gk, gv = kc[:, :, s].cpu(), vc[:, :, s].cpu()          # [B, H, T, d]
        if c < 0:
            assert torch.isnan(gk.float()).all() and torch.isnan(gv.float()).all(), f"slot {s} written"
        else:
            ek, ev = chunks[c]
            assert torch.equal(_bits(gk), _bits(ek.permute(0, 2, 1, 3).contiguous())), s
            assert torch.equal(_bits(gv), _bits(ev.permute(0, 2, 1, 3).contiguous())), s


def stream_and_check_commit(wl, dev, *, chunks, schedule="auto", check_at=None, n_rows=None,
                            check_cache=True, append_at=(), keep_last=None, gen_on_device=False,
                            out_dtype=torch.float32, seed=0, tol=None, fp8=None):
    """Stream through a handle created with commit_in_forward: per chunk, the first step's
    forward, then the last step's forward_commit (its K_cur / V_cur become the chunk's cache
    entry) -- or, at the chunks in `append_at`, a plain forward plus append_chunk.  After every
    chunk the table is compared with the oracle's table for the ring with a spare slot and (with
    check_cache) the cache with the oracle's ring model, bit for bit; at the chunks in
    `check_at` (all if None) both outputs are compared with the oracle.  fp8 = "qk" or "qkv": an
    e4m3 handle (e4m3 Q/K, and V too with "qkv"); the cache is compared with the e4m3 tensors
    committed, the outputs with the oracle on the dequantised inputs (E4M3_P_TOL with "qkv").
    Returns a list of (k, step, max_abs, mean_rel)."""
    pv8 = fp8 == "qkv"
    if tol is None:
        tol = E4M3_P_TOL if pv8 else (MAX_ABS, MEAN_REL)
    if fp8:
        sc = synth.FP8_SCALE
        h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                   out_dtype=out_dtype, max_short_q=-1, schedule=schedule, commit_in_forward=True,
                                   qk_fp8=True, q_scale=sc, k_scale=sc, pv_fp8=pv8, v_scale=sc, device=dev)
    else:
        h = make_handle(wl, dev, out_dtype=out_dtype, max_short_q=-1, schedule=schedule, commit_in_forward=True)
    deq_qk = synth.from_e4m3 if fp8 else (lambda t: t)
    deq_v = synth.from_e4m3 if pv8 else (lambda t: t)
    R = h.R
    if check_cache:
        poison_cache(h)
    gdev = dev if gen_on_device else "cpu"
    if fp8:
        Kc, Vc = synth.cond_inputs_fp8(wl, seed=seed, device=gdev, v8=pv8)
    else:
        Kc, Vc = synth.cond_inputs(wl, seed=seed, device=gdev)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    Kc, Vc = deq_qk(Kc.cpu()), deq_v(Vc.cpu())
    ring = oracle.Ring(B=wl.B, H=wl.H, d=wl.d, T=wl.T, n_cond=0, W=wl.W, sink=wl.sink, Kc=None, Vc=None, R=R) \
        if check_cache else None
    hist_K, hist_V, committed, results = [], [], {}, []
    for k in range(chunks):
        for step in range(wl.steps):
            if fp8:
                Q, K, V = synth.chunk_inputs_fp8(wl, k, step, seed=seed, device=gdev, v8=pv8)
            else:
                Q, K, V = synth.chunk_inputs(wl, k, step, seed=seed, device=gdev)
            last = step == wl.steps - 1
            if last and k not in append_at:
                out = h.forward_commit(Q.to(dev), K.to(dev), V.to(dev))
            else:
                out = h.forward(Q.to(dev), K.to(dev), V.to(dev))
            if check_at is None or k in check_at:
                r = None if n_rows is None else sample_rows(wl.T, n_rows, seed=1000 * k + step)
                ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink,
                                       k=k, Kc=Kc, Vc=Vc, hist_K=hist_K, hist_V=hist_V, Q=deq_qk(Q.cpu()),
                                       K_cur=deq_qk(K.cpu()), V_cur=deq_v(V.cpu()), rows=r)
                got = out.float().cpu().numpy()
                if r is not None:
                    got = got[:, r]
                ma, mr = compare(got, ref, *tol)
                results.append((k, step, ma, mr))
        if k in append_at:
            h.append_chunk(K.to(dev), V.to(dev))
        Kh, Vh = K.cpu(), V.cpu()
        hist_K.append(deq_qk(Kh))
        hist_V.append(deq_v(Vh))
        torch.cuda.synchronize()
        check_table(h.table().cpu().numpy(), k + 1, wl.W, wl.sink, wl.n_cond, wl.T, R=R)
        if check_cache:
            ring.append(deq_qk(Kh), deq_v(Vh))
            committed[k] = (Kh, Vh)
            check_cache_against_ring(h, ring, committed)
        if keep_last is not None:
            for c in range(1, max(1, len(hist_K) - keep_last)):
                hist_K[c] = None
                hist_V[c] = None
    torch.cuda.synchronize()
    assert h.status() == 0, f"device status {h.status():#x}"
    return results


# The error an e4m3 P adds.  The kernel rounds P to the MMA's operand type and divides by the sum
# of the rounded weights, so the output's error from P scales with that type's unit roundoff:
# 2^-8 for bf16 (8 significant bits), 2^-4 for e4m3 (4).  The parity tolerance above is the one
# bf16 P meets; with e4m3 P it is scaled by the ratio of the two, 2^4.
E4M3_P_TOL = (MAX_ABS * 16, MEAN_REL * 16)


def stream_and_check_fp8(wl, dev, *, chunks, check_at=None, n_rows=None, keep_last=None,
                         gen_on_device=False, out_dtype=torch.float32, seed=0, joint=False,
                         tol=None, pv8=False, n_q=None, schedule="auto"):
    """Stream through a handle with e4m3 queries and keys (and, with pv8, e4m3 values: P V on
    kind::f8f6f4): 2 forwards then an append per chunk, every e4m3 tensor with scale FP8_SCALE.
    The oracle computes the same attention on the dequantised values (exact in float32).  With
    joint, the forward also carries e4m3 condition queries; with n_q (<= 128) the forwards take
    the chunk's first n_q queries (the split-K path).  Tolerance: the parity one, or E4M3_P_TOL
    with pv8.  Returns a list of (k, step, which, max_abs, mean_rel)."""
    sc = synth.FP8_SCALE
    if tol is None:
        tol = E4M3_P_TOL if pv8 else (MAX_ABS, MEAN_REL)
    h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                               out_dtype=out_dtype, qk_fp8=True, q_scale=sc, k_scale=sc, pv_fp8=pv8,
                               v_scale=sc, schedule=schedule, device=dev)
    gdev = dev if gen_on_device else "cpu"
    deq_v = (lambda t: synth.from_e4m3(t)) if pv8 else (lambda t: t)
    Kc8, Vc = synth.cond_inputs_fp8(wl, seed=seed, device=gdev, v8=pv8)
    h.set_cond(Kc8.to(dev), Vc.to(dev))
    Kc = synth.from_e4m3(Kc8).cpu()
    Vc = deq_v(Vc).cpu()
    hist_K, hist_V, results = [], [], []
    for k in range(chunks):
        for step in range(wl.steps):
            Q8, K8, V = synth.chunk_inputs_fp8(wl, k, step, seed=seed, n_q=n_q, device=gdev, v8=pv8)
            if joint:
                Qc8 = synth.to_e4m3(synth.cond_queries(wl, k, step, seed=seed, device=gdev))
                out, out_c = h.forward_joint(Q8.to(dev), Qc8.to(dev), K8.to(dev), V.to(dev))
                sets = (("chunk", Q8, out, wl.T), ("cond", Qc8, out_c, wl.n_cond))
            else:
                out = h.forward(Q8.to(dev), K8.to(dev), V.to(dev))
                sets = (("chunk", Q8, out, Q8.shape[1]),)
            if check_at is None or k in check_at:
                for which, q8, o, n in sets:
                    r = None if n_rows is None else sample_rows(n, n_rows, seed=1000 * k + step)
                    ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink,
                                           k=k, Kc=Kc, Vc=Vc, hist_K=hist_K, hist_V=hist_V,
                                           Q=synth.from_e4m3(q8).cpu(), K_cur=synth.from_e4m3(K8).cpu(),
                                           V_cur=deq_v(V).cpu(), rows=r)
                    got = o.float().cpu().numpy()
                    if r is not None:
                        got = got[:, r]
                    ma, mr = compare(got, ref, *tol)
                    results.append((k, step, which, ma, mr))
        h.append_chunk(K8.to(dev), V.to(dev))
        hist_K.append(synth.from_e4m3(K8).cpu())
        hist_V.append(deq_v(V).cpu())
        if keep_last is not None:
            for c in range(1, max(1, len(hist_K) - keep_last)):
                hist_K[c] = None
                hist_V[c] = None
    torch.cuda.synchronize()
    assert h.status() == 0, f"device status {h.status():#x}"
    return results
