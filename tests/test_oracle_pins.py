"""Pins for the FP64 oracle, against things other than the oracle itself (CPU only).

* hand enumeration of the pages' visibility rule (tests/golden/);
* a pure-Python brute force (its own cache simulation with a deque, math.fsum sums);
* a closed form: Q = 0 gives uniform weights, so with one-hot group values the output is
  n_tokens(group) / N_vis exactly;
* a library special case: when every chunk is visible, the result is plain softmax attention
  (torch scaled_dot_product_attention in float64) over the concatenated keys;
* four invariants: invisible keys have zero influence, the sink is always visible, permuting
  keys inside the visible set changes nothing, and streaming through the ring buffer equals
  recomputation from the full history.
The visibility rule is from the agifrontier tutorial (section "从双向编辑到分块因果架构的蜕变")
and the neurohive review (section "Чанки и борьба с дрейфом").
"""
from __future__ import annotations

import collections
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).float().numpy()


# ------------------------------------------------------------------ brute force (independent)

def brute_visible(k, W, sink):
    """Visible history of chunk k by simulating the cache: a deque of the W most recent
    commits plus a pinned first chunk."""
    window = collections.deque()
    pinned = set()
    for c in range(k):
        window.append(c)
        if len(window) > W:
            window.popleft()
        if sink and c == 0:
            pinned.add(0)
    return sorted(set(window) | pinned)


def brute_slots(n_commits, W, sink):
    """Physical slot of each committed chunk: the sink keeps slot 0; a new window chunk takes
    the lowest slot whose chunk has left the window (or an empty one)."""
    S = W + (1 if sink else 0)
    holder = [None] * S
    window = collections.deque()
    where = {}
    for c in range(n_commits):
        window.append(c)
        if len(window) > W:
            window.popleft()
        if sink and c == 0:
            holder[0] = 0
            where[c] = 0
            continue
        if W == 0:
            where[c] = -1
            continue
        base = 1 if sink else 0
        for s in range(base, S):
            if holder[s] is None or holder[s] not in window:
                holder[s] = c
                where[c] = s
                break
    return where


def brute_slots_spare(n_commits, W, sink):
    """Physical slots of a ring that keeps one spare window slot (W + 1 in all, none for
    W = 0), written while the chunk's own forward still reads its history: chunk c takes the
    lowest window slot whose chunk is not visible to chunk c, or an empty one."""
    R = W + 1 if W > 0 else 0
    base = 1 if sink else 0
    holder = [None] * (base + R)
    where = {}
    for c in range(n_commits):
        if sink and c == 0:
            holder[0] = 0
            where[c] = 0
            continue
        if R == 0:
            where[c] = -1
            continue
        vis = set(brute_visible(c, W, sink))
        for s_ in range(base, base + R):
            if holder[s_] is None or holder[s_] not in vis:
                holder[s_] = c
                where[c] = s_
                break
    return where


def brute_attention(Kc, Vc, hist_K, hist_V, Q, Kcur, Vcur, W, sink, scale):
    B, n_q, H, d = Q.shape
    k = len(hist_K)
    vis = brute_visible(k, W, sink)
    out = np.zeros((B, n_q, H, d))
    for b in range(B):
        for h in range(H):
            keys, vals = [], []
            for j in range(Kc.shape[1] if Kc is not None else 0):
                keys.append(Kc[b, j, h]); vals.append(Vc[b, j, h])
            for c in vis:
                for t in range(hist_K[c].shape[1]):
                    keys.append(hist_K[c][b, t, h]); vals.append(hist_V[c][b, t, h])
            for t in range(Kcur.shape[1]):
                keys.append(Kcur[b, t, h]); vals.append(Vcur[b, t, h])
            for i in range(n_q):
                q = Q[b, i, h]
                s = [scale * math.fsum(float(q[c]) * float(kk[c]) for c in range(d)) for kk in keys]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                den = math.fsum(w)
                for c in range(d):
                    out[b, i, h, c] = math.fsum(w[j] * float(vals[j][c]) for j in range(len(w))) / den
    return out


def _stream(B, H, d, T, n_cond, n_chunks, seed, n_q=None):
    Kc = _rand((B, n_cond, H, d), seed + 1) if n_cond else None
    Vc = _rand((B, n_cond, H, d), seed + 2) if n_cond else None
    ks = [_rand((B, T, H, d), seed + 10 + 3 * c) for c in range(n_chunks)]
    vs = [_rand((B, T, H, d), seed + 11 + 3 * c) for c in range(n_chunks)]
    qs = [_rand((B, n_q or T, H, d), seed + 12 + 3 * c) for c in range(n_chunks)]
    return Kc, Vc, ks, vs, qs


# ------------------------------------------------------------------ golden: the pages' rule

def _golden_rules():
    rows = []
    with open(os.path.join(GOLDEN, "visibility_rule.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, vis, slots = [p.strip() for p in line.split("|")]
            W, sink, k = (int(x) for x in head.split())
            vis = [] if vis == "-" else [int(x) for x in vis.split()]
            slots = [] if slots == "-" else [int(x) for x in slots.split()]
            rows.append((W, bool(sink), k, vis, slots))
    return rows


@pytest.mark.parametrize("W,sink,k,vis,slots", _golden_rules())
def test_golden_visibility_rule(oracle_mod, W, sink, k, vis, slots):
    got = [j for j in range(k) if oracle_mod.visible(k, W, sink, j)]
    assert got == vis
    assert [oracle_mod.slot(j, W, sink) for j in vis] == slots
    # and the canonical table carries the same chunks and slots
    tab = oracle_mod.table(k, W, sink, n_cond=5, T=7)
    segs = tab[3:].reshape(-1, 4)
    cache = segs[segs[:, 0] == 1]
    assert list(cache[:, 1]) == vis and list(cache[:, 2]) == slots
    # and the chunk bitmap row marks exactly those chunks
    row = oracle_mod.vis_row(k, W, sink)
    assert row.shape == (k,) and list(np.flatnonzero(row)) == vis


def test_golden_visible_keys(oracle_mod):
    with open(os.path.join(GOLDEN, "visible_keys.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, T, n_cond, W, k, nvis = line.split()
            tab = oracle_mod.table(int(k), int(W), True, int(n_cond), int(T))
            assert tab[2] == int(nvis), line
            assert tab[3:].reshape(-1, 4)[:, 3].sum() == int(nvis)


# ------------------------------------------------------------------ tables vs brute force

@pytest.mark.parametrize("sink", [True, False])
@pytest.mark.parametrize("W", [0, 1, 2, 3, 5, 6])
def test_tables_brute_force(oracle_mod, W, sink):
    where = brute_slots(40, W, sink)
    for k in range(40):
        vis = brute_visible(k, W, sink)
        assert [j for j in range(k) if oracle_mod.visible(k, W, sink, j)] == vis
        # causal across chunks: neither the active chunk itself nor a later one is history
        assert not any(oracle_mod.visible(k, W, sink, j) for j in (k, k + 1, k + W + 2, -1))
        tab = oracle_mod.table(k, W, sink, n_cond=3, T=11)
        segs = tab[3:].reshape(-1, 4)
        assert tab[0] == k and tab[1] == len(segs)
        kinds = list(segs[:, 0])
        assert kinds == [0] + [1] * len(vis) + [2]          # canonical order
        assert list(segs[1:-1, 1]) == vis                   # ascending chunk ids, sink first
        assert list(segs[1:-1, 2]) == [where[j] for j in vis]
        assert tuple(segs[-1]) == (2, k, -1, 11)
        assert tab[2] == 3 + 11 * (len(vis) + 1)
        # the chunk bitmap row: vis[k][j] = [j in Hist(k)] for every j < k, 0/1 only
        row = oracle_mod.vis_row(k, W, sink)
        assert row.shape == (k,) and set(np.unique(row)) <= {0, 1}
        assert list(np.flatnonzero(row)) == vis
        # |Hist(k)| = min(k, W+1) with the sink, min(k, W) without
        assert len(vis) == (min(k, W + 1) if sink else min(k, W))
        if sink and k >= 1:
            assert vis[0] == 0                              # the sink is always visible
        # every slot index is in range and no two visible chunks share a slot
        sl = [where[j] for j in vis]
        assert all(0 <= s < oracle_mod.num_slots(W, sink) for s in sl)
        assert len(set(sl)) == len(sl)


@pytest.mark.parametrize("sink", [True, False])
@pytest.mark.parametrize("W", [0, 1, 2, 3, 5, 6])
def test_tables_spare_slot(oracle_mod, W, sink):
    """A ring with one spare window slot: the same visible chunks, other slots.  The slot
    chunk k is committed into is never one that chunk k's own forward reads."""
    R = W + 1 if W > 0 else 0
    where = brute_slots_spare(40, W, sink)
    for k in range(40):
        vis = brute_visible(k, W, sink)
        plain = oracle_mod.table(k, W, sink, n_cond=3, T=11)
        tab = oracle_mod.table(k, W, sink, n_cond=3, T=11, R=R)
        segs, psegs = tab[3:].reshape(-1, 4), plain[3:].reshape(-1, 4)
        assert tab[:3].tolist() == plain[:3].tolist()
        assert segs[:, [0, 1, 3]].tolist() == psegs[:, [0, 1, 3]].tolist()   # only slots differ
        assert list(segs[1:-1, 2]) == [where[j] for j in vis]
        sl = [where[j] for j in vis]
        assert all(0 <= x < oracle_mod.num_slots(W, sink, R) for x in sl) and len(set(sl)) == len(sl)
        own = oracle_mod.slot(k, W, sink, R)
        assert own == where[k]
        assert own not in sl or own < 0                                     # never read while written


def test_ring_holds_exactly_hist(oracle_mod):
    """The occupied slots after committing chunks 0..k-1 hold exactly Hist(k)."""
    B, H, d, T = 1, 1, 4, 2
    for W in (0, 1, 2, 4):
        for sink in (True, False):
            ring = oracle_mod.Ring(B=B, H=H, d=d, T=T, n_cond=0, W=W, sink=sink, Kc=None, Vc=None)
            for k in range(12):
                held = sorted(c for c in ring.slot_chunks() if c >= 0)
                assert held == brute_visible(k, W, sink), (W, sink, k)
                z = np.zeros((B, T, H, d), np.float32)
                ring.append(z, z)


# ------------------------------------------------------------------ attention vs brute force

@pytest.mark.parametrize("T,W,sink,n_cond", [
    (1, 0, True, 8), (3, 1, True, 0), (3, 2, False, 8), (16, 1, True, 8), (3, 5, True, 8),
    (3, 0, False, 8), (2, 2, True, 3)])
def test_attention_brute_force(oracle_mod, T, W, sink, n_cond):
    B, H, d, nch = 2, 2, 8, 7
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, nch, seed=100 + T + 7 * W)
    for k in range(nch):
        ref = brute_attention(Kc, Vc, ks[:k], vs[:k], qs[k], ks[k], vs[k], W, sink, d ** -0.5)
        got = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, k=k, Kc=Kc, Vc=Vc,
                                   hist_K=ks[:k], hist_V=vs[:k], Q=qs[k], K_cur=ks[k], V_cur=vs[k])
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_attention_short_queries_and_rows(oracle_mod):
    """n_q < T queries, and the row-subset mode, against the brute force."""
    B, H, d, T, n_cond, W = 1, 3, 8, 6, 4, 2
    Kc, Vc, ks, vs, _ = _stream(B, H, d, T, n_cond, 5, seed=7)
    Q = _rand((B, 3, H, d), 99)
    k = 4
    ref = brute_attention(Kc, Vc, ks[:k], vs[:k], Q, ks[k], vs[k], W, True, d ** -0.5)
    got = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=True, k=k, Kc=Kc, Vc=Vc,
                               hist_K=ks[:k], hist_V=vs[:k], Q=Q, K_cur=ks[k], V_cur=vs[k])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    sub = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=True, k=k, Kc=Kc, Vc=Vc,
                               hist_K=ks[:k], hist_V=vs[:k], Q=Q, K_cur=ks[k], V_cur=vs[k],
                               rows=[2, 0])
    np.testing.assert_array_equal(sub[:, 0], got[:, 2])
    np.testing.assert_array_equal(sub[:, 1], got[:, 0])


# ------------------------------------------------------------------ closed form

@pytest.mark.parametrize("W,sink", [(0, True), (1, True), (3, True), (2, False), (0, False)])
def test_closed_form_uniform(oracle_mod, W, sink):
    """Q = 0 => uniform weights over the visible keys.  V = one-hot of each key's group
    (0 = condition, 1 + c = history chunk c, 1 + k = current chunk) => out[g] is exactly
    n_tokens(g) / N_vis for visible groups and 0 for invisible ones."""
    B, H, T, n_cond, nch = 1, 2, 5, 3, 9
    d = nch + 2
    for k in range(nch):
        Kc = _rand((B, n_cond, H, d), 1)
        Vc = np.zeros((B, n_cond, H, d), np.float32); Vc[..., 0] = 1
        hk = [_rand((B, T, H, d), 10 + c) for c in range(k)]
        hv = []
        for c in range(k):
            v = np.zeros((B, T, H, d), np.float32); v[..., 1 + c] = 1; hv.append(v)
        Kcur = _rand((B, T, H, d), 50)
        Vcur = np.zeros((B, T, H, d), np.float32); Vcur[..., 1 + k] = 1
        Q = np.zeros((B, T, H, d), np.float32)
        out = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, k=k, Kc=Kc, Vc=Vc,
                                   hist_K=hk, hist_V=hv, Q=Q, K_cur=Kcur, V_cur=Vcur)
        # expected: counts over the visible set of the independent cache simulation
        vis = brute_visible(k, W, sink)
        nvis = n_cond + T * (len(vis) + 1)
        exp = np.zeros(d)
        exp[0] = n_cond / nvis
        for c in vis:
            exp[1 + c] = T / nvis
        exp[1 + k] = T / nvis
        np.testing.assert_allclose(out, np.broadcast_to(exp, out.shape), rtol=0, atol=1e-15)
        if sink and k >= 1:
            assert out[0, 0, 0, 1] == pytest.approx(T / nvis, abs=1e-15)   # sink share


# ------------------------------------------------------------------ library special case

@pytest.mark.parametrize("B,H,d,T,n_cond,k", [(2, 3, 32, 20, 8, 3), (1, 2, 64, 9, 0, 2)])
def test_all_visible_equals_sdpa(oracle_mod, B, H, d, T, n_cond, k):
    """Sink on and W >= k: every committed chunk is visible, so the result is unmasked softmax
    attention over [cond; chunk 0; ...; chunk k-1; current] (torch SDPA, float64)."""
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, k + 1, seed=321)
    got = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=k, sink=True, k=k, Kc=Kc, Vc=Vc,
                               hist_K=ks[:k], hist_V=vs[:k], Q=qs[k], K_cur=ks[k], V_cur=vs[k])
    parts_k = ([Kc] if n_cond else []) + ks[: k + 1]
    parts_v = ([Vc] if n_cond else []) + vs[: k + 1]
    Kall = torch.from_numpy(np.concatenate(parts_k, axis=1)).double().permute(0, 2, 1, 3)
    Vall = torch.from_numpy(np.concatenate(parts_v, axis=1)).double().permute(0, 2, 1, 3)
    Qt = torch.from_numpy(qs[k]).double().permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(Qt, Kall, Vall).permute(0, 2, 1, 3)
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_no_history_equals_sdpa(oracle_mod):
    """W = 0, sink off: attention over condition + current chunk only, for every k."""
    B, H, d, T, n_cond = 1, 2, 16, 12, 6
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, 4, seed=5)
    k = 3
    got = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=0, sink=False, k=k, Kc=Kc, Vc=Vc,
                               hist_K=ks[:k], hist_V=vs[:k], Q=qs[k], K_cur=ks[k], V_cur=vs[k])
    Kall = torch.from_numpy(np.concatenate([Kc, ks[k]], 1)).double().permute(0, 2, 1, 3)
    Vall = torch.from_numpy(np.concatenate([Vc, vs[k]], 1)).double().permute(0, 2, 1, 3)
    Qt = torch.from_numpy(qs[k]).double().permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(Qt, Kall, Vall).permute(0, 2, 1, 3)
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ invariants

@pytest.mark.parametrize("W,sink", [(1, True), (2, False), (3, True)])
def test_invisible_keys_have_zero_influence(oracle_mod, W, sink):
    """Overwrite every invisible chunk with NaN / +-1e30: output bit-identical; passing None
    for an invisible chunk is accepted, for a visible one it is an error."""
    B, H, d, T, n_cond, k = 1, 2, 16, 6, 4, 7
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, k + 1, seed=11)
    kw = dict(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, k=k, Kc=Kc, Vc=Vc,
              Q=qs[k], K_cur=ks[k], V_cur=vs[k])
    base = oracle_mod.attention(hist_K=ks[:k], hist_V=vs[:k], **kw)
    vis = brute_visible(k, W, sink)
    pk, pv, nk, nv = list(ks[:k]), list(vs[:k]), list(ks[:k]), list(vs[:k])
    for c in range(k):
        if c not in vis:
            pk[c] = np.full_like(ks[c], np.nan)
            pv[c] = np.where(np.arange(d) % 2 == 0, 1e30, -1e30).astype(np.float32) * np.ones_like(vs[c])
            nk[c] = None
            nv[c] = None
    np.testing.assert_array_equal(oracle_mod.attention(hist_K=pk, hist_V=pv, **kw), base)
    np.testing.assert_array_equal(oracle_mod.attention(hist_K=nk, hist_V=nv, **kw), base)
    bad_k = list(ks[:k]); bad_k[vis[-1]] = None
    with pytest.raises(ValueError):
        oracle_mod.attention(hist_K=bad_k, hist_V=vs[:k], **kw)


def test_visible_keys_do_have_influence(oracle_mod):
    """Guard for the test above: perturbing a VISIBLE chunk (the sink) changes the output."""
    B, H, d, T, n_cond, k, W = 1, 2, 16, 6, 4, 7, 2
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, k + 1, seed=12)
    kw = dict(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=True, k=k, Kc=Kc, Vc=Vc,
              Q=qs[k], K_cur=ks[k], V_cur=vs[k])
    base = oracle_mod.attention(hist_K=ks[:k], hist_V=vs[:k], **kw)
    pv = list(vs[:k]); pv[0] = pv[0] + 1.0
    assert np.abs(oracle_mod.attention(hist_K=ks[:k], hist_V=pv, **kw) - base).max() > 1e-3


def test_permutation_invariance(oracle_mod):
    """Permuting keys (with their values) inside the visible set leaves the output unchanged:
    rows of the current chunk, rows of the condition block, and whole visible chunks swapped."""
    B, H, d, T, n_cond, k, W = 2, 2, 16, 9, 5, 6, 2
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, k + 1, seed=13)
    kw = dict(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=True, k=k, Q=qs[k])
    base = oracle_mod.attention(Kc=Kc, Vc=Vc, hist_K=ks[:k], hist_V=vs[:k], K_cur=ks[k], V_cur=vs[k], **kw)
    rng = np.random.default_rng(0)
    p = rng.permutation(T)
    pc = rng.permutation(n_cond)
    hk, hv = list(ks[:k]), list(vs[:k])
    vis = brute_visible(k, W, True)          # [0, 4, 5]
    hk[vis[0]], hk[vis[-1]] = ks[vis[-1]], ks[vis[0]]
    hv[vis[0]], hv[vis[-1]] = vs[vis[-1]], vs[vis[0]]
    hk[vis[1]] = ks[vis[1]][:, p]; hv[vis[1]] = vs[vis[1]][:, p]
    got = oracle_mod.attention(Kc=Kc[:, pc], Vc=Vc[:, pc], hist_K=hk, hist_V=hv,
                               K_cur=ks[k][:, p], V_cur=vs[k][:, p], **kw)
    np.testing.assert_allclose(got, base, rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,H,d,T,n_cond,W,sink,n_chunks", [
    (1, 2, 64, 16, 8, 1, True, 4),      # the tiny workload's shapes
    (2, 2, 8, 5, 3, 2, False, 12),
    (1, 2, 32, 70, 16, 2, True, 16),    # 480p-like, scaled down
    (1, 1, 16, 64, 8, 3, True, 225),    # long horizon, reduced T
    (1, 2, 8, 4, 0, 0, True, 6),
])
def test_streaming_equals_recompute(oracle_mod, B, H, d, T, n_cond, W, sink, n_chunks):
    """Ring buffer (S slots, evicting) vs dense mask over the full history, every chunk and
    both denoise steps."""
    Kc, Vc, _, _, _ = _stream(B, H, d, T, n_cond, 0, seed=17)
    ring = oracle_mod.Ring(B=B, H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, Kc=Kc, Vc=Vc)
    hk, hv = [], []
    for k in range(n_chunks):
        for step in range(2):
            s = 1000 * k + 10 * step
            Q, Kn, Vn = _rand((B, T, H, d), s + 1), _rand((B, T, H, d), s + 2), _rand((B, T, H, d), s + 3)
            a = ring.forward(Q, Kn, Vn)
            keep = set(brute_visible(k, W, sink))
            b = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, k=k, Kc=Kc, Vc=Vc,
                                     hist_K=[x if c in keep else None for c, x in enumerate(hk)],
                                     hist_V=[x if c in keep else None for c, x in enumerate(hv)],
                                     Q=Q, K_cur=Kn, V_cur=Vn)
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
        ring.append(Kn, Vn)
        hk.append(Kn); hv.append(Vn)


@pytest.mark.parametrize("W,sink", [(1, True), (2, False), (3, True), (0, True)])
def test_spare_slot_ring_streaming_equals_recompute(oracle_mod, W, sink):
    """The ring with a spare window slot holds one chunk that has left the window; its forward
    skips it and equals the dense mask over the full history, every chunk."""
    B, H, d, T, n_cond, n_chunks = 1, 2, 8, 5, 3, 10
    R = W + 1 if W > 0 else 0
    Kc, Vc, _, _, _ = _stream(B, H, d, T, n_cond, 0, seed=23)
    ring = oracle_mod.Ring(B=B, H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, Kc=Kc, Vc=Vc, R=R)
    hk, hv = [], []
    for k in range(n_chunks):
        held = sorted(c for c in ring.slot_chunks() if c >= 0)
        vis = brute_visible(k, W, sink)
        assert set(vis) <= set(held) and len(held) <= len(vis) + 1
        Q, Kn, Vn = _rand((B, T, H, d), 7 * k + 1), _rand((B, T, H, d), 7 * k + 2), _rand((B, T, H, d), 7 * k + 3)
        a = ring.forward(Q, Kn, Vn)
        b = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=sink, k=k, Kc=Kc, Vc=Vc,
                                 hist_K=hk, hist_V=hv, Q=Q, K_cur=Kn, V_cur=Vn)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
        ring.append(Kn, Vn)
        hk.append(Kn); hv.append(Vn)


def test_stress_outliers_stay_finite(oracle_mod):
    """Keys with sigma 4 outliers: the oracle stays finite and matches the brute force."""
    B, H, d, T, n_cond, W, k = 1, 2, 16, 8, 4, 2, 4
    Kc, Vc, ks, vs, qs = _stream(B, H, d, T, n_cond, k + 1, seed=23)
    ks = [x * np.where(np.random.default_rng(c).random(x.shape[:-1]) < 0.2, 4.0, 1.0)[..., None]
          .astype(np.float32) for c, x in enumerate(ks)]
    ref = brute_attention(Kc, Vc, ks[:k], vs[:k], qs[k], ks[k], vs[k], W, True, d ** -0.5)
    got = oracle_mod.attention(H=H, d=d, T=T, n_cond=n_cond, W=W, sink=True, k=k, Kc=Kc, Vc=Vc,
                               hist_K=ks[:k], hist_V=vs[:k], Q=qs[k], K_cur=ks[k], V_cur=vs[k])
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
