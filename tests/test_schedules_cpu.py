"""The full-path schedules, enumerated on the host with the kernels' own schedule code
(sw_attn_schedule_pieces).  For the persistent (pairs of Q tiles), three-buffer (Q tiles) and
CTA-pair (pairs of Q tiles over CTA pairs) kernels:
  * every (unit, key tile) is processed exactly once;
  * a unit's pieces lie in consecutive CTAs, in key-tile order;
  * a CTA has at most two split pieces, its first and its last stream-K piece, and the partial
    slots the merging piece reads (two per CTA: 2g for its first stream-K piece, 2g + 1 for the
    other) are exactly the slots the unit's pieces wrote;
  * the live Q tiles of a unit are what its position in the head gives.
Checked on the workloads' shapes, on small shapes cut into many pieces, and on 300 seeded random
shapes per schedule.  Host only: no device memory is touched.
"""
from __future__ import annotations

import numpy as np
import pytest

from block_causal_attention_sliding_b200 import _native as N

# (nqt, nt, B*H, SMs): 720p, 480p, the stress workload, and small shapes whose units are cut into
# many pieces (few items per CTA), odd and even tile counts
SHAPES = [
    (25, 127, 24, 148), (11, 45, 16, 148), (25, 204, 128, 148), (3, 8, 6, 148), (1, 3, 1, 148),
    (2, 5, 3, 7), (7, 11, 5, 13), (13, 40, 2, 148), (5, 9, 7, 148), (4, 2, 1, 148), (9, 1, 3, 148),
    (26, 30, 11, 148), (3, 129, 2, 5),
]
KINDS = [("persistent", N.SW_SCHED_PERSISTENT), ("tri", N.SW_SCHED_TRI), ("pair", N.SW_SCHED_PAIR)]


def load_schedule_lib(path):
    """A library built from other copies of the schedule sources (the mutation check), typed
    like the package's own."""
    import ctypes
    L = ctypes.CDLL(path)
    L.sw_attn_schedule_pieces.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_int]
    L.sw_attn_schedule_pieces.restype = ctypes.c_int
    return L


def pieces(kind, nqt, nt, bh, ctas, lib=None):
    L = lib if lib is not None else N.lib()
    cap = 1 << 20
    out = np.zeros((cap, 6), dtype=np.int32)
    n = L.sw_attn_schedule_pieces(kind, nqt, nt, bh, ctas, out.ctypes.data, cap)
    assert n >= 0, n
    return out[:n]


@pytest.mark.parametrize("name,kind", KINDS)
@pytest.mark.parametrize("nqt,nt,bh,sms", SHAPES)
def test_schedule_covers_and_merges(name, kind, nqt, nt, bh, sms):
    ctas = sms // 2 if kind == N.SW_SCHED_PAIR else sms   # the pair kernel runs one cluster per 2 SMs
    check_schedule(kind, nqt, nt, bh, ctas)


@pytest.mark.parametrize("name,kind", KINDS)
def test_schedule_random_shapes(name, kind):
    """The same checks on 300 seeded random shapes per schedule: small and large tile counts,
    CTA counts from 1 to above the number of units, so every mix of whole rounds, many-way
    splits and idle CTAs comes up."""
    rng = np.random.default_rng(20260 + kind)
    for _ in range(300):
        nqt = int(rng.integers(1, 40))
        nt = int(rng.integers(1, 150))
        bh = int(rng.integers(1, 40))
        ctas = int(rng.integers(1, 200))
        check_schedule(kind, nqt, nt, bh, ctas)


def check_all(lib=None, n_random=100):
    """Every check above on every fixed shape and n_random seeded random shapes per schedule."""
    for _, kind in KINDS:
        for nqt, nt, bh, sms in SHAPES:
            check_schedule(kind, nqt, nt, bh, sms // 2 if kind == N.SW_SCHED_PAIR else sms, lib)
        rng = np.random.default_rng(20260 + kind)
        for _ in range(n_random):
            check_schedule(kind, int(rng.integers(1, 40)), int(rng.integers(1, 150)), int(rng.integers(1, 40)),
                           int(rng.integers(1, 200)), lib)


def check_schedule(kind, nqt, nt, bh, ctas, lib=None):
    per_bh = nqt if kind == N.SW_SCHED_TRI else (nqt + 1) // 2
    rows = pieces(kind, nqt, nt, bh, ctas, lib)
    assert len(rows) > 0

    # every (unit, key tile) exactly once; a unit's pieces in consecutive CTAs, in key-tile order
    by_unit = {}
    for g, u, j0, j1, sk, live in rows:
        assert 0 <= g < ctas and 0 <= u < bh * per_bh and 0 <= j0 < j1 <= nt
        by_unit.setdefault(int(u), []).append((int(j0), int(j1), int(g), int(live)))
        if kind == N.SW_SCHED_TRI:
            assert live == 1
        else:
            assert live == min(2, nqt - 2 * (u % per_bh))
    assert sorted(by_unit) == list(range(bh * per_bh))
    for u, ps in by_unit.items():
        ps.sort()
        assert ps[0][0] == 0 and ps[-1][1] == nt, (u, ps)
        for a, b in zip(ps, ps[1:]):
            assert a[1] == b[0], (u, ps)                      # contiguous, no overlap
            assert b[2] == a[2] + 1, (u, ps)                  # next piece on the next CTA

    # partial slots: the kernel writes slot 2g for a CTA's first stream-K piece and 2g + 1 for any
    # other; the merging piece reads, for CTA gg of the unit's range, 2gg if gg > g_first or if
    # g_first's first stream-K piece belongs to this unit, else 2gg + 1
    sk_list = {}
    for g, u, j0, j1, sk, live in rows:
        if sk:
            sk_list.setdefault(int(g), []).append((int(u), int(j0), int(j1)))
    slot_of = {}
    for g, lst in sk_list.items():
        split = [i for i, (u, j0, j1) in enumerate(lst) if j1 - j0 < nt]
        assert all(i in (0, len(lst) - 1) for i in split), (g, lst)   # only first and last may be split
        for i, (u, j0, j1) in enumerate(lst):
            if j1 - j0 < nt:
                slot_of[(u, g)] = 2 * g if i == 0 else 2 * g + 1
    written = set()
    for u, ps in by_unit.items():
        if len(ps) == 1:
            assert ps[0][0] == 0 and ps[0][1] == nt
            continue
        gs = [g for _, _, g, _ in ps]
        g_first = gs[0]
        opens_first = sk_list[g_first][0][0] == u
        for gg in gs:
            want = 2 * gg if (gg > g_first or opens_first) else 2 * gg + 1
            assert slot_of[(u, gg)] == want, (u, gg, slot_of[(u, gg)], want)
            assert want not in written                       # no two pieces share a slot
            written.add(want)


def test_schedule_hook_rejects_bad_arguments():
    L = N.lib()
    buf = np.zeros((4, 6), dtype=np.int32)
    assert L.sw_attn_schedule_pieces(N.SW_SCHED_GRID, 4, 4, 1, 4, buf.ctypes.data, 4) == N.SW_EINVAL
    assert L.sw_attn_schedule_pieces(N.SW_SCHED_TRI, 0, 4, 1, 4, buf.ctypes.data, 4) == N.SW_EINVAL
    assert L.sw_attn_schedule_pieces(N.SW_SCHED_TRI, 4, 4, 1, 4, None, 4) == N.SW_EINVAL
    assert L.sw_attn_schedule_pieces(N.SW_SCHED_TRI, 40, 40, 4, 4, buf.ctypes.data, 4) == N.SW_ESHAPE
