"""FP64 CPU oracle for block-causal sink + sliding-window attention (test infrastructure).

Only the tests, the package's smoke check and the benchmark's CPU-baseline and reference legs
may import this package.  The product path (the CUDA library and its binding) never touches it,
and it shares no code with that path.

The arithmetic lives in ``swattn_oracle.c`` (plain C, double precision, OpenMP); this module
only builds it with gcc and marshals numpy arrays.  What it computes follows the JoyAI-Video-Edit
pages: the agifrontier tutorial "JoyAI-Video-Edit：单卡720p 30帧，两步蒸馏攻克流式视频编辑",
section "从双向编辑到分块因果架构的蜕变" (block-causal mask, bounded window, first-chunk sink),
and the neurohive review, section "Чанки и борьба с дрейфом".

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` (brute force on
tiny inputs, closed forms, a library special case, four invariants).  The pages print no
worked numeric example, so nothing is pinned against printed values; the visibility tables
are pinned against a hand enumeration of the pages' rule in ``tests/golden/``.
``tests/test_oracle_mutants.py`` plants plausible mistakes in a private copy of this package and
checks that each one fails a pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libswattn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP) next to its source; return the .so path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    i32, dbl, vp = ctypes.c_int, ctypes.c_double, ctypes.c_void_p
    lib.swo_visible.argtypes = [i32, i32, i32, i32]
    lib.swo_visible.restype = i32
    lib.swo_num_slots.argtypes = [i32, i32]
    lib.swo_num_slots.restype = i32
    lib.swo_slot.argtypes = [i32, i32, i32]
    lib.swo_slot.restype = i32
    lib.swo_table.argtypes = [i32, i32, i32, i32, i32, vp, i32]
    lib.swo_table.restype = i32
    lib.swo_num_slots_r.argtypes = [i32, i32]
    lib.swo_num_slots_r.restype = i32
    lib.swo_slot_r.argtypes = [i32, i32, i32]
    lib.swo_slot_r.restype = i32
    lib.swo_table_r.argtypes = [i32, i32, i32, i32, i32, i32, vp, i32]
    lib.swo_table_r.restype = i32
    lib.swo_vis_row.argtypes = [i32, i32, i32, vp, i32]
    lib.swo_vis_row.restype = i32
    lib.swo_ring_create_r.argtypes = [i32] * 8 + [vp, vp]
    lib.swo_ring_create_r.restype = vp
    lib.swo_attention.argtypes = [i32] * 8 + [vp, vp, vp, vp, vp, i32, vp, vp, dbl, vp, i32, vp]
    lib.swo_attention.restype = i32
    lib.swo_ring_create.argtypes = [i32] * 7 + [vp, vp]
    lib.swo_ring_create.restype = vp
    lib.swo_ring_destroy.argtypes = [vp]
    lib.swo_ring_append.argtypes = [vp, vp, vp]
    lib.swo_ring_slot_chunk.argtypes = [vp, i32]
    lib.swo_ring_slot_chunk.restype = i32
    lib.swo_ring_forward.argtypes = [vp, vp, i32, vp, vp, dbl, vp]
    lib.swo_ring_forward.restype = i32
    lib.swo_num_threads.restype = i32
    lib.swo_set_num_threads.argtypes = [i32]
    lib.swo_set_num_threads.restype = None
    _lib = lib
    return lib


def _f32(a) -> np.ndarray:
    """Accept numpy or a CPU torch tensor (any float dtype); return contiguous float32.

    bf16 values are exact in float32, so nothing is rounded here."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(_load().swo_num_threads())


def set_num_threads(n: int) -> None:
    """OpenMP threads for the oracle's calls made from this thread from now on."""
    _load().swo_set_num_threads(int(n))


def visible(k: int, W: int, sink: bool, j: int) -> bool:
    return bool(_load().swo_visible(k, W, int(sink), j))


def num_slots(W: int, sink: bool, R: int | None = None) -> int:
    """Ring slots; R window slots (default W; W + 1 keeps a spare slot)."""
    return int(_load().swo_num_slots_r(W if R is None else R, int(sink)))


def slot(c: int, W: int, sink: bool, R: int | None = None) -> int:
    return int(_load().swo_slot_r(c, W if R is None else R, int(sink)))


def table(k: int, W: int, sink: bool, n_cond: int, T: int, R: int | None = None) -> np.ndarray:
    """Canonical visibility table: [k, n_segments, N_vis, (kind, chunk_id, slot, n_tokens)...];
    slots of a ring with R window slots (default W)."""
    cap = 3 + 4 * (k + 3)
    out = np.zeros(cap, dtype=np.int32)
    n = _load().swo_table_r(k, W, W if R is None else R, int(sink), n_cond, T, out.ctypes.data, cap)
    if n < 0:
        raise RuntimeError("swo_table: capacity")
    return out[:n].copy()


def vis_row(k: int, W: int, sink: bool) -> np.ndarray:
    """Chunk bitmap row of the visibility table: uint8 [k], entry j = 1 iff history chunk j is
    visible to active chunk k (the current chunk itself is not part of the row)."""
    out = np.zeros(max(k, 1), dtype=np.uint8)
    n = _load().swo_vis_row(k, W, int(sink), out.ctypes.data, out.shape[0])
    if n < 0:
        raise RuntimeError("swo_vis_row: bad arguments")
    return out[:n].copy()


def attention(*, H: int, d: int, T: int, n_cond: int, W: int, sink: bool, k: int,
              Kc, Vc, hist_K, hist_V, Q, K_cur, V_cur, scale: float | None = None,
              rows=None) -> np.ndarray:
    """Dense-mask full-history attention in float64.

    Shapes (user layout): Kc/Vc [B, n_cond, H, d]; hist_K/hist_V lists of k arrays
    [B, T, H, d] (an entry may be None if that chunk is invisible; a None for a visible
    chunk raises); Q [B, n_q, H, d]; K_cur/V_cur [B, T, H, d].  ``rows`` selects query rows.
    Returns [B, n_rows, H, d] float64.
    """
    lib = _load()
    Qf = _f32(Q)
    B, n_q = Qf.shape[0], Qf.shape[1]
    assert Qf.shape[2] == H and Qf.shape[3] == d
    Kcf, Vcf = (_f32(Kc), _f32(Vc)) if n_cond > 0 else (None, None)
    Kcur_f, Vcur_f = _f32(K_cur), _f32(V_cur)
    hk = [(_f32(x) if x is not None else None) for x in hist_K]
    hv = [(_f32(x) if x is not None else None) for x in hist_V]
    assert len(hk) == k and len(hv) == k
    PArr = ctypes.c_void_p * max(k, 1)
    kp = PArr(*([_ptr(x) for x in hk] or [None]))
    vp = PArr(*([_ptr(x) for x in hv] or [None]))
    if rows is None:
        r_arr, n_rows = None, n_q
    else:
        r_arr = np.ascontiguousarray(rows, dtype=np.int32)
        n_rows = int(r_arr.shape[0])
        assert r_arr.min() >= 0 and r_arr.max() < n_q
    out = np.empty((B, n_rows, H, d), dtype=np.float64)
    s = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    rc = lib.swo_attention(B, H, d, T, n_cond, W, int(sink), k, _ptr(Kcf), _ptr(Vcf),
                           ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p),
                           _ptr(Qf), n_q, _ptr(Kcur_f), _ptr(Vcur_f), s,
                           _ptr(r_arr), n_rows, out.ctypes.data)
    if rc == -2:
        raise ValueError("oracle: a visible history chunk was passed as None")
    if rc != 0:
        raise RuntimeError(f"oracle: swo_attention failed ({rc})")
    return out


class Ring:
    """The ring-buffer statement of the same attention (bounded cache with pinned sink)."""

    def __init__(self, *, B: int, H: int, d: int, T: int, n_cond: int, W: int, sink: bool, Kc, Vc,
                 R: int | None = None):
        assert d <= 512
        self._lib = _load()
        self.B, self.H, self.d, self.T = B, H, d, T
        R = W if R is None else R
        self._Kc, self._Vc = (_f32(Kc), _f32(Vc)) if n_cond > 0 else (None, None)
        self._h = self._lib.swo_ring_create_r(B, H, d, T, n_cond, W, R, int(sink),
                                              _ptr(self._Kc), _ptr(self._Vc))
        if not self._h:
            raise MemoryError("swo_ring_create")
        self.S = num_slots(W, sink, R)

    def append(self, K, V) -> None:
        Kf, Vf = _f32(K), _f32(V)
        self._lib.swo_ring_append(self._h, _ptr(Kf), _ptr(Vf))

    def slot_chunks(self) -> list[int]:
        return [int(self._lib.swo_ring_slot_chunk(self._h, s)) for s in range(self.S)]

    def forward(self, Q, K_cur, V_cur, scale: float | None = None) -> np.ndarray:
        Qf, Kf, Vf = _f32(Q), _f32(K_cur), _f32(V_cur)
        B, n_q = Qf.shape[0], Qf.shape[1]
        out = np.empty((B, n_q, self.H, self.d), dtype=np.float64)
        s = (1.0 / np.sqrt(self.d)) if scale is None else float(scale)
        self._lib.swo_ring_forward(self._h, _ptr(Qf), n_q, _ptr(Kf), _ptr(Vf), s, out.ctypes.data)
        return out

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.swo_ring_destroy(h)
            self._h = None
