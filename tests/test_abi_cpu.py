"""The C-ABI library on a machine without a GPU: it loads, exports every declared symbol, and
its host-only calls (create, workspace sizing, argument checks) behave as documented."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def native():
    from block_causal_attention_sliding_b200 import build as B
    B.build()
    from block_causal_attention_sliding_b200 import _native
    return _native


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "swattn.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"SW_API\s+[\w\s\*]*?\b(sw_attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for name in ("sw_attn_create", "sw_attn_append_chunk", "sw_attn_forward"):
        assert name in syms


def test_library_exports_every_declared_symbol(native):
    L = native.lib()
    syms = _declared_symbols()
    assert sorted(native.EXPORTS) == syms
    for name in syms:
        assert hasattr(L, name), name


def _create(native, **kw):
    cfg = dict(B=1, H=24, d=128, tokens_per_chunk=3180, W=3, n_cond=256, sink=1, out_dtype=0,
               scale=0.0, max_short_q=0, schedule=0)
    cfg.update(kw)
    c = native.SwAttnConfig(**cfg)
    h = ctypes.c_void_p()
    rc = native.lib().sw_attn_create_ex(ctypes.byref(c), ctypes.byref(h))
    return rc, h


def test_create_and_workspace_bytes(native):
    L = native.lib()
    rc, h = _create(native)
    assert rc == 0 and h.value
    ws = L.sw_attn_workspace_bytes(h)
    # ring K+V: 2 * 24 heads * 4 slots * 3180 * 128 * 2 B; cond K+V: 2 * 24 * 256 * 128 * 2 B
    ring = 2 * 24 * 4 * 3180 * 128 * 2
    cond = 2 * 24 * 256 * 128 * 2
    # plus split-K partials and the persistent schedule's merge scratch (tens of MB)
    assert ring + cond <= ws <= ring + cond + 64 * 2 ** 20
    assert L.sw_attn_table_ints(h) == 3 + 4 * (3 + 3) + 3
    ko, vo = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.sw_attn_cache_offsets(h, ctypes.byref(ko), ctypes.byref(vo)) == 0
    assert ko.value % 1024 == 0 and vo.value - ko.value >= ring // 2
    L.sw_attn_destroy(h)
    # the simple constructor: B = 1, sink on
    h2 = ctypes.c_void_p()
    assert L.sw_attn_create(24, 128, 3180, 3, 256, ctypes.byref(h2)) == 0
    assert L.sw_attn_workspace_bytes(h2) == ws
    L.sw_attn_destroy(h2)


def test_workspace_constant_in_stream_length(native):
    """Cache memory depends on W, not on how many chunks will be streamed."""
    L = native.lib()
    sizes = []
    for W in (1, 3, 6):
        rc, h = _create(native, W=W)
        assert rc == 0
        sizes.append(L.sw_attn_workspace_bytes(h))
        L.sw_attn_destroy(h)
    assert sizes[0] < sizes[1] < sizes[2]


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), -2), (dict(d=0), -2), (dict(H=0), -2), (dict(B=0), -2),
    (dict(tokens_per_chunk=0), -2), (dict(W=-1), -2), (dict(W=65), -2), (dict(n_cond=-3), -2),
    (dict(sink=2), -1), (dict(out_dtype=7), -1), (dict(max_short_q=129), -2),
    (dict(scale=float("inf")), -1), (dict(schedule=5), -1),
    (dict(schedule=4, d=64), -2),   # the CTA-pair schedule is d = 128 only
    (dict(schedule=1, qk_fp8=1), -2),   # no e4m3 form of the grid schedule
])
def test_create_rejects_bad_config(native, kw, code):
    rc, h = _create(native, **kw)
    assert rc == code
    assert not h.value
    assert native.lib().sw_attn_last_error().decode()


def test_fp8_configs_accepted(native):
    """e4m3 handles are accepted with the committing forward and with the schedules that have an
    e4m3 form (automatic, persistent, three-buffer), e4m3 V only on top of e4m3 Q/K."""
    L = native.lib()
    for kw in (dict(qk_fp8=1), dict(qk_fp8=1, pv_fp8=1), dict(qk_fp8=1, commit_in_forward=1),
               dict(qk_fp8=1, pv_fp8=1, commit_in_forward=1), dict(qk_fp8=1, schedule=native.SW_SCHED_TRI),
               dict(qk_fp8=1, schedule=native.SW_SCHED_AUTO)):
        rc, h = _create(native, **kw)
        assert rc == 0, (kw, L.sw_attn_last_error())
        L.sw_attn_destroy(h)
    for kw in (dict(pv_fp8=1), dict(qk_fp8=1, d=64), dict(qk_fp8=1, schedule=native.SW_SCHED_PAIR)):
        rc, h = _create(native, **kw)
        assert rc == native.SW_ESHAPE, kw
        assert not h.value


def test_calls_before_workspace_fail_cleanly(native):
    L = native.lib()
    rc, h = _create(native, H=2, d=64, tokens_per_chunk=16, W=1, n_cond=8)
    assert rc == 0
    dummy = ctypes.c_void_p(0x1000)
    assert L.sw_attn_forward(h, dummy, dummy, dummy, dummy, 16, None) == native.SW_ESTATE
    assert b"workspace" in L.sw_attn_last_error()
    assert L.sw_attn_append_chunk(h, dummy, dummy, None) == native.SW_ESTATE
    assert L.sw_attn_set_cond(h, dummy, dummy, None) == native.SW_ESTATE
    assert L.sw_attn_reset(h, None) == native.SW_ESTATE
    st = ctypes.c_int32()
    assert L.sw_attn_get_status(h, ctypes.byref(st)) == native.SW_ESTATE
    # bind: null and misaligned pointers and short buffers are refused before any CUDA call
    assert L.sw_attn_bind_workspace(h, None, 1 << 20, None) == native.SW_EINVAL
    assert L.sw_attn_bind_workspace(h, ctypes.c_void_p(0x1008), 1 << 30, None) == native.SW_EALIGN
    assert L.sw_attn_bind_workspace(h, ctypes.c_void_p(0x10000), 16, None) == native.SW_ESHAPE
    L.sw_attn_destroy(h)


def test_null_handle(native):
    L = native.lib()
    assert L.sw_attn_workspace_bytes(None) == 0
    assert L.sw_attn_forward(None, None, None, None, None, 1, None) == native.SW_EINVAL
    L.sw_attn_destroy(None)   # ignored


def test_schedule_resolution(native):
    """Auto picks the two-tile persistent kernel when there are at least as many 128-row Q-tile
    pairs as SMs (148 before a device is bound), the three-buffer kernel otherwise; explicit
    schedules are returned as given.  Host only."""
    L = native.lib()
    cases = [
        (dict(schedule=native.SW_SCHED_AUTO), 3180, native.SW_SCHED_PERSISTENT),        # 24 x 13 = 312 pairs
        (dict(schedule=native.SW_SCHED_AUTO, H=16, tokens_per_chunk=1400), 1400, native.SW_SCHED_TRI),  # 96
        (dict(schedule=native.SW_SCHED_GRID), 3180, native.SW_SCHED_GRID),
        (dict(schedule=native.SW_SCHED_TRI), 3180, native.SW_SCHED_TRI),
        # the CTA-pair kernel needs a device that holds a pair of its CTAs: before a workspace is
        # bound (no device known) it resolves to the three-buffer kernel
        (dict(schedule=native.SW_SCHED_PAIR), 3180, native.SW_SCHED_TRI),
    ]
    for kw, n_q, want in cases:
        rc, h = _create(native, **kw)
        assert rc == 0
        assert L.sw_attn_schedule_for(h, n_q) == want, (kw, n_q)
        L.sw_attn_destroy(h)
    # the boundary: 147 pairs -> tri, 148 pairs -> persistent (H heads x 1 pair with n_q <= 256)
    for H, want in ((147, native.SW_SCHED_TRI), (148, native.SW_SCHED_PERSISTENT)):
        rc, h = _create(native, schedule=native.SW_SCHED_AUTO, H=H, tokens_per_chunk=256, n_cond=0)
        assert rc == 0
        assert L.sw_attn_schedule_for(h, 256) == want
        L.sw_attn_destroy(h)
    rc, h = _create(native, schedule=native.SW_SCHED_AUTO)
    assert L.sw_attn_schedule_for(h, 0) == native.SW_EINVAL
    assert L.sw_attn_schedule_for(None, 10) == native.SW_EINVAL
    L.sw_attn_destroy(h)


def test_fp8_handles_halve_the_cache(native):
    """An e4m3 K (and V) cache takes one byte per element: the K cache of a qk_fp8 handle and the
    K and V caches of a qk_fp8 + pv_fp8 handle are half their bf16 sizes, and nothing else in the
    workspace changes.  Host only."""
    L = native.lib()
    ring_half = 24 * 4 * 3180 * 128          # one of K or V in the ring, bytes at 2 B per element / 2
    cond_half = 24 * 256 * 128

    def layout(**kw):
        rc, h = _create(native, **kw)
        assert rc == 0, L.sw_attn_last_error()
        ko, vo = ctypes.c_size_t(), ctypes.c_size_t()
        assert L.sw_attn_cache_offsets(h, ctypes.byref(ko), ctypes.byref(vo)) == 0
        ws = L.sw_attn_workspace_bytes(h)
        L.sw_attn_destroy(h)
        return ws, ko.value, vo.value

    ws16, ko16, vo16 = layout()
    ws8k, ko8k, vo8k = layout(qk_fp8=1)
    ws8, ko8, vo8 = layout(qk_fp8=1, pv_fp8=1)
    assert ko16 == ko8k == ko8                               # the state header comes first, unchanged
    assert vo16 - ko16 == 2 * ring_half                      # bf16 K cache (already 1 KB aligned)
    assert vo8k - ko8k == ring_half and vo8 - ko8 == ring_half
    # K ring + K cond halve on the qk_fp8 handle; V ring + V cond too with pv_fp8
    assert ws16 - ws8k == ring_half + cond_half
    assert ws16 - ws8 == 2 * (ring_half + cond_half)


def test_commit_in_forward_keeps_one_spare_slot(native):
    """The committing forward writes the chunk into a slot its own forward does not read, so the
    ring has W + 1 window slots (plus the sink): one more slot of K and V.  W = 0 keeps none."""
    L = native.lib()
    slot = 2 * 24 * 3180 * 128 * 2           # one slot of K and V, bf16

    def ws(**kw):
        rc, h = _create(native, **kw)
        assert rc == 0, L.sw_attn_last_error()
        n = L.sw_attn_workspace_bytes(h)
        L.sw_attn_destroy(h)
        return n

    assert ws(commit_in_forward=1) - ws() == slot
    assert ws(commit_in_forward=1, W=0) == ws(W=0)
    assert ws(commit_in_forward=1, qk_fp8=1, pv_fp8=1) - ws(qk_fp8=1, pv_fp8=1) == slot // 2


def test_destroyed_and_unknown_handles_are_refused(native):
    """A destroyed handle, or a pointer that never was a handle, is refused by every call with
    SW_EINVAL (0 from the size queries) before anything is dereferenced; a second destroy and the
    destroy of an unknown pointer are ignored.  Host only."""
    L = native.lib()
    rc, h = _create(native, H=2, d=64, tokens_per_chunk=16, W=1, n_cond=8)
    assert rc == 0 and L.sw_attn_workspace_bytes(h) > 0
    L.sw_attn_destroy(h)
    fake = ctypes.c_void_p(0x7000)           # never dereferenced: the set of live handles says no
    dummy = ctypes.c_void_p(0x1000)
    st = ctypes.c_int32()
    ko, vo = ctypes.c_size_t(), ctypes.c_size_t()
    for bad in (h, fake):
        assert L.sw_attn_workspace_bytes(bad) == 0
        assert L.sw_attn_table_ints(bad) == 0
        calls = [
            L.sw_attn_bind_workspace(bad, ctypes.c_void_p(0x10000), 1 << 30, None),
            L.sw_attn_set_cond(bad, dummy, dummy, None),
            L.sw_attn_append_chunk(bad, dummy, dummy, None),
            L.sw_attn_forward(bad, dummy, dummy, dummy, dummy, 16, None),
            L.sw_attn_forward_commit(bad, dummy, dummy, dummy, dummy, None),
            L.sw_attn_forward_joint(bad, dummy, dummy, dummy, dummy, dummy, dummy, None),
            L.sw_attn_forward_short_noalloc(bad, dummy, dummy, dummy, dummy, 16, None),
            L.sw_attn_reset(bad, None),
            L.sw_attn_get_table(bad, dummy, None),
            L.sw_attn_get_status(bad, ctypes.byref(st)),
            L.sw_attn_cache_offsets(bad, ctypes.byref(ko), ctypes.byref(vo)),
            L.sw_attn_schedule_for(bad, 16),
            L.sw_attn_commit_kind(bad),
            L.sw_attn_selftest_timeout(bad, 1000, None),
        ]
        assert calls == [native.SW_EINVAL] * len(calls)
        assert b"unknown or destroyed handle" in L.sw_attn_last_error()
        arr = (ctypes.c_void_p * 1)(bad)
        ptrs = (ctypes.c_void_p * 1)(dummy)
        assert L.sw_attn_append_chunk_batched(arr, 1, ptrs, ptrs, None) == native.SW_EINVAL
        assert b"unknown or destroyed handle 0" in L.sw_attn_last_error()
        L.sw_attn_destroy(bad)                # ignored: destroyed before, or never created
    # another handle created afterwards is unaffected, and is refused once destroyed in turn
    rc, h2 = _create(native, H=2, d=64, tokens_per_chunk=16, W=1, n_cond=8)
    assert rc == 0 and L.sw_attn_workspace_bytes(h2) > 0
    L.sw_attn_destroy(h2)
    assert L.sw_attn_workspace_bytes(h2) == 0


def test_missing_library_fails_loudly(monkeypatch):
    """Without the built library the binding raises at first use: there is no fallback."""
    from block_causal_attention_sliding_b200 import _native as N
    monkeypatch.setattr(N, "_lib", None)
    monkeypatch.setattr(N, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libswattn.so"))
    with pytest.raises(ImportError, match="not built"):
        N.lib()


def test_product_path_never_touches_the_oracle():
    """The package (binding, API, build, inputs) imports, loads and names nothing under oracle/."""
    pkg = os.path.join(ROOT, "block_causal_attention_sliding_b200")
    for dirpath, _, files in os.walk(pkg):
        for name in files:
            if name.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, name), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), name
                assert "swattn_oracle" not in text and "libswattn_oracle" not in text, name


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the behaviour without a GPU")
def test_api_without_a_gpu_raises():
    """On a machine without a GPU the Python API raises when it needs the device: no CPU path."""
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    with pytest.raises((RuntimeError, AssertionError)):
        SlidingWindowAttention(H=2, d=64, T=16, W=1, n_cond=8)


def test_bench_reaches_the_oracle_only_from_its_baseline_legs():
    """bench.py imports the oracle only inside the functions of its CPU-baseline and reference
    legs, never at module level or in the CUDA arm."""
    import ast
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    allowed = {"oracle_inputs", "cpu_baseline", "cpu_stream_ms", "run_reference"}
    found = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found.append(func)
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                found.append(func)
            visit(child, f)

    visit(tree, None)
    assert found and set(found) <= allowed, found
