"""Mutation check of the schedule tests (CPU only; nvcc builds host code without a GPU).

The stream-K schedules that the persistent, three-buffer and CTA-pair kernels run are plain
host/device code (persist_sched.cuh, tri_common.cuh), which sw_attn_schedule_pieces enumerates
on the host.  Each mutant below plants one plausible mistake in a private copy of those sources
(an off-by-one, a dropped correction term, a wrong index), builds the enumeration hook from the
copy into a scratch library, and runs the checks of test_schedules_cpu.py against it in a
subprocess: they must fail on every mutant and pass on an unmutated copy.  The package's own
sources and library are never touched.  Mistakes in the cost positions of the persistent
schedule's stream-K line (its odd-tile correction dropped, for one) are left out: they make the
enumeration loop stop advancing instead of producing wrong pieces, so they hang rather than fail.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_causal_attention_sliding_b200", "csrc")
PERSIST = "persist_sched.cuh"
TRI = "tri_common.cuh"

# (name, file, text, replacement)
MUTANTS = [
    # persistent kernel: whole pairs of Q tiles in rounds, then one stream-K line of (pair, key tile)
    ("persistent: one round too many", PERSIST, "rounds = P / G;", "rounds = (P + G - 1) / G;"),
    ("persistent: stream-K CTA floor dropped", PERSIST,
     "Gsk = Csk > 0 ? (int)min((long long)G, max(1LL, Csk / 2)) : 0;", "Gsk = Csk > 0 ? G : 0;"),
    ("persistent: round-robin stride off by one", PERSIST,
     "const int p = s.g + it.r * s.G;", "const int p = s.g + it.r * (s.G - 1);"),
    ("persistent: stream-K line starts one pair late", PERSIST,
     "p0 = rounds * G;", "p0 = rounds * G + (rounds * G < P ? 1 : 0);"),
    ("persistent: first key tile rounded down", PERSIST,
     "const int j0 = (int)((it.cur - ps + lv - 1) / lv);", "const int j0 = (int)((it.cur - ps) / lv);"),
    ("persistent: live tiles from the head index", PERSIST,
     "return min(2, nqt - 2 * (p % npairs));", "return min(2, nqt - 2 * (p / npairs));"),
    ("persistent: last key tile one past the range", PERSIST,
     "const int j1 = (int)(e < s.nt ? e : s.nt);", "const int j1 = (int)(e + 1 < s.nt ? e + 1 : s.nt);"),
    ("persistent: a CTA's range ends one item early", PERSIST,
     "c1 = cta < Gsk ? (long long)(cta + 1) * Csk / Gsk : 0;",
     "c1 = cta < Gsk ? (long long)(cta + 1) * Csk / Gsk - (cta + 1 < Gsk ? 1 : 0) : 0;"),
    # three-buffer and CTA-pair kernels: units in rounds, then a stream-K line of (unit, key tile)
    ("tri: one round too many", TRI, "rounds = U / G;", "rounds = (U + G - 1) / G;"),
    ("tri: cursor skips an item", TRI, "it.cur += j1 - j0;", "it.cur += j1 - j0 + 1;"),
    ("tri: piece runs one item past the range", TRI,
     "const long long left = s.c1 - it.cur;", "const long long left = s.c1 - it.cur + 1;"),
    ("tri: a CTA's range ends one item early", TRI,
     "c1 = cta < Gsk ? (long long)(cta + 1) * Csk / Gsk : 0;",
     "c1 = cta < Gsk ? (long long)(cta + 1) * Csk / Gsk - (cta + 1 < Gsk ? 1 : 0) : 0;"),
    ("tri: stream-K CTA floor dropped", TRI,
     "Gsk = Csk > 0 ? (int)min((long long)G, max(1LL, Csk / 2)) : 0;", "Gsk = Csk > 0 ? G : 0;"),
    ("tri: first unit of the stream-K line off by one", TRI,
     "const int u = s.u0 + (int)(it.cur / s.nt);", "const int u = s.u0 + (int)(it.cur / s.nt) + (it.cur > 0);"),
]


def _build(tmp: str, mutant) -> str:
    from block_causal_attention_sliding_b200 import build as B
    dst = os.path.join(tmp, "csrc")
    os.makedirs(dst)
    for name in os.listdir(CSRC):
        if name.endswith((".cuh", ".h")) or name == "sched_host.cu":
            shutil.copy(os.path.join(CSRC, name), os.path.join(dst, name))
    if mutant is not None:
        path = os.path.join(dst, mutant[1])
        with open(path, encoding="utf-8") as f:
            text = f.read()
        assert text.count(mutant[2]) == 1, mutant[0]
        with open(path, "w", encoding="utf-8") as f:
            f.write(text.replace(mutant[2], mutant[3]))
    lib = os.path.join(tmp, "libsched.so")
    subprocess.run([B._nvcc(), *B.NVCC_FLAGS, "-I", B.INCLUDE, "-I", dst, "-shared",
                    os.path.join(dst, "sched_host.cu"), "-o", lib],
                   check=True, capture_output=True, timeout=600)
    return lib


def _run_checks(mutant) -> tuple[int, str]:
    with tempfile.TemporaryDirectory(prefix="sched_mutant_") as tmp:
        lib = _build(tmp, mutant)
        code = ("import sys; sys.path[:0] = [%r, %r]; import test_schedules_cpu as t; "
                "t.check_all(t.load_schedule_lib(%r))" % (os.path.join(ROOT, "tests"), ROOT, lib))
        env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
        p = subprocess.run([sys.executable, "-c", code], cwd=tmp, env=env, capture_output=True, text=True,
                           timeout=180)
        return p.returncode, p.stderr[-1500:]


def test_mutation_sites_exist():
    assert len({m[0] for m in MUTANTS}) == len(MUTANTS)
    for name, fname, old, new in MUTANTS:
        with open(os.path.join(CSRC, fname), encoding="utf-8") as f:
            assert f.read().count(old) == 1, name
        assert old != new, name


@pytest.mark.timeout(1800)
def test_every_schedule_mutant_fails_a_check():
    """The unmutated copy passes every schedule check; each mutant fails one of them with a
    failed assertion (never an interpreter crash or a hang)."""
    jobs = [None] + MUTANTS
    with cf.ThreadPoolExecutor(max_workers=max(1, min(6, os.cpu_count() or 1))) as ex:
        results = list(ex.map(_run_checks, jobs))
    rc0, log0 = results[0]
    assert rc0 == 0, "unmutated copy fails the schedule checks:\n" + log0
    survivors = [(m[0], rc, log) for m, (rc, log) in zip(MUTANTS, results[1:])
                 if rc != 1 or "AssertionError" not in log]
    assert not survivors, "\n\n".join(f"{n}: exit {rc}\n{log}" for n, rc, log in survivors)
