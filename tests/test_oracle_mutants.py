"""Mutation check of the oracle's pins (CPU only).

Each mutant below plants one plausible mistake in a private copy of the oracle: a dropped term,
an off-by-one window, a wrong sign or index, a transposed operand.  The pin suite
(test_oracle_pins.py, with its golden files) then runs against that copy in a subprocess and
must fail, so each kind of mistake is caught by at least one pin.  An unmutated copy run the
same way must pass, which shows the harness itself works.

The repository's oracle is never modified: the copies live in a temporary directory, build their
own library there, and are imported ahead of the repository's one.
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
C_SRC = "swattn_oracle.c"
PY_SRC = "__init__.py"

# (name, file, text, replacement, which occurrence of text (0-based))
MUTANTS = [
    # the visibility rule: Hist(k) = the W most recent chunks plus the sink
    ("window one chunk short", C_SRC, "if (j >= k - W) return 1;", "if (j > k - W) return 1;", 0),
    ("window one chunk long", C_SRC, "if (j >= k - W) return 1;", "if (j >= k - W - 1) return 1;", 0),
    ("sink dropped", C_SRC, "if (sink && j == 0) return 1;", "if (sink && j == 1) return 1;", 0),
    ("a chunk sees itself as history", C_SRC, "if (j < 0 || j >= k) return 0;",
     "if (j < 0 || j > k) return 0;", 0),
    # ring slots
    ("sink ring slot off by one", C_SRC, "return 1 + (c - 1) % R;", "return 1 + c % R;", 0),
    ("plain ring slot off by one", C_SRC, "return c % R;", "return (c + 1) % R;", 0),
    ("spare-slot table uses W slots", C_SRC, "swo_slot_r(j, R, sink)", "swo_slot_r(j, W, sink)", 0),
    # the canonical table and the bitmap row
    ("chunk id and slot transposed", C_SRC,
     "out[pos++] = 1; out[pos++] = j; out[pos++] = swo_slot_r(j, R, sink);",
     "out[pos++] = 1; out[pos++] = swo_slot_r(j, R, sink); out[pos++] = j;", 0),
    ("N_vis misses the current chunk", C_SRC,
     "out[pos++] = 2; out[pos++] = k; out[pos++] = -1; out[pos++] = T;\n    nseg++; nvis += T;",
     "out[pos++] = 2; out[pos++] = k; out[pos++] = -1; out[pos++] = T;\n    nseg++;", 0),
    ("bitmap row ignores the sink", C_SRC, "swo_visible(k, W, sink, j);", "swo_visible(k, W, 0, j);", 0),
    # the dense definition
    ("dot product drops a term", C_SRC, "for (int c = 0; c < d; c++) s += ",
     "for (int c = 1; c < d; c++) s += ", 0),
    ("mask taken from the next chunk", C_SRC, "swo_visible(k, W, sink, c);",
     "swo_visible(k, W, sink, c + 1);", 0),
    ("scale dropped on condition keys", C_SRC, "sc[jj] = scale * dot_f(q, kr, d);",
     "sc[jj] = dot_f(q, kr, d);", 0),
    ("exponent sign flipped on history keys", C_SRC, "const double e = exp(sc[jj] - mx);",
     "const double e = exp(mx - sc[jj]);", 1),
    ("condition keys left out of the denominator", C_SRC, "den += e;", "(void)e;", 0),
    ("output not normalised", C_SRC, "o[c] = acc[c] / den;", "o[c] = acc[c];", 0),
    ("K used as V for the current chunk", C_SRC,
     "const float *vr = Vcur + (((long)b * T + t) * H + h) * d;",
     "const float *vr = Kcur + (((long)b * T + t) * H + h) * d;", 0),
    ("row selection ignored", C_SRC, "const int i = rows ? rows[r] : r;", "const int i = r;", 0),
    ("every head reads head 0's query", C_SRC,
     "const float *q = Q + (((long)b * n_q + i) * H + h) * d;",
     "const float *q = Q + (((long)b * n_q + i) * H + 0) * d;", 0),
    ("current keys of batch 0 for every batch", C_SRC,
     "const float *kr = Kcur + (((long)b * T + t) * H + h) * d;",
     "const float *kr = Kcur + (((long)0 * T + t) * H + h) * d;", 0),
    # the ring statement
    ("ring evicts the wrong chunk", C_SRC, "r->slot_chunk[q] == c - r->R)",
     "r->slot_chunk[q] == c - r->R + 1)", 0),
    ("ring reads one chunk past the window", C_SRC, "if (held < r->n_committed - r->W && ",
     "if (held < r->n_committed - r->W - 1 && ", 0),
    ("ring skips the sink", C_SRC,
     "if (held < r->n_committed - r->W && !(r->sink && held == 0)) continue;",
     "if (held < r->n_committed - r->W) continue;", 0),
    ("online softmax does not rescale its sum", C_SRC, "l *= f;", "(void)f;", 0),
    ("ring uses K as the condition values", C_SRC, "Kb = r->Kc; Vb = r->Vc;", "Kb = r->Kc; Vb = r->Kc;", 0),
    # the binding's default softmax scale, 1/sqrt(d)
    ("default scale 1/d", PY_SRC, "s = (1.0 / np.sqrt(d)) if scale is None else float(scale)",
     "s = (1.0 / d) if scale is None else float(scale)", 0),
]


def _replace_nth(text: str, old: str, new: str, n: int) -> str:
    at = -1
    for _ in range(n + 1):
        at = text.find(old, at + 1)
        assert at >= 0, f"mutation site not found: {old!r} (occurrence {n})"
    return text[:at] + new + text[at + len(old):]


def _stage(dst: str, mutant) -> None:
    """A private copy of the oracle (sources only; it builds its own library) and of the pins."""
    os.makedirs(os.path.join(dst, "oracle"))
    os.makedirs(os.path.join(dst, "tests"))
    for name in (C_SRC, PY_SRC):
        with open(os.path.join(ROOT, "oracle", name), encoding="utf-8") as f:
            text = f.read()
        if mutant is not None and mutant[1] == name:
            text = _replace_nth(text, mutant[2], mutant[3], mutant[4])
        with open(os.path.join(dst, "oracle", name), "w", encoding="utf-8") as f:
            f.write(text)
    for name in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(dst, "tests", name))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))


def _run_pins(mutant) -> tuple[int, str]:
    with tempfile.TemporaryDirectory(prefix="oracle_mutant_") as tmp:
        _stage(tmp, mutant)
        env = dict(os.environ, OMP_NUM_THREADS="2", PYTHONDONTWRITEBYTECODE="1")
        env.pop("PYTHONPATH", None)
        p = subprocess.run(
            [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
             os.path.join("tests", "test_oracle_pins.py")],
            cwd=tmp, env=env, capture_output=True, text=True, timeout=600)
        return p.returncode, p.stdout[-2000:] + p.stderr[-2000:]


def test_mutants_sites_are_unique_enough():
    """Every mutation site exists in the current sources, and names are distinct."""
    assert len({m[0] for m in MUTANTS}) == len(MUTANTS)
    for name, fname, old, new, n in MUTANTS:
        with open(os.path.join(ROOT, "oracle", fname), encoding="utf-8") as f:
            text = f.read()
        assert text.count(old) > n, name
        assert old != new, name


@pytest.mark.timeout(1200)
def test_every_mutant_fails_a_pin():
    """The unmutated copy passes the pins; every mutant fails at least one of them (a failed
    assertion or a raised error in a test, never a crash of the interpreter)."""
    jobs = [None] + MUTANTS
    with cf.ThreadPoolExecutor(max_workers=max(1, min(6, (os.cpu_count() or 2) // 2))) as ex:
        results = list(ex.map(_run_pins, jobs))
    rc0, log0 = results[0]
    assert rc0 == 0, "unmutated copy of the oracle fails its pins:\n" + log0
    survivors = [(m[0], rc, log) for m, (rc, log) in zip(MUTANTS, results[1:]) if rc != 1]
    assert not survivors, "\n\n".join(f"{n}: exit {rc}\n{log}" for n, rc, log in survivors)
