"""The table builder (K1) run on the host with the device's own code (sw_attn_table_host),
bit for bit against the oracle's canonical table and chunk bitmap row, over far more chunks,
windows and ring sizes than a GPU run visits; plus the counter advance and its overflow flag.
The visibility rule is from the agifrontier tutorial, section "从双向编辑到分块因果架构的蜕变",
and the neurohive review, section "Чанки и борьба с дрейфом".  Host only.
"""
from __future__ import annotations

import numpy as np
import pytest

from block_causal_attention_sliding_b200 import _native as N

HEADER = 16   # state ints before the table: [0] chunks committed, [1] status bits


def table_host(k, W, R, sink, n_cond, T, advance=0):
    cap = HEADER + 3 + 4 * (W + 3) + 3
    out = np.full(cap, 12345, dtype=np.int32)
    n = N.lib().sw_attn_table_host(k, W, R, int(sink), n_cond, T, advance, out.ctypes.data, cap)
    assert n == cap, n
    return out


@pytest.mark.parametrize("sink", [False, True])
@pytest.mark.parametrize("W", [0, 1, 2, 3, 4, 5, 6, 7, 31, 63, 64])
def test_table_builder_matches_oracle(oracle_mod, W, sink):
    import parity_util as PU
    for R in sorted({W, W + 1 if W > 0 else 0}):
        for n_cond in (0, 5):
            for k in range(0, min(200, 3 * W + 12)):
                out = table_host(k, W, R, sink, n_cond, T=11)
                assert out[0] == k and out[1] == 0
                PU.check_table(out[HEADER:], k, W, sink, n_cond, 11, R=R)


def test_table_builder_advance_and_overflow(oracle_mod):
    import parity_util as PU
    for k in (0, 1, 4, 99):
        out = table_host(k, 3, 3, True, 256, 3180, advance=1)
        assert out[0] == k + 1 and out[1] == 0              # a commit advances the counter
        PU.check_table(out[HEADER:], k + 1, 3, True, 256, 3180)
    out = table_host(1 << 30, 3, 3, True, 0, 16, advance=1)
    assert out[0] == 1 << 30                                 # the counter stops
    assert out[1] & N.SW_STATUS_OVERFLOW                     # and the overflow bit is raised


def test_table_hook_rejects_bad_arguments():
    L = N.lib()
    buf = np.zeros(64, dtype=np.int32)
    p = buf.ctypes.data
    assert L.sw_attn_table_host(0, 3, 3, 1, 0, 16, 0, None, 64) == N.SW_EINVAL
    assert L.sw_attn_table_host(-1, 3, 3, 1, 0, 16, 0, p, 64) == N.SW_EINVAL
    assert L.sw_attn_table_host(0, 65, 65, 1, 0, 16, 0, p, 64) == N.SW_EINVAL   # W <= 64
    assert L.sw_attn_table_host(0, 3, 5, 1, 0, 16, 0, p, 64) == N.SW_EINVAL     # R is W or W + 1
    assert L.sw_attn_table_host(0, 0, 1, 1, 0, 16, 0, p, 64) == N.SW_EINVAL     # W = 0 keeps no slot
    assert L.sw_attn_table_host(0, 3, 3, 2, 0, 16, 0, p, 64) == N.SW_EINVAL
    assert L.sw_attn_table_host(0, 3, 3, 1, 0, 0, 0, p, 64) == N.SW_EINVAL
    assert L.sw_attn_table_host(0, 3, 3, 1, 0, 16, 0, p, 20) == N.SW_ESHAPE      # cap too small
