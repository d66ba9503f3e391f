"""Failure detection on the GPU without a GPU fault: a kernel whose bounded wait runs out (on a
barrier nothing completes) records SW_STATUS_TIMEOUT and returns; the status is read on the
host, cleared by reset, and the same handle computes correctly afterwards."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_sliding_b200 import _native, synth
from block_causal_attention_sliding_b200.configs import WORKLOADS

from parity_util import compare, make_handle

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = WORKLOADS["tiny"]
    h = make_handle(wl, dev, max_short_q=-1)
    lib = _native.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert h.status() == 0
    assert lib.sw_attn_selftest_timeout(h._h, 50_000_000, stream) == 0      # 50 ms limit
    assert h.status() & _native.SW_STATUS_TIMEOUT
    assert lib.sw_attn_selftest_timeout(h._h, 10, stream) == _native.SW_EINVAL
    h.reset()
    assert h.status() == 0
    # the context and the handle still work
    Kc, Vc = synth.cond_inputs(wl)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    Q, K, V = synth.chunk_inputs(wl, 0, 0)
    got = h.forward(Q.to(dev), K.to(dev), V.to(dev)).cpu().numpy()
    ref = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=0, Kc=Kc, Vc=Vc,
                           hist_K=[], hist_V=[], Q=Q, K_cur=K, V_cur=V)
    compare(got, ref)
    assert h.status() == 0
