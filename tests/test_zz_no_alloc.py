"""The allocation-free short-query forward, called through the C ABI.

sw_attn_forward_short_noalloc serves callers that cannot allocate device memory when they
call (a host framework's fixed pool, a fixed-footprint server): its split-K partials live in
a fixed array inside the library instead of the handle's workspace.  On two calls in a row
(the second reuses the array the first one left behind) its output must equal the ordinary
entry point's bit for bit -- both run the same split kernel and combine with the same split
count -- and match the FP64 oracle within the parity tolerance.  Kept in a file of its own so
a run that stops at the first failure has already run everything else; it must pass both alone
and after the other tests.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from block_causal_attention_sliding_b200 import _native, synth
from block_causal_attention_sliding_b200.configs import Workload

from parity_util import E4M3_P_TOL, MAX_ABS, MEAN_REL, compare, make_handle

pytestmark = pytest.mark.gpu


def test_noalloc_matches_forward_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_attention_sliding_b200 import build as B
    B.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    import oracle
    oracle.build()
    wl = Workload("noalloc", B=2, H=3, d=128, T=300, n_cond=40, W=2, sink=True, chunks=4, steps=1)
    h = make_handle(wl, dev)   # fp32 output
    Kc, Vc = synth.cond_inputs(wl)
    h.set_cond(Kc.to(dev), Vc.to(dev))
    hist_K, hist_V = [], []
    for k in range(3):
        _, K, V = synth.chunk_inputs(wl, k, 0)
        h.append_chunk(K.to(dev), V.to(dev))
        hist_K.append(K)
        hist_V.append(V)
    lib = _native.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call, n_q in enumerate((64, 17)):
        Qh, Kh, Vh = synth.chunk_inputs(wl, 3, call, n_q=n_q)
        Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
        ref = h.forward(Q, K, V)                      # existing entry point (workspace scratch)
        out = torch.full_like(ref, float("nan"))
        rc = lib.sw_attn_forward_short_noalloc(h._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                               out.data_ptr(), n_q, ctypes.c_void_p(stream))
        assert rc == 0, lib.sw_attn_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from sw_attn_forward"
        exact = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=3, Kc=Kc, Vc=Vc,
                                 hist_K=hist_K, hist_V=hist_V, Q=Qh, K_cur=Kh, V_cur=Vh)
        compare(out.cpu().numpy(), exact, MAX_ABS, MEAN_REL)
    assert h.status() == 0
    # a shape that cannot fit even one split in the fixed array is refused, not truncated
    big = make_handle(Workload("big", B=1, H=256, d=128, T=8, n_cond=0, W=0, sink=False, chunks=1, steps=1), dev)
    q = torch.zeros((1, 8, 256, 128), dtype=torch.bfloat16, device=dev)
    o = torch.empty((1, 8, 256, 128), dtype=torch.float32, device=dev)
    rc = lib.sw_attn_forward_short_noalloc(big._h, q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), 8,
                                           ctypes.c_void_p(stream))
    assert rc == _native.SW_ESHAPE and b"scratch" in lib.sw_attn_last_error()


@pytest.mark.parametrize("pv8", [False, True])
def test_noalloc_fp8_matches_forward(pv8):
    """Handles with e4m3 Q and K (and V with pv8) take the same split kernel: the allocation-free
    entry equals sw_attn_forward bit for bit and the oracle on the dequantised inputs."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_attention_sliding_b200 import build as B
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    B.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    import oracle
    oracle.build()
    wl = Workload("noalloc8", B=2, H=3, d=128, T=300, n_cond=40, W=2, sink=True, chunks=4, steps=1)
    sc = synth.FP8_SCALE
    h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                               out_dtype=torch.float32, qk_fp8=True, q_scale=sc, k_scale=sc, pv_fp8=pv8,
                               v_scale=sc, device=dev)
    deq_v = synth.from_e4m3 if pv8 else (lambda t: t)
    Kc8, Vc = synth.cond_inputs_fp8(wl, v8=pv8)
    h.set_cond(Kc8.to(dev), Vc.to(dev))
    hist_K, hist_V = [], []
    for k in range(3):
        _, K8, V = synth.chunk_inputs_fp8(wl, k, 0, v8=pv8)
        h.append_chunk(K8.to(dev), V.to(dev))
        hist_K.append(synth.from_e4m3(K8))
        hist_V.append(deq_v(V))
    lib = _native.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call, n_q in enumerate((64, 17)):
        Q8h, K8h, Vh = synth.chunk_inputs_fp8(wl, 3, call, n_q=n_q, v8=pv8)
        Q8, K8, V = Q8h.to(dev), K8h.to(dev), Vh.to(dev)
        ref = h.forward(Q8, K8, V)
        out = torch.full_like(ref, float("nan"))
        rc = lib.sw_attn_forward_short_noalloc(h._h, Q8.data_ptr(), K8.data_ptr(), V.data_ptr(),
                                               out.data_ptr(), n_q, ctypes.c_void_p(stream))
        assert rc == 0, lib.sw_attn_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from sw_attn_forward"
        exact = oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=3,
                                 Kc=synth.from_e4m3(Kc8), Vc=deq_v(Vc), hist_K=hist_K, hist_V=hist_V,
                                 Q=synth.from_e4m3(Q8h), K_cur=synth.from_e4m3(K8h), V_cur=deq_v(Vh))
        compare(out.cpu().numpy(), exact, *(E4M3_P_TOL if pv8 else (MAX_ABS, MEAN_REL)))
    assert h.status() == 0
