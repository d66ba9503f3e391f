"""Seeded synthetic inputs for the streaming attention (no method arithmetic lives here).

Both the CUDA path's tests and the oracle draw from this module, so the two see bit-identical
bf16 inputs.  Recipe (stated once, used everywhere):
  * each tensor is drawn from its own CPU ``torch.Generator`` seeded with
    ``seed * 1_000_000 + chunk * 100 + step * 10 + tensor_id``;
  * values are N(0, 1) in float32, then rounded to bf16 (round to nearest even);
  * with ``outlier_p > 0`` every key row (b, token, h) is independently an outlier with that
    probability and is multiplied by 4 (an N(0, 16) draw), in K_cur, committed K and the
    condition K alike;
  * tensor ids: Q = 0, K_cur = 1, V_cur = 2, condition K = 3, condition V = 4, condition-stream
    queries = 5; condition K/V use chunk 0, step 0 for the first prompt and chunk v, step 0 for
    prompt version v (a prompt changed mid-stream); condition queries use the (chunk, step) of
    the forward they belong to.
  * FP8 inputs (queries and keys of an e4m3 handle, and values too on a handle with e4m3 V): the
    same draws divided by a power-of-two scale (FP8_SCALE, exact) and rounded to OCP e4m3
    (float8_e4m3fn, round to nearest even); the dequantised values x8 * FP8_SCALE are what the
    attention sees.
The user layout is [B, N, H, d] contiguous.
"""
from __future__ import annotations

import torch

TID_Q, TID_K, TID_V, TID_KC, TID_VC, TID_QC = 0, 1, 2, 3, 4, 5


def stream_seed(seed: int, chunk: int, step: int, tensor_id: int) -> int:
    return seed * 1_000_000 + chunk * 100 + step * 10 + tensor_id


def draw(shape, seed_int: int, *, outlier_p: float = 0.0, device="cpu") -> torch.Tensor:
    """N(0,1) float32 -> bf16, optional sigma-4 outlier rows along the last dim."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed_int))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if outlier_p > 0.0:
        sel = torch.rand(tuple(shape[:-1]), generator=g, device=device) < outlier_p
        x = torch.where(sel.unsqueeze(-1), x * 4.0, x)
    return x.to(torch.bfloat16)


def chunk_inputs(wl, chunk: int, step: int, *, seed: int = 0, n_q: int | None = None,
                 device="cpu"):
    """Q [B, n_q, H, d], K_cur and V_cur [B, T, H, d] for one (chunk, step)."""
    nq = wl.T if n_q is None else n_q
    qshape = (wl.B, nq, wl.H, wl.d)
    kshape = (wl.B, wl.T, wl.H, wl.d)
    if nq == wl.T:
        Q = draw(qshape, stream_seed(seed, chunk, step, TID_Q), device=device)
    else:
        # short query sets are the first n_q rows of a full draw
        Q = draw(kshape, stream_seed(seed, chunk, step, TID_Q), device=device)[:, :nq].contiguous()
    K = draw(kshape, stream_seed(seed, chunk, step, TID_K), outlier_p=wl.outlier_p, device=device)
    V = draw(kshape, stream_seed(seed, chunk, step, TID_V), device=device)
    return Q, K, V


def cond_inputs(wl, *, seed: int = 0, version: int = 0, device="cpu"):
    """Condition K, V [B, n_cond, H, d] of prompt version `version` (0: the stream's first)."""
    shape = (wl.B, wl.n_cond, wl.H, wl.d)
    Kc = draw(shape, stream_seed(seed, version, 0, TID_KC), outlier_p=wl.outlier_p, device=device)
    Vc = draw(shape, stream_seed(seed, version, 0, TID_VC), device=device)
    return Kc, Vc


def cond_queries(wl, chunk: int, step: int, *, seed: int = 0, device="cpu"):
    """Condition-stream queries Q_cond [B, n_cond, H, d] for one (chunk, step)."""
    return draw((wl.B, wl.n_cond, wl.H, wl.d), stream_seed(seed, chunk, step, TID_QC), device=device)


FP8_SCALE = 2.0 ** -4   # |x| / FP8_SCALE stays below the e4m3 limit (448) even for sigma-4 outlier keys


def to_e4m3(x: torch.Tensor, scale: float = FP8_SCALE) -> torch.Tensor:
    """x / scale rounded to e4m3 (scale a power of two, so the division is exact)."""
    return (x.float() / scale).to(torch.float8_e4m3fn)


def from_e4m3(x8: torch.Tensor, scale: float = FP8_SCALE) -> torch.Tensor:
    """The dequantised values x8 * scale, exact in float32."""
    return x8.float() * scale


def chunk_inputs_fp8(wl, chunk: int, step: int, *, seed: int = 0, n_q: int | None = None, device="cpu",
                     v8: bool = False):
    """Q and K_cur in e4m3, V_cur in bf16 (e4m3 with v8), for one (chunk, step) of an e4m3 handle."""
    Q, K, V = chunk_inputs(wl, chunk, step, seed=seed, n_q=n_q, device=device)
    return to_e4m3(Q), to_e4m3(K), (to_e4m3(V) if v8 else V)


def cond_inputs_fp8(wl, *, seed: int = 0, version: int = 0, device="cpu", v8: bool = False):
    """Condition K in e4m3, V in bf16 (e4m3 with v8)."""
    Kc, Vc = cond_inputs(wl, seed=seed, version=version, device=device)
    return to_e4m3(Kc), (to_e4m3(Vc) if v8 else Vc)
