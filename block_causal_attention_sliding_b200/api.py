"""Python face of libswattn: one handle = one layer's bounded KV cache on one GPU.

PyTorch provides the device memory (the workspace and the caller's tensors) and the stream;
the library's kernels do every step of the computation.  Calls enqueue on the current torch
stream and never synchronise, so a chunk step can be captured in a CUDA graph.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native as N


def _stream_ptr(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dev_ptr(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return int(t.data_ptr())


class SlidingWindowAttention:
    """Streaming block-causal attention over [condition ; sink ; window ; current chunk].

    One handle holds one layer's cache (sw_attn_create_ex + a torch-allocated workspace).
    schedule: "auto", "persistent", "tri", "grid" or "pair" (the full-path kernel); qk_fp8 /
    pv_fp8: e4m3 queries and keys / values with per-tensor scales; commit_in_forward: keep a spare
    window slot for forward_commit; commit_path: "auto", "tma" or "copy" for chunk commits."""

    def __init__(self, *, H: int, d: int, T: int, W: int, n_cond: int, B: int = 1,
                 sink: bool = True, out_dtype=torch.bfloat16, scale: float | None = None,
                 max_short_q: int = 0, schedule: str = "auto", commit_in_forward: bool = False,
                 qk_fp8: bool = False, q_scale: float = 1.0, k_scale: float = 1.0, commit_path: str = "auto",
                 pv_fp8: bool = False, v_scale: float = 1.0, device=None):
        self._lib = N.lib()
        cfg = N.SwAttnConfig(B=B, H=H, d=d, tokens_per_chunk=T, W=W, n_cond=n_cond,
                             sink=int(bool(sink)),
                             out_dtype=N.SW_OUT_F32 if out_dtype == torch.float32 else N.SW_OUT_BF16,
                             scale=0.0 if scale is None else float(scale), max_short_q=max_short_q,
                             schedule={"persistent": N.SW_SCHED_PERSISTENT, "grid": N.SW_SCHED_GRID,
                                       "tri": N.SW_SCHED_TRI, "pair": N.SW_SCHED_PAIR,
                                       "auto": N.SW_SCHED_AUTO}[schedule],
                             commit_in_forward=int(bool(commit_in_forward)), qk_fp8=int(bool(qk_fp8)),
                             q_scale=float(q_scale), k_scale=float(k_scale),
                             commit_path={"auto": N.SW_COMMIT_AUTO, "copy": N.SW_COMMIT_COPY,
                                          "tma": N.SW_COMMIT_TMA}[commit_path],
                             pv_fp8=int(bool(pv_fp8)), v_scale=float(v_scale))
        if out_dtype not in (torch.float32, torch.bfloat16):
            raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
        h = ctypes.c_void_p()
        N.check(self._lib.sw_attn_create_ex(ctypes.byref(cfg), ctypes.byref(h)))
        self._h = h
        self.B, self.H, self.d, self.T, self.W, self.n_cond, self.sink = B, H, d, T, W, n_cond, bool(sink)
        # window slots of the ring: W, or W + 1 (a spare slot) with commit_in_forward
        self.R = W + 1 if (commit_in_forward and W > 0) else W
        # e4m3 queries and keys (FP8 handle), bf16 otherwise
        self.qk_fp8 = bool(qk_fp8)
        self.qk_dtype = torch.float8_e4m3fn if self.qk_fp8 else torch.bfloat16
        # e4m3 V as well (pv_fp8), bf16 otherwise
        self.pv_fp8 = bool(pv_fp8)
        self.v_dtype = torch.float8_e4m3fn if self.pv_fp8 else torch.bfloat16
        self.out_dtype = out_dtype
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        nbytes = int(self._lib.sw_attn_workspace_bytes(h))
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            N.check(self._lib.sw_attn_bind_workspace(h, self.workspace.data_ptr(), nbytes, _stream_ptr()))
        self.table_ints = int(self._lib.sw_attn_table_ints(h))

    def commit_kind(self) -> str:
        """How chunk commits move K and V into the ring: "tma" (bulk copies) or "copy" (kernel)."""
        r = int(self._lib.sw_attn_commit_kind(self._h))
        if r < 0:
            N.check(r)
        return "tma" if r == N.SW_COMMIT_TMA else "copy"

    def schedule_for(self, n_q: int | None = None) -> str:
        """The schedule a full-path forward of n_q queries (default T) runs with."""
        r = int(self._lib.sw_attn_schedule_for(self._h, self.T if n_q is None else n_q))
        if r < 0:
            N.check(r)
        return {N.SW_SCHED_PERSISTENT: "persistent", N.SW_SCHED_GRID: "grid", N.SW_SCHED_TRI: "tri",
                N.SW_SCHED_PAIR: "pair"}[r]

    # -- stream control
    def set_cond(self, K_cond: torch.Tensor, V_cond: torch.Tensor, stream=None) -> None:
        shape = (self.B, self.n_cond, self.H, self.d)
        for name, t in (("K_cond", K_cond), ("V_cond", V_cond)):
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
        N.check(self._lib.sw_attn_set_cond(self._h, _dev_ptr(K_cond, "K_cond", self.qk_dtype),
                                           _dev_ptr(V_cond, "V_cond", self.v_dtype), _stream_ptr(stream)))

    def append_chunk(self, K: torch.Tensor, V: torch.Tensor, stream=None) -> None:
        shape = (self.B, self.T, self.H, self.d)
        for name, t in (("K", K), ("V", V)):
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
        N.check(self._lib.sw_attn_append_chunk(self._h, _dev_ptr(K, "K", self.qk_dtype),
                                               _dev_ptr(V, "V", self.v_dtype), _stream_ptr(stream)))

    def forward(self, Q: torch.Tensor, K_cur: torch.Tensor, V_cur: torch.Tensor,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        if Q.dim() != 4 or Q.shape[0] != self.B or Q.shape[2] != self.H or Q.shape[3] != self.d:
            raise ValueError(f"Q must be [B, n_q, H, d] = [{self.B}, n_q, {self.H}, {self.d}]")
        n_q = int(Q.shape[1])
        kv_shape = (self.B, self.T, self.H, self.d)
        for name, t in (("K_cur", K_cur), ("V_cur", V_cur)):
            if tuple(t.shape) != kv_shape:
                raise ValueError(f"{name} must have shape {kv_shape}, got {tuple(t.shape)}")
        if out is None:
            out = torch.empty((self.B, n_q, self.H, self.d), dtype=self.out_dtype, device=Q.device)
        elif tuple(out.shape) != tuple(Q.shape) or out.dtype != self.out_dtype:
            raise ValueError("out must match Q's shape and the handle's out_dtype")
        N.check(self._lib.sw_attn_forward(self._h, _dev_ptr(Q, "Q", self.qk_dtype),
                                          _dev_ptr(K_cur, "K_cur", self.qk_dtype),
                                          _dev_ptr(V_cur, "V_cur", self.v_dtype),
                                          _dev_ptr(out, "out"), n_q, _stream_ptr(stream)))
        return out

    __call__ = forward

    def forward_commit(self, Q: torch.Tensor, K_cur: torch.Tensor, V_cur: torch.Tensor,
                       out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """The chunk's clean pass: forward of all T queries that also commits K_cur / V_cur to the
        cache (sw_attn_forward_commit; the handle needs commit_in_forward)."""
        shape = (self.B, self.T, self.H, self.d)
        for name, t in (("Q", Q), ("K_cur", K_cur), ("V_cur", V_cur)):
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
        if out is None:
            out = torch.empty(shape, dtype=self.out_dtype, device=Q.device)
        elif tuple(out.shape) != shape or out.dtype != self.out_dtype:
            raise ValueError("out must be [B, T, H, d] in the handle's out_dtype")
        N.check(self._lib.sw_attn_forward_commit(self._h, _dev_ptr(Q, "Q", self.qk_dtype),
                                                 _dev_ptr(K_cur, "K_cur", self.qk_dtype),
                                                 _dev_ptr(V_cur, "V_cur", self.v_dtype),
                                                 _dev_ptr(out, "out"), _stream_ptr(stream)))
        return out

    def forward_joint(self, Q: torch.Tensor, Q_cond: torch.Tensor, K_cur: torch.Tensor, V_cur: torch.Tensor,
                      out: torch.Tensor | None = None, out_cond: torch.Tensor | None = None,
                      stream=None) -> tuple[torch.Tensor, torch.Tensor]:
        """The chunk's queries (all T rows) and the condition-stream queries ([B, n_cond, H, d]) over
        the same visible keys, in one launch (sw_attn_forward_joint).  Returns (out, out_cond)."""
        q_shape = (self.B, self.T, self.H, self.d)
        qc_shape = (self.B, self.n_cond, self.H, self.d)
        for name, t, shp in (("Q", Q, q_shape), ("K_cur", K_cur, q_shape), ("V_cur", V_cur, q_shape),
                             ("Q_cond", Q_cond, qc_shape)):
            if tuple(t.shape) != shp:
                raise ValueError(f"{name} must have shape {shp}, got {tuple(t.shape)}")
        if out is None:
            out = torch.empty(q_shape, dtype=self.out_dtype, device=Q.device)
        if out_cond is None:
            out_cond = torch.empty(qc_shape, dtype=self.out_dtype, device=Q.device)
        for name, t, shp in (("out", out, q_shape), ("out_cond", out_cond, qc_shape)):
            if tuple(t.shape) != shp or t.dtype != self.out_dtype:
                raise ValueError(f"{name} must be {shp} in the handle's out_dtype")
        N.check(self._lib.sw_attn_forward_joint(self._h, _dev_ptr(Q, "Q", self.qk_dtype),
                                                _dev_ptr(Q_cond, "Q_cond", self.qk_dtype),
                                                _dev_ptr(K_cur, "K_cur", self.qk_dtype),
                                                _dev_ptr(V_cur, "V_cur", self.v_dtype),
                                                _dev_ptr(out, "out"), _dev_ptr(out_cond, "out_cond"),
                                                _stream_ptr(stream)))
        return out, out_cond

    def reset(self, stream=None) -> None:
        N.check(self._lib.sw_attn_reset(self._h, _stream_ptr(stream)))

    # -- inspection
    def table(self, stream=None) -> torch.Tensor:
        t = torch.empty(self.table_ints, dtype=torch.int32, device=self.device)
        N.check(self._lib.sw_attn_get_table(self._h, t.data_ptr(), _stream_ptr(stream)))
        return t

    def status(self) -> int:
        v = ctypes.c_int32(0)
        N.check(self._lib.sw_attn_get_status(self._h, ctypes.byref(v)))
        return int(v.value)

    def workspace_bytes(self) -> int:
        return int(self._lib.sw_attn_workspace_bytes(self._h))

    def cache_views(self):
        """(K_cache, V_cache) as [B, H, S, T, d] bf16 views of the workspace (for inspection)."""
        S = self.R + (1 if self.sink else 0)
        ko, vo = ctypes.c_size_t(0), ctypes.c_size_t(0)
        N.check(self._lib.sw_attn_cache_offsets(self._h, ctypes.byref(ko), ctypes.byref(vo)))
        n = 2 * self.B * self.H * S * self.T * self.d
        shape = (self.B, self.H, S, self.T, self.d)
        nk = n // 2 if self.qk_fp8 else n
        nv = n // 2 if self.pv_fp8 else n
        kc = self.workspace[ko.value: ko.value + nk].view(self.qk_dtype).view(shape)
        vc = self.workspace[vo.value: vo.value + nv].view(self.v_dtype).view(shape)
        return kc, vc

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.sw_attn_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def append_chunk_batched(handles, Ks, Vs, stream=None) -> None:
    """Commit the finished chunk of several handles (e.g. every layer of a model) in one copy
    launch and one table launch (sw_attn_append_chunk_batched).  Handles share B, H, d, T."""
    n = len(handles)
    if n < 1 or len(Ks) != n or len(Vs) != n:
        raise ValueError("need one K and one V per handle")
    for h, K, V in zip(handles, Ks, Vs):
        shape = (h.B, h.T, h.H, h.d)
        if tuple(K.shape) != shape or tuple(V.shape) != shape:
            raise ValueError(f"K and V must have shape {shape}")
    lib = handles[0]._lib
    hp = (ctypes.c_void_p * n)(*[h._h.value for h in handles])
    kp = (ctypes.c_void_p * n)(*[_dev_ptr(K, "K", h.qk_dtype) for h, K in zip(handles, Ks)])
    vp = (ctypes.c_void_p * n)(*[_dev_ptr(V, "V", h.v_dtype) for h, V in zip(handles, Vs)])
    N.check(lib.sw_attn_append_chunk_batched(ctypes.cast(hp, ctypes.c_void_p), n, ctypes.cast(kp, ctypes.c_void_p),
                                             ctypes.cast(vp, ctypes.c_void_p), _stream_ptr(stream)))
