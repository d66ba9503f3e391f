"""Workload shapes for streaming block-causal sink + sliding-window attention.

Token counts follow the JoyAI-Video-Edit pages: one latent frame per chunk (8 video frames)
and a VAE that maps 24x24 pixels to one token (neurohive review, section "Архитектура
JoyAI-Video-Edit"), so a 720x1280 chunk holds 30x53 = 1590 tokens per side; a chunk carries
aligned source and target tokens (agifrontier tutorial, section "从双向编辑到分块因果架构的蜕变"),
so T = 2 * 1590 = 3180 queries.  Two denoise steps run per chunk (same tutorial, section
"SA-DMD"), after which the clean chunk is committed to the cache.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int          # independent streams
    H: int          # heads
    d: int          # head dim
    T: int          # tokens per chunk (source + target)
    n_cond: int     # condition tokens, always visible
    W: int          # window: number of most recent history chunks kept
    sink: bool      # first chunk pinned as a permanent global sink
    chunks: int     # chunks streamed
    steps: int      # denoise steps (forwards) per chunk
    outlier_p: float = 0.0   # probability a key row is drawn with sigma 4 (variance 16)

    @property
    def scale(self) -> float:
        return self.d ** -0.5

    @property
    def slots(self) -> int:
        return self.W + (1 if self.sink else 0)

    def n_hist(self, k: int) -> int:
        """Number of visible history chunks for active chunk k (window union sink)."""
        win = min(k, self.W)
        extra = 1 if (self.sink and k >= 1 and k - self.W > 0) else 0
        return win + extra

    def n_vis(self, k: int) -> int:
        return self.n_cond + self.T * (self.n_hist(k) + 1)

    def flops_forward(self, k: int, n_q: int | None = None) -> float:
        """Algorithmic FLOPs of one forward: QK^T and PV over the visible keys only."""
        nq = self.T if n_q is None else n_q
        return 4.0 * self.B * self.H * nq * self.n_vis(k) * self.d

    def steady_k(self) -> int:
        """First chunk index with the full window plus the sink visible."""
        return self.W + 1 if self.sink else self.W


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, d=64, T=16, n_cond=8, W=1, sink=True, chunks=4, steps=2),
    "480p": Workload("480p", B=1, H=16, d=128, T=1400, n_cond=64, W=2, sink=True, chunks=16, steps=2),
    "720p": Workload("720p", B=1, H=24, d=128, T=3180, n_cond=256, W=3, sink=True, chunks=32, steps=2),
    "long720p": Workload("long720p", B=1, H=24, d=128, T=3180, n_cond=256, W=3, sink=True,
                         chunks=225, steps=2),
    "stress": Workload("stress", B=4, H=32, d=128, T=3180, n_cond=512, W=6, sink=True, chunks=32,
                       steps=2, outlier_p=0.01),
}
