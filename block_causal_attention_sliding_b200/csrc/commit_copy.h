// commit_copy.h -- the TMA form of the chunk commit (append/evict): declarations shared by the
// kernel (cache_kernels.cu) and the host code (swattn_host.cu).
#pragma once
#include "swattn_internal.h"

namespace swattn {

// src maps over the caller's K and V ([B, T, H, d], dimensions ordered {d, t, h, b}); dst maps
// over the ring ({d, T, S, H, B}); boxes of whole d rows x kCommitRows rows x min(H, kCommitHeads)
// heads, unswizzled on both sides (no thread reads the buffers), so a loaded box is stored as it
// lies.  With H <= kCommitHeads a source box is kCommitRows whole token rows, contiguous.
struct CommitMaps {
    CUtensorMap src_k, src_v, dst_k, dst_v;
};
constexpr int kCommitRows = 4;
constexpr int kCommitHeads = 24;
constexpr int kCommitBufs = 8;   // buffers per CTA (one CTA per SM)

// Up to kCommitBatch handles (layers) in one launch: each handle's maps, device state, table
// advance and slot count (16 x 512 B of maps keeps the launch parameters near 9 KB).
constexpr int kCommitBatch = 16;
struct alignas(64) CommitBatch {
    CommitMaps maps[kCommitBatch];
    int32_t* state[kCommitBatch];
    TableAdvance ta[kCommitBatch];
    int S[kCommitBatch];
    int n;
};

// The chunk commit of cb.n handles of the same B, T, H, d and formats: ctas_per_handle blocks
// split each handle's items; each handle's last block advances its own counter and table.
cudaError_t launch_commit_tma_batch(const CommitBatch& cb, int B, int T, int H, int d, int k_esz, int v_esz,
                                    int ctas_per_handle, cudaStream_t stream);

// Copy the finished chunk into the ring slot the device counter names, then (last CTA) advance
// the counter and rebuild the table.  ctas: one per SM.  k_esz, v_esz: bytes per K and V element
// (1: e4m3, 2: bf16).
cudaError_t launch_commit_tma(const CommitMaps& maps, int B, int T, int H, int d, int k_esz, int v_esz,
                              int32_t* state, const TableAdvance& ta, int S, int ctas, cudaStream_t stream);

}  // namespace swattn
