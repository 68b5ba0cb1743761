// ca_internal.h — declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/compactattn.h"

namespace ca {

// Most sequences one call accepts (chunk starts travel in the kernel parameters).
constexpr int kMaxBatch = 128;

// Workspace layout (bytes): [0, 4) status word, [4, 8) work-item counter,
// [8, 12) finished-CTA counter; padded to 256.
constexpr size_t kWorkspaceHeader = 256;

int launch_build_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                        int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                        cudaStream_t stream);

struct AttnArgs {
    const void *Q, *K, *V;
    const int32_t *tables, *counts;  // NULL for the dense path
    const int32_t *chunk_start;      // host
    int B, H_q, H_kv, C, L_max, D, blk;
    float scale;
    void *O;
    float *LSE;
    void *workspace;
};

// Attention kernel modes: walk the tables over the cache in place; every block
// of the visible length (the dense path); or the tables' blocks gathered into a
// compact buffer (block t of a table at row t * blk, masked by its original
// position — the explicit-compaction ablation).
constexpr int kModeTables = 0;
constexpr int kModeDense = 1;
constexpr int kModeCompact = 2;
// Per-tile block-sparse ablation: one work item per (b, query head, 256 chunk
// rows), walking that head's span table (entries j | Q-block bits << 24).
constexpr int kModePerTile = 3;

// Chunk rows of one per-tile work item (two 128-row tiles of one head); the
// span tables group a head's Q-blocks by it.
constexpr int kTileItemRows = 256;
// Low bits of a span-table entry that hold the KV block index.
constexpr int kSpanEntryBits = 24;

int launch_tile_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int span,
                       int32_t *tables, int32_t *counts, cudaStream_t stream);

int launch_chunk_attention(const AttnArgs &a, int mode, cudaStream_t stream);

// Copies the K and V blocks each table selects into compact buffers: block
// tables[b,g,t] of the cache goes to rows [t * blk, (t + 1) * blk) of Kc / Vc.
int launch_compact_kv(const void *K, const void *V, const int32_t *tables, const int32_t *counts,
                      int B, int H_kv, int L_max, int D, int blk, void *Kc, void *Vc,
                      cudaStream_t stream);

}  // namespace ca
