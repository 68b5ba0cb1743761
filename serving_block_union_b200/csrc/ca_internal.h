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

// page_ids: CSR indices hold global pages (b * H_kv + g) * nKVmax + j.
int launch_build_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                        int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                        bool page_ids, cudaStream_t stream);

// The same from a bit-packed mask (uint32 [B, H_q, nQ, ceil(nKVmax / 32)]).
int launch_build_tables_bits(const uint32_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                             int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                             bool page_ids, cudaStream_t stream);

struct AttnArgs {
    const void *Q, *K, *V;
    const int32_t *tables, *counts;  // NULL for the dense path
    const int32_t *chunk_start;      // host
    int B, H_q, H_kv, C, L_max, D, blk;
    float scale;
    void *O;
    float *LSE;
    void *workspace;
    size_t workspace_bytes;
    // paged form (kModeTables only): tables = kv_indices (global pages, nnz
    // entries), counts unused, rows of (b, g) at kv_indptr[b*H_kv+g] ..
    const int32_t *kv_indptr = nullptr;
    long long nnz = 0;
    const int32_t *chunk_len = nullptr;  // host [B], NULL: every chunk is C rows
    // FP8 inputs: Q, K, V hold E4M3 codes; the real values are the codes times
    // descale[0] (Q), descale[1] (K), descale[2] (V)
    bool fp8 = false;
    float descale[3] = {1.0f, 1.0f, 1.0f};
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

// Host-side argument checks shared by every attention entry point (dense: no
// tables / counts; chunk_len: NULL when every chunk has C rows). Returns CA_OK
// or the error code the entry point reports; enqueues nothing.
int check_attention(const void *Q, const void *K, const void *V, const int32_t *tables,
                    const int32_t *counts, bool dense, const int32_t *chunk_start, int B, int H_q,
                    int H_kv, int C, int L_max, int D, int blk, float scale, const void *O,
                    const float *LSE, const void *workspace, size_t workspace_bytes,
                    const int32_t *chunk_len = nullptr);

// ---- split of the last wave (split-KV with an LSE merge)
//
// One CTA runs one work item (two 128-row tiles against a block list) and one
// CTA fits an SM, so n_items CTAs take ceil(n_items / SMs) waves and the last
// wave can be mostly empty (256 items on 148 SMs: 1.73 waves of work in 2).
// The plan keeps the full waves [0, n_first) whole and cuts each remaining
// item's block list into `split` segments run by separate CTAs, choosing the
// split that makes those segment waves shortest. Each segment CTA writes a
// normalised partial O (bf16) and its base-2 LSE (fp32) to the workspace;
// the last of an item's CTAs to finish merges them in fp32 (workspace
// counters, no waiting). The kernel keeps a split item whole where its table
// prefix is shorter than kMinSegEntries blocks per segment: measured on B200
// at split 4, segments of ~22 blocks (2% density, full-prefill chunk 25)
// gain nothing, ~33 (chunk 40) gain 2%, ~50 (5% density) 3%; the host
// cannot see the table lengths, the kernel can.
constexpr int kMaxSplit = 8;
constexpr int kMinSegEntries = 24;
constexpr int kRowsPerItem = 256;     // packed rows of one item (two tiles)
constexpr int kSplitMinBlocks = 64;   // items shorter than this are not split

struct SplitPlan {
    int n_items = 0, n_first = 0, split = 1;
    size_t bytes = kWorkspaceHeader;  // workspace this plan needs
    size_t lse_off = 0, o_off = 0;    // byte offsets of the partial LSE / O arrays
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline SplitPlan plan_split(int n_items, int num_sms, int D, bool allow) {
    SplitPlan p;
    p.n_items = p.n_first = n_items;
    if (!allow || num_sms <= 0 || n_items <= 0) return p;
    const int n_first = (n_items / num_sms) * num_sms;
    const int n_rest = n_items - n_first;
    if (n_rest == 0) return p;
    int best_s = 1;
    long long best_waves = 1, best_den = 1;  // last waves' length as a fraction
    for (int s = 2; s <= kMaxSplit; ++s) {
        const long long waves = ((long long)n_rest * s + num_sms - 1) / num_sms;
        if (waves * best_den < best_waves * s) {  // waves / s < best
            best_s = s;
            best_waves = waves;
            best_den = s;
        }
    }
    if (best_s == 1) return p;
    const size_t rows = (size_t)n_rest * best_s * kRowsPerItem;
    p.n_first = n_first;
    p.split = best_s;
    p.lse_off = kWorkspaceHeader + align256(4 * (size_t)n_rest);
    p.o_off = p.lse_off + align256(4 * rows);
    p.bytes = p.o_off + 2 * rows * (size_t)D;  // bf16 partial O
    return p;
}

// Work items of one attention launch: B * units * pairs, the unit a KV group
// (G query heads packed per tile) or, in the per-tile mode, a query head.
inline int attention_items(int B, int H_q, int H_kv, int C, bool per_tile) {
    const int pack = per_tile ? 1 : H_q / H_kv;
    const int R = 128 / pack;
    const int n_pairs = ((C + R - 1) / R + 1) / 2;
    return B * (per_tile ? H_q : H_kv) * n_pairs;
}

// SM count of the current device (cached per device; 148 if it cannot be read).
int current_sm_count();

// Copies the K and V blocks each table selects into compact buffers: block
// tables[b,g,t] of the cache goes to rows [t * blk, (t + 1) * blk) of Kc / Vc.
int launch_compact_kv(const void *K, const void *V, const int32_t *tables, const int32_t *counts,
                      int B, int H_kv, int L_max, int D, int blk, void *Kc, void *Vc,
                      cudaStream_t stream);

// Merge of n attention results over disjoint key sets (2 <= n <= kMaxMergeParts):
// LSE = ln sum_i exp(LSE_i), O = sum_i exp(LSE_i - LSE) O_i; bf16 O, fp32 LSE.
constexpr int kMaxMergeParts = 8;
int launch_merge_states(const void *const *O_parts, const float *const *LSE_parts, int n,
                        long long rows, int D, void *O, float *LSE, cudaStream_t stream);

}  // namespace ca
