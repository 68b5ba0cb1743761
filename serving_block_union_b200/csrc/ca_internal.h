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

int launch_chunk_attention(const AttnArgs &a, bool dense, cudaStream_t stream);

}  // namespace ca
