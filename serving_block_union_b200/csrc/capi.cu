// capi.cu — the extern "C" boundary: host-side argument checks, then one
// asynchronous launch on the caller's stream. See include/compactattn.h for
// the contract of every entry point.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ca_internal.h"
#include "sm100_ptx.cuh"

namespace {

inline bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline bool supported_group(int G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }

}  // namespace

namespace ca {

int check_attention(const void *Q, const void *K, const void *V, const int32_t *tables,
                    const int32_t *counts, bool dense, const int32_t *chunk_start, int B, int H_q,
                    int H_kv, int C, int L_max, int D, int blk, float scale, const void *O,
                    const float *LSE, const void *workspace, size_t workspace_bytes,
                    const int32_t *chunk_len) {
    if (!Q || !K || !V || !O || !chunk_start || !workspace) return CA_ERR_INVALID_ARG;
    if (!dense && (!tables || !counts)) return CA_ERR_INVALID_ARG;
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || C <= 0 || L_max <= 0 || D <= 0 || blk <= 0)
        return CA_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !isfinite(scale)) return CA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return CA_ERR_SHAPE;
    if (L_max % blk != 0) return CA_ERR_SHAPE;
    for (int b = 0; b < B && b < ca::kMaxBatch; ++b) {
        const long long cs = chunk_start[b];
        const long long len = chunk_len ? chunk_len[b] : C;
        if (len < 0 || len > C) return CA_ERR_SHAPE;
        if (cs < 0 || cs + len > L_max) return CA_ERR_SHAPE;
    }
    if (!(D == 64 || D == 128) || !(blk == 64 || blk == 128)) return CA_ERR_UNSUPPORTED;
    if (!supported_group(H_q / H_kv)) return CA_ERR_UNSUPPORTED;
    if (B > ca::kMaxBatch) return CA_ERR_UNSUPPORTED;
    // element counts must stay inside 32-bit TMA coordinates and int indexing
    if ((long long)B * H_q * C >= (1LL << 31) || (long long)B * H_kv * L_max >= (1LL << 31))
        return CA_ERR_SHAPE;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
        return CA_ERR_ALIGN;
    if ((LSE && !aligned(LSE, 4)) || (tables && !aligned(tables, 4)) ||
        (counts && !aligned(counts, 4)))
        return CA_ERR_ALIGN;
    if (!aligned(workspace, 256) || workspace_bytes < ca::kWorkspaceHeader)
        return CA_ERR_WORKSPACE;
    return CA_OK;
}

}  // namespace ca

using ca::check_attention;

extern "C" {

const char *ca_status_string(int status) {
    switch (status) {
        case CA_OK: return "CA_OK";
        case CA_ERR_INVALID_ARG: return "CA_ERR_INVALID_ARG";
        case CA_ERR_SHAPE: return "CA_ERR_SHAPE";
        case CA_ERR_ALIGN: return "CA_ERR_ALIGN";
        case CA_ERR_UNSUPPORTED: return "CA_ERR_UNSUPPORTED";
        case CA_ERR_WORKSPACE: return "CA_ERR_WORKSPACE";
        case CA_ERR_TABLE: return "CA_ERR_TABLE";
        case CA_ERR_TIMEOUT: return "CA_ERR_TIMEOUT";
        case CA_ERR_CUDA: return "CA_ERR_CUDA";
        default: return "CA_ERR_UNKNOWN";
    }
}

int ca_version(void) { return 200; }

size_t ca_workspace_bytes(int B, int H_q, int H_kv, int C, int blk) {
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || C <= 0 || blk <= 0 || H_q % H_kv != 0) return 0;
    // room for the last-wave split of either item layout, at the largest D
    const int sms = ca::current_sm_count();
    size_t bytes = ca::kWorkspaceHeader;
    for (int per_tile = 0; per_tile < 2; ++per_tile) {
        const int n = ca::attention_items(B, H_q, H_kv, C, per_tile != 0);
        const ca::SplitPlan plan = ca::plan_split(n, sms, 128, true);
        if (plan.bytes > bytes) bytes = plan.bytes;
    }
    return bytes;
}

int ca_build_block_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                          int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                          void *stream) {
    if (!mask || !tables || !counts) return CA_ERR_INVALID_ARG;
    if (indices && !indptr) return CA_ERR_INVALID_ARG;
    if (B <= 0 || H_q <= 0 || nQ <= 0 || nKVmax <= 0 || group <= 0) return CA_ERR_INVALID_ARG;
    if (H_q % group != 0) return CA_ERR_SHAPE;
    if ((long long)B * H_q * nQ * nKVmax >= (1LL << 40)) return CA_ERR_SHAPE;
    if ((long long)B * (H_q / group) * nKVmax >= (1LL << 31)) return CA_ERR_SHAPE;
    if (!aligned(tables, 4) || !aligned(counts, 4) || (indptr && !aligned(indptr, 4)) ||
        (indices && !aligned(indices, 4)))
        return CA_ERR_ALIGN;
    return ca::launch_build_tables(mask, B, H_q, nQ, nKVmax, group, tables, counts, indptr,
                                   indices, false, static_cast<cudaStream_t>(stream));
}

int ca_build_block_tables_bits(const uint32_t *mask_bits, int B, int H_q, int nQ, int nKVmax,
                               int group, int32_t *tables, int32_t *counts, int32_t *indptr,
                               int32_t *indices, void *stream) {
    if (!mask_bits || !tables || !counts) return CA_ERR_INVALID_ARG;
    if (indices && !indptr) return CA_ERR_INVALID_ARG;
    if (B <= 0 || H_q <= 0 || nQ <= 0 || nKVmax <= 0 || group <= 0) return CA_ERR_INVALID_ARG;
    if (H_q % group != 0) return CA_ERR_SHAPE;
    if ((long long)B * H_q * nQ * ((nKVmax + 31) / 32) >= (1LL << 38)) return CA_ERR_SHAPE;
    if ((long long)B * (H_q / group) * nKVmax >= (1LL << 31)) return CA_ERR_SHAPE;
    if (!aligned(mask_bits, 4) || !aligned(tables, 4) || !aligned(counts, 4) ||
        (indptr && !aligned(indptr, 4)) || (indices && !aligned(indices, 4)))
        return CA_ERR_ALIGN;
    return ca::launch_build_tables_bits(mask_bits, B, H_q, nQ, nKVmax, group, tables, counts,
                                        indptr, indices, false,
                                        static_cast<cudaStream_t>(stream));
}

int ca_build_kv_pages(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                      int32_t *tables, int32_t *counts, int32_t *kv_indptr, int32_t *kv_indices,
                      void *stream) {
    if (!kv_indptr || !kv_indices) return CA_ERR_INVALID_ARG;
    if (!mask || !tables || !counts) return CA_ERR_INVALID_ARG;
    if (B <= 0 || H_q <= 0 || nQ <= 0 || nKVmax <= 0 || group <= 0) return CA_ERR_INVALID_ARG;
    if (H_q % group != 0) return CA_ERR_SHAPE;
    if ((long long)B * H_q * nQ * nKVmax >= (1LL << 40)) return CA_ERR_SHAPE;
    if ((long long)B * (H_q / group) * nKVmax >= (1LL << 31)) return CA_ERR_SHAPE;
    if (!aligned(tables, 4) || !aligned(counts, 4) || !aligned(kv_indptr, 4) ||
        !aligned(kv_indices, 4))
        return CA_ERR_ALIGN;
    return ca::launch_build_tables(mask, B, H_q, nQ, nKVmax, group, tables, counts, kv_indptr,
                                   kv_indices, true, static_cast<cudaStream_t>(stream));
}

int ca_paged_chunk_attention(const void *Q, const void *K, const void *V,
                             const int32_t *kv_indptr, const int32_t *kv_indices, long long nnz,
                             const int32_t *chunk_start, const int32_t *chunk_len, int B, int H_q,
                             int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                             float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
    if (!kv_indptr || !kv_indices || nnz < 0) return CA_ERR_INVALID_ARG;
    const int st = check_attention(Q, K, V, kv_indices, kv_indptr, false, chunk_start, B, H_q,
                                   H_kv, C, L_max, D, blk, scale, O, LSE, workspace,
                                   workspace_bytes, chunk_len);
    if (st != CA_OK) return st;
    ca::AttnArgs a{Q, K, V, kv_indices, nullptr, chunk_start, B, H_q, H_kv, C, L_max, D, blk,
                   scale, O, LSE, workspace, workspace_bytes};
    a.kv_indptr = kv_indptr;
    a.nnz = nnz;
    a.chunk_len = chunk_len;
    return ca::launch_chunk_attention(a, ca::kModeTables, static_cast<cudaStream_t>(stream));
}

int ca_chunk_attention_fp8(const void *Q8, const void *K8, const void *V8, float q_descale,
                           float k_descale, float v_descale, const int32_t *tables,
                           const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                           int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                           float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
    const bool dense = tables == nullptr;
    if (dense && counts) return CA_ERR_INVALID_ARG;
    const int st = check_attention(Q8, K8, V8, tables, counts, dense, chunk_start, B, H_q, H_kv,
                                   C, L_max, D, blk, scale, O, LSE, workspace, workspace_bytes);
    if (st != CA_OK) return st;
    for (float d : {q_descale, k_descale, v_descale})
        if (!(d > 0.0f) || !isfinite(d)) return CA_ERR_INVALID_ARG;
    if (D != 128) return CA_ERR_UNSUPPORTED;
    ca::AttnArgs a{Q8, K8, V8, tables, counts, chunk_start, B, H_q, H_kv, C, L_max, D, blk,
                   scale, O, LSE, workspace, workspace_bytes};
    a.fp8 = true;
    a.descale[0] = q_descale;
    a.descale[1] = k_descale;
    a.descale[2] = v_descale;
    return ca::launch_chunk_attention(a, dense ? ca::kModeDense : ca::kModeTables,
                                      static_cast<cudaStream_t>(stream));
}

int ca_chunk_attention(const void *Q, const void *K, const void *V, const int32_t *tables,
                       const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                       int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                       float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
    const int st = check_attention(Q, K, V, tables, counts, false, chunk_start, B, H_q, H_kv, C,
                                   L_max, D, blk, scale, O, LSE, workspace, workspace_bytes);
    if (st != CA_OK) return st;
    ca::AttnArgs a{Q, K, V, tables, counts, chunk_start, B, H_q, H_kv, C, L_max, D, blk,
                   scale, O, LSE, workspace, workspace_bytes};
    return ca::launch_chunk_attention(a, ca::kModeTables, static_cast<cudaStream_t>(stream));
}

int ca_dense_chunk_attention(const void *Q, const void *K, const void *V,
                             const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                             int L_max, int D, int blk, float scale, void *O, float *LSE,
                             void *workspace, size_t workspace_bytes, void *stream) {
    const int st = check_attention(Q, K, V, nullptr, nullptr, true, chunk_start, B, H_q, H_kv, C,
                                   L_max, D, blk, scale, O, LSE, workspace, workspace_bytes);
    if (st != CA_OK) return st;
    ca::AttnArgs a{Q, K, V, nullptr, nullptr, chunk_start, B, H_q, H_kv, C, L_max, D, blk,
                   scale, O, LSE, workspace, workspace_bytes};
    return ca::launch_chunk_attention(a, ca::kModeDense, static_cast<cudaStream_t>(stream));
}

int ca_compact_kv_blocks(const void *K, const void *V, const int32_t *tables,
                         const int32_t *counts, int B, int H_kv, int L_max, int D, int blk,
                         void *Kc, void *Vc, void *stream) {
    if (!K || !V || !tables || !counts || !Kc || !Vc) return CA_ERR_INVALID_ARG;
    if (B <= 0 || H_kv <= 0 || L_max <= 0 || D <= 0 || blk <= 0) return CA_ERR_INVALID_ARG;
    if (L_max % blk != 0) return CA_ERR_SHAPE;
    if (!(D == 64 || D == 128) || !(blk == 64 || blk == 128)) return CA_ERR_UNSUPPORTED;
    if ((long long)B * H_kv * L_max >= (1LL << 31)) return CA_ERR_SHAPE;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Kc, 16) || !aligned(Vc, 16) ||
        !aligned(tables, 4) || !aligned(counts, 4))
        return CA_ERR_ALIGN;
    return ca::launch_compact_kv(K, V, tables, counts, B, H_kv, L_max, D, blk, Kc, Vc,
                                 static_cast<cudaStream_t>(stream));
}

int ca_compacted_chunk_attention(const void *Q, const void *Kc, const void *Vc,
                                 const int32_t *tables, const int32_t *counts,
                                 const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                                 int L_max, int D, int blk, float scale, void *O, float *LSE,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    const int st = check_attention(Q, Kc, Vc, tables, counts, false, chunk_start, B, H_q, H_kv,
                                   C, L_max, D, blk, scale, O, LSE, workspace, workspace_bytes);
    if (st != CA_OK) return st;
    ca::AttnArgs a{Q, Kc, Vc, tables, counts, chunk_start, B, H_q, H_kv, C, L_max, D, blk,
                   scale, O, LSE, workspace, workspace_bytes};
    return ca::launch_chunk_attention(a, ca::kModeCompact, static_cast<cudaStream_t>(stream));
}

int ca_merge_attention_states_n(const void *const *O_parts, const float *const *LSE_parts, int n,
                                long long rows, int D, void *O, float *LSE, void *stream) {
    if (!O_parts || !LSE_parts || !O || n < 2 || rows < 0 || D <= 0) return CA_ERR_INVALID_ARG;
    if (n > ca::kMaxMergeParts) return CA_ERR_UNSUPPORTED;
    if (D % 8 != 0) return CA_ERR_SHAPE;
    if (D > 2048) return CA_ERR_UNSUPPORTED;
    for (int i = 0; i < n; ++i) {
        if (!O_parts[i] || !LSE_parts[i]) return CA_ERR_INVALID_ARG;
        if (!aligned(O_parts[i], 16) || !aligned(LSE_parts[i], 4)) return CA_ERR_ALIGN;
    }
    if (!aligned(O, 16) || (LSE && !aligned(LSE, 4))) return CA_ERR_ALIGN;
    return ca::launch_merge_states(O_parts, LSE_parts, n, rows, D, O, LSE,
                                   static_cast<cudaStream_t>(stream));
}

int ca_merge_attention_states(const void *O_a, const float *LSE_a, const void *O_b,
                              const float *LSE_b, long long rows, int D, void *O, float *LSE,
                              void *stream) {
    const void *o[2] = {O_a, O_b};
    const float *l[2] = {LSE_a, LSE_b};
    return ca_merge_attention_states_n(o, l, 2, rows, D, O, LSE, stream);
}

int ca_tile_span(int blk) {
    return (blk == 64 || blk == 128) ? ca::kTileItemRows / blk : 0;
}

int ca_build_tile_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int blk,
                         int32_t *tables, int32_t *counts, void *stream) {
    if (!mask || !tables || !counts) return CA_ERR_INVALID_ARG;
    if (B <= 0 || H_q <= 0 || nQ <= 0 || nKVmax <= 0 || blk <= 0) return CA_ERR_INVALID_ARG;
    const int span = ca_tile_span(blk);
    if (span == 0) return CA_ERR_UNSUPPORTED;
    if (nKVmax >= (1 << ca::kSpanEntryBits)) return CA_ERR_SHAPE;
    const long long nS = (nQ + span - 1) / span;
    if ((long long)B * H_q * nQ * nKVmax >= (1LL << 40)) return CA_ERR_SHAPE;
    if ((long long)B * H_q * nS >= (1LL << 31)) return CA_ERR_SHAPE;
    if (!aligned(tables, 4) || !aligned(counts, 4)) return CA_ERR_ALIGN;
    return ca::launch_tile_tables(mask, B, H_q, nQ, nKVmax, span, tables, counts,
                                  static_cast<cudaStream_t>(stream));
}

int ca_tile_chunk_attention(const void *Q, const void *K, const void *V, const int32_t *tables,
                            const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                            int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                            float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
    const int st = check_attention(Q, K, V, tables, counts, false, chunk_start, B, H_q, H_kv, C,
                                   L_max, D, blk, scale, O, LSE, workspace, workspace_bytes);
    if (st != CA_OK) return st;
    if (L_max / blk >= (1 << ca::kSpanEntryBits)) return CA_ERR_SHAPE;
    ca::AttnArgs a{Q, K, V, tables, counts, chunk_start, B, H_q, H_kv, C, L_max, D, blk,
                   scale, O, LSE, workspace, workspace_bytes};
    return ca::launch_chunk_attention(a, ca::kModePerTile, static_cast<cudaStream_t>(stream));
}

int ca_read_device_status(const void *workspace, void *stream) {
    if (!workspace) return CA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return CA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CA_ERR_CUDA;
    if (word & ca::kDevErrTable) return CA_ERR_TABLE;
    if (word & ca::kDevErrTimeout) return CA_ERR_TIMEOUT;
    return CA_OK;
}

}  // extern "C"
