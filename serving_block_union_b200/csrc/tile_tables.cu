// tile_tables.cu — span tables for the per-tile block-sparse ablation path.
//
// CompactAttention pages, "Problem" (block-sparse kernels in the Q << KV
// regime) and the efficiency ablation in "Experimental results": the baseline
// that executes the 2D mask directly, every head and Q-block with its own KV
// blocks, no union. The attention kernel's work item covers 256 chunk rows of
// one head (two 128-row tiles), i.e. a span of 256 / blk Q-blocks, so the table
// of an item lists, ascending, every KV block that some Q-block of its span
// selects, with one bit per Q-block saying which of them use it:
//     entry = j | (bit u set iff Q-block span * s + u selects j) << 24.
// The rows of a tile that do not select a listed block skip it; executed as a
// whole, the result is per-tile block-sparse attention exactly.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ca_internal.h"

namespace ca {

namespace {

constexpr int kWarpsPerCta = 8;

// One warp per (b, h, span); lanes sweep the KV blocks 32 at a time and
// compact the selected ones with a ballot.
__global__ void __launch_bounds__(32 * kWarpsPerCta)
    tile_span_tables_kernel(const uint8_t *__restrict__ mask, int n_items, int nQ, int nKVmax,
                            int span, int nS, int32_t *__restrict__ tables,
                            int32_t *__restrict__ counts) {
    const int item = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (item >= n_items) return;
    const int s = item % nS;
    const int bh = item / nS;
    const int q0 = s * span;
    const int nrows = min(span, nQ - q0);
    const uint8_t *rows = mask + ((size_t)bh * nQ + q0) * (size_t)nKVmax;
    int32_t *T = tables + (size_t)item * nKVmax;
    int n = 0;
    for (int j0 = 0; j0 < nKVmax; j0 += 32) {
        const int j = j0 + lane;
        int bits = 0;
        if (j < nKVmax) {
            for (int u = 0; u < nrows; ++u)
                bits |= (__ldg(rows + (size_t)u * nKVmax + j) != 0 ? 1 : 0) << u;
        }
        const unsigned sel = __ballot_sync(0xffffffffu, bits != 0);
        if (bits) T[n + __popc(sel & ((1u << lane) - 1u))] = j | (bits << 24);
        n += __popc(sel);
    }
    for (int t = n + lane; t < nKVmax; t += 32) T[t] = -1;
    if (lane == 0) counts[item] = n;
}

// The same with 32-bit loads: lane l reads blocks 4l .. 4l+3 of every mask row
// of the span as one word (rows 4-byte aligned: nKVmax % 4 == 0), and a warp
// scan of the per-lane counts places the entries, 128 blocks per step.
__global__ void __launch_bounds__(32 * kWarpsPerCta)
    tile_span_tables_x4_kernel(const uint8_t *__restrict__ mask, int n_items, int nQ,
                               int nKVmax, int span, int nS, int32_t *__restrict__ tables,
                               int32_t *__restrict__ counts) {
    const int item = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (item >= n_items) return;
    const int s = item % nS;
    const int bh = item / nS;
    const int q0 = s * span;
    const int nrows = min(span, nQ - q0);
    const uint32_t *rows =
        reinterpret_cast<const uint32_t *>(mask + ((size_t)bh * nQ + q0) * (size_t)nKVmax);
    const int words = nKVmax >> 2;
    int32_t *T = tables + (size_t)item * nKVmax;
    int n = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        int bits[4] = {0, 0, 0, 0};  // Q-block bits of blocks 4w .. 4w+3
        if (w < words) {
            for (int u = 0; u < nrows; ++u) {
                const uint32_t v = __ldg(rows + (size_t)u * words + w);
#pragma unroll
                for (int k = 0; k < 4; ++k) bits[k] |= (((v >> (8 * k)) & 0xFFu) != 0 ? 1 : 0) << u;
            }
        }
        const int mine = (bits[0] != 0) + (bits[1] != 0) + (bits[2] != 0) + (bits[3] != 0);
        int incl = mine;  // inclusive warp scan of the per-lane counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int pos = n + incl - mine;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (bits[k]) T[pos++] = (4 * w + k) | (bits[k] << 24);
        n += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int t = n + lane; t < nKVmax; t += 32) T[t] = -1;
    if (lane == 0) counts[item] = n;
}

}  // namespace

int launch_tile_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int span,
                       int32_t *tables, int32_t *counts, cudaStream_t stream) {
    const int nS = (nQ + span - 1) / span;
    const int n_items = B * H_q * nS;
    const unsigned grid = static_cast<unsigned>((n_items + kWarpsPerCta - 1) / kWarpsPerCta);
    if (nKVmax % 4 == 0 && (reinterpret_cast<uintptr_t>(mask) & 3u) == 0)
        tile_span_tables_x4_kernel<<<grid, 32 * kWarpsPerCta, 0, stream>>>(
            mask, n_items, nQ, nKVmax, span, nS, tables, counts);
    else
        tile_span_tables_kernel<<<grid, 32 * kWarpsPerCta, 0, stream>>>(mask, n_items, nQ, nKVmax,
                                                                        span, nS, tables, counts);
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

}  // namespace ca
