// compact_kv.cu — the explicit-compaction ablation's copy step.
//
// The CompactAttention pages contrast zero-copy paged execution with methods
// that gather the selected KV entries into a compact buffer before dense
// attention ("Experimental results": zero-copy beats explicit KV compaction
// even with the metadata build counted). This kernel is that gather at block
// granularity, so the two can be timed on the same tables: block
// tables[b, g, t] of the cache is copied to rows [t * blk, (t + 1) * blk) of
// the compact buffers. Table entries outside [0, L_max / blk) leave their
// destination rows zero.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ca_internal.h"

namespace ca {

namespace {

// One CTA per (b, g, t); 16-byte vector copies of the block's K and V rows.
__global__ void __launch_bounds__(256)
    compact_kv_kernel(const uint4 *__restrict__ K, const uint4 *__restrict__ V,
                      const int32_t *__restrict__ tables, const int32_t *__restrict__ counts,
                      int H_kv, int L_max, int D, int blk, uint4 *__restrict__ Kc,
                      uint4 *__restrict__ Vc) {
    const int nKVmax = L_max / blk;
    const int t = blockIdx.x;
    const int bg = blockIdx.y;
    const int cnt = counts[bg];
    if (cnt < 0 || cnt > nKVmax || t >= cnt) return;
    const int j = tables[(size_t)bg * nKVmax + t];
    const size_t vec_per_block = (size_t)blk * D / 8;  // 8 bf16 per 16 bytes
    const size_t plane = (size_t)L_max * D / 8;
    uint4 *kd = Kc + (size_t)bg * plane + (size_t)t * vec_per_block;
    uint4 *vd = Vc + (size_t)bg * plane + (size_t)t * vec_per_block;
    if (j < 0 || j >= nKVmax) {
        for (size_t i = threadIdx.x; i < vec_per_block; i += blockDim.x) {
            kd[i] = make_uint4(0, 0, 0, 0);
            vd[i] = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const uint4 *ks = K + (size_t)bg * plane + (size_t)j * vec_per_block;
    const uint4 *vs = V + (size_t)bg * plane + (size_t)j * vec_per_block;
    for (size_t i = threadIdx.x; i < vec_per_block; i += blockDim.x) {
        kd[i] = __ldg(ks + i);
        vd[i] = __ldg(vs + i);
    }
}

}  // namespace

int launch_compact_kv(const void *K, const void *V, const int32_t *tables, const int32_t *counts,
                      int B, int H_kv, int L_max, int D, int blk, void *Kc, void *Vc,
                      cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(L_max / blk), static_cast<unsigned>(B * H_kv));
    compact_kv_kernel<<<grid, 256, 0, stream>>>(
        static_cast<const uint4 *>(K), static_cast<const uint4 *>(V), tables, counts, H_kv, L_max,
        D, blk, static_cast<uint4 *>(Kc), static_cast<uint4 *>(Vc));
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

}  // namespace ca
