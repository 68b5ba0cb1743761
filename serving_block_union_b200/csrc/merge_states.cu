// merge_states.cu — merge of attention results over disjoint key sets.
//
// Split-KV execution (not on the CompactAttention pages: the standard way to
// spread one query row's attention over several segments of its KV blocks)
// leaves, per segment i, an output O_i normalised over its own keys and the
// log-sum-exp LSE_i of its scores. Attention over the union of the key sets
// is then
//     LSE = ln sum_i exp(LSE_i),   O = sum_i exp(LSE_i - LSE) O_i,
// evaluated here with the largest LSE_i subtracted first. The chunk kernel
// does this merge itself for the segments of one launch; this kernel is the
// user-facing form, for results produced by separate calls (other tables,
// other streams, other GPUs).
//
// Pure HBM streaming: per row, n * D bf16 (+ n fp32) in and D bf16 (+ one
// fp32) out. A row is handled by D / 8 threads, 16 bytes each; a 256-thread
// CTA covers 256 / (D / 8) rows per pass; grid-stride over rows with a grid
// of a few CTAs per SM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ca_internal.h"

namespace ca {

namespace {

constexpr int kMergeThreads = 256;

struct MergeParts {
    const uint4 *O[kMaxMergeParts];
    const float *L[kMaxMergeParts];
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h;
        memcpy(&h, &w[i], 4);
        const float2 p = __bfloat1622float2(h);
        f[2 * i] = p.x;
        f[2 * i + 1] = p.y;
    }
}

__device__ __forceinline__ uint4 f32_to_bf16x8(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        memcpy(&w[i], &h, 4);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// n parts (2 <= n <= NP <= kMaxMergeParts; NP is a compile-time bound so that
// the common two-part merge keeps few registers and many CTAs per SM).
// vpr = D / 8 vectors per row; rpp rows per pass of the CTA. The pass loop is
// uniform over the CTA so that, when the output LSE aliases an input LSE, a
// barrier separates every thread's reads of the row's LSE_i from the single
// store of its merged LSE.
template <int NP>
__global__ void __launch_bounds__(kMergeThreads)
    merge_states_kernel(MergeParts parts, int n, long long rows, int vpr, int rpp,
                        uint4 *O, float *LSE, int lse_alias) {
    const int rsub = threadIdx.x / vpr;
    const int c = threadIdx.x - rsub * vpr;
    const long long step = (long long)gridDim.x * rpp;
    for (long long base = (long long)blockIdx.x * rpp; base < rows; base += step) {
        const long long r = base + rsub;
        const bool active = rsub < rpp && r < rows;
        float lse = -INFINITY;
        if (active) {
            float l[NP];
            float m = -INFINITY;
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                l[i] = i < n ? __ldg(parts.L[i] + r) : -INFINITY;
                m = fmaxf(m, l[i]);
            }
            uint4 v[NP];
            const size_t off = (size_t)r * vpr + c;
#pragma unroll
            for (int i = 0; i < NP; ++i)
                if (i < n) v[i] = __ldcs(parts.O[i] + off);
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
            if (m != -INFINITY) {
                float w[NP];
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    w[i] = i < n ? expf(l[i] - m) : 0.f;
                    s += w[i];
                }
                const float inv = 1.f / s;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    if (i < n) {
                        float f[8];
                        bf16x8_to_f32(v[i], f);
                        const float wi = w[i] * inv;
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wi, f[e], acc[e]);
                    }
                }
                lse = m + logf(s);
            }
            __stcs(O + off, f32_to_bf16x8(acc));
        }
        if (LSE) {
            if (lse_alias) __syncthreads();
            if (active && c == 0) LSE[r] = lse;
        }
    }
}

}  // namespace

int launch_merge_states(const void *const *O_parts, const float *const *LSE_parts, int n,
                        long long rows, int D, void *O, float *LSE, cudaStream_t stream) {
    if (rows == 0) return CA_OK;
    MergeParts p{};
    int alias = 0;
    for (int i = 0; i < n; ++i) {
        p.O[i] = static_cast<const uint4 *>(O_parts[i]);
        p.L[i] = LSE_parts[i];
        if (LSE && LSE_parts[i] == LSE) alias = 1;
    }
    const int vpr = D / 8;
    const int rpp = kMergeThreads / vpr;
    const long long passes = (rows + rpp - 1) / rpp;
    const long long cap = (long long)current_sm_count() * 8;
    const unsigned grid = static_cast<unsigned>(passes < cap ? passes : cap);
    if (n == 2)
        merge_states_kernel<2><<<grid, kMergeThreads, 0, stream>>>(
            p, n, rows, vpr, rpp, static_cast<uint4 *>(O), LSE, alias);
    else
        merge_states_kernel<kMaxMergeParts><<<grid, kMergeThreads, 0, stream>>>(
            p, n, rows, vpr, rpp, static_cast<uint4 *>(O), LSE, alias);
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

}  // namespace ca
