// build_tables.cu — Block-Union KV table construction on the GPU.
//
// CompactAttention pages, "Methodology", selection stage: the per-head 2D block
// mask is reduced by a Q-block union (over the chunk's query blocks) and an
// intra-group union (over the query heads sharing a KV head) into the minimal
// per-(batch, KV-group) table T_{b,g}; the CSR form is the kv_indptr /
// kv_indices metadata handed to the paged kernel.
//
// Three forms. With few (b, g), each is spread over a cluster of CTAs (the
// cluster kernel below). With many, one CTA per (b, g) reads the group's
// contiguous G * nQ mask rows with bulk copies into shared memory (the bulk
// kernel below). Where neither applies (rows not 16-byte multiples, or wider
// than the bulk form takes), one CTA per (b, g) reads with register loads:
// thread (rg, c) owns 16 consecutive KV blocks (chunk c) and ORs 16-byte
// vectors of the mask rows rg, rg + RG, ... of the group's rows (coalesced:
// consecutive threads read consecutive 16-byte words of a row). Row groups
// are OR-combined through shared memory, every chunk turns its 16 bytes into
// a 16-bit set, and a block-wide exclusive prefix sum of the popcounts (warp
// shuffles + one shared-memory pass) gives each chunk its write offset, so
// the table comes out ascending without a sort.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <type_traits>

#include "ca_internal.h"
#include "sm100_ptx.cuh"

namespace ca {

namespace {

constexpr int kMaxThreads = 1024;

__device__ __forceinline__ uint32_t nonzero_nibble(uint32_t w) {
    // 4 bits: bit k = (byte k of w != 0)
    const uint32_t m = __vcmpne4(w, 0u);  // 0xFF in every nonzero byte
    return ((m >> 7) & 1u) | ((m >> 14) & 2u) | ((m >> 21) & 4u) | ((m >> 28) & 8u);
}

__device__ __forceinline__ uint32_t nonzero_bytes16(uint4 v) {
    // bit k of the result = (byte k of v != 0), bytes in memory order
    return nonzero_nibble(v.x) | (nonzero_nibble(v.y) << 4) | (nonzero_nibble(v.z) << 8) |
           (nonzero_nibble(v.w) << 12);
}

// Block-wide exclusive scan of `x` over the first `n_active` threads (a multiple
// of 32). Returns the exclusive prefix; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int x, int tid, int n_active, int *warp_sums,
                                                    int *total) {
    const int lane = tid & 31, warp = tid >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    const int n_warps = n_active >> 5;
    if (warp == 0) {
        int s = lane < n_warps ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < n_warps) warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int warp_base = warp > 0 ? warp_sums[warp - 1] : 0;
    *total = warp_sums[n_warps - 1];
    return warp_base + incl - x;
}

// chp: chunk threads per row group (multiple of 32), rg: row groups,
// blockDim.x = chp * rg. vec: mask rows are 16-byte aligned and nKVmax % 16 == 0.
__global__ void __launch_bounds__(kMaxThreads)
    union_tables_kernel(const uint8_t *__restrict__ mask, int H_q, int nQ, int nKVmax, int G,
                        int chp, int rg, int vec, int32_t *__restrict__ tables,
                        int32_t *__restrict__ counts) {
    extern __shared__ uint32_t sm_bits[];  // [rg][chp]
    __shared__ int warp_sums[32];
    __shared__ int s_base;

    const int bg = blockIdx.x;
    const int H_kv = H_q / G;
    const int b = bg / H_kv, g = bg % H_kv;
    const int tid = threadIdx.x;
    const int c_local = tid % chp, r_grp = tid / chp;
    const int n_rows = G * nQ;
    const int n_chunks = (nKVmax + 15) >> 4;
    const uint8_t *base = mask + ((size_t)b * H_q + (size_t)g * G) * nQ * (size_t)nKVmax;
    int32_t *T = tables + (size_t)bg * nKVmax;

    if (tid == 0) s_base = 0;
    __syncthreads();

    for (int round0 = 0; round0 < n_chunks; round0 += chp) {
        const int chunk = round0 + c_local;
        const int j0 = chunk << 4;
        uint32_t bits = 0;
        if (chunk < n_chunks) {
            if (vec) {
                uint4 acc = make_uint4(0, 0, 0, 0);
#pragma unroll 8
                for (int row = r_grp; row < n_rows; row += rg) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
                        base + (size_t)row * nKVmax + j0));
                    acc.x |= v.x; acc.y |= v.y; acc.z |= v.z; acc.w |= v.w;
                }
                bits = nonzero_bytes16(acc);
            } else {
                const int nb = min(16, nKVmax - j0);
                for (int row = r_grp; row < n_rows; row += rg) {
                    const uint8_t *p = base + (size_t)row * nKVmax + j0;
                    for (int k = 0; k < nb; ++k) bits |= (uint32_t)(__ldg(p + k) != 0) << k;
                }
            }
        }
        sm_bits[r_grp * chp + c_local] = bits;
        __syncthreads();
        int total = 0;
        if (r_grp == 0) {
            for (int q = 1; q < rg; ++q) bits |= sm_bits[q * chp + c_local];
        }
        // every thread takes part in the scan (barriers inside); only row group 0 counts
        const int cnt = (r_grp == 0) ? __popc(bits) : 0;
        const int off = block_exclusive_scan(cnt, tid, chp * rg, warp_sums, &total);
        if (r_grp == 0 && bits) {
            int w = s_base + off;
            uint32_t m = bits;
            while (m) {
                const int k = __ffs(m) - 1;
                T[w++] = j0 + k;
                m &= m - 1;
            }
        }
        __syncthreads();
        if (tid == 0) s_base += total;
        __syncthreads();
    }
    const int n = s_base;
    for (int t = n + tid; t < nKVmax; t += blockDim.x) T[t] = -1;
    if (tid == 0) counts[bg] = n;
}

// The same union from a bit-packed mask: uint32 words [B, H_q, nQ, nW],
// nW = ceil(nKVmax / 32), bit k of word w selects KV block 32 * w + k (bits
// at or past nKVmax are ignored). Thread (r_grp, w) ORs word w of rows
// r_grp, r_grp + rg, ...; the row groups combine through shared memory and a
// block-wide scan of the popcounts places each word's blocks.
__global__ void __launch_bounds__(kMaxThreads)
    union_bits_kernel(const uint32_t *__restrict__ mask, int H_q, int nQ, int nKVmax, int G,
                      int wpr, int rg, int32_t *__restrict__ tables,
                      int32_t *__restrict__ counts) {
    extern __shared__ uint32_t sm_words[];  // [rg][wpr]
    __shared__ int warp_sums[32];
    __shared__ int s_base;

    const int bg = blockIdx.x;
    const int H_kv = H_q / G;
    const int b = bg / H_kv, g = bg % H_kv;
    const int tid = threadIdx.x;
    const int w_local = tid % wpr, r_grp = tid / wpr;
    const int n_rows = G * nQ;
    const int nW = (nKVmax + 31) >> 5;
    const uint32_t *base = mask + ((size_t)b * H_q + (size_t)g * G) * nQ * (size_t)nW;
    int32_t *T = tables + (size_t)bg * nKVmax;

    if (tid == 0) s_base = 0;
    __syncthreads();

    for (int round0 = 0; round0 < nW; round0 += wpr) {
        const int w = round0 + w_local;
        uint32_t bits = 0;
        if (w < nW) {
#pragma unroll 8
            for (int row = r_grp; row < n_rows; row += rg) bits |= __ldg(base + (size_t)row * nW + w);
            const int valid = nKVmax - (w << 5);  // blocks this word can name
            if (valid < 32) bits &= (1u << valid) - 1u;
        }
        sm_words[r_grp * wpr + w_local] = bits;
        __syncthreads();
        int total = 0;
        if (r_grp == 0) {
            for (int q = 1; q < rg; ++q) bits |= sm_words[q * wpr + w_local];
        }
        const int cnt = (r_grp == 0) ? __popc(bits) : 0;
        const int off = block_exclusive_scan(cnt, tid, wpr * rg, warp_sums, &total);
        if (r_grp == 0 && bits) {
            int o = s_base + off;
            uint32_t m = bits;
            while (m) {
                const int k = __ffs(m) - 1;
                T[o++] = (w << 5) + k;
                m &= m - 1;
            }
        }
        __syncthreads();
        if (tid == 0) s_base += total;
        __syncthreads();
    }
    const int n = s_base;
    for (int t = n + tid; t < nKVmax; t += blockDim.x) T[t] = -1;
    if (tid == 0) counts[bg] = n;
}

// Bulk-copy form of the one-CTA-per-(b, g) union, for many (b, g) (a batch
// of sequences). A (b, g)'s G * nQ mask rows are contiguous in memory, so the
// CTA reads them as pieces of `rpp` whole rows, one cp.async.bulk copy per
// piece into a two-stage shared-memory ring (completion counted in bytes on
// the stage's mbarrier): two pieces, up to 64 KB, in flight per CTA without a
// register per byte, against a few loads per thread in the register form.
// Thread t ORs units t, t + 256, ... (16-byte vectors of a byte mask, or
// 32-bit words of a bit-packed one) over every row of every piece; a
// block-wide scan of the units' popcounts, in unit order, places each
// unit's entries (ascending without a sort). Every wait is bounded: a piece
// that never lands (not seen in practice) leaves the CTA's count at -1,
// which the attention kernels reject, after the copies it issued are drained.
constexpr int kBulkThreads = 256;
constexpr int kBulkPieceBytes = 32 * 1024;  // one stage of the ring
constexpr int kBulkMaxUnitsPerThread = 4;   // units per row <= 1024

__device__ __forceinline__ void or_into(uint4 &a, const uint4 &v) {
    a.x |= v.x;
    a.y |= v.y;
    a.z |= v.z;
    a.w |= v.w;
}
__device__ __forceinline__ void or_into(uint32_t &a, uint32_t v) { a |= v; }

template <bool BITS, int UPT>
__global__ void __launch_bounds__(kBulkThreads)
    union_tables_bulk_kernel(const void *__restrict__ mask, int H_q, int nQ, int nKVmax, int G,
                             int rpp, int32_t *__restrict__ tables,
                             int32_t *__restrict__ counts) {
    using Unit = typename std::conditional<BITS, uint32_t, uint4>::type;
    constexpr int UB = BITS ? 32 : 16;  // KV blocks per unit
    extern __shared__ uint8_t bulk_raw[];
    __shared__ uint64_t full[2];
    __shared__ int warp_sums[32];
    __shared__ int s_abort;

    const int bg = blockIdx.x, tid = threadIdx.x;
    const int H_kv = H_q / G;
    const int b = bg / H_kv, g = bg % H_kv;
    const int n_rows = G * nQ;
    const int n_units = (nKVmax + UB - 1) / UB;
    const size_t row_bytes = (size_t)n_units * sizeof(Unit);
    const uint8_t *src = static_cast<const uint8_t *>(mask) +
                         ((size_t)b * H_q + (size_t)g * G) * nQ * row_bytes;
    uint8_t *stage0 = bulk_raw + ((128u - (smem_u32(bulk_raw) & 127u)) & 127u);
    const uint32_t stage_bytes = (uint32_t)((size_t)rpp * row_bytes);
    const int n_pieces = (n_rows + rpp - 1) / rpp;
    int32_t *T = tables + (size_t)bg * nKVmax;
    const AbortState ab{&s_abort, nullptr};  // a timeout shows as count -1

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // thread 0 issues piece p (rows [p * rpp, ...)) into stage p & 1
    int issued = 0;
    auto issue = [&](int p) {
        const int r0 = p * rpp;
        const uint32_t bytes = (uint32_t)((size_t)min(rpp, n_rows - r0) * row_bytes);
        uint64_t *bar = &full[p & 1];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(stage0 + (p & 1) * stage_bytes, src + (size_t)r0 * row_bytes, bytes, bar);
        issued = p + 1;
    };
    if (tid == 0) {
        issue(0);
        if (n_pieces > 1) issue(1);
    }
    Unit acc[UPT];
#pragma unroll
    for (int k = 0; k < UPT; ++k) acc[k] = Unit{};
    int landed = 0;  // pieces this thread saw complete
    for (int p = 0; p < n_pieces; ++p) {
        // every thread reaches every barrier below, whether its wait held or not
        if (mbar_wait(&full[p & 1], (p >> 1) & 1, ab)) {
            landed = p + 1;
            const uint8_t *st = stage0 + (p & 1) * stage_bytes;
            const int nr = min(rpp, n_rows - p * rpp);
#pragma unroll 4
            for (int r = 0; r < nr; ++r) {
                const Unit *row = reinterpret_cast<const Unit *>(st + (size_t)r * row_bytes);
#pragma unroll
                for (int k = 0; k < UPT; ++k) {
                    const int u = tid + k * kBulkThreads;
                    if (u < n_units) or_into(acc[k], row[u]);
                }
            }
        }
        __syncthreads();  // stage p & 1 is free again
        if (tid == 0 && p + 2 < n_pieces && !s_abort) issue(p + 2);
    }
    if (s_abort) {  // the barrier above made the flag visible to every thread
        if (tid == 0) {
            for (int p = landed; p < issued; ++p) mbar_wait_drain(&full[p & 1], (p >> 1) & 1);
            counts[bg] = -1;
        }
        return;
    }
    // The table is assembled in the ring's shared memory (free now: every
    // piece has been consumed) where it fits, then written out with
    // consecutive threads on consecutive entries; a unit's entries written
    // straight to global memory would be one scattered 4-byte store each.
    const bool in_smem = (size_t)nKVmax * 4 <= (n_pieces > 1 ? 2u : 1u) * (size_t)stage_bytes;
    int32_t *dst = in_smem ? reinterpret_cast<int32_t *>(stage0) : T;
    int run = 0;
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
        const int u = tid + k * kBulkThreads;
        uint32_t bits = 0;
        if (u < n_units) {
            if constexpr (BITS) {
                bits = acc[k];
                const int valid = nKVmax - u * 32;  // blocks this word can name
                if (valid < 32) bits &= (1u << valid) - 1u;
            } else {
                bits = nonzero_bytes16(acc[k]);
            }
        }
        int tot = 0;
        const int off = block_exclusive_scan(__popc(bits), tid, kBulkThreads, warp_sums, &tot);
        int w = run + off;
        const int j0 = u * UB;
        while (bits) {
            dst[w++] = j0 + __ffs(bits) - 1;
            bits &= bits - 1;
        }
        run += tot;
        __syncthreads();  // warp_sums is reused by the next round; dst complete
    }
    if (in_smem) {
        for (int t = tid; t < nKVmax; t += kBulkThreads) T[t] = t < run ? dst[t] : -1;
    } else {
        for (int t = run + tid; t < nKVmax; t += kBulkThreads) T[t] = -1;
    }
    if (tid == 0) counts[bg] = run;
}

// Cluster form of the same union: a (b, g) row set is spread over a cluster of
// kClusterCtas CTAs, CTA q taking units [q * upc, (q + 1) * upc) of the KV
// range (a unit is 16 blocks of a byte mask, one 16-byte load per row, or 32
// blocks of a bit mask, one 32-bit word per row). Each CTA ORs its units over
// the group's G * nQ rows (one load per (row, unit) pair, consecutive threads
// on consecutive units of a row, folded into shared memory by atomicOr), scans
// its popcounts, and writes its entry total into every CTA's shared memory
// (distributed shared memory stores); after one cluster barrier each CTA has
// all the totals, which give its write offset and the table length. So one
// (b, g) is read by kClusterCtas SMs at once instead of one, and the table
// still comes out ascending without a sort.
constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = 256;
constexpr int kMaxUnitsPerCta = 1024;

template <bool BITS>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kClusterThreads)
    union_tables_cluster_kernel(const void *__restrict__ mask, int H_q, int nQ, int nKVmax, int G,
                                int upc, int32_t *__restrict__ tables,
                                int32_t *__restrict__ counts) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ uint32_t s_bits[kMaxUnitsPerCta];
    __shared__ int s_off[kMaxUnitsPerCta];
    __shared__ int warp_sums[32];
    __shared__ int s_totals[kClusterCtas];  // entry totals of every CTA of the cluster
    __shared__ int s_base, s_n;

    constexpr int UB = BITS ? 32 : 16;  // KV blocks per unit
    const int q = static_cast<int>(cluster.block_rank());
    const int bg = blockIdx.y;
    const int H_kv = H_q / G;
    const int b = bg / H_kv, g = bg % H_kv;
    const int tid = threadIdx.x;
    const int n_units = (nKVmax + UB - 1) / UB;
    const int u0 = q * upc;
    const int nu = max(0, min(upc, n_units - u0));
    const int n_rows = G * nQ;
    const size_t row0 = ((size_t)b * H_q + (size_t)g * G) * nQ;
    int32_t *T = tables + (size_t)bg * nKVmax;

    for (int u = tid; u < nu; u += kClusterThreads) s_bits[u] = 0;
    __syncthreads();
    // pass 1: the union of this CTA's units, four (row, unit) loads in flight
    // per thread before their results are folded in
    const int pairs = n_rows * nu;
    for (int p0 = tid; p0 < pairs; p0 += 4 * kClusterThreads) {
        uint32_t bits[4];
        int unit[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int p = p0 + k * kClusterThreads;
            bits[k] = 0;
            unit[k] = 0;
            if (p < pairs) {
                const int row = p / nu;
                const int u = p - row * nu;
                unit[k] = u;
                if constexpr (BITS) {
                    const int nW = n_units;
                    bits[k] = __ldg(static_cast<const uint32_t *>(mask) + (row0 + row) * nW + u0 + u);
                } else {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
                        static_cast<const uint8_t *>(mask) + (row0 + row) * (size_t)nKVmax +
                        (size_t)(u0 + u) * 16));
                    bits[k] = nonzero_bytes16(v);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (bits[k]) atomicOr(&s_bits[unit[k]], bits[k]);
    }
    __syncthreads();
    if constexpr (BITS) {
        // bits at or past nKVmax name no block
        if (tid == 0 && nu > 0) {
            const int valid = nKVmax - (u0 + nu - 1) * 32;
            if (valid < 32) s_bits[nu - 1] &= (1u << valid) - 1u;
        }
        __syncthreads();
    }
    // pass 2: CTA-local exclusive scan of the units' popcounts
    int run = 0;
    for (int r0 = 0; r0 < nu; r0 += kClusterThreads) {
        const int u = r0 + tid;
        const int c = u < nu ? __popc(s_bits[u]) : 0;
        int tot = 0;
        const int off = block_exclusive_scan(c, tid, kClusterThreads, warp_sums, &tot);
        if (u < nu) s_off[u] = run + off;
        run += tot;
        __syncthreads();  // warp_sums is reused by the next round
    }
    // publish this CTA's total into slot q of every CTA of the cluster; after
    // the barrier (release / acquire) every slot is filled and no CTA touches
    // another's shared memory again, so none has to wait for the others to
    // finish before it exits
    if (tid < kClusterCtas) *cluster.map_shared_rank(&s_totals[q], tid) = run;
    cluster.sync();
    // this CTA's offset (totals of the lower ranks) and the table length
    if (tid < 32) {
        const int t = tid < kClusterCtas ? s_totals[tid] : 0;
        int below = tid < q ? t : 0;
        int all = t;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            below += __shfl_xor_sync(0xffffffffu, below, o);
            all += __shfl_xor_sync(0xffffffffu, all, o);
        }
        if (tid == 0) {
            s_base = below;
            s_n = all;
        }
    }
    __syncthreads();
    const int base = s_base, n = s_n;
    for (int u = tid; u < nu; u += kClusterThreads) {
        uint32_t m = s_bits[u];
        int w = base + s_off[u];
        const int j0 = (u0 + u) * UB;
        while (m) {
            const int k = __ffs(m) - 1;
            T[w++] = j0 + k;
            m &= m - 1;
        }
    }
    for (int t = n + q * kClusterThreads + tid; t < nKVmax; t += kClusterCtas * kClusterThreads)
        T[t] = -1;
    if (q == 0 && tid == 0) counts[bg] = n;
}

// Units per CTA of the cluster form, or 0 where it does not apply. It pays
// only while one CTA per (b, g) leaves most SMs idle (a single sequence or a
// few): measured at 128K (G = 4, 16 Q-blocks), 8 (b, g) build in 10.8 us
// against 14.7 us with one CTA each, but 512 (b, g) take 36.6 us against 20.6.
int cluster_upc(int n_units, int n_bg) {
    if (n_bg <= 0 || n_bg > 65535 || n_bg > current_sm_count() / 4) return 0;
    const int upc = (n_units + kClusterCtas - 1) / kClusterCtas;
    return upc <= kMaxUnitsPerCta ? upc : 0;
}

// Rows per piece of the bulk form, or 0 where it does not apply (a row wider
// than a piece, more than four units per thread). Bit-packed rows are 4-byte
// multiples, so there the pieces hold a multiple of four rows and start on
// 16 bytes; the caller checks the region's own alignment. The piece count is
// the least that fits, the rows spread evenly over it.
int bulk_rpp(int n_rows, size_t row_bytes, int n_units, bool bits) {
    if (n_units > kBulkThreads * kBulkMaxUnitsPerThread || row_bytes > (size_t)kBulkPieceBytes)
        return 0;
    int rpp = (int)(kBulkPieceBytes / row_bytes);
    if (rpp >= n_rows) return n_rows;  // one piece
    if (bits) rpp &= ~3;
    if (rpp <= 0) return 0;
    const int n_pieces = (n_rows + rpp - 1) / rpp;
    int even = (n_rows + n_pieces - 1) / n_pieces;
    if (bits) even = (even + 3) & ~3;  // still <= rpp, a multiple of 4
    return even;
}

template <bool BITS, int UPT>
int launch_bulk_t(const void *mask, int B, int H_q, int nQ, int nKVmax, int group, int rpp,
                  size_t smem, int32_t *tables, int32_t *counts, cudaStream_t stream) {
    auto kern = union_tables_bulk_kernel<BITS, UPT>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        2 * kBulkPieceBytes + 128);
    });
    if (attr_err != cudaSuccess) return CA_ERR_CUDA;
    kern<<<B * (H_q / group), kBulkThreads, smem, stream>>>(mask, H_q, nQ, nKVmax, group, rpp,
                                                            tables, counts);
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

template <bool BITS>
int launch_bulk(const void *mask, int B, int H_q, int nQ, int nKVmax, int group, int rpp,
                int32_t *tables, int32_t *counts, cudaStream_t stream) {
    const int n_rows = group * nQ;
    const int n_units = BITS ? (nKVmax + 31) / 32 : nKVmax / 16;
    const size_t row_bytes = (size_t)n_units * (BITS ? 4 : 16);
    const int stages = rpp < n_rows ? 2 : 1;
    const size_t smem = (size_t)stages * rpp * row_bytes + 128;
    const int upt = (n_units + kBulkThreads - 1) / kBulkThreads;
    if (upt <= 1)
        return launch_bulk_t<BITS, 1>(mask, B, H_q, nQ, nKVmax, group, rpp, smem, tables,
                                      counts, stream);
    if (upt <= 2)
        return launch_bulk_t<BITS, 2>(mask, B, H_q, nQ, nKVmax, group, rpp, smem, tables,
                                      counts, stream);
    return launch_bulk_t<BITS, 4>(mask, B, H_q, nQ, nKVmax, group, rpp, smem, tables, counts,
                                  stream);
}

// CSR form: indptr[bg] = sum of counts before bg; indices = valid prefixes.
__global__ void __launch_bounds__(256)
    csr_kernel(const int32_t *__restrict__ tables, const int32_t *__restrict__ counts, int n_bg,
               int nKVmax, bool page_ids, int32_t *__restrict__ indptr,
               int32_t *__restrict__ indices) {
    __shared__ int red[256];
    const int bg = blockIdx.x, tid = threadIdx.x;
    int s = 0;
    for (int k = tid; k < bg; k += blockDim.x) s += counts[k];
    red[tid] = s;
    __syncthreads();
    for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
        if (tid < w) red[tid] += red[tid + w];
        __syncthreads();
    }
    const int off = red[0];
    const int n = counts[bg];
    if (tid == 0) {
        indptr[bg] = off;
        if (bg == n_bg - 1) indptr[n_bg] = off + n;
    }
    if (indices) {
        // block j of (b, g), or its global page (b * H_kv + g) * nKVmax + j
        const int32_t *T = tables + (size_t)bg * nKVmax;
        const int32_t base = page_ids ? bg * nKVmax : 0;
        for (int t = tid; t < n; t += blockDim.x) indices[off + t] = base + T[t];
    }
}

int launch_csr(const int32_t *tables, const int32_t *counts, int n_bg, int nKVmax,
               bool page_ids, int32_t *indptr, int32_t *indices, cudaStream_t stream) {
    if (!indptr) return CA_OK;
    csr_kernel<<<n_bg, 256, 0, stream>>>(tables, counts, n_bg, nKVmax, page_ids, indptr, indices);
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

}  // namespace

int launch_build_tables_bits(const uint32_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                             int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                             bool page_ids, cudaStream_t stream) {
    const int H_kv = H_q / group;
    const int nW = (nKVmax + 31) / 32;
    if (const int upc = cluster_upc(nW, B * H_kv)) {
        union_tables_cluster_kernel<true><<<dim3(kClusterCtas, B * H_kv), kClusterThreads, 0,
                                            stream>>>(mask, H_q, nQ, nKVmax, group, upc, tables,
                                                      counts);
        if (cudaGetLastError() != cudaSuccess) return CA_ERR_CUDA;
        return launch_csr(tables, counts, B * H_kv, nKVmax, page_ids, indptr, indices, stream);
    }
    // the bulk form where the (b, g) regions and pieces start on 16 bytes
    const int n_rows = group * nQ;
    if ((reinterpret_cast<uintptr_t>(mask) & 15u) == 0 && ((size_t)n_rows * nW) % 4 == 0) {
        if (const int rpp = bulk_rpp(n_rows, (size_t)nW * 4, nW, true)) {
            const int st = launch_bulk<true>(mask, B, H_q, nQ, nKVmax, group, rpp, tables,
                                             counts, stream);
            if (st != CA_OK) return st;
            return launch_csr(tables, counts, B * H_kv, nKVmax, page_ids, indptr, indices,
                              stream);
        }
    }
    int wpr = ((nW + 31) / 32) * 32;
    if (wpr > kMaxThreads) wpr = kMaxThreads;
    int rg = 512 / wpr;
    if (rg < 1) rg = 1;
    if (rg > group * nQ) rg = group * nQ;
    const int threads = wpr * rg;
    const size_t smem = sizeof(uint32_t) * (size_t)threads;
    union_bits_kernel<<<B * H_kv, threads, smem, stream>>>(mask, H_q, nQ, nKVmax, group, wpr, rg,
                                                            tables, counts);
    if (cudaGetLastError() != cudaSuccess) return CA_ERR_CUDA;
    return launch_csr(tables, counts, B * H_kv, nKVmax, page_ids, indptr, indices, stream);
}

int launch_build_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                        int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                        bool page_ids, cudaStream_t stream) {
    const int H_kv = H_q / group;
    const int n_chunks = (nKVmax + 15) / 16;
    const int vec = ((reinterpret_cast<uintptr_t>(mask) & 15u) == 0 && (nKVmax % 16) == 0) ? 1 : 0;
    if (const int upc = vec ? cluster_upc(n_chunks, B * H_kv) : 0) {
        union_tables_cluster_kernel<false><<<dim3(kClusterCtas, B * H_kv), kClusterThreads, 0,
                                             stream>>>(mask, H_q, nQ, nKVmax, group, upc, tables,
                                                       counts);
        if (cudaGetLastError() != cudaSuccess) return CA_ERR_CUDA;
        return launch_csr(tables, counts, B * H_kv, nKVmax, page_ids, indptr, indices, stream);
    }
    if (const int rpp = vec ? bulk_rpp(group * nQ, (size_t)nKVmax, n_chunks, false) : 0) {
        const int st = launch_bulk<false>(mask, B, H_q, nQ, nKVmax, group, rpp, tables, counts,
                                          stream);
        if (st != CA_OK) return st;
        return launch_csr(tables, counts, B * H_kv, nKVmax, page_ids, indptr, indices, stream);
    }
    int chp = ((n_chunks + 31) / 32) * 32;
    if (chp > kMaxThreads) chp = kMaxThreads;
    int rg = kMaxThreads / chp;
    const int n_rows = group * nQ;
    if (rg > n_rows) rg = n_rows;
    // keep CTAs modest when the chunk count is small: at most 512 threads
    while (rg > 1 && chp * rg > 512) --rg;
    if (rg < 1) rg = 1;
    const int threads = chp * rg;
    const size_t smem = sizeof(uint32_t) * (size_t)threads;
    union_tables_kernel<<<B * H_kv, threads, smem, stream>>>(mask, H_q, nQ, nKVmax, group, chp,
                                                              rg, vec, tables, counts);
    if (cudaGetLastError() != cudaSuccess) return CA_ERR_CUDA;
    return launch_csr(tables, counts, B * H_kv, nKVmax, page_ids, indptr, indices, stream);
}

}  // namespace ca
