// chunk_attention.cu — zero-copy paged chunk attention over Block-Union tables
// (tcgen05 + TMEM + TMA, sm_100a).
//
// CompactAttention pages, "Methodology", execution stage: dense attention of
// every query head of a GQA group over the KV blocks of T_{b,g}, read in place
// from the KV-head-major cache [B, H_kv, L, D] (each (b, KV head, block) is one
// contiguous region, so a block is a single TMA box) with no gather copy.
//
// Work item (one CTA): (b, g, pair of 128-row tiles). A tile packs G query
// heads x R = 128 / G chunk rows into the MMA's M = 128 rows (row m = head
// (m / R), chunk row r0 + (m % R)), so each selected KV block is brought into
// shared memory once and serves the whole group; the two tiles of the pair
// share every K/V stage as well. Both tiles' rows lie in the same positions
// window, so they walk the same prefix of the (ascending) table:
//   n_eff  = #{t : T[t] <= last position / blk}          (later blocks unread)
//   n_full = #{t : T[t] <= (first position + 1) / blk - 1} (no causal mask)
//
// Grid: one CTA per item, items ordered group by group (all tile pairs of a
// group, the last rows first, then the next group): the CTAs resident
// together hold every tile pair of a few groups, start each group's table at
// the same time and walk its blocks in lockstep, so each block comes from HBM
// once and then from L2,
// and the items past the last full wave (split below) cover the last groups
// whole, whose tables the full waves did not read. (A persistent stream-K
// schedule that balances the last wave staggers the CTAs instead and read
// several times more DRAM; under the 1 kW power cap that sustained runs
// reach, it was not faster either.) When
// the items do not fill the SMs evenly, the items past the last full wave are
// cut into segments of their block lists (split-KV): each segment CTA writes a
// normalised partial O (bf16) and its LSE (fp32) to the workspace and the
// item's last CTA merges them in fp32 (an atomic counter, no waiting). An
// item whose table would give segments shorter than kMinSegEntries blocks
// runs whole on its first segment's CTA (decided here, from the count).
//
// FP8 (template flag): E4M3 Q, K, V, kind::f8f6f4 MMAs (K = 32 per step), P
// rounded to E4M3 as 2^(x + 4) in TMEM (four values per column); O and the
// LSE are normalised by the fp32 sum of the unrounded P, as in the bf16 path.
//
// Warp roles (384 threads, one CTA per SM):
//   warps 0-3  softmax + epilogue of tile 0 (thread = TMEM lane = packed row)
//   warps 4-7  softmax + epilogue of tile 1
//   warp 8     MMA issue (one elected lane) + TMEM allocation
//   warp 9     TMA producer (Q once, then K and V of T[0..n_eff) in a ring)
//   warps 10-11 idle (they complete the third warpgroup of the register split)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512);
// P (bf16 pairs) overwrites the first blk/2 columns of S and feeds the P.V MMA
// straight from tensor memory, in chunks of 64 keys as the softmax produces
// them.
// MMA order per block j: PV0(j), S0(j+1), PV1(j), S1(j+1): while tile 0's
// softmax works on S0(j+1) the tensor core runs tile 1's products and the
// other way round.
//
// Online softmax in base 2 (x = s * scale * log2 e); the running max is only
// raised when it grows by more than 16 (a factor 2^16), so O is rescaled in
// TMEM rarely (P stays below 2^16, far inside bf16 / fp32 range; a threshold
// of 8 rescaled often enough to cost 2.6% of the time); the final O / l and
// LSE = (m + log2 l) ln 2 use the same max.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "ca_internal.h"
#include "sm100_ptx.cuh"

namespace ca {

namespace {

constexpr int kTileM = 128;
// Register split (setmaxnreg): three warpgroups — two softmax warpgroups (one
// per tile) and one holding the MMA issuer, the TMA producer and two idle
// warps. Launched at kLaunchRegs registers per thread (the most 384 threads
// can have: three warps share each SM sub-partition's 16K registers); the
// softmax warpgroups then grow to kSoftmaxRegs and the third shrinks to
// kControlRegs, so that per sub-partition (one warp of each warpgroup)
// 2 * kSoftmaxRegs + kControlRegs = 3 * kLaunchRegs (208 + 208 + 88 = 504).
constexpr int kSoftmaxWarps = 8;
constexpr int kMmaWarp = kSoftmaxWarps;
constexpr int kTmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 4);
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
// per SM sub-partition: one warp of each softmax warpgroup plus one control warp
constexpr int kControlRegs = 3 * kLaunchRegs - 2 * kSoftmaxRegs;
static_assert(kSoftmaxRegs % 8 == 0 && kControlRegs % 8 == 0 && kControlRegs >= 24,
              "setmaxnreg counts are multiples of 8, at least 24");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 16.0f;
constexpr float kLn2 = 0.693147180559945309f;
constexpr int kSmemBudget = 227 * 1024;
constexpr int kSmemFloor = 120 * 1024;  // keeps one CTA (and one TMEM owner) per SM
// Keys per P chunk handed from the softmax to the P.V MMA (measured: 32- and
// 128-key chunks were slower).
constexpr int kPChunkKeysMax = 64;

struct Params {
    int B, H_q, H_kv, C, L_max, G, R, n_pairs, nKVmax;
    int n_items, n_first, split;  // split of the last wave (split == 1: none)
    unsigned int *counters;       // [n_items - n_first] finished segments per item
    float *part_lse;              // [n_rest][split][256] base-2 LSE of a segment's rows
    uint16_t *part_o;             // [n_rest][split][256][D] normalised partial O (bf16)
    float scale_log2;
    float o_scale;              // factor on O (the V descale of FP8 inputs, else 1)
    const int32_t *tables;      // or, in the paged form, kv_indices (global pages)
    const int32_t *counts;
    const int32_t *kv_indptr;   // paged form: rows of (b, g) in kv_indices; else NULL
    long long nnz;              // paged form: entries of kv_indices
    uint16_t *O;
    float *LSE;
    unsigned int *status;
    int chunk_start[kMaxBatch];
    int chunk_len[kMaxBatch];   // rows of each sequence's chunk (<= C)
    unsigned char b_order[kMaxBatch];
};

template <int D, int BLK, bool F8 = false>
struct Layout {
    static constexpr int kEB = F8 ? 1 : 2;           // bytes per Q / K / V element
    static constexpr int kQTile = kTileM * D * kEB;  // D*kEB/128 sub-tiles of 128 rows x 128 B
    static constexpr int kKV = BLK * D * kEB;        // D*kEB/128 sub-tiles of BLK rows x 128 B
    static constexpr int kRoom = kSmemBudget - 2048 - 2 * kQTile;
    // K and V ring stages (equal rings): as many as fit, at most 4
    static constexpr int kFit = kRoom / kKV;  // K + V stages that fit
    static constexpr int kStages = kFit / 2 > 4 ? 4 : kFit / 2;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = 2 * kQTile;
    static constexpr int kVOff = kKOff + kStages * kKV;
    static constexpr int kBarOff = kVOff + kStages * kKV;
    static constexpr int kPChunkKeys = kPChunkKeysMax < BLK ? kPChunkKeysMax : BLK;
    static constexpr int kPChunks = BLK / kPChunkKeys;  // P reaches the MMA chunk by chunk
    static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 * kPChunks + 2 + 1;
    static constexpr int kEnd = kBarOff + kNumBars * 8 + 16;
    static constexpr int kDynamic = (kEnd + 1024) > kSmemFloor ? (kEnd + 1024) : kSmemFloor;
    static_assert(kStages >= 2, "need two K / V stages");
    static_assert(kDynamic <= kSmemBudget, "shared memory budget exceeded");
};

// KV block index of a table entry (span-table entries carry Q-block bits
// above kSpanEntryBits).
template <bool SPAN>
__device__ __forceinline__ int block_of(int e) {
    return SPAN ? (e & ((1 << kSpanEntryBits) - 1)) : e;
}

// Entries of the ascending prefix T[0, n) that are <= bound; warp-cooperative
// (all 32 lanes), scanning windows of 32 from the end (the answer is normally
// in the last window: only blocks inside the chunk can lie past the bound).
template <bool SPAN>
__device__ __forceinline__ int count_le(const int32_t *T, int n, int bound, int lane, int base) {
    int hi = n;
    while (hi > 0) {
        const int lo = hi > 32 ? hi - 32 : 0;
        const int idx = lo + lane;
        const int v = idx < hi ? block_of<SPAN>(__ldg(T + idx)) - base : 0;
        const unsigned gt = __ballot_sync(0xffffffffu, idx < hi && v > bound);
        const int ngt = __popc(gt);
        if (ngt < hi - lo) return hi - ngt;
        hi = lo;
    }
    return 0;
}

// Named barrier 1 over the softmax warps only (barrier 0 is __syncthreads).
__device__ __forceinline__ void softmax_bar_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxWarps * 32) : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_row<128>(uint32_t taddr, uint32_t (&r)[128]) {
    tmem_ld128(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_row<64>(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld64(taddr, r);
}

template <int D, int BLK, int MODE, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params P) {
    using L = Layout<D, BLK, F8>;
    constexpr bool DENSE = MODE == kModeDense;
    constexpr bool COMPACT = MODE == kModeCompact;  // K/V block t sits at row t * BLK
    constexpr bool PERTILE = MODE == kModePerTile;  // one head per tile, span tables
    constexpr int NST = L::kStages;
    // FP8 (E4M3 Q, K, V; kind::f8f6f4 MMAs; P rounded to E4M3 in TMEM)
    constexpr int EB = L::kEB;
    constexpr int DCH = D * EB / 128;  // 128-byte sub-tiles along D
    constexpr int XIN = 128 / EB;      // elements in a 128-byte sub-tile row
    constexpr int KS = 32 / EB;        // elements per MMA K step (32 bytes)
    constexpr uint32_t kIdescS =
        F8 ? idesc_e4m3_f32(kTileM, BLK, false) : idesc_bf16_f32(kTileM, BLK, false);
    constexpr uint32_t kIdescPV =
        F8 ? idesc_e4m3_f32(kTileM, D, true) : idesc_bf16_f32(kTileM, D, true);
    // FP8 P is 2^(x + 4) with the running max raised whenever a row max grows
    // by more than 4.5, so P <= 2^8.5 fits E4M3 (max 448); the row's largest P
    // is at least 2^4, values down to 2^-10 of the reference stay normal and
    // the subnormals reach 2^-13 (measured: bias 8 / threshold 1/2 rescaled O
    // often enough to cost 3.5% with the same errors). bf16 P is 2^x,
    // threshold 16.
    constexpr float kThresh = F8 ? 4.5f : kRescaleThreshold;
    constexpr float kPBias = F8 ? 4.0f : 0.0f;
    static_assert(!F8 || MODE == kModeTables || MODE == kModeDense,
                  "FP8 runs the table and dense paths");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + NST;
    uint64_t *v_full = k_empty + NST;
    uint64_t *v_empty = v_full + NST;
    constexpr int NPC = L::kPChunks;
    uint64_t *s_full = v_empty + NST;     // [2]
    uint64_t *p_full = s_full + 2;        // [2][NPC]: P chunk c of tile t stored in TMEM
    uint64_t *o_full = p_full + 2 * NPC;  // [2]
    uint64_t *mma_done = o_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    int *last_flag = abort_flag + 1;  // split items: this CTA merges the segments

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item: (b, pair, unit), the unit a KV group, or a query head in
    // the per-tile mode. CTAs [0, n_first) run items [0, n_first) whole; the
    // rest run one of `split` segments of an item's block list each
    // (segment-major, so that the CTAs resident together walk the same blocks).
    int item = blockIdx.x, seg = 0, nseg = 1;
    if (item >= P.n_first) {
        const int k = item - P.n_first;
        const int n_rest = P.n_items - P.n_first;
        seg = k / n_rest;
        item = P.n_first + k % n_rest;
        nseg = P.split;
    }
    const int units = PERTILE ? P.H_q : P.H_kv;
    const int per_b = units * P.n_pairs;
    const int b = P.b_order[item / per_b];
    const int rem = item % per_b;
    const int unit = rem / P.n_pairs;  // group by group
    // within a group the last rows first: they see the most causal blocks, so
    // the longest items start first (2-5% on the short early chunks of a
    // prefill, no change at 128K)
    const int pair = P.n_pairs - 1 - rem % P.n_pairs;
    const int g = PERTILE ? unit / P.G : unit;     // KV head
    const int head0 = PERTILE ? unit : g * P.G;  // query head of packed row 0
    const int cs = P.chunk_start[b];
    const int len_b = P.chunk_len[b];  // this sequence's chunk rows
    const int R = P.R;
    const int r0 = pair * 2 * R;
    const int r_end = min(r0 + 2 * R, len_b);
    const int p_min = cs + r0;
    const int p_max = cs + r_end - 1;
    const int jlast = p_max / BLK;
    const int jfull = (p_min + 1) / BLK - 1;

    // ---- table prefix this item walks (every role computes it the same way)
    const int32_t *T = nullptr;
    int base = 0;  // paged form: entries are base + block index
    int n_eff, n_full;
    if (r0 >= len_b) {  // a pair past a shorter chunk's end: no rows, no work
        n_eff = n_full = 0;
    } else if (DENSE) {
        n_eff = jlast + 1;
        n_full = jfull + 1 > 0 ? jfull + 1 : 0;
    } else {
        const size_t trow = PERTILE ? ((size_t)b * P.H_q + unit) * P.n_pairs + pair
                                    : (size_t)b * P.H_kv + g;
        int cnt;
        if (!PERTILE && P.kv_indptr != nullptr) {
            const long long start = __ldg(P.kv_indptr + trow);
            const long long end = __ldg(P.kv_indptr + trow + 1);
            cnt = (int)(end - start);
            if (start < 0 || end > P.nnz || end < start || end - start > P.nKVmax) {
                if (threadIdx.x == 0) atomicOr(P.status, kDevErrTable);
                cnt = 0;
            }
            T = P.tables + (cnt > 0 ? start : 0);
            base = (int)trow * P.nKVmax;
        } else {
            cnt = __ldg(P.counts + trow);
            if (cnt < 0 || cnt > P.nKVmax) {
                if (threadIdx.x == 0) atomicOr(P.status, kDevErrTable);
                cnt = 0;
            }
            T = P.tables + trow * P.nKVmax;
        }
        n_eff = count_le<PERTILE>(T, cnt, jlast, lane, base);
        n_full = count_le<PERTILE>(T, n_eff, jfull, lane, base);
    }
    // A split item whose prefix is short is not split after all: segments of
    // fewer than kMinSegEntries blocks each cost more in their own prologue,
    // epilogue and merge than they save (the table's length is known only
    // here, on the device). Every segment of the item reads the same count, so
    // all agree; segment 0 then takes the whole item and the others leave
    // before they touch shared memory, TMEM or the merge counters.
    if (nseg > 1 && n_eff < kMinSegEntries * nseg) {
        if (seg > 0) return;
        nseg = 1;
    }
    // this CTA's segment of the prefix: table entries [t0, t0 + n_run)
    const int t0 = (int)((long long)seg * n_eff / nseg);
    const int n_run = (int)((long long)(seg + 1) * n_eff / nseg) - t0;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full + t, 1);
            for (int c = 0; c < NPC; ++c) mbar_init(p_full + t * NPC + c, 4);
            mbar_init(o_full + t, 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kTmaWarp && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState ab{abort_flag, P.status};

    // Role code sits inside the branch that re-sized its registers, so the
    // compiler allocates each role within its own budget.
    if (warp >= kMmaWarp) {
      regs_dec<kControlRegs>();
      if (warp == kTmaWarp) {
        // ================================================================ producer
        int k_issued = 0, v_issued = 0;  // loads started (for the drain below)
        bool q_issued = false;
        if (n_run > 0) {
            if (lane == 0) {
                mbar_arrive_expect_tx(q_full, 2 * L::kQTile);
                for (int t = 0; t < 2; ++t)
                    for (int dc = 0; dc < DCH; ++dc)
                        tma_load_3d(smem + L::kQOff + t * L::kQTile + dc * (kTileM * 128), &tmQ,
                                    q_full, dc * XIN, r0 + t * R, b * P.H_q + head0);
            }
            q_issued = true;
            // K(j) and V(j) into ring stage j % NST (lane 0 only); false if a
            // wait gave up
            auto load_kv = [&](int j, int blk_idx) -> bool {
                const int s = j % NST;
                const uint32_t par = ((j / NST) & 1) ^ 1;
                if (!mbar_wait(k_empty + s, par, ab)) return false;
                mbar_arrive_expect_tx(k_full + s, L::kKV);
                for (int dc = 0; dc < DCH; ++dc)
                    tma_load_3d(smem + L::kKOff + s * L::kKV + dc * (BLK * 128), &tmK,
                                k_full + s, dc * XIN, blk_idx * BLK, b * P.H_kv + g);
                k_issued = j + 1;
                if (!mbar_wait(v_empty + s, par, ab)) return false;
                mbar_arrive_expect_tx(v_full + s, L::kKV);
                for (int dc = 0; dc < DCH; ++dc)
                    tma_load_3d(smem + L::kVOff + s * L::kKV + dc * (BLK * 128), &tmV,
                                v_full + s, dc * XIN, blk_idx * BLK, b * P.H_kv + g);
                v_issued = j + 1;
                return true;
            };
            int prev_last = -1;
            bool ok = true;
            for (int w0 = 0; w0 < n_run && ok; w0 += 32) {
                const int jj = t0 + w0 + lane;  // table index
                const int nwin = min(32, n_run - w0);
                int jb = DENSE ? jj : (lane < nwin ? block_of<PERTILE>(__ldg(T + jj)) - base : 0);
                if (!DENSE) {
                    int prv = __shfl_up_sync(0xffffffffu, jb, 1);
                    if (lane == 0) prv = prev_last;
                    const bool out = jb < 0 || jb >= P.nKVmax;
                    const bool bad = lane < nwin && (out || jb <= prv);
                    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(P.status, kDevErrTable);
                    prev_last = __shfl_sync(0xffffffffu, jb, nwin - 1);
                    // an out-of-range entry is fetched from one block past the cache end:
                    // the copy lands zero-filled and nothing outside K / V is touched
                    if (out) jb = P.nKVmax;
                }
                for (int q = 0; q < nwin; ++q) {
                    const int j = w0 + q;
                    const int blk_idx = COMPACT ? t0 + j : __shfl_sync(0xffffffffu, jb, q);
                    int good = 1;
                    if (lane == 0) good = load_kv(j, blk_idx);
                    good = __shfl_sync(0xffffffffu, good, 0);
                    if (!good) {
                        ok = false;
                        break;
                    }
                }
            }
        }
        // drain: every copy this warp started has landed before the CTA exits
        if (lane == 0) {
            if (q_issued) mbar_wait_drain(q_full, 0);
            for (int j = k_issued > NST ? k_issued - NST : 0; j < k_issued; ++j)
                mbar_wait_drain(k_full + j % NST, (j / NST) & 1);
            for (int j = v_issued > NST ? v_issued - NST : 0; j < v_issued; ++j)
                mbar_wait_drain(v_full + j % NST, (j / NST) & 1);
        }
        __syncwarp();
      } else if (warp == kMmaWarp) {
        // ================================================================ MMA issue
        if (n_run > 0 && lane == 0) {
            // Descriptors: the high words are constant; the low words of the Q
            // tiles are fixed for the item and those of a K / V stage are a base
            // plus the stage offset, so each MMA costs one add and the issue.
            const uint64_t dq = sdesc_sw128(sbase + L::kQOff, 16, 1024);
            const uint64_t dk = sdesc_sw128(sbase + L::kKOff, 16, 1024);
            const uint64_t dv = sdesc_sw128(sbase + L::kVOff, BLK * 128, 1024);
            const uint32_t q_lo = static_cast<uint32_t>(dq), q_hi = static_cast<uint32_t>(dq >> 32);
            const uint32_t k_lo = static_cast<uint32_t>(dk), k_hi = static_cast<uint32_t>(dk >> 32);
            const uint32_t v_lo = static_cast<uint32_t>(dv), v_hi = static_cast<uint32_t>(dv >> 32);
            constexpr uint32_t kStageUnits = L::kKV >> 4;  // one stage, in descriptor units
            auto issue_s = [&](int t, int slot) {
                const uint32_t a0 = q_lo + t * (L::kQTile >> 4);
                const uint32_t b0 = k_lo + slot * kStageUnits;
#pragma unroll
                for (int kk = 0; kk < D / KS; ++kk) {
                    // 32-byte K steps (16 bf16 / 32 E4M3) inside a 128-B swizzle
                    // row; a new 128-byte sub-tile every 4 steps
                    const uint32_t ao = ((kk >> 2) * (kTileM * 128) + (kk & 3) * 32) >> 4;
                    const uint32_t bo = ((kk >> 2) * (BLK * 128) + (kk & 3) * 32) >> 4;
                    if constexpr (F8)
                        mma_ss_w8(tmem + t * 128, a0 + ao, q_hi, b0 + bo, k_hi, kIdescS,
                                  kk > 0 ? 1u : 0u);
                    else
                        mma_ss_w(tmem + t * 128, a0 + ao, q_hi, b0 + bo, k_hi, kIdescS,
                                 kk > 0 ? 1u : 0u);
                }
            };
            // P.V of tile t, chunk by chunk as the softmax hands P over; false if a
            // wait gave up.
            auto issue_pv = [&](int t, int slot, bool acc, uint32_t par) -> bool {
                const uint32_t b0 = v_lo + slot * kStageUnits;
#pragma unroll
                for (int c = 0; c < NPC; ++c) {
                    if (!mbar_wait(p_full + t * NPC + c, par, ab)) return false;
                    tc_fence_after();
                    constexpr int KPC = L::kPChunkKeys / KS;  // MMAs (one K step each) per chunk
#pragma unroll
                    for (int kk = KPC * c; kk < KPC * c + KPC; ++kk) {
                        // a K step is 8 TMEM columns of P (2 bf16 or 4 E4M3 per
                        // column) and KS rows of V (128 bytes per row)
                        if constexpr (F8)
                            mma_ts_w8(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                                      b0 + ((kk * (KS * 128)) >> 4), v_hi, kIdescPV,
                                      (acc || kk > 0) ? 1u : 0u);
                        else
                            mma_ts_w(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                                     b0 + ((kk * (KS * 128)) >> 4), v_hi, kIdescPV,
                                     (acc || kk > 0) ? 1u : 0u);
                    }
                }
                return true;
            };
            bool ok = mbar_wait(q_full, 0, ab) && mbar_wait(k_full, 0, ab);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                tc_commit(s_full + 0);
                issue_s(1, 0);
                tc_commit(s_full + 1);
                tc_commit(k_empty + 0);
            }
            // per block j: P.V(j) of tile 0, S(j + 1) of tile 0, P.V(j) of tile 1,
            // S(j + 1) of tile 1 (S overwrites the P columns the P.V before it read;
            // the tensor core runs one CTA's MMAs in issue order)
            for (int j = 0; j < n_run && ok; ++j) {
                const int s = j % NST;
                const uint32_t ph = (j / NST) & 1;
                const bool more = j + 1 < n_run;
                const int s1 = (j + 1) % NST;
                const uint32_t ph1 = ((j + 1) / NST) & 1;
                if (!(ok = mbar_wait(v_full + s, ph, ab))) break;
                if (!(ok = issue_pv(0, s, j > 0, j & 1))) break;
                if (more) {
                    if (!(ok = mbar_wait(k_full + s1, ph1, ab))) break;
                    tc_fence_after();
                    issue_s(0, s1);
                    tc_commit(s_full + 0);
                } else {
                    tc_commit(o_full + 0);
                }
                if (!(ok = issue_pv(1, s, j > 0, j & 1))) break;
                tc_commit(v_empty + s);
                if (more) {
                    issue_s(1, s1);
                    tc_commit(s_full + 1);
                    tc_commit(k_empty + s1);
                } else {
                    tc_commit(o_full + 1);
                }
            }
            // drain: all MMAs issued by this thread have completed
            tc_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
        __syncwarp();
      }
    } else {
        regs_inc<kSoftmaxRegs>();
        // ================================================================ softmax
        // Warp (t, qw): tile t, TMEM lanes / packed rows 32*qw .. 32*qw + 31.
        const int t = warp / 4;
        const int qw = warp & 3;
        const int m = qw * 32 + lane;
        const int h_local = m / R;
        const int r = r0 + t * R + (m % R);
        const bool valid = r < len_b;
        const int p = cs + r;
        const int h = head0 + h_local;
        // per-tile mode: bit of this row's Q-block in the span-table entries
        // (the 32 rows of a warp share one Q-block, so it is warp-uniform)
        const int member_shift = kSpanEntryBits + (r / BLK - r0 / BLK);
        const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
        const uint32_t tS = tmem + lane_base + t * 128;
        const uint32_t tO = tmem + lane_base + 256 + t * 128;
        const float sl2 = P.scale_log2;
        // Table entries the softmax needs, fetched ahead into one register per
        // lane: the blocks that need the causal mask (at most a few: entries
        // past n_full; lane i holds entry n_full + i), or, in the per-tile mode,
        // a window of 32 entries of the walk (lane i holds entry t0 + w + i).
        const int j_mask = n_full - t0;  // walk index from which blocks are masked
        int tab_reg = 0;
        if (!DENSE && !PERTILE) {
            const int e = n_full + lane;
            tab_reg = e < n_eff ? __ldg(T + e) - base : 0;
        }
        if (PERTILE) tab_reg = lane < n_run ? __ldg(T + t0 + lane) : 0;

        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < n_run; ++j) {
            int e_j = 0;
            if (PERTILE) {
                e_j = __shfl_sync(0xffffffffu, tab_reg, j & 31);
                if ((j & 31) == 31) {  // next window of 32 entries
                    const int e = t0 + j + 1 + lane;
                    tab_reg = e < t0 + n_run ? __ldg(T + e) : 0;
                }
            }
            ok = mbar_wait(s_full + t, j & 1, ab);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (PERTILE && ((e_j >> member_shift) & 1) == 0) {
                // block not selected by this row's Q-block: P = 0, the running
                // max and sum are unchanged
                uint32_t zero[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
                for (int c = 0; c < NPC; ++c) {
                    constexpr int CK = L::kPChunkKeys;
#pragma unroll
                    for (int q = 0; q < CK / 32; ++q) tmem_st16(tS + c * (CK / 2) + q * 16, zero);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    mbar_arrive_lane0(p_full + t * NPC + c, lane);
                }
                continue;
            }
            float s[BLK];
            {
                uint32_t v[BLK];
                tmem_ld_row<BLK>(tS, v);  // the whole S row in one round trip
#pragma unroll
                for (int i = 0; i < BLK; ++i) s[i] = __uint_as_float(v[i]);
            }
            if (j >= j_mask) {
                int jb = DENSE ? t0 + j
                               : (PERTILE ? block_of<true>(e_j)
                                          : __shfl_sync(0xffffffffu, tab_reg, (j - j_mask) & 31));
                jb = min(max(jb, 0), P.nKVmax);  // only matters for a flagged, invalid table
                const int lim = p - jb * BLK;  // columns c <= lim are visible
#pragma unroll
                for (int c = 0; c < BLK; ++c)
                    if (c > lim) s[c] = -INFINITY;
            }
            // row max: 8 independent chains of 3-input max, then a short tree
            float mx8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = s[k];
#pragma unroll
            for (int c = 8; c + 8 < BLK; c += 16)
#pragma unroll
                for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], s[c + k], s[c + 8 + k]);
            if ((BLK - 8) % 16 != 0) {
#pragma unroll
                for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], s[BLK - 8 + k]);
            }
            const float pmax = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                                     fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
            const float m_blk = pmax * sl2;
            const float m_new = fmaxf(m_run, m_blk);
            const bool old_finite = m_run != -INFINITY;
            const bool upd = old_finite ? (m_new > m_run + kThresh) : (m_new != -INFINITY);
            float alpha = 1.0f;
            if (upd) {
                alpha = old_finite ? ex2_approx(m_run - m_new) : 0.0f;
                m_run = m_new;
            }
            // O rescale (rare: only when a row's max grew past the threshold). O is
            // stable here: S(j) was committed after P.V(j-1) was issued. It must land
            // before the first P chunk is handed over.
            const bool need = upd && old_finite && j > 0;
            if (__any_sync(0xffffffffu, need)) {
                const float a = need ? alpha : 1.0f;
#pragma unroll
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t v[16];
                    tmem_ld16(tO + c * 16, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * a);
                    tmem_st16(tO + c * 16, v);
                }
            }
            const float m_use = m_run == -INFINITY ? 0.0f : m_run;
            l_run *= alpha;
            // exponentials in pairs: x = s * scale_log2 - m as one f32x2 FMA, the
            // row sum in four f32x2 accumulators
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            const uint64_t nm2 = f2_pack(kPBias - m_use, kPBias - m_use);
            uint64_t acc2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc2[k] = 0ull;
#pragma unroll
            for (int c = 0; c < NPC; ++c) {
                constexpr int CK = L::kPChunkKeys;
                constexpr int PCOLS = CK * EB / 4;  // TMEM columns of a P chunk
                uint32_t pk[CK / 2];  // bf16 pairs; FP8: E4M3 quads in pk[0, CK/4)
                uint64_t p_prev = 0ull;
#pragma unroll
                for (int i = 0; i < CK / 2; ++i) {
                    const int e0 = c * CK + 2 * i;
                    const uint64_t x2 = f2_fma(f2_pack(s[e0], s[e0 + 1]), sl2x2, nm2);
                    // FP8: every 4th pair on the FMA pipe (the FP8 products are
                    // short, so the exponentials set the softmax: 2.3% faster
                    // at 128K; in bf16 the same split was 4.8% slower)
                    const uint64_t p2 =
                        (F8 && (c * CK / 2 + i) % 4 == 3)
                            ? exp2_poly2(x2)
                            : f2_pack(ex2_approx(f2_lo(x2)), ex2_approx(f2_hi(x2)));
                    acc2[i & 3] = f2_add(acc2[i & 3], p2);
                    if constexpr (F8) {
                        // P.V takes P rounded to E4M3; O and the LSE are both
                        // normalised by the fp32 sum of the unrounded P
                        if (i & 1) {
                            pk[i >> 1] = pack_e4m3x4(f2_lo(p_prev), f2_hi(p_prev), f2_lo(p2),
                                                     f2_hi(p2));
                        } else {
                            p_prev = p2;
                        }
                    } else {
                        pk[i] = pack_bf16x2(f2_lo(p2), f2_hi(p2));
                    }
                }
#pragma unroll
                for (int q = 0; q < PCOLS / 16; ++q) tmem_st16(tS + c * PCOLS + q * 16, pk + q * 16);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                mbar_arrive_lane0(p_full + t * NPC + c, lane);
            }
            acc2[0] = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
            l_run += f2_lo(acc2[0]) + f2_hi(acc2[0]);
        }
        bool have_o = false;
        if (n_run > 0 && __all_sync(0xffffffffu, ok)) {
            const bool got = mbar_wait(o_full + t, 0, ab);
            have_o = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        const float inv_l = l_run > 0.0f ? P.o_scale / l_run : 0.0f;
        const float lse2 = (l_run > 0.0f && have_o) ? m_run + log2f(l_run) - kPBias : -INFINITY;
        uint16_t *orow = P.O + (((size_t)b * P.H_q + h) * P.C + r) * D;
        float *lse_out = (valid && P.LSE != nullptr) ? P.LSE + ((size_t)b * P.H_q + h) * P.C + r
                                                      : nullptr;
        if (nseg == 1) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (have_o) {
                    tmem_ld32(tO + c * 32, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l,
                                        __uint_as_float(v[2 * i + 1]) * inv_l);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            if (lse_out) *lse_out = lse2 * kLn2;
        } else {
            // Segment of a split item: its normalised O (bf16) and base-2 LSE
            // (fp32) go to the workspace, one slot row per packed row.
            // (recomputed from the block index: nothing of the item decode has
            // to stay live across the block loop for this rare path)
            const int kseg = (int)blockIdx.x - P.n_first;
            const int n_rest_ = P.n_items - P.n_first;
            const int rest = kseg % n_rest_;
            const int seg_ = kseg / n_rest_;
            const int m_ = (warp & 3) * 32 + lane;
            const size_t row0 = (size_t)rest * P.split * kRowsPerItem + (warp / 4) * 128 + m_;
            const size_t mine = row0 + (size_t)seg_ * kRowsPerItem;
            uint16_t *po = P.part_o + mine * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (have_o) {
                    tmem_ld32(tO + c * 32, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l,
                                        __uint_as_float(v[2 * i + 1]) * inv_l);
                uint4 *dst = reinterpret_cast<uint4 *>(po + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
            P.part_lse[mine] = lse2;
            // publish, count this segment in, and let the item's last CTA merge
            __threadfence();
            softmax_bar_sync();
            if (threadIdx.x == 0) {
                const unsigned prev = atomicAdd(P.counters + rest, 1u);
                *last_flag = prev + 1 == (unsigned)nseg;
            }
            softmax_bar_sync();
            if (*last_flag) {
                __threadfence();
                float ls[kMaxSplit];
                float mx = -INFINITY;
#pragma unroll
                for (int sg = 0; sg < kMaxSplit; ++sg) {
                    ls[sg] = sg < nseg ? __ldcg(P.part_lse + row0 + (size_t)sg * kRowsPerItem)
                                       : -INFINITY;
                    mx = fmaxf(mx, ls[sg]);
                }
                float wsum = 0.0f;
#pragma unroll
                for (int sg = 0; sg < kMaxSplit; ++sg) {
                    ls[sg] = mx == -INFINITY ? 0.0f : exp2f(ls[sg] - mx);  // weight
                    wsum += ls[sg];
                }
                const float inv_w = wsum > 0.0f ? 1.0f / wsum : 0.0f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    float acc[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
                    for (int sg = 0; sg < nseg; ++sg) {
                        const float w = ls[sg] * inv_w;
                        // eight bf16 per 16-byte load; a bf16 widens to fp32
                        // by moving its bits to the high half
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            P.part_o + (row0 + (size_t)sg * kRowsPerItem) * D + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 x = __ldcg(src + i);
                            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                acc[8 * i + 2 * k] =
                                    fmaf(w, __uint_as_float(xw[k] << 16), acc[8 * i + 2 * k]);
                                acc[8 * i + 2 * k + 1] = fmaf(
                                    w, __uint_as_float(xw[k] & 0xffff0000u), acc[8 * i + 2 * k + 1]);
                            }
                        }
                    }
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pack_bf16x2(acc[8 * i], acc[8 * i + 1]),
                                                pack_bf16x2(acc[8 * i + 2], acc[8 * i + 3]),
                                                pack_bf16x2(acc[8 * i + 4], acc[8 * i + 5]),
                                                pack_bf16x2(acc[8 * i + 6], acc[8 * i + 7]));
                    }
                }
                if (lse_out) *lse_out = wsum > 0.0f ? (mx + log2f(wsum)) * kLn2 : -INFINITY;
                if (threadIdx.x == 0) P.counters[rest] = 0u;  // ready for the next launch
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D tiled map over a contiguous [d2][d1][d0] tensor of bf16 (eb = 2) or
// 8-bit (eb = 1, E4M3 codes moved as bytes) elements, 128-byte swizzle.
bool encode_3d(CUtensorMap *map, const void *base, int eb, uint64_t d0, uint64_t d1,
               uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * eb, d0 * d1 * eb};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt =
        eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = fn(map, dt, 3, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, int BLK, int MODE, bool F8 = false>
int launch_t(const AttnArgs &a, cudaStream_t stream) {
    using L = Layout<D, BLK, F8>;
    auto kern = chunk_attn_kernel<D, BLK, MODE, F8>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        L::kDynamic);
    });
    if (attr_err != cudaSuccess) return CA_ERR_CUDA;
    // The in-kernel register split assumes exactly kLaunchRegs registers per
    // thread at launch; any other count could leave a warpgroup waiting for
    // registers that never come, so refuse to launch instead.
    static int num_regs = -1;
    if (num_regs < 0) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return CA_ERR_CUDA;
        num_regs = fa.numRegs;
    }
    if (num_regs != kLaunchRegs) return CA_ERR_UNSUPPORTED;

    const int G = a.H_q / a.H_kv;
    const int pack = MODE == kModePerTile ? 1 : G;  // query heads packed into a tile
    const int R = kTileM / pack;
    const int n_tiles = (a.C + R - 1) / R;
    const int n_pairs = (n_tiles + 1) / 2;

    constexpr int EB = L::kEB;
    constexpr uint32_t XIN = 128 / EB;  // box width: one 128-byte swizzle row
    CUtensorMap tq, tk, tv;
    if (!encode_3d(&tq, a.Q, EB, (uint64_t)D, (uint64_t)a.C, (uint64_t)a.B * a.H_q, XIN, R,
                   pack) ||
        !encode_3d(&tk, a.K, EB, (uint64_t)D, (uint64_t)a.L_max, (uint64_t)a.B * a.H_kv, XIN, BLK,
                   1) ||
        !encode_3d(&tv, a.V, EB, (uint64_t)D, (uint64_t)a.L_max, (uint64_t)a.B * a.H_kv, XIN, BLK,
                   1))
        return CA_ERR_CUDA;

    Params P;
    P.B = a.B;
    P.H_q = a.H_q;
    P.H_kv = a.H_kv;
    P.C = a.C;
    P.L_max = a.L_max;
    P.G = G;
    P.R = R;
    P.n_pairs = n_pairs;
    P.nKVmax = a.L_max / BLK;
    P.scale_log2 = a.scale * 1.4426950408889634f * (F8 ? a.descale[0] * a.descale[1] : 1.0f);
    P.o_scale = F8 ? a.descale[2] : 1.0f;
    P.tables = a.tables;
    P.counts = a.counts;
    P.kv_indptr = a.kv_indptr;
    P.nnz = a.nnz;
    P.O = static_cast<uint16_t *>(a.O);
    P.LSE = a.LSE;
    P.status = static_cast<unsigned int *>(a.workspace);
    // longest visible lengths first: their items are the heaviest
    auto len_of = [&](int i) { return a.chunk_len ? a.chunk_len[i] : a.C; };
    auto reach = [&](int i) { return (long long)a.chunk_start[i] + len_of(i); };
    int order[kMaxBatch];
    for (int i = 0; i < a.B; ++i) order[i] = i;
    for (int i = 1; i < a.B; ++i) {
        const int x = order[i];
        int k = i - 1;
        while (k >= 0 && reach(order[k]) < reach(x)) {
            order[k + 1] = order[k];
            --k;
        }
        order[k + 1] = x;
    }
    for (int i = 0; i < kMaxBatch; ++i) {
        P.chunk_start[i] = i < a.B ? a.chunk_start[i] : 0;
        P.chunk_len[i] = i < a.B ? len_of(i) : 0;
        P.b_order[i] = static_cast<unsigned char>(i < a.B ? order[i] : 0);
    }
    // split the last wave when the items are alike (one cache length) and long
    const int units = MODE == kModePerTile ? a.H_q : a.H_kv;
    const int n_items = a.B * units * n_pairs;
    bool alike = true;
    int nkv_max = 0;
    for (int i = 0; i < a.B; ++i) {
        alike = alike && a.chunk_start[i] == a.chunk_start[0] && len_of(i) == len_of(0);
        nkv_max = max(nkv_max, (a.chunk_start[i] + len_of(i) + BLK - 1) / BLK);
    }
    SplitPlan plan = plan_split(n_items, current_sm_count(), D,
                                alike && nkv_max >= kSplitMinBlocks);
    if (plan.split > 1 && a.workspace_bytes < plan.bytes)
        plan = plan_split(n_items, 0, D, false);  // workspace too small: no split
    unsigned char *ws = static_cast<unsigned char *>(a.workspace);
    P.n_items = n_items;
    P.n_first = plan.n_first;
    P.split = plan.split;
    P.counters = reinterpret_cast<unsigned int *>(ws + kWorkspaceHeader);
    P.part_lse = reinterpret_cast<float *>(ws + plan.lse_off);
    P.part_o = reinterpret_cast<uint16_t *>(ws + plan.o_off);
    const unsigned grid = static_cast<unsigned>(plan.n_first +
                                                (n_items - plan.n_first) * plan.split);
    kern<<<grid, kThreads, L::kDynamic, stream>>>(tq, tk, tv, P);
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

}  // namespace

int current_sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            n <= 0)
            return 148;
        cache[dev] = n;
    }
    return cache[dev];
}

int launch_chunk_attention(const AttnArgs &a, int mode, cudaStream_t stream) {
    if (a.fp8) {
        if (a.D != 128 || (mode != kModeTables && mode != kModeDense)) return CA_ERR_UNSUPPORTED;
        const bool dense = mode == kModeDense;
        if (a.blk == 128)
            return dense ? launch_t<128, 128, kModeDense, true>(a, stream)
                         : launch_t<128, 128, kModeTables, true>(a, stream);
        if (a.blk == 64)
            return dense ? launch_t<128, 64, kModeDense, true>(a, stream)
                         : launch_t<128, 64, kModeTables, true>(a, stream);
        return CA_ERR_UNSUPPORTED;
    }
#define CA_DISPATCH(D_, BLK_)                                                         \
    if (a.D == D_ && a.blk == BLK_) {                                                 \
        if (mode == kModeDense) return launch_t<D_, BLK_, kModeDense>(a, stream);     \
        if (mode == kModeCompact) return launch_t<D_, BLK_, kModeCompact>(a, stream); \
        if (mode == kModePerTile) return launch_t<D_, BLK_, kModePerTile>(a, stream); \
        return launch_t<D_, BLK_, kModeTables>(a, stream);                            \
    }
    CA_DISPATCH(128, 128)
    CA_DISPATCH(128, 64)
    CA_DISPATCH(64, 128)
    CA_DISPATCH(64, 64)
#undef CA_DISPATCH
    return CA_ERR_UNSUPPORTED;
}

}  // namespace ca
