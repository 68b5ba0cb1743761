/*
 * compactattn.h — C ABI of the B200 (sm_100a) CompactAttention chunked-prefill
 * hot path: Block-Union KV table construction and zero-copy paged attention.
 *
 * Method: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
 * Selection" (arXiv 2605.16839; gist.science / hotpaper.ai / fugumt.com pages,
 * section "Methodology" / abstract).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All pointers except `chunk_start` are DEVICE pointers owned by the caller.
 *   The library never allocates, frees or synchronises device memory, except
 *   ca_read_device_status(), which synchronises its stream.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and returns a ca_status. Argument checks run on the host
 *   before anything is enqueued; on a non-OK return nothing was launched.
 * - bf16 tensors are raw IEEE bfloat16 (uint16 bit patterns), row-major and
 *   contiguous in the stated layout; 16-byte aligned base pointers.
 * - Notation: B sequences, H_q query heads, H_kv KV heads, G = H_q / H_kv
 *   (query head h reads KV head h / G), D head dim, blk block size (the Q-block
 *   size, the KV-block size and the cache page size are all blk), C chunk
 *   length, L_max allocated cache rows per (b, KV head), nKVmax = L_max / blk,
 *   nQ = C / blk, chunk_start[b] = tokens already cached for sequence b.
 */
#ifndef COMPACTATTN_H
#define COMPACTATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ca_status {
    CA_OK = 0,
    CA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, non-finite scale   */
    CA_ERR_SHAPE = 2,       /* shape precondition violated                          */
    CA_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                     */
    CA_ERR_UNSUPPORTED = 4, /* D, blk or G outside the compiled set                 */
    CA_ERR_WORKSPACE = 5,   /* workspace NULL, misaligned or smaller than required  */
    CA_ERR_TABLE = 6,       /* device: table entry/count out of range or unsorted   */
    CA_ERR_TIMEOUT = 7,     /* device: a bounded wait inside a kernel expired       */
    CA_ERR_CUDA = 8         /* a CUDA runtime / driver call failed                  */
} ca_status;

/* Human-readable name of a status code (static storage). */
const char *ca_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int ca_version(void);

/*
 * Block-Union KV table construction (pages: "Methodology", selection stage —
 * Q-block union, then intra-group union, giving the minimal per-(batch,
 * KV-group) block table T_{b,g}; the CSR form is the kv_indptr / kv_indices
 * metadata of the execution stage).
 *
 *   U[b,g,j] = OR_{h in group g} OR_{i < nQ} (mask[b,h,i,j] != 0)
 *   tables[b,g,:]  = the j with U[b,g,j] = 1, ascending, then -1 up to nKVmax
 *   counts[b,g]    = number of such j
 *   indptr[k]      = sum of counts over flattened (b,g) < k   (k = 0..B*H_kv)
 *   indices[...]   = the tables' valid prefixes, concatenated in (b,g) order
 *
 * mask    uint8 [B, H_q, nQ, nKVmax], nonzero = tile selected (block j is
 *         absolute: cached blocks first, then the chunk's).
 * tables  int32 [B, H_kv, nKVmax]   (H_kv = H_q / group), written in full.
 * counts  int32 [B, H_kv].
 * indptr  int32 [B*H_kv + 1] or NULL; indices int32 [B*H_kv*nKVmax] or NULL
 *         (indices needs indptr). Bit-exact, deterministic.
 * Errors: CA_ERR_INVALID_ARG (NULL / non-positive), CA_ERR_SHAPE (group does
 * not divide H_q), CA_ERR_ALIGN (tables/counts/indptr/indices not 4-byte
 * aligned), CA_ERR_CUDA (launch failure). On the device, with many (b, g),
 * a (b, g) whose mask rows do not land in shared memory within the bounded
 * wait (never seen in practice) gets count -1 and its table is left as it
 * was; the attention calls reject such a count (status bit 0).
 */
int ca_build_block_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                          int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices,
                          void *stream);

/*
 * ca_build_block_tables from a bit-packed mask: mask_bits uint32
 * [B, H_q, nQ, ceil(nKVmax / 32)], bit k (value 1 << k) of word w selects KV
 * block 32 * w + k; bits naming blocks at or past nKVmax are ignored. Eight
 * times less mask traffic than the byte mask. Outputs, errors and results are
 * those of ca_build_block_tables for the equivalent byte mask (mask_bits must
 * be 4-byte aligned).
 */
int ca_build_block_tables_bits(const uint32_t *mask_bits, int B, int H_q, int nQ, int nKVmax,
                               int group, int32_t *tables, int32_t *counts, int32_t *indptr,
                               int32_t *indices, void *stream);

/* Bytes of device workspace the attention entry points use for these sizes on
 * the current device, for D <= 128: a 256-byte header (status word) plus room
 * for the split of the last wave of work items (split-KV: when the items do
 * not fill the SMs evenly, the remaining items' block lists are cut into
 * segments run by separate CTAs; each writes a partial O and LSE, merged by
 * the item's last CTA). Any workspace of at least 256 bytes is valid; one
 * smaller than this value runs without the split. Allocate it once, 256-byte
 * aligned and zero-filled, and reuse it for later calls on the same stream;
 * after a call that reported a device error, zero it again. Returns 0 for
 * invalid sizes. */
size_t ca_workspace_bytes(int B, int H_q, int H_kv, int C, int blk);

/*
 * Zero-copy paged chunk attention over the Block-Union tables (pages:
 * "Methodology", execution stage — dense attention of every query head of the
 * group over the selected KV blocks, read in place from the KV-head-major
 * cache [B, H_kv, L, D], with no gather / compaction copy).
 *
 * For each sequence b, query head h (g = h / G) and chunk row r, with position
 * p = chunk_start[b] + r and key set
 *     K_set = { k : k / blk in T_{b,g}, k <= p }      (causal, bottom-right)
 * it computes s_k = scale * <Q[b,h,r,:], K[b,g,k,:]> and
 *     LSE[b,h,r] = ln sum_{k in K_set} exp(s_k)
 *     O[b,h,r,:] = sum_{k in K_set} exp(s_k - LSE) * V[b,g,k,:]
 * (O = 0 and LSE = -inf when K_set is empty). Blocks lying wholly after a
 * row's position are never read. Inputs bf16, products accumulated in fp32,
 * probabilities rounded to bf16 before the P.V product, O rounded to bf16.
 *
 * Q       bf16 [B, H_q, C, D]               (16-byte aligned)
 * K, V    bf16 [B, H_kv, L_max, D]          (16-byte aligned; rows
 *         [chunk_start[b], chunk_start[b] + C) already hold the chunk's keys)
 * tables  int32 [B, H_kv, nKVmax] ascending prefixes (as built above)
 * counts  int32 [B, H_kv]
 * chunk_start  HOST int32 [B], 0 <= chunk_start[b], chunk_start[b] + C <= L_max
 * O       bf16 [B, H_q, C, D] (16-byte aligned), LSE fp32 [B, H_q, C] or NULL
 * workspace   >= 256 bytes (ca_workspace_bytes(...) to allow the last-wave
 *         split), 256-byte aligned, zeroed once.
 * Supported: D in {64, 128}, blk in {64, 128}, G in {1, 2, 4, 8, 16},
 * 1 <= B <= 128, L_max % blk == 0.
 * Errors (host): CA_ERR_INVALID_ARG, CA_ERR_SHAPE, CA_ERR_ALIGN,
 * CA_ERR_UNSUPPORTED, CA_ERR_WORKSPACE, CA_ERR_CUDA. Errors found on the
 * device (a count outside [0, nKVmax], an entry outside [0, nKVmax) or a
 * table that is not strictly ascending; an expired bounded wait) never trap:
 * the kernel records them in the workspace status word, skips or zero-fills
 * the affected work, and ca_read_device_status() reports them.
 */
int ca_chunk_attention(const void *Q, const void *K, const void *V, const int32_t *tables,
                       const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                       int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                       float *LSE, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Block-Union tables in the paged-kernel metadata form (pages: "Methodology",
 * execution stage — the tables reach the paged attention kernel as
 * kv_indptr / kv_indices). Same union as ca_build_block_tables (tables and
 * counts are written too), and
 *   kv_indptr[k]  = sum of counts over flattened (b, g) < k   (k = 0..B*H_kv)
 *   kv_indices[kv_indptr[b*H_kv+g] + t] = (b*H_kv + g) * nKVmax + T_{b,g}[t]
 * i.e. global page ids of the cache viewed as B*H_kv*nKVmax pages of blk rows.
 * kv_indptr int32 [B*H_kv + 1], kv_indices int32 [B*H_kv*nKVmax] (capacity;
 * the first kv_indptr[B*H_kv] entries are written). Errors as
 * ca_build_block_tables; both pointers are required.
 */
int ca_build_kv_pages(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                      int32_t *tables, int32_t *counts, int32_t *kv_indptr, int32_t *kv_indices,
                      void *stream);

/*
 * ca_chunk_attention over the paged metadata form, with chunks of different
 * lengths (ragged batches): the block list of (b, g) is
 *   { kv_indices[t] - (b*H_kv + g) * nKVmax : kv_indptr[b*H_kv+g] <= t < kv_indptr[b*H_kv+g+1] },
 * ascending, and sequence b has chunk_len[b] rows (0 <= chunk_len[b] <= C;
 * NULL = all C). Q / O stay padded [B, H_q, C, D] (LSE [B, H_q, C]); rows
 * r >= chunk_len[b] are neither read for their result nor written. Each row's
 * result is the one ca_chunk_attention defines, with
 * chunk_start[b] + chunk_len[b] <= L_max instead of chunk_start[b] + C.
 * kv_indptr int32 [B*H_kv + 1] and kv_indices int32 [nnz] are device arrays.
 * A row range outside [0, nnz], longer than nKVmax or decreasing, or an entry
 * that is not a page of its own (b, g), is a device error (CA_ERR_TABLE) that
 * skips the affected work. Other arguments and errors as ca_chunk_attention.
 */
int ca_paged_chunk_attention(const void *Q, const void *K, const void *V,
                             const int32_t *kv_indptr, const int32_t *kv_indices, long long nnz,
                             const int32_t *chunk_start, const int32_t *chunk_len, int B, int H_q,
                             int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                             float *LSE, void *workspace, size_t workspace_bytes, void *stream);

/*
 * ca_chunk_attention on an FP8 (E4M3) cache. The pages use bf16; this is an
 * extension for caches stored in 8 bits. Q8, K8, V8 hold E4M3 codes (one byte
 * per element, same layouts as the bf16 tensors) and the attention inputs are
 * q_descale * Q8, k_descale * K8, v_descale * V8 (per-tensor factors, > 0).
 * Q.K^T and P.V run as E4M3 tensor-core products with fp32 accumulation; P
 * is rounded to E4M3 as 2^(x + 4) with the running row max raised whenever a
 * row max grows by more than 4.5, so it never saturates (P <= 2^8.5 < 448);
 * O and LSE are normalised by the fp32 sum of the unrounded P. A quarter of
 * the exponentials are a polynomial (relative error <= 1.02e-4).
 * O (bf16) and LSE (fp32) as ca_chunk_attention; tables == NULL (and counts
 * == NULL) runs the dense path over every visible block. Supported: D = 128,
 * blk in {64, 128}; other arguments and errors as ca_chunk_attention, plus
 * CA_ERR_INVALID_ARG for a descale that is not a positive finite number.
 */
int ca_chunk_attention_fp8(const void *Q8, const void *K8, const void *V8, float q_descale,
                           float k_descale, float v_descale, const int32_t *tables,
                           const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                           int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                           float *LSE, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The dense paged path (pages: the "dense attention baseline" the speedup is
 * quoted against): identical to ca_chunk_attention with
 * T_{b,g} = [0, ceil((chunk_start[b] + C) / blk)) for every group.
 * Same arguments minus tables / counts; same errors.
 */
int ca_dense_chunk_attention(const void *Q, const void *K, const void *V,
                             const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                             int L_max, int D, int blk, float scale, void *O, float *LSE,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Explicit-compaction ablation, step 1 (pages: "Experimental results" — the
 * efficiency ablation comparing zero-copy paged execution with explicit KV
 * compaction, the copy that token-level selection methods need): gathers the
 * K and V blocks each table selects into compact buffers. Block
 * tables[b,g,t] (t < counts[b,g]) of K / V is copied to rows
 * [t*blk, (t+1)*blk) of Kc / Vc; entries outside [0, nKVmax) give zero rows;
 * rows at t >= counts[b,g] are not written.
 * K, V, Kc, Vc bf16 [B, H_kv, L_max, D] (16-byte aligned); tables / counts as
 * for ca_chunk_attention. Errors: CA_ERR_INVALID_ARG, CA_ERR_SHAPE,
 * CA_ERR_ALIGN, CA_ERR_UNSUPPORTED, CA_ERR_CUDA.
 */
int ca_compact_kv_blocks(const void *K, const void *V, const int32_t *tables,
                         const int32_t *counts, int B, int H_kv, int L_max, int D, int blk,
                         void *Kc, void *Vc, void *stream);

/*
 * Explicit-compaction ablation, step 2: ca_chunk_attention over the compact
 * buffers of ca_compact_kv_blocks — block t of a table is read from rows
 * [t*blk, (t+1)*blk) of Kc / Vc and masked by its original position
 * tables[b,g,t]*blk. Same arguments, results and errors as
 * ca_chunk_attention, with Kc / Vc in place of K / V.
 */
int ca_compacted_chunk_attention(const void *Q, const void *Kc, const void *Vc,
                                 const int32_t *tables, const int32_t *counts,
                                 const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                                 int L_max, int D, int blk, float scale, void *O, float *LSE,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Per-tile block-sparse ablation (pages: "Problem", block-sparse kernels that
 * execute the 2D mask directly in the Q << KV regime, and the efficiency
 * ablation under "Experimental results"): every query head and Q-block
 * attends to its own selected blocks, with no Q-block or intra-group union:
 *   K_set(b, h, r) = { k : mask[b, h, r / blk, k / blk] != 0, k <= p }.
 *
 * Q-blocks per span: the per-tile kernel processes 256 chunk rows of one head
 * per work item, so its tables group each head's Q-blocks in spans of
 * 256 / blk. Returns that number (2 for blk 128, 4 for blk 64), 0 if blk is
 * unsupported.
 */
int ca_tile_span(int blk);

/*
 * Per-tile ablation, step 1: span tables from the mask. For each (b, h,
 * span s), nS = ceil(nQ / span) spans with span = ca_tile_span(blk):
 *   tables[b, h, s, 0 : counts[b, h, s]] = ascending KV blocks j that some
 *   Q-block i = span * s + u (u < span, i < nQ) selects, each stored as
 *   j | (bit u set iff mask[b, h, span * s + u, j] != 0) << 24;
 *   tables[b, h, s, counts[b, h, s] :] = -1.
 * mask    device uint8 [B, H_q, nQ, nKVmax], nonzero = selected
 * tables  device int32 [B, H_q, nS, nKVmax] (written), counts int32
 *         [B, H_q, nS] (written); caller-owned, 4-byte aligned.
 * Requires nKVmax < 2^24. Errors: CA_ERR_INVALID_ARG, CA_ERR_SHAPE,
 * CA_ERR_ALIGN, CA_ERR_UNSUPPORTED (blk), CA_ERR_CUDA.
 */
int ca_build_tile_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int blk,
                         int32_t *tables, int32_t *counts, void *stream);

/*
 * Per-tile ablation, step 2: attention over the span tables of
 * ca_build_tile_tables, read in place from the cache. A work item holds two
 * 128-row tiles of one query head and walks its span's table; a tile's rows
 * skip (P = 0) every block their own Q-block did not select, so the result is
 * per-tile block-sparse attention. Each head loads its own K/V blocks (no
 * sharing across the GQA group). Arguments and errors as ca_chunk_attention,
 * with tables / counts shaped [B, H_q, nS, L_max / blk] / [B, H_q, nS],
 * nS = ceil(C / 256) (the mask had nQ = ceil(C / blk) Q-blocks); requires
 * L_max / blk < 2^24.
 */
int ca_tile_chunk_attention(const void *Q, const void *K, const void *V, const int32_t *tables,
                            const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                            int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                            float *LSE, void *workspace, size_t workspace_bytes, void *stream);

/*
 * ca_chunk_attention without a caller workspace, for callers that cannot
 * allocate device memory when they run attention (an engine whose device
 * memory is sized once at start-up, code inside a fixed memory pool, a host
 * path that must not enter the allocator). The paper has no counterpart: this
 * is a deployment convenience of this library.
 *
 * Same arguments, results and host-side error codes as ca_chunk_attention
 * minus the workspace (the checks run before anything is enqueued, so a
 * rejected call touches nothing on the GPU); it allocates nothing (no
 * cudaMalloc / cudaFree, no allocating library call).
 * The scratch it needs comes from a fixed 4096-byte array inside the library,
 * held by every GPU that loads the library until the process exits. That
 * holds the status word and header the kernels need at minimum, not the
 * partial results of the last-wave split, so calls through this entry point
 * always run unsplit (same results within rounding, sometimes slower).
 * The first call on each device looks up that device's copy of the array
 * (cudaGetSymbolAddress, with that device current), so make that first call
 * before any stream capture. Every call on a device shares the one array:
 * calls that overlap on the GPU (for example on two streams at once) race, so
 * serialise them. Each call clears the device status word first; if
 * device_status (a device pointer to one uint32, or NULL) is given, the call
 * copies the final status word there on the same stream: bit 0 set = an
 * invalid table or count was found, bit 1 set = a bounded wait expired.
 */
int ca_chunk_attention_noalloc(const void *Q, const void *K, const void *V, const int32_t *tables,
                               const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                               int H_kv, int C, int L_max, int D, int blk, float scale, void *O,
                               float *LSE, unsigned int *device_status, void *stream);

/*
 * Merge of attention results over disjoint key sets. The CompactAttention
 * pages do not describe split-KV; this is the standard log-sum-exp identity
 * split-KV execution rests on (one query row's attention cut over several
 * segments of its table, each segment normalised on its own), the same one
 * ca_chunk_attention applies inside a launch to its last-wave segments, here
 * for results of separate calls (other tables, streams or GPUs).
 * Each part i holds, for the same query rows, O_i normalised over its own
 * keys and LSE_i = ln sum exp(score) over them (natural log, the convention of
 * ca_chunk_attention's LSE output). The merged result is attention over the
 * union of the key sets:
 *     LSE[r]   = ln sum_i exp(LSE_i[r])
 *     O[r, :]  = sum_i exp(LSE_i[r] - LSE[r]) * O_i[r, :]
 * computed in fp32 with the largest LSE_i[r] subtracted first. A part with
 * LSE_i[r] = -inf (no visible key) has weight 0; if every part has -inf the
 * row gets O = 0, LSE = -inf. LSE_i must be finite or -inf.
 *
 * O_a, O_b, O  bf16 [rows, D] row-major (any leading shape flattened to rows,
 *              e.g. [B, H_q, C] of ca_chunk_attention), 16-byte aligned;
 * LSE_a, LSE_b fp32 [rows], 4-byte aligned; LSE fp32 [rows] or NULL (not
 *              written). O may be the same buffer as O_a or O_b (in place) and
 *              LSE the same as LSE_a or LSE_b; partial overlaps are not allowed.
 * D: a multiple of 8, at most 2048. rows == 0 is a no-op. All pointers are
 * device memory owned by the caller; the call is asynchronous on `stream`.
 * Errors: CA_ERR_INVALID_ARG (NULL input / negative rows / D <= 0),
 * CA_ERR_SHAPE (D not a multiple of 8), CA_ERR_UNSUPPORTED (D > 2048),
 * CA_ERR_ALIGN, CA_ERR_CUDA (launch failure).
 */
int ca_merge_attention_states(const void *O_a, const float *LSE_a, const void *O_b,
                              const float *LSE_b, long long rows, int D, void *O, float *LSE,
                              void *stream);

/* The same merge over n parts (2 <= n <= 8, else CA_ERR_UNSUPPORTED; n == 1
 * is CA_ERR_INVALID_ARG). O_parts / LSE_parts are HOST arrays of n device
 * pointers (read during the call only), each part laid out as O_a / LSE_a
 * above. One pass over the data: no intermediate rounding to bf16. */
int ca_merge_attention_states_n(const void *const *O_parts, const float *const *LSE_parts, int n,
                                long long rows, int D, void *O, float *LSE, void *stream);

/* Self-test of the kernels' bounded waits: one kernel waits on a barrier that
 * nothing ever completes; after limit_cycles SM clock cycles (at most about
 * 2 s) the wait gives up, sets the timeout bit of the workspace status word
 * and the kernel returns. ca_read_device_status() then reports CA_ERR_TIMEOUT
 * and the context stays usable. Nothing faults, traps or hangs. */
int ca_selftest_bounded_wait(void *workspace, long long limit_cycles, void *stream);

/* Synchronises `stream`, then reads the workspace status word written by the
 * kernels: CA_OK, CA_ERR_TABLE or CA_ERR_TIMEOUT (sticky until the workspace is
 * zeroed again; CA_ERR_TABLE wins if both are set). CA_ERR_CUDA if the stream
 * reports an error. Meant for tests and debugging, not the hot path. */
int ca_read_device_status(const void *workspace, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* COMPACTATTN_H */
