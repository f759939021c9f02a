/*
 * s2attn.h -- C ABI of the B200 (sm_100a) HHST sparse-attention library.
 *
 * The operation. "S2-Attention: Hardware-aware context sharding among attention
 * heads" (OpenReview forum page, Abstract, and the arXiv 2407.17678 abstract)
 * introduces the Head-Heterogenous Strided Transformer (HHST): attention is
 * restricted per head to a strided subset of the context plus a local window,
 * different heads take different subsets so that together they cover all of
 * it, and dense heads may be mixed in ("hybrid"). The pages state the pattern
 * only in words; this library uses the explicit block rule
 *
 *     key block j is active for (head h, query block i)  iff  j <= i and
 *     (dense[h]  or  i - j < L  or  (j + h) mod S == 0)
 *
 * with block size B (query block i = q / B, key block j = k / B), vertical
 * stride S and L local blocks, plus token-level causality (k <= q) inside the
 * diagonal block. The result is exact softmax attention under that mask:
 * O[q] = sum_k softmax_k(scale * Q[q].K[k]) V[k] over the visible keys k.
 *
 * Conventions for every entry point:
 *  - Returns an int status (S2_OK = 0, else one of the S2_ERR_* codes). No C++
 *    exception crosses the ABI. A call that returns an error launches nothing.
 *  - The caller owns every buffer. No call allocates, frees or synchronises
 *    device memory (s2_device_status is the one synchronous call). The library
 *    does hold three fixed file-scope device arrays on every GPU that loads it,
 *    until the process exits: the error flags, 1024 work-counter slots (16 KB)
 *    and the 8 MiB scratch of s2_attn_decode_noalloc (see there).
 *  - Device pointers must stay valid until the work queued on `stream` ends.
 *    `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Launches are asynchronous.
 *  - Launches on different streams may overlap. The persistent kernels
 *    (prefill, chunked prefill, backward) take their work items from a counter
 *    slot that each launch owns from start to end; slots are handed out in
 *    turn, and a launch whose slot is still held by an earlier launch that has
 *    not finished waits for it (within the wait bound below, after which its
 *    CTAs stop taking items and S2_ERR_TIMEOUT is reported). So any number of
 *    launches may be in flight at once without sharing counters. The one
 *    shared buffer is the scratch of s2_attn_decode_noalloc.
 *  - The device addresses of those arrays are looked up once per device and
 *    kept for the life of the process: after cudaDeviceReset, or anything else
 *    that replaces the device's primary context, unload and reload the library.
 *  - `scale` (the logits' multiplier) 0 selects 1/sqrt(head_dim).
 *  - Tensors are bf16 (IEEE bfloat16 bit patterns in uint16 storage), dense and
 *    row-major with the innermost dimension last, 16-byte aligned.
 *  - Device waits inside the kernels are bounded. A wait that runs out sets a
 *    device flag that s2_device_status reports as S2_ERR_TIMEOUT. While that
 *    flag is set, any kernel wait that is not already satisfied gives up at
 *    once (so one stuck CTA does not stall the rest); s2_device_status(1, ...)
 *    clears it.
 */
#ifndef S2ATTN_H
#define S2ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    S2_OK = 0,
    S2_ERR_INVALID_ARG = 1, /* a null pointer, a bad size, or a malformed layout */
    S2_ERR_UNSUPPORTED = 2, /* head_dim, block size or page size outside the built set;
                               no sm_100 device */
    S2_ERR_CAPACITY = 3,    /* an output array or workspace is too small */
    S2_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed */
    S2_ERR_TIMEOUT = 5,     /* a bounded device wait ran out (s2_device_status) */
    S2_ERR_DEVICE_INDEX = 6 /* a kernel met an index outside its buffers and skipped it
                               (s2_device_status) */
};

/* Human-readable name of a status code (static storage, never NULL). */
const char* s2_status_string(int status);

/* ------------------------------------------------------------------------ */
/* Layout builder (host only)                                                */
/* ------------------------------------------------------------------------ */

/* Parameters of one HHST layout (the block rule in the file header). */
typedef struct s2_layout_desc {
    int32_t num_heads;       /* H >= 1 */
    int32_t block_size;      /* B >= 1 tokens per query/key block */
    int32_t vertical_stride; /* S >= 1 */
    int32_t local_blocks;    /* L >= 1 (so every row holds its diagonal block) */
    int32_t num_blocks;      /* nb >= 1 query/key blocks (ceil(seq / B)) */
    const uint8_t* dense_head_mask; /* host, [num_heads], nonzero = dense causal head;
                                       NULL = no dense heads */
} s2_layout_desc;

/*
 * Build the per-head compacted key-block index lists (CSR) of a layout.
 *
 * Two-call protocol: with col_idx == NULL only *nnz_out is set (row_ptr is
 * still filled when non-NULL). Otherwise:
 *   row_ptr [H * (nb + 1)] (host, written): row_ptr[h*(nb+1) + i] is the offset
 *     into col_idx of the list for (head h, query block i); the list ends at
 *     row_ptr[h*(nb+1) + i + 1]. Offsets are global across heads, so
 *     row_ptr[h*(nb+1) + nb] == row_ptr[(h+1)*(nb+1)] and row_ptr[0] == 0.
 *   col_idx [col_idx_cap] (host, written): active key blocks j, ascending within
 *     each list, so the diagonal block i is always last.
 *   *nnz_out = total entries. S2_ERR_CAPACITY when col_idx_cap < nnz, or when
 *   nnz exceeds INT32_MAX (offsets are int32).
 * S2_ERR_INVALID_ARG for a NULL desc or nnz_out, a parameter out of range, or
 * col_idx given without row_ptr. The lists are enumerated directly (cost
 * O(nnz)); call once per layout and copy the arrays to the device.
 */
int s2_build_layout(const s2_layout_desc* desc, int32_t* row_ptr, int32_t* col_idx,
                    int64_t col_idx_cap, int64_t* nnz_out);

/* One context range of a head's pattern (s2_build_layout_ranges). */
typedef struct s2_context_range {
    int32_t end_block;       /* exclusive end on the key-block axis; strictly ascending within
                                a head, the head's last range ends at num_blocks */
    int32_t vertical_stride; /* S >= 0; 0 = the range has no strided blocks */
    int32_t local_blocks;    /* L >= 0 */
    int32_t dense;           /* nonzero = every causal block of the range is active */
} s2_context_range;

/*
 * Layouts customised per head and per context range. The arXiv abstract of
 * "S2-Attention: Hardware-aware context sharding among attention heads" says
 * the patterns can be set at both levels and gives no formula; the reading
 * here: head h's ranges, ranges[range_ptr[h]] .. ranges[range_ptr[h+1] - 1],
 * cut its key-block axis [0, num_blocks) into consecutive pieces, and key
 * block j <= i is active for query block i of head h iff, with the (S, L,
 * dense) of the range that holds j,
 *
 *     dense  or  i - j < L  or  (S > 0 and (j + h) mod S == 0).
 *
 * One range [0, nb) with S >= 1, L >= 1 is the HHST rule of s2_build_layout.
 * A dense first range gives every head the opening blocks of the context; a
 * range with S = 0 keeps only its local window.
 *
 *   range_ptr  host int32 [num_heads + 1] (read): range_ptr[0] == 0, at least
 *              one range per head (range_ptr[h] < range_ptr[h+1]).
 *   ranges     host [range_ptr[num_heads]] (read).
 * Output arrays, the two-call protocol and S2_ERR_CAPACITY as s2_build_layout.
 * A list may be empty (a range pattern may leave a query block with no key):
 * the kernels then write a zero output row and LSE = -inf for its queries.
 * S2_ERR_INVALID_ARG for NULL pointers, num_heads or num_blocks < 1, and
 * ranges that are empty, not ascending, do not end at num_blocks, or have a
 * negative S or L. Cost O(nnz + number of ranges * num_blocks).
 */
int s2_build_layout_ranges(int32_t num_heads, int32_t num_blocks, const int32_t* range_ptr,
                           const s2_context_range* ranges, int32_t* row_ptr,
                           int32_t* col_idx, int64_t col_idx_cap, int64_t* nnz_out);

/*
 * Layout from any per-head block mask (the generic form of a per-head
 * pattern): block_mask is host uint8 [num_heads][num_blocks][num_blocks],
 * nonzero at [h][i][j] when key block j is active for query block i of head
 * h. Causality inside the diagonal block is still applied by the kernels.
 * Entries above the diagonal (j > i) must be zero: the kernels treat every
 * listed block other than the diagonal as fully visible, so such an entry is
 * rejected with S2_ERR_INVALID_ARG rather than silently dropped. Output
 * arrays, the two-call protocol and S2_ERR_CAPACITY as s2_build_layout; lists
 * may be empty as in s2_build_layout_ranges. Cost O(num_heads * num_blocks^2).
 */
int s2_build_layout_mask(int32_t num_heads, int32_t num_blocks, const uint8_t* block_mask,
                         int32_t* row_ptr, int32_t* col_idx, int64_t col_idx_cap,
                         int64_t* nnz_out);

/*
 * Transposed lists for the backward pass: for each head h and key block j,
 * the ascending query blocks i whose list (in row_ptr/col_idx, from any of
 * the builders above) holds j.
 *   row_ptr, col_idx, nnz  host layout (read); lists must be strictly
 *                          ascending with 0 <= j <= i and global offsets.
 *   col_ptr  host int32 [num_heads * (num_blocks + 1)] (written): global
 *            offsets into row_idx, col_ptr[h*(nb+1) + j] .. col_ptr[h*(nb+1) + j + 1].
 *   row_idx  host int32 [nnz] (written).
 * S2_ERR_INVALID_ARG for NULL pointers or a malformed layout. Cost O(nnz + H nb).
 */
int s2_build_layout_transpose(int32_t num_heads, int32_t num_blocks, const int32_t* row_ptr,
                              const int32_t* col_idx, int64_t nnz, int32_t* col_ptr,
                              int32_t* row_idx);

/*
 * Key tiles of the backward for block_size 64: the dK/dV kernel works on
 * 128-row key tiles of two 64-row key blocks and walks the union of their
 * transposed lists, so blocks whose lists overlap should share a tile. Per
 * head, blocks are ordered by transposed-list length (longest first, ties by
 * j) and paired consecutively (under HHST: strided blocks j and j + S, and
 * neighbouring local-only blocks).
 *   col_ptr    host transposed offsets from s2_build_layout_transpose (read).
 *   key_tiles  host int32 [num_heads][ceil(num_blocks / 2)][2] (written): the
 *              two key blocks of each tile; -1 for the missing second block
 *              when num_blocks is odd. Every block appears exactly once.
 * S2_ERR_INVALID_ARG for NULL pointers, sizes < 1 or decreasing offsets.
 */
int s2_build_key_tiles(int32_t num_heads, int32_t num_blocks, const int32_t* col_ptr,
                       int32_t* key_tiles);

/* ------------------------------------------------------------------------ */
/* Prefill: block-sparse causal attention over whole sequences               */
/* ------------------------------------------------------------------------ */

/*
 * O = HHST-masked softmax(scale * Q K^T) V for every query row.
 *
 * "S2-Attention: Hardware-aware context sharding among attention heads"
 * (OpenReview forum page, Abstract): each head attends to its own strided
 * share of the context plus a local window, the heads together cover it, and
 * the sparsity turns into wall-clock speed only through a FlashAttention-style
 * kernel that works at the block granularity of the pattern. This is that
 * forward pass over whole sequences (training and prefill).
 *
 *   q, k, v   device bf16 [batch][heads][seq][head_dim] (read).
 *   o         device bf16 [batch][heads][seq][head_dim] (written).
 *   lse       device fp32 [batch][heads][seq] or NULL: natural-log
 *             log-sum-exp of the scaled visible logits of each row (written).
 *   head_dim  64 or 128.  block_size 64 or 128.  Any seq >= 1: the last
 *             block may be partial (its missing keys are never visible).
 *   num_blocks == ceil(seq / block_size).
 *   row_ptr, col_idx, nnz: a layout from one of the s2_build_layout*
 *             builders for (heads, num_blocks), copied to device memory
 *             (read). Lists must be strictly ascending with j <= i; nnz may be
 *             0 (then col_idx may be NULL). A query row whose list is empty
 *             gets a zero output row and LSE = -inf.
 *   scale     multiplier of the logits, > 0; 0 selects 1/sqrt(head_dim).
 * Runs tcgen05 tensor-core tiles of 128 query rows; only the listed key blocks
 * are visited and causality is applied inside the diagonal block only.
 * num_blocks is at most 2046 (union lists are staged in shared memory).
 */
int s2_attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                    int32_t batch, int32_t heads, int32_t seq, int32_t head_dim,
                    float scale, int32_t block_size, int32_t num_blocks,
                    const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                    void* stream);

/*
 * s2_attn_prefill with grouped key/value heads (GQA/MQA; the pages do not
 * mention it): k and v are [batch][heads_kv][seq][head_dim], heads_kv divides
 * heads, and query head h reads key/value head h / (heads / heads_kv). The
 * layout (rows per query head) is applied per query head, so heads of one
 * group may visit different key blocks. heads_kv == heads is s2_attn_prefill.
 * S2_ERR_INVALID_ARG when heads_kv < 1 or does not divide heads.
 */
int s2_attn_prefill_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                        int32_t batch, int32_t heads, int32_t heads_kv, int32_t seq,
                        int32_t head_dim, float scale, int32_t block_size, int32_t num_blocks,
                        const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                        void* stream);

/* ------------------------------------------------------------------------ */
/* Chunked prefill: a chunk of queries per sequence over a paged KV cache    */
/* ------------------------------------------------------------------------ */

/*
 * Each sequence s appends a chunk of q_start[s+1] - q_start[s] query tokens at
 * the end of its context of ctx_lens[s] tokens, whose keys and values (the
 * chunk's own included) are already in the paged cache. Chunk row t of
 * sequence s sits at position ctx_lens[s] - (q_start[s+1] - t) and attends to
 * keys 0..position under the layout (query block = position / block_size),
 * with token causality inside the diagonal block: the prefill definition
 * restricted to the chunk rows. One-token chunks are decode. Serving prefills
 * long prompts this way; the arXiv abstract of "S2-Attention: Hardware-aware
 * context sharding among attention heads" reports 7B inference in vLLM, and
 * PagedAttention is in its reference list.
 *
 *   q            device bf16 [total_q][heads][head_dim] (read): packed rows.
 *   k_cache,     device bf16 [num_pages][heads_kv][page_size][head_dim] (read),
 *   v_cache      as s2_attn_decode_gqa (heads_kv divides heads).
 *   block_table  device int32 [batch][max_pages] (read).
 *   ctx_lens     device int32 [batch] (read): context length including the chunk.
 *   q_start      device int32 [batch + 1] (read): q_start[0] = 0, ascending,
 *                q_start[batch] = total_q, and each chunk no longer than
 *                max_q_len or its context.
 *   max_q_len    host bound on the chunk lengths (sizes the grid).
 *   page_size 16. head_dim 64 or 128. block_size 64 or 128.
 *   row_ptr, col_idx, nnz, num_blocks: device layout covering the longest
 *                context ((ctx_len - 1) / block_size < num_blocks).
 *   out          device bf16 [total_q][heads][head_dim] (written).
 *   lse          device fp32 [total_q][heads] or NULL (written).
 * Cache rows past a context inside its last page may hold anything: the
 * kernel never lets them reach the output. A sequence whose q_start, length
 * or page ids are out of range is skipped and reported by s2_device_status as
 * S2_ERR_DEVICE_INDEX. Errors before launch: S2_ERR_INVALID_ARG (null
 * pointers, sizes, alignment, scale), S2_ERR_UNSUPPORTED (head_dim,
 * block_size, page_size, num_blocks > 2046, sizes past the int32 ranges).
 */
int s2_attn_chunk_prefill(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_table, const int32_t* ctx_lens,
                          const int32_t* q_start, int32_t batch, int32_t heads, int32_t heads_kv,
                          int32_t head_dim, int32_t page_size, int32_t max_pages,
                          int64_t num_pages, int32_t max_q_len, int64_t total_q,
                          int32_t block_size, int32_t num_blocks, const int32_t* row_ptr,
                          const int32_t* col_idx, int64_t nnz, float scale, void* out,
                          float* lse, void* stream);

/* ------------------------------------------------------------------------ */
/* Backward: gradients of the prefill                                        */
/* ------------------------------------------------------------------------ */

/* Bytes of device workspace s2_attn_backward needs: 8 bytes per query row,
 * rows padded to a multiple of 128 per (batch, head). */
size_t s2_attn_backward_workspace_size(int32_t batch, int32_t heads, int32_t seq);

/*
 * dQ, dK, dV of s2_attn_prefill. The arXiv abstract of "S2-Attention:
 * Hardware-aware context sharding among attention heads" reports training
 * speedups; the gradients are those of the same masked softmax attention:
 * with P = exp(scale Q K^T - LSE) over the visible keys and D = rowsum(dO * O),
 *     dV = P^T dO,   dS = P * (dO V^T - D),   dQ = scale dS K,   dK = scale dS^T Q.
 *
 *   q, o        device bf16 [batch][heads][seq][head_dim] (read): the forward's
 *               queries and output.
 *   k, v        device bf16 [batch][heads_kv][seq][head_dim] (read).
 *   dout        device bf16 [batch][heads][seq][head_dim] (read): dL/dO.
 *   lse         device fp32 [batch][heads][seq] (read): the forward's LSE.
 *   dq          device bf16 [batch][heads][seq][head_dim] (written).
 *   dk, dv      device bf16 [batch][heads_kv][seq][head_dim] (written): with
 *               grouped heads (heads_kv < heads, query head h reading K/V head
 *               h / (heads / heads_kv)) they sum over the group's query heads.
 *   heads_kv    divides heads; a group is at most 16 query heads and, when
 *               heads_kv < heads, (heads / heads_kv) * num_blocks <= 4096
 *               (S2_ERR_UNSUPPORTED otherwise).
 *   seq, head_dim, scale, block_size, num_blocks: as s2_attn_prefill.
 *   row_ptr, col_idx, nnz  device layout the forward used (read).
 *   col_ptr, row_idx       device transposed layout from
 *                          s2_build_layout_transpose (read).
 *   key_tiles              device key tiles from s2_build_key_tiles (read;
 *                          required when block_size is 64, ignored otherwise).
 *   workspace   device, >= s2_attn_backward_workspace_size(batch, heads, seq)
 *               bytes, 256-byte aligned (scratch, clobbered).
 * Runs three kernels: row statistics (D, LSE in the log2 domain), dQ over the
 * query tiles' key-block lists, and dK/dV over the key tiles' transposed
 * lists; S and dP are recomputed by both, so no accumulator is shared between
 * CTAs (no atomics; results are deterministic). Rows with an empty list get
 * zero gradients. Errors: S2_ERR_INVALID_ARG (null pointers, sizes, alignment,
 * a bad scale), S2_ERR_CAPACITY (workspace too small), S2_ERR_UNSUPPORTED
 * (head_dim, block_size, group limits above), S2_ERR_CUDA (launch failure).
 */
int s2_attn_backward(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     int32_t batch, int32_t heads, int32_t heads_kv, int32_t seq,
                     int32_t head_dim, float scale, int32_t block_size, int32_t num_blocks,
                     const int32_t* row_ptr, const int32_t* col_idx, const int32_t* col_ptr,
                     const int32_t* row_idx, const int32_t* key_tiles, int64_t nnz,
                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode: one query token per sequence over a paged KV cache               */
/* ------------------------------------------------------------------------ */

/* Bytes of device workspace s2_attn_decode needs for this shape and split
 * count (num_splits <= 0 means the automatic choice for this shape). */
size_t s2_attn_decode_workspace_size(int32_t batch, int32_t heads, int32_t head_dim,
                                     int32_t num_splits);

/* The split count s2_attn_decode uses when given num_splits <= 0: about one
 * wave of resident CTAs on a B200, ceil(370 / (batch * heads)), at most 16.
 * (With up to 256 sequences the split kernel starts the sequences with the
 * longest contexts first, which evens out the last wave.) */
int32_t s2_attn_decode_auto_splits(int32_t batch, int32_t heads);

/*
 * Split-KV decode: for each sequence s and head h, the query at position
 * n-1 (n = ctx_lens[s]) attends to keys 0..n-1 of its own context under the
 * same block rule (query block i = (n-1) / block_size).
 *
 * The inference side of "S2-Attention: Hardware-aware context sharding among
 * attention heads" (arXiv abstract on the mlsanity index page: a 7B HHST model
 * served through vLLM runs 4.5x faster than its dense counterpart;
 * PagedAttention is in its reference list): one new token per sequence over a
 * paged KV cache, reading only the active blocks. The splits of a context are
 * merged by the log-sum-exp rule (online softmax as an associative reduction,
 * the LeanAttention summary on the SampleAttention page).
 *
 *   q            device bf16 [batch][heads][head_dim] (read).
 *   k_cache,     device bf16 [num_pages][heads][page_size][head_dim] (read):
 *   v_cache      token t of sequence s is row t % page_size of physical page
 *                block_table[s][t / page_size].
 *   block_table  device int32 [batch][max_pages] (read); entries past a
 *                sequence's last page are ignored (-1 by convention).
 *   ctx_lens     device int32 [batch] (read), 1 <= n <= min(max_pages *
 *                page_size, num_blocks * block_size).
 *   page_size 16.  head_dim 64 or 128.  block_size a multiple of page_size.
 *   row_ptr, col_idx, nnz: device layout for (heads, num_blocks) from one of
 *                the s2_build_layout* builders; an empty list gives a zero
 *                output and LSE = -inf.
 *   scale        multiplier of the logits, any finite value; 0 selects
 *                1/sqrt(head_dim).
 *   out          device bf16 [batch][heads][head_dim] (written).
 *   lse          device fp32 [batch][heads] or NULL (written).
 *   workspace    device, >= s2_attn_decode_workspace_size(...) bytes, 256-byte
 *                aligned; holds per-split partial results (scratch, clobbered).
 * A ctx_lens entry out of range, or a block-table entry outside [0, num_pages)
 * inside a context, is skipped by the kernel and reported by s2_device_status
 * as S2_ERR_DEVICE_INDEX.
 */
int s2_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_table, const int32_t* ctx_lens,
                   int32_t batch, int32_t heads, int32_t head_dim, int32_t page_size,
                   int32_t max_pages, int64_t num_pages, int32_t block_size,
                   int32_t num_blocks, const int32_t* row_ptr, const int32_t* col_idx,
                   int64_t nnz, float scale, void* out, float* lse,
                   void* workspace, size_t workspace_bytes, int32_t num_splits,
                   void* stream);

/*
 * s2_attn_decode with grouped key/value heads: the caches are
 * [num_pages][heads_kv][page_size][head_dim] and query head h reads key/value
 * head h / (heads / heads_kv) (heads_kv divides heads; S2_ERR_INVALID_ARG
 * otherwise). Each query head walks its own layout row, so one group's heads
 * may read different pages. heads_kv == heads is s2_attn_decode.
 */
int s2_attn_decode_gqa(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_table, const int32_t* ctx_lens,
                       int32_t batch, int32_t heads, int32_t heads_kv, int32_t head_dim,
                       int32_t page_size, int32_t max_pages, int64_t num_pages,
                       int32_t block_size, int32_t num_blocks, const int32_t* row_ptr,
                       const int32_t* col_idx, int64_t nnz, float scale, void* out,
                       float* lse, void* workspace, size_t workspace_bytes,
                       int32_t num_splits, void* stream);

/*
 * Decode that allocates nothing: s2_attn_decode with the split partials kept
 * in a scratch array inside the library instead of a caller workspace.
 *
 * This entry point has no counterpart in the paper; it exists for callers that
 * cannot call cudaMalloc: plug-ins whose host framework owns every device
 * allocation and gives them none, C programs that link this library without a
 * device allocator of their own, and latency-critical loops that must not
 * allocate or free because cudaMalloc and cudaFree can synchronise the device.
 *
 * Arguments, layouts and results are those of s2_attn_decode, without
 * workspace and workspace_bytes. The scratch is a file-scope device array of
 * S2_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU loading the library holds
 * until the process exits. A shape whose partials need more than that
 * (s2_attn_decode_workspace_size(batch, heads, head_dim, num_splits) >
 * S2_NOALLOC_SCRATCH_BYTES) is rejected with S2_ERR_CAPACITY before anything
 * runs. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. All calls share the one array, which keeps the
 * last call's contents (nothing in it has to start at zero): calls that can
 * overlap on the GPU, on different streams, race on it and must be ordered by
 * the caller. The function calls no cudaMalloc, cudaFree or other allocating
 * routine.
 */
#define S2_NOALLOC_SCRATCH_BYTES (8u << 20)
int s2_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_table, const int32_t* ctx_lens,
                           int32_t batch, int32_t heads, int32_t head_dim, int32_t page_size,
                           int32_t max_pages, int64_t num_pages, int32_t block_size,
                           int32_t num_blocks, const int32_t* row_ptr, const int32_t* col_idx,
                           int64_t nnz, float scale, void* out, float* lse,
                           int32_t num_splits, void* stream);

/* ------------------------------------------------------------------------ */
/* Device status and limits                                                  */
/* ------------------------------------------------------------------------ */

/*
 * Synchronise the current device and report the kernels' error flags:
 * S2_OK, S2_ERR_TIMEOUT (a bounded wait ran out) or S2_ERR_DEVICE_INDEX (an
 * index was out of range and skipped). *flags_out (may be NULL) receives the
 * raw bit set (1 = timeout, 2 = index). reset != 0 clears the flags and, when
 * a timeout was flagged, also frees every work-counter slot (a launch that
 * timed out may not have released its own); call it while no other thread is
 * launching this library's kernels on the device.
 */
int s2_device_status(int reset, uint32_t* flags_out);

/* Bound, in nanoseconds, of every device wait in kernels launched after this
 * call (process-wide; default 2e9). 0 makes any wait that is not already
 * satisfied give up at once, which tests use to exercise the timeout path. */
int s2_set_wait_timeout_ns(uint64_t ns);

/* Library version string. */
const char* s2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H */
