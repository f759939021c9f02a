// layout.cpp -- host builders of the per-head compacted key-block lists (CSR).
//
// HHST ("S2-Attention: Hardware-aware context sharding among attention heads",
// Abstract) gives each head its own strided share of the context plus a local
// window. For head h and query block i the active key blocks are
//   the L local blocks  max(0, i-L+1) .. i, and
//   the strided blocks  j < i-L+1 with j = -h (mod S),
// or every block 0..i for a dense head. This file enumerates them directly in
// ascending order (strided ones first, then the local run), which is O(nnz)
// rather than a test of every (i, j) pair, and emits CSR offsets.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <vector>

#include "s2attn.h"

namespace {

// Number of active blocks in row (h, i).
int64_t row_count(int64_t h, int64_t i, int64_t S, int64_t L, bool dense)
{
    if (dense) return i + 1;
    const int64_t lo = i - L + 1 > 0 ? i - L + 1 : 0;  // first local block
    const int64_t first = (S - h % S) % S;             // smallest j >= 0 with (j+h) % S == 0
    const int64_t strided = lo > first ? (lo - 1 - first) / S + 1 : 0;
    return strided + (i - lo + 1);
}

// Write the ascending list of row (h, i) to out; returns the count.
int64_t row_fill(int64_t h, int64_t i, int64_t S, int64_t L, bool dense, int32_t* out)
{
    int64_t n = 0;
    if (dense) {
        for (int64_t j = 0; j <= i; ++j) out[n++] = (int32_t)j;
        return n;
    }
    const int64_t lo = i - L + 1 > 0 ? i - L + 1 : 0;
    for (int64_t j = (S - h % S) % S; j < lo; j += S) out[n++] = (int32_t)j;
    for (int64_t j = lo; j <= i; ++j) out[n++] = (int32_t)j;
    return n;
}

}  // namespace

extern "C" int s2_build_layout(const s2_layout_desc* d, int32_t* row_ptr, int32_t* col_idx,
                               int64_t col_idx_cap, int64_t* nnz_out)
{
    if (!d || !nnz_out) return S2_ERR_INVALID_ARG;
    const int64_t H = d->num_heads, B = d->block_size, S = d->vertical_stride,
                  L = d->local_blocks, nb = d->num_blocks;
    if (H < 1 || B < 1 || S < 1 || L < 1 || nb < 1) return S2_ERR_INVALID_ARG;
    if (col_idx && !row_ptr) return S2_ERR_INVALID_ARG;

    int64_t nnz = 0;
    for (int64_t h = 0; h < H; ++h) {
        const bool dense = d->dense_head_mask && d->dense_head_mask[h] != 0;
        for (int64_t i = 0; i < nb; ++i) nnz += row_count(h, i, S, L, dense);
    }
    *nnz_out = nnz;
    if (nnz > INT32_MAX) return S2_ERR_CAPACITY;  // offsets are int32
    if (!row_ptr) return S2_OK;

    int64_t off = 0;
    for (int64_t h = 0; h < H; ++h) {
        const bool dense = d->dense_head_mask && d->dense_head_mask[h] != 0;
        for (int64_t i = 0; i < nb; ++i) {
            row_ptr[h * (nb + 1) + i] = (int32_t)off;
            off += row_count(h, i, S, L, dense);
        }
        row_ptr[h * (nb + 1) + nb] = (int32_t)off;
    }
    if (!col_idx) return S2_OK;
    if (col_idx_cap < nnz) return S2_ERR_CAPACITY;

    for (int64_t h = 0; h < H; ++h) {
        const bool dense = d->dense_head_mask && d->dense_head_mask[h] != 0;
        for (int64_t i = 0; i < nb; ++i)
            row_fill(h, i, S, L, dense, col_idx + row_ptr[h * (nb + 1) + i]);
    }
    return S2_OK;
}

// ---------------------------------------------------------------------------
// Per-context-range layouts. The arXiv abstract of S2-Attention says patterns
// can be customised per head and per context range; here a head's key-block
// axis is cut into consecutive ranges with their own (S, L, dense), and key
// block j follows the range that holds it. Enumeration per (h, i) walks the
// ranges left to right and, inside each, emits the strided blocks below the
// local window and then the window itself, so lists come out ascending.
// ---------------------------------------------------------------------------

namespace {

// Visit the active blocks of row (h, i) under one range [a, b): dense, or the
// strided j = -h (mod S) below the window, then the window i-L+1 .. i.
template <class F>
void range_row(int64_t h, int64_t i, int64_t a, int64_t b, const s2_context_range& r, F&& emit)
{
    const int64_t hi = b < i + 1 ? b : i + 1;  // exclusive
    if (a >= hi) return;
    if (r.dense) {
        for (int64_t j = a; j < hi; ++j) emit(j);
        return;
    }
    const int64_t L = r.local_blocks, S = r.vertical_stride;
    int64_t lo = i - L + 1;  // first block of the local window
    if (lo < a) lo = a;
    if (lo > hi) lo = hi;
    if (S > 0) {
        const int64_t j0 = a + ((S - (a + h) % S) % S);  // first j >= a with (j + h) % S == 0
        for (int64_t j = j0; j < lo; j += S) emit(j);
    }
    for (int64_t j = lo; j < hi; ++j) emit(j);
}

int64_t range_row_count(int64_t h, int64_t i, int64_t a, int64_t b, const s2_context_range& r)
{
    const int64_t hi = b < i + 1 ? b : i + 1;
    if (a >= hi) return 0;
    if (r.dense) return hi - a;
    const int64_t L = r.local_blocks, S = r.vertical_stride;
    int64_t lo = i - L + 1;
    if (lo < a) lo = a;
    if (lo > hi) lo = hi;
    int64_t n = hi - lo;
    if (S > 0) {
        const int64_t j0 = a + ((S - (a + h) % S) % S);
        if (j0 < lo) n += (lo - 1 - j0) / S + 1;
    }
    return n;
}

// Shared second half of the builders: row offsets from per-row counts, then
// the lists. count(h, i) and fill(h, i, out) describe one row.
template <class Count, class Fill>
int emit_csr(int64_t H, int64_t nb, Count&& count, Fill&& fill, int32_t* row_ptr,
             int32_t* col_idx, int64_t col_idx_cap, int64_t* nnz_out)
{
    int64_t nnz = 0;
    for (int64_t h = 0; h < H; ++h)
        for (int64_t i = 0; i < nb; ++i) nnz += count(h, i);
    *nnz_out = nnz;
    if (nnz > INT32_MAX) return S2_ERR_CAPACITY;
    if (!row_ptr) return S2_OK;
    int64_t off = 0;
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t i = 0; i < nb; ++i) {
            row_ptr[h * (nb + 1) + i] = (int32_t)off;
            off += count(h, i);
        }
        row_ptr[h * (nb + 1) + nb] = (int32_t)off;
    }
    if (!col_idx) return S2_OK;
    if (col_idx_cap < nnz) return S2_ERR_CAPACITY;
    for (int64_t h = 0; h < H; ++h)
        for (int64_t i = 0; i < nb; ++i) fill(h, i, col_idx + row_ptr[h * (nb + 1) + i]);
    return S2_OK;
}

}  // namespace

extern "C" int s2_build_layout_ranges(int32_t num_heads, int32_t num_blocks,
                                      const int32_t* range_ptr, const s2_context_range* ranges,
                                      int32_t* row_ptr, int32_t* col_idx, int64_t col_idx_cap,
                                      int64_t* nnz_out)
{
    if (!range_ptr || !ranges || !nnz_out || num_heads < 1 || num_blocks < 1)
        return S2_ERR_INVALID_ARG;
    if (col_idx && !row_ptr) return S2_ERR_INVALID_ARG;
    const int64_t H = num_heads, nb = num_blocks;
    if (range_ptr[0] != 0) return S2_ERR_INVALID_ARG;
    for (int64_t h = 0; h < H; ++h) {
        const int32_t r0 = range_ptr[h], r1 = range_ptr[h + 1];
        if (r1 <= r0) return S2_ERR_INVALID_ARG;
        int64_t prev = 0;
        for (int32_t r = r0; r < r1; ++r) {
            const s2_context_range& c = ranges[r];
            if (c.end_block <= prev || c.vertical_stride < 0 || c.local_blocks < 0)
                return S2_ERR_INVALID_ARG;
            prev = c.end_block;
        }
        if (prev != nb) return S2_ERR_INVALID_ARG;
    }
    auto count = [&](int64_t h, int64_t i) {
        int64_t n = 0, a = 0;
        for (int32_t r = range_ptr[h]; r < range_ptr[h + 1] && a <= i; ++r) {
            n += range_row_count(h, i, a, ranges[r].end_block, ranges[r]);
            a = ranges[r].end_block;
        }
        return n;
    };
    auto fill = [&](int64_t h, int64_t i, int32_t* out) {
        int64_t n = 0, a = 0;
        for (int32_t r = range_ptr[h]; r < range_ptr[h + 1] && a <= i; ++r) {
            range_row(h, i, a, ranges[r].end_block, ranges[r],
                      [&](int64_t j) { out[n++] = (int32_t)j; });
            a = ranges[r].end_block;
        }
    };
    return emit_csr(H, nb, count, fill, row_ptr, col_idx, col_idx_cap, nnz_out);
}

extern "C" int s2_build_layout_mask(int32_t num_heads, int32_t num_blocks,
                                    const uint8_t* block_mask, int32_t* row_ptr, int32_t* col_idx,
                                    int64_t col_idx_cap, int64_t* nnz_out)
{
    if (!block_mask || !nnz_out || num_heads < 1 || num_blocks < 1) return S2_ERR_INVALID_ARG;
    if (col_idx && !row_ptr) return S2_ERR_INVALID_ARG;
    const int64_t H = num_heads, nb = num_blocks;
    for (int64_t h = 0; h < H; ++h)
        for (int64_t i = 0; i < nb; ++i) {
            const uint8_t* m = block_mask + (h * nb + i) * nb;
            for (int64_t j = i + 1; j < nb; ++j)
                if (m[j]) return S2_ERR_INVALID_ARG;  // above the diagonal
        }
    auto count = [&](int64_t h, int64_t i) {
        const uint8_t* m = block_mask + (h * nb + i) * nb;
        int64_t n = 0;
        for (int64_t j = 0; j <= i; ++j) n += m[j] != 0;
        return n;
    };
    auto fill = [&](int64_t h, int64_t i, int32_t* out) {
        const uint8_t* m = block_mask + (h * nb + i) * nb;
        int64_t n = 0;
        for (int64_t j = 0; j <= i; ++j)
            if (m[j]) out[n++] = (int32_t)j;
    };
    return emit_csr(H, nb, count, fill, row_ptr, col_idx, col_idx_cap, nnz_out);
}

// ---------------------------------------------------------------------------
// Transposed lists for the backward pass: for each head h and key block j, the
// ascending query blocks i whose list holds j. A counting sort per head: count
// the entries per j, turn the counts into offsets, then visit the rows in
// ascending i so that every transposed list comes out ascending.
// ---------------------------------------------------------------------------
extern "C" int s2_build_layout_transpose(int32_t num_heads, int32_t num_blocks,
                                         const int32_t* row_ptr, const int32_t* col_idx,
                                         int64_t nnz, int32_t* col_ptr, int32_t* row_idx)
{
    if (!row_ptr || !col_ptr || num_heads < 1 || num_blocks < 1 || nnz < 0 || nnz > INT32_MAX ||
        ((!col_idx || !row_idx) && nnz > 0))
        return S2_ERR_INVALID_ARG;
    const int64_t H = num_heads, nb = num_blocks;
    // validate: global offsets, rows within [0, nnz], j ascending with j <= i
    int64_t prev_end = 0;
    for (int64_t h = 0; h < H; ++h)
        for (int64_t i = 0; i < nb; ++i) {
            const int64_t a = row_ptr[h * (nb + 1) + i], b = row_ptr[h * (nb + 1) + i + 1];
            if (a != prev_end || b < a || b > nnz) return S2_ERR_INVALID_ARG;
            prev_end = b;
            for (int64_t e = a; e < b; ++e) {
                const int32_t j = col_idx[e];
                if (j < 0 || j > i || (e > a && j <= col_idx[e - 1])) return S2_ERR_INVALID_ARG;
            }
        }
    if (prev_end != nnz) return S2_ERR_INVALID_ARG;
    for (int64_t h = 0; h < H; ++h) {
        int32_t* cp = col_ptr + h * (nb + 1);
        for (int64_t j = 0; j <= nb; ++j) cp[j] = 0;
        const int64_t base = row_ptr[h * (nb + 1)];
        for (int64_t e = base; e < row_ptr[h * (nb + 1) + nb]; ++e) ++cp[col_idx[e] + 1];
        cp[0] = (int32_t)base;
        for (int64_t j = 1; j <= nb; ++j) cp[j] += cp[j - 1];
        // fill: a running cursor per j (reuse the start offsets, then restore)
        for (int64_t i = 0; i < nb; ++i)
            for (int64_t e = row_ptr[h * (nb + 1) + i]; e < row_ptr[h * (nb + 1) + i + 1]; ++e)
                row_idx[cp[col_idx[e]]++] = (int32_t)i;
        for (int64_t j = nb; j > 0; --j) cp[j] = cp[j - 1];
        cp[0] = (int32_t)base;
    }
    return S2_OK;
}

// ---------------------------------------------------------------------------
// Key tiles of the backward's dK/dV kernel for 64-row blocks: each 128-row key
// tile holds two key blocks and walks the union of their transposed lists, so
// blocks whose lists overlap should share a tile. Per head, the blocks are
// ordered by transposed-list length (longest first, then by j) and paired
// consecutively: under HHST the strided blocks j and j + S pair up (both are
// listed by nearly every later query block) and the other blocks pair with
// their neighbours (overlapping local windows).
// ---------------------------------------------------------------------------
extern "C" int s2_build_key_tiles(int32_t num_heads, int32_t num_blocks, const int32_t* col_ptr,
                                  int32_t* key_tiles)
{
    if (!col_ptr || !key_tiles || num_heads < 1 || num_blocks < 1) return S2_ERR_INVALID_ARG;
    const int64_t H = num_heads, nb = num_blocks, ntk = (nb + 1) / 2;
    std::vector<int32_t> order((size_t)nb);
    for (int64_t h = 0; h < H; ++h) {
        const int32_t* cp = col_ptr + h * (nb + 1);
        for (int64_t j = 0; j < nb; ++j) {
            if (cp[j + 1] < cp[j]) return S2_ERR_INVALID_ARG;
            order[(size_t)j] = (int32_t)j;
        }
        std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
            return cp[a + 1] - cp[a] > cp[b + 1] - cp[b];
        });
        for (int64_t t = 0; t < ntk; ++t) {
            key_tiles[(h * ntk + t) * 2] = order[(size_t)(2 * t)];
            key_tiles[(h * ntk + t) * 2 + 1] = 2 * t + 1 < nb ? order[(size_t)(2 * t + 1)] : -1;
        }
    }
    return S2_OK;
}
