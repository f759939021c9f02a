// layout.cpp -- host builder of the HHST per-head compacted key-block lists.
//
// HHST ("S2-Attention: Hardware-aware context sharding among attention heads",
// Abstract) gives each head its own strided share of the context plus a local
// window. For head h and query block i the active key blocks are
//   the L local blocks  max(0, i-L+1) .. i, and
//   the strided blocks  j < i-L+1 with j = -h (mod S),
// or every block 0..i for a dense head. This file enumerates them directly in
// ascending order (strided ones first, then the local run), which is O(nnz)
// rather than a test of every (i, j) pair, and emits CSR offsets.
#include <climits>
#include <cstdint>

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
