// lists.cuh -- walking compacted block lists (CSR) on the device.
//
// A tile of M = 128 rows covers one or more consecutive blocks; its work is
// the ascending union of those blocks' lists, each element tagged with the
// blocks (rows of the CSR) that list it. Used by the prefill kernel (query
// blocks over key-block lists) and by the backward kernels (also over the
// transposed lists: key blocks over the query blocks that list them).
#pragma once

#include <climits>
#include <cstdint>

#include "ptx.cuh"

namespace s2 {

// Warp-wide bounded wait (every lane polls: measured faster than one lane
// polling and broadcasting).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl)
{
    const bool ok = mbar_wait(bar, parity, ctl);
    return __all_sync(0xffffffffu, ok);
}

// Union-list entry: key block j (bits 0..23), row tags (bits 24..27).
__device__ __forceinline__ uint32_t list_pack(int j, int bits) { return (uint32_t)j | ((uint32_t)bits << 24); }
__device__ __forceinline__ int list_j(uint32_t e) { return (int)(e & 0xFFFFFFu); }
__device__ __forceinline__ int list_bits(uint32_t e) { return (int)((e >> 24) & 0xFu); }

// Walks the ascending union of up to ROWS compacted lists (CSR rows
// qb0 .. qb0+ROWS-1 of one head) and tags each element with the rows that
// list it. Elements outside [imin, imax] are malformed: for the key-block
// lists of query blocks that is [0, last query block of the tile]; for the
// transposed lists (query blocks listing a key block) it is
// [first key block of the tile, nb - 1].
template <int ROWS>
struct UnionWalk {
    int a[ROWS], e[ROWS];
    int imin, imax;

    // `any` tells whether a list is non-empty.
    bool any;

    // Key-block lists of query blocks qb0..: returns false for offsets outside [0, nnz].
    __device__ __forceinline__ bool init(const int32_t* row_ptr, int rp, int qb0, int nb, int64_t nnz)
    {
        const bool ok = init_rows(row_ptr, rp, qb0, nb, nnz);
        imin = 0;
        return ok;
    }

    // Transposed lists of the key blocks kb[0..ROWS-1] (kb[r] < 0: no block):
    // the same walk, valid range [smallest key block, nb - 1].
    __device__ __forceinline__ bool init_transposed(const int32_t* col_ptr, int rp, const int* kb, int nb,
                                                    int64_t nnz)
    {
        const bool ok = init_rows(col_ptr, rp, kb, nb, nnz);
        imin = INT_MAX;
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
            if (kb[r] >= 0 && kb[r] < imin) imin = kb[r];
        imax = nb - 1;
        return ok;
    }

    __device__ __forceinline__ bool init_rows(const int32_t* row_ptr, int rp, int qb0, int nb, int64_t nnz)
    {
        int rows[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) rows[r] = qb0 + r;
        return init_rows(row_ptr, rp, rows, nb, nnz);
    }

    // CSR rows rows[0..ROWS-1] (a row outside [0, nb) is absent).
    __device__ __forceinline__ bool init_rows(const int32_t* row_ptr, int rp, const int* rows, int nb,
                                              int64_t nnz)
    {
        bool ok = true;
        any = false;
        imax = -1;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            a[r] = e[r] = 0;
            const int qb = rows[r];
            if (qb >= 0 && qb < nb) {
                a[r] = __ldg(row_ptr + rp + qb);
                e[r] = __ldg(row_ptr + rp + qb + 1);
                ok = ok && a[r] >= 0 && a[r] <= e[r] && e[r] <= nnz;
                any = any || e[r] > a[r];
                imax = qb;
            }
        }
        if (!ok) {
#pragma unroll
            for (int r = 0; r < ROWS; ++r) a[r] = e[r] = 0;
            any = false;
        }
        return ok;
    }

    // Next union element j, its row tag bits, and whether it is the last.
    // A malformed entry (j outside [imin, imax]) comes out as j = imin with no tags.
    __device__ __forceinline__ void next(const int32_t* col, int& j, int& bits, bool& last, bool& bad)
    {
        int jm = INT_MAX;
        int cur[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            cur[r] = a[r] < e[r] ? __ldg(col + a[r]) : INT_MAX;
            jm = cur[r] < jm ? cur[r] : jm;
        }
        bits = 0;
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
            if (cur[r] == jm) {
                bits |= 1 << r;
                ++a[r];
            }
        last = true;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) last = last && a[r] >= e[r];
        bad = jm < imin || jm > imax;
        if (bad) {
            jm = imin;
            bits = 0;
        }
        j = jm;
    }
};

// Warp-cooperative version of the walk, for a list built once per CTA before
// the main loop: all 32 lanes copy the CSR rows rows[0..ROWS-1] (coalesced)
// into `scratch` (ROWS * cap ints) and lane 0 merges them from shared memory,
// which avoids a dependent global load per element. Writes the tagged union
// into `list` and returns its length on every lane. Rows outside [0, nb) are
// absent; offsets outside [0, nnz], lists longer than cap and elements
// outside [lo, hi] set kFlagIndex (a bad element becomes lo with no tags).
template <int ROWS>
__device__ __forceinline__ int warp_union_list(const int32_t* row_ptr, const int32_t* col, int rp,
                                               const int* rows, int nb, int64_t nnz, int lo, int hi,
                                               uint32_t* list, int cap, int32_t* scratch,
                                               uint32_t* gflags)
{
    const int lane = threadIdx.x & 31;
    int a[ROWS], n[ROWS];
    bool ok = true;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        a[r] = n[r] = 0;
        if (rows[r] >= 0 && rows[r] < nb) {
            const int b0 = __ldg(row_ptr + rp + rows[r]), b1 = __ldg(row_ptr + rp + rows[r] + 1);
            ok = ok && b0 >= 0 && b0 <= b1 && b1 <= nnz && b1 - b0 <= cap;
            a[r] = b0;
            n[r] = b1 - b0;
        }
    }
    if (!ok) {
        if (lane == 0) atomicOr(gflags, kFlagIndex);
        return 0;
    }
    auto checked = [&](int j, int bits) {
        if (j < lo || j > hi) {
            atomicOr(gflags, kFlagIndex);
            return list_pack(lo, 0);
        }
        return list_pack(j, bits);
    };
    if constexpr (ROWS == 1) {
        for (int t = lane; t < n[0]; t += 32) list[t] = checked(__ldg(col + a[0] + t), 1);
        __syncwarp();
        return n[0];
    }
    else {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
        for (int t = lane; t < n[r]; t += 32) scratch[r * cap + t] = __ldg(col + a[r] + t);
    __syncwarp();
    int len = 0;
    if (lane == 0) {
        int i[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) i[r] = 0;
        for (;;) {
            int jm = INT_MAX;
#pragma unroll
            for (int r = 0; r < ROWS; ++r)
                if (i[r] < n[r]) jm = min(jm, scratch[r * cap + i[r]]);
            if (jm == INT_MAX) break;
            int bits = 0;
#pragma unroll
            for (int r = 0; r < ROWS; ++r)
                if (i[r] < n[r] && scratch[r * cap + i[r]] == jm) {
                    bits |= 1 << r;
                    ++i[r];
                }
            if (len >= cap) {  // cannot happen for ascending lists with nb <= cap
                atomicOr(gflags, kFlagIndex);
                break;
            }
            list[len++] = checked(jm, bits);
        }
    }
    __syncwarp();
    return __shfl_sync(0xffffffffu, len, 0);
    }
}

}  // namespace s2
