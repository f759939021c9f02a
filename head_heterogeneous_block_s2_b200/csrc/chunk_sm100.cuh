// chunk_sm100.cuh -- chunked prefill over a paged KV cache on sm_100a.
//
// Serving runs prefill in chunks: each sequence appends a chunk of query
// tokens at the end of its context, whose keys and values (the chunk's own
// included) already sit in a paged cache addressed through a block table
// (PagedAttention is in the reference list of the arXiv page of "S2-Attention:
// Hardware-aware context sharding among attention heads"; the abstract reports
// 7B inference in vLLM). Chunk row t of sequence s sits at position
// ctx_lens[s] - (q_start[s+1] - t) and attends, under the same compacted
// block lists as the prefill, to the keys up to its position.
//
// The kernel is the prefill pair kernel's pipeline (one MMA thread for both
// tiles, prefill_pair_sm100.cuh) with chunk addressing:
//  * a work item is up to two adjacent 128-row tiles of absolute positions of
//    one (sequence, head), cut to the chunk; a sequence's pairs are taken from
//    the end of its chunk (the heaviest first), sequence after sequence, heads
//    innermost; the CTAs are persistent and take items from a device counter;
//  * Q comes by TMA from the packed chunk rows [total_q][heads][D] (rows
//    outside the chunk read zeros or other rows and are never stored);
//  * a key block is B / 16 pages: each page is one TMA box (per 64-column
//    panel) of a 3-D map over the cache [num_pages * heads_kv][16][D], issued
//    by one lane of the K/V warp each; pages past the context (or with an
//    invalid id, which is flagged) load zeros through an out-of-range
//    coordinate;
//  * rows past the context inside the last page hold whatever the cache holds
//    there, so the softmax threads zero them in the V stage before their
//    tile's P V product reads it (their P is 0 anyway, but 0 times a NaN would
//    not be);
//  * the output and the LSE go to the packed chunk rows;
//  * each tile has its own Q buffer barriers: the tile's last S MMA of an item
//    releases its Q and the next item's Q of that tile loads at once (the
//    first tile usually sees its last key block one element before the second,
//    whose diagonal block ends the list), and the tile's O is complete with its
//    last PV, so its epilogue runs while the other tile finishes the item.
// Roles: warp 2 maps items (a warp-parallel prefix over the sequences),
// builds the union list of the item's query blocks and loads Q; warp 0
// streams K and V; warp 1 owns TMEM and issues tcgen05.mma (S_t = Q_t K^T,
// O_t += P_t V); warps 4..7 and 8..11 are the softmax of tile 0 and tile 1.
// Every wait is bounded; a CTA that gives up drains its own copies and MMAs
// and exits with the device timeout flag set.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>

#include "lists.cuh"
#include "ptx.cuh"
#include "store.cuh"  // store_bf16_row
#include "umma.cuh"

namespace s2 {

struct ChunkParams {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t nnz;
    const int32_t* block_table;  // [batch][max_pages]
    const int32_t* ctx_lens;     // [batch]: context length including the chunk
    const int32_t* q_start;      // [batch + 1]: chunk rows of sequence s are q_start[s] .. q_start[s+1]-1
    uint16_t* out;               // [total_q][heads][HD]
    float* lse;                  // [total_q][heads] or null
    int64_t num_pages, total_q;
    int32_t batch, heads, heads_kv, max_pages, nb, max_q_len;
    float scale_log2;
    uint64_t timeout_ns;
    uint32_t* gflags;
    int* sched;                  // work-counter slot (sched_claim / sched_take / sched_leave)
    int sched_id;                // this launch's nonzero id
};

constexpr int kChunkPage = 16;  // tokens per cache page

template <int HD, int BK>
struct ChunkCfg {
    static constexpr int M = 128;                          // rows per tile
    static constexpr int TROWS = M / BK;                   // query blocks per tile
    static constexpr int ROWS = 2 * TROWS;                 // query blocks per item
    static constexpr int NK = BK;                          // S columns
    static constexpr int PPB = BK / kChunkPage;            // cache pages per key block
    static constexpr uint32_t QBYTES = M * HD * 2;         // one tile's Q
    static constexpr uint32_t KVBYTES = BK * HD * 2;       // one K (or V) block
    static constexpr int LIST_CAP = 2048;                  // union entries per item (>= nb + 1)
    static constexpr uint32_t LIST_BYTES = 2 * LIST_CAP * 4;  // double-buffered
    static constexpr int ST = (2 * QBYTES + 4 * 2 * KVBYTES + LIST_BYTES <= 220 * 1024) ? 4 : 2;
    static constexpr uint32_t KPANEL = ST * BK * 128;      // bytes of one 64-column K panel, all stages
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + 2 * QBYTES;  // [panel][stage][BK rows x 128 B]
    static constexpr uint32_t OFF_V = OFF_K + ST * KVBYTES;  // [stage][panel][BK rows x 128 B]
    static constexpr uint32_t OFF_LIST = OFF_V + ST * KVBYTES;
    static constexpr uint32_t OFF_BAR = OFF_LIST + LIST_BYTES;
    // barriers: q_full[0], q_empty[0], kv_full[ST], kv_empty[ST], s_full[2], p_full[2],
    // pv_done[2], drain, list_full[2], list_empty[2], q_full[1], q_empty[1]
    static constexpr int NBAR = 2 + 2 * ST + 6 + 1 + 4 + 2;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    // misc ints: [0] tmem, [1] abort, [2..3] list lengths, [4..5] item of each
    // list buffer (-1: no more), [8..15] and [16..23] the buffers' item fields
    static constexpr uint32_t SMEM = OFF_MISC + 96;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    static constexpr uint32_t LIST_CONSUMERS = 10;  // K/V producer, MMA issuer, 8 softmax warps
    __host__ __device__ static constexpr uint32_t colS(int t) { return (uint32_t)(t * NK); }
    __host__ __device__ static constexpr uint32_t colO(int t) { return (uint32_t)(2 * NK + t * HD); }
    // When TMEM has room for both tiles' Q (HD/2 columns each), S = Q K^T reads
    // Q from TMEM and only K from shared memory.
    static constexpr bool Q_IN_TMEM = 2 * NK + 3 * HD <= 512;
    __host__ __device__ static constexpr uint32_t colQ(int t) { return (uint32_t)(2 * NK + 2 * HD + t * (HD / 2)); }
    static constexpr int TMEM_NEED = 2 * NK + 2 * HD + (Q_IN_TMEM ? HD : 0);
    static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// One work item; stored in shared memory by the scheduler warp for the other roles.
struct ChunkItem {
    int s, h, hkv, qt0;  // sequence, query head, K/V head, first tile (absolute 128-row tile)
    int tile1;           // 1 if the tile qt0 + 1 belongs to the item
    int n, c0, q0;       // context length, first chunk position, first chunk row
};
static_assert(sizeof(ChunkItem) == 32, "eight ints");

// Chunk geometry of sequence s: false for inconsistent metadata; `pairs` = the
// number of tile pairs (0 for an empty or inconsistent chunk).
template <int BK>
__device__ __forceinline__ bool chunk_seq(const ChunkParams& p, int s, int& n, int& q0, int& ql, int& pairs)
{
    n = __ldg(p.ctx_lens + s);
    q0 = __ldg(p.q_start + s);
    ql = __ldg(p.q_start + s + 1) - q0;
    pairs = 0;
    const bool ok = ql >= 0 && ql <= p.max_q_len && ql <= n && q0 >= 0 && (int64_t)q0 + ql <= p.total_q &&
                    (int64_t)n <= (int64_t)p.max_pages * kChunkPage && (n == 0 || (n - 1) / BK < p.nb);
    if (ok && ql > 0) {
        const int tiles = (n - 1) / 128 - (n - ql) / 128 + 1;
        pairs = (tiles + 1) >> 1;
    }
    return ok;
}

// Item w (warp-collective): heads innermost, then the sequences' tile pairs in
// order, each sequence's from the end of its chunk. False if w is out of range.
template <int BK>
__device__ __forceinline__ bool chunk_item(const ChunkParams& p, int64_t w, int lane, ChunkItem& I)
{
    const int h = (int)(w % p.heads);
    int64_t g = w / p.heads;  // pair slot over the batch
    for (int s0 = 0; s0 < p.batch; s0 += 32) {
        const int s = s0 + lane;
        int n = 0, q0 = 0, ql = 0, np = 0;
        if (s < p.batch) chunk_seq<BK>(p, s, n, q0, ql, np);
        int incl = np;  // inclusive prefix over the lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        if (g < tot) {
            const unsigned hit = __ballot_sync(0xffffffffu, g < incl);
            const int src = __ffs(hit) - 1;
            const int pr = (int)g - (__shfl_sync(0xffffffffu, incl, src) - __shfl_sync(0xffffffffu, np, src));
            I.s = s0 + src;
            I.n = __shfl_sync(0xffffffffu, n, src);
            I.q0 = __shfl_sync(0xffffffffu, q0, src);
            I.c0 = I.n - __shfl_sync(0xffffffffu, ql, src);
            I.h = h;
            I.hkv = h / (p.heads / p.heads_kv);
            const int tfirst = I.c0 / 128, hi = (I.n - 1) / 128 - 2 * pr;
            I.tile1 = hi - 1 >= tfirst ? 1 : 0;
            I.qt0 = I.tile1 ? hi - 1 : hi;
            return true;
        }
        g -= tot;
    }
    return false;
}

// Tile t's share of a union element's row tags (one query block per tile
// with 128-key blocks, two with 64-key blocks).
template <int BK>
__device__ __forceinline__ bool tile_sees_chunk(int bits, int t)
{
    return BK == 128 ? ((bits >> t) & 1) != 0 : ((bits >> (2 * t)) & 3) != 0;
}

template <int HD, int BK>
__global__ void __launch_bounds__(384, 1)
s2_chunk_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const ChunkParams p)
{
    using C = ChunkCfg<HD, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Q of tile t: loaded (q_full) and released by the tile's last S MMA of an item (q_empty)
    auto bar_q = [&](int t) { return sb + C::OFF_BAR + 8u * (t == 0 ? 0 : 13 + 2 * C::ST); };
    auto bar_qe = [&](int t) { return sb + C::OFF_BAR + 8u * (t == 0 ? 1 : 14 + 2 * C::ST); };
    auto bar_kf = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + s); };  // K and V of a stage
    auto bar_ke = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + C::ST + s); };
    auto bar_sf = [&](int t) { return sb + C::OFF_BAR + 8u * (2 + 2 * C::ST + t); };
    auto bar_pf = [&](int t) { return sb + C::OFF_BAR + 8u * (4 + 2 * C::ST + t); };
    auto bar_pv = [&](int t) { return sb + C::OFF_BAR + 8u * (6 + 2 * C::ST + t); };
    const uint32_t bar_dr = sb + C::OFF_BAR + 8u * (8 + 2 * C::ST);
    auto bar_lf = [&](int b) { return sb + C::OFF_BAR + 8u * (9 + 2 * C::ST + b); };
    auto bar_le = [&](int b) { return sb + C::OFF_BAR + 8u * (11 + 2 * C::ST + b); };
    const uint32_t* list = reinterpret_cast<const uint32_t*>(smem + C::OFF_LIST);
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_cta = misc + 1;
    volatile int* list_len = misc + 2;
    volatile int* list_item = misc + 4;
    ChunkItem* items = reinterpret_cast<ChunkItem*>(misc + 8);  // [2]: one per list buffer

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_q(t), 1);
            mbar_init(bar_qe(t), 1);
        }
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_ke(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_sf(t), 1);
            mbar_init(bar_pf(t), 128);
            mbar_init(bar_pv(t), 1);
            mbar_init(bar_lf(t), 1);
            mbar_init(bar_le(t), C::LIST_CONSUMERS);
        }
        mbar_init(bar_dr, 1);
        *abort_cta = 0;
        misc[6] = sched_claim(p.sched, p.sched_id, WaitCtl{p.timeout_ns, p.gflags, abort_cta});
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl ctl{p.timeout_ns, p.gflags, abort_cta};
    constexpr uint64_t kDrainNs = 200000000ull;

    if (warp == 2) {
        // ------------------------------------------------------------ items, union lists, Q
        // items in this launch: tile pairs over the batch times heads (a sequence
        // with inconsistent metadata counts none and is flagged)
        int64_t pairs = 0;
        for (int s0 = 0; s0 < p.batch; s0 += 32) {
            int n = 0, q0 = 0, ql = 0, np = 0;
            if (s0 + lane < p.batch && !chunk_seq<BK>(p, s0 + lane, n, q0, ql, np)) atomicOr(p.gflags, kFlagIndex);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) np += __shfl_xor_sync(0xffffffffu, np, o);
            pairs += np;
        }
        const int64_t num_items = pairs * p.heads;
        uint32_t* wlist = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
        int64_t w = blockIdx.x;  // first item static, the rest from the work counter
        int k = 0;
        int qn[2] = {0, 0};  // Q phases started per tile
        for (;; ++k) {
            const int b = k & 1;
            // union list of this item into buffer b (free once item k-2 is consumed)
            if (!warp_wait(bar_le(b), ((k >> 1) & 1) ^ 1, ctl)) break;
            ChunkItem I;
            if (w >= num_items || !chunk_item<BK>(p, w, lane, I)) {  // no more work for any role
                if (lane == 0) {
                    list_item[b] = -1;
                    list_len[b] = 0;
                    mbar_arrive(bar_lf(b));
                }
                break;
            }
            int64_t w_next = 0;
            if (lane == 0) w_next = misc[6] ? (int64_t)gridDim.x + sched_take(p.sched) : num_items;
            w_next = __shfl_sync(0xffffffffu, w_next, 0);
            if (lane == 0) {
                // the item's query blocks, without those wholly before the chunk or
                // past the context (their rows are never stored)
                int rows[C::ROWS];
#pragma unroll
                for (int r = 0; r < C::ROWS; ++r) {
                    const int qb = I.qt0 * C::TROWS + r;
                    const bool in = (r < C::TROWS || I.tile1) && (qb + 1) * BK > I.c0 && qb * BK < I.n;
                    rows[r] = in ? qb : -1;
                }
                UnionWalk<C::ROWS> it;
                const bool ok = it.init_rows(p.row_ptr, I.h * (p.nb + 1), rows, p.nb, p.nnz);
                it.imin = 0;
                int len = 0;
                if (it.any) {  // an item whose rows are all empty publishes an empty list
                    for (;;) {
                        int j, bits;
                        bool last, bad;
                        it.next(p.col_idx, j, bits, last, bad);
                        if (bad) atomicOr(p.gflags, kFlagIndex);
                        if (len >= C::LIST_CAP - 1) {  // cannot happen when nb <= LIST_CAP - 1
                            atomicOr(p.gflags, kFlagIndex);
                            last = true;
                        }
                        wlist[b * C::LIST_CAP + len++] = list_pack(j, bits);
                        if (last) break;
                    }
                } else if (!ok) {
                    atomicOr(p.gflags, kFlagIndex);
                }
                items[b] = I;
                list_len[b] = len;
                list_item[b] = (int)(w & 0x7fffffff);
                mbar_arrive(bar_lf(b));
            }
            // Q of each tile, once the previous item's last S MMA of that tile is done
            // with its buffer (tile 0 usually sees its last key block one element
            // before tile 1, so its Q reloads earlier); tile row r is chunk row
            // q0 + 128 (qt0 + t) - c0 + r. An absent second tile only completes its
            // barrier phase.
            int q_ok = 1;
            if (lane == 0) {
                for (int t = 0; t < 2; ++t) {
                    if (!mbar_wait(bar_qe(t), (k & 1) ^ 1, ctl)) {
                        q_ok = 0;
                        break;
                    }
                    if (t == 0 || I.tile1) {
                        mbar_arrive_expect_tx(bar_q(t), C::QBYTES);
#pragma unroll
                        for (int pn = 0; pn < HD / 64; ++pn)
                            tma_load_3d(sb + C::OFF_Q + t * C::QBYTES + pn * (C::M * 128), &tmQ, pn * 64, I.h,
                                        I.q0 + (I.qt0 + t) * C::M - I.c0, bar_q(t));
                    } else {
                        mbar_arrive(bar_q(t));
                    }
                    ++qn[t];
                }
            }
            if (!__shfl_sync(0xffffffffu, q_ok, 0)) break;  // Q of item k was not (wholly) issued
            w = w_next;
        }
        if (lane == 0 && *abort_cta)  // let this CTA's own Q loads land before exit
            for (int t = 0; t < 2; ++t)
                if (qn[t] > 0) mbar_drain(bar_q(t), (qn[t] - 1) & 1, kDrainNs);
        __syncwarp();
    } else if (warp == 0) {
        // ------------------------------------------------------------ K/V producer
        // Lane pg < B/16 loads page pg of each key block (K and V, every panel).
        const int32_t oob_plane = (int32_t)(p.num_pages * p.heads_kv);  // reads zeros
        int n = 0, k = 0;
        bool stop = false;
        for (; !stop; ++k) {
            const int b = k & 1;
            if (!warp_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
            if (list_item[b] < 0) break;
            const ChunkItem I = items[b];
            const uint32_t* L = list + b * C::LIST_CAP;
            const int len = list_len[b];
            // the cache plane of this lane's page of element e (the block-table
            // read of the next element is issued before waiting for its stage)
            auto page_plane = [&](int e) {
                const int lp = list_j(L[e]) * C::PPB + lane;  // logical page of this lane
                int32_t pl = oob_plane;
                if (lane < C::PPB && lp * kChunkPage < I.n) {
                    const int32_t phys = __ldg(p.block_table + (int64_t)I.s * p.max_pages + lp);
                    if (phys < 0 || phys >= p.num_pages)
                        atomicOr(p.gflags, kFlagIndex);
                    else
                        pl = phys * p.heads_kv + I.hkv;
                }
                return pl;
            };
            int32_t plane_next = len > 0 ? page_plane(0) : oob_plane;
            for (int e = 0; e < len; ++e, ++n) {
                const int st = n % C::ST;
                const int32_t plane = plane_next;
                if (e + 1 < len) plane_next = page_plane(e + 1);
                if (!warp_wait(bar_ke(st), ((n / C::ST) & 1) ^ 1, ctl)) {
                    stop = true;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(bar_kf(st), 2 * C::KVBYTES);
                __syncwarp();
                if (lane < C::PPB) {
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_3d(sb + C::OFF_K + pn * C::KPANEL + st * (BK * 128) + lane * (kChunkPage * 128),
                                    &tmK, pn * 64, 0, plane, bar_kf(st));
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_3d(sb + C::OFF_V + st * C::KVBYTES + pn * (BK * 128) + lane * (kChunkPage * 128),
                                    &tmV, pn * 64, 0, plane, bar_kf(st));
                }
                __syncwarp();
            }
            if (!stop && lane == 0) mbar_arrive(bar_le(b));
        }
        if (lane == 0 && *abort_cta)  // let this CTA's own loads land before exit
            for (int m = (n > C::ST ? n - C::ST : 0); m < n; ++m)
                mbar_drain(bar_kf(m % C::ST), (m / C::ST) & 1, kDrainNs);
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc(128, C::NK, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc(128, HD, 0, 1);
            constexpr int KSTEPS = BK / 16;  // PV k-steps per key block
            bool issued = false, fail = false;
            int pvc[2] = {0, 0};  // PV MMAs issued per tile (all items)
            bool first_pv[2] = {true, true};
            int n = 0;            // union elements consumed (all items)
            // S_t = Q_t K^T over the block in stage st
            auto issue_s = [&](int t, int st) {
                const uint64_t dq = umma_sdesc(sb + C::OFF_Q + t * C::QBYTES, 16, 1024);
                const uint64_t dk = umma_sdesc(sb + C::OFF_K + st * (BK * 128), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t bk = dk + (((kk >> 2) * C::KPANEL + (kk & 3) * 32) >> 4);
                    if constexpr (C::Q_IN_TMEM)
                        umma_bf16_ts(tmem + C::colS(t), tmem + C::colQ(t) + kk * 8, bk, idesc_s, kk > 0 ? 1u : 0u);
                    else
                        umma_bf16_ss(tmem + C::colS(t), dq + (((kk >> 2) * (C::M * 128) + (kk & 3) * 32) >> 4),
                                     bk, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_sf(t));
                issued = true;
            };
            // O_t += P_t V over the block in stage st
            auto issue_pv = [&](int t, int st) {
                const uint32_t acc0 = first_pv[t] ? 0u : 1u;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk)
                    umma_bf16_ts(tmem + C::colO(t), tmem + C::colS(t) + kk * 8,
                                 umma_sdesc(sb + C::OFF_V + st * C::KVBYTES + kk * 2048, BK * 128, 1024), idesc_o,
                                 kk > 0 ? 1u : acc0);
                ++pvc[t];
                first_pv[t] = false;
            };
            auto wait_k = [&](int m) { return mbar_wait(bar_kf(m % C::ST), (m / C::ST) & 1, ctl); };
            for (int k = 0; !fail; ++k) {
                const int b = k & 1;
                if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                if (list_item[b] < 0) break;
                const bool two = items[b].tile1 != 0;
                const uint32_t* L = list + b * C::LIST_CAP;
                const int len = list_len[b];
                // The last element each tile sees (-1: none): its S MMA is the tile's
                // last read of its Q buffer, its PV completes the tile's O.
                int lastS[2] = {-1, -1};
                for (int g = len - 1; g >= 0 && (lastS[0] < 0 || (two && lastS[1] < 0)); --g) {
                    const int gb = list_bits(L[g]);
#pragma unroll
                    for (int t = 0; t < 2; ++t)
                        if (lastS[t] < 0 && tile_sees_chunk<BK>(gb, t)) lastS[t] = g;
                }
                bool q_in[2] = {false, false};  // this item's phase of the tile's Q barrier observed
                auto take_q = [&](int t) {
                    if (!q_in[t]) {
                        if (!mbar_wait(bar_q(t), k & 1, ctl)) return false;
                        q_in[t] = true;
                        tc_fence_after();
                    }
                    return true;
                };
                if (len == 0) {
                    if (!take_q(0) || !take_q(1)) break;
                    umma_commit(bar_qe(0));
                    umma_commit(bar_qe(1));
                    mbar_arrive(bar_le(b));
                    continue;
                }
                for (int t = 0; t < 2 && !fail; ++t) {
                    if constexpr (C::Q_IN_TMEM) {
                        // Q of the tile into TMEM (after the previous item's S MMAs, in
                        // issue order), then its shared-memory buffer is free at once.
                        if (!take_q(t)) {
                            fail = true;
                            break;
                        }
                        if (t == 0 || two) {
                            const uint64_t dq = umma_sdesc(sb + C::OFF_Q + t * C::QBYTES, 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk)
                                tmem_cp_128x256b(tmem + C::colQ(t) + kk * 8,
                                                 dq + (((kk >> 2) * (C::M * 128) + (kk & 3) * 32) >> 4));
                        }
                        umma_commit(bar_qe(t));
                    } else if (lastS[t] < 0) {  // the tile reads no Q in this item
                        if (!take_q(t)) {
                            fail = true;
                            break;
                        }
                        umma_commit(bar_qe(t));
                    }
                }
                if (fail) break;
                // S_t of element e (in stage st), once the tile's Q has landed; the
                // tile's last one releases the Q buffer
                auto s_tile = [&](int t, int e, int st) {
                    if (!C::Q_IN_TMEM && !take_q(t)) return false;
                    issue_s(t, st);
                    if (!C::Q_IN_TMEM && e == lastS[t]) umma_commit(bar_qe(t));
                    return true;
                };
                first_pv[0] = first_pv[1] = true;
                int bits = list_bits(L[0]);
                if (!wait_k(n)) break;
                tc_fence_after();
                for (int t = 0; t < 2 && !fail; ++t)
                    if (tile_sees_chunk<BK>(bits, t) && !s_tile(t, 0, n % C::ST)) fail = true;
                if (fail) break;
                for (int g = 0;; ++g, ++n) {
                    const bool last = g + 1 == len;
                    const int nbits = last ? 0 : list_bits(L[g + 1]);
                    const int st = n % C::ST;
                    const int st1 = (n + 1) % C::ST;
                    bool k_next_ready = false;
                    if (bits == 0) {  // malformed element no tile sees: let its loads land first
                        if (!wait_k(n)) {
                            fail = true;
                            break;
                        }
                    }
                    const int last_t = tile_sees_chunk<BK>(bits, 1) ? 1 : (tile_sees_chunk<BK>(bits, 0) ? 0 : 1);
                    for (int t = 0; t < 2 && !fail; ++t) {
                        if (tile_sees_chunk<BK>(bits, t)) {
                            if (!mbar_wait(bar_pf(t), pvc[t] & 1, ctl)) { fail = true; break; }
                            tc_fence_after();
                            issue_pv(t, st);
                            // O_t of the item is complete with the tile's last PV: its
                            // softmax warps start the epilogue while the other tile runs on
                            if (g == lastS[t]) umma_commit(bar_pv(t));
                        }
                        if (t == last_t) umma_commit(bar_ke(st));
                        if (!last && tile_sees_chunk<BK>(nbits, t)) {
                            if (!k_next_ready) {
                                if (!wait_k(n + 1)) { fail = true; break; }
                                k_next_ready = true;
                                tc_fence_after();
                            }
                            if (!s_tile(t, g + 1, st1)) { fail = true; break; }
                        }
                    }
                    if (fail) break;
                    if (last) {
                        ++n;
                        break;
                    }
                    bits = nbits;
                }
                if (!fail) mbar_arrive(bar_le(b));
            }
            if (*abort_cta && issued) {
                umma_commit(bar_dr);
                mbar_drain(bar_dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax + epilogue
        const int t = (warp - 4) >> 2;              // tile of this warpgroup
        const int quad = warp & 3;                  // TMEM lane quadrant
        const int r = quad * 32 + lane;             // row within the tile
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const float sc = p.scale_log2;              // > 0
        int cnt = 0;                                // S_t blocks processed (all items)
        int n_ep = 0;                               // items with a PV of this tile (pv_done phases)
        int n0 = 0;                                 // union elements of the earlier items
        bool fail = false;
        for (int k = 0; !fail; ++k) {
            const int b = k & 1;
            if (!warp_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
            if (list_item[b] < 0) break;
            const ChunkItem I = items[b];
            const int qpos = (I.qt0 + t) * C::M + r;  // absolute position of this row
            const int rowbit = (BK == 128) ? t : 2 * t + (r >> 6);
            const bool active = (t == 0) || I.tile1;
            const bool row_valid = active && qpos >= I.c0 && qpos < I.n;
            const int n16 = ((I.n + kChunkPage - 1) / kChunkPage) * kChunkPage;  // end of the last page
            const uint32_t* L = list + b * C::LIST_CAP;
            const int len = list_len[b];
            const int n_item = n0;
            n0 += len;
            float m_used = -1e30f, l = 0.f;
            int cnt_item = 0;
            if (active) {
                for (int g = 0; g < len; ++g) {
                    const uint32_t ent = L[g];
                    if (!tile_sees_chunk<BK>(list_bits(ent), t)) continue;
                    const int j = list_j(ent);
                    if (!warp_wait(bar_sf(t), cnt & 1, ctl)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    uint32_t sr[C::NK];  // S row; packed P overwrites its front as it is consumed
#pragma unroll
                    for (int c = 0; c < C::NK / 32; ++c)
                        tmem_ld32(tl + C::colS(t) + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
                    tmem_wait_ld();
                    const bool vis = (list_bits(ent) >> rowbit) & 1;
                    const int lim = qpos - j * BK;  // key column c visible iff vis && c <= lim
                    if (!__all_sync(0xffffffffu, vis && lim >= BK - 1)) {
#pragma unroll
                        for (int c = 0; c < C::NK; ++c)
                            if (!(vis && c <= lim)) sr[c] = 0xff800000u;  // -inf
                    }
                    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < C::NK; c += 8) {
                        mx[0] = fmax3(mx[0], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                        mx[1] = fmax3(mx[1], __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
                        mx[2] = fmax3(mx[2], __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
                        mx[3] = fmax3(mx[3], __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
                    }
                    const float mt = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;
                    const float m_cand = fmaxf(m_used, mt);
                    const bool move = m_cand - m_used > 8.0f;  // rescale O only when the max grew by > 2^8
                    const float alpha = move ? ex2(m_used - m_cand) : 1.0f;
                    if (move) m_used = m_cand;
                    const float neg_m = -m_used;
                    float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int q = 0; q < C::NK / 2; ++q) {  // column pair (2q, 2q+1)
                        const float p0 = ex2(fmaf(__uint_as_float(sr[2 * q]), sc, neg_m));
                        const float p1 = ex2(fmaf(__uint_as_float(sr[2 * q + 1]), sc, neg_m));
                        rs[(2 * q) & 3] += p0;
                        rs[(2 * q + 1) & 3] += p1;
                        sr[q] = pack_bf16x2(p0, p1);  // slot q <= 2q: already read
                    }
                    l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
                    // P (bf16 pairs) over the first NK/2 columns of S_t.
#pragma unroll
                    for (int c = 0; c < C::NK / 64; ++c)
                        tmem_st32(tl + C::colS(t) + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32 * c]));
                    static_assert(C::NK % 64 == 0, "P stored in 32-column chunks");
                    // Rows of this block past the context inside its last page hold
                    // stale cache data: zero them in V before this tile's P V reads
                    // them (the block's loads have landed: S of it has completed).
                    const int z0 = I.n - j * BK, z1 = min(BK, n16 - j * BK);
                    if (z0 < z1) {
                        if (r >= z0 && r < z1) {
                            const int st = (n_item + g) % C::ST;
#pragma unroll
                            for (int pn = 0; pn < HD / 64; ++pn) {
                                uint4* row = reinterpret_cast<uint4*>(smem + C::OFF_V + st * C::KVBYTES +
                                                                      pn * (BK * 128) + r * 128);
#pragma unroll
                                for (int w2 = 0; w2 < 8; ++w2) row[w2] = make_uint4(0, 0, 0, 0);
                            }
                        }
                        fence_proxy_async_smem();  // generic-proxy writes read by the MMA
                    }
                    if (cnt_item > 0 && __any_sync(0xffffffffu, move)) {
                        // O_t is stable: S_t of this block was issued after PV_t of the
                        // previous one, and the next PV waits for this block's P.
#pragma unroll
                        for (int c = 0; c < HD / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tl + C::colO(t) + 32 * c, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e2 = 0; e2 < 32; ++e2) o[e2] = __float_as_uint(__uint_as_float(o[e2]) * alpha);
                            tmem_st32(tl + C::colO(t) + 32 * c, o);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_pf(t));
                    ++cnt;
                    ++cnt_item;
                }
            }
            if (fail) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_le(b));
            const int64_t orow = (int64_t)(I.q0 + qpos - I.c0) * p.heads + I.h;  // packed output row
            if (cnt_item > 0) {
                if (!warp_wait(bar_pv(t), (n_ep++) & 1, ctl)) break;  // the item's last PV of this tile
                tc_fence_after();
                const float inv = l > 0.f ? 1.0f / l : 0.f;
                uint16_t* og = p.out + orow * HD;
                // 32-byte stores (whole L2 sectors, half the store instructions) when
                // the output is 32-byte aligned: output rows of a tile are heads * HD
                // elements apart, so every store of the tile touches its own sectors
                const bool st32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tl + C::colO(t) + 32 * c, o);
                    tmem_wait_ld();
                    if (row_valid) store_bf16_row<32>(og + 32 * c, o, inv, st32);
                }
                if (row_valid && p.lse) p.lse[orow] = l > 0.f ? (m_used + lg2(l)) * 0.69314718055994531f : -INFINITY;
            } else if (row_valid) {  // no row of this tile lists a key block: zero output
                uint16_t* og = p.out + orow * HD;
                for (int d = 0; d < HD; d += 8) *reinterpret_cast<uint4*>(og + d) = make_uint4(0, 0, 0, 0);
                if (p.lse) p.lse[orow] = -INFINITY;
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    // every CTA has stopped taking items by now; the last one frees the slot
    if (threadIdx.x == 0 && misc[6]) sched_leave(p.sched);
}

}  // namespace s2
