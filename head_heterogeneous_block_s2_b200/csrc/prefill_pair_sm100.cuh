// prefill_pair_sm100.cuh -- block-sparse HHST prefill, two query tiles per CTA.
//
// S2-Attention ("S2-Attention: Hardware-aware context sharding among attention
// heads", Abstract) needs a FlashAttention-style kernel for sparsity to pay off;
// HHST shards the context across heads at block granularity, so the block is
// the tile here. One work item is a pair of adjacent 128-row query tiles of
// one (batch, head). Adjacent tiles share their strided key blocks and most
// local ones, so the CTA walks the union of their key-block lists, loads each
// key block once, and runs each tile's MMAs only on the blocks that tile sees.
//
// Key blocks are consumed in groups of G blocks (one S MMA of N = G * B keys
// and one softmax pass per group). K is stored panel-major across the stage
// ring so that G adjacent stages form one G*B-row K operand, and union lists
// are padded to a multiple of G with a fully masked entry. G = 2 for B = 64
// (N = 128 MMAs) was measured and lost to the extra masked work it issues
// (a tile computes both blocks of a group if it sees either), so G = 1.
//
// The kernel is persistent: one CTA per SM takes work items from a device
// counter (its first item is its block index), so the next item's loads and
// S MMAs overlap the current item's last groups and epilogue and the load
// balances itself (item order: see pair_item).
//
// CTA = 12 warps (14 with 64-key blocks):
//   warp 2      scheduler, list builder and Q producer: takes the next item
//               from the work counter, writes the item's union list and index
//               into a double-buffered shared-memory list, loads the item's Q
//               tiles once the previous item releases the shared-memory Q
//               buffer, and prefetches the next item's Q into L2.
//   warp 0      K/V producer: K and V of each union block, item after item,
//               into an ST-stage ring (TMA, SWIZZLE_128B, 64-column panels).
//   warp 1      owns TMEM; one thread issues the tcgen05.mma ops
//               S_t = Q_t K^T into TMEM and O_t += P_t V with P_t read from
//               TMEM (A operand) and V from shared memory (MN-major B operand).
//   warps 4..7  softmax of tile 0, warps 8..11 softmax of tile 1: thread = one
//               query row = one TMEM lane. Loads its S row of a group, masks
//               (union tag bit of its query block; token causality where the
//               key block reaches its own block), keeps a running max and sum
//               in the log2 domain, writes P (bf16 pairs) over the S columns
//               in TMEM, and at the end normalises O and stores it with the LSE.
//
// Two pipelines, chosen by block size (PairCfg):
//  * 64-key blocks (SDB): each tile has two S buffers in TMEM, and S of the
//    tile's next blocks is issued ahead of the softmax, so the tensor core
//    computes S of block i+1 while the softmax works on block i. With 64-key
//    blocks a single thread's chain of barrier waits, commits and MMA issues
//    (about 0.1-0.2k cycles each) was the limit, so four threads issue: per
//    tile one for S (warps 1 and 3) and one for PV (warps 12 and 13), each
//    walking the same union list; a K/V stage is released when all four have
//    committed, the Q buffer when both S issuers have. Q stays in shared
//    memory (TMEM is full).
//  * 128-key blocks: one S buffer per tile and one issuer for both tiles; the
//    two softmax warpgroups ping-pong (while one computes exponentials for its
//    tile, the tensor core runs the other tile's MMAs). When TMEM has room
//    (head dim 64), Q is copied into TMEM by tcgen05.cp at the start of the
//    item and S reads only K from shared memory. Warp 3 is idle.
//
// Ordering facts the pipelines rely on:
//  * tcgen05.mma and tcgen05.cp ops of one thread execute in issue order and a
//    commit tracks all earlier ones of that thread (so the next item's Q copy
//    lands after the current item's last S MMA has read Q from TMEM).
//  * One S buffer: S_t(next) is issued after PV_t(current), so when the
//    softmax sees S_t(next) complete, PV_t(current) has finished: P_t's TMEM
//    columns (aliased on S_t) are free and O_t is stable for a rescale.
//  * Two S buffers: S_t(i+2) is issued once PV_t(i) (same buffer) has
//    completed. The softmax waits for PV_t(i-1)'s own commit before it
//    rescales O_t at block i and before the epilogue; S_t(i) complete implies
//    PV_t(i-2) complete, so that barrier's phase cannot alias. Every S/P/PV
//    barrier is per buffer, for the same reason.
//  * Every issuing thread waits for each union element's loads, in order, and
//    commits kv_empty for it, including elements its tile skips: a stage can
//    then never be refilled before every thread has passed it, which keeps
//    each kv_full parity wait within one phase of the element it wants. (An S
//    thread that skipped unseen elements could see a stage one phase behind
//    as complete, or, waiting on them, one phase ahead that needs its own S.)
//  * A tile's first P of the next item is published only after its warpgroup
//    has read O out of TMEM (tcgen05.wait::ld) for the previous item, so the
//    next item's first PV (which overwrites O) cannot race the epilogue.
//  * The running-max reference only moves when the max grows by more than
//    2^8 (kRescaleLog2), so O rescales are rare; P values stay <= 256.
// Every wait is bounded; on a timeout the CTA drains its own copies and MMAs,
// frees TMEM and exits with the device timeout flag set.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"
#include "lists.cuh"  // union lists of compacted key-block rows
#include "umma.cuh"   // PrefillParams, umma_sdesc, umma_idesc

namespace s2 {


template <int HD, int BK>
struct PairCfg {
    static constexpr int M = 128;                          // rows per tile
    static constexpr int ROWS = (BK == 128) ? 2 : 4;       // query blocks per item
    static constexpr int G = 1;                            // key blocks per group (see below)
    static constexpr int NK = BK * G;                      // keys per group = S columns
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
    // barriers: q_full, q_empty, kv_full[ST] (K and V of a stage), kv_empty[ST],
    // s_full[2][2], p_full[2][2], pv_done[2][2] ([tile][S buffer]), drain[4]
    // (one per MMA issuer), list_full[2], list_empty[2]
    static constexpr int NBAR = 2 + 2 * ST + 12 + 4 + 4;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 32;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    // S double-buffered per tile (64-key blocks): the S MMA of a tile's next
    // block runs while the softmax works on the current one, so a tile's chain
    // is no longer S -> softmax -> PV -> S. Takes 4 NK + 2 HD TMEM columns, so
    // Q stays in shared memory. This pipeline has four MMA issuer threads, an
    // S issuer and a PV issuer per tile (warps 1 and 3: S of tiles 0 and 1;
    // warps 12 and 13: PV of tiles 0 and 1), in a 14-warp CTA.
    static constexpr bool SDB = BK == 64 && 4 * NK + 2 * HD <= 512;
    static constexpr int SBUF = SDB ? 2 : 1;
    static constexpr int THREADS = SDB ? 448 : 384;
    // threads that commit once per union element to kv_empty (and S issuers:
    // once per item to q_empty)
    static constexpr uint32_t KV_RELEASERS = SDB ? 4 : 1;
    static constexpr uint32_t Q_RELEASERS = SDB ? 2 : 1;
    // list_empty arrivals per item: K/V producer, MMA issuer(s), 8 softmax warps
    static constexpr uint32_t LIST_CONSUMERS = 9 + KV_RELEASERS;
    __host__ __device__ static constexpr uint32_t colS(int t, int u = 0) { return (uint32_t)((t * SBUF + u) * NK); }
    __host__ __device__ static constexpr uint32_t colO(int t) { return (uint32_t)(2 * SBUF * NK + t * HD); }
    // Without S double-buffering, when TMEM has room for both tiles' Q (HD/2
    // columns each) S = Q K^T reads Q from TMEM and only K from shared memory.
    static constexpr bool Q_IN_TMEM = !SDB && 2 * NK + 3 * HD <= 512;
    __host__ __device__ static constexpr uint32_t colQ(int t) { return (uint32_t)(2 * NK + 2 * HD + t * (HD / 2)); }
    static constexpr int TMEM_NEED = 2 * SBUF * NK + 2 * HD + (Q_IN_TMEM ? HD : 0);
    static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "TMEM budget");
    static_assert(!SDB || G == 1, "the double-buffered pipeline walks single blocks");
    static_assert(ST % G == 0, "groups must not wrap the stage ring");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

constexpr float kRescaleLog2 = 8.0f;

// Tile t's share of a union element's row tags.
template <int BK>
__device__ __forceinline__ bool tile_sees(int bits, int t)
{
    return BK == 128 ? ((bits >> t) & 1) != 0 : ((bits >> (2 * t)) & 3) != 0;
}

// Item order switch: head-major from this many tile pairs per head (measured:
// 32 pairs per head ran 5% faster in global heaviest-first order, 128 and 512
// pairs per head 11% faster head-major).
constexpr int kHeadMajorPairs = 64;

// One work item: a pair of adjacent 128-row query tiles of one (batch, head).
struct PairItem {
    int qt0, qb0, rp;
    bool tile1;
    int bh, bkv;       // (batch, query head) and (batch, K/V head) plane indices
    int64_t row_base;  // first output row of the plane: bh * seq
};

template <int BK>
__device__ __forceinline__ PairItem pair_item(const PrefillParams& p, int w)
{
    // Long sequences (many pairs per head): head by head, heaviest pairs first
    // within a head, so CTAs running together share one head's strided key
    // blocks in L2. Short ones: heaviest pairs of all heads first (the K/V of
    // every head is small, and a global heaviest-first order balances better).
    const int npairs = (p.nqt + 1) >> 1;
    const int BH = p.batch * p.heads;
    const bool head_major = npairs >= kHeadMajorPairs;
    const int pr = npairs - 1 - (head_major ? w % npairs : w / BH);
    const int bh = head_major ? w / npairs : w % BH;
    PairItem it;
    it.qt0 = 2 * pr;
    it.tile1 = it.qt0 + 1 < p.nqt;
    it.qb0 = (BK == 128) ? it.qt0 : 2 * it.qt0;
    it.rp = (bh % p.heads) * (p.nb + 1);
    it.bh = bh;
    it.bkv = (bh / p.heads) * p.heads_kv + (bh % p.heads) / (p.heads / p.heads_kv);
    it.row_base = (int64_t)bh * p.seq;
    return it;
}

template <int HD, int BK>
__global__ void __launch_bounds__(PairCfg<HD, BK>::THREADS, 1)
s2_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillParams p)
{
    using C = PairCfg<HD, BK>;
    constexpr int G = C::G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_items = p.batch * p.heads * ((p.nqt + 1) >> 1);

    const uint32_t bar_q = sb + C::OFF_BAR;
    const uint32_t bar_qe = sb + C::OFF_BAR + 8u;
    // K and V of a stage land on one barrier: the MMA thread waits once per
    // block (the loads run well ahead of it; a separate V barrier only added a
    // wait to its critical path).
    auto bar_kf = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + s); };
    auto bar_ke = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + C::ST + s); };
    // [tile][S buffer]
    auto bar_sf = [&](int t, int u = 0) { return sb + C::OFF_BAR + 8u * (2 + 2 * C::ST + 2 * t + u); };
    auto bar_pf = [&](int t, int u = 0) { return sb + C::OFF_BAR + 8u * (6 + 2 * C::ST + 2 * t + u); };
    auto bar_pv = [&](int t, int u = 0) { return sb + C::OFF_BAR + 8u * (10 + 2 * C::ST + 2 * t + u); };
    const uint32_t bar_dr = sb + C::OFF_BAR + 8u * (14 + 2 * C::ST);  // [4]: one per MMA issuer
    auto bar_lf = [&](int b) { return sb + C::OFF_BAR + 8u * (18 + 2 * C::ST + b); };
    auto bar_le = [&](int b) { return sb + C::OFF_BAR + 8u * (20 + 2 * C::ST + b); };
    const uint32_t* list = reinterpret_cast<const uint32_t*>(smem + C::OFF_LIST);
    // [0] tmem, [1] abort, [2..3] list lengths, [4..5] item of each list buffer (-1: no more)
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_cta = misc + 1;
    volatile int* list_len = misc + 2;
    volatile int* list_item = misc + 4;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_qe, C::Q_RELEASERS);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_ke(s), C::KV_RELEASERS);
        }
        for (int t = 0; t < 2; ++t) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(bar_sf(t, u), 1);
                mbar_init(bar_pf(t, u), 128);
                mbar_init(bar_pv(t, u), 1);
            }
            mbar_init(bar_lf(t), 1);
            mbar_init(bar_le(t), C::LIST_CONSUMERS);
        }
        for (int i = 0; i < 4; ++i) mbar_init(bar_dr + 8u * i, 1);
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
        // ------------------------------------------------------------ list builder + Q producer
        if (lane == 0) {
            int k = 0;
            uint32_t* wlist = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
            int w = blockIdx.x;  // first item static, the rest from the work counter
            for (;; ++k) {
                const int b = k & 1;
                // union list of this item into buffer b (free once item k-2 is consumed)
                if (!mbar_wait(bar_le(b), ((k >> 1) & 1) ^ 1, ctl)) break;
                if (w >= num_items) {  // tell every role there is no more work
                    list_item[b] = -1;
                    list_len[b] = 0;
                    mbar_arrive(bar_lf(b));
                    break;
                }
                const int w_next = misc[6] ? (int)gridDim.x + sched_take(p.sched) : num_items;
                const PairItem I = pair_item<BK>(p, w);
                UnionWalk<C::ROWS> it;
                int len = 0;
                const bool ok = it.init(p.row_ptr, I.rp, I.qb0, p.nb, p.nnz);
                if (it.any) {  // an item whose rows are all empty publishes an empty list
                    for (;;) {
                        int j, bits;
                        bool last, bad;
                        it.next(p.col_idx, j, bits, last, bad);
                        if (bad) atomicOr(p.gflags, kFlagIndex);
                        if (len >= C::LIST_CAP - G) {  // cannot happen when nb <= LIST_CAP - G
                            atomicOr(p.gflags, kFlagIndex);
                            last = true;
                        }
                        wlist[b * C::LIST_CAP + len++] = list_pack(j, bits);
                        if (last) break;
                    }
                    while (len % G) wlist[b * C::LIST_CAP + len++] = list_pack(0, 0);  // masked pad
                } else if (!ok) {
                    atomicOr(p.gflags, kFlagIndex);
                }
                list_len[b] = len;
                list_item[b] = w;
                mbar_arrive(bar_lf(b));
                // Q of both tiles, once the previous item's S MMAs are done with the buffer
                if (!mbar_wait(bar_qe, (k & 1) ^ 1, ctl)) break;
                mbar_arrive_expect_tx(bar_q, (I.tile1 ? 2 : 1) * C::QBYTES);
                for (int t = 0; t < (I.tile1 ? 2 : 1); ++t)
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_3d(sb + C::OFF_Q + t * C::QBYTES + pn * (C::M * 128), &tmQ, pn * 64,
                                    (I.qt0 + t) * C::M, I.bh, bar_q);
                if (w_next < num_items) {  // next item's Q into L2
                    const PairItem J = pair_item<BK>(p, w_next);
                    for (int t = 0; t < (J.tile1 ? 2 : 1); ++t)
                        for (int pn = 0; pn < HD / 64; ++pn)
                            tma_prefetch_3d(&tmQ, pn * 64, (J.qt0 + t) * C::M, J.bh);
                }
                w = w_next;
            }
            if (*abort_cta && k > 0) mbar_drain(bar_q, (k - 1) & 1, kDrainNs);
        }
        __syncwarp();
    } else if (warp == 0) {
        // ------------------------------------------------------------ K/V producer
        if (lane == 0) {
            int n = 0, k = 0;
            bool stop = false;
            for (; !stop; ++k) {
                const int b = k & 1;
                if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                const int w = list_item[b];
                if (w < 0) break;
                const PairItem I = pair_item<BK>(p, w);
                const uint32_t* L = list + b * C::LIST_CAP;
                const int len = list_len[b];
                for (int e = 0; e < len; ++e, ++n) {
                    const int st = n % C::ST;
                    if (!mbar_wait(bar_ke(st), ((n / C::ST) & 1) ^ 1, ctl)) {
                        stop = true;
                        break;
                    }
                    const int32_t krow = list_j(L[e]) * BK;
                    mbar_arrive_expect_tx(bar_kf(st), 2 * C::KVBYTES);
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_3d(sb + C::OFF_K + pn * C::KPANEL + st * (BK * 128), &tmK, pn * 64, krow,
                                    I.bkv, bar_kf(st));
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_3d(sb + C::OFF_V + st * C::KVBYTES + pn * (BK * 128), &tmV, pn * 64,
                                    krow, I.bkv, bar_kf(st));
                }
                if (!stop) mbar_arrive(bar_le(b));
            }
            if (*abort_cta)  // let this CTA's own loads land before exit
                for (int m = (n > C::ST ? n - C::ST : 0); m < n; ++m)
                    mbar_drain(bar_kf(m % C::ST), (m / C::ST) & 1, kDrainNs);
        }
        __syncwarp();
    } else if (warp == 1 || (C::SDB && (warp == 3 || warp >= 12))) {
        // ------------------------------------------------------------ MMA issuer(s)
        if constexpr (C::SDB) {
            // Per tile an S issuer (warp 1: tile 0, warp 3: tile 1) and a PV issuer
            // (warp 12: tile 0, warp 13: tile 1), each walking the same union list.
            // The i-th S of a tile goes to its S buffer i & 1; S_{i+2} reuses the
            // buffer of block i, so the S issuer waits for PV_i's commit first
            // (the two threads' MMAs have no issue-order relation). Both commit
            // kv_empty once per union element: a stage is free when K (read by
            // S) and V (read by PV) of both tiles are done.
            const bool s_role = warp == 1 || warp == 3;
            const int T = s_role ? (warp == 1 ? 0 : 1) : warp - 12;
            const uint32_t my_dr = bar_dr + 8u * (s_role ? T : 2 + T);
            if (lane == 0) {
                constexpr uint32_t idesc_s = umma_idesc(128, C::NK, 0, 0);
                constexpr uint32_t idesc_o = umma_idesc(128, HD, 0, 1);
                bool issued = false, fail = false;
                int cnt = 0;  // S (or PV) MMAs of tile T issued so far (all items)
                int n0 = 0;   // union elements of the earlier items
                const uint64_t dq = umma_sdesc(sb + C::OFF_Q + T * C::QBYTES, 16, 1024);
                for (int k = 0; !fail; ++k) {
                    const int b = k & 1;
                    if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                    if (list_item[b] < 0) break;
                    const uint32_t* L = list + b * C::LIST_CAP;
                    const int len = list_len[b];
                    const bool mine = T == 0 || pair_item<BK>(p, list_item[b]).tile1;  // tile T exists
                    int last_seen = -1;  // last element tile T sees in this item
                    if (s_role) {
                        if (!mbar_wait(bar_q, k & 1, ctl)) break;
                        for (int e = len - 1; mine && e >= 0; --e)
                            if (tile_sees<BK>(list_bits(L[e]), T)) {
                                last_seen = e;
                                break;
                            }
                        if (last_seen < 0) umma_commit(bar_qe);  // Q_T unused in this item
                    }
                    bool first = true;
                    for (int e = 0; e < len; ++e) {
                        const int n = n0 + e, st = n % C::ST;
                        const bool sees = mine && tile_sees<BK>(list_bits(L[e]), T);
                        if (s_role) {
                            // S buffer cnt & 1 is free once PV_{cnt-2} completed (PV_{cnt-4}
                            // completed before S_{cnt-2} was issued: no phase aliasing)
                            if (sees && cnt >= 2 &&
                                !mbar_wait(bar_pv(T, cnt & 1), ((cnt - 2) >> 1) & 1, ctl)) {
                                fail = true;
                                break;
                            }
                            if (!mbar_wait(bar_kf(st), (n / C::ST) & 1, ctl)) {
                                fail = true;
                                break;
                            }
                            if (sees) {
                                tc_fence_after();
                                const uint64_t dk = umma_sdesc(sb + C::OFF_K + st * (BK * 128), 16, 1024);
#pragma unroll
                                for (int kk = 0; kk < HD / 16; ++kk)
                                    umma_bf16_ss(tmem + C::colS(T, cnt & 1),
                                                 dq + (((kk >> 2) * (C::M * 128) + (kk & 3) * 32) >> 4),
                                                 dk + (((kk >> 2) * C::KPANEL + (kk & 3) * 32) >> 4), idesc_s,
                                                 kk > 0 ? 1u : 0u);
                                umma_commit(bar_sf(T, cnt & 1));
                                ++cnt;
                                issued = true;
                                if (e == last_seen) umma_commit(bar_qe);  // no more S of this item reads Q_T
                            }
                        } else if (sees) {
                            if (!mbar_wait(bar_pf(T, cnt & 1), (cnt >> 1) & 1, ctl)) {
                                fail = true;
                                break;
                            }
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < C::NK / 16; ++kk)
                                umma_bf16_ts(tmem + C::colO(T), tmem + C::colS(T, cnt & 1) + kk * 8,
                                             umma_sdesc(sb + C::OFF_V + st * C::KVBYTES + kk * 2048, BK * 128, 1024),
                                             idesc_o, (kk > 0 || !first) ? 1u : 0u);
                            // the softmax waits on this before an O rescale and the epilogue,
                            // the S issuer before reusing the buffer
                            umma_commit(bar_pv(T, cnt & 1));
                            ++cnt;
                            first = false;
                            issued = true;
                        } else if (!mbar_wait(bar_kf(st), (n / C::ST) & 1, ctl)) {
                            // a block tile T skips: its loads land before the stage is released
                            // (so this arrival cannot count toward an earlier use of the stage)
                            fail = true;
                            break;
                        }
                        umma_commit(bar_ke(st));
                    }
                    if (fail) break;
                    n0 += len;
                    mbar_arrive(bar_le(b));
                }
                if (*abort_cta && issued) {
                    umma_commit(my_dr);
                    mbar_drain(my_dr, 0, kDrainNs);
                }
            }
        } else {
            if (lane == 0) {
                constexpr uint32_t idesc_s = umma_idesc(128, C::NK, 0, 0);
                constexpr uint32_t idesc_o = umma_idesc(128, HD, 0, 1);
                constexpr int KSTEPS_BLK = BK / 16;  // PV k-steps per key block
                bool issued = false, fail = false;
                int pvc[2] = {0, 0};  // PV groups issued per tile (all items)
                bool first_pv[2] = {true, true};
                int n = 0;            // union elements consumed (all items); a multiple of G
                // S_t = Q_t K^T over the G blocks of the group starting at stage st (N = 128).
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
                // O_t += P_t V over the group's G blocks (stages st .. st+G-1).
                auto issue_pv = [&](int t, int st) {
                    const uint32_t acc0 = first_pv[t] ? 0u : 1u;
#pragma unroll
                    for (int kk = 0; kk < C::NK / 16; ++kk) {
                        const int s = st + kk / KSTEPS_BLK;
                        const uint64_t dv = umma_sdesc(sb + C::OFF_V + s * C::KVBYTES + (kk % KSTEPS_BLK) * 2048,
                                                       BK * 128, 1024);
                        umma_bf16_ts(tmem + C::colO(t), tmem + C::colS(t) + kk * 8, dv, idesc_o,
                                     kk > 0 ? 1u : acc0);
                    }
                    ++pvc[t];
                    first_pv[t] = false;
                };
                int k = 0;
                for (; !fail; ++k) {
                    const int b = k & 1;
                    if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                    if (list_item[b] < 0) break;
                    const uint32_t* L = list + b * C::LIST_CAP;
                    const int len = list_len[b];
                    if (!mbar_wait(bar_q, k & 1, ctl)) break;
                    if (len == 0) {
                        umma_commit(bar_qe);
                        mbar_arrive(bar_le(b));
                        continue;
                    }
                    if constexpr (C::Q_IN_TMEM) {
                        // Q of both tiles into TMEM (after the previous item's S MMAs, in
                        // issue order), then the shared-memory Q buffer is free at once.
                        tc_fence_after();
                        const bool two = pair_item<BK>(p, list_item[b]).tile1;
                        for (int t = 0; t < (two ? 2 : 1); ++t) {
                            const uint64_t dq = umma_sdesc(sb + C::OFF_Q + t * C::QBYTES, 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk)
                                tmem_cp_128x256b(tmem + C::colQ(t) + kk * 8,
                                                 dq + (((kk >> 2) * (C::M * 128) + (kk & 3) * 32) >> 4));
                        }
                        umma_commit(bar_qe);
                    }
                    const int ngroups = len / G;
                    first_pv[0] = first_pv[1] = true;
                    auto gbits = [&](int g) {
                        int bits = 0;
#pragma unroll
                        for (int i = 0; i < G; ++i) bits |= list_bits(L[g * G + i]);
                        return bits;
                    };
                    auto wait_k = [&](int n0) {
                        for (int i = 0; i < G; ++i)
                            if (!mbar_wait(bar_kf((n0 + i) % C::ST), ((n0 + i) / C::ST) & 1, ctl)) return false;
                        return true;
                    };
                    int bits = gbits(0);
                    if (!wait_k(n)) break;
                    tc_fence_after();
                    for (int t = 0; t < 2; ++t)
                        if (tile_sees<BK>(bits, t)) issue_s(t, n % C::ST);
                    for (int g = 0;; ++g, n += G) {
                        const bool last = g + 1 == ngroups;
                        const int nbits = last ? 0 : gbits(g + 1);
                        const int st = n % C::ST;
                        const int st1 = (n + G) % C::ST;
                        if (last && !C::Q_IN_TMEM) umma_commit(bar_qe);  // no more S MMAs of this item read Q
                        // K and V of this group landed together: S of the group was issued
                        // after waiting for them (or the malformed case below waits)
                        bool k_next_ready = false;
                        if (bits == 0) {  // malformed group no tile sees: let its loads land first
                            if (!wait_k(n)) {
                                fail = true;
                                break;
                            }
                        }
                        const int last_t = tile_sees<BK>(bits, 1) ? 1 : (tile_sees<BK>(bits, 0) ? 0 : 1);
                        for (int t = 0; t < 2 && !fail; ++t) {
                            if (tile_sees<BK>(bits, t)) {
                                if (!mbar_wait(bar_pf(t), pvc[t] & 1, ctl)) { fail = true; break; }
                                tc_fence_after();
                                issue_pv(t, st);
                            }
                            if (t == last_t)
                                for (int i = 0; i < G; ++i) umma_commit(bar_ke(st + i));
                            if (!last && tile_sees<BK>(nbits, t)) {
                                if (!k_next_ready) {
                                    if (!wait_k(n + G)) { fail = true; break; }
                                    k_next_ready = true;
                                    tc_fence_after();
                                }
                                issue_s(t, st1);
                            }
                        }
                        if (fail) break;
                        if (last) {
                            n += G;
                            break;
                        }
                        bits = nbits;
                    }
                    if (!fail) {
                        // O_t of this item is complete once its last PV is: one commit per
                        // tile and item (the softmax reads O only in the epilogue)
                        for (int t = 0; t < 2; ++t)
                            if (!first_pv[t]) umma_commit(bar_pv(t));
                        mbar_arrive(bar_le(b));
                    }
                }
                if (*abort_cta && issued) {
                    umma_commit(bar_dr);
                    mbar_drain(bar_dr, 0, kDrainNs);
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax
        const int t = (warp - 4) >> 2;              // tile of this warpgroup
        const int quad = warp & 3;                  // TMEM lane quadrant
        const int r = quad * 32 + lane;             // row within the tile
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const float sc = p.scale_log2;              // > 0
        int cnt = 0;                                // S_t groups processed (all items)
        int n_ep = 0;                               // items with a PV of this tile (pv_done phases)
        bool fail = false;
        int k = 0;
        for (; !fail; ++k) {
            const int b = k & 1;
            if (!warp_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
            const int w = list_item[b];
            if (w < 0) break;
            const PairItem I = pair_item<BK>(p, w);
            const int qpos = (I.qt0 + t) * C::M + r;
            const int rowbit = (BK == 128) ? t : 2 * t + (r >> 6);
            const bool active = (t == 0) || I.tile1;
            const bool row_valid = active && qpos < p.seq && (I.qb0 + rowbit) < p.nb;
            const uint32_t* L = list + b * C::LIST_CAP;
            const int len = list_len[b];
            float m_used = -1e30f, l = 0.f;
            int cnt_item = 0;
            if (active) {
                for (int g = 0; g < len / G; ++g) {
                    uint32_t ent[G];
                    int bits = 0;
#pragma unroll
                    for (int i = 0; i < G; ++i) {
                        ent[i] = L[g * G + i];
                        bits |= list_bits(ent[i]);
                    }
                    if (!tile_sees<BK>(bits, t)) continue;
                    // S buffer of this block and the phase of its barriers
                    const int u = C::SDB ? (cnt & 1) : 0;
                    const uint32_t par = C::SDB ? ((cnt >> 1) & 1) : (cnt & 1);
                    if (!warp_wait(bar_sf(t, u), par, ctl)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    uint32_t sr[C::NK];  // S row; packed P overwrites its front as it is consumed
#pragma unroll
                    for (int c = 0; c < C::NK / 32; ++c)
                        tmem_ld32(tl + C::colS(t, u) + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
                    tmem_wait_ld();
                    bool vis[G];
                    int lim[G];  // key column c of block i visible iff vis[i] && c <= lim[i]
                    bool full = true;
#pragma unroll
                    for (int i = 0; i < G; ++i) {
                        vis[i] = (list_bits(ent[i]) >> rowbit) & 1;
                        lim[i] = qpos - list_j(ent[i]) * BK;
                        full = full && vis[i] && lim[i] >= BK - 1;
                    }
                    if (!__all_sync(0xffffffffu, full)) {
#pragma unroll
                        for (int c = 0; c < C::NK; ++c)
                            if (!(vis[c / BK] && (c % BK) <= lim[c / BK])) sr[c] = 0xff800000u;  // -inf
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
                    const bool move = m_cand - m_used > kRescaleLog2;
                    const float alpha = move ? ex2(m_used - m_cand) : 1.0f;
                    if (move) m_used = m_cand;
                    const float neg_m = -m_used;
                    float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int q = 0; q < C::NK / 2; ++q) {  // column pair (2q, 2q+1)
                        float p0, p1;
                        if constexpr (C::SDB) {
                            // packed pair FMA and ADD: 5 instructions per pair instead of 7
                            // (this loop's instruction count, not the exponential unit,
                            // is what the softmax spends its time on)
                            float x0, x1;
                            ffma2(x0, x1, __uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1]), sc, neg_m);
                            p0 = ex2(x0);
                            p1 = ex2(x1);
                            fadd2(rs[(q & 1) * 2], rs[(q & 1) * 2 + 1], p0, p1);
                        } else {
                            p0 = ex2(fmaf(__uint_as_float(sr[2 * q]), sc, neg_m));
                            p1 = ex2(fmaf(__uint_as_float(sr[2 * q + 1]), sc, neg_m));
                            rs[(2 * q) & 3] += p0;
                            rs[(2 * q + 1) & 3] += p1;
                        }
                        sr[q] = pack_bf16x2(p0, p1);  // slot q <= 2q: already read
                    }
                    l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
                    // P (bf16 pairs) over the first NK/2 columns of S_t.
#pragma unroll
                    for (int c = 0; c < C::NK / 64; ++c)
                        tmem_st32(tl + C::colS(t, u) + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32 * c]));
                    static_assert(C::NK % 64 == 0, "P stored in 32-column chunks");
                    if (cnt_item > 0 && __any_sync(0xffffffffu, move)) {
                        // O_t must hold PV_t of the previous block and no later one (the
                        // next PV waits for this block's P). Single S buffer: S_t of this
                        // block was issued after that PV, so it has completed. Double
                        // buffer: wait for that PV's commit (the PV before it completed
                        // before this block's S did, so the phase cannot alias).
                        if constexpr (C::SDB) {
                            if (!warp_wait(bar_pv(t, (cnt - 1) & 1), ((cnt - 1) >> 1) & 1, ctl)) {
                                fail = true;
                                break;
                            }
                            tc_fence_after();
                        }
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
                    mbar_arrive(bar_pf(t, u));
                    ++cnt;
                    ++cnt_item;
                }
            }
            if (fail) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_le(b));
            if (cnt_item > 0) {
                // O_t complete: the commit after this item's last PV (single S buffer:
                // one commit per item; double buffer: one per PV, the last one's phase)
                const bool ok = C::SDB ? warp_wait(bar_pv(t, (cnt - 1) & 1), ((cnt - 1) >> 1) & 1, ctl)
                                       : warp_wait(bar_pv(t), (n_ep++) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                const float inv = l > 0.f ? 1.0f / l : 0.f;
                uint16_t* orow = p.o + (I.row_base + qpos) * HD;
                if constexpr (C::SDB) {
                    // Each thread writes its own row: 32-byte stores (whole L2 sectors,
                    // half the store instructions of 16-byte ones) when O is 32-byte
                    // aligned, and 64 columns loaded per tcgen05 wait. (The 128-key
                    // kernel is at its register cap and keeps 32-column loads and
                    // 16-byte stores: the wider form spilled and ran 7% slower there.)
                    const bool st32 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
#pragma unroll
                    for (int c = 0; c < HD / 64; ++c) {
                        uint32_t o[64];
                        tmem_ld32(tl + C::colO(t) + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                        tmem_ld32(tl + C::colO(t) + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                        tmem_wait_ld();
                        if (row_valid) {
#pragma unroll
                            for (int e2 = 0; e2 < 64; e2 += 16) {
                                uint32_t w[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    w[i] = pack_bf16x2(__uint_as_float(o[e2 + 2 * i]) * inv,
                                                       __uint_as_float(o[e2 + 2 * i + 1]) * inv);
                                if (st32) {
                                    st_global_v8(orow + 64 * c + e2, w);
                                } else {
                                    *reinterpret_cast<uint4*>(orow + 64 * c + e2) = make_uint4(w[0], w[1], w[2], w[3]);
                                    *reinterpret_cast<uint4*>(orow + 64 * c + e2 + 8) =
                                        make_uint4(w[4], w[5], w[6], w[7]);
                                }
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tl + C::colO(t) + 32 * c, o);
                        tmem_wait_ld();
                        if (row_valid) {
#pragma unroll
                            for (int e2 = 0; e2 < 32; e2 += 8) {
                                uint4 v;
                                v.x = pack_bf16x2(__uint_as_float(o[e2 + 0]) * inv, __uint_as_float(o[e2 + 1]) * inv);
                                v.y = pack_bf16x2(__uint_as_float(o[e2 + 2]) * inv, __uint_as_float(o[e2 + 3]) * inv);
                                v.z = pack_bf16x2(__uint_as_float(o[e2 + 4]) * inv, __uint_as_float(o[e2 + 5]) * inv);
                                v.w = pack_bf16x2(__uint_as_float(o[e2 + 6]) * inv, __uint_as_float(o[e2 + 7]) * inv);
                                *reinterpret_cast<uint4*>(orow + 32 * c + e2) = v;
                            }
                        }
                    }
                }
                if (row_valid && p.lse)
                    p.lse[I.row_base + qpos] = l > 0.f ? (m_used + lg2(l)) * 0.69314718055994531f : -INFINITY;
            } else if (row_valid) {  // no row of this tile lists a key block: zero output
                uint16_t* orow = p.o + (I.row_base + qpos) * HD;
                for (int d = 0; d < HD; d += 8) *reinterpret_cast<uint4*>(orow + d) = make_uint4(0, 0, 0, 0);
                if (p.lse) p.lse[I.row_base + qpos] = -INFINITY;
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
