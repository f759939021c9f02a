// backward_sm100.cuh -- block-sparse backward (dQ, dK, dV) of the HHST
// attention on sm_100a.
//
// The arXiv abstract of "S2-Attention: Hardware-aware context sharding among
// attention heads" reports training speedups over FlashAttention-2, so the
// gradients run on the same compacted block lists as the forward. With the
// forward's LSE and an upstream gradient dO, per visible (q, k):
//
//   P = exp(s - LSE_q),  dP = dO_q . V_k,  D_q = dO_q . O_q,  dS = P (dP - D_q)
//   dQ_q = scale sum_k dS K_k,  dK_k = scale sum_q dS Q_q,  dV_k = sum_q P dO_q
//
// (D_q = sum_k P dP because O_q = sum_k P V_k.) Three kernels:
//
//   s2_bwd_stats_kernel  per query row: (LSE * log2 e, D_q) into a row-padded
//                        fp32 workspace; rows past seq get (+inf, 0) so that
//                        any P computed for them is exactly 0.
//   s2_bwd_dq_kernel     persistent; one 128-row query tile per work item,
//                        walking the union of its query blocks' key-block
//                        lists (the forward's lists): S = Q K^T and dP = dO V^T
//                        into TMEM, dS (bf16) written back over dP, dQ += dS K
//                        with dS read from TMEM and K from shared memory as an
//                        MN-major B. An element is 128 keys: one 128-key
//                        block, or two list entries with 64-key blocks.
//   s2_bwd_dkv_kernel    one 128-row key tile per CTA, walking the union of
//                        its key blocks' transposed lists (query blocks that
//                        list them): S^T = K Q^T and dP^T = V dO^T into TMEM,
//                        P^T and dS^T (bf16) written back over them, then
//                        dV += P^T dO and dK += dS^T Q with the A operands
//                        read from TMEM. 128-key blocks.
//   s2_bwd_dkv_persistent_kernel
//                        the same per key tile for 64-key blocks (two blocks
//                        per tile), persistent over tiles like the dQ kernel,
//                        with K and V in TMEM.
// dQ and dK/dV are computed by separate kernels (S and dP are recomputed by
// both) so that no accumulator is shared between CTAs: no atomics, and the
// results are deterministic.
//
// CTA = 12 warps: warp 0 TMA producer; warp 1 TMEM owner and MMA issuer (one
// thread); warp 2 builds the union list in shared memory (in the persistent
// kernels item after item, double-buffered, and it also loads the item's Q
// and dO, or K and V); warps 4..11 the element-wise passes and the epilogue:
// thread = one tile row = one TMEM lane, warps 4..7 on the first half of the
// columns and warps 8..11 on the second (two warps per SM sub-partition hide
// the exponential and TMEM latencies; a single warpgroup was measured to leave
// the tensor core idle most of the time). In the persistent dK/dV kernel
// (N = 64 products, which one thread issues at half the tensor core's rate) a
// thread of warp 3 issues too: dV(G) then S^T(G+1) from warp 1, dK(G) then
// dP^T(G+1) from warp 3.
// With B = 64 a 128-row tile holds two blocks and every row masks by its own
// block's tag. Every wait is bounded; on a timeout the CTA drains its own
// copies and MMAs, frees TMEM and exits with the device timeout flag set.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>

#include "lists.cuh"
#include "ptx.cuh"
#include "store.cuh"  // store_bf16_row
#include "umma.cuh"

namespace s2 {

struct BackwardParams {
    const int32_t* row_ptr;  // key-block lists of query blocks (the forward's layout)
    const int32_t* col_idx;
    const int32_t* col_ptr;  // query-block lists of key blocks (its transpose)
    const int32_t* row_idx;
    const int32_t* key_tiles;  // B = 64: [heads][ntiles][2] key blocks of each key tile (-1: none)
    int64_t nnz;
    const uint16_t* o;     // [batch][heads][seq][HD] forward output (stats kernel)
    const uint16_t* dout;  // [batch][heads][seq][HD] upstream gradient (stats kernel)
    const float* lse;      // [batch][heads][seq] forward LSE, natural log (stats kernel)
    float* stats;          // [batch * heads][seq_pad / 128][2][128]: LSE * log2 e, then D
    uint16_t* dq;          // [batch][heads][seq][HD]
    uint16_t* dk;          // [batch][heads_kv][seq][HD]: summed over each K/V head's query heads
    uint16_t* dv;
    int32_t batch, heads, heads_kv, seq, seq_pad, nb, ntiles;  // query head h reads K/V head h / (heads / heads_kv)
    float scale;       // logit scale
    float scale_log2;  // scale * log2 e
    uint64_t timeout_ns;
    uint32_t* gflags;
    int* sched;     // dQ kernel work-counter slot (sched_claim / sched_take / sched_leave)
    int* sched_kv;  // the same for the persistent dK/dV kernel (64-key blocks)
    int sched_id, sched_kv_id;  // the two launches' nonzero ids
};

// Descriptor offset (16-byte units) of k-step kk (16 elements) of a K-major
// SWIZZLE_128B operand of `rows` rows stored as 64-column panels.
__device__ __forceinline__ uint64_t kstep(int kk, int rows)
{
    return (uint64_t)((((kk >> 2) * (rows * 128)) + (kk & 3) * 32) >> 4);
}

// N consecutive 32-bit TMEM columns of this thread's lane (N = 16, 32 or 64).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N])
{
    if constexpr (N == 16) {
        tmem_ld16(taddr, r);
    } else {
#pragma unroll
        for (int c = 0; c < N / 32; ++c)
            tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N])
{
    if constexpr (N == 16) {
        tmem_st16(taddr, r);
    } else {
#pragma unroll
        for (int c = 0; c < N / 32; ++c)
            tmem_st32(taddr + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&r[32 * c]));
    }
}

// TMEM column of k-step kk (16 rows of K) of a bf16 A operand written by the
// two element-wise warpgroups: half g = kk / (BK / 32) of the BK columns was
// packed into the first BK / 4 columns of that half's own range.
template <int BK>
__host__ __device__ constexpr uint32_t packed_col(int kk)
{
    return (uint32_t)((kk / (BK / 32)) * (BK / 2) + (kk % (BK / 32)) * 8);
}

// ------------------------------------------------------------------ stats

// One group of HD/8 threads per row (8 bf16 of dO and O per thread); the loop
// runs warp by warp so that every lane of a warp takes part in each shuffle.
template <int HD>
__global__ void __launch_bounds__(256) s2_bwd_stats_kernel(const BackwardParams p)
{
    constexpr int TPR = HD / 8;
    constexpr int RPW = 32 / TPR;  // rows per warp
    const int64_t rows = (int64_t)p.batch * p.heads * p.seq_pad;
    const int lane = threadIdx.x & 31, sub = lane % TPR;
    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp_id * RPW; base < rows; base += nwarps * RPW) {
        const int64_t r = base + lane / TPR;
        const int64_t bh = r / p.seq_pad;
        const int q = (int)(r % p.seq_pad);
        float d = 0.f;
        if (r < rows && q < p.seq) {
            const int64_t off = (bh * p.seq + q) * HD + sub * 8;
            const uint4 a = *reinterpret_cast<const uint4*>(p.o + off);
            const uint4 b = *reinterpret_cast<const uint4*>(p.dout + off);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                d = fmaf(bf16lo(av[i]), bf16lo(bv[i]), fmaf(bf16hi(av[i]), bf16hi(bv[i]), d));
        }
#pragma unroll
        for (int w = TPR / 2; w > 0; w >>= 1) d += __shfl_xor_sync(0xffffffffu, d, w);
        if (sub == 0 && r < rows) {  // planar per 128-row tile: 128 values of L2, then 128 of D
            float* t = p.stats + (r / 128) * 256 + (r % 128);
            t[0] = q < p.seq ? p.lse[bh * p.seq + q] * 1.4426950408889634f : INFINITY;
            t[128] = q < p.seq ? d : 0.f;
        }
    }
}

// ------------------------------------------------------------------ dQ

template <int HD, int BK>
struct BwdQCfg {
    static constexpr int M = 128;
    static constexpr int ROWS = (BK == 128) ? 1 : 2;  // query blocks per tile
    // One element = NK = 128 keys: one 128-key block, or two consecutive
    // entries of the union list with 64-key blocks (an odd last entry is
    // paired with a fully masked pad). The two entries of a pair need not be
    // adjacent blocks: each element-wise warpgroup masks its own 64 columns
    // by its own entry, and every row of the tile computes every element of
    // the union anyway, so pairing adds no masked work beyond the pad. S, dP
    // and dQ are then N = 128 / K = 128 products, which one thread issues at
    // the tensor core's rate.
    static constexpr int NK = 128;
    static constexpr int KPE = NK / BK;               // list entries per element
    static constexpr uint32_t TBYTES = M * HD * 2;    // Q or dO tile
    static constexpr uint32_t KVBYTES = NK * HD * 2;  // K or V of one element
    static constexpr int ST = 2;
    static constexpr int LIST_CAP = 2048;
    static constexpr uint32_t LIST_BYTES = 2 * LIST_CAP * 4;  // double-buffered
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_DO = TBYTES;
    static constexpr uint32_t OFF_K = 2 * TBYTES;              // [stage][panel][NK rows x 128 B]
    static constexpr uint32_t OFF_V = OFF_K + ST * KVBYTES;
    static constexpr uint32_t OFF_LIST = OFF_V + ST * KVBYTES;
    static constexpr uint32_t OFF_BAR = OFF_LIST + LIST_BYTES;
    // barriers: qd_full, qd_empty, k_full[ST], v_full[ST], kv_empty[ST], s_full, ds_full, acc_done,
    // drain, dp_full, s_free, list_full[2], list_empty[2]
    static constexpr int NBAR = 2 + 3 * ST + 6 + 4;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 32;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    // producer, MMA issuer, 8 element-wise warps
    static constexpr uint32_t LIST_CONSUMERS = 10;
    static constexpr uint32_t COL_S = 0, COL_DP = NK, COL_ACC = 2 * NK;
    // Q and dO, the A operands of every S and dP MMA of an item, sit in TMEM
    // (HD/2 columns each): those MMAs read only K or V from shared memory.
    static constexpr uint32_t COL_QA = 2 * NK + HD, COL_DOA = 2 * NK + HD + HD / 2;
    static constexpr uint32_t TMEM_COLS = (2 * NK + 2 * HD) <= 256 ? 256 : 512;
    static_assert(2 * NK + 2 * HD <= 512, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Persistent: each CTA takes work items (one 128-row query tile of one plane,
// the tiles with the longest lists first) from a device counter; a warp
// builds the next item's union list and loads its Q and dO while the current
// item runs, so items follow one another without a prologue.
template <int HD, int BK>
__global__ void __launch_bounds__(384, 1)
s2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const BackwardParams p)
{
    using C = BwdQCfg<HD, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BH = p.batch * p.heads;
    const int num_items = p.ntiles * BH;
    auto item_qt = [&](int w) { return p.ntiles - 1 - w / BH; };  // longest lists first
    auto item_bh = [&](int w) { return w % BH; };

    const uint32_t bar_qd = sb + C::OFF_BAR;
    const uint32_t bar_qe = sb + C::OFF_BAR + 8u;
    auto bar_kf = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + s); };
    auto bar_vf = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + C::ST + s); };
    auto bar_ke = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + 2 * C::ST + s); };
    const uint32_t bar_s = sb + C::OFF_BAR + 8u * (2 + 3 * C::ST);
    const uint32_t bar_ds = bar_s + 8u;
    const uint32_t bar_acc = bar_s + 16u;
    const uint32_t bar_dr = bar_s + 24u;
    const uint32_t bar_dp = bar_s + 32u;
    const uint32_t bar_sfree = bar_s + 40u;
    auto bar_lf = [&](int b) { return bar_s + 48u + 8u * b; };
    auto bar_le = [&](int b) { return bar_s + 64u + 8u * b; };
    const uint32_t* list = reinterpret_cast<const uint32_t*>(smem + C::OFF_LIST);
    // [0] tmem, [1] abort, [2..3] list lengths, [4..5] item of each list buffer (-1: no more)
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_cta = misc + 1;
    volatile int* list_len = misc + 2;
    volatile int* list_item = misc + 4;

    if (threadIdx.x == 0) {
        mbar_init(bar_qd, 1);
        mbar_init(bar_qe, 1);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_vf(s), 1);
            mbar_init(bar_ke(s), 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_ds, 256);
        mbar_init(bar_acc, 1);
        mbar_init(bar_dr, 1);
        mbar_init(bar_dp, 1);
        mbar_init(bar_sfree, 256);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_lf(b), 1);
            mbar_init(bar_le(b), C::LIST_CONSUMERS);
        }
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
        // ------------------------------------------------------------ items, union lists, Q and dO
        if (lane == 0) {
            int k = 0;
            uint32_t* wlist = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
            int w = blockIdx.x;  // first item static, the rest from the work counter
            for (;; ++k) {
                const int b = k & 1;
                // list buffer b is free once item k-2 is consumed
                if (!mbar_wait(bar_le(b), ((k >> 1) & 1) ^ 1, ctl)) break;
                if (w >= num_items) {  // tell every role there is no more work
                    list_item[b] = -1;
                    list_len[b] = 0;
                    mbar_arrive(bar_lf(b));
                    break;
                }
                const int w_next = misc[6] ? (int)gridDim.x + sched_take(p.sched) : num_items;
                const int qt = item_qt(w), bh = item_bh(w), h = bh % p.heads;
                UnionWalk<C::ROWS> it;
                int len = 0;
                const bool ok = it.init(p.row_ptr, h * (p.nb + 1), qt * C::ROWS, p.nb, p.nnz);
                if (it.any) {
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
                list_len[b] = len;
                list_item[b] = w;
                mbar_arrive(bar_lf(b));
                // Q and dO of the tile, once the previous item's copies into TMEM are done
                if (!mbar_wait(bar_qe, (k & 1) ^ 1, ctl)) break;
                mbar_arrive_expect_tx(bar_qd, 2 * C::TBYTES);
#pragma unroll
                for (int pn = 0; pn < HD / 64; ++pn) {
                    tma_load_3d(sb + C::OFF_Q + pn * (C::M * 128), &tmQ, pn * 64, qt * C::M, bh, bar_qd);
                    tma_load_3d(sb + C::OFF_DO + pn * (C::M * 128), &tmDO, pn * 64, qt * C::M, bh, bar_qd);
                }
                w = w_next;
            }
            if (*abort_cta && k > 0) mbar_drain(bar_qd, (k - 1) & 1, kDrainNs);
        }
        __syncwarp();
    } else if (warp == 0) {
        // ------------------------------------------------------------ K and V producer
        if (lane == 0) {
            int n = 0, k = 0;
            bool stop = false;
            for (; !stop; ++k) {
                const int b = k & 1;
                if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                const int w = list_item[b];
                if (w < 0) break;
                const int bh = item_bh(w);
                const int bkv = (bh / p.heads) * p.heads_kv + (bh % p.heads) / (p.heads / p.heads_kv);
                const uint32_t* L = list + b * C::LIST_CAP;
                const int len = list_len[b];
                const int nel = (len + C::KPE - 1) / C::KPE;
                for (int e = 0; e < nel; ++e, ++n) {
                    const int st = n % C::ST;
                    if (!mbar_wait(bar_ke(st), ((n / C::ST) & 1) ^ 1, ctl)) {
                        stop = true;
                        break;
                    }
                    // entry h of the element into rows h*BK.. of the stage (a pad loads
                    // the first entry's block again: finite data, masked)
                    mbar_arrive_expect_tx(bar_kf(st), C::KVBYTES);
#pragma unroll
                    for (int h = 0; h < C::KPE; ++h) {
                        const int ei = e * C::KPE + h;
                        const int32_t krow = list_j(L[ei < len ? ei : e * C::KPE]) * BK;
#pragma unroll
                        for (int pn = 0; pn < HD / 64; ++pn)
                            tma_load_3d(sb + C::OFF_K + st * C::KVBYTES + pn * (C::NK * 128) + h * (BK * 128), &tmK,
                                        pn * 64, krow, bkv, bar_kf(st));
                    }
                    mbar_arrive_expect_tx(bar_vf(st), C::KVBYTES);
#pragma unroll
                    for (int h = 0; h < C::KPE; ++h) {
                        const int ei = e * C::KPE + h;
                        const int32_t krow = list_j(L[ei < len ? ei : e * C::KPE]) * BK;
#pragma unroll
                        for (int pn = 0; pn < HD / 64; ++pn)
                            tma_load_3d(sb + C::OFF_V + st * C::KVBYTES + pn * (C::NK * 128) + h * (BK * 128), &tmV,
                                        pn * 64, krow, bkv, bar_vf(st));
                    }
                }
                if (!stop) mbar_arrive(bar_le(b));
            }
            if (*abort_cta)  // let this CTA's own loads land before exit
                for (int m = (n > C::ST ? n - C::ST : 0); m < n; ++m) {
                    mbar_drain(bar_kf(m % C::ST), (m / C::ST) & 1, kDrainNs);
                    mbar_drain(bar_vf(m % C::ST), (m / C::ST) & 1, kDrainNs);
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc(128, C::NK, 0, 0);  // S = Q K^T, dP = dO V^T
            constexpr uint32_t idesc_q = umma_idesc(128, HD, 0, 1);     // dQ += dS K (K as MN-major B)
            const uint64_t dq_desc = umma_sdesc(sb + C::OFF_Q, 16, 1024);
            const uint64_t ddo_desc = umma_sdesc(sb + C::OFF_DO, 16, 1024);
            bool issued = false, fail = false;
            // Element G (counted over all items) uses stage G % ST; S(G) and dP(G)
            // are committed separately so that the element-wise warps start on P
            // while dP is still running. Order per element: [S(G) read out]
            // S(G+1); [dS(G) ready] dQ(G), dP(G+1). The warps keep P in
            // registers, so S(G+1) may overwrite S(G) as soon as they have
            // loaded it; dS(G) sits in dP's columns and dP(G+1) is issued after
            // dQ(G) has read it.
            auto issue_s = [&](int G) {
                const int st = G % C::ST;
                if (!mbar_wait(bar_kf(st), (G / C::ST) & 1, ctl)) return false;
                tc_fence_after();
                const uint64_t dk_desc = umma_sdesc(sb + C::OFF_K + st * C::KVBYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    umma_bf16_ts(tmem + C::COL_S, tmem + C::COL_QA + kk * 8, dk_desc + kstep(kk, C::NK), idesc_s,
                                 kk > 0 ? 1u : 0u);
                umma_commit(bar_s);
                issued = true;
                return true;
            };
            auto issue_dp = [&](int G) {
                const int st = G % C::ST;
                if (!mbar_wait(bar_vf(st), (G / C::ST) & 1, ctl)) return false;
                tc_fence_after();
                const uint64_t dv_desc = umma_sdesc(sb + C::OFF_V + st * C::KVBYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    umma_bf16_ts(tmem + C::COL_DP, tmem + C::COL_DOA + kk * 8, dv_desc + kstep(kk, C::NK),
                                 idesc_s, kk > 0 ? 1u : 0u);
                umma_commit(bar_dp);
                return true;
            };
            int G = 0;
            for (int k = 0; !fail; ++k) {
                const int b = k & 1;
                if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                if (list_item[b] < 0) break;
                const int len = (list_len[b] + C::KPE - 1) / C::KPE;  // elements
                if (!mbar_wait(bar_qd, k & 1, ctl)) break;
                // Q and dO into TMEM (after the previous item's MMAs that read them,
                // in issue order); the shared-memory buffers are then free.
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    tmem_cp_128x256b(tmem + C::COL_QA + kk * 8, dq_desc + kstep(kk, C::M));
                    tmem_cp_128x256b(tmem + C::COL_DOA + kk * 8, ddo_desc + kstep(kk, C::M));
                }
                umma_commit(bar_qe);
                issued = true;
                if (len > 0) {
                    // S's columns are free once the warps have loaded S of the previous
                    // element; dP's (its dS) were read by its dQ, issued before.
                    if (G > 0 && !mbar_wait(bar_sfree, (G - 1) & 1, ctl)) break;
                    tc_fence_after();
                    if (!issue_s(G) || !issue_dp(G)) break;
                    for (int n = 0; n < len; ++n, ++G) {
                        const int st = G % C::ST;
                        const bool more = n + 1 < len;
                        if (more) {
                            if (!mbar_wait(bar_sfree, G & 1, ctl)) {
                                fail = true;
                                break;
                            }
                            tc_fence_after();
                            if (!issue_s(G + 1)) {
                                fail = true;
                                break;
                            }
                        }
                        if (!mbar_wait(bar_ds, G & 1, ctl)) {
                            fail = true;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < C::NK / 16; ++kk) {
                            const uint64_t bk =
                                umma_sdesc(sb + C::OFF_K + st * C::KVBYTES + kk * 2048, C::NK * 128, 1024);
                            umma_bf16_ts(tmem + C::COL_ACC, tmem + C::COL_DP + packed_col<C::NK>(kk), bk, idesc_q,
                                         (n > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(bar_ke(st));
                        if (more && !issue_dp(G + 1)) {
                            fail = true;
                            break;
                        }
                    }
                    if (fail) break;
                    umma_commit(bar_acc);  // dQ of this item is complete once its last MMA is
                }
                mbar_arrive(bar_le(b));
            }
            if (*abort_cta && issued) {
                umma_commit(bar_dr);
                mbar_drain(bar_dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ element-wise passes + epilogue
        constexpr int HALF = C::NK / 2;  // key columns per warpgroup (one entry's block when paired)
        const int quad = warp & 3, g = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const float sc = p.scale_log2;
        const int rowbit = (BK == 128) ? 0 : (r >> 6);
        bool fail = false;
        int G = 0, n_acc = 0;  // elements, and items with a dQ accumulation, so far
        for (int k = 0; !fail; ++k) {
            const int b = k & 1;
            if (!warp_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
            const int w = list_item[b];
            if (w < 0) break;
            const int qt = item_qt(w), bh = item_bh(w);
            const int qpos = qt * C::M + r;
            const bool row_valid = qpos < p.seq;
            float lx = 0.f, dy = 0.f;  // this row's LSE * log2 e and D
            if (row_valid) {
                const float* sp = p.stats + ((int64_t)bh * p.ntiles + qt) * 256 + r;
                lx = sp[0];
                dy = sp[128];
            }
            const uint32_t* L = list + b * C::LIST_CAP;
            const int nent = list_len[b];
            const int len = (nent + C::KPE - 1) / C::KPE;  // elements
            for (int n = 0; n < len; ++n, ++G) {
                // this warpgroup's entry: the element's block (128-key blocks), or
                // entry g of the pair (64-key blocks; past the list: a masked pad)
                const int ei = n * C::KPE + (C::KPE == 2 ? g : 0);
                const uint32_t ent = ei < nent ? L[ei] : 0u;
                if (!warp_wait(bar_s, G & 1, ctl)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                const bool vis = row_valid && ((list_bits(ent) >> rowbit) & 1);
                // column c of this half visible iff c <= lim
                const int lim = qpos - list_j(ent) * BK - (C::KPE == 2 ? 0 : g * HALF);
                // P pass (needs S only; dP may still be running): P as bf16 pairs in registers
                uint32_t sr[HALF], pk[HALF / 2];
                tmem_ld_cols<HALF>(tl + C::COL_S + g * HALF, sr);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar_sfree);  // S(G) is in registers: S(G+1) may be written
#pragma unroll
                for (int c = 0; c < HALF; c += 2) {
                    const float p0 = (vis && c <= lim) ? ex2(fmaf(__uint_as_float(sr[c]), sc, -lx)) : 0.f;
                    const float p1 = (vis && c + 1 <= lim) ? ex2(fmaf(__uint_as_float(sr[c + 1]), sc, -lx)) : 0.f;
                    pk[c / 2] = pack_bf16x2(p0, p1);
                }
                if (!warp_wait(bar_dp, G & 1, ctl)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                // dS pass: dS = P (dP - D), bf16 pairs over the first HALF/2 columns
                // of this half of dP (already read)
                tmem_ld_cols<HALF>(tl + C::COL_DP + g * HALF, sr);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < HALF; c += 2) {
                    const float d0 = bf16lo(pk[c / 2]) * (__uint_as_float(sr[c]) - dy);
                    const float d1 = bf16hi(pk[c / 2]) * (__uint_as_float(sr[c + 1]) - dy);
                    pk[c / 2] = pack_bf16x2(d0, d1);
                }
                tmem_st_cols<HALF / 2>(tl + C::COL_DP + g * HALF, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_ds);
            }
            if (fail) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_le(b));
            // warpgroup g stores output columns g * HD/2 .. (g + 1) * HD/2 - 1; the
            // next item's first dQ MMA (which overwrites the accumulator) waits
            // for this warpgroup's first dS of that item, so it follows these loads
            uint16_t* drow = p.dq + ((int64_t)bh * p.seq + qpos) * HD + g * (HD / 2);
            if (len > 0) {
                if (!warp_wait(bar_acc, (n_acc++) & 1, ctl)) break;
                tc_fence_after();
                // HD/2 columns per warpgroup, 32 per TMEM load, one wait
                const bool st32 = (reinterpret_cast<uintptr_t>(p.dq) & 31u) == 0;
                uint32_t o[HD / 2];
#pragma unroll
                for (int c = 0; c < HD / 64; ++c)
                    tmem_ld32(tl + C::COL_ACC + g * (HD / 2) + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&o[32 * c]));
                tmem_wait_ld();
                if (row_valid) store_bf16_row<HD / 2>(drow, o, p.scale, st32);
            } else if (row_valid) {  // no key block listed for this tile
                for (int d = 0; d < HD / 2; d += 8) *reinterpret_cast<uint4*>(drow + d) = make_uint4(0, 0, 0, 0);
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

// ------------------------------------------------------------------ dK, dV

template <int HD, int BK>
struct BwdKVCfg {
    static_assert(BK == 128, "64-key blocks use s2_bwd_dkv_persistent_kernel");
    static constexpr int M = 128;                      // one key block per tile
    static constexpr uint32_t TBYTES = M * HD * 2;     // K or V tile
    static constexpr uint32_t QBYTES = BK * HD * 2;    // one query block of Q or dO
    static constexpr uint32_t STATBYTES = BK * 8;      // L2 of the BK queries, then their D
    static constexpr int ST = 2;
    static constexpr int LIST_CAP = 4096;  // grouped heads: the lists of every query head of the group
    static constexpr uint32_t OFF_K = 0;
    static constexpr uint32_t OFF_V = TBYTES;
    static constexpr uint32_t OFF_Q = 2 * TBYTES;              // [stage][panel][BK rows x 128 B]
    static constexpr uint32_t OFF_DO = OFF_Q + ST * QBYTES;
    static constexpr uint32_t OFF_STAT = OFF_DO + ST * QBYTES;
    static constexpr uint32_t OFF_LIST = OFF_STAT + ST * STATBYTES;
    static constexpr uint32_t OFF_BAR = OFF_LIST + LIST_CAP * 4;
    // barriers: kv_full, q_full[ST], q_empty[ST], s_full, p_full, acc_done, drain, dp_full, ds_full
    static constexpr int NBAR = 1 + 2 * ST + 6;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 32;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    static constexpr uint32_t COL_S = 0, COL_DP = BK, COL_DV = 2 * BK, COL_DK = 2 * BK + HD;
    // When TMEM has room (head_dim 64), K and V, the A operands of every S^T
    // and dP^T MMA of the CTA, sit in TMEM (HD/2 columns each).
    static constexpr bool A_IN_TMEM = 2 * BK + 3 * HD <= 512;
    static constexpr uint32_t COL_KA = 2 * BK + 2 * HD, COL_VA = 2 * BK + 2 * HD + HD / 2;
    static constexpr uint32_t TMEM_COLS = (2 * BK + 2 * HD + (A_IN_TMEM ? HD : 0)) <= 256 ? 256 : 512;
    static_assert(2 * BK + 2 * HD <= 512, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// One key tile per CTA; launched for 128-key blocks (64-key blocks use the
// persistent kernel below).
template <int HD, int BK>
__global__ void __launch_bounds__(384, 1)
s2_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const BackwardParams p)
{
    using C = BwdKVCfg<HD, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // One key tile of one K/V plane; with grouped heads the tile collects the
    // gradients of every query head of its group (list entries carry the head).
    const int BHk = p.batch * p.heads_kv;
    const int kt = (int)(blockIdx.x / BHk);
    const int bkv = (int)(blockIdx.x % BHk);
    const int grp = p.heads / p.heads_kv;
    const int h = (bkv % p.heads_kv) * grp;         // first query head of the group
    const int bq0 = (bkv / p.heads_kv) * p.heads + h;  // its (batch, head) plane
    int kb[1] = {kt};  // the tile's key block

    const uint32_t bar_kv = sb + C::OFF_BAR;
    auto bar_qf = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + s); };
    auto bar_qe = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + C::ST + s); };
    const uint32_t bar_s = sb + C::OFF_BAR + 8u * (1 + 2 * C::ST);
    const uint32_t bar_p = bar_s + 8u;
    const uint32_t bar_acc = bar_s + 16u;
    const uint32_t bar_dr = bar_s + 24u;
    const uint32_t bar_dp = bar_s + 32u;
    const uint32_t bar_ds = bar_s + 40u;
    uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);  // [0] tmem, [1] abort, [2] list length
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_cta = misc + 1;

    if (threadIdx.x == 0) {
        mbar_init(bar_dp, 1);
        mbar_init(bar_ds, 256);
        mbar_init(bar_kv, 1);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_qf(s), 1);
            mbar_init(bar_qe(s), 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_acc, 1);
        mbar_init(bar_dr, 1);
        *abort_cta = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {  // K and V of the tile do not depend on the list: load them now
        mbar_arrive_expect_tx(bar_kv, 2 * C::TBYTES);
        const int32_t krow = kt * BK;
#pragma unroll
        for (int pn = 0; pn < HD / 64; ++pn) {
            tma_load_3d(sb + C::OFF_K + pn * (C::M * 128), &tmK, pn * 64, krow, bkv, bar_kv);
            tma_load_3d(sb + C::OFF_V + pn * (C::M * 128), &tmV, pn * 64, krow, bkv, bar_kv);
        }
    }
    if (warp == 2) {  // the tile's key block's query-block lists
        int total = 0;
        for (int hh = 0; hh < grp; ++hh) {  // the group's query heads, one list after another
            const int n = warp_union_list<1>(p.col_ptr, p.row_idx, (h + hh) * (p.nb + 1), kb, p.nb, p.nnz, kt,
                                             p.nb - 1, list + total, C::LIST_CAP - total, nullptr, p.gflags);
            for (int t = lane; t < n; t += 32) list[total + t] |= (uint32_t)hh << 28;
            __syncwarp();
            total += n;
        }
        if (lane == 0) misc[2] = total;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int len = misc[2];
    const WaitCtl ctl{p.timeout_ns, p.gflags, abort_cta};
    constexpr uint64_t kDrainNs = 200000000ull;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && len == 0) mbar_drain(bar_kv, 0, kDrainNs);  // nothing to do: let K, V land
        if (lane == 0 && len > 0) {
            int n = 0;
            for (; n < len; ++n) {
                const int st = n % C::ST;
                if (!mbar_wait(bar_qe(st), ((n / C::ST) & 1) ^ 1, ctl)) break;
                const int i = list_j(list[n]);
                const int bq = bq0 + (int)(list[n] >> 28);  // query plane of this entry
                mbar_arrive_expect_tx(bar_qf(st), 2 * C::QBYTES + C::STATBYTES);
#pragma unroll
                for (int pn = 0; pn < HD / 64; ++pn) {
                    tma_load_3d(sb + C::OFF_Q + st * C::QBYTES + pn * (BK * 128), &tmQ, pn * 64, i * BK,
                                bq, bar_qf(st));
                    tma_load_3d(sb + C::OFF_DO + st * C::QBYTES + pn * (BK * 128), &tmDO, pn * 64, i * BK,
                                bq, bar_qf(st));
                }
                const float* sx = p.stats + ((int64_t)bq * p.ntiles + (i * BK) / 128) * 256 + (i * BK) % 128;
                bulk_load(sb + C::OFF_STAT + st * C::STATBYTES, sx, BK * 4, bar_qf(st));
                bulk_load(sb + C::OFF_STAT + st * C::STATBYTES + BK * 4, sx + 128, BK * 4, bar_qf(st));
            }
            if (*abort_cta) {
                mbar_drain(bar_kv, 0, kDrainNs);
                for (int m = (n > C::ST ? n - C::ST : 0); m < n; ++m)
                    mbar_drain(bar_qf(m % C::ST), (m / C::ST) & 1, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && len > 0) {
            constexpr uint32_t idesc_s = umma_idesc(128, BK, 0, 0);   // S^T = K Q^T, dP^T = V dO^T
            constexpr uint32_t idesc_a = umma_idesc(128, HD, 0, 1);   // dV += P^T dO, dK += dS^T Q
            const uint64_t dk_desc = umma_sdesc(sb + C::OFF_K, 16, 1024);
            const uint64_t dv_desc = umma_sdesc(sb + C::OFF_V, 16, 1024);
            bool issued = false;
            // S^T(n) and dP^T(n) are committed separately so that the element-wise
            // warps compute P^T while dP^T is still running. Order per element n:
            // [P^T(n) ready] dV(n), S^T(n+1); [dS^T(n) ready] dK(n), dP^T(n+1).
            // S^T(n+1) overwrites P^T(n) after dV(n) has read it (MMAs of one
            // thread run in issue order; the warps keep P in registers for the
            // dS pass); dP^T(n+1) overwrites dS^T(n) after dK(n).
            auto issue_st = [&](int n) {
                const int st = n % C::ST;
                if (!mbar_wait(bar_qf(st), (n / C::ST) & 1, ctl)) return false;
                tc_fence_after();
                const uint64_t dq_desc = umma_sdesc(sb + C::OFF_Q + st * C::QBYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    if constexpr (C::A_IN_TMEM)
                        umma_bf16_ts(tmem + C::COL_S, tmem + C::COL_KA + kk * 8, dq_desc + kstep(kk, BK), idesc_s,
                                     kk > 0 ? 1u : 0u);
                    else
                        umma_bf16_ss(tmem + C::COL_S, dk_desc + kstep(kk, C::M), dq_desc + kstep(kk, BK), idesc_s,
                                     kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_s);
                issued = true;
                return true;
            };
            auto issue_dpt = [&](int n) {  // stage already waited for by issue_st(n)
                const int st = n % C::ST;
                const uint64_t ddo_desc = umma_sdesc(sb + C::OFF_DO + st * C::QBYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    if constexpr (C::A_IN_TMEM)
                        umma_bf16_ts(tmem + C::COL_DP, tmem + C::COL_VA + kk * 8, ddo_desc + kstep(kk, BK),
                                     idesc_s, kk > 0 ? 1u : 0u);
                    else
                        umma_bf16_ss(tmem + C::COL_DP, dv_desc + kstep(kk, C::M), ddo_desc + kstep(kk, BK),
                                     idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_dp);
            };
            const bool kv_ok = mbar_wait(bar_kv, 0, ctl);
            if (kv_ok && C::A_IN_TMEM) {  // K and V into TMEM, before every MMA that reads them
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    tmem_cp_128x256b(tmem + C::COL_KA + kk * 8, dk_desc + kstep(kk, C::M));
                    tmem_cp_128x256b(tmem + C::COL_VA + kk * 8, dv_desc + kstep(kk, C::M));
                }
                issued = true;
            }
            if (kv_ok && issue_st(0)) {
                issue_dpt(0);
                for (int n = 0; n < len; ++n) {
                    const int st = n % C::ST;
                    const bool more = n + 1 < len;
                    if (!mbar_wait(bar_p, n & 1, ctl)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t bdo = umma_sdesc(sb + C::OFF_DO + st * C::QBYTES + kk * 2048, BK * 128, 1024);
                        umma_bf16_ts(tmem + C::COL_DV, tmem + C::COL_S + packed_col<BK>(kk), bdo, idesc_a,
                                     (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (more && !issue_st(n + 1)) break;
                    if (!mbar_wait(bar_ds, n & 1, ctl)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t bq = umma_sdesc(sb + C::OFF_Q + st * C::QBYTES + kk * 2048, BK * 128, 1024);
                        umma_bf16_ts(tmem + C::COL_DK, tmem + C::COL_DP + packed_col<BK>(kk), bq, idesc_a,
                                     (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_qe(st));
                    if (more) issue_dpt(n + 1);
                }
                if (!*abort_cta) umma_commit(bar_acc);
            }
            if (*abort_cta && issued) {
                umma_commit(bar_dr);
                mbar_drain(bar_dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ element-wise passes + epilogue
        constexpr int HALF = BK / 2;  // query columns per warpgroup
        const int quad = warp & 3, g = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int kbit = 0;  // the list entries' row tag of the tile's one key block
        const int kpos = kt * BK + r;
        const bool row_valid = kpos < p.seq;
        const float sc = p.scale_log2;
        bool fail = false;
        for (int n = 0; n < len; ++n) {
            const int st = n % C::ST;
            const uint32_t ent = list[n];
            // the stage's query statistics came by bulk copy: observe its barrier
            // too (already complete: the MMAs of this element waited for it)
            if (!warp_wait(bar_qf(st), (n / C::ST) & 1, ctl) || !warp_wait(bar_s, n & 1, ctl)) {
                fail = true;
                break;
            }
            tc_fence_after();
            const float* sx = reinterpret_cast<const float*>(smem + C::OFF_STAT + st * C::STATBYTES) + g * HALF;
            const float* sy = sx + BK;
            const bool vis = row_valid && ((list_bits(ent) >> kbit) & 1);
            const int lim = kpos - list_j(ent) * BK - g * HALF;  // column c of this half visible iff c >= lim
            // P pass (needs S^T only): P^T as bf16 pairs over the first HALF/2
            // columns of this half of S^T (already read), kept in registers too
            uint32_t sr[HALF], pk[HALF / 2];
            tmem_ld_cols<HALF>(tl + C::COL_S + g * HALF, sr);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < HALF; c += 4) {
                const float4 x = *reinterpret_cast<const float4*>(sx + c);
                const float p0 = (vis && c >= lim) ? ex2(fmaf(__uint_as_float(sr[c]), sc, -x.x)) : 0.f;
                const float p1 = (vis && c + 1 >= lim) ? ex2(fmaf(__uint_as_float(sr[c + 1]), sc, -x.y)) : 0.f;
                const float p2 = (vis && c + 2 >= lim) ? ex2(fmaf(__uint_as_float(sr[c + 2]), sc, -x.z)) : 0.f;
                const float p3 = (vis && c + 3 >= lim) ? ex2(fmaf(__uint_as_float(sr[c + 3]), sc, -x.w)) : 0.f;
                pk[c / 2] = pack_bf16x2(p0, p1);
                pk[c / 2 + 1] = pack_bf16x2(p2, p3);
            }
            tmem_st_cols<HALF / 2>(tl + C::COL_S + g * HALF, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p);
            if (!warp_wait(bar_dp, n & 1, ctl)) {
                fail = true;
                break;
            }
            tc_fence_after();
            // dS pass: dS^T = P^T (dP^T - D) over the first HALF/2 columns of this half of dP^T
            tmem_ld_cols<HALF>(tl + C::COL_DP + g * HALF, sr);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < HALF; c += 4) {
                const float4 y = *reinterpret_cast<const float4*>(sy + c);
                const float d0 = bf16lo(pk[c / 2]) * (__uint_as_float(sr[c]) - y.x);
                const float d1 = bf16hi(pk[c / 2]) * (__uint_as_float(sr[c + 1]) - y.y);
                const float d2 = bf16lo(pk[c / 2 + 1]) * (__uint_as_float(sr[c + 2]) - y.z);
                const float d3 = bf16hi(pk[c / 2 + 1]) * (__uint_as_float(sr[c + 3]) - y.w);
                pk[c / 2] = pack_bf16x2(d0, d1);
                pk[c / 2 + 1] = pack_bf16x2(d2, d3);
            }
            tmem_st_cols<HALF / 2>(tl + C::COL_DP + g * HALF, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_ds);
        }
        if (!fail) {
            // warpgroup 0 stores dV, warpgroup 1 stores dK (times the scale)
            const int64_t row = (int64_t)bkv * p.seq + kpos;
            uint16_t* grow = (g == 0 ? p.dv : p.dk) + row * HD;
            if (len > 0) {
                if (warp_wait(bar_acc, 0, ctl)) {
                    tc_fence_after();
                    const float f = g == 0 ? 1.0f : p.scale;
                    const uint32_t col = g == 0 ? C::COL_DV : C::COL_DK;
                    const bool st32 = (reinterpret_cast<uintptr_t>(g == 0 ? p.dv : p.dk) & 31u) == 0;
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tl + col + 32 * c, o);
                        tmem_wait_ld();
                        if (row_valid) store_bf16_row<32>(grow + 32 * c, o, f, st32);
                    }
                }
            } else if (row_valid) {  // no query block lists this tile's key blocks
                for (int d = 0; d < HD; d += 8) *reinterpret_cast<uint4*>(grow + d) = make_uint4(0, 0, 0, 0);
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ dK, dV (persistent, B = 64)

// 64-key blocks: each CTA takes work items (one 128-row key tile = two 64-key
// blocks of one K/V plane, in the order above: key tiles outermost, so the
// tiles seen by the most query blocks come first) from a device counter.
// K and V are only the A operands of S^T and dP^T, and sit in TMEM, so their
// shared-memory copy is needed only for the tcgen05.cp at the start of an
// item: one buffer suffices, and the next tile's K and V (and its union list,
// double-buffered) load while the current tile runs. Element counters run over
// all items of the CTA, so stages, barrier phases and the S^T/dP^T ->
// dV/dK hand-offs carry across item boundaries unchanged.
template <int HD>
struct BwdKVPCfg {
    static constexpr int BK = 64;
    static constexpr int M = 128;
    static constexpr int ROWS = 2;                     // key blocks per tile
    static constexpr uint32_t TBYTES = M * HD * 2;     // K or V tile
    static constexpr uint32_t QBYTES = BK * HD * 2;    // one query block of Q or dO
    static constexpr uint32_t STATBYTES = BK * 8;      // L2 of the BK queries, then their D
    static constexpr int ST = 2;
    static constexpr int LIST_CAP = 4096;  // grouped heads: the lists of every query head of the group
    static constexpr uint32_t OFF_K = 0;
    static constexpr uint32_t OFF_V = TBYTES;
    static constexpr uint32_t OFF_Q = 2 * TBYTES;              // [stage][panel][BK rows x 128 B]
    static constexpr uint32_t OFF_DO = OFF_Q + ST * QBYTES;
    static constexpr uint32_t OFF_STAT = OFF_DO + ST * QBYTES;
    static constexpr uint32_t OFF_LIST = OFF_STAT + ST * STATBYTES;  // two list buffers
    static constexpr uint32_t OFF_SCR = OFF_LIST + 2 * LIST_CAP * 4;  // list-merge scratch
    static constexpr uint32_t OFF_BAR = OFF_SCR + ROWS * LIST_CAP * 4;
    // barriers: kv_full, kv_empty, q_full[ST], q_empty[ST], s_full, p_full, acc_done, dp_full,
    // ds_full, drain x 2, list_full[2], list_empty[2]
    static constexpr int NBAR = 2 + 2 * ST + 7 + 4;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 48;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    // Q/dO producer, the two MMA threads, 8 element-wise warps
    static constexpr uint32_t LIST_CONSUMERS = 11;
    static constexpr uint32_t COL_S = 0, COL_DP = BK, COL_DV = 2 * BK, COL_DK = 2 * BK + HD;
    static constexpr uint32_t COL_KA = 2 * BK + 2 * HD, COL_VA = 2 * BK + 2 * HD + HD / 2;
    static constexpr uint32_t TMEM_COLS = (2 * BK + 3 * HD) <= 256 ? 256 : 512;
    static_assert(2 * BK + 3 * HD <= 512, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Work item w of the dK/dV kernels: key tile kt of K/V plane bkv, the first
// query head h of its group and that head's (batch, head) plane.
struct KvItem {
    int kt, bkv, h, bq0;
};

__device__ __forceinline__ KvItem kv_item(const BackwardParams& p, int w)
{
    const int BHk = p.batch * p.heads_kv, grp = p.heads / p.heads_kv;
    KvItem it;
    it.kt = w / BHk;
    it.bkv = w % BHk;
    it.h = (it.bkv % p.heads_kv) * grp;
    it.bq0 = (it.bkv / p.heads_kv) * p.heads + it.h;
    return it;
}

// Key block r (0 or 1) of a 64-key tile, -1 if none.
__device__ __forceinline__ int kv_item_block(const BackwardParams& p, const KvItem& it, int r)
{
    const int j = __ldg(p.key_tiles + ((int64_t)it.h * p.ntiles + it.kt) * 2 + r);
    return j < p.nb ? j : -1;
}

template <int HD>
__global__ void __launch_bounds__(384, 1)
s2_bwd_dkv_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                             const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                             const BackwardParams p)
{
    using C = BwdKVPCfg<HD>;
    constexpr int BK = C::BK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_items = p.ntiles * p.batch * p.heads_kv;
    const int grp = p.heads / p.heads_kv;

    const uint32_t bar_kv = sb + C::OFF_BAR;
    const uint32_t bar_kve = bar_kv + 8u;  // K and V copied into TMEM (one commit each): refill
    auto bar_qf = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + s); };
    auto bar_qe = [&](int s) { return sb + C::OFF_BAR + 8u * (2 + C::ST + s); };
    const uint32_t bar_s = sb + C::OFF_BAR + 8u * (2 + 2 * C::ST);
    const uint32_t bar_p = bar_s + 8u;
    const uint32_t bar_acc = bar_s + 16u;
    const uint32_t bar_dp = bar_s + 24u;
    const uint32_t bar_ds = bar_s + 32u;
    const uint32_t bar_dr = bar_s + 40u;
    const uint32_t bar_dr2 = bar_s + 48u;
    auto bar_lf = [&](int b) { return bar_s + 56u + 8u * b; };
    auto bar_le = [&](int b) { return bar_s + 72u + 8u * b; };
    const uint32_t* list = reinterpret_cast<const uint32_t*>(smem + C::OFF_LIST);
    // [0] tmem, [1] abort, [2..3] list lengths, [4..5] item of each list buffer (-1: no more),
    // [6] this CTA holds the work-counter slot, [8..11] the key blocks of each buffer's tile
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_cta = misc + 1;
    volatile int* list_len = misc + 2;
    volatile int* list_item = misc + 4;
    volatile int* list_kb = misc + 8;  // [buffer][key block r of the tile] (-1: none)

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        mbar_init(bar_kve, 2);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_qf(s), 1);
            mbar_init(bar_qe(s), 2);  // one commit from each MMA thread
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_acc, 2);
        mbar_init(bar_dp, 1);
        mbar_init(bar_ds, 256);
        mbar_init(bar_dr, 1);
        mbar_init(bar_dr2, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_lf(b), 1);
            mbar_init(bar_le(b), C::LIST_CONSUMERS);
        }
        *abort_cta = 0;
        misc[6] = sched_claim(p.sched_kv, p.sched_kv_id, WaitCtl{p.timeout_ns, p.gflags, abort_cta});
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
        // ------------------------------------------------------------ items, union lists, K and V
        uint32_t* wlist = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
        int32_t* scratch = reinterpret_cast<int32_t*>(smem + C::OFF_SCR);
        int w = blockIdx.x;  // first item static, the rest from the work counter
        int m = 0;           // K/V loads issued (items with a non-empty list)
        for (int k = 0;; ++k) {
            const int b = k & 1;
            // list buffer b is free once item k-2 is consumed
            if (!warp_wait(bar_le(b), ((k >> 1) & 1) ^ 1, ctl)) break;
            if (w >= num_items) {  // tell every role there is no more work
                if (lane == 0) {
                    list_item[b] = -1;
                    list_len[b] = 0;
                    mbar_arrive(bar_lf(b));
                }
                break;
            }
            int w_next = 0;
            if (lane == 0) w_next = misc[6] ? (int)gridDim.x + sched_take(p.sched_kv) : num_items;
            w_next = __shfl_sync(0xffffffffu, w_next, 0);
            const KvItem it = kv_item(p, w);
            int kb[C::ROWS];
            int lo = INT_MAX;
#pragma unroll
            for (int r = 0; r < C::ROWS; ++r) {
                kb[r] = kv_item_block(p, it, r);
                if (kb[r] >= 0 && kb[r] < lo) lo = kb[r];
            }
            uint32_t* L = wlist + b * C::LIST_CAP;
            int total = 0;
            for (int hh = 0; hh < grp; ++hh) {  // the group's query heads, one list after another
                const int n = warp_union_list<C::ROWS>(p.col_ptr, p.row_idx, (it.h + hh) * (p.nb + 1), kb, p.nb,
                                                       p.nnz, lo, p.nb - 1, L + total, C::LIST_CAP - total,
                                                       scratch, p.gflags);
                for (int t = lane; t < n; t += 32) L[total + t] |= (uint32_t)hh << 28;
                __syncwarp();
                total += n;
            }
            if (lane == 0) {
                list_len[b] = total;
                list_item[b] = w;
#pragma unroll
                for (int r = 0; r < C::ROWS; ++r) list_kb[2 * b + r] = kb[r];
                mbar_arrive(bar_lf(b));
            }
            if (total > 0) {
                // K and V of the tile, once the previous tile's copies into TMEM are done
                if (!warp_wait(bar_kve, (m & 1) ^ 1, ctl)) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar_kv, 2 * C::TBYTES);
                    const int kany = kb[0] >= 0 ? kb[0] : kb[1];  // a missing block loads the other's rows
#pragma unroll
                    for (int r = 0; r < C::ROWS; ++r) {
                        const int32_t krow = (kb[r] >= 0 ? kb[r] : kany) * BK;
#pragma unroll
                        for (int pn = 0; pn < HD / 64; ++pn) {
                            tma_load_3d(sb + C::OFF_K + pn * (C::M * 128) + r * (BK * 128), &tmK, pn * 64, krow,
                                        it.bkv, bar_kv);
                            tma_load_3d(sb + C::OFF_V + pn * (C::M * 128) + r * (BK * 128), &tmV, pn * 64, krow,
                                        it.bkv, bar_kv);
                        }
                    }
                }
                ++m;
            }
            w = w_next;
        }
        if (lane == 0 && *abort_cta && m > 0) mbar_drain(bar_kv, (m - 1) & 1, kDrainNs);
        __syncwarp();
    } else if (warp == 0) {
        // ------------------------------------------------------------ Q, dO and statistics producer
        if (lane == 0) {
            int n = 0;  // elements over all items; element n uses stage n % ST
            bool stop = false;
            for (int k = 0; !stop; ++k) {
                const int b = k & 1;
                if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                const int w = list_item[b];
                if (w < 0) break;
                const int bq0 = kv_item(p, w).bq0;
                const uint32_t* L = list + b * C::LIST_CAP;
                const int len = list_len[b];
                for (int e = 0; e < len; ++e, ++n) {
                    const int st = n % C::ST;
                    if (!mbar_wait(bar_qe(st), ((n / C::ST) & 1) ^ 1, ctl)) {
                        stop = true;
                        break;
                    }
                    const int i = list_j(L[e]);
                    const int bq = bq0 + (int)(L[e] >> 28);  // query plane of this entry
                    mbar_arrive_expect_tx(bar_qf(st), 2 * C::QBYTES + C::STATBYTES);
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn) {
                        tma_load_3d(sb + C::OFF_Q + st * C::QBYTES + pn * (BK * 128), &tmQ, pn * 64, i * BK, bq,
                                    bar_qf(st));
                        tma_load_3d(sb + C::OFF_DO + st * C::QBYTES + pn * (BK * 128), &tmDO, pn * 64, i * BK, bq,
                                    bar_qf(st));
                    }
                    const float* sx = p.stats + ((int64_t)bq * p.ntiles + (i * BK) / 128) * 256 + (i * BK) % 128;
                    bulk_load(sb + C::OFF_STAT + st * C::STATBYTES, sx, BK * 4, bar_qf(st));
                    bulk_load(sb + C::OFF_STAT + st * C::STATBYTES + BK * 4, sx + 128, BK * 4, bar_qf(st));
                }
                if (!stop) mbar_arrive(bar_le(b));
            }
            if (*abort_cta)  // let this CTA's own loads land before exit
                for (int m = (n > C::ST ? n - C::ST : 0); m < n; ++m)
                    mbar_drain(bar_qf(m % C::ST), (m / C::ST) & 1, kDrainNs);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------------------ MMA issuers
        // Thread A (warp 1): K into TMEM, then per element dV(G) += P^T(G) dO
        // followed by S^T(G+1) = K Q^T. Thread B (warp 3): V into TMEM, then
        // dK(G) += dS^T(G) Q followed by dP^T(G+1) = V dO^T. S^T(G+1) overwrites
        // P^T(G) and dP^T(G+1) overwrites dS^T(G), each after the MMA of the same
        // thread that reads it (one thread: issue order), and after the
        // element-wise threads have read S^T(G) / dP^T(G) (they wrote P^T(G) /
        // dS^T(G) before arriving). Both threads read every stage, so a stage is
        // released by one commit from each (after dV(G) and after dK(G)); so are
        // the tile's accumulators (after its last dV and dK) and the shared-memory
        // K/V buffer (after each thread's copy into TMEM). A tile's first dV and
        // dK overwrite the accumulators: their P^T and dS^T come from
        // element-wise threads that have already read the previous tile's out.
        if (lane == 0) {
            const bool tA = warp == 1;
            constexpr uint32_t idesc_s = umma_idesc(128, BK, 0, 0);  // S^T = K Q^T, dP^T = V dO^T
            constexpr uint32_t idesc_a = umma_idesc(128, HD, 0, 1);  // dV += P^T dO, dK += dS^T Q
            const uint64_t a_desc = umma_sdesc(sb + (tA ? C::OFF_K : C::OFF_V), 16, 1024);
            const uint32_t col_a = tA ? C::COL_KA : C::COL_VA;      // K or V in TMEM
            const uint32_t col_x = tA ? C::COL_S : C::COL_DP;       // S^T / P^T or dP^T / dS^T
            const uint32_t col_acc = tA ? C::COL_DV : C::COL_DK;
            const uint32_t off_b = tA ? C::OFF_Q : C::OFF_DO;       // B of S^T / dP^T
            const uint32_t off_b2 = tA ? C::OFF_DO : C::OFF_Q;      // B of dV / dK
            const uint32_t bar_x = tA ? bar_s : bar_dp;             // S^T / dP^T written
            const uint32_t bar_y = tA ? bar_p : bar_ds;             // P^T / dS^T written
            bool issued = false, fail = false;
            int G = 0, m = 0;
            auto issue_x = [&](int g) {  // S^T(g) or dP^T(g)
                const int st = g % C::ST;
                if (!mbar_wait(bar_qf(st), (g / C::ST) & 1, ctl)) return false;
                tc_fence_after();
                const uint64_t b_desc = umma_sdesc(sb + off_b + st * C::QBYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    umma_bf16_ts(tmem + col_x, tmem + col_a + kk * 8, b_desc + kstep(kk, BK), idesc_s,
                                 kk > 0 ? 1u : 0u);
                umma_commit(bar_x);
                return true;
            };
            for (int k = 0; !fail; ++k) {
                const int b = k & 1;
                if (!mbar_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
                if (list_item[b] < 0) break;
                const int len = list_len[b];
                if (len > 0) {
                    if (!mbar_wait(bar_kv, m & 1, ctl)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        tmem_cp_128x256b(tmem + col_a + kk * 8, a_desc + kstep(kk, C::M));
                    umma_commit(bar_kve);
                    issued = true;
                    ++m;
                    if (!issue_x(G)) break;
                }
                for (int n = 0; n < len; ++n, ++G) {
                    const int st = G % C::ST;
                    if (!mbar_wait(bar_y, G & 1, ctl)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t bb = umma_sdesc(sb + off_b2 + st * C::QBYTES + kk * 2048, BK * 128, 1024);
                        umma_bf16_ts(tmem + col_acc, tmem + col_x + packed_col<BK>(kk), bb, idesc_a,
                                     (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_qe(st));
                    if (n + 1 == len) {
                        umma_commit(bar_acc);  // the tile's dV (dK) is complete with it
                    } else if (!issue_x(G + 1)) {
                        fail = true;
                        break;
                    }
                }
                if (fail) break;
                mbar_arrive(bar_le(b));
            }
            if (*abort_cta && issued) {
                const uint32_t dr = tA ? bar_dr : bar_dr2;
                umma_commit(dr);
                mbar_drain(dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ element-wise passes + epilogue
        constexpr int HALF = BK / 2;  // query columns per warpgroup
        const int quad = warp & 3, g = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int kbit = r >> 6;  // key block of this row within the tile
        const float sc = p.scale_log2;
        bool fail = false;
        int G = 0, n_acc = 0;  // elements, and tiles with an accumulation, so far
        for (int k = 0; !fail; ++k) {
            const int b = k & 1;
            if (!warp_wait(bar_lf(b), (k >> 1) & 1, ctl)) break;
            const int w = list_item[b];
            if (w < 0) break;
            const KvItem it = kv_item(p, w);
            const int kbr = list_kb[2 * b + kbit];  // kv_item_block(p, it, kbit), read by the scheduler
            const int kpos = kbr * BK + (r % BK);
            const bool row_valid = kbr >= 0 && kpos < p.seq;
            const uint32_t* L = list + b * C::LIST_CAP;
            const int len = list_len[b];
            for (int n = 0; n < len; ++n, ++G) {
                const int st = G % C::ST;
                const uint32_t ent = L[n];
                // the stage's query statistics came by bulk copy: observe its barrier
                // too (already complete: the MMAs of this element waited for it)
                if (!warp_wait(bar_qf(st), (G / C::ST) & 1, ctl) || !warp_wait(bar_s, G & 1, ctl)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                const float* sx = reinterpret_cast<const float*>(smem + C::OFF_STAT + st * C::STATBYTES) + g * HALF;
                const float* sy = sx + BK;
                const bool vis = row_valid && ((list_bits(ent) >> kbit) & 1);
                const int lim = kpos - list_j(ent) * BK - g * HALF;  // column c of this half visible iff c >= lim
                // P pass (needs S^T only): P^T as bf16 pairs, kept in registers too
                uint32_t sr[HALF], pk[HALF / 2];
                tmem_ld_cols<HALF>(tl + C::COL_S + g * HALF, sr);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < HALF; c += 4) {
                    const float4 x = *reinterpret_cast<const float4*>(sx + c);
                    const float p0 = (vis && c >= lim) ? ex2(fmaf(__uint_as_float(sr[c]), sc, -x.x)) : 0.f;
                    const float p1 = (vis && c + 1 >= lim) ? ex2(fmaf(__uint_as_float(sr[c + 1]), sc, -x.y)) : 0.f;
                    const float p2 = (vis && c + 2 >= lim) ? ex2(fmaf(__uint_as_float(sr[c + 2]), sc, -x.z)) : 0.f;
                    const float p3 = (vis && c + 3 >= lim) ? ex2(fmaf(__uint_as_float(sr[c + 3]), sc, -x.w)) : 0.f;
                    pk[c / 2] = pack_bf16x2(p0, p1);
                    pk[c / 2 + 1] = pack_bf16x2(p2, p3);
                }
                tmem_st_cols<HALF / 2>(tl + C::COL_S + g * HALF, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_p);
                if (!warp_wait(bar_dp, G & 1, ctl)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                // dS pass: dS^T = P^T (dP^T - D)
                tmem_ld_cols<HALF>(tl + C::COL_DP + g * HALF, sr);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < HALF; c += 4) {
                    const float4 y = *reinterpret_cast<const float4*>(sy + c);
                    const float d0 = bf16lo(pk[c / 2]) * (__uint_as_float(sr[c]) - y.x);
                    const float d1 = bf16hi(pk[c / 2]) * (__uint_as_float(sr[c + 1]) - y.y);
                    const float d2 = bf16lo(pk[c / 2 + 1]) * (__uint_as_float(sr[c + 2]) - y.z);
                    const float d3 = bf16hi(pk[c / 2 + 1]) * (__uint_as_float(sr[c + 3]) - y.w);
                    pk[c / 2] = pack_bf16x2(d0, d1);
                    pk[c / 2 + 1] = pack_bf16x2(d2, d3);
                }
                tmem_st_cols<HALF / 2>(tl + C::COL_DP + g * HALF, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_ds);
            }
            if (fail) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_le(b));
            // warpgroup 0 stores dV, warpgroup 1 stores dK (times the scale); the
            // next tile's first dV/dK MMA waits for this thread's next P^T/dS^T,
            // so it follows these loads
            const int64_t row = (int64_t)it.bkv * p.seq + kpos;
            uint16_t* grow = (g == 0 ? p.dv : p.dk) + row * HD;
            if (len > 0) {
                if (!warp_wait(bar_acc, (n_acc++) & 1, ctl)) break;
                tc_fence_after();
                const float f = g == 0 ? 1.0f : p.scale;
                const uint32_t col = g == 0 ? C::COL_DV : C::COL_DK;
                // 64 columns per TMEM wait, and 32-byte stores (whole L2 sectors) when
                // the gradient is 32-byte aligned
                const bool st32 = (reinterpret_cast<uintptr_t>(g == 0 ? p.dv : p.dk) & 31u) == 0;
#pragma unroll
                for (int c = 0; c < HD / 64; ++c) {
                    uint32_t o[64];
                    tmem_ld32(tl + col + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                    tmem_ld32(tl + col + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                    tmem_wait_ld();
                    if (row_valid) store_bf16_row<64>(grow + 64 * c, o, f, st32);
                }
            } else if (row_valid) {  // no query block lists this tile's key blocks
                for (int d = 0; d < HD; d += 8) *reinterpret_cast<uint4*>(grow + d) = make_uint4(0, 0, 0, 0);
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
    if (threadIdx.x == 0 && misc[6]) sched_leave(p.sched_kv);
}

}  // namespace s2
