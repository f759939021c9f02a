// prefill_pair_sm100.cuh -- block-sparse HHST prefill, two query tiles per CTA.
//
// S2-Attention ("S2-Attention: Hardware-aware context sharding among attention
// heads", Abstract) needs a FlashAttention-style kernel for sparsity to pay off;
// HHST shards the context across heads at block granularity, so the block is
// the tile here. One CTA owns two adjacent 128-row query tiles of one
// (batch, head). Adjacent tiles share their strided key blocks and most local
// ones, so the CTA walks the union of their key-block lists, loads each key
// block once, and runs each tile's MMAs only on the blocks that tile sees.
//
// CTA = 12 warps:
//   warp 0      TMA producer: Q of both tiles once, then K and V of each union
//               block into an ST-stage ring (SWIZZLE_128B, 64-column panels).
//   warp 1      owns TMEM; one thread issues tcgen05.mma:
//               S_t = Q_t K^T (A and B from shared memory) into TMEM, and
//               O_t += P_t V with P_t read from TMEM (A operand) and V from
//               shared memory (MN-major B operand).
//   warps 4..7  softmax of tile 0, warps 8..11 softmax of tile 1: thread = one
//               query row = one TMEM lane. Loads its S row, masks (union tag
//               bit of its query block; token causality where the key block
//               reaches its own block), keeps a running max and sum in the
//               log2 domain, writes P (bf16 pairs) over the S columns in TMEM,
//               and at the end normalises O and stores it with the LSE.
//   warps 2, 3  idle (no work; they only take part in block-wide barriers).
// The two softmax warpgroups ping-pong: while one computes exponentials for
// its tile, the tensor core runs the other tile's MMAs.
//
// Ordering facts the pipeline relies on:
//  * tcgen05.mma ops of one thread execute in issue order and a commit tracks
//    all earlier ones. S_t(next) is issued after PV_t(current), so when the
//    softmax sees S_t(next) complete, PV_t(current) has finished: P_t's TMEM
//    columns (aliased on S_t) are free and O_t is stable for a rescale.
//  * The running-max reference only moves when the max grows by more than
//    2^8 (kRescaleLog2), so O rescales are rare; P values stay <= 256.
// Every role walks the union list itself from the CSR arrays, so no shared
// per-stage record can be overwritten under a warpgroup that lags behind.
// Every wait is bounded; on a timeout the CTA drains its own copies and MMAs,
// frees TMEM and exits with the device timeout flag set.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"
#include "prefill_sm100.cuh"  // PrefillParams, umma_sdesc, umma_idesc

namespace s2 {

template <int HD, int BK>
struct PairCfg {
    static constexpr int M = 128;                          // rows per tile
    static constexpr int ROWS = (BK == 128) ? 2 : 4;       // query blocks per CTA
    static constexpr uint32_t QBYTES = M * HD * 2;         // one tile's Q
    static constexpr uint32_t KVBYTES = BK * HD * 2;       // one K (or V) block
    static constexpr int ST = (2 * QBYTES + 4 * 2 * KVBYTES <= 200 * 1024) ? 4 : 2;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + 2 * QBYTES;
    static constexpr uint32_t OFF_V = OFF_K + ST * KVBYTES;
    static constexpr uint32_t OFF_BAR = OFF_V + ST * KVBYTES;
    // barriers: q_full, k_full[ST], v_full[ST], kv_empty[ST], s_full[2], p_full[2], pv_done[2], drain
    static constexpr int NBAR = 1 + 3 * ST + 6 + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 16;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    static constexpr uint32_t TMEM_COLS = (2 * BK + 2 * HD) <= 256 ? 256 : 512;
    __host__ __device__ static constexpr uint32_t colS(int t) { return (uint32_t)(t * BK); }
    __host__ __device__ static constexpr uint32_t colO(int t) { return (uint32_t)(2 * BK + t * HD); }
    static_assert(2 * BK + 2 * HD <= 512, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

constexpr float kRescaleLog2 = 8.0f;

// Walks the ascending union of up to ROWS compacted lists (query blocks
// qb0 .. qb0+ROWS-1 of one head) and tags each key block with the rows that
// list it. Every role runs its own copy; all copies see the same sequence.
template <int ROWS>
struct UnionWalk {
    int a[ROWS], e[ROWS];
    int imax;

    __device__ __forceinline__ bool init(const int32_t* row_ptr, int rp, int qb0, int nb, int64_t nnz)
    {
        bool ok = true;
        bool any = false;
        imax = -1;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            a[r] = e[r] = 0;
            const int qb = qb0 + r;
            if (qb < nb) {
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
        }
        return ok && any;
    }

    // Next union element: key block j, row tag bits, and whether it is the last.
    // A malformed entry (j outside [0, imax]) comes out as j = 0 with no tags.
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
        bad = jm < 0 || jm > imax;
        if (bad) {
            jm = 0;
            bits = 0;
        }
        j = jm;
    }
};

// Tile t's share of a union element's row tags.
template <int BK>
__device__ __forceinline__ bool tile_sees(int bits, int t)
{
    return BK == 128 ? ((bits >> t) & 1) != 0 : ((bits >> (2 * t)) & 3) != 0;
}

template <int HD, int BK>
__global__ void __launch_bounds__(384, 1)
s2_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillParams p)
{
    using C = PairCfg<HD, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Heaviest pairs (largest query blocks) first.
    const int npairs = (p.nqt + 1) >> 1;
    const int BH = p.batch * p.heads;
    const int pr = npairs - 1 - (int)(blockIdx.x / BH);
    const int bh = (int)(blockIdx.x % BH);
    const int h = bh % p.heads;
    const int qt0 = 2 * pr;                        // first query tile
    const bool tile1 = qt0 + 1 < p.nqt;            // second tile exists
    const int qb0 = (BK == 128) ? qt0 : 2 * qt0;   // first query block
    const int64_t row_base = (int64_t)bh * p.seq;

    const uint32_t bar_q = sb + C::OFF_BAR;
    auto bar_kf = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + s); };
    auto bar_vf = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + C::ST + s); };
    auto bar_ke = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + 2 * C::ST + s); };
    auto bar_sf = [&](int t) { return sb + C::OFF_BAR + 8u * (1 + 3 * C::ST + t); };
    auto bar_pf = [&](int t) { return sb + C::OFF_BAR + 8u * (3 + 3 * C::ST + t); };
    auto bar_pv = [&](int t) { return sb + C::OFF_BAR + 8u * (5 + 3 * C::ST + t); };
    const uint32_t bar_dr = sb + C::OFF_BAR + 8u * (7 + 3 * C::ST);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_cta = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_vf(s), 1);
            mbar_init(bar_ke(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_sf(t), 1);
            mbar_init(bar_pf(t), 128);
            mbar_init(bar_pv(t), 1);
        }
        mbar_init(bar_dr, 1);
        *abort_cta = 0;
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
    const int rp = h * (p.nb + 1);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            UnionWalk<C::ROWS> it;
            const bool ok = it.init(p.row_ptr, rp, qb0, p.nb, p.nnz);
            if (!ok) atomicOr(p.gflags, kFlagIndex);
            int n = 0;
            if (ok) {
                mbar_arrive_expect_tx(bar_q, (tile1 ? 2 : 1) * C::QBYTES);
                for (int t = 0; t < (tile1 ? 2 : 1); ++t)
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_2d(sb + C::OFF_Q + t * C::QBYTES + pn * (C::M * 128), &tmQ, pn * 64,
                                    (int32_t)(row_base + (qt0 + t) * C::M), bar_q);
                for (;;) {
                    int j, bits;
                    bool last, bad;
                    it.next(p.col_idx, j, bits, last, bad);
                    if (bad) atomicOr(p.gflags, kFlagIndex);
                    const int st = n % C::ST;
                    if (!mbar_wait(bar_ke(st), ((n / C::ST) & 1) ^ 1, ctl)) break;
                    const int32_t krow = (int32_t)(row_base + (int64_t)j * BK);
                    mbar_arrive_expect_tx(bar_kf(st), C::KVBYTES);
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_2d(sb + C::OFF_K + st * C::KVBYTES + pn * (BK * 128), &tmK, pn * 64,
                                    krow, bar_kf(st));
                    mbar_arrive_expect_tx(bar_vf(st), C::KVBYTES);
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_2d(sb + C::OFF_V + st * C::KVBYTES + pn * (BK * 128), &tmV, pn * 64,
                                    krow, bar_vf(st));
                    ++n;
                    if (last) break;
                }
            }
            if (*abort_cta && ok) {  // let this CTA's own loads land before exit
                mbar_drain(bar_q, 0, kDrainNs);
                for (int m = (n > C::ST ? n - C::ST : 0); m < n; ++m) {
                    mbar_drain(bar_kf(m % C::ST), (m / C::ST) & 1, kDrainNs);
                    mbar_drain(bar_vf(m % C::ST), (m / C::ST) & 1, kDrainNs);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            UnionWalk<C::ROWS> it;
            const bool ok = it.init(p.row_ptr, rp, qb0, p.nb, p.nnz);
            constexpr uint32_t idesc_s = umma_idesc(128, BK, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc(128, HD, 0, 1);
            bool issued = false;
            int pvc[2] = {0, 0};
            auto issue_s = [&](int t, int st) {
                const uint32_t d = tmem + C::colS(t);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t a = sb + C::OFF_Q + t * C::QBYTES + (kk >> 2) * (C::M * 128) + (kk & 3) * 32;
                    const uint32_t b = sb + C::OFF_K + st * C::KVBYTES + (kk >> 2) * (BK * 128) + (kk & 3) * 32;
                    umma_bf16_ss(d, umma_sdesc(a, 16, 1024), umma_sdesc(b, 16, 1024), idesc_s,
                                 kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_sf(t));
                issued = true;
            };
            auto issue_pv = [&](int t, int st) {
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t b = sb + C::OFF_V + st * C::KVBYTES + kk * (16 * 128);
                    umma_bf16_ts(tmem + C::colO(t), tmem + C::colS(t) + kk * 8,
                                 umma_sdesc(b, BK * 128, 1024), idesc_o,
                                 (pvc[t] > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar_pv(t));
                ++pvc[t];
            };
            do {
                if (!ok) break;
                int j, bits, nbits;
                bool last, nlast, bad;
                it.next(p.col_idx, j, bits, last, bad);
                if (!mbar_wait(bar_q, 0, ctl)) break;
                if (!mbar_wait(bar_kf(0), 0, ctl)) break;
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (tile_sees<BK>(bits, t)) issue_s(t, 0);
                bool fail = false;
                for (int n = 0;; ++n) {
                    const int st = n % C::ST;
                    const int st1 = (n + 1) % C::ST;
                    nbits = 0;
                    nlast = true;
                    if (!last) it.next(p.col_idx, j, nbits, nlast, bad);
                    bool v_ready = false, k_next_ready = false;
                    if (bits == 0) {  // malformed entry no tile sees: let its loads land first
                        if (!mbar_wait(bar_kf(st), (n / C::ST) & 1, ctl) ||
                            !mbar_wait(bar_vf(st), (n / C::ST) & 1, ctl))
                            break;
                    }
                    const int last_t = tile_sees<BK>(bits, 1) ? 1 : (tile_sees<BK>(bits, 0) ? 0 : 1);
                    for (int t = 0; t < 2 && !fail; ++t) {
                        if (tile_sees<BK>(bits, t)) {
                            if (!mbar_wait(bar_pf(t), pvc[t] & 1, ctl)) { fail = true; break; }
                            if (!v_ready) {
                                if (!mbar_wait(bar_vf(st), (n / C::ST) & 1, ctl)) { fail = true; break; }
                                v_ready = true;
                            }
                            tc_fence_after();
                            issue_pv(t, st);
                        }
                        if (t == last_t) umma_commit(bar_ke(st));
                        if (!last && tile_sees<BK>(nbits, t)) {
                            if (!k_next_ready) {
                                if (!mbar_wait(bar_kf(st1), ((n + 1) / C::ST) & 1, ctl)) { fail = true; break; }
                                k_next_ready = true;
                                tc_fence_after();
                            }
                            issue_s(t, st1);
                        }
                    }
                    if (fail || last) break;
                    bits = nbits;
                    last = nlast;
                }
            } while (0);
            if (*abort_cta && issued) {
                umma_commit(bar_dr);
                mbar_drain(bar_dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax
        const int t = (warp - 4) >> 2;              // tile of this warpgroup
        const int quad = warp & 3;                  // TMEM lane quadrant
        const int r = quad * 32 + lane;             // row within the tile
        const int qpos = (qt0 + t) * C::M + r;      // query position
        const int rowbit = (BK == 128) ? t : 2 * t + (r >> 6);
        const bool active = (t == 0) || tile1;
        const bool row_valid = active && qpos < p.seq && (qb0 + rowbit) < p.nb;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        float m_used = -1e30f, l = 0.f;
        int cnt = 0;
        bool done = false;
        UnionWalk<C::ROWS> it;
        const bool ok = it.init(p.row_ptr, rp, qb0, p.nb, p.nnz);
        if (ok && active) {
            for (;;) {
                int j, bits;
                bool last, bad;
                it.next(p.col_idx, j, bits, last, bad);
                if (tile_sees<BK>(bits, t)) {
                    bool w = mbar_wait(bar_sf(t), cnt & 1, ctl);
                    if (!__all_sync(0xffffffffu, w)) break;
                    tc_fence_after();
                    uint32_t sr[BK];
#pragma unroll
                    for (int c = 0; c < BK / 32; ++c)
                        tmem_ld32(tl + C::colS(t) + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
                    tmem_wait_ld();
                    const bool vis = (bits >> rowbit) & 1;
                    const int lim = qpos - j * BK;  // key column c visible iff c <= lim
                    float mt = -INFINITY;
#pragma unroll
                    for (int c = 0; c < BK; ++c) {
                        const float x = (vis && c <= lim) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
                        sr[c] = __float_as_uint(x);
                        mt = fmaxf(mt, x);
                    }
                    const float m_cand = fmaxf(m_used, mt);
                    const bool move = m_cand - m_used > kRescaleLog2;
                    const float alpha = move ? ex2(m_used - m_cand) : 1.0f;
                    if (move) m_used = m_cand;
                    float rs = 0.f;
#pragma unroll
                    for (int c = 0; c < BK / 2; ++c) {
                        const float p0 = ex2(__uint_as_float(sr[2 * c]) - m_used);
                        const float p1 = ex2(__uint_as_float(sr[2 * c + 1]) - m_used);
                        rs += p0 + p1;
                        sr[c] = pack_bf16x2(p0, p1);
                    }
                    l = l * alpha + rs;
                    // P (bf16 pairs) over the first BK/2 columns of S_t.
#pragma unroll
                    for (int c = 0; c < BK / 64; ++c)
                        tmem_st32(tl + C::colS(t) + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32 * c]));
                    if (cnt > 0 && __any_sync(0xffffffffu, move)) {
                        // O_t is stable: S_t of this block completed after PV_t of the last one.
#pragma unroll
                        for (int c = 0; c < HD / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tl + C::colO(t) + 32 * c, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st32(tl + C::colO(t) + 32 * c, o);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_pf(t));
                    ++cnt;
                }
                if (last) {
                    done = true;
                    break;
                }
            }
        }
        if (done && cnt > 0) {
            const bool w = mbar_wait(bar_pv(t), (cnt - 1) & 1, ctl);
            if (__all_sync(0xffffffffu, w)) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.0f / l : 0.f;
                uint16_t* orow = p.o + (row_base + qpos) * HD;
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tl + C::colO(t) + 32 * c, o);
                    tmem_wait_ld();
                    if (row_valid) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv, __uint_as_float(o[e + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                            *reinterpret_cast<uint4*>(orow + 32 * c + e) = v;
                        }
                    }
                }
                if (row_valid && p.lse)
                    p.lse[row_base + qpos] = l > 0.f ? (m_used + lg2(l)) * 0.69314718055994531f : -INFINITY;
            }
        } else if (row_valid && !ok) {
            uint16_t* orow = p.o + (row_base + qpos) * HD;
            for (int d = 0; d < HD; d += 8) *reinterpret_cast<uint4*>(orow + d) = make_uint4(0, 0, 0, 0);
            if (p.lse) p.lse[row_base + qpos] = -INFINITY;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace s2
