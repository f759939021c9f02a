// prefill_sm100.cuh -- block-sparse HHST prefill attention on sm_100a.
//
// S2-Attention ("S2-Attention: Hardware-aware context sharding among attention
// heads", Abstract) argues that sparse attention only pays off with a
// FlashAttention-style, hardware-aware kernel; HHST shards the context across
// heads at block granularity. This kernel makes the block the tile: one CTA
// owns 128 query rows of one (batch, head) and visits only the key blocks in
// that row's compacted list, with an online softmax across them.
//
// CTA = 6 warps:
//   warp 0      TMA producer: Q once, then K and V tiles of each listed key
//               block into an ST-stage ring (SWIZZLE_128B, 64-column panels).
//   warp 1      owns TMEM and issues tcgen05.mma from one thread:
//               S = Q K^T into one of two TMEM score buffers, then
//               O += P V into the TMEM output accumulator.
//   warps 2..5  softmax: thread = one query row = one TMEM lane. Loads its
//               score row, masks (block bits; token causality only where the
//               key block reaches the row's own block), keeps running max and
//               sum, rescales O in TMEM when the max grows, writes P (bf16) to
//               shared memory in the UMMA K-major SWIZZLE_128B layout, and at
//               the end normalises O and stores it with the log-sum-exp.
// With block size 64 one 128-row tile holds two query blocks; the producer
// walks the union of their two lists and tags each key block with which
// halves see it.
//
// Every wait is bounded (WaitCtl); on a timeout the CTA drains its own copies
// and MMAs, frees TMEM and exits with the device timeout flag set.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"

namespace s2 {

struct PrefillParams {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t nnz;
    uint16_t* o;  // bf16 bits
    float* lse;   // may be null
    int32_t batch, heads, seq, nb, nqt;
    float scale_log2;  // scale * log2(e)
    uint64_t timeout_ns;
    uint32_t* gflags;
    int* sched;  // pair kernel work counter {next item, CTAs done}, zero at launch
};

template <int HD, int BK>
struct PrefillCfg {
    static constexpr int M = 128;          // query rows per tile
    static constexpr int ST = (HD == 128 && BK == 128) ? 2 : 4;
    static constexpr uint32_t QBYTES = M * HD * 2;
    static constexpr uint32_t KVBYTES = BK * HD * 2;
    static constexpr uint32_t PBYTES = M * BK * 2;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + QBYTES;
    static constexpr uint32_t OFF_V = OFF_K + ST * KVBYTES;
    static constexpr uint32_t OFF_P = OFF_V + ST * KVBYTES;
    static constexpr uint32_t OFF_BAR = OFF_P + PBYTES;
    // barriers: q_full, k_full[ST], v_full[ST], kv_empty[ST], s_full[2], p_full, pv_done, drain
    static constexpr int NBAR = 1 + 3 * ST + 2 + 3;
    static constexpr uint32_t OFF_INFO = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t OFF_MISC = OFF_INFO + ST * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 16;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;  // slack for 1024-byte alignment
    static constexpr uint32_t TMEM_COLS = (2 * BK + HD) <= 256 ? 256 : 512;
    static constexpr uint32_t COL_O = 2 * BK;
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
    static_assert(HD % 64 == 0 && BK % 64 == 0, "64-column panels");
};

// UMMA shared-memory descriptor, SWIZZLE_128B, version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// UMMA instruction descriptor: bf16 x bf16 -> fp32, M x N, operand majors.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, int a_mn_major, int b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
           ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int HD, int BK>
__global__ void __launch_bounds__(192, 1)
s2_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const PrefillParams p)
{
    using C = PrefillCfg<HD, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Heaviest tiles (largest query block) first; all (batch, head) pairs of
    // one query tile are adjacent in launch order.
    const int BH = p.batch * p.heads;
    const int qt = p.nqt - 1 - (int)(blockIdx.x / BH);
    const int bh = (int)(blockIdx.x % BH);
    const int h = bh % p.heads;
    const int i0 = (BK == 128) ? qt : 2 * qt;
    const int i1 = (BK == 128) ? -1 : (2 * qt + 1 < p.nb ? 2 * qt + 1 : -1);
    const int imax = i1 >= 0 ? i1 : i0;

    const uint32_t bar_q = sb + C::OFF_BAR;
    auto bar_kf = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + s); };
    auto bar_vf = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + C::ST + s); };
    auto bar_ke = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + 2 * C::ST + s); };
    auto bar_sf = [&](int b) { return sb + C::OFF_BAR + 8u * (1 + 3 * C::ST + b); };
    const uint32_t bar_pf = sb + C::OFF_BAR + 8u * (3 + 3 * C::ST);
    const uint32_t bar_pv = sb + C::OFF_BAR + 8u * (4 + 3 * C::ST);
    const uint32_t bar_dr = sb + C::OFF_BAR + 8u * (5 + 3 * C::ST);
    int4* info = reinterpret_cast<int4*>(smem + C::OFF_INFO);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_cta = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_vf(s), 1);
            mbar_init(bar_ke(s), 1);
        }
        mbar_init(bar_sf(0), 1);
        mbar_init(bar_sf(1), 1);
        mbar_init(bar_pf, 128);
        mbar_init(bar_pv, 1);
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

    // Row ranges of the tile's query blocks, validated against the list size.
    const int rp = h * (p.nb + 1);
    int a0 = p.row_ptr[rp + i0], e0 = p.row_ptr[rp + i0 + 1];
    int a1 = 0, e1 = 0;
    if (i1 >= 0) {
        a1 = p.row_ptr[rp + i1];
        e1 = p.row_ptr[rp + i1 + 1];
    }
    bool rows_ok = a0 >= 0 && a0 <= e0 && e0 <= p.nnz && a1 >= 0 && a1 <= e1 && e1 <= p.nnz &&
                   (e0 > a0 || e1 > a1);
    if (!rows_ok && threadIdx.x == 0) atomicOr(p.gflags, kFlagIndex);

    const int64_t row_base = (int64_t)bh * p.seq;  // first row of this (b, h) in [rows, HD]

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && rows_ok) {
            int n = 0;
            mbar_arrive_expect_tx(bar_q, C::QBYTES);
#pragma unroll
            for (int pn = 0; pn < HD / 64; ++pn)
                tma_load_2d(sb + C::OFF_Q + pn * (C::M * 128), &tmQ, pn * 64,
                            (int32_t)(row_base + qt * C::M), bar_q);
            for (;;) {
                const int ja = a0 < e0 ? p.col_idx[a0] : INT_MAX;
                const int jb = a1 < e1 ? p.col_idx[a1] : INT_MAX;
                int j = ja < jb ? ja : jb;
                int bits = (ja == j ? 1 : 0) | (jb == j ? 2 : 0);
                if (ja == j) ++a0;
                if (jb == j) ++a1;
                const int last = (a0 >= e0 && a1 >= e1) ? 1 : 0;
                if (j < 0 || j > imax) {  // malformed list: load block 0, mask it out
                    atomicOr(p.gflags, kFlagIndex);
                    j = 0;
                    bits = 0;
                }
                const int st = n % C::ST;
                if (!mbar_wait(bar_ke(st), ((n / C::ST) & 1) ^ 1, ctl)) break;
                info[st] = make_int4(j, bits, last, 0);
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
            if (*abort_cta) {  // let this CTA's own loads land before exit
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
        if (lane == 0 && rows_ok) {
            constexpr uint32_t idesc_s = umma_idesc(128, BK, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc(128, HD, 0, 1);
            bool issued = false;
            auto issue_s = [&](int n) {
                const int st = n % C::ST;
                const uint32_t d = tmem + (uint32_t)((n & 1) * BK);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t a = sb + C::OFF_Q + (kk >> 2) * (C::M * 128) + (kk & 3) * 32;
                    const uint32_t b = sb + C::OFF_K + st * C::KVBYTES + (kk >> 2) * (BK * 128) +
                                       (kk & 3) * 32;
                    umma_bf16_ss(d, umma_sdesc(a, 16, 1024), umma_sdesc(b, 16, 1024), idesc_s,
                                 kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_sf(n & 1));
                issued = true;
            };
            do {
                if (!mbar_wait(bar_q, 0, ctl)) break;
                if (!mbar_wait(bar_kf(0), 0, ctl)) break;
                tc_fence_after();
                issue_s(0);
                for (int n = 0;; ++n) {
                    const int st = n % C::ST;
                    const int4 inf = info[st];
                    if (!inf.z) {
                        const int n1 = n + 1;
                        if (!mbar_wait(bar_kf(n1 % C::ST), (n1 / C::ST) & 1, ctl)) break;
                        tc_fence_after();
                        issue_s(n1);
                    }
                    if (!mbar_wait(bar_pf, n & 1, ctl)) break;
                    if (!mbar_wait(bar_vf(st), (n / C::ST) & 1, ctl)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t a = sb + C::OFF_P + (kk >> 2) * (C::M * 128) + (kk & 3) * 32;
                        const uint32_t b = sb + C::OFF_V + st * C::KVBYTES + kk * (16 * 128);
                        umma_bf16_ss(tmem + C::COL_O, umma_sdesc(a, 16, 1024),
                                     umma_sdesc(b, BK * 128, 1024), idesc_o,
                                     (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_ke(st));
                    umma_commit(bar_pv);
                    if (inf.z) break;
                }
            } while (0);
            if (*abort_cta && issued) {
                umma_commit(bar_dr);
                mbar_drain(bar_dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3;            // TMEM lane quadrant of this warp
        const int r = quad * 32 + lane;       // tile row
        const int qpos = qt * C::M + r;       // query position in the sequence
        const int half = (BK == 64) ? (r >> 6) : 0;
        const bool row_valid = qpos < p.seq && (half == 0 || i1 >= 0);
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        float m = -1e30f, l = 0.f;
        int n = 0;
        bool done = false;
        if (rows_ok) {
            for (;; ++n) {
                const int st = n % C::ST;
                bool ok = mbar_wait(bar_kf(st), (n / C::ST) & 1, ctl);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int4 inf = info[st];
                ok = mbar_wait(bar_sf(n & 1), (n >> 1) & 1, ctl);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();

                uint32_t sr[BK];
#pragma unroll
                for (int c = 0; c < BK / 32; ++c)
                    tmem_ld32(tl + (uint32_t)((n & 1) * BK + 32 * c),
                              *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
                tmem_wait_ld();

                const bool vis = (inf.y >> half) & 1;
                const int lim = qpos - inf.x * BK;  // key column c visible iff c <= lim
                float mt = -INFINITY;
#pragma unroll
                for (int c = 0; c < BK; ++c) {
                    const float x = (vis && c <= lim) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
                    sr[c] = __float_as_uint(x);
                    mt = fmaxf(mt, x);
                }
                const float m_new = fmaxf(m, mt);
                const float alpha = ex2(m - m_new);
                float rs = 0.f;
#pragma unroll
                for (int c = 0; c < BK; ++c) {
                    const float pc = ex2(__uint_as_float(sr[c]) - m_new);
                    rs += pc;
                    sr[c] = __float_as_uint(pc);
                }
                if (n > 0) {
                    ok = mbar_wait(bar_pv, (n - 1) & 1, ctl);
                    if (!__all_sync(0xffffffffu, ok)) break;
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
                        for (int c = 0; c < HD / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tl + C::COL_O + 32 * c, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st32(tl + C::COL_O + 32 * c, o);
                        }
                        tmem_wait_st();
                    }
                }
                l = l * alpha + rs;
                m = m_new;
                // P row -> shared memory, UMMA K-major SWIZZLE_128B (64-key panels).
                uint8_t* prow = smem + C::OFF_P + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int ch = 0; ch < BK / 8; ++ch) {
                    const int pn = ch >> 3, cc = ch & 7;
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(sr[8 * ch + 0]), __uint_as_float(sr[8 * ch + 1]));
                    v.y = pack_bf16x2(__uint_as_float(sr[8 * ch + 2]), __uint_as_float(sr[8 * ch + 3]));
                    v.z = pack_bf16x2(__uint_as_float(sr[8 * ch + 4]), __uint_as_float(sr[8 * ch + 5]));
                    v.w = pack_bf16x2(__uint_as_float(sr[8 * ch + 6]), __uint_as_float(sr[8 * ch + 7]));
                    *reinterpret_cast<uint4*>(prow + pn * (C::M * 128) + ((cc ^ (r & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar_pf);
                if (inf.z) {
                    done = true;
                    break;
                }
            }
        }
        if (done) {
            const bool ok = mbar_wait(bar_pv, n & 1, ctl);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.0f / l : 0.f;
                uint16_t* orow = p.o + (row_base + qpos) * HD;
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tl + C::COL_O + 32 * c, o);
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
                    p.lse[row_base + qpos] = l > 0.f ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
            }
        } else if (!rows_ok && row_valid) {
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
