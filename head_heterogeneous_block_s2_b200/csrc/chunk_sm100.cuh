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
// One CTA = one 128-row tile of absolute positions [128 t, 128 t + 128) of one
// (sequence, head), cut to the chunk; it walks the union of the tile's query
// blocks' key-block lists. Q comes by TMA from the packed chunk rows
// [total_q][heads][D] (rows outside the chunk read zeros or other rows and are
// never stored). A key block is B / 16 pages: each page is one TMA box of a
// 3-D map over the cache [num_pages * heads_kv][16][D]; pages past the
// context (or with an invalid id, which is flagged) load zeros through an
// out-of-range coordinate. Rows past the context inside the last page hold
// whatever the cache holds there, so the element-wise warps zero them in
// shared memory before the P V product uses them (their P is 0 anyway, but
// 0 times a NaN would not be).
//
// CTA = 12 warps: warp 0 lane 0 loads Q and streams K (3 stages), warp 3
// lane 0 streams V (2 stages), warp 1 owns TMEM and issues tcgen05.mma
// (S = Q K^T into one of two TMEM buffers, O += P V with P from TMEM), warp 2
// builds the union list, warps 4..11 run the online softmax and the epilogue:
// thread = row = TMEM lane, warps 4..7 on the first half of each block's
// columns and warps 8..11 on the second; the two halves of a row exchange
// their maxima through shared memory once per block (an mbarrier of the 256
// softmax threads, waited with the same bound as every other wait, so a CTA
// that gives up cannot strand the others) and keep partial sums that meet in
// the epilogue. S is
// double-buffered, so the softmax of one key block overlaps the MMAs of the
// next.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>

#include "lists.cuh"
#include "ptx.cuh"
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
};

constexpr int kChunkPage = 16;  // tokens per cache page

template <int HD, int BK>
struct ChunkCfg {
    static constexpr int M = 128;
    static constexpr int ROWS = 128 / BK;              // query blocks per tile
    static constexpr uint32_t QBYTES = M * HD * 2;
    static constexpr uint32_t KVBYTES = BK * HD * 2;   // one K or V block
    static constexpr int KST = 3, VST = 2;             // K and V ring depths
    static constexpr int LIST_CAP = 2048;
    static constexpr uint32_t OFF_Q = 0;                       // [panel][128 rows x 128 B]
    static constexpr uint32_t OFF_K = QBYTES;                  // [stage][panel][BK rows x 128 B]
    static constexpr uint32_t OFF_V = OFF_K + KST * KVBYTES;
    static constexpr uint32_t OFF_LIST = OFF_V + VST * KVBYTES;
    static constexpr uint32_t OFF_SCR = OFF_LIST + LIST_CAP * 4;
    // exchange slots [3][2][128] floats: row maxima by block parity, then partial sums
    static constexpr uint32_t OFF_XCH = OFF_SCR + (ROWS > 1 ? ROWS * LIST_CAP * 4 : 0);
    static constexpr uint32_t OFF_BAR = OFF_XCH + 3 * 2 * 128 * 4;
    // barriers: q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], p_full,
    // pv_done, drain, xch[2], xch_sum
    static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 8;
    static constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) / 16) * 16;
    static constexpr uint32_t SMEM = OFF_MISC + 32;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
    __host__ __device__ static constexpr uint32_t colS(int b) { return (uint32_t)(b * BK); }
    static constexpr uint32_t COL_O = 2 * BK;
    static constexpr uint32_t COL_QA = 2 * BK + HD;  // Q, the A operand of every S MMA (HD/2 columns)
    static constexpr uint32_t TMEM_COLS = (2 * BK + HD + HD / 2) <= 256 ? 256 : 512;
    static_assert(2 * BK + HD + HD / 2 <= 512, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

template <int HD, int BK>
__global__ void __launch_bounds__(384, 1)
s2_chunk_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const ChunkParams p)
{
    using C = ChunkCfg<HD, BK>;
    const int u = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    // ---- this CTA's tile (uniform over the CTA: every thread may leave together)
    const int n = __ldg(p.ctx_lens + s);
    const int q0 = __ldg(p.q_start + s), ql = __ldg(p.q_start + s + 1) - q0;
    const bool seq_ok = ql >= 0 && ql <= p.max_q_len && ql <= n && q0 >= 0 && (int64_t)q0 + ql <= p.total_q &&
                        (int64_t)n <= (int64_t)p.max_pages * kChunkPage && (n == 0 || (n - 1) / BK < p.nb);
    if (!seq_ok) {
        if (u == 0 && h == 0 && threadIdx.x == 0) atomicOr(p.gflags, kFlagIndex);
        return;
    }
    if (ql == 0) return;
    const int c0 = n - ql;                   // first chunk position
    const int t = c0 / C::M + u;             // absolute 128-row tile
    if (t * C::M >= n) return;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hkv = h / (p.heads / p.heads_kv);

    const uint32_t bar_q = sb + C::OFF_BAR;
    auto bar_kf = [&](int i) { return sb + C::OFF_BAR + 8u * (1 + i); };
    auto bar_ke = [&](int i) { return sb + C::OFF_BAR + 8u * (1 + C::KST + i); };
    auto bar_vf = [&](int i) { return sb + C::OFF_BAR + 8u * (1 + 2 * C::KST + i); };
    auto bar_ve = [&](int i) { return sb + C::OFF_BAR + 8u * (1 + 2 * C::KST + C::VST + i); };
    auto bar_sf = [&](int b) { return sb + C::OFF_BAR + 8u * (1 + 2 * C::KST + 2 * C::VST + b); };
    const uint32_t bar_p = sb + C::OFF_BAR + 8u * (3 + 2 * C::KST + 2 * C::VST);
    const uint32_t bar_pv = bar_p + 8u;
    const uint32_t bar_dr = bar_p + 16u;
    auto bar_x = [&](int b) { return bar_p + 24u + 8u * b; };  // max exchange, by block parity
    const uint32_t bar_xl = bar_p + 40u;                        // partial-sum exchange
    uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);  // [0] tmem, [1] abort, [2] list length
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_cta = misc + 1;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < C::KST; ++i) {
            mbar_init(bar_kf(i), 1);
            mbar_init(bar_ke(i), 1);
        }
        for (int i = 0; i < C::VST; ++i) {
            mbar_init(bar_vf(i), 1);
            mbar_init(bar_ve(i), 1);
        }
        mbar_init(bar_sf(0), 1);
        mbar_init(bar_sf(1), 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_pv, 1);
        mbar_init(bar_dr, 1);
        mbar_init(bar_x(0), 256);
        mbar_init(bar_x(1), 256);
        mbar_init(bar_xl, 256);
        *abort_cta = 0;
        fence_mbar_init();
        // Q of the tile: chunk row of position t*128 is q0 + t*128 - c0 (may be
        // negative or past the end: those rows read zeros and are not stored)
        mbar_arrive_expect_tx(bar_q, C::QBYTES);
#pragma unroll
        for (int pn = 0; pn < HD / 64; ++pn)
            tma_load_3d(sb + C::OFF_Q + pn * (C::M * 128), &tmQ, pn * 64, h, q0 + t * C::M - c0, bar_q);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 2) {
        int rows[C::ROWS];
#pragma unroll
        for (int r = 0; r < C::ROWS; ++r) rows[r] = t * C::ROWS + r;
        const int len = warp_union_list<C::ROWS>(p.row_ptr, p.col_idx, h * (p.nb + 1), rows, p.nb, p.nnz, 0,
                                                 min(t * C::ROWS + C::ROWS, p.nb) - 1, list, C::LIST_CAP,
                                                 reinterpret_cast<int32_t*>(smem + C::OFF_SCR), p.gflags);
        if (lane == 0) misc[2] = len;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int len = misc[2];
    const WaitCtl ctl{p.timeout_ns, p.gflags, abort_cta};
    constexpr uint64_t kDrainNs = 200000000ull;
    const int32_t oob_plane = (int32_t)(p.num_pages * p.heads_kv);  // reads zeros

    // Cache plane (page * heads_kv + hkv) of logical page lp, or the zero plane.
    auto page_plane = [&](int lp) -> int32_t {
        if (lp * kChunkPage >= n) return oob_plane;
        const int32_t phys = __ldg(p.block_table + (int64_t)s * p.max_pages + lp);
        if (phys < 0 || phys >= p.num_pages) {
            atomicOr(p.gflags, kFlagIndex);
            return oob_plane;
        }
        return phys * p.heads_kv + hkv;
    };

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------------------ K (warp 0) and V (warp 3) producers
        const bool is_k = warp == 0;
        if (lane == 0 && len == 0 && is_k) mbar_drain(bar_q, 0, kDrainNs);  // nothing to do: let Q land
        if (lane == 0 && len > 0) {
            const int NST = is_k ? C::KST : C::VST;
            const uint32_t base = is_k ? C::OFF_K : C::OFF_V;
            const CUtensorMap* map = is_k ? &tmK : &tmV;
            int e = 0;
            for (; e < len; ++e) {
                const int st = e % NST;
                const uint32_t full = is_k ? bar_kf(st) : bar_vf(st);
                if (!mbar_wait(is_k ? bar_ke(st) : bar_ve(st), ((e / NST) & 1) ^ 1, ctl)) break;
                const int j = list_j(list[e]);
                mbar_arrive_expect_tx(full, C::KVBYTES);
                for (int pg = 0; pg < BK / kChunkPage; ++pg) {
                    const int32_t plane = page_plane(j * (BK / kChunkPage) + pg);
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn)
                        tma_load_3d(sb + base + st * C::KVBYTES + pn * (BK * 128) + pg * (kChunkPage * 128), map,
                                    pn * 64, 0, plane, full);
                }
            }
            if (*abort_cta) {  // let this CTA's own loads land before exit
                if (is_k) mbar_drain(bar_q, 0, kDrainNs);
                for (int m = (e > NST ? e - NST : 0); m < e; ++m)
                    mbar_drain(is_k ? bar_kf(m % NST) : bar_vf(m % NST), (m / NST) & 1, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && len > 0) {
            constexpr uint32_t idesc_s = umma_idesc(128, BK, 0, 0);   // S = Q K^T
            constexpr uint32_t idesc_o = umma_idesc(128, HD, 0, 1);   // O += P V (V as MN-major B)
            const uint64_t dq = umma_sdesc(sb + C::OFF_Q, 16, 1024);
            bool issued = false;
            // S(e) goes to TMEM buffer e & 1; S(e+2) is issued after PV(e), which
            // reads P(e) from that buffer (MMAs of one thread run in issue order).
            auto issue_s = [&](int e) {
                const int st = e % C::KST;
                if (!mbar_wait(bar_kf(st), (e / C::KST) & 1, ctl)) return false;
                tc_fence_after();
                const uint64_t dk = umma_sdesc(sb + C::OFF_K + st * C::KVBYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t off_q = (uint64_t)((((kk >> 2) * (C::M * 128)) + (kk & 3) * 32) >> 4);
                    const uint64_t off_k = (uint64_t)((((kk >> 2) * (BK * 128)) + (kk & 3) * 32) >> 4);
                    (void)off_q;
                    umma_bf16_ts(tmem + C::colS(e & 1), tmem + C::COL_QA + kk * 8, dk + off_k, idesc_s,
                                 kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_ke(st));
                umma_commit(bar_sf(e & 1));
                issued = true;
                return true;
            };
            const bool q_ok = mbar_wait(bar_q, 0, ctl);
            if (q_ok) {  // Q into TMEM, in issue order before every S MMA
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    tmem_cp_128x256b(tmem + C::COL_QA + kk * 8,
                                     dq + (uint64_t)((((kk >> 2) * (C::M * 128)) + (kk & 3) * 32) >> 4));
                issued = true;
            }
            if (q_ok && issue_s(0) && (len < 2 || issue_s(1))) {
                for (int e = 0; e < len; ++e) {
                    const int vs = e % C::VST;
                    if (!mbar_wait(bar_p, e & 1, ctl)) break;
                    if (!mbar_wait(bar_vf(vs), (e / C::VST) & 1, ctl)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t dv = umma_sdesc(sb + C::OFF_V + vs * C::KVBYTES + kk * 2048, BK * 128, 1024);
                        // the two softmax halves packed P into the first quarter of each half
                        const uint32_t pcol = (kk / (BK / 32)) * (BK / 2) + (kk % (BK / 32)) * 8;
                        umma_bf16_ts(tmem + C::COL_O, tmem + C::colS(e & 1) + pcol, dv, idesc_o,
                                     (e > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_ve(vs));
                    umma_commit(bar_pv);
                    if (e + 2 < len && !issue_s(e + 2)) break;
                }
            }
            if (*abort_cta && issued) {
                umma_commit(bar_dr);
                mbar_drain(bar_dr, 0, kDrainNs);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ online softmax + epilogue
        constexpr int HALF = BK / 2;  // key columns per warpgroup
        const int quad = warp & 3, g = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);  // [slot][half][row]
        const int pos = t * C::M + r;
        const int rowbit = (BK == 128) ? 0 : (r >> 6);
        const bool row_valid = pos >= c0 && pos < n;
        const float sc = p.scale_log2;  // > 0
        const int n16 = ((n + kChunkPage - 1) / kChunkPage) * kChunkPage;  // end of the last loaded page
        float m_used = -1e30f, l = 0.f;  // l: this half's partial row sum
        bool fail = false;
        for (int e = 0; e < len; ++e) {
            const uint32_t ent = list[e];
            const int j = list_j(ent);
            const int b = e & 1;
            if (!warp_wait(bar_sf(b), (e >> 1) & 1, ctl)) {
                fail = true;
                break;
            }
            tc_fence_after();
            uint32_t sr[HALF];
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c)
                tmem_ld32(tl + C::colS(b) + g * HALF + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
            tmem_wait_ld();
            const bool vis = row_valid && ((list_bits(ent) >> rowbit) & 1);
            const int lim = pos - j * BK - g * HALF;  // column c of this half visible iff c <= lim
#pragma unroll
            for (int c = 0; c < HALF; ++c)
                if (!(vis && c <= lim)) sr[c] = 0xff800000u;  // -inf
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < HALF; c += 2) mx = fmax3(mx, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
            // the row's maximum over both halves (slots alternate by block parity, so
            // a slot is rewritten only after its reader has passed the next barrier)
            xch[(b * 2 + g) * 128 + r] = mx;
            mbar_arrive(bar_x(b));
            if (!warp_wait(bar_x(b), (e >> 1) & 1, ctl)) {
                fail = true;
                break;
            }
            mx = fmaxf(mx, xch[(b * 2 + (g ^ 1)) * 128 + r]);
            const float m_cand = fmaxf(m_used, mx * sc);
            const bool move = m_cand - m_used > 8.0f;  // rescale O only when the max grew by > 2^8
            const float alpha = move ? ex2(m_used - m_cand) : 1.0f;
            if (move) m_used = m_cand;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < HALF / 2; ++c) {
                const float p0 = ex2(fmaf(__uint_as_float(sr[2 * c]), sc, -m_used));
                const float p1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), sc, -m_used));
                rs += p0 + p1;
                sr[c] = pack_bf16x2(p0, p1);  // slot c <= 2c: already read
            }
            l = l * alpha + rs;
            if constexpr (HALF / 2 == 32) {
                tmem_st32(tl + C::colS(b) + g * HALF, *reinterpret_cast<const uint32_t(*)[32]>(&sr[0]));
            } else {
                tmem_st16(tl + C::colS(b) + g * HALF, *reinterpret_cast<const uint32_t(*)[16]>(&sr[0]));
            }
            // Rows of this block past the context inside its last loaded page hold
            // stale cache data: zero them in V before the P V product reads them.
            const int z0 = n - j * BK, z1 = min(BK, n16 - j * BK);
            if (z0 < z1 && g == 0) {
                const int vs = e % C::VST;
                if (!warp_wait(bar_vf(vs), (e / C::VST) & 1, ctl)) {
                    fail = true;
                    break;
                }
                if (r >= z0 && r < z1) {
#pragma unroll
                    for (int pn = 0; pn < HD / 64; ++pn) {
                        uint4* line = reinterpret_cast<uint4*>(smem + C::OFF_V + vs * C::KVBYTES + pn * (BK * 128) + r * 128);
#pragma unroll
                        for (int w = 0; w < 8; ++w) line[w] = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
            }
            // O is stable once PV(e-1) is done: each half rescales its HD/2 columns
            if (e > 0 && !warp_wait(bar_pv, (e - 1) & 1, ctl)) {
                fail = true;
                break;
            }
            tc_fence_after();
            if (e > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
                for (int c = 0; c < HD / 64; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tl + C::COL_O + g * (HD / 2) + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e2 = 0; e2 < 32; ++e2) o[e2] = __float_as_uint(__uint_as_float(o[e2]) * alpha);
                    tmem_st32(tl + C::COL_O + g * (HD / 2) + 32 * c, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p);
        }
        if (!fail) {  // the two halves' partial sums meet
            xch[(4 + g) * 128 + r] = l;  // slot 2: never used by the max exchange
            mbar_arrive(bar_xl);
            fail = !warp_wait(bar_xl, 0, ctl);
            l += xch[(4 + (g ^ 1)) * 128 + r];
        }
        if (!fail) {
            // every lane takes part in the waits and TMEM loads; only chunk rows store
            const bool acc_ok = len > 0 && warp_wait(bar_pv, (len - 1) & 1, ctl);
            const int64_t orow = (int64_t)(q0 + pos - c0) * p.heads + h;
            uint16_t* og = p.out + orow * HD + g * (HD / 2);
            if (acc_ok) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
                for (int c = 0; c < HD / 64; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tl + C::COL_O + g * (HD / 2) + 32 * c, o);
                    tmem_wait_ld();
                    if (row_valid) {
#pragma unroll
                        for (int e2 = 0; e2 < 32; e2 += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(o[e2 + 0]) * inv, __uint_as_float(o[e2 + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(o[e2 + 2]) * inv, __uint_as_float(o[e2 + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(o[e2 + 4]) * inv, __uint_as_float(o[e2 + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(o[e2 + 6]) * inv, __uint_as_float(o[e2 + 7]) * inv);
                            *reinterpret_cast<uint4*>(og + 32 * c + e2) = v;
                        }
                    }
                }
                if (row_valid && g == 0 && p.lse)
                    p.lse[orow] = l > 0.f ? (m_used + lg2(l)) * 0.69314718055994531f : -INFINITY;
            } else if (len == 0 && row_valid) {  // no key block listed for this tile
                for (int d = 0; d < HD / 2; d += 8) *reinterpret_cast<uint4*>(og + d) = make_uint4(0, 0, 0, 0);
                if (g == 0 && p.lse) p.lse[orow] = -INFINITY;
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

}  // namespace s2
