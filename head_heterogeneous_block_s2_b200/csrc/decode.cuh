// decode.cuh -- split-KV HHST decode over a paged KV cache, and its combine.
//
// At inference HHST is served from a paged KV cache ("S2-Attention" abstract:
// 4.5x faster 7B inference in vLLM; PagedAttention is in the arXiv page's
// reference list). One query token per sequence attends to the tokens of the
// key blocks listed for its query block. The work of one (sequence, head) is
// the list of 16-token pages of its active key blocks; it is cut into
// num_splits contiguous page ranges, one CTA each.
//
// CTA = 5 warps. Warp 0 (one thread) streams K and V pages with untiled bulk
// copies (4 KB per page and head at head_dim 128, contiguous in the
// [page][head][token][dim] cache) into an NS-stage ring. Warps 1..4 each take
// every 4th page: a lane pair computes one token's q.k (each lane half of the
// dimensions, read from shared memory in a rotated order that keeps all 32
// banks busy), the warp keeps an online softmax (running max, sum) and
// accumulates p * V with each lane owning head_dim / 32 output dimensions.
// The four warps then merge their states. With one split the CTA writes the
// final bf16 output; otherwise it writes fp32 partials (un-normalised O, max,
// sum) that s2_decode_combine_kernel merges by the associative log-sum-exp
// rule (the online-softmax reduction LeanAttention describes as a reduction).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace s2 {

struct DecodeParams {
    const uint16_t* q;       // [batch][H][HD]
    const uint16_t* k_cache; // [pages][H_kv][16][HD]; query head h reads K/V head h / (H / H_kv)
    const uint16_t* v_cache;
    const int32_t* block_table;  // [batch][max_pages]
    const int32_t* ctx_lens;     // [batch]
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t nnz, num_pages;
    int32_t batch, heads, heads_kv, max_pages, block_size, nb, num_splits;
    float scale_log2;
    uint16_t* out;   // [batch][H][HD] (num_splits == 1)
    float* lse;      // [batch][H] or null (num_splits == 1)
    float* ws_o;     // [batch][H][splits][HD] partial un-normalised outputs
    float2* ws_ml;   // [batch][H][splits] (max, sum) in the log2 domain
    uint64_t timeout_ns;
    uint32_t* gflags;
};

constexpr int kPage = 16;

template <int HD>
struct DecodeCfg {
    static constexpr int NS = 8;                         // pipeline stages (pages)
    static constexpr uint32_t PAGE_BYTES = kPage * HD * 2;
    static constexpr uint32_t STAGE_BYTES = 2 * PAGE_BYTES;  // K page + V page
    static constexpr uint32_t OFF_BAR = NS * STAGE_BYTES;    // full[NS], empty[NS]
    static constexpr uint32_t OFF_META = OFF_BAR + 2 * NS * 8;
    static constexpr uint32_t OFF_MERGE = OFF_META + NS * 8;  // 4 warps x (HD + 2) floats
    static constexpr uint32_t OFF_MISC = OFF_MERGE + 4 * (HD + 2) * 4;
    // batches of up to LPT_MAX sequences start their longest contexts first
    static constexpr int LPT_MAX = 256;
    static constexpr uint32_t OFF_CTX = OFF_MISC + 32;  // [LPT_MAX] context lengths
    static constexpr uint32_t SMEM = OFF_CTX + LPT_MAX * 4;
    static constexpr int DPL = HD / 32;  // output dims per lane
};

// Pages of key block j visible from a context of n tokens.
__device__ __forceinline__ int block_pages(int j, int bs, int n)
{
    const int t0 = j * bs;
    const int t1 = min(t0 + bs, n);
    return t1 > t0 ? (t1 - t0 + kPage - 1) / kPage : 0;
}

template <int HD>
__global__ void __launch_bounds__(160)
s2_decode_split_kernel(const DecodeParams p)
{
    using C = DecodeCfg<HD>;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sp = blockIdx.x, h = blockIdx.y;
    const int H = p.heads;
    const int hkv = h / (H / p.heads_kv);

    auto bar_full = [&](int st) { return sb + C::OFF_BAR + 8u * st; };
    auto bar_empty = [&](int st) { return sb + C::OFF_BAR + 8u * (C::NS + st); };
    int2* meta = reinterpret_cast<int2*>(smem + C::OFF_META);
    int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);
    volatile int* abort_cta = reinterpret_cast<volatile int*>(misc + 7);

    // Sequence of this CTA. CTAs start in grid order, so with up to LPT_MAX
    // sequences the z-th grid slice takes the sequence with the z-th longest
    // context (ties by index; the ranks are a permutation): the longest
    // page lists start first and short ones fill the last wave. Larger
    // batches keep the index order.
    int s = blockIdx.z;
    if (p.batch <= C::LPT_MAX) {
        int* ctxs = reinterpret_cast<int*>(smem + C::OFF_CTX);
        for (int i = threadIdx.x; i < p.batch; i += blockDim.x) ctxs[i] = p.ctx_lens[i];
        __syncthreads();
        for (int c = threadIdx.x; c < p.batch; c += blockDim.x) {
            const int nc = ctxs[c];
            int rank = 0;
            for (int j = 0; j < p.batch; ++j) {
                const int nj = ctxs[j];
                rank += (nj > nc || (nj == nc && j < c)) ? 1 : 0;
            }
            if (rank == (int)blockIdx.z) misc[5] = c;
        }
        __syncthreads();
        s = misc[5];
    }

    // Work of this CTA: pages [pg0, pg1) of the (s, h) page list.
    if (threadIdx.x == 0) {
        for (int st = 0; st < C::NS; ++st) {
            mbar_init(bar_full(st), 1);
            mbar_init(bar_empty(st), 1);
        }
        *abort_cta = 0;
        const int n = p.ctx_lens[s];
        int ok = n >= 1 && (int64_t)n <= (int64_t)p.max_pages * kPage &&
                 (n - 1) / p.block_size < p.nb;
        int r0 = 0, r1 = 0, total = 0;
        if (ok) {
            const int i = (n - 1) / p.block_size;
            r0 = p.row_ptr[h * (p.nb + 1) + i];
            r1 = p.row_ptr[h * (p.nb + 1) + i + 1];
            ok = r0 >= 0 && r0 <= r1 && r1 <= p.nnz;
        }
        if (ok) {
            const int i = (n - 1) / p.block_size;
            for (int e = r0; e < r1; ++e) {
                const int j = p.col_idx[e];
                if (j < 0 || j > i) { ok = 0; break; }  // every listed block holds >= 1 page
                total += block_pages(j, p.block_size, n);
            }
        }
        if (!ok) {
            atomicOr(p.gflags, kFlagIndex);
            total = 0;
        }
        const int chunk = (total + p.num_splits - 1) / p.num_splits;
        const int pg0 = min(total, sp * chunk), pg1 = min(total, pg0 + chunk);
        misc[0] = n;
        misc[1] = r0;
        misc[2] = r1;
        misc[3] = pg0;
        misc[4] = pg1;
        fence_mbar_init();
    }
    __syncthreads();
    const int n_ctx = misc[0], r0 = misc[1];
    const int pg0 = misc[3], pg1 = misc[4];
    const int cnt = pg1 - pg0;
    const WaitCtl ctl{p.timeout_ns, p.gflags, abort_cta};
    constexpr uint64_t kDrainNs = 200000000ull;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && cnt > 0) {
            // Find the block holding page pg0 of the list.
            int e = r0, skip = pg0, blk_pages = 0;
            for (;;) {
                blk_pages = block_pages(p.col_idx[e], p.block_size, n_ctx);
                if (skip < blk_pages) break;
                skip -= blk_pages;
                ++e;
            }
            int in_blk = skip;
            int n = 0;
            for (; n < cnt; ++n) {
                const int j = p.col_idx[e];
                const int lp = j * (p.block_size / kPage) + in_blk;  // logical page
                const int tok0 = lp * kPage;
                int valid = min(kPage, n_ctx - tok0);
                const int64_t phys = p.block_table[(int64_t)s * p.max_pages + lp];
                if (phys < 0 || phys >= p.num_pages) {
                    atomicOr(p.gflags, kFlagIndex);
                    valid = 0;
                }
                const int st = n % C::NS;
                if (!mbar_wait(bar_empty(st), ((n / C::NS) & 1) ^ 1, ctl)) break;
                meta[st] = make_int2(tok0, valid);
                if (valid > 0) {
                    const int64_t off = ((phys * p.heads_kv + hkv) * kPage) * HD;
                    mbar_arrive_expect_tx(bar_full(st), C::STAGE_BYTES);
                    bulk_load(sb + st * C::STAGE_BYTES, p.k_cache + off, C::PAGE_BYTES, bar_full(st));
                    bulk_load(sb + st * C::STAGE_BYTES + C::PAGE_BYTES, p.v_cache + off, C::PAGE_BYTES,
                              bar_full(st));
                } else {
                    mbar_arrive(bar_full(st));
                }
                if (++in_blk == blk_pages && n + 1 < cnt) {
                    ++e;
                    in_blk = 0;
                    blk_pages = block_pages(p.col_idx[e], p.block_size, n_ctx);
                }
            }
            if (*abort_cta)
                for (int m = (n > C::NS ? n - C::NS : 0); m < n; ++m)
                    mbar_drain(bar_full(m % C::NS), (m / C::NS) & 1, kDrainNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ consumers
        const int cw = warp - 1;
        const int t = lane >> 1, hf = lane & 1;
        // q half of this lane, in the rotated chunk order used for K reads,
        // pre-multiplied by scale * log2(e).
        float qr[HD / 2];
        const uint16_t* qg = p.q + ((int64_t)s * H + h) * HD + hf * (HD / 2);
#pragma unroll
        for (int c = 0; c < HD / 16; ++c) {
            const int cc = (c + t) & (HD / 16 - 1);
            const uint4 v = *reinterpret_cast<const uint4*>(qg + cc * 8);
            qr[8 * c + 0] = bf16lo(v.x) * p.scale_log2;
            qr[8 * c + 1] = bf16hi(v.x) * p.scale_log2;
            qr[8 * c + 2] = bf16lo(v.y) * p.scale_log2;
            qr[8 * c + 3] = bf16hi(v.y) * p.scale_log2;
            qr[8 * c + 4] = bf16lo(v.z) * p.scale_log2;
            qr[8 * c + 5] = bf16hi(v.z) * p.scale_log2;
            qr[8 * c + 6] = bf16lo(v.w) * p.scale_log2;
            qr[8 * c + 7] = bf16hi(v.w) * p.scale_log2;
        }
        float m = -1e30f, l = 0.f, acc[C::DPL];
#pragma unroll
        for (int d = 0; d < C::DPL; ++d) acc[d] = 0.f;

        for (int n = cw; n < cnt; n += 4) {
            const int st = n % C::NS;
            const bool ok = mbar_wait(bar_full(st), (n / C::NS) & 1, ctl);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int2 mt = meta[st];
            const uint8_t* kp = smem + st * C::STAGE_BYTES;
            const uint8_t* vp = kp + C::PAGE_BYTES;
            // score of token t (lane pair)
            float sc = 0.f;
            const uint8_t* krow = kp + t * (HD * 2) + hf * HD;
#pragma unroll
            for (int c = 0; c < HD / 16; ++c) {
                const int cc = (c + t) & (HD / 16 - 1);
                const uint4 v = *reinterpret_cast<const uint4*>(krow + cc * 16);
                sc = fmaf(qr[8 * c + 0], bf16lo(v.x), sc);
                sc = fmaf(qr[8 * c + 1], bf16hi(v.x), sc);
                sc = fmaf(qr[8 * c + 2], bf16lo(v.y), sc);
                sc = fmaf(qr[8 * c + 3], bf16hi(v.y), sc);
                sc = fmaf(qr[8 * c + 4], bf16lo(v.z), sc);
                sc = fmaf(qr[8 * c + 5], bf16hi(v.z), sc);
                sc = fmaf(qr[8 * c + 6], bf16lo(v.w), sc);
                sc = fmaf(qr[8 * c + 7], bf16hi(v.w), sc);
            }
            sc += __shfl_xor_sync(0xffffffffu, sc, 1);
            const float x = t < mt.y ? sc : -INFINITY;
            float mx = x;
#pragma unroll
            for (int o = 16; o >= 2; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m, mx);
            const float alpha = ex2(m - m_new);
            const float pt = ex2(x - m_new);
            float ps = hf == 0 ? pt : 0.f;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l = l * alpha + ps;
            m = m_new;
#pragma unroll
            for (int d = 0; d < C::DPL; ++d) acc[d] *= alpha;
            for (int tt = 0; tt < mt.y; ++tt) {
                const float w = __shfl_sync(0xffffffffu, pt, 2 * tt);
                const uint8_t* vrow = vp + tt * (HD * 2) + lane * (C::DPL * 2);
                if constexpr (C::DPL == 4) {
                    const uint2 v = *reinterpret_cast<const uint2*>(vrow);
                    acc[0] = fmaf(w, bf16lo(v.x), acc[0]);
                    acc[1] = fmaf(w, bf16hi(v.x), acc[1]);
                    acc[2] = fmaf(w, bf16lo(v.y), acc[2]);
                    acc[3] = fmaf(w, bf16hi(v.y), acc[3]);
                } else {
                    const uint32_t v = *reinterpret_cast<const uint32_t*>(vrow);
                    acc[0] = fmaf(w, bf16lo(v), acc[0]);
                    acc[1] = fmaf(w, bf16hi(v), acc[1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty(st));
        }
        // merge the four warps' states
        float* mg = reinterpret_cast<float*>(smem + C::OFF_MERGE) + cw * (HD + 2);
#pragma unroll
        for (int d = 0; d < C::DPL; ++d) mg[lane * C::DPL + d] = acc[d];
        if (lane == 0) {
            mg[HD] = m;
            mg[HD + 1] = l;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (cw == 0) {
            const float* base = reinterpret_cast<const float*>(smem + C::OFF_MERGE);
            float M = -1e30f;
#pragma unroll
            for (int w = 0; w < 4; ++w) M = fmaxf(M, base[w * (HD + 2) + HD]);
            float L = 0.f, o[C::DPL];
#pragma unroll
            for (int d = 0; d < C::DPL; ++d) o[d] = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float f = ex2(base[w * (HD + 2) + HD] - M);
                L += f * base[w * (HD + 2) + HD + 1];
#pragma unroll
                for (int d = 0; d < C::DPL; ++d) o[d] += f * base[w * (HD + 2) + lane * C::DPL + d];
            }
            const int64_t sh = (int64_t)s * H + h;
            if (p.num_splits == 1) {
                const float inv = L > 0.f ? 1.f / L : 0.f;
                uint16_t* og = p.out + sh * HD + lane * C::DPL;
                if constexpr (C::DPL == 4) {
                    uint2 v;
                    v.x = pack_bf16x2(o[0] * inv, o[1] * inv);
                    v.y = pack_bf16x2(o[2] * inv, o[3] * inv);
                    *reinterpret_cast<uint2*>(og) = v;
                } else {
                    *reinterpret_cast<uint32_t*>(og) = pack_bf16x2(o[0] * inv, o[1] * inv);
                }
                if (lane == 0 && p.lse)
                    p.lse[sh] = L > 0.f ? (M + lg2(L)) * 0.69314718055994531f : -INFINITY;
            } else {
                const int64_t part = sh * p.num_splits + sp;
                float* og = p.ws_o + part * HD + lane * C::DPL;
#pragma unroll
                for (int d = 0; d < C::DPL; ++d) og[d] = o[d];
                if (lane == 0) p.ws_ml[part] = make_float2(L > 0.f ? M : -INFINITY, L);
            }
        }
    }
}

// One CTA per (sequence, head), one thread per output dimension.
template <int HD>
__global__ void __launch_bounds__(HD)
s2_decode_combine_kernel(const float* __restrict__ ws_o, const float2* __restrict__ ws_ml,
                         int num_splits, uint16_t* __restrict__ out, float* __restrict__ lse)
{
    const int64_t sh = blockIdx.x;
    const int d = threadIdx.x;
    const float2* ml = ws_ml + sh * num_splits;
    float M = -INFINITY;
    for (int q = 0; q < num_splits; ++q) M = fmaxf(M, ml[q].x);
    float L = 0.f, o = 0.f;
    if (M > -INFINITY) {
        for (int q = 0; q < num_splits; ++q) {
            const float2 v = ml[q];
            if (v.x == -INFINITY) continue;
            const float f = ex2(v.x - M);
            L += f * v.y;
            o += f * ws_o[(sh * num_splits + q) * HD + d];
        }
    }
    const float r = L > 0.f ? o / L : 0.f;
    out[sh * HD + d] = (uint16_t)(pack_bf16x2(r, 0.f) & 0xffffu);
    if (d == 0 && lse) lse[sh] = L > 0.f ? (M + lg2(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace s2
