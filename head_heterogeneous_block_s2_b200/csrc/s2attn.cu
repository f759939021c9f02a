// s2attn.cu -- C ABI of the HHST sparse-attention library (see include/s2attn.h).
//
// Host side of the prefill, decode and backward paths: argument validation, TMA tensor
// maps (encoded through the driver entry point, so the library does not link
// libcuda and loads on machines without a GPU), launches, and the device
// error flags shared by all kernels of this translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "s2attn.h"
#include "ptx.cuh"
#include "backward_sm100.cuh"
#include "chunk_sm100.cuh"
#include "decode.cuh"
#include "prefill_pair_sm100.cuh"

namespace {

__device__ uint32_t g_s2_flags;

// Work counters of the persistent kernels (prefill, chunked prefill, and the
// backward's dQ and 64-key dK/dV kernels): a ring of slots {owner, next item,
// CTAs done, unused}. Each launch gets the next slot in turn and a nonzero id;
// its CTAs claim the slot before taking items and the last one frees it, so a
// slot reused while an earlier launch still holds it makes the new launch
// wait for that one (see sched_claim), never share its counters.
constexpr int kSchedSlots = 1024;
__device__ int g_s2_sched[s2::kSchedWords * kSchedSlots];
std::atomic<uint32_t> g_launch_seq{0};


std::atomic<uint64_t> g_timeout_ns{2000000000ull};

constexpr int kMaxDevices = 64;
struct DevInfo {
    int checked = 0;  // 0 unknown, 1 sm_100, -1 other
    int num_sms = 0;
    uint32_t* flags = nullptr;
    int* sched = nullptr;
    bool prefill_attr_done[4] = {false, false, false, false};
    bool decode_attr_done[2] = {false, false};
    bool backward_attr_done[4] = {false, false, false, false};
    bool chunk_attr_done[4] = {false, false, false, false};
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

// The slot and id of the next persistent launch on device `dev`.
int* next_sched(int dev, int* id)
{
    const uint32_t s = g_launch_seq.fetch_add(1);
    *id = (int)(s % 0x7ffffffeu) + 1;
    return g_dev[dev].sched + s2::kSchedWords * (int)(s % kSchedSlots);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Device checks, once per device: compute capability 10.x and the address of
// the error flags.
int device_ready(int* dev_out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return S2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return S2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& d = g_dev[dev];
    if (d.checked == 0) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return S2_ERR_CUDA;
        if (major != 10) {
            d.checked = -1;
        } else {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_s2_flags) != cudaSuccess) return S2_ERR_CUDA;
            d.flags = static_cast<uint32_t*>(p);
            void* q = nullptr;
            if (cudaGetSymbolAddress(&q, g_s2_sched) != cudaSuccess) return S2_ERR_CUDA;
            d.sched = static_cast<int*>(q);
            d.num_sms = sms;
            d.checked = 1;
        }
    }
    if (d.checked != 1) return S2_ERR_UNSUPPORTED;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return S2_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    *dev_out = dev;
    return S2_OK;
}

// 2-D bf16 tensor map over [rows][cols], box [box_rows][64], SWIZZLE_128B.
// 3-D bf16 tensor map over [planes][seq][cols] (cols innermost), 64-column
// SWIZZLE_128B boxes of box_rows rows; rows at or past seq read as zeros.
int make_map(CUtensorMap* m, const void* base, uint64_t planes, uint64_t seq, uint64_t cols,
             uint32_t box_rows)
{
    const cuuint64_t dims[3] = {cols, seq, planes};
    const cuuint64_t strides[2] = {cols * 2, seq * cols * 2};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? S2_OK : S2_ERR_CUDA;
}

// Packed chunk rows [rows][heads][cols]: one head's 128 consecutive rows per box.
int make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads, uint64_t cols)
{
    const cuuint64_t dims[3] = {cols, heads, rows};
    const cuuint64_t strides[2] = {cols * 2, heads * cols * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? S2_OK : S2_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The logits' multiplier: 0 selects 1/sqrt(head_dim). Returns false for a
// non-finite value, and for a negative one where `positive` is required (the
// prefill-type kernels take the row maximum of the unscaled logits).
bool resolve_scale(float& scale, int32_t head_dim, bool positive)
{
    if (!std::isfinite(scale)) return false;
    if (scale == 0.f) scale = 1.0f / std::sqrt((float)head_dim);
    return !positive || scale > 0.f;
}

template <int HD, int BK>
int launch_prefill(const void* q, const void* k, const void* v, s2::PrefillParams& pp, int dev,
                   int attr_slot, cudaStream_t stream)
{
    using C = s2::PairCfg<HD, BK>;
    const uint64_t qplanes = (uint64_t)pp.batch * pp.heads, kvplanes = (uint64_t)pp.batch * pp.heads_kv;
    CUtensorMap mq, mk, mv;
    if (make_map(&mq, q, qplanes, pp.seq, HD, 128) || make_map(&mk, k, kvplanes, pp.seq, HD, BK) ||
        make_map(&mv, v, kvplanes, pp.seq, HD, BK))
        return S2_ERR_CUDA;
    auto kern = s2::s2_prefill_pair_kernel<HD, BK>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].prefill_attr_done[attr_slot]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::SMEM_ALLOC) != cudaSuccess)
                return S2_ERR_CUDA;

            g_dev[dev].prefill_attr_done[attr_slot] = true;
        }
    }
    // Persistent: one CTA per SM (one fits by shared memory), each walking a
    // static share of the tile pairs.
    const uint64_t items = (uint64_t)pp.batch * pp.heads * ((pp.nqt + 1) / 2);
    const uint64_t grid = items < (uint64_t)g_dev[dev].num_sms ? items : (uint64_t)g_dev[dev].num_sms;
    kern<<<(unsigned)grid, C::THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv, pp);
    return cudaGetLastError() == cudaSuccess ? S2_OK : S2_ERR_CUDA;
}

// Backward: row statistics, then the dQ kernel and the dK/dV kernel (neither
// writes what the other reads). The dQ kernel is persistent; so is the dK/dV
// kernel for 64-key blocks (one CTA per 128-row key tile for 128-key blocks).
template <int HD, int BK>
int launch_backward(const void* q, const void* k, const void* v, s2::BackwardParams& bp, int dev,
                    int attr_slot, cudaStream_t stream)
{
    using CQ = s2::BwdQCfg<HD, BK>;
    using CK = s2::BwdKVCfg<HD, BK>;
    using CKP = s2::BwdKVPCfg<HD>;
    const uint64_t planes = (uint64_t)bp.batch * bp.heads, kvplanes = (uint64_t)bp.batch * bp.heads_kv;
    CUtensorMap q128, do128, kbk, vbk, qbk, dobk;
    if (make_map(&q128, q, planes, bp.seq, HD, 128) || make_map(&do128, bp.dout, planes, bp.seq, HD, 128) ||
        make_map(&kbk, k, kvplanes, bp.seq, HD, BK) || make_map(&vbk, v, kvplanes, bp.seq, HD, BK) ||
        make_map(&qbk, q, planes, bp.seq, HD, BK) || make_map(&dobk, bp.dout, planes, bp.seq, HD, BK))
        return S2_ERR_CUDA;
    auto kq = s2::s2_bwd_dq_kernel<HD, BK>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].backward_attr_done[attr_slot]) {
            cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, CQ::SMEM_ALLOC);
            if constexpr (BK == 64)
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(s2::s2_bwd_dkv_persistent_kernel<HD>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, CKP::SMEM_ALLOC);
            if constexpr (BK != 64)
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(s2::s2_bwd_dkv_kernel<HD, BK>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, CK::SMEM_ALLOC);
            if (e != cudaSuccess) return S2_ERR_CUDA;
            g_dev[dev].backward_attr_done[attr_slot] = true;
        }
    }
    const int64_t rows = (int64_t)planes * bp.seq_pad;
    const int64_t rows_per_cta = 256 / (HD / 8);
    int64_t grid0 = (rows + rows_per_cta - 1) / rows_per_cta;
    if (grid0 > (int64_t)g_dev[dev].num_sms * 16) grid0 = (int64_t)g_dev[dev].num_sms * 16;
    s2::s2_bwd_stats_kernel<HD><<<(unsigned)grid0, 256, 0, stream>>>(bp);
    if (cudaGetLastError() != cudaSuccess) return S2_ERR_CUDA;
    // dQ: persistent, at most one CTA per SM (work counter slot in bp.sched)
    const uint64_t qitems = planes * (uint64_t)bp.ntiles;
    const uint64_t qgrid = qitems < (uint64_t)g_dev[dev].num_sms ? qitems : (uint64_t)g_dev[dev].num_sms;
    kq<<<(unsigned)qgrid, 384, CQ::SMEM_ALLOC, stream>>>(q128, do128, kbk, vbk, bp);
    if (cudaGetLastError() != cudaSuccess) return S2_ERR_CUDA;
    const uint64_t kvitems = kvplanes * (uint64_t)bp.ntiles;
    if constexpr (BK == 64) {  // persistent, at most one CTA per SM (work counter slot in bp.sched_kv)
        const uint64_t kvgrid = kvitems < (uint64_t)g_dev[dev].num_sms ? kvitems : (uint64_t)g_dev[dev].num_sms;
        s2::s2_bwd_dkv_persistent_kernel<HD>
            <<<(unsigned)kvgrid, 384, CKP::SMEM_ALLOC, stream>>>(qbk, dobk, kbk, vbk, bp);
    } else {
        s2::s2_bwd_dkv_kernel<HD, BK><<<(unsigned)kvitems, 384, CK::SMEM_ALLOC, stream>>>(qbk, dobk, kbk, vbk, bp);
    }
    return cudaGetLastError() == cudaSuccess ? S2_OK : S2_ERR_CUDA;
}

// Chunked prefill: persistent CTAs over (sequence, head, tile pair) items.
template <int HD, int BK>
int launch_chunk(const void* q, const void* kc, const void* vc, s2::ChunkParams& cp, int dev, int attr_slot,
                 cudaStream_t stream)
{
    using C = s2::ChunkCfg<HD, BK>;
    CUtensorMap mq, mk, mv;
    const uint64_t planes = (uint64_t)cp.num_pages * cp.heads_kv;
    if (make_rows_map(&mq, q, (uint64_t)cp.total_q, cp.heads, HD) ||
        make_map(&mk, kc, planes, s2::kChunkPage, HD, s2::kChunkPage) ||
        make_map(&mv, vc, planes, s2::kChunkPage, HD, s2::kChunkPage))
        return S2_ERR_CUDA;
    auto kern = s2::s2_chunk_prefill_kernel<HD, BK>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].chunk_attr_done[attr_slot]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) !=
                cudaSuccess)
                return S2_ERR_CUDA;
            g_dev[dev].chunk_attr_done[attr_slot] = true;
        }
    }
    // Persistent: at most one CTA per SM; the kernel counts the items (tile
    // pairs x heads) from the device-side chunk metadata, bounded here by the
    // largest chunk (a chunk of L rows spans at most L / 128 + 2 tiles).
    const uint64_t pairs_max = ((uint64_t)(cp.max_q_len + 127) / 128 + 2) / 2;
    const uint64_t items = (uint64_t)cp.batch * cp.heads * pairs_max;
    const uint64_t grid = items < (uint64_t)g_dev[dev].num_sms ? items : (uint64_t)g_dev[dev].num_sms;
    kern<<<(unsigned)grid, 384, C::SMEM_ALLOC, stream>>>(mq, mk, mv, cp);
    return cudaGetLastError() == cudaSuccess ? S2_OK : S2_ERR_CUDA;
}

template <int HD>
int launch_decode(s2::DecodeParams& dp, int dev, cudaStream_t stream)
{
    using C = s2::DecodeCfg<HD>;
    auto kern = s2::s2_decode_split_kernel<HD>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        const int slot = HD == 128 ? 1 : 0;
        if (!g_dev[dev].decode_attr_done[slot]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
                cudaSuccess)
                return S2_ERR_CUDA;
            g_dev[dev].decode_attr_done[slot] = true;
        }
    }
    dim3 grid(dp.num_splits, dp.heads, dp.batch);
    kern<<<grid, 160, C::SMEM, stream>>>(dp);
    if (cudaGetLastError() != cudaSuccess) return S2_ERR_CUDA;
    if (dp.num_splits > 1) {
        s2::s2_decode_combine_kernel<HD><<<(unsigned)(dp.batch * dp.heads), HD, 0, stream>>>(
            dp.ws_o, dp.ws_ml, dp.num_splits, dp.out, dp.lse);
        if (cudaGetLastError() != cudaSuccess) return S2_ERR_CUDA;
    }
    return S2_OK;
}

constexpr int kMaxSplits = 64;

size_t ws_bytes(int64_t batch, int64_t heads, int64_t head_dim, int64_t splits)
{
    if (splits <= 1) return 0;
    const size_t o = (size_t)(batch * heads * splits * head_dim) * sizeof(float);
    const size_t o_pad = (o + 255) & ~size_t(255);
    return o_pad + (size_t)(batch * heads * splits) * sizeof(float2);
}

}  // namespace

extern "C" {

const char* s2_status_string(int status)
{
    switch (status) {
    case S2_OK: return "S2_OK";
    case S2_ERR_INVALID_ARG: return "S2_ERR_INVALID_ARG";
    case S2_ERR_UNSUPPORTED: return "S2_ERR_UNSUPPORTED";
    case S2_ERR_CAPACITY: return "S2_ERR_CAPACITY";
    case S2_ERR_CUDA: return "S2_ERR_CUDA";
    case S2_ERR_TIMEOUT: return "S2_ERR_TIMEOUT";
    case S2_ERR_DEVICE_INDEX: return "S2_ERR_DEVICE_INDEX";
    default: return "S2_ERR_UNKNOWN";
    }
}

const char* s2_version(void) { return "s2attn-b200 0.1 (sm_100a)"; }

int s2_set_wait_timeout_ns(uint64_t ns)
{
    g_timeout_ns.store(ns);
    return S2_OK;
}

int s2_device_status(int reset, uint32_t* flags_out)
{
    int dev = 0;
    const int rc = device_ready(&dev);
    if (rc) return rc;
    uint32_t f = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return S2_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&f, g_s2_flags, sizeof f) != cudaSuccess) return S2_ERR_CUDA;
    if (reset) {
        const uint32_t z = 0;
        if (cudaMemcpyToSymbol(g_s2_flags, &z, sizeof z) != cudaSuccess) return S2_ERR_CUDA;
        // After a timeout a work-counter slot may still be held by a launch whose
        // CTAs did not all claim it; with the device idle every slot is free.
        if ((f & s2::kFlagTimeout) &&
            (cudaMemset(g_dev[dev].sched, 0, sizeof(int) * s2::kSchedWords * kSchedSlots) != cudaSuccess ||
             cudaDeviceSynchronize() != cudaSuccess))
            return S2_ERR_CUDA;
    }
    if (flags_out) *flags_out = f;
    if (f & s2::kFlagTimeout) return S2_ERR_TIMEOUT;
    if (f & s2::kFlagIndex) return S2_ERR_DEVICE_INDEX;
    return S2_OK;
}

int s2_attn_prefill_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                        int32_t batch, int32_t heads, int32_t heads_kv, int32_t seq,
                        int32_t head_dim, float scale, int32_t block_size, int32_t num_blocks,
                        const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz, void* stream)
{
    if (!q || !k || !v || !o || !row_ptr || (!col_idx && nnz > 0)) return S2_ERR_INVALID_ARG;
    if (batch < 1 || heads < 1 || seq < 1 || nnz < 0 || !resolve_scale(scale, head_dim, true))
        return S2_ERR_INVALID_ARG;
    if (heads_kv < 1 || heads % heads_kv != 0) return S2_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return S2_ERR_UNSUPPORTED;
    if (block_size != 64 && block_size != 128) return S2_ERR_UNSUPPORTED;
    if (num_blocks > 2046) return S2_ERR_UNSUPPORTED;  // union lists are staged in shared memory
    if (num_blocks != (seq + block_size - 1) / block_size) return S2_ERR_INVALID_ARG;
    // work items are counted in int on the device
    if ((int64_t)batch * heads * (((seq + 127) / 128 + 1) / 2) >= (int64_t)(INT32_MAX / 2))
        return S2_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return S2_ERR_INVALID_ARG;
    int dev = 0;
    int rc = device_ready(&dev);
    if (rc) return rc;

    s2::PrefillParams pp;
    pp.row_ptr = row_ptr;
    pp.col_idx = col_idx;
    pp.nnz = nnz;
    pp.o = static_cast<uint16_t*>(o);
    pp.lse = lse;
    pp.batch = batch;
    pp.heads = heads;
    pp.heads_kv = heads_kv;
    pp.seq = seq;
    pp.nb = num_blocks;
    pp.nqt = (seq + 127) / 128;
    pp.scale_log2 = scale * 1.4426950408889634f;
    pp.timeout_ns = g_timeout_ns.load();
    pp.gflags = g_dev[dev].flags;
    pp.sched = next_sched(dev, &pp.sched_id);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128 && block_size == 128) return launch_prefill<128, 128>(q, k, v, pp, dev, 0, st);
    if (head_dim == 128 && block_size == 64) return launch_prefill<128, 64>(q, k, v, pp, dev, 1, st);
    if (head_dim == 64 && block_size == 128) return launch_prefill<64, 128>(q, k, v, pp, dev, 2, st);
    return launch_prefill<64, 64>(q, k, v, pp, dev, 3, st);
}

size_t s2_attn_backward_workspace_size(int32_t batch, int32_t heads, int32_t seq)
{
    if (batch < 1 || heads < 1 || seq < 1) return 0;
    const int64_t seq_pad = ((int64_t)seq + 127) / 128 * 128;
    return (size_t)((int64_t)batch * heads * seq_pad * 8);
}

int s2_attn_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int32_t batch, int32_t heads,
                     int32_t heads_kv, int32_t seq, int32_t head_dim, float scale,
                     int32_t block_size, int32_t num_blocks, const int32_t* row_ptr,
                     const int32_t* col_idx, const int32_t* col_ptr, const int32_t* row_idx,
                     const int32_t* key_tiles, int64_t nnz, void* workspace,
                     size_t workspace_bytes, void* stream)
{
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !row_ptr || !col_ptr ||
        ((!col_idx || !row_idx) && nnz > 0) || !workspace || (block_size == 64 && !key_tiles))
        return S2_ERR_INVALID_ARG;
    if (batch < 1 || heads < 1 || seq < 1 || nnz < 0 || !resolve_scale(scale, head_dim, true))
        return S2_ERR_INVALID_ARG;
    if (heads_kv < 1 || heads % heads_kv != 0) return S2_ERR_INVALID_ARG;
    // grouped heads: a key tile walks every query head's list of its group (tags of 4 bits)
    if (heads / heads_kv > 16 || (heads != heads_kv && (int64_t)(heads / heads_kv) * num_blocks > 4096))
        return S2_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return S2_ERR_UNSUPPORTED;
    if (block_size != 64 && block_size != 128) return S2_ERR_UNSUPPORTED;
    if (num_blocks > 2046) return S2_ERR_UNSUPPORTED;  // union lists are staged in shared memory
    if (num_blocks != (seq + block_size - 1) / block_size) return S2_ERR_INVALID_ARG;
    const int64_t ntiles = ((int64_t)seq + 127) / 128;
    if ((int64_t)batch * heads * ntiles >= (int64_t)INT32_MAX) return S2_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return S2_ERR_INVALID_ARG;
    if (workspace_bytes < s2_attn_backward_workspace_size(batch, heads, seq)) return S2_ERR_CAPACITY;
    int dev = 0;
    int rc = device_ready(&dev);
    if (rc) return rc;

    s2::BackwardParams bp;
    bp.row_ptr = row_ptr;
    bp.col_idx = col_idx;
    bp.col_ptr = col_ptr;
    bp.row_idx = row_idx;
    bp.key_tiles = key_tiles;
    bp.nnz = nnz;
    bp.o = static_cast<const uint16_t*>(o);
    bp.dout = static_cast<const uint16_t*>(dout);
    bp.lse = lse;
    bp.stats = static_cast<float*>(workspace);
    bp.dq = static_cast<uint16_t*>(dq);
    bp.dk = static_cast<uint16_t*>(dk);
    bp.dv = static_cast<uint16_t*>(dv);
    bp.batch = batch;
    bp.heads = heads;
    bp.heads_kv = heads_kv;
    bp.seq = seq;
    bp.seq_pad = (int32_t)(ntiles * 128);
    bp.nb = num_blocks;
    bp.ntiles = (int32_t)ntiles;
    bp.scale = scale;
    bp.scale_log2 = scale * 1.4426950408889634f;
    bp.timeout_ns = g_timeout_ns.load();
    bp.gflags = g_dev[dev].flags;
    bp.sched = next_sched(dev, &bp.sched_id);
    bp.sched_kv = next_sched(dev, &bp.sched_kv_id);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128 && block_size == 128) return launch_backward<128, 128>(q, k, v, bp, dev, 0, st);
    if (head_dim == 128 && block_size == 64) return launch_backward<128, 64>(q, k, v, bp, dev, 1, st);
    if (head_dim == 64 && block_size == 128) return launch_backward<64, 128>(q, k, v, bp, dev, 2, st);
    return launch_backward<64, 64>(q, k, v, bp, dev, 3, st);
}

int s2_attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                    int32_t batch, int32_t heads, int32_t seq, int32_t head_dim, float scale,
                    int32_t block_size, int32_t num_blocks, const int32_t* row_ptr,
                    const int32_t* col_idx, int64_t nnz, void* stream)
{
    return s2_attn_prefill_gqa(q, k, v, o, lse, batch, heads, heads, seq, head_dim, scale,
                               block_size, num_blocks, row_ptr, col_idx, nnz, stream);
}

int s2_attn_chunk_prefill(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_table, const int32_t* ctx_lens, const int32_t* q_start,
                          int32_t batch, int32_t heads, int32_t heads_kv, int32_t head_dim,
                          int32_t page_size, int32_t max_pages, int64_t num_pages, int32_t max_q_len,
                          int64_t total_q, int32_t block_size, int32_t num_blocks,
                          const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz, float scale,
                          void* out, float* lse, void* stream)
{
    if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !q_start || !row_ptr ||
        (!col_idx && nnz > 0) || !out)
        return S2_ERR_INVALID_ARG;
    if (batch < 1 || heads < 1 || max_pages < 1 || num_pages < 1 || num_blocks < 1 || nnz < 0 ||
        max_q_len < 1 || total_q < 1 || !resolve_scale(scale, head_dim, true))
        return S2_ERR_INVALID_ARG;
    if (heads_kv < 1 || heads % heads_kv != 0) return S2_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return S2_ERR_UNSUPPORTED;
    if (page_size != s2::kChunkPage) return S2_ERR_UNSUPPORTED;
    if (block_size != 64 && block_size != 128) return S2_ERR_UNSUPPORTED;
    if (num_blocks > 2046) return S2_ERR_UNSUPPORTED;  // union lists are staged in shared memory
    if (batch > 65535 || heads > 65535 || total_q >= INT32_MAX / 2 || max_q_len > (1 << 24))
        return S2_ERR_UNSUPPORTED;
    if (num_pages * heads_kv >= (int64_t)INT32_MAX) return S2_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return S2_ERR_INVALID_ARG;
    int dev = 0;
    int rc = device_ready(&dev);
    if (rc) return rc;
    s2::ChunkParams cp;
    cp.row_ptr = row_ptr;
    cp.col_idx = col_idx;
    cp.nnz = nnz;
    cp.block_table = block_table;
    cp.ctx_lens = ctx_lens;
    cp.q_start = q_start;
    cp.out = static_cast<uint16_t*>(out);
    cp.lse = lse;
    cp.num_pages = num_pages;
    cp.total_q = total_q;
    cp.batch = batch;
    cp.heads = heads;
    cp.heads_kv = heads_kv;
    cp.max_pages = max_pages;
    cp.nb = num_blocks;
    cp.max_q_len = max_q_len;
    cp.scale_log2 = scale * 1.4426950408889634f;
    cp.timeout_ns = g_timeout_ns.load();
    cp.gflags = g_dev[dev].flags;
    cp.sched = next_sched(dev, &cp.sched_id);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128 && block_size == 128) return launch_chunk<128, 128>(q, k_cache, v_cache, cp, dev, 0, st);
    if (head_dim == 128 && block_size == 64) return launch_chunk<128, 64>(q, k_cache, v_cache, cp, dev, 1, st);
    if (head_dim == 64 && block_size == 128) return launch_chunk<64, 128>(q, k_cache, v_cache, cp, dev, 2, st);
    return launch_chunk<64, 64>(q, k_cache, v_cache, cp, dev, 3, st);
}

int32_t s2_attn_decode_auto_splits(int32_t batch, int32_t heads)
{
    if (batch < 1 || heads < 1) return 1;
    // About one wave of resident CTAs (148 SMs x ~2.5): the split kernel starts
    // the longest contexts first, so the short ones even out the last wave and
    // more splits only add partials to merge. Measured on 32 heads, contexts
    // U[4096, 32768] (active K+V GB/s, one launch after an L2 flush), the best
    // counts were 3 at batch 4, 2 at batch 8 and 1 at batches 16, 32 and 64;
    // this rule gives exactly those.
    const int64_t bh = (int64_t)batch * heads;
    const int64_t target = 370;
    int64_t sp = (target + bh - 1) / bh;
    if (sp < 1) sp = 1;
    if (sp > 16) sp = 16;
    return (int32_t)sp;
}

size_t s2_attn_decode_workspace_size(int32_t batch, int32_t heads, int32_t head_dim,
                                     int32_t num_splits)
{
    if (batch < 1 || heads < 1 || head_dim < 1) return 0;
    const int32_t sp = num_splits > 0 ? num_splits : s2_attn_decode_auto_splits(batch, heads);
    return ws_bytes(batch, heads, head_dim, sp);
}

int s2_attn_decode_gqa(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_table, const int32_t* ctx_lens, int32_t batch,
                       int32_t heads, int32_t heads_kv, int32_t head_dim, int32_t page_size,
                       int32_t max_pages, int64_t num_pages, int32_t block_size,
                       int32_t num_blocks, const int32_t* row_ptr, const int32_t* col_idx,
                       int64_t nnz, float scale, void* out, float* lse, void* workspace,
                       size_t workspace_bytes, int32_t num_splits, void* stream)
{
    if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !row_ptr ||
        (!col_idx && nnz > 0) || !out)
        return S2_ERR_INVALID_ARG;
    if (batch < 1 || heads < 1 || max_pages < 1 || num_pages < 1 || num_blocks < 1 || nnz < 0 ||
        !resolve_scale(scale, head_dim, false) || num_splits > kMaxSplits)
        return S2_ERR_INVALID_ARG;
    if (heads_kv < 1 || heads % heads_kv != 0) return S2_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return S2_ERR_UNSUPPORTED;
    if (page_size != s2::kPage) return S2_ERR_UNSUPPORTED;
    if (block_size < page_size || block_size % page_size != 0) return S2_ERR_UNSUPPORTED;
    if (batch > 65535 || heads > 65535) return S2_ERR_UNSUPPORTED;
    if (num_pages * heads_kv * page_size * head_dim >= (int64_t)1 << 62) return S2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return S2_ERR_INVALID_ARG;
    const int32_t sp = num_splits > 0 ? num_splits : s2_attn_decode_auto_splits(batch, heads);
    const size_t need = ws_bytes(batch, heads, head_dim, sp);
    if (need > 0) {
        if (!workspace) return S2_ERR_INVALID_ARG;
        if (workspace_bytes < need) return S2_ERR_CAPACITY;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return S2_ERR_INVALID_ARG;
    }
    int dev = 0;
    int rc = device_ready(&dev);
    if (rc) return rc;

    s2::DecodeParams dp;
    dp.q = static_cast<const uint16_t*>(q);
    dp.k_cache = static_cast<const uint16_t*>(k_cache);
    dp.v_cache = static_cast<const uint16_t*>(v_cache);
    dp.block_table = block_table;
    dp.ctx_lens = ctx_lens;
    dp.row_ptr = row_ptr;
    dp.col_idx = col_idx;
    dp.nnz = nnz;
    dp.num_pages = num_pages;
    dp.batch = batch;
    dp.heads = heads;
    dp.heads_kv = heads_kv;
    dp.max_pages = max_pages;
    dp.block_size = block_size;
    dp.nb = num_blocks;
    dp.num_splits = sp;
    dp.scale_log2 = scale * 1.4426950408889634f;
    dp.out = static_cast<uint16_t*>(out);
    dp.lse = lse;
    const size_t o_bytes = ((size_t)batch * heads * sp * head_dim * sizeof(float) + 255) & ~size_t(255);
    dp.ws_o = need ? static_cast<float*>(workspace) : nullptr;
    dp.ws_ml = need ? reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + o_bytes) : nullptr;
    dp.timeout_ns = g_timeout_ns.load();
    dp.gflags = g_dev[dev].flags;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return head_dim == 128 ? launch_decode<128>(dp, dev, st) : launch_decode<64>(dp, dev, st);
}

int s2_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_table, const int32_t* ctx_lens, int32_t batch,
                   int32_t heads, int32_t head_dim, int32_t page_size, int32_t max_pages,
                   int64_t num_pages, int32_t block_size, int32_t num_blocks,
                   const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz, float scale,
                   void* out, float* lse, void* workspace, size_t workspace_bytes,
                   int32_t num_splits, void* stream)
{
    return s2_attn_decode_gqa(q, k_cache, v_cache, block_table, ctx_lens, batch, heads, heads,
                              head_dim, page_size, max_pages, num_pages, block_size, num_blocks,
                              row_ptr, col_idx, nnz, scale, out, lse, workspace, workspace_bytes,
                              num_splits, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- decode without allocation
//
// s2_attn_decode_noalloc: the same split-KV decode, but its split partials go
// to a scratch array that lives in this library's own device image instead of
// a caller-supplied workspace. Meant for callers that cannot allocate device
// memory themselves (see the header). The array is a file-scope device
// variable: every GPU that loads the library holds S2_NOALLOC_SCRATCH_BYTES of
// it until the process exits, and all calls share it.
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[S2_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device. In host code the symbol
// name is only a host-side stand-in, so the real address is looked up once
// per device (with that device current) and passed to the kernels.
void* g_noalloc_addr[kMaxDevices] = {};

int noalloc_scratch(int dev, void** out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return S2_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return S2_OK;
}

}  // namespace

extern "C" int s2_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_table, const int32_t* ctx_lens,
                                      int32_t batch, int32_t heads, int32_t head_dim,
                                      int32_t page_size, int32_t max_pages, int64_t num_pages,
                                      int32_t block_size, int32_t num_blocks,
                                      const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                                      float scale, void* out, float* lse, int32_t num_splits,
                                      void* stream)
{
    if (batch < 1 || heads < 1 || num_splits > kMaxSplits) return S2_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return S2_ERR_UNSUPPORTED;
    const int32_t sp = num_splits > 0 ? num_splits : s2_attn_decode_auto_splits(batch, heads);
    if (ws_bytes(batch, heads, head_dim, sp) > S2_NOALLOC_SCRATCH_BYTES) return S2_ERR_CAPACITY;
    int dev = 0;
    int rc = device_ready(&dev);
    if (rc) return rc;
    void* scratch = nullptr;
    rc = noalloc_scratch(dev, &scratch);
    if (rc) return rc;
    // Nothing in the scratch has to start at zero: the split kernel writes
    // every partial (max, sum, output) that the combine kernel then reads.
    return s2_attn_decode(q, k_cache, v_cache, block_table, ctx_lens, batch, heads, head_dim,
                          page_size, max_pages, num_pages, block_size, num_blocks, row_ptr,
                          col_idx, nnz, scale, out, lse, scratch, S2_NOALLOC_SCRATCH_BYTES, sp,
                          stream);
}
