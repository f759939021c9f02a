// umma.cuh -- parameters of the prefill kernel and the sm_100 UMMA descriptors
// (shared-memory matrix descriptor and instruction descriptor) it issues.
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
    int32_t batch, heads, heads_kv, seq, nb, nqt;  // query head h reads K/V head h / (heads / heads_kv)
    float scale_log2;  // scale * log2(e)
    uint64_t timeout_ns;
    uint32_t* gflags;
    int* sched;    // work-counter slot of this launch (sched_claim / sched_take / sched_leave)
    int sched_id;  // this launch's nonzero id
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

}  // namespace s2
