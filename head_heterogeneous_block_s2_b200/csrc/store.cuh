// store.cuh -- bf16 row stores for the epilogues (one thread writes one row of
// its TMEM lane).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace s2 {

// Scales N fp32 values (bit patterns in o) by f, rounds them to bf16 and stores
// them at dst (N a multiple of 16, dst 16-byte aligned): 32-byte stores (whole
// L2 sectors, half the store instructions) when st32 says dst is 32-byte
// aligned, else 16-byte ones.
template <int N>
__device__ __forceinline__ void store_bf16_row(uint16_t* dst, const uint32_t* o, float f, bool st32)
{
#pragma unroll
    for (int e = 0; e < N; e += 16) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i] = pack_bf16x2(__uint_as_float(o[e + 2 * i]) * f, __uint_as_float(o[e + 2 * i + 1]) * f);
        if (st32) {
            st_global_v8(dst + e, w);
        } else {
            *reinterpret_cast<uint4*>(dst + e) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(dst + e + 8) = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

}  // namespace s2
