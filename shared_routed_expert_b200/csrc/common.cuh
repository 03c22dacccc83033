// Device helpers shared by the layer's kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace sre {

// Device status word layout at the start of the workspace.
struct DevStatus {
    unsigned int code;      // 0 ok, else a moe_status value
    unsigned int info;      // first offending index / wait site
    unsigned int timeouts;  // number of waits that ran out
    unsigned int pad[61];
};
static_assert(sizeof(DevStatus) == 256, "status block is 256 bytes");

__device__ __forceinline__ void report(DevStatus* st, unsigned code, unsigned info) {
    if (st == nullptr) return;
    if (atomicCAS(&st->code, 0u, code) == 0u) st->info = info;
    if (code == MOE_ERR_TIMEOUT) atomicAdd(&st->timeouts, 1u);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

// two floats -> packed bf16x2 (low half = a)
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __nv_fp8_e4m3 v;
    v.__x = c;
    return static_cast<float>(v);
}


// Power-of-two exponent k for a chunk whose largest magnitude is amax, so that
// amax * 2^-k lies in [2^14, 2^15) (fp16 keeps 11 significant bits there and
// cannot overflow). k is clamped to [-100, 113]; amax = 0 gives k = 0.
__device__ __forceinline__ int f16_chunk_exp(float amax) {
    if (!(amax > 0.0f)) return 0;
    const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
    return max(-100, min(113, ex - 14));
}

__device__ __forceinline__ float exp2_int(int k) {   // 2^k for k in [-126, 127]
    return __uint_as_float(static_cast<uint32_t>(127 + k) << 23);
}

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t v) {
    return __half22float2(*reinterpret_cast<__half2*>(&v));
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + __expf(-g)); }

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace sre
