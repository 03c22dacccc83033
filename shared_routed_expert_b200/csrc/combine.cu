// Weighted aggregation of the expert outputs.
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1: all expert
// outputs are aggregated with weights. With the fusion the shared expert is
// slot K of every token (weight shared_weight), so one weighted sum over the
// S = K + 1 slots gives the layer output:
//     out[t] = sum_{k<S} w[t,k] * y[inv[t*S + k]]
// accumulated in fp32 in slot order and rounded once to the output dtype
// (the moe_combine entry point, over expert rows y). moe_forward does the same
// sum inside the down-projection's epilogue and only needs round_rows here.
// `add` (weight add_w) is an optional extra [T, H] term added last.
#include <algorithm>

#include "kernels.cuh"

namespace sre {

namespace {

constexpr int CB_THREADS = 128;

// bf16 rows: each thread owns 8-element vectors of the token's row.
__global__ void __launch_bounds__(CB_THREADS) combine_bf16_kernel(int T, int S, int H,
                                                                  const uint4* __restrict__ y,
                                                                  const int32_t* __restrict__ inv,
                                                                  const float* __restrict__ w,
                                                                  const uint4* __restrict__ add,
                                                                  float add_w,
                                                                  uint4* __restrict__ out) {
    const int t = blockIdx.x;
    const int nv = H / 8;
    __shared__ int32_t s_row[64];
    __shared__ float s_w[64];
    for (int k = threadIdx.x; k < S; k += blockDim.x) {
        s_row[k] = inv[static_cast<size_t>(t) * S + k];
        s_w[k] = w[static_cast<size_t>(t) * S + k];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
        for (int k = 0; k < S; ++k) {
            const uint4 q = y[static_cast<size_t>(s_row[k]) * nv + i];
            const float wk = s_w[k];
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[2 * j] = __fmaf_rn(wk, __uint_as_float(u[j] << 16), acc[2 * j]);
                acc[2 * j + 1] = __fmaf_rn(wk, __uint_as_float(u[j] & 0xFFFF0000u), acc[2 * j + 1]);
            }
        }
        if (add != nullptr) {
            const uint4 q = add[static_cast<size_t>(t) * nv + i];
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[2 * j] = __fmaf_rn(add_w, __uint_as_float(u[j] << 16), acc[2 * j]);
                acc[2 * j + 1] = __fmaf_rn(add_w, __uint_as_float(u[j] & 0xFFFF0000u), acc[2 * j + 1]);
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        out[static_cast<size_t>(t) * nv + i] = o;
    }
}

__global__ void __launch_bounds__(CB_THREADS) combine_f32_kernel(int T, int S, int H,
                                                                 const float4* __restrict__ y,
                                                                 const int32_t* __restrict__ inv,
                                                                 const float* __restrict__ w,
                                                                 const float4* __restrict__ add,
                                                                 float add_w,
                                                                 float4* __restrict__ out) {
    const int t = blockIdx.x;
    const int nv = H / 4;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < S; ++k) {
            const int r = inv[static_cast<size_t>(t) * S + k];
            const float wk = w[static_cast<size_t>(t) * S + k];
            const float4 q = y[static_cast<size_t>(r) * nv + i];
            acc.x = __fmaf_rn(wk, q.x, acc.x);
            acc.y = __fmaf_rn(wk, q.y, acc.y);
            acc.z = __fmaf_rn(wk, q.z, acc.z);
            acc.w = __fmaf_rn(wk, q.w, acc.w);
        }
        if (add != nullptr) {
            const float4 q = add[static_cast<size_t>(t) * nv + i];
            acc.x = __fmaf_rn(add_w, q.x, acc.x);
            acc.y = __fmaf_rn(add_w, q.y, acc.y);
            acc.z = __fmaf_rn(add_w, q.z, acc.z);
            acc.w = __fmaf_rn(add_w, q.w, acc.w);
        }
        out[static_cast<size_t>(t) * nv + i] = acc;
    }
}

// out = bf16(acc), 8 elements per thread-step
__global__ void __launch_bounds__(256) round_rows_kernel(size_t n8, const float4* __restrict__ acc,
                                                         uint4* __restrict__ out) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const float4 a = acc[2 * i], b = acc[2 * i + 1];
        out[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                            pack_bf16x2(b.z, b.w));
    }
}

}  // namespace

cudaError_t launch_round_rows(int T, int H, const float* acc, uint16_t* out, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const size_t n8 = static_cast<size_t>(T) * H / 8;
    const int blocks = static_cast<int>(std::min<size_t>((n8 + 255) / 256, 148 * 8));
    ProfileScope ps("round_out", stream);
    round_rows_kernel<<<blocks, 256, 0, stream>>>(n8, reinterpret_cast<const float4*>(acc),
                                                   reinterpret_cast<uint4*>(out));
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_combine(int T, int S, int H, int act_dtype, const void* y, const int32_t* inv,
                           const float* w, const void* add, float add_w, void* out,
                           cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    ProfileScope ps("combine", stream);
    if (act_dtype == MOE_BF16)
        combine_bf16_kernel<<<T, CB_THREADS, 0, stream>>>(
            T, S, H, static_cast<const uint4*>(y), inv, w, static_cast<const uint4*>(add), add_w,
            static_cast<uint4*>(out));
    else
        combine_f32_kernel<<<T, CB_THREADS, 0, stream>>>(
            T, S, H, static_cast<const float4*>(y), inv, w, static_cast<const float4*>(add), add_w,
            static_cast<float4*>(out));
    note_launch();
    return cudaGetLastError();
}

}  // namespace sre
