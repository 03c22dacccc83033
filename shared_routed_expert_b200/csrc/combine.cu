// Weighted aggregation of the expert outputs.
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1: all expert
// outputs are aggregated with weights. With the fusion the shared expert is
// slot K of every token (weight shared_weight), so one weighted sum over the
// S = K + 1 slots gives the layer output:
//     out[t] = sum_{k<S} w[t,k] * y[inv[t*S + k]]
// accumulated in fp32 in slot order and rounded once to the output dtype
// The moe_combine entry point runs it over bf16/fp32 expert rows; moe_forward
// over the scaled-fp16 rows its down-projection writes (11 significant bits,
// so that storing the rows adds ~2^-12 relative error per slot instead of
// bf16's 2^-9). `add` (weight add_w) is an optional [T, H] term added last:
// the unfused layer's separately computed shared expert.
#include <algorithm>

#include "kernels.cuh"

namespace sre {

namespace {

constexpr int CB_THREADS = 128;
constexpr int CB_BATCH = 9;      // slot rows loaded together (S = 9: all at once)

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

// Scaled-fp16 rows (see the GEMM2 epilogue): value = fp16 * 2^k, one k per 32
// columns. Each thread owns 8-column vectors of the token's row (4 threads per
// exponent byte). The sum is written rounded to bf16, or as fp32 (kF32Out: a
// tensor-parallel rank's partial output).
template <bool kF32Out>
__global__ void __launch_bounds__(CB_THREADS) combine_f16s_kernel(int T, int S, int H,
                                                                  const uint4* __restrict__ y,
                                                                  const int8_t* __restrict__ yexp,
                                                                  const int32_t* __restrict__ inv,
                                                                  const float* __restrict__ w,
                                                                  const uint4* __restrict__ add,
                                                                  const int8_t* __restrict__ addexp,
                                                                  float add_w, void* __restrict__ out) {
    const int t = blockIdx.x;
    const int nv = H / 8, ne = H / 32;
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
        // slots in groups of CB_BATCH: the group's row loads are all in flight
        // before the first of them is accumulated (accumulation stays in slot order)
        for (int k0 = 0; k0 < S; k0 += CB_BATCH) {
            uint4 q[CB_BATCH];
            int8_t ex[CB_BATCH];
#pragma unroll
            for (int g = 0; g < CB_BATCH; ++g) {
                if (k0 + g < S) {
                    const size_t r = static_cast<size_t>(s_row[k0 + g]);
                    q[g] = y[r * nv + i];
                    ex[g] = yexp[r * ne + (i >> 2)];
                }
            }
#pragma unroll
            for (int g = 0; g < CB_BATCH; ++g) {
                if (k0 + g < S) {
                    const float wk = s_w[k0 + g] * exp2_int(ex[g]);
                    const uint32_t u[4] = {q[g].x, q[g].y, q[g].z, q[g].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = unpack_f16x2(u[j]);
                        acc[2 * j] = __fmaf_rn(wk, f.x, acc[2 * j]);
                        acc[2 * j + 1] = __fmaf_rn(wk, f.y, acc[2 * j + 1]);
                    }
                }
            }
        }
        if (add != nullptr) {
            const uint4 q = add[static_cast<size_t>(t) * nv + i];
            const float wk = add_w * exp2_int(addexp[static_cast<size_t>(t) * ne + (i >> 2)]);
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = unpack_f16x2(u[j]);
                acc[2 * j] = __fmaf_rn(wk, f.x, acc[2 * j]);
                acc[2 * j + 1] = __fmaf_rn(wk, f.y, acc[2 * j + 1]);
            }
        }
        if constexpr (kF32Out) {
            float4* o = static_cast<float4*>(out) + (static_cast<size_t>(t) * nv + i) * 2;
            o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
            static_cast<uint4*>(out)[static_cast<size_t>(t) * nv + i] =
                make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
        }
    }
}

__global__ void __launch_bounds__(256) cast_f32_bf16_kernel(size_t n4, const float4* __restrict__ in,
                                                            uint2* __restrict__ out) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const float4 v = in[i];
        out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
}

}  // namespace

cudaError_t launch_combine_f16s(int T, int S, int H, const uint16_t* y16, const int8_t* yexp,
                                const int32_t* inv, const float* w, const uint16_t* add16,
                                const int8_t* addexp, float add_w, void* out, bool out_f32, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    ProfileScope ps("combine", stream);
    if (out_f32)
        combine_f16s_kernel<true><<<T, CB_THREADS, 0, stream>>>(T, S, H, reinterpret_cast<const uint4*>(y16), yexp,
                                                                inv, w, reinterpret_cast<const uint4*>(add16),
                                                                addexp, add_w, out);
    else
        combine_f16s_kernel<false><<<T, CB_THREADS, 0, stream>>>(T, S, H, reinterpret_cast<const uint4*>(y16),
                                                                 yexp, inv, w, reinterpret_cast<const uint4*>(add16),
                                                                 addexp, add_w, out);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_cast_f32_bf16(size_t n, const float* in, uint16_t* out, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    ProfileScope ps("cast_bf16", stream);
    const size_t n4 = n / 4;
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n4 + 255) / 256, 148 * 16));
    cast_f32_bf16_kernel<<<blocks, 256, 0, stream>>>(n4, reinterpret_cast<const float4*>(in),
                                                     reinterpret_cast<uint2*>(out));
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
