// Grouped SwiGLU expert FFN on CUDA cores (fp32 layers; also a slow
// cross-check of the tensor-core kernels for bf16 / E4M3 weights).
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1: the shared and
// routed experts have identical tensor shapes and computation flow, so one
// grouped pass over the expert-sorted rows serves all S slots of every token.
// Per row r of expert e (offsets[e] <= r < offsets[e+1]):
//     h = silu(gate_e . v) * (up_e . v)        gate rows [0, I), up rows [I, 2I) of w13[e]
//     y = w2[e] . h
// E4M3 layers carry per-row activation scales and per-output-channel weight
// scales; both factor out of the K-sum and are applied in the epilogue.
//
// Work is cut into (expert m-tile of 128 rows, n-tile) blocks; m-tiles never
// straddle two experts. The grid covers an upper bound of the m-tile count;
// blocks past the real count (tile_off[E]) exit at once.
#include "kernels.cuh"

namespace sre {

namespace {

constexpr int SM_BM = kTileM;   // 128 rows
constexpr int SM_BK = 16;

template <int DT>
__device__ __forceinline__ void load8(const void* base, size_t idx, float* v) {
    if constexpr (DT == MOE_F32) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
        const float4 a = p[0], b = p[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else if constexpr (DT == MOE_BF16) {
        const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx);
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = __uint_as_float(u[j] << 16);
            v[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
    } else {
        const uint2 q = *reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(base) + idx);
        const uint32_t u[2] = {q.x, q.y};
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = e4m3_to_f32(static_cast<uint8_t>(u[j >> 2] >> ((j & 3) * 8)));
    }
}

__device__ __forceinline__ int find_expert(const int32_t* tile_off, int E, int mt) {
    int lo = 0, hi = E - 1;   // largest e with tile_off[e] <= mt
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_off[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// GEMM1 + SwiGLU. Block: 128 rows x 32 h-columns (gate and up), 256 threads,
// 4 rows x 4 columns (x2 for gate/up) per thread.
template <int ADT, int WDT>
__global__ void __launch_bounds__(256) simt_gemm1_kernel(FfnArgs a) {
    constexpr int BN = 32;
    __shared__ __align__(16) float As[SM_BK][SM_BM + 4];
    __shared__ __align__(16) float Bs[SM_BK][2 * BN + 4];
    const int mt = blockIdx.x;
    if (mt >= a.tile_off[a.E]) return;
    const int e = find_expert(a.tile_off, a.E, mt);
    const int row0 = a.offsets[e] + (mt - a.tile_off[e]) * SM_BM;
    const int row_end = a.offsets[e + 1];
    const int n0 = blockIdx.y * BN;
    const int H = a.H, I = a.I;
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    const size_t wbase = static_cast<size_t>(e) * 2 * I * H;

    float g[4][4], u[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { g[i][j] = 0.f; u[i][j] = 0.f; }

    for (int k0 = 0; k0 < H; k0 += SM_BK) {
        {   // A: 128 rows x 16 k, 8 values per thread
            const int r = tid >> 1, kh = (tid & 1) * 8;
            float v[8];
            const int row = row0 + r;
            if (row < row_end) load8<ADT>(a.xp, static_cast<size_t>(row) * H + k0 + kh, v);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) As[kh + j][r] = v[j];
        }
        if (tid < 2 * BN * 2) {   // B: 64 weight rows (32 gate, 32 up) x 16 k
            const int r = tid >> 1, kh = (tid & 1) * 8;
            const int n = (r < BN) ? (n0 + r) : (I + n0 + r - BN);
            float v[8];
            load8<WDT>(a.w13, wbase + static_cast<size_t>(n) * H + k0 + kh, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) Bs[kh + j][r] = v[j];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < SM_BK; ++k) {
            const float4 av = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
            const float4 gv = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
            const float4 uv = *reinterpret_cast<const float4*>(&Bs[k][BN + tx * 4]);
            const float ar[4] = {av.x, av.y, av.z, av.w};
            const float gr[4] = {gv.x, gv.y, gv.z, gv.w};
            const float ur[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    g[i][j] = fmaf(ar[i], gr[j], g[i][j]);
                    u[i][j] = fmaf(ar[i], ur[j], u[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = row0 + ty * 4 + i;
        if (row >= row_end) continue;
        const float xs = (WDT == MOE_E4M3) ? a.xp_scale[row] : 1.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            float gv = g[i][j], uv = u[i][j];
            if (WDT == MOE_E4M3) {
                gv = gv * xs * a.s13[static_cast<size_t>(e) * 2 * I + n];
                uv = uv * xs * a.s13[static_cast<size_t>(e) * 2 * I + I + n];
            }
            const float hv = silu_f32(gv) * uv;
            if (ADT == MOE_F32 && WDT == MOE_F32)
                static_cast<float*>(a.h)[static_cast<size_t>(row) * I + n] = hv;
            else
                static_cast<uint16_t*>(a.h)[static_cast<size_t>(row) * I + n] = f32_to_bf16(hv);
        }
    }
}

// GEMM2. Block: 128 rows x 64 output columns, 256 threads, 4 rows x 8 columns each.
template <int HDT, int WDT>
__global__ void __launch_bounds__(256) simt_gemm2_kernel(FfnArgs a) {
    constexpr int BN = 64;
    __shared__ __align__(16) float As[SM_BK][SM_BM + 4];
    __shared__ __align__(16) float Bs[SM_BK][BN + 4];
    const int mt = blockIdx.x;
    if (mt >= a.tile_off[a.E]) return;
    const int e = find_expert(a.tile_off, a.E, mt);
    const int row0 = a.offsets[e] + (mt - a.tile_off[e]) * SM_BM;
    const int row_end = a.offsets[e + 1];
    const int n0 = blockIdx.y * BN;
    const int H = a.H, I = a.I;
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    const size_t wbase = static_cast<size_t>(e) * H * I;
    const void* A = (HDT == MOE_E4M3) ? static_cast<const void*>(a.hq) : a.h;

    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < I; k0 += SM_BK) {
        {
            const int r = tid >> 1, kh = (tid & 1) * 8;
            float v[8];
            const int row = row0 + r;
            if (row < row_end) load8<HDT>(A, static_cast<size_t>(row) * I + k0 + kh, v);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) As[kh + j][r] = v[j];
        }
        if (tid < BN * 2) {
            const int r = tid >> 1, kh = (tid & 1) * 8;
            float v[8];
            load8<WDT>(a.w2, wbase + static_cast<size_t>(n0 + r) * I + k0 + kh, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) Bs[kh + j][r] = v[j];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < SM_BK; ++k) {
            const float4 av = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[k][tx * 8]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[k][tx * 8 + 4]);
            const float ar[4] = {av.x, av.y, av.z, av.w};
            const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
        }
        __syncthreads();
    }
    // Scaled-fp16 rows: the 32-column chunk of a row is spread over 4 lanes
    // (tx = 4c..4c+3), so its amax is reduced over lane bits 0-1. Every lane
    // runs the shuffles; only valid rows store.
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = row0 + ty * 4 + i;
        const bool valid = row < row_end;
        const float hs = (WDT == MOE_E4M3 && valid) ? a.h_scale[row] : 1.0f;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int n = n0 + tx * 8 + j;
            v[j] = acc[i][j];
            if (WDT == MOE_E4M3 && valid) v[j] = v[j] * hs * a.s2[static_cast<size_t>(e) * H + n];
        }
        if (a.yexp != nullptr) {
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
            const int k = f16_chunk_exp(amax);
            const float down = exp2_int(-k);
            if (valid) {
                uint16_t* dst = static_cast<uint16_t*>(a.y) + static_cast<size_t>(row) * H + n0 + tx * 8;
                *reinterpret_cast<uint4*>(dst) =
                    make_uint4(pack_f16x2(v[0] * down, v[1] * down), pack_f16x2(v[2] * down, v[3] * down),
                               pack_f16x2(v[4] * down, v[5] * down), pack_f16x2(v[6] * down, v[7] * down));
                if ((tx & 3) == 0) a.yexp[static_cast<size_t>(row) * (H / 32) + (n0 + tx * 8) / 32] = static_cast<int8_t>(k);
            }
        } else if (valid) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = n0 + tx * 8 + j;
                if (HDT == MOE_F32)
                    static_cast<float*>(a.y)[static_cast<size_t>(row) * H + n] = v[j];
                else
                    static_cast<uint16_t*>(a.y)[static_cast<size_t>(row) * H + n] = f32_to_bf16(v[j]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_ffn_simt(const FfnArgs& in, cudaStream_t stream) {
    if (in.R == 0 || in.max_mtiles == 0) return cudaSuccess;
    FfnArgs a = in;
    if (a.perm != nullptr) {
        // rows of the grouped pass gathered from the token matrix
        const int eb = (a.w_dtype == MOE_E4M3) ? 1 : (a.act_dtype == MOE_F32 ? 4 : 2);
        cudaError_t err = launch_gather_rows(a.R, a.S, a.H, eb, a.xt, a.xt_scale, a.perm, a.xp, a.xp_scale, nullptr, stream);
        if (err != cudaSuccess) return err;
    } else {
        a.xp = const_cast<void*>(a.xt);           // row r is token r
        a.xp_scale = const_cast<float*>(a.xt_scale);
    }
    const dim3 g1(a.max_mtiles, a.I / 32), g2(a.max_mtiles, a.H / 64);
    {
        ProfileScope ps("gemm1_simt", stream);
        if (a.w_dtype == MOE_F32) simt_gemm1_kernel<MOE_F32, MOE_F32><<<g1, 256, 0, stream>>>(a);
        else if (a.w_dtype == MOE_BF16) simt_gemm1_kernel<MOE_BF16, MOE_BF16><<<g1, 256, 0, stream>>>(a);
        else simt_gemm1_kernel<MOE_E4M3, MOE_E4M3><<<g1, 256, 0, stream>>>(a);
        note_launch();
    }
    if (a.w_dtype == MOE_E4M3) {
        cudaError_t err = launch_quant_rows(a.R, a.I, static_cast<const uint16_t*>(a.h), a.hq,
                                            a.h_scale, stream, "quant_h");
        if (err != cudaSuccess) return err;
    }
    {
        ProfileScope ps("gemm2_simt", stream);
        if (a.w_dtype == MOE_F32) simt_gemm2_kernel<MOE_F32, MOE_F32><<<g2, 256, 0, stream>>>(a);
        else if (a.w_dtype == MOE_BF16) simt_gemm2_kernel<MOE_BF16, MOE_BF16><<<g2, 256, 0, stream>>>(a);
        else simt_gemm2_kernel<MOE_E4M3, MOE_E4M3><<<g2, 256, 0, stream>>>(a);
        note_launch();
    }
    return cudaGetLastError();
}

}  // namespace sre
