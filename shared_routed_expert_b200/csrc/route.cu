// Router of the GLM4-MoE expert layer: logits, top-K, slot weights.
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1 "Shared Experts
// Fusion": each token's router selects its top-8 routed experts; with the
// fusion the shared expert (index n_routed) is fixed in the 9th slot.
//
// Logits are fp32 in one fixed order so that routing is reproducible bit for
// bit: H is cut into 256-wide segments; inside a segment an fma chain starting
// at +0 runs over ascending h; segment sums are added in ascending order to a
// running total starting at +0; the bias is added last. The tile kernel below
// either walks all segments of its (token, expert) tile itself (large T) or
// computes one segment per block and leaves the ordered sum of the segment
// partials to the top-K kernel (small T, where there are too few tiles to fill
// the GPU). Both give the same bits.
#include "kernels.cuh"

namespace sre {

namespace {

constexpr int RT_BT = 32;     // tokens per block
constexpr int RT_BE = 32;     // experts per block
constexpr int RT_KC = 32;     // h per shared-memory chunk
constexpr int RT_SEG = 256;   // segment length of the fixed order
constexpr int RT_PAD = 36;    // row pitch (floats) of the transposed tiles

template <bool kBf16>
__device__ __forceinline__ void load_x_chunk(const void* x, int T, int H, int t0, int h0,
                                             float (*xs)[RT_PAD]) {
    const int i = threadIdx.x;          // 64 threads: token i/2, half i%2
    const int t = t0 + (i >> 1);
    const int hb = h0 + (i & 1) * 16;
    float v[16];
    if (t < T) {
        if constexpr (kBf16) {
            const uint4* p = reinterpret_cast<const uint4*>(
                static_cast<const uint16_t*>(x) + static_cast<size_t>(t) * H + hb);
            uint4 a = p[0], b = p[1];
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                v[2 * j] = __uint_as_float(w[j] << 16);
                v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        } else {
            const float4* p = reinterpret_cast<const float4*>(
                static_cast<const float*>(x) + static_cast<size_t>(t) * H + hb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 q = p[j];
                v[4 * j] = q.x; v[4 * j + 1] = q.y; v[4 * j + 2] = q.z; v[4 * j + 3] = q.w;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
    }
    const int col = i >> 1, rb = (i & 1) * 16;
#pragma unroll
    for (int j = 0; j < 16; ++j) xs[rb + j][col] = v[j];
}

__device__ __forceinline__ void load_w_chunk(const float* wr, int E, int H, int e0, int h0,
                                             float (*ws)[RT_PAD]) {
    const int i = threadIdx.x;
    const int e = e0 + (i >> 1);
    const int hb = h0 + (i & 1) * 16;
    float v[16];
    if (e < E) {
        const float4* p = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H + hb);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float4 q = p[j];
            v[4 * j] = q.x; v[4 * j + 1] = q.y; v[4 * j + 2] = q.z; v[4 * j + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
    }
    const int col = i >> 1, rb = (i & 1) * 16;
#pragma unroll
    for (int j = 0; j < 16; ++j) ws[rb + j][col] = v[j];
}

// grid (ceil(T/32), ceil(E/32), n_split); 64 threads, 4x4 (token, expert) each.
// n_split == 1: P[t][e] = ordered sum over all segments.
// n_split == H/256: P[s][t][e] = sum of segment s (blockIdx.z).
template <bool kBf16>
__global__ void __launch_bounds__(64) router_logits_kernel(const void* __restrict__ x,
                                                           const float* __restrict__ wr,
                                                           float* __restrict__ P, int T, int H,
                                                           int E, int n_split) {
    __shared__ __align__(16) float xs[RT_KC][RT_PAD];
    __shared__ __align__(16) float ws[RT_KC][RT_PAD];
    const int t0 = blockIdx.x * RT_BT, e0 = blockIdx.y * RT_BE;
    const int ty = threadIdx.x >> 3, tx = threadIdx.x & 7;   // tokens ty*4.., experts tx*4..
    const int nseg = H / RT_SEG;
    int s_begin = 0, s_end = nseg;
    if (n_split > 1) { s_begin = blockIdx.z; s_end = blockIdx.z + 1; }

    float total[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) total[a][b] = 0.0f;

    for (int s = s_begin; s < s_end; ++s) {
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
        for (int kc = 0; kc < RT_SEG; kc += RT_KC) {
            const int h0 = s * RT_SEG + kc;
            load_x_chunk<kBf16>(x, T, H, t0, h0, xs);
            load_w_chunk(wr, E, H, e0, h0, ws);
            __syncthreads();
#pragma unroll 8
            for (int k = 0; k < RT_KC; ++k) {
                const float4 xa = *reinterpret_cast<const float4*>(&xs[k][ty * 4]);
                const float4 wb = *reinterpret_cast<const float4*>(&ws[k][tx * 4]);
                const float xv[4] = {xa.x, xa.y, xa.z, xa.w};
                const float wv[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(xv[a], wv[b], acc[a][b]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
                total[a][b] = (n_split > 1) ? acc[a][b] : __fadd_rn(total[a][b], acc[a][b]);
    }
    float* out = P + (n_split > 1 ? static_cast<size_t>(blockIdx.z) * T * E : 0);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int t = t0 + ty * 4 + a;
        if (t >= T) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int e = e0 + tx * 4 + b;
            if (e < E) out[static_cast<size_t>(t) * E + e] = total[a][b];
        }
    }
}

__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
    return v1 > v2 || (v1 == v2 && i1 < i2);
}

constexpr int TK_MAXPL = 8;   // logits per lane: n_routed <= 256

// One warp per token. P holds n_part ordered partials [n_part][T][E].
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ P, int n_part,
                                                   const float* __restrict__ bias, int T, int E,
                                                   int K, int renormalize, int shared_id,
                                                   float shared_weight, int32_t* __restrict__ ids,
                                                   float* __restrict__ wts,
                                                   float* __restrict__ logits_out) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int t = warp;
    const int S = K + (shared_id >= 0 ? 1 : 0);
    float key[TK_MAXPL];
#pragma unroll
    for (int j = 0; j < TK_MAXPL; ++j) {
        const int e = lane + 32 * j;
        float v = -INFINITY;
        if (e < E) {
            float tot = 0.0f;
            for (int p = 0; p < n_part; ++p)
                tot = __fadd_rn(tot, P[(static_cast<size_t>(p) * T + t) * E + e]);
            if (bias != nullptr) tot = __fadd_rn(tot, bias[e]);
            if (logits_out != nullptr) logits_out[static_cast<size_t>(t) * E + e] = tot;
            v = isnan(tot) ? -INFINITY : tot;
        }
        key[j] = v;
    }
    unsigned taken = 0;    // bit j: element lane + 32j taken
    float sel_v[32];
    int my_id = -1;
    float my_v = 0.0f;
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < TK_MAXPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E && !((taken >> j) & 1u) && better(key[j], e, bv, bi)) { bv = key[j]; bi = e; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        sel_v[k] = bv;
        if (lane == k) { my_id = bi; my_v = bv; }
    }
    float m, den = 0.0f;
    if (renormalize) {
        m = sel_v[0];
        for (int k = 0; k < K; ++k) den += expf(sel_v[k] - m);
    } else {
        m = -INFINITY;
#pragma unroll
        for (int j = 0; j < TK_MAXPL; ++j) m = fmaxf(m, key[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        float part = 0.0f;
#pragma unroll
        for (int j = 0; j < TK_MAXPL; ++j)
            if (lane + 32 * j < E) part += expf(key[j] - m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
        den = part;
    }
    if (lane < K) {
        ids[static_cast<size_t>(t) * S + lane] = my_id;
        wts[static_cast<size_t>(t) * S + lane] = expf(my_v - m) / den;
    }
    if (shared_id >= 0 && lane == 0) {
        ids[static_cast<size_t>(t) * S + K] = shared_id;
        wts[static_cast<size_t>(t) * S + K] = shared_weight;
    }
}

}  // namespace

int router_split_count(int T, int H) {
    // Split into segments when the (token, expert) tiles alone cannot fill the GPU.
    return (T <= 512) ? H / RT_SEG : 1;
}

size_t router_partial_floats(int T, int H, int E) {
    return static_cast<size_t>(router_split_count(T, H)) * T * E;
}

cudaError_t launch_route(const moe_shape& s, const void* x, const float* wr, const float* bias,
                         int32_t* ids, float* wts, float* logits, float* partials, int shared_id,
                         cudaStream_t st) {
    const int T = s.T, H = s.H, E = s.n_routed;
    const int split = router_split_count(T, H);
    dim3 grid(ceil_div(T, RT_BT), ceil_div(E, RT_BE), split);
    {
        ProfileScope ps("route_logits", st);
        if (s.act_dtype == MOE_BF16)
            router_logits_kernel<true><<<grid, 64, 0, st>>>(x, wr, partials, T, H, E, split);
        else
            router_logits_kernel<false><<<grid, 64, 0, st>>>(x, wr, partials, T, H, E, split);
        note_launch();
    }
    {
        ProfileScope ps("route_topk", st);
        topk_kernel<<<ceil_div(T * 32, 256), 256, 0, st>>>(partials, split, bias, T, E, s.top_k,
                                                          s.renormalize, shared_id,
                                                          s.shared_weight, ids, wts, logits);
        note_launch();
    }
    return cudaGetLastError();
}

}  // namespace sre
