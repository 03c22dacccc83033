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
// computes one segment's chains per block (T x E x H/256 independent chains:
// enough parallelism to fill the GPU at any T), and the top-K kernel adds the
// segment partials in order.
#include "kernels.cuh"

namespace sre {

namespace {

constexpr int RT_BT = 128;    // tokens per block
constexpr int RT_BE = 32;     // experts per block
constexpr int RT_KC = 32;     // h per shared-memory chunk
constexpr int RT_SEG = 256;   // segment length of the fixed order
constexpr int RT_XP = RT_BT + 4;   // row pitch (floats) of the transposed x tile
constexpr int RT_WP = RT_BE + 4;   // row pitch (floats) of the transposed w tile

// x chunk: 128 tokens x 32 h -> xs[h][t]; thread i loads tokens i and i + 64
template <bool kBf16>
__device__ __forceinline__ void load_x_chunk(const void* x, int T, int H, int t0, int h0,
                                             float (*xs)[RT_XP]) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int tl = threadIdx.x + half * 64;
        const int t = t0 + tl;
        float v[32];
        if (t < T) {
            if constexpr (kBf16) {
                const uint4* p = reinterpret_cast<const uint4*>(
                    static_cast<const uint16_t*>(x) + static_cast<size_t>(t) * H + h0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 a = p[q];
                    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[8 * q + 2 * j] = __uint_as_float(w[j] << 16);
                        v[8 * q + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                    }
                }
            } else {
                const float4* p = reinterpret_cast<const float4*>(
                    static_cast<const float*>(x) + static_cast<size_t>(t) * H + h0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 a = p[q];
                    v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) xs[j][tl] = v[j];
    }
}

// w chunk: 32 experts x 32 h -> ws[h][e]; thread i loads expert i/2, h-half i%2
__device__ __forceinline__ void load_w_chunk(const float* wr, int E, int H, int e0, int h0,
                                             float (*ws)[RT_WP]) {
    const int i = threadIdx.x;
    const int e = e0 + (i >> 1);
    const int hb = (i & 1) * 16;
    float v[16];
    if (e < E) {
        const float4* p = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H + h0 + hb);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 q = p[j];
            v[4 * j] = q.x; v[4 * j + 1] = q.y; v[4 * j + 2] = q.z; v[4 * j + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) ws[hb + j][i >> 1] = v[j];
}

// grid (ceil(T/128), ceil(E/32), H/256); 64 threads, 8 tokens x 8 experts each.
// P[s][t][e] = fma chain over the 256 h of segment s (blockIdx.z), from +0.
template <bool kBf16>
__global__ void __launch_bounds__(64) router_segment_kernel(const void* __restrict__ x,
                                                            const float* __restrict__ wr,
                                                            float* __restrict__ P, int T, int H,
                                                            int E) {
    __shared__ __align__(16) float xs[RT_KC][RT_XP];
    __shared__ __align__(16) float ws[RT_KC][RT_WP];
    const int t0 = blockIdx.x * RT_BT, e0 = blockIdx.y * RT_BE, s = blockIdx.z;
    const int ty = threadIdx.x >> 2, tx = threadIdx.x & 3;   // tokens ty*8.., experts tx*8..

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;

    for (int kc = 0; kc < RT_SEG; kc += RT_KC) {
        const int h0 = s * RT_SEG + kc;
        load_x_chunk<kBf16>(x, T, H, t0, h0, xs);
        load_w_chunk(wr, E, H, e0, h0, ws);
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < RT_KC; ++k) {
            const float4 x0 = *reinterpret_cast<const float4*>(&xs[k][ty * 8]);
            const float4 x1 = *reinterpret_cast<const float4*>(&xs[k][ty * 8 + 4]);
            const float4 w0 = *reinterpret_cast<const float4*>(&ws[k][tx * 8]);
            const float4 w1 = *reinterpret_cast<const float4*>(&ws[k][tx * 8 + 4]);
            const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = __fmaf_rn(xv[a], wv[b], acc[a][b]);
        }
        __syncthreads();
    }
    float* out = P + static_cast<size_t>(s) * T * E;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int t = t0 + ty * 8 + a;
        if (t >= T) continue;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int e = e0 + tx * 8 + b;
            if (e < E) out[static_cast<size_t>(t) * E + e] = acc[a][b];
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
    (void)T;
    return H / RT_SEG;    // one partial per segment: parallel over T x E x segments
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
            router_segment_kernel<true><<<grid, 64, 0, st>>>(x, wr, partials, T, H, E);
        else
            router_segment_kernel<false><<<grid, 64, 0, st>>>(x, wr, partials, T, H, E);
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
