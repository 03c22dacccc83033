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
#include <mutex>

#include "kernels.cuh"

namespace sre {

namespace {

constexpr int RT_EL = 16;      // expert lanes per block; a thread owns kEJ experts strided by RT_EL
constexpr int RT_KC = 32;      // h per shared-memory chunk
constexpr int RT_SEG = 256;    // segment length of the fixed order
constexpr int RT_WP = RT_KC + 4;       // row pitch (floats) of the w tile ws[e][k]: 144 B rows

// Block shape: kTY token groups x RT_EL expert lanes (kTY * 16 threads); thread
// (ty, tx) owns kTPT tokens and kEJ experts, so a block covers kTY * kTPT tokens
// and RT_EL * kEJ experts of one segment.
template <int kTY, int kTPT, int kEJ>
struct RouterTile {
    static constexpr int THREADS = kTY * RT_EL;
    static constexpr int BT = kTY * kTPT;          // tokens per block
    static constexpr int BE = RT_EL * kEJ;         // experts per block
    static constexpr int XP = BT + 4;              // row pitch (floats) of the transposed x tile xs[k][t]
    static constexpr int XG = BT * RT_KC / 8 / THREADS;   // x pieces of 8 h per thread and chunk
    struct Smem {
        float xs[2][RT_KC][XP];
        float ws[2][BE][RT_WP];
    };
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// w chunk: rows e0.. (kBE experts) x 32 h, copied as is into ws[e][k]
// (16-byte pieces; rows past E are left unwritten: their results are never stored)
template <int kBE, int kThreads>
__device__ __forceinline__ void issue_w_chunk(const float* wr, int E, int H, int e0, int h0,
                                              float (*ws)[RT_WP]) {
    static_assert((kBE * RT_KC / 4) % kThreads == 0, "whole pieces per thread");
#pragma unroll
    for (int i = 0; i < (kBE * RT_KC / 4) / kThreads; ++i) {
        const int piece = threadIdx.x + i * kThreads;
        const int e = piece >> 3, c = piece & 7;
        if (e0 + e < E) cp_async16(&ws[e][c * 4], wr + static_cast<size_t>(e0 + e) * H + h0 + c * 4);
    }
    cp_async_commit();
}

// The next chunk's x is held raw (bf16 pairs or fp32 bits) in registers while
// the current chunk is multiplied, and converted when stored. Piece p = thread
// + kThreads g holds token t0 + p % BT, h h0 + 8 (p / BT) .. +7.
template <bool kBf16, int kXG>
struct XStage {
    static constexpr int N = kXG * (kBf16 ? 4 : 8);   // 32-bit words per thread
    uint32_t w[N];
};

template <bool kBf16, int kXG, int kBT, int kThreads>
__device__ __forceinline__ void load_x_chunk(const void* x, int T, int H, int t0, int h0, XStage<kBf16, kXG>& st) {
#pragma unroll
    for (int g = 0; g < kXG; ++g) {
        const int piece = threadIdx.x + g * kThreads;
        const int t = t0 + (piece % kBT);
        const int q = (piece / kBT) * 8;
        if constexpr (kBf16) {
            uint4 a = make_uint4(0u, 0u, 0u, 0u);
            if (t < T)
                a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + static_cast<size_t>(t) * H + h0 + q);
            st.w[4 * g] = a.x; st.w[4 * g + 1] = a.y; st.w[4 * g + 2] = a.z; st.w[4 * g + 3] = a.w;
        } else {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (t < T) {
                const float* p = static_cast<const float*>(x) + static_cast<size_t>(t) * H + h0 + q;
                a = *reinterpret_cast<const float4*>(p);
                b = *reinterpret_cast<const float4*>(p + 4);
            }
            st.w[8 * g] = __float_as_uint(a.x); st.w[8 * g + 1] = __float_as_uint(a.y);
            st.w[8 * g + 2] = __float_as_uint(a.z); st.w[8 * g + 3] = __float_as_uint(a.w);
            st.w[8 * g + 4] = __float_as_uint(b.x); st.w[8 * g + 5] = __float_as_uint(b.y);
            st.w[8 * g + 6] = __float_as_uint(b.z); st.w[8 * g + 7] = __float_as_uint(b.w);
        }
    }
}

// transposed into xs[k][t] as fp32 (bf16 -> fp32 is exact)
template <bool kBf16, int kXG, int kBT, int kThreads, int kXP>
__device__ __forceinline__ void store_x_chunk(const XStage<kBf16, kXG>& st, float (*xs)[kXP]) {
#pragma unroll
    for (int g = 0; g < kXG; ++g) {
        const int piece = threadIdx.x + g * kThreads;
        const int tl = piece % kBT;
        const int q = (piece / kBT) * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float v;
            if constexpr (kBf16) {
                const uint32_t pr = st.w[4 * g + (j >> 1)];
                v = __uint_as_float((j & 1) ? (pr & 0xFFFF0000u) : (pr << 16));
            } else {
                v = __uint_as_float(st.w[8 * g + j]);
            }
            xs[q + j][tl] = v;
        }
    }
}

// grid (ceil(T/BT), ceil(E/BE), H/256): thread (ty, tx) = (threadIdx / 16,
// threadIdx % 16) owns tokens t0 + kTPT ty .. +kTPT-1 and experts e0 + tx + 16 j
// (j < kEJ). P[s][t][e] = fma chain over the 256 h of segment s (blockIdx.z),
// from +0, h ascending. The next chunk's copies are in flight while this one is
// multiplied.
template <bool kBf16, int kTY, int kTPT, int kEJ, int kMinB>
__global__ void __launch_bounds__(kTY * RT_EL, kMinB) router_segment_kernel(const void* __restrict__ x,
                                                                          const float* __restrict__ wr,
                                                                          float* __restrict__ P, int T, int H,
                                                                          int E) {
    using RT = RouterTile<kTY, kTPT, kEJ>;
    constexpr int NT = RT::THREADS, BT = RT::BT, XP = RT::XP, XG = RT::XG;
    extern __shared__ __align__(16) uint8_t rt_smem[];
    using Smem = typename RT::Smem;
    Smem& sm = *reinterpret_cast<Smem*>(rt_smem);
    const int t0 = blockIdx.x * BT, e0 = blockIdx.y * RT::BE, s = blockIdx.z;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;

    float acc[kTPT][kEJ];
#pragma unroll
    for (int a = 0; a < kTPT; ++a)
#pragma unroll
        for (int j = 0; j < kEJ; ++j) acc[a][j] = 0.0f;

    constexpr int NCHUNK = RT_SEG / RT_KC;
    XStage<kBf16, XG> xnext;
    issue_w_chunk<RT::BE, NT>(wr, E, H, e0, s * RT_SEG, sm.ws[0]);
    load_x_chunk<kBf16, XG, BT, NT>(x, T, H, t0, s * RT_SEG, xnext);
    store_x_chunk<kBf16, XG, BT, NT, XP>(xnext, sm.xs[0]);
    cp_async_wait_all();
    __syncthreads();

#pragma unroll 1
    for (int c = 0; c < NCHUNK; ++c) {
        const int buf = c & 1;
        const bool more = c + 1 < NCHUNK;
        if (more) {
            const int h1 = s * RT_SEG + (c + 1) * RT_KC;
            issue_w_chunk<RT::BE, NT>(wr, E, H, e0, h1, sm.ws[buf ^ 1]);
            load_x_chunk<kBf16, XG, BT, NT>(x, T, H, t0, h1, xnext);
        }
        const float (*xs)[XP] = sm.xs[buf];
        const float (*ws)[RT_WP] = sm.ws[buf];
        // 8-token tiles: two k steps unrolled keep the operands within the register budget
        constexpr int kUnroll = kTPT >= 8 ? 2 : RT_KC / 4;
#pragma unroll kUnroll
        for (int k4 = 0; k4 < RT_KC; k4 += 4) {
            float xv[kTPT][4];   // [token][k]
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int a4 = 0; a4 < kTPT; a4 += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(&xs[k4 + kk][ty * kTPT + a4]);
                    xv[a4][kk] = v.x; xv[a4 + 1][kk] = v.y; xv[a4 + 2][kk] = v.z; xv[a4 + 3][kk] = v.w;
                }
            }
#pragma unroll
            for (int j = 0; j < kEJ; ++j) {
                const float4 w = *reinterpret_cast<const float4*>(&ws[tx + RT_EL * j][k4]);
#pragma unroll
                for (int a = 0; a < kTPT; ++a) {
                    float r = acc[a][j];
                    r = __fmaf_rn(xv[a][0], w.x, r);
                    r = __fmaf_rn(xv[a][1], w.y, r);
                    r = __fmaf_rn(xv[a][2], w.z, r);
                    r = __fmaf_rn(xv[a][3], w.w, r);
                    acc[a][j] = r;
                }
            }
        }
        if (more) {
            store_x_chunk<kBf16, XG, BT, NT, XP>(xnext, sm.xs[buf ^ 1]);
            cp_async_wait_all();
        }
        __syncthreads();
    }
    float* out = P + static_cast<size_t>(s) * T * E;
#pragma unroll
    for (int a = 0; a < kTPT; ++a) {
        const int t = t0 + ty * kTPT + a;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < kEJ; ++j) {
            const int e = e0 + tx + RT_EL * j;
            if (e < E) out[static_cast<size_t>(t) * E + e] = acc[a][j];
        }
    }
}

__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
    return v1 > v2 || (v1 == v2 && i1 < i2);
}

constexpr int TK_MAXPL = 8;   // logits per lane: n_routed <= 256

// One warp per token. P holds n_part ordered partials [n_part][T][E].
// key = ranking score (logit + bias, fp32, bias added last); the weights use
// the key, or the logit without the bias when bias_select_only; routed slots
// weigh routed_scale * softmax.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ P, int n_part,
                                                   const float* __restrict__ bias, int T, int E,
                                                   int K, int renormalize, int shared_id,
                                                   float shared_weight, float routed_scale,
                                                   int bias_select_only, int32_t* __restrict__ ids,
                                                   float* __restrict__ wts,
                                                   float* __restrict__ logits_out) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int t = warp;
    const int S = K + (shared_id >= 0 ? 1 : 0);
    // segment partials summed in segment order; TK_PB segments' loads are in
    // flight before the first of them is added
    constexpr int TK_PB = 4;
    float tot[TK_MAXPL];
#pragma unroll
    for (int j = 0; j < TK_MAXPL; ++j) tot[j] = 0.0f;
    for (int p0 = 0; p0 < n_part; p0 += TK_PB) {
        float v[TK_PB][TK_MAXPL];
#pragma unroll
        for (int q = 0; q < TK_PB; ++q)
#pragma unroll
            for (int j = 0; j < TK_MAXPL; ++j) {
                const int e = lane + 32 * j;
                v[q][j] = (p0 + q < n_part && e < E) ? P[(static_cast<size_t>(p0 + q) * T + t) * E + e] : 0.0f;
            }
#pragma unroll
        for (int q = 0; q < TK_PB; ++q)
            if (p0 + q < n_part)
#pragma unroll
                for (int j = 0; j < TK_MAXPL; ++j) tot[j] = __fadd_rn(tot[j], v[q][j]);
    }
    float key[TK_MAXPL], wlog[TK_MAXPL];
#pragma unroll
    for (int j = 0; j < TK_MAXPL; ++j) {
        const int e = lane + 32 * j;
        float v = -INFINITY, u = -INFINITY;
        if (e < E) {
            float tj = tot[j];
            const float raw = isnan(tj) ? -INFINITY : tj;
            if (bias != nullptr) tj = __fadd_rn(tj, bias[e]);
            if (logits_out != nullptr) logits_out[static_cast<size_t>(t) * E + e] = tj;
            v = isnan(tj) ? -INFINITY : tj;
            u = (bias_select_only && bias != nullptr) ? raw : v;
        }
        key[j] = v;
        wlog[j] = u;
    }
    unsigned taken = 0;    // bit j: element lane + 32j taken
    float sel_w[32];       // weight logits of the selected experts, in rank order
    int my_id = -1;
    float my_w = 0.0f;
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
        float wv = 0.0f;     // the owner lane's weight logit of expert bi
#pragma unroll
        for (int j = 0; j < TK_MAXPL; ++j)
            if (j == (bi >> 5)) wv = wlog[j];
        wv = __shfl_sync(0xFFFFFFFFu, wv, bi & 31);
        sel_w[k] = wv;
        if (lane == k) { my_id = bi; my_w = wv; }
    }
    float m = -INFINITY, den = 0.0f;
    if (renormalize) {
        for (int k = 0; k < K; ++k) m = fmaxf(m, sel_w[k]);
        for (int k = 0; k < K; ++k) den += expf(sel_w[k] - m);
    } else {
#pragma unroll
        for (int j = 0; j < TK_MAXPL; ++j) m = fmaxf(m, wlog[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        float part = 0.0f;
#pragma unroll
        for (int j = 0; j < TK_MAXPL; ++j)
            if (lane + 32 * j < E) part += expf(wlog[j] - m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
        den = part;
    }
    if (lane < K) {
        ids[static_cast<size_t>(t) * S + lane] = my_id;
        wts[static_cast<size_t>(t) * S + lane] = routed_scale * (expf(my_w - m) / den);
    }
    if (shared_id >= 0 && lane == 0) {
        ids[static_cast<size_t>(t) * S + K] = shared_id;
        wts[static_cast<size_t>(t) * S + K] = shared_weight;
    }
}

template <int kTY, int kTPT, int kEJ, int kMinB>
cudaError_t launch_router_segments(const moe_shape& s, const void* x, const float* wr, float* partials, int T,
                                   int H, int E, int split, cudaStream_t st) {
    using RT = RouterTile<kTY, kTPT, kEJ>;
    constexpr int smem = static_cast<int>(sizeof(typename RT::Smem));
    auto kb = router_segment_kernel<true, kTY, kTPT, kEJ, kMinB>;
    auto kf = router_segment_kernel<false, kTY, kTPT, kEJ, kMinB>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [kb, kf] {
        attr_err = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    dim3 grid(ceil_div(T, RT::BT), ceil_div(E, RT::BE), split);
    ProfileScope ps("route_logits", st);
    if (s.act_dtype == MOE_BF16)
        kb<<<grid, RT::THREADS, smem, st>>>(x, wr, partials, T, H, E);
    else
        kf<<<grid, RT::THREADS, smem, st>>>(x, wr, partials, T, H, E);
    note_launch();
    return cudaGetLastError();
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
                         int32_t* ids, float* wts, float* logits, float* partials, void* route_scratch,
                         int shared_id, DevStatus* status, cudaStream_t st) {
    const int T = s.T, H = s.H, E = s.n_routed;
#ifndef SRE_ROUTE_TC
#define SRE_ROUTE_TC 1
#endif
    // the same ids and weights from approximate tensor-core logits, verified exactly
    if (SRE_ROUTE_TC && route_scratch != nullptr && route_tc_applies(s, logits))
        return launch_route_tc(s, x, wr, bias, ids, wts, partials, route_scratch, shared_id, status, st);
    const int split = router_split_count(T, H);
    // small batches: 32 experts per block (5x the blocks at 160 routed experts)
#ifndef SRE_RT_WIDE
#define SRE_RT_WIDE 1
#endif
    const bool narrow = T <= 256;
    cudaError_t err;
    if (narrow)
        err = launch_router_segments<16, 4, 2, 2>(s, x, wr, partials, T, H, E, split, st);
    else if (SRE_RT_WIDE == 1)
        err = launch_router_segments<8, 8, 10, 3>(s, x, wr, partials, T, H, E, split, st);
    else
        err = launch_router_segments<16, 4, 10, 2>(s, x, wr, partials, T, H, E, split, st);
    if (err != cudaSuccess) return err;
    {
        ProfileScope ps("route_topk", st);
        topk_kernel<<<ceil_div(T * 32, 256), 256, 0, st>>>(partials, split, bias, T, E, s.top_k,
                                                          s.renormalize, shared_id, s.shared_weight,
                                                          s.routed_scale, s.bias_select_only, ids, wts,
                                                          logits);
        note_launch();
    }
    return cudaGetLastError();
}

}  // namespace sre
