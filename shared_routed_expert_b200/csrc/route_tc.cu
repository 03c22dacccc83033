// Routing through approximate logits on the tensor cores, verified exactly.
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1: every token's
// router picks its top-8 routed experts; with the fusion the shared expert
// takes the 9th slot. The ids and weights produced here are those of the
// fixed-order fp32 logits of route.cu (per 256-wide segment of H an fma chain
// from +0 over ascending h, segment sums added in ascending order to a total
// starting at +0, then the bias), bit for bit: the tensor cores only narrow
// down which experts' logits must be formed that way.
//
//   A. split       w = w_hi + w_lo + r, w_hi = bf16(w), w_lo = bf16(w - w_hi),
//                  so |r| <= 2^-16 |w|; ||w_e||_2 per expert.
//   B. approximate a[t][e] = x_t . w_hi_e + x_t . w_lo_e by tcgen05 MMAs (bf16
//                  operands, fp32 accumulators), over KS slices of H.
//   C. candidates  |a - L| <= eps_e = RV_C ||x_t|| ||w_e|| for the fixed-order
//                  logit L: sum_h |x_h w_h| <= ||x|| ||w|| (Cauchy-Schwarz) bounds
//                  the split residual (2^-16 = 1.5e-5), the fixed order's own
//                  rounding (< 280 u = 1.7e-5), the sum of the KS slices and the
//                  tensor cores' fp32 accumulation (at one ulp per 16-product
//                  step, H / 16 steps: 1.9e-5 at H = 5120), about 5e-5 in all;
//                  RV_C is twice that. (Measured on B200 over random, Zipf-biased,
//                  x100-scaled and 256-expert inputs: at most 2.9e-7.) Let A be the K experts of largest approximate key
//                  (a + bias) and Tk the smallest of their keys. Every expert of
//                  A has an exact key >= Tk - max eps, so an expert whose
//                  approximate key is below Tk - max eps - eps_e is beaten by K
//                  experts and is not in the exact top-K: the exact top-K lies in
//                  S = {e : key_e + eps_e >= Tk - max eps}.
//   D. verify      the fixed-order segment partials of the candidates only: the
//                  (token, candidate) pairs are bucketed by expert, so a warp
//                  works on pairs of one expert (its weights read once for all
//                  lanes) and each lane streams its token's activations.
//   E. select      ordered segment sums, the bias, the ranking (key descending,
//                  id ascending) and the softmax over the selected slots, with
//                  the arithmetic of route.cu's top-K kernel.
// A token with a non-finite approximation or norm, or with more candidates
// than RV_MAXC, forms every expert's logit in step E (slow, exact). The path
// serves renormalised top-K over bf16 activations when no logits are asked
// for; route.cu serves the rest.
#include <algorithm>
#include <atomic>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace sre {

namespace {

constexpr int RV_MAXC = 32;                 // candidate slots per token
constexpr float RV_C = 1.0e-4f;             // eps coefficient (see step C)
constexpr int RV_SEG = 256;                 // the fixed order's segment length
constexpr int RV_CPAD = 32;                 // ints between two experts' pair counters (one 128-byte line each)
constexpr int RTC_THREADS = 192;            // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int RTC_MAX_STAGES = 6;
constexpr int RTC_RING = 192 * 1024;
constexpr int RTC_MIN_SMEM = 120 * 1024;    // one CTA per SM: its 512 TMEM columns never wait
constexpr int WS_ROWS = 256;                // rows per half of the split weights

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
    return v > bv || (v == bv && e < be);
}
__device__ __forceinline__ float rank_key(float v) { return isnan(v) ? -INFINITY : v; }

// ---------------------------------------------------------------- A. split
// Also zeroes the per-expert pair counters that step C fills.
__global__ void __launch_bounds__(256) route_split_kernel(const float* __restrict__ wr, int E, int H,
                                                          __nv_bfloat16* __restrict__ ws, float* __restrict__ nw,
                                                          int32_t* __restrict__ bcnt) {
    // H <= 8192: every thread's (up to 8) float4 loads are in flight together
    constexpr int VM = 8;
    const int e = blockIdx.x;
    if (threadIdx.x == 0) bcnt[e * RV_CPAD] = 0;
    const int nv = H / 4;
    float4 v[VM];
#pragma unroll
    for (int i = 0; i < VM; ++i) {
        const int q = threadIdx.x + i * 256;
        v[i] = (e < E && q < nv) ? reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H)[q]
                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < VM; ++i) {
        const int q = threadIdx.x + i * 256;
        if (q >= nv) continue;
        const float w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint16_t hb[4], lb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(w[j]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(w[j] - __bfloat162float(hi));
            hb[j] = __bfloat16_as_ushort(hi);
            lb[j] = __bfloat16_as_ushort(lo);
            ss = fmaf(w[j], w[j], ss);
        }
        const uint2 hv = make_uint2(hb[0] | (static_cast<uint32_t>(hb[1]) << 16), hb[2] | (static_cast<uint32_t>(hb[3]) << 16));
        const uint2 lv = make_uint2(lb[0] | (static_cast<uint32_t>(lb[1]) << 16), lb[2] | (static_cast<uint32_t>(lb[3]) << 16));
        reinterpret_cast<uint2*>(ws + static_cast<size_t>(e) * H)[q] = hv;
        reinterpret_cast<uint2*>(ws + (static_cast<size_t>(WS_ROWS) + e) * H)[q] = lv;
    }
    __shared__ float red[8];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int i = 0; i < (blockDim.x >> 5); ++i) t += red[i];
        nw[e] = sqrtf(t) * 1.00390625f;     // 1 + 2^-8 covers the norm's own rounding
    }
}

// ---------------------------------------------------------------- B. approximate logits
// CTA (mt, ks): tokens 128 mt .. +127 x all experts, h in k-blocks
// ks * kb_per .. +kb_per of 64. D_hi in TMEM columns 0.., D_lo in 256..
__global__ void __launch_bounds__(RTC_THREADS, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int E,
                    int NP, int kb_per, int nstage, float* __restrict__ approx, DevStatus* status,
                    long long wait_limit, int inject_stall) {
    constexpr int A_BYTES = 128 * 128;
    const int B_BYTES = 2 * NP * 128;
    const int STAGE = A_BYTES + B_BYTES;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[RTC_MAX_STAGES], empty_bar[RTC_MAX_STAGES], tfull_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    volatile int* abort_flag = &s_abort;
    const int mt = blockIdx.x, ks = blockIdx.y;
    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        ptx::mbar_init(&tfull_bar, 1);
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmX);
        ptx::prefetch_tmap(&tmW);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&s_tmem, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        if (lane == 0 && !inject_stall) {       // testing hook: no loads, so the waits below run out
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = 0; kb < kb_per; ++kb) {
                if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, wait_limit, status, 21u)) break;
                ptx::mbar_arrive_expect_tx(&full_bar[stage], static_cast<uint32_t>(STAGE));
                uint8_t* st = base + stage * STAGE;
                const int kx = (ks * kb_per + kb) * 64;
                ptx::tma_load_2d(st, &tmX, &full_bar[stage], kx, mt * 128);
                ptx::tma_load_2d(st + A_BYTES, &tmW, &full_bar[stage], kx, 0);
                ptx::tma_load_2d(st + A_BYTES + NP * 128, &tmW, &full_bar[stage], kx, WS_ROWS);
                if (++stage == nstage) { stage = 0; phase ^= 1u; }
            }
            if (*abort_flag) {
                // every armed stage's copies land before the CTA may leave
                for (int s = 0; s < nstage; ++s) {
                    const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
                    const long long t0 = clock64();
                    while (!ptx::mbar_try_wait(&full_bar[s], par) && clock64() - t0 < wait_limit) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = ptx::instr_desc(128, NP, 1u);
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = 0; kb < kb_per; ++kb) {
                if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag, wait_limit, status, 22u)) break;
                ptx::tc_fence_after();
                const uint32_t a = ptx::smem_u32(base + stage * STAGE);
                const uint32_t b = a + A_BYTES;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ad = ptx::smem_desc_sw<128>(a + k * 32);
                    const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
                    ptx::mma_f16(tmem, ad, ptx::smem_desc_sw<128>(b + k * 32), idesc, acc);
                    ptx::mma_f16(tmem + 256, ad, ptx::smem_desc_sw<128>(b + NP * 128 + k * 32), idesc, acc);
                }
                ptx::mma_commit(&empty_bar[stage]);
                if (++stage == nstage) { stage = 0; phase ^= 1u; }
            }
            // completes once every MMA issued above has finished; waited for here
            // as well, so that its arrival lands before the CTA may leave
            ptx::mma_commit(&tfull_bar);
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&tfull_bar, 0u) && clock64() - t0 < wait_limit) {
            }
        }
    } else {
        const int sub = warp & 3;
        int ok = 0;
        if (lane == 0) ok = ptx::mbar_wait(&tfull_bar, 0u, abort_flag, wait_limit, status, 23u) && !*abort_flag;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok) {
            ptx::tc_fence_after();
            const int row = mt * 128 + sub * 32 + lane;
            float* out = approx + (static_cast<size_t>(ks) * T + row) * E;
            const uint32_t tl = tmem + (static_cast<uint32_t>(sub * 32) << 16);
            for (int c = 0; c < NP / 32; ++c) {
                uint32_t h[32], l[32];
                ptx::tmem_ld_32x32b_x32(tl + c * 32, h);
                ptx::tmem_ld_32x32b_x32(tl + 256 + c * 32, l);
                ptx::tmem_ld_wait(h);
                ptx::tmem_ld_wait(l);
                if (row < T) {
                    if ((E & 3) == 0 && c * 32 + 32 <= E) {
                        // rows of E floats start on 16-byte boundaries
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(out + c * 32 + j) =
                                make_float4(__fadd_rn(__uint_as_float(h[j]), __uint_as_float(l[j])),
                                            __fadd_rn(__uint_as_float(h[j + 1]), __uint_as_float(l[j + 1])),
                                            __fadd_rn(__uint_as_float(h[j + 2]), __uint_as_float(l[j + 2])),
                                            __fadd_rn(__uint_as_float(h[j + 3]), __uint_as_float(l[j + 3])));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j < E)
                                out[c * 32 + j] = __fadd_rn(__uint_as_float(h[j]), __uint_as_float(l[j]));
                    }
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- C. candidates
// One warp per token. cand_n[t] = |S| (every expert when the token's bound is
// not usable); cand[t][0 .. min(|S|, RV_MAXC)) the candidate ids, ascending.
// A token whose |S| <= RV_MAXC also appends each pair (t, slot) to its expert's
// bucket: bucket[e][bcnt[e * RV_CPAD]++] = t * RV_MAXC + slot. Each counter sits
// on a cache line of its own, so that the atomics spread over the L2 slices.
// The order inside a bucket is that of the atomics; every pair's result is
// formed on its own, so it does not matter.
__global__ void __launch_bounds__(256) route_candidates_kernel(const float* __restrict__ approx, int KS,
                                                               const float* __restrict__ bias,
                                                               const float* __restrict__ nw,
                                                               const uint16_t* __restrict__ x, int T, int H, int E,
                                                               int K, int32_t* __restrict__ cand_n,
                                                               int32_t* __restrict__ cand,
                                                               int32_t* __restrict__ bcnt,
                                                               int32_t* __restrict__ bucket) {
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    // ||x_t||_2 (bf16 -> fp32 is exact)
    float ss = 0.0f;
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
    for (int i0 = lane; i0 < H / 8; i0 += 32 * 8) {
        uint4 q[8];                              // eight loads in flight per lane
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u;
            q[u] = i < H / 8 ? xr[i] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
                ss = fmaf(a, a, ss);
                ss = fmaf(b, b, ss);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    const float nx = sqrtf(ss) * 1.00390625f;
    bool usable = isfinite(nx);
    constexpr int J = 8;                        // E <= 256
    float key[J], eps[J];
    float eps_max = 0.0f;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        key[j] = -INFINITY;
        eps[j] = 0.0f;
        if (e < E) {
            float av[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) av[k] = k < KS ? approx[(static_cast<size_t>(k) * T + t) * E + e] : 0.0f;
            float a = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < KS) a = __fadd_rn(a, av[k]);
            usable = usable && isfinite(a);
            const float kv = bias != nullptr ? __fadd_rn(a, bias[e]) : a;
            key[j] = rank_key(kv);
            const float ej = RV_C * (nx * nw[e]) + 9.5367431640625e-07f * fabsf(kv);   // + 2^-20 |key|
            eps[j] = ej;
            eps_max = fmaxf(eps_max, ej);
        }
    }
    usable = __all_sync(0xFFFFFFFFu, usable);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) eps_max = fmaxf(eps_max, __shfl_xor_sync(0xFFFFFFFFu, eps_max, off));
    // Tk: the K-th largest approximate key
    unsigned taken = 0;
    float tk = INFINITY;
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < J; ++j) {
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
        tk = bv;
    }
    const float lim = tk - eps_max;             // -inf when Tk is -inf: every expert
    usable = usable && isfinite(eps_max);
    int n = 0;
    int slot[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        const bool c = e < E && (!usable || key[j] + eps[j] >= lim);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, c);
        slot[j] = c ? n + __popc(m & ((1u << lane) - 1u)) : RV_MAXC;
        if (slot[j] < RV_MAXC) cand[static_cast<size_t>(t) * RV_MAXC + slot[j]] = e;
        n += __popc(m);
    }
    if (lane == 0) cand_n[t] = usable ? n : E + 1;    // E + 1: not usable, every logit in step E
    if (usable && n <= RV_MAXC) {
        // every atomic of the lane is issued before the first result is used
        int pos[J];
#pragma unroll
        for (int j = 0; j < J; ++j)
            pos[j] = slot[j] < RV_MAXC ? atomicAdd(&bcnt[(lane + 32 * j) * RV_CPAD], 1) : -1;
#pragma unroll
        for (int j = 0; j < J; ++j)
            if (pos[j] >= 0) bucket[static_cast<size_t>(lane + 32 * j) * T + pos[j]] = t * RV_MAXC + slot[j];
    }
}

// ---------------------------------------------------------------- D. verify
// A warp item is (segment s, expert e, 32 of e's bucketed pairs); lane = pair
// (t, c). The segment is taken in chunks of RV_KC h. For each chunk the warp
// copies its 32 tokens' activations (8 lanes per 128-byte row, coalesced) and
// the expert's RV_KC weights into one of its two shared-memory buffers with
// cp.async; while one buffer is multiplied the next chunk (of this item, or
// the first of the warp's next item) is in flight. Each lane reads its own row
// back (row pitch 144 bytes: the 8 lanes of a quarter-warp hit distinct bank
// groups), the weights as broadcasts, and extends its fma chain. Items are
// numbered segment-major, so the activations in use at a time are one
// segment's columns of x (T x 512 bytes), which stay in L2.
// pc[s][t][c] = segment partial of candidate c.
constexpr int RV_KC = 64;                   // h per chunk
constexpr int RV_PITCH = RV_KC * 2 + 16;    // bytes per staged activation row
constexpr int RV_WARPS = 4;                 // warps per block
constexpr int RV_BUF = 32 * RV_PITCH + RV_KC * 4;   // a chunk: 32 rows, then the weights

__device__ __forceinline__ void rv_cp16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// the pairs of one item, as this lane sees them
struct RvItem {
    int s, e, t, c;
    bool valid;
    int rowtok[8];                          // tokens of the rows this lane copies
};

__device__ __forceinline__ RvItem rv_item(int item, int per_seg, const int* pre, int E, int T,
                                          const int32_t* __restrict__ bcnt, const int32_t* __restrict__ bucket,
                                          int lane) {
    RvItem it;
    it.s = item / per_seg;
    const int r = item - it.s * per_seg;
    int lo = 0, hi = E;                     // pre[lo] <= r < pre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= r) lo = mid;
        else hi = mid;
    }
    it.e = lo;
    const int p = (r - pre[lo]) * 32 + lane;
    it.valid = p < bcnt[lo * RV_CPAD];
    const int code = it.valid ? bucket[static_cast<size_t>(lo) * T + p] : 0;
    it.t = code / RV_MAXC;
    it.c = code % RV_MAXC;
    return it;
}

// the tokens of the rows this lane copies (apart from rv_item so that the
// bucket load of the next item is waited for only when its first chunk is
// copied)
__device__ __forceinline__ void rv_rows(RvItem& it, int lane) {
#pragma unroll
    for (int j = 0; j < 8; ++j) it.rowtok[j] = __shfl_sync(0xFFFFFFFFu, it.t, (lane >> 3) + 4 * j);
}

// chunk kc of an item into the buffer at `dst` (shared-memory address)
__device__ __forceinline__ void rv_copy(const RvItem& it, int kc, uint32_t dst, const uint16_t* __restrict__ x,
                                        const float* __restrict__ wr, int H, int lane) {
    const int h0 = it.s * RV_SEG + kc * RV_KC;
    const int piece = lane & 7;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        rv_cp16(dst + ((lane >> 3) + 4 * j) * RV_PITCH + piece * 16,
                x + static_cast<size_t>(it.rowtok[j]) * H + h0 + piece * 8);
    if (lane < RV_KC / 4) rv_cp16(dst + 32 * RV_PITCH + lane * 16, wr + static_cast<size_t>(it.e) * H + h0 + lane * 4);
}

__global__ void __launch_bounds__(RV_WARPS * 32) route_verify_kernel(const uint16_t* __restrict__ x,
                                                                     const float* __restrict__ wr, int T, int H,
                                                                     int E, const int32_t* __restrict__ bcnt,
                                                                     const int32_t* __restrict__ bucket,
                                                                     float* __restrict__ pc) {
    extern __shared__ __align__(16) uint8_t rv_x[];    // [RV_WARPS][2][RV_BUF]
    __shared__ int pre[257];                // pre[e]: first item of expert e within a segment
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp == 0) {
        int v[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            v[j] = e < E ? (bcnt[e * RV_CPAD] + 31) >> 5 : 0;
            sum += v[j];
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        int run = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            pre[lane * 8 + j] = run;
            run += v[j];
        }
        if (lane == 31) pre[256] = incl;
    }
    __syncthreads();
    const int per_seg = pre[256];
    const int total = per_seg * (H / RV_SEG);
    const int nwarp = gridDim.x * RV_WARPS;
    const uint32_t sbuf = static_cast<uint32_t>(__cvta_generic_to_shared(rv_x)) + warp * 2 * RV_BUF;
    const uint8_t* gbuf = rv_x + warp * 2 * RV_BUF;
    int item = blockIdx.x * RV_WARPS + warp;
    if (item >= total) return;
    RvItem cur = rv_item(item, per_seg, pre, E, T, bcnt, bucket, lane);
    rv_rows(cur, lane);
    rv_copy(cur, 0, sbuf, x, wr, H, lane);
    asm volatile("cp.async.commit_group;" ::: "memory");
    int b = 0;
    constexpr int NKC = RV_SEG / RV_KC;
    while (true) {
        const int nitem = item + nwarp;
        const bool more = nitem < total;
        RvItem nxt = cur;
        if (more) nxt = rv_item(nitem, per_seg, pre, E, T, bcnt, bucket, lane);
        float acc = 0.0f;
#pragma unroll 1
        for (int kc = 0; kc < NKC; ++kc) {
            // the next chunk's copy goes out before this one is multiplied
            if (kc + 1 < NKC) rv_copy(cur, kc + 1, sbuf + (b ^ 1) * RV_BUF, x, wr, H, lane);
            else if (more) {
                rv_rows(nxt, lane);
                rv_copy(nxt, 0, sbuf + (b ^ 1) * RV_BUF, x, wr, H, lane);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 1;" ::: "memory");
            __syncwarp();                       // every lane's pieces of this chunk have landed
            const uint8_t* row = gbuf + b * RV_BUF + lane * RV_PITCH;
            const float* wc = reinterpret_cast<const float*>(gbuf + b * RV_BUF + 32 * RV_PITCH);
#pragma unroll
            for (int q = 0; q < RV_KC / 8; ++q) {
                const uint4 xv = *reinterpret_cast<const uint4*>(row + q * 16);
                const float4 wa = *reinterpret_cast<const float4*>(wc + q * 8);
                const float4 wb = *reinterpret_cast<const float4*>(wc + q * 8 + 4);
                // bf16 -> fp32 is exact; h ascending within the segment
                acc = __fmaf_rn(__uint_as_float(xv.x << 16), wa.x, acc);
                acc = __fmaf_rn(__uint_as_float(xv.x & 0xFFFF0000u), wa.y, acc);
                acc = __fmaf_rn(__uint_as_float(xv.y << 16), wa.z, acc);
                acc = __fmaf_rn(__uint_as_float(xv.y & 0xFFFF0000u), wa.w, acc);
                acc = __fmaf_rn(__uint_as_float(xv.z << 16), wb.x, acc);
                acc = __fmaf_rn(__uint_as_float(xv.z & 0xFFFF0000u), wb.y, acc);
                acc = __fmaf_rn(__uint_as_float(xv.w << 16), wb.z, acc);
                acc = __fmaf_rn(__uint_as_float(xv.w & 0xFFFF0000u), wb.w, acc);
            }
            __syncwarp();                       // the buffer is copied into again on the next chunk
            b ^= 1;
        }
        if (cur.valid) pc[(static_cast<size_t>(cur.s) * T + cur.t) * RV_MAXC + cur.c] = acc;
        if (!more) break;
        item = nitem;
        cur = nxt;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------- E. select
// One warp per token: exact logits of the candidates (or of every expert when
// the token has no usable candidate set), then route.cu's ranking and weights.
__global__ void __launch_bounds__(256) route_select_kernel(const float* __restrict__ pc, int nseg,
                                                           const int32_t* __restrict__ cand_n,
                                                           const int32_t* __restrict__ cand,
                                                           const uint16_t* __restrict__ x,
                                                           const float* __restrict__ wr,
                                                           const float* __restrict__ bias, int T, int H, int E,
                                                           int K, int shared_id, float shared_weight,
                                                           float routed_scale, int bias_select_only,
                                                           int32_t* __restrict__ ids, float* __restrict__ wts) {
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const int S = K + (shared_id >= 0 ? 1 : 0);
    const int n = cand_n[t];
    const bool full = n > RV_MAXC;
    const int J = full ? (E + 31) / 32 : 1;     // experts per lane
    constexpr int JM = 8;
    float key[JM], wlog[JM];
    int eid[JM];
#pragma unroll
    for (int j = 0; j < JM; ++j) {
        key[j] = -INFINITY;
        wlog[j] = -INFINITY;
        eid[j] = 0x7FFFFFFF;
        if (j >= J) continue;
        int e = -1;
        float tot = 0.0f;
        if (full) {
            e = lane + 32 * j;
            if (e < E) {
                // the fixed order: segment chains from +0, segment sums in order
                const uint16_t* xr = x + static_cast<size_t>(t) * H;
                const float* w = wr + static_cast<size_t>(e) * H;
                for (int sg = 0; sg < nseg; ++sg) {
                    float r = 0.0f;
                    for (int h = sg * RV_SEG; h < (sg + 1) * RV_SEG; ++h)
                        r = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(xr[h]) << 16), w[h], r);
                    tot = __fadd_rn(tot, r);
                }
            } else {
                e = -1;
            }
        } else if (lane < n) {
            e = cand[static_cast<size_t>(t) * RV_MAXC + lane];
            for (int sg = 0; sg < nseg; ++sg)
                tot = __fadd_rn(tot, pc[(static_cast<size_t>(sg) * T + t) * RV_MAXC + lane]);
        }
        if (e >= 0) {
            const float raw = isnan(tot) ? -INFINITY : tot;
            const float tj = bias != nullptr ? __fadd_rn(tot, bias[e]) : tot;
            const float v = rank_key(tj);
            key[j] = v;
            wlog[j] = (bias_select_only && bias != nullptr) ? raw : v;
            eid[j] = e;
        }
    }
    unsigned taken = 0;
    float sel_w[32];
    int my_id = -1;
    float my_w = 0.0f;
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF, bj = 0;
#pragma unroll
        for (int j = 0; j < JM; ++j)
            if (j < J && eid[j] != 0x7FFFFFFF && !((taken >> j) & 1u) && better(key[j], eid[j], bv, bi)) {
                bv = key[j];
                bi = eid[j];
                bj = j;
            }
        // owner lane of the winner: carried with it through the reduction
        int bl = lane * JM + bj;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            const int ol = __shfl_xor_sync(0xFFFFFFFFu, bl, off);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; bl = ol; }
        }
        const int owner = bl / JM, oj = bl % JM;
        if (owner == lane) taken |= 1u << oj;
        float wv = 0.0f;
#pragma unroll
        for (int j = 0; j < JM; ++j)
            if (j == oj) wv = wlog[j];
        wv = __shfl_sync(0xFFFFFFFFu, wv, owner);
        sel_w[k] = wv;
        if (lane == k) { my_id = bi; my_w = wv; }
    }
    float m = -INFINITY, den = 0.0f;
    for (int k = 0; k < K; ++k) m = fmaxf(m, sel_w[k]);
    for (int k = 0; k < K; ++k) den += expf(sel_w[k] - m);
    if (lane < K) {
        ids[static_cast<size_t>(t) * S + lane] = my_id;
        wts[static_cast<size_t>(t) * S + lane] = routed_scale * (expf(my_w - m) / den);
    }
    if (shared_id >= 0 && lane == 0) {
        ids[static_cast<size_t>(t) * S + K] = shared_id;
        wts[static_cast<size_t>(t) * S + K] = shared_weight;
    }
}

inline size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

std::atomic<int> g_inject_route{0};

int rv_split(int H) {
    const int nkb = H / 64, nseg = H / RV_SEG;
    if (nseg >= 4 && nkb % 4 == 0) return 4;
    if (nseg >= 2 && nkb % 2 == 0) return 2;
    return 1;
}

}  // namespace

void route_tc_inject_stall(int n_calls) { g_inject_route.store(n_calls); }

bool route_tc_applies(const moe_shape& s, const float* logits_out) {
    return logits_out == nullptr && s.act_dtype == MOE_BF16 && s.renormalize != 0 && s.T > 256 &&
           s.n_routed >= 32 && s.n_routed <= 256 && s.top_k <= 16 && s.H % RV_SEG == 0 && s.H <= 8192;
}

size_t route_tc_scratch_bytes(int T, int H, int E) {
    if (E < 32 || E > 256 || T <= 256 || H % RV_SEG != 0 || H > 8192) return 0;
    return align256(static_cast<size_t>(2) * WS_ROWS * H * 2) + align256(256 * 4) +
           align256(static_cast<size_t>(T) * 4) + align256(static_cast<size_t>(T) * RV_MAXC * 4) +
           align256(256 * RV_CPAD * 4) + align256(static_cast<size_t>(E) * T * 4);
}

cudaError_t launch_route_tc(const moe_shape& s, const void* x, const float* wr, const float* bias, int32_t* ids,
                            float* wts, float* partials, void* scratch, int shared_id, DevStatus* status,
                            cudaStream_t st) {
    const int T = s.T, H = s.H, E = s.n_routed, K = s.top_k;
    const int NP = (E + 31) & ~31;
    const int KS = rv_split(H);
    const int nseg = H / RV_SEG;
    uint8_t* p = static_cast<uint8_t*>(scratch);
    __nv_bfloat16* wsplit = reinterpret_cast<__nv_bfloat16*>(p);
    p += align256(static_cast<size_t>(2) * WS_ROWS * H * 2);
    float* nw = reinterpret_cast<float*>(p);
    p += align256(256 * 4);
    int32_t* cand_n = reinterpret_cast<int32_t*>(p);
    p += align256(static_cast<size_t>(T) * 4);
    int32_t* cand = reinterpret_cast<int32_t*>(p);
    p += align256(static_cast<size_t>(T) * RV_MAXC * 4);
    int32_t* bcnt = reinterpret_cast<int32_t*>(p);
    p += align256(256 * RV_CPAD * 4);
    int32_t* bucket = reinterpret_cast<int32_t*>(p);
    // the router partials buffer ([H/256][T][E] floats) holds the approximate
    // slices first ([KS][T][E], KS <= H/256) and the candidates' exact segment
    // partials after them ([H/256][T][RV_MAXC], RV_MAXC <= E)
    float* approx = partials;
    float* pc = partials;

    CUtensorMap tmX, tmW;
    if (!make_map_bf16_2d(&tmX, x, H, T, 128) || !make_map_bf16_2d(&tmW, wsplit, H, 2 * WS_ROWS, NP))
        return cudaErrorInvalidValue;
    {
        ProfileScope ps("route_split", st);
        route_split_kernel<<<NP, 256, 0, st>>>(wr, E, H, wsplit, nw, bcnt);
        note_launch();
    }
    {
        const int stage = 128 * 128 + 2 * NP * 128;
        const int nstage = std::min(RTC_MAX_STAGES, RTC_RING / stage);
        const int smem = std::max(nstage * stage + 1024, RTC_MIN_SMEM);
        static int attr = 0;
        if (smem > attr) {
            const cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       RTC_RING + 2048);
            if (e != cudaSuccess) return e;
            attr = RTC_RING + 2048;
        }
        int inject = 0;
        {
            int cur = g_inject_route.load();
            while (cur > 0 && !g_inject_route.compare_exchange_weak(cur, cur - 1)) {
            }
            inject = cur > 0 ? 1 : 0;
        }
        ProfileScope ps("route_approx", st);
        route_tc_kernel<<<dim3((T + 127) / 128, KS), RTC_THREADS, smem, st>>>(
            tmX, tmW, T, E, NP, H / 64 / KS, nstage, approx, status, inject ? (20ll << 20) : (4ll << 30), inject);
        note_launch();
    }
    {
        ProfileScope ps("route_candidates", st);
        route_candidates_kernel<<<(T * 32 + 255) / 256, 256, 0, st>>>(approx, KS, bias, nw,
                                                                     static_cast<const uint16_t*>(x), T, H, E, K,
                                                                     cand_n, cand, bcnt, bucket);
        note_launch();
    }
    {
        static int grid = 0;
        if (grid == 0) {
            int dev = 0, nsm = 0, per = 0;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
            cudaError_t e = cudaFuncSetAttribute(route_verify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 RV_WARPS * 2 * RV_BUF);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, route_verify_kernel, RV_WARPS * 32,
                                                                  RV_WARPS * 2 * RV_BUF);
            if (e != cudaSuccess) return e;
            grid = std::max(1, nsm * per);
        }
        ProfileScope ps("route_verify", st);
        route_verify_kernel<<<grid, RV_WARPS * 32, RV_WARPS * 2 * RV_BUF, st>>>(static_cast<const uint16_t*>(x), wr,
                                                                               T, H, E, bcnt, bucket, pc);
        note_launch();
    }
    {
        ProfileScope ps("route_topk", st);
        route_select_kernel<<<(T * 32 + 255) / 256, 256, 0, st>>>(pc, nseg, cand_n, cand,
                                                                 static_cast<const uint16_t*>(x), wr, bias, T, H, E,
                                                                 K, shared_id, s.shared_weight, s.routed_scale,
                                                                 s.bias_select_only, ids, wts);
        note_launch();
    }
    return cudaGetLastError();
}

}  // namespace sre
