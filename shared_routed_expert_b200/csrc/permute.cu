// Token permutation for the single routed-MoE pass of the fused layer.
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1: the shared
// expert joins the routed experts so that one routed-MoE pass computes all
// top-(K+1) slots. That pass needs the R = T*S slots grouped by expert:
// counts, exclusive offsets and a permutation, experts in id order and, inside
// an expert, stable by flat slot index (so the result is deterministic and the
// shared expert's block is tokens 0..T-1 in order).
//
// Three kernels, no atomics on the order-defining path:
//   hist:    per 512-slot chunk, per-expert counts (shared-memory histogram)
//   scan:    one block; warp-parallel scans over chunks (per expert) and over
//            experts give each chunk's first row inside each expert's group,
//            the counts, the offsets and the GEMM tile prefix
//   scatter: one warp per chunk walks its slots in order, 32 at a time;
//            __match_any_sync ranks equal experts inside a group.
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace sre {

namespace {

// per 512-slot chunk c: counts of each expert -> chunk_hist[e][c] (expert-major)
__global__ void __launch_bounds__(128) perm_hist_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                        int n_chunks, int32_t* __restrict__ chunk_hist,
                                                        DevStatus* status) {
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int base = blockIdx.x * kPermChunk;
#pragma unroll
    for (int i = threadIdx.x; i < kPermChunk; i += 128) {
        const int f = base + i;
        if (f < R) {
            const int e = ids[f];
            if (e < 0 || e >= E) report(status, MOE_ERR_DEVICE, static_cast<unsigned>(f));
            else atomicAdd(&hist[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_hist[static_cast<size_t>(e) * n_chunks + blockIdx.x] = hist[e];
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

// One block of 1024 threads. Warp w owns experts w, w+32, ...: the expert's
// row of chunk counts is read 32 consecutive chunks per instruction, every
// load of the row in flight before the scans (rows of up to 32 * kScanVals
// chunks; longer rows go 32 chunks per round trip). Writes
// chunk_hist[e][c] <- sum_{c' < c} chunk_hist[e][c'] (the chunk's first row
// inside expert e's group) and counts[e]; warp 0 then scans the counts into
// offsets and the GEMM tile prefix tile_off[e] = sum_{e' < e} ceil(counts[e'] /
// kTileM). The scatter adds offsets[e].
constexpr int kScanVals = 12;    // 32-chunk groups per row held in registers (n_chunks <= 384)
__global__ void __launch_bounds__(1024) perm_scan_kernel(int n_chunks, int E, int32_t* __restrict__ chunk_hist,
                                                         int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ tile_off) {
    __shared__ int32_t s_cnt[1024];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = ceil_div(n_chunks, 32);
    for (int e = warp; e < E; e += 32) {
        int32_t* row = chunk_hist + static_cast<size_t>(e) * n_chunks;
        int carry = 0;
        if (groups <= kScanVals) {
            int v[kScanVals];
#pragma unroll
            for (int g = 0; g < kScanVals; ++g) {
                const int c = g * 32 + lane;
                v[g] = (g < groups && c < n_chunks) ? row[c] : 0;
            }
#pragma unroll
            for (int g = 0; g < kScanVals; ++g) {
                if (g < groups) {
                    const int c = g * 32 + lane;
                    const int inc = warp_inclusive_scan(v[g], lane);
                    if (c < n_chunks) row[c] = carry + inc - v[g];
                    carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
                }
            }
        } else {
            for (int cb = 0; cb < n_chunks; cb += 32) {
                const int c = cb + lane;
                const int v = (c < n_chunks) ? row[c] : 0;
                const int inc = warp_inclusive_scan(v, lane);
                if (c < n_chunks) row[c] = carry + inc - v;
                carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
            }
        }
        if (lane == 0) s_cnt[e] = carry;
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0, tcarry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int c = (e < E) ? s_cnt[e] : 0;
            const int tc = ceil_div(c, kTileM);
            const int inc = warp_inclusive_scan(c, lane);
            const int tinc = warp_inclusive_scan(tc, lane);
            if (e < E) {
                counts[e] = c;
                offsets[e] = carry + inc - c;
                tile_off[e] = tcarry + tinc - tc;
            }
            carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
            tcarry += __shfl_sync(0xFFFFFFFFu, tinc, 31);
        }
        if (lane == 0) {
            offsets[E] = carry;
            tile_off[E] = tcarry;
        }
    }
}

// One warp per chunk: the chunk's ids are loaded first (all loads in flight
// at once), then ranked 32 at a time in slot order; __match_any_sync groups
// equal experts, the rank inside a group is the count of lower lanes.
constexpr int kPermPerLane = kPermChunk / 32;
__global__ void __launch_bounds__(32) perm_scatter_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                          int n_chunks,
                                                          const int32_t* __restrict__ chunk_base,
                                                          const int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv) {
    extern __shared__ int32_t next[];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32)
        next[e] = offsets[e] + chunk_base[static_cast<size_t>(e) * n_chunks + blockIdx.x];
    const int base = blockIdx.x * kPermChunk;
    int my[kPermPerLane];
#pragma unroll
    for (int g = 0; g < kPermPerLane; ++g) {
        const int f = base + g * 32 + lane;
        int e = (f < R) ? ids[f] : -1;
        my[g] = (e < 0 || e >= E) ? -1 : e;
    }
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int g = 0; g < kPermPerLane; ++g) {
        const int f = base + g * 32 + lane;
        const int e = my[g];
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
        if (e >= 0) {
            const int row = next[e] + __popc(peers & lt);
            perm[row] = f;
            inv[f] = row;
        }
        __syncwarp();
        if (e >= 0 && (peers & lt) == 0) next[e] += __popc(peers);   // lowest lane of the group
        __syncwarp();
    }
}

// The three kernels above as one cooperative launch (every block resident at
// once), one block of kFusedWarps warps per 512-slot chunk, E <= 256:
//   1. warp w counts the experts of its 64 slots (chunk slots 64 w .. 64 w + 63)
//      and the block writes the chunk's column chunk_hist[.][c];
//   2. grid barrier: each block adds 1 to *bar (zeroed before the launch) and
//      waits, bounded, until it reads n_chunks (on expiry MOE_ERR_TIMEOUT and
//      the block returns);
//   3. warp w sums rows e = w, w + 8, ... of chunk_hist: the expert's rows in
//      chunks before c and in all chunks; a scan over experts turns the totals
//      into offsets (block 0 also writes counts, offsets and tile_off), and a
//      scan over the block's warps gives each warp its first row per expert;
//   4. each warp ranks its slots in slot order with __match_any_sync.
// Rows follow slot order inside each expert (chunk, then warp, then lane), as
// in the three kernels.
constexpr int kFusedWarps = kPermChunk / 64;
__global__ void __launch_bounds__(kFusedWarps * 32) perm_fused_kernel(
    const int32_t* __restrict__ ids, int R, int E, int n_chunks, int32_t* __restrict__ chunk_hist,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ tile_off,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, unsigned* bar, long long wait_limit,
    DevStatus* status) {
    __shared__ int32_t s_w[kFusedWarps][256];   // per warp: slots of expert e, then its first row
    __shared__ int32_t s_pre[256], s_tot[256];
    __shared__ int s_ok;
    const int c = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < kFusedWarps * 256; i += kFusedWarps * 32) s_w[i / 256][i % 256] = 0;
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    int my[2];
    unsigned peers[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int f = c * kPermChunk + warp * 64 + g * 32 + lane;
        int e = (f < R) ? ids[f] : -1;
        if (f < R && (e < 0 || e >= E)) report(status, MOE_ERR_DEVICE, static_cast<unsigned>(f));
        if (e >= E) e = -1;
        my[g] = e < 0 ? -1 : e;
        peers[g] = __match_any_sync(0xFFFFFFFFu, my[g]);
    }
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        if (my[g] >= 0 && (peers[g] & lt) == 0) s_w[warp][my[g]] += __popc(peers[g]);   // one leader per expert
        __syncwarp();
    }
    __syncthreads();
    for (int e = tid; e < E; e += kFusedWarps * 32) {
        int h = 0;
#pragma unroll
        for (int w = 0; w < kFusedWarps; ++w) h += s_w[w][e];
        chunk_hist[static_cast<size_t>(e) * n_chunks + c] = h;
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        atomicAdd(bar, 1u);
        volatile int never = 0;
        s_ok = ptx::counter_wait(bar, static_cast<unsigned>(n_chunks), &never, wait_limit, status, 30u);
    }
    __syncthreads();
    if (!s_ok) return;
    __threadfence();
    {
        // warp w: experts w + kFusedWarps i; every expert's loads of a 32-chunk
        // round are in flight together
        constexpr int IPW = 256 / kFusedWarps;
        int pre[IPW], tot[IPW];
#pragma unroll
        for (int i = 0; i < IPW; ++i) pre[i] = tot[i] = 0;
        for (int c0 = 0; c0 < n_chunks; c0 += 32) {
            const int cc = c0 + lane;
#pragma unroll
            for (int i = 0; i < IPW; ++i) {
                const int e = warp + kFusedWarps * i;
                if (e < E && cc < n_chunks) {
                    const int v = __ldcg(chunk_hist + static_cast<size_t>(e) * n_chunks + cc);
                    tot[i] += v;
                    pre[i] += cc < c ? v : 0;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < IPW; ++i) {
            const int e = warp + kFusedWarps * i;
            if (e >= E) break;                  // warp-uniform
            int t = tot[i], p = pre[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                t += __shfl_xor_sync(0xFFFFFFFFu, t, off);
                p += __shfl_xor_sync(0xFFFFFFFFu, p, off);
            }
            if (lane == 0) {
                s_pre[e] = p;
                s_tot[e] = t;
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0, tcarry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int n = (e < E) ? s_tot[e] : 0;
            const int tc = ceil_div(n, kTileM);
            const int inc = warp_inclusive_scan(n, lane);
            const int tinc = warp_inclusive_scan(tc, lane);
            if (e < E) {
                if (c == 0) {
                    counts[e] = n;
                    offsets[e] = carry + inc - n;
                    tile_off[e] = tcarry + tinc - tc;
                }
                s_pre[e] += carry + inc - n;        // the chunk's first row of expert e
            }
            carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
            tcarry += __shfl_sync(0xFFFFFFFFu, tinc, 31);
        }
        if (lane == 0 && c == 0) {
            offsets[E] = carry;
            tile_off[E] = tcarry;
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kFusedWarps * 32) {   // exclusive scan over the block's warps
        int run = s_pre[e];
#pragma unroll
        for (int w = 0; w < kFusedWarps; ++w) {
            const int n = s_w[w][e];
            s_w[w][e] = run;
            run += n;
        }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int f = c * kPermChunk + warp * 64 + g * 32 + lane;
        const int e = my[g];
        if (e >= 0) {
            const int row = s_w[warp][e] + __popc(peers[g] & lt);
            perm[row] = f;
            inv[f] = row;
        }
        __syncwarp();
        if (e >= 0 && (peers[g] & lt) == 0) s_w[warp][e] += __popc(peers[g]);
        __syncwarp();
    }
}

// Small batches (R <= kSmallR slots, E <= kSmallE experts): the whole
// permutation in one block of 1024 threads, same result as the three kernels
// above. Counts by shared-memory histogram; offsets and tile prefix by a warp
// scan; then rounds of 1024 slots in slot order: warp w ranks its 32 slots
// with __match_any_sync, per-expert counts of the warps are scanned across
// warps, and each slot's row is run[e] + (slots of e in lower warps) + rank.
constexpr int kSmallR = 8192;
constexpr int kSmallE = 256;
__global__ void __launch_bounds__(1024) perm_small_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ tile_off,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv, DevStatus* status) {
    __shared__ int32_t s_cnt[kSmallE];
    __shared__ int32_t s_run[kSmallE];
    __shared__ int32_t s_w[32][kSmallE];      // per round: slots of expert e in warp w, then its first row
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < E; e += 1024) s_cnt[e] = 0;
    __syncthreads();
    for (int f = tid; f < R; f += 1024) {
        const int e = ids[f];
        if (e < 0 || e >= E) report(status, MOE_ERR_DEVICE, static_cast<unsigned>(f));
        else atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0, tcarry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int c = (e < E) ? s_cnt[e] : 0;
            const int tc = ceil_div(c, kTileM);
            const int inc = warp_inclusive_scan(c, lane);
            const int tinc = warp_inclusive_scan(tc, lane);
            if (e < E) {
                counts[e] = c;
                offsets[e] = carry + inc - c;
                tile_off[e] = tcarry + tinc - tc;
                s_run[e] = carry + inc - c;
            }
            carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
            tcarry += __shfl_sync(0xFFFFFFFFu, tinc, 31);
        }
        if (lane == 0) {
            offsets[E] = carry;
            tile_off[E] = tcarry;
        }
    }
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < R; base += 1024) {
        for (int i = tid; i < 32 * E; i += 1024) s_w[i / E][i % E] = 0;
        __syncthreads();
        const int f = base + tid;
        int e = (f < R) ? ids[f] : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
        if (e >= 0 && (peers & lt) == 0) s_w[warp][e] = __popc(peers);
        __syncthreads();
        for (int x = tid; x < E; x += 1024) {       // exclusive scan over warps, in warp order
            int run = s_run[x];
            for (int w = 0; w < 32; ++w) {
                const int c = s_w[w][x];
                s_w[w][x] = run;
                run += c;
            }
            s_run[x] = run;
        }
        __syncthreads();
        if (e >= 0) {
            const int row = s_w[warp][e] + __popc(peers & lt);
            perm[row] = f;
            inv[f] = row;
        }
        __syncthreads();
    }
}

// Xp[r] = x[perm[r] / S]: one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(int R, int S, int row_vecs,
                                                          const uint4* __restrict__ x,
                                                          const float* __restrict__ xscale,
                                                          const int32_t* __restrict__ perm,
                                                          uint4* __restrict__ xp,
                                                          float* __restrict__ xpscale,
                                                          const int32_t* __restrict__ skip) {
    const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= R) return;
    if (skip != nullptr && r >= skip[0] && r < skip[1]) return;
    const int f = perm[r];
    if (f < 0 || f >= R) return;          // a slot dropped for a bad id leaves no row
    const int t = f / S;
    const uint4* src = x + static_cast<size_t>(t) * row_vecs;
    uint4* dst = xp + static_cast<size_t>(r) * row_vecs;
    for (int i = lane; i < row_vecs; i += 32) dst[i] = src[i];
    if (xscale != nullptr && lane == 0) xpscale[r] = xscale[t];
}

// v / s correctly rounded, from y = RN(1 / s): Markstein's theorem (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990): q0 = RN(v y) lies within an ulp of v / s, the
// residual v - s q0 is then exact (one fma), and RN(q0 + r y) = RN(v / s),
// provided no intermediate underflows or overflows.
__device__ __forceinline__ float div_by_recip(float v, float s, float y) {
    const float q0 = __fmul_rn(v, y);
    const float r = __fmaf_rn(-q0, s, v);
    return __fmaf_rn(r, y, q0);
}

// One warp per row: amax (fp32), scale = amax / 448 (IEEE divide, amax = 0 -> 1),
// codes = E4M3_rn_satfinite(v / scale) with the quotient rounded as the IEEE
// divide rounds it: by div_by_recip when amax >= 2^-60 (then every quotient of
// 2^-11 or more, the only ones whose code depends on its last bit, has a normal
// residual; smaller ones are codes of +-0 either way), by the divide otherwise.
constexpr float kMarksteinMinAmax = 8.6736174e-19f;    // 2^-60

// the quantiser of a row whose largest magnitude is amax
struct RowQuant {
    float scale, y;
    bool by_recip;
};
__device__ __forceinline__ RowQuant row_quant(float amax) {
    RowQuant q;
    q.scale = (amax > 0.0f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
    q.by_recip = amax >= kMarksteinMinAmax && amax <= 3.4028235e38f;     // warp-uniform
    q.y = q.by_recip ? __frcp_rn(q.scale) : 0.0f;
    return q;
}

__device__ __forceinline__ float amax_bf16x8(float amax, const uint4 q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
    return amax;
}

// eight bf16 values -> eight E4M3 codes (round to nearest even, saturated to
// +-448; in order, little-endian); kRecip:
// the quotients by div_by_recip (rq.by_recip, decided once per row), else by
// the IEEE divide. Two quotients go through one paired conversion (the first
// in the low byte), the same rounding as one at a time.
template <bool kRecip>
__device__ __forceinline__ uint2 codes_bf16x8(const uint4 q, const RowQuant& rq) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
        float2 qv;
        if constexpr (kRecip) {
            qv = make_float2(div_by_recip(a, rq.scale, rq.y), div_by_recip(b, rq.scale, rq.y));
        } else {
            qv = make_float2(__fdiv_rn(a, rq.scale), __fdiv_rn(b, rq.scale));
        }
        const uint32_t two = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(qv, __NV_SATFINITE, __NV_E4M3));
        packed[j >> 1] |= two << ((j & 1) * 16);
    }
    return make_uint2(packed[0], packed[1]);
}

__global__ void __launch_bounds__(256) quant_rows_kernel(int rows, int cols,
                                                         const uint16_t* __restrict__ in,
                                                         uint8_t* __restrict__ codes,
                                                         float* __restrict__ scales) {
    const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const uint4* src = reinterpret_cast<const uint4*>(in + static_cast<size_t>(r) * cols);
    const int nv = cols / 8;
    float amax = 0.0f;
    for (int i = lane; i < nv; i += 32) amax = amax_bf16x8(amax, src[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const RowQuant rq = row_quant(amax);
    uint2* dst = reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * cols);
    if (rq.by_recip) {
        for (int i = lane; i < nv; i += 32) dst[i] = codes_bf16x8<true>(src[i], rq);
    } else {
        for (int i = lane; i < nv; i += 32) dst[i] = codes_bf16x8<false>(src[i], rq);
    }
    if (lane == 0) scales[r] = rq.scale;
}

// Token-major gather of the grouped pass's rows: one 128-thread block per token
// t reads its row once into registers (H <= kScatterMaxH bf16 values, a
// quarter of the row per warp) and writes it to the rows inv[t * S + k] of its
// slots, leaving out rows in [skip[0], skip[1]) (a group the GEMM reads from
// the token matrix directly) and slots without a row. Four warps per token
// keep the items small, so the grid has no tail of whole-row warps.
// kQuant (E4M3 layers): the row is quantised as quant_rows_kernel does it (the
// row's amax is a max, so its order does not matter) and its codes and scale go
// to the token matrix (xq, xscale) as well as to the slots' rows (xp,
// xpscale); otherwise the bf16 row itself is copied.
constexpr int kScatterThreads = 128;
constexpr int kScatterVec = 8;                  // 16-byte vectors per thread
constexpr int kScatterMaxH = kScatterVec * kScatterThreads * 8;

template <bool kQuant>
__global__ void __launch_bounds__(kScatterThreads) scatter_rows_kernel(int T, int S, int R, int H,
                                                                       const uint4* __restrict__ x,
                                                                       const int32_t* __restrict__ inv,
                                                                       const int32_t* __restrict__ skip,
                                                                       uint8_t* __restrict__ xq,
                                                                       float* __restrict__ xscale,
                                                                       void* __restrict__ xp,
                                                                       float* __restrict__ xpscale) {
    const int t = blockIdx.x;
    const int i = threadIdx.x;
    const int nv = H / 8;
    uint4 v[kScatterVec];
    const uint4* src = x + static_cast<size_t>(t) * nv;
#pragma unroll
    for (int j = 0; j < kScatterVec; ++j)
        if (j * kScatterThreads + i < nv) v[j] = src[j * kScatterThreads + i];
    const int s0 = skip != nullptr ? skip[0] : 0, s1 = skip != nullptr ? skip[1] : 0;
    const int32_t* tinv = inv + static_cast<size_t>(t) * S;
    if constexpr (kQuant) {
        __shared__ float s_amax[kScatterThreads / 32];
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < kScatterVec; ++j)
            if (j * kScatterThreads + i < nv) amax = amax_bf16x8(amax, v[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        if ((i & 31) == 0) s_amax[i >> 5] = amax;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kScatterThreads / 32; ++w) amax = fmaxf(amax, s_amax[w]);
        const RowQuant rq = row_quant(amax);
        uint2 c[kScatterVec];
        if (rq.by_recip) {
#pragma unroll
            for (int j = 0; j < kScatterVec; ++j)
                if (j * kScatterThreads + i < nv) c[j] = codes_bf16x8<true>(v[j], rq);
        } else {
#pragma unroll
            for (int j = 0; j < kScatterVec; ++j)
                if (j * kScatterThreads + i < nv) c[j] = codes_bf16x8<false>(v[j], rq);
        }
        uint2* dq = reinterpret_cast<uint2*>(xq + static_cast<size_t>(t) * H);
#pragma unroll
        for (int j = 0; j < kScatterVec; ++j)
            if (j * kScatterThreads + i < nv) dq[j * kScatterThreads + i] = c[j];
        if (i == 0) xscale[t] = rq.scale;
        for (int k = 0; k < S; ++k) {
            const int r = tinv[k];
            if (r < 0 || r >= R || (r >= s0 && r < s1)) continue;       // block-uniform
            uint2* d = reinterpret_cast<uint2*>(static_cast<uint8_t*>(xp) + static_cast<size_t>(r) * H);
#pragma unroll
            for (int j = 0; j < kScatterVec; ++j)
                if (j * kScatterThreads + i < nv) d[j * kScatterThreads + i] = c[j];
            if (i == 0) xpscale[r] = rq.scale;
        }
    } else {
        for (int k = 0; k < S; ++k) {
            const int r = tinv[k];
            if (r < 0 || r >= R || (r >= s0 && r < s1)) continue;       // block-uniform
            uint4* d = static_cast<uint4*>(xp) + static_cast<size_t>(r) * nv;
#pragma unroll
            for (int j = 0; j < kScatterVec; ++j)
                if (j * kScatterThreads + i < nv) d[j * kScatterThreads + i] = v[j];
        }
    }
}

}  // namespace

size_t permute_scratch_ints(int R, int E) {
    return static_cast<size_t>(ceil_div(R, kPermChunk)) * E;
}

// blocks of perm_fused_kernel that can be resident at once
int fused_capacity() {
    static int cap = -1;
    if (cap < 0) {
        int dev = 0, nsm = 0, per = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, perm_fused_kernel, kFusedWarps * 32, 0) !=
            cudaSuccess)
            per = 0;
        cap = nsm * per;
    }
    return cap;
}

cudaError_t launch_permute(int R, int E, const int32_t* ids, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* tile_off, int32_t* scratch,
                           DevStatus* st, cudaStream_t stream, unsigned* fused_bar) {
    if (R <= kSmallR && E <= kSmallE) {
        ProfileScope ps("permute_small", stream);
        perm_small_kernel<<<1, 1024, 0, stream>>>(ids, R, E, counts, offsets, tile_off, perm, inv, st);
        note_launch();
        return cudaGetLastError();
    }
    const int n_chunks = ceil_div(R, kPermChunk);
    if (fused_bar != nullptr && E <= 256 && n_chunks <= fused_capacity()) {
        cudaError_t err = cudaMemsetAsync(fused_bar, 0, sizeof(unsigned), stream);
        if (err != cudaSuccess) return err;
        ProfileScope ps("permute_fused", stream);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(n_chunks), 1, 1);
        cfg.blockDim = dim3(kFusedWarps * 32, 1, 1);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, perm_fused_kernel, ids, R, E, n_chunks, scratch, counts, offsets, tile_off,
                                 perm, inv, fused_bar, 4ll << 30, st);
        note_launch();
        return err;
    }
    const size_t hsm = static_cast<size_t>(E) * sizeof(int32_t);
    if (n_chunks > 0) {
        ProfileScope ps("permute_hist", stream);
        perm_hist_kernel<<<n_chunks, 128, hsm, stream>>>(ids, R, E, n_chunks, scratch, st);
        note_launch();
    }
    {
        ProfileScope ps("permute_scan", stream);
        perm_scan_kernel<<<1, 1024, 0, stream>>>(n_chunks, E, scratch, counts, offsets, tile_off);
        note_launch();
    }
    if (n_chunks > 0) {
        ProfileScope ps("permute_scatter", stream);
        perm_scatter_kernel<<<n_chunks, 32, hsm, stream>>>(ids, R, E, n_chunks, scratch, offsets, perm, inv);
        note_launch();
    }
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(int R, int S, int H, int elem_bytes, const void* x,
                               const float* xscale, const int32_t* perm, void* xp, float* xpscale,
                               const int32_t* skip, cudaStream_t stream) {
    if (R == 0) return cudaSuccess;
    const int row_vecs = H * elem_bytes / 16;
    ProfileScope ps("gather", stream);
    gather_rows_kernel<<<ceil_div(R * 32, 256), 256, 0, stream>>>(
        R, S, row_vecs, static_cast<const uint4*>(x), xscale, perm, static_cast<uint4*>(xp), xpscale, skip);
    note_launch();
    return cudaGetLastError();
}

bool scatter_rows_supported(int H) { return H > 0 && H % 8 == 0 && H <= kScatterMaxH; }

cudaError_t launch_scatter_rows(int T, int S, int R, int H, const void* x, const int32_t* inv,
                                const int32_t* skip, uint8_t* xq, float* xscale, void* xp, float* xpscale,
                                cudaStream_t stream) {
    if (!scatter_rows_supported(H)) return cudaErrorNotSupported;
    if (T == 0) return cudaSuccess;
    ProfileScope ps("gather", stream);
    if (xq != nullptr)
        scatter_rows_kernel<true><<<T, kScatterThreads, 0, stream>>>(
            T, S, R, H, static_cast<const uint4*>(x), inv, skip, xq, xscale, xp, xpscale);
    else
        scatter_rows_kernel<false><<<T, kScatterThreads, 0, stream>>>(
            T, S, R, H, static_cast<const uint4*>(x), inv, skip, nullptr, nullptr, xp, nullptr);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(int rows, int cols, const uint16_t* in, uint8_t* codes,
                              float* scales, cudaStream_t stream, const char* name) {
    if (rows == 0) return cudaSuccess;
    ProfileScope ps(name, stream);
    quant_rows_kernel<<<ceil_div(rows * 32, 256), 256, 0, stream>>>(rows, cols, in, codes, scales);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sre
