// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (tcgen05).
//
// "Optimizing GLM4-MoE for production" (Novita AI), section 1: the shared
// expert has the same tensor shapes and computation flow as the routed ones,
// so it joins them as one more group of the same grouped GEMM (expert index
// n_routed, rows = every token) and one pass computes all S slots.
//
// Two persistent kernels per layer, one CTA per SM:
//   GEMM1: G = Xp[rows of e] . W13[e]^T; the epilogue applies SwiGLU
//          h = silu(G_gate) * G_up and stores bf16 h [R, I]
//   GEMM2: Y = h[rows of e] . W2[e]^T, stored as bf16 rows [R, H] (the
//          moe_grouped_ffn entry point) or, inside moe_forward, as fp16 rows
//          scaled by a power of two per 32 columns (11 significant bits, same
//          bytes as bf16) for the fp32 weighted combine that follows
// E4M3 layers run kind::f8f6f4 with per-row activation scales and
// per-output-channel weight scales applied in the epilogue (they factor out of
// the K-sum).
//
// CTA layout (320 threads; 448 in grouped_gemm_swap_kernel, whose 12 epilogue
// warps are described there): warp 0 = TMA producer, warp 1 = TMEM allocator
// and single-thread MMA issuer, warps 2-9 = epilogue (warp w reads TMEM lanes
// 32*(w%4)..+31; two warps per lane group split the columns or, for 256-row
// units, take one accumulator each). Stages hold 128 bytes of K per row (64
// bf16 or 128 E4M3 values) of the A tile(s) and of an N-row B tile, written by
// TMA with the 128-byte swizzle. For 128-row units two TMEM accumulators
// (columns 0 and 256) let the epilogue of one unit overlap the MMAs of the next.
//
// Tiles are ordered expert-major, then n-tile, then m-tile, so CTAs running at
// the same time share each weight tile through L2. An m-tile never straddles
// two experts: rows past the expert's end are computed on whatever TMA loads
// there (zero past R) and masked at the store.
//
// Every mbarrier wait is bounded; a wait that runs out raises an abort flag
// that makes the other roles leave their loops, records MOE_ERR_TIMEOUT in the
// status word, drains the copies and MMAs in flight and frees TMEM.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace sre {

namespace {

constexpr int TC_BM = 128;
constexpr int TC_RING_BYTES = 192 * 1024;          // shared memory for the stage ring
#ifndef SRE_STAGE_ROW_BYTES
#define SRE_STAGE_ROW_BYTES 128
#endif
constexpr int TC_MAXE = 260;

constexpr uint32_t TC_TMEM_COLS = 512;

struct TcParams {
    // output rows leave by TMA stores through this map (16-bit elements, 32 x 32
    // boxes, 64-byte swizzle: the staging slices' layout) when out_tma is set;
    // the kernels take TcParams as a __grid_constant__ parameter so that the
    // map's address is valid for the TMA unit
    CUtensorMap tm_out;
    int out_tma;
    int E, H, I;
    int n_tiles_n;          // n-tiles per m-tile
    int bn_out;             // output columns per n-tile (GEMM1: I columns; GEMM2: H columns)
    int k_blocks;           // K / (128 bytes per row)
    const int32_t* offsets; // [E+1]
    const int32_t* tile_off;// [E+1]
    uint16_t* out;          // GEMM1: h [R, I]; GEMM2: y [R, H] (bf16)
    int out_ld;
    const float* row_scale; // E4M3: per-row activation scale [R]
    int direct_e;           // GEMM1: expert whose A rows are read from the token matrix (tmA2), or -1
    int first_e;            // tokens-as-N kernel: expert whose units run first (the largest group), or -1
    const float* direct_scale;  // E4M3: per-token scale of that expert's rows
    const float* col_scale; // E4M3: per-output-channel weight scale (s13 [E, 2I] or s2 [E, H])
    // GEMM2 with yexp != null: rows stored as fp16(v * 2^-k), k per 32 columns in yexp
    int8_t* yexp;
    // GEMM2 with the weighted combine folded in (fold_e >= 0): the fold_e group's
    // units (the shared expert's; its rows are the tokens in order, its units the
    // last ones) also write the layer output, summing each token's slots; see
    // fold_combine
    int fold_e;
    int fold_S;                 // slots per token; the fold_e group's slot is the last
    const int32_t* fold_inv;    // [T * S] flat slot -> row
    const float* fold_w;        // [T * S] slot weights
    void* fold_out;             // [T, H] bf16, or fp32 when fold_out_f32
    int fold_out_f32;
    unsigned* ready;            // [n_tiles_n] routed-unit epilogue warps done, per n-tile (zero at launch)
    unsigned fold_extra;        // testing hook: added to the arrivals a fold_e unit waits for (never reached)
    DevStatus* status;
    long long wait_limit;   // SM clock cycles per wait
    int inject_stall;       // testing hook: the producer never issues its loads
};

struct TileInfo {
    int e, row0, row_end, n0;
    bool two;       // pair units: the second 128-row m-tile exists
};

// Work unit `id` -> (expert, m-tile or m-tile pair, n-tile). Units are ordered
// expert-major, then n-tile, then m-unit; s_unit is the prefix of m-units per
// expert (m-tiles, or pairs of m-tiles when kPair).
template <bool kPair>
__device__ __forceinline__ TileInfo decode_unit(int id, const int* s_unit, const int* s_off, int E, int NT,
                                                int bn_out) {
    int lo = 0, hi = E - 1;   // largest e with s_unit[e] * NT <= id
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_unit[mid] * NT <= id) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int mue = s_unit[e + 1] - s_unit[e];
    const int local = id - s_unit[e] * NT;
    const int nt = local / mue;
    const int mu = local - nt * mue;
    TileInfo t;
    t.e = e;
    t.row0 = s_off[e] + mu * (kPair ? 2 * TC_BM : TC_BM);
    t.row_end = s_off[e + 1];
    t.n0 = nt * bn_out;
    t.two = kPair && (t.row0 + TC_BM < t.row_end);
    return t;
}

// A warp's staging slice is free again: the TMA store that last read it (if
// any; issued by lane 0, whose bulk groups these are) has read it.
__device__ __forceinline__ void slice_acquire(const CUtensorMap* tm, int lane) {
    if (tm != nullptr) {
        if (lane == 0) ptx::bulk_wait_read_all();
        __syncwarp();
    }
}

// A whole 32 x 32 block staged in the slice (64-byte rows, 16-byte chunks
// XOR-swizzled by (row >> 1) & 3: the TMA 64-byte swizzle) leaves by one TMA
// store; the warp goes on while the TMA unit reads the slice.
__device__ __forceinline__ void slice_tma_store(const CUtensorMap* tm, const uint8_t* slice, int lane, int row0,
                                                int col0) {
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        ptx::tma_store_2d(tm, slice, col0, row0);
        ptx::bulk_commit();
    }
}

// One warp's 32 rows x 32 columns of 16-bit results (lane = row, packed[] = its
// 64 bytes) go to global memory through a 2 KB shared-memory slice: written
// with the 16-byte chunks of row r XOR-swizzled by (r >> 1) & 3 (conflict-free),
// then either stored by TMA (tm set and all 32 rows below row_end) or read
// back so that 4 lanes cover one row's 64 contiguous bytes (8 rows per
// instruction) and stored without the rows at or past row_end (those belong
// to the next group).
__device__ __forceinline__ void stage_store(uint8_t* slice, const uint32_t (&packed)[16], int lane, uint16_t* out,
                                            int ld, int row0, int row_end, int col0, const CUtensorMap* tm) {
    slice_acquire(tm, lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int pc = q ^ ((lane >> 1) & 3);
        *reinterpret_cast<uint4*>(slice + lane * 64 + pc * 16) =
            make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
    }
    if (tm != nullptr && row0 + 32 <= row_end) {
        slice_tma_store(tm, slice, lane, row0, col0);
        return;
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = j * 8 + (lane >> 2);
        const int c = lane & 3;
        const uint4 v = *reinterpret_cast<const uint4*>(slice + r * 64 + ((c ^ ((r >> 1) & 3)) * 16));
        const int grow = row0 + r;
        if (grow < row_end)
            *reinterpret_cast<uint4*>(out + static_cast<size_t>(grow) * ld + col0 + c * 8) = v;
    }
    __syncwarp();
}

// E4M3 layers: this warp's per-output-channel weight scales of a unit (GEMM2:
// columns n0 + 32 c_begin .. n0 + 32 c_end of expert e; GEMM1: the gate columns
// of those h columns, then the up columns) copied once into its 1 KB shared
// area, coalesced, so that the epilogue reads them as broadcasts instead of one
// global load per value and chunk.
template <bool kGemm1>
__device__ __forceinline__ void stage_scales(const TcParams& p, const TileInfo& t, int c_begin, int c_end,
                                             float* dst, int lane) {
    const int n = (c_end - c_begin) * 32;
    __syncwarp();                                    // the previous unit's reads are done
    if constexpr (kGemm1) {
        const float* g = p.col_scale + static_cast<size_t>(t.e) * 2 * p.I + t.n0 + c_begin * 32;
        for (int i = lane; i < n; i += 32) {
            dst[i] = g[i];
            dst[n + i] = g[p.I + i];
        }
    } else {
        const float* g = p.col_scale + static_cast<size_t>(t.e) * p.H + t.n0 + c_begin * 32;
        for (int i = lane; i < n; i += 32) dst[i] = g[i];
    }
    __syncwarp();
}

// max |a[j]| over 32 registers as four independent chains (max is exact, so
// the order does not change the result; a single chain is 32 dependent steps)
__device__ __forceinline__ float abs_max32(const float (&a)[32]) {
    float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < 32; ++j) m[j & 3] = fmaxf(m[j & 3], fabsf(a[j]));
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Epilogue of one unit for one warp: TMEM columns [c_begin, c_end) x 32 of the
// lane group at `tb` (row = this lane's output row, valid if it is stored)
// become bf16 h (GEMM1, SwiGLU applied) or bf16 / scaled-fp16 y rows (GEMM2),
// leaving through this warp's staging slice (rows wrow0..wrow0+31).
template <bool kFp8, bool kGemm1, int kBN>
__device__ __forceinline__ void epilogue_rows(const TcParams& p, const TileInfo& t, uint32_t tb, int c_begin,
                                              int c_end, uint8_t* stage_w, int lane, int row, bool valid,
                                              float rs, int wrow0, const float* scs) {
    constexpr int HALF = kBN / 2;
    const CUtensorMap* tmo = p.out_tma ? &p.tm_out : nullptr;
    if constexpr (kGemm1) {
#pragma unroll 1
        for (int c = c_begin; c < c_end; ++c) {
            uint32_t g[32], u[32];
            ptx::tmem_ld_32x32b_x32(tb + c * 32, g);
            ptx::tmem_ld_32x32b_x32(tb + HALF + c * 32, u);
            ptx::tmem_ld_wait(g);
            ptx::tmem_ld_wait(u);
            // this warp's staged weight scales: gate columns, then up columns (broadcast reads)
            const float* sg = scs + (c - c_begin) * 32;
            const float* su = scs + (c_end - c_begin) * 32 + (c - c_begin) * 32;
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float g0 = __uint_as_float(g[j]), g1 = __uint_as_float(g[j + 1]);
                float u0 = __uint_as_float(u[j]), u1 = __uint_as_float(u[j + 1]);
                if constexpr (kFp8) {
                    // (v * rs) * scale, two at a time; rows past the group end are
                    // computed too and not stored
                    const float2 rs2 = make_float2(rs, rs);
                    const float2 gg = __fmul2_rn(__fmul2_rn(make_float2(g0, g1), rs2), make_float2(sg[j], sg[j + 1]));
                    const float2 uu = __fmul2_rn(__fmul2_rn(make_float2(u0, u1), rs2), make_float2(su[j], su[j + 1]));
                    g0 = gg.x;
                    g1 = gg.y;
                    u0 = uu.x;
                    u1 = uu.y;
                }
                packed[j >> 1] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
            }
            stage_store(stage_w, packed, lane, p.out, p.out_ld, wrow0, t.row_end, t.n0 + c * 32, tmo);
        }
    } else {
        // chunk c's TMEM load is in flight while chunk c-1 is converted and stored
        uint64_t exps = 0;
        auto process = [&](const uint32_t (&v)[32], int c) {
            const float* sc = scs + (c - c_begin) * 32;      // this warp's staged weight scales
            float a[32];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float2 q = make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                if constexpr (kFp8) {
                    // (a * rs) * sc per element, two at a time; rows past the group end are not stored
                    q = __fmul2_rn(__fmul2_rn(q, make_float2(rs, rs)), make_float2(sc[j], sc[j + 1]));
                }
                a[j] = q.x;
                a[j + 1] = q.y;
            }
            uint32_t packed[16];
            if (p.yexp != nullptr) {
                const float amax = abs_max32(a);
                const int k = f16_chunk_exp(amax);
                const float down = exp2_int(-k);
                const float2 down2 = make_float2(down, down);
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float2 q = __fmul2_rn(make_float2(a[j], a[j + 1]), down2);
                    packed[j >> 1] = pack_f16x2(q.x, q.y);
                }
                exps |= static_cast<uint64_t>(static_cast<uint8_t>(static_cast<int8_t>(k))) << (8 * (c - c_begin));
            } else {
#pragma unroll
                for (int j = 0; j < 32; j += 2) packed[j >> 1] = pack_bf16x2(a[j], a[j + 1]);
            }
            stage_store(stage_w, packed, lane, p.out, p.out_ld, wrow0, t.row_end, t.n0 + c * 32, tmo);
        };
        if constexpr (kFp8) {
            // E4M3: one chunk at a time (the scale products need the registers)
#pragma unroll 1
            for (int c = c_begin; c < c_end; ++c) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tb + c * 32, v);
                ptx::tmem_ld_wait(v);
                process(v, c);
            }
        } else {
            uint32_t va[32], vb[32];
            ptx::tmem_ld_32x32b_x32(tb + c_begin * 32, va);
            ptx::tmem_ld_wait(va);
#pragma unroll 1
            for (int c = c_begin; c < c_end; c += 2) {
                const bool has_b = c + 1 < c_end;
                if (has_b) ptx::tmem_ld_32x32b_x32(tb + (c + 1) * 32, vb);
                process(va, c);
                if (has_b) {
                    ptx::tmem_ld_wait(vb);
                    const bool has_a = c + 2 < c_end;
                    if (has_a) ptx::tmem_ld_32x32b_x32(tb + (c + 2) * 32, va);
                    process(vb, c + 1);
                    if (has_a) ptx::tmem_ld_wait(va);
                }
            }
        }
        if (p.yexp != nullptr && valid) {
            // one store of the run's exponent bytes: a run of n = 8, 4 or 2 chunks
            // starts at a multiple of n (and H / 32, n0 / 32 are multiples of 8)
            int8_t* e = p.yexp + static_cast<size_t>(row) * (p.H / 32) + t.n0 / 32 + c_begin;
            const int n = c_end - c_begin;
            if (n == 8) {
                *reinterpret_cast<uint64_t*>(e) = exps;
            } else if (n == 4) {
                *reinterpret_cast<uint32_t*>(e) = static_cast<uint32_t>(exps);
            } else if (n == 2) {
                *reinterpret_cast<uint16_t*>(e) = static_cast<uint16_t>(exps);
            } else {
                for (int i = 0; i < n; ++i) e[i] = static_cast<int8_t>(exps >> (8 * i));
            }
        }
    }
}

// Weighted combine inside the down-projection ("Optimizing GLM4-MoE for
// production" (Novita AI), section 1: the outputs of a token's experts are
// aggregated with weights), done by the fold_e group's units (the shared
// expert's, whose rows are the tokens in order and whose units come last)
// when moe_forward is asked for it (MOE_FFN_COMBINE_FOLD): one launch less,
// and the reads overlap the MMAs of the units that follow. A warp first stores
// its rows of the unit as every unit does (epilogue_rows), frees the
// accumulator so that the next unit's MMAs start, waits until every routed
// unit of this n-tile has stored its rows (p.ready), and then, for each of its
// 32 tokens and its columns [col0, col0 + ncols),
//     out[tok, cols] = sum_{k < S} w[tok, k] * y[inv[tok * S + k], cols]
// accumulating in fp32 in slot order (one fma per slot with the slot's weight
// times its chunk's power of two; the unit's own row is the last slot) and
// rounding once: the operations of the separate combine kernel in the same
// order, so the output is the same bit for bit. Sixteen lanes cover 128
// contiguous columns (8 each) of one token's rows, so every load reads 256
// contiguous bytes of a row. Measured on B200 this is slower than the separate
// combine pass (prefill_bf16 GEMM2 0.97 ms against 0.61 + 0.08 ms): the eight
// epilogue warps keep ~20 KB of loads in flight per SM where the separate pass
// keeps several times that, so the aggregation is latency-bound here.
constexpr int FOLD_SLOTS = 5;    // slot rows whose loads are issued together

__device__ __forceinline__ void fold_store(const TcParams& p, int tok, int col, const float (&acc)[8]) {
    if (p.fold_out_f32) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.fold_out) + static_cast<size_t>(tok) * p.H + col);
        o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.fold_out) + static_cast<size_t>(tok) * p.H + col) =
            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
    }
}

__device__ __forceinline__ void fold_fma(const uint4& q, float wgt, float (&acc)[8]) {
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const float2 f = unpack_f16x2(u[h]);
        acc[2 * h] = __fmaf_rn(wgt, f.x, acc[2 * h]);
        acc[2 * h + 1] = __fmaf_rn(wgt, f.y, acc[2 * h + 1]);
    }
}

// The combine of one warp's 32 rows (unit rows wrow0 .. +31, tokens wrow0 -
// grp0 ..) over columns [col0, col0 + ncols), ncols a multiple of 128. Work item
// i = (token pair i % 16, 128-column block i / 16); lanes 0-15 take the pair's
// first token, 16-31 its second, 8 columns per lane; the loads of FOLD_SLOTS
// slot rows are in flight together.
__device__ __forceinline__ void fold_combine(const TcParams& p, int row_end, int lane, int wrow0, int grp0,
                                             int col0, int ncols) {
    const int S = p.fold_S;
    const int ne = p.H / 32;
    const int items = 16 * (ncols >> 7);
    const int half = lane >> 4;
    const int cl = (lane & 15) * 8;
#pragma unroll 1
    for (int it = 0; it < items; ++it) {
        const int row = wrow0 + 2 * (it % 16) + half;
        const int col = col0 + (it / 16) * 128 + cl;
        if (row >= row_end) continue;
        const int tok = row - grp0;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll 1
        for (int k0 = 0; k0 < S; k0 += FOLD_SLOTS) {
            uint4 q[FOLD_SLOTS];
            int ex[FOLD_SLOTS];
            float wk[FOLD_SLOTS];
#pragma unroll
            for (int g = 0; g < FOLD_SLOTS; ++g) {
                if (k0 + g < S) {
                    const size_t f = static_cast<size_t>(tok) * S + k0 + g;
                    const size_t r = static_cast<size_t>(p.fold_inv[f]);
                    q[g] = *reinterpret_cast<const uint4*>(p.out + r * p.H + col);
                    ex[g] = p.yexp[r * ne + (col >> 5)];
                    wk[g] = p.fold_w[f];
                }
            }
#pragma unroll
            for (int g = 0; g < FOLD_SLOTS; ++g)
                if (k0 + g < S) fold_fma(q[g], wk[g] * exp2_int(ex[g]), acc);
        }
        fold_store(p, tok, col, acc);
    }
}

// A routed unit's epilogue warp is done storing: its rows become visible at GPU
// scope before the n-tile's counter counts it.
__device__ __forceinline__ void fold_arrive(const TcParams& p, int nt, int lane) {
    __threadfence();
    __syncwarp();
    if (lane == 0) ptx::red_release_gpu_add(p.ready + nt, 1u);
}

// Before a fold_e unit reads routed rows: wait until every routed unit's
// epilogue warps have counted themselves on this n-tile (bounded; false on
// timeout or abort).
__device__ __forceinline__ bool fold_wait(const TcParams& p, int nt, unsigned target, volatile int* abort,
                                          int lane) {
    int ok = 1;
    if (lane == 0) ok = ptx::counter_wait(p.ready + nt, target, abort, p.wait_limit, p.status, 5u);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();          // the warp's own stores of this unit are visible to all its lanes
    __threadfence();
    return ok != 0;
}

// kBN: MMA N (GEMM1: gate half + up half; GEMM2: 256 output columns).
// kPair: a work unit is two consecutive 128-row m-tiles of one expert that share
// each weight (B) stage in shared memory (an M = 256 tile: every weight byte is
// fetched by one CTA and used for 256 rows). Its two fp32 accumulators fill
// TMEM (columns 0 and 256), so there is no second buffer; the 8 epilogue warps
// drain them 4 per accumulator. Otherwise a unit is one m-tile, the two TMEM
// buffers alternate between units, and the 8 epilogue warps split each tile's
// columns in two halves (two warps per TMEM sub-partition).
// kRowB: bytes of K per row per stage (128: 128-byte swizzle; 64: 64-byte swizzle,
// twice as many stages of half the size).
template <int kRowB, int kBN, bool kPair>
struct Ring {
    static constexpr int A_TILE = TC_BM * kRowB;
    static constexpr int STAGE = (kPair ? 2 : 1) * A_TILE + kBN * kRowB;
    static constexpr int N = (TC_RING_BYTES / STAGE) > 8 ? 8 : (TC_RING_BYTES / STAGE);
    // + epilogue staging (2 KB per warp), weight scales (1 KB per warp), alignment
    static constexpr int SMEM = N * STAGE + 8 * 2048 + 8 * 1024 + 1024;
};

template <bool kFp8, bool kGemm1, int kBN, bool kPair, int kRowB>
__global__ void __launch_bounds__(320, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ TcParams p) {
    using RG = Ring<kRowB, kBN, kPair>;
    constexpr int NSTAGE = RG::N;
    constexpr int TC_ABYTES = RG::A_TILE;           // one 128-row A tile per stage
    constexpr int ABYTES = (kPair ? 2 : 1) * TC_ABYTES;
    constexpr int BBYTES = kBN * kRowB;
    constexpr int HALF = kBN / 2;
    constexpr int KEL = kFp8 ? kRowB : kRowB / 2;   // K elements per stage
    constexpr int KSTEPS = kRowB / 32;              // MMAs (32 bytes of K each) per stage
    constexpr int EPI_WARPS = 8;
    constexpr uint32_t IDESC = ptx::instr_desc(TC_BM, kBN, kFp8 ? 0u : 1u);

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[NSTAGE], empty_bar[NSTAGE], tfull_bar[2], tempty_bar[2], drain_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_off[TC_MAXE], s_unit[TC_MAXE];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + NSTAGE * ABYTES;
    uint8_t* sStage = sB + NSTAGE * BBYTES;         // EPI_WARPS x 2 KB
    float* sScale = reinterpret_cast<float*>(sStage + EPI_WARPS * 2048);   // EPI_WARPS x 1 KB (E4M3 weight scales)
    volatile int* abort_flag = &s_abort;

    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_off[i] = p.offsets[i];
    if constexpr (kPair) {
        // prefix of m-tile pairs per expert (warp scan over the m-tile counts)
        if (warp == 0) {
            int carry = 0;
            for (int e0 = 0; e0 <= p.E; e0 += 32) {
                const int e = e0 + lane;
                const int pairs = (e < p.E) ? (p.tile_off[e + 1] - p.tile_off[e] + 1) >> 1 : 0;
                int inc = pairs;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
                    if (lane >= off) inc += o;
                }
                if (e <= p.E) s_unit[e] = carry + inc - pairs;
                carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
            }
        }
    } else {
        for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_unit[i] = p.tile_off[i];
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull_bar[b], 1);
            ptx::mbar_init(&tempty_bar[b], EPI_WARPS * 32);
        }
        ptx::mbar_init(&drain_bar, 1);
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        if (p.direct_e >= 0) ptx::prefetch_tmap(&tmA2);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&s_tmem, TC_TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = s_tmem;
    const int total = s_unit[p.E] * p.n_tiles_n;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // The whole warp walks the tiles; lane 0 waits and issues every load.
        if (!p.inject_stall) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                const TileInfo t = decode_unit<kPair>(tile, s_unit, s_off, p.E, p.n_tiles_n, p.bn_out);
                int ok = 1;
                if (lane == 0) {
                    const uint32_t tx = (t.two ? 2 : 1) * TC_ABYTES + BBYTES;
                    for (int kb = 0; kb < p.k_blocks; ++kb) {
                        if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_limit, p.status, 1u)) {
                            ok = 0;
                            break;
                        }
                        ptx::mbar_arrive_expect_tx(&full_bar[stage], tx);
                        const int kx = kb * KEL;
                        // A rows: gathered copy, or the token matrix itself for the direct group
                        const bool direct = t.e == p.direct_e;
                        const CUtensorMap* am = direct ? &tmA2 : &tmA;
                        const int ar = direct ? t.row0 - s_off[t.e] : t.row0;
                        ptx::tma_load_2d(sA + stage * ABYTES, am, &full_bar[stage], kx, ar);
                        if (t.two)
                            ptx::tma_load_2d(sA + stage * ABYTES + TC_ABYTES, am, &full_bar[stage], kx, ar + TC_BM);
                        if constexpr (kGemm1) {
                            ptx::tma_load_3d(sB + stage * BBYTES, &tmB, &full_bar[stage], kx, t.n0, 2 * t.e);
                            ptx::tma_load_3d(sB + stage * BBYTES + HALF * kRowB, &tmB, &full_bar[stage], kx, t.n0,
                                             2 * t.e + 1);
                        } else {
                            ptx::tma_load_2d(sB + stage * BBYTES, &tmB, &full_bar[stage], kx, t.e * p.H + t.n0);
                        }
                        if (++stage == NSTAGE) { stage = 0; phase ^= 1u; }
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                __syncwarp();
                if (!ok) break;
            }
            if (lane == 0 && *abort_flag) {
                // let every copy in flight land before the CTA can exit: each
                // stage's last armed phase completes when its bytes arrive
                for (int s = 0; s < NSTAGE; ++s) {
                    // stages below `stage` were armed in the current round (phase),
                    // the others in the previous one (phase ^ 1) if ever
                    const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
                    const long long t0 = clock64();
                    while (!ptx::mbar_try_wait(&full_bar[s], par) && clock64() - t0 < p.wait_limit) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                bool two = false;
                if constexpr (kPair) two = decode_unit<kPair>(tile, s_unit, s_off, p.E, p.n_tiles_n, p.bn_out).two;
                if (!ptx::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, p.wait_limit, p.status, 2u)) break;
                ptx::tc_fence_after();
                const uint32_t d0 = tmem_base + static_cast<uint32_t>(kPair ? 0 : acc * 256);
                const uint32_t d1 = tmem_base + 256u;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_limit, p.status, 3u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(sA + stage * ABYTES);
                    const uint32_t b_addr = ptx::smem_u32(sB + stage * BBYTES);
#pragma unroll
                    for (int k = 0; k < KSTEPS; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw<kRowB>(a_addr + k * 32);
                        const uint64_t bd = ptx::smem_desc_sw<kRowB>(b_addr + k * 32);
                        if constexpr (kFp8) ptx::mma_f8(d0, ad, bd, IDESC, (kb | k) != 0);
                        else ptx::mma_f16(d0, ad, bd, IDESC, (kb | k) != 0);
                        if (kPair && two) {
                            const uint64_t ad1 = ptx::smem_desc_sw<kRowB>(a_addr + TC_ABYTES + k * 32);
                            if constexpr (kFp8) ptx::mma_f8(d1, ad1, bd, IDESC, (kb | k) != 0);
                            else ptx::mma_f16(d1, ad1, bd, IDESC, (kb | k) != 0);
                        }
                    }
                    ptx::mma_commit(&empty_bar[stage]);
                    if (++stage == NSTAGE) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit(&tfull_bar[acc]);
                if constexpr (kPair) {
                    acc_phase ^= 1u;      // one buffer: every unit flips its phase
                } else {
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1u;
                }
            }
            // every MMA this thread issued has finished before TMEM is freed
            ptx::mma_commit(&drain_bar);
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&drain_bar, 0) && clock64() - t0 < p.wait_limit) {
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int sub = warp & 3;                  // TMEM lanes 32*sub .. +31
        const int eg = (warp - 2) >> 2;            // pair: accumulator; single: column half
        const int r_local = (kPair ? eg * TC_BM : 0) + sub * 32 + lane;
        constexpr int NCH = kGemm1 ? HALF / 32 : kBN / 32;   // 32-column chunks per unit
        constexpr int PER = kPair ? NCH : (NCH + 1) / 2;
        const int c_begin = kPair ? 0 : eg * PER;
        const int c_end = kPair ? NCH : min(NCH, c_begin + PER);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileInfo t = decode_unit<kPair>(tile, s_unit, s_off, p.E, p.n_tiles_n, p.bn_out);
            // one lane waits and the warp takes its result: tcgen05.ld below needs the whole warp
            int ok = 0;
            if (lane == 0) ok = ptx::mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, p.wait_limit, p.status, 4u);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            ptx::tc_fence_after();
            const bool active = (!kPair || eg == 0 || t.two) && c_begin < c_end;    // warp-uniform
            const int row = t.row0 + r_local;
            const bool valid = active && row < t.row_end;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) +
                                static_cast<uint32_t>(kPair ? eg * 256 : acc * 256);
            float rs = 1.0f;
            if (kFp8 && valid)
                rs = (t.e == p.direct_e) ? p.direct_scale[row - s_off[t.e]] : p.row_scale[row];
            const bool fold = !kGemm1 && t.e == p.fold_e;
            const int wrow0 = t.row0 + (kPair ? eg * TC_BM : 0) + sub * 32;   // first unit row of this warp
            if (active) {
                // 16-bit outputs leave through this warp's 2 KB staging slice so that
                // global stores cover whole 64-byte row segments (see stage_store)
                uint8_t* stage_w = sStage + (warp - 2) * 2048;
                float* scs = sScale + (warp - 2) * 256;
                if constexpr (kFp8) stage_scales<kGemm1>(p, t, c_begin, c_end, scs, lane);
                epilogue_rows<kFp8, kGemm1, kBN>(p, t, tb, c_begin, c_end, stage_w, lane, row, valid, rs, wrow0, scs);
            }
            if (!kGemm1 && p.fold_e >= 0 && !fold) fold_arrive(p, t.n0 / p.bn_out, lane);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&tempty_bar[acc]);
            if (fold && active) {
                // the accumulator is free for the next unit; the combine reads global memory only
                // arrivals on the n-tile's counter once every routed unit is stored
                const unsigned target =
                    static_cast<unsigned>(s_unit[p.E] - (s_unit[p.fold_e + 1] - s_unit[p.fold_e])) * EPI_WARPS +
                    p.fold_extra;
                if (!fold_wait(p, t.n0 / p.bn_out, target, abort_flag, lane)) break;
                fold_combine(p, t.row_end, lane, wrow0, s_off[t.e], t.n0 + c_begin * 32, (c_end - c_begin) * 32);
            }
            if constexpr (kPair) {
                acc_phase ^= 1u;
            } else {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
        }
        // this warp's TMA stores have left shared memory and reached global memory
        if (lane == 0) ptx::bulk_wait_all();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TC_TMEM_COLS);
    }
}

// ------------------------------------------------------------------ CTA-pair kernel
// 256-row units on a cluster of two CTAs (the two SMs of a TPC) with
// tcgen05.mma.cta_group::2: CTA r holds A rows row0 + 128 r .. +127 and half
// of the unit's B rows, and receives D rows 128 r .. +127 for all columns in
// its own TMEM. Each weight byte is fetched once per 256 rows, as with
// single-CTA 256-row units, but each SM stages only half of it.
//
// kNSUB = 1: one N = kBN MMA per K step; the two TMEM buffers (columns 0 and
//   256) alternate between units, so the epilogue of one unit overlaps the
//   MMAs of the next. B halves: GEMM1 the gate rows in rank 0 and the up rows
//   in rank 1; GEMM2 output columns n0 + 128 r .. +127.
// kNSUB = 2: two N = 256 MMAs per K step share the A stage (a 256 x 512 tile
//   per pair: half the A traffic per FLOP, a quarter less staged per FLOP),
//   filling all 512 TMEM columns; sub-tile j accumulates in columns 256 j.
//   GEMM1: rank 0 stages gate rows n0 .. n0+255 and rank 1 the up rows, so
//   sub-tile j holds gate and up of h columns n0 + 128 j .. +127; GEMM2: rank r
//   stages output rows n0 + 256 j + 128 r .. +127 for sub-tile j, so sub-tile j
//   holds output columns n0 + 256 j .. +255. Warps 2-5 drain sub-tile 0 and
//   warps 6-9 sub-tile 1; the next unit's MMAs wait for both.
//
// Rank 0 arms its full barriers for the bytes of both CTAs and issues every
// MMA; the commit that frees a stage or fills an accumulator arrives on the
// barrier of that index in both CTAs. The epilogue threads of both CTAs arrive
// on rank 0's TMEM-empty barriers. A wait that runs out raises the abort flag
// of both CTAs.
template <int kRowB, int kBN, int kNSUB>
struct Ring2 {
    static constexpr int A_TILE = TC_BM * kRowB;
    static constexpr int B_SUB = (kBN / 2) * kRowB;           // one CTA's rows of one sub-tile
    static constexpr int B_HALF = kNSUB * B_SUB;
    static constexpr int STAGE = A_TILE + B_HALF;
    static constexpr int N = (TC_RING_BYTES / STAGE) > 8 ? 8 : (TC_RING_BYTES / STAGE);
    static constexpr int SMEM = N * STAGE + 8 * 2048 + 8 * 1024 + 1024;
};

template <bool kFp8, bool kGemm1, int kBN, int kNSUB, int kRowB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ TcParams p) {
    static_assert(kNSUB == 1 || kBN == 256, "two sub-tiles of N = 256");
    using RG = Ring2<kRowB, kBN, kNSUB>;
    constexpr int NSTAGE = RG::N;
    constexpr int ABYTES = RG::A_TILE;
    constexpr int BBYTES = RG::B_HALF;
    constexpr int HALF = kBN / 2;
    constexpr int KEL = kFp8 ? kRowB : kRowB / 2;
    constexpr int KSTEPS = kRowB / 32;
    constexpr int EPI_WARPS = 8;
    constexpr uint32_t IDESC = ptx::instr_desc(2 * TC_BM, kBN, kFp8 ? 0u : 1u);

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[NSTAGE], empty_bar[NSTAGE], tfull_bar[2], tempty_bar[2], drain_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_off[TC_MAXE], s_unit[TC_MAXE];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + NSTAGE * ABYTES;
    uint8_t* sStage = sB + NSTAGE * BBYTES;
    float* sScale = reinterpret_cast<float*>(sStage + EPI_WARPS * 2048);   // EPI_WARPS x 1 KB (E4M3 weight scales)
    volatile int* abort_flag = &s_abort;
    const uint32_t peer_abort = ptx::mapa(&s_abort, rank ^ 1u);

    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_off[i] = p.offsets[i];
    if (warp == 0) {
        // prefix of 256-row units per expert
        int carry = 0;
        for (int e0 = 0; e0 <= p.E; e0 += 32) {
            const int e = e0 + lane;
            const int pairs = (e < p.E) ? (p.tile_off[e + 1] - p.tile_off[e] + 1) >> 1 : 0;
            int inc = pairs;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
                if (lane >= off) inc += o;
            }
            if (e <= p.E) s_unit[e] = carry + inc - pairs;
            carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull_bar[b], 1);
            // epilogue threads of both CTAs that drain this buffer
            ptx::mbar_init(&tempty_bar[b], 2 * (EPI_WARPS / kNSUB) * 32);
        }
        ptx::mbar_init(&drain_bar, 1);
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        if (p.direct_e >= 0) ptx::prefetch_tmap(&tmA2);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(&s_tmem, TC_TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();        // rank 0's barriers exist before the peer's copies name them
    ptx::tc_fence_after();
    const uint32_t tmem_base = s_tmem;
    const int total = s_unit[p.E] * p.n_tiles_n;

    if (warp == 0) {
        // ---------------------------------------------------------------- producers (both CTAs)
        if (!p.inject_stall) {
            int stage = 0;
            uint32_t phase = 0;
            for (int u = cluster; u < total; u += nclusters) {
                const TileInfo t = decode_unit<true>(u, s_unit, s_off, p.E, p.n_tiles_n, p.bn_out);
                int ok = 1;
                if (lane == 0) {
                    // rank 1's A tile exists only when the unit has a second m-tile;
                    // otherwise its rows of D are never stored and its MMA rows read
                    // whatever the stage last held
                    const bool load_a = rank == 0 || t.two;
                    const uint32_t tx = (t.two ? 2 : 1) * ABYTES + 2 * BBYTES;
                    const bool direct = t.e == p.direct_e;
                    const CUtensorMap* am = direct ? &tmA2 : &tmA;
                    const int ar = (direct ? t.row0 - s_off[t.e] : t.row0) + static_cast<int>(rank) * TC_BM;
                    for (int kb = 0; kb < p.k_blocks; ++kb) {
                        if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_limit, p.status, 1u)) {
                            ok = 0;
                            break;
                        }
                        const uint32_t fb = ptx::mapa(&full_bar[stage], 0);
                        if (rank == 0) ptx::mbar_arrive_expect_tx(&full_bar[stage], tx);
                        const int kx = kb * KEL;
                        uint8_t* b_dst = sB + stage * BBYTES;
                        if (load_a) ptx::tma_load_2d_pair(sA + stage * ABYTES, am, fb, kx, ar);
                        if constexpr (kGemm1) {
                            // one box of kNSUB * HALF gate (rank 0) or up (rank 1) rows
                            ptx::tma_load_3d_pair(b_dst, &tmB, fb, kx, t.n0, 2 * t.e + static_cast<int>(rank));
                        } else {
#pragma unroll
                            for (int j = 0; j < kNSUB; ++j)
                                ptx::tma_load_2d_pair(b_dst + j * RG::B_SUB, &tmB, fb, kx,
                                                      t.e * p.H + t.n0 + j * kBN + static_cast<int>(rank) * HALF);
                        }
                        if (++stage == NSTAGE) { stage = 0; phase ^= 1u; }
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                __syncwarp();
                if (!ok) break;
            }
            if (lane == 0 && *abort_flag) {
                ptx::st_remote_u32(peer_abort, 1u);
                if (rank == 0) {
                    // every stage's last armed phase completes when both CTAs' bytes land
                    for (int s = 0; s < NSTAGE; ++s) {
                        const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
                        const long long t0 = clock64();
                        while (!ptx::mbar_try_wait(&full_bar[s], par) && clock64() - t0 < p.wait_limit) {
                        }
                    }
                } else {
                    // rank 1 cannot see its copies land (they count on rank 0's
                    // barriers): give any in flight ample time
                    const long long t0 = clock64();
                    while (clock64() - t0 < (1ll << 21)) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (rank 0)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;                // kNSUB = 1: buffer of this unit
            uint32_t acc_phase = 0;     // parity of the buffer's current use
            for (int u = cluster; u < total; u += nclusters) {
                bool ok = true;
#pragma unroll
                for (int j = 0; j < kNSUB; ++j) {
                    const int b = kNSUB == 1 ? acc : j;
                    ok = ok && ptx::mbar_wait_cluster(&tempty_bar[b], acc_phase ^ 1u, abort_flag, p.wait_limit,
                                                      p.status, 2u);
                }
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(acc * 256);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_limit, p.status, 3u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(sA + stage * ABYTES);
                    const uint32_t b_addr = ptx::smem_u32(sB + stage * BBYTES);
#pragma unroll
                    for (int k = 0; k < KSTEPS; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw<kRowB>(a_addr + k * 32);
#pragma unroll
                        for (int j = 0; j < kNSUB; ++j) {
                            const uint64_t bd = ptx::smem_desc_sw<kRowB>(b_addr + j * RG::B_SUB + k * 32);
                            const uint32_t dj = d + static_cast<uint32_t>(j * 256);
                            if constexpr (kFp8) ptx::mma_f8_pair(dj, ad, bd, IDESC, (kb | k) != 0);
                            else ptx::mma_f16_pair(dj, ad, bd, IDESC, (kb | k) != 0);
                        }
                    }
                    ptx::mma_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == NSTAGE) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
#pragma unroll
                for (int j = 0; j < kNSUB; ++j) ptx::mma_commit_pair(&tfull_bar[kNSUB == 1 ? acc : j], 0x3);
                if constexpr (kNSUB == 1) {
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1u;
                } else {
                    acc_phase ^= 1u;
                }
            }
            if (*abort_flag) ptx::st_remote_u32(peer_abort, 1u);
            // every MMA has finished (in both CTAs' TMEM and shared memory) before teardown
            ptx::mma_commit_pair(&drain_bar, 0x3);
        }
        if (lane == 0) {
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&drain_bar, 0) && clock64() - t0 < p.wait_limit) {
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int sub = warp & 3;
        const int eg = (warp - 2) >> 2;            // kNSUB = 1: column half; 2: sub-tile
        constexpr int NCH = kGemm1 ? HALF / 32 : kBN / 32;
        constexpr int PER = kNSUB == 1 ? (NCH + 1) / 2 : NCH;
        const int c_begin = kNSUB == 1 ? eg * PER : 0;
        const int c_end = min(NCH, c_begin + PER);
        const int r_local = static_cast<int>(rank) * TC_BM + sub * 32 + lane;
        const uint32_t tempty0 = ptx::mapa(&tempty_bar[0], 0);
        const uint32_t tempty1 = ptx::mapa(&tempty_bar[1], 0);
        uint8_t* stage_w = sStage + (warp - 2) * 2048;
        int acc = kNSUB == 1 ? 0 : eg;
        uint32_t acc_phase = 0;
        for (int u = cluster; u < total; u += nclusters) {
            TileInfo t = decode_unit<true>(u, s_unit, s_off, p.E, p.n_tiles_n, p.bn_out);
            int ok = 0;
            if (lane == 0) ok = ptx::mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, p.wait_limit, p.status, 4u);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) {
                if (lane == 0) ptx::st_remote_u32(peer_abort, 1u);
                break;
            }
            ptx::tc_fence_after();
            const int nt = t.n0 / p.bn_out;
            if constexpr (kNSUB == 2) t.n0 += eg * (kGemm1 ? HALF : kBN);   // this sub-tile's output columns
            const bool active = (rank == 0 || t.two) && c_begin < c_end;    // warp-uniform
            const int row = t.row0 + r_local;
            const bool valid = active && row < t.row_end;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(acc * 256);
            float rs = 1.0f;
            if (kFp8 && valid)
                rs = (t.e == p.direct_e) ? p.direct_scale[row - s_off[t.e]] : p.row_scale[row];
            const bool fold = !kGemm1 && t.e == p.fold_e;
            const int wrow0 = t.row0 + static_cast<int>(rank) * TC_BM + sub * 32;
            if (active) {
                float* scs = sScale + (warp - 2) * 256;
                if constexpr (kFp8) stage_scales<kGemm1>(p, t, c_begin, c_end, scs, lane);
                epilogue_rows<kFp8, kGemm1, kBN>(p, t, tb, c_begin, c_end, stage_w, lane, row, valid, rs, wrow0, scs);
            }
            if (!kGemm1 && p.fold_e >= 0 && !fold) fold_arrive(p, nt, lane);
            ptx::tc_fence_before();
            ptx::mbar_arrive_remote(acc == 0 ? tempty0 : tempty1);
            if (fold && active) {
                // the accumulator is free for the next unit; the combine reads global memory only
                // arrivals (both CTAs' epilogue warps) on the n-tile's counter once
                // every routed unit is stored
                const unsigned target =
                    static_cast<unsigned>(s_unit[p.E] - (s_unit[p.fold_e + 1] - s_unit[p.fold_e])) * 2u * EPI_WARPS +
                    p.fold_extra;
                if (!fold_wait(p, nt, target, abort_flag, lane)) {
                    if (lane == 0) ptx::st_remote_u32(peer_abort, 1u);
                    break;
                }
                fold_combine(p, t.row_end, lane, wrow0, s_off[t.e], t.n0 + c_begin * 32, (c_end - c_begin) * 32);
            }
            if constexpr (kNSUB == 1) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
        // this warp's TMA stores have left shared memory and reached global memory
        if (lane == 0) ptx::bulk_wait_all();
    }

    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();        // no CTA leaves while its peer may still name its memory
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
    }
}

// ------------------------------------------------------------------ tokens as the N dimension
// grouped_gemm_swap_kernel computes the transposed products, D^T = W . X^T: a
// unit is 256 weight rows (M, 128 per CTA of the pair) times up to 256 token
// rows of one expert (N, a multiple of 16, half staged by each CTA). A group
// of c rows is cut into ceil(c / 256) units of equal size rounded up to 16
// rows, so a routed group of ~205 rows costs 208 rows of MMA work instead of a
// 256-row M tile. The group scheduled first (the shared expert's, every token)
// is cut into units of the routed groups' mean size (16-row multiple in
// [192, 256]) so that all units cost about the same. TMEM lane = output
// feature, column = token.
//   GEMM1: sub-tile 0 = gate rows n0 + 128 r .. +127 of W13[e] (CTA rank r),
//          sub-tile 1 = the up rows of the same h columns; accumulators in
//          TMEM columns 0 and 256; every epilogue warp reads both and applies
//          SwiGLU, the three warps of a lane group taking every third
//          32-token chunk, written out transposed through the warp's slice.
//   GEMM2: sub-tile j = output columns n0 + 256 j + 128 r .. +127; the three
//          warps of a lane group share the chunks of both sub-tiles. A
//          scaled-fp16 chunk (32 output columns of one row) lies across one
//          warp's 32 lanes, so each block goes through the slice as fp32 and is
//          read back two lanes per row before its exponent is taken.
// Both sub-tiles of a stage share the token tile. TMEM is full, so the next
// unit's MMAs wait for the epilogue of this one (12 epilogue warps keep it
// short). The pair protocol (rank 0
// arms and issues, commits multicast to both CTAs, epilogues arrive on rank
// 0's barrier, bounded waits and abort) is that of grouped_gemm_pair_kernel.

struct SwapUnit {
    int e, row0, rows, n0;
};

__device__ __forceinline__ SwapUnit decode_swap(int id, const int* s_unit, const int* s_off, const int* s_rpu,
                                                int E, int NT, int bn_out) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_unit[mid] * NT <= id) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int nu = s_unit[e + 1] - s_unit[e];
    const int local = id - s_unit[e] * NT;
    const int nt = local / nu;
    const int mu = local - nt * nu;
    const int count = s_off[e + 1] - s_off[e];
    const int rpu = s_rpu[e];                                 // rows per unit, <= 256
    SwapUnit t;
    t.e = e;
    t.row0 = s_off[e] + mu * rpu;
    t.rows = min(rpu, count - mu * rpu);                      // >= 1
    t.n0 = nt * bn_out;
    return t;
}

// One warp's 32 x 32 block of 16-bit results with lane = output column col0 +
// lane and v[i] = output row row0 + i: written column-wise into the warp's 2 KB
// slice (rows of 64 bytes, 16-byte chunks XOR-swizzled by (row >> 1) & 3: each
// instruction writes one row, conflict-free), then stored as stage_store does
// (one TMA store for a whole block; rows at or past row_end are not stored).
__device__ __forceinline__ void stage_store_t(uint8_t* slice, const uint16_t (&v)[32], int lane, uint16_t* out,
                                              int ld, int row0, int row_end, int col0, const CUtensorMap* tm) {
    const int chunk = lane >> 3, within = (lane & 7) * 2;
    slice_acquire(tm, lane);
#pragma unroll
    for (int i = 0; i < 32; ++i)
        *reinterpret_cast<uint16_t*>(slice + i * 64 + ((chunk ^ ((i >> 1) & 3)) * 16) + within) = v[i];
    if (tm != nullptr && row0 + 32 <= row_end) {
        slice_tma_store(tm, slice, lane, row0, col0);
        return;
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = j * 8 + (lane >> 2);
        const int c = lane & 3;
        const uint4 w = *reinterpret_cast<const uint4*>(slice + r * 64 + ((c ^ ((r >> 1) & 3)) * 16));
        const int grow = row0 + r;
        if (grow < row_end)
            *reinterpret_cast<uint4*>(out + static_cast<size_t>(grow) * ld + col0 + c * 8) = w;
    }
    __syncwarp();
}

__device__ __forceinline__ uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// 12 epilogue warps (three per TMEM lane group): TMEM holds one unit, so the
// epilogue is not overlapped with MMAs and its length is paid in full
constexpr int SW_EPI_WARPS = 12;
constexpr int SW_THREADS = (2 + SW_EPI_WARPS) * 32;

template <int kRowB>
struct RingS {
    static constexpr int A_SUB = TC_BM * kRowB;         // 128 weight rows of one sub-tile
    static constexpr int A_TILE = 2 * A_SUB;
    static constexpr int B_TILE = 128 * kRowB;          // this CTA's token rows (N / 2 <= 128)
    static constexpr int STAGE = A_TILE + B_TILE;
    static constexpr int N = (TC_RING_BYTES / STAGE) > 8 ? 8 : (TC_RING_BYTES / STAGE);
    static constexpr int SMEM = N * STAGE + SW_EPI_WARPS * 2048 + 1024;
};

// silu(g) = g / (1 + e^-g) with the hardware's approximate reciprocal (a few
// ulp; e^-g = inf gives 0) instead of an IEEE division
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <bool kFp8, bool kGemm1, int kRowB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SW_THREADS, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                             const __grid_constant__ CUtensorMap tmX2, const __grid_constant__ TcParams p) {
    using RG = RingS<kRowB>;
    constexpr int NSTAGE = RG::N;
    constexpr int KEL = kFp8 ? kRowB : kRowB / 2;
    constexpr int KSTEPS = kRowB / 32;
    constexpr int EPI_WARPS = SW_EPI_WARPS;
    constexpr int EG = EPI_WARPS / 4;           // epilogue warps per TMEM lane group

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[NSTAGE], empty_bar[NSTAGE], tfull_bar, tempty_bar, drain_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_off[TC_MAXE], s_unit[TC_MAXE], s_rpu[TC_MAXE];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + NSTAGE * RG::A_TILE;
    uint8_t* sStage = sB + NSTAGE * RG::B_TILE;
    volatile int* abort_flag = &s_abort;
    const uint32_t peer_abort = ptx::mapa(&s_abort, rank ^ 1u);

    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_off[i] = p.offsets[i];
    if (warp == 0) {
        // units per expert and their rows: ceil(count / 256) units of equal size
        // rounded up to 16 rows; the first-scheduled group in units of the other
        // groups' mean size
        int target = 256;
        if (p.first_e >= 0 && p.E > 1) {
            const int cf = p.offsets[p.first_e + 1] - p.offsets[p.first_e];
            const int mean = (p.offsets[p.E] - cf) / (p.E - 1);
            target = min(256, max(192, (mean + 15) & ~15));
        }
        int carry = 0;
        for (int e0 = 0; e0 <= p.E; e0 += 32) {
            const int e = e0 + lane;
            int units = 0;
            if (e < p.E) {
                const int c = p.offsets[e + 1] - p.offsets[e];
                int rpu;
                if (e == p.first_e) {
                    units = (c + target - 1) / target;
                    rpu = target;
                } else {
                    units = (c + 255) >> 8;
                    rpu = units ? (((c + units - 1) / units + 15) & ~15) : 0;
                }
                s_rpu[e] = rpu;
            }
            int inc = units;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
                if (lane >= off) inc += o;
            }
            if (e <= p.E) s_unit[e] = carry + inc - units;
            carry += __shfl_sync(0xFFFFFFFFu, inc, 31);
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        ptx::mbar_init(&tfull_bar, 1);
        ptx::mbar_init(&tempty_bar, 2 * EPI_WARPS * 32);     // every epilogue thread of both CTAs
        ptx::mbar_init(&drain_bar, 1);
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmW);
        ptx::prefetch_tmap(&tmX);
        if (p.direct_e >= 0) ptx::prefetch_tmap(&tmX2);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(&s_tmem, TC_TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem_base = s_tmem;
    const int total = s_unit[p.E] * p.n_tiles_n;
    // the largest group's units (all 256 rows) go first, so that the last wave
    // holds the smaller routed units; every role walks the same rotated order.
    // (Spreading them evenly through the schedule instead, so that tensor-bound
    // shared units run beside HBM-bound routed ones, measured 1-1.5% slower.)
    const int rot = p.first_e >= 0 ? s_unit[p.first_e] * p.n_tiles_n : 0;
    auto unit = [&](int u) {
        const int v = u + rot;
        return decode_swap(v < total ? v : v - total, s_unit, s_off, s_rpu, p.E, p.n_tiles_n, p.bn_out);
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- producers (both CTAs)
        if (!p.inject_stall) {
            int stage = 0;
            uint32_t phase = 0;
            for (int u = cluster; u < total; u += nclusters) {
                const SwapUnit t = unit(u);
                int ok = 1;
                if (lane == 0) {
                    const bool direct = t.e == p.direct_e;
                    const CUtensorMap* xm = direct ? &tmX2 : &tmX;
                    const int n_half = ((t.rows + 15) & ~15) >> 1;
                    const int xr = (direct ? t.row0 - s_off[t.e] : t.row0) + static_cast<int>(rank) * n_half;
                    constexpr uint32_t tx = 2u * (RG::A_TILE + RG::B_TILE);
                    for (int kb = 0; kb < p.k_blocks; ++kb) {
                        if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.wait_limit, p.status, 1u)) {
                            ok = 0;
                            break;
                        }
                        const uint32_t fb = ptx::mapa(&full_bar[stage], 0);
                        if (rank == 0) ptx::mbar_arrive_expect_tx(&full_bar[stage], tx);
                        const int kx = kb * KEL;
                        uint8_t* a_dst = sA + stage * RG::A_TILE;
                        if constexpr (kGemm1) {
                            const int wr = t.n0 + static_cast<int>(rank) * TC_BM;
                            ptx::tma_load_3d_pair(a_dst, &tmW, fb, kx, wr, 2 * t.e);
                            ptx::tma_load_3d_pair(a_dst + RG::A_SUB, &tmW, fb, kx, wr, 2 * t.e + 1);
                        } else {
#pragma unroll
                            for (int j = 0; j < 2; ++j)
                                ptx::tma_load_2d_pair(a_dst + j * RG::A_SUB, &tmW, fb, kx,
                                                      t.e * p.H + t.n0 + j * 256 + static_cast<int>(rank) * TC_BM);
                        }
                        ptx::tma_load_2d_pair(sB + stage * RG::B_TILE, xm, fb, kx, xr);
                        if (++stage == NSTAGE) { stage = 0; phase ^= 1u; }
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                __syncwarp();
                if (!ok) break;
            }
            if (lane == 0 && *abort_flag) {
                ptx::st_remote_u32(peer_abort, 1u);
                if (rank == 0) {
                    for (int s = 0; s < NSTAGE; ++s) {
                        const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
                        const long long t0 = clock64();
                        while (!ptx::mbar_try_wait(&full_bar[s], par) && clock64() - t0 < p.wait_limit) {
                        }
                    }
                } else {
                    const long long t0 = clock64();
                    while (clock64() - t0 < (1ll << 21)) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (rank 0)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phase = 0;
            for (int u = cluster; u < total; u += nclusters) {
                const SwapUnit t = unit(u);
                const uint32_t idesc = ptx::instr_desc(2 * TC_BM, (t.rows + 15) & ~15, kFp8 ? 0u : 1u);
                bool ok = ptx::mbar_wait_cluster(&tempty_bar, acc_phase ^ 1u, abort_flag, p.wait_limit, p.status, 2u);
                if (!ok) break;
                ptx::tc_fence_after();
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag, p.wait_limit, p.status, 3u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(sA + stage * RG::A_TILE);
                    const uint32_t b_addr = ptx::smem_u32(sB + stage * RG::B_TILE);
#pragma unroll
                    for (int k = 0; k < KSTEPS; ++k) {
                        const uint64_t bd = ptx::smem_desc_sw<kRowB>(b_addr + k * 32);
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const uint64_t ad = ptx::smem_desc_sw<kRowB>(a_addr + j * RG::A_SUB + k * 32);
                            const uint32_t dj = tmem_base + static_cast<uint32_t>(j * 256);
                            if constexpr (kFp8) ptx::mma_f8_pair(dj, ad, bd, idesc, (kb | k) != 0);
                            else ptx::mma_f16_pair(dj, ad, bd, idesc, (kb | k) != 0);
                        }
                    }
                    ptx::mma_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == NSTAGE) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit_pair(&tfull_bar, 0x3);
                acc_phase ^= 1u;
            }
            if (*abort_flag) ptx::st_remote_u32(peer_abort, 1u);
            ptx::mma_commit_pair(&drain_bar, 0x3);
        }
        if (lane == 0) {
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&drain_bar, 0) && clock64() - t0 < p.wait_limit) {
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int sub = warp & 3;
        const int eg = (warp - 2) >> 2;          // 0 .. EG-1
        const uint32_t tempty0 = ptx::mapa(&tempty_bar, 0);
        uint8_t* stage_w = sStage + (warp - 2) * 2048;
        const CUtensorMap* tmo = (kGemm1 && p.out_tma) ? &p.tm_out : nullptr;
        uint32_t acc_phase = 0;
        for (int u = cluster; u < total; u += nclusters) {
            const SwapUnit t = unit(u);
            int ok = 0;
            if (lane == 0) ok = ptx::mbar_wait(&tfull_bar, acc_phase, abort_flag, p.wait_limit, p.status, 4u);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) {
                if (lane == 0) ptx::st_remote_u32(peer_abort, 1u);
                break;
            }
            ptx::tc_fence_after();
            const int nch = (t.rows + 31) >> 5;
            const int row_end = t.row0 + t.rows;
            const uint32_t lanes = static_cast<uint32_t>(sub * 32) << 16;
            const bool direct = t.e == p.direct_e;
            if constexpr (kGemm1) {
                const int col0 = t.n0 + static_cast<int>(rank) * TC_BM + sub * 32;   // h columns of this warp
                float sg = 1.0f, su = 1.0f;
                if constexpr (kFp8) {
                    const float* s = p.col_scale + static_cast<size_t>(t.e) * 2 * p.I + col0 + lane;
                    sg = s[0];
                    su = s[p.I];
                }
#pragma unroll 1
                for (int c = eg; c < nch; c += EG) {
                    uint32_t g[32], v[32];
                    ptx::tmem_ld_32x32b_x32(tmem_base + lanes + c * 32, g);
                    ptx::tmem_ld_32x32b_x32(tmem_base + lanes + 256 + c * 32, v);
                    float my_rs = 1.0f;
                    if constexpr (kFp8) {
                        const int r = c * 32 + lane;
                        if (r < t.rows) my_rs = direct ? p.direct_scale[t.row0 - s_off[t.e] + r] : p.row_scale[t.row0 + r];
                    }
                    ptx::tmem_ld_wait(g);
                    ptx::tmem_ld_wait(v);
                    uint16_t o[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float gi = __uint_as_float(g[i]), ui = __uint_as_float(v[i]);
                        if constexpr (kFp8) {
                            const float rs = __shfl_sync(0xFFFFFFFFu, my_rs, i);
                            gi = gi * rs * sg;
                            ui = ui * rs * su;
                        }
                        o[i] = bf16_bits(silu_fast(gi) * ui);
                    }
                    stage_store_t(stage_w, o, lane, p.out, p.out_ld, t.row0 + c * 32, row_end, col0, tmo);
                }
            } else {
                // Each 32-token chunk goes through the warp's slice as fp32 in two
                // halves of 16 tokens: written one token row (128 bytes) per
                // instruction, 16-byte chunks XOR-swizzled by row & 7; read back with
                // two lanes per row, 16 columns each, so that the chunk exponent is a
                // max over 16 registers and one shuffle.
#pragma unroll 1
                for (int q = eg; q < 2 * nch; q += EG) {
                    const int j = q & 1, c = q >> 1;     // sub-tile, 32-token chunk
                    const int col0 = t.n0 + j * 256 + static_cast<int>(rank) * TC_BM + sub * 32;   // y columns
                    float sc = 1.0f;
                    if constexpr (kFp8) sc = p.col_scale[static_cast<size_t>(t.e) * p.H + col0 + lane];
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(tmem_base + lanes + static_cast<uint32_t>(j * 256) + c * 32, v);
                    ptx::tmem_ld_wait(v);
                    const int r = lane >> 1, hh = lane & 1;      // read side: row, column half
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float a = __uint_as_float(v[h2 * 16 + i]);
                            if constexpr (kFp8) a *= sc;
                            *reinterpret_cast<float*>(stage_w + i * 128 + (((lane >> 2) ^ (i & 7)) << 4) +
                                                      (lane & 3) * 4) = a;
                        }
                        __syncwarp();
                        float a[16];
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const float4 w4 = *reinterpret_cast<const float4*>(
                                stage_w + r * 128 + (((hh * 4 + k4) ^ (r & 7)) << 4));
                            a[4 * k4] = w4.x;
                            a[4 * k4 + 1] = w4.y;
                            a[4 * k4 + 2] = w4.z;
                            a[4 * k4 + 3] = w4.w;
                        }
                        __syncwarp();
                        const int rr = c * 32 + h2 * 16 + r;     // row within the unit
                        const bool valid = rr < t.rows;
                        if constexpr (kFp8) {
                            const float rs = valid ? p.row_scale[t.row0 + rr] : 0.0f;
#pragma unroll
                            for (int k = 0; k < 16; ++k) a[k] *= rs;
                        }
                        uint32_t pk[8];
                        int kexp = 0;
                        if (p.yexp != nullptr) {
                            float amax = 0.0f;
#pragma unroll
                            for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(a[k]));
                            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
                            kexp = f16_chunk_exp(amax);
                            const float down = exp2_int(-kexp);
#pragma unroll
                            for (int k = 0; k < 16; k += 2) pk[k >> 1] = pack_f16x2(a[k] * down, a[k + 1] * down);
                        } else {
#pragma unroll
                            for (int k = 0; k < 16; k += 2) pk[k >> 1] = pack_bf16x2(a[k], a[k + 1]);
                        }
                        if (valid) {
                            uint4* dst = reinterpret_cast<uint4*>(
                                p.out + static_cast<size_t>(t.row0 + rr) * p.out_ld + col0 + hh * 16);
                            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                            if (p.yexp != nullptr && hh == 0)
                                p.yexp[static_cast<size_t>(t.row0 + rr) * (p.H / 32) + col0 / 32] =
                                    static_cast<int8_t>(kexp);
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive_remote(tempty0);
            acc_phase ^= 1u;
        }
        // this warp's TMA stores have left shared memory and reached global memory
        if (lane == 0) ptx::bulk_wait_all();
    }

    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// rank-2/3 K-major map with a {row_bytes of K, box_rows[, 1]} box and the
// swizzle of that width (128 or 64 bytes)
bool make_map(CUtensorMap* m, const void* ptr, bool fp8, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides_bytes, cuuint32_t box_rows, int row_bytes) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(fp8 ? row_bytes : row_bytes / 2), box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    const CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          static_cast<cuuint32_t>(rank), const_cast<void*>(ptr), dims, strides_bytes, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Map of a 16-bit [rows, cols] output (row pitch cols) for the epilogues' TMA
// stores: 32 x 32 boxes, 64-byte swizzle. 0 where TMA cannot address it (the
// epilogues then store every row themselves).
int out_map(CUtensorMap* m, const void* out, int cols, int rows) {
    if (rows <= 0 || (reinterpret_cast<uintptr_t>(out) & 15) != 0 || (cols * 2) % 16 != 0) return 0;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    return make_map(m, out, false, 2, dims, strides, 32, 64) ? 1 : 0;
}

int num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

int gemm1_half(int I) {
    if (I % 128 == 0) return 128;
    if (I % 96 == 0) return 96;
    return 64;
}

std::atomic<int> g_inject{0};
std::atomic<int> g_inject_fold{0};

// Launch of a persistent grid; cooperative (every CTA resident at once, or the
// launch fails) when the kernel's CTAs wait on one another (the folded combine)
template <typename Kern>
cudaError_t launch_grid(Kern kern, int grid, int threads, int smem, bool coop, cudaStream_t st,
                        const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2, const TcParams& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = coop ? attr : nullptr;
    cfg.numAttrs = coop ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a, b, a2, p);
}

template <bool kFp8, bool kGemm1, int kBN, bool kPair>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2, const TcParams& p,
                       cudaStream_t st, const char* name) {
    constexpr int kRowB = SRE_STAGE_ROW_BYTES;
    constexpr int smem = Ring<kRowB, kBN, kPair>::SMEM;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(grouped_gemm_kernel<kFp8, kGemm1, kBN, kPair, kRowB>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    ProfileScope ps(name, st);
    const cudaError_t err = launch_grid(grouped_gemm_kernel<kFp8, kGemm1, kBN, kPair, kRowB>, num_sms(), 320, smem,
                                        p.fold_e >= 0, st, a, b, a2, p);
    note_launch();
    return err;
}

// CTA pairs: as many clusters of two as can be resident at once (a TPC with
// one usable SM holds none), each walking the units persistently
template <bool kFp8, bool kGemm1, int kBN, int kNSUB>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2, const TcParams& p,
                        cudaStream_t st, const char* name) {
    constexpr int kRowB = SRE_STAGE_ROW_BYTES;
    constexpr int smem = Ring2<kRowB, kBN, kNSUB>::SMEM;
    auto kern = grouped_gemm_pair_kernel<kFp8, kGemm1, kBN, kNSUB, kRowB>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    static int clusters = 0;
    std::call_once(once, [kern] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (attr_err != cudaSuccess) return;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1), 1, 1);
        cfg.blockDim = dim3(320, 1, 1);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        attr_err = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        clusters = n;
        if (attr_err == cudaSuccess && n < 1) attr_err = cudaErrorNotSupported;
    });
    if (attr_err != cudaSuccess) return attr_err;
    ProfileScope ps(name, st);
    const cudaError_t err = launch_grid(kern, 2 * clusters, 320, smem, p.fold_e >= 0, st, a, b, a2, p);
    note_launch();
    return err;
}

// tokens as N on CTA pairs: sized like launch_pair
template <bool kFp8, bool kGemm1>
cudaError_t launch_swap(const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& x2, const TcParams& p,
                        cudaStream_t st, const char* name) {
    constexpr int kRowB = SRE_STAGE_ROW_BYTES;
    constexpr int smem = RingS<kRowB>::SMEM;
    auto kern = grouped_gemm_swap_kernel<kFp8, kGemm1, kRowB>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    static int clusters = 0;
    std::call_once(once, [kern] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (attr_err != cudaSuccess) return;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1), 1, 1);
        cfg.blockDim = dim3(SW_THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        attr_err = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        clusters = n;
        if (attr_err == cudaSuccess && n < 1) attr_err = cudaErrorNotSupported;
    });
    if (attr_err != cudaSuccess) return attr_err;
    ProfileScope ps(name, st);
    kern<<<2 * clusters, SW_THREADS, smem, st>>>(w, x, x2, p);
    note_launch();
    return cudaGetLastError();
}

template <bool kFp8, bool kPair>
cudaError_t launch_gemm1(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2, const TcParams& p,
                         int half, cudaStream_t st) {
    if (half == 128) return launch_one<kFp8, true, 256, kPair>(a, b, a2, p, st, "gemm1_tc");
    if (half == 96) return launch_one<kFp8, true, 192, kPair>(a, b, a2, p, st, "gemm1_tc");
    return launch_one<kFp8, true, 128, kPair>(a, b, a2, p, st, "gemm1_tc");
}

template <bool kFp8>
cudaError_t launch_gemm1_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2, const TcParams& p,
                              int half, bool wide, cudaStream_t st) {
    if (wide) return launch_pair<kFp8, true, 256, 2>(a, b, a2, p, st, "gemm1_tc");
    if (half == 128) return launch_pair<kFp8, true, 256, 1>(a, b, a2, p, st, "gemm1_tc");
    if (half == 96) return launch_pair<kFp8, true, 192, 1>(a, b, a2, p, st, "gemm1_tc");
    return launch_pair<kFp8, true, 128, 1>(a, b, a2, p, st, "gemm1_tc");
}

}  // namespace

bool make_map_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    return make_map(m, ptr, false, 2, dims, strides, box_rows, 128);
}

void ffn_tc_inject_stall(int n_launches) { g_inject.store(n_launches); }
void ffn_tc_inject_fold_stall(int n_launches) { g_inject_fold.store(n_launches); }

bool ffn_tc_supported(const FfnArgs& a) {
    if (a.act_dtype != MOE_BF16) return false;
    if (a.w_dtype != MOE_BF16 && a.w_dtype != MOE_E4M3) return false;
    if (a.H % 256 != 0 || a.I % 64 != 0) return false;
    if (a.E + 1 > TC_MAXE) return false;
    if (encode_fn() == nullptr) return false;
    return true;
}

cudaError_t launch_ffn_tc(const FfnArgs& a, cudaStream_t st) {
    if (a.R == 0) return cudaSuccess;
    const bool fp8 = a.w_dtype == MOE_E4M3;
    const int esz = fp8 ? 1 : 2;
    const int half = gemm1_half(a.I);
    constexpr int kRowBytes = SRE_STAGE_ROW_BYTES;
    const int kel = fp8 ? kRowBytes : kRowBytes / 2;
    // rows of the grouped pass gathered from the token matrix (rows are the
    // tokens themselves when perm is null)
    const void* xp = a.xt;
    const float* xp_scale = a.xt_scale;
    if (a.perm != nullptr && a.xp_ready) {
        xp = a.xp;
        xp_scale = a.xp_scale;
    } else if (a.perm != nullptr) {
        // the direct group's rows are not copied: GEMM1 reads them from xt
        const int32_t* skip = a.direct_e >= 0 ? a.offsets + a.direct_e : nullptr;
        const cudaError_t e = launch_gather_rows(a.R, a.S, a.H, esz, a.xt, a.xt_scale, a.perm, a.xp, a.xp_scale,
                                                 skip, st);
        if (e != cudaSuccess) return e;
        xp = a.xp;
        xp_scale = a.xp_scale;
    }
    int inject = 0;
    {
        int cur = g_inject.load();
        while (cur > 0 && !g_inject.compare_exchange_weak(cur, cur - 1)) {
        }
        inject = cur > 0 ? 1 : 0;
    }

    // CTA pairs (cta_pair > 0); 256 x 512 pair tiles (cta_pair == 2) where the
    // output width divides into them (GEMM1: I % 256, GEMM2: H % 512). Chosen by
    // default for bf16 layers whose groups average >= 192 rows: measured on B200,
    // prefill_bf16 GEMM1 + GEMM2 1.86 ms with pair tiles vs 1.91 ms with
    // single-CTA 256-row units; E4M3 layers and small groups are faster on
    // single-CTA 128-row units (prefill_fp8 4.95 vs 6.29 ms per layer).
    // cta_pair == 3: tokens as the MMA's N dimension (grouped_gemm_swap_kernel)
    // where the widths divide (GEMM1: I % 256, GEMM2: H % 512), else as 2.
    // cta_pair == 4 (the default for large bf16 groups): GEMM1 as 3, GEMM2 as 2.
    const bool big_bf16 = a.w_dtype == MOE_BF16 && a.R >= 192 * a.E;
    const int cta_pair = a.cta_pair >= 0 ? a.cta_pair : ((a.unit_rows == 0 && big_bf16) ? 4 : 0);
    const bool two_sm = cta_pair > 0;
    const bool swap1 = (cta_pair == 3 || cta_pair == 4) && a.I % 256 == 0;
    const bool swap2 = cta_pair == 3 && a.H % 512 == 0;
    const bool wide1 = cta_pair >= 2 && half == 128 && a.I % 256 == 0;
    const bool wide2 = cta_pair >= 2 && a.H % 512 == 0;
    const int bn1 = wide1 ? 2 * half : half;     // h columns per unit (swap: 256 as well)

    // GEMM1: A = Xp [R, H] (rows gathered by the gather kernel); B = W13 viewed as
    // [2E][I][H] (gate/up halves separately clipped at I)
    CUtensorMap ta, tb;
    {
        const cuuint64_t ad[2] = {static_cast<cuuint64_t>(a.H), static_cast<cuuint64_t>(a.R)};
        const cuuint64_t as[1] = {static_cast<cuuint64_t>(a.H) * esz};
        const cuuint64_t bd[3] = {static_cast<cuuint64_t>(a.H), static_cast<cuuint64_t>(a.I),
                                  static_cast<cuuint64_t>(2 * a.E)};
        const cuuint64_t bs[2] = {static_cast<cuuint64_t>(a.H) * esz, static_cast<cuuint64_t>(a.I) * a.H * esz};
        // swap: each CTA stages 128 gate and 128 up rows of the 256 h columns
        if (!make_map(&ta, xp, fp8, 2, ad, as, TC_BM, kRowBytes) ||
            !make_map(&tb, a.w13, fp8, 3, bd, bs, swap1 ? TC_BM : bn1, kRowBytes))
            return cudaErrorInvalidValue;
    }
    // the direct group's A: the token matrix [T, H]
    CUtensorMap ta2 = ta;
    const int direct_e = (a.perm != nullptr) ? a.direct_e : -1;
    if (direct_e >= 0) {
        const cuuint64_t ad[2] = {static_cast<cuuint64_t>(a.H), static_cast<cuuint64_t>(a.T)};
        const cuuint64_t as[1] = {static_cast<cuuint64_t>(a.H) * esz};
        if (!make_map(&ta2, a.xt, fp8, 2, ad, as, TC_BM, kRowBytes)) return cudaErrorInvalidValue;
    }
    TcParams p;
    p.E = a.E; p.H = a.H; p.I = a.I;
    p.n_tiles_n = ceil_div(a.I, bn1);
    p.bn_out = bn1;
    p.k_blocks = ceil_div(a.H, kel);
    p.offsets = a.offsets;
    p.tile_off = a.tile_off;
    p.out = static_cast<uint16_t*>(a.h);
    p.out_ld = a.I;
    p.out_tma = out_map(&p.tm_out, a.h, a.I, a.R);
    p.row_scale = fp8 ? xp_scale : nullptr;
    p.direct_e = direct_e;
    p.first_e = a.perm != nullptr ? a.direct_e : -1;
    p.direct_scale = fp8 ? a.xt_scale : nullptr;
    p.col_scale = fp8 ? a.s13 : nullptr;
    p.yexp = nullptr;
    p.fold_e = -1;
    p.fold_S = 0;
    p.fold_inv = nullptr;
    p.fold_w = nullptr;
    p.fold_out = nullptr;
    p.fold_out_f32 = 0;
    p.ready = nullptr;
    p.fold_extra = 0;
    p.status = a.status;
    p.wait_limit = inject ? (20ll << 20) : (4ll << 30);
    p.inject_stall = inject;
    // single-CTA units: M = 256 (two m-tiles sharing each weight stage) when
    // forced, 128 rows otherwise (measured on B200: E4M3 layers are faster with
    // 128-row units, prefill_fp8 4.95 vs 6.04 ms, skewed_fp8 0.84 vs 0.99 ms)
    const bool pair = a.unit_rows == 256;
    cudaError_t err;
    if (swap1)
        err = fp8 ? launch_swap<true, true>(tb, ta, ta2, p, st, "gemm1_tc")
                  : launch_swap<false, true>(tb, ta, ta2, p, st, "gemm1_tc");
    else if (two_sm)
        err = fp8 ? launch_gemm1_pair<true>(ta, tb, ta2, p, half, wide1, st)
                  : launch_gemm1_pair<false>(ta, tb, ta2, p, half, wide1, st);
    else
        err = fp8 ? (pair ? launch_gemm1<true, true>(ta, tb, ta2, p, half, st)
                          : launch_gemm1<true, false>(ta, tb, ta2, p, half, st))
                  : (pair ? launch_gemm1<false, true>(ta, tb, ta2, p, half, st)
                          : launch_gemm1<false, false>(ta, tb, ta2, p, half, st));
    if (err != cudaSuccess) return err;

    const void* hA = a.h;
    if (fp8) {
        err = launch_quant_rows(a.R, a.I, static_cast<const uint16_t*>(a.h), a.hq, a.h_scale, st, "quant_h");
        if (err != cudaSuccess) return err;
        hA = a.hq;
    }
    // GEMM2: A = h [R, I]; B = W2 viewed as [E*H][I]
    {
        const cuuint64_t ad[2] = {static_cast<cuuint64_t>(a.I), static_cast<cuuint64_t>(a.R)};
        const cuuint64_t as[1] = {static_cast<cuuint64_t>(a.I) * esz};
        const cuuint64_t bd[2] = {static_cast<cuuint64_t>(a.I), static_cast<cuuint64_t>(a.E) * a.H};
        const cuuint64_t bs[1] = {static_cast<cuuint64_t>(a.I) * esz};
        // a CTA pair stages 128 of the 256 weight rows in each CTA
        if (!make_map(&ta, hA, fp8, 2, ad, as, TC_BM, kRowBytes) ||
            !make_map(&tb, a.w2, fp8, 2, bd, bs, two_sm ? 128 : 256, kRowBytes))
            return cudaErrorInvalidValue;
    }
    p.n_tiles_n = a.H / (wide2 ? 512 : 256);
    p.bn_out = wide2 ? 512 : 256;
    p.k_blocks = ceil_div(a.I, kel);
    p.out = static_cast<uint16_t*>(a.y);
    p.out_ld = a.H;
    p.out_tma = out_map(&p.tm_out, a.y, a.H, a.R);
    p.row_scale = fp8 ? a.h_scale : nullptr;
    p.direct_e = -1;
    p.col_scale = fp8 ? a.s2 : nullptr;
    p.yexp = a.yexp;
    if (swap2)
        return fp8 ? launch_swap<true, false>(tb, ta, ta, p, st, "gemm2_tc")
                   : launch_swap<false, false>(tb, ta, ta, p, st, "gemm2_tc");
    // the weighted combine folded into the shared expert's units (its group is
    // the last one, rows = tokens in order): the kernels below, with scaled-fp16
    // rows and a layer output to write
    const bool fold = a.fold_out != nullptr && a.yexp != nullptr && a.fold_ready != nullptr &&
                      direct_e == a.E - 1;
    if (fold) {
        p.fold_e = direct_e;
        // the folded combine reads rows other units stored (release / acquire
        // on p.ready): those rows are written by plain stores
        p.out_tma = 0;
        p.fold_S = a.S;
        p.fold_inv = a.fold_inv;
        p.fold_w = a.fold_w;
        p.fold_out = a.fold_out;
        p.fold_out_f32 = a.fold_out_f32;
        p.ready = a.fold_ready;
        int cur = g_inject_fold.load();
        while (cur > 0 && !g_inject_fold.compare_exchange_weak(cur, cur - 1)) {
        }
        if (cur > 0) {
            p.fold_extra = 1;                 // the fold_e units wait for an arrival that never comes
            p.wait_limit = 20ll << 20;
        }
        err = cudaMemsetAsync(a.fold_ready, 0, static_cast<size_t>(p.n_tiles_n) * sizeof(unsigned), st);
        if (err != cudaSuccess) return err;
    }
    auto gemm2 = [&]() -> cudaError_t {
        if (wide2)
            return fp8 ? launch_pair<true, false, 256, 2>(ta, tb, ta, p, st, "gemm2_tc")
                       : launch_pair<false, false, 256, 2>(ta, tb, ta, p, st, "gemm2_tc");
        if (two_sm)
            return fp8 ? launch_pair<true, false, 256, 1>(ta, tb, ta, p, st, "gemm2_tc")
                       : launch_pair<false, false, 256, 1>(ta, tb, ta, p, st, "gemm2_tc");
        if (fp8)
            return pair ? launch_one<true, false, 256, true>(ta, tb, ta, p, st, "gemm2_tc")
                        : launch_one<true, false, 256, false>(ta, tb, ta, p, st, "gemm2_tc");
        return pair ? launch_one<false, false, 256, true>(ta, tb, ta, p, st, "gemm2_tc")
                    : launch_one<false, false, 256, false>(ta, tb, ta, p, st, "gemm2_tc");
    };
    err = gemm2();
    if (fold && err != cudaSuccess) {
        // the cooperative launch was refused (the grid cannot be made co-resident):
        // rows of every group, combined separately by the caller
        cudaGetLastError();
        p.fold_e = -1;
        p.ready = nullptr;
        p.fold_extra = 0;
        return gemm2();
    }
    if (fold && err == cudaSuccess && a.folded != nullptr) *a.folded = true;
    return err;
}

}  // namespace sre
