// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace sre {

// ---- launch accounting / optional per-kernel timing (api.cu)
void note_launch();
struct ProfileScope {
    ProfileScope(const char* name, cudaStream_t st);
    ~ProfileScope();
    int slot;
    cudaStream_t stream;
};

// ---- router (route.cu)
int router_split_count(int T, int H);
size_t router_partial_floats(int T, int H, int E);
// route_scratch: route_tc_scratch_bytes(T, H, n_routed) bytes (may be null when 0)
cudaError_t launch_route(const moe_shape& s, const void* x, const float* wr, const float* bias,
                         int32_t* ids, float* wts, float* logits, float* partials, void* route_scratch,
                         int shared_id, DevStatus* status, cudaStream_t st);

// ---- routing through approximate tensor-core logits, verified exactly (route_tc.cu)
bool route_tc_applies(const moe_shape& s, const float* logits_out);
size_t route_tc_scratch_bytes(int T, int H, int E);
void route_tc_inject_stall(int n_calls);     // testing hook (moe_inject_route_timeout)
cudaError_t launch_route_tc(const moe_shape& s, const void* x, const float* wr, const float* bias, int32_t* ids,
                            float* wts, float* partials, void* scratch, int shared_id, DevStatus* status,
                            cudaStream_t st);
// 2-D TMA map of a bf16 row-major [rows, cols] matrix: boxes of 64 columns
// (128 bytes, 128-byte swizzle) by box_rows rows (ffn_tc.cu)
bool make_map_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows);

// ---- permutation (permute.cu)
constexpr int kPermChunk = 512;      // flat slots per scatter chunk
constexpr int kTileM = 128;          // rows per expert GEMM tile (tile schedule granularity)
size_t permute_scratch_ints(int R, int E);
// Also fills tile_off[E+1] (exclusive scan of ceil(count/kTileM)). With
// fused_bar (one unsigned of device memory) the batches the three-kernel path
// would take run as one cooperative kernel where its grid fits on the device.
cudaError_t launch_permute(int R, int E, const int32_t* ids, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* tile_off, int32_t* scratch,
                           DevStatus* st, cudaStream_t stream, unsigned* fused_bar = nullptr);
// Xp[r] = x[perm[r] / S] (bf16 or fp32 rows, or E4M3 codes + per-row scale);
// rows in [skip[0], skip[1]) are left out when skip != null (a group whose rows
// the GEMM reads from x directly)
cudaError_t launch_gather_rows(int R, int S, int H, int elem_bytes, const void* x,
                               const float* xscale, const int32_t* perm, void* xp, float* xpscale,
                               const int32_t* skip, cudaStream_t stream);
// Token-major form of the same rows from bf16 tokens x [T, H]: for each token t
// and slot k, row inv[t * S + k] of xp (rows in [skip[0], skip[1]) and slots
// without a row in [0, R) are left out). With xq != null (E4M3 layers) the
// token's row is quantised per row first (codes and scale to xq[t], xscale[t],
// the same codes as launch_quant_rows) and xp / xpscale receive the codes.
bool scatter_rows_supported(int H);
cudaError_t launch_scatter_rows(int T, int S, int R, int H, const void* x, const int32_t* inv,
                                const int32_t* skip, uint8_t* xq, float* xscale, void* xp, float* xpscale,
                                cudaStream_t stream);
// per-row E4M3 quantisation of bf16 rows
cudaError_t launch_quant_rows(int rows, int cols, const uint16_t* in, uint8_t* codes,
                              float* scales, cudaStream_t stream, const char* name = "quant_rows");

// ---- expert FFN, CUDA-core path (ffn_simt.cu)
struct FfnArgs {
    int R, H, I, E;               // rows, hidden, intermediate, experts in this pass
    int act_dtype, w_dtype;
    // activations: the token matrix and how rows map to it
    const void* xt;               // [T, H] x (act dtype) or its E4M3 codes
    const float* xt_scale;        // [T] per-token E4M3 scale
    int T;
    const int32_t* perm;          // [R] row -> flat slot t*S + k; null: row r is token r
    int S;
    // rows gathered from xt into xp before the GEMMs
    void* xp;                     // [R, H] (act dtype, or E4M3 codes)
    float* xp_scale;              // [R] (E4M3)
    int xp_ready = 0;             // tensor-core path: xp already holds the rows (token-major gather)
    const int32_t* offsets;       // [E+1]
    const int32_t* tile_off;      // [E+1] m-tile prefix (kTileM rows)
    const void* w13; const float* s13;
    const void* w2;  const float* s2;
    void* h;                      // [R, I] act dtype (bf16 or f32)
    uint8_t* hq; float* h_scale;  // [R, I] codes, [R] (E4M3)
    void* y;                      // [R, H] expert rows: act dtype, or fp16 when yexp != null
    // scaled-fp16 rows (yexp != null): y holds fp16(v * 2^-k) and
    // yexp[r * H/32 + c] = k (int8), one power-of-two exponent per 32 columns,
    // chosen so the chunk's largest |v| maps into [2^14, 2^15)
    int8_t* yexp;
    int unit_rows;                // tensor-core work unit: 0 auto, 128 or 256 rows
    int cta_pair;                 // tensor-core: 256-row units split over a CTA pair (cta_group::2)
    int direct_e;                 // expert whose rows are tokens 0..T-1 in order (A read from
                                  // xt directly, not gathered), or -1
    int max_mtiles;               // upper bound of sum_e ceil(count_e / kTileM)
    // moe_forward, fused layer: the weighted combine folded into GEMM2's units of
    // the direct_e group (the last one) where the tensor-core GEMM2 supports it;
    // *folded is set when it ran (the caller then skips the combine pass)
    const int32_t* fold_inv;      // [T*S] flat slot -> row, or null (no fold)
    const float* fold_w;          // [T*S] slot weights
    void* fold_out;               // [T, H] layer output (bf16, or fp32 when fold_out_f32)
    int fold_out_f32;
    unsigned* fold_ready;         // [H / 256] per n-tile counters (zeroed by the launch)
    bool* folded;
    DevStatus* status;
};
cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t stream);

// ---- fused QK-norm + partial RoPE (qknorm.cu)
bool qk_norm_rope_supported(int head_dim, int rot);
cudaError_t launch_qk_norm_rope(int T, int n_q, int n_kv, int head_dim, int rot, float eps, uint16_t* qkv,
                                const int32_t* pos, int max_pos, const uint16_t* q_w, const uint16_t* k_w,
                                const float* cos_sin, int32_t* bad, cudaStream_t st);

// ---- expert FFN, tcgen05 tensor-core path (ffn_tc.cu)
bool ffn_tc_supported(const FfnArgs& a);
cudaError_t launch_ffn_tc(const FfnArgs& a, cudaStream_t stream);
// testing hook: the next n grouped-FFN calls on the tensor-core path run with a
// producer that never issues its loads and a ~10 ms wait limit
void ffn_tc_inject_stall(int n_calls);
// testing hook: in the next n calls that fold the weighted combine into GEMM2,
// the shared expert's units wait for one routed arrival more than there will
// be, with a ~10 ms wait limit
void ffn_tc_inject_fold_stall(int n_calls);

// ---- combine (combine.cu)
// out[t] = sum_k w[t,k] * y[inv[t*S+k]] (+ add_w * add[t] if add != null)
cudaError_t launch_combine(int T, int S, int H, int act_dtype, const void* y, const int32_t* inv,
                           const float* w, const void* add, float add_w, void* out,
                           cudaStream_t stream);
// same over scaled-fp16 rows (y16/yexp, add16/addexp as produced by the GEMM2 epilogue), bf16 out
cudaError_t launch_combine_f16s(int T, int S, int H, const uint16_t* y16, const int8_t* yexp,
                                const int32_t* inv, const float* w, const uint16_t* add16,
                                const int8_t* addexp, float add_w, void* out, bool out_f32, cudaStream_t stream);
// fp32 -> bf16, round to nearest even (the last step of a tensor-parallel layer)
cudaError_t launch_cast_f32_bf16(size_t n, const float* in, uint16_t* out, cudaStream_t stream);

}  // namespace sre
