// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

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
// zero_rows (optional): [T, H] fp32 rows the top-K kernel clears (the combine accumulator)
cudaError_t launch_route(const moe_shape& s, const void* x, const float* wr, const float* bias,
                         int32_t* ids, float* wts, float* logits, float* partials, int shared_id,
                         float* zero_rows, cudaStream_t st);

// ---- permutation (permute.cu)
constexpr int kPermChunk = 512;      // flat slots per scatter chunk
constexpr int kTileM = 128;          // rows per expert GEMM tile (tile schedule granularity)
size_t permute_scratch_ints(int R, int E);
// Also fills tile_off[E+1] (exclusive scan of ceil(count/kTileM)).
cudaError_t launch_permute(int R, int E, const int32_t* ids, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* tile_off, int32_t* scratch,
                           DevStatus* st, cudaStream_t stream);
// Xp[r] = x[perm[r] / S] (bf16 or fp32 rows, or E4M3 codes + per-row scale)
cudaError_t launch_gather_rows(int R, int S, int H, int elem_bytes, const void* x,
                               const float* xscale, const int32_t* perm, void* xp, float* xpscale,
                               cudaStream_t stream);
// per-row E4M3 quantisation of bf16 rows
cudaError_t launch_quant_rows(int rows, int cols, const uint16_t* in, uint8_t* codes,
                              float* scales, cudaStream_t stream);

// ---- expert FFN, CUDA-core path (ffn_simt.cu)
struct FfnArgs {
    int R, H, I, E;               // rows, hidden, intermediate, experts in this pass
    int act_dtype, w_dtype;
    const void* xp;               // [R, H] gathered activations (act dtype, or E4M3 codes)
    const float* xp_scale;        // [R] (E4M3)
    const int32_t* offsets;       // [E+1]
    const int32_t* tile_off;      // [E+1] m-tile prefix (kTileM rows)
    const void* w13; const float* s13;
    const void* w2;  const float* s2;
    void* h;                      // [R, I] act dtype (bf16 or f32)
    uint8_t* hq; float* h_scale;  // [R, I] codes, [R] (E4M3)
    void* y;                      // [R, H] act dtype (row-output mode)
    // combine mode (out_acc != null): instead of writing y, GEMM2 adds
    // w * y_row into out_acc[token] (fp32, [T, H]); token = f / S with
    // f = perm[row] (perm == null: f = row); w = slot_w[f] (slot_w == null: w_const)
    float* out_acc;
    const int32_t* perm;
    int S;
    const float* slot_w;
    float w_const;
    int max_mtiles;               // upper bound of sum_e ceil(count_e / kTileM)
    DevStatus* status;
};
cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t stream);

// ---- expert FFN, tcgen05 tensor-core path (ffn_tc.cu)
bool ffn_tc_supported(const FfnArgs& a);
cudaError_t launch_ffn_tc(const FfnArgs& a, cudaStream_t stream);
// testing hook: the next n grouped-FFN calls on the tensor-core path run with a
// producer that never issues its loads and a ~10 ms wait limit
void ffn_tc_inject_stall(int n_calls);

// ---- combine (combine.cu)
// out[t] = bf16(acc[t]) for the fp32 combine accumulator
cudaError_t launch_round_rows(int T, int H, const float* acc, uint16_t* out, cudaStream_t stream);
// out[t] = sum_k w[t,k] * y[inv[t*S+k]] (+ add_w * add[t] if add != null)
cudaError_t launch_combine(int T, int S, int H, int act_dtype, const void* y, const int32_t* inv,
                           const float* w, const void* add, float add_w, void* out,
                           cudaStream_t stream);

}  // namespace sre
