// C ABI of the shared-experts-fused MoE layer (declared in include/moe.h).
//
// Host side only: argument validation, workspace carving, kernel dispatch on
// the caller's stream, the device status word, launch counting and optional
// per-kernel event timing. No device memory is allocated here.
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.cuh"

namespace sre {

// ------------------------------------------------------------ launch counting
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// ------------------------------------------------------------ profiling
namespace {
struct ProfRec {
    std::string name;
    cudaEvent_t start = nullptr, stop = nullptr;
    bool used = false;
};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof;
std::atomic<bool> g_prof_on{false};
}  // namespace

ProfileScope::ProfileScope(const char* name, cudaStream_t st) : slot(-1), stream(st) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    int idx = -1;
    for (size_t i = 0; i < g_prof.size(); ++i)
        if (!g_prof[i].used) { idx = static_cast<int>(i); break; }
    if (idx < 0) {
        ProfRec r;
        if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return;
        g_prof.push_back(r);
        idx = static_cast<int>(g_prof.size()) - 1;
    }
    g_prof[idx].name = name;
    g_prof[idx].used = true;
    cudaEventRecord(g_prof[idx].start, st);
    slot = idx;
}

ProfileScope::~ProfileScope() {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEventRecord(g_prof[slot].stop, stream);
}

// ------------------------------------------------------------ workspace layout
namespace {

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int act_bytes(int dt) { return dt == MOE_F32 ? 4 : 2; }

struct Layout {
    size_t status, partials, route, ids, wts, counts, offsets, tile_off, perm, inv, chunk, pbar, ready;
    size_t xq, xscale, xp, xp_scale, h, hq, h_scale, y, yexp;
    // unfused only: the shared expert's dense pass
    size_t sh_off, sh_tile, sh_h, sh_hq, sh_hscale, sh_y, sh_yexp;
    size_t total;
};

struct Dims {
    int T, H, I, Er, K, S, E, R;
    bool fused, shared;
};

Dims dims_of(const moe_shape& s, bool fused) {
    Dims d;
    d.T = s.T; d.H = s.H; d.I = s.I; d.Er = s.n_routed; d.K = s.top_k;
    d.shared = s.shared_id >= 0;
    d.fused = fused;
    const bool in_pass = fused && d.shared;      // shared expert inside the grouped pass
    d.S = d.K + (in_pass ? 1 : 0);
    d.E = d.Er + (in_pass ? 1 : 0);
    d.R = d.T * d.S;
    return d;
}

Layout layout_of(const moe_shape& s, const Dims& d) {
    Layout L;
    std::memset(&L, 0, sizeof(L));
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
    const bool fp8 = s.w_dtype == MOE_E4M3;
    const int ab = act_bytes(s.act_dtype);
    L.status = take(sizeof(DevStatus));
    L.partials = take(router_partial_floats(d.T, d.H, d.Er) * 4);
    L.route = take(route_tc_scratch_bytes(d.T, d.H, d.Er));
    L.ids = take(static_cast<size_t>(d.T) * d.S * 4);
    L.wts = take(static_cast<size_t>(d.T) * d.S * 4);
    L.counts = take(static_cast<size_t>(d.E) * 4);
    L.offsets = take(static_cast<size_t>(d.E + 1) * 4);
    L.tile_off = take(static_cast<size_t>(d.E + 1) * 4);
    L.perm = take(static_cast<size_t>(d.R) * 4);
    L.inv = take(static_cast<size_t>(d.R) * 4);
    L.chunk = take(permute_scratch_ints(d.R, d.E) * 4);
    L.pbar = take(4);
    L.ready = take(static_cast<size_t>(d.H / 256) * 4);
    if (fp8) {
        L.xq = take(static_cast<size_t>(d.T) * d.H);
        L.xscale = take(static_cast<size_t>(d.T) * 4);
    }
    L.xp = take(static_cast<size_t>(d.R) * d.H * (fp8 ? 1 : ab));
    L.xp_scale = take(static_cast<size_t>(d.R) * 4);
    L.h = take(static_cast<size_t>(d.R) * d.I * ab);
    if (fp8) {
        L.hq = take(static_cast<size_t>(d.R) * d.I);
        L.h_scale = take(static_cast<size_t>(d.R) * 4);
    }
    // expert rows: fp32 for fp32 layers, else scaled fp16 + one exponent byte per 32 columns
    L.y = take(static_cast<size_t>(d.R) * d.H * ab);
    if (s.act_dtype != MOE_F32) L.yexp = take(static_cast<size_t>(d.R) * (d.H / 32));
    if (!d.fused && d.shared) {
        L.sh_off = take(2 * 4);
        L.sh_tile = take(2 * 4);
        L.sh_h = take(static_cast<size_t>(d.T) * d.I * ab);
        if (fp8) {
            L.sh_hq = take(static_cast<size_t>(d.T) * d.I);
            L.sh_hscale = take(static_cast<size_t>(d.T) * 4);
        }
        L.sh_y = take(static_cast<size_t>(d.T) * d.H * ab);
        if (s.act_dtype != MOE_F32) L.sh_yexp = take(static_cast<size_t>(d.T) * (d.H / 32));
    }
    L.total = off;
    return L;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status check_shape(const moe_shape* s) {
    if (s == nullptr) return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->T > (1 << 20)) return MOE_ERR_INVALID_ARG;
    if (s->H <= 0 || s->I <= 0 || s->n_routed <= 0 || s->top_k <= 0) return MOE_ERR_INVALID_ARG;
    if (s->top_k > s->n_routed) return MOE_ERR_INVALID_ARG;
    if (s->shared_id != -1 && s->shared_id != s->n_routed) return MOE_ERR_INVALID_ARG;
    if (s->renormalize != 0 && s->renormalize != 1) return MOE_ERR_INVALID_ARG;
    if (!(s->routed_scale > 0.0f) || !isfinite(s->routed_scale)) return MOE_ERR_INVALID_ARG;
    if (s->bias_select_only != 0 && s->bias_select_only != 1) return MOE_ERR_INVALID_ARG;
    if (s->out_f32 != 0 && s->out_f32 != 1) return MOE_ERR_INVALID_ARG;
    if (s->H % 256 != 0 || s->I % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (s->n_routed > 256 || s->top_k > 32) return MOE_ERR_UNSUPPORTED;
    const bool ok_dt = (s->act_dtype == MOE_F32 && s->w_dtype == MOE_F32) ||
                       (s->act_dtype == MOE_BF16 && s->w_dtype == MOE_BF16) ||
                       (s->act_dtype == MOE_BF16 && s->w_dtype == MOE_E4M3);
    if (!ok_dt) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

__global__ void dense_offsets_kernel(int rows, int32_t* off, int32_t* tile_off) {
    off[0] = 0;
    off[1] = rows;
    tile_off[0] = 0;
    tile_off[1] = ceil_div(rows, kTileM);
}

__global__ void tile_prefix_kernel(int E, const int32_t* __restrict__ off, int32_t* __restrict__ tile_off) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
        tile_off[e] = acc;
        acc += ceil_div(off[e + 1] - off[e], kTileM);
    }
    tile_off[E] = acc;
}

// Expert FFN over already-gathered rows (xp). Runs quantisation of h in between
// for E4M3 layers.
bool tc_forced_impl(int impl) {
    return impl == MOE_FFN_TCGEN05 || impl == MOE_FFN_TCGEN05_M128 || impl == MOE_FFN_TCGEN05_M256 ||
           impl == MOE_FFN_TCGEN05_PAIR || impl == MOE_FFN_TCGEN05_WIDE || impl == MOE_FFN_TCGEN05_SWAP;
}

// run_ffn takes the tensor-core path for these arguments
bool ffn_takes_tc(const FfnArgs& in, int impl) {
    return ffn_tc_supported(in) && (tc_forced_impl(impl) || (impl == MOE_FFN_AUTO && in.w_dtype != MOE_F32));
}

cudaError_t run_ffn(const FfnArgs& in, int impl, cudaStream_t st) {
    const bool tc_ok = ffn_tc_supported(in);
    const bool tc_forced = tc_forced_impl(impl);
    if (tc_forced || (impl == MOE_FFN_AUTO && in.w_dtype != MOE_F32 && tc_ok)) {
        if (!tc_ok) return cudaErrorNotSupported;
        FfnArgs a = in;
        a.unit_rows = impl == MOE_FFN_TCGEN05_M128 ? 128 : (impl == MOE_FFN_TCGEN05_M256 ? 256 : 0);
        a.cta_pair = impl == MOE_FFN_TCGEN05_PAIR ? 1 : impl == MOE_FFN_TCGEN05_WIDE ? 2
                   : impl == MOE_FFN_TCGEN05_SWAP ? 3
                   : (impl == MOE_FFN_AUTO || impl == MOE_FFN_TCGEN05) ? -1 : 0;
        return launch_ffn_tc(a, st);
    }
    return launch_ffn_simt(in, st);
}

moe_status check_impl(int impl, const moe_shape& s) {
    impl &= ~MOE_FFN_COMBINE_FOLD;
    if (impl < MOE_FFN_AUTO || impl > MOE_FFN_TCGEN05_SWAP) return MOE_ERR_INVALID_ARG;
    if (impl >= MOE_FFN_TCGEN05 && s.w_dtype == MOE_F32) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// Quantises x per token to E4M3 for E4M3 layers; returns the token matrix the
// grouped pass reads (x itself otherwise).
cudaError_t prepare_tokens(const moe_shape& s, const Dims& d, const Layout& L, void* ws, const void* x,
                           const void** xt, const float** xt_scale, cudaStream_t st) {
    if (s.w_dtype == MOE_E4M3) {
        *xt = at<uint8_t>(ws, L.xq);
        *xt_scale = at<float>(ws, L.xscale);
        return launch_quant_rows(d.T, d.H, static_cast<const uint16_t*>(x), at<uint8_t>(ws, L.xq),
                                 at<float>(ws, L.xscale), st, "quant_x");
    }
    *xt = x;
    *xt_scale = nullptr;
    return cudaSuccess;
}

FfnArgs ffn_args(const moe_shape& s, const Dims& d, const Layout& L, void* ws, const void* xt,
                 const float* xt_scale, const int32_t* perm, const void* w13, const float* s13,
                 const void* w2, const float* s2, void* y) {
    FfnArgs a;
    a.R = d.R; a.H = d.H; a.I = d.I; a.E = d.E;
    a.act_dtype = s.act_dtype; a.w_dtype = s.w_dtype;
    a.xt = xt;
    a.xt_scale = xt_scale;
    a.T = d.T;
    a.perm = perm;
    a.S = d.S;
    a.xp = at<void>(ws, L.xp);
    a.xp_scale = at<float>(ws, L.xp_scale);
    a.offsets = at<int32_t>(ws, L.offsets);
    a.tile_off = at<int32_t>(ws, L.tile_off);
    a.w13 = w13; a.s13 = s13; a.w2 = w2; a.s2 = s2;
    a.h = at<void>(ws, L.h);
    a.hq = s.w_dtype == MOE_E4M3 ? at<uint8_t>(ws, L.hq) : nullptr;
    a.h_scale = s.w_dtype == MOE_E4M3 ? at<float>(ws, L.h_scale) : nullptr;
    a.y = y;
    a.yexp = nullptr;
    a.unit_rows = 0;
    a.cta_pair = 0;
    a.direct_e = -1;
    a.max_mtiles = d.R / kTileM + d.E;
    a.fold_inv = nullptr;
    a.fold_w = nullptr;
    a.fold_out = nullptr;
    a.fold_out_f32 = 0;
    a.fold_ready = nullptr;
    a.folded = nullptr;
    a.status = at<DevStatus>(ws, L.status);
    return a;
}

}  // namespace
}  // namespace sre

using namespace sre;

extern "C" {

size_t moe_workspace_size(const moe_shape* shape, int fuse_shared) {
    if (check_shape(shape) != MOE_OK) return 0;
    const Dims d = dims_of(*shape, fuse_shared != 0);
    return layout_of(*shape, d).total;
}

// the routing path's scratch (split router weights, candidate lists), or null
// where that path does not apply to the shape
void* route_scratch(const moe_shape& s, void* ws, const Layout& L) {
    return route_tc_scratch_bytes(s.T, s.H, s.n_routed) ? at<uint8_t>(ws, L.route) : nullptr;
}

moe_status moe_route_topk(const moe_shape* shape, const void* x, const float* router_w,
                          const float* router_bias, int32_t* ids, float* weights, float* logits,
                          void* ws, size_t ws_bytes, void* stream) {
    moe_status rc = check_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!x || !router_w || !ids || !weights || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return MOE_ERR_INVALID_ARG;
    const Dims d = dims_of(*shape, true);
    const Layout L = layout_of(*shape, d);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (shape->T == 0) return MOE_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_route(*shape, x, router_w, router_bias, ids, weights, logits,
                                    at<float>(ws, L.partials), route_scratch(*shape, ws, L), shape->shared_id,
                                    at<DevStatus>(ws, L.status), st));
}

moe_status moe_permute(const moe_shape* shape, const int32_t* ids, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                       void* stream) {
    moe_status rc = check_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!ids || !counts || !offsets || !perm || !inv || !ws) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_INVALID_ARG;
    const Dims d = dims_of(*shape, true);
    const Layout L = layout_of(*shape, d);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_permute(d.R, d.E, ids, counts, offsets, perm, inv,
                                      at<int32_t>(ws, L.tile_off), at<int32_t>(ws, L.chunk),
                                      at<DevStatus>(ws, L.status), st, at<unsigned>(ws, L.pbar)));
}

moe_status moe_grouped_ffn(const moe_shape* shape, const void* x, const int32_t* perm,
                           const int32_t* offsets, const void* w13, const float* s13,
                           const void* w2, const float* s2, void* y, void* ws, size_t ws_bytes,
                           int ffn_impl, void* stream) {
    moe_status rc = check_shape(shape);
    if (rc != MOE_OK) return rc;
    if (ffn_impl & MOE_FFN_COMBINE_FOLD) return MOE_ERR_INVALID_ARG;   // no aggregation here
    if ((rc = check_impl(ffn_impl, *shape)) != MOE_OK) return rc;
    if (!x || !perm || !offsets || !w13 || !w2 || !y || !ws) return MOE_ERR_INVALID_ARG;
    const bool fp8 = shape->w_dtype == MOE_E4M3;
    if (fp8 && (!s13 || !s2)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return MOE_ERR_INVALID_ARG;
    const Dims d = dims_of(*shape, true);
    const Layout L = layout_of(*shape, d);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (shape->T == 0) return MOE_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the grouped passes read offsets and their m-tile prefix from the workspace
    cudaError_t err = cudaMemcpyAsync(at<int32_t>(ws, L.offsets), offsets,
                                      static_cast<size_t>(d.E + 1) * 4, cudaMemcpyDeviceToDevice, st);
    if (err == cudaSuccess) {
        tile_prefix_kernel<<<1, 1, 0, st>>>(d.E, at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.tile_off));
        note_launch();
        err = cudaGetLastError();
    }
    const void* xt = nullptr;
    const float* xt_scale = nullptr;
    if (err == cudaSuccess) err = prepare_tokens(*shape, d, L, ws, x, &xt, &xt_scale, st);
    if (err == cudaSuccess)
        err = run_ffn(ffn_args(*shape, d, L, ws, xt, xt_scale, perm, w13, s13, w2, s2, y), ffn_impl, st);
    return cuda_status(err);
}

moe_status moe_combine(const moe_shape* shape, const void* y, const int32_t* inv,
                       const float* weights, void* out, void* stream) {
    moe_status rc = check_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!y || !inv || !weights || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const Dims d = dims_of(*shape, true);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_combine(d.T, d.S, d.H, shape->act_dtype, y, inv, weights, nullptr,
                                      0.0f, out, st));
}

moe_status moe_cast_f32_bf16(size_t n, const float* in, void* out, void* stream) {
    if (n % 4 != 0 || (n > 0 && (!in || !out))) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!aligned16(in) || (reinterpret_cast<uintptr_t>(out) & 7u))) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_cast_f32_bf16(n, in, static_cast<uint16_t*>(out), static_cast<cudaStream_t>(stream)));
}

moe_status moe_forward(const moe_shape* shape, const void* x, const float* router_w,
                       const float* router_bias, const void* w13, const float* s13,
                       const void* w2, const float* s2, int fuse_shared, void* out, void* ws,
                       size_t ws_bytes, int ffn_impl, void* stream) {
    moe_status rc = check_shape(shape);
    if (rc != MOE_OK) return rc;
    if ((rc = check_impl(ffn_impl, *shape)) != MOE_OK) return rc;
    if (!x || !router_w || !w13 || !w2 || !out || !ws) return MOE_ERR_INVALID_ARG;
    const bool fp8 = shape->w_dtype == MOE_E4M3;
    if (fp8 && (!s13 || !s2)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(w13) || !aligned16(w2) ||
        !aligned16(out) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return MOE_ERR_INVALID_ARG;
    const bool fused = fuse_shared != 0;
    if (!fused && shape->shared_id < 0) return MOE_ERR_INVALID_ARG;
    const bool fold_combine = (ffn_impl & MOE_FFN_COMBINE_FOLD) != 0;
    ffn_impl &= ~MOE_FFN_COMBINE_FOLD;
    const Dims d = dims_of(*shape, fused);
    const Layout L = layout_of(*shape, d);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (shape->T == 0) return MOE_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    int32_t* ids = at<int32_t>(ws, L.ids);
    float* wts = at<float>(ws, L.wts);
    const bool f32_act = shape->act_dtype == MOE_F32;
    const int route_shared = fused ? shape->shared_id : -1;
    cudaError_t err = launch_route(*shape, x, router_w, router_bias, ids, wts, nullptr,
                                   at<float>(ws, L.partials), route_scratch(*shape, ws, L), route_shared,
                                   at<DevStatus>(ws, L.status), st);
    if (err == cudaSuccess)
        err = launch_permute(d.R, d.E, ids, at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets),
                             at<int32_t>(ws, L.perm), at<int32_t>(ws, L.inv),
                             at<int32_t>(ws, L.tile_off), at<int32_t>(ws, L.chunk),
                             at<DevStatus>(ws, L.status), st, at<unsigned>(ws, L.pbar));
    // the token matrix of the grouped pass: x, or its per-token E4M3 codes
    const void* xt = fp8 ? static_cast<const void*>(at<uint8_t>(ws, L.xq)) : x;
    const float* xt_scale = fp8 ? at<float>(ws, L.xscale) : nullptr;
    bool folded = false;
    FfnArgs a = ffn_args(*shape, d, L, ws, xt, xt_scale, at<int32_t>(ws, L.perm), w13, s13, w2, s2,
                         at<void>(ws, L.y));
    a.yexp = f32_act ? nullptr : at<int8_t>(ws, L.yexp);
    // fused layout: the shared expert's group is every token in order (stable
    // permutation, shared id last), so its rows need no gather
    a.direct_e = (fused && d.shared) ? d.E - 1 : -1;
    if (err == cudaSuccess) {
        if (shape->act_dtype == MOE_BF16 && d.T >= 1024 && scatter_rows_supported(d.H) &&
            ffn_takes_tc(a, ffn_impl)) {
            // the grouped rows by token (each token's row read once, quantised
            // there for E4M3 layers) instead of quantising the tokens and then
            // gathering row by row inside the tensor-core pass; small batches
            // keep the row gather (a few tokens leave most SMs idle:
            // decode_bf16, 64 tokens, 25 against 11 us with a warp per token)
            err = launch_scatter_rows(d.T, d.S, d.R, d.H, x, at<int32_t>(ws, L.inv),
                                      a.direct_e >= 0 ? at<int32_t>(ws, L.offsets) + a.direct_e : nullptr,
                                      fp8 ? at<uint8_t>(ws, L.xq) : nullptr, fp8 ? at<float>(ws, L.xscale) : nullptr,
                                      a.xp, a.xp_scale, st);
            a.xp_ready = 1;
        } else {
            err = prepare_tokens(*shape, d, L, ws, x, &xt, &xt_scale, st);
        }
    }
    if (err == cudaSuccess) {
        if (a.direct_e >= 0 && !f32_act && fold_combine) {
            // the weighted combine inside GEMM2's shared-expert units, where the
            // tensor-core GEMM2 runs it (folded tells whether it did)
            a.fold_inv = at<int32_t>(ws, L.inv);
            a.fold_w = wts;
            a.fold_out = out;
            a.fold_out_f32 = shape->out_f32 != 0;
            a.fold_ready = at<unsigned>(ws, L.ready);
            a.folded = &folded;
        }
        err = run_ffn(a, ffn_impl, st);
    }

    if (err == cudaSuccess && !fused) {
        // Unfused: the shared expert as its own dense pass over x (rows = tokens);
        // the combine adds it with weight shared_weight.
        const int esz = fp8 ? 1 : act_bytes(shape->w_dtype);
        const size_t sid = static_cast<size_t>(shape->shared_id);
        FfnArgs a;
        a.R = d.T; a.H = d.H; a.I = d.I; a.E = 1;
        a.act_dtype = shape->act_dtype; a.w_dtype = shape->w_dtype;
        a.xt = xt;
        a.xt_scale = xt_scale;
        a.T = d.T;
        a.perm = nullptr;          // rows are the tokens in order
        a.S = 1;
        a.xp = nullptr;
        a.xp_scale = nullptr;
        a.offsets = at<int32_t>(ws, L.sh_off);
        a.tile_off = at<int32_t>(ws, L.sh_tile);
        a.w13 = static_cast<const char*>(w13) + sid * 2 * d.I * d.H * esz;
        a.s13 = fp8 ? s13 + sid * 2 * d.I : nullptr;
        a.w2 = static_cast<const char*>(w2) + sid * d.H * d.I * esz;
        a.s2 = fp8 ? s2 + sid * d.H : nullptr;
        a.h = at<void>(ws, L.sh_h);
        a.hq = fp8 ? at<uint8_t>(ws, L.sh_hq) : nullptr;
        a.h_scale = fp8 ? at<float>(ws, L.sh_hscale) : nullptr;
        a.y = at<void>(ws, L.sh_y);
        a.yexp = f32_act ? nullptr : at<int8_t>(ws, L.sh_yexp);
        a.unit_rows = 0;
        a.cta_pair = 0;
        a.direct_e = -1;
        a.max_mtiles = ceil_div(d.T, kTileM);
        a.fold_inv = nullptr;
        a.fold_w = nullptr;
        a.fold_out = nullptr;
        a.fold_out_f32 = 0;
        a.fold_ready = nullptr;
        a.folded = nullptr;
        a.status = at<DevStatus>(ws, L.status);
        dense_offsets_kernel<<<1, 1, 0, st>>>(d.T, at<int32_t>(ws, L.sh_off), at<int32_t>(ws, L.sh_tile));
        note_launch();
        err = cudaGetLastError();
        if (err == cudaSuccess) err = run_ffn(a, ffn_impl, st);
    }
    if (err == cudaSuccess && !folded) {
        const int32_t* inv = at<int32_t>(ws, L.inv);
        if (f32_act)
            err = launch_combine(d.T, d.S, d.H, MOE_F32, at<void>(ws, L.y), inv, wts,
                                 fused ? nullptr : at<void>(ws, L.sh_y), shape->shared_weight, out, st);
        else
            err = launch_combine_f16s(d.T, d.S, d.H, at<uint16_t>(ws, L.y), at<int8_t>(ws, L.yexp), inv, wts,
                                      fused ? nullptr : at<uint16_t>(ws, L.sh_y),
                                      fused ? nullptr : at<int8_t>(ws, L.sh_yexp), shape->shared_weight,
                                      out, shape->out_f32 != 0, st);
    }
    return cuda_status(err);
}

moe_status moe_quant_rows_e4m3(int32_t rows, int32_t cols, const void* in, uint8_t* codes,
                               float* scales, void* stream) {
    if (rows < 0 || cols <= 0 || cols % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (!in || !codes || !scales || !aligned16(in) || (reinterpret_cast<uintptr_t>(codes) & 7u))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_quant_rows(rows, cols, static_cast<const uint16_t*>(in), codes, scales,
                                         static_cast<cudaStream_t>(stream)));
}

moe_status moe_qk_norm_rope(int32_t T, int32_t n_q, int32_t n_kv, int32_t head_dim, int32_t rot_dim, float eps,
                            void* qkv, const int32_t* positions, int32_t max_pos, const void* q_norm_w,
                            const void* k_norm_w, const float* cos_sin, int32_t* bad_positions, void* stream) {
    if (T < 0 || n_q < 0 || n_kv < 0 || max_pos <= 0 || !(eps >= 0.0f) || !isfinite(eps))
        return MOE_ERR_INVALID_ARG;
    if (!qkv || !positions || !q_norm_w || !k_norm_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(q_norm_w) || !aligned16(k_norm_w)) return MOE_ERR_INVALID_ARG;
    if (rot_dim > 0 && (!cos_sin || !aligned16(cos_sin))) return MOE_ERR_INVALID_ARG;   // unused when rot_dim == 0
    if (!qk_norm_rope_supported(head_dim, rot_dim)) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_qk_norm_rope(T, n_q, n_kv, head_dim, rot_dim, eps, static_cast<uint16_t*>(qkv),
                                           positions, max_pos, static_cast<const uint16_t*>(q_norm_w),
                                           static_cast<const uint16_t*>(k_norm_w), cos_sin, bad_positions,
                                           static_cast<cudaStream_t>(stream)));
}

moe_status moe_get_status(void* ws, void* stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus h;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemset(ws, 0, sizeof(DevStatus)) != cudaSuccess) return MOE_ERR_CUDA;
    return static_cast<moe_status>(h.code);
}

moe_status moe_clear_status(void* ws, void* stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(DevStatus), static_cast<cudaStream_t>(stream)));
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_DEVICE: return "bad data on device (expert id out of range)";
    }
    return "unknown status";
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

void moe_inject_wait_timeout(int n_calls) { ffn_tc_inject_stall(n_calls > 0 ? n_calls : 0); }

void moe_inject_fold_timeout(int n_calls) { ffn_tc_inject_fold_stall(n_calls > 0 ? n_calls : 0); }

void moe_inject_route_timeout(int n_calls) { route_tc_inject_stall(n_calls > 0 ? n_calls : 0); }

void moe_profile_enable(int on) { g_prof_on.store(on != 0); }

void moe_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : g_prof) r.used = false;
}

moe_status moe_profile_read(const char* name, int64_t* launches, double* total_ms) {
    if (!name || !launches || !total_ms) return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    int64_t n = 0;
    double ms = 0.0;
    for (auto& r : g_prof) {
        if (!r.used || r.name != name) continue;
        if (cudaEventSynchronize(r.stop) != cudaSuccess) return MOE_ERR_CUDA;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return MOE_ERR_CUDA;
        ms += t;
        ++n;
    }
    *launches = n;
    *total_ms = ms;
    return MOE_OK;
}

}  // extern "C"
