/*
 * moe.h - C ABI of the shared-experts-fused MoE expert layer for B200 (sm_100a).
 *
 * The layer (GLM4-MoE expert layer, "Optimizing GLM4-MoE for production",
 * Novita AI, section 1 "Shared Experts Fusion"): every token goes through one
 * shared expert and through the top-k routed experts its router picks, and the
 * expert outputs are aggregated with weights. The fusion appends the shared
 * expert to the routed ones as expert number n_routed (160 for GLM-4.7) and
 * gives every token top_k + 1 slots, the shared expert fixed in the last slot,
 * so that one routed-MoE pass computes all of them.
 *
 * Conventions for every entry point
 *  - Pointers named x, w13, ids, ... are DEVICE pointers; the caller owns every
 *    buffer, including the workspace `ws`. The library never allocates device
 *    memory and never synchronises except in moe_get_status.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it; calls on one workspace must not
 *    overlap on the GPU.
 *  - Tensors are dense, row-major, with the shapes written in brackets.
 *    bf16 tensors are passed as raw 16-bit patterns, E4M3 tensors as bytes
 *    (OCP E4M3FN codes), fp32 as float.
 *  - Errors found on the host (null or misaligned pointers, unsupported sizes or
 *    dtypes, a workspace that is too small) return immediately with nothing
 *    enqueued. Errors found on the device (an expert id out of range, a bounded
 *    wait that ran out) are recorded in the workspace's status word and read
 *    back by moe_get_status; kernels never trap.
 *  - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *  - Calls are thread-safe; no state is kept between calls except the optional
 *    profiling and launch counters below.
 */
#ifndef SRE_MOE_H
#define SRE_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer or inconsistent shape */
    MOE_ERR_UNSUPPORTED = 2,   /* sizes or dtype combination this build does not run */
    MOE_ERR_WORKSPACE = 3,     /* ws_bytes smaller than moe_workspace_size() */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    MOE_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out (device-side) */
    MOE_ERR_DEVICE = 6         /* bad data seen on the device (e.g. expert id out of range) */
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2 } moe_dtype;

/* Shape and options of one layer call.
 *   T            tokens
 *   H            hidden size; multiple of 256 (router reduction order, tiles)
 *   I            per-expert intermediate size; multiple of 64
 *   n_routed     routed experts E_r (1..256)
 *   top_k        routed experts per token K (1..min(n_routed, 32))
 *   shared_id    n_routed: a shared expert is stored as expert n_routed (the
 *                fused layout); -1: no shared expert
 *   shared_weight  weight of the shared slot (1.0 reproduces the unfused sum)
 *   renormalize  1: softmax over the K selected logits; 0: full softmax over
 *                all n_routed logits evaluated at the selected ids
 *   act_dtype    dtype of x, out and of the expert rows y: MOE_F32 or MOE_BF16
 *   w_dtype      expert weight dtype: MOE_F32 (with act F32), MOE_BF16 or
 *                MOE_E4M3 (both with act BF16)
 *   routed_scale routed scaling factor s (> 0, finite; 1.0 = none): the routed
 *                slots' weights are s * softmax; the shared slot keeps
 *                shared_weight (engines that scale the whole fused sum by s
 *                give the shared slot 1/s instead: the same output)
 *   bias_select_only  0: router_bias is added to the logits used for both
 *                ranking and weights; 1: the bias only ranks (ids), the
 *                weights use the logits without it
 *   out_f32      0: moe_forward writes out in act_dtype; 1: out is fp32, the
 *                unrounded sum (a tensor-parallel rank's partial output, to
 *                be summed across ranks and rounded once, moe_cast_f32_bf16)
 * Derived: S = top_k + (shared_id >= 0) slots per token in the fused layout,
 * E = n_routed + (shared_id >= 0) experts, R = T*S expert rows. */
typedef struct moe_shape {
    int32_t T, H, I, n_routed, top_k, shared_id;
    float shared_weight;
    int32_t renormalize;
    int32_t act_dtype, w_dtype;
    float routed_scale;
    int32_t bias_select_only;
    int32_t out_f32;
} moe_shape;

/* Kernel choice for the expert GEMMs. AUTO picks the tcgen05 tensor-core
 * kernels for bf16/E4M3 weights and the CUDA-core kernels for fp32. TCGEN05
 * picks the tensor-core work unit itself: for bf16 weights whose groups average
 * >= 192 rows, CTA pairs with GEMM1 as TCGEN05_SWAP and GEMM2 as TCGEN05_WIDE,
 * else 128-row units on single CTAs (as TCGEN05_M128);
 * TCGEN05_M128 / TCGEN05_M256 force one of them; TCGEN05_PAIR forces 256-row
 * units split over a pair of CTAs on the two SMs of a TPC (tcgen05 cta_group::2,
 * each SM staging half of every weight tile); TCGEN05_WIDE the same with
 * 256 x 512 tiles per pair (two N = 256 MMAs sharing each activation stage)
 * where the output width allows (GEMM1: I % 256 == 0, GEMM2: H % 512 == 0;
 * 256 x 256 pair tiles otherwise); TCGEN05_SWAP runs CTA pairs with the
 * operands exchanged: 256 weight rows are the MMA's M and up to 256 rows of one
 * expert's group its N, in steps of 16, so a group pads to a multiple of 16
 * rows instead of a multiple of 128 (GEMM1 where I % 256 == 0, GEMM2 where
 * H % 512 == 0; as TCGEN05_WIDE otherwise). */
typedef enum moe_ffn_impl {
    MOE_FFN_AUTO = 0, MOE_FFN_SIMT = 1, MOE_FFN_TCGEN05 = 2,
    MOE_FFN_TCGEN05_M128 = 3, MOE_FFN_TCGEN05_M256 = 4, MOE_FFN_TCGEN05_PAIR = 5,
    MOE_FFN_TCGEN05_WIDE = 6, MOE_FFN_TCGEN05_SWAP = 7
} moe_ffn_impl;

/* Flag OR'ed into ffn_impl of moe_forward: run the weighted aggregation of the
 * fused layer inside the down-projection's units of the shared expert instead
 * of as its own pass over the stored expert rows (where the tensor-core
 * down-projection runs, i.e. not with TCGEN05_SWAP or SIMT). The output is the
 * same bit for bit either way. The separate pass is the default: measured on
 * B200 it is faster (the in-kernel aggregation is bound by the loads a few
 * epilogue warps can keep in flight). */
#define MOE_FFN_COMBINE_FOLD 512

/* Bytes of workspace moe_forward needs for this shape (fused or not). The
 * other entry points need at most this much. Returns 0 for an invalid shape. */
size_t moe_workspace_size(const moe_shape* shape, int fuse_shared);

/* Router: logits, top-K selection and slot weights.
 * Follows the write-up's section 1: each token's router picks its top-8 routed
 * experts; with the fusion the shared expert takes the 9th slot.
 *   x        [T, H] act_dtype       router_w [n_routed, H] fp32
 *   router_bias [n_routed] fp32 or NULL (added to the logits before ranking)
 *   ids      [T, S] int32 out: slots 0..K-1 = routed ids ranked by
 *            (logit desc, id asc); slot K = shared_id when shared_id >= 0
 *   weights  [T, S] fp32 out: softmax weights of the routed slots;
 *            shared_weight in slot K
 *   logits   [T, n_routed] fp32 out, or NULL. Logits are fp32 in a fixed order:
 *            per 256-wide segment of H an fma chain from +0 over ascending h,
 *            segment sums added in ascending order to a total starting at +0,
 *            then the bias; so they are reproducible bit for bit.
 * ids and weights are those of these logits either way. Without logits, a
 * batch of more than 256 tokens (bf16 activations, renormalised top-K, 32 to
 * 256 routed experts, K <= 16, H <= 8192) ranks approximate logits from the
 * tensor cores and forms in the fixed order only the logits of the experts
 * within the approximation's error bound of the K-th key: the same ids and
 * weights, bit for bit.
 * Needs moe_workspace_size(shape, 1) bytes of ws. */
moe_status moe_route_topk(const moe_shape* shape, const void* x, const float* router_w,
                          const float* router_bias, int32_t* ids, float* weights,
                          float* logits, void* ws, size_t ws_bytes, void* stream);

/* Sort the R = T*S slots by expert: the token permutation of "one routed-MoE
 * pass" (section 1). Experts in id order; inside an expert, stable by flat slot
 * index t*S + k, so the shared expert's block is tokens 0..T-1 in order.
 *   ids      [T, S] int32 with values in [0, E); S = top_k + (shared_id >= 0)
 *   counts   [E] int32 out     offsets [E + 1] int32 out (exclusive scan)
 *   perm     [R] int32 out: perm[row] = flat slot index
 *   inv      [R] int32 out: inv[flat] = row
 * An id outside [0, E) sets MOE_ERR_DEVICE in the status word (that slot is
 * dropped). */
moe_status moe_permute(const moe_shape* shape, const int32_t* ids, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                       size_t ws_bytes, void* stream);

/* Expert FFNs for all R rows, grouped by expert (section 1: the shared and
 * routed experts have identical tensor shapes and computation flow, so one
 * grouped pass serves both). Row r belongs to expert e with
 * offsets[e] <= r < offsets[e+1] and reads token perm[r] / S of x.
 * Per row: h = silu(gate . v) * (up . v) (rounded to bf16 for bf16 layers),
 * y = w2[e] . h. E4M3 layers quantise v per token and h per row to E4M3 with
 * scale amax/448, and apply the weight scales per output channel.
 *   x    [T, H] act_dtype
 *   w13  [E, 2I, H] w_dtype: rows [0, I) gate, [I, 2I) up;  s13 [E, 2I] fp32 (E4M3 only, else NULL)
 *   w2   [E, H, I]  w_dtype;                                  s2  [E, H]  fp32 (E4M3 only, else NULL)
 *   y    [R, H] act_dtype out, rows in permuted order
 * Needs moe_workspace_size(shape, 1) bytes of ws. */
moe_status moe_grouped_ffn(const moe_shape* shape, const void* x, const int32_t* perm,
                           const int32_t* offsets, const void* w13, const float* s13,
                           const void* w2, const float* s2, void* y, void* ws,
                           size_t ws_bytes, int ffn_impl, void* stream);

/* Weighted aggregation of the expert outputs (section 1: "all expert outputs
 * are aggregated with weights"):
 *   out[t] = sum_{k<S} weights[t, k] * y[inv[t*S + k]], fp32, slot order,
 *   rounded once to act_dtype.
 *   y [R, H], inv [R], weights [T, S], out [T, H]. */
moe_status moe_combine(const moe_shape* shape, const void* y, const int32_t* inv,
                       const float* weights, void* out, void* stream);

/* The whole layer. fuse_shared = 1: the fused top-(K+1) pass (route -> permute
 * -> grouped FFN over all E experts -> weighted aggregation). fuse_shared = 0: the unfused layer of the
 * pseudocode in section 2.1 of "GLM4-MoE生产环境优化：SGLang降低65%首Token延迟":
 * routed top-K pass plus a separate dense pass of the shared expert added with
 * weight shared_weight (the GPU baseline the fusion is measured against; needs
 * shared_id >= 0).
 * The expert rows are kept as fp16 scaled by a power of two per 32 columns
 * (11 significant bits) and aggregated in fp32 in slot order, rounded once to
 * act_dtype (or left in fp32 when shape->out_f32); the result is deterministic.
 * With MOE_FFN_COMBINE_FOLD in ffn_impl the fused layer's aggregation runs
 * inside the down-projection's units of the shared expert, which come last:
 * each stores its rows, waits (bounded; MOE_ERR_TIMEOUT if it runs out) until
 * the routed units of its columns have stored theirs, and sums every slot of
 * its tokens in slot order (one launch less: the write-up's section 1 argument
 * for the fusion). That kernel is a cooperative launch, all of its CTAs resident
 * at once; where the launch is refused the aggregation runs as its own pass.
 *   x [T, H], router_w [n_routed, H], router_bias [n_routed] or NULL,
 *   w13 [E, 2I, H], s13, w2 [E, H, I], s2 as in moe_grouped_ffn, out [T, H]
 *   (act_dtype, or fp32 when out_f32).
 * Tensor parallelism: a rank that holds every expert's slice of the
 * intermediate dimension (w13 rows gate[j0, j1) and up[j0, j1), w2 columns
 * [j0, j1), I = j1 - j0, with their E4M3 scales) and calls this with out_f32 = 1
 * computes its exact share of the layer: the SwiGLU is per intermediate column,
 * so the ranks' outputs sum to the layer's (E4M3 layers quantise h per row of
 * the slice). Sum the shares across ranks, then moe_cast_f32_bf16.
 * Needs moe_workspace_size(shape, fuse_shared) bytes of ws. */
moe_status moe_forward(const moe_shape* shape, const void* x, const float* router_w,
                       const float* router_bias, const void* w13, const float* s13,
                       const void* w2, const float* s2, int fuse_shared, void* out,
                       void* ws, size_t ws_bytes, int ffn_impl, void* stream);

/* out[i] = bf16(in[i]), round to nearest even; n a multiple of 4, in 16-byte
 * and out 8-byte aligned. */
moe_status moe_cast_f32_bf16(size_t n, const float* in, void* out, void* stream);

/* Per-row E4M3 quantisation used before each E4M3 GEMM: scale = amax/448 in
 * fp32 (amax = 0 -> 1), codes = E4M3_rn_satfinite(v / scale) (fp32 divide).
 *   in [rows, cols] bf16, codes [rows, cols] u8 out, scales [rows] fp32 out.
 * cols must be a multiple of 8. */
moe_status moe_quant_rows_e4m3(int32_t rows, int32_t cols, const void* in, uint8_t* codes,
                               float* scales, void* stream);

/* Synchronises `stream`, reads the workspace status word and clears it.
 * Returns MOE_OK, MOE_ERR_DEVICE or MOE_ERR_TIMEOUT (or MOE_ERR_CUDA). */
moe_status moe_get_status(void* ws, void* stream);

/* Zero the workspace status word (asynchronously on stream). */
moe_status moe_clear_status(void* ws, void* stream);

const char* moe_status_string(moe_status s);

/* Number of kernels this library has launched in this process. */
uint64_t moe_launch_count(void);

/* Optional per-kernel timing: while enabled, every launch is bracketed by CUDA
 * events on its stream. moe_profile_read synchronises those events and returns,
 * for kernel name `name`, the number of launches and their summed device time
 * in milliseconds since the last moe_profile_reset. */
void moe_profile_enable(int on);
void moe_profile_reset(void);
moe_status moe_profile_read(const char* name, int64_t* launches, double* total_ms);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory themselves: code whose device buffers all come from a host framework
 * that owns every allocation and gives plugins no allocator; code that must not
 * call cudaMalloc where it enqueues work (it may synchronise the device, and is
 * not allowed while a stream is being captured); callers with a fixed device
 * footprint. The method on the pages has no counterpart of this call; it is a
 * deployment convenience.
 * Arguments and results are those of moe_permute (ids [T, S] in, counts [E],
 * offsets [E+1], perm [R], inv [R] out, all caller-owned device buffers); the
 * kernels are the same. Their scratch lives in one 1 MiB array in the library's
 * device globals, which every GPU that loads the library holds until the
 * process exits. Limit, with E the number of expert groups (n_routed, + 1 with
 * a shared expert) and S the slots per token:
 *     ceil(T*S / 512) * E <= (1048576 - 256 - round256(4 * (E + 1))) / 4,
 * round256 rounding up to a multiple of 256. The right side is 262016 for
 * E <= 63, 261952 for E in 64..127, 261888 for 128..191 (161 experts and 9
 * slots: T <= 92501), 261824 for 192..255 and 261760 for 256..257. Larger
 * calls return MOE_ERR_UNSUPPORTED before enqueuing anything.
 * The library allocates nothing in this call.
 * The first call on a device looks up the array's device address (once per
 * device and CUDA context, with that device current); make that first call
 * before any stream capture. After cudaDeviceReset the next call is again a
 * first call. All calls share the array and it keeps the last call's contents, so
 * calls that overlap on the GPU (other streams, other host threads) race and
 * must be serialised by the caller. Out-of-range ids are dropped as in
 * moe_permute, but not reported: this call has no status word the caller can
 * read. */
moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* ids, int32_t* counts,
                               int32_t* offsets, int32_t* perm, int32_t* inv, void* stream);

/* Failure-injection hook for tests of the bounded waits: the next n_calls
 * grouped-FFN passes on the tensor-core path run with a TMA producer that never
 * issues its loads and a wait limit of about 10 ms, so their waits run out; the
 * kernels then drain, free TMEM, return, and leave MOE_ERR_TIMEOUT in the status
 * word (the outputs of those calls are garbage). No GPU fault is involved. */
void moe_inject_wait_timeout(int n_calls);

/* Failure-injection hook for the wait of the aggregation inside the fused
 * layer's down-projection: in the next n_calls moe_forward calls that run it,
 * the shared expert's units wait for one more routed-unit arrival than there
 * will be, with a limit of about 10 ms; the waits run out, the kernel drains,
 * frees TMEM and returns, and MOE_ERR_TIMEOUT is left in the status word (the
 * outputs of those calls are garbage). No GPU fault is involved. */
void moe_inject_fold_timeout(int n_calls);

/* Failure-injection hook for the routing through approximate tensor-core
 * logits (moe_route_topk / moe_forward on batches over 256 tokens): in the
 * next n_calls calls that take that path, the approximate-logit kernel issues
 * no loads and waits with a limit of about 10 ms; its waits run out, it drains,
 * frees TMEM and returns, and MOE_ERR_TIMEOUT is left in the status word (the
 * routing of those calls is garbage, but every id stays in range). No GPU fault
 * is involved. */
void moe_inject_route_timeout(int n_calls);

/* Fused QK-norm + partial RoPE on the attention's q and k heads, in place.
 * "GLM4-MoE生产环境优化：SGLang降低65%首Token延迟", section 2.2 QK-Norm-RoPE
 * fusion, and the de/en pages, section 2 "Qknorm Fusion": both steps are
 * head-wise and run as one kernel; in GLM4-MoE only half of each head's
 * dimensions rotate. For token t and each q and k head:
 *   u = v / sqrt(mean(v^2) + eps) * w     (RMSNorm over head_dim; w = q_norm_w
 *                                          for q heads, k_norm_w for k heads)
 *   (u_i, u_{i+rot_dim/2}) -> (u_i c_i - u_{i+rot_dim/2} s_i,
 *                              u_{i+rot_dim/2} c_i + u_i s_i),  i < rot_dim/2
 * with c_i = cos_sin[positions[t]][i], s_i = cos_sin[positions[t]][rot_dim/2 + i];
 * dimensions from rot_dim on pass through. fp32 arithmetic, one rounding.
 *   qkv        [T][(n_q + 2*n_kv) * head_dim] bf16, caller-owned; each row is
 *              q heads | k heads | v heads; q and k are overwritten, v is not
 *              touched
 *   positions  [T] int32, each in [0, max_pos)
 *   q_norm_w, k_norm_w  [head_dim] bf16
 *   cos_sin    [max_pos][rot_dim] fp32 (may be NULL when rot_dim == 0)
 *   eps        >= 0
 *   bad_positions  device int32 counter or NULL: a token whose position is out
 *              of range leaves its heads unchanged and adds one per head
 * head_dim 64, 128 or 256; rot_dim even, <= head_dim, rot_dim/2 a multiple of
 * head_dim/32 (GLM4-MoE: 128 and 64). Asynchronous on `stream`. Returns
 * MOE_ERR_INVALID_ARG for null or misaligned pointers (16 bytes) or bad sizes,
 * MOE_ERR_UNSUPPORTED for other head shapes, MOE_ERR_CUDA on launch failure. */
moe_status moe_qk_norm_rope(int32_t T, int32_t n_q, int32_t n_kv, int32_t head_dim, int32_t rot_dim, float eps,
                            void* qkv, const int32_t* positions, int32_t max_pos, const void* q_norm_w,
                            const void* k_norm_w, const float* cos_sin, int32_t* bad_positions, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SRE_MOE_H */
