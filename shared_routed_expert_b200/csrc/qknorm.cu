// Fused QK-norm + partial RoPE on the attention's q and k heads.
//
// "GLM4-MoE生产环境优化：SGLang降低65%首Token延迟", section 2.2 QK-Norm-RoPE
// fusion, and the de/en pages, section 2 "Qknorm Fusion": normalisation and
// rotary embedding are both head-wise, so one kernel does both; in GLM4-MoE
// only half of each head's dimensions rotate.
//
// Per token t and q/k head h (the fused qkv row is q heads | k heads | v heads;
// v is not touched):
//   u = v / sqrt(mean(v^2) + eps) * w            (RMSNorm over head_dim; w per
//                                                 dimension, q or k weight)
//   for i < rot/2: (u_i, u_{i+rot/2}) -> (u_i c - u_{i+rot/2} s,
//                                         u_{i+rot/2} c + u_i s)
//   with c, s the table's cos/sin of angle i at the token's position; the
//   dimensions from rot on pass through. fp32 arithmetic, one bf16 rounding.
//
// One warp per eight heads of a token: lane l holds dimensions EPL*l ..
// EPL*l + EPL-1 of each (EPL = head_dim / 32), the sum of squares is a warp
// reduction, and a dimension's rotation partner (rot/2 away) sits
// rot/2 / EPL lanes away, fetched by one shuffle. Memory-bound: each head is
// read and written once.
#include "kernels.cuh"

namespace sre {

namespace {

constexpr int QK_WARPS = 8;

template <int EPL>
struct Vec;
template <>
struct Vec<2> { using T = uint32_t; };
template <>
struct Vec<4> { using T = uint2; };
template <>
struct Vec<8> { using T = uint4; };

template <int EPL>
__device__ __forceinline__ void unpack(const typename Vec<EPL>::T& v, float (&f)[EPL]) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
    for (int j = 0; j < EPL / 2; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// HPW consecutive heads of one token per warp, all loads in flight before the
// arithmetic (the kernel is bound by bytes in flight, not by its few flops)
constexpr int QK_HPW = 8;

template <int EPL>
__global__ void __launch_bounds__(QK_WARPS * 32) qk_norm_rope_kernel(
    int T, int n_q, int n_kv, int rot, float eps, uint16_t* __restrict__ qkv, const int32_t* __restrict__ pos,
    int max_pos, const uint16_t* __restrict__ q_w, const uint16_t* __restrict__ k_w,
    const float* __restrict__ cos_sin, int32_t* __restrict__ bad) {
    constexpr int D = 32 * EPL;
    using V = typename Vec<EPL>::T;
    const int lane = threadIdx.x & 31;
    const int heads = n_q + n_kv;
    const int groups = (heads + QK_HPW - 1) / QK_HPW;           // head groups per token
    const long long item = static_cast<long long>(blockIdx.x) * QK_WARPS + (threadIdx.x >> 5);
    if (item >= static_cast<long long>(T) * groups) return;
    const int t = static_cast<int>(item / groups);
    const int h0 = static_cast<int>(item % groups) * QK_HPW;
    const int nh = min(QK_HPW, heads - h0);
    const int p = pos[t];
    if (p < 0 || p >= max_pos) {
        if (lane == 0 && bad != nullptr) atomicAdd(bad, nh);
        return;
    }
    V* base = reinterpret_cast<V*>(qkv + static_cast<size_t>(t) * (heads + n_kv) * D + static_cast<size_t>(h0) * D);
    V raw[QK_HPW];
#pragma unroll
    for (int k = 0; k < QK_HPW; ++k)
        if (k < nh) raw[k] = base[k * 32 + lane];
    float wq[EPL], wk[EPL];
    unpack<EPL>(reinterpret_cast<const V*>(q_w)[lane], wq);
    unpack<EPL>(reinterpret_cast<const V*>(k_w)[lane], wk);

    const int half = rot >> 1;
    const int i0 = lane * EPL;                 // first dimension of this lane
    const int lane_off = half / EPL;           // rotation partners are this many lanes apart
    const int src = (i0 < half) ? lane + lane_off : (i0 < rot ? lane - lane_off : lane);
    // this lane's cos/sin (one row per token, shared by its heads)
    float c[EPL], sn[EPL];
    const float* cs = cos_sin + static_cast<size_t>(p) * rot;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        const int i = i0 + j;
        const int a = i < half ? i : i - half;
        c[j] = i < rot ? cs[a] : 1.0f;
        sn[j] = i < rot ? (i < half ? -cs[half + a] : cs[half + a]) : 0.0f;
    }

#pragma unroll
    for (int k = 0; k < QK_HPW; ++k) {
        if (k >= nh) break;                                      // warp-uniform
        float v[EPL];
        unpack<EPL>(raw[k], v);
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) ss = fmaf(v[j], v[j], ss);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
        const float r = rsqrtf(ss / D + eps);
        const bool is_q = h0 + k < n_q;
        uint32_t o[EPL / 2];
#pragma unroll
        for (int j = 0; j < EPL; j += 2) {
            float y[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float u = v[j + q] * r * (is_q ? wq[j + q] : wk[j + q]);
                const float partner = __shfl_sync(0xFFFFFFFFu, u, src);
                // first half: u c - partner s; second half: u c + partner s; pass-through: u
                y[q] = u * c[j + q] + partner * sn[j + q];
            }
            o[j >> 1] = pack_bf16x2(y[0], y[1]);
        }
        base[k * 32 + lane] = *reinterpret_cast<const V*>(o);
    }
}

template <int EPL>
void launch_epl(int T, int n_q, int n_kv, int rot, float eps, uint16_t* qkv, const int32_t* pos, int max_pos,
                const uint16_t* q_w, const uint16_t* k_w, const float* cos_sin, int32_t* bad, cudaStream_t st) {
    const long long items = static_cast<long long>(T) * ((n_q + n_kv + QK_HPW - 1) / QK_HPW);
    const unsigned blocks = static_cast<unsigned>((items + QK_WARPS - 1) / QK_WARPS);
    qk_norm_rope_kernel<EPL><<<blocks, QK_WARPS * 32, 0, st>>>(T, n_q, n_kv, rot, eps, qkv, pos, max_pos, q_w,
                                                                k_w, cos_sin, bad);
}

}  // namespace

bool qk_norm_rope_supported(int head_dim, int rot) {
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return false;
    const int epl = head_dim / 32;
    return rot >= 0 && rot <= head_dim && rot % 2 == 0 && (rot / 2) % epl == 0;
}

cudaError_t launch_qk_norm_rope(int T, int n_q, int n_kv, int head_dim, int rot, float eps, uint16_t* qkv,
                                const int32_t* pos, int max_pos, const uint16_t* q_w, const uint16_t* k_w,
                                const float* cos_sin, int32_t* bad, cudaStream_t st) {
    if (T == 0 || n_q + n_kv == 0) return cudaSuccess;
    ProfileScope ps("qk_norm_rope", st);
    if (head_dim == 64)
        launch_epl<2>(T, n_q, n_kv, rot, eps, qkv, pos, max_pos, q_w, k_w, cos_sin, bad, st);
    else if (head_dim == 128)
        launch_epl<4>(T, n_q, n_kv, rot, eps, qkv, pos, max_pos, q_w, k_w, cos_sin, bad, st);
    else
        launch_epl<8>(T, n_q, n_kv, rot, eps, qkv, pos, max_pos, q_w, k_w, cos_sin, bad, st);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sre
