// moe_permute_noalloc: the expert permutation without a caller-provided
// workspace, for callers that cannot allocate device memory themselves.
//
// Who needs it: code that gets device buffers only from a host framework that
// owns every allocation and offers no allocator to plugins; code that must not
// call cudaMalloc at the point of use because it may synchronise the device or
// is not allowed there (for example while a stream is being captured into a
// graph); and callers with a hard cap on their device footprint that cannot
// budget a per-call workspace. They still pass ids and the four outputs.
//
// The kernels are the same as moe_permute's; only their scratch (the status
// word, the tile prefix and the per-chunk expert histograms) lives in one
// file-scope __device__ array of kNoAllocScratchBytes instead of a workspace.
// Every GPU that loads the library holds that array until the process exits.
//
// Host code must not pass the array's name to a kernel: on the host it is a
// stand-in symbol, not a device address. The device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first
// call made on it (so make the first call outside any stream capture), and
// cached together with the unique id of the CUDA context it belongs to. A
// cudaDeviceReset ends that context and the module is loaded again in the next
// one, where the array may sit at another address: a call that finds another
// current context looks the address up again (and is then, again, a first
// call).
//
// All calls share the array and it keeps the last call's contents. The status
// word is cleared at the start of every call (report() needs it at zero); the
// histograms are fully rewritten by each call. Calls that overlap on the GPU
// (two streams, or two host threads) race on the array and give wrong results:
// serialise them.
#include <cuda.h>

#include <mutex>

#include "kernels.cuh"

namespace sre {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB per GPU
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_permute_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // unique id of the context the address belongs to

// The driver's cuCtxGetCurrent and cuCtxGetId, looked up through the runtime
// (the library links no driver library).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
template <typename Fn>
Fn driver_fn(const char* name) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(ptr);
}

// Unique id of the calling thread's current context (ids are never reused, unlike
// context handles); 0 when no context is current or the driver calls are missing.
unsigned long long current_context_id() {
    static const CtxGetCurrentFn get = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get == nullptr || get_id == nullptr || get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    unsigned long long ctx = current_context_id();    // 0 before the runtime first used this thread
    if (g_scratch_addr[dev] == nullptr || ctx == 0 || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);    // makes the device's context current
        if (e != cudaSuccess) return e;
        ctx = current_context_id();
        if (ctx == 0) return cudaErrorInitializationError;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

}  // namespace
}  // namespace sre

using namespace sre;

extern "C" moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* ids, int32_t* counts,
                                          int32_t* offsets, int32_t* perm, int32_t* inv, void* stream) {
    if (shape == nullptr || !ids || !counts || !offsets || !perm || !inv) return MOE_ERR_INVALID_ARG;
    const moe_shape& s = *shape;
    if (s.T < 0 || s.T > (1 << 20) || s.n_routed <= 0 || s.top_k <= 0 || s.top_k > s.n_routed)
        return MOE_ERR_INVALID_ARG;
    if (s.shared_id != -1 && s.shared_id != s.n_routed) return MOE_ERR_INVALID_ARG;
    if (s.n_routed > 256 || s.top_k > 32) return MOE_ERR_UNSUPPORTED;
    const int S = s.top_k + (s.shared_id >= 0 ? 1 : 0);
    const int E = s.n_routed + (s.shared_id >= 0 ? 1 : 0);
    const int R = s.T * S;

    // scratch layout: [status word][tile prefix, E+1 ints][chunk histograms]
    const size_t off_tile = round256(sizeof(DevStatus));
    const size_t off_hist = off_tile + round256(static_cast<size_t>(E + 1) * sizeof(int32_t));
    const size_t need = off_hist + permute_scratch_ints(R, E) * sizeof(int32_t);
    if (need > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;   // too many tokens for the fixed array

    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
    char* b = static_cast<char*>(base);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(b, 0, sizeof(DevStatus), st) != cudaSuccess) return MOE_ERR_CUDA;
    const cudaError_t e = launch_permute(R, E, ids, counts, offsets, perm, inv,
                                         reinterpret_cast<int32_t*>(b + off_tile),
                                         reinterpret_cast<int32_t*>(b + off_hist),
                                         reinterpret_cast<DevStatus*>(b), st);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
