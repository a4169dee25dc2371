// Clean-pass state update that allocates nothing: arl2_state_update_noalloc.
//
// Some callers cannot allocate device memory at the point where they run
// the update: a plugin inside a host framework that only hands out its own
// fixed buffers, or a process whose caching allocator has reserved the
// device memory up front so that a cudaMalloc would fail or fragment it.
// For them this entry point runs the same SIMT kernels as the handle's
// clean-pass update, but on a state buffer the caller owns and with its two
// fp32 scratch arrays (k' and v', then r = v' - k' S) taken from a
// file-scope device array instead of a handle.
//
// The array is a static __device__ object: every GPU that loads this
// library holds it (2 x ARL2_NOALLOC_MAX_ELEMENTS floats, 32 MiB) until the
// process exits.  Host code cannot use its name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress
// (with that device current) and caches it; that first call also sets the
// kernels' shared-memory limits.  Both are kept for the life of the process:
// after a cudaDeviceReset the cached address and attributes are stale, so
// the call must not be used across one.  Every call shares the array and
// leaves its contents behind; calls whose work overlaps on the GPU race on
// it.
#include "arl2.h"
#include "internal.h"

#include <cstdint>
#include <mutex>

namespace {

constexpr size_t kMaxElems = ARL2_NOALLOC_MAX_ELEMENTS;
constexpr int kMaxDevices = 64;
// The same caps as arl2_create: heads and batch are grid dimensions of the
// SIMT kernels (at most 65535 each).
constexpr int kMaxHeads = 1024;
constexpr int kMaxBatch = 65535;

// [0, kMaxElems): k' (fp32); [kMaxElems, 2 kMaxElems): v', then r.
static __device__ __align__(256) float g_update_scratch[2 * kMaxElems];

std::mutex g_setup_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_update_scratch on the current device (set up once).
arl2_status scratch_for_current_device(float** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ARL2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ARL2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_update_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return ARL2_ERR_CUDA;
        }
        if (arl2::simt_init() != cudaSuccess) {
            cudaGetLastError();
            return ARL2_ERR_CUDA;
        }
        g_scratch_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_ptr[dev];
    return ARL2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" arl2_status arl2_state_update_noalloc(int batch, int heads, int head_dim, int tokens,
                                                 arl2_dtype dtype, const void* k, const void* v,
                                                 const void* w_k, const void* w_v,
                                                 const float* alpha, const float* beta,
                                                 float* state, cudaStream_t stream) {
    if (!k || !v || !w_k || !w_v || !alpha || !beta || !state) return ARL2_ERR_INVALID_ARG;
    if (dtype != ARL2_BF16 && dtype != ARL2_FP32) return ARL2_ERR_INVALID_ARG;
    if (batch < 1 || batch > kMaxBatch || heads < 1 || heads > kMaxHeads || tokens < 1 || head_dim < 1 ||
        head_dim > 128)
        return ARL2_ERR_SHAPE;
    const size_t elems = (size_t)batch * (size_t)tokens * (size_t)heads * (size_t)head_dim;
    if (elems > kMaxElems) return ARL2_ERR_SHAPE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(w_k) || !aligned16(w_v) || !aligned16(state))
        return ARL2_ERR_ALIGN;
    float* scratch = nullptr;
    arl2_status s = scratch_for_current_device(&scratch);
    if (s != ARL2_OK) return s;
    float* kp = scratch;
    float* vr = scratch + kMaxElems;
    const arl2::Dims dm{batch, heads, head_dim, tokens};
    const bool bf16 = dtype == ARL2_BF16;
    // Every element of kp and vr that a later kernel reads is written first by
    // the phi kernels of this same call, so nothing needs clearing.
    if (arl2::launch_phi_simt(bf16, k, w_k, true, kp, nullptr, dm, stream) != cudaSuccess ||
        arl2::launch_phi_simt(bf16, v, w_v, false, vr, nullptr, dm, stream) != cudaSuccess ||
        arl2::launch_residual_simt(kp, vr, state, dm, stream) != cudaSuccess ||
        arl2::launch_accum_simt(kp, vr, alpha, 0, beta, state, dm, stream) != cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}
