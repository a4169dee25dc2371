// The softmax teacher layer with a KV cache: the C ABI of include/arl2.h
// (arl2_kv_*) and the kernel that appends a clean pass to the cache.
//
// "Attend Locally, Remember Linearly", technical summary §1 ("KV Cache
// Growth") and §4 ("Efficiency"): the layers of the stack that the hybrid
// layer does not replace keep full softmax attention over the keys and
// values of every frame generated so far.  Frame N's queries attend to the
// clean keys/values of frames 0..N-1 (the cache) and, bidirectionally, to
// their own pass's keys/values; the clean pass then appends its keys and
// values.  Memory grows by 2 B L H d elements per frame, the cost the
// hybrid layer's fixed-size state removes.
//
// The cache is one allocation of max_frames frames, made at create time, so
// no later call allocates.  Attention reads the two key runs in place (the
// first Lc = N L rows of the cache, then the pass's own k, v): no pass
// copies its keys anywhere except the clean pass's append.
//
// Kernels per call:
//   tensor-core path (bf16, d = 128): attn_tc_kernel<no state read> (1),
//                                     + kv_append_kernel on a clean pass (2)
//   SIMT path (fp32, other d):        attn_simt_kernel (1), + append (2)
#include "arl2.h"
#include "internal.h"
#include "attn_tc.h"
#include "tma.h"

#include <cmath>
#include <cstdint>
#include <new>

using arl2::Dims;

struct arl2_kv_handle {
    int device = -1;
    Dims dm{};
    arl2_dtype dtype = ARL2_BF16;
    bool use_tc = false;
    float scale = 0.f;
    size_t esz = 0;
    size_t n_tok = 0;          // B*L*H*d
    int cap_frames = 0;        // cache capacity in frames
    int frames = 0;            // frames whose clean pass is in the cache
    size_t bytes = 0;          // device bytes held
    void* kc = nullptr;        // [B][cap_frames * L][H][d] in dtype
    void* vc = nullptr;
    void* attn_ws = nullptr;   // split-tile partials and flags of the attention kernel
    arl2::TokenMapCache* maps = nullptr;
    arl2::AttnTc* tc = nullptr;
    CUtensorMap tm_kc{}, tm_vc{};  // maps of the first tm_rows cache rows
    int tm_rows = 0;
    void* stage_tok[4] = {nullptr, nullptr, nullptr, nullptr};  // q, k, v, out (host entry)
    int* err = nullptr;
    unsigned long long launches = 0;
};

namespace arl2 {
namespace {

// Grid-stride copy of one frame of k and v into cache frame `slot`, in
// units of U (the widest of 16, 8, 4, 2 bytes dividing a frame's bytes).
template <typename U>
__global__ void __launch_bounds__(256) kv_append_kernel(const U* __restrict__ k, const U* __restrict__ v,
                                                        U* __restrict__ kc, U* __restrict__ vc,
                                                        size_t frame_units, size_t batch_units,
                                                        size_t slot_units, int B) {
    const size_t per = (size_t)B * frame_units;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * per;
         i += (size_t)gridDim.x * blockDim.x) {
        const bool is_v = i >= per;
        const size_t j = is_v ? i - per : i;
        const size_t b = j / frame_units, e = j - b * frame_units;
        const size_t dst = b * batch_units + slot_units + e;
        if (is_v)
            vc[dst] = __ldcs(v + j);
        else
            kc[dst] = __ldcs(k + j);
    }
}

template <typename U>
cudaError_t append_as(const void* k, const void* v, void* kc, void* vc, size_t frame_bytes, int slot,
                      int cap_frames, int B, cudaStream_t st) {
    const size_t fu = frame_bytes / sizeof(U);
    const size_t total = 2 * (size_t)B * fu;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t want = (total + 255) / 256;
    const unsigned grid = (unsigned)(want < (size_t)sms * 8 ? want : (size_t)sms * 8);
    kv_append_kernel<U><<<grid, 256, 0, st>>>(static_cast<const U*>(k), static_cast<const U*>(v),
                                              static_cast<U*>(kc), static_cast<U*>(vc), fu,
                                              fu * (size_t)cap_frames, fu * (size_t)slot, B);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_append(const void* k, const void* v, void* kc, void* vc, size_t esz, int slot,
                             int cap_frames, Dims dm, cudaStream_t st) {
    const size_t fb = (size_t)dm.L * dm.H * dm.d * esz;  // one frame of one stream
    const uintptr_t a = reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
                        reinterpret_cast<uintptr_t>(kc) | reinterpret_cast<uintptr_t>(vc);
    if (fb % 16 == 0 && a % 16 == 0) return append_as<uint4>(k, v, kc, vc, fb, slot, cap_frames, dm.B, st);
    if (fb % 8 == 0 && a % 8 == 0) return append_as<uint2>(k, v, kc, vc, fb, slot, cap_frames, dm.B, st);
    if (fb % 4 == 0 && a % 4 == 0) return append_as<uint32_t>(k, v, kc, vc, fb, slot, cap_frames, dm.B, st);
    return append_as<uint16_t>(k, v, kc, vc, fb, slot, cap_frames, dm.B, st);
}

}  // namespace arl2

namespace {

constexpr int kMaxHeads = 1024;
constexpr int kMaxBatch = 65535;
constexpr int kMaxHeadDim = 128;
constexpr long long kMaxCacheRows = 1ll << 26;  // max_frames * tokens_per_frame

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

arl2_status check_device(const arl2_kv_handle* h) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ARL2_ERR_CUDA;
    return dev == h->device ? ARL2_OK : ARL2_ERR_INVALID_ARG;
}

template <typename T>
arl2_status dalloc(arl2_kv_handle* h, T** p, size_t bytes) {
    void* q = nullptr;
    if (cudaMalloc(&q, bytes) != cudaSuccess) {
        cudaGetLastError();
        return ARL2_ERR_OOM;
    }
    *p = static_cast<T*>(q);
    h->bytes += bytes;
    return ARL2_OK;
}

void release(arl2_kv_handle* h) {
    if (!h) return;
    if (h->tc) arl2::attn_tc_destroy(h->tc);
    delete h->maps;
    void* ptrs[] = {h->kc, h->vc, h->attn_ws, h->stage_tok[0], h->stage_tok[1], h->stage_tok[2],
                    h->stage_tok[3], h->err};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    delete h;
}

size_t cache_elems(const arl2_kv_handle* h) {
    return (size_t)h->dm.B * h->cap_frames * h->dm.L * h->dm.H * h->dm.d;
}

}  // namespace

extern "C" {

arl2_status arl2_kv_create(const arl2_kv_config* cfg, cudaStream_t stream, arl2_kv_handle** out) {
    if (!cfg || !out) return ARL2_ERR_INVALID_ARG;
    *out = nullptr;
    if (cfg->dtype != ARL2_BF16 && cfg->dtype != ARL2_FP32) return ARL2_ERR_INVALID_ARG;
    if (cfg->impl != ARL2_IMPL_AUTO && cfg->impl != ARL2_IMPL_SIMT) return ARL2_ERR_INVALID_ARG;
    if (cfg->batch < 1 || cfg->batch > kMaxBatch || cfg->heads < 1 || cfg->heads > kMaxHeads ||
        cfg->tokens_per_frame < 1 || cfg->head_dim < 1 || cfg->head_dim > kMaxHeadDim || cfg->max_frames < 1 ||
        (long long)cfg->max_frames * cfg->tokens_per_frame > kMaxCacheRows)
        return ARL2_ERR_SHAPE;
    if (!(cfg->softmax_scale >= 0.f) || std::isinf(cfg->softmax_scale)) return ARL2_ERR_INVALID_ARG;
    if (cfg->max_ctas < 0) return ARL2_ERR_INVALID_ARG;
    const bool use_tc = cfg->impl == ARL2_IMPL_AUTO && cfg->dtype == ARL2_BF16;
    if (use_tc && cfg->head_dim != 128) return ARL2_ERR_UNSUPPORTED;

    arl2_kv_handle* h = new (std::nothrow) arl2_kv_handle();
    if (!h) return ARL2_ERR_OOM;
    if (cudaGetDevice(&h->device) != cudaSuccess) {
        delete h;
        return ARL2_ERR_CUDA;
    }
    h->dm = Dims{cfg->batch, cfg->heads, cfg->head_dim, cfg->tokens_per_frame};
    h->dtype = cfg->dtype;
    h->use_tc = use_tc;
    h->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->head_dim);
    h->esz = cfg->dtype == ARL2_BF16 ? 2 : 4;
    h->cap_frames = cfg->max_frames;
    const Dims& dm = h->dm;
    h->n_tok = (size_t)dm.B * dm.L * dm.H * dm.d;

    arl2_status s = dalloc(h, &h->kc, cache_elems(h) * h->esz);
    if (s == ARL2_OK) s = dalloc(h, &h->vc, cache_elems(h) * h->esz);
    if (s == ARL2_OK) s = dalloc(h, &h->err, sizeof(int));
    if (s == ARL2_OK && use_tc) s = dalloc(h, &h->attn_ws, arl2::attn_tc_workspace_bytes(dm));
    if (s == ARL2_OK && cfg->host_staging)
        for (int i = 0; i < 4 && s == ARL2_OK; ++i) s = dalloc(h, &h->stage_tok[i], h->n_tok * h->esz);
    if (s == ARL2_OK && arl2::simt_init() != cudaSuccess) s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && use_tc) {
        h->maps = new (std::nothrow) arl2::TokenMapCache(dm);
        h->tc = arl2::attn_tc_create(dm, h->attn_ws, cfg->max_ctas);
        if (!h->maps || !h->maps->ok() || !h->tc) s = ARL2_ERR_CUDA;
    }
    if (s == ARL2_OK && cudaMemsetAsync(h->err, 0, sizeof(int), stream) != cudaSuccess) s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && use_tc &&
        cudaMemsetAsync(h->attn_ws, 0, arl2::attn_tc_workspace_bytes(dm), stream) != cudaSuccess)
        s = ARL2_ERR_CUDA;
    if (s != ARL2_OK) {
        cudaStreamSynchronize(stream);
        release(h);
        return s;
    }
    *out = h;
    return ARL2_OK;
}

arl2_status arl2_kv_frame_forward(arl2_kv_handle* h, const void* q, const void* k, const void* v,
                                  int clean_pass, void* out, cudaStream_t stream) {
    if (!h || !q || !k || !v || !out) return ARL2_ERR_INVALID_ARG;
    if (out == q || out == k || out == v) return ARL2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ARL2_ERR_ALIGN;
    if (clean_pass && h->frames >= h->cap_frames) return ARL2_ERR_SHAPE;  // the cache is full
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const Dims& dm = h->dm;
    const int Lc = h->frames * dm.L;
    const long long cap_rows = (long long)h->cap_frames * dm.L;
    ++h->launches;
    if (h->use_tc) {
        if (Lc > 0 && h->tm_rows != Lc) {
            if (!arl2::tma_encode_token_rows(&h->tm_kc, h->kc, dm.B, dm.H, Lc, cap_rows) ||
                !arl2::tma_encode_token_rows(&h->tm_vc, h->vc, dm.B, dm.H, Lc, cap_rows)) {
                h->tm_rows = 0;
                return ARL2_ERR_CUDA;
            }
            h->tm_rows = Lc;
        }
        if (arl2::attn_tc_launch_cached(h->tc, *h->maps, q, k, v, &h->tm_kc, &h->tm_vc, Lc, out, h->scale,
                                        h->err, stream) != cudaSuccess)
            return ARL2_ERR_CUDA;
    } else {
        if (arl2::launch_attn_simt_cached(h->dtype == ARL2_BF16, q, k, v, h->kc, h->vc, Lc, cap_rows, nullptr,
                                          nullptr, out, h->scale, dm, stream) != cudaSuccess)
            return ARL2_ERR_CUDA;
    }
    if (clean_pass) {
        ++h->launches;
        if (arl2::launch_kv_append(k, v, h->kc, h->vc, h->esz, h->frames, h->cap_frames, dm, stream) !=
            cudaSuccess)
            return ARL2_ERR_CUDA;
        ++h->frames;
    }
    return ARL2_OK;
}

arl2_status arl2_kv_frame_forward_host(arl2_kv_handle* h, const void* q, const void* k, const void* v,
                                       int clean_pass, void* out, cudaStream_t stream) {
    if (!h || !q || !k || !v || !out) return ARL2_ERR_INVALID_ARG;
    if (!h->stage_tok[0]) return ARL2_ERR_INVALID_ARG;
    if (clean_pass && h->frames >= h->cap_frames) return ARL2_ERR_SHAPE;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const size_t tb = h->n_tok * h->esz;
    const void* src[3] = {q, k, v};
    for (int i = 0; i < 3; ++i)
        if (cudaMemcpyAsync(h->stage_tok[i], src[i], tb, cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return ARL2_ERR_CUDA;
    s = arl2_kv_frame_forward(h, h->stage_tok[0], h->stage_tok[1], h->stage_tok[2], clean_pass,
                              h->stage_tok[3], stream);
    if (s != ARL2_OK) return s;
    if (cudaMemcpyAsync(out, h->stage_tok[3], tb, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

arl2_status arl2_kv_reset(arl2_kv_handle* h) {
    if (!h) return ARL2_ERR_INVALID_ARG;
    h->frames = 0;
    return ARL2_OK;
}

int arl2_kv_frames(const arl2_kv_handle* h) { return h ? h->frames : -1; }

arl2_status arl2_kv_cache_get(arl2_kv_handle* h, void* k_dst, void* v_dst, cudaStream_t stream) {
    if (!h || !k_dst || !v_dst) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    if (h->frames == 0) return ARL2_OK;
    const size_t frame_b = (size_t)h->dm.L * h->dm.H * h->dm.d * h->esz;
    const size_t width = frame_b * h->frames, pitch = frame_b * h->cap_frames;
    if (cudaMemcpy2DAsync(k_dst, width, h->kc, pitch, width, h->dm.B, cudaMemcpyDeviceToDevice, stream) !=
            cudaSuccess ||
        cudaMemcpy2DAsync(v_dst, width, h->vc, pitch, width, h->dm.B, cudaMemcpyDeviceToDevice, stream) !=
            cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

arl2_status arl2_kv_cache_set(arl2_kv_handle* h, const void* k_src, const void* v_src, int frames,
                              cudaStream_t stream) {
    if (!h || frames < 0 || (frames > 0 && (!k_src || !v_src))) return ARL2_ERR_INVALID_ARG;
    if (frames > h->cap_frames) return ARL2_ERR_SHAPE;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    if (frames > 0) {
        const size_t frame_b = (size_t)h->dm.L * h->dm.H * h->dm.d * h->esz;
        const size_t width = frame_b * frames, pitch = frame_b * h->cap_frames;
        if (cudaMemcpy2DAsync(h->kc, pitch, k_src, width, width, h->dm.B, cudaMemcpyDeviceToDevice, stream) !=
                cudaSuccess ||
            cudaMemcpy2DAsync(h->vc, pitch, v_src, width, width, h->dm.B, cudaMemcpyDeviceToDevice, stream) !=
                cudaSuccess)
            return ARL2_ERR_CUDA;
    }
    h->frames = frames;
    return ARL2_OK;
}

arl2_status arl2_kv_device_status(arl2_kv_handle* h, cudaStream_t stream) {
    if (!h) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    int word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ARL2_ERR_CUDA;
    if (cudaMemcpy(&word, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ARL2_ERR_CUDA;
    if (word != 0) {
        if (cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) return ARL2_ERR_CUDA;
        if (h->use_tc) {
            size_t nflags = 0;
            int* flags = arl2::attn_tc_flags(h->tc, &nflags);
            if (cudaMemset(flags, 0, nflags * sizeof(int)) != cudaSuccess) return ARL2_ERR_CUDA;
        }
        return ARL2_ERR_TIMEOUT;
    }
    return ARL2_OK;
}

size_t arl2_kv_device_bytes(const arl2_kv_handle* h) { return h ? h->bytes : 0; }

size_t arl2_kv_cache_bytes(const arl2_kv_handle* h) {
    return h ? 2 * (size_t)h->frames * h->dm.B * h->dm.L * h->dm.H * h->dm.d * h->esz : 0;
}

unsigned long long arl2_kv_kernel_launches(const arl2_kv_handle* h) { return h ? h->launches : 0; }

void arl2_kv_destroy(arl2_kv_handle* h) {
    if (!h) return;
    const int dev = h->device;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
    cudaDeviceSynchronize();
    release(h);
    if (prev >= 0 && prev != dev) cudaSetDevice(prev);
}

}  // extern "C"
