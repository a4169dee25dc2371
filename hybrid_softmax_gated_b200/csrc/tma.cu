// Host-side TMA tensor-map encoding (see tma.h).
#include "tma.h"

#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <new>

namespace arl2 {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_once;

void resolve() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess && fn)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
        cudaGetLastError();
}

bool encode4(CUtensorMap* m, const void* p, const cuuint64_t dims[4], const cuuint64_t strides[3],
             const cuuint32_t box[4]) {
    if (!tma_available()) return false;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace

bool tma_available() {
    std::call_once(g_once, resolve);
    return g_encode != nullptr;
}

bool tma_encode_tokens(CUtensorMap* m, const void* p, const Dims& dm) {
    const cuuint64_t dims[4] = {128, (cuuint64_t)dm.H, (cuuint64_t)dm.L, (cuuint64_t)dm.B};
    const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)dm.H * 128 * 2,
                                   (cuuint64_t)dm.L * dm.H * 128 * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    return encode4(m, p, dims, strides, box);
}

bool tma_encode_token_rows(CUtensorMap* m, const void* p, int B, int H, int rows, long long capacity) {
    if (rows < 1 || rows > capacity) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)H * 128 * 2, (cuuint64_t)capacity * H * 128 * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    return encode4(m, p, dims, strides, box);
}

bool tma_encode_rows_2d(CUtensorMap* m, const void* p, long long inner, long long rows, long long outer,
                        int box_rows) {
    if (inner < 64 || (inner * 2) % 16 != 0 || rows < 1 || outer < 1 || box_rows < 1 || box_rows > 256)
        return false;
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)outer, 1};
    const cuuint64_t strides[3] = {(cuuint64_t)inner * 2, (cuuint64_t)(inner * 2 * rows),
                                   (cuuint64_t)(inner * 2 * rows * outer)};
    const cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    return encode4(m, p, dims, strides, box);
}

bool tma_encode_tiles(CUtensorMap* m, const void* p, int outer) {
    const cuuint64_t dims[4] = {128, 128, (cuuint64_t)outer, 1};
    const cuuint64_t strides[3] = {128 * 2, 128 * 128 * 2, (cuuint64_t)outer * 128 * 128 * 2};
    const cuuint32_t box[4] = {64, 128, 1, 1};
    return encode4(m, p, dims, strides, box);
}

TokenMapCache::TokenMapCache(const Dims& dm) : dm_(dm), entries_(new (std::nothrow) Entry[kSlots]) {
    if (entries_)
        for (int i = 0; i < kSlots; ++i) entries_[i].p = nullptr;
}

TokenMapCache::~TokenMapCache() { delete[] entries_; }

bool TokenMapCache::get(const void* p, CUtensorMap* out) {
    Entry& e = entries_[(reinterpret_cast<uintptr_t>(p) >> 8) % kSlots];
    if (e.p != p) {
        if (!tma_encode_tokens(&e.m, p, dm_)) {
            e.p = nullptr;
            return false;
        }
        e.p = p;
    }
    *out = e.m;
    return true;
}

}  // namespace arl2
