// Host-side TMA tensor-map encoding shared by the tensor-core kernels.
//
// All operand tiles are 128 rows x 128 bf16, loaded as two boxes of
// 128 rows x 64 columns (128 bytes, the 128-byte swizzle span).
#pragma once

#include <cuda.h>
#include <cstdint>

#include "internal.h"

namespace arl2 {

// Resolve cuTensorMapEncodeTiled through the runtime (no libcuda link).
bool tma_available();

// Token tensor [B][L][H][128] bf16: dims {128, H, L, B}; box {64, 1, 128, 1}.
bool tma_encode_tokens(CUtensorMap* m, const void* p, const Dims& dm);

// The first `rows` token rows of a [B][capacity][H][128] bf16 buffer (a KV
// cache): dims {128, H, rows, B}, batch stride capacity rows; rows past
// `rows` read as zeros.
bool tma_encode_token_rows(CUtensorMap* m, const void* p, int B, int H, int rows, long long capacity);

// Row-major bf16 matrices [outer][rows][inner] (inner contiguous, a
// multiple of 8 elements): dims {inner, rows, outer, 1}; box {64, box_rows,
// 1, 1}, rows past the end read as zeros.
bool tma_encode_rows_2d(CUtensorMap* m, const void* p, long long inner, long long rows, long long outer,
                        int box_rows);

// Square bf16 tiles [outer][128][128] (outer = H or B*H flattened, the
// innermost dimension contiguous): dims {128, 128, outer}; box {64, 128, 1}.
bool tma_encode_tiles(CUtensorMap* m, const void* p, int outer);

// Direct-mapped cache of token-tensor maps keyed by pointer (one per
// handle; its dimensions never change).
class TokenMapCache {
public:
    explicit TokenMapCache(const Dims& dm);
    ~TokenMapCache();
    bool ok() const { return entries_ != nullptr; }
    // Returns a copy of the map for p (false if encoding failed).
    bool get(const void* p, CUtensorMap* out);

private:
    static constexpr int kSlots = 1024;
    struct Entry {
        const void* p;
        CUtensorMap m;
    };
    Dims dm_;
    Entry* entries_;
};

}  // namespace arl2
