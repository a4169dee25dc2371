// Token-level (sequential) state access on the tensor cores: bf16 layers,
// head_dim 128 (token_level_tc.cu).  The intra-frame term is written to out
// first (the attention kernel with a zero state); this adds the token-level
// reads and, on the clean pass, stores the frame's last state in S.
#pragma once

#include "internal.h"
#include "tma.h"

namespace arl2 {

struct TlTc;

// bf16 workspace: five 128 x 128 tiles per 128-token chunk of each (stream, head).
size_t tl_tc_workspace_bytes(const Dims& dm);
// w_all: bf16 [3][H][128][128] (W_q, W_k, W_v); the workspace is the caller's.
TlTc* tl_tc_create(const Dims& dm, const void* w_all, void* workspace);
void tl_tc_destroy(TlTc* t);
// Two kernels: the per-chunk preparation (all chunks in parallel) and the
// scan (one CTA per stream and head, chunks in order).  alpha [B][H] (or
// [B][H][128] with alpha_per_key), beta [B][H][L] fp32; S fp32 [B][H][128][128].
cudaError_t tl_tc_launch(TlTc* t, TokenMapCache& maps, const void* q, const void* k, const void* v,
                         const float* alpha, int alpha_per_key, const float* beta, float* S, void* out,
                         bool clean, int* err, cudaStream_t st);

}  // namespace arl2
