// Tensor-core (tcgen05) clean-pass state update of the ARL2 layer, bf16
// operands, fp32 accumulation and fp32 master state; head_dim 128.
//
//   K' = rownorm(K W_k), V' = V W_v
//   dS = K'^T diag(beta) (V' - K' S_{N-1})        (per 128-token chunk)
//   S_N = alpha S_{N-1} + sum_chunks dS
//   then Mt = (W_q S_N)^T and S_N in bf16 (the fold kernel)
#pragma once

#include "internal.h"
#include "tma.h"

namespace arl2 {

struct UpdateTc;

// Buffers owned by the handle that the update reads and writes.
struct UpdateBuffers {
    const void* w_all;  // bf16 [3][H][128][128]: W_q, W_k, W_v
    float* S;           // fp32 [B][H][128][128] master state, row = key feature
    void* Sb;           // bf16 copy of S (read by the next update)
    void* Mt;           // bf16 (W_q S)^T (read by the attention kernel)
    float* part_s;      // fp32 [B][H][chunks] blocks of 128 x 128, in column quads
};

int update_tc_chunks(const Dims& dm);
UpdateTc* update_tc_create(const Dims& dm, const UpdateBuffers& buf);
void update_tc_destroy(UpdateTc* u);

// Enqueue the update for one clean pass (three kernels: chunk, finalize,
// fold).  k, v: token
// tensors of the pass; alpha [B][H], beta [B][H][L] fp32.
cudaError_t update_tc_launch(UpdateTc* u, TokenMapCache& maps, const void* k, const void* v,
                             const float* alpha, int alpha_per_key, const float* beta, int* err,
                             cudaStream_t st);

}  // namespace arl2
