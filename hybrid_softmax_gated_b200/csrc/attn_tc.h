// Tensor-core (tcgen05) kernel for the per-pass read of the ARL2 layer:
//   out = softmax(Q K^T scale) V + Q (W_q S_{N-1})
// and, without the state read, for the softmax teacher layer whose keys and
// values run on from a KV cache into the frame's own.
// bf16 in, fp32 accumulate in TMEM, bf16 out; head_dim 128.
#pragma once

#include "internal.h"
#include "tma.h"

namespace arl2 {

struct AttnTc;

// Device workspace the kernel needs (split-tile partials and flags).
size_t attn_tc_workspace_bytes(const Dims& dm);

// Configure the kernel for the given dimensions.  workspace: device buffer
// of attn_tc_workspace_bytes(dm) bytes, its flag words zeroed (see
// attn_tc_flags).  max_ctas > 0 caps the persistent grid (else one CTA per
// SM).  Returns nullptr on failure (no tensor-map encoder, bad dims).
AttnTc* attn_tc_create(Dims dm, void* workspace, int max_ctas);
void attn_tc_destroy(AttnTc* t);

// The split-tile flag words inside the workspace (count of them in *count);
// they must be zero between launches.
int* attn_tc_flags(AttnTc* t, size_t* count);

// q, k, v, out: [B][L][H][128] bf16.  Mt: [B][H][128][128] bf16 holding
// (W_q S)^T.  err: device error word (bit kErrTimeoutAttn on a timeout).
cudaError_t attn_tc_launch(AttnTc* t, TokenMapCache& maps, const void* q, const void* k,
                           const void* v, const void* Mt, void* out, float scale, int* err,
                           cudaStream_t st);

// Plain softmax attention of the frame's queries over Lc cached keys, then
// the frame's own L keys (the softmax teacher layer with a KV cache):
//   out = softmax([Q Kc^T, Q K^T] scale) [Vc; V]
// kc, vc: maps of the cache's first Lc rows (tma_encode_token_rows); unused
// (may be null) when Lc = 0.
cudaError_t attn_tc_launch_cached(AttnTc* t, TokenMapCache& maps, const void* q, const void* k,
                                  const void* v, const CUtensorMap* kc, const CUtensorMap* vc, int Lc,
                                  void* out, float scale, int* err, cudaStream_t st);

}  // namespace arl2
