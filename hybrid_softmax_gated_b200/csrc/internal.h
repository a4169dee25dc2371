// Internal declarations shared by the host library and the kernel files of
// libarl2.so.  Nothing here is part of the C ABI (see include/arl2.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>

namespace arl2 {

// Problem dimensions of one handle: B streams, H heads, head width d,
// L tokens per frame.  Token tensors are [B][L][H][d].
struct Dims {
    int B, H, d, L;
};

// Error word bits set by kernels whose bounded waits ran out.
enum : int {
    kErrTimeoutAttn = 1 << 0,
    kErrTimeoutUpdate = 1 << 1,
    kErrTimeoutTokenLevel = 1 << 2,
};

// ---- failure path self-test (simt.cu) -------------------------------------
// One thread waits for *flag to become nonzero with the same bounded spin
// the kernels' inter-CTA waits use; after limit_ns it sets kErrTimeoutAttn
// in *err and returns.
cudaError_t launch_selftest_wait(const int* flag, unsigned long long limit_ns, int* err, cudaStream_t st);

// ---- SIMT kernels (fp32 arithmetic; T = float or __nv_bfloat16) ----------

// One-time kernel attribute setup (dynamic shared memory limits); called by
// arl2_create so that no launch path changes attributes (graph capture).
cudaError_t simt_init();

// out = x W[h] per head, optionally with L2-normalised rows.  Exactly one of
// out_f (fp32) and out_t (element type of x) is non-null.
cudaError_t launch_phi_simt(bool bf16, const void* x, const void* w, bool l2norm,
                            float* out_f, void* out_t, Dims dm, cudaStream_t st);

// out = softmax(Q K^T scale) V + qp S   (qp = Q W_q, fp32 [B][L][H][d])
cudaError_t launch_attn_simt(bool bf16, const void* q, const void* k, const void* v,
                             const float* qp, const float* S, void* out, float scale,
                             Dims dm, cudaStream_t st);

// The same attention with Lc leading keys from a KV cache kc, vc
// ([B][cap][H][d], element type of q); S == nullptr: no inter term (the
// softmax teacher layer), qp unused then.
cudaError_t launch_attn_simt_cached(bool bf16, const void* q, const void* k, const void* v,
                                    const void* kc, const void* vc, int Lc, long long cap,
                                    const float* qp, const float* S, void* out, float scale, Dims dm,
                                    cudaStream_t st);

// Copy a frame's k and v ([B][L][H][d], esz bytes per element) into frames
// [slot, slot + 1) of the caches kc, vc ([B][cap_frames * L][H][d]).
cudaError_t launch_kv_append(const void* k, const void* v, void* kc, void* vc, size_t esz, int slot,
                             int cap_frames, Dims dm, cudaStream_t st);

// r = vp - kp S, written over vp (fp32 [B][L][H][d]); S is the pre-update state.
cudaError_t launch_residual_simt(const float* kp, float* vp_to_r, const float* S, Dims dm,
                                 cudaStream_t st);

// S = alpha S + kp^T diag(beta) r, in place.
cudaError_t launch_accum_simt(const float* kp, const float* r, const float* alpha, int alpha_per_key,
                              const float* beta, float* S, Dims dm, cudaStream_t st);

// Copies of the state derived from S alone, used by the tensor-core kernels:
// Mt[b][h][n][a] = bf16(sum_c Wq[h][a][c] S[b][h][c][n])   ((W_q S)^T)
// Sb[b][h][c][n] = bf16(S[b][h][c][n])
cudaError_t launch_fold_state(const void* wq_bf16, const float* S, void* Mt, void* Sb, Dims dm,
                              cudaStream_t st);

// ---- token-level (sequential) access, fp32 (token_level.cu) ------------
// Chunks of the frame and the fp32 workspace of one pass.
int tl_chunks(const Dims& dm);
size_t tl_workspace_floats(const Dims& dm);
cudaError_t tl_init();  // kernel attributes, once (arl2_create)
// Adds q'_i S^(i) to out for every token (out already holds the intra-frame
// term) and, when clean, stores S^(L) in S.  qp, kp (row-normalised), vp:
// fp32 [B][L][H][d]; alpha [B][H] or [B][H][d]; beta [B][H][L].
cudaError_t launch_tl(const float* qp, const float* kp, const float* vp, const float* alpha,
                      int alpha_per_key, const float* beta, float* ws, float* S, void* out, bool bf16,
                      bool clean, Dims dm, cudaStream_t st);

}  // namespace arl2

namespace arl2 {

// ---- gate projections (gates.cu) ----------------------------------------
// alpha [B][H] and beta [B][H][L] from hidden states x [B][L][D] and the
// transposed weights wt [gate_padded_outputs(H)][D] (launch_gate_transpose
// of w [D][2H]; x, w in the layer dtype), bias fp32 [2H].  part_a: fp32
// [B][gate_tiles(L)][H] scratch; count: [B] zeroed words (left zeroed).
int gate_tiles(int L);
bool gate_shape_ok(int D, int H);
int gate_padded_outputs(int H);
cudaError_t gate_init();  // kernel attributes, once (arl2_create)
cudaError_t launch_gate_transpose(bool bf16, const void* w, void* wt, int D, int H, cudaStream_t st);
cudaError_t launch_gate_proj(bool bf16, const void* x, const void* wt, const float* bias, int B, int L, int D,
                             int H, float* beta, float* part_a, float* alpha, unsigned* count,
                             cudaStream_t st);

// The tensor-core form for bf16 (gates_tc.cu): wt as above, wt_rows rows.
struct GateTc;
int gate_tc_outputs(int H);  // padded outputs N of its products: 32, 64 or 96
// alpha-logit partials per stream that either kernel writes (part_a holds
// B * gate_part_count(L) * H floats)
int gate_part_count(int L);
GateTc* gate_tc_create(int B, int L, int D, int H, const void* wt, int wt_rows);  // nullptr: not usable
void gate_tc_destroy(GateTc* g);
cudaError_t gate_tc_launch(GateTc* g, const void* x, const float* bias, float* beta, float* part_a, float* alpha,
                           unsigned* count, int* err, cudaStream_t st);

}  // namespace arl2
