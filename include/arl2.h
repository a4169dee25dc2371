/*
 * arl2.h — C ABI of the ARL2 hybrid attention layer for NVIDIA B200 (sm_100a).
 *
 * The layer ("Attend Locally, Remember Linearly", technical summary §2.1
 * Hybrid Attention Decomposition and §2.2 Memory State Management) runs once
 * per latent frame and denoising pass.  For every stream b and head h:
 *
 *   O = softmax(Q K^T * scale) V  +  (Q W_q[h]) S_{N-1}[b,h]
 *
 * the first term being the intra-frame bidirectional softmax branch over the
 * frame's L tokens (§2.1 item 1) and the second the inter-frame read of the
 * fixed-size state through the per-head feature map phi_q (§2.1 "Adaptation",
 * "Output"), every token reading the same pre-update state (§2.2 "Frame-Level
 * Access").  On the clean pass only (§2.2 "Clean-Pass Updates"), after the
 * read, the state is updated once for the frame (§2.1 "State Update"):
 *
 *   K' = rownorm(K W_k[h]),  V' = V W_v[h]
 *   S_N = alpha S_{N-1} + K'^T diag(beta) (V' - K' S_{N-1})
 *
 * Conventions used by every entry point:
 *   - Token tensors (q, k, v, out, x) are [B][L][H][d], dense, in the
 *     handle's dtype, device memory, 16-byte aligned.
 *   - Feature maps W are [H][d][d] with row = input feature (x' = x W).
 *   - The state S is fp32 [B][H][d][d], row = key feature, column = value
 *     feature.  It is owned by the handle.
 *   - alpha is fp32 [B][H] (one forget gate per stream and head for the
 *     frame; headwise gating, the form the pages adopt), or, for a handle
 *     created with gating = ARL2_GATE_ELEMENTWISE, fp32 [B][H][d] (one gate
 *     per key feature: S_N = diag(alpha) S_{N-1} + ..., the variant the
 *     atlas summary's "Surprising findings" compares).  beta is fp32
 *     [B][H][L] (one rate per token).
 *   - Every call is asynchronous and stream-ordered on the given stream: it
 *     makes no host synchronisation and allocates nothing after
 *     arl2_create.  A call that returns anything but ARL2_OK enqueued
 *     nothing, except ARL2_ERR_CUDA, which reports a failed launch or copy.
 *   - The caller keeps ownership of every pointer it passes; the handle owns
 *     the state, its derived copies, the weight copies and all workspaces.
 *   - The caller's current CUDA device must be the handle's device.
 *   - A handle is not thread-safe: calls on one handle must be serialised
 *     by the caller, and calls enqueued on different streams must not
 *     overlap on the GPU.
 */
#ifndef ARL2_H
#define ARL2_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ARL2_OK = 0,
    ARL2_ERR_INVALID_ARG = -1,  /* null pointer, bad flag, wrong device     */
    ARL2_ERR_SHAPE = -2,        /* a dimension out of the supported range   */
    ARL2_ERR_ALIGN = -3,        /* a tensor pointer not 16-byte aligned     */
    ARL2_ERR_CUDA = -4,         /* a CUDA runtime or driver call failed     */
    ARL2_ERR_OOM = -5,          /* device allocation failed in arl2_create  */
    ARL2_ERR_TIMEOUT = -6,      /* a kernel's bounded wait ran out          */
    ARL2_ERR_UNSUPPORTED = -7   /* valid, but not built for this dtype/size */
} arl2_status;

typedef enum { ARL2_BF16 = 0, ARL2_FP32 = 1 } arl2_dtype;

/* Kernel family.  AUTO picks the tensor-core (tcgen05) kernels for bf16 with
 * head_dim 128 and the fp32 SIMT kernels for fp32.  SIMT forces the SIMT
 * kernels (fp32 arithmetic) for either dtype; it exists to cross-check the
 * tensor-core kernels on the GPU and is not a fallback: AUTO never falls
 * back to it. */
typedef enum { ARL2_IMPL_AUTO = 0, ARL2_IMPL_SIMT = 1 } arl2_impl;

/* Granularity of the forget gate alpha (see the conventions above). */
typedef enum { ARL2_GATE_HEADWISE = 0, ARL2_GATE_ELEMENTWISE = 1 } arl2_gating;

/* How the frame's tokens reach the state.  FRAME (the method, technical
 * summary §2.2 "Frame-Level Access"): every token reads S_{N-1} and the
 * clean pass updates once.  TOKEN (the ablation the pages compare with it):
 * token i reads the state left by tokens 0..i-1 of the pass and then updates
 * it with the delta rule, S <- G_i S + beta_i k'_i^T (v'_i - k'_i S), the
 * forget gate acting once with token 0 (G_0 = alpha, G_i = 1); every pass
 * reads through its own sequential states, so alpha and beta are required on
 * every pass, and only the clean pass keeps the final state.  With bf16 and
 * d = 128 TOKEN runs on tensor-core kernels (a per-chunk preparation, then a
 * scan over 128-token chunks with the fp32 state in TMEM and bf16 chunk
 * operands); otherwise on fp32 SIMT kernels (bf16 inputs are widened).  With
 * bf16 its output is rounded twice (the intra-frame term, then the sum). */
typedef enum { ARL2_ACCESS_FRAME = 0, ARL2_ACCESS_TOKEN = 1 } arl2_access;

typedef struct arl2_handle arl2_handle;

typedef struct {
    int batch;             /* B >= 1: independent streams                     */
    int heads;             /* H >= 1                                          */
    int head_dim;          /* d: 128 for bf16 tensor-core kernels; 1..128 SIMT */
    int tokens_per_frame;  /* L >= 1                                          */
    arl2_dtype dtype;      /* dtype of q, k, v, out and the feature maps      */
    const void* w_q;       /* device [H][d][d], dtype; copied at create       */
    const void* w_k;
    const void* w_v;
    float softmax_scale;   /* 0 selects 1/sqrt(d)                             */
    int host_staging;      /* 0: none; 1: device staging buffers for the
                              host-buffer calls (arl2_frame_forward_host,
                              arl2_frame_forward_hidden_host), copies on the
                              caller's stream; 2: two sets of them, and the
                              copies run on the handle's own streams so that
                              one call's input copies overlap the previous
                              call's pass and output copy (see
                              arl2_frame_forward_host); other nonzero values
                              act as 1                                        */
    arl2_impl impl;
    int max_ctas;          /* 0: the tensor-core attention kernel may use every
                              SM; > 0 caps its persistent grid (co-scheduling
                              with other work, tests of the split schedule)   */
    arl2_gating gating;    /* HEADWISE: alpha [B][H]; ELEMENTWISE: [B][H][d]  */
    arl2_access access;    /* FRAME (the method) or TOKEN (the ablation)      */
    /* Optional gate projections (see arl2_frame_forward_hidden).  NULL w_gate:
     * none, and hidden_dim, b_gate are ignored. */
    int hidden_dim;        /* D: width of the hidden states; a multiple of 8;
                              needs 2 H <= 96                                 */
    const void* w_gate;    /* device [D][2H] in dtype, 16-byte aligned; column
                              h gives head h's alpha logit, column H + h its
                              beta logit; copied at create                    */
    const float* b_gate;   /* device fp32 [2H], 16-byte aligned; copied       */
} arl2_config;

/* Create a layer on the current device.  Validates cfg, allocates the zeroed
 * state S_0 = 0 and every workspace, and copies the three feature maps
 * (stream-ordered on `stream`).  On success *out receives the handle.
 * Errors: INVALID_ARG (null cfg/out/weights, w_gate without b_gate), SHAPE
 * (also hidden_dim with w_gate), ALIGN (weights), UNSUPPORTED (dtype/head_dim
 * the chosen kernels do not handle; gate projections with elementwise
 * gating), OOM, CUDA. */
arl2_status arl2_create(const arl2_config* cfg, cudaStream_t stream, arl2_handle** out);

/* One denoising pass of one latent frame (technical summary §2.1, §2.2).
 * Writes out = O_intra + O_inter for every token, reading S_{N-1}.  When
 * clean_pass is nonzero, then also updates the state in place to S_N; alpha
 * and beta are read only in that case and may be NULL otherwise (with
 * access = ARL2_ACCESS_TOKEN they are read on every pass, see above).
 * q, k, v, out: device [B][L][H][d] dtype, 16-byte aligned; out must not
 * alias q, k or v.  alpha: device fp32 [B][H] ([B][H][d] with elementwise
 * gating); beta: device fp32 [B][H][L]. */
arl2_status arl2_frame_forward(arl2_handle* h, const void* q, const void* k, const void* v,
                               const float* alpha, const float* beta, int clean_pass,
                               void* out, cudaStream_t stream);

/* arl2_frame_forward on HOST buffers: copies q, k, v (and alpha, beta on a
 * clean pass) from host memory into the handle's device staging buffers,
 * runs the pass, and copies out back to host memory.  The call is complete
 * when `stream` reaches its end; host buffers should be pinned for the
 * copies to be asynchronous, and the caller must not touch them until then.
 * host_staging = 1: every copy is ordered on `stream`.  host_staging = 2:
 * consecutive calls alternate between two staging sets; the input copies
 * run on the handle's copy-in stream (once the pass that last used the set
 * is done) and may start before earlier work on `stream` has finished, so
 * the host inputs must hold their values when the call is made; the pass
 * runs on `stream` after them; the output copy runs on the copy-out stream
 * and `stream` waits for it.  Needs a handle created with host_staging != 0
 * (INVALID_ARG otherwise). */
arl2_status arl2_frame_forward_host(arl2_handle* h, const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, int clean_pass,
                                    void* out, cudaStream_t stream);

/* Gate projections (technical summary §2.1 "State Update": alpha and beta
 * are learned per-token projections; the pages give no form, and this is
 * the reading the library takes).  For hidden states x (device [B][L][D] in
 * dtype, 16-byte aligned; the input of the layer's QKV projection):
 *   a_ih = x_i . w_gate[:, h] + b_gate[h],  g_ih = x_i . w_gate[:, H+h] + b_gate[H+h]
 *   beta[b][h][i] = sigmoid(g_ih)
 *   alpha[b][h]   = sigmoid((1/L) sum_i a_ih)   (one forget gate per frame)
 * Writes alpha (device fp32 [B][H]) and beta (device fp32 [B][H][L]).
 * Needs a handle created with w_gate (INVALID_ARG otherwise); fp32
 * accumulation; one kernel. */
arl2_status arl2_gates_apply(arl2_handle* h, const void* x, float* alpha, float* beta, cudaStream_t stream);

/* arl2_frame_forward with the gates projected from the hidden states x
 * (arl2_gates_apply into the handle's own buffers) on the passes that read
 * them: the clean pass (and, with token-level access, every pass).  x may be
 * NULL on other passes.  Needs a handle created with w_gate. */
arl2_status arl2_frame_forward_hidden(arl2_handle* h, const void* q, const void* k, const void* v,
                                      const void* x, int clean_pass, void* out, cudaStream_t stream);

/* arl2_frame_forward_hidden on HOST buffers (q, k, v, out [B][L][H][d] and x
 * [B][L][D], pinned for asynchronous copies), stream-ordered like
 * arl2_frame_forward_host.  Needs host_staging and w_gate at create. */
arl2_status arl2_frame_forward_hidden_host(arl2_handle* h, const void* q, const void* k, const void* v,
                                           const void* x, int clean_pass, void* out, cudaStream_t stream);

/* S := 0 for every stream and head (the start of a new video stream). */
arl2_status arl2_state_reset(arl2_handle* h, cudaStream_t stream);

/* Copy the fp32 state [B][H][d][d] to device memory dst (checkpoint, parity). */
arl2_status arl2_state_get(arl2_handle* h, float* dst_device, cudaStream_t stream);

/* Replace the state by the fp32 [B][H][d][d] device buffer src (resume). */
arl2_status arl2_state_set(arl2_handle* h, const float* src_device, cudaStream_t stream);

/* Apply one of the handle's per-head feature maps to a token tensor:
 * which = 0: out = x W_q;  1: out = rownorm(x W_k);  2: out = x W_v
 * (technical summary §2.1 "Adaptation").  x, out: device [B][L][H][d] in
 * the handle's dtype.  This is the stand-alone form of the projection the
 * forward pass fuses; it exists for step-level checks. */
arl2_status arl2_phi_apply(arl2_handle* h, int which, const void* x, void* out,
                           cudaStream_t stream);

/* Synchronise `stream`, then read and clear the handle's device error word.
 * Returns ARL2_ERR_TIMEOUT if a kernel gave up a bounded wait since the last
 * check (its outputs are then undefined), ARL2_ERR_CUDA on a CUDA error,
 * else ARL2_OK.  This is the one call that blocks the host. */
arl2_status arl2_device_status(arl2_handle* h, cudaStream_t stream);

/* Self-test of the failure path: one thread waits, with the bounded spin
 * the kernels' inter-CTA waits use, for a device word that nothing ever
 * sets; after limit_us (1 .. 1,000,000) it gives up, sets the handle's error
 * word and returns.  arl2_device_status then reports ARL2_ERR_TIMEOUT and
 * clears it; the context stays usable.  No fault, trap or unbounded wait. */
arl2_status arl2_selftest_wait_timeout(arl2_handle* h, unsigned limit_us, cudaStream_t stream);

/* Device bytes the handle holds (state, copies, weights, workspaces). */
size_t arl2_device_bytes(const arl2_handle* h);

/* Number of kernels this handle has enqueued (or recorded into a CUDA graph
 * capture) since creation; memsets and copies are not counted.  0 for NULL. */
unsigned long long arl2_kernel_launches(const arl2_handle* h);

/* Largest batch * tokens * heads * head_dim that arl2_state_update_noalloc
 * accepts: 4,194,304 elements (a 1560-token, 12-head, 128-wide frame of one
 * stream is 2,396,160). */
#define ARL2_NOALLOC_MAX_ELEMENTS (1u << 22)

/* The clean-pass state update, for callers that cannot allocate device
 * memory.  The ARL2 pages have no counterpart to this call: it exists for
 * deployment.  Some callers cannot call cudaMalloc where they run this step
 * (a plugin that only gets fixed buffers from its host framework, or a
 * process whose caching allocator has already reserved the device memory),
 * and arl2_create allocates.  This call allocates nothing: the caller owns
 * the state, and the two fp32 scratch arrays the update needs live in a
 * static device array inside the library (2 x ARL2_NOALLOC_MAX_ELEMENTS
 * floats = 32 MiB, held on every GPU that loads the library until exit).
 *
 * Computes, in place on `state` (fp32 [B][H][d][d], row = key feature):
 *   S = alpha S + K'^T diag(beta) (V' - K' S),  K' = rownorm(K W_k), V' = V W_v
 * k, v: device [B][L][H][d] in dtype; w_k, w_v: device [H][d][d] in dtype;
 * alpha: device fp32 [B][H]; beta: device fp32 [B][H][L].  All pointers
 * 16-byte aligned.  Uses the fp32 SIMT kernels for either dtype.
 *
 * The first call on each device looks up the scratch array's device address
 * (cudaGetSymbolAddress, with that device current) and sets kernel
 * attributes; make that first call before any stream capture.  That set-up
 * is cached for the life of the process, so do not use this call across a
 * cudaDeviceReset (the cached address and attributes would be stale).  Every
 * call shares the one scratch array and leaves its contents behind, so calls
 * whose work overlaps on the GPU (other streams, other threads) race: keep
 * them ordered.  Errors: INVALID_ARG (null pointer, bad dtype), SHAPE (a
 * dimension out of range: batch above 65535, heads above 1024, head_dim
 * above 128, or B*L*H*d > ARL2_NOALLOC_MAX_ELEMENTS), ALIGN, CUDA; nothing
 * is enqueued on an error other than CUDA. */
arl2_status arl2_state_update_noalloc(int batch, int heads, int head_dim, int tokens,
                                      arl2_dtype dtype, const void* k, const void* v,
                                      const void* w_k, const void* w_v, const float* alpha,
                                      const float* beta, float* state, cudaStream_t stream);

/* Release everything the handle owns.  Synchronises the device first.
 * NULL is ignored. */
void arl2_destroy(arl2_handle* h);

/* ------------------------------------------------------------------------
 * Softmax teacher layer with a KV cache.
 *
 * The attention the hybrid layer replaces, kept by the layers of a stack
 * that stay softmax: technical summary §1 ("KV Cache Growth": the cache of
 * keys and values grows with every generated frame) and §4 ("Efficiency":
 * the speedup of the hybrid stack grows with video length as that cache
 * comes to dominate).  The pages fix the cache's role, not its arithmetic;
 * this layer reads it as chunk-causal attention at frame granularity.  For
 * one pass of frame N (N = arl2_kv_frames before the call):
 *   O = softmax([Q Kc^T, Q K^T] * scale) [Vc; V]
 * where (Kc, Vc) hold the keys and values of the clean passes of frames
 * 0..N-1 in frame order, and (K, V) are this pass's own, attended
 * bidirectionally.  A clean pass then appends its k and v to the cache (the
 * same passes that update the hybrid layer's state, §2.2 "Clean-Pass
 * Updates"); other passes leave the cache alone.
 *
 * The cache holds max_frames frames and is allocated by arl2_kv_create; no
 * later call allocates.  Device memory held: 2 B max_frames L H d elements
 * of dtype plus workspaces; the part in use grows by 2 B L H d elements per
 * frame (arl2_kv_cache_bytes). */
typedef struct arl2_kv_handle arl2_kv_handle;

typedef struct {
    int batch;             /* B >= 1                                          */
    int heads;             /* H >= 1                                          */
    int head_dim;          /* d: 128 for the bf16 tensor-core kernel; 1..128 SIMT */
    int tokens_per_frame;  /* L >= 1                                          */
    int max_frames;        /* cache capacity in frames, >= 1; max_frames * L
                              <= 2^26                                         */
    arl2_dtype dtype;      /* dtype of q, k, v, out and the cache             */
    float softmax_scale;   /* 0 selects 1/sqrt(d)                             */
    int host_staging;      /* nonzero: staging buffers for
                              arl2_kv_frame_forward_host                      */
    arl2_impl impl;
    int max_ctas;          /* as in arl2_config                               */
} arl2_kv_config;

/* Create a teacher layer with an empty cache on the current device.
 * Errors: INVALID_ARG, SHAPE, UNSUPPORTED (dtype/head_dim), OOM, CUDA. */
arl2_status arl2_kv_create(const arl2_kv_config* cfg, cudaStream_t stream, arl2_kv_handle** out);

/* One pass of one frame: out = the attention above over the cached frames
 * and this pass's k, v; with clean_pass nonzero, then appends k and v to the
 * cache.  q, k, v, out: device [B][L][H][d] dtype, 16-byte aligned; out must
 * not alias q, k or v.  SHAPE (nothing enqueued) for a clean pass when the
 * cache already holds max_frames frames.  The frame count lives on the host:
 * a call recorded into a CUDA graph keeps the cache length it saw. */
arl2_status arl2_kv_frame_forward(arl2_kv_handle* h, const void* q, const void* k, const void* v,
                                  int clean_pass, void* out, cudaStream_t stream);

/* arl2_kv_frame_forward on HOST buffers (pinned for asynchronous copies):
 * q, k, v are copied into the handle's staging buffers, and out back, all
 * stream-ordered.  Needs host_staging != 0 (INVALID_ARG otherwise). */
arl2_status arl2_kv_frame_forward_host(arl2_kv_handle* h, const void* q, const void* k, const void* v,
                                       int clean_pass, void* out, cudaStream_t stream);

/* Empty the cache (the start of a new video stream).  Host-side only. */
arl2_status arl2_kv_reset(arl2_kv_handle* h);

/* Frames in the cache; -1 for NULL. */
int arl2_kv_frames(const arl2_kv_handle* h);

/* Copy the cached keys and values to device buffers k_dst, v_dst, each
 * [B][frames * L][H][d] dtype (dense).  Nothing is copied while empty. */
arl2_status arl2_kv_cache_get(arl2_kv_handle* h, void* k_dst, void* v_dst, cudaStream_t stream);

/* Replace the cache by `frames` frames from device buffers k_src, v_src,
 * each [B][frames * L][H][d] dtype (dense): resume from a checkpoint taken
 * with arl2_kv_cache_get.  frames = 0 empties the cache.  Errors:
 * INVALID_ARG, SHAPE (frames > max_frames), CUDA. */
arl2_status arl2_kv_cache_set(arl2_kv_handle* h, const void* k_src, const void* v_src, int frames,
                              cudaStream_t stream);

/* As arl2_device_status, for the teacher layer's kernels. */
arl2_status arl2_kv_device_status(arl2_kv_handle* h, cudaStream_t stream);

/* Device bytes the handle holds (the whole cache capacity included). */
size_t arl2_kv_device_bytes(const arl2_kv_handle* h);

/* Bytes of the cache in use: 2 B frames L H d elements of dtype. */
size_t arl2_kv_cache_bytes(const arl2_kv_handle* h);

/* Kernels this handle has enqueued since creation. */
unsigned long long arl2_kv_kernel_launches(const arl2_kv_handle* h);

/* Release the handle (synchronises the device first); NULL is ignored. */
void arl2_kv_destroy(arl2_kv_handle* h);

/* Static string for a status code. */
const char* arl2_status_string(arl2_status s);

/* ABI version: major * 10000 + minor * 100 + patch. */
int arl2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ARL2_H */
