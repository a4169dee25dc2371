// Host side of libarl2.so: the C ABI declared in include/arl2.h.
//
// The handle owns the fp32 state S[B][H][d][d], its derived copies, one
// copy of the three feature maps, and every workspace.  All of it is
// allocated in arl2_create; no later call allocates, which keeps device
// memory flat over arbitrarily long streams (the constant-memory property
// the ARL2 pages claim for the fixed-size state, technical summary §1 and
// §4 "Memory").
//
// Kernels per call (tensor-core path, bf16, head_dim 128):
//   read-only pass : attn_tc_kernel                         (1 launch)
//   clean pass     : attn_tc_kernel, update_chunk_kernel,
//                    update_finalize_kernel, fold_state      (4 launches)
// SIMT path (fp32, or impl = ARL2_IMPL_SIMT):
//   read-only pass : phi (q'), attn_simt                     (2 launches)
//   clean pass     : + phi (k'), phi (v'), residual, accum   (6 launches)
#include "arl2.h"
#include "internal.h"
#include "attn_tc.h"
#include "tma.h"
#include "token_level_tc.h"
#include "update_tc.h"

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>

using arl2::Dims;

struct arl2_handle {
    int device = -1;
    Dims dm{};
    arl2_dtype dtype = ARL2_BF16;
    arl2_impl impl = ARL2_IMPL_AUTO;
    bool use_tc = false;      // tensor-core kernels for attention and update
    float scale = 0.f;
    size_t esz = 0;           // bytes per element of dtype
    size_t n_tok = 0;         // B*L*H*d
    size_t n_state = 0;       // B*H*d*d
    size_t bytes = 0;         // device bytes held
    void* w_all = nullptr;    // feature maps [3][H][d][d] in dtype: W_q, W_k, W_v
    void* w[3] = {nullptr, nullptr, nullptr};
    float* S = nullptr;       // fp32 master state
    // tensor-core path (both copies are functions of S alone)
    void* Mt = nullptr;       // bf16 (W_q S)^T, read by the attention kernel
    void* Sb = nullptr;       // bf16 S, read by the update kernel
    float* part_s = nullptr;  // fp32 update partials [B][H][chunks], d x d each
    void* attn_ws = nullptr;  // attention split-tile partials and flags
    arl2::TokenMapCache* maps = nullptr;
    arl2::AttnTc* tc = nullptr;
    arl2::UpdateTc* up = nullptr;
    // SIMT path
    float* qp = nullptr;      // fp32 workspaces [B][L][H][d]
    float* kp = nullptr;
    float* vp = nullptr;
    // host staging: one slot (host_staging = 1), or two whose copies run on
    // the handle's own streams (host_staging = 2, see host_pass)
    int stage_slots = 0;
    int stage_next = 0;                   // slot of the next host call
    void* stage_tok[2][4] = {};           // [slot] q, k, v, out
    float* stage_alpha[2] = {};
    float* stage_beta[2] = {};
    void* stage_x[2] = {};                // [slot] x [B][L][D] (gate projections)
    cudaStream_t copy_in = nullptr;       // two slots: input copies
    cudaStream_t copy_out = nullptr;      // two slots: output copies
    cudaEvent_t ev_in[2] = {};            // [slot] input copies done
    cudaEvent_t ev_fwd[2] = {};           // [slot] the pass that read the slot done
    cudaEvent_t ev_out[2] = {};           // [slot] output copy done
    int alpha_per_key = 0;    // elementwise gating: alpha [B][H][d] instead of [B][H]
    int token_level = 0;      // token-level (sequential) access instead of frame-level
    float* tl_ws = nullptr;   // token-level chunk workspace (SIMT path)
    void* tltc_ws = nullptr;  // token-level chunk tiles (tensor-core path)
    arl2::TlTc* tltc = nullptr;
    void* zero_read = nullptr;  // zero state for the intra-only attention launch
                                // (bf16 Mt on the tensor-core path, fp32 S on SIMT)
    // gate projections (optional): weights, and the gates they produce
    int hidden = 0;             // D, 0 without projections
    void* w_gate = nullptr;     // transposed: [gate_padded_outputs(H)][D] in dtype
    float* b_gate = nullptr;    // [2H]
    float* g_alpha = nullptr;   // [B][H]
    float* g_beta = nullptr;    // [B][H][L]
    float* g_part = nullptr;    // [B][gate_tiles(L)][H]
    unsigned* g_count = nullptr;  // [B], zero between launches
    arl2::GateTc* gtc = nullptr;  // tensor-core gate projection (bf16), else the SIMT kernel
    int* quiet = nullptr;       // a zero word nothing ever sets (the failure-path self-test)
    int* err = nullptr;       // device error word
    unsigned long long launches = 0;  // kernels enqueued by this handle
};

namespace {

constexpr int kMaxHeads = 1024;
constexpr int kMaxBatch = 65535;
constexpr int kMaxTokens = 1 << 20;
constexpr int kMaxHeadDim = 128;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

arl2_status check_device(const arl2_handle* h) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ARL2_ERR_CUDA;
    return dev == h->device ? ARL2_OK : ARL2_ERR_INVALID_ARG;
}

template <typename T>
arl2_status dalloc(arl2_handle* h, T** p, size_t bytes) {
    void* q = nullptr;
    if (cudaMalloc(&q, bytes) != cudaSuccess) {
        cudaGetLastError();
        return ARL2_ERR_OOM;
    }
    *p = static_cast<T*>(q);
    h->bytes += bytes;
    return ARL2_OK;
}

void release(arl2_handle* h) {
    if (!h) return;
    if (h->tc) arl2::attn_tc_destroy(h->tc);
    if (h->up) arl2::update_tc_destroy(h->up);
    if (h->gtc) arl2::gate_tc_destroy(h->gtc);
    if (h->tltc) arl2::tl_tc_destroy(h->tltc);
    delete h->maps;
    void* ptrs[] = {h->w_all, h->S, h->Mt, h->Sb, h->part_s, h->attn_ws, h->qp, h->kp,
                    h->vp, h->err, h->tl_ws, h->zero_read,
                    h->w_gate, h->b_gate, h->g_alpha, h->g_beta, h->g_part, h->g_count,
                    h->quiet, h->tltc_ws};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    for (int sl = 0; sl < 2; ++sl) {
        for (void* p : h->stage_tok[sl])
            if (p) cudaFree(p);
        void* more[] = {h->stage_alpha[sl], h->stage_beta[sl], h->stage_x[sl]};
        for (void* p : more)
            if (p) cudaFree(p);
        cudaEvent_t evs[] = {h->ev_in[sl], h->ev_fwd[sl], h->ev_out[sl]};
        for (cudaEvent_t e : evs)
            if (e) cudaEventDestroy(e);
    }
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
    delete h;
}

arl2_status zero_state(arl2_handle* h, cudaStream_t st) {
    if (cudaMemsetAsync(h->S, 0, h->n_state * sizeof(float), st) != cudaSuccess) return ARL2_ERR_CUDA;
    if (h->use_tc && (cudaMemsetAsync(h->Mt, 0, h->n_state * 2, st) != cudaSuccess ||
                      cudaMemsetAsync(h->Sb, 0, h->n_state * 2, st) != cudaSuccess))
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

// Recompute the tensor-core copies of the state after arl2_state_set.
arl2_status refresh_derived(arl2_handle* h, cudaStream_t st) {
    if (!h->use_tc) return ARL2_OK;
    ++h->launches;
    if (arl2::launch_fold_state(h->w[0], h->S, h->Mt, h->Sb, h->dm, st) != cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

arl2_status clean_update(arl2_handle* h, const void* k, const void* v, const float* alpha,
                         const float* beta, cudaStream_t st) {
    if (h->use_tc) {
        h->launches += 2;
        return arl2::update_tc_launch(h->up, *h->maps, k, v, alpha, h->alpha_per_key, beta, h->err, st) ==
                       cudaSuccess
                   ? ARL2_OK
                   : ARL2_ERR_CUDA;
    }
    const bool bf16 = h->dtype == ARL2_BF16;
    h->launches += 4;
    if (arl2::launch_phi_simt(bf16, k, h->w[1], true, h->kp, nullptr, h->dm, st) != cudaSuccess ||
        arl2::launch_phi_simt(bf16, v, h->w[2], false, h->vp, nullptr, h->dm, st) != cudaSuccess ||
        arl2::launch_residual_simt(h->kp, h->vp, h->S, h->dm, st) != cudaSuccess ||
        arl2::launch_accum_simt(h->kp, h->vp, alpha, h->alpha_per_key, beta, h->S, h->dm, st) != cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

struct HostCopy {
    void* dst;
    const void* src;
    size_t bytes;
};

// One pass on host buffers through staging slot `slot`: the input copies,
// then `pass` (which enqueues the pass on `stream`, writing the slot's output
// staging), then the copy of the output back to `out`.  With one slot every
// copy runs on `stream`, in order.  With two, the input copies run on the
// handle's copy-in stream once the pass that last read the slot is done,
// the pass waits for them, the output copy runs on the copy-out stream, and
// `stream` waits for that: the call is still complete when `stream` reaches
// its end, while the next call's input copies overlap this pass and its
// output copy.  They may also start before earlier work on `stream` ends, so
// the host inputs must hold their values when the call is made.
template <typename Pass>
arl2_status host_pass(arl2_handle* h, int slot, const HostCopy* in, int n_in, void* out, cudaStream_t stream,
                      Pass&& pass) {
    const bool piped = h->stage_slots == 2;
    const cudaStream_t cin = piped ? h->copy_in : stream;
    if (piped && cudaStreamWaitEvent(cin, h->ev_fwd[slot], 0) != cudaSuccess) return ARL2_ERR_CUDA;
    for (int i = 0; i < n_in; ++i)
        if (cudaMemcpyAsync(in[i].dst, in[i].src, in[i].bytes, cudaMemcpyHostToDevice, cin) != cudaSuccess)
            return ARL2_ERR_CUDA;
    // the pass waits for its inputs and for the slot's previous output copy
    // (already behind `stream` when consecutive calls share it)
    if (piped && (cudaEventRecord(h->ev_in[slot], cin) != cudaSuccess ||
                  cudaStreamWaitEvent(stream, h->ev_in[slot], 0) != cudaSuccess ||
                  cudaStreamWaitEvent(stream, h->ev_out[slot], 0) != cudaSuccess))
        return ARL2_ERR_CUDA;
    const arl2_status s = pass();
    if (s != ARL2_OK) return s;
    const cudaStream_t cout = piped ? h->copy_out : stream;
    if (piped && (cudaEventRecord(h->ev_fwd[slot], stream) != cudaSuccess ||
                  cudaStreamWaitEvent(cout, h->ev_fwd[slot], 0) != cudaSuccess))
        return ARL2_ERR_CUDA;
    if (cudaMemcpyAsync(out, h->stage_tok[slot][3], h->n_tok * h->esz, cudaMemcpyDeviceToHost, cout) !=
        cudaSuccess)
        return ARL2_ERR_CUDA;
    if (piped && (cudaEventRecord(h->ev_out[slot], cout) != cudaSuccess ||
                  cudaStreamWaitEvent(stream, h->ev_out[slot], 0) != cudaSuccess))
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

// The staging slot of the next host call.
int next_slot(arl2_handle* h) {
    const int slot = h->stage_next;
    h->stage_next = h->stage_slots == 2 ? slot ^ 1 : 0;
    return slot;
}

}  // namespace

extern "C" {

int arl2_version(void) { return 10300; }

const char* arl2_status_string(arl2_status s) {
    switch (s) {
        case ARL2_OK: return "ok";
        case ARL2_ERR_INVALID_ARG: return "invalid argument";
        case ARL2_ERR_SHAPE: return "unsupported shape";
        case ARL2_ERR_ALIGN: return "pointer not 16-byte aligned";
        case ARL2_ERR_CUDA: return "CUDA error";
        case ARL2_ERR_OOM: return "device out of memory";
        case ARL2_ERR_TIMEOUT: return "kernel wait timed out";
        case ARL2_ERR_UNSUPPORTED: return "unsupported dtype or head_dim for these kernels";
    }
    return "unknown status";
}

arl2_status arl2_create(const arl2_config* cfg, cudaStream_t stream, arl2_handle** out) {
    if (!cfg || !out) return ARL2_ERR_INVALID_ARG;
    *out = nullptr;
    if (cfg->dtype != ARL2_BF16 && cfg->dtype != ARL2_FP32) return ARL2_ERR_INVALID_ARG;
    if (cfg->impl != ARL2_IMPL_AUTO && cfg->impl != ARL2_IMPL_SIMT) return ARL2_ERR_INVALID_ARG;
    if (!cfg->w_q || !cfg->w_k || !cfg->w_v) return ARL2_ERR_INVALID_ARG;
    if (cfg->batch < 1 || cfg->batch > kMaxBatch || cfg->heads < 1 || cfg->heads > kMaxHeads ||
        cfg->tokens_per_frame < 1 || cfg->tokens_per_frame > kMaxTokens || cfg->head_dim < 1 ||
        cfg->head_dim > kMaxHeadDim)
        return ARL2_ERR_SHAPE;
    if (!(cfg->softmax_scale >= 0.f) || std::isinf(cfg->softmax_scale)) return ARL2_ERR_INVALID_ARG;
    if (cfg->max_ctas < 0) return ARL2_ERR_INVALID_ARG;
    if (cfg->gating != ARL2_GATE_HEADWISE && cfg->gating != ARL2_GATE_ELEMENTWISE)
        return ARL2_ERR_INVALID_ARG;
    if (cfg->access != ARL2_ACCESS_FRAME && cfg->access != ARL2_ACCESS_TOKEN) return ARL2_ERR_INVALID_ARG;
    if (!aligned16(cfg->w_q) || !aligned16(cfg->w_k) || !aligned16(cfg->w_v)) return ARL2_ERR_ALIGN;
    const bool use_tc = cfg->impl == ARL2_IMPL_AUTO && cfg->dtype == ARL2_BF16;
    if (use_tc && cfg->head_dim != 128) return ARL2_ERR_UNSUPPORTED;
    if (cfg->w_gate) {
        if (!cfg->b_gate) return ARL2_ERR_INVALID_ARG;
        if (!arl2::gate_shape_ok(cfg->hidden_dim, cfg->heads)) return ARL2_ERR_SHAPE;
        if (!aligned16(cfg->w_gate) || !aligned16(cfg->b_gate)) return ARL2_ERR_ALIGN;
        if (cfg->gating != ARL2_GATE_HEADWISE) return ARL2_ERR_UNSUPPORTED;  // one alpha per head
    }

    arl2_handle* h = new (std::nothrow) arl2_handle();
    if (!h) return ARL2_ERR_OOM;
    if (cudaGetDevice(&h->device) != cudaSuccess) {
        delete h;
        return ARL2_ERR_CUDA;
    }
    h->dm = Dims{cfg->batch, cfg->heads, cfg->head_dim, cfg->tokens_per_frame};
    h->dtype = cfg->dtype;
    h->impl = cfg->impl;
    h->use_tc = use_tc;
    h->alpha_per_key = cfg->gating == ARL2_GATE_ELEMENTWISE ? 1 : 0;
    h->token_level = cfg->access == ARL2_ACCESS_TOKEN ? 1 : 0;
    h->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->head_dim);
    h->esz = cfg->dtype == ARL2_BF16 ? 2 : 4;
    const Dims& dm = h->dm;
    h->n_tok = (size_t)dm.B * dm.L * dm.H * dm.d;
    h->n_state = (size_t)dm.B * dm.H * dm.d * dm.d;
    const size_t wbytes = (size_t)dm.H * dm.d * dm.d * h->esz;

    arl2_status s = dalloc(h, &h->w_all, 3 * wbytes);
    if (s == ARL2_OK) {
        for (int i = 0; i < 3; ++i) h->w[i] = static_cast<char*>(h->w_all) + i * wbytes;
        s = dalloc(h, &h->S, h->n_state * sizeof(float));
    }
    if (s == ARL2_OK) s = dalloc(h, &h->err, sizeof(int));
    if (s == ARL2_OK) s = dalloc(h, &h->quiet, sizeof(int));
    if (use_tc) {
        const size_t parts = (size_t)dm.B * dm.H * arl2::update_tc_chunks(dm) * dm.d * dm.d;
        if (s == ARL2_OK) s = dalloc(h, &h->Mt, h->n_state * 2);
        if (s == ARL2_OK) s = dalloc(h, &h->Sb, h->n_state * 2);
        if (s == ARL2_OK) s = dalloc(h, &h->part_s, parts * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->attn_ws, arl2::attn_tc_workspace_bytes(dm));
    }
    if (!use_tc) {
        if (s == ARL2_OK) s = dalloc(h, &h->qp, h->n_tok * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->kp, h->n_tok * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->vp, h->n_tok * sizeof(float));
    }
    if (h->token_level) {
        if (use_tc) {
            if (s == ARL2_OK) s = dalloc(h, &h->tltc_ws, arl2::tl_tc_workspace_bytes(dm));
        } else {
            if (s == ARL2_OK) s = dalloc(h, &h->tl_ws, arl2::tl_workspace_floats(dm) * sizeof(float));
            if (s == ARL2_OK && arl2::tl_init() != cudaSuccess) s = ARL2_ERR_CUDA;
        }
        if (s == ARL2_OK) s = dalloc(h, &h->zero_read, h->n_state * (use_tc ? 2 : sizeof(float)));
    }
    h->stage_slots = cfg->host_staging == 2 ? 2 : (cfg->host_staging ? 1 : 0);
    for (int sl = 0; sl < h->stage_slots && s == ARL2_OK; ++sl) {
        for (int i = 0; i < 4 && s == ARL2_OK; ++i) s = dalloc(h, &h->stage_tok[sl][i], h->n_tok * h->esz);
        if (s == ARL2_OK)
            s = dalloc(h, &h->stage_alpha[sl], (size_t)dm.B * dm.H * (h->alpha_per_key ? dm.d : 1) * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->stage_beta[sl], (size_t)dm.B * dm.H * dm.L * sizeof(float));
    }
    if (s == ARL2_OK && h->stage_slots == 2) {
        if (cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking) != cudaSuccess)
            s = ARL2_ERR_CUDA;
        for (int sl = 0; sl < 2 && s == ARL2_OK; ++sl)
            if (cudaEventCreateWithFlags(&h->ev_in[sl], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&h->ev_fwd[sl], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&h->ev_out[sl], cudaEventDisableTiming) != cudaSuccess)
                s = ARL2_ERR_CUDA;
    }
    const size_t gate_w_bytes =
        cfg->w_gate ? (size_t)cfg->hidden_dim * arl2::gate_padded_outputs(dm.H) * h->esz : 0;
    if (s == ARL2_OK && cfg->w_gate) {
        h->hidden = cfg->hidden_dim;
        s = dalloc(h, &h->w_gate, gate_w_bytes);
        if (s == ARL2_OK) s = dalloc(h, &h->b_gate, 2 * (size_t)dm.H * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->g_alpha, (size_t)dm.B * dm.H * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->g_beta, (size_t)dm.B * dm.H * dm.L * sizeof(float));
        if (s == ARL2_OK)
            s = dalloc(h, &h->g_part, (size_t)dm.B * arl2::gate_part_count(dm.L) * dm.H * sizeof(float));
        if (s == ARL2_OK) s = dalloc(h, &h->g_count, (size_t)dm.B * sizeof(unsigned));
        for (int sl = 0; sl < h->stage_slots && s == ARL2_OK; ++sl)
            s = dalloc(h, &h->stage_x[sl], (size_t)dm.B * dm.L * h->hidden * h->esz);
    }
    if (s == ARL2_OK && arl2::simt_init() != cudaSuccess) s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && h->w_gate && arl2::gate_init() != cudaSuccess) s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && h->w_gate && use_tc)  // nullptr (shapes it does not take): the SIMT kernel
        h->gtc = arl2::gate_tc_create(dm.B, dm.L, h->hidden, dm.H, h->w_gate, arl2::gate_padded_outputs(dm.H));
    if (s == ARL2_OK && use_tc) {
        h->maps = new (std::nothrow) arl2::TokenMapCache(dm);
        h->tc = arl2::attn_tc_create(dm, h->attn_ws, cfg->max_ctas);
        const arl2::UpdateBuffers ub{h->w_all, h->S, h->Sb, h->Mt, h->part_s};
        h->up = arl2::update_tc_create(dm, ub);
        if (!h->maps || !h->maps->ok() || !h->tc || !h->up) s = ARL2_ERR_CUDA;
        if (s == ARL2_OK && h->token_level) {
            h->tltc = arl2::tl_tc_create(dm, h->w_all, h->tltc_ws);
            if (!h->tltc) s = ARL2_ERR_CUDA;
        }
    }
    if (s != ARL2_OK) {
        release(h);
        return s;
    }
    const void* src[3] = {cfg->w_q, cfg->w_k, cfg->w_v};
    for (int i = 0; i < 3; ++i)
        if (cudaMemcpyAsync(h->w[i], src[i], wbytes, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
            s = ARL2_ERR_CUDA;
    if (s == ARL2_OK) s = zero_state(h, stream);
    if (s == ARL2_OK && (cudaMemsetAsync(h->err, 0, sizeof(int), stream) != cudaSuccess ||
                         cudaMemsetAsync(h->quiet, 0, sizeof(int), stream) != cudaSuccess))
        s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && h->w_gate &&
        (arl2::launch_gate_transpose(h->dtype == ARL2_BF16, cfg->w_gate, h->w_gate, h->hidden, dm.H, stream) !=
             cudaSuccess ||
         cudaMemcpyAsync(h->b_gate, cfg->b_gate, 2 * (size_t)dm.H * sizeof(float), cudaMemcpyDeviceToDevice,
                         stream) != cudaSuccess ||
         cudaMemsetAsync(h->g_count, 0, (size_t)dm.B * sizeof(unsigned), stream) != cudaSuccess))
        s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && use_tc &&
        cudaMemsetAsync(h->attn_ws, 0, arl2::attn_tc_workspace_bytes(dm), stream) != cudaSuccess)
        s = ARL2_ERR_CUDA;
    if (s == ARL2_OK && h->token_level &&
        cudaMemsetAsync(h->zero_read, 0, h->n_state * (use_tc ? 2 : sizeof(float)), stream) != cudaSuccess)
        s = ARL2_ERR_CUDA;
    if (s != ARL2_OK) {
        cudaStreamSynchronize(stream);
        release(h);
        return s;
    }
    *out = h;
    return ARL2_OK;
}

// Token-level access: the intra-frame term through the usual attention
// kernel reading a zero state, the phi maps in fp32, then the chunked
// sequential read/update (token_level.cu), which adds q'_i S^(i) to out and
// keeps S^(L) on the clean pass.
static arl2_status token_level_pass(arl2_handle* h, const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, bool clean, void* out,
                                    cudaStream_t st) {
    const bool bf16 = h->dtype == ARL2_BF16;
    const Dims& dm = h->dm;
    if (h->use_tc) {
        // the intra-frame term (the attention kernel reading a zero state),
        // then the token-level reads and states on the tensor cores
        h->launches += 3;
        if (arl2::attn_tc_launch(h->tc, *h->maps, q, k, v, h->zero_read, out, h->scale, h->err, st) !=
                cudaSuccess ||
            arl2::tl_tc_launch(h->tltc, *h->maps, q, k, v, alpha, h->alpha_per_key, beta, h->S, out, clean,
                               h->err, st) != cudaSuccess)
            return ARL2_ERR_CUDA;
        if (clean) return refresh_derived(h, st);
        return ARL2_OK;
    } else {
        h->launches += 2;
        if (arl2::launch_phi_simt(bf16, q, h->w[0], false, h->qp, nullptr, dm, st) != cudaSuccess ||
            arl2::launch_attn_simt(bf16, q, k, v, h->qp, static_cast<const float*>(h->zero_read), out,
                                   h->scale, dm, st) != cudaSuccess)
            return ARL2_ERR_CUDA;
    }
    h->launches += 4;
    if (arl2::launch_phi_simt(bf16, k, h->w[1], true, h->kp, nullptr, dm, st) != cudaSuccess ||
        arl2::launch_phi_simt(bf16, v, h->w[2], false, h->vp, nullptr, dm, st) != cudaSuccess ||
        arl2::launch_tl(h->qp, h->kp, h->vp, alpha, h->alpha_per_key, beta, h->tl_ws, h->S, out, bf16,
                        clean, dm, st) != cudaSuccess)
        return ARL2_ERR_CUDA;
    // the tensor-core copies of the state follow S (checkpoint consistency)
    if (clean) return refresh_derived(h, st);
    return ARL2_OK;
}

arl2_status arl2_frame_forward(arl2_handle* h, const void* q, const void* k, const void* v,
                               const float* alpha, const float* beta, int clean_pass, void* out,
                               cudaStream_t stream) {
    if (!h || !q || !k || !v || !out) return ARL2_ERR_INVALID_ARG;
    // token-level access reads through the gates on every pass
    if ((clean_pass || h->token_level) && (!alpha || !beta)) return ARL2_ERR_INVALID_ARG;
    if (out == q || out == k || out == v) return ARL2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ARL2_ERR_ALIGN;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const bool bf16 = h->dtype == ARL2_BF16;
    if (h->token_level) return token_level_pass(h, q, k, v, alpha, beta, clean_pass != 0, out, stream);
    if (h->use_tc) {
        ++h->launches;
        if (arl2::attn_tc_launch(h->tc, *h->maps, q, k, v, h->Mt, out, h->scale, h->err, stream) !=
            cudaSuccess)
            return ARL2_ERR_CUDA;
    } else {
        h->launches += 2;
        if (arl2::launch_phi_simt(bf16, q, h->w[0], false, h->qp, nullptr, h->dm, stream) != cudaSuccess ||
            arl2::launch_attn_simt(bf16, q, k, v, h->qp, h->S, out, h->scale, h->dm, stream) !=
                cudaSuccess)
            return ARL2_ERR_CUDA;
    }
    if (clean_pass) return clean_update(h, k, v, alpha, beta, stream);
    return ARL2_OK;
}

arl2_status arl2_frame_forward_host(arl2_handle* h, const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, int clean_pass,
                                    void* out, cudaStream_t stream) {
    if (!h || !q || !k || !v || !out) return ARL2_ERR_INVALID_ARG;
    if (h->stage_slots == 0) return ARL2_ERR_INVALID_ARG;
    const bool gates = clean_pass || h->token_level;  // the passes that read alpha and beta
    if (gates && (!alpha || !beta)) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const Dims& dm = h->dm;
    const int sl = next_slot(h);
    void* const* st = h->stage_tok[sl];
    const size_t tb = h->n_tok * h->esz;
    HostCopy in[5] = {{st[0], q, tb}, {st[1], k, tb}, {st[2], v, tb}, {}, {}};
    int n_in = 3;
    if (gates) {
        in[n_in++] = {h->stage_alpha[sl], alpha, (size_t)dm.B * dm.H * (h->alpha_per_key ? dm.d : 1) * sizeof(float)};
        in[n_in++] = {h->stage_beta[sl], beta, (size_t)dm.B * dm.H * dm.L * sizeof(float)};
    }
    return host_pass(h, sl, in, n_in, out, stream, [&]() {
        return arl2_frame_forward(h, st[0], st[1], st[2], gates ? h->stage_alpha[sl] : nullptr,
                                  gates ? h->stage_beta[sl] : nullptr, clean_pass, st[3], stream);
    });
}

arl2_status arl2_gates_apply(arl2_handle* h, const void* x, float* alpha, float* beta, cudaStream_t stream) {
    if (!h || !x || !alpha || !beta) return ARL2_ERR_INVALID_ARG;
    if (!h->w_gate) return ARL2_ERR_INVALID_ARG;
    if (!aligned16(x)) return ARL2_ERR_ALIGN;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const Dims& dm = h->dm;
    ++h->launches;
    const cudaError_t e =
        h->gtc ? arl2::gate_tc_launch(h->gtc, x, h->b_gate, beta, h->g_part, alpha, h->g_count, h->err, stream)
               : arl2::launch_gate_proj(h->dtype == ARL2_BF16, x, h->w_gate, h->b_gate, dm.B, dm.L, h->hidden, dm.H,
                                        beta, h->g_part, alpha, h->g_count, stream);
    if (e != cudaSuccess) return ARL2_ERR_CUDA;
    return ARL2_OK;
}

arl2_status arl2_frame_forward_hidden(arl2_handle* h, const void* q, const void* k, const void* v,
                                      const void* x, int clean_pass, void* out, cudaStream_t stream) {
    if (!h || !q || !k || !v || !out) return ARL2_ERR_INVALID_ARG;
    if (!h->w_gate) return ARL2_ERR_INVALID_ARG;
    const bool gates = clean_pass || h->token_level;  // the passes that read alpha and beta
    if (!gates) return arl2_frame_forward(h, q, k, v, nullptr, nullptr, 0, out, stream);
    arl2_status s = arl2_gates_apply(h, x, h->g_alpha, h->g_beta, stream);
    if (s != ARL2_OK) return s;
    return arl2_frame_forward(h, q, k, v, h->g_alpha, h->g_beta, clean_pass, out, stream);
}

arl2_status arl2_frame_forward_hidden_host(arl2_handle* h, const void* q, const void* k, const void* v,
                                           const void* x, int clean_pass, void* out, cudaStream_t stream) {
    if (!h || !q || !k || !v || !out) return ARL2_ERR_INVALID_ARG;
    if (h->stage_slots == 0 || !h->w_gate) return ARL2_ERR_INVALID_ARG;
    const bool gates = clean_pass || h->token_level;
    if (gates && !x) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const int sl = next_slot(h);
    void* const* st = h->stage_tok[sl];
    const size_t tb = h->n_tok * h->esz;
    HostCopy in[4] = {{st[0], q, tb}, {st[1], k, tb}, {st[2], v, tb}, {}};
    int n_in = 3;
    if (gates) in[n_in++] = {h->stage_x[sl], x, (size_t)h->dm.B * h->dm.L * h->hidden * h->esz};
    return host_pass(h, sl, in, n_in, out, stream, [&]() {
        return arl2_frame_forward_hidden(h, st[0], st[1], st[2], gates ? h->stage_x[sl] : nullptr, clean_pass,
                                         st[3], stream);
    });
}

arl2_status arl2_state_reset(arl2_handle* h, cudaStream_t stream) {
    if (!h) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    return zero_state(h, stream);
}

arl2_status arl2_state_get(arl2_handle* h, float* dst, cudaStream_t stream) {
    if (!h || !dst) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    if (cudaMemcpyAsync(dst, h->S, h->n_state * sizeof(float), cudaMemcpyDeviceToDevice, stream) !=
        cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

arl2_status arl2_state_set(arl2_handle* h, const float* src, cudaStream_t stream) {
    if (!h || !src) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    if (cudaMemcpyAsync(h->S, src, h->n_state * sizeof(float), cudaMemcpyDeviceToDevice, stream) !=
        cudaSuccess)
        return ARL2_ERR_CUDA;
    return refresh_derived(h, stream);
}

arl2_status arl2_phi_apply(arl2_handle* h, int which, const void* x, void* out,
                           cudaStream_t stream) {
    if (!h || !x || !out || which < 0 || which > 2) return ARL2_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return ARL2_ERR_ALIGN;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    const bool bf16 = h->dtype == ARL2_BF16;
    ++h->launches;
    if (arl2::launch_phi_simt(bf16, x, h->w[which], which == 1, nullptr, out, h->dm, stream) !=
        cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

arl2_status arl2_device_status(arl2_handle* h, cudaStream_t stream) {
    if (!h) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    int word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ARL2_ERR_CUDA;
    if (cudaMemcpy(&word, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return ARL2_ERR_CUDA;
    if (word != 0) {
        // a kernel gave up: clear the error word and any split-tile flags it
        // may have left set, so that the next launch starts clean
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

arl2_status arl2_selftest_wait_timeout(arl2_handle* h, unsigned limit_us, cudaStream_t stream) {
    if (!h || limit_us == 0 || limit_us > 1000000u) return ARL2_ERR_INVALID_ARG;
    arl2_status s = check_device(h);
    if (s != ARL2_OK) return s;
    ++h->launches;
    if (arl2::launch_selftest_wait(h->quiet, (unsigned long long)limit_us * 1000ull, h->err, stream) != cudaSuccess)
        return ARL2_ERR_CUDA;
    return ARL2_OK;
}

size_t arl2_device_bytes(const arl2_handle* h) { return h ? h->bytes : 0; }

unsigned long long arl2_kernel_launches(const arl2_handle* h) { return h ? h->launches : 0; }

void arl2_destroy(arl2_handle* h) {
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
