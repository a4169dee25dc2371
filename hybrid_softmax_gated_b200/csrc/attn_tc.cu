// Fused intra-frame softmax attention + inter-frame state read on sm_100a.
//
// "Attend Locally, Remember Linearly", technical summary §2.1: the
// intra-frame branch is bidirectional softmax attention among one frame's
// tokens (item 1); the inter-frame branch reads the fixed-size state through
// phi_q, O_inter = Q' S_{N-1} ("Output"), with every token of the frame
// reading the same pre-update state (§2.2 "Frame-Level Access").
//
// Since phi_q is a plain linear map, Q' S = Q (W_q S): the product
// M = W_q S is formed once per frame when the state changes, and the read
// becomes one extra 128x128x128 tensor-core product of the Q tile this CTA
// already holds in shared memory.  O = O_intra + O_inter leaves the kernel
// once, in bf16.
//
// One CTA owns 128 query rows of one (stream, head):
//   warp 0      TMA producer: Q, then K/V blocks of 128 keys through a
//               2-stage ring, then the (W_q S)^T tile in the K ring
//   warp 1      UMMA issuer (one thread): S_j = Q K_j^T into TMEM
//               (double-buffered), O += P_j V_j, O_inter = Q M
//   warp 2      TMEM allocator
//   warps 4-7   softmax + epilogue: thread i owns query row i (TMEM lane i)
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,384) O,
// [384,512) O_inter, all fp32.
// Online softmax with lazy rescaling: the running row max only moves when
// it grows by more than 2^8; the final 1/l uses the same max as the
// numerator, so the result is exact up to rounding.
#include "attn_tc.h"
#include "ptx.cuh"

#include <cuda_bf16.h>

#include <cmath>
#include <cstring>
#include <new>

namespace arl2 {
namespace {

constexpr int kBM = 128;                       // query rows per CTA
constexpr int kBN = 128;                       // keys per block
constexpr int kD = 128;                        // head dim
using ptx::kHalfBytes;
using ptx::kTileBytes;
using ptx::kmajor_desc;
using ptx::mnmajor_desc;
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColOi = 384;
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr float kRescaleLog2 = 8.0f;

struct __align__(1024) Smem {
    uint8_t q[kTileBytes];
    uint8_t k[kStages][kTileBytes];
    uint8_t v[kStages][kTileBytes];
    uint8_t p[kTileBytes];
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full, o_ready, done;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
                   __nv_bfloat16* __restrict__ out, int L, int H, float scale_log2, int* err) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int n_kv = (L + kBN - 1) / kBN;
    volatile int* abort = &sm.abort;
    const int no_abort = 0;

    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&sm.q_full), 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(ptx::smem_u32(&sm.k_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.k_empty[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.v_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.v_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(ptx::smem_u32(&sm.s_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.s_empty[s]), kBM);
        }
        ptx::mbar_init(ptx::smem_u32(&sm.p_full), kBM);
        ptx::mbar_init(ptx::smem_u32(&sm.o_ready), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.done), 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_u32(&sm.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    auto fail = [&]() {
        atomicOr(err, kErrTimeoutAttn);
        *abort = 1;
    };

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer --
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
        ptx::tma_prefetch_desc(&tm_m);
        const uint32_t q_s = ptx::smem_u32(sm.q);
        const int t0 = qt * kBM;
        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&sm.q_full), kTileBytes);
        ptx::tma_load_4d(q_s, &tm_q, 0, h, t0, b, ptx::smem_u32(&sm.q_full));
        ptx::tma_load_4d(q_s + kHalfBytes, &tm_q, 64, h, t0, b, ptx::smem_u32(&sm.q_full));
        // Block i of the K ring is keys [128 i, 128 i + 128); block n_kv is
        // the (W_q S)^T tile.  Loads follow the order the UMMA warp
        // consumes them: K0, then (K_{j+1}, V_j) for j = 0 .. n_kv-1.
        auto load_k = [&](int i) -> bool {
            const int s = i & 1;
            if (i >= 2 &&
                !ptx::mbar_wait_bounded(ptx::smem_u32(&sm.k_empty[s]), ((i >> 1) - 1) & 1, abort,
                                        kWaitLimitNs))
                return false;
            const uint32_t bar = ptx::smem_u32(&sm.k_full[s]);
            const uint32_t dst = ptx::smem_u32(sm.k[s]);
            ptx::mbar_arrive_expect_tx(bar, kTileBytes);
            if (i < n_kv) {
                ptx::tma_load_4d(dst, &tm_k, 0, h, i * kBN, b, bar);
                ptx::tma_load_4d(dst + kHalfBytes, &tm_k, 64, h, i * kBN, b, bar);
            } else {
                ptx::tma_load_4d(dst, &tm_m, 0, 0, b * H + h, 0, bar);
                ptx::tma_load_4d(dst + kHalfBytes, &tm_m, 64, 0, b * H + h, 0, bar);
            }
            return true;
        };
        auto load_v = [&](int j) -> bool {
            const int s = j & 1;
            if (j >= 2 &&
                !ptx::mbar_wait_bounded(ptx::smem_u32(&sm.v_empty[s]), ((j >> 1) - 1) & 1, abort,
                                        kWaitLimitNs))
                return false;
            const uint32_t bar = ptx::smem_u32(&sm.v_full[s]);
            const uint32_t dst = ptx::smem_u32(sm.v[s]);
            ptx::mbar_arrive_expect_tx(bar, kTileBytes);
            ptx::tma_load_4d(dst, &tm_v, 0, h, j * kBN, b, bar);
            ptx::tma_load_4d(dst + kHalfBytes, &tm_v, 64, h, j * kBN, b, bar);
            return true;
        };
        bool ok = load_k(0);
        int k_issued = ok ? 1 : 0, v_issued = 0;
        for (int j = 0; ok && j < n_kv; ++j) {
            ok = load_k(j + 1);
            if (ok) k_issued = j + 2;
            if (ok) ok = load_v(j);
            if (ok) v_issued = j + 1;
        }
        if (!ok) fail();
        // Drain: every load this thread issued has landed before the CTA
        // may exit (consumed phases return at once).
        ptx::mbar_wait_bounded(ptx::smem_u32(&sm.q_full), 0, &no_abort, kWaitLimitNs);
        for (int i = k_issued - 2; i < k_issued; ++i)
            if (i >= 0)
                ptx::mbar_wait_bounded(ptx::smem_u32(&sm.k_full[i & 1]), (i >> 1) & 1, &no_abort,
                                       kWaitLimitNs);
        for (int j = v_issued - 2; j < v_issued; ++j)
            if (j >= 0)
                ptx::mbar_wait_bounded(ptx::smem_u32(&sm.v_full[j & 1]), (j >> 1) & 1, &no_abort,
                                       kWaitLimitNs);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------- UMMA issuer --
        constexpr uint32_t idesc_kk = ptx::idesc_bf16_f32(kBM, kBN, false, false);
        constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kBM, kD, false, true);
        const uint32_t q_s = ptx::smem_u32(sm.q);
        const uint32_t p_s = ptx::smem_u32(sm.p);
        bool ok = ptx::mbar_wait_bounded(ptx::smem_u32(&sm.q_full), 0, abort, kWaitLimitNs);
        auto issue_qk = [&](int i) -> bool {  // S_i = Q K_i^T into buffer i & 1
            const int s = i & 1;
            if (!ptx::mbar_wait_bounded(ptx::smem_u32(&sm.k_full[s]), (i >> 1) & 1, abort,
                                        kWaitLimitNs))
                return false;
            if (i >= 2 && !ptx::mbar_wait_bounded(ptx::smem_u32(&sm.s_empty[s]), ((i >> 1) - 1) & 1,
                                                  abort, kWaitLimitNs))
                return false;
            ptx::tc_fence_after();
            const uint32_t k_s = ptx::smem_u32(sm.k[s]);
            const uint32_t d = tmem + kColS + (uint32_t)s * kBN;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
                ptx::umma_f16_ss(d, kmajor_desc(q_s, kk), kmajor_desc(k_s, kk), idesc_kk, kk > 0);
            ptx::umma_commit(ptx::smem_u32(&sm.s_full[s]));
            ptx::umma_commit(ptx::smem_u32(&sm.k_empty[s]));
            return true;
        };
        if (ok) ok = issue_qk(0);
        for (int j = 0; ok && j < n_kv; ++j) {
            if (j + 1 < n_kv) ok = issue_qk(j + 1);
            if (!ok) break;
            // O += P_j V_j
            const int s = j & 1;
            ok = ptx::mbar_wait_bounded(ptx::smem_u32(&sm.p_full), j & 1, abort, kWaitLimitNs) &&
                 ptx::mbar_wait_bounded(ptx::smem_u32(&sm.v_full[s]), (j >> 1) & 1, abort,
                                        kWaitLimitNs);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t v_s = ptx::smem_u32(sm.v[s]);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                ptx::umma_f16_ss(tmem + kColO, kmajor_desc(p_s, kk), mnmajor_desc(v_s, kk), idesc_pv,
                                 (j > 0 || kk > 0) ? 1u : 0u);
            ptx::umma_commit(ptx::smem_u32(&sm.v_empty[s]));
            ptx::umma_commit(ptx::smem_u32(&sm.o_ready));
        }
        if (ok) {
            // O_inter = Q (W_q S)^T^T, the folded state tile sits in K slot n_kv
            const int s = n_kv & 1;
            ok = ptx::mbar_wait_bounded(ptx::smem_u32(&sm.k_full[s]), (n_kv >> 1) & 1, abort,
                                        kWaitLimitNs);
            if (ok) {
                ptx::tc_fence_after();
                const uint32_t m_s = ptx::smem_u32(sm.k[s]);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    ptx::umma_f16_ss(tmem + kColOi, kmajor_desc(q_s, kk), kmajor_desc(m_s, kk),
                                     idesc_kk, kk > 0);
            }
        }
        if (!ok) fail();
        // Completion of everything issued above (also on the failure path,
        // so that no UMMA is in flight when TMEM is released).
        ptx::umma_commit(ptx::smem_u32(&sm.done));
        if (!ok)
            ptx::mbar_wait_bounded(ptx::smem_u32(&sm.done), 0, &no_abort, kWaitLimitNs);
    } else if (warp >= 4) {
        // ---------------------------------------- softmax + epilogue --
        const int row = threadIdx.x - 128;                 // query row in tile = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t p_row = ptx::smem_u32(sm.p) + (uint32_t)row * 128u;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int s = j & 1;
            // The decision to stop is made warp-wide, so that every lane
            // reaches (or skips) the warp-collective tcgen05 ops together.
            ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(ptx::smem_u32(&sm.s_full[s]),
                                                                (j >> 1) & 1, abort, kWaitLimitNs));
            if (!ok) break;
            ptx::tc_fence_after();
            uint32_t raw[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                ptx::tmem_ld32(tmem + lane_base + kColS + (uint32_t)s * kBN + (uint32_t)c * 32, raw[c]);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::reg_fence(raw[c]);
            ptx::tc_fence_before();
            ptx::mbar_arrive(ptx::smem_u32(&sm.s_empty[s]));

            float x[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(raw[c][i]) * scale_log2;
            const int valid = L - j * kBN;  // keys of this block inside the frame
            if (valid < kBN) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i >= valid) x[i] = -INFINITY;
            }
            float mx = x[0];
#pragma unroll
            for (int i = 1; i < 128; ++i) mx = fmaxf(mx, x[i]);
            const float m_new = fmaxf(m_run, mx);
            const bool need = m_new > m_run + kRescaleLog2;
            const float m_use = need ? m_new : m_run;
            const float corr = need ? ptx::ex2(m_run - m_new) : 1.f;
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < 128; ++i) {
                x[i] = ptx::ex2(x[i] - m_use);
                sum += x[i];
            }
            l_run = l_run * corr + sum;
            m_run = m_use;

            if (j >= 1) {
                // PV_{j-1} done: O is stable and the P buffer is free.
                ok = __all_sync(0xffffffffu,
                                ptx::mbar_wait_bounded(ptx::smem_u32(&sm.o_ready), (j - 1) & 1,
                                                       abort, kWaitLimitNs));
                if (!ok) break;
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        const uint32_t ta = tmem + lane_base + kColO + (uint32_t)c * 32;
                        ptx::tmem_ld32(ta, o);
                        ptx::tmem_wait_ld();
                        ptx::reg_fence(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
                        ptx::tmem_st32(ta, o);
                    }
                    ptx::tmem_wait_st();
                }
            }
            // P row -> shared memory, bf16, 128-byte swizzled K-major layout
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
                const int half = ch >> 3, c16 = ch & 7;
                const __nv_bfloat162 p0 = __floats2bfloat162_rn(x[ch * 8 + 0], x[ch * 8 + 1]);
                const __nv_bfloat162 p1 = __floats2bfloat162_rn(x[ch * 8 + 2], x[ch * 8 + 3]);
                const __nv_bfloat162 p2 = __floats2bfloat162_rn(x[ch * 8 + 4], x[ch * 8 + 5]);
                const __nv_bfloat162 p3 = __floats2bfloat162_rn(x[ch * 8 + 6], x[ch * 8 + 7]);
                const uint32_t addr =
                    p_row + (uint32_t)half * kHalfBytes + (uint32_t)((c16 ^ (row & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                             "r"(*reinterpret_cast<const uint32_t*>(&p0)),
                             "r"(*reinterpret_cast<const uint32_t*>(&p1)),
                             "r"(*reinterpret_cast<const uint32_t*>(&p2)),
                             "r"(*reinterpret_cast<const uint32_t*>(&p3))
                             : "memory");
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(ptx::smem_u32(&sm.p_full));
        }
        if (ok)
            ok = ptx::mbar_wait_bounded(ptx::smem_u32(&sm.o_ready), (n_kv - 1) & 1, abort,
                                        kWaitLimitNs) &&
                 ptx::mbar_wait_bounded(ptx::smem_u32(&sm.done), 0, abort, kWaitLimitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
            fail();
        } else {
            ptx::tc_fence_after();
            const float inv_l = 1.f / l_run;
            const int t = qt * kBM + row;
            __nv_bfloat16* orow = out + (((size_t)b * L + t) * H + h) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32], oi[32];
                ptx::tmem_ld32(tmem + lane_base + kColO + (uint32_t)c * 32, o);
                ptx::tmem_ld32(tmem + lane_base + kColOi + (uint32_t)c * 32, oi);
                ptx::tmem_wait_ld();
                ptx::reg_fence(o);
                ptx::reg_fence(oi);
                if (t < L) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = g * 8 + e * 2;
                            const float a0 = fmaf(__uint_as_float(o[i]), inv_l, __uint_as_float(oi[i]));
                            const float a1 =
                                fmaf(__uint_as_float(o[i + 1]), inv_l, __uint_as_float(oi[i + 1]));
                            const __nv_bfloat162 pr = __floats2bfloat162_rn(a0, a1);
                            w[e] = *reinterpret_cast<const uint32_t*>(&pr);
                        }
                        *reinterpret_cast<uint4*>(orow + c * 32 + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

// ------------------------------------------------------------------ host --

struct AttnTc {
    Dims dm{};
    const void* m_ptr = nullptr;
    CUtensorMap tm_m{};
};

AttnTc* attn_tc_create(Dims dm) {
    if (dm.d != kD || dm.L < 1 || dm.H < 1 || dm.B < 1 || !tma_available()) return nullptr;
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    AttnTc* t = new (std::nothrow) AttnTc();
    if (t) t->dm = dm;
    return t;
}

void attn_tc_destroy(AttnTc* t) { delete t; }

cudaError_t attn_tc_launch(AttnTc* t, TokenMapCache& maps, const void* q, const void* k,
                           const void* v, const void* Mt, void* out, float scale, int* err,
                           cudaStream_t st) {
    const Dims& dm = t->dm;
    if (Mt != t->m_ptr) {
        if (!tma_encode_tiles(&t->tm_m, Mt, dm.B * dm.H)) return cudaErrorInvalidValue;
        t->m_ptr = Mt;
    }
    CUtensorMap cq, ck, cv;
    if (!maps.get(q, &cq) || !maps.get(k, &ck) || !maps.get(v, &cv)) return cudaErrorInvalidValue;
    const dim3 grid((dm.L + kBM - 1) / kBM, dm.H, dm.B);
    attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(cq, ck, cv, t->tm_m,
                                                       static_cast<__nv_bfloat16*>(out), dm.L, dm.H,
                                                       scale * 1.4426950408889634f, err);
    return cudaGetLastError();
}

}  // namespace arl2
