// Token-level (sequential) state access on sm_100a tensor cores, bf16 layers
// with head_dim 128.
//
// The ablation the pages compare with frame-level access ("Attend Locally,
// Remember Linearly", technical summary §2.2 "Frame-Level Access"; atlas
// summary "Surprising findings"): within the frame token i reads the state
// left by tokens 0..i-1, then updates it with the delta rule; the frame's
// forget gate G (alpha, or diag(alpha) per key feature) acts once, with
// token 0's update.  Every pass reads through its own sequential states;
// only the clean pass keeps the last one.
//
// Chunked form, chunks of C = 128 tokens, S_0 the state at the chunk start
// (G applying in chunk 0 only):
//   A[j][i] = beta_i k'_j . k'_i (i < j),  T = (I + A)^-1   (lower triangular)
//   k~_j = k'_j G and q~_j = q'_j G for j >= 1 of chunk 0, else k'_j, q'_j
//   U    = T V' - (T K~) S_0                   (the chunk's residuals)
//   o_j += q~_j S_0 + sum_{i<j} P[j][i] u_i,   P[j][i] = beta_i q'_j . k'_i
//   S_C  = G S_0 + (diag(beta) K')^T U
// tl_tc_prep_kernel (one CTA per chunk, all chunks in parallel) computes on
// tcgen05 Q' = Q W_q, K' = rownorm(K W_k), V' = V W_v, then K' K'^T and
// Q' K'^T, solves for T by forward substitution in fp32 (shared memory),
// and forms T K~ and T V' on tcgen05.  It writes five bf16 128 x 128 tiles
// per chunk: T K~, Q~, P, diag(beta) K' and T V'.  tl_tc_scan_kernel (one
// CTA per stream and head) runs the chunks in order with the fp32 state in
// TMEM: W = (T K~) S_0 and O = Q~ S_0, then U = T V' - W (bf16, shared
// memory), O += P U and S += (diag(beta) K')^T U, adding O to the output
// (which holds the intra-frame term) and refreshing S_0 (bf16) for the
// next chunk.  The scan splits the value features (the columns of S evolve
// independently) over two CTAs per (stream, head).
#include "internal.h"
#include "ptx.cuh"
#include "tma.h"

#include <cuda_bf16.h>

#include <cmath>
#include <new>

namespace arl2 {
namespace {

using ptx::kHalfBytes;
using ptx::kTileBytes;
using ptx::kmajor_desc;
using ptx::mnmajor_desc;

constexpr int kC = 128;  // tokens per chunk
constexpr int kD = 128;  // head dim
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr int kTilesPerChunk = 5;  // T K~, Q~, P, diag(beta) K', T V'
enum TileKind : int { kTK = 0, kQG = 1, kP = 2, kBK = 3, kTV = 4 };

// Byte offset of element (r, c) (c in [0, 128)) of a 128 x 128 bf16 tile in
// the 128-byte-swizzled layout TMA writes for two {64, 128} boxes.
__device__ __forceinline__ uint32_t tile_elem(int r, int c) {
    return ptx::tile_chunk_offset(r, c >> 3) + (uint32_t)((c & 7) * 2);
}

// Row r of a tile as 16 columns at a time: c16 = 0..7 (16 bf16 = two
// 16-byte chunks).
__device__ __forceinline__ void st_row16(uint32_t tile, int r, int c16, const float* x) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const float* s = x + 8 * g;
        ptx::st_shared_v4(tile + ptx::tile_chunk_offset(r, 2 * c16 + g), ptx::pack_bf16x2(s[0], s[1]),
                          ptx::pack_bf16x2(s[2], s[3]), ptx::pack_bf16x2(s[4], s[5]),
                          ptx::pack_bf16x2(s[6], s[7]));
    }
}

// ---------------------------------------------------------------- prep --
constexpr int kPrepThreads = 256;

struct __align__(1024) PrepSmem {
    // seven 32 KB regions, reused through the phases:
    //   t[0] K chunk -> K' (bf16)           -> A fp32 (with t[1])
    //   t[1] Q chunk -> Q' (bf16)
    //   t[2] V chunk -> K~ (bf16, B operand)
    //   t[3] W_k     -> V' (bf16, B operand)
    //   t[4] W_q     -> T fp32 (with t[5])
    //   t[5] W_v
    //   t[6]            T (bf16, A operand)
    uint8_t t[7][kTileBytes];
    float beta[kC];
    float gate[kD];  // G per key feature (headwise: the head's alpha in every entry)
    uint64_t ld[3];  // K with W_k, Q with W_q, V with W_v
    uint64_t phi;    // K W_k, Q W_q, V W_v in TMEM
    uint64_t ap;     // K' K'^T, Q' K'^T in TMEM
    uint64_t tv;     // T K~, T V' in TMEM
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kPrepSmem = sizeof(PrepSmem) + 1024;
static_assert(kPrepSmem <= 232448, "prep shared memory");

// Row r of tile `kind` of chunk c of (stream, head) bh in the workspace:
// bf16 [B H][chunks][kind][128][128], rows contiguous.
__device__ __forceinline__ __nv_bfloat16* ws_row(__nv_bfloat16* ws, size_t bh, int nc, int c, int kind, int r) {
    return ws + ((((bh * nc + c) * kTilesPerChunk + kind) * kC + r) * (size_t)kD);
}

// 16 values -> 16 bf16 at p (32 bytes, 16-byte aligned)
__device__ __forceinline__ void st_global_bf16x16(__nv_bfloat16* p, const float* x) {
    uint4* q = reinterpret_cast<uint4*>(p);
    q[0] = make_uint4(ptx::pack_bf16x2(x[0], x[1]), ptx::pack_bf16x2(x[2], x[3]), ptx::pack_bf16x2(x[4], x[5]),
                      ptx::pack_bf16x2(x[6], x[7]));
    q[1] = make_uint4(ptx::pack_bf16x2(x[8], x[9]), ptx::pack_bf16x2(x[10], x[11]),
                      ptx::pack_bf16x2(x[12], x[13]), ptx::pack_bf16x2(x[14], x[15]));
}

// One CTA per (chunk, head, stream).  Warp 0 lane 0 loads and issues; warps
// 4-7 (thread = chunk row = TMEM lane) run the epilogues; threads 0-127
// (thread = column) solve for T.  Phases are separated by commits (the
// epilogue warps wait for the tensor cores) and by named barrier 1 over all
// 256 threads (the issuer waits for the epilogues and the solve).
__global__ void __launch_bounds__(kPrepThreads, 1)
    tl_tc_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                      const float* __restrict__ alpha, int alpha_per_key, const float* __restrict__ beta,
                      __nv_bfloat16* __restrict__ ws, int L, int H, int nc, int* err) {
    extern __shared__ uint8_t smem_raw[];
    PrepSmem& sm = *reinterpret_cast<PrepSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // chunk-major order: the last (ragged) chunks of every (stream, head)
    // are dispatched last, so that when the grid takes more than one wave
    // the later wave holds the chunks with the least solve work
    const int n_bh = (int)(gridDim.x / (unsigned)nc);
    const int c = (int)blockIdx.x / n_bh;
    const int bhi = (int)blockIdx.x - c * n_bh;
    const int b = bhi / H, h = bhi - b * H;
    const size_t bh = (size_t)b * H + h;
    const int t0 = c * kC;
    const int vrows = L - t0 < kC ? L - t0 : kC;  // the chunk's tokens (rows past them are zero)
    volatile int* abort = &sm.abort;
    const int no_abort = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) ptx::mbar_init(ptx::smem_u32(&sm.ld[i]), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.phi), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.ap), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.tv), 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (threadIdx.x < kC) {
        const int t = t0 + threadIdx.x;
        sm.beta[threadIdx.x] = t < L ? beta[bh * L + t] : 0.f;
        sm.gate[threadIdx.x] = alpha_per_key ? alpha[bh * kD + threadIdx.x] : alpha[bh];
    }
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_u32(&sm.tmem_base), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t tl[7];
#pragma unroll
    for (int i = 0; i < 7; ++i) tl[i] = ptx::smem_u32(sm.t[i]);
    auto fail = [&]() {
        atomicOr(err, kErrTimeoutTokenLevel);
        *abort = 1;
    };
    auto bar = [&]() { ptx::named_bar_sync(1, kPrepThreads); };
    // issuer: lane 0 of warp 0 (waits bounded; on failure the error word is set)
    const bool issuer = warp == 0 && lane == 0;
    constexpr uint32_t id_k_mn = ptx::idesc_bf16_f32(kC, kD, false, true);
    constexpr uint32_t id_k_k = ptx::idesc_bf16_f32(kC, kC, false, false);
    bool ok = true;

    // ---- phase 1: loads and Q', K', V' (fp32 in TMEM columns 128, 0, 256)
    if (issuer) {
        const uint32_t kt[3] = {tl[0], tl[1], tl[2]};  // K, Q, V chunks
        const uint32_t wt[3] = {tl[3], tl[4], tl[5]};  // W_k, W_q, W_v
        const CUtensorMap* xm[3] = {&tm_k, &tm_q, &tm_v};
        const int widx[3] = {H + h, h, 2 * H + h};
        for (int i = 0; i < 3; ++i) {
            const uint32_t bb = ptx::smem_u32(&sm.ld[i]);
            ptx::mbar_arrive_expect_tx(bb, 2 * kTileBytes);
            ptx::tma_load_4d(kt[i], xm[i], 0, h, t0, b, bb);
            ptx::tma_load_4d(kt[i] + kHalfBytes, xm[i], 64, h, t0, b, bb);
            ptx::tma_load_4d(wt[i], &tm_w, 0, 0, widx[i], 0, bb);
            ptx::tma_load_4d(wt[i] + kHalfBytes, &tm_w, 64, 0, widx[i], 0, bb);
        }
        const uint32_t dcol[3] = {0u, 128u, 256u};  // K', Q', V'
        for (int i = 0; ok && i < 3; ++i) {
            ok = ptx::mbar_wait_bounded(ptx::smem_u32(&sm.ld[i]), 0, abort, kWaitLimitNs);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem + dcol[i], kmajor_desc(kt[i], kk), mnmajor_desc(wt[i], kk), id_k_mn, kk > 0);
        }
        if (!ok) fail();
        ptx::umma_commit(ptx::smem_u32(&sm.phi));  // (also after a failure: drained below)
    }
    const int row = ((warp & 3) << 5) + lane;  // epilogue warps: chunk row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const bool epi = warp >= 4;
    const int t_row = t0 + row;
    const bool gated_row = c == 0 && row >= 1;  // G applies to tokens 1.. of chunk 0
    if (epi) {
        ok = ptx::mbar_wait_warp(ptx::smem_u32(&sm.phi), 0, abort, kWaitLimitNs);
        if (ok) {
            ptx::tc_fence_after();
            // K' = Kp / max(|Kp|, 1e-6): its bf16 row into t[0] (the A/B
            // operand of K' K'^T and Q' K'^T), K~ into t[2] (the B operand
            // of T K~), diag(beta) K' to the workspace
            float ss = 0.f;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t raw[32];
                ptx::tmem_ld32(tmem + lane_base + (uint32_t)q * 32, raw);
                ptx::tmem_wait_ld();
                ptx::reg_fence(raw);
#pragma unroll
                for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(raw[i]), __uint_as_float(raw[i]), ss);
            }
            const float inv = 1.f / fmaxf(sqrtf(ss), 1e-6f);
            const float beta_r = sm.beta[row];
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {  // 16 columns at a time
                uint32_t raw[16];
                ptx::tmem_ld16(tmem + lane_base + (uint32_t)q * 16, raw);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(raw);
                float kn[16], kt[16], bk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    kn[i] = __uint_as_float(raw[i]) * inv;
                    kt[i] = gated_row ? kn[i] * sm.gate[q * 16 + i] : kn[i];
                    bk[i] = beta_r * kn[i];
                }
                st_row16(tl[0], row, q, kn);
                st_row16(tl[2], row, q, kt);
                st_global_bf16x16(ws_row(ws, bh, nc, c, kBK, row) + q * 16, bk);
            }
            // Q' (unscaled) into t[1]; Q~ to the workspace; V' into t[3]
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {
                uint32_t rq[16], rv[16];
                ptx::tmem_ld16(tmem + lane_base + 128u + (uint32_t)q * 16, rq);
                ptx::tmem_ld16(tmem + lane_base + 256u + (uint32_t)q * 16, rv);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(rq);
                ptx::reg_fence16(rv);
                float qv[16], qg[16], vv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    qv[i] = __uint_as_float(rq[i]);
                    qg[i] = gated_row ? qv[i] * sm.gate[q * 16 + i] : qv[i];
                    vv[i] = __uint_as_float(rv[i]);
                }
                st_row16(tl[1], row, q, qv);
                st_row16(tl[3], row, q, vv);
                st_global_bf16x16(ws_row(ws, bh, nc, c, kQG, row) + q * 16, qg);
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
        }
        if (!ok) fail();
    }
    (void)t_row;
    bar();  // #1: K', Q', K~, V' tiles written

    // ---- phase 2: K' K'^T (TMEM 0) and Q' K'^T (TMEM 128)
    if (issuer) {
        if (ok) {
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem, kmajor_desc(tl[0], kk), kmajor_desc(tl[0], kk), id_k_k, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem + 128u, kmajor_desc(tl[1], kk), kmajor_desc(tl[0], kk), id_k_k, kk > 0);
        }
        ptx::umma_commit(ptx::smem_u32(&sm.ap));
    }
    // A^T (masked, times beta_i) as fp32 [i][j] over t[0..1]; P (masked,
    // times beta_i) to the workspace
    float* At = reinterpret_cast<float*>(sm.t[0]);
    if (epi) {
        ok = ptx::mbar_wait_warp(ptx::smem_u32(&sm.ap), 0, abort, kWaitLimitNs);
        if (ok) {
            ptx::tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {
                uint32_t ra[16], rp[16];
                ptx::tmem_ld16(tmem + lane_base + (uint32_t)q * 16, ra);
                ptx::tmem_ld16(tmem + lane_base + 128u + (uint32_t)q * 16, rp);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(ra);
                ptx::reg_fence16(rp);
                float pv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int col = q * 16 + i;
                    const float bi = col < row ? sm.beta[col] : 0.f;  // strictly lower
                    At[col * kC + row] = bi * __uint_as_float(ra[i]);
                    pv[i] = bi * __uint_as_float(rp[i]);
                }
                st_global_bf16x16(ws_row(ws, bh, nc, c, kP, row) + q * 16, pv);
            }
            ptx::tc_fence_before();
        }
        if (!ok) fail();
    }
    bar();  // #2: A^T written; TMEM 0-255 read out

    // ---- phase 3: T = (I + A)^-1, fp32.  With A in 2 x 2 blocks,
    //   T = [[T11, 0], [T21, T22]],  T11 = (I + A11)^-1,  T22 = (I + A22)^-1,
    //   T21 = -T22 A21 T11,
    // applied twice: the four 32-row diagonal blocks are solved at once by
    // forward substitution (thread = column e: T[j][e] = [j == e] -
    // sum_{r0 <= i < j} A[j][i] T[i][e], T[i][e] = 0 for i < e, so every
    // thread of a block runs the same rows and reads A broadcast; rows in
    // groups of 8: the group's sums over earlier rows first, then the
    // triangle inside the group), the lower 32-block of each 64-row half
    // follows from two 32^3 products, and the lower 64-block from two 64^3
    // products, all on 256 threads.  T fp32 [j][e] over t[4..5], its bf16
    // copy into t[6] (the A operand of T K~ and T V').  A^T[i][j] for
    // i >= 64 > j is zero and unused: the products' X = A21 T11 go there.
    float* Tf = reinterpret_cast<float*>(sm.t[4]);
    auto st_t_bf16 = [&](int j, int e, float x) {
        const __nv_bfloat16 hv = __float2bfloat16_rn(x);
        asm volatile("st.shared.b16 [%0], %1;" ::"r"(tl[6] + tile_elem(j, e)),
                     "h"(*reinterpret_cast<const unsigned short*>(&hv))
                     : "memory");
    };
    const bool go = ok && !*abort;
    if (go && threadIdx.x < kC) {
        const int r0 = threadIdx.x & ~31;  // the diagonal block's first row
        const int e = threadIdx.x;
#pragma unroll 1
        for (int jb = r0; jb < r0 + 32; jb += 8) {
            if (jb >= vrows) {
                // rows of padding: k' = 0 there, so A's row is zero and T's is e_j
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float x = jb + r == e ? 1.f : 0.f;
                    Tf[(jb + r) * kC + e] = x;
                    st_t_bf16(jb + r, e, x);
                }
                continue;
            }
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int i = r0; i < jb; ++i) {
                const float ti = Tf[i * kC + e];
                const float4 a0 = *reinterpret_cast<const float4*>(At + i * kC + jb);
                const float4 a1 = *reinterpret_cast<const float4*>(At + i * kC + jb + 4);
                acc[0] = fmaf(a0.x, ti, acc[0]);
                acc[1] = fmaf(a0.y, ti, acc[1]);
                acc[2] = fmaf(a0.z, ti, acc[2]);
                acc[3] = fmaf(a0.w, ti, acc[3]);
                acc[4] = fmaf(a1.x, ti, acc[4]);
                acc[5] = fmaf(a1.y, ti, acc[5]);
                acc[6] = fmaf(a1.z, ti, acc[6]);
                acc[7] = fmaf(a1.w, ti, acc[7]);
            }
            float tv[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float x = (jb + r == e ? 1.f : 0.f) - acc[r];
#pragma unroll
                for (int i = 0; i < r; ++i) x = fmaf(-At[(jb + i) * kC + jb + r], tv[i], x);
                tv[r] = x;
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                Tf[(jb + r) * kC + e] = tv[r];
                st_t_bf16(jb + r, e, tv[r]);
            }
        }
    } else if (go) {
        const int u = threadIdx.x - kC;
        // T12 = 0: rows 0-63, columns 64-127 (bf16 only: no product reads it)
        {
            const int e = 64 + (u & 63);
#pragma unroll 4
            for (int j = (u >> 6) & 1; j < 64; j += 2) st_t_bf16(j, e, 0.f);
        }
        // the 32-blocks above the diagonal inside each half (fp32 too: the
        // 64-level products read T11 and T22 whole)
        {
            const int hb = u >> 6;
            const int e = 64 * hb + 32 + (u & 31);
#pragma unroll 4
            for (int j = 64 * hb + ((u >> 5) & 1); j < 64 * hb + 32; j += 2) {
                Tf[j * kC + e] = 0.f;
                st_t_bf16(j, e, 0.f);
            }
        }
    }
    bar();  // #3a: the diagonal 32-blocks, and zeros above them
    {
        // inside half hh: X' = A21' T11' (32 x 32, into A^T's unused rows),
        // then T21' = -T22' X'; thread = 2 rows x 4 columns of one half
        const int hh = threadIdx.x >> 7;
        const int idx = threadIdx.x & 127;
        const int pk = (idx >> 3) * 2, pe = (idx & 7) * 4;
        const int o = 64 * hh;  // the half's first row and column
        const bool lower32 = go && vrows > o + 32;  // else A21' = 0 (rows of padding) and T21' = 0
        float* Xs = At + (64 + 32 * hh) * kC + 32 * hh;  // X'[k][e] at Xs[k * kC + e]
        if (lower32) {
            float acc[2][4] = {};
#pragma unroll 4
            for (int i = 0; i < 32; ++i) {
                const float a0 = At[(o + i) * kC + o + 32 + pk];  // A[o + 32 + pk][o + i]
                const float a1 = At[(o + i) * kC + o + 33 + pk];
                const float4 t = *reinterpret_cast<const float4*>(Tf + (o + i) * kC + o + pe);
                const float tv4[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    acc[0][v] = fmaf(a0, tv4[v], acc[0][v]);
                    acc[1][v] = fmaf(a1, tv4[v], acc[1][v]);
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
                *reinterpret_cast<float4*>(Xs + (pk + r) * kC + pe) =
                    make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        }
        bar();  // #3b: X' written
        if (lower32) {
            float acc[2][4] = {};
#pragma unroll 4
            for (int m = 0; m < 32; ++m) {
                const float t0 = Tf[(o + 32 + pk) * kC + o + 32 + m];  // T22'[pk][m]
                const float t1 = Tf[(o + 33 + pk) * kC + o + 32 + m];
                const float4 x = *reinterpret_cast<const float4*>(Xs + m * kC + pe);
                const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    acc[0][v] = fmaf(t0, xv[v], acc[0][v]);
                    acc[1][v] = fmaf(t1, xv[v], acc[1][v]);
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    Tf[(o + 32 + pk + r) * kC + o + pe + v] = -acc[r][v];
                    st_t_bf16(o + 32 + pk + r, o + pe + v, -acc[r][v]);
                }
        } else if (go) {
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    Tf[(o + 32 + pk + r) * kC + o + pe + v] = 0.f;
                    st_t_bf16(o + 32 + pk + r, o + pe + v, 0.f);
                }
        }
    }
    bar();  // #3c: T11, T22 (and T12 = 0) written
    // X = A21 T11 (64 x 64): thread = 4 rows j x 4 columns e
    const int mj = (threadIdx.x >> 4) * 4, me = (threadIdx.x & 15) * 4;
    float* X = At + 64 * kC;  // X[k][e] at A^T row 64 + k (e < 64)
    // with no token past row 63, A21 = 0 and T21 = 0
    const bool lower = go && vrows > 64;
    if (lower) {
        float acc[4][4] = {};
#pragma unroll 4
        for (int i = 0; i < 64; ++i) {
            const float4 a = *reinterpret_cast<const float4*>(At + i * kC + 64 + mj);  // A[64 + mj..][i]
            const float4 t = *reinterpret_cast<const float4*>(Tf + i * kC + me);       // T11[i][me..]
            const float av[4] = {a.x, a.y, a.z, a.w}, tv4[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], tv4[v], acc[u][v]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            *reinterpret_cast<float4*>(X + (mj + u) * kC + me) = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    bar();  // #3b: X written
    // T21 = -T22 X
    if (lower) {
        float acc[4][4] = {};
#pragma unroll 4
        for (int k = 0; k < 64; ++k) {
            const float4 x = *reinterpret_cast<const float4*>(X + k * kC + me);
            const float xv[4] = {x.x, x.y, x.z, x.w};
            float tv4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) tv4[u] = Tf[(64 + mj + u) * kC + 64 + k];  // T22[mj + u][k]
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(tv4[u], xv[v], acc[u][v]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) st_t_bf16(64 + mj + u, me + v, -acc[u][v]);
    } else if (go) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) st_t_bf16(64 + mj + u, me + v, 0.f);
    }
    if (go) ptx::fence_proxy_async_smem();  // (after every st.shared of this thread into t[6])
    bar();  // #3: T (bf16) complete

    // ---- phase 4: T K~ (TMEM 0) and T V' (TMEM 128)
    if (issuer) {
        if (ok && !*abort) {
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem, kmajor_desc(tl[6], kk), mnmajor_desc(tl[2], kk), id_k_mn, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem + 128u, kmajor_desc(tl[6], kk), mnmajor_desc(tl[3], kk), id_k_mn, kk > 0);
        }
        ptx::umma_commit(ptx::smem_u32(&sm.tv));
    }
    if (epi) {
        ok = ptx::mbar_wait_warp(ptx::smem_u32(&sm.tv), 0, abort, kWaitLimitNs);
        if (ok) {
            ptx::tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {
                uint32_t rk[16], rv[16];
                ptx::tmem_ld16(tmem + lane_base + (uint32_t)q * 16, rk);
                ptx::tmem_ld16(tmem + lane_base + 128u + (uint32_t)q * 16, rv);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(rk);
                ptx::reg_fence16(rv);
                float xk[16], xv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    xk[i] = __uint_as_float(rk[i]);
                    xv[i] = __uint_as_float(rv[i]);
                }
                st_global_bf16x16(ws_row(ws, bh, nc, c, kTK, row) + q * 16, xk);
                st_global_bf16x16(ws_row(ws, bh, nc, c, kTV, row) + q * 16, xv);
            }
        }
        if (!ok) fail();
    }
    // Drain: every load has landed and every product finished before exit.
    if (issuer) {
        for (int i = 0; i < 3; ++i) ptx::mbar_wait_bounded(ptx::smem_u32(&sm.ld[i]), 0, &no_abort, kWaitLimitNs);
        ptx::mbar_wait_bounded(ptx::smem_u32(&sm.tv), 0, &no_abort, kWaitLimitNs);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- scan --
constexpr int kScanThreads = 256;
constexpr int kNv = 64;  // value features per scan CTA (the columns of S evolve independently)
constexpr uint32_t kNvBytes = kC * kNv * 2;  // a 128 x 64 bf16 operand: one 128-byte swizzle span wide

struct __align__(1024) ScanSmem {
    uint8_t s0[kNvBytes];    // S_0 columns [n0, n0 + 64) in bf16, rows = key feature (B, MN-major)
    uint8_t u[kNvBytes];     // U columns [n0, n0 + 64) in bf16, rows = token (B, MN-major)
    uint8_t tv[kNvBytes];    // T V' columns [n0, n0 + 64)
    uint8_t tk[kTileBytes];  // T K~ of the chunk (A operand)
    uint8_t qg[kTileBytes];  // Q~ (A operand)
    uint8_t p[kTileBytes];   // P (A operand)
    uint8_t bk[kTileBytes];  // diag(beta) K' (A operand, MN-major: read as its transpose)
    uint64_t full_a, full_tv, full_b;  // chunk tiles landed: T K~ and Q~, T V', P and diag(beta) K'
    uint64_t c1;        // W = T K~ S_0 and O = Q~ S_0 done
    uint64_t c2;        // O += P U and S += (diag(beta) K')^T U done
    uint64_t s0_ready;  // 4 warp arrivals: S_0 (bf16) written
    uint64_t u_ready;   // 4 warp arrivals: U written (and W, T V' read)
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kScanSmem = sizeof(ScanSmem) + 1024;
static_assert(kScanSmem <= 232448, "scan shared memory");

// Byte offset of the 16-byte chunk c16 (0..7) of row r in a 128 x 64 bf16
// operand (one 128-byte swizzle span wide).
__device__ __forceinline__ uint32_t nv_chunk_offset(int r, int c16) {
    return (uint32_t)r * 128u + (uint32_t)((c16 ^ (r & 7)) << 4);
}
__device__ __forceinline__ void st_nv16(uint32_t tile, int r, int c16x2, const float* x) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const float* s = x + 8 * g;
        ptx::st_shared_v4(tile + nv_chunk_offset(r, 2 * c16x2 + g), ptx::pack_bf16x2(s[0], s[1]),
                          ptx::pack_bf16x2(s[2], s[3]), ptx::pack_bf16x2(s[4], s[5]),
                          ptx::pack_bf16x2(s[6], s[7]));
    }
}

// One CTA per (value-feature half, head, stream): the chunks in order.  Warp
// 0 lane 0 loads the chunk tiles (tensor map over the workspace tiles) and
// issues; warps 4-7 (thread = TMEM lane: token j for W and O, key feature m
// for S) run the epilogues.  TMEM: S fp32 at 0, W at 64, O at 128 + 64 (c & 1)
// (two buffers: chunk c's output is read out while chunk c + 1's first
// products run).
template <bool kClean>
__global__ void __launch_bounds__(kScanThreads, 1)
    tl_tc_scan_kernel(const __grid_constant__ CUtensorMap tm_ws, const float* __restrict__ alpha,
                      int alpha_per_key, float* __restrict__ S, __nv_bfloat16* __restrict__ out, int L, int H,
                      int nc, int* err) {
    extern __shared__ uint8_t smem_raw[];
    ScanSmem& sm = *reinterpret_cast<ScanSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kNv, h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * H + h;
    volatile int* abort = &sm.abort;
    const int no_abort = 0;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&sm.full_a), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.full_tv), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.full_b), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.c1), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.c2), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.s0_ready), 4);
        ptx::mbar_init(ptx::smem_u32(&sm.u_ready), 4);
        sm.abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_u32(&sm.tmem_base), 256);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    auto fail = [&]() {
        atomicOr(err, kErrTimeoutTokenLevel);
        *abort = 1;
    };
    auto tile_index = [&](int c, int kind) { return (int)((bh * nc + c) * kTilesPerChunk + kind); };
    constexpr uint32_t kColW = 64, kColO = 128;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------- loads and products --
        constexpr uint32_t id_k_mn = ptx::idesc_bf16_f32(kC, kNv, false, true);
        constexpr uint32_t id_mn_mn = ptx::idesc_bf16_f32(kC, kNv, true, true);
        const uint32_t s0 = ptx::smem_u32(sm.s0), u = ptx::smem_u32(sm.u), tv = ptx::smem_u32(sm.tv);
        const uint32_t tk = ptx::smem_u32(sm.tk), qg = ptx::smem_u32(sm.qg);
        const uint32_t pp = ptx::smem_u32(sm.p), bk = ptx::smem_u32(sm.bk);
        auto load2 = [&](uint32_t bar, uint32_t d0, int i0, uint32_t d1, int i1) {
            ptx::mbar_arrive_expect_tx(bar, 2 * kTileBytes);
            ptx::tma_load_4d(d0, &tm_ws, 0, 0, i0, 0, bar);
            ptx::tma_load_4d(d0 + kHalfBytes, &tm_ws, 64, 0, i0, 0, bar);
            ptx::tma_load_4d(d1, &tm_ws, 0, 0, i1, 0, bar);
            ptx::tma_load_4d(d1 + kHalfBytes, &tm_ws, 64, 0, i1, 0, bar);
        };
        auto load_tv = [&](int c) {  // this CTA's 64 columns of T V'
            const uint32_t bar = ptx::smem_u32(&sm.full_tv);
            ptx::mbar_arrive_expect_tx(bar, kNvBytes);
            ptx::tma_load_4d(tv, &tm_ws, n0, 0, tile_index(c, kTV), 0, bar);
        };
        auto wt = [&](uint64_t* bar, uint32_t par) {
            return ptx::mbar_wait_bounded(ptx::smem_u32(bar), par, abort, kWaitLimitNs);
        };
        load2(ptx::smem_u32(&sm.full_a), tk, tile_index(0, kTK), qg, tile_index(0, kQG));
        load_tv(0);
        load2(ptx::smem_u32(&sm.full_b), pp, tile_index(0, kP), bk, tile_index(0, kBK));
        bool ok = true;
        for (int c = 0; ok && c < nc; ++c) {
            const uint32_t par = c & 1;
            const uint32_t o_col = tmem + kColO + (uint32_t)(c & 1) * kNv;
            // W = (T K~) S_0 and O = Q~ S_0
            ok = wt(&sm.full_a, par) && wt(&sm.s0_ready, par);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem + kColW, kmajor_desc(tk, kk), mnmajor_desc(s0, kk), id_k_mn, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(o_col, kmajor_desc(qg, kk), mnmajor_desc(s0, kk), id_k_mn, kk > 0);
            ptx::umma_commit(ptx::smem_u32(&sm.c1));
            // the next chunk's T K~ and Q~ once these products are done
            ok = wt(&sm.c1, par);
            if (!ok) break;
            if (c + 1 < nc) load2(ptx::smem_u32(&sm.full_a), tk, tile_index(c + 1, kTK), qg, tile_index(c + 1, kQG));
            // O += P U and S += (diag(beta) K')^T U
            ok = wt(&sm.u_ready, par);
            if (!ok) break;
            if (c + 1 < nc) load_tv(c + 1);
            ok = wt(&sm.full_b, par);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(o_col, kmajor_desc(pp, kk), mnmajor_desc(u, kk), id_k_mn, 1u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ptx::umma_f16_ss(tmem, mnmajor_desc(bk, kk), mnmajor_desc(u, kk), id_mn_mn, 1u);
            ptx::umma_commit(ptx::smem_u32(&sm.c2));
            ok = wt(&sm.c2, par);
            if (!ok) break;
            if (c + 1 < nc) load2(ptx::smem_u32(&sm.full_b), pp, tile_index(c + 1, kP), bk, tile_index(c + 1, kBK));
        }
        if (!ok) {
            fail();
            // nothing may still run on the tensor cores when TMEM is released
            ptx::umma_commit(ptx::smem_u32(&sm.c2));
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------ epilogues --
        const int r = ((warp & 3) << 5) + lane;  // TMEM lane
        const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s0 = ptx::smem_u32(sm.s0), u = ptx::smem_u32(sm.u), tv = ptx::smem_u32(sm.tv);
        auto warp_arrive = [&](uint64_t* bar) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(bar));
        };
        auto ww = [&](uint64_t* bar, uint32_t par) {
            return ptx::mbar_wait_warp(ptx::smem_u32(bar), par, abort, kWaitLimitNs);
        };
        float* Srow = S + (bh * kD + r) * kD + n0;  // S row m = r, this CTA's columns
        // S_{N-1} into TMEM (fp32) and S_0 (bf16) into shared memory
        {
            const float g = alpha_per_key ? alpha[bh * kD + r] : alpha[bh];
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                uint32_t x[32];
                float f[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 v = *reinterpret_cast<const float4*>(Srow + q * 32 + 4 * i);
                    f[4 * i] = v.x;
                    f[4 * i + 1] = v.y;
                    f[4 * i + 2] = v.z;
                    f[4 * i + 3] = v.w;
                }
                st_nv16(s0, r, 2 * q, f);
                st_nv16(s0, r, 2 * q + 1, f + 16);
                // the TMEM copy starts as G S_{N-1}: the gate of the frame acts
                // once, with the first token's update (the products of chunk 0
                // read the ungated S_0 from shared memory)
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = __float_as_uint(g * f[i]);
                ptx::tmem_st32(tmem + lb + (uint32_t)q * 32, x);
            }
            ptx::tmem_wait_st();
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            warp_arrive(&sm.s0_ready);
        }
        bool ok = true;
        for (int c = 0; ok && c < nc; ++c) {
            const uint32_t par = c & 1;
            const int t = c * kC + r;
            // this row's intra-frame output (columns n0..n0+63), read early
            uint4 o_in[8];
            __nv_bfloat16* orow = out + (((size_t)b * L + t) * H + h) * kD + n0;
            if (t < L) {
#pragma unroll
                for (int i = 0; i < 8; ++i) o_in[i] = __ldcg(reinterpret_cast<const uint4*>(orow) + i);
            }
            // U = T V' - W -> bf16
            ok = ww(&sm.c1, par) && ww(&sm.full_tv, par);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t w[16];
                ptx::tmem_ld16(tmem + lb + kColW + (uint32_t)q * 16, w);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(w);
                float uu[16];
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    uint32_t v4[4];
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(v4[0]), "=r"(v4[1]), "=r"(v4[2]), "=r"(v4[3])
                                 : "r"(tv + nv_chunk_offset(r, 2 * q + g)));
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(v4[e] << 16), hi = __uint_as_float(v4[e] & 0xffff0000u);
                        uu[8 * g + 2 * e] = lo - __uint_as_float(w[8 * g + 2 * e]);
                        uu[8 * g + 2 * e + 1] = hi - __uint_as_float(w[8 * g + 2 * e + 1]);
                    }
                }
                st_nv16(u, r, q, uu);
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            warp_arrive(&sm.u_ready);
            ok = ww(&sm.c2, par);
            if (!ok) break;
            ptx::tc_fence_after();
            // S -> S_0 (bf16) first: the next chunk's products need only that
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t sv[16];
                ptx::tmem_ld16(tmem + lb + (uint32_t)q * 16, sv);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(sv);
                float sf[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) sf[i] = __uint_as_float(sv[i]);
                st_nv16(s0, r, q, sf);
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            warp_arrive(&sm.s0_ready);
            // then O (this chunk's buffer) -> the output, added to the intra term
            const uint32_t o_col = tmem + lb + kColO + (uint32_t)(c & 1) * kNv;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t o[16];
                ptx::tmem_ld16(o_col + (uint32_t)q * 16, o);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(o);
                if (t < L) {
                    float y[16];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        const uint4 v = o_in[2 * q + g];
                        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            y[8 * g + 2 * e] = __uint_as_float(vv[e] << 16) + __uint_as_float(o[8 * g + 2 * e]);
                            y[8 * g + 2 * e + 1] =
                                __uint_as_float(vv[e] & 0xffff0000u) + __uint_as_float(o[8 * g + 2 * e + 1]);
                        }
                    }
                    st_global_bf16x16(orow + q * 16, y);
                }
            }
        }
        if (ok && kClean) {
            // the frame's last state
            ptx::tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                uint32_t x[32];
                ptx::tmem_ld32(tmem + lb + (uint32_t)q * 32, x);
                ptx::tmem_wait_ld();
                ptx::reg_fence(x);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4*>(Srow + q * 32 + 4 * i) =
                        make_float4(__uint_as_float(x[4 * i]), __uint_as_float(x[4 * i + 1]),
                                    __uint_as_float(x[4 * i + 2]), __uint_as_float(x[4 * i + 3]));
            }
        }
        if (!ok) fail();
    }
    // drain: the last products are complete before exit
    if (warp == 0 && lane == 0) {
        ptx::mbar_wait_bounded(ptx::smem_u32(&sm.c2), (nc - 1) & 1, &no_abort, kWaitLimitNs);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 256);
    }
}

}  // namespace

// ------------------------------------------------------------------ host --
struct TlTc {
    Dims dm{};
    int nc = 0;
    __nv_bfloat16* ws = nullptr;
    CUtensorMap tm_w{}, tm_ws{};
};

size_t tl_tc_workspace_bytes(const Dims& dm) {
    const size_t nc = (size_t)(dm.L + kC - 1) / kC;
    return (size_t)dm.B * dm.H * nc * kTilesPerChunk * kC * kD * sizeof(__nv_bfloat16);
}

TlTc* tl_tc_create(const Dims& dm, const void* w_all, void* workspace) {
    if (dm.d != kD || !tma_available() || !w_all || !workspace) return nullptr;
    if (cudaFuncSetAttribute(tl_tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrepSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(tl_tc_scan_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kScanSmem) != cudaSuccess ||
        cudaFuncSetAttribute(tl_tc_scan_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kScanSmem) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    TlTc* t = new (std::nothrow) TlTc();
    if (!t) return nullptr;
    t->dm = dm;
    t->nc = (dm.L + kC - 1) / kC;
    t->ws = static_cast<__nv_bfloat16*>(workspace);
    if (!tma_encode_tiles(&t->tm_w, w_all, 3 * dm.H) ||
        !tma_encode_tiles(&t->tm_ws, workspace, dm.B * dm.H * t->nc * kTilesPerChunk)) {
        delete t;
        return nullptr;
    }
    return t;
}

void tl_tc_destroy(TlTc* t) { delete t; }

cudaError_t tl_tc_launch(TlTc* t, TokenMapCache& maps, const void* q, const void* k, const void* v,
                         const float* alpha, int alpha_per_key, const float* beta, float* S, void* out,
                         bool clean, int* err, cudaStream_t st) {
    const Dims& dm = t->dm;
    CUtensorMap cq, ck, cv;
    if (!maps.get(q, &cq) || !maps.get(k, &ck) || !maps.get(v, &cv)) return cudaErrorInvalidValue;
    tl_tc_prep_kernel<<<dim3(t->nc * dm.H * dm.B), kPrepThreads, kPrepSmem, st>>>(
        cq, ck, cv, t->tm_w, alpha, alpha_per_key, beta, t->ws, dm.L, dm.H, t->nc, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (clean)
        tl_tc_scan_kernel<true><<<dim3(kD / kNv, dm.H, dm.B), kScanThreads, kScanSmem, st>>>(t->tm_ws, alpha, alpha_per_key,
                                                                                 S, o, dm.L, dm.H, t->nc, err);
    else
        tl_tc_scan_kernel<false><<<dim3(kD / kNv, dm.H, dm.B), kScanThreads, kScanSmem, st>>>(t->tm_ws, alpha, alpha_per_key,
                                                                                  S, o, dm.L, dm.H, t->nc, err);
    return cudaGetLastError();
}

}  // namespace arl2
