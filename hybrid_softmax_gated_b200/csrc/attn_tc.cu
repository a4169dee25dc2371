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
// becomes one extra 128x128x128 tensor-core product of a Q tile that is in
// shared memory anyway.  O = O_intra + O_inter leaves the kernel once, bf16.
//
// Work decomposition.  A tile is 128 query rows of one (stream, head); a
// unit is one tile against one block of 128 keys.  When there are more
// tiles than SMs the grid is persistent (at most one CTA per SM) and CTA c
// takes the contiguous unit range
// [c U / G, (c+1) U / G).  A tile cut by a range boundary has a head piece
// (its first key blocks, at the end of CTA c's range) and a tail piece (the
// rest, at the start of CTA c+1's range).  Each CTA runs its head piece
// FIRST and writes it as an fp32 partial (unnormalised O, running max, row
// sum) with a release flag; it runs its tail piece LAST, then acquires the
// flag of the partial the previous CTA wrote at its start and merges the
// two.  A CTA only ever waits for the CTA before it, which the block
// scheduler has dispatched first; the waits are bounded all the same.  With
// no more tiles than SMs, one CTA per tile.
//
// One CTA, 384 threads:
//   warp 0       TMA producer (whole warp, one elected lane issues): Q
//                tiles (2 slots), K and V blocks (2-stage rings), the
//                (W_q S)^T tile through the K ring
//   warp 1       UMMA issuer (whole warp, one elected lane issues)
//   warp 2       TMEM allocator
//   warp 3       epilogue helper: publishes head partials (release flag),
//                acquires the flag of a tail's head partial, issues the TMA
//                stores of staged outputs
//   warps 4-7    softmax warpgroup 0: even key blocks, accumulator O_0
//   warps 8-11   softmax warpgroup 1: odd key blocks, accumulator O_1
// The two warpgroups split the key blocks, not the columns: each thread
// owns one row (TMEM lane) of a whole 128-key block, so the row max needs
// no exchange, and each warpgroup keeps its own running max, row sum and
// accumulator.  Their softmax work interleaves with the other's products
// on the tensor core.  The epilogue combines (m_0, l_0, O_0) and
// (m_1, l_1, O_1) once per segment.
// TMEM columns: [0,256) two S/P buffers, [256,512) O_0 and O_1, fp32 (P:
// bf16 pairs packed over the first half of its S buffer).  Buffers rotate
// over "virtual blocks": each key block of a segment, then (for a segment
// that finishes its tile) one more for O_inter, read by the epilogue.
// Issue order per segment: S_0, S_1, then P V_j followed by the next item
// into buffer j & 1 (S_{j+2}, or O_inter = Q (W_q S) after P V_{n-2}).
// Online softmax with lazy rescaling: the running row max only moves when
// it grows by more than 2^8; the final 1/l uses the same max as the
// numerator, so the result is exact up to rounding.  Exponentials run on
// the SFU (ex2.approx).  A share on the FMA pipe (a Cody-Waite reduced
// polynomial in packed f32x2 arithmetic) measured slower: it costs several
// issue slots per exponential where the SFU costs one.
// Outputs leave through a TMA store staged in the segment's Q slot; split
// partials are stored so that a warp's lanes write consecutive 16 bytes.
#include "attn_tc.h"
#include "ptx.cuh"

#include <cuda_bf16.h>

#include <cmath>
#include <cstring>
#include <new>
#include <type_traits>

namespace arl2 {
namespace {

using ptx::kHalfBytes;
using ptx::kTileBytes;
using ptx::kmajor_desc;
using ptx::mnmajor_desc;

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per block
constexpr int kD = 128;   // head dim
constexpr int kThreads = 384;
constexpr int kSoftmaxWarps = 8;  // arrivals on the softmax barriers: one per warp
constexpr int kWgWarps = 4;       // warps of one softmax warpgroup
// Registers per thread: at launch (384 threads, one CTA per SM), then after
// the split: warpgroup 0 (producer, issuer, allocator, helper) gives up
// registers to the two softmax warpgroups.
constexpr int kRegsLaunch = 168, kRegsLow = 96, kRegsHigh = 200;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;  // S/P buffers at 0, 128; O_0, O_1 at 256, 384
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr float kRescaleLog2 = 8.0f;

enum SegKind : int { kFull = 0, kHead = 1, kTail = 2 };

struct Seg {
    int tile, kv0, kv1, kind;
};

// Unit schedule shared by every role of every CTA.
struct Sched {
    int n_q, n_kv, T;  // tiles per (stream, head), key blocks, tiles in total
    int n_c;           // leading key blocks read from the KV cache (0: none)
    int G;             // CTAs
    int split;         // 1: persistent unit ranges, 0: one tile per CTA
    long long U;       // units
};

struct CtaRange {
    int n_segs;
    int has_head, has_tail;
    int t_first, t_last, e0, e1;  // e0: first key block of t_first; e1: end block of t_last
    int full_lo, full_hi;         // full tiles [full_lo, full_hi)
};

__device__ __forceinline__ CtaRange cta_range(const Sched& s, int c) {
    CtaRange r{};
    if (!s.split) {
        r.n_segs = 1;
        r.full_lo = c;
        r.full_hi = c + 1;
        return r;
    }
    const long long u0 = (long long)c * s.U / s.G, u1 = (long long)(c + 1) * s.U / s.G;
    r.t_first = (int)(u0 / s.n_kv);
    r.e0 = (int)(u0 - (long long)r.t_first * s.n_kv);
    r.t_last = (int)((u1 - 1) / s.n_kv);
    r.e1 = (int)(u1 - (long long)r.t_last * s.n_kv);
    r.has_tail = r.e0 > 0;
    r.has_head = r.e1 < s.n_kv;  // (t_last > t_first whenever units per CTA >= n_kv)
    r.full_lo = r.t_first + (r.has_tail ? 1 : 0);
    r.full_hi = r.t_last + (r.has_head ? 0 : 1);
    if (r.full_hi < r.full_lo) r.full_hi = r.full_lo;
    r.n_segs = r.has_head + (r.full_hi - r.full_lo) + r.has_tail;
    return r;
}

// Segment i of the CTA: head piece first, full tiles, tail piece last.
__device__ __forceinline__ Seg seg_at(const Sched& s, const CtaRange& r, int i) {
    if (r.has_head) {
        if (i == 0) return Seg{r.t_last, 0, r.e1, kHead};
        --i;
    }
    const int nf = r.full_hi - r.full_lo;
    if (i < nf) return Seg{r.full_lo + i, 0, s.n_kv, kFull};
    return Seg{r.t_first, r.e0, s.n_kv, kTail};
}

struct __align__(1024) Smem {
    uint8_t q[2][kTileBytes];
    uint8_t k[2][kTileBytes];
    uint8_t v[2][kTileBytes];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    // Per S/P buffer b (= the softmax warpgroup that owns it): a buffer's
    // next S needs the P V of its previous block issued, so neither barrier
    // runs more than one phase ahead of its waiter.
    uint64_t s_full[2];  // one commit: S of the buffer's block is in TMEM
    uint64_t p_half[2];  // 4 warp arrivals: P of the block's first 64 keys written (O_b rescaled)
    uint64_t p_full[2];  // 4 warp arrivals: P of the other 64 keys written
    uint64_t drain;      // the issuer's last commit before it gives up after a failed wait
    uint64_t o_free;     // 8 warp arrivals per segment: O_0, O_1 and O_inter read out
    uint64_t ebar;       // 8 warp arrivals: epilogue exchange of row maxima and sums
    uint64_t stage_free[2];  // 1 arrival per segment: the Q slot used as output staging is free
    uint64_t staged[2];      // 8 warp arrivals per segment (by si & 1): output staged / head
                             // partial written; a slot's next use needs stage_free, so warp 3
                             // can never fall two phases behind on one of them
    uint64_t head_ready;     // 1 arrival: the head partial of this CTA's tail piece is visible
    float red_m[2][kBM];     // [warpgroup][row] running max (log2 units) of the segment
    float red_l[2][kBM];     // [warpgroup][row] row sum against that max
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__device__ __forceinline__ int valid_keys(int L, int kv) {
    const int v = L - kv * kBN;
    return v < kBN ? v : kBN;
}

// Keys of block kv: the first nc blocks cover the Lc cached keys, the rest
// the frame's own L keys; each run ends in its own ragged block.
__device__ __forceinline__ int block_keys(int nc, int L, int Lc, int kv) {
    return kv < nc ? valid_keys(Lc, kv) : valid_keys(L, kv - nc);
}

// K-ring items of a segment: its key blocks, then (with the inter-frame
// read, for a segment that finishes its tile) the (W_q S)^T tile.
template <bool kInter>
__device__ __forceinline__ int seg_items(const Seg& sg) {
    return sg.kv1 - sg.kv0 + (kInter && sg.kind != kHead ? 1 : 0);
}

// kInter: add the inter-frame read Q (W_q S) (the hybrid layer); without
// it, plain softmax attention whose first Lc keys come from a KV cache
// (tm_kc, tm_vc) and the rest from the frame (tm_k, tm_v).
template <bool kInter>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_m,
                   const __grid_constant__ CUtensorMap tm_o, float* __restrict__ part_o,
                   float* __restrict__ part_ml, int* __restrict__ flags, int L, int Lc, int H, Sched sch,
                   float scale_log2, int* err) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // key blocks from the KV cache (the hybrid layer has none: a constant 0)
    const int nc = kInter ? 0 : sch.n_c;
    volatile int* abort = &sm.abort;
    const int no_abort = 0;
    const CtaRange rng = cta_range(sch, blockIdx.x);
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(ptx::smem_u32(&sm.q_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.q_empty[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.k_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.k_empty[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.v_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.v_empty[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.s_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.p_half[s]), kWgWarps);
            ptx::mbar_init(ptx::smem_u32(&sm.p_full[s]), kWgWarps);
            ptx::mbar_init(ptx::smem_u32(&sm.stage_free[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.staged[s]), kSoftmaxWarps);
        }
        ptx::mbar_init(ptx::smem_u32(&sm.drain), 1);
        ptx::mbar_init(ptx::smem_u32(&sm.o_free), kSoftmaxWarps);
        ptx::mbar_init(ptx::smem_u32(&sm.ebar), kSoftmaxWarps);
        ptx::mbar_init(ptx::smem_u32(&sm.head_ready), 1);
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
    // Nothing of this kernel touches global memory before the previous kernel
    // has finished: every role starts with that wait (griddepcontrol.wait),
    // and only then lets the next kernel launch, so that the state update
    // that follows a clean pass may load the pass's inputs before its own
    // wait.

    auto fail = [&]() {
        atomicOr(err, kErrTimeoutAttn);
        *abort = 1;
    };
    // bounded wait with a warp-uniform result (every role runs as whole warps)
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
        return ptx::mbar_wait_warp(ptx::smem_u32(bar), parity, abort, kWaitLimitNs);
    };

    // Warpgroup 0 (producer, issuer, allocator, helper) hands registers to
    // the two softmax warpgroups, before it has any asynchronous copy in
    // flight (the hand-off would wait for those).
    if (warp < 4) ptx::setmaxnreg_dec<kRegsLow>();
    if (warp == 0) {
        // (the whole warp runs the producer; one elected lane issues)
        // ------------------------------------------------ TMA producer --
        ptx::pdl_wait_then_trigger();
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
        if (nc > 0) {
            ptx::tma_prefetch_desc(&tm_kc);
            ptx::tma_prefetch_desc(&tm_vc);
        }
        if (kInter) ptx::tma_prefetch_desc(&tm_m);
        int kc = 0, vc = 0;  // ring counters (same sequence as the UMMA issuer)
        // A K slot is free again once its previous item is consumed: a key
        // block is released by the softmax warpgroup that saw its S (k_empty,
        // one phase per key block in the slot), the (W_q S)^T tile by the
        // commit after O_inter (q_empty of its segment).
        int m_seg0 = -1, m_seg1 = -1;  // segment whose (W_q S)^T tile is in slot 0 / 1, or -1
        uint32_t kr_par = 0;            // bit s: parity of the next k_empty[s] phase
        int si = 0;
        bool ok = true;
        auto load_k = [&](int b, int h, int kv) -> bool {  // kv < 0: the (W_q S)^T tile
            const int s = kc & 1;
            const int m_seg = s ? m_seg1 : m_seg0;
            if (kc >= 2) {
                bool w;
                if (m_seg >= 0) {
                    w = wwait(&sm.q_empty[m_seg & 1], (m_seg >> 1) & 1);
                } else {
                    w = wwait(&sm.k_empty[s], (kr_par >> s) & 1);
                    kr_par ^= 1u << s;
                }
                if (!w) return false;
            }
            if (s)
                m_seg1 = kv < 0 ? si : -1;
            else
                m_seg0 = kv < 0 ? si : -1;
            const uint32_t bar = ptx::smem_u32(&sm.k_full[s]), dst = ptx::smem_u32(sm.k[s]);
            ptx::mbar_arrive_expect_tx_w(bar, kTileBytes);
            if (kv >= 0) {
                const CUtensorMap* tm = kv < nc ? &tm_kc : &tm_k;
                const int row = (kv < nc ? kv : kv - nc) * kBN;
                ptx::tma_load_4d_w(dst, tm, 0, h, row, b, bar);
                ptx::tma_load_4d_w(dst + kHalfBytes, tm, 64, h, row, b, bar);
            } else {
                ptx::tma_load_4d_w(dst, &tm_m, 0, 0, b * H + h, 0, bar);
                ptx::tma_load_4d_w(dst + kHalfBytes, &tm_m, 64, 0, b * H + h, 0, bar);
            }
            ++kc;
            return true;
        };
        auto load_v = [&](int b, int h, int kv) -> bool {
            const int s = vc & 1;
            if (vc >= 2 && !wwait(&sm.v_empty[s], ((vc >> 1) - 1) & 1)) return false;
            const uint32_t bar = ptx::smem_u32(&sm.v_full[s]), dst = ptx::smem_u32(sm.v[s]);
            ptx::mbar_arrive_expect_tx_w(bar, kTileBytes);
            const CUtensorMap* tm = kv < nc ? &tm_vc : &tm_v;
            const int row = (kv < nc ? kv : kv - nc) * kBN;
            ptx::tma_load_4d_w(dst, tm, 0, h, row, b, bar);
            ptx::tma_load_4d_w(dst + kHalfBytes, tm, 64, h, row, b, bar);
            ++vc;
            return true;
        };
        for (; ok && si < rng.n_segs; ++si) {
            const Seg sg = seg_at(sch, rng, si);
            const int bh = sg.tile / sch.n_q, qt = sg.tile - bh * sch.n_q;
            const int b = bh / H, h = bh - b * H;
            const int qs = si & 1;
            // the slot's previous Q is consumed and its output staging stored
            if (si >= 2 && !(wwait(&sm.q_empty[qs], ((si >> 1) - 1) & 1) &&
                             wwait(&sm.stage_free[qs], ((si >> 1) - 1) & 1))) {
                ok = false;
                break;
            }
            const uint32_t qbar = ptx::smem_u32(&sm.q_full[qs]), qdst = ptx::smem_u32(sm.q[qs]);
            ptx::mbar_arrive_expect_tx_w(qbar, kTileBytes);
            ptx::tma_load_4d_w(qdst, &tm_q, 0, h, qt * kBM, b, qbar);
            ptx::tma_load_4d_w(qdst + kHalfBytes, &tm_q, 64, h, qt * kBM, b, qbar);
            // The K ring carries the segment's key blocks, then (unless the
            // segment is a head piece) the (W_q S)^T tile; the issuer takes
            // items 0 and 1 first and item j + 2 after the P V of block j.
            const int n = sg.kv1 - sg.kv0;
            const int nk = seg_items<kInter>(sg);
            auto load_item = [&](int i) { return load_k(b, h, i < n ? sg.kv0 + i : -1); };
            for (int i = 0; ok && i < 2 && i < nk; ++i) ok = load_item(i);
            for (int j = 0; ok && j < n; ++j) {
                ok = load_v(b, h, sg.kv0 + j);
                if (ok && j + 2 < nk) ok = load_item(j + 2);
            }
        }
        if (!ok) fail();
        // Drain: the last loads of each ring have landed before exit.
        for (int i = kc - 2; i < kc; ++i)
            if (i >= 0) ptx::mbar_wait_bounded(ptx::smem_u32(&sm.k_full[i & 1]), (i >> 1) & 1, &no_abort, kWaitLimitNs);
        for (int i = vc - 2; i < vc; ++i)
            if (i >= 0) ptx::mbar_wait_bounded(ptx::smem_u32(&sm.v_full[i & 1]), (i >> 1) & 1, &no_abort, kWaitLimitNs);
        for (int i = si - 2; i < si; ++i)
            if (i >= 0) ptx::mbar_wait_bounded(ptx::smem_u32(&sm.q_full[i & 1]), (i >> 1) & 1, &no_abort, kWaitLimitNs);
    } else if (warp == 1) {
        // (the whole warp runs the issuer; one elected lane issues)
        // ------------------------------------------------- UMMA issuer --
        ptx::pdl_wait_then_trigger();
        const uint32_t idesc_pv = ptx::idesc_bf16_f32(kBM, kD, false, true);  // V: MN-major
        const uint32_t idesc_qm = ptx::idesc_bf16_f32(kBM, kD, false, false);
        int kc = 0, vc = 0;
        int vb = 0;           // virtual blocks so far: block vb + j of a segment uses buffer (vb + j) & 1
        uint32_t p_par = 0;   // bit b: phase parity of p_half[b] and p_full[b] to wait for
        int prev_oi_buf = -1; // buffer holding the previous segment's O_inter
        bool ok = true;
        int si = 0;
        for (; ok && si < rng.n_segs; ++si) {
            const Seg sg = seg_at(sch, rng, si);
            const int qs = si & 1;
            const int n = sg.kv1 - sg.kv0;
            const int nk = seg_items<kInter>(sg);
            if (!wwait(&sm.q_full[qs], (si >> 1) & 1)) {
                ok = false;
                break;
            }
            const uint32_t q_s = ptx::smem_u32(sm.q[qs]);
            // O_0, O_1 and the buffer with the previous segment's O_inter are
            // free once that segment's epilogue has read them (o_free).
            bool freed = si == 0;
            auto make_free = [&](int buf) -> bool {
                if (freed || (buf >= 0 && buf != prev_oi_buf)) return true;
                freed = true;
                return wwait(&sm.o_free, (si - 1) & 1);
            };
            // K-ring item i: S = Q K_i^T (i < n) or O_inter = Q (W_q S) (i == n),
            // into buffer (vb + i) & 1.  item_ready waits for what the item
            // needs besides the tensor pipe's order (its buffer's previous
            // contents read out, its K-ring tile), item_issue issues it.
            auto item_ready = [&](int i) -> bool {
                return make_free((vb + i) & 1) && wwait(&sm.k_full[kc & 1], (kc >> 1) & 1);
            };
            auto item_issue = [&](int i) {
                const int buf = (vb + i) & 1;
                const int s = kc & 1;
                ptx::tc_fence_after();
                const uint32_t k_s = ptx::smem_u32(sm.k[s]);
                const uint32_t d = tmem + kColS + (uint32_t)buf * kBN;
                if (i < n) {
                    const int valid = block_keys(nc, L, Lc, sg.kv0 + i);
                    const uint32_t idesc = ptx::idesc_bf16_f32(kBM, (valid + 15) & ~15, false, false);
                    ptx::umma_ss8_kk(d, kmajor_desc(q_s, 0), kmajor_desc(k_s, 0), idesc, 0u);
                    ptx::umma_commit_w(ptx::smem_u32(&sm.s_full[buf]));
                    // the last use of Q: a head piece's (once per CTA at most), or
                    // every segment's without the inter-frame read
                    if ((!kInter || sg.kind == kHead) && i == n - 1)
                        ptx::umma_commit_w(ptx::smem_u32(&sm.q_empty[qs]));
                } else {
                    // O_inter: the last use of Q and of the (W_q S)^T tile
                    ptx::umma_ss8_kk(d, kmajor_desc(q_s, 0), kmajor_desc(k_s, 0), idesc_qm, 0u);
                    ptx::umma_commit_w(ptx::smem_u32(&sm.q_empty[qs]));
                }
                ++kc;
            };
            for (int i = 0; ok && i < 2 && i < nk; ++i) {
                ok = item_ready(i);
                if (ok) item_issue(i);
            }
            if (ok) ok = make_free(-1);  // the first P V of each O_b starts it afresh
            for (int j = 0; ok && j < n; ++j) {
                const int buf = (vb + j) & 1;
                const int vs = vc & 1;
                const uint32_t par = (p_par >> buf) & 1;
                p_par ^= 1u << buf;
                // (V first: it has landed long before P, whose hand-off
                // should start the products without a further check)
                ok = wwait(&sm.v_full[vs], (vc >> 1) & 1) && wwait(&sm.p_half[buf], par);
                if (!ok) break;
                ptx::tc_fence_after();
                const int ksteps = (block_keys(nc, L, Lc, sg.kv0 + j) + 15) >> 4;
                const uint32_t p_t = tmem + kColS + (uint32_t)buf * kBN;
                const uint32_t o_t = tmem + kColO + (uint32_t)buf * kD;
                const uint32_t v_s = ptx::smem_u32(sm.v[vs]);
                const uint32_t acc0 = j >= 2 ? 1u : 0u;
                // O_b += P V, P from TMEM, in two halves of 64 keys: the first
                // runs while the softmax warps compute the second half's P.
                // A full half is one short issue sequence (the issue rate of a
                // single warp bounds the tensor pipe).
                const int k_half = ksteps < 4 ? ksteps : 4;
                if (k_half == 4) {
                    ptx::umma_ts4_mn(o_t, p_t, mnmajor_desc(v_s, 0), idesc_pv, acc0);
                } else {
                    for (int kk = 0; kk < k_half; ++kk)
                        ptx::umma_f16_ts_w(o_t, p_t + (uint32_t)kk * 8u, mnmajor_desc(v_s, kk), idesc_pv,
                                           kk > 0 ? 1u : acc0);
                }
                // The next item into this buffer follows the P V that reads it;
                // what else it needs is awaited now, while P is completed.
                const bool next = j + 2 < nk;
                ok = (!next || item_ready(j + 2)) && wwait(&sm.p_full[buf], par);
                if (!ok) break;
                ptx::tc_fence_after();
                if (ksteps == kBN / 16) {
                    ptx::umma_ts4_mn(o_t, p_t + 32u, mnmajor_desc(v_s, 4), idesc_pv, 1u);
                } else {
                    for (int kk = 4; kk < ksteps; ++kk)
                        ptx::umma_f16_ts_w(o_t, p_t + (uint32_t)kk * 8u, mnmajor_desc(v_s, kk), idesc_pv, 1u);
                }
                ptx::umma_commit_w(ptx::smem_u32(&sm.v_empty[vs]));
                ++vc;
                if (next) item_issue(j + 2);
            }
            if (!ok) break;
            prev_oi_buf = kInter && sg.kind != kHead ? (vb + n) & 1 : -1;
            vb += nk;
        }
        if (!ok) {
            fail();
            // nothing may still run on the tensor cores when TMEM is released
            ptx::umma_commit_w(ptx::smem_u32(&sm.drain));
            ptx::mbar_wait_bounded(ptx::smem_u32(&sm.drain), 0, &no_abort, kWaitLimitNs);
        }
    } else if (warp == 2) {
        // the TMEM allocator has no role in between; it triggers like the others
        ptx::pdl_wait_then_trigger();
    } else if (warp == 3) {
        // ------------------------------------------- epilogue helper --
        if (lane == 0 && rng.n_segs > 0) {
            // Warm L2 with the first tiles this CTA reads (Q, K_0, K_1, V_0) while
            // the previous kernel may still be running: only a hint, the loads
            // proper follow the wait for that kernel.  (After the register
            // hand-off, which would otherwise wait for these to complete.)
            const Seg sg = seg_at(sch, rng, 0);
            const int bh = sg.tile / sch.n_q, qt = sg.tile - bh * sch.n_q;
            const int b = bh / H, h = bh - b * H;
            for (int half = 0; half < 2; ++half) {
                ptx::tma_prefetch_l2_4d(&tm_q, half * 64, h, qt * kBM, b);
                for (int i = 0; i < 2 && sg.kv0 + i < sg.kv1; ++i) {
                    const int kv = sg.kv0 + i;
                    const int row = (kv < nc ? kv : kv - nc) * kBN;
                    ptx::tma_prefetch_l2_4d(kv < nc ? &tm_kc : &tm_k, half * 64, h, row, b);
                    if (i == 0) ptx::tma_prefetch_l2_4d(kv < nc ? &tm_vc : &tm_v, half * 64, h, row, b);
                }
            }
        }
        __syncwarp();
        ptx::pdl_wait_then_trigger();
        bool ok = true;
        for (int si = 0; ok && si < rng.n_segs; ++si) {
            const Seg sg = seg_at(sch, rng, si);
            const int bh = sg.tile / sch.n_q, qt = sg.tile - bh * sch.n_q;
            const int b = bh / H, h = bh - b * H;
            if (sg.kind == kTail) {
                // acquire the previous CTA's head partial of this tile
                if (lane == 0) {
                    const uint64_t t0 = ptx::globaltimer_ns();
                    while (ptx::ld_acquire_gpu(flags + sg.tile) == 0) {
                        if (*abort || ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                            ok = false;
                            break;
                        }
                    }
                    ptx::mbar_arrive(ptx::smem_u32(&sm.head_ready));
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            ok = wwait(&sm.staged[si & 1], (si >> 1) & 1);
            if (!ok) break;
            if (sg.kind == kHead) {
                // the head partial written by the softmax warps -> release flag
                if (lane == 0) ptx::st_release_gpu(flags + sg.tile, 1);
            } else {
                const uint32_t stage = ptx::smem_u32(sm.q[si & 1]);
                if (lane == 0) {
                    if (sg.kind == kTail) flags[sg.tile] = 0;  // read: clear for the next launch
                    ptx::tma_store_4d(&tm_o, stage, 0, h, qt * kBM, b);
                    ptx::tma_store_4d(&tm_o, stage + kHalfBytes, 64, h, qt * kBM, b);
                    ptx::bulk_commit_group();
                    ptx::bulk_wait_group_read0();
                }
                __syncwarp();
            }
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&sm.stage_free[si & 1]));
        }
        if (!ok) fail();
    } else if (warp >= 4) {
        // ---------------------------------------- softmax + epilogue --
        ptx::setmaxnreg_inc<kRegsHigh>();
        ptx::pdl_wait_then_trigger();
        const int wg = (warp - 4) >> 2;               // S/P buffer, O accumulator and key blocks
        const int row = ((warp & 3) << 5) + lane;     // tile row = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t sbuf = tmem + lane_base + kColS + (uint32_t)wg * kBN;
        const uint32_t obuf = tmem + lane_base + kColO + (uint32_t)wg * kD;
        int vb = 0;                  // virtual blocks so far (see the issuer)
        int kc0 = 0, vc0 = 0;        // K-ring items and P V products before this segment
        uint32_t s_par = 0;          // phase parity of s_full[wg] to wait for
        uint32_t e_uses = 0;         // completed uses of ebar
        bool ok = true;
        // One arrival per warp on the softmax barriers: the warp's lanes
        // are synchronised (and their shared-memory writes ordered) by
        // __syncwarp, then lane 0 arrives.
        auto warp_arrive = [&](uint64_t* bar) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(bar));
        };
        // all 8 softmax warps meet at ebar (arrive, then a bounded wait)
        auto meet_e = [&]() -> bool {
            warp_arrive(&sm.ebar);
            return wwait(&sm.ebar, (e_uses++) & 1);
        };
        const float2 sl2 = make_float2(scale_log2, scale_log2);
        for (int si = 0; ok && si < rng.n_segs; ++si) {
            const Seg sg = seg_at(sch, rng, si);
            const int n = sg.kv1 - sg.kv0;
            float m_run = -INFINITY, l_run = 0.f;
            // this warpgroup's blocks of the segment: j = j0, j0 + 2, ...
            const int j0 = ((vb & 1) == wg) ? 0 : 1;
            for (int j = j0; j < n; j += 2) {
                ok = wwait(&sm.s_full[wg], s_par);
                s_par ^= 1u;
                if (!ok) break;
                // S is done: the K tile it was computed from may be reloaded
                if ((warp & 3) == 0 && lane == 0) ptx::mbar_arrive(ptx::smem_u32(&sm.k_empty[(kc0 + j) & 1]));
                ptx::tc_fence_after();
                uint32_t raw[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) ptx::tmem_ld32(sbuf + (uint32_t)c * 32, raw[c]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) ptx::reg_fence(raw[c]);
                float x[128];
#pragma unroll
                for (int i = 0; i < 128; ++i) x[i] = __uint_as_float(raw[i >> 5][i & 31]);
                const int valid = block_keys(nc, L, Lc, sg.kv0 + j);
                if (valid < kBN) {
#pragma unroll
                    for (int i = 0; i < 128; ++i)
                        if (i >= valid) x[i] = -INFINITY;
                }
                // row max: 3-input max tree
                float m16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    m16[i] = ptx::max3(ptx::max3(x[8 * i], x[8 * i + 1], x[8 * i + 2]),
                                       ptx::max3(x[8 * i + 3], x[8 * i + 4], x[8 * i + 5]),
                                       fmaxf(x[8 * i + 6], x[8 * i + 7]));
                float m4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    m4[i] = ptx::max3(m16[4 * i], m16[4 * i + 1], fmaxf(m16[4 * i + 2], m16[4 * i + 3]));
                const float mx = ptx::max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
                const float m_new = fmaxf(m_run, mx * scale_log2);
                const bool need = m_new > m_run + kRescaleLog2;
                const float m_use = need ? m_new : m_run;
                const float corr = need ? ptx::ex2(m_run - m_new) : 1.f;
                const float2 nm = make_float2(-m_use, -m_use);
                float2 sum4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
                uint32_t pk[64];
                // P (bf16 pairs) over the first 64 columns of the S buffer, in
                // two halves of 64 keys, each handed to the issuer when stored.
                // A block of at most 64 keys (a frame's ragged last block) has
                // no second half: its P V reads the first half only.
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    if (hf == 1 && valid <= kBN / 2) {
                        warp_arrive(&sm.p_full[wg]);
                        continue;
                    }
#pragma unroll
                    for (int i = 32 * hf; i < 32 * hf + 32; ++i) {
                        // SFU exponentials
                        const float2 a = ptx::fma2(make_float2(x[2 * i], x[2 * i + 1]), sl2, nm);
                        float2 p;
                        p.x = ptx::ex2(a.x);
                        p.y = ptx::ex2(a.y);
                        sum4[i & 3] = ptx::add2(sum4[i & 3], p);
                        pk[i] = ptx::pack_bf16x2(p.x, p.y);
                    }
                    if (hf == 0 && j >= 2 && __any_sync(0xffffffffu, need)) {
                        // rescale O_wg before the first half's P V adds to it
                        // (after that half's exponentials, when fewer of S's
                        // registers are live): S of this block was committed
                        // after the P V of this warpgroup's previous block, so
                        // that is done
#pragma unroll 1
                        for (int c = 0; c < 4; ++c) {
                            uint32_t o[32];
                            ptx::tmem_ld32(obuf + (uint32_t)c * 32, o);
                            ptx::tmem_wait_ld();
                            ptx::reg_fence(o);
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
                            ptx::tmem_st32(obuf + (uint32_t)c * 32, o);
                        }
                    }
                    ptx::tmem_st32_u(sbuf + 32u * hf, pk + 32 * hf);
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    warp_arrive(hf == 0 ? &sm.p_half[wg] : &sm.p_full[wg]);
                }
                const float2 s2 = ptx::add2(ptx::add2(sum4[0], sum4[1]), ptx::add2(sum4[2], sum4[3]));
                l_run = l_run * corr + (s2.x + s2.y);
                m_run = m_use;
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue --
            // combine the two warpgroups' running (max, sum) of each row
            const bool has0 = n >= 2 || (vb & 1) == 0;
            const bool has1 = n >= 2 || (vb & 1) == 1;
            sm.red_m[wg][row] = m_run;
            sm.red_l[wg][row] = l_run;
            ok = meet_e();
            if (!ok) break;
            const float m0 = sm.red_m[0][row], m1 = sm.red_m[1][row];
            const float l0 = sm.red_l[0][row], l1 = sm.red_l[1][row];
            const float m_seg = fmaxf(has0 ? m0 : -INFINITY, has1 ? m1 : -INFINITY);
            const float a0 = has0 ? ptx::ex2(m0 - m_seg) : 0.f;
            const float a1 = has1 ? ptx::ex2(m1 - m_seg) : 0.f;
            const float l_seg = a0 * l0 + a1 * l1;
            // partial of (tile, column half): float4 chunk i of row r at [i][r], so
            // that the 32 lanes of a warp touch 512 consecutive bytes
            float4* pbase = reinterpret_cast<float4*>(part_o) + ((size_t)sg.tile * 2 + wg) * 16 * kBM + row;
            // A tail piece merges the head partial the previous CTA wrote at its
            // start (warp 3 acquires its flag): its 16 float4 of this thread's
            // row half are loaded now, so that their L2 latency overlaps the
            // wait for the last product and the accumulator loads.
            float4 ph[4];  // chunk 0 now; each chunk loads the next one's first
            float2 ml = make_float2(0.f, 0.f);
            if (sg.kind == kTail) {
                ok = wwait(&sm.head_ready, 0);
                if (!ok) break;
                ml = __ldcg(reinterpret_cast<const float2*>(part_ml + ((size_t)sg.tile * kBM + row) * 2));
#pragma unroll
                for (int i = 0; i < 4; ++i) ph[i] = __ldcg(pbase + (size_t)i * kBM);
            }
            // the segment's last P V: its commit covers every product before it
            ok = wwait(&sm.v_empty[(vc0 + n - 1) & 1], ((vc0 + n - 1) >> 1) & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            // this warpgroup's output columns [64 wg, 64 wg + 64) of
            // a0 O_0 + a1 O_1 (unnormalised, against m_seg)
            const uint32_t ocol = tmem + lane_base + kColO + (uint32_t)wg * 64;
            // a0 O_0 + a1 O_1 over 32 columns, and (with_oi) O_inter's, in one round trip
            auto load_acc = [&](int c, float (&acc)[32], auto with_oi, uint32_t oi_col, uint32_t (&oi)[32]) {
                // (a warpgroup without blocks in this segment left its O stale:
                // it is loaded but not used)
                uint32_t o0[32], o1[32];
                ptx::tmem_ld32(ocol + (uint32_t)c * 32, o0);
                ptx::tmem_ld32(ocol + kD + (uint32_t)c * 32, o1);
                if constexpr (decltype(with_oi)::value) ptx::tmem_ld32(oi_col + (uint32_t)c * 32, oi);
                ptx::tmem_wait_ld();
                ptx::reg_fence(o0);
                ptx::reg_fence(o1);
                if constexpr (decltype(with_oi)::value) ptx::reg_fence(oi);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float v0 = has0 ? a0 * __uint_as_float(o0[i]) : 0.f;
                    acc[i] = has1 ? fmaf(a1, __uint_as_float(o1[i]), v0) : v0;
                }
            };
            if (sg.kind == kHead) {
                // unnormalised O, running max and row sum -> partial, then the flag
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float acc[32];
                    uint32_t unused[32];
                    load_acc(c, acc, std::false_type{}, 0u, unused);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        pbase[(size_t)(c * 8 + i) * kBM] =
                            make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
                }
                if (wg == 0)
                    *reinterpret_cast<float2*>(part_ml + ((size_t)sg.tile * kBM + row) * 2) =
                        make_float2(m_seg, l_seg);
                // warp 3 publishes it: these writes happen before its release
                warp_arrive(&sm.staged[si & 1]);
            } else if (sg.kind == kTail) {
                // merge with the head partial: four chunks of 16 columns,
                // unrolled so that the preloaded partial stays in registers
                const float mm = fmaxf(ml.x, m_seg);
                const float a_h = ptx::ex2(ml.x - mm);
                const float a_t = ptx::ex2(m_seg - mm);
                const float inv_l = 1.f / (a_h * ml.y + a_t * l_seg);
                const uint32_t stage = ptx::smem_u32(sm.q[si & 1]);  // the segment's Q slot
                const uint32_t o0c = tmem + lane_base + kColO + (uint32_t)wg * 64;
                const uint32_t oi_col = tmem + lane_base + kColS + (uint32_t)((vb + n) & 1) * kBN + (uint32_t)wg * 64;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float4 pn[4];
                    if (c < 3) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) pn[i] = __ldcg(pbase + (size_t)((c + 1) * 4 + i) * kBM);
                    }
                    uint32_t o0[16], o1[16], oi[16];
                    ptx::tmem_ld16(o0c + (uint32_t)c * 16, o0);
                    ptx::tmem_ld16(o0c + kD + (uint32_t)c * 16, o1);
                    if (kInter) ptx::tmem_ld16(oi_col + (uint32_t)c * 16, oi);
                    ptx::tmem_wait_ld();
                    ptx::reg_fence16(o0);
                    ptx::reg_fence16(o1);
                    if (kInter) ptx::reg_fence16(oi);
                    float acc[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float v0 = has0 ? a0 * __uint_as_float(o0[i]) : 0.f;
                        acc[i] = (has1 ? fmaf(a1, __uint_as_float(o1[i]), v0) : v0) * a_t;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 p4 = ph[i];
                        acc[4 * i] = fmaf(a_h, p4.x, acc[4 * i]);
                        acc[4 * i + 1] = fmaf(a_h, p4.y, acc[4 * i + 1]);
                        acc[4 * i + 2] = fmaf(a_h, p4.z, acc[4 * i + 2]);
                        acc[4 * i + 3] = fmaf(a_h, p4.w, acc[4 * i + 3]);
                    }
#pragma unroll
                    for (int gq = 0; gq < 2; ++gq) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = gq * 8 + e * 2;
                            const float i0 = kInter ? __uint_as_float(oi[i]) : 0.f;
                            const float i1 = kInter ? __uint_as_float(oi[i + 1]) : 0.f;
                            w[e] = ptx::pack_bf16x2(fmaf(acc[i], inv_l, i0), fmaf(acc[i + 1], inv_l, i1));
                        }
                        ptx::st_shared_v4(stage + ptx::tile_chunk_offset(row, wg * 8 + c * 2 + gq), w[0], w[1],
                                          w[2], w[3]);
                    }
                    if (c < 3) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) ph[i] = pn[i];
                    }
                }
                ptx::fence_proxy_async_smem();
                // staged (and the partial read): warp 3 stores it
                warp_arrive(&sm.staged[si & 1]);
            } else {
                const float inv_l = 1.f / l_seg;
                const uint32_t stage = ptx::smem_u32(sm.q[si & 1]);  // the segment's Q slot
                const uint32_t oi_col = tmem + lane_base + kColS + (uint32_t)((vb + n) & 1) * kBN + (uint32_t)wg * 64;
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float acc[32];
                    uint32_t oi[32];
                    load_acc(c, acc, std::bool_constant<kInter>{}, oi_col, oi);
                    // bf16 output row chunk -> the staging tile (128-byte swizzle)
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = gq * 8 + e * 2;
                            const float i0 = kInter ? __uint_as_float(oi[i]) : 0.f;
                            const float i1 = kInter ? __uint_as_float(oi[i + 1]) : 0.f;
                            w[e] = ptx::pack_bf16x2(fmaf(acc[i], inv_l, i0), fmaf(acc[i + 1], inv_l, i1));
                        }
                        ptx::st_shared_v4(stage + ptx::tile_chunk_offset(row, wg * 8 + c * 4 + gq), w[0], w[1],
                                          w[2], w[3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                // staged (and the partial read): warp 3 stores it
                warp_arrive(&sm.staged[si & 1]);
            }
            ptx::tc_fence_before();
            warp_arrive(&sm.o_free);
            vb += seg_items<kInter>(sg);
            kc0 += seg_items<kInter>(sg);
            vc0 += n;
        }
        if (!ok) fail();
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
    int G = 0;  // CTAs the persistent grid may use
    const void* m_ptr = nullptr;
    CUtensorMap tm_m{};
    Sched sch{};  // the schedule without cached keys
    float* part_o = nullptr;
    float* part_ml = nullptr;
    int* flags = nullptr;
};

namespace {

// Tiles of 128 query rows against n_c + ceil(L / 128) key blocks.  The
// split-tile workspace depends on the tiles only, so one workspace serves
// every cache length.
Sched make_sched(const Dims& dm, int Lc, int G) {
    Sched s{};
    s.n_q = (dm.L + kBM - 1) / kBM;
    s.n_c = (Lc + kBN - 1) / kBN;
    s.n_kv = s.n_c + (dm.L + kBN - 1) / kBN;
    s.T = dm.B * dm.H * s.n_q;
    s.U = (long long)s.T * s.n_kv;
    s.split = s.T > G ? 1 : 0;
    s.G = s.split ? G : s.T;
    return s;
}

template <bool kInter>
bool kernel_ready() {
    if (cudaFuncSetAttribute(attn_tc_kernel<kInter>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    // the warpgroups' register split needs the launch count it was sized for
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, attn_tc_kernel<kInter>) != cudaSuccess || fa.numRegs != kRegsLaunch) {
        cudaGetLastError();
        return false;
    }
    return true;
}

template <bool kInter>
cudaError_t launch(const AttnTc* t, const Sched& sch, const CUtensorMap& cq, const CUtensorMap& ck,
                   const CUtensorMap& cv, const CUtensorMap& ckc, const CUtensorMap& cvc,
                   const CUtensorMap& co, int Lc, float scale, int* err, cudaStream_t st) {
    const float sl2 = scale * 1.4426950408889634f;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sch.G, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    // Programmatic dependent launch: the CTAs start (set-up only) while the
    // previous kernel drains.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_tc_kernel<kInter>, cq, ck, cv, ckc, cvc, t->tm_m, co, t->part_o,
                              t->part_ml, t->flags, t->dm.L, Lc, t->dm.H, sch, sl2, err);
}

}  // namespace

size_t attn_tc_workspace_bytes(const Dims& dm) {
    const size_t tiles = (size_t)dm.B * dm.H * ((dm.L + kBM - 1) / kBM);
    return tiles * ((size_t)kBM * kD * 4 + (size_t)kBM * 2 * 4 + 4);
}

AttnTc* attn_tc_create(Dims dm, void* workspace, int max_ctas) {
    if (dm.d != kD || dm.L < 1 || dm.H < 1 || dm.B < 1 || !tma_available() || !workspace) return nullptr;
    if (!kernel_ready<true>() || !kernel_ready<false>()) return nullptr;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
        cudaGetLastError();
        return nullptr;
    }
    AttnTc* t = new (std::nothrow) AttnTc();
    if (!t) return nullptr;
    t->dm = dm;
    t->G = max_ctas > 0 && max_ctas < sms ? max_ctas : sms;
    t->sch = make_sched(dm, 0, t->G);
    const size_t tiles = (size_t)t->sch.T;
    char* w = static_cast<char*>(workspace);
    t->part_o = reinterpret_cast<float*>(w);
    t->part_ml = reinterpret_cast<float*>(w + tiles * kBM * kD * 4);
    t->flags = reinterpret_cast<int*>(w + tiles * kBM * kD * 4 + tiles * kBM * 2 * 4);
    return t;
}

int* attn_tc_flags(AttnTc* t, size_t* count) {
    *count = (size_t)t->sch.T;
    return t->flags;
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
    CUtensorMap cq, ck, cv, co;
    if (!maps.get(q, &cq) || !maps.get(k, &ck) || !maps.get(v, &cv) || !maps.get(out, &co))
        return cudaErrorInvalidValue;
    return launch<true>(t, t->sch, cq, ck, cv, ck, cv, co, 0, scale, err, st);
}

cudaError_t attn_tc_launch_cached(AttnTc* t, TokenMapCache& maps, const void* q, const void* k,
                                  const void* v, const CUtensorMap* kc, const CUtensorMap* vc, int Lc,
                                  void* out, float scale, int* err, cudaStream_t st) {
    if (Lc < 0 || (Lc > 0 && (!kc || !vc))) return cudaErrorInvalidValue;
    CUtensorMap cq, ck, cv, co;
    if (!maps.get(q, &cq) || !maps.get(k, &ck) || !maps.get(v, &cv) || !maps.get(out, &co))
        return cudaErrorInvalidValue;
    const Sched sch = Lc > 0 ? make_sched(t->dm, Lc, t->G) : t->sch;
    return launch<false>(t, sch, cq, ck, cv, Lc > 0 ? *kc : ck, Lc > 0 ? *vc : cv, co, Lc, scale, err, st);
}

}  // namespace arl2
