// Gate projections on the tensor cores (bf16 layers).
//
// The same reading of "learned per-token projections" (technical summary
// §2.1 "State Update") as the SIMT kernel in gates.cu: per token i and head
// h, logits a_ih = x_i . w[:, h] + b[h] and g_ih = x_i . w[:, H+h] + b[H+h];
// beta_ih = sigmoid(g_ih); alpha_h = sigmoid(mean_i a_ih).
//
// The logits are one product [L x D] . [D x 2H] per stream.  Here a CTA
// takes 128 tokens (the TMEM lanes) against the transposed weights padded to
// NP = 32, 64 or 96 outputs (tcgen05 kind::f16, M = 128, N = NP, bf16 in,
// fp32 accumulate in TMEM); its hidden features are split over a
// thread-block cluster of up to 8 CTAs, each streaming its slice of x and
// w^T through a 4-stage TMA ring.  The slices' fp32 logit tiles meet through
// distributed shared memory: rank r reads its share of the rows of every
// rank's tile (in rank order, so the sum is deterministic), adds the bias,
// writes those rows' beta and their per-head sum of alpha logits; the last
// of a stream's row groups (an atomic count) turns the sums into alpha.
//
// One CTA, 128 threads: warp 0 lane 0 issues the TMA loads, warp 1 lane 0
// the MMAs; all four warps read the accumulator (warp w: TMEM lanes
// 32w..32w+31) and run the epilogue.  Every wait on an mbarrier is bounded;
// a CTA that gives up sets the error word and still takes both cluster
// barriers, so its cluster never waits on it.
#include "internal.h"
#include "ptx.cuh"
#include "tma.h"

#include <cuda_bf16.h>

#include <new>

namespace arl2 {
namespace {

constexpr int kTM = 128;        // tokens per tile
constexpr int kKC = 64;         // hidden features per chunk (one 128-byte swizzle span)
constexpr int kStages = 4;
constexpr int kMaxSplit = 8;    // cluster size (portable bound)
constexpr int kThreads = 128;
constexpr uint64_t kWaitLimitNs = 4000000000ull;


__device__ __forceinline__ float gate_sigmoid(float z) { return 1.f / (1.f + expf(-z)); }

template <int NP>
struct __align__(1024) GSmem {
    uint8_t a[kStages][kTM * kKC * 2];  // x chunks: 128 tokens x 64 features (16 KB)
    uint8_t b[kStages][NP * kKC * 2];   // w^T chunks: NP outputs x 64 features
    uint64_t full[kStages], empty[kStages], done;
    uint32_t tmem_base;
    int abort;
    float red[kTM][NP + 4];             // this rank's rows of the summed logit tile
    int last;
};
// After the products, the fp32 logit tile [128][NP + 4] reuses the x ring.
template <int NP>
constexpr int kPartLd = NP + 4;
static_assert(kTM * (96 + 4) * 4 <= kStages * kTM * kKC * 2, "logit tile fits the x ring");

template <int NP>
__host__ __device__ constexpr uint32_t tmem_cols() {
    return NP <= 32 ? 32u : 128u;
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const float* __restrict__ bias, int L, int D, int H, float* __restrict__ beta,
                   float* __restrict__ part_a, float* __restrict__ alpha, unsigned* __restrict__ count,
                   int* __restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    GSmem<NP>& sm = *reinterpret_cast<GSmem<NP>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                  ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x, b = blockIdx.y, n_tiles = gridDim.x;
    const uint32_t rank = ptx::cluster_ctarank();
    const int n_split = gridDim.z;  // the cluster spans z
    const int nch = (D + kKC - 1) / kKC;
    const int per = (nch + n_split - 1) / n_split;
    const int c_lo = (int)rank * per;
    const int n = max(0, min(nch, c_lo + per) - c_lo);  // this rank's chunks
    volatile int* abort = &sm.abort;
    const int no_abort = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(ptx::smem_u32(&sm.full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sm.empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(&sm.done), 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(&sm.tmem_base), tmem_cols<NP>());
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    auto fail = [&]() {
        atomicOr(err, kErrTimeoutUpdate);
        *abort = 1;
    };

    constexpr uint32_t kABytes = kTM * kKC * 2, kBBytes = NP * kKC * 2;
    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------- TMA producer
        ptx::tma_prefetch_desc(&tm_x);
        ptx::tma_prefetch_desc(&tm_w);
        int issued = 0;
        for (int i = 0; i < n; ++i) {
            const int s = i % kStages;
            if (i >= kStages &&
                !ptx::mbar_wait_bounded(ptx::smem_u32(&sm.empty[s]), ((i / kStages) - 1) & 1, abort, kWaitLimitNs)) {
                fail();
                break;
            }
            const uint32_t bar = ptx::smem_u32(&sm.full[s]);
            const int c0 = (c_lo + i) * kKC;
            ptx::mbar_arrive_expect_tx(bar, kABytes + kBBytes);
            ptx::tma_load_4d(ptx::smem_u32(sm.a[s]), &tm_x, c0, tile * kTM, b, 0, bar);
            ptx::tma_load_4d(ptx::smem_u32(sm.b[s]), &tm_w, c0, 0, 0, 0, bar);
            issued = i + 1;
        }
        // every load issued has landed before the ring is reused or the CTA
        // exits (on the normal path the products already consumed them)
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
            ptx::mbar_wait_bounded(ptx::smem_u32(&sm.full[i % kStages]), (i / kStages) & 1, &no_abort, kWaitLimitNs);
    } else if (warp == 1 && lane == 0) {
        // ----------------------------------------------------- MMA issuer
        const uint32_t idesc = ptx::idesc_bf16_f32(kTM, NP, false, false);  // both K-major
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const int s = i % kStages;
            if (!ptx::mbar_wait_bounded(ptx::smem_u32(&sm.full[s]), (i / kStages) & 1, abort, kWaitLimitNs)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t as = ptx::smem_u32(sm.a[s]), bs = ptx::smem_u32(sm.b[s]);
#pragma unroll
            for (int kk = 0; kk < kKC / 16; ++kk)
                ptx::umma_f16_ss(tmem, ptx::sdesc_sw128(as + kk * 32u, 16u, 1024u),
                                 ptx::sdesc_sw128(bs + kk * 32u, 16u, 1024u), idesc, (i > 0 || kk > 0) ? 1u : 0u);
            ptx::umma_commit(ptx::smem_u32(&sm.empty[s]));
        }
        if (!ok) fail();
        // every product issued (or none): done arrives when they are complete
        ptx::umma_commit(ptx::smem_u32(&sm.done));
    }
    __syncwarp();

    // ------------------------------------------- this rank's logit tile
    const int row = threadIdx.x;  // = TMEM lane (warp w reads lanes 32w..32w+31)
    float* part = reinterpret_cast<float*>(sm.a[0]);
    const bool done_ok = ptx::mbar_wait_bounded(ptx::smem_u32(&sm.done), 0, &no_abort, kWaitLimitNs);
    if (!done_ok && threadIdx.x == 0) fail();
    ptx::tc_fence_after();
    // (the barrier below also keeps the ring's last TMA writes ordered before
    // the tile overwrites it: every load was consumed by a completed product)
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NP / 32; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c * 32, v);
        ptx::tmem_wait_ld();
        ptx::reg_fence(v);
        const bool have = n > 0 && done_ok && !*abort;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(part + row * kPartLd<NP> + c * 32 + j) =
                have ? make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                                   __uint_as_float(v[j + 3]))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // #1: every rank's tile is written

    // Rank r sums rows [R r, R r + R) of the tile (R = 128 / ranks) over
    // every rank's slice, in rank order, one group of 4 columns of one row
    // per step; a step's loads from the cluster's ranks are all in flight
    // before its adds.
    const int R = (kTM + n_split - 1) / n_split;
    const int row_lo = (int)rank * R, rows = max(0, min(kTM, row_lo + R) - row_lo);
    for (int idx = threadIdx.x; idx < rows * (NP / 4); idx += kThreads) {
        const int rr = idx / (NP / 4), g = idx - rr * (NP / 4);
        const uint32_t a = ptx::smem_u32(part + (row_lo + rr) * kPartLd<NP> + 4 * g);
        float4 t[kMaxSplit];
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q)
            if (q < n_split) t[q] = ptx::ld_shared_cluster_v4(ptx::mapa_shared(a, (uint32_t)q));
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q)
            if (q < n_split) {
                sum.x += t[q].x;
                sum.y += t[q].y;
                sum.z += t[q].z;
                sum.w += t[q].w;
            }
        *reinterpret_cast<float4*>(&sm.red[rr][4 * g]) = sum;
    }
    ptx::cluster_sync();  // #2: every remote read is done; ranks may go on alone
    __syncthreads();

    // beta of the rank's rows, and their per-head sum of alpha logits
    const int row0 = tile * kTM + row_lo;
    for (int i = threadIdx.x; i < rows * H; i += kThreads) {
        const int r = i / H, h = i - r * H;
        if (row0 + r < L) beta[((size_t)b * H + h) * L + row0 + r] = gate_sigmoid(sm.red[r][H + h] + bias[H + h]);
    }
    const int n_parts = n_tiles * n_split;
    const int part_idx = (b * n_tiles + tile) * n_split + (int)rank;
    for (int h = threadIdx.x; h < H; h += kThreads) {
        float s = 0.f;
        for (int r = 0; r < rows && row0 + r < L; ++r) s += sm.red[r][h] + bias[h];
        part_a[(size_t)part_idx * H + h] = s;
    }
    // the last of the stream's parts turns the sums into alpha
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        sm.last = atomicAdd(&count[b], 1u) == (unsigned)(n_parts - 1);
        if (sm.last) __threadfence();
    }
    __syncthreads();
    if (sm.last) {
        // thread t sums partials k = t, t + 128, ... for every head (each
        // partial's H values are contiguous), then a fixed tree over the
        // threads: the same order on every run
        float* acc = &sm.red[0][0];  // [kThreads][H] (the rows are not needed any more)
        __syncthreads();
        float s[48];
#pragma unroll
        for (int h = 0; h < 48; ++h) s[h] = 0.f;
        for (int k = threadIdx.x; k < n_parts; k += kThreads) {
            const float* p = part_a + ((size_t)b * n_parts + k) * H;
#pragma unroll
            for (int h = 0; h < 48; ++h)
                if (h < H) s[h] += __ldcg(p + h);
        }
#pragma unroll
        for (int h = 0; h < 48; ++h)
            if (h < H) acc[threadIdx.x * H + h] = s[h];
        __syncthreads();
        for (int step = kThreads / 2; step > 0; step >>= 1) {
            for (int i = threadIdx.x; i < step * H; i += kThreads) acc[i] += acc[i + step * H];
            __syncthreads();
        }
        for (int h = threadIdx.x; h < H; h += kThreads) alpha[(size_t)b * H + h] = gate_sigmoid(acc[h] / (float)L);
        if (threadIdx.x == 0) count[b] = 0;  // re-armed for the next launch
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tmem_cols<NP>());
    }
}

template <int NP>
constexpr size_t smem_bytes() {
    return sizeof(GSmem<NP>) + 1024;
}

template <int NP>
bool set_attr() {
    if (cudaFuncSetAttribute(gate_tc_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_bytes<NP>()) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return true;
}

}  // namespace

struct GateTc {
    int B = 0, L = 0, D = 0, H = 0, NP = 0, split = 1;
    CUtensorMap tm_w{};
    const void* x_ptr = nullptr;
    CUtensorMap tm_x{};
};

int gate_tc_outputs(int H) { return 2 * H <= 32 ? 32 : 2 * H <= 64 ? 64 : 96; }

int gate_part_count(int L) {
    const int simt = gate_tiles(L), tc = ((L + kTM - 1) / kTM) * kMaxSplit;
    return simt > tc ? simt : tc;
}

GateTc* gate_tc_create(int B, int L, int D, int H, const void* wt, int wt_rows) {
    if (!gate_shape_ok(D, H) || D < kKC || H > 48 || !tma_available()) return nullptr;
    const int NP = gate_tc_outputs(H);
    if (wt_rows < NP) return nullptr;
    const bool ok = NP == 32 ? set_attr<32>() : NP == 64 ? set_attr<64>() : set_attr<96>();
    if (!ok) return nullptr;
    GateTc* g = new (std::nothrow) GateTc();
    if (!g) return nullptr;
    g->B = B;
    g->L = L;
    g->D = D;
    g->H = H;
    g->NP = NP;
    const int nch = (D + kKC - 1) / kKC;
    g->split = nch < kMaxSplit ? nch : kMaxSplit;
    if (!tma_encode_rows_2d(&g->tm_w, wt, D, wt_rows, 1, NP)) {
        delete g;
        return nullptr;
    }
    return g;
}

void gate_tc_destroy(GateTc* g) { delete g; }

cudaError_t gate_tc_launch(GateTc* g, const void* x, const float* bias, float* beta, float* part_a, float* alpha,
                           unsigned* count, int* err, cudaStream_t st) {
    if (x != g->x_ptr) {
        if (!tma_encode_rows_2d(&g->tm_x, x, g->D, g->L, g->B, kTM)) return cudaErrorInvalidValue;
        g->x_ptr = x;
    }
    const int n_tiles = (g->L + kTM - 1) / kTM;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(n_tiles, g->B, g->split);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = g->split;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (g->NP) {
        case 32:
            cfg.dynamicSmemBytes = smem_bytes<32>();
            return cudaLaunchKernelEx(&cfg, gate_tc_kernel<32>, g->tm_x, g->tm_w, bias, g->L, g->D, g->H, beta,
                                      part_a, alpha, count, err);
        case 64:
            cfg.dynamicSmemBytes = smem_bytes<64>();
            return cudaLaunchKernelEx(&cfg, gate_tc_kernel<64>, g->tm_x, g->tm_w, bias, g->L, g->D, g->H, beta,
                                      part_a, alpha, count, err);
        default:
            cfg.dynamicSmemBytes = smem_bytes<96>();
            return cudaLaunchKernelEx(&cfg, gate_tc_kernel<96>, g->tm_x, g->tm_w, bias, g->L, g->D, g->H, beta,
                                      part_a, alpha, count, err);
    }
}

}  // namespace arl2
