// Gate projections: the forget gate alpha and the per-token rates beta from
// the layer's hidden states.
//
// "Attend Locally, Remember Linearly", technical summary §2.1 ("State
// Update"): alpha and beta are learned per-token projections.  The pages
// give no form; this file computes the reading the oracle states: per token
// i and head h two logits, a_ih = x_i . w[:, h] + bias[h] and
// g_ih = x_i . w[:, H + h] + bias[H + h]; beta_ih = sigmoid(g_ih); the
// frame's forget gate alpha_h = sigmoid(mean_i a_ih) (one update per frame,
// §2.2 "Frame-Level Access"; headwise gating, §4).
//
// A skinny product, [L x D] by [D x 2H] per stream (2H = 24 at 1.3B
// scale): too narrow for the tensor cores to pay, and its 115 MFLOP per
// 480p frame take ~1.5 us of the fp32 FMA pipes against ~0.7 us to read x
// once from HBM.  SIMT, fp32 accumulation:
//   CTA = 16 tokens of one stream, 16 warps.  x and the matching rows of w
//   stream through shared memory in chunks of 256 features (128 for wide
//   outputs), double buffered (the next chunk's global loads wait in
//   registers while the current one is used), converted to fp32 once; w is
//   kept transposed, [output][feature] (zero-padded to 8U outputs, done once
//   when the weights are loaded), with padded shared-memory rows.  Warp w takes 1/16 of
//   every chunk's features; lane (tg, og) keeps a 4-token x U-output register
//   tile, so 4 features cost 4 + U shared 16-byte reads (the x reads
//   broadcast within a token group, the w reads conflict-free) for 16 U FMAs.
//   The 8 warps' partial sums meet in shared memory; the CTA writes beta
//   for its tokens and, per head, the sum of its tokens' alpha logits.  The
//   last CTA of a stream (an atomic count) sums those partials, a warp per
//   head in a fixed order (deterministic), writes alpha and re-arms the
//   count.
#include "internal.h"

#include <cuda_bf16.h>

namespace arl2 {
namespace {

constexpr int kGTok = 16;       // tokens per CTA: 4 token groups of 4
constexpr int kGWarps = 16;
constexpr int kGThreads = kGWarps * 32;
constexpr int kGMaxU = 12;      // outputs per lane: 2H <= 8 U <= 96

__device__ __forceinline__ float gate_sigmoid(float z) { return 1.f / (1.f + expf(-z)); }

// chunk of hidden features staged per step: 256, or 128 for wide outputs
// (two fp32 buffers of {x [16][C + 4], w^T [8U][C + 4]} fit in shared memory)
template <int U>
struct GateShape {
    static constexpr int kC = U <= 6 ? 256 : 128;
    static constexpr int kLd = kC + 4;                   // padded row: conflict-free 16-byte reads
    static constexpr int kO = 8 * U;                     // outputs, padded
    static constexpr int kBuf = (kGTok + kO) * kLd;      // floats per buffer
    static constexpr int kRows = kGTok + kO;             // x rows, then w^T rows
    static constexpr int kPieces = kRows * kC / 8;       // 8-element pieces of a chunk
    static constexpr int kPer = (kPieces + kGThreads - 1) / kGThreads;
    static constexpr int kSteps = kC / kGWarps / 4;      // 4-feature steps per warp and chunk
    static constexpr int kRedLd = kO + 1;
    static constexpr size_t kSmem = sizeof(float) * (2 * (size_t)kBuf);
    static_assert((size_t)kGWarps * kGTok * kRedLd <= 2 * (size_t)kBuf, "reduction fits the buffers");
};

template <typename T>
__device__ __forceinline__ void piece_load(const T* p, uint4 (&r)[2]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    r[0] = q[0];
    if (sizeof(T) == 4) r[1] = q[1];
}

__device__ __forceinline__ void piece_floats(const uint4 (&r)[2], const __nv_bfloat16*, float (&v)[8]) {
    const uint32_t w[4] = {r[0].x, r[0].y, r[0].z, r[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void piece_floats(const uint4 (&r)[2], const float*, float (&v)[8]) {
    v[0] = __uint_as_float(r[0].x); v[1] = __uint_as_float(r[0].y);
    v[2] = __uint_as_float(r[0].z); v[3] = __uint_as_float(r[0].w);
    v[4] = __uint_as_float(r[1].x); v[5] = __uint_as_float(r[1].y);
    v[6] = __uint_as_float(r[1].z); v[7] = __uint_as_float(r[1].w);
}

// Lane (tg, og) = (lane / 8, lane % 8) owns tokens 4 tg .. 4 tg + 3 and
// outputs og U .. og U + U - 1; warp w owns features [w C/16, (w+1) C/16) of
// every chunk.  Per 4 features: 4 + U shared 16-byte reads, 16 U FMAs.
// wt: the weights transposed and zero-padded, [8U][D] (gate_transpose).
template <typename T, int U>
__global__ void __launch_bounds__(kGThreads) gate_proj_kernel(
    const T* __restrict__ x, const T* __restrict__ wt, const float* __restrict__ bias, int L, int D, int H,
    float* __restrict__ beta, float* __restrict__ part_a, float* __restrict__ alpha,
    unsigned* __restrict__ count) {
    using S = GateShape<U>;
    extern __shared__ __align__(16) float gsm[];
    __shared__ float alogit[kGTok][4 * kGMaxU];  // alpha logits, heads < H <= 48
    __shared__ bool last;
    const int O = 2 * H;  // <= S::kO
    const int b = blockIdx.y, tile = blockIdx.x, n_tiles = gridDim.x;
    const int t0 = tile * kGTok;
    const int nt = min(kGTok, L - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tg = lane >> 3, og = lane & 7;
    const T* xb = x + ((size_t)b * L + t0) * D;

    uint4 rg[S::kPer][2];
    // global -> registers: piece p of the chunk at feature c0 is row
    // p / (C/8) (x rows of this tile, then w^T rows), features e..e+7;
    // zeros past D or L, so every piece of the buffer is rewritten per chunk
    auto fetch = [&](int c0) {
        const int nc = min(S::kC, D - c0);
#pragma unroll
        for (int k = 0; k < S::kPer; ++k) {
            const int p = threadIdx.x + k * kGThreads;
            const int row = p / (S::kC / 8), e = (p % (S::kC / 8)) * 8;
            rg[k][0] = rg[k][1] = make_uint4(0, 0, 0, 0);
            if (p < S::kPieces && e < nc) {
                if (row < kGTok) {
                    if (row < nt) piece_load(xb + (size_t)row * D + c0 + e, rg[k]);
                } else {
                    piece_load(wt + (size_t)(row - kGTok) * D + c0 + e, rg[k]);
                }
            }
        }
    };
    // registers -> one shared buffer, fp32
    auto stash = [&](float* buf) {
        float v[8];
#pragma unroll
        for (int k = 0; k < S::kPer; ++k) {
            const int p = threadIdx.x + k * kGThreads;
            if (p >= S::kPieces) break;
            const int row = p / (S::kC / 8), e = (p % (S::kC / 8)) * 8;
            piece_floats(rg[k], static_cast<const T*>(nullptr), v);
            float* dst = buf + row * S::kLd + e;
            *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
        }
    };

    float acc[4][U];
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int u = 0; u < U; ++u) acc[t][u] = 0.f;

    fetch(0);
    int cur = 0;
    for (int c0 = 0; c0 < D; c0 += S::kC) {
        float* buf = gsm + cur * S::kBuf;
        stash(buf);  // (its previous use ended before the last barrier)
        __syncthreads();
        if (c0 + S::kC < D) fetch(c0 + S::kC);  // in flight while this chunk is used
        const float* xs = buf + (4 * tg) * S::kLd;
        const float* ws = buf + kGTok * S::kLd + (og * U) * S::kLd;
#pragma unroll
        for (int s = 0; s < S::kSteps; ++s) {
            const int e = warp * (S::kC / kGWarps) + s * 4;
            float4 xv[4], wv[U];
#pragma unroll
            for (int t = 0; t < 4; ++t) xv[t] = *reinterpret_cast<const float4*>(xs + t * S::kLd + e);
#pragma unroll
            for (int u = 0; u < U; ++u) wv[u] = *reinterpret_cast<const float4*>(ws + u * S::kLd + e);
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float a = acc[t][u];
                    a = fmaf(xv[t].x, wv[u].x, a);
                    a = fmaf(xv[t].y, wv[u].y, a);
                    a = fmaf(xv[t].z, wv[u].z, a);
                    a = fmaf(xv[t].w, wv[u].w, a);
                    acc[t][u] = a;
                }
        }
        cur ^= 1;
    }

    // the warps' partial sums meet in shared memory (over the buffers)
    __syncthreads();
    float* red = gsm;  // [kGWarps][kGTok][kRedLd]
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int u = 0; u < U; ++u) red[(warp * kGTok + 4 * tg + t) * S::kRedLd + og * U + u] = acc[t][u];
    __syncthreads();
    for (int i = threadIdx.x; i < kGTok * O; i += kGThreads) {
        const int t = i / O, o = i - t * O;
        float z = bias[o];
#pragma unroll
        for (int k = 0; k < kGWarps; ++k) z += red[(k * kGTok + t) * S::kRedLd + o];
        if (o >= H) {
            if (t < nt) beta[((size_t)b * H + (o - H)) * L + t0 + t] = gate_sigmoid(z);
        } else {
            alogit[t][o] = z;
        }
    }
    __syncthreads();
    // per head, the sum of this tile's alpha logits (fixed order)
    for (int h = threadIdx.x; h < H; h += kGThreads) {
        float sa = 0.f;
        for (int t = 0; t < nt; ++t) sa += alogit[t][h];
        part_a[((size_t)b * n_tiles + tile) * H + h] = sa;
    }
    // the last tile of the stream turns the partial sums into alpha
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&count[b], 1u) == (unsigned)(n_tiles - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    // warp per head: lanes take tiles lane, lane + 32, ... (independent
    // loads), then a fixed shuffle tree: the same sum order on every run
    for (int h = warp; h < H; h += kGWarps) {
        float sa = 0.f;
        for (int k = lane; k < n_tiles; k += 32) sa += __ldcg(&part_a[((size_t)b * n_tiles + k) * H + h]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sa += __shfl_xor_sync(0xffffffffu, sa, off);
        if (lane == 0) alpha[(size_t)b * H + h] = gate_sigmoid(sa / (float)L);
    }
    if (threadIdx.x == 0) count[b] = 0;  // re-armed for the next launch
}

// wt[o][e] = w[e][o] for o < O, 0 for O <= o < Opad
template <typename T>
__global__ void gate_transpose_kernel(const T* __restrict__ w, T* __restrict__ wt, int D, int O, int Opad) {
    const size_t n = (size_t)Opad * D;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int o = (int)(i / D), e = (int)(i - (size_t)o * D);
        wt[i] = o < O ? w[(size_t)e * O + o] : T(0.f);
    }
}

template <int U>
cudaError_t gate_attr() {
    const int mx = (int)GateShape<U>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(gate_proj_kernel<__nv_bfloat16, U>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gate_proj_kernel<float, U>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    return e;
}

template <int U>
void gate_launch(bool bf16, dim3 grid, cudaStream_t st, const void* x, const void* wt, const float* bias, int L,
                 int D, int H, float* beta, float* part_a, float* alpha, unsigned* count) {
    const size_t smem = GateShape<U>::kSmem;
    if (bf16)
        gate_proj_kernel<__nv_bfloat16, U><<<grid, kGThreads, smem, st>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(wt), bias, L, D, H, beta,
            part_a, alpha, count);
    else
        gate_proj_kernel<float, U><<<grid, kGThreads, smem, st>>>(static_cast<const float*>(x),
                                                                  static_cast<const float*>(wt), bias, L, D, H,
                                                                  beta, part_a, alpha, count);
}

// the instantiated widths: U = outputs per lane, 2H rounded up to 8 U
constexpr int kUs[] = {1, 2, 3, 4, 6, 8, 12};
int pick_u(int H) {
    for (int u : kUs)
        if (2 * H <= 8 * u) return u;
    return 0;
}

}  // namespace

int gate_tiles(int L) { return (L + kGTok - 1) / kGTok; }

bool gate_shape_ok(int D, int H) { return D >= 8 && D % 8 == 0 && H >= 1 && 2 * H <= 8 * kGMaxU; }

int gate_padded_outputs(int H) {
    // rows of the transposed weights: the SIMT tile's 8U, and the 32-row
    // multiple the tensor-core kernel reads (both zero past 2H)
    const int simt = 8 * pick_u(H), tc = gate_tc_outputs(H);
    return simt > tc ? simt : tc;
}

cudaError_t launch_gate_transpose(bool bf16, const void* w, void* wt, int D, int H, cudaStream_t st) {
    const int O = 2 * H, Opad = gate_padded_outputs(H);
    const size_t n = (size_t)Opad * D;
    const unsigned grid = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    if (bf16)
        gate_transpose_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w),
                                                                   static_cast<__nv_bfloat16*>(wt), D, O, Opad);
    else
        gate_transpose_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(w), static_cast<float*>(wt), D,
                                                           O, Opad);
    return cudaGetLastError();
}

cudaError_t gate_init() {
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = gate_attr<1>();
    if (e == cudaSuccess) e = gate_attr<2>();
    if (e == cudaSuccess) e = gate_attr<3>();
    if (e == cudaSuccess) e = gate_attr<4>();
    if (e == cudaSuccess) e = gate_attr<6>();
    if (e == cudaSuccess) e = gate_attr<8>();
    if (e == cudaSuccess) e = gate_attr<12>();
    if (e != cudaSuccess) cudaGetLastError();
    return e;
}

cudaError_t launch_gate_proj(bool bf16, const void* x, const void* wt, const float* bias, int B, int L, int D,
                             int H, float* beta, float* part_a, float* alpha, unsigned* count,
                             cudaStream_t st) {
    const dim3 grid(gate_tiles(L), B);
    switch (pick_u(H)) {
        case 1: gate_launch<1>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        case 2: gate_launch<2>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        case 3: gate_launch<3>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        case 4: gate_launch<4>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        case 6: gate_launch<6>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        case 8: gate_launch<8>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        case 12: gate_launch<12>(bf16, grid, st, x, wt, bias, L, D, H, beta, part_a, alpha, count); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace arl2
