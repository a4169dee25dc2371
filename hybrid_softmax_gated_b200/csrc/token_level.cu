// Token-level (sequential) state access, fp32 arithmetic.
//
// The ablation the pages compare with frame-level access ("Attend Locally,
// Remember Linearly", technical summary §2.2 "Frame-Level Access"; atlas
// summary "Surprising findings"): within the frame, token i reads the state
// left by tokens 0..i-1 and then updates it with the delta rule; the frame's
// forget gate G (alpha, or diag(alpha) per key feature) acts once, with
// token 0's update:
//   S^(0) = S_{N-1};  o_i += q'_i S^(i);
//   S^(i+1) = G_i S^(i) + beta_i k'_i^T (v'_i - k'_i S^(i)),  G_0 = G, G_i = I.
// Every pass reads through its own sequential states; only the clean pass
// keeps S^(L).
//
// Chunked form (chunks of C tokens; S_0 the state at the chunk's start, and
// G applying in chunk 0 only).  With u_j = v'_j - k'_j S^(j) for the chunk's
// tokens, S^(j) = G S_0 + sum_{i<j} beta_i k'_i^T u_i for j >= 1 gives
//   (I + A) U = V' - K~ S_0,   A[j][i] = beta_i k'_j . k'_i  (i < j),
//   k~_j = k'_j G (j >= 1, chunk 0), k~_j = k'_j otherwise,
//   o_j  += q~_j S_0 + sum_{i<j} P[j][i] u_i,  P[j][i] = beta_i q'_j . k'_i,
//   S_C  = G S_0 + (diag(beta) K')^T U.
// tl_prep_kernel forms, for every chunk independently, T K~ and T V' with
// T = (I + A)^{-1} (by forward substitution), Q~, diag(beta) K' and P; tl_scan_kernel then runs the chunks
// in order for a slice of value features (the columns of S evolve
// independently), adding the reads into out and, on the clean pass, storing
// the final state.
#include "internal.h"

namespace arl2 {
namespace {

constexpr int kTlChunk = 64;     // C
constexpr int kTlCols = 16;      // value features per scan CTA
constexpr int kTlThreads = 256;
constexpr int kPad = 4;          // row padding of [C][d] staging (bank spread)

// Row stride of [C][d] staging in shared memory: a multiple of 4 floats (for
// float4 access) plus kPad (bank spread).
__host__ __device__ inline int padded(int d) { return ((d + 3) & ~3) + kPad; }

__device__ __forceinline__ size_t tokidx(int b, int t, int h, int c, const Dims& dm) {
    return (((size_t)b * dm.L + t) * dm.H + h) * dm.d + c;
}

// Per (stream, head, chunk): [T K~ | T V' | Q~ | diag(beta) K'] each C x d,
// then P (C x C), fp32.
__host__ __device__ inline size_t tl_chunk_floats(int d) {
    return (size_t)4 * kTlChunk * d + (size_t)kTlChunk * kTlChunk;
}

__global__ void __launch_bounds__(kTlThreads) tl_prep_kernel(const float* __restrict__ qp,
                                                            const float* __restrict__ kp,
                                                            const float* __restrict__ vp,
                                                            const float* __restrict__ alpha,
                                                            int alpha_per_key,
                                                            const float* __restrict__ beta,
                                                            float* __restrict__ ws, Dims dm,
                                                            int n_chunks) {
    extern __shared__ float sm[];
    const int d = dm.d, dp = padded(d), d4 = (d + 3) / 4;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kTlChunk;
    float* Ks = sm;                       // [C][dp] k'
    float* Qs = Ks + kTlChunk * dp;       // [C][dp] q'
    float* Vs = Qs + kTlChunk * dp;       // [C][dp] v'
    float* A = Vs + kTlChunk * dp;        // [C][C]
    float* P = A + kTlChunk * kTlChunk;   // [C][C]
    float* bs = P + kTlChunk * kTlChunk;  // [C] beta
    float* gs = bs + kTlChunk;            // [d] gate of chunk 0 per key feature
    const size_t bh = (size_t)b * dm.H + h;
    for (int i = threadIdx.x; i < kTlChunk * dp; i += blockDim.x) {
        const int j = i / dp, e = i - j * dp, t = t0 + j;
        const bool ok = t < dm.L && e < d;  // (the row padding is zero: float4 dots)
        Ks[i] = ok ? kp[tokidx(b, t, h, e, dm)] : 0.f;
        Qs[i] = ok ? qp[tokidx(b, t, h, e, dm)] : 0.f;
        Vs[i] = ok ? vp[tokidx(b, t, h, e, dm)] : 0.f;
    }
    for (int j = threadIdx.x; j < kTlChunk; j += blockDim.x)
        bs[j] = t0 + j < dm.L ? beta[bh * dm.L + t0 + j] : 0.f;
    for (int e = threadIdx.x; e < d; e += blockDim.x)
        gs[e] = alpha_per_key ? alpha[bh * d + e] : alpha[bh];
    __syncthreads();
    // A[j][i] = beta_i k'_j . k'_i and P[j][i] = beta_i q'_j . k'_i for i < j
    for (int p = threadIdx.x; p < kTlChunk * kTlChunk; p += blockDim.x) {
        const int j = p / kTlChunk, i = p - j * kTlChunk;
        float a = 0.f, q = 0.f;
        if (i < j) {
            const float4* kj = reinterpret_cast<const float4*>(Ks + j * dp);
            const float4* ki = reinterpret_cast<const float4*>(Ks + i * dp);
            const float4* qj = reinterpret_cast<const float4*>(Qs + j * dp);
            for (int e4 = 0; e4 < d4; ++e4) {
                const float4 x = kj[e4], y = ki[e4], z = qj[e4];
                a = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, a))));
                q = fmaf(z.x, y.x, fmaf(z.y, y.y, fmaf(z.z, y.z, fmaf(z.w, y.w, q))));
            }
            a *= bs[i];
            q *= bs[i];
        }
        A[p] = a;
        P[p] = q;
    }
    __syncthreads();
    float* out = ws + (bh * n_chunks + c) * tl_chunk_floats(d);
    float* TK = out;
    float* TV = TK + (size_t)kTlChunk * d;
    float* QG = TV + (size_t)kTlChunk * d;
    float* BK = QG + (size_t)kTlChunk * d;
    float* Pg = BK + (size_t)kTlChunk * d;
    // T K~ and T V' with T = (I + A)^{-1}: forward substitution, one
    // right-hand-side column per thread (K~'s columns, then V''s), rows in
    // order: x_j = r_j - sum_{i<j} A[j][i] x_i.  k~_i = k'_i G for i >= 1 in
    // chunk 0.  The solutions overwrite Ks / Vs in place.
    for (int col = threadIdx.x; col < 2 * d; col += blockDim.x) {
        const bool is_k = col < d;
        const int e = is_k ? col : col - d;
        float* X = is_k ? Ks : Vs;
        const float g = (is_k && c == 0) ? gs[e] : 1.f;
        for (int j = 0; j < kTlChunk; ++j) {
            float x = X[j * dp + e];
            if (is_k && j >= 1) x *= g;
            if (is_k) BK[j * d + e] = bs[j] * X[j * dp + e];  // diag(beta) K' (before overwrite)
            for (int i = 0; i < j; ++i) x = fmaf(-A[j * kTlChunk + i], X[i * dp + e], x);
            X[j * dp + e] = x;
        }
    }
    __syncthreads();
    for (int p = threadIdx.x; p < kTlChunk * d; p += blockDim.x) {
        const int j = p / d, e = p - j * d;
        TK[p] = Ks[j * dp + e];
        TV[p] = Vs[j * dp + e];
        QG[p] = (c == 0 && j >= 1) ? Qs[j * dp + e] * gs[e] : Qs[j * dp + e];
    }
    for (int p = threadIdx.x; p < kTlChunk * kTlChunk; p += blockDim.x) Pg[p] = P[p];
}

template <typename T>
__device__ __forceinline__ float load_f(const T* p);
template <>
__device__ __forceinline__ float load_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <typename T>
__device__ __forceinline__ void store_f(T* p, float x);
template <>
__device__ __forceinline__ void store_f<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_f<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// One CTA: value features [n0, n0 + 16) of one (stream, head), all chunks in
// order.  256 threads: for U and the reads, thread = (token j, 4 features);
// for the state, thread = (key feature m, 8 features).
template <typename OutT>
__global__ void __launch_bounds__(kTlThreads) tl_scan_kernel(const float* __restrict__ ws,
                                                            float* __restrict__ S,
                                                            OutT* __restrict__ out,
                                                            const float* __restrict__ alpha,
                                                            int alpha_per_key, int clean, Dims dm,
                                                            int n_chunks) {
    extern __shared__ float sm[];
    const int d = dm.d, dp = padded(d);
    const int n0 = blockIdx.x * kTlCols, h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * dm.H + h;
    float* Ss = sm;                          // [d][16] state slice
    float* Us = Ss + d * kTlCols;            // [C][16]
    float* TKs = Us + kTlChunk * kTlCols;    // [C][dp]
    float* QGs = TKs + kTlChunk * dp;        // [C][dp]
    float* BKs = QGs + kTlChunk * dp;        // [C][dp]
    float* Ps = BKs + kTlChunk * dp;         // [C][C]
    float* TVs = Ps + kTlChunk * kTlChunk;   // [C][16]
    const int ncols = min(kTlCols, d - n0);
    float* Sg = S + bh * d * d;
    for (int i = threadIdx.x; i < d * kTlCols; i += blockDim.x) {
        const int m = i / kTlCols, n = i - m * kTlCols;
        Ss[i] = n < ncols ? Sg[(size_t)m * d + n0 + n] : 0.f;
    }
    const int j = threadIdx.x >> 2, ng = (threadIdx.x & 3) * 4;       // U / reads
    const int m_own = threadIdx.x >> 1, nh = (threadIdx.x & 1) * 8;   // state update
    for (int c = 0; c < n_chunks; ++c) {
        const float* src = ws + (bh * n_chunks + c) * tl_chunk_floats(d);
        const float* TK = src;
        const float* TV = TK + (size_t)kTlChunk * d;
        const float* QG = TV + (size_t)kTlChunk * d;
        const float* BK = QG + (size_t)kTlChunk * d;
        const float* P = BK + (size_t)kTlChunk * d;
        __syncthreads();  // the previous chunk is done with the staging buffers
        if ((d & 3) == 0) {
            // float4 loads, many in flight (the chunk's inputs come from L2)
            const int d4 = d >> 2, n4 = kTlChunk * d4;
#pragma unroll 4
            for (int i = threadIdx.x; i < n4; i += blockDim.x) {
                const int r = i / d4, e = (i - r * d4) * 4;
                const float4 x = __ldg(reinterpret_cast<const float4*>(TK) + i);
                const float4 y = __ldg(reinterpret_cast<const float4*>(QG) + i);
                const float4 z = __ldg(reinterpret_cast<const float4*>(BK) + i);
                *reinterpret_cast<float4*>(TKs + r * dp + e) = x;
                *reinterpret_cast<float4*>(QGs + r * dp + e) = y;
                *reinterpret_cast<float4*>(BKs + r * dp + e) = z;
            }
        } else {
            for (int i = threadIdx.x; i < kTlChunk * d; i += blockDim.x) {
                const int r = i / d, e = i - r * d;
                TKs[r * dp + e] = __ldg(TK + i);
                QGs[r * dp + e] = __ldg(QG + i);
                BKs[r * dp + e] = __ldg(BK + i);
            }
        }
        for (int i = threadIdx.x; i < kTlChunk * kTlChunk; i += blockDim.x) Ps[i] = __ldg(P + i);
        for (int i = threadIdx.x; i < kTlChunk * kTlCols; i += blockDim.x) {
            const int r = i / kTlCols, n = i - r * kTlCols;
            TVs[i] = n < ncols ? __ldg(TV + (size_t)r * d + n0 + n) : 0.f;
        }
        __syncthreads();
        // U = T V' - T K~ S_0 (rows j, features ng..ng+3)
        {
            float u[4] = {TVs[j * kTlCols + ng], TVs[j * kTlCols + ng + 1], TVs[j * kTlCols + ng + 2],
                          TVs[j * kTlCols + ng + 3]};
            for (int m = 0; m < d; ++m) {
                const float tk = TKs[j * dp + m];
                const float4 s = *reinterpret_cast<const float4*>(Ss + m * kTlCols + ng);
                u[0] = fmaf(-tk, s.x, u[0]);
                u[1] = fmaf(-tk, s.y, u[1]);
                u[2] = fmaf(-tk, s.z, u[2]);
                u[3] = fmaf(-tk, s.w, u[3]);
            }
            *reinterpret_cast<float4*>(Us + j * kTlCols + ng) = make_float4(u[0], u[1], u[2], u[3]);
        }
        __syncthreads();
        // reads: o_j += q~_j S_0 + sum_{i<j} P[j][i] u_i
        {
            float o[4] = {0.f, 0.f, 0.f, 0.f};
            for (int m = 0; m < d; ++m) {
                const float q = QGs[j * dp + m];
                const float4 s = *reinterpret_cast<const float4*>(Ss + m * kTlCols + ng);
                o[0] = fmaf(q, s.x, o[0]);
                o[1] = fmaf(q, s.y, o[1]);
                o[2] = fmaf(q, s.z, o[2]);
                o[3] = fmaf(q, s.w, o[3]);
            }
            for (int i = 0; i < j; ++i) {
                const float pji = Ps[j * kTlChunk + i];
                const float4 uu = *reinterpret_cast<const float4*>(Us + i * kTlCols + ng);
                o[0] = fmaf(pji, uu.x, o[0]);
                o[1] = fmaf(pji, uu.y, o[1]);
                o[2] = fmaf(pji, uu.z, o[2]);
                o[3] = fmaf(pji, uu.w, o[3]);
            }
            const int t = c * kTlChunk + j;
            if (t < dm.L) {
                for (int e = 0; e < 4; ++e) {
                    if (ng + e >= ncols) break;
                    OutT* p = out + tokidx(b, t, h, n0 + ng + e, dm);
                    store_f(p, load_f(p) + o[e]);
                }
            }
        }
        __syncthreads();  // every read of S_0 is done
        // S_C = G S_0 + (diag(beta) K')^T U   (G: the frame's gate, chunk 0 only)
        {
            if (m_own < d) {
                const float g = c == 0 ? (alpha_per_key ? alpha[bh * d + m_own] : alpha[bh]) : 1.f;
                float s[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) s[e] = g * Ss[m_own * kTlCols + nh + e];
                for (int jj = 0; jj < kTlChunk; ++jj) {
                    const float bk = BKs[jj * dp + m_own];
#pragma unroll
                    for (int e = 0; e < 8; ++e) s[e] = fmaf(bk, Us[jj * kTlCols + nh + e], s[e]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) Ss[m_own * kTlCols + nh + e] = s[e];
            }
        }
    }
    __syncthreads();
    if (clean) {
        for (int i = threadIdx.x; i < d * kTlCols; i += blockDim.x) {
            const int m = i / kTlCols, n = i - m * kTlCols;
            if (n < ncols) Sg[(size_t)m * d + n0 + n] = Ss[i];
        }
    }
}

size_t prep_smem(int d) {
    return sizeof(float) * ((size_t)3 * kTlChunk * padded(d) + 2 * kTlChunk * kTlChunk + kTlChunk + d);
}
size_t scan_smem(int d) {
    return sizeof(float) * ((size_t)d * kTlCols + kTlChunk * kTlCols + 3 * (size_t)kTlChunk * padded(d) +
                            kTlChunk * kTlChunk + kTlChunk * kTlCols);
}

}  // namespace

int tl_chunks(const Dims& dm) { return (dm.L + kTlChunk - 1) / kTlChunk; }

size_t tl_workspace_floats(const Dims& dm) {
    return (size_t)dm.B * dm.H * tl_chunks(dm) * tl_chunk_floats(dm.d);
}

cudaError_t tl_init() {
    cudaError_t e = cudaFuncSetAttribute(tl_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)prep_smem(128));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tl_scan_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)scan_smem(128));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(tl_scan_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)scan_smem(128));
}

cudaError_t launch_tl(const float* qp, const float* kp, const float* vp, const float* alpha,
                      int alpha_per_key, const float* beta, float* ws, float* S, void* out, bool bf16,
                      bool clean, Dims dm, cudaStream_t st) {
    const int nc = tl_chunks(dm);
    tl_prep_kernel<<<dim3(nc, dm.H, dm.B), kTlThreads, prep_smem(dm.d), st>>>(qp, kp, vp, alpha, alpha_per_key,
                                                                               beta, ws, dm, nc);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const dim3 grid((dm.d + kTlCols - 1) / kTlCols, dm.H, dm.B);
    if (bf16)
        tl_scan_kernel<__nv_bfloat16><<<grid, kTlThreads, scan_smem(dm.d), st>>>(
            ws, S, static_cast<__nv_bfloat16*>(out), alpha, alpha_per_key, clean ? 1 : 0, dm, nc);
    else
        tl_scan_kernel<float><<<grid, kTlThreads, scan_smem(dm.d), st>>>(
            ws, S, static_cast<float*>(out), alpha, alpha_per_key, clean ? 1 : 0, dm, nc);
    return cudaGetLastError();
}

}  // namespace arl2
