// SIMT kernels of the ARL2 layer, fp32 arithmetic on fp32 or bf16 storage.
//
// These carry the fp32 workloads (whose 1e-4 tolerance no bf16/tf32 tensor
// core operand can meet) and serve as an independent GPU cross-check of the
// tensor-core kernels.  Steps ("Attend Locally, Remember Linearly",
// technical summary §2.1 and §2.2):
//   phi      x' = x W[h] (+ row L2 norm for k')          §2.1 Adaptation
//   attn     softmax(Q K^T s) V + (Q W_q) S_{N-1}          §2.1 items 1-2, Output
//   residual r = v' - k' S_{N-1}                           §2.1 State Update
//   accum    S = alpha S + k'^T diag(beta) r               §2.1 State Update
#include "internal.h"

#include <cmath>

namespace arl2 {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ size_t tok(int b, int t, int h, int c, const Dims& dm) {
    return (((size_t)b * dm.L + t) * dm.H + h) * dm.d + c;
}

// ---------------------------------------------------------------- phi ----
// One CTA: 128 tokens of one (b, h); 256 threads, thread (rg, cg) computes
// rows 8 rg .. 8 rg + 7 and columns 8 cg .. 8 cg + 7 of x W[h] from W and
// the token rows staged in shared memory (fp32), then the optional row
// L2 norm (the 16 threads of a row group hold a whole row: half a warp).
constexpr int kPhiRows = 128;
constexpr int kPhiThreads = 256;

template <typename T>
__device__ __forceinline__ void store8(T* p, const float* y, bool full, int n);
template <>
__device__ __forceinline__ void store8<float>(float* p, const float* y, bool full, int n) {
    if (full) {
        reinterpret_cast<float4*>(p)[0] = make_float4(y[0], y[1], y[2], y[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
        for (int e = 0; e < n; ++e) p[e] = y[e];
    }
}
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float* y, bool full, int n) {
    if (full) {
        uint4 u;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]), h3 = __floats2bfloat162_rn(y[6], y[7]);
        u.x = *reinterpret_cast<uint32_t*>(&h0);
        u.y = *reinterpret_cast<uint32_t*>(&h1);
        u.z = *reinterpret_cast<uint32_t*>(&h2);
        u.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(p) = u;
    } else {
        for (int e = 0; e < n; ++e) p[e] = __float2bfloat16_rn(y[e]);
    }
}

template <typename T>
__global__ void __launch_bounds__(kPhiThreads) phi_simt_kernel(const T* __restrict__ x,
                                                               const T* __restrict__ w, int l2norm,
                                                               float* __restrict__ out_f,
                                                               T* __restrict__ out_t, Dims dm) {
    extern __shared__ float sm[];
    const int d = dm.d;
    float* Ws = sm;                 // [d][128]
    float* Xs = Ws + d * 128;       // [kPhiRows][d]
    const int h = blockIdx.y, b = blockIdx.z;
    const int t0 = blockIdx.x * kPhiRows;
    const int nt = min(kPhiRows, dm.L - t0);
    for (int i = threadIdx.x; i < d * 128; i += blockDim.x) {
        const int a = i >> 7, c = i & 127;
        Ws[i] = c < d ? to_f(w[((size_t)h * d + a) * d + c]) : 0.f;
    }
    for (int i = threadIdx.x; i < kPhiRows * d; i += blockDim.x) {
        const int r = i / d, c = i - r * d;
        Xs[i] = r < nt ? to_f(x[tok(b, t0 + r, h, c, dm)]) : 0.f;
    }
    __syncthreads();
    const int rg = threadIdx.x >> 4, cg = threadIdx.x & 15;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[i][jj] = 0.f;
    for (int a = 0; a < d; ++a) {
        float xr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) xr[i] = Xs[(rg * 8 + i) * d + a];
        const float4 w0 = *reinterpret_cast<const float4*>(Ws + a * 128 + cg * 8);
        const float4 w1 = *reinterpret_cast<const float4*>(Ws + a * 128 + cg * 8 + 4);
        const float wc[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) acc[i][jj] = fmaf(xr[i], wc[jj], acc[i][jj]);
    }
    const int c0 = cg * 8;
    const int ncol = max(0, min(8, d - c0));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float inv = 1.f;
        if (l2norm) {
            float ss = 0.f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) ss = fmaf(acc[i][jj], acc[i][jj], ss);
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            inv = 1.f / fmaxf(sqrtf(ss), 1e-6f);
        }
        const int r = rg * 8 + i;
        if (r >= nt || ncol == 0) continue;
        float y[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) y[jj] = acc[i][jj] * inv;
        const size_t o = tok(b, t0 + r, h, c0, dm);
        const bool full = ncol == 8 && (d & 7) == 0;
        if (out_f) store8<float>(out_f + o, y, full, ncol);
        else store8<T>(out_t + o, y, full, ncol);
    }
}

// --------------------------------------------------------------- attn ----
// One block: 32 query rows of one (b, h); 256 threads, thread (r, g) with
// r = tid / 8 owns output columns g, g+8, g+16, ... of row r.  Keys stream
// through shared memory 32 at a time with an online softmax: first the Lc
// keys of a KV cache (kc, vc: [B][cap][H][d], the softmax teacher layer),
// then the frame's own L.  S == nullptr: no inter-frame read.
constexpr int kAQ = 32, kAK = 32, kAThreads = 256, kAColsPerThread = 16;

template <typename T>
__global__ void __launch_bounds__(kAThreads) attn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ kc, const T* __restrict__ vc, int Lc, long long cap,
    const float* __restrict__ qp, const float* __restrict__ S, T* __restrict__ out,
    float scale_log2, Dims dm) {
    extern __shared__ float sm[];
    const int d = dm.d;
    float* Qs = sm;                    // [kAQ][d]
    float* Ks = Qs + kAQ * d;          // [kAK][d + 1]
    float* Vs = Ks + kAK * (d + 1);    // [kAK][d]
    float* Ps = Vs + kAK * d;          // [kAQ][kAK + 1]
    float* Ss = Ps + kAQ * (kAK + 1);  // [d][d]
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * kAQ;
    const int nq = min(kAQ, dm.L - q0);
    const int tid = threadIdx.x, r = tid >> 3, g = tid & 7;

    for (int i = tid; i < kAQ * d; i += kAThreads) {
        const int rr = i / d, c = i - rr * d;
        Qs[i] = rr < nq ? to_f(q[tok(b, q0 + rr, h, c, dm)]) : 0.f;
    }
    float o[kAColsPerThread];
#pragma unroll
    for (int i = 0; i < kAColsPerThread; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int Lk = Lc + dm.L;
    for (int k0 = 0; k0 < Lk; k0 += kAK) {
        const int nk = min(kAK, Lk - k0);
        __syncthreads();  // previous tile fully consumed (and Qs written)
        for (int i = tid; i < kAK * d; i += kAThreads) {
            const int j = i / d, c = i - j * d;
            const int t = k0 + j;
            float kx = 0.f, vx = 0.f;
            if (j < nk && t < Lc) {
                const size_t o = (((size_t)b * cap + t) * dm.H + h) * d + c;
                kx = to_f(kc[o]);
                vx = to_f(vc[o]);
            } else if (j < nk) {
                kx = to_f(k[tok(b, t - Lc, h, c, dm)]);
                vx = to_f(v[tok(b, t - Lc, h, c, dm)]);
            }
            Ks[j * (d + 1) + c] = kx;
            Vs[j * d + c] = vx;
        }
        __syncthreads();
        float s[4];
        float tmax = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = g * 4 + jj;
            float dot = 0.f;
            for (int a = 0; a < d; ++a) dot = fmaf(Qs[r * d + a], Ks[j * (d + 1) + a], dot);
            s[jj] = j < nk ? dot * scale_log2 : -INFINITY;
            tmax = fmaxf(tmax, s[jj]);
        }
        for (int off = 1; off < 8; off <<= 1)
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
        const float m_new = fmaxf(m, tmax);
        const float corr = exp2f(m - m_new);
        float psum = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const float p = exp2f(s[jj] - m_new);
            Ps[r * (kAK + 1) + g * 4 + jj] = p;
            psum += p;
        }
        for (int off = 1; off < 8; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l = l * corr + psum;
        m = m_new;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kAColsPerThread; ++i) o[i] *= corr;
        for (int j = 0; j < nk; ++j) {
            const float p = Ps[r * (kAK + 1) + j];
#pragma unroll
            for (int i = 0; i < kAColsPerThread; ++i) {
                const int c = g + 8 * i;
                if (c < d) o[i] = fmaf(p, Vs[j * d + c], o[i]);
            }
        }
    }
    const float inv_l = 1.f / l;
    if (!S) {
        if (r < nq) {
#pragma unroll
            for (int i = 0; i < kAColsPerThread; ++i) {
                const int c = g + 8 * i;
                if (c < d) out[tok(b, q0 + r, h, c, dm)] = from_f<T>(o[i] * inv_l);
            }
        }
        return;
    }
    __syncthreads();
    // inter-frame read: (q W_q) S with the pre-update state
    const float* Sbh = S + ((size_t)b * dm.H + h) * d * d;
    for (int i = tid; i < d * d; i += kAThreads) Ss[i] = Sbh[i];
    for (int i = tid; i < kAQ * d; i += kAThreads) {
        const int rr = i / d, c = i - rr * d;
        Qs[i] = rr < nq ? qp[tok(b, q0 + rr, h, c, dm)] : 0.f;
    }
    __syncthreads();
    if (r < nq) {
#pragma unroll
        for (int i = 0; i < kAColsPerThread; ++i) {
            const int c = g + 8 * i;
            if (c >= d) continue;
            float acc = 0.f;
            for (int a = 0; a < d; ++a) acc = fmaf(Qs[r * d + a], Ss[a * d + c], acc);
            out[tok(b, q0 + r, h, c, dm)] = from_f<T>(o[i] * inv_l + acc);
        }
    }
}

// ----------------------------------------------------------- residual ----
constexpr int kRRows = 32;

__global__ void __launch_bounds__(128) residual_simt_kernel(const float* __restrict__ kp,
                                                            float* __restrict__ vr,
                                                            const float* __restrict__ S, Dims dm) {
    extern __shared__ float sm[];
    const int d = dm.d;
    float* Ss = sm;          // [d][d]
    float* Kt = Ss + d * d;  // [kRRows][d]
    const int h = blockIdx.y, b = blockIdx.z;
    const int t0 = blockIdx.x * kRRows;
    const int nt = min(kRRows, dm.L - t0);
    const float* Sbh = S + ((size_t)b * dm.H + h) * d * d;
    for (int i = threadIdx.x; i < d * d; i += blockDim.x) Ss[i] = Sbh[i];
    for (int i = threadIdx.x; i < nt * d; i += blockDim.x) {
        const int rr = i / d, c = i - rr * d;
        Kt[i] = kp[tok(b, t0 + rr, h, c, dm)];
    }
    __syncthreads();
    const int n = threadIdx.x;
    if (n >= d) return;
    for (int rr = 0; rr < nt; ++rr) {
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(Kt[rr * d + c], Ss[c * d + n], acc);
        const size_t o = tok(b, t0 + rr, h, n, dm);
        vr[o] = vr[o] - acc;
    }
}

// -------------------------------------------------------------- accum ----
constexpr int kCRows = 8;

__global__ void __launch_bounds__(128) accum_simt_kernel(const float* __restrict__ kp,
                                                         const float* __restrict__ r,
                                                         const float* __restrict__ alpha,
                                                         int alpha_per_key,
                                                         const float* __restrict__ beta,
                                                         float* __restrict__ S, Dims dm) {
    const int d = dm.d;
    const int h = blockIdx.y, b = blockIdx.z;
    const int c0 = blockIdx.x * kCRows;
    const int n = threadIdx.x;
    if (n >= d) return;
    float acc[kCRows];
#pragma unroll
    for (int i = 0; i < kCRows; ++i) acc[i] = 0.f;
    const float* bt = beta + ((size_t)b * dm.H + h) * dm.L;
    for (int t = 0; t < dm.L; ++t) {
        const float rb = bt[t] * r[tok(b, t, h, n, dm)];
        const float* krow = kp + tok(b, t, h, 0, dm);
#pragma unroll
        for (int i = 0; i < kCRows; ++i)
            if (c0 + i < d) acc[i] = fmaf(krow[c0 + i], rb, acc[i]);
    }
    // headwise: one gate for the head; elementwise: one per key feature c
    const float* a_bh = alpha + ((size_t)b * dm.H + h) * (alpha_per_key ? d : 1);
    float* Sbh = S + ((size_t)b * dm.H + h) * d * d;
#pragma unroll
    for (int i = 0; i < kCRows; ++i) {
        const int c = c0 + i;
        if (c < d) Sbh[c * d + n] = fmaf(a_bh[alpha_per_key ? c : 0], Sbh[c * d + n], acc[i]);
    }
}


template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Dynamic shared memory of each kernel at the largest head_dim (128).
constexpr size_t kPhiSmemMax = sizeof(float) * (128 * 128 + kPhiRows * 128);
constexpr size_t kAttnSmemMax =
    sizeof(float) * (kAQ * 128 + kAK * 129 + kAK * 128 + kAQ * (kAK + 1) + 128 * 128);
constexpr size_t kResidualSmemMax = sizeof(float) * (128 * 128 + kRRows * 128);

}  // namespace

cudaError_t simt_init() {
    cudaError_t e;
    if ((e = set_smem(phi_simt_kernel<float>, kPhiSmemMax)) != cudaSuccess) return e;
    if ((e = set_smem(phi_simt_kernel<__nv_bfloat16>, kPhiSmemMax)) != cudaSuccess) return e;
    if ((e = set_smem(attn_simt_kernel<float>, kAttnSmemMax)) != cudaSuccess) return e;
    if ((e = set_smem(attn_simt_kernel<__nv_bfloat16>, kAttnSmemMax)) != cudaSuccess) return e;
    return set_smem(residual_simt_kernel, kResidualSmemMax);
}

cudaError_t launch_phi_simt(bool bf16, const void* x, const void* w, bool l2norm, float* out_f,
                            void* out_t, Dims dm, cudaStream_t st) {
    const size_t smem = sizeof(float) * ((size_t)dm.d * 128 + (size_t)kPhiRows * dm.d);
    const dim3 grid((dm.L + kPhiRows - 1) / kPhiRows, dm.H, dm.B);
    if (bf16) {
        phi_simt_kernel<__nv_bfloat16><<<grid, kPhiThreads, smem, st>>>(
            (const __nv_bfloat16*)x, (const __nv_bfloat16*)w, l2norm, out_f, (__nv_bfloat16*)out_t, dm);
    } else {
        phi_simt_kernel<float><<<grid, kPhiThreads, smem, st>>>((const float*)x, (const float*)w, l2norm, out_f,
                                     (float*)out_t, dm);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------ self-test ----
__global__ void selftest_wait_kernel(const int* __restrict__ flag, unsigned long long limit_ns, int* err) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v != 0) return;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > limit_ns) {
            atomicOr(err, kErrTimeoutAttn);
            return;
        }
    }
}

cudaError_t launch_selftest_wait(const int* flag, unsigned long long limit_ns, int* err, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(flag, limit_ns, err);
    return cudaGetLastError();
}

cudaError_t launch_attn_simt_cached(bool bf16, const void* q, const void* k, const void* v,
                                    const void* kc, const void* vc, int Lc, long long cap,
                                    const float* qp, const float* S, void* out, float scale, Dims dm,
                                    cudaStream_t st) {
    const int d = dm.d;
    const size_t smem = sizeof(float) * ((size_t)kAQ * d + (size_t)kAK * (d + 1) +
                                         (size_t)kAK * d + (size_t)kAQ * (kAK + 1) + (size_t)d * d);
    const dim3 grid((dm.L + kAQ - 1) / kAQ, dm.H, dm.B);
    const float scale_log2 = scale * 1.4426950408889634f;
    if (bf16) {
        attn_simt_kernel<__nv_bfloat16><<<grid, kAThreads, smem, st>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)kc,
            (const __nv_bfloat16*)vc, Lc, cap, qp, S, (__nv_bfloat16*)out, scale_log2, dm);
    } else {
        attn_simt_kernel<float><<<grid, kAThreads, smem, st>>>((const float*)q, (const float*)k, (const float*)v,
                                                               (const float*)kc, (const float*)vc, Lc, cap, qp, S,
                                                               (float*)out, scale_log2, dm);
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_simt(bool bf16, const void* q, const void* k, const void* v,
                             const float* qp, const float* S, void* out, float scale, Dims dm,
                             cudaStream_t st) {
    return launch_attn_simt_cached(bf16, q, k, v, nullptr, nullptr, 0, 0, qp, S, out, scale, dm, st);
}

cudaError_t launch_residual_simt(const float* kp, float* vp_to_r, const float* S, Dims dm,
                                 cudaStream_t st) {
    const size_t smem = sizeof(float) * ((size_t)dm.d * dm.d + (size_t)kRRows * dm.d);
    const dim3 grid((dm.L + kRRows - 1) / kRRows, dm.H, dm.B);
    residual_simt_kernel<<<grid, 128, smem, st>>>(kp, vp_to_r, S, dm);
    return cudaGetLastError();
}

cudaError_t launch_accum_simt(const float* kp, const float* r, const float* alpha, int alpha_per_key,
                              const float* beta, float* S, Dims dm, cudaStream_t st) {
    const dim3 grid((dm.d + kCRows - 1) / kCRows, dm.H, dm.B);
    accum_simt_kernel<<<grid, 128, 0, st>>>(kp, r, alpha, alpha_per_key, beta, S, dm);
    return cudaGetLastError();
}


}  // namespace arl2
