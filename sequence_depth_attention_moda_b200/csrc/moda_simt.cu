// moda_simt.cu -- CUDA-core (fp32) forward and backward of the MoDA operator.
//
// This is the fp32 dtype path (fp32 storage and arithmetic, for tight-
// tolerance checks); the bf16 storage instantiation is kept for debugging the
// tensor-core path on the device.  One warp owns one query row (forward, dQ)
// or one key row (dK/dV); each lane holds d/32 coordinates and dot products
// are warp reductions.  Softmax statistics are base-2 with the log2(e)/sqrt(d)
// scale folded in; exp2(x) = exp(x ln 2) so the result is the same operator.
//
// Operator: paper summary of arXiv 2603.15619, "Mixture-of-Depths Attention
// (MoDA): The Unified Operator" (one softmax over causal sequence keys j <= t
// and the token's own L depth rows t*L .. t*L+L-1), online-softmax update of
// "Fused online-softmax (Algorithm 1)"; GQA head h -> KV head h / G
// ("moda-attention 0.1.0", "Key Design Choices").
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "moda_internal.h"

namespace moda {
namespace {

constexpr int kWarps = 4;             // warps per block
constexpr int kMaxPerLane = 4;        // d <= 128

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__device__ __forceinline__ void load_row(const T* p, int d, int lane, float (&x)[kMaxPerLane]) {
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int c = lane + 32 * i;
        x[i] = c < d ? to_f(p[c]) : 0.0f;
    }
}

template <typename T>
__device__ __forceinline__ float dot_row(const float (&x)[kMaxPerLane], const T* p, int d,
                                         int lane) {
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c < d) s += x[i] * to_f(p[c]);
    }
    return warp_sum(s);
}

// ---------------------------------------------------------------- forward --
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
fwd_simt_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ K,
                const T* __restrict__ V, const T* __restrict__ Kd, const T* __restrict__ Vd,
                T* __restrict__ O, float* __restrict__ LSE) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long nrows = (long long)p.B * p.Hq * p.T;
    if (row >= nrows) return;
    const int t = (int)(row % p.T);
    const int h = (int)((row / p.T) % p.Hq);
    const int b = (int)(row / ((long long)p.T * p.Hq));
    const int hk = h / p.G;
    const int d = p.d;
    const long long kv0 = ((long long)b * p.Hk + hk) * p.T;

    float q[kMaxPerLane], acc[kMaxPerLane] = {0.f, 0.f, 0.f, 0.f};
    load_row(Q + row * d, d, lane, q);
    float m = -INFINITY, l = 0.0f;
    auto visit = [&](const T* krow, const T* vrow) {
        const float s = dot_row(q, krow, d, lane) * p.scale_log2;
        const float m_new = fmaxf(m, s);
        const float alpha = exp2f(m - m_new);
        const float pr = exp2f(s - m_new);
        l = l * alpha + pr;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int c = lane + 32 * i;
            acc[i] = acc[i] * alpha + (c < d ? pr * to_f(vrow[c]) : 0.0f);
        }
        m = m_new;
    };
    const int jmax = p.causal ? t : p.T - 1;   // last visible sequence key
    for (int j = 0; j <= jmax; ++j) visit(K + (kv0 + j) * d, V + (kv0 + j) * d);
    for (int l2 = p.win_lo; l2 < p.L; ++l2) {
        const long long r = (kv0 + t) * p.L + l2;
        visit(Kd + r * d, Vd + r * d);
    }
    const float inv = 1.0f / l;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c < d) O[row * d + c] = from_f<T>(acc[i] * inv);
    }
    if (lane == 0) LSE[row] = (m + log2f(l)) * 0.6931471805599453f;
}

// ---------------------------------------------------------------- backward -
// D[row] = sum_c dO[row, c] * O[row, c]
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_rowdot_kernel(long long nrows, int d, const T* __restrict__ O, const T* __restrict__ dO,
                  float* __restrict__ D) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (row >= nrows) return;
    float s = 0.0f;
    for (int c = lane; c < d; c += 32) s += to_f(O[row * d + c]) * to_f(dO[row * d + c]);
    s = warp_sum(s);
    if (lane == 0) D[row] = s;
}

// One warp per query row: dQ over sequence keys and depth rows.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_dq_simt_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ K,
                   const T* __restrict__ V, const T* __restrict__ Kd, const T* __restrict__ Vd,
                   const float* __restrict__ LSE, const T* __restrict__ dO,
                   const float* __restrict__ D, T* __restrict__ dQ) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long nrows = (long long)p.B * p.Hq * p.T;
    if (row >= nrows) return;
    const int t = (int)(row % p.T);
    const int h = (int)((row / p.T) % p.Hq);
    const int b = (int)(row / ((long long)p.T * p.Hq));
    const int hk = h / p.G;
    const int d = p.d;
    const long long kv0 = ((long long)b * p.Hk + hk) * p.T;
    float q[kMaxPerLane], go[kMaxPerLane], dq[kMaxPerLane] = {0.f, 0.f, 0.f, 0.f};
    load_row(Q + row * d, d, lane, q);
    load_row(dO + row * d, d, lane, go);
    const float lse2 = LSE[row] * 1.4426950408889634f;
    const float Dr = D[row];
    auto visit = [&](const T* krow, const T* vrow) {
        const float pr = exp2f(dot_row(q, krow, d, lane) * p.scale_log2 - lse2);
        const float ds = pr * (dot_row(go, vrow, d, lane) - Dr);
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int c = lane + 32 * i;
            if (c < d) dq[i] += ds * to_f(krow[c]);
        }
    };
    const int jmax = p.causal ? t : p.T - 1;   // last visible sequence key
    for (int j = 0; j <= jmax; ++j) visit(K + (kv0 + j) * d, V + (kv0 + j) * d);
    for (int l2 = p.win_lo; l2 < p.L; ++l2) {
        const long long r = (kv0 + t) * p.L + l2;
        visit(Kd + r * d, Vd + r * d);
    }
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c < d) dQ[row * d + c] = from_f<T>(dq[i] * p.scale);
    }
}

// One warp per depth row (b, hk, t, l): sum over the group's G heads at token t.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_ddepth_simt_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ Kd,
                       const T* __restrict__ Vd, const float* __restrict__ LSE,
                       const T* __restrict__ dO, const float* __restrict__ D,
                       T* __restrict__ dKd, T* __restrict__ dVd) {
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long nrows = (long long)p.B * p.Hk * p.T * p.L;
    if (r >= nrows) return;
    const long long tok = r / p.L;               // (b*Hk + hk)*T + t
    const bool in_window = (int)(r - tok * p.L) >= p.win_lo;
    const int t = (int)(tok % p.T);
    const long long bh = tok / p.T;
    const int hk = (int)(bh % p.Hk);
    const int b = (int)(bh / p.Hk);
    const int d = p.d;
    float kd[kMaxPerLane], vd[kMaxPerLane];
    float dk[kMaxPerLane] = {0.f, 0.f, 0.f, 0.f}, dv[kMaxPerLane] = {0.f, 0.f, 0.f, 0.f};
    load_row(Kd + r * d, d, lane, kd);
    load_row(Vd + r * d, d, lane, vd);
    for (int g = 0; g < (in_window ? p.G : 0); ++g) {
        const long long qrow = ((long long)b * p.Hq + hk * p.G + g) * p.T + t;
        const float pr =
            exp2f(dot_row(kd, Q + qrow * d, d, lane) * p.scale_log2 - LSE[qrow] * 1.4426950408889634f);
        const float ds = pr * (dot_row(vd, dO + qrow * d, d, lane) - D[qrow]);
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int c = lane + 32 * i;
            if (c < d) {
                dk[i] += ds * to_f(Q[qrow * d + c]);
                dv[i] += pr * to_f(dO[qrow * d + c]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c < d) {
            dKd[r * d + c] = from_f<T>(dk[i] * p.scale);
            dVd[r * d + c] = from_f<T>(dv[i]);
        }
    }
}

// One warp per sequence key row (b, hk, j): every head of the group, t >= j.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_dkdv_simt_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ K,
                     const T* __restrict__ V, const float* __restrict__ LSE,
                     const T* __restrict__ dO, const float* __restrict__ D, T* __restrict__ dK,
                     T* __restrict__ dV) {
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long nrows = (long long)p.B * p.Hk * p.T;
    if (r >= nrows) return;
    const int j = (int)(r % p.T);
    const long long bh = r / p.T;
    const int hk = (int)(bh % p.Hk);
    const int b = (int)(bh / p.Hk);
    const int d = p.d;
    float k[kMaxPerLane], v[kMaxPerLane];
    float dk[kMaxPerLane] = {0.f, 0.f, 0.f, 0.f}, dv[kMaxPerLane] = {0.f, 0.f, 0.f, 0.f};
    load_row(K + r * d, d, lane, k);
    load_row(V + r * d, d, lane, v);
    for (int g = 0; g < p.G; ++g) {
        const long long q0 = ((long long)b * p.Hq + hk * p.G + g) * p.T;
        for (int t = p.causal ? j : 0; t < p.T; ++t) {
            const long long qrow = q0 + t;
            const float pr = exp2f(dot_row(k, Q + qrow * d, d, lane) * p.scale_log2 -
                                   LSE[qrow] * 1.4426950408889634f);
            const float ds = pr * (dot_row(v, dO + qrow * d, d, lane) - D[qrow]);
#pragma unroll
            for (int i = 0; i < kMaxPerLane; ++i) {
                const int c = lane + 32 * i;
                if (c < d) {
                    dk[i] += ds * to_f(Q[qrow * d + c]);
                    dv[i] += pr * to_f(dO[qrow * d + c]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c < d) {
            dK[r * d + c] = from_f<T>(dk[i] * p.scale);
            dV[r * d + c] = from_f<T>(dv[i]);
        }
    }
}

unsigned blocks_for(long long rows) { return (unsigned)((rows + kWarps - 1) / kWarps); }

template <typename T>
cudaError_t fwd_impl(const Problem& p, const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd, void* O, float* LSE, cudaStream_t s) {
    const long long rows = (long long)p.B * p.Hq * p.T;
    fwd_simt_kernel<T><<<blocks_for(rows), kWarps * 32, 0, s>>>(
        p, (const T*)Q, (const T*)K, (const T*)V, (const T*)Kd, (const T*)Vd, (T*)O, LSE);
    return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_impl(const Problem& p, const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd, const void* O, const float* LSE,
                     const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                     float* D, cudaStream_t s) {
    const long long rows = (long long)p.B * p.Hq * p.T;
    bwd_rowdot_kernel<T><<<blocks_for(rows), kWarps * 32, 0, s>>>(rows, p.d, (const T*)O,
                                                                  (const T*)dO, D);
    phase_mark(1, s);
    bwd_dq_simt_kernel<T><<<blocks_for(rows), kWarps * 32, 0, s>>>(
        p, (const T*)Q, (const T*)K, (const T*)V, (const T*)Kd, (const T*)Vd, LSE, (const T*)dO,
        D, (T*)dQ);
    const long long krows = (long long)p.B * p.Hk * p.T;
    bwd_dkdv_simt_kernel<T><<<blocks_for(krows), kWarps * 32, 0, s>>>(
        p, (const T*)Q, (const T*)K, (const T*)V, LSE, (const T*)dO, D, (T*)dK, (T*)dV);
    phase_mark(2, s);
    if (p.L > 0) {
        const long long drows = krows * p.L;
        bwd_ddepth_simt_kernel<T><<<blocks_for(drows), kWarps * 32, 0, s>>>(
            p, (const T*)Q, (const T*)Kd, (const T*)Vd, LSE, (const T*)dO, D, (T*)dKd, (T*)dVd);
    }
    phase_mark(3, s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const void* Kd, const void* Vd, void* O, float* LSE,
                            cudaStream_t stream) {
    return p.elem_bytes == 4 ? fwd_impl<float>(p, Q, K, V, Kd, Vd, O, LSE, stream)
                             : fwd_impl<__nv_bfloat16>(p, Q, K, V, Kd, Vd, O, LSE, stream);
}

cudaError_t launch_bwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const void* Kd, const void* Vd, const void* O, const float* LSE,
                            const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                            float* Dws, cudaStream_t stream) {
    return p.elem_bytes == 4
               ? bwd_impl<float>(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, Dws, stream)
               : bwd_impl<__nv_bfloat16>(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd,
                                         Dws, stream);
}

}  // namespace moda
