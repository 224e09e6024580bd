// moda_decode.cu -- MoDA decoding: one new token per sequence against a
// cached sequence of T keys plus the token's own L depth rows.
//
// Operator: paper summary of arXiv 2603.15619, "Mixture-of-Depths Attention
// (MoDA): The Unified Operator" -- the query at the newest position sees every
// cached key (the causal mask admits all of them) and its own depth rows,
// under one softmax scaled by 1/sqrt(d); "Complexity Analysis" (Table 1)
// gives the decoding cost O(L*T*D + L^2*D) per token across layers.
//
// Decoding reads each cached K/V row once for only the G query heads of its
// group, so it is bound by HBM bandwidth, not by math: the kernels run on the
// CUDA cores.  Split-K over the keys:
//  1. decode_split_kernel: CTA (split, b*Hk + hk), 8 warps.  Split s covers
//     keys [s*kps, (s+1)*kps); one extra split (when L > 0) covers the depth
//     rows.  A warp takes 32 keys at a time: lane = key for the G scores
//     (q, pre-scaled to base 2, read from shared memory by broadcast), an
//     online softmax per head across the warp, then lane = head dimensions
//     for P V (each key's weight broadcast by shuffle).  Every warp writes
//     its partial (m, l, o) to the workspace.
//  2. decode_combine_kernel: one CTA per query head merges the partials:
//     o = sum_i o_i 2^(m_i - M) / sum_i l_i 2^(m_i - M), LSE = (M + log2 l) ln 2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "moda_internal.h"
#include "moda_ptx.cuh"

namespace moda {
namespace {

using namespace ptx;

constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;

struct DecArgs {
    const void* q;      // [B, Hq, D]
    const void* K;      // [B, Hk, T, D] cached keys
    const void* V;
    const void* Kd;     // [B, Hk, L, D] depth rows of the new token
    const void* Vd;
    float* part;        // [B*Hq][n_part][D + 2]: m (base 2), l, o[D]
    int B, Hq, Hk, T, L, G, win_lo;
    int n_seq_split, kps, n_part;
    float scale_log2;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// 8 consecutive elements starting at element 8*c of a row.
__device__ __forceinline__ void load8(const __nv_bfloat16* row, int c, float* v) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* row, int c, float* v) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row) + 2 * c);
    const float4 b = __ldg(reinterpret_cast<const float4*>(row) + 2 * c + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// N consecutive elements (N = 2 or 4) at `p`.
template <int N>
__device__ __forceinline__ void loadn(const __nv_bfloat16* p, float* v) {
    if (N == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else {
        const unsigned int u = __ldg(reinterpret_cast<const unsigned int*>(p));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        v[0] = a.x; v[1] = a.y;
    }
}
template <int N>
__device__ __forceinline__ void loadn(const float* p, float* v) {
    if (N == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
        const float2 a = __ldg(reinterpret_cast<const float2*>(p));
        v[0] = a.x; v[1] = a.y;
    }
}

// Raw V row slice of one lane (NDL elements), kept packed until used.
template <typename E, int N> struct VRaw;
template <> struct VRaw<__nv_bfloat16, 4> {
    uint2 u;
    __device__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint2*>(p)); }
    __device__ void get(float* v) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    }
};
template <> struct VRaw<__nv_bfloat16, 2> {
    unsigned int u;
    __device__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const unsigned int*>(p)); }
    __device__ void get(float* v) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        v[0] = a.x; v[1] = a.y;
    }
};

#ifndef MODA_DEC_PREFETCH_V
#define MODA_DEC_PREFETCH_V 1
#endif

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename E, int D, int GMAX>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecArgs a) {
    constexpr int NDL = D / 32;                   // head dimensions per lane in P V
    __shared__ __align__(16) float qs[GMAX * D];
    const int split = static_cast<int>(blockIdx.x);
    const int bh = static_cast<int>(blockIdx.y);
    const int b = bh / a.Hk;
    const int hk = bh - b * a.Hk;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const E* q = static_cast<const E*>(a.q) + (static_cast<size_t>(b) * a.Hq + hk * a.G) * D;
    for (int i = threadIdx.x; i < GMAX * D; i += kDecThreads) {
        const int g = i / D;
        qs[i] = g < a.G ? to_f(q[i]) * a.scale_log2 : 0.0f;
    }
    __syncthreads();

    const bool dep = split == a.n_seq_split;      // the depth split (only when L > 0)
    const E* kb;
    const E* vb;
    int k0, k1;
    if (!dep) {
        kb = static_cast<const E*>(a.K) + static_cast<size_t>(bh) * a.T * D;
        vb = static_cast<const E*>(a.V) + static_cast<size_t>(bh) * a.T * D;
        k0 = split * a.kps;
        k1 = min(a.T, k0 + a.kps);
    } else {
        kb = static_cast<const E*>(a.Kd) + static_cast<size_t>(bh) * a.L * D;
        vb = static_cast<const E*>(a.Vd) + static_cast<size_t>(bh) * a.L * D;
        k0 = a.win_lo;
        k1 = a.L;
    }

    float m[GMAX], l[GMAX], o[GMAX][NDL];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int e = 0; e < NDL; ++e) o[g][e] = 0.0f;
    }
    // bf16 tiles of 32 keys load their V rows (lane = head dimensions) before
    // the scores, so that latency overlaps the score work
    constexpr bool kPre = MODA_DEC_PREFETCH_V && sizeof(E) == 2;
    using VR = VRaw<__nv_bfloat16, NDL>;
    for (int kt = k0 + warp * 32; kt < k1; kt += 32 * kDecWarps) {
        const int nk = min(32, k1 - kt);
        const E* vt = vb + static_cast<size_t>(kt) * D + lane * NDL;
        VR vpre[kPre ? 32 : 1];
        if (kPre && nk == 32) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
                vpre[jj].load(reinterpret_cast<const __nv_bfloat16*>(vt + static_cast<size_t>(jj) * D));
        }
        // scores of this lane's key for the G heads (base 2)
        const int key = kt + lane;
        const bool valid = key < k1;
        float s[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) s[g] = 0.0f;
        if (valid) {
            const E* kr = kb + static_cast<size_t>(key) * D;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                float kv[8];
                load8(kr, c, kv);
#pragma unroll
                for (int g = 0; g < GMAX; ++g) {
                    const float4 qa = *reinterpret_cast<const float4*>(&qs[g * D + 8 * c]);
                    const float4 qb = *reinterpret_cast<const float4*>(&qs[g * D + 8 * c + 4]);
                    s[g] = fmaf(qa.x, kv[0], s[g]); s[g] = fmaf(qa.y, kv[1], s[g]);
                    s[g] = fmaf(qa.z, kv[2], s[g]); s[g] = fmaf(qa.w, kv[3], s[g]);
                    s[g] = fmaf(qb.x, kv[4], s[g]); s[g] = fmaf(qb.y, kv[5], s[g]);
                    s[g] = fmaf(qb.z, kv[6], s[g]); s[g] = fmaf(qb.w, kv[7], s[g]);
                }
            }
        }
        // online softmax per head across the warp's 32 keys (lane 0's key is
        // always valid, so the tile maximum is finite)
        float p[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            const float sg = valid ? s[g] : -INFINITY;
            const float mn = fmaxf(m[g], warp_max(sg));
            const float alpha = ex2(m[g] - mn);
            p[g] = valid ? ex2(sg - mn) : 0.0f;
            l[g] = l[g] * alpha + warp_sum(p[g]);
            m[g] = mn;
#pragma unroll
            for (int e = 0; e < NDL; ++e) o[g][e] *= alpha;
        }
        // O += P V with lane = head dimensions [NDL*lane, NDL*lane + NDL)
        auto accumulate = [&](int jj, const float* vv) {
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                const float pj = __shfl_sync(0xffffffffu, p[g], jj);
#pragma unroll
                for (int e = 0; e < NDL; ++e) o[g][e] = fmaf(pj, vv[e], o[g][e]);
            }
        };
        if (kPre && nk == 32) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                float vv[NDL];
                vpre[jj].get(vv);
                accumulate(jj, vv);
            }
        } else if (nk == 32) {           // full tile: several V rows in flight
#pragma unroll 8
            for (int jj = 0; jj < 32; ++jj) {
                float vv[NDL];
                loadn<NDL>(vt + static_cast<size_t>(jj) * D, vv);
                accumulate(jj, vv);
            }
        } else {
            for (int jj = 0; jj < nk; ++jj) {
                float vv[NDL];
                loadn<NDL>(vt + static_cast<size_t>(jj) * D, vv);
                accumulate(jj, vv);
            }
        }
    }
    // this warp's partial for each head of the group
    const int slot = split * kDecWarps + warp;
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
        if (g < a.G) {
            float* pr = a.part + ((static_cast<size_t>(b) * a.Hq + hk * a.G + g) * a.n_part + slot) * (D + 2);
            if (lane == 0) {
                pr[0] = m[g];
                pr[1] = l[g];
            }
#pragma unroll
            for (int e = 0; e < NDL; ++e) pr[2 + lane * NDL + e] = o[g][e];
        }
    }
}

__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// One CTA (D threads) per query head: merge the n_part partials.
template <typename E, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ part, int n_part,
                                                            E* __restrict__ out, float* __restrict__ lse) {
    const size_t row = blockIdx.x;
    const float* pr = part + row * n_part * (D + 2);
    float M = -INFINITY;
    for (int i = 0; i < n_part; ++i) M = fmaxf(M, pr[i * (D + 2)]);
    float l = 0.0f, acc = 0.0f;
    for (int i = 0; i < n_part; ++i) {
        const float mi = pr[i * (D + 2)];
        if (mi == -INFINITY) continue;            // a warp that saw no key
        const float w = ex2(mi - M);
        l = fmaf(pr[i * (D + 2) + 1], w, l);
        acc = fmaf(pr[i * (D + 2) + 2 + threadIdx.x], w, acc);
    }
    store_out(out + row * D + threadIdx.x, acc / l);
    if (threadIdx.x == 0) lse[row] = (M + log2f(l)) * 0.6931471805599453f;
}

#ifndef MODA_DEC_CTAS_PER_SM
#define MODA_DEC_CTAS_PER_SM 4
#endif
int seq_splits(const Problem& p) {
    const long long bh = static_cast<long long>(p.B) * p.Hk;
    // enough CTAs to fill every SM (loads in flight hide the HBM latency)
    const long long want = (static_cast<long long>(MODA_DEC_CTAS_PER_SM) * device_sm_count() + bh - 1) / bh;
    const long long by_len = (static_cast<long long>(p.T) + 255) / 256;  // >= 256 keys each
    long long n = want < by_len ? want : by_len;
    return static_cast<int>(n < 1 ? 1 : n);
}

template <typename E, int D, int GMAX>
cudaError_t launch_e(const Problem& p, const DecArgs& a, void* out, float* lse, cudaStream_t s) {
    dim3 grid(a.n_seq_split + (p.L > 0 ? 1 : 0), p.B * p.Hk);
    decode_split_kernel<E, D, GMAX><<<grid, kDecThreads, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<E, D><<<p.B * p.Hq, D, 0, s>>>(a.part, a.n_part, static_cast<E*>(out), lse);
    return cudaGetLastError();
}

template <typename E, int D>
cudaError_t launch_g(const Problem& p, const DecArgs& a, void* out, float* lse, cudaStream_t s) {
    if (p.G <= 4) return launch_e<E, D, 4>(p, a, out, lse, s);
    if (p.G <= 8) return launch_e<E, D, 8>(p, a, out, lse, s);
    return launch_e<E, D, 16>(p, a, out, lse, s);
}

}  // namespace

size_t decode_workspace_bytes(const Problem& p) {
    const size_t n_part = static_cast<size_t>(seq_splits(p) + (p.L > 0 ? 1 : 0)) * kDecWarps;
    const size_t bytes = static_cast<size_t>(p.B) * p.Hq * n_part * (p.d + 2) * sizeof(float);
    return (bytes + 255) & ~static_cast<size_t>(255);
}

cudaError_t launch_decode(const Problem& p, const void* q, const void* K, const void* V,
                          const void* Kd, const void* Vd, void* out, float* lse, void* ws,
                          cudaStream_t stream) {
    DecArgs a;
    a.q = q; a.K = K; a.V = V; a.Kd = Kd; a.Vd = Vd;
    a.part = static_cast<float*>(ws);
    a.B = p.B; a.Hq = p.Hq; a.Hk = p.Hk; a.T = p.T; a.L = p.L; a.G = p.G; a.win_lo = p.win_lo;
    a.n_seq_split = seq_splits(p);
    a.kps = (p.T + a.n_seq_split - 1) / a.n_seq_split;
    a.n_part = (a.n_seq_split + (p.L > 0 ? 1 : 0)) * kDecWarps;
    a.scale_log2 = p.scale_log2;
    if (p.elem_bytes == 2) {
        if (p.d == 128) return launch_g<__nv_bfloat16, 128>(p, a, out, lse, stream);
        if (p.d == 64) return launch_g<__nv_bfloat16, 64>(p, a, out, lse, stream);
    } else {
        if (p.d == 128) return launch_g<float, 128>(p, a, out, lse, stream);
        if (p.d == 64) return launch_g<float, 64>(p, a, out, lse, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace moda
