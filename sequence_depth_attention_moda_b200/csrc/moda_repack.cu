// moda_repack.cu -- depth-KV repack: layer-major [L, B, Hk, T, d] to the
// token-major (flash-compatible) [B, Hk, T*L, d] with row t*L + l (paper
// summary of arXiv 2603.15619, "Hardware-Efficient Implementation").
//
// Pure HBM traffic: every byte is read once and written once.  Each warp
// moves whole rows with 16-byte accesses (a 256-byte row is 16 lanes), and
// every thread keeps kUnroll independent loads in flight before storing.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moda_internal.h"

namespace moda {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// One 16-byte vector per step.  dst vector index i -> (row r, vector v);
// r = (bh*T + t)*L + l reads source row (l*BH + bh)*T + t.
__global__ void __launch_bounds__(kThreads) repack_vec16_kernel(const uint4* __restrict__ src,
                                                                 uint4* __restrict__ dst, int L,
                                                                 long long BH, int T,
                                                                 int vecs_per_row,
                                                                 long long total) {
    const long long stride = (long long)gridDim.x * kThreads;
    long long i = (long long)blockIdx.x * kThreads + threadIdx.x;
    for (; i < total; i += stride * kUnroll) {
        uint4 v[kUnroll];
        long long idx[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            idx[u] = i + u * stride;
            if (idx[u] < total) {
                const long long r = idx[u] / vecs_per_row;
                const int c = (int)(idx[u] - r * vecs_per_row);
                const int l = (int)(r % L);
                const long long bt = r / L;
                const long long bh = bt / T;
                const long long t = bt - bh * T;
                const long long sr = ((long long)l * BH + bh) * T + t;
                v[u] = __ldcs(src + sr * vecs_per_row + c);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (idx[u] < total) __stcs(dst + idx[u], v[u]);
    }
}

// Any row size: element-wise copy of 16-bit units (fp32 rows are even units).
__global__ void __launch_bounds__(kThreads) repack_u16_kernel(const uint16_t* __restrict__ src,
                                                               uint16_t* __restrict__ dst, int L,
                                                               long long BH, int T, int units,
                                                               long long total) {
    const long long stride = (long long)gridDim.x * kThreads;
    for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < total; i += stride) {
        const long long r = i / units;
        const int c = (int)(i - r * units);
        const int l = (int)(r % L);
        const long long bt = r / L;
        const long long bh = bt / T;
        const long long t = bt - bh * T;
        dst[i] = src[(((long long)l * BH + bh) * T + t) * units + c];
    }
}

}  // namespace

cudaError_t launch_repack(int B, int Hk, int T, int d, int L, int elem_bytes, const void* src,
                          void* dst, cudaStream_t stream) {
    const long long BH = (long long)B * Hk;
    const long long row_bytes = (long long)d * elem_bytes;
    const long long rows = BH * T * L;
    const int sms = device_sm_count();
    if (row_bytes % 16 == 0) {
        const int vpr = (int)(row_bytes / 16);
        const long long total = rows * vpr;
        long long blocks = (total + (long long)kThreads * kUnroll - 1) / ((long long)kThreads * kUnroll);
        const long long cap = (long long)sms * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        repack_vec16_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(
            static_cast<const uint4*>(src), static_cast<uint4*>(dst), L, BH, T, vpr, total);
    } else {
        const int units = (int)(row_bytes / 2);
        const long long total = rows * units;
        long long blocks = (total + kThreads - 1) / kThreads;
        const long long cap = (long long)sms * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        repack_u16_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(
            static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), L, BH, T, units, total);
    }
    return cudaGetLastError();
}

}  // namespace moda
