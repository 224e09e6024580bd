// moda_repack.cu -- depth-KV repack: layer-major [L, B, Hk, T, d] to the
// token-major (flash-compatible) [B, Hk, T*L, d] with row t*L + l (paper
// summary of arXiv 2603.15619, "Hardware-Efficient Implementation").
//
// Pure HBM traffic: every byte is read once and written once.  One warp
// moves one token (b, hk, t) at a time: its L rows are L separate rows of the
// source (one per layer, B*Hk*T rows apart) and one contiguous run of L rows
// of the destination.  Lanes take consecutive 16-byte vectors of that run
// (a 256-byte row is 16 lanes), so every load and store instruction of a
// warp covers whole rows, and each lane keeps kUnroll loads in flight before
// storing.  Index arithmetic is 32-bit and per token, not per vector.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moda_internal.h"

namespace moda {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;

// VPR: 16-byte vectors per row when known at compile time (0: runtime vpr).
template <int VPR>
__global__ void __launch_bounds__(kThreads) repack_vec16_kernel(const uint4* __restrict__ src,
                                                                 uint4* __restrict__ dst, int L,
                                                                 int BHT, int vpr_rt) {
    const int vpr = VPR > 0 ? VPR : vpr_rt;
    const int lane = threadIdx.x & 31;
    const int wpb = kThreads / 32;
    const int n_warps = gridDim.x * wpb;
    const int per_token = L * vpr;                        // vectors of one token
    for (int item = blockIdx.x * wpb + (threadIdx.x >> 5); item < BHT; item += n_warps) {
        const uint4* s0 = src + static_cast<size_t>(item) * vpr;          // layer 0 row of the token
        uint4* d0 = dst + static_cast<size_t>(item) * per_token;
        for (int base = 0; base < per_token; base += 32 * kUnroll) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int e = base + u * 32 + lane;
                if (e < per_token) {
                    const int l = e / vpr;
                    const int c = e - l * vpr;
                    v[u] = __ldcs(s0 + static_cast<size_t>(l) * BHT * vpr + c);
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int e = base + u * 32 + lane;
                if (e < per_token) __stcs(d0 + e, v[u]);
            }
        }
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
    if (row_bytes % 16 == 0 && (long long)L * (row_bytes / 16) < (1LL << 30)) {
        const int vpr = (int)(row_bytes / 16);
        const long long BHT = BH * T;                         // tokens; < 2^31 (validated)
        const long long warps = (long long)sms * 8 * (kThreads / 32);
        long long blocks = BHT < warps ? (BHT + kThreads / 32 - 1) / (kThreads / 32) : (long long)sms * 8;
        if (blocks < 1) blocks = 1;
        if (vpr == 16)
            repack_vec16_kernel<16><<<(unsigned)blocks, kThreads, 0, stream>>>(
                static_cast<const uint4*>(src), static_cast<uint4*>(dst), L, (int)BHT, vpr);
        else if (vpr == 8)
            repack_vec16_kernel<8><<<(unsigned)blocks, kThreads, 0, stream>>>(
                static_cast<const uint4*>(src), static_cast<uint4*>(dst), L, (int)BHT, vpr);
        else
            repack_vec16_kernel<0><<<(unsigned)blocks, kThreads, 0, stream>>>(
                static_cast<const uint4*>(src), static_cast<uint4*>(dst), L, (int)BHT, vpr);
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
