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
// group (2G multiply-adds per byte), so it is bound by HBM bandwidth.  Both
// paths split the keys, write partial (m, l, o) records and merge them.
//
// bf16 (decode_mma_kernel): one CTA per SM walks a contiguous range of the
// flattened list of 64-row items (per KV head: its depth tiles, then its
// sequence tiles).  A producer warp streams K and V tiles into a ring of
// shared-memory stages with TMA (128-byte swizzle); three consumer warps take
// the items round-robin and do the two small contractions on the tensor cores
// with mma.sync m16n8k16 (M = the G <= 16 query heads of the group): the
// scores S = q K^T with K read by ldmatrix, an online softmax on the score
// fragments, and O += P V with V read by ldmatrix.trans, P passed from the
// score accumulators as the A operand without leaving registers.  The tensor
// cores are not what bounds this kernel: they only keep the CUDA cores' issue
// slots free so that one CTA per SM can keep enough tile loads in flight.
// Each warp writes one partial per (KV head, CTA) it touches.
//
// fp32 (decode_split_kernel): CTA (split, b*Hk + hk), 8 warps.  Split s covers
// keys [s*kps, (s+1)*kps); one extra split (when L > 0) covers the depth rows.
// A warp takes 32 keys at a time: lane = key for the G scores, an online
// softmax per head across the warp, then lane = head dimensions for P V.
//
// decode_combine_kernel: one CTA per query head merges the partials:
// o = sum_i o_i 2^(m_i - M) / sum_i l_i 2^(m_i - M), LSE = (M + log2 l) ln 2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <cstring>

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
// 8 consecutive elements starting at element 8*c of a row.
__device__ __forceinline__ void load8(const float* row, int c, float* v) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row) + 2 * c);
    const float4 b = __ldg(reinterpret_cast<const float4*>(row) + 2 * c + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// N consecutive elements (N = 2 or 4) at `p`.
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
    for (int kt = k0 + warp * 32; kt < k1; kt += 32 * kDecWarps) {
        const int nk = min(32, k1 - kt);
        const E* vt = vb + static_cast<size_t>(kt) * D + lane * NDL;
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
        if (nk == 32) {           // full tile: several V rows in flight
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

// ------------------------------------------------------------------------
// bf16 path: TMA-staged tiles, mma.sync contractions, flattened schedule.
constexpr int kMmaWarps = 3;                        // consumer warps
constexpr int kMmaThreads = 32 * (kMmaWarps + 1);   // + one producer warp
constexpr int kTileRows = 64;                       // keys per item
constexpr int kRingBytes = 192 * 1024;

template <int D>
struct DecLay {
    static constexpr int kSlabs = D / 64;                        // 128-byte slabs along d
    static constexpr int kSlabBytes = kTileRows * 128;
    static constexpr int kHalf = kSlabs * kSlabBytes;            // one K (or V) tile
    static constexpr int kStage = 2 * kHalf;
    static constexpr int kStages = kRingBytes / kStage;
    // Item i sits in stage i % kStages and goes to warp i % kMmaWarps.  With
    // kStages a multiple of kMmaWarps every use of a stage belongs to the same
    // warp, so a warp never waits on a stage two phases ahead of its barrier
    // (a parity wait cannot tell phase k + 2 from phase k).
    static_assert(kStages % kMmaWarps == 0, "each stage must have a single consumer warp");
    static constexpr int kBar = kStages * kStage;
    static constexpr int kSmem = kBar + 2 * kStages * 8 + 16 + 1024;   // + 1024-byte alignment slack
};

struct DecMmaArgs {
    TmaMap tk, tv;       // [B*Hk, T, D] cached keys / values, box 64 x seq_rows
    TmaMap tkd, tvd;     // [B*Hk, L, D] depth rows, box 64 x dep_rows
    const __nv_bfloat16* q;   // [B, Hq, D]
    float* part;         // [B*Hq][maxc][kMmaWarps][D + 2]: m (base 2), l, o[D]
    unsigned int* status;
    long long n_items;   // B*Hk*ipb
    int G, T, L, win_lo;
    int n_dep, ipb;      // items per KV head: depth tiles first, then sequence tiles
    int n_cta, maxc;
    int seq_rows, dep_rows;   // rows a TMA box brings (min(64, extent))
    float scale_log2;
};

// The CTA whose item range holds item x; CTA c owns [c*n/P, (c+1)*n/P).
__host__ __device__ __forceinline__ long long dec_owner(long long x, long long n_items, int n_cta) {
    return ((x + 1) * n_cta - 1) / n_items;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
// c (16x8 fp32) += a (16x16 bf16, row) * b (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared address of the 16-byte chunk `ch` (8 elements along d) of row `row`
// of a tile written by TMA with 128-byte swizzle: slab ch/8, chunk position
// (ch % 8) XOR (row % 8) inside the row's 128 bytes.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t tile, int row, int ch) {
    return tile + (ch >> 3) * (kTileRows * 128) + row * 128 + ((((ch & 7) ^ (row & 7))) << 4);
}

template <int D>
__global__ void __launch_bounds__(kMmaThreads, 1) decode_mma_kernel(const __grid_constant__ DecMmaArgs a) {
    using Lay = DecLay<D>;
    constexpr int S = Lay::kStages;
    constexpr int NT = kTileRows / 8;     // 8-key score tiles per item
    constexpr int ND = D / 8;             // 8-dim output tiles
    extern __shared__ unsigned char dec_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
    uint64_t* empty = full + S;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long cta = blockIdx.x;
    const long long lo = cta * a.n_items / a.n_cta;
    const long long hi = (cta + 1) * a.n_items / a.n_cta;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (a.seq_rows < kTileRows || a.dep_rows < kTileRows) {
        // boxes shorter than a tile leave rows unwritten: make them finite
        uint4* z = reinterpret_cast<uint4*>(smem);
        for (int i = threadIdx.x; i < S * Lay::kStage / 16; i += kMmaThreads) z[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp == kMmaWarps) {
        // ---------------------------------------------------------- producer --
        if (lane == 0) {
            prefetch_tmap(&a.tk);
            prefetch_tmap(&a.tv);
            if (a.n_dep > 0) {
                prefetch_tmap(&a.tkd);
                prefetch_tmap(&a.tvd);
            }
            const int n = static_cast<int>(hi - lo);
            int issued = 0;
            for (int i = 0; i < n; ++i) {
                const int st = i % S;
                if (i >= S && !mbar_wait(&empty[st], ((i / S) - 1) & 1, a.status, abort_flag)) break;
                const long long x = lo + i;
                const int bh = static_cast<int>(x / a.ipb);
                const int t = static_cast<int>(x - static_cast<long long>(bh) * a.ipb);
                const bool dep = t < a.n_dep;
                const int r0 = dep ? a.win_lo + t * kTileRows : (t - a.n_dep) * kTileRows;
                const uint32_t rows = dep ? a.dep_rows : a.seq_rows;
                unsigned char* dst = smem + st * Lay::kStage;
                mbar_arrive_expect_tx(&full[st], 2u * Lay::kSlabs * 128u * rows);
#pragma unroll
                for (int s = 0; s < Lay::kSlabs; ++s) {
                    tma_load_3d(dst + s * Lay::kSlabBytes, dep ? &a.tkd : &a.tk, &full[st], s * 64, r0, bh);
                    tma_load_3d(dst + Lay::kHalf + s * Lay::kSlabBytes, dep ? &a.tvd : &a.tv, &full[st],
                                s * 64, r0, bh);
                }
                issued = i + 1;
            }
            // every load this thread started lands before the CTA retires
            // (bounded by time only: these waits ignore the abort flag)
            int no_abort = 0;
            for (int i = max(0, issued - S); i < issued; ++i)
                mbar_wait(&full[i % S], (i / S) & 1, a.status, &no_abort);
        }
        return;
    }

    // -------------------------------------------------------------- consumers --
    // Fragment coordinates of mma m16n8k16: rows g and g + 8 (query heads of
    // the group), columns 2*tig and 2*tig + 1.
    const int g = lane >> 2;
    const int tig = lane & 3;
    const uint32_t sbase = smem_u32(smem);
    const int bh_first = static_cast<int>(lo / a.ipb);
    const int bh_last = hi > lo ? static_cast<int>((hi - 1) / a.ipb) : bh_first - 1;
    bool ok = true;
    for (int bh = bh_first; ok && bh <= bh_last; ++bh) {
        // q of this KV head's group as A fragments; rows >= G are zero
        uint32_t qa[D / 16][4];
        {
            const __nv_bfloat16* q0 = a.q + (static_cast<size_t>(bh) * a.G + g) * D;
            const __nv_bfloat16* q1 = q0 + 8 * D;
            const bool v0 = g < a.G, v1 = g + 8 < a.G;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int c = 16 * ks + 2 * tig;
                qa[ks][0] = v0 ? __ldg(reinterpret_cast<const unsigned int*>(q0 + c)) : 0u;
                qa[ks][1] = v1 ? __ldg(reinterpret_cast<const unsigned int*>(q1 + c)) : 0u;
                qa[ks][2] = v0 ? __ldg(reinterpret_cast<const unsigned int*>(q0 + c + 8)) : 0u;
                qa[ks][3] = v1 ? __ldg(reinterpret_cast<const unsigned int*>(q1 + c + 8)) : 0u;
            }
        }
        float o[ND][4];
#pragma unroll
        for (int nd = 0; nd < ND; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.0f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;

        const long long x0 = max(lo, static_cast<long long>(bh) * a.ipb);
        const long long x1 = min(hi, static_cast<long long>(bh + 1) * a.ipb);
        long long i = x0 - lo;
        i += (warp - static_cast<int>(i % kMmaWarps) + kMmaWarps) % kMmaWarps;   // this warp's first item
        for (; lo + i < x1; i += kMmaWarps) {
            const int st = static_cast<int>(i % S);
            ok = __all_sync(0xffffffffu, mbar_wait(&full[st], static_cast<uint32_t>((i / S) & 1), a.status,
                                                   abort_flag));
            if (!ok) break;
            const int t = static_cast<int>(lo + i - static_cast<long long>(bh) * a.ipb);
            const bool dep = t < a.n_dep;
            const int nvalid = dep ? min(kTileRows, a.L - (a.win_lo + t * kTileRows))
                                   : min(kTileRows, a.T - (t - a.n_dep) * kTileRows);
            const uint32_t sk = sbase + st * Lay::kStage;
            const uint32_t sv = sk + Lay::kHalf;

            // S = q K^T: 16 heads x 64 keys
            float s[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
            for (int kp = 0; kp < D / 32; ++kp) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t b[4];
                    ldsm_x4(sw128_chunk(sk, nt * 8 + (lane & 7), kp * 4 + (lane >> 3)), b);
                    mma_bf16_16816(s[nt], qa[2 * kp], b[0], b[1]);
                    mma_bf16_16816(s[nt], qa[2 * kp + 1], b[2], b[3]);
                }
            }
            // online softmax in base 2 on rows g (values 0, 1) and g + 8 (2, 3)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = s[nt][e] * a.scale_log2;
                    if (nvalid < kTileRows && nt * 8 + 2 * tig + (e & 1) >= nvalid) v = -INFINITY;
                    s[nt][e] = v;
                }
                mx0 = fmax3(mx0, s[nt][0], s[nt][1]);
                mx1 = fmax3(mx1, s[nt][2], s[nt][3]);
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);   // finite: key 0 is valid
            const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                s[nt][0] = ex2(s[nt][0] - mn0);
                s[nt][1] = ex2(s[nt][1] - mn0);
                s[nt][2] = ex2(s[nt][2] - mn1);
                s[nt][3] = ex2(s[nt][3] - mn1);
                ps0 += s[nt][0] + s[nt][1];
                ps1 += s[nt][2] + s[nt][3];
            }
            l0 = fmaf(l0, al0, ps0);
            l1 = fmaf(l1, al1, ps1);
#pragma unroll
            for (int nd = 0; nd < ND; ++nd) {
                o[nd][0] *= al0;
                o[nd][1] *= al0;
                o[nd][2] *= al1;
                o[nd][3] *= al1;
            }
            // O += P V: P (16 x 64, bf16) from the score fragments, V by
            // transposing loads (rows = keys, columns = head dimensions)
#pragma unroll
            for (int kk = 0; kk < kTileRows / 16; ++kk) {
                uint32_t pa[4];
                pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
                for (int np = 0; np < ND / 2; ++np) {
                    uint32_t b[4];
                    ldsm_x4_t(sw128_chunk(sv, kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7), np * 2 + (lane >> 4)),
                              b);
                    mma_bf16_16816(o[2 * np], pa, b[0], b[1]);
                    mma_bf16_16816(o[2 * np + 1], pa, b[2], b[3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (!ok) break;
        // this warp's partial for (bh, this CTA)
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const int cc = static_cast<int>(cta - dec_owner(static_cast<long long>(bh) * a.ipb, a.n_items, a.n_cta));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = g + 8 * h;
            if (row < a.G) {
                float* pr = a.part +
                            (((static_cast<size_t>(bh) * a.G + row) * a.maxc + cc) * kMmaWarps + warp) * (D + 2);
                if (tig == 0) {
                    pr[0] = h ? m1 : m0;
                    pr[1] = h ? l1 : l0;
                }
#pragma unroll
                for (int nd = 0; nd < ND; ++nd)
                    *reinterpret_cast<float2*>(pr + 2 + nd * 8 + 2 * tig) = make_float2(o[nd][2 * h], o[nd][2 * h + 1]);
            }
        }
    }
}

__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Which partial records a query head merges.  Fixed splits: n_part records.
// Item ranges (bf16 path): the CTAs owning the KV head's items, kMmaWarps
// records each, out of maxc * kMmaWarps slots.
struct CombineRange {
    int n_part;          // > 0: fixed count
    int G, ipb, n_cta, maxc;
    long long n_items;
};

// One CTA (D threads) per query head: merge its partials.
template <typename E, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ part, const CombineRange r,
                                                            E* __restrict__ out, float* __restrict__ lse) {
    const size_t row = blockIdx.x;
    int n_part, stride;
    if (r.n_part > 0) {
        n_part = stride = r.n_part;
    } else {
        const long long bh = static_cast<long long>(row / r.G);
        const long long c0 = dec_owner(bh * r.ipb, r.n_items, r.n_cta);
        const long long c1 = dec_owner((bh + 1) * r.ipb - 1, r.n_items, r.n_cta);
        n_part = static_cast<int>(c1 - c0 + 1) * kMmaWarps;
        stride = r.maxc * kMmaWarps;
    }
    const float* pr = part + row * stride * (D + 2);
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

// Item ranges of the bf16 path.
struct MmaPlan {
    int n_dep, ipb, n_cta, maxc;
    long long n_items;
};
MmaPlan mma_plan(const Problem& p) {
    MmaPlan m;
    const int ld = p.L - p.win_lo;
    m.n_dep = ld > 0 ? (ld + kTileRows - 1) / kTileRows : 0;
    m.ipb = m.n_dep + (p.T + kTileRows - 1) / kTileRows;
    const long long bhs = static_cast<long long>(p.B) * p.Hk;
    m.n_items = bhs * m.ipb;
    const long long sms = device_sm_count();
    m.n_cta = static_cast<int>(m.n_items < sms ? m.n_items : sms);
    m.maxc = 1;
    for (long long bh = 0; bh < bhs && m.n_items > 0; ++bh) {
        const long long c = dec_owner((bh + 1) * m.ipb - 1, m.n_items, m.n_cta) -
                            dec_owner(bh * m.ipb, m.n_items, m.n_cta) + 1;
        if (c > m.maxc) m.maxc = static_cast<int>(c);
    }
    return m;
}

template <typename E, int D, int GMAX>
cudaError_t launch_e(const Problem& p, const DecArgs& a, void* out, float* lse, cudaStream_t s) {
    dim3 grid(a.n_seq_split + (p.L > 0 ? 1 : 0), p.B * p.Hk);
    decode_split_kernel<E, D, GMAX><<<grid, kDecThreads, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CombineRange r{};
    r.n_part = a.n_part;
    decode_combine_kernel<E, D><<<p.B * p.Hq, D, 0, s>>>(a.part, r, static_cast<E*>(out), lse);
    return cudaGetLastError();
}

template <typename E, int D>
cudaError_t launch_g(const Problem& p, const DecArgs& a, void* out, float* lse, cudaStream_t s) {
    if (p.G <= 4) return launch_e<E, D, 4>(p, a, out, lse, s);
    if (p.G <= 8) return launch_e<E, D, 8>(p, a, out, lse, s);
    return launch_e<E, D, 16>(p, a, out, lse, s);
}

template <int D>
cudaError_t launch_mma(const Problem& p, const void* q, const void* K, const void* V, const void* Kd,
                       const void* Vd, void* out, float* lse, void* ws, cudaStream_t s) {
    using Lay = DecLay<D>;
    const MmaPlan m = mma_plan(p);
    if (m.n_items == 0) return cudaSuccess;
    DecMmaArgs a;
    std::memset(&a, 0, sizeof(a));
    const uint64_t bhs = static_cast<uint64_t>(p.B) * p.Hk;
    a.seq_rows = p.T < kTileRows ? p.T : kTileRows;
    a.dep_rows = p.L <= 0 ? kTileRows : (p.L < kTileRows ? p.L : kTileRows);
    cudaError_t e;
    if ((e = make_tma_3d_bf16(&a.tk, K, D, p.T, bhs, a.seq_rows, 1)) != cudaSuccess) return e;
    if ((e = make_tma_3d_bf16(&a.tv, V, D, p.T, bhs, a.seq_rows, 1)) != cudaSuccess) return e;
    if (m.n_dep > 0) {
        if ((e = make_tma_3d_bf16(&a.tkd, Kd, D, p.L, bhs, a.dep_rows, 1)) != cudaSuccess) return e;
        if ((e = make_tma_3d_bf16(&a.tvd, Vd, D, p.L, bhs, a.dep_rows, 1)) != cudaSuccess) return e;
    }
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.part = static_cast<float*>(ws);
    a.status = device_status_word();
    a.n_items = m.n_items;
    a.G = p.G;
    a.T = p.T;
    a.L = p.L;
    a.win_lo = p.win_lo;
    a.n_dep = m.n_dep;
    a.ipb = m.ipb;
    a.n_cta = m.n_cta;
    a.maxc = m.maxc;
    a.scale_log2 = p.scale_log2;
    if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(decode_mma_kernel<D>), Lay::kSmem)) != cudaSuccess)
        return e;
    decode_mma_kernel<D><<<m.n_cta, kMmaThreads, Lay::kSmem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CombineRange r;
    r.n_part = 0;
    r.G = p.G;
    r.ipb = m.ipb;
    r.n_cta = m.n_cta;
    r.maxc = m.maxc;
    r.n_items = m.n_items;
    decode_combine_kernel<__nv_bfloat16, D><<<p.B * p.Hq, D, 0, s>>>(
        a.part, r, static_cast<__nv_bfloat16*>(out), lse);
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(const Problem& p) {
    size_t bytes;
    if (p.elem_bytes == 2) {
        const MmaPlan m = mma_plan(p);
        bytes = static_cast<size_t>(p.B) * p.Hq * m.maxc * kMmaWarps * (p.d + 2) * sizeof(float);
    } else {
        const size_t n_part = static_cast<size_t>(seq_splits(p) + (p.L > 0 ? 1 : 0)) * kDecWarps;
        bytes = static_cast<size_t>(p.B) * p.Hq * n_part * (p.d + 2) * sizeof(float);
    }
    return (bytes + 255) & ~static_cast<size_t>(255);
}

cudaError_t launch_decode(const Problem& p, const void* q, const void* K, const void* V,
                          const void* Kd, const void* Vd, void* out, float* lse, void* ws,
                          cudaStream_t stream) {
    if (p.elem_bytes == 2) {
        if (p.d == 128) return launch_mma<128>(p, q, K, V, Kd, Vd, out, lse, ws, stream);
        if (p.d == 64) return launch_mma<64>(p, q, K, V, Kd, Vd, out, lse, ws, stream);
        return cudaErrorInvalidValue;
    }
    DecArgs a;
    a.q = q; a.K = K; a.V = V; a.Kd = Kd; a.Vd = Vd;
    a.part = static_cast<float*>(ws);
    a.B = p.B; a.Hq = p.Hq; a.Hk = p.Hk; a.T = p.T; a.L = p.L; a.G = p.G; a.win_lo = p.win_lo;
    a.n_seq_split = seq_splits(p);
    a.kps = (p.T + a.n_seq_split - 1) / a.n_seq_split;
    a.n_part = (a.n_seq_split + (p.L > 0 ? 1 : 0)) * kDecWarps;
    a.scale_log2 = p.scale_log2;
    if (p.d == 128) return launch_g<float, 128>(p, a, out, lse, stream);
    if (p.d == 64) return launch_g<float, 64>(p, a, out, lse, stream);
    return cudaErrorInvalidValue;
}

}  // namespace moda
