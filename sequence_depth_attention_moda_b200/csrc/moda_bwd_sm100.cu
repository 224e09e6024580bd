// moda_bwd_sm100.cu -- MoDA backward for sm_100a (tcgen05 + TMEM + TMA).
//
// The pages give no backward formulas; this is the derivative of the forward
// definition (paper summary of arXiv 2603.15619, "Mixture-of-Depths Attention
// (MoDA): The Unified Operator": one softmax over [causal sequence keys |
// the token's own L depth rows]).  With P the softmax weights recomputed from
// the saved LSE, and D = rowsum(dO * O):
//     dS = P * (dO . v - D)
//     dQ = scale * (sum_j dS_j K_j + sum_l dS'_l Kd_l)
//     dK_j = scale * sum over the group's heads and rows t >= j of dS q
//     dV_j = sum over the same rows of P dO
//     dKd[t*L+l] = scale * sum over the group's heads of dS'_l q[h,t]
//     dVd[t*L+l] = sum over the group's heads of P'_l dO[h,t]
// Non-causal: "rows t >= j" becomes all rows.  Depth window S: only the last S
// depth rows of a token take part; the gradients of the others are zero.
//
// Three launches, no floating-point atomics (bitwise repeatable):
//  1. rowdot:  D[b,h,t] = sum_c dO * O                      (CUDA cores, HBM)
//  2. dkdv:    one CTA per 128-key tile of one KV head.  M = 128 keys:
//              S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and dS^T written
//              back to TMEM as bf16, then dV += P^T dO and dK += dS^T Q with
//              the A operand read from TMEM.  The group's G heads are all
//              iterated inside the CTA, so dK/dV are complete sums.  With the
//              full workspace, store warps also write every dS^T row into
//              the dq kernel's operand tiles (stored dS); the query blocks
//              are then token-major (64 / G tokens of all G heads, row
//              t * G + g), the dq tile's row order.
//  3. dq:      one CTA per 128-row query tile (G heads x 128/G tokens, as in
//              the forward; token-major rows with stored dS).  Sequence
//              blocks: dQ += dS K, dS either read from the stored tiles (no
//              S, dP, exponentials) or recomputed from S = Q K^T and
//              dP = dO V^T.  Depth blocks: S', dP' and
//              dS' recomputed, P' and dS' (bf16) also staged in shared
//              memory, and the token-local depth gradients come out as
//              dKd^T = Q^T dS' and dVd^T = dO^T P' (M = d, N = depth rows):
//              each depth row belongs to exactly one query tile, so these
//              are complete without atomics.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <cmath>

#include "moda_internal.h"
#include "moda_ptx.cuh"

namespace moda {
namespace {

using namespace ptx;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 352;            // dq: warp 0 TMA, warps 1 and 6 MMA, warps 2..5 and 7..10 math
constexpr int kMathThreads = 256;
constexpr int kKvMathWarps = 8;          // dkdv: warps 2..9, two per TMEM lane quarter
constexpr int kKvGradWarp = 2 + kKvMathWarps;   // dkdv: issuer of dV and dK (warp 10)
constexpr int kKvStoreWarp0 = kKvGradWarp + 1;  // dkdv: warps 11..14 store dS (one per lane quarter)
constexpr int kKvThreads = 32 * (kKvStoreWarp0 + 4);
constexpr uint32_t kSlabBytes = 128 * 128;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------ 1. rowdot ----
template <int D>
__global__ void __launch_bounds__(256) rowdot_kernel(long long nrows,
                                                      const __nv_bfloat16* __restrict__ O,
                                                      const __nv_bfloat16* __restrict__ dO,
                                                      float* __restrict__ Dout) {
    constexpr int kLanesPerRow = D / 8;              // 16 B per lane
    constexpr int kRowsPerWarp = 32 / kLanesPerRow;
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long row = warp * kRowsPerWarp + lane / kLanesPerRow;
    float s = 0.0f;
    if (row < nrows) {
        const uint4 a = reinterpret_cast<const uint4*>(O + row * D)[lane % kLanesPerRow];
        const uint4 b = reinterpret_cast<const uint4*>(dO + row * D)[lane % kLanesPerRow];
        const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 fa = __bfloat1622float2(pa[e]);
            const float2 fb = __bfloat1622float2(pb[e]);
            s = fmaf(fa.x, fb.x, s);
            s = fmaf(fa.y, fb.y, s);
        }
    }
#pragma unroll
    for (int o = kLanesPerRow / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (row < nrows && lane % kLanesPerRow == 0) Dout[row] = s;
}

// -------------------------------------------------------------- 2. dkdv ----
// Query blocks are 64 rows, so S^T and dP^T are double-buffered in TMEM:
//   S^T0 [0,64) S^T1 [64,128) | dP^T0 [128,192) dP^T1 [192,256) |
//   dV [256, 256+D) | dK [384, 384+D)
// The per-query statistics enter through the MMAs: one more K=16 step per
// product multiplies a constant key-side tile whose rows are (1, 1, 0, ...)
// by query-side rows (-b_hi, -b_lo, 0, ...), where b_hi + b_lo is LSE / scale
// (for S^T) or D (for dP^T) split into two bf16 parts.  TMEM then holds
// s - LSE/scale and dP - D, and the math warps need no statistics at all:
// P^T = 2^(scale*log2(e) * S'^T), dS^T = P^T * dP'^T.
struct DkdvArgs {
    TmaMap tk, tv, tq, tdo;
    const float* LSE;
    const float* Drow;
    __nv_bfloat16* dK;
    __nv_bfloat16* dV;
    unsigned int* status;
    int B, Hq, Hk, T, G, n_kt, n_qb;     // n_qb counts 64-row query blocks
    int band;                            // (b, KV head) pairs per band (banded_item)
    int causal;
    float scale, scale_log2;
    // Stored dS (nullptr: not stored): the tiles the dq kernel reads instead
    // of recomputing S and dP; see store_ds_row.
    unsigned char* dS;
    int n_qt, n_kb, tq_log2;             // dq query tiles (Tq = 1 << tq_log2 tokens), 64-key blocks
    // Token-major query blocks (kTok, with stored dS): block i holds tokens
    // [i * TB, (i + 1) * TB), TB = 64 / G = 1 << tb_log2, of all G heads, row
    // t * G + g (tq / tdo are 4-D head-strided maps); otherwise the blocks are
    // 64 tokens of one head, head by head.
    int tb_log2, g_log2, n_tb;
    int n_items, persist;                // key tiles; persist: CTAs walk several (snake_tile)
};

// Stored dS tiles.  Tile (bh, qt, kb) holds dS = P * (dP - D) (unscaled, bf16)
// for the 128 rows of dq query tile qt (token-major: row r = (t - qt * Tq) * G
// + g, as in the forward's tile) and the 64 keys of key block kb, laid out byte for byte as
// the dq kernel's shared-memory A operand, MN-major without swizzle: the 16
// bytes of rows 8c .. 8c + 7 for key k at byte c * 1024 + k * 16.  The dK/dV
// kernel's store warps hold one key row each (a warp: 32 consecutive keys),
// so every store instruction writes 512 contiguous bytes.  Tiles are 16 KB,
// at ((bh * n_qt + qt) * n_kb + kb) * 16 KB.
constexpr uint32_t kDsTileBytes = 128 * 64 * 2;

// One key row's dS for the 64 rows of a token-major query block (32 packed
// bf16 pairs in v: tokens t0 .. t0 + TB - 1 of all G heads, row t * G + g)
// into the tiles: the block is 64 consecutive rows of one dq query tile (TB
// divides Tq), so its 8 chunks of 8 rows go to 8 consecutive 1 KB row groups
// of that tile.  Keys past T get zeros; key blocks past the last are skipped.
__device__ __forceinline__ void store_ds_row(const DkdvArgs& a, int bh, int key, int t0, const uint32_t* v) {
    const int kb = key >> 6, k = key & 63;
    if (kb >= a.n_kb) return;
    const bool live = key < a.T;
    const int qt = t0 >> a.tq_log2;
    const int r0 = (t0 - (qt << a.tq_log2)) << a.g_log2;   // first row of the block in the tile
    unsigned char* dst = a.dS + (static_cast<size_t>(bh * a.n_qt + qt) * a.n_kb + kb) * kDsTileBytes +
                         (r0 >> 3) * 1024 + k * 16;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        // streaming store (evict first): the tiles are read once, by the dQ
        // kernel, and must not push the Q / dO tiles this kernel re-reads out of L2
        __stcs(reinterpret_cast<uint4*>(dst + j * 1024),
               live ? make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]) : make_uint4(0, 0, 0, 0));
    }
}

constexpr int kKvBQ = 64;               // query rows per iteration
constexpr int kKvStages = 4;            // Q/dO ring depth
constexpr uint32_t kKvSlab = 64 * 128;
// Bias tiles: K = 16 (one MMA step), K-major without swizzle.  Core matrices
// of 8 rows x 16 bytes; element (row r, k) at (r / 8) * 256 + (k / 8) * 128 +
// (r % 8) * 16 + (k % 8) * 2, so the K-adjacent core matrix is 128 B further
// and the next 8-row group 256 B further.
constexpr uint32_t kBiasLbo = 128, kBiasSbo = 256;
__host__ __device__ constexpr uint32_t bias_chunk(int r, int c) {   // 16-byte chunk c (k = 8c .. 8c + 7) of row r
    return (r >> 3) * kBiasSbo + c * kBiasLbo + (r & 7) * 16;
}

template <int D>
struct DkdvLayout {
    static constexpr int kSlabs = D / 64;
    static constexpr uint32_t kKTile = kSlabs * kSlabBytes;     // 128 key rows
    static constexpr uint32_t kQTile = kSlabs * kKvSlab;        // 64 query rows
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kKTile;
    static constexpr uint32_t kQ = 2 * kKTile;                  // kKvStages stages
    static constexpr uint32_t kDO = kQ + kKvStages * kQTile;    // kKvStages stages
    // bias tiles of each stage (64 query rows x K = 16): LSE / scale, then D
    static constexpr uint32_t kBiasQ = 64 * 32;
    static constexpr uint32_t kAL = kDO + kKvStages * kQTile;
    static constexpr uint32_t kAD = kAL + kKvStages * kBiasQ;
    static constexpr uint32_t kAA = kAD + kKvStages * kBiasQ;   // key-side (1, 1, 0, ...) rows, 128 x K = 16
    static constexpr uint32_t kBar = kAA + 128 * 32;
    static constexpr uint32_t kBytes = kBar + 256;
    static constexpr uint32_t kDynSmem = kBytes + 1024 > 120u * 1024 ? kBytes + 1024 : 120u * 1024;
};

// Per S/dP buffer b (iteration it uses b = it & 1): SFull / DPFull (S^T /
// dP^T products done), PReady / DSReady (P^T / dS^T written over them by the
// math warps), SFree (dV product done: the S columns may be overwritten),
// DSRead (store warps hold the dS^T rows).  The Q/dO stage release QEmpty
// follows the dK product, the last reader of the stage and of dS^T.
enum { kA_KVFull = 0, kA_QFull = 1, kA_QEmpty = 1 + kKvStages, kA_SFull = 1 + 2 * kKvStages,
       kA_DPFull = 3 + 2 * kKvStages, kA_PReady = 5 + 2 * kKvStages, kA_DSReady = 7 + 2 * kKvStages,
       kA_SFree = 9 + 2 * kKvStages, kA_Final = 11 + 2 * kKvStages, kA_DSRead = 12 + 2 * kKvStages,
       kA_AccFree = 14 + 2 * kKvStages, kA_NumBars = 15 + 2 * kKvStages };
static_assert(kA_NumBars * 8 + 8 <= 256, "dK/dV barriers, TMEM address and abort flag fit the barrier area");

// kTok: token-major query blocks (the stored-dS backward), see DkdvArgs.
template <int D, bool kTok>
__global__ void __launch_bounds__(kKvThreads, 1) dkdv_kernel(const __grid_constant__ DkdvArgs a) {
    using Lay = DkdvLayout<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kA_NumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    // The dQ kernel may start on SMs this grid has left: its depth blocks
    // need nothing from this kernel, and it waits for this grid's completion
    // before its first stored dS tile.
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nbh = a.B * a.Hk;
    // Work items: key tiles (b * Hk + hk, kt), the longest (small kt) first
    // within bands of heads (banded_item).  A persistent launch deals them to
    // its CTAs in a snake over rounds of gridDim.x items (snake_tile);
    // otherwise CTA c takes item c.  Every role walks the same items and keeps
    // a running iteration count for ring stages, TMEM buffers and barrier
    // phases; the next item's K/V load and first score products overlap the
    // previous item's dK/dV read-out.
    const int n_ctas = static_cast<int>(gridDim.x);
    const int n_rounds = a.persist ? (a.n_items + n_ctas - 1) / n_ctas : 1;
    auto item_of = [&](int rnd) {
        return a.persist ? snake_tile(rnd, static_cast<int>(blockIdx.x), n_ctas) : static_cast<int>(blockIdx.x);
    };
    struct Item {
        int kt, bh, b, hk, qb0, nqb, tb0, n_it;
    };
    // Iteration it of an item -> query block: its first token tq0 and, head by
    // head, its head g (token-major blocks hold all G heads).  Causal: the
    // first block that sees the key tile is the one holding token kt * BN.
    auto decode = [&](int idx) {
        Item I;
        banded_item(idx, a.n_kt, nbh, a.band, &I.kt, &I.bh);
        I.b = I.bh / a.Hk;
        I.hk = I.bh - I.b * a.Hk;
        I.qb0 = a.causal ? I.kt * (BN / kKvBQ) : 0;
        I.nqb = a.n_qb - I.qb0;
        I.tb0 = a.causal ? (I.kt * BN) >> a.tb_log2 : 0;
        I.n_it = kTok ? a.n_tb - I.tb0 : a.G * I.nqb;
        return I;
    };
    auto block_of = [&](const Item& I, int it, int* g, int* tq0) {
        if (kTok) {
            *g = 0;
            *tq0 = (I.tb0 + it) << a.tb_log2;
        } else {
            *g = it / I.nqb;
            *tq0 = (I.qb0 + it - *g * I.nqb) * kKvBQ;
        }
    };

    if (threadIdx.x == 0) {
        mbar_init(&bars[kA_KVFull], 1);
        for (int s = 0; s < kKvStages; ++s) {
            mbar_init(&bars[kA_QFull + s], 1);
            mbar_init(&bars[kA_QEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kA_SFull + s], 1);
            mbar_init(&bars[kA_DPFull + s], 1);
            mbar_init(&bars[kA_PReady + s], kKvMathWarps);   // one arrive per math warp
            mbar_init(&bars[kA_DSReady + s], kKvMathWarps);
            mbar_init(&bars[kA_SFree + s], 1);
        }
        mbar_init(&bars[kA_Final], 1);
        mbar_init(&bars[kA_AccFree], kKvMathWarps);         // dK/dV of an item read out
        for (int s = 0; s < 2; ++s) mbar_init(&bars[kA_DSRead + s], 4);   // one arrive per store warp
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    // key-side bias rows: elements 0 and 1 are 1.0, the rest zero; in the
    // query-side tiles the second chunk (k = 8 .. 15) of every row stays zero
    for (int i = threadIdx.x; i < 2 * BN; i += kKvThreads) {
        const int r = i >> 1, c = i & 1;
        *reinterpret_cast<uint4*>(smem + Lay::kAA + bias_chunk(r, c)) =
            c == 0 ? make_uint4(pack_bf16(1.0f, 1.0f), 0u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = threadIdx.x; i < 2 * kKvStages * kKvBQ; i += kKvThreads) {
        const int r = i % kKvBQ, t = i / kKvBQ;          // t: tile (AL, AD of each stage)
        *reinterpret_cast<uint4*>(smem + Lay::kAL + t * Lay::kBiasQ + bias_chunk(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // producer, whole warp: per item the K and V tiles, then per query
        // block the bias rows (lanes write rows lane and lane + 32) and Q and
        // dO by TMA (lane 0)
        if (lane == 0) {
            prefetch_tmap(&a.tk); prefetch_tmap(&a.tv); prefetch_tmap(&a.tq); prefetch_tmap(&a.tdo);
        }
        const float inv_scale = 1.0f / a.scale;
        float nl[2], nd[2];
        int it0 = 0, n_done = 0, issued = 0;
        bool ok = true;
        for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
            const int idx = item_of(rnd);
            if (idx >= a.n_items) continue;
            const Item I = decode(idx);
            // the item's K and V replace the previous item's once its last dK
            // product (and so every product reading K or V) has completed
            if (lane == 0) {
                if (n_done > 0 && !mbar_wait(&bars[kA_QEmpty + (it0 - 1) % kKvStages],
                                             ((it0 - 1) / kKvStages) & 1, a.status, abort_flag))
                    ok = false;
                if (ok) {
                    mbar_arrive_expect_tx(&bars[kA_KVFull], 2 * Lay::kKTile);
                    for (int s = 0; s < Lay::kSlabs; ++s) {
                        tma_load_3d(smem + Lay::kK + s * kSlabBytes, &a.tk, &bars[kA_KVFull], s * 64, I.kt * BN, I.bh);
                        tma_load_3d(smem + Lay::kV + s * kSlabBytes, &a.tv, &bars[kA_KVFull], s * 64, I.kt * BN, I.bh);
                    }
                }
            }
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            // LSE and D of a query block are read one iteration ahead, so their
            // global-load latency overlaps the wait for the stage to free up
            auto fetch_stats = [&](int it) {
                int g, tq0;
                block_of(I, it, &g, &tq0);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int rr = lane + 32 * h2;                 // row of the block
                    const int gr = kTok ? (rr & (a.G - 1)) : g;
                    const int t = tq0 + (kTok ? rr >> a.g_log2 : rr);
                    const size_t qrow = static_cast<size_t>(I.b * a.Hq + I.hk * a.G + gr) * a.T + t;
                    nl[h2] = t < a.T ? a.LSE[qrow] : INFINITY;     // rows past T: p = 0
                    nd[h2] = t < a.T ? a.Drow[qrow] : 0.0f;
                }
            };
            if (I.n_it > 0) fetch_stats(0);
            for (int it = 0; it < I.n_it; ++it) {
                const int git = it0 + it;
                const int st = git % kKvStages;
                if (git >= kKvStages &&
                    !__all_sync(0xffffffffu, mbar_wait(&bars[kA_QEmpty + st], ((git / kKvStages) - 1) & 1,
                                                       a.status, abort_flag))) {
                    ok = false;
                    break;
                }
                int g, tq0;
                block_of(I, it, &g, &tq0);
                float cl[2] = {nl[0], nl[1]}, cd[2] = {nd[0], nd[1]};
                if (it + 1 < I.n_it) fetch_stats(it + 1);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int rr = lane + 32 * h2;                 // query row of the block
                    const float bl = -cl[h2] * inv_scale;
                    const float bd = -cd[h2];
                    const float lh = __bfloat162float(__float2bfloat16_rn(bl));
                    const float ll = bl == -INFINITY ? 0.0f : bl - lh;
                    const float dh = __bfloat162float(__float2bfloat16_rn(bd));
                    const float dl = bd - dh;
                    const uint32_t o0 = bias_chunk(rr, 0);
                    *reinterpret_cast<uint4*>(smem + Lay::kAL + st * Lay::kBiasQ + o0) = make_uint4(pack_bf16(lh, ll), 0u, 0u, 0u);
                    *reinterpret_cast<uint4*>(smem + Lay::kAD + st * Lay::kBiasQ + o0) = make_uint4(pack_bf16(dh, dl), 0u, 0u, 0u);
                }
                fence_proxy_async_smem();   // generic writes -> the tensor core's reads
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars[kA_QFull + st], 2 * Lay::kQTile);
                    for (int s = 0; s < Lay::kSlabs; ++s) {
                        unsigned char* dq_ = smem + Lay::kQ + st * Lay::kQTile + s * kKvSlab;
                        unsigned char* ddo = smem + Lay::kDO + st * Lay::kQTile + s * kKvSlab;
                        if (kTok) {   // box (64, G, TB, 1): rows t * G + g
                            tma_load_4d(dq_, &a.tq, &bars[kA_QFull + st], s * 64, 0, tq0, I.bh);
                            tma_load_4d(ddo, &a.tdo, &bars[kA_QFull + st], s * 64, 0, tq0, I.bh);
                        } else {
                            const int qh = I.b * a.Hq + I.hk * a.G + g;
                            tma_load_3d(dq_, &a.tq, &bars[kA_QFull + st], s * 64, tq0, qh);
                            tma_load_3d(ddo, &a.tdo, &bars[kA_QFull + st], s * 64, tq0, qh);
                        }
                    }
                }
                issued = git + 1;
            }
            it0 += I.n_it;
            ++n_done;
        }
        // Let every load this warp started land before the CTA retires.
        if (lane == 0) {
            if (n_done > 0) mbar_wait(&bars[kA_KVFull], (n_done - 1) & 1, a.status, abort_flag);
            for (int it = max(0, issued - kKvStages); it < issued; ++it)
                mbar_wait(&bars[kA_QFull + it % kKvStages], (it / kKvStages) & 1, a.status, abort_flag);
        }
    } else if (warp == 1 || warp == kKvGradWarp) {
        // Two issuers on different sub-partitions: warp 1 the score products
        // S^T, dP^T, warp kKvGradWarp the gradient products dV, dK.  One
        // elected thread of each runs the loop; a commit tracks only its own
        // thread's MMAs.  The two halves of an iteration are chained
        // separately -- S^T -> P^T -> dV and dP^T -> dS^T -> dK -- so the math
        // warps start on P while dP^T is still computing, and dV runs while
        // they compute dS.
        if (elect_one()) {
            const uint32_t id_s = idesc_bf16(128, kKvBQ, false, false);
            const uint32_t id_g = idesc_bf16(128, D, false, true);
            const uint64_t kd0 = desc_kmajor_sw128(smem_u32(smem + Lay::kK));
            const uint64_t vd0 = desc_kmajor_sw128(smem_u32(smem + Lay::kV));
            const uint64_t ad0 = desc_noswizzle(smem_u32(smem + Lay::kAA), kBiasLbo, kBiasSbo);
            bool ok = true;
            int it0 = 0, n_done = 0;
            for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
                const int idx = item_of(rnd);
                if (idx >= a.n_items) continue;
                const Item I = decode(idx);
                if (warp == 1) {
                    // the item's K and V tiles
                    if (!mbar_wait(&bars[kA_KVFull], n_done & 1, a.status, abort_flag)) { ok = false; break; }
                    for (int it = 0; it < I.n_it; ++it) {
                        const int git = it0 + it;
                        const int st = git % kKvStages;
                        const int buf = git & 1;
                        if (!mbar_wait(&bars[kA_QFull + st], (git / kKvStages) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        // S^T = K Q^T - LSE/scale into the S columns of buffer buf,
                        // which held P^T two iterations back: its dV product must be done
                        if (git >= 2 &&
                            !mbar_wait(&bars[kA_SFree + buf], ((git - 2) >> 1) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t qd = desc_kmajor_sw128(smem_u32(smem + Lay::kQ + st * Lay::kQTile));
                        const uint64_t dd = desc_kmajor_sw128(smem_u32(smem + Lay::kDO + st * Lay::kQTile));
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t offk = ((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4;
                            const uint64_t offq = ((kk >> 2) * kKvSlab + (kk & 3) * 32) >> 4;
                            umma_ss(tmem + buf * 64, kd0 + offk, qd + offq, id_s, kk > 0 ? 1u : 0u);
                        }
                        umma_ss(tmem + buf * 64, ad0,
                                desc_noswizzle(smem_u32(smem + Lay::kAL + st * Lay::kBiasQ), kBiasLbo, kBiasSbo),
                                id_s, 1u);
                        umma_commit(&bars[kA_SFull + buf]);
                        // dP^T = V dO^T - D over dS^T of two iterations back: its dK
                        // product must be done (that iteration's stage release)
                        // and, with stored dS, the store warps must have read it
                        if (git >= 2 && !mbar_wait(&bars[kA_QEmpty + (git - 2) % kKvStages],
                                                   ((git - 2) / kKvStages) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (git >= 2 && a.dS &&
                            !mbar_wait(&bars[kA_DSRead + buf], ((git - 2) >> 1) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t offk = ((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4;
                            const uint64_t offq = ((kk >> 2) * kKvSlab + (kk & 3) * 32) >> 4;
                            umma_ss(tmem + 128 + buf * 64, vd0 + offk, dd + offq, id_s, kk > 0 ? 1u : 0u);
                        }
                        umma_ss(tmem + 128 + buf * 64, ad0,
                                desc_noswizzle(smem_u32(smem + Lay::kAD + st * Lay::kBiasQ), kBiasLbo, kBiasSbo),
                                id_s, 1u);
                        umma_commit(&bars[kA_DPFull + buf]);
                    }
                } else {
                    for (int it = 0; it < I.n_it; ++it) {
                        const int git = it0 + it;
                        const int st = git % kKvStages;
                        const int buf = git & 1;
                        const uint32_t acc0 = it > 0 ? 1u : 0u;
                        // dV += P^T dO (A: P^T from TMEM), then release the S columns
                        if (!mbar_wait(&bars[kA_PReady + buf], (git >> 1) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        // an item's first products overwrite dV / dK: the math
                        // warps must have read out the previous item's
                        if (it == 0 && n_done > 0 &&
                            !mbar_wait(&bars[kA_AccFree], (n_done - 1) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t dmn = desc_mnmajor_sw128(smem_u32(smem + Lay::kDO + st * Lay::kQTile), kKvSlab);
#pragma unroll
                        for (int kk = 0; kk < kKvBQ / 16; ++kk)
                            umma_ts(tmem + 256, tmem + buf * 64 + kk * 8, dmn + kk * (2048 >> 4), id_g,
                                    kk > 0 ? 1u : acc0);
                        umma_commit(&bars[kA_SFree + buf]);
                        // dK += dS^T Q, then release the Q/dO stage (and dS^T)
                        if (!mbar_wait(&bars[kA_DSReady + buf], (git >> 1) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t qmn = desc_mnmajor_sw128(smem_u32(smem + Lay::kQ + st * Lay::kQTile), kKvSlab);
#pragma unroll
                        for (int kk = 0; kk < kKvBQ / 16; ++kk)
                            umma_ts(tmem + 384, tmem + 128 + buf * 64 + kk * 8, qmn + kk * (2048 >> 4), id_g,
                                    kk > 0 ? 1u : acc0);
                        umma_commit(&bars[kA_QEmpty + st]);
                    }
                    umma_commit(&bars[kA_Final]);
                }
                it0 += I.n_it;
                ++n_done;
            }
        }
        __syncwarp();
    } else if (warp >= kKvStoreWarp0) {
        // Store warps (stored dS only): once the math warps have written an
        // iteration's dS^T into TMEM (DSReady), each reads its lane quarter's
        // 32 key rows x 64 packed queries, releases the buffer for the next
        // score products (DSRead) and writes the rows into the dQ kernel's
        // tiles -- off the math warps' path.
        if (a.dS) {
            const int quarter = warp & 3;
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            bool ok = true;
            int it0 = 0;
            for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
                const int idx = item_of(rnd);
                if (idx >= a.n_items) continue;
                const Item I = decode(idx);
                const int k = I.kt * BN + quarter * 32 + lane;
                for (int it = 0; it < I.n_it; ++it) {
                    int g, tq0;
                    block_of(I, it, &g, &tq0);
                    const int git = it0 + it;
                    const int buf = git & 1;
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars[kA_DSReady + buf], (git >> 1) & 1, a.status,
                                                           abort_flag))) { ok = false; break; }
                    tc_fence_after();
                    uint32_t v[32];
                    tmem_ld32(lane_base + 128 + buf * 64, v);
                    tmem_wait_ld();
                    reg_fence<32>(v);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[kA_DSRead + buf]);
                    store_ds_row(a, I.bh, k, tq0, v);
                }
                it0 += I.n_it;
            }
        }
    } else {
        // Math warps 2..9: two per TMEM lane quarter, each on 16 key rows;
        // threads t and t + 16 of a warp share a key row and hold query
        // columns [0, 32) and [32, 64) of the block (16x32bx2 TMEM shapes).
        const int quarter = warp & 3;
        const int sub = (warp - 2) >> 2;
        const int half = lane >> 4;
        const int kr = quarter * 32 + sub * 16 + (lane & 15);   // key row within the tile
        const int c0 = half * 32;                          // first query column of this thread
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32 + sub * 16) << 16);
        const float sl2 = a.scale_log2;
        bool ok = true;
        int it0 = 0, n_done = 0;
        for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
            const int idx = item_of(rnd);
            if (idx >= a.n_items) continue;
            const Item I = decode(idx);
            const int k = I.kt * BN + kr;
            for (int it = 0; it < I.n_it; ++it) {
                int g, tq0;
                block_of(I, it, &g, &tq0);
                const int git = it0 + it;
                const int buf = git & 1;
                // P^T = 2^(scale*log2(e) * (s - LSE/scale)) once S^T is in
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[kA_SFull + buf], (git >> 1) & 1, a.status,
                                                       abort_flag))) { ok = false; break; }
                tc_fence_after();
                const bool diag = a.causal && tq0 < I.kt * BN + BN;   // some key after some query
                uint32_t s[32], dp[32], pk[16], dk[16];
                tmem_ld16x2_32<32>(lane_base + buf * 64, s);          // s - LSE/scale
                tmem_wait_ld();
                reg_fence<32>(s);
                if (!diag) {                   // every column visible (CTA-uniform branch)
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[e] = __float_as_uint(ex2(__uint_as_float(s[e]) * sl2));
                } else {
                    // visible columns: token >= k, i.e. c >= k - tq0 (head by head)
                    // or c >= (k - tq0) * G (token-major); a select, no branch per
                    // element (masked: score -inf, so P = dS = 0)
                    const int vlo = (kTok ? (k - tq0) * a.G : k - tq0) - c0;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        s[e] = __float_as_uint(ex2((e >= vlo ? __uint_as_float(s[e]) : -INFINITY) * sl2));
                }
#pragma unroll
                for (int e = 0; e < 32; e += 2) pk[e / 2] = pack_bf16(__uint_as_float(s[e]), __uint_as_float(s[e + 1]));
                // P^T (bf16 pairs) over the S columns this warp has read
                __syncwarp();
                tmem_st16x2_16<16>(lane_base + buf * 64, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kA_PReady + buf]);
                // dS^T = P^T * (dP^T - D) once dP^T is in
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[kA_DPFull + buf], (git >> 1) & 1, a.status,
                                                       abort_flag))) { ok = false; break; }
                tc_fence_after();
                tmem_ld16x2_32<32>(lane_base + 128 + buf * 64, dp);   // dP - D
                tmem_wait_ld();
                reg_fence<32>(dp);
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    dk[e / 2] = pack_bf16(__uint_as_float(s[e]) * __uint_as_float(dp[e]),
                                          __uint_as_float(s[e + 1]) * __uint_as_float(dp[e + 1]));
                __syncwarp();
                tmem_st16x2_16<16>(lane_base + 128 + buf * 64, dk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kA_DSReady + buf]);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kA_Final], n_done & 1, a.status, abort_flag));
            if (ok) {
                tc_fence_after();
                // dK (scaled) then dV; this thread writes columns [half*D/2, (half+1)*D/2).
                // Once both are in registers the next item's products may overwrite them.
#pragma unroll
                for (int which = 0; which < 2; ++which) {
                    uint32_t gr[D / 2];
#pragma unroll
                    for (int c = 0; c < D / 2; c += 32)
                        tmem_ld16x2_32<D / 2>(lane_base + (which ? 256 : 384) + c, gr + c);
                    tmem_wait_ld();
                    reg_fence<D / 2>(gr);
                    if (which == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars[kA_AccFree]);
                    }
                    if (k < a.T) {
                        const size_t row = static_cast<size_t>(I.bh) * a.T + k;
                        uint4* dst = reinterpret_cast<uint4*>((which ? a.dV : a.dK) + row * D + half * (D / 2));
                        const float sc = which ? 1.0f : a.scale;
#pragma unroll
                        for (int c = 0; c < D / 2; c += 8) {
                            uint4 u;
                            u.x = pack_bf16(__uint_as_float(gr[c]) * sc, __uint_as_float(gr[c + 1]) * sc);
                            u.y = pack_bf16(__uint_as_float(gr[c + 2]) * sc, __uint_as_float(gr[c + 3]) * sc);
                            u.z = pack_bf16(__uint_as_float(gr[c + 4]) * sc, __uint_as_float(gr[c + 5]) * sc);
                            u.w = pack_bf16(__uint_as_float(gr[c + 6]) * sc, __uint_as_float(gr[c + 7]) * sc);
                            dst[c / 8] = u;
                        }
                    }
                }
            }
            it0 += I.n_it;
            ++n_done;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- 3. dq ----
// Key and depth blocks are 64 rows, so S and dP are double-buffered in TMEM:
// the MMAs of block i+1 run while the math warps work on block i.
//   TMEM columns: S0 [0,64) S1 [64,128) | dP0 [128,192) dP1 [192,256) |
//                 dQ [256, 256+D) | dKd^T [384,448) | dVd^T [448,512)
struct DqArgs {
    TmaMap tq, tdo, tk, tv, tkd, tvd;
    const float* LSE;
    const float* Drow;
    __nv_bfloat16* dQ;
    __nv_bfloat16* dKd;
    __nv_bfloat16* dVd;
    unsigned int* status;
    int B, Hq, Hk, T, L, G, Tq, n_qt, dep_rows;
    int causal, win_lo;
    int band;                            // (b, KV head) pairs per band (banded_item)
    float scale, scale_log2;
    const unsigned char* dS;             // stored dS tiles (written by the dK/dV kernel), kStored only
    int n_kb;                            // 64-key blocks per head
    int g_log2;                          // kStored: G = 1 << g_log2
    int layer;                           // Kd, Vd, dKd, dVd layer-major [L, B, Hk, T, d]
};

constexpr int kDqBN = 64;            // rows per key / depth block
constexpr int kDqStages = 4;         // K/V ring depth (stored dS: K + dS tile per stage)
constexpr uint32_t kDqSlab = 64 * 128;   // 64 rows x 64 bf16

template <int D>
struct DqLayout {
    static constexpr int kSlabs = D / 64;
    static constexpr uint32_t kQTile = kSlabs * kSlabBytes;      // 128 rows
    static constexpr uint32_t kKTile = kSlabs * kDqSlab;         // 64 rows
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kDO = kQTile;
    static constexpr uint32_t kK = 2 * kQTile;                   // kDqStages stages
    static constexpr uint32_t kV = kK + kDqStages * kKTile;      // kDqStages stages
    static constexpr uint32_t kDS = kV + kDqStages * kKTile;     // [128 q][64 depth] bf16, 128-B swizzle
    static constexpr uint32_t kP = kDS + kSlabBytes;
    static constexpr uint32_t kBar = kP + kSlabBytes;
    static constexpr uint32_t kBytes = kBar + 256;
    static constexpr uint32_t kDynSmem = kBytes + 1024 > 120u * 1024 ? kBytes + 1024 : 120u * 1024;
};

enum { kB_QFull = 0, kB_KVFull = 1, kB_KVEmpty = 1 + kDqStages, kB_SFull = 1 + 2 * kDqStages,
       kB_PReady = 3 + 2 * kDqStages, kB_DDFull = 5 + 2 * kDqStages, kB_Final = 6 + 2 * kDqStages,
       kB_NumBars = 7 + 2 * kDqStages };

constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColDKd = 384, kColDVd = 448;

// One bf16 to global memory with the streaming (evict-first) cache hint.
__device__ __forceinline__ void st_cs_bf16(__nv_bfloat16* p, __nv_bfloat16 v) {
    asm volatile("st.global.cs.b16 [%0], %1;" ::"l"(p), "h"(*reinterpret_cast<const unsigned short*>(&v))
                 : "memory");
}

// dK_d, dV_d of one thread's 32 depth rows (its d index fixed) into the
// layer-major tensors, when the rows are 32 / kL whole tokens: layer outer,
// token inner, so the warps of a depth block write each layer plane's rows
// together, and with the streaming hint, so those L2 lines leave for DRAM
// together, instead of hopping across the kL planes row by row (which left
// the lines of a plane to scattered evictions: dQ 0.306 against 0.246 ms at
// the layer workload).  base: element index of (layer 0, the first row's
// token, this d); lstride: elements between layer planes.
template <int kL>
__device__ __forceinline__ void store_depth_grads_layer(__nv_bfloat16* dKd, __nv_bfloat16* dVd, size_t base,
                                                        size_t lstride, int nvalid, float scale, int D,
                                                        const uint32_t* xk, const uint32_t* xv) {
    constexpr int kTok = 32 / kL;
#pragma unroll
    for (int l = 0; l < kL; ++l) {
#pragma unroll
        for (int tk = 0; tk < kTok; ++tk) {
            const int c = tk * kL + l;
            if (c < nvalid) {
                const size_t off = base + l * lstride + static_cast<size_t>(tk) * D;
                st_cs_bf16(dKd + off, __float2bfloat16_rn(__uint_as_float(xk[c]) * scale));
                st_cs_bf16(dVd + off, __float2bfloat16_rn(__uint_as_float(xv[c])));
            }
        }
    }
}

// kStored: the sequence part reads the dS tiles the dK/dV kernel stored
// (dQ += dS K straight from shared memory, no recomputation of S and dP, no
// math); the tile's depth blocks come first and run as before.  Otherwise
// every block recomputes S and dP, sequence blocks first.
template <int D, bool kStored>
__global__ void __launch_bounds__(kThreads, 1) dq_kernel(const __grid_constant__ DqArgs a) {
    using Lay = DqLayout<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kB_NumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nbh = a.B * a.Hk;
    int outer, bh;
    banded_item(static_cast<int>(blockIdx.x), a.n_qt, nbh, a.band, &outer, &bh);
    const int qt = a.n_qt - 1 - outer;                  // longest query tiles first
    const int b = bh / a.Hk;
    const int hk = bh - b * a.Hk;
    const int t0 = qt * a.Tq;
    const int R = a.G * a.Tq;
    const int t_end = min(t0 + a.Tq, a.T);
    const int n_seq = ((a.causal ? t_end : a.T) - 1) / kDqBN + 1;
    const int dep_total = a.L > 0 ? (t_end - t0) * a.L : 0;
    const int n_dep = (dep_total + a.dep_rows - 1) / a.dep_rows;
    const int nb = n_seq + n_dep;
    // Block i of the tile, in the order of the variant.
    auto is_dep = [&](int i) { return kStored ? i < n_dep : i >= n_seq; };
    auto seq_idx = [&](int i) { return kStored ? i - n_dep : i; };
    auto dep_idx = [&](int i) { return kStored ? i : i - n_seq; };

    if (threadIdx.x == 0) {
        mbar_init(&bars[kB_QFull], 1);
        for (int s = 0; s < kDqStages; ++s) {
            mbar_init(&bars[kB_KVFull + s], 1);
            mbar_init(&bars[kB_KVEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kB_SFull + s], 1);
            mbar_init(&bars[kB_PReady + s], kMathThreads);
        }
        mbar_init(&bars[kB_DDFull], 1);
        mbar_init(&bars[kB_Final], 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (R < BM) {  // rows the Q / dO boxes do not cover: zeros
        const int per = (BM - R) * 8;
        for (int i = threadIdx.x; i < 2 * Lay::kSlabs * per; i += kThreads) {
            const int which = i / (Lay::kSlabs * per);       // 0: Q, 1: dO
            const int rem0 = i - which * Lay::kSlabs * per;
            const int slab = rem0 / per;
            const int rem = rem0 - slab * per;
            const int row = R + rem / 8;
            reinterpret_cast<uint4*>(smem + (which ? Lay::kDO : Lay::kQ) + slab * kSlabBytes +
                                     row * 128)[rem % 8] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        if (lane == 0) {
            prefetch_tmap(&a.tq); prefetch_tmap(&a.tdo); prefetch_tmap(&a.tk); prefetch_tmap(&a.tv);
            if (a.L > 0) { prefetch_tmap(&a.tkd); prefetch_tmap(&a.tvd); }
            const uint32_t q_bytes = Lay::kSlabs * 128u * a.Tq * a.G;
            const uint64_t once = policy_evict_first();
            mbar_arrive_expect_tx(&bars[kB_QFull], 2 * q_bytes);
            for (int s = 0; s < Lay::kSlabs; ++s) {
                if (kStored) {   // token-major: box (64, G, Tq, 1) lands as rows t * G + g
                    tma_load_4d(smem + Lay::kQ + s * kSlabBytes, &a.tq, &bars[kB_QFull], s * 64, 0, t0, bh);
                    tma_load_4d(smem + Lay::kDO + s * kSlabBytes, &a.tdo, &bars[kB_QFull], s * 64, 0, t0, bh);
                } else {
                    tma_load_3d(smem + Lay::kQ + s * kSlabBytes, &a.tq, &bars[kB_QFull], s * 64, t0, b * a.Hq + hk * a.G);
                    tma_load_3d(smem + Lay::kDO + s * kSlabBytes, &a.tdo, &bars[kB_QFull], s * 64, t0, b * a.Hq + hk * a.G);
                }
            }
            int issued = 0;
            for (int i = 0; i < nb; ++i) {
                const int st = i % kDqStages;
                if (i >= kDqStages &&
                    !mbar_wait(&bars[kB_KVEmpty + st], ((i / kDqStages) - 1) & 1, a.status, abort_flag))
                    break;
                // this kernel may have started before the dK/dV kernel ended
                // (programmatic dependent launch): the stored dS tiles are
                // read only after that grid has completed
                if (kStored && i == n_dep) griddep_wait();
                unsigned char* dk = smem + Lay::kK + st * Lay::kKTile;
                unsigned char* dv = smem + Lay::kV + st * Lay::kKTile;
                const bool seq = !is_dep(i);
                const int row0 = seq ? seq_idx(i) * kDqBN : t0 * a.L + dep_idx(i) * a.dep_rows;
                const uint32_t bytes = Lay::kSlabs * 128u * (seq ? kDqBN : a.dep_rows);
                if (kStored && seq) {
                    // K tile by TMA into the K slot, the stored dS tile (16 KB,
                    // already in operand layout) by one bulk copy into the V slot
                    static_assert(!kStored || Lay::kKTile == kDsTileBytes, "dS tile must fill the V slot");
                    const unsigned char* tile =
                        a.dS + (static_cast<size_t>(bh * a.n_qt + qt) * a.n_kb + seq_idx(i)) * kDsTileBytes;
                    mbar_arrive_expect_tx(&bars[kB_KVFull + st], bytes + kDsTileBytes);
                    for (int s = 0; s < Lay::kSlabs; ++s)
                        tma_load_3d(dk + s * kDqSlab, &a.tk, &bars[kB_KVFull + st], s * 64, row0, bh);
                    bulk_load_hint(dv, tile, kDsTileBytes, &bars[kB_KVFull + st], once);
                    issued = i + 1;
                    continue;
                }
                const void* mk = seq ? static_cast<const void*>(&a.tk) : static_cast<const void*>(&a.tkd);
                const void* mv = seq ? static_cast<const void*>(&a.tv) : static_cast<const void*>(&a.tvd);
                mbar_arrive_expect_tx(&bars[kB_KVFull + st], 2 * bytes);
                for (int s = 0; s < Lay::kSlabs; ++s) {
                    if (seq) {
                        tma_load_3d(dk + s * kDqSlab, mk, &bars[kB_KVFull + st], s * 64, row0, bh);
                        tma_load_3d(dv + s * kDqSlab, mv, &bars[kB_KVFull + st], s * 64, row0, bh);
                    } else if (a.layer) {   // box (64, L, dep_rows / L, 1): whole tokens from row0 / L
                        tma_load_4d_hint(dk + s * kDqSlab, mk, &bars[kB_KVFull + st], s * 64, 0, row0 / a.L, bh, once);
                        tma_load_4d_hint(dv + s * kDqSlab, mv, &bars[kB_KVFull + st], s * 64, 0, row0 / a.L, bh, once);
                    } else {   // depth tiles are read exactly once
                        tma_load_3d_hint(dk + s * kDqSlab, mk, &bars[kB_KVFull + st], s * 64, row0, bh, once);
                        tma_load_3d_hint(dv + s * kDqSlab, mv, &bars[kB_KVFull + st], s * 64, row0, bh, once);
                    }
                }
                issued = i + 1;
            }
            mbar_wait(&bars[kB_QFull], 0, a.status, abort_flag);
            for (int i = max(0, issued - kDqStages); i < issued; ++i)
                mbar_wait(&bars[kB_KVFull + i % kDqStages], (i / kDqStages) & 1, a.status, abort_flag);
        }
    } else if (warp == 1 || warp == 6) {
        // ------------------------------------------------------ MMA issuers -
        // Two warps on different sub-partitions share the issue work: warp 6
        // the score products S(j), dP(j); warp 1 dQ(i) and the depth
        // gradients.  One elected thread of each runs the loop; a commit
        // tracks only its own thread's MMAs, and the waits below order every
        // TMEM reuse across the two.
        if (elect_one()) {
            const uint32_t id_seq = idesc_bf16(128, kDqBN, false, false);
            const uint32_t id_dep = idesc_bf16(128, a.dep_rows, false, false);
            const uint32_t id_dq = idesc_bf16(128, D, false, true);
            const uint32_t id_dd = idesc_bf16(128, a.dep_rows, true, true);
            const uint32_t q_addr = smem_u32(smem + Lay::kQ);
            const uint32_t do_addr = smem_u32(smem + Lay::kDO);
            const uint32_t ds_addr = smem_u32(smem + Lay::kDS);
            const uint32_t p_addr = smem_u32(smem + Lay::kP);
            const uint64_t qd0 = desc_kmajor_sw128(q_addr);
            const uint64_t dod0 = desc_kmajor_sw128(do_addr);
            // S(j) = Q K_j^T and dP(j) = dO V_j^T into buffer j & 1.
            auto issue_s = [&](int j) -> bool {
                const int st = j % kDqStages;
                const int buf = j & 1;
                if (!mbar_wait(&bars[kB_KVFull + st], (j / kDqStages) & 1, a.status, abort_flag)) return false;
                tc_fence_after();
                const uint32_t id = is_dep(j) ? id_dep : id_seq;
                const uint64_t kd = desc_kmajor_sw128(smem_u32(smem + Lay::kK + st * Lay::kKTile));
                const uint64_t vd = desc_kmajor_sw128(smem_u32(smem + Lay::kV + st * Lay::kKTile));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t offq = ((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4;
                    const uint64_t offk = ((kk >> 2) * kDqSlab + (kk & 3) * 32) >> 4;
                    umma_ss(tmem + kColS + buf * 64, qd0 + offq, kd + offk, id, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t offq = ((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4;
                    const uint64_t offk = ((kk >> 2) * kDqSlab + (kk & 3) * 32) >> 4;
                    umma_ss(tmem + kColDP + buf * 64, dod0 + offq, vd + offk, id, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[kB_SFull + buf]);
                return true;
            };
            if (warp == 6) {
                // kStored: only the depth blocks (blocks 0 .. n_dep-1) need S and dP
                const int n_sdp = kStored ? n_dep : nb;
                bool ok = mbar_wait(&bars[kB_QFull], 0, a.status, abort_flag);
                for (int j = 0; ok && j < n_sdp; ++j) {
                    // buffer j & 1 last held dS(j-2), which dQ(j-2) reads: wait
                    // until that has completed (its K/V-stage release)
                    if (j >= 2 && !mbar_wait(&bars[kB_KVEmpty + (j - 2) % kDqStages], ((j - 2) / kDqStages) & 1,
                                             a.status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!issue_s(j)) { ok = false; break; }
                }
            } else {
                bool ok = true;
                const uint32_t id_dqs = idesc_bf16(128, D, true, true);   // A = stored dS, MN-major
                for (int i = 0; ok && i < nb; ++i) {
                    const int st = i % kDqStages;
                    const int buf = i & 1;
                    const bool seq = !is_dep(i);
                    if (kStored && seq) {
                        // dQ += dS K: A = the dS tile in the V slot (MN-major,
                        // no swizzle: 8 keys 128 B apart, 8 rows 1024 B apart; 16
                        // keys = 256 B per K step), B = the K tile, MN-major
                        if (!mbar_wait(&bars[kB_KVFull + st], (i / kDqStages) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + Lay::kV + st * Lay::kKTile);
                        const uint64_t kmn = desc_mnmajor_sw128(smem_u32(smem + Lay::kK + st * Lay::kKTile), kDqSlab);
#pragma unroll
                        for (int kk = 0; kk < kDqBN / 16; ++kk)
                            umma_ss(tmem + kColDQ, desc_mnmajor_noswizzle(a_addr + kk * 256, 128, 1024),
                                    kmn + kk * (2048 >> 4), id_dqs, (i > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&bars[kB_KVEmpty + st]);
                        continue;
                    }
                    const int n = seq ? kDqBN : a.dep_rows;
                    if (!mbar_wait(&bars[kB_PReady + buf], (i >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t kmn = desc_mnmajor_sw128(smem_u32(smem + Lay::kK + st * Lay::kKTile), kDqSlab);
                    // depth block: the gradient products first, so their
                    // completion (which the math warps wait for before the next
                    // depth block) does not queue behind this block's dQ.  Their
                    // K dimension is the tile's query rows, and P', dS' are zero
                    // outside the rows of the block's own tokens (each query
                    // row sees only its own token's depth rows), so only the
                    // 16-row K steps that hold such rows are issued.
                    if (!seq) {
                        const int r0 = dep_idx(i) * a.dep_rows;
                        const int tok_lo = r0 / a.L;
                        const int tok_hi = (min(r0 + a.dep_rows, dep_total) - 1) / a.L;
                        uint32_t steps = 0xffu;
                        if (kStored) {       // token-major: rows [tok_lo * G, (tok_hi + 1) * G)
                            const int s0 = (tok_lo << a.g_log2) >> 4;
                            const int s1 = (min((tok_hi + 1) << a.g_log2, R) - 1) >> 4;
                            steps = ((2u << s1) - 1u) & ~((1u << s0) - 1u);
                        } else if (a.G <= 8) {
                            steps = 0;
                            for (int g = 0, base = 0; g < a.G && base < R; ++g, base += a.Tq) {
                                const int s0 = (base + tok_lo) >> 4;
                                const int s1 = min(base + tok_hi, R - 1) >> 4;
                                steps |= ((2u << s1) - 1u) & ~((1u << s0) - 1u);
                            }
                            if (steps == 0) steps = 1;   // (cannot happen) keep the accumulators defined
                        }
                        uint32_t acc = 0;
#pragma unroll
                        for (int kk = 0; kk < BM / 16; ++kk) {
                            if (!((steps >> kk) & 1u)) continue;
                            umma_ss(tmem + kColDKd, desc_mnmajor_sw128(q_addr + kk * 2048, kSlabBytes),
                                    desc_mnmajor_sw128(ds_addr + kk * 2048, kSlabBytes), id_dd, acc);
                            umma_ss(tmem + kColDVd, desc_mnmajor_sw128(do_addr + kk * 2048, kSlabBytes),
                                    desc_mnmajor_sw128(p_addr + kk * 2048, kSlabBytes), id_dd, acc);
                            acc = 1;
                        }
                        umma_commit(&bars[kB_DDFull]);
                    }
                    // dS of keys [16kk, 16kk + 16) sits at column (kk / 2) * 32 +
                    // (kk % 2) * 8 of the buffer (each math half packs its 32 keys
                    // into the first 16 of its own 32 columns)
                    if (n == kDqBN) {
#pragma unroll
                        for (int kk = 0; kk < kDqBN / 16; ++kk)
                            umma_ts(tmem + kColDQ, tmem + kColS + buf * 64 + (kk >> 1) * 32 + (kk & 1) * 8,
                                    kmn + kk * (2048 >> 4), id_dq, (i > 0 || kk > 0) ? 1u : 0u);
                    } else {
                        for (int kk = 0; kk < n / 16; ++kk)
                            umma_ts(tmem + kColDQ, tmem + kColS + buf * 64 + (kk >> 1) * 32 + (kk & 1) * 8,
                                    kmn + kk * (2048 >> 4), id_dq, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&bars[kB_KVEmpty + st]);
                }
                umma_commit(&bars[kB_Final]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ math --------
        // Warps 2..5 and 7..10: two per TMEM lane quarter (they share its
        // sub-partition and interleave).  Thread = query row r; the warp's
        // half takes columns [c0, c0 + 32) of every 64-row block.  Rows are
        // token-major with stored dS (r = t * G + g: a warp's 32 rows are
        // 32 / G tokens, so most depth blocks hold none of its rows' depth
        // rows and the warp skips them), head by head otherwise (r = g * Tq + t).
        const int quarter = warp & 3;
        const int half = warp >= 7 ? 1 : 0;
        const int c0 = 32 * half;
        const int r = quarter * 32 + lane;
        const bool row_real = r < R;
        const int g = row_real ? (kStored ? r & (a.G - 1) : r / a.Tq) : 0;
        const int t_row = row_real ? t0 + (kStored ? r >> a.g_log2 : r - g * a.Tq) : t0;
        const bool row_live = row_real && t_row < a.T;
        const size_t qrow = (static_cast<size_t>(b) * a.Hq + hk * a.G + g) * a.T + t_row;
        const float lse2 = row_live ? a.LSE[qrow] * kLog2e : INFINITY;
        const float Dr = row_live ? a.Drow[qrow] : 0.0f;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const float sl2 = a.scale_log2;
        unsigned char* sDS = smem + Lay::kDS;
        unsigned char* sP = smem + Lay::kP;
        const size_t dep_base = (static_cast<size_t>(bh) * a.T + t0) * a.L;  // first depth row of the tile

        // dKd / dVd of depth block jd: TMEM lane = d index, column = depth row,
        // so for each depth row the four warps of a half store 128 consecutive
        // d values (64 contiguous bytes per warp) straight to global memory;
        // the half takes depth rows [c0, c0 + 32) of the block.
        // The accumulators are read into registers (epi_load) before the next
        // depth block's gradient MMAs may overwrite them, and written out
        // (epi_store) after this thread's P-ready arrive, so the global stores
        // are off the serial chain MMA -> read-out -> next block's MMA.
        auto epi_load = [&](uint32_t* xk, uint32_t* xv) {
            tmem_ld32(lane_base + kColDKd + c0, xk);
            tmem_ld32(lane_base + kColDVd + c0, xv);
            tmem_wait_ld();
            reg_fence<32>(xk);
            reg_fence<32>(xv);
        };
        auto epi_store = [&](int jd, const uint32_t* xk, const uint32_t* xv) {
            if (r < D) {
                const int row0 = jd * a.dep_rows + c0;
                const int nvalid = min(a.dep_rows, dep_total - jd * a.dep_rows) - c0;
                if (a.layer && a.L <= 16 && 32 % a.L == 0) {
                    // whole tokens per thread (32 % L == 0 and row0 % L == 0: L
                    // divides the depth blocks and 32)
                    const size_t lstride = static_cast<size_t>(a.B) * a.Hk * a.T * D;
                    const size_t base = (static_cast<size_t>(bh) * a.T + t0 + row0 / a.L) * D + r;
                    switch (a.L) {
                        case 1: store_depth_grads_layer<1>(a.dKd, a.dVd, base, lstride, nvalid, a.scale, D, xk, xv); break;
                        case 2: store_depth_grads_layer<2>(a.dKd, a.dVd, base, lstride, nvalid, a.scale, D, xk, xv); break;
                        case 4: store_depth_grads_layer<4>(a.dKd, a.dVd, base, lstride, nvalid, a.scale, D, xk, xv); break;
                        case 8: store_depth_grads_layer<8>(a.dKd, a.dVd, base, lstride, nvalid, a.scale, D, xk, xv); break;
                        default: store_depth_grads_layer<16>(a.dKd, a.dVd, base, lstride, nvalid, a.scale, D, xk, xv); break;
                    }
                } else if (a.layer) {
                    // depth row q of the tile = token t0 + q / L, layer q % L, at
                    // row (l * B * Hk + bh) * T + t of the layer-major tensors
                    const size_t lstride = static_cast<size_t>(a.B) * a.Hk * a.T * D;
                    int tq = row0 / a.L;
                    int l = row0 - tq * a.L;
                    size_t off = static_cast<size_t>(l) * lstride + (static_cast<size_t>(bh) * a.T + t0 + tq) * D + r;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (c < nvalid) {
                            a.dKd[off] = __float2bfloat16_rn(__uint_as_float(xk[c]) * a.scale);
                            a.dVd[off] = __float2bfloat16_rn(__uint_as_float(xv[c]));
                        }
                        if (++l == a.L) {
                            l = 0;
                            off += D - static_cast<size_t>(a.L - 1) * lstride;
                        } else {
                            off += lstride;
                        }
                    }
                } else {
                    __nv_bfloat16* gk = a.dKd + (dep_base + row0) * D + r;
                    __nv_bfloat16* gv = a.dVd + (dep_base + row0) * D + r;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (c < nvalid) {
                            st_cs_bf16(gk + static_cast<size_t>(c) * D, __float2bfloat16_rn(__uint_as_float(xk[c]) * a.scale));
                            st_cs_bf16(gv + static_cast<size_t>(c) * D, __float2bfloat16_rn(__uint_as_float(xv[c])));
                        }
                    }
                }
            }
        };

        bool ok = true;
        int jd = 0;
        const int n_math = kStored ? n_dep : nb;      // kStored: depth blocks only (blocks 0 .. n_dep-1)
        for (int i = 0; i < n_math; ++i) {
            const int buf = i & 1;
            const bool seq = !is_dep(i);
            if (!mbar_wait(&bars[kB_SFull + buf], (i >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[32], dp[32], dsk[16], pk[16];
            int lo = 0, hi = kDqBN, kb = 0;
            const int lim = a.causal ? t_row : a.T - 1;   // last visible sequence key
            if (seq) {
                kb = seq_idx(i) * kDqBN;
            } else {
                const int base = t_row * a.L - (t0 * a.L + jd * a.dep_rows);
                lo = base + a.win_lo;
                hi = min(base + a.L, a.dep_rows);
            }
            // A depth block none of the warp's rows can see in its half of the
            // columns (token-major rows): P' and dS' are exactly 0 there, written
            // without loading or exponentiating.
            const bool skip = kStored && !seq &&
                              __all_sync(0xffffffffu, !row_live || max(lo, c0) >= min(hi, c0 + 32));
            const bool all_visible = seq && kb + c0 + 31 <= lim;
            if (!skip) {
                tmem_ld32(lane_base + kColS + buf * 64 + c0, s);
                tmem_ld32(lane_base + kColDP + buf * 64 + c0, dp);
                tmem_wait_ld();
                reg_fence<32>(s);
                reg_fence<32>(dp);
            }
            // Masked entries get score -inf and dP 0 by selects (no branch per
            // element), so exp2 runs unconditionally and yields exactly 0.
            if (skip) {
#pragma unroll
                for (int e = 0; e < 16; ++e) dsk[e] = pk[e] = 0u;
            } else if (all_visible) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float p0 = ex2(fmaf(__uint_as_float(s[e]), sl2, -lse2));
                    const float p1 = ex2(fmaf(__uint_as_float(s[e + 1]), sl2, -lse2));
                    dsk[e / 2] = pack_bf16(p0 * (__uint_as_float(dp[e]) - Dr),
                                           p1 * (__uint_as_float(dp[e + 1]) - Dr));
                    pk[e / 2] = pack_bf16(p0, p1);
                }
            } else {
                // visible block columns: seq c <= t_row - kb; depth lo <= c < hi
                const int vlo = seq ? 0 : lo;
                const int vhi = seq ? lim - kb + 1 : hi;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float p2[2], d2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int c = c0 + e + u;
                        const bool vis = c >= vlo && c < vhi;
                        const float sv = vis ? __uint_as_float(s[e + u]) : -INFINITY;
                        const float dv = vis ? __uint_as_float(dp[e + u]) : Dr;
                        p2[u] = ex2(fmaf(sv, sl2, -lse2));
                        d2[u] = p2[u] * (dv - Dr);
                    }
                    dsk[e / 2] = pack_bf16(d2[0], d2[1]);
                    pk[e / 2] = pack_bf16(p2[0], p2[1]);
                }
            }
            // packed dS of keys [c0, c0 + 32) into columns [c0, c0 + 16): inside
            // this half's own score columns, which only it reads
            tmem_st16(lane_base + kColS + buf * 64 + c0, dsk);
            uint32_t xk[32], xv[32];                      // depth gradients of block jd - 1
            if (!seq) {
                // the previous depth block's MMAs are done before its staging
                // tiles and TMEM columns are reused
                if (jd >= 1) {
                    if (!mbar_wait(&bars[kB_DDFull], (jd - 1) & 1, a.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    epi_load(xk, xv);
                }
                // row r of the [q][depth] staging tiles, 128-byte swizzle;
                // this half's depth columns are 16-byte chunks 4*half .. 4*half+3
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const uint32_t off = r * 128 + (((4 * half + ch) ^ (r & 7)) << 4);
                    *reinterpret_cast<uint4*>(sDS + off) =
                        make_uint4(dsk[4 * ch], dsk[4 * ch + 1], dsk[4 * ch + 2], dsk[4 * ch + 3]);
                    *reinterpret_cast<uint4*>(sP + off) =
                        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
                }
                fence_proxy_async_smem();
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[kB_PReady + buf]);
            if (!seq) {
                if (jd >= 1) epi_store(jd - 1, xk, xv);
                ++jd;
            }
        }
        if (ok && n_dep > 0) {
            if (mbar_wait(&bars[kB_DDFull], (n_dep - 1) & 1, a.status, abort_flag)) {
                tc_fence_after();
                uint32_t xk[32], xv[32];
                epi_load(xk, xv);
                epi_store(n_dep - 1, xk, xv);
            } else {
                ok = false;
            }
        }
        if (ok) ok = mbar_wait(&bars[kB_Final], 0, a.status, abort_flag);
        if (ok) {
            tc_fence_after();
            uint32_t o[D / 2];                                // this half's D/2 columns of dQ
#pragma unroll
            for (int c = 0; c < D / 2; c += 32) tmem_ld32(lane_base + kColDQ + half * (D / 2) + c, o + c);
            tmem_wait_ld();
            reg_fence<D / 2>(o);
            if (row_live) {
                uint4* dst = reinterpret_cast<uint4*>(a.dQ + qrow * D + half * (D / 2));
                const float sc = a.scale;
#pragma unroll
                for (int c = 0; c < D / 2; c += 8) {
                    uint4 v;
                    v.x = pack_bf16(__uint_as_float(o[c]) * sc, __uint_as_float(o[c + 1]) * sc);
                    v.y = pack_bf16(__uint_as_float(o[c + 2]) * sc, __uint_as_float(o[c + 3]) * sc);
                    v.z = pack_bf16(__uint_as_float(o[c + 4]) * sc, __uint_as_float(o[c + 5]) * sc);
                    v.w = pack_bf16(__uint_as_float(o[c + 6]) * sc, __uint_as_float(o[c + 7]) * sc);
                    dst[c / 8] = v;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    // never complete before the dK/dV kernel (this one may have started early)
    if (threadIdx.x == 0) griddep_wait();
}

// The stored-dS backward: d = 128, G in {1, 2, 4, 8} (Tq = 128 / G >= 16, a
// power of two, so a dK/dV thread's 32 queries fall in whole chunks of one or
// two dq tiles), and at most this many bytes of tiles.
constexpr double kMaxStoredDsBytes = 16.0 * 1024 * 1024 * 1024;

// Launch with programmatic stream serialization: the kernel may start before
// the previous kernel in the stream has completed (see griddep_wait).
template <typename Args>
cudaError_t launch_dependent(void (*kernel)(Args), unsigned grid, unsigned threads, uint32_t smem,
                             cudaStream_t stream, const Args& args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args);
}

int log2_exact(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return (1 << l) == x ? l : -1;
}

template <int D>
cudaError_t launch_d(const Problem& p, const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd, const void* O, const float* LSE,
                     const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                     void* ws, size_t ws_bytes, cudaStream_t stream) {
    cudaError_t e;
    float* Dws = static_cast<float*>(ws);
    const size_t ds_bytes = bwd_ds_bytes(p);
    bool stored = ds_bytes > 0 && ws_bytes >= bwd_workspace_bytes(p) + ds_bytes;
    const int Tq = BM / p.G;
    // Stored dS runs both kernels on token-major query rows: Q and dO as
    // (d, head g, token, b * Hk + hk) with byte strides (T * d * 2, d * 2,
    // G * T * d * 2), whose boxes (64, G, tokens, 1) land as rows t * G + g.
    // If the driver declines these views, the backward recomputes dS instead.
    TmaMap q_kv, do_kv, q_dq, do_dq;
    if (stored) {
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.G, (uint64_t)p.T, (uint64_t)p.B * p.Hk};
        const uint64_t strides[3] = {(uint64_t)p.T * D * 2, (uint64_t)D * 2, (uint64_t)p.G * p.T * D * 2};
        const uint32_t box_kv[4] = {64, (uint32_t)p.G, (uint32_t)(kKvBQ / p.G), 1};
        const uint32_t box_dq[4] = {64, (uint32_t)p.G, (uint32_t)Tq, 1};
        stored = make_tma_4d_bf16(&q_kv, Q, dims, strides, box_kv) == cudaSuccess &&
                 make_tma_4d_bf16(&do_kv, dO, dims, strides, box_kv) == cudaSuccess &&
                 make_tma_4d_bf16(&q_dq, Q, dims, strides, box_dq) == cudaSuccess &&
                 make_tma_4d_bf16(&do_dq, dO, dims, strides, box_dq) == cudaSuccess;
    }
    unsigned char* ds_tiles = stored ? static_cast<unsigned char*>(ws) + bwd_workspace_bytes(p) : nullptr;
    const int n_qt = (p.T + Tq - 1) / Tq;
    const int n_kb = (p.T + kDqBN - 1) / kDqBN;
    // 1. D = rowsum(dO * O)
    const long long nrows = (long long)p.B * p.Hq * p.T;
    constexpr int kRowsPerBlock = 8 * (32 / (D / 8));
    rowdot_kernel<D><<<(unsigned)((nrows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, stream>>>(
        nrows, static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), Dws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    phase_mark(1, stream);

    // 2. dK, dV
    DkdvArgs A;
    A.B = p.B; A.Hq = p.Hq; A.Hk = p.Hk; A.T = p.T; A.G = p.G;
    A.n_kt = (p.T + BN - 1) / BN;
    A.n_qb = (p.T + kKvBQ - 1) / kKvBQ;
    A.scale = p.scale; A.scale_log2 = p.scale_log2;
    A.causal = p.causal;
    A.LSE = LSE; A.Drow = Dws;
    A.dK = static_cast<__nv_bfloat16*>(dK);
    A.dV = static_cast<__nv_bfloat16*>(dV);
    A.status = device_status_word();
    A.band = l2_band(p.B * p.Hk, 2.0 * p.G * p.T * D * 2);   // Q and dO of one group
    A.dS = ds_tiles;
    A.n_qt = n_qt;
    A.n_kb = n_kb;
    A.tq_log2 = stored ? log2_exact(Tq) : 0;
    A.g_log2 = stored ? log2_exact(p.G) : 0;
    A.tb_log2 = stored ? 6 - A.g_log2 : 0;
    A.n_tb = stored ? (p.T + (1 << A.tb_log2) - 1) >> A.tb_log2 : 0;
    if ((e = make_tma_3d_bf16(&A.tk, K, D, p.T, (uint64_t)p.B * p.Hk, BN, 1)) != cudaSuccess) return e;
    if ((e = make_tma_3d_bf16(&A.tv, V, D, p.T, (uint64_t)p.B * p.Hk, BN, 1)) != cudaSuccess) return e;
    if (stored) {
        A.tq = q_kv;
        A.tdo = do_kv;
    } else {
        if ((e = make_tma_3d_bf16(&A.tq, Q, D, p.T, (uint64_t)p.B * p.Hq, kKvBQ, 1)) != cudaSuccess) return e;
        if ((e = make_tma_3d_bf16(&A.tdo, dO, D, p.T, (uint64_t)p.B * p.Hq, kKvBQ, 1)) != cudaSuccess) return e;
    }
    {
        const uint32_t smem = DkdvLayout<D>::kDynSmem;
        const void* fn = stored ? reinterpret_cast<const void*>(dkdv_kernel<D, true>)
                                : reinterpret_cast<const void*>(dkdv_kernel<D, false>);
        if ((e = set_max_dynamic_smem(fn, (int)smem)) != cudaSuccess) return e;
        // One CTA per SM walks a snake of the longest-first key tiles when there
        // are more tiles than SMs and the order is longest-first overall (one
        // band of heads: the snake balances a decreasing order); otherwise one
        // CTA per tile, which the hardware schedules greedily.
        const long long n_items = (long long)p.B * p.Hk * A.n_kt;
        if (n_items > 0x7fffffffLL) return cudaErrorInvalidValue;
        const long long sms = device_sm_count() > 0 ? device_sm_count() : 1;
        A.n_items = static_cast<int>(n_items);
        A.persist = n_items > sms && A.band >= p.B * p.Hk ? 1 : 0;
        const long long grid = A.persist ? sms : n_items;
        if (stored)
            dkdv_kernel<D, true><<<(unsigned)grid, kKvThreads, smem, stream>>>(A);
        else
            dkdv_kernel<D, false><<<(unsigned)grid, kKvThreads, smem, stream>>>(A);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        phase_mark(2, stream);
    }

    // 3. dQ, dKd, dVd
    DqArgs B;
    B.B = p.B; B.Hq = p.Hq; B.Hk = p.Hk; B.T = p.T; B.L = p.L; B.G = p.G;
    B.Tq = BM / p.G;
    B.n_qt = (p.T + B.Tq - 1) / B.Tq;
    const int dep = B.Tq * p.L;
    B.dep_rows = dep >= 64 ? 64 : ((dep + 15) / 16) * 16;
    if (B.dep_rows < 16) B.dep_rows = 16;
    B.scale = p.scale; B.scale_log2 = p.scale_log2;
    B.causal = p.causal; B.win_lo = p.win_lo;
    B.LSE = LSE; B.Drow = Dws;
    B.dQ = static_cast<__nv_bfloat16*>(dQ);
    B.dKd = static_cast<__nv_bfloat16*>(dKd);
    B.dVd = static_cast<__nv_bfloat16*>(dVd);
    B.status = device_status_word();
    B.band = l2_band(p.B * p.Hk, 2.0 * p.T * D * 2);          // K and V of one head
    B.dS = ds_tiles;
    B.n_kb = n_kb;
    B.g_log2 = stored ? log2_exact(p.G) : 0;
    if (stored) {
        B.tq = q_dq;
        B.tdo = do_dq;
    } else {
        if ((e = make_tma_3d_bf16(&B.tq, Q, D, p.T, (uint64_t)p.B * p.Hq, B.Tq, p.G)) != cudaSuccess) return e;
        if ((e = make_tma_3d_bf16(&B.tdo, dO, D, p.T, (uint64_t)p.B * p.Hq, B.Tq, p.G)) != cudaSuccess) return e;
    }
    if ((e = make_tma_3d_bf16(&B.tk, K, D, p.T, (uint64_t)p.B * p.Hk, kDqBN, 1)) != cudaSuccess) return e;
    if ((e = make_tma_3d_bf16(&B.tv, V, D, p.T, (uint64_t)p.B * p.Hk, kDqBN, 1)) != cudaSuccess) return e;
    B.layer = p.depth_layer;
    if (p.L > 0 && p.depth_layer) {
        // layer-major cache [L, B, Hk, T, d] viewed as (d, layer, token, b * Hk + hk)
        if (B.dep_rows % p.L != 0) return cudaErrorInvalidValue;
        const uint64_t nbh = (uint64_t)p.B * p.Hk;
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.L, (uint64_t)p.T, nbh};
        const uint64_t strides[3] = {nbh * p.T * D * 2, (uint64_t)D * 2, (uint64_t)p.T * D * 2};
        const uint32_t box[4] = {64, (uint32_t)p.L, (uint32_t)(B.dep_rows / p.L), 1};
        if ((e = make_tma_4d_bf16(&B.tkd, Kd, dims, strides, box)) != cudaSuccess) return e;
        if ((e = make_tma_4d_bf16(&B.tvd, Vd, dims, strides, box)) != cudaSuccess) return e;
    } else if (p.L > 0) {
        const uint64_t rows = (uint64_t)p.T * p.L;
        if ((e = make_tma_3d_bf16(&B.tkd, Kd, D, rows, (uint64_t)p.B * p.Hk, B.dep_rows, 1)) != cudaSuccess) return e;
        if ((e = make_tma_3d_bf16(&B.tvd, Vd, D, rows, (uint64_t)p.B * p.Hk, B.dep_rows, 1)) != cudaSuccess) return e;
    } else {
        B.tkd = B.tk;
        B.tvd = B.tv;
    }
    {
        const uint32_t smem = DqLayout<D>::kDynSmem;
        const long long grid = (long long)p.B * p.Hk * B.n_qt;
        bool launched = false;
        if constexpr (D == 128) {
            if (stored) {
                if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(dq_kernel<D, true>), (int)smem)) !=
                    cudaSuccess)
                    return e;
                if ((e = launch_dependent(dq_kernel<D, true>, (unsigned)grid, kThreads, smem, stream, B)) !=
                    cudaSuccess)
                    return e;
                launched = true;
            }
        }
        if (!launched) {
            if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(dq_kernel<D, false>), (int)smem)) !=
                cudaSuccess)
                return e;
            if ((e = launch_dependent(dq_kernel<D, false>, (unsigned)grid, kThreads, smem, stream, B)) !=
                cudaSuccess)
                return e;
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        phase_mark(3, stream);
    }
    return cudaSuccess;
}

}  // namespace


size_t bwd_ds_bytes(const Problem& p) {
    if (p.elem_bytes != 2 || p.d != 128 || !(p.G == 1 || p.G == 2 || p.G == 4 || p.G == 8)) return 0;
    const double Tq = BM / p.G;
    const double tiles = double(p.B) * p.Hk * std::ceil(p.T / Tq) * std::ceil(p.T / double(kDqBN));
    const double bytes = tiles * kDsTileBytes;
    return bytes <= kMaxStoredDsBytes ? static_cast<size_t>(bytes) : 0;
}

cudaError_t launch_bwd_sm100(const Problem& p, const void* Q, const void* K, const void* V,
                             const void* Kd, const void* Vd, const void* O, const float* LSE,
                             const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                             void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (p.d == 128)
        return launch_d<128>(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, ws, ws_bytes, stream);
    if (p.d == 64)
        return launch_d<64>(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, ws, ws_bytes, stream);
    return cudaErrorInvalidValue;
}

}  // namespace moda
