// moda_fwd_sm100.cu -- fused MoDA forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Operator: paper summary of arXiv 2603.15619, "Mixture-of-Depths Attention
// (MoDA): The Unified Operator" -- one softmax over the causal sequence keys
// (j <= t) and the token's own L depth rows, scaled by 1/sqrt(d); the online
// form is "Fused online-softmax (Algorithm 1)" (running max / sum / output in
// base 2, sequence blocks then depth blocks, o / acc at the end).  Two options
// change only the visible sets: non-causal (every row sees keys 0..T-1; the
// README's "TODO" non-causal kernel) and a depth window (the last S of the L
// depth rows; bounded depth slots, summary "6. Limitations and Trade-offs").
//
// Work unit: one query tile of 128 rows = the G heads of one KV head times
// Tq = 128/G consecutive tokens (row r -> head g = r / Tq, token t0 + r % Tq).
// This is the pages' group-aware idea in B200 form: every K/V tile and every
// depth tile is loaded once into shared memory and used by all G heads of the
// group, and the depth rows of the tile's Tq tokens are one contiguous range
// [t0*L, (t0+Tq)*L) of the token-major depth tensor.
//
// CTA roles (384 threads):
//   warp 0      TMA producer of Q (once) and of the K (or K_depth) tiles;
//   warp 10     TMA producer of the V (or V_depth) tiles.  K and V have rings
//               of their own: a K stage frees as soon as S_i = Q K_i^T is
//               done, a V stage only when O += P_i V_i is, so the next K
//               tiles stream in while PV still holds older V tiles.
//   warp 11     score-MMA issuer: S_i = Q K_i^T into one of three TMEM S
//               buffers, up to three blocks ahead of the PV products, so
//               score tiles are ready before the softmax needs them and the
//               tensor pipe's issue-to-completion latency (hundreds of
//               cycles) is off the softmax's critical path.
//   warp 1      TMEM allocator and PV-MMA issuer: O += P_i V_i with P read
//               from TMEM.  The two issuers sit on different sub-partitions.
//   warps 2..9  softmax, two warps per TMEM lane quarter (16 rows each) and
//               two threads per tile row: with the 16x32bx2 TMEM shapes,
//               thread t < 16 holds columns [0, 64) of its row and thread
//               t + 16 columns [64, 128), so the row max and sum take one
//               shuffle.  Per block: tcgen05.ld of S, masks, running max,
//               exp2, row sum, P (bf16) written back over S with tcgen05.st;
//               O in TMEM is rescaled only when the running max grew by more
//               than 2^8 (exact: the final o / acc cancels it).  Two warps
//               per SM sub-partition keep its MUFU (exp2) unit fed.
// TMEM columns: S0 [0,128), S1 [128,256), S2 [256,384), O [384, 384+d).
// Softmax: row max as four partial maxima of three-input max; exp2 on the
// MUFU unit (moving a share of the exponentials to a polynomial on the FMA
// pipe measured slower: the softmax warps are issue-bound, not MUFU-bound).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "moda_internal.h"
#include "moda_ptx.cuh"

namespace moda {
namespace {

using namespace ptx;

constexpr int BM = 128;          // query rows per tile
constexpr int BN = 128;          // sequence keys per block
constexpr int kKStages = 3;      // K ring: a stage frees when S_i is done
constexpr int kVStages = 3;      // V ring: a stage frees when PV_i is done
constexpr int kSoftmaxWarps = 8;             // warps 2..9
constexpr int kVWarp = 2 + kSoftmaxWarps;    // V producer
constexpr int kSWarp = kVWarp + 1;           // score-MMA issuer (sub-partition 3)
constexpr int kThreads = 32 * (kSWarp + 1);
constexpr float kLazyLimit = 1024.0f;     // largest half-row sum of p kept without a rescale
constexpr uint32_t kSlabBytes = 128 * 128;   // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 512;
constexpr int kSBufs = 3;            // S / P buffers in TMEM
constexpr uint32_t kColO = 384;      // O accumulator after the three S buffers

struct FwdArgs {
    TmaMap tq, tk, tv, tkd, tvd;
    __nv_bfloat16* O;
    float* LSE;
    unsigned int* status;
    int B, Hq, Hk, T, L, G, Tq, n_qt, dep_rows;
    int causal;       // 0: every row sees keys 0..T-1
    int win_lo;       // first visible depth row of a token
    int n_tiles;      // B * Hk * n_qt query tiles, longest first within a band of heads
    int band;         // (b, KV head) pairs per band (banded_item)
    int tok_major;    // query tile rows token-major (r = t * G + g), else head-major (r = g * Tq + t)
    int layer;        // depth tiles from the layer-major cache (4-D view, dep_rows / L whole tokens)
    float scale_log2;
};

// Query tile `idx`: heads in bands (banded_item), and within a band the last
// query tiles (the longest) of every (b, hk) first.  Blocks are n_seq key
// blocks, then the depth blocks.
struct FwdTile {
    int b, hk, bh, t0, t_end, n_seq, nb;
};
__device__ __forceinline__ FwdTile fwd_tile(const FwdArgs& a, int idx) {
    FwdTile t;
    int outer;
    banded_item(idx, a.n_qt, a.B * a.Hk, a.band, &outer, &t.bh);
    const int qt = a.n_qt - 1 - outer;
    t.b = t.bh / a.Hk;
    t.hk = t.bh - t.b * a.Hk;
    t.t0 = qt * a.Tq;
    t.t_end = min(t.t0 + a.Tq, a.T);                   // one past the last real token
    t.n_seq = ((a.causal ? t.t_end : a.T) - 1) / BN + 1;
    const int n_dep = a.L > 0 ? ((t.t_end - t.t0) * a.L + a.dep_rows - 1) / a.dep_rows : 0;
    t.nb = t.n_seq + n_dep;
    return t;
}

template <int D>
struct Layout {
    static constexpr int kSlabs = D / 64;
    static constexpr uint32_t kTile = kSlabs * kSlabBytes;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kTile;
    static constexpr uint32_t kV = kK + kKStages * kTile;
    static constexpr uint32_t kBar = kV + kVStages * kTile;
    static constexpr uint32_t kBytes = kBar + 256;
    // + alignment slack; never below 120 KB so that one CTA (and one 512-column
    // TMEM allocation) is resident per SM.
    static constexpr uint32_t kDynSmem = kBytes + 1024 > 120u * 1024 ? kBytes + 1024 : 120u * 1024;
};

// Barrier slots.
enum { kQFull = 0, kKFull = 1, kVFull = kKFull + kKStages, kVEmpty = kVFull + kVStages,
       kSFull = kVEmpty + kVStages, kPReady = kSFull + kSBufs, kOFinal = kPReady + kSBufs,
       kOFree = kOFinal + 1, kNumBars = kOFree + 1 };
static_assert(kKStages == kSBufs, "a K stage is released by the score barrier of its S buffer");
static_assert(kVStages == kSBufs, "an S buffer is free again at the V-stage release of its PV");

// kPersist: CTAs walk several tiles (grid = SM count); otherwise each CTA
// takes exactly tile blockIdx.x and the tile loops compile away.
template <int D, bool kPersist>
__global__ void __launch_bounds__(kThreads, 1) moda_fwd_sm100_kernel(const __grid_constant__ FwdArgs a) {
    using Lay = Layout<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    unsigned char* sQ = smem + Lay::kQ;
    unsigned char* sK = smem + Lay::kK;
    unsigned char* sV = smem + Lay::kV;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Persistent: CTA c takes tile snake_tile(r, c, gridDim.x) of every round
    // r.  Ring stages and barrier phases follow a per-CTA running block count j
    // over all of its tiles, which every role computes alike.
    const int R = a.G * a.Tq;
    const int cta = static_cast<int>(blockIdx.x);
    const int tstep = static_cast<int>(gridDim.x);
    const int n_rounds = kPersist ? (a.n_tiles + tstep - 1) / tstep : 1;
    auto tile_of = [&](int rnd) { return kPersist ? snake_tile(rnd, cta, tstep) : cta; };

    if (threadIdx.x == 0) {
        mbar_init(&bars[kQFull], 1);
        for (int s = 0; s < kKStages; ++s) mbar_init(&bars[kKFull + s], 1);
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&bars[kVFull + s], 1);
            mbar_init(&bars[kVEmpty + s], 1);
        }
        for (int s = 0; s < kSBufs; ++s) {
            mbar_init(&bars[kSFull + s], 1);
            mbar_init(&bars[kPReady + s], kSoftmaxWarps);   // one arrive per softmax warp
        }
        mbar_init(&bars[kOFinal], 1);
        mbar_init(&bars[kOFree], kSoftmaxWarps);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (R < BM) {  // rows the Q box does not cover: make them finite (zeros)
        for (int i = threadIdx.x; i < Lay::kSlabs * (BM - R) * 8; i += kThreads) {
            const int slab = i / ((BM - R) * 8);
            const int rem = i - slab * (BM - R) * 8;
            const int row = R + rem / 8;
            reinterpret_cast<uint4*>(sQ + slab * kSlabBytes + row * 128)[rem % 8] =
                make_uint4(0, 0, 0, 0);
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

    if (warp == 0 || warp == kVWarp) {
        // ------------------------------------------------------ producers ---
        // warp 0: Q, then K_i (sequence) / K_depth tiles; warp kVWarp: V tiles.
        if (lane == 0) {
            const bool is_k = warp == 0;
            const int nst = is_k ? kKStages : kVStages;
            uint64_t* full = &bars[is_k ? kKFull : kVFull];
            uint64_t* empty = &bars[is_k ? kSFull : kVEmpty];
            unsigned char* ring = is_k ? sK : sV;
            const void* m_seq = is_k ? static_cast<const void*>(&a.tk) : static_cast<const void*>(&a.tv);
            const void* m_dep = is_k ? static_cast<const void*>(&a.tkd) : static_cast<const void*>(&a.tvd);
            const uint64_t once = policy_evict_first();   // depth tiles are read exactly once
            prefetch_tmap(m_seq);
            if (a.L > 0) prefetch_tmap(m_dep);
            if (is_k) prefetch_tmap(&a.tq);
            const uint32_t q_bytes = Lay::kSlabs * 128u * a.Tq * a.G;
            int j = 0, kt = 0, issued = 0, nq = 0;
            bool ok = true;
            for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
                const int tile = tile_of(rnd);
                if (tile >= a.n_tiles) continue;
                const FwdTile T = fwd_tile(a, tile);
                if (is_k) {
                    // Q has one buffer: the previous tile's last score MMA must
                    // be done before it is overwritten (the next phase of that
                    // S buffer needs this Q, so the parity is exact)
                    if (kt > 0 && !mbar_wait(&bars[kSFull + (j - 1) % kSBufs], ((j - 1) / kSBufs) & 1,
                                             a.status, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bars[kQFull], q_bytes);
                    for (int s = 0; s < Lay::kSlabs; ++s) {
                        if (a.tok_major)
                            tma_load_4d(sQ + s * kSlabBytes, &a.tq, &bars[kQFull], s * 64, 0, T.t0, T.bh);
                        else
                            tma_load_3d(sQ + s * kSlabBytes, &a.tq, &bars[kQFull], s * 64, T.t0,
                                        T.b * a.Hq + T.hk * a.G);
                    }
                    ++nq;
                }
                for (int i = 0; i < T.nb; ++i, ++j) {
                    const int st = j % nst;
                    // K stage of block j-nst is free once S(j-nst) is done: that
                    // is the score barrier of its buffer (three K stages, three S
                    // buffers), so no separate commit is needed for K.
                    if (j >= nst && !mbar_wait(&empty[st], ((j / nst) - 1) & 1, a.status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    unsigned char* dst = ring + st * Lay::kTile;
                    const bool seq = i < T.n_seq;
                    const int row0 = seq ? i * BN : T.t0 * a.L + (i - T.n_seq) * a.dep_rows;
                    const uint32_t bytes = Lay::kSlabs * 128u * (seq ? BN : a.dep_rows);
                    mbar_arrive_expect_tx(&full[st], bytes);
                    for (int s = 0; s < Lay::kSlabs; ++s) {
                        if (seq)
                            tma_load_3d(dst + s * kSlabBytes, m_seq, &full[st], s * 64, row0, T.bh);
                        else if (a.layer)   // box (64, L, dep_rows / L, 1) from token row0 / L
                            tma_load_4d_hint(dst + s * kSlabBytes, m_dep, &full[st], s * 64, 0, row0 / a.L, T.bh,
                                             once);
                        else
                            tma_load_3d_hint(dst + s * kSlabBytes, m_dep, &full[st], s * 64, row0, T.bh, once);
                    }
                    issued = j + 1;
                }
                ++kt;
            }
            // Let every load this thread started land before the CTA retires.
            if (nq > 0) mbar_wait(&bars[kQFull], (nq - 1) & 1, a.status, abort_flag);
            for (int i = max(0, issued - nst); i < issued; ++i)
                mbar_wait(&full[i % nst], (i / nst) & 1, a.status, abort_flag);
        }
    } else if (warp == 1 || warp == kSWarp) {
        // ------------------------------------------------------ MMA issuers -
        // Two warps issue: warp kSWarp the score products S(j), warp 1 the
        // PV(j) products, on two sub-partitions.  One elected thread of each
        // runs the whole loop (waits, MMAs, commits): an MMA issue blocks until
        // the tensor pipe takes it, so the issue path's own cost is pipe idle
        // time, and single-thread waits and issues cost about half of the
        // warp-collective forms.  A commit tracks only its own thread's MMAs.
        if (elect_one()) {
            const uint32_t id_seq = idesc_bf16(128, BN, false, false);
            const uint32_t id_dep = idesc_bf16(128, a.dep_rows, false, false);
            const uint32_t id_pv = idesc_bf16(128, D, false, true);
            // Descriptors are built once; a K step adds its byte offset / 16 to
            // the 14-bit address field (shared addresses stay < 256 KB).
            const uint64_t qd0 = desc_kmajor_sw128(smem_u32(sQ));
            // S(j) = Q K_j^T into buffer j % 3 (i: the block's index in its tile).
            // The buffer last held P(j-3), read by PV(j-3): the caller waits for
            // that product's completion (its V-stage release) first.
            auto issue_s = [&](int j, int i, const FwdTile& T) -> bool {
                const int st = j % kKStages;
                const int sb = j % kSBufs;
                if (!mbar_wait(&bars[kKFull + st], (j / kKStages) & 1, a.status, abort_flag)) return false;
                tc_fence_after();
                const uint64_t kd0 = desc_kmajor_sw128(smem_u32(sK + st * Lay::kTile));
                const uint32_t id = i < T.n_seq ? id_seq : id_dep;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4;
                    umma_ss(tmem + sb * 128, qd0 + off, kd0 + off, id, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[kSFull + sb]);
                return true;
            };
            // O += P(j) V_j with P read from TMEM buffer j % 3; the tile's first
            // block overwrites O.
            auto issue_pv = [&](int j, int i, const FwdTile& T) -> bool {
                const int st = j % kVStages;
                const int sb = j % kSBufs;
                if (!mbar_wait(&bars[kPReady + sb], (j / kSBufs) & 1, a.status, abort_flag)) return false;
                if (!mbar_wait(&bars[kVFull + st], (j / kVStages) & 1, a.status, abort_flag)) return false;
                tc_fence_after();
                const int krows = i < T.n_seq ? BN : a.dep_rows;
                const uint64_t vd0 = desc_mnmajor_sw128(smem_u32(sV + st * Lay::kTile), kSlabBytes);
                if (krows == BN) {
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        umma_ts(tmem + kColO, tmem + sb * 128 + kk * 8, vd0 + kk * (2048 >> 4), id_pv,
                                (i > 0 || kk > 0) ? 1u : 0u);
                } else {
                    for (int kk = 0; kk < krows / 16; ++kk)
                        umma_ts(tmem + kColO, tmem + sb * 128 + kk * 8, vd0 + kk * (2048 >> 4), id_pv,
                                (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[kVEmpty + st]);
                return true;
            };
            // The score issuer runs up to three blocks ahead of the PV issuer
            // (three S buffers), so two score tiles are ready before the softmax
            // needs them.
            bool ok = true;
            int j0 = 0, kt = 0;
            const bool s_role = warp == kSWarp;
            for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
                const int tile = tile_of(rnd);
                if (tile >= a.n_tiles) continue;
                const FwdTile T = fwd_tile(a, tile);
                if (s_role) {
                    ok = mbar_wait(&bars[kQFull], kt & 1, a.status, abort_flag);
                    for (int i = 0; ok && i < T.nb; ++i) {
                        const int j = j0 + i;
                        // buffer j % 3 held P(j-3): PV(j-3) must have completed
                        if (j >= kSBufs && !mbar_wait(&bars[kVEmpty + (j - kSBufs) % kVStages],
                                                      ((j - kSBufs) / kVStages) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (!issue_s(j, i, T)) { ok = false; break; }
                    }
                } else {
                    for (int i = 0; ok && i < T.nb; ++i) {
                        // the tile's first PV overwrites O: the softmax warps must
                        // have read the previous tile's O out
                        if (i == 0 && kt > 0 &&
                            !mbar_wait(&bars[kOFree], (kt - 1) & 1, a.status, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (i == 0) tc_fence_after();
                        if (!issue_pv(j0 + i, i, T)) { ok = false; break; }
                    }
                    umma_commit(&bars[kOFinal]);
                }
                j0 += T.nb;
                ++kt;
            }
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 2 + kSoftmaxWarps) {
        // ------------------------------------------------------ softmax -----
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ..
        const int sub = (warp - 2) >> 2;              // rows 16*sub .. of the quarter
        const int half = lane >> 4;                   // column half of the row
        const int r = quarter * 32 + sub * 16 + (lane & 15);   // tile row
        const bool row_real = r < R;
        // the row's head and token offset within the tile
        const int g = row_real ? (a.tok_major ? r % a.G : r / a.Tq) : 0;
        const int t_off = row_real ? (a.tok_major ? r / a.G : r - g * a.Tq) : 0;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32 + sub * 16) << 16);
        const int c0 = half * 64;                     // first S column this thread holds
        const float sl2 = a.scale_log2;
        bool ok = true;
        int j0 = 0, kt = 0;
        for (int rnd = 0; ok && rnd < n_rounds; ++rnd) {
            const int tile = tile_of(rnd);
            if (tile >= a.n_tiles) continue;
            const FwdTile T = fwd_tile(a, tile);
            const int t0 = T.t0, n_seq = T.n_seq, nb = T.nb;
            const int t_row = t0 + t_off;
            float m = -INFINITY, l = 0.0f;                // l: this half's share of the row sum
            for (int i = 0; i < nb; ++i) {
                const int j = j0 + i;                     // running block count: ring phases
                const int sb = j % kSBufs;
                // every wait result is made warp-uniform: the shuffles and the
                // .sync.aligned TMEM accesses below need the whole warp
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[kSFull + sb], (j / kSBufs) & 1, a.status,
                                                       abort_flag))) { ok = false; break; }
                tc_fence_after();
                const uint32_t s_addr = lane_base + sb * 128;
                if (i >= n_seq) {
                    // A depth block none of the warp's 16 rows can see (each
                    // row sees only its own token's rows): every score would be
                    // masked to -inf, so P is exactly 0 and the row sums do not
                    // change.  Write the zeros without loading or exponentiating.
                    const int base = t_row * a.L - (t0 * a.L + (i - n_seq) * a.dep_rows) - c0;
                    const int vis_lo = max(base + a.win_lo, 0);
                    const int vis_hi = min(min(base + a.L, a.dep_rows - c0), 64);
                    if (__all_sync(0xffffffffu, vis_lo >= vis_hi)) {
                        uint32_t zero[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) zero[c] = 0u;
                        __syncwarp();
                        tmem_st16x2_32<32>(s_addr, zero);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars[kPReady + sb]);
                        continue;
                    }
                }
                uint32_t sr[64];
                tmem_ld16x2_32<64>(s_addr, sr);            // columns c0 .. c0+31
                tmem_ld16x2_32<64>(s_addr + 32, sr + 32);  // columns c0+32 .. c0+63
                tmem_wait_ld();
                reg_fence<64>(sr);
                // masks: invisible scores become -inf (p = 0)
                if (i < n_seq) {
                    const int kb = i * BN + c0;
                    const int lim = a.causal ? t_row : a.T - 1;   // last visible key
                    if (kb + 63 > lim) {
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (kb + c > lim) sr[c] = __float_as_uint(-INFINITY);
                    }
                } else {
                    const int base = t_row * a.L - (t0 * a.L + (i - n_seq) * a.dep_rows) - c0;
                    const int lo = base + a.win_lo;
                    const int hi = min(base + a.L, a.dep_rows - c0);
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < lo || c >= hi) sr[c] = __float_as_uint(-INFINITY);
                }
                // Row max of this block (both halves of the row), base 2.
                auto block_max = [&]() -> float {
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 64; c += 8) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            mx4[u] = fmax3(mx4[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
                    }
                    float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    return mx * sl2;
                };
                // p = 2^(s*sl2 - m) for this thread's 64 columns, packed to bf16;
                // returns this half-row's sum.
                uint32_t pk[32];
                auto exp_block = [&]() -> float {
                    float rs4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float x0 = fmaf(__uint_as_float(sr[2 * c]), sl2, -m);
                        const float x1 = fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -m);
                        const float p0 = ex2(x0);
                        const float p1 = ex2(x1);
                        rs4[c & 3] += p0 + p1;
                        pk[c] = pack_bf16(p0, p1);
                    }
                    return (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
                };
                // The online softmax is exact for any reference point m, so a
                // block is first exponentiated against the running m without
                // computing its max.  Only when some p could exceed 2^10 (a
                // half-row sum above 2^10 is necessary for that, and catches
                // overflow too) does the warp take the block max, rescale O and
                // l to the new reference and recompute P.  The first block sets m.
                if (i == 0) m = block_max();
                float rs = exp_block();
                if (i > 0 && __any_sync(0xffffffffu, !(rs <= kLazyLimit))) {
                    const float m_new = fmaxf(m, block_max());
                    // O must hold P_{i-1} V_{i-1} before it is rescaled: wait for
                    // the V-stage release PV_{i-1} commits.  S_i was issued after
                    // PV_{i-2}, so at most PV_{i-1} is in flight, and PV_{i+2}
                    // (the stage's next use) needs P_{i+2}: the parity is exact.
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars[kVEmpty + (j - 1) % kVStages],
                                                           ((j - 1) / kVStages) & 1, a.status, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float alpha = ex2(m - m_new);
                    l *= alpha;
                    m = m_new;
#pragma unroll
                    for (int c = 0; c < D / 2; c += 32) {   // this thread's half of the O row
                        uint32_t o[32];
                        tmem_ld16x2_32<D / 2>(lane_base + kColO + c, o);
                        tmem_wait_ld();
                        reg_fence<32>(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st16x2_32<D / 2>(lane_base + kColO + c, o);
                    }
                    tmem_wait_st();
                    rs = exp_block();
                }
                l += rs;
                // P columns c0/2 .. c0/2+31 (bf16 pairs) over the S columns this
                // warp has already read (its own loads completed above)
                __syncwarp();
                tmem_st16x2_32<32>(s_addr, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kPReady + sb]);
            }
            // ---------------------------------------------------- epilogue ------
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kOFinal], kt & 1, a.status, abort_flag));
            const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
            if (ok) {
                tc_fence_after();
                uint32_t o[D / 2];
#pragma unroll
                for (int c = 0; c < D / 2; c += 32) tmem_ld16x2_32<D / 2>(lane_base + kColO + c, o + c);
                tmem_wait_ld();
                reg_fence<D / 2>(o);
                // O is in registers: the next tile's first PV may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kOFree]);
                if (row_real && t_row < a.T) {
                    const float inv = 1.0f / l_row;
                    const size_t qrow = (static_cast<size_t>(T.b) * a.Hq + T.hk * a.G + g) * a.T + t_row;
                    uint4* dst = reinterpret_cast<uint4*>(a.O + qrow * D + half * (D / 2));
#pragma unroll
                    for (int c = 0; c < D / 2; c += 8) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(o[c + 0]) * inv, __uint_as_float(o[c + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(o[c + 4]) * inv, __uint_as_float(o[c + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(o[c + 6]) * inv, __uint_as_float(o[c + 7]) * inv);
                        dst[c / 8] = v;
                    }
                    if (half == 0) a.LSE[qrow] = (m + log2f(l_row)) * 0.6931471805599453f;
                }
            }
            j0 += nb;
            ++kt;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t launch_d(const Problem& p, const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd, void* O, float* LSE, cudaStream_t stream) {
    FwdArgs a;
    a.B = p.B; a.Hq = p.Hq; a.Hk = p.Hk; a.T = p.T; a.L = p.L; a.G = p.G;
    a.Tq = BM / p.G;
    a.n_qt = (p.T + a.Tq - 1) / a.Tq;
    const int dep = a.Tq * p.L;
    a.dep_rows = dep >= 128 ? 128 : ((dep + 15) / 16) * 16;
    if (a.dep_rows < 16) a.dep_rows = 16;
    a.scale_log2 = p.scale_log2;
    a.causal = p.causal;
    a.win_lo = p.win_lo;
    a.O = static_cast<__nv_bfloat16*>(O);
    a.LSE = LSE;
    a.status = device_status_word();
    cudaError_t e;
    // Query tile token-major: a 4-D view of Q as (d, head g, token, b * Hk + hk)
    // with byte strides (T * d * 2, d * 2, G * T * d * 2): the box (64, G, Tq, 1)
    // lands as rows t * G + g.  Each warp's rows then cover few tokens, so
    // most depth blocks hold none of a warp's visible depth rows and the
    // warp skips them.  Head-major (a 3-D box) if the driver declines the view.
    {
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.G, (uint64_t)p.T, (uint64_t)p.B * p.Hk};
        const uint64_t strides[3] = {(uint64_t)p.T * D * 2, (uint64_t)D * 2, (uint64_t)p.G * p.T * D * 2};
        const uint32_t box[4] = {64, (uint32_t)p.G, (uint32_t)a.Tq, 1};
        a.tok_major = make_tma_4d_bf16(&a.tq, Q, dims, strides, box) == cudaSuccess ? 1 : 0;
    }
    if (!a.tok_major &&
        (e = make_tma_3d_bf16(&a.tq, Q, D, p.T, (uint64_t)p.B * p.Hq, a.Tq, p.G)) != cudaSuccess)
        return e;
    if ((e = make_tma_3d_bf16(&a.tk, K, D, p.T, (uint64_t)p.B * p.Hk, BN, 1)) != cudaSuccess) return e;
    if ((e = make_tma_3d_bf16(&a.tv, V, D, p.T, (uint64_t)p.B * p.Hk, BN, 1)) != cudaSuccess) return e;
    a.layer = p.depth_layer;
    if (p.L > 0 && p.depth_layer) {
        // layer-major cache [L, B, Hk, T, d] viewed as (d, layer, token, b * Hk + hk):
        // a box of dep_rows / L whole tokens lands as rows t * L + l, the same
        // shared-memory tile as the token-major layout's dep_rows rows
        if (a.dep_rows % p.L != 0) return cudaErrorInvalidValue;
        const uint64_t nbh = (uint64_t)p.B * p.Hk;
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.L, (uint64_t)p.T, nbh};
        const uint64_t strides[3] = {nbh * p.T * D * 2, (uint64_t)D * 2, (uint64_t)p.T * D * 2};
        const uint32_t box[4] = {64, (uint32_t)p.L, (uint32_t)(a.dep_rows / p.L), 1};
        if ((e = make_tma_4d_bf16(&a.tkd, Kd, dims, strides, box)) != cudaSuccess) return e;
        if ((e = make_tma_4d_bf16(&a.tvd, Vd, dims, strides, box)) != cudaSuccess) return e;
    } else if (p.L > 0) {
        const uint64_t rows = (uint64_t)p.T * p.L;
        if ((e = make_tma_3d_bf16(&a.tkd, Kd, D, rows, (uint64_t)p.B * p.Hk, a.dep_rows, 1)) != cudaSuccess) return e;
        if ((e = make_tma_3d_bf16(&a.tvd, Vd, D, rows, (uint64_t)p.B * p.Hk, a.dep_rows, 1)) != cudaSuccess) return e;
    } else {
        a.tkd = a.tk;
        a.tvd = a.tv;
    }
    const uint32_t smem = Layout<D>::kDynSmem;
    e = set_max_dynamic_smem(reinterpret_cast<const void*>(moda_fwd_sm100_kernel<D, true>), (int)smem);
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem(reinterpret_cast<const void*>(moda_fwd_sm100_kernel<D, false>), (int)smem);
    if (e != cudaSuccess) return e;
    // Short tiles (on average fewer than 64 key blocks): one persistent CTA per
    // SM walks its share, so tile start-up and epilogue overlap the previous
    // tile.  Long tiles: one CTA per tile (each takes exactly its own tile),
    // which measured faster there.
    const long long n_tiles = (long long)p.B * p.Hk * a.n_qt;
    if (n_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    a.n_tiles = static_cast<int>(n_tiles);
    a.band = l2_band(p.B * p.Hk, 2.0 * p.T * D * 2);   // K and V of one head
    const long long seq_blocks = p.causal ? ((long long)p.T + BN - 1) / BN / 2 + 1 : ((long long)p.T + BN - 1) / BN;
    const long long avg_blocks = seq_blocks + ((long long)a.Tq * p.L + a.dep_rows - 1) / a.dep_rows;
    const long long sms = device_sm_count() > 0 ? device_sm_count() : 1;
    if (avg_blocks < 64 && n_tiles > sms)
        moda_fwd_sm100_kernel<D, true><<<(unsigned)sms, kThreads, smem, stream>>>(a);
    else
        moda_fwd_sm100_kernel<D, false><<<(unsigned)n_tiles, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace


cudaError_t launch_fwd_sm100(const Problem& p, const void* Q, const void* K, const void* V,
                             const void* Kd, const void* Vd, void* O, float* LSE,
                             cudaStream_t stream) {
    if (p.d == 128) return launch_d<128>(p, Q, K, V, Kd, Vd, O, LSE, stream);
    if (p.d == 64) return launch_d<64>(p, Q, K, V, Kd, Vd, O, LSE, stream);
    return cudaErrorInvalidValue;
}

}  // namespace moda
