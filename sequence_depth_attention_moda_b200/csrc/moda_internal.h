// moda_internal.h -- interface between the C-ABI host layer (moda_api.cu) and
// the kernel launchers.  Not installed; not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moda.h"

namespace moda {

// A validated problem.  Index conventions follow the C ABI (include/moda.h).
struct Problem {
    int B, Hq, Hk, T, d, L, G;
    float scale;        // softmax scale on the natural-log scale
    float scale_log2;   // scale * log2(e): scores go straight into exp2
    int elem_bytes;     // 2 (bf16) or 4 (fp32)
    int causal;         // 1: key j visible to row t iff j <= t; 0: all keys
    int win_lo;         // first visible depth row of a token (L - window, or 0)
    int depth_layer;    // 1: Kd, Vd (and dKd, dVd) layer-major [L, B, Hk, T, d]
};

// Kernel-side status bits written into the per-device status word.
enum : unsigned int {
    kStatusTimeout = 1u,   // a bounded mbarrier / flag wait ran out
};

// Address of the calling device's status word (device memory), or nullptr.
unsigned int* device_status_word();
// Shape validation and error recording of the API layer, for entry points
// defined outside moda_api.cu.
moda_status api_validate(const moda_shape* shape, Problem* p);
moda_status api_fail(moda_status s, const char* msg);

// SM count of the current device (cached).
int device_sm_count();

// Tile of CTA c in round r of a persistent launch with G CTAs: rounds of G
// tiles of a longest-first order, dealt alternately forwards and backwards
// (a snake), so every CTA's total stays close to the mean.  Only the last
// round can run past the tile count; callers skip such slots.
__host__ __device__ inline int snake_tile(int r, int c, int G) {
    return r * G + ((r & 1) ? G - 1 - c : c);
}

// Work item `idx` of a list of n_outer x nbh items, in bands of `band`
// (b, KV head) pairs: every item of the first band's heads (outer index 0,
// 1, ... for each head in turn), then the next band.  Items that run at the
// same time then share the K/V (or Q/dO) of only a few heads, which stay in
// L2 while the band lasts instead of being re-read from HBM for every outer
// index.  With band >= nbh this is the plain outer-major order.
__host__ __device__ inline void banded_item(int idx, int n_outer, int nbh, int band, int* outer,
                                            int* bh) {
    const int per_band = band * n_outer;
    const int bi = idx / per_band;
    const int local = idx - bi * per_band;
    const int h0 = bi * band;
    const int hb = nbh - h0 < band ? nbh - h0 : band;
    *outer = local / hb;
    *bh = h0 + (local - *outer * hb);
}

// Heads per band.  When every head's re-read operands (`bytes_per_head`
// each) fit in half of the 126 MB L2 together, no banding (nbh: the plain
// longest-first order over all heads keeps the best load balance); else as
// many heads as fit in a 32 MB share, at least one.
inline int l2_band(int nbh, double bytes_per_head) {
    const double mib = 1024.0 * 1024.0;
    if (bytes_per_head <= 0 || nbh * bytes_per_head <= 64.0 * mib) return nbh;
    const int b = static_cast<int>(32.0 * mib / bytes_per_head);
    return b < 1 ? 1 : (b > nbh ? nbh : b);
}

// Records the calling thread's k-th phase marker on `stream`, if one is set
// (see moda_set_phase_events); a no-op otherwise.
void phase_mark(int k, cudaStream_t stream);

// ---- decoding (moda_decode.cu) ----------------------------------------------
// One query token per (b, Hq head) against T cached keys and L depth rows;
// ws holds decode_workspace_bytes(p) bytes of partials.
size_t decode_workspace_bytes(const Problem& p);
cudaError_t launch_decode(const Problem& p, const void* q, const void* K, const void* V,
                          const void* Kd, const void* Vd, void* out, float* lse, void* ws,
                          cudaStream_t stream);

// ---- depth repack (moda_repack.cu) -----------------------------------------
cudaError_t launch_repack(int B, int Hk, int T, int d, int L, int elem_bytes,
                          const void* src, void* dst, cudaStream_t stream);

// ---- CUDA-core path (moda_simt.cu): fp32 dtype; bf16 inputs for debugging --
cudaError_t launch_fwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const void* Kd, const void* Vd, void* O, float* LSE,
                            cudaStream_t stream);
cudaError_t launch_bwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const void* Kd, const void* Vd, const void* O, const float* LSE,
                            const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                            float* Dws, cudaStream_t stream);

// ---- tensor-core path, sm_100a (moda_fwd_sm100.cu, moda_bwd_sm100.cu) -------
// Each returns cudaSuccess, or an error; on error nothing was launched.
cudaError_t launch_fwd_sm100(const Problem& p, const void* Q, const void* K, const void* V,
                             const void* Kd, const void* Vd, void* O, float* LSE,
                             cudaStream_t stream);
// ws holds D = rowsum(dO * O) (bwd_workspace_bytes) and, when ws_bytes also
// covers bwd_ds_bytes after it, the stored dS tiles; otherwise the dQ kernel
// recomputes S and dP.
cudaError_t launch_bwd_sm100(const Problem& p, const void* Q, const void* K, const void* V,
                             const void* Kd, const void* Vd, const void* O, const float* LSE,
                             const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                             void* ws, size_t ws_bytes, cudaStream_t stream);

// Workspace bytes the backward needs at least: D = rowsum(dO * O), fp32
// [B, Hq, T], rounded up to 256 bytes.
size_t bwd_workspace_bytes(const Problem& p);
// Bytes of stored dS tiles the faster backward uses on top of that (0 when it
// does not apply to this shape).
size_t bwd_ds_bytes(const Problem& p);

// ---- TMA descriptors (moda_tma.cu) -------------------------------------------
// A 3-D bf16 tensor map over a row-major [outer, rows, d] tensor, box
// [box_outer, box_rows, 64] with 128-byte swizzle (d split in 64-wide slabs).
struct TmaMap { alignas(64) unsigned char bytes[128]; };
cudaError_t make_tma_3d_bf16(TmaMap* out, const void* base, uint64_t d, uint64_t rows,
                             uint64_t outer, uint32_t box_rows, uint32_t box_outer);

// A 4-D bf16 tensor map (dims[0] = d, innermost; byte strides of dims 1..3),
// box `box` with 128-byte swizzle (box[0] = 64: one 128-byte row).  The
// strides need not grow with the dimension: the forward reads a query tile
// token-major (heads inner to tokens) through one.  Memoised like the 3-D maps.
cudaError_t make_tma_4d_bf16(TmaMap* out, const void* base, const uint64_t dims[4],
                             const uint64_t strides_bytes[3], const uint32_t box[4]);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) for `func` on the current
// device, done once per (device, function): later calls only look it up.
cudaError_t set_max_dynamic_smem(const void* func, int bytes);

}  // namespace moda
