// moda_api.cu -- the C ABI declared in include/moda.h: argument validation,
// workspace sizing, dispatch to the kernel launchers, status reporting.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "moda.h"
#include "moda_internal.h"

namespace moda {
namespace {

// Kernel-side status word, one per device (this is a device variable: every
// device that loads the library gets its own copy).
__device__ unsigned int g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
unsigned int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

thread_local std::string g_last_error;

constexpr int kMaxPhaseEvents = 8;
thread_local cudaEvent_t g_phase_events[kMaxPhaseEvents] = {};
thread_local int g_n_phase_events = 0;

moda_status fail(moda_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

moda_status cuda_fail(cudaError_t e, const char* what) {
    return fail(MODA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validate a shape; fill *p.  `tensor_core` selects the bf16 limits.
moda_status validate(const moda_shape* s, Problem* p) {
    if (!s) return fail(MODA_ERR_INVALID_ARG, "shape is NULL");
    if (s->dtype != MODA_BF16 && s->dtype != MODA_FP32)
        return fail(MODA_ERR_INVALID_ARG, "unknown dtype %d", (int)s->dtype);
    if (s->depth_layout != MODA_DEPTH_FLAT && s->depth_layout != MODA_DEPTH_CHUNKED &&
        s->depth_layout != MODA_DEPTH_LAYER)
        return fail(MODA_ERR_INVALID_ARG, "unknown depth layout %d", (int)s->depth_layout);
    if (s->B < 0 || s->T < 0 || s->L < 0)
        return fail(MODA_ERR_INVALID_ARG, "B=%d T=%d L=%d must be >= 0", s->B, s->T, s->L);
    if (s->Hq < 1 || s->Hk < 1 || s->Hq % s->Hk != 0)
        return fail(MODA_ERR_INVALID_ARG, "need Hq >= 1, Hk >= 1 and Hq %% Hk == 0 (Hq=%d Hk=%d)",
                    s->Hq, s->Hk);
    if (s->d < 1) return fail(MODA_ERR_INVALID_ARG, "d=%d must be >= 1", s->d);
    if (!(s->softmax_scale >= 0.0f) || std::isinf(s->softmax_scale))
        return fail(MODA_ERR_INVALID_ARG, "softmax_scale must be finite (<= 0 for 1/sqrt(d))");
    if (s->depth_layout == MODA_DEPTH_CHUNKED) {
        if (s->C < 1) return fail(MODA_ERR_INVALID_ARG, "chunked layout needs C >= 1 (C=%d)", s->C);
        if (s->T % s->C != 0)
            return fail(MODA_ERR_INVALID_ARG, "chunked layout needs T %% C == 0 (T=%d C=%d)", s->T,
                        s->C);
    } else if (s->C < 0) {
        return fail(MODA_ERR_INVALID_ARG, "C=%d must be >= 0", s->C);
    }
    if (s->flags & ~MODA_FLAG_NONCAUSAL)
        return fail(MODA_ERR_INVALID_ARG, "unknown flags 0x%x", (unsigned)s->flags);
    if (s->depth_window < 0 || s->depth_window > s->L)
        return fail(MODA_ERR_INVALID_ARG, "depth_window=%d must be in 0..L (L=%d)", s->depth_window,
                    s->L);
    const int G = s->Hq / s->Hk;
    if (s->dtype == MODA_BF16) {
        if (s->d != 64 && s->d != 128)
            return fail(MODA_ERR_UNSUPPORTED, "bf16 path supports d in {64, 128} (d=%d)", s->d);
        if (G > 128) return fail(MODA_ERR_UNSUPPORTED, "bf16 path supports G <= 128 (G=%d)", G);
    } else if (s->d > 128) {
        return fail(MODA_ERR_UNSUPPORTED, "fp32 path supports d <= 128 (d=%d)", s->d);
    }
    const bool layer = s->depth_layout == MODA_DEPTH_LAYER && s->L > 0;
    if (layer) {
        // whole tokens per depth block: the forward's blocks of n(128) rows and
        // the dQ kernel's of n(64) rows, n(c) = min(c, Tq*L rounded up to 16)
        if (s->dtype != MODA_BF16)
            return fail(MODA_ERR_UNSUPPORTED, "the layer-major depth layout needs the bf16 path");
        const long long dep = (long long)(128 / G) * s->L;
        const long long r16 = (dep + 15) / 16 * 16;
        const long long n128 = r16 < 128 ? r16 : 128, n64 = r16 < 64 ? r16 : 64;
        if (n128 % s->L != 0 || n64 % s->L != 0)
            return fail(MODA_ERR_UNSUPPORTED,
                        "layer-major depth layout: L=%d does not split the depth blocks (%lld, %lld rows) "
                        "into whole tokens; repack to the flat layout",
                        s->L, n128, n64);
    }
    // 64-bit element counts must stay addressable; the kernels index rows with
    // 32-bit (b*H + h) and token coordinates.
    const double rows_q = double(s->B) * s->Hq * s->T;
    const double rows_d = double(s->B) * s->Hk * s->T * double(s->L);
    if (rows_q > 2147483647.0 || rows_d > 2147483647.0 || double(s->T) * s->L > 2147483647.0)
        return fail(MODA_ERR_UNSUPPORTED, "problem too large for 32-bit row indices");
    p->B = s->B; p->Hq = s->Hq; p->Hk = s->Hk; p->T = s->T; p->d = s->d; p->L = s->L; p->G = G;
    p->scale = s->softmax_scale > 0.0f ? s->softmax_scale : 1.0f / std::sqrt(float(s->d));
    p->scale_log2 = p->scale * 1.4426950408889634f;
    p->elem_bytes = s->dtype == MODA_BF16 ? 2 : 4;
    p->causal = (s->flags & MODA_FLAG_NONCAUSAL) ? 0 : 1;
    p->win_lo = s->depth_window > 0 ? s->L - s->depth_window : 0;
    p->depth_layer = layer ? 1 : 0;
    return MODA_OK;
}

moda_status check_ptrs(std::initializer_list<std::pair<const void*, const char*>> ptrs) {
    for (auto& pr : ptrs) {
        if (!pr.first) return fail(MODA_ERR_INVALID_ARG, "%s is NULL", pr.second);
        if (!aligned16(pr.first))
            return fail(MODA_ERR_MISALIGNED, "%s is not 16-byte aligned", pr.second);
    }
    return MODA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

size_t bwd_workspace_bytes(const Problem& p) {
    return round_up(size_t(p.B) * p.Hq * p.T * sizeof(float), 256);
}

unsigned int* device_status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    if (!g_status_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<unsigned int*>(ptr);
    }
    return g_status_ptr[dev];
}

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    if (!g_sm_count[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_sm_count[dev] = n > 0 ? n : 148;
    }
    return g_sm_count[dev];
}

void phase_mark(int k, cudaStream_t stream) {
    if (k >= 0 && k < g_n_phase_events && g_phase_events[k]) cudaEventRecord(g_phase_events[k], stream);
}

// Hooks for entry points that live in other files of the library.
moda_status api_validate(const moda_shape* shape, Problem* p) { return validate(shape, p); }
moda_status api_fail(moda_status s, const char* msg) { return fail(s, "%s", msg); }

}  // namespace moda

using namespace moda;

extern "C" {

size_t moda_workspace_size(const moda_shape* shape, int for_bwd) {
    Problem p;
    if (validate(shape, &p) != MODA_OK) return static_cast<size_t>(-1);
    if (for_bwd < 0 || for_bwd > 2) return static_cast<size_t>(-1);
    if (!for_bwd) return 0;
    if (for_bwd == 2) return bwd_workspace_bytes(p);
    return bwd_workspace_bytes(p) + bwd_ds_bytes(p);
}

moda_status moda_repack_depth(const moda_shape* shape, const void* src, void* dst,
                              moda_stream_t stream) {
    Problem p;
    // the repack's layouts are fixed (layer-major in, token-major out)
    moda_shape flat;
    if (shape) {
        flat = *shape;
        flat.depth_layout = MODA_DEPTH_FLAT;
    }
    moda_status st = validate(shape ? &flat : nullptr, &p);
    if (st != MODA_OK) return st;
    if (p.B == 0 || p.T == 0 || p.L == 0) return MODA_OK;
    if ((st = check_ptrs({{src, "src"}, {dst, "dst"}})) != MODA_OK) return st;
    if (src == dst) return fail(MODA_ERR_INVALID_ARG, "repack cannot run in place");
    cudaError_t e = launch_repack(p.B, p.Hk, p.T, p.d, p.L, p.elem_bytes, src, dst,
                                  reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MODA_OK : cuda_fail(e, "repack launch");
}

moda_status moda_fwd(const moda_shape* shape, const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd, void* O, float* LSE, void* ws,
                     size_t ws_bytes, moda_stream_t stream) {
    (void)ws; (void)ws_bytes;
    Problem p;
    moda_status st = validate(shape, &p);
    if (st != MODA_OK) return st;
    if (p.B == 0 || p.T == 0) return MODA_OK;
    if ((st = check_ptrs({{Q, "Q"}, {K, "K"}, {V, "V"}, {O, "O"}, {LSE, "LSE"}})) != MODA_OK)
        return st;
    if (p.L > 0 && (st = check_ptrs({{Kd, "Kd"}, {Vd, "Vd"}})) != MODA_OK) return st;
    if (!device_status_word()) return fail(MODA_ERR_CUDA, "no usable CUDA device");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    phase_mark(0, s);
    cudaError_t e = p.elem_bytes == 2
                        ? launch_fwd_sm100(p, Q, K, V, Kd, Vd, O, LSE, s)
                        : launch_fwd_simt(p, Q, K, V, Kd, Vd, O, LSE, s);
    if (e == cudaSuccess) phase_mark(1, s);
    return e == cudaSuccess ? MODA_OK : cuda_fail(e, "forward launch");
}

moda_status moda_bwd(const moda_shape* shape, const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd, const void* O, const float* LSE,
                     const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                     void* ws, size_t ws_bytes, moda_stream_t stream) {
    Problem p;
    moda_status st = validate(shape, &p);
    if (st != MODA_OK) return st;
    if (p.B == 0 || p.T == 0) return MODA_OK;
    if ((st = check_ptrs({{Q, "Q"}, {K, "K"}, {V, "V"}, {O, "O"}, {LSE, "LSE"}, {dO, "dO"},
                          {dQ, "dQ"}, {dK, "dK"}, {dV, "dV"}})) != MODA_OK)
        return st;
    if (p.L > 0 &&
        (st = check_ptrs({{Kd, "Kd"}, {Vd, "Vd"}, {dKd, "dKd"}, {dVd, "dVd"}})) != MODA_OK)
        return st;
    const size_t need = bwd_workspace_bytes(p);
    if (!ws || ws_bytes < need)
        return fail(MODA_ERR_WORKSPACE, "backward needs %zu workspace bytes (got %zu%s)", need,
                    ws_bytes, ws ? "" : ", NULL");
    if (!aligned16(ws)) return fail(MODA_ERR_MISALIGNED, "ws is not 16-byte aligned");
    if (!device_status_word()) return fail(MODA_ERR_CUDA, "no usable CUDA device");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float* Dws = static_cast<float*>(ws);
    phase_mark(0, s);
    cudaError_t e =
        p.elem_bytes == 2
            ? launch_bwd_sm100(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, ws, ws_bytes, s)
            : launch_bwd_simt(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, Dws, s);
    return e == cudaSuccess ? MODA_OK : cuda_fail(e, "backward launch");
}

namespace {
// Decoding limits on top of the shared shape checks.
moda_status validate_decode(const moda_shape* shape, moda::Problem* p) {
    using namespace moda;
    // the depth layout has no effect on decoding (Kd, Vd are the new token's rows)
    moda_shape flat;
    if (shape) {
        flat = *shape;
        flat.depth_layout = MODA_DEPTH_FLAT;
    }
    moda_status st = validate(shape ? &flat : nullptr, p);
    if (st != MODA_OK) return st;
    if (p->B > 0 && p->T < 1) return fail(MODA_ERR_INVALID_ARG, "decoding needs T >= 1 cached keys");
    if (p->d != 64 && p->d != 128)
        return fail(MODA_ERR_UNSUPPORTED, "decoding supports d in {64, 128} (d=%d)", p->d);
    if (p->G > 16) return fail(MODA_ERR_UNSUPPORTED, "decoding supports G <= 16 (G=%d)", p->G);
    return MODA_OK;
}
}  // namespace

size_t moda_decode_workspace_size(const moda_shape* shape) {
    moda::Problem p;
    if (validate_decode(shape, &p) != MODA_OK) return static_cast<size_t>(-1);
    if (p.B == 0) return 0;
    return moda::decode_workspace_bytes(p);
}

moda_status moda_decode(const moda_shape* shape, const void* q, const void* K, const void* V,
                        const void* Kd, const void* Vd, void* o, float* lse, void* ws,
                        size_t ws_bytes, moda_stream_t stream) {
    using namespace moda;
    Problem p;
    moda_status st = validate_decode(shape, &p);
    if (st != MODA_OK) return st;
    if (p.B == 0) return MODA_OK;
    if ((st = check_ptrs({{q, "q"}, {K, "K"}, {V, "V"}, {o, "o"}, {lse, "lse"}, {ws, "ws"}})) != MODA_OK)
        return st;
    if (p.L > 0 && (st = check_ptrs({{Kd, "Kd"}, {Vd, "Vd"}})) != MODA_OK) return st;
    if (!device_status_word()) return fail(MODA_ERR_CUDA, "no usable CUDA device");
    const size_t need = decode_workspace_bytes(p);
    if (ws_bytes < need)
        return fail(MODA_ERR_WORKSPACE, "decoding needs %zu bytes of workspace (got %zu)", need, ws_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    phase_mark(0, s);
    cudaError_t e = launch_decode(p, q, K, V, Kd, Vd, o, lse, ws, s);
    if (e == cudaSuccess) phase_mark(1, s);
    return e == cudaSuccess ? MODA_OK : cuda_fail(e, "decode launch");
}

moda_status moda_check_status(moda_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int* w = device_status_word();
    if (!w) return fail(MODA_ERR_CUDA, "no usable CUDA device");
    unsigned int v = 0;
    e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (v) {
        const unsigned int zero = 0;
        e = cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "status clear");
        if (v & kStatusTimeout) return fail(MODA_ERR_TIMEOUT, "a kernel wait timed out");
    }
    return MODA_OK;
}

const char* moda_status_string(moda_status status) {
    switch (status) {
        case MODA_OK: return "MODA_OK";
        case MODA_ERR_INVALID_ARG: return "MODA_ERR_INVALID_ARG";
        case MODA_ERR_MISALIGNED: return "MODA_ERR_MISALIGNED";
        case MODA_ERR_UNSUPPORTED: return "MODA_ERR_UNSUPPORTED";
        case MODA_ERR_WORKSPACE: return "MODA_ERR_WORKSPACE";
        case MODA_ERR_CUDA: return "MODA_ERR_CUDA";
        case MODA_ERR_TIMEOUT: return "MODA_ERR_TIMEOUT";
    }
    return "MODA_ERR_UNKNOWN";
}

const char* moda_last_error_message(void) { return g_last_error.c_str(); }

moda_status moda_set_phase_events(void* const* events, int n) {
    if (n < 0 || n > kMaxPhaseEvents) return fail(MODA_ERR_INVALID_ARG, "n=%d must be 0..%d", n, kMaxPhaseEvents);
    if (n > 0 && !events) return fail(MODA_ERR_INVALID_ARG, "events is NULL");
    for (int i = 0; i < kMaxPhaseEvents; ++i)
        g_phase_events[i] = i < n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
    g_n_phase_events = n;
    return MODA_OK;
}

int moda_version(void) { return 10200; }

}  // extern "C"
