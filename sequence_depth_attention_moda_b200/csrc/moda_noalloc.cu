// moda_noalloc.cu -- moda_bwd_noalloc: the backward for callers that cannot
// allocate device memory.  The only scratch the backward needs (D, one fp32
// per query row) lives in a fixed array compiled into the library instead of a
// caller-provided workspace.  The pages have no counterpart to this.
#include <cstdio>
#include <mutex>
#include <utility>

#include "moda.h"
#include "moda_internal.h"

namespace moda {
namespace {

// Capacity in query rows (B * Hq * T): 4 Mi rows = 16 MiB of fp32.  Every
// device that loads the library holds this array until the process exits.
constexpr size_t kScratchRows = size_t(4) << 20;
__device__ __align__(256) float g_bwd_scratch[kScratchRows];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_bwd_scratch on the current device.  In host code the
// array's name only stands in for the symbol, so the address is looked up
// once per device (with that device current) and cached.
moda_status scratch_for_current_device(float** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return api_fail(MODA_ERR_CUDA, "moda_bwd_noalloc: no usable CUDA device");
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
        if (e != cudaSuccess || !ptr) {
            char msg[160];
            snprintf(msg, sizeof(msg), "moda_bwd_noalloc: cudaGetSymbolAddress failed: %s",
                     cudaGetErrorString(e));
            return api_fail(MODA_ERR_CUDA, msg);
        }
        g_scratch_ptr[dev] = static_cast<float*>(ptr);
    }
    *out = g_scratch_ptr[dev];
    return MODA_OK;
}

// The same pointer rules and status codes as moda_bwd: NULL is an invalid
// argument, an address off a 16-byte boundary is misaligned.
moda_status check_ptr(const void* p, const char* name) {
    char msg[120];
    if (!p) {
        snprintf(msg, sizeof(msg), "moda_bwd_noalloc: %s is NULL", name);
        return api_fail(MODA_ERR_INVALID_ARG, msg);
    }
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) {
        snprintf(msg, sizeof(msg), "moda_bwd_noalloc: %s is not 16-byte aligned", name);
        return api_fail(MODA_ERR_MISALIGNED, msg);
    }
    return MODA_OK;
}

}  // namespace
}  // namespace moda

using namespace moda;

extern "C" moda_status moda_bwd_noalloc(const moda_shape* shape, const void* Q, const void* K,
                                        const void* V, const void* Kd, const void* Vd,
                                        const void* O, const float* LSE, const void* dO, void* dQ,
                                        void* dK, void* dV, void* dKd, void* dVd,
                                        moda_stream_t stream) {
    Problem p;
    moda_status st = api_validate(shape, &p);
    if (st != MODA_OK) return st;
    if (p.B == 0 || p.T == 0) return MODA_OK;
    const std::pair<const void*, const char*> need[] = {
        {Q, "Q"}, {K, "K"}, {V, "V"}, {O, "O"}, {LSE, "LSE"}, {dO, "dO"}, {dQ, "dQ"}, {dK, "dK"}, {dV, "dV"}};
    for (const auto& pr : need)
        if ((st = check_ptr(pr.first, pr.second)) != MODA_OK) return st;
    if (p.L > 0) {
        const std::pair<const void*, const char*> dep[] = {{Kd, "Kd"}, {Vd, "Vd"}, {dKd, "dKd"}, {dVd, "dVd"}};
        for (const auto& pr : dep)
            if ((st = check_ptr(pr.first, pr.second)) != MODA_OK) return st;
    }
    const size_t rows = size_t(p.B) * p.Hq * p.T;
    if (rows > kScratchRows) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "moda_bwd_noalloc: B*Hq*T = %zu exceeds its built-in scratch of %zu rows; "
                 "use moda_bwd with a workspace", rows, kScratchRows);
        return api_fail(MODA_ERR_WORKSPACE, msg);
    }
    if (!device_status_word()) return api_fail(MODA_ERR_CUDA, "moda_bwd_noalloc: no usable CUDA device");
    float* scratch = nullptr;
    if ((st = scratch_for_current_device(&scratch)) != MODA_OK) return st;
    // D rows need no clearing: the first kernel of the call writes every row
    // of [0, B*Hq*T) before any later kernel reads it.  Only the D rows are
    // offered, so the dQ kernel recomputes S and dP (no stored dS tiles).
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    phase_mark(0, s);
    cudaError_t e =
        p.elem_bytes == 2
            ? launch_bwd_sm100(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, scratch,
                               bwd_workspace_bytes(p), s)
            : launch_bwd_simt(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, scratch, s);
    if (e != cudaSuccess) {
        char msg[160];
        snprintf(msg, sizeof(msg), "moda_bwd_noalloc: launch failed: %s", cudaGetErrorString(e));
        return api_fail(MODA_ERR_CUDA, msg);
    }
    return MODA_OK;
}
