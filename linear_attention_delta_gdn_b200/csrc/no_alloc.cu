// no_alloc.cu -- gdn2_bwd_no_alloc: the backward without a caller-supplied workspace.
//
// Some callers cannot call cudaMalloc at the point where they need gradients:
// code that runs inside another component's memory management (a framework's
// caching allocator, or a plugin handed only the tensors it reads and writes),
// code that must not synchronise the device (cudaMalloc and cudaFree may), and
// code that must not be able to fail for lack of memory after start-up. For
// them this entry point takes the scratch memory of the backward from a fixed
// array in this library instead of from the caller. It allocates nothing.
//
// The array (GDN2_NO_ALLOC_SCRATCH_BYTES) lives in device memory of every GPU
// that loads the library, for as long as the library stays loaded. All calls on
// one device share it and it keeps the last call's contents; the backward writes
// every scratch byte it reads, so nothing in it has to start at zero. Calls
// whose work overlaps on the GPU (different streams, or different host threads,
// on the same device) race on the array and give wrong results: order them.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdio.h>

#include <mutex>

#include "gdn2.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)GDN2_NO_ALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 256;
void* g_scratch_ptr[kMaxDevices];   // device address of g_scratch, per device (null: not set up)
std::mutex g_setup_mutex;

thread_local char g_no_alloc_err[256];

gdn2_status report(gdn2_status s) {
    gdn2::set_last_error(g_no_alloc_err);
    return s;
}

// Device address of the scratch array on the current device. The host-side
// symbol is only a stand-in: its device address has to be looked up, once per
// device, with that device current.
gdn2_status scratch_for_current_device(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        snprintf(g_no_alloc_err, sizeof(g_no_alloc_err), "gdn2_bwd_no_alloc: no usable current device (%s)",
                 cudaGetErrorString(e));
        return GDN2_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) {
            snprintf(g_no_alloc_err, sizeof(g_no_alloc_err),
                     "gdn2_bwd_no_alloc: cudaGetSymbolAddress failed on device %d (%s)", dev, cudaGetErrorString(e));
            return GDN2_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GDN2_OK;
}

}  // namespace

extern "C" {

size_t gdn2_no_alloc_scratch_bytes(void) { return kScratchBytes; }

gdn2_status gdn2_bwd_no_alloc(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                              const void* w, const float* S0, const void* dout, const float* dST, void* dq,
                              void* dk, void* dv, void* dlog_alpha, void* db, void* dw, float* dS0, int B, int T,
                              int H, int Dk, int Dv, int chunk, gdn2_dtype dt, void* stream) {
    const size_t need = gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt);
    if (need > kScratchBytes) {
        snprintf(g_no_alloc_err, sizeof(g_no_alloc_err),
                 "gdn2_bwd_no_alloc: this problem needs %zu scratch bytes, the fixed array holds %zu "
                 "(use gdn2_bwd with a workspace)", need, kScratchBytes);
        return report(GDN2_ERR_WORKSPACE);
    }
    void* scratch = nullptr;
    gdn2_status st = scratch_for_current_device(&scratch);
    if (st != GDN2_OK) return report(st);
    // The chunk-start states are recomputed into the scratch (states_saved = 0).
    return gdn2_bwd(q, k, v, log_alpha, b, w, S0, dout, dST, dq, dk, dv, dlog_alpha, db, dw, dS0, B, T, H, Dk, Dv,
                    chunk, dt, 0, scratch, kScratchBytes, stream);
}

}  // extern "C"
