// trace.cu -- optional per-kernel timing of the library's launches.
//
// While tracing is on (gdn2_trace_enable(1)), each kernel launch is bracketed by
// two CUDA events recorded on the launch's stream. gdn2_trace_read() waits for
// the recorded events, returns per kernel the number of launches and the summed
// device time, and forgets them. Off by default; when off the launch path only
// reads one flag.
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "gdn2.h"
#include "internal.h"

namespace gdn2 {
namespace {

const char* kNames[KERNEL_COUNT] = {"chunk_fwd_kernel", "chunk_bwd_kernel", "recurrent_fwd_kernel",
                                    "recurrent_bwd_kernel", "decode_kernel", "gate_expand_kernel",
                                    "gate_reduce_kernel", "pad_copy_kernel", "split_prefix_kernel",
                                    "state_affine_kernel", "gates_fwd_kernel", "gates_bwd_kernel"};

std::atomic<int> g_on{0};
std::mutex g_mu;
struct Rec {
    int kernel;
    cudaEvent_t start, stop;
};
std::vector<Rec> g_recs;

}  // namespace

TraceScope::TraceScope(KernelId id, cudaStream_t s) : id_(id), stream_(s), start_(nullptr), active_(false) {
    if (!g_on.load(std::memory_order_relaxed)) return;
    if (cudaEventCreate(&start_) != cudaSuccess) return;
    if (cudaEventRecord(start_, stream_) != cudaSuccess) {
        cudaEventDestroy(start_);
        return;
    }
    active_ = true;
}

TraceScope::~TraceScope() {
    if (!active_) return;
    cudaEvent_t stop = nullptr;
    if (cudaEventCreate(&stop) != cudaSuccess || cudaEventRecord(stop, stream_) != cudaSuccess) {
        if (stop) cudaEventDestroy(stop);
        cudaEventDestroy(start_);
        return;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    g_recs.push_back(Rec{(int)id_, start_, stop});
}

}  // namespace gdn2

extern "C" {

void gdn2_trace_enable(int on) { gdn2::g_on.store(on ? 1 : 0); }

int gdn2_trace_read(char* names, size_t names_cap, int* launches, double* ms, int max_kernels) {
    using namespace gdn2;
    std::vector<Rec> recs;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        recs.swap(g_recs);
    }
    int cnt[KERNEL_COUNT] = {0};
    double tot[KERNEL_COUNT] = {0.0};
    for (const Rec& r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) == cudaSuccess && cudaEventElapsedTime(&t, r.start, r.stop) == cudaSuccess) {
            cnt[r.kernel] += 1;
            tot[r.kernel] += t;
        }
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    int n = 0;
    size_t used = 0;
    if (names && names_cap) names[0] = '\0';
    for (int k = 0; k < KERNEL_COUNT && n < max_kernels; ++k) {
        if (!cnt[k]) continue;
        if (launches) launches[n] = cnt[k];
        if (ms) ms[n] = tot[k];
        if (names) {
            int w = snprintf(names + used, names_cap > used ? names_cap - used : 0, "%s%s", n ? "," : "", kNames[k]);
            if (w > 0) used += (size_t)w;
        }
        ++n;
    }
    return n;
}

}  // extern "C"
