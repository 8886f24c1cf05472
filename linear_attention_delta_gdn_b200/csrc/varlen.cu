// varlen.cu -- variable-length sequences packed along the token axis (cu_seqlens).
//
// The sequences of a batch of different lengths are packed back to back, [Ttot, H, D]; sequence n holds
// tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 and has its own initial and final state. The calls copy the
// packed tensors into a zero-padded [N, Tmax, H, D] layout in the workspace, run gdn2_fwd / gdn2_bwd on it,
// and copy the results back. Padding is exact, not an approximation: a padded token has k = q = v = b = w = 0
// and log_alpha = 0, so it maps the state to itself (S_t = (I - 0) Diag(1) S + 0) and leaves the final state
// and every gradient of the real tokens unchanged; its own outputs are dropped. Every chunk of the padded run
// starts at a sequence's start, so each sequence ends in its own ragged chunk.
//
// cu_seqlens stays in device memory (nothing synchronises); the caller passes N, Tmax (the longest length,
// rounded up as it likes) and Ttot (the packed length). A sequence longer than Tmax is cut at Tmax, and a
// sequence reaching past Ttot (or a decreasing cu_seqlens) is dropped from the copies; both are reported by
// gdn2_device_status (GDN2_ERR_INVALID, detail "cu_seqlens").
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "common.cuh"
#include "gdn2.h"
#include "internal.h"

namespace gdn2 {

__device__ unsigned int g_varlen_error;   // bit 1: a sequence longer than Tmax; bit 2: one outside [0, Ttot)

namespace {

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

// pad[n][t][h][:] = t < len_n ? packed[cu[n] + t][h][:] : 0 (gather), or the reverse copy for t < len_n
// (scatter). One thread per 16 bytes of a row; rows are (n, t, h) of the padded layout.
__global__ void pad_copy_kernel(const int* __restrict__ cu, int N, int Tmax, long long Ttot, int H, int row_bytes,
                                const unsigned char* __restrict__ src, unsigned char* __restrict__ dst, int gather) {
    const int per = row_bytes / 16;
    const long long total = (long long)N * Tmax * H * per;
    for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        const int p = (int)(x % per);
        const long long row = x / per;
        const int h = (int)(row % H);
        const long long nt = row / H;
        const int t = (int)(nt % Tmax), n = (int)(nt / Tmax);
        const int start = cu[n], len = cu[n + 1] - start;
        const bool inside = start >= 0 && len >= 0 && (long long)start + len <= Ttot;
        if (t == 0 && h == 0 && p == 0) {
            if (len > Tmax) atomicOr(&g_varlen_error, 1u);
            if (!inside) atomicOr(&g_varlen_error, 2u);
        }
        const bool real = inside && t < len;
        const long long prow = ((long long)start + t) * H + h;   // row of the packed tensor
        const size_t poff = (size_t)prow * row_bytes + 16 * p, qoff = (size_t)row * row_bytes + 16 * p;
        if (gather) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (real) v = *reinterpret_cast<const uint4*>(src + poff);
            *reinterpret_cast<uint4*>(dst + qoff) = v;
        } else if (real) {
            *reinterpret_cast<uint4*>(dst + poff) = *reinterpret_cast<const uint4*>(src + qoff);
        }
    }
}

cudaError_t pad_copy(const int* cu, int N, int Tmax, long long Ttot, int H, int D, size_t es, const void* src,
                     void* dst, bool gather, cudaStream_t s) {
    const int row_bytes = (int)(D * es);
    const long long work = (long long)N * Tmax * H * (row_bytes / 16);
    if (work == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (work + 255) / 256, cap = (long long)sms * 16;
    TraceScope trace(K_VARLEN_COPY, s);
    pad_copy_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(cu, N, Tmax, Ttot, H, row_bytes,
                                                                   static_cast<const unsigned char*>(src),
                                                                   static_cast<unsigned char*>(dst), gather ? 1 : 0);
    return cudaGetLastError();
}

// Workspace (each region 256-byte aligned): [gdn2 workspace for (B = N, T = Tmax), of GDN2_OP_FWD for a plain
// forward, else of GDN2_OP_BWD] then the padded q, k, log_alpha, b (Dk) and v, w (Dv), then the padded o (Dv)
// for the forward, or the padded dout (Dv), dq, dk, dlog_alpha, db (Dk), dv, dw (Dv) for the backward.
struct VLayout {
    size_t base;
    size_t in[6];       // q, k, v, log_alpha, b, w
    size_t out[7];      // forward: o; backward: dout, dq, dk, dv, dlog_alpha, db, dw
    size_t total;
};
VLayout vlayout(gdn2_op op, int N, int Tmax, int H, int Dk, int Dv, int chunk, gdn2_dtype dt) {
    VLayout L{};
    const size_t es = dt == GDN2_BF16 ? 2 : 4, rows = (size_t)N * Tmax * H;
    const size_t kb = al256(rows * Dk * es), vb = al256(rows * Dv * es);
    L.base = al256(gdn2_workspace_size(op == GDN2_OP_FWD ? GDN2_OP_FWD : GDN2_OP_BWD, N, Tmax, H, Dk, Dv, chunk, dt));
    size_t off = L.base;
    const int in_dim[6] = {Dk, Dk, Dv, Dk, Dk, Dv};
    for (int i = 0; i < 6; ++i) {
        L.in[i] = off;
        off += in_dim[i] == Dk ? kb : vb;
    }
    if (op == GDN2_OP_BWD) {
        const int out_dim[7] = {Dv, Dk, Dk, Dv, Dk, Dk, Dv};
        for (int i = 0; i < 7; ++i) {
            L.out[i] = off;
            off += out_dim[i] == Dk ? kb : vb;
        }
    } else {
        L.out[0] = off;
        off += vb;
    }
    L.total = off;
    return L;
}

thread_local char g_err[256];
gdn2_status report(gdn2_status s) {
    set_last_error(g_err);
    return s;
}

gdn2_status check(const int* cu_seqlens, int N, int Tmax, long long Ttot, int H, int Dk, int Dv, int chunk,
                  gdn2_dtype dt, size_t need, void* ws, size_t ws_bytes, const char* fn) {
    if (N < 1 || Tmax < 0 || Ttot < 0) {
        snprintf(g_err, sizeof(g_err), "%s: N=%d must be >= 1, Tmax=%d and Ttot=%lld >= 0", fn, N, Tmax, Ttot);
        return report(GDN2_ERR_INVALID);
    }
    if (!cu_seqlens) {
        snprintf(g_err, sizeof(g_err), "%s: cu_seqlens must not be NULL", fn);
        return report(GDN2_ERR_INVALID);
    }
    if (Tmax > 0 && gdn2_workspace_size(GDN2_OP_BWD, N, Tmax, H, Dk, Dv, chunk, dt) == 0) {
        snprintf(g_err, sizeof(g_err), "%s: unsupported sizes (H=%d, Dk=%d, Dv=%d, chunk=%d, dtype=%d)", fn, H, Dk,
                 Dv, chunk, (int)dt);
        return report(GDN2_ERR_UNSUPPORTED);
    }
    if (need && (!ws || ws_bytes < need)) {
        snprintf(g_err, sizeof(g_err), "%s needs %zu workspace bytes, got %zu", fn, need, ws ? ws_bytes : 0);
        return report(GDN2_ERR_WORKSPACE);
    }
    if (need && ((uintptr_t)ws & 255)) {
        snprintf(g_err, sizeof(g_err), "%s: ws must be 256-byte aligned", fn);
        return report(GDN2_ERR_INVALID);
    }
    return GDN2_OK;
}

gdn2_status check_ptrs(const void* const* ptrs, int n, const char* fn) {
    for (int i = 0; i < n; ++i) {
        if (!ptrs[i]) {
            snprintf(g_err, sizeof(g_err), "%s: token tensors must not be NULL", fn);
            return report(GDN2_ERR_INVALID);
        }
        if ((uintptr_t)ptrs[i] & 15) {
            snprintf(g_err, sizeof(g_err), "%s: token tensors must be 16-byte aligned", fn);
            return report(GDN2_ERR_INVALID);
        }
    }
    return GDN2_OK;
}

gdn2_status cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_err, sizeof(g_err), "%s: %s", where, cudaGetErrorString(e));
    return report(GDN2_ERR_CUDA);
}

}  // namespace

cudaError_t varlen_take_errors(unsigned int* bits) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, g_varlen_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_varlen_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn2

using namespace gdn2;

extern "C" {

size_t gdn2_varlen_workspace_size(gdn2_op op, int N, int Tmax, int H, int Dk, int Dv, int chunk, gdn2_dtype dt) {
    if (N < 1 || Tmax < 0) return 0;
    if (Tmax > 0 && gdn2_workspace_size(GDN2_OP_BWD, N, Tmax, H, Dk, Dv, chunk, dt) == 0) return 0;
    return vlayout(op, N, Tmax, H, Dk, Dv, chunk, dt).total;
}

gdn2_status gdn2_varlen_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                            const void* w, const int* cu_seqlens, int N, int Tmax, long long Ttot, const float* S0,
                            void* o,
                            float* ST, int H, int Dk, int Dv, int chunk, gdn2_dtype dt, int save_states, void* ws,
                            size_t ws_bytes, void* stream) {
    const gdn2_op op = save_states ? GDN2_OP_FWD_SAVE : GDN2_OP_FWD;
    const VLayout L = vlayout(op, N, Tmax, H, Dk, Dv, chunk, dt);
    gdn2_status st = check(cu_seqlens, N, Tmax, Ttot, H, Dk, Dv, chunk, dt, L.total, ws, ws_bytes, "gdn2_varlen_fwd");
    if (st != GDN2_OK) return st;
    if (Tmax > 0) {
        const void* ptrs[7] = {q, k, v, log_alpha, b, w, o};
        if ((st = check_ptrs(ptrs, 7, "gdn2_varlen_fwd")) != GDN2_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* w8 = static_cast<unsigned char*>(ws);
    const size_t es = dt == GDN2_BF16 ? 2 : 4;
    const void* src[6] = {q, k, v, log_alpha, b, w};
    const int dim[6] = {Dk, Dk, Dv, Dk, Dk, Dv};
    for (int i = 0; i < 6 && Tmax > 0; ++i) {
        cudaError_t e = pad_copy(cu_seqlens, N, Tmax, Ttot, H, dim[i], es, src[i], w8 + L.in[i], true, s);
        if (e != cudaSuccess) return cuda_fail(e, "gdn2_varlen_fwd (padding)");
    }
    st = gdn2_fwd(w8 + L.in[0], w8 + L.in[1], w8 + L.in[2], w8 + L.in[3], w8 + L.in[4], w8 + L.in[5], S0,
                  w8 + L.out[0], ST, N, Tmax, H, Dk, Dv, chunk, dt, save_states, ws, L.base, stream);
    if (st != GDN2_OK || Tmax == 0) return st;
    cudaError_t e = pad_copy(cu_seqlens, N, Tmax, Ttot, H, Dv, es, w8 + L.out[0], o, false, s);
    return e == cudaSuccess ? GDN2_OK : cuda_fail(e, "gdn2_varlen_fwd (unpadding)");
}

gdn2_status gdn2_varlen_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                            const void* w, const int* cu_seqlens, int N, int Tmax, long long Ttot, const float* S0,
                            const void* dout,
                            const float* dST, void* dq, void* dk, void* dv, void* dlog_alpha, void* db, void* dw,
                            float* dS0, int H, int Dk, int Dv, int chunk, gdn2_dtype dt, int states_saved, void* ws,
                            size_t ws_bytes, void* stream) {
    const VLayout L = vlayout(GDN2_OP_BWD, N, Tmax, H, Dk, Dv, chunk, dt);
    gdn2_status st = check(cu_seqlens, N, Tmax, Ttot, H, Dk, Dv, chunk, dt, L.total, ws, ws_bytes, "gdn2_varlen_bwd");
    if (st != GDN2_OK) return st;
    if (Tmax > 0) {
        const void* ptrs[13] = {q, k, v, log_alpha, b, w, dout, dq, dk, dv, dlog_alpha, db, dw};
        if ((st = check_ptrs(ptrs, 13, "gdn2_varlen_bwd")) != GDN2_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* w8 = static_cast<unsigned char*>(ws);
    const size_t es = dt == GDN2_BF16 ? 2 : 4;
    const void* src[7] = {q, k, v, log_alpha, b, w, dout};
    const size_t dst[7] = {L.in[0], L.in[1], L.in[2], L.in[3], L.in[4], L.in[5], L.out[0]};
    const int dim[7] = {Dk, Dk, Dv, Dk, Dk, Dv, Dv};
    for (int i = 0; i < 7 && Tmax > 0; ++i) {
        cudaError_t e = pad_copy(cu_seqlens, N, Tmax, Ttot, H, dim[i], es, src[i], w8 + dst[i], true, s);
        if (e != cudaSuccess) return cuda_fail(e, "gdn2_varlen_bwd (padding)");
    }
    st = gdn2_bwd(w8 + L.in[0], w8 + L.in[1], w8 + L.in[2], w8 + L.in[3], w8 + L.in[4], w8 + L.in[5], S0,
                  w8 + L.out[0], dST, w8 + L.out[1], w8 + L.out[2], w8 + L.out[3], w8 + L.out[4], w8 + L.out[5],
                  w8 + L.out[6], dS0, N, Tmax, H, Dk, Dv, chunk, dt, states_saved, ws, L.base, stream);
    if (st != GDN2_OK || Tmax == 0) return st;
    void* outs[6] = {dq, dk, dv, dlog_alpha, db, dw};
    const int odim[6] = {Dk, Dk, Dv, Dk, Dk, Dv};
    for (int i = 0; i < 6; ++i) {
        cudaError_t e = pad_copy(cu_seqlens, N, Tmax, Ttot, H, odim[i], es, w8 + L.out[1 + i], outs[i], false, s);
        if (e != cudaSuccess) return cuda_fail(e, "gdn2_varlen_bwd (unpadding)");
    }
    return GDN2_OK;
}

}  // extern "C"
