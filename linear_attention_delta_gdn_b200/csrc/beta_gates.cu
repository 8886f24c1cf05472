// beta_gates.cu -- KDA and Gated DeltaNet through the Gated Delta Rule-2 kernels.
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention" (README "Strict Generalization"
// bullet, arXiv abstract) states that the operator reduces to KDA when the erase and write gates are one
// scalar beta_t per head and token (b_t = w_t = beta_t 1), and further to Gated DeltaNet when the decay is
// also one scalar per head and token. These entry points take the reduced gates. On the tensor-core path
// (bf16, Dk = Dv = 128) the chunk kernels have instances for a scalar erase and write gate and for a scalar
// decay too: beta (and log_a) go in as they are, and dbeta_t = sum_i db_ti + sum_j dw_tj (and dlog_a_t =
// sum_i dlog_alpha_ti) come out of the backward's gradient units. Elsewhere (or with beta, log_a not 4-byte
// aligned) the gates are broadcast into the workspace, gdn2_fwd / gdn2_bwd run on them, and their gradients
// are summed back over the channels, by memory-bound elementwise kernels (a row per lane group, 16-byte
// pieces, a few rows in flight per warp); each call broadcasts what it needs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "common.cuh"
#include "gdn2.h"
#include "internal.h"

namespace gdn2 {
namespace {

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

// One 16-byte piece of copies of v (8 bf16 or 4 fp32)
__device__ __forceinline__ void store_piece(__nv_bfloat16* dst, __nv_bfloat16 v) {
    const uint32_t x = (uint32_t)__bfloat16_as_ushort(v) * 0x10001u;
    *reinterpret_cast<uint4*>(dst) = make_uint4(x, x, x, x);
}
__device__ __forceinline__ void store_piece(float* dst, float v) {
    *reinterpret_cast<float4*>(dst) = make_float4(v, v, v, v);
}
// The sum of one 16-byte piece
__device__ __forceinline__ float sum_piece(const __nv_bfloat16* src) {
    const uint4 x = *reinterpret_cast<const uint4*>(src);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        s += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xFFFF0000u);
    return s;
}
__device__ __forceinline__ float sum_piece(const float* src) {
    const float4 x = *reinterpret_cast<const float4*>(src);
    return (x.x + x.y) + (x.z + x.w);
}

constexpr int ROWS_PER_WARP = 4;   // row steps a warp has in flight (their loads issued before any store)

// Lanes that share a row: the pieces per row rounded up to a power of two, at most the warp.
__device__ __forceinline__ int lanes_per_row(int per) {
    int g = 1;
    while (g < per && g < 32) g <<= 1;
    return g;
}

// Per-row broadcast: row r = (b, t, h); b[r][0:Dk] = beta[r], w[r][0:Dv] = beta[r] (unless b, w are null),
// la[r][0:Dk] = la_s[r] (scalar decay only). G lanes share a row (32 / G rows per warp at a time, ROWS_PER_WARP
// times over); lane g of a row writes the 16-byte pieces g, g + G, ... of its [b | w | la] concatenation (Dk,
// Dv are multiples of 16: whole pieces).
template <typename Tin>
__global__ void expand_kernel(const Tin* __restrict__ beta, const Tin* __restrict__ la_s, Tin* __restrict__ b,
                              Tin* __restrict__ w, Tin* __restrict__ la, long long rows, int Dk, int Dv) {
    constexpr int E = 16 / (int)sizeof(Tin);
    const int lane = threadIdx.x & 31;
    const int nb = b ? Dk / E : 0, nw = w ? Dv / E : 0, per = nb + nw + (la_s ? Dk / E : 0);
    const int G = lanes_per_row(per), rps = 32 / G, sub = lane / G, gl = lane % G;
    const long long step = (long long)ROWS_PER_WARP * rps;   // rows per warp and pass
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r0 = (blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5)) * step; r0 < rows;
         r0 += warps * step) {
        Tin bv[ROWS_PER_WARP], lv[ROWS_PER_WARP];
#pragma unroll
        for (int j = 0; j < ROWS_PER_WARP; ++j) {
            long long r = r0 + j * rps + sub;
            if (r >= rows) r = rows - 1;
            bv[j] = nb + nw ? beta[r] : Tin{};
            lv[j] = la_s ? la_s[r] : bv[j];
        }
#pragma unroll
        for (int j = 0; j < ROWS_PER_WARP; ++j) {
            const long long r = r0 + j * rps + sub;
            if (r >= rows) break;
            for (int p = gl; p < per; p += G) {
                if (p < nb)
                    store_piece(b + r * Dk + E * p, bv[j]);
                else if (p < nb + nw)
                    store_piece(w + r * Dv + E * (p - nb), bv[j]);
                else
                    store_piece(la + r * Dk + E * (p - nb - nw), lv[j]);
            }
        }
    }
}

// Per-row sums: dbeta[r] = sum db[r] + sum dw[r] (unless db, dw are null); dla_s[r] = sum dla[r] (scalar decay
// only). Rows shared out as in expand_kernel; all of a pass's 16-byte pieces are loaded before the sums.
template <typename Tin>
__global__ void reduce_kernel(const Tin* __restrict__ db, const Tin* __restrict__ dw, const Tin* __restrict__ dla,
                              Tin* __restrict__ dbeta, Tin* __restrict__ dla_s, long long rows, int Dk, int Dv) {
    constexpr int E = 16 / (int)sizeof(Tin);
    const int lane = threadIdx.x & 31;
    const int nb = db ? Dk / E : 0, nw = dw ? Dv / E : 0, per = nb + nw + (dla ? Dk / E : 0);
    const int G = lanes_per_row(per), rps = 32 / G, sub = lane / G, gl = lane % G;
    const long long step = (long long)ROWS_PER_WARP * rps;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r0 = (blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5)) * step; r0 < rows;
         r0 += warps * step) {
        float sb[ROWS_PER_WARP], sl[ROWS_PER_WARP];
#pragma unroll
        for (int j = 0; j < ROWS_PER_WARP; ++j) {
            sb[j] = 0.f;
            sl[j] = 0.f;
            const long long r = r0 + j * rps + sub;
            if (r >= rows) continue;
            for (int p = gl; p < per; p += G) {
                if (p < nb)
                    sb[j] += sum_piece(db + r * Dk + E * p);
                else if (p < nb + nw)
                    sb[j] += sum_piece(dw + r * Dv + E * (p - nb));
                else
                    sl[j] += sum_piece(dla + r * Dk + E * (p - nb - nw));
            }
        }
#pragma unroll
        for (int j = 0; j < ROWS_PER_WARP; ++j) {
            for (int m = G >> 1; m >= 1; m >>= 1) {   // within the G lanes of the row
                sb[j] += __shfl_xor_sync(0xffffffffu, sb[j], m);
                sl[j] += __shfl_xor_sync(0xffffffffu, sl[j], m);
            }
            const long long r = r0 + j * rps + sub;
            if (gl == 0 && r < rows) {
                if (nb + nw) dbeta[r] = from_f32<Tin>(sb[j]);
                if (dla) dla_s[r] = from_f32<Tin>(sl[j]);
            }
        }
    }
}

// Enough blocks of `block` threads for `work` threads, at most as many as are resident at once (a whole
// number of waves: the kernels are grid-stride loops)
template <typename K>
int grid_for(K kernel, long long work, int block) {
    int dev = 0, sms = 148, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, block, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const long long want = (work + block - 1) / block;
    const long long cap = (long long)sms * per_sm;
    return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

template <typename Tin>
cudaError_t launch_expand(const void* beta, const void* la_s, void* b, void* w, void* la, long long rows, int Dk,
                          int Dv, cudaStream_t s) {
    TraceScope trace(K_GATE_EXPAND, s);
    expand_kernel<Tin><<<grid_for(expand_kernel<Tin>, rows * 32 / ROWS_PER_WARP, 256), 256, 0, s>>>(static_cast<const Tin*>(beta), static_cast<const Tin*>(la_s),
                                                          static_cast<Tin*>(b), static_cast<Tin*>(w),
                                                          static_cast<Tin*>(la), rows, Dk, Dv);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_reduce(const void* db, const void* dw, const void* dla, void* dbeta, void* dla_s, long long rows,
                          int Dk, int Dv, cudaStream_t s) {
    TraceScope trace(K_GATE_REDUCE, s);
    reduce_kernel<Tin><<<grid_for(reduce_kernel<Tin>, rows * 32 / ROWS_PER_WARP, 256), 256, 0, s>>>(
        static_cast<const Tin*>(db), static_cast<const Tin*>(dw), static_cast<const Tin*>(dla),
        static_cast<Tin*>(dbeta), static_cast<Tin*>(dla_s), rows, Dk, Dv);
    return cudaGetLastError();
}

// Workspace of the reduced-gate calls (each region 256-byte aligned):
//   [gdn2 workspace: gdn2_workspace_size(GDN2_OP_FWD) for a plain forward, else the larger of the
//    GDN2_OP_FWD_SAVE and GDN2_OP_BWD sizes, so that a forward that saves its states and the backward on
//    them find the broadcast gates at the same offsets]
//   [b: rows x Dk][w: rows x Dv][log_alpha: rows x Dk (scalar decay)]
//   backward only: [db: rows x Dk][dw: rows x Dv][dlog_alpha: rows x Dk (scalar decay)]
struct Layout {
    size_t base, b, w, la, db, dw, dla, total;
};
Layout layout(gdn2_gate gate, gdn2_op op, int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt) {
    Layout L{};
    const size_t es = dt == GDN2_BF16 ? 2 : 4;
    const size_t rows = (size_t)B * T * H;
    const bool scalar = gate == GDN2_GATE_GDN;
    if (op == GDN2_OP_FWD) {
        L.base = al256(gdn2_workspace_size(GDN2_OP_FWD, B, T, H, Dk, Dv, chunk, dt));
    } else {
        const size_t save = gdn2_workspace_size(GDN2_OP_FWD_SAVE, B, T, H, Dk, Dv, chunk, dt);
        const size_t bwd = gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt);
        L.base = al256(save > bwd ? save : bwd);
    }
    L.b = L.base;
    L.w = L.b + al256(rows * Dk * es);
    L.la = L.w + al256(rows * Dv * es);
    L.db = L.la + (scalar ? al256(rows * Dk * es) : 0);
    L.dw = L.db + al256(rows * Dk * es);
    L.dla = L.dw + al256(rows * Dv * es);
    L.total = op == GDN2_OP_BWD ? L.dla + (scalar ? al256(rows * Dk * es) : 0) : L.db;
    return L;
}

thread_local char g_err[256];
gdn2_status report(gdn2_status s) {
    set_last_error(g_err);
    return s;
}

}  // namespace
}  // namespace gdn2

using namespace gdn2;

extern "C" {

size_t gdn2_beta_workspace_size(gdn2_gate gate, gdn2_op op, int B, int T, int H, int Dk, int Dv, int chunk,
                                gdn2_dtype dt) {
    if (gate != GDN2_GATE_KDA && gate != GDN2_GATE_GDN) return 0;
    if (gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt) == 0 && T > 0) return 0;
    return layout(gate, op, B, T, H, Dk, Dv, chunk, dt).total;
}

gdn2_status gdn2_beta_fwd(gdn2_gate gate, const void* q, const void* k, const void* v, const void* log_alpha,
                          const void* beta, const float* S0, void* o, float* ST, int B, int T, int H, int Dk, int Dv,
                          int chunk, gdn2_dtype dt, int save_states, void* ws, size_t ws_bytes, void* stream) {
    if (gate != GDN2_GATE_KDA && gate != GDN2_GATE_GDN) {
        snprintf(g_err, sizeof(g_err), "gate=%d is not GDN2_GATE_KDA or GDN2_GATE_GDN", (int)gate);
        return report(GDN2_ERR_INVALID);
    }
    if (T > 0 && (!beta || !log_alpha)) {
        snprintf(g_err, sizeof(g_err), "%s must not be NULL", beta ? "log_alpha" : "beta");
        return report(GDN2_ERR_INVALID);
    }
    const gdn2_op op = save_states ? GDN2_OP_FWD_SAVE : GDN2_OP_FWD;
    const Layout L = layout(gate, op, B, T, H, Dk, Dv, chunk, dt);
    if (T > 0) {
        if (gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt) == 0)   // invalid sizes: let gdn2_fwd say why
            return gdn2_fwd(q, k, v, log_alpha, log_alpha, log_alpha, S0, o, ST, B, T, H, Dk, Dv, chunk, dt,
                            save_states, ws, ws_bytes, stream);
        if (!ws || ws_bytes < L.total || ((uintptr_t)ws & 255)) {
            snprintf(g_err, sizeof(g_err), "gdn2_beta_fwd needs a 256-byte aligned workspace of %zu bytes, got %zu",
                     L.total, ws ? ws_bytes : 0);
            return report(ws && ws_bytes >= L.total ? GDN2_ERR_INVALID : GDN2_ERR_WORKSPACE);
        }
    }
    unsigned char* w8 = static_cast<unsigned char*>(ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool scalar = gate == GDN2_GATE_GDN;
    const bool tc = tc_path(dt, Dk, Dv) && ((uintptr_t)beta & 3) == 0;   // the chunk kernels take beta as it is
    const bool tc_la = tc && scalar && ((uintptr_t)log_alpha & 3) == 0;    // and the scalar decay
    const void* la_full = log_alpha;
    if (T > 0 && (!tc || (scalar && !tc_la))) {
        const long long rows = (long long)B * T * H;
        void* bf = tc ? nullptr : w8 + L.b;
        void* wf = tc ? nullptr : w8 + L.w;
        cudaError_t e = dt == GDN2_BF16
                            ? launch_expand<__nv_bfloat16>(beta, scalar ? log_alpha : nullptr, bf, wf, w8 + L.la, rows,
                                                           Dk, Dv, s)
                            : launch_expand<float>(beta, scalar ? log_alpha : nullptr, bf, wf, w8 + L.la, rows, Dk, Dv,
                                                   s);
        if (e != cudaSuccess) {
            snprintf(g_err, sizeof(g_err), "gdn2_beta_fwd (gate broadcast): %s", cudaGetErrorString(e));
            return report(GDN2_ERR_CUDA);
        }
        if (scalar) la_full = w8 + L.la;
    }
    if (T > 0 && tc)
        return fwd_impl(q, k, v, la_full, beta, beta, S0, o, ST, B, T, H, Dk, Dv, chunk, dt, save_states, ws, L.base,
                        stream, beta, tc_la);
    return gdn2_fwd(q, k, v, la_full, T > 0 ? w8 + L.b : nullptr, T > 0 ? w8 + L.w : nullptr, S0, o, ST, B, T, H,
                    Dk, Dv, chunk, dt, save_states, ws, L.base, stream);
}

gdn2_status gdn2_beta_bwd(gdn2_gate gate, const void* q, const void* k, const void* v, const void* log_alpha,
                          const void* beta, const float* S0, const void* dout, const float* dST, void* dq, void* dk,
                          void* dv, void* dlog_alpha, void* dbeta, float* dS0, int B, int T, int H, int Dk, int Dv,
                          int chunk, gdn2_dtype dt, int states_saved, void* ws, size_t ws_bytes, void* stream) {
    if (gate != GDN2_GATE_KDA && gate != GDN2_GATE_GDN) {
        snprintf(g_err, sizeof(g_err), "gate=%d is not GDN2_GATE_KDA or GDN2_GATE_GDN", (int)gate);
        return report(GDN2_ERR_INVALID);
    }
    const Layout L = layout(gate, GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt);
    if (T > 0) {
        if (!beta || !log_alpha || !dbeta || !dlog_alpha) {
            snprintf(g_err, sizeof(g_err), "beta, log_alpha, dbeta and dlog_alpha must not be NULL");
            return report(GDN2_ERR_INVALID);
        }
        if (gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt) == 0)
            return gdn2_bwd(q, k, v, log_alpha, log_alpha, log_alpha, S0, dout, dST, dq, dk, dv, dlog_alpha, dbeta,
                            dbeta, dS0, B, T, H, Dk, Dv, chunk, dt, states_saved, ws, ws_bytes, stream);
        if (!ws || ws_bytes < L.total || ((uintptr_t)ws & 255)) {
            snprintf(g_err, sizeof(g_err), "gdn2_beta_bwd needs a 256-byte aligned workspace of %zu bytes, got %zu",
                     L.total, ws ? ws_bytes : 0);
            return report(ws && ws_bytes >= L.total ? GDN2_ERR_INVALID : GDN2_ERR_WORKSPACE);
        }
    }
    unsigned char* w8 = static_cast<unsigned char*>(ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool scalar = gate == GDN2_GATE_GDN;
    const bool tc = tc_path(dt, Dk, Dv) && ((uintptr_t)beta & 3) == 0;   // the chunk kernels take beta as it is
    const bool tc_la = tc && scalar && ((uintptr_t)log_alpha & 3) == 0;    // and the scalar decay
    const long long rows = (long long)B * T * H;
    if (T > 0 && (!tc || (scalar && !tc_la))) {   // the broadcast gates
        void* bf = tc ? nullptr : w8 + L.b;
        void* wf = tc ? nullptr : w8 + L.w;
        cudaError_t e = dt == GDN2_BF16
                            ? launch_expand<__nv_bfloat16>(beta, scalar ? log_alpha : nullptr, bf, wf, w8 + L.la, rows,
                                                           Dk, Dv, s)
                            : launch_expand<float>(beta, scalar ? log_alpha : nullptr, bf, wf, w8 + L.la, rows, Dk, Dv,
                                                   s);
        if (e != cudaSuccess) {
            snprintf(g_err, sizeof(g_err), "gdn2_beta_bwd (gate broadcast): %s", cudaGetErrorString(e));
            return report(GDN2_ERR_CUDA);
        }
    }
    void* dla_full = scalar ? static_cast<void*>(w8 + L.dla) : dlog_alpha;
    if (T > 0 && tc) {
        const bool bcast_la = scalar && !tc_la;
        gdn2_status st = bwd_impl(q, k, v, bcast_la ? static_cast<const void*>(w8 + L.la) : log_alpha, beta, beta, S0,
                                  dout, dST, dq, dk, dv, bcast_la ? dla_full : dlog_alpha, dbeta, dbeta, dS0, B, T, H,
                                  Dk, Dv, chunk, dt, states_saved, ws, L.base, stream, beta, dbeta, tc_la);
        if (st != GDN2_OK || !bcast_la) return st;
        cudaError_t e = launch_reduce<__nv_bfloat16>(nullptr, nullptr, w8 + L.dla, dbeta, dlog_alpha, rows, Dk, Dv, s);
        if (e != cudaSuccess) {
            snprintf(g_err, sizeof(g_err), "gdn2_beta_bwd (decay gradient sum): %s", cudaGetErrorString(e));
            return report(GDN2_ERR_CUDA);
        }
        return GDN2_OK;
    }
    gdn2_status st = gdn2_bwd(q, k, v, scalar ? static_cast<const void*>(w8 + L.la) : log_alpha,
                              T > 0 ? w8 + L.b : nullptr, T > 0 ? w8 + L.w : nullptr, S0, dout, dST, dq, dk, dv,
                              T > 0 ? dla_full : dlog_alpha, T > 0 ? w8 + L.db : dbeta, T > 0 ? w8 + L.dw : dbeta,
                              dS0, B, T, H, Dk, Dv, chunk, dt, states_saved, ws, L.base, stream);
    if (st != GDN2_OK || T == 0) return st;
    cudaError_t e = dt == GDN2_BF16
                        ? launch_reduce<__nv_bfloat16>(w8 + L.db, w8 + L.dw, scalar ? w8 + L.dla : nullptr, dbeta,
                                                       scalar ? dlog_alpha : nullptr, rows, Dk, Dv, s)
                        : launch_reduce<float>(w8 + L.db, w8 + L.dw, scalar ? w8 + L.dla : nullptr, dbeta,
                                               scalar ? dlog_alpha : nullptr, rows, Dk, Dv, s);
    if (e != cudaSuccess) {
        snprintf(g_err, sizeof(g_err), "gdn2_beta_bwd (gate sums): %s", cudaGetErrorString(e));
        return report(GDN2_ERR_CUDA);
    }
    return GDN2_OK;
}

}  // extern "C"
