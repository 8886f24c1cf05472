// gdn2_api.cu -- the C ABI of libgdn2.so (declared in include/gdn2.h).
//
// Host-side argument checks, workspace layout and dispatch between the
// tensor-core chunkwise kernels (bf16, Dk = Dv = 128, chunk 64) and the fp32
// token-recurrent kernels (everything else). Nothing here allocates memory or
// synchronises; every launch goes to the caller's stream.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "gdn2.h"
#include "internal.h"

using namespace gdn2;

namespace {
// An NVTX range around an entry point (visible in Nsight timelines; free when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace

namespace {

thread_local char g_err[512];

gdn2_status fail(gdn2_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
gdn2_status fail(gdn2_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

gdn2_status cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return GDN2_OK;
    return fail(GDN2_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64; }
bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Checks sizes; returns GDN2_OK or an error status with detail.
gdn2_status check_dims(int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt, bool seq) {
    if (dt != GDN2_F32 && dt != GDN2_BF16) return fail(GDN2_ERR_INVALID, "dtype %d is not GDN2_F32 or GDN2_BF16", (int)dt);
    if (B < 1 || H < 1) return fail(GDN2_ERR_INVALID, "B=%d and H=%d must be >= 1", B, H);
    if (seq && T < 0) return fail(GDN2_ERR_INVALID, "T=%d must be >= 0", T);
    if (!dim_ok(Dk) || !dim_ok(Dv))
        return fail(GDN2_ERR_UNSUPPORTED, "Dk=%d, Dv=%d: each must be 16, 32, 64 or 128", Dk, Dv);
    if (seq && !chunk_ok(chunk)) return fail(GDN2_ERR_UNSUPPORTED, "chunk=%d: must be 16, 32 or 64", chunk);
    // element counts must stay well inside size_t and int grid limits
    const double elems = (double)B * (seq ? (double)T : 1.0) * H * (Dk > Dv ? Dk : Dv);
    if (elems > 4.0e15) return fail(GDN2_ERR_INVALID, "problem too large");
    if ((double)B * H > 2147483647.0) return fail(GDN2_ERR_INVALID, "B*H too large");
    return GDN2_OK;
}

// Tensor-core workspace (units = B*H*NC chunks), each region 256-byte aligned:
//   [states: units x TC_STATE_BYTES][Delta^T: units x TC_DELTA_BYTES]  (training only)
//   [WY images: units x TC_WY_BYTES][ready flags]
//   then, for the backward, [dZ^T: units x TC_STATE_BYTES][dDelta^T: units x TC_DELTA_BYTES][flags].
size_t tc_units(const Dims& d) { return (size_t)d.B * d.H * (size_t)d.nchunks(); }
size_t tc_split_bytes(const Dims& d) { return align256(chunk_fwd_split_bytes(d.B * d.H, d.nchunks())); }
// WY images, ready flags, then the segment states and maps of a long sequence (if it can be cut)
size_t tc_wy_bytes(const Dims& d) {
    return tc_units(d) * TC_WY_BYTES + align256(tc_units(d) * sizeof(unsigned int)) + tc_split_bytes(d);
}

// Forward-saved region: chunk-start states (and, on the tensor-core path, Delta^T, the WY images and flags).
size_t states_bytes(const Dims& d, gdn2_dtype dt) {
    const size_t units = tc_units(d);
    return tc_path(dt, d.Dk, d.Dv) ? units * (TC_STATE_BYTES + TC_DELTA_BYTES) + tc_wy_bytes(d)
                                                  : units * d.Dk * d.Dv * sizeof(float);
}
size_t tc_delta_offset(const Dims& d) { return tc_units(d) * TC_STATE_BYTES; }
size_t tc_tp_offset(const Dims& d) { return tc_units(d) * (TC_STATE_BYTES + TC_DELTA_BYTES); }
size_t tc_flags_offset(const Dims& d, bool with_states) {
    return (with_states ? tc_tp_offset(d) : 0) + tc_units(d) * TC_WY_BYTES;
}
size_t tc_split_offset(const Dims& d, bool with_states) {
    return tc_flags_offset(d, with_states) + align256(tc_units(d) * sizeof(unsigned int));
}

// GDN2_OP_MAP: [WY images][flags, work counter, abort word][segment maps of a long piece]
size_t map_sbuf_offset(const Dims& d) {
    return align256(tc_units(d) * TC_WY_BYTES) + align256((tc_units(d) + 2) * sizeof(unsigned int));
}

size_t bwd_extra_bytes(const Dims& d, gdn2_dtype dt) {
    if (tc_path(dt, d.Dk, d.Dv))   // dZ and dDelta images, ready flags, work counter, abort word
        return tc_units(d) * (TC_STATE_BYTES + TC_DELTA_BYTES) + align256((tc_units(d) + 2) * sizeof(unsigned int));
    const size_t seg = (size_t)d.B * d.H * d.chunk * d.Dk * d.Dv * sizeof(float);
    const size_t del = (size_t)d.B * d.H * d.chunk * d.Dv * sizeof(float);
    return align256(seg) + align256(del);
}

#define REQUIRE_PTR(p)                                                                      \
    do {                                                                                    \
        if (!(p)) return fail(GDN2_ERR_INVALID, "%s must not be NULL", #p);                 \
        if (!aligned((p), 16)) return fail(GDN2_ERR_INVALID, "%s must be 16-byte aligned", #p); \
    } while (0)
#define OPTIONAL_PTR(p)                                                                     \
    do {                                                                                    \
        if ((p) && !aligned((p), 16)) return fail(GDN2_ERR_INVALID, "%s must be 16-byte aligned", #p); \
    } while (0)

// T == 0: the final state is the initial state and no token work exists.
gdn2_status copy_or_zero_state(float* dst, const float* src, const Dims& d, cudaStream_t s) {
    if (!dst || dst == src) return GDN2_OK;
    const size_t bytes = (size_t)d.B * d.H * d.Dk * d.Dv * sizeof(float);
    cudaError_t e = src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(dst, 0, bytes, s);
    return cuda_status(e, "state copy");
}

}  // namespace

namespace gdn2 {
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
static bool env_flag(const char* name) {
    const char* v = getenv(name);
    return v && v[0] && !(v[0] == '0' && v[1] == 0);
}
bool cooperative_disabled() { return env_flag("GDN2_NO_COOPERATIVE"); }
bool test_skip_producers() { return env_flag("GDN2_TEST_SKIP_PRODUCERS"); }
bool split_disabled() { return env_flag("GDN2_NO_SPLIT"); }
}  // namespace gdn2

extern "C" {

int gdn2_version(void) { return 100; }

const char* gdn2_status_string(gdn2_status s) {
    switch (s) {
    case GDN2_OK: return "GDN2_OK";
    case GDN2_ERR_INVALID: return "GDN2_ERR_INVALID: invalid argument";
    case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED: shape or dtype not supported";
    case GDN2_ERR_WORKSPACE: return "GDN2_ERR_WORKSPACE: workspace missing or too small";
    case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA: CUDA runtime error";
    case GDN2_ERR_TIMEOUT: return "GDN2_ERR_TIMEOUT: device-side wait gave up";
    }
    return "unknown gdn2_status";
}

const char* gdn2_last_error(void) { return g_err; }

gdn2_status gdn2_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "gdn2_device_status (stream)");
    unsigned int fwd = 0, bwd = 0;
    if ((e = chunk_fwd_take_errors(&fwd)) != cudaSuccess) return cuda_status(e, "gdn2_device_status (forward record)");
    if ((e = chunk_bwd_take_errors(&bwd)) != cudaSuccess) return cuda_status(e, "gdn2_device_status (backward record)");
    unsigned int vl = 0;
    if ((e = varlen_take_errors(&vl)) != cudaSuccess) return cuda_status(e, "gdn2_device_status (varlen record)");
    if (vl)
        return fail(GDN2_ERR_INVALID, "cu_seqlens: %s%s", (vl & 1u) ? "a sequence was longer than Tmax (cut) " : "",
                    (vl & 2u) ? "a sequence lay outside [0, Ttot) or had a negative length (dropped)" : "");
    if ((fwd | bwd) & GDN2_DBG_BIT)
        return fail(GDN2_ERR_INVALID,
                    "index check failed (debug build; the accesses it guarded were skipped): chunk_fwd_kernel bits "
                    "0x%x, chunk_bwd_kernel bits 0x%x",
                    fwd, bwd);
    if (fwd | bwd)
        return fail(GDN2_ERR_TIMEOUT,
                    "device wait gave up: chunk_fwd_kernel bits 0x%x, chunk_bwd_kernel bits 0x%x "
                    "(1 MMA completion, 2 tile loads, 4 forward ready flag / gradient unit, 8 backward ready flag, "
                    "16 launched with a block size the kernel is not built for)",
                    fwd, bwd);
    return GDN2_OK;
}

size_t gdn2_workspace_size(gdn2_op op, int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt) {
    if (check_dims(B, T, H, Dk, Dv, chunk, dt, true) != GDN2_OK) return 0;
    const Dims d = run_dims(B, T, H, Dk, Dv, chunk, dt);
    switch (op) {
    case GDN2_OP_FWD: return tc_path(dt, Dk, Dv) ? align256(tc_wy_bytes(d)) : 0;
    case GDN2_OP_FWD_SAVE: return align256(states_bytes(d, dt));
    case GDN2_OP_BWD: return align256(states_bytes(d, dt)) + align256(bwd_extra_bytes(d, dt));
    case GDN2_OP_MAP:   // WY images, ready flags with the backward's work counter and abort word, segment maps
        return tc_path(dt, Dk, Dv) ? map_sbuf_offset(d) + tc_split_bytes(d) : 0;
    }
    return 0;
}

}  // extern "C"

namespace gdn2 {

gdn2_status fwd_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                     const void* w, const float* S0, void* o, float* ST, int B, int T, int H, int Dk,
                     int Dv, int chunk, gdn2_dtype dt, int save_states, void* ws, size_t ws_bytes,
                     void* stream, const void* beta, bool scalar_decay) {
    NvtxRange nvtx("gdn2_fwd");
    gdn2_status st = check_dims(B, T, H, Dk, Dv, chunk, dt, true);
    if (st != GDN2_OK) return st;
    const Dims d = run_dims(B, T, H, Dk, Dv, chunk, dt);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    OPTIONAL_PTR(S0);
    OPTIONAL_PTR(ST);
    if (T == 0) return copy_or_zero_state(ST, S0, d, s);
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(log_alpha);
    REQUIRE_PTR(b); REQUIRE_PTR(w); REQUIRE_PTR(o);
    {
        const size_t need = gdn2_workspace_size(save_states ? GDN2_OP_FWD_SAVE : GDN2_OP_FWD, B, T, H, Dk, Dv, chunk, dt);
        if (need && (!ws || ws_bytes < need))
            return fail(GDN2_ERR_WORKSPACE, "gdn2_fwd%s needs %zu workspace bytes, got %zu",
                        save_states ? " with save_states" : "", need, ws ? ws_bytes : 0);
        if (need && !aligned(ws, 256)) return fail(GDN2_ERR_INVALID, "ws must be 256-byte aligned");
    }
    if (tc_path(dt, Dk, Dv)) {
        ChunkFwdArgs a{};
        a.d = d;
        a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w;
        a.beta = beta;
        a.scalar_decay = beta != nullptr && scalar_decay;
        a.S0 = S0; a.o = o; a.ST = ST;
        unsigned char* wsb = static_cast<unsigned char*>(ws);
        const bool keep = save_states != 0;
        a.states = keep ? wsb : nullptr;
        a.deltas = keep ? wsb + tc_delta_offset(d) : nullptr;
        a.wy = wsb + (keep ? tc_tp_offset(d) : 0);
        a.flags = reinterpret_cast<unsigned int*>(wsb + tc_flags_offset(d, keep));
        a.sbuf = tc_split_bytes(d) ? reinterpret_cast<float*>(wsb + tc_split_offset(d, keep)) : nullptr;
        return cuda_status(chunk_fwd_launch(a, s), "gdn2_fwd (tensor-core path)");
    }
    RecurrentArgs a{};
    a.op = RecurrentArgs::FWD;
    a.dt = dt;
    a.d = d;
    a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w;
    a.S0 = S0; a.o = o; a.ST = ST;
    a.states = save_states ? static_cast<float*>(ws) : nullptr;
    return cuda_status(recurrent_launch(a, s), "gdn2_fwd (recurrent path)");
}

gdn2_status bwd_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                     const void* w, const float* S0, const void* dout, const float* dST, void* dq,
                     void* dk, void* dv, void* dlog_alpha, void* db, void* dw, float* dS0, int B, int T,
                     int H, int Dk, int Dv, int chunk, gdn2_dtype dt, int states_saved, void* ws,
                     size_t ws_bytes, void* stream, const void* beta, void* dbeta, bool scalar_decay) {
    NvtxRange nvtx("gdn2_bwd");
    gdn2_status st = check_dims(B, T, H, Dk, Dv, chunk, dt, true);
    if (st != GDN2_OK) return st;
    const Dims d = run_dims(B, T, H, Dk, Dv, chunk, dt);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    OPTIONAL_PTR(S0);
    OPTIONAL_PTR(dST);
    OPTIONAL_PTR(dS0);
    if (T == 0) return copy_or_zero_state(dS0, dST, d, s);
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(log_alpha);
    REQUIRE_PTR(b); REQUIRE_PTR(w); REQUIRE_PTR(dout);
    REQUIRE_PTR(dq); REQUIRE_PTR(dk); REQUIRE_PTR(dv); REQUIRE_PTR(dlog_alpha);
    REQUIRE_PTR(db); REQUIRE_PTR(dw);
    const size_t need = gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt);
    if (!ws || ws_bytes < need)
        return fail(GDN2_ERR_WORKSPACE, "gdn2_bwd needs %zu workspace bytes, got %zu", need, ws ? ws_bytes : 0);
    if (!aligned(ws, 256)) return fail(GDN2_ERR_INVALID, "ws must be 256-byte aligned");
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    unsigned char* extra = wsb + align256(states_bytes(d, dt));

    if (tc_path(dt, Dk, Dv)) {
        if (!states_saved) {
            ChunkFwdArgs f{};
            f.d = d;
            f.q = q; f.k = k; f.v = v; f.la = log_alpha; f.b = b; f.w = w;
            f.beta = beta;
            f.scalar_decay = beta != nullptr && scalar_decay;
            f.S0 = S0; f.o = nullptr; f.ST = nullptr; f.states = wsb; f.deltas = wsb + tc_delta_offset(d);
            f.wy = wsb + tc_tp_offset(d);
            f.flags = reinterpret_cast<unsigned int*>(wsb + tc_flags_offset(d, true));
            f.sbuf = tc_split_bytes(d) ? reinterpret_cast<float*>(wsb + tc_split_offset(d, true)) : nullptr;
            gdn2_status e = cuda_status(chunk_fwd_launch(f, s), "gdn2_bwd state recompute");
            if (e != GDN2_OK) return e;
        }
        ChunkBwdArgs a{};
        a.d = d;
        a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w; a.dout = dout;
        a.dST = dST;
        a.dq = dq; a.dk = dk; a.dv = dv; a.dla = dlog_alpha; a.db = db; a.dw = dw; a.dS0 = dS0;
        a.beta = beta; a.dbeta = dbeta;
        a.scalar_decay = beta != nullptr && scalar_decay;
        a.states = wsb;
        a.tp = wsb + tc_tp_offset(d);
        a.deltas = wsb + tc_delta_offset(d);
        a.dstates = extra;
        a.ddeltas = extra + tc_units(d) * TC_STATE_BYTES;
        a.flags = reinterpret_cast<unsigned int*>(extra + tc_units(d) * (TC_STATE_BYTES + TC_DELTA_BYTES));
        // the forward's segment region (dead once the forward is done) serves the backward's segments
        a.sbuf = tc_split_bytes(d) ? reinterpret_cast<float*>(wsb + tc_split_offset(d, true)) : nullptr;
        return cuda_status(chunk_bwd_launch(a, s), "gdn2_bwd (tensor-core path)");
    }

    RecurrentArgs a{};
    a.dt = dt;
    a.d = d;
    a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w;
    a.S0 = S0;
    a.states = reinterpret_cast<float*>(wsb);
    if (!states_saved) {
        a.op = RecurrentArgs::FWD;
        a.o = nullptr;
        a.ST = nullptr;
        gdn2_status e = cuda_status(recurrent_launch(a, s), "gdn2_bwd state recompute");
        if (e != GDN2_OK) return e;
    }
    a.op = RecurrentArgs::BWD;
    a.dout = dout; a.dST = dST;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dla = dlog_alpha; a.db = db; a.dw = dw; a.dS0 = dS0;
    const size_t seg = (size_t)B * H * d.chunk * Dk * Dv * sizeof(float);
    a.seg = reinterpret_cast<float*>(extra);
    a.segdelta = reinterpret_cast<float*>(extra + align256(seg));
    return cuda_status(recurrent_launch(a, s), "gdn2_bwd (recurrent path)");
}

}  // namespace gdn2

extern "C" {

gdn2_status gdn2_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                     const void* w, const float* S0, void* o, float* ST, int B, int T, int H, int Dk,
                     int Dv, int chunk, gdn2_dtype dt, int save_states, void* ws, size_t ws_bytes,
                     void* stream) {
    return fwd_impl(q, k, v, log_alpha, b, w, S0, o, ST, B, T, H, Dk, Dv, chunk, dt, save_states, ws, ws_bytes,
                    stream, nullptr);
}

gdn2_status gdn2_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                     const void* w, const float* S0, const void* dout, const float* dST, void* dq,
                     void* dk, void* dv, void* dlog_alpha, void* db, void* dw, float* dS0, int B, int T,
                     int H, int Dk, int Dv, int chunk, gdn2_dtype dt, int states_saved, void* ws,
                     size_t ws_bytes, void* stream) {
    return bwd_impl(q, k, v, log_alpha, b, w, S0, dout, dST, dq, dk, dv, dlog_alpha, db, dw, dS0, B, T, H, Dk, Dv,
                    chunk, dt, states_saved, ws, ws_bytes, stream, nullptr, nullptr);
}

// Shared checks of gdn2_fwd_map / gdn2_bwd_map; T == 0 writes the maps of an empty piece.
static gdn2_status map_prologue(const char* name, const void* q, const void* k, const void* v, const void* la,
                                const void* b, const void* w, const void* dout, bool need_dout, float* Mx, float* Nx,
                                int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt, void* ws, size_t ws_bytes,
                                cudaStream_t s, bool* done) {
    *done = false;
    gdn2_status st = check_dims(B, T, H, Dk, Dv, chunk, dt, true);
    if (st != GDN2_OK) return st;
    if (!tc_path(dt, Dk, Dv))
        return fail(GDN2_ERR_UNSUPPORTED, "%s: maps are computed on the tensor-core path only (bf16, Dk = Dv = 128)", name);
    if (!Mx || !aligned(Mx, 16) || !Nx || !aligned(Nx, 16))
        return fail(GDN2_ERR_INVALID, "%s: both map outputs must be non-NULL and 16-byte aligned", name);
    const Dims d = run_dims(B, T, H, Dk, Dv, chunk, dt);
    if (T == 0) {
        *done = true;
        cudaError_t e = state_identity_launch(Mx, B * H, Dk, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(Nx, 0, (size_t)B * H * Dk * Dv * sizeof(float), s);
        return cuda_status(e, name);
    }
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(la); REQUIRE_PTR(b); REQUIRE_PTR(w);
    if (need_dout) REQUIRE_PTR(dout);
    const size_t need = gdn2_workspace_size(GDN2_OP_MAP, B, T, H, Dk, Dv, chunk, dt);
    if (!ws || ws_bytes < need) return fail(GDN2_ERR_WORKSPACE, "%s needs %zu workspace bytes, got %zu", name, need, ws ? ws_bytes : 0);
    if (!aligned(ws, 256)) return fail(GDN2_ERR_INVALID, "ws must be 256-byte aligned");
    (void)d;
    return GDN2_OK;
}

gdn2_status gdn2_fwd_map(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                         const void* w, float* M, float* N, int B, int T, int H, int Dk, int Dv, int chunk,
                         gdn2_dtype dt, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx("gdn2_fwd_map");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    bool done = false;
    gdn2_status st = map_prologue("gdn2_fwd_map", q, k, v, log_alpha, b, w, nullptr, false, M, N, B, T, H, Dk, Dv,
                                  chunk, dt, ws, ws_bytes, s, &done);
    if (st != GDN2_OK || done) return st;
    const Dims d = run_dims(B, T, H, Dk, Dv, chunk, dt);
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    ChunkFwdArgs a{};
    a.d = d;
    a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w;
    a.wy = wsb;
    a.flags = reinterpret_cast<unsigned int*>(wsb + align256(tc_units(d) * TC_WY_BYTES));
    a.sbuf = tc_split_bytes(d) ? reinterpret_cast<float*>(wsb + map_sbuf_offset(d)) : nullptr;
    a.map_N = N; a.map_M = M;
    return cuda_status(chunk_fwd_launch(a, s), "gdn2_fwd_map");
}

gdn2_status gdn2_bwd_map(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                         const void* w, const void* dout, float* A, float* Bm, int B, int T, int H, int Dk,
                         int Dv, int chunk, gdn2_dtype dt, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx("gdn2_bwd_map");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    bool done = false;
    gdn2_status st = map_prologue("gdn2_bwd_map", q, k, v, log_alpha, b, w, dout, true, A, Bm, B, T, H, Dk, Dv,
                                  chunk, dt, ws, ws_bytes, s, &done);
    if (st != GDN2_OK || done) return st;
    const Dims d = run_dims(B, T, H, Dk, Dv, chunk, dt);
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    unsigned int* flags = reinterpret_cast<unsigned int*>(wsb + align256(tc_units(d) * TC_WY_BYTES));
    // the WY images of the piece (the forward's producers alone), then the reverse pass twice per head
    ChunkFwdArgs f{};
    f.d = d;
    f.q = q; f.k = k; f.v = v; f.la = log_alpha; f.b = b; f.w = w;
    f.wy = wsb; f.flags = flags;
    cudaError_t e = chunk_fwd_wy_launch(f, s);
    if (e != cudaSuccess) return cuda_status(e, "gdn2_bwd_map (WY images)");
    ChunkBwdArgs a{};
    a.d = d;
    a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w; a.dout = dout;
    a.tp = wsb; a.flags = flags;
    a.sbuf = tc_split_bytes(d) ? reinterpret_cast<float*>(wsb + map_sbuf_offset(d)) : nullptr;
    a.map_A = A; a.map_B = Bm;
    return cuda_status(chunk_bwd_launch(a, s), "gdn2_bwd_map");
}

gdn2_status gdn2_state_affine(const float* M, const float* N, const float* S_in, float* S_out, int B, int H, int Dk,
                              int Dv, void* stream) {
    NvtxRange nvtx("gdn2_state_affine");
    gdn2_status st = check_dims(B, 1, H, Dk, Dv, 64, GDN2_F32, false);
    if (st != GDN2_OK) return st;
    REQUIRE_PTR(M); REQUIRE_PTR(S_out);
    OPTIONAL_PTR(N); OPTIONAL_PTR(S_in);
    if ((const float*)S_out == M) return fail(GDN2_ERR_INVALID, "S_out must not alias M");
    return cuda_status(state_affine_launch(M, N, S_in, S_out, B * H, Dk, Dv, static_cast<cudaStream_t>(stream)),
                       "gdn2_state_affine");
}

gdn2_status gdn2_layer_gates_fwd(const void* z, const float* a_bias, void* q, void* k, void* v, void* b, void* w,
                                 void* log_alpha, int B, int T, int H, int Dk, int Dv, gdn2_dtype dt, void* stream) {
    NvtxRange nvtx("gdn2_layer_gates_fwd");
    gdn2_status st = check_dims(B, T, H, Dk, Dv, 64, dt, true);
    if (st != GDN2_OK) return st;
    if (T == 0) return GDN2_OK;
    REQUIRE_PTR(z); REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(b); REQUIRE_PTR(w);
    REQUIRE_PTR(log_alpha); OPTIONAL_PTR(a_bias);
    return cuda_status(gates_fwd_launch(z, q, k, v, b, w, log_alpha, a_bias, (long long)B * T * H, H, Dk, Dv, dt,
                                        static_cast<cudaStream_t>(stream)),
                       "gdn2_layer_gates_fwd");
}

gdn2_status gdn2_layer_gates_bwd(const void* z, const float* a_bias, const void* dq, const void* dk, const void* dv,
                                 const void* db, const void* dw, const void* dlog_alpha, void* dz, int B, int T, int H,
                                 int Dk, int Dv, gdn2_dtype dt, void* stream) {
    NvtxRange nvtx("gdn2_layer_gates_bwd");
    gdn2_status st = check_dims(B, T, H, Dk, Dv, 64, dt, true);
    if (st != GDN2_OK) return st;
    if (T == 0) return GDN2_OK;
    REQUIRE_PTR(z); REQUIRE_PTR(dq); REQUIRE_PTR(dk); REQUIRE_PTR(dv); REQUIRE_PTR(db); REQUIRE_PTR(dw);
    REQUIRE_PTR(dlog_alpha); REQUIRE_PTR(dz); OPTIONAL_PTR(a_bias);
    return cuda_status(gates_bwd_launch(z, dq, dk, dv, db, dw, dlog_alpha, a_bias, dz, (long long)B * T * H, H, Dk, Dv, dt,
                                        static_cast<cudaStream_t>(stream)),
                       "gdn2_layer_gates_bwd");
}

gdn2_status gdn2_decode_step(const void* q, const void* k, const void* v, const void* log_alpha,
                             const void* b, const void* w, float* S, void* o, int B, int H, int Dk,
                             int Dv, gdn2_dtype dt, void* stream) {
    NvtxRange nvtx("gdn2_decode_step");
    gdn2_status st = check_dims(B, 1, H, Dk, Dv, 64, dt, false);
    if (st != GDN2_OK) return st;
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(log_alpha);
    REQUIRE_PTR(b); REQUIRE_PTR(w); REQUIRE_PTR(S); REQUIRE_PTR(o);
    RecurrentArgs a{};
    a.op = RecurrentArgs::DECODE;
    a.dt = dt;
    a.d = Dims{B, 1, H, Dk, Dv, 64};
    a.q = q; a.k = k; a.v = v; a.la = log_alpha; a.b = b; a.w = w;
    a.S = S; a.o = o;
    return cuda_status(recurrent_launch(a, static_cast<cudaStream_t>(stream)), "gdn2_decode_step");
}

}  // extern "C"
