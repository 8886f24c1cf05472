// internal.h -- launch interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace gdn2 {

// fp32 token-recurrent kernels (recurrent.cu).
struct RecurrentArgs {
    enum Op { DECODE, FWD, BWD } op;
    gdn2_dtype dt;
    Dims d;
    const void *q, *k, *v, *la, *b, *w, *dout;
    const float *S0, *dST;
    float* S;            // decode: state in/out
    void* o;             // output (may be null in FWD: states only)
    float *ST, *dS0;
    void *dq, *dk, *dv, *dla, *db, *dw;
    float* states;       // [B,H,NC,Dk,Dv] fp32 chunk-start states (FWD writes if non-null, BWD reads)
    float* seg;          // BWD scratch [B,H,chunk,Dk,Dv]
    float* segdelta;     // BWD scratch [B,H,chunk,Dv]
};
cudaError_t recurrent_launch(const RecurrentArgs& a, cudaStream_t s);

// Tensor-core chunkwise kernels (chunk_fwd.cu, chunk_bwd.cu): bf16, Dk = Dv = 128, chunk = 64.
constexpr int TC_D = 128;
constexpr int TC_C = 64;
// bytes of one saved state image (bf16 128 x 128, 128B-swizzled panels)
constexpr size_t TC_STATE_BYTES = (size_t)TC_D * TC_D * 2;
// One WY image per chunk, written by the forward's producers: bf16 row tiles T [64 x 64], P [64 x 64],
// Wm, Qt, Kt [64 x 128 each], then gC (fp32 [128]), the chunk's untame-channel mask (4 x 32 bits, bit =
// key channel) and padding to a 1 KB multiple, then a Kh = k * exp(G_C - G_t) tile [64 x 128] that is
// written (and read) only for chunks whose mask is not zero.
constexpr size_t TC_WY_T = 0, TC_WY_P = 8192, TC_WY_WM = 16384, TC_WY_QT = 32768, TC_WY_KT = 49152,
                 TC_WY_GC = 65536, TC_WY_MASK = 66048, TC_WY_KH = 66560;
constexpr size_t TC_WY_BYTES = 82944;
// bytes of one saved Delta^T (forward) or dDelta^T (backward) image: bf16 128 x 64 row tile
constexpr size_t TC_DELTA_BYTES = (size_t)TC_D * TC_C * 2;

struct ChunkFwdArgs {
    Dims d;
    const void *q, *k, *v, *la, *b, *w;
    const float* S0;
    void* o;               // may be null: states only
    float* ST;
    unsigned char* states; // [B,H,NC] chunk-start state images, or null
    unsigned char* deltas; // [B,H,NC] Delta^T images (with states), or null
    unsigned char* wy;     // [B,H,NC] WY images (T | P | Wm), always written
    unsigned int* flags;   // [B,H,NC] ready flags (scratch)
    float* sbuf;           // segment states and maps of long sequences (chunk_fwd_split_bytes), or null
    float *map_N, *map_M;  // both set: compute the affine map of each head's sequence instead ([BH][128][128])
    const void* beta;      // [B,T,H] bf16, or null: erase and write gates one scalar per head and token
                           // (b = w = beta 1; b and w are then not read)
    bool scalar_decay;     // with beta: la is [B,T,H] (one decay per head and token, broadcast over Dk)
};
cudaError_t chunk_fwd_launch(const ChunkFwdArgs& a, cudaStream_t s);
cudaError_t chunk_fwd_map_launch(const ChunkFwdArgs& a, cudaStream_t s);   // map_N / map_M of every head
cudaError_t chunk_fwd_wy_launch(const ChunkFwdArgs& a, cudaStream_t s);    // the WY images (and flags) alone
// Long sequences with few heads: a head's chunks may be cut into segments that run on separate CTAs (segment
// maps, a prefix over them, then the segments again from their start states). Workspace for that, 0 if the
// problem never qualifies.
constexpr int TC_SPLIT_MAX_BH = 32;
constexpr int TC_SPLIT_MIN_CHUNKS_PER_SEG = 16;
size_t chunk_fwd_split_bytes(int BH, int nc);
// The segment count for a problem (0: no split), and the fp32 prefix over the segment maps, shared by the
// forward and the backward (whose reverse segments use the same per-head layout of states and maps).
int split_segments_for(int BH, int nc, int slots, bool have_buf);
// Segments of the maps of a piece (gdn2_fwd_map / gdn2_bwd_map), in the same workspace region, slot-major
// ([slot][B*H][128][128]): 0 for none.
int map_segments_for(int BH, int nc, int slots, bool have_buf);
cudaError_t split_prefix_launch(float* sbuf, int R, int BH, cudaStream_t s);
bool split_disabled();   // environment variable GDN2_NO_SPLIT set: keep every head on one chain

struct ChunkBwdArgs {
    Dims d;
    const void *q, *k, *v, *la, *b, *w, *dout;
    const float *dST;
    void *dq, *dk, *dv, *dla, *db, *dw;
    float* dS0;
    const unsigned char* states;  // [B,H,NC] chunk-start state images
    const unsigned char* deltas;  // [B,H,NC] Delta^T images saved by the forward
    const unsigned char* tp;      // [B,H,NC] WY images (T | P | Wm) of every chunk
    unsigned char* dstates;       // [B,H,NC] images of Diag(gC) dL/dS' per chunk (scratch)
    unsigned char* ddeltas;       // [B,H,NC] dDelta^T images (scratch)
    unsigned int* flags;          // [B,H,NC] ready flags, then work counter and abort word (scratch)
    float* sbuf;                  // segment gradients and maps of long sequences (chunk_fwd_split_bytes), or null
    float *map_B, *map_A;         // both set: compute the reverse affine map of each head's sequence instead
    const void* beta;             // [B,T,H] bf16, or null: b = w = beta 1 (b and w are then not read, db and dw
    void* dbeta;                  // not written; dbeta [B,T,H] bf16 = sum_i db_ti + sum_j dw_tj instead)
    bool scalar_decay;            // with beta: la and dla are [B,T,H] (dla_t = sum_i dlog_alpha_ti)
};
cudaError_t chunk_bwd_launch(const ChunkBwdArgs& a, cudaStream_t s);
// gdn2_fwd / gdn2_bwd with one scalar erase and write gate per head and token (beta [B,T,H], dbeta), taken on
// the tensor-core path only (tc_path); b and w must be non-null but are not read there, nor db and dw written.
// scalar_decay (with beta): log_alpha and dlog_alpha are [B,T,H]; beta and log_alpha 4-byte aligned.
gdn2_status fwd_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* b, const void* w,
                     const float* S0, void* o, float* ST, int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt,
                     int save_states, void* ws, size_t ws_bytes, void* stream, const void* beta,
                     bool scalar_decay = false);
gdn2_status bwd_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* b, const void* w,
                     const float* S0, const void* dout, const float* dST, void* dq, void* dk, void* dv,
                     void* dlog_alpha, void* db, void* dw, float* dS0, int B, int T, int H, int Dk, int Dv, int chunk,
                     gdn2_dtype dt, int states_saved, void* ws, size_t ws_bytes, void* stream, const void* beta,
                     void* dbeta, bool scalar_decay = false);
// dst = M src + N per head, fp32 [BH][128][128] operands, in place allowed for src == dst
cudaError_t state_affine_launch(const float* M, const float* N, const float* src, float* dst, int BH, int Dk, int Dv,
                                cudaStream_t s);
cudaError_t state_identity_launch(float* dst, int BH, int Dk, cudaStream_t s);   // dst = I per head [Dk][Dk]

// Gate activations of the layer (layer_gates.cu): z [rows][4 Dk + 2 Dv] -> q, k, v, b, w, log_alpha and back.
cudaError_t gates_fwd_launch(const void* z, void* q, void* k, void* v, void* b, void* w, void* la, const float* abias,
                             long long rows, int H, int Dk, int Dv, gdn2_dtype dt, cudaStream_t s);
cudaError_t gates_bwd_launch(const void* z, const void* dq, const void* dk, const void* dv, const void* db, const void* dw,
                             const void* dla, const float* abias, void* dz, long long rows, int H, int Dk, int Dv,
                             gdn2_dtype dt, cudaStream_t s);

// Kernels of the library, for gdn2_trace_read().
enum KernelId { K_CHUNK_FWD = 0, K_CHUNK_BWD, K_REC_FWD, K_REC_BWD, K_DECODE, K_GATE_EXPAND, K_GATE_REDUCE,
                K_VARLEN_COPY, K_SPLIT_PREFIX, K_STATE_AFFINE, K_LAYER_GATES, K_LAYER_GATES_BWD, KERNEL_COUNT };

// Brackets one kernel launch with CUDA events on its stream while tracing is on.
class TraceScope {
  public:
    TraceScope(KernelId id, cudaStream_t s);
    ~TraceScope();
    TraceScope(const TraceScope&) = delete;
    TraceScope& operator=(const TraceScope&) = delete;

  private:
    KernelId id_;
    cudaStream_t stream_;
    cudaEvent_t start_;
    bool active_;
};

// True when the environment variable GDN2_NO_COOPERATIVE is set: the chunkwise kernels then run
// their producer and consumer work as two ordinary launches instead of one cooperative launch.
bool cooperative_disabled();
bool test_skip_producers();   // host-side fault injection for the forward's two-launch form
// Read and clear the device-side error words of the tensor-core kernels (bit set: a bounded wait gave up).
cudaError_t chunk_fwd_take_errors(unsigned int* bits);
cudaError_t chunk_bwd_take_errors(unsigned int* bits);
cudaError_t varlen_take_errors(unsigned int* bits);   // bit 1: a sequence longer than Tmax; 2: outside [0, Ttot)

// Sets the detail string returned by gdn2_last_error() on this host thread.
void set_last_error(const char* msg);

// Whether the tensor-core kernels handle this problem: bf16 with d_k = d_v = 128. They always run the
// WY algorithm on 64-token chunks; the result does not depend on the chunk length in exact arithmetic,
// so a requested chunk of 16 or 32 is served by the same kernels.
inline bool tc_path(gdn2_dtype dt, int Dk, int Dv) { return dt == GDN2_BF16 && Dk == TC_D && Dv == TC_D; }
// The sizes a call runs with: on the tensor-core path the chunk is the kernels' 64.
inline Dims run_dims(int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt) {
    return Dims{B, T, H, Dk, Dv, tc_path(dt, Dk, Dv) ? TC_C : chunk};
}

}  // namespace gdn2
