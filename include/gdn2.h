/*
 * gdn2.h -- C ABI of libgdn2.so: the Gated Delta Rule-2 sequence-mixing
 * operator of Gated DeltaNet-2 on NVIDIA B200 (sm_100a).
 *
 * The operator ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
 * Attention"; GitHub README method bullets and arXiv abstract 2605.22791): per
 * batch element and head, a d_k x d_v state S evolves with a channel-wise decay
 * alpha_t, a channel-wise erase gate b_t in [0,1]^{d_k} acting on the key side
 * of the decayed state and a channel-wise write gate w_t in [0,1]^{d_v} acting
 * on the value side of the new content:
 *
 *     S_t = (I - k_t (b_t*k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t*v_t)^T
 *     o_t = S_t^T q_t
 *
 * ('*' is the elementwise product; alpha_t = exp(log_alpha_t)). The README's
 * "Hardware-efficient Training" bullet and the abstract name the method of
 * computation: a chunkwise WY algorithm with the channel-wise decay absorbed
 * into asymmetric erase factors, and a gate-aware backward.
 *
 * Conventions for every call below
 *   - Pointers are DEVICE pointers to contiguous row-major tensors, unless a
 *     comment says otherwise. Token tensors are [B, T, H, D]; single-token
 *     (decode) tensors are [B, H, D]; states are [B, H, Dk, Dv] float32 with
 *     rows indexing keys and columns indexing values.
 *   - dt is the element type of q, k, v, log_alpha, b, w, o, dout and of the
 *     token gradients dq, dk, dv, dlog_alpha, db, dw. States and their
 *     gradients are always float32.
 *   - stream is a cudaStream_t (NULL: the legacy default stream). All work is
 *     enqueued on it; no call allocates memory, and none but
 *     gdn2_device_status synchronises the host.
 *   - The caller owns every buffer, including the workspace.
 *   - Arguments are checked on the host before anything is launched. On an
 *     error status nothing has been launched and no output was touched, except
 *     GDN2_ERR_CUDA, which reports a launch failure or an earlier asynchronous
 *     error of the device (outputs are then undefined).
 *   - Gate values are not range-checked (that would cost a pass over HBM).
 *   - log_alpha is a log-decay (alpha in (0, 1]); any value <= 0 is handled,
 *     however strong. On the tensor-core path a channel whose log-decay over
 *     a 64-token chunk exceeds 60 is left out of that chunk's tensor-core
 *     products and its terms are summed exactly on CUDA cores instead (same
 *     results, slower: such chunks cost several times a typical one).
 *     Positive log_alpha (growth) is accepted as long as the cumulative sum
 *     inside a chunk stays below about +60; beyond that the tensor-core path
 *     overflows (the recurrent kernels have no such limit).
 *   - Supported sizes: Dk, Dv in {16, 32, 64, 128}; chunk in {16, 32, 64};
 *     any T >= 0 (a ragged last chunk is allowed); B, H >= 1.
 *     The tensor-core path runs for dt = GDN2_BF16, Dk = Dv = 128, with any
 *     chunk argument: its kernels always use 64-token chunks (the chunkwise
 *     algorithm is exact, so the chunk length does not change the result).
 *     Every other supported combination runs on the fp32 recurrent kernels,
 *     where chunk is the spacing of the state checkpoints of the backward.
 *   - Thread safety: calls may be made from several host threads; error
 *     detail strings are per thread.
 *   - Launches: on the tensor-core path the forward and the backward each run
 *     as one cooperative launch when the device allows it (the per-head chain
 *     and the per-chunk work share the SMs and hand chunks over through ready
 *     flags in the workspace), else as two ordinary launches with the same
 *     results. Setting the environment variable GDN2_NO_COOPERATIVE (to any
 *     value but "0") selects the two-launch form, e.g. for tools that do not
 *     support cooperative launches. GDN2_TEST_SKIP_PRODUCERS (same rule) is a
 *     test hook of the forward's two-launch form: the producer launch is left
 *     out, so the consumers' ready-flag waits run out and gdn2_device_status
 *     reports GDN2_ERR_TIMEOUT; outputs are then not valid.
 *     With few heads (B*H <= 32) and long sequences (at least 64 chunks) each
 *     head's chunks are cut into 4 to 8 segments that run on separate CTAs
 *     (the segments' affine state maps, a prefix over them, then the segments
 *     from their start states): more launches per call, the same results up
 *     to rounding. GDN2_NO_SPLIT (same rule) keeps one chain per head.
 *   - A debug build of the library (libgdn2_debug.so, compiled with
 *     -DGDN2_DEBUG) checks the kernels' task, segment and unit indexes; a
 *     failed check skips the access and gdn2_device_status reports it as
 *     GDN2_ERR_INVALID ("index check"). The release build has no such checks.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn2_status {
    GDN2_OK = 0,
    GDN2_ERR_INVALID = 1,     /* null pointer, bad size or option; nothing launched */
    GDN2_ERR_UNSUPPORTED = 2, /* valid but not built for this shape/dtype; nothing launched */
    GDN2_ERR_WORKSPACE = 3,   /* workspace missing or too small; nothing launched */
    GDN2_ERR_CUDA = 4,        /* CUDA runtime error (see gdn2_last_error) */
    GDN2_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (reported by gdn2_device_status) */
} gdn2_status;

typedef enum gdn2_dtype {
    GDN2_F32 = 0,
    GDN2_BF16 = 1
} gdn2_dtype;

typedef enum gdn2_op {
    GDN2_OP_FWD = 0,      /* gdn2_fwd with save_states = 0 */
    GDN2_OP_FWD_SAVE = 1, /* gdn2_fwd with save_states = 1 */
    GDN2_OP_BWD = 2,      /* gdn2_bwd (either value of states_saved) */
    GDN2_OP_MAP = 3       /* gdn2_fwd_map and gdn2_bwd_map */
} gdn2_op;

/*
 * Bytes of device workspace that gdn2_fwd / gdn2_bwd need for one problem.
 * The workspace of GDN2_OP_BWD starts with the region that GDN2_OP_FWD_SAVE
 * fills, so one buffer of gdn2_workspace_size(GDN2_OP_BWD, ...) bytes serves a
 * gdn2_fwd(save_states = 1) followed by a gdn2_bwd(states_saved = 1).
 * GDN2_OP_FWD needs a workspace only on the tensor-core path (dt = GDN2_BF16,
 * Dk = Dv = 128): there the forward keeps, per chunk, the image of the WY step
 * (the T, P and Wm tiles, the scaled query and key tiles, the chunk's decay and
 * its strongly decaying channels) and a ready flag that hands it from the CTAs
 * that compute it to the CTAs that walk the chunks of a head.
 * Returns 0 for an invalid or unsupported problem and for a forward that needs
 * no workspace. The workspace must be 256-byte aligned; its contents on entry
 * do not matter. On the tensor-core path it is about 81 KB per 64-token
 * chunk and head for GDN2_OP_FWD and GDN2_OP_MAP, 129 KB for GDN2_OP_FWD_SAVE
 * and 177 KB for GDN2_OP_BWD; with B*H <= 32 and at least 32 chunks, 1.2 MB
 * per head is added for the segment states and maps of long sequences.
 */
size_t gdn2_workspace_size(gdn2_op op, int B, int T, int H, int Dk, int Dv, int chunk,
                           gdn2_dtype dt);

/*
 * Forward over whole sequences.
 *   q, k, log_alpha, b : [B, T, H, Dk] dt      (query, key, log-decay, erase gate)
 *   v, w               : [B, T, H, Dv] dt      (value, write gate)
 *   S0                 : [B, H, Dk, Dv] float32, or NULL for a zero initial state
 *   o                  : [B, T, H, Dv] dt       output, o_t = S_t^T q_t
 *   ST                 : [B, H, Dk, Dv] float32 final state, or NULL
 *   chunk              : chunk length of the WY algorithm (16, 32 or 64)
 *   save_states        : nonzero -> keep the chunk-start states in ws for a
 *                        later gdn2_bwd(states_saved = 1) on the same inputs
 *   ws, ws_bytes       : workspace of >= gdn2_workspace_size(GDN2_OP_FWD, or
 *                        GDN2_OP_FWD_SAVE when save_states) bytes; may be NULL
 *                        when that size is 0
 * S0 and ST may alias (the state is updated in place).
 */
gdn2_status gdn2_fwd(const void* q, const void* k, const void* v, const void* log_alpha,
                     const void* b, const void* w, const float* S0, void* o, float* ST,
                     int B, int T, int H, int Dk, int Dv, int chunk, gdn2_dtype dt,
                     int save_states, void* ws, size_t ws_bytes, void* stream);

/*
 * Gate-aware backward of gdn2_fwd for the loss L = <dout, o> + <dST, S_T>.
 *   q .. w, S0         : the forward's inputs (S0 may be NULL: zeros)
 *   dout               : [B, T, H, Dv] dt, gradient of o
 *   dST                : [B, H, Dk, Dv] float32 gradient of S_T, or NULL (zero)
 *   dq, dk, dlog_alpha, db : [B, T, H, Dk] dt   (outputs)
 *   dv, dw             : [B, T, H, Dv] dt       (outputs)
 *   dS0                : [B, H, Dk, Dv] float32 gradient of S0, or NULL
 *   states_saved       : nonzero -> ws holds the chunk-start states written by
 *                        gdn2_fwd(save_states = 1) with the same inputs, S0,
 *                        sizes and chunk; zero -> they are recomputed here
 *   ws, ws_bytes       : >= gdn2_workspace_size(GDN2_OP_BWD, ...) bytes
 * All six token gradients must be given; they must not alias the inputs.
 */
gdn2_status gdn2_bwd(const void* q, const void* k, const void* v, const void* log_alpha,
                     const void* b, const void* w, const float* S0, const void* dout,
                     const float* dST, void* dq, void* dk, void* dv, void* dlog_alpha, void* db,
                     void* dw, float* dS0, int B, int T, int H, int Dk, int Dv, int chunk,
                     gdn2_dtype dt, int states_saved, void* ws, size_t ws_bytes, void* stream);

/*
 * One recurrent decode step for every (b, h), state updated in place -- the
 * constant-memory decoding of the arXiv abstract.
 *   q, k, log_alpha, b : [B, H, Dk] dt ;  v, w : [B, H, Dv] dt
 *   S                  : [B, H, Dk, Dv] float32, read and overwritten with S_t
 *   o                  : [B, H, Dv] dt, o = S_t^T q
 */
gdn2_status gdn2_decode_step(const void* q, const void* k, const void* v, const void* log_alpha,
                             const void* b, const void* w, float* S, void* o, int B, int H,
                             int Dk, int Dv, gdn2_dtype dt, void* stream);

/*
 * The two recurrences that the operator generalises, run through the same
 * kernels (README "Strict Generalization" bullet, arXiv abstract). With the
 * erase and write gates one scalar beta_t per head and token, b_t = w_t =
 * beta_t 1, the operator is KDA,
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 * and with the decay also one scalar per head and token it is Gated DeltaNet
 * (published with the state transposed, d_v x d_k; here the state keeps the
 * [B, H, Dk, Dv] layout of gdn2_fwd, the transpose of the published one).
 *   gate       GDN2_GATE_KDA: log_alpha [B, T, H, Dk] (channel-wise decay)
 *              GDN2_GATE_GDN: log_alpha [B, T, H]     (one decay per head and token)
 *   beta       [B, T, H] dt
 *   dbeta      [B, T, H] dt (output of the backward); for GDN2_GATE_GDN dlog_alpha
 *              is [B, T, H], else [B, T, H, Dk]
 * Everything else as gdn2_fwd / gdn2_bwd, including the chunk and the paths
 * taken. On the tensor-core path (bf16, Dk = Dv = 128) with beta 4-byte
 * aligned, the chunk kernels' scalar-gate instances read beta per token and
 * the backward sums dbeta_t = sum_i db_ti + sum_j dw_tj itself, and likewise
 * a scalar decay (GDN2_GATE_GDN, log_alpha 4-byte aligned): dlog_a_t =
 * sum_i dlog_alpha_ti. Otherwise the reduced gates are broadcast into the
 * workspace, gdn2_fwd / gdn2_bwd run on them and their gradients are summed
 * back (each call broadcasts what it needs).
 * Workspace: gdn2_beta_workspace_size(gate, op, ...) bytes, 256-byte aligned;
 * one buffer of the GDN2_OP_BWD size serves gdn2_beta_fwd(save_states = 1)
 * followed by gdn2_beta_bwd(states_saved = 1). Returns 0 for an invalid gate
 * or problem.
 */
typedef enum gdn2_gate {
    GDN2_GATE_KDA = 1,   /* beta per head and token, channel-wise decay */
    GDN2_GATE_GDN = 2    /* beta and the decay per head and token */
} gdn2_gate;
size_t gdn2_beta_workspace_size(gdn2_gate gate, gdn2_op op, int B, int T, int H, int Dk, int Dv, int chunk,
                                gdn2_dtype dt);
gdn2_status gdn2_beta_fwd(gdn2_gate gate, const void* q, const void* k, const void* v, const void* log_alpha,
                          const void* beta, const float* S0, void* o, float* ST, int B, int T, int H, int Dk,
                          int Dv, int chunk, gdn2_dtype dt, int save_states, void* ws, size_t ws_bytes,
                          void* stream);
gdn2_status gdn2_beta_bwd(gdn2_gate gate, const void* q, const void* k, const void* v, const void* log_alpha,
                          const void* beta, const float* S0, const void* dout, const float* dST, void* dq,
                          void* dk, void* dv, void* dlog_alpha, void* dbeta, float* dS0, int B, int T, int H,
                          int Dk, int Dv, int chunk, gdn2_dtype dt, int states_saved, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * Sequences of different lengths packed along the token axis. Sequence n
 * holds packed tokens cu_seqlens[n] .. cu_seqlens[n+1] - 1 and has its own
 * initial and final state; the state does not pass from one sequence to the
 * next.
 *   q, k, log_alpha, b : [Ttot, H, Dk] dt ;  v, w, o, dout : [Ttot, H, Dv] dt
 *   cu_seqlens         : [N + 1] int32, DEVICE memory, non-decreasing, from 0
 *   N, Tmax, Ttot      : number of sequences, a bound on their lengths (host
 *                        ints; the work is sized by N x Tmax), packed length
 *   S0, ST, dST, dS0   : [N, H, Dk, Dv] float32 (nullable as in gdn2_fwd/bwd)
 * Token gradients are packed like the inputs. The calls copy the packed
 * tensors into a zero-padded [N, Tmax, H, D] layout in the workspace, run
 * gdn2_fwd / gdn2_bwd on it and copy the results back (a zero token maps the
 * state to itself, so the padding changes no result). cu_seqlens is not read
 * on the host: a sequence longer than Tmax is cut at Tmax, one outside
 * [0, Ttot) is skipped, and gdn2_device_status then returns GDN2_ERR_INVALID
 * with the detail "cu_seqlens".
 * Workspace: gdn2_varlen_workspace_size(op, ...) bytes, 256-byte aligned; the
 * GDN2_OP_BWD size serves gdn2_varlen_fwd(save_states = 1) followed by
 * gdn2_varlen_bwd(states_saved = 1).
 */
size_t gdn2_varlen_workspace_size(gdn2_op op, int N, int Tmax, int H, int Dk, int Dv, int chunk, gdn2_dtype dt);
gdn2_status gdn2_varlen_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                            const void* w, const int* cu_seqlens, int N, int Tmax, long long Ttot, const float* S0,
                            void* o, float* ST, int H, int Dk, int Dv, int chunk, gdn2_dtype dt, int save_states,
                            void* ws, size_t ws_bytes, void* stream);
gdn2_status gdn2_varlen_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                            const void* w, const int* cu_seqlens, int N, int Tmax, long long Ttot, const float* S0,
                            const void* dout, const float* dST, void* dq, void* dk, void* dv, void* dlog_alpha,
                            void* db, void* dw, float* dS0, int H, int Dk, int Dv, int chunk, gdn2_dtype dt,
                            int states_saved, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward without a caller-supplied workspace. The paper has no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc where they
 * need gradients -- code running inside another component's memory management
 * (a framework's caching allocator, a plugin handed only its tensors), code
 * that must not synchronise the device (cudaMalloc/cudaFree may), or code that
 * must not be able to fail for lack of memory after start-up.
 *
 * Same arguments and results as gdn2_bwd with states_saved = 0, minus the
 * workspace: the scratch memory lives in a fixed array of
 * GDN2_NO_ALLOC_SCRATCH_BYTES bytes inside the library, present on every GPU
 * that loads the library until it is unloaded. Nothing is allocated.
 *   - Problems whose gdn2_workspace_size(GDN2_OP_BWD, ...) exceeds that size
 *     are rejected with GDN2_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current). Under lazy module loading
 *     (CUDA_MODULE_LOADING=LAZY, the default) that first lookup also loads the
 *     library's device code and commits the array's memory, so it can fail for
 *     lack of memory and it can synchronise: make the first call on each device
 *     during start-up, and before any stream capture on the device.
 *   - The looked-up address is kept for the life of the process. After a reset
 *     of the device (cudaDeviceReset, or a primary context that was released
 *     and created again) it is stale, and this entry point must not be used on
 *     that device any more.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents (nothing in it needs to start at zero). Calls whose work overlaps
 *     on the GPU -- other streams or host threads on the same device -- race on
 *     it: order them.
 */
#define GDN2_NO_ALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
gdn2_status gdn2_bwd_no_alloc(const void* q, const void* k, const void* v, const void* log_alpha,
                              const void* b, const void* w, const float* S0, const void* dout,
                              const float* dST, void* dq, void* dk, void* dv, void* dlog_alpha,
                              void* db, void* dw, float* dS0, int B, int T, int H, int Dk, int Dv,
                              int chunk, gdn2_dtype dt, void* stream);

/* Size in bytes of the fixed scratch array used by gdn2_bwd_no_alloc. */
size_t gdn2_no_alloc_scratch_bytes(void);

/*
 * Affine maps of a sequence piece, for one sequence cut into pieces that run on
 * several devices (context parallelism). The recurrence is linear in the state
 * (S_t = (I - k_t (b_t*k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t*v_t)^T, the
 * state update of the GitHub README's introduction; the abstract's fixed-size
 * state is what crosses a piece boundary), so a piece maps its start state to its end
 * state as S_end = M S_start + N, and its backward maps the end gradient to the
 * start gradient as dS_start = A dS_end + B (A = M^T in exact arithmetic; B is
 * the start gradient from a zero end gradient). With the maps of the pieces
 * before it, a device forms its start state (and with those after it, its end
 * gradient) and then runs gdn2_fwd / gdn2_bwd on its own piece.
 *   q .. w, dout : one piece [B, T, H, D] dt, as in gdn2_fwd / gdn2_bwd
 *   M, A         : [B, H, Dk, Dk] float32 out
 *   N, Bm        : [B, H, Dk, Dv] float32 out
 * Tensor-core path only (dt = GDN2_BF16, Dk = Dv = 128); other problems return
 * GDN2_ERR_UNSUPPORTED. T = 0 gives M = A = I and N = Bm = 0. Workspace:
 * gdn2_workspace_size(GDN2_OP_MAP, ...) bytes, 256-byte aligned (the WY images
 * of the piece and their flags; with few heads and a long piece also the maps
 * of its segments, which run in parallel and are then composed). The maps go
 * to the caller's buffers; nothing else outside the workspace is written.
 */
gdn2_status gdn2_fwd_map(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                         const void* w, float* M, float* N, int B, int T, int H, int Dk, int Dv, int chunk,
                         gdn2_dtype dt, void* ws, size_t ws_bytes, void* stream);
gdn2_status gdn2_bwd_map(const void* q, const void* k, const void* v, const void* log_alpha, const void* b,
                         const void* w, const void* dout, float* A, float* Bm, int B, int T, int H, int Dk,
                         int Dv, int chunk, gdn2_dtype dt, void* ws, size_t ws_bytes, void* stream);
/*
 * S_out = M S_in + N per (batch, head), in float32: the step that chains the
 * maps above. M: [B, H, Dk, Dk]; S_in, N, S_out: [B, H, Dk, Dv]; S_in NULL
 * reads as zero, N NULL as zero. S_out may alias S_in or N (not M). Device
 * pointers, 16-byte aligned.
 */
gdn2_status gdn2_state_affine(const float* M, const float* N, const float* S_in, float* S_out, int B, int H,
                              int Dk, int Dv, void* stream);

/*
 * Gate activations of a Gated DeltaNet-2 layer: the operator's inputs from one
 * projection of the hidden state. The pages name the two per-channel gate
 * computations (GitHub README method bullets; the aiexpert.news article puts
 * the overhead over KDA on them) but not their parameterisation; the plainest
 * reading is used. Per token and head, z = [z_q | z_k | z_v | z_b | z_w | z_a]
 * (widths Dk, Dk, Dv, Dk, Dv, Dk) gives
 *   q = z_q / ||z_q||,  k = z_k / ||z_k||   (L2 over the head's channels, 1e-6
 *                                            added under the root)
 *   v = z_v,  b = sigmoid(z_b),  w = sigmoid(z_w),
 *   log_alpha = -softplus(z_a + a_bias)
 *   z                   : [B, T, H, 4 Dk + 2 Dv] dt
 *   a_bias              : [H, Dk] float32 decay bias, or NULL for none
 *   q, k, b, log_alpha  : [B, T, H, Dk] dt ;  v, w : [B, T, H, Dv] dt
 * gdn2_layer_gates_bwd writes dz (same layout as z) from z and the gradients of
 * the six outputs (as gdn2_bwd returns them); the gradient of a_bias is the sum
 * of dz_a over batch and tokens. Device pointers, 16-byte aligned;
 * no workspace; any Dk, Dv the operator supports; fp32 arithmetic.
 */
gdn2_status gdn2_layer_gates_fwd(const void* z, const float* a_bias, void* q, void* k, void* v, void* b, void* w,
                                 void* log_alpha, int B, int T, int H, int Dk, int Dv, gdn2_dtype dt, void* stream);
gdn2_status gdn2_layer_gates_bwd(const void* z, const float* a_bias, const void* dq, const void* dk, const void* dv,
                                 const void* db, const void* dw, const void* dlog_alpha, void* dz, int B, int T, int H,
                                 int Dk, int Dv, gdn2_dtype dt, void* stream);

/*
 * Per-kernel timing, for profiling. gdn2_trace_enable(1) makes every later
 * kernel launch of the library record a CUDA event before and after it on the
 * launch's stream (gdn2_trace_enable(0) stops it; off by default).
 * gdn2_trace_read waits for the recorded events, writes up to max_kernels
 * entries -- comma-separated kernel names into names (capacity names_cap),
 * launch counts into launches, summed device milliseconds into ms -- returns
 * the number of entries, and clears the record. Host pointers; any may be NULL.
 */
void gdn2_trace_enable(int on);
int gdn2_trace_read(char* names, size_t names_cap, int* launches, double* ms, int max_kernels);

/* Device-side status of the tensor-core kernels. Every wait inside them (on an
 * mbarrier or on a ready flag written by another CTA) gives up after ~2 s; the
 * kernel then records the event in device memory, lets its own copies in flight
 * land, skips the rest of its work and exits (the outputs of that call are not
 * valid, the CUDA context stays usable). This call synchronises `stream` (a
 * cudaStream_t, NULL for the default stream), returns GDN2_ERR_TIMEOUT if such
 * an event was recorded since the previous call (gdn2_last_error names the
 * kernel and the kind of wait) and clears the record; GDN2_ERR_CUDA if the
 * stream holds a CUDA error, and GDN2_ERR_INVALID if a packed-sequence call met
 * an inconsistent cu_seqlens (see gdn2_varlen_fwd). The entry points above never
 * synchronise, so this is the call that checks a finished step after the fact.
 */
gdn2_status gdn2_device_status(void* stream);

/* Static description of a status code. */
const char* gdn2_status_string(gdn2_status s);

/* Detail of the last non-OK status returned on the calling host thread. */
const char* gdn2_last_error(void);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
int gdn2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
