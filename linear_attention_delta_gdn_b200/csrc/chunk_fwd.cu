// chunk_fwd.cu -- chunkwise WY forward of the Gated Delta Rule-2 operator on
// tcgen05 tensor cores (bf16 operands, fp32 TMEM accumulators, fp32 state).
//
// Chunk algebra ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
// Attention", arXiv abstract: chunkwise WY algorithm, decay absorbed into
// asymmetric erase factors), per head and chunk of 64 tokens starting from S:
//   prep     Et = g*b*k, Qt = g*q, Kt = k/g, U = w*v          (g = exp(cumsum log_alpha))
//   WY       [A; P] = [Et; Qt] Kt^T,  T = (I + strict_lower(A))^{-1},  Wm = T Et
//   state    Delta^T = U^T T^T - S^T Wm^T,  O = Qt S + P Delta,  S'^T = (S^T + Delta^T Kt) Diag(gC)
// Chunks with untame channels (see chunk_common.cuh) leave those channels out of [A; P] = [Et; Qt] Kt^T,
// add their terms exactly on CUDA cores, and update the state as S'^T = S^T Diag(gC) + Delta^T Kh with
// Kh = k*exp(G_C - G) (an extra tile of their WY image), since Kt itself would overflow.
// The WY step does not depend on S; the state step is a chain over the chunks of a head.
//
// One launch, two kinds of CTA (256 threads each, one CTA per SM):
//   * producers run two independent WY pipelines each (one warpgroup per pipeline, its own named
//     barrier, mbarriers and TMEM columns), over the chunks of all heads in chunk-major order; a
//     pipeline writes T, P, Wm, Qt, Kt, gC and the untame-channel mask of its chunk ("WY image", 65 KB,
//     plus Kh for chunks with untame channels) to the workspace and sets the chunk's ready flag (release)
//     once those stores have completed;
//   * consumers (one per head, or several heads each when heads outnumber them) walk their head's
//     chunks in order: they wait for the chunk's flag (acquire), copy its WY image into shared
//     memory and run the state step. The state S^T lives in TMEM (lane j = value channel, column
//     i = key channel) in fp32 with a bf16 copy in shared memory as the UMMA operand.
// With few heads the producers run on the SMs that the consumers leave idle, in the same
// cooperative launch (all CTAs resident, so every wait ends; each wait is also bounded in time).
// Otherwise the producers run as one launch and the consumers as a second one.
// For training, the chunk-start states are written as bf16 images; the WY images stay in the
// workspace for the backward.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

using namespace chunk;

// ---- consumer (state pass) shared memory, bytes from a 1024-aligned base
namespace sp {
constexpr uint32_t QQ = 0;          // 2 x [64 x 128] Qt from the WY image (by chunk parity)
constexpr uint32_t KT = 32768;      // 2 x [64 x 128] Kt (Kh for chunks with untame channels) from the WY image
constexpr uint32_t UU = 65536;      // [64 x 128] v -> U (even chunks)
constexpr uint32_t WW = 81920;      // [64 x 128] w (even chunks)
constexpr uint32_t WY = 98304;      // WY image head: T [64 x 64] | P [64 x 64] | Wm [64 x 128]
constexpr uint32_t TT = WY, PP = WY + 8192, WM = WY + 16384;
constexpr uint32_t ST = 131072;     // [128 x 128] S^T (bf16)
constexpr uint32_t DT = 163840;     // [128 x 64] Delta^T (bf16)
constexpr uint32_t GC = 180224;     // 2 x fp32 gC[128] from the WY image (by chunk parity)
constexpr uint32_t BAR = 181248;    // 4 mbarriers (load even, mma, load odd, unused), tmem base, abort flag
constexpr uint32_t MASK = BAR + 64; // 2 x untame-channel mask (4 words) from the WY image (by chunk parity)
constexpr uint32_t UU1 = 182272;    // [64 x 128] v -> U (odd chunks)
constexpr uint32_t WW1 = 198656;    // [64 x 128] w (odd chunks)
constexpr uint32_t END = 215040;
}  // namespace sp
// ---- producer (WY) shared memory: two independent pipelines of one warpgroup (4 warps) each, so that one
// unit's tensor-core round trips and barriers overlap the other unit's work
namespace wy {
constexpr uint32_t PIPE = 105472;   // bytes per pipeline
constexpr uint32_t QE = 0;          // [128 x 128]: rows 0..63 b -> Et, rows 64..127 q -> Qt
constexpr uint32_t KH = 32768;      // k, then fp32 A [64 x 64] (sq_idx) once the prep has read k
constexpr uint32_t KT = 49152;      // log_alpha -> Kt
constexpr uint32_t IMG = 65536;     // T | P (bf16 64 x 64 each), then Wm (bf16 64 x 128): the image's first 48 KB
constexpr uint32_t TT = IMG, PP = IMG + 8192;
constexpr uint32_t TF = 81920;      // fp32 T [64 x 64] (sq_idx), then Wm once the solve is done
constexpr uint32_t SX = 98304;      // solve temporaries (4 warps x 16 x XS fp32) | prep scan scratch (fp32 [8][128])
                                    // | list of the untame channels (exact path)
constexpr uint32_t GC = 104448;     // 2 x fp32 gC[128] (by unit parity)
constexpr uint32_t STAGE = TF;      // exact path for untame channels: fp32 [4][64][16] raw-input stage
constexpr uint32_t BAR = 2 * PIPE;  // 4 mbarriers (inputs, mma per pipeline), tmem base, abort flag
constexpr uint32_t UMASK = BAR + 64;  // untame-channel masks: [pipeline][unit parity][4 words]
constexpr uint32_t BETA = UMASK + 64; // scalar gates (and a scalar decay): [pipeline][unit parity][beta | log_alpha]
                                      // [64 tokens] 32-bit words holding them
}  // namespace wy
constexpr uint32_t SMEM_BYTES = (sp::END > wy::BETA + 2048 ? sp::END : wy::BETA + 2048) + 1024;
static_assert(sp::MASK + 32 <= sp::UU1 && sp::UU1 % 1024 == 0 && sp::WW1 % 1024 == 0, "consumer layout");
static_assert(4 * 16 * XS * 4 <= wy::GC - wy::SX && 8 * 128 * 4 <= wy::GC - wy::SX, "producer scratch fits");
static_assert(4 * 64 * 16 * 4 == TILE_64x128 && wy::STAGE + 4 * 64 * 16 * 4 <= wy::SX, "untame stage fits");
static_assert(TC_WY_QT == 32768 && TC_WY_KT == 49152 && TC_WY_GC == 65536 && TC_WY_MASK == 66048 &&
              TC_WY_KH == 66560, "WY image: T | P | Wm | Qt | Kt | gC | mask | (Kh)");
static_assert(wy::TF == wy::IMG + TC_WY_WM, "T | P | Wm contiguous in shared memory as in the image");
// The per-thread copy loops below are written for NT threads: copy_wy moves 8 (T | P | Wm) and 4 (Qt, Kt)
// 16-byte pieces per thread, the U = w*v loop 4 rows of 8 values. The kernel checks blockDim.x == NT.
static_assert(8 * 16 * NT == TC_WY_QT && 4 * 16 * NT == TILE_64x128 && 4 * NT * 8 == C * D, "NT-thread loops");

// TMEM columns. Consumer: S^T (fp32 state), Ut^T -> Delta^T, O x 2 (M=64). Producer pipeline g: [A; P] at
// 256 g, Wm (M=64) at 256 g + 64.
constexpr uint32_t TM_S = 0, TM_D = 128, TM_O = 256;   // O: two buffers of 128 columns (chunk parity)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t CONS_LOAD_BYTES = 2 * 64 * 128 * 2;   // v, w
constexpr uint32_t PROD_LOAD_BYTES = 4 * 64 * 128 * 2;

__device__ unsigned int g_fwd_error;

struct FwdParams {
    int T, H, BH, nc;
    int ncons, nprod;              // CTAs [0, ncons) are consumers, the next nprod are producers
    const __nv_bfloat16 *q, *k, *la, *b;   // raw inputs, read directly only by the untame-channel path
    const float* S0;
    __nv_bfloat16* o;              // may be null (states only)
    float* ST;
    unsigned char* states;         // [BH, nc] chunk-start state images, or null
    unsigned char* deltas;         // [BH, nc] Delta^T images, or null
    unsigned char* wyimg;          // [BH, nc] WY images
    unsigned int* flags;           // [BH, nc] ready flags (zero at launch)
    int split_R;                   // > 0: the chunks of a head are cut into split_R segments (long sequences)
    int phase;                     // with split_R: 1 (first segment, segment maps) or 3 (the other segments);
                                   // 5: the maps of the whole sequence of every head (map_N, map_M)
    float* sbuf;                   // with split_R: per head, segment start states, then the maps N and M
    float *map_N, *map_M;          // phase 5: [BH][D][D] each
    const __nv_bfloat16* beta;     // [B, T, H] erase and write gates b = w = beta 1 (kernels instantiated for
                                   // them: no b or w tiles are loaded), else null
};

// ---- consumer tasks
// Without a split, task t walks every chunk of head t from S0 (zero if none) and writes o, S_T and, for training,
// the chunk-start state and Delta images. A long sequence with few heads is cut into R segments instead; with
// the state after segment s-1 written S_s, a segment is an affine map S_{s+1} = M_s S_s + N_s, where N_s is the
// segment's final state from a zero start and M_s (d_k x d_k) the one from an identity start with no input
// (U = 0). Phase 1 walks segment 0 for real (its end is S_1) and, for s = 1 .. R-2, N_s and M_s as separate
// tasks; a prefix kernel then forms S_2 .. S_{R-1}; phase 3 walks segments 1 .. R-1 for real from S_s.
struct Task {
    int head, c0, c1;
    const float* start;   // start state [D][D] (row = key), or null: zero, or identity when ident
    bool ident;           // start from the identity (a segment's M)
    bool zero_u;          // no input: U = 0 (a segment's M)
    bool out;             // the real chain: o and, if requested, the training images
    float* fin;           // where the final state goes [D][D], or null
};
// per head: R-1 start states S_1 .. S_{R-1}, then N_1 .. N_{R-2}, then M_1 .. M_{R-2}
constexpr int SPLIT_R_MAX = 8;
constexpr size_t SPLIT_MATS_PER_HEAD = (SPLIT_R_MAX - 1) + 2 * (SPLIT_R_MAX - 2);
__host__ __device__ inline int seg_begin(int s, int nc, int R) { return (int)((long long)s * nc / R); }
__device__ __forceinline__ float* split_mat(const FwdParams& p, int head, int kind, int s) {   // kind 0: S, 1: N, 2: M
    const int R = p.split_R;
    const int idx = kind == 0 ? s - 1 : (kind == 1 ? (R - 1) + (s - 1) : (R - 1) + (R - 2) + (s - 1));
    if (!GDN2_IN(g_fwd_error, idx >= 0 && idx < (int)SPLIT_MATS_PER_HEAD && head < p.BH)) return nullptr;
    return p.sbuf + ((size_t)head * SPLIT_MATS_PER_HEAD + idx) * D * D;
}
__device__ __forceinline__ int task_count(const FwdParams& p) {
    if (p.phase == 5) return 2 * p.BH * (p.split_R ? p.split_R : 1);
    if (!p.split_R) return p.BH;
    return p.phase == 1 ? p.BH * (1 + 2 * (p.split_R - 2)) : p.BH * (p.split_R - 1);
}
__device__ Task task_at(const FwdParams& p, int t) {
    Task k{};
    k.head = t % p.BH;
    const size_t hd = (size_t)k.head * D * D;
    if (p.phase == 5) {   // the whole sequence as one piece: N from a zero start, M from the identity without input
        if (p.split_R) {      // per segment j: N_j into slot j, M_j into slot R + j (slot-major: [slot][BH][D][D])
            const int R = p.split_R, j = t / p.BH, s2 = j < R ? j : j - R;
            k.c0 = seg_begin(s2, p.nc, R); k.c1 = s2 == R - 1 ? p.nc : seg_begin(s2 + 1, p.nc, R);
            if (j >= R) { k.ident = true; k.zero_u = true; }
            k.fin = p.sbuf + ((size_t)j * p.BH + k.head) * D * D;
            return k;
        }
        k.c0 = 0; k.c1 = p.nc;
        if (t < p.BH) {
            k.fin = p.map_N + hd;
        } else {
            k.ident = true; k.zero_u = true; k.fin = p.map_M + hd;
        }
        return k;
    }
    if (!p.split_R) {
        k.c0 = 0; k.c1 = p.nc; k.start = p.S0 ? p.S0 + hd : nullptr; k.out = true; k.fin = p.ST ? p.ST + hd : nullptr;
        return k;
    }
    const int R = p.split_R, j = t / p.BH;
    if (p.phase == 1) {
        if (j == 0) {
            k.c0 = 0; k.c1 = seg_begin(1, p.nc, R); k.start = p.S0 ? p.S0 + hd : nullptr; k.out = true;
            k.fin = split_mat(p, k.head, 0, 1);
        } else if (j <= R - 2) {
            k.c0 = seg_begin(j, p.nc, R); k.c1 = seg_begin(j + 1, p.nc, R); k.fin = split_mat(p, k.head, 1, j);
        } else {
            const int s2 = j - (R - 2);
            k.c0 = seg_begin(s2, p.nc, R); k.c1 = seg_begin(s2 + 1, p.nc, R); k.ident = true; k.zero_u = true;
            k.fin = split_mat(p, k.head, 2, s2);
        }
    } else {
        const int s2 = 1 + j;
        k.c0 = seg_begin(s2, p.nc, R); k.c1 = s2 == R - 1 ? p.nc : seg_begin(s2 + 1, p.nc, R);
        k.start = split_mat(p, k.head, 0, s2); k.out = true;
        k.fin = (s2 == R - 1 && p.ST) ? p.ST + hd : nullptr;
    }
    return k;
}

struct Maps {
    CUtensorMap q, k, v, la, b, w;
};

__device__ __forceinline__ void sync_for_mma() {   // smem written by threads + TMEM accesses done -> MMA issuer
    tc::fence_async_smem();
    tc::tc_fence_before();
    __syncthreads();
}

// ------------------------------------------------------------------ producer
// The helpers below run on one warpgroup (wt = thread in the group, wq = warp in the group, which is
// also the TMEM lane quarter it may read) and synchronise it with wg_sync() (a named barrier).

// Gate prep of one chunk: thread = (8-token block tb = wt / 16, 8-channel group cg = wt % 16);
//   reads  log_alpha (KT), k (KH), b (QE rows 0..63), q (QE rows 64..127)
//   writes Et = g*b*k -> QE rows 0..63, Qt = g*q -> QE rows 64..127, Kt = k/g -> KT, gC;
//   block totals of the cumsum go through red (fp32 [8][128]). The threads of the last token block, which
//   hold G_C, OR the untame channels (log-decay over the chunk, -G_C, above TAME_LOG_DECAY) into umask
//   (bit = channel); their Kt is still written here and cleared afterwards (untame chunks only).
// One scalar gate per head and token (beta [B, T, H] bf16, 4-byte aligned): the 64 tokens of a chunk are copied
// into shared memory as the 32-bit words that hold them (cp.async, 4 bytes each, zeros past the end of the
// sequence); token row r of a chunk whose first element is e0 = (b T + t0) H + h sits in the high half of its
// word when e0 + r H is odd.
__device__ __forceinline__ void beta_words_copy(uint32_t* dst, const __nv_bfloat16* beta, int b, int h, int t0, int T,
                                                int H, int row) {
    const size_t e = ((size_t)b * T + t0 + row) * H + h;
    const bool valid = t0 + row < T;
    tc::cp_async4(dst + row, valid ? beta + (e & ~(size_t)1) : beta, valid);
}
__device__ __forceinline__ float beta_word_value(const uint32_t* words, int row, int e0_odd, int H_odd) {
    const uint32_t w = words[row];
    return __uint_as_float(((e0_odd ^ (row & H_odd)) ? w >> 16 : w & 0xFFFFu) << 16);
}

// With BETA, b is one value per token, read from the chunk's beta words (bw, e0_odd, H_odd: beta_word_value;
// QE rows 0..63 hold no b tile).
template <bool BETA, typename Sync>
__device__ __forceinline__ void gate_prep_wg(unsigned char* QE, const unsigned char* KH, unsigned char* KT,
                                             float* gC_out, float* red, unsigned int* umask, int wt, const uint32_t* bw,
                                             int e0_odd, int H_odd, Sync&& wg_sync) {
    constexpr int RB = 8;
    const int cg = wt & 15, tb = wt >> 4;
    float G[RB][8];
#pragma unroll
    for (int u = 0; u < RB; ++u) {
        tc::ld_row8(KT, C, RB * tb + u, cg, G[u]);
        if (u > 0) {
#pragma unroll
            for (int c = 0; c < 8; ++c) G[u][c] += G[u - 1][c];
        }
    }
    *reinterpret_cast<float4*>(red + tb * 128 + 8 * cg) = make_float4(G[RB - 1][0], G[RB - 1][1], G[RB - 1][2], G[RB - 1][3]);
    *reinterpret_cast<float4*>(red + tb * 128 + 8 * cg + 4) = make_float4(G[RB - 1][4], G[RB - 1][5], G[RB - 1][6], G[RB - 1][7]);
    wg_sync();
    float pre[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int q = 0; q < tb; ++q) {
        const float4 x0 = *reinterpret_cast<const float4*>(red + q * 128 + 8 * cg);
        const float4 x1 = *reinterpret_cast<const float4*>(red + q * 128 + 8 * cg + 4);
        pre[0] += x0.x; pre[1] += x0.y; pre[2] += x0.z; pre[3] += x0.w;
        pre[4] += x1.x; pre[5] += x1.y; pre[6] += x1.z; pre[7] += x1.w;
    }
    if (tb == C / RB - 1) {
        unsigned int bits = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float tot = pre[c] + G[RB - 1][c];
            gC_out[8 * cg + c] = fast_exp(tot);
            bits |= (tot < -TAME_LOG_DECAY ? 1u : 0u) << c;
        }
        if (bits) atomicOr(umask + (cg >> 2), bits << (8 * (cg & 3)));
    }
#pragma unroll
    for (int u = 0; u < RB; ++u) {
        const int row = RB * tb + u;
        float kk[8], bb[8], qq[8], e[8], kt[8];
        tc::ld_row8(KH, C, row, cg, kk);
        if constexpr (BETA) {
            const float bv = beta_word_value(bw, row, e0_odd, H_odd);
#pragma unroll
            for (int c = 0; c < 8; ++c) bb[c] = bv;
        } else {
            tc::ld_row8(QE, 2 * C, row, cg, bb);
        }
        tc::ld_row8(QE, 2 * C, C + row, cg, qq);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float Gv = pre[c] + G[u][c];
            const float g = fast_exp(Gv), ig = fast_exp(-Gv);
            e[c] = g * bb[c] * kk[c];
            kt[c] = kk[c] * ig;
            qq[c] *= g;
        }
        tc::st_row8(QE, 2 * C, row, cg, e);
        tc::st_row8(KT, C, row, cg, kt);
        tc::st_row8(QE, 2 * C, C + row, cg, qq);
    }
}

// The same prep with one decay and one erase / write gate per token (Gated DeltaNet): the cumulative log-decay
// G_t and g_t = exp(G_t) are the same for every channel, so each thread keeps one value per row; log_alpha
// and beta come from their words (lw, bw), not from tiles. Every channel is untame or none is.
template <typename Sync>
__device__ __forceinline__ void gate_prep_scalar_wg(unsigned char* QE, const unsigned char* KH, unsigned char* KT,
                                                    float* gC_out, float* red, unsigned int* umask, int wt,
                                                    const uint32_t* bw, const uint32_t* lw, int e0_odd, int H_odd,
                                                    Sync&& wg_sync) {
    constexpr int RB = 8;
    const int cg = wt & 15, tb = wt >> 4;
    float G[RB];
#pragma unroll
    for (int u = 0; u < RB; ++u) G[u] = beta_word_value(lw, RB * tb + u, e0_odd, H_odd) + (u > 0 ? G[u - 1] : 0.f);
    if (cg == 0) red[tb] = G[RB - 1];
    wg_sync();
    float pre = 0.f;
#pragma unroll 1
    for (int q = 0; q < tb; ++q) pre += red[q];
    if (tb == C / RB - 1) {
        const float tot = pre + G[RB - 1];
        const float gc = fast_exp(tot);
#pragma unroll
        for (int c = 0; c < 8; ++c) gC_out[8 * cg + c] = gc;
        if (tot < -TAME_LOG_DECAY && cg == 0)
            for (int w = 0; w < 4; ++w) atomicOr(umask + w, 0xFFFFFFFFu);
    }
#pragma unroll
    for (int u = 0; u < RB; ++u) {
        const int row = RB * tb + u;
        float kk[8], qq[8], e[8], kt[8];
        tc::ld_row8(KH, C, row, cg, kk);
        tc::ld_row8(QE, 2 * C, C + row, cg, qq);
        const float Gv = pre + G[u];
        const float g = fast_exp(Gv), ig = fast_exp(-Gv);
        const float gb = g * beta_word_value(bw, row, e0_odd, H_odd);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            e[c] = gb * kk[c];
            kt[c] = kk[c] * ig;
            qq[c] *= g;
        }
        tc::st_row8(QE, 2 * C, row, cg, e);
        tc::st_row8(KT, C, row, cg, kt);
        tc::st_row8(QE, 2 * C, C + row, cg, qq);
    }
}

// Clears the Kt columns of the untame channels (umask) of the thread's 8 x 8 block (prep mapping), so that the
// tensor-core pair products leave them out.
__device__ __noinline__ void clear_untame_kt(unsigned char* KT, const unsigned int* umask, int wt) {
    const int cg = wt & 15, tb = wt >> 4;
    const unsigned int bits = (umask[cg >> 2] >> (8 * (cg & 3))) & 0xFFu;
    if (!bits) return;
#pragma unroll 1
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if ((bits >> c) & 1u) tc::st_bf16(KT, tc::tile_off(C, 8 * tb + u, 8 * cg + c), 0.f);
}

// Exact contributions of the untame channels (bits of umask) to A (sA: fp32, strictly lower) and P (PP: bf16,
// lower with the diagonal): for each such channel i and pair s <= t of the chunk,
//   A_ts += e_ti k_si L,  P_ts += q_ti k_si L,   L = prod_{s < tau <= t} alpha_tau,i = exp(G_ti - G_si) <= 1,
// e = b*k; and their column of the image's Kh tile, Kh_ti = k_ti prod_{tau > t} alpha_tau,i. The chunk's raw
// inputs are read from global memory, 16 channels at a time, into an fp32 stage ([alpha | k | e | q][64
// tokens][16]); thread (column s = wt % 64, A or P = wt / 64) keeps its 64 sums in registers and adds them at
// the end. Called by the whole warpgroup; ends with a barrier.
__device__ __noinline__ void untame_fixup_wg(int T, int H, const __nv_bfloat16* gq, const __nv_bfloat16* gk,
                                             const __nv_bfloat16* gla, const __nv_bfloat16* gb,
                                             const __nv_bfloat16* gbeta, bool sdec, int b, int h, int t0,
                                             const unsigned int* umask, float* sA, unsigned char* PP, float* stage,
                                             unsigned char* list, unsigned char* kh_img, int wt, int wg) {
    auto wg_sync = [&]() { tc::named_sync(1 + wg, 128); };
    const int w = wt >> 5, bit = wt & 31;
    int before = 0;
    for (int i = 0; i < w; ++i) before += __popc(umask[i]);
    const int nU = __popc(umask[0]) + __popc(umask[1]) + __popc(umask[2]) + __popc(umask[3]);
    if ((umask[w] >> bit) & 1u) list[before + __popc(umask[w] & ((1u << bit) - 1u))] = (unsigned char)wt;
    const int s = wt & 63;
    const bool isP = wt >= 64;
    const int L = min(C, T - t0);
    float* sAl = stage;
    float* sK = stage + 64 * 16;
    float* sE = stage + 2 * 64 * 16;
    float* sQ = stage + 3 * 64 * 16;
    float acc[C];
#pragma unroll
    for (int t = 0; t < C; ++t) acc[t] = 0.f;
    for (int g0 = 0; g0 < nU; g0 += 16) {
        wg_sync();   // the list is complete; the previous group's stage is no longer read
        {
            const int c = wt & 15, tb = wt >> 4;
            const int ch = g0 + c < nU ? (int)list[g0 + c] : -1;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int tau = 8 * tb + u;
                float al = 1.f, kk = 0.f, ee = 0.f, qq = 0.f;
                if (ch >= 0 && tau < L) {
                    const size_t off = tok_off(b, t0 + tau, h, T, H, D) + ch;
                    al = fast_exp(__bfloat162float(sdec ? gla[((size_t)b * T + t0 + tau) * H + h] : gla[off]));
                    kk = __bfloat162float(gk[off]);
                    ee = (gbeta ? __bfloat162float(gbeta[((size_t)b * T + t0 + tau) * H + h])
                                : __bfloat162float(gb[off])) * kk;
                    qq = __bfloat162float(gq[off]);
                }
                sAl[tau * 16 + c] = al;
                sK[tau * 16 + c] = kk;
                sE[tau * 16 + c] = ee;
                sQ[tau * 16 + c] = qq;
            }
        }
        wg_sync();
        if (wt < 16 && g0 + wt < nU) {   // Kh of channel list[g0 + wt]: suffix products of alpha
            const int ch = list[g0 + wt];
            float suf = 1.f;
            for (int t = C - 1; t >= 0; --t) {
                tc::st_bf16(kh_img, tc::tile_off(C, t, ch), sK[t * 16 + wt] * suf);
                suf *= sAl[t * 16 + wt];
            }
        }
        const float* X = isP ? sQ : sE;
        for (int c = 0; c < 16; ++c) {
            const float ks = sK[s * 16 + c];
            float Lp = 1.f;
#pragma unroll
            for (int t = 0; t < C; ++t) {
                if (t > s) Lp *= sAl[t * 16 + c];
                if (t > s || (isP && t == s)) acc[t] += X[t * 16 + c] * ks * Lp;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < C; ++t) {
        if (!isP && t > s) sA[sq_idx(t, s)] += acc[t];
        if (isP && t >= s) {
            const uint32_t off = tc::tile_off(C, t, s);
            tc::st_bf16(PP, off, tc::ld_bf16(PP, off) + acc[t]);
        }
    }
    wg_sync();
}

// [A; P] from TMEM (lanes 0..63 A, 64..127 P; 64 columns): warp wq reads its lane quarter; the strictly
// lower part of A goes to the fp32 scratch sA, the causal part of P to the bf16 tile PP.
__device__ __forceinline__ void extract_AP_wg(uint32_t lane_base_ap, float* sA, unsigned char* PP, int wq, int lane) {
    float v[32];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int c0 = 32 * hf;
        tc::tmem_ld32(lane_base_ap + c0, v);
        tc::tmem_wait_ld(v);
        if (wq < 2) {
            const int t = 32 * wq + lane;
#pragma unroll
            for (int u = 0; u < 32; ++u) sA[sq_idx(t, c0 + u)] = v[u];
        } else {
            const int t = 32 * (wq - 2) + lane;
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = (c0 + u <= t) ? v[u] : 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) tc::st_row8(PP, C, t, (c0 >> 3) + g, v + 8 * g);
        }
    }
}

// (I + A)^{-1} on one warpgroup: the diagonal 16 x 16 blocks by substitution (warp wq: block wq, which
// also clears its block row above the diagonal), then the off-diagonal blocks by diagonals, each warp
// taking both 8-column halves of its block in turn (warp-level tf32 products, mma.sync m16n8k8).
template <typename Sync>
__device__ __forceinline__ void solve_unit_lower_wg(const float* __restrict__ sA, float* __restrict__ sTf,
                                                    float* __restrict__ sX, unsigned char* Ttile, int wq, int lane,
                                                    Sync&& wg_sync) {
    switch (wq) {
    case 0: diag_inverse16<0>(sA, sTf, Ttile, lane); break;
    case 1: diag_inverse16<16>(sA, sTf, Ttile, lane); break;
    case 2: diag_inverse16<32>(sA, sTf, Ttile, lane); break;
    default: diag_inverse16<48>(sA, sTf, Ttile, lane); break;
    }
    {   // zeros above the diagonal block: block row wq, columns 16 wq + 16 .. 63
        const int base = 16 * wq, ngrp = (C - base - 16) / 8;
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int e = lane; e < 16 * ngrp; e += 32) tc::st_row8(Ttile, C, base + (e / ngrp), (base + 16) / 8 + (e % ngrp), z);
    }
    wg_sync();
    float* Xw = sX + wq * 16 * XS;
    float acc[4], p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};   // p0, p1: T_30's sums (warp 3)
    // X (16 x 8) -> per-warp temporary -> T_ij[:, nc..] = -T_ii X
    auto finish = [&](float (&x)[4], int i, int j, int nc, bool keep) {
        warp_store16x8(x, Xw, 0, 0, false, 1.f, lane);
        __syncwarp();
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sTf, 16 * i, 16 * i, Xw, 0, 0, false, lane);
        if (keep) warp_store16x8(acc, sTf, 16 * i, 16 * j + nc, true, -1.f, lane);
        warp_store16x8_tile(acc, Ttile, 16 * i, 16 * j + nc, -1.f, lane);
        __syncwarp();
    };
    // diagonal 1: T_{j+1,j} (warps 0..2); warp 3 starts T_30's sums with A_30 T_00
    if (wq < 3) {
        const int j = wq, i = j + 1;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            warp_mm16x8(x, sA, 16 * i, 16 * j, sTf, 16 * j, 16 * j + 8 * nt, true, lane);
            finish(x, i, j, 8 * nt, true);
        }
    } else {
        warp_mm16x8(p0, sA, 48, 0, sTf, 0, 0, true, lane);
        warp_mm16x8(p1, sA, 48, 0, sTf, 0, 8, true, lane);
    }
    wg_sync();
    // diagonal 2: T_20 (warp 0), T_31 (warp 1); warp 3 adds A_31 T_10
    if (wq < 2) {
        const int j = wq, i = j + 2;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            warp_mm16x8(x, sA, 16 * i, 16 * j, sTf, 16 * j, 16 * j + 8 * nt, true, lane);
            warp_mm16x8(x, sA, 16 * i, 16 * (j + 1), sTf, 16 * (j + 1), 16 * j + 8 * nt, true, lane);
            finish(x, i, j, 8 * nt, true);
        }
    } else if (wq == 3) {
        warp_mm16x8(p0, sA, 48, 16, sTf, 16, 0, true, lane);
        warp_mm16x8(p1, sA, 48, 16, sTf, 16, 8, true, lane);
    }
    wg_sync();
    // diagonal 3: T_30 = -T_33 (A_30 T_00 + A_31 T_10 + A_32 T_20)   (warp 3)
    if (wq == 3) {
        warp_mm16x8(p0, sA, 48, 32, sTf, 32, 0, true, lane);
        finish(p0, 3, 0, 0, false);
        warp_mm16x8(p1, sA, 48, 32, sTf, 32, 8, true, lane);
        finish(p1, 3, 0, 8, false);
    }
}

// Wm (M=64 accumulator, 128 columns) into rows 0..63 of a bf16 row tile with R rows: warp wq takes rows
// 16 wq .. 16 wq + 15 (its lane quarter's lanes 0..15).
__device__ __forceinline__ void tmem_m64_to_tile_wg(uint32_t lane_base_col, unsigned char* dst, int R, int wq, int lane) {
    const int r = 16 * wq + (lane & 15);
    float v[32];
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
        tc::tmem_ld32(lane_base_col + c0, v);
        tc::tmem_wait_ld(v);
        if (lane < 16) {
#pragma unroll
            for (int g = 0; g < 4; ++g) tc::st_row8(dst, R, r, (c0 >> 3) + g, v + 8 * g);
        }
    }
}

template <bool BETA, bool SDEC>
__device__ void run_producer(const Maps& m, const FwdParams& p, unsigned char* sm, uint32_t tmem, int pid) {
    // no b tile with BETA, no log_alpha tile with SDEC
    constexpr uint32_t LOAD_BYTES = PROD_LOAD_BYTES - (BETA ? 64u * 128u * 2u : 0u) - (SDEC ? 64u * 128u * 2u : 0u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, wq = warp & 3, wt = tid & 127;   // pipeline, warp and thread in it
    unsigned char* pb = sm + wg * wy::PIPE;
    unsigned char* QE = pb + wy::QE;
    unsigned char* KH = pb + wy::KH;
    unsigned char* KT = pb + wy::KT;
    unsigned char* TT = pb + wy::TT;
    unsigned char* PP = pb + wy::PP;
    float* sA = reinterpret_cast<float*>(pb + wy::KH);
    float* sTf = reinterpret_cast<float*>(pb + wy::TF);
    float* sX = reinterpret_cast<float*>(pb + wy::SX);
    uint64_t* bar_in = reinterpret_cast<uint64_t*>(sm + wy::BAR) + 2 * wg;
    uint64_t* bar_mma = bar_in + 1;
    int* abort_flag = reinterpret_cast<int*>(sm + wy::BAR + 36);
    const uint32_t lane_base = tmem + ((uint32_t)(32 * wq) << 16);
    const uint32_t tm_ap = tmem + 256 * wg, tm_w = tmem + 256 * wg + 64;
    const uint32_t sQE = tc::smem_u32(QE), sKT = tc::smem_u32(KT), sTT = tc::smem_u32(TT);
    constexpr uint32_t ID_M1 = tc::idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_M2 = tc::idesc_bf16(64, 128, false, true);
    auto wg_sync = [&]() { tc::named_sync(1 + wg, 128); };
    auto sync_for_mma_wg = [&]() {
        tc::fence_async_smem();
        tc::tc_fence_before();
        wg_sync();
    };
    uint32_t ph_in = 0, ph_mma = 0;
    auto wait_mma = [&]() {
        if (!tc::mbar_wait(bar_mma, ph_mma)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 1u); }
        ph_mma ^= 1;
        tc::tc_fence_after();
    };
    const int units = p.BH * p.nc, npipe = 2 * p.nprod;
    // The WY image of a unit is written by bulk stores of the pipeline's thread 0 in two groups: Qt, Kt and
    // gC right after the prep (with the untame mask, a plain store; the Kh tile of a chunk with untame
    // channels comes from the prep's own plain stores), T | P | Wm at the end of the unit. The same thread
    // sets the unit's flag at
    // the end of the pipeline's next unit, when its stores have long completed (the wait for them and the
    // release fence then cost little). The next unit's tiles are loaded as soon as their
    // buffers are free: q and log_alpha (over Qt, Kt) once M1 and the first group have read them, k (over
    // A) after the solve, b (over Et) once M2 has read it. Before the solve writes T | P | Wm, the previous
    // unit's second group has read them (thread 0 waits for that before issuing M1, whose completion the
    // other threads wait for).
    long long unreleased = -1;
    int kunit = 0;
    bool inflight = false;   // the next unit's loads are issued
    auto coords = [&](int u, int& b, int& h, int& t0) {
        const int c = u / p.BH, head = u % p.BH;
        b = head / p.H; h = head % p.H; t0 = c * C;
    };
    const int u0 = 2 * pid + wg;
    if (u0 < units && wt == 0) {   // the first unit's tiles
        int b, h, t0;
        coords(u0, b, h, t0);
        tc::mbar_arrive_expect_tx(bar_in, LOAD_BYTES);
        tma_tile(QE, 2 * C, C, &m.q, b, h, t0, bar_in);
        if (!SDEC) tma_tile(KT, C, 0, &m.la, b, h, t0, bar_in);
        tma_tile(KH, C, 0, &m.k, b, h, t0, bar_in);
        if (!BETA) tma_tile(QE, 2 * C, 0, &m.b, b, h, t0, bar_in);
    }
    // BETA: a unit's beta words (and with SDEC its log_alpha words), by unit parity, copied by threads 0..63 of
    // the pipeline at the start of the unit before. The beta words are read after the prep's first barrier:
    // those threads wait for them at the start of the unit; the log_alpha words are read before it: with SDEC
    // they wait at the end of the unit before, ahead of its last barrier.
    uint32_t* betaw = reinterpret_cast<uint32_t*>(sm + wy::BETA) + 256 * wg;
    auto copy_beta = [&](int u, int par) {
        int b_, h_, t0_;
        coords(u, b_, h_, t0_);
        beta_words_copy(betaw + 128 * par, p.beta, b_, h_, t0_, p.T, p.H, wt);
        if (SDEC) beta_words_copy(betaw + 128 * par + 64, p.la, b_, h_, t0_, p.T, p.H, wt);
        tc::cp_async_commit();
    };
    if (BETA && u0 < units) {
        if (wt < 64) copy_beta(u0, 0);
        if (SDEC) {
            if (wt < 64) tc::cp_async_wait_all();
            wg_sync();
        }
    }
    for (int u = u0; u < units; u += npipe, ++kunit) {
        const int c = u / p.BH, head = u % p.BH;
        const bool next = u + npipe < units;
        int nb = 0, nh = 0, nt0 = 0;
        if (next) coords(u + npipe, nb, nh, nt0);
        if (BETA && wt < 64) {
            if (next) copy_beta(u + npipe, (kunit + 1) & 1);
            if (!SDEC) {   // this unit's words
                if (next) tc::cp_async_wait_but1();
                else tc::cp_async_wait_all();
            }
        }
        float* gC = reinterpret_cast<float*>(pb + wy::GC + (kunit & 1) * 512);
        if (!tc::mbar_wait(bar_in, ph_in)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 2u); }
        ph_in ^= 1;
        inflight = false;

        // untame-channel mask of this unit (by unit parity; the other parity is cleared for the next unit,
        // whose prep sets bits only after a barrier of this pipeline)
        unsigned int* umask = reinterpret_cast<unsigned int*>(sm + wy::UMASK) + 8 * wg + 4 * (kunit & 1);
        if (wt < 4) reinterpret_cast<unsigned int*>(sm + wy::UMASK)[8 * wg + 4 * ((kunit + 1) & 1) + wt] = 0u;
        unsigned char* img = p.wyimg + ((size_t)head * p.nc + c) * TC_WY_BYTES;
        const bool img_ok = GDN2_IN(g_fwd_error, head < p.BH && c < p.nc);   // else the image is not written
        {
            const int e0 = (int)((((size_t)(head / p.H) * p.T + (size_t)c * C) * p.H + head % p.H) & 1);
            if constexpr (SDEC)
                gate_prep_scalar_wg(QE, KH, KT, gC, sX, umask, wt, betaw + 128 * (kunit & 1),
                                    betaw + 128 * (kunit & 1) + 64, e0, p.H & 1, wg_sync);
            else
                gate_prep_wg<BETA>(QE, KH, KT, gC, sX, umask, wt, betaw + 128 * (kunit & 1), e0, p.H & 1, wg_sync);
        }
        sync_for_mma_wg();
        const bool untame = (umask[0] | umask[1] | umask[2] | umask[3]) != 0u;   // the same on every thread
        if (untame) {   // their Kt columns are cleared before the image's Kt and M1 read KT
            clear_untame_kt(KT, umask, wt);
            sync_for_mma_wg();
        }
        if (wt == 0 && img_ok) {   // first image group: Qt, Kt, gC (final after the prep), and the untame mask
            tc::bulk_store(img + TC_WY_QT, QE + 8192, 8192u);               // Qt (two 64-row halves of the
            tc::bulk_store(img + TC_WY_QT + 8192, QE + 24576, 8192u);       //  128-row tile, 16 KB apart)
            tc::bulk_store(img + TC_WY_KT, KT, 16384u);                     // Kt
            tc::bulk_store(img + TC_WY_GC, gC, 512u);                       // gC
            tc::bulk_commit();
            *reinterpret_cast<uint4*>(img + TC_WY_MASK) = make_uint4(umask[0], umask[1], umask[2], umask[3]);
        }
        if (wt == 0) {   // [A; P] = [Et; Qt] Kt^T
            tc::bulk_wait_read_but1();   // the previous unit's T | P | Wm may be overwritten
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tm_ap, tc::desc_k(sQE, 2 * C, 0, kk), tc::desc_k(sKT, C, 0, kk), ID_M1, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        if (wt == 0 && next) {   // the next unit's q and log_alpha over Qt, Kt
            tc::bulk_wait_read();
            tc::mbar_arrive_expect_tx(bar_in, LOAD_BYTES);
            tma_tile(QE, 2 * C, C, &m.q, nb, nh, nt0, bar_in);
            if (!SDEC) tma_tile(KT, C, 0, &m.la, nb, nh, nt0, bar_in);
            inflight = true;
        }
        extract_AP_wg(lane_base + (tm_ap - tmem), sA, PP, wq, lane);   // A over k: the prep has read k
        tc::tc_fence_before();
        wg_sync();
        if (untame && img_ok) {   // exact terms of the channels left out of M1 (TF is free until the solve)
            int b, h, t0;
            coords(u, b, h, t0);
            untame_fixup_wg(p.T, p.H, p.q, p.k, p.la, p.b, BETA ? p.beta : nullptr, SDEC, b, h, t0, umask, sA, PP,
                            reinterpret_cast<float*>(pb + wy::STAGE), reinterpret_cast<unsigned char*>(sX),
                            img + TC_WY_KH, wt, wg);
        }
        solve_unit_lower_wg(sA, sTf, sX, TT, wq, lane, wg_sync);   // T = (I + A)^{-1}
        sync_for_mma_wg();
        if (wt == 0) {   // Wm = T Et ; the next unit's k over A (which the solve has finished with)
            if (next) tma_tile(KH, C, 0, &m.k, nb, nh, nt0, bar_in);
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tm_w, tc::desc_k(sTT, C, 0, kk), tc::desc_mn(sQE, 2 * C, 0, kk), ID_M2, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        if (!BETA && wt == 0 && next) tma_tile(QE, 2 * C, 0, &m.b, nb, nh, nt0, bar_in);   // the next unit's b over Et
        tmem_m64_to_tile_wg(lane_base + (tm_w - tmem), pb + wy::TF, C, wq, lane);   // Wm over the fp32 T
        sync_for_mma_wg();
        if (wt == 0) {   // the previous unit's flag (all its stores are older than this unit's first group);
                         // second image group: T | P | Wm
            if (unreleased >= 0 && !*abort_flag) tc::flag_release_after_bulk_but1(p.flags + unreleased, 1u);
            const size_t unit = (size_t)head * p.nc + c;
            if (img_ok) tc::bulk_store(p.wyimg + unit * TC_WY_BYTES + TC_WY_T, TT, 32768u);
            tc::bulk_commit();
            unreleased = (long long)unit;
        }
        if (SDEC && wt < 64) tc::cp_async_wait_all();   // the next unit's words (published by the barrier)
        // all 128 threads leave together if any has seen the abort flag (the other pipeline may set it at
        // any time, so separate reads could split the threads that synchronise on this barrier)
        if (tc::named_sync_or(1 + wg, 128, *abort_flag != 0)) break;
    }
    if (wt == 0) {   // the last unit's flag; every image store completes before the CTA leaves
        if (unreleased >= 0 && !*abort_flag) tc::flag_release_after_bulk(p.flags + unreleased, 1u);
        tc::bulk_wait_all();
    }
    // after an abort: the next unit's loads land before the CTA's shared memory is released
    if (wt == 0 && inflight) (void)tc::mbar_wait(bar_in, ph_in);
    if (BETA) tc::cp_async_wait_all();   // and the beta words in flight
}

// ------------------------------------------------------------------ consumer

// Kh of a chunk with untame channels, in place of its Kt tile (bf16 [64 x 128] row tile): Kt * gC on the
// tame columns, and on the untame ones (bits of msk) the values that the producer wrote to the image's Kh
// tile (kh_img, global memory). NT threads, 4 pieces of 8 columns each.
__device__ __noinline__ void kh_from_kt(unsigned char* KT, const unsigned char* kh_img, const float* gC, uint4 msk,
                                        int tid) {
    const unsigned int mw[4] = {msk.x, msk.y, msk.z, msk.w};
#pragma unroll 1
    for (int e = 0; e < 4; ++e) {
        const int idx = tid + NT * e, row = idx >> 4, g = idx & 15;
        float x[8];
        tc::ld_row8(KT, C, row, g, x);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int col = 8 * g + c;
            x[c] = ((mw[col >> 5] >> (col & 31)) & 1u) ? tc::ld_bf16(kh_img, tc::tile_off(C, row, col)) : x[c] * gC[col];
        }
        tc::st_row8(KT, C, row, g, x);
    }
}

template <bool BETA>
__device__ void run_consumer(const Maps& m, const FwdParams& p, unsigned char* sm, uint32_t tmem, int cid) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // v and w tiles by chunk parity: chunk c + 2 is loaded while chunk c + 1's tiles wait in the other pair
    auto UUp = [&](int c) { return sm + ((c & 1) ? sp::UU1 : sp::UU); };
    auto WWp = [&](int c) { return sm + ((c & 1) ? sp::WW1 : sp::WW); };
    unsigned char* STt = sm + sp::ST;
    unsigned char* DT = sm + sp::DT;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + sp::BAR);
    uint64_t* bar_mma = bars + 1;
    auto bar_ld = [&](int c) { return bars + ((c & 1) ? 2 : 0); };
    int* abort_flag = reinterpret_cast<int*>(sm + sp::BAR + 36);
    const uint32_t lane_base = tmem + ((uint32_t)(tm_quarter(warp) * 32) << 16);   // this warp's TMEM lanes
    const int jrow = 32 * tm_quarter(warp) + lane, cpart = 64 * tm_part(warp);      // lane row, column half
    const int T = p.T, H = p.H, nc = p.nc;

    const uint32_t sST = tc::smem_u32(STt), sDT = tc::smem_u32(DT),
                   sTT = tc::smem_u32(sm + sp::TT), sPP = tc::smem_u32(sm + sp::PP), sWM = tc::smem_u32(sm + sp::WM);
    constexpr uint32_t ID_M3 = tc::idesc_bf16(128, 64, true, false);
    constexpr uint32_t ID_M4 = tc::idesc_bf16(128, 64, false, false, true);
    constexpr uint32_t ID_M56 = tc::idesc_bf16(64, 128, false, false);
    constexpr uint32_t ID_M7 = tc::idesc_bf16(128, 128, false, true);

    uint32_t ph_load = 0, ph_mma = 0;   // ph_load: bit p is the phase of the load barrier of parity p
    auto wait_mma = [&]() {
        if (!tc::mbar_wait(bar_mma, ph_mma)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 1u); }
        ph_mma ^= 1;
        tc::tc_fence_after();
    };
    // thread 0 waits for the WY image of (head, c); the caller synchronises the CTA afterwards
    auto wait_wy = [&](size_t head, int c) {
        if (!tc::flag_wait(p.flags + head * nc + c, 1u)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 4u); }
    };
    // the WY image of (head, c): T | P | Wm to WY, Qt and Kt to this chunk's parity buffers, gC and the mask
    auto copy_wy = [&](size_t head, int c) {
        const unsigned char* src = p.wyimg + (head * nc + c) * TC_WY_BYTES;
        const int par = c & 1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int o = 16 * (tid + NT * i);
            tc::cp_async16_cg(sm + sp::WY + o, src + o);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int o = 16 * (tid + NT * i);
            tc::cp_async16_cg(sm + sp::QQ + par * TILE_64x128 + o, src + TC_WY_QT + o);
            tc::cp_async16_cg(sm + sp::KT + par * TILE_64x128 + o, src + TC_WY_KT + o);
        }
        if (tid < 32) tc::cp_async16_cg(sm + sp::GC + par * 512 + 16 * tid, src + TC_WY_GC + 16 * tid);
        if (tid == 32) tc::cp_async16_cg(sm + sp::MASK + par * 16, src + TC_WY_MASK);
        tc::cp_async_commit();
    };

    const int ntasks = task_count(p);
    for (int ti = cid; ti < ntasks; ti += p.ncons) {
        const Task task = task_at(p, ti);
        if (!GDN2_IN(g_fwd_error, task.head >= 0 && task.head < p.BH && 0 <= task.c0 && task.c0 < task.c1 &&
                                      task.c1 <= nc))
            continue;   // the same on every thread, before any barrier of the task
        const int headi = task.head, c0 = task.c0, c1 = task.c1;
        const size_t head = (size_t)headi;
        const int h = headi % H, b = headi / H;
        const bool want_o = task.out && p.o != nullptr;
        unsigned char* const states = task.out ? p.states : nullptr;   // training images: real chains only
        unsigned char* const deltas = task.out ? p.deltas : nullptr;
        const bool zero_u = task.zero_u;
        // v and w of chunk c (issued by lane 0 of warps 0 and 1 at once; a TMA issue takes ~100 cycles)
        auto issue_loads = [&](int c) {
            if (lane != 0 || warp > 1) return;
            const int t0 = c * C;
            if (warp == 0) {
                tc::mbar_arrive_expect_tx(bar_ld(c), CONS_LOAD_BYTES - (BETA ? 64u * 128u * 2u : 0u));
                tma_tile(UUp(c), C, 0, &m.v, b, h, t0, bar_ld(c));
            } else if (!BETA) {
                tma_tile(WWp(c), C, 0, &m.w, b, h, t0, bar_ld(c));
            }
        };
        // o rows of chunk c from its M=64 accumulator (16-byte stores)
        auto store_o = [&](int c) {
            const int t0 = c * C, L = min(C, T - t0);
            const int t = m64_row(warp, lane);
            const uint32_t ob = lane_base + TM_O + 128 * (c & 1);
            float v[32];
#pragma unroll
            for (int c0 = cpart; c0 < cpart + 64; c0 += 32) {
                tc::tmem_ld32(ob + c0, v);
                tc::tmem_wait_ld(v);
                if (lane < 16 && t < L) {
                    uint4* dst = reinterpret_cast<uint4*>(p.o + tok_off(b, t0 + t, h, T, H, D) + c0);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        dst[g] = make_uint4(tc::pack_bf16x2(v[8 * g], v[8 * g + 1]), tc::pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                            tc::pack_bf16x2(v[8 * g + 4], v[8 * g + 5]), tc::pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
                }
            }
        };
        if (!zero_u) {
            issue_loads(c0);
            if (c0 + 1 < c1) issue_loads(c0 + 1);
        }
        // BETA: w is the gate of the token; chunk c's beta words go into its (unused) w tile, copied with its v
        // tile two chunks ahead and complete at the cp.async wait of the chunk before
        auto copy_beta = [&](int c) {
            if (tid < 64) {
                beta_words_copy(reinterpret_cast<uint32_t*>(WWp(c)), p.beta, b, h, c * C, T, H, tid);
                tc::cp_async_commit();
            }
        };
        if (BETA && !zero_u) {
            copy_beta(c0);
            if (c0 + 1 < c1) copy_beta(c0 + 1);
            tc::cp_async_wait_all();   // chunk c0's words, before the barrier below
        }
        if (tid == 0) wait_wy(head, c0);
        // start state: S^T row j = column j of the start matrix (zero if none, or the identity)
        {
            const int j = jrow;
            float v[32];
#pragma unroll 1
            for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
#pragma unroll
                for (int u = 0; u < 32; ++u)
                    v[u] = task.start ? task.start[(i0 + u) * D + j] : (task.ident && i0 + u == j ? 1.f : 0.f);
                tc::tmem_st32(lane_base + TM_S + i0, v);
#pragma unroll
                for (int g = 0; g < 4; ++g) tc::st_row8(STt, D, j, (i0 >> 3) + g, v + 8 * g);
            }
            tc::tmem_wait_st();
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        copy_wy(head, c0);
        if (states && tid == 0) {
            tc::bulk_store(states + (head * nc + c0) * TC_STATE_BYTES, STt, (uint32_t)TC_STATE_BYTES);
            tc::bulk_commit();
        }

        int c = c0;
        for (; c < c1; ++c) {
            const int par = c & 1;
            const uint32_t sQQ = tc::smem_u32(sm + sp::QQ + par * TILE_64x128),
                           sKT = tc::smem_u32(sm + sp::KT + par * TILE_64x128);
            const float* sGC = reinterpret_cast<const float*>(sm + sp::GC + par * 512);
            const uint32_t tm_o = tmem + TM_O + 128 * par;
            unsigned char* UU = UUp(c);
            const unsigned char* WW = WWp(c);
            const uint32_t sUU = tc::smem_u32(UU);
            if (!zero_u) {
                if (!tc::mbar_wait(bar_ld(c), (ph_load >> par) & 1u)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 2u); }
                ph_load ^= 1u << par;
            }

            // ---- U = w * v (Qt, Kt and gC come with the WY image): 4 row chunks of 8 values per thread
#pragma unroll
            for (int e = 0; e < 4 && !zero_u; ++e) {
                const int idx = tid + NT * e, row = idx >> 4, g = idx & 15;
                float vv[8], ww[8];
                tc::ld_row8(UU, C, row, g, vv);
                if constexpr (BETA) {
                    const float bv = beta_word_value(reinterpret_cast<const uint32_t*>(WW), row,
                                                     (int)((((size_t)b * T + (size_t)c * C) * H + h) & 1), H & 1);
#pragma unroll
                    for (int x = 0; x < 8; ++x) ww[x] = bv;
                } else {
                    tc::ld_row8(WW, C, row, g, ww);
                }
#pragma unroll
                for (int x = 0; x < 8; ++x) vv[x] *= ww[x];
                tc::st_row8(UU, C, row, g, vv);
            }

            tc::cp_async_wait_all();   // this chunk's WY image
            sync_for_mma();
            // a chunk with untame channels updates the state with Kh on a state scaled by gC first, the others
            // with Kt and a scaling afterwards
            const uint4 msk = *reinterpret_cast<const uint4*>(sm + sp::MASK + par * 16);
            const bool khm = (msk.x | msk.y | msk.z | msk.w) != 0u;   // the same on every thread
            if (khm) kh_from_kt(sm + sp::KT + par * TILE_64x128, p.wyimg + (head * nc + c) * TC_WY_BYTES + TC_WY_KH,
                                sGC, msk, tid);   // in the shadow of M3-M5, which do not read it

            // ---- M3: Delta^T := U^T T^T ;  M4: Delta^T -= S^T Wm^T  (commit) ;  M5: O = Qt S
            if (tid == 0) {
                tc::tc_fence_after();
                if (!zero_u) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tmem + TM_D, tc::desc_mn(sUU, C, 0, kk), tc::desc_k(sTT, C, 0, kk), ID_M3, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_D, tc::desc_k(sST, D, 0, kk), tc::desc_k(sWM, C, 0, kk), ID_M4,
                                 (zero_u && kk == 0) ? 0u : 1u);
                tc::mma_commit(bar_mma);
                if (want_o) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16(tm_o, tc::desc_k(sQQ, C, 0, kk), tc::desc_k(sST, D, 0, kk), ID_M56, kk > 0);
                }
                if (c + 1 < c1) wait_wy(head, c + 1);   // overlaps the MMAs
            }
            if (want_o && c > c0) store_o(c - 1);     // previous chunk's output, in the MMAs' shadow
            if (khm) {   // S^T := S^T Diag(gC) on the fp32 state, in the MMAs' shadow (M3-M5 read its bf16 copy); M7
                         // then adds Delta^T Kh
                float v[32];
#pragma unroll 1
                for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
                    tc::tmem_ld32(lane_base + TM_S + i0, v);
                    tc::tmem_wait_ld(v);
#pragma unroll
                    for (int u = 0; u < 32; ++u) v[u] *= sGC[i0 + u];
                    tc::tmem_st32(lane_base + TM_S + i0, v);
                }
                tc::tmem_wait_st();
            }
            wait_mma();
            // this chunk's v (read by M3) and w buffers are free: chunk c + 2's tiles go there
            if (!zero_u && c + 2 < c1) {
                issue_loads(c + 2);
                if (BETA) copy_beta(c + 2);
            }
            tmem_to_tile_rows<64>(lane_base + TM_D, DT, warp, lane);   // Delta^T (lane j) -> bf16 rows
            sync_for_mma();
            if (deltas && tid == 0) {   // Delta^T of this chunk for the backward
                tc::bulk_store(deltas + (head * nc + c) * TC_DELTA_BYTES, DT, (uint32_t)TC_DELTA_BYTES);
                tc::bulk_commit();
            }

            // ---- M6: O += P Delta ;  M7: Z^T = S^T + Delta^T Kt  (or S'^T = S^T Diag(gC) + Delta^T Kh)
            if (tid == 0) {
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (want_o)
                        tc::mma_bf16(tm_o, tc::desc_k(sPP, C, 0, kk), tc::desc_k(sDT, D, 0, kk), ID_M56, 1);
                    tc::mma_bf16(tmem + TM_S, tc::desc_k(sDT, D, 0, kk), tc::desc_mn(sKT, C, 0, kk), ID_M7, 1);
                }
                tc::mma_commit(bar_mma);
            }
            wait_mma();
            // S'^T = Z^T Diag(gC) (unless already scaled), and a bf16 copy of the new state for the next chunk
            // (the bulk stores of the previous state image and of this chunk's Delta^T must have read their tiles)
            if (states && tid == 0) tc::bulk_wait_read();
            __syncthreads();   // also orders thread 0's flag acquire before the image copy
            if (c + 1 < c1) copy_wy(head, c + 1);
            {
                const int j = jrow;
                float v[32];
#pragma unroll 1
                for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
                    tc::tmem_ld32(lane_base + TM_S + i0, v);
                    tc::tmem_wait_ld(v);
                    if (!khm) {
#pragma unroll
                        for (int u = 0; u < 32; ++u) v[u] *= sGC[i0 + u];
                        tc::tmem_st32(lane_base + TM_S + i0, v);
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g) tc::st_row8(STt, D, j, (i0 >> 3) + g, v + 8 * g);
                }
                if (!khm) tc::tmem_wait_st();
            }
            sync_for_mma();
            tc::tc_fence_after();
            if (states && tid == 0 && c + 1 < c1) {
                tc::bulk_store(states + (head * nc + c + 1) * TC_STATE_BYTES, STt, (uint32_t)TC_STATE_BYTES);
                tc::bulk_commit();
            }
            if (*abort_flag) {   // let the next chunk's loads land before leaving
                if (!zero_u && tid == 0 && c + 1 < c1) (void)tc::mbar_wait(bar_ld(c + 1), (ph_load >> ((c + 1) & 1)) & 1u);
                if (!zero_u && tid == 0 && c + 2 < c1) (void)tc::mbar_wait(bar_ld(c + 2), ((ph_load >> (c & 1)) & 1u));
                break;
            }
        }
        if (want_o && c == c1) store_o(c1 - 1);

        // final state (fp32): fin[i][j] from S^T (lane j)
        if (task.fin) {
            const int j = jrow;
            float v[32];
#pragma unroll 1
            for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
                tc::tmem_ld32(lane_base + TM_S + i0, v);
                tc::tmem_wait_ld(v);
#pragma unroll
                for (int u = 0; u < 32; ++u) task.fin[(i0 + u) * D + j] = v[u];
            }
        }
        tc::cp_async_wait_all();
        if (states && tid == 0) tc::bulk_wait_all();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        if (*abort_flag) break;
    }
}

template <bool BETA, bool SDEC>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_kernel(const __grid_constant__ Maps maps, const FwdParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays in the shared window
    const int tid = threadIdx.x, warp = tid >> 5;
    if (blockDim.x != NT) {   // the index arithmetic assumes NT threads: refuse any other launch shape
        if (tid == 0) atomicOr(&g_fwd_error, 16u);
        return;
    }
    const bool consumer = (int)blockIdx.x < p.ncons;
    const uint32_t bar_off = consumer ? sp::BAR : wy::BAR;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + bar_off);
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(sm + bar_off + 32);
    int* abort_flag = reinterpret_cast<int*>(sm + bar_off + 36);
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) tc::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        if (!consumer)
            for (int i = 0; i < 16; ++i) reinterpret_cast<unsigned int*>(sm + wy::UMASK)[i] = 0u;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&maps.q); tc::tma_prefetch_desc(&maps.k);
        if (!SDEC) tc::tma_prefetch_desc(&maps.la);
        if (consumer) {
            tc::tma_prefetch_desc(&maps.v);
            if (!BETA) tc::tma_prefetch_desc(&maps.w);
        } else if (!BETA) {
            tc::tma_prefetch_desc(&maps.b);
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base_ptr, TM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_base_ptr;
    if (consumer) run_consumer<BETA>(maps, p, sm, tmem, blockIdx.x);
    else run_producer<BETA, SDEC>(maps, p, sm, tmem, blockIdx.x - p.ncons);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TM_COLS);
    }
}

// Segment start states S_2 .. S_{R-1} from S_1 and the segment maps, S_{s+1} = M_s S_s + N_s, in fp32. The value
// columns of a state never mix, so CTA (head, block of 16 columns) runs the whole prefix for its columns. Thread
// (row group rq = tid / 4: rows rq + 32 r, r < 4; column quarter cq = tid % 4: 4 columns) keeps a 4 x 4 block of
// sums in registers, so one pass over the 128 terms of a product costs 8 shared-memory vector loads per 64
// FMAs. M_s goes to shared memory by cp.async, the next step's while this one runs (two buffers; rows padded
// to 132 floats so that the 8 rows a warp reads at once fall in distinct bank groups).
constexpr int PREFIX_LD = D + 4;
constexpr int PREFIX_THREADS = 128;
constexpr uint32_t PREFIX_SMEM = (uint32_t)(2 * D * PREFIX_LD + D * 16) * sizeof(float);
static_assert(D * D / 4 == 32 * PREFIX_THREADS && D == 4 * 32, "prefix thread mapping");
__global__ void __launch_bounds__(PREFIX_THREADS) split_prefix_kernel(float* sbuf, int R) {
    extern __shared__ float4 prefix_smem[];
    float* Mbuf = reinterpret_cast<float*>(prefix_smem);   // 2 x [D][PREFIX_LD]
    float(*Sc)[16] = reinterpret_cast<float(*)[16]>(Mbuf + 2 * D * PREFIX_LD);
    if (!GDN2_IN(g_fwd_error, R >= 4 && R <= SPLIT_R_MAX)) return;   // the slots of a head hold R <= SPLIT_R_MAX
    const int head = blockIdx.x / (D / 16), j0 = (blockIdx.x % (D / 16)) * 16;
    const int tid = threadIdx.x, cq = tid & 3, rq = tid >> 2;
    float* base = sbuf + (size_t)head * SPLIT_MATS_PER_HEAD * D * D;
    auto mat = [&](int kind, int s) { return base + (size_t)((kind == 0 ? 0 : (kind == 1 ? R - 1 : 2 * R - 3)) + s - 1) * D * D; };
    auto stage = [&](int s, int buf) {   // M_s -> buffer buf, 32 16-byte copies per thread
        const float4* src = reinterpret_cast<const float4*>(mat(2, s));
        float* dst = Mbuf + buf * D * PREFIX_LD;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int idx = tid + PREFIX_THREADS * e, r = idx >> 5, c4 = idx & 31;
            tc::cp_async16_cg(dst + r * PREFIX_LD + 4 * c4, src + idx);
        }
        tc::cp_async_commit();
    };
    stage(1, 0);
    const float* S1 = mat(0, 1);
    for (int e = tid; e < D * 16; e += PREFIX_THREADS) Sc[e >> 4][e & 15] = S1[(e >> 4) * D + j0 + (e & 15)];
    for (int s = 1; s <= R - 2; ++s) {
        const int buf = (s - 1) & 1;
        const float* N = mat(1, s);
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float4 n = *reinterpret_cast<const float4*>(N + (size_t)(rq + 32 * r) * D + j0 + 4 * cq);
            acc[r][0] = n.x; acc[r][1] = n.y; acc[r][2] = n.z; acc[r][3] = n.w;
        }
        if (s + 1 <= R - 2) {   // the next step's M goes to the other buffer (read last in step s - 1)
            stage(s + 1, buf ^ 1);
            tc::cp_async_wait_but1();
        } else {
            tc::cp_async_wait_all();
        }
        __syncthreads();   // every thread's copies of M_s, and S_s in Sc
        const float* Ms = Mbuf + buf * D * PREFIX_LD;
#pragma unroll 2
        for (int l = 0; l < D; l += 4) {
            float4 m[4], sv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) m[r] = *reinterpret_cast<const float4*>(Ms + (rq + 32 * r) * PREFIX_LD + l);
#pragma unroll
            for (int u = 0; u < 4; ++u) sv[u] = *reinterpret_cast<const float4*>(&Sc[l + u][4 * cq]);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float mr[4] = {m[r].x, m[r].y, m[r].z, m[r].w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    acc[r][0] += mr[u] * sv[u].x;
                    acc[r][1] += mr[u] * sv[u].y;
                    acc[r][2] += mr[u] * sv[u].z;
                    acc[r][3] += mr[u] * sv[u].w;
                }
            }
        }
        __syncthreads();   // every thread has read Sc and this buffer
        float* Sn = mat(0, s + 1);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = rq + 32 * r;
            *reinterpret_cast<float4*>(&Sc[i][4 * cq]) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
            *reinterpret_cast<float4*>(Sn + (size_t)i * D + j0 + 4 * cq) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        }
    }
    tc::cp_async_wait_all();
}

// Number of segments a head's chunks are cut into (0: none). Only when the heads leave most CTA slots idle
// and every segment keeps a few dozen chunks; bounded by the workspace reserved for the maps.
int split_segments(int BH, int nc, int slots, bool have_buf) {
    if (!have_buf || split_disabled() || BH <= 0 || BH > TC_SPLIT_MAX_BH) return 0;
    int R = (slots / BH - 1) / 2 + 2;   // phase 1 runs BH (1 + 2 (R - 2)) chains at once
    if (R > SPLIT_R_MAX) R = SPLIT_R_MAX;
    if (R > nc / TC_SPLIT_MIN_CHUNKS_PER_SEG) R = nc / TC_SPLIT_MIN_CHUNKS_PER_SEG;
    return R < 4 ? 0 : R;   // three segments lose in the backward (measured at B2 H16 T32K)
}

}  // namespace

cudaError_t split_prefix_launch(float* sbuf, int R, int BH, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(split_prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREFIX_SMEM);
    if (e != cudaSuccess) return e;
    TraceScope trace(K_SPLIT_PREFIX, s);
    split_prefix_kernel<<<BH * (D / 16), PREFIX_THREADS, PREFIX_SMEM, s>>>(sbuf, R);
    return cudaGetLastError();
}

int split_segments_for(int BH, int nc, int slots, bool have_buf) { return split_segments(BH, nc, slots, have_buf); }

// Segments of a piece's map computation: its 2 B*H chains (N and M, or B and A) become 2 B*H R chains over
// R segments, composed afterwards (R - 1 steps of gdn2_state_affine per map); as many as the CTA slots hold.
int map_segments_for(int BH, int nc, int slots, bool have_buf) {
    if (!have_buf || split_disabled() || BH <= 0 || BH > TC_SPLIT_MAX_BH) return 0;
    int R = slots / (2 * BH);
    if (R > SPLIT_R_MAX) R = SPLIT_R_MAX;
    if (R > nc / TC_SPLIT_MIN_CHUNKS_PER_SEG) R = nc / TC_SPLIT_MIN_CHUNKS_PER_SEG;
    return R < 2 ? 0 : R;
}

// The producers alone (with_maps: then per head two chains over the whole sequence, a piece of a longer one:
// N from a zero start with the inputs, M from the identity without input).
static cudaError_t fwd_pieces_launch(const ChunkFwdArgs& a, cudaStream_t s, bool with_maps) {
    const Dims& d = a.d;
    if (d.T == 0 || d.B * d.H == 0) return cudaSuccess;
    Maps maps;
    const void* ptrs[6] = {a.q, a.k, a.v, a.la, a.b, a.w};
    CUtensorMap* mp[6] = {&maps.q, &maps.k, &maps.v, &maps.la, &maps.b, &maps.w};
    for (int i = 0; i < 6; ++i)
        if (make_token_map(mp[i], ptrs[i], d.B, d.T, d.H) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    LaunchFacts lf{};
    cudaError_t e = launch_facts(chunk_fwd_kernel<false, false>, NT, SMEM_BYTES, &lf);
    if (e != cudaSuccess) return e;
    const int BH = d.B * d.H, nc = d.nchunks(), units = BH * nc, slots = lf.nsm * lf.occ;
    FwdParams p{};
    p.T = d.T; p.H = d.H; p.BH = BH; p.nc = nc;
    p.q = static_cast<const __nv_bfloat16*>(a.q); p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.la = static_cast<const __nv_bfloat16*>(a.la); p.b = static_cast<const __nv_bfloat16*>(a.b);
    p.wyimg = a.wy; p.flags = a.flags;
    if ((e = cudaMemsetAsync(a.flags, 0, (size_t)units * sizeof(unsigned int), s)) != cudaSuccess) return e;
    FwdParams pp = p;
    pp.ncons = 0;
    pp.nprod = units < slots ? units : slots;
    {
        TraceScope trace(K_CHUNK_FWD, s);
        chunk_fwd_kernel<false, false><<<pp.nprod, NT, SMEM_BYTES, s>>>(maps, pp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (!with_maps) return cudaSuccess;
    FwdParams pc = p;
    pc.phase = 5; pc.nprod = 0; pc.map_N = a.map_N; pc.map_M = a.map_M;
    const int R = map_segments_for(BH, nc, slots, a.sbuf != nullptr);
    pc.split_R = R;
    pc.sbuf = a.sbuf;
    const int ntasks = 2 * BH * (R ? R : 1);
    pc.ncons = ntasks < slots ? ntasks : slots;
    {
        TraceScope trace(K_CHUNK_FWD, s);
        chunk_fwd_kernel<false, false><<<pc.ncons, NT, SMEM_BYTES, s>>>(maps, pc);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (!R) return cudaSuccess;
    // compose the segments in order: N = M_{R-1} (... (M_1 N_0 + N_1) ...) + N_{R-1}, M = M_{R-1} ... M_1 M_0
    const size_t DD = (size_t)D * D;
    auto slot = [&](int j) { return a.sbuf + (size_t)j * BH * DD; };
    for (int s2 = 1; s2 < R; ++s2) {
        if ((e = state_affine_launch(slot(R + s2), slot(s2), s2 == 1 ? slot(0) : a.map_N, a.map_N, BH, D, D, s)) != cudaSuccess)
            return e;
        if ((e = state_affine_launch(slot(R + s2), nullptr, s2 == 1 ? slot(R) : a.map_M, a.map_M, BH, D, D, s)) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

cudaError_t chunk_fwd_map_launch(const ChunkFwdArgs& a, cudaStream_t s) { return fwd_pieces_launch(a, s, true); }
cudaError_t chunk_fwd_wy_launch(const ChunkFwdArgs& a, cudaStream_t s) { return fwd_pieces_launch(a, s, false); }

size_t chunk_fwd_split_bytes(int BH, int nc) {
    if (BH > TC_SPLIT_MAX_BH || nc < TC_SPLIT_MIN_CHUNKS_PER_SEG * 2) return 0;   // also the maps' segments (R >= 2)
    return (size_t)BH * SPLIT_MATS_PER_HEAD * TC_D * TC_D * sizeof(float);
}

cudaError_t chunk_fwd_launch(const ChunkFwdArgs& a, cudaStream_t s) {
    if (a.map_N && a.map_M) return chunk_fwd_map_launch(a, s);
    const Dims& d = a.d;
    if (d.T == 0 || d.B * d.H == 0) return cudaSuccess;
    // one scalar gate per head and token: the kernels built for it (the b and w maps are then never read)
    // (and one decay per head and token: the la map is then never read either)
    const bool sdec = a.beta && a.scalar_decay;
    void (*kern)(const Maps, const FwdParams) = !a.beta ? chunk_fwd_kernel<false, false>
                                                : (sdec ? chunk_fwd_kernel<true, true> : chunk_fwd_kernel<true, false>);
    Maps maps;
    const void* ptrs[6] = {a.q, a.k, a.v, sdec ? a.q : a.la, a.beta ? a.q : a.b, a.beta ? a.v : a.w};
    CUtensorMap* mp[6] = {&maps.q, &maps.k, &maps.v, &maps.la, &maps.b, &maps.w};
    for (int i = 0; i < 6; ++i)
        if (make_token_map(mp[i], ptrs[i], d.B, d.T, d.H) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    LaunchFacts lf{};
    cudaError_t e = launch_facts(kern, NT, SMEM_BYTES, &lf);
    if (e != cudaSuccess) return e;
    const int nsm = lf.nsm, coop = lf.coop, occ = lf.occ;
    const int BH = d.B * d.H, nc = d.nchunks();
    const int units = BH * nc;
    const int slots = nsm * occ;

    FwdParams p{};
    p.T = d.T; p.H = d.H; p.BH = BH; p.nc = nc;
    p.q = static_cast<const __nv_bfloat16*>(a.q); p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.la = static_cast<const __nv_bfloat16*>(a.la); p.b = static_cast<const __nv_bfloat16*>(a.b);
    p.beta = static_cast<const __nv_bfloat16*>(a.beta);
    p.S0 = a.S0; p.o = static_cast<__nv_bfloat16*>(a.o); p.ST = a.ST;
    p.states = a.states; p.deltas = a.deltas; p.wyimg = a.wy; p.flags = a.flags;
    if ((e = cudaMemsetAsync(a.flags, 0, (size_t)units * sizeof(unsigned int), s)) != cudaSuccess) return e;

    const int R = split_segments(BH, nc, slots, a.sbuf != nullptr);
    if (R) {   // producers, then the first segments and the segment maps, the prefix, then the other segments
        p.split_R = R;
        p.sbuf = a.sbuf;
        FwdParams pp = p;
        pp.ncons = 0;
        pp.nprod = units < slots ? units : slots;
        {
            TraceScope trace(K_CHUNK_FWD, s);
            if (!test_skip_producers()) {
                kern<<<pp.nprod, NT, SMEM_BYTES, s>>>(maps, pp);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
        }
        for (int phase = 1; phase <= 3; phase += 2) {
            FwdParams pc = p;
            pc.phase = phase;
            pc.nprod = 0;
            const int ntasks = phase == 1 ? BH * (1 + 2 * (R - 2)) : BH * (R - 1);
            pc.ncons = ntasks < slots ? ntasks : slots;
            {
                TraceScope trace(K_CHUNK_FWD, s);
                kern<<<pc.ncons, NT, SMEM_BYTES, s>>>(maps, pc);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
            if (phase == 1 && (e = split_prefix_launch(a.sbuf, R, BH, s)) != cudaSuccess) return e;
        }
        return cudaSuccess;
    }

    TraceScope trace(K_CHUNK_FWD, s);
    // Heads share the launch with the producers while the producers keep pace: per chunk step the
    // BH consumer chunks take about as long as BH WY units spread over the remaining CTAs.
    if (coop && !cooperative_disabled() && !test_skip_producers() && slots >= 2 && 16 * BH <= 9 * slots) {
        p.ncons = BH;
        p.nprod = slots - BH < units ? slots - BH : units;
        void* args[2] = {&maps, &p};
        e = cudaLaunchCooperativeKernel((const void*)kern, dim3(p.ncons + p.nprod), dim3(NT), args,
                                        SMEM_BYTES, s);
        if (e == cudaSuccess) return cudaSuccess;
        (void)cudaGetLastError();   // not launched: fall back to two launches
    }
    FwdParams pp = p;   // producers only
    pp.ncons = 0;
    pp.nprod = units < slots ? units : slots;
    if (!test_skip_producers()) {
        kern<<<pp.nprod, NT, SMEM_BYTES, s>>>(maps, pp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    FwdParams pc = p;   // consumers only; every flag is set when they start
    pc.ncons = BH;
    pc.nprod = 0;
    kern<<<BH, NT, SMEM_BYTES, s>>>(maps, pc);
    return cudaGetLastError();
}

cudaError_t chunk_fwd_take_errors(unsigned int* bits) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, g_fwd_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_fwd_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn2
