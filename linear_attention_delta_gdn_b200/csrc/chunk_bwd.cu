// chunk_bwd.cu -- gate-aware backward of the chunkwise Gated Delta Rule-2 operator
// on tcgen05 tensor cores (bf16 operands, fp32 TMEM accumulators).
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention" (arXiv
// abstract) names a gate-aware backward that keeps training parallel; the page
// prints no equations. The adjoint of the chunk form (see chunk_common.cuh), for
// one chunk with start state S, S' = Diag(gC) S + Kh^T Delta (Kh = gC*Kt), next-state gradient
// dS' and output gradient dO; dZ = Diag(gC) dS':
//   dDelta = Kh dS' + P^T dO = Kt dZ + P^T dO        (P = tril(Qt Kt^T))
//   dS     = dZ + Qt^T dO - Wm^T dDelta              -> gradient of the chunk-start state
//   dU     = T^T dDelta                              -> dv = dU*w, dw = dU*v
//   dP     = (dO Delta^T) * incl,  dA = -(dU Delta^T) * strict
//   dQt    = dO S^T + dP Kt,       dEt = -dU S^T + dA Kt
//   dKt    = dP^T Qt + dA^T Et,    dKh = Delta dS'^T  (so Delta dZ^T = gC*dKh)
// (dA uses T^T dT T^T = dU Delta^T, since dT = dDelta (U - Et S)^T = dDelta Delta^T (I + A)^T.)
// Gate chain through g = exp(G) (G = in-chunk cumsum of log_alpha):
//   dq = g*dQt;  dE = g*dEt;  dkK = dKt/g + (gC/g)*dKh;  db = dE*k;  dk = dkK + dE*b
//   dG_t = q*dq + e*dE - k*dkK   (e = b*k);  the last position also gets
//   E = rowsum(dZ * S) + sum_t Kh_t * dKh_t   (the dependence of S' on gC)
//   dlog_alpha_t = sum_{tau >= t} dG_tau + E
// Chunks without untame channels (chunk_common.cuh) carry dZ (reverse pass image), Kt and 1/g; chunks
// with untame channels carry dS', Kh and h = gC/g instead (Kt = k/g would overflow), and the pair terms of
// dq, dE and dkK of their untame channels (left out of the tensor-core products) are summed exactly on
// CUDA cores with exp(G_t - G_s) as a running product of alpha. The forward's WY image of the chunk
// records which channels are untame.
//
// One launch, two kinds of work, both reading the forward's per-chunk T and P tiles instead of
// redoing the solve:
//   reverse pass    one CTA per (batch, head) walks the chunks backwards carrying dS^T in TMEM
//                   (fp32); per chunk it writes dZ^T (dS'^T) as a bf16 image and then sets the chunk's
//                   ready flag (release);
//   chunk gradients every other CTA takes (head, chunk) units from a shared counter, in the
//                   order the reverse pass produces them, waits for the unit's flag (acquire) and
//                   computes every gradient of the chunk from the saved S, Delta (forward), dZ (dS'),
//                   dDelta (reverse pass), T, P, the inputs and dout. Reverse-pass CTAs join them
//                   once their head is done.
// With few heads this is one cooperative launch (all CTAs resident, so every wait ends; each wait is
// also bounded in time); otherwise the reverse pass and the gradients run as two launches.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

using namespace chunk;

__device__ unsigned int g_bwd_error;

// The backward runs 512 threads per CTA: 16 warps, four per TMEM lane quarter (warp w reads lanes
// 32 (w % 4) .. + 31; the four warps of a quarter, part = w / 4, split the columns of a read-out).
constexpr int BT = 512;
constexpr int BPARTS = BT / 128;
// The copy loops move whole images in 16-byte pieces per thread and the gate chain maps thread tid to
// (key channel tid % 128, token quarter tid / 128): both need exactly BT threads (checked at kernel entry).
static_assert(TC_STATE_BYTES % (16 * BT) == 0 && TC_DELTA_BYTES % (16 * BT) == 0 && BPARTS * 16 == 64,
              "BT-thread loops");

// The sum of the 8 bf16 values of a 16-byte piece of shared memory
__device__ __forceinline__ float row8_sum(const unsigned char* src) {
    const uint4 x = *reinterpret_cast<const uint4*>(src);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) s += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xFFFF0000u);
    return s;
}

// Copy a [128 lanes x NCOL] fp32 accumulator into a bf16 row tile of 128 rows (row = lane); each of
// the four warps of a lane quarter takes NCOL / 4 columns.
template <int NCOL>
__device__ __forceinline__ void tmem_rows_to_tile(uint32_t lane_base_col, unsigned char* dst, int warp, int lane) {
    static_assert(NCOL == 64, "16 columns per warp");
    const int row = 32 * tm_quarter(warp) + lane, c0 = (NCOL / BPARTS) * tm_part(warp);
    float v[16];
    tc::tmem_ld16(lane_base_col + c0, v);
    tc::tmem_wait_ld(v);
    tc::st_row8(dst, 128, row, (c0 >> 3), v);
    tc::st_row8(dst, 128, row, (c0 >> 3) + 1, v + 8);
}

// Exact pair terms of an untame channel i at token t (see the gate chain): with L = exp(G_t - G_s) as a
// running product of alpha (tables of alpha and of the raw q, fp32 [64 tokens][128 channels]),
//   fq = sum_{s<=t} dP_ts k_s L,  fe = sum_{s<t} dA_ts k_s L,
//   fk = sum_{t2>=t} (dP_{t2,t} q_t2 + dA_{t2,t} e_t2) exp(G_t2 - G_t)      (e = b*k)
// dP^T and dA^T are the bf16 tiles PP and TT (row s, column t); k and b the raw tiles KH and WW.
struct PairTerms {
    float fq, fe, fk;
};
__device__ __noinline__ PairTerms untame_pair_terms(const unsigned char* KH, const unsigned char* WW,
                                                    const unsigned char* PP, const unsigned char* TT,
                                                    const float* atab, const float* qtab, int i, int t) {
    float fq = 0.f, fe = 0.f, fk = 0.f, L = 1.f;
    for (int s = t; s >= 0; --s) {
        if (s < t) L *= atab[(s + 1) * 128 + i];
        const float ks = tc::ld_bf16(KH, tc::tile_off(C, s, i)) * L;
        fq += tc::ld_bf16(PP, tc::tile_off(C, s, t)) * ks;
        fe += tc::ld_bf16(TT, tc::tile_off(C, s, t)) * ks;   // dA_tt = 0
    }
    L = 1.f;
    for (int t2 = t; t2 < C; ++t2) {
        if (t2 > t) L *= atab[t2 * 128 + i];
        const float e2 = tc::ld_bf16(WW, tc::tile_off(C, t2, i)) * tc::ld_bf16(KH, tc::tile_off(C, t2, i));
        fk += (tc::ld_bf16(PP, tc::tile_off(C, t, t2)) * qtab[t2 * 128 + i] + tc::ld_bf16(TT, tc::tile_off(C, t, t2)) * e2) * L;
    }
    return PairTerms{fq, fe, fk};
}

// For a chunk with untame channels, before the gate chain: thread (channel i, token quarter qt) of an
// untame channel replaces, for its 16 tokens, G1 by dq = g G1 + fq, G2 by dE = g G2 + fe, G3 by fk and g by 1
// in TMEM, and Qt, Et by the raw q and e = b*k in QE, so that the gate chain's uniform formulas give the
// exact gradients (see untame_pair_terms). Whole warps (the TMEM accesses are warp-wide).
__device__ __noinline__ void untame_prepass(uint32_t lane_base, unsigned char* QE, const unsigned char* KH,
                                            const unsigned char* WW, const unsigned char* PP, const unsigned char* TT,
                                            const float* atab, const float* qtab, int i, int qt, bool untame,
                                            uint32_t tm_g1, uint32_t tm_g2, uint32_t tm_g3, uint32_t tm_gv) {
    const uint32_t col128 = (uint32_t)((i >> 6) * 128 * 128 + ((i & 7) << 1));
    const uint32_t chk = (uint32_t)((i & 63) >> 3);
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
        const int tq = 16 * qt + 8 * hh;
        float g1[8], g2[8], g3[8], gv[8];
        tc::tmem_ld8(lane_base + tm_g1 + tq, g1);
        tc::tmem_ld8(lane_base + tm_g2 + tq, g2);
        tc::tmem_ld8(lane_base + tm_g3 + tq, g3);
        tc::tmem_ld8(lane_base + tm_gv + tq, gv);
        tc::tmem_wait_ld(g1, g2, g3, gv);
        if (untame) {
#pragma unroll 1
            for (int u = 0; u < 8; ++u) {
                const int t = tq + u;
                const PairTerms f = untame_pair_terms(KH, WW, PP, TT, atab, qtab, i, t);
                g1[u] = gv[u] * g1[u] + f.fq;
                g2[u] = gv[u] * g2[u] + f.fe;
                g3[u] = f.fk;
                gv[u] = 1.f;
                const uint32_t sw = (uint32_t)t * 128 + ((chk ^ ((uint32_t)t & 7)) << 4);
                tc::st_bf16(QE, col128 + C * 128 + sw, qtab[t * 128 + i]);                          // q
                tc::st_bf16(QE, col128 + sw, tc::ld_bf16(WW, tc::tile_off(C, t, i)) *
                                                 tc::ld_bf16(KH, tc::tile_off(C, t, i)));           // e = b*k
            }
        }
        tc::tmem_st8(lane_base + tm_g1 + tq, g1);
        tc::tmem_st8(lane_base + tm_g2 + tq, g2);
        tc::tmem_st8(lane_base + tm_g3 + tq, g3);
        tc::tmem_st8(lane_base + tm_gv + tq, gv);
    }
    tc::tmem_wait_st();
}

// Gradient-unit prep, thread = (key channel i = tid % 128, token quarter qt = tid / 128: tokens
// 16 qt .. 16 qt + 15):
//   reads  log_alpha (KT), k (KH), b (QE rows 0..63), q (QE rows 64..127)
//   writes Et -> QE rows 0..63, Qt -> QE rows 64..127, Kt -> KT (zero when channel i is untame; k stays in
//   KH); g[t][i] = exp(G) and r[t][i] go to TMEM at tmem_g and tmem_r (lane i, column t) for the gate chain,
//   r = 1/g, or h = exp(G_C - G) when the chunk has untame channels (khm). Quarter sums of log_alpha are
//   exchanged through qsum (fp32 [4][128]). Returns gC = exp(G_C) of channel i. Contains one __syncthreads.
__device__ __forceinline__ float grad_prep(unsigned char* QE, const unsigned char* KH, unsigned char* KT,
                                           float* qsum, int tid, uint32_t tmem_g, uint32_t tmem_r, bool untame,
                                           bool khm) {
    const int i = tid & 127, qt = tid >> 7;
    const uint32_t col64 = (uint32_t)((i >> 6) * 64 * 128 + ((i & 7) << 1));
    const uint32_t col128 = (uint32_t)((i >> 6) * 128 * 128 + ((i & 7) << 1));
    const uint32_t chunk = (uint32_t)((i & 63) >> 3);
    float la[16];
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const uint32_t t = (uint32_t)(16 * qt + u);
        la[u] = tc::ld_bf16(KT, col64 + t * 128 + ((chunk ^ (t & 7)) << 4));
        if (u & 1) s1 += la[u]; else s0 += la[u];
    }
    qsum[qt * 128 + i] = s0 + s1;
    __syncthreads();   // also: every log_alpha is read before Kt overwrites it
    float G = 0.f, tot = 0.f;
#pragma unroll
    for (int q = 0; q < BPARTS; ++q) {
        const float x = qsum[q * 128 + i];
        tot += x;
        if (q < qt) G += x;
    }
    const float shift = khm ? tot : 0.f;   // r = exp(shift - G)
    const float igC = khm ? 1.f / fast_exp(tot) : 1.f;   // 1/g = r * igC (used on tame channels only)
    float gvals[16], rvals[16];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float kk[8], bb[8], qq[8];
        uint32_t o64[8], o128[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t t = (uint32_t)(16 * qt + 8 * half + u);
            const uint32_t sw = t * 128 + ((chunk ^ (t & 7)) << 4);
            o64[u] = col64 + sw;
            o128[u] = col128 + sw;
            kk[u] = tc::ld_bf16(KH, o64[u]);
            bb[u] = tc::ld_bf16(QE, o128[u]);
            qq[u] = tc::ld_bf16(QE, o128[u] + C * 128);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            G += la[8 * half + u];
            const float g = fast_exp(G), r = fast_exp(shift - G), ig = r * igC;
            gvals[8 * half + u] = g;
            rvals[8 * half + u] = r;
            tc::st_bf16(QE, o128[u], g * bb[u] * kk[u]);                  // Et
            tc::st_bf16(QE, o128[u] + C * 128, g * qq[u]);                // Qt
            tc::st_bf16(KT, o64[u], untame ? 0.f : kk[u] * ig);           // Kt = k/g
        }
    }
    tc::tmem_st16(tmem_g + 16 * qt, gvals);
    tc::tmem_st16(tmem_r + 16 * qt, rvals);
    tc::tmem_wait_st();
    return fast_exp(tot);
}

constexpr uint32_t TILE_C = 64 * 64 * 2;   // bytes of a 64 x 64 bf16 tile

// Barrier block shared by both kinds of work (above every tile of either layout):
// 4 mbarriers (load, mma, k, b), TMEM base, abort flag, next unit (2 ints), prefetch mbarrier at +48,
// "this unit has an untame channel" flag at +56.
constexpr uint32_t OFF_BARS = 229888;
constexpr uint32_t SMEM_BYTES_ALL = 229952 + 1024;

struct BwdMaps {
    CUtensorMap q, k, v, la, b, w, dout, dq, dk, db, dla, dv, dw;
};
struct BwdParams {
    int T, H, BH, nc;
    const __nv_bfloat16 *q_raw, *la_raw;   // raw inputs, read directly only for untame channels
    const __nv_bfloat16* beta;       // [B, T, H] erase and write gates b = w = beta 1 (kernels instantiated for
    __nv_bfloat16* dbeta;            // them), and their gradient sum_i db_ti + sum_j dw_tj; else null
    __nv_bfloat16* dla_s;            // one decay per head and token (la_raw [B, T, H]): its gradient [B, T, H]
    int nrev;                        // CTAs [0, nrev) run the reverse pass of head blockIdx.x
    int join;                        // reverse-pass CTAs take gradient units afterwards
    int grad;                        // this launch computes gradient units
    const float* dST;
    float* dS0;
    __nv_bfloat16 *dv, *dw;
    const unsigned char* states;     // chunk-start state images
    const unsigned char* deltas;     // Delta^T images of the forward
    const unsigned char* tp;         // WY images (T | P | Wm)
    unsigned char* dstates;          // dS'^T images
    unsigned char* ddeltas;          // dDelta^T images
    unsigned int* flags;             // [BH, nc] dS' ready flags (zero at launch)
    unsigned int* counter;           // [0]: next gradient unit, [1]: abort word (zero at launch)
    int split_R;                     // > 0: the reverse pass of a head is cut into split_R segments
    int phase;                       // with split_R: 1 (last segment, segment maps) or 3 (the other segments);
                                     // 5: the reverse maps of every head's whole sequence (map_B, map_A)
    float* sbuf;                     // with split_R: per head, segment end gradients, then the maps B and A
    float *map_B, *map_A;            // phase 5: [BH][D][D] each
};

// ---- reverse-pass tasks
// Without a split, task t walks every chunk of head t backwards from dST (zero if none). A long sequence with
// few heads is cut into R segments as in the forward; with E_s the gradient at the end of segment s (E_{R-1} =
// dST), walking a segment backwards is an affine map E_{s-1} = A_s E_s + B_s, where B_s is the result from a
// zero end gradient and A_s (d_k x d_k) the one from an identity end gradient without output gradients (dO =
// 0). Phase 1 walks the last segment for real (its start gradient is E_{R-2}) and, for s = 1 .. R-2, B_s and
// A_s as separate tasks; the forward's prefix kernel then forms E_{R-3} .. E_0 (its slot k holds E_{R-1-k},
// its maps those of segment R-1-k); phase 3 walks segments 0 .. R-2 for real, next to the gradient workers.
struct RevTask {
    int head, c_hi, c_lo;    // chunks c_hi down to c_lo
    const float* start;      // end gradient [D][D] (row = key), or null: zero, or identity when ident
    bool ident, zero_do;     // A_s: identity start, no output gradient
    bool real;               // the real chain: dZ and dDelta images, ready flags
    float* fin;              // where the gradient at chunk c_lo's start goes, or null
};
constexpr int SPLIT_R_MAX = 8;
constexpr size_t SPLIT_MATS_PER_HEAD = (SPLIT_R_MAX - 1) + 2 * (SPLIT_R_MAX - 2);
__host__ __device__ inline int seg_begin(int s, int nc, int R) { return (int)((long long)s * nc / R); }
__device__ __forceinline__ float* rsplit_mat(const BwdParams& p, int head, int kind, int k) {   // 0: E, 1: B, 2: A
    const int R = p.split_R;
    const int idx = kind == 0 ? k - 1 : (kind == 1 ? (R - 1) + (k - 1) : (R - 1) + (R - 2) + (k - 1));
    if (!GDN2_IN(g_bwd_error, idx >= 0 && idx < (int)SPLIT_MATS_PER_HEAD && head < p.BH)) return nullptr;
    return p.sbuf + ((size_t)head * SPLIT_MATS_PER_HEAD + idx) * D * D;
}
__device__ __forceinline__ int rev_task_count(const BwdParams& p) {
    if (p.phase == 5) return 2 * p.BH * (p.split_R ? p.split_R : 1);
    if (!p.split_R) return p.BH;
    return p.phase == 1 ? p.BH * (1 + 2 * (p.split_R - 2)) : p.BH * (p.split_R - 1);
}
__device__ RevTask rev_task_at(const BwdParams& p, int t) {
    RevTask k{};
    k.head = t % p.BH;
    const size_t hd = (size_t)k.head * D * D;
    if (p.phase == 5) {   // the whole sequence as one piece: B from a zero end gradient, A from the identity
        if (p.split_R) {      // per segment j: B_j into slot j, A_j into slot R + j (slot-major: [slot][BH][D][D])
            const int R = p.split_R, j = t / p.BH, s2 = j < R ? j : j - R;
            k.c_lo = seg_begin(s2, p.nc, R);
            k.c_hi = (s2 == R - 1 ? p.nc : seg_begin(s2 + 1, p.nc, R)) - 1;
            if (j >= R) { k.ident = true; k.zero_do = true; }
            k.fin = p.sbuf + ((size_t)j * p.BH + k.head) * D * D;
            return k;
        }
        k.c_hi = p.nc - 1; k.c_lo = 0;
        if (t < p.BH) {
            k.fin = p.map_B + hd;
        } else {
            k.ident = true; k.zero_do = true; k.fin = p.map_A + hd;
        }
        return k;
    }
    if (!p.split_R) {
        k.c_hi = p.nc - 1; k.c_lo = 0; k.start = p.dST ? p.dST + hd : nullptr; k.real = true;
        k.fin = p.dS0 ? p.dS0 + hd : nullptr;
        return k;
    }
    const int R = p.split_R, j = t / p.BH;
    auto seg_lo = [&](int s2) { return seg_begin(s2, p.nc, R); };
    auto seg_hi = [&](int s2) { return (s2 == R - 1 ? p.nc : seg_begin(s2 + 1, p.nc, R)) - 1; };
    if (p.phase == 1) {
        if (j == 0) {   // the last segment, for real, from dST; its start gradient is E_{R-2} = slot 1
            k.c_hi = seg_hi(R - 1); k.c_lo = seg_lo(R - 1); k.start = p.dST ? p.dST + hd : nullptr; k.real = true;
            k.fin = rsplit_mat(p, k.head, 0, 1);
        } else if (j <= R - 2) {   // B of segment s2 = R-1-j into slot j
            const int s2 = R - 1 - j;
            k.c_hi = seg_hi(s2); k.c_lo = seg_lo(s2); k.fin = rsplit_mat(p, k.head, 1, j);
        } else {   // A of segment s2 into slot j - (R-2)
            const int kk = j - (R - 2), s2 = R - 1 - kk;
            k.c_hi = seg_hi(s2); k.c_lo = seg_lo(s2); k.ident = true; k.zero_do = true;
            k.fin = rsplit_mat(p, k.head, 2, kk);
        }
    } else {   // segment s2 = j (0 .. R-2) for real from E_{s2} = slot R-1-s2
        const int s2 = j;
        k.c_hi = seg_hi(s2); k.c_lo = seg_lo(s2); k.start = rsplit_mat(p, k.head, 0, R - 1 - s2); k.real = true;
        k.fin = (s2 == 0 && p.dS0) ? p.dS0 + hd : nullptr;
    }
    return k;
}
// Gradient units in the order the reverse pass produces them. Without a split: chunks from the last, heads
// inside. With a split (phase 3): the last segment's units first (ready from phase 1), then the other
// segments' units interleaved by position from their ends. Returns false for an index that names no unit
// (segments of unequal length).
__device__ __forceinline__ int unit_slots(const BwdParams& p) {
    if (!p.split_R) return p.BH * p.nc;
    const int R = p.split_R, last = p.nc - seg_begin(R - 1, p.nc, R);
    int lmax = 0;
    for (int s2 = 0; s2 < R - 1; ++s2) {
        const int l = seg_begin(s2 + 1, p.nc, R) - seg_begin(s2, p.nc, R);
        lmax = l > lmax ? l : lmax;
    }
    return p.BH * last + p.BH * (R - 1) * lmax;
}
__device__ __forceinline__ bool unit_at_unchecked(const BwdParams& p, int u, int* head, int* c) {
    if (!p.split_R) {
        *c = p.nc - 1 - u / p.BH;
        *head = u % p.BH;
        return true;
    }
    const int R = p.split_R, lo_last = seg_begin(R - 1, p.nc, R), nlast = p.BH * (p.nc - lo_last);
    if (u < nlast) {
        *c = p.nc - 1 - u / p.BH;
        *head = u % p.BH;
        return true;
    }
    const int v = u - nlast, per = p.BH * (R - 1), jpos = v / per, rem = v % per, s2 = rem / p.BH;
    *head = rem % p.BH;
    const int lo = seg_begin(s2, p.nc, R), hi = seg_begin(s2 + 1, p.nc, R) - 1;
    *c = hi - jpos;
    return *c >= lo;
}
__device__ __forceinline__ bool unit_at(const BwdParams& p, int u, int* head, int* c) {
    return unit_at_unchecked(p, u, head, c) && GDN2_IN(g_bwd_error, *head >= 0 && *head < p.BH && *c >= 0 && *c < p.nc);
}
// mbarrier parities carried across the units a CTA works on
struct Phases {
    uint32_t load = 0, mma = 0, k = 0, b = 0, pre = 0;
};
// The next gradient unit of a CTA, handed between units through shared memory (OFF_BARS + 40):
// [0] unit index, [1] nonzero once its S, T and dS'^T images are being prefetched (flag acquired).
struct NextUnit {
    int unit, prefetched;
};

// Kh of a chunk with untame channels, in place of its Kt tile (bf16 [64 x 128] row tile): Kt * gC on the
// tame columns, and on the untame ones (bits of msk) the values that the forward wrote to the image's Kh tile
// (kh_img, global memory). BT threads, 2 pieces of 8 columns each.
__device__ __noinline__ void kh_from_kt(unsigned char* KT, const unsigned char* kh_img, const float* gC, uint4 msk,
                                        int tid) {
    const unsigned int mw[4] = {msk.x, msk.y, msk.z, msk.w};
#pragma unroll 1
    for (int e = 0; e < 2; ++e) {
        const int idx = tid + BT * e, row = idx >> 4, g = idx & 15;
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

// ====================================================================== reverse state pass

namespace rs {
// Qt, Kt, dout, Wm, gC and the mask alternate between two buffers by chunk parity, so the next chunk's
// tiles can land while this chunk's MMAs read the current ones; P has one buffer. Qt, Kt (Kh), Wm, P, gC
// and the mask come from the forward's WY image.
constexpr uint32_t OFF_QQ = 0;           // 2 x Qt (64 rows), at +0 / +16384
constexpr uint32_t OFF_KT0 = 49152;      // Kt or Kh (even chunks)
constexpr uint32_t OFF_DO0 = 65536;      // dout (even chunks)
constexpr uint32_t OFF_WW0 = 81920;      // Wm (even chunks)
constexpr uint32_t OFF_ST = 98304;       // dZ^T or dS'^T (bf16)
constexpr uint32_t OFF_DT = 131072;      // dDelta^T (bf16)
constexpr uint32_t OFF_PP = 147456;      // P
constexpr uint32_t OFF_DO1 = 163840;     // dout (odd chunks)
constexpr uint32_t OFF_WW1 = 180224;     // Wm (odd chunks)
constexpr uint32_t OFF_KT1 = 196608;     // Kt or Kh (odd chunks)
constexpr uint32_t OFF_GC = 212992;      // 2 x fp32 gC[128] (by parity)
constexpr uint32_t OFF_MASK = 214016;    // 2 x untame-channel mask (4 words, by parity)
constexpr uint32_t TM_S = 0, TM_D = 128;
constexpr uint32_t LOAD_BYTES = 4 * 64 * 128 * 2 + TILE_C + 512 + 16;   // Qt, Kt, dout, Wm, P, gC, mask
}  // namespace rs
static_assert(rs::OFF_MASK + 32 <= OFF_BARS, "reverse-pass layout lies below the barrier block");

__device__ void run_reverse(const BwdMaps& m, const BwdParams& p, unsigned char* sm, uint32_t tmem,
                            const RevTask& task, Phases& ph) {
    using namespace rs;
    unsigned char* STt = sm + OFF_ST;
    unsigned char* DT = sm + OFF_DT;
    unsigned char* PP = sm + OFF_PP;
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* bar_mma = bar_load + 1;
    int* abort_flag = reinterpret_cast<int*>(sm + OFF_BARS + 36);
    auto QQ = [&](int c) { return sm + OFF_QQ + (c & 1) * TILE_64x128; };
    auto KT = [&](int c) { return sm + ((c & 1) ? OFF_KT1 : OFF_KT0); };
    auto DO = [&](int c) { return sm + ((c & 1) ? OFF_DO1 : OFF_DO0); };
    auto WW = [&](int c) { return sm + ((c & 1) ? OFF_WW1 : OFF_WW0); };
    auto GC = [&](int c) { return reinterpret_cast<float*>(sm + OFF_GC + (c & 1) * 512); };
    auto MASK = [&](int c) { return sm + OFF_MASK + (c & 1) * 16; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int headi = task.head, c_hi = task.c_hi, c_lo = task.c_lo;
    const bool zero_do = task.zero_do, real = task.real;
    const int h = headi % p.H, b = headi / p.H;
    const size_t head = (size_t)headi;
    const int nc = p.nc;
    const uint32_t lane_base = tmem + ((uint32_t)(tm_quarter(warp) * 32) << 16);
    const int jrow = 32 * tm_quarter(warp) + lane, cpart = 32 * tm_part(warp);      // lane row, column quarter

    // chunk c's tiles arrive on one barrier phase, issued in three groups as their buffers free up
    // dout, Qt, Kt, Wm, gC, mask (buffers of this parity are free): issued by lane 0 of warps 0-5 at once
    // (a task without output gradients, zero_do, needs neither dout, nor Qt and P)
    auto issue_first = [&](int c) {
        if (lane != 0 || warp > 5) return;
        const unsigned char* img = p.tp + (head * nc + c) * TC_WY_BYTES;
        switch (warp) {
        case 0:
            tc::mbar_arrive_expect_tx(bar_load, zero_do ? LOAD_BYTES - 2 * 64 * 128 * 2 - TILE_C : LOAD_BYTES);
            if (!zero_do) tma_tile(DO(c), C, 0, &m.dout, b, h, c * C, bar_load);
            break;
        case 1: if (!zero_do) tc::bulk_load(QQ(c), img + TC_WY_QT, 64 * 128 * 2, bar_load); break;
        case 2: tc::bulk_load(KT(c), img + TC_WY_KT, 64 * 128 * 2, bar_load); break;
        case 3: tc::bulk_load(WW(c), img + TC_WY_WM, 64 * 128 * 2, bar_load); break;
        case 4: tc::bulk_load(GC(c), img + TC_WY_GC, 512, bar_load); break;
        default: tc::bulk_load(MASK(c), img + TC_WY_MASK, 16, bar_load); break;
        }
    };
    auto issue_p = [&](int c) {   // after the MMAs that read P
        tc::bulk_load(PP, p.tp + (head * nc + c) * TC_WY_BYTES + TILE_C, TILE_C, bar_load);
    };
    issue_first(c_hi);
    if (tid == 0 && !zero_do) issue_p(c_hi);

    {   // the gradient at the end of the range: lane j holds column j of the start matrix (dST, zero or I)
        const int j = jrow;
        float v[32];
#pragma unroll 1
        for (int i0 = cpart; i0 < cpart + 32; i0 += 32) {
#pragma unroll
            for (int u = 0; u < 32; ++u)
                v[u] = task.start ? task.start[(i0 + u) * D + j] : (task.ident && i0 + u == j ? 1.f : 0.f);
            tc::tmem_st32(lane_base + TM_S + i0, v);
        }
        tc::tmem_wait_st();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    const uint32_t sST = tc::smem_u32(STt), sDT = tc::smem_u32(DT), sPP = tc::smem_u32(PP);
    constexpr uint32_t ID_N1a = tc::idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_N1b = tc::idesc_bf16(128, 64, true, true);
    constexpr uint32_t ID_N2a = tc::idesc_bf16(128, 128, true, true);
    constexpr uint32_t ID_N2b = tc::idesc_bf16(128, 128, false, true, true);

    auto wait_mma = [&]() {
        if (!tc::mbar_wait(bar_mma, ph.mma)) { atomicExch(abort_flag, 1); atomicOr(&g_bwd_error, 1u); }
        ph.mma ^= 1;
        tc::tc_fence_after();
    };
    auto sync_for_mma = [&]() {
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
    };

    int unreleased = -1;   // chunk whose dS' image is written but whose flag is not yet set
    for (int c = c_hi; c >= c_lo; --c) {
        const uint32_t sQQ = tc::smem_u32(QQ(c)), sKT = tc::smem_u32(KT(c)), sDO = tc::smem_u32(DO(c)),
                       sWW = tc::smem_u32(WW(c));
        if (!tc::mbar_wait(bar_load, ph.load)) { atomicExch(abort_flag, 1); atomicOr(&g_bwd_error, 2u); }
        ph.load ^= 1;
        // the other parity's buffers were last read by chunk c + 1, whose MMAs are complete
        if (c > c_lo) issue_first(c - 1);

        const float* sGC = GC(c);   // Qt, Kt, gC and the mask came with the forward's WY image
        const uint4 msk = *reinterpret_cast<const uint4*>(MASK(c));
        const bool khm = (msk.x | msk.y | msk.z | msk.w) != 0u;   // the same on every thread
        if (khm)   // untame channels in this chunk: Kh replaces Kt, dS' replaces dZ
            kh_from_kt(KT(c), p.tp + (head * nc + c) * TC_WY_BYTES + TC_WY_KH, sGC, msk, tid);
        // the fp32 gradient scaled in place, dZ^T = dS'^T Diag(gC) (the first term of dS^T), and a bf16 copy of
        // dZ^T, or of dS'^T (taken before the scaling) in a chunk with untame channels: the operand of dDelta
        // and the image for the gradient units
        {
            const int j = jrow;
            float v[32];
#pragma unroll 1
            for (int i0 = cpart; i0 < cpart + 32; i0 += 32) {
                tc::tmem_ld32(lane_base + TM_S + i0, v);
                tc::tmem_wait_ld(v);
                if (khm) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) tc::st_row8(STt, D, j, (i0 >> 3) + g, v + 8 * g);
                }
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] *= sGC[i0 + u];
                tc::tmem_st32(lane_base + TM_S + i0, v);
                if (!khm) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) tc::st_row8(STt, D, j, (i0 >> 3) + g, v + 8 * g);
                }
            }
            tc::tmem_wait_st();
        }
        sync_for_mma();

        // dDelta^T = dZ^T Kt^T (= dS'^T Kh^T) + dO^T P (commit) ;  dS^T = dZ^T + dO^T Qt (continues below)
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_D, tc::desc_k(sST, D, 0, kk), tc::desc_k(sKT, C, 0, kk), ID_N1a, kk > 0);
            if (!zero_do) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_D, tc::desc_mn(sDO, C, 0, kk), tc::desc_mn(sPP, C, 0, kk), ID_N1b, 1);
            }
            tc::mma_commit(bar_mma);
            if (!zero_do) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_S, tc::desc_mn(sDO, C, 0, kk), tc::desc_mn(sQQ, C, 0, kk), ID_N2a, 1);
            }
        }
        // the previous chunk's dZ image stores have drained: publish it while the MMAs run
        if (real && tid == 32 && unreleased >= 0 && !*abort_flag) tc::flag_release(p.flags + head * nc + unreleased, 1u);
        if (real) {   // this chunk's dZ^T (dS'^T) image for the gradient units (plain stores, published one chunk later)
            uint4* dst = reinterpret_cast<uint4*>(p.dstates + (head * nc + c) * TC_STATE_BYTES);
            const uint4* src = reinterpret_cast<const uint4*>(STt);
#pragma unroll
            for (int i = 0; i < (int)(TC_STATE_BYTES / 16 / BT); ++i) dst[tid + BT * i] = src[tid + BT * i];
            unreleased = c;
        }
        wait_mma();
        if (tid == 0 && c > c_lo && !zero_do) issue_p(c - 1);
        tmem_rows_to_tile<64>(lane_base + TM_D, DT, warp, lane);   // dDelta^T rows
        sync_for_mma();
        if (real) {   // dDelta^T image for the gradient units (published with the dZ^T image)
            uint4* dst = reinterpret_cast<uint4*>(p.ddeltas + (head * nc + c) * TC_DELTA_BYTES);
            const uint4* src = reinterpret_cast<const uint4*>(DT);
#pragma unroll
            for (int i = 0; i < (int)(TC_DELTA_BYTES / 16 / BT); ++i) dst[tid + BT * i] = src[tid + BT * i];
        }

        // dS^T -= dDelta^T Wm
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_k(sDT, D, 0, kk), tc::desc_mn(sWW, C, 0, kk), ID_N2b, 1);
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        if (*abort_flag) {   // let the next chunk's loads land before leaving
            if (tid == 0) {
                atomicExch(p.counter + 1, 1u);   // gradient units of this head will never be ready
                if (c > c_lo) (void)tc::mbar_wait(bar_load, ph.load);
            }
            break;
        }
    }
    if (tid == 32 && unreleased >= 0 && !*abort_flag) tc::flag_release(p.flags + head * nc + unreleased, 1u);

    if (task.fin) {   // the gradient at the start of the range, fin[i][j] from dS^T (lane j): dS0 or a segment's
        const int j = jrow;
        float v[32];
#pragma unroll 1
        for (int i0 = cpart; i0 < cpart + 32; i0 += 32) {
            tc::tmem_ld32(lane_base + TM_S + i0, v);
            tc::tmem_wait_ld(v);
#pragma unroll
            for (int u = 0; u < 32; ++u) task.fin[(i0 + u) * D + j] = v[u];
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
}

// ====================================================================== per-chunk gradients

namespace cg {
constexpr uint32_t OFF_QE = 0;           // rows 0..63: b -> Et, rows 64..127: q -> Qt
constexpr uint32_t OFF_KH = 32768;       // k
constexpr uint32_t OFF_KT = 49152;       // log_alpha -> Kt
constexpr uint32_t OFF_DU = 65536;       // [128 x 128]: rows 0..63 dout (later staged dq), rows 64..127
                                         // v -> -dU (later staged dlog_alpha): one N = 128 operand
constexpr uint32_t OFF_WW = 98304;       // w, later b (reloaded)
constexpr uint32_t OFF_ST = 114688;      // S^T image (chunk start)
constexpr uint32_t OFF_DS = 147456;      // dS'^T image
constexpr uint32_t OFF_DT = 180224;      // Delta^T [128 x 64] (forward image), later staged dk
constexpr uint32_t OFF_DDT = 196608;     // dDelta^T [128 x 64] (reverse-pass image), later staged db
constexpr uint32_t OFF_PP = 212992;      // prep scratch, then dP^T [64 x 64]; with TT: dw staging, and
constexpr uint32_t OFF_TT = 221184;      // T, later dA^T   [dP^T | dA^T] as one N = 128 operand
constexpr uint32_t OFF_SDBW = 229376;    // one scalar gate per token: the dw tile's row sums (64 floats)
// TMEM columns (M=64 accumulators use lanes 0-15 of each 32-lane quarter)
constexpr uint32_t TM_AP = 0,      // dP^T (M=64)
    TM_W = 64,                     // dA^T (M=64, 64 columns)
    TM_DU = 320,                   // dU (M=64, 128 columns), later G1 = dQt^T, G2 = dEt^T
    TM_G1 = 320, TM_G2 = 384, TM_G3 = 256, TM_G4 = 192,   // G3 = dKt^T (P and A paths), G4 = (Delta dS'^T)^T = dKh^T
    TM_GV = 448,                   // g[t] = exp(G) per key channel
    TM_HV = 128;                   // r[t] = 1/g, or exp(G_C - G) in a chunk with untame channels
constexpr uint32_t LOAD_GATE = 4 * 64 * 128 * 2;                             // b, q, k, log_alpha: the prep's
constexpr uint32_t LOAD_REST = 3 * 64 * 128 * 2 + (uint32_t)TC_DELTA_BYTES;   // v, w, dout, Delta^T
constexpr uint32_t LOAD_PRE = (uint32_t)TC_STATE_BYTES + TILE_C;     // S image, T (dS'^T: cp.async)
static_assert(OFF_TT + TILE_C <= OFF_SDBW && OFF_SDBW + 64 * 4 <= OFF_BARS, "gradient-unit layout below the barriers");
}  // namespace cg

// Gradients of chunk c of head `headi`; returns false if a bounded wait gave up. `prefetched`: the S, T
// and dS'^T images of this unit were requested by the previous unit (S, T on the prefetch barrier).
// Lane 0 of warp 9 takes the CTA's next unit from the counter while this one runs and acquires its flag
// while the G MMAs run; once this unit has finished with the S^T, T and dS'^T tiles, the next unit's
// images are requested into them. The next unit is published in *nxt.
// BETA (b = w = beta 1): the b rows of QE and the w tile hold the gate of each token, written by the threads
// at the start of the unit (no b or w tiles are loaded and b is not reloaded); dw and db are not stored, their
// row sums (over the value and key channels) go out as dbeta. SDEC (with BETA; one decay per head and token):
// the log_alpha tile is written the same way, and dlog_alpha goes out as its row sums.
template <bool BETA, bool SDEC>
__device__ bool grad_unit(const BwdMaps& m, const BwdParams& p, unsigned char* sm, uint32_t tmem, int headi, int c,
                          Phases& ph, bool prefetched, NextUnit* nxt) {
    using namespace cg;
    unsigned char* QE = sm + OFF_QE;
    unsigned char* KH = sm + OFF_KH;
    unsigned char* KT = sm + OFF_KT;
    unsigned char* DU = sm + OFF_DU;
    unsigned char* WW = sm + OFF_WW;
    unsigned char* STt = sm + OFF_ST;
    unsigned char* DS = sm + OFF_DS;
    unsigned char* DT = sm + OFF_DT;
    unsigned char* DDT = sm + OFF_DDT;
    unsigned char* TT = sm + OFF_TT;
    unsigned char* PP = sm + OFF_PP;
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* bar_mma = bar_load + 1;
    uint64_t* bar_rest = bar_load + 2;
    uint64_t* bar_b = bar_load + 3;
    uint64_t* bar_pre = reinterpret_cast<uint64_t*>(sm + OFF_BARS + 48);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, H = p.H, nc = p.nc;
    const int units = unit_slots(p);
    const int h = headi % H, b = headi / H;
    const size_t head = (size_t)headi;
    const int t0 = c * C;
    const int L = min(C, T - t0);
    const CUtensorMap *mq = &m.q, *mk = &m.k, *mv = &m.v, *mla = &m.la, *mb = &m.b, *mw = &m.w, *mdo = &m.dout;
    const CUtensorMap *mdq = &m.dq, *mdk = &m.dk, *mdb = &m.db, *mdla = &m.dla;

    // the chunk's untame channels, as recorded by the forward (a chunk with any takes the Kh / dS' form); loaded
    // first, used after the tile loads
    const uint4 msk = *reinterpret_cast<const uint4*>(p.tp + (head * nc + c) * TC_WY_BYTES + TC_WY_MASK);
    bool ok = true;
    int next_unit = units;    // lane 0 of warp 9: the CTA's next unit (its atomic returns while this unit runs)
    // BETA: the gates of rows tid / 16 and tid / 16 + 32 (bf16 bits, 0 past the end of the sequence), loaded
    // first and written out as b and w rows below
    uint32_t bet16[2] = {0u, 0u}, la16[2] = {0u, 0u};
    if constexpr (BETA) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int row = (tid >> 4) + 32 * x;
            if (t0 + row < T) {
                bet16[x] = __bfloat16_as_ushort(p.beta[((size_t)b * T + t0 + row) * H + h]);
                if (SDEC) la16[x] = __bfloat16_as_ushort(p.la_raw[((size_t)b * T + t0 + row) * H + h]);
            }
        }
    }
    // The loads are issued by lane 0 of several warps at once (a TMA issue takes ~100 cycles); a barrier
    // phase cannot complete before the arrival that carries its expected bytes. Two groups: the prep's
    // inputs (b, q, k, log_alpha, into tiles no output is staged in) go out at once; the rest (v, w, dout,
    // Delta^T, and S^T, T unless prefetched) after thread 0 has seen the previous unit's output stores read
    // DU, DT and DDT, and land while the prep runs.
    // (*nxt is rewritten only after the next barriers: every thread has read it by then.)
    if (lane == 0) {
        switch (warp) {
        case 0:
            tc::mbar_arrive_expect_tx(bar_load, LOAD_GATE - (BETA ? 64u * 128u * 2u : 0u) - (SDEC ? 64u * 128u * 2u : 0u));
            if (!BETA) tma_tile(QE, 2 * C, 0, mb, b, h, t0, bar_load);
            break;
        case 1: tma_tile(QE, 2 * C, C, mq, b, h, t0, bar_load); break;
        case 2: tma_tile(KH, C, 0, mk, b, h, t0, bar_load); break;
        case 3: if (!SDEC) tma_tile(KT, C, 0, mla, b, h, t0, bar_load); break;
        case 9: next_unit = (int)atomicAdd(p.counter, 1u); break;   // first needed at the G MMAs
        default: break;
        }
    }
    if (tid == 0) {
        if (!prefetched && !tc::flag_wait(p.flags + head * nc + c, 1u)) {   // dS'^T of this chunk: the reverse pass
            ok = false;
            atomicOr(&g_bwd_error, 8u);
            atomicExch(p.counter + 1, 1u);
        }
        tc::bulk_wait_read();   // the previous unit's dq, dlog_alpha stores have read DU
    }
    if (lane == 0 && (warp == 1 || warp == 2)) tc::bulk_wait_read();   // its dk, db stores: DT, DDT
    if constexpr (BETA) {   // rows r and r + 32 of b (QE rows 0..63) and w (WW): 8 copies of beta per piece
        const int r = tid >> 4, panel = (tid >> 3) & 1, chunk = tid & 7;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int row = r + 32 * x;
            const uint32_t v16 = bet16[x] * 0x10001u;
            const uint4 v = make_uint4(v16, v16, v16, v16);
            *reinterpret_cast<uint4*>(QE + panel * (2 * C * 128) + row * 128 + chunk * 16) = v;
            *reinterpret_cast<uint4*>(WW + panel * (C * 128) + row * 128 + chunk * 16) = v;
            if (SDEC) {
                const uint32_t l16 = la16[x] * 0x10001u;
                *reinterpret_cast<uint4*>(KT + panel * (C * 128) + row * 128 + chunk * 16) =
                    make_uint4(l16, l16, l16, l16);
            }
        }
    }
    __syncthreads();   // orders thread 0's acquire and its wait before the loads and copies below
    if (lane == 0) {
        const unsigned char* src = p.tp + (head * nc + c) * TC_WY_BYTES;   // T | P | Wm
        switch (warp) {
        case 4:
            tc::mbar_arrive_expect_tx(bar_rest, (prefetched ? LOAD_REST : LOAD_REST + LOAD_PRE) -
                                                    (BETA ? 64u * 128u * 2u : 0u));
            tma_tile(DU, 2 * C, C, mv, b, h, t0, bar_rest);
            break;
        case 5: if (!BETA) tma_tile(WW, C, 0, mw, b, h, t0, bar_rest); break;
        case 6: tma_tile(DU, 2 * C, 0, mdo, b, h, t0, bar_rest); break;
        case 7:
            tc::bulk_load(DT, p.deltas + (head * nc + c) * TC_DELTA_BYTES, (uint32_t)TC_DELTA_BYTES, bar_rest);
            break;
        case 8:
            if (!prefetched) {
                tc::bulk_load(STt, p.states + (head * nc + c) * TC_STATE_BYTES, (uint32_t)TC_STATE_BYTES, bar_rest);
                tc::bulk_load(TT, src, TILE_C, bar_rest);
            }
            break;
        default: break;
        }
    }
    {   // the reverse pass's images of this chunk: dS'^T (unless prefetched) and dDelta^T
        if (!prefetched) {
            const unsigned char* src = p.dstates + (head * nc + c) * TC_STATE_BYTES;
#pragma unroll
            for (int i = 0; i < (int)(TC_STATE_BYTES / 16 / BT); ++i)
                tc::cp_async16_cg(DS + 16 * (tid + BT * i), src + 16 * (tid + BT * i));
        }
        const unsigned char* src = p.ddeltas + (head * nc + c) * TC_DELTA_BYTES;
#pragma unroll
        for (int i = 0; i < (int)(TC_DELTA_BYTES / 16 / BT); ++i)
            tc::cp_async16_cg(DDT + 16 * (tid + BT * i), src + 16 * (tid + BT * i));
        tc::cp_async_commit();
    }
    const uint32_t lane_base = tmem + ((uint32_t)(tm_quarter(warp) * 32) << 16);
    const int jrow = 32 * tm_quarter(warp) + lane, cpart = 32 * tm_part(warp);      // lane row, column quarter
    (void)jrow;
    ok = tc::mbar_wait(bar_load, ph.load) && ok;   // the prep's inputs
    ph.load ^= 1;
    auto wait_mma = [&]() {
        ok = tc::mbar_wait(bar_mma, ph.mma) && ok;
        ph.mma ^= 1;
        tc::tc_fence_after();
    };
    auto sync_for_mma = [&]() {
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
    };

    const uint32_t sQE = tc::smem_u32(QE), sKT = tc::smem_u32(KT),
                   sDU = tc::smem_u32(DU), sST = tc::smem_u32(STt),
                   sDS = tc::smem_u32(DS), sDT = tc::smem_u32(DT), sDDT = tc::smem_u32(DDT),
                   sTT = tc::smem_u32(TT), sPP = tc::smem_u32(PP);

    // ---- factors (G kept in TMEM)
    const bool khm = (msk.x | msk.y | msk.z | msk.w) != 0u;   // the same on every thread
    const int ich = tid & 127;
    const bool untame = ((ich < 64 ? (ich < 32 ? msk.x : msk.y) : (ich < 96 ? msk.z : msk.w)) >> (ich & 31)) & 1u;
    const float gC = grad_prep(QE, KH, KT, reinterpret_cast<float*>(PP), tid, lane_base + TM_GV, lane_base + TM_HV,
                               untame, khm);   // PP: scratch
    ok = tc::mbar_wait(bar_rest, ph.k) && ok;   // the rest of the unit's tiles, loaded during the prep
    ph.k ^= 1;
    if (prefetched) {
        ok = tc::mbar_wait(bar_pre, ph.pre) && ok;
        ph.pre ^= 1;
    }
    tc::cp_async_wait_all();
    sync_for_mma();

    // ---- dU = T^T dDelta (M=64)
    if (tid == 0) {
        tc::tc_fence_after();
        constexpr uint32_t id = tc::idesc_bf16(64, 128, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + TM_DU, tc::desc_mn(sTT, C, 0, kk), tc::desc_k(sDDT, D, 0, kk), id, kk > 0);
        tc::mma_commit(bar_mma);
    }
    wait_mma();
    {   // dv = dU*w -> DDT, dw = dU*v -> PP|TT (bf16 row tiles for TMA stores; the dU MMA has read T
        // and dDelta^T, the prep its scratch); -dU replaces v
        const int t = m64_row(warp, lane);
        float v[32];
        const int c0 = cpart;
        tc::tmem_ld32(lane_base + TM_DU + c0, v);
        tc::tmem_wait_ld(v);
        if (lane < 16) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float x[8], y[8];
                const float* d = v + 8 * g;
                tc::ld_row8(WW, C, t, (c0 >> 3) + g, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = d[e] * x[e];
                tc::st_row8(DDT, C, t, (c0 >> 3) + g, y);            // dv
                tc::ld_row8(DU, 2 * C, C + t, (c0 >> 3) + g, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = d[e] * x[e];
                tc::st_row8(PP, C, t, (c0 >> 3) + g, y);             // dw (PP and TT form one 64 x 128 tile)
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = -d[e];
                tc::st_row8(DU, 2 * C, C + t, (c0 >> 3) + g, y);     // -dU over v
            }
        }
    }
    sync_for_mma();
    // store dv (lane 0 of warp 1) and dw (warp 2; rows past the end of the sequence are skipped), and bring b
    // back for the gate chain (warp 3; w is consumed), while thread 0 issues the MMAs below
    if (lane == 0 && (warp == 1 || (!BETA && (warp == 2 || warp == 3)))) {
        if (warp == 3) {
            tc::mbar_arrive_expect_tx(bar_b, 64 * 128 * 2);
            tma_tile(WW, C, 0, mb, b, h, t0, bar_b);
        } else {
            const CUtensorMap* map = warp == 1 ? &m.dv : &m.dw;
            unsigned char* tile = warp == 1 ? DDT : PP;
            tc::tma_store_4d(map, 0, h, t0, b, tile);
            tc::tma_store_4d(map, 64, h, t0, b, tile + C * 128);
            tc::bulk_commit();
        }
    }

    // ---- dP^T = Delta dO^T (M=64), dA^T = -Delta dU^T (M=64)
    if (tid == 0) {
        tc::tc_fence_after();
        constexpr uint32_t id_pa = tc::idesc_bf16(64, 128, true, false);   // the tile holds -dU: no negation
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // [dP^T | dA^T] (TM_AP, TM_W adjacent) as one N = 128 product over DU
            tc::mma_bf16(tmem + TM_AP, tc::desc_mn(sDT, D, 0, kk), tc::desc_k(sDU, 2 * C, 0, kk), id_pa, kk > 0);
        tc::mma_commit(bar_mma);
    }
    if (lane == 0 && (warp == 1 || warp == 2))
        tc::bulk_wait_read();   // the dv, dw stores have read their tiles (DDT, TT, PP are overwritten below)
    if constexpr (BETA) {   // row t of the dw tile (PP | TT) summed over the value channels, while the MMAs run
        const int t = tid >> 3, part = tid & 7;
        float sdw = row8_sum(PP + t * 128 + part * 16) + row8_sum(PP + C * 128 + t * 128 + part * 16);
        sdw += __shfl_xor_sync(0xffffffffu, sdw, 1);
        sdw += __shfl_xor_sync(0xffffffffu, sdw, 2);
        sdw += __shfl_xor_sync(0xffffffffu, sdw, 4);
        if (part == 0) reinterpret_cast<float*>(sm + OFF_SDBW)[t] = sdw;
    }
    wait_mma();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    {   // M=64 accumulators: rows s = 16 q + lane (lanes < 16); the warps of a quarter take 16 columns each
        const int s_ = m64_row(warp, lane), c0 = 16 * tm_part(warp);
        float v[16];
        tc::tmem_ld16(lane_base + TM_AP + c0, v);
        tc::tmem_wait_ld(v);
        if (lane < 16) {
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = (s_ <= c0 + u) ? v[u] : 0.f;   // dP[t][s], t >= s
#pragma unroll
            for (int g = 0; g < 2; ++g) tc::st_row8(PP, C, s_, (c0 >> 3) + g, v + 8 * g);
        }
        tc::tmem_ld16(lane_base + TM_W + c0, v);
        tc::tmem_wait_ld(v);
        if (lane < 16) {
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = (s_ < c0 + u) ? v[u] : 0.f;    // dA[t][s], t > s
#pragma unroll
            for (int g = 0; g < 2; ++g) tc::st_row8(TT, C, s_, (c0 >> 3) + g, v + 8 * g);
        }
    }
    sync_for_mma();

    // ---- G1 = dQt^T = S dO^T + Kt^T dP^T ; G2 = dEt^T = -S dU^T + Kt^T dA^T
    //      G3 = Qt^T dP + Et^T dA ;        G4 = dZ Delta^T          (all [key channel i][token t])
    // G1 and G2 (adjacent in TMEM) share their A operands: [G1 | G2] = S [dO; -dU]^T + Kt^T [dP^T | dA^T]
    // as N = 128 products (DU rows; PP and TT panels).
    if (tid == 0) {
        tc::tc_fence_after();
        constexpr uint32_t id_mk = tc::idesc_bf16(128, 64, true, false);
        constexpr uint32_t id_mk2 = tc::idesc_bf16(128, 128, true, false);
        constexpr uint32_t id_mm = tc::idesc_bf16(128, 64, true, true);
        constexpr uint32_t id_mm2 = tc::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            tc::mma_bf16(tmem + TM_G1, tc::desc_mn(sST, D, 0, kk), tc::desc_k(sDU, 2 * C, 0, kk), id_mk2, kk > 0);
            tc::mma_bf16(tmem + TM_G4, tc::desc_mn(sDS, D, 0, kk), tc::desc_mn(sDT, D, 0, kk), id_mm, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            tc::mma_bf16(tmem + TM_G1, tc::desc_mn(sKT, C, 0, kk), tc::desc_mn(sPP, C, 0, kk), id_mm2, 1);
            tc::mma_bf16(tmem + TM_G3, tc::desc_mn(sQE, 2 * C, C, kk), tc::desc_k(sPP, C, 0, kk), id_mk, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + TM_G3, tc::desc_mn(sQE, 2 * C, 0, kk), tc::desc_k(sTT, C, 0, kk), id_mk, 1);
        tc::mma_commit(bar_mma);
    }

    // rowsum(dZ * S) (or gC rowsum(dS' * S)) for key channel i over this quarter's value channels (both images
    // hold row j = value channel)
    const int i = tid & 127, qt = tid >> 7;
    float Epart = 0.f;
    {
        float e1 = 0.f, e2 = 0.f;
#pragma unroll 8
        for (int j = 32 * qt; j < 32 * qt + 32; j += 2) {
            e1 += tc::ld_bf16(DS, tc::tile_off(D, j, i)) * tc::ld_bf16(STt, tc::tile_off(D, j, i));
            e2 += tc::ld_bf16(DS, tc::tile_off(D, j + 1, i)) * tc::ld_bf16(STt, tc::tile_off(D, j + 1, i));
        }
        Epart = (e1 + e2) * (khm ? gC : 1.f);
    }
    if (warp == 9 && lane == 0) {   // while the G MMAs run: the CTA's next unit, published at the next barrier
        if (*reinterpret_cast<volatile unsigned int*>(p.counter + 1)) next_unit = units;   // a CTA gave up
        int ready = 0;
        int nh = 0, nc_ = 0;
        if (next_unit < units && unit_at(p, next_unit, &nh, &nc_))   // acquire: usually set long ago
            ready = tc::ld_acquire(p.flags + (size_t)nh * nc + nc_) == 1u;
        nxt->unit = next_unit;
        nxt->prefetched = ready;
    }
    wait_mma();
    if (!BETA) {
        ok = tc::mbar_wait(bar_b, ph.b) && ok;
        ph.b ^= 1;
    }

    // ---- untame channels: their pair terms are summed exactly below, from alpha and the raw q of the chunk
    // (fp32 [64 tokens][128 channels] tables over the S^T and dS'^T tiles, which the G MMAs and the rowsum
    // have finished with; the next unit's images are fetched into them only after pass 1)
    const bool slow = khm;
    float* atab = reinterpret_cast<float*>(STt);
    float* qtab = reinterpret_cast<float*>(DS);
    if (slow) {
        __syncthreads();   // every thread's rowsum has read S^T and dS'^T
        for (int x = tid; x < C * D; x += BT) {
            const int tau = x >> 7, ch = x & 127;
            float al = 1.f, qq = 0.f;
            if (tau < L) {
                const size_t off = tok_off(b, t0 + tau, h, T, H, D) + ch;
                al = fast_exp(__bfloat162float(SDEC ? p.la_raw[((size_t)b * T + t0 + tau) * H + h] : p.la_raw[off]));
                qq = __bfloat162float(p.q_raw[off]);
            }
            atab[x] = al;
            qtab[x] = qq;
        }
        __syncthreads();
        untame_prepass(lane_base, QE, KH, WW, PP, TT, atab, qtab, i, qt, untame, TM_G1, TM_G2, TM_G3, TM_GV);
        __syncthreads();   // every exact sum has read dP^T (PP) before the gate chain's exchange reuses it
    }

    // ---- gate chain, thread = (key channel i, token quarter qt: tokens 16 qt .. 16 qt + 15). Pass 1: dq,
    // dk, db and dG_t; partial sums of E and dG are exchanged between the quarters (in the consumed dP^T
    // tile). Pass 2: dlog_alpha_t = sum_{tau >= t} dG_tau + E. Results go to bf16 row tiles (dq -> DU rows
    // 0..63, dk -> DT, db -> DDT, dlog_alpha -> DU rows 64..127), stored by TMA.
    const uint32_t col64 = (uint32_t)((i >> 6) * 64 * 128 + ((i & 7) << 1));
    const uint32_t col128 = (uint32_t)((i >> 6) * 128 * 128 + ((i & 7) << 1));
    const uint32_t chk = (uint32_t)((i & 63) >> 3);
    // tame channels: dkK = (G3 a + G4) r with r = 1/g, a = 1 (G4 = Delta dZ^T), or r = gC/g, a = 1/gC (G4 = dKh)
    const float a_ = khm ? (untame ? 0.f : 1.f / gC) : 1.f;
    float dG[16];
    float dGsum = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {   // two halves of 8 tokens (keeps the TMEM read-outs in registers)
        const int tq = 16 * qt + 8 * hh;
        float g1[8], g2[8], g3[8], g4[8], gv[8], hv[8];
        tc::tmem_ld8(lane_base + TM_G1 + tq, g1);
        tc::tmem_ld8(lane_base + TM_G2 + tq, g2);
        tc::tmem_ld8(lane_base + TM_G3 + tq, g3);
        tc::tmem_ld8(lane_base + TM_G4 + tq, g4);
        tc::tmem_ld8(lane_base + TM_GV + tq, gv);
        tc::tmem_ld8(lane_base + TM_HV + tq, hv);
        tc::tmem_wait_ld(g1, g2, g3, g4, gv, hv);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = tq + u;
            const uint32_t sw = (uint32_t)t * 128 + ((chk ^ ((uint32_t)t & 7)) << 4);
            const float kk = tc::ld_bf16(KH, col64 + sw);
            const float bb = tc::ld_bf16(WW, col64 + sw);
            const float g = gv[u], r = hv[u];
            const float qv = tc::ld_bf16(QE, col128 + C * 128 + sw);   // Qt (raw q on an untame channel)
            const float et = tc::ld_bf16(QE, col128 + sw);             // Et (raw e on an untame channel)
            const float dq = g * g1[u], dE = g * g2[u];
            const float dkK = g3[u] * (untame ? 1.f : r * a_) + g4[u] * r;   // dKt/g + (gC/g) dKh
            const float dGt = qv * g1[u] + et * g2[u] - kk * dkK;
            dG[8 * hh + u] = dGt;
            dGsum += dGt;
            Epart += kk * r * g4[u];                                        // Kh dKh (= Kt Delta dZ^T)
            tc::st_bf16(DU, col128 + sw, dq);                               // dq
            tc::st_bf16(DT, col64 + sw, dkK + dE * bb);                     // dk
            tc::st_bf16(DDT, col64 + sw, dE * kk);                          // db
        }
    }
    float* xch = reinterpret_cast<float*>(PP);                      // [2 quantities][4 quarters][128]
    xch[(0 * BPARTS + qt) * 128 + i] = Epart;
    xch[(1 * BPARTS + qt) * 128 + i] = dGsum;
    tc::fence_async_smem();   // every read of S^T and dS'^T (G MMAs, rowsum) precedes the prefetch below, and
                              // dq, dk, db (final after pass 1) are visible to the tensor stores
    __syncthreads();          // also orders warp 9's acquire before every thread's copy of the next dS'^T
    if (lane == 0 && warp < (BETA ? 2 : 3)) {   // dq, dk, db (lane 0 of warps 0, 1, 2) go out while pass 2 runs; rows past
                                   // the end of the sequence are skipped
        const CUtensorMap* map = warp == 0 ? mdq : (warp == 1 ? mdk : mdb);
        const unsigned char* tile = warp == 0 ? DU : (warp == 1 ? DT : DDT);
        const uint32_t panel = warp == 0 ? 2 * C * 128 : C * 128;   // second 64 channels
        tc::tma_store_4d(map, 0, h, t0, b, tile);
        tc::tma_store_4d(map, 64, h, t0, b, tile + panel);
        tc::bulk_commit();
    }
    if constexpr (BETA) {   // dbeta_t: row t of the db tile (DDT) summed over the key channels, plus the dw sum
        const int t = tid >> 3, part = tid & 7;
        float sdb = row8_sum(DDT + t * 128 + part * 16) + row8_sum(DDT + C * 128 + t * 128 + part * 16);
        sdb += __shfl_xor_sync(0xffffffffu, sdb, 1);
        sdb += __shfl_xor_sync(0xffffffffu, sdb, 2);
        sdb += __shfl_xor_sync(0xffffffffu, sdb, 4);
        if (part == 0 && t < L)
            p.dbeta[((size_t)b * T + t0 + t) * H + h] =
                __float2bfloat16(sdb + reinterpret_cast<const float*>(sm + OFF_SDBW)[t]);
    }
    int nxt_head = 0, nxt_c = 0;
    if (nxt->prefetched) unit_at(p, nxt->unit, &nxt_head, &nxt_c);
    if (tid == 0 && nxt->prefetched) {   // S^T and T of the next unit into the tiles this unit has finished with
        const size_t nu = (size_t)nxt_head * nc + nxt_c;
        tc::mbar_arrive_expect_tx(bar_pre, LOAD_PRE);
        tc::bulk_load(STt, p.states + nu * TC_STATE_BYTES, (uint32_t)TC_STATE_BYTES, bar_pre);
        tc::bulk_load(TT, p.tp + nu * TC_WY_BYTES, TILE_C, bar_pre);
    }
    if (nxt->prefetched) {
        const size_t nu = (size_t)nxt_head * nc + nxt_c;
        const unsigned char* src = p.dstates + nu * TC_STATE_BYTES;
#pragma unroll
        for (int i = 0; i < (int)(TC_STATE_BYTES / 16 / BT); ++i)
            tc::cp_async16_cg(DS + 16 * (tid + BT * i), src + 16 * (tid + BT * i));
        tc::cp_async_commit();
    }
    float E = 0.f, suffix = 0.f;                                    // suffix: dG of the later quarters
#pragma unroll
    for (int q = 0; q < BPARTS; ++q) {
        E += xch[(0 * BPARTS + q) * 128 + i];
        if (q > qt) suffix += xch[(1 * BPARTS + q) * 128 + i];
    }
#pragma unroll
    for (int u = 15; u >= 0; --u) {
        const uint32_t t = (uint32_t)(16 * qt + u);
        suffix += dG[u];
        tc::st_bf16(DU, col128 + C * 128 + t * 128 + ((chk ^ (t & 7)) << 4), suffix + E);   // dlog_alpha
    }
    tc::fence_async_smem();
    __syncthreads();
    if (!SDEC && tid == 0) {   // dlog_alpha; the next unit waits for the stores' reads before it reuses their tiles
        tc::tma_store_4d(mdla, 0, h, t0, b, DU + C * 128);
        tc::tma_store_4d(mdla, 64, h, t0, b, DU + C * 128 + 2 * C * 128);
        tc::bulk_commit();
    }
    if constexpr (SDEC) {   // one decay per token: row t of the dlog_alpha tile (DU rows 64..127) summed
        const int t = tid >> 3, part = tid & 7;
        float sla = row8_sum(DU + C * 128 + t * 128 + part * 16) + row8_sum(DU + 3 * C * 128 + t * 128 + part * 16);
        sla += __shfl_xor_sync(0xffffffffu, sla, 1);
        sla += __shfl_xor_sync(0xffffffffu, sla, 2);
        sla += __shfl_xor_sync(0xffffffffu, sla, 4);
        if (part == 0 && t < L) p.dla_s[((size_t)b * T + t0 + t) * H + h] = __float2bfloat16(sla);
    }
    if (!ok) atomicOr(&g_bwd_error, 4u);
    tc::tc_fence_before();
    ok = __syncthreads_and(ok) != 0;   // the same answer on every thread: the CTA leaves the loop together
    tc::tc_fence_after();
    return ok;
}

template <bool BETA, bool SDEC>
__global__ void __launch_bounds__(BT, 1) chunk_bwd_kernel(const __grid_constant__ BwdMaps maps, const BwdParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays in the shared window
    const int tid = threadIdx.x, warp = tid >> 5;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(sm + OFF_BARS + 32);
    int* abort_flag = reinterpret_cast<int*>(sm + OFF_BARS + 36);
    NextUnit* nxt = reinterpret_cast<NextUnit*>(sm + OFF_BARS + 40);
    if (blockDim.x != BT) {   // the index arithmetic assumes BT threads: refuse any other launch shape
        if (tid == 0) atomicOr(&g_bwd_error, 16u);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) tc::mbar_init(&bars[i], 1);
        tc::mbar_init(reinterpret_cast<uint64_t*>(sm + OFF_BARS + 48), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base_ptr, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_base_ptr;
    Phases ph;
    const bool reverse = (int)blockIdx.x < p.nrev;
    if (reverse) {   // the CTA's reverse-pass tasks (one each in a launch with gradient workers)
        const int ntasks = rev_task_count(p);
        for (int t = blockIdx.x; t < ntasks && !*abort_flag; t += p.nrev) {
            const RevTask task = rev_task_at(p, t);
            if (GDN2_IN(g_bwd_error, task.head >= 0 && task.head < p.BH && 0 <= task.c_lo && task.c_lo <= task.c_hi &&
                                         task.c_hi < p.nc))
                run_reverse(maps, p, sm, tmem, task, ph);
        }
    }
    if (p.grad && (!reverse || p.join) && !*abort_flag) {
        const int units = unit_slots(p);
        if (tid == 0) {   // stop taking units once any CTA of the launch has given up
            nxt->unit = *reinterpret_cast<volatile unsigned int*>(p.counter + 1) ? units : (int)atomicAdd(p.counter, 1u);
            nxt->prefetched = 0;
        }
        __syncthreads();
        int u = nxt->unit;
        bool pre = false;
        while (u < units) {
            // units in the order the reverse pass produces them (unit_at)
            int c = 0, headi = 0;
            if (!unit_at(p, u, &headi, &c)) {   // an index that names no unit: take the next one
                if (tid == 0) {
                    nxt->unit = *reinterpret_cast<volatile unsigned int*>(p.counter + 1) ? units : (int)atomicAdd(p.counter, 1u);
                    nxt->prefetched = 0;
                }
                __syncthreads();
                u = nxt->unit;
                pre = false;
                __syncthreads();
                continue;
            }
            if (!grad_unit<BETA, SDEC>(maps, p, sm, tmem, headi, c, ph, pre, nxt)) {
                // a bounded wait gave up: let a prefetch in flight land before leaving
                if (tid == 0 && nxt->prefetched) (void)tc::mbar_wait(reinterpret_cast<uint64_t*>(sm + OFF_BARS + 48), ph.pre);
                tc::cp_async_wait_all();
                break;
            }
            u = nxt->unit;   // written by thread 0 before the unit's last barrier
            pre = nxt->prefetched != 0;
        }
        if ((tid & 31) == 0 && warp < 3) tc::bulk_wait_read();   // the last unit's output stores have read their tiles
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t chunk_bwd_launch(const ChunkBwdArgs& a, cudaStream_t s) {
    const Dims& d = a.d;
    if (d.T == 0 || d.B * d.H == 0) return cudaSuccess;
    // one scalar gate per head and token: the kernels built for it (the b, w, db and dw maps are never used)
    // (and one decay per head and token: the la and dla maps are then never used either)
    const bool beta = a.beta != nullptr && !(a.map_A && a.map_B);
    const bool sdec = beta && a.scalar_decay;
    void (*kern)(const BwdMaps, const BwdParams) = !beta ? chunk_bwd_kernel<false, false>
                                                   : (sdec ? chunk_bwd_kernel<true, true> : chunk_bwd_kernel<true, false>);
    BwdMaps maps;
    const void* ptrs[13] = {a.q, a.k, a.v, sdec ? a.q : a.la, beta ? a.q : a.b, beta ? a.v : a.w, a.dout, a.dq, a.dk,
                            beta ? a.dq : a.db, sdec ? a.dq : a.dla, a.dv, beta ? a.dv : a.dw};
    CUtensorMap* mp[13] = {&maps.q, &maps.k, &maps.v, &maps.la, &maps.b, &maps.w, &maps.dout,
                           &maps.dq, &maps.dk, &maps.db, &maps.dla, &maps.dv, &maps.dw};
    if (a.map_A && a.map_B)   // no gradient units run: their output maps only need a valid address
        for (int i = 7; i < 13; ++i) ptrs[i] = a.dout;
    for (int i = 0; i < 13; ++i)
        if (make_token_map(mp[i], ptrs[i], d.B, d.T, d.H) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    LaunchFacts lf{};
    cudaError_t e = launch_facts(kern, BT, SMEM_BYTES_ALL, &lf);
    if (e != cudaSuccess) return e;
    const int nsm = lf.nsm, coop = lf.coop, occ = lf.occ;
    const int BH = d.B * d.H, nc = d.nchunks();
    const int units = BH * nc;
    const int slots = nsm * occ;

    BwdParams p{};
    p.T = d.T; p.H = d.H; p.BH = BH; p.nc = nc;
    p.q_raw = static_cast<const __nv_bfloat16*>(a.q); p.la_raw = static_cast<const __nv_bfloat16*>(a.la);
    if (beta) {
        p.beta = static_cast<const __nv_bfloat16*>(a.beta);
        p.dbeta = static_cast<__nv_bfloat16*>(a.dbeta);
        if (sdec) p.dla_s = static_cast<__nv_bfloat16*>(a.dla);
    }
    p.dST = a.dST; p.dS0 = a.dS0;
    p.dv = static_cast<__nv_bfloat16*>(a.dv); p.dw = static_cast<__nv_bfloat16*>(a.dw);
    p.states = a.states; p.deltas = a.deltas; p.tp = a.tp; p.dstates = a.dstates; p.ddeltas = a.ddeltas;
    p.flags = a.flags; p.counter = a.flags + units;
    if ((e = cudaMemsetAsync(a.flags, 0, ((size_t)units + 2) * sizeof(unsigned int), s)) != cudaSuccess) return e;

    if (a.map_A && a.map_B) {   // reverse maps only: the reverse pass of every head (or segment) twice, no gradients
        BwdParams pm = p;
        pm.phase = 5; pm.grad = 0; pm.join = 0; pm.map_A = a.map_A; pm.map_B = a.map_B;
        const int R = map_segments_for(BH, nc, slots, a.sbuf != nullptr);
        pm.split_R = R;
        pm.sbuf = a.sbuf;
        const int ntasks = 2 * BH * (R ? R : 1);
        pm.nrev = ntasks < slots ? ntasks : slots;
        {
            TraceScope trace(K_CHUNK_BWD, s);
            kern<<<pm.nrev, BT, SMEM_BYTES_ALL, s>>>(maps, pm);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (!R) return cudaSuccess;
        // compose from the last segment: B = A_0 (... (A_{R-2} B_{R-1} + B_{R-2}) ...) + B_0, A = A_0 A_1 ... A_{R-1}
        const size_t DD = (size_t)D * D;
        auto slot = [&](int j) { return a.sbuf + (size_t)j * BH * DD; };
        for (int s2 = R - 2; s2 >= 0; --s2) {
            const bool first = s2 == R - 2;
            if ((e = state_affine_launch(slot(R + s2), slot(s2), first ? slot(R - 1) : a.map_B, a.map_B, BH, D, D, s)) !=
                cudaSuccess)
                return e;
            if ((e = state_affine_launch(slot(R + s2), nullptr, first ? slot(2 * R - 1) : a.map_A, a.map_A, BH, D, D, s)) !=
                cudaSuccess)
                return e;
        }
        return cudaSuccess;
    }
    const int R = split_segments_for(BH, nc, slots, a.sbuf != nullptr);
    if (R) {   // the last segments and the segment maps, the prefix, then the other segments with the gradients
        p.split_R = R;
        p.sbuf = a.sbuf;
        BwdParams p1 = p;
        p1.phase = 1; p1.grad = 0; p1.join = 0;
        const int n1 = BH * (1 + 2 * (R - 2));
        p1.nrev = n1 < slots ? n1 : slots;
        {
            TraceScope trace(K_CHUNK_BWD, s);
            kern<<<p1.nrev, BT, SMEM_BYTES_ALL, s>>>(maps, p1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if ((e = split_prefix_launch(a.sbuf, R, BH, s)) != cudaSuccess) return e;
        BwdParams p3 = p;
        p3.phase = 3;
        const int n3 = BH * (R - 1);
        TraceScope trace(K_CHUNK_BWD, s);
        if (coop && !cooperative_disabled() && n3 < slots) {
            p3.nrev = n3; p3.join = 1; p3.grad = 1;
            void* args[2] = {&maps, &p3};
            e = cudaLaunchCooperativeKernel((const void*)kern, dim3(slots), dim3(BT), args, SMEM_BYTES_ALL, s);
            if (e == cudaSuccess) return cudaSuccess;
            (void)cudaGetLastError();
        }
        BwdParams pr = p3;
        pr.nrev = n3 < slots ? n3 : slots; pr.join = 0; pr.grad = 0;
        kern<<<pr.nrev, BT, SMEM_BYTES_ALL, s>>>(maps, pr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        BwdParams pg = p3;
        pg.nrev = 0; pg.join = 0; pg.grad = 1;
        kern<<<units < slots ? units : slots, BT, SMEM_BYTES_ALL, s>>>(maps, pg);
        return cudaGetLastError();
    }

    TraceScope trace(K_CHUNK_BWD, s);
    // Every head's reverse pass plus at least one gradient worker resident at once: one launch.
    if (coop && !cooperative_disabled() && BH < slots) {
        p.nrev = BH; p.join = 1; p.grad = 1;
        void* args[2] = {&maps, &p};
        e = cudaLaunchCooperativeKernel((const void*)kern, dim3(slots), dim3(BT), args, SMEM_BYTES_ALL, s);
        if (e == cudaSuccess) return cudaSuccess;
        (void)cudaGetLastError();   // not launched: fall back to two launches
    }
    BwdParams pr = p;   // reverse pass only
    pr.nrev = BH; pr.join = 0; pr.grad = 0;
    kern<<<BH, BT, SMEM_BYTES_ALL, s>>>(maps, pr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    BwdParams pg = p;   // gradient units only; every flag is set when they start
    pg.nrev = 0; pg.join = 0; pg.grad = 1;
    kern<<<units < slots ? units : slots, BT, SMEM_BYTES_ALL, s>>>(maps, pg);
    return cudaGetLastError();
}

cudaError_t chunk_bwd_take_errors(unsigned int* bits) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, g_bwd_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn2
