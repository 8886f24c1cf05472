// chunk_common.cuh -- pieces shared by the chunkwise tensor-core kernels
// (bf16 inputs, d_k = d_v = 128, chunk C = 64, one warpgroup of 128 threads).
//
// Chunk algebra ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
// Attention", arXiv abstract and README "Hardware-efficient Training" bullet:
// a chunkwise WY algorithm with the channel-wise decay absorbed into asymmetric
// erase factors). Per head and chunk of C tokens starting from state S:
//   G_t = sum_{tau<=t} log_alpha_tau (inclusive, within the chunk), g = exp(G), gC = g_{C-1}
//   Et = g*(b*k)      erase factor scaled forward
//   Kt = k/g          key scaled backward
//   Qt = g*q,  Kh = (gC/g)*k = gC*Kt,  U = w*v
//   A  = strictly_lower(Et Kt^T),  T = (I + A)^{-1},  Wm = T Et,  Ut = T U
//   Delta = Ut - Wm S;   O = Qt S + tril(Qt Kt^T) Delta;   S' = Diag(gC) S + Kh^T Delta
// The kernels apply the last step as S' = Diag(gC) (S + Kt^T Delta) (Kh = gC*Kt), scaling the
// fp32 accumulator after the contraction, so no Kh tile is formed.
// Rows past the end of the sequence are zero-filled by TMA: they give zero
// factors, a flat cumulative decay and an identity block of T, so a ragged
// last chunk needs no special case except masked stores.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {
namespace chunk {

constexpr int D = 128;        // d_k = d_v
constexpr int C = 64;         // chunk length
constexpr int NT = 256;       // threads per CTA (two warpgroups)
// TMEM access: warp w reads lane quarter (w % 4), i.e. lanes 32 (w % 4) .. +31; the two warps of a
// quarter (w and w + 4) split the columns of each read-out between them (part = w / 4).
__device__ __forceinline__ int tm_quarter(int warp) { return warp & 3; }
__device__ __forceinline__ int tm_part(int warp) { return warp >> 2; }
constexpr uint32_t TILE_64x128 = 64 * 128 * 2;    // bytes of a [64 x 128] bf16 row tile

// ------------------------------------------------------------ host: TMA maps

// Tensor map of a [B, T, H, 128] bf16 tensor; box = 64 channels x 1 head x 64 tokens x 1,
// 128-byte swizzle, zero fill past the end of the sequence.
inline CUresult make_token_map(CUtensorMap* map, const void* ptr, int B, int T, int H) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return CUDA_ERROR_NOT_FOUND;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// ------------------------------------------------------------ device

// Load one [64 tokens x 128 channels] tile of (b, h) starting at token t0 into a
// row tile at `dst` (rows dst_row0.., tile of R rows): two 64-channel boxes.
__device__ __forceinline__ void tma_tile(unsigned char* dst, int R, int dst_row0, const CUtensorMap* map,
                                         int b, int h, int t0, uint64_t* bar) {
    tc::tma_load_4d(dst + dst_row0 * 128, map, 0, h, t0, b, bar);
    tc::tma_load_4d(dst + R * 128 + dst_row0 * 128, map, 64, h, t0, b, bar);
}

// Gate preparation, channel-major variant: thread = (key/value channel i = tid % 128,
// token half hf = tid / 128: tokens 32 hf .. 32 hf + 31), tokens in blocks of 8:
//   reads  log_alpha (KT), k (KH), b (QE rows 0..63), q (QE rows 64..127), v (UU), w (WW)
//   writes Et = g*b*k -> QE rows 0..63, Qt = g*q -> QE rows 64..127, Kt = k/g -> KT,
//          U = w*v -> KH (over k, which the thread has read); UU and WW keep v and w.
//   g = exp(G), G = inclusive cumsum of log_alpha; gC[i] = g at the last row.
//   G[t][i] is also stored to TMEM at tmem_g (lane i, column t); tmem_g is the thread's lane base.
__device__ __forceinline__ void gate_prep_cols(unsigned char* QE, unsigned char* KH, unsigned char* KT,
                                               const unsigned char* UU, const unsigned char* WW, float* gC_out,
                                               int tid, uint32_t tmem_g) {
    const int i = tid & 127, hf = tid >> 7;
    const uint32_t col64 = (uint32_t)((i >> 6) * 64 * 128 + ((i & 7) << 1));
    const uint32_t col128 = (uint32_t)((i >> 6) * 128 * 128 + ((i & 7) << 1));
    const uint32_t chunk = (uint32_t)((i & 63) >> 3);
    float G = 0.f;
    if (hf) {   // the second half starts from the sum over the first 32 tokens
        float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
        for (int t = 0; t < 32; t += 2) {
            s0 += tc::ld_bf16(KT, col64 + (uint32_t)t * 128 + ((chunk ^ (uint32_t)(t & 7)) << 4));
            s1 += tc::ld_bf16(KT, col64 + (uint32_t)(t + 1) * 128 + ((chunk ^ (uint32_t)((t + 1) & 7)) << 4));
        }
        G = s0 + s1;
    }
    __syncthreads();   // every thread has read the log_alpha it needs before Kt overwrites it
#pragma unroll 1
    for (int tb2 = 0; tb2 < 2; ++tb2) {
        float gvals[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int tb = 4 * hf + 2 * tb2 + half;
            float la[8], kk[8], bb[8], qq[8], vv[8], ww[8];
            uint32_t o64[8], o128[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t row = (uint32_t)(8 * tb + u);
                const uint32_t sw = ((chunk ^ (uint32_t)u) << 4);
                o64[u] = col64 + row * 128 + sw;
                o128[u] = col128 + row * 128 + sw;
                la[u] = tc::ld_bf16(KT, o64[u]);
                kk[u] = tc::ld_bf16(KH, o64[u]);
                bb[u] = tc::ld_bf16(QE, o128[u]);
                qq[u] = tc::ld_bf16(QE, o128[u] + C * 128);
                vv[u] = tc::ld_bf16(UU, o64[u]);
                ww[u] = tc::ld_bf16(WW, o64[u]);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                G += la[u];
                gvals[half * 8 + u] = G;
                const float g = fast_exp(G), ig = fast_exp(-G);
                tc::st_bf16(QE, o128[u], g * bb[u] * kk[u]);          // Et
                tc::st_bf16(QE, o128[u] + C * 128, g * qq[u]);        // Qt
                tc::st_bf16(KT, o64[u], kk[u] * ig);                  // Kt
                tc::st_bf16(KH, o64[u], ww[u] * vv[u]);               // U
            }
        }
        tc::tmem_st16(tmem_g + 32 * hf + 16 * tb2, gvals);
    }
    tc::tmem_wait_st();
    if (hf) gC_out[i] = fast_exp(G);
}

// Inclusive cumulative log-decay of the chunk for one thread = (4-token block tb = tid / 16,
// 8-channel group cg = tid % 16): on return G[u][c] + pre[c] is G at row 4 tb + u, channel 8 cg + c.
// The thread's log_alpha rows are read from KT (row tile of 64 rows); block totals are exchanged
// through `red` (fp32 [16][128], 8 KB). gC[i] = exp(G) at the last row when gC_out is not null.
// Contains one __syncthreads; afterwards the thread may overwrite its own rows and channels of KT.
__device__ __forceinline__ void chunk_cumsum(const unsigned char* KT, float* red, float* gC_out, int tid,
                                             float (&G)[4][8], float (&pre)[8]) {
    constexpr int RB = 4;
    const int cg = tid & 15, tb = tid >> 4;
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
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 8; ++c) pre[c] = 0.f;
#pragma unroll 1
    for (int p = 0; p < tb; ++p) {
        const float4 x0 = *reinterpret_cast<const float4*>(red + p * 128 + 8 * cg);
        const float4 x1 = *reinterpret_cast<const float4*>(red + p * 128 + 8 * cg + 4);
        pre[0] += x0.x; pre[1] += x0.y; pre[2] += x0.z; pre[3] += x0.w;
        pre[4] += x1.x; pre[5] += x1.y; pre[6] += x1.z; pre[7] += x1.w;
    }
    if (gC_out && tb == C / RB - 1) {
#pragma unroll
        for (int c = 0; c < 8; ++c) gC_out[8 * cg + c] = fast_exp(pre[c] + G[RB - 1][c]);
    }
}

// Gate preparation, vectorised: thread = (4-token block tb = tid / 16, 8-channel group cg = tid % 16),
// 16-byte shared-memory accesses:
//   reads  log_alpha (KT), k (KH), b (QE rows 0..63), q (QE rows 64..127), v (UU), w (WW)
//   writes Et = g*b*k -> QE rows 0..63, Qt = g*q -> QE rows 64..127 (want_q),
//          Kt = k/g -> KT, U = w*v -> UU (want_u); KH keeps k.
//   g = exp(G), G = inclusive cumsum of log_alpha over the chunk; gC[i] = g at the last row.
// Contains one __syncthreads.
__device__ __forceinline__ void gate_prep(unsigned char* QE, const unsigned char* KH, unsigned char* KT,
                                          unsigned char* UU, const unsigned char* WW, float* gC_out,
                                          float* red, int tid, bool want_q, bool want_u) {
    constexpr int RB = 4;
    const int cg = tid & 15, tb = tid >> 4;
    float G[RB][8], pre[8];
    chunk_cumsum(KT, red, gC_out, tid, G, pre);
#pragma unroll
    for (int u = 0; u < RB; ++u) {
        const int row = RB * tb + u;
        float kk[8], bb[8], qq[8], vv[8], ww[8];
        tc::ld_row8(KH, C, row, cg, kk);
        tc::ld_row8(QE, 2 * C, row, cg, bb);
        if (want_q) tc::ld_row8(QE, 2 * C, C + row, cg, qq);
        if (want_u) { tc::ld_row8(UU, C, row, cg, vv); tc::ld_row8(WW, C, row, cg, ww); }
        float e[8], kt[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float Gv = pre[c] + G[u][c];
            const float g = fast_exp(Gv), ig = fast_exp(-Gv);
            e[c] = g * bb[c] * kk[c];
            kt[c] = kk[c] * ig;
            if (want_q) qq[c] *= g;
            if (want_u) vv[c] *= ww[c];
        }
        tc::st_row8(QE, 2 * C, row, cg, e);
        tc::st_row8(KT, C, row, cg, kt);
        if (want_q) tc::st_row8(QE, 2 * C, C + row, cg, qq);
        if (want_u) tc::st_row8(UU, C, row, cg, vv);
    }
}

// Gate preparation of the state passes (no erase factor): same thread layout as gate_prep;
//   reads  log_alpha (KT), k (KH), q (QQ, 64 rows), v (UU), w (WW)
//   writes Qt = g*q -> QQ, Kt = k/g -> KT, U = w*v -> UU (kU), gC.
// Contains one __syncthreads.
template <bool kU = true>
__device__ __forceinline__ void gate_prep_state(unsigned char* QQ, const unsigned char* KH, unsigned char* KT,
                                                unsigned char* UU, const unsigned char* WW, float* gC_out,
                                                float* red, int tid) {
    constexpr int RB = 4;
    const int cg = tid & 15, tb = tid >> 4;
    float G[RB][8], pre[8];
    chunk_cumsum(KT, red, gC_out, tid, G, pre);
#pragma unroll
    for (int u = 0; u < RB; ++u) {
        const int row = RB * tb + u;
        float kk[8], qq[8], vv[8], ww[8];
        tc::ld_row8(KH, C, row, cg, kk);
        tc::ld_row8(QQ, C, row, cg, qq);
        if (kU) {
            tc::ld_row8(UU, C, row, cg, vv);
            tc::ld_row8(WW, C, row, cg, ww);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float Gv = pre[c] + G[u][c];
            const float g = fast_exp(Gv), ig = fast_exp(-Gv);
            kk[c] *= ig;
            qq[c] *= g;
            if (kU) vv[c] *= ww[c];
        }
        tc::st_row8(KT, C, row, cg, kk);
        tc::st_row8(QQ, C, row, cg, qq);
        if (kU) tc::st_row8(UU, C, row, cg, vv);
    }
}

// fp32 64 x 64 scratch matrices (A and its inverse) are stored with row stride
// 64 and the column index XOR-ed with (row % 32): row-wise and column-wise
// accesses by a warp are then both free of bank conflicts.
__device__ __forceinline__ int sq_idx(int r, int c) { return r * 64 + (c ^ (r & 31)); }

// Copy the strictly lower part of [A; P] from TMEM (lanes 0..63 = A, 64..127 = P,
// 64 columns at the warp's lane base + column 0) into the fp32 scratch sA and, if want_p,
// the causal part of P into the bf16 row tile PP. Each warp handles 32 of the 64 columns.
__device__ __forceinline__ void extract_AP(uint32_t lane_base_ap, float* sA, unsigned char* PP, bool want_p,
                                           int warp, int lane) {
    const int q = tm_quarter(warp), c0 = 32 * tm_part(warp);
    float v[32];
    tc::tmem_ld32(lane_base_ap + c0, v);
    tc::tmem_wait_ld(v);
    if (q < 2) {
        const int t = 32 * q + lane;
#pragma unroll
        for (int u = 0; u < 32; ++u) sA[sq_idx(t, c0 + u)] = v[u];
    } else if (want_p) {
        const int t = 32 * (q - 2) + lane;
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = (c0 + u <= t) ? v[u] : 0.f;
#pragma unroll
        for (int g = 0; g < 4; ++g) tc::st_row8(PP, C, t, (c0 >> 3) + g, v + 8 * g);
    }
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Row stride of the per-warp 16 x 8 fp32 temporaries (conflict-free fragment loads).
constexpr int XS = 24;
// acc (16 x 8, one m16n8 C fragment) += A[ar.., ac..] (16 x 16) * B[br.., bc..] (16 x 8), one warp,
// tf32 inputs, fp32 accumulation. A comes from a 64 x 64 scratch (sq_idx layout); B from the same
// layout (b_sq) or from a per-warp 16 x 8 temporary with row stride XS.
__device__ __forceinline__ void warp_mm16x8(float (&acc)[4], const float* __restrict__ A, int ar, int ac,
                                            const float* __restrict__ Bm, int br, int bc, bool b_sq, int lane) {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = to_tf32(A[sq_idx(ar + g, ac + 8 * ks + t4)]);
        const uint32_t a1 = to_tf32(A[sq_idx(ar + g + 8, ac + 8 * ks + t4)]);
        const uint32_t a2 = to_tf32(A[sq_idx(ar + g, ac + 8 * ks + t4 + 4)]);
        const uint32_t a3 = to_tf32(A[sq_idx(ar + g + 8, ac + 8 * ks + t4 + 4)]);
        const int r0 = br + 8 * ks + t4, c0 = bc + g;
        const float x0 = b_sq ? Bm[sq_idx(r0, c0)] : Bm[r0 * XS + c0];
        const float x1 = b_sq ? Bm[sq_idx(r0 + 4, c0)] : Bm[(r0 + 4) * XS + c0];
        mma_tf32_16x8x8(acc, a0, a1, a2, a3, to_tf32(x0), to_tf32(x1));
    }
}
// Store a 16 x 8 accumulator (times scale) to a sq_idx scratch at (rr, cc) or to a per-warp temporary.
__device__ __forceinline__ void warp_store16x8(const float (&acc)[4], float* dst, int rr, int cc, bool sq, float scale,
                                               int lane) {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int r = rr + g + ((e >> 1) << 3), c = cc + 2 * t4 + (e & 1);
        if (sq) dst[sq_idx(r, c)] = scale * acc[e];
        else dst[r * XS + c] = scale * acc[e];
    }
}
__device__ __forceinline__ void warp_load16x8(float (&acc)[4], const float* src, int lane) {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = src[(g + ((e >> 1) << 3)) * XS + 2 * t4 + (e & 1)];
}
// bf16 copy of a 16 x 8 accumulator (times scale) into the T row tile (64 x 64) at (rr, cc).
__device__ __forceinline__ void warp_store16x8_tile(const float (&acc)[4], unsigned char* Ttile, int rr, int cc,
                                                    float scale, int lane) {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int r = rr + g + 8 * hf, c = cc + 2 * t4;
        *reinterpret_cast<uint32_t*>(Ttile + tc::tile_off(C, r, c)) =
            tc::pack_bf16x2(scale * acc[2 * hf], scale * acc[2 * hf + 1]);
    }
}

// Inverse of the unit lower 16 x 16 diagonal block at (BASE, BASE) of I + A by right-looking forward
// substitution, one warp, lane = column (lanes 16..31 repeat lanes 0..15). The block's 120 strictly lower
// entries are read into registers first (compile-time addresses), so the 15 dependent steps run on
// registers. Writes the block to sTf (fp32, sq_idx layout) and to the bf16 T tile.
template <int BASE>
__device__ __forceinline__ void diag_inverse16(const float* __restrict__ sA, float* __restrict__ sTf,
                                               unsigned char* Ttile, int lane) {
    const int s = lane & 15;
    float a[120];
#pragma unroll
    for (int m = 0, idx = 0; m < 15; ++m)
#pragma unroll
        for (int r = m + 1; r < 16; ++r, ++idx) a[idx] = sA[sq_idx(BASE + r, BASE + m)];
    float acc[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) acc[r] = (r == s) ? 1.f : 0.f;
#pragma unroll
    for (int m = 0, idx = 0; m < 15; ++m) {
        const float xm = acc[m];
#pragma unroll
        for (int r = m + 1; r < 16; ++r, ++idx) acc[r] -= a[idx] * xm;
    }
    if (lane < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            sTf[sq_idx(BASE + r, BASE + s)] = acc[r];
            tc::st_bf16(Ttile, tc::tile_off(C, BASE + r, BASE + s), acc[r]);
        }
    }
}

// (I + A)^{-1} for the strictly lower 64 x 64 matrix A (fp32 scratch sA, sq_idx layout), 8 warps.
// Writes the inverse to sTf (lower triangle incl. the unit diagonal is valid) and the bf16 row
// tile T (64 x 64, zeros above the diagonal).
//   1. 16 x 16 diagonal blocks T_ii by right-looking forward substitution (warp i < 4, lane =
//      column); warps 4..7 clear T above the diagonal blocks meanwhile.
//   2. off-diagonal blocks T_ij = -T_ii * sum_{k=j}^{i-1} A_ik T_kj, by diagonals i - j = 1, 2, 3,
//      as warp-level tf32 tensor-core products (mma.sync m16n8k8); the warps w and w + 4 take the
//      left and right 8 columns of a block.
// sX: 8 warps x 16 x XS floats (12 KB), must not alias the T tile.
__device__ __forceinline__ void solve_unit_lower(const float* __restrict__ sA, float* __restrict__ sTf,
                                                 float* __restrict__ sX, unsigned char* Ttile, int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < 4) {
        switch (warp) {
        case 0: diag_inverse16<0>(sA, sTf, Ttile, lane); break;
        case 1: diag_inverse16<16>(sA, sTf, Ttile, lane); break;
        case 2: diag_inverse16<32>(sA, sTf, Ttile, lane); break;
        default: diag_inverse16<48>(sA, sTf, Ttile, lane); break;
        }
    } else {
        // zeros above the diagonal blocks: block row br = warp - 4, columns 16 br + 16 .. 63
        const int br = warp - 4, base = 16 * br;
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const int ngrp = (C - base - 16) / 8;
        for (int e = lane; e < 16 * ngrp; e += 32)
            tc::st_row8(Ttile, C, base + (e / ngrp), (base + 16) / 8 + (e % ngrp), z);
    }
    __syncthreads();
    const int blk = warp & 3, nt = warp >> 2, nc = 8 * nt;     // warp pair blk, column half nt
    float* Xw = sX + warp * 16 * XS;
    float acc[4];
    // diagonal 1: T_{j+1,j} (pairs 0..2); pair 3 starts T_30's sum with A_30 T_00
    if (blk < 3) {
        const int j = blk, i = j + 1;
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sA, 16 * i, 16 * j, sTf, 16 * j, 16 * j + nc, true, lane);
        warp_store16x8(acc, Xw, 0, 0, false, 1.f, lane);
        __syncwarp();
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sTf, 16 * i, 16 * i, Xw, 0, 0, false, lane);
        warp_store16x8(acc, sTf, 16 * i, 16 * j + nc, true, -1.f, lane);
        warp_store16x8_tile(acc, Ttile, 16 * i, 16 * j + nc, -1.f, lane);
    } else {
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sA, 48, 0, sTf, 0, nc, true, lane);          // A_30 T_00
        warp_store16x8(acc, Xw, 0, 0, false, 1.f, lane);
    }
    __syncthreads();
    // diagonal 2: T_20 (pair 0), T_31 (pair 1); pair 3 adds A_31 T_10 to its partial
    if (blk < 2) {
        const int j = blk, i = j + 2;
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sA, 16 * i, 16 * j, sTf, 16 * j, 16 * j + nc, true, lane);
        warp_mm16x8(acc, sA, 16 * i, 16 * (j + 1), sTf, 16 * (j + 1), 16 * j + nc, true, lane);
        warp_store16x8(acc, Xw, 0, 0, false, 1.f, lane);
        __syncwarp();
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sTf, 16 * i, 16 * i, Xw, 0, 0, false, lane);
        warp_store16x8(acc, sTf, 16 * i, 16 * j + nc, true, -1.f, lane);
        warp_store16x8_tile(acc, Ttile, 16 * i, 16 * j + nc, -1.f, lane);
    } else if (blk == 3) {
        warp_load16x8(acc, Xw, lane);
        warp_mm16x8(acc, sA, 48, 16, sTf, 16, nc, true, lane);         // + A_31 T_10
        __syncwarp();
        warp_store16x8(acc, Xw, 0, 0, false, 1.f, lane);
    }
    __syncthreads();
    // diagonal 3: T_30 = -T_33 (A_30 T_00 + A_31 T_10 + A_32 T_20)   (pair 3)
    if (blk == 3) {
        warp_load16x8(acc, Xw, lane);
        warp_mm16x8(acc, sA, 48, 32, sTf, 32, nc, true, lane);
        __syncwarp();
        warp_store16x8(acc, Xw, 0, 0, false, 1.f, lane);
        __syncwarp();
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        warp_mm16x8(acc, sTf, 48, 48, Xw, 0, 0, false, lane);
        warp_store16x8_tile(acc, Ttile, 48, nc, -1.f, lane);
    }
}

// Copy a [128 lanes x NCOL] fp32 TMEM accumulator into a bf16 row tile of 128 rows (row = lane);
// the two warps of a lane quarter take half of the columns each.
template <int NCOL>
__device__ __forceinline__ void tmem_to_tile_rows(uint32_t lane_base_col, unsigned char* dst, int warp, int lane) {
    const int row = 32 * tm_quarter(warp) + lane, c0 = (NCOL / 2) * tm_part(warp);
    float v[32];
#pragma unroll
    for (int cc = 0; cc < NCOL / 2; cc += 32) {
        tc::tmem_ld32(lane_base_col + c0 + cc, v);
        tc::tmem_wait_ld(v);
#pragma unroll
        for (int g = 0; g < 4; ++g) tc::st_row8(dst, 128, row, ((c0 + cc) >> 3) + g, v + 8 * g);
    }
}

// M = 64 accumulators (cta_group::1): row r of D lives in TMEM lane (r % 16) + 32 (r / 16).
// In lane quarter q, lanes 0..15 hold rows 16 q .. 16 q + 15. All 32 lanes must execute the loads.
__device__ __forceinline__ int m64_row(int warp, int lane) { return 16 * tm_quarter(warp) + (lane & 15); }

// Copy a [64 rows x 128 columns] M=64 accumulator into a bf16 row tile of 64 rows; the two warps of
// a lane quarter take 64 columns each.
__device__ __forceinline__ void tmem_m64_to_tile(uint32_t lane_base_col, unsigned char* dst, int warp, int lane) {
    const int r = m64_row(warp, lane), c0 = 64 * tm_part(warp);
    float v[32];
#pragma unroll
    for (int cc = 0; cc < 64; cc += 32) {
        tc::tmem_ld32(lane_base_col + c0 + cc, v);
        tc::tmem_wait_ld(v);
        if (lane < 16) {
#pragma unroll
            for (int g = 0; g < 4; ++g) tc::st_row8(dst, C, r, ((c0 + cc) >> 3) + g, v + 8 * g);
        }
    }
}

}  // namespace chunk
}  // namespace gdn2
