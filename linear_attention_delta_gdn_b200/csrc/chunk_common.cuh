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
constexpr int NT = 128;       // threads per CTA (one warpgroup; thread i <-> TMEM lane i)
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

// Gate preparation, one thread per channel i (= threadIdx.x):
//   reads q (rows 64.. of QE), b (rows 0.. of QE), k (KH), log_alpha (KT), v (UU), w (WW)
//   writes Et -> QE rows 0..63, Qt -> QE rows 64..127, Kt -> KT, Kh -> KH, U -> UU,
//   gC[i] -> gC_out. Each element is read and rewritten by the same thread.
// With want_u = false, v/w are left untouched.
__device__ __forceinline__ void gate_prep(unsigned char* QE, unsigned char* KH, unsigned char* KT,
                                          unsigned char* UU, const unsigned char* WW, float* gC_out, int i,
                                          bool want_q, bool want_u) {
    float G = 0.f;
#pragma unroll 8
    for (int t = 0; t < C; ++t) G += tc::ld_bf16(KT, tc::tile_off(C, t, i));
    const float gC = fast_exp(G);
    gC_out[i] = gC;
    G = 0.f;
#pragma unroll 4
    for (int t = 0; t < C; ++t) {
        const uint32_t o64 = tc::tile_off(C, t, i);
        G += tc::ld_bf16(KT, o64);
        const float g = fast_exp(G), ig = fast_exp(-G);
        const float kk = tc::ld_bf16(KH, o64);
        const uint32_t oe = tc::tile_off(2 * C, t, i);
        const float bb = tc::ld_bf16(QE, oe);
        tc::st_bf16(QE, oe, g * bb * kk);                    // Et
        if (want_q) {
            const uint32_t oq = tc::tile_off(2 * C, C + t, i);
            tc::st_bf16(QE, oq, g * tc::ld_bf16(QE, oq));     // Qt
        }
        const float kt = kk * ig;
        tc::st_bf16(KT, o64, kt);                            // Kt
        tc::st_bf16(KH, o64, gC * kt);                       // Kh
        if (want_u) tc::st_bf16(UU, o64, tc::ld_bf16(WW, o64) * tc::ld_bf16(UU, o64));   // U = w*v
    }
}

// fp32 64 x 64 scratch matrices (A and its inverse) are stored with row stride
// 64 and the column index XOR-ed with (row % 32): row-wise and column-wise
// accesses by a warp are then both free of bank conflicts.
__device__ __forceinline__ int sq_idx(int r, int c) { return r * 64 + (c ^ (r & 31)); }

// Copy the strictly lower part of [A; P] from TMEM (lanes 0..63 = A, 64..127 = P,
// 64 columns at tm_ap) into the fp32 scratch sA (warps 0, 1) and, if want_p,
// the causal part of P into the bf16 row tile PP (warps 2, 3).
__device__ __forceinline__ void extract_AP(uint32_t lane_base_ap, float* sA, unsigned char* PP, bool want_p,
                                           int tid) {
    float v[32];
    if (tid < 64) {
        const int t = tid;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            tc::tmem_ld32(lane_base_ap + 32 * h2, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) sA[sq_idx(t, 32 * h2 + u)] = v[u];
        }
    } else {
        const int t = tid - 64;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            tc::tmem_ld32(lane_base_ap + 32 * h2, v);
            tc::tmem_wait_ld();
            if (want_p) {
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = (32 * h2 + u <= t) ? v[u] : 0.f;
#pragma unroll
                for (int g = 0; g < 4; ++g) tc::st_row8(PP, C, t, 4 * h2 + g, v + 8 * g);
            }
        }
    }
}

// (I + A)^{-1} for the strictly lower 64 x 64 matrix A (fp32 scratch sA).
// Writes the fp32 inverse to sTf (lower triangle incl. the unit diagonal is
// valid) and the bf16 row tile T (64 x 64, zeros above the diagonal).
// 16 x 16 diagonal blocks by forward substitution (one warp per block), then the
// off-diagonal blocks by diagonals: T_ij = -T_ii * sum_{k=j}^{i-1} A_ik T_kj.
// sX (768 floats) may alias the T tile: it is dead before T is written.
__device__ __forceinline__ void solve_unit_lower(const float* sA, float* sTf, float* sX, unsigned char* Ttile,
                                                 int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    if (lane < 16) {
        const int s = lane, base = 16 * warp;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == s) ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) acc -= sA[sq_idx(base + r, base + m)] * x[m];
            x[r] = acc;
            sTf[sq_idx(base + r, base + s)] = acc;
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;
        for (int e = tid; e < nb * 256; e += NT) {
            const int j = e >> 8, i = j + d, r = (e >> 4) & 15, c = e & 15;
            float acc = 0.f;
            for (int kb = j; kb < i; ++kb) {
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc += sA[sq_idx(16 * i + r, 16 * kb + m)] * sTf[sq_idx(16 * kb + m, 16 * j + c)];
            }
            sX[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < nb * 256; e += NT) {
            const int j = e >> 8, i = j + d, r = (e >> 4) & 15, c = e & 15;
            float acc = 0.f;
            for (int m = 0; m <= r; ++m) acc += sTf[sq_idx(16 * i + r, 16 * i + m)] * sX[(j << 8) + m * 16 + c];
            sTf[sq_idx(16 * i + r, 16 * j + c)] = -acc;
        }
        __syncthreads();
    }
    if (tid < C) {
        const int t = tid;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = 8 * g + u;
                x[u] = (s <= t) ? sTf[sq_idx(t, s)] : 0.f;
            }
            tc::st_row8(Ttile, C, t, g, x);
        }
    }
}

// Transpose a [128 lanes x 64 columns] fp32 TMEM accumulator (lane = channel,
// column = token) into the bf16 row tile dst [64 tokens x 128 channels].
__device__ __forceinline__ void tmem_to_tile_transposed(uint32_t lane_base_col, unsigned char* dst, int tid) {
    float v[32];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        tc::tmem_ld32(lane_base_col + 32 * h2, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) tc::st_bf16(dst, tc::tile_off(C, 32 * h2 + u, tid), v[u]);
    }
}

// Copy a [128 lanes x ncol] fp32 TMEM accumulator into a bf16 row tile of 128
// rows (row = lane), ncol in {64, 128}.
template <int NCOL>
__device__ __forceinline__ void tmem_to_tile_rows(uint32_t lane_base_col, unsigned char* dst, int tid) {
    float v[32];
#pragma unroll
    for (int c0 = 0; c0 < NCOL; c0 += 32) {
        tc::tmem_ld32(lane_base_col + c0, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) tc::st_row8(dst, 128, tid, (c0 >> 3) + g, v + 8 * g);
    }
}

// Multiply a [128 lanes x 128 columns] fp32 TMEM state by gC[column] in place.
__device__ __forceinline__ void tmem_scale_columns(uint32_t lane_base_col, const float* gC) {
    float v[32];
#pragma unroll 1
    for (int i0 = 0; i0 < D; i0 += 32) {
        tc::tmem_ld32(lane_base_col + i0, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] *= gC[i0 + u];
        tc::tmem_st32(lane_base_col + i0, v);
    }
    tc::tmem_wait_st();
}

}  // namespace chunk
}  // namespace gdn2
