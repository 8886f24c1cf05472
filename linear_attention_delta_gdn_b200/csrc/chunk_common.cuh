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
// The kernels scale the fp32 state by gC, then let the contraction add Kh^T Delta to it; the WY image
// of a chunk carries Kh (bounded) in place of Kt.
// Rows past the end of the sequence are zero-filled by TMA: they give zero
// factors, a flat cumulative decay and an identity block of T, so a ragged
// last chunk needs no special case except masked stores.
//
// Range of the factors. Qt, Et and Kh carry exp(G_t) or exp(G_C - G_t) <= 1 (log_alpha <= 0), but Kt
// carries exp(-G_t), which overflows once a channel decays by more than ~e^88 inside one chunk. A channel
// is "tame" in a chunk when the sum of |log_alpha| over the chunk is at most TAME_LOG_DECAY: then every
// factor stays within e^{+-60} and the products inside the fp32 accumulators stay finite. For the other
// ("untame") channels Kt is set to zero, so the tensor-core products that pair two tokens of the chunk
// (A, P in the forward; dQt, dEt, dKt in the backward) leave them out, and their exact contribution,
// sum over channels of x_t y_s exp(G_t - G_s), is added on CUDA cores with exp(G_t - G_s) formed as the
// running product of alpha over (s, t] (every factor <= 1). The state updates use Kh, so they need no
// fix-up. Typical decays (|G| of a few units per chunk) never take the exact path.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {
namespace chunk {

constexpr int D = 128;        // d_k = d_v
constexpr int C = 64;         // chunk length
constexpr int NT = 256;       // threads per CTA (two warpgroups)
constexpr float TAME_LOG_DECAY = 60.f;   // largest sum of |log_alpha| over a chunk on the tensor-core products
// TMEM access: warp w reads lane quarter (w % 4), i.e. lanes 32 (w % 4) .. +31; the two warps of a
// quarter (w and w + 4) split the columns of each read-out between them (part = w / 4).
__device__ __forceinline__ int tm_quarter(int warp) { return warp & 3; }
__device__ __forceinline__ int tm_part(int warp) { return warp >> 2; }
constexpr uint32_t TILE_64x128 = 64 * 128 * 2;    // bytes of a [64 x 128] bf16 row tile

// ------------------------------------------------------------ host: TMA maps

// Tensor map of a [B, T, H, 128] bf16 tensor; box = 64 channels x 1 head x 64 tokens x 1,
// 128-byte swizzle, zero fill past the end of the sequence.
inline CUresult encode_token_map(CUtensorMap* map, const void* ptr, int B, int T, int H) {
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

// The same, from a small per-thread cache keyed by (pointer, B, T, H): a training step passes the same
// tensors call after call, and encoding a map is host work on every launch otherwise. A map describes
// only addresses and sizes, so a hit is exact; the cache never dereferences the pointer.
inline CUresult make_token_map(CUtensorMap* map, const void* ptr, int B, int T, int H) {
    struct Entry {
        const void* ptr;
        int B, T, H;
        CUtensorMap map;
    };
    constexpr int N = 64;
    thread_local Entry cache[N] = {};
    const uintptr_t key = reinterpret_cast<uintptr_t>(ptr);
    const int slot = (int)(((key >> 8) ^ (key >> 20) ^ (uintptr_t)T * 31u ^ (uintptr_t)B * 7u ^ (uintptr_t)H) % N);
    Entry& e = cache[slot];
    if (e.ptr == ptr && e.B == B && e.T == T && e.H == H && ptr) {
        *map = e.map;
        return CUDA_SUCCESS;
    }
    const CUresult r = encode_token_map(map, ptr, B, T, H);
    if (r == CUDA_SUCCESS) e = Entry{ptr, B, T, H, *map};
    return r;
}

// Per-device launch facts of a kernel that never change once known: SM count, cooperative-launch support,
// resident CTAs per SM at the kernel's shared-memory size. The shared-memory attribute itself is set on every
// call (a device reset clears it).
struct LaunchFacts {
    int nsm, coop, occ;
};
template <typename Kernel>
inline cudaError_t launch_facts(Kernel kernel, int threads, uint32_t smem, LaunchFacts* out) {
    constexpr int kMaxDev = 64;
    static LaunchFacts facts[kMaxDev];
    static bool known[kMaxDev];
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < kMaxDev && known[dev]) {
        *out = facts[dev];
        return cudaSuccess;
    }
    LaunchFacts f{};
    if ((e = cudaDeviceGetAttribute(&f.nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&f.coop, cudaDevAttrCooperativeLaunch, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&f.occ, kernel, threads, smem)) != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDev) {
        facts[dev] = f;
        known[dev] = true;
    }
    *out = f;
    return cudaSuccess;
}

// ------------------------------------------------------------ device

// Load one [64 tokens x 128 channels] tile of (b, h) starting at token t0 into a
// row tile at `dst` (rows dst_row0.., tile of R rows): two 64-channel boxes.
__device__ __forceinline__ void tma_tile(unsigned char* dst, int R, int dst_row0, const CUtensorMap* map,
                                         int b, int h, int t0, uint64_t* bar) {
    tc::tma_load_4d(dst + dst_row0 * 128, map, 0, h, t0, b, bar);
    tc::tma_load_4d(dst + R * 128 + dst_row0 * 128, map, 64, h, t0, b, bar);
}

// fp32 64 x 64 scratch matrices (A and its inverse) are stored with row stride
// 64 and the column index XOR-ed with (row % 32): row-wise and column-wise
// accesses by a warp are then both free of bank conflicts.
__device__ __forceinline__ int sq_idx(int r, int c) { return r * 64 + (c ^ (r & 31)); }

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

}  // namespace chunk
}  // namespace gdn2
