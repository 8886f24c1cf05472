// chunk_fwd.cu -- chunkwise WY forward of the Gated Delta Rule-2 operator on
// tcgen05 tensor cores (bf16 operands, fp32 TMEM accumulators, fp32 state).
//
// One CTA (256 threads) per (batch, head) walks the chunks in order; the state
// is carried across chunks in TMEM as S^T (lane j = value channel, column i =
// key channel) in fp32, with a bf16 copy in shared memory as the UMMA operand.
// Per chunk ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
// Attention", arXiv abstract: chunkwise WY algorithm, decay absorbed into
// asymmetric erase factors):
//   TMA      q, k, v, log_alpha, b, w tiles (64 tokens x 128, bf16, 128B swizzle)
//   prep     Et = g*b*k, Qt = g*q, Kt = k/g, Kh = gC*Kt, U = w*v       (g = exp(cumsum log_alpha))
//   M1       [A; P] = [Et; Qt] Kt^T                                     (M=128, N=64, K=128)
//   solve    T = (I + strict_lower(A))^{-1}     (16x16 blocks, off-diagonal merges on mma.sync tf32)
//   M2, M3   Wm = T Et (M=64, N=128) ,  Delta^T := U^T T^T (M=128, N=64)
//   M4, M5   Delta^T -= S^T Wm^T (M=128) ,  O = Qt S (M=64, N=128)
//   M6, M7   O += P Delta (M=64) ,  Z^T = S^T + Delta^T Kt (M=128, N=128)
//   scale    S'^T = Z^T Diag(gC) on the fp32 accumulator, bf16 copy for the next chunk
// For training, the chunk-start states and the T and P tiles of every chunk are written
// (bf16 shared-memory images) for the backward.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

using namespace chunk;

// shared-memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_QE = 0;           // [128 x 128] rows 0..63: b -> Et, rows 64..127: q -> Qt
constexpr uint32_t OFF_KH = 32768;       // [64 x 128] k
constexpr uint32_t OFF_KT = 49152;       // [64 x 128] log_alpha -> Kt
constexpr uint32_t OFF_UU = 65536;       // [64 x 128] v -> U
constexpr uint32_t OFF_WW = 81920;       // [64 x 128] w -> solve temporaries -> Wm
constexpr uint32_t OFF_ST = 98304;       // [128 x 128] S^T (bf16)
constexpr uint32_t OFF_DT = 131072;      // [128 x 64] Delta^T (bf16)  | fp32 A scratch [64 x 64]
constexpr uint32_t OFF_TF = 147456;      // fp32 T [64 x 64] | prep scan scratch
constexpr uint32_t OFF_TT = 163840;      // [64 x 64] T (bf16)
constexpr uint32_t OFF_PP = 172032;      // [64 x 64] P (bf16)
constexpr uint32_t OFF_GC = 180224;      // fp32 gC[128]
constexpr uint32_t OFF_BAR = 180736;     // 2 mbarriers, tmem base, abort flag
constexpr uint32_t SMEM_BYTES = 180800 + 1024;

// TMEM columns: S^T (fp32 state), [A; P], Ut^T -> Delta^T, Wm (M=64), O (M=64)
constexpr uint32_t TM_S = 0, TM_AP = 128, TM_D = 192, TM_W = 256, TM_O = 384, TM_COLS = 512;

constexpr uint32_t LOAD_BYTES = 6 * 64 * 128 * 2;

__device__ unsigned int g_fwd_error;

__global__ void __launch_bounds__(NT, 1)
chunk_fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                 const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mla,
                 const __grid_constant__ CUtensorMap mb, const __grid_constant__ CUtensorMap mw,
                 const float* __restrict__ S0, __nv_bfloat16* __restrict__ o, float* __restrict__ ST,
                 unsigned char* __restrict__ states, unsigned char* __restrict__ tp, int T, int H) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays in the shared window
    unsigned char* QE = sm + OFF_QE;
    unsigned char* KH = sm + OFF_KH;
    unsigned char* KT = sm + OFF_KT;
    unsigned char* UU = sm + OFF_UU;
    unsigned char* WW = sm + OFF_WW;
    unsigned char* STt = sm + OFF_ST;
    unsigned char* DT = sm + OFF_DT;
    float* sA = reinterpret_cast<float*>(sm + OFF_DT);
    float* sTf = reinterpret_cast<float*>(sm + OFF_TF);
    float* sX = reinterpret_cast<float*>(sm + OFF_WW);   // w is consumed by the prep, Wm written after M2
    unsigned char* TT = sm + OFF_TT;
    unsigned char* PP = sm + OFF_PP;
    float* sGC = reinterpret_cast<float*>(sm + OFF_GC);
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_mma = bar_load + 1;
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 16);
    int* abort_flag = reinterpret_cast<int*>(sm + OFF_BAR + 20);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const size_t head = blockIdx.x;
    const int nc = (T + C - 1) / C;
    const bool want_o = (o != nullptr);
    const bool save = (states != nullptr);          // training: keep S, T and P of every chunk
    const bool want_qp = want_o || save;

    if (tid == 0) {
        tc::mbar_init(bar_load, 1);
        tc::mbar_init(bar_mma, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&mq); tc::tma_prefetch_desc(&mk); tc::tma_prefetch_desc(&mv);
        tc::tma_prefetch_desc(&mla); tc::tma_prefetch_desc(&mb); tc::tma_prefetch_desc(&mw);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base_ptr, TM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_base_ptr;
    const uint32_t lane_base = tmem + ((uint32_t)(tm_quarter(warp) * 32) << 16);   // this warp's TMEM lanes
    const int jrow = 32 * tm_quarter(warp) + lane, cpart = 64 * tm_part(warp);      // lane row, column half

    auto issue_loads = [&](int c) {
        const int t0 = c * C;
        tc::mbar_arrive_expect_tx(bar_load, LOAD_BYTES);
        tma_tile(QE, 2 * C, 0, &mb, b, h, t0, bar_load);
        tma_tile(QE, 2 * C, C, &mq, b, h, t0, bar_load);
        tma_tile(KH, C, 0, &mk, b, h, t0, bar_load);
        tma_tile(KT, C, 0, &mla, b, h, t0, bar_load);
        tma_tile(UU, C, 0, &mv, b, h, t0, bar_load);
        tma_tile(WW, C, 0, &mw, b, h, t0, bar_load);
    };
    if (tid == 0 && nc > 0) issue_loads(0);

    // initial state: S^T row j = column j of S0
    {
        const int j = jrow;
        float v[32];
#pragma unroll 1
        for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = S0 ? S0[(head * D + i0 + u) * D + j] : 0.f;
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
    if (states && tid == 0) {
        tc::bulk_store(states + (head * nc + 0) * TC_STATE_BYTES, STt, (uint32_t)TC_STATE_BYTES);
        tc::bulk_commit();
    }

    const uint32_t sQE = tc::smem_u32(QE), sKT = tc::smem_u32(KT), sUU = tc::smem_u32(UU),
                   sWW = tc::smem_u32(WW), sST = tc::smem_u32(STt), sDT = tc::smem_u32(DT),
                   sTT = tc::smem_u32(TT), sPP = tc::smem_u32(PP);
    constexpr uint32_t ID_M1 = tc::idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_M2 = tc::idesc_bf16(64, 128, false, true);
    constexpr uint32_t ID_M3 = tc::idesc_bf16(128, 64, true, false);
    constexpr uint32_t ID_M4 = tc::idesc_bf16(128, 64, false, false, true);
    constexpr uint32_t ID_M56 = tc::idesc_bf16(64, 128, false, false);
    constexpr uint32_t ID_M7 = tc::idesc_bf16(128, 128, false, true);

    uint32_t ph_load = 0, ph_mma = 0;
    auto wait_mma = [&]() {
        if (!tc::mbar_wait(bar_mma, ph_mma)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 1u); }
        ph_mma ^= 1;
        tc::tc_fence_after();
    };
    auto sync_for_mma = [&]() {   // smem written by threads + TMEM accesses done -> visible to the MMA issuer
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
    };

    for (int c = 0; c < nc; ++c) {
        const int t0 = c * C;
        const int L = min(C, T - t0);
        if (!tc::mbar_wait(bar_load, ph_load)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 2u); }
        ph_load ^= 1;

        // ---- gate prep (thread = channel)
        gate_prep(QE, KH, KT, UU, WW, sGC, sTf, tid, want_qp, true);
        sync_for_mma();

        // ---- M1: [A; P] = [Et; Qt] Kt^T
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_AP, tc::desc_k(sQE, 2 * C, 0, kk), tc::desc_k(sKT, C, 0, kk), ID_M1, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        extract_AP(lane_base + TM_AP, sA, PP, want_qp, warp, lane);
        tc::tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^{-1}
        solve_unit_lower(sA, sTf, sX, TT, tid);
        sync_for_mma();
        if (save && tid == 0) {   // T and P of this chunk for the backward
            unsigned char* dst = tp + (head * nc + c) * TC_TP_BYTES;
            tc::bulk_store(dst, TT, (uint32_t)(TC_TP_BYTES / 2));
            tc::bulk_store(dst + TC_TP_BYTES / 2, PP, (uint32_t)(TC_TP_BYTES / 2));
            tc::bulk_commit();
        }

        // ---- M2: Wm = T Et ;  M3: Delta^T := U^T T^T
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                tc::mma_bf16(tmem + TM_W, tc::desc_k(sTT, C, 0, kk), tc::desc_mn(sQE, 2 * C, 0, kk), ID_M2, kk > 0);
                tc::mma_bf16(tmem + TM_D, tc::desc_mn(sUU, C, 0, kk), tc::desc_k(sTT, C, 0, kk), ID_M3, kk > 0);
            }
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        tmem_m64_to_tile(lane_base + TM_W, WW, warp, lane);   // Wm rows [t][i]
        sync_for_mma();

        // ---- M4: Delta^T -= S^T Wm^T ;  M5: O = Qt S
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                tc::mma_bf16(tmem + TM_D, tc::desc_k(sST, D, 0, kk), tc::desc_k(sWW, C, 0, kk), ID_M4, 1);
                if (want_o)
                    tc::mma_bf16(tmem + TM_O, tc::desc_k(sQE, 2 * C, C, kk), tc::desc_k(sST, D, 0, kk), ID_M56, kk > 0);
            }
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        tmem_to_tile_rows<64>(lane_base + TM_D, DT, warp, lane);   // Delta^T (lane j) -> bf16 rows
        sync_for_mma();

        // ---- M6: O += P Delta ;  M7: Z^T = S^T + Delta^T Kt
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                if (want_o)
                    tc::mma_bf16(tmem + TM_O, tc::desc_k(sPP, C, 0, kk), tc::desc_k(sDT, D, 0, kk), ID_M56, 1);
                tc::mma_bf16(tmem + TM_S, tc::desc_k(sDT, D, 0, kk), tc::desc_mn(sKT, C, 0, kk), ID_M7, 1);
            }
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        // all smem input tiles of this chunk are consumed: prefetch the next chunk
        if (tid == 0 && c + 1 < nc) issue_loads(c + 1);

        if (want_o) {   // o rows t from the M=64 accumulator: 16-byte stores
            const int t = m64_row(warp, lane);
            float v[32];
#pragma unroll
            for (int c0 = cpart; c0 < cpart + 64; c0 += 32) {
                tc::tmem_ld32(lane_base + TM_O + c0, v);
                tc::tmem_wait_ld();
                if (lane < 16 && t < L) {
                    uint4* dst = reinterpret_cast<uint4*>(o + tok_off(b, t0 + t, h, T, H, D) + c0);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        dst[g] = make_uint4(tc::pack_bf16x2(v[8 * g], v[8 * g + 1]), tc::pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                            tc::pack_bf16x2(v[8 * g + 4], v[8 * g + 5]), tc::pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
                }
            }
        }
        // S'^T = Z^T Diag(gC): scale the fp32 state, keep a bf16 copy for the next chunk
        if (states && tid == 0) tc::bulk_wait_read();
        __syncthreads();
        {
            const int j = jrow;
            float v[32];
#pragma unroll 1
            for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
                tc::tmem_ld32(lane_base + TM_S + i0, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] *= sGC[i0 + u];
                tc::tmem_st32(lane_base + TM_S + i0, v);
#pragma unroll
                for (int g = 0; g < 4; ++g) tc::st_row8(STt, D, j, (i0 >> 3) + g, v + 8 * g);
            }
            tc::tmem_wait_st();
        }
        sync_for_mma();
        tc::tc_fence_after();
        if (states && tid == 0 && c + 1 < nc) {
            tc::bulk_store(states + (head * nc + c + 1) * TC_STATE_BYTES, STt, (uint32_t)TC_STATE_BYTES);
            tc::bulk_commit();
        }
        if (*abort_flag) break;
    }

    // final state (fp32): ST[i][j] from S^T (lane j)
    if (ST) {
        const int j = jrow;
        float v[32];
#pragma unroll 1
        for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
            tc::tmem_ld32(lane_base + TM_S + i0, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) ST[(head * D + i0 + u) * D + j] = v[u];
        }
    }
    if (states && tid == 0) tc::bulk_wait_all();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace

cudaError_t chunk_fwd_launch(const ChunkFwdArgs& a, cudaStream_t s) {
    const Dims& d = a.d;
    if (d.T == 0 || d.B * d.H == 0) return cudaSuccess;
    CUtensorMap mq, mk, mv, mla, mb, mw;
    const void* ptrs[6] = {a.q, a.k, a.v, a.la, a.b, a.w};
    CUtensorMap* maps[6] = {&mq, &mk, &mv, &mla, &mb, &mw};
    for (int i = 0; i < 6; ++i)
        if (make_token_map(maps[i], ptrs[i], d.B, d.T, d.H) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    TraceScope trace(K_CHUNK_FWD, s);
    chunk_fwd_kernel<<<d.B * d.H, NT, SMEM_BYTES, s>>>(mq, mk, mv, mla, mb, mw, a.S0,
                                                       static_cast<__nv_bfloat16*>(a.o), a.ST, a.states, a.tp, d.T, d.H);
    return cudaGetLastError();
}

}  // namespace gdn2
