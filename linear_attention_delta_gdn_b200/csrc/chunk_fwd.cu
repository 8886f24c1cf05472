// chunk_fwd.cu -- chunkwise WY forward of the Gated Delta Rule-2 operator on
// tcgen05 tensor cores (bf16 operands, fp32 TMEM accumulators, fp32 state).
//
// Chunk algebra ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
// Attention", arXiv abstract: chunkwise WY algorithm, decay absorbed into
// asymmetric erase factors), per head and chunk of 64 tokens starting from S:
//   prep     Et = g*b*k, Qt = g*q, Kt = k/g, U = w*v          (g = exp(cumsum log_alpha))
//   WY       [A; P] = [Et; Qt] Kt^T,  T = (I + strict_lower(A))^{-1},  Wm = T Et
//   state    Delta^T = U^T T^T - S^T Wm^T,  O = Qt S + P Delta,  S'^T = (S^T + Delta^T Kt) Diag(gC)
// The WY step does not depend on S; the state step is a chain over the chunks of a head.
//
// One launch, two kinds of CTA (256 threads each, one CTA per SM):
//   * producers walk the chunks of all heads in chunk-major order and compute the WY step; each
//     writes T, P and Wm of its chunk ("WY image", 32 KB) to the workspace and then sets the
//     chunk's ready flag (release);
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
constexpr uint32_t KT = 32768;      // 2 x [64 x 128] Kt from the WY image (by chunk parity)
constexpr uint32_t UU = 65536;      // [64 x 128] v -> U
constexpr uint32_t WW = 81920;      // [64 x 128] w
constexpr uint32_t WY = 98304;      // WY image head: T [64 x 64] | P [64 x 64] | Wm [64 x 128]
constexpr uint32_t TT = WY, PP = WY + 8192, WM = WY + 16384;
constexpr uint32_t ST = 131072;     // [128 x 128] S^T (bf16)
constexpr uint32_t DT = 163840;     // [128 x 64] Delta^T (bf16)
constexpr uint32_t GC = 180224;     // 2 x fp32 gC[128] from the WY image (by chunk parity)
constexpr uint32_t BAR = 181248;    // 3 mbarriers (load, mma, unused), tmem base, abort flag
}  // namespace sp
// ---- producer (WY) shared memory: two input stages, then the solve scratch and the WY image
namespace wy {
constexpr uint32_t STAGE = 65536;   // per stage: [b; q] rows (32 KB) at 0, k at 32768, log_alpha at 49152
constexpr uint32_t QE = 0, KH = 32768, KT = 49152;
constexpr uint32_t SA = 131072;     // fp32 A [64 x 64] (sq_idx) | prep scan scratch
constexpr uint32_t TF = 147456;     // fp32 T [64 x 64]
constexpr uint32_t SX = 163840;     // solve temporaries, 12 KB
constexpr uint32_t IMG = 176128;    // WY image: T | P | Wm (32 KB)
constexpr uint32_t TT = IMG, PP = IMG + 8192, WM = IMG + 16384;
constexpr uint32_t BAR = 208896;    // 3 mbarriers (2 stages, mma), tmem base, abort flag
constexpr uint32_t GC = 208960;     // 2 x fp32 gC[128] (by stage)
}  // namespace wy
constexpr uint32_t SMEM_BYTES = 209984 + 1024;
static_assert(sp::BAR + 64 <= wy::BAR + 64, "consumer layout fits");
static_assert(TC_WY_QT == 32768 && TC_WY_KT == 49152 && TC_WY_GC == 65536, "WY image: T | P | Wm | Qt | Kt | gC");

// TMEM columns. Consumer: S^T (fp32 state), Ut^T -> Delta^T, O x 2 (M=64). Producer: [A; P], Wm (M=64).
constexpr uint32_t TM_S = 0, TM_D = 128, TM_O = 256;   // O: two buffers of 128 columns (chunk parity)
constexpr uint32_t TM_AP = 0, TM_W = 128;
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t CONS_LOAD_BYTES = 2 * 64 * 128 * 2;   // v, w
constexpr uint32_t PROD_LOAD_BYTES = 4 * 64 * 128 * 2;

__device__ unsigned int g_fwd_error;

struct FwdParams {
    int T, H, BH, nc;
    int ncons, nprod;              // CTAs [0, ncons) are consumers, the next nprod are producers
    const float* S0;
    __nv_bfloat16* o;              // may be null (states only)
    float* ST;
    unsigned char* states;         // [BH, nc] chunk-start state images, or null
    unsigned char* deltas;         // [BH, nc] Delta^T images, or null
    unsigned char* wyimg;          // [BH, nc] WY images
    unsigned int* flags;           // [BH, nc] ready flags (zero at launch)
};

struct Maps {
    CUtensorMap q, k, v, la, b, w;
};

__device__ __forceinline__ void sync_for_mma() {   // smem written by threads + TMEM accesses done -> MMA issuer
    tc::fence_async_smem();
    tc::tc_fence_before();
    __syncthreads();
}

// ------------------------------------------------------------------ producer
__device__ void run_producer(const Maps& m, const FwdParams& p, unsigned char* sm, uint32_t tmem, int pid) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bar_in = reinterpret_cast<uint64_t*>(sm + wy::BAR);   // [2]
    uint64_t* bar_mma = bar_in + 2;
    int* abort_flag = reinterpret_cast<int*>(sm + wy::BAR + 28);
    float* sA = reinterpret_cast<float*>(sm + wy::SA);
    float* sTf = reinterpret_cast<float*>(sm + wy::TF);
    float* sX = reinterpret_cast<float*>(sm + wy::SX);
    unsigned char* TT = sm + wy::TT;
    unsigned char* PP = sm + wy::PP;
    unsigned char* WM = sm + wy::WM;
    const uint32_t lane_base = tmem + ((uint32_t)(tm_quarter(warp) * 32) << 16);
    const uint32_t sTT = tc::smem_u32(TT);
    constexpr uint32_t ID_M1 = tc::idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_M2 = tc::idesc_bf16(64, 128, false, true);
    const int units = p.BH * p.nc;

    // The four tiles of unit u, issued by lane 0 of warps 0-2 (a TMA issue takes ~100 cycles). q and
    // log_alpha land on Qt and Kt of the stage, which the previous image stores read: thread 32 issues
    // them (part 2) only after waiting for those reads.
    auto tile_coords = [&](int u, int& b, int& h, int& t0) {
        const int c = u / p.BH, head = u % p.BH;
        b = head / p.H; h = head % p.H; t0 = c * C;
    };
    auto issue_loads_1 = [&](int stage, int u) {
        if (lane != 0 || (warp != 0 && warp != 2)) return;
        int b, h, t0;
        tile_coords(u, b, h, t0);
        unsigned char* base = sm + stage * wy::STAGE;
        if (warp == 0) {
            tc::mbar_arrive_expect_tx(&bar_in[stage], PROD_LOAD_BYTES);
            tma_tile(base + wy::QE, 2 * C, 0, &m.b, b, h, t0, &bar_in[stage]);
        } else {
            tma_tile(base + wy::KH, C, 0, &m.k, b, h, t0, &bar_in[stage]);
        }
    };
    auto issue_loads_2 = [&](int stage, int u) {   // lane 0 of warps 1 and 2
        if (lane != 0 || (warp != 1 && warp != 2)) return;
        int b, h, t0;
        tile_coords(u, b, h, t0);
        unsigned char* base = sm + stage * wy::STAGE;
        if (warp == 1) tma_tile(base + wy::QE, 2 * C, C, &m.q, b, h, t0, &bar_in[stage]);
        else tma_tile(base + wy::KT, C, 0, &m.la, b, h, t0, &bar_in[stage]);
    };
    if (pid < units) {
        issue_loads_1(0, pid);
        issue_loads_2(0, pid);
    }

    uint32_t ph_in = 0, ph_mma = 0;   // ph_in: bit s = phase parity of input stage s
    auto wait_mma = [&]() {
        if (!tc::mbar_wait(bar_mma, ph_mma)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 1u); }
        ph_mma ^= 1;
        tc::tc_fence_after();
    };
    int stage = 0;
    bool pending = false;   // a prefetch into the other stage is in flight (thread 0's view)
    // The WY image of a unit is written by bulk stores that thread 32 issues at the end of the unit; the
    // same thread sets the unit's flag one unit later (once the stores are complete) and, before any
    // tile they read is overwritten, waits until they have read it.
    long long unreleased = -1;   // unit whose WY image is being written but whose flag is not yet set
    for (int u = pid; u < units; u += p.nprod, stage ^= 1) {
        const int c = u / p.BH, head = u % p.BH;
        unsigned char* base = sm + stage * wy::STAGE;
        unsigned char* QE = base + wy::QE;
        if (!tc::mbar_wait(&bar_in[stage], (ph_in >> stage) & 1u)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 2u); }
        ph_in ^= 1u << stage;
        // the other stage was last read by the previous unit's MMAs, which have completed, and by its image
        // stores: b and k do not overlap what those read; q and log_alpha follow below
        pending = u + p.nprod < units;
        if (pending) issue_loads_1(stage ^ 1, u + p.nprod);

        gate_prep(QE, base + wy::KH, base + wy::KT, nullptr, nullptr, reinterpret_cast<float*>(sm + wy::GC + stage * 512),
                  sA, tid, true, false);
        // the previous image stores have read T | P | Wm (rewritten after this barrier) and the other
        // stage's Qt, Kt (reloaded below)
        if (tid == 32) tc::bulk_wait_read();
        sync_for_mma();
        const uint32_t sQE = tc::smem_u32(QE), sKT = tc::smem_u32(base + wy::KT);
        if (tid == 0) {   // [A; P] = [Et; Qt] Kt^T
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_AP, tc::desc_k(sQE, 2 * C, 0, kk), tc::desc_k(sKT, C, 0, kk), ID_M1, kk > 0);
            tc::mma_commit(bar_mma);
        }
        // while M1 runs, warps 1 and 2 (outside the MMA-issuing warp) issue the prefetch's q and log_alpha
        // (the image stores have read the tiles they overwrite: thread 32 waited before the barrier), and
        // thread 32 sets the previous unit's flag (its image stores have completed during this unit's prep)
        if (pending) issue_loads_2(stage ^ 1, u + p.nprod);
        if (tid == 32 && unreleased >= 0 && !*abort_flag) tc::flag_release_after_bulk(p.flags + unreleased, 1u);
        unreleased = -1;
        wait_mma();
        extract_AP(lane_base + TM_AP, sA, PP, true, warp, lane);
        tc::tc_fence_before();
        __syncthreads();
        solve_unit_lower(sA, sTf, sX, TT, tid);   // T = (I + A)^{-1}
        sync_for_mma();
        if (tid == 0) {   // Wm = T Et
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_W, tc::desc_k(sTT, C, 0, kk), tc::desc_mn(sQE, 2 * C, 0, kk), ID_M2, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_mma();
        tmem_m64_to_tile(lane_base + TM_W, WM, warp, lane);
        tc::fence_async_smem();   // the tiles written by threads are read by the image's bulk stores
        tc::tc_fence_before();
        __syncthreads();
        // the WY image of (head, c): T | P | Wm, then Qt (rows 64..127 of the [b; q] tile, whose two 64-channel
        // panels are 16 KB apart), Kt and gC, by bulk stores
        const size_t unit = (size_t)head * p.nc + c;
        if (tid == 32) {
            unsigned char* img = p.wyimg + unit * TC_WY_BYTES;
            tc::bulk_store(img, sm + wy::IMG, 32768u);
            tc::bulk_store(img + TC_WY_QT, QE + 8192, 8192u);
            tc::bulk_store(img + TC_WY_QT + 8192, QE + 16384 + 8192, 8192u);
            tc::bulk_store(img + TC_WY_KT, base + wy::KT, 16384u);
            tc::bulk_store(img + TC_WY_GC, sm + wy::GC + stage * 512, 512u);
            tc::bulk_commit();
        }
        unreleased = (long long)unit;
        if (*abort_flag) break;
        pending = false;
    }
    if (tid == 32) {   // the last unit's flag; every image store completes before the CTA leaves
        if (unreleased >= 0 && !*abort_flag) tc::flag_release_after_bulk(p.flags + unreleased, 1u);
        tc::bulk_wait_all();
    }
    // after an abort: let the prefetch in flight land before the CTA's shared memory is released
    if (tid == 0 && pending) (void)tc::mbar_wait(&bar_in[stage ^ 1], (ph_in >> (stage ^ 1)) & 1u);
}

// ------------------------------------------------------------------ consumer
__device__ void run_consumer(const Maps& m, const FwdParams& p, unsigned char* sm, uint32_t tmem, int cid) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    unsigned char* UU = sm + sp::UU;
    unsigned char* WW = sm + sp::WW;
    unsigned char* STt = sm + sp::ST;
    unsigned char* DT = sm + sp::DT;
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + sp::BAR);
    uint64_t* bar_mma = bar_load + 1;
    int* abort_flag = reinterpret_cast<int*>(sm + sp::BAR + 28);
    const uint32_t lane_base = tmem + ((uint32_t)(tm_quarter(warp) * 32) << 16);   // this warp's TMEM lanes
    const int jrow = 32 * tm_quarter(warp) + lane, cpart = 64 * tm_part(warp);      // lane row, column half
    const int T = p.T, H = p.H, nc = p.nc;
    const bool want_o = (p.o != nullptr);

    const uint32_t sUU = tc::smem_u32(UU), sST = tc::smem_u32(STt), sDT = tc::smem_u32(DT),
                   sTT = tc::smem_u32(sm + sp::TT), sPP = tc::smem_u32(sm + sp::PP), sWM = tc::smem_u32(sm + sp::WM);
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
    // thread 0 waits for the WY image of (head, c); the caller synchronises the CTA afterwards
    auto wait_wy = [&](size_t head, int c) {
        if (!tc::flag_wait(p.flags + head * nc + c, 1u)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 4u); }
    };
    // the WY image of (head, c): T | P | Wm to WY, Qt and Kt to this chunk's parity buffers, gC
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
        tc::cp_async_commit();
    };

    for (int headi = cid; headi < p.BH; headi += p.ncons) {
        const size_t head = (size_t)headi;
        const int h = headi % H, b = headi / H;
        // v and w of chunk c (issued by lane 0 of warps 0 and 1 at once; a TMA issue takes ~100 cycles)
        auto issue_loads = [&](int c) {
            if (lane != 0 || warp > 1) return;
            const int t0 = c * C;
            if (warp == 0) {
                tc::mbar_arrive_expect_tx(bar_load, CONS_LOAD_BYTES);
                tma_tile(UU, C, 0, &m.v, b, h, t0, bar_load);
            } else {
                tma_tile(WW, C, 0, &m.w, b, h, t0, bar_load);
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
                tc::tmem_wait_ld();
                if (lane < 16 && t < L) {
                    uint4* dst = reinterpret_cast<uint4*>(p.o + tok_off(b, t0 + t, h, T, H, D) + c0);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        dst[g] = make_uint4(tc::pack_bf16x2(v[8 * g], v[8 * g + 1]), tc::pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                            tc::pack_bf16x2(v[8 * g + 4], v[8 * g + 5]), tc::pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
                }
            }
        };
        issue_loads(0);
        if (tid == 0) wait_wy(head, 0);
        // initial state: S^T row j = column j of S0
        {
            const int j = jrow;
            float v[32];
#pragma unroll 1
            for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = p.S0 ? p.S0[(head * D + i0 + u) * D + j] : 0.f;
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
        copy_wy(head, 0);
        if (p.states && tid == 0) {
            tc::bulk_store(p.states + (head * nc + 0) * TC_STATE_BYTES, STt, (uint32_t)TC_STATE_BYTES);
            tc::bulk_commit();
        }

        int c = 0;
        for (; c < nc; ++c) {
            const int par = c & 1;
            const uint32_t sQQ = tc::smem_u32(sm + sp::QQ + par * TILE_64x128),
                           sKT = tc::smem_u32(sm + sp::KT + par * TILE_64x128);
            const float* sGC = reinterpret_cast<const float*>(sm + sp::GC + par * 512);
            const uint32_t tm_o = tmem + TM_O + 128 * par;
            if (!tc::mbar_wait(bar_load, ph_load)) { atomicExch(abort_flag, 1); atomicOr(&g_fwd_error, 2u); }
            ph_load ^= 1;

            // ---- U = w * v (Qt, Kt and gC come with the WY image): 4 row chunks of 8 values per thread
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int idx = tid + NT * e, row = idx >> 4, g = idx & 15;
                float vv[8], ww[8];
                tc::ld_row8(UU, C, row, g, vv);
                tc::ld_row8(WW, C, row, g, ww);
#pragma unroll
                for (int x = 0; x < 8; ++x) vv[x] *= ww[x];
                tc::st_row8(UU, C, row, g, vv);
            }
            tc::cp_async_wait_all();   // this chunk's WY image
            sync_for_mma();

            // ---- M3: Delta^T := U^T T^T ;  M4: Delta^T -= S^T Wm^T  (commit) ;  M5: O = Qt S
            if (tid == 0) {
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_D, tc::desc_mn(sUU, C, 0, kk), tc::desc_k(sTT, C, 0, kk), ID_M3, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_D, tc::desc_k(sST, D, 0, kk), tc::desc_k(sWM, C, 0, kk), ID_M4, 1);
                tc::mma_commit(bar_mma);
                if (want_o) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16(tm_o, tc::desc_k(sQQ, C, 0, kk), tc::desc_k(sST, D, 0, kk), ID_M56, kk > 0);
                }
                if (c + 1 < nc) wait_wy(head, c + 1);   // overlaps the MMAs
            }
            if (want_o && c > 0) store_o(c - 1);      // previous chunk's output, in the MMAs' shadow
            wait_mma();
            // v (read by M3) and w are free: prefetch the next chunk's
            if (c + 1 < nc) issue_loads(c + 1);
            tmem_to_tile_rows<64>(lane_base + TM_D, DT, warp, lane);   // Delta^T (lane j) -> bf16 rows
            sync_for_mma();
            if (p.deltas && tid == 0) {   // Delta^T of this chunk for the backward
                tc::bulk_store(p.deltas + (head * nc + c) * TC_DELTA_BYTES, DT, (uint32_t)TC_DELTA_BYTES);
                tc::bulk_commit();
            }

            // ---- M6: O += P Delta ;  M7: Z^T = S^T + Delta^T Kt
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
            // S'^T = Z^T Diag(gC): scale the fp32 state, keep a bf16 copy for the next chunk (the bulk
            // stores of the previous state image and of this chunk's Delta^T must have read their tiles)
            if (p.states && tid == 0) tc::bulk_wait_read();
            __syncthreads();   // also orders thread 0's flag acquire before the image copy
            if (c + 1 < nc) copy_wy(head, c + 1);
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
            if (p.states && tid == 0 && c + 1 < nc) {
                tc::bulk_store(p.states + (head * nc + c + 1) * TC_STATE_BYTES, STt, (uint32_t)TC_STATE_BYTES);
                tc::bulk_commit();
            }
            if (*abort_flag) {   // let the next chunk's loads land before leaving
                if (tid == 0 && c + 1 < nc) (void)tc::mbar_wait(bar_load, ph_load);
                break;
            }
        }
        if (want_o && c == nc) store_o(nc - 1);

        // final state (fp32): ST[i][j] from S^T (lane j)
        if (p.ST) {
            const int j = jrow;
            float v[32];
#pragma unroll 1
            for (int i0 = cpart; i0 < cpart + 64; i0 += 32) {
                tc::tmem_ld32(lane_base + TM_S + i0, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) p.ST[(head * D + i0 + u) * D + j] = v[u];
            }
        }
        tc::cp_async_wait_all();
        if (p.states && tid == 0) tc::bulk_wait_all();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        if (*abort_flag) break;
    }
}

__global__ void __launch_bounds__(NT, 1) chunk_fwd_kernel(const __grid_constant__ Maps maps, const FwdParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays in the shared window
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool consumer = (int)blockIdx.x < p.ncons;
    const uint32_t bar_off = consumer ? sp::BAR : wy::BAR;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + bar_off);
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(sm + bar_off + 24);
    int* abort_flag = reinterpret_cast<int*>(sm + bar_off + 28);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) tc::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&maps.q); tc::tma_prefetch_desc(&maps.k); tc::tma_prefetch_desc(&maps.la);
        if (consumer) { tc::tma_prefetch_desc(&maps.v); tc::tma_prefetch_desc(&maps.w); }
        else tc::tma_prefetch_desc(&maps.b);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base_ptr, TM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_base_ptr;
    if (consumer) run_consumer(maps, p, sm, tmem, blockIdx.x);
    else run_producer(maps, p, sm, tmem, blockIdx.x - p.ncons);
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
    Maps maps;
    const void* ptrs[6] = {a.q, a.k, a.v, a.la, a.b, a.w};
    CUtensorMap* mp[6] = {&maps.q, &maps.k, &maps.v, &maps.la, &maps.b, &maps.w};
    for (int i = 0; i < 6; ++i)
        if (make_token_map(mp[i], ptrs[i], d.B, d.T, d.H) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, coop = 0, occ = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, chunk_fwd_kernel, NT, SMEM_BYTES)) != cudaSuccess)
        return e;
    const int BH = d.B * d.H, nc = d.nchunks();
    const int units = BH * nc;
    const int slots = nsm * occ;

    FwdParams p{};
    p.T = d.T; p.H = d.H; p.BH = BH; p.nc = nc;
    p.S0 = a.S0; p.o = static_cast<__nv_bfloat16*>(a.o); p.ST = a.ST;
    p.states = a.states; p.deltas = a.deltas; p.wyimg = a.wy; p.flags = a.flags;
    if ((e = cudaMemsetAsync(a.flags, 0, (size_t)units * sizeof(unsigned int), s)) != cudaSuccess) return e;

    TraceScope trace(K_CHUNK_FWD, s);
    // Heads share the launch with the producers while the producers keep pace: per chunk step the
    // BH consumer chunks take about as long as BH WY units spread over the remaining CTAs.
    if (coop && !cooperative_disabled() && slots >= 2 && 16 * BH <= 9 * slots) {
        p.ncons = BH;
        p.nprod = slots - BH < units ? slots - BH : units;
        void* args[2] = {&maps, &p};
        e = cudaLaunchCooperativeKernel((const void*)chunk_fwd_kernel, dim3(p.ncons + p.nprod), dim3(NT), args,
                                        SMEM_BYTES, s);
        if (e == cudaSuccess) return cudaSuccess;
        (void)cudaGetLastError();   // not launched: fall back to two launches
    }
    FwdParams pp = p;   // producers only
    pp.ncons = 0;
    pp.nprod = units < slots ? units : slots;
    chunk_fwd_kernel<<<pp.nprod, NT, SMEM_BYTES, s>>>(maps, pp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    FwdParams pc = p;   // consumers only; every flag is set when they start
    pc.ncons = BH;
    pc.nprod = 0;
    chunk_fwd_kernel<<<BH, NT, SMEM_BYTES, s>>>(maps, pc);
    return cudaGetLastError();
}

}  // namespace gdn2
