// tc.cuh -- inline-PTX wrappers for sm_100a: tcgen05 (TMEM, UMMA), TMA, mbarriers,
// and the shared-memory tile layout used by the chunkwise kernels.
//
// Tile layout ("row tile"): a bf16 matrix of R rows and 64*P columns is stored
// as P panels of R x 64; panel p holds columns [64p, 64p+64). Each row of a
// panel is 128 bytes, and the 16-byte chunk g of row r sits at chunk position
// g ^ (r % 8) (the 128-byte swizzle of TMA and UMMA). Every tile starts on a
// 1024-byte boundary. One tile serves as
//   * a K-major UMMA operand (rows = M or N index, columns = K index): per
//     16-wide K step kk the descriptor starts at panel kk/4, byte (kk%4)*32 of
//     the row, SBO = 1024 (8-row groups), LBO unused;
//   * an MN-major UMMA operand (rows = K index, columns = M or N index): per K
//     step kk the descriptor starts at row 16*kk, LBO = panel stride R*128
//     (next 64 M/N elements), SBO = 1024 (next 8 K rows).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace gdn2 {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ row-tile addressing

// byte offset of element (r, c) inside a row tile with R rows
__device__ __forceinline__ uint32_t tile_off(int R, int r, int c) {
    return (uint32_t)((c >> 6) * R * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}
// byte offset of the 16-byte chunk holding columns [8g, 8g+8) of row r
__device__ __forceinline__ uint32_t tile_chunk_off(int R, int r, int g) {
    return (uint32_t)((g >> 3) * R * 128 + r * 128 + (((g & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ float ld_bf16(const unsigned char* tile, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + off));
}
__device__ __forceinline__ void st_bf16(unsigned char* tile, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16*>(tile + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// store 8 consecutive columns [8g, 8g+8) of row r
__device__ __forceinline__ void st_row8(unsigned char* tile, int R, int r, int g, const float* x) {
    uint4 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    v.z = pack_bf16x2(x[4], x[5]);
    v.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(tile + tile_chunk_off(R, r, g)) = v;
}
// store / load 4 consecutive columns [4g, 4g+4) of row r (8 bytes, half of a 16-byte chunk)
__device__ __forceinline__ void st_row4(unsigned char* tile, int R, int r, int g, const float* x) {
    uint2 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    *reinterpret_cast<uint2*>(tile + tile_chunk_off(R, r, g >> 1) + ((g & 1) << 3)) = v;
}
__device__ __forceinline__ void ld_row4(const unsigned char* tile, int R, int r, int g, float* x) {
    uint2 v = *reinterpret_cast<const uint2*>(tile + tile_chunk_off(R, r, g >> 1) + ((g & 1) << 3));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void ld_row8(const unsigned char* tile, int R, int r, int g, float* x) {
    uint4 v = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(R, r, g));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// ------------------------------------------------------------ UMMA descriptors

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;          // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;          // SWIZZLE_128B
    return d;
}
// K-major operand from a row tile (R rows) starting at row r0, K step kk
__device__ __forceinline__ uint64_t desc_k(uint32_t tile, int R, int r0, int kk) {
    return sdesc(tile + (uint32_t)((kk >> 2) * R * 128 + r0 * 128 + (kk & 3) * 32), 16, 1024);
}
// MN-major operand from a row tile (R rows): K rows start at r0, K step kk
__device__ __forceinline__ uint64_t desc_mn(uint32_t tile, int R, int r0, int kk) {
    return sdesc(tile + (uint32_t)((r0 + 16 * kk) * 128), (uint32_t)(R * 128), 1024);
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn, bool neg_a = false) {
    return (1u << 4)                       // D format: f32
           | (1u << 7)                     // A format: bf16
           | (1u << 10)                    // B format: bf16
           | ((neg_a ? 1u : 0u) << 13)     // negate A
           | ((a_mn ? 1u : 0u) << 15)      // A major: 0 = K, 1 = MN
           | ((b_mn ? 1u : 0u) << 16)      // B major
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// ------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier once all previously issued MMAs of this thread are complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// tcgen05.ld fills its destination registers asynchronously: they may be read only after
// tcgen05.wait::ld. The wait takes the arrays that the outstanding loads fill and, after the wait
// instruction, marks each of their registers as rewritten (an empty asm), so that the compiler cannot
// schedule any use of them (a conversion, a multiply) above the wait.
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}
template <typename... Arrays>
__device__ __forceinline__ void tmem_wait_ld(Arrays&... arrays) {
    static_assert(sizeof...(Arrays) > 0, "name the registers the loads fill");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    (reg_fence(arrays), ...);
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Warp-wide: each thread reads 8 / 16 / 32 consecutive 32-bit columns of its own lane. The loads write
// straight into the caller's float registers (no copy that could be scheduled before the wait).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
          "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    tmem_ld16(taddr, v);
    tmem_ld16(taddr + 16, v + 16);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    tmem_st16(taddr, v);
    tmem_st16(taddr + 16, v + 16);
}

// ------------------------------------------------------------ mbarriers, fences

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase with parity `phase` to complete. Gives up after ~2 s and
// returns false (the caller records an error and stops).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase) {
    const uint32_t addr = smem_u32(bar);
    uint32_t done = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(phase)
        : "memory");
    if (done) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr), "r"(phase)
            : "memory");
        if (done) return true;
        if (global_timer_ns() - t0 > 2000000000ull) return false;
    }
}
// Named barrier `id` over `count` threads (a multiple of 32), in the non-aligned form: every thread
// counts on its own, so it is correct even when a warp arrives diverged, e.g. right after a block that
// only one of its threads executes (the aligned bar.sync would count the whole warp at once).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t count) {
    asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also returns whether `pred` held on any participating thread (the same answer on
// every thread, so a loop can leave on it without splitting the threads that synchronise on `id`).
__device__ __forceinline__ bool named_sync_or(uint32_t id, uint32_t count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\tbarrier.red.or.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
// Make generic-proxy shared-memory writes visible to the async proxy (UMMA, TMA).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ TMA and bulk copies

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
// Tiled shared -> global copy of one box (current bulk group). Elements outside the tensor are skipped.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3, const void* src) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(map),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// Contiguous global -> shared copy (16-byte aligned, size multiple of 16), completes on bar.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Contiguous shared -> global copy in the current bulk group.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until the shared-memory sources of all committed bulk stores may be reused
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// same, for all but the most recently committed bulk group
__device__ __forceinline__ void bulk_wait_read_but1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// wait until all committed bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 16-byte global -> shared copy through L2 only (not L1), completed by cp_async_wait_all().
__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// 4-byte global -> shared copy (through L1); with valid false the 4 bytes are zeros and src is not read.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// all committed groups but the most recent one are complete
__device__ __forceinline__ void cp_async_wait_but1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// ------------------------------------------------------------ flags between CTAs of one launch
// Publishing: every thread writes its data, __syncthreads(), then one thread calls flag_release
// (a gpu-scope acq_rel fence orders the whole CTA's earlier writes before the flag store).
__device__ __forceinline__ void flag_release(unsigned int* flag, unsigned int value) {
    asm volatile("fence.acq_rel.gpu;\n\tst.relaxed.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(value) : "memory");
}
// Same, for data this thread wrote with bulk (async-proxy) stores: wait until they are complete, order
// them before the thread's generic accesses (proxy fence), then release the flag.
__device__ __forceinline__ void flag_release_after_bulk(unsigned int* flag, unsigned int value) {
    asm volatile("cp.async.bulk.wait_group 0;\n\tfence.proxy.async.global;\n\tfence.acq_rel.gpu;\n\t"
                 "st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(value) : "memory");
}
// Same, when the most recent bulk group belongs to later data: waits for all groups but that one.
__device__ __forceinline__ void flag_release_after_bulk_but1(unsigned int* flag, unsigned int value) {
    asm volatile("cp.async.bulk.wait_group 1;\n\tfence.proxy.async.global;\n\tfence.acq_rel.gpu;\n\t"
                 "st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(value) : "memory");
}
__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* flag) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    return v;
}
// One thread waits until *flag == value (acquire), then the CTA synchronises before reading the
// published data. Gives up after ~2 s and returns false.
__device__ __forceinline__ bool flag_wait(const unsigned int* flag, unsigned int value) {
    if (ld_acquire(flag) == value) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire(flag) == value) return true;
        if (global_timer_ns() - t0 > 2000000000ull) return false;
    }
}

}  // namespace tc
}  // namespace gdn2
