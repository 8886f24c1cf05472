// state_maps.cu -- chaining the affine maps of sequence pieces.
//
// A piece of a sequence maps its start state to its end state as S_end = M S_start + N (and its backward
// the end gradient to the start gradient as dS_start = A dS_end + B); the maps themselves come from the
// chunk kernels (chunk_fwd_map_launch, and the backward's map mode). Chaining them is one small product
// per head: dst = M src + N, fp32, Dk x Dk times Dk x Dv.
#include <cuda_runtime.h>

#include "internal.h"

namespace gdn2 {
namespace {

constexpr int AF_COLS = 16;      // state columns per CTA
constexpr int AF_THREADS = 128;  // thread = (row group rq = tid / 4: rows rq + 32 r; column quarter cq = tid % 4)

// CTA = (head, block of 16 state columns). M goes to shared memory (rows padded by 4 floats, so the 8 rows a
// warp reads at once fall in distinct bank groups) and the CTA's column block of src beside it, both before
// any thread writes; so dst may alias src (other CTAs touch other columns) and N (each element is read by the
// thread that then writes it). Each thread keeps a (Dk / 32) x 4 block of sums in registers.
__global__ void __launch_bounds__(AF_THREADS) state_affine_kernel(const float* __restrict__ M, const float* N,
                                                                   const float* src, float* dst, int Dk, int Dv) {
    extern __shared__ float4 af_smem[];
    const int LD = Dk + 4;
    float* Ms = reinterpret_cast<float*>(af_smem);   // [Dk][LD]
    float* Sc = Ms + Dk * LD;                        // [Dk][AF_COLS]
    const size_t head = blockIdx.x;
    const int cb = blockIdx.y * AF_COLS;
    const int tid = threadIdx.x, cq = tid & 3, rq = tid >> 2;
    const float4* M4 = reinterpret_cast<const float4*>(M + head * Dk * Dk);
    const size_t so = head * Dk * Dv;
    for (int idx = tid; idx < Dk * Dk / 4; idx += AF_THREADS) {
        const int r = idx / (Dk / 4), c4 = idx % (Dk / 4);
        *reinterpret_cast<float4*>(Ms + r * LD + 4 * c4) = M4[idx];
    }
    for (int e = tid; e < Dk * AF_COLS; e += AF_THREADS) {
        const int r = e / AF_COLS, c = e % AF_COLS;
        Sc[e] = src ? src[so + (size_t)r * Dv + cb + c] : 0.f;
    }
    __syncthreads();
    const int rows = Dk / 32 > 0 ? Dk / 32 : 1;   // rows per thread (Dk = 16: threads rq < 16 take one)
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][e] = 0.f;
    for (int l = 0; l < Dk; l += 4) {
        float4 sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) sv[u] = *reinterpret_cast<const float4*>(Sc + (l + u) * AF_COLS + 4 * cq);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = rq + 32 * r;
            if (r >= rows || i >= Dk) break;
            const float4 m = *reinterpret_cast<const float4*>(Ms + i * LD + l);
            const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[r][0] += mv[u] * sv[u].x;
                acc[r][1] += mv[u] * sv[u].y;
                acc[r][2] += mv[u] * sv[u].z;
                acc[r][3] += mv[u] * sv[u].w;
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = rq + 32 * r;
        if (r >= rows || i >= Dk) break;
        const size_t o = so + (size_t)i * Dv + cb + 4 * cq;
        float4 n = N ? *reinterpret_cast<const float4*>(N + o) : make_float4(0.f, 0.f, 0.f, 0.f);
        n.x += acc[r][0]; n.y += acc[r][1]; n.z += acc[r][2]; n.w += acc[r][3];
        *reinterpret_cast<float4*>(dst + o) = n;
    }
}

// dst = I per head ([Dk][Dk]).
__global__ void identity_kernel(float* dst, int Dk, size_t total) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i % ((size_t)Dk * Dk);
        dst[i] = (e / Dk == e % Dk) ? 1.f : 0.f;
    }
}

}  // namespace

cudaError_t state_affine_launch(const float* M, const float* N, const float* src, float* dst, int BH, int Dk, int Dv,
                                cudaStream_t s) {
    if (BH <= 0) return cudaSuccess;
    const int smem = (Dk * (Dk + 4) + Dk * AF_COLS) * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(state_affine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    TraceScope trace(K_STATE_AFFINE, s);
    state_affine_kernel<<<dim3(BH, (Dv + AF_COLS - 1) / AF_COLS), AF_THREADS, smem, s>>>(M, N, src, dst, Dk, Dv);
    return cudaGetLastError();
}

cudaError_t state_identity_launch(float* dst, int BH, int Dk, cudaStream_t s) {
    const size_t total = (size_t)BH * Dk * Dk;
    if (total == 0) return cudaSuccess;
    const size_t blocks = (total + 255) / 256;
    TraceScope trace(K_STATE_AFFINE, s);
    identity_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(dst, Dk, total);
    return cudaGetLastError();
}

}  // namespace gdn2
