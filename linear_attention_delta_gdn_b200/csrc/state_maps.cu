// state_maps.cu -- chaining the affine maps of sequence pieces.
//
// A piece of a sequence maps its start state to its end state as S_end = M S_start + N (and its backward
// the end gradient to the start gradient as dS_start = A dS_end + B); the maps themselves come from the
// chunk kernels (chunk_fwd_map_launch, and the backward's map mode). Chaining them is one small product
// per head: dst = M src + N, fp32, 128 x 128 x 128 at most -- a few microseconds, far from any roofline
// that matters next to the pieces themselves.
#include <cuda_runtime.h>

#include "internal.h"

namespace gdn2 {
namespace {

constexpr int AF_COLS = 16;      // state columns per CTA
constexpr int AF_THREADS = 256;

// CTA = (head, block of 16 state columns). The CTA reads its column block of src into shared memory before
// any thread writes, so dst may alias src (other CTAs touch other columns) and N (each element is read by
// the thread that then writes it).
__global__ void __launch_bounds__(AF_THREADS) state_affine_kernel(const float* __restrict__ M, const float* N,
                                                                   const float* src, float* dst, int Dk, int Dv) {
    __shared__ float col[TC_D * AF_COLS];   // Dk <= 128
    const size_t head = blockIdx.x;
    const int cb = blockIdx.y * AF_COLS;
    const size_t mo = head * Dk * Dk, so = head * Dk * Dv;
    for (int i = threadIdx.x; i < Dk * AF_COLS; i += AF_THREADS) {
        const int r = i / AF_COLS, c = i % AF_COLS;
        col[i] = (src && cb + c < Dv) ? src[so + (size_t)r * Dv + cb + c] : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < Dk * AF_COLS; i += AF_THREADS) {
        const int r = i / AF_COLS, c = i % AF_COLS;
        if (cb + c >= Dv) continue;
        const size_t o = so + (size_t)r * Dv + cb + c;
        float acc = N ? N[o] : 0.f;
        const float* mr = M + mo + (size_t)r * Dk;
        for (int kk = 0; kk < Dk; ++kk) acc = fmaf(mr[kk], col[kk * AF_COLS + c], acc);
        dst[o] = acc;
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
    TraceScope trace(K_STATE_AFFINE, s);
    state_affine_kernel<<<dim3(BH, (Dv + AF_COLS - 1) / AF_COLS), AF_THREADS, 0, s>>>(M, N, src, dst, Dk, Dv);
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
