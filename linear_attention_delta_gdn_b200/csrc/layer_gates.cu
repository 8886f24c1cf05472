// layer_gates.cu -- the gate activations of a Gated DeltaNet-2 layer, between its input projection and the
// operator, and their backward.
//
// The pages describe the layer only as the operator plus "two additional per-channel gate computations" (the
// erase gate b_t in [0,1]^{d_k} and the write gate w_t in [0,1]^{d_v}, GitHub README method bullets; the
// aiexpert.news article attributes the overhead over KDA to them) next to KDA's channel-wise decay. The
// plainest reading, used here: one projection z = x W_in per token gives, per head, the pre-activations
// [z_q | z_k | z_v | z_b | z_w | z_a] (widths Dk, Dk, Dv, Dk, Dv, Dk), and
//   q = z_q / ||z_q||,  k = z_k / ||z_k||   (L2 norm over the head's channels, eps 1e-6 under the root)
//   v = z_v,  b = sigmoid(z_b),  w = sigmoid(z_w),  log_alpha = -softplus(z_a + a_bias)
// with an optional per-(head, channel) decay bias (fp32 [H][Dk]; a layer sets the decay's resting rate with it).
// Backward: dz_q = (dq - q (q.dq)) / ||z_q|| (same for k), dz_v = dv, dz_b = db b (1 - b),
// dz_w = dw w (1 - w), dz_a = -dlog_alpha sigmoid(z_a + a_bias) (the bias gradient is the sum of dz_a).
//
// Two (token, head) rows per warp, one per half-warp: HBM-bound elementwise work with two half-warp reductions
// (the norms); every lane moves 16-byte pieces, a row's loads all in flight before any arithmetic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace gdn2 {
namespace {

constexpr int GT_WARPS = 8;   // warps per CTA
constexpr float GT_EPS = 1e-6f;

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }
// softplus(x) = log(1 + e^x), computed as max(x, 0) + log1p(e^{-|x|}) so that it neither overflows nor loses
// the small values
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x))); }

// 16-byte pieces of a row: E = 8 bf16 or 4 fp32 values.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    __device__ static void store(__nv_bfloat16* p, const float (&v)[8]) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};
template <> struct Vec16<float> {
    static constexpr int E = 4;
    __device__ static void load(const float* p, float (&v)[4]) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
    __device__ static void store(float* p, const float (&v)[4]) { *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]); }
};

// sum over the 16 lanes of a half-warp (the lanes of one row)
__device__ __forceinline__ float half_sum(float x) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Two rows per warp, one per half-warp: lane hl = lane % 16 of a half takes the 16-byte pieces hl + 16 m of every
// segment of its row, so each warp instruction works on one segment (one activation, no divergence) and moves
// 2 x 16 x 16 contiguous bytes; the six segments' pieces are loaded before any arithmetic. M = pieces per lane
// and segment for d <= 128 (1 for bf16, 2 for fp32).
template <typename Tin>
__global__ void __launch_bounds__(32 * GT_WARPS) gates_fwd_kernel(const Tin* __restrict__ z, Tin* __restrict__ q,
                                                                  Tin* __restrict__ k, Tin* __restrict__ v,
                                                                  Tin* __restrict__ b, Tin* __restrict__ w,
                                                                  Tin* __restrict__ la, const float* __restrict__ abias,
                                                                  long long rows, int H, int Dk, int Dv) {
    constexpr int E = Vec16<Tin>::E, M = 128 / E / 16;
    const int hl = threadIdx.x & 15;
    const int W = 4 * Dk + 2 * Dv;
    const int width[6] = {Dk, Dk, Dv, Dk, Dv, Dk};
    const int start[6] = {0, Dk, 2 * Dk, 2 * Dk + Dv, 3 * Dk + Dv, 3 * Dk + 2 * Dv};
    Tin* const outs[6] = {q, k, v, b, w, la};
    const long long nwarps = (long long)gridDim.x * GT_WARPS;
    for (long long r2 = (long long)blockIdx.x * GT_WARPS + (threadIdx.x >> 5); 2 * r2 < rows; r2 += nwarps) {
        const long long r = 2 * r2 + ((threadIdx.x >> 4) & 1);
        const bool live = r < rows;
        const Tin* zr = z + (live ? r : 0) * W;
        float x[6][M][E];
#pragma unroll
        for (int s = 0; s < 6; ++s)
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const int pc = hl + 16 * m;
                if (live && pc * E < width[s]) Vec16<Tin>::load(zr + start[s] + pc * E, x[s][m]);
                else {
#pragma unroll
                    for (int e = 0; e < E; ++e) x[s][m][e] = 0.f;
                }
            }
        float nq = 0.f, nk = 0.f;
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int e = 0; e < E; ++e) { nq += x[0][m][e] * x[0][m][e]; nk += x[1][m][e] * x[1][m][e]; }
        const float iq = rsqrtf(half_sum(nq) + GT_EPS), ik = rsqrtf(half_sum(nk) + GT_EPS);
        if (!live) continue;
        const float* bb = abias ? abias + (size_t)(r % H) * Dk : nullptr;
#pragma unroll
        for (int s = 0; s < 6; ++s)
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const int pc = hl + 16 * m;
                if (pc * E >= width[s]) continue;
                float y[E];
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float t = x[s][m][e];
                    y[e] = s == 0 ? t * iq : s == 1 ? t * ik : s == 2 ? t : (s == 3 || s == 4) ? sigmoid_f(t)
                                                                                              : -softplus_f(t + (bb ? bb[pc * E + e] : 0.f));
                }
                Vec16<Tin>::store(outs[s] + r * width[s] + pc * E, y);
            }
    }
}

// The backward: one warp per row (8-byte pieces per lane, 4 values per segment and lane): with the z and
// gradient pieces of a whole row held at once (as the forward does), its registers would leave half the warps.
template <typename T> struct Vec4;
template <> struct Vec4<__nv_bfloat16> {
    __device__ static void load(const __nv_bfloat16* p, float (&v)[4]) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
        v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
    }
    __device__ static void store(__nv_bfloat16* p, const float (&v)[4]) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
        uint2 u;
        u.x = *reinterpret_cast<const unsigned int*>(&a);
        u.y = *reinterpret_cast<const unsigned int*>(&b);
        *reinterpret_cast<uint2*>(p) = u;
    }
};
template <> struct Vec4<float> {
    __device__ static void load(const float* p, float (&v)[4]) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
    __device__ static void store(float* p, const float (&v)[4]) { *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]); }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Segment of the pre-activation row: 0 q, 1 k, 2 v, 3 b, 4 w, 5 a, with offsets in the row and in the outputs.
struct Seg {
    int Dk, Dv;
    __device__ int width(int s) const { return (s == 2 || s == 4) ? Dv : Dk; }
    __device__ int begin(int s) const {
        const int w[6] = {Dk, Dk, Dv, Dk, Dv, Dk};
        int o = 0;
        for (int i = 0; i < s; ++i) o += w[i];
        return o;
    }
};

// dz from z, the outputs q, k, b, w (recomputed from z) and their gradients.
template <typename Tin>
__global__ void __launch_bounds__(32 * GT_WARPS) gates_bwd_kernel(const Tin* __restrict__ z, const Tin* __restrict__ dq,
                                                                  const Tin* __restrict__ dk, const Tin* __restrict__ dv,
                                                                  const Tin* __restrict__ db, const Tin* __restrict__ dw,
                                                                  const Tin* __restrict__ dla, const float* __restrict__ abias,
                                                                  Tin* __restrict__ dz, long long rows, int H, int Dk, int Dv) {
    const int lane = threadIdx.x & 31;
    const Seg sg{Dk, Dv};
    const int W = 4 * Dk + 2 * Dv;
    for (long long r = (long long)blockIdx.x * GT_WARPS + (threadIdx.x >> 5); r < rows;
         r += (long long)gridDim.x * GT_WARPS) {
        const Tin* zr = z + r * W;
        Tin* dzr = dz + r * W;
        // norms and the projections q.dq, k.dk (on the unnormalised z: q.dq = (z_q.dq) / ||z_q||)
        float nq = 0.f, nk = 0.f, pq = 0.f, pk = 0.f;
        for (int j = 4 * lane; j < Dk; j += 128) {
            float a[4], c[4], ga[4], gc[4];
            Vec4<Tin>::load(zr + j, a);
            Vec4<Tin>::load(zr + Dk + j, c);
            Vec4<Tin>::load(dq + r * Dk + j, ga);
            Vec4<Tin>::load(dk + r * Dk + j, gc);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                nq += a[e] * a[e]; nk += c[e] * c[e];
                pq += a[e] * ga[e]; pk += c[e] * gc[e];
            }
        }
        const float iq = rsqrtf(warp_sum(nq) + GT_EPS), ik = rsqrtf(warp_sum(nk) + GT_EPS);
        const float sq = warp_sum(pq) * iq * iq, sk = warp_sum(pk) * ik * ik;   // (q.dq) / ||z_q||, as a factor of z_q
        const Tin* const grads[6] = {dq, dk, dv, db, dw, dla};
#pragma unroll
        for (int s = 0; s < 6; ++s) {
            const int D = sg.width(s), o = sg.begin(s);
            for (int j = 4 * lane; j < D; j += 128) {
                float x[4], g[4];
                Vec4<Tin>::load(zr + o + j, x);
                Vec4<Tin>::load(grads[s] + r * D + j, g);
                if (s == 5 && abias) {
                    const float* bb = abias + (size_t)(r % H) * Dk + j;
#pragma unroll
                    for (int e = 0; e < 4; ++e) x[e] += bb[e];
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float t = x[e], gg = g[e];
                    float d;
                    if (s == 0) d = (gg - t * sq) * iq;
                    else if (s == 1) d = (gg - t * sk) * ik;
                    else if (s == 2) d = gg;
                    else if (s == 5) d = -gg * sigmoid_f(t);
                    else { const float y = sigmoid_f(t); d = gg * y * (1.f - y); }
                    x[e] = d;
                }
                Vec4<Tin>::store(dzr + o + j, x);
            }
        }
    }
}

int gates_grid(long long rows) {
    static int nsm = 0;
    if (!nsm) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            nsm = 148;
    }
    const long long want = ((rows + 1) / 2 + GT_WARPS - 1) / GT_WARPS;   // a warp takes two rows
    const long long cap = (long long)nsm * 16;   // 16 CTAs of 8 warps per SM: full occupancy, grid-stride beyond
    return (int)(want < cap ? want : cap);
}

}  // namespace

cudaError_t gates_fwd_launch(const void* z, void* q, void* k, void* v, void* b, void* w, void* la, const float* abias,
                             long long rows, int H, int Dk, int Dv, gdn2_dtype dt, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    TraceScope trace(K_LAYER_GATES, s);
    const int grid = gates_grid(rows);
    if (dt == GDN2_BF16) {
        using T = __nv_bfloat16;
        gates_fwd_kernel<T><<<grid, 32 * GT_WARPS, 0, s>>>(static_cast<const T*>(z), static_cast<T*>(q), static_cast<T*>(k),
                                                           static_cast<T*>(v), static_cast<T*>(b), static_cast<T*>(w),
                                                           static_cast<T*>(la), abias, rows, H, Dk, Dv);
    } else {
        gates_fwd_kernel<float><<<grid, 32 * GT_WARPS, 0, s>>>(static_cast<const float*>(z), static_cast<float*>(q),
                                                               static_cast<float*>(k), static_cast<float*>(v),
                                                               static_cast<float*>(b), static_cast<float*>(w),
                                                               static_cast<float*>(la), abias, rows, H, Dk, Dv);
    }
    return cudaGetLastError();
}

cudaError_t gates_bwd_launch(const void* z, const void* dq, const void* dk, const void* dv, const void* db, const void* dw,
                             const void* dla, const float* abias, void* dz, long long rows, int H, int Dk, int Dv,
                             gdn2_dtype dt, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    TraceScope trace(K_LAYER_GATES_BWD, s);
    const int grid = gates_grid(rows);
    if (dt == GDN2_BF16) {
        using T = __nv_bfloat16;
        gates_bwd_kernel<T><<<grid, 32 * GT_WARPS, 0, s>>>(static_cast<const T*>(z), static_cast<const T*>(dq),
                                                           static_cast<const T*>(dk), static_cast<const T*>(dv),
                                                           static_cast<const T*>(db), static_cast<const T*>(dw),
                                                           static_cast<const T*>(dla), abias, static_cast<T*>(dz), rows, H,
                                                           Dk, Dv);
    } else {
        gates_bwd_kernel<float><<<grid, 32 * GT_WARPS, 0, s>>>(static_cast<const float*>(z), static_cast<const float*>(dq),
                                                               static_cast<const float*>(dk), static_cast<const float*>(dv),
                                                               static_cast<const float*>(db), static_cast<const float*>(dw),
                                                               static_cast<const float*>(dla), abias, static_cast<float*>(dz),
                                                               rows, H, Dk, Dv);
    }
    return cudaGetLastError();
}

}  // namespace gdn2
