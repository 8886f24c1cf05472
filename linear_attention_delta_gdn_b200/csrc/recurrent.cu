// recurrent.cu -- token-recurrent fp32 kernels of the Gated Delta Rule-2 operator.
//
//  * decode step: one token per (b, h), state [Dk, Dv] fp32 read from and written
//    back to HBM (the constant-memory decoding of "Gated DeltaNet-2: Decoupling
//    Erase and Write in Linear Attention", arXiv abstract). Memory-bound: 128-bit
//    coalesced loads/stores of the state, column reductions through shared memory.
//  * forward / backward over whole sequences with fp32 arithmetic throughout,
//    used for fp32 inputs (where bf16 tensor-core operands would not meet an fp32
//    accuracy budget) and for shapes outside the tensor-core path.
//
// Recurrence (GitHub README method bullets: erase gate b on the key side of the
// decayed state, write gate w on the value side, channel-wise decay alpha):
//     P = Diag(alpha_t) S_{t-1};  r = P^T (b_t*k_t);  S_t = P + k_t (w_t*v_t - r)^T;  o_t = S_t^T q_t
//
// Thread layout (all three kernels): a CTA owns one (b, h); thread tid owns the
// float4 column group c4 = tid % C4 (C4 = Dv/4) and the rows
// i = tid / C4 + r * (NT / C4), r < RPT, of the d_k x d_v state, kept in registers.
// Sums over rows (r_j, o_j, ddelta_j) go through shared memory; sums over
// columns (dq_i, dk_i, de_i, dlog_alpha_i) are shuffles among the C4 lanes of a row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

template <int DK, int DV>
struct Layout {
    static constexpr int C4 = DV / 4;                                  // float4 groups per row
    static constexpr int NT = (DK * C4 >= 256) ? 256 : DK * C4;        // threads per CTA
    static constexpr int RSTEP = NT / C4;                              // rows per pass
    static constexpr int RPT = DK / RSTEP;                             // rows per thread
    static_assert(DV % 4 == 0 && C4 <= 32 && (32 % C4) == 0, "Dv/4 must divide 32");
    static_assert(NT % C4 == 0 && DK % RSTEP == 0, "bad layout");
};

// Sum of a value over the C4 consecutive lanes that hold one state row.
template <int C4>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int m = C4 / 2; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// Per-token vectors staged in shared memory.
template <int DK, int DV>
struct TokVec {
    float q[DK], k[DK], alpha[DK], e[DK], b[DK], la[DK];
    float u[DV], v[DV], w[DV], dout[DV], delta[DV], ddelta[DV];
};

template <typename Tin, int DK, int DV>
__device__ __forceinline__ void load_tok(TokVec<DK, DV>& tv, const Tin* q, const Tin* k,
                                         const Tin* v, const Tin* la, const Tin* b, const Tin* w,
                                         const Tin* dout, int tid, int nt) {
    for (int i = tid; i < DK; i += nt) {
        float kk = to_f32(k[i]), bb = to_f32(b[i]), l = to_f32(la[i]);
        tv.q[i] = to_f32(q[i]);
        tv.k[i] = kk;
        tv.b[i] = bb;
        tv.la[i] = l;
        tv.alpha[i] = expf(l);
        tv.e[i] = bb * kk;
    }
    for (int j = tid; j < DV; j += nt) {
        float vv = to_f32(v[j]), ww = to_f32(w[j]);
        tv.v[j] = vv;
        tv.w[j] = ww;
        tv.u[j] = ww * vv;
        if (dout) tv.dout[j] = to_f32(dout[j]);
    }
}

// Column sums over all rows: each thread contributes part[4] for its columns.
// red is [RSTEP][DV]; result lands in out[DV]. Ends with a barrier.
template <int DK, int DV>
__device__ __forceinline__ void col_sum(float (*red)[DV], const float part[4], float* out, int tid) {
    using L = Layout<DK, DV>;
    const int c4 = tid % L::C4, rs = tid / L::C4;
#pragma unroll
    for (int c = 0; c < 4; ++c) red[rs][c4 * 4 + c] = part[c];
    __syncthreads();
    for (int j = tid; j < DV; j += L::NT) {
        float s = 0.f;
#pragma unroll 8
        for (int r = 0; r < L::RSTEP; ++r) s += red[r][j];
        out[j] = s;
    }
    __syncthreads();
}

// One recurrence step on the register-resident state S (rows owned by this
// thread). Writes delta_j to tv.delta and, if o != nullptr, o_j.
template <typename Tin, int DK, int DV>
__device__ __forceinline__ void fwd_step(float (&S)[Layout<DK, DV>::RPT][4], TokVec<DK, DV>& tv,
                                         float (*red)[DV], Tin* o, int tid) {
    using L = Layout<DK, DV>;
    const int c4 = tid % L::C4, r0 = tid / L::C4;
    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < L::RPT; ++r) {
        const int i = r0 + r * L::RSTEP;
        const float a = tv.alpha[i], e = tv.e[i];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            S[r][c] *= a;                 // P = Diag(alpha) S
            part[c] += S[r][c] * e;       // r_j = sum_i P_ij e_i
        }
    }
    col_sum<DK, DV>(red, part, tv.delta, tid);
    for (int j = tid; j < DV; j += L::NT) tv.delta[j] = tv.u[j] - tv.delta[j];   // delta = u - r
    __syncthreads();
    float dl[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) { dl[c] = tv.delta[c4 * 4 + c]; part[c] = 0.f; }
#pragma unroll
    for (int r = 0; r < L::RPT; ++r) {
        const int i = r0 + r * L::RSTEP;
        const float kk = tv.k[i], qq = tv.q[i];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            S[r][c] += kk * dl[c];        // S = P + k delta^T
            part[c] += S[r][c] * qq;      // o = S^T q
        }
    }
    if (o) {
        float* osum = tv.ddelta;          // scratch
        col_sum<DK, DV>(red, part, osum, tid);
        for (int j = tid; j < DV; j += L::NT) o[j] = from_f32<Tin>(osum[j]);
    }
}

template <int DK, int DV>
__device__ __forceinline__ void load_state(float (&S)[Layout<DK, DV>::RPT][4], const float* src, int tid) {
    using L = Layout<DK, DV>;
    const int c4 = tid % L::C4, r0 = tid / L::C4;
#pragma unroll
    for (int r = 0; r < L::RPT; ++r) {
        const int i = r0 + r * L::RSTEP;
        if (src) {
            float4 x = reinterpret_cast<const float4*>(src + (size_t)i * DV)[c4];
            S[r][0] = x.x; S[r][1] = x.y; S[r][2] = x.z; S[r][3] = x.w;
        } else {
            S[r][0] = S[r][1] = S[r][2] = S[r][3] = 0.f;
        }
    }
}

template <int DK, int DV>
__device__ __forceinline__ void store_state(const float (&S)[Layout<DK, DV>::RPT][4], float* dst, int tid) {
    using L = Layout<DK, DV>;
    const int c4 = tid % L::C4, r0 = tid / L::C4;
#pragma unroll
    for (int r = 0; r < L::RPT; ++r) {
        const int i = r0 + r * L::RSTEP;
        reinterpret_cast<float4*>(dst + (size_t)i * DV)[c4] = make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
    }
}

// ---------------------------------------------------------------- decode

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(Layout<DK, DV>::NT)
decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
              const Tin* __restrict__ la, const Tin* __restrict__ b, const Tin* __restrict__ w,
              float* __restrict__ S, Tin* __restrict__ o) {
    using L = Layout<DK, DV>;
    __shared__ TokVec<DK, DV> tv;
    __shared__ float red[L::RSTEP][DV];
    const int tid = threadIdx.x;
    const size_t head = blockIdx.x;
    float* Sh = S + head * DK * DV;
    float St[L::RPT][4];
    load_state<DK, DV>(St, Sh, tid);     // issue the state loads first
    load_tok<Tin, DK, DV>(tv, q + head * DK, k + head * DK, v + head * DV, la + head * DK,
                          b + head * DK, w + head * DV, nullptr, tid, L::NT);
    __syncthreads();
    fwd_step<Tin, DK, DV>(St, tv, red, o + head * DV, tid);
    store_state<DK, DV>(St, Sh, tid);
}

// ---------------------------------------------------------------- forward

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(Layout<DK, DV>::NT)
fwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
           const Tin* __restrict__ la, const Tin* __restrict__ b, const Tin* __restrict__ w,
           const float* __restrict__ S0, Tin* __restrict__ o, float* __restrict__ ST,
           float* __restrict__ states, int T, int H, int chunk) {
    using L = Layout<DK, DV>;
    __shared__ TokVec<DK, DV> tv;
    __shared__ float red[L::RSTEP][DV];
    const int tid = threadIdx.x;
    const int h = blockIdx.x % H, bb = blockIdx.x / H;
    const size_t head = blockIdx.x;
    const int nc = (T + chunk - 1) / chunk;
    float St[L::RPT][4];
    load_state<DK, DV>(St, S0 ? S0 + head * DK * DV : nullptr, tid);
    for (int t = 0; t < T; ++t) {
        if (states && t % chunk == 0)
            store_state<DK, DV>(St, states + (head * nc + t / chunk) * DK * DV, tid);
        const size_t ok = tok_off(bb, t, h, T, H, DK), ov = tok_off(bb, t, h, T, H, DV);
        load_tok<Tin, DK, DV>(tv, q + ok, k + ok, v + ov, la + ok, b + ok, w + ov, nullptr, tid, L::NT);
        __syncthreads();
        fwd_step<Tin, DK, DV>(St, tv, red, o ? o + ov : nullptr, tid);
        __syncthreads();
    }
    if (ST) store_state<DK, DV>(St, ST + head * DK * DV, tid);
}

// ---------------------------------------------------------------- backward
//
// Reverse-mode adjoint of the step, per token going backwards, dS = dL/dS_t:
//   dS += q dout^T ; dq = S_t dout ; dk = dS delta ; ddelta = dS^T k ; dr = -ddelta
//   de = P dr ; dP = dS + e dr^T ; dlog_alpha = rowsum(dP * P) ; dS = Diag(alpha) dP
//   dv = ddelta * w ; dw = ddelta * v ; db = de * k ; dk += de * b
// S_{t-1} comes from a per-chunk recompute out of the chunk-start checkpoints;
// the recomputed states and deltas of the current chunk go to a per-head scratch.

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(Layout<DK, DV>::NT)
bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
           const Tin* __restrict__ la, const Tin* __restrict__ b, const Tin* __restrict__ w,
           const Tin* __restrict__ dout, const float* __restrict__ dST,
           Tin* __restrict__ dq, Tin* __restrict__ dk, Tin* __restrict__ dv, Tin* __restrict__ dla,
           Tin* __restrict__ db, Tin* __restrict__ dw, float* __restrict__ dS0,
           const float* __restrict__ states, float* __restrict__ seg, float* __restrict__ segdelta,
           int T, int H, int chunk) {
    using L = Layout<DK, DV>;
    __shared__ TokVec<DK, DV> tv;
    __shared__ float red[L::RSTEP][DV];
    const int tid = threadIdx.x;
    const int c4 = tid % L::C4, r0 = tid / L::C4;
    const int h = blockIdx.x % H, bb = blockIdx.x / H;
    const size_t head = blockIdx.x;
    const int nc = (T + chunk - 1) / chunk;
    float* segh = seg + head * (size_t)chunk * DK * DV;
    float* segd = segdelta + head * (size_t)chunk * DV;
    float dS[L::RPT][4];
    load_state<DK, DV>(dS, dST ? dST + head * DK * DV : nullptr, tid);
    float St[L::RPT][4];

    for (int c = nc - 1; c >= 0; --c) {
        const int t0 = c * chunk, t1 = min(T, t0 + chunk);
        // recompute: seg[tt] = state before token t0+tt, segd[tt] = delta of token t0+tt
        load_state<DK, DV>(St, states + (head * nc + c) * DK * DV, tid);
        for (int t = t0; t < t1; ++t) {
            store_state<DK, DV>(St, segh + (size_t)(t - t0) * DK * DV, tid);
            const size_t ok = tok_off(bb, t, h, T, H, DK), ov = tok_off(bb, t, h, T, H, DV);
            load_tok<Tin, DK, DV>(tv, q + ok, k + ok, v + ov, la + ok, b + ok, w + ov, nullptr, tid, L::NT);
            __syncthreads();
            fwd_step<Tin, DK, DV>(St, tv, red, static_cast<Tin*>(nullptr), tid);
            for (int j = tid; j < DV; j += L::NT) segd[(size_t)(t - t0) * DV + j] = tv.delta[j];
            __syncthreads();
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const size_t ok = tok_off(bb, t, h, T, H, DK), ov = tok_off(bb, t, h, T, H, DV);
            load_tok<Tin, DK, DV>(tv, q + ok, k + ok, v + ov, la + ok, b + ok, w + ov, dout + ov, tid, L::NT);
            for (int j = tid; j < DV; j += L::NT) tv.delta[j] = segd[(size_t)(t - t0) * DV + j];
            load_state<DK, DV>(St, segh + (size_t)(t - t0) * DK * DV, tid);   // S_{t-1}
            __syncthreads();
            float dl[4], dov[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) { dl[cc] = tv.delta[c4 * 4 + cc]; dov[cc] = tv.dout[c4 * 4 + cc]; }
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            float rq[L::RPT], rk[L::RPT];
#pragma unroll
            for (int r = 0; r < L::RPT; ++r) {
                const int i = r0 + r * L::RSTEP;
                const float a = tv.alpha[i], kk = tv.k[i], qq = tv.q[i];
                float sq = 0.f, sk = 0.f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    St[r][cc] *= a;                                   // P
                    const float s_t = St[r][cc] + kk * dl[cc];        // S_t
                    sq += s_t * dov[cc];                              // dq = S_t dout
                    dS[r][cc] += qq * dov[cc];                        // dS += q dout^T
                    sk += dS[r][cc] * dl[cc];                         // dk = dS delta
                    part[cc] += dS[r][cc] * kk;                       // ddelta = dS^T k
                }
                rq[r] = sq;
                rk[r] = sk;
            }
            col_sum<DK, DV>(red, part, tv.ddelta, tid);
            float dr[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) dr[cc] = -tv.ddelta[c4 * 4 + cc];
            for (int j = tid; j < DV; j += L::NT) {
                dv[ov + j] = from_f32<Tin>(tv.ddelta[j] * tv.w[j]);
                dw[ov + j] = from_f32<Tin>(tv.ddelta[j] * tv.v[j]);
            }
#pragma unroll
            for (int r = 0; r < L::RPT; ++r) {
                const int i = r0 + r * L::RSTEP;
                const float a = tv.alpha[i], e = tv.e[i];
                float sde = 0.f, sla = 0.f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    sde += St[r][cc] * dr[cc];                        // de = P dr
                    const float dp = dS[r][cc] + e * dr[cc];          // dP
                    sla += dp * St[r][cc];                            // rowsum(dP * P)
                    dS[r][cc] = a * dp;                               // dS_{t-1}
                }
                const float sq = row_sum<L::C4>(rq[r]);
                const float sk = row_sum<L::C4>(rk[r]);
                sde = row_sum<L::C4>(sde);
                sla = row_sum<L::C4>(sla);
                if (c4 == 0) {
                    dq[ok + i] = from_f32<Tin>(sq);
                    dk[ok + i] = from_f32<Tin>(sk + sde * tv.b[i]);
                    db[ok + i] = from_f32<Tin>(sde * tv.k[i]);
                    dla[ok + i] = from_f32<Tin>(sla);
                }
            }
            __syncthreads();
        }
    }
    if (dS0) store_state<DK, DV>(dS, dS0 + head * DK * DV, tid);
}

// ---------------------------------------------------------------- dispatch

template <typename Tin, int DK, int DV>
cudaError_t launch_all(const RecurrentArgs& a, cudaStream_t s) {
    using L = Layout<DK, DV>;
    const Dims& d = a.d;
    const unsigned grid = (unsigned)((size_t)d.B * d.H);
    if (grid == 0) return cudaSuccess;
    const Tin* q = static_cast<const Tin*>(a.q);
    const Tin* k = static_cast<const Tin*>(a.k);
    const Tin* v = static_cast<const Tin*>(a.v);
    const Tin* la = static_cast<const Tin*>(a.la);
    const Tin* b = static_cast<const Tin*>(a.b);
    const Tin* w = static_cast<const Tin*>(a.w);
    switch (a.op) {
    case RecurrentArgs::DECODE: {
        TraceScope trace(K_DECODE, s);
        decode_kernel<Tin, DK, DV><<<grid, L::NT, 0, s>>>(q, k, v, la, b, w, a.S, static_cast<Tin*>(a.o));
        break;
    }
    case RecurrentArgs::FWD: {
        TraceScope trace(K_REC_FWD, s);
        fwd_kernel<Tin, DK, DV><<<grid, L::NT, 0, s>>>(q, k, v, la, b, w, a.S0, static_cast<Tin*>(a.o),
                                                       a.ST, a.states, d.T, d.H, d.chunk);
        break;
    }
    case RecurrentArgs::BWD: {
        TraceScope trace(K_REC_BWD, s);
        bwd_kernel<Tin, DK, DV><<<grid, L::NT, 0, s>>>(
            q, k, v, la, b, w, static_cast<const Tin*>(a.dout), a.dST, static_cast<Tin*>(a.dq),
            static_cast<Tin*>(a.dk), static_cast<Tin*>(a.dv), static_cast<Tin*>(a.dla),
            static_cast<Tin*>(a.db), static_cast<Tin*>(a.dw), a.dS0, a.states, a.seg, a.segdelta,
            d.T, d.H, d.chunk);
        break;
    }
    }
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dt(const RecurrentArgs& a, cudaStream_t s) {
    const int dk = a.d.Dk, dv = a.d.Dv;
#define GDN2_CASE(DK_, DV_) \
    if (dk == DK_ && dv == DV_) return launch_all<Tin, DK_, DV_>(a, s);
#define GDN2_ROW(DK_) GDN2_CASE(DK_, 16) GDN2_CASE(DK_, 32) GDN2_CASE(DK_, 64) GDN2_CASE(DK_, 128)
    GDN2_ROW(16) GDN2_ROW(32) GDN2_ROW(64) GDN2_ROW(128)
#undef GDN2_ROW
#undef GDN2_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t recurrent_launch(const RecurrentArgs& a, cudaStream_t s) {
    return a.dt == GDN2_BF16 ? launch_dt<__nv_bfloat16>(a, s) : launch_dt<float>(a, s);
}

}  // namespace gdn2
