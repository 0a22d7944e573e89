// One-token decode step of the delta-rule family on a resident fp32 state.
//
// For streaming inference the state S of every head stays in HBM between tokens and one
// call applies exactly one step of the per-token recurrence to it:
//     S' = S diag(a)          a = 1 (DeltaNet), alpha (GDN), alpha[:] (KDA)
//     r  = v - S' k           residual against the decayed state
//     S  = S' + beta r k^T    (plain linear attention: S = S + v k^T)
//     o  = S q                readout after the write
// Gated DeltaNet-2 takes e = b (.) k for k and z = w (.) v for v; u = beta r (the write
// value) is optionally stored.
// Rows of S are independent given (q, k, v[i], alpha, beta), so the step streams S once
// from HBM and back: the bound is HBM bandwidth (2*dv*dk*4 bytes per head per token).
// A warp owns 4 consecutive rows of one head; lane l holds key channels
// [l*EPL, (l+1)*EPL) of each row (EPL = DK/32), so every row is one coalesced
// 4*DK-byte access, and the row dot products are warp reductions, four rows at a time.
#pragma once

#include "common.cuh"
#include "dr_sequential.cuh"

namespace drscan {

constexpr int DEC_ROWS = 4;     // rows of S per warp
constexpr int DEC_WARPS = 8;    // warps per CTA
constexpr int DEC_THREADS = 32 * DEC_WARPS;

template <int EPL>
__device__ __forceinline__ void ld_f32(const float* p, float* x) {
    if constexpr (EPL == 4) {
        const float4 t = *reinterpret_cast<const float4*>(p);
        x[0] = t.x, x[1] = t.y, x[2] = t.z, x[3] = t.w;
    } else if constexpr (EPL == 2) {
        const float2 t = *reinterpret_cast<const float2*>(p);
        x[0] = t.x, x[1] = t.y;
    } else {
        x[0] = *p;
    }
}

template <int EPL>
__device__ __forceinline__ void st_f32(float* p, const float* x) {
    if constexpr (EPL == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    } else if constexpr (EPL == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
        *p = x[0];
    }
}

template <typename TIn, int EPL>
__device__ __forceinline__ void ld_in(const TIn* p, float* x) {
    if constexpr (sizeof(TIn) == 4) {
        ld_f32<EPL>(reinterpret_cast<const float*>(p), x);
    } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) x[e] = to_f32<TIn>(p[e]);
    }
}

// grid: ceil(B*H*dv / (DEC_ROWS*DEC_WARPS)); block: DEC_THREADS. dv is a multiple of 32, so
// the DEC_ROWS rows of a warp belong to one head.
template <typename TIn, int MODE, int DK>
__global__ void __launch_bounds__(DEC_THREADS) dr_decode_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ gate,
    const float* __restrict__ erase, const float* __restrict__ write, const float* S_in,
    float* S_out, TIn* __restrict__ out, TIn* __restrict__ u_out, long rows, int dv) {
    constexpr int EPL = DK / 32;
    const int lane = threadIdx.x & 31;
    const long r0 = ((long)blockIdx.x * DEC_WARPS + (threadIdx.x >> 5)) * DEC_ROWS;
    if (r0 >= rows) return;
    const long bh = r0 / dv;
    const int i0 = (int)(r0 - bh * dv);
    const int c0 = lane * EPL;  // first key channel of this lane

    float kk[EPL], qq[EPL], a[EPL];
    ld_in<TIn, EPL>(k + bh * DK + c0, kk);
    ld_in<TIn, EPL>(q + bh * DK + c0, qq);
    if constexpr (MODE == DR_GDN2) {
        float eb[EPL];
        ld_f32<EPL>(erase + bh * DK + c0, eb);
#pragma unroll
        for (int e = 0; e < EPL; ++e) kk[e] *= eb[e];
    }
    if constexpr (MODE == DR_KDA) {
        ld_f32<EPL>(gate + bh * DK + c0, a);
    } else {
        const float g = (MODE == DR_GDN || MODE == DR_GDN2) ? gate[bh] : 1.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a[e] = g;
    }
    const float b = MODE == DR_LINEAR ? 1.f : beta[bh];

    float s[DEC_ROWS][EPL], vi[DEC_ROWS];
#pragma unroll
    for (int j = 0; j < DEC_ROWS; ++j) {
        const long row = r0 + j;
        if (S_in) {
            ld_f32<EPL>(S_in + row * DK + c0, s[j]);
        } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[j][e] = 0.f;
        }
        vi[j] = to_f32<TIn>(v[bh * dv + i0 + j]);
        if constexpr (MODE == DR_GDN2) vi[j] *= write[bh * dv + i0 + j];
    }
    // prediction (S' k)_i, reduced over the warp for the four rows at once
    float p[DEC_ROWS];
#pragma unroll
    for (int j = 0; j < DEC_ROWS; ++j) {
        p[j] = 0.f;
        if constexpr (MODE != DR_LINEAR) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                s[j][e] *= a[e];
                p[j] = fmaf(s[j][e], kk[e], p[j]);
            }
        }
    }
    if constexpr (MODE != DR_LINEAR) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int j = 0; j < DEC_ROWS; ++j) p[j] += __shfl_xor_sync(0xffffffffu, p[j], off);
    }
    // write, then the readout (S q)_i
    float o[DEC_ROWS], u[DEC_ROWS];
#pragma unroll
    for (int j = 0; j < DEC_ROWS; ++j) {
        const float w = MODE == DR_LINEAR ? vi[j] : b * (vi[j] - p[j]);
        u[j] = w;
        o[j] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            s[j][e] = fmaf(w, kk[e], s[j][e]);
            o[j] = fmaf(s[j][e], qq[e], o[j]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int j = 0; j < DEC_ROWS; ++j) o[j] += __shfl_xor_sync(0xffffffffu, o[j], off);
    if (S_out) {
#pragma unroll
        for (int j = 0; j < DEC_ROWS; ++j) st_f32<EPL>(S_out + (r0 + j) * DK + c0, s[j]);
    }
    if (lane < DEC_ROWS) {
        float oj = o[0], uj = u[0];
#pragma unroll
        for (int j = 1; j < DEC_ROWS; ++j) {
            oj = lane == j ? o[j] : oj;
            uj = lane == j ? u[j] : uj;
        }
        out[bh * dv + i0 + lane] = from_f32<TIn>(oj);
        if (u_out) u_out[bh * dv + i0 + lane] = from_f32<TIn>(uj);
    }
}

}  // namespace drscan
