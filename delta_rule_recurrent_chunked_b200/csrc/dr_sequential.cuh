// Per-token delta-rule scan with an fp32 state on CUDA cores.
//
// Every row of S evolves independently given (k_t, alpha_t, beta_t): with
// S' = S_{t-1} diag(a_t), row i of the update is
//     s_i <- a (.) s_i + u_t[i] k_t,   u_t[i] = beta_t (v_t[i] - (a (.) s_i) . k_t)
// and o_t[i] = s_i . q_t (readout after the write). Gated DeltaNet-2 runs the same rows
// with k_t replaced by its erase direction e_t = b_t (.) k_t and v_t by its write target
// z_t = w_t (.) v_t. The write values u_t are optionally stored. One thread owns one row of
// S in registers, so a token costs ~4*dk FMAs per thread and no cross-thread communication.
// A CTA is one warp covering 32 consecutive rows (value channels) of one (b,h); tokens
// are staged through shared memory in tiles and broadcast to the warp. For fp32 inputs
// without per-channel gates the tiles are double-buffered: the next tile is copied with
// cp.async while the current one is scanned.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace drscan {

constexpr int SEQ_TILE = 16;  // tokens staged per shared-memory tile

template <typename TIn>
__device__ __forceinline__ float to_f32(TIn x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
    return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename TIn>
__device__ __forceinline__ TIn from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
    return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// grid: (B*H, dv/32); block: 32 threads.
template <typename TIn, int MODE, int DK>
__global__ void __launch_bounds__(32) dr_sequential_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ gate,
    const float* __restrict__ erase, const float* __restrict__ write,
    const float* __restrict__ S0, TIn* __restrict__ out, float* __restrict__ S_final,
    TIn* __restrict__ u_out, int T, int dv) {
    constexpr bool kScalarGate = MODE == DR_GDN || MODE == DR_GDN2;
    // double-buffered asynchronous tile copies (fp32 inputs, no per-channel gates)
    constexpr bool kAsync = std::is_same<TIn, float>::value && MODE != DR_KDA && MODE != DR_GDN2;
    constexpr int NBUF = kAsync ? 2 : 1;
    __shared__ __align__(16) float skb[NBUF][SEQ_TILE][DK];
    __shared__ __align__(16) float sqb[NBUF][SEQ_TILE][DK];
    __shared__ __align__(16) float sa[MODE == DR_KDA ? SEQ_TILE : 1][MODE == DR_KDA ? DK : 4];
    __shared__ __align__(16) float svb[NBUF][SEQ_TILE][32];
    __shared__ __align__(16) float sbb[NBUF][SEQ_TILE];
    __shared__ __align__(16) float sgb[NBUF][SEQ_TILE];

    const int lane = threadIdx.x;
    const long bh = blockIdx.x;
    const int row = blockIdx.y * 32 + lane;

    const TIn* qh = q + bh * (long)T * DK;
    const TIn* kh = k + bh * (long)T * DK;
    const TIn* vh = v + bh * (long)T * dv;
    TIn* oh = out + bh * (long)T * dv;
    TIn* uh = u_out ? u_out + bh * (long)T * dv : nullptr;

    float s[DK];
    if (S0) {
        const float* src = S0 + (bh * dv + row) * (long)DK;
#pragma unroll
        for (int j = 0; j < DK; j += 4) {
            float4 x = *reinterpret_cast<const float4*>(src + j);
            s[j] = x.x;
            s[j + 1] = x.y;
            s[j + 2] = x.z;
            s[j + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < DK; ++j) s[j] = 0.f;
    }

    // asynchronous copy of the tile starting at token t0c into buffer b: the k and q rows,
    // this warp's 32 value channels of v, and the per-token beta and gate
    auto copy_tile = [&](int t0c, int b) {
        const int ntc = min(SEQ_TILE, T - t0c);
        for (int e = lane; e < ntc * DK / 4; e += 32) {
            const int tt = (4 * e) / DK, j = (4 * e) % DK;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&skb[b][tt][j])),
                         "l"(reinterpret_cast<const float*>(kh) + (long)(t0c + tt) * DK + j)
                         : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&sqb[b][tt][j])),
                         "l"(reinterpret_cast<const float*>(qh) + (long)(t0c + tt) * DK + j)
                         : "memory");
        }
        for (int e = lane; e < ntc * 8; e += 32) {  // 8 pieces of 16 bytes per token
            const int tt = e >> 3, j = 4 * (e & 7);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&svb[b][tt][j])),
                         "l"(reinterpret_cast<const float*>(vh) + (long)(t0c + tt) * dv +
                             blockIdx.y * 32 + j)
                         : "memory");
        }
        if (lane < ntc) {
            if (MODE != DR_LINEAR)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&sbb[b][lane])),
                             "l"(beta + bh * T + t0c + lane)
                             : "memory");
            if (kScalarGate)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&sgb[b][lane])),
                             "l"(gate + bh * T + t0c + lane)
                             : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if constexpr (kAsync) {
        if (T > 0) copy_tile(0, 0);
    }

    for (int t0 = 0, it = 0; t0 < T; t0 += SEQ_TILE, ++it) {
        const int nt = min(SEQ_TILE, T - t0);
        const int cur = kAsync ? (it & 1) : 0;
        float(*sk)[DK] = skb[cur];
        float(*sq)[DK] = sqb[cur];
        float(*sv)[32] = svb[cur];
        float* sb = sbb[cur];
        float* sg = sgb[cur];
        __syncwarp();
        if constexpr (kAsync) {
            // the next tile goes out now; this one's copies are waited for
            if (t0 + SEQ_TILE < T) {
                copy_tile(t0 + SEQ_TILE, cur ^ 1);
                asm volatile("cp.async.wait_group 1;" ::: "memory");
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
        }
        for (int e = lane; e < (kAsync ? 0 : nt * DK); e += 32) {
            const int tt = e / DK, j = e % DK;
            const long kt = (bh * T + t0 + tt) * (long)DK + j;
            sk[tt][j] = to_f32(kh[(long)(t0 + tt) * DK + j]);
            if constexpr (MODE == DR_GDN2) sk[tt][j] *= erase[kt];  // e = b (.) k
            sq[tt][j] = to_f32(qh[(long)(t0 + tt) * DK + j]);
            if constexpr (MODE == DR_KDA) sa[tt][j] = gate[kt];
        }
        if constexpr (!kAsync) {
            for (int tt = 0; tt < nt; ++tt) {
                float x = to_f32(vh[(long)(t0 + tt) * dv + row]);
                if constexpr (MODE == DR_GDN2) x *= write[(bh * T + t0 + tt) * (long)dv + row];  // z
                sv[tt][lane] = x;
            }
        }
        if (lane < nt) {
            if (!kAsync || MODE == DR_LINEAR) sb[lane] = (MODE == DR_LINEAR) ? 1.f : beta[bh * T + t0 + lane];
            if (!kAsync || !kScalarGate) sg[lane] = kScalarGate ? gate[bh * T + t0 + lane] : 1.f;
        }
        __syncwarp();

        for (int tt = 0; tt < nt; ++tt) {
            const float vi = sv[tt][lane];
            if constexpr (MODE == DR_LINEAR) {
#pragma unroll
                for (int j = 0; j < DK; ++j) s[j] = fmaf(vi, sk[tt][j], s[j]);
                if (uh) uh[(long)(t0 + tt) * dv + row] = from_f32<TIn>(vi);
            } else {
                if constexpr (kScalarGate) {
                    const float a = sg[tt];
#pragma unroll
                    for (int j = 0; j < DK; ++j) s[j] *= a;
                } else if constexpr (MODE == DR_KDA) {
#pragma unroll
                    for (int j = 0; j < DK; ++j) s[j] *= sa[tt][j];
                }
                float p0 = 0.f, p1 = 0.f;
#pragma unroll
                for (int j = 0; j < DK; j += 2) {
                    p0 = fmaf(s[j], sk[tt][j], p0);
                    p1 = fmaf(s[j + 1], sk[tt][j + 1], p1);
                }
                const float w = sb[tt] * (vi - (p0 + p1));
#pragma unroll
                for (int j = 0; j < DK; ++j) s[j] = fmaf(w, sk[tt][j], s[j]);
                if (uh) uh[(long)(t0 + tt) * dv + row] = from_f32<TIn>(w);
            }
            float o0 = 0.f, o1 = 0.f;
#pragma unroll
            for (int j = 0; j < DK; j += 2) {
                o0 = fmaf(s[j], sq[tt][j], o0);
                o1 = fmaf(s[j + 1], sq[tt][j + 1], o1);
            }
            oh[(long)(t0 + tt) * dv + row] = from_f32<TIn>(o0 + o1);
        }
    }

    if (S_final) {
        float* dst = S_final + (bh * dv + row) * (long)DK;
#pragma unroll
        for (int j = 0; j < DK; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
    }
}

}  // namespace drscan
