// Chunked delta-rule scan on sm_100a tensor cores (DeltaNet, Gated DeltaNet, KDA).
//
// The sequence is cut into chunks of C = 64 tokens. Inside a chunk with entering state
// S0 (dv x dk), g_t the running sum of log-decay (scalar for GDN, per key channel for
// KDA, 0 for DeltaNet) and gamma = exp(g), the per-token recurrence
//     S_t = S_{t-1} diag(a_t) + beta_t (v_t - S_{t-1} diag(a_t) k_t) k_t^T,  o_t = S_t q_t
// is exactly (WY/UT representation of the triangular system of writes)
//     A[t,i] = beta_t (k_t.k_i) gamma_t/gamma_i  (i < t)        strictly lower, C x C
//     P[t,i] = (q_t.k_i) gamma_t/gamma_i          (i <= t)
//     T      = (I + A)^{-1} diag(beta)                          unit-lower solve
//     Y      = V - diag(gamma) K S0^T                           residual vs decayed state
//     O      = diag(gamma) Q S0^T + (P T) Y
//     S_C^T  = diag(gamma_C) S0^T + Khat^T Y,  Khat^T = K^T diag(gamma_C/gamma) T
// (KDA: the decay sits inside the operands, K*gamma, Q*gamma and K/gamma per channel.)
//
// Contractions on tcgen05 (bf16 operands in 128-byte-swizzled shared memory, fp32
// accumulators in tensor memory), one CTA per (b, h, slice of BV value channels):
//   Gram   D_G  = [K;Q] K^T                M=128 N=64 K=128
//   H      D_H  = K^T Ttilde               M=128 N=64 K=64   (A operand M/N-major)
//   PT     D_PT = P T                      M=128 N=64 K=64
//   MMA1   D1   = [K;Q] S0^T               M=128 N=BV K=128
//   MMA2   D2   = [T;PT] Y                 M=128 N=BV K=64
//   MMA3   S^T += Khat^T Y                 M=128 N=BV K=64   (fp32 state stays in TMEM)
// The unit-lower solve runs on CUDA cores in fp32. q/k/v tiles arrive by TMA; rows past
// T are zero-filled by the copy engine and masked in the gate arithmetic.
//
// This version runs the stages of a chunk one after another in a single warpgroup
// (thread r <-> TMEM lane r); loads for the next chunks are in flight meanwhile.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace drscan {

constexpr int CK = 64;    // chunk length
constexpr int CDK = 128;  // key dimension of the chunked kernel

template <int MODE, int BV>
struct ChunkLayout {
    static constexpr bool kKda = MODE == DR_KDA;
    static constexpr int NS = kKda ? 1 : 2;  // input stages
    static constexpr int KQ_B = 32768;       // [K;Q] bf16: 2 panels x 128 rows x 128 B
    static constexpr int KN_B = kKda ? 16384 : 0;
    static constexpr int V_B = CK * BV * 2;
    static constexpr int GATE_B = kKda ? CK * CDK * 4 : 0;

    static constexpr int KQ = 0;
    static constexpr int KN = KQ + NS * KQ_B;        // KDA: K/gamma, 2 panels x 64 rows
    static constexpr int TP = KN + NS * KN_B;        // [T; PT]: 128 rows x 64 cols
    static constexpr int KH = TP + 16384;            // Khat^T: 128 rows (dk) x 64 cols (t)
    static constexpr int PM = KH + 16384;            // P: rows 0-63 (rows 64-127 zero)
    static constexpr int TT = PM + 16384;            // T^T: 64 rows x 64
    static constexpr int TTS = TT + 8192;            // (diag(gamma_C/gamma) T)^T
    static constexpr int SS = TTS + 8192;            // S bf16: 2 panels x BV rows
    static constexpr int SY = SS + BV * 256;         // Y^T: BV rows x 64 (t)
    static constexpr int V = SY + ((BV * 128 + 1023) / 1024) * 1024;
    static constexpr int GATE = V + NS * V_B;        // KDA gate fp32 [64][128] (then g)
    static constexpr int AM = kKda ? GATE : GATE + NS * GATE_B;  // A fp32 [64][68]
    static constexpr int AM_B = CK * 68 * 4;
    static constexpr int GV = kKda ? GATE + GATE_B : AM + AM_B;  // g, gamma / gamma_C
    static constexpr int BAR = GV + 1024;
    static constexpr int TOTAL = BAR + 128;
    static_assert(!kKda || AM_B <= GATE_B, "A aliases the KDA gate buffer");
    static_assert(TOTAL + 1024 <= 232448, "shared memory budget");

    static constexpr int COL_G = 0;   // D_G, then D_PT
    static constexpr int COL_H = 64;  // D_H
    static constexpr int COL_D1 = 128;
    static constexpr int COL_D2 = 128 + BV;
    static constexpr int COL_S = 128 + 2 * BV;
    static constexpr int NCOLS = (128 + 3 * BV) <= 256 ? 256 : 512;
    static constexpr uint32_t TX_BYTES = KQ_B + V_B + GATE_B;
};

// bf16 bits of 8 consecutive columns of a row, stored as one 16-byte swizzled chunk.
__device__ __forceinline__ void st_row_chunk(uint8_t* panel, int row, int chunk, const float* x) {
    uint4 w;
    w.x = pack_bf16(x[0], x[1]);
    w.y = pack_bf16(x[2], x[3]);
    w.z = pack_bf16(x[4], x[5]);
    w.w = pack_bf16(x[6], x[7]);
    *reinterpret_cast<uint4*>(panel + row * 128 + ((chunk ^ (row & 7)) << 4)) = w;
}

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float ld_bf16(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

template <int MODE, int BV>
__global__ void __launch_bounds__(128, 1) dr_chunked_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmGate,
    const float* __restrict__ beta, const float* __restrict__ gate, const float* __restrict__ S0,
    __nv_bfloat16* __restrict__ out, float* __restrict__ S_final, int T, int dv) {
    using L = ChunkLayout<MODE, BV>;
    constexpr bool kGdn = MODE == DR_GDN;
    constexpr bool kKda = MODE == DR_KDA;
    constexpr int NS = L::NS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);  // [0,NS): full, NS: mma
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::BAR + 64);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::BAR + 80);
    float* sG = reinterpret_cast<float*>(sm + L::GV);        // GDN: g[64]; KDA: gamma_C[128]
    float* sGam = sG + 64;                                    // GDN: gamma[64], gamma_C at [64]
    float* sA = reinterpret_cast<float*>(sm + L::AM);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const long bh = blockIdx.x;
    const int v0 = blockIdx.y * BV;
    const int nchunks = (T + CK - 1) / CK;
    const uint32_t bar_mma = smem_u32(&bars[NS]);

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(smem_u32(&bars[s]), 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        mbar_init_fence();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmV);
        if constexpr (kKda) tma_prefetch_desc(&tmGate);
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_holder), L::NCOLS);
    // P's rows 64-127 are never written: keep them zero.
    for (int e = tid; e < 8192 / 16; e += 128)
        reinterpret_cast<uint4*>(sm + L::PM + 8192)[e] = make_uint4(0, 0, 0, 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t trow = tmem + lane_base;  // this thread's TMEM lane

    auto issue_loads = [&](int chunk, int s) {
        const uint32_t full = smem_u32(&bars[s]);
        mbar_arrive_expect_tx(full, L::TX_BYTES);
        uint8_t* kq = sm + L::KQ + s * L::KQ_B;
        const int t0 = chunk * CK;
        for (int p = 0; p < 2; ++p) {
            tma_load_3d(smem_u32(kq + p * 16384), &tmK, full, p * 64, t0, (int)bh);
            tma_load_3d(smem_u32(kq + p * 16384 + 8192), &tmQ, full, p * 64, t0, (int)bh);
        }
        tma_load_3d(smem_u32(sm + L::V + s * L::V_B), &tmV, full, v0, t0, (int)bh);
        if constexpr (kKda) tma_load_3d(smem_u32(sm + L::GATE), &tmGate, full, 0, t0, (int)bh);
    };

    if (tid == 0) {
        for (int c = 0; c < NS && c < nchunks; ++c) issue_loads(c, c);
    }

    // ---- initial state: S^T row j (lane j = key channel) in TMEM, bf16 copy in smem
    {
        float sv[BV];
        const float* src = S0 ? S0 + (bh * dv + v0) * (long)CDK + tid : nullptr;
#pragma unroll
        for (int v = 0; v < BV; ++v) sv[v] = src ? src[(long)v * CDK] : 0.f;
#pragma unroll
        for (int v = 0; v < BV; ++v) st_bf16(sm + L::SS, sw128_offset(v, tid, BV), sv[v]);
#pragma unroll
        for (int c16 = 0; c16 < BV; c16 += 16) tmem_st16(trow + L::COL_S + c16, sv + c16);
        tmem_wait_st();
    }
    fence_async_smem();

    // per-token scalars of the next chunk, prefetched into registers (threads 0..63)
    float nb = 0.f, ng = 1.f;
    if (tid < CK && tid < T) {
        nb = beta[bh * T + tid];
        if constexpr (kGdn) ng = gate[bh * T + tid];
    }

    uint32_t mma_phase = 0;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
        const int s = c % NS;
        const int t0 = c * CK;
        const int nvalid = min(CK, T - t0);
        const float b_t = nb;  // beta of row t = tid (threads < 64)
        const float a_t = ng;  // alpha of row t (GDN)
        if (tid < CK) {
            const int tn = t0 + CK + tid;
            nb = 0.f;
            ng = 1.f;
            if (tn < T) {
                nb = beta[bh * T + tn];
                if constexpr (kGdn) ng = gate[bh * T + tn];
            }
        }
        uint8_t* kq = sm + L::KQ + s * L::KQ_B;
        uint8_t* kn = sm + L::KN + s * L::KN_B;
        const uint8_t* vt = sm + L::V + s * L::V_B;

        if (!mbar_wait(smem_u32(&bars[s]), (uint32_t)((c / NS) & 1), abort_flag)) {
            ok = false;
            break;
        }

        // ---- gate prefix sums
        if constexpr (kGdn) {
            if (tid < CK) {
                float x = (tid < nvalid) ? logf(a_t) : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if ((tid & 31) >= off) x += y;
                }
                if (tid == 31) sG[200] = x;  // scratch: total of rows 0..31
                sG[tid] = x;
            }
            __syncthreads();
            if (tid >= 32 && tid < CK) sG[tid] += sG[200];
            __syncthreads();
            if (tid < CK) sGam[tid] = expf(sG[tid]);
            if (tid == 0) sGam[64] = expf(sG[CK - 1]);
        } else if constexpr (kKda) {
            // thread j owns key channel j: running log-decay over the chunk's rows; rewrite
            // K and Q in place as K*gamma, Q*gamma and store K/gamma.
            const float* gt = reinterpret_cast<const float*>(sm + L::GATE);
            float run = 0.f;
            for (int t = 0; t < CK; ++t) {
                if (t < nvalid) run += logf(gt[t * CDK + tid]);
                const float e = expf(run);
                const float ei = expf(-run);
                const uint32_t ok_ = sw128_offset(t, tid, 128);
                const uint32_t oq = sw128_offset(64 + t, tid, 128);
                const float kv = ld_bf16(kq, ok_);
                st_bf16(kq, ok_, kv * e);
                st_bf16(kq, oq, ld_bf16(kq, oq) * e);
                st_bf16(kn, sw128_offset(t, tid, 64), kv * ei);
            }
            sG[tid] = expf(run);  // gamma_C per key channel
            fence_async_smem();
        }
        __syncthreads();

        // ---- decay the carried state: S^T row j *= gamma_C (before MMA3 accumulates)
        if constexpr (MODE != DR_DELTANET) {
            const float gC = kKda ? sG[tid] : sGam[64];
            float sv[BV];
#pragma unroll
            for (int c16 = 0; c16 < BV; c16 += 16) tmem_ld16(trow + L::COL_S + c16, sv + c16);
            tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < BV; ++v) sv[v] *= gC;
#pragma unroll
            for (int c16 = 0; c16 < BV; c16 += 16) tmem_st16(trow + L::COL_S + c16, sv + c16);
            tmem_wait_st();
        }

        // ---- Gram: D_G = [K;Q] K^T  (KDA: [K*g; Q*g] (K/g)^T)
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int p = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t a = smem_desc_sw128(smem_u32(kq + p * 16384 + ko), 16, 1024);
                const uint64_t b = kKda ? smem_desc_sw128(smem_u32(kn + p * 8192 + ko), 16, 1024)
                                        : a;
                tc_mma_bf16(tmem + L::COL_G, a, b, idesc, kk > 0);
            }
            tc_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, abort_flag)) {
            ok = false;
            break;
        }
        mma_phase ^= 1;
        tc_fence_after();

        // ---- Gram epilogue: A (fp32, rows 0-63) and P (bf16 operand)
        {
            float gr[64];
#pragma unroll
            for (int c16 = 0; c16 < 64; c16 += 16) tmem_ld16(trow + L::COL_G + c16, gr + c16);
            tmem_wait_ld();
            const int t = tid & 63;
            const float gt = kGdn ? sG[t] : 0.f;
            if (tid < 64) {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    float a = 0.f;
                    if (i < t) a = b_t * gr[i] * (kGdn ? expf(gt - sG[i]) : 1.f);
                    gr[i] = a;
                }
#pragma unroll
                for (int i = 0; i < 64; i += 4)
                    *reinterpret_cast<float4*>(sA + t * 68 + i) =
                        make_float4(gr[i], gr[i + 1], gr[i + 2], gr[i + 3]);
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    float p = 0.f;
                    if (i <= t) p = gr[i] * (kGdn ? expf(gt - sG[i]) : 1.f);
                    gr[i] = p;
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_row_chunk(sm + L::PM, t, ch, gr + ch * 8);
            }
        }
        __syncthreads();

        // ---- UT solve on CUDA cores: column j of X = (I + A)^{-1}; T = X diag(beta)
        if (tid < 64) {
            const int j = tid;
            float x[64];
#pragma unroll
            for (int t = 0; t < 64; ++t) {
                float acc = (t == j) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < t; i += 4) {
                    const float4 a4 = *reinterpret_cast<const float4*>(sA + t * 68 + i);
                    acc = fmaf(-a4.x, x[i], acc);
                    if (i + 1 < t) acc = fmaf(-a4.y, x[i + 1], acc);
                    if (i + 2 < t) acc = fmaf(-a4.z, x[i + 2], acc);
                    if (i + 3 < t) acc = fmaf(-a4.w, x[i + 3], acc);
                }
                x[t] = acc;
            }
#pragma unroll
            for (int t = 0; t < 64; ++t) x[t] *= b_t;  // column j scaled by beta_j
            // [T; PT] rows 0-63 (row t, column j)
#pragma unroll
            for (int t = 0; t < 64; ++t) st_bf16(sm + L::TP, sw128_offset(t, j, 128), x[t]);
            // T^T row j
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_row_chunk(sm + L::TT, j, ch, x + ch * 8);
            if constexpr (kGdn) {
                const float gC = sGam[64];
#pragma unroll
                for (int t = 0; t < 64; ++t) x[t] *= gC / sGam[t];
            }
            if constexpr (!kKda) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_row_chunk(sm + L::TTS, j, ch, x + ch * 8);
            }
        }
        fence_async_smem();
        __syncthreads();

        // ---- H: Khat^T = K^T Ttilde (KDA: (K/g)^T T); PT = P T
        if (tid == 0) {
            constexpr uint32_t idesc_h = idesc_bf16(128, 64, 1, 0);
            constexpr uint32_t idesc_p = idesc_bf16(128, 64, 0, 0);
            const uint8_t* bt = sm + (kKda ? L::TT : L::TTS);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = kKda ? smem_desc_sw128(smem_u32(kn + kk * 2048), 8192, 1024)
                                        : smem_desc_sw128(smem_u32(kq + kk * 2048), 16384, 1024);
                const uint64_t b = smem_desc_sw128(smem_u32(bt + kk * 32), 16, 1024);
                tc_mma_bf16(tmem + L::COL_H, a, b, idesc_h, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_sw128(smem_u32(sm + L::PM + kk * 32), 16, 1024);
                const uint64_t b = smem_desc_sw128(smem_u32(sm + L::TT + kk * 32), 16, 1024);
                tc_mma_bf16(tmem + L::COL_G, a, b, idesc_p, kk > 0);
            }
            tc_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, abort_flag)) {
            ok = false;
            break;
        }
        mma_phase ^= 1;
        tc_fence_after();
        {
            float h[64];
#pragma unroll
            for (int c16 = 0; c16 < 64; c16 += 16) tmem_ld16(trow + L::COL_H + c16, h + c16);
            tmem_wait_ld();
            if constexpr (kKda) {
                const float gC = sG[tid];
#pragma unroll
                for (int i = 0; i < 64; ++i) h[i] *= gC;
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_row_chunk(sm + L::KH, tid, ch, h + ch * 8);
            if (tid < 64) {
#pragma unroll
                for (int c16 = 0; c16 < 64; c16 += 16) tmem_ld16(trow + L::COL_G + c16, h + c16);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_row_chunk(sm + L::TP, 64 + tid, ch, h + ch * 8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- MMA1: D1 = [K;Q] S0^T (KDA: [K*g; Q*g] S0^T)
        if (tid == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, BV, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int p = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t a = smem_desc_sw128(smem_u32(kq + p * 16384 + ko), 16, 1024);
                const uint64_t b =
                    smem_desc_sw128(smem_u32(sm + L::SS + p * (BV * 128) + ko), 16, 1024);
                tc_mma_bf16(tmem + L::COL_D1, a, b, idesc, kk > 0);
            }
            tc_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, abort_flag)) {
            ok = false;
            break;
        }
        mma_phase ^= 1;
        tc_fence_after();

        // ---- residual Y = V - gamma (K S0^T), stored as the B operand Y^T
        if (tid < 64) {
            const int t = tid;
            const float gt = kGdn ? sGam[t] : 1.f;
            float xr[BV];
#pragma unroll
            for (int c16 = 0; c16 < BV; c16 += 16) tmem_ld16(trow + L::COL_D1 + c16, xr + c16);
            tmem_wait_ld();
            const uint4* vrow = reinterpret_cast<const uint4*>(vt + t * BV * 2);
#pragma unroll
            for (int c8 = 0; c8 < BV / 8; ++c8) {
                const uint4 w = vrow[c8];
                const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int v = c8 * 8 + e;
                    st_bf16(sm + L::SY, sw128_offset(v, t, BV),
                            __bfloat162float(hv[e]) - gt * xr[v]);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- MMA2: D2 = [T; PT] Y;  MMA3: S^T += Khat^T Y
        if (tid == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, BV, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_sw128(smem_u32(sm + L::TP + kk * 32), 16, 1024);
                const uint64_t b = smem_desc_sw128(smem_u32(sm + L::SY + kk * 32), 16, 1024);
                tc_mma_bf16(tmem + L::COL_D2, a, b, idesc, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_sw128(smem_u32(sm + L::KH + kk * 32), 16, 1024);
                const uint64_t b = smem_desc_sw128(smem_u32(sm + L::SY + kk * 32), 16, 1024);
                tc_mma_bf16(tmem + L::COL_S, a, b, idesc, 1);
            }
            tc_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, abort_flag)) {
            ok = false;
            break;
        }
        mma_phase ^= 1;
        tc_fence_after();

        // ---- output rows: O = gamma (Q S0^T) + PT Y  (warps 2-3 own rows 64-127)
        if (tid >= 64) {
            const int t = tid - 64;
            const float gt = kGdn ? sGam[t] : 1.f;
#pragma unroll
            for (int c16 = 0; c16 < BV; c16 += 16) {
                float z[16], d[16];
                tmem_ld16(trow + L::COL_D1 + c16, z);
                tmem_ld16(trow + L::COL_D2 + c16, d);
                tmem_wait_ld();
                if (t < nvalid) {
                    uint4 w[2];
                    uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        wp[e] = pack_bf16(fmaf(gt, z[2 * e], d[2 * e]),
                                          fmaf(gt, z[2 * e + 1], d[2 * e + 1]));
                    uint4* dst = reinterpret_cast<uint4*>(out + (bh * T + t0 + t) * (long)dv + v0 +
                                                          c16);
                    dst[0] = w[0];
                    dst[1] = w[1];
                }
            }
        }
        // ---- carried state: bf16 copy for the next MMA1, fp32 S_final after the last chunk
        {
            float sv[BV];
#pragma unroll
            for (int c16 = 0; c16 < BV; c16 += 16) tmem_ld16(trow + L::COL_S + c16, sv + c16);
            tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < BV; ++v) st_bf16(sm + L::SS, sw128_offset(v, tid, BV), sv[v]);
            if (c == nchunks - 1 && S_final) {
                float* dst = S_final + (bh * dv + v0) * (long)CDK + tid;
#pragma unroll
                for (int v = 0; v < BV; ++v) dst[(long)v * CDK] = sv[v];
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && c + NS < nchunks) issue_loads(c + NS, s);
    }

    if (!ok && tid == 0) {
        // give outstanding copies and MMAs a bounded chance to land before TMEM is freed
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 50000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::NCOLS);
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3D map over a [BH, T, inner] row-major tensor, box {box_inner, 64 rows, 1}.
inline bool make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize,
                        long BH, int T, int inner, int box_inner, bool swizzle128) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * T};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)CK, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool chunked_supported(int variant, int dk, int dv) {
    return dk == CDK && (dv == 32 || dv == 64 || dv == 128) &&
           (variant == DR_DELTANET || variant == DR_GDN || variant == DR_KDA);
}

template <int MODE, int BV>
int launch_chunked_bv(const void* q, const void* k, const void* v, const float* beta,
                      const float* gate, const float* S0, void* out, float* S_final, int BH, int T,
                      int dv, cudaStream_t stream) {
    using L = ChunkLayout<MODE, BV>;
    CUtensorMap mk, mq, mv, mg;
    if (!make_map_3d(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, BH, T, CDK, 64, true) ||
        !make_map_3d(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, BH, T, CDK, 64, true) ||
        !make_map_3d(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, BH, T, dv, BV, false))
        return DR_ERR_CUDA;
    mg = mk;
    if (MODE == DR_KDA &&
        !make_map_3d(&mg, gate, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, BH, T, CDK, CDK, false))
        return DR_ERR_CUDA;
    const int smem = L::TOTAL + 1024;
    auto kern = dr_chunked_kernel<MODE, BV>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return DR_ERR_CUDA;
    dim3 grid((unsigned)BH, (unsigned)(dv / BV));
    kern<<<grid, 128, smem, stream>>>(mk, mq, mv, mg, beta, gate, S0,
                                      static_cast<__nv_bfloat16*>(out), S_final, T, dv);
    return cudaGetLastError() == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

// Value-slice width: the widest that still gives about one CTA per SM.
inline int pick_bv(int variant, long BH, int dv) {
    const int opts_gdn[3] = {64, 32, 16};
    const int opts_kda[4] = {128, 64, 32, 16};
    const int* opts = variant == DR_KDA ? opts_kda : opts_gdn;
    const int n = variant == DR_KDA ? 4 : 3;
    int best = opts[n - 1];
    for (int i = n - 1; i >= 0; --i) {
        const int bv = opts[i];
        if (bv > dv) continue;
        if (BH * (dv / bv) >= 111) best = bv;
    }
    return best;
}

template <int MODE>
int launch_chunked_mode(const void* q, const void* k, const void* v, const float* beta,
                        const float* gate, const float* S0, void* out, float* S_final, int BH,
                        int T, int dv, cudaStream_t stream) {
    switch (pick_bv(MODE, BH, dv)) {
        case 16:
            return launch_chunked_bv<MODE, 16>(q, k, v, beta, gate, S0, out, S_final, BH, T, dv,
                                               stream);
        case 32:
            return launch_chunked_bv<MODE, 32>(q, k, v, beta, gate, S0, out, S_final, BH, T, dv,
                                               stream);
        case 64:
            return launch_chunked_bv<MODE, 64>(q, k, v, beta, gate, S0, out, S_final, BH, T, dv,
                                               stream);
        case 128:
            if constexpr (MODE == DR_KDA)
                return launch_chunked_bv<MODE, 128>(q, k, v, beta, gate, S0, out, S_final, BH, T,
                                                    dv, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

inline int launch_chunked(const void* q, const void* k, const void* v, const float* beta,
                          const float* gate, const float* S0, void* out, float* S_final, int BH,
                          int T, int dk, int dv, int variant, cudaStream_t stream) {
    (void)dk;
    switch (variant) {
        case DR_DELTANET:
            return launch_chunked_mode<DR_DELTANET>(q, k, v, beta, gate, S0, out, S_final, BH, T,
                                                    dv, stream);
        case DR_GDN:
            return launch_chunked_mode<DR_GDN>(q, k, v, beta, gate, S0, out, S_final, BH, T, dv,
                                               stream);
        case DR_KDA:
            return launch_chunked_mode<DR_KDA>(q, k, v, beta, gate, S0, out, S_final, BH, T, dv,
                                               stream);
    }
    return DR_ERR_UNSUPPORTED;
}

}  // namespace drscan
