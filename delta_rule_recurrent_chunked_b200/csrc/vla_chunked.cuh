// Chunked Variational Linear Attention scan, fp32, C = 64 tokens per chunk, two kernels.
//
// A-phase (vla_aphase_kernel, one CTA per (b,h)). Over a chunk with entering inverse penalty
// A_c, the Sherman-Morrison steps of its tokens add up to the Woodbury identity
//     A_t = A_c - A_c U_{<=t}^T (I + U_{<=t} A_c U_{<=t}^T)^-1 U_{<=t} A_c,
// where U_{<=t} holds the chunk's u rows up to token t. With the Cholesky factor
// M = I + U A_c U^T = L L^T (positive definite, every pivot >= 1 for a positive definite A_c)
// and W = L^-1 U A_c, the leading t rows of W depend on the leading t rows of U alone, so
//     A_t k_t = A_c k_t - sum_{s<=t} w_s (w_s . k_t),   A_{c+1} = A_c - W^T W,
// and the write directions of the whole chunk are Y = K A_c - tril(K W^T) W, normalised by
// rows. Everything but the 64 x 64 factorisation is a dense product; the serial chain per
// token of the per-token recurrence becomes a 16 x 16 register factorisation per 16 tokens.
// The directions go to a scratch array in global memory, one row per token.
//
// S-phase (vla_sphase_kernel, one CTA per (b,h) and 32 rows of S). Given the directions,
// S_t = S_{t-1} + r_t alpha_hat_t^T with r_t = v_t - S_{t-1} k_t is a delta rule whose read
// key k_t and write key alpha_hat_t differ. Over a chunk entering with S_c:
//     (I + G) R = V - K S_c^T,  G = strictly lower part of K Alpha^T,
//     O = Q S_c^T + tril(Q Alpha^T) R,   S_{c+1} = S_c + R^T Alpha,
// the WY form of the chunked delta rule with two keys. Rows of S are independent given the
// directions, so the state is split over CTAs by rows. The ratio readout's n_t follows the
// same write with its value held at 1: it is one more row of the state in every CTA, and
// the readout divides by its output n_t q_t.
//
// Fused (vla_fused_kernel, one cluster per (b,h)): the A-phase CTA keeps only what the next
// chunk needs, [U A_c; K A_c], M, its factor and A_{c+1}; it hands W and K A_c to the S-phase
// CTAs of the cluster, each of which forms Y and the directions itself before its S-phase
// step. Every CTA of a cluster runs one of the two phases at a time, on its own SM.
//
// Everything is fp32 on CUDA cores: the tolerance of fp32 inputs is below what one tf32
// tensor-core pass keeps.
#pragma once

#include "common.cuh"

namespace drscan {

constexpr int VC_C = 64;          // tokens per chunk
constexpr int VC_THREADS = 256;   // threads of either kernel
constexpr int VC_RS = 32;         // rows of S per S-phase CTA

// Copies nrows token rows of D floats (row-major) into a padded shared-memory tile with
// 16-byte asynchronous copies; rows from nvalid on are filled with zeros.
template <int D>
__device__ __forceinline__ void vc_load_rows(float (*dst)[D + 4], const float* src, int nvalid,
                                             int tid) {
    constexpr int V4 = D / 4;
    for (int e = tid; e < VC_C * V4; e += VC_THREADS) {
        const int r = e / V4, c4 = e - r * V4;
        const uint32_t d = smem_u32(&dst[r][4 * c4]);
        const bool ok = r < nvalid;
        const float* s = ok ? src + (long)r * D + 4 * c4 : src;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(s),
                     "r"(ok ? 16 : 0)
                     : "memory");
    }
}

// Same for a slice of columns [c0, c0 + W) of rows of D floats.
template <int D, int W>
__device__ __forceinline__ void vc_load_cols(float (*dst)[W + 4], const float* src, int c0,
                                             int nvalid, int tid) {
    constexpr int V4 = W / 4;
    for (int e = tid; e < VC_C * V4; e += VC_THREADS) {
        const int r = e / V4, c4 = e - r * V4;
        const uint32_t d = smem_u32(&dst[r][4 * c4]);
        const bool ok = r < nvalid;
        const float* s = ok ? src + (long)r * D + c0 + 4 * c4 : src;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(s),
                     "r"(ok ? 16 : 0)
                     : "memory");
    }
}

__device__ __forceinline__ void vc_wait_copies() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// N consecutive floats of a shared-memory row (N in {1, 2, 4, 6, 8}; p aligned to
// 8 bytes, and to 16 when N is a multiple of 4).
template <int N>
__device__ __forceinline__ void vc_ld(const float* p, float* x) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 f = *reinterpret_cast<const float4*>(p + i);
            x[i] = f.x;
            x[i + 1] = f.y;
            x[i + 2] = f.z;
            x[i + 3] = f.w;
        }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            const float2 f = *reinterpret_cast<const float2*>(p + i);
            x[i] = f.x;
            x[i + 1] = f.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) x[i] = p[i];
    }
}

__device__ __forceinline__ float vc_comp(const float4& f, int q) {
    return q == 0 ? f.x : (q == 1 ? f.y : (q == 2 ? f.z : f.w));
}

// ---- cluster hand-off of the write directions (fused kernel)
// Once a chunk's Cholesky factor is done, one thread of the A-phase CTA (cluster rank 0)
// copies its W and K A_c tiles (adjacent in shared memory) into a slot pair of every S-phase
// CTA (ranks 1 ..) with one bulk copy that completes its bytes on that CTA's `full` barrier
// of the pair. An S-phase CTA arms that barrier (expected bytes) for the pair's next chunk
// before it hands the pair back by arriving on the A-phase CTA's `empty` barrier of the pair. Every wait is bounded (mbar-style, with the
// CTA's abort flag); after a timeout a CTA stops sending and receiving and runs its loops to
// the end, so every thread reaches the cluster barrier that ends the kernel.
struct VcLink {
    uint32_t al_base;    // shared::cta address of the S-phase layout's al[0][0][0]
    uint32_t full_bar;   // shared::cta address of full[0] (full[1] at +8)
    uint32_t empty_bar;  // shared::cta address of empty[0] (empty[1] at +8)
    int nranks;          // S-phase CTAs of the cluster
    volatile int* abort;
};

__device__ __forceinline__ uint32_t vc_cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Bytes of one chunk's alpha_hat tile (64 rows of D floats, padded rows of D + 4).
template <int D>
constexpr uint32_t vc_tile_bytes() {
    return (uint32_t)(VC_C * (D + 4) * 4);
}

// Slot pairs (W, K A_c) of an S-phase CTA in the fused kernel: two, so that a chunk's copy
// lands while the previous chunk is worked on, where shared memory has room for them (up to
// D = 96); one at D = 128.
template <int D>
constexpr int vc_nslot() {
    return D <= 96 ? 2 : 1;
}

// Phase wait with cluster-scope acquire (the data behind the barrier was written by another
// CTA of the cluster), bounded like mbar_wait.
__device__ __forceinline__ bool vc_wait_cluster(uint32_t bar, uint32_t parity,
                                                volatile int* abort) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
        if ((it & 31u) == 31u && global_timer_ns() - t0 > DRSCAN_WAIT_LIMIT_NS) {
            raise_status(DR_ERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------
// Write directions of one chunk
// ---------------------------------------------------------------------------------------
// From the chunk's K rows, W = L^-1 (U A_c) and K A_c (shared-memory tiles of row stride
// D + 4): Y = K A_c - tril(K W^T) W (s <= t) and alpha_hat_t = Y_t / |Y_t|. g is a 64 x 68
// scratch for tril(K W^T). TO_GLOBAL: rows t < nv go to dst (row per token); otherwise
// alpha_hat replaces K A_c in place, rows past the end of the sequence set to zero, and the
// block is synchronised at the end. The A-phase kernel and the S-phase CTAs of the fused
// kernel run this same code, so both forms give the same bits.
template <int D, bool TO_GLOBAL>
__device__ __forceinline__ void vc_alpha_hat(const float (*k)[D + 4], const float (*w)[D + 4],
                                             float (*ka)[D + 4], float (*g)[VC_C + 4], int nv,
                                             float* __restrict__ dst, int tid) {
    constexpr int CT = D / 16;
    const int rg = tid >> 4, cg = tid & 15;
    // tril(K W^T): rows rg + 16 i, columns cg + 16 j
    {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 2
        for (int kk = 0; kk < D; kk += 4) {
            float4 a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = *reinterpret_cast<const float4*>(&k[rg + 16 * i][kk]);
                b[i] = *reinterpret_cast<const float4*>(&w[cg + 16 * i][kk]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][j] = fmaf(a[i].x, b[j].x, acc[i][j]);
                    acc[i][j] = fmaf(a[i].y, b[j].y, acc[i][j]);
                    acc[i][j] = fmaf(a[i].z, b[j].z, acc[i][j]);
                    acc[i][j] = fmaf(a[i].w, b[j].w, acc[i][j]);
                }
        }
        __syncthreads();  // every thread is done with what g held before it is overwritten
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = rg + 16 * i, s = cg + 16 * j;
                g[r][s] = s <= r ? acc[i][j] : 0.f;
            }
    }
    __syncthreads();
    // Y = K A_c - tril(K W^T) W (rows rg + 16 i, columns cg*CT + j), normalised by rows over
    // the 16 threads of a row group
    {
        float acc[4][CT];
#pragma unroll
        for (int i = 0; i < 4; ++i) vc_ld<CT>(&ka[rg + 16 * i][cg * CT], acc[i]);
#pragma unroll 2
        for (int s = 0; s < VC_C; s += 4) {
            float4 a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(&g[rg + 16 * i][s]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float b[CT];
                vc_ld<CT>(&w[s + q][cg * CT], b);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float av = vc_comp(a[i], q);
#pragma unroll
                    for (int j = 0; j < CT; ++j) acc[i][j] = fmaf(-av, b[j], acc[i][j]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float n2 = 0.f;
#pragma unroll
            for (int j = 0; j < CT; ++j) n2 = fmaf(acc[i][j], acc[i][j], n2);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, off);
            const int r = rg + 16 * i;
            if constexpr (TO_GLOBAL) {
                if (r < nv) {
                    const float inv = rsqrtf(n2);
                    float* o = dst + (long)r * D + cg * CT;
#pragma unroll
                    for (int j = 0; j < CT; ++j) o[j] = acc[i][j] * inv;
                }
            } else {
                // each thread rewrites only the K A_c entries it read
                const float inv = r < nv ? rsqrtf(n2) : 0.f;
                float* o = &ka[r][cg * CT];
#pragma unroll
                for (int j = 0; j < CT; ++j) o[j] = acc[i][j] * inv;
            }
        }
    }
    if constexpr (!TO_GLOBAL) __syncthreads();
}

// ---------------------------------------------------------------------------------------
// A-phase
// ---------------------------------------------------------------------------------------
template <int D>
struct VcASmem {
    static constexpr int P = D + 4;  // padded row stride: rows 1 apart sit 4 banks apart
    float A[D][P];                   // A_c (symmetric)
    float u[VC_C][P];
    float k[VC_C][P];
    float ua[VC_C][P];               // U A_c, then W = L^-1 U A_c
    float ka[VC_C][P];               // K A_c
    float m[VC_C][VC_C + 4];         // I + U A_c U^T, then L's diagonal blocks, then tril(K W^T)
    float pt[16][VC_C + 4];          // the panel of L below the current diagonal block, transposed
    float dinv[VC_C];                // 1 / L_tt
};

// One head's A-phase. PUSH = false: alpha_hat to global memory (row per token); PUSH = true:
// into the S-phase CTAs of the cluster through `link`.
template <int D, bool PUSH>
__device__ __forceinline__ void vc_aphase(unsigned char* smem_raw, long bh,
                                          const float* __restrict__ k,
                                          const float* __restrict__ u,
                                          const float* __restrict__ A0, float lambda0,
                                          float* __restrict__ A_final, float* __restrict__ alpha,
                                          int T, const VcLink& link) {
    VcASmem<D>& sm = *reinterpret_cast<VcASmem<D>*>(smem_raw);
    constexpr int CT = D / 16;  // columns per thread in the 16-column-group tilings
    const int tid = threadIdx.x;
    const int rg = tid >> 4, cg = tid & 15;
    const float* kh = k + bh * (long)T * D;
    const float* uh = u + bh * (long)T * D;
    float* ah = PUSH ? nullptr : alpha + bh * (long)T * D;
    const int nchunks = (T + VC_C - 1) / VC_C;

    for (int e = tid; e < D * D; e += VC_THREADS) {
        const int r = e / D, c = e - r * D;
        sm.A[r][c] = A0 ? A0[bh * D * D + e] : (r == c ? 1.f / lambda0 : 0.f);
    }
    if (nchunks > 0) {
        vc_load_rows<D>(sm.u, uh, min(VC_C, T), tid);
        vc_load_rows<D>(sm.k, kh, min(VC_C, T), tid);
    }
    vc_wait_copies();
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * VC_C;
        const int nv = min(VC_C, T - t0);
        const int nv_next = min(VC_C, T - t0 - VC_C);

        // 1. [U A_c; K A_c]: rows rg + 16 i (i < 4 from U, i >= 4 from K), columns cg*CT + j
        {
            float acc[8][CT];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < CT; ++j) acc[i][j] = 0.f;
#pragma unroll 2
            for (int kk = 0; kk < D; kk += 4) {
                float4 a[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    a[i] = *reinterpret_cast<const float4*>(
                        i < 4 ? &sm.u[rg + 16 * i][kk] : &sm.k[rg + 16 * (i - 4)][kk]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float b[CT];
                    vc_ld<CT>(&sm.A[kk + q][cg * CT], b);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float av = vc_comp(a[i], q);
#pragma unroll
                        for (int j = 0; j < CT; ++j) acc[i][j] = fmaf(av, b[j], acc[i][j]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float* dst = i < 4 ? &sm.ua[rg + 16 * i][cg * CT] : &sm.ka[rg + 16 * (i - 4)][cg * CT];
#pragma unroll
                for (int j = 0; j < CT; ++j) dst[j] = acc[i][j];
            }
        }
        __syncthreads();

        // 2. M = I + U (U A_c)^T: rows rg + 16 i, columns cg + 16 j
        {
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 2
            for (int kk = 0; kk < D; kk += 4) {
                float4 a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    a[i] = *reinterpret_cast<const float4*>(&sm.u[rg + 16 * i][kk]);
                    b[i] = *reinterpret_cast<const float4*>(&sm.ua[cg + 16 * i][kk]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[i][j] = fmaf(a[i].x, b[j].x, acc[i][j]);
                        acc[i][j] = fmaf(a[i].y, b[j].y, acc[i][j]);
                        acc[i][j] = fmaf(a[i].z, b[j].z, acc[i][j]);
                        acc[i][j] = fmaf(a[i].w, b[j].w, acc[i][j]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = rg + 16 * i, s = cg + 16 * j;
                    sm.m[r][s] = acc[i][j] + (r == s ? 1.f : 0.f);
                }
        }
        __syncthreads();
        // U is not read again in this chunk (nor K when the S-phase CTAs form the write
        // directions): fetch the next chunk's rows under the factorisation
        if (nv_next > 0) {
            vc_load_rows<D>(sm.u, uh + (long)(t0 + VC_C) * D, nv_next, tid);
            if constexpr (PUSH) vc_load_rows<D>(sm.k, kh + (long)(t0 + VC_C) * D, nv_next, tid);
        }

        // 3. M = L L^T by 16 x 16 blocks. Per block: warp 1 first applies the previous block's
        //    contribution to this diagonal block and hands it to warp 0 on a named barrier;
        //    warp 0 factors it while warps 1-7 apply that contribution to the rest of the
        //    trailing rows of M and of U A_c; then the block rows of W = L^-1 (U A_c) (forward
        //    substitution, a thread per column) and the panel below the block (a thread per row).
        // M[i0..i0+3][s0..s0+3] -= P[i0..][.] P[s0..][.]^T, P = the panel (rows of L below the
        // previous diagonal block, held transposed in pt: four rows are one float4 per t)
        auto m_tile = [&](int i0, int s0) {
            float li[4][16], ls[4][16];
            float acc[4][4];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float4 x = *reinterpret_cast<const float4*>(&sm.pt[t][i0]);
                const float4 y = *reinterpret_cast<const float4*>(&sm.pt[t][s0]);
                li[0][t] = x.x, li[1][t] = x.y, li[2][t] = x.z, li[3][t] = x.w;
                ls[0][t] = y.x, ls[1][t] = y.y, ls[2][t] = y.z, ls[3][t] = y.w;
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) vc_ld<4>(&sm.m[i0 + a][s0], acc[a]);
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int t = 0; t < 16; ++t) acc[a][bb] = fmaf(-li[a][t], ls[bb][t], acc[a][bb]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
                *reinterpret_cast<float4*>(&sm.m[i0 + a][s0]) =
                    make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        };
#pragma unroll 1
        for (int jb = 0; jb < 4; ++jb) {
            const int b0 = 16 * jb;
            if (tid < 32) {
                // diagonal block in one warp: lane l (l < 16) holds row b0 + l in registers
                const int l = tid & 15;
                // warp 1 has applied the previous block's contribution to this block
                if (jb > 0) asm volatile("bar.sync 1, 64;" ::: "memory");
                float r[16];
                vc_ld<16>(&sm.m[b0 + l][b0], r);
                float my_inv = 0.f;
                bool bad = false;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float piv = __shfl_sync(0xffffffffu, r[j], j);
                    bad |= !(piv > 0.f);
                    const float inv = rsqrtf(piv);
                    if (l == j) {
                        r[j] = piv * inv;
                        my_inv = inv;
                    } else if (l > j) {
                        r[j] *= inv;
                    }
                    const float lj = r[j];
#pragma unroll
                    for (int mm = 1; mm < 16; ++mm) {
                        if (mm > j) {
                            const float lm = __shfl_sync(0xffffffffu, lj, mm);
                            if (l >= mm) r[mm] = fmaf(-lj, lm, r[mm]);
                        }
                    }
                }
                if (tid < 16) {
#pragma unroll
                    for (int mm = 0; mm < 16; ++mm)
                        if (mm <= l) sm.m[b0 + l][b0 + mm] = r[mm];
                    sm.dinv[b0 + l] = my_inv;
                    if (bad && l == 0) raise_status(DR_ERR_NOT_SPD);
                }
            } else if (jb > 0) {
                const int p0 = b0 - 16;  // the block whose contribution is applied
                if (tid < 64) {
                    // warp 1: the ten lower 4 x 4 tiles of this diagonal block first (tile q
                    // is row group ti, column group ts <= ti), then release warp 0
                    const int q = tid - 32;
                    if (q < 10) {
                        const int ti = q < 1 ? 0 : q < 3 ? 1 : q < 6 ? 2 : 3;
                        const int ts = q - ti * (ti + 1) / 2;
                        m_tile(b0 + 4 * ti, b0 + 4 * ts);
                    }
                    __syncwarp();
                    __threadfence_block();
                    asm volatile("bar.arrive 1, 64;" ::: "memory");
                }
                const int n4 = (VC_C - 16 - p0) / 4;  // trailing rows, in groups of four
                const int nm = n4 * n4;               // 4 x 4 tiles of the trailing block of M
                const int nu = n4 * (D / 4);          // 4 x 4 tiles of the trailing rows of U A_c
                for (int e = tid - 32; e < nm + nu; e += VC_THREADS - 32) {
                    if (e < nm) {
                        const int ti = e / n4, ts = e - ti * n4;
                        const int i0 = p0 + 16 + 4 * ti, s0 = p0 + 16 + 4 * ts;
                        if (s0 > i0 + 3) continue;  // strictly above the diagonal: unused
                        if (ti < 4 && ts < 4) continue;  // the diagonal block: done above
                        m_tile(i0, s0);
                    } else {
                        float li[4][16];
                        float acc[4][4];
                        const int f = e - nm;
                        const int ti = f / (D / 4), tc = f - ti * (D / 4);
                        const int i0 = p0 + 16 + 4 * ti, c0 = 4 * tc;
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const float4 x = *reinterpret_cast<const float4*>(&sm.pt[t][i0]);
                            li[0][t] = x.x, li[1][t] = x.y, li[2][t] = x.z, li[3][t] = x.w;
                        }
#pragma unroll
                        for (int a = 0; a < 4; ++a) vc_ld<4>(&sm.ua[i0 + a][c0], acc[a]);
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            float w4[4];
                            vc_ld<4>(&sm.ua[p0 + t][c0], w4);
#pragma unroll
                            for (int a = 0; a < 4; ++a)
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    acc[a][j] = fmaf(-li[a][t], w4[j], acc[a][j]);
                        }
#pragma unroll
                        for (int a = 0; a < 4; ++a)
                            *reinterpret_cast<float4*>(&sm.ua[i0 + a][c0]) =
                                make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
                    }
                }
            }
            __syncthreads();
            if (tid < D) {
                // W rows b0..b0+15, column tid: L_bb x = (U A_c)_b
                float x[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) x[t] = sm.ua[b0 + t][tid];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    x[t] *= sm.dinv[b0 + t];
#pragma unroll
                    for (int mm = t + 1; mm < 16; ++mm)
                        x[mm] = fmaf(-sm.m[b0 + mm][b0 + t], x[t], x[mm]);
                }
#pragma unroll
                for (int t = 0; t < 16; ++t) sm.ua[b0 + t][tid] = x[t];
            } else if (tid - D < VC_C - 16 - b0) {
                // panel row i below the block: x L_bb^T = M_i,b
                const int i = b0 + 16 + (tid - D);
                float x[16];
                vc_ld<16>(&sm.m[i][b0], x);
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    x[t] *= sm.dinv[b0 + t];
#pragma unroll
                    for (int s = t + 1; s < 16; ++s) x[s] = fmaf(-x[t], sm.m[b0 + s][b0 + t], x[s]);
                }
                // into the transposed panel, which only the next block's updates read
#pragma unroll
                for (int t = 0; t < 16; ++t) sm.pt[t][i] = x[t];
            }
            __syncthreads();
        }

        if constexpr (PUSH) {
            // W (in place of U A_c) and K A_c, adjacent tiles, go to every S-phase CTA, which
            // forms the chunk's write directions itself: the next chunk's A-phase needs only
            // W. The CTAs release the slot pair once they are done with the chunk.
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                // pair sp last held chunk c - NSL: its release is phase c / NSL - 1 of `empty`
                constexpr int NSL = vc_nslot<D>();
                const int sp = c % NSL;
                if (c >= NSL)
                    vc_wait_cluster(link.empty_bar + 8u * sp, (uint32_t)((c / NSL - 1) & 1),
                                    link.abort);
                if (!*link.abort) {
                    for (int qr = 1; qr <= link.nranks; ++qr)
                        bulk_copy_to_peer(
                            cluster_map(link.al_base + sp * 2 * vc_tile_bytes<D>(), (uint32_t)qr),
                            smem_u32(&sm.ua[0][0]), 2 * vc_tile_bytes<D>(),
                            cluster_map(link.full_bar + 8u * sp, (uint32_t)qr));
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            }
        } else {
            // 4-5. the chunk's write directions, written out row per token (L's storage
            //      takes tril(K W^T))
            vc_alpha_hat<D, true>(sm.k, sm.ua, sm.ka, sm.m, nv, ah + (long)t0 * D, tid);
            if (nv_next > 0) vc_load_rows<D>(sm.k, kh + (long)(t0 + VC_C) * D, nv_next, tid);
        }

        // 6. A_{c+1} = A_c - W^T W: rows rg*CT + i, columns cg*CT + j
        {
            float acc[CT][CT];
#pragma unroll
            for (int i = 0; i < CT; ++i)
#pragma unroll
                for (int j = 0; j < CT; ++j) acc[i][j] = 0.f;
#pragma unroll 4
            for (int s = 0; s < VC_C; ++s) {
                float a[CT], b[CT];
                vc_ld<CT>(&sm.ua[s][rg * CT], a);
                vc_ld<CT>(&sm.ua[s][cg * CT], b);
#pragma unroll
                for (int i = 0; i < CT; ++i)
#pragma unroll
                    for (int j = 0; j < CT; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
#pragma unroll
            for (int i = 0; i < CT; ++i) {
                float* dst = &sm.A[rg * CT + i][cg * CT];
#pragma unroll
                for (int j = 0; j < CT; ++j) dst[j] -= acc[i][j];
            }
        }
        if constexpr (PUSH) {
            // the next chunk's first step rewrites the tile: its copies must have read it
            if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
        vc_wait_copies();
        __syncthreads();
    }
    if constexpr (PUSH) {
        if (tid == 0) bulk_wait_all();  // every copy has landed before the kernel can end
    }

    if (A_final) {
        for (int e = tid; e < D * D; e += VC_THREADS) {
            const int r = e / D, c = e - r * D;
            A_final[bh * D * D + e] = sm.A[r][c];
        }
    }
}

// grid: B*H; block: VC_THREADS; dynamic shared memory: sizeof(VcASmem<D>).
template <int D>
__global__ void __launch_bounds__(VC_THREADS, 1)
    vla_aphase_kernel(const float* __restrict__ k, const float* __restrict__ u,
                      const float* __restrict__ A0, float lambda0, float* __restrict__ A_final,
                      float* __restrict__ alpha, int T) {
    extern __shared__ __align__(16) unsigned char vc_smem_raw[];
    vc_aphase<D, false>(vc_smem_raw, blockIdx.x, k, u, A0, lambda0, A_final, alpha, T, VcLink{});
}

// ---------------------------------------------------------------------------------------
// S-phase
// ---------------------------------------------------------------------------------------
template <int D>
struct VcSSmem {
    static constexpr int P = D + 4;
    static constexpr int PR = VC_RS + 4;
    float k[VC_C][P];
    float q[VC_C][P];
    // alpha_hat rows, double buffered; fused: slot pair s holds W in al[2s] and K A_c, then
    // alpha_hat in its place, in al[2s + 1]
    float al[2 * vc_nslot<D>()][VC_C][P];
    float S[VC_RS + 1][P];       // this CTA's rows of S (+ n for the ratio readout)
    float g[VC_C][VC_C + 4];     // strictly lower part of K Alpha^T
    float p[VC_C][VC_C + 4];     // lower part (diagonal included) of Q Alpha^T
    float v[VC_C][PR];           // this CTA's value columns
    float r[VC_C][PR + 4];       // V - K S^T, then R (column VC_RS: the n row's residual)
    float o[VC_C][PR];           // Q S^T
    float on[VC_C];              // ratio readout: q_t . n_c
};

// One head's S-phase for rows row0 .. row0 + 31 of S. PULL = false: alpha_hat from global
// memory; PULL = true: W and K A_c of each chunk arrive from the cluster's A-phase CTA
// (`link`) into al[0] and al[1], and this CTA forms alpha_hat in al[1].
template <int D, bool RATIO, bool PULL>
__device__ __forceinline__ void vc_sphase(unsigned char* smem_raw, long bh, int row0,
                                          const float* __restrict__ q,
                                          const float* __restrict__ k,
                                          const float* __restrict__ v,
                                          const float* __restrict__ alpha,
                                          const float* __restrict__ S0,
                                          const float* __restrict__ n0, float* __restrict__ out,
                                          float* __restrict__ S_final,
                                          float* __restrict__ n_final, int T,
                                          const VcLink& link) {
    VcSSmem<D>& sm = *reinterpret_cast<VcSSmem<D>*>(smem_raw);
    constexpr int CT = D / 16;
    constexpr int NRC = VC_RS + (RATIO ? 1 : 0);  // columns of R (value rows + n)
    const int tid = threadIdx.x;
    const int rg = tid >> 4, cg = tid & 15;
    const long seq = bh * (long)T * D;
    const int nchunks = (T + VC_C - 1) / VC_C;

    for (int e = tid; e < VC_RS * D; e += VC_THREADS) {
        const int r = e / D, c = e - r * D;
        sm.S[r][c] = S0 ? S0[bh * D * D + (long)(row0 + r) * D + c] : 0.f;
    }
    if constexpr (RATIO) {
        for (int c = tid; c < D; c += VC_THREADS) sm.S[VC_RS][c] = n0 ? n0[bh * D + c] : 0.f;
    }
    if (nchunks > 0) {
        const int nv = min(VC_C, T);
        vc_load_rows<D>(sm.k, k + seq, nv, tid);
        vc_load_rows<D>(sm.q, q + seq, nv, tid);
        if constexpr (!PULL) vc_load_rows<D>(sm.al[0], alpha + seq, nv, tid);
        vc_load_cols<D, VC_RS>(sm.v, v + seq, row0, nv, tid);
    }
    vc_wait_copies();
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * VC_C;
        const int nv = min(VC_C, T - t0);
        const int nv_next = min(VC_C, T - t0 - VC_C);
        const int b = c & 1;
        constexpr int NSL = vc_nslot<D>();
        const int sp = c % NSL;  // fused: this chunk's slot pair
        if constexpr (PULL) {
            // this chunk's W and K A_c: the k-th fill of pair sp completes its phase k
            vc_wait_cluster(link.full_bar + 8u * sp, (uint32_t)((c / NSL) & 1), link.abort);
            vc_alpha_hat<D, false>(sm.k, sm.al[2 * sp], sm.al[2 * sp + 1], sm.p, nv, nullptr, tid);
        } else {
            if (nv_next > 0)
                vc_load_rows<D>(sm.al[b ^ 1], alpha + seq + (long)(t0 + VC_C) * D, nv_next, tid);
        }
        float (*alh)[VcSSmem<D>::P] = sm.al[PULL ? 2 * sp + 1 : b];  // this chunk's alpha_hat

        // 1. [G; P] = [K; Q] Alpha^T: rows rg + 16 i (i < 4 from K, i >= 4 from Q),
        //    columns cg + 16 j
        {
            float acc[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 2
            for (int kk = 0; kk < D; kk += 4) {
                float4 a[8], bb[4];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    a[i] = *reinterpret_cast<const float4*>(
                        i < 4 ? &sm.k[rg + 16 * i][kk] : &sm.q[rg + 16 * (i - 4)][kk]);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    bb[j] = *reinterpret_cast<const float4*>(&alh[cg + 16 * j][kk]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[i][j] = fmaf(a[i].x, bb[j].x, acc[i][j]);
                        acc[i][j] = fmaf(a[i].y, bb[j].y, acc[i][j]);
                        acc[i][j] = fmaf(a[i].z, bb[j].z, acc[i][j]);
                        acc[i][j] = fmaf(a[i].w, bb[j].w, acc[i][j]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = rg + 16 * i, s = cg + 16 * j;
                    sm.g[t][s] = s < t ? acc[i][j] : 0.f;
                    sm.p[t][s] = s <= t ? acc[i + 4][j] : 0.f;
                }
        }

        // 2. V - K S^T and Q S^T: rows rg + 16 i, columns cg*2 + j of this CTA's rows of S
        {
            float acc[8][2];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = 0.f;
#pragma unroll 2
            for (int kk = 0; kk < D; kk += 4) {
                float4 a[8], bb[2];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    a[i] = *reinterpret_cast<const float4*>(
                        i < 4 ? &sm.k[rg + 16 * i][kk] : &sm.q[rg + 16 * (i - 4)][kk]);
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    bb[j] = *reinterpret_cast<const float4*>(&sm.S[cg * 2 + j][kk]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        acc[i][j] = fmaf(a[i].x, bb[j].x, acc[i][j]);
                        acc[i][j] = fmaf(a[i].y, bb[j].y, acc[i][j]);
                        acc[i][j] = fmaf(a[i].z, bb[j].z, acc[i][j]);
                        acc[i][j] = fmaf(a[i].w, bb[j].w, acc[i][j]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = rg + 16 * i;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    sm.r[t][cg * 2 + j] = sm.v[t][cg * 2 + j] - acc[i][j];
                    sm.o[t][cg * 2 + j] = acc[i + 4][j];
                }
            }
            if constexpr (RATIO) {
                // the n row: 1 - k_t . n and q_t . n, one dot product per thread
                if (tid < 2 * VC_C) {
                    const int t = tid & (VC_C - 1);
                    const float* x = tid < VC_C ? sm.k[t] : sm.q[t];
                    float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                    for (int kk = 0; kk < D; kk += 4) {
                        const float4 a = *reinterpret_cast<const float4*>(x + kk);
                        const float4 n4 = *reinterpret_cast<const float4*>(&sm.S[VC_RS][kk]);
                        d4[0] = fmaf(a.x, n4.x, d4[0]);
                        d4[1] = fmaf(a.y, n4.y, d4[1]);
                        d4[2] = fmaf(a.z, n4.z, d4[2]);
                        d4[3] = fmaf(a.w, n4.w, d4[3]);
                    }
                    const float dn = (d4[0] + d4[1]) + (d4[2] + d4[3]);
                    if (tid < VC_C)
                        sm.r[t][VC_RS] = t < nv ? 1.f - dn : 0.f;
                    else
                        sm.on[t] = dn;
                }
            }
        }
        __syncthreads();
        // K, Q and V are not read again in this chunk: fetch the next chunk's rows
        if (nv_next > 0) {
            const long nx = seq + (long)(t0 + VC_C) * D;
            vc_load_rows<D>(sm.k, k + nx, nv_next, tid);
            vc_load_rows<D>(sm.q, q + nx, nv_next, tid);
            vc_load_cols<D, VC_RS>(sm.v, v + nx, row0, nv_next, tid);
        }

        // 3. (I + G) R = V - K S^T by 16-row blocks: a column per thread within the block,
        //    then the rows below take the block's contribution
#pragma unroll 1
        for (int jb = 0; jb < 4; ++jb) {
            const int b0 = 16 * jb;
            if (tid < NRC) {
                float x[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) x[t] = sm.r[b0 + t][tid];
#pragma unroll
                for (int t = 0; t < 16; ++t)
#pragma unroll
                    for (int mm = t + 1; mm < 16; ++mm)
                        x[mm] = fmaf(-sm.g[b0 + mm][b0 + t], x[t], x[mm]);
#pragma unroll
                for (int t = 0; t < 16; ++t) sm.r[b0 + t][tid] = x[t];
            }
            __syncthreads();
            if (jb < 3) {
                const int nrow = VC_C - 16 - b0;
                // rows below x (pairs of columns; the n column rides with the last pair)
                for (int e = tid; e < nrow * (VC_RS / 2); e += VC_THREADS) {
                    const int i = b0 + 16 + e / (VC_RS / 2), c2 = 2 * (e % (VC_RS / 2));
                    float gi[16];
                    vc_ld<16>(&sm.g[i][b0], gi);
                    float a0 = sm.r[i][c2], a1 = sm.r[i][c2 + 1];
                    float a2 = 0.f;
                    const bool extra = RATIO && c2 == VC_RS - 2;
                    if (extra) a2 = sm.r[i][VC_RS];
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const float2 x2 = *reinterpret_cast<const float2*>(&sm.r[b0 + t][c2]);
                        a0 = fmaf(-gi[t], x2.x, a0);
                        a1 = fmaf(-gi[t], x2.y, a1);
                        if (extra) a2 = fmaf(-gi[t], sm.r[b0 + t][VC_RS], a2);
                    }
                    sm.r[i][c2] = a0;
                    sm.r[i][c2 + 1] = a1;
                    if (extra) sm.r[i][VC_RS] = a2;
                }
                __syncthreads();
            }
        }

        // 4. O = Q S^T + tril(Q Alpha^T) R: rows rg + 16 i, columns cg*2 + j; the ratio
        //    readout divides by n_t q_t = q_t . n_c + tril(Q Alpha^T) r_n
        {
            float acc[4][2], dn[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[i][0] = sm.o[rg + 16 * i][cg * 2];
                acc[i][1] = sm.o[rg + 16 * i][cg * 2 + 1];
                dn[i] = RATIO ? sm.on[rg + 16 * i] : 0.f;
            }
#pragma unroll 2
            for (int s = 0; s < VC_C; s += 4) {
                float4 a[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    a[i] = *reinterpret_cast<const float4*>(&sm.p[rg + 16 * i][s]);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const float2 x2 = *reinterpret_cast<const float2*>(&sm.r[s + qq][cg * 2]);
                    const float xn = RATIO ? sm.r[s + qq][VC_RS] : 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float av = vc_comp(a[i], qq);
                        acc[i][0] = fmaf(av, x2.x, acc[i][0]);
                        acc[i][1] = fmaf(av, x2.y, acc[i][1]);
                        if constexpr (RATIO) dn[i] = fmaf(av, xn, dn[i]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = rg + 16 * i;
                if (t < nv) {
                    float2 o2 = make_float2(acc[i][0], acc[i][1]);
                    if constexpr (RATIO) {
                        o2.x /= dn[i];
                        o2.y /= dn[i];
                    }
                    *reinterpret_cast<float2*>(out + seq + (long)(t0 + t) * D + row0 + cg * 2) = o2;
                }
            }
        }

        // 5. S += R^T Alpha: rows rg*2 + i, columns cg*CT + j (and n += r_n^T Alpha)
        {
            float acc[2][CT];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < CT; ++j) acc[i][j] = 0.f;
            float accn = 0.f;
#pragma unroll 4
            for (int s = 0; s < VC_C; ++s) {
                const float2 x2 = *reinterpret_cast<const float2*>(&sm.r[s][rg * 2]);
                float bb[CT];
                vc_ld<CT>(&alh[s][cg * CT], bb);
#pragma unroll
                for (int j = 0; j < CT; ++j) {
                    acc[0][j] = fmaf(x2.x, bb[j], acc[0][j]);
                    acc[1][j] = fmaf(x2.y, bb[j], acc[1][j]);
                }
                if constexpr (RATIO) {
                    if (tid < D) accn = fmaf(sm.r[s][VC_RS], alh[s][tid], accn);
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float* dst = &sm.S[rg * 2 + i][cg * CT];
#pragma unroll
                for (int j = 0; j < CT; ++j) dst[j] += acc[i][j];
            }
            if constexpr (RATIO) {
                if (tid < D) sm.S[VC_RS][tid] += accn;
            }
        }
        vc_wait_copies();
        __syncthreads();
        if constexpr (PULL) {
            // pair sp is read (alpha_hat by steps 1 and 5): arm it for chunk c + NSL, then hand
            // it back to the A-phase CTA
            if (tid == 0 && !*link.abort) {
                if (c + NSL < nchunks)
                    mbar_arrive_expect_tx(link.full_bar + 8u * sp, 2 * vc_tile_bytes<D>());
                mbar_arrive_remote(cluster_map(link.empty_bar + 8u * sp, 0));
            }
        }
    }

    if (S_final) {
        for (int e = tid; e < VC_RS * D; e += VC_THREADS) {
            const int r = e / D, c = e - r * D;
            S_final[bh * D * D + (long)(row0 + r) * D + c] = sm.S[r][c];
        }
    }
    if constexpr (RATIO) {
        if (n_final && row0 == 0)
            for (int c = tid; c < D; c += VC_THREADS) n_final[bh * D + c] = sm.S[VC_RS][c];
    }
}

// grid: (B*H, D / VC_RS); block: VC_THREADS; dynamic shared memory: sizeof(VcSSmem<D>).
template <int D, bool RATIO>
__global__ void __launch_bounds__(VC_THREADS, 1)
    vla_sphase_kernel(const float* __restrict__ q, const float* __restrict__ k,
                      const float* __restrict__ v, const float* __restrict__ alpha,
                      const float* __restrict__ S0, const float* __restrict__ n0,
                      float* __restrict__ out, float* __restrict__ S_final,
                      float* __restrict__ n_final, int T) {
    extern __shared__ __align__(16) unsigned char vc_smem_raw[];
    vc_sphase<D, RATIO, false>(vc_smem_raw, blockIdx.x, (int)blockIdx.y * VC_RS, q, k, v, alpha,
                               S0, n0, out, S_final, n_final, T, VcLink{});
}

// ---------------------------------------------------------------------------------------
// Fused: both phases in one cluster per head
// ---------------------------------------------------------------------------------------
// Cluster of 1 + D/32 CTAs per (b,h): rank 0 runs the A-phase and hands every chunk's W and
// K A_c to ranks 1 .. D/32 (the S-phase for 32 rows of S each, which first form the chunk's
// alpha_hat rows) through their shared memory, so that both phases run at once on different
// SMs, the A-phase's serial chain holds only what the next chunk needs, and no scratch
// memory is needed.
template <int D>
constexpr int vc_fused_bar_offset() {
    constexpr int a = (int)sizeof(VcASmem<D>), b = (int)sizeof(VcSSmem<D>);
    return ((a > b ? a : b) + 15) / 16 * 16;
}

template <int D>
constexpr int vc_fused_smem_bytes() {
    return vc_fused_bar_offset<D>() + 48;  // full[2] (at +0), empty[2] (at +16), abort (at +32)
}
static_assert(vc_fused_smem_bytes<32>() <= 232448 && vc_fused_smem_bytes<64>() <= 232448 &&
                  vc_fused_smem_bytes<96>() <= 232448 && vc_fused_smem_bytes<128>() <= 232448,
              "shared memory per CTA");

// grid: B*H*(1 + D/32) with clusters of (1 + D/32, 1, 1); block: VC_THREADS; dynamic shared
// memory: vc_fused_smem_bytes<D>().
template <int D, bool RATIO>
__global__ void __launch_bounds__(VC_THREADS, 1)
    vla_fused_kernel(const float* __restrict__ q, const float* __restrict__ k,
                     const float* __restrict__ v, const float* __restrict__ u,
                     const float* __restrict__ S0, const float* __restrict__ A0,
                     const float* __restrict__ n0, float lambda0, float* __restrict__ out,
                     float* __restrict__ S_final, float* __restrict__ A_final,
                     float* __restrict__ n_final, int T) {
    extern __shared__ __align__(16) unsigned char vc_smem_raw[];
    constexpr int NS = D / VC_RS;  // S-phase CTAs per head
    uint8_t* bars = vc_smem_raw + vc_fused_bar_offset<D>();
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 32);
    const uint32_t rank = vc_cluster_rank();
    const long bh = blockIdx.x / (NS + 1);
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(bars), 1);        // full[0]: armed by this CTA, bytes from rank 0
        mbar_init(smem_u32(bars + 8), 1);    // full[1]
        mbar_init(smem_u32(bars + 16), NS);  // empty[0]: one arrival per S-phase CTA
        mbar_init(smem_u32(bars + 24), NS);  // empty[1]
        *abort_flag = 0;
        if (rank != 0) {
            // the slot pairs of the first chunks, armed before any copy can be issued
            const int nchunks = (T + VC_C - 1) / VC_C;
            for (int c = 0; c < vc_nslot<D>() && c < nchunks; ++c)
                mbar_arrive_expect_tx(smem_u32(bars + 8 * c), 2 * vc_tile_bytes<D>());
        }
        mbar_init_fence();
    }
    __syncthreads();
    cluster_sync_all();  // every barrier of the cluster is initialised before any remote arrival

    VcLink link;
    link.al_base = smem_u32(&reinterpret_cast<VcSSmem<D>*>(vc_smem_raw)->al[0][0][0]);
    link.full_bar = smem_u32(bars);
    link.empty_bar = smem_u32(bars + 16);
    link.nranks = NS;
    link.abort = abort_flag;
    if (rank == 0)
        vc_aphase<D, true>(vc_smem_raw, bh, k, u, A0, lambda0, A_final, nullptr, T, link);
    else
        vc_sphase<D, RATIO, true>(vc_smem_raw, bh, (int)(rank - 1) * VC_RS, q, k, v, nullptr, S0,
                                  n0, out, S_final, n_final, T, link);
    // no CTA may leave while another can still write into its shared memory or arrive on it
    cluster_sync_all();
}

}  // namespace drscan
