// Log-linear attention over a Fenwick hierarchy of linear-attention memories ("Adaptive memory
// decay for log-linear attention", problem definition and method sections), chunked.
//
// At step t the prefix [0, t] splits into the token itself (level 0) and one block of 2^b
// earlier tokens per set bit b of t (level b + 1); the output is the lambda_t-weighted sum
// of the levels' readouts. With chunks of C = 64 tokens aligned to multiples of 64:
//   * a pair (t, s <= t) inside one chunk has level bitlen(t ^ s) <= 6, so the in-chunk part
//     is (Q K^T (.) W) V with W[t, s] = lambda_t^(bitlen(t ^ s)) for s <= t;
//   * a token s of an earlier chunk c' < c has level 7 + floor(log2(c ^ c')): the earlier
//     chunks split into one block of 2^b chunks per set bit b of c, and
//     O[t] += sum_{b : bit b of c} lambda_t^(7+b) (M_b q_t),   M_b = sum_{s in block b} v_s k_s^T.
// The block states M_b are a binary counter over chunks: after chunk c, with j = the number of
// trailing ones of c, M_j = V_c^T K_c + sum_{b<j} M_b and M_b = 0 for b < j.
//
// One CTA per (b, h, slice of BV value channels) walks the chunks in order. Eight warps: four
// own 16 query rows each for the in-chunk part and then 32 key channels each for the chunk
// state and the merge, four the same rows for the block-state readouts; every contraction is a bf16
// m16n8k16 warp MMA with fp32 accumulation (the tiles are 16-64 rows, the level bookkeeping
// sits between them). The block states stay in shared memory in fp32
// (dk x BV per level, for up to LL_LEVELS chunk levels: T <= 64 * 2^LL_LEVELS). The next
// chunk's tiles are loaded into registers while the current chunk computes (the level
// states leave no room for a second shared-memory stage) and stored once it is done.
#pragma once

#include "common.cuh"

namespace drscan {

constexpr int LL_C = 64;         // chunk length
constexpr int LL_DK = 128;       // key dimension
constexpr int LL_BV = 32;        // value channels per CTA
constexpr int LL_LEVELS = 9;     // chunk levels kept (T <= 32768)
constexpr int LL_LMAX = 16;      // lambda levels per token read (7 in-chunk + LL_LEVELS)
constexpr int LL_THREADS = 256;
constexpr int LL_QS = LL_DK + 8;   // bf16 row stride of the Q and K tiles (conflict-free ldmatrix)
constexpr int LL_VS = LL_BV + 8;   // bf16 row stride of the V tile
constexpr int LL_MS = LL_DK + 8;   // fp32 row stride of a block state (rows = value channels)

struct LoglinearSmem {
    __nv_bfloat16 q[LL_C][LL_QS];
    __nv_bfloat16 k[LL_C][LL_QS];
    __nv_bfloat16 v[LL_C][LL_VS];
    float lam[LL_C][LL_LMAX];
    float m[LL_LEVELS][LL_BV][LL_MS];  // block states M_b: value channel rows, key columns
    float o[LL_C][LL_BV + 2];          // the block-state part of the chunk's outputs
};

__device__ __forceinline__ void ll_mma(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ll_ldsm_x4(uint32_t* r, const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ll_ldsm_x4_t(uint32_t* r, const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ int ll_bitlen(int x) { return 32 - __clz(x); }

// Read-only global loads issued exactly where they stand (volatile asm keeps their place among
// the kernel's barriers), so that the next chunk's prefetch overlaps the current chunk's work.
__device__ __forceinline__ uint4 ll_ld_pinned_u4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float ll_ld_pinned_f(const float* p) {
    float r;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r) : "l"(p));
    return r;
}

// One chunk's tiles in registers, spread over the CTA's threads (rows past T as zeros, their
// lambdas as zero): loaded from HBM early, stored to shared memory when the tiles are free.
struct LoglinearStage {
    static constexpr int NQK = LL_C * (LL_DK / 8) / LL_THREADS;  // 16-byte pieces per thread
    static constexpr int NV = LL_C * (LL_BV / 8) / LL_THREADS;
    static constexpr int NL = LL_C * LL_LMAX / LL_THREADS;
    uint4 qv[NQK], kv[NQK], vv[NV];
    float lv[NL];

    __device__ __forceinline__ void load(const __nv_bfloat16* __restrict__ q,
                                         const __nv_bfloat16* __restrict__ k,
                                         const __nv_bfloat16* __restrict__ v,
                                         const float* __restrict__ lam, long bh, int T, int dv,
                                         int v0, int L, int t0, int tid) {
#pragma unroll
        for (int i = 0; i < NQK; ++i) {
            const int e = tid + i * LL_THREADS;
            const int r = e / (LL_DK / 8), c8 = (e % (LL_DK / 8)) * 8;
            qv[i] = kv[i] = make_uint4(0, 0, 0, 0);
            if (t0 + r < T) {
                qv[i] = ll_ld_pinned_u4(q + (bh * T + t0 + r) * (long)LL_DK + c8);
                kv[i] = ll_ld_pinned_u4(k + (bh * T + t0 + r) * (long)LL_DK + c8);
            }
        }
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int e = tid + i * LL_THREADS;
            const int r = e / (LL_BV / 8), c8 = (e % (LL_BV / 8)) * 8;
            vv[i] = make_uint4(0, 0, 0, 0);
            if (t0 + r < T) vv[i] = ll_ld_pinned_u4(v + (bh * T + t0 + r) * (long)dv + v0 + c8);
        }
#pragma unroll
        for (int i = 0; i < NL; ++i) {
            const int e = tid + i * LL_THREADS;
            const int r = e / LL_LMAX, l = e % LL_LMAX;
            lv[i] = (t0 + r < T && l < L) ? ll_ld_pinned_f(lam + (bh * T + t0 + r) * (long)L + l) : 0.f;
        }
    }

    __device__ __forceinline__ void store(LoglinearSmem& sm) const;
};

__device__ __forceinline__ void LoglinearStage::store(LoglinearSmem& sm) const {
    const int tid = threadIdx.x;
#pragma unroll
    for (int i = 0; i < NQK; ++i) {
        const int e = tid + i * LL_THREADS;
        const int r = e / (LL_DK / 8), c8 = (e % (LL_DK / 8)) * 8;
        *reinterpret_cast<uint4*>(&sm.q[r][c8]) = qv[i];
        *reinterpret_cast<uint4*>(&sm.k[r][c8]) = kv[i];
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = tid + i * LL_THREADS;
        const int r = e / (LL_BV / 8), c8 = (e % (LL_BV / 8)) * 8;
        *reinterpret_cast<uint4*>(&sm.v[r][c8]) = vv[i];
    }
#pragma unroll
    for (int i = 0; i < NL; ++i) {
        const int e = tid + i * LL_THREADS;
        sm.lam[e / LL_LMAX][e % LL_LMAX] = lv[i];
    }
}

// grid: (B*H, dv / LL_BV); block: LL_THREADS; dynamic shared memory: sizeof(LoglinearSmem).
// Warps 0-3 take the in-chunk part of the outputs (query rows 16w .. 16w+15) and the chunk
// state (key channels 32w .. +31), which they merge into the block states once the readouts
// are done; warps 4-7 the readouts of the block states for the same rows. The two halves of
// the outputs meet in shared memory before the store.
__global__ void __launch_bounds__(LL_THREADS) loglinear_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ lam,
    __nv_bfloat16* __restrict__ out, int T, int dv, int L) {
    extern __shared__ __align__(16) unsigned char ll_smem_raw[];
    LoglinearSmem& sm = *reinterpret_cast<LoglinearSmem*>(ll_smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tg = lane & 3;
    const bool intra = warp < 4;
    const int wq = warp & 3;  // row block (both halves) / key-channel block (state)
    const long bh = blockIdx.x;
    const int v0 = blockIdx.y * LL_BV;
    const int nchunks = (T + LL_C - 1) / LL_C;
    const int r0 = 16 * wq;
    const int ta = r0 + g, tb = r0 + g + 8;  // this thread's two rows (in-chunk positions)

    for (int e = tid; e < LL_LEVELS * LL_BV * LL_MS; e += LL_THREADS) (&sm.m[0][0][0])[e] = 0.f;
    LoglinearStage stage;
    if (nchunks > 0) stage.load(q, k, v, lam, bh, T, dv, v0, L, 0, tid);

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * LL_C;
        __syncthreads();  // the previous chunk is done with every tile
        stage.store(sm);
        __syncthreads();
        if (c + 1 < nchunks) stage.load(q, k, v, lam, bh, T, dv, v0, L, t0 + LL_C, tid);

        float o[LL_BV / 8][4];
#pragma unroll
        for (int n = 0; n < LL_BV / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        float s[2][LL_BV / 8][4];  // this chunk's state V^T K (in-chunk warps)
        if (intra) {
            // P = Q K^T over the chunk's 64 keys, weighted by lambda of the pair's level
            float p[LL_C / 8][4];
#pragma unroll
            for (int n = 0; n < LL_C / 8; ++n) p[n][0] = p[n][1] = p[n][2] = p[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < LL_DK / 16; ++kk) {
                uint32_t a[4];
                ll_ldsm_x4(a, &sm.q[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
#pragma unroll
                for (int n2 = 0; n2 < LL_C / 16; ++n2) {
                    // keys 16*n2 .. +15 as two n8 tiles: rows = keys, columns = channels
                    uint32_t b[4];
                    ll_ldsm_x4(b, &sm.k[n2 * 16 + (lane & 7) + ((lane >> 4) << 3)]
                                       [kk * 16 + ((lane >> 3) & 1) * 8]);
                    const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
                    ll_mma(p[2 * n2], a, b0);
                    ll_mma(p[2 * n2 + 1], a, b1);
                }
            }
#pragma unroll
            for (int n = 0; n < LL_C / 8; ++n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = (e < 2) ? ta : tb;
                    const int s = 8 * n + 2 * tg + (e & 1);
                    p[n][e] = (s <= t) ? p[n][e] * sm.lam[t][ll_bitlen(t ^ s)] : 0.f;
                }
            }
            // O = P V (P from the accumulators as bf16 A fragments)
#pragma unroll
            for (int kk = 0; kk < LL_C / 16; ++kk) {
                uint32_t a[4];
                a[0] = pack_bf16(p[2 * kk][0], p[2 * kk][1]);
                a[1] = pack_bf16(p[2 * kk][2], p[2 * kk][3]);
                a[2] = pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
                a[3] = pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
                for (int n2 = 0; n2 < LL_BV / 16; ++n2) {
                    uint32_t b[4];
                    ll_ldsm_x4_t(b, &sm.v[kk * 16 + (lane & 15)][n2 * 16 + (lane >> 4) * 8]);
                    const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
                    ll_mma(o[2 * n2], a, b0);
                    ll_mma(o[2 * n2 + 1], a, b1);
                }
            }
            // this chunk's state V^T K, transposed (rows = key channels 32*wq .. +31), here so
            // that it overlaps the other warps' block-state readouts
            if (c + 1 < nchunks) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int n = 0; n < LL_BV / 8; ++n)
                        s[mt][n][0] = s[mt][n][1] = s[mt][n][2] = s[mt][n][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < LL_C / 16; ++kk) {  // over the chunk's tokens
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        // A (m = key channel, k = token) = K^T: transposed 8x8 loads of the K tile
                        uint32_t a[4];
                        const int kc0 = 32 * wq + 16 * mt;
                        ll_ldsm_x4_t(a, &sm.k[kk * 16 + (lane & 7) + ((lane >> 4) << 3)]
                                             [kc0 + ((lane >> 3) & 1) * 8]);
#pragma unroll
                        for (int n2 = 0; n2 < LL_BV / 16; ++n2) {
                            uint32_t b[4];
                            ll_ldsm_x4_t(b, &sm.v[kk * 16 + (lane & 15)][n2 * 16 + (lane >> 4) * 8]);
                            const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
                            ll_mma(s[mt][2 * n2], a, b0);
                            ll_mma(s[mt][2 * n2 + 1], a, b1);
                        }
                    }
                }
            }
        } else {
            // earlier chunks: one readout per set bit b of c, weighted by lambda^(7+b)
            for (int b = 0; b < LL_LEVELS; ++b) {
                if (!((c >> b) & 1)) continue;
                float z[LL_BV / 8][4];
#pragma unroll
                for (int n = 0; n < LL_BV / 8; ++n) z[n][0] = z[n][1] = z[n][2] = z[n][3] = 0.f;
                const float(*mb)[LL_MS] = sm.m[b];
#pragma unroll 4
                for (int kk = 0; kk < LL_DK / 16; ++kk) {
                    uint32_t a[4];
                    ll_ldsm_x4(a, &sm.q[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
#pragma unroll
                    for (int n = 0; n < LL_BV / 8; ++n) {
                        // B (k = key channel, n = value channel) from the fp32 state, as bf16:
                        // two adjacent key channels of one value row per 8-byte load
                        const int kc = kk * 16 + 2 * tg, vc = 8 * n + g;
                        const float2 lo = *reinterpret_cast<const float2*>(&mb[vc][kc]);
                        const float2 hi = *reinterpret_cast<const float2*>(&mb[vc][kc + 8]);
                        uint32_t bb[2];
                        bb[0] = pack_bf16(lo.x, lo.y);
                        bb[1] = pack_bf16(hi.x, hi.y);
                        ll_mma(z[n], a, bb);
                    }
                }
                const float la = sm.lam[ta][7 + b], lb = sm.lam[tb][7 + b];
#pragma unroll
                for (int n = 0; n < LL_BV / 8; ++n) {
                    o[n][0] = fmaf(la, z[n][0], o[n][0]);
                    o[n][1] = fmaf(la, z[n][1], o[n][1]);
                    o[n][2] = fmaf(lb, z[n][2], o[n][2]);
                    o[n][3] = fmaf(lb, z[n][3], o[n][3]);
                }
            }
            // hand the block-state part of the outputs to the in-chunk warps
#pragma unroll
            for (int n = 0; n < LL_BV / 8; ++n) {
                const int col = 8 * n + 2 * tg;
                *reinterpret_cast<float2*>(&sm.o[ta][col]) = make_float2(o[n][0], o[n][1]);
                *reinterpret_cast<float2*>(&sm.o[tb][col]) = make_float2(o[n][2], o[n][3]);
            }
        }
        __syncthreads();  // the block-state readouts are done (and their outputs are in sm.o)
        if (intra) {
#pragma unroll
            for (int n = 0; n < LL_BV / 8; ++n) {
                const int col = 8 * n + 2 * tg;
                const float2 xa = *reinterpret_cast<const float2*>(&sm.o[ta][col]);
                const float2 xb = *reinterpret_cast<const float2*>(&sm.o[tb][col]);
                if (t0 + ta < T)
                    *reinterpret_cast<uint32_t*>(out + (bh * T + t0 + ta) * (long)dv + v0 + col) =
                        pack_bf16(o[n][0] + xa.x, o[n][1] + xa.y);
                if (t0 + tb < T)
                    *reinterpret_cast<uint32_t*>(out + (bh * T + t0 + tb) * (long)dv + v0 + col) =
                        pack_bf16(o[n][2] + xb.x, o[n][3] + xb.y);
            }
            // binary counter: M_j = this chunk + sum_{b<j} M_b, M_b = 0 for b < j. Each thread
            // touches only its own (key channel, value channel) positions, and every readout
            // of the block states finished before the barrier above.
            if (c + 1 < nchunks) {
                int j = 0;
                while ((c >> j) & 1) ++j;
                if (j < LL_LEVELS) {
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
                        for (int n = 0; n < LL_BV / 8; ++n) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int kc = 32 * wq + 16 * mt + g + ((e & 2) ? 8 : 0);
                                const int vc = 8 * n + 2 * tg + (e & 1);
                                float x = s[mt][n][e];
                                for (int b = 0; b < j; ++b) {
                                    x += sm.m[b][vc][kc];
                                    sm.m[b][vc][kc] = 0.f;
                                }
                                sm.m[j][vc][kc] = x;
                            }
                        }
                    }
                }
            }
        }
    }
}

}  // namespace drscan
