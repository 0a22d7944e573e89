// Variational Linear Attention scan, warp-specialised, fp32, one CTA per (b,h).
//
// Two thread groups of d threads each:
//  * the A-group owns A (row i in thread i's registers) and produces the write direction
//    alpha_hat_t for every token: z = A_{t-1} u and y = A_{t-1} k in one pass over the row,
//    then ONE group reduction of u.z, k.z, y.y, y.z and z.z. With c = 1/(1 + u.z) and
//    w = c (k.z), A_t k = y - w z (Sherman-Morrison applied to the vector, so no second
//    dependent mat-vec) and ||A_t k||^2 = y.y - 2 w y.z + w^2 z.z, so the norm needs no
//    reduction of its own; then the rank-1 update of A's row;
//  * the S-group owns S (row i in thread i's registers); given alpha_hat_t its rows are
//    independent: r_i = v_i - s_i.k, s_i += r_i alpha_hat, and the readout after the write
//    o_i = s_i.q + r_i (alpha_hat.q), with s_i the row before the write: the two dot products
//    of a token run side by side. alpha_hat.q comes from the A-group (y.q and z.q join its
//    reduction: alpha_hat.q = (y.q - w z.q) / ||A_t k||). No reductions in the S-group.
// The groups run one token tile apart: while the A-group produces the directions of tile n
// into a shared-memory ring, the S-group consumes tile n-1. One __syncthreads per tile.
//
// Ratio readout (RATIO): o_t = S_t q_t / (n_t q_t) with n_t = n_{t-1} + (1 - n_{t-1} k_t)
// alpha_hat_t^T, the same write applied to a value held at 1. The A-group keeps n (element i
// in thread i) and computes the denominator without another serial reduction: n.k, n.q,
// y.q and z.q join the first reduction, and with c = 1/(1 + u.z),
//     alpha_hat.q = (y.q - c (k.z)(z.q)) / ||A_t k||,   n_t q = n.q + (1 - n.k) alpha_hat.q.
// The denominator rides in the ring next to alpha_hat; the S-group divides its readout.
#pragma once

#include "common.cuh"

namespace drscan {

constexpr int VLA_TILE = 16;

template <int D>
struct VlaSmem {
    float uA[2][VLA_TILE][D];
    float kA[2][VLA_TILE][D];
    float qA[2][VLA_TILE][D];  // the A-group's copy of q
    float kS[2][VLA_TILE][D];
    float vS[2][VLA_TILE][D];
    float qS[2][VLA_TILE][D];
    float ring[2][VLA_TILE][D];
    float aq[2][VLA_TILE];     // alpha_hat_t . q_t
    float den[2][VLA_TILE];    // ratio readout: n_t q_t
    // alternate tokens use alternate buffers: a token's writes never meet a slower thread's
    // reads of the previous token (one group barrier per token separates them)
    float zbuf[2][D];
    float red1[2][9][4];  // a token's partial sums, one slot per value and warp
};

// Sums N values over the D threads of a group (warp shuffles, then one named barrier to
// join the warps when D > 32); every thread gets the N totals.
template <int D, int N>
__device__ __forceinline__ void vla_group_sum(float* x, float (*red)[4], int i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int e = 0; e < N; ++e) x[e] += __shfl_xor_sync(0xffffffffu, x[e], off);
    if constexpr (D > 32) {
        if ((i & 31) == 0) {
#pragma unroll
            for (int e = 0; e < N; ++e) red[e][i >> 5] = x[e];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(D) : "memory");
#pragma unroll
        for (int e = 0; e < N; ++e) {
            x[e] = 0.f;
#pragma unroll
            for (int w = 0; w < D / 32; ++w) x[e] += red[e][w];
        }
    } else {
        __syncwarp();
    }
}

// Starts the copy of nt token rows of one operand into a tile buffer: 16-byte asynchronous
// copies (cp.async), so the issuing thread does not wait for HBM; vla_tiles_landed() waits
// for this thread's copies before the tile barrier that publishes them.
template <int D>
__device__ __forceinline__ void vla_load_tile(float (*dst)[D], const float* src, int nt, int tid) {
    const char* s = reinterpret_cast<const char*>(src);
    const uint32_t d = smem_u32(&dst[0][0]);
    for (int e = tid; e < nt * D / 4; e += D)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + 16u * e),
                     "l"(s + 16l * e)
                     : "memory");
}

__device__ __forceinline__ void vla_tiles_landed() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// grid: B*H; block: 2*D threads; dynamic shared memory: sizeof(VlaSmem<D>).
template <int D, bool RATIO>
__global__ void __launch_bounds__(2 * D) vla_sequential_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ u, const float* __restrict__ S0, const float* __restrict__ A0,
    const float* __restrict__ n0, float lambda0, float* __restrict__ out,
    float* __restrict__ S_final, float* __restrict__ A_final, float* __restrict__ n_final,
    int T) {
    extern __shared__ __align__(16) unsigned char vla_smem_raw[];
    VlaSmem<D>& sm = *reinterpret_cast<VlaSmem<D>*>(vla_smem_raw);

    const int tid = threadIdx.x;
    const bool is_a = tid < D;
    const int i = is_a ? tid : tid - D;
    const long bh = blockIdx.x;
    const long seq = bh * (long)T * D;
    const long mat = bh * (long)D * D;
    const int ntiles = (T + VLA_TILE - 1) / VLA_TILE;

    float m[D];  // row i of A (A-group) or of S (S-group)
    float nrm = 0.f;  // ratio readout: element i of n (A-group)
    if (is_a) {
        if constexpr (RATIO) nrm = n0 ? n0[bh * D + i] : 0.f;
        if (A0) {
#pragma unroll
            for (int j = 0; j < D; ++j) m[j] = A0[mat + (long)i * D + j];
        } else {
            const float inv = 1.f / lambda0;
#pragma unroll
            for (int j = 0; j < D; ++j) m[j] = (j == i) ? inv : 0.f;
        }
        if (ntiles > 0) {
            const int nt = min(VLA_TILE, T);
            vla_load_tile<D>(sm.uA[0], u + seq, nt, i);
            vla_load_tile<D>(sm.kA[0], k + seq, nt, i);
            vla_load_tile<D>(sm.qA[0], q + seq, nt, i);
            vla_tiles_landed();
        }
    } else {
        if (S0) {
#pragma unroll
            for (int j = 0; j < D; ++j) m[j] = S0[mat + (long)i * D + j];
        } else {
#pragma unroll
            for (int j = 0; j < D; ++j) m[j] = 0.f;
        }
    }
    __syncthreads();

    for (int it = 0; it <= ntiles; ++it) {
        if (is_a) {
            if (it + 1 < ntiles) {
                const int t0 = (it + 1) * VLA_TILE;
                const int nt = min(VLA_TILE, T - t0);
                vla_load_tile<D>(sm.uA[(it + 1) & 1], u + seq + (long)t0 * D, nt, i);
                vla_load_tile<D>(sm.kA[(it + 1) & 1], k + seq + (long)t0 * D, nt, i);
                vla_load_tile<D>(sm.qA[(it + 1) & 1], q + seq + (long)t0 * D, nt, i);
            }
            if (it < ntiles) {
                const int b = it & 1;
                const int nt = min(VLA_TILE, T - it * VLA_TILE);
                for (int tt = 0; tt < nt; ++tt) {
                    const int par = tt & 1;  // VLA_TILE is even: parity of the token index
                    const float* uu = sm.uA[b][tt];
                    const float* kk = sm.kA[b][tt];
                    // four partial sums per product (dependent FMA chains of D/4); the shared
                    // operands are read four at a time
                    float z4[4] = {0.f, 0.f, 0.f, 0.f}, y4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int j = 0; j < D; j += 4) {
                        const float4 u4 = *reinterpret_cast<const float4*>(uu + j);
                        const float4 k4 = *reinterpret_cast<const float4*>(kk + j);
                        z4[0] = fmaf(m[j], u4.x, z4[0]);
                        z4[1] = fmaf(m[j + 1], u4.y, z4[1]);
                        z4[2] = fmaf(m[j + 2], u4.z, z4[2]);
                        z4[3] = fmaf(m[j + 3], u4.w, z4[3]);
                        y4[0] = fmaf(m[j], k4.x, y4[0]);
                        y4[1] = fmaf(m[j + 1], k4.y, y4[1]);
                        y4[2] = fmaf(m[j + 2], k4.z, y4[2]);
                        y4[3] = fmaf(m[j + 3], k4.w, y4[3]);
                    }
                    const float z = (z4[0] + z4[1]) + (z4[2] + z4[3]);
                    const float y = (y4[0] + y4[1]) + (y4[2] + y4[3]);
                    sm.zbuf[par][i] = z;
                    // u.z, k.z, y.y, y.z, z.z, y.q, z.q (and for the ratio readout n.k, n.q)
                    constexpr int NR = RATIO ? 9 : 7;
                    float r1[NR];
                    const float qi = sm.qA[b][tt][i];
                    r1[0] = uu[i] * z;
                    r1[1] = kk[i] * z;
                    r1[2] = y * y;
                    r1[3] = y * z;
                    r1[4] = z * z;
                    r1[5] = y * qi;
                    r1[6] = z * qi;
                    if constexpr (RATIO) {
                        r1[7] = nrm * kk[i];
                        r1[8] = nrm * qi;
                    }
                    vla_group_sum<D, NR>(r1, sm.red1[par], i);
                    const float c = 1.f / (1.f + r1[0]);
                    const float w = c * r1[1];
                    const float* zb = sm.zbuf[par];
                    const float cz = -c * z;
#pragma unroll
                    for (int j = 0; j < D; j += 4) {
                        const float4 z4v = *reinterpret_cast<const float4*>(zb + j);
                        m[j] = fmaf(cz, z4v.x, m[j]);
                        m[j + 1] = fmaf(cz, z4v.y, m[j + 1]);
                        m[j + 2] = fmaf(cz, z4v.z, m[j + 2]);
                        m[j + 3] = fmaf(cz, z4v.w, m[j + 3]);
                    }
                    const float yt = fmaf(-w, z, y);  // A_t k = A_{t-1}k - c z (z.k)
                    const float n2 = fmaf(w * w, r1[4], fmaf(-2.f * w, r1[3], r1[2]));
                    const float inv = rsqrtf(n2);
                    sm.ring[b][tt][i] = yt * inv;
                    const float aq = fmaf(-w, r1[6], r1[5]) * inv;  // alpha_hat.q
                    if (i == 0) sm.aq[b][tt] = aq;
                    if constexpr (RATIO) {
                        const float g = 1.f - r1[7];  // 1 - n.k
                        nrm = fmaf(g, yt * inv, nrm);
                        if (i == 0) sm.den[b][tt] = fmaf(g, aq, r1[8]);  // n_t q_t
                    }
                }
            }
        } else {
            if (it < ntiles) {
                const int t0 = it * VLA_TILE;
                const int nt = min(VLA_TILE, T - t0);
                vla_load_tile<D>(sm.kS[it & 1], k + seq + (long)t0 * D, nt, i);
                vla_load_tile<D>(sm.vS[it & 1], v + seq + (long)t0 * D, nt, i);
                vla_load_tile<D>(sm.qS[it & 1], q + seq + (long)t0 * D, nt, i);
            }
            if (it >= 1) {
                const int b = (it - 1) & 1;
                const int t0 = (it - 1) * VLA_TILE;
                const int nt = min(VLA_TILE, T - t0);
                for (int tt = 0; tt < nt; ++tt) {
                    const float* kk = sm.kS[b][tt];
                    const float* qq = sm.qS[b][tt];
                    const float* al = sm.ring[b][tt];
                    // s.k and s.q of the row before the write, side by side
                    float p4[4] = {0.f, 0.f, 0.f, 0.f}, o4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int j = 0; j < D; j += 4) {
                        const float4 k4 = *reinterpret_cast<const float4*>(kk + j);
                        const float4 q4 = *reinterpret_cast<const float4*>(qq + j);
                        p4[0] = fmaf(m[j], k4.x, p4[0]);
                        p4[1] = fmaf(m[j + 1], k4.y, p4[1]);
                        p4[2] = fmaf(m[j + 2], k4.z, p4[2]);
                        p4[3] = fmaf(m[j + 3], k4.w, p4[3]);
                        o4[0] = fmaf(m[j], q4.x, o4[0]);
                        o4[1] = fmaf(m[j + 1], q4.y, o4[1]);
                        o4[2] = fmaf(m[j + 2], q4.z, o4[2]);
                        o4[3] = fmaf(m[j + 3], q4.w, o4[3]);
                    }
                    const float o0 = (o4[0] + o4[1]) + (o4[2] + o4[3]), o1 = 0.f;
                    const float r = sm.vS[b][tt][i] - ((p4[0] + p4[1]) + (p4[2] + p4[3]));
#pragma unroll
                    for (int j = 0; j < D; j += 4) {
                        const float4 a4 = *reinterpret_cast<const float4*>(al + j);
                        m[j] = fmaf(r, a4.x, m[j]);
                        m[j + 1] = fmaf(r, a4.y, m[j + 1]);
                        m[j + 2] = fmaf(r, a4.z, m[j + 2]);
                        m[j + 3] = fmaf(r, a4.w, m[j + 3]);
                    }
                    const float o = fmaf(r, sm.aq[b][tt], o0 + o1);  // s_t.q after the write
                    if constexpr (RATIO)
                        out[seq + (long)(t0 + tt) * D + i] = o / sm.den[b][tt];
                    else
                        out[seq + (long)(t0 + tt) * D + i] = o;
                }
            }
        }
        vla_tiles_landed();  // the next tile's copies are in shared memory before the barrier
        __syncthreads();
    }

    float* dst = is_a ? A_final : S_final;
    if (dst) {
#pragma unroll
        for (int j = 0; j < D; ++j) dst[mat + (long)i * D + j] = m[j];
    }
    if constexpr (RATIO) {
        if (is_a && n_final) n_final[bh * D + i] = nrm;
    }
}

}  // namespace drscan
