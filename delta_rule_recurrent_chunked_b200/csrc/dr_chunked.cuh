// Chunked delta-rule scan on sm_100a tensor cores (DeltaNet, Gated DeltaNet, KDA, Gated
// DeltaNet-2).
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
// (KDA: the decay sits inside the operands, K*gamma, Q*gamma and K/gamma per channel, and
// Khat^T = diag(gamma_C) (K/gamma)^T T. Gated DeltaNet-2 is Gated DeltaNet run on its erase
// directions e = b (.) k and write targets z = w (.) v, which its entry point forms in
// scratch before this kernel runs.) Rows 0-63 of MMA2 below are
// T Y = U, the chunk's write values u_t = beta_t r_t, stored when the caller asks for them.
//
// Contractions on tcgen05 (bf16 operands in 128-byte-swizzled shared memory, fp32
// accumulators in tensor memory), one CTA per (b, h, slice of BV value channels):
//   Gram   D_G  = [K;Q] K^T                M=128 N=64 K=128
//   PT     D_PT = P T                      M=128 N=64 K=64   (B read M/N-major)
//   H      D_H  = K^T Ttilde               M=128 N=64 K=64   (A and B read M/N-major)
//   MMA1   D1   = [K;Q] S0^T               M=128 N=BV K=128
//   MMA2   D2   = [T;PT] Y                 M=128 N=BV K=64
//   MMA3   S^T += Khat^T Y                 M=128 N=BV K=64   (fp32 state stays in TMEM)
// The unit-lower inverse (I + A)^{-1} is built on the CUDA cores: 16x16 diagonal blocks by
// substitution in fp32, then the off-diagonal blocks by two levels of block products
// (X21 = -X22 A21 X11) on tf32 mma.sync, whose 16-row tiles are below tcgen05's minimum M.
//
// Warp roles (512 threads), one CTA per (head, value slice) doing both sides:
//   warp 0      TMA producer of K and Q tiles; beta and GDN gate scalars
//   warp 1      chain MMA issuer (MMA1, MMA2, MMA3)
//   warp 2      prep MMA issuer (Gram, PT, H)
//   warp 3      tensor-memory allocation, then the TMA producer of V tiles
//   warps 4-7   chain warpgroup: residual Y, output rows, carried state (TMEM lane = row)
//   warps 8-15  prep warps: gates, Gram epilogue, UT inverse, operand staging
// The prep side runs up to one chunk ahead of the chain; the only serial dependency
// between chunks is the state (MMA1 -> residual -> MMA3 -> state copy -> MMA1).
// Split clusters (few heads; SPLIT): per head, 1-4 prep CTAs and 2 chain CTAs.
//   prep CTA:  warps 0 and 4 K/Q producers (one stage each), warp 1 distributor (bulk copies
//              of each prepared slot into the chain CTAs), warps 2 and 3 prep MMA issuers,
//              warps 8-11 and 12-15 two prep groups on alternate chunks;
//   chain CTA: warp 0 K/Q producer, warp 1 MMA1 issuer, warp 2 MMA3/MMA2 issuer, warp 3 V
//              producer, warps 4-7 and 8-11 two chain warpgroups sharing the value columns,
//              warp 12 slot releaser.
// Every wait is bounded: on a timeout the status word is latched, the CTA-wide abort flag
// is raised and all roles run to the end without waiting or issuing.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>


#include "common.cuh"

namespace drscan {

constexpr int CK = 64;    // chunk length
// KDA: lowest summed log alpha of one key channel over one chunk that the anchored
// factorisation represents exactly (its factors stay below exp(85) in fp32 and bf16)
constexpr float KDA_MIN_LOG_DECAY = -170.f;
constexpr int CDK = 128;  // key dimension of the chunked kernel
constexpr int CHUNK_THREADS = 512;

// Shared-memory layout (byte offsets from a 1024-aligned base) and TMEM columns.
// Unsplit: one CTA holds the prep and the chain operands side by side.
// SPLIT: prep CTAs and chain CTAs of a cluster share one layout in which the chain operands
// (two sub-chains' S and Y, the V stages) overlay the prep temporaries of two prep groups.
template <int MODE, int BV, bool SPLIT = false>
struct ChunkLayout {
    static constexpr bool kKda = MODE == DR_KDA;
    static constexpr bool kGdn = MODE == DR_GDN;  // scalar gate
    static_assert(!(SPLIT && kKda), "KDA is never split");
    static_assert(MODE != DR_GDN2, "Gated DeltaNet-2 runs as Gated DeltaNet on (q, e, z)");
    static constexpr int NS = 2;                          // K/Q stages
    static constexpr int NSV = (kKda && BV == 128) ? 1 : 2;  // V stages
    static constexpr int NP = (kKda && BV >= 64) ? 1 : 2;    // prepared-operand slots
    static constexpr int NKN = kKda ? 1 : 0;

    static constexpr int KQ_B = 32768;  // [K;Q] bf16: 2 panels x 128 rows x 128 B
    static constexpr int V_B = CK * BV * 2;
    // BV >= 64: the V tile is stored as 128-byte-swizzled panels of 64 channels (8 KB each),
    // so that the residual threads, each reading its own row, hit distinct banks
    static constexpr bool V_SWZ = BV >= 64;
    // The chain MMAs run with N = NB >= 64 so that Y and the bf16 state are stored as
    // M/N-major B operands in 64-column swizzled groups (whole-row 16-byte stores); columns
    // beyond the real ones are zero padding. Group g of S / Y sits at SS + g*16384 /
    // SY + g*8192.
    static constexpr int NB = BV < 64 ? 64 : BV;
    static constexpr int NG = NB / 64;
    static constexpr int SY_B = NG * 8192;   // Y: 64 rows (t) x 64 columns per group
    static constexpr int SS_B = NG * 16384;  // S: 128 rows (key channel) x 64 columns per group

    // A prepared-operand slot: [T; PT] (128 rows x 64), Khat^T (128 rows (dk) x 64 (t)),
    // gamma vector. Contiguous, so that one bulk copy hands it to another CTA of the cluster.
    static constexpr int SLOT_TP = 0, SLOT_KH = 16384, SLOT_GAM = 32768;
    static constexpr int SLOT_B = 32768 + 1024;
    // A split cluster copies only what the chain reads: PT rows, Khat^T and the gammas (the
    // T rows feed the prep CTA's own PT and H; the chain's MMA2 rows 0-63 are never read).
    static constexpr int COPY_OFF = SLOT_TP + 8192, COPY_B = SLOT_GAM + 512 - COPY_OFF;

    // prep temporaries of one group: P (64 rows, A operand of an M=64 MMA), Ttilde (GDN:
    // diag(gamma_C/gamma) T), A then X = (I+A)^{-1} (fp32 [64][68]), block scratch [32][36]
    static constexpr int AM_B = CK * 68 * 4, ZS_B = 32 * 36 * 4;

    static constexpr int KQ = 0;
    static constexpr int KN = KQ + NS * KQ_B;    // KDA: K/gamma, 2 panels x 64 rows
    static constexpr int SLOT = KN + NKN * 16384;
    static constexpr int X0 = SLOT + NP * SLOT_B;  // 1024-aligned
    // ---- unsplit
    static constexpr int U_PM = X0, U_TTS = X0 + 8192;
    static constexpr int U_SS = U_TTS + (kGdn ? 8192 : 0);
    static constexpr int U_SY = U_SS + SS_B;
    static constexpr int U_V = U_SY + SY_B;
    static constexpr int U_AM = U_V + NSV * V_B;
    static constexpr int U_END = U_AM + AM_B + ZS_B;
    // ---- split: prep view and chain view of the same region
    static constexpr int S_PM = X0, S_TTS = X0 + 8192, S_PM2 = X0 + 16384, S_TTS2 = X0 + 24576;
    static constexpr int S_AM = X0 + 32768, S_ZS = S_AM + AM_B;
    static constexpr int S_AM2 = S_ZS + ZS_B, S_ZS2 = S_AM2 + AM_B;
    static constexpr int S_SS = X0, S_SY = X0 + SS_B, S_V = S_SY + SY_B;
    // a chain CTA's third prepared-operand slot (its ring is three deep when the cluster has
    // two or more prep CTAs)
    static constexpr int SLOT2 = (S_V + NSV * V_B + 1023) / 1024 * 1024;
    static constexpr int S_END_PREP = S_ZS2 + ZS_B, S_END_CHAIN = SLOT2 + SLOT_B;
    static constexpr int S_END = S_END_PREP > S_END_CHAIN ? S_END_PREP : S_END_CHAIN;

    static constexpr int PM = SPLIT ? S_PM : U_PM;
    static constexpr int TTS = SPLIT ? S_TTS : U_TTS;
    static constexpr int PM2 = S_PM2, TTS2 = S_TTS2, AM2 = S_AM2, ZS2 = S_ZS2;
    static constexpr int SS = SPLIT ? S_SS : U_SS;  // S bf16, M/N-major B operand
    static constexpr int SY = SPLIT ? S_SY : U_SY;  // Y bf16, M/N-major B operand
    static constexpr int V = SPLIT ? S_V : U_V;     // V stages: 64 rows x BV bf16
    static constexpr int AM = SPLIT ? S_AM : U_AM;
    static constexpr int ZS = AM + AM_B;
    // per stage: beta[64]; GDN: g[64], 1/gamma[64], gamma[64] (cumulative log-decay and its
    // exponentials, computed by the producer warp)
    static constexpr int BG_B = 1024;
    static constexpr int BG = SPLIT ? S_END : U_END;
    static constexpr int PG = BG + NS * BG_B;    // prep-private: KDA scan exchange, gamma_C[128]
    static constexpr int BAR = PG + 3072;
    static constexpr int TOTAL = BAR + 512;
    static_assert(TOTAL + 1024 <= 232448, "shared memory budget");
    static_assert(NS % 2 == 0, "each of two prep groups owns whole K/Q stages");
    static_assert(X0 % 1024 == 0 && SS % 1024 == 0 && SY % 1024 == 0 && PM % 1024 == 0 &&
                      TTS % 1024 == 0 && PM2 % 1024 == 0 && TTS2 % 1024 == 0,
                  "swizzled operands need 1024-byte alignment");

    // TMEM columns. Prep: D_G then D_PT at COL_G, D_H at COL_H (second prep group: +128).
    // Chain: sub-chain g's D1, D2 and fp32 state at COL_D1/COL_D2/COL_S + 64 g; split chain
    // CTAs keep two D1 buffers (chunk parity b at +128 b) so that a chunk's outputs can still
    // be read while the next chunk's MMA1 runs.
    static constexpr int COL_G = 0;
    static constexpr int COL_H = 64;
    static constexpr int COL_D1 = SPLIT ? 0 : 128;
    static constexpr int COL_D2 = SPLIT ? 256 : 128 + NB;
    static constexpr int COL_S = SPLIT ? 384 : 128 + 2 * NB;
    static constexpr int NCOLS = SPLIT ? 512 : ((128 + 3 * NB) <= 256 ? 256 : 512);
};

// mbarrier indices inside the BAR block
enum ChunkBar {
    B_KQ_FULL = 0,    // [2]
    B_KQ_EMPTY = 2,   // [2]
    B_V_FULL = 4,     // [2]
    B_V_EMPTY = 6,    // [2]
    B_GO = 8,         // prep -> prep MMA: Gram operands ready, D_G free
    B_GRAM = 9,       // Gram done
    B_TREADY = 10,    // prep -> prep MMA: T staged
    B_HDONE = 11,     // PT and H done
    B_PREP = 12,      // [2] slot ready for the chain
    B_SLOT_EMPTY = 14,  // [2] slot consumed by the chain
    B_MMA1 = 16,
    B_YREADY = 17,
    B_MMA23 = 18,     // MMA2 and MMA3 done (split chain CTA: MMA3 done)
    B_STATE = 19,     // bf16 state copy ready for MMA1
    B_PEER_FREE = 20,  // [2] prep CTA: every chain CTA freed its copy of the slot
    B_GRP1 = 22,       // second prep group's GO, GRAM, TREADY, HDONE (prep CTA of a split)
    B_ODONE = 26,      // split chain CTA: the output rows are read out of TMEM
    B_PREP2 = 27,      // split chain CTA: third slot ready
    B_MMA2 = 28,       // split chain CTA: MMA2 done
    B_SFREE = 29,      // [3] split chain CTA: chain slot i read by every thread and every MMA
    B_COUNT = 32
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

__device__ __forceinline__ uint32_t tf32_bits(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D(16x8, fp32) += A(16x8, tf32, row) * B(8x8, tf32, col). Fragments: lane = 4*g + tg;
// A {(g,tg), (g+8,tg), (g,tg+4), (g+8,tg+4)}, B {(k=tg,n=g), (k=tg+4,n=g)},
// D {(g,2tg), (g,2tg+1), (g+8,2tg), (g+8,2tg+1)}.
__device__ __forceinline__ void mma_tf32(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// A fragment of the 16x8 tile at (r0, k0) of a row-major fp32 matrix with row stride ld.
__device__ __forceinline__ void frag_a(uint32_t* a, const float* m, int ld, int r0, int k0,
                                       int g, int tg) {
    a[0] = tf32_bits(m[(r0 + g) * ld + k0 + tg]);
    a[1] = tf32_bits(m[(r0 + g + 8) * ld + k0 + tg]);
    a[2] = tf32_bits(m[(r0 + g) * ld + k0 + tg + 4]);
    a[3] = tf32_bits(m[(r0 + g + 8) * ld + k0 + tg + 4]);
}

// B fragment of the 8x8 tile at (k0, n0) of a row-major (K rows) fp32 matrix.
__device__ __forceinline__ void frag_b(uint32_t* b, const float* m, int ld, int k0, int n0, int g,
                                       int tg) {
    b[0] = tf32_bits(m[(k0 + tg) * ld + n0 + g]);
    b[1] = tf32_bits(m[(k0 + tg + 4) * ld + n0 + g]);
}

// Store -D (16x8 fragment) at (r0, n0) of a row-major fp32 matrix.
__device__ __forceinline__ void store_neg_frag(float* m, int ld, int r0, int n0, const float* d,
                                               int g, int tg, float sign) {
    m[(r0 + g) * ld + n0 + 2 * tg] = sign * d[0];
    m[(r0 + g) * ld + n0 + 2 * tg + 1] = sign * d[1];
    m[(r0 + g + 8) * ld + n0 + 2 * tg] = sign * d[2];
    m[(r0 + g + 8) * ld + n0 + 2 * tg + 1] = sign * d[3];
}

// Named barrier of one prep group (ids 1 and 3; id 2 belongs to the chain warpgroup).
__device__ __forceinline__ void group_sync(int gi, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + 2 * gi), "r"(nthreads) : "memory");
}

// Per-launch options of the segmented scan (all off in a plain launch):
//   Ts         tokens from one sequence's start to the next in beta, gate, out and u_out (the
//              K/Q/V tensor maps carry the same stride); T for a plain launch
//   S_ckpt     when set, the state after the first ckpt_chunks chunks of each sequence is
//              written there too ([seq, dv, dk] fp32, like S_final)
//   expand     when set, a token whose step could grow a state difference (beta_t |k_t|^2 > 2,
//              or a gate above 1) ORs 1 into *expand
//   run_if     when set, the launch does nothing unless *run_if != 0 (every CTA returns first)
//   G, ext     G > 1: sequence bh is segment bh % G of head bh / G (T tokens each, Ts = T);
//              every segment but the last runs on for ext more tokens (a multiple of 64) into
//              the next one, whose outputs there it writes, and every segment but the first
//              writes no output for its own first ext tokens; S0 is [heads, dv, dk] and enters
//              segment 0 only (the others start from zero)
struct ChunkSeg {
    long Ts;
    float* S_ckpt;
    int ckpt_chunks;
    int* expand;
    const int* run_if;
    int G, ext;
};

// Per-device counts of segmented scans and of the chained reruns their checks asked for.
__device__ unsigned long long g_seg_scans = 0, g_seg_reruns = 0;

// SEG: the segment launch of the segmented scan (Gated DeltaNet on split clusters, KDA on
// one CTA per sequence), the only instances that read seg.G, seg.ext, seg.S_ckpt and
// seg.expand; the others compile without that code.
template <int MODE, int BV, bool SPLIT, bool SEG = false>
__global__ void __launch_bounds__(CHUNK_THREADS, 1) dr_chunked_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmV, const float* __restrict__ beta,
    const float* __restrict__ gate, const float* __restrict__ S0,
    __nv_bfloat16* __restrict__ out, float* __restrict__ S_final,
    __nv_bfloat16* __restrict__ u_out, int T_seq, int dv, int nprep, const ChunkSeg seg) {
    // a conditional launch whose condition is off: every CTA leaves before any barrier
    if (seg.run_if && *seg.run_if == 0) return;
    if (seg.run_if && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        atomicAdd(&g_seg_reruns, 1ull);
    static_assert(!SEG || (SPLIT && (MODE == DR_GDN || MODE == DR_DELTANET)) ||
                      (!SPLIT && MODE == DR_KDA),
                  "segments run on split DeltaNet / Gated DeltaNet and on unsplit KDA");
    const long Ts = seg.Ts;
    const int gseg = SEG ? (int)(blockIdx.x % seg.G) : 0;
    // tokens this CTA runs, and the chunks whose outputs it leaves to the segment before
    const int T = SEG ? T_seq + (gseg < seg.G - 1 ? seg.ext : 0) : T_seq;
    const int cskip = SEG ? (gseg > 0 ? seg.ext / CK : 0) : 0;
    // the one-CTA chain path below is compiled into split instances too (unused there): it
    // carries the segment code only in the unsplit segment instances
    constexpr bool kSegU = SEG && !SPLIT;
    const float* S0q = !S0   ? nullptr
                       : SEG ? (gseg == 0 ? S0 + (long)(blockIdx.x / seg.G) * dv * CDK : nullptr)
                             : S0 + (long)blockIdx.x * dv * CDK;
    using L = ChunkLayout<MODE, BV, SPLIT>;
    constexpr bool kGdn = L::kGdn;  // scalar gate (Gated DeltaNet)
    constexpr bool kKda = MODE == DR_KDA;
    constexpr int NS = L::NS, NSV = L::NSV, NP = L::NP;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::BAR + 8 * B_COUNT);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::BAR + 8 * B_COUNT + 16);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const long bh = blockIdx.x;
    const int nchunks = (T + CK - 1) / CK;
    // SPLIT: the CTAs of one head form a cluster; ranks 0..nprep-1 prepare the chunks'
    // operands ([T; PT], Khat^T, gamma), NGR consecutive chunks per rank in turn, and copy
    // them into the shared memory of ranks nprep.., each of which runs the chain for one
    // slice of BV value channels. Otherwise one CTA does both for its slice.
    static_assert(!(SPLIT && kKda), "KDA is never split");
    constexpr bool split = SPLIT;
    const int NPREP = SPLIT ? nprep : 1;
    constexpr int NGR = SPLIT ? 2 : 1;  // prep groups per prep CTA
    const int rank = split ? (int)blockIdx.y : 0;
    const int NCC = split ? (int)gridDim.y - NPREP : 1;  // chain CTAs per head
    const bool is_prep = !split || rank < NPREP;
    const bool is_chain = !split || rank >= NPREP;
    const int v0 = (split ? rank - NPREP : (int)blockIdx.y) * BV;
    // Chunks are dealt to the prep CTAs one at a time, so consecutive chunks are prepared and
    // copied by different CTAs. The chunks this CTA loads, in order: all of them, or (prep
    // CTA of a split cluster) chunk_of(m) = rank + m * NPREP; ordinal_of inverts it. A prep
    // CTA's groups take alternate ordinals and its prepared-operand slots follow the ordinal.
    const int pSP = is_chain ? 1 : NPREP, pbase = is_chain ? 0 : rank;
    auto chunk_of = [&](int m) { return pbase + m * pSP; };
    auto ordinal_of = [&](int c) { return (c - pbase) / pSP; };
    auto owner_of = [&](int c) { return c % NPREP; };           // prep rank of chunk c
    auto pslot_of = [&](int c) { return (c / NPREP) % NP; };    // its slot in that prep CTA
    // Chain-side slot ring: NP slots, or three in a split cluster with two or more prep CTAs
    // (then no two of the first three chunks share a prep CTA and prep slot, so the initial
    // credits complete distinct barrier phases).
    const int npc = (SPLIT && NPREP >= 2) ? 3 : NP;
    auto cslot = [&](int i) -> uint8_t* {
        if constexpr (SPLIT) {
            if (i == 2) return sm + L::SLOT2;
        }
        return sm + L::SLOT + i * L::SLOT_B;
    };
    auto cprep = [&](int i) { return bar(i == 2 ? B_PREP2 : B_PREP + i); };
    // a split cluster copies the PT rows, Khat^T and the gammas of each slot, and the T rows
    // as well when the chain CTAs export the write values (rows 0-63 of MMA2)
    const uint32_t copy_off = u_out ? (uint32_t)L::SLOT_TP : (uint32_t)L::COPY_OFF;
    const uint32_t copy_b = u_out ? (uint32_t)(L::COPY_B + 8192) : (uint32_t)L::COPY_B;
    auto slot = [&](int p) { return sm + L::SLOT + p * L::SLOT_B; };

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_KQ_FULL + s), 2);
            mbar_init(bar(B_KQ_EMPTY + s), split ? 1 : 2);
            mbar_init(bar(B_V_FULL + s), 1);
            mbar_init(bar(B_V_EMPTY + s), SPLIT ? 128 : 64);  // residual threads
            mbar_init(bar(B_PREP + s), 1);
            mbar_init(bar(B_SLOT_EMPTY + s), 1);
            mbar_init(bar(B_PEER_FREE + s), split ? NCC : 1);
        }
        mbar_init(bar(B_PREP2), 1);
        mbar_init(bar(B_MMA2), 1);
        for (int i = 0; i < 3; ++i) mbar_init(bar(B_SFREE + i), 257);  // 256 chain threads + MMA2
        const uint32_t gthreads = 256 / NGR;  // threads per prep group
        mbar_init(bar(B_GO), gthreads);
        mbar_init(bar(B_GRAM), 1);
        mbar_init(bar(B_TREADY), gthreads);
        mbar_init(bar(B_HDONE), 1);
        mbar_init(bar(B_GRP1 + 0), gthreads);
        mbar_init(bar(B_GRP1 + 1), 1);
        mbar_init(bar(B_GRP1 + 2), gthreads);
        mbar_init(bar(B_GRP1 + 3), 1);
        // output rows read out of D2 (and, when exporting, the write-value rows)
        mbar_init(bar(B_ODONE), u_out ? 256 : 128);
        mbar_init(bar(B_MMA1), 1);
        // split chain CTA: the residual threads arrive after writing Y, the others once the
        // state they rescaled in tensor memory for the next MMA3 is stored
        mbar_init(bar(B_YREADY), SPLIT ? 256 : 128);
        mbar_init(bar(B_MMA23), 1);
        mbar_init(bar(B_STATE), SPLIT ? 256 : 128);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 3) tmem_alloc(smem_u32(tmem_holder), L::NCOLS);
    // The padding columns of S and Y are read by the chain MMAs: keep them zero.
    for (int e = tid; e < (L::SS_B + L::SY_B) / 16; e += CHUNK_THREADS)
        reinterpret_cast<uint4*>(sm + L::SS)[e] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if constexpr (SPLIT) cluster_sync_all();  // peers' barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0 || (SPLIT && warp == 4 && !is_chain)) {
        // ------------------------------------------------------------------ producer
        // (a split prep CTA gives each prep group's K/Q stage its own producer: warp 0 loads
        // the even positions m, warp 4 the odd ones, so neither waits on the other's group)
        const int mstep = (SPLIT && !is_chain) ? 2 : 1;
        const int mfirst = (SPLIT && !is_chain && warp == 4) ? 1 : 0;
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmV);
        }
        for (int m = mfirst;; m += mstep) {
            const int c = chunk_of(m);
            if (c >= nchunks) break;
            const int s = m % NS;
            const int t0 = c * CK;
            if (m >= NS) mbar_wait(bar(B_KQ_EMPTY + s), (uint32_t)(((m / NS) - 1) & 1), abort_flag);
            // the tile loads go out first; the per-token scalars are computed while they fly
            // and the stage completes with the second arrival
            if (lane == 0 && !*abort_flag) {
                uint8_t* kq = sm + L::KQ + s * L::KQ_B;
                mbar_arrive_expect_tx(bar(B_KQ_FULL + s), L::KQ_B);
                for (int p = 0; p < 2; ++p) {
                    tma_load_3d(smem_u32(kq + p * 16384), &tmK, bar(B_KQ_FULL + s), p * 64, t0,
                                (int)bh);
                    tma_load_3d(smem_u32(kq + p * 16384 + 8192), &tmQ, bar(B_KQ_FULL + s), p * 64,
                                t0, (int)bh);
                }
            } else if (lane == 0) {
                mbar_arrive(bar(B_KQ_FULL + s));
            }
            float* bg = reinterpret_cast<float*>(sm + L::BG + s * L::BG_B);
            const float b0 = t0 + lane < T ? beta[bh * Ts + t0 + lane] : 0.f;
            const float b1 = t0 + 32 + lane < T ? beta[bh * Ts + t0 + 32 + lane] : 0.f;
            if constexpr (kGdn) {
                // g_t = sum of log alpha over the chunk's rows up to t (masked rows add 0)
                const float a0 = t0 + lane < T ? gate[bh * Ts + t0 + lane] : 1.f;
                const float a1 = t0 + 32 + lane < T ? gate[bh * Ts + t0 + 32 + lane] : 1.f;
                if (SEG && (a0 > 1.f || a1 > 1.f)) atomicOr(seg.expand, 1);
                float x0 = t0 + lane < T ? __logf(a0) : 0.f;
                float x1 = t0 + 32 + lane < T ? __logf(a1) : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
                    const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
                    if (lane >= off) {
                        x0 += y0;
                        x1 += y1;
                    }
                }
                x1 += __shfl_sync(0xffffffffu, x0, 31);
                bg[64 + lane] = x0;
                bg[96 + lane] = x1;
                bg[128 + lane] = __expf(-x0);
                bg[160 + lane] = __expf(-x1);
                bg[192 + lane] = __expf(x0);
                bg[224 + lane] = __expf(x1);
            }
            bg[lane] = b0;
            bg[32 + lane] = b1;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_KQ_FULL + s));
        }
    } else if (warp == 3 && is_chain) {
        // ------------------------------------------------------------------ V producer
        for (int c = 0; c < nchunks; ++c) {
            const int sv = c % NSV;
            if (lane == 0) {
                if (c >= NSV)
                    mbar_wait(bar(B_V_EMPTY + sv), (uint32_t)(((c / NSV) - 1) & 1), abort_flag);
                if (!*abort_flag) {
                    mbar_arrive_expect_tx(bar(B_V_FULL + sv), L::V_B);
                    constexpr int VB = L::V_SWZ ? 64 : BV;  // channels per TMA box
#pragma unroll
                    for (int pn = 0; pn < BV / VB; ++pn)
                        tma_load_3d(smem_u32(sm + L::V + sv * L::V_B + pn * CK * VB * 2), &tmV,
                                    bar(B_V_FULL + sv), v0 + pn * VB, c * CK, (int)bh);
                }
            }
        }
    } else if (warp == 1 && !is_chain) {
        // ------------------------------------------------------------------ slot distributor
        // (prep CTA of a split cluster): ships each prepared slot to the chain CTAs once all
        // of them have freed their copy, then hands the slot back to the prep warps
        if (lane == 0) {
            for (int m = 0;; ++m) {
                const int c = chunk_of(m);
                if (c >= nchunks) break;
                const int p = m % NP;
                const uint32_t ph = (uint32_t)((m / NP) & 1);
                mbar_wait(bar(B_PREP + p), ph, abort_flag);
                mbar_wait(bar(B_PEER_FREE + p), ph, abort_flag);
                if (!*abort_flag) {
                    // into chain slot c % npc of every chain rank
                    const uint32_t src = smem_u32(slot(p)) + copy_off;
                    const uint32_t dst = smem_u32(cslot(c % npc)) + copy_off;
                    for (int q = NPREP; q < NPREP + NCC; ++q)  // the chain ranks
                        bulk_copy_to_peer(cluster_map(dst, q), src, copy_b,
                                          cluster_map(cprep(c % npc), q));
                    bulk_commit_and_wait_read();
                }
                mbar_arrive(bar(B_SLOT_EMPTY + p));
            }
            // No copy may still be writing into a chain CTA when the cluster's final barrier
            // lets it exit (after a timeout its chain no longer waits for every slot).
            bulk_wait_all();
        }
    } else if (warp == 1 || (SPLIT && warp == 2 && is_chain)) {
        // ------------------------------------------------------------------ chain MMA issuer
        // Unsplit: warp 1 issues MMA1, MMA2 and MMA3. Split chain CTA: warp 1 issues MMA1 (it
        // needs only K/Q and the state copy), warp 2 the state update MMA3 and then MMA2, so
        // neither issuer's waits delay the other's step of the chain.
        if (lane == 0) {
            constexpr uint32_t id1 = idesc_bf16(128, L::NB, 0, 1);
            const bool do_mma1 = warp == 1, do_mma23 = !SPLIT || warp == 2;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                uint8_t* kq = sm + L::KQ + s * L::KQ_B;
                if (do_mma1) {
                    mbar_wait(bar(B_KQ_FULL + s), (uint32_t)((c / NS) & 1), abort_flag);
                    if constexpr (!SPLIT)
                        mbar_wait(cprep(c % npc), (uint32_t)((c / npc) & 1), abort_flag);
                    mbar_wait(bar(B_STATE), (uint32_t)(c & 1), abort_flag);
                    tc_fence_after();
                    if (!*abort_flag) {
                        const uint32_t d1 = L::COL_D1 + (SPLIT ? 128 * (c & 1) : 0);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const int pn = kk >> 2, ko = (kk & 3) * 32;
                            tc_mma_bf16(tmem + d1,
                                        smem_desc_sw128(smem_u32(kq + pn * 16384 + ko), 16, 1024),
                                        smem_desc_sw128(smem_u32(sm + L::SS + kk * 2048), 16384, 1024),
                                        id1, kk > 0);
                        }
                        tc_commit(bar(B_MMA1));
                        tc_commit(bar(B_KQ_EMPTY + s));
                    }
                }
                if (!do_mma23) continue;
                if constexpr (SPLIT) mbar_wait(cprep(c % npc), (uint32_t)((c / npc) & 1), abort_flag);
                const uint8_t* tp = cslot(c % npc) + L::SLOT_TP;
                const uint8_t* kh = cslot(c % npc) + L::SLOT_KH;
                mbar_wait(bar(B_YREADY), (uint32_t)(c & 1), abort_flag);
                tc_fence_after();
                auto mma3 = [&]() {  // S^T += Khat^T Y
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem + L::COL_S, smem_desc_sw128(smem_u32(kh + kk * 32), 16, 1024),
                                    smem_desc_sw128(smem_u32(sm + L::SY + kk * 2048), 8192, 1024), id1,
                                    1);
                };
                auto mma2 = [&]() {  // D2 = [T; PT] Y
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem + L::COL_D2, smem_desc_sw128(smem_u32(tp + kk * 32), 16, 1024),
                                    smem_desc_sw128(smem_u32(sm + L::SY + kk * 2048), 8192, 1024), id1,
                                    kk > 0);
                };
                if constexpr (SPLIT) {
                    // the state update first (it is on the chain's critical path), then the
                    // output rows once the previous chunk's are out of D2
                    if (!*abort_flag) {
                        mma3();
                        tc_commit(bar(B_MMA23));
                    }
                    if (c > 0) mbar_wait(bar(B_ODONE), (uint32_t)((c - 1) & 1), abort_flag);
                    tc_fence_after();
                    if (!*abort_flag) {
                        mma2();
                        tc_commit(bar(B_MMA2));
                        tc_commit(bar(B_SFREE + c % npc));  // last reader of the slot
                    }
                } else {
                    if (!*abort_flag) {
                        mma2();
                        mma3();
                        tc_commit(bar(B_MMA23));
                    }
                }
            }
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------------ prep MMA issuer
        // warp 2 serves prep group 0; warp 3 serves group 1 in the prep CTA of a split cluster
        const int gi = warp - 2;
        if (!is_prep || gi >= NGR) goto done;
        if (lane == 0) {
            constexpr uint32_t idg = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idp = idesc_bf16(64, 64, 0, 1);  // D row m -> lane m%16 + 32*(m/16)
            constexpr uint32_t idh = idesc_bf16(128, 64, 1, 1);
            const int gb = gi ? B_GRP1 : B_GO;
            const uint32_t cg = L::COL_G + 128 * gi, chh = L::COL_H + 128 * gi;
            uint8_t* pm = sm + (gi ? L::PM2 : L::PM);
            uint8_t* tts = sm + (gi ? L::TTS2 : L::TTS);
            int k = 0;  // the group's chunk ordinal
            for (int c = pbase + gi * pSP; c < nchunks; c += NGR * pSP, ++k) {
                const int s = ordinal_of(c) % NS, p = ordinal_of(c) % NP;
                uint8_t* kq = sm + L::KQ + s * L::KQ_B;
                uint8_t* kn = sm + L::KN;
                const uint32_t jp = (uint32_t)(k & 1);
                mbar_wait(bar(gb + 0), jp, abort_flag);
                tc_fence_after();
                if (!*abort_flag) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int pn = kk >> 2, ko = (kk & 3) * 32;
                        const uint64_t a = smem_desc_sw128(smem_u32(kq + pn * 16384 + ko), 16, 1024);
                        const uint64_t b =
                            kKda ? smem_desc_sw128(smem_u32(kn + pn * 8192 + ko), 16, 1024) : a;
                        tc_mma_bf16(tmem + cg, a, b, idg, kk > 0);
                    }
                    tc_commit(bar(gb + 1));
                }
                mbar_wait(bar(gb + 2), jp, abort_flag);
                tc_fence_after();
                if (!*abort_flag) {
                    const uint8_t* tp = slot(p) + L::SLOT_TP;
                    // PT = P T: B = T read M/N-major from the slot's rows 0-63
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem + cg, smem_desc_sw128(smem_u32(pm + kk * 32), 16, 1024),
                                    smem_desc_sw128(smem_u32(tp + kk * 2048), 1024, 1024), idp, kk > 0);
                    // H: A = K^T (KDA: (K/g)^T) M/N-major, B = Ttilde (or T) M/N-major
                    const uint8_t* bt = kGdn ? tts : tp;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a =
                            kKda ? smem_desc_sw128(smem_u32(kn + kk * 2048), 8192, 1024)
                                 : smem_desc_sw128(smem_u32(kq + kk * 2048), 16384, 1024);
                        tc_mma_bf16(tmem + chh, a,
                                    smem_desc_sw128(smem_u32(bt + kk * 2048), 1024, 1024), idh,
                                    kk > 0);
                    }
                    tc_commit(bar(gb + 3));
                    tc_commit(bar(B_KQ_EMPTY + s));
                }
            }
        }
    } else if (SPLIT && is_chain && warp >= 4 && warp < 12) {
        // ------------------------------------------------------------------ chain warpgroups
        // of a split chain CTA. Warps 4-7 and 8-11 reach the same TMEM lanes and share the
        // value columns: warpgroup h takes HC columns from cb (with 16 channels the second only
        // keeps the barrier counts). Threads 0-63 of each (TMEM lanes of the K rows) write the
        // residuals, threads 64-127 (Q rows) the outputs, all (lane = key channel) the state.
        // Per chunk: the residuals; then the state, already scaled by the next chunk's gamma_C
        // and handed straight to MMA1; then the outputs, which overlap the next residuals.
        const int h = warp >= 8 ? 1 : 0;
        constexpr int HC = BV >= 32 ? BV / 2 : BV;  // columns per warpgroup
        const bool active = BV >= 32 || h == 0;
        const int cb = h * HC;                     // first column (0, 16 or 32)
        constexpr int LW = HC < 16 ? 16 : HC;      // TMEM columns read (one piece: <= 32)
        constexpr int NV8 = HC / 8;                // real 8-column chunks
        static_assert(!SPLIT || LW <= 32, "one epilogue piece per warpgroup");
        const int r = tid - (h ? 256 : 128);  // TMEM lane: row t (Y, O) or key channel j (state)
        const uint32_t trow = tmem + ((uint32_t)(r & ~31) << 16);
        // gamma_t of row r & 63 for the next chunk: each chunk's slot is waited for, and its
        // gammas read, one chunk ahead (under the previous chunk's MMA3 latency)
        float gt_next = 1.f;
        {
            // slots start empty: expect the prep CTAs' copies of the first chunks
            if (h == 0 && r == 0) {
                for (int c = 0; c < npc && c < nchunks; ++c) {
                    mbar_arrive_expect_tx(cprep(c), copy_b);
                    mbar_arrive_remote(cluster_map(bar(B_PEER_FREE + pslot_of(c)), owner_of(c)));
                }
            }
            float gC0 = 1.f;
            if (nchunks > 0) {
                mbar_wait(cprep(0), 0u, abort_flag);
                if constexpr (kGdn) {
                    const float* gam = reinterpret_cast<const float*>(cslot(0) + L::SLOT_GAM);
                    gt_next = gam[r & 63];
                    gC0 = gam[64];
                }
                mbar_arrive(bar(B_SFREE + 0));  // this thread is done reading slot 0
            }
            if (active) {
                const float* src = S0q ? S0q + (v0 + cb) * (long)CDK + r : nullptr;
                float sv[LW];
#pragma unroll
                for (int v = 0; v < LW; ++v) sv[v] = (src && v < HC) ? src[(long)v * CDK] : 0.f;
#pragma unroll
                for (int i = 0; i < NV8; ++i) st_row_chunk(sm + L::SS, r, cb / 8 + i, sv + 8 * i);
#pragma unroll
                for (int c16 = 0; c16 < LW; c16 += 16) {
                    float w[16];
#pragma unroll
                    for (int v = 0; v < 16; ++v) w[v] = sv[c16 + v] * gC0;
                    tmem_st16(trow + L::COL_S + cb + c16, w);
                }
            }
            if (h == 0) {  // the padding columns of the fp32 state start at zero
                float w[16];
#pragma unroll
                for (int v = 0; v < 16; ++v) w[v] = 0.f;
                for (int c16 = (BV + 15) / 16 * 16; c16 < 64; c16 += 16) tmem_st16(trow + L::COL_S + c16, w);
            }
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bar(B_STATE));
            if (r >= 64) mbar_arrive(bar(B_YREADY));  // the first MMA3 may use the state
        }
        // write values U = T Y of chunk c (rows 0-63 of D2), read by the residual threads once
        // MMA2 of that chunk is done; D2 is reused only after they (and the output threads)
        // arrive on B_ODONE
        auto export_u = [&](int c) {
            mbar_wait(bar(B_MMA2), (uint32_t)(c & 1), abort_flag);
            tc_fence_after();
            if (active) {
                float d[LW];
#pragma unroll
                for (int c16 = 0; c16 < LW; c16 += 16) tmem_ld16(trow + L::COL_D2 + cb + c16, d + c16);
                tmem_wait_ld();
                if (c * CK + r < T && (!SEG || c >= cskip)) {
                    uint4* dst = reinterpret_cast<uint4*>(u_out + (bh * Ts + c * CK + r) * (long)dv + v0 + cb);
#pragma unroll
                    for (int i = 0; i < NV8; ++i) {
                        uint4 w;
                        uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e) wp[e] = pack_bf16(d[8 * i + 2 * e], d[8 * i + 2 * e + 1]);
                        dst[i] = w;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_ODONE));
        };
        for (int c = 0; c < nchunks; ++c) {
            const int svi = c % NSV;
            const int t0 = c * CK;
            const int nvalid = min(CK, T - t0);
            const uint32_t d1 = L::COL_D1 + 128 * (c & 1);
            const float gt = gt_next;
            const bool last = c == nchunks - 1;
            if (u_out && r < 64 && c > 0) export_u(c - 1);
            // ---- residuals Y = V - gamma_t (S0 k_t), stored as the B operand Y^T
            if (r < 64) {
                if (active) {
                    mbar_wait(bar(B_MMA1), (uint32_t)(c & 1), abort_flag);
                    tc_fence_after();
                    mbar_wait(bar(B_V_FULL + svi), (uint32_t)((c / NSV) & 1), abort_flag);
                    const uint8_t* vst = sm + L::V + svi * L::V_B + r * BV * 2;  // row r of V
                    float x[LW];
                    uint4 vw[NV8];
#pragma unroll
                    for (int c16 = 0; c16 < LW; c16 += 16) tmem_ld16(trow + d1 + cb + c16, x + c16);
#pragma unroll
                    for (int i = 0; i < NV8; ++i) {
                        const int j = cb / 8 + i;  // 16-byte chunk of the row
                        vw[i] = *reinterpret_cast<const uint4*>(
                            vst + ((L::V_SWZ ? (j ^ (r & 7)) : j) << 4));
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < NV8; ++i) {
                        const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&vw[i]);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = fmaf(-gt, x[8 * i + e], __bfloat162float(hv[e]));
                        st_row_chunk(sm + L::SY, r, cb / 8 + i, y);
                    }
                }
                mbar_arrive(bar(B_V_EMPTY + svi));
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bar(B_YREADY));
            }
            // ---- carried state: bf16 copy for MMA1 of the next chunk, fp32 S_final after the
            // last; the fp32 state takes the next chunk's gamma_C (from its slot, waited here
            // under the MMA3 latency) before that chunk's MMA3
            float gCn = 1.f;
            if (!last) {
                const int pn = (c + 1) % npc;
                mbar_wait(cprep(pn), (uint32_t)(((c + 1) / npc) & 1), abort_flag);
                if constexpr (kGdn) {
                    const float* gam = reinterpret_cast<const float*>(cslot(pn) + L::SLOT_GAM);
                    gt_next = gam[r & 63];
                    gCn = gam[64];
                }
                mbar_arrive(bar(B_SFREE + pn));  // this thread is done reading that slot
            }
            mbar_wait(bar(B_MMA23), (uint32_t)(c & 1), abort_flag);
            tc_fence_after();
            // the bf16 copy goes to MMA1 first; the fp32 state is rescaled for the next MMA3
            // after that hand-off (MMA3 waits for it through B_YREADY)
            float sv[LW];
            if (active) {
#pragma unroll
                for (int c16 = 0; c16 < LW; c16 += 16) tmem_ld16(trow + L::COL_S + cb + c16, sv + c16);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < NV8; ++i) st_row_chunk(sm + L::SS, r, cb / 8 + i, sv + 8 * i);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bar(B_STATE));
            if (active) {
                if (last && S_final) {
                    float* dst = S_final + (bh * dv + v0 + cb) * (long)CDK + r;
#pragma unroll
                    for (int v = 0; v < HC; ++v) dst[(long)v * CDK] = sv[v];
                }
                if (SEG && c + 1 == seg.ckpt_chunks) {
                    float* dst = seg.S_ckpt + (bh * dv + v0 + cb) * (long)CDK + r;
#pragma unroll
                    for (int v = 0; v < HC; ++v) dst[(long)v * CDK] = sv[v];
                }
                if constexpr (kGdn) {
                    if (!last) {
#pragma unroll
                        for (int v = 0; v < LW; ++v) sv[v] *= gCn;
#pragma unroll
                        for (int c16 = 0; c16 < LW; c16 += 16) tmem_st16(trow + L::COL_S + cb + c16, sv + c16);
                        tmem_wait_st();
                    }
                }
            }
            if (r >= 64 && !last) {
                tc_fence_before();
                mbar_arrive(bar(B_YREADY));  // for the next chunk's MMA3
            }
            // ---- outputs O = gamma_t (S0 q_t) + (P T Y)_t, overlapping the next residuals
            if (r >= 64) {
                const int t = r - 64;
                mbar_wait(bar(B_MMA2), (uint32_t)(c & 1), abort_flag);
                tc_fence_after();
                if (active) {
                    float z[LW], dd[LW];
#pragma unroll
                    for (int c16 = 0; c16 < LW; c16 += 16) {
                        tmem_ld16(trow + d1 + cb + c16, z + c16);
                        tmem_ld16(trow + L::COL_D2 + cb + c16, dd + c16);
                    }
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(bar(B_ODONE));
                    if (t < nvalid && (!SEG || c >= cskip)) {
                        uint4* dst = reinterpret_cast<uint4*>(out + (bh * Ts + t0 + t) * (long)dv + v0 + cb);
#pragma unroll
                        for (int i = 0; i < NV8; ++i) {
                            uint4 w;
                            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                wp[e] = pack_bf16(fmaf(gt, z[8 * i + 2 * e], dd[8 * i + 2 * e]),
                                                  fmaf(gt, z[8 * i + 2 * e + 1], dd[8 * i + 2 * e + 1]));
                            dst[i] = w;
                        }
                    }
                } else {
                    mbar_arrive(bar(B_ODONE));
                }
            }
        }
        if (u_out && r < 64 && nchunks > 0) export_u(nchunks - 1);
    } else if (warp >= 4 && warp < 8) {
        if (!is_chain) goto done;
        // ------------------------------------------------------------------ chain warpgroup
        const int r = tid - 128;  // TMEM lane: value row t (Y, O) or key channel j (state)
        const uint32_t trow = tmem + ((uint32_t)(r & ~31) << 16);
        // KDA: the bf16 copy of a chunk's entering state is scaled per key channel (lane r) by
        // exp(m), m the chunk's anchor, published by the prep warps before they release the
        // Gram operands of that chunk (phase c of B_GO)
        auto state_anchor = [&](int c) -> float {
            if constexpr (kKda) {
                mbar_wait(bar(B_GO), (uint32_t)(c & 1), abort_flag);
                return reinterpret_cast<const float*>(sm + L::BG + (c % NS) * L::BG_B)[128 + r];
            } else {
                return 1.f;
            }
        };
        {
            const float* src = S0q ? S0q + (long)v0 * CDK + r : nullptr;
            const float em = state_anchor(0);
#pragma unroll
            for (int c16 = 0; c16 < L::NB; c16 += 16) {
                float sv[16], sb[16];
#pragma unroll
                for (int v = 0; v < 16; ++v) {
                    sv[v] = (src && c16 < BV) ? src[(long)(c16 + v) * CDK] : 0.f;
                    sb[v] = sv[v] * em;
                }
                if (c16 < BV) {
                    uint8_t* grp = sm + L::SS + (c16 >> 6) * 16384;
                    st_row_chunk(grp, r, (c16 & 63) >> 3, sb);
                    st_row_chunk(grp, r, ((c16 & 63) >> 3) + 1, sb + 8);
                }
                tmem_st16(trow + L::COL_S + c16, sv);
            }
            tmem_wait_st();
            fence_async_smem();
            mbar_arrive(bar(B_STATE));
            // slots start empty: expect the prep CTA's copies of the first chunks
        }
        auto prescale = [&](int c) {  // S^T *= gamma_C of chunk c, before MMA3(c)
            if constexpr (MODE != DR_DELTANET) {
                const int p = c % NP;
                mbar_wait(bar(B_PREP + p), (uint32_t)((c / NP) & 1), abort_flag);
                const float* gam = reinterpret_cast<const float*>(slot(p) + L::SLOT_GAM);
                const float gC = kKda ? gam[r] : gam[64];
                constexpr int PW = BV < 32 ? BV : 32;  // columns per tensor-memory round trip
#pragma unroll
                for (int c0 = 0; c0 < BV; c0 += PW) {
                    float sv[PW];
#pragma unroll
                    for (int c16 = 0; c16 < PW; c16 += 16) tmem_ld16(trow + L::COL_S + c0 + c16, sv + c16);
                    tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < PW; ++v) sv[v] *= gC;
#pragma unroll
                    for (int c16 = 0; c16 < PW; c16 += 16) tmem_st16(trow + L::COL_S + c0 + c16, sv + c16);
                }
                tmem_wait_st();
            }
        };
        if (nchunks > 0) prescale(0);
        for (int c = 0; c < nchunks; ++c) {
            const int p = c % NP, svi = c % NSV;
            const int t0 = c * CK;
            const int nvalid = min(CK, T - t0);
            const float* gam = reinterpret_cast<const float*>(slot(p) + L::SLOT_GAM);
            mbar_wait(bar(B_MMA1), (uint32_t)(c & 1), abort_flag);
            tc_fence_after();
            if (r < 64) {
                // residual Y = V - gamma_t (S0 k_t), stored as the B operand Y^T
                mbar_wait(bar(B_V_FULL + svi), (uint32_t)((c / NSV) & 1),
                          abort_flag);
                const float gt = kGdn ? gam[r] : 1.f;
                // row r of V: 16-byte piece jj (channels 8jj .. 8jj+7)
                const uint8_t* vtile = sm + L::V + svi * L::V_B;
                auto vpiece = [&](int jj) -> uint4 {
                    if constexpr (L::V_SWZ)
                        return *reinterpret_cast<const uint4*>(
                            vtile + (jj >> 3) * (CK * 128) + r * 128 + (((jj & 7) ^ (r & 7)) << 4));
                    else
                        return *reinterpret_cast<const uint4*>(vtile + r * BV * 2 + jj * 16);
                };
                constexpr int HW = BV < 64 ? BV : 64;  // columns per pass
#pragma unroll
                for (int c0 = 0; c0 < BV; c0 += HW) {
                    float x[HW];
                    uint4 vw[HW / 8];
#pragma unroll
                    for (int c16 = 0; c16 < HW; c16 += 16) tmem_ld16(trow + L::COL_D1 + c0 + c16, x + c16);
#pragma unroll
                    for (int i = 0; i < HW / 8; ++i) vw[i] = vpiece(c0 / 8 + i);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < HW / 8; ++i) {
                        const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&vw[i]);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = fmaf(-gt, x[8 * i + e], __bfloat162float(hv[e]));
                        const int col = c0 + 8 * i;
                        st_row_chunk(sm + L::SY + (col >> 6) * 8192, r, (col & 63) >> 3, y);
                    }
                }
                mbar_arrive(bar(B_V_EMPTY + svi));
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bar(B_YREADY));

            mbar_wait(bar(B_MMA23), (uint32_t)(c & 1), abort_flag);
            tc_fence_after();
            if (r < 64 && u_out) {
                // write values U = T Y (rows 0-63 of D2)
#pragma unroll
                for (int c16 = 0; c16 < BV; c16 += 16) {
                    float d[16];
                    tmem_ld16(trow + L::COL_D2 + c16, d);
                    tmem_wait_ld();
                    if (r < nvalid && (!kSegU || c >= cskip)) {
                        uint4 w[2];
                        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                        for (int e = 0; e < 8; ++e) wp[e] = pack_bf16(d[2 * e], d[2 * e + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(u_out + (bh * Ts + t0 + r) * (long)dv +
                                                              v0 + c16);
                        dst[0] = w[0];
                        dst[1] = w[1];
                    }
                }
            }
            if (r >= 64) {
                // output rows: O = gamma_t (S0 q_t) + (P T Y)_t
                const int t = r - 64;
                const float gt = kGdn ? gam[t] : 1.f;
                constexpr int PW = BV < 32 ? BV : 32;  // columns per tensor-memory round trip
#pragma unroll
                for (int c0 = 0; c0 < BV; c0 += PW) {
                    float z[PW], d[PW];
#pragma unroll
                    for (int c16 = 0; c16 < PW; c16 += 16) {
                        tmem_ld16(trow + L::COL_D1 + c0 + c16, z + c16);
                        tmem_ld16(trow + L::COL_D2 + c0 + c16, d + c16);
                    }
                    tmem_wait_ld();
                    if (t < nvalid && (!kSegU || c >= cskip)) {
                        uint4* dst = reinterpret_cast<uint4*>(out + (bh * Ts + t0 + t) * (long)dv +
                                                              v0 + c0);
#pragma unroll
                        for (int i = 0; i < PW / 8; ++i) {
                            uint4 w;
                            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                wp[e] = pack_bf16(fmaf(gt, z[8 * i + 2 * e], d[8 * i + 2 * e]),
                                                  fmaf(gt, z[8 * i + 2 * e + 1], d[8 * i + 2 * e + 1]));
                            dst[i] = w;
                        }
                    }
                }
            }
            // carried state: bf16 copy for the next MMA1; fp32 S_final after the last chunk
            {
                float* dst = (c == nchunks - 1 && S_final)
                                 ? S_final + (bh * dv + v0) * (long)CDK + r
                                 : nullptr;
                float* dck = (kSegU && c + 1 == seg.ckpt_chunks)
                                 ? seg.S_ckpt + (bh * dv + v0) * (long)CDK + r
                                 : nullptr;
                const float em = (kKda && c + 1 < nchunks) ? state_anchor(c + 1) : 1.f;
                constexpr int HW = BV < 64 ? BV : 64;
#pragma unroll
                for (int c0 = 0; c0 < BV; c0 += HW) {
                    float sv[HW];
#pragma unroll
                    for (int c16 = 0; c16 < HW; c16 += 16) tmem_ld16(trow + L::COL_S + c0 + c16, sv + c16);
                    tmem_wait_ld();
                    if (dst) {
#pragma unroll
                        for (int v = 0; v < HW; ++v) dst[(long)(c0 + v) * CDK] = sv[v];
                    }
                    if (kSegU && dck) {
#pragma unroll
                        for (int v = 0; v < HW; ++v) dck[(long)(c0 + v) * CDK] = sv[v];
                    }
                    if constexpr (kKda) {
#pragma unroll
                        for (int v = 0; v < HW; ++v) sv[v] *= em;
                    }
#pragma unroll
                    for (int i = 0; i < HW / 8; ++i) {
                        const int col = c0 + 8 * i;
                        st_row_chunk(sm + L::SS + (col >> 6) * 16384, r, (col & 63) >> 3, sv + 8 * i);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bar(B_STATE));
            // slot p is free once every chain thread is done with it (MMA2/3 completed before
            // the wait above); hand it to whoever fills it next
            asm volatile("bar.sync 2, 128;" ::: "memory");
            if (r == 0 && c + NP < nchunks) mbar_arrive(bar(B_SLOT_EMPTY + p));
            if (c + 1 < nchunks) prescale(c + 1);
        }
    } else if (SPLIT && warp == 12 && is_chain) {
        // ------------------------------------------------------------------ slot releaser
        // (split chain CTA): once every chain thread and every MMA is done with chain slot
        // c % npc (warp 12), expect chunk c + npc in it and credit the prep CTA that owns it.
        // The slot's next phase needs this release, so the waits here never fall two phases
        // behind.
        if (lane == 0) {
            for (int c = 0; c + npc < nchunks; ++c) {
                mbar_wait(bar(B_SFREE + c % npc), (uint32_t)((c / npc) & 1), abort_flag);
                mbar_arrive_expect_tx(cprep(c % npc), copy_b);
                mbar_arrive_remote(cluster_map(bar(B_PEER_FREE + pslot_of(c + npc)), owner_of(c + npc)));
            }
        }
    } else if (warp >= 8) {
        if (!is_prep) goto done;
        // ------------------------------------------------------------------ prep warps
        // Without `split`, warps 8-15 form one prep group. In the prep CTA of a split cluster
        // they form two groups of four warps (8-11 and 12-15) that take alternate chunks, each
        // with its own TMEM columns, temporaries, mbarriers and named barrier. Group-local
        // thread u; lq = the TMEM lane this thread reaches (warp 8+i reaches 32*(i%4) .. +31).
        constexpr int GT = 256 / NGR;  // threads per group; each loop below runs NGR times
        const int gi = (tid - 256) / GT;
        const int u = (tid - 256) - gi * GT;
        const int lq = (tid - 256) & 127;
        constexpr int GW = GT >> 5;
        const int wq = u >> 5, g8 = lane >> 2, tg = lane & 3;
        const uint32_t trow = tmem + 128 * gi + ((uint32_t)(lq & ~31) << 16);
        const int gb = gi ? B_GRP1 : B_GO;
        uint8_t* pm = sm + (gi ? L::PM2 : L::PM);
        uint8_t* tts = sm + (gi ? L::TTS2 : L::TTS);
        float* sA = reinterpret_cast<float*>(sm + (gi ? L::AM2 : L::AM));
        float* sZ = reinterpret_cast<float*>(sm + (gi ? L::ZS2 : L::ZS));
        auto gsync = [&]() { group_sync(gi, GT); };
        // KDA (always one group) scan exchange: pg[128*q + ch] = summed log alpha over row
        // quarter q; exp(G - m) at pg[512 + ch], gamma_C = exp(G) at pg[640 + ch]
        float* pg = reinterpret_cast<float*>(sm + L::PG);
        // KDA: thread u owns key channels 2*(u%64), 2*(u%64)+1 on rows 16*(u/64) .. +15 of a
        // chunk; the next owned chunk's alpha values are prefetched into registers.
        const int kc = 2 * (u & 63), kq4 = u >> 6;
        constexpr bool kChan = kKda;  // per-key-channel values prefetched per chunk
        // Byte offsets of (row 16*kq4 + i, channels kc, kc+1) in the 128-byte-swizzled K/Q
        // stage (128 rows per panel) and K/gamma tile (64 rows per panel): the swizzle of row
        // i depends on i & 7 only, so row i's offset is a per-thread base plus the 16-byte
        // chunk position xsw(i & 7) plus a constant, and no swizzle arithmetic is left per
        // access in the loops below.
        const uint32_t kq_row0 = (uint32_t)(kc >> 6) * 128u * 128u + (uint32_t)(16 * kq4) * 128u +
                                 (uint32_t)(kc & 7) * 2u;
        const uint32_t kn_row0 = (uint32_t)(kc >> 6) * 64u * 128u + (uint32_t)(16 * kq4) * 128u +
                                 (uint32_t)(kc & 7) * 2u;
        const uint32_t kc_chunk = (uint32_t)((kc & 63) >> 3);
        auto xsw = [&](int i) -> uint32_t { return ((kc_chunk ^ (uint32_t)(i & 7)) << 4); };
        const float* chan = gate;
        float2 gpf[kChan ? 16 : 1];
        if constexpr (kChan) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = 16 * kq4 + i;
                gpf[i] = t < T ? *reinterpret_cast<const float2*>(chan + (bh * Ts + t) * (long)CDK + kc)
                               : make_float2(1.f, 1.f);
            }
        }
        int k = 0;  // the group's chunk ordinal
        for (int c = pbase + gi * pSP; c < nchunks; c += NGR * pSP, ++k) {
            const int mo = ordinal_of(c);  // position among the chunks this CTA loads
            const int s = mo % NS, p = mo % NP;
            const uint32_t jp = (uint32_t)(k & 1);
            const int t0 = c * CK;
            const int nvalid = min(CK, T - t0);
            uint8_t* kq = sm + L::KQ + s * L::KQ_B;
            const float* bg = reinterpret_cast<const float*>(sm + L::BG + s * L::BG_B);
            // NGR divides NS, so a group waits on every phase of the stages it reads, in order
            // (a parity wait cannot tell a completed phase from the one before it still pending)
            mbar_wait(bar(B_KQ_FULL + s), (uint32_t)((mo / NS) & 1), abort_flag);

            // ---- 1. gates. GDN: g, 1/gamma, gamma come from the producer; the factored form
            // gamma_t * (1/gamma_i) of exp(g_t - g_i) is used when it cannot overflow.
            bool fact = true;
            if constexpr (kGdn) {
                fact = bg[64 + 63] > -80.f;
            } else if constexpr (kKda) {
                // Per key channel c, G = summed log alpha over the chunk (four row quarters
                // joined through shared memory) and the anchor m = G/2. K and Q are rewritten
                // in place as K*exp(g - m), Q*exp(g - m) and K*exp(m - g) is stored, so every
                // factor of exp(g_t - g_i) = exp(g_t - m) * exp(m - g_i) stays within
                // exp(+-|G|/2): exact for G down to KDA_MIN_LOG_DECAY. The chain multiplies its
                // bf16 state copy by exp(m) per channel, which restores exp(g_t) in MMA1.
                uint8_t* kn = sm + L::KN;
                // summed log alpha of this thread's 16 rows: the log of their product, or,
                // where that product would underflow, the sum of the rows' logs
                // rows past the end of a ragged chunk count as alpha = 1 (so that every loop
                // below runs without a per-row test)
                if (nvalid < CK) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (16 * kq4 + i >= nvalid) gpf[i] = make_float2(1.f, 1.f);
                }
                if constexpr (SEG) {
                    // a gate above 1 could grow a state difference
                    bool up = false;
#pragma unroll
                    for (int i = 0; i < 16; ++i) up |= gpf[i].x > 1.f || gpf[i].y > 1.f;
                    if (up) atomicOr(seg.expand, 1);
                }
                float2 part = make_float2(1.f, 1.f);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    part.x *= gpf[i].x;
                    part.y *= gpf[i].y;
                }
                float2 lp = make_float2(__logf(part.x), __logf(part.y));
                if (part.x < 1e-30f || part.y < 1e-30f) {
                    lp = make_float2(0.f, 0.f);
                    for (int i = 0; i < 16; ++i) {
                        lp.x += __logf(gpf[i].x);
                        lp.y += __logf(gpf[i].y);
                    }
                }
                *reinterpret_cast<float2*>(pg + 128 * kq4 + kc) = lp;
                gsync();
                float2 G = make_float2(0.f, 0.f), Lb = make_float2(0.f, 0.f);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 pq = *reinterpret_cast<const float2*>(pg + 128 * q + kc);
                    if (q < kq4) {
                        Lb.x += pq.x;
                        Lb.y += pq.y;
                    }
                    G.x += pq.x;
                    G.y += pq.y;
                }
                const float2 m = make_float2(0.5f * G.x, 0.5f * G.y);
                if (kq4 == 0) {
                    if (G.x < KDA_MIN_LOG_DECAY || G.y < KDA_MIN_LOG_DECAY)
                        raise_status(DR_ERR_GATE_RANGE);
                    // exp(m) for the chain's copy of the entering state of this chunk
                    float* bgw = reinterpret_cast<float*>(sm + L::BG + s * L::BG_B);
                    *reinterpret_cast<float2*>(bgw + 128 + kc) = make_float2(__expf(m.x), __expf(m.y));
                }
                float2 run = make_float2(__expf(Lb.x - m.x), __expf(Lb.y - m.y));
                uint8_t* kr = kq + kq_row0;  // K row 16*kq4 (Q rows sit 64 rows further on)
                uint8_t* nr = kn + kn_row0;
#pragma unroll
                for (int i0 = 0; i0 < 16; i0 += 8) {
                    uint32_t kw[8], qw[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        kw[i] = *reinterpret_cast<const uint32_t*>(kr + xsw(i) + (i0 + i) * 128);
                        qw[i] = *reinterpret_cast<const uint32_t*>(kr + xsw(i) + (64 + i0 + i) * 128);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        run.x *= gpf[i0 + i].x;
                        run.y *= gpf[i0 + i].y;
                        const float2 k2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&kw[i]));
                        const float2 q2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&qw[i]));
                        const float ix = __fdividef(1.f, run.x), iy = __fdividef(1.f, run.y);
                        *reinterpret_cast<uint32_t*>(kr + xsw(i) + (i0 + i) * 128) =
                            pack_bf16(k2.x * run.x, k2.y * run.y);
                        *reinterpret_cast<uint32_t*>(kr + xsw(i) + (64 + i0 + i) * 128) =
                            pack_bf16(q2.x * run.x, q2.y * run.y);
                        *reinterpret_cast<uint32_t*>(nr + xsw(i) + (i0 + i) * 128) =
                            pack_bf16(k2.x * ix, k2.y * iy);
                    }
                }
                if (kq4 == 3) {
                    // exp(G - m) scales Khat^T's rows; gamma_C = exp(G) decays the state
                    *reinterpret_cast<float2*>(pg + 512 + kc) = run;
                    *reinterpret_cast<float2*>(pg + 640 + kc) = make_float2(__expf(G.x), __expf(G.y));
                }
                fence_async_smem();
                gsync();
            }
            tc_fence_before();
            mbar_arrive(bar(gb + 0));
            if constexpr (kChan) {
                // the next owned chunk's per-channel gates, issued after this stage's proxy
                // fence so that the fence does not wait for them; they land under the rest of
                // this chunk's prep
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int tn = (c + NGR * pSP) * CK + 16 * kq4 + i;
                    gpf[i] = tn < T ? *reinterpret_cast<const float2*>(chan + (bh * Ts + tn) * (long)CDK + kc)
                                    : make_float2(1.f, 1.f);
                }
            }

            // ---- 2. Gram epilogue: A (fp32, rows 0-63) and P (bf16, rows 0-63 of pm); a
            // thread takes one or both 32-column halves of TMEM row lq
            mbar_wait(bar(gb + 1), jp, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int i = 0; i < NGR; ++i) {
                const int hf = (u >> 7) + i;  // column half
                const int t = lq & 63;
                const int c32 = 32 * hf;
                float rowf = (lq < 64) ? bg[t] : 1.f;  // beta_t on A rows
                float gt = 0.f;
                if constexpr (kGdn) {
                    gt = bg[64 + t];
                    if (fact) rowf *= bg[192 + t];
                }
                float gr[32];
                tmem_ld16(trow + L::COL_G + c32, gr);
                tmem_ld16(trow + L::COL_G + c32 + 16, gr + 16);
                float dec[32];
                if constexpr (kGdn) {
                    if (fact) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 d4 = *reinterpret_cast<const float4*>(bg + 128 + c32 + e);
                            dec[e] = d4.x;
                            dec[e + 1] = d4.y;
                            dec[e + 2] = d4.z;
                            dec[e + 3] = d4.w;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            dec[e] = __expf(fminf(gt - bg[64 + c32 + e], 0.f));
                    }
                }
                tmem_wait_ld();
                if (SEG && lq < 64 && (t >> 5) == hf) {
                    // the step's transition diag(a)(I - beta k k^T) is non-expansive while
                    // beta |k|^2 <= 2 (|k|^2 is the Gram's diagonal)
                    float kk = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) kk = (c32 + e == t) ? gr[e] : kk;
                    if (bg[t] * kk > 2.f) atomicOr(seg.expand, 1);
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = c32 + e;
                    const bool keep = (lq < 64) ? (i < t) : (i <= t);
                    const float v = kGdn ? rowf * gr[e] * dec[e] : rowf * gr[e];
                    gr[e] = keep ? v : 0.f;
                }
                if (lq < 64) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(sA + t * 68 + c32 + e) =
                            make_float4(gr[e], gr[e + 1], gr[e + 2], gr[e + 3]);
                } else {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) st_row_chunk(pm, t, c32 / 8 + ch, gr + 8 * ch);
                }
            }
            gsync();

            // ---- 3. X = (I + A)^{-1}, in place in sA
            float xcol[16];
            if (u < 64) {  // diagonal 16x16 blocks, one column per thread
                const int b = u >> 4, cc = u & 15;
#pragma unroll
                for (int t = 0; t < 16; ++t) xcol[t] = (t == cc) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i)
#pragma unroll
                    for (int t = i + 1; t < 16; ++t)
                        xcol[t] = fmaf(-sA[(16 * b + t) * 68 + 16 * b + i], xcol[i], xcol[t]);
            }
            gsync();
            if (u < 64) {
                const int b = u >> 4, cc = u & 15;
#pragma unroll
                for (int t = 0; t < 16; ++t) sA[(16 * b + t) * 68 + 16 * b + cc] = xcol[t];
            }
            gsync();
            if (wq < 2) {  // X(b+1,b) = -X(b+1,b+1) A(b+1,b) X(b,b) for b = 0, 2
                const int b0 = 32 * wq, b1 = b0 + 16;
                float* z = sZ + wq * 16 * 20;
                float acc[2][4] = {};
#pragma unroll
                for (int kk = 0; kk < 16; kk += 8) {
                    uint32_t a[4], bb[2];
                    frag_a(a, sA, 68, b1, b0 + kk, g8, tg);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        frag_b(bb, sA, 68, b0 + kk, b0 + 8 * nt, g8, tg);
                        mma_tf32(acc[nt], a, bb);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) store_neg_frag(z, 20, 0, 8 * nt, acc[nt], g8, tg, 1.f);
                __syncwarp();
                float acc2[2][4] = {};
#pragma unroll
                for (int kk = 0; kk < 16; kk += 8) {
                    uint32_t a[4], bb[2];
                    frag_a(a, sA, 68, b1, b1 + kk, g8, tg);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        frag_b(bb, z, 20, kk, 8 * nt, g8, tg);
                        mma_tf32(acc2[nt], a, bb);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
                    store_neg_frag(sA, 68, b1, b0 + 8 * nt, acc2[nt], g8, tg, -1.f);
            }
            gsync();
            // X[32:64, 0:32] = -X[32:64, 32:64] A[32:64, 0:32] X[0:32, 0:32], in eight 16x8
            // tiles per product, spread over the group's warps
#pragma unroll
            for (int i = 0; i < NGR; ++i) {
                const int tile = wq + i * GW;
                const int m0 = 32 + 16 * (tile >> 2), n0 = 8 * (tile & 3);
                float acc[4] = {};
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    uint32_t a[4], bb[2];
                    frag_a(a, sA, 68, m0, kk, g8, tg);
                    frag_b(bb, sA, 68, kk, n0, g8, tg);
                    mma_tf32(acc, a, bb);
                }
                store_neg_frag(sZ, 36, m0 - 32, n0, acc, g8, tg, 1.f);
            }
            gsync();
#pragma unroll
            for (int i = 0; i < NGR; ++i) {
                const int tile = wq + i * GW;
                const int m0 = 32 + 16 * (tile >> 2), n0 = 8 * (tile & 3);
                float acc2[4] = {};
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    uint32_t a[4], bb[2];
                    frag_a(a, sA, 68, m0, 32 + kk, g8, tg);
                    frag_b(bb, sZ, 36, kk, n0, g8, tg);
                    mma_tf32(acc2, a, bb);
                }
                store_neg_frag(sA, 68, m0, n0, acc2, g8, tg, -1.f);
            }
            gsync();

            // ---- 4. stage T = X diag(beta) into the slot (and Ttilde for GDN's H): virtual
            // thread v writes half (v/64 % 2) of row v % 64 of T (v < 128) or of Ttilde
            if (mo >= NP) {
                // the previous use of slot p must be finished: by this CTA's chain, or (split)
                // by the distributor's copies to the chain CTAs
                mbar_wait(bar(B_SLOT_EMPTY + p), (uint32_t)(((mo / NP) - 1) & 1), abort_flag);
            }
            uint8_t* tp = slot(p) + L::SLOT_TP;
            float* gam = reinterpret_cast<float*>(slot(p) + L::SLOT_GAM);
#pragma unroll
            for (int i = 0; i < NGR; ++i) {
                const int v = u + i * GT;
                const int t = v & 63, half = (v >> 6) & 1;
                float scale = 1.f;
                uint8_t* dst = tp;
                if (v >= 128) {
                    if constexpr (kGdn) {
                        scale = __expf(bg[64 + 63] - bg[64 + t]);  // gamma_C / gamma_t
                        dst = tts;
                    } else {
                        dst = nullptr;
                    }
                }
                if (dst) {
                    float row[32];
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 x4 = *reinterpret_cast<const float4*>(sA + t * 68 + 32 * half + e);
                        const float4 b4 = *reinterpret_cast<const float4*>(bg + 32 * half + e);
                        row[e] = x4.x * b4.x * scale;
                        row[e + 1] = x4.y * b4.y * scale;
                        row[e + 2] = x4.z * b4.z * scale;
                        row[e + 3] = x4.w * b4.w * scale;
                    }
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) st_row_chunk(dst, t, 4 * half + ch, row + 8 * ch);
                }
                if constexpr (kGdn) {
                    if (v < 64) gam[v] = bg[192 + v];
                    if (v == 64) gam[64] = bg[192 + 63];
                } else if constexpr (kKda) {
                    if (v < 128) gam[v] = pg[640 + v];
                }
            }
            fence_async_smem();
            mbar_arrive(bar(gb + 2));

            // ---- 5. Khat^T -> slot (row lq); PT rows -> slot rows 64-127
            mbar_wait(bar(gb + 3), jp, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int i = 0; i < NGR; ++i) {
                const int hf = (u >> 7) + i;  // column half
                uint8_t* kh = slot(p) + L::SLOT_KH;
                const int c32 = 32 * hf;
                float h[32];
                tmem_ld16(trow + L::COL_H + c32, h);
                tmem_ld16(trow + L::COL_H + c32 + 16, h + 16);
                tmem_wait_ld();
                if constexpr (kKda) {
                    const float gC = pg[512 + lq];
#pragma unroll
                    for (int e = 0; e < 32; ++e) h[e] *= gC;
                }
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) st_row_chunk(kh, lq, c32 / 8 + ch, h + 8 * ch);
                // P T was an M=64 MMA: its row 16*q + l sits in lane l (< 16) of quadrant q
                tmem_ld16(trow + L::COL_G + c32, h);
                tmem_ld16(trow + L::COL_G + c32 + 16, h + 16);
                tmem_wait_ld();
                if ((lq & 31) < 16) {
                    const int t = 16 * (lq >> 5) + (lq & 15);
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) st_row_chunk(tp, 64 + t, c32 / 8 + ch, h + 8 * ch);
                }
            }
            fence_async_smem();
            tc_fence_before();
            gsync();
            if (u == 0) mbar_arrive(bar(B_PREP + p));
        }
    }

done:
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // give copies and MMAs issued before the abort a bounded chance to land
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 50000000ull) {
        }
    }
    __syncthreads();
    if constexpr (SPLIT) cluster_sync_all();  // no CTA leaves while the others may still address it
    tc_fence_after();
    if (warp == 3) tmem_dealloc(tmem, L::NCOLS);
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

// 3D map over BH sequences of T rows of `inner` elements, row-major, Ts rows from one
// sequence's start to the next (Ts = T: a [BH, T, inner] tensor); box {box_inner, 64 rows, 1}.
inline bool make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize,
                        long BH, int T, long Ts, int inner, int box_inner, bool swizzle128) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * Ts};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)CK, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Shapes and variants the chunked path takes (Gated DeltaNet-2 through its pre-scaled inputs).
inline bool chunked_supported(int variant, int dk, int dv) {
    return dk == CDK && (dv == 32 || dv == 64 || dv == 128) &&
           (variant == DR_DELTANET || variant == DR_GDN || variant == DR_KDA ||
            variant == DR_GDN2);
}

// Arguments of one chunked launch (device pointers as dr_scan_fwd_ex receives them; erase
// and write are read only by the Gated DeltaNet-2 pre-scaling).
struct ChunkArgs {
    const void *q, *k, *v;
    const float *beta, *gate, *erase, *write, *S0;
    void* out;
    float* S_final;
    void* u_out;
    int BH, T, dv;
};

// The last tensor map encoded for each (thread, slot): a scan called again on the same
// buffers and shape (the usual case in a loop) reuses it instead of encoding anew.
struct MapCacheEntry {
    const void* base = nullptr;
    long BH = 0, Ts = 0;
    int T = 0, inner = 0, box = 0;
    bool swz = false;
    int dev = -1;
    CUtensorMap map;
};

inline bool cached_map_3d(int slot, CUtensorMap* m, const void* base, long BH, int T, long Ts,
                          int inner, int box_inner, bool swizzle128) {
    thread_local MapCacheEntry cache[16];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    MapCacheEntry& e = cache[slot & 15];
    if (e.base == base && e.BH == BH && e.T == T && e.Ts == Ts && e.inner == inner &&
        e.box == box_inner && e.swz == swizzle128 && e.dev == dev) {
        *m = e.map;
        return true;
    }
    if (!make_map_3d(&e.map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, BH, T, Ts, inner,
                     box_inner, swizzle128)) {
        e.base = nullptr;
        return false;
    }
    e.base = base, e.BH = BH, e.T = T, e.Ts = Ts, e.inner = inner, e.box = box_inner;
    e.swz = swizzle128;
    e.dev = dev;
    *m = e.map;
    return true;
}

// A plain launch: sequences back to back, no checkpoint, no checks, unconditional.
inline ChunkSeg plain_seg(const ChunkArgs& a) {
    return ChunkSeg{(long)a.T, nullptr, 0, nullptr, nullptr, 0, 0};
}

// `maps` picks the set of cached tensor-map slots (0, 1, 2: the launches of one segmented
// scan keep their own maps).
template <int MODE, int BV, bool SPLIT, bool SEG = false>
int launch_chunked_bv(const ChunkArgs& a, int nprep, const ChunkSeg& sg, int maps,
                      cudaStream_t stream) {
    using L = ChunkLayout<MODE, BV, SPLIT>;
    CUtensorMap mk, mq, mv;
    const int m0 = 4 * maps;
    const int rows = a.T + (sg.G > 1 ? sg.ext : 0);  // tokens one sequence may read
    if (!cached_map_3d(m0, &mk, a.k, a.BH, rows, sg.Ts, CDK, 64, true) ||
        !cached_map_3d(m0 + 1, &mq, a.q, a.BH, rows, sg.Ts, CDK, 64, true) ||
        !cached_map_3d(m0 + 2, &mv, a.v, a.BH, rows, sg.Ts, a.dv, L::V_SWZ ? 64 : BV, L::V_SWZ))
        return DR_ERR_CUDA;
    const int smem = L::TOTAL + 1024;
    auto kern = dr_chunked_kernel<MODE, BV, SPLIT, SEG>;
    // the shared-memory opt-in is a per-device property of the function: set it once
    static bool attr_set[16] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DR_ERR_CUDA;
    if (dev < 0 || dev >= 16 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return DR_ERR_CUDA;
        if (dev >= 0 && dev < 16) attr_set[dev] = true;
    }
    const int split = SPLIT ? nprep : 0;  // prep CTAs per head
    const int ny = a.dv / BV + split;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.BH, (unsigned)ny);
    cfg.blockDim = dim3(CHUNK_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = split ? ny : 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = split ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, mk, mq, mv, a.beta, a.gate, a.S0,
                           static_cast<__nv_bfloat16*>(a.out), a.S_final,
                           static_cast<__nv_bfloat16*>(a.u_out), a.T, a.dv, split, sg) != cudaSuccess)
        return DR_ERR_CUDA;
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

// Clusters of `size` CTAs of the chunked kernel (one CTA per SM) that can be resident at
// once on the current device; cached per device.
inline int max_active_clusters(int size) {
    static int cache[16][9] = {};
    int dev = 0;
    if (size < 1 || size > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16)
        return 0;
    if (cache[dev][size] == 0) {
        using L = ChunkLayout<DR_GDN, 64, true>;
        auto kern = dr_chunked_kernel<DR_GDN, 64, true>;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1, (unsigned)size);
        cfg.blockDim = dim3(CHUNK_THREADS);
        cfg.dynamicSmemBytes = L::TOTAL + 1024;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = (unsigned)size;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 L::TOTAL + 1024) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
            n = -1;
        cache[dev][size] = n;
    }
    return cache[dev][size] > 0 ? cache[dev][size] : 0;
}

// Split mode (a cluster per head of `nprep` prep CTAs and dv/BV chain CTAs) for the
// scalar-gate variants when the heads are too few to fill the GPU otherwise. Measured on
// B200 (GDN, dk = dv = 128): two chain CTAs per head (BV = dv/2) beat four, whose extra slot
// copies cost more than their shorter chain saves; more prep CTAs help a little (16 heads,
// T = 32768: 2 / 3 / 4 prep CTAs 0.839 / 0.824 / 0.815 ms), so the plan takes as many as fit,
// up to four. Every cluster must be resident at once (clusters of 7-8 CTAs fit 15 at a time
// on B200, which would put 16 heads into two waves) and the grid must fit 148 SMs.
struct SplitPlan {
    int bv = 0, nprep = 0;  // nprep == 0: unsplit
};

inline SplitPlan pick_split(int variant, long BH, int dv) {
    SplitPlan plan;
    if (variant == DR_KDA || dv < 32) return plan;
    const int bv = dv / 2, ncc = 2;
    for (int np = 4; np >= 1; --np) {
        if (BH * (np + ncc) <= 148 && BH <= max_active_clusters(np + ncc)) {
            plan.bv = bv;
            plan.nprep = np;
            break;
        }
    }
    return plan;
}

// One launch with a given plan (nprep == 0: unsplit, value slice plan.bv, or pick_bv's when
// 0). SEG: the segment launch of the segmented scan (split Gated DeltaNet, unsplit KDA).
template <int MODE, bool SEG = false>
int launch_chunked_plan(const ChunkArgs& a, const SplitPlan& plan, const ChunkSeg& sg, int maps,
                        cudaStream_t stream) {
    static_assert(!SEG || MODE == DR_GDN || MODE == DR_KDA || MODE == DR_DELTANET,
                  "segments: DeltaNet, GDN and KDA");
    if constexpr (MODE != DR_KDA) {
        if (plan.nprep > 0) {
            switch (plan.bv) {
                case 16:
                    return launch_chunked_bv<MODE, 16, true, SEG>(a, plan.nprep, sg, maps, stream);
                case 32:
                    return launch_chunked_bv<MODE, 32, true, SEG>(a, plan.nprep, sg, maps, stream);
                case 64:
                    return launch_chunked_bv<MODE, 64, true, SEG>(a, plan.nprep, sg, maps, stream);
            }
            return DR_ERR_UNSUPPORTED;
        }
    }
    if constexpr (SEG && MODE != DR_KDA) {
        return DR_ERR_UNSUPPORTED;
    } else {
        switch (plan.bv ? plan.bv : pick_bv(MODE, a.BH, a.dv)) {
            case 16:
                if constexpr (!SEG) return launch_chunked_bv<MODE, 16, false>(a, 0, sg, maps, stream);
                break;
            case 32:
                return launch_chunked_bv<MODE, 32, false, SEG>(a, 0, sg, maps, stream);
            case 64:
                return launch_chunked_bv<MODE, 64, false, SEG>(a, 0, sg, maps, stream);
            case 128:
                if constexpr (MODE == DR_KDA)
                    return launch_chunked_bv<MODE, 128, false, SEG>(a, 0, sg, maps, stream);
        }
        return DR_ERR_UNSUPPORTED;
    }
}

template <int MODE>
int launch_chunked_mode(const ChunkArgs& a, cudaStream_t stream) {
    return launch_chunked_plan<MODE>(a, pick_split(MODE, a.BH, a.dv), plain_seg(a), 0, stream);
}

// ---------------------------------------------------------------------------------------
// Segmented scan (Gated DeltaNet, few heads, long sequences)
//
// With few heads the chained kernel leaves SMs idle and runs one chain of T/64 dependent
// chunks per head. The segmented form cuts each head into G equal segments and runs them in
// one launch as independent sequences:
//   1. segment g starts from a zero state (segment 0 from S0) and writes its outputs, except
//      for its first SEG_WINDOW chunks when g > 0; it records its state Z after those chunks.
//      Every segment but the last then runs SEG_WINDOW chunks on into the next segment,
//      carrying its state, and writes the outputs there: the next segment's window is thus
//      computed from the state that segment g reached, and X, the state at the end, is that
//      same point once more, reached through the segments before;
//   2. a check per boundary: the outputs of segment g after its window, computed from Z_g,
//      are kept only if every value row of X_{g-1} - Z_g is at most SEG_EPS times the
//      largest row norm of X_{g-1}. While every step's transition diag(a)(I - beta k k^T) is
//      non-expansive (gate <= 1 and beta |k|^2 <= 2, checked by the kernel on every token),
//      that difference never grows afterwards, so every later output and the end state move
//      by at most that much. By induction over the segments, X_{g-1} is itself the chained
//      state to within the same bound. SEG_EPS = 2^-7 sits above the kernel's own rounding:
//      its bf16 copy of the state rounds two nearly equal states apart by up to one bf16
//      step (2^-8 of an element), so two runs whose states agree to far below that still
//      differ by up to about 2^-8 of the row norm (measured on B200: 0.3e-3 to 2.1e-3 under
//      the Gated DeltaNet workload's gates; 2.8e-2 and more once the gate's log-mean is -6 or
//      weaker, too little decay);
//   3. when any check fails, a conditional launch of the chained kernel recomputes everything
//      (it returns at once when the checks passed): the result is always the chained one to
//      within SEG_EPS of the state's scale.
// A gate strictly below 1 makes the difference decay by gamma_C per chunk, so with the
// decays these models use the window's eight chunks shrink it far below the threshold (to
// about 4e-8 of the row norm in fp64 for gates exp(-softplus(x)), x ~ N(-4, 1)).
// ---------------------------------------------------------------------------------------
constexpr int SEG_WINDOW = 8;        // chunks of overlap between consecutive segments
constexpr int SEG_MIN_CHUNKS = 32;   // shortest segment (four windows)
// DeltaNet has no gate: a state difference shrinks only along the keys written, by about
// 0.85 per chunk for keys spread over all directions (fp64 on the workloads' inputs: 0.26,
// 7e-2, 1.7e-2, 4.7e-3 of the row norm after 8, 16, 24, 32 chunks), so its window is 48
// chunks (about 3e-4) and its segments at least twice that
constexpr int SEG_WINDOW_DN = 48;
constexpr int SEG_MIN_CHUNKS_DN = 96;
constexpr float SEG_EPS = 1.0f / 128.f;

struct SegPlan {
    int nseg = 1;               // segments per head (1: the chained kernel alone)
    int window = SEG_WINDOW;    // chunks of overlap
    SplitPlan split;            // plan of the segment launch (BH * nseg sequences)
};

// Segments pay where the chain is long: measured on B200 (Gated DeltaNet, dk = dv = 128), a
// chained chunk step takes about 3.1 K cycles and a step of the segment launch (two prep
// CTAs per cluster) about 3.65 K; the check and the conditional launch add about 8 us. In
// units of a chained step:
//   chained   nch
//   segmented 1.18 * (nch / G + SEG_WINDOW) + 5
// The plan takes the G with the lowest estimate among those that keep every segment at
// least SEG_MIN_CHUNKS long and let all B*H*G segments run at once as clusters of at least
// two prep and two chain CTAs, and segments only when that estimate is below 0.9 * nch.
//
// KDA runs unsplit, one CTA per (head, value slice), and its prep, about 13.9 K cycles per
// chunk on B200, sets the pace whatever the slice width: with few heads the chained plan
// splits the values into narrow slices whose CTAs each repeat the whole prep. The segment
// launch gives every sequence one CTA with all dv value channels instead, so in units of a
// chunk step (chained nch) the segmented scan takes nch / G + SEG_WINDOW + 2, for the G that
// keeps B*H*G CTAs within one per SM.
inline SegPlan pick_segments(int variant, long BH, int T, int dv) {
    SegPlan sp;
    if (variant == DR_KDA) {
        if (T % CK != 0) return sp;
        const int nch = T / CK;
        double best = 0.9 * nch;
        for (int G = 2; G <= nch / SEG_MIN_CHUNKS; ++G) {
            if (nch % G) continue;
            if (BH * G > 148) break;
            const double est = nch / G + SEG_WINDOW + 2.0;
            if (est < best) {
                best = est;
                sp.nseg = G;
                sp.split.bv = dv;
                sp.split.nprep = 0;
            }
        }
        return sp;
    }
    if ((variant != DR_GDN && variant != DR_DELTANET) || dv < 32 || T % CK != 0) return sp;
    const int nch = T / CK;
    const int window = variant == DR_DELTANET ? SEG_WINDOW_DN : SEG_WINDOW;
    const int min_chunks = variant == DR_DELTANET ? SEG_MIN_CHUNKS_DN : SEG_MIN_CHUNKS;
    double best = 0.9 * nch;
    for (int G = 2; G <= nch / min_chunks; ++G) {
        if (nch % G) continue;
        const long n = BH * G;
        if (n * 4 > 148 || n > max_active_clusters(4)) break;
        const SplitPlan p = pick_split(variant, n, dv);
        if (p.nprep < 2) continue;
        const double est = 1.18 * (nch / G + window) + 5.0;
        if (est < best) {
            best = est;
            sp.nseg = G;
            sp.window = window;
            sp.split = p;
        }
    }
    return sp;
}

// Step 2 of the segmented scan, one block per sequence s = head * G + segment. X and Z are
// [BH * G, dv, CDK] fp32: X[s] is where segment s's run ended (the state after the window of
// segment s + 1, or the head's final state for the last segment), Z[s] the zero-start state
// after segment s's own window. The last segment's X is the head's final state (a failed
// check's rerun overwrites it). Any failed check ORs 2 into *flag. A warp takes dv/16 value
// rows and issues all their loads before it reduces.
constexpr int SEG_CHECK_THREADS = 512;
__global__ void __launch_bounds__(SEG_CHECK_THREADS) seg_handoff_check_kernel(
    const float* __restrict__ X, const float* __restrict__ Z, float* __restrict__ S_final,
    int* __restrict__ flag, int G, int dv, float eps) {
    constexpr int NW = SEG_CHECK_THREADS / 32, RMAX = CDK / NW;  // rows per warp, dv <= 128
    const long s = blockIdx.x;
    const int g = (int)(s % G);
    const long head = s / G;
    const long n = (long)dv * CDK;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (s == 0 && tid == 0) atomicAdd(&g_seg_scans, 1ull);
    if (g == G - 1 && S_final) {
        const float4* src = reinterpret_cast<const float4*>(X + s * n);
        float4* dst = reinterpret_cast<float4*>(S_final + head * n);
        for (long e = tid; e < n / 4; e += SEG_CHECK_THREADS) dst[e] = src[e];
    }
    if (g == 0) return;
    const float* xs = X + (s - 1) * n;  // the true state after segment s's window
    const float* zs = Z + s * n;
    __shared__ float red[2][NW];
    float4 x[RMAX], z[RMAX];
#pragma unroll
    for (int i = 0; i < RMAX; ++i) {
        const int row = warp + NW * i;
        if (row < dv) {
            x[i] = reinterpret_cast<const float4*>(xs + (long)row * CDK)[lane];
            z[i] = reinterpret_cast<const float4*>(zs + (long)row * CDK)[lane];
        }
    }
    float dmax = 0.f, xmax = 0.f;
#pragma unroll
    for (int i = 0; i < RMAX; ++i) {
        if (warp + NW * i >= dv) break;
        float d2 = (x[i].x - z[i].x) * (x[i].x - z[i].x) + (x[i].y - z[i].y) * (x[i].y - z[i].y) +
                   (x[i].z - z[i].z) * (x[i].z - z[i].z) + (x[i].w - z[i].w) * (x[i].w - z[i].w);
        float x2 = x[i].x * x[i].x + x[i].y * x[i].y + x[i].z * x[i].z + x[i].w * x[i].w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            d2 += __shfl_xor_sync(0xffffffffu, d2, off);
            x2 += __shfl_xor_sync(0xffffffffu, x2, off);
        }
        // a NaN anywhere makes the comparison below fail
        dmax = (d2 > dmax || d2 != d2) ? d2 : dmax;
        xmax = fmaxf(xmax, x2);
    }
    if (lane == 0) {
        red[0][warp] = dmax;
        red[1][warp] = xmax;
    }
    __syncthreads();
    if (tid == 0) {
        float d = 0.f, xm = 0.f;
        for (int w = 0; w < NW; ++w) {
            d = (red[0][w] > d || red[0][w] != red[0][w]) ? red[0][w] : d;
            xm = fmaxf(xm, red[1][w]);
        }
        if (!(d <= eps * eps * xm)) atomicOr(flag, 2);
    }
}

inline int launch_chunked(const ChunkArgs& a, int variant, cudaStream_t stream) {
    switch (variant) {
        case DR_DELTANET:
            return launch_chunked_mode<DR_DELTANET>(a, stream);
        case DR_GDN:
            return launch_chunked_mode<DR_GDN>(a, stream);
        case DR_KDA:
            return launch_chunked_mode<DR_KDA>(a, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

}  // namespace drscan
