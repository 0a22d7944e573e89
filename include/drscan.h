/*
 * drscan: forward recurrent-memory scan of delta-rule linear attention on B200 (sm_100a).
 *
 * C ABI. Every tensor argument is a DEVICE pointer owned by the caller, row-major and
 * contiguous; the library never allocates, frees or keeps a pointer past the call.
 * Calls are asynchronous on `stream`: the return value covers argument validation and
 * the kernel launch only. Conditions detected on the device (a bounded wait that ran
 * out) are latched in a per-device status word and read by dr_poll_error().
 *
 * Per head and per token the delta-rule family computes, with S in R^{dv x dk} mapping
 * keys to values ("Mechanisms, trade-offs and cross-layer routing of linear-attention
 * architectures", section "Technical details": memory W in R^{d_v x d_phi}, DeltaNet
 * prediction vbar = W_{t-1} kappa, residual r = v - vbar, write W <- W + beta r (x) kappa;
 * Gated DeltaNet W <- alpha W + beta r_alpha (x) kappa; Kimi Delta Attention decays each
 * key-feature channel):
 *
 *     S'  = S_{t-1} diag(a_t)              a_t = 1 (DeltaNet), alpha_t (GDN), alpha_t[:] (KDA)
 *     r_t = v_t - S' k_t                   residual against the decayed state
 *     S_t = S' + beta_t r_t k_t^T
 *     o_t = S_t q_t                        readout after the write
 *
 * and plain linear attention S_t = S_{t-1} + v_t k_t^T ("Variational Linear Attention
 * (VLA)", section 2.1). The kernels apply no feature map and no 1/sqrt(dk) scale: q and
 * k arrive as the caller prepared them (normally L2-normalised per token).
 *
 * Gated DeltaNet-2 (same page, sections "Methodology" and "Technical details": a
 * per-key-channel erase gate b and a per-value-channel write gate w, erase direction
 * e = b (.) kappa, write target z = w (.) v, residual r = z - W~ e) runs the recurrence
 * above with a_t = alpha_t (scalar) and k_t, v_t replaced by e_t, z_t: W~ = alpha_t S_{t-1}
 * is the decayed memory and the residual is written along e_t.
 *
 * The write value of a token is u_t = beta_t r_t, the vector the step adds to memory along
 * its key (S_t = S' + u_t k_t^T; u_t = v_t for plain linear attention). It is the internal
 * signal the page's cross-layer routing (CLER / CLVR) passages carry to later layers;
 * dr_scan_fwd_ex and dr_decode_step_ex can return it per token.
 */
#ifndef DRSCAN_H
#define DRSCAN_H

#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

/* variant, in the low byte of `mode` */
enum {
    DR_LINEAR = 0,   /* S_t = S_{t-1} + v_t k_t^T; beta and gate ignored (may be NULL) */
    DR_DELTANET = 1, /* a_t = 1 */
    DR_GDN = 2,      /* a_t = alpha_t, one scalar per (b,h,t) */
    DR_KDA = 3,      /* a_t = alpha_t[0..dk), one value per key channel */
    DR_GDN2 = 4      /* Gated DeltaNet-2: a_t = alpha_t, k -> b (.) k, v -> w (.) v; only
                        through dr_scan_fwd_ex / dr_decode_step_ex, which take b and w */
};
#define DR_MODE_MASK 0xFF
/* q, k, v and out are bf16 (else fp32). beta, gate, S0 and S_final are always fp32. */
#define DR_IN_BF16 0x100
/* Use the per-token kernel (fp32 state, CUDA cores) even where the chunked tensor-core
 * kernel applies. Same results up to rounding; slower. For testing and as a baseline. */
#define DR_FORCE_SEQUENTIAL 0x200
/* Keep DeltaNet, Gated DeltaNet and KDA on the chained chunked kernel (one pass, one dependent
 * chain of chunks per head) where dr_scan_fwd would take the segmented scan (see dr_scan_fwd). */
#define DR_CHAINED 0x400

/* status codes */
enum {
    DR_OK = 0,
    DR_ERR_INVALID_ARG = -1, /* null/misaligned pointer, negative size, bad flag */
    DR_ERR_UNSUPPORTED = -2, /* a valid request outside the compiled shapes */
    DR_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed (launch, attributes) */
    DR_ERR_TIMEOUT = -4,     /* device: a bounded wait on a barrier ran out; outputs invalid */
    DR_ERR_DEVICE_BOUNDS = -5, /* device: an index check failed; outputs invalid */
    DR_ERR_GATE_RANGE = -6,  /* device: a KDA gate decayed past the chunked kernel's range
                                (see dr_scan_fwd); outputs invalid */
    DR_ERR_NOT_SPD = -7,     /* device: the chunked VLA scan met a non-positive pivot in
                                I + U A U^T, i.e. A was not positive definite (an A0 that is
                                not an inverse penalty); outputs invalid */
    DR_ERR_SCRATCH_LIMIT = -8 /* vla_scan_fwd_noalloc: B*H*T*d is above
                                 VLA_NOALLOC_MAX_FLOATS, the size of its fixed scratch array */
};

/*
 * dr_scan_fwd -- delta-rule scan over B*H independent sequences of T tokens.
 *
 *   q, k     [B,H,T,dk]  bf16 if (mode & DR_IN_BF16) else fp32
 *   v        [B,H,T,dv]  same type as q
 *   beta     [B,H,T] fp32, the write strength in (0,1); NULL allowed only for DR_LINEAR
 *   gate     alpha values in (0,1], fp32 (not logs): NULL for DR_LINEAR / DR_DELTANET,
 *            [B,H,T] for DR_GDN, [B,H,T,dk] for DR_KDA
 *   S0       [B,H,dv,dk] fp32 initial state, or NULL for zeros
 *   out      [B,H,T,dv] same type as v (written)
 *   S_final  [B,H,dv,dk] fp32 final state, or NULL to skip (written)
 *   mode     variant | DR_IN_BF16? | DR_FORCE_SEQUENTIAL? | DR_CHAINED?
 *
 * Supported: dk, dv in {32, 64, 128}; B, H >= 0 (B*H < 2^31); T >= 0 (T = 0 copies S0
 * into S_final). Every non-NULL pointer must be 16-byte aligned; when B*H*T == 0 the
 * per-token tensors (q, k, v, beta, gate, out) are not read and may be NULL. bf16 inputs with dk = 128 and
 * variant DeltaNet/GDN/KDA run the chunked kernel (chunks of 64 tokens, WY/UT form on
 * tcgen05 tensor cores, bf16 operands, fp32 state in tensor memory); everything else
 * runs the per-token kernel with an fp32 state. out may not alias an input.
 *
 * KDA on the chunked kernel factors the in-chunk decay exp(g_t - g_i) (g = running sum
 * of log alpha per key channel) as exp(g_t - m) * exp(m - g_i) with the anchor m = G/2,
 * G the channel's summed log alpha over the 64-token chunk. This is exact for G >= -170
 * (alpha about 0.07 per token, every token, every channel); a chunk with any channel
 * below that latches DR_ERR_GATE_RANGE, which dr_poll_error() reports (the outputs of
 * that call are then invalid: rerun it with DR_FORCE_SEQUENTIAL, which has no such limit).
 *
 * Segmented scan (DeltaNet, Gated DeltaNet and KDA, bf16, dk = 128, T a multiple of 64, heads
 * too few to fill the GPU; see dr_chunked_plan_ex). A sequence's state carries over from chunk to chunk,
 * so the chained kernel runs T/64 dependent chunk steps per head ("Mechanisms, trade-offs and
 * cross-layer routing of linear-attention architectures", Technical details: the state is
 * decayed by alpha and corrected by the delta rule at every token). With few heads the call
 * instead cuts each head into G equal segments and runs them at once, in one launch: every
 * segment from a zero state (the first from S0); every segment but the last runs a window of
 * 8 chunks (48 for DeltaNet, which has no gate) on into the next one, carrying its state, and
 * writes the outputs there, while the next one writes none for those chunks. A check per
 * boundary then compares the carried state at the end of the window with the next segment's
 * zero-start state there: they must agree
 * within 2^-7 of the carried state's largest value-row norm (row-wise 2-norm). A step whose
 * transition diag(alpha)(I - beta k k^T) could grow a difference (any alpha > 1 or
 * beta |k|^2 > 2, both checked on every token) also fails the check. When every check
 * passes, the outputs and S_final stand: they differ from the chained scan's by at most that
 * bound (times |q|), the size of the kernel's own rounding: its bf16 copy of the state
 * already sets two runs from nearly equal states up to about 2^-8 of the row norm apart.
 * When any check fails, the chained kernel reruns the whole call on the device (no host
 * round trip), so the result is the chained one; a gate close to 1 everywhere makes the
 * check fail and the call then costs up to about twice the chained kernel. The segmented
 * scan takes 2 * B*H*G * dv*dk*4 bytes of scratch from the library's stream-ordered pool
 * (DR_ERR_CUDA if it cannot be had). DR_CHAINED turns it off; dr_segment_counters counts its
 * calls and reruns.
 *
 * Returns DR_OK or a negative status; on error nothing is launched.
 */
int dr_scan_fwd(const void* q, const void* k, const void* v, const float* beta,
                const float* gate, const float* S0, void* out, float* S_final,
                int B, int H, int T, int dk, int dv, int mode, cudaStream_t stream);

/*
 * dr_scan_fwd_ex -- dr_scan_fwd with Gated DeltaNet-2 and the per-token write values.
 * Same arguments, rules and return values as dr_scan_fwd, plus:
 *
 *   erase    [B,H,T,dk] fp32, the erase gate b of DR_GDN2 (NULL for every other variant)
 *   write    [B,H,T,dv] fp32, the write gate w of DR_GDN2 (NULL for every other variant)
 *   u_out    [B,H,T,dv] same type as v, or NULL: receives u_t = beta_t r_t for every token
 *            (v_t for DR_LINEAR). May not alias any other argument.
 *
 * DR_GDN2 takes gate [B,H,T] (alpha) like DR_GDN. With bf16 inputs and dk = 128 it runs
 * as two kernels on `stream`: the first writes e = b (.) k and z = w (.) v in bf16 (each
 * product in fp32, rounded to nearest even) into B*H*T*(dk+dv)*2 bytes of scratch taken
 * stream-ordered from a memory pool of the library's own (kept between calls, released in
 * stream order after the call's last kernel); the second is the chunked Gated DeltaNet
 * kernel, with its plan, on (q, e, z). DR_ERR_CUDA if the scratch cannot be had. Other
 * inputs of DR_GDN2 take the per-token kernel, which applies b and w itself.
 * Asking for u_out adds one [B,H,T,dv] store (and, in a split launch, 8 KB more of each
 * chunk's operands copied between the CTAs of a cluster).
 */
int dr_scan_fwd_ex(const void* q, const void* k, const void* v, const float* beta,
                   const float* gate, const float* erase, const float* write, const float* S0,
                   void* out, float* S_final, void* u_out,
                   int B, int H, int T, int dk, int dv, int mode, cudaStream_t stream);

/*
 * dr_decode_step -- one token of the same recurrence for B*H heads whose state S stays
 * resident (streaming inference): on entry S holds S_{t-1}, on return S_t, and out
 * receives o_t. Same definitions and readings as dr_scan_fwd with T = 1.
 *
 *   q, k     [B,H,dk]    bf16 if (mode & DR_IN_BF16) else fp32
 *   v        [B,H,dv]    same type as q
 *   beta     [B,H] fp32; NULL allowed only for DR_LINEAR
 *   gate     alpha values, fp32: NULL for DR_LINEAR / DR_DELTANET, [B,H] for DR_GDN,
 *            [B,H,dk] for DR_KDA
 *   S        [B,H,dv,dk] fp32, read and updated in place
 *   out      [B,H,dv] same type as v (written); may not alias any other argument
 *   mode     variant | DR_IN_BF16?
 *
 * Supported: dk, dv in {32, 64, 128}; B, H >= 0 (B*H = 0 launches nothing). Every pointer
 * must be 16-byte aligned and, when B*H > 0, non-NULL except as allowed above. The kernel
 * streams each head's state from HBM and back once (one warp per four rows of S, fp32
 * arithmetic on CUDA cores). Returns DR_OK or a negative status; on error nothing is
 * launched.
 */
int dr_decode_step(const void* q, const void* k, const void* v, const float* beta,
                   const float* gate, float* S, void* out, int B, int H, int dk, int dv, int mode,
                   cudaStream_t stream);

/*
 * dr_decode_step_ex -- dr_decode_step with Gated DeltaNet-2 and the write value:
 *   erase [B,H,dk] and write [B,H,dv] fp32, DR_GDN2's gates (NULL otherwise);
 *   u_out [B,H,dv] same type as v, or NULL: receives this token's u = beta r.
 * Same rules and return values as dr_decode_step.
 */
int dr_decode_step_ex(const void* q, const void* k, const void* v, const float* beta,
                      const float* gate, const float* erase, const float* write, float* S,
                      void* out, void* u_out, int B, int H, int dk, int dv, int mode,
                      cudaStream_t stream);

/*
 * vla_scan_fwd -- Variational Linear Attention scan ("Variational Linear Attention
 * (VLA)", sections 2.2-2.3): per head and token, with A the inverse penalty matrix,
 *
 *     z_t = A_{t-1} u_t
 *     A_t = A_{t-1} - z_t z_t^T / (1 + u_t^T z_t)        (Sherman-Morrison)
 *     alpha_hat_t = A_t k_t / ||A_t k_t||
 *     S_t = S_{t-1} + (v_t - S_{t-1} k_t) alpha_hat_t^T
 *     o_t = S_t q_t
 *
 *   q, k, v, u, out   [B,H,T,d] fp32 (k and q normally unit-norm per token)
 *   S0, A0            [B,H,d,d] fp32, or NULL for zeros / I / lambda0
 *   lambda0           > 0 when A0 is NULL (ignored otherwise)
 *   S_final, A_final  [B,H,d,d] fp32, or NULL to skip
 *
 * Supported: d in {32, 64, 96, 128}; T >= 0. Non-NULL pointers 16-byte aligned; when
 * B*H*T == 0, q, k, v, u and out are not read and may be NULL. A0, when given, must be
 * symmetric positive definite (it is the inverse of a penalty matrix).
 *
 * The scan runs chunked, 64 tokens at a time. An A-phase turns the chunk's Sherman-Morrison
 * steps into one Woodbury update (a 64 x 64 Cholesky factorisation of I + U A U^T) and
 * produces every alpha_hat_t; an S-phase applies the write and readout in the WY form of a
 * delta rule whose read key is k_t and write key alpha_hat_t, 32 rows of S per CTA. By
 * default both run at once in one kernel, a cluster of 1 + d/32 CTAs per head whose A-phase
 * CTA passes each chunk's W = L^-1 U A and K A through shared memory to the S-phase CTAs,
 * which form alpha_hat themselves (no scratch). Where A stops being positive definite the
 * device latches DR_ERR_NOT_SPD.
 * Returns DR_OK or a negative status; on error nothing is launched.
 */
int vla_scan_fwd(const float* q, const float* k, const float* v, const float* u,
                 const float* S0, const float* A0, float lambda0,
                 float* out, float* S_final, float* A_final,
                 int B, int H, int T, int d, cudaStream_t stream);

/* vla_scan_fwd_ex flag: the ratio readout (see below). */
#define VLA_RATIO_READOUT 0x1
/* vla_scan_fwd_ex flag: the per-token kernel (one CTA per head, the Sherman-Morrison steps
 * one token at a time) instead of the chunked scan. Same results up to rounding, no
 * scratch memory; slower. For testing and as a baseline. */
#define VLA_SEQUENTIAL 0x2
/* vla_scan_fwd_ex flag: the chunked scan as two kernels, the A-phase for every head first,
 * then the S-phase, with alpha_hat in B*H*T*d*4 bytes of scratch taken stream-ordered from a
 * memory pool of the library's own (kept between calls) and released in stream order after
 * the second kernel. Same results as the fused kernel; slower (the phases do not overlap).
 * The fused kernel also falls back to this pair where its cluster does not fit. */
#define VLA_TWO_KERNEL 0x4

/*
 * vla_scan_fwd_ex -- vla_scan_fwd with the ratio readout of "Variational Linear Attention
 * (VLA)", section 2.3 (the output is a ratio of recurrences, as in standard linear
 * attention, with an ELU+1 feature map). With flags = VLA_RATIO_READOUT the scan also keeps
 * the denominator state n (a row of d values: the same write applied to one more value
 * channel held at 1),
 *
 *     n_t = n_{t-1} + (1 - n_{t-1} k_t) alpha_hat_t^T,     o_t = S_t q_t / (n_t q_t),
 *
 * and S, A follow vla_scan_fwd exactly. The feature map is the caller's: q holds phi(q)
 * (ELU+1 of the raw query) and k the unit-norm phi(k) / ||phi(k)||.
 *
 *   n0       [B,H,d] fp32 initial denominator state, or NULL for zeros (ratio readout only)
 *   n_final  [B,H,d] fp32 final denominator state, or NULL to skip (ratio readout only)
 *   flags    0 (o_t = S_t q_t, exactly vla_scan_fwd) or VLA_RATIO_READOUT, optionally
 *            with one of VLA_SEQUENTIAL and VLA_TWO_KERNEL
 *
 * Other arguments, rules and return values as vla_scan_fwd; n0 / n_final with flags = 0
 * return DR_ERR_INVALID_ARG. The denominator is not guarded: where n_t q_t is zero the output
 * is not finite.
 */
int vla_scan_fwd_ex(const float* q, const float* k, const float* v, const float* u,
                    const float* S0, const float* A0, const float* n0, float lambda0,
                    float* out, float* S_final, float* A_final, float* n_final,
                    int B, int H, int T, int d, int flags, cudaStream_t stream);

/* Largest B*H*T*d that vla_scan_fwd_noalloc accepts: its scratch array holds this many
 * floats (64 MiB). */
#define VLA_NOALLOC_MAX_FLOATS 16777216

/*
 * vla_scan_fwd_noalloc -- vla_scan_fwd_ex with VLA_TWO_KERNEL, without any memory allocation.
 * The pages have no counterpart: this entry point exists for callers that must not allocate
 * device memory, such as a serving engine that reserves all device memory up front for its
 * own allocator and forbids later allocations, or code that runs where a driver allocation
 * may block or synchronise (a latency-bound step, an allocator's own callback). The
 * two-kernel form of the chunked VLA scan needs B*H*T*d floats of scratch for the write
 * directions between its kernels; vla_scan_fwd_ex takes them from a memory pool, this entry
 * point from a fixed array compiled into the library, which every GPU that loads the library
 * holds (VLA_NOALLOC_MAX_FLOATS floats, 64 MiB) until the process exits. (The default fused
 * form of vla_scan_fwd_ex needs no scratch either, where its cluster fits on the device.)
 *
 * Arguments, layout and results are those of vla_scan_fwd_ex; flags is 0 or
 * VLA_RATIO_READOUT (other flags return DR_ERR_INVALID_ARG: the two-kernel pair is always
 * the one that runs). B*H*T*d above VLA_NOALLOC_MAX_FLOATS returns DR_ERR_SCRATCH_LIMIT before
 * anything is launched. The call makes no cudaMalloc, cudaFree or pool allocation.
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * once per device, with that device current); make that first call before any stream
 * capture. Every call on a device shares the one array, and the array keeps the last call's
 * contents (every element a call reads is written by that call first). Calls that overlap on
 * the GPU (different streams, or different host threads) race on the array: serialise them.
 * Returns DR_OK or a negative status; on error nothing is launched.
 */
int vla_scan_fwd_noalloc(const float* q, const float* k, const float* v, const float* u,
                         const float* S0, const float* A0, const float* n0, float lambda0,
                         float* out, float* S_final, float* A_final, float* n_final,
                         int B, int H, int T, int d, int flags, cudaStream_t stream);

/*
 * loglinear_scan_fwd -- log-linear attention over a Fenwick hierarchy of linear-attention
 * memories ("Adaptive memory decay for log-linear attention", problem definition and method
 * sections: the memory is a Fenwick-tree hierarchy whose state grows as O(log T), and every
 * output is a weighted sum of memory levels with weights lambda_t^(l)). At step t the
 * prefix [0, t] splits into level 0 = {t} and, per set bit b of t, level b + 1 = a block of
 * 2^b earlier tokens (the Fenwick split of the prefix); with M_l the sum of v_s k_s^T over
 * level l's tokens,
 *
 *     o_t = sum_l lambda_t^(l) M_l q_t.
 *
 *   q, k     [B,H,T,dk] bf16 (mode = DR_IN_BF16)
 *   v, out   [B,H,T,dv] bf16
 *   lambda   [B,H,T,L] fp32 level weights (produced by the caller, e.g. the page's
 *            softplus MLP); L >= 1 + bit length of T - 1, L <= 16
 *
 * Supported: dk = 128, dv in {32, 64, 128}, T <= 32768. Starts from empty memories (no
 * state in or out). Every non-NULL pointer 16-byte aligned; with B*H*T == 0 nothing is read.
 * Returns DR_OK or a negative status; on error nothing is launched.
 */
int loglinear_scan_fwd(const void* q, const void* k, const void* v, const float* lambda,
                       void* out, int B, int H, int T, int dk, int dv, int L, int mode,
                       cudaStream_t stream);

/* Static, human-readable text for a status code (never NULL). */
const char* dr_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the status word that kernels on the
 * current device latch when a bounded wait runs out, an index check fails or a gate is out
 * of the chunked kernel's range (DR_OK, DR_ERR_TIMEOUT, DR_ERR_DEVICE_BOUNDS,
 * DR_ERR_GATE_RANGE), or DR_ERR_CUDA if the synchronisation
 * itself failed. The word is a static device variable: the library allocates nothing.
 */
int dr_poll_error(cudaStream_t stream);

/*
 * The launch shape dr_scan_fwd picks for the chunked tensor-core kernel on the current
 * device, for `BH` = B*H sequences and the same `mode` word (variant | flags; DR_GDN2 gets
 * DR_GDN's plan, the kernel its chunked path runs on the pre-scaled inputs):
 *   *bv    value channels per chain CTA;
 *   *nprep prep CTAs per head in a split cluster (a cluster of *nprep prep CTAs and dv/(*bv)
 *          chain CTAs per head, used when the heads are too few to fill the GPU), or 0 when
 *          one CTA per (head, value slice) does both sides.
 * Returns DR_OK; DR_ERR_UNSUPPORTED (both set to 0) when the request would run the
 * per-token kernel instead (fp32 inputs, DR_FORCE_SEQUENTIAL, dk != 128, dv not in
 * {32, 64, 128}, or plain linear attention); DR_ERR_INVALID_ARG for null pointers, BH < 1
 * or unknown mode bits. Launches nothing; queries the device's cluster occupancy once.
 */
int dr_chunked_plan(int mode, long long BH, int dk, int dv, int* bv, int* nprep);

/*
 * dr_chunked_plan with the sequence length: also reports, in *nseg, how many segments per
 * head the segmented scan of dr_scan_fwd cuts each sequence into (1: the chained kernel
 * alone; then *bv and *nprep are dr_chunked_plan's). With *nseg > 1, *bv and *nprep are
 * the plan of the segment launches, which run B*H*(*nseg) sequences of T/(*nseg) tokens.
 * Same return values as dr_chunked_plan; T < 0 is DR_ERR_INVALID_ARG.
 */
int dr_chunked_plan_ex(int mode, long long BH, int T, int dk, int dv, int* bv, int* nprep,
                       int* nseg);

/*
 * How often the segmented scan ran on the current device since the library was loaded
 * (*scans) and how many of those calls failed a hand-off check and were recomputed by the
 * chained kernel (*reruns). Waits for the device to finish its work first. Returns DR_OK,
 * DR_ERR_INVALID_ARG for null pointers, DR_ERR_CUDA if the device cannot be read.
 */
int dr_segment_counters(unsigned long long* scans, unsigned long long* reruns);

/*
 * Test hook for the failure path: launches a one-block kernel on `stream` that waits on
 * a shared-memory barrier nothing ever arrives on, with a spin limit of `spin_limit`
 * polls, then latches DR_ERR_TIMEOUT and returns. Nothing faults or hangs.
 * Returns DR_OK if the launch succeeded.
 */
int dr_debug_timeout_probe(int spin_limit, cudaStream_t stream);

/* Library version as 10000*major + 100*minor + patch. */
int dr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DRSCAN_H */
