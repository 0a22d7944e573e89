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
    DR_KDA = 3       /* a_t = alpha_t[0..dk), one value per key channel */
};
#define DR_MODE_MASK 0xFF
/* q, k, v and out are bf16 (else fp32). beta, gate, S0 and S_final are always fp32. */
#define DR_IN_BF16 0x100
/* Use the per-token kernel (fp32 state, CUDA cores) even where the chunked tensor-core
 * kernel applies. Same results up to rounding; slower. For testing and as a baseline. */
#define DR_FORCE_SEQUENTIAL 0x200

/* status codes */
enum {
    DR_OK = 0,
    DR_ERR_INVALID_ARG = -1, /* null/misaligned pointer, negative size, bad flag */
    DR_ERR_UNSUPPORTED = -2, /* a valid request outside the compiled shapes */
    DR_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed (launch, attributes) */
    DR_ERR_TIMEOUT = -4,     /* device: a bounded wait on a barrier ran out; outputs invalid */
    DR_ERR_DEVICE_BOUNDS = -5 /* device: an index check failed; outputs invalid */
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
 *   mode     variant | DR_IN_BF16? | DR_FORCE_SEQUENTIAL?
 *
 * Supported: dk, dv in {32, 64, 128}; B, H >= 0 (B*H < 2^31); T >= 0 (T = 0 copies S0
 * into S_final). Every non-NULL pointer must be 16-byte aligned; when B*H*T == 0 the
 * per-token tensors (q, k, v, beta, gate, out) are not read and may be NULL. bf16 inputs with dk = 128 and
 * variant DeltaNet/GDN/KDA run the chunked kernel (chunks of 64 tokens, WY/UT form on
 * tcgen05 tensor cores, bf16 operands, fp32 state in tensor memory); everything else
 * runs the per-token kernel with an fp32 state. out may not alias an input.
 *
 * KDA on the chunked kernel factors exp(g_t - g_i) as exp(g_t) * exp(-g_i) inside a
 * chunk (g = running sum of log alpha): the summed log-decay of any key channel over
 * one 64-token chunk must stay above -80, else results are inexact (no error is raised).
 *
 * Returns DR_OK or a negative status; on error nothing is launched.
 */
int dr_scan_fwd(const void* q, const void* k, const void* v, const float* beta,
                const float* gate, const float* S0, void* out, float* S_final,
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
 * B*H*T == 0, q, k, v, u and out are not read and may be NULL.
 * Returns DR_OK or a negative status; on error nothing is launched.
 */
int vla_scan_fwd(const float* q, const float* k, const float* v, const float* u,
                 const float* S0, const float* A0, float lambda0,
                 float* out, float* S_final, float* A_final,
                 int B, int H, int T, int d, cudaStream_t stream);

/* Static, human-readable text for a status code (never NULL). */
const char* dr_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the status word that kernels on the
 * current device latch when a bounded wait runs out or an index check fails
 * (DR_OK, DR_ERR_TIMEOUT, DR_ERR_DEVICE_BOUNDS), or DR_ERR_CUDA if the synchronisation
 * itself failed. The word is a static device variable: the library allocates nothing.
 */
int dr_poll_error(cudaStream_t stream);

/*
 * The launch shape dr_scan_fwd picks for the chunked tensor-core kernel on the current
 * device, for `BH` = B*H sequences and the same `mode` word (variant | flags):
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
