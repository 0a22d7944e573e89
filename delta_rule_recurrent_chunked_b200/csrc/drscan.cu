// C-ABI entry points of libdrscan: argument validation, kernel selection and launch.
// The declarations, with the meaning and layout of every argument, are in drscan.h.
// All kernels live in this one translation unit so that they share the device status
// word without relocatable device code.
#include <climits>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "dr_chunked.cuh"
#include "dr_decode.cuh"
#include "dr_sequential.cuh"
#include "loglinear.cuh"
#include "vla_chunked.cuh"
#include "vla_sequential.cuh"

using namespace drscan;

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }
bool dim_supported(int d) { return d == 32 || d == 64 || d == 128; }

int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

// Arguments of a decode step (device pointers as dr_decode_step_ex receives them).
struct DecodeArgs {
    const void *q, *k, *v;
    const float *beta, *gate, *erase, *write;
    float* S;
    void *out, *u_out;
    long rows;
    int dv;
};

template <typename TIn, int MODE, int DK>
int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    constexpr long per_cta = (long)DEC_ROWS * DEC_WARPS;
    dr_decode_kernel<TIn, MODE, DK><<<(unsigned)((a.rows + per_cta - 1) / per_cta), DEC_THREADS,
                                       0, stream>>>(
        static_cast<const TIn*>(a.q), static_cast<const TIn*>(a.k), static_cast<const TIn*>(a.v),
        a.beta, a.gate, a.erase, a.write, a.S, a.S, static_cast<TIn*>(a.out),
        static_cast<TIn*>(a.u_out), a.rows, a.dv);
    return launch_status();
}

template <typename TIn, int MODE>
int dispatch_decode_dk(const DecodeArgs& a, int dk, cudaStream_t stream) {
    switch (dk) {
        case 32:
            return launch_decode<TIn, MODE, 32>(a, stream);
        case 64:
            return launch_decode<TIn, MODE, 64>(a, stream);
        case 128:
            return launch_decode<TIn, MODE, 128>(a, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

template <typename TIn>
int dispatch_decode(const DecodeArgs& a, int dk, int variant, cudaStream_t stream) {
    switch (variant) {
        case DR_LINEAR:
            return dispatch_decode_dk<TIn, DR_LINEAR>(a, dk, stream);
        case DR_DELTANET:
            return dispatch_decode_dk<TIn, DR_DELTANET>(a, dk, stream);
        case DR_GDN:
            return dispatch_decode_dk<TIn, DR_GDN>(a, dk, stream);
        case DR_KDA:
            return dispatch_decode_dk<TIn, DR_KDA>(a, dk, stream);
        case DR_GDN2:
            return dispatch_decode_dk<TIn, DR_GDN2>(a, dk, stream);
    }
    return DR_ERR_INVALID_ARG;
}

template <typename TIn, int MODE, int DK>
int launch_sequential(const ChunkArgs& a, cudaStream_t stream) {
    dim3 grid((unsigned)a.BH, (unsigned)(a.dv / 32));
    dr_sequential_kernel<TIn, MODE, DK><<<grid, 32, 0, stream>>>(
        static_cast<const TIn*>(a.q), static_cast<const TIn*>(a.k), static_cast<const TIn*>(a.v),
        a.beta, a.gate, a.erase, a.write, a.S0, static_cast<TIn*>(a.out), a.S_final,
        static_cast<TIn*>(a.u_out), a.T, a.dv);
    return launch_status();
}

template <typename TIn, int MODE>
int dispatch_sequential_dk(const ChunkArgs& a, int dk, cudaStream_t stream) {
    switch (dk) {
        case 32:
            return launch_sequential<TIn, MODE, 32>(a, stream);
        case 64:
            return launch_sequential<TIn, MODE, 64>(a, stream);
        case 128:
            return launch_sequential<TIn, MODE, 128>(a, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

template <typename TIn>
int dispatch_sequential(const ChunkArgs& a, int dk, int variant, cudaStream_t stream) {
    switch (variant) {
        case DR_LINEAR:
            return dispatch_sequential_dk<TIn, DR_LINEAR>(a, dk, stream);
        case DR_DELTANET:
            return dispatch_sequential_dk<TIn, DR_DELTANET>(a, dk, stream);
        case DR_GDN:
            return dispatch_sequential_dk<TIn, DR_GDN>(a, dk, stream);
        case DR_KDA:
            return dispatch_sequential_dk<TIn, DR_KDA>(a, dk, stream);
        case DR_GDN2:
            return dispatch_sequential_dk<TIn, DR_GDN2>(a, dk, stream);
    }
    return DR_ERR_INVALID_ARG;
}

// State handed through unchanged when there are no tokens: S_final = S0 (or zeros).
int copy_state(float* dst, const float* src, size_t count, cudaStream_t stream) {
    if (!dst) return DR_OK;
    cudaError_t e = src ? cudaMemcpyAsync(dst, src, count * sizeof(float),
                                          cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(dst, 0, count * sizeof(float), stream);
    return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

// Gated DeltaNet-2's erase directions e = b (.) k and write targets z = w (.) v in bf16 (each
// product in fp32, rounded to nearest even), for the chunked path, which then runs Gated
// DeltaNet on (q, e, z). A thread per 8 consecutive elements: the k part, then the v part.
__global__ void gdn2_prescale_kernel(const __nv_bfloat16* __restrict__ k,
                                     const float* __restrict__ b,
                                     const __nv_bfloat16* __restrict__ v,
                                     const float* __restrict__ w, __nv_bfloat16* __restrict__ e,
                                     __nv_bfloat16* __restrict__ z, long nk8, long nv8) {
    const long u = blockIdx.x * (long)blockDim.x + threadIdx.x;
    if (u >= nk8 + nv8) return;
    const bool kpart = u < nk8;
    const long o = 8 * (kpart ? u : u - nk8);
    const __nv_bfloat16* x = kpart ? k : v;
    const float* g = kpart ? b : w;
    const uint4 xr = *reinterpret_cast<const uint4*>(x + o);
    const float4 g0 = *reinterpret_cast<const float4*>(g + o);
    const float4 g1 = *reinterpret_cast<const float4*>(g + o + 4);
    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xr);
    const float2 a0 = __bfloat1622float2(xp[0]), a1 = __bfloat1622float2(xp[1]);
    const float2 a2 = __bfloat1622float2(xp[2]), a3 = __bfloat1622float2(xp[3]);
    uint4 y;
    y.x = pack_bf16(a0.x * g0.x, a0.y * g0.y);
    y.y = pack_bf16(a1.x * g0.z, a1.y * g0.w);
    y.z = pack_bf16(a2.x * g1.x, a2.y * g1.y);
    y.w = pack_bf16(a3.x * g1.z, a3.y * g1.w);
    *reinterpret_cast<uint4*>((kpart ? e : z) + o) = y;
}

__global__ void scaled_identity_kernel(float* A, int d, long count, float diag) {
    long e = blockIdx.x * (long)blockDim.x + threadIdx.x;
    if (e < count) {
        const long rc = e % ((long)d * d);
        A[e] = (rc / d == rc % d) ? diag : 0.f;
    }
}

template <int D, bool RATIO>
int launch_vla(const float* q, const float* k, const float* v, const float* u, const float* S0,
               const float* A0, const float* n0, float lambda0, float* out, float* S_final,
               float* A_final, float* n_final, long BH, int T, cudaStream_t stream) {
    const int smem = (int)sizeof(VlaSmem<D>);
    auto kern = vla_sequential_kernel<D, RATIO>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return DR_ERR_CUDA;
    kern<<<(unsigned)BH, 2 * D, smem, stream>>>(q, k, v, u, S0, A0, n0, lambda0, out, S_final,
                                                A_final, n_final, T);
    return launch_status();
}

// Stream-ordered scratch from a memory pool of this library's own, one per device, that
// keeps its memory between calls (release threshold at the maximum), so that a call after
// the first one does not go to the driver for memory.
int scratch_alloc(void** p, size_t bytes, cudaStream_t stream) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static cudaMemPool_t pools[kMaxDev] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return DR_ERR_CUDA;
    cudaMemPool_t pool;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!pools[dev]) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.handleTypes = cudaMemHandleTypeNone;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t created;
            if (cudaMemPoolCreate(&created, &props) != cudaSuccess) return DR_ERR_CUDA;
            uint64_t keep = UINT64_MAX;
            cudaMemPoolSetAttribute(created, cudaMemPoolAttrReleaseThreshold, &keep);
            pools[dev] = created;
        }
        pool = pools[dev];
    }
    return cudaMallocFromPoolAsync(p, bytes, pool, stream) == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

// The segmented scan (steps in dr_chunked.cuh) of Gated DeltaNet or KDA: scratch for two sets
// of per-segment states and the check word, stream-ordered from the library's pool.
template <int MODE>
int launch_segmented(const ChunkArgs& a, const SegPlan& sp, cudaStream_t stream) {
    const int G = sp.nseg;
    const long nseq = (long)a.BH * G;
    const size_t sn = (size_t)a.dv * CDK;  // floats per state
    void* scratch = nullptr;
    int rc = scratch_alloc(&scratch, 2 * nseq * sn * sizeof(float) + 256, stream);
    if (rc != DR_OK) return rc;
    float* X = static_cast<float*>(scratch);  // end state of each segment's run
    float* Z = X + nseq * sn;                 // zero-start state after the window
    int* flag = reinterpret_cast<int*>(Z + nseq * sn);
    rc = cudaMemsetAsync(flag, 0, sizeof(int), stream) == cudaSuccess ? DR_OK : DR_ERR_CUDA;
    // 1. all segments at once, each but the last running on through the next one's window
    ChunkArgs p = a;
    p.BH = (int)nseq;
    p.T = a.T / G;
    p.S_final = X;
    if (rc == DR_OK)
        rc = launch_chunked_plan<MODE, true>(
            p, sp.split, ChunkSeg{(long)p.T, Z, sp.window, flag, nullptr, G, sp.window * CK}, 1,
            stream);
    // 2. the hand-off checks (and the final states)
    if (rc == DR_OK) {
        seg_handoff_check_kernel<<<(unsigned)nseq, SEG_CHECK_THREADS, 0, stream>>>(
            X, Z, a.S_final, flag, G, a.dv, SEG_EPS);
        rc = launch_status();
    }
    // 3. the chained scan, run only if a check failed
    if (rc == DR_OK)
        rc = launch_chunked_plan<MODE>(a, pick_split(MODE, a.BH, a.dv),
                                       ChunkSeg{(long)a.T, nullptr, 0, nullptr, flag, 0, 0}, 2,
                                       stream);
    if (cudaFreeAsync(scratch, stream) != cudaSuccess && rc == DR_OK) rc = DR_ERR_CUDA;
    return rc;
}

// The chunked path: the segmented scan where its plan applies (few heads, long sequences; not
// with DR_CHAINED), else one launch of the chained kernel.
int launch_chunked_auto(const ChunkArgs& a, int variant, bool chained, cudaStream_t stream) {
    if (!chained) {
        const SegPlan sp = pick_segments(variant, a.BH, a.T, a.dv);
        if (sp.nseg > 1) {
            switch (variant) {
                case DR_DELTANET:
                    return launch_segmented<DR_DELTANET>(a, sp, stream);
                case DR_GDN:
                    return launch_segmented<DR_GDN>(a, sp, stream);
                case DR_KDA:
                    return launch_segmented<DR_KDA>(a, sp, stream);
            }
        }
    }
    return launch_chunked(a, variant, stream);
}

// Gated DeltaNet-2 on the chunked path: e and z into stream-ordered scratch, then the Gated
// DeltaNet kernel (and its plan) on (q, e, z).
int launch_gdn2_chunked(ChunkArgs a, int dk, bool chained, cudaStream_t stream) {
    const long nk = (long)a.BH * a.T * dk, nv = (long)a.BH * a.T * a.dv;
    void* scratch = nullptr;
    int rc = scratch_alloc(&scratch, (size_t)(nk + nv) * sizeof(__nv_bfloat16), stream);
    if (rc != DR_OK) return rc;
    __nv_bfloat16* e = static_cast<__nv_bfloat16*>(scratch);
    __nv_bfloat16* z = e + nk;
    const long units = (nk + nv) / 8;
    gdn2_prescale_kernel<<<(unsigned)((units + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.k), a.erase, static_cast<const __nv_bfloat16*>(a.v),
        a.write, e, z, nk / 8, nv / 8);
    rc = launch_status();
    if (rc == DR_OK) {
        a.k = e;
        a.v = z;
        a.erase = a.write = nullptr;
        rc = launch_chunked_auto(a, DR_GDN, chained, stream);
    }
    if (cudaFreeAsync(scratch, stream) != cudaSuccess && rc == DR_OK) rc = DR_ERR_CUDA;
    return rc;
}

// The chunked pair: the A-phase writes alpha_hat into scratch, the S-phase reads it.
template <int D, bool RATIO>
int launch_vla_chunked(const float* q, const float* k, const float* v, const float* u,
                       const float* S0, const float* A0, const float* n0, float lambda0,
                       float* out, float* S_final, float* A_final, float* n_final, long BH,
                       int T, cudaStream_t stream) {
    const int smem_a = (int)sizeof(VcASmem<D>);
    const int smem_s = (int)sizeof(VcSSmem<D>);
    auto ka = vla_aphase_kernel<D>;
    auto ks = vla_sphase_kernel<D, RATIO>;
    if (cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_a) !=
            cudaSuccess ||
        cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_s) !=
            cudaSuccess)
        return DR_ERR_CUDA;
    void* scratch = nullptr;
    int rc = scratch_alloc(&scratch, (size_t)BH * T * D * sizeof(float), stream);
    if (rc != DR_OK) return rc;
    float* alpha = static_cast<float*>(scratch);
    ka<<<(unsigned)BH, VC_THREADS, smem_a, stream>>>(k, u, A0, lambda0, A_final, alpha, T);
    rc = launch_status();
    if (rc == DR_OK) {
        ks<<<dim3((unsigned)BH, D / VC_RS), VC_THREADS, smem_s, stream>>>(
            q, k, v, alpha, S0, n0, out, S_final, n_final, T);
        rc = launch_status();
    }
    if (cudaFreeAsync(scratch, stream) != cudaSuccess && rc == DR_OK) rc = DR_ERR_CUDA;
    return rc;
}

// The fused kernel: one cluster of 1 + D/32 CTAs per head, both phases at once, no scratch.
// Returns DR_ERR_UNSUPPORTED (nothing launched) when no such cluster fits on the device.
template <int D, bool RATIO>
int launch_vla_fused(const float* q, const float* k, const float* v, const float* u,
                     const float* S0, const float* A0, const float* n0, float lambda0,
                     float* out, float* S_final, float* A_final, float* n_final, long BH, int T,
                     cudaStream_t stream) {
    constexpr int CS = 1 + D / VC_RS;
    const int smem = vc_fused_smem_bytes<D>();
    auto kern = vla_fused_kernel<D, RATIO>;
    if (BH * CS > INT_MAX) return DR_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return DR_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(BH * CS));
    cfg.blockDim = dim3(VC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) return DR_ERR_CUDA;
    if (clusters < 1) return DR_ERR_UNSUPPORTED;
    if (cudaLaunchKernelEx(&cfg, kern, q, k, v, u, S0, A0, n0, lambda0, out, S_final, A_final,
                           n_final, T) != cudaSuccess)
        return DR_ERR_CUDA;
    return launch_status();
}

template <int D>
int launch_vla_readout(bool ratio, bool sequential, bool two_kernel, const float* q,
                       const float* k, const float* v, const float* u, const float* S0,
                       const float* A0, const float* n0, float lambda0, float* out,
                       float* S_final, float* A_final, float* n_final, long BH, int T,
                       cudaStream_t stream) {
    if (!sequential && !two_kernel) {
        const int rc = ratio ? launch_vla_fused<D, true>(q, k, v, u, S0, A0, n0, lambda0, out,
                                                         S_final, A_final, n_final, BH, T, stream)
                             : launch_vla_fused<D, false>(q, k, v, u, S0, A0, nullptr, lambda0,
                                                          out, S_final, A_final, nullptr, BH, T,
                                                          stream);
        if (rc != DR_ERR_UNSUPPORTED) return rc;  // else: the two-kernel pair below
    }
    if (sequential) {
        if (ratio)
            return launch_vla<D, true>(q, k, v, u, S0, A0, n0, lambda0, out, S_final, A_final,
                                       n_final, BH, T, stream);
        return launch_vla<D, false>(q, k, v, u, S0, A0, nullptr, lambda0, out, S_final,
                                    A_final, nullptr, BH, T, stream);
    }
    if (ratio)
        return launch_vla_chunked<D, true>(q, k, v, u, S0, A0, n0, lambda0, out, S_final,
                                           A_final, n_final, BH, T, stream);
    return launch_vla_chunked<D, false>(q, k, v, u, S0, A0, nullptr, lambda0, out, S_final,
                                        A_final, nullptr, BH, T, stream);
}

__global__ void timeout_probe_kernel(int spin_limit) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool done = false;
        for (int i = 0; i < spin_limit && !done; ++i) done = mbar_test(b, 0);
        if (!done) raise_status(DR_ERR_TIMEOUT);
    }
}

// ---- scratch of the no-allocation VLA entry point

// Write directions of vla_scan_fwd_noalloc: a fixed array instead of pool memory. Every GPU
// that loads the library holds it until the process exits. Host code only ever passes its
// device address, looked up per device below (the array's name is a host-side stand-in).
static __device__ __align__(256) float g_vla_noalloc_scratch[VLA_NOALLOC_MAX_FLOATS];

// Device address of g_vla_noalloc_scratch on the current device, looked up once per device
// (the first call on a device, with that device current).
int noalloc_scratch(float** out) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static float* addr[kMaxDev] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return DR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_vla_noalloc_scratch) != cudaSuccess || !p)
            return DR_ERR_CUDA;
        addr[dev] = static_cast<float*>(p);
    }
    *out = addr[dev];
    return DR_OK;
}

// The chunked pair with the directions in the fixed array (nothing allocated or freed).
template <int D, bool RATIO>
int launch_vla_noalloc(const float* q, const float* k, const float* v, const float* u,
                       const float* S0, const float* A0, const float* n0, float lambda0,
                       float* out, float* S_final, float* A_final, float* n_final, long BH,
                       int T, float* alpha, cudaStream_t stream) {
    const int smem_a = (int)sizeof(VcASmem<D>);
    const int smem_s = (int)sizeof(VcSSmem<D>);
    auto ka = vla_aphase_kernel<D>;
    auto ks = vla_sphase_kernel<D, RATIO>;
    if (cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_a) !=
            cudaSuccess ||
        cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_s) !=
            cudaSuccess)
        return DR_ERR_CUDA;
    ka<<<(unsigned)BH, VC_THREADS, smem_a, stream>>>(k, u, A0, lambda0, A_final, alpha, T);
    int rc = launch_status();
    if (rc != DR_OK) return rc;
    ks<<<dim3((unsigned)BH, D / VC_RS), VC_THREADS, smem_s, stream>>>(q, k, v, alpha, S0, n0, out,
                                                                    S_final, n_final, T);
    return launch_status();
}

template <int D>
int launch_vla_noalloc_readout(bool ratio, const float* q, const float* k, const float* v,
                               const float* u, const float* S0, const float* A0,
                               const float* n0, float lambda0, float* out, float* S_final,
                               float* A_final, float* n_final, long BH, int T, float* alpha,
                               cudaStream_t stream) {
    if (ratio)
        return launch_vla_noalloc<D, true>(q, k, v, u, S0, A0, n0, lambda0, out, S_final,
                                           A_final, n_final, BH, T, alpha, stream);
    return launch_vla_noalloc<D, false>(q, k, v, u, S0, A0, nullptr, lambda0, out, S_final,
                                        A_final, nullptr, BH, T, alpha, stream);
}

}  // namespace

extern "C" {

int dr_version(void) { return kVersion; }

const char* dr_status_string(int status) {
    switch (status) {
        case DR_OK:
            return "ok";
        case DR_ERR_INVALID_ARG:
            return "invalid argument (null or misaligned pointer, negative size, bad mode flag)";
        case DR_ERR_UNSUPPORTED:
            return "unsupported shape (dk, dv or d outside the compiled set)";
        case DR_ERR_CUDA:
            return "CUDA runtime or driver error";
        case DR_ERR_TIMEOUT:
            return "device: a bounded barrier wait ran out; outputs are invalid";
        case DR_ERR_DEVICE_BOUNDS:
            return "device: an index check failed; outputs are invalid";
        case DR_ERR_GATE_RANGE:
            return "device: a KDA gate's summed log-decay over one chunk is below the chunked "
                   "kernel's range; outputs are invalid (rerun with DR_FORCE_SEQUENTIAL)";
        case DR_ERR_NOT_SPD:
            return "device: VLA's inverse penalty A is not positive definite (a non-positive "
                   "pivot in I + U A U^T); outputs are invalid";
        case DR_ERR_SCRATCH_LIMIT:
            return "request too large for vla_scan_fwd_noalloc's fixed scratch array "
                   "(B*H*T*d > VLA_NOALLOC_MAX_FLOATS); use vla_scan_fwd_ex";
    }
    return "unknown status";
}

int dr_scan_fwd_ex(const void* q, const void* k, const void* v, const float* beta,
                   const float* gate, const float* erase, const float* write, const float* S0,
                   void* out, float* S_final, void* u_out, int B, int H, int T, int dk, int dv,
                   int mode, cudaStream_t stream) {
    const int variant = mode & DR_MODE_MASK;
    if (mode & ~(DR_MODE_MASK | DR_IN_BF16 | DR_FORCE_SEQUENTIAL | DR_CHAINED))
        return DR_ERR_INVALID_ARG;
    if (variant > DR_GDN2) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    const bool gated = variant == DR_GDN || variant == DR_KDA || variant == DR_GDN2;
    // per-token tensors are read only when there are tokens (empty tensors may be NULL)
    const bool tokens = BH > 0 && T > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(out)))
        return DR_ERR_INVALID_ARG;
    if (tokens && variant != DR_LINEAR && !ok_ptr(beta)) return DR_ERR_INVALID_ARG;
    if (tokens && gated && !ok_ptr(gate)) return DR_ERR_INVALID_ARG;
    if (tokens && variant == DR_GDN2 && (!ok_ptr(erase) || !ok_ptr(write)))
        return DR_ERR_INVALID_ARG;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(out) || !ok_opt(beta) ||
        !ok_opt(gate) || !ok_opt(erase) || !ok_opt(write) || !ok_opt(S0) ||
        !ok_opt(S_final) || !ok_opt(u_out))
        return DR_ERR_INVALID_ARG;
    if (!dim_supported(dk) || !dim_supported(dv)) return DR_ERR_UNSUPPORTED;
    if (BH == 0) return DR_OK;
    if (T == 0) return copy_state(S_final, S0, (size_t)BH * dv * dk, stream);

    const bool bf16 = (mode & DR_IN_BF16) != 0;
    ChunkArgs a{q, k, v, variant == DR_LINEAR ? nullptr : beta, gated ? gate : nullptr,
                variant == DR_GDN2 ? erase : nullptr, variant == DR_GDN2 ? write : nullptr,
                S0, out, S_final, u_out, (int)BH, T, dv};
    if (bf16 && !(mode & DR_FORCE_SEQUENTIAL) && chunked_supported(variant, dk, dv))
        return variant == DR_GDN2
                   ? launch_gdn2_chunked(a, dk, (mode & DR_CHAINED) != 0, stream)
                   : launch_chunked_auto(a, variant, (mode & DR_CHAINED) != 0, stream);
    if (bf16) return dispatch_sequential<__nv_bfloat16>(a, dk, variant, stream);
    return dispatch_sequential<float>(a, dk, variant, stream);
}

int dr_scan_fwd(const void* q, const void* k, const void* v, const float* beta, const float* gate,
                const float* S0, void* out, float* S_final, int B, int H, int T, int dk, int dv,
                int mode, cudaStream_t stream) {
    // Gated DeltaNet-2 needs its erase and write gates: only dr_scan_fwd_ex takes them
    if ((mode & DR_MODE_MASK) == DR_GDN2) return DR_ERR_INVALID_ARG;
    return dr_scan_fwd_ex(q, k, v, beta, gate, nullptr, nullptr, S0, out, S_final, nullptr, B, H,
                          T, dk, dv, mode, stream);
}

int dr_decode_step_ex(const void* q, const void* k, const void* v, const float* beta,
                      const float* gate, const float* erase, const float* write, float* S,
                      void* out, void* u_out, int B, int H, int dk, int dv, int mode,
                      cudaStream_t stream) {
    const int variant = mode & DR_MODE_MASK;
    if (mode & ~(DR_MODE_MASK | DR_IN_BF16)) return DR_ERR_INVALID_ARG;
    if (variant > DR_GDN2) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || dk <= 0 || dv <= 0) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    const bool gated = variant == DR_GDN || variant == DR_KDA || variant == DR_GDN2;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(out) || !ok_opt(beta) ||
        !ok_opt(gate) || !ok_opt(erase) || !ok_opt(write) || !ok_opt(S) || !ok_opt(u_out))
        return DR_ERR_INVALID_ARG;
    if (BH > 0) {
        if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(out) || !ok_ptr(S))
            return DR_ERR_INVALID_ARG;
        if (variant != DR_LINEAR && !ok_ptr(beta)) return DR_ERR_INVALID_ARG;
        if (gated && !ok_ptr(gate)) return DR_ERR_INVALID_ARG;
        if (variant == DR_GDN2 && (!ok_ptr(erase) || !ok_ptr(write))) return DR_ERR_INVALID_ARG;
    }
    if (!dim_supported(dk) || !dim_supported(dv)) return DR_ERR_UNSUPPORTED;
    if (BH == 0) return DR_OK;
    const long rows = BH * dv;
    if (rows / ((long)DEC_ROWS * DEC_WARPS) >= INT_MAX) return DR_ERR_UNSUPPORTED;
    DecodeArgs a{q, k, v, variant == DR_LINEAR ? nullptr : beta, gated ? gate : nullptr,
                 variant == DR_GDN2 ? erase : nullptr, variant == DR_GDN2 ? write : nullptr, S,
                 out, u_out, rows, dv};
    if (mode & DR_IN_BF16) return dispatch_decode<__nv_bfloat16>(a, dk, variant, stream);
    return dispatch_decode<float>(a, dk, variant, stream);
}

int dr_decode_step(const void* q, const void* k, const void* v, const float* beta,
                   const float* gate, float* S, void* out, int B, int H, int dk, int dv, int mode,
                   cudaStream_t stream) {
    if ((mode & DR_MODE_MASK) == DR_GDN2) return DR_ERR_INVALID_ARG;
    return dr_decode_step_ex(q, k, v, beta, gate, nullptr, nullptr, S, out, nullptr, B, H, dk, dv,
                             mode, stream);
}

int vla_scan_fwd_ex(const float* q, const float* k, const float* v, const float* u,
                    const float* S0, const float* A0, const float* n0, float lambda0, float* out,
                    float* S_final, float* A_final, float* n_final, int B, int H, int T, int d,
                    int flags, cudaStream_t stream) {
    if (flags & ~(VLA_RATIO_READOUT | VLA_SEQUENTIAL | VLA_TWO_KERNEL)) return DR_ERR_INVALID_ARG;
    const bool ratio = (flags & VLA_RATIO_READOUT) != 0;
    const bool sequential = (flags & VLA_SEQUENTIAL) != 0;
    const bool two_kernel = (flags & VLA_TWO_KERNEL) != 0;
    if (sequential && two_kernel) return DR_ERR_INVALID_ARG;
    if (!ratio && (n0 || n_final)) return DR_ERR_INVALID_ARG;
    if (!ok_opt(n0) || !ok_opt(n_final)) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || d <= 0) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    const bool tokens = BH > 0 && T > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(u) || !ok_ptr(out)))
        return DR_ERR_INVALID_ARG;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(u) || !ok_opt(out) || !ok_opt(S0) ||
        !ok_opt(A0) || !ok_opt(S_final) || !ok_opt(A_final))
        return DR_ERR_INVALID_ARG;
    if (!A0 && !(lambda0 > 0.f)) return DR_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 96 && d != 128) return DR_ERR_UNSUPPORTED;
    if (BH == 0) return DR_OK;
    if (T == 0) {
        const size_t n = (size_t)BH * d * d;
        int rc = copy_state(S_final, S0, n, stream);
        if (rc == DR_OK && ratio) rc = copy_state(n_final, n0, (size_t)BH * d, stream);
        if (rc != DR_OK || !A_final) return rc;
        if (A0) return copy_state(A_final, A0, n, stream);
        scaled_identity_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(A_final, d, (long)n,
                                                                               1.f / lambda0);
        return launch_status();
    }
    switch (d) {
        case 32:
            return launch_vla_readout<32>(ratio, sequential, two_kernel, q, k, v, u, S0, A0, n0,
                                          lambda0, out, S_final, A_final, n_final, BH, T, stream);
        case 64:
            return launch_vla_readout<64>(ratio, sequential, two_kernel, q, k, v, u, S0, A0, n0,
                                          lambda0, out, S_final, A_final, n_final, BH, T, stream);
        case 96:
            return launch_vla_readout<96>(ratio, sequential, two_kernel, q, k, v, u, S0, A0, n0,
                                          lambda0, out, S_final, A_final, n_final, BH, T, stream);
        case 128:
            return launch_vla_readout<128>(ratio, sequential, two_kernel, q, k, v, u, S0, A0, n0,
                                           lambda0, out, S_final, A_final, n_final, BH, T, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

int vla_scan_fwd(const float* q, const float* k, const float* v, const float* u, const float* S0,
                 const float* A0, float lambda0, float* out, float* S_final, float* A_final, int B,
                 int H, int T, int d, cudaStream_t stream) {
    return vla_scan_fwd_ex(q, k, v, u, S0, A0, nullptr, lambda0, out, S_final, A_final, nullptr,
                           B, H, T, d, 0, stream);
}

int vla_scan_fwd_noalloc(const float* q, const float* k, const float* v, const float* u,
                         const float* S0, const float* A0, const float* n0, float lambda0,
                         float* out, float* S_final, float* A_final, float* n_final, int B,
                         int H, int T, int d, int flags, cudaStream_t stream) {
    if (flags & ~VLA_RATIO_READOUT) return DR_ERR_INVALID_ARG;
    const bool ratio = (flags & VLA_RATIO_READOUT) != 0;
    if (!ratio && (n0 || n_final)) return DR_ERR_INVALID_ARG;
    if (!ok_opt(n0) || !ok_opt(n_final)) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || d <= 0) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    const bool tokens = BH > 0 && T > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(u) || !ok_ptr(out)))
        return DR_ERR_INVALID_ARG;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(u) || !ok_opt(out) || !ok_opt(S0) ||
        !ok_opt(A0) || !ok_opt(S_final) || !ok_opt(A_final))
        return DR_ERR_INVALID_ARG;
    if (!A0 && !(lambda0 > 0.f)) return DR_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 96 && d != 128) return DR_ERR_UNSUPPORTED;
    if ((double)BH * (double)T * (double)d > (double)VLA_NOALLOC_MAX_FLOATS)
        return DR_ERR_SCRATCH_LIMIT;
    if (!tokens)  // no scan to run: the state copies of vla_scan_fwd_ex, which allocate nothing
        return vla_scan_fwd_ex(q, k, v, u, S0, A0, n0, lambda0, out, S_final, A_final, n_final,
                               B, H, T, d, flags, stream);
    float* alpha = nullptr;
    const int rc = noalloc_scratch(&alpha);
    if (rc != DR_OK) return rc;
    switch (d) {
        case 32:
            return launch_vla_noalloc_readout<32>(ratio, q, k, v, u, S0, A0, n0, lambda0, out,
                                                  S_final, A_final, n_final, BH, T, alpha, stream);
        case 64:
            return launch_vla_noalloc_readout<64>(ratio, q, k, v, u, S0, A0, n0, lambda0, out,
                                                  S_final, A_final, n_final, BH, T, alpha, stream);
        case 96:
            return launch_vla_noalloc_readout<96>(ratio, q, k, v, u, S0, A0, n0, lambda0, out,
                                                  S_final, A_final, n_final, BH, T, alpha, stream);
        case 128:
            return launch_vla_noalloc_readout<128>(ratio, q, k, v, u, S0, A0, n0, lambda0, out,
                                                   S_final, A_final, n_final, BH, T, alpha,
                                                   stream);
    }
    return DR_ERR_UNSUPPORTED;
}

int loglinear_scan_fwd(const void* q, const void* k, const void* v, const float* lambda,
                       void* out, int B, int H, int T, int dk, int dv, int L, int mode,
                       cudaStream_t stream) {
    if (mode & ~DR_IN_BF16) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || L < 1) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    // every position needs its level: level 0 plus one per bit of T - 1
    int need = 1;
    while (need < 31 && ((long)(T > 0 ? T - 1 : 0) >> (need - 1)) > 0) ++need;
    if (L < need) return DR_ERR_INVALID_ARG;
    const bool tokens = BH > 0 && T > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(lambda) || !ok_ptr(out)))
        return DR_ERR_INVALID_ARG;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(lambda) || !ok_opt(out))
        return DR_ERR_INVALID_ARG;
    if (!(mode & DR_IN_BF16) || dk != LL_DK || (dv != 32 && dv != 64 && dv != 128) ||
        L > LL_LMAX || (long)T > (long)LL_C << LL_LEVELS)
        return DR_ERR_UNSUPPORTED;
    if (!tokens) return DR_OK;
    const int smem = (int)sizeof(LoglinearSmem);
    static bool attr_set[16] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DR_ERR_CUDA;
    if (dev < 0 || dev >= 16 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(loglinear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess)
            return DR_ERR_CUDA;
        if (dev >= 0 && dev < 16) attr_set[dev] = true;
    }
    loglinear_kernel<<<dim3((unsigned)BH, (unsigned)(dv / LL_BV)), LL_THREADS, smem, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), lambda, static_cast<__nv_bfloat16*>(out), T, dv, L);
    return launch_status();
}

int dr_poll_error(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return DR_ERR_CUDA;
    int status = 0;
    if (cudaMemcpyFromSymbol(&status, g_status, sizeof(int)) != cudaSuccess) return DR_ERR_CUDA;
    if (status != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return DR_ERR_CUDA;
    }
    return status;
}

int dr_segment_counters(unsigned long long* scans, unsigned long long* reruns) {
    if (!scans || !reruns) return DR_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(scans, drscan::g_seg_scans, sizeof(*scans)) != cudaSuccess ||
        cudaMemcpyFromSymbol(reruns, drscan::g_seg_reruns, sizeof(*reruns)) != cudaSuccess)
        return DR_ERR_CUDA;
    return DR_OK;
}

int dr_chunked_plan_ex(int mode, long long BH, int T, int dk, int dv, int* bv, int* nprep,
                       int* nseg) {
    if (!nseg || T < 0) return DR_ERR_INVALID_ARG;
    *nseg = 1;
    int rc = dr_chunked_plan(mode, BH, dk, dv, bv, nprep);
    if (rc != DR_OK || (mode & DR_CHAINED)) return rc;
    const int variant = mode & DR_MODE_MASK;
    const drscan::SegPlan sp = drscan::pick_segments(
        variant == DR_GDN2 ? DR_GDN : variant, (long)BH, T, dv);
    if (sp.nseg > 1) {
        *nseg = sp.nseg;
        *bv = sp.split.bv;
        *nprep = sp.split.nprep;
    }
    return DR_OK;
}

int dr_chunked_plan(int mode, long long BH, int dk, int dv, int* bv, int* nprep) {
    if ((mode & DR_MODE_MASK) > DR_GDN2) return DR_ERR_INVALID_ARG;
    if (!bv || !nprep) return DR_ERR_INVALID_ARG;
    *bv = 0;
    *nprep = 0;
    const int variant = mode & DR_MODE_MASK;
    if (mode & ~(DR_MODE_MASK | DR_IN_BF16 | DR_FORCE_SEQUENTIAL | DR_CHAINED))
        return DR_ERR_INVALID_ARG;
    if (BH < 1 || BH > INT_MAX) return DR_ERR_INVALID_ARG;
    if (!(mode & DR_IN_BF16) || (mode & DR_FORCE_SEQUENTIAL) ||
        !drscan::chunked_supported(variant, dk, dv))
        return DR_ERR_UNSUPPORTED;
    const drscan::SplitPlan plan = drscan::pick_split(variant, (long)BH, dv);
    *nprep = plan.nprep;
    *bv = plan.nprep ? plan.bv : drscan::pick_bv(variant, (long)BH, dv);
    return DR_OK;
}

int dr_debug_timeout_probe(int spin_limit, cudaStream_t stream) {
    if (spin_limit < 1 || spin_limit > 1000000) return DR_ERR_INVALID_ARG;
    timeout_probe_kernel<<<1, 32, 0, stream>>>(spin_limit);
    return launch_status();
}

}  // extern "C"
