// C-ABI entry points of libdrscan: argument validation, kernel selection and launch.
// The declarations, with the meaning and layout of every argument, are in drscan.h.
// All kernels live in this one translation unit so that they share the device status
// word without relocatable device code.
#include <climits>
#include <cstdint>
#include <cstdio>

#include "common.cuh"
#include "dr_chunked.cuh"
#include "dr_decode.cuh"
#include "dr_sequential.cuh"
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

template <typename TIn, int MODE, int DK>
int launch_decode(const void* q, const void* k, const void* v, const float* beta, const float* gate,
                  float* S, void* out, long rows, int dv, cudaStream_t stream) {
    constexpr long per_cta = (long)DEC_ROWS * DEC_WARPS;
    dr_decode_kernel<TIn, MODE, DK><<<(unsigned)((rows + per_cta - 1) / per_cta), DEC_THREADS, 0,
                                       stream>>>(
        static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), beta,
        gate, S, S, static_cast<TIn*>(out), rows, dv);
    return launch_status();
}

template <typename TIn, int MODE>
int dispatch_decode_dk(const void* q, const void* k, const void* v, const float* beta,
                       const float* gate, float* S, void* out, long rows, int dk, int dv,
                       cudaStream_t stream) {
    switch (dk) {
        case 32:
            return launch_decode<TIn, MODE, 32>(q, k, v, beta, gate, S, out, rows, dv, stream);
        case 64:
            return launch_decode<TIn, MODE, 64>(q, k, v, beta, gate, S, out, rows, dv, stream);
        case 128:
            return launch_decode<TIn, MODE, 128>(q, k, v, beta, gate, S, out, rows, dv, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

template <typename TIn>
int dispatch_decode(const void* q, const void* k, const void* v, const float* beta,
                    const float* gate, float* S, void* out, long rows, int dk, int dv, int variant,
                    cudaStream_t stream) {
    switch (variant) {
        case DR_LINEAR:
            return dispatch_decode_dk<TIn, DR_LINEAR>(q, k, v, beta, gate, S, out, rows, dk, dv,
                                                      stream);
        case DR_DELTANET:
            return dispatch_decode_dk<TIn, DR_DELTANET>(q, k, v, beta, gate, S, out, rows, dk, dv,
                                                        stream);
        case DR_GDN:
            return dispatch_decode_dk<TIn, DR_GDN>(q, k, v, beta, gate, S, out, rows, dk, dv, stream);
        case DR_KDA:
            return dispatch_decode_dk<TIn, DR_KDA>(q, k, v, beta, gate, S, out, rows, dk, dv, stream);
    }
    return DR_ERR_INVALID_ARG;
}

template <typename TIn, int MODE, int DK>
int launch_sequential(const void* q, const void* k, const void* v, const float* beta,
                      const float* gate, const float* S0, void* out, float* S_final, long BH,
                      int T, int dv, cudaStream_t stream) {
    dim3 grid((unsigned)BH, (unsigned)(dv / 32));
    dr_sequential_kernel<TIn, MODE, DK><<<grid, 32, 0, stream>>>(
        static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), beta,
        gate, S0, static_cast<TIn*>(out), S_final, T, dv);
    return launch_status();
}

template <typename TIn, int MODE>
int dispatch_sequential_dk(const void* q, const void* k, const void* v, const float* beta,
                           const float* gate, const float* S0, void* out, float* S_final, long BH,
                           int T, int dk, int dv, cudaStream_t stream) {
    switch (dk) {
        case 32:
            return launch_sequential<TIn, MODE, 32>(q, k, v, beta, gate, S0, out, S_final, BH, T,
                                                    dv, stream);
        case 64:
            return launch_sequential<TIn, MODE, 64>(q, k, v, beta, gate, S0, out, S_final, BH, T,
                                                    dv, stream);
        case 128:
            return launch_sequential<TIn, MODE, 128>(q, k, v, beta, gate, S0, out, S_final, BH, T,
                                                     dv, stream);
    }
    return DR_ERR_UNSUPPORTED;
}

template <typename TIn>
int dispatch_sequential(const void* q, const void* k, const void* v, const float* beta,
                        const float* gate, const float* S0, void* out, float* S_final, long BH,
                        int T, int dk, int dv, int variant, cudaStream_t stream) {
    switch (variant) {
        case DR_LINEAR:
            return dispatch_sequential_dk<TIn, DR_LINEAR>(q, k, v, beta, gate, S0, out, S_final,
                                                          BH, T, dk, dv, stream);
        case DR_DELTANET:
            return dispatch_sequential_dk<TIn, DR_DELTANET>(q, k, v, beta, gate, S0, out, S_final,
                                                            BH, T, dk, dv, stream);
        case DR_GDN:
            return dispatch_sequential_dk<TIn, DR_GDN>(q, k, v, beta, gate, S0, out, S_final, BH,
                                                       T, dk, dv, stream);
        case DR_KDA:
            return dispatch_sequential_dk<TIn, DR_KDA>(q, k, v, beta, gate, S0, out, S_final, BH,
                                                       T, dk, dv, stream);
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

__global__ void scaled_identity_kernel(float* A, int d, long count, float diag) {
    long e = blockIdx.x * (long)blockDim.x + threadIdx.x;
    if (e < count) {
        const long rc = e % ((long)d * d);
        A[e] = (rc / d == rc % d) ? diag : 0.f;
    }
}

template <int D>
int launch_vla(const float* q, const float* k, const float* v, const float* u, const float* S0,
               const float* A0, float lambda0, float* out, float* S_final, float* A_final,
               long BH, int T, cudaStream_t stream) {
    const int smem = (int)sizeof(VlaSmem<D>);
    if (cudaFuncSetAttribute(vla_sequential_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
        return DR_ERR_CUDA;
    vla_sequential_kernel<D><<<(unsigned)BH, 2 * D, smem, stream>>>(
        q, k, v, u, S0, A0, lambda0, out, S_final, A_final, T);
    return launch_status();
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
    }
    return "unknown status";
}

int dr_scan_fwd(const void* q, const void* k, const void* v, const float* beta, const float* gate,
                const float* S0, void* out, float* S_final, int B, int H, int T, int dk, int dv,
                int mode, cudaStream_t stream) {
    const int variant = mode & DR_MODE_MASK;
    if (mode & ~(DR_MODE_MASK | DR_IN_BF16 | DR_FORCE_SEQUENTIAL)) return DR_ERR_INVALID_ARG;
    if (variant > DR_KDA) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    // per-token tensors are read only when there are tokens (empty tensors may be NULL)
    const bool tokens = BH > 0 && T > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(out)))
        return DR_ERR_INVALID_ARG;
    if (tokens && variant != DR_LINEAR && !ok_ptr(beta)) return DR_ERR_INVALID_ARG;
    if (tokens && (variant == DR_GDN || variant == DR_KDA) && !ok_ptr(gate))
        return DR_ERR_INVALID_ARG;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(out) || !ok_opt(beta) ||
        !ok_opt(gate) || !ok_opt(S0) || !ok_opt(S_final))
        return DR_ERR_INVALID_ARG;
    if (!dim_supported(dk) || !dim_supported(dv)) return DR_ERR_UNSUPPORTED;
    if (BH == 0) return DR_OK;
    if (T == 0) return copy_state(S_final, S0, (size_t)BH * dv * dk, stream);

    const bool bf16 = (mode & DR_IN_BF16) != 0;
    if (variant == DR_LINEAR) beta = nullptr;
    if (variant == DR_LINEAR || variant == DR_DELTANET) gate = nullptr;
    if (bf16 && !(mode & DR_FORCE_SEQUENTIAL) && chunked_supported(variant, dk, dv))
        return launch_chunked(q, k, v, beta, gate, S0, out, S_final, (int)BH, T, dk, dv, variant,
                              stream);
    if (bf16)
        return dispatch_sequential<__nv_bfloat16>(q, k, v, beta, gate, S0, out, S_final, BH, T, dk,
                                                  dv, variant, stream);
    return dispatch_sequential<float>(q, k, v, beta, gate, S0, out, S_final, BH, T, dk, dv,
                                      variant, stream);
}

int dr_decode_step(const void* q, const void* k, const void* v, const float* beta,
                   const float* gate, float* S, void* out, int B, int H, int dk, int dv, int mode,
                   cudaStream_t stream) {
    const int variant = mode & DR_MODE_MASK;
    if (mode & ~(DR_MODE_MASK | DR_IN_BF16)) return DR_ERR_INVALID_ARG;
    if (variant > DR_KDA) return DR_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || dk <= 0 || dv <= 0) return DR_ERR_INVALID_ARG;
    const long BH = (long)B * (long)H;
    if (BH > INT_MAX) return DR_ERR_INVALID_ARG;
    if (!ok_opt(q) || !ok_opt(k) || !ok_opt(v) || !ok_opt(out) || !ok_opt(beta) ||
        !ok_opt(gate) || !ok_opt(S))
        return DR_ERR_INVALID_ARG;
    if (BH > 0) {
        if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(out) || !ok_ptr(S))
            return DR_ERR_INVALID_ARG;
        if (variant != DR_LINEAR && !ok_ptr(beta)) return DR_ERR_INVALID_ARG;
        if ((variant == DR_GDN || variant == DR_KDA) && !ok_ptr(gate)) return DR_ERR_INVALID_ARG;
    }
    if (!dim_supported(dk) || !dim_supported(dv)) return DR_ERR_UNSUPPORTED;
    if (BH == 0) return DR_OK;
    const long rows = BH * dv;
    if (rows / ((long)DEC_ROWS * DEC_WARPS) >= INT_MAX) return DR_ERR_UNSUPPORTED;
    if (variant == DR_LINEAR) beta = nullptr;
    if (variant == DR_LINEAR || variant == DR_DELTANET) gate = nullptr;
    if (mode & DR_IN_BF16)
        return dispatch_decode<__nv_bfloat16>(q, k, v, beta, gate, S, out, rows, dk, dv, variant,
                                              stream);
    return dispatch_decode<float>(q, k, v, beta, gate, S, out, rows, dk, dv, variant, stream);
}

int vla_scan_fwd(const float* q, const float* k, const float* v, const float* u, const float* S0,
                 const float* A0, float lambda0, float* out, float* S_final, float* A_final, int B,
                 int H, int T, int d, cudaStream_t stream) {
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
        if (rc != DR_OK || !A_final) return rc;
        if (A0) return copy_state(A_final, A0, n, stream);
        scaled_identity_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(A_final, d, (long)n,
                                                                               1.f / lambda0);
        return launch_status();
    }
    switch (d) {
        case 32:
            return launch_vla<32>(q, k, v, u, S0, A0, lambda0, out, S_final, A_final, BH, T,
                                  stream);
        case 64:
            return launch_vla<64>(q, k, v, u, S0, A0, lambda0, out, S_final, A_final, BH, T,
                                  stream);
        case 96:
            return launch_vla<96>(q, k, v, u, S0, A0, lambda0, out, S_final, A_final, BH, T,
                                  stream);
        case 128:
            return launch_vla<128>(q, k, v, u, S0, A0, lambda0, out, S_final, A_final, BH, T,
                                   stream);
    }
    return DR_ERR_UNSUPPORTED;
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

int dr_chunked_plan(int mode, long long BH, int dk, int dv, int* bv, int* nprep) {
    if (!bv || !nprep) return DR_ERR_INVALID_ARG;
    *bv = 0;
    *nprep = 0;
    const int variant = mode & DR_MODE_MASK;
    if (mode & ~(DR_MODE_MASK | DR_IN_BF16 | DR_FORCE_SEQUENTIAL)) return DR_ERR_INVALID_ARG;
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
