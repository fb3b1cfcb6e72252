// sscan_backward.cu -- C ABI of the backward pass (kernel in kernel_backward.cuh).
//
// Shape-based like sscan_forward_noalloc: the backward needs no plan state
// beyond the shape, the I/O type and the ZOH flag.  Argument checks, output
// zeroing (dA, dB, dC are accumulated with atomics) and the launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "device_utils.cuh"
#include "kernel_backward.cuh"
#include "sscan.h"

using namespace sscan;

namespace {

bool aligned16_b(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlaps_b(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}
int64_t div_up(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t bwd_dpad(int64_t D) { return div_up(D, kBwdThreads) * kBwdThreads; }
int64_t bwd_chunks(int64_t L) { return div_up(L, kChunk); }

template <class IO, bool ZOH>
int launch_backward(int64_t B, int64_t L, int64_t D, const void *u, const void *delta, const float *A,
                    const void *Bm, const void *Cm, const float *h0, const void *dy, const float *dhf, void *du,
                    void *ddelta, float *dA, float *dB, float *dC, float *dh0, void *ws, cudaStream_t s) {
    if (smem_opt_in<sscan_backward_kernel<IO, ZOH>>(kBwdSmem) != cudaSuccess) return SSCAN_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(bwd_dpad(D) / kBwdThreads), static_cast<unsigned>(B));
    sscan_backward_kernel<IO, ZOH><<<grid, kBwdThreads, kBwdSmem, s>>>(
        static_cast<const IO *>(u), static_cast<const IO *>(delta), A, static_cast<const IO *>(Bm),
        static_cast<const IO *>(Cm), h0, static_cast<const IO *>(dy), dhf, static_cast<IO *>(du),
        static_cast<IO *>(ddelta), dA, dB, dC, dh0, static_cast<float *>(ws), L, D, bwd_dpad(D), bwd_chunks(L));
    return cudaGetLastError() == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t sscan_backward_workspace_bytes(int64_t B, int64_t L, int64_t D, int64_t N) {
    if (B < 1 || D < 1 || L < 1 || N != 16) return 0;
    const size_t bytes = size_t(B) * size_t(bwd_dpad(D)) * size_t(bwd_chunks(L)) * 16 * sizeof(float);
    return (bytes + 255) / 256 * 256;
}

int sscan_backward(int64_t B, int64_t L, int64_t D, int64_t N, int dtype, uint32_t flags, const void *u,
                   const void *delta, const float *A, const void *Bm, const void *Cm, const float *h0,
                   const void *dy, const float *dh_final, void *du, void *ddelta, float *dA, float *dB, float *dC,
                   float *dh0, void *workspace, void *stream) {
    if (B < 1 || D < 1 || L < 0) return SSCAN_ERR_INVALID;
    if (B > 65535 || D > (int64_t(1) << 31) || L > (int64_t(1) << 40)) return SSCAN_ERR_UNSUPPORTED;
    if (dtype != SSCAN_F32 && dtype != SSCAN_BF16) return SSCAN_ERR_INVALID;
    if (flags & ~static_cast<uint32_t>(SSCAN_ZOH | SSCAN_DELTA_SOFTPLUS)) return SSCAN_ERR_INVALID;
    if (N != 16 || (flags & SSCAN_DELTA_SOFTPLUS)) return SSCAN_ERR_UNSUPPORTED;
    const size_t es = dtype == SSCAN_F32 ? 4 : 2;
    const size_t n_bld = static_cast<size_t>(B * L * D), n_bln = static_cast<size_t>(B * L * N);
    const size_t n_dn = static_cast<size_t>(D * N), n_bdn = static_cast<size_t>(B * D * N);
    if (!A || !dA) return SSCAN_ERR_INVALID;
    if (n_bld && (!u || !delta || !Bm || !Cm || !dy || !du || !ddelta || !dB || !dC)) return SSCAN_ERR_INVALID;
    const void *ptrs[] = {u, delta, A, Bm, Cm, h0, dy, dh_final, du, ddelta, dA, dB, dC, dh0, workspace};
    for (const void *q : ptrs)
        if (q && !aligned16_b(q)) return SSCAN_ERR_ALIGN;
    // outputs must not overlap inputs or each other
    const void *ins[] = {u, delta, A, Bm, Cm, h0, dy, dh_final};
    const size_t insz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * es, n_bln * es, n_bdn * 4, n_bld * es, n_bdn * 4};
    const void *outs[] = {du, ddelta, dA, dB, dC, dh0};
    const size_t outsz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * 4, n_bln * 4, n_bdn * 4};
    for (int i = 0; i < 6; ++i) {
        for (int k = 0; k < 8; ++k)
            if (overlaps_b(outs[i], outsz[i], ins[k], insz[k])) return SSCAN_ERR_INVALID;
        for (int k = i + 1; k < 6; ++k)
            if (overlaps_b(outs[i], outsz[i], outs[k], outsz[k])) return SSCAN_ERR_INVALID;
    }
    const size_t ws = sscan_backward_workspace_bytes(B, L, D, N);
    if (ws && !workspace) return SSCAN_ERR_WORKSPACE;
    for (int k = 0; k < 8; ++k)
        if (ws && overlaps_b(workspace, ws, ins[k], insz[k])) return SSCAN_ERR_WORKSPACE;
    for (int i = 0; i < 6; ++i)
        if (ws && overlaps_b(workspace, ws, outs[i], outsz[i])) return SSCAN_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // dA, dB, dC are accumulated with atomics
    if (cudaMemsetAsync(dA, 0, n_dn * 4, s) != cudaSuccess) return SSCAN_ERR_CUDA;
    if (n_bln && (cudaMemsetAsync(dB, 0, n_bln * 4, s) != cudaSuccess ||
                  cudaMemsetAsync(dC, 0, n_bln * 4, s) != cudaSuccess))
        return SSCAN_ERR_CUDA;
    if (L == 0) {  // no tokens: dh0 = dh_final
        if (dh0 && (dh_final ? cudaMemcpyAsync(dh0, dh_final, n_bdn * 4, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dh0, 0, n_bdn * 4, s)) != cudaSuccess)
            return SSCAN_ERR_CUDA;
        return SSCAN_OK;
    }
    const bool zoh = (flags & SSCAN_ZOH) != 0;
    if (dtype == SSCAN_F32)
        return zoh ? launch_backward<float, true>(B, L, D, u, delta, A, Bm, Cm, h0, dy, dh_final, du, ddelta, dA, dB,
                                                  dC, dh0, workspace, s)
                   : launch_backward<float, false>(B, L, D, u, delta, A, Bm, Cm, h0, dy, dh_final, du, ddelta, dA,
                                                   dB, dC, dh0, workspace, s);
    return zoh ? launch_backward<uint16_t, true>(B, L, D, u, delta, A, Bm, Cm, h0, dy, dh_final, du, ddelta, dA, dB,
                                                 dC, dh0, workspace, s)
               : launch_backward<uint16_t, false>(B, L, D, u, delta, A, Bm, Cm, h0, dy, dh_final, du, ddelta, dA, dB,
                                                  dC, dh0, workspace, s);
}

}  // extern "C"
