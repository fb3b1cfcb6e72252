// sscan_backward.cu -- C ABI of the backward pass (kernel in kernel_backward.cuh).
//
// Shape-based like sscan_forward_noalloc: the backward needs no plan state
// beyond the shape, the I/O type and the flags.  Argument checks, output
// zeroing (dA, dB, dC and the bias gradient are accumulated with atomics) and
// the launch.
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
int64_t bwd_dpad(int64_t D, int64_t N) { return div_up(D, bwd_block_channels(static_cast<int>(N))) * bwd_block_channels(static_cast<int>(N)); }
int64_t bwd_chunks(int64_t L) { return div_up(L, kChunk); }

// States per lane: 4 for every N (2 and 1, with twice and four times the warps,
// measured slower: the extra lane-sum work outweighs the latency hidden).
constexpr int bwd_states(int64_t) { return 4; }
// backward blocks per batch row (planes of the dB / dC partial sums)
int64_t bwd_planes(int64_t D, int64_t N) {
    return bwd_dpad(D, N) / bwd_block_channels_s(static_cast<int>(N), bwd_states(N));
}
size_t bwd_ckpt_bytes(int64_t B, int64_t L, int64_t D, int64_t N) {
    const size_t bytes = size_t(B) * size_t(bwd_dpad(D, N)) * size_t(bwd_chunks(L)) * size_t(N) * sizeof(float);
    return (bytes + 255) / 256 * 256;
}

template <class IO, int N, int S, bool ZOH, bool FUSED, bool STAGED>
int launch_backward_k(int64_t B, const BwdParams &prm, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>(prm.Dpad / bwd_block_channels_s(N, S)), static_cast<unsigned>(B));
    constexpr int smem = bwd_smem_bytes<IO, N, S, STAGED>();
    if (smem_opt_in<sscan_backward_kernel<IO, N, S, ZOH, FUSED, STAGED>>(smem) != cudaSuccess) return SSCAN_ERR_CUDA;
    sscan_backward_kernel<IO, N, S, ZOH, FUSED, STAGED><<<grid, kBwdThreads, smem, s>>>(prm);
    return cudaGetLastError() == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

// The staged kernel copies 4-byte words of every row: fp32, or bf16 with an even D.
template <class IO, int N, int S, bool ZOH, bool FUSED>
int launch_backward_t(int64_t B, const BwdParams &prm, cudaStream_t s) {
    if (sizeof(IO) == 4 || prm.D % 2 == 0) return launch_backward_k<IO, N, S, ZOH, FUSED, true>(B, prm, s);
    return launch_backward_k<IO, N, S, ZOH, FUSED, false>(B, prm, s);
}

template <class IO, int N, int S>
int launch_backward_s(int64_t B, bool zoh, bool fused, const BwdParams &prm, cudaStream_t s) {
    if (fused)
        return zoh ? launch_backward_t<IO, N, S, true, true>(B, prm, s) : launch_backward_t<IO, N, S, false, true>(B, prm, s);
    return zoh ? launch_backward_t<IO, N, S, true, false>(B, prm, s) : launch_backward_t<IO, N, S, false, false>(B, prm, s);
}

template <class IO>
int launch_backward(int64_t B, int64_t N, bool zoh, bool fused, const BwdParams &prm, cudaStream_t s) {
    switch (N) {
        case 16: return launch_backward_s<IO, 16, bwd_states(16)>(B, zoh, fused, prm, s);
        case 32: return launch_backward_s<IO, 32, bwd_states(32)>(B, zoh, fused, prm, s);
        default: return launch_backward_s<IO, 64, bwd_states(64)>(B, zoh, fused, prm, s);
    }
}

}  // namespace

extern "C" {

size_t sscan_backward_workspace_bytes(int64_t B, int64_t L, int64_t D, int64_t N) {
    if (B < 1 || D < 1 || L < 1 || (N != 16 && N != 32 && N != 64)) return 0;
    const size_t part = size_t(bwd_planes(D, N)) * size_t(B) * size_t(L) * 2 * size_t(N) * sizeof(float);
    return bwd_ckpt_bytes(B, L, D, N) + (part + 255) / 256 * 256;
}

int sscan_backward_gated(int64_t B, int64_t L, int64_t D, int64_t N, int dtype, uint32_t flags, const void *u,
                         const void *delta, const float *A, const void *Bm, const void *Cm, const float *h0,
                         const float *delta_bias, const void *z, const void *dy, const float *dh_final, void *du,
                         void *ddelta, float *dA, float *dB, float *dC, float *dh0, float *ddelta_bias, void *dz,
                         void *workspace, void *stream) {
    if (B < 1 || D < 1 || L < 0) return SSCAN_ERR_INVALID;
    if (B > 65535 || D > (int64_t(1) << 31) || L > (int64_t(1) << 40)) return SSCAN_ERR_UNSUPPORTED;
    if (dtype != SSCAN_F32 && dtype != SSCAN_BF16) return SSCAN_ERR_INVALID;
    if (flags & ~static_cast<uint32_t>(SSCAN_ZOH | SSCAN_DELTA_SOFTPLUS)) return SSCAN_ERR_INVALID;
    if (N != 16 && N != 32 && N != 64) return SSCAN_ERR_UNSUPPORTED;
    const bool softplus = (flags & SSCAN_DELTA_SOFTPLUS) != 0;
    const bool fused = softplus || delta_bias != nullptr || z != nullptr;
    const size_t es = dtype == SSCAN_F32 ? 4 : 2;
    const size_t n_bld = static_cast<size_t>(B * L * D), n_bln = static_cast<size_t>(B * L * N);
    const size_t n_dn = static_cast<size_t>(D * N), n_bdn = static_cast<size_t>(B * D * N);
    if (!A || !dA) return SSCAN_ERR_INVALID;
    if (n_bld && (!u || !delta || !Bm || !Cm || !dy || !du || !ddelta || !dB || !dC)) return SSCAN_ERR_INVALID;
    if (z && n_bld && !dz) return SSCAN_ERR_INVALID;
    if (delta_bias && !ddelta_bias) return SSCAN_ERR_INVALID;
    const void *ptrs[] = {u, delta, A, Bm, Cm, h0, delta_bias, z, dy, dh_final, du, ddelta, dA, dB, dC, dh0,
                          ddelta_bias, dz, workspace};
    for (const void *q : ptrs)
        if (q && !aligned16_b(q)) return SSCAN_ERR_ALIGN;
    // outputs must not overlap inputs or each other
    const void *ins[] = {u, delta, A, Bm, Cm, h0, dy, dh_final, delta_bias, z};
    const size_t insz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * es, n_bln * es, n_bdn * 4, n_bld * es, n_bdn * 4,
                           static_cast<size_t>(D) * 4, n_bld * es};
    const void *outs[] = {du, ddelta, dA, dB, dC, dh0, ddelta_bias, dz};
    const size_t outsz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * 4, n_bln * 4, n_bdn * 4,
                            static_cast<size_t>(D) * 4, n_bld * es};
    for (int i = 0; i < 8; ++i) {
        for (int k = 0; k < 10; ++k)
            if (overlaps_b(outs[i], outsz[i], ins[k], insz[k])) return SSCAN_ERR_INVALID;
        for (int k = i + 1; k < 8; ++k)
            if (overlaps_b(outs[i], outsz[i], outs[k], outsz[k])) return SSCAN_ERR_INVALID;
    }
    const size_t ws = sscan_backward_workspace_bytes(B, L, D, N);
    if (ws && !workspace) return SSCAN_ERR_WORKSPACE;
    for (int k = 0; k < 10; ++k)
        if (ws && overlaps_b(workspace, ws, ins[k], insz[k])) return SSCAN_ERR_WORKSPACE;
    for (int i = 0; i < 8; ++i)
        if (ws && overlaps_b(workspace, ws, outs[i], outsz[i])) return SSCAN_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // dA and the bias gradient are accumulated with atomics (dB and dC are written whole)
    if (cudaMemsetAsync(dA, 0, n_dn * 4, s) != cudaSuccess) return SSCAN_ERR_CUDA;
    if (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, static_cast<size_t>(D) * 4, s) != cudaSuccess)
        return SSCAN_ERR_CUDA;
    if (L == 0) {  // no tokens: dh0 = dh_final
        if (dh0 && (dh_final ? cudaMemcpyAsync(dh0, dh_final, n_bdn * 4, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dh0, 0, n_bdn * 4, s)) != cudaSuccess)
            return SSCAN_ERR_CUDA;
        return SSCAN_OK;
    }
    BwdParams prm;
    prm.u = u; prm.delta = delta; prm.Bm = Bm; prm.Cm = Cm; prm.dy = dy; prm.z = z;
    prm.A = A; prm.h0 = h0; prm.dhf = dh_final; prm.bias = delta_bias;
    prm.du = du; prm.ddelta = ddelta; prm.dz = dz;
    prm.dA = dA; prm.dB = dB; prm.dC = dC; prm.dh0 = dh0; prm.dbias = ddelta_bias;
    prm.ckpt = static_cast<float *>(workspace);
    prm.part = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + bwd_ckpt_bytes(B, L, D, N));
    prm.L = L; prm.D = D; prm.Dpad = bwd_dpad(D, N); prm.nchunks = bwd_chunks(L);
    prm.softplus = softplus ? 1 : 0;
    const bool zoh = (flags & SSCAN_ZOH) != 0;
    const int rc = dtype == SSCAN_F32 ? launch_backward<float>(B, N, zoh, fused, prm, s)
                                      : launch_backward<uint16_t>(B, N, zoh, fused, prm, s);
    if (rc != SSCAN_OK) return rc;
    const int64_t quads = B * L * 2 * (N / 4);
    const int64_t rblocks = div_up(quads, 256) < 148 * 64 ? div_up(quads, 256) : 148 * 64;  // grid-stride beyond
    sscan_backward_reduce_kernel<<<static_cast<unsigned>(rblocks), 256, 0, s>>>(
        prm.part, dB, dC, B * L, static_cast<int>(N), bwd_planes(D, N));
    return cudaGetLastError() == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

int sscan_backward(int64_t B, int64_t L, int64_t D, int64_t N, int dtype, uint32_t flags, const void *u,
                   const void *delta, const float *A, const void *Bm, const void *Cm, const float *h0,
                   const void *dy, const float *dh_final, void *du, void *ddelta, float *dA, float *dB, float *dC,
                   float *dh0, void *workspace, void *stream) {
    return sscan_backward_gated(B, L, D, N, dtype, flags, u, delta, A, Bm, Cm, h0, nullptr, nullptr, dy, dh_final,
                                du, ddelta, dA, dB, dC, dh0, nullptr, nullptr, workspace, stream);
}

}  // extern "C"
