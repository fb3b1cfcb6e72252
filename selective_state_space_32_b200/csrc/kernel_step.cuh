// kernel_step.cuh -- the selective-scan forward for short sequences, in
// particular the single-token decode step ("tm_ssm_selective", section "What it
// costs at inference, and on a CPU": generation is a constant-size state update
// per token, h = Abar h + Bbar u, y = C . h).
//
// At L = 1 the work is a stream over the [B, D, N] fp32 state: read h0, one
// update, write h_final; the 4-byte-per-state round trip is almost all of the
// HBM traffic (a [B, D] u, delta, y is N times smaller), so the kernel is
// shaped for bandwidth: each thread owns four consecutive states of one
// channel (one 16-byte load and store), the N/4 threads of a channel are
// adjacent lanes, so a warp's state loads and stores are one contiguous
// 512-byte run, and each thread carries ITEMS channels so that every thread
// has that many independent 16-byte loads in flight.  A (a [D, N] table
// re-read by every batch row) comes from L2; B and C rows of a batch row are
// the same for all its channels (broadcast loads).  Longer sequences (up to
// the chained kernel's minimum length) run the same code token by token with
// the state in registers.  Any D; every pointer 16-byte aligned.
#pragma once

#include "device_utils.cuh"

namespace sscan {

constexpr int kStepThreads = 256;
constexpr int kStepItems = 2;  // channels per thread

// 4 values of B or C (row p[0..3]) as fp32
template <class IO> __device__ __forceinline__ float4 ld4(const IO *p);
template <> __device__ __forceinline__ float4 ld4<float>(const float *p) {
    return __ldg(reinterpret_cast<const float4 *>(p));
}
template <> __device__ __forceinline__ float4 ld4<uint16_t>(const uint16_t *p) {
    const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xffff0000u));
}

// Batch row b = blockIdx.y; thread (channel slot k of ITEMS, lane group g): states
// 4g .. 4g+3 of channel d = (blockIdx.x * ITEMS + k) * CPB + threadIdx.x / LPC;
// LPC = N/4 adjacent lanes share a channel.  (A 2-D grid: no index division.)
template <class IO, int N, bool ZOH>
__global__ void __launch_bounds__(kStepThreads)
sscan_step_kernel(const IO *__restrict__ u, const IO *__restrict__ delta, const float *__restrict__ A,
                  const IO *__restrict__ Bm, const IO *__restrict__ Cm, const float *h0, IO *__restrict__ y,
                  float *h_final, int64_t L, int64_t D, const float *__restrict__ delta_bias,
                  const IO *__restrict__ z, int softplus) {
    constexpr int LPC = N / 4;
    constexpr int CPB = kStepThreads / LPC;  // channels per block slice
    const int g = threadIdx.x % LPC;
    const int n0 = 4 * g;
    int64_t b[kStepItems], d[kStepItems];
    bool valid[kStepItems];
    f2 A2[kStepItems][2], A1[kStepItems][2], iA[kStepItems][2], h[kStepItems][2];
#pragma unroll
    for (int k = 0; k < kStepItems; ++k) {
        const int64_t dd = (static_cast<int64_t>(blockIdx.x) * kStepItems + k) * CPB + threadIdx.x / LPC;
        valid[k] = dd < D;
        b[k] = blockIdx.y;
        d[k] = valid[k] ? dd : D - 1;  // ragged tail: read a real channel, store nothing
    }
    // every independent load first: A rows, states, then the per-token inputs
#pragma unroll
    for (int k = 0; k < kStepItems; ++k) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(A + d[k] * N + n0));
        A2[k][0] = pack2(static_cast<float>(static_cast<double>(a.x) * 1.4426950408889634),
                         static_cast<float>(static_cast<double>(a.y) * 1.4426950408889634));
        A2[k][1] = pack2(static_cast<float>(static_cast<double>(a.z) * 1.4426950408889634),
                         static_cast<float>(static_cast<double>(a.w) * 1.4426950408889634));
        if (ZOH) {  // 1/A and -1/A for the ZOH coefficient
            iA[k][0] = pack2(1.0f / a.x, 1.0f / a.y);
            iA[k][1] = pack2(1.0f / a.z, 1.0f / a.w);
            A1[k][0] = pack2(-1.0f / a.x, -1.0f / a.y);
            A1[k][1] = pack2(-1.0f / a.z, -1.0f / a.w);
        }
        if (h0 != nullptr) {
            const float4 v = *reinterpret_cast<const float4 *>(h0 + (b[k] * D + d[k]) * N + n0);
            h[k][0] = pack2(v.x, v.y);
            h[k][1] = pack2(v.z, v.w);
        } else {
            h[k][0] = h[k][1] = splat2(0.0f);
        }
    }
    for (int64_t t = 0; t < L; ++t) {
        float x[kStepItems], dl[kStepItems];
        float4 Bv[kStepItems], Cv[kStepItems];
#pragma unroll
        for (int k = 0; k < kStepItems; ++k) {
            const int64_t row = b[k] * L + t;
            x[k] = Io<IO>::widen(Io<IO>::ld(u + row * D + d[k]));
            dl[k] = Io<IO>::widen(Io<IO>::ld(delta + row * D + d[k]));
            Bv[k] = ld4<IO>(Bm + row * N + n0);
            Cv[k] = ld4<IO>(Cm + row * N + n0);
        }
#pragma unroll
        for (int k = 0; k < kStepItems; ++k) {
            float dv = dl[k];
            if (delta_bias != nullptr) dv += __ldg(delta_bias + d[k]);
            if (softplus) dv = softplus_f(dv);
            const f2 dd = splat2(dv);
            const f2 b01 = pack2(Bv[k].x, Bv[k].y), b23 = pack2(Bv[k].z, Bv[k].w);
            f2 ya = splat2(0.0f);
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float e0, e1;
                const f2 e = mul2(dd, A2[k][p]);
                unpack2(e, e0, e1);
                const f2 abar = pack2(ex2(e0), ex2(e1));
                const f2 bp = p ? b23 : b01;
                const f2 bu = ZOH ? mul2(zoh_coef_pair(dd, e, iA[k][p], A1[k][p], abar), mul2(bp, splat2(x[k])))
                                  : mul2(bp, splat2(dv * x[k]));
                h[k][p] = fma2(abar, h[k][p], bu);
                ya = fma2(p ? pack2(Cv[k].z, Cv[k].w) : pack2(Cv[k].x, Cv[k].y), h[k][p], ya);
            }
            float y0, y1;
            unpack2(ya, y0, y1);
            float yv = y0 + y1;
#pragma unroll
            for (int o = 1; o < LPC; o <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
            if (valid[k] && g == 0) {
                const int64_t idx = (b[k] * L + t) * D + d[k];
                if (z != nullptr) yv *= silu_f(Io<IO>::widen(Io<IO>::ld(z + idx)));
                Io<IO>::st(y + idx, yv);
            }
        }
    }
    if (h_final != nullptr) {
#pragma unroll
        for (int k = 0; k < kStepItems; ++k) {
            if (!valid[k]) continue;
            float a0, a1, a2, a3;
            unpack2(h[k][0], a0, a1);
            unpack2(h[k][1], a2, a3);
            *reinterpret_cast<float4 *>(h_final + (b[k] * D + d[k]) * N + n0) = make_float4(a0, a1, a2, a3);
        }
    }
}

}  // namespace sscan
