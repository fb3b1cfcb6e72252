// kernel_backward.cuh -- backward pass of the selective scan (N = 16).
//
// Gradients of a loss through h_t = Abar_t h_{t-1} + beta_t u_t,
// y_t = sum_n C_t[n] h_t[n], Abar_t = exp(delta_t A), beta_t = delta_t B_t
// (Euler) or (Abar_t - 1)/A B_t (ZOH), from dy (and optionally dh_final):
//
//   g_t = C_t dy_t + Abar_{t+1} g_{t+1}            (g = dLoss/dh, a reverse scan)
//   du_t = sum_n g_t beta_t         ddelta_t = sum_n g_t (h_{t-1} A Abar_t + u_t dbeta/ddelta)
//   dA  += g_t (h_{t-1} delta_t Abar_t + u_t dbeta/dA)      (summed over b and t)
//   dB_t += g_t u_t dbeta/dB        dC_t += dy_t h_t          (summed over channels d)
//   dh0 = Abar_0 g_0
//
// "Selective State-Space Models (Mamba) and Hardware-Aware Scans", section 3:
// the backward pass recomputes the states instead of reading a stored
// [B, L, D, N] tensor.  Here a first pass runs the recurrence forward and keeps
// the state every kChunk tokens (a checkpoint per channel, in the workspace);
// the reverse sweep then takes the chunks last to first, recomputes each
// chunk's kChunk states from its checkpoint into shared memory, and runs the
// reverse recurrence over them.
//
// Mapping: one lane per channel holding all 16 states, a warp = 32 consecutive
// channels of one batch row, so du, ddelta and dA need no cross-lane work.  dB
// and dC are sums over channels: per token each lane's 16 values are
// reduce-scattered over the warp (16 + 16 shuffles), and 16 lanes add one value
// each into the fp32 output with an atomic (outputs zeroed by the host).
#pragma once

#include "device_utils.cuh"

namespace sscan {

constexpr int kBwdThreads = 128;  // 4 warps = 128 channels of one batch row
constexpr int kChunk = 8;         // tokens per recomputed chunk
constexpr int kBwdSmem = kChunk * 16 * kBwdThreads * 4;  // dynamic shared memory (64 KB)

// Sum 16 per-lane values over the 32 lanes of the warp; afterwards lane l
// (l < 16) holds the total of value l (lanes 16..31 hold duplicates).
__device__ __forceinline__ float warp_sum16(float (&v)[16], int lane) {
    // levels 16, 8, 4, 2: each lane keeps the half of its values its partner does not
#pragma unroll
    for (int m = 16, cnt = 16; m >= 2; m >>= 1, cnt >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < cnt / 2; ++i) {
            const float send = up ? v[i] : v[i + cnt / 2];
            const float keep = up ? v[i + cnt / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    // one value left: the value index is the lane's bits 4, 3, 2, 1 (halves kept at
    // each level), summed over those bits; the last level sums over bit 0
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// Value index held by lane l after warp_sum16's first four levels.
__device__ __forceinline__ int warp_sum16_index(int lane) {
    return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}

template <class IO, bool ZOH>
__global__ void __launch_bounds__(kBwdThreads)
sscan_backward_kernel(const IO *__restrict__ u, const IO *__restrict__ delta, const float *__restrict__ A,
                      const IO *__restrict__ Bm, const IO *__restrict__ Cm, const float *__restrict__ h0,
                      const IO *__restrict__ dy, const float *__restrict__ dhf, IO *__restrict__ du,
                      IO *__restrict__ ddelta, float *__restrict__ dA, float *__restrict__ dB,
                      float *__restrict__ dC, float *__restrict__ dh0, float *__restrict__ ckpt,
                      int64_t L, int64_t D, int64_t Dpad, int64_t nchunks) {
    constexpr int N = 16;
    extern __shared__ float hs[];  // [kChunk][N][kBwdThreads]: the current chunk's states
    const int lane = threadIdx.x & 31;
    const int64_t b = blockIdx.y;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * kBwdThreads + threadIdx.x;
    const bool valid = d < D;
    const int64_t dc = valid ? d : D - 1;  // past the last channel: compute on a real one, store nothing

    float a2[N], a1[N], ia[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        const float an = __ldg(A + dc * N + n);
        a2[n] = static_cast<float>(static_cast<double>(an) * 1.4426950408889634);
        a1[n] = an;
        ia[n] = an != 0.0f ? 1.0f / an : 0.0f;
    }
    const IO *up = u + b * L * D + dc;
    const IO *dp = delta + b * L * D + dc;
    const IO *gp = dy + b * L * D + dc;
    const IO *bp = Bm + b * L * N;
    const IO *cp = Cm + b * L * N;
    float *ck = ckpt + (b * Dpad + d) * nchunks * N;  // this lane's checkpoints (own slot even past D)

    // beta and its derivatives for one state
    auto coefs = [&](int n, float dl, float abar, float Bn, float &beta, float &dbdl, float &dbda, float &dbdb) {
        if (!ZOH) {
            beta = dl * Bn; dbdl = Bn; dbda = 0.0f; dbdb = dl;
        } else if (a1[n] != 0.0f) {
            const float z = dl * a1[n];
            // (e^z - 1)/A: the small-|z| form keeps the relative accuracy of e^z - 1
            const float em1 = fabsf(z) < 0.25f ? z * (1.0f + z * (0.5f + z * (1.0f / 6.0f + z * (1.0f / 24.0f + z * (1.0f / 120.0f)))))
                                              : abar - 1.0f;
            dbdb = em1 * ia[n];
            beta = dbdb * Bn;
            dbdl = abar * Bn;
            // (delta abar A - (abar - 1)) / A^2 = delta^2 sum_{k>=2} z^(k-2) (k-1)/k!: the series
            // for |z| < 1 (terms to k = 10, truncation < 5e-7 relative), where the direct
            // form cancels; the direct form beyond
            const float ser = 0.5f + z * (1.0f / 3.0f + z * (0.125f + z * (1.0f / 30.0f + z * (1.0f / 144.0f +
                              z * (1.0f / 840.0f + z * (1.0f / 5760.0f + z * (1.0f / 45360.0f + z * (1.0f / 403200.0f))))))));
            const float num = fabsf(z) < 1.0f ? dl * dl * ser : (dl * abar * a1[n] - em1) * ia[n] * ia[n];
            dbda = Bn * num;
        } else {
            beta = dl * Bn; dbdl = Bn; dbda = 0.5f * dl * dl * Bn; dbdb = dl;
        }
    };

    // ---- pass 1: forward, keeping the state entering every chunk ----
    float h[N];
#pragma unroll
    for (int n = 0; n < N; ++n) h[n] = h0 != nullptr ? h0[(b * D + dc) * N + n] : 0.0f;
    for (int64_t t = 0; t < L; ++t) {
        if (t % kChunk == 0) {
            float *dst = ck + (t / kChunk) * N;
#pragma unroll
            for (int n = 0; n < N; n += 4) *reinterpret_cast<float4 *>(dst + n) = make_float4(h[n], h[n + 1], h[n + 2], h[n + 3]);
        }
        const float x = Io<IO>::widen(Io<IO>::ld(up + t * D));
        const float dl = Io<IO>::widen(Io<IO>::ld(dp + t * D));
#pragma unroll
        for (int n = 0; n < N; ++n) {
            const float abar = ex2(dl * a2[n]);
            float beta, q0, q1, q2;
            coefs(n, dl, abar, Io<IO>::widen(Io<IO>::ld(bp + t * N + n)), beta, q0, q1, q2);
            h[n] = fmaf(abar, h[n], beta * x);
        }
    }

    // ---- pass 2: reverse sweep over the chunks ----
    float g[N], dacc[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        g[n] = dhf != nullptr ? dhf[(b * D + dc) * N + n] : 0.0f;
        dacc[n] = 0.0f;
    }
    const int vi = warp_sum16_index(lane);
    for (int64_t c = nchunks - 1; c >= 0; --c) {
        const int64_t t0 = c * kChunk;
        const int nt = static_cast<int>(L - t0 < kChunk ? L - t0 : kChunk);
        // recompute the chunk's states h_{t0 .. t0+nt-1} from its checkpoint
        float hc[N];
        const float *src = ck + c * N;
#pragma unroll
        for (int n = 0; n < N; n += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(src + n);
            hc[n] = v.x; hc[n + 1] = v.y; hc[n + 2] = v.z; hc[n + 3] = v.w;
        }
        for (int k = 0; k < nt; ++k) {
            const int64_t t = t0 + k;
            const float x = Io<IO>::widen(Io<IO>::ld(up + t * D));
            const float dl = Io<IO>::widen(Io<IO>::ld(dp + t * D));
#pragma unroll
            for (int n = 0; n < N; ++n) {
                const float abar = ex2(dl * a2[n]);
                float beta, q0, q1, q2;
                coefs(n, dl, abar, Io<IO>::widen(Io<IO>::ld(bp + t * N + n)), beta, q0, q1, q2);
                hc[n] = fmaf(abar, hc[n], beta * x);
                hs[(k * N + n) * kBwdThreads + threadIdx.x] = hc[n];
            }
        }
        // reverse over the chunk's tokens
        for (int k = nt - 1; k >= 0; --k) {
            const int64_t t = t0 + k;
            const float x = Io<IO>::widen(Io<IO>::ld(up + t * D));
            const float dl = Io<IO>::widen(Io<IO>::ld(dp + t * D));
            const float dyt = valid ? Io<IO>::widen(Io<IO>::ld(gp + t * D)) : 0.0f;  // idle lanes add nothing
            float vb[N], vc[N];
            float dut = 0.0f, ddt = 0.0f;
#pragma unroll
            for (int n = 0; n < N; ++n) {
                // h_{t-1}: the previous token of this chunk, or the chunk's checkpoint
                const float hprev = k > 0 ? hs[((k - 1) * N + n) * kBwdThreads + threadIdx.x] : ck[c * N + n];
                const float ht = hs[(k * N + n) * kBwdThreads + threadIdx.x];
                const float Bn = Io<IO>::widen(Io<IO>::ld(bp + t * N + n));
                const float Cn = Io<IO>::widen(Io<IO>::ld(cp + t * N + n));
                const float abar = ex2(dl * a2[n]);
                float beta, dbdl, dbda, dbdb;
                coefs(n, dl, abar, Bn, beta, dbdl, dbda, dbdb);
                g[n] = fmaf(Cn, dyt, g[n]);
                dut = fmaf(g[n], beta, dut);
                ddt = fmaf(g[n], fmaf(hprev * a1[n], abar, x * dbdl), ddt);
                dacc[n] = fmaf(g[n], fmaf(hprev * dl, abar, x * dbda), dacc[n]);
                vb[n] = g[n] * x * dbdb;
                vc[n] = dyt * ht;
                g[n] *= abar;
            }
            if (valid) {
                Io<IO>::st(du + (b * L + t) * D + d, dut);
                Io<IO>::st(ddelta + (b * L + t) * D + d, ddt);
            } else {
#pragma unroll
                for (int n = 0; n < N; ++n) vb[n] = 0.0f;  // idle lanes add nothing to dB
            }
            const float sb = warp_sum16(vb, lane);
            const float sc = warp_sum16(vc, lane);
            if ((lane & 1) == 0) {  // one of the two lanes holding each total
                atomicAdd(dB + (b * L + t) * N + vi, sb);
                atomicAdd(dC + (b * L + t) * N + vi, sc);
            }
        }
    }
    if (valid) {
        if (dh0 != nullptr) {
#pragma unroll
            for (int n = 0; n < N; n += 4)
                *reinterpret_cast<float4 *>(dh0 + (b * D + d) * N + n) = make_float4(g[n], g[n + 1], g[n + 2], g[n + 3]);
        }
#pragma unroll
        for (int n = 0; n < N; ++n) atomicAdd(dA + d * N + n, dacc[n]);
    }
}

}  // namespace sscan
