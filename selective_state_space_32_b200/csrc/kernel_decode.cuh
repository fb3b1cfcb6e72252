// kernel_decode.cuh -- the single-token decode step with a carried state
// ("tm_ssm_selective", section "What it costs at inference, and on a CPU":
// generation updates a constant-size state per token, h = Abar h + Bbar u,
// y = C . h, so a step streams the whole [B, D, N] fp32 state through once).
//
// The step is an HBM stream: h0 in, h_final out, 8 bytes per state against
// 4 + 4 + ES bytes per channel of u, delta and y.  The kernel keeps many
// bytes in flight with bulk copies instead of per-thread loads.  A tile is
// one batch row x TD channels (8 KB of state).  Each persistent block owns
// one range of TD channels (several ranges when there are more ranges than
// blocks) and walks batch rows, so the per-channel constants (A, scaled once
// by log2(e), and the bias) are loaded into registers once per range; a
// producer warp copies each tile's state rows, u, delta (and z) and the row's
// B and C into a ring of shared-memory stages with cp.async.bulk (no
// multicast), several tiles ahead of the four consumer warps.  A consumer
// thread owns four consecutive states of a channel (the N/4 threads of a
// channel are adjacent lanes) in kDecItems channel slots, reads them from the stage,
// releases it, updates, and stores h_final with 16-byte stores (a warp's are
// one contiguous 512-byte run) and y from the first lane of each channel.
// h_final may be h0: a tile's state is in shared memory before any of it is
// overwritten, and tiles are disjoint.  Every wait is bounded; a wait that
// gives up latches an error bit in the status word, and the producer waits
// (bounded) for the copies it issued before it returns.
// Requirements (checked on the host): D a multiple of 8 (every bulk copy a
// multiple of 16 bytes at a 16-byte-aligned address), h0 present.
#pragma once

#include "device_utils.cuh"

namespace sscan {

constexpr int kDecConsumers = 128;                 // four consumer warps
constexpr int kDecThreads = kDecConsumers + 32;    // + one producer warp
constexpr int kDecStages = 4;
constexpr int kDecTileStateBytes = 8192;           // state bytes per tile
constexpr int kDecItems = kDecTileStateBytes / (kDecConsumers * 16);  // channel slots per thread (4 states each)

constexpr int dec_round16(int v) { return (v + 15) / 16 * 16; }

template <class IO, int N> struct DecodeCfg {
    static constexpr int LPC = N / 4;                  // threads per channel
    static constexpr int CPS = kDecConsumers / LPC;    // channels per slot
    static constexpr int TD = kDecItems * CPS;         // channels per tile
    static constexpr int ES = static_cast<int>(sizeof(IO));
    static_assert(TD * N * 4 == kDecTileStateBytes, "tile size");
    static constexpr int oH = 0;                       // state rows [TD][N] fp32
    static constexpr int oU = oH + TD * N * 4;         // u [TD]
    static constexpr int oDl = oU + dec_round16(TD * ES);
    static constexpr int oZ = oDl + dec_round16(TD * ES);
    static constexpr int oB = oZ + dec_round16(TD * ES);  // B row [N]
    static constexpr int oC = oB + dec_round16(N * ES);
    static constexpr int kStage = (oC + dec_round16(N * ES) + 127) / 128 * 128;
    static constexpr int kBarOff = kDecStages * kStage;
    static constexpr int kSmem = kBarOff + 2 * kDecStages * 8 + 128;  // + alignment slack
};

// The tiles of block `blk` of `grid`: channel ranges r = r0, r0 + r_step, ...
// (R ranges of TD channels), for each range batch rows b = b0, b0 + b_step, ...
// With R <= grid the grid is a multiple of R (K = grid / R blocks per range);
// otherwise every block takes whole ranges, all batch rows.
struct DecodeWalk {
    int64_t r0, r_step, b0, b_step;
    __device__ DecodeWalk(int64_t blk, int64_t grid, int64_t R) {
        if (R <= grid) {
            r0 = blk % R;
            r_step = R;
            b0 = blk / R;
            b_step = grid / R;
        } else {
            r0 = blk;
            r_step = grid;
            b0 = 0;
            b_step = 1;
        }
    }
};

// One cp.async.bulk global -> shared copy of `bytes` (a multiple of 16, both
// addresses 16-byte aligned), completing on `bar`.  No multicast.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

template <class IO> __device__ __forceinline__ float lds_widen(const unsigned char *p, int i) {
    if constexpr (sizeof(IO) == 4) {
        return reinterpret_cast<const float *>(p)[i];
    } else {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t *>(p)[i]) << 16);
    }
}

template <class IO> __device__ __forceinline__ float4 lds_widen4(const unsigned char *p) {
    if constexpr (sizeof(IO) == 4) {
        return *reinterpret_cast<const float4 *>(p);
    } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                           __uint_as_float(v.y & 0xffff0000u));
    }
}

template <class IO, int N, bool ZOH>
__global__ void __launch_bounds__(kDecThreads, 4)
sscan_decode_kernel(const IO *__restrict__ u, const IO *__restrict__ delta, const float *__restrict__ A,
                    const IO *__restrict__ Bm, const IO *__restrict__ Cm, const float *h0, IO *__restrict__ y,
                    float *h_final, int64_t B, int64_t D, const float *__restrict__ delta_bias,
                    const IO *__restrict__ z, int softplus, int *status) {
    using Cfg = DecodeCfg<IO, N>;
    constexpr int TD = Cfg::TD, LPC = Cfg::LPC, CPS = Cfg::CPS, ES = Cfg::ES;
    extern __shared__ unsigned char dyn_smem[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dyn_smem) + 127) & ~uintptr_t(127));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *empty = full + kDecStages;
    const int64_t R = (D + TD - 1) / TD;
    const DecodeWalk walk(blockIdx.x, gridDim.x, R);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecConsumers / 32);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (threadIdx.x >= kDecConsumers) {  // producer warp: one lane issues the copies
        if (threadIdx.x != kDecConsumers) return;
        const uint32_t bc = static_cast<uint32_t>(N * ES);
        uint32_t issued = 0;  // tiles issued by this block
        bool ok = true;
        for (int64_t r = walk.r0; r < R && ok; r += walk.r_step) {
            const int64_t d0 = r * TD;
            const int td = static_cast<int>(D - d0 < TD ? D - d0 : TD);
            const uint32_t hb = static_cast<uint32_t>(td * N * 4), vb = static_cast<uint32_t>(td * ES);
            const uint32_t bytes = hb + 2 * vb + (z ? vb : 0) + 2 * bc;
            for (int64_t b = walk.b0; b < B; b += walk.b_step, ++issued) {
                const int s = static_cast<int>(issued % kDecStages);
                if (issued >= kDecStages && !mbar_wait(&empty[s], ((issued / kDecStages) - 1) & 1)) {
                    atomicOr(status, 1);
                    ok = false;
                    break;
                }
                const int64_t row = b * D + d0;
                unsigned char *st = smem + s * Cfg::kStage;
                mbar_expect_tx(&full[s], bytes);
                bulk_load(st + Cfg::oH, h0 + row * N, hb, &full[s]);
                bulk_load(st + Cfg::oU, u + row, vb, &full[s]);
                bulk_load(st + Cfg::oDl, delta + row, vb, &full[s]);
                if (z) bulk_load(st + Cfg::oZ, z + row, vb, &full[s]);
                bulk_load(st + Cfg::oB, Bm + b * N, bc, &full[s]);
                bulk_load(st + Cfg::oC, Cm + b * N, bc, &full[s]);
            }
        }
        // wait (bounded) for the copies still in flight before the block may end
        const uint32_t first = issued > kDecStages ? issued - kDecStages : 0;
        for (uint32_t j = first; j < issued; ++j)
            if (!mbar_wait(&full[j % kDecStages], (j / kDecStages) & 1)) atomicOr(status, 1);
        return;
    }

    // consumers
    const int g = threadIdx.x % LPC;
    const int n0 = 4 * g;
    const int lane = threadIdx.x & 31;
    const int c0 = threadIdx.x / LPC;  // the thread's channels within a tile: c0 + k * CPS
    uint32_t i = 0;                    // tiles consumed by this block
    for (int64_t r = walk.r0; r < R; r += walk.r_step) {
        const int64_t d0 = r * TD;
        const int td = static_cast<int>(D - d0 < TD ? D - d0 : TD);
        int cc[kDecItems];  // ragged range: slots past the end read a loaded channel, store nothing
        // the range's per-channel constants, once: A * log2(e) (and 1/A for ZOH), the bias
        f2 a2[kDecItems][2], ia[kDecItems][2];
        float bias[kDecItems];
#pragma unroll
        for (int k = 0; k < kDecItems; ++k) {
            const int c = c0 + k * CPS;
            cc[k] = c < td ? c : td - 1;
            const float4 a = __ldg(reinterpret_cast<const float4 *>(A + (d0 + cc[k]) * N + n0));
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                a2[k][p] = pack2(static_cast<float>(static_cast<double>(av[2 * p]) * 1.4426950408889634),
                                 static_cast<float>(static_cast<double>(av[2 * p + 1]) * 1.4426950408889634));
                if constexpr (ZOH) ia[k][p] = pack2(1.0f / av[2 * p], 1.0f / av[2 * p + 1]);
            }
            bias[k] = delta_bias ? __ldg(delta_bias + d0 + cc[k]) : 0.0f;
        }
        for (int64_t b = walk.b0; b < B; b += walk.b_step, ++i) {
            const int s = static_cast<int>(i % kDecStages);
            if (!mbar_wait_sleep(&full[s], (i / kDecStages) & 1)) {
                atomicOr(status, 1);
                return;
            }
            const unsigned char *st = smem + s * Cfg::kStage;
            float4 hv[kDecItems];
            float x[kDecItems], dl[kDecItems], zz[kDecItems];
#pragma unroll
            for (int k = 0; k < kDecItems; ++k) {
                hv[k] = *reinterpret_cast<const float4 *>(st + Cfg::oH + (cc[k] * N + n0) * 4);
                x[k] = lds_widen<IO>(st + Cfg::oU, cc[k]);
                dl[k] = lds_widen<IO>(st + Cfg::oDl, cc[k]) + bias[k];
                zz[k] = z ? lds_widen<IO>(st + Cfg::oZ, cc[k]) : 0.0f;
            }
            const float4 bv = lds_widen4<IO>(st + Cfg::oB + n0 * ES);
            const float4 cv = lds_widen4<IO>(st + Cfg::oC + n0 * ES);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);  // the stage's contents are in registers

            const int64_t row = b * D + d0;
            float *hf_t = h_final ? h_final + row * N + n0 : nullptr;  // this tile's rows, this thread's states
            IO *y_t = y + row;
            const f2 bp[2] = {pack2(bv.x, bv.y), pack2(bv.z, bv.w)};
            const f2 cp[2] = {pack2(cv.x, cv.y), pack2(cv.z, cv.w)};
#pragma unroll
            for (int k = 0; k < kDecItems; ++k) {
                float dv = dl[k];
                if (softplus) dv = softplus_f(dv);
                const f2 dd = splat2(dv);
                const f2 hin[2] = {pack2(hv[k].x, hv[k].y), pack2(hv[k].z, hv[k].w)};
                f2 hn[2];
                f2 ya = splat2(0.0f);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    float e0, e1;
                    const f2 e = mul2(dd, a2[k][p]);
                    unpack2(e, e0, e1);
                    const f2 abar = pack2(ex2(e0), ex2(e1));
                    f2 bu;
                    if constexpr (ZOH) {
                        float i0, i1;
                        unpack2(ia[k][p], i0, i1);
                        bu = mul2(zoh_coef_pair(dd, e, ia[k][p], pack2(-i0, -i1), abar), mul2(bp[p], splat2(x[k])));
                    } else {
                        bu = mul2(bp[p], splat2(dv * x[k]));
                    }
                    hn[p] = fma2(abar, hin[p], bu);
                    ya = fma2(cp[p], hn[p], ya);
                }
                float y0, y1;
                unpack2(ya, y0, y1);
                float yv = y0 + y1;
#pragma unroll
                for (int o = 1; o < LPC; o <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
                const int c = c0 + k * CPS;
                if (c < td) {
                    if (h_final != nullptr) {
                        float a0, a1, a2v, a3;
                        unpack2(hn[0], a0, a1);
                        unpack2(hn[1], a2v, a3);
                        *reinterpret_cast<float4 *>(hf_t + c * N) = make_float4(a0, a1, a2v, a3);
                    }
                    if (g == 0) {
                        if (z != nullptr) yv *= silu_f(zz[k]);
                        Io<IO>::st(y_t + c, yv);
                    }
                }
            }
        }
    }
}

}  // namespace sscan
