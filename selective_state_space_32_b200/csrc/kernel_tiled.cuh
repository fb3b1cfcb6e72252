// kernel_tiled.cuh -- the persistent chained forward with block-wide tiles, for
// shapes whose per-warp tile rows are narrower than an L2 fill.
//
// The chained kernel (kernel_chained.cuh) gives every warp its own chain and its
// own TMA stages.  At N = 64 a warp holds 4 to 8 channels, so a warp's u / delta
// row is 8-16 bytes of bf16: the 64-byte L2 fill around it belongs to chains that
// other warps reach at other times, and the inputs cross HBM several times.
// Here the unit of the schedule is a block-chain: one batch row b and the
// CPB = WPC * CPW consecutive channels of the block's WPC consumer warps, over
// the whole sequence ("Selective State-Space Models (Mamba) and Hardware-Aware
// Scans", section 2: the recurrence is sequential in time, channels are
// independent).  All consumer warps of a block walk the same block-chain
// segments in lockstep, so one TMA box of CPB channels per token row feeds them
// all (a whole row of sectors), and the stage's B and C tiles ([T][N], the same
// for every channel of row b) are loaded and widened once per block instead of
// once per warp.
//
// Roles.  Warp WPC (the producer) issues the 2-D TMA loads of every stage
// (u, delta [T][CPB]; B, C [T][N]) on a "full" mbarrier, waits for each stage to
// land, copies its B and C tiles into padded fp32 rows (bf16 widened) and
// arrives on the stage's "ready" mbarrier.  Consumer warp w runs channels
// w*CPW .. w*CPW + CPW - 1 of the block-chain with the lane layout of the
// chained kernel (LPC lanes per channel, NL states per lane in registers), and
// arrives on the stage's "empty" mbarrier (WPC arrivals release the slot).
//
// Schedule.  The block-chains are laid end to end (chain-major, then time) and
// cut into equal segments, one per block (the chained kernel's Segment walk
// with one worker per block).  A block-chain cut between two blocks hands its
// state over per warp: the earlier block runs the head first and publishes each
// warp's state at the cut; the later block runs the tail last, each warp
// reading its own part (epoch-tagged flags, bounded waits; the grid is launched
// cooperatively, so every block is resident).  Arithmetic per state update is
// the chained kernel's (discretize / advance, kernel_chained.cuh), except the
// bf16-precision ZOH coefficient of warps whose every A is <= 0, which takes a
// select-free form (discretize_zoh_min).
#pragma once

#include <type_traits>

#include "kernel_chained.cuh"

namespace sscan {

template <class IO, int N_, int NL_, int T_, int STAGES_, int WPC_>
struct TiledCfg {
    static constexpr int N = N_, NL = NL_, T = T_, STAGES = STAGES_, WPC = WPC_;
    static constexpr int LPC = N / NL;       // lanes per channel
    static constexpr int CPW = 32 / LPC;     // channels per consumer warp
    static constexpr int CPB = WPC * CPW;    // channels per block-chain (tile row)
    static constexpr int NP = NL / 2;        // packed pairs per lane
    // tokens per discretize group: bounded by the registers of WPC + 1 warps per SM
    static constexpr int G = NL >= 16 ? 2 : (WPC >= 16 ? 4 : 8);   // Euler (Abar ahead)
    static constexpr int GZ = NL >= 16 ? 2 : (WPC >= 16 ? 2 : 4);  // ZOH
    static constexpr int ES = sizeof(IO);
    static constexpr int kU = T * CPB * ES;  // one u or delta tile
    static constexpr int kB = T * N * ES;    // one B or C tile
    static constexpr int kStage = 2 * kU + 2 * kB;
    static constexpr int kStageF = kStage + kU;  // fused calls with a gate: z [T][CPB] too
    // fp32 B, C rows: each lane group's NL values followed by 4 floats of padding
    // when a warp reads 4 or more groups (groups 32 or 64 bytes apart would share banks)
    static constexpr int kPadG = LPC >= 4 ? 4 : 0;
    static constexpr int kRowW = N + LPC * kPadG;
    static constexpr int kConv = 2 * T * kRowW * 4;
    static constexpr int kStageA = (kStageF + 127) / 128 * 128;
    static constexpr int kSlot = kStageA + (kConv + 127) / 128 * 128;
    // fused calls: each consumer warp's delta' = softplus(delta + bias) and silu(z), fp32 [T][CPW]
    static constexpr int kDsf = T * CPW * 4;
    static constexpr int kScratch = WPC * 2 * kDsf;
    static constexpr int kBars = (3 * STAGES * 8 + 127) / 128 * 128;  // full, ready, empty
    static constexpr int kSmem = STAGES * kSlot + kScratch + kBars;
    static constexpr int kThreads = (WPC + 1) * 32;
    static_assert(LPC >= 1 && LPC <= 8 && N % NL == 0 && NL % 4 == 0, "bad split");
    static_assert(CPB * ES % 16 == 0 && N * ES % 16 == 0, "TMA rows must be 16-byte multiples");
    static_assert(CPB <= 256 && T <= 256, "TMA box dimensions");
    static_assert(kU % 128 == 0 && kB % 128 == 0, "tile alignment");
    static_assert(NL % (16 / ES) == 0, "a 16-byte chunk of B or C never spans two lane groups");
    static_assert(T % 8 == 0, "token groups divide a stage");
    static_assert(T * CPW % 32 == 0 && kScratch % 128 == 0, "fused tile entries per lane");
};

// Exact ZOH at bf16 precision without a select, for a warp whose every A is <= 0:
// the coefficient (Abar - 1)/A as min(Abar (1/A) - (1 + 2^-21)/A, delta).  The bias
// 2^-21/|A| exceeds the error of Abar (ex2.approx, about 2^-22) and makes the first
// form an upper bound of the exact c = delta phi(delta A) in the signed sense, and
// c <= delta for A <= 0, so where the first form has lost its relative accuracy
// (|delta A| below about 2^-10) the min takes delta (relative error |delta A|/2),
// and elsewhere the first form (relative error 2^-21 / |delta A|): at most about
// 2^-11, against the 2^-9 rounding of a bf16 output.  A = 0: 1/A is infinite, the
// first form NaN, and fminf returns delta, the exact limit.
template <int NP>
__device__ __forceinline__ void discretize_zoh_min(f2 (&ab)[NP], f2 (&bu)[NP], const f2 (&A2)[NP],
                                                   const f2 (&iA)[NP], float x, float dl, const float *Bs) {
    const f2 dd = splat2(dl), xx = splat2(x);
    const f2 kBias = splat2(-(1.0f + 0x1p-21f));
#pragma unroll
    for (int i = 0; i < NP / 2; ++i) {
        const float4 bv = reinterpret_cast<const float4 *>(Bs)[i];
        const f2 b01 = pack2(bv.x, bv.y), b23 = pack2(bv.z, bv.w);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int p = 2 * i + q;
            float e0, e1;
            unpack2(mul2(dd, A2[p]), e0, e1);
            ab[p] = pack2(ex2(e0), ex2(e1));
            float c0, c1;
            unpack2(fma2(ab[p], iA[p], mul2(iA[p], kBias)), c0, c1);
            bu[p] = mul2(pack2(fminf(c0, dl), fminf(c1, dl)), mul2(q ? b23 : b01, xx));
        }
    }
}

// The producer warp: TMA issue in the block's processing order, at most STAGES
// stages ahead of the consumers, and the fp32 copy of every landed stage's B and
// C tiles.  All lanes walk the same stages; lane 0 issues the copies.  On a wait
// that gives up it records the failure and waits (bounded) for its copies in
// flight before returning.
template <class IO, class Cfg, bool FUSED>
__device__ __forceinline__ void tiled_produce(const CUtensorMap *tm_u, const CUtensorMap *tm_d,
                                              const CUtensorMap *tm_b, const CUtensorMap *tm_c,
                                              const CUtensorMap *tm_z, const ChainedParams &P,
                                              unsigned char *smem, uint64_t *full, uint64_t *ready,
                                              uint64_t *empty, int lane) {
    constexpr int T = Cfg::T, STAGES = Cfg::STAGES, N = Cfg::N, NL = Cfg::NL, CPB = Cfg::CPB;
    if (lane == 0) {
        tma_prefetch_desc(tm_u);
        tma_prefetch_desc(tm_d);
        tma_prefetch_desc(tm_b);
        tma_prefetch_desc(tm_c);
        if (FUSED && P.z != nullptr) tma_prefetch_desc(tm_z);
    }
    const bool zt = FUSED && P.z != nullptr;  // the gate tile is loaded with each stage
    const int64_t L = P.L;
    const Segment sg(static_cast<int64_t>(blockIdx.x), P);
    // issue walk (ki, ti, tei, r_i) and widening walk (kw, tw, tew, r_w) over the same stages
    int64_t ki = 0, ti = 0, tei = 0, kw = 0, tw = 0, tew = 0, r_i = 0, r_w = 0;
    int xi = 0, rowi = 0;
    auto begin_issue = [&]() {
        int64_t c;
        sg.part(ki, L, c, ti, tei);
        const int64_t b = c / P.chains_per_row;
        xi = static_cast<int>((c - b * P.chains_per_row) * CPB);
        rowi = static_cast<int>(b * L);
    };
    auto begin_widen = [&]() {
        int64_t c;
        sg.part(kw, L, c, tw, tew);
    };
    if (sg.n_parts > 0) {
        begin_issue();
        begin_widen();
    }
    bool failed = false;
    while (kw < sg.n_parts) {
        // issue ahead: up to STAGES stages beyond the one to widen, as slots are released
        while (ki < sg.n_parts && r_i < r_w + STAGES) {
            const int s = static_cast<int>(r_i % STAGES);
            if (r_i >= STAGES) {
                const uint32_t par = static_cast<uint32_t>((r_i / STAGES - 1) & 1);
                bool freed;
                if (r_i == r_w)
                    freed = mbar_wait(&empty[s], par);  // nothing else to do until it is free
                else
                    freed = mbar_test_wait(&empty[s], par);
                freed = __all_sync(0xffffffffu, freed);
                if (!freed) {
                    if (r_i == r_w) failed = true;
                    break;
                }
            }
            if (lane == 0) {
                unsigned char *slot = smem + s * Cfg::kSlot;
                uint64_t *bar = &full[s];
                const int yrow = rowi + static_cast<int>(ti);
                mbar_expect_tx(bar, zt ? Cfg::kStageF : Cfg::kStage);
                tma_load_2d(slot, tm_u, xi, yrow, bar);
                tma_load_2d(slot + Cfg::kU, tm_d, xi, yrow, bar);
                tma_load_2d(slot + 2 * Cfg::kU, tm_b, 0, yrow, bar);
                tma_load_2d(slot + 2 * Cfg::kU + Cfg::kB, tm_c, 0, yrow, bar);
                if (zt) tma_load_2d(slot + Cfg::kStage, tm_z, xi, yrow, bar);
            }
            __syncwarp();
            ++r_i;
            ti += T;
            if (ti >= tei && ++ki < sg.n_parts) begin_issue();
        }
        if (failed) break;
        // widen the oldest issued stage once it has landed
        const int s = static_cast<int>(r_w % STAGES);
        const bool landed = __all_sync(0xffffffffu, mbar_wait(&full[s], static_cast<uint32_t>((r_w / STAGES) & 1)));
        if (!landed) {
            failed = true;
            break;
        }
        unsigned char *slot = smem + s * Cfg::kSlot;
        float *convB = reinterpret_cast<float *>(slot + Cfg::kStageA);
        float *convC = convB + T * Cfg::kRowW;
        constexpr int kPer = 16 / Cfg::ES;        // values per 16-byte chunk
        constexpr int kChunks = T * N / kPer;
        const uint4 *rb = reinterpret_cast<const uint4 *>(slot + 2 * Cfg::kU);
        const uint4 *rc = reinterpret_cast<const uint4 *>(slot + 2 * Cfg::kU + Cfg::kB);
#pragma unroll 4
        for (int q = lane; q < kChunks; q += 32) {
            const uint4 vb = rb[q], vc = rc[q];
            const int col = (kPer * q) % N, row = (kPer * q) / N;
            const int dst = row * Cfg::kRowW + (col / NL) * (NL + Cfg::kPadG) + col % NL;
            float4 *ob = reinterpret_cast<float4 *>(convB + dst);
            float4 *oc = reinterpret_cast<float4 *>(convC + dst);
            if constexpr (Cfg::ES == 4) {
                ob[0] = make_float4(__uint_as_float(vb.x), __uint_as_float(vb.y), __uint_as_float(vb.z),
                                    __uint_as_float(vb.w));
                oc[0] = make_float4(__uint_as_float(vc.x), __uint_as_float(vc.y), __uint_as_float(vc.z),
                                    __uint_as_float(vc.w));
            } else {
                ob[0] = make_float4(__uint_as_float(vb.x << 16), __uint_as_float(vb.x & 0xffff0000u),
                                    __uint_as_float(vb.y << 16), __uint_as_float(vb.y & 0xffff0000u));
                ob[1] = make_float4(__uint_as_float(vb.z << 16), __uint_as_float(vb.z & 0xffff0000u),
                                    __uint_as_float(vb.w << 16), __uint_as_float(vb.w & 0xffff0000u));
                oc[0] = make_float4(__uint_as_float(vc.x << 16), __uint_as_float(vc.x & 0xffff0000u),
                                    __uint_as_float(vc.y << 16), __uint_as_float(vc.y & 0xffff0000u));
                oc[1] = make_float4(__uint_as_float(vc.z << 16), __uint_as_float(vc.z & 0xffff0000u),
                                    __uint_as_float(vc.w << 16), __uint_as_float(vc.w & 0xffff0000u));
            }
        }
        __syncwarp();  // every lane's rows before the arrive (release)
        if (lane == 0) mbar_arrive(&ready[s]);
        ++r_w;
        tw += T;
        if (tw >= tew && ++kw < sg.n_parts) begin_widen();
    }
    if (failed) {
        if (lane == 0) atomicOr(P.status, 4);
        // copies issued but not yet seen landing: wait for them (bounded) before leaving
        for (int64_t r = r_w; r < r_i; ++r) mbar_wait(&full[r % STAGES], static_cast<uint32_t>((r / STAGES) & 1));
        __syncwarp();
    }
}

// Fused calls: a consumer warp's delta' = softplus(delta + bias) (or delta + bias)
// and silu(z) (or 1) for its CPW channels of one stage, from the block's
// [T][CPB] tiles into its own fp32 [T][CPW] tiles.  Entry i = lane + 32k is
// token i / CPW, channel i % CPW = lane % CPW (32 is a multiple of CPW).
template <class IO, class Cfg>
__device__ __forceinline__ void tiled_fused_tile(const IO *dsm, const IO *zs, float *dsf, float *gsf, int ch0,
                                                 float biasv, bool softplus, bool gate, int lane) {
    constexpr int CPW = Cfg::CPW, CPB = Cfg::CPB, kPer = Cfg::T * CPW / 32;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = lane + 32 * k;
        const int src = (i / CPW) * CPB + ch0 + i % CPW;
        const float v = Io<IO>::widen(dsm[src]) + biasv;
        dsf[i] = softplus ? softplus_f(v) : v;
        gsf[i] = gate ? silu_f(Io<IO>::widen(zs[src])) : 1.0f;
    }
}

template <class IO, class Cfg, bool ZOH, bool FUSED>
__global__ void __launch_bounds__(Cfg::kThreads, 1)
sscan_tiled_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_d,
                   const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                   const __grid_constant__ CUtensorMap tm_z, const ChainedParams P) {
    constexpr int N = Cfg::N, NL = Cfg::NL, T = Cfg::T, STAGES = Cfg::STAGES, WPC = Cfg::WPC;
    constexpr int LPC = Cfg::LPC, CPW = Cfg::CPW, CPB = Cfg::CPB, NP = Cfg::NP;
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * Cfg::kSlot + Cfg::kScratch);
    uint64_t *full = bars, *ready = bars + STAGES, *empty = bars + 2 * STAGES;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&ready[i], 1);
            mbar_init(&empty[i], WPC);
        }
        mbar_fence_init();
    }
    __syncthreads();  // the only block-wide barrier
    if (warp == WPC) {
        tiled_produce<IO, Cfg, FUSED>(&tm_u, &tm_d, &tm_b, &tm_c, &tm_z, P, smem, full, ready, empty, lane);
        return;
    }

    const int64_t L = P.L, D = P.D;
    const Segment seg(static_cast<int64_t>(blockIdx.x), P);
    if (seg.n_parts == 0) return;  // this block has no work
    const int cl = lane / LPC;   // channel within the warp
    const int g = lane % LPC;    // state group
    const int n0 = g * NL;
    const int ch = warp * CPW + cl;                   // channel within the block-chain
    const int gofs = g * (NL + Cfg::kPadG);           // this lane's group in a padded fp32 row
    constexpr int RS = Cfg::kRowW;
    constexpr int G = Cfg::G, GZ = Cfg::GZ;
    float *dsf = reinterpret_cast<float *>(smem + STAGES * Cfg::kSlot) + warp * 2 * (T * CPW);  // FUSED
    float *gsf = dsf + T * CPW;
    const bool gate = FUSED && P.z != nullptr;
    int64_t consumed = 0;
    bool failed = false;

    for (int64_t k = 0; k < seg.n_parts && !failed; ++k) {
        int64_t c, ts, te;
        seg.part(k, L, c, ts, te);
        const int64_t b = c / P.chains_per_row, cg = c - b * P.chains_per_row;
        const int64_t d = cg * CPB + ch;
        const bool valid = d < D;
        const int64_t dcl = valid ? d : D - 1;
        const int64_t wc = c * WPC + warp;  // this warp's share of the block-chain: carry index

        f2 A2[NP], A1[NP], iA[NP], h[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const float a0 = __ldg(P.A + dcl * N + n0 + 2 * p);
            const float a1 = __ldg(P.A + dcl * N + n0 + 2 * p + 1);
            A2[p] = pack2(static_cast<float>(static_cast<double>(a0) * 1.4426950408889634),
                          static_cast<float>(static_cast<double>(a1) * 1.4426950408889634));
            iA[p] = ZOH ? pack2(1.0f / a0, 1.0f / a1) : splat2(0.0f);
            A1[p] = splat2(0.0f);  // -1/A: fp32 I/O only (bf16-precision ZOH takes it from 1/A)
        }
        if (ZOH && Cfg::ES == 4) {
#pragma unroll
            for (int p = 0; p < NP; ++p) A1[p] = neg2(iA[p]);
        }

        if (ts == 0) {
            if (P.h0 != nullptr) {
                const float *src = P.h0 + (b * D + dcl) * N + n0;
#pragma unroll
                for (int p = 0; p < NP; p += 2) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + 2 * p);
                    h[p] = pack2(v.x, v.y);
                    h[p + 1] = pack2(v.z, v.w);
                }
            } else {
#pragma unroll
                for (int p = 0; p < NP; ++p) h[p] = splat2(0.0f);
            }
        } else {
            // the state at the cut, published by this warp's counterpart in the previous block
            int bad = 0;
            if (lane == 0) {
                const unsigned long long want = P.epoch_hi | static_cast<unsigned long long>(ts);
                uint32_t it = 0;
                while (ld_acquire_u64(P.flags + wc) != want) {
                    if (++it > (kSpinLimit >> 2)) {
                        bad = 1;
                        atomicOr(P.status, 1);
                        break;
                    }
                    __nanosleep(128);
                }
            }
            bad = __shfl_sync(0xffffffffu, bad, 0);
            __syncwarp();  // order every lane's reads after lane 0's acquire
            const float *src = P.carry + (wc * 32 + lane) * NL;
#pragma unroll
            for (int p = 0; p < NP; p += 2) {
                const float4 v = bad ? make_float4(0.f, 0.f, 0.f, 0.f)
                                     : __ldcg(reinterpret_cast<const float4 *>(src + 2 * p));
                h[p] = pack2(v.x, v.y);
                h[p + 1] = pack2(v.z, v.w);
            }
        }

        // lanes past the last channel store into their own sink slot (unconditional stores)
        IO *ybase = valid ? static_cast<IO *>(P.y) + b * L * D + d
                          : reinterpret_cast<IO *>(static_cast<float *>(P.ysink) +
                                                   (static_cast<int64_t>(blockIdx.x) * WPC + warp) * 32 + lane);
        const int64_t ystr = valid ? D : 0;
        float biasv = 0.0f;
        if (FUSED && P.delta_bias != nullptr) {
            const int64_t dp = cg * CPB + warp * CPW + lane % CPW;
            biasv = dp < D ? __ldg(P.delta_bias + dp) : 0.0f;
        }
        // bf16 ZOH: the select-free coefficient when every A of the warp is <= 0 (decided
        // once per part, the same for every stage: two copies of the stage loop)
        bool a_nonpos = true;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float x0, x1;
            unpack2(A2[p], x0, x1);
            a_nonpos = a_nonpos && x0 <= 0.0f && x1 <= 0.0f;
        }
        a_nonpos = __all_sync(0xffffffffu, a_nonpos);
        auto stages = [&](auto min_tag) {
        constexpr bool MINF = decltype(min_tag)::value;
        for (int64_t t0 = ts; t0 < te; t0 += T) {
            const int s = static_cast<int>(consumed % STAGES);
            const uint32_t par = static_cast<uint32_t>((consumed / STAGES) & 1);
            // the TMA tiles of the stage, then the producer's fp32 B and C rows
            const bool landed = mbar_wait(&full[s], par) && mbar_wait(&ready[s], par);
            if (!__all_sync(0xffffffffu, landed)) {
                if (lane == 0) atomicOr(P.status, 2);
                failed = true;
                break;
            }
            const unsigned char *slot = smem + s * Cfg::kSlot;
            const IO *us = reinterpret_cast<const IO *>(slot) + ch;
            const IO *dsm = reinterpret_cast<const IO *>(slot + Cfg::kU) + ch;
            const float *Bs = reinterpret_cast<const float *>(slot + Cfg::kStageA) + gofs;
            const float *Cs = Bs + T * RS;
            if (FUSED) {
                tiled_fused_tile<IO, Cfg>(reinterpret_cast<const IO *>(slot + Cfg::kU),
                                          reinterpret_cast<const IO *>(slot + Cfg::kStage), dsf, gsf, warp * CPW,
                                          biasv, P.softplus != 0, gate, lane);
                __syncwarp();
            }
            auto delta_at = [&](int j1) { return FUSED ? dsf[j1 * CPW + cl] : Io<IO>::widen(dsm[j1 * CPB]); };
            auto x_at = [&](int j1) { return Io<IO>::widen(us[j1 * CPB]); };
            const int nsteps = static_cast<int>(te - t0 < T ? te - t0 : T);
            IO *yp = ybase + t0 * ystr;
            int j = 0;
            auto group_euler = [&](int j0) {
                constexpr int KEEP = G / LPC > 0 ? G / LPC : 1;
                const bool g_store = LPC <= G || (g & (LPC / G - 1)) == 0;
                f2 ab[G][NP];
                float duv[G];
#pragma unroll
                for (int q = 0; q < G; ++q) {
                    const float x = x_at(j0 + q);
                    const float dl = delta_at(j0 + q);
                    duv[q] = dl * x;
                    discretize_abar<NP, false, 0>(ab[q], A2, 0.0f, dl);
                }
                float yv[G];
#pragma unroll
                for (int q = 0; q < G; ++q)
                    yv[q] = advance_euler<NP>(h, ab[q], duv[q], Bs + (j0 + q) * RS, Cs + (j0 + q) * RS);
                const int base = reduce_scatter<LPC, G>(yv, g);
                if (FUSED) {
#pragma unroll
                    for (int q = 0; q < KEEP; ++q) yv[q] *= gsf[(j0 + base + q) * CPW + cl];
                }
                if (g_store) {
#pragma unroll
                    for (int q = 0; q < KEEP; ++q) Io<IO>::st(yp + (j0 + base + q) * ystr, yv[q]);
                }
            };
            auto group_zoh = [&](int j0) {  // Abar and Bbar u ahead, then the updates
                constexpr int KEEP = GZ / LPC > 0 ? GZ / LPC : 1;
                const bool g_store = LPC <= GZ || (g & (LPC / GZ - 1)) == 0;
                f2 ab[GZ][NP], bu[GZ][NP];
#pragma unroll
                for (int q = 0; q < GZ; ++q) {
                    if constexpr (MINF)
                        discretize_zoh_min<NP>(ab[q], bu[q], A2, iA, x_at(j0 + q), delta_at(j0 + q),
                                               Bs + (j0 + q) * RS);
                    else
                        discretize<NP, true, false, 0, Cfg::ES == 2, true>(ab[q], bu[q], A2, A1, iA, 0.0f,
                                                                     x_at(j0 + q), delta_at(j0 + q),
                                                                     Bs + (j0 + q) * RS);
                }
                float yv[GZ];
#pragma unroll
                for (int q = 0; q < GZ; ++q) yv[q] = advance<NP>(h, ab[q], bu[q], Cs + (j0 + q) * RS);
                const int base = reduce_scatter<LPC, GZ>(yv, g);
                if (FUSED) {
#pragma unroll
                    for (int q = 0; q < KEEP; ++q) yv[q] *= gsf[(j0 + base + q) * CPW + cl];
                }
                if (g_store) {
#pragma unroll
                    for (int q = 0; q < KEEP; ++q) Io<IO>::st(yp + (j0 + base + q) * ystr, yv[q]);
                }
            };
            if (!ZOH) {
                if (nsteps == T) {
#pragma unroll
                    for (int j0 = 0; j0 < T; j0 += G) group_euler(j0);
                    j = T;
                } else {
                    for (; j + G <= nsteps; j += G) group_euler(j);
                }
            } else {
                if (nsteps == T) {
#pragma unroll
                    for (int j0 = 0; j0 < T; j0 += GZ) group_zoh(j0);
                    j = T;
                } else {
                    for (; j + GZ <= nsteps; j += GZ) group_zoh(j);
                }
            }
            for (; j < nsteps; ++j) {  // ragged end of a part
                f2 ab[NP], bu[NP];
                const float x = x_at(j);
                const float dl = delta_at(j);
                discretize<NP, ZOH, false, 0, Cfg::ES == 2, true>(ab, bu, A2, A1, iA, 0.0f, x, dl, Bs + j * RS);
                float yv = advance<NP>(h, ab, bu, Cs + j * RS);
#pragma unroll
                for (int o = 1; o < LPC; o <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
                if (FUSED) yv *= gsf[j * CPW + cl];
                if (g == 0) Io<IO>::st(yp + j * ystr, yv);
            }
            // every lane is done reading the slot: release it to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            ++consumed;
        }
        };
        if (ZOH && Cfg::ES == 2 && a_nonpos)
            stages(std::true_type());
        else
            stages(std::false_type());
        if (failed) break;

        if (te < L && !P.drop_publish) {
            // publish this warp's state at the cut for its counterpart in the next block
            float *dst = P.carry + (wc * 32 + lane) * NL;
#pragma unroll
            for (int p = 0; p < NP; p += 2) {
                float a, bq, cq, e;
                unpack2(h[p], a, bq);
                unpack2(h[p + 1], cq, e);
                __stcg(reinterpret_cast<float4 *>(dst + 2 * p), make_float4(a, bq, cq, e));
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(P.flags + wc, P.epoch_hi | static_cast<unsigned long long>(te));
        } else if (te == L && P.h_final != nullptr && valid) {
            float *dst = P.h_final + (b * D + d) * N + n0;
#pragma unroll
            for (int p = 0; p < NP; p += 2) {
                float a, bq, cq, e;
                unpack2(h[p], a, bq);
                unpack2(h[p + 1], cq, e);
                *reinterpret_cast<float4 *>(dst + 2 * p) = make_float4(a, bq, cq, e);
            }
        }
    }
}

}  // namespace sscan
