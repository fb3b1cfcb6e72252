// kernel_chained.cuh -- persistent selective-scan forward with TMA-staged
// inputs and a static, exactly balanced schedule of chain segments.
//
// Work unit.  A "chain" is one batch row b and CPW = 32/LPC consecutive
// channels over the whole sequence; one warp runs a chain with lane
// (c, g) = (channel c of the chain, state group g) owning NL = N/LPC states of
// channel c in registers.  The recurrence h = Abar*h + Bbar u is sequential in
// time ("Selective State-Space Models (Mamba) and Hardware-Aware Scans",
// section 2), so a chain's steps must run in order; chains are independent.
//
// Schedule.  The B*ceil(D/CPW) chains are laid end to end (chain-major, then
// time) and cut into W segments of S = ceil(chains*L / W) chain-steps on
// average, one per warp of a persistent grid, so every warp does the same
// number of state updates (up to a small shift that evens out finishing times:
// the warps sharing an SM sub-partition with the producer run S - 3x steps, the
// others S + x).  With segments >= L a chain is cut at most once, between two
// consecutive warps: the earlier warp runs the chain's head (from t = 0) FIRST
// and publishes the state at the cut; the later warp runs its own head and
// whole chains first and the chain's tail LAST, after reading that state.
// This is "scan within a block, carry the block's state forward"
// ("tm_ssm_selective", section "What it costs at inference, and on a CPU"):
// the carry is the exact state, so there is no fix-up pass and no exponent is
// computed twice.  The wait cannot deadlock (the grid is launched
// cooperatively, so all warps are resident, and a warp only waits for a head
// that its predecessor runs before anything else) and is bounded anyway.
//
// Pipeline.  Each consumer warp owns a ring of STAGES shared-memory stages of T
// tokens: u and delta tiles [T][CPW] and B, C tiles [T][N].  A producer warp per
// block loads them with 2-D TMA (no multicast) on a "full" mbarrier per slot and
// refills a slot after its consumer releases it on an "empty" mbarrier, so the
// (slow) TMA issue never stalls a consumer and the compute loop only reads
// shared memory.  bf16 B/C tiles are widened once per stage by the warp.
//
// Arithmetic per state update: Abar = 2^(delta*A*log2 e) on the MUFU pipe (an
// option, POLY, moves a quarter of the states to the FMA pipe, exp2_fma_pair;
// measured slower with one consumer warp per SM sub-partition, so off by
// default); Bbar u (Euler or exact ZOH), h = Abar*h + Bbar u and y += C*h on
// packed f32x2 instructions.  y is reduced over the LPC lanes of a channel
// with shuffles and stored directly (lanes past the last channel store into a
// sink slot, so no store is guarded).
//
// Fused kernels (FUSED): each stage also carries the gate tile z, and the
// stage's delta' = softplus(delta + bias) and silu(z) are computed once per
// tile entry into fp32 tiles (fused_tile) -- by a helper warp per consumer on
// the same SM sub-partition for 4-consumer shapes (help), else by the
// consumer itself; y is stored multiplied by silu(z).
#pragma once

#include "device_utils.cuh"

namespace sscan {

struct ChainedParams {
    const float *A;                // [D][N]
    const float *h0;               // [B][D][N] or null
    void *y;                       // [B][L][D]
    float *h_final;                // [B][D][N] or null
    float *carry;                  // [chains][32][NL] state at a cut
    unsigned long long *flags;     // [chains] (epoch << 32) | cut position
    int *status;                   // device status word
    unsigned long long epoch_hi;   // this launch's epoch << 32
    int64_t L, D;
    int64_t chains_per_row;        // ceil(D / CPW)
    int64_t chains;                // B * chains_per_row
    int64_t seg;                   // chain-steps per warp (S), on average
    int64_t seg_shift;             // x: warps j = 0 mod 4 of a block run S - 3x steps, the others S + x
    int wpc;                       // consumer warps per block
    // split mode (chains cut into several pieces that are scanned concurrently)
    const void *delta;             // [B][L][D], read again by the fix-up
    const void *Cm;                // [B][L][N], read again by the fix-up
    float *rec_h;                  // [chains][max_pieces][32][NL] local end state of a piece
    float *rec_s;                  // [chains][max_pieces][32] sum of delta over the piece
    int *rec_mono;                 // [chains][max_pieces] delta >= 0 over the piece and A <= 0
    unsigned long long *rec_flags; // [chains][max_pieces] (epoch << 32) | 1 once published
    int64_t max_pieces;
    void *ysink;                   // [warps][32] 4-byte slots: y stores of lanes past the last channel
    // fused prologue / epilogue (FUSED kernels only)
    const float *delta_bias;       // [D] added to delta, or null
    const void *z;                 // [B][L][D] gate: y *= silu(z), or null
    int softplus;                  // delta <- softplus(delta + bias)
    int drop_publish;              // failure-detection tests only: heads never publish their carry
};

template <class IO, int N_, int NL_, int T_, int STAGES_, int WPC_>
struct ChainedCfg {
    static constexpr int N = N_, NL = NL_, T = T_, STAGES = STAGES_, WPC = WPC_;
    static constexpr int LPC = N / NL;      // lanes per channel
    static constexpr int CPW = 32 / LPC;    // channels per warp (chain width)
    static constexpr int NP = NL / 2;       // packed pairs per lane
    // tokens per discretize group: as many as registers allow (more independent
// exponentials per warp measured faster); ZOH keeps more per-token values live
    static constexpr int G = NL >= 16 ? 2 : (T < 16 ? T : 16);
    static constexpr int GZ = NL >= 16 ? 2 : 8;
    static constexpr int ES = sizeof(IO);
    static constexpr int kU = T * CPW * ES;                 // one u or delta tile
    static constexpr int kB = T * N * ES;                   // one B or C tile
    static constexpr int kStage = 2 * kU + 2 * kB;          // TMA bytes per stage
    // widened B, C (bf16 I/O): fp32 rows of N states; with 16 states per lane each
    // lane's group is followed by 4 floats of padding, so that the LPC groups a warp
    // reads with one 16-byte load per lane fall on disjoint banks (unpadded, groups
    // 64 bytes apart pair up on the same banks)
    static constexpr int kPadG = (ES == 2 && NL >= 16) ? 4 : 0;
    static constexpr int kRowW = N + LPC * kPadG;             // floats per widened row
    static constexpr int kConv = ES == 2 ? 2 * T * kRowW * 4 : 0;
    static constexpr int kWarp = ((STAGES * kStage + kConv) + 127) / 128 * 128;
    static constexpr int kBars = (2 * WPC * STAGES * 8 + 127) / 128 * 128;  // full + empty per slot
    static constexpr int kSmem = WPC * kWarp + kBars;
    // fused kernels: each stage also holds the gate tile z [T][CPW]; two fp32 [T][CPW]
    // tiles hold the stage's delta after bias / softplus and silu(z)
    static constexpr int kStageF = kStage + kU;
    static constexpr int kDsf = T * CPW * 4;
    static constexpr int kWarpF = ((STAGES * kStageF + kConv + 2 * kDsf) + 127) / 128 * 128;
    static constexpr int kSmemF = WPC * kWarpF + kBars;
    // fused kernels of 4-consumer shapes: one helper warp per consumer, on the same SM
    // sub-partition, computes those two tiles for every stage into a ring of STAGES
    // (the consumer's MUFU pipe is idle during its state updates; a ninth warp fits the
    // register file at the consumer's register count)
    static constexpr int kWarpH = ((STAGES * kStageF + kConv + 2 * STAGES * kDsf) + 127) / 128 * 128;
    static constexpr int kBarsH = (3 * WPC * STAGES * 8 + 127) / 128 * 128;  // full, empty, ready
    static constexpr int kSmemH = WPC * kWarpH + kBarsH;
    static constexpr int kThreadsH = (2 * WPC + 1) * 32;
    static constexpr bool kHelp = WPC == 4 && kSmemH <= 227 * 1024;
    static constexpr int kThreads = (WPC + 1) * 32;  // WPC consumer warps + 1 producer warp
    static_assert(LPC >= 1 && LPC <= 8 && N % NL == 0 && NL % 4 == 0, "bad split");
    static_assert(CPW * ES % 16 == 0 && N * ES % 16 == 0, "TMA rows must be 16-byte multiples");
    static_assert(kU % 128 == 0 && kB % 128 == 0, "tile alignment");
    static_assert(ES == 4 || (T * N) % 256 == 0, "bf16 widening splits the tile in 8-value chunks");
};

// Discretize one token for one lane: Abar and Bbar u for the lane's NL states.
// Independent of the state, so a group of tokens is discretized ahead of the
// (sequential) state updates and the MUFU latency overlaps them.  PAR is the
// token's parity; it selects which pairs take 2^x on the FMA pipe (a quarter
// of all pairs across two tokens).  COARSE (bf16 I/O) takes the ZOH coefficient
// to bf16 precision (zoh_coef_pair_bf16; CFMA: its fused multiply-add form).
template <int NP, bool ZOH, bool POLY, int PAR, bool COARSE = false, bool CFMA = false>
__device__ __forceinline__ void discretize(f2 (&ab)[NP], f2 (&bu)[NP], const f2 (&A2)[NP], const f2 (&nA)[NP],
                                           const f2 (&iA)[NP], float cap, float x, float dl,
                                           const float *Bs) {
    const f2 dd = splat2(dl);
    f2 du2, xx, ddc;
    if (ZOH)
        xx = splat2(x);
    else
        du2 = splat2(dl * x);
    if (POLY) ddc = splat2(fminf(dl, cap));
#pragma unroll
    for (int i = 0; i < NP / 2; ++i) {
        const float4 bv = reinterpret_cast<const float4 *>(Bs)[i];
        const f2 b01 = pack2(bv.x, bv.y), b23 = pack2(bv.z, bv.w);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int p = 2 * i + q;
            const f2 bp = q ? b23 : b01;
            const f2 e = mul2(dd, A2[p]);
            if (POLY && ((PAR * NP + p) % 4 == 3)) {
                ab[p] = exp2_fma_pair(ddc, A2[p]);
            } else {
                float e0, e1;
                unpack2(e, e0, e1);
                ab[p] = pack2(ex2(e0), ex2(e1));
            }
            if (ZOH && COARSE)  // no -1/A registers to keep
                bu[p] = mul2(zoh_coef_pair_bf16<CFMA>(dd, e, iA[p], ab[p]), mul2(bp, xx));
            else if (ZOH)
                bu[p] = mul2(zoh_coef_pair(dd, e, iA[p], nA[p], ab[p]), mul2(bp, xx));
            else
                bu[p] = mul2(bp, du2);
        }
    }
}

// The state update and readout of one token: h = Abar*h + Bbar u, partial y = C.h.
template <int NP>
__device__ __forceinline__ float advance(f2 (&h)[NP], const f2 (&ab)[NP], const f2 (&bu)[NP], const float *Cs) {
    f2 ya = splat2(0.0f);
#pragma unroll
    for (int i = 0; i < NP / 2; ++i) {
        const float4 cv = reinterpret_cast<const float4 *>(Cs)[i];
        h[2 * i] = fma2(ab[2 * i], h[2 * i], bu[2 * i]);
        ya = fma2(pack2(cv.x, cv.y), h[2 * i], ya);
        h[2 * i + 1] = fma2(ab[2 * i + 1], h[2 * i + 1], bu[2 * i + 1]);
        ya = fma2(pack2(cv.z, cv.w), h[2 * i + 1], ya);
    }
    float y0, y1;
    unpack2(ya, y0, y1);
    return y0 + y1;
}

// Euler path, split in two so that a longer run of tokens fits in registers:
// discretize_abar computes only Abar (the exponentials, independent of h) ...
template <int NP, bool POLY, int PAR>
__device__ __forceinline__ void discretize_abar(f2 (&ab)[NP], const f2 (&A2)[NP], float cap, float dl) {
    const f2 dd = splat2(dl);
    f2 ddc;
    if (POLY) ddc = splat2(fminf(dl, cap));
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        if (POLY && ((PAR * NP + p) % 4 == 3)) {
            ab[p] = exp2_fma_pair(ddc, A2[p]);
        } else {
            float e0, e1;
            unpack2(mul2(dd, A2[p]), e0, e1);
            ab[p] = pack2(ex2(e0), ex2(e1));
        }
    }
}

// ... and advance_euler forms Bbar u = B * (delta * u) while updating the state.
template <int NP>
__device__ __forceinline__ float advance_euler(f2 (&h)[NP], const f2 (&ab)[NP], float du, const float *Bs,
                                               const float *Cs) {
    const f2 du2 = splat2(du);
    f2 ya = splat2(0.0f);
#pragma unroll
    for (int i = 0; i < NP / 2; ++i) {
        const float4 bv = reinterpret_cast<const float4 *>(Bs)[i];
        const float4 cv = reinterpret_cast<const float4 *>(Cs)[i];
        h[2 * i] = fma2(ab[2 * i], h[2 * i], mul2(pack2(bv.x, bv.y), du2));
        ya = fma2(pack2(cv.x, cv.y), h[2 * i], ya);
        h[2 * i + 1] = fma2(ab[2 * i + 1], h[2 * i + 1], mul2(pack2(bv.z, bv.w), du2));
        ya = fma2(pack2(cv.z, cv.w), h[2 * i + 1], ya);
    }
    float y0, y1;
    unpack2(ya, y0, y1);
    return y0 + y1;
}

// Sum G per-token partial outputs over the LPC lanes of a channel and scatter
// the totals: afterwards this lane holds the full y of tokens
// base .. base + cnt - 1 in v[0 .. cnt), cnt = max(1, G / LPC).  Each level
// halves the token set a lane keeps and sends the other half to its partner.
template <int LPC, int G>
__device__ __forceinline__ int reduce_scatter(float (&v)[G], int g) {
    int base = 0;
#pragma unroll
    for (int m = LPC / 2, cnt = G; m >= 1; m >>= 1) {
        if (cnt >= 2) {
            const bool up = (g & m) != 0;
#pragma unroll
            for (int i = 0; i < cnt / 2; ++i) {
                const float send = up ? v[i] : v[i + cnt / 2];
                const float keep = up ? v[i + cnt / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
            if (up) base += cnt / 2;
            cnt /= 2;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
    return base;
}

// The chain-steps [q0, q1) of one warp's segment, as parts: [head of the last
// chain] [whole chains] [tail of the first chain], in that order of processing.
struct Segment {
    int64_t c_first, t_first, c_last, t_last, f_lo, n_full, n_parts;
    int n_head;
    bool single;
    // First chain-step of warp w: w*S shifted by x per heavier warp before it in its
    // block minus 3x per lighter one (a block's total stays WPC*S).
    static __device__ __forceinline__ int64_t start(int64_t w, const ChainedParams &P) {
        const int j = static_cast<int>(w % P.wpc);
        return w * P.seg + P.seg_shift * (j - 4 * ((j + 3) / 4));
    }
    __device__ __forceinline__ Segment(int64_t wk, const ChainedParams &P) {
        const int64_t L = P.L, Q = P.chains * L;
        const int64_t q0 = start(wk, P);
        if (q0 >= Q) {
            n_parts = 0;
            c_first = t_first = c_last = t_last = f_lo = n_full = 0;
            n_head = 0;
            single = true;
            return;
        }
        const int64_t q1e = start(wk + 1, P);
        const int64_t q1 = q1e < Q ? q1e : Q;
        c_first = q0 / L;
        t_first = q0 - c_first * L;
        c_last = (q1 - 1) / L;
        t_last = q1 - c_last * L;  // in [1, L]
        single = c_first == c_last;
        n_head = (!single && t_last < L) ? 1 : 0;
        const int n_tail = (!single && t_first > 0) ? 1 : 0;
        f_lo = t_first == 0 ? c_first : c_first + 1;
        const int64_t f_hi = t_last == L ? c_last : c_last - 1;
        n_full = single ? 0 : (f_hi >= f_lo ? f_hi - f_lo + 1 : 0);
        n_parts = single ? 1 : n_head + n_full + n_tail;
    }
    __device__ __forceinline__ void part(int64_t k, int64_t L, int64_t &c, int64_t &ts, int64_t &te) const {
        if (single) {
            c = c_first; ts = t_first; te = t_last;
        } else if (k < n_head) {
            c = c_last; ts = 0; te = t_last;
        } else if (k < n_head + n_full) {
            c = f_lo + (k - n_head); ts = 0; te = L;
        } else {
            c = c_first; ts = t_first; te = L;
        }
    }
};

// Split mode, second phase for one piece [ts, te) of chain c (ts > 0) that was
// scanned from a zero state.  Its carried-in state is the inclusive state of
// the previous pieces: h_in = sum_i (prod_{k>i} P_k) hloc_i over the earlier
// pieces i, where P_k = prod Abar over piece k = 2^(A*log2e * sum delta) (one
// exponent per state and piece).  The records are published at the end of
// every piece's local scan, so the look-back never waits for another fix-up.
// The exact output is y_t = y_local,t + C_t . z_t with z_t = Abar_t z_{t-1},
// z = h_in before ts; the loop stops once every |z| has fallen below
// 2^-40 max(1, |h_in|) and delta >= 0, A <= 0 over the piece guarantee that
// it can only shrink further ("Delta is a gate": large steps reset the state,
// "tm_ssm_selective").  The piece's final state is hloc + P_piece h_in.
template <class IO, class Cfg, bool FUSED>
__device__ __noinline__ void split_fixup(const ChainedParams &P, int64_t c, int64_t ts, int64_t te,
                                         int64_t wk, int lane) {
    constexpr int N = Cfg::N, NL = Cfg::NL, LPC = Cfg::LPC, CPW = Cfg::CPW, NP = Cfg::NP;
    constexpr int FB = NL <= 8 ? 8 : 4;  // tokens per block of loads
    const int64_t L = P.L, D = P.D;
    const int cl = lane / LPC, g = lane % LPC, n0 = g * NL;
    const int64_t b = c / P.chains_per_row, cw = c - b * P.chains_per_row;
    const int64_t d = cw * CPW + cl;
    const bool valid = d < D;
    const int64_t dcl = valid ? d : D - 1;
    f2 A2[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const float a0 = __ldg(P.A + dcl * N + n0 + 2 * p), a1 = __ldg(P.A + dcl * N + n0 + 2 * p + 1);
        A2[p] = pack2(static_cast<float>(static_cast<double>(a0) * 1.4426950408889634),
                      static_cast<float>(static_cast<double>(a1) * 1.4426950408889634));
    }
    const int64_t jp = wk - (c * L) / P.seg;  // index of this piece within chain c
    f2 acc_h[NP], acc_p[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        acc_h[p] = splat2(0.0f);
        acc_p[p] = splat2(1.0f);
    }
    for (int64_t i = jp - 1; i >= 0; --i) {
        const int64_t r = c * P.max_pieces + i;
        int bad = 0;
        if (lane == 0) {
            uint32_t it = 0;
            while (ld_acquire_u64(P.rec_flags + r) != (P.epoch_hi | 1ull)) {
                if (++it > (kSpinLimit >> 2)) {
                    bad = 1;
                    atomicOr(P.status, 1);
                    break;
                }
                __nanosleep(128);
            }
        }
        bad = __shfl_sync(0xffffffffu, bad, 0);
        __syncwarp();
        if (bad) break;
        const float sd = __ldcg(P.rec_s + r * 32 + lane);
        const float *src = P.rec_h + (r * 32 + lane) * NL;
        bool all_zero = true;
#pragma unroll
        for (int p = 0; p < NP; p += 2) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + 2 * p));
            const f2 hl[2] = {pack2(v.x, v.y), pack2(v.z, v.w)};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float e0, e1;
                unpack2(mul2(splat2(sd), A2[p + q]), e0, e1);
                acc_h[p + q] = fma2(acc_p[p + q], hl[q], acc_h[p + q]);
                acc_p[p + q] = mul2(acc_p[p + q], pack2(ex2(e0), ex2(e1)));
                float p0, p1;
                unpack2(acc_p[p + q], p0, p1);
                all_zero = all_zero && p0 == 0.0f && p1 == 0.0f;
            }
        }
        if (__all_sync(0xffffffffu, all_zero)) break;  // older pieces are multiplied by exact zeros
    }
    // this piece's own record: local end state, sum of delta, monotone flag
    const int64_t ro = c * P.max_pieces + jp;
    const bool mono = __ldcg(P.rec_mono + ro) != 0;
    float hmax = 0.0f;
    f2 z[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        z[p] = acc_h[p];
        float a, bq;
        unpack2(z[p], a, bq);
        hmax = fmaxf(hmax, fmaxf(fabsf(a), fabsf(bq)));
    }
    const float tau = ldexpf(fmaxf(1.0f, hmax), -40);
    const IO *dptr = static_cast<const IO *>(P.delta) + b * L * D + dcl;
    const IO *cptr = static_cast<const IO *>(P.Cm) + b * L * N + n0;
    IO *yptr = static_cast<IO *>(P.y) + b * L * D + dcl;
    const bool writer = valid && g == 0;
    // fused: the same delta transform as the scan; the correction is gated like y
    const float biasv = (FUSED && P.delta_bias != nullptr) ? __ldg(P.delta_bias + dcl) : 0.0f;
    const bool gate = FUSED && P.z != nullptr;
    const IO *zptr = gate ? static_cast<const IO *>(P.z) + b * L * D + dcl : nullptr;
    for (int64_t tb = ts; tb < te; tb += FB) {
        const int nb = static_cast<int>(te - tb < FB ? te - tb : FB);
        float dl[FB], yo[FB], gq[FB];
        f2 cv[FB][NP];
#pragma unroll
        for (int q = 0; q < FB; ++q) {
            const int64_t t = tb + (q < nb ? q : 0);
            dl[q] = Io<IO>::widen(Io<IO>::ld(dptr + t * D));
            if (FUSED) {
                dl[q] += biasv;
                if (P.softplus) dl[q] = softplus_f(dl[q]);
            }
            Io<IO>::template ld_pairs<NP>(cptr + t * N, cv[q]);
            yo[q] = writer ? Io<IO>::widen(__ldcg(yptr + t * D)) : 0.0f;
            gq[q] = (gate && writer) ? silu_f(Io<IO>::widen(Io<IO>::ld(zptr + t * D))) : 1.0f;
        }
#pragma unroll
        for (int q = 0; q < FB; ++q) {
            if (q < nb) {
                f2 ya = splat2(0.0f);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    float e0, e1;
                    unpack2(mul2(splat2(dl[q]), A2[p]), e0, e1);
                    z[p] = mul2(pack2(ex2(e0), ex2(e1)), z[p]);
                    ya = fma2(cv[q][p], z[p], ya);
                }
                float y0, y1;
                unpack2(ya, y0, y1);
                float corr = y0 + y1;
#pragma unroll
                for (int o = 1; o < LPC; o <<= 1) corr += __shfl_xor_sync(0xffffffffu, corr, o);
                if (writer) Io<IO>::st(yptr + (tb + q) * D, yo[q] + corr * gq[q]);
            }
        }
        if (mono) {
            float zmax = 0.0f;
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                float a, bq;
                unpack2(z[p], a, bq);
                zmax = fmaxf(zmax, fmaxf(fabsf(a), fabsf(bq)));
            }
            if (__all_sync(0xffffffffu, zmax <= tau)) break;
        }
    }
    if (te == L && P.h_final != nullptr) {
        const float sd = __ldcg(P.rec_s + ro * 32 + lane);
        const float *src = P.rec_h + (ro * 32 + lane) * NL;
        float *dst = P.h_final + (b * D + d) * N + n0;
#pragma unroll
        for (int p = 0; p < NP; p += 2) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + 2 * p));
            float o[4];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float e0, e1;
                unpack2(mul2(splat2(sd), A2[p + q]), e0, e1);
                float h0v, h1v;
                unpack2(acc_h[p + q], h0v, h1v);
                o[2 * q] = (q ? v.z : v.x) + ex2(e0) * h0v;
                o[2 * q + 1] = (q ? v.w : v.y) + ex2(e1) * h1v;
            }
            if (valid) *reinterpret_cast<float4 *>(dst + 2 * p) = make_float4(o[0], o[1], o[2], o[3]);
        }
    }
}

// The fused per-stage transform of one [T][CPW] tile: delta' = softplus(delta + bias)
// (or delta + bias) and silu(z) (or 1) in fp32, lane-strided entries (entry i is
// channel i % CPW, the same for every entry of a lane since 32 is a multiple of CPW).
// A fixed trip count keeps the independent exponentials in flight together.
template <class IO, class Cfg>
__device__ __forceinline__ void fused_tile(const IO *dsm, const IO *zs, float *dsf, float *gsf, float biasv,
                                           bool softplus, bool gate, int lane) {
    constexpr int kPer = Cfg::T * Cfg::CPW / 32;
    static_assert(Cfg::T * Cfg::CPW % 32 == 0, "tile entries per lane");
    if (softplus) {
#pragma unroll
        for (int k = 0; k < kPer; ++k)
            dsf[lane + 32 * k] = softplus_f(Io<IO>::widen(dsm[lane + 32 * k]) + biasv);
    } else {
#pragma unroll
        for (int k = 0; k < kPer; ++k) dsf[lane + 32 * k] = Io<IO>::widen(dsm[lane + 32 * k]) + biasv;
    }
    if (gate) {
#pragma unroll
        for (int k = 0; k < kPer; ++k) gsf[lane + 32 * k] = silu_f(Io<IO>::widen(zs[lane + 32 * k]));
    } else {
#pragma unroll
        for (int k = 0; k < kPer; ++k) gsf[lane + 32 * k] = 1.0f;
    }
}

// Helper warp j (fused 4-consumer shapes): walks consumer j's stages in its order,
// waits for each stage to land, writes its transformed tiles into ring slot s and
// arrives on ready[s].  It never runs more than a ring ahead: a slot is refilled
// only after the consumer has released it.  Every wait is bounded.
template <class IO, class Cfg>
__device__ __forceinline__ void help(const ChainedParams &P, unsigned char *smem, uint64_t *full,
                                     uint64_t *ready, int j, int lane) {
    constexpr int T = Cfg::T, STAGES = Cfg::STAGES, CPW = Cfg::CPW;
    const int64_t L = P.L, D = P.D;
    const Segment sg(static_cast<int64_t>(blockIdx.x) * Cfg::WPC + j, P);
    unsigned char *wbase = smem + j * Cfg::kWarpH;
    float *dring = reinterpret_cast<float *>(wbase + STAGES * Cfg::kStageF + Cfg::kConv);
    float *gring = dring + STAGES * T * CPW;
    const bool gate = P.z != nullptr;
    int64_t r = 0;
    for (int64_t k = 0; k < sg.n_parts; ++k) {
        int64_t c, ts, te;
        sg.part(k, L, c, ts, te);
        const int64_t cw = c % P.chains_per_row;
        float biasv = 0.0f;
        if (P.delta_bias != nullptr) {
            const int64_t dp = cw * CPW + lane % CPW;
            biasv = dp < D ? __ldg(P.delta_bias + dp) : 0.0f;
        }
        for (int64_t t0 = ts; t0 < te; t0 += T, ++r) {
            const int s = static_cast<int>(r % STAGES);
            const bool landed = mbar_wait(&full[s], static_cast<uint32_t>((r / STAGES) & 1));
            if (!__all_sync(0xffffffffu, landed)) {
                if (lane == 0) atomicOr(P.status, 8);
                return;  // the consumer's bounded wait on ready[s] then gives up too
            }
            const IO *dsm = reinterpret_cast<const IO *>(wbase + s * Cfg::kStageF + Cfg::kU);
            const IO *zs = reinterpret_cast<const IO *>(wbase + s * Cfg::kStageF + Cfg::kStage);
            fused_tile<IO, Cfg>(dsm, zs, dring + s * T * CPW, gring + s * T * CPW, biasv, P.softplus != 0,
                                gate, lane);
            __syncwarp();  // every lane's tile entries before the arrive (release)
            if (lane == 0) mbar_arrive(&ready[s]);
        }
    }
}

// The producer: the block's last warp keeps every consumer warp's ring filled,
// lane i serving consumer warp i, all lanes in lockstep so that one TMA
// instruction issues the loads of every consumer that has a free slot (issuing
// a TMA load costs the issuing warp on the order of a hundred cycles).
// Consumer i's stages are loaded in its processing order (the same Segment walk
// the consumer does) into slot r % STAGES once the consumer has released the
// stage that used the slot before.  No lane ever blocks on one consumer (a
// consumer may be waiting for another warp's carry): each lane tests its
// consumer's barrier, and the warp backs off briefly when no lane could issue.
template <class IO, class Cfg, bool FUSED, int kRegion>
__device__ __forceinline__ void produce(const CUtensorMap *tm_u, const CUtensorMap *tm_d, const CUtensorMap *tm_b,
                                        const CUtensorMap *tm_c, const CUtensorMap *tm_z, const ChainedParams &P,
                                        unsigned char *smem,
                                        uint64_t *full, uint64_t *empty, int lane) {
    constexpr int WPC = Cfg::WPC, T = Cfg::T, STAGES = Cfg::STAGES, CPW = Cfg::CPW;
    if (lane == 0) {
        tma_prefetch_desc(tm_u);
        tma_prefetch_desc(tm_d);
        tma_prefetch_desc(tm_b);
        tma_prefetch_desc(tm_c);
        if (FUSED && P.z != nullptr) tma_prefetch_desc(tm_z);
    }
    constexpr int kStageB = FUSED ? Cfg::kStageF : Cfg::kStage;
    const bool zt = FUSED && P.z != nullptr;  // the gate tile is loaded with each stage
    const int64_t L = P.L;
    const int i = lane;  // the consumer this lane serves
    const Segment sg(static_cast<int64_t>(blockIdx.x) * WPC + (i < WPC ? i : 0), P);
    int64_t k = (i < WPC && sg.n_parts > 0) ? 0 : -1;
    int64_t te = 0, t = 0, r = 0;
    int x = 0, row = 0;
    auto begin_part = [&]() {
        int64_t c, ts;
        sg.part(k, L, c, ts, te);
        t = ts;
        const int64_t b = c / P.chains_per_row;
        x = static_cast<int>((c - b * P.chains_per_row) * CPW);
        row = static_cast<int>(b * L);
    };
    if (k >= 0) begin_part();
    unsigned char *ring = smem + (i < WPC ? i : 0) * kRegion;
    uint32_t idle = 0;
    while (__any_sync(0xffffffffu, k >= 0)) {
        const int s = static_cast<int>(r % STAGES);
        const bool ready = k >= 0 && (r < STAGES || mbar_test_wait(&empty[i * STAGES + s],
                                                                   static_cast<uint32_t>((r / STAGES - 1) & 1)));
        if (ready) {
            unsigned char *slot = ring + s * kStageB;
            uint64_t *bar = &full[i * STAGES + s];
            const int yrow = row + static_cast<int>(t);
            mbar_expect_tx(bar, zt ? Cfg::kStageF : Cfg::kStage);
            tma_load_2d(slot, tm_u, x, yrow, bar);
            tma_load_2d(slot + Cfg::kU, tm_d, x, yrow, bar);
            tma_load_2d(slot + 2 * Cfg::kU, tm_b, 0, yrow, bar);
            tma_load_2d(slot + 2 * Cfg::kU + Cfg::kB, tm_c, 0, yrow, bar);
            if (zt) tma_load_2d(slot + Cfg::kStage, tm_z, x, yrow, bar);
            ++r;
            t += T;
            if (t >= te) {
                if (++k < sg.n_parts)
                    begin_part();
                else
                    k = -1;
            }
        }
        if (__any_sync(0xffffffffu, ready)) {
            idle = 0;
        } else {
            if (++idle > (kSpinLimit << 2)) {  // consumers stopped releasing slots
                if (lane == 0) atomicOr(P.status, 4);
                return;
            }
            __nanosleep(64);
        }
    }
}

template <class IO, class Cfg, bool ZOH, bool POLY, bool SPLIT, bool FUSED>
__global__ void __launch_bounds__((FUSED && Cfg::kHelp) ? Cfg::kThreadsH : Cfg::kThreads, 1)
sscan_chained_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_d,
                     const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_z, const ChainedParams P) {
    constexpr int N = Cfg::N, NL = Cfg::NL, T = Cfg::T, STAGES = Cfg::STAGES;
    constexpr int LPC = Cfg::LPC, CPW = Cfg::CPW, NP = Cfg::NP;
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool HELP = FUSED && Cfg::kHelp;  // helper warps compute the fused tiles
    constexpr int kWarpB = HELP ? Cfg::kWarpH : (FUSED ? Cfg::kWarpF : Cfg::kWarp);  // one consumer's region
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::WPC * kWarpB);
    if (threadIdx.x == 0) {
        for (int i = 0; i < (HELP ? 3 : 2) * Cfg::WPC * STAGES; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    __syncthreads();  // the only block-wide barrier
    if (warp == (HELP ? 2 * Cfg::WPC : Cfg::WPC)) {
        produce<IO, Cfg, FUSED, kWarpB>(&tm_u, &tm_d, &tm_b, &tm_c, &tm_z, P, smem, bars,
                                        bars + Cfg::WPC * STAGES, lane);
        return;
    }
    if (HELP && warp >= Cfg::WPC) {
        const int j = warp - Cfg::WPC;
        help<IO, Cfg>(P, smem, bars + j * STAGES, bars + (2 * Cfg::WPC + j) * STAGES, j, lane);
        return;
    }
    constexpr int kStageB = FUSED ? Cfg::kStageF : Cfg::kStage;  // bytes of one stage
    unsigned char *wbase = smem + warp * kWarpB;
    float *convB = reinterpret_cast<float *>(wbase + STAGES * kStageB);
    float *convC = convB + T * Cfg::kRowW;
    float *dsf0 = reinterpret_cast<float *>(wbase + STAGES * kStageB + Cfg::kConv);  // FUSED: delta'
    float *gsf0 = dsf0 + (HELP ? STAGES : 1) * T * CPW;                               // FUSED: silu(z)
    uint64_t *full = bars + warp * STAGES;
    uint64_t *empty = bars + (Cfg::WPC + warp) * STAGES;
    uint64_t *ready = bars + (2 * Cfg::WPC + warp) * STAGES;  // HELP only

    const int64_t L = P.L, D = P.D;
    const int64_t wk = static_cast<int64_t>(blockIdx.x) * Cfg::WPC + warp;  // this warp's segment
    const Segment seg(wk, P);
    if (seg.n_parts == 0) return;  // this warp has no work
    const int64_t n_parts = seg.n_parts;
    auto part = [&](int64_t k, int64_t &c, int64_t &ts, int64_t &te) { seg.part(k, L, c, ts, te); };

    auto tile_u = [&](int s) { return reinterpret_cast<IO *>(wbase + s * kStageB); };
    auto tile_d = [&](int s) { return reinterpret_cast<IO *>(wbase + s * kStageB + Cfg::kU); };
    auto tile_b = [&](int s) { return reinterpret_cast<IO *>(wbase + s * kStageB + 2 * Cfg::kU); };
    auto tile_c = [&](int s) {
        return reinterpret_cast<IO *>(wbase + s * kStageB + 2 * Cfg::kU + Cfg::kB);
    };
    auto tile_z = [&](int s) { return reinterpret_cast<IO *>(wbase + s * kStageB + Cfg::kStage); };

    const int cl = lane / LPC;   // channel within the chain
    const int g = lane % LPC;    // state group
    const int n0 = g * NL;
    // B, C tiles: row stride and this lane's group offset (TMA tiles for fp32 I/O,
    // padded widened tiles for bf16)
    constexpr int RS = Cfg::ES == 4 ? N : Cfg::kRowW;
    const int gofs = Cfg::ES == 4 ? n0 : g * (NL + Cfg::kPadG);
    int64_t consumed = 0;
    bool failed = false;

    for (int64_t k = 0; k < n_parts && !failed; ++k) {
        int64_t c, ts, te;
        part(k, c, ts, te);
        const int64_t b = c / P.chains_per_row, cw = c - b * P.chains_per_row;
        const int64_t d = cw * CPW + cl;
        const bool valid = d < D;
        const int64_t dcl = valid ? d : D - 1;

        f2 A2[NP], A1[NP], iA[NP], h[NP];
        float amax = 0.0f;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const float a0 = __ldg(P.A + dcl * N + n0 + 2 * p);
            const float a1 = __ldg(P.A + dcl * N + n0 + 2 * p + 1);
            A2[p] = pack2(static_cast<float>(static_cast<double>(a0) * 1.4426950408889634),
                          static_cast<float>(static_cast<double>(a1) * 1.4426950408889634));
            if (ZOH) {
                iA[p] = pack2(1.0f / a0, 1.0f / a1);
                A1[p] = pack2(-1.0f / a0, -1.0f / a1);  // -1/A for the ZOH coefficient
            }
            if (POLY && (p % 2 == 1)) {  // pairs that may take the FMA-pipe exponent
                float x0, x1;
                unpack2(A2[p], x0, x1);
                amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
            }
        }
        // |delta * A2| <= 125 on the FMA-pipe pairs keeps 2^x in the normal range;
        // clamping delta there changes nothing visible (2^-125 vs 0 in Abar).
        const float cap = amax > 0.0f ? 125.0f / amax : 3.0e38f;

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
        } else if (SPLIT) {
#pragma unroll
            for (int p = 0; p < NP; ++p) h[p] = splat2(0.0f);  // local scan; carried in later
        } else {
            // the state at the cut, published by the previous warp
            int bad = 0;
            if (lane == 0) {
                const unsigned long long want = P.epoch_hi | static_cast<unsigned long long>(ts);
                uint32_t it = 0;
                while (ld_acquire_u64(P.flags + c) != want) {
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
            const float *src = P.carry + (c * 32 + lane) * NL;
#pragma unroll
            for (int p = 0; p < NP; p += 2) {
                const float4 v = bad ? make_float4(0.f, 0.f, 0.f, 0.f)
                                     : __ldcg(reinterpret_cast<const float4 *>(src + 2 * p));
                h[p] = pack2(v.x, v.y);
                h[p + 1] = pack2(v.z, v.w);
            }
        }

        double dsum = 0.0;      // split mode: sum of delta over the part (for prod Abar)
        float dmin = 3.0e38f;   // split mode: smallest delta of the part
        // Lanes past the last channel (d >= D) store into their own sink slot
        // (stride 0) instead of skipping the store: the stores of a stage are then
        // unconditional, which measured faster than a per-lane guard.
        IO *ybase = valid ? static_cast<IO *>(P.y) + b * L * D + d
                          : reinterpret_cast<IO *>(static_cast<float *>(P.ysink) + wk * 32 + lane);
        const int64_t ystr = valid ? D : 0;
        // fused prologue: this lane transforms tile entries lane, lane + 32, ...,
        // all of channel lane % CPW of the chain (32 is a multiple of CPW)
        float biasv = 0.0f;
        if (FUSED && P.delta_bias != nullptr) {
            const int64_t dp = cw * CPW + lane % CPW;
            biasv = dp < D ? __ldg(P.delta_bias + dp) : 0.0f;
        }
        const bool gate = FUSED && P.z != nullptr;
        for (int64_t t0 = ts; t0 < te; t0 += T) {
            const int s = static_cast<int>(consumed % STAGES);
            const uint32_t par = static_cast<uint32_t>((consumed / STAGES) & 1);
            bool landed = mbar_wait(&full[s], par);
            if (HELP) landed = landed && mbar_wait(&ready[s], par);  // the helper's tiles of this stage
            if (!__all_sync(0xffffffffu, landed)) {
                if (lane == 0) atomicOr(P.status, 2);
                failed = true;
                break;
            }
            const IO *us = tile_u(s);
            const IO *dsm = tile_d(s);
            const float *Bs;
            const float *Cs;
            if (Cfg::ES == 4) {
                Bs = reinterpret_cast<const float *>(tile_b(s));
                Cs = reinterpret_cast<const float *>(tile_c(s));
            } else {
                // widen the stage's B and C tiles to fp32 once for all lanes (padded rows)
                constexpr int kChunks = T * N / 8;  // 8 bf16 per 16-byte chunk
                const uint4 *rb = reinterpret_cast<const uint4 *>(tile_b(s));
                const uint4 *rc = reinterpret_cast<const uint4 *>(tile_c(s));
#pragma unroll
                for (int q = lane; q < kChunks; q += 32) {
                    const uint4 vb = rb[q], vc = rc[q];
                    const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
                    const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w};
                    const int col = (8 * q) % N, row = (8 * q) / N;  // a chunk never spans two groups
                    const int dst = row * Cfg::kRowW + (col / NL) * (NL + Cfg::kPadG) + col % NL;
                    float4 *ob = reinterpret_cast<float4 *>(convB + dst);
                    float4 *oc = reinterpret_cast<float4 *>(convC + dst);
                    ob[0] = make_float4(__uint_as_float(wb[0] << 16), __uint_as_float(wb[0] & 0xffff0000u),
                                        __uint_as_float(wb[1] << 16), __uint_as_float(wb[1] & 0xffff0000u));
                    ob[1] = make_float4(__uint_as_float(wb[2] << 16), __uint_as_float(wb[2] & 0xffff0000u),
                                        __uint_as_float(wb[3] << 16), __uint_as_float(wb[3] & 0xffff0000u));
                    oc[0] = make_float4(__uint_as_float(wc[0] << 16), __uint_as_float(wc[0] & 0xffff0000u),
                                        __uint_as_float(wc[1] << 16), __uint_as_float(wc[1] & 0xffff0000u));
                    oc[1] = make_float4(__uint_as_float(wc[2] << 16), __uint_as_float(wc[2] & 0xffff0000u),
                                        __uint_as_float(wc[3] << 16), __uint_as_float(wc[3] & 0xffff0000u));
                }
                __syncwarp();
                Bs = convB;
                Cs = convC;
            }
            // fused tiles of this stage: the helper's ring slot, or computed here
            const float *dsf = HELP ? dsf0 + s * T * CPW : dsf0;
            const float *gsf = HELP ? gsf0 + s * T * CPW : gsf0;
            if (FUSED && !HELP) {
                fused_tile<IO, Cfg>(dsm, tile_z(s), dsf0, gsf0, biasv, P.softplus != 0, gate, lane);
                __syncwarp();
            }
            auto delta_at = [&](int idx) { return FUSED ? dsf[idx] : Io<IO>::widen(dsm[idx]); };
            const int nsteps = static_cast<int>(te - t0 < T ? te - t0 : T);
            IO *yp = ybase + t0 * ystr;
            int j = 0;
            float ssum = 0.0f;  // split mode: this stage's share of dsum
            // Groups of G tokens: discretize the whole group first (independent of h),
            // then its sequential state updates, then one reduce-scatter of the G
            // partial outputs over the channel's lanes, so every lane stores.
            constexpr int G = Cfg::G;
            constexpr int GZ = Cfg::GZ;
            constexpr int KEEP = G / LPC > 0 ? G / LPC : 1;
            const bool g_store = LPC <= G || (g & (LPC / G - 1)) == 0;
            auto group_euler = [&](int j0) {
                f2 ab[G][NP];
                float duv[G];
#pragma unroll
                for (int q = 0; q < G; ++q) {
                    const float x = Io<IO>::widen(us[(j0 + q) * CPW + cl]);
                    const float dl = delta_at((j0 + q) * CPW + cl);
                    if (SPLIT) {
                        ssum += dl;
                        dmin = fminf(dmin, dl);
                    }
                    duv[q] = dl * x;
                    if (q & 1)
                        discretize_abar<NP, POLY, 1>(ab[q], A2, cap, dl);
                    else
                        discretize_abar<NP, POLY, 0>(ab[q], A2, cap, dl);
                }
                float yv[G];
#pragma unroll
                for (int q = 0; q < G; ++q)
                    yv[q] = advance_euler<NP>(h, ab[q], duv[q], Bs + (j0 + q) * RS + gofs, Cs + (j0 + q) * RS + gofs);
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
            auto group = [&](int j0) {  // ZOH: Abar and the ZOH coefficient per token
                constexpr int G = GZ;
                constexpr int KEEP = G / LPC > 0 ? G / LPC : 1;
                const bool g_store = LPC <= G || (g & (LPC / G - 1)) == 0;
                f2 ab[G][NP], bu[G][NP];
#pragma unroll
                for (int q = 0; q < G; ++q) {
                    const float x = Io<IO>::widen(us[(j0 + q) * CPW + cl]);
                    const float dl = delta_at((j0 + q) * CPW + cl);
                    if (SPLIT) {
                        ssum += dl;
                        dmin = fminf(dmin, dl);
                    }
                    if (q & 1)
                        discretize<NP, ZOH, POLY, 1, sizeof(IO) == 2>(ab[q], bu[q], A2, A1, iA, cap, x, dl, Bs + (j0 + q) * RS + gofs);
                    else
                        discretize<NP, ZOH, POLY, 0, sizeof(IO) == 2>(ab[q], bu[q], A2, A1, iA, cap, x, dl, Bs + (j0 + q) * RS + gofs);
                }
                float yv[G];
#pragma unroll
                for (int q = 0; q < G; ++q) yv[q] = advance<NP>(h, ab[q], bu[q], Cs + (j0 + q) * RS + gofs);
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
                    for (int j0 = 0; j0 < T; j0 += GZ) group(j0);
                    j = T;
                } else {
                    for (; j + GZ <= nsteps; j += GZ) group(j);
                }
            }
            for (; j < nsteps; ++j) {  // ragged end of a part
                f2 ab[NP], bu[NP];
                const float x = Io<IO>::widen(us[j * CPW + cl]);
                const float dl = delta_at(j * CPW + cl);
                if (SPLIT) {
                    ssum += dl;
                    dmin = fminf(dmin, dl);
                }
                discretize<NP, ZOH, POLY, 0, sizeof(IO) == 2>(ab, bu, A2, A1, iA, cap, x, dl, Bs + j * RS + gofs);
                float yv = advance<NP>(h, ab, bu, Cs + j * RS + gofs);
#pragma unroll
                for (int o = 1; o < LPC; o <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
                if (FUSED) yv *= gsf[j * CPW + cl];
                if (g == 0) Io<IO>::st(yp + j * ystr, yv);
            }
            if (SPLIT) dsum += static_cast<double>(ssum);
            // every lane is done reading the slot: release it to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            ++consumed;
        }
        if (failed) break;

        if (SPLIT && (ts > 0 || te < L)) {
            // publish this piece's record: local end state, sum of delta, monotone flag
            const int64_t r = c * P.max_pieces + (wk - (c * L) / P.seg);
            float *dst = P.rec_h + (r * 32 + lane) * NL;
            bool a_nonpos = true;
#pragma unroll
            for (int p = 0; p < NP; p += 2) {
                float a, bq, cq, e;
                unpack2(h[p], a, bq);
                unpack2(h[p + 1], cq, e);
                __stcg(reinterpret_cast<float4 *>(dst + 2 * p), make_float4(a, bq, cq, e));
            }
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                float x0, x1;
                unpack2(A2[p], x0, x1);
                a_nonpos = a_nonpos && x0 <= 0.0f && x1 <= 0.0f;
            }
            __stcg(P.rec_s + r * 32 + lane, static_cast<float>(dsum));
            const bool mono = __all_sync(0xffffffffu, a_nonpos && dmin >= 0.0f);
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                __stcg(P.rec_mono + r, mono ? 1 : 0);
                __threadfence();
                st_release_u64(P.rec_flags + r, P.epoch_hi | 1ull);
            }
        } else if (te < L && !P.drop_publish) {
            // publish the state at the cut for the warp that runs the rest of this chain
            float *dst = P.carry + (c * 32 + lane) * NL;
#pragma unroll
            for (int p = 0; p < NP; p += 2) {
                float a, bq, cq, e;
                unpack2(h[p], a, bq);
                unpack2(h[p + 1], cq, e);
                __stcg(reinterpret_cast<float4 *>(dst + 2 * p), make_float4(a, bq, cq, e));
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(P.flags + c, P.epoch_hi | static_cast<unsigned long long>(te));
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
    if (SPLIT && !failed) {
        __syncwarp();
        __threadfence_block();  // phase-1 y stores of every lane before the fix-up reads them
        for (int64_t k = 0; k < n_parts; ++k) {
            int64_t c, ts, te;
            part(k, c, ts, te);
            if (ts == 0) continue;
            split_fixup<IO, Cfg, FUSED>(P, c, ts, te, wk, lane);
        }
    }
    if (failed) {
        // drain loads that may still be in flight into this warp's ring (the producer
        // refills only released slots, so at most STAGES) before leaving; bounded
        if (lane == 0)
            for (int64_t i = consumed; i < consumed + STAGES; ++i)
                mbar_wait(&full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1));
        __syncwarp();
    }
}

}  // namespace sscan
