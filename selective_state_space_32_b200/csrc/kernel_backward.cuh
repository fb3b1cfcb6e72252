// kernel_backward.cuh -- backward pass of the selective scan (N = 16, 32, 64),
// with the fused prologue (delta' = softplus(delta + bias)) and gate
// (y' = y silu(z)) of the forward.
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
// and, for the fused layer, with s = delta_raw + bias and ys the scan's output:
//   dy_scan = dy silu(z),   dz = dy ys silu'(z),   silu'(z) = sig(z) (1 + z (1 - sig(z))),
//   ddelta_raw = ddelta' sig(s) (softplus' = sigmoid; 1 without softplus),
//   dbias[d] = sum over b and t of ddelta_raw.
//
// "Selective State-Space Models (Mamba) and Hardware-Aware Scans", section 3:
// the backward pass recomputes the states instead of reading a stored
// [B, L, D, N] tensor.  A forward pass keeps the state entering every chunk of
// KC tokens (a checkpoint per channel, in the workspace); the reverse sweep
// takes the chunks last to first, recomputes each chunk's states from its
// checkpoint into registers and runs the reverse recurrence over them.
//
// Mapping: each lane holds S consecutive states of one channel (S = 4, 2 or 1;
// LPC = N/S adjacent lanes per channel, CPW = 32/LPC channels per warp); a block
// of four warps covers CPB = 4 CPW consecutive channels of one batch row, and
// its warps walk the same chunks in the same order.  The reverse sweep over a
// chunk keeps every cross-lane sum out of the token loop: each lane writes its
// per-token partials (its states' share of du, ddelta and the gate's ys, and
// its contributions to dB and dC) to shared memory; after the chunk the block's
// threads reduce them data-parallel: du, ddelta (and dz) of each (token,
// channel) over the channel's LPC lanes, stored with coalesced writes, and dB,
// dC of each (token, four states) over the block's channels, stored in the
// block's own plane of a workspace array.  A second kernel sums the planes
// into dB and dC: the blocks of a batch row walk the same tokens at the same
// time, so atomics on dB and dC would all meet on the same few lines.  dA
// needs no cross-lane sum (one atomic per lane at the end).  The recompute
// keeps each token's Abar in registers for the reverse sweep.  When every row
// of the block's channels is 4-byte aligned (fp32, or bf16 with an even D) the
// chunk's inputs are staged in shared memory by cp.async one chunk ahead
// (STAGED: the L1 kept only about a third of the prefetched rows, and the
// reverse sweep waited on L2 for the rest).
#pragma once

#include "device_utils.cuh"

namespace sscan {

constexpr int kBwdWarps = 4;
constexpr int kBwdThreads = 32 * kBwdWarps;
constexpr int kChunk = 8;   // tokens per recomputed chunk

// channels a backward block covers with S states per lane
__host__ __device__ constexpr int bwd_block_channels_s(int N, int S) { return kBwdWarps * (32 / (N / S)); }
// channel padding of the checkpoint workspace: the widest block (S = 4), a
// multiple of every block width
__host__ __device__ constexpr int bwd_block_channels(int N) { return bwd_block_channels_s(N, 4); }
// blocks per SM the register budget is set for
template <int S> constexpr int bwd_min_blocks() { return S == 4 ? 3 : S == 2 ? 6 : 10; }

struct BwdParams {
    const void *u, *delta, *Bm, *Cm, *dy, *z;
    const float *A, *h0, *dhf, *bias;
    void *du, *ddelta, *dz;
    float *dA, *dB, *dC, *dh0, *dbias;
    float *ckpt;           // [B][Dpad][nchunks][N]
    float *part;           // [Dpad / CPB][B][L][2][N]: each block's dB, dC sums over its channels
    int64_t L, D, Dpad, nchunks;
    int softplus;
};

// S consecutive fp32 values (S = 4, 2, 1): load (read-only path or plain), store, atomic add
template <int S> __device__ __forceinline__ void ldv(const float *p, float (&v)[S], bool ro = true) {
    if constexpr (S == 4) {
        const float4 t = ro ? __ldg(reinterpret_cast<const float4 *>(p)) : *reinterpret_cast<const float4 *>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (S == 2) {
        const float2 t = ro ? __ldg(reinterpret_cast<const float2 *>(p)) : *reinterpret_cast<const float2 *>(p);
        v[0] = t.x; v[1] = t.y;
    } else {
        v[0] = ro ? __ldg(p) : *p;
    }
}
template <int S> __device__ __forceinline__ void stv(float *p, const float (&v)[S]) {
    if constexpr (S == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else if constexpr (S == 2) *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    else *p = v[0];
}
template <int S> __device__ __forceinline__ void atomic_addv(float *p, const float (&v)[S]) {
    if constexpr (S == 4) atomicAdd(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    else if constexpr (S == 2) atomicAdd(reinterpret_cast<float2 *>(p), make_float2(v[0], v[1]));
    else atomicAdd(p, v[0]);
}
// S consecutive values of a B or C row in the I/O type, widened to fp32
template <class IO, int S> __device__ __forceinline__ void ldv_io(const IO *p, float (&v)[S]) {
    if constexpr (sizeof(IO) == 4) {
        ldv<S>(reinterpret_cast<const float *>(p), v);
    } else if constexpr (S == 4) {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
        v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
    } else if constexpr (S == 2) {
        const uint32_t t = __ldg(reinterpret_cast<const unsigned int *>(p));
        v[0] = __uint_as_float(t << 16); v[1] = __uint_as_float(t & 0xffff0000u);
    } else {
        v[0] = __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short *>(p))) << 16);
    }
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void prefetch_l1(const void *p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// 4-byte asynchronous global -> shared copies (cp.async, no register staging)
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// S consecutive values of a staged B or C row (shared memory, I/O type), widened to fp32
template <class IO, int S> __device__ __forceinline__ void ldv_sm(const IO *p, float (&v)[S]) {
    static_assert(S == 4, "four states per lane");
    if constexpr (sizeof(IO) == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
        const uint2 t = *reinterpret_cast<const uint2 *>(p);
        v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
    }
}

// One buffer of a chunk's staged inputs, in the I/O type: delta, u, dy, z as
// [KC][CPB] (the block's channels fastest), B and C as [KC][N].
template <class IO, int N, int S>
struct BwdStage {
    static constexpr int CPB = bwd_block_channels_s(N, S), KC = kChunk;
    static constexpr int kDl = 0, kU = KC * CPB, kDy = 2 * KC * CPB, kZ = 3 * KC * CPB;
    static constexpr int kB = 4 * KC * CPB, kC = kB + KC * N;
    static constexpr int kElems = ((kC + KC * N) * int(sizeof(IO)) + 15) / 16 * 16 / int(sizeof(IO));
};
// dynamic shared memory of the backward kernel: the per-chunk partials, and two
// staging buffers when STAGED
// A row of the per-token dB / dC contributions ([channel][N] of one token): 16 floats of
// padding put consecutive tokens' rows on opposite halves of the banks, so the
// threads of the channel sums (one per token and four states) read 16-byte words
// spread over all 32 banks.
template <int S> constexpr int bwd_vrow() { return kBwdThreads * S + 16; }
template <class IO, int N, int S, bool STAGED>
constexpr int bwd_smem_bytes() {
    return (3 * kChunk * kBwdThreads + 2 * kChunk * bwd_vrow<S>()) * 4 +
           (STAGED ? 2 * BwdStage<IO, N, S>::kElems * int(sizeof(IO)) + 2 * kBwdThreads * S * 4 : 0);
}

// Sum of LPC consecutive floats in shared memory (16-byte aligned when LPC >= 4).
template <int LPC> __device__ __forceinline__ float sum_lanes(const float *p) {
    float acc = 0.0f;
    if constexpr (LPC >= 4) {
#pragma unroll
        for (int i = 0; i < LPC; i += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(p + i);
            acc += (v.x + v.y) + (v.z + v.w);
        }
    } else {
#pragma unroll
        for (int i = 0; i < LPC; ++i) acc += p[i];
    }
    return acc;
}

template <class IO, int N, int S, bool ZOH, bool FUSED, bool STAGED>
__global__ void __launch_bounds__(kBwdThreads, bwd_min_blocks<S>())
sscan_backward_kernel(const BwdParams P) {
    constexpr int LPC = N / S, CPW = 32 / LPC, CPB = kBwdWarps * CPW, KC = kChunk;
    // keep each token's Abar from the recompute for the reverse sweep (S = 4), or
    // take it again from the MUFU pipe there (fewer registers: S = 2, 1)
    constexpr bool kKeepAbar = S >= 4;
    constexpr int KA = kKeepAbar ? KC : 1;
    // per chunk: each lane's partials of du, ddelta (of the raw step) and the gate's ys per
    // token, and its S contributions to dB and dC per token ([k][channel][N] order)
    extern __shared__ __align__(16) unsigned char bsm[];
    float(*s_tok)[KC][kBwdThreads] = reinterpret_cast<float(*)[KC][kBwdThreads]>(bsm);
    constexpr int VR = bwd_vrow<S>();
    float(*s_vb)[VR] = reinterpret_cast<float(*)[VR]>(bsm + 3 * KC * kBwdThreads * 4);
    float(*s_vc)[VR] = s_vb + KC;
    // STAGED: two buffers of a chunk's inputs (BwdStage), filled by cp.async a chunk ahead
    using St = BwdStage<IO, N, S>;
    IO *stage_base = reinterpret_cast<IO *>(bsm + (3 * KC * kBwdThreads + 2 * KC * VR) * 4);
    // STAGED: two buffers of each lane's checkpoint for the reverse sweep, [buffer][thread][S]
    float *ck_stage = reinterpret_cast<float *>(stage_base + 2 * St::kElems);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cl = lane / LPC, g = lane % LPC, n0 = S * g;
    const int64_t L = P.L, D = P.D;
    const int64_t b = blockIdx.y;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * CPB + warp * CPW + cl;
    const bool valid = d < D;
    const int64_t dc = valid ? d : D - 1;  // past the last channel: compute on a real one, add nothing
    const IO *u = static_cast<const IO *>(P.u) + b * L * D + dc;
    const IO *dl_in = static_cast<const IO *>(P.delta) + b * L * D + dc;
    const IO *dyp = static_cast<const IO *>(P.dy) + b * L * D + dc;
    const IO *zp = FUSED && P.z ? static_cast<const IO *>(P.z) + b * L * D + dc : nullptr;
    const IO *Bp = static_cast<const IO *>(P.Bm) + b * L * N + n0;
    const IO *Cp = static_cast<const IO *>(P.Cm) + b * L * N + n0;
    float *ck = P.ckpt + (b * P.Dpad + d) * P.nchunks * N + n0;  // own slot even past D

    float a1[S], a2[S], ia[S];
    ldv<S>(P.A + dc * N + n0, a1);
#pragma unroll
    for (int i = 0; i < S; ++i) {
        a2[i] = static_cast<float>(static_cast<double>(a1[i]) * 1.4426950408889634);
        ia[i] = a1[i] != 0.0f ? 1.0f / a1[i] : 0.0f;
    }
    const float biasv = FUSED && P.bias ? __ldg(P.bias + dc) : 0.0f;
    // the step the scan uses, and (fused) softplus' = sigmoid of its argument, from the raw
    // delta of this lane's channel
    auto step_raw = [&](float raw, float &sig) {
        if (!FUSED) {
            sig = 1.0f;
            return raw;
        }
        const float s = raw + biasv;
        if (!P.softplus) {
            sig = 1.0f;
            return s;
        }
        sig = 1.0f / (1.0f + ex2(-s * 1.4426950408889634f));
        return softplus_f(s);
    };
    // beta and its derivatives for state i
    auto coefs = [&](int i, float dl, float abar, float Bn, float &beta, float &dbdl, float &dbda, float &dbdb) {
        if (!ZOH) {
            beta = dl * Bn; dbdl = Bn; dbda = 0.0f; dbdb = dl;
        } else if (a1[i] != 0.0f) {
            const float z = dl * a1[i];
            // (e^z - 1)/A: the small-|z| series keeps the relative accuracy of e^z - 1
            const float em1 = fabsf(z) < 0.25f ? z * (1.0f + z * (0.5f + z * (1.0f / 6.0f + z * (1.0f / 24.0f + z * (1.0f / 120.0f)))))
                                              : abar - 1.0f;
            dbdb = em1 * ia[i];
            beta = dbdb * Bn;
            dbdl = abar * Bn;
            // (delta abar A - (abar - 1)) / A^2 = delta^2 sum_{k>=2} z^(k-2) (k-1)/k!: the series
            // for |z| < 1 (terms to k = 10, truncation < 5e-7 relative), where the direct
            // form cancels; the direct form beyond
            const float ser = 0.5f + z * (1.0f / 3.0f + z * (0.125f + z * (1.0f / 30.0f + z * (1.0f / 144.0f +
                              z * (1.0f / 840.0f + z * (1.0f / 5760.0f + z * (1.0f / 45360.0f + z * (1.0f / 403200.0f))))))));
            const float num = fabsf(z) < 1.0f ? dl * dl * ser : (dl * abar * a1[i] - em1) * ia[i] * ia[i];
            dbda = Bn * num;
        } else {
            beta = dl * Bn; dbdl = Bn; dbda = 0.5f * dl * dl * Bn; dbdb = dl;
        }
    };

    // Unstaged: the rows a chunk reads (delta, u, dy, z of this warp's channels, B and C)
    // are prefetched ahead of it: into L1 one chunk ahead, into L2 two chunks ahead; lane
    // l takes token l % KC of row kind l / KC.  Prefetches are hints: addresses stay
    // inside the tensors (tokens clamped to the sequence).  (STAGED: the cp.async copies,
    // issued a whole chunk ahead, need none; the L2 prefetches measured 8 % slower there.)
    auto prefetch_chunk = [&](int64_t c, bool l1, bool with_dy) {
        if (c < 0 || c >= P.nchunks) return;
        const int64_t t = c * KC + lane % KC < L ? c * KC + lane % KC : L - 1;
        const void *a;
        switch (lane / KC) {
            case 0: a = dl_in + t * D; break;
            case 1: a = u + t * D; break;
            case 2: a = with_dy ? static_cast<const void *>(dyp + t * D) : static_cast<const void *>(Bp + t * N); break;
            default: a = (with_dy && zp) ? static_cast<const void *>(zp + t * D) : static_cast<const void *>(Cp + t * N); break;
        }
        if (l1) prefetch_l1(a); else prefetch_l2(a);
        if (with_dy && lane / KC >= 2) {  // B and C rows too
            const void *bc = lane / KC == 2 ? static_cast<const void *>(Bp + t * N) : static_cast<const void *>(Cp + t * N);
            if (l1) prefetch_l1(bc); else prefetch_l2(bc);
        }
    };

    // STAGED: chunk c's inputs into buffer `buf` with 4-byte cp.async copies, issued by
    // all threads (consecutive threads take consecutive words of a token row: coalesced),
    // one commit group per chunk; the caller waits and synchronises before reading.
    // Tokens past the sequence's end repeat its last token (unused); words past D read the
    // row's last word (D is a multiple of the elements per word), lanes there add nothing.
    constexpr int EPW = 4 / int(sizeof(IO));  // elements per 4-byte word
    const int64_t d0 = static_cast<int64_t>(blockIdx.x) * CPB;
    const IO *dl_row = static_cast<const IO *>(P.delta) + b * L * D;
    const IO *u_row = static_cast<const IO *>(P.u) + b * L * D;
    const IO *dy_row = static_cast<const IO *>(P.dy) + b * L * D;
    const IO *z_row = FUSED && P.z ? static_cast<const IO *>(P.z) + b * L * D : nullptr;
    const IO *B_row = static_cast<const IO *>(P.Bm) + b * L * N;
    const IO *C_row = static_cast<const IO *>(P.Cm) + b * L * N;
    auto issue = [&](int64_t c, int buf, bool rev) {
        IO *sb = stage_base + buf * St::kElems;
        const int64_t t0 = c * KC;
        const int nt = static_cast<int>(L - t0 < KC ? L - t0 : KC);
        constexpr int WPR = CPB / EPW;  // words per token row of the block's channels
        for (int e = threadIdx.x; e < KC * WPR; e += kBwdThreads) {
            const int k = e / WPR, w = e % WPR;
            const int64_t t = t0 + (k < nt ? k : nt - 1);
            const int64_t col = d0 + w * EPW < D ? d0 + w * EPW : D - EPW;
            const int64_t gi = t * D + col;
            const int si = k * CPB + w * EPW;
            cp_async4(sb + St::kDl + si, dl_row + gi);
            cp_async4(sb + St::kU + si, u_row + gi);
            if (rev) {
                cp_async4(sb + St::kDy + si, dy_row + gi);
                if (FUSED && z_row != nullptr) cp_async4(sb + St::kZ + si, z_row + gi);
            }
        }
        constexpr int WPN = N / EPW;
        for (int e = threadIdx.x; e < (rev ? 2 : 1) * KC * WPN; e += kBwdThreads) {
            const int which = e / (KC * WPN), r = e % (KC * WPN), k = r / WPN, w = r % WPN;
            const int64_t t = t0 + (k < nt ? k : nt - 1);
            cp_async4(sb + (which ? St::kC : St::kB) + k * N + w * EPW, (which ? C_row : B_row) + t * N + w * EPW);
        }
        if (rev) cp_async16(ck_stage + (buf * kBwdThreads + threadIdx.x) * S, ck + c * N);  // this lane's own
        cp_async_commit();
    };
    const int ch = warp * CPW + cl;  // this lane's channel within the block
    // token k of chunk c (token t): staged or straight from global memory
    auto in_dl = [&](const IO *sb, int k, int64_t t) {
        if constexpr (STAGED) return Io<IO>::widen(sb[St::kDl + k * CPB + ch]);
        else return Io<IO>::widen(Io<IO>::ld(dl_in + t * D));
    };
    auto in_x = [&](const IO *sb, int k, int64_t t) {
        if constexpr (STAGED) return Io<IO>::widen(sb[St::kU + k * CPB + ch]);
        else return Io<IO>::widen(Io<IO>::ld(u + t * D));
    };
    auto in_dy = [&](const IO *sb, int k, int64_t t) {
        if constexpr (STAGED) return Io<IO>::widen(sb[St::kDy + k * CPB + ch]);
        else return Io<IO>::widen(Io<IO>::ld(dyp + t * D));
    };
    auto in_z = [&](const IO *sb, int k, int64_t t) {
        if constexpr (STAGED) return Io<IO>::widen(sb[St::kZ + k * CPB + ch]);
        else return Io<IO>::widen(Io<IO>::ld(zp + t * D));
    };
    auto in_B = [&](const IO *sb, int k, int64_t t, float (&v)[S]) {
        if constexpr (STAGED) ldv_sm<IO, S>(sb + St::kB + k * N + n0, v);
        else ldv_io<IO, S>(Bp + t * N, v);
    };
    auto in_C = [&](const IO *sb, int k, int64_t t, float (&v)[S]) {
        if constexpr (STAGED) ldv_sm<IO, S>(sb + St::kC + k * N + n0, v);
        else ldv_io<IO, S>(Cp + t * N, v);
    };

    // ---- pass 1: forward, keeping the state entering every chunk ----
    // (chunk by chunk: a chunk's loads sit in one straight-line block, ahead of its
    // dependent updates).  States are held as packed pairs: the Euler updates run on
    // f32x2 instructions; ZOH works on the unpacked values.
    constexpr int SP = S / 2;  // state pairs per lane
    static_assert(S % 2 == 0, "states per lane come in pairs");
    f2 a2p[SP], a1p[SP];
#pragma unroll
    for (int p = 0; p < SP; ++p) {
        a2p[p] = pack2(a2[2 * p], a2[2 * p + 1]);
        a1p[p] = pack2(a1[2 * p], a1[2 * p + 1]);
    }
    auto abar_pair = [&](float dl, int p) {
        float e0, e1;
        unpack2(mul2(splat2(dl), a2p[p]), e0, e1);
        return pack2(ex2(e0), ex2(e1));
    };
    auto ld_pairs = [&](const float *src, f2 (&v)[SP], bool ro) {
        float t[S];
        ldv<S>(src, t, ro);
#pragma unroll
        for (int p = 0; p < SP; ++p) v[p] = pack2(t[2 * p], t[2 * p + 1]);
    };
    auto st_pairs = [&](float *dst, const f2 (&v)[SP]) {
        float t[S];
#pragma unroll
        for (int p = 0; p < SP; ++p) unpack2(v[p], t[2 * p], t[2 * p + 1]);
        stv<S>(dst, t);
    };
    // ZOH state update of one pair (scalar: the coefficient's series need the single values)
    auto zoh_step = [&](f2 hp, int p, float dl, float x, float b0, float b1, f2 &abp) {
        float h0v, h1v;
        unpack2(hp, h0v, h1v);
        const float ab0 = ex2(dl * a2[2 * p]), ab1 = ex2(dl * a2[2 * p + 1]);
        float beta0, beta1, q0, q1, q2;
        coefs(2 * p, dl, ab0, b0, beta0, q0, q1, q2);
        coefs(2 * p + 1, dl, ab1, b1, beta1, q0, q1, q2);
        abp = pack2(ab0, ab1);
        return pack2(fmaf(ab0, h0v, beta0 * x), fmaf(ab1, h1v, beta1 * x));
    };
    f2 h[SP];
    if (P.h0) {
        ld_pairs(P.h0 + (b * D + dc) * N + n0, h, false);
    } else {
#pragma unroll
        for (int p = 0; p < SP; ++p) h[p] = splat2(0.0f);
    }
    if constexpr (STAGED) {
        issue(0, 0, false);
    } else {
        prefetch_chunk(0, true, false);
        prefetch_chunk(1, false, false);
    }
    for (int64_t c = 0; c < P.nchunks; ++c) {
        const int64_t t0 = c * KC;
        const int nt = static_cast<int>(L - t0 < KC ? L - t0 : KC);
        const IO *sb = stage_base + (c & 1) * St::kElems;
        if constexpr (STAGED) {
            // chunk c has landed (this thread's copies), then every thread's; every thread is
            // also done with chunk c - 1, whose buffer takes chunk c + 1
            cp_async_wait_all();
            __syncthreads();
            if (c + 1 < P.nchunks) issue(c + 1, (c + 1) & 1, false);
        } else {
            prefetch_chunk(c + 1, true, false);
            prefetch_chunk(c + 2, false, false);
        }
        st_pairs(ck + c * N, h);
        float xs[KC], ds[KC], Bs[KC][S];
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int64_t t = t0 + (k < nt ? k : nt - 1);
            float sg;
            ds[k] = step_raw(in_dl(sb, k, t), sg);
            xs[k] = in_x(sb, k, t);
            in_B(sb, k, t, Bs[k]);
        }
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (k < nt) {
                const f2 dx2 = splat2(ds[k] * xs[k]);  // Euler: Bbar u = B (delta u)
#pragma unroll
                for (int p = 0; p < SP; ++p) {
                    if constexpr (ZOH) {
                        f2 abp;
                        h[p] = zoh_step(h[p], p, ds[k], xs[k], Bs[k][2 * p], Bs[k][2 * p + 1], abp);
                    } else {
                        h[p] = fma2(abar_pair(ds[k], p), h[p], mul2(pack2(Bs[k][2 * p], Bs[k][2 * p + 1]), dx2));
                    }
                }
            }
        }
    }

    // ---- pass 2: reverse sweep over the chunks ----
    f2 gs[SP], dacc[SP];
    if (P.dhf && valid) {
        ld_pairs(P.dhf + (b * D + dc) * N + n0, gs, false);
    } else {
#pragma unroll
        for (int p = 0; p < SP; ++p) gs[p] = splat2(0.0f);
    }
#pragma unroll
    for (int p = 0; p < SP; ++p) dacc[p] = splat2(0.0f);
    float dbias_acc = 0.0f;
    if constexpr (STAGED) {
        __syncthreads();  // every thread is done with the forward pass's buffers
        issue(P.nchunks - 1, (P.nchunks - 1) & 1, true);
    } else {
        prefetch_chunk(P.nchunks - 1, true, true);
    }
    for (int64_t c = P.nchunks - 1; c >= 0; --c) {
        const int64_t t0 = c * KC;
        const int nt = static_cast<int>(L - t0 < KC ? L - t0 : KC);
        const IO *sb = stage_base + (c & 1) * St::kElems;
        if constexpr (STAGED) {
            // chunk c has landed; every thread is done with chunk c + 1 (its buffer takes
            // chunk c - 1) and with the previous chunk's sums in shared memory
            cp_async_wait_all();
            __syncthreads();
            if (c >= 1) issue(c - 1, (c - 1) & 1, true);
        } else {
            prefetch_chunk(c - 1, true, true);
            prefetch_chunk(c - 2, false, true);
        }
        if (!STAGED && c >= 1) prefetch_l1(ck + (c - 1) * N);
        // recompute the chunk's states h_{t0 .. t0+nt-1} (and each token's Abar) from its checkpoint
        f2 h_in[SP], hk[KC][SP], ab[KA][SP];
        if constexpr (STAGED) {
            const float4 v = *reinterpret_cast<const float4 *>(ck_stage + ((c & 1) * kBwdThreads + threadIdx.x) * S);
            h_in[0] = pack2(v.x, v.y);
            h_in[1] = pack2(v.z, v.w);
        } else {
            ld_pairs(ck + c * N, h_in, false);
        }
        {
            f2 hc[SP];
#pragma unroll
            for (int p = 0; p < SP; ++p) hc[p] = h_in[p];
#pragma unroll
            for (int k = 0; k < KC; ++k) {
                const int64_t t = t0 + (k < nt ? k : nt - 1);  // loads need not wait behind work
                float sg;
                const float dl = step_raw(in_dl(sb, k, t), sg);
                const float x = in_x(sb, k, t);
                float Bv[S];
                in_B(sb, k, t, Bv);
                const f2 dx2 = splat2(dl * x);
#pragma unroll
                for (int p = 0; p < SP; ++p) {
                    f2 abp, hn;
                    if constexpr (ZOH) {
                        hn = zoh_step(hc[p], p, dl, x, Bv[2 * p], Bv[2 * p + 1], abp);
                    } else {
                        abp = abar_pair(dl, p);
                        hn = fma2(abp, hc[p], mul2(pack2(Bv[2 * p], Bv[2 * p + 1]), dx2));
                    }
                    if (k < nt) hc[p] = hn;
                    hk[k][p] = hc[p];
                    if constexpr (kKeepAbar) ab[k][p] = abp;
                }
            }
        }
        // reverse over the chunk's tokens
#pragma unroll
        for (int k = KC - 1; k >= 0; --k) {
            // the token's inputs are loaded unconditionally (past the sequence's end: its last
            // token, unused), so the loads need not wait behind the previous token's work
            const int64_t t = t0 + (k < nt ? k : nt - 1);
            float sg;
            const float dl = step_raw(in_dl(sb, k, t), sg);
            const float x = in_x(sb, k, t);
            float dyt = valid ? in_dy(sb, k, t) : 0.0f;  // idle lanes add nothing
            float Bv[S], Cv[S];
            in_B(sb, k, t, Bv);
            in_C(sb, k, t, Cv);
            const float zraw = (FUSED && zp != nullptr) ? in_z(sb, k, t) : 0.0f;
            if (k < nt) {
                float ysp = 0.0f;
                if (FUSED && zp != nullptr) {
                    // the gate: this lane's share of the scan's own output ys = C . h_t
#pragma unroll
                    for (int p = 0; p < SP; ++p) {
                        float h0v, h1v;
                        unpack2(hk[k][p], h0v, h1v);
                        ysp = fmaf(Cv[2 * p], h0v, ysp);
                        ysp = fmaf(Cv[2 * p + 1], h1v, ysp);
                    }
                    const float sz = 1.0f / (1.0f + ex2(-zraw * 1.4426950408889634f));
                    dyt *= zraw * sz;  // dy of the scan = dy silu(z)
                }
                float dut = 0.0f, ddt = 0.0f;
                f2 vb[SP], vc[SP];
                const f2 dy2 = splat2(dyt);
                if constexpr (ZOH) {
#pragma unroll
                    for (int p = 0; p < SP; ++p) {
                        float hp0, hp1, hk0, hk1, g0, g1, da0, da1;
                        unpack2(k > 0 ? hk[k > 0 ? k - 1 : 0][p] : h_in[p], hp0, hp1);
                        unpack2(hk[k][p], hk0, hk1);
                        unpack2(gs[p], g0, g1);
                        unpack2(dacc[p], da0, da1);
                        float abv[2];
                        if constexpr (kKeepAbar) unpack2(ab[k][p], abv[0], abv[1]);
                        else { abv[0] = ex2(dl * a2[2 * p]); abv[1] = ex2(dl * a2[2 * p + 1]); }
                        float gv[2] = {g0, g1}, dav[2] = {da0, da1}, vbv[2], vcv[2];
                        const float hpv[2] = {hp0, hp1}, hkv[2] = {hk0, hk1};
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int i = 2 * p + q;
                            float beta, dbdl, dbda, dbdb;
                            coefs(i, dl, abv[q], Bv[i], beta, dbdl, dbda, dbdb);
                            gv[q] = fmaf(Cv[i], dyt, gv[q]);
                            dut = fmaf(gv[q], beta, dut);
                            ddt = fmaf(gv[q], fmaf(hpv[q] * a1[i], abv[q], x * dbdl), ddt);
                            dav[q] = fmaf(gv[q], fmaf(hpv[q] * dl, abv[q], x * dbda), dav[q]);
                            vbv[q] = gv[q] * x * dbdb;
                            vcv[q] = dyt * hkv[q];
                            gv[q] *= abv[q];
                        }
                        gs[p] = pack2(gv[0], gv[1]);
                        dacc[p] = pack2(dav[0], dav[1]);
                        vb[p] = pack2(vbv[0], vbv[1]);
                        vc[p] = pack2(vcv[0], vcv[1]);
                    }
                } else {
                    // Euler (beta = delta B): du = delta sum g B, ddelta = sum g hprev A Abar + u sum g B,
                    // dA += g hprev delta Abar, dB += g u delta; the shared factors once per state
                    const f2 xdl2 = splat2(x * dl), dl2 = splat2(dl);
                    f2 sgb = splat2(0.0f), sqa = splat2(0.0f);
#pragma unroll
                    for (int p = 0; p < SP; ++p) {
                        const f2 hprev = k > 0 ? hk[k > 0 ? k - 1 : 0][p] : h_in[p];
                        const f2 abp = kKeepAbar ? ab[k > KA - 1 ? KA - 1 : k][p] : abar_pair(dl, p);
                        gs[p] = fma2(pack2(Cv[2 * p], Cv[2 * p + 1]), dy2, gs[p]);
                        sgb = fma2(gs[p], pack2(Bv[2 * p], Bv[2 * p + 1]), sgb);
                        const f2 q = mul2(mul2(gs[p], hprev), abp);
                        sqa = fma2(q, a1p[p], sqa);
                        dacc[p] = fma2(q, dl2, dacc[p]);
                        vb[p] = mul2(gs[p], xdl2);
                        vc[p] = mul2(dy2, hk[k][p]);
                        gs[p] = mul2(gs[p], abp);
                    }
                    float sb0, sb1, sq0, sq1;
                    unpack2(sgb, sb0, sb1);
                    unpack2(sqa, sq0, sq1);
                    const float sgbv = sb0 + sb1;
                    dut = dl * sgbv;
                    ddt = fmaf(x, sgbv, sq0 + sq1);
                }
                s_tok[0][k][threadIdx.x] = dut;
                s_tok[1][k][threadIdx.x] = ddt * sg;  // the gradient of the raw step (softplus' = sigmoid)
                if (FUSED && zp != nullptr) s_tok[2][k][threadIdx.x] = ysp;
                st_pairs(&s_vb[k][threadIdx.x * S], vb);
                st_pairs(&s_vc[k][threadIdx.x * S], vc);
            }
        }
        __syncthreads();
        // du, ddelta (and dz) of each (token, channel): the channel's LPC lanes are the
        // consecutive threads j LPC .. j LPC + LPC - 1
        for (int e = threadIdx.x; e < KC * CPB; e += kBwdThreads) {
            const int k = e / CPB, j = e % CPB;
            const int64_t dj = static_cast<int64_t>(blockIdx.x) * CPB + j;
            if (k >= nt || dj >= D) continue;
            const int64_t idx = (b * L + t0 + k) * D + dj;
            const float dut = sum_lanes<LPC>(&s_tok[0][k][j * LPC]);
            const float ddt = sum_lanes<LPC>(&s_tok[1][k][j * LPC]);
            Io<IO>::st(static_cast<IO *>(P.du) + idx, dut);
            Io<IO>::st(static_cast<IO *>(P.ddelta) + idx, ddt);
            dbias_acc += ddt;  // this thread's channel is always j = threadIdx.x % CPB
            if (FUSED && zp != nullptr) {
                const float ys = sum_lanes<LPC>(&s_tok[2][k][j * LPC]);
                const float zt = Io<IO>::widen(Io<IO>::ld(static_cast<const IO *>(P.z) + idx));
                const float dy0 = Io<IO>::widen(Io<IO>::ld(static_cast<const IO *>(P.dy) + idx));
                const float sz = 1.0f / (1.0f + ex2(-zt * 1.4426950408889634f));
                Io<IO>::st(static_cast<IO *>(P.dz) + idx, dy0 * ys * sz * fmaf(zt, 1.0f - sz, 1.0f));
            }
        }
        // dB, dC of each (token, four states): summed over the block's channels (the
        // contributions sit in [k][channel][N] order) into this block's plane.  Two adjacent
        // lanes share an item, one over the even channels and one over the odd, and meet by a
        // shuffle (2 KC N/4 items: a multiple of the block's threads, so every lane takes part
        // in every shuffle; rows past the chunk's end are summed and not stored).
        constexpr int kQ = N / 4;
        static_assert((4 * KC * kQ) % kBwdThreads == 0 && CPB % 2 == 0, "two lanes per item, every lane busy");
        float *plane = P.part + static_cast<int64_t>(blockIdx.x) * gridDim.y * L * 2 * N;
        for (int e = threadIdx.x; e < 4 * KC * kQ; e += kBwdThreads) {
            const int item = e >> 1, half = e & 1;
            const int which = item / (KC * kQ), r = item % (KC * kQ), k = r / kQ, q = r % kQ;
            const float *src = (which ? &s_vc[k][0] : &s_vb[k][0]) + 4 * q + half * N;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int j = 0; j < CPB / 2; ++j) {
                const float4 v = *reinterpret_cast<const float4 *>(src + 2 * j * N);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 1);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 1);
            acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 1);
            acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 1);
            if (half == 0 && k < nt)
                *reinterpret_cast<float4 *>(plane + ((b * L + t0 + k) * 2 + which) * N + 4 * q) = acc;
        }
        // every thread done with this chunk's sums before the next chunk writes them (STAGED:
        // the barrier at the top of the next chunk)
        if constexpr (!STAGED) __syncthreads();
    }
    if (valid) {
        if (P.dh0 != nullptr) st_pairs(P.dh0 + (b * D + d) * N + n0, gs);
        float da[S];
#pragma unroll
        for (int p = 0; p < SP; ++p) unpack2(dacc[p], da[2 * p], da[2 * p + 1]);
        atomic_addv<S>(P.dA + d * N + n0, da);
    }
    if (FUSED && P.dbias != nullptr && threadIdx.x < KC * CPB) {
        const int64_t dj = static_cast<int64_t>(blockIdx.x) * CPB + threadIdx.x % CPB;
        if (dj < D) atomicAdd(P.dbias + dj, dbias_acc);
    }
}

// dB and dC: the sum of the backward blocks' planes ([planes][rows][2][N],
// rows = B L), one thread per four outputs, the planes read with coalesced
// 16-byte loads.
__global__ void __launch_bounds__(256)
sscan_backward_reduce_kernel(const float *__restrict__ part, float *__restrict__ dB, float *__restrict__ dC,
                             int64_t rows, int N, int64_t planes) {
    const int64_t per_plane = rows * 2 * (N / 4);
    for (int64_t q4 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q4 < per_plane;
         q4 += static_cast<int64_t>(gridDim.x) * blockDim.x) {  // float4 index within a plane
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 *p = reinterpret_cast<const float4 *>(part) + q4;
        for (int64_t k = 0; k < planes; ++k) {
            const float4 v = __ldg(p + k * per_plane);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        const int64_t row = q4 / (2 * (N / 4));
        const int rem = static_cast<int>(q4 % (2 * (N / 4)));
        const int which = rem / (N / 4), q = rem % (N / 4);
        *reinterpret_cast<float4 *>((which ? dC : dB) + row * N + 4 * q) = acc;
    }
}

}  // namespace sscan
