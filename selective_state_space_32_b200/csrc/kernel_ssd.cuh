// kernel_ssd.cuh -- Mamba-2 state-space-duality (SSD) forward on the sm_100a
// tensor cores (tcgen05.mma, accumulators in tensor memory, TMA-staged tiles).
//
// What is computed ("Mamba & Mamba-2 Architecture", section 3, "Mamba-2 and
// State Space Duality (SSD)"): the transition is one scalar per head,
// a_t = exp(delta_t * A_h), so within a block of tokens the sequence map is
// the 1-semiseparable matrix M o (C Bbar^T) applied to the head's inputs X,
// with Bbar_s = delta_s B_s and M[t, s] = prod_{k = s+1 .. t} a_k (s <= t).
// The sequence is cut into blocks ("partitions the sequence into blocks ... and
// executes the intra-block computations using GPU Tensor Cores"); the state
// h [N x P] carries the earlier blocks into each block.  For one block of
// Q = 128 tokens of one (batch row b, head h), with cs_t = sum_{k <= t} delta_k
// A_h inside the block:
//
//   S      = C Bᵀ                                   [Q x Q]   MMA 1 (K = N)
//   P      = S o L,  L[t, s] = delta_s exp(cs_t - cs_s) for s <= t, else 0
//   Y      = P X  +  diag(exp(cs_t)) C h_in         [Q x P]   MMA 2 + MMA 3 (K = Q, K = N)
//   S_blk  = Bᵀ diag(w) X,  w_s = delta_s exp(cs_end - cs_s)   [N x P]   MMA 4 (K = Q)
//   h_out  = exp(cs_end) h_in + S_blk               (fp32, in registers)
//
// which is exactly the chunked algorithm of the fp64 SSD oracle, with blocks
// of 128 tokens (the page's "e.g. block size 64" names a size, not a rule; 128
// is the tcgen05 MMA's natural M, and any block size gives the same result).
//
// Work unit.  One CTA per (b, h) walks the blocks in order; the state passing
// is sequential, but it is only the cheap last line above, so the blocks are
// pipelined: block c+2 is being loaded and the MMAs of block c+1 run while the
// CUDA cores finish block c.  One CTA per SM (211 KB of shared memory, 448 of
// the 512 TMEM columns).
//
// Roles (9 warps).
//   warp 8, lane 0  TMA loads (C, B: two 64-state boxes each; X: one box) into
//                   two stages, and every tcgen05.mma and commit;
//   warps 0-3 (P)   decays of the block, then P from S (TMEM) back into TMEM as
//                   the bf16 A operand of MMA 2 (over S's first 64 columns);
//   warps 4-7 (Y)   w X (bf16, shared memory) for MMA 4, the fp32 state h and
//                   its bf16 copy h_in for MMA 3 (two buffers), and y.
// Thread i of a warpgroup is TMEM lane i: token row i of S, P and Y, state row
// i of S_blk and h.  Each warpgroup scans the block's steps itself.
//
// Tensor memory (512 columns allocated, 448 used; lanes x 32-bit columns):
// S of even blocks [0, 128), of odd blocks [128, 256) (P over the first 64 of
// them); P X [256, 320); C h_in [320, 384); S_blk [384, 448).
//
// Precision.  bf16 operands, fp32 accumulation; P, h_in and w X are rounded
// to bf16 as MMA operands, the state and the decays stay fp32.
//
// Every wait is bounded; a wait that gives up sets an abort flag that every
// other wait of the CTA checks, latches a bit in the caller's status word, and
// the CTA drains its last MMAs, releases its tensor memory and exits.  Every
// thread of a warpgroup runs the same named barriers whatever happens.
#pragma once

#include "device_utils.cuh"

namespace sscan {
namespace ssd {

constexpr int kQ = 128;          // tokens per block (M of the MMAs over tokens)
constexpr int kN = 128;          // state size
constexpr int kP = 64;           // head dimension
constexpr int kWG = 128;         // threads per warpgroup
constexpr int kThreads = 2 * kWG + 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColY1 = 256, kColY2 = 320, kColSblk = 384;  // S of block c at kColS + 128 (c & 1)

// Shared memory, from a 1024-byte aligned base (the 128-byte swizzle atom).
constexpr int kBox = kQ * 128;                 // one TMA box: 128 rows x 128 bytes
constexpr int kStage = 5 * kBox;               // C (2 boxes), B (2 boxes), X
constexpr int kOffStage = 0;                   // 2 stages
constexpr int kOffWX = 2 * kStage;             // w X, [token s][head dim p]
constexpr int kOffH = kOffWX + kBox;           // h_in as bf16, [state n][head dim p], 2 buffers
constexpr int kOffCs = kOffH + 2 * kBox;       // warpgroup P: float cs2[128] (cumulative delta*A*log2 e)
constexpr int kOffDt = kOffCs + 512;           //              float delta[128]
constexpr int kOffColf = kOffDt + 512;         //              float column factors[128]
constexpr int kOffWarp = kOffColf + 512;       // float scan totals [2 warpgroups][4 warps]
constexpr int kOffBars = kOffWarp + 64;        // mbarriers
constexpr int kNumBars = 13;
constexpr int kOffTmem = kOffBars + 8 * kNumBars;
constexpr int kOffAbort = kOffTmem + 4;
constexpr int kSmemUsed = kOffAbort + 4;
constexpr int kSmemBytes = kSmemUsed + 1024;   // + slack to align the base
constexpr uint32_t kLoadBytes = kStage;        // C, B and X per block
constexpr int kOffC = 0, kOffB = 2 * kBox, kOffX = 4 * kBox;  // within a stage

// mbarriers; a per-stage barrier completes once per two blocks, the others once per block
enum {
    BAR_FULL = 0,      // [2] TMA of a stage landed                      (count 1 + bytes)
    BAR_SDONE = 2,     // [2] MMA 1 of the stage's block done             (commit)
    BAR_PREADY = 4,    // [2] P of the stage's block in TMEM              (warpgroup P)
    BAR_WXREADY = 6,   // w X of the block written                        (warpgroup Y)
    BAR_M4 = 7,        // MMA 4 of the block done: S_blk ready, w X free  (commit)
    BAR_SBLKFREE = 8,  // S_blk of the block read                         (warpgroup Y)
    BAR_HREADY = 9,    // h_in of the next block written                  (warpgroup Y)
    BAR_YREADY = 10,   // MMAs 2 and 3 of the block done (and everything before them)
    BAR_YFREE = 11,    // P X and C h_in of the block read                (warpgroup Y)
    BAR_DRAIN = 12,    // every MMA of the CTA done (before the tensor memory is released)
};

struct Params {
    const float *dt;       // [B][L][H] step delta (after softplus)
    const float *A;        // [H]
    const float *h0;       // [B][H][N][P] or null
    uint16_t *y;           // [B][L][H][P] bf16
    float *h_final;        // [B][H][N][P] or null
    int *status;           // error bits, or null
    int64_t L;
    int H;
    int nblocks;
};

// ------------------------------------------------------ tcgen05 primitives

// Instruction descriptor of kind::f16 with bf16 A and B and an fp32 accumulator:
// bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format, 15 A
// major (0 = K, 1 = MN), 16 B major, 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading and
// stride byte offsets (all >> 4), version 1 (bits 46-47), layout 2 (bits 61-63).
// K-major operands: rows of 128 bytes, 8-row atoms SBO = 1024 bytes apart (LBO
// unused, 16).  MN-major operands: 64 contiguous elements per 128-byte row, K
// along rows, 8-row groups SBO = 1024 bytes apart, further 64-element MN
// chunks LBO bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A B with A and B in shared memory
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// D (+)= A B with A in tensor memory (M lanes x K/2 columns of packed pairs)
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// arrive on bar once every earlier tcgen05.mma of this thread has completed
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane; the wait is part of the
// call, with the registers passed through it so no use is scheduled before it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
          "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
          "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
          "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

// bf16 pair (round to nearest even): lo in bits 0-15, hi in bits 16-31
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Byte offset of 16-byte chunk c (0-7) of row r in a 128-byte-swizzled tile (the
// layout TMA writes with SWIZZLE_128B into a 1024-byte aligned box).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return uint32_t(r) * 128u + (uint32_t(c ^ (r & 7)) << 4); }

// Bounded wait on an mbarrier phase that also gives up once another thread of the
// CTA has aborted; on its own timeout it raises the abort flag and the status bit.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              int *status, int bit) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63 && *abort_flag) return false;
    }
    *abort_flag = 1;
    if (status) atomicOr(status, bit);
    return false;
}

// --------------------------------------------------------------- the kernel

// Inclusive scan of v over the 128 threads of a warpgroup (named barrier `bar_id`,
// warp totals in tot4[4]); returns the thread's prefix and the block total.
__device__ __forceinline__ float wg_scan(float v, int wl, int lane, float *tot4, int bar_id, float &total) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) tot4[wl] = v;
    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
    float pre = 0.0f, tot = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float wt = tot4[i];
        pre += i < wl ? wt : 0.0f;
        tot += wt;
    }
    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");  // totals read before the next block's scan
    total = tot;
    return v + pre;
}

__global__ void __launch_bounds__(kThreads, 1)
ssd_forward_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const Params prm) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char *sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / prm.H, h = blockIdx.x % prm.H;
    const int64_t L = prm.L;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffTmem);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffAbort);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[BAR_FULL + i], 1);
            mbar_init(&bars[BAR_SDONE + i], 1);
            mbar_init(&bars[BAR_PREADY + i], kWG);
        }
        mbar_init(&bars[BAR_WXREADY], kWG);
        mbar_init(&bars[BAR_M4], 1);
        mbar_init(&bars[BAR_SBLKFREE], kWG);
        mbar_init(&bars[BAR_HREADY], kWG);
        mbar_init(&bars[BAR_YREADY], 1);
        mbar_init(&bars[BAR_YFREE], kWG);
        mbar_init(&bars[BAR_DRAIN], 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 8) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const int nb = prm.nblocks;
    const float a2 = __ldg(prm.A + h) * 1.4426950408889634f;  // A_h log2(e): decays as powers of 2

    if (warp == 8) {
        if (lane == 0) {
            // ------------------------------------------------ TMA and MMA issue
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            tma_prefetch_desc(&tm_c);
            constexpr uint32_t id_s = idesc_bf16(kQ, kQ, 0, 0);    // C (K-major) x B^T (K-major)
            constexpr uint32_t id_y = idesc_bf16(kQ, kP, 0, 1);    // P or C (K-major) x X or h (MN-major)
            constexpr uint32_t id_st = idesc_bf16(kN, kP, 1, 1);   // B^T (MN-major) x wX (MN-major)
            const uint32_t sWX = sbase + kOffWX;
            auto load = [&](int c) {  // block c into stage c & 1
                const uint32_t st = sbase + kOffStage + (c & 1) * kStage;
                uint64_t *bar = &bars[BAR_FULL + (c & 1)];
                const int t0 = c * kQ;
                mbar_expect_tx(bar, kLoadBytes);
                tma_load_3d(st + kOffC, &tm_c, 0, t0, b, bar);
                tma_load_3d(st + kOffC + kBox, &tm_c, 64, t0, b, bar);
                tma_load_3d(st + kOffB, &tm_b, 0, t0, b, bar);
                tma_load_3d(st + kOffB + kBox, &tm_b, 64, t0, b, bar);
                tma_load_4d(st + kOffX, &tm_x, 0, h, t0, b, bar);
            };
            auto wait = [&](int bar, uint32_t parity) {
                return wait_or_abort(&bars[bar], parity, abort_flag, prm.status, 16);
            };
            bool issued = false;
            auto mma1 = [&](int c) {  // S of block c = C B^T, K = N in 8 steps of 16 states
                const uint32_t st = sbase + kOffStage + (c & 1) * kStage;
                const uint32_t sC = st + kOffC, sB = st + kOffB;
                const uint32_t tS = tbase + kColS + 128 * (c & 1);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
                    mma_ss(tS, sdesc_sw128(sC + off, 16, 1024), sdesc_sw128(sB + off, 16, 1024), id_s, k > 0);
                }
                mma_commit(&bars[BAR_SDONE + (c & 1)]);
                issued = true;
            };
            // Issue order: MMA 1 of block c+1 goes ahead of MMAs 2 and 3 of block c, so that
            // warpgroup P forms P of block c+1 while they run.  The S buffer of block c+1 last
            // held block c-1's P, read by its MMA 2: done once BAR_YREADY of c-1 was seen.
            load(0);
            if (nb > 1) load(1);
            bool run = wait(BAR_FULL, 0);
            if (run) {
                tc_fence_after();
                mma1(0);
            }
            for (int c = 0; run && c < nb; ++c) {
                const int s = c & 1;
                const uint32_t ps = (c >> 1) & 1, pc = c & 1, pp = (c - 1) & 1;
                const uint32_t st = sbase + kOffStage + s * kStage;
                const uint32_t sC = st + kOffC, sB = st + kOffB, sX = st + kOffX;
                const uint32_t sH = sbase + kOffH + s * kBox;  // h_in of this block
                const uint32_t tS = tbase + kColS + 128 * s;
                // MMA 4: S_blk = B^T (w X), M = N (two 64-state chunks kBox apart), K = Q.
                // h_in of this block is waited for here, before MMA 4: warpgroup Y arrives
                // for the next block's h_in as soon as MMA 4 is done, and a phase-parity
                // wait must never fall two phases behind its barrier.
                if (!wait(BAR_WXREADY, pc)) break;
                if (c > 0 && !wait(BAR_SBLKFREE, pp)) break;
                if (!wait(BAR_HREADY, pc)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss(tbase + kColSblk, sdesc_sw128(sB + k * 2048, kBox, 1024),
                           sdesc_sw128(sWX + k * 2048, kBox, 1024), id_st, k > 0);
                mma_commit(&bars[BAR_M4]);
                // MMA 1 of the next block
                if (c + 1 < nb) {
                    if (!wait(BAR_FULL + (s ^ 1), ((c + 1) >> 1) & 1)) break;
                    tc_fence_after();
                    mma1(c + 1);
                }
                // MMA 2: Y1 = P X (P: TMEM columns 8k.. of packed pairs), MMA 3: Y2 = C h_in
                if (!wait(BAR_PREADY + s, ps)) break;
                if (c > 0 && !wait(BAR_YFREE, pp)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts(tbase + kColY1, tS + 8 * k, sdesc_sw128(sX + k * 2048, kBox, 1024), id_y, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
                    mma_ss(tbase + kColY2, sdesc_sw128(sC + off, 16, 1024), sdesc_sw128(sH + k * 2048, kBox, 1024),
                           id_y, k > 0);
                }
                mma_commit(&bars[BAR_YREADY]);
                // block c+2 goes into this stage once every MMA of block c is done
                if (c + 2 < nb) {
                    if (!wait(BAR_YREADY, pc)) break;
                    load(c + 2);
                }
            }
            // the tensor memory is released below: every MMA issued must be done first.  A
            // commit tracks all earlier MMAs of this thread: one more on its own barrier,
            // waited for with a bound (also after an abort)
            if (issued) {
                mma_commit(&bars[BAR_DRAIN]);
                for (uint32_t i = 0; i < kSpinLimit; ++i)
                    if (mbar_try_wait(&bars[BAR_DRAIN], 0)) break;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ the two warpgroups
        const bool is_p = warp < 4;
        const int wl = warp & 3;               // warp within the warpgroup
        const int t = threadIdx.x & 127;       // TMEM lane = token row = state row
        const uint32_t lane_base = tbase + (uint32_t(wl * 32) << 16);
        float *tot4 = reinterpret_cast<float *>(sm + kOffWarp) + (is_p ? 0 : 4);
        const int bar_id = is_p ? 1 : 2;
        bool ok = true;
        auto wait_warp = [&](int bar, uint32_t parity) {
            const bool r = ok && wait_or_abort(&bars[bar], parity, abort_flag, prm.status, 32);
            return __all_sync(0xffffffffu, r);
        };
        const float *dtp = prm.dt + int64_t(b) * L * prm.H + h;
        float dt_next = t < L ? __ldg(dtp + int64_t(t) * prm.H) : 0.0f;
        // y of block c: P X + 2^cs (C h_in), rows inside the sequence only (warpgroup P, after
        // forming the next block's P; its TMEM reads end before YFREE lets MMAs 2, 3 reuse them)
        auto emit_y = [&](int c, float cs) {
            ok = wait_warp(BAR_YREADY, c & 1);
            if (!ok) return;
            tc_fence_after();
            const float e = ex2(cs);
            uint32_t o[2][16];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t y1[32], y2[32];
                tmem_ld32(lane_base + kColY1 + 32 * half, y1);
                tmem_ld32(lane_base + kColY2 + 32 * half, y2);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    o[half][j] = pack_bf16(fmaf(e, __uint_as_float(y2[2 * j]), __uint_as_float(y1[2 * j])),
                                           fmaf(e, __uint_as_float(y2[2 * j + 1]), __uint_as_float(y1[2 * j + 1])));
            }
            tc_fence_before();
            mbar_arrive(&bars[BAR_YFREE]);
            const int64_t tok = int64_t(c) * kQ + t;
            if (tok < L) {
                uint4 *d4 = reinterpret_cast<uint4 *>(prm.y + ((int64_t(b) * L + tok) * prm.H + h) * kP);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    d4[q] = make_uint4(o[q >> 2][4 * (q & 3)], o[q >> 2][4 * (q & 3) + 1],
                                       o[q >> 2][4 * (q & 3) + 2], o[q >> 2][4 * (q & 3) + 3]);
            }
        };

        if (is_p) {
            // ============================================ warpgroup P
            float *s_cs = reinterpret_cast<float *>(sm + kOffCs);
            float *s_dt = reinterpret_cast<float *>(sm + kOffDt);
            float *s_colf = reinterpret_cast<float *>(sm + kOffColf);
            float cs_prev = 0.0f;
            for (int c = 0; c < nb; ++c) {
                const int s = c & 1;
                const uint32_t ps = (c >> 1) & 1;
                const float dt = dt_next;
                const int64_t nxt = int64_t(c + 1) * kQ + t;
                dt_next = nxt < L ? __ldg(dtp + nxt * prm.H) : 0.0f;  // next block's step, in flight
                float tot;
                const float cs = wg_scan(dt * a2, wl, lane, tot4, bar_id, tot);
                s_cs[t] = cs;
                s_dt[t] = dt;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                // column factor of token s = t for its 16-token group: delta_s 2^(r_g - cs_s),
                // r_g = cs at the group's last token (<= 1 for A <= 0)
                s_colf[t] = dt * ex2(s_cs[(t & ~15) + 15] - cs);
                asm volatile("bar.sync 1, 128;" ::: "memory");
                // P = S o L into TMEM (packed bf16 pairs over S's first 64 columns)
                ok = wait_warp(BAR_SDONE + s, ps);
                if (ok) {
                    tc_fence_after();
                    const uint32_t tS = lane_base + kColS + 128 * s;
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk) {  // columns 32kk .. 32kk+31 (groups 2kk, 2kk+1)
                        uint32_t pk[16];
                        if (kk < wl) {
                            // groups entirely before this warp's rows: 2^(cs_t - cs_s) = 2^(cs_t - r_g) 2^(r_g - cs_s)
                            uint32_t s_raw[32];
                            tmem_ld32(tS + 32 * kk, s_raw);
                            const float rf0 = ex2(cs - s_cs[32 * kk + 15]);
                            const float rf1 = ex2(cs - s_cs[32 * kk + 31]);
#pragma unroll
                            for (int j = 0; j < 32; j += 2) {
                                const float rf = j < 16 ? rf0 : rf1;
                                const float p0 = __uint_as_float(s_raw[j]) * s_colf[32 * kk + j] * rf;
                                const float p1 = __uint_as_float(s_raw[j + 1]) * s_colf[32 * kk + j + 1] * rf;
                                pk[j / 2] = pack_bf16(p0, p1);
                            }
                        } else if (kk == wl) {
                            // the groups holding this warp's diagonal: 2^(cs_t - cs_s) directly, 0 above it
                            uint32_t s_raw[32];
                            tmem_ld32(tS + 32 * kk, s_raw);
#pragma unroll
                            for (int j = 0; j < 32; j += 2) {
                                const int s0 = 32 * kk + j;
                                const float p0 =
                                    s0 <= t ? __uint_as_float(s_raw[j]) * s_dt[s0] * ex2(cs - s_cs[s0]) : 0.0f;
                                const float p1 = s0 + 1 <= t ? __uint_as_float(s_raw[j + 1]) * s_dt[s0 + 1] *
                                                                   ex2(cs - s_cs[s0 + 1])
                                                             : 0.0f;
                                pk[j / 2] = pack_bf16(p0, p1);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) pk[j] = 0u;
                        }
                        tmem_st16(tS + 16 * kk, pk);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bars[BAR_PREADY + s]);
                }
                if (ok && c > 0) emit_y(c - 1, cs_prev);
                cs_prev = cs;
            }
            if (ok && nb > 0) emit_y(nb - 1, cs_prev);
        } else {
            // ============================================ warpgroup Y
            float hs[kP];  // state row n = t, fp32
            {
                const float *src = prm.h0 ? prm.h0 + ((int64_t(b) * prm.H + h) * kN + t) * kP : nullptr;
#pragma unroll
                for (int j = 0; j < kP; j += 4) {
                    const float4 v = src ? __ldg(reinterpret_cast<const float4 *>(src + j)) : make_float4(0, 0, 0, 0);
                    hs[j] = v.x;
                    hs[j + 1] = v.y;
                    hs[j + 2] = v.z;
                    hs[j + 3] = v.w;
                }
            }
            auto write_h = [&](int buf) {  // h_in row n = t as bf16 into the swizzled [n][p] tile
                unsigned char *row = sm + kOffH + buf * kBox;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint4 v;
                    v.x = pack_bf16(hs[8 * q + 0], hs[8 * q + 1]);
                    v.y = pack_bf16(hs[8 * q + 2], hs[8 * q + 3]);
                    v.z = pack_bf16(hs[8 * q + 4], hs[8 * q + 5]);
                    v.w = pack_bf16(hs[8 * q + 6], hs[8 * q + 7]);
                    *reinterpret_cast<uint4 *>(row + sw128(t, q)) = v;
                }
                fence_proxy_async_smem();  // generic writes -> the MMA's operand reads
            };
            write_h(0);
            mbar_arrive(&bars[BAR_HREADY]);
            // Per block c: w X of block c first (MMA 4 of block c can start at once), then
            // the state passing of block c (warpgroup P emits y).  The h_in buffer written
            // for block c+1 was read by MMA 3 of block c-1: done once MMA 4 of block c is,
            // as a commit tracks every earlier MMA of the issuing thread.
            for (int c = 0; c < nb; ++c) {
                const int s = c & 1;
                const uint32_t ps = (c >> 1) & 1, pc = c & 1;
                const float dt = dt_next;
                const int64_t nxt = int64_t(c + 1) * kQ + t;
                dt_next = nxt < L ? __ldg(dtp + nxt * prm.H) : 0.0f;
                float tot;
                const float cs = wg_scan(dt * a2, wl, lane, tot4, bar_id, tot);
                // ---- w X for MMA 4: X of this block landed; w X's buffer was freed by MMA 4
                // of block c-1 (waited for in the state step of the previous block)
                ok = wait_warp(BAR_FULL + s, ps);
                if (ok) {
                    const float wv = dt * ex2(tot - cs);  // w_s of the block end state, s = t
                    const unsigned char *xr = sm + kOffStage + s * kStage + kOffX;
                    unsigned char *wr = sm + kOffWX;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint4 v4 = *reinterpret_cast<const uint4 *>(xr + sw128(t, q));
                        v4.x = pack_bf16(bf16_lo(v4.x) * wv, bf16_hi(v4.x) * wv);
                        v4.y = pack_bf16(bf16_lo(v4.y) * wv, bf16_hi(v4.y) * wv);
                        v4.z = pack_bf16(bf16_lo(v4.z) * wv, bf16_hi(v4.z) * wv);
                        v4.w = pack_bf16(bf16_lo(v4.w) * wv, bf16_hi(v4.w) * wv);
                        *reinterpret_cast<uint4 *>(wr + sw128(t, q)) = v4;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&bars[BAR_WXREADY]);
                }
                // ---- state passing: h = 2^cs_end h + S_blk (row n = t); then h_in of block c+1,
                // into the buffer MMA 3 of block c-1 read
                ok = wait_warp(BAR_M4, pc);
                if (ok) {
                    tc_fence_after();
                    const float aend = ex2(tot);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t sb[32];
                        tmem_ld32(lane_base + kColSblk + 32 * half, sb);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            hs[32 * half + j] = fmaf(aend, hs[32 * half + j], __uint_as_float(sb[j]));
                    }
                    tc_fence_before();
                    mbar_arrive(&bars[BAR_SBLKFREE]);
                    write_h((c + 1) & 1);
                    mbar_arrive(&bars[BAR_HREADY]);
                }
            }
            if (ok && prm.h_final) {
                float *dst = prm.h_final + ((int64_t(b) * prm.H + h) * kN + t) * kP;
#pragma unroll
                for (int j = 0; j < kP; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(hs[j], hs[j + 1], hs[j + 2], hs[j + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace ssd
}  // namespace sscan
