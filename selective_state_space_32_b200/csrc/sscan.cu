// sscan.cu -- host side of the B200 (sm_100a) selective-scan forward library:
// plans, schedule choice, TMA descriptors, launches, and the C ABI declared in
// include/sscan.h (the host-buffer entry point is in host_pipe.cu, the
// backward in sscan_backward.cu, the SSD form in ssd.cu).
//
// What is computed ("tm_ssm_selective" (Transformer Math page on selective
// SSMs), section "Discretization becomes a per-token operation"; the
// selective_scan reference loop of "12. Selective State Space"):
//     Abar = exp(delta*A[d,n]);   Bbar u = delta*B[n]*u  (Euler) or
//     (exp(delta*A)-1)/A*B[n]*u (ZOH);   h = Abar*h + Bbar u;   y = sum_n C[n]*h.
//
// Kernels:
//  * chained (kernel_chained.cuh): persistent, cooperative, one warp per
//    chain segment, TMA-staged inputs, exactly balanced work per warp;
//  * tiled (kernel_tiled.cuh): the same recurrence with one block per
//    block-chain segment, its warps sharing each stage's tiles (shapes whose
//    per-warp rows are narrower than an L2 fill);
//  * step (kernel_step.cuh): four states per thread, shaped for the state's
//    HBM round trip; sequences shorter than the chained kernel's minimum
//    (the decode kernel, kernel_decode.cuh, takes the single-token step with
//    a state);
//  * generic (kernel_generic.cuh): one thread per (channel, state group),
//    plain loads; for the longer shapes the chained kernel cannot take.
// Every one keeps each (b,d) state row in registers; the [B,L,D,N] tensors
// never reach memory.  The path is ALU bound on B200 (one 2^x and four FMA-pipe
// operations per state update against 1-3 bytes of HBM traffic), so there are
// no tensor-core stages.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "device_utils.cuh"
#include "kernel_chained.cuh"
#include "kernel_decode.cuh"
#include "kernel_generic.cuh"
#include "kernel_step.cuh"
#include "kernel_tiled.cuh"
#include "plan.cuh"
#include "sscan.h"

#define SSCAN_VERSION 200  // 0.2.0

using namespace sscan;

namespace {

// Chained-kernel shapes compiled into the library.  NL states per lane, T
// tokens per pipeline stage, STAGES stages per warp, WPC warps per block.
struct KCfg {
    int N, NL, T, STAGES, WPC;
};
// In order of preference for a shape; a shape is taken when the problem has at
// least one chain per warp of the persistent grid (148 blocks x WPC warps).
// Measured on B200: the MUFU pipe saturates from 2 warps per SM sub-partition
// at 8 states per lane and from ~4 at 4 states per lane.
constexpr KCfg kChainedCfgs[] = {
    {16, 8, 32, 4, 8},   // 0: 16 channels per warp, 2 warps per SM sub-partition (bf16 only: smem)
    {16, 4, 16, 4, 12},  // 1: 8 channels per warp, 3 warps per sub-partition
    {16, 4, 16, 4, 8},   // 2: 8 channels per warp, 2 warps per sub-partition
    {16, 8, 32, 4, 4},   // 3: 16 channels per warp, 1 warp per sub-partition
    {16, 4, 16, 4, 4},   // 4: 8 channels per warp, 1 warp per sub-partition
    {32, 8, 32, 4, 4},   // 5: 8 channels per warp
    {64, 16, 16, 3, 8},  // 6: 8 channels per warp, 2 warps per sub-partition
};
// Order in which the shapes are tried (measured on B200: for N = 16 both I/O
// types run fastest at 8 states per lane and one consumer warp per SM
// sub-partition, then at 4 states per lane and two).
constexpr int kPrefF32[] = {3, 2, 1, 4, 5, 6, 0};
constexpr int kPrefBF16[] = {3, 0, 2, 1, 4, 5, 6};
// The split mode can use any number of warps (pieces are independent until the
// fix-up), so it prefers two consumer warps per sub-partition.
constexpr int kPrefSplitF32[] = {2, 3, 1, 4, 5, 6, 0};
constexpr int kPrefSplitBF16[] = {0, 2, 3, 1, 4, 5, 6};
constexpr int kNumCfgs = sizeof(kChainedCfgs) / sizeof(kChainedCfgs[0]);

// Block-tiled shapes (kernel_tiled.cuh): N, NL states per lane, T tokens per
// stage, STAGES stages per block, WPC consumer warps per block.
constexpr KCfg kTiledCfgs[] = {
    {64, 8, 32, 3, 12},  // 0: 48 channels per block, 3 consumer warps per SM sub-partition
    {64, 8, 16, 4, 16},  // 1: 64 channels per block, 4 per sub-partition
    {32, 8, 16, 4, 12},  // 2: 96 channels per block
};
constexpr int kNumTiledCfgs = sizeof(kTiledCfgs) / sizeof(kTiledCfgs[0]);
// Shapes the schedule takes without being asked, in order of preference: measured
// on B200 for bf16 I/O at N = 64 (exact ZOH, B = 16, L = 1024, D = 5120: 2.09 ms
// against 2.29 ms for the chained kernel's best shape); the others are built for
// SSCAN_TUNE and the tests.
constexpr int kTiledAuto[] = {0};

std::atomic<uint32_t> g_epoch{1};  // launch tags of the chained kernel (unique per process)

constexpr int kMaxSmem = 227 * 1024;  // dynamic shared memory per block on B200
// The consumer warps that share an SM sub-partition with the producer warp (warp
// index a multiple of 4) ran ~4% slower than the other three on B200, and the
// launch ends with its slowest warp; they get 3x fewer chain-steps and the others
// x more, x = S * kLightPermille / 1000, which evens out the finishing times.
constexpr int kLightPermille = 10;
constexpr int64_t kMinChainedL = 64;  // shorter sequences use the step kernel

// Shared memory of a chained-kernel shape (mirrors ChainedCfg::kSmem; a fused call on a
// shape whose larger ChainedCfg::kSmemF does not fit runs the generic kernel).
int chained_smem_bytes(const KCfg &k, int es) {
    const int lpc = k.N / k.NL, cpw = 32 / lpc;
    const int kU = k.T * cpw * es, kB = k.T * k.N * es;
    const int rowW = k.N + ((es == 2 && k.NL >= 16) ? 4 * lpc : 0);  // ChainedCfg::kRowW
    const int stage = 2 * kU + 2 * kB, conv = es == 2 ? 2 * k.T * rowW * 4 : 0;
    const int warp = (k.STAGES * stage + conv + 127) / 128 * 128;
    const int bars = (2 * k.WPC * k.STAGES * 8 + 127) / 128 * 128;
    return k.WPC * warp + bars;
}

// Shared memory of a tiled-kernel shape (mirrors TiledCfg::kSmem).
int tiled_smem_bytes(const KCfg &k, int es) {
    const int lpc = k.N / k.NL, cpw = 32 / lpc, cpb = k.WPC * cpw;
    const int kU = k.T * cpb * es, kB = k.T * k.N * es;
    const int stageF = 2 * kU + 2 * kB + kU;
    const int rowW = k.N + (lpc >= 4 ? 4 * lpc : 0);
    const int conv = 2 * k.T * rowW * 4;
    const int slot = (stageF + 127) / 128 * 128 + (conv + 127) / 128 * 128;
    const int scratch = k.WPC * 2 * k.T * cpw * 4;
    const int bars = (3 * k.STAGES * 8 + 127) / 128 * 128;
    return k.STAGES * slot + scratch + bars;
}

}  // namespace

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Optional tuning override read at plan creation, e.g. SSCAN_TUNE="cfg=1,poly=0,sms=4":
// cfg indexes the chained shapes above (-1 forces the generic kernel), poly=0
// keeps every exponent on the MUFU pipe, sms limits the chained grid to that
// many blocks, split=1 forces the split mode (tests use the last two to cut
// chains on small problems), nopublish=1 makes the warps running a chain's
// head skip publishing the carried state (failure-detection tests: the
// bounded waits of the warps running the tails must give up and report it),
// light=<per mille> sets how much shorter the segments of the warps that share
// an SM sub-partition with the producer warp are (see kLightPermille), decode=0
// runs a decode step (L = 1) on the step kernel instead of the decode kernel,
// tiled=<i> forces the block-tiled shape i (kTiledCfgs), tiled=-1 keeps the
// schedule off the tiled kernel.
void read_tune(int &cfg, int &poly, int &sms, int &split, int &nopublish, int &light, int &decode,
               int &tiled) {
    cfg = -2;
    poly = -1;
    sms = 0;
    split = 0;
    nopublish = 0;
    light = -1;
    decode = 1;
    tiled = -2;
    const char *s = getenv("SSCAN_TUNE");
    if (!s) return;
    if (const char *c = strstr(s, "cfg=")) cfg = atoi(c + 4);
    if (const char *c = strstr(s, "poly=")) poly = atoi(c + 5);
    if (const char *c = strstr(s, "sms=")) sms = atoi(c + 4);
    if (const char *c = strstr(s, "split=")) split = atoi(c + 6);
    if (const char *c = strstr(s, "nopublish=")) nopublish = atoi(c + 10);
    if (const char *c = strstr(s, "light=")) light = atoi(c + 6);
    if (const char *c = strstr(s, "decode=")) decode = atoi(c + 7);
    if (const char *c = strstr(s, "tiled=")) tiled = atoi(c + 6);
}

void choose_schedule(sscan_plan *p) {
    const int es = p->dtype == SSCAN_F32 ? 4 : 2;
    p->mode = kGeneric;
    p->g_nl = p->N == 16 ? 8 : 16;
    p->g_lpc = static_cast<int>(p->N) / p->g_nl;
    int want = -2, poly = -1, sms = 0, force_split = 0, nopublish = 0, light = -1, decode = 1, tiled = -2;
    read_tune(want, poly, sms, force_split, nopublish, light, decode, tiled);
    p->drop_publish = nopublish != 0;
    const int blocks = (sms > 0 && sms < p->sm_count) ? sms : p->sm_count;
    // the FMA-pipe exponent measured slower than MUFU alone at every occupancy: off unless asked
    p->poly = (p->flags & SSCAN_ZOH) ? false : (poly == 1);
    // very short sequences (e.g. one decode step, L = 1) are a stream over the state:
    // the step kernel, not a persistent grid with a TMA pipeline
    if (p->L < kMinChainedL && want != -1) {
        p->mode = kStep;
        // one token with every bulk copy a multiple of 16 bytes: the decode kernel
        // (calls with a state; without one the step kernel runs)
        p->decode = p->L == 1 && p->D % 8 == 0 && decode != 0;
        return;
    }
    if (want == -1) return;
    // the chained kernel needs TMA-compatible rows and int32 TMA row coordinates
    if ((p->D * es) % 16 != 0 || p->B * p->L >= (int64_t(1) << 31) || p->L >= (int64_t(1) << 32)) return;
    // 0) tiled: block-chains of the block's channels, at least about one per block
    if (tiled != -1 && want < 0 && !force_split) {
        const int n_try = tiled >= 0 ? 1 : static_cast<int>(sizeof(kTiledAuto) / sizeof(kTiledAuto[0]));
        for (int oi = 0; oi < n_try; ++oi) {
            const int i = tiled >= 0 ? tiled : kTiledAuto[oi];
            if (i < 0 || i >= kNumTiledCfgs) continue;
            const KCfg &k = kTiledCfgs[i];
            if (k.N != p->N || tiled_smem_bytes(k, es) > kMaxSmem) continue;
            if (tiled < 0 && es != 2) continue;  // fp32 I/O: not measured faster than the chained kernel
            const int64_t cpb = int64_t(32 / (k.N / k.NL)) * k.WPC;
            const int64_t cpr = ceil_div(p->D, cpb);
            const int64_t chains = p->B * cpr;
            if (tiled < 0 && chains * 20 < int64_t(blocks) * 17) continue;
            p->mode = kTiled;
            p->split = false;
            p->cfg = i;
            p->chains_per_row = cpr;
            p->chains = chains;
            p->workers = int64_t(blocks) * k.WPC;
            p->seg = ceil_div(chains * p->L, blocks);
            p->seg_shift = 0;
            p->max_pieces = 0;
            p->rec_s_off = p->rec_mono_off = 0;
            // carried state and flag per (block-chain, consumer warp)
            p->flag_off = align_up(size_t(chains) * k.WPC * 32 * k.NL * sizeof(float), 256);
            p->flag_bytes = size_t(chains) * k.WPC * sizeof(unsigned long long);
            p->sink_off = p->flag_off + align_up(p->flag_bytes, 256);
            p->ws_bytes = p->sink_off + align_up(size_t(p->workers) * 32 * sizeof(float), 256);
            return;
        }
    }
    // 1) chained: enough chains that each is cut at most once (segment >= L)
    // 2) split: fewer chains than warps; cut them into pieces scanned concurrently
    for (int pass = force_split ? 1 : 0; pass < 2; ++pass) {
        for (int oi = 0; oi < kNumCfgs; ++oi) {
            const int i = pass == 0 ? (es == 4 ? kPrefF32[oi] : kPrefBF16[oi])
                                    : (es == 4 ? kPrefSplitF32[oi] : kPrefSplitBF16[oi]);
            const KCfg &k = kChainedCfgs[i];
            if (k.N != p->N) continue;
            if (want >= 0 && want != i) continue;
            const int lpc = k.N / k.NL, cpw = 32 / lpc;
            if ((cpw * es) % 16 != 0) continue;
            if (chained_smem_bytes(k, es) > kMaxSmem) continue;
            const int64_t cpr = ceil_div(p->D, cpw);
            const int64_t chains = p->B * cpr;
            int64_t workers = int64_t(blocks) * k.WPC;
            const bool split = pass == 1;
            // segments somewhat shorter than L cut a few chains twice (a short wait for the
            // middle piece); measured cheaper than fewer warps down to ~0.85 L
            if (!split && chains * 20 < workers * 17 && want < 0) continue;
            if (split && !force_split) {  // at least 256 tokens per warp; whole blocks
                const int64_t cap = (chains * p->L / 256) / k.WPC * k.WPC;
                if (cap < workers) workers = cap > k.WPC ? cap : k.WPC;
            }
            p->mode = kChained;
            p->split = split && chains < workers;  // else the capped grid already fits whole chains
            p->cfg = i;
            p->chains_per_row = cpr;
            p->chains = chains;
            // Segments are equal over the whole grid, in split mode too.  Cutting every chain
            // into the same whole number of pieces would line up the pieces of neighbouring
            // chains (which share the 64-byte L2 lines of their u and delta rows) and read
            // each input byte from DRAM once instead of 1.6 times, but leaves warps idle
            // (1152 of 1184 on the 131072-token sequence) and measured 3 % slower on B200:
            // the kernel is bound by its ALUs, not by DRAM.
            p->seg = ceil_div(chains * p->L, workers);
            p->workers = workers;
            // split mode indexes pieces by equal segments; the chained mode balances time
            p->seg_shift = p->split ? 0 : p->seg * (light >= 0 ? light : kLightPermille) / 1000;
            if (p->split) {
                p->max_pieces = p->L / p->seg + 2;
                const size_t recs = size_t(chains) * size_t(p->max_pieces);
                p->rec_s_off = align_up(recs * 32 * k.NL * sizeof(float), 256);
                p->rec_mono_off = p->rec_s_off + align_up(recs * 32 * sizeof(float), 256);
                p->flag_off = p->rec_mono_off + align_up(recs * sizeof(int), 256);
                p->flag_bytes = recs * sizeof(unsigned long long);
            } else {
                p->max_pieces = 0;
                p->rec_s_off = p->rec_mono_off = 0;
                p->flag_off = align_up(size_t(chains) * 32 * k.NL * sizeof(float), 256);
                p->flag_bytes = size_t(chains) * sizeof(unsigned long long);
            }
            p->sink_off = p->flag_off + align_up(p->flag_bytes, 256);
            p->ws_bytes = p->sink_off + align_up(size_t(workers) * 32 * sizeof(float), 256);
            return;
        }
    }
}

// Arguments of the fused prologue / epilogue of one call.
struct Fused {
    const float *bias;  // [D] or null
    const void *z;      // [B][L][D] gate or null
    bool softplus;      // plan flag SSCAN_DELTA_SOFTPLUS
    bool on() const { return bias != nullptr || z != nullptr || softplus; }
};

// ------------------------------------------------------------ generic launch

template <class IO, int NL, int LPC>
cudaError_t launch_generic_t(const sscan_plan *p, const void *u, const void *dl, const float *A,
                             const void *Bm, const void *Cm, const float *h0, void *y, float *hf,
                             const Fused &fu, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>(ceil_div(p->D, kGenericThreads / LPC)), static_cast<unsigned>(p->B));
    auto kern = (p->flags & SSCAN_ZOH) ? sscan_generic_kernel<IO, NL, LPC, true>
                                       : sscan_generic_kernel<IO, NL, LPC, false>;
    kern<<<grid, kGenericThreads, 0, s>>>(
        static_cast<const IO *>(u), static_cast<const IO *>(dl), A, static_cast<const IO *>(Bm),
        static_cast<const IO *>(Cm), h0, static_cast<IO *>(y), hf, p->L, p->D, fu.bias,
        static_cast<const IO *>(fu.z), fu.softplus ? 1 : 0);
    return cudaGetLastError();
}

template <class IO>
cudaError_t launch_generic(const sscan_plan *p, const void *u, const void *dl, const float *A,
                           const void *Bm, const void *Cm, const float *h0, void *y, float *hf,
                           const Fused &fu, cudaStream_t s) {
    switch (p->N) {
        case 16: return launch_generic_t<IO, 8, 2>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
        case 32: return launch_generic_t<IO, 16, 2>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
        default: return launch_generic_t<IO, 16, 4>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
    }
}

// --------------------------------------------------------------- step launch

template <class IO, int N>
cudaError_t launch_step_t(const sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                          const void *Cm, const float *h0, void *y, float *hf, const Fused &fu, cudaStream_t s) {
    constexpr int per_block = kStepThreads / (N / 4) * kStepItems;  // channels per block
    const dim3 grid(static_cast<unsigned>(ceil_div(p->D, per_block)), static_cast<unsigned>(p->B));
    auto kern = (p->flags & SSCAN_ZOH) ? sscan_step_kernel<IO, N, true> : sscan_step_kernel<IO, N, false>;
    kern<<<grid, kStepThreads, 0, s>>>(static_cast<const IO *>(u), static_cast<const IO *>(dl), A,
                                       static_cast<const IO *>(Bm), static_cast<const IO *>(Cm), h0,
                                       static_cast<IO *>(y), hf, p->L, p->D, fu.bias,
                                       static_cast<const IO *>(fu.z), fu.softplus ? 1 : 0);
    return cudaGetLastError();
}

template <class IO>
cudaError_t launch_step(const sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                        const void *Cm, const float *h0, void *y, float *hf, const Fused &fu, cudaStream_t s) {
    switch (p->N) {
        case 16: return launch_step_t<IO, 16>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
        case 32: return launch_step_t<IO, 32>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
        default: return launch_step_t<IO, 64>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
    }
}

template <class IO, int N, bool ZOH>
int launch_decode_t(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm, const void *Cm,
                    const float *h0, void *y, float *hf, const Fused &fu, cudaStream_t s) {
    using Cfg = DecodeCfg<IO, N>;
    auto kern = sscan_decode_kernel<IO, N, ZOH>;
    if (smem_opt_in<sscan_decode_kernel<IO, N, ZOH>>(Cfg::kSmem) != cudaSuccess) return SSCAN_ERR_CUDA;
    if (p->dec_grid == 0) {
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kDecThreads, Cfg::kSmem) != cudaSuccess)
            return SSCAN_ERR_CUDA;
        // the walk of sscan_decode_kernel: with R channel ranges and at most `slots` resident
        // blocks, K = min(B, slots / R) blocks per range (grid K * R), else one block per slot
        const int64_t R = ceil_div(p->D, Cfg::TD);
        const int64_t slots = static_cast<int64_t>(occ > 0 ? occ : 1) * p->sm_count;
        const int64_t K = std::min<int64_t>(p->B, slots / R);
        p->dec_grid = static_cast<int>(R <= slots ? K * R : slots);
    }
    kern<<<p->dec_grid, kDecThreads, Cfg::kSmem, s>>>(
        static_cast<const IO *>(u), static_cast<const IO *>(dl), A, static_cast<const IO *>(Bm),
        static_cast<const IO *>(Cm), h0, static_cast<IO *>(y), hf, p->B, p->D, fu.bias,
        static_cast<const IO *>(fu.z), fu.softplus ? 1 : 0, p->d_status);
    return cudaGetLastError() == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

template <class IO>
int launch_decode(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm, const void *Cm,
                  const float *h0, void *y, float *hf, const Fused &fu, cudaStream_t s) {
    const bool zoh = (p->flags & SSCAN_ZOH) != 0;
    switch (p->N) {
        case 16: return zoh ? launch_decode_t<IO, 16, true>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s)
                            : launch_decode_t<IO, 16, false>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
        case 32: return zoh ? launch_decode_t<IO, 32, true>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s)
                            : launch_decode_t<IO, 32, false>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
        default: return zoh ? launch_decode_t<IO, 64, true>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s)
                            : launch_decode_t<IO, 64, false>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s);
    }
}

// ------------------------------------------------------------ chained launch

// L2 promotion of 64 bytes: a u or delta tile row is only CPW * es bytes (16 to 64)
// and the neighbouring channels of the same row belong to other chains, reached by
// other warps at other times; 256-byte promotion measured 1.4x (f32, 64-byte rows)
// to 10x (bf16 with N = 64, 16-byte rows) the DRAM bytes the inputs hold.
bool encode_map(CUtensorMap *m, const void *ptr, int es, uint64_t inner, uint64_t rows, uint32_t box_inner,
                uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * static_cast<uint64_t>(es)};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(m, es == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                           const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_64B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <class IO, int CFG, bool ZOH, bool POLY, bool SPLIT, bool FUSED>
int launch_chained_t(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                     const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                     cudaStream_t s) {
    constexpr KCfg k = kChainedCfgs[CFG];
    using Cfg = ChainedCfg<IO, k.N, k.NL, k.T, k.STAGES, k.WPC>;
    if constexpr (FUSED && !Cfg::kHelp && Cfg::kSmemF > kMaxSmem) {
        // the fused stage ring of this shape does not fit: the generic kernel serves the call
        (void)ws;
        return launch_generic<IO>(p, u, dl, A, Bm, Cm, h0, y, hf, fu, s) == cudaSuccess ? SSCAN_OK
                                                                                       : SSCAN_ERR_CUDA;
    } else {
    constexpr bool help = FUSED && Cfg::kHelp;  // helper warps (see ChainedCfg::kHelp)
    constexpr int smem_bytes = help ? Cfg::kSmemH : (FUSED ? Cfg::kSmemF : Cfg::kSmem);
    constexpr int threads = help ? Cfg::kThreadsH : Cfg::kThreads;
    auto kern = sscan_chained_kernel<IO, Cfg, ZOH, POLY, SPLIT, FUSED>;
    if (smem_opt_in<sscan_chained_kernel<IO, Cfg, ZOH, POLY, SPLIT, FUSED>>(smem_bytes) != cudaSuccess)
        return SSCAN_ERR_CUDA;

    const int es = sizeof(IO);
    const void *ptrs[5] = {u, dl, Bm, Cm, fu.z};
    if (!p->tm_valid || memcmp(ptrs, p->tm_ptr, sizeof ptrs) != 0) {
        const uint64_t rows = static_cast<uint64_t>(p->B * p->L);
        if (!encode_map(&p->tm[0], u, es, p->D, rows, Cfg::CPW, Cfg::T) ||
            !encode_map(&p->tm[1], dl, es, p->D, rows, Cfg::CPW, Cfg::T) ||
            !encode_map(&p->tm[2], Bm, es, p->N, rows, p->N, Cfg::T) ||
            !encode_map(&p->tm[3], Cm, es, p->N, rows, p->N, Cfg::T) ||
            (fu.z != nullptr && !encode_map(&p->tm[4], fu.z, es, p->D, rows, Cfg::CPW, Cfg::T))) {
            p->tm_valid = false;
            return SSCAN_ERR_CUDA;
        }
        if (fu.z == nullptr) p->tm[4] = p->tm[0];  // never loaded (the kernel sees no gate)
        memcpy(p->tm_ptr, ptrs, sizeof ptrs);
        p->tm_valid = true;
    }
    unsigned char *w = static_cast<unsigned char *>(ws);
    unsigned long long *flags = reinterpret_cast<unsigned long long *>(w + p->flag_off);
    if (ws != p->last_ws) {  // a workspace seen for the first time: clear its flags once
        if (cudaMemsetAsync(flags, 0, p->flag_bytes, s) != cudaSuccess) return SSCAN_ERR_CUDA;
        p->last_ws = ws;
    }
    uint32_t ep = g_epoch.fetch_add(1);
    if (ep == 0) ep = g_epoch.fetch_add(1);
    ChainedParams prm;
    prm.A = A;
    prm.h0 = h0;
    prm.y = y;
    prm.h_final = hf;
    prm.carry = reinterpret_cast<float *>(w);
    prm.flags = flags;
    prm.delta = dl;
    prm.Cm = Cm;
    prm.rec_h = reinterpret_cast<float *>(w);
    prm.rec_s = reinterpret_cast<float *>(w + p->rec_s_off);
    prm.rec_mono = reinterpret_cast<int *>(w + p->rec_mono_off);
    prm.rec_flags = flags;
    prm.max_pieces = p->max_pieces;
    prm.ysink = w + p->sink_off;
    prm.drop_publish = p->drop_publish ? 1 : 0;
    prm.status = p->d_status;
    prm.epoch_hi = static_cast<unsigned long long>(ep) << 32;
    prm.L = p->L;
    prm.D = p->D;
    prm.chains_per_row = p->chains_per_row;
    prm.chains = p->chains;
    prm.seg = p->seg;
    prm.seg_shift = p->seg_shift;
    prm.wpc = k.WPC;
    prm.delta_bias = fu.bias;
    prm.z = fu.z;
    prm.softplus = fu.softplus ? 1 : 0;
    void *args[] = {&p->tm[0], &p->tm[1], &p->tm[2], &p->tm[3], &p->tm[4], &prm};
    const dim3 grid(static_cast<unsigned>(p->workers / k.WPC)), block(threads);
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), grid, block, args,
                                                      smem_bytes, s);
    return e == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
    }
}

// Fused calls (bias, softplus or gate) take the FUSED kernels, which keep every
// exponent on the MUFU pipe.
template <class IO, int CFG, bool SPLIT>
int launch_chained_mode(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                        const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                        cudaStream_t s) {
    const bool zoh = (p->flags & SSCAN_ZOH) != 0;
    if (fu.on())
        return zoh ? launch_chained_t<IO, CFG, true, false, SPLIT, true>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s)
                   : launch_chained_t<IO, CFG, false, false, SPLIT, true>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
    if (zoh)
        return launch_chained_t<IO, CFG, true, false, SPLIT, false>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
    if (p->poly)
        return launch_chained_t<IO, CFG, false, true, SPLIT, false>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
    return launch_chained_t<IO, CFG, false, false, SPLIT, false>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
}

template <class IO, int CFG>
int launch_chained_cfg(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                       const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                       cudaStream_t s) {
    return p->split ? launch_chained_mode<IO, CFG, true>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s)
                    : launch_chained_mode<IO, CFG, false>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
}

template <class IO>
int launch_chained(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                   const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                   cudaStream_t s) {
    switch (p->cfg) {
        case 0: return launch_chained_cfg<IO, 0>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 1: return launch_chained_cfg<IO, 1>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 2: return launch_chained_cfg<IO, 2>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 3: return launch_chained_cfg<IO, 3>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 4: return launch_chained_cfg<IO, 4>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 5: return launch_chained_cfg<IO, 5>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 6: return launch_chained_cfg<IO, 6>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        default: return SSCAN_ERR_UNSUPPORTED;
    }
}

// ------------------------------------------------------------- tiled launch

template <class IO, int CFG, bool ZOH, bool FUSED>
int launch_tiled_t(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                   const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                   cudaStream_t s) {
    constexpr KCfg k = kTiledCfgs[CFG];
    using Cfg = TiledCfg<IO, k.N, k.NL, k.T, k.STAGES, k.WPC>;
    auto kern = sscan_tiled_kernel<IO, Cfg, ZOH, FUSED>;
    if (smem_opt_in<sscan_tiled_kernel<IO, Cfg, ZOH, FUSED>>(Cfg::kSmem) != cudaSuccess) return SSCAN_ERR_CUDA;
    const int es = sizeof(IO);
    const void *ptrs[5] = {u, dl, Bm, Cm, fu.z};
    if (!p->tm_valid || memcmp(ptrs, p->tm_ptr, sizeof ptrs) != 0) {
        const uint64_t rows = static_cast<uint64_t>(p->B * p->L);
        if (!encode_map(&p->tm[0], u, es, p->D, rows, Cfg::CPB, Cfg::T) ||
            !encode_map(&p->tm[1], dl, es, p->D, rows, Cfg::CPB, Cfg::T) ||
            !encode_map(&p->tm[2], Bm, es, p->N, rows, p->N, Cfg::T) ||
            !encode_map(&p->tm[3], Cm, es, p->N, rows, p->N, Cfg::T) ||
            (fu.z != nullptr && !encode_map(&p->tm[4], fu.z, es, p->D, rows, Cfg::CPB, Cfg::T))) {
            p->tm_valid = false;
            return SSCAN_ERR_CUDA;
        }
        if (fu.z == nullptr) p->tm[4] = p->tm[0];  // never loaded (the kernel sees no gate)
        memcpy(p->tm_ptr, ptrs, sizeof ptrs);
        p->tm_valid = true;
    }
    unsigned char *w = static_cast<unsigned char *>(ws);
    unsigned long long *flags = reinterpret_cast<unsigned long long *>(w + p->flag_off);
    if (ws != p->last_ws) {  // a workspace seen for the first time: clear its flags once
        if (cudaMemsetAsync(flags, 0, p->flag_bytes, s) != cudaSuccess) return SSCAN_ERR_CUDA;
        p->last_ws = ws;
    }
    uint32_t ep = g_epoch.fetch_add(1);
    if (ep == 0) ep = g_epoch.fetch_add(1);
    ChainedParams prm;
    memset(&prm, 0, sizeof prm);
    prm.A = A;
    prm.h0 = h0;
    prm.y = y;
    prm.h_final = hf;
    prm.carry = reinterpret_cast<float *>(w);
    prm.flags = flags;
    prm.ysink = w + p->sink_off;
    prm.drop_publish = p->drop_publish ? 1 : 0;
    prm.status = p->d_status;
    prm.epoch_hi = static_cast<unsigned long long>(ep) << 32;
    prm.L = p->L;
    prm.D = p->D;
    prm.chains_per_row = p->chains_per_row;
    prm.chains = p->chains;
    prm.seg = p->seg;
    prm.seg_shift = 0;
    prm.wpc = 1;  // one segment per block
    prm.delta_bias = fu.bias;
    prm.z = fu.z;
    prm.softplus = fu.softplus ? 1 : 0;
    void *args[] = {&p->tm[0], &p->tm[1], &p->tm[2], &p->tm[3], &p->tm[4], &prm};
    const dim3 grid(static_cast<unsigned>(p->workers / k.WPC)), block(Cfg::kThreads);
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), grid, block, args,
                                                      Cfg::kSmem, s);
    return e == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

template <class IO, int CFG>
int launch_tiled_cfg(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                     const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                     cudaStream_t s) {
    const bool zoh = (p->flags & SSCAN_ZOH) != 0;
    if (fu.on())
        return zoh ? launch_tiled_t<IO, CFG, true, true>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s)
                   : launch_tiled_t<IO, CFG, false, true>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
    return zoh ? launch_tiled_t<IO, CFG, true, false>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s)
               : launch_tiled_t<IO, CFG, false, false>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
}

template <class IO>
int launch_tiled(sscan_plan *p, const void *u, const void *dl, const float *A, const void *Bm,
                 const void *Cm, const float *h0, void *y, float *hf, void *ws, const Fused &fu,
                 cudaStream_t s) {
    switch (p->cfg) {
        case 0: return launch_tiled_cfg<IO, 0>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 1: return launch_tiled_cfg<IO, 1>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        case 2: return launch_tiled_cfg<IO, 2>(p, u, dl, A, Bm, Cm, h0, y, hf, ws, fu, s);
        default: return SSCAN_ERR_UNSUPPORTED;
    }
}

}  // namespace

void sscan_choose_schedule(sscan_plan *p) { choose_schedule(p); }

// No tokens: the final state is the initial one (zero without h0).
int step_empty(const sscan_plan *p, const float *h0, float *hf, cudaStream_t s) {
    if (hf == nullptr || hf == h0) return SSCAN_OK;
    const size_t bytes = static_cast<size_t>(p->B * p->D * p->N) * sizeof(float);
    const cudaError_t e = h0 ? cudaMemcpyAsync(hf, h0, bytes, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(hf, 0, bytes, s);
    return e == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

// ------------------------------------------------ allocation-free entry point

namespace {

// Scratch for sscan_forward_noalloc: a fixed array in the library's own device
// image instead of a caller- or library-allocated buffer.  Every device that
// loads the library holds these bytes until the process exits.  Layout: the
// 4-byte device status word at offset 0, the kernel's workspace from offset 256.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr size_t kNoAllocWorkspaceOffset = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_addr[kMaxDevices] = {};

// The scratch array's device address on device `dev` (the current device).  In
// host code the symbol itself is only a host-side stand-in, so the address is
// looked up once per device and cached.
int noalloc_scratch(int dev, unsigned char **out) {
    if (dev < 0 || dev >= kMaxDevices) return SSCAN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SSCAN_ERR_CUDA;
        g_noalloc_addr[dev] = ptr;
    }
    *out = static_cast<unsigned char *>(g_noalloc_addr[dev]);
    return SSCAN_OK;
}

}  // namespace

extern "C" {

int sscan_version(void) { return SSCAN_VERSION; }

const char *sscan_status_string(int status) {
    switch (status) {
        case SSCAN_OK: return "ok";
        case SSCAN_ERR_INVALID: return "invalid argument";
        case SSCAN_ERR_UNSUPPORTED: return "unsupported configuration";
        case SSCAN_ERR_ALIGN: return "pointer not 16-byte aligned";
        case SSCAN_ERR_CUDA: return "CUDA error";
        case SSCAN_ERR_TIMEOUT: return "device wait timed out";
        case SSCAN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        default: return "unknown status";
    }
}

int sscan_plan_create(sscan_plan_t *plan, int64_t B, int64_t L, int64_t D, int64_t N, int dtype,
                      uint32_t flags) {
    if (!plan) return SSCAN_ERR_INVALID;
    *plan = nullptr;
    if (B < 1 || D < 1 || L < 0) return SSCAN_ERR_INVALID;
    if (B > 65535 || D > (int64_t(1) << 31) || L > (int64_t(1) << 40)) return SSCAN_ERR_UNSUPPORTED;
    if (dtype != SSCAN_F32 && dtype != SSCAN_BF16) return SSCAN_ERR_INVALID;
    if (flags & ~static_cast<uint32_t>(SSCAN_ZOH | SSCAN_DELTA_SOFTPLUS)) return SSCAN_ERR_INVALID;
    if (N != 16 && N != 32 && N != 64) return SSCAN_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSCAN_ERR_UNSUPPORTED;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SSCAN_ERR_CUDA;
    sscan_plan *p = new (std::nothrow) sscan_plan();
    if (!p) return SSCAN_ERR_INVALID;
    p->B = B;
    p->L = L;
    p->D = D;
    p->N = N;
    p->dtype = dtype;
    p->flags = flags;
    p->device = dev;
    p->sm_count = sms;
    p->d_status = nullptr;
    p->last_ws = nullptr;
    p->tm_valid = false;
    p->ws_bytes = 0;
    p->host = nullptr;
    choose_schedule(p);
    if (cudaMalloc(&p->d_status, sizeof(int)) != cudaSuccess ||
        cudaMemset(p->d_status, 0, sizeof(int)) != cudaSuccess) {
        if (p->d_status) cudaFree(p->d_status);
        delete p;
        return SSCAN_ERR_CUDA;
    }
    *plan = p;
    return SSCAN_OK;
}

void sscan_plan_destroy(sscan_plan_t plan) {
    if (!plan) return;
    sscan_host_pipe_free(plan->host);
    if (plan->d_status) cudaFree(plan->d_status);
    delete plan;
}

size_t sscan_workspace_bytes(sscan_plan_t plan) { return plan ? plan->ws_bytes : 0; }

int sscan_plan_describe(sscan_plan_t plan, char *buf, size_t len) {
    if (!plan) return -1;
    char tmp[512];
    int n;
    if (plan->mode == kTiled) {
        const KCfg &k = kTiledCfgs[plan->cfg];
        n = snprintf(tmp, sizeof tmp,
                     "kernel=tiled B=%lld L=%lld D=%lld N=%lld dtype=%s zoh=%d states_per_thread=%d "
                     "threads_per_channel=%d channels_per_warp=%d warps_per_block=%d channels_per_block=%d "
                     "tokens_per_stage=%d stages=%d split=0 chains=%lld blocks=%lld segment=%lld workspace=%zu "
                     "sms=%d",
                     (long long)plan->B, (long long)plan->L, (long long)plan->D, (long long)plan->N,
                     plan->dtype == SSCAN_F32 ? "f32" : "bf16", (plan->flags & SSCAN_ZOH) ? 1 : 0, k.NL,
                     k.N / k.NL, 32 / (k.N / k.NL), k.WPC, k.WPC * (32 / (k.N / k.NL)), k.T, k.STAGES,
                     (long long)plan->chains, (long long)(plan->workers / k.WPC), (long long)plan->seg,
                     plan->ws_bytes, plan->sm_count);
    } else if (plan->mode == kChained) {
        const KCfg &k = kChainedCfgs[plan->cfg];
        n = snprintf(tmp, sizeof tmp,
                     "kernel=chained B=%lld L=%lld D=%lld N=%lld dtype=%s zoh=%d states_per_thread=%d "
                     "threads_per_channel=%d channels_per_warp=%d warps_per_block=%d tokens_per_stage=%d "
                     "stages=%d fma_pipe_exp=%d split=%d chains=%lld warps=%lld segment=%lld shift=%lld workspace=%zu "
                     "sms=%d",
                     (long long)plan->B, (long long)plan->L, (long long)plan->D, (long long)plan->N,
                     plan->dtype == SSCAN_F32 ? "f32" : "bf16", (plan->flags & SSCAN_ZOH) ? 1 : 0, k.NL,
                     k.N / k.NL, 32 / (k.N / k.NL), k.WPC, k.T, k.STAGES, plan->poly ? 1 : 0,
                     plan->split ? 1 : 0,
                     (long long)plan->chains, (long long)plan->workers, (long long)plan->seg, (long long)plan->seg_shift, plan->ws_bytes,
                     plan->sm_count);
    } else if (plan->mode == kStep && plan->decode) {
        n = snprintf(tmp, sizeof tmp,
                     "kernel=decode B=%lld L=%lld D=%lld N=%lld dtype=%s zoh=%d states_per_thread=4 "
                     "threads_per_channel=%lld stages=%d tile_state_bytes=%d threads=%d sms=%d "
                     "(the step kernel when h0 is NULL)",
                     (long long)plan->B, (long long)plan->L, (long long)plan->D, (long long)plan->N,
                     plan->dtype == SSCAN_F32 ? "f32" : "bf16", (plan->flags & SSCAN_ZOH) ? 1 : 0,
                     (long long)(plan->N / 4), kDecStages, kDecTileStateBytes, kDecThreads, plan->sm_count);
    } else if (plan->mode == kStep) {
        n = snprintf(tmp, sizeof tmp,
                     "kernel=step B=%lld L=%lld D=%lld N=%lld dtype=%s zoh=%d states_per_thread=4 "
                     "threads_per_channel=%lld channels_per_thread=%d block=%d sms=%d",
                     (long long)plan->B, (long long)plan->L, (long long)plan->D, (long long)plan->N,
                     plan->dtype == SSCAN_F32 ? "f32" : "bf16", (plan->flags & SSCAN_ZOH) ? 1 : 0,
                     (long long)(plan->N / 4), kStepItems, kStepThreads, plan->sm_count);
    } else {
        n = snprintf(tmp, sizeof tmp,
                     "kernel=generic B=%lld L=%lld D=%lld N=%lld dtype=%s zoh=%d states_per_thread=%d "
                     "threads_per_channel=%d block=%d sms=%d",
                     (long long)plan->B, (long long)plan->L, (long long)plan->D, (long long)plan->N,
                     plan->dtype == SSCAN_F32 ? "f32" : "bf16", (plan->flags & SSCAN_ZOH) ? 1 : 0,
                     plan->g_nl, plan->g_lpc, kGenericThreads, plan->sm_count);
    }
    if (buf && len) {
        strncpy(buf, tmp, len - 1);
        buf[len - 1] = '\0';
    }
    return n;
}

int sscan_forward(sscan_plan_t plan, const void *u, const void *delta, const float *A,
                  const void *B, const void *C, const float *h0, void *y, float *h_final,
                  void *workspace, void *stream) {
    return sscan_forward_gated(plan, u, delta, A, B, C, h0, nullptr, nullptr, y, h_final, workspace, stream);
}

int sscan_forward_gated(sscan_plan_t plan, const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *h0, const float *delta_bias,
                        const void *z, void *y, float *h_final, void *workspace, void *stream) {
    if (!plan) return SSCAN_ERR_INVALID;
    sscan_plan *p = plan;
    const size_t es = p->dtype == SSCAN_F32 ? 4 : 2;
    const size_t n_bld = static_cast<size_t>(p->B * p->L * p->D);
    const size_t n_bln = static_cast<size_t>(p->B * p->L * p->N);
    const size_t n_dn = static_cast<size_t>(p->D * p->N);
    const size_t n_bdn = static_cast<size_t>(p->B * p->D * p->N);
    if (!A) return SSCAN_ERR_INVALID;
    if (n_bld && (!u || !delta || !y)) return SSCAN_ERR_INVALID;
    if (n_bln && (!B || !C)) return SSCAN_ERR_INVALID;
    const void *ptrs[] = {u, delta, A, B, C, h0, y, h_final, delta_bias, z};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSCAN_ERR_ALIGN;
    // y must not overlap any input; h_final may equal h0 but not overlap anything else
    const void *ins[] = {u, delta, A, B, C, delta_bias, z, h0};
    const size_t insz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * es, n_bln * es,
                           static_cast<size_t>(p->D) * 4, n_bld * es, n_bdn * 4};
    for (int i = 0; i < 8; ++i) {
        if (overlaps(y, n_bld * es, ins[i], insz[i])) return SSCAN_ERR_INVALID;
        if (i < 7 && overlaps(h_final, n_bdn * 4, ins[i], insz[i])) return SSCAN_ERR_INVALID;
    }
    const Fused fu{delta_bias, z, (p->flags & SSCAN_DELTA_SOFTPLUS) != 0};
    if (h0 && h_final && h0 != h_final && overlaps(h_final, n_bdn * 4, h0, n_bdn * 4))
        return SSCAN_ERR_INVALID;
    if (overlaps(h_final, n_bdn * 4, y, n_bld * es)) return SSCAN_ERR_INVALID;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p->mode == kChained || p->mode == kTiled) {
        if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SSCAN_ERR_WORKSPACE;
        const size_t sz[10] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * es, n_bln * es,
                               n_bdn * 4, n_bld * es, n_bdn * 4, static_cast<size_t>(p->D) * 4, n_bld * es};
        for (int i = 0; i < 10; ++i)
            if (overlaps(workspace, p->ws_bytes, ptrs[i], sz[i])) return SSCAN_ERR_WORKSPACE;
        if (p->mode == kTiled)
            return p->dtype == SSCAN_F32
                       ? launch_tiled<float>(p, u, delta, A, B, C, h0, y, h_final, workspace, fu, s)
                       : launch_tiled<uint16_t>(p, u, delta, A, B, C, h0, y, h_final, workspace, fu, s);
        return p->dtype == SSCAN_F32
                   ? launch_chained<float>(p, u, delta, A, B, C, h0, y, h_final, workspace, fu, s)
                   : launch_chained<uint16_t>(p, u, delta, A, B, C, h0, y, h_final, workspace, fu, s);
    }
    if (p->mode == kStep) {
        if (p->L == 0) return step_empty(p, h0, h_final, s);
        if (p->decode && h0 != nullptr)
            return p->dtype == SSCAN_F32 ? launch_decode<float>(p, u, delta, A, B, C, h0, y, h_final, fu, s)
                                         : launch_decode<uint16_t>(p, u, delta, A, B, C, h0, y, h_final, fu, s);
        const cudaError_t e =
            p->dtype == SSCAN_F32 ? launch_step<float>(p, u, delta, A, B, C, h0, y, h_final, fu, s)
                                  : launch_step<uint16_t>(p, u, delta, A, B, C, h0, y, h_final, fu, s);
        return e == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
    }
    const cudaError_t e =
        p->dtype == SSCAN_F32 ? launch_generic<float>(p, u, delta, A, B, C, h0, y, h_final, fu, s)
                              : launch_generic<uint16_t>(p, u, delta, A, B, C, h0, y, h_final, fu, s);
    return e == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

int sscan_get_status(sscan_plan_t plan, void *stream) {
    if (!plan) return SSCAN_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, plan->d_status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(plan->d_status, 0, sizeof(int), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SSCAN_ERR_CUDA;
    return v == 0 ? SSCAN_OK : SSCAN_ERR_TIMEOUT;
}

int sscan_noalloc_status(void *stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSCAN_ERR_UNSUPPORTED;
    unsigned char *scratch = nullptr;
    const int rc = noalloc_scratch(dev, &scratch);
    if (rc != SSCAN_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, scratch, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(scratch, 0, sizeof(int), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return SSCAN_ERR_CUDA;
    return v == 0 ? SSCAN_OK : SSCAN_ERR_TIMEOUT;
}

int sscan_forward_noalloc(int64_t B, int64_t L, int64_t D, int64_t N, int dtype, uint32_t flags,
                          const void *u, const void *delta, const float *A, const void *Bm, const void *Cm,
                          const float *h0, void *y, float *h_final, void *stream) {
    // the same size checks as sscan_plan_create, without allocating a plan
    if (B < 1 || D < 1 || L < 0) return SSCAN_ERR_INVALID;
    if (B > 65535 || D > (int64_t(1) << 31) || L > (int64_t(1) << 40)) return SSCAN_ERR_UNSUPPORTED;
    if (dtype != SSCAN_F32 && dtype != SSCAN_BF16) return SSCAN_ERR_INVALID;
    if (flags & ~static_cast<uint32_t>(SSCAN_ZOH | SSCAN_DELTA_SOFTPLUS)) return SSCAN_ERR_INVALID;
    if (N != 16 && N != 32 && N != 64) return SSCAN_ERR_UNSUPPORTED;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSCAN_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SSCAN_ERR_CUDA;
    unsigned char *scratch = nullptr;
    const int rc = noalloc_scratch(dev, &scratch);
    if (rc != SSCAN_OK) return rc;
    sscan_plan p{};  // on the stack: same schedule as a plan for this shape
    p.B = B;
    p.L = L;
    p.D = D;
    p.N = N;
    p.dtype = dtype;
    p.flags = flags;
    p.device = dev;
    p.sm_count = sms;
    p.last_ws = nullptr;  // the launch clears the workspace flags it uses
    p.tm_valid = false;
    p.ws_bytes = 0;
    choose_schedule(&p);
    if (p.ws_bytes > kNoAllocScratchBytes - kNoAllocWorkspaceOffset) return SSCAN_ERR_WORKSPACE;
    p.d_status = reinterpret_cast<int *>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(p.d_status, 0, sizeof(int), s) != cudaSuccess) return SSCAN_ERR_CUDA;
    return sscan_forward(&p, u, delta, A, Bm, Cm, h0, y, h_final,
                         p.ws_bytes ? scratch + kNoAllocWorkspaceOffset : nullptr, stream);
}

}  // extern "C"
