// sscan.cu -- selective-scan (Mamba / S6) forward for B200 (sm_100a), and the
// C ABI declared in include/sscan.h.
//
// What is computed ("tm_ssm_selective" (Transformer Math page on selective
// SSMs), section "Discretization becomes a per-token operation"; the
// selective_scan reference loop of "12. Selective State Space"):
//     Abar = exp(delta*A[d,n]);   Bbar u = delta*B[n]*u  (Euler) or
//     (exp(delta*A)-1)/A*B[n]*u (ZOH);   h = Abar*h + Bbar u;   y = sum_n C[n]*h.
//
// Design (B200-first; the pages' SRAM-fused kernel for older GPUs is prior art):
//  * Each thread owns NL of the N states of one (b,d) channel in registers
//    for the whole sequence; LPC = N/NL neighbouring lanes share a channel and
//    combine their partial y with warp shuffles.  The [B,L,D,N] tensors
//    (Abar, Bbar u, h over time) never exist outside registers.
//  * fp32 arithmetic throughout, on packed f32x2 FMA/MUL/ADD (two states per
//    instruction) to halve the issue slots; exp through ex2.approx on the
//    MUFU pipe with the log2(e) factor folded into A once per thread.
//  * u/delta are streamed along D (adjacent lanes -> adjacent channels, so
//    loads coalesce) with an 8-token register prefetch ring; B/C rows are
//    shared by every channel of a batch row and come from L1.
//  * The path is ALU bound on B200 (one exp and four FMA-pipe operations per
//    state update against 1-3 bytes of HBM traffic), so no tensor cores.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>

#include "sscan.h"

#define SSCAN_VERSION 100  // 0.1.0

namespace {

// ---------------------------------------------------------------- device utils

typedef unsigned long long f2;  // two fp32 values in one 64-bit register pair

__device__ __forceinline__ f2 pack2(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(f2 v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
    f2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// 2^x on the MUFU pipe (flushes results below 2^-126 to zero)
__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Storage types: fp32 as float, bf16 as its 16-bit pattern.
template <class IO> struct Io;
template <> struct Io<float> {
    static __device__ __forceinline__ float ld(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ float widen(float v) { return v; }
    static __device__ __forceinline__ void st(float *p, float v) { *p = v; }
    // NP consecutive pairs (2*NP values) starting at p (16-byte aligned)
    template <int NP>
    static __device__ __forceinline__ void ld_pairs(const float *p, f2 (&out)[NP]) {
#pragma unroll
        for (int i = 0; i < NP / 2; ++i) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(p) + i);
            out[2 * i] = pack2(v.x, v.y);
            out[2 * i + 1] = pack2(v.z, v.w);
        }
    }
};
template <> struct Io<uint16_t> {
    static __device__ __forceinline__ uint16_t ld(const uint16_t *p) { return __ldg(p); }
    static __device__ __forceinline__ float widen(uint16_t v) {
        return __uint_as_float(static_cast<uint32_t>(v) << 16);
    }
    static __device__ __forceinline__ void st(uint16_t *p, float v) {
        uint16_t r;
        asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
        *p = r;
    }
    template <int NP>
    static __device__ __forceinline__ void ld_pairs(const uint16_t *p, f2 (&out)[NP]) {
#pragma unroll
        for (int i = 0; i < NP / 4; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p) + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)  // low half = even state, high half = odd state
                out[4 * i + j] = pack2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
        }
    }
};

constexpr int kThreads = 128;  // threads per block
constexpr int kPrefetch = 8;   // tokens of u/delta kept in flight per thread

// phi(z) = (exp(z) - 1) / z = sum_k z^k / (k+1)!, truncated after z^7; for
// |z| <= 1/2 the first omitted term is below 1.1e-8 relative.  Coefficients
// are the Taylor series 1/(k+1)!, highest first.
__device__ __forceinline__ f2 phi2(f2 z) {
    const f2 c7 = pack2(1.0f / 40320.0f, 1.0f / 40320.0f);
    const f2 c6 = pack2(1.0f / 5040.0f, 1.0f / 5040.0f);
    const f2 c5 = pack2(1.0f / 720.0f, 1.0f / 720.0f);
    const f2 c4 = pack2(1.0f / 120.0f, 1.0f / 120.0f);
    const f2 c3 = pack2(1.0f / 24.0f, 1.0f / 24.0f);
    const f2 c2 = pack2(1.0f / 6.0f, 1.0f / 6.0f);
    const f2 c1 = pack2(0.5f, 0.5f);
    const f2 c0 = pack2(1.0f, 1.0f);
    f2 q = fma2(c7, z, c6);
    q = fma2(q, z, c5);
    q = fma2(q, z, c4);
    q = fma2(q, z, c3);
    q = fma2(q, z, c2);
    q = fma2(q, z, c1);
    return fma2(q, z, c0);
}

// ------------------------------------------------------------------ kernel

// One block: kThreads/LPC channels of batch row blockIdx.y, channels
// blockIdx.x*(kThreads/LPC) ...; thread (channel c, group g) owns states
// [g*NL, (g+1)*NL).  Lanes of one channel are adjacent (g fastest).
template <class IO, int NL, int LPC, bool ZOH>
__global__ void __launch_bounds__(kThreads)
sscan_fwd_kernel(const IO *__restrict__ u, const IO *__restrict__ delta,
                 const float *__restrict__ A, const IO *__restrict__ Bm,
                 const IO *__restrict__ Cm, const float *h0, IO *__restrict__ y,
                 float *h_final, int64_t L, int64_t D) {
    constexpr int N = NL * LPC;
    constexpr int NP = NL / 2;  // packed pairs per thread
    constexpr int CPB = kThreads / LPC;
    const int g = threadIdx.x % LPC;
    const int64_t b = blockIdx.y;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * CPB + threadIdx.x / LPC;
    const bool valid = d < D;
    const int64_t dc = valid ? d : D - 1;  // ragged tail: read a real channel, store nothing
    const int n0 = g * NL;

    // per-thread constants: A*log2(e) (Abar = 2^(delta*A2)); ZOH also needs A and 1/A
    f2 A2[NP], A1[NP], iA[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const float a0 = __ldg(A + dc * N + n0 + 2 * p), a1 = __ldg(A + dc * N + n0 + 2 * p + 1);
        A2[p] = pack2(static_cast<float>(static_cast<double>(a0) * 1.4426950408889634),
                      static_cast<float>(static_cast<double>(a1) * 1.4426950408889634));
        if (ZOH) {
            A1[p] = pack2(a0, a1);
            iA[p] = pack2(1.0f / a0, 1.0f / a1);
        }
    }
    f2 h[NP];
    const int64_t srow = (b * D + dc) * N + n0;
    if (h0 != nullptr) {
#pragma unroll
        for (int p = 0; p < NP; p += 2) {
            const float4 v = *reinterpret_cast<const float4 *>(h0 + srow + 2 * p);
            h[p] = pack2(v.x, v.y);
            h[p + 1] = pack2(v.z, v.w);
        }
    } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) h[p] = pack2(0.0f, 0.0f);
    }

    const IO *up = u + b * L * D + dc;
    const IO *dp = delta + b * L * D + dc;
    const IO *bp = Bm + b * L * N + n0;
    const IO *cp = Cm + b * L * N + n0;
    IO *yp = y + b * L * D + dc;
    const bool writer = valid && g == 0;

    IO ubuf[kPrefetch], dbuf[kPrefetch];
#pragma unroll
    for (int k = 0; k < kPrefetch; ++k)
        if (k < L) {
            ubuf[k] = Io<IO>::ld(up + k * D);
            dbuf[k] = Io<IO>::ld(dp + k * D);
        }

    for (int64_t t0 = 0; t0 < L; t0 += kPrefetch) {
#pragma unroll
        for (int k = 0; k < kPrefetch; ++k) {
            const int64_t t = t0 + k;
            if (t < L) {
                const float x = Io<IO>::widen(ubuf[k]);
                const float dl = Io<IO>::widen(dbuf[k]);
                if (t + kPrefetch < L) {
                    ubuf[k] = Io<IO>::ld(up + (t + kPrefetch) * D);
                    dbuf[k] = Io<IO>::ld(dp + (t + kPrefetch) * D);
                }
                f2 Bp[NP], Cp[NP];
                Io<IO>::template ld_pairs<NP>(bp + t * N, Bp);
                Io<IO>::template ld_pairs<NP>(cp + t * N, Cp);

                const f2 dd = pack2(dl, dl);
                const float du = dl * x;
                const f2 du2 = pack2(du, du);
                const f2 xx = pack2(x, x);
                f2 ya = pack2(0.0f, 0.0f), yb = pack2(0.0f, 0.0f);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    float e0, e1;
                    unpack2(mul2(dd, A2[p]), e0, e1);
                    const f2 abar = pack2(ex2(e0), ex2(e1));
                    f2 bu;
                    if (!ZOH) {
                        bu = mul2(Bp[p], du2);
                    } else {
                        // (exp(z)-1)/A * B*u with z = delta*A: delta*phi(z) for |z| <= 1/2
                        // (exact at A = 0), (Abar - 1) * (1/A) otherwise.
                        const f2 z = mul2(dd, A1[p]);
                        const f2 small = mul2(dd, phi2(z));
                        const f2 big = mul2(add2(abar, pack2(-1.0f, -1.0f)), iA[p]);
                        float z0, z1, s0, s1, g0, g1;
                        unpack2(z, z0, z1);
                        unpack2(small, s0, s1);
                        unpack2(big, g0, g1);
                        const f2 coef = pack2(fabsf(z0) <= 0.5f ? s0 : g0, fabsf(z1) <= 0.5f ? s1 : g1);
                        bu = mul2(coef, mul2(Bp[p], xx));
                    }
                    h[p] = fma2(abar, h[p], bu);
                    if (p & 1)
                        yb = fma2(Cp[p], h[p], yb);
                    else
                        ya = fma2(Cp[p], h[p], ya);
                }
                float y0, y1;
                unpack2(add2(ya, yb), y0, y1);
                float yv = y0 + y1;
#pragma unroll
                for (int o = 1; o < LPC; o <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
                if (writer) Io<IO>::st(yp + t * D, yv);
            }
        }
    }
    if (h_final != nullptr && valid) {
#pragma unroll
        for (int p = 0; p < NP; p += 2) {
            float a, bq, c, e;
            unpack2(h[p], a, bq);
            unpack2(h[p + 1], c, e);
            *reinterpret_cast<float4 *>(h_final + (b * D + d) * N + n0 + 2 * p) = make_float4(a, bq, c, e);
        }
    }
}

// ------------------------------------------------------------------- host side

struct Schedule {
    int nl;   // states per thread
    int lpc;  // threads per channel
};

}  // namespace

struct sscan_plan {
    int64_t B, L, D, N;
    int dtype;
    uint32_t flags;
    int device;
    int sm_count;
    Schedule sched;
    int *d_status;  // device status word
};

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

Schedule choose_schedule(int64_t N) {
    if (N == 16) return {8, 2};
    if (N == 32) return {16, 2};
    return {16, 4};  // N == 64
}

template <class IO, int NL, int LPC>
cudaError_t launch_t(const sscan_plan *p, const void *u, const void *dl, const float *A,
                     const void *Bm, const void *Cm, const float *h0, void *y, float *hf,
                     cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>((p->D + kThreads / LPC - 1) / (kThreads / LPC)),
                    static_cast<unsigned>(p->B));
    if (p->flags & SSCAN_ZOH)
        sscan_fwd_kernel<IO, NL, LPC, true><<<grid, kThreads, 0, s>>>(
            static_cast<const IO *>(u), static_cast<const IO *>(dl), A, static_cast<const IO *>(Bm),
            static_cast<const IO *>(Cm), h0, static_cast<IO *>(y), hf, p->L, p->D);
    else
        sscan_fwd_kernel<IO, NL, LPC, false><<<grid, kThreads, 0, s>>>(
            static_cast<const IO *>(u), static_cast<const IO *>(dl), A, static_cast<const IO *>(Bm),
            static_cast<const IO *>(Cm), h0, static_cast<IO *>(y), hf, p->L, p->D);
    return cudaGetLastError();
}

template <class IO>
cudaError_t launch_io(const sscan_plan *p, const void *u, const void *dl, const float *A,
                      const void *Bm, const void *Cm, const float *h0, void *y, float *hf,
                      cudaStream_t s) {
    switch (p->N) {
        case 16: return launch_t<IO, 8, 2>(p, u, dl, A, Bm, Cm, h0, y, hf, s);
        case 32: return launch_t<IO, 16, 2>(p, u, dl, A, Bm, Cm, h0, y, hf, s);
        default: return launch_t<IO, 16, 4>(p, u, dl, A, Bm, Cm, h0, y, hf, s);
    }
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
    if (flags & ~static_cast<uint32_t>(SSCAN_ZOH)) return SSCAN_ERR_INVALID;
    if (N != 16 && N != 32 && N != 64) return SSCAN_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSCAN_ERR_UNSUPPORTED;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SSCAN_ERR_CUDA;
    sscan_plan *p = new (std::nothrow) sscan_plan;
    if (!p) return SSCAN_ERR_INVALID;
    p->B = B;
    p->L = L;
    p->D = D;
    p->N = N;
    p->dtype = dtype;
    p->flags = flags;
    p->device = dev;
    p->sm_count = sms;
    p->sched = choose_schedule(N);
    p->d_status = nullptr;
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
    if (plan->d_status) cudaFree(plan->d_status);
    delete plan;
}

size_t sscan_workspace_bytes(sscan_plan_t plan) {
    (void)plan;
    return 0;
}

int sscan_plan_describe(sscan_plan_t plan, char *buf, size_t len) {
    if (!plan) return -1;
    char tmp[256];
    const int n = snprintf(tmp, sizeof tmp,
                           "B=%lld L=%lld D=%lld N=%lld dtype=%s zoh=%d states_per_thread=%d "
                           "threads_per_channel=%d block=%d sms=%d",
                           (long long)plan->B, (long long)plan->L, (long long)plan->D,
                           (long long)plan->N, plan->dtype == SSCAN_F32 ? "f32" : "bf16",
                           (plan->flags & SSCAN_ZOH) ? 1 : 0, plan->sched.nl, plan->sched.lpc,
                           kThreads, plan->sm_count);
    if (buf && len) {
        strncpy(buf, tmp, len - 1);
        buf[len - 1] = '\0';
    }
    return n;
}

int sscan_forward(sscan_plan_t plan, const void *u, const void *delta, const float *A,
                  const void *B, const void *C, const float *h0, void *y, float *h_final,
                  void *workspace, void *stream) {
    (void)workspace;
    if (!plan) return SSCAN_ERR_INVALID;
    const sscan_plan *p = plan;
    const size_t es = p->dtype == SSCAN_F32 ? 4 : 2;
    const size_t n_bld = static_cast<size_t>(p->B * p->L * p->D);
    const size_t n_bln = static_cast<size_t>(p->B * p->L * p->N);
    const size_t n_dn = static_cast<size_t>(p->D * p->N);
    const size_t n_bdn = static_cast<size_t>(p->B * p->D * p->N);
    if (!A) return SSCAN_ERR_INVALID;
    if (n_bld && (!u || !delta || !y)) return SSCAN_ERR_INVALID;
    if (n_bln && (!B || !C)) return SSCAN_ERR_INVALID;
    const void *ptrs[] = {u, delta, A, B, C, h0, y, h_final};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSCAN_ERR_ALIGN;
    // y must not overlap any input; h_final may equal h0 but not overlap anything else
    const void *ins[] = {u, delta, A, B, C, h0};
    const size_t insz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * es, n_bln * es, n_bdn * 4};
    for (int i = 0; i < 6; ++i) {
        if (overlaps(y, n_bld * es, ins[i], insz[i])) return SSCAN_ERR_INVALID;
        if (i < 5 && overlaps(h_final, n_bdn * 4, ins[i], insz[i])) return SSCAN_ERR_INVALID;
    }
    if (h0 && h_final && h0 != h_final && overlaps(h_final, n_bdn * 4, h0, n_bdn * 4))
        return SSCAN_ERR_INVALID;
    if (overlaps(h_final, n_bdn * 4, y, n_bld * es)) return SSCAN_ERR_INVALID;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        p->dtype == SSCAN_F32
            ? launch_io<float>(p, u, delta, A, B, C, h0, y, h_final, s)
            : launch_io<uint16_t>(p, u, delta, A, B, C, h0, y, h_final, s);
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
    return v;
}

}  // extern "C"
