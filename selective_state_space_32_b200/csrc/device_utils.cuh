// device_utils.cuh -- device helpers shared by the selective-scan kernels:
// packed f32x2 arithmetic, 2^x on the MUFU and on the FMA pipe, storage-type
// conversion, and the mbarrier / TMA / flag primitives of the chained kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace sscan {

// Opt kernel KERN into `bytes` of dynamic shared memory (above the 48 KB default).
// The attribute belongs to the device that is current when it is set, so it is
// set once per (kernel, device): one bit per device ordinal below 64, and every
// call on a higher ordinal sets it again.
template <auto KERN>
inline cudaError_t smem_opt_in(int bytes) {
    static std::atomic<unsigned long long> done{0};
    int dev = 0;
    const cudaError_t g = cudaGetDevice(&dev);
    if (g != cudaSuccess) return g;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// ------------------------------------------------------------ packed fp32 pairs

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
__device__ __forceinline__ f2 splat2(float v) { return pack2(v, v); }
// -a for a pair (the two sign bits flipped: integer operations, no FP pipe)
__device__ __forceinline__ f2 neg2(f2 a) { return a ^ 0x8000000080000000ull; }

// 2^x on the MUFU pipe (ex2.approx; results below 2^-126 flush to zero)
__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 2^(d*a) for a pair on the FMA pipe, |d*a| <= 125 (the caller clamps d).
// Range reduction: t = d*a + 1.5*2^23 leaves j = round(d*a) in the low
// mantissa bits; f = d*a - j in [-1/2, 1/2]; 2^f = 1 + f*q(f) with q of degree
// 4 fitted for minimax relative error on [-1/2, 1/2] (csrc/gen_exp2_poly.py,
// max relative error 1.7e-7 in fp32); the result's exponent is then raised by
// j with one integer add of j << 23 (t's low bits shifted into the exponent).
__device__ __forceinline__ f2 exp2_fma_pair(f2 dd, f2 a) {
    const f2 kShift = splat2(12582912.0f);  // 1.5 * 2^23
    const f2 kNeg1 = splat2(-1.0f);
    const f2 t = fma2(dd, a, kShift);
    const f2 jn = fma2(t, kNeg1, kShift);   // -round(d*a), exact
    const f2 f = fma2(dd, a, jn);           // d*a - round(d*a)
    f2 q = fma2(splat2(1.326472731307149e-03f), f, splat2(9.671512991189957e-03f));
    q = fma2(q, f, splat2(5.550733581185341e-02f));
    q = fma2(q, f, splat2(2.402224242687225e-01f));
    q = fma2(q, f, splat2(6.931470036506653e-01f));
    q = fma2(q, f, splat2(1.0f));
    float t0, t1, q0, q1;
    unpack2(t, t0, t1);
    unpack2(q, q0, q1);
    const uint32_t r0 = __float_as_uint(q0) + (__float_as_uint(t0) << 23);
    const uint32_t r1 = __float_as_uint(q1) + (__float_as_uint(t1) << 23);
    return pack2(__uint_as_float(r0), __uint_as_float(r1));
}

// psi(e) = phi(e ln 2), phi(z) = (exp(z) - 1) / z, for |e| <= 1/(8 ln 2), i.e.
// |z| <= 1/8, in the variable e = z / ln 2 = delta * A * log2(e) that the
// exponential 2^e already needs: a degree-3 polynomial fitted for minimax
// relative error (csrc/gen_phi_poly.py 3 0.125 --log2; 3.3e-7 max relative
// error of the fp32 Horner evaluation).
__device__ __forceinline__ f2 psi2(f2 e) {
    f2 q = fma2(splat2(1.387602649629116e-02f), e, splat2(8.013805747032166e-02f));
    q = fma2(q, e, splat2(3.4657374024391174e-01f));
    return fma2(q, e, splat2(9.999997615814209e-01f));
}

// Exact ZOH coefficient (exp(z) - 1) / A for a pair, z = d*A, from e = d*A*log2(e)
// (the exponent of abar = 2^e), ia = 1/A and nia = -1/A: d*psi(e) when |z| <= 1/8
// (also at A = 0, where ia is not finite and the other branch is not taken),
// abar*(1/A) - 1/A otherwise (there |abar - 1| >= 0.117, so the 2^-22 relative
// error of abar stays below ~2e-6).
__device__ __forceinline__ f2 zoh_coef_pair(f2 dd, f2 e, f2 ia, f2 nia, f2 abar) {
    const f2 small = mul2(dd, psi2(e));
    const f2 big = fma2(abar, ia, nia);
    float e0, e1, s0, s1, g0, g1;
    unpack2(e, e0, e1);
    unpack2(small, s0, s1);
    unpack2(big, g0, g1);
    constexpr float kLim = 0.18033688011112042f;  // 1/8 / ln 2
    return pack2(fabsf(e0) <= kLim ? s0 : g0, fabsf(e1) <= kLim ? s1 : g1);
}

// The ZOH coefficient to the precision of bf16 I/O, in two packed operations and a
// select: d (the z -> 0 limit: relative error |phi(z) - 1| <= |z|/2) when
// |z| <= 2^-10.5, (abar - 1)/A beyond, as (abar - 1) * (1/A) (abar - 1 is exact
// for abar in [1/2, 2]) or, with FMA, as abar * (1/A) - 1/A in one fused
// operation (-1/A from the sign bits of 1/A); the relative error of abar itself,
// about 2^-22, becomes 2^-22 / |z|.  Both forms stay below 3.5e-4 relative,
// against the 2^-9 rounding of a bf16 output and the bf16 tolerance of 5e-3
// relative L2.  (A = 0 takes the first form: e = 0 there, and ia is not finite.)
// The chained kernel measured faster with the first form on B200, the tiled one
// with the second.
constexpr float kZohBf16Lim = 9.9606e-4f;  // 2^-10.5 / ln 2: the bound on |e| = |delta A| log2 e
template <bool FMA = false>
__device__ __forceinline__ f2 zoh_coef_pair_bf16(f2 dd, f2 e, f2 ia, f2 abar) {
    const f2 big = FMA ? fma2(abar, ia, neg2(ia)) : mul2(add2(abar, splat2(-1.0f)), ia);
    float e0, e1, d0, d1, g0, g1;
    unpack2(e, e0, e1);
    unpack2(dd, d0, d1);
    unpack2(big, g0, g1);
    return pack2(fabsf(e0) <= kZohBf16Lim ? d0 : g0, fabsf(e1) <= kZohBf16Lim ? d1 : g1);
}

// softplus(s) = log(1 + e^s) for the fused prologue.  s itself above 20 (the
// remainder log1p(e^-s) < 2.1e-9 is below half an ulp of s); otherwise with
// w = e^s (MUFU ex2, relative error ~2^-22): for w < 1/8 the Taylor series of
// log1p(w) to w^8 (truncation below w^9/9, i.e. < 7e-9 relative), else
// ln 2 * log2(1 + w) on the MUFU (result >= 0.117 there, so the lg2
// approximation's ~2^-22 absolute error stays below ~2e-6 relative).  Both
// branches are evaluated and one is selected (no divergence).
__device__ __forceinline__ float softplus_f(float s) {
    const float w = ex2(fminf(s, 20.0f) * 1.4426950408889634f);
    float q = fmaf(w, -0.125f, 0.14285714285714285f);
    q = fmaf(q, w, -0.16666666666666666f);
    q = fmaf(q, w, 0.2f);
    q = fmaf(q, w, -0.25f);
    q = fmaf(q, w, 0.3333333333333333f);
    q = fmaf(q, w, -0.5f);
    q = fmaf(q, w, 1.0f);
    const float series = w * q;
    float l;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.0f + w));
    const float big = l * 0.6931471805599453f;
    return s > 20.0f ? s : (w < 0.125f ? series : big);
}

// silu(z) = z * sigmoid(z) = z / (1 + e^-z) with the MUFU reciprocal (relative
// error ~2^-23); 1 + e^-z = inf (z < -88) gives rcp = 0 and silu = -0.
__device__ __forceinline__ float silu_f(float z) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + ex2(-z * 1.4426950408889634f)));
    return z * r;
}

// ------------------------------------------------------------- storage types

template <class IO> struct Io;
template <> struct Io<float> {
    static constexpr int kBytes = 4;
    static __device__ __forceinline__ float ld(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ float widen(float v) { return v; }
    static __device__ __forceinline__ void st(float *p, float v) { *p = v; }
    // NP consecutive pairs (2*NP values) starting at a 16-byte aligned p
    template <int NP>
    static __device__ __forceinline__ void ld_pairs(const float *p, f2 (&out)[NP]) {
        static_assert(NP % 2 == 0, "pairs are loaded 4 values at a time");
#pragma unroll
        for (int i = 0; i < NP / 2; ++i) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(p) + i);
            out[2 * i] = pack2(v.x, v.y);
            out[2 * i + 1] = pack2(v.z, v.w);
        }
    }
};
template <> struct Io<uint16_t> {  // bf16 bit patterns
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ uint16_t ld(const uint16_t *p) { return __ldg(p); }
    static __device__ __forceinline__ float widen(uint16_t v) {
        return __uint_as_float(static_cast<uint32_t>(v) << 16);
    }
    static __device__ __forceinline__ void st(uint16_t *p, float v) {
        uint16_t r;
        asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
        *p = r;
    }
    // NP consecutive pairs (2*NP bf16 values) starting at p (8-byte aligned for NP = 2,
    // 16-byte aligned otherwise); each 32-bit word holds one pair
    template <int NP>
    static __device__ __forceinline__ void ld_pairs(const uint16_t *p, f2 (&out)[NP]) {
        static_assert(NP == 2 || NP % 4 == 0, "pairs are loaded 2 or 4 words at a time");
        if constexpr (NP == 2) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
            out[0] = pack2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u));
            out[1] = pack2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
        } else {
#pragma unroll
            for (int i = 0; i < NP / 4; ++i) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p) + i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)  // low half = even state, high half = odd state
                    out[4 * i + j] = pack2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
            }
        }
    }
};

// ------------------------------------------------- mbarrier / TMA / flag wait

constexpr uint32_t kSpinLimit = 1u << 22;  // bound on every device-side wait loop

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase with the given parity to complete; false if the bound ran out.
// A non-blocking test first: a stage loaded well ahead is normally complete already.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
// mbar_wait for a waiter that is expected to wait: each try suspends the thread
// for up to kSleepHintNs (it resumes as soon as the phase completes) instead of
// spinning through issue slots the other warps need.  Bounded by kSleepLimit tries.
constexpr uint32_t kSleepHintNs = 20000;
constexpr uint32_t kSleepLimit = 1u << 16;
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < kSleepLimit; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(kSleepHintNs)
            : "memory");
        if (ok) return true;
    }
    return false;
}
// 2-D tiled TMA load (no multicast) of box {x, y} into shared memory, completing on bar.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Order this thread's (and, after a warp/CTA barrier, its peers') generic-proxy
// shared-memory accesses before later async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

}  // namespace sscan
