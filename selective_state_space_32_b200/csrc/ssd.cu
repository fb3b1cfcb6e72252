// ssd.cu -- C ABI of the Mamba-2 SSD forward (kernel in kernel_ssd.cuh):
// argument checks, the TMA tensor maps of x, B and C, and the launch.
//
// Shapes ("Mamba & Mamba-2 Architecture", section 3, read with the shapes of
// its section 1): x, y [B][L][H][P] bf16 (H heads of P channels), delta
// [B][L][H] fp32 (one step per head and token), A [H] fp32 (one scalar
// transition per head), B, C [B][L][N] bf16 (shared by all heads), h0 and
// h_final [B][H][N][P] fp32.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "device_utils.cuh"
#include "kernel_ssd.cuh"
#include "sscan.h"

using namespace sscan;

namespace {

bool aligned16_s(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlaps_s(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// bf16 tensor map with a 128-byte swizzle: dims[0] is the contiguous one; the box
// is 64 elements (128 bytes) along it.  Loads outside the tensor read zeros.
bool encode_bf16(CUtensorMap *m, const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
                 const uint32_t *box) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) st[i] = strides_bytes[i];
    }
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), d, st, bx, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

int sscan_ssd_forward(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, const void *x, const float *delta,
                      const float *A, const void *Bm, const void *Cm, const float *h0, void *y, float *h_final,
                      int *status, void *stream) {
    if (B < 1 || H < 1 || L < 0 || P < 1 || N < 1) return SSCAN_ERR_INVALID;
    if (P != ssd::kP || N != ssd::kN) return SSCAN_ERR_UNSUPPORTED;
    if (B * H > (int64_t(1) << 31) - 1 || L > (int64_t(1) << 31) - ssd::kQ || B > (int64_t(1) << 31) - 1)
        return SSCAN_ERR_UNSUPPORTED;
    if (!A) return SSCAN_ERR_INVALID;
    if (L > 0 && (!x || !delta || !Bm || !Cm || !y)) return SSCAN_ERR_INVALID;
    const void *ptrs[] = {x, delta, A, Bm, Cm, h0, y, h_final, status};
    for (const void *q : ptrs)
        if (q && !aligned16_s(q) && q != status) return SSCAN_ERR_ALIGN;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return SSCAN_ERR_ALIGN;
    const size_t n_x = size_t(B) * size_t(L) * size_t(H) * size_t(P);
    const size_t n_bc = size_t(B) * size_t(L) * size_t(N);
    const size_t n_dt = size_t(B) * size_t(L) * size_t(H);
    const size_t n_h = size_t(B) * size_t(H) * size_t(N) * size_t(P);
    const void *ins[] = {x, delta, A, Bm, Cm, h0};
    const size_t insz[] = {n_x * 2, n_dt * 4, size_t(H) * 4, n_bc * 2, n_bc * 2, n_h * 4};
    for (int i = 0; i < 6; ++i) {
        if (overlaps_s(y, n_x * 2, ins[i], insz[i])) return SSCAN_ERR_INVALID;
        if (i < 5 && overlaps_s(h_final, n_h * 4, ins[i], insz[i])) return SSCAN_ERR_INVALID;
    }
    if (h0 && h_final && h0 != h_final && overlaps_s(h_final, n_h * 4, h0, n_h * 4)) return SSCAN_ERR_INVALID;
    if (overlaps_s(h_final, n_h * 4, y, n_x * 2)) return SSCAN_ERR_INVALID;
    if (status && (overlaps_s(status, 4, y, n_x * 2) || overlaps_s(status, 4, h_final, n_h * 4)))
        return SSCAN_ERR_INVALID;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (L == 0) {  // no tokens: the final state is the initial one
        if (!h_final) return SSCAN_OK;
        const cudaError_t e = h0 ? (h0 == h_final ? cudaSuccess
                                                  : cudaMemcpyAsync(h_final, h0, n_h * 4, cudaMemcpyDeviceToDevice, s))
                                 : cudaMemsetAsync(h_final, 0, n_h * 4, s);
        return e == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
    }
    // x as [B][L][H][P]: dims (P, H, L, B), box (64, 1, 128, 1); B and C as [B][L][N]:
    // dims (N, L, B), box (64, 128, 1), loaded as two boxes of 64 states
    CUtensorMap tm_x, tm_b, tm_c;
    const uint64_t dx[4] = {uint64_t(P), uint64_t(H), uint64_t(L), uint64_t(B)};
    const uint64_t sx[3] = {uint64_t(P) * 2, uint64_t(H) * P * 2, uint64_t(L) * H * P * 2};
    const uint32_t bx[4] = {64, 1, ssd::kQ, 1};
    const uint64_t dbc[3] = {uint64_t(N), uint64_t(L), uint64_t(B)};
    const uint64_t sbc[2] = {uint64_t(N) * 2, uint64_t(L) * N * 2};
    const uint32_t bbc[3] = {64, ssd::kQ, 1};
    if (!encode_bf16(&tm_x, x, 4, dx, sx, bx) || !encode_bf16(&tm_b, Bm, 3, dbc, sbc, bbc) ||
        !encode_bf16(&tm_c, Cm, 3, dbc, sbc, bbc))
        return SSCAN_ERR_CUDA;
    if (smem_opt_in<ssd::ssd_forward_kernel>(ssd::kSmemBytes) != cudaSuccess) return SSCAN_ERR_CUDA;
    ssd::Params prm;
    prm.dt = delta;
    prm.A = A;
    prm.h0 = h0;
    prm.y = static_cast<uint16_t *>(y);
    prm.h_final = h_final;
    prm.status = status;
    prm.L = L;
    prm.H = static_cast<int>(H);
    prm.nblocks = static_cast<int>((L + ssd::kQ - 1) / ssd::kQ);
    ssd::ssd_forward_kernel<<<static_cast<unsigned>(B * H), ssd::kThreads, ssd::kSmemBytes, s>>>(tm_x, tm_b, tm_c,
                                                                                                    prm);
    return cudaGetLastError() == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

}  // extern "C"
