// host_pipe.cu -- sscan_forward_host: the forward pass on host buffers, its
// copies overlapping the scan (pieces of the problem through two device buffer
// slots and three streams).  Host code only: it launches the library's scan
// through sscan_forward_gated on sub-plans of the caller's plan.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>

#include "plan.cuh"
#include "sscan.h"

namespace {

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

// sscan_forward_host cuts the problem into pieces and runs them as a
// three-stage pipeline: copy a piece's inputs in (stream s_in), scan it (the
// caller's stream), copy its outputs out (stream s_out).  Two buffer slots let
// the copies of the neighbouring pieces run while a piece is scanned.  Pieces
// are cut along L, the state carried from piece to piece in one device buffer
// (each piece's h_final is the next one's h0, the split-call resume the scan
// supports exactly), or, for short sequences (a decode step), along the batch
// rows, which are independent (each slot then holds its rows' state).
struct HostPipe {
    bool along_b = false;         // pieces of batch rows (else of tokens)
    int64_t piece = 0, pieces = 0;  // tokens or rows per piece; number of pieces
    sscan_plan *sub[2] = {};  // plans for a full piece and for a shorter last piece
    size_t off_ws[2] = {}, off_A = 0, off_bias = 0, off_h = 0, bytes = 0;
    size_t off_slot[2][7] = {};  // per slot: u, delta, z, B, C, y, and (along_b) the rows' state
    size_t max_pitch = 0;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_join = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
    bool streams_ready = false;
};

namespace {

// A call is cut into at most kHostPieces pieces along L, kHostPiecesB along the batch
// rows.  Measured on B200 with pinned host memory: a host-to-device copy has a large
// fixed cost (4 MB in 0.34 ms, 38 MB in 0.72 ms), so the row pieces of a decode step
// (256 x 2048 x 16 fp32 state) are fastest as two (1.24 ms per call, 1.40 ms as one,
// 1.45 ms as eight); along L (8 x 2048 x 1536 fp32) eight pieces took 4.6 ms, one 5.8 ms.
constexpr int64_t kHostPieces = 8;
constexpr int64_t kHostPiecesB = 2;
constexpr int64_t kHostPieceAlign = 64; // piece lengths along L are multiples of this many tokens

sscan_plan *host_sub_plan(const sscan_plan *p, int64_t B, int64_t L) {
    sscan_plan *q = new (std::nothrow) sscan_plan();
    if (!q) return nullptr;
    q->B = B;
    q->L = L;
    q->D = p->D;
    q->N = p->N;
    q->dtype = p->dtype;
    q->flags = p->flags;
    q->device = p->device;
    q->sm_count = p->sm_count;
    q->d_status = p->d_status;  // shared: sscan_get_status on the parent sees the pieces' waits
    q->last_ws = nullptr;
    q->tm_valid = false;
    q->ws_bytes = 0;
    q->host = nullptr;
    sscan_choose_schedule(q);
    return q;
}

}  // namespace

void sscan_host_pipe_free(HostPipe *h) {
    if (!h) return;
    if (h->s_in) cudaStreamDestroy(h->s_in);
    if (h->s_out) cudaStreamDestroy(h->s_out);
    cudaEvent_t evs[] = {h->ev_join, h->ev_in[0], h->ev_in[1], h->ev_comp[0], h->ev_comp[1],
                         h->ev_out[0], h->ev_out[1]};
    for (cudaEvent_t e : evs)
        if (e) cudaEventDestroy(e);
    delete h->sub[0];  // sub-plans own no device memory (the status word is the parent's)
    delete h->sub[1];
    delete h;
}

namespace {

// Piece schedule and device-workspace layout of sscan_forward_host (host
// arithmetic only; made once per plan).
HostPipe *host_layout(sscan_plan *p) {
    if (p->host) return p->host;
    HostPipe *h = new (std::nothrow) HostPipe();
    if (!h) return nullptr;
    const int64_t L = p->L;
    // sequences too short for several 64-token pieces, with several rows: cut the rows
    h->along_b = L >= 1 && L < kHostPieces * kHostPieceAlign && p->B >= 2;
    int64_t npc = h->along_b ? kHostPiecesB : kHostPieces;  // SSCAN_TUNE="hostpieces=K": 1..64
    if (const char *t = getenv("SSCAN_TUNE"))
        if (const char *c = strstr(t, "hostpieces=")) {
            const int v = atoi(c + 11);
            if (v >= 1 && v <= 64) npc = v;
        }
    int64_t ext, pc;
    if (h->along_b) {
        ext = p->B;
        pc = ceil_div(p->B, npc);
    } else {
        ext = L;
        pc = ceil_div(ceil_div(L, npc), kHostPieceAlign) * kHostPieceAlign;
        if (pc > L) pc = L;
    }
    h->piece = pc;
    h->pieces = ext == 0 ? 1 : ceil_div(ext, pc);
    const int64_t last = ext - (h->pieces - 1) * pc;
    h->sub[0] = h->along_b ? host_sub_plan(p, pc, L) : host_sub_plan(p, p->B, pc);
    h->sub[1] = last == pc ? nullptr : h->along_b ? host_sub_plan(p, last, L) : host_sub_plan(p, p->B, last);
    if (!h->sub[0] || (last != pc && !h->sub[1])) {
        sscan_host_pipe_free(h);
        return nullptr;
    }
    const size_t es = p->dtype == SSCAN_F32 ? 4 : 2;
    size_t o = 0;
    auto take = [&o](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    h->off_ws[0] = take(h->sub[0]->ws_bytes);
    h->off_ws[1] = take(h->sub[1] ? h->sub[1]->ws_bytes : 0);
    h->off_A = take(static_cast<size_t>(p->D * p->N) * 4);
    h->off_bias = take(static_cast<size_t>(p->D) * 4);
    h->off_h = take(h->along_b ? 0 : static_cast<size_t>(p->B * p->D * p->N) * 4);
    const int64_t rows = h->along_b ? pc : p->B, toks = h->along_b ? L : pc;
    const size_t bld = static_cast<size_t>(rows * toks * p->D) * es;
    const size_t bln = static_cast<size_t>(rows * toks * p->N) * es;
    const size_t bdn = h->along_b ? static_cast<size_t>(rows * p->D * p->N) * 4 : 0;
    for (int j = 0; j < 2; ++j) {
        const size_t sizes[7] = {bld, bld, bld, bln, bln, bld, bdn};
        for (int i = 0; i < 7; ++i) h->off_slot[j][i] = take(sizes[i]);
    }
    h->bytes = o;
    p->host = h;
    return h;
}

int host_streams(HostPipe *h, int dev) {
    if (h->streams_ready) return SSCAN_OK;
    int mp = 0;
    bool ok = cudaDeviceGetAttribute(&mp, cudaDevAttrMaxPitch, dev) == cudaSuccess && mp > 0;
    h->max_pitch = static_cast<size_t>(mp);
    if (ok && !h->s_in) ok = cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking) == cudaSuccess;
    if (ok && !h->s_out) ok = cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t *evs[] = {&h->ev_join, &h->ev_in[0], &h->ev_in[1], &h->ev_comp[0], &h->ev_comp[1],
                          &h->ev_out[0], &h->ev_out[1]};
    for (cudaEvent_t *e : evs)
        if (ok && !*e) ok = cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return SSCAN_ERR_CUDA;  // what was made is kept and freed with the plan
    h->streams_ready = true;
    return SSCAN_OK;
}

// `rows` rows of `width` bytes, source rows `spitch` apart, destination rows
// `dpitch` apart (one 2-D copy; row by row past the device's pitch limit).
cudaError_t copy_rows(void *dst, size_t dpitch, const void *src, size_t spitch, size_t width,
                      int64_t rows, size_t max_pitch, cudaStream_t s) {
    if (width == 0 || rows == 0) return cudaSuccess;
    if (dpitch == width && spitch == width)
        return cudaMemcpyAsync(dst, src, width * static_cast<size_t>(rows), cudaMemcpyDefault, s);
    if (dpitch <= max_pitch && spitch <= max_pitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, static_cast<size_t>(rows), cudaMemcpyDefault, s);
    for (int64_t r = 0; r < rows; ++r) {
        const cudaError_t e = cudaMemcpyAsync(static_cast<char *>(dst) + r * dpitch,
                                              static_cast<const char *>(src) + r * spitch, width,
                                              cudaMemcpyDefault, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t sscan_host_workspace_bytes(sscan_plan_t plan) {
    if (!plan) return 0;
    const HostPipe *h = host_layout(plan);
    return h ? h->bytes : 0;
}

int sscan_forward_host(sscan_plan_t plan, const void *u, const void *delta, const float *A,
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
    // the same aliasing rules as sscan_forward_gated, on the caller's buffers
    const void *ins[] = {u, delta, A, B, C, delta_bias, z, h0};
    const size_t insz[] = {n_bld * es, n_bld * es, n_dn * 4, n_bln * es, n_bln * es,
                           static_cast<size_t>(p->D) * 4, n_bld * es, n_bdn * 4};
    for (int i = 0; i < 8; ++i) {
        if (overlaps(y, n_bld * es, ins[i], insz[i])) return SSCAN_ERR_INVALID;
        if (i < 7 && overlaps(h_final, n_bdn * 4, ins[i], insz[i])) return SSCAN_ERR_INVALID;
    }
    if (h0 && h_final && h0 != h_final && overlaps(h_final, n_bdn * 4, h0, n_bdn * 4)) return SSCAN_ERR_INVALID;
    if (overlaps(h_final, n_bdn * 4, y, n_bld * es)) return SSCAN_ERR_INVALID;
    HostPipe *h = host_layout(p);
    if (!h) return SSCAN_ERR_INVALID;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SSCAN_ERR_WORKSPACE;
    for (int i = 0; i < 8; ++i)
        if (overlaps(workspace, h->bytes, ins[i], insz[i])) return SSCAN_ERR_WORKSPACE;
    if (overlaps(workspace, h->bytes, y, n_bld * es) || overlaps(workspace, h->bytes, h_final, n_bdn * 4))
        return SSCAN_ERR_WORKSPACE;
    const int src = host_streams(h, p->device);
    if (src != SSCAN_OK) return src;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char *w = static_cast<unsigned char *>(workspace);
    float *dA = reinterpret_cast<float *>(w + h->off_A);
    float *dbias = reinterpret_cast<float *>(w + h->off_bias);
    float *dh = reinterpret_cast<float *>(w + h->off_h);
    int rc = SSCAN_OK;
    auto ok = [&rc](cudaError_t e) {
        if (e != cudaSuccess && rc == SSCAN_OK) rc = SSCAN_ERR_CUDA;
        return rc == SSCAN_OK;
    };
    do {
        // the internal streams start after the work already queued on `stream`
        if (!ok(cudaEventRecord(h->ev_join, s)) || !ok(cudaStreamWaitEvent(h->s_in, h->ev_join, 0)) ||
            !ok(cudaStreamWaitEvent(h->s_out, h->ev_join, 0)))
            break;
        if (!ok(cudaMemcpyAsync(dA, A, n_dn * 4, cudaMemcpyDefault, h->s_in))) break;
        if (delta_bias && !ok(cudaMemcpyAsync(dbias, delta_bias, static_cast<size_t>(p->D) * 4,
                                              cudaMemcpyDefault, h->s_in)))
            break;
        if (!h->along_b && h0 && !ok(cudaMemcpyAsync(dh, h0, n_bdn * 4, cudaMemcpyDefault, h->s_in))) break;
        const size_t pitch_d = static_cast<size_t>(p->L * p->D) * es, pitch_n = static_cast<size_t>(p->L * p->N) * es;
        const size_t row_h = static_cast<size_t>(p->D * p->N) * 4;  // one batch row's state
        for (int64_t k = 0; k < h->pieces && rc == SSCAN_OK; ++k) {
            const int j = static_cast<int>(k & 1);
            // piece k: batch rows [b0, b0 + nb) x tokens [l0, l0 + lk)
            const int64_t b0 = h->along_b ? k * h->piece : 0;
            const int64_t nb = h->along_b ? std::min(h->piece, p->B - b0) : p->B;
            const int64_t l0 = h->along_b ? 0 : k * h->piece;
            const int64_t lk = h->along_b ? p->L : std::min(h->piece, p->L - l0);
            const int which = (h->along_b ? nb : lk) == h->piece ? 0 : 1;
            sscan_plan *q = h->sub[which];
            unsigned char *slot[7];
            for (int i = 0; i < 7; ++i) slot[i] = w + h->off_slot[j][i];
            // the state: carried in dh along L; the piece's own rows in slot 6 along B (in place)
            float *hst = h->along_b ? reinterpret_cast<float *>(slot[6]) : dh;
            const size_t row_d = static_cast<size_t>(lk * p->D) * es, row_n = static_cast<size_t>(lk * p->N) * es;
            const size_t at_d = static_cast<size_t>((b0 * p->L + l0) * p->D) * es;
            const size_t at_n = static_cast<size_t>((b0 * p->L + l0) * p->N) * es;
            // inputs of piece k into slot j, once the scan of piece k-2 has read it (and, along
            // B, once its state has been copied out of the slot)
            if (k >= 2 && !ok(cudaStreamWaitEvent(h->s_in, h->ev_comp[j], 0))) break;
            if (k >= 2 && h->along_b && !ok(cudaStreamWaitEvent(h->s_in, h->ev_out[j], 0))) break;
            if (!ok(copy_rows(slot[0], row_d, static_cast<const char *>(u) + at_d, pitch_d, row_d, nb, h->max_pitch, h->s_in)) ||
                !ok(copy_rows(slot[1], row_d, static_cast<const char *>(delta) + at_d, pitch_d, row_d, nb, h->max_pitch, h->s_in)) ||
                (z && !ok(copy_rows(slot[2], row_d, static_cast<const char *>(z) + at_d, pitch_d, row_d, nb, h->max_pitch, h->s_in))) ||
                !ok(copy_rows(slot[3], row_n, static_cast<const char *>(B) + at_n, pitch_n, row_n, nb, h->max_pitch, h->s_in)) ||
                !ok(copy_rows(slot[4], row_n, static_cast<const char *>(C) + at_n, pitch_n, row_n, nb, h->max_pitch, h->s_in)) ||
                (h->along_b && h0 && !ok(cudaMemcpyAsync(hst, h0 + b0 * p->D * p->N, static_cast<size_t>(nb) * row_h,
                                                         cudaMemcpyDefault, h->s_in))) ||
                !ok(cudaEventRecord(h->ev_in[j], h->s_in)))
                break;
            // scan piece k once its inputs are in and slot j's previous y has been copied out
            if (!ok(cudaStreamWaitEvent(s, h->ev_in[j], 0))) break;
            if (k >= 2 && !ok(cudaStreamWaitEvent(s, h->ev_out[j], 0))) break;
            const bool has_h0 = h->along_b ? h0 != nullptr : (k > 0 || h0 != nullptr);
            const int frc = sscan_forward_gated(q, slot[0], slot[1], dA, slot[3], slot[4], has_h0 ? hst : nullptr,
                                                delta_bias ? dbias : nullptr, z ? slot[2] : nullptr, slot[5], hst,
                                                w + h->off_ws[which], s);
            if (frc != SSCAN_OK) {
                rc = frc;
                break;
            }
            // y (and, along B, the rows' final state) of piece k out of slot j
            if (!ok(cudaEventRecord(h->ev_comp[j], s)) || !ok(cudaStreamWaitEvent(h->s_out, h->ev_comp[j], 0)) ||
                !ok(copy_rows(static_cast<char *>(y) + at_d, pitch_d, slot[5], row_d, row_d, nb, h->max_pitch, h->s_out)) ||
                (h->along_b && h_final && !ok(cudaMemcpyAsync(h_final + b0 * p->D * p->N, hst, static_cast<size_t>(nb) * row_h,
                                                              cudaMemcpyDefault, h->s_out))) ||
                !ok(cudaEventRecord(h->ev_out[j], h->s_out)))
                break;
        }
        if (rc == SSCAN_OK && h_final && !h->along_b)
            ok(cudaMemcpyAsync(h_final, dh, n_bdn * 4, cudaMemcpyDefault, h->s_out));
    } while (false);
    // `stream` waits for everything queued on the internal streams, on success and on error
    const bool joined = cudaEventRecord(h->ev_join, h->s_in) == cudaSuccess &&
                        cudaStreamWaitEvent(s, h->ev_join, 0) == cudaSuccess &&
                        cudaEventRecord(h->ev_join, h->s_out) == cudaSuccess &&
                        cudaStreamWaitEvent(s, h->ev_join, 0) == cudaSuccess;
    if (!joined && rc == SSCAN_OK) rc = SSCAN_ERR_CUDA;
    return rc;
}

}  // extern "C"
