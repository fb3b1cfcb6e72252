// plan.cuh -- the plan object of the selective-scan library, shared by the
// library's translation units (sscan.cu: schedules and launches; host_pipe.cu:
// the host-buffer entry point).  Not part of the C ABI.
#pragma once

#include <cuda.h>

#include <cstddef>
#include <cstdint>

enum SscanMode { kGeneric = 0, kChained = 1, kStep = 2, kTiled = 3 };

struct HostPipe;

struct sscan_plan {
    int64_t B, L, D, N;
    int dtype;
    uint32_t flags;
    int device;
    int sm_count;
    int *d_status;
    SscanMode mode;
    // chained kernel
    int cfg;           // index into kChainedCfgs (kTiled: into kTiledCfgs)
    bool poly;         // part of the exponents on the FMA pipe
    bool split;        // chains cut into concurrently scanned pieces + look-back fix-up
    bool drop_publish; // failure-detection tests: heads skip publishing (see read_tune)
    int64_t chains_per_row, chains, workers, seg, max_pieces;
    int64_t seg_shift;  // segment re-balancing unit x (see ChainedParams::seg_shift)
    size_t flag_off, flag_bytes;                // flags cleared on a workspace's first use
    size_t rec_s_off, rec_mono_off, ws_bytes;   // split-mode record arrays (rec_h at 0)
    size_t sink_off;                            // y sink of lanes past the last channel
    const void *last_ws;  // workspace whose flags were last cleared
    // tensor-map cache
    const void *tm_ptr[5];
    CUtensorMap tm[5];  // u, delta, B, C, gate z (z: fused calls with a gate; else a copy of u's)
    bool tm_valid;
    // generic kernel
    int g_nl, g_lpc;
    // decode kernel (L = 1 with a state)
    bool decode;
    int dec_grid;  // persistent grid, set on the first launch
    // sscan_forward_host: piece schedule, sub-plans and streams (made on first use)
    HostPipe *host;
};

// The kernel schedule of a plan's shape (host arithmetic only; reads SSCAN_TUNE).
void sscan_choose_schedule(sscan_plan *p);
// Release a plan's host-buffer pipeline (its sub-plans, streams and events).
void sscan_host_pipe_free(HostPipe *h);
