// The visible key set of a query chunk, as a short list of token runs.
//
// Method: HGA paper-review page, section 3, routing policy ("确定性可见性",
// deterministic visibility) and exact token output attention: a query token
// of chunk c sees the sink chunks 0..F-1, the recent closed chunks c-L..c-1,
// the previous chunk c-1 (forced when L == 0), the routed groups, and the
// causal part of its own chunk.  Each token appears once: sinks and recent
// chunks are merged when they overlap, and routed groups are middle-chunk
// groups, which never overlap either window.
#pragma once
#include "hga_internal.cuh"

namespace hga {

struct RunList {
    static constexpr int kMaxRuns = 1024 + 3;
    int start[kMaxRuns];   // first token of the run
    int off[kMaxRuns + 1]; // prefix offsets into the key list
    int n;                 // number of runs
    int cur_off;           // key-list offset where the current chunk starts
};

// Thread 0 builds the run list for current chunk c: fixed windows, routed
// groups (sel: K_g ids, ascending, -1 padded) and n_cur tokens of chunk c.
// Returns the total key count through rl.off[rl.n].
__device__ __forceinline__ void build_runs(RunList &rl, int c, int F, int L, int g_s,
                                           const int32_t *__restrict__ sel, int K_g, int n_cur) {
    int n = 0, o = 0;
    const int nsink = min(F, c);
    if (nsink > 0) {
        rl.start[n] = 0;
        rl.off[n++] = o;
        o += nsink * kChunk;
    }
    const int rec_lo = max(c - max(L, 1), nsink);
    if (rec_lo < c) {
        rl.start[n] = rec_lo * kChunk;
        rl.off[n++] = o;
        o += (c - rec_lo) * kChunk;
    }
    for (int j = 0; j < K_g; ++j) {
        const int g = sel[j];
        if (g < 0) continue;
        rl.start[n] = g * g_s;
        rl.off[n++] = o;
        o += g_s;
    }
    rl.cur_off = o;
    rl.start[n] = c * kChunk;
    rl.off[n++] = o;
    o += n_cur;
    rl.off[n] = o;
    rl.n = n;
}

// Fill keys[0..total) with token indices from the runs (whole CTA).
__device__ __forceinline__ void fill_keys(const RunList &rl, int *keys) {
    for (int r = 0; r < rl.n; ++r) {
        const int s = rl.start[r], o = rl.off[r], len = rl.off[r + 1] - o;
        for (int k = threadIdx.x; k < len; k += blockDim.x) keys[o + k] = s + k;
    }
}

}  // namespace hga
