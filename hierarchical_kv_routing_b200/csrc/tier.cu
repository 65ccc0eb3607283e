// Host-resident K/V tier for prefill (hga_forward mode HGA_PREFILL_HOSTKV).
//
// Method: HGA paper-review page, section 3, "三层 K/V 存储" (three-tier K/V
// store): the full token K/V history lives in host RAM, the GPU holds the
// chunk and group summaries, and routing fetches only the token K/V of the
// routed groups (store operation "gather token K/V"); attention is the same
// exact softmax over the visible set (eq. (1) restricted).  The gist.science
// page, "Memory Architecture", describes the same cold tier.
//
// Design.  K (raw) and V stay in the caller's pinned host arrays.  Stage 1
// reads K across the host link once (zero-copy loads) to build the summaries
// on the GPU; stage 2 routes every query block on the GPU.  Stage 3 runs in
// waves of up to kWave query blocks.  For each wave a gather kernel on a side
// stream reads, over the link, the wave's sink chunks (first use of each
// buffer only), the window of recent and current chunks (chunks already in
// the other buffer are copied on the device instead) and the routed groups of
// every (block, KV head), rotates the keys on the way (same rounding as
// stage 1), and writes them into one of two HBM staging buffers; the
// tensor-core attention of the wave reads that buffer on the caller's stream
// while the next wave is gathered into the other one.
#include <mutex>

#include "hga_internal.cuh"

namespace hga {
namespace {

constexpr int kWave = 32;            // query blocks per wave
constexpr int kGatherThreads = 256;
constexpr int kMaxDevices = 64;

using bf16 = __nv_bfloat16;

struct GatherArgs {
    int B, T, Hkv, K_g, g_s, NB;
    int c0, c1, R;                   // wave blocks; staging rows per sequence
    int sink_tok;                    // tokens [0, sink_tok) -> rows [0, sink_tok)
    int win_tok0, win_tok1, win_row0;
    int prev_tok0, prev_tok1;        // window already held by the other buffer
    int rt_row0;
    long long n_sink, n_win, n_rt;   // (token, head) rows of each part, all sequences
    const bf16 *k_host, *v_host;     // device addresses of the pinned host arrays
    const int32_t *pos, *sel_group;
    bf16 *sk, *sv;                   // this wave's buffer
    const bf16 *psk, *psv;           // the other buffer
    Rope rope;
};

// Plain 16-byte global load (host memory is read without the read-only path).
__device__ __forceinline__ uint4 ld16(const bf16 *p) {
    uint4 w;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                 : "l"(p));
    return w;
}

// One (token, head) row per D/16 threads; thread q moves the 8 pairs whose
// first elements are 8q..8q+7 (two 16-byte words of K and two of V).
template <int D>
__global__ void __launch_bounds__(kGatherThreads) k_tier_gather(const GatherArgs A) {
    constexpr int H = D / 2, TPU = D / 16;
    const long long total = A.n_sink + A.n_win + A.n_rt;
    const int q = threadIdx.x % TPU;
    const long long stride = (long long)gridDim.x * (kGatherThreads / TPU);
    for (long long u = (long long)blockIdx.x * (kGatherThreads / TPU) + threadIdx.x / TPU;
         u < total; u += stride) {
        int b, tok, h, row;
        bool from_prev = false;
        if (u < A.n_sink) {
            const long long per = (long long)A.sink_tok * A.Hkv;
            b = (int)(u / per);
            const int rem = (int)(u % per);
            tok = rem / A.Hkv;
            h = rem % A.Hkv;
            row = tok;
        } else if (u < A.n_sink + A.n_win) {
            const long long v = u - A.n_sink;
            const long long per = (long long)(A.win_tok1 - A.win_tok0) * A.Hkv;
            b = (int)(v / per);
            const int rem = (int)(v % per);
            tok = A.win_tok0 + rem / A.Hkv;
            h = rem % A.Hkv;
            row = A.win_row0 + tok - A.win_tok0;
            from_prev = tok >= A.prev_tok0 && tok < A.prev_tok1;
        } else {
            const long long v = u - A.n_sink - A.n_win;
            const long long per = (long long)(A.c1 - A.c0) * A.Hkv * A.K_g * A.g_s;
            b = (int)(v / per);
            int rem = (int)(v % per);
            const int e = rem % A.g_s;
            rem /= A.g_s;
            const int j = rem % A.K_g;
            rem /= A.K_g;
            h = rem % A.Hkv;
            const int cb = rem / A.Hkv;
            const int sel = A.sel_group[(((long long)b * A.NB + A.c0 + cb) * A.Hkv + h) * A.K_g + j];
            if (sel < 0) continue;
            tok = sel * A.g_s + e;
            row = A.rt_row0 + (cb * A.K_g + j) * A.g_s + e;
        }
        const long long dst = (((long long)b * A.R + row) * A.Hkv + h) * D;
        uint4 *dk = reinterpret_cast<uint4 *>(A.sk + dst);
        uint4 *dv = reinterpret_cast<uint4 *>(A.sv + dst);
        if (from_prev) {
            // rotated already: a device-to-device copy from the other buffer
            const long long src =
                (((long long)b * A.R + A.win_row0 + tok - A.prev_tok0) * A.Hkv + h) * D;
            const uint4 *pk = reinterpret_cast<const uint4 *>(A.psk + src);
            const uint4 *pv = reinterpret_cast<const uint4 *>(A.psv + src);
            const uint4 k0 = pk[q], k1 = pk[q + TPU], v0 = pv[q], v1 = pv[q + TPU];
            dk[q] = k0;
            dk[q + TPU] = k1;
            dv[q] = v0;
            dv[q + TPU] = v1;
            continue;
        }
        const long long src = (((long long)b * A.T + tok) * A.Hkv + h) * D;
        const uint4 k0 = ld16(A.k_host + src + 8 * q), k1 = ld16(A.k_host + src + H + 8 * q);
        const uint4 v0 = ld16(A.v_host + src + 8 * q), v1 = ld16(A.v_host + src + H + 8 * q);
        dv[q] = v0;
        dv[q + TPU] = v1;
        const int32_t p = A.pos[(long long)b * A.T + tok];
        const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(&k0);
        const __nv_bfloat162 *y2 = reinterpret_cast<const __nv_bfloat162 *>(&k1);
        uint4 o0, o1;
        __nv_bfloat162 *a2 = reinterpret_cast<__nv_bfloat162 *>(&o0);
        __nv_bfloat162 *c2 = reinterpret_cast<__nv_bfloat162 *>(&o1);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(x2[e]), y = __bfloat1622float2(y2[e]);
            const float2 r0 = rot_pair(x.x, y.x, rope_cs_int(A.rope, p, 8 * q + 2 * e));
            const float2 r1 = rot_pair(x.y, y.y, rope_cs_int(A.rope, p, 8 * q + 2 * e + 1));
            a2[e] = __floats2bfloat162_rn(r0.x, r1.x);
            c2[e] = __floats2bfloat162_rn(r0.y, r1.y);
        }
        dk[q] = o0;
        dk[q + TPU] = o1;
    }
}

// Workspace: summaries, selections, two staging buffers (K and V each).
struct TierWs {
    size_t s_chunk, s_group, sel_c, sel_g, stage[4], total;
    int W, R;
};

inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

TierWs tier_ws(const Geo &g) {
    TierWs w;
    w.W = g.NB < kWave ? g.NB : kWave;
    const int Lw = g.L > 1 ? g.L : 1;
    w.R = g.F * g.C + (w.W + Lw) * g.C + w.W * g.K_g * g.g_s;
    size_t o = 0;
    w.s_chunk = o;
    o += up256((size_t)g.B * g.Hkv * g.NC * g.D * 4);
    w.s_group = o;
    o += up256((size_t)g.B * g.Hkv * g.NC * g.gpc * g.D * 4);
    w.sel_c = o;
    o += up256((size_t)g.B * g.NB * g.Hkv * g.K_c * 4);
    w.sel_g = o;
    o += up256((size_t)g.B * g.NB * g.Hkv * g.K_g * 4);
    const size_t stage = up256((size_t)g.B * w.R * g.Hkv * g.D * sizeof(bf16));
    for (int i = 0; i < 4; ++i) {
        w.stage[i] = o;
        o += stage;
    }
    w.total = o;
    return w;
}

// Per-device side stream and events, created on first use.  One mutex keeps
// the enqueue sequence of a call (which reuses these events) whole when
// several host threads call at once.
struct SideRes {
    bool ready = false;
    cudaStream_t side = nullptr;
    cudaEvent_t start = nullptr, ready_ev[2] = {}, free_ev[2] = {};
};
std::mutex g_tier_mu;
SideRes g_side[kMaxDevices];

cudaError_t side_resources(int dev, SideRes **out) {
    SideRes &s = g_side[dev];
    if (!s.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&s.side, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.start, cudaEventDisableTiming);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&s.ready_ev[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.free_ev[i], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return e;
        s.ready = true;
    }
    *out = &s;
    return cudaSuccess;
}

template <int D>
hga_status gather(const GatherArgs &a, cudaStream_t st) {
    constexpr int per_cta = kGatherThreads / (D / 16);
    const long long total = a.n_sink + a.n_win + a.n_rt;
    if (total == 0) return HGA_OK;
    long long grid = (total + per_cta - 1) / per_cta;
    if (grid > 148 * 8) grid = 148 * 8;
    k_tier_gather<D><<<(unsigned)grid, kGatherThreads, 0, st>>>(a);
    return cuda_status(cudaGetLastError());
}

}  // namespace

size_t hostkv_workspace_bytes(const Geo &g) { return tier_ws(g).total; }

hga_status launch_prefill_hostkv(const Geo &g, const Rope &r, const hga_io &io, void *ws,
                                 cudaStream_t st) {
    if (!attend_tc_supported(g, HGA_BF16)) return HGA_ERR_UNSUPPORTED;
    void *dk = nullptr, *dv = nullptr;
    if (cudaHostGetDevicePointer(&dk, const_cast<void *>(io.k), 0) != cudaSuccess ||
        cudaHostGetDevicePointer(&dv, const_cast<void *>(io.v), 0) != cudaSuccess) {
        cudaGetLastError();   // not pinned and mapped host memory: not sticky
        return HGA_ERR_INVALID_ARG;
    }
    const TierWs w = tier_ws(g);
    char *base = static_cast<char *>(ws);
    float *s_chunk = reinterpret_cast<float *>(base + w.s_chunk);
    float *s_group = reinterpret_cast<float *>(base + w.s_group);
    int32_t *sel_c = io.sel_chunk ? io.sel_chunk : reinterpret_cast<int32_t *>(base + w.sel_c);
    int32_t *sel_g = io.sel_group ? io.sel_group : reinterpret_cast<int32_t *>(base + w.sel_g);
    bf16 *stage[4];
    for (int i = 0; i < 4; ++i) stage[i] = reinterpret_cast<bf16 *>(base + w.stage[i]);

    // stages 1 and 2: summaries from the host keys (one pass over the link)
    hga_status s = launch_summaries(g, r, HGA_BF16, dk, nullptr, io.pos, g.T, nullptr, nullptr,
                                    nullptr, g.T, s_chunk, s_group, g.NC, nullptr, nullptr, st,
                                    /*host_src=*/true);
    if (s != HGA_OK) return s;
    s = launch_route(g, r, HGA_BF16, io.q, io.pos, s_chunk, s_group, g.NC, sel_c, sel_g, st);
    if (s != HGA_OK) return s;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return HGA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_tier_mu);
    SideRes *sr = nullptr;
    if ((e = side_resources(dev, &sr)) != cudaSuccess) return cuda_status(e);
    // the side stream starts after everything already on the caller's stream
    if ((e = cudaEventRecord(sr->start, st)) != cudaSuccess) return cuda_status(e);
    if ((e = cudaStreamWaitEvent(sr->side, sr->start, 0)) != cudaSuccess) return cuda_status(e);

    const int Lw = g.L > 1 ? g.L : 1;
    const int sink_rows = g.F * g.C;
    const int win_row0 = sink_rows;
    const int rt_row0 = sink_rows + (w.W + Lw) * g.C;
    int prev_tok0 = 0, prev_tok1 = 0;
    for (int wave = 0, c0 = 0; c0 < g.NB; ++wave, c0 += w.W) {
        const int c1 = c0 + w.W < g.NB ? c0 + w.W : g.NB;
        const int buf = wave & 1;
        const int nsink0 = c0 < g.F ? c0 : g.F;
        const int rec_lo0 = c0 - Lw > nsink0 ? c0 - Lw : nsink0;
        const int wlo = rec_lo0 > g.F ? rec_lo0 : g.F;
        GatherArgs a;
        a.B = g.B;
        a.T = g.T;
        a.Hkv = g.Hkv;
        a.K_g = g.K_g;
        a.g_s = g.g_s;
        a.NB = g.NB;
        a.c0 = c0;
        a.c1 = c1;
        a.R = w.R;
        a.sink_tok = wave < 2 ? (sink_rows < g.T ? sink_rows : g.T) : 0;
        a.win_tok0 = wlo * g.C;
        a.win_tok1 = c1 * g.C < g.T ? c1 * g.C : g.T;
        if (a.win_tok1 < a.win_tok0) a.win_tok1 = a.win_tok0;
        a.win_row0 = win_row0;
        a.prev_tok0 = wave > 0 ? prev_tok0 : 0;
        a.prev_tok1 = wave > 0 ? prev_tok1 : 0;
        a.rt_row0 = rt_row0;
        a.n_sink = (long long)g.B * a.sink_tok * g.Hkv;
        a.n_win = (long long)g.B * (a.win_tok1 - a.win_tok0) * g.Hkv;
        a.n_rt = (long long)g.B * (c1 - c0) * g.Hkv * g.K_g * g.g_s;
        a.k_host = static_cast<const bf16 *>(dk);
        a.v_host = static_cast<const bf16 *>(dv);
        a.pos = io.pos;
        a.sel_group = sel_g;
        a.sk = stage[2 * buf];
        a.sv = stage[2 * buf + 1];
        a.psk = stage[2 * (buf ^ 1)];
        a.psv = stage[2 * (buf ^ 1) + 1];
        a.rope = r;
        prev_tok0 = a.win_tok0;
        prev_tok1 = a.win_tok1;

        // gather into `buf` once the attention two waves back has read it
        if (wave >= 2 && (e = cudaStreamWaitEvent(sr->side, sr->free_ev[buf], 0)) != cudaSuccess)
            return cuda_status(e);
        s = g.D == 128 ? gather<128>(a, sr->side) : gather<64>(a, sr->side);
        if (s != HGA_OK) return s;
        if ((e = cudaEventRecord(sr->ready_ev[buf], sr->side)) != cudaSuccess) return cuda_status(e);
        if ((e = cudaStreamWaitEvent(st, sr->ready_ev[buf], 0)) != cudaSuccess) return cuda_status(e);
        TierWave tw;
        tw.c0 = c0;
        tw.c1 = c1;
        tw.sink_rows = sink_rows;
        tw.win_tok0 = a.win_tok0;
        tw.win_row0 = win_row0;
        tw.rt_row0 = rt_row0;
        s = launch_attend_tc(g, r, io.q, io.pos, a.sk, w.R, a.sv, w.R, sel_g, io.out, io.lse, st,
                             &tw);
        if (s != HGA_OK) return s;
        if ((e = cudaEventRecord(sr->free_ev[buf], st)) != cudaSuccess) return cuda_status(e);
    }
    return HGA_OK;
}

}  // namespace hga
