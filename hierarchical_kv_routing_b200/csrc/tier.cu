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
// waves of up to kWave query blocks.  Per wave, on a side stream:
//   k_tier_cache (one CTA per (sequence, KV head)): the warm tier, a bounded
//       cache of routed groups in HBM (the pages' warm VRAM tier).  The
//       wave's routed group ids are de-duplicated (a bitmap over the
//       sequence's groups); an id already cached is a hit; each miss takes a
//       slot by CLOCK order (a hand sweeps the slots; a slot is free or was
//       last used more than one wave ago, so neither the wave being attended
//       nor this one loses a slot it reads).  The kernel writes the fetch list
//       of misses and the wave's row map (routed slot -> cache row).
//   k_tier_gather: reads over the link the wave's sink chunks (first use of
//       each staging buffer), the window of recent and current chunks (chunks
//       the other buffer already holds are copied on the device) and the
//       fetch list's groups, rotating keys on the way (same rounding as stage
//       1), into one of two staging buffers and the cache.
// The tensor-core attention of the wave reads the buffer and the cache on
// the caller's stream while the next wave is prepared.  Each sequence's rows
// form one space per tensor (staging buffer 0, buffer 1, cache), so one
// tensor map covers every key a wave reads.  The cache holds two waves'
// worth of routed groups per (sequence, KV head) (the fewest that CLOCK can
// always serve), or every group of the sequence when that is fewer, unless
// the caller's workspace says otherwise: a larger one holds more slots (up
// to every group), a smaller one shrinks the wave so the staging buffers and
// the two-wave cache fit (down to one query block per wave).
#include <mutex>

#include "hga_internal.cuh"

namespace hga {
namespace {

constexpr int kWave = 32;            // query blocks per wave
constexpr int kGatherThreads = 256;
constexpr int kCacheThreads = 256;
constexpr int kMaxDevices = 64;

using bf16 = __nv_bfloat16;

__device__ int g_tier_error = 0;
__device__ unsigned long long g_tier_link_bytes = 0;   // host bytes the gathers read

struct GatherArgs {
    int B, T, Hkv, K_g, g_s, NB, W;
    int c0, c1, RT;                  // wave blocks; rows per sequence (buffers + cache)
    int buf_row0, pbuf_row0;         // this wave's staging buffer, the other one
    int sink_tok;                    // tokens [0, sink_tok) -> rows buf_row0 + token
    int win_tok0, win_tok1, win_row0;
    int prev_tok0, prev_tok1;        // window already held by the other buffer
    int cache_row0;                  // first row of the group cache
    long long n_sink, n_win, n_rt;   // (token, head) rows of each part, all sequences
    const bf16 *k_host, *v_host;     // device addresses of the pinned host arrays
    const int32_t *pos;
    const int2 *fetch;               // [B, Hkv, W * K_g]: (cache slot, group id) of each miss
    const int32_t *n_fetch;          // [B, Hkv]
    bf16 *kk, *vv;                   // [B, RT, Hkv, D]
    Rope rope;
};

struct CacheArgs {
    int B, Hkv, K_g, g_s, NB, NG, NS, W;
    int c0, c1, wave, cache_row0;
    const int32_t *sel_group;        // [B, NB, Hkv, K_g]
    int32_t *slot_of;                // [B, Hkv, NG]: cache slot of a group, or -1
    int32_t *gid_of, *stamp;         // [B, Hkv, NS]: group in a slot (-1: free), last wave used
    int32_t *hand;                   // [B, Hkv]: the CLOCK hand
    int2 *fetch;                     // [B, Hkv, W * K_g]
    int32_t *n_fetch;                // [B, Hkv]
    int32_t *rt_map;                 // [B, W, Hkv, K_g]: first row of each routed group
};

// Exclusive prefix sum of one value per thread over the CTA (s: kCacheThreads
// ints of shared scratch); returns this thread's offset, *total the sum.
__device__ __forceinline__ int block_excl_scan(int v, int *s, int *total) {
    const int t = threadIdx.x;
    s[t] = v;
    __syncthreads();
    for (int o = 1; o < kCacheThreads; o <<= 1) {
        const int a = t >= o ? s[t - o] : 0;
        __syncthreads();
        s[t] += a;
        __syncthreads();
    }
    *total = s[kCacheThreads - 1];
    const int incl = s[t];
    __syncthreads();
    return incl - v;
}

// The warm tier for one wave and one (sequence, KV head): de-duplicate the
// wave's routed groups, keep hits, give each miss a slot by CLOCK order,
// write the fetch list and the wave's row map.
__global__ void __launch_bounds__(kCacheThreads) k_tier_cache(const CacheArgs A) {
    extern __shared__ uint32_t bits[];                        // NG bits, then three lists
    __shared__ int s_scan[kCacheThreads];
    const int h = blockIdx.x, b = blockIdx.y, u = b * A.Hkv + h, tid = threadIdx.x;
    const int nwords = (A.NG + 31) / 32, WK = A.W * A.K_g;
    int *uniq = reinterpret_cast<int *>(bits + nwords);
    int *miss = uniq + WK;
    int *victim = miss + WK;
    int32_t *slot_of = A.slot_of + (long long)u * A.NG;
    int32_t *gid_of = A.gid_of + (long long)u * A.NS;
    int32_t *stamp = A.stamp + (long long)u * A.NS;
    const int nids = (A.c1 - A.c0) * A.K_g;
    auto sel_at = [&](int i) {
        const int c = A.c0 + i / A.K_g, j = i % A.K_g;
        return A.sel_group[(((long long)b * A.NB + c) * A.Hkv + h) * A.K_g + j];
    };
    for (int w = tid; w < nwords; w += kCacheThreads) bits[w] = 0u;
    __syncthreads();
    for (int i = tid; i < nids; i += kCacheThreads) {
        const int g = sel_at(i);
        if (g >= 0 && g < A.NG) atomicOr(&bits[g >> 5], 1u << (g & 31));
    }
    __syncthreads();
    // the wave's distinct groups, ascending
    const int wpt = (nwords + kCacheThreads - 1) / kCacheThreads;
    int cnt = 0;
    for (int w = tid * wpt; w < min(nwords, (tid + 1) * wpt); ++w) cnt += __popc(bits[w]);
    int nu = 0;
    int off = block_excl_scan(cnt, s_scan, &nu);
    for (int w = tid * wpt; w < min(nwords, (tid + 1) * wpt); ++w) {
        uint32_t m = bits[w];
        while (m) {
            const int bit = __ffs(m) - 1;
            m &= m - 1;
            uniq[off++] = w * 32 + bit;
        }
    }
    __syncthreads();
    // hits keep their slot (stamped with this wave); misses, ascending
    const int upt = (nu + kCacheThreads - 1) / kCacheThreads;
    int nmiss = 0;
    for (int i = tid * upt; i < min(nu, (tid + 1) * upt); ++i) {
        const int s = slot_of[uniq[i]];
        if (s >= 0) stamp[s] = A.wave;
        else ++nmiss;
    }
    int m = 0;
    off = block_excl_scan(nmiss, s_scan, &m);
    for (int i = tid * upt; i < min(nu, (tid + 1) * upt); ++i)
        if (slot_of[uniq[i]] < 0) miss[off++] = uniq[i];
    __syncthreads();
    // victims: from the hand on, slots that are free or were last used more
    // than one wave ago (the previous wave may still be attended)
    const int hand0 = A.hand[u];
    int found = 0;
    for (int base = 0; base < A.NS && found < m; base += kCacheThreads) {
        const int k = base + tid;
        const int s = (hand0 + k) % A.NS;
        const int ok = k < A.NS && (gid_of[s] < 0 || stamp[s] < A.wave - 1);
        int n_ok = 0;
        const int rank = block_excl_scan(ok, s_scan, &n_ok);
        if (ok && found + rank < m) victim[found + rank] = s;
        found += n_ok;
    }
    if (found > m) found = m;
    if (found < m && tid == 0) atomicExch(&g_tier_error, (int)HGA_ERR_UNSUPPORTED);
    __syncthreads();
    for (int i = tid; i < found; i += kCacheThreads) {
        const int old = gid_of[victim[i]];
        if (old >= 0) slot_of[old] = -1;
    }
    __syncthreads();
    int2 *fetch = A.fetch + (long long)u * WK;
    for (int i = tid; i < found; i += kCacheThreads) {
        const int s = victim[i], g = miss[i];
        slot_of[g] = s;
        gid_of[s] = g;
        stamp[s] = A.wave;
        fetch[i] = make_int2(s, g);
    }
    if (tid == 0) {
        A.n_fetch[u] = found;
        if (found > 0) A.hand[u] = (victim[found - 1] + 1) % A.NS;
    }
    __syncthreads();
    // the wave's row map
    for (int i = tid; i < nids; i += kCacheThreads) {
        const int g = sel_at(i);
        const int s = g >= 0 && g < A.NG ? slot_of[g] : -1;
        const int c = i / A.K_g, j = i % A.K_g;
        A.rt_map[(((long long)b * A.W + c) * A.Hkv + h) * A.K_g + j] =
            s >= 0 ? A.cache_row0 + s * A.g_s : -1;
    }
}

// Adds link bytes that no gather counted (the cold tier's group summaries).
__global__ void k_tier_count(unsigned long long bytes) { atomicAdd(&g_tier_link_bytes, bytes); }

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
    const int WK = A.W * A.K_g;
    unsigned host_bytes = 0;
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
            row = A.buf_row0 + tok;
        } else if (u < A.n_sink + A.n_win) {
            const long long v = u - A.n_sink;
            const long long per = (long long)(A.win_tok1 - A.win_tok0) * A.Hkv;
            b = (int)(v / per);
            const int rem = (int)(v % per);
            tok = A.win_tok0 + rem / A.Hkv;
            h = rem % A.Hkv;
            row = A.buf_row0 + A.win_row0 + tok - A.win_tok0;
            from_prev = tok >= A.prev_tok0 && tok < A.prev_tok1;
        } else {
            // a group the cache did not hold: into its cache slot
            const long long v = u - A.n_sink - A.n_win;
            const long long per = (long long)A.Hkv * WK * A.g_s;
            b = (int)(v / per);
            int rem = (int)(v % per);
            const int e = rem % A.g_s;
            rem /= A.g_s;
            const int i = rem % WK;
            h = rem / WK;
            if (i >= A.n_fetch[b * A.Hkv + h]) continue;
            const int2 f = A.fetch[((long long)b * A.Hkv + h) * WK + i];
            tok = f.y * A.g_s + e;
            row = A.cache_row0 + f.x * A.g_s + e;
        }
        const long long dst = (((long long)b * A.RT + row) * A.Hkv + h) * D;
        uint4 *dk = reinterpret_cast<uint4 *>(A.kk + dst);
        uint4 *dv = reinterpret_cast<uint4 *>(A.vv + dst);
        if (from_prev) {
            // rotated already: a device-to-device copy from the other buffer
            const long long src =
                (((long long)b * A.RT + A.pbuf_row0 + A.win_row0 + tok - A.prev_tok0) * A.Hkv + h) * D;
            const uint4 *pk = reinterpret_cast<const uint4 *>(A.kk + src);
            const uint4 *pv = reinterpret_cast<const uint4 *>(A.vv + src);
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
        host_bytes += 64;
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
    // bytes read over the link, one atomic per warp
    host_bytes = __reduce_add_sync(0xffffffffu, host_bytes);
    if ((threadIdx.x & 31) == 0 && host_bytes)
        atomicAdd(&g_tier_link_bytes, (unsigned long long)host_bytes);
}

// Workspace: summaries, selections, the K and V row spaces (per sequence:
// staging buffer 0, buffer 1, the group cache), the cache tables and the two
// row maps.
struct TierWs {
    size_t s_chunk, s_group, sel_c, sel_g, kk, vv, slot_of, gid_of, stamp, hand, n_fetch,
        fetch, rt_map, total;
    int W, Rs, NG, NS, RT, cache_row0;
};

inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout for waves of W query blocks and a warm cache of NS group
// slots per (sequence, KV head).
TierWs tier_ws(const Geo &g, int W, long long NS) {
    TierWs w;
    w.W = W;
    const int Lw = g.L > 1 ? g.L : 1;
    w.Rs = g.F * g.C + (w.W + Lw) * g.C;          // sinks and window of one buffer
    w.NG = g.NC * g.gpc;                          // groups of the sequence's closed chunks
    w.NS = (int)(NS < 1 ? 1 : NS);
    w.cache_row0 = 2 * w.Rs;
    w.RT = w.cache_row0 + w.NS * g.g_s;
    const size_t BH = (size_t)g.B * g.Hkv;
    size_t o = 0;
    w.s_chunk = o;
    o += up256((size_t)g.B * g.Hkv * g.NC * g.D * 4);
    w.s_group = o;
    o += up256((size_t)g.B * g.Hkv * g.NC * g.gpc * g.D * 4);
    w.sel_c = o;
    o += up256((size_t)g.B * g.NB * g.Hkv * g.K_c * 4);
    w.sel_g = o;
    o += up256((size_t)g.B * g.NB * g.Hkv * g.K_g * 4);
    const size_t rows = up256((size_t)g.B * w.RT * g.Hkv * g.D * sizeof(bf16));
    w.kk = o;
    o += rows;
    w.vv = o;
    o += rows;
    w.slot_of = o;
    o += up256(BH * (w.NG > 0 ? w.NG : 1) * 4);
    w.gid_of = o;
    o += up256(BH * w.NS * 4);
    w.stamp = o;
    o += up256(BH * w.NS * 4);
    w.hand = o;
    o += up256(BH * 4);
    w.n_fetch = o;
    o += up256(BH * 4);
    w.fetch = o;
    o += up256(BH * w.W * g.K_g * sizeof(int2));
    w.rt_map = o;
    o += up256(2 * (size_t)g.B * w.W * g.Hkv * g.K_g * 4);
    w.total = o;
    return w;
}

// The fewest slots that CLOCK can always serve for waves of W blocks: a wave
// reads at most W * K_g distinct groups and may not evict the previous
// wave's, so two waves' worth; never more than the sequence has groups.
long long min_slots(const Geo &g, int W) {
    const long long ng = (long long)g.NC * g.gpc, two = 2ll * W * g.K_g;
    return ng < two ? ng : two;
}

int full_wave(const Geo &g) { return g.NB < kWave ? g.NB : kWave; }

// The default plan: full waves, a cache of two waves' worth of groups.
TierWs tier_default(const Geo &g) { return tier_ws(g, full_wave(g), min_slots(g, full_wave(g))); }

// The plan for a workspace of `budget` bytes (the warm tier's VRAM budget):
// with at least the default size, full waves and as many cache slots as fit,
// up to every group of the sequence; with less, the wave shrinks (its
// staging buffers and the cache's two-wave floor with it) until the layout
// fits, down to one query block per wave.  ok = false when even that does
// not fit.
TierWs tier_plan(const Geo &g, size_t budget, bool *ok) {
    const TierWs def = tier_default(g);
    *ok = true;
    if (budget >= def.total) {
        long long lo = def.NS, hi = (long long)g.NC * g.gpc;
        if (hi < lo) hi = lo;
        while (lo < hi) {                         // largest NS whose layout fits
            const long long mid = lo + (hi - lo + 1) / 2;
            if (tier_ws(g, def.W, mid).total <= budget) lo = mid;
            else hi = mid - 1;
        }
        return tier_ws(g, def.W, lo);
    }
    for (int W = def.W - 1; W >= 1; --W) {
        const TierWs t = tier_ws(g, W, min_slots(g, W));
        if (t.total <= budget) return t;
    }
    *ok = false;
    return tier_ws(g, 1, min_slots(g, 1));
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
        if (e != cudaSuccess) {
            // release what was made, so a later call starts from nothing
            for (int i = 0; i < 2; ++i) {
                if (s.free_ev[i]) cudaEventDestroy(s.free_ev[i]);
                if (s.ready_ev[i]) cudaEventDestroy(s.ready_ev[i]);
            }
            if (s.start) cudaEventDestroy(s.start);
            if (s.side) cudaStreamDestroy(s.side);
            s = SideRes();
            return e;
        }
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

size_t hostkv_workspace_bytes(const Geo &g) { return tier_default(g).total; }

hga_status hostkv_plan(const Geo &g, size_t workspace_bytes, hga_hostkv_plan *plan) {
    bool ok = true;
    const TierWs t = tier_plan(g, workspace_bytes, &ok);
    plan->wave_blocks = t.W;
    plan->cache_slots = t.NS;
    plan->bytes = ok ? t.total : 0;
    plan->min_bytes = tier_ws(g, 1, min_slots(g, 1)).total;
    const long long ng = (long long)g.NC * g.gpc;
    plan->max_bytes = tier_ws(g, full_wave(g), ng > min_slots(g, full_wave(g)) ? ng
                                                 : min_slots(g, full_wave(g))).total;
    return ok ? HGA_OK : HGA_ERR_WORKSPACE;
}

hga_status launch_prefill_hostkv(const Geo &g, const Rope &r, const hga_io &io, void *ws,
                                 size_t ws_bytes, cudaStream_t st) {
    if (!attend_tc_supported(g, HGA_BF16)) return HGA_ERR_UNSUPPORTED;
    void *dk = nullptr, *dv = nullptr;
    if (cudaHostGetDevicePointer(&dk, const_cast<void *>(io.k), 0) != cudaSuccess ||
        cudaHostGetDevicePointer(&dv, const_cast<void *>(io.v), 0) != cudaSuccess) {
        cudaGetLastError();   // not pinned and mapped host memory: not sticky
        return HGA_ERR_INVALID_ARG;
    }
    bool fits = true;
    const TierWs w = tier_plan(g, ws_bytes, &fits);
    if (!fits) return HGA_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    float *s_chunk = reinterpret_cast<float *>(base + w.s_chunk);
    float *s_group = reinterpret_cast<float *>(base + w.s_group);
    // group summaries in the cold tier: the caller's pinned host table
    const bool host_groups = io.s_group_host != nullptr;
    if (host_groups) {
        void *dg = nullptr;
        if (cudaHostGetDevicePointer(&dg, io.s_group_host, 0) != cudaSuccess) {
            cudaGetLastError();   // not pinned and mapped host memory: not sticky
            return HGA_ERR_INVALID_ARG;
        }
        s_group = static_cast<float *>(dg);
    }
    int32_t *sel_c = io.sel_chunk ? io.sel_chunk : reinterpret_cast<int32_t *>(base + w.sel_c);
    int32_t *sel_g = io.sel_group ? io.sel_group : reinterpret_cast<int32_t *>(base + w.sel_g);
    bf16 *kk = reinterpret_cast<bf16 *>(base + w.kk);
    bf16 *vv = reinterpret_cast<bf16 *>(base + w.vv);
    int32_t *slot_of = reinterpret_cast<int32_t *>(base + w.slot_of);
    int32_t *gid_of = reinterpret_cast<int32_t *>(base + w.gid_of);
    int32_t *stamp = reinterpret_cast<int32_t *>(base + w.stamp);
    int32_t *hand = reinterpret_cast<int32_t *>(base + w.hand);
    int32_t *n_fetch = reinterpret_cast<int32_t *>(base + w.n_fetch);
    int2 *fetch = reinterpret_cast<int2 *>(base + w.fetch);
    int32_t *rt_map = reinterpret_cast<int32_t *>(base + w.rt_map);
    const size_t BH = (size_t)g.B * g.Hkv;
    const size_t map_wave = (size_t)g.B * w.W * g.Hkv * g.K_g;

    // stages 1 and 2: summaries from the host keys (one pass over the link)
    hga_status s = launch_summaries(g, r, HGA_BF16, dk, nullptr, io.pos, g.T, nullptr, nullptr,
                                    nullptr, g.T, s_chunk, s_group, g.NC, nullptr, nullptr, st,
                                    /*host_src=*/true);
    if (s != HGA_OK) return s;
    s = launch_route(g, r, HGA_BF16, io.q, io.pos, s_chunk, s_group, g.NC, sel_c, sel_g, st,
                     host_groups);
    if (s != HGA_OK) return s;
    if (host_groups) {
        // the group table written over the link, and the group rows of every
        // block's routed chunks read back
        long long rows = 0;
        for (int c = 0; c < g.NB; ++c) {
            const int n_mid = max(0, (g.L == 0 ? c - 2 : c - g.L - 1) - g.F + 1);
            rows += min(g.K_c, n_mid);
        }
        const unsigned long long bytes =
            ((unsigned long long)g.NC + (unsigned long long)rows) * g.gpc * g.D * 4ull * g.B * g.Hkv;
        k_tier_count<<<1, 1, 0, st>>>(bytes);
        cudaError_t ce = cudaGetLastError();
        if (ce != cudaSuccess) return cuda_status(ce);
    }
    // an empty group cache for this call
    cudaError_t e = cudaMemsetAsync(slot_of, 0xff, BH * (w.NG > 0 ? w.NG : 1) * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(gid_of, 0xff, BH * w.NS * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(stamp, 0, BH * w.NS * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(hand, 0, BH * 4, st);
    if (e != cudaSuccess) return cuda_status(e);

    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return HGA_ERR_UNSUPPORTED;
    const size_t cache_smem = 4 * ((size_t)(w.NG + 31) / 32 + 3 * (size_t)w.W * g.K_g);
    if ((e = ensure_smem((const void *)k_tier_cache, cache_smem)) != cudaSuccess)
        return cuda_status(e);
    std::lock_guard<std::mutex> lock(g_tier_mu);
    SideRes *sr = nullptr;
    if ((e = side_resources(dev, &sr)) != cudaSuccess) return cuda_status(e);
    // the side stream starts after everything already on the caller's stream
    if ((e = cudaEventRecord(sr->start, st)) != cudaSuccess) return cuda_status(e);
    if ((e = cudaStreamWaitEvent(sr->side, sr->start, 0)) != cudaSuccess) return cuda_status(e);

    const int Lw = g.L > 1 ? g.L : 1;
    const int sink_rows = g.F * g.C;
    const int win_row0 = sink_rows;
    int prev_tok0 = 0, prev_tok1 = 0;
    for (int wave = 0, c0 = 0; c0 < g.NB; ++wave, c0 += w.W) {
        const int c1 = c0 + w.W < g.NB ? c0 + w.W : g.NB;
        const int buf = wave & 1;
        const int nsink0 = c0 < g.F ? c0 : g.F;
        const int rec_lo0 = c0 - Lw > nsink0 ? c0 - Lw : nsink0;
        const int wlo = rec_lo0 > g.F ? rec_lo0 : g.F;
        int32_t *map = rt_map + buf * map_wave;

        CacheArgs ca;
        ca.B = g.B;
        ca.Hkv = g.Hkv;
        ca.K_g = g.K_g;
        ca.g_s = g.g_s;
        ca.NB = g.NB;
        ca.NG = w.NG;
        ca.NS = w.NS;
        ca.W = w.W;
        ca.c0 = c0;
        ca.c1 = c1;
        ca.wave = wave;
        ca.cache_row0 = w.cache_row0;
        ca.sel_group = sel_g;
        ca.slot_of = slot_of;
        ca.gid_of = gid_of;
        ca.stamp = stamp;
        ca.hand = hand;
        ca.fetch = fetch;
        ca.n_fetch = n_fetch;
        ca.rt_map = map;

        GatherArgs a;
        a.B = g.B;
        a.T = g.T;
        a.Hkv = g.Hkv;
        a.K_g = g.K_g;
        a.g_s = g.g_s;
        a.NB = g.NB;
        a.W = w.W;
        a.c0 = c0;
        a.c1 = c1;
        a.RT = w.RT;
        a.buf_row0 = buf * w.Rs;
        a.pbuf_row0 = (buf ^ 1) * w.Rs;
        a.sink_tok = wave < 2 ? (sink_rows < g.T ? sink_rows : g.T) : 0;
        a.win_tok0 = wlo * g.C;
        a.win_tok1 = c1 * g.C < g.T ? c1 * g.C : g.T;
        if (a.win_tok1 < a.win_tok0) a.win_tok1 = a.win_tok0;
        a.win_row0 = win_row0;
        a.prev_tok0 = wave > 0 ? prev_tok0 : 0;
        a.prev_tok1 = wave > 0 ? prev_tok1 : 0;
        a.cache_row0 = w.cache_row0;
        a.n_sink = (long long)g.B * a.sink_tok * g.Hkv;
        a.n_win = (long long)g.B * (a.win_tok1 - a.win_tok0) * g.Hkv;
        a.n_rt = (long long)g.B * g.Hkv * w.W * g.K_g * g.g_s;
        a.k_host = static_cast<const bf16 *>(dk);
        a.v_host = static_cast<const bf16 *>(dv);
        a.pos = io.pos;
        a.fetch = fetch;
        a.n_fetch = n_fetch;
        a.kk = kk;
        a.vv = vv;
        a.rope = r;
        prev_tok0 = a.win_tok0;
        prev_tok1 = a.win_tok1;

        // the cache and `buf` change once the attention two waves back has
        // read them (the cache only evicts slots no later wave used)
        if (wave >= 2 && (e = cudaStreamWaitEvent(sr->side, sr->free_ev[buf], 0)) != cudaSuccess)
            return cuda_status(e);
        k_tier_cache<<<dim3(g.Hkv, g.B), kCacheThreads, cache_smem, sr->side>>>(ca);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
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
        tw.buf_row0 = a.buf_row0;
        tw.rt_W = w.W;
        tw.rt_map = map;
        s = launch_attend_tc(g, r, io.q, io.pos, kk, w.RT, vv, w.RT, sel_g, io.out, io.lse, st, &tw);
        if (s != HGA_OK) return s;
        if ((e = cudaEventRecord(sr->free_ev[buf], st)) != cudaSuccess) return cuda_status(e);
    }
    return HGA_OK;
}

// Reads (and optionally resets) the bytes the host tier's gathers have read
// over the link, after the work queued on `st`.
hga_status tier_link_bytes_take(cudaStream_t st, unsigned long long *bytes, bool clear) {
    unsigned long long v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_tier_link_bytes, sizeof(v), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear) {
        const unsigned long long zero = 0;
        e = cudaMemcpyToSymbolAsync(g_tier_link_bytes, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    *bytes = v;
    return HGA_OK;
}

// Reads this file's device error word on `st` and optionally resets it.
hga_status tier_error_take(cudaStream_t st, bool clear) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_tier_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_tier_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    return (hga_status)v;
}

}  // namespace hga
