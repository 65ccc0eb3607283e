// Decode step: one new token per sequence, appended to the K/V cache, routed
// with its own query and attended over its visible set.
//
// Method: HGA paper-review page, section 3: the store's "append closed
// chunk" operation (a chunk's mixed-RoPE summaries exist once its last token
// is written), the routing policy and selection equation applied to one query
// token, and exact token output attention (eq. (1) over the visible set).
// The pages check decode against a full recompute (Table 7); the tests here
// do the same against the oracle.
//
// Two kernels per step, both HBM-bound:
//   k_decode_scan   grid (scan splits, KV heads, sequences).  Split 0 of each
//                   (sequence, KV head) appends the token (rotated key, value,
//                   position, raw key into the open-chunk buffer) and, when the
//                   token closes its chunk, writes that chunk's summaries.  Every
//                   split scores its 64-chunk slice of the middle-chunk table
//                   with the token's routing query (fp64 accumulation) and
//                   keeps its top K_c keys; the last split to finish (atomic
//                   counter) merges them, scores the groups of the chosen
//                   chunks and keeps the top K_g.
//   k_decode_attend grid (key splits, KV heads, sequences).  Each CTA takes a
//                   slice of the token's visible key list, stages its K/V rows
//                   in shared memory with 16-byte loads, and computes partial
//                   softmax sums for the KV head's G query heads; the last CTA
//                   per (sequence, KV head) combines the partials, and the last
//                   of those per sequence increments lens.
// Counters live in the workspace; each last CTA resets its counter, so the
// workspace only has to be zeroed before its first use.
#include "hga_internal.cuh"
#include "route_common.cuh"
#include "vec.cuh"
#include "visible.cuh"

namespace hga {

__device__ int g_decode_error = 0;

namespace {

constexpr int kThreads = 256;
constexpr int kScanChunks = 64;   // middle chunks per scan split
constexpr int kAttSplits = 8;     // key-list splits per (sequence, KV head)

struct DecodeArgs {
    int B, Tc, Hq, Hkv, G, C, g_s, gpc, F, L, K_c, K_g, nc_cap, ns_scan, keys_max, per_max;
    const void *q_new, *k_new, *v_new;
    const int32_t *pos_new;
    void *k_rot, *v;
    int32_t *pos;
    void *k_open;
    float *s_chunk, *s_group;
    int32_t *lens;
    void *out;
    float *lse;
    int32_t *sel_c, *sel_g;          // [B, Hkv, K]
    unsigned long long *cand;        // [B, Hkv, ns_scan, K_c]
    float *part;                     // [B, Hq, kAttSplits, D + 2]
    int32_t *scan_done, *att_done, *seq_done;
    float scale_log2;
    Rope rope;
};

template <typename T>
__device__ __forceinline__ float ld_elem(const T *p) {
    return to_f(*p);
}

// Summaries of chunk c of (b, h) from the open-chunk raw keys (its last key
// was written by this CTA just before), positions from the cache except the
// last one (pos_last).  One work item per (set, pair): sets 0..gpc-1 are the
// groups, set gpc the chunk.  High pairs: mean of rotated keys; low pairs:
// mean raw key rotated at the set's mean position.
template <typename T, int D>
__device__ void close_chunk(const DecodeArgs &A, int b, int h, int c, int32_t pos_last) {
    constexpr int H = D / 2;
    const T *ko = static_cast<const T *>(A.k_open) + ((int64_t)b * A.Hkv + h) * A.C * D;
    const int32_t *pc = A.pos + (int64_t)b * A.Tc + (int64_t)c * A.C;
    for (int e = threadIdx.x; e < (A.gpc + 1) * H; e += blockDim.x) {
        const int set = e / H, i = e % H;
        const int lo = set < A.gpc ? set * A.g_s : 0, cnt = set < A.gpc ? A.g_s : A.C;
        const bool hf = is_high(A.rope, i);
        double a = 0.0, d2 = 0.0, pm = 0.0;
        for (int j = lo; j < lo + cnt; ++j) {
            const int32_t pj = j == A.C - 1 ? pos_last : pc[j];
            pm += (double)pj;
            const float x = ld_elem(ko + (int64_t)j * D + i), y = ld_elem(ko + (int64_t)j * D + i + H);
            if (hf) {
                const float2 r = rope_cs(A.rope, (double)pj, i);
                a += (double)(x * r.x - y * r.y);
                d2 += (double)(y * r.x + x * r.y);
            } else {
                a += (double)x;
                d2 += (double)y;
            }
        }
        a /= (double)cnt;
        d2 /= (double)cnt;
        float o0 = (float)a, o1 = (float)d2;
        if (!hf) {
            const float2 r = rope_cs(A.rope, pm / (double)cnt, i);
            o0 = (float)(a * (double)r.x - d2 * (double)r.y);
            o1 = (float)(d2 * (double)r.x + a * (double)r.y);
        }
        float *dst = set < A.gpc
            ? A.s_group + ((((int64_t)b * A.Hkv + h) * A.nc_cap + c) * A.gpc + set) * D
            : A.s_chunk + (((int64_t)b * A.Hkv + h) * A.nc_cap + c) * D;
        dst[i] = o0;
        dst[i + H] = o1;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) k_decode_scan(const DecodeArgs A) {
    constexpr int H = D / 2;
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(smem);
    __shared__ double qr[D];
    __shared__ RouteScratch rs;
    __shared__ int s_last;

    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t = A.lens[b];
    if (t < 0 || t >= A.Tc) {
        if (threadIdx.x == 0) atomicExch(&g_decode_error, (int)HGA_ERR_BOUNDS);
        return;   // every CTA of this sequence sees the same lens and skips
    }
    const int c = t / A.C;
    const int32_t pnew = A.pos_new[b];

    // ---- append (split 0 of each KV head)
    if (s == 0) {
        const T *kn = static_cast<const T *>(A.k_new) + ((int64_t)b * A.Hkv + h) * D;
        const T *vn = static_cast<const T *>(A.v_new) + ((int64_t)b * A.Hkv + h) * D;
        const int64_t row = ((int64_t)b * A.Tc + t) * A.Hkv + h;
        T *kr = static_cast<T *>(A.k_rot) + row * D;
        T *vr = static_cast<T *>(A.v) + row * D;
        T *ko = static_cast<T *>(A.k_open) + (((int64_t)b * A.Hkv + h) * A.C + t % A.C) * D;
        for (int i = threadIdx.x; i < H; i += blockDim.x) {
            const float x = to_f(kn[i]), y = to_f(kn[i + H]);
            const float2 r = rope_cs(A.rope, (double)pnew, i);
            kr[i] = from_f<T>(x * r.x - y * r.y);
            kr[i + H] = from_f<T>(y * r.x + x * r.y);
            ko[i] = kn[i];
            ko[i + H] = kn[i + H];
        }
        for (int i = threadIdx.x; i < D; i += blockDim.x) vr[i] = vn[i];
        if (h == 0 && threadIdx.x == 0) A.pos[(int64_t)b * A.Tc + t] = pnew;
        __syncthreads();
        if (t % A.C == A.C - 1) close_chunk<T, D>(A, b, h, c, pnew);
    }

    // ---- routing query of the token: sum over the KV head's query heads
    if (threadIdx.x < H) {
        const int i = threadIdx.x;
        const float2 r = rope_cs(A.rope, (double)pnew, i);
        const T *qb = static_cast<const T *>(A.q_new) + ((int64_t)b * A.Hq + (int64_t)h * A.G) * D;
        double a = 0.0, d2 = 0.0;
        for (int g = 0; g < A.G; ++g) {
            const float x = to_f(qb[g * D + i]), y = to_f(qb[g * D + i + H]);
            a += (double)(x * r.x - y * r.y);
            d2 += (double)(y * r.x + x * r.y);
        }
        qr[i] = a;
        qr[i + H] = d2;
    }
    __syncthreads();

    // ---- this split's slice of the middle chunks, top K_c keys
    const int mlo = A.F, mhi = middle_hi(c, A.L);
    const int first = max(mlo, s * kScanChunks);
    const int last = min(mhi, s * kScanChunks + kScanChunks - 1);
    const int n = max(0, last - first + 1);
    const float *Sc = A.s_chunk + ((int64_t)b * A.Hkv + h) * A.nc_cap * D;
    score_rows<D>(qr, Sc, first, n, cand);
    __syncthreads();
    unsigned long long *mine = A.cand + (((int64_t)b * A.Hkv + h) * A.ns_scan + s) * A.K_c;
    topk_keys(cand, n, A.K_c, mine, rs);

    // ---- the last split merges and routes the groups
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int done = atomicAdd(&A.scan_done[b * A.Hkv + h], 1);
        s_last = done == A.ns_scan - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const unsigned long long *all = A.cand + ((int64_t)b * A.Hkv + h) * A.ns_scan * A.K_c;
    const int ntot = A.ns_scan * A.K_c;
    for (int r = threadIdx.x; r < ntot; r += blockDim.x) cand[r] = __ldcg(all + r);
    __syncthreads();
    // keys of 0 are padding: they never beat a real key, and only min(K_c,
    // real) keys are kept, so count the real ones
    int nreal = 0;
    for (int r = 0; r < ntot; ++r) nreal += cand[r] != 0;
    // compact (stable) so padding does not count as a candidate
    __syncthreads();
    if (threadIdx.x == 0) {
        int w = 0;
        for (int r = 0; r < ntot; ++r)
            if (cand[r] != 0) cand[w++] = cand[r];
    }
    __syncthreads();
    const int kc = topk_select(cand, nreal, A.K_c, rs.sel_c, rs);
    int32_t *oc = A.sel_c + ((int64_t)b * A.Hkv + h) * A.K_c;
    for (int r = threadIdx.x; r < A.K_c; r += blockDim.x) oc[r] = r < kc ? rs.sel_c[r] : -1;
    const float *Sg = A.s_group + ((int64_t)b * A.Hkv + h) * A.nc_cap * A.gpc * D;
    __syncthreads();
    score_group_rows<D>(qr, Sg, rs.sel_c, A.gpc, kc * A.gpc, cand);
    __syncthreads();
    const int kg = topk_select(cand, kc * A.gpc, A.K_g, rs.sel_g, rs);
    int32_t *og = A.sel_g + ((int64_t)b * A.Hkv + h) * A.K_g;
    for (int r = threadIdx.x; r < A.K_g; r += blockDim.x) og[r] = r < kg ? rs.sel_g[r] : -1;
    if (threadIdx.x == 0) A.scan_done[b * A.Hkv + h] = 0;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) k_decode_attend(const DecodeArgs A) {
    constexpr int H = D / 2, DL = D / 32;   // dims per lane
    extern __shared__ __align__(16) unsigned char smem[];
    // regions: keys (int, keys_max rounded to 4), q [G][D], scores [G][per_max]
    // (per_max a multiple of 4), K and V rows [per_max][D]; all 16-byte aligned
    int *keys = reinterpret_cast<int *>(smem);
    float *qs = reinterpret_cast<float *>(smem + sizeof(int) * ((A.keys_max + 3) & ~3));
    float *sc = qs + A.G * D;
    T *Ks = reinterpret_cast<T *>(sc + A.G * A.per_max);
    T *Vs = Ks + (size_t)A.per_max * D;
    __shared__ RunList rl;
    __shared__ int s_last, s_seq_last;

    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int t = A.lens[b];
    if (t < 0 || t >= A.Tc) return;
    const int c = t / A.C;
    const int32_t pnew = A.pos_new[b];

    if (threadIdx.x == 0)
        build_runs(rl, c, A.F, A.L, A.g_s, A.sel_g + ((int64_t)b * A.Hkv + h) * A.K_g, A.K_g,
                   t - c * A.C + 1);
    // rotated, pre-scaled queries of the G heads
    const T *qb = static_cast<const T *>(A.q_new) + ((int64_t)b * A.Hq + (int64_t)h * A.G) * D;
    for (int e = threadIdx.x; e < A.G * H; e += blockDim.x) {
        const int g = e / H, i = e % H;
        const float2 r = rope_cs(A.rope, (double)pnew, i);
        const float x = to_f(qb[g * D + i]), y = to_f(qb[g * D + i + H]);
        qs[g * D + i] = (x * r.x - y * r.y) * A.scale_log2;
        qs[g * D + i + H] = (y * r.x + x * r.y) * A.scale_log2;
    }
    __syncthreads();
    fill_keys(rl, keys);
    const int nkeys = rl.off[rl.n];
    const int per = (nkeys + kAttSplits - 1) / kAttSplits;
    const int k0 = min(nkeys, s * per), nk = min(nkeys, k0 + per) - k0;
    __syncthreads();

    // stage this slice's K and V rows (16-byte loads)
    constexpr int VPR = D * (int)sizeof(T) / 16;   // 16-byte vectors per row
    const T *kbase = static_cast<const T *>(A.k_rot);
    const T *vbase = static_cast<const T *>(A.v);
    for (int e = threadIdx.x; e < nk * VPR; e += blockDim.x) {
        const int k = e / VPR, part = e % VPR;
        const int64_t row = ((int64_t)b * A.Tc + keys[k0 + k]) * A.Hkv + h;
        reinterpret_cast<uint4 *>(Ks + (size_t)k * D)[part] =
            __ldg(reinterpret_cast<const uint4 *>(kbase + row * D) + part);
        reinterpret_cast<uint4 *>(Vs + (size_t)k * D)[part] =
            __ldg(reinterpret_cast<const uint4 *>(vbase + row * D) + part);
    }
    __syncthreads();

    // scores: one warp per key, lanes over dims, all G heads
    for (int k = warp; k < nk; k += nw) {
        float kv[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) kv[e] = to_f(Ks[(size_t)k * D + lane * DL + e]);
        for (int g = 0; g < A.G; ++g) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < DL; ++e) a = fmaf(qs[g * D + lane * DL + e], kv[e], a);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (lane == 0) sc[g * A.per_max + k] = a;
        }
    }
    __syncthreads();

    // per head: max, exponentials, sum, then P.V over this slice
    float *part_b = A.part + ((int64_t)b * A.Hq + (int64_t)h * A.G) * kAttSplits * (D + 2);
    for (int g = warp; g < A.G; g += nw) {
        float m = -INFINITY;
        for (int k = lane; k < nk; k += 32) m = fmaxf(m, sc[g * A.per_max + k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int k = lane; k < nk; k += 32) {
            const float p = nk > 0 ? exp2f(sc[g * A.per_max + k] - m) : 0.f;
            sc[g * A.per_max + k] = p;
            l += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        __syncwarp();
        float o_acc[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) o_acc[e] = 0.f;
        for (int k = 0; k < nk; ++k) {
            const float p = sc[g * A.per_max + k];
#pragma unroll
            for (int e = 0; e < DL; ++e)
                o_acc[e] = fmaf(p, to_f(Vs[(size_t)k * D + lane * DL + e]), o_acc[e]);
        }
        float *dst = part_b + ((int64_t)g * kAttSplits + s) * (D + 2);
#pragma unroll
        for (int e = 0; e < DL; ++e) dst[2 + lane * DL + e] = o_acc[e];
        if (lane == 0) {
            dst[0] = nk > 0 ? m : -INFINITY;
            dst[1] = l;
        }
    }

    // ---- the last split of this (sequence, KV head) combines
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int done = atomicAdd(&A.att_done[b * A.Hkv + h], 1);
        s_last = done == kAttSplits - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int g = warp; g < A.G; g += nw) {
        const float *src = part_b + (int64_t)g * kAttSplits * (D + 2);
        float M = -INFINITY;
        for (int sp = 0; sp < kAttSplits; ++sp) M = fmaxf(M, __ldcg(src + sp * (D + 2)));
        float L = 0.f, o_acc[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) o_acc[e] = 0.f;
        for (int sp = 0; sp < kAttSplits; ++sp) {
            const float ms = __ldcg(src + sp * (D + 2));
            if (ms == -INFINITY) continue;
            const float w = exp2f(ms - M);
            L += w * __ldcg(src + sp * (D + 2) + 1);
#pragma unroll
            for (int e = 0; e < DL; ++e) o_acc[e] += w * __ldcg(src + sp * (D + 2) + 2 + lane * DL + e);
        }
        const float inv = 1.f / L;
        T *o = static_cast<T *>(A.out) + ((int64_t)b * A.Hq + (int64_t)h * A.G + g) * D;
#pragma unroll
        for (int e = 0; e < DL; ++e) o[lane * DL + e] = from_f<T>(o_acc[e] * inv);
        if (A.lse && lane == 0)
            A.lse[(int64_t)b * A.Hq + (int64_t)h * A.G + g] = (M + __log2f(L)) * 0.6931471805599453f;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        A.att_done[b * A.Hkv + h] = 0;
        __threadfence();
        const int done = atomicAdd(&A.seq_done[b], 1);
        s_seq_last = done == A.Hkv - 1;
        if (s_seq_last) {
            A.seq_done[b] = 0;
            A.lens[b] = t + 1;
        }
    }
}

struct Ws {
    size_t counters, cand, sel_c, sel_g, part, total;
};

inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

Ws layout(const Geo &g) {
    const int ns = ((g.T / g.C) + kScanChunks - 1) / kScanChunks;
    Ws w;
    size_t o = 0;
    w.counters = o;
    o += up256(sizeof(int32_t) * (size_t)(2 * g.B * g.Hkv + g.B));
    w.cand = o;
    o += up256(sizeof(unsigned long long) * (size_t)g.B * g.Hkv * ns * g.K_c);
    w.sel_c = o;
    o += up256(sizeof(int32_t) * (size_t)g.B * g.Hkv * g.K_c);
    w.sel_g = o;
    o += up256(sizeof(int32_t) * (size_t)g.B * g.Hkv * g.K_g);
    w.part = o;
    o += up256(sizeof(float) * (size_t)g.B * g.Hq * kAttSplits * (g.D + 2));
    w.total = o;
    return w;
}

template <typename T, int D>
hga_status run(const Geo &g, const Rope &r, const hga_io &io, void *ws, cudaStream_t st) {
    const Ws w = layout(g);
    char *base = static_cast<char *>(ws);
    DecodeArgs A;
    A.B = g.B;
    A.Tc = g.T;
    A.Hq = g.Hq;
    A.Hkv = g.Hkv;
    A.G = g.G;
    A.C = g.C;
    A.g_s = g.g_s;
    A.gpc = g.gpc;
    A.F = g.F;
    A.L = g.L;
    A.K_c = g.K_c;
    A.K_g = g.K_g;
    A.nc_cap = g.T / g.C;
    A.ns_scan = (A.nc_cap + kScanChunks - 1) / kScanChunks;
    A.keys_max = (int)min((long long)(g.F + max(g.L, 1) + 1) * g.C + (long long)g.K_g * g.g_s,
                          (long long)g.T);
    A.per_max = (((A.keys_max + kAttSplits - 1) / kAttSplits) + 3) & ~3;
    A.q_new = io.q_new;
    A.k_new = io.k_new;
    A.v_new = io.v_new;
    A.pos_new = io.pos_new;
    A.k_rot = io.cache.k_rot;
    A.v = io.cache.v;
    A.pos = io.cache.pos;
    A.k_open = io.cache.k_open;
    A.s_chunk = io.cache.s_chunk;
    A.s_group = io.cache.s_group;
    A.lens = io.cache.lens;
    A.out = io.out;
    A.lse = io.lse;
    A.sel_c = io.sel_chunk ? io.sel_chunk : reinterpret_cast<int32_t *>(base + w.sel_c);
    A.sel_g = io.sel_group ? io.sel_group : reinterpret_cast<int32_t *>(base + w.sel_g);
    A.cand = reinterpret_cast<unsigned long long *>(base + w.cand);
    A.part = reinterpret_cast<float *>(base + w.part);
    int32_t *cnt = reinterpret_cast<int32_t *>(base + w.counters);
    A.scan_done = cnt;
    A.att_done = cnt + g.B * g.Hkv;
    A.seq_done = cnt + 2 * g.B * g.Hkv;
    A.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    A.rope = r;

    const size_t smem_scan = sizeof(unsigned long long) *
        (size_t)max(max(kScanChunks, A.ns_scan * g.K_c), g.K_c * g.gpc);
    const size_t smem_att = sizeof(int) * (size_t)((A.keys_max + 3) & ~3) +
        sizeof(float) * (size_t)(g.G * D + g.G * A.per_max) + 2 * sizeof(T) * (size_t)A.per_max * D;
    if (smem_scan > 200 * 1024 || smem_att > 200 * 1024) return HGA_ERR_UNSUPPORTED;
    auto ks = k_decode_scan<T, D>;
    auto ka = k_decode_attend<T, D>;
    cudaError_t e = ensure_smem((const void *)ks, smem_scan);
    if (e == cudaSuccess)
        e = ensure_smem((const void *)ka, smem_att);
    if (e != cudaSuccess) return cuda_status(e);
    ks<<<dim3(A.ns_scan, g.Hkv, g.B), kThreads, smem_scan, st>>>(A);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
    ka<<<dim3(kAttSplits, g.Hkv, g.B), kThreads, smem_att, st>>>(A);
    return cuda_status(cudaGetLastError());
}

}  // namespace

size_t decode_workspace_bytes(const Geo &g) { return layout(g).total; }

hga_status launch_decode(const Geo &g, const Rope &r, int dtype, const hga_io &io, void *ws,
                         cudaStream_t st) {
    if (dtype == HGA_BF16)
        return g.D == 128 ? run<__nv_bfloat16, 128>(g, r, io, ws, st)
                          : run<__nv_bfloat16, 64>(g, r, io, ws, st);
    return g.D == 128 ? run<float, 128>(g, r, io, ws, st) : run<float, 64>(g, r, io, ws, st);
}

}  // namespace hga
