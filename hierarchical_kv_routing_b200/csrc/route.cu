// Stage 2: two-level routing per (query block, KV head).
//
// Method: HGA paper-review page, section 3, routing policy ("路由策略") and
// the selection equation: the query scores the chunk summaries of the middle
// context (score_m = q . c_m), keeps the top K_c chunks, then scores the group
// summaries inside those chunks and keeps the top K_g groups, whose exact
// token K/V are then opened.  The routing query of a 64-token prefill block
// and KV head is the block's RoPE-rotated queries summed over its tokens and
// over the KV head's query heads.
//
// Design: one CTA per (run of up to 8 consecutive query blocks, KV head,
// sequence).  Phase 1 streams the run's queries from HBM (the only large
// read: every thread keeps one token's G head rows in flight as 16-byte
// loads, sums the heads in fp32 (RoPE is linear), rotates, and accumulates
// over tokens in fp64; warp shuffles and one shared-memory pass reduce over
// tokens).  All of a run's CTAs stream at once, so the GPU's whole load
// capacity works on Q.  Phase 2 reads each middle-chunk summary row once and
// scores it against all the run's routing queries (fp64 dot products, the
// query broadcast from shared memory), which cuts the chunk table's L2
// traffic by the run length; one warp per block then takes its top K_c
// (keys below a threshold that cannot reach the top K_c dropped first, then
// warp bitonic sort and merge of packed (fp32 score, id) keys), scores the
// groups of its chunks and takes the top K_g.  K above 32 falls back to
// CTA-wide selection rounds, one block at a time.
#include <climits>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "hga_internal.cuh"
#include "route_common.cuh"
#include "route_schedule.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kBlk = 8;                          // query blocks per CTA at most
constexpr size_t kCandBytes = 160 * 1024;        // shared candidate table budget

struct RouteArgs {
    const void *q;
    __nv_bfloat16 *q_rot;        // optional (bf16 only): rotated queries out
    const int32_t *pos;
    int T, Hq, Hkv, G, NB, F, L, K_c, K_g, gpc, nc_cap, nblk, ncap;
    const float *s_chunk, *s_group;
    int32_t *sel_chunk, *sel_group;
    Rope rope;
};

// kHostGroups: the group summary table is in pinned host memory (the host
// tier's cold store) and its rows are read over the link with plain loads.
// kWriteQ (bf16): every head's rotated query is also written to A.q_rot; the
// (token, pair) angles are then held across the head loop, so fewer head
// rows are kept in flight to stay within the register budget.
template <typename T, int D, bool kHostGroups, bool kWriteQ>
__global__ void __launch_bounds__(kThreads, 2) k_route(const RouteArgs A) {
    constexpr int H = D / 2;
    constexpr int EPW = 16 / (int)sizeof(T);     // elements per 16-byte word
    constexpr int NS = H / EPW;                  // words per half row
    constexpr int TP = kThreads / NS;            // tokens per pass
    constexpr int HB = sizeof(T) == 2 && !kWriteQ ? 8 : 4;   // head rows in flight per thread
    extern __shared__ __align__(16) unsigned char smem[];
    double *qr = reinterpret_cast<double *>(smem);                            // [kBlk][D]
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(qr + kBlk * D);
    __shared__ double part[kThreads / 32][D];
    __shared__ int sel_s[kBlk][32];
    __shared__ int kc_s[kBlk];
    __shared__ unsigned long long lists[kThreads];
    __shared__ RouteScratch rs;

    int run, unit;
    pair_slot((int)((blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x), (int)gridDim.x,
              (int)(gridDim.y * gridDim.z), &run, &unit);
    const int h = unit % (int)gridDim.y, b = unit / (int)gridDim.y;
    const int c0 = run * A.nblk;
    const int nb = min(A.nblk, A.NB - c0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T *q = static_cast<const T *>(A.q);

    // Launched as a programmatic dependent of the previous kernel on the
    // stream: nothing that kernel may write is read before it completes.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- phase 1: routing queries sum_i sum_{h'} R_{p_i}(q_{i,h'}), per block
    const int w = threadIdx.x % NS, jt = threadIdx.x / NS;
    for (int blk = 0; blk < nb; ++blk) {
        const int t0 = (c0 + blk) * kChunk;
        const int n = min(kChunk, A.T - t0);
        double al[EPW], ah[EPW];
#pragma unroll
        for (int e = 0; e < EPW; ++e) al[e] = ah[e] = 0.0;
        for (int j = jt; j < n; j += TP) {
            const int64_t row0 = ((int64_t)b * A.T + t0 + j) * A.Hq + (int64_t)h * A.G;
            const T *row = q + row0 * D;
            const int32_t p = A.pos[(int64_t)b * A.T + t0 + j];
            // the angles of this word's pairs serve every head and the sum
            // (formed up front only when every head is rotated and written)
            float2 cs[EPW];
            if constexpr (kWriteQ)
#pragma unroll
                for (int e = 0; e < EPW; ++e) cs[e] = rope_cs_int(A.rope, p, w * EPW + e);
            float lo[EPW], hi[EPW];
#pragma unroll
            for (int e = 0; e < EPW; ++e) lo[e] = hi[e] = 0.f;
            for (int g0 = 0; g0 < A.G; g0 += HB) {
                uint4 wl[HB], wh[HB];
#pragma unroll
                for (int u = 0; u < HB; ++u)
                    if (g0 + u < A.G) {
                        wl[u] = __ldg(reinterpret_cast<const uint4 *>(row + (g0 + u) * D) + w);
                        wh[u] = __ldg(reinterpret_cast<const uint4 *>(row + (g0 + u) * D + H) + w);
                    }
#pragma unroll
                for (int u = 0; u < HB; ++u)
                    if (g0 + u < A.G) {
                        float a[EPW], c[EPW];
                        unpack_words<T, EPW>(reinterpret_cast<const uint4(&)[1]>(wl[u]), a);
                        unpack_words<T, EPW>(reinterpret_cast<const uint4(&)[1]>(wh[u]), c);
#pragma unroll
                        for (int e = 0; e < EPW; ++e) {
                            lo[e] += a[e];
                            hi[e] += c[e];
                        }
                        if constexpr (kWriteQ && sizeof(T) == 2) {
                            // this head's rotated query, rounded as the
                            // attention kernel rounds its own rotation
                            {
                                uint4 ol, oh;
                                __nv_bfloat162 *pl = reinterpret_cast<__nv_bfloat162 *>(&ol);
                                __nv_bfloat162 *ph = reinterpret_cast<__nv_bfloat162 *>(&oh);
#pragma unroll
                                for (int e = 0; e < EPW / 2; ++e) {
                                    const float2 r0 = rot_pair(a[2 * e], c[2 * e], cs[2 * e]);
                                    const float2 r1 = rot_pair(a[2 * e + 1], c[2 * e + 1], cs[2 * e + 1]);
                                    pl[e] = __floats2bfloat162_rn(r0.x, r1.x);
                                    ph[e] = __floats2bfloat162_rn(r0.y, r1.y);
                                }
                                __nv_bfloat16 *orow = A.q_rot + (row0 + g0 + u) * D;
                                reinterpret_cast<uint4 *>(orow)[w] = ol;
                                reinterpret_cast<uint4 *>(orow + H)[w] = oh;
                            }
                        }
                    }
            }
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
                if constexpr (!kWriteQ) cs[e] = rope_cs_int(A.rope, p, w * EPW + e);
                const float2 rr = rot_pair(lo[e], hi[e], cs[e]);
                al[e] += (double)rr.x;
                ah[e] += (double)rr.y;
            }
        }
        // lanes holding the same word: reduce over their tokens
#pragma unroll
        for (int off = NS; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
                al[e] += __shfl_xor_sync(0xffffffffu, al[e], off);
                ah[e] += __shfl_xor_sync(0xffffffffu, ah[e], off);
            }
        if (lane < NS)
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
                part[warp][w * EPW + e] = al[e];
                part[warp][H + w * EPW + e] = ah[e];
            }
        __syncthreads();
        if (threadIdx.x < D) {
            double sum = 0.0;
#pragma unroll
            for (int wp = 0; wp < kThreads / 32; ++wp) sum += part[wp][threadIdx.x];
            qr[blk * D + threadIdx.x] = sum;
        }
        __syncthreads();
    }

    // the next kernel (stage 3) may be launched as this one winds down
    asm volatile("griddepcontrol.launch_dependents;");

    // ---- phase 2: chunk scores for every block of the run, one row read once
    const float *Sc = A.s_chunk + ((int64_t)b * A.Hkv + h) * A.nc_cap * D;
    const float *Sg = A.s_group + ((int64_t)b * A.Hkv + h) * A.nc_cap * A.gpc * D;
    const int n_rows = max(0, middle_hi(c0 + nb - 1, A.L) - A.F + 1);
    // two rows per thread (r and r + kThreads): each query value read from
    // shared memory (as a pair of dims) serves both rows
    for (int r = threadIdx.x; r < n_rows; r += 2 * kThreads) {
        const int r2 = r + kThreads;
        const bool two = r2 < n_rows;
        const float4 *ra = reinterpret_cast<const float4 *>(Sc + (int64_t)(A.F + r) * D);
        const float4 *rb = reinterpret_cast<const float4 *>(Sc + (int64_t)(A.F + (two ? r2 : r)) * D);
        double acc[kBlk], acc2[kBlk];
#pragma unroll
        for (int k = 0; k < kBlk; ++k) acc[k] = acc2[k] = 0.0;
#pragma unroll 1
        for (int base = 0; base < D / 4; base += 4) {
            float4 va[4], vb[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                va[e] = __ldg(ra + base + e);
                vb[e] = __ldg(rb + base + e);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = 4 * (base + e);
#pragma unroll
                for (int k = 0; k < kBlk; ++k) {
                    if (k < nb) {
                        const double2 q01 = *reinterpret_cast<const double2 *>(qr + k * D + d);
                        const double2 q23 = *reinterpret_cast<const double2 *>(qr + k * D + d + 2);
                        acc[k] = fma(q01.x, (double)va[e].x, acc[k]);
                        acc2[k] = fma(q01.x, (double)vb[e].x, acc2[k]);
                        acc[k] = fma(q01.y, (double)va[e].y, acc[k]);
                        acc2[k] = fma(q01.y, (double)vb[e].y, acc2[k]);
                        acc[k] = fma(q23.x, (double)va[e].z, acc[k]);
                        acc2[k] = fma(q23.x, (double)vb[e].z, acc2[k]);
                        acc[k] = fma(q23.y, (double)va[e].w, acc[k]);
                        acc2[k] = fma(q23.y, (double)vb[e].w, acc2[k]);
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kBlk; ++k)
            if (k < nb) {
                const int mh = middle_hi(c0 + k, A.L);
                cand[k * A.ncap + r] = A.F + r <= mh ? pack_key((float)acc[k], A.F + r) : 0ull;
                if (two)
                    cand[k * A.ncap + r2] = A.F + r2 <= mh ? pack_key((float)acc2[k], A.F + r2) : 0ull;
            }
    }
    __syncthreads();

    if (A.K_c <= 32 && A.K_g <= 32) {
        // one warp per block: top K_c chunks, then its groups and top K_g
        for (int k = warp; k < nb; k += kThreads / 32) {
            const int c = c0 + k;
            const int n_mid = max(0, middle_hi(c, A.L) - A.F + 1);
            const unsigned long long top = warp_topk_filtered(cand + k * A.ncap, n_mid, A.K_c);
            const bool take = lane < A.K_c && top != 0ull;
            const int id = warp_sort_asc_int(take ? key_id(top) : 0x7fffffff);
            const int kc = min(A.K_c, n_mid);
            sel_s[k][lane] = id;
            int32_t *oc = A.sel_chunk + (((int64_t)b * A.NB + c) * A.Hkv + h) * A.K_c;
            if (lane < A.K_c) oc[lane] = lane < kc ? id : -1;
            if (lane == 0) kc_s[k] = kc;
        }
        __syncthreads();
        // group candidates of every block at once (the chunk table is free)
        const int slots = A.K_c * A.gpc;
        for (int x = threadIdx.x; x < nb * slots; x += kThreads) {
            const int k = x / slots, r = x % slots;
            if (r < kc_s[k] * A.gpc) {
                const int gid = sel_s[k][r / A.gpc] * A.gpc + r % A.gpc;
                cand[k * A.ncap + r] =
                    pack_key((float)thread_dot_row<D, kHostGroups>(qr + k * D, Sg + (int64_t)gid * D), gid);
            }
        }
        __syncthreads();
        for (int k = warp; k < nb; k += kThreads / 32) {
            const int c = c0 + k;
            const int ng = kc_s[k] * A.gpc;
            const unsigned long long top = warp_topk_filtered(cand + k * A.ncap, ng, A.K_g);
            const bool take = lane < A.K_g && top != 0ull;
            const int id = warp_sort_asc_int(take ? key_id(top) : 0x7fffffff);
            const int kg = min(A.K_g, ng);
            int32_t *og = A.sel_group + (((int64_t)b * A.NB + c) * A.Hkv + h) * A.K_g;
            if (lane < A.K_g) og[lane] = lane < kg ? id : -1;
        }
        return;
    }

    // K above 32: CTA-wide selection rounds, one block at a time
    for (int k = 0; k < nb; ++k) {
        const int c = c0 + k;
        const int n_mid = max(0, middle_hi(c, A.L) - A.F + 1);
        unsigned long long *ck = cand + k * A.ncap;
        const int kc = min(A.K_c, n_mid);
        if (A.K_c <= 32) block_topk32(ck, n_mid, A.K_c, rs.sel_c, lists);
        else topk_select(ck, n_mid, A.K_c, rs.sel_c, rs);
        int32_t *oc = A.sel_chunk + (((int64_t)b * A.NB + c) * A.Hkv + h) * A.K_c;
        for (int r = threadIdx.x; r < A.K_c; r += kThreads) oc[r] = r < kc ? rs.sel_c[r] : -1;
        __syncthreads();
        const int ng = kc * A.gpc;
        for (int r = threadIdx.x; r < ng; r += kThreads) {
            const int gid = rs.sel_c[r / A.gpc] * A.gpc + r % A.gpc;
            ck[r] = pack_key((float)thread_dot_row<D, kHostGroups>(qr + k * D, Sg + (int64_t)gid * D), gid);
        }
        __syncthreads();
        const int kg = min(A.K_g, ng);
        if (A.K_g <= 32) block_topk32(ck, ng, A.K_g, rs.sel_g, lists);
        else topk_select(ck, ng, A.K_g, rs.sel_g, rs);
        int32_t *og = A.sel_group + (((int64_t)b * A.NB + c) * A.Hkv + h) * A.K_g;
        for (int r = threadIdx.x; r < A.K_g; r += kThreads) og[r] = r < kg ? rs.sel_g[r] : -1;
        __syncthreads();
    }
}

// SM count and resident CTAs per SM of `kern` at `smem` bytes on the current
// device (looked up once per kernel, size and device).
cudaError_t residency(const void *kern, size_t smem, int *sms, int *per_sm) {
    static std::mutex mu;
    static std::map<std::tuple<const void *, size_t, int>, std::pair<int, int>> seen;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(kern, smem, dev);
    auto it = seen.find(key);
    if (it == seen.end()) {
        int n = 0, k = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&k, kern, kThreads, smem);
        if (e != cudaSuccess) return e;
        it = seen.emplace(key, std::make_pair(n, k)).first;
    }
    *sms = it->second.first;
    *per_sm = it->second.second;
    return cudaSuccess;
}

template <typename T, int D>
hga_status run(const Geo &g, const Rope &r, const void *q, const int32_t *pos,
               const float *s_chunk, const float *s_group, int nc_cap, int32_t *sel_chunk,
               int32_t *sel_group, cudaStream_t st, bool host_groups, void *q_rot) {
    RouteArgs a;
    a.q = q;
    a.q_rot = static_cast<__nv_bfloat16 *>(q_rot);
    a.pos = pos;
    a.T = g.T;
    a.Hq = g.Hq;
    a.Hkv = g.Hkv;
    a.G = g.G;
    a.NB = g.NB;
    a.F = g.F;
    a.L = g.L;
    a.K_c = g.K_c;
    a.K_g = g.K_g;
    a.gpc = g.gpc;
    a.nc_cap = nc_cap;
    // candidate rows per block: middle chunks, or the selected chunks' groups
    a.ncap = (int)max(max((long long)g.NC, 1ll), (long long)min(g.K_c, g.NC) * g.gpc);
    const size_t row_bytes = sizeof(unsigned long long) * (size_t)a.ncap;
    if (row_bytes > kCandBytes) return HGA_ERR_UNSUPPORTED;   // must fit on chip
    const int nmax = (int)min((size_t)kBlk, kCandBytes / row_bytes);
    a.s_chunk = s_chunk;
    a.s_group = s_group;
    a.sel_chunk = sel_chunk;
    a.sel_group = sel_group;
    a.rope = r;
    // shared memory sized for the longest run, so the residency does not
    // depend on the run length picked below
    const size_t smem = sizeof(double) * kBlk * D + row_bytes * nmax;
    auto kern = host_groups ? k_route<T, D, true, false>
                            : (q_rot ? k_route<T, D, false, true> : k_route<T, D, false, false>);
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    int sms = 0, per_sm = 0;
    e = residency((const void *)kern, smem, &sms, &per_sm);
    if (e != cudaSuccess) return cuda_status(e);
    a.nblk = per_sm > 0 ? pick_run(g.NB, g.Hkv * g.B, nmax, sms, per_sm) : nmax;
    // the kernel forms a 32-bit linear CTA index
    if ((long long)((g.NB + a.nblk - 1) / a.nblk) * g.Hkv * g.B > (long long)INT32_MAX)
        return HGA_ERR_UNSUPPORTED;
    // a programmatic dependent of the previous kernel on the stream: when
    // that is stage 1 (which triggers early), the launch and set-up overlap it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((g.NB + a.nblk - 1) / a.nblk, g.Hkv, g.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, a));
}

}  // namespace

hga_status launch_route(const Geo &g, const Rope &r, int dtype, const void *q, const int32_t *pos,
                        const float *s_chunk, const float *s_group, int nc_cap,
                        int32_t *sel_chunk, int32_t *sel_group, cudaStream_t st,
                        bool host_groups, void *q_rot) {
    if (g.NB <= 0) return HGA_OK;
    if (dtype == HGA_BF16)
        return g.D == 128 ? run<__nv_bfloat16, 128>(g, r, q, pos, s_chunk, s_group, nc_cap,
                                                     sel_chunk, sel_group, st, host_groups, q_rot)
                          : run<__nv_bfloat16, 64>(g, r, q, pos, s_chunk, s_group, nc_cap,
                                                    sel_chunk, sel_group, st, host_groups, q_rot);
    if (q_rot) return HGA_ERR_UNSUPPORTED;       // rotated queries are written in bf16 only
    return g.D == 128 ? run<float, 128>(g, r, q, pos, s_chunk, s_group, nc_cap, sel_chunk,
                                        sel_group, st, host_groups, nullptr)
                      : run<float, 64>(g, r, q, pos, s_chunk, s_group, nc_cap, sel_chunk,
                                       sel_group, st, host_groups, nullptr);
}

}  // namespace hga
