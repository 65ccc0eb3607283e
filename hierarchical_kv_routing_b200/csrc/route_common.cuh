// Scoring and top-K selection shared by the prefill and decode routers
// (256-thread CTAs).  Method: HGA paper-review page, section 3, routing
// policy and selection equation: scores are plain dot products q . s; the top
// K candidates are kept, the lower id winning on equal scores.
#pragma once
#include "hga_internal.cuh"
#include "vec.cuh"

namespace hga {

constexpr int kRouteThreads = 256;
constexpr int kMaxK = 1024;     // largest K_c or K_g a router accepts

struct RouteScratch {
    int sel_c[kMaxK];           // selected chunk ids, ascending
    int sel_g[kMaxK];           // selected group ids, ascending
    int tmp[kMaxK];
    unsigned long long wmax[kRouteThreads / 32];
    unsigned long long best;
};

// One fp64 dot product of q (shared, fp64) with an fp32 row, by one warp.
template <int D>
__device__ __forceinline__ double warp_dot_row(const double *qr, const float *__restrict__ row) {
    const int lane = threadIdx.x & 31;
    double s = 0.0;
    if constexpr (D == 128) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(row) + lane);
        s = qr[4 * lane] * v.x + qr[4 * lane + 1] * v.y + qr[4 * lane + 2] * v.z +
            qr[4 * lane + 3] * v.w;
    } else {
        const float2 v = __ldg(reinterpret_cast<const float2 *>(row) + lane);
        s = qr[2 * lane] * v.x + qr[2 * lane + 1] * v.y;
    }
    return warp_sum_f64(s);
}

// cand[r] = key(q . S[first + r], first + r) for r < n (one warp per row).
template <int D>
__device__ __forceinline__ void score_rows(const double *qr, const float *__restrict__ S, int first,
                                           int n, unsigned long long *cand) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int r = warp; r < n; r += nw) {
        const double s = warp_dot_row<D>(qr, S + (int64_t)(first + r) * D);
        if (lane == 0) cand[r] = pack_key((float)s, first + r);
    }
}

// cand[r] = key(q . Sg[gid], gid), gid = sel_c[r / gpc] * gpc + r % gpc.
template <int D>
__device__ __forceinline__ void score_group_rows(const double *qr, const float *__restrict__ Sg,
                                                 const int *sel_c, int gpc, int n,
                                                 unsigned long long *cand) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int r = warp; r < n; r += nw) {
        const int gid = sel_c[r / gpc] * gpc + r % gpc;
        const double s = warp_dot_row<D>(qr, Sg + (int64_t)gid * D);
        if (lane == 0) cand[r] = pack_key((float)s, gid);
    }
}

// Ascending sort of k ids (rank sort; ids are distinct).  in != out.
__device__ __forceinline__ void sort_ids(const int *in, int *out, int k) {
    for (int t = threadIdx.x; t < k; t += blockDim.x) {
        const int v = in[t];
        int rank = 0;
        for (int u = 0; u < k; ++u) rank += in[u] < v;
        out[rank] = v;
    }
    __syncthreads();
}

// Top-K of n candidate keys (cand is consumed).  Writes the chosen ids,
// ascending, to out; returns min(K, n).  Call with the whole CTA.
__device__ __forceinline__ int topk_select(unsigned long long *cand, int n, int K, int *out,
                                           RouteScratch &rs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = min(K, n);
    if (n <= K) {
        for (int r = threadIdx.x; r < n; r += blockDim.x) rs.tmp[r] = key_id(cand[r]);
        __syncthreads();
        sort_ids(rs.tmp, out, n);
        return n;
    }
    for (int round = 0; round < k; ++round) {
        unsigned long long m = 0;
        for (int r = threadIdx.x; r < n; r += blockDim.x) m = cand[r] > m ? cand[r] : m;
        m = warp_max_u64(m);
        if (lane == 0) rs.wmax[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long b = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = rs.wmax[w] > b ? rs.wmax[w] : b;
            rs.best = b;
            rs.tmp[round] = key_id(b);
        }
        __syncthreads();
        const unsigned long long b = rs.best;
        for (int r = threadIdx.x; r < n; r += blockDim.x)
            if (cand[r] == b) cand[r] = 0;
    }
    __syncthreads();
    sort_ids(rs.tmp, out, k);
    return k;
}

}  // namespace hga

namespace hga {

// The K largest candidate keys (cand is consumed), written to out[0..K)
// (global or shared), descending, padded with 0.  Returns min(K, n).
__device__ __forceinline__ int topk_keys(unsigned long long *cand, int n, int K,
                                         unsigned long long *out, RouteScratch &rs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = min(K, n);
    for (int round = 0; round < k; ++round) {
        unsigned long long m = 0;
        for (int r = threadIdx.x; r < n; r += blockDim.x) m = cand[r] > m ? cand[r] : m;
        m = warp_max_u64(m);
        if (lane == 0) rs.wmax[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long b = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = rs.wmax[w] > b ? rs.wmax[w] : b;
            rs.best = b;
            out[round] = b;
        }
        __syncthreads();
        const unsigned long long b = rs.best;
        for (int r = threadIdx.x; r < n; r += blockDim.x)
            if (cand[r] == b) cand[r] = 0;
    }
    for (int r = k + threadIdx.x; r < K; r += blockDim.x) out[r] = 0;
    __syncthreads();
    return k;
}

}  // namespace hga

namespace hga {

// ---- register top-K for K <= 32: warp bitonic sort and merge of packed keys

// Sort the warp's 32 keys, one per lane, descending (lane 0 = largest).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const unsigned long long p = __shfl_xor_sync(0xffffffffu, v, j);
            const bool take_max = ((lane & j) == 0) == ((lane & k) == 0);
            v = take_max ? (p > v ? p : v) : (p < v ? p : v);
        }
    }
    return v;
}

// Top 32 of two descending lists a and b (one key per lane), descending.
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long a,
                                                              unsigned long long b) {
    const int lane = threadIdx.x & 31;
    const unsigned long long br = __shfl_sync(0xffffffffu, b, 31 - lane);
    unsigned long long v = a > br ? a : br;   // bitonic: the top 32 of the union
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const unsigned long long p = __shfl_xor_sync(0xffffffffu, v, j);
        v = ((lane & j) == 0) ? (p > v ? p : v) : (p < v ? p : v);
    }
    return v;
}

// Ascending sort of 32 ints across a warp (padding = INT_MAX).
__device__ __forceinline__ int warp_sort_asc_int(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int p = __shfl_xor_sync(0xffffffffu, v, j);
            const bool take_min = ((lane & j) == 0) == ((lane & k) == 0);
            v = take_min ? min(v, p) : max(v, p);
        }
    }
    return v;
}

// The warp's top 32 of n keys in smem/global (strided by the warp count),
// descending.  warp_index/n_warps split the candidates between warps.
__device__ __forceinline__ unsigned long long warp_top32(const unsigned long long *cand, int n,
                                                         int warp_index, int n_warps) {
    const int lane = threadIdx.x & 31;
    unsigned long long acc = 0;
    for (int base = warp_index * 32; base < n; base += n_warps * 32) {
        const unsigned long long x = base + lane < n ? cand[base + lane] : 0ull;
        acc = warp_merge_desc(acc, warp_sort_desc(x));
    }
    return acc;
}

// The warp's top 32 of n keys in shared memory, descending, where only the
// top K (K <= 32) will be used.  At least K lanes hold a key as large as the
// K-th largest of the lanes' maxima (tau), so every top-K key is >= tau:
// the keys below tau are dropped first (cand is compacted in place), which
// leaves the sort-and-merge rounds a few dozen keys instead of n.
__device__ __forceinline__ unsigned long long warp_topk_filtered(unsigned long long *cand, int n,
                                                                 int K) {
    const int lane = threadIdx.x & 31;
    if (n <= 64) return warp_top32(cand, n, 0, 1);
    unsigned long long m = 0ull;
    for (int i = lane; i < n; i += 32) m = cand[i] > m ? cand[i] : m;
    const unsigned long long tau = __shfl_sync(0xffffffffu, warp_sort_desc(m), K - 1);
    int w = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const unsigned long long x = i < n ? cand[i] : 0ull;
        const bool keep = x != 0ull && x >= tau;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        // writes land below base + 32: never on keys not read yet
        if (keep) cand[w + __popc(bal & ((1u << lane) - 1u))] = x;
        w += __popc(bal);
        __syncwarp();
    }
    return warp_top32(cand, w, 0, 1);
}

// Top-K (K <= 32) of n candidate keys with the whole CTA: every warp reduces
// its share to a sorted top 32, warp 0 merges them.  Writes the chosen ids
// ascending to out (K entries, the unused ones -1); returns min(K, n).
// lists: shared scratch of 32 * (blockDim.x / 32) keys.
__device__ __forceinline__ int block_topk32(const unsigned long long *cand, int n, int K, int *out,
                                            unsigned long long *lists) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const unsigned long long mine = warp_top32(cand, n, warp, nw);
    lists[warp * 32 + lane] = mine;
    __syncthreads();
    if (warp == 0) {
        unsigned long long acc = lists[lane];
        for (int w = 1; w < nw; ++w) acc = warp_merge_desc(acc, lists[w * 32 + lane]);
        const bool take = lane < K && acc != 0ull;
        const int id = warp_sort_asc_int(take ? key_id(acc) : 0x7fffffff);
        if (lane < K) out[lane] = id == 0x7fffffff ? -1 : id;
    }
    __syncthreads();
    return min(K, n);
}

}  // namespace hga

namespace hga {

// fp64 dot product of q (shared, fp64) with one fp32 row by a quad of
// adjacent lanes (each a quarter of the row, all its loads in flight), the
// partial sums combined across the quad; every lane of the quad returns it.
template <int D>
__device__ __forceinline__ double quad_dot_row(const double *qr, const float *__restrict__ row) {
    constexpr int kPer = D / 16;                  // float4 loads per lane
    const int part = threadIdx.x & 3;
    const float4 *r4 = reinterpret_cast<const float4 *>(row) + part * kPer;
    const double2 *q2 = reinterpret_cast<const double2 *>(qr) + part * kPer * 2;
    float4 v[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) v[e] = __ldg(r4 + e);
    double s0 = 0.0, s1 = 0.0;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
        const double2 a = q2[2 * e], b = q2[2 * e + 1];
        s0 = fma(a.x, (double)v[e].x, s0);
        s1 = fma(a.y, (double)v[e].y, s1);
        s0 = fma(b.x, (double)v[e].z, s0);
        s1 = fma(b.y, (double)v[e].w, s1);
    }
    double s = s0 + s1;
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    return s;
}

// fp64 dot product of q (shared, fp64) with one fp32 row, by one thread
// (the whole row streams through this thread's 16-byte loads).
template <int D, bool kPlain = false, int kBatch = 8>
__device__ __forceinline__ double thread_dot_row(const double *qr, const float *__restrict__ row) {
    // kBatch 16-byte loads in flight per batch (8 by default: several rows per
    // thread and CTAs per SM cover the latency, within few registers).
    // kPlain: the row is in pinned host memory, read with plain loads (not
    // the read-only path)
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
    const double2 *q2 = reinterpret_cast<const double2 *>(qr);
    double s0 = 0.0, s1 = 0.0;
#pragma unroll
    for (int base = 0; base < D / 4; base += kBatch) {
        float4 v[kBatch];
#pragma unroll
        for (int e = 0; e < kBatch; ++e) {
            if constexpr (kPlain) {
                const float4 *p = r4 + base + e;
                asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(v[e].x), "=f"(v[e].y), "=f"(v[e].z), "=f"(v[e].w)
                             : "l"(p));
            } else {
                v[e] = __ldg(r4 + base + e);
            }
        }
#pragma unroll
        for (int e = 0; e < kBatch; ++e) {
            const double2 a = q2[2 * (base + e)], b = q2[2 * (base + e) + 1];
            s0 = fma(a.x, (double)v[e].x, s0);
            s1 = fma(a.y, (double)v[e].y, s1);
            s0 = fma(b.x, (double)v[e].z, s0);
            s1 = fma(b.y, (double)v[e].w, s1);
        }
    }
    return s0 + s1;
}

// Top-K (K <= 32) keys of n candidates with the whole CTA, written to out
// (global or shared) descending, padded with 0.
__device__ __forceinline__ void block_topk32_keys(const unsigned long long *cand, int n, int K,
                                                  unsigned long long *out,
                                                  unsigned long long *lists) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const unsigned long long mine = warp_top32(cand, n, warp, nw);
    lists[warp * 32 + lane] = mine;
    __syncthreads();
    if (warp == 0) {
        unsigned long long acc = lists[lane];
        for (int w = 1; w < nw; ++w) acc = warp_merge_desc(acc, lists[w * 32 + lane]);
        if (lane < K) out[lane] = acc;
    }
    __syncthreads();
}

}  // namespace hga

namespace hga {

// ---- selection by counting ranks (no dependent shuffle chains)

// The K largest of n distinct candidate keys (0 = padding, never chosen) by
// rank: a key is chosen when fewer than K keys exceed it.  top[0..K)
// (shared) receives them descending, 0-padded.  Whole CTA.
__device__ __forceinline__ void rank_topk(const unsigned long long *cand, int n, int K,
                                          unsigned long long *top) {
    for (int r = threadIdx.x; r < K; r += blockDim.x) top[r] = 0ull;
    __syncthreads();
    // four lanes per candidate, each counting a quarter of the others
    const int part = threadIdx.x & 3;
    for (int base = 0; base < n; base += (int)blockDim.x / 4) {
        const int i = base + (int)threadIdx.x / 4;
        const unsigned long long k = i < n ? cand[i] : 0ull;
        int r = 0;
        if (k) {
            int j = part;
            for (; j + 28 < n; j += 32) {      // eight loads in flight
                unsigned long long c[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) c[u] = cand[j + 4 * u];
#pragma unroll
                for (int u = 0; u < 8; ++u) r += c[u] > k;
            }
            for (; j < n; j += 4) r += cand[j] > k;
        }
        r += __shfl_xor_sync(0xffffffffu, r, 1);
        r += __shfl_xor_sync(0xffffffffu, r, 2);
        if (part == 0 && k && r < K) top[r] = k;
    }
    __syncthreads();
}

// The same over nl descending, 0-padded lists of len keys each (lists[b *
// len + p]): a key's rank is the number of keys above it in every list,
// found by binary search.  Whole CTA.
__device__ __forceinline__ void rank_topk_lists(const unsigned long long *lists, int nl, int len,
                                                int K, unsigned long long *top) {
    for (int r = threadIdx.x; r < K; r += blockDim.x) top[r] = 0ull;
    __syncthreads();
    for (int i = threadIdx.x; i < nl * len; i += blockDim.x) {
        const unsigned long long x = lists[i];
        if (!x) continue;
        int r = 0;
        for (int b = 0; b < nl; ++b) {
            const unsigned long long *Lb = lists + b * len;
            int lo = 0, hi = len;                 // first index whose key is not above x
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (Lb[mid] > x) lo = mid + 1;
                else hi = mid;
            }
            r += lo;
        }
        if (r < K) top[r] = x;
    }
    __syncthreads();
}

// Ids of top[0..K) (descending keys, 0-padded) in ascending order into
// out[0..K), the unused entries -1; returns how many were chosen.  Whole CTA.
__device__ __forceinline__ int ids_ascending(const unsigned long long *top, int K, int *out) {
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
        const unsigned long long k = top[i];
        if (!k) {
            out[i] = -1;
            continue;
        }
        const int id = key_id(k);
        int r = 0;
#pragma unroll 8
        for (int j = 0; j < K; ++j) {
            const unsigned long long kj = top[j];
            r += kj != 0ull && key_id(kj) < id;
        }
        out[r] = id;
    }
    __syncthreads();
    int n = 0;
    for (int i = 0; i < K; ++i) n += top[i] != 0ull;
    return n;
}

}  // namespace hga
