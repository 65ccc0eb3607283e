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
