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
// Design: one CTA per (block, KV head, sequence), HBM-bound on the Q stream.
// Each thread sums its token's G query heads on a quarter of the pairs with
// 16-byte loads (RoPE is linear, so heads are summed before rotating), the
// rotated rows meet in shared memory and 128 threads reduce them over the
// block's tokens in fp64.  Scores are fp64 dot products, one summary row per
// thread (its 16-byte loads all in flight), ranked as packed (fp32 score, id)
// keys; the top-K runs in registers (warp bitonic sort and merge) for K <= 32
// and by CTA-wide rounds above that.
#include "hga_internal.cuh"
#include "route_common.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_route(const T *__restrict__ q, const int32_t *__restrict__ pos, int Tlen, int Hq, int Hkv,
        const float *__restrict__ s_chunk, const float *__restrict__ s_group, int nc_cap,
        int F, int L, int K_c, int K_g, int gpc, int ncand, int32_t *__restrict__ sel_chunk,
        int32_t *__restrict__ sel_group, Rope rope) {
    constexpr int H = D / 2, PS = H / 4;
    extern __shared__ __align__(16) unsigned char smem[];
    float *rot = reinterpret_cast<float *>(smem);                              // [64][D]
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(rot + kChunk * D);
    __shared__ __align__(16) double qr[D];
    __shared__ unsigned long long lists[kThreads];
    __shared__ RouteScratch rs;

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int NB = gridDim.x;
    const int G = Hq / Hkv;
    const int t0 = c * kChunk;
    const int n = min(kChunk, Tlen - t0);

    // ---- routing query: sum_i sum_{h'} R_{p_i}(q_{i,h'})
    {
        const int j = threadIdx.x >> 2, sl = threadIdx.x & 3;
        float lo[PS], hi[PS];
#pragma unroll
        for (int p = 0; p < PS; ++p) lo[p] = hi[p] = 0.f;
        if (j < n) {
            const T *row = q + (((int64_t)b * Tlen + t0 + j) * Hq + (int64_t)h * G) * D;
            // several heads' rows in flight at a time, kept packed until summed
            constexpr int kVec = PS * (int)sizeof(T) / 16;        // 16-byte words per half
            constexpr int kBatch = sizeof(T) == 2 ? 4 : 2;
            for (int h0 = 0; h0 < G; h0 += kBatch) {
                uint4 wa[kBatch][kVec], wb[kBatch][kVec];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    if (h0 + u < G) {
                        const uint4 *pa = reinterpret_cast<const uint4 *>(row + (h0 + u) * D + sl * PS);
                        const uint4 *pb = reinterpret_cast<const uint4 *>(row + (h0 + u) * D + H + sl * PS);
#pragma unroll
                        for (int v = 0; v < kVec; ++v) {
                            wa[u][v] = __ldg(pa + v);
                            wb[u][v] = __ldg(pb + v);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    if (h0 + u < G) {
                        float a[PS], d2[PS];
                        unpack_words<T, PS>(wa[u], a);
                        unpack_words<T, PS>(wb[u], d2);
#pragma unroll
                        for (int p = 0; p < PS; ++p) {
                            lo[p] += a[p];
                            hi[p] += d2[p];
                        }
                    }
                }
            }
            const int32_t pj = pos[(int64_t)b * Tlen + t0 + j];
#pragma unroll
            for (int p = 0; p < PS; ++p) {
                const float2 r = rope_cs_int(rope, pj, sl * PS + p);
                const float x = lo[p], y = hi[p];
                lo[p] = x * r.x - y * r.y;
                hi[p] = y * r.x + x * r.y;
            }
        }
#pragma unroll
        for (int p = 0; p < PS; ++p) {
            rot[j * D + sl * PS + p] = lo[p];
            rot[j * D + H + sl * PS + p] = hi[p];
        }
        __syncthreads();
        if (threadIdx.x < D) {
            double s = 0.0;
            for (int jj = 0; jj < n; ++jj) s += (double)rot[jj * D + threadIdx.x];
            qr[threadIdx.x] = s;
        }
        __syncthreads();
    }

    // ---- chunk level: middle chunks F..hi, top K_c
    const int hi_m = middle_hi(c, L);
    const int n_mid = max(0, hi_m - F + 1);
    const float *Sc = s_chunk + ((int64_t)b * Hkv + h) * nc_cap * D;
    for (int r = threadIdx.x; r < n_mid; r += kThreads)
        cand[r] = pack_key((float)thread_dot_row<D>(qr, Sc + (int64_t)(F + r) * D), F + r);
    __syncthreads();
    const int kc = min(K_c, n_mid);
    if (K_c <= 32) block_topk32(cand, n_mid, K_c, rs.sel_c, lists);
    else topk_select(cand, n_mid, K_c, rs.sel_c, rs);
    int32_t *out_c = sel_chunk + (((int64_t)b * NB + c) * Hkv + h) * K_c;
    for (int r = threadIdx.x; r < K_c; r += kThreads) out_c[r] = r < kc ? rs.sel_c[r] : -1;

    // ---- group level: the groups of the selected chunks, top K_g
    const float *Sg = s_group + ((int64_t)b * Hkv + h) * nc_cap * gpc * D;
    const int n_g = kc * gpc;
    __syncthreads();
    for (int r = threadIdx.x; r < n_g; r += kThreads) {
        const int gid = rs.sel_c[r / gpc] * gpc + r % gpc;
        cand[r] = pack_key((float)thread_dot_row<D>(qr, Sg + (int64_t)gid * D), gid);
    }
    __syncthreads();
    const int kg = min(K_g, n_g);
    if (K_g <= 32) block_topk32(cand, n_g, K_g, rs.sel_g, lists);
    else topk_select(cand, n_g, K_g, rs.sel_g, rs);
    int32_t *out_g = sel_group + (((int64_t)b * NB + c) * Hkv + h) * K_g;
    for (int r = threadIdx.x; r < K_g; r += kThreads) out_g[r] = r < kg ? rs.sel_g[r] : -1;
}

template <typename T, int D>
hga_status run(const Geo &g, const Rope &r, const void *q, const int32_t *pos,
               const float *s_chunk, const float *s_group, int nc_cap, int32_t *sel_chunk,
               int32_t *sel_group, cudaStream_t st) {
    const long long ncand = max(max((long long)g.NC, 1ll), (long long)min(g.K_c, g.NC) * g.gpc);
    const size_t smem = sizeof(float) * kChunk * D + sizeof(unsigned long long) * (size_t)ncand;
    if (smem > 180 * 1024) return HGA_ERR_UNSUPPORTED;   // candidate table must fit on chip
    auto kern = k_route<T, D>;
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 grid(g.NB, g.Hkv, g.B);
    kern<<<grid, kThreads, smem, st>>>(static_cast<const T *>(q), pos, g.T, g.Hq, g.Hkv, s_chunk,
                                       s_group, nc_cap, g.F, g.L, g.K_c, g.K_g, g.gpc,
                                       (int)ncand, sel_chunk, sel_group, r);
    return cuda_status(cudaGetLastError());
}

}  // namespace

hga_status launch_route(const Geo &g, const Rope &r, int dtype, const void *q, const int32_t *pos,
                        const float *s_chunk, const float *s_group, int nc_cap,
                        int32_t *sel_chunk, int32_t *sel_group, cudaStream_t st) {
    if (g.NB <= 0) return HGA_OK;
    if (dtype == HGA_BF16)
        return g.D == 128 ? run<__nv_bfloat16, 128>(g, r, q, pos, s_chunk, s_group, nc_cap,
                                                     sel_chunk, sel_group, st)
                          : run<__nv_bfloat16, 64>(g, r, q, pos, s_chunk, s_group, nc_cap,
                                                    sel_chunk, sel_group, st);
    return g.D == 128 ? run<float, 128>(g, r, q, pos, s_chunk, s_group, nc_cap, sel_chunk,
                                        sel_group, st)
                      : run<float, 64>(g, r, q, pos, s_chunk, s_group, nc_cap, sel_chunk,
                                       sel_group, st);
}

}  // namespace hga
