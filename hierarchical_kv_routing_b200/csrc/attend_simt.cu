// Stage 3 on CUDA cores: exact softmax attention over the routed token set,
// fp32 arithmetic (the fp32 path, and the fallback for shapes the tensor-core
// kernel does not take).
//
// Method: HGA paper-review page, section 3, exact token output attention with
// eq. (1): softmax(q_i . k_j / sqrt(D)) over the visible set only, exact, with
// no summary tokens, gates or calibration.
//
// Design: one CTA per (block, KV head, sequence, 64-row slice) where the
// block's 64*G query rows are ordered (token, head).  Four threads share a
// row, each holding a quarter of its rotate-half pairs in registers; key and
// value tiles of 32 gathered rows are staged in shared memory (padded so the
// four slices hit distinct banks); online softmax in base 2.
#include "hga_internal.cuh"
#include "vec.cuh"
#include "visible.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 64;   // query rows per CTA
constexpr int kTile = 32;   // keys per tile

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_attend_simt(const T *__restrict__ q, const int32_t *__restrict__ pos, int Tlen, int Hq, int Hkv,
              const T *__restrict__ k_rot, int k_T, const T *__restrict__ v, int v_T,
              const int32_t *__restrict__ sel_group, int NB, int F, int L, int K_g, int g_s,
              T *__restrict__ out, float *__restrict__ lse, Rope rope, float scale_log2) {
    constexpr int H = D / 2, PS = H / 4, SW = 2 * PS + 1;   // slice width + pad
    extern __shared__ __align__(16) unsigned char smem[];
    float *Kt = reinterpret_cast<float *>(smem);            // [kTile][4][SW]
    float *Vt = Kt + kTile * 4 * SW;                        // [kTile][4][SW]
    int *keys = reinterpret_cast<int *>(Vt + kTile * 4 * SW);
    __shared__ RunList rl;

    const int G = Hq / Hkv;
    const int n_rc = (kChunk * G + kRows - 1) / kRows;
    const int c = blockIdx.x / n_rc, rc = blockIdx.x % n_rc;
    const int h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk;
    const int n_cur = min(kChunk, Tlen - t0);

    if (threadIdx.x == 0)
        build_runs(rl, c, F, L, g_s, sel_group + (((int64_t)b * NB + c) * Hkv + h) * K_g, K_g,
                   n_cur);
    __syncthreads();
    fill_keys(rl, keys);
    const int nkeys = rl.off[rl.n];

    // this thread's row and slice
    const int r = threadIdx.x >> 2, sl = threadIdx.x & 3;
    const int R = rc * kRows + r;
    const int tok = t0 + R / G, hq = h * G + R % G;
    const bool valid = (R < kChunk * G) && (tok < Tlen);
    float qv[2 * PS], o[2 * PS];
#pragma unroll
    for (int e = 0; e < 2 * PS; ++e) qv[e] = o[e] = 0.f;
    if (valid) {
        const T *qrow = q + (((int64_t)b * Tlen + tok) * Hq + hq) * D;
        float lo[PS], hi[PS];
        load_slice<T, PS>(qrow + sl * PS, lo);
        load_slice<T, PS>(qrow + H + sl * PS, hi);
        const int32_t pp = pos[(int64_t)b * Tlen + tok];
#pragma unroll
        for (int p = 0; p < PS; ++p) {
            const float2 cs = rope_cs_int(rope, pp, sl * PS + p);
            qv[p] = (lo[p] * cs.x - hi[p] * cs.y) * scale_log2;
            qv[PS + p] = (hi[p] * cs.x + lo[p] * cs.y) * scale_log2;
        }
    }
    float m = -INFINITY, l = 0.f;
    __syncthreads();

    // loader mapping: key kk = tid / 8, part pp = tid % 8 (D/8 elements,
    // which lie inside one slice's low or high half)
    const int lk = threadIdx.x >> 3, lp = threadIdx.x & 7;
    const int l_sl = lp & 3, l_half = lp >> 2;
    for (int base = 0; base < nkeys; base += kTile) {
        if (base + lk < nkeys) {
            const int kt = keys[base + lk];
            const int64_t krow = ((int64_t)b * k_T + kt) * Hkv + h;
            const int64_t vrow = ((int64_t)b * v_T + kt) * Hkv + h;
            const int d0 = l_half * H + l_sl * PS;
            float a[PS], w[PS];
            load_slice<T, PS>(k_rot + krow * D + d0, a);
            load_slice<T, PS>(v + vrow * D + d0, w);
            float *kd = Kt + (lk * 4 + l_sl) * SW + l_half * PS;
            float *vd = Vt + (lk * 4 + l_sl) * SW + l_half * PS;
#pragma unroll
            for (int e = 0; e < PS; ++e) {
                kd[e] = a[e];
                vd[e] = w[e];
            }
        }
        __syncthreads();
        const int nk = min(kTile, nkeys - base);
        float s[kTile];
        float mt = -INFINITY;
#pragma unroll
        for (int kk = 0; kk < kTile; ++kk) {
            float acc = 0.f;
            const float *kr = Kt + (kk * 4 + sl) * SW;
#pragma unroll
            for (int e = 0; e < 2 * PS; ++e) acc = fmaf(qv[e], kr[e], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            const bool ok = kk < nk && keys[base + kk] <= tok;
            s[kk] = ok ? acc : -INFINITY;
            mt = fmaxf(mt, s[kk]);
        }
        if (valid && mt > -INFINITY) {
            const float mn = fmaxf(m, mt);
            const float corr = exp2f(m - mn);   // m = -inf on the first live tile: 0
            l *= corr;
#pragma unroll
            for (int e = 0; e < 2 * PS; ++e) o[e] *= corr;
#pragma unroll
            for (int kk = 0; kk < kTile; ++kk) {
                const float p = exp2f(s[kk] - mn);
                l += p;
                const float *vr = Vt + (kk * 4 + sl) * SW;
#pragma unroll
                for (int e = 0; e < 2 * PS; ++e) o[e] = fmaf(p, vr[e], o[e]);
            }
            m = mn;
        }
        __syncthreads();
    }
    if (valid) {
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < 2 * PS; ++e) o[e] *= inv;
        T *orow = out + (((int64_t)b * Tlen + tok) * Hq + hq) * D;
        float lo[PS], hi[PS];
#pragma unroll
        for (int p = 0; p < PS; ++p) {
            lo[p] = o[p];
            hi[p] = o[PS + p];
        }
        store_slice<T, PS>(orow + sl * PS, lo);
        store_slice<T, PS>(orow + H + sl * PS, hi);
        if (lse && sl == 0)
            lse[((int64_t)b * Hq + hq) * Tlen + tok] = (m + __log2f(l)) * 0.6931471805599453f;
    }
}

}  // namespace
size_t attend_simt_smem(const Geo &g);
namespace {

template <typename T, int D>
hga_status run(const Geo &g, const Rope &r, const void *q, const int32_t *pos, const void *k_rot,
               int k_T, const void *v, int v_T, const int32_t *sel_group, void *out, float *lse,
               cudaStream_t st) {
    const size_t smem = attend_simt_smem(g);
    if (smem > 200 * 1024) return HGA_ERR_UNSUPPORTED;
    auto kern = k_attend_simt<T, D>;
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    const int n_rc = (kChunk * g.G + kRows - 1) / kRows;
    dim3 grid(g.NB * n_rc, g.Hkv, g.B);
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    kern<<<grid, kThreads, smem, st>>>(static_cast<const T *>(q), pos, g.T, g.Hq, g.Hkv,
                                       static_cast<const T *>(k_rot), k_T,
                                       static_cast<const T *>(v), v_T, sel_group, g.NB, g.F, g.L,
                                       g.K_g, g.g_s, static_cast<T *>(out), lse, r, scale_log2);
    return cuda_status(cudaGetLastError());
}

}  // namespace

// Key list bound: the fixed windows, the routed tokens and the current chunk,
// and never more than T distinct tokens.
size_t attend_simt_smem(const Geo &g) {
    const long long max_keys =
        min((long long)(g.F + max(g.L, 1) + 1) * kChunk + (long long)g.K_g * g.g_s, (long long)g.T);
    return sizeof(float) * 2 * kTile * 4 * (g.D / 4 + 1) + sizeof(int) * (size_t)max_keys;
}

hga_status launch_attend_simt(const Geo &g, const Rope &r, int dtype, const void *q,
                              const int32_t *pos, const void *k_rot, int k_T, const void *v,
                              int v_T, const int32_t *sel_group, void *out, float *lse,
                              cudaStream_t st) {
    if (g.NB <= 0) return HGA_OK;
    if (dtype == HGA_BF16)
        return g.D == 128
            ? run<__nv_bfloat16, 128>(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st)
            : run<__nv_bfloat16, 64>(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st);
    return g.D == 128 ? run<float, 128>(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st)
                      : run<float, 64>(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st);
}

}  // namespace hga
