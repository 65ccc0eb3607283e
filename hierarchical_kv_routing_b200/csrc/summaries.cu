// Stage 1: rotate keys (K_rot = RoPE(K)) and build the mixed-RoPE chunk and
// group summaries of every closed chunk.
//
// Method: HGA paper-review page, section 3, "Mixed-RoPE Routing Summaries":
// for a token set G (a 64-token chunk or a g_s-token group) the summary's
// high-frequency pairs are the mean of the per-token rotated keys, and its
// low-frequency pairs are the mean raw key rotated at the set's mean position.
// Summaries are routing keys only; they never enter the attention output.
//
// Design (HBM-bound stream): one CTA per (chunk, sequence) handles all KV
// heads, so each (token, pair) angle is computed once into shared memory and
// reused Hkv times.  Each key row is read once with 16-byte vector loads and
// written once (K_rot); set sums are accumulated in fp64 from shared memory.
#include "hga_internal.cuh"
#include "vec.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;

// Shared memory: cos/sin per (token, pair) [64][D/2] float2, then the values
// to be averaged per (token, dim) [64][D] float (rotated on high pairs, raw on
// low pairs).
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_summaries(const T *__restrict__ k_raw, const T *__restrict__ v_raw,
            const int32_t *__restrict__ pos, int in_T, int Hkv, T *__restrict__ k_rot,
            T *__restrict__ v_out, int32_t *__restrict__ pos_out, int out_T,
            float *__restrict__ s_chunk, float *__restrict__ s_group, int nc_cap,
            T *__restrict__ k_open, int32_t *__restrict__ lens, int g_s, Rope rope) {
    constexpr int C = kChunk, H = D / 2, PS = H / 4;  // pairs per thread slice
    extern __shared__ __align__(16) unsigned char smem[];
    float2 *cs = reinterpret_cast<float2 *>(smem);                // [C][H]
    float *val = reinterpret_cast<float *>(smem + sizeof(float2) * C * H);  // [C][D]
    __shared__ double s_pmid[C + 1];

    const int m = blockIdx.x, b = blockIdx.y;
    const int t0 = m * C;
    const int n = min(C, in_T - t0);
    const bool closed = (n == C);
    const int gpc = C / g_s;
    const int32_t *pb = pos + (int64_t)b * in_T + t0;

    for (int e = threadIdx.x; e < C * H; e += kThreads) {
        const int j = e / H, i = e % H;
        if (j < n) cs[e] = rope_cs(rope, (double)pb[j], i);
    }
    if (pos_out)
        for (int j = threadIdx.x; j < n; j += kThreads) pos_out[(int64_t)b * out_T + t0 + j] = pb[j];
    if (lens && m == 0 && threadIdx.x == 0) lens[b] = in_T;
    // mean positions: chunk (index gpc) and groups (0..gpc-1)
    if (closed && threadIdx.x <= gpc) {
        const int g = threadIdx.x;
        const int lo = g < gpc ? g * g_s : 0, cnt = g < gpc ? g_s : C;
        double acc = 0.0;
        for (int j = 0; j < cnt; ++j) acc += (double)pb[lo + j];
        s_pmid[g] = acc / (double)cnt;
    }
    __syncthreads();

    const int j = threadIdx.x >> 2, sl = threadIdx.x & 3;
    for (int h = 0; h < Hkv; ++h) {
        if (j < n) {
            const int64_t in_row = ((int64_t)b * in_T + t0 + j) * Hkv + h;
            const int64_t out_row = ((int64_t)b * out_T + t0 + j) * Hkv + h;
            float lo[PS], hi[PS], rlo[PS], rhi[PS];
            load_slice<T, PS>(k_raw + in_row * D + sl * PS, lo);
            load_slice<T, PS>(k_raw + in_row * D + H + sl * PS, hi);
#pragma unroll
            for (int p = 0; p < PS; ++p) {
                const float2 c = cs[j * H + sl * PS + p];
                rlo[p] = lo[p] * c.x - hi[p] * c.y;
                rhi[p] = hi[p] * c.x + lo[p] * c.y;
            }
            if (k_rot) {
                store_slice<T, PS>(k_rot + out_row * D + sl * PS, rlo);
                store_slice<T, PS>(k_rot + out_row * D + H + sl * PS, rhi);
            }
            if (v_out) {
                float a[PS], c2[PS];
                load_slice<T, PS>(v_raw + in_row * D + sl * PS, a);
                load_slice<T, PS>(v_raw + in_row * D + H + sl * PS, c2);
                store_slice<T, PS>(v_out + out_row * D + sl * PS, a);
                store_slice<T, PS>(v_out + out_row * D + H + sl * PS, c2);
            }
            if (!closed && k_open) {
                T *ko = k_open + (((int64_t)b * Hkv + h) * C + j) * D;
                store_slice<T, PS>(ko + sl * PS, lo);
                store_slice<T, PS>(ko + H + sl * PS, hi);
            }
            if (closed) {
#pragma unroll
                for (int p = 0; p < PS; ++p) {
                    const int i = sl * PS + p;
                    const bool hf = is_high(rope, i);
                    val[j * D + i] = hf ? rlo[p] : lo[p];
                    val[j * D + i + H] = hf ? rhi[p] : hi[p];
                }
            }
        }
        __syncthreads();
        if (closed) {
            // one work item per (set, pair): sets 0..gpc-1 are groups, gpc the chunk
            for (int e = threadIdx.x; e < (gpc + 1) * H; e += kThreads) {
                const int set = e / H, i = e % H;
                const int lo = set < gpc ? set * g_s : 0, cnt = set < gpc ? g_s : C;
                double a = 0.0, c2 = 0.0;
                for (int jj = 0; jj < cnt; ++jj) {
                    a += (double)val[(lo + jj) * D + i];
                    c2 += (double)val[(lo + jj) * D + i + H];
                }
                a /= (double)cnt;
                c2 /= (double)cnt;
                float o0, o1;
                if (is_high(rope, i)) {
                    o0 = (float)a;
                    o1 = (float)c2;
                } else {
                    const float2 r = rope_cs(rope, s_pmid[set], i);
                    o0 = (float)(a * (double)r.x - c2 * (double)r.y);
                    o1 = (float)(c2 * (double)r.x + a * (double)r.y);
                }
                float *dst = set < gpc
                    ? s_group + ((((int64_t)b * Hkv + h) * nc_cap + m) * gpc + set) * D
                    : s_chunk + (((int64_t)b * Hkv + h) * nc_cap + m) * D;
                dst[i] = o0;
                dst[i + H] = o1;
            }
            __syncthreads();
        }
    }
}

template <typename T, int D>
hga_status run(const Geo &g, const Rope &r, const void *k_raw, const void *v_raw,
               const int32_t *pos, int in_T, void *k_rot, void *v_out, int32_t *pos_out,
               int out_T, float *s_chunk, float *s_group, int nc_cap, void *k_open,
               int32_t *lens, cudaStream_t st) {
    const size_t smem = sizeof(float2) * kChunk * (D / 2) + sizeof(float) * kChunk * D;
    auto kern = k_summaries<T, D>;
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 grid((in_T + kChunk - 1) / kChunk, g.B);
    kern<<<grid, kThreads, smem, st>>>(
        static_cast<const T *>(k_raw), static_cast<const T *>(v_raw), pos, in_T, g.Hkv,
        static_cast<T *>(k_rot), static_cast<T *>(v_out), pos_out, out_T, s_chunk, s_group,
        nc_cap, static_cast<T *>(k_open), lens, g.g_s, r);
    return cuda_status(cudaGetLastError());
}

}  // namespace

hga_status launch_summaries(const Geo &g, const Rope &r, int dtype, const void *k_raw,
                            const void *v_raw, const int32_t *pos, int in_T, void *k_rot,
                            void *v_out, int32_t *pos_out, int out_T, float *s_chunk,
                            float *s_group, int nc_cap, void *k_open, int32_t *lens,
                            cudaStream_t st) {
    if (in_T <= 0) return HGA_OK;
    if (dtype == HGA_BF16) {
        if (g.D == 128)
            return run<__nv_bfloat16, 128>(g, r, k_raw, v_raw, pos, in_T, k_rot, v_out, pos_out,
                                           out_T, s_chunk, s_group, nc_cap, k_open, lens, st);
        return run<__nv_bfloat16, 64>(g, r, k_raw, v_raw, pos, in_T, k_rot, v_out, pos_out, out_T,
                                      s_chunk, s_group, nc_cap, k_open, lens, st);
    }
    if (g.D == 128)
        return run<float, 128>(g, r, k_raw, v_raw, pos, in_T, k_rot, v_out, pos_out, out_T, s_chunk,
                               s_group, nc_cap, k_open, lens, st);
    return run<float, 64>(g, r, k_raw, v_raw, pos, in_T, k_rot, v_out, pos_out, out_T, s_chunk,
                          s_group, nc_cap, k_open, lens, st);
}

}  // namespace hga
