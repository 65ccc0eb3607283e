// Stage 1: rotate keys (K_rot = RoPE(K)) and build the mixed-RoPE chunk and
// group summaries of every closed chunk.
//
// Method: HGA paper-review page, section 3, "Mixed-RoPE Routing Summaries":
// for a token set G (a 64-token chunk or a g_s-token group) the summary's
// high-frequency pairs are the mean of the per-token rotated keys, and its
// low-frequency pairs are the mean raw key rotated at the set's mean position.
// Summaries are routing keys only; they never enter the attention output.
//
// Design (HBM-bound stream): one CTA per (chunk, sequence).  The chunk's key
// rows (all KV heads, or a slab of heads when they do not fit) arrive in
// shared memory as one bulk copy while the CTA computes every (token, pair)
// angle once for all heads.  Then each thread owns one (head, pair): it walks
// the 64 tokens, rotates in place, and keeps the group and chunk sums in fp64
// registers, so no shared-memory reduction is needed; the rotated rows leave
// as one bulk store (K_rot).  Keys that live in pinned host memory (the
// host-resident tier) are read with plain loads instead of the bulk copy.
#include "hga_internal.cuh"
#include "sm100.cuh"

namespace hga {

__device__ int g_summaries_error = 0;
// Test hooks (hga_set_test_hooks): skip the keys' bulk copy, so the wait for
// it runs out, and the limit of that wait.
__device__ int g_summaries_skip_copy = 0;
__device__ unsigned long long g_summaries_wait_ns = sm100::kMaxWaitNs;

namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kSlabBytes = 64 * 1024;   // key rows of one head slab of one chunk

struct SumArgs {
    const void *k_raw, *v_raw;
    const int32_t *pos;
    int in_T, Hkv, HS;          // HS: heads per slab
    void *k_rot, *v_out;
    int32_t *pos_out;
    int out_T;
    float *s_chunk, *s_group;
    int nc_cap;
    void *k_open;
    int32_t *lens;
    int g_s;
    Rope rope;
};

// Plain 16-byte load (no read-only path; used for pinned host memory).
__device__ __forceinline__ uint4 ld16_plain(const void *p) {
    uint4 w;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                 : "l"(p));
    return w;
}

// Summary of one set for pair i from its fp64 sums: high pairs are the mean
// of the rotated keys; low pairs the mean raw key rotated at the set's mean
// position.
__device__ __forceinline__ void write_summary(const Rope &rope, bool hf, int i, int H, double sx,
                                              double sy, int cnt, double pmid, float *dst) {
    const double a = sx / (double)cnt, c2 = sy / (double)cnt;
    float o0, o1;
    if (hf) {
        o0 = (float)a;
        o1 = (float)c2;
    } else {
        const float2 r = rope_cs(rope, pmid, i);
        o0 = (float)(a * (double)r.x - c2 * (double)r.y);
        o1 = (float)(c2 * (double)r.x + a * (double)r.y);
    }
    dst[i] = o0;
    dst[i + H] = o1;
}

template <typename T, int D, bool kHost>
__global__ void __launch_bounds__(kThreads, 2) k_summaries(const SumArgs A) {
    constexpr int C = kChunk, H = D / 2;
    extern __shared__ __align__(128) unsigned char smem[];
    T *kb = reinterpret_cast<T *>(smem);                          // [n][nh][D]
    float2 *cs = reinterpret_cast<float2 *>(smem + kSlabBytes);   // [n][H]
    __shared__ double s_pmid[C + 1];
    __shared__ int32_t s_pos[C];
    __shared__ __align__(8) uint64_t bar;

    const int m = blockIdx.x, b = blockIdx.y;
    const int t0 = m * C;
    const int n = min(C, A.in_T - t0);
    const bool closed = n == C;
    const int gpc = C / A.g_s;
    const int32_t *pb = A.pos + (int64_t)b * A.in_T + t0;
    const T *kin = static_cast<const T *>(A.k_raw);

    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    // the chunk's positions, one coalesced load
    if (threadIdx.x < n) s_pos[threadIdx.x] = pb[threadIdx.x];
    __syncthreads();
    // a kernel launched after this one as a programmatic dependent (stage 2)
    // may start now: it reads what this kernel writes only after its
    // griddepcontrol.wait
    asm volatile("griddepcontrol.launch_dependents;");

    int pass = 0;
    for (int hs0 = 0; hs0 < A.Hkv; hs0 += A.HS, ++pass) {
        const int nh = min(A.HS, A.Hkv - hs0);
        const uint32_t row_bytes = (uint32_t)(nh * D * sizeof(T));
        const T *src0 = kin + (((int64_t)b * A.in_T + t0) * A.Hkv + hs0) * D;
        if constexpr (!kHost) {
            if (threadIdx.x == 0) {
                mbar_arrive_expect_tx(&bar, row_bytes * n);
                if (g_summaries_skip_copy) {
                    // test hook: the copy is not issued and the wait below runs out
                } else if (nh == A.Hkv) {
                    bulk_load(kb, src0, row_bytes * n, &bar);       // contiguous rows
                } else {
                    for (int j = 0; j < n; ++j)
                        bulk_load(kb + (size_t)j * nh * D, src0 + (int64_t)j * A.Hkv * D, row_bytes,
                                  &bar);
                }
            }
        } else {
            // eight independent loads in flight per thread (the link's latency
            // is microseconds), then the shared-memory stores
            const int wpr = (int)(row_bytes / 16), nw = n * wpr;
            for (int base = 0; base < nw; base += 8 * kThreads) {
                uint4 w[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int idx = base + u * kThreads + threadIdx.x;
                    if (idx < nw)
                        w[u] = ld16_plain(reinterpret_cast<const uint4 *>(
                                              src0 + (int64_t)(idx / wpr) * A.Hkv * D) + idx % wpr);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int idx = base + u * kThreads + threadIdx.x;
                    if (idx < nw) reinterpret_cast<uint4 *>(kb)[idx] = w[u];
                }
            }
        }
        if (pass == 0) {
            // while the keys are in flight: angles, mean positions, copies
            for (int e = threadIdx.x; e < n * H; e += kThreads)
                cs[e] = rope_cs_int(A.rope, s_pos[e / H], e % H);
            if (closed && threadIdx.x < 32) {
                // mean positions: lane l holds positions l and l + 32 (64-bit
                // sums are exact); each set is a run of lanes
                const int l = threadIdx.x;
                const long long p0 = s_pos[l], p1 = s_pos[l + 32];
                long long tot = p0 + p1;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
                if (l == 0) s_pmid[gpc] = (double)tot / (double)C;
                for (int g = 0; g < gpc; ++g) {
                    const int lo = g * A.g_s;
                    long long part = 0;
                    for (int j = l; j < A.g_s; j += 32) part += s_pos[lo + j];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                    if (l == 0) s_pmid[g] = (double)part / (double)A.g_s;
                }
            }
            if (A.pos_out)
                for (int j = threadIdx.x; j < n; j += kThreads)
                    A.pos_out[(int64_t)b * A.out_T + t0 + j] = s_pos[j];
            if (A.lens && m == 0 && threadIdx.x == 0) A.lens[b] = A.in_T;
            if (A.v_out) {
                const int wpr = A.Hkv * D * (int)sizeof(T) / 16;
                const uint4 *vs = reinterpret_cast<const uint4 *>(
                    static_cast<const T *>(A.v_raw) + ((int64_t)b * A.in_T + t0) * A.Hkv * D);
                uint4 *vd = reinterpret_cast<uint4 *>(
                    static_cast<T *>(A.v_out) + ((int64_t)b * A.out_T + t0) * A.Hkv * D);
                for (int w = threadIdx.x; w < n * wpr; w += kThreads) vd[w] = __ldg(vs + w);
            }
        }
        __syncthreads();
        if constexpr (!kHost) {
            if (!mbar_wait(&bar, pass & 1, g_summaries_wait_ns)) {
                if (threadIdx.x == 0) atomicExch(&g_summaries_error, (int)HGA_ERR_TIMEOUT);
                return;
            }
        }

        // one (head, pair) per thread: rotate in place, fp64 set sums with
        // four independent accumulators (tokens j, j+1, j+2, j+3 in flight)
        for (int e = threadIdx.x; e < nh * H; e += kThreads) {
            const int hh = e / H, i = e % H;
            const int h = hs0 + hh;
            const bool hf = is_high(A.rope, i);
            T *col = kb + (size_t)hh * D + i;          // token j at col + j * js
            const size_t js = (size_t)nh * D;
            if (!closed) {
                T *ko = A.k_open ? static_cast<T *>(A.k_open) + ((int64_t)b * A.Hkv + h) * C * D
                                 : nullptr;
                for (int j = 0; j < n; ++j) {
                    T *px = col + j * js;
                    const T x0 = px[0], y0 = px[H];
                    const float2 rr = rot_pair(to_f(x0), to_f(y0), cs[j * H + i]);
                    if (ko) {
                        ko[(int64_t)j * D + i] = x0;
                        ko[(int64_t)j * D + i + H] = y0;
                    }
                    px[0] = from_f<T>(rr.x);
                    px[H] = from_f<T>(rr.y);
                }
                continue;
            }
            float *sg = A.s_group + (((int64_t)b * A.Hkv + h) * A.nc_cap + m) * gpc * D;
            double cx = 0.0, cy = 0.0;
            for (int set = 0; set < gpc; ++set) {
                double ax[4] = {0.0, 0.0, 0.0, 0.0}, ay[4] = {0.0, 0.0, 0.0, 0.0};
                const int j0 = set * A.g_s;
                int jj = 0;
                for (; jj + 4 <= A.g_s; jj += 4) {
                    float x[4], y[4];
                    float2 c4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const T *px = col + (j0 + jj + u) * js;
                        x[u] = to_f(px[0]);
                        y[u] = to_f(px[H]);
                        c4[u] = cs[(j0 + jj + u) * H + i];
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 rr = rot_pair(x[u], y[u], c4[u]);
                        T *px = col + (j0 + jj + u) * js;
                        px[0] = from_f<T>(rr.x);
                        px[H] = from_f<T>(rr.y);
                        ax[u] += (double)(hf ? rr.x : x[u]);
                        ay[u] += (double)(hf ? rr.y : y[u]);
                    }
                }
                for (; jj < A.g_s; ++jj) {
                    T *px = col + (j0 + jj) * js;
                    const float x = to_f(px[0]), y = to_f(px[H]);
                    const float2 rr = rot_pair(x, y, cs[(j0 + jj) * H + i]);
                    px[0] = from_f<T>(rr.x);
                    px[H] = from_f<T>(rr.y);
                    ax[0] += (double)(hf ? rr.x : x);
                    ay[0] += (double)(hf ? rr.y : y);
                }
                const double gx = (ax[0] + ax[1]) + (ax[2] + ax[3]);
                const double gy = (ay[0] + ay[1]) + (ay[2] + ay[3]);
                write_summary(A.rope, hf, i, H, gx, gy, A.g_s, s_pmid[set], sg + (int64_t)set * D);
                cx += gx;
                cy += gy;
            }
            write_summary(A.rope, hf, i, H, cx, cy, C, s_pmid[gpc],
                          A.s_chunk + (((int64_t)b * A.Hkv + h) * A.nc_cap + m) * D);
        }
        // rotated rows out
        if (A.k_rot) {
            fence_proxy_async_smem();
            __syncthreads();
            if (threadIdx.x == 0) {
                T *dst0 = static_cast<T *>(A.k_rot) + (((int64_t)b * A.out_T + t0) * A.Hkv + hs0) * D;
                if (nh == A.Hkv) {
                    bulk_store(dst0, kb, row_bytes * n);
                } else {
                    for (int j = 0; j < n; ++j)
                        bulk_store(dst0 + (int64_t)j * A.Hkv * D, kb + (size_t)j * nh * D, row_bytes);
                }
                bulk_commit();
                bulk_wait_read();
            }
        }
        __syncthreads();
    }
}

template <typename T, int D, bool kHost>
hga_status run(const Geo &g, const SumArgs &a, int in_T, cudaStream_t st) {
    const size_t smem = kSlabBytes + sizeof(float2) * kChunk * (D / 2);
    auto kern = k_summaries<T, D, kHost>;
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 grid((in_T + kChunk - 1) / kChunk, g.B);
    kern<<<grid, kThreads, smem, st>>>(a);
    return cuda_status(cudaGetLastError());
}

}  // namespace

hga_status launch_summaries(const Geo &g, const Rope &r, int dtype, const void *k_raw,
                            const void *v_raw, const int32_t *pos, int in_T, void *k_rot,
                            void *v_out, int32_t *pos_out, int out_T, float *s_chunk,
                            float *s_group, int nc_cap, void *k_open, int32_t *lens,
                            cudaStream_t st, bool host_src) {
    if (in_T <= 0) return HGA_OK;
    const size_t es = dtype == HGA_BF16 ? 2 : 4;
    SumArgs a;
    a.k_raw = k_raw;
    a.v_raw = v_raw;
    a.pos = pos;
    a.in_T = in_T;
    a.Hkv = g.Hkv;
    const int fit = (int)(kSlabBytes / (kChunk * g.D * es));
    a.HS = fit < 1 ? 1 : (fit < g.Hkv ? fit : g.Hkv);
    a.k_rot = k_rot;
    a.v_out = v_out;
    a.pos_out = pos_out;
    a.out_T = out_T;
    a.s_chunk = s_chunk;
    a.s_group = s_group;
    a.nc_cap = nc_cap;
    a.k_open = k_open;
    a.lens = lens;
    a.g_s = g.g_s;
    a.rope = r;
    if (host_src) {
        // the host-resident tier: bf16 keys only, no copies to the device
        if (dtype != HGA_BF16 || v_raw || v_out || k_open) return HGA_ERR_UNSUPPORTED;
        return g.D == 128 ? run<__nv_bfloat16, 128, true>(g, a, in_T, st)
                          : run<__nv_bfloat16, 64, true>(g, a, in_T, st);
    }
    if (dtype == HGA_BF16)
        return g.D == 128 ? run<__nv_bfloat16, 128, false>(g, a, in_T, st)
                          : run<__nv_bfloat16, 64, false>(g, a, in_T, st);
    return g.D == 128 ? run<float, 128, false>(g, a, in_T, st) : run<float, 64, false>(g, a, in_T, st);
}


// Reads this file's device error word on `st` (after the work queued on it)
// and optionally resets it; returns the recorded status (HGA_OK if none).
hga_status summaries_test_hooks(int skip_copy, unsigned long long wait_ns, cudaStream_t st) {
    const unsigned long long ns = wait_ns ? wait_ns : sm100::kMaxWaitNs;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_summaries_skip_copy, &skip_copy, sizeof(int), 0,
                                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_summaries_wait_ns, &ns, sizeof(ns), 0,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e);
}

hga_status summaries_error_take(cudaStream_t st, bool clear) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_summaries_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_summaries_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    return (hga_status)v;
}

}  // namespace hga
