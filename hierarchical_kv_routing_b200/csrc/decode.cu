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
// Three kernels per step, all HBM-bound.  The visible set splits into a part
// routing does not touch (sinks, recent chunks, the current chunk) and the
// routed groups, so the fixed part is attended on a second stream while the
// step routes, and only the routed groups wait for the routing.
//   k_decode_a  grid (scan splits, KV heads, sequences): split 0 appends the
//               token (rotated key, value, position, raw key of the open
//               chunk) and, when the token closes its chunk, writes that
//               chunk's summaries.  Each CTA scores its 256 middle chunks, one
//               summary row per thread (fp64 dot products), and keeps its top
//               K_c keys; the last one to finish (atomic counter) merges them,
//               scores the groups of the chosen chunks and keeps the top K_g.
//   k_decode_fixed  grid (nF, KV heads, sequences), on a second stream forked
//               before and joined after the step, beside k_decode_a: attends
//               the KV head's G query heads over a slice of the fixed keys
//               (the new token's key and value straight from the step's
//               inputs, everything else from the cache) and writes partial
//               softmax sums.
//   k_decode_b  grid (nR, KV heads, sequences), launched as a programmatic
//               dependent of k_decode_a: it rotates the queries, then waits
//               for k_decode_a and attends over a slice of the routed groups.
// A slice holds at most slice_keys keys (128 for bf16, D = 128): their key
// and value rows are staged in shared memory, and Q.K runs register-blocked
// (each query slice read from shared memory serves four keys).
// The last of the nF + nR slice CTAs (fixed or routed) of a (sequence, KV head)
// combines all partials; the last of those per sequence increments lens.
// Counters live in the workspace; each last CTA resets its counter, so the
// workspace only has to be zeroed before its first use.
#include <mutex>

#include "hga_internal.cuh"
#include "route_common.cuh"
#include "vec.cuh"

namespace hga {

__device__ int g_decode_error = 0;

namespace {

constexpr int kThreads = 256;
constexpr int kScanChunks = 256;  // middle chunks per scan CTA (one per thread)
// Keys per attention slice CTA: its key and value rows (32 KB each) are
// staged in shared memory, which keeps two slice CTAs per SM.
template <typename T, int D>
constexpr int slice_keys() {
    return (32 * 1024) / (D * (int)sizeof(T)) < kThreads ? (32 * 1024) / (D * (int)sizeof(T))
                                                          : kThreads;
}
constexpr int kMinSliceKeys = 64;     // the smallest slice_keys of any type and size
constexpr int kMaxG = 16;
constexpr int kMaxCand = 1024;    // merge and group candidate table

struct DecodeArgs {
    int B, Tc, Hq, Hkv, G, C, g_s, gpc, F, L, K_c, K_g, nc_cap, ns_scan;
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
    float *part;                     // [B, Hq, nparts, D + 2]
    int nF, nR, nparts;              // fixed and routed slice CTAs per (sequence, KV head)
    int32_t *scan_done, *att_done, *seq_done;
    float scale_log2;
    Rope rope;
};

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
            const float x = to_f(ko[(int64_t)j * D + i]), y = to_f(ko[(int64_t)j * D + i + H]);
            if (hf) {
                const float2 r = rope_cs_int(A.rope, pj, i);
                const float2 rr = rot_pair(x, y, r);
                a += (double)rr.x;
                d2 += (double)rr.y;
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

// Rotated, pre-scaled queries of the KV head's G heads -> qs[G][D].
template <typename T, int D>
__device__ __forceinline__ void load_queries(const DecodeArgs &A, int b, int h, int32_t pnew,
                                             float *qs) {
    constexpr int H = D / 2;
    const T *qb = static_cast<const T *>(A.q_new) + ((int64_t)b * A.Hq + (int64_t)h * A.G) * D;
    for (int e = threadIdx.x; e < A.G * H; e += blockDim.x) {
        const int g = e / H, i = e % H;
        const float2 r = rope_cs_int(A.rope, pnew, i);
        const float x = to_f(qb[g * D + i]), y = to_f(qb[g * D + i + H]);
        qs[g * D + i] = (x * r.x - y * r.y) * A.scale_log2;
        qs[g * D + i + H] = (y * r.x + x * r.y) * A.scale_log2;
    }
}

// The step's new key, rotated and rounded to the cache's type exactly like
// the appended row, into knew[D] (shared, cache type), by D/2 threads.
template <typename T, int D>
__device__ __forceinline__ void rotate_new_key(const DecodeArgs &A, int b, int h, int32_t pnew,
                                               T *knew) {
    constexpr int H = D / 2;
    if (threadIdx.x < H) {
        const int i = threadIdx.x;
        const T *kn = static_cast<const T *>(A.k_new) + ((int64_t)b * A.Hkv + h) * D;
        const float x = to_f(kn[i]), y = to_f(kn[i + H]);
        const float2 r = rope_cs_int(A.rope, pnew, i);
        const float2 rr = rot_pair(x, y, r);
        knew[i] = from_f<T>(rr.x);
        knew[i + H] = from_f<T>(rr.y);
    }
}

// q . k for one packed 16-byte slice of k (8 bf16 or 4 fp32 values).
template <typename T>
__device__ __forceinline__ float dot16(const uint4 &w, const float *q) {
    if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
        const float4 qa = *reinterpret_cast<const float4 *>(q);
        const float4 qb = *reinterpret_cast<const float4 *>(q + 4);
        const float2 a = __bfloat1622float2(h2[0]), b = __bfloat1622float2(h2[1]);
        const float2 c = __bfloat1622float2(h2[2]), d = __bfloat1622float2(h2[3]);
        float s = qa.x * a.x;
        s = fmaf(qa.y, a.y, s);
        s = fmaf(qa.z, b.x, s);
        s = fmaf(qa.w, b.y, s);
        s = fmaf(qb.x, c.x, s);
        s = fmaf(qb.y, c.y, s);
        s = fmaf(qb.z, d.x, s);
        return fmaf(qb.w, d.y, s);
    } else {
        const float4 qa = *reinterpret_cast<const float4 *>(q);
        float s = qa.x * __uint_as_float(w.x);
        s = fmaf(qa.y, __uint_as_float(w.y), s);
        s = fmaf(qa.z, __uint_as_float(w.z), s);
        return fmaf(qa.w, __uint_as_float(w.w), s);
    }
}

// DL consecutive elements (shared memory) as one packed load.
template <typename T, int DL>
__device__ __forceinline__ void load_lane_slice(const T *p, float (&x)[DL]) {
    if constexpr (sizeof(T) == 2 && DL == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.x));
        const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.y));
        x[0] = a.x;
        x[1] = a.y;
        x[2] = c.x;
        x[3] = c.y;
    } else if constexpr (sizeof(T) == 2 && DL == 2) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
        x[0] = a.x;
        x[1] = a.y;
    } else if constexpr (sizeof(T) == 4 && DL == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        x[0] = a.x;
        x[1] = a.y;
        x[2] = a.z;
        x[3] = a.w;
    } else {
#pragma unroll
        for (int e = 0; e < DL; ++e) x[e] = to_f(p[e]);
    }
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}

// Partial attention of the G heads over keys key_of(0..nk), nk <=
// slice_keys.  The key and value rows are staged in shared memory with
// cp.async (the token's own key from knew, its value from the step's
// inputs).  Q.K: lane s of a key group holds 16-byte slice s of 4 keys and
// scores them for 8 heads at a time (each q slice read from shared memory
// serves 4 keys); the group's lanes reduce-scatter the 32 partial sums.
// Softmax and P.V then run one warp per head with lanes over dims.  Writes
// (m, l, o[D]) for part index `pi`.
template <typename T, int D, typename KeyOf>
__device__ void attend_part(const DecodeArgs &A, int b, int h, int t, int nk, KeyOf key_of,
                            int pi, const float *qs, const T *knew, float *sc, int *kt_s, T *Ks,
                            T *Vs) {
    constexpr int DL = D / 32;
    constexpr int NV = D * (int)sizeof(T) / 16;     // 16-byte slices per row
    constexpr int EV = 16 / (int)sizeof(T);         // elements per slice
    constexpr int KPG = 4;                          // keys per Q.K lane
    constexpr int NVAL = KPG * 8;                   // partial sums per lane
    constexpr int R = NVAL / NV;                    // sums per lane after the reduce
    constexpr int KPP = KPG * kThreads / NV;        // keys per Q.K pass
    static_assert(32 % NV == 0 && NVAL % NV == 0, "Q.K lane groups");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int k = threadIdx.x; k < nk; k += blockDim.x) kt_s[k] = key_of(k);
    __syncthreads();
    const T *kbase = static_cast<const T *>(A.k_rot);
    const T *vbase = static_cast<const T *>(A.v);
    const T *vn = static_cast<const T *>(A.v_new) + ((int64_t)b * A.Hkv + h) * D;
    for (int idx = threadIdx.x; idx < nk * NV; idx += blockDim.x) {
        const int k = idx / NV, pv = idx % NV;
        const int kv = kt_s[k];
        const int64_t row = (((int64_t)b * A.Tc + kv) * A.Hkv + h) * D;
        uint4 *kd = reinterpret_cast<uint4 *>(Ks + (size_t)k * D) + pv;
        if (kv == t) *kd = reinterpret_cast<const uint4 *>(knew)[pv];
        else cp_async16(kd, reinterpret_cast<const uint4 *>(kbase + row) + pv);
        cp_async16(reinterpret_cast<uint4 *>(Vs + (size_t)k * D) + pv,
                   reinterpret_cast<const uint4 *>(kv == t ? vn : vbase + row) + pv);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    {
        const int sl = threadIdx.x % NV, kgp = threadIdx.x / NV;
        for (int k0 = 0; k0 < nk; k0 += KPP) {
            float kx[KPG][EV];
#pragma unroll
            for (int j = 0; j < KPG; ++j) {
                const int key = k0 + kgp * KPG + j;
                uint4 w = make_uint4(0u, 0u, 0u, 0u);
                if (key < nk) w = reinterpret_cast<const uint4 *>(Ks + (size_t)key * D)[sl];
                if constexpr (sizeof(T) == 2) {
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
                    for (int z = 0; z < 4; ++z) {
                        const float2 f = __bfloat1622float2(h2[z]);
                        kx[j][2 * z] = f.x;
                        kx[j][2 * z + 1] = f.y;
                    }
                } else {
                    kx[j][0] = __uint_as_float(w.x);
                    kx[j][1] = __uint_as_float(w.y);
                    kx[j][2] = __uint_as_float(w.z);
                    kx[j][3] = __uint_as_float(w.w);
                }
            }
            for (int g0 = 0; g0 < A.G; g0 += 8) {
                float v[NVAL];
#pragma unroll
                for (int x = 0; x < NVAL; ++x) v[x] = 0.f;
#pragma unroll
                for (int hh = 0; hh < 8; ++hh) {
                    if (g0 + hh < A.G) {
                        const float4 *q4 = reinterpret_cast<const float4 *>(qs + (g0 + hh) * D + sl * EV);
#pragma unroll
                        for (int z = 0; z < EV / 4; ++z) {
                            const float4 qv = q4[z];
#pragma unroll
                            for (int j = 0; j < KPG; ++j) {
                                float a = v[j * 8 + hh];
                                a = fmaf(qv.x, kx[j][4 * z], a);
                                a = fmaf(qv.y, kx[j][4 * z + 1], a);
                                a = fmaf(qv.z, kx[j][4 * z + 2], a);
                                a = fmaf(qv.w, kx[j][4 * z + 3], a);
                                v[j * 8 + hh] = a;
                            }
                        }
                    }
                }
                // reduce-scatter over the group's lanes: lane s keeps sums
                // [s R, s R + R) of the group's 4 keys x 8 heads
#pragma unroll
                for (int st = NV / 2, n = NVAL; st >= 1; st >>= 1, n >>= 1) {
                    const bool up = (lane & st) != 0;
#pragma unroll
                    for (int x = 0; x < n / 2; ++x) {
                        const float send = up ? v[x] : v[x + n / 2];
                        const float keep = up ? v[x + n / 2] : v[x];
                        v[x] = keep + __shfl_xor_sync(0xffffffffu, send, st);
                    }
                }
#pragma unroll
                for (int x = 0; x < R; ++x) {
                    const int id = sl * R + x, key = k0 + kgp * KPG + id / 8, g = g0 + id % 8;
                    if (key < nk && g < A.G) sc[g * kThreads + key] = v[x];
                }
            }
        }
    }
    __syncthreads();
    float *part_b = A.part + ((int64_t)b * A.Hq + (int64_t)h * A.G) * A.nparts * (D + 2);
    for (int g = warp; g < A.G; g += nw) {
        float m = -INFINITY;
        for (int k = lane; k < nk; k += 32) m = fmaxf(m, sc[g * kThreads + k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int k = lane; k < nk; k += 32) {
            const float p = exp2f(sc[g * kThreads + k] - m);
            sc[g * kThreads + k] = p;
            l += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        __syncwarp();
        float acc[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[e] = 0.f;
#pragma unroll 4
        for (int k = 0; k < nk; ++k) {
            const float p = sc[g * kThreads + k];
            float vv[DL];
            load_lane_slice<T, DL>(Vs + (size_t)k * D + lane * DL, vv);
#pragma unroll
            for (int e = 0; e < DL; ++e) acc[e] = fmaf(p, vv[e], acc[e]);
        }
        float *dst = part_b + ((int64_t)g * A.nparts + pi) * (D + 2);
#pragma unroll
        for (int e = 0; e < DL; ++e) dst[2 + lane * DL + e] = acc[e];
        if (lane == 0) {
            dst[0] = nk > 0 ? m : -INFINITY;
            dst[1] = l;
        }
    }
}

// ---- bf16 slices on warp-level tensor-core tiles (mma.sync m16n8k16) ----
// A slice is a [G x D] . [D x keys] product: the G <= 16 query heads of a KV
// head are the 16 rows of an m16 tile (rows >= G are zero).  Rows in shared
// memory are padded by 16 bytes, so the eight 16-byte rows an ldmatrix reads
// fall in distinct banks.
constexpr int kQRows = 16;

__device__ __forceinline__ uint32_t su32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(su32(p))
                 : "memory");
}
__device__ __forceinline__ void ldsm4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(su32(p))
                 : "memory");
}
__device__ __forceinline__ void ldsm2_t(uint32_t (&r)[2], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(su32(p))
                 : "memory");
}
// d (16x8 f32) += a (16x16 bf16, row major) . b (16x8 bf16, column major)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__host__ __device__ constexpr int tc_row() { return D + 8; }                                // K, V and Q rows
template <int D>
__host__ __device__ constexpr int tc_prow() { return (32 * 1024) / (D * 2) + 8; }  // P rows
template <int D>
__host__ __device__ constexpr size_t tc_tile_bytes() {                                      // Q and P tiles
    return sizeof(__nv_bfloat16) * kQRows * (size_t)(tc_row<D>() + tc_prow<D>());
}
template <int D>
__host__ __device__ constexpr size_t tc_dyn_bytes() {                   // K and V rows
    return 2 * sizeof(__nv_bfloat16) * (size_t)(tc_prow<D>() - 8) * tc_row<D>();
}

// Rotated queries of the KV head's G heads, scaled by log2(e)/sqrt(D) and
// rounded to bf16, as the 16-row A tile Qb (rows >= G zero).
template <int D>
__device__ __forceinline__ void load_queries_tc(const DecodeArgs &A, int b, int h, int32_t pnew,
                                                __nv_bfloat16 *Qb) {
    constexpr int H = D / 2, RE = tc_row<D>();
    const __nv_bfloat16 *qb =
        static_cast<const __nv_bfloat16 *>(A.q_new) + ((int64_t)b * A.Hq + (int64_t)h * A.G) * D;
    for (int e = threadIdx.x; e < kQRows * H; e += blockDim.x) {
        const int g = e / H, i = e % H;
        float o0 = 0.f, o1 = 0.f;
        if (g < A.G) {
            const float2 r = rope_cs_int(A.rope, pnew, i);
            const float x = to_f(qb[g * D + i]), y = to_f(qb[g * D + i + H]);
            o0 = (x * r.x - y * r.y) * A.scale_log2;
            o1 = (y * r.x + x * r.y) * A.scale_log2;
        }
        Qb[g * RE + i] = __float2bfloat16_rn(o0);
        Qb[g * RE + i + H] = __float2bfloat16_rn(o1);
    }
}

// attend_part for bf16 on tensor-core tiles.  Same inputs and partial
// (m, l, o[D]) output; P is rounded to bf16 for P.V and l sums the rounded
// weights, so the weights of a row sum to exactly l.
template <int D, typename KeyOf>
__device__ void attend_part_tc(const DecodeArgs &A, int b, int h, int t, int nk, KeyOf key_of,
                               int pi, const __nv_bfloat16 *Qb, const __nv_bfloat16 *knew,
                               float *sc, int *kt_s, __nv_bfloat16 *Pb, __nv_bfloat16 *Ks,
                               __nv_bfloat16 *Vs) {
    using bf = __nv_bfloat16;
    constexpr int RE = tc_row<D>(), PE = tc_prow<D>();
    constexpr int NV = D / 8;                           // 16-byte chunks per row
    static_assert(D % 32 == 0 && kThreads == 256, "8 warps, two k-steps per ldmatrix");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int nk16 = (nk + 15) & ~15;
    for (int k = threadIdx.x; k < nk; k += blockDim.x) kt_s[k] = key_of(k);
    __syncthreads();
    const bf *kbase = static_cast<const bf *>(A.k_rot);
    const bf *vbase = static_cast<const bf *>(A.v);
    const bf *vn = static_cast<const bf *>(A.v_new) + ((int64_t)b * A.Hkv + h) * D;
    for (int idx = threadIdx.x; idx < nk16 * NV; idx += blockDim.x) {
        const int k = idx / NV, pv = idx % NV;
        uint4 *kd = reinterpret_cast<uint4 *>(Ks + (size_t)k * RE) + pv;
        uint4 *vd = reinterpret_cast<uint4 *>(Vs + (size_t)k * RE) + pv;
        if (k >= nk) {                                  // pad rows: P.V must see zeros
            *kd = make_uint4(0u, 0u, 0u, 0u);
            *vd = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        const int kv = kt_s[k];
        const int64_t row = (((int64_t)b * A.Tc + kv) * A.Hkv + h) * D;
        if (kv == t) *kd = reinterpret_cast<const uint4 *>(knew)[pv];
        else cp_async16(kd, reinterpret_cast<const uint4 *>(kbase + row) + pv);
        cp_async16(vd, reinterpret_cast<const uint4 *>(kv == t ? vn : vbase + row) + pv);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    const int g_lo = lane >> 2, c2 = (lane & 3) * 2;
    // S = Q K^T: 8-key column tiles over the warps, the Q fragments held
    {
        uint32_t qa[D / 16][4];
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8, cc = (lane >> 4) * 8;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) ldsm4(qa[kk], Qb + r * RE + kk * 16 + cc);
        for (int nt = warp; nt < nk16 / 8; nt += nw) {
            const int n0 = nt * 8;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; kk += 2) {
                uint32_t kb[4];
                ldsm4(kb, Ks + (size_t)(n0 + (lane & 7)) * RE + kk * 16 + (lane >> 3) * 8);
                mma16816(acc, qa[kk], kb[0], kb[1]);
                mma16816(acc, qa[kk + 1], kb[2], kb[3]);
            }
            const int key = n0 + c2;
            if (g_lo < A.G) {
                if (key < nk) sc[g_lo * kThreads + key] = acc[0];
                if (key + 1 < nk) sc[g_lo * kThreads + key + 1] = acc[1];
            }
            if (g_lo + 8 < A.G) {
                if (key < nk) sc[(g_lo + 8) * kThreads + key] = acc[2];
                if (key + 1 < nk) sc[(g_lo + 8) * kThreads + key + 1] = acc[3];
            }
        }
    }
    __syncthreads();
    // softmax per head (base 2, scores pre-scaled): P as bf16 into the A tile
    float *part_b = A.part + ((int64_t)b * A.Hq + (int64_t)h * A.G) * A.nparts * (D + 2);
    for (int g = warp; g < kQRows; g += nw) {
        if (g >= A.G) {
            for (int k = lane; k < nk16; k += 32) Pb[g * PE + k] = __float2bfloat16_rn(0.f);
            continue;
        }
        float m = -INFINITY;
        for (int k = lane; k < nk; k += 32) m = fmaxf(m, sc[g * kThreads + k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int k = lane; k < nk16; k += 32) {
            const bf p = __float2bfloat16_rn(k < nk ? exp2f(sc[g * kThreads + k] - m) : 0.f);
            Pb[g * PE + k] = p;
            l += __bfloat162float(p);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            float *dst = part_b + ((int64_t)g * A.nparts + pi) * (D + 2);
            dst[0] = nk > 0 ? m : -INFINITY;
            dst[1] = l;
        }
    }
    __syncthreads();
    // O = P V: warp w owns output dims [w D/8, (w + 1) D/8)
    {
        constexpr int NT = D / 64;                      // 8-dim column tiles per warp
        const int d0 = warp * (D / 8);
        float o[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        const int pr = (lane & 7) + ((lane >> 3) & 1) * 8, pc = (lane >> 4) * 8;
        const int vr = (lane & 7) + ((lane >> 3) & 1) * 8;
        for (int k0 = 0; k0 < nk16; k0 += 16) {
            uint32_t pa[4];
            ldsm4(pa, Pb + pr * PE + k0 + pc);
            if constexpr (NT == 2) {
                uint32_t vb[4];
                ldsm4_t(vb, Vs + (size_t)(k0 + vr) * RE + d0 + (lane >> 4) * 8);
                mma16816(o[0], pa, vb[0], vb[1]);
                mma16816(o[1], pa, vb[2], vb[3]);
            } else {
                uint32_t vb[2];
                ldsm2_t(vb, Vs + (size_t)(k0 + vr) * RE + d0);
                mma16816(o[0], pa, vb[0], vb[1]);
            }
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int d = d0 + 8 * j + c2;
            if (g_lo < A.G) {
                float *dst = part_b + ((int64_t)g_lo * A.nparts + pi) * (D + 2) + 2;
                dst[d] = o[j][0];
                dst[d + 1] = o[j][1];
            }
            if (g_lo + 8 < A.G) {
                float *dst = part_b + ((int64_t)(g_lo + 8) * A.nparts + pi) * (D + 2) + 2;
                dst[d] = o[j][2];
                dst[d + 1] = o[j][3];
            }
        }
    }
}

// Every slice CTA (fixed or routed) ends here: the last of the nparts
// slices of (b, h) to finish combines all partial softmax sums into the
// output, and the last (b, h) of a sequence increments its lens.
template <typename T, int D>
__device__ void finish_slice(const DecodeArgs &A, int b, int h, int t, int *s_last) {
    constexpr int DL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int done = atomicAdd(&A.att_done[b * A.Hkv + h], 1);
        *s_last = done == A.nparts - 1;
    }
    __syncthreads();
    if (!*s_last) return;
    __threadfence();
    const float *part_b = A.part + ((int64_t)b * A.Hq + (int64_t)h * A.G) * A.nparts * (D + 2);
    for (int g = warp; g < A.G; g += nw) {
        const float *src = part_b + (int64_t)g * A.nparts * (D + 2);
        float M = -INFINITY;
#pragma unroll 4
        for (int sp = 0; sp < A.nparts; ++sp) M = fmaxf(M, __ldcg(src + sp * (D + 2)));
        float L = 0.f, acc[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[e] = 0.f;
#pragma unroll 4
        for (int sp = 0; sp < A.nparts; ++sp) {
            const float *ps = src + sp * (D + 2);
            const float m = __ldcg(ps);
            const float w = m == -INFINITY ? 0.f : exp2f(m - M);
            L += w * __ldcg(ps + 1);
#pragma unroll
            for (int e = 0; e < DL; ++e) acc[e] += w * __ldcg(ps + 2 + lane * DL + e);
        }
        const float inv = 1.f / L;
        T *o = static_cast<T *>(A.out) + ((int64_t)b * A.Hq + (int64_t)h * A.G + g) * D;
#pragma unroll
        for (int e = 0; e < DL; ++e) o[lane * DL + e] = from_f<T>(acc[e] * inv);
        if (A.lse && lane == 0)
            A.lse[(int64_t)b * A.Hq + (int64_t)h * A.G + g] = (M + __log2f(L)) * 0.6931471805599453f;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        A.att_done[b * A.Hkv + h] = 0;
        __threadfence();
        const int done = atomicAdd(&A.seq_done[b], 1);
        if (done == A.Hkv - 1) {
            A.seq_done[b] = 0;
            A.lens[b] = t + 1;
        }
    }
}

// The fixed keys of the token's visible set (sinks, recent chunks, the
// current chunk up to the token; the new key and value straight from the
// step's inputs, everything else from the cache), split in nF slices.
// Runs beside k_decode_a on a second stream: it needs no routing.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) k_decode_fixed(const DecodeArgs A) {
    constexpr bool kTc = sizeof(T) == 2;                              // bf16: tensor-core tiles
    __shared__ __align__(16) float qs[kTc ? 4 : kMaxG * D];
    __shared__ __align__(16) unsigned char tct[kTc ? tc_tile_bytes<D>() : 16];
    __shared__ __align__(16) T knew[D];
    __shared__ float sc[kMaxG * kThreads];
    __shared__ int kt_s[kThreads];
    __shared__ int s_last;
    extern __shared__ __align__(16) unsigned char dyn[];
    T *Ks = reinterpret_cast<T *>(dyn);                               // [slice_keys][row]
    constexpr int kSK = (32 * 1024) / (D * (int)sizeof(T)) < kThreads ? (32 * 1024) / (D * (int)sizeof(T)) : kThreads;
    constexpr int kRow = kTc ? tc_row<D>() : D;
    T *Vs = Ks + (size_t)kSK * kRow;
    __nv_bfloat16 *Qb = reinterpret_cast<__nv_bfloat16 *>(tct);
    __nv_bfloat16 *Pb = Qb + kQRows * tc_row<D>();
    const int f = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t = A.lens[b];
    if (t < 0 || t >= A.Tc) {
        if (threadIdx.x == 0) atomicExch(&g_decode_error, (int)HGA_ERR_BOUNDS);
        return;   // every CTA of this sequence sees the same lens and skips
    }
    const int c = t / A.C;
    const int32_t pnew = A.pos_new[b];
    const int nsink = min(A.F, c);
    const int rec_lo = max(c - max(A.L, 1), nsink);
    const int n1 = nsink * A.C, n2 = n1 + (c - rec_lo) * A.C;
    const int nfix = n2 + (t - c * A.C + 1);
    const int per = (nfix + A.nF - 1) / A.nF;
    const int k0 = min(nfix, f * per), nk = min(nfix, k0 + per) - k0;
    if constexpr (kTc) load_queries_tc<D>(A, b, h, pnew, Qb);
    else load_queries<T, D>(A, b, h, pnew, qs);
    rotate_new_key<T, D>(A, b, h, pnew, knew);
    __syncthreads();
    auto key_of = [&](int k) {
        const int i = k0 + k;
        return i < n1 ? i : (i < n2 ? rec_lo * A.C + (i - n1) : c * A.C + (i - n2));
    };
    if constexpr (kTc)
        attend_part_tc<D>(A, b, h, t, nk, key_of, f, Qb, knew, sc, kt_s, Pb, Ks, Vs);
    else
        attend_part<T, D>(A, b, h, t, nk, key_of, f, qs, knew, sc, kt_s, Ks, Vs);
    finish_slice<T, D>(A, b, h, t, &s_last);
}

// Shared memory of k_decode_a (chunk scan and routing).
template <typename T, int D>
struct ScanSmem {
    double qr[D];
    unsigned long long cand[kMaxCand];
    unsigned long long top[kMaxK];
    unsigned long long lists[kThreads];
    int sel_c[kMaxK], sel_g[kMaxK];
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 4) k_decode_a(const DecodeArgs A) {
    constexpr int H = D / 2;
    __shared__ ScanSmem<T, D> ss;
    __shared__ int s_last;
    double *qr = ss.qr;
    unsigned long long *cand = ss.cand;
    int *sel_c = ss.sel_c, *sel_g = ss.sel_g;

    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t = A.lens[b];
    if (t < 0 || t >= A.Tc) {
        if (threadIdx.x == 0) atomicExch(&g_decode_error, (int)HGA_ERR_BOUNDS);
        return;   // every CTA of this sequence sees the same lens and skips
    }
    const int c = t / A.C;
    const int32_t pnew = A.pos_new[b];

    // ------------------------------------------------------------- scan --
    if (s == 0) {
        const T *kn = static_cast<const T *>(A.k_new) + ((int64_t)b * A.Hkv + h) * D;
        const T *vn = static_cast<const T *>(A.v_new) + ((int64_t)b * A.Hkv + h) * D;
        const int64_t row = ((int64_t)b * A.Tc + t) * A.Hkv + h;
        T *kr = static_cast<T *>(A.k_rot) + row * D;
        T *vr = static_cast<T *>(A.v) + row * D;
        T *ko = static_cast<T *>(A.k_open) + (((int64_t)b * A.Hkv + h) * A.C + t % A.C) * D;
        for (int i = threadIdx.x; i < H; i += blockDim.x) {
            const float x = to_f(kn[i]), y = to_f(kn[i + H]);
            const float2 r = rope_cs_int(A.rope, pnew, i);
            const float2 rr = rot_pair(x, y, r);
            kr[i] = from_f<T>(rr.x);
            kr[i + H] = from_f<T>(rr.y);
            ko[i] = kn[i];
            ko[i + H] = kn[i + H];
        }
        for (int i = threadIdx.x; i < D; i += blockDim.x) vr[i] = vn[i];
        if (h == 0 && threadIdx.x == 0) A.pos[(int64_t)b * A.Tc + t] = pnew;
        __syncthreads();
        if (t % A.C == A.C - 1) close_chunk<T, D>(A, b, h, c, pnew);
    }

    // routing query of the token: the KV head's query heads summed, in fp64
    if (threadIdx.x < H) {
        const int i = threadIdx.x;
        const float2 r = rope_cs_int(A.rope, pnew, i);
        const T *qb = static_cast<const T *>(A.q_new) + ((int64_t)b * A.Hq + (int64_t)h * A.G) * D;
        double a = 0.0, d2 = 0.0;
#pragma unroll
        for (int g = 0; g < kMaxG; ++g) {
            if (g < A.G) {
                const float x = to_f(qb[g * D + i]), y = to_f(qb[g * D + i + H]);
                a += (double)(x * r.x - y * r.y);
                d2 += (double)(y * r.x + x * r.y);
            }
        }
        qr[i] = a;
        qr[i + H] = d2;
    }
    __syncthreads();

    // this CTA's slice of the middle chunks, one row per thread
    const int mlo = A.F, mhi = middle_hi(c, A.L);
    const int first = max(mlo, s * kScanChunks);
    const int last = min(mhi, s * kScanChunks + kScanChunks - 1);
    const int n = max(0, last - first + 1);
    const float *Sc = A.s_chunk + ((int64_t)b * A.Hkv + h) * A.nc_cap * D;
    if (threadIdx.x < n)
        cand[threadIdx.x] = pack_key(
            (float)thread_dot_row<D, false, 8>(qr, Sc + (int64_t)(first + threadIdx.x) * D),
            first + threadIdx.x);
    __syncthreads();
    // this CTA's top K_c keys, descending and 0-padded
    unsigned long long *mine = A.cand + (((int64_t)b * A.Hkv + h) * A.ns_scan + s) * A.K_c;
    if (A.K_c <= 32) {
        block_topk32_keys(cand, n, A.K_c, mine, ss.lists);
    } else {
        rank_topk(cand, n, A.K_c, ss.top);
        for (int r = threadIdx.x; r < A.K_c; r += blockDim.x) mine[r] = ss.top[r];
    }

    // the last scan CTA of (b, h) merges and routes the groups
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int done = atomicAdd(&A.scan_done[b * A.Hkv + h], 1);
        s_last = done == A.ns_scan - 1;
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;");
    if (!s_last) return;
    __threadfence();
    const unsigned long long *all = A.cand + ((int64_t)b * A.Hkv + h) * A.ns_scan * A.K_c;
    const int ntot = A.ns_scan * A.K_c;
    for (int r = threadIdx.x; r < ntot; r += blockDim.x) cand[r] = __ldcg(all + r);
    __syncthreads();
    // the scan CTAs' lists are descending: ranks by binary search
    rank_topk_lists(cand, A.ns_scan, A.K_c, A.K_c, ss.top);
    const int kc = ids_ascending(ss.top, A.K_c, sel_c);
    int32_t *oc = A.sel_c + ((int64_t)b * A.Hkv + h) * A.K_c;
    for (int r = threadIdx.x; r < A.K_c; r += blockDim.x) oc[r] = sel_c[r];
    const float *Sg = A.s_group + ((int64_t)b * A.Hkv + h) * A.nc_cap * A.gpc * D;
    const int ng = kc * A.gpc;
    // four lanes per group row (all of a row's loads in one round trip)
    for (int x = threadIdx.x; x < ((ng + 63) / 64) * 256; x += blockDim.x) {
        const int r = x >> 2;
        const int rr = r < ng ? r : 0;            // whole quads stay converged
        const int gid = sel_c[rr / A.gpc] * A.gpc + rr % A.gpc;
        const double sv = ng > 0 ? quad_dot_row<D>(qr, Sg + (int64_t)gid * D) : 0.0;
        if (r < ng && (x & 3) == 0) cand[r] = pack_key((float)sv, gid);
    }
    __syncthreads();
    rank_topk(cand, ng, A.K_g, ss.top);
    ids_ascending(ss.top, A.K_g, sel_g);
    int32_t *og = A.sel_g + ((int64_t)b * A.Hkv + h) * A.K_g;
    for (int r = threadIdx.x; r < A.K_g; r += blockDim.x) og[r] = sel_g[r];
    if (threadIdx.x == 0) A.scan_done[b * A.Hkv + h] = 0;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) k_decode_b(const DecodeArgs A) {
    constexpr bool kTc = sizeof(T) == 2;                              // bf16: tensor-core tiles
    __shared__ __align__(16) float qs[kTc ? 4 : kMaxG * D];
    __shared__ __align__(16) unsigned char tct[kTc ? tc_tile_bytes<D>() : 16];
    __shared__ __align__(16) T knew[D];
    __shared__ float sc[kMaxG * kThreads];
    __shared__ int kt_s[kThreads];
    __shared__ int sel[kMaxK];
    __shared__ int s_last;
    extern __shared__ __align__(16) unsigned char dyn[];
    T *Ks = reinterpret_cast<T *>(dyn);                               // [slice_keys][row]
    constexpr int kSK = (32 * 1024) / (D * (int)sizeof(T)) < kThreads ? (32 * 1024) / (D * (int)sizeof(T)) : kThreads;
    constexpr int kRow = kTc ? tc_row<D>() : D;
    T *Vs = Ks + (size_t)kSK * kRow;
    __nv_bfloat16 *Qb = reinterpret_cast<__nv_bfloat16 *>(tct);
    __nv_bfloat16 *Pb = Qb + kQRows * tc_row<D>();

    const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t = A.lens[b];          // written only by the previous step
    const int32_t pnew = A.pos_new[b];
    if (t >= 0 && t < A.Tc) {
        if constexpr (kTc) load_queries_tc<D>(A, b, h, pnew, Qb);
        else load_queries<T, D>(A, b, h, pnew, qs);
    }
    // everything below reads what k_decode_a wrote
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (t < 0 || t >= A.Tc) return;
    for (int j = threadIdx.x; j < A.K_g; j += blockDim.x)
        sel[j] = A.sel_g[((int64_t)b * A.Hkv + h) * A.K_g + j];
    __syncthreads();
    int kg = 0;
    for (int j = 0; j < A.K_g; ++j) kg += sel[j] >= 0;
    const int nrt = kg * A.g_s;
    const int per = (nrt + A.nR - 1) / A.nR;
    const int k0 = min(nrt, r * per), nk = min(nrt, k0 + per) - k0;
    auto key_of = [&](int k) {
        const int i = k0 + k;
        return sel[i / A.g_s] * A.g_s + i % A.g_s;
    };
    if constexpr (kTc)
        attend_part_tc<D>(A, b, h, t, nk, key_of, A.nF + r, Qb, knew, sc, kt_s, Pb, Ks, Vs);
    else
        attend_part<T, D>(A, b, h, t, nk, key_of, A.nF + r, qs, knew, sc, kt_s, Ks, Vs);

    finish_slice<T, D>(A, b, h, t, &s_last);
}

struct Ws {
    size_t counters, cand, sel_c, sel_g, part, total;
};

// Scan CTAs: scan CTA s holds middle chunks [256 s, 256 s + 256); the highest
// middle chunk a step can have is nc - L - 2 (nc - 3 with L = 0).
int scan_splits(const Geo &g) {
    const int nc = g.T / g.C;
    return max(0, nc - 2 - g.L) / kScanChunks + 1;
}

inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Fixed and routed slice CTAs per (sequence, KV head) for a slice size.
struct Slices {
    int nF, nR;
};
Slices slices(const Geo &g, int keys) {
    Slices s;
    s.nF = ((g.F + max(g.L, 1) + 1) * g.C + keys - 1) / keys;
    const long long routed = min((long long)g.K_g * g.g_s, (long long)g.T);
    s.nR = max(1, (int)((routed + keys - 1) / keys));
    return s;
}

Ws layout(const Geo &g) {
    const int ns = scan_splits(g);
    const Slices sl = slices(g, kMinSliceKeys);      // the most partials of any type
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
    o += up256(sizeof(float) * (size_t)g.B * g.Hq * (sl.nF + sl.nR) * (g.D + 2));
    w.total = o;
    return w;
}

// Per-device side stream and fork / join events for the fixed-key slices,
// created on the first decode step of a device and kept for the process.
// One mutex keeps a step's enqueue sequence (which reuses the events) whole.
struct DecodeSide {
    bool ready = false;
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_dec_mu;
DecodeSide g_dec_side[64];

cudaError_t decode_side(int dev, DecodeSide **out) {
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    DecodeSide &d = g_dec_side[dev];
    if (!d.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&d.side, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&d.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&d.join, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            // release what was made, so a later call starts from nothing
            if (d.join) cudaEventDestroy(d.join);
            if (d.fork) cudaEventDestroy(d.fork);
            if (d.side) cudaStreamDestroy(d.side);
            d = DecodeSide();
            return e;
        }
        d.ready = true;
    }
    *out = &d;
    return cudaSuccess;
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
    A.ns_scan = scan_splits(g);
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

    const Slices sl = slices(g, slice_keys<T, D>());
    A.nF = sl.nF;
    A.nR = sl.nR;
    A.nparts = sl.nF + sl.nR;
    const size_t vs_bytes = sizeof(T) == 2 ? tc_dyn_bytes<D>()
                                           : 2 * sizeof(T) * (size_t)slice_keys<T, D>() * D;
    cudaError_t e = ensure_smem((const void *)k_decode_fixed<T, D>, vs_bytes);
    if (e == cudaSuccess) e = ensure_smem((const void *)k_decode_b<T, D>, vs_bytes);
    if (e != cudaSuccess) return cuda_status(e);
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_status(e);
    std::lock_guard<std::mutex> lock(g_dec_mu);
    DecodeSide *sd = nullptr;
    if ((e = decode_side(dev, &sd)) != cudaSuccess) return cuda_status(e);
    // caller's stream: scan and routing, then the routed slices as its
    // programmatic dependents; side stream (forked before, joined after):
    // the fixed slices, which need no routing
    if ((e = cudaEventRecord(sd->fork, st)) != cudaSuccess) return cuda_status(e);
    k_decode_a<T, D><<<dim3(A.ns_scan, g.Hkv, g.B), kThreads, 0, st>>>(A);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(A.nR, g.Hkv, g.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = vs_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, k_decode_b<T, D>, A)) != cudaSuccess) return cuda_status(e);
    if ((e = cudaStreamWaitEvent(sd->side, sd->fork, 0)) != cudaSuccess) return cuda_status(e);
    k_decode_fixed<T, D><<<dim3(A.nF, g.Hkv, g.B), kThreads, vs_bytes, sd->side>>>(A);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    if ((e = cudaEventRecord(sd->join, sd->side)) != cudaSuccess) return cuda_status(e);
    return cuda_status(cudaStreamWaitEvent(st, sd->join, 0));
}

}  // namespace

// Shapes the fixed-size tables hold: the merge and group candidates fit
// kMaxCand, the query heads of a KV head kMaxG.
bool decode_supported(const Geo &g) {
    const long long ns = scan_splits(g);
    return g.G <= kMaxG && ns * g.K_c <= kMaxCand && (long long)g.K_c * g.gpc <= kMaxCand;
}

size_t decode_workspace_bytes(const Geo &g) { return layout(g).total; }

hga_status launch_decode(const Geo &g, const Rope &r, int dtype, const hga_io &io, void *ws,
                         cudaStream_t st) {
    if (!decode_supported(g)) return HGA_ERR_UNSUPPORTED;
    if (dtype == HGA_BF16)
        return g.D == 128 ? run<__nv_bfloat16, 128>(g, r, io, ws, st)
                          : run<__nv_bfloat16, 64>(g, r, io, ws, st);
    return g.D == 128 ? run<float, 128>(g, r, io, ws, st) : run<float, 64>(g, r, io, ws, st);
}


// Reads this file's device error word on `st` (after the work queued on it)
// and optionally resets it; returns the recorded status (HGA_OK if none).
hga_status decode_error_take(cudaStream_t st, bool clear) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_decode_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_decode_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    return (hga_status)v;
}

}  // namespace hga
