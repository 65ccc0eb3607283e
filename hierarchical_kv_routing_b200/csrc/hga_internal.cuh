// Internal declarations of the HGA sm_100a library: per-call constants,
// device helpers shared by the kernels, and the host-side launchers that the
// C ABI (api.cu) calls after validating its arguments.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hga.h"

namespace hga {

constexpr int kChunk = 64;      // C; also the prefill query block
constexpr int kMaxHalf = 64;    // D/2 for D <= 128

// RoPE constants of one call: omega_i = theta^(-2i/D) (rotate-half pair
// (i, i + D/2)) and the high-frequency mask (pair i high iff its wavelength
// 2*pi/omega_i is below hf_wavelength).  Passed by value as a kernel
// parameter.
struct Rope {
    double omega[kMaxHalf];
    unsigned long long turn[kMaxHalf];  // round(omega_i / (2 pi) * 2^64): turns per position
    unsigned long long high;  // bit i set: pair i is high-frequency
    int half;                 // D / 2
};

// Shape and policy of one call, as the kernels see it.
struct Geo {
    int B, T, Hq, Hkv, D, G;    // T = tokens (prefill) or capacity (decode)
    int C, g_s, gpc, F, L, K_c, K_g;
    int NC;                     // closed chunks present (prefill: T / C)
    int NB;                     // query blocks: ceil(T / C)
};

// ---------------------------------------------------------------- device --

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// (cos, sin) of p * omega_i.  The angle is formed and reduced to [-pi, pi]
// in fp64 (two-term 2*pi, Cody-Waite), so positions up to 2^31 keep fp32
// accuracy; the reduced angle goes to the accurate sincosf.
__device__ __forceinline__ float2 rope_cs(const Rope &r, double p, int i) {
    const double a = p * r.omega[i];
    const double k = rint(a * 0.15915494309189535);           // 1 / (2 pi)
    double red = fma(-k, 6.283185307179586, a);                // 2 pi, high part
    red = fma(-k, 2.4492935982947064e-16, red);                // 2 pi, low part
    float s, c;
    sincosf((float)red, &s, &c);
    return make_float2(c, s);
}

// (cos, sin) of p * omega_i for an integer position p, without floating
// point range reduction: the angle in turns, p * omega_i / (2 pi), is formed
// modulo 1 in 64-bit fixed point (an integer product that wraps), its top 32
// bits taken as a signed fraction of a half turn, and passed to sincospif.
// The angle error is below pi * 2^-24 for |p| < 2^31, the same as rounding
// the reduced angle to fp32.
__device__ __forceinline__ float2 rope_cs_int(const Rope &r, int32_t p, int i) {
    const unsigned long long u = (unsigned long long)(long long)p * r.turn[i];
    const float x = (float)(int)(u >> 32) * 0x1p-31f;     // angle / pi in [-1, 1)
    float s, c;
    sincospif(x, &s, &c);
    return make_float2(c, s);
}

__device__ __forceinline__ bool is_high(const Rope &r, int i) { return (r.high >> i) & 1ull; }

// Rotate the pair (x, y) by the angle whose (cos, sin) is cs.  The rounding
// is spelled out (one product rounded, then one fused multiply-add) so every
// kernel that writes rotated keys produces the same bits for the same input.
__device__ __forceinline__ float2 rot_pair(float x, float y, float2 cs) {
    return make_float2(__fmaf_rn(x, cs.x, -__fmul_rn(y, cs.y)),
                       __fmaf_rn(y, cs.x, __fmul_rn(x, cs.y)));
}

// Routing keys: a score and a candidate id packed so that a larger key means
// a higher score, and on equal scores the lower id.  0 = no candidate.
__device__ __forceinline__ unsigned long long pack_key(float score, int id) {
    unsigned u = __float_as_uint(score);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)id);
}
__device__ __forceinline__ int key_id(unsigned long long k) {
    return (int)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull));
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Middle chunks of current chunk c: F <= m <= c-L-1, and with L == 0 the
// forced previous chunk c-1 is left out (it is always visible).
__device__ __forceinline__ int middle_hi(int c, int L) { return L == 0 ? c - 2 : c - L - 1; }

// ----------------------------------------------------------------- host --

hga_status set_rope(Rope *r, int D, double theta, double hf_wavelength, int C);
hga_status cuda_status(cudaError_t e);

// Raise a kernel's dynamic shared-memory limit to at least `bytes`, calling
// cudaFuncSetAttribute only when the limit has to grow (so repeated launches,
// including launches inside a stream capture, make no such call).
cudaError_t ensure_smem(const void *kernel, size_t bytes);

// Stage 1.  k_rot/v_out/pos_out/k_open/lens may be null.  in_T: tokens per
// sequence of the inputs; out_T: token capacity of k_rot/v_out/pos_out;
// nc_cap: chunk capacity of s_chunk/s_group.  host_src: k_raw is the device
// address of pinned host memory (read with plain loads; bf16, summaries only).
hga_status launch_summaries(const Geo &g, const Rope &r, int dtype, const void *k_raw,
                            const void *v_raw, const int32_t *pos, int in_T, void *k_rot,
                            void *v_out, int32_t *pos_out, int out_T, float *s_chunk,
                            float *s_group, int nc_cap, void *k_open, int32_t *lens,
                            cudaStream_t st, bool host_src = false);

// Stage 2 (prefill blocks).  host_groups: s_group is the device address of
// pinned host memory (read with plain loads).  q_rot (bf16 only, may be
// null): the rotated queries [B, T, Hq, D] are written there, rounded as the
// tensor-core attention rounds its own rotation.
hga_status launch_route(const Geo &g, const Rope &r, int dtype, const void *q, const int32_t *pos,
                        const float *s_chunk, const float *s_group, int nc_cap,
                        int32_t *sel_chunk, int32_t *sel_group, cudaStream_t st,
                        bool host_groups = false, void *q_rot = nullptr);

// Stage 3 (prefill blocks).  k_T / v_T: token capacity per sequence of k_rot
// and v.  The CUDA-core kernel takes every shape; the tensor-core kernel
// takes bf16 with g_s a multiple of 8.
hga_status launch_attend_simt(const Geo &g, const Rope &r, int dtype, const void *q,
                              const int32_t *pos, const void *k_rot, int k_T, const void *v,
                              int v_T, const int32_t *sel_group, void *out, float *lse,
                              cudaStream_t st);
size_t attend_simt_smem(const Geo &g);
bool attend_tc_supported(const Geo &g, int dtype);

// One wave of query blocks [c0, c1) whose keys and values sit in a staging
// buffer of the host-resident tier (rows per sequence: the buffer's k_T):
// tokens below sink_rows at row = token, other fixed-window and current
// tokens at row = win_row0 + token - win_tok0, and group slot j of block c at
// rows rt_row0 + ((c - c0) * K_g + j) * g_s (slot j holds the j-th routed id).
// One wave of the host tier: blocks [c0, c1); sinks and the recent/current
// window sit in a staging buffer starting at row buf_row0 (token tok < sink_rows
// at buf_row0 + tok, others at buf_row0 + win_row0 + tok - win_tok0); routed
// group slot j of (block c, KV head h, sequence b) starts at row
// rt_map[((b * rt_W + c - c0) * Hkv + h) * K_g + j] (the group cache).
struct TierWave {
    int c0, c1, sink_rows, win_tok0, win_row0, buf_row0, rt_W;
    const int32_t *rt_map;
};

// tw == nullptr: every query block, keys at their token rows.  q_rot
// non-null: the queries are already rotated (stage 2 wrote them) and q is
// not read.
hga_status launch_attend_tc(const Geo &g, const Rope &r, const void *q, const int32_t *pos,
                            const void *k_rot, int k_T, const void *v, int v_T,
                            const int32_t *sel_group, void *out, float *lse, cudaStream_t st,
                            const TierWave *tw = nullptr, const void *q_rot = nullptr);

// Prefill with K and V in pinned host memory (hga_forward HGA_PREFILL_HOSTKV).
size_t hostkv_workspace_bytes(const Geo &g);
hga_status hostkv_plan(const Geo &g, size_t workspace_bytes, hga_hostkv_plan *plan);
hga_status launch_prefill_hostkv(const Geo &g, const Rope &r, const hga_io &io, void *ws,
                                 size_t ws_bytes, cudaStream_t st);

// Backward of stage 3 (hga_attend_backward): dq [B,T,Hq,D], dk and dv
// [B,T,Hkv,D], fp32.  Workspace: per query row (LSE in base 2, Delta), and
// for the tensor-core path the rotated queries in bf16.
size_t backward_workspace_bytes(const Geo &g, int dtype);
hga_status launch_attend_backward(const Geo &g, const Rope &r, int dtype, const void *q,
                                  const int32_t *pos, const void *k_rot, const void *v,
                                  const int32_t *sel_group, const float *lse,
                                  const void *dout, float *dq, float *dk, float *dv, void *ws,
                                  const void *q_rot, cudaStream_t st);
hga_status backward_error_take(cudaStream_t st, bool clear);

// Device error words (bounded-wait timeouts, bounds checks) of each kernel
// file: read on a stream after its queued work, optionally reset.
hga_status attend_tc_error_take(cudaStream_t st, bool clear);
hga_status decode_error_take(cudaStream_t st, bool clear);
hga_status summaries_error_take(cudaStream_t st, bool clear);
hga_status summaries_test_hooks(int skip_copy, unsigned long long wait_ns, cudaStream_t st);
hga_status tier_error_take(cudaStream_t st, bool clear);
hga_status tier_link_bytes_take(cudaStream_t st, unsigned long long *bytes, bool clear);

// Decode step (append, close-chunk summaries, route, split attention).
size_t decode_workspace_bytes(const Geo &g);
hga_status launch_decode(const Geo &g, const Rope &r, int dtype, const hga_io &io, void *ws,
                         cudaStream_t st);

}  // namespace hga
