// The C ABI of include/hga.h: host-side argument checks, workspace layout and
// kernel dispatch.  Nothing here allocates device memory; every kernel is
// enqueued on the caller's stream.
#include <climits>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "hga_internal.cuh"
#include "route_common.cuh"

namespace hga {

static thread_local int g_last_cuda_error = 0;

hga_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return HGA_OK;
    g_last_cuda_error = (int)e;
    return HGA_ERR_CUDA;
}

// The opt-in belongs to the kernel as loaded on one device, so the record of
// what was granted is kept per (kernel, device).
cudaError_t ensure_smem(const void *kernel, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> granted;
    int dev = 0;
    const cudaError_t de = cudaGetDevice(&dev);
    if (de != cudaSuccess) return de;
    std::lock_guard<std::mutex> lock(mu);
    size_t &have = granted[std::make_pair(kernel, dev)];
    if (bytes <= have) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) have = bytes;
    return e;
}

hga_status set_rope(Rope *r, int D, double theta, double hf_wavelength, int C) {
    std::memset(r, 0, sizeof(*r));
    const double hf = hf_wavelength > 0 ? hf_wavelength : (double)C;
    r->half = D / 2;
    for (int i = 0; i < D / 2; ++i) {
        r->omega[i] = std::pow(theta, -2.0 * (double)i / (double)D);
        if (2.0 * M_PI / r->omega[i] < hf) r->high |= 1ull << i;
        // turns per position as a 64-bit fraction (extended precision on the host)
        const long double two_pi = 6.283185307179586476925286766559L;
        const long double t = (long double)r->omega[i] / two_pi * 18446744073709551616.0L;
        r->turn[i] = (unsigned long long)llroundl(t);
    }
    return HGA_OK;
}

namespace {

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

constexpr int kMaxGridYZ = 65535;

hga_status check_common(const hga_dims *d, const hga_params *p) {
    if (!d || !p) return HGA_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 0 || d->Hq < 1 || d->Hkv < 1 || d->Hq % d->Hkv) return HGA_ERR_INVALID_ARG;
    if (d->dtype != HGA_F32 && d->dtype != HGA_BF16) return HGA_ERR_INVALID_ARG;
    if (p->C < 1 || p->g_s < 1 || p->C % p->g_s || p->F < 0 || p->L < 0 || p->K_c < 0 || p->K_g < 0)
        return HGA_ERR_INVALID_ARG;
    if (!(p->rope_theta > 1.0) || !std::isfinite(p->rope_theta) || std::isnan(p->hf_wavelength))
        return HGA_ERR_INVALID_ARG;
    if (d->D != 64 && d->D != 128) return HGA_ERR_UNSUPPORTED;
    // B and Hkv index grid axes (65535 at most); token rows b * T + t are
    // 32-bit tensor-map coordinates
    if (d->B > kMaxGridYZ || d->Hkv > kMaxGridYZ || (long long)d->B * d->T > (long long)INT32_MAX)
        return HGA_ERR_UNSUPPORTED;
    if (p->C != kChunk) return HGA_ERR_UNSUPPORTED;
    if (p->K_c > kMaxK || p->K_g > kMaxK) return HGA_ERR_UNSUPPORTED;
    return HGA_OK;
}

Geo make_geo(const hga_dims *d, const hga_params *p) {
    Geo g;
    g.B = d->B;
    g.T = d->T;
    g.Hq = d->Hq;
    g.Hkv = d->Hkv;
    g.D = d->D;
    g.G = d->Hq / d->Hkv;
    g.C = p->C;
    g.g_s = p->g_s;
    g.gpc = p->C / p->g_s;
    g.F = p->F;
    g.L = p->L;
    g.K_c = p->K_c;
    g.K_g = p->K_g;
    g.NC = d->T / p->C;
    g.NB = (d->T + p->C - 1) / p->C;
    return g;
}

inline size_t esize(int dtype) { return dtype == HGA_BF16 ? 2 : 4; }
inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Prefill workspace: K_rot, chunk and group summaries, selections, and (for
// shapes the tensor-core attention takes, when the workspace has room) the
// rotated queries stage 2 writes for stage 3.  `min` is the size without
// them.
struct PrefillWs {
    size_t k_rot, s_chunk, s_group, sel_c, sel_g, q_rot, min, total;
};

PrefillWs prefill_ws(const Geo &g, int dtype) {
    PrefillWs w;
    size_t o = 0;
    w.k_rot = o;
    o += up256((size_t)g.B * g.T * g.Hkv * g.D * esize(dtype));
    w.s_chunk = o;
    o += up256((size_t)g.B * g.Hkv * g.NC * g.D * 4);
    w.s_group = o;
    o += up256((size_t)g.B * g.Hkv * g.NC * g.gpc * g.D * 4);
    w.sel_c = o;
    o += up256((size_t)g.B * g.NB * g.Hkv * g.K_c * 4);
    w.sel_g = o;
    o += up256((size_t)g.B * g.NB * g.Hkv * g.K_g * 4);
    w.min = o;
    w.q_rot = o;
    if (dtype == HGA_BF16 && attend_tc_supported(g, dtype))
        o += up256((size_t)g.B * g.T * g.Hq * g.D * 2);
    w.total = o;
    return w;
}

hga_status attend_dispatch(const Geo &g, const Rope &r, int dtype, const void *q, const int32_t *pos,
                           const void *k_rot, int k_T, const void *v, int v_T,
                           const int32_t *sel_group, void *out, float *lse, cudaStream_t st,
                           const void *q_rot = nullptr) {
    if (attend_tc_supported(g, dtype))
        return launch_attend_tc(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st,
                                nullptr, q_rot);
    return launch_attend_simt(g, r, dtype, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st);
}

}  // namespace
}  // namespace hga

using namespace hga;

extern "C" {

hga_status hga_build_summaries(const hga_dims *dims, const hga_params *prm, const void *k_raw,
                               const int32_t *pos, void *k_rot, float *s_chunk, float *s_group,
                               void *stream) {
    hga_status s = check_common(dims, prm);
    if (s != HGA_OK) return s;
    if (dims->T == 0) return HGA_OK;
    const bool has_closed = dims->T >= prm->C;   // summary tables may be empty (NULL)
    if (!k_raw || !pos || (has_closed && (!s_chunk || !s_group))) return HGA_ERR_INVALID_ARG;
    if (!aligned16(k_raw) || (k_rot && !aligned16(k_rot)) || !aligned16(s_chunk) || !aligned16(s_group))
        return HGA_ERR_INVALID_ARG;
    const Geo g = make_geo(dims, prm);
    Rope r;
    set_rope(&r, g.D, prm->rope_theta, prm->hf_wavelength, prm->C);
    return launch_summaries(g, r, dims->dtype, k_raw, nullptr, pos, g.T, k_rot, nullptr, nullptr,
                            g.T, s_chunk, s_group, g.NC, nullptr, nullptr,
                            (cudaStream_t)stream);
}

hga_status hga_route(const hga_dims *dims, const hga_params *prm, const void *q, const int32_t *pos,
                     const float *s_chunk, const float *s_group, int32_t *sel_chunk,
                     int32_t *sel_group, void *q_rot, void *stream) {
    hga_status s = check_common(dims, prm);
    if (s != HGA_OK) return s;
    if (dims->T == 0) return HGA_OK;
    const bool has_closed = dims->T >= prm->C;
    if (!q || !pos || (has_closed && (!s_chunk || !s_group)) ||
        (prm->K_c > 0 && !sel_chunk) || (prm->K_g > 0 && !sel_group))
        return HGA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(s_chunk) || !aligned16(s_group) || !aligned16(q_rot))
        return HGA_ERR_INVALID_ARG;
    if (q_rot && dims->dtype != HGA_BF16) return HGA_ERR_UNSUPPORTED;
    const Geo g = make_geo(dims, prm);
    Rope r;
    set_rope(&r, g.D, prm->rope_theta, prm->hf_wavelength, prm->C);
    return launch_route(g, r, dims->dtype, q, pos, s_chunk, s_group, g.NC, sel_chunk, sel_group,
                        (cudaStream_t)stream, false, q_rot);
}

hga_status hga_attend(const hga_dims *dims, const hga_params *prm, const void *q, const int32_t *pos,
                      const void *k_rot, const void *v, const int32_t *sel_group, void *out,
                      float *lse, const void *q_rot, void *stream) {
    hga_status s = check_common(dims, prm);
    if (s != HGA_OK) return s;
    if (dims->T == 0) return HGA_OK;
    if (!q || !pos || !k_rot || !v || (prm->K_g > 0 && !sel_group) || !out)
        return HGA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_rot) || !aligned16(v) || !aligned16(out) ||
        !aligned16(q_rot))
        return HGA_ERR_INVALID_ARG;
    if (q_rot && dims->dtype != HGA_BF16) return HGA_ERR_UNSUPPORTED;
    const Geo g = make_geo(dims, prm);
    Rope r;
    set_rope(&r, g.D, prm->rope_theta, prm->hf_wavelength, prm->C);
    return attend_dispatch(g, r, dims->dtype, q, pos, k_rot, g.T, v, g.T, sel_group, out, lse,
                           (cudaStream_t)stream, q_rot);
}

size_t hga_prefill_workspace_min(const hga_dims *dims, const hga_params *prm) {
    if (check_common(dims, prm) != HGA_OK) return 0;
    return prefill_ws(make_geo(dims, prm), dims->dtype).min;
}

size_t hga_workspace_size(int mode, const hga_dims *dims, const hga_params *prm) {
    if (check_common(dims, prm) != HGA_OK) return 0;
    const Geo g = make_geo(dims, prm);
    if (mode == HGA_PREFILL) return prefill_ws(g, dims->dtype).total;
    if (mode == HGA_DECODE) return decode_workspace_bytes(g);
    if (mode == HGA_PREFILL_HOSTKV) return hostkv_workspace_bytes(g);
    if (mode == HGA_ATTEND_BACKWARD) return backward_workspace_bytes(g, dims->dtype);
    return 0;
}

hga_status hga_hostkv_plan_for(const hga_dims *dims, const hga_params *prm,
                               size_t workspace_bytes, hga_hostkv_plan *plan) {
    if (!plan) return HGA_ERR_INVALID_ARG;
    const hga_status s = check_common(dims, prm);
    if (s != HGA_OK) return s;
    return hostkv_plan(make_geo(dims, prm), workspace_bytes, plan);
}

hga_status hga_attend_backward(const hga_dims *dims, const hga_params *prm, const void *q,
                               const int32_t *pos, const void *k_rot, const void *v,
                               const int32_t *sel_group, const float *lse, const void *d_out,
                               const void *q_rot, float *dq, float *dk, float *dv,
                               void *workspace, size_t workspace_bytes, void *stream) {
    hga_status s = check_common(dims, prm);
    if (s != HGA_OK) return s;
    if (dims->T == 0) return HGA_OK;
    if (!q || !pos || !k_rot || !v || (prm->K_g > 0 && !sel_group) || !lse || !d_out || !dq ||
        !dk || !dv)
        return HGA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_rot) || !aligned16(v) || !aligned16(d_out) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(q_rot))
        return HGA_ERR_INVALID_ARG;
    if (q_rot && dims->dtype != HGA_BF16) return HGA_ERR_UNSUPPORTED;
    const Geo g = make_geo(dims, prm);
    const size_t need = backward_workspace_bytes(g, dims->dtype);
    if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u))
        return HGA_ERR_WORKSPACE;
    Rope r;
    set_rope(&r, g.D, prm->rope_theta, prm->hf_wavelength, prm->C);
    return launch_attend_backward(g, r, dims->dtype, q, pos, k_rot, v, sel_group, lse, d_out,
                                  dq, dk, dv, workspace, q_rot, (cudaStream_t)stream);
}

hga_status hga_forward(int mode, const hga_dims *dims, const hga_params *prm, const hga_io *io,
                       void *workspace, size_t workspace_bytes, void *stream) {
    hga_status s = check_common(dims, prm);
    if (s != HGA_OK) return s;
    if (!io) return HGA_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    const Geo g = make_geo(dims, prm);
    Rope r;
    set_rope(&r, g.D, prm->rope_theta, prm->hf_wavelength, prm->C);
    size_t need = hga_workspace_size(mode, dims, prm);
    if (mode == HGA_PREFILL) need = prefill_ws(g, dims->dtype).min;   // q_rot when it fits
    if (mode == HGA_PREFILL_HOSTKV) {
        // any workspace the warm tier's smallest plan fits in
        hga_hostkv_plan pl;
        hostkv_plan(g, 0, &pl);
        need = pl.min_bytes;
    }
    const bool ws_ok =
        need == 0 || (workspace && workspace_bytes >= need && !((uintptr_t)workspace & 255u));
    char *ws = static_cast<char *>(workspace);

    if (io->s_group_host && mode != HGA_PREFILL_HOSTKV) return HGA_ERR_INVALID_ARG;
    if (mode == HGA_PREFILL) {
        if (dims->T == 0) return HGA_OK;
        const hga_kv_cache &cc = io->cache;
        const bool fill = cc.k_rot != nullptr;
        // cache fill only: no queries, no output (stage 1 into the cache)
        const bool fill_only = fill && !io->q && !io->out;
        if (!io->k || !io->v || !io->pos || (!fill_only && (!io->q || !io->out)))
            return HGA_ERR_INVALID_ARG;
        if ((io->q && !aligned16(io->q)) || !aligned16(io->k) || !aligned16(io->v) ||
            (io->out && !aligned16(io->out)))
            return HGA_ERR_INVALID_ARG;
        if (!fill_only && !ws_ok) return HGA_ERR_WORKSPACE;   // fill only needs none
        if (fill) {
            if ((long long)dims->B * cc.capacity > (long long)INT32_MAX) return HGA_ERR_UNSUPPORTED;
            if (cc.capacity < dims->T || cc.capacity % prm->C || !cc.v || !cc.pos || !cc.k_open ||
                !cc.s_chunk || !cc.s_group || !cc.lens)
                return HGA_ERR_INVALID_ARG;
            if (!aligned16(cc.k_rot) || !aligned16(cc.v) || !aligned16(cc.k_open) ||
                !aligned16(cc.s_chunk) || !aligned16(cc.s_group))
                return HGA_ERR_INVALID_ARG;
        }
        const PrefillWs w = prefill_ws(g, dims->dtype);
        void *k_rot = fill ? cc.k_rot : (void *)(ws + w.k_rot);
        const int k_T = fill ? cc.capacity : g.T;
        const int nc_cap = fill ? cc.capacity / prm->C : g.NC;
        float *s_chunk = fill ? cc.s_chunk : (float *)(ws + w.s_chunk);
        float *s_group = fill ? cc.s_group : (float *)(ws + w.s_group);
        int32_t *sel_c = io->sel_chunk ? io->sel_chunk : (int32_t *)(ws + w.sel_c);
        int32_t *sel_g = io->sel_group ? io->sel_group : (int32_t *)(ws + w.sel_g);
        s = launch_summaries(g, r, dims->dtype, io->k, fill ? io->v : nullptr, io->pos, g.T, k_rot,
                             fill ? cc.v : nullptr, fill ? cc.pos : nullptr, k_T, s_chunk, s_group,
                             nc_cap, fill ? cc.k_open : nullptr, fill ? cc.lens : nullptr, st);
        if (s != HGA_OK || fill_only) return s;
        // the rotated queries pass from stage 2 to stage 3 when the shape
        // takes the tensor-core attention and the workspace holds them
        void *q_rot = w.total > w.min && workspace_bytes >= w.total ? (void *)(ws + w.q_rot)
                                                                    : nullptr;
        s = launch_route(g, r, dims->dtype, io->q, io->pos, s_chunk, s_group, nc_cap, sel_c, sel_g,
                         st, false, q_rot);
        if (s != HGA_OK) return s;
        return attend_dispatch(g, r, dims->dtype, io->q, io->pos, k_rot, k_T, io->v, g.T, sel_g,
                               io->out, io->lse, st, q_rot);
    }
    if (mode == HGA_DECODE) {
        if (!ws_ok) return HGA_ERR_WORKSPACE;
        const hga_kv_cache &cc = io->cache;
        if (!io->q_new || !io->k_new || !io->v_new || !io->pos_new || !io->out) return HGA_ERR_INVALID_ARG;
        if (!cc.k_rot || !cc.v || !cc.pos || !cc.k_open || !cc.s_chunk || !cc.s_group || !cc.lens)
            return HGA_ERR_INVALID_ARG;
        if (cc.capacity != dims->T || cc.capacity < prm->C || cc.capacity % prm->C)
            return HGA_ERR_INVALID_ARG;
        if (!aligned16(io->q_new) || !aligned16(io->k_new) || !aligned16(io->v_new) ||
            !aligned16(io->out) || !aligned16(cc.k_rot) || !aligned16(cc.v) ||
            !aligned16(cc.k_open) || !aligned16(cc.s_chunk) || !aligned16(cc.s_group))
            return HGA_ERR_INVALID_ARG;
        return launch_decode(g, r, dims->dtype, *io, workspace, st);
    }
    if (mode == HGA_PREFILL_HOSTKV) {
        if (dims->T == 0) return HGA_OK;
        if (!ws_ok) return HGA_ERR_WORKSPACE;
        if (dims->dtype != HGA_BF16) return HGA_ERR_UNSUPPORTED;
        if (!io->q || !io->k || !io->v || !io->pos || !io->out || io->cache.k_rot)
            return HGA_ERR_INVALID_ARG;
        if (!aligned16(io->q) || !aligned16(io->k) || !aligned16(io->v) || !aligned16(io->out) ||
            !aligned16(io->s_group_host))
            return HGA_ERR_INVALID_ARG;
        return launch_prefill_hostkv(g, r, *io, workspace, workspace_bytes, st);
    }
    return HGA_ERR_INVALID_ARG;
}

const char *hga_status_string(hga_status s) {
    switch (s) {
    case HGA_OK: return "ok";
    case HGA_ERR_INVALID_ARG: return "invalid argument";
    case HGA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case HGA_ERR_CUDA: return "CUDA error";
    case HGA_ERR_TIMEOUT: return "bounded device wait timed out";
    case HGA_ERR_BOUNDS: return "device-side index check failed";
    case HGA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    }
    return "unknown status";
}

int hga_last_cuda_error(void) { return g_last_cuda_error; }

hga_status hga_device_status(void *stream, int clear) {
    const cudaStream_t st = (cudaStream_t)stream;
    hga_status first = HGA_OK;
    const hga_status parts[5] = {summaries_error_take(st, clear != 0),
                                 attend_tc_error_take(st, clear != 0),
                                 decode_error_take(st, clear != 0),
                                 tier_error_take(st, clear != 0),
                                 backward_error_take(st, clear != 0)};
    for (hga_status p : parts)
        if (p != HGA_OK && first == HGA_OK) first = p;
    return first;
}

hga_status hga_set_test_hooks(int skip_summaries_copy, unsigned long long summaries_wait_ns,
                              void *stream) {
    return summaries_test_hooks(skip_summaries_copy != 0 ? 1 : 0, summaries_wait_ns,
                                (cudaStream_t)stream);
}

hga_status hga_hostkv_link_bytes(void *stream, unsigned long long *bytes, int clear) {
    if (!bytes) return HGA_ERR_INVALID_ARG;
    return tier_link_bytes_take((cudaStream_t)stream, bytes, clear != 0);
}

}  // extern "C"
