// Backward of stage 3: gradients of exact softmax attention over the routed
// token set with respect to the raw (pre-RoPE) queries and keys and the
// values, the routed groups held fixed (routing is a discrete choice, so no
// gradient reaches the summaries).
//
// Method: HGA paper-review page, section 6, Tab. 8 (a training step through
// the routed attention) and Sec. 5.9 (QK fine-tuning through it in the
// exact-token mode).  The page gives no formula; this is the derivative of
// eq. (1) restricted to each query token's visible set V(i):
//   S_ij = q~_i . k~_j / sqrt(D),  P_ij = exp(S_ij - LSE_i),  j in V(i)
//   dV_j  = sum_i P_ij dO_i
//   dS_ij = P_ij (dO_i . v_j - Delta_i),  Delta_i = sum_j P_ij dO_i . v_j
//   dq_i  = R_{p_i}^T  sum_j dS_ij k~_j / sqrt(D)
//   dk_j  = R_{p_j}^T  sum_i dS_ij q~_i / sqrt(D)
// where q~ = R_p(q), k~ = R_p(k) and i runs over the query rows of every
// query head of k_j's KV head.  Delta_i equals dO_i . O_i; it is formed from
// the kernels' own P and dO . v (a first pass over the keys) rather than from
// the stored output, so that the difference dO_i . v_j - Delta_i, which
// cancels heavily on rows whose weight sits on few keys, is taken between
// values with the same rounding (with a bf16 output the error of dO . O
// dominated such rows' dq).
//
// Kernels (bf16 on the tensor cores; fp32, and bf16 shapes the tensor-core
// kernels do not take, on the CUDA cores):
//   k_bwd_prep   per query row: q~ rounded to bf16 exactly as the forward
//                rounds it, and the LSE (in base 2 for the tensor cores).
//   k_bwd_dq_tc  query-major, like the forward: one CTA per (block, KV head,
//                256-row half), two 128-row M-tiles ping-ponging; per 64-key
//                tile S = Q~ K~^T and dP = dO V^T into TMEM.  A first pass
//                over the tiles sums Delta = P . dP per row (and stores it for
//                the dK/dV kernel); in the second the softmax warpgroups form
//                dS (bf16, over the S columns) and the tensor core
//                accumulates dQ~ += dS K~ in TMEM; the epilogue rotates dQ~
//                back and stores fp32 rows.
//   k_bwd_dkv_tc key-major inside a unit: one CTA per (block, KV head) owns
//                all 64*G query rows; per 128-key tile and 64-row subtile
//                S^T = K~ Q~^T and dP^T = V dO^T into TMEM (lane = key), the
//                softmax warpgroups form P^T and dS^T (bf16, in place), and
//                the tensor core accumulates dV += P^T dO and dK~ += dS^T Q~
//                in TMEM over the unit's rows; each key tile's sums leave by
//                vector reductions (red.global.add.v4.f32) into fp32 rows,
//                since a key is seen by many units.
//   k_bwd_finish dk = R_p^T dk~ in place at every key's position.
#include <cudaTypedefs.h>

#include "hga_internal.cuh"
#include "sm100.cuh"
#include "vec.cuh"
#include "visible.cuh"

namespace hga {

__device__ int g_bwd_error = 0;

namespace {

using namespace sm100;

constexpr int kDummy = 0x7fffffff;       // padding segment
constexpr int kMaxSeg = 2048;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

// Inverse rotation of the pair (x, y) by the angle whose (cos, sin) is cs.
__device__ __forceinline__ float2 unrot_pair(float x, float y, float2 cs) {
    return make_float2(fmaf(x, cs.x, y * cs.y), fmaf(y, cs.x, -x * cs.y));
}

// ------------------------------------------------------------------ prep --
// One thread per 8 rotate-half pairs of a query row (b, t, hq): 16-byte
// loads of the pairs' low and high halves; writes q~ (bf16, rounded exactly
// as the forward rounds its rotated queries) when qt is non-null.  The
// word's first thread also writes rowstat.x = LSE, to base 2 (times log2 e)
// for the tensor-core kernels, which exponentiate with ex2, natural for the
// CUDA-core kernel.  rowstat.y (Delta) is written by the main kernels' first
// pass.
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_bwd_prep(const T *__restrict__ q, const int32_t *__restrict__ pos,
           const float *__restrict__ lse, int Tlen, int Hq, long long rows, int log2_lse,
           __nv_bfloat16 *__restrict__ qt, float2 *__restrict__ rowstat, Rope rope) {
    constexpr int H = D / 2, W = H / 8;       // words of 8 pairs per row
    const long long x = (long long)blockIdx.x * 256 + threadIdx.x;
    if (x >= rows * W) return;
    const long long r = x / W;
    const int w = (int)(x % W);
    const long long bt = r / Hq;              // (b, t)
    const int hq = (int)(r % Hq);
    const long long b = bt / Tlen, t = bt % Tlen;
    if (qt) {
        float lo[8], hi[8];
        load_slice<T, 8>(q + r * D + w * 8, lo);
        load_slice<T, 8>(q + r * D + H + w * 8, hi);
        const int32_t p = pos[bt];
        uint4 ol, oh;
        __nv_bfloat162 *pl = reinterpret_cast<__nv_bfloat162 *>(&ol);
        __nv_bfloat162 *ph = reinterpret_cast<__nv_bfloat162 *>(&oh);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 r0 = rot_pair(lo[2 * e], hi[2 * e], rope_cs_int(rope, p, w * 8 + 2 * e));
            const float2 r1 =
                rot_pair(lo[2 * e + 1], hi[2 * e + 1], rope_cs_int(rope, p, w * 8 + 2 * e + 1));
            pl[e] = __floats2bfloat162_rn(r0.x, r1.x);
            ph[e] = __floats2bfloat162_rn(r0.y, r1.y);
        }
        reinterpret_cast<uint4 *>(qt + r * D)[w] = ol;
        reinterpret_cast<uint4 *>(qt + r * D + H)[w] = oh;
    }
    if (w == 0) {
        const float l = lse[(b * Hq + hq) * Tlen + t];
        rowstat[r] = make_float2(log2_lse ? l * kLog2e : l, 0.f);
    }
}

// ------------------------------------------------------------- finish --
// dk = R_p^T dk~ in place, one warp per key row (b, t, h).
template <int D>
__global__ void __launch_bounds__(256)
k_bwd_finish(const int32_t *__restrict__ pos, int Hkv, long long rows, float *__restrict__ dk,
             Rope rope) {
    constexpr int H = D / 2, PL = H / 32;
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int32_t p = pos[r / Hkv];
    float *row = dk + r * D;
#pragma unroll
    for (int e = 0; e < PL; ++e) {
        const int i = lane * PL + e;
        const float2 o = unrot_pair(row[i], row[i + H], rope_cs_int(rope, p, i));
        row[i] = o.x;
        row[i + H] = o.y;
    }
}

// ------------------------------------------------------ CUDA-core path --
// One CTA per (block, KV head, sequence); one warp per query row of the
// unit: the row's probabilities are recomputed from the forward's LSE, dq~
// accumulates in registers, and dk~ and dv accumulate into fp32 rows by
// atomic adds (a key is shared by many rows and units).
constexpr int kSimtThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_bwd_simt(const T *__restrict__ q, const int32_t *__restrict__ pos, int Tlen, int Hq, int Hkv,
           const T *__restrict__ k_rot, const T *__restrict__ v,
           const int32_t *__restrict__ sel_group, int NB, int F, int L, int K_g, int g_s,
           const float2 *__restrict__ rowstat, const T *__restrict__ dout,
           float *__restrict__ dq, float *__restrict__ dk_acc, float *__restrict__ dv, Rope rope,
           float scale) {
    // scale = 1/sqrt(D); rowstat.x = natural-log LSE
    constexpr int H = D / 2, PL = H / 32;     // pairs per lane: dims (i, i+H) of i = lane*PL+e
    extern __shared__ int keys[];
    __shared__ RunList rl;
    const int G = Hq / Hkv;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk, n_cur = min(kChunk, Tlen - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kSimtThreads / 32;
    if (threadIdx.x == 0)
        build_runs(rl, c, F, L, g_s, sel_group + (((int64_t)b * NB + c) * Hkv + h) * K_g, K_g,
                   n_cur);
    __syncthreads();
    fill_keys(rl, keys);
    __syncthreads();
    for (int R = warp; R < n_cur * G; R += nw) {
        const int tok = t0 + R / G, hq = h * G + R % G;
        const int64_t row = ((int64_t)b * Tlen + tok) * Hq + hq;
        const int32_t p = pos[(int64_t)b * Tlen + tok];
        float ql[PL], qh[PL], gl[PL], gh[PL], dl[PL], dh[PL];
#pragma unroll
        for (int e = 0; e < PL; ++e) {
            const int i = lane * PL + e;
            const float2 rr = rot_pair(to_f(q[row * D + i]), to_f(q[row * D + i + H]),
                                       rope_cs_int(rope, p, i));
            ql[e] = rr.x;
            qh[e] = rr.y;
            gl[e] = to_f(dout[row * D + i]);
            gh[e] = to_f(dout[row * D + i + H]);
            dl[e] = dh[e] = 0.f;
        }
        const float lse_i = rowstat[row].x;
        const int nvis = rl.cur_off + (tok - t0 + 1);
        // first pass: Delta = sum_j P_ij dO_i . v_j with this kernel's own P
        float delta = 0.f;
        for (int kk = 0; kk < nvis; ++kk) {
            const int j = keys[kk];
            const int64_t kr = (((int64_t)b * Tlen + j) * Hkv + h) * D;
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int e = 0; e < PL; ++e) {
                const int i = lane * PL + e;
                s = fmaf(ql[e], to_f(k_rot[kr + i]), fmaf(qh[e], to_f(k_rot[kr + i + H]), s));
                dp = fmaf(gl[e], to_f(v[kr + i]), fmaf(gh[e], to_f(v[kr + i + H]), dp));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                dp += __shfl_xor_sync(0xffffffffu, dp, o);
            }
            delta = fmaf(expf(fmaf(s, scale, -lse_i)), dp, delta);
        }
        for (int kk = 0; kk < nvis; ++kk) {
            const int j = keys[kk];
            const int64_t kr = (((int64_t)b * Tlen + j) * Hkv + h) * D;
            float kl[PL], kh[PL], vl[PL], vh[PL], s = 0.f, dp = 0.f;
#pragma unroll
            for (int e = 0; e < PL; ++e) {
                const int i = lane * PL + e;
                kl[e] = to_f(k_rot[kr + i]);
                kh[e] = to_f(k_rot[kr + i + H]);
                vl[e] = to_f(v[kr + i]);
                vh[e] = to_f(v[kr + i + H]);
                s = fmaf(ql[e], kl[e], fmaf(qh[e], kh[e], s));
                dp = fmaf(gl[e], vl[e], fmaf(gh[e], vh[e], dp));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                dp += __shfl_xor_sync(0xffffffffu, dp, o);
            }
            const float pr = expf(fmaf(s, scale, -lse_i));
            const float ds = pr * (dp - delta) * scale;
#pragma unroll
            for (int e = 0; e < PL; ++e) {
                const int i = lane * PL + e;
                dl[e] = fmaf(ds, kl[e], dl[e]);
                dh[e] = fmaf(ds, kh[e], dh[e]);
                atomicAdd(dk_acc + kr + i, ds * ql[e]);
                atomicAdd(dk_acc + kr + i + H, ds * qh[e]);
                atomicAdd(dv + kr + i, pr * gl[e]);
                atomicAdd(dv + kr + i + H, pr * gh[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < PL; ++e) {
            const int i = lane * PL + e;
            const float2 o = unrot_pair(dl[e], dh[e], rope_cs_int(rope, p, i));
            dq[row * D + i] = o.x;
            dq[row * D + i + H] = o.y;
        }
    }
}

// ------------------------------------------------ tensor-core kernels --

constexpr int kThreads = 384;
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsCtl = 56;
constexpr uint32_t kRegsSoftmax = 224;

struct BwdArgs {
    int T, Hq, Hkv, G, NB, F, L, K_g, g_s;
    int rows_per_unit, ctas_per_unit, tokM, tokS;
    const int32_t *sel_group;
    const int32_t *pos;
    float2 *rowstat;      // (LSE in base 2, Delta): Delta written by the dQ kernel
    float *dq, *dk, *dv;
    float scale_log2;     // log2(e) / sqrt(D)
    float inv_sqrt_d;
    Rope rope;
};

struct BwdCtl {
    uint64_t q_full[2], s_full[2], p_full[2], o_full[2];
    uint64_t kv_full[4], kv_empty[4], row_full[4], row_empty[4];
    uint64_t acc_done, acc_free, fin;
    uint32_t tmem_base;
    int nseg, first_cur, nkeys;
    volatile int abort;
    int seg_tok[kMaxSeg];
};

__device__ __forceinline__ void bwd_fail(BwdCtl &ctl) {
    ctl.abort = 1;
    atomicExch(&g_bwd_error, (int)HGA_ERR_TIMEOUT);
}

// The unit's visible set as 8-token segments (warp-wide): sinks, recent
// chunks, routed groups, then the current chunk up to token max_tok; padded
// to an even count with a dummy segment.  Returns through ctl.
__device__ __forceinline__ void build_segments(BwdCtl &ctl, const BwdArgs &A, int b, int c, int h,
                                               int max_tok) {
    const int lane = threadIdx.x & 31;
    const int t0 = c * kChunk;
    const int nsink = min(A.F, c);
    const int rec_lo = max(c - max(A.L, 1), nsink);
    const int n_fixed = 8 * (nsink + (c - rec_lo));
    for (int s = lane; s < n_fixed; s += 32)
        ctl.seg_tok[s] = s < 8 * nsink ? s * 8 : rec_lo * kChunk + (s - 8 * nsink) * 8;
    const int32_t *sel = A.sel_group + (((int64_t)b * A.NB + c) * A.Hkv + h) * A.K_g;
    const int gseg = A.g_s / 8;
    int kg = 0;
    for (int base = 0; base < A.K_g; base += 32) {
        const int v = base + lane < A.K_g ? sel[base + lane] : -1;
        kg += __popc(__ballot_sync(0xffffffffu, v >= 0));
    }
    for (int j = lane; j < kg; j += 32)
        for (int e = 0; e < gseg; ++e) ctl.seg_tok[n_fixed + j * gseg + e] = sel[j] * A.g_s + e * 8;
    const int n_route = n_fixed + kg * gseg;
    const int ncur = (max_tok - t0) / 8 + 1;
    for (int e = lane; e < ncur; e += 32) ctl.seg_tok[n_route + e] = t0 + e * 8;
    int nseg = n_route + ncur;
    if (lane == 0) {
        if (nseg & 1) ctl.seg_tok[nseg++] = kDummy;
        ctl.nseg = nseg;
        ctl.first_cur = n_route;
        ctl.nkeys = n_route * 8 + (max_tok - t0 + 1);
    }
}

// Loads nsj segments (8 key rows each) of one tensor into a 128B-swizzled
// tile whose D-halves are half_bytes apart; runs of 8 or 2 consecutive
// segments go as one 64- or 16-row box.
__device__ __forceinline__ void load_segments(uint8_t *tile, uint32_t half_bytes, int halves,
                                              const int *sg, int nsj, const CUtensorMap *m8,
                                              const CUtensorMap *m16, const CUtensorMap *m64,
                                              uint64_t *bar, int h, int zbase, uint64_t policy) {
    for (int e = 0; e < nsj;) {
        const int st = sg[e];
        int run = 1;
        if (st != kDummy) {
            if ((e & 7) == 0 && e + 8 <= nsj) {
                run = 8;
                for (int i = 1; i < 8; ++i)
                    if (sg[e + i] != st + 8 * i) { run = 1; break; }
            }
            if (run == 1 && (e & 1) == 0 && e + 2 <= nsj && sg[e + 1] == st + 8) run = 2;
        }
        const CUtensorMap *m = run == 8 ? m64 : (run == 2 ? m16 : m8);
        const int z = zbase + (st == kDummy ? 0 : st);
        for (int hf = 0; hf < halves; ++hf)
            tma_load_3d_hint(tile + hf * half_bytes + e * 1024, m, bar, hf * 64, h, z, policy);
        e += run;
    }
}

// ---- dQ: query-major -------------------------------------------------------

template <int D>
struct DqCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kSegPerTile = 8;                  // 64 keys
    static constexpr int kStages = 2;
    static constexpr uint32_t kQHalf = 128 * 128;          // 128 rows x 128 B
    static constexpr uint32_t kQTile = kHalves * kQHalf;
    static constexpr uint32_t kKHalf = 64 * 128;           // 64 keys x 128 B
    static constexpr uint32_t kKTile = kHalves * kKHalf;
    static constexpr uint32_t oQ = 0;
    static constexpr uint32_t oG = oQ + 2 * kQTile;        // dO tiles
    static constexpr uint32_t oK = oG + 2 * kQTile;
    static constexpr uint32_t oV = oK + kStages * kKTile;
    static constexpr uint32_t oEnd = oV + kStages * kKTile;
};

// TMEM per M-tile mt (256 columns): S at mt*256 (64), dP at +64 (64), dQ~ at
// +128 (D).  dS (bf16) is written over the S columns.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dq_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
            const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
            const __grid_constant__ CUtensorMap tmK16, const __grid_constant__ CUtensorMap tmV16,
            const __grid_constant__ CUtensorMap tmK64, const __grid_constant__ CUtensorMap tmV64,
            const BwdArgs A) {
    using C = DqCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ BwdCtl ctl;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x / A.ctas_per_unit, cu = blockIdx.x % A.ctas_per_unit;
    const int h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk;
    const int row0 = cu * 256;
    const int rows = min(256, A.rows_per_unit - row0);
    const int NT = (rows + 127) >> 7;
    const int max_tok = min(t0 + (row0 + rows - 1) / A.G, A.T - 1);

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl.q_full[i], 1);
            mbar_init(&ctl.s_full[i], 1);
            mbar_init(&ctl.p_full[i], 128);
            mbar_init(&ctl.o_full[i], 1);
        }
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&ctl.kv_full[i], 1);
            mbar_init(&ctl.kv_empty[i], 1);
        }
        mbar_init(&ctl.fin, 1);
        ctl.abort = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmG);
        // this CTA's query rows are read once: they should not push the
        // gathered K and V (read twice by every unit that sees them) out of L2
        const uint64_t once = l2_policy_evict_first();
        for (int mt = 0; mt < NT; ++mt) {
            const int tok_first = t0 + (row0 + mt * 128) / A.G;
            mbar_arrive_expect_tx(&ctl.q_full[mt], (uint32_t)(2 * A.G * A.tokM * D * 2));
            for (int hf = 0; hf < C::kHalves; ++hf) {
                tma_load_3d_hint(smem + C::oQ + mt * C::kQTile + hf * C::kQHalf, &tmQ,
                                 &ctl.q_full[mt], hf * 64, h * A.G, b * A.T + tok_first, once);
                tma_load_3d_hint(smem + C::oG + mt * C::kQTile + hf * C::kQHalf, &tmG,
                                 &ctl.q_full[mt], hf * 64, h * A.G, b * A.T + tok_first, once);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, 512);
        tc_fence_before();
    }
    if (warp == 2) build_segments(ctl, A, b, c, h, max_tok);
    __syncthreads();
    tc_fence_after();
    static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
    const uint32_t tmem = ctl.tmem_base;
    const int nseg = ctl.nseg;
    const int ntiles = (nseg + C::kSegPerTile - 1) / C::kSegPerTile;
    const int first_cur = ctl.first_cur;

    if (warp < 4) {
        regs_dec<kRegsCtl>();
        if (warp == 0 && lane == 0) {
            // ---- producer: K~ and V tiles of 64 keys into a 2-stage ring
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            prefetch_tensormap(&tmK16);
            prefetch_tensormap(&tmV16);
            prefetch_tensormap(&tmK64);
            prefetch_tensormap(&tmV64);
            // every tile twice: the Delta pass, then the dS / dQ pass
            const uint64_t keep = l2_policy_evict_last();
            for (int t = 0; t < 2 * ntiles && !ctl.abort; ++t) {
                const int j = t % ntiles, s = t % C::kStages;
                if (t >= C::kStages && !mbar_wait(&ctl.kv_empty[s], ((t / C::kStages) - 1) & 1)) {
                    bwd_fail(ctl);
                    break;
                }
                const int nsj = min(C::kSegPerTile, nseg - j * C::kSegPerTile);
                mbar_arrive_expect_tx(&ctl.kv_full[s], (uint32_t)(2 * nsj * 8 * D * 2));
                const int *sg = ctl.seg_tok + j * C::kSegPerTile;
                load_segments(smem + C::oK + s * C::kKTile, C::kKHalf, C::kHalves, sg, nsj, &tmK,
                              &tmK16, &tmK64, &ctl.kv_full[s], h, b * A.T, keep);
                load_segments(smem + C::oV + s * C::kKTile, C::kKHalf, C::kHalves, sg, nsj, &tmV,
                              &tmV16, &tmV64, &ctl.kv_full[s], h, b * A.T, keep);
            }
        } else if (warp == 1 && lane == 0) {
            // ---- MMA issuer
            const uint32_t idesc_dq = idesc_bf16_f32(128, D, false, true);
            bool ok = true;
            for (int mt = 0; mt < NT && ok; ++mt) ok = mbar_wait(&ctl.q_full[mt], 0);
            tc_fence_after();
            // step t < ntiles: the Delta pass over tile t; t >= ntiles: the
            // dS / dQ pass over tile t - ntiles
            const int T2 = 2 * ntiles;
            for (int t = 0; t <= T2 && ok; ++t) {
                const int s = t % C::kStages;
                const int j = t % ntiles;
                for (int mt = 0; mt < NT && ok; ++mt) {
                    if (t > 0) {
                        if (!(ok = mbar_wait(&ctl.p_full[mt], (t - 1) & 1))) break;
                        tc_fence_after();
                        if (t - 1 >= ntiles) {
                            // dQ~ += dS K~ of the previous tile: A from TMEM,
                            // K~ as an MN-major B
                            const int jp = (t - 1) - ntiles;
                            const int sp = (t - 1) % C::kStages;
                            const int nsj = min(C::kSegPerTile, nseg - jp * C::kSegPerTile);
                            const uint32_t kbase = smem_addr(smem + C::oK + sp * C::kKTile);
                            for (int ks = 0; ks < nsj / 2; ++ks)
                                mma_ts(tmem + mt * 256 + 128, tmem + mt * 256 + ks * 8,
                                       smem_desc_sw128(kbase + ks * 2048, C::kKHalf, 1024),
                                       idesc_dq, (jp > 0 || ks > 0) ? 1u : 0u);
                            if (t == T2) mma_commit(&ctl.o_full[mt]);
                            else if (mt == NT - 1) mma_commit(&ctl.kv_empty[sp]);
                        }
                    }
                    if (t < T2) {
                        if (mt == 0) {
                            if (!(ok = mbar_wait(&ctl.kv_full[s], (t / C::kStages) & 1))) break;
                            tc_fence_after();
                        }
                        const int nsj = min(C::kSegPerTile, nseg - j * C::kSegPerTile);
                        const uint32_t idesc = idesc_bf16_f32(128, nsj * 8, false, false);
                        const uint32_t qb = smem_addr(smem + C::oQ + mt * C::kQTile);
                        const uint32_t gb = smem_addr(smem + C::oG + mt * C::kQTile);
                        const uint32_t kb = smem_addr(smem + C::oK + s * C::kKTile);
                        const uint32_t vb = smem_addr(smem + C::oV + s * C::kKTile);
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t oa = (kk >> 2) * C::kQHalf + (kk & 3) * 32;
                            const uint32_t ob = (kk >> 2) * C::kKHalf + (kk & 3) * 32;
                            mma_ss(tmem + mt * 256, smem_desc_sw128(qb + oa, 16, 1024),
                                   smem_desc_sw128(kb + ob, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                        }
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t oa = (kk >> 2) * C::kQHalf + (kk & 3) * 32;
                            const uint32_t ob = (kk >> 2) * C::kKHalf + (kk & 3) * 32;
                            mma_ss(tmem + mt * 256 + 64, smem_desc_sw128(gb + oa, 16, 1024),
                                   smem_desc_sw128(vb + ob, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&ctl.s_full[mt]);
                        // a Delta-pass tile is done with its stage once S and dP are
                        if (t < ntiles && mt == NT - 1) mma_commit(&ctl.kv_empty[s]);
                    }
                }
            }
            if (!ok) bwd_fail(ctl);
            mma_commit(&ctl.fin);
            if (!mbar_wait(&ctl.fin, 0)) bwd_fail(ctl);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // ---- softmax warpgroups: thread = TMEM lane = query row
        const int mt = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const int R = row0 + mt * 128 + r;
        const int tok = t0 + R / A.G;
        const int head = R % A.G;
        const bool valid = mt < NT && (mt * 128 + r) < rows && tok < A.T;
        const int64_t grow = ((int64_t)b * A.T + tok) * A.Hq + (int64_t)h * A.G + head;
        const float lse2 = valid ? A.rowstat[grow].x : 0.f;
        const int nvis = valid ? first_cur * 8 + (tok - t0 + 1) : 0;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16) + mt * 256;
        const float sc = A.scale_log2, isd = A.inv_sqrt_d;
        bool ok = true;
        if (mt < NT) {
            float delta = 0.f;
            for (int t = 0; t < 2 * ntiles && ok; ++t) {
                if (!(ok = mbar_wait(&ctl.s_full[mt], t & 1))) {
                    bwd_fail(ctl);
                    break;
                }
                tc_fence_after();
                uint32_t sv[64], dp[64];
                tmem_ld32(lane_base + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(lane_base + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_ld32(lane_base + 64, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
                tmem_ld32(lane_base + 96, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
                tmem_ld_wait();
                const int gc0 = (t % ntiles) * C::kSegPerTile * 8;
                if (gc0 + 64 > nvis) {
                    // the row's visible keys end inside this tile: the later
                    // columns (and any past the tile's keys, which hold stale
                    // values) get P = 0 and dP = 0, with no per-column branch
#pragma unroll
                    for (int col = 0; col < 64; ++col)
                        if (gc0 + col >= nvis) {
                            sv[col] = __float_as_uint(-INFINITY);
                            dp[col] = 0u;
                        }
                }
                // pairs of columns in packed two-lane fp32: x = s * scale - LSE
                const uint64_t sc2 = f2_pack(sc, sc), nl2 = f2_pack(-lse2, -lse2);
                if (t < ntiles) {
                    // Delta pass: sum of P dP over the row's visible keys
                    uint64_t d4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) d4[u] = f2_pack(0.f, 0.f);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float2 x = f2_unpack(f2_fma(
                            f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2, nl2));
                        d4[e & 3] = f2_fma(f2_pack(ex2(x.x), ex2(x.y)),
                                           f2_pack(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])),
                                           d4[e & 3]);
                    }
                    const float2 da = f2_unpack(f2_add(d4[0], d4[1])), db = f2_unpack(f2_add(d4[2], d4[3]));
                    delta += (da.x + da.y) + (db.x + db.y);
                    if (t == ntiles - 1 && valid) A.rowstat[grow].y = delta;
                } else {
                    const uint64_t nd2 = f2_pack(-delta, -delta), is2 = f2_pack(isd, isd);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float2 x = f2_unpack(f2_fma(
                            f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2, nl2));
                        const float2 ds = f2_unpack(f2_mul(
                            f2_mul(f2_pack(ex2(x.x), ex2(x.y)),
                                   f2_add(f2_pack(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])), nd2)),
                            is2));
                        sv[e] = pack_bf16(ds.x, ds.y);
                    }
                    tmem_st32(lane_base + 0, *reinterpret_cast<const uint32_t(*)[32]>(&sv[0]));
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(&ctl.p_full[mt]);
            }
            // epilogue: dq = R_p^T dQ~ (fp32 row)
            if (ok && !mbar_wait(&ctl.o_full[mt], 0)) {
                bwd_fail(ctl);
                ok = false;
            }
            tc_fence_after();
            if (ok) {
                const int32_t p = valid ? A.pos[(int64_t)b * A.T + tok] : 0;
                float *dqrow = A.dq + grow * D;
                constexpr int H = D / 2;
                for (int cb = 0; cb < H / 32; ++cb) {
                    uint32_t lo[32], hi[32];
                    tmem_ld32(lane_base + 128 + cb * 32, lo);
                    tmem_ld32(lane_base + 128 + H + cb * 32, hi);
                    tmem_ld_wait();
                    if (valid) {
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            float a[4], bb[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int e = e4 * 4 + u;
                                const float2 o = unrot_pair(__uint_as_float(lo[e]), __uint_as_float(hi[e]),
                                                            rope_cs_int(A.rope, p, cb * 32 + e));
                                a[u] = o.x;
                                bb[u] = o.y;
                            }
                            __stcs(reinterpret_cast<float4 *>(dqrow + cb * 32) + e4,
                                   make_float4(a[0], a[1], a[2], a[3]));
                            __stcs(reinterpret_cast<float4 *>(dqrow + H + cb * 32) + e4,
                                   make_float4(bb[0], bb[1], bb[2], bb[3]));
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- dK, dV: key-major inside a unit ----------------------------------------

template <int D>
struct DkvCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kSegPerTile = 16;                 // 128 keys
    static constexpr int kRowStages = 4;
    static constexpr uint32_t kKHalf = 128 * 128;          // 128 keys x 128 B
    static constexpr uint32_t kKTile = kHalves * kKHalf;
    static constexpr uint32_t kRHalf = 64 * 128;           // 64 rows x 128 B
    static constexpr uint32_t kRTile = kHalves * kRHalf;
    static constexpr uint32_t oK = 0;
    static constexpr uint32_t oV = oK + kKTile;
    static constexpr uint32_t oQ = oV + kKTile;            // row stages: q~ then dO
    static constexpr uint32_t oG = oQ + kRowStages * kRTile;
    static constexpr uint32_t oStat = oG + kRowStages * kRTile;   // float2 per unit row
};

// TMEM: buffer bb (0, 1) holds S^T at bb*128 (64 columns: the subtile's
// rows) and dP^T at bb*128 + 64; P^T and dS^T (bf16) are written over them.
// dV at 256 (D columns), dK~ at 384.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dkv_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
             const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
             const __grid_constant__ CUtensorMap tmK16, const __grid_constant__ CUtensorMap tmV16,
             const __grid_constant__ CUtensorMap tmK64, const __grid_constant__ CUtensorMap tmV64,
             const BwdArgs A) {
    using C = DkvCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ BwdCtl ctl;
    float2 *stat = reinterpret_cast<float2 *>(smem + C::oStat);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk;
    const int max_tok = min(t0 + kChunk - 1, A.T - 1);
    const int nrows = (max_tok - t0 + 1) * A.G;           // valid rows of the unit
    const int nsub = (nrows + 63) >> 6;                   // 64-row subtiles

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl.s_full[i], 1);
            mbar_init(&ctl.p_full[i], 128);
        }
        mbar_init(&ctl.kv_full[0], 1);
        mbar_init(&ctl.kv_empty[0], 1);
        for (int i = 0; i < C::kRowStages; ++i) {
            mbar_init(&ctl.row_full[i], 1);
            mbar_init(&ctl.row_empty[i], 1);
        }
        mbar_init(&ctl.acc_done, 1);
        mbar_init(&ctl.acc_free, 256);
        mbar_init(&ctl.fin, 1);
        ctl.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, 512);
        tc_fence_before();
    }
    if (warp == 2) build_segments(ctl, A, b, c, h, max_tok);
    if (warp == 3) {
        // (-LSE * log2 e, -Delta) of every row of the unit (negated: they
        // are added below); rows past the end of the sequence get -inf, so
        // their probabilities are zero
        for (int R = lane; R < nsub * 64; R += 32) {
            const int tok = t0 + R / A.G;
            float2 st = make_float2(-INFINITY, 0.f);
            if (R < nrows) {
                st = A.rowstat[((int64_t)b * A.T + tok) * A.Hq + (int64_t)h * A.G + R % A.G];
                st = make_float2(-st.x, -st.y);
            }
            stat[R] = st;
        }
    }
    __syncthreads();
    tc_fence_after();
    static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
    const uint32_t tmem = ctl.tmem_base;
    const int nseg = ctl.nseg;
    const int ntiles = (nseg + C::kSegPerTile - 1) / C::kSegPerTile;
    const int first_cur = ctl.first_cur;
    const int nkeys = ctl.nkeys;
    const int nsteps = ntiles * nsub;

    if (warp < 4) {
        regs_dec<kRegsCtl>();
        if (warp == 0 && lane == 0) {
            // ---- producer: one K~ and V tile of 128 keys (single stage)
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            prefetch_tensormap(&tmK16);
            prefetch_tensormap(&tmV16);
            prefetch_tensormap(&tmK64);
            prefetch_tensormap(&tmV64);
            const uint64_t keep = l2_policy_evict_last();   // other units read these keys too
            for (int j = 0; j < ntiles && !ctl.abort; ++j) {
                if (j > 0 && !mbar_wait(&ctl.kv_empty[0], (j - 1) & 1)) {
                    bwd_fail(ctl);
                    break;
                }
                const int nsj = min(C::kSegPerTile, nseg - j * C::kSegPerTile);
                mbar_arrive_expect_tx(&ctl.kv_full[0], (uint32_t)(2 * nsj * 8 * D * 2));
                const int *sg = ctl.seg_tok + j * C::kSegPerTile;
                load_segments(smem + C::oK, C::kKHalf, C::kHalves, sg, nsj, &tmK, &tmK16, &tmK64,
                              &ctl.kv_full[0], h, b * A.T, keep);
                load_segments(smem + C::oV, C::kKHalf, C::kHalves, sg, nsj, &tmV, &tmV16, &tmV64,
                              &ctl.kv_full[0], h, b * A.T, keep);
            }
        } else if (warp == 2 && lane == 0) {
            // ---- producer: q~ and dO row subtiles of 64 rows, re-streamed per key tile
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmG);
            // the unit's query rows are re-read once per key tile
            const uint64_t keep = l2_policy_evict_last();
            for (int n = 0; n < nsteps && !ctl.abort; ++n) {
                const int s = n % C::kRowStages;
                if (n >= C::kRowStages &&
                    !mbar_wait(&ctl.row_empty[s], ((n / C::kRowStages) - 1) & 1)) {
                    bwd_fail(ctl);
                    break;
                }
                const int i = n % nsub;
                const int tok_first = t0 + i * A.tokS;
                mbar_arrive_expect_tx(&ctl.row_full[s], (uint32_t)(2 * A.G * A.tokS * D * 2));
                for (int hf = 0; hf < C::kHalves; ++hf) {
                    tma_load_3d_hint(smem + C::oQ + s * C::kRTile + hf * C::kRHalf, &tmQ,
                                     &ctl.row_full[s], hf * 64, h * A.G, b * A.T + tok_first, keep);
                    tma_load_3d_hint(smem + C::oG + s * C::kRTile + hf * C::kRHalf, &tmG,
                                     &ctl.row_full[s], hf * 64, h * A.G, b * A.T + tok_first, keep);
                }
            }
        } else if (warp == 1 && lane == 0) {
            // ---- MMA issuer.  Step n: S^T and dP^T of subtile n, then dV and
            // dK~ of subtile n-1 (whose P^T / dS^T the softmax has written)
            const uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
            const uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
            bool ok = true;
            for (int n = 0; n <= nsteps && ok; ++n) {
                if (n < nsteps) {
                    const int j = n / nsub, i = n % nsub, bb = n & 1, s = n % C::kRowStages;
                    if (i == 0) {
                        if (!(ok = mbar_wait(&ctl.kv_full[0], j & 1))) break;
                    }
                    if (!(ok = mbar_wait(&ctl.row_full[s], (n / C::kRowStages) & 1))) break;
                    tc_fence_after();
                    const uint32_t kb = smem_addr(smem + C::oK), vb = smem_addr(smem + C::oV);
                    const uint32_t qb = smem_addr(smem + C::oQ + s * C::kRTile);
                    const uint32_t gb = smem_addr(smem + C::oG + s * C::kRTile);
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * C::kKHalf + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * C::kRHalf + (kk & 3) * 32;
                        mma_ss(tmem + bb * 128, smem_desc_sw128(kb + oa, 16, 1024),
                               smem_desc_sw128(qb + ob, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * C::kKHalf + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * C::kRHalf + (kk & 3) * 32;
                        mma_ss(tmem + bb * 128 + 64, smem_desc_sw128(vb + oa, 16, 1024),
                               smem_desc_sw128(gb + ob, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&ctl.s_full[bb]);
                    if (i == nsub - 1) mma_commit(&ctl.kv_empty[0]);
                }
                if (n >= 1) {
                    const int m = n - 1;
                    const int jm = m / nsub, im = m % nsub, bm = m & 1, sm = m % C::kRowStages;
                    if (!(ok = mbar_wait(&ctl.p_full[bm], (m >> 1) & 1))) break;
                    if (im == 0 && jm > 0) {
                        if (!(ok = mbar_wait(&ctl.acc_free, (jm - 1) & 1))) break;
                    }
                    tc_fence_after();
                    const uint32_t qb = smem_addr(smem + C::oQ + sm * C::kRTile);
                    const uint32_t gb = smem_addr(smem + C::oG + sm * C::kRTile);
                    for (int ks = 0; ks < 4; ++ks) {      // 64 rows, 16 per product
                        mma_ts(tmem + 256, tmem + bm * 128 + ks * 8,
                               smem_desc_sw128(gb + ks * 2048, C::kRHalf, 1024), idesc_acc,
                               (im > 0 || ks > 0) ? 1u : 0u);
                        mma_ts(tmem + 384, tmem + bm * 128 + 64 + ks * 8,
                               smem_desc_sw128(qb + ks * 2048, C::kRHalf, 1024), idesc_acc,
                               (im > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(&ctl.row_empty[sm]);
                    if (im == nsub - 1) mma_commit(&ctl.acc_done);
                }
            }
            if (!ok) bwd_fail(ctl);
            mma_commit(&ctl.fin);
            if (!mbar_wait(&ctl.fin, 0)) bwd_fail(ctl);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // ---- two warpgroups, alternating subtiles; thread = TMEM lane = key
        const int wg = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int kl = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const float sc = A.scale_log2, isd = A.inv_sqrt_d;
        bool ok = true;
        for (int j = 0; j < ntiles && ok; ++j) {
            const int kidx = j * C::kSegPerTile * 8 + kl;
            // rows R see this key iff R >= rmin (the causal part of the
            // current chunk); keys past the last real one are seen by none
            const int rmin = kidx >= nkeys ? 1 << 30
                           : (kidx < first_cur * 8 ? 0 : (kidx - first_cur * 8) * A.G);
            for (int i = 0; i < nsub && ok; ++i) {
                const int n = j * nsub + i;
                if ((n & 1) != wg) continue;
                const int bb = n & 1;
                if (!(ok = mbar_wait(&ctl.s_full[bb], (n >> 1) & 1))) {
                    bwd_fail(ctl);
                    break;
                }
                tc_fence_after();
                const uint32_t base = tmem + lane_off + bb * 128;
                uint32_t sv[64], dp[64];
                tmem_ld32(base + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(base + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_ld32(base + 64, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
                tmem_ld32(base + 96, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
                tmem_ld_wait();
                const int R0 = i * 64;
                if (R0 < rmin) {
                    // rows before rmin do not see this key (and keys past the
                    // last real one are seen by none): their entries get
                    // P = 0 and dS = 0 whatever the tile's unused rows hold
#pragma unroll
                    for (int col = 0; col < 64; ++col)
                        if (R0 + col < rmin) {
                            sv[col] = __float_as_uint(-INFINITY);
                            dp[col] = 0u;
                        }
                }
                const float4 *st4 = reinterpret_cast<const float4 *>(stat + R0);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float4 st = st4[e];           // (-lse, -delta) of rows R0 + 2e, + 1
                    const float p0 = ex2(fmaf(__uint_as_float(sv[2 * e]), sc, st.x));
                    const float p1 = ex2(fmaf(__uint_as_float(sv[2 * e + 1]), sc, st.z));
                    const float d0 = p0 * (__uint_as_float(dp[2 * e]) + st.y) * isd;
                    const float d1 = p1 * (__uint_as_float(dp[2 * e + 1]) + st.w) * isd;
                    sv[e] = pack_bf16(p0, p1);
                    dp[e] = pack_bf16(d0, d1);
                }
                tmem_st32(base + 0, *reinterpret_cast<const uint32_t(*)[32]>(&sv[0]));
                tmem_st32(base + 64, *reinterpret_cast<const uint32_t(*)[32]>(&dp[0]));
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&ctl.p_full[bb]);
            }
            if (!ok) break;
            // epilogue of key tile j: warpgroup 0 adds dV, warpgroup 1 dK~
            if (!(ok = mbar_wait(&ctl.acc_done, j & 1))) {
                bwd_fail(ctl);
                break;
            }
            tc_fence_after();
            // the key's row (keys past the last real one, and padding, have none)
            int tok = -1;
            if (kidx < nkeys) {
                const int sgt = ctl.seg_tok[kidx >> 3];
                if (sgt != kDummy) tok = sgt + (kidx & 7);
            }
            float *dst = tok >= 0
                ? (wg == 0 ? A.dv : A.dk) + (((int64_t)b * A.T + tok) * A.Hkv + h) * D : nullptr;
            const uint32_t acc = tmem + lane_off + (wg == 0 ? 256 : 384);
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t v[32];
                tmem_ld32(acc + cb * 32, v);
                tmem_ld_wait();
                if (dst) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4)
                        red_add_v4(dst + cb * 32 + e4 * 4, __uint_as_float(v[e4 * 4]),
                                   __uint_as_float(v[e4 * 4 + 1]), __uint_as_float(v[e4 * 4 + 2]),
                                   __uint_as_float(v[e4 * 4 + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(&ctl.acc_free);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3-D bf16 map over rows of [n_rows][heads][D]: box (64, box_heads,
// box_rows), 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap *m, const void *base, int D, int heads, long long n_rows, int box_heads,
              int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)n_rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
hga_status run_tc(const Geo &g, const Rope &r, const __nv_bfloat16 *qt, const int32_t *pos,
                  const void *k_rot, const void *v, const int32_t *sel_group,
                  float2 *rowstat, const void *dout, float *dq, float *dk, float *dv,
                  cudaStream_t st) {
    BwdArgs a;
    a.T = g.T;
    a.Hq = g.Hq;
    a.Hkv = g.Hkv;
    a.G = g.G;
    a.NB = g.NB;
    a.F = g.F;
    a.L = g.L;
    a.K_g = g.K_g;
    a.g_s = g.g_s;
    a.rows_per_unit = kChunk * g.G;
    a.ctas_per_unit = (a.rows_per_unit + 255) / 256;
    a.tokM = min(128, kChunk * g.G) / g.G;
    a.tokS = 64 / g.G;
    a.sel_group = sel_group;
    a.pos = pos;
    a.rowstat = rowstat;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    a.inv_sqrt_d = (float)(1.0 / sqrt((double)D));
    a.rope = r;
    const long long qrows = (long long)g.B * g.T, krows = (long long)g.B * g.T;
    CUtensorMap mq, mg, mqs, mgs, mk, mv, mk16, mv16, mk64, mv64;
    if (!make_map(&mq, qt, D, g.Hq, qrows, g.G, a.tokM) ||
        !make_map(&mg, dout, D, g.Hq, qrows, g.G, a.tokM) ||
        !make_map(&mqs, qt, D, g.Hq, qrows, g.G, a.tokS) ||
        !make_map(&mgs, dout, D, g.Hq, qrows, g.G, a.tokS) ||
        !make_map(&mk, k_rot, D, g.Hkv, krows, 1, 8) || !make_map(&mv, v, D, g.Hkv, krows, 1, 8) ||
        !make_map(&mk16, k_rot, D, g.Hkv, krows, 1, 16) ||
        !make_map(&mv16, v, D, g.Hkv, krows, 1, 16) ||
        !make_map(&mk64, k_rot, D, g.Hkv, krows, 1, 64) ||
        !make_map(&mv64, v, D, g.Hkv, krows, 1, 64))
        return HGA_ERR_CUDA;
    {
        const size_t smem = DqCfg<D>::oEnd + 1024;
        auto kern = k_bwd_dq_tc<D>;
        cudaError_t e = ensure_smem((const void *)kern, smem);
        if (e != cudaSuccess) return cuda_status(e);
        dim3 grid(g.NB * a.ctas_per_unit, g.Hkv, g.B);
        kern<<<grid, kThreads, smem, st>>>(mq, mg, mk, mv, mk16, mv16, mk64, mv64, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    }
    {
        const int max_rows = ((kChunk * g.G + 63) / 64) * 64;
        const size_t smem = DkvCfg<D>::oStat + sizeof(float2) * (size_t)max_rows + 1024;
        auto kern = k_bwd_dkv_tc<D>;
        cudaError_t e = ensure_smem((const void *)kern, smem);
        if (e != cudaSuccess) return cuda_status(e);
        dim3 grid(g.NB, g.Hkv, g.B);
        kern<<<grid, kThreads, smem, st>>>(mqs, mgs, mk, mv, mk16, mv16, mk64, mv64, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    }
    return HGA_OK;
}

template <typename T, int D>
hga_status run_simt(const Geo &g, const Rope &r, const void *q, const int32_t *pos,
                    const void *k_rot, const void *v, const int32_t *sel_group,
                    const float2 *rowstat, const void *dout, float *dq, float *dk, float *dv,
                    cudaStream_t st) {
    const size_t nk = (size_t)(g.F + max(g.L, 1) + 1) * kChunk + (size_t)g.K_g * g.g_s;
    const size_t smem = sizeof(int) * nk;
    auto kern = k_bwd_simt<T, D>;
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    kern<<<dim3(g.NB, g.Hkv, g.B), kSimtThreads, smem, st>>>(
        static_cast<const T *>(q), pos, g.T, g.Hq, g.Hkv, static_cast<const T *>(k_rot),
        static_cast<const T *>(v), sel_group, g.NB, g.F, g.L, g.K_g, g.g_s, rowstat,
        static_cast<const T *>(dout), dq, dk, dv, r, (float)(1.0 / sqrt((double)D)));
    return cuda_status(cudaGetLastError());
}

template <typename T, int D>
hga_status run_all(const Geo &g, const Rope &r, bool tc, const void *q, const int32_t *pos,
                   const void *k_rot, const void *v, const int32_t *sel_group,
                   const float *lse, const void *dout, float *dq, float *dk, float *dv, void *ws,
                   const void *q_rot, cudaStream_t st) {
    const long long qrows = (long long)g.B * g.T * g.Hq, krows = (long long)g.B * g.T * g.Hkv;
    char *w = static_cast<char *>(ws);
    float2 *rowstat = reinterpret_cast<float2 *>(w);
    // the rotated queries: the caller's (the forward's routing wrote them),
    // else rotated here into the workspace
    __nv_bfloat16 *qt = tc && !q_rot ? reinterpret_cast<__nv_bfloat16 *>(
                                           w + ((sizeof(float2) * qrows + 255) & ~(size_t)255))
                                     : nullptr;
    cudaError_t e = cudaMemsetAsync(dk, 0, sizeof(float) * krows * D, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, sizeof(float) * krows * D, st);
    if (e != cudaSuccess) return cuda_status(e);
    constexpr int W = D / 16;
    k_bwd_prep<T, D><<<(unsigned)((qrows * W + 255) / 256), 256, 0, st>>>(
        static_cast<const T *>(q), pos, lse, g.T, g.Hq, qrows, tc ? 1 : 0, qt, rowstat, r);
    if (tc && q_rot) qt = const_cast<__nv_bfloat16 *>(static_cast<const __nv_bfloat16 *>(q_rot));
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    hga_status s;
    if constexpr (sizeof(T) == 2) {
        s = tc ? run_tc<D>(g, r, qt, pos, k_rot, v, sel_group, rowstat, dout, dq, dk, dv, st)
               : run_simt<T, D>(g, r, q, pos, k_rot, v, sel_group, rowstat, dout, dq, dk, dv, st);
    } else {
        s = run_simt<T, D>(g, r, q, pos, k_rot, v, sel_group, rowstat, dout, dq, dk, dv, st);
    }
    if (s != HGA_OK) return s;
    k_bwd_finish<D><<<(unsigned)((krows + 7) / 8), 256, 0, st>>>(pos, g.Hkv, krows, dk, r);
    return cuda_status(cudaGetLastError());
}

}  // namespace

size_t backward_workspace_bytes(const Geo &g, int dtype) {
    const size_t qrows = (size_t)g.B * g.T * g.Hq;
    size_t n = (sizeof(float2) * qrows + 255) & ~(size_t)255;
    if (dtype == HGA_BF16 && attend_tc_supported(g, dtype))
        n += (qrows * g.D * 2 + 255) & ~(size_t)255;
    return n;
}

hga_status launch_attend_backward(const Geo &g, const Rope &r, int dtype, const void *q,
                                  const int32_t *pos, const void *k_rot, const void *v,
                                  const int32_t *sel_group, const float *lse,
                                  const void *dout, float *dq, float *dk, float *dv, void *ws,
                                  const void *q_rot, cudaStream_t st) {
    if (g.NB <= 0) return HGA_OK;
    const bool tc = dtype == HGA_BF16 && attend_tc_supported(g, dtype);
    if (dtype == HGA_BF16)
        return g.D == 128 ? run_all<__nv_bfloat16, 128>(g, r, tc, q, pos, k_rot, v, sel_group,
                                                        lse, dout, dq, dk, dv, ws, q_rot, st)
                          : run_all<__nv_bfloat16, 64>(g, r, tc, q, pos, k_rot, v, sel_group,
                                                       lse, dout, dq, dk, dv, ws, q_rot, st);
    return g.D == 128 ? run_all<float, 128>(g, r, false, q, pos, k_rot, v, sel_group, lse,
                                            dout, dq, dk, dv, ws, q_rot, st)
                      : run_all<float, 64>(g, r, false, q, pos, k_rot, v, sel_group, lse,
                                           dout, dq, dk, dv, ws, q_rot, st);
}

hga_status backward_error_take(cudaStream_t st, bool clear) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_bwd_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_bwd_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    return (hga_status)v;
}

}  // namespace hga
