// Stage 3 on the 5th-generation tensor cores (sm_100a, bf16): exact softmax
// attention over the routed token set of each 64-token query block.
//
// Method: HGA paper-review page, section 3, exact token output attention with
// eq. (1): the block's queries attend, with scale 1/sqrt(D), to the sink
// chunks, the recent chunks, the previous chunk, the routed groups and the
// causal part of their own chunk, and nothing else.
//
// Design.  One CTA owns up to 256 query rows of one (block, KV head) unit
// (rows ordered token-major, head-minor, so the G query heads of a KV head
// share every key tile) as two 128-row M-tiles.  The unit's visible set is a
// list of 8-token segments; 16 segments make one 128-key tile.
//   warp 0      TMA producer: both Q tiles once, then per key tile one
//               8x64-element box per segment and D-half for K and for V, into
//               128-byte-swizzled shared memory (a 2- or 4-stage ring).
//   warp 1      TMEM owner and MMA issuer (one thread): S = Q K^T into TMEM
//               (SS form), then O += P V with P read from TMEM (TS form).
//   warps 2-3   build the segment list at start.
//   warps 4-11  two softmax warpgroups, one per M-tile; thread = TMEM lane =
//               query row.  Unless stage 2 already wrote the rotated queries
//               (then the Q tiles are loaded rotated), they rotate their Q
//               rows in shared memory (RoPE),
//               read S from TMEM, keep a running max in base 2 and rescale O
//               in TMEM only when the max grows by more than 2^8 (exact: the
//               final normalisation uses the same reference), write P (bf16)
//               over the S columns, and finally normalise O and store it.
// The two M-tiles ping-pong so the tensor core computes one tile's S and PV
// while the other's softmax runs.  Every mbarrier wait is bounded; a timeout
// records an error word and the CTA winds down.
#include <cudaTypedefs.h>

#include <algorithm>

#include "hga_internal.cuh"
#include "sm100.cuh"

namespace hga {

__device__ int g_attend_tc_error = 0;

namespace {

using namespace sm100;

// Two shapes of CTA.  The general one: 384 threads, two 128-row M-tiles,
// one CTA per SM (all 512 TMEM columns).  kOne (units of at most 128 query
// rows, i.e. Hq/Hkv <= 2): 256 threads, one M-tile, 256 TMEM columns and a
// 2-stage ring, so two CTAs share an SM and one's softmax, set-up and
// epilogue overlap the other's products.
template <bool kOne> struct Shape {
    static constexpr int kThreads = kOne ? 256 : 384;
    static constexpr uint32_t kRegsLaunch = kOne ? 128 : 168;   // 65536 / (threads x CTAs per SM)
    static constexpr uint32_t kRegsCtl = 56;                    // warps 0-3: TMA producers, MMA issuer
    static constexpr uint32_t kRegsSoftmax = kOne ? 200 : 224;  // softmax and epilogue warps
    static constexpr uint32_t kTmemCols = kOne ? 256 : 512;
    static_assert(128 * kRegsCtl + (kThreads - 128) * kRegsSoftmax <= kThreads * kRegsLaunch,
                  "register split");
};
constexpr int kMaxSeg = 2048;
constexpr int kSegPerTile = 16;          // 16 x 8 tokens = 128 keys
constexpr int kDummy = 0x7fffffff;       // padding segment

template <int D, bool kOne = false>
struct Cfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kStages = (D == 128 || kOne) ? 2 : 4;
    static constexpr uint32_t kHalfBytes = 128 * 128;          // 128 rows x 128 B
    static constexpr uint32_t kTileBytes = kHalves * kHalfBytes;
    static constexpr uint32_t oQ = 0;
    static constexpr uint32_t oK = oQ + (kOne ? 1 : 2) * kTileBytes;
    static constexpr uint32_t oV = oK + kStages * kTileBytes;
    static constexpr uint32_t oEnd = oV + kStages * kTileBytes;
    static constexpr uint32_t oCS = oEnd;                       // optional cos/sin table
};

struct Ctl {
    uint64_t q_full[2], q_ready[2], s_full[2], p_full[2], o_full[2];
    uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
    uint64_t fin;
    uint32_t tmem_base;
    int nseg, first_cur;
    int early;                // tile 0 was issued during set-up
    volatile int abort;
    int s_pos[kChunk];        // positions of this CTA's query tokens
    int seg_tok[kMaxSeg];
};

struct TcArgs {
    int T, Hq, Hkv, G, NB, F, L, K_g, g_s, k_T, v_T;
    int rows_per_unit, ctas_per_unit, tokM;
    int cs_tokens;            // > 0: the CTA's (token, pair) cos/sin table is in smem
    int prerot;               // the Q tiles are already rotated (stage 2 wrote them)
    int tma_out;              // O leaves through the output map (else row stores)
    int c0;                   // first query block of this launch
    int B, nblk;              // sequences and query blocks of this launch (persistent form)
    // Host-resident tier: K/V rows come from the tier's buffers, not from the
    // token layout.  Tokens below sink_rows sit at row buf_row0 + token, other
    // fixed tokens at buf_row0 + win_row0 + token - win_tok0; routed group
    // slot j of (block c, head h, sequence b) at the row rt_map gives.
    int sink_rows, win_tok0, win_row0, buf_row0, rt_W;
    const int32_t *rt_map;
    const int32_t *sel_group;
    const int32_t *pos;
    __nv_bfloat16 *out;
    float *lse;
    float scale_log2;
    Rope rope;
};

__device__ __forceinline__ void fail(Ctl &ctl) {
    ctl.abort = 1;
    atomicExch(&g_attend_tc_error, (int)HGA_ERR_TIMEOUT);
}

// Loads nsj segments (8 key rows each, rows sg[e] of sequence b's token
// layout) of one tensor into a 128B-swizzled tile whose D-halves are
// half_bytes apart; runs of 8 or 2 consecutive segments go as one 64- or
// 16-row box.
template <int kHalves>
__device__ __forceinline__ void load_tile(uint8_t *tile, uint32_t half_bytes, const int *sg,
                                          int nsj, const CUtensorMap *m8, const CUtensorMap *m16,
                                          const CUtensorMap *m64, uint64_t *full, int h, int zb) {
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
        const int z = zb + (st == kDummy ? 0 : st);
        for (int hf = 0; hf < kHalves; ++hf)
            tma_load_3d(tile + hf * half_bytes + e * 1024, m, full, hf * 64, h, z);
        e += run;
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// One key tile of the online softmax for one query row (thread = TMEM lane
// of its M-tile; lane_base addresses the row's S columns, O follows at +128):
// reads S, masks the columns at or past nvis (gc0 = the tile's first column
// in the key list), updates the base-2 reference m_ref and the row sum l,
// writes P (bf16) over the S columns and rescales O in TMEM when the
// reference grows.  Ends with the TMEM stores complete.
template <int D>
__device__ __forceinline__ void softmax_tile(uint32_t lane_base, int gc0, int nvis, bool valid,
                                             float sc, float &m_ref, float &l) {
    // the row's visible keys are the first nvis columns of the list
    const bool need_mask = gc0 + kSegPerTile * 8 > nvis;
    // one TMEM pass: the S row (up to 128 columns) into registers
    uint32_t v[128];
    tmem_ld32(lane_base + 0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
    tmem_ld32(lane_base + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
    tmem_ld32(lane_base + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
    tmem_ld32(lane_base + 96, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
    tmem_ld_wait();
    if (need_mask) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
            if (gc0 + e >= nvis) v[e] = __float_as_uint(-INFINITY);
    }
    // row max with 8 independent chains of three-input maxima
    float mx8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(__uint_as_float(v[u]), __uint_as_float(v[u + 8]));
#pragma unroll
    for (int e = 16; e < 128; e += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u)
            mx8[u] = max3f(mx8[u], __uint_as_float(v[e + u]), __uint_as_float(v[e + 8 + u]));
    float mx = fmaxf(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]));
    mx = max3f(mx, mx8[6], mx8[7]);
    if (!valid) mx = -INFINITY;
    const float mt_new = mx * sc;
    // The reference grows only when the row max rises by more than
    // 2^8; P uses the new reference, and O (accumulated under the
    // old one) is rescaled below, before this tile's P.V.
    const bool grow = mt_new > m_ref + 8.0f;
    const bool rescale = grow && m_ref != -INFINITY;
    const float f = rescale ? ex2(m_ref - mt_new) : 1.0f;
    if (grow) m_ref = mt_new;
    l *= f;
    // P = 2^(s*scale - m_ref) as packed bf16, in place, over the S columns
    // A row with no reference yet has every column masked (a valid row sees
    // a key of its first tile), so s * scale + 0 is -inf and P is 0 without
    // a per-column branch; rows past the end are never stored.
    const float neg = m_ref != -INFINITY ? -m_ref : 0.f;
    // pairs of columns in packed two-lane fp32: s * scale - m_ref
    // and the row sum (4 chains of pairs), ex2 per column
    const uint64_t sc2 = f2_pack(sc, sc), neg2 = f2_pack(neg, neg);
    uint64_t l4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) l4[u] = f2_pack(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < 64; ++e) {
        const float2 x = f2_unpack(f2_fma(
            f2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2, neg2));
        const float p0 = ex2(x.x), p1 = ex2(x.y);
        l4[e & 3] = f2_add(l4[e & 3], f2_pack(p0, p1));
        v[e] = pack_bf16(p0, p1);
    }
    const float2 la = f2_unpack(f2_add(l4[0], l4[1])), lb = f2_unpack(f2_add(l4[2], l4[3]));
    l += (la.x + la.y) + (lb.x + lb.y);
    tmem_st32(lane_base + 0, *reinterpret_cast<const uint32_t(*)[32]>(&v[0]));
    tmem_st32(lane_base + 32, *reinterpret_cast<const uint32_t(*)[32]>(&v[32]));
    // tcgen05.ld/st are warp-collective: the warp rescales O
    // together when any of its rows needs it (factor 1 elsewhere)
    if (__any_sync(0xffffffffu, rescale)) {
        for (int cb = 0; cb < D / 32; ++cb) {
            uint32_t o[32];
            tmem_ld32(lane_base + 128 + cb * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(lane_base + 128 + cb * 32, o);
        }
    }
    tmem_st_wait();
}

// kTier: keys come from the host tier's buffers and group cache (TcArgs tier
// fields) instead of the token layout; a separate instantiation, so the
// in-HBM prefill's code is not touched by it.
template <int D, bool kTier, bool kOne>
__global__ void __launch_bounds__(Shape<kOne>::kThreads, kOne ? 2 : 1)
k_attend_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK16,
            const __grid_constant__ CUtensorMap tmV16, const __grid_constant__ CUtensorMap tmK64,
            const __grid_constant__ CUtensorMap tmV64, const __grid_constant__ CUtensorMap tmO,
            const TcArgs A) {
    using C = Cfg<D, kOne>;
    using SH = Shape<kOne>;
    constexpr int kThreads = SH::kThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ Ctl ctl;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = A.c0 + blockIdx.x / A.ctas_per_unit, cu = blockIdx.x % A.ctas_per_unit;
    const int h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk;
    const int row0 = cu * 256;
    const int rows = min(256, A.rows_per_unit - row0);
    const int NT = (rows + 127) >> 7;
    const int max_tok = min(t0 + (row0 + rows - 1) / A.G, A.T - 1);

    // ---------------------------------------------------------- set-up --
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl.q_full[i], 1);
            mbar_init(&ctl.q_ready[i], 128);
            mbar_init(&ctl.s_full[i], 1);
            mbar_init(&ctl.p_full[i], 128);
            mbar_init(&ctl.o_full[i], 1);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&ctl.k_full[i], 1);
            mbar_init(&ctl.v_full[i], 1);
            mbar_init(&ctl.k_empty[i], 1);
            mbar_init(&ctl.v_empty[i], 1);
        }
        mbar_init(&ctl.fin, 1);
        ctl.abort = 0;
        fence_barrier_init();
        // Q tiles first, so they load while the cos/sin table is computed
        prefetch_tensormap(&tmQ);
        for (int mt = 0; mt < NT; ++mt) {
            const int tok_first = t0 + (row0 + mt * 128) / A.G;
            mbar_arrive_expect_tx(&ctl.q_full[mt], (uint32_t)(A.G * A.tokM * D * 2));
            for (int hf = 0; hf < C::kHalves; ++hf)
                tma_load_3d(smem + C::oQ + mt * C::kTileBytes + hf * C::kHalfBytes, &tmQ,
                            &ctl.q_full[mt], hf * 64, h * A.G, b * A.T + tok_first);
        }
        // The first key tile, when the fixed windows fill it, depends on no
        // routed id: its K and V start loading now, before the segment list
        // is built (its 16 segments are the list's first 16, the same rule).
        const int nsink = min(A.F, c);
        const int rec_lo = max(c - max(A.L, 1), nsink);
        ctl.early = 8 * (nsink + (c - rec_lo)) >= kSegPerTile;
        if (ctl.early) {
            int sg[kSegPerTile];
            for (int e = 0; e < kSegPerTile; ++e) {
                const int tok = e < 8 * nsink ? e * 8 : rec_lo * kChunk + (e - 8 * nsink) * 8;
                if constexpr (kTier)
                    sg[e] = A.buf_row0 + (tok < A.sink_rows ? tok : A.win_row0 + tok - A.win_tok0);
                else
                    sg[e] = tok;
            }
            prefetch_tensormap(&tmK64);
            prefetch_tensormap(&tmV64);
            mbar_arrive_expect_tx(&ctl.k_full[0], (uint32_t)kSegPerTile * 8 * D * 2);
            load_tile<C::kHalves>(smem + C::oK, C::kHalfBytes, sg, kSegPerTile, &tmK, &tmK16,
                                  &tmK64, &ctl.k_full[0], h, b * A.k_T);
            mbar_arrive_expect_tx(&ctl.v_full[0], (uint32_t)kSegPerTile * 8 * D * 2);
            load_tile<C::kHalves>(smem + C::oV, C::kHalfBytes, sg, kSegPerTile, &tmV, &tmV16,
                                  &tmV64, &ctl.v_full[0], h, b * A.v_T);
        }
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, SH::kTmemCols);
        tc_fence_before();
    }
    if (warp == 3 && !A.prerot) {
        // positions of the CTA's tokens (for the rotation), one coalesced load
        const int tk0 = t0 + row0 / A.G;
        for (int j = lane; j < kChunk; j += 32)
            ctl.s_pos[j] = tk0 + j < A.T ? A.pos[(int64_t)b * A.T + tk0 + j] : 0;
    }
    if (warp == 2) {
        // the visible set as 8-token segments: sinks, recent, routed groups,
        // then the current chunk up to this CTA's last query token
        const int nsink = min(A.F, c);
        const int rec_lo = max(c - max(A.L, 1), nsink);
        const int n_fixed = 8 * (nsink + (c - rec_lo));
        // load row of a token: itself, or its place in the tier's window
        auto row_of = [&](int tok) {
            if constexpr (kTier)
                return A.buf_row0 + (tok < A.sink_rows ? tok : A.win_row0 + tok - A.win_tok0);
            else
                return tok;
        };
        for (int s = lane; s < n_fixed; s += 32)
            ctl.seg_tok[s] = row_of(s < 8 * nsink ? s * 8 : rec_lo * kChunk + (s - 8 * nsink) * 8);
        const int32_t *sel = A.sel_group + (((int64_t)b * A.NB + c) * A.Hkv + h) * A.K_g;
        const int gseg = A.g_s / 8;
        int kg = 0;
        for (int base = 0; base < A.K_g; base += 32) {
            const int v = base + lane < A.K_g ? sel[base + lane] : -1;
            kg += __popc(__ballot_sync(0xffffffffu, v >= 0));
        }
        for (int j = lane; j < kg; j += 32) {
            int r0;
            if constexpr (kTier)
                r0 = A.rt_map[(((int64_t)b * A.rt_W + (c - A.c0)) * A.Hkv + h) * A.K_g + j];
            else
                r0 = sel[j] * A.g_s;
            for (int e = 0; e < gseg; ++e) ctl.seg_tok[n_fixed + j * gseg + e] = r0 + e * 8;
        }
        const int n_route = n_fixed + kg * gseg;
        const int ncur = (max_tok - t0) / 8 + 1;
        for (int e = lane; e < ncur; e += 32) ctl.seg_tok[n_route + e] = row_of(t0 + e * 8);
        int nseg = n_route + ncur;
        if (lane == 0) {
            if (nseg & 1) ctl.seg_tok[nseg++] = kDummy;
            ctl.nseg = nseg;
            ctl.first_cur = n_route;
        }
    }
    __syncthreads();
    const int tok0 = t0 + row0 / A.G;
    float2 *cs_tab = reinterpret_cast<float2 *>(smem + C::oCS);
    tc_fence_after();
    // Registers: the producer / MMA warpgroup needs few, the two softmax
    // warpgroups hold a 128-column S row each.  128 x 56 + 256 x 224 equals
    // the launch allocation of 384 x 168.

    const uint32_t tmem = ctl.tmem_base;
    const int nseg = ctl.nseg;
    const int ntiles = (nseg + kSegPerTile - 1) / kSegPerTile;
    const int first_cur = ctl.first_cur;

    if (warp < 4) {
    regs_dec<SH::kRegsCtl>();
    if (warp == 0 || warp == 2) {
        // ------------------------------------------------------ producers --
        // warp 0 streams the K tiles, warp 2 the V tiles, each through its own
        // stage ring: a K tile is needed one P.V earlier than its V tile, so
        // the K stream must not wait behind V stage releases
        if (lane == 0) {
            const bool is_k = warp == 0;
            const CUtensorMap *m8 = is_k ? &tmK : &tmV;
            const CUtensorMap *m16 = is_k ? &tmK16 : &tmV16;
            const CUtensorMap *m64 = is_k ? &tmK64 : &tmV64;
            prefetch_tensormap(m8);
            prefetch_tensormap(m16);
            prefetch_tensormap(m64);
            const int kvT = is_k ? A.k_T : A.v_T;
            for (int j = 0; j < ntiles && !ctl.abort; ++j) {
                const int s = j % C::kStages;
                const uint32_t ph = ((j / C::kStages) - 1) & 1;
                uint64_t *empty = is_k ? &ctl.k_empty[s] : &ctl.v_empty[s];
                uint64_t *full = is_k ? &ctl.k_full[s] : &ctl.v_full[s];
                if (j >= C::kStages && !mbar_wait(empty, ph)) {
                    fail(ctl);
                    break;
                }
                if (j == 0 && ctl.early) continue;      // tile 0 is already loading
                const int nsj = min(kSegPerTile, nseg - j * kSegPerTile);
                uint8_t *tile = smem + (is_k ? C::oK : C::oV) + s * C::kTileBytes;
                mbar_arrive_expect_tx(full, (uint32_t)nsj * 8 * D * 2);
                load_tile<C::kHalves>(tile, C::kHalfBytes, ctl.seg_tok + j * kSegPerTile, nsj, m8,
                                      m16, m64, full, h, b * kvT);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
            bool ok = true;
            // rotated Q tiles are ready as soon as they land
            for (int mt = 0; mt < NT && ok; ++mt)
                ok = mbar_wait(A.prerot ? &ctl.q_full[mt] : &ctl.q_ready[mt], 0);
            tc_fence_after();
            auto issue_pv = [&](int mt, int jj) {
                const int sp = jj % C::kStages;
                const int nsj = min(kSegPerTile, nseg - jj * kSegPerTile);
                const uint32_t vbase = smem_addr(smem + C::oV + sp * C::kTileBytes);
                for (int ks = 0; ks < nsj / 2; ++ks) {
                    const uint64_t bd = smem_desc_sw128(vbase + ks * 2048, C::kHalfBytes, 1024);
                    mma_ts(tmem + mt * 256 + 128, tmem + mt * 256 + ks * 8, bd, idesc_pv,
                           (jj > 0 || ks > 0) ? 1u : 0u);
                }
            };
            auto issue_s = [&](int mt, int jj) {
                const int s = jj % C::kStages;
                const int nsj = min(kSegPerTile, nseg - jj * kSegPerTile);
                const uint32_t idesc = idesc_bf16_f32(128, nsj * 8, false, false);
                const uint32_t qb = smem_addr(smem + C::oQ + mt * C::kTileBytes);
                const uint32_t kb = smem_addr(smem + C::oK + s * C::kTileBytes);
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + mt * 256, smem_desc_sw128(qb + off, 16, 1024),
                           smem_desc_sw128(kb + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                }
            };
            // per tile j: P.V of tile j-1 first (it needs no new data), then
            // S of tile j once its K tile has landed; K stages are released
            // after both S products, V stages after both P.V products
            for (int j = 0; j <= ntiles && ok; ++j) {
                const int s = j % C::kStages;
                for (int mt = 0; mt < NT && ok; ++mt) {
                    if (j > 0) {
                        if (!(ok = mbar_wait(&ctl.p_full[mt], (j - 1) & 1))) break;
                        tc_fence_after();
                        const int sp = (j - 1) % C::kStages;
                        if (mt == 0) {
                            if (!(ok = mbar_wait(&ctl.v_full[sp], ((j - 1) / C::kStages) & 1))) break;
                            tc_fence_after();
                        }
                        issue_pv(mt, j - 1);
                        if (j == ntiles) mma_commit(&ctl.o_full[mt]);
                        else if (mt == NT - 1) mma_commit(&ctl.v_empty[sp]);
                    }
                    if (j < ntiles) {
                        if (mt == 0) {
                            if (!(ok = mbar_wait(&ctl.k_full[s], (j / C::kStages) & 1))) break;
                            tc_fence_after();
                        }
                        issue_s(mt, j);
                        mma_commit(&ctl.s_full[mt]);
                        if (mt == NT - 1) mma_commit(&ctl.k_empty[s]);
                    }
                }
            }
            if (!ok) fail(ctl);
            // all issued tensor-core work retires before TMEM is released
            mma_commit(&ctl.fin);
            if (!mbar_wait(&ctl.fin, 0)) fail(ctl);
        }
    }
    } else {
        regs_inc<SH::kRegsSoftmax>();
        // ------------------------------------------------------- softmax --
        // cos/sin of every (token, pair) of this CTA's rows, shared by the G
        // query heads of a token (each angle formed once instead of G times);
        // built by the softmax warps alone while the producers already load
        // the first key and value tiles
        if (A.cs_tokens > 0) {
            // rows padded to H + 1 entries: the 4 tokens a warp reads differ in bank
            constexpr int H = D / 2;
            for (int e = threadIdx.x - 128; e < A.cs_tokens * H; e += kThreads - 128) {
                const int tj = e / H;
                if (tok0 + tj < A.T) cs_tab[tj * (H + 1) + e % H] = rope_cs_int(A.rope, ctl.s_pos[tj], e % H);
            }
            named_bar(1, kThreads - 128);
        }
        const int mt = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const int R = row0 + mt * 128 + r;
        const int tok = t0 + R / A.G;
        const int head = R % A.G;
        const bool valid = mt < NT && (mt * 128 + r) < rows && tok < A.T;
        // Visible keys of this row, in key-list order: every fixed and routed
        // key (first_cur segments), then the current chunk's tokens up to the
        // row's own; only the trailing padding follows.  So a key column is
        // visible iff its index in the list is below nvis.
        const int nvis = first_cur * 8 + (tok - t0 + 1);
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16) + mt * 256;
        if (mt < NT) {
            // RoPE of this row's query, in place in the swizzled Q tile
            // (rotated tiles need no wait here: the MMA issuer waits for them)
            bool ok = A.prerot || mbar_wait(&ctl.q_full[mt], 0);
            if (!ok) fail(ctl);
            if (ok && valid && !A.prerot) {
                uint8_t *qt = smem + C::oQ + mt * C::kTileBytes;
                const int32_t p = ctl.s_pos[tok - tok0];
                const float2 *csr = cs_tab + (tok - tok0) * (D / 2 + 1);
                constexpr int kGroups = D / 16;       // 8 pairs per 16-byte chunk
                for (int g = 0; g < kGroups; ++g) {
                    const int lo_half = 0, hi_half = D == 128 ? 1 : 0;
                    const int lo_chunk = g, hi_chunk = D == 128 ? g : g + 4;
                    uint4 *lo = reinterpret_cast<uint4 *>(qt + lo_half * C::kHalfBytes + r * 128 +
                                                          ((lo_chunk ^ (r & 7)) << 4));
                    uint4 *hi = reinterpret_cast<uint4 *>(qt + hi_half * C::kHalfBytes + r * 128 +
                                                          ((hi_chunk ^ (r & 7)) << 4));
                    uint4 a = *lo, bb = *hi;
                    __nv_bfloat162 *pa = reinterpret_cast<__nv_bfloat162 *>(&a);
                    __nv_bfloat162 *pb = reinterpret_cast<__nv_bfloat162 *>(&bb);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(pa[e]);
                        const float2 y = __bfloat1622float2(pb[e]);
                        const float2 c0 = A.cs_tokens > 0 ? csr[g * 8 + 2 * e]
                                                          : rope_cs_int(A.rope, p, g * 8 + 2 * e);
                        const float2 c1 = A.cs_tokens > 0 ? csr[g * 8 + 2 * e + 1]
                                                          : rope_cs_int(A.rope, p, g * 8 + 2 * e + 1);
                        // the same rounding as every other rotation in the library
                        const float2 r0 = rot_pair(x.x, y.x, c0), r1 = rot_pair(x.y, y.y, c1);
                        pa[e] = __floats2bfloat162_rn(r0.x, r1.x);
                        pb[e] = __floats2bfloat162_rn(r0.y, r1.y);
                    }
                    *lo = a;
                    *hi = bb;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&ctl.q_ready[mt]);

            float m_ref = -INFINITY, l = 0.f;
            const float sc = A.scale_log2;
            for (int j = 0; j < ntiles && ok; ++j) {
                if (!(ok = mbar_wait(&ctl.s_full[mt], j & 1))) {
                    fail(ctl);
                    break;
                }
                tc_fence_after();
                softmax_tile<D>(lane_base, j * kSegPerTile * 8, nvis, valid, sc, m_ref, l);
                tc_fence_before();
                mbar_arrive(&ctl.p_full[mt]);
            }
            // epilogue: O / l -> out, LSE
            if (ok) {
                if (!mbar_wait(&ctl.o_full[mt], 0)) {
                    fail(ctl);
                    ok = false;
                }
            }
            tc_fence_after();
            // With the output map, the normalised rows are staged in this
            // M-tile's Q tile (its last S product completed before its last
            // P.V), in the 128B-swizzled layout of the map's box (the Q
            // tile's own), and leave as one tensor store per D-half; rows
            // past the sequence's end fall outside the map and are not written.
            uint8_t *ot = smem + C::oQ + mt * C::kTileBytes;
            if (ok) {
                const float inv = valid && l > 0.f ? 1.f / l : 0.f;
                __nv_bfloat16 *orow =
                    A.out + (((int64_t)b * A.T + tok) * A.Hq + (int64_t)h * A.G + head) * D;
#pragma unroll
                for (int hb = 0; hb < D / 64; ++hb) {
                    uint32_t v[64];
                    tmem_ld32(lane_base + 128 + hb * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                    tmem_ld32(lane_base + 128 + hb * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                    tmem_ld_wait();
                    if (valid) {
#pragma unroll
                        for (int q8 = 0; q8 < 8; ++q8) {
                            uint4 w;
                            uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                wp[e] = pack_bf16(__uint_as_float(v[q8 * 8 + 2 * e]) * inv,
                                                  __uint_as_float(v[q8 * 8 + 2 * e + 1]) * inv);
                            if (A.tma_out)
                                *reinterpret_cast<uint4 *>(ot + hb * C::kHalfBytes + r * 128 +
                                                           ((q8 ^ (r & 7)) << 4)) = w;
                            else
                                reinterpret_cast<uint4 *>(orow)[hb * 8 + q8] = w;
                        }
                    }
                }
                if (valid && A.lse)
                    A.lse[((int64_t)b * A.Hq + (int64_t)h * A.G + head) * A.T + tok] =
                        (m_ref + __log2f(l)) * 0.6931471805599453f;
            }
            if (A.tma_out) {
                // every thread of the warpgroup reaches this barrier once
                fence_proxy_async_smem();
                if (mt == 0) named_bar(2, 128);
                else named_bar(3, 128);
                if (r == 0 && ok && !ctl.abort) {
                    const int tok_first = t0 + (row0 + mt * 128) / A.G;
                    for (int hf = 0; hf < C::kHalves; ++hf)
                        tma_store_4d(&tmO, ot + hf * C::kHalfBytes, hf * 64, h * A.G, tok_first, b);
                    bulk_commit();
                    bulk_wait_read();      // the tile is read before the CTA exits
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, SH::kTmemCols);
    }
}

// ------------------------------------------------------------------------
// Persistent form (rotated queries given, units of at least 256 rows, no
// tier): one CTA per SM walks the units blockIdx.x, blockIdx.x + gridDim.x,
// ... (the order of the one-unit-per-CTA grid).  Stage rings and barrier
// phases run on across units, so a unit's set-up and epilogue overlap the
// key loops around it:
//   warp 3      builds the segment list of each unit into one of two buffers
//               and loads its two rotated Q tiles, each as soon as the
//               previous unit's last S product on that tile has completed.
//   warps 0, 2  stream the K and V tiles of unit after unit.
//   warp 1      issues the products; a unit's first S follows the previous
//               unit's last P.V on the same M-tile.
//   warps 4-11  softmax as above; each M-tile's epilogue (O from TMEM to
//               row stores) runs while the tensor core starts the next unit,
//               whose first P.V waits for the softmax warps anyway.
constexpr int kMaxSegP = 1024;

struct CtlP {
    uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_full[2];
    uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
    uint64_t seg_full[2], seg_empty[2];
    uint64_t fin;
    uint32_t tmem_base;
    volatile int abort;
    int nseg[2], first_cur[2];
    int seg_tok[2][kMaxSegP];
};
constexpr uint32_t kSegConsumers = 3 + 8;   // K, V producers, MMA issuer, 8 softmax warps

struct UnitP {
    int c, cu, h, b;
};

// Unit u in the one-unit-per-CTA grid's order: (block, row half) fastest,
// then KV head, then sequence.
__device__ __forceinline__ UnitP unit_at(const TcArgs &A, int u) {
    UnitP p;
    const int per_h = A.nblk * A.ctas_per_unit;
    const int per_b = per_h * A.Hkv;
    p.b = u / per_b;
    const int rem = u - p.b * per_b;
    p.h = rem / per_h;
    const int x = rem - p.h * per_h;
    p.c = A.c0 + x / A.ctas_per_unit;
    p.cu = x - (x / A.ctas_per_unit) * A.ctas_per_unit;
    return p;
}

__device__ __forceinline__ void fail_p(CtlP &ctl) {
    ctl.abort = 1;
    atomicExch(&g_attend_tc_error, (int)HGA_ERR_TIMEOUT);
}

// The visible set of one unit's rows as 8-token segments (sinks, recent
// chunks, routed groups, then the current chunk up to the unit's last query
// token), written by one whole warp into buffer buf.
__device__ __forceinline__ void build_segments_p(CtlP &ctl, int buf, const TcArgs &A,
                                                 const UnitP &un) {
    const int lane = threadIdx.x & 31;
    const int c = un.c, t0 = c * kChunk;
    const int row0 = un.cu * 256;
    const int rows = min(256, A.rows_per_unit - row0);
    const int max_tok = min(t0 + (row0 + rows - 1) / A.G, A.T - 1);
    int *seg = ctl.seg_tok[buf];
    const int nsink = min(A.F, c);
    const int rec_lo = max(c - max(A.L, 1), nsink);
    const int n_fixed = 8 * (nsink + (c - rec_lo));
    for (int s = lane; s < n_fixed; s += 32)
        seg[s] = s < 8 * nsink ? s * 8 : rec_lo * kChunk + (s - 8 * nsink) * 8;
    const int32_t *sel = A.sel_group + (((int64_t)un.b * A.NB + c) * A.Hkv + un.h) * A.K_g;
    const int gseg = A.g_s / 8;
    int kg = 0;
    for (int base = 0; base < A.K_g; base += 32) {
        const int v = base + lane < A.K_g ? sel[base + lane] : -1;
        kg += __popc(__ballot_sync(0xffffffffu, v >= 0));
    }
    for (int j = lane; j < kg; j += 32) {
        const int r0 = sel[j] * A.g_s;
        for (int e = 0; e < gseg; ++e) seg[n_fixed + j * gseg + e] = r0 + e * 8;
    }
    const int n_route = n_fixed + kg * gseg;
    const int ncur = (max_tok - t0) / 8 + 1;
    for (int e = lane; e < ncur; e += 32) seg[n_route + e] = t0 + e * 8;
    __syncwarp();
    if (lane == 0) {
        int nseg = n_route + ncur;
        if (nseg & 1) seg[nseg++] = kDummy;
        ctl.nseg[buf] = nseg;
        ctl.first_cur[buf] = n_route;
    }
    __syncwarp();
}

template <int D>
__global__ void __launch_bounds__(384, 1)
k_attend_tcp(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK16,
             const __grid_constant__ CUtensorMap tmV16, const __grid_constant__ CUtensorMap tmK64,
             const __grid_constant__ CUtensorMap tmV64, const TcArgs A) {
    using C = Cfg<D, false>;
    using SH = Shape<false>;
    constexpr int kS = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ CtlP ctl;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NU = A.B * A.Hkv * A.nblk * A.ctas_per_unit;

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl.q_full[i], 1);
            mbar_init(&ctl.q_empty[i], 1);
            mbar_init(&ctl.s_full[i], 1);
            mbar_init(&ctl.p_full[i], 128);
            mbar_init(&ctl.o_full[i], 1);
            mbar_init(&ctl.seg_full[i], 1);
            mbar_init(&ctl.seg_empty[i], kSegConsumers);
        }
        for (int i = 0; i < kS; ++i) {
            mbar_init(&ctl.k_full[i], 1);
            mbar_init(&ctl.v_full[i], 1);
            mbar_init(&ctl.k_empty[i], 1);
            mbar_init(&ctl.v_empty[i], 1);
        }
        mbar_init(&ctl.fin, 1);
        ctl.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, SH::kTmemCols);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    // launched as a programmatic dependent of stage 2: the set-up above ran
    // while it finished; the routed sets and rotated queries are read below
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp < 4) {
        regs_dec<SH::kRegsCtl>();
        if ((warp == 0 || warp == 2) && lane == 0) {
            // ------------------------------------------------- producers --
            const bool is_k = warp == 0;
            const CUtensorMap *m8 = is_k ? &tmK : &tmV;
            const CUtensorMap *m16 = is_k ? &tmK16 : &tmV16;
            const CUtensorMap *m64 = is_k ? &tmK64 : &tmV64;
            prefetch_tensormap(m8);
            prefetch_tensormap(m16);
            prefetch_tensormap(m64);
            uint64_t *full = is_k ? ctl.k_full : ctl.v_full;
            uint64_t *empty = is_k ? ctl.k_empty : ctl.v_empty;
            const uint32_t ring = is_k ? C::oK : C::oV;
            const int kvT = is_k ? A.k_T : A.v_T;
            int gt = 0;          // tiles issued so far, over all units
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int u = blockIdx.x + i * gridDim.x;
                if (u >= NU || ctl.abort) break;
                const int buf = i & 1;
                if (!(ok = mbar_wait_ab(&ctl.seg_full[buf], (i >> 1) & 1, &ctl.abort))) break;
                const UnitP un = unit_at(A, u);
                const int nseg = ctl.nseg[buf];
                const int ntiles = (nseg + kSegPerTile - 1) / kSegPerTile;
                const int *sg = ctl.seg_tok[buf];
                for (int j = 0; j < ntiles; ++j, ++gt) {
                    const int s = gt % kS;
                    if (gt >= kS && !(ok = mbar_wait_ab(&empty[s], ((gt / kS) - 1) & 1, &ctl.abort)))
                        break;
                    const int nsj = min(kSegPerTile, nseg - j * kSegPerTile);
                    mbar_arrive_expect_tx(&full[s], (uint32_t)nsj * 8 * D * 2);
                    load_tile<C::kHalves>(smem + ring + s * C::kTileBytes, C::kHalfBytes,
                                          sg + j * kSegPerTile, nsj, m8, m16, m64, &full[s], un.h,
                                          un.b * kvT);
                }
                if (ok) mbar_arrive(&ctl.seg_empty[buf]);
            }
            if (!ok) {
                fail_p(ctl);
                // let the copies already issued land before the CTA exits
                for (int t = max(0, gt - kS); t < gt; ++t)
                    mbar_wait(&full[t % kS], (t / kS) & 1, 100000000ull);
            }
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------ MMA issuer --
            const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
            auto issue_pv = [&](int mt, int sp, int nsj, bool acc) {
                const uint32_t vbase = smem_addr(smem + C::oV + sp * C::kTileBytes);
                for (int ks = 0; ks < nsj / 2; ++ks) {
                    const uint64_t bd = smem_desc_sw128(vbase + ks * 2048, C::kHalfBytes, 1024);
                    mma_ts(tmem + mt * 256 + 128, tmem + mt * 256 + ks * 8, bd, idesc_pv,
                           (acc || ks > 0) ? 1u : 0u);
                }
            };
            auto issue_s = [&](int mt, int s, int nsj) {
                const uint32_t idesc = idesc_bf16_f32(128, nsj * 8, false, false);
                const uint32_t qb = smem_addr(smem + C::oQ + mt * C::kTileBytes);
                const uint32_t kb = smem_addr(smem + C::oK + s * C::kTileBytes);
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + mt * 256, smem_desc_sw128(qb + off, 16, 1024),
                           smem_desc_sw128(kb + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                }
            };
            bool ok = true;
            int g0 = 0;          // global index of the unit's first tile
            for (int i = 0; ok; ++i) {
                const int u = blockIdx.x + i * gridDim.x;
                if (u >= NU || ctl.abort) break;
                const int buf = i & 1;
                if (!(ok = mbar_wait_ab(&ctl.seg_full[buf], (i >> 1) & 1, &ctl.abort))) break;
                const int nseg = ctl.nseg[buf];
                mbar_arrive(&ctl.seg_empty[buf]);
                const int ntiles = (nseg + kSegPerTile - 1) / kSegPerTile;
                // per tile j: P.V of tile j-1 (it needs no new data), then S
                // of tile j; K stages are released after both S products, V
                // stages after both P.V products
                for (int j = 0; j <= ntiles && ok; ++j) {
                    const int gs = g0 + j;
                    const int s = gs % kS;
                    for (int mt = 0; mt < 2 && ok; ++mt) {
                        if (j > 0) {
                            if (!(ok = mbar_wait_ab(&ctl.p_full[mt], (gs - 1) & 1, &ctl.abort))) break;
                            tc_fence_after();
                            const int sp = (gs - 1) % kS;
                            if (mt == 0) {
                                if (!(ok = mbar_wait_ab(&ctl.v_full[sp], ((gs - 1) / kS) & 1, &ctl.abort)))
                                    break;
                                tc_fence_after();
                            }
                            issue_pv(mt, sp, min(kSegPerTile, nseg - (j - 1) * kSegPerTile), j > 1);
                            if (j == ntiles) mma_commit(&ctl.o_full[mt]);
                            if (mt == 1) mma_commit(&ctl.v_empty[sp]);
                        }
                        if (j < ntiles) {
                            if (j == 0) {
                                if (!(ok = mbar_wait_ab(&ctl.q_full[mt], i & 1, &ctl.abort))) break;
                                tc_fence_after();
                            }
                            if (mt == 0) {
                                if (!(ok = mbar_wait_ab(&ctl.k_full[s], (gs / kS) & 1, &ctl.abort))) break;
                                tc_fence_after();
                            }
                            issue_s(mt, s, min(kSegPerTile, nseg - j * kSegPerTile));
                            mma_commit(&ctl.s_full[mt]);
                            if (j == ntiles - 1) mma_commit(&ctl.q_empty[mt]);
                            if (mt == 1) mma_commit(&ctl.k_empty[s]);
                        }
                    }
                }
                g0 += ntiles;
            }
            if (!ok) fail_p(ctl);
            // all issued tensor-core work retires before TMEM is released
            mma_commit(&ctl.fin);
            if (!mbar_wait(&ctl.fin, 0)) fail_p(ctl);
        } else if (warp == 3) {
            // ------------------------------- segment lists and Q tiles --
            bool ok = true;
            int issued = 0;      // units whose Q tiles were issued
            for (int i = 0; ok; ++i) {
                const int u = blockIdx.x + i * gridDim.x;
                if (u >= NU || ctl.abort) break;
                const int buf = i & 1;
                if (i >= 2) {
                    if (lane == 0)
                        ok = mbar_wait_ab(&ctl.seg_empty[buf], ((i >> 1) - 1) & 1, &ctl.abort);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                }
                const UnitP un = unit_at(A, u);
                build_segments_p(ctl, buf, A, un);
                if (lane == 0) {
                    mbar_arrive(&ctl.seg_full[buf]);
                    if (i == 0) prefetch_tensormap(&tmQ);
                    for (int mt = 0; mt < 2 && ok; ++mt) {
                        if (i >= 1 && !(ok = mbar_wait_ab(&ctl.q_empty[mt], (i - 1) & 1, &ctl.abort)))
                            break;
                        const int tok_first = un.c * kChunk + (un.cu * 256 + mt * 128) / A.G;
                        mbar_arrive_expect_tx(&ctl.q_full[mt], (uint32_t)(A.G * A.tokM * D * 2));
                        for (int hf = 0; hf < C::kHalves; ++hf)
                            tma_load_3d(smem + C::oQ + mt * C::kTileBytes + hf * C::kHalfBytes, &tmQ,
                                        &ctl.q_full[mt], hf * 64, un.h * A.G,
                                        un.b * A.T + tok_first);
                    }
                    if (ok) issued = i + 1;
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
            }
            if (lane == 0 && !ok) {
                fail_p(ctl);
                // the last unit's Q tiles land before the CTA exits
                if (issued > 0)
                    for (int mt = 0; mt < 2; ++mt)
                        mbar_wait(&ctl.q_full[mt], (issued - 1) & 1, 100000000ull);
            }
        }
    } else {
        regs_inc<SH::kRegsSoftmax>();
        // ------------------------------------------------------- softmax --
        const int mt = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16) + mt * 256;
        const float sc = A.scale_log2;
        bool ok = true;
        int g0 = 0;
        for (int i = 0; ok; ++i) {
            const int u = blockIdx.x + i * gridDim.x;
            if (u >= NU || ctl.abort) break;
            const int buf = i & 1;
            if (!(ok = mbar_wait_ab(&ctl.seg_full[buf], (i >> 1) & 1, &ctl.abort))) break;
            const int first_cur = ctl.first_cur[buf];
            const int nseg = ctl.nseg[buf];
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.seg_empty[buf]);
            const UnitP un = unit_at(A, u);
            const int t0 = un.c * kChunk;
            const int R = un.cu * 256 + mt * 128 + r;
            const int tok = t0 + R / A.G;
            const int head = R % A.G;
            const bool valid = tok < A.T;
            const int nvis = first_cur * 8 + (tok - t0 + 1);
            const int ntiles = (nseg + kSegPerTile - 1) / kSegPerTile;
            float m_ref = -INFINITY, l = 0.f;
            for (int j = 0; j < ntiles; ++j) {
                if (!(ok = mbar_wait_ab(&ctl.s_full[mt], (g0 + j) & 1, &ctl.abort))) break;
                tc_fence_after();
                softmax_tile<D>(lane_base, j * kSegPerTile * 8, nvis, valid, sc, m_ref, l);
                tc_fence_before();
                mbar_arrive(&ctl.p_full[mt]);
            }
            g0 += ntiles;
            if (!ok || !(ok = mbar_wait_ab(&ctl.o_full[mt], i & 1, &ctl.abort))) break;
            tc_fence_after();
            // epilogue: O / l -> out (row stores), LSE; the TMEM reads complete
            // before this warp's next p_full arrival lets the next unit's
            // first P.V overwrite O
            const float inv = valid && l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow =
                A.out + (((int64_t)un.b * A.T + tok) * A.Hq + (int64_t)un.h * A.G + head) * D;
            {
                uint32_t v[D];
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb)
                    tmem_ld32(lane_base + 128 + cb * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[cb * 32]));
                tmem_ld_wait();
                if (valid) {
#pragma unroll
                    for (int q8 = 0; q8 < D / 8; ++q8) {
                        uint4 w;
                        uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            wp[e] = pack_bf16(__uint_as_float(v[q8 * 8 + 2 * e]) * inv,
                                              __uint_as_float(v[q8 * 8 + 2 * e + 1]) * inv);
                        reinterpret_cast<uint4 *>(orow)[q8] = w;
                    }
                }
            }
            if (valid && A.lse)
                A.lse[((int64_t)un.b * A.Hq + (int64_t)un.h * A.G + head) * A.T + tok] =
                    (m_ref + __log2f(l)) * 0.6931471805599453f;
        }
        if (!ok) fail_p(ctl);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, SH::kTmemCols);
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

// 3-D bf16 map over rows of [n_rows][heads][D]: box (64, box_heads, box_rows),
// 128-byte swizzle, zero fill out of bounds.
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

// 4-D bf16 map over [n_seq][T][heads][D]: box (64, box_heads, box_rows, 1),
// 128-byte swizzle; a box never reaches past its own sequence's last token.
bool make_map_4d(CUtensorMap *m, const void *base, int D, int heads, int T, int n_seq,
                 int box_heads, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)n_seq};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2,
                             (cuuint64_t)T * heads * D * 2};
    cuuint32_t box[4] = {64u, (cuuint32_t)box_heads, (cuuint32_t)box_rows, 1u};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
hga_status run(const Geo &g, const Rope &r, const void *q, const int32_t *pos, const void *k_rot,
               int k_T, const void *v, int v_T, const int32_t *sel_group, void *out, float *lse,
               cudaStream_t st, const TierWave *tw, const void *q_rot) {
    TcArgs a;
    a.prerot = q_rot != nullptr;
    a.c0 = tw ? tw->c0 : 0;
    a.sink_rows = tw ? tw->sink_rows : 0;
    a.win_tok0 = tw ? tw->win_tok0 : 0;
    a.win_row0 = tw ? tw->win_row0 : 0;
    a.buf_row0 = tw ? tw->buf_row0 : 0;
    a.rt_W = tw ? tw->rt_W : 0;
    a.rt_map = tw ? tw->rt_map : nullptr;
    const int nblk = tw ? tw->c1 - tw->c0 : g.NB;
    a.T = g.T;
    a.Hq = g.Hq;
    a.Hkv = g.Hkv;
    a.G = g.G;
    a.NB = g.NB;
    a.F = g.F;
    a.L = g.L;
    a.K_g = g.K_g;
    a.g_s = g.g_s;
    a.k_T = k_T;
    a.v_T = v_T;
    a.rows_per_unit = kChunk * g.G;
    a.ctas_per_unit = (a.rows_per_unit + 255) / 256;
    a.tokM = min(128, kChunk * g.G) / g.G;
    {
        // the table costs tokens x D/2 x 8 bytes; keep the CTA inside 227 KB
        const int tok_cta = (min(256, a.rows_per_unit) + g.G - 1) / g.G;
        const size_t tab = (size_t)tok_cta * (D / 2 + 1) * sizeof(float2);
        a.cs_tokens = !a.prerot && Cfg<D>::oEnd + 1024 + tab + sizeof(Ctl) <= 232448 ? tok_cta : 0;
    }
    // units of at most 128 rows take the one-M-tile CTA (two per SM)
    const bool one = a.rows_per_unit <= 128;
    a.sel_group = sel_group;
    a.pos = pos;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    a.rope = r;
    CUtensorMap mq, mk, mv, mk16, mv16, mk64, mv64;
    if (!make_map(&mq, q_rot ? q_rot : q, D, g.Hq, (long long)g.B * g.T, g.G, a.tokM) ||
        !make_map(&mk, k_rot, D, g.Hkv, (long long)g.B * k_T, 1, 8) ||
        !make_map(&mv, v, D, g.Hkv, (long long)g.B * v_T, 1, 8) ||
        !make_map(&mk16, k_rot, D, g.Hkv, (long long)g.B * k_T, 1, 16) ||
        !make_map(&mv16, v, D, g.Hkv, (long long)g.B * v_T, 1, 16) ||
        !make_map(&mk64, k_rot, D, g.Hkv, (long long)g.B * k_T, 1, 64) ||
        !make_map(&mv64, v, D, g.Hkv, (long long)g.B * v_T, 1, 64))
        return HGA_ERR_CUDA;
    const size_t smem = (one ? Cfg<D, true>::oEnd : Cfg<D>::oEnd) + 1024 +
                        (size_t)a.cs_tokens * (D / 2 + 1) * sizeof(float2);
    auto kern = tw ? (one ? k_attend_tc<D, true, true> : k_attend_tc<D, true, false>)
                   : (one ? k_attend_tc<D, false, true> : k_attend_tc<D, false, false>);
    a.B = g.B;
    a.nblk = nblk;
    // rotated queries, no tier, units of at least 256 rows: the persistent
    // form, one CTA per SM
    const long long n_units = (long long)g.B * g.Hkv * nblk * a.ctas_per_unit;
    const long long segs = 8ll * (g.F + max(g.L, 1) + 1) + (long long)g.K_g * (g.g_s / 8) + 2;
    if (q_rot && !tw && a.rows_per_unit >= 256 && segs <= kMaxSegP && n_units < (1ll << 30)) {
        int dev = 0, nsm = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_status(e);
        const size_t psmem = Cfg<D>::oEnd + 1024;
        auto pk = k_attend_tcp<D>;
        if ((e = ensure_smem((const void *)pk, psmem)) != cudaSuccess) return cuda_status(e);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)std::min<long long>(n_units, std::max(nsm, 1)));
        cfg.blockDim = dim3(Shape<false>::kThreads);
        cfg.dynamicSmemBytes = psmem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cuda_status(cudaLaunchKernelEx(&cfg, pk, mq, mk, mv, mk16, mv16, mk64, mv64, a));
    }
    // the calls check that out is 16-byte aligned (the map needs it); row
    // stores remain for any other base
    CUtensorMap mo;
    a.tma_out = (reinterpret_cast<uintptr_t>(out) & 15) == 0 &&
                make_map_4d(&mo, out, D, g.Hq, g.T, g.B, g.G, a.tokM);
    if (!a.tma_out) mo = mq;      // unused
    cudaError_t e = ensure_smem((const void *)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 grid(nblk * a.ctas_per_unit, g.Hkv, g.B);
    kern<<<grid, one ? Shape<true>::kThreads : Shape<false>::kThreads, smem, st>>>(
        mq, mk, mv, mk16, mv16, mk64, mv64, mo, a);
    return cuda_status(cudaGetLastError());
}

}  // namespace

bool attend_tc_supported(const Geo &g, int dtype) {
    if (dtype != HGA_BF16 || (g.D != 64 && g.D != 128)) return false;
    if (g.G < 1 || g.G > 16 || (g.G & (g.G - 1))) return false;
    if (g.g_s % 8) return false;
    const long long segs = 8ll * (g.F + max(g.L, 1) + 1) + (long long)g.K_g * (g.g_s / 8) + 2;
    return segs <= kMaxSeg;
}

hga_status launch_attend_tc(const Geo &g, const Rope &r, const void *q, const int32_t *pos,
                            const void *k_rot, int k_T, const void *v, int v_T,
                            const int32_t *sel_group, void *out, float *lse, cudaStream_t st,
                            const TierWave *tw, const void *q_rot) {
    if (g.NB <= 0 || (tw && tw->c1 <= tw->c0)) return HGA_OK;
    return g.D == 128
        ? run<128>(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st, tw, q_rot)
        : run<64>(g, r, q, pos, k_rot, k_T, v, v_T, sel_group, out, lse, st, tw, q_rot);
}


// Reads this file's device error word on `st` (after the work queued on it)
// and optionally resets it; returns the recorded status (HGA_OK if none).
hga_status attend_tc_error_take(cudaStream_t st, bool clear) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_attend_tc_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_attend_tc_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    return (hga_status)v;
}

}  // namespace hga
