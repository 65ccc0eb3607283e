/*
 * hga.h — C ABI of the B200 (sm_100a) library for Hierarchical Global
 * Attention (HGA): routed exact-token causal attention.
 *
 * Sources.  The operations follow the HGA paper-review page ("HGA:
 * Hierarchical Global Attention — Drop-In Exact-Token Routing for Pretrained
 * Long-Context Transformers", xllm-io), section 3 (技术架构): the mixed-RoPE
 * summary formula, the routing policy (deterministic visibility, middle
 * routing, the selection equation M_sel = topK_c, G_sel = topK_g), exact
 * token output attention (eq. (1) restricted to the routed set) and the
 * store's four operations (append closed chunk, read chunk summaries, fetch
 * group summaries, gather token K/V, section "三层 K/V 存储").  The
 * gist.science page "Hierarchical Global Attention (HGA)", technical summary,
 * "Core Mechanism", restates the same mechanism.
 *
 * Conventions for every call.
 *  - Pointers are DEVICE pointers (cudaMalloc / PyTorch CUDA memory) unless a
 *    comment says host.  The caller owns every buffer; the library allocates
 *    nothing and keeps no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued asynchronously; no call synchronises the host
 *    except where stated.
 *  - Layouts are dense row-major with the last index fastest:
 *      Q, O      [B, T, Hq,  D]      query head hq uses KV head hq / (Hq/Hkv)
 *      K, V, K_rot [B, T, Hkv, D]    K is the RAW (pre-RoPE) key projection
 *      pos       [B, T] int32        RoPE positions (any values; causality
 *                                    follows the token index, not pos)
 *      s_chunk   [B, Hkv, NC, D] f32 NC = T / C closed chunks (a partial last
 *                                    chunk is open and has no summary)
 *      s_group   [B, Hkv, NC*C/g_s, D] f32, group j of chunk m at m*C/g_s + j
 *      sel_chunk [B, NB, Hkv, K_c] int32, NB = ceil(T / C) query blocks
 *      sel_group [B, NB, Hkv, K_g] int32 global group ids
 *      lse       [B, Hq, T] f32      natural-log softmax denominators
 *    Selected ids are ascending and padded with -1.
 *  - dtype (hga_dims.dtype) is the element type of Q, K, V, K_rot and O:
 *    HGA_F32 or HGA_BF16.  Summaries, scores and accumulation are fp32 or
 *    wider.
 *  - Every tensor pointer (inputs, outputs, caches, summaries) must be
 *    16-byte aligned; another base is HGA_ERR_INVALID_ARG.
 *  - Errors: arguments are checked on the host first; a failing check
 *    returns HGA_ERR_INVALID_ARG or HGA_ERR_UNSUPPORTED and launches nothing.
 *    Size limits of this build (HGA_ERR_UNSUPPORTED beyond them): B <= 65535,
 *    Hkv <= 65535, and B * T (B * capacity for a K/V cache) below 2^31.
 *    A launch failure returns HGA_ERR_CUDA (the CUDA error is not cleared by
 *    the library; hga_last_cuda_error() gives its code).
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hga_status {
    HGA_OK = 0,
    HGA_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size or a bad layout */
    HGA_ERR_UNSUPPORTED = 2,   /* valid, but not a shape this build handles  */
    HGA_ERR_CUDA = 3,          /* a CUDA launch or copy failed               */
    HGA_ERR_TIMEOUT = 4,       /* a bounded device wait gave up              */
    HGA_ERR_BOUNDS = 5,        /* a device-side index check failed           */
    HGA_ERR_WORKSPACE = 6      /* workspace missing or smaller than required */
} hga_status;

typedef enum hga_dtype { HGA_F32 = 0, HGA_BF16 = 1 } hga_dtype;

typedef enum hga_mode {
    HGA_PREFILL = 0, HGA_DECODE = 1, HGA_PREFILL_HOSTKV = 2,
    HGA_ATTEND_BACKWARD = 3     /* hga_workspace_size only: hga_attend_backward */
} hga_mode;

/* Method parameters (page section 3 and its setup table in section 6). */
typedef struct hga_params {
    int32_t C;            /* chunk length in tokens; this build needs C == 64,
                             which is also the prefill query block            */
    int32_t g_s;          /* group length; divides C                          */
    int32_t F;            /* sink chunks 0..F-1, always visible               */
    int32_t L;            /* recent closed chunks, always visible; with L == 0
                             the previous chunk is still forced visible       */
    int32_t K_c;          /* middle chunks routed per block and KV head (>=0) */
    int32_t K_g;          /* groups opened inside those chunks (>= 0)         */
    double rope_theta;    /* RoPE base: omega_i = theta^(-2i/D), pair (i, i+D/2) */
    double hf_wavelength; /* pair i is high-frequency iff 2*pi/omega_i is below
                             this; <= 0 selects C; +inf makes every pair high */
} hga_params;

/* Problem shape. */
typedef struct hga_dims {
    int32_t B;      /* sequences                                              */
    int32_t T;      /* prefill: tokens per sequence; decode: cache capacity   */
    int32_t Hq;     /* query heads, a multiple of Hkv                         */
    int32_t Hkv;    /* key/value heads                                        */
    int32_t D;      /* head dimension: 64 or 128                              */
    int32_t dtype;  /* hga_dtype                                              */
} hga_dims;

/* Decode state, all device memory owned by the caller, for `capacity` tokens
 * per sequence (Tc below; a multiple of C).  hga_forward(HGA_PREFILL) fills
 * it when io.cache.k_rot is non-NULL; every hga_forward(HGA_DECODE) appends
 * one token per sequence and increments lens. */
typedef struct hga_kv_cache {
    int32_t capacity;  /* Tc                                                  */
    void *k_rot;       /* [B, Tc, Hkv, D] rotated keys                        */
    void *v;           /* [B, Tc, Hkv, D] values                              */
    int32_t *pos;      /* [B, Tc] positions of the cached tokens              */
    void *k_open;      /* [B, Hkv, C, D] raw keys of each sequence's open chunk
                          (needed for the low-frequency pairs when it closes) */
    float *s_chunk;    /* [B, Hkv, Tc/C, D]                                   */
    float *s_group;    /* [B, Hkv, Tc/g_s, D]                                 */
    int32_t *lens;     /* [B] tokens already cached                           */
} hga_kv_cache;

/* Inputs and outputs of hga_forward.  Unused members must be NULL. */
typedef struct hga_io {
    /* HGA_PREFILL */
    const void *q;             /* [B, T, Hq, D]                                */
    const void *k;             /* [B, T, Hkv, D] raw keys                      */
    const void *v;             /* [B, T, Hkv, D]                               */
    const int32_t *pos;        /* [B, T]                                       */
    /* HGA_DECODE: one new token per sequence, at index lens[b]               */
    const void *q_new;         /* [B, Hq, D]                                   */
    const void *k_new;         /* [B, Hkv, D] raw key                          */
    const void *v_new;         /* [B, Hkv, D]                                  */
    const int32_t *pos_new;    /* [B]                                          */
    /* outputs */
    void *out;                 /* prefill [B, T, Hq, D]; decode [B, Hq, D]     */
    float *lse;                /* optional: prefill [B, Hq, T]; decode [B, Hq] */
    int32_t *sel_chunk;        /* optional: prefill [B, NB, Hkv, K_c];
                                  decode [B, Hkv, K_c]                         */
    int32_t *sel_group;        /* optional: prefill [B, NB, Hkv, K_g];
                                  decode [B, Hkv, K_g]                         */
    hga_kv_cache cache;        /* decode: required; prefill: optional output   */
    /* HGA_PREFILL_HOSTKV only, optional: a HOST pointer to pinned, mapped
     * memory [B, Hkv, NC*C/g_s, D] f32 that holds the group summaries in the
     * cold tier (page section 3's store table puts them in host RAM beside
     * the token K/V).  Stage 1 writes them there over the link and stage 2
     * reads only the groups of each block's routed chunks over the link
     * (store operation "fetch group summaries"); NULL keeps them in the
     * workspace on the GPU. */
    float *s_group_host;
} hga_io;

/* Stage 1 — rotate keys and build mixed-RoPE summaries ("append closed
 * chunk").  Page section 3, "Mixed-RoPE Routing Summaries": for each closed
 * chunk and each g_s-token group, high-frequency pairs are the mean of the
 * per-token rotated keys; low-frequency pairs are the mean raw key rotated at
 * the set's mean position.  Also writes K_rot = RoPE(K) for attention.
 * k_rot may be NULL (summaries only).  Shapes as in the header comment. */
hga_status hga_build_summaries(const hga_dims *dims, const hga_params *prm,
                               const void *k_raw, const int32_t *pos,
                               void *k_rot, float *s_chunk, float *s_group,
                               void *stream);

/* Stage 2 — two-level routing per 64-token query block and KV head.  Page
 * section 3, "路由策略" (routing policy) and the selection equation: the
 * routing query is the block's RoPE-rotated queries summed over its tokens and
 * over the KV head's query heads; middle chunks F..b-L-1 (minus the forced
 * previous chunk when L == 0) are scored by q.c_m, the top K_c kept, their
 * groups scored by q.g_{m,g} and the top K_g kept.  Ties in score go to the
 * lower index.  Outputs sel_chunk / sel_group as in the header comment.
 * q_rot (bf16 only, may be NULL; HGA_ERR_UNSUPPORTED for fp32): when given,
 * [B, T, Hq, D] bf16 receives every query rotated at its position, rounded
 * as hga_attend rounds its own rotation, for hga_attend's q_rot. */
hga_status hga_route(const hga_dims *dims, const hga_params *prm,
                     const void *q, const int32_t *pos,
                     const float *s_chunk, const float *s_group,
                     int32_t *sel_chunk, int32_t *sel_group, void *q_rot, void *stream);

/* Stage 3 — exact softmax attention over the routed token set.  Page section
 * 3, "精确 Token 输出注意力" (exact token output attention) with eq. (1): each
 * query token i of block b attends, with scale 1/sqrt(D), to the union of
 * sink chunks 0..F-1, recent chunks b-L..b-1, chunk b-1, the tokens of
 * sel_group, and tokens b*C..i of its own chunk.  q is raw (pre-RoPE) and is
 * rotated inside; k_rot comes from hga_build_summaries.  lse may be NULL.
 * q_rot (bf16 only, may be NULL): the rotated queries hga_route wrote; the
 * tensor-core kernel then loads them as they are instead of rotating q (the
 * result is bit-identical), q is still required for the CUDA-core kernel.
 * Which kernel runs: bf16 with Hq/Hkv a power of two <= 16, g_s a multiple
 * of 8 and a visible set of at most 2048 8-token segments runs on the tensor
 * cores (tcgen05): with q_rot given, Hq/Hkv >= 4 and at most 1024 segments
 * as one persistent CTA per SM walking the (block, KV head, 256-row) units,
 * else one CTA per unit; fp32, and bf16 outside those limits, run on the
 * CUDA cores in fp32 arithmetic.  Both give the same result within rounding (bf16
 * outputs are rounded from fp32 accumulators). */
hga_status hga_attend(const hga_dims *dims, const hga_params *prm,
                      const void *q, const int32_t *pos,
                      const void *k_rot, const void *v,
                      const int32_t *sel_group, void *out, float *lse,
                      const void *q_rot, void *stream);

/* Backward of stage 3 (training through the routed attention).  Page
 * section 6, Tab. 8 (a training step through HGA attention) and Sec. 5.9
 * (QK fine-tuning through it in the exact-token mode).  The page prints no
 * formula; this is the derivative of eq. (1) restricted to each query's
 * visible set, the routed groups held fixed (routing is a discrete choice, so
 * no gradient reaches the summaries):
 *   P_ij = exp(q~_i . k~_j / sqrt(D) - LSE_i) over j in V(i) (q~, k~ rotated)
 *   dv_j = sum_i P_ij dO_i
 *   dS_ij = P_ij (dO_i . v_j - Delta_i),  Delta_i = sum_j P_ij dO_i . v_j
 *   dq_i = R_{p_i}^T sum_j dS_ij k~_j / sqrt(D)
 *   dk_j = R_{p_j}^T sum_i dS_ij q~_i / sqrt(D)
 * with i over the query rows of every query head of k_j's KV head.  Delta_i
 * equals dO_i . O_i; the library forms it from its own P and dO . v, so the
 * forward output is not an input (with a rounded output, the cancellation in
 * dO . v_j - Delta_i on rows whose weight sits on few keys would magnify its
 * rounding error).
 * Inputs: q (raw), pos, k_rot, v and sel_group as given to hga_attend; lse as
 * hga_attend returned it (required); d_out [B, T, Hq, D] in the dtype of q;
 * q_rot (bf16, may be NULL) the rotated queries hga_route wrote for the
 * forward, which spares the backward rotating q again (same results).  Outputs, fp32: dq [B, T, Hq, D] with respect to the raw
 * q, dk [B, T, Hkv, D] with respect to the RAW k (the rotation undone at each
 * key's position), dv [B, T, Hkv, D]; every element is written.  workspace:
 * hga_workspace_size(HGA_ATTEND_BACKWARD) bytes, 256-byte aligned.  bf16 with
 * the tensor-core forward's shape limits runs on the tensor cores (tcgen05),
 * everything else on the CUDA cores.  dk and dv are sums over units formed by
 * atomic additions, so their low bits may differ between runs. */
hga_status hga_attend_backward(const hga_dims *dims, const hga_params *prm,
                               const void *q, const int32_t *pos, const void *k_rot,
                               const void *v, const int32_t *sel_group, const float *lse,
                               const void *d_out, const void *q_rot, float *dq, float *dk,
                               float *dv, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Bytes of device workspace hga_forward (or, for HGA_ATTEND_BACKWARD,
 * hga_attend_backward) needs for `mode` (0 if none).  For HGA_PREFILL this
 * includes room for the rotated queries stage 2 hands to stage 3 (bf16
 * shapes of the tensor-core attention); hga_forward(HGA_PREFILL) also accepts
 * a workspace of hga_prefill_workspace_min bytes and then rotates the
 * queries inside stage 3 instead (same results). */
size_t hga_workspace_size(int mode, const hga_dims *dims, const hga_params *prm);

/* The smallest workspace hga_forward(HGA_PREFILL) accepts (0 if the
 * arguments are malformed): rotated keys, summaries and routed ids only. */
size_t hga_prefill_workspace_min(const hga_dims *dims, const hga_params *prm);

/* The whole path in one call.
 * HGA_PREFILL: stages 1-3 over the T prompt tokens (K_rot, summaries and
 *   selections live in the workspace unless io.cache / io.sel_* are given).
 *   With io.cache.k_rot set (capacity >= T), the cache is filled for decoding:
 *   K_rot, V, pos, summaries, the open chunk's raw keys, and lens = T.  With
 *   the cache set and io.q and io.out both NULL, only the cache is filled
 *   (stage 1; no routing or attention is computed).
 * HGA_DECODE: dims.T must equal io.cache.capacity.  For each sequence b, appends the new token at t = lens[b]
 *   (rotated key, value, position, raw key of the open chunk), builds the
 *   summaries of chunk t/C if t closes it (page section 3, store operation
 *   "append closed chunk"), routes with the token's own query (summed over the
 *   KV head's query heads), attends over the visible set of token t and
 *   increments lens[b].  Requires lens[b] < dims.T.  The attention over the
 *   keys routing does not choose (sinks, recent and current chunks) runs on
 *   a library-owned side stream (one per device, created on the first decode
 *   call) forked from and joined back into `stream` inside the call, so the
 *   caller sees ordinary stream order and can capture steps in a CUDA graph.
 * HGA_PREFILL_HOSTKV: the prefill of HGA_PREFILL with the token K/V history
 *   in host RAM (page section 3, the three-tier K/V store: the summaries stay
 *   on the GPU and only routed groups are fetched).  io.k and io.v are HOST
 *   pointers to pinned, mapped memory (cudaHostAlloc / cudaMallocHost /
 *   cudaHostRegister with mapping) holding raw K and V [B, T, Hkv, D]; q,
 *   pos and out (and lse, sel_chunk, sel_group when given) are device
 *   pointers; io.cache must be empty.  bf16 only, shapes the tensor-core
 *   attention takes (g_s a multiple of 8, Hq/Hkv a power of two <= 16).
 *   Stage 1 reads K over the host link once (with io.s_group_host set, it
 *   also writes the group summaries there, and stage 2 reads the routed
 *   chunks' group rows from there); stage 3 runs in waves of 32
 *   query blocks whose sink, recent and current K/V rows are fetched by the
 *   GPU over the link into two HBM staging buffers in the workspace, and
 *   whose routed groups go through a warm tier: a cache of routed groups in
 *   the workspace (page section 3's warm VRAM tier; CLOCK replacement) from
 *   which hits are read and into which misses are fetched.  The wave size
 *   and the cache's slots follow the workspace size (hga_hostkv_plan_for):
 *   by default 32 blocks and two waves' worth of groups per sequence and KV
 *   head (or all of them when fewer).
 *   This runs on a library-owned side stream (one per device, created on
 *   the first such call), the next wave's fetch overlapping this wave's
 *   attention; the call joins that stream back into `stream` before
 *   returning, so the caller sees ordinary stream order.  The cache lives
 *   for one call.  Host memory that is not pinned and
 *   mapped returns HGA_ERR_INVALID_ARG.  The outputs equal HGA_PREFILL's.
 * workspace: hga_workspace_size(mode) bytes of device memory, 256-byte
 * aligned (HGA_PREFILL_HOSTKV: any size from the plan's min_bytes up; see
 * hga_hostkv_plan_for).  For HGA_DECODE it must be zero-filled before its first use; the
 * library leaves it zeroed between calls.  Calls that share a workspace must
 * not overlap on the GPU. */
hga_status hga_forward(int mode, const hga_dims *dims, const hga_params *prm,
                       const hga_io *io, void *workspace, size_t workspace_bytes,
                       void *stream);

/* hga_forward(HGA_PREFILL) for callers that cannot allocate device memory.
 * The paper has no counterpart to this call: it is a convenience of this
 * library.  It is meant for code that only holds its inputs and outputs at
 * call time and may not call cudaMalloc then, for example a serving step
 * whose device memory belongs to another allocator or to a fixed arena
 * (a cudaMalloc there can fail, or stall the device mid-step), or a plug-in
 * that a host runtime hands nothing but tensors.
 *
 * Arguments are those of hga_forward(HGA_PREFILL) without a workspace: q, k,
 * v, pos and out as in the header comment, lse optional (NULL to skip).  The
 * scratch (rotated keys, summaries, routed ids) lives in one fixed 16 MiB
 * array inside the library's device image, which every GPU that loads the
 * library keeps until the process exits.  A shape whose scratch
 * (hga_prefill_workspace_min) exceeds 16 MiB is rejected with
 * HGA_ERR_WORKSPACE before anything is launched; about 14K tokens fit at
 * Hkv=4, D=128, bf16.  Nothing in the scratch needs to start at zero.
 *
 * The first call on a device, with that device current, looks up the
 * array's device address (cudaGetSymbolAddress) and caches it; make that
 * first call before any stream capture.  The cached address belongs to the
 * device's primary context as it was then: after cudaDeviceReset on that
 * device the address is stale, so do not call this entry point on a device
 * after resetting it (load the library in a fresh process instead).  All
 * calls share the one array:
 * calls that overlap on the GPU (other streams, other threads, without
 * ordering between them) race on it and give wrong results. */
hga_status hga_forward_prefill_noalloc(const hga_dims *dims, const hga_params *prm,
                                       const void *q, const void *k, const void *v,
                                       const int32_t *pos, void *out, float *lse, void *stream);

/* How HGA_PREFILL_HOSTKV uses a workspace of a given size: the warm tier
 * (page section 3's bounded VRAM cache of routed groups, which shrinks to
 * leave a configurable VRAM headroom) takes whatever the caller's workspace
 * holds.  hga_workspace_size(HGA_PREFILL_HOSTKV) is the default: waves of 32
 * query blocks and a cache of two waves' worth of routed groups per
 * (sequence, KV head).  A larger workspace keeps more groups cached (fewer
 * link bytes), up to every group of the sequence (max_bytes); a smaller one
 * shrinks the wave, and with it the staging buffers and the cache's floor of
 * two waves' worth, down to one query block per wave (min_bytes).  Outputs
 * are the same for every plan.  A caller that wants a headroom sizes the
 * workspace as the free device memory minus the headroom, clamped to
 * [min_bytes, max_bytes]. */
typedef struct hga_hostkv_plan {
    int32_t wave_blocks;   /* query blocks per wave                            */
    int32_t cache_slots;   /* warm-cache slots (one routed group each) per
                              (sequence, KV head)                              */
    size_t bytes;          /* workspace bytes this plan uses (0 if none fits)  */
    size_t min_bytes;      /* the smallest workspace any plan fits in          */
    size_t max_bytes;      /* the workspace that caches every group            */
} hga_hostkv_plan;

/* The plan hga_forward(HGA_PREFILL_HOSTKV) follows for workspace_bytes.
 * Host only.  Returns HGA_ERR_WORKSPACE (with min_bytes filled in) when the
 * workspace is below min_bytes; *plan must be a host pointer. */
hga_status hga_hostkv_plan_for(const hga_dims *dims, const hga_params *prm,
                               size_t workspace_bytes, hga_hostkv_plan *plan);

/* Status recorded by the kernels themselves since the last reset: a bounded
 * wait that gave up (HGA_ERR_TIMEOUT: the kernel recorded it, released what
 * it held and returned without finishing its tile) or a device-side index
 * check that refused an access (HGA_ERR_BOUNDS, e.g. a decode step for a
 * sequence whose lens[b] is outside [0, capacity); that sequence is skipped,
 * the others proceed).  Kernels never trap: a launch that met such a
 * condition still completes, and only this call reports it.  Waits for the
 * work already queued on `stream`, then reads the library's error words;
 * clear != 0 resets them.  Returns HGA_OK when none is set, the first set
 * status otherwise, or HGA_ERR_CUDA if the copies fail. */
hga_status hga_device_status(void *stream, int clear);

/* Bytes the host tier (HGA_PREFILL_HOSTKV) has moved over the host link
 * since the last reset: for stage 3 the K and V rows of sinks, windows and
 * the routed groups its warm cache did not hold; with the group summaries in
 * host memory also the summaries stage 1 wrote there and the group rows
 * stage 2 read (stage 1's single pass over K is not counted).  Waits for the work queued on `stream`; clear != 0 resets the
 * count.  *bytes must be a host pointer (HGA_ERR_INVALID_ARG if NULL). */
hga_status hga_hostkv_link_bytes(void *stream, unsigned long long *bytes, int clear);

/* Test hook, not for production use: exercises the bounded-wait timeout
 * path of a real kernel without a GPU fault.  With skip_summaries_copy != 0
 * the summaries kernel (stage 1, device-memory keys) does not issue the bulk
 * copy of its keys, so its wait for them runs out after summaries_wait_ns
 * (0 = the default limit of 2 s); the kernel then records HGA_ERR_TIMEOUT
 * (read by hga_device_status) and returns with nothing in flight, and its
 * outputs are left unwritten.  hga_set_test_hooks(0, 0, stream) restores
 * normal operation.  The settings are per device and apply to every call
 * that follows; the call waits for `stream`. */
hga_status hga_set_test_hooks(int skip_summaries_copy, unsigned long long summaries_wait_ns,
                              void *stream);

/* Static description of a status code. */
const char *hga_status_string(hga_status s);

/* The last CUDA error code seen by a failing call on this thread (0 = none). */
int hga_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* HGA_H */
