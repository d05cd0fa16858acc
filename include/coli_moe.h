/*
 * coli_moe.h -- C ABI of the B200 (sm_100a) quantised Mixture-of-Experts layer.
 *
 * One MoE decoder layer of a GLM-5.2-class model as the pages describe it:
 *   [HN] "Show HN: 遅いコンピュータで GLM 5.2 を実行する" (ja.news.hada.io/topic?id=31297),
 *        section "実装済みの主な機能" (implemented features):
 *          router bullet       -- DeepSeek-V3-style sigmoid router, noaux_tc,
 *                                 routed_scaling_factor, shared expert;
 *          integer-dot bullet  -- Q8_0-style int8 activations, integer dot;
 *          quantisation bullet -- int8 / packed int4 / packed int2 weights with
 *                                 per-row scales, dequantised on use;
 *          batch-union bullet  -- each distinct expert of a batch is read once
 *                                 and applied to every position routed to it.
 *   [DT] "Comment exécuter un réseau de neurones de 744 milliards de paramètres
 *        sur un ordinateur ordinaire" (devtrends.cc), section "Comment fonctionne
 *        le moteur": requests for identical experts are merged; an expert is its
 *        gate, up and down matrices, read together.
 *
 * Conventions shared by every entry point:
 *   - Pointers named *_host are host memory; every other pointer is device
 *     memory of the current CUDA device.  Device pointers must be 16-byte
 *     aligned.  The library never frees memory it did not allocate.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and never synchronises the host, except
 *     coli_moe_forward_host, which returns with its result in host memory.
 *   - Argument errors are detected on the host before any launch and return
 *     COLI_EINVAL with nothing enqueued; launch failures return COLI_ECUDA.
 *     coli_last_error() gives a one-line message for the calling thread.
 *     Nothing throws across this boundary.
 *   - A coli_moe handle is not thread-safe: use one handle per stream.
 *   - NaN or Inf inputs give unspecified (but memory-safe) results.
 *
 * Numerics (identical on every path):
 *   Q8_0: d = amax/127 rounded to fp32; q = clamp(round-half-even(x/d), +-127)
 *         with IEEE fp32 division; amax == 0 gives d = 0, q = 0.
 *   int dot: per 32-block integer sums S_b (exact int32); acc = sum_b S_b*d_b
 *         in fp64 (each product exact); value = (float)(acc * row_scale).
 *   router: fp64 logits of fp32 inputs, fp64 sigmoid and selection.
 *   SwiGLU: h = (float)(g/(1+exp(-g)) * u) in fp64.
 *   combine: fp64, shared experts first (weight 1), then routed slots in order.
 */
#ifndef COLI_MOE_H
#define COLI_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define COLI_ABI_VERSION 2

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *coli_stream_t;

typedef enum {
    COLI_OK = 0,
    COLI_EINVAL = 1,       /* bad argument: null/misaligned pointer, bad size or shape */
    COLI_ENOMEM = 2,       /* device allocation failed */
    COLI_ECUDA = 3,        /* a CUDA call or kernel launch failed */
    COLI_EUNSUPPORTED = 4, /* valid request this build does not implement */
    COLI_ETIMEOUT = 5      /* a bounded device-side wait gave up */
} coli_status;

/* Weight code formats ([HN] quantisation bullet).  Codes are two's complement
 * inside their field, the lowest-indexed element in the lowest bits:
 *   COLI_W_INT8: one code per byte, [-127, 127], scale = amax/127
 *   COLI_W_INT4: two per byte (element 2j in the low nibble of byte j),
 *                [-8, 7], scale = amax/7
 *   COLI_W_INT2: four per byte (element 4j+i in bits 2i..2i+1 of byte j),
 *                [-2, 1], scale = amax/2 (so +amax saturates to +1) */
typedef enum { COLI_W_INT8 = 8, COLI_W_INT4 = 4, COLI_W_INT2 = 2 } coli_wfmt;

/* Shape of one layer.
 *   hidden (H), inter (I): multiples of 32 (of 64 for COLI_W_INT2), <= 16384.
 *   n_routed (E) in [1, 1024], n_shared (S) in [0, 4].
 *   n_group (G) divides E; topk_group (gk) in [1, G];
 *   top_k (k) in [1, min(32, gk*E/G)].
 *   A dense layer ([HN] router bullet: the first three layers are dense) is
 *   E = 0 with k = 0 and S >= 1 (G and gk ignored): every token through the
 *   shared experts only; its router pointers may be NULL.
 *   max_tokens: largest T any call on this handle will pass, >= 1.
 *   expert_top_p: adaptive expert top-p ([HN] モデルのダウンロードと実行,
 *     --topp; 0 or >= 1: off).  For p in (0, 1), after the group-limited
 *     top-k the selected experts are kept by descending sigmoid score (ties:
 *     the earlier slot) while the kept scores sum to less than p times the
 *     top-k's score sum, the first always; the other slots are dropped
 *     (idx -1, weight 0, no expert computed) and the weights renormalised
 *     over the kept experts. */
typedef struct {
    int hidden, inter, n_routed, n_shared, top_k, n_group, topk_group;
    float routed_scaling_factor;
    int wfmt; /* a coli_wfmt */
    int max_tokens;
    float expert_top_p;
} coli_moe_config;

/* One quantised matrix: codes [rows][K*bits/8] bytes, row-major with K
 * contiguous; scales [rows] fp32.  Device pointers. */
typedef struct {
    const void *codes;
    const float *scales;
} coli_qmat;

/* One SwiGLU expert ([DT]): gate and up are [I][H], down is [H][I]. */
typedef struct {
    coli_qmat gate, up, down;
} coli_expert;

typedef struct coli_moe coli_moe; /* opaque */

const char *coli_status_str(coli_status s);
/* Message for the calling thread's last failed call ("" if none). */
const char *coli_last_error(void);
int coli_abi_version(void);

/* Q8_0 quantisation of rows of activations ([HN] integer-dot bullet).
 *   x [rows][len] fp32 -> q [rows][len] int8, d [rows][len/32] fp32.
 *   len % 32 == 0; rows >= 0 (rows == 0 is a no-op). */
coli_status coli_quant_q8(const float *x, int64_t rows, int64_t len, int8_t *q, float *d,
                          coli_stream_t stream);

/* Per-row weight quantisation and packing ([HN] quantisation bullet).
 *   w [rows][K] fp32 -> codes [rows][K*wfmt/8] bytes, scales [rows] fp32.
 *   K % 32 == 0 (K % 64 == 0 for COLI_W_INT2). */
coli_status coli_quant_weights(const float *w, int64_t rows, int64_t K, int wfmt, void *codes,
                               float *scales, coli_stream_t stream);

/* FP8 checkpoint weights -> per-row weight format ([HN] 実装済みの主な機能,
 * offline-converter bullet: the FP8 shards are dequantised with 128 x 128
 * block scales, then requantised into the engine's container).
 *   w_fp8 [rows][K] one e4m3 code per byte (1 sign, 4 exponent bits with
 *     bias 7, 3 mantissa bits, no infinities, S.1111.111 NaN); device,
 *     16-byte aligned;
 *   block_scale [ceil(rows/block)][ceil(K/block)] fp32, device: the block's
 *     multiplier, w = fp32(e4m3(code) * block_scale[r/block][k/block]);
 *   block: a positive multiple of 16 (the checkpoints use 128);
 *   -> codes [rows][K*wfmt/8], scales [rows] exactly as coli_quant_weights
 *     of the dequantised rows.
 *   K % 32 == 0 (K % 64 == 0 for COLI_W_INT2); rows == 0 is a no-op.  NaN
 *   codes give unspecified (memory-safe) results. */
coli_status coli_requant_fp8(const void *w_fp8, const float *block_scale, int64_t rows, int64_t K,
                            int64_t block, int wfmt, void *codes, float *scales,
                            coli_stream_t stream);

/* Create a layer handle ([HN] router and batch-union bullets).
 *   router_w [E][H] fp32 and bias [E] fp32 (e_score_correction_bias) are
 *   device pointers; experts is a HOST array of E + S coli_expert records
 *   (routed experts 0..E-1, then the shared experts) holding device pointers.
 *   All of them are borrowed: they must stay valid and unchanged for the
 *   handle's lifetime; nothing is copied or repacked.  The handle allocates
 *   its own device workspace, sized by max_tokens.  On failure *out is NULL. */
coli_status coli_moe_create(const coli_moe_config *cfg, const float *router_w, const float *bias,
                            const coli_expert *experts, coli_moe **out);

/* Routing only ([HN] router bullet):  x [T][H] fp32 ->
 *   idx [T][k] int32: selected experts sorted by descending choice score
 *                     c = sigmoid(x.W_r) + bias (ties: lower index); -1 for a
 *                     slot the adaptive expert top-p dropped;
 *   w   [T][k] fp32:  sigmoid scores of idx renormalised to sum 1, times
 *                     routed_scaling_factor (the bias is not in w).
 * Group-limited: a group's score is the sum of its two best c; only the
 * topk_group best groups are eligible.  1 <= T <= max_tokens. */
coli_status coli_router(coli_moe *m, const float *x, int T, int32_t *idx, float *w,
                        coli_stream_t stream);

/* The whole layer ([HN] router, integer-dot, quantisation and batch-union
 * bullets; [DT] expert = gate, up, down):
 *   out[t] = sum_shared e_s(x_t) + sum_j w[t][j] * e_{idx[t][j]}(x_t)
 *   e(x) = down . Q8_0( SwiGLU( gate . Q8_0(x), up . Q8_0(x) ) )
 * x [T][H] fp32 (device), out [T][H] fp32 (device, overwritten; must not
 * alias x).  1 <= T <= max_tokens.
 * Execution (results are the same to the stated tolerance on every path):
 * T <= 8 runs one persistent cooperative kernel when the shared-memory plan
 * fits; larger T runs the router kernels and grouped expert GEMMs on the
 * tensor cores (tcgen05 int8 MMA) when hidden and inter are multiples of
 * 256, else CUDA-core grouped kernels.  Setting COLI_NO_TC=1 in the
 * environment before coli_moe_create keeps the CUDA-core grouped kernels
 * for that handle. */
coli_status coli_moe_forward(coli_moe *m, const float *x, int T, float *out,
                             coli_stream_t stream);

/* coli_moe_forward from and to HOST memory: copies x_host [T][H] in, runs
 * the layer, copies out_host [T][H] back and synchronises `stream` before
 * returning.  Pinned host buffers make the copies asynchronous DMA;
 * pageable buffers also work, more slowly. */
coli_status coli_moe_forward_host(coli_moe *m, const float *x_host, int T, float *out_host,
                                  coli_stream_t stream);

/* Expert parallelism over several GPUs (one handle per GPU): the layer's
 * routed experts are split into contiguous ranges, one per GPU, the router
 * is replicated and one GPU also computes the shared experts; every GPU's
 * partial output covers the (token, expert) pairs it owns, and the partials
 * are summed in a fixed GPU order.  ("Comment exécuter un réseau de neurones
 * de 744 milliards de paramètres sur un ordinateur ordinaire", devtrends.cc,
 * "Les chiffres réels de vitesse": six GPUs keep the experts entirely in
 * video memory; the pages do not say how they are split.)
 *
 * coli_moe_set_experts: later forwards on this handle compute only routed
 *   experts e_lo <= e < e_hi and, if own_shared, the shared experts (every
 *   token still routes over all experts).  Expert weights outside the range
 *   are never read, so they may be placeholders.  0 <= e_lo <= e_hi <= E.
 *
 * coli_moe_forward_partial: as coli_moe_forward, but writes the fp64 sum of
 *   this handle's slots, unrounded, shared experts first and then routed
 *   slots in order:  y_partial[t][r] = sum_{owned shared} e + sum_{owned j}
 *   w[t][j] e_j  (device, [T][H] fp64, 16-byte aligned, not aliasing x).
 *
 * coli_combine_partials: out[i] = (float)(parts[0][i] + parts[1][i] + ...)
 *   in fp64 in part order; parts is [n_parts][n] fp64 (device), out [n] fp32.
 *   With one part holding every expert the result equals coli_moe_forward
 *   bit for bit; with several it differs only in the association of the fp64
 *   sum (the same for every call: deterministic). */
coli_status coli_moe_set_experts(coli_moe *m, int e_lo, int e_hi, int own_shared);
coli_status coli_moe_forward_partial(coli_moe *m, const float *x, int T, double *y_partial,
                                     coli_stream_t stream);
coli_status coli_combine_partials(const double *parts, int n_parts, int64_t n, float *out,
                                  coli_stream_t stream);

/* Release the handle and its workspace (not the borrowed weights).  Waits for
 * work already enqueued on the handle's last stream.  NULL is a no-op. */
void coli_moe_destroy(coli_moe *m);

/* Bytes of device workspace coli_moe_create would allocate (0 if cfg is invalid). */
size_t coli_moe_workspace_bytes(const coli_moe_config *cfg);

/* Synchronise `stream` and report device-side failures of earlier calls on
 * this handle: every wait inside the library's kernels is bounded (about one
 * second); a wait that gives up records COLI_ETIMEOUT in the handle's error
 * word and its kernel returns early, leaving that call's outputs undefined.
 * Returns COLI_ETIMEOUT (and clears the word) if that happened, else COLI_OK. */
coli_status coli_moe_device_status(coli_moe *m, coli_stream_t stream);

/* Kernel launches made by this library in this process so far. */
uint64_t coli_launch_count(void);

/* Optional per-kernel timing with CUDA events on the launching stream.
 * While enabled, every kernel of coli_moe_forward is bracketed by events;
 * coli_moe_profile_read synchronises on them and returns, per kernel name,
 * the launches and summed milliseconds since the last read. */
typedef struct {
    const char *name; /* static string */
    int launches;
    double ms;
} coli_kernel_time;
coli_status coli_moe_profile(coli_moe *m, int enable);
coli_status coli_moe_profile_read(coli_moe *m, coli_kernel_time *out, int max_entries,
                                  int *n_entries);

/* ---------------------------------------------------------------------------
 * Parity exports (used by the tests; same library, prefixed coli_dbg_).
 * ------------------------------------------------------------------------ */

/* Integer block sums of one matrix against T Q8_0 vectors ([HN] integer-dot
 * bullet):  S[t][r][b] = sum_{k in block b} code[r][k] * xq[t][k]  (int32).
 *   codes [rows][K*wfmt/8], xq [T][K] int8 -> S [T][rows][K/32] int32. */
coli_status coli_dbg_block_sums(const void *codes, int wfmt, int64_t rows, int64_t K,
                                const int8_t *xq, int T, int32_t *S, coli_stream_t stream);

/* The routing decision and the intermediate Q8_0(h) of the last
 * coli_moe_forward on this handle, per (token, slot): slot j < k is routed
 * slot j, slot k + i is shared expert i.
 *   idx [T][k] int32, w [T][k] fp32, hq [T][k+S][I] int8, hd [T][k+S][I/32]
 *   fp32 (device).  Any output may be NULL.  T must equal that call's T. */
coli_status coli_dbg_last_forward(coli_moe *m, int T, int32_t *idx, float *w, int8_t *hq,
                                  float *hd, coli_stream_t stream);

/* Routing that allocates nothing (no counterpart on the pages; the pages'
 * engine runs on the CPU and never faces this).  Same result as coli_router
 * for the same inputs, but without a coli_moe handle: the router's scratch
 * (fp64 sigmoid and choice scores and a completion ticket) lives in one
 * fixed array inside the library instead of a workspace that
 * coli_moe_create would cudaMalloc.  It is for callers that cannot allocate
 * device memory at the point where they route: a process whose memory is
 * already handed out to a caching allocator or a fixed budget, or a
 * latency-critical loop that cannot take cudaMalloc's implicit
 * synchronisation.  The call itself makes no cudaMalloc, cudaFree or other
 * allocating call.
 *   cfg:      layer shape (only hidden, n_routed, n_shared, top_k, n_group,
 *             topk_group and routed_scaling_factor are used; the config must
 *             still be valid as for coli_moe_create);
 *   router_w [E][H], bias [E], x [T][H] fp32 device pointers;
 *   idx [T][k] int32, w [T][k] fp32 device outputs, as coli_router.
 * Limits: 1 <= T <= 8 tokens and n_routed <= 1024; larger requests return
 * COLI_EINVAL.  The fixed array holds 131,328 bytes on every GPU that loads
 * the library, until the process exits.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current.  Every call on a device
 * shares the one array and it keeps the last call's contents (the ticket is
 * cleared at the start of each call): calls that overlap on the GPU, e.g. on
 * two streams, race.  A dense layer (n_routed = 0) returns COLI_EINVAL. */
coli_status coli_router_static(const coli_moe_config *cfg, const float *router_w,
                               const float *bias, const float *x, int T, int32_t *idx, float *w,
                               coli_stream_t stream);

/* Test hook for the bounded waits of the layer's own kernels (no counterpart
 * on the pages).  Sets how many SM cycles a wait on another part of a kernel
 * may last before that kernel gives up (records COLI_ETIMEOUT in the handle's
 * error word, leaves without finishing the call, and the call's outputs are
 * undefined); cycles <= 0 restores the default of about one second.  Waits for
 * work already issued (bulk copies, tensor-core MMAs) keep the default, so a
 * kernel that gives up still leaves no copy in flight and no tensor memory
 * held.  Applies to later calls on this handle; returns once the new limit is
 * in place. */
coli_status coli_dbg_set_wait_limit(coli_moe *m, long long cycles, coli_stream_t stream);

/* Test hook for the bounded waits (no counterpart on the pages): one thread
 * waits on an mbarrier that nothing ever arrives at, through the same bounded
 * wait the pipelined kernels use.  The wait gives up after about one second
 * and records COLI_ETIMEOUT in the handle's error word, which the next
 * coli_moe_device_status reports.  Nothing faults or hangs. */
coli_status coli_dbg_wait_probe(coli_moe *m, coli_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* COLI_MOE_H */
