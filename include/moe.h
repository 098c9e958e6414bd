/* split_weight_b200: the data-parallel MoE expert block of DWDP on one B200.
 *
 * DWDP ("DWDP: Distributed Weight Data Parallelism for High-Performance LLM
 * Inference on NVL72", arXiv 2604.01621, abstract) keeps every GPU data
 * parallel: a rank runs the MoE block on its own tokens, and only the expert
 * weights are split between peers, the missing ones being fetched
 * asynchronously instead of through a layer-boundary collective.  The
 * explainer "Distributed Weight Data Parallelism cuts LLM inference stalls"
 * shows (split-weight figure) that the local and remote expert weights have
 * to reach the grouped GEMM; this library reaches them through a per-expert
 * (pool, slot) table spanning both pools, with no merge copy, and prefetches
 * the next layer's remote experts into an alternate buffer on a copy-engine
 * stream (prefetch-timeline figure).
 *
 * One layer, all calls enqueued on one compute stream:
 *   moe_route -> moe_permute -> moe_grouped_ffn -> moe_combine
 * and, on a copy stream, moe_prefetch_layer for a later layer.
 *
 * Conventions (all entry points):
 *   - Every function returns a moe_status; nothing aborts, exits or traps.
 *     moe_last_error() gives a thread-local description of the last failure.
 *   - Shapes, pointers and alignment are checked on the host before any
 *     launch; a bad argument returns MOE_ERR_INVALID_ARG (or
 *     MOE_ERR_UNSUPPORTED for a legal but unimplemented case) and enqueues
 *     nothing.
 *   - The caller owns all memory.  The library allocates no device memory;
 *     calls that need scratch take (workspace, workspace_bytes), sized by the
 *     matching *_workspace_size query; too small -> MOE_ERR_WORKSPACE.
 *   - Device pointers must be 16-byte aligned.  Every call is asynchronous on
 *     the given stream and never synchronises.  Errors of the launch itself
 *     return MOE_ERR_CUDA; faults inside a kernel surface at the caller's
 *     next synchronisation.  Kernels never wait without a time limit: a wait
 *     that runs out sets the device error word that moe_check_device() reads
 *     (MOE_ERR_TIMEOUT) and the kernel returns.
 *   - Matrices are row-major.  bf16 is IEEE bfloat16, e4m3 is the OCP FP8
 *     E4M3 "fn" format (max 448, no infinities).
 */
#ifndef SPLIT_WEIGHT_B200_MOE_H
#define SPLIT_WEIGHT_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_TIMEOUT = 5,
    MOE_ERR_DEVICE_CHECK = 6
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2 } moe_dtype;

typedef enum moe_score { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score;

/* Static text for a status code. */
MOE_API const char *moe_status_string(moe_status s);
/* Thread-local description of the last failing call ("" if none). */
MOE_API const char *moe_last_error(void);
/* MOE_ABI_VERSION of the loaded library. */
MOE_API int32_t moe_abi_version(void);
/* Number of kernels this library has launched in this process (all threads,
 * all devices), counted after each launch the runtime accepted.  Copies
 * issued by moe_prefetch_layer are not kernels and are not counted.  A
 * caller takes the difference of two readings around a region of calls. */
MOE_API uint64_t moe_kernel_launches(void);

/* ------------------------------------------------------------------------
 * Routing: router logits, scores and top-k selection.
 *
 * The pages run "the MoE expert layer" of DeepSeek-R1 on every rank (arXiv
 * 2604.01621, abstract; explainer, first figure) but give no router
 * arithmetic; this is the DeepSeek-R1 layer shape read plainly:
 *   logits  l[t,e] = sum_h x[t,h] W_g[e,h] in fp32, in a fixed order: h in
 *           chunks of 256, each a chain of fused multiply-adds from 0 in
 *           ascending h, the chunk sums added in ascending order.
 *   SOFTMAX: the k largest logits; w_j = exp(l_j - l_max) / sum over the k
 *           chosen (renormalize != 0) or over all E (renormalize == 0).
 *   SIGMOID: s = sigmoid(l) (evaluated in fp64, rounded to fp32); selection
 *           key s + bias[e] (fp32); groups are n_group contiguous blocks of
 *           E/n_group experts scored by the sum of their two largest keys;
 *           the topk_group best groups are kept and the k best keys inside
 *           them chosen; w_j = s_j / sum_i s_i (fp32, i in output order) when
 *           renormalize != 0, else s_j.
 *   Both: w_j *= routed_scale.  Ties go to the lower index everywhere.
 * Results are bit-for-bit reproducible (the exponent of the sigmoid is this
 * library's own fp64 routine).
 *
 * x        [T, H] device, dtype MOE_F32 or MOE_BF16.
 * w_gate   [E, H] fp32 device.   bias [E] fp32 device or NULL (SIGMOID only).
 * topk_idx [T, k] int32 out, experts in descending key order.
 * topk_w   [T, k] fp32 out.
 * Limits: 1 <= E <= 1024, 1 <= k <= 32, H % 32 == 0, T >= 0;
 *         SIGMOID: E % n_group == 0, n_group <= 32,
 *                  1 <= topk_group <= n_group, k <= topk_group * E / n_group.
 * ---------------------------------------------------------------------- */
typedef struct moe_route_cfg {
    int32_t T, H, E, k;
    int32_t score;       /* moe_score */
    int32_t n_group;     /* SIGMOID: number of expert groups (1 = no grouping) */
    int32_t topk_group;  /* SIGMOID: groups kept per token */
    float routed_scale;  /* multiplies every routing weight */
    int32_t renormalize; /* see above */
} moe_route_cfg;

/* Workspace of moe_route (device, 16-byte aligned): the fp32 logits [T, E],
 * or, when the logits kernel splits the h chunks over its grid (small and
 * large batches), one [T, E] plane per 256-wide chunk, ceil(H/256) planes,
 * summed in chunk order by the call (about 235 MB at T = 8192, H = 7168,
 * E = 256).  0 for an invalid cfg. */
MOE_API size_t moe_route_workspace_size(const moe_route_cfg *cfg);
MOE_API moe_status moe_route(const moe_route_cfg *cfg, const void *x, moe_dtype x_dtype,
                     const float *w_gate, const float *bias, int32_t *topk_idx, float *topk_w,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Permutation: expert histogram, scan, stable scatter and row gather.
 *
 * Groups each rank's token-expert assignments by expert so that one grouped
 * GEMM serves all of them (explainer, split-weight figure: the grouped GEMM
 * of the block).  With a = t*k + j the assignments in ascending order:
 *   offsets[e]  = number of assignments to experts < e   ([E+1], offsets[E] = T*k)
 *   row of a    = offsets[e] + #{a' < a with the same expert}   (stable)
 *   perm_src[row] = t,  inv_pos[t,j] = row
 *   x_perm[row]   = x[t] converted to perm_dtype;
 *   with_shared != 0: rows T*k .. T*k+T-1 of x_perm are x[0..T-1] (input of
 *   the always-on shared expert).
 * perm_dtype MOE_BF16: x_perm [rows, H] bf16 (fp32 x is rounded to nearest
 * even).  perm_dtype MOE_E4M3: x_perm [rows, H] e4m3 plus x_perm_scales
 * [H/128, rows] fp32 (one row of scales per 128-column block, so a block's
 * scales for consecutive rows are contiguous): per row and 128 columns
 * s = amax/448, code = e4m3(v/s).
 * topk_idx entries must lie in [0, E).  This is checked on the device: an
 * entry outside sets the device error word (moe_check_device() then returns
 * MOE_ERR_DEVICE_CHECK) and is skipped.  A skipped assignment has no row:
 * offsets[E] is then less than T*k, its inv_pos entry is -1, the rows
 * offsets[E] .. T*k-1 of perm_src are left unwritten and the same rows of
 * x_perm hold no defined value.  The gather checks every perm_src value
 * against [0, T) before it reads x: a value outside is reported the same way
 * and its row is zero-filled, so x is never read out of bounds.
 * Limits: H % 128 == 0, 1 <= E <= 1024, 1 <= k <= 32.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_permute_workspace_size(int32_t T, int32_t k, int32_t E);
MOE_API moe_status moe_permute(int32_t T, int32_t k, int32_t E, int32_t H, const int32_t *topk_idx,
                       const void *x, moe_dtype x_dtype, moe_dtype perm_dtype, int32_t with_shared,
                       int32_t *offsets, int32_t *perm_src, int32_t *inv_pos, void *x_perm,
                       float *x_perm_scales, void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/* Allocation-free moe_permute.  The DWDP pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory, not
 * even a workspace of their own - for example a plug-in inside a host
 * application or serving runtime that has reserved all device memory for its
 * own pool and forbids any other allocation, or code on a latency-critical
 * path where a cudaMalloc (which may synchronise the whole device) is not
 * allowed.
 *
 * Same arguments and results as moe_permute without (workspace,
 * workspace_bytes): the scratch lives in a fixed 1 MiB array in the
 * library's device code module.  CUDA places it on a device when it loads
 * that module there (with the default lazy module loading, at the first
 * permutation call or symbol lookup on that device, not when the library is
 * opened); from then on that GPU holds it until the process exits.  The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 * Arguments are checked as in moe_permute before any CUDA call is made.
 *   - Limit: moe_permute_workspace_size(T, k, E) <= 1 MiB, i.e.
 *     8 * ceil(T*k / 2048) * E bytes (E = 256: up to 1,048,576 token-expert
 *     assignments).  Larger sizes return MOE_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each word is written before it is
 *     read within a call).  Calls that overlap on the GPU (other streams,
 *     other host threads) race on it: serialise them. */
MOE_API moe_status moe_permute_noalloc(int32_t T, int32_t k, int32_t E, int32_t H,
                               const int32_t *topk_idx, const void *x, moe_dtype x_dtype,
                               moe_dtype perm_dtype, int32_t with_shared, int32_t *offsets,
                               int32_t *perm_src, int32_t *inv_pos, void *x_perm,
                               float *x_perm_scales, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Expert weight images and the split-weight table.
 *
 * One expert image (a "slot") holds, at the offsets moe_expert_layout_get
 * returns: w_gu [2I, H] (gate rows 0..I-1, up rows I..2I-1) and w_down
 * [H, I], both row-major in w_dtype; for MOE_E4M3 also fp32 block scales
 * s_gu [2I/128, H/128] and s_down [H/128, I/128] (weight = code * scale).
 * A pool is `count` slots `stride` bytes apart (stride >= layout.bytes,
 * stride % 256 == 0, base 1024-byte aligned).
 *
 * The table spans two pools that need not be adjacent or related in any way
 * (the explainer's split-weight figure: local and remote weights reach the
 * grouped GEMM without being merged into one contiguous buffer):
 *   pool_slot[e] = (pool << 31) | slot,  pool 0 = local, pool 1 = remote.
 * pool_slot is a HOST array of E entries, read during the call.
 * ---------------------------------------------------------------------- */
typedef struct moe_expert_layout {
    int64_t gu_offset, down_offset;             /* bytes from the slot start */
    int64_t gu_scale_offset, down_scale_offset; /* -1 unless MOE_E4M3 */
    int64_t bytes;                              /* bytes of one image (256-byte multiple) */
} moe_expert_layout;

MOE_API moe_status moe_expert_layout_get(int32_t H, int32_t I, moe_dtype w_dtype, moe_expert_layout *out);

typedef struct moe_expert_table {
    const void *local_base;
    int32_t local_count;
    int64_t local_stride;
    const void *remote_base;
    int32_t remote_count;
    int64_t remote_stride;
    const void *shared;        /* one image of the shared expert, or NULL */
    const int32_t *pool_slot;  /* HOST [E] */
} moe_expert_table;

/* ------------------------------------------------------------------------
 * Grouped SwiGLU expert FFN over the split pools (the block's grouped GEMM;
 * explainer, split-weight figure).
 *
 * For every routed expert e with n_e = offsets[e+1] - offsets[e] > 0 and,
 * when has_shared, for the shared expert on rows T*k .. T*k+T-1:
 *   G = X_e W_gu[e]^T                     X_e = x_perm rows of e
 *   h = silu(G[:, :I]) * G[:, I:]         -> h rows of e   (act_dtype)
 *   y = h W_down[e]^T                     -> y_perm rows of e (bf16)
 * fp32 accumulation on the tensor cores.
 * x_perm  [rows, H] act_dtype (rows = T*k + (has_shared ? T : 0)).
 * h       [rows, I] act_dtype (intermediate, caller-owned).
 * y_perm  [rows, H] bf16 out.
 * Supported (w_dtype, act_dtype):
 *   MOE_BF16 / MOE_BF16  bf16 weights and activations, bf16 tensor-core MMA.
 *   MOE_E4M3 / MOE_BF16  e4m3 weights (code x fp32 128x128 block scale), bf16
 *                        activations: the weights are dequantised to bf16 in
 *                        shared memory and the bf16 MMA runs.
 *   MOE_E4M3 / MOE_E4M3  both GEMMs on the fp8 tensor cores.  x_perm is e4m3
 *                        with x_perm_scales [H/128, rows] fp32 as moe_permute
 *                        writes them (x = code x scale per row and 128
 *                        columns); h is e4m3 [rows, I] and its scales
 *                        [I/128, rows] fp32 go to the workspace, which must
 *                        hold moe_grouped_ffn_workspace_size(d) bytes.
 *                        Requires H % 256 == 0.
 * x_perm_scales is ignored (may be NULL) in the two bf16-activation
 * combinations.  There the workspace is optional: with
 * moe_grouped_ffn_workspace_size(d) bytes (16-byte aligned) the kernels
 * take their tiles from two counters in it, each CTA the next tile when it
 * is ready for one, which balances tiles of unequal size; with NULL (or
 * fewer bytes) each CTA takes a fixed round-robin share.  The results are
 * the same bits either way.  A workspace serves one call at a time.
 * Limits: H % 128 == 0, I % 128 == 0, 1 <= E <= 1024, 1 <= k <= 32.
 * ---------------------------------------------------------------------- */
typedef struct moe_ffn_desc {
    int32_t T, H, I, E, k;
    int32_t w_dtype;    /* moe_dtype of the expert weights */
    int32_t act_dtype;  /* moe_dtype of x_perm */
    int32_t has_shared; /* shared expert present */
} moe_ffn_desc;

MOE_API size_t moe_grouped_ffn_workspace_size(const moe_ffn_desc *d);
MOE_API moe_status moe_grouped_ffn(const moe_ffn_desc *d, const moe_expert_table *tbl, const void *x_perm,
                           const float *x_perm_scales, const int32_t *offsets, void *h,
                           void *y_perm, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* Per-expert readiness (explainer, prefetch caption: the fetch of a layer's
 * remote experts runs while the rank computes; here the grouped GEMM may
 * start before the fetch has finished).  With a gate, moe_grouped_ffn_gated
 * does not need the fetch's ready event: before the first weight load of a
 * tile of a REMOTE-pool expert in slot s it waits until
 *   (int32_t)(flags[s / slots_per_flag] - epoch) >= 0
 * i.e. until moe_prefetch_layer_flagged has landed the chunk that holds s.
 * Tiles run local experts first, then the shared one, then remote experts in
 * slot order, the order a fetch fills them in.  The wait polls with a time
 * limit (timeout_ns; 0 = 2 s); if it runs out the kernels stop early, the
 * outputs are undefined and moe_check_device() reports MOE_ERR_TIMEOUT.
 * flags: device, n_flags words, 4-byte aligned, written only by the copy
 * stream.  A NULL gate (or moe_grouped_ffn) reads the remote pool as it is:
 * the caller orders the fetch before the call (e.g. with the ready event).
 * The waiting CTAs (one per SM) must leave room on their SMs for the fetch:
 * between two buffers of one GPU cudaMemcpyAsync runs as a copy kernel on
 * the SMs.  A gated call whose kernel would hold more than 55,296 registers
 * per SM (the most measured to leave the copy running) returns MOE_ERR_CUDA
 * instead of launching it; every kernel of this library is within it. */
typedef struct moe_ready_gate {
    const uint32_t *flags;
    uint32_t epoch;
    int32_t slots_per_flag;  /* remote slots per flag (a flag covers one copy chunk) */
    int32_t n_flags;         /* >= ceil(remote_count / slots_per_flag) */
    int64_t timeout_ns;
} moe_ready_gate;

MOE_API moe_status moe_grouped_ffn_gated(const moe_ffn_desc *d, const moe_expert_table *tbl,
                                 const moe_ready_gate *gate, const void *x_perm,
                                 const float *x_perm_scales, const int32_t *offsets, void *h,
                                 void *y_perm, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream);

/* moe_grouped_ffn_gated with GEMM1's token rows read from x itself instead
 * of x_perm: the row gather of moe_permute is fused into the GEMM's operand
 * load (TMA tile::gather4 through perm_src), so x_perm need not be written
 * (moe_permute with x_perm = NULL).  Routed row r of expert e reads
 * x[perm_src[r]]; the shared expert's rows are x[0 .. T-1].
 * x [T, H] bf16 (act_dtype must be MOE_BF16; w_dtype MOE_BF16 or MOE_E4M3);
 * perm_src [T*k] int32 as moe_permute wrote it, 16-byte aligned.  A perm_src
 * value outside [0, T) is reported through the device error word
 * (MOE_ERR_DEVICE_CHECK) and token 0 is read in its place.  gate may be NULL.
 * Everything else as moe_grouped_ffn. */
MOE_API moe_status moe_grouped_ffn_x(const moe_ffn_desc *d, const moe_expert_table *tbl,
                             const moe_ready_gate *gate, const void *x, const int32_t *perm_src,
                             const int32_t *offsets, void *h, void *y_perm, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/* Progress reports of a grouped-GEMM call, by which a later fetch is paced
 * (moe_prefetch_layer_paced): the explainer's prefetch caption has the fetch
 * run while the rank computes; reporting lets the copy spread over that
 * compute instead of running as one burst beside it.
 *   word   device, 4-byte aligned: written only by these reports and read by
 *          the copy stream.  Over one call it takes base + 1 .. base + steps
 *          as the tiles' MMAs are issued (the gate/up launch covers the first
 *          round(2 steps / 3) steps, the down launch the rest, each in equal
 *          parts of its tiles; a wrap-around maximum, never lowered), then
 *          base + steps + 1 once the call's launches have ended on `stream`,
 *          finished or stopped early.  A caller that runs calls back to back
 *          gives call n the base b0 + n (steps + 1).
 *   tiles  device, two 4-byte words of scratch (tile counters of the two
 *          launches), reset by the call.
 *   steps  >= 2. */
typedef struct moe_progress {
    uint32_t *word;
    uint32_t *tiles;
    uint32_t base;
    int32_t steps;
} moe_progress;

/* moe_grouped_ffn_x / moe_grouped_ffn_gated with progress reports.  Token
 * rows come from x through perm_src when both are given (as in
 * moe_grouped_ffn_x, x_perm ignored), else from x_perm; gate may be NULL,
 * progress must not be.  The final write of the progress word is issued
 * even when the call fails after its argument checks. */
MOE_API moe_status moe_grouped_ffn_paced(const moe_ffn_desc *d, const moe_expert_table *tbl,
                                 const moe_ready_gate *gate, const moe_progress *progress,
                                 const void *x_perm, const float *x_perm_scales, const void *x,
                                 const int32_t *perm_src, const int32_t *offsets, void *h,
                                 void *y_perm, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Weighted combine (unpermute):
 *   y[t] = sum_{j=0..k-1, ascending} topk_w[t,j] * y_perm[inv_pos[t,j]]
 *          + (with_shared ? y_perm[T*k + t] : 0)
 * in fp32, rounded once to y_dtype (MOE_F32 or MOE_BF16).
 * y_perm [rows, H] bf16; inv_pos [T, k] int32; topk_w [T, k] fp32; y [T, H].
 * Limits: H % 8 == 0, 1 <= k <= 32.
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_combine(int32_t T, int32_t k, int32_t H, const void *y_perm, const int32_t *inv_pos,
                       const float *topk_w, int32_t with_shared, void *y, moe_dtype y_dtype,
                       cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Remote-expert prefetch into the alternate buffer (explainer, prefetch
 * figure: while a rank computes layer l, the copy engine fetches layer l+1's
 * remote experts into the alternate buffer; fetch-path figure: the pull is a
 * cudaMemcpyAsync on the copy engine, not on the SMs).  Between two buffers
 * of one GPU the driver runs the copy as a kernel on the SMs (measured on
 * B200), so there the fetch competes with the compute for the SMs.
 *
 * Enqueues on copy_stream: a wait on wait_free (if not NULL: the event the
 * compute stream recorded after the last use of dst), the copy of `bytes`
 * from src to dst (cudaMemcpyAsync device-to-device, in pieces of
 * chunk_bytes if chunk_bytes > 0), and a record of ready_out (if not NULL),
 * which the consumer waits on before moe_grouped_ffn reads dst.  src may be
 * another GPU's memory when peer access is enabled.
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_prefetch_layer(const void *src, void *dst, size_t bytes, size_t chunk_bytes,
                              cudaStream_t copy_stream, cudaEvent_t wait_free,
                              cudaEvent_t ready_out);

/* ------------------------------------------------------------------------
 * Peer fetch inside a DWDP group (explainer, fetch-path caption: a rank
 * pulls the experts it lacks from a peer's memory with cudaMemcpyAsync over
 * NVLink, on the copy engine; contention caption: several destinations can
 * converge on one source, which time-division multiplexed slicing across
 * destinations removes).
 *
 * A group has G ranks (2 <= G <= 64).  Rank r owns one pool of its experts,
 * bytes_per_rank bytes (its slots x stride; a multiple of 256).  Its remote
 * buffer holds the other G-1 pools back to back in rank order, skipping r
 * (with n experts per rank, rank q owning experts [q*n, q*n+n) in slot
 * order, expert e of rank q != r sits in slot (q < r ? q : q-1)*n + e - q*n
 * of rank r's remote buffer).
 *
 * The slice plan: each source pool is cut into P = min(slices,
 * bytes_per_rank/256) pieces, each a multiple of 256 bytes except that the
 * last takes the rest.  Step j = 0 .. (G-1)*P - 1 of rank r copies piece
 * floor(j / (G-1)) of source s = (r + 1 + j mod (G-1)) mod G.  At any step j
 * the map r -> s is the same rotation on every rank, with no fixed point, so
 * G ranks pulling at the same pace read G different sources: no source ever
 * serves two destinations in the same step.
 * ---------------------------------------------------------------------- */
typedef struct moe_peer_copy {
    int32_t step;        /* position in the schedule (0-based) */
    int32_t src_rank;    /* rank whose pool is read */
    int64_t src_offset;  /* bytes from the start of that pool */
    int64_t dst_offset;  /* bytes from the start of the remote buffer */
    int64_t bytes;
} moe_peer_copy;

/* The plan of `rank` (host only, no CUDA call).  plan == NULL: only
 * *plan_len is set (a size query).  Otherwise plan must hold plan_capacity
 * >= *plan_len entries; they are written in step order. */
MOE_API moe_status moe_peer_fetch_plan(int32_t group_size, int32_t rank, int64_t bytes_per_rank,
                               int32_t slices, moe_peer_copy *plan, int32_t plan_capacity,
                               int32_t *plan_len);

/* Enqueues rank's plan on copy_stream: a wait on wait_free (if not NULL),
 * one cudaMemcpyAsync per step from src_pools[src_rank] + src_offset to
 * dst + dst_offset, and a record of ready_out (if not NULL).
 * src_pools: HOST array of G device pointers, the pools of the group's ranks
 * as this process addresses them (peer access or moe_pool_import);
 * src_pools[rank] is not read.  dst: (G-1) * bytes_per_rank bytes, 256-byte
 * aligned, on this rank's device.  Pools must be 256-byte aligned and must
 * not overlap dst.  No kernel reads a peer's memory: only the copy engine
 * does. */
MOE_API moe_status moe_prefetch_peers(int32_t group_size, int32_t rank, const void *const *src_pools,
                              int64_t bytes_per_rank, int32_t slices, void *dst,
                              cudaStream_t copy_stream, cudaEvent_t wait_free,
                              cudaEvent_t ready_out);

/* Lets the current device read peer_device's memory (one process driving
 * several GPUs).  Already enabled is not an error; MOE_ERR_UNSUPPORTED when
 * the pair has no peer path. */
MOE_API moe_status moe_enable_peer_access(int32_t peer_device);

/* One process per GPU: a rank exports its pool, every other rank imports it.
 * The handle names the CUDA allocation that contains `base` (cudaMalloc'd,
 * e.g. by a caching allocator) and base's offset inside it. */
typedef struct moe_pool_handle {
    char ipc[64];    /* cudaIpcMemHandle_t of the allocation */
    int64_t offset;  /* bytes from the allocation start to the pool */
} moe_pool_handle;

MOE_API moe_status moe_pool_export(const void *base, moe_pool_handle *out);
/* Maps an exported pool into this process: *base_out is the pool, and
 * *mapping_out the mapping to pass to moe_pool_close once no copy reads it. */
MOE_API moe_status moe_pool_import(const moe_pool_handle *h, void **base_out, void **mapping_out);
MOE_API moe_status moe_pool_close(void *mapping);

/* moe_prefetch_layer with per-chunk readiness flags for a gated grouped GEMM:
 * the copy is issued in chunks of chunk_bytes (> 0; the last takes the
 * rest), and after chunk c the copy stream writes flags[c] = epoch (a stream
 * memory operation, ordered after the chunk's copy, executed without SMs).
 * flags: device, ceil(bytes / chunk_bytes) words.  For a remote pool with
 * slot stride S, chunk_bytes = slots_per_flag * S makes flag c cover slots
 * [c*slots_per_flag, (c+1)*slots_per_flag).  MOE_ERR_UNSUPPORTED if the
 * driver does not provide cuStreamWriteValue32. */
MOE_API moe_status moe_prefetch_layer_flagged(const void *src, void *dst, size_t bytes,
                                      size_t chunk_bytes, cudaStream_t copy_stream,
                                      cudaEvent_t wait_free, uint32_t *flags, uint32_t epoch,
                                      cudaEvent_t ready_out);

/* moe_prefetch_layer_flagged paced by a grouped-GEMM call's progress (see
 * moe_progress): before chunk c of n a one-thread kernel on the copy stream
 * waits until
 *   (int32_t)(*pace->word - moe_pace_threshold(c, n, lead_chunks, pace->base,
 *                                              pace->steps)) >= 0
 * or 200 ms have passed, whichever comes first (a wait that runs out lets
 * the chunk go: pacing spreads the copy, the flags order it).  The first
 * lead_chunks chunks go at once; the others are spread evenly over the
 * call's reports, the last one released by report base + steps.  Enqueue
 * the pacing call BEFORE this fetch: streams may share a hardware queue, and
 * a wait queued ahead of its call would then hold the call back until it
 * runs out.  Only the word is read (pace->tiles unused).
 * MOE_ERR_UNSUPPORTED if the driver lacks cuStreamWriteValue32. */
MOE_API moe_status moe_prefetch_layer_paced(const void *src, void *dst, size_t bytes,
                                    size_t chunk_bytes, cudaStream_t copy_stream,
                                    cudaEvent_t wait_free, uint32_t *flags, uint32_t epoch,
                                    const moe_progress *pace, int32_t lead_chunks,
                                    cudaEvent_t ready_out);

/* The release threshold of moe_prefetch_layer_paced's chunk c of n:
 *   c <  lead_chunks:  base
 *   c >= lead_chunks:  base + floor((c - lead_chunks + 1) (steps + 1)
 *                                   / (n - lead_chunks + 1))
 * Host function (no device work). */
MOE_API uint32_t moe_pace_threshold(int64_t chunk, int64_t n_chunks, int32_t lead_chunks,
                                    uint32_t base, int32_t steps);

/* Selective prefetch (the predicted-routing prefetch of the offloading
 * diagram on the pages; this library's reading: fetch only the remote experts
 * a layer is predicted to touch, then the ones the prediction missed).
 * Copies slots[0 .. n) of a remote pool image of pool_slots slots, slot s
 * being the slot_bytes at offset s * slot_bytes of src and of dst (both
 * pool_slots * slot_bytes long, not overlapping); a run of consecutive
 * indices is one cudaMemcpyAsync, after which the copy stream writes
 * flags[s] = epoch for each slot s of the run (per-slot readiness: a
 * moe_ready_gate with slots_per_flag = 1, n_flags = pool_slots).
 * slots: host array, values in [0, pool_slots) (else MOE_ERR_INVALID_ARG
 * before anything is enqueued); flags: device, pool_slots words, 4-byte
 * aligned.  wait_free / ready_out as for moe_prefetch_layer.  n = 0 copies
 * nothing. */
MOE_API moe_status moe_prefetch_slots(const void *src, void *dst, size_t slot_bytes,
                              int32_t pool_slots, const int32_t *slots, int32_t n,
                              cudaStream_t copy_stream, cudaEvent_t wait_free, uint32_t *flags,
                              uint32_t epoch, cudaEvent_t ready_out);

/* The experts a routing selects: touched[e] = 1 if some entry of topk_idx
 * [A] equals e, else 0 (touched: device, E bytes, zeroed by the call on
 * `stream`).  Entries outside [0, E) are reported through the device error
 * word (MOE_ERR_DEVICE_CHECK) and skipped.  Used to predict a layer's
 * remote experts from a look-ahead routing and to find those a prediction
 * missed. */
MOE_API moe_status moe_experts_touched(const int32_t *topk_idx, int64_t A, int32_t E,
                               uint8_t *touched, cudaStream_t stream);

/* Host-side poll of an event with a deadline: MOE_OK once it has completed,
 * MOE_ERR_TIMEOUT after timeout_ms milliseconds, MOE_ERR_CUDA on error. */
MOE_API moe_status moe_wait_ready(cudaEvent_t ev, int32_t timeout_ms);

/* Synchronises the current device, then reads and clears the device error
 * word: MOE_OK, MOE_ERR_TIMEOUT (a kernel wait ran out) or
 * MOE_ERR_DEVICE_CHECK (an index outside its range was seen and skipped). */
MOE_API moe_status moe_check_device(void);

/* Test hook: the next `count` CUDA runtime calls the library makes report
 * failure (MOE_ERR_CUDA) without being issued.  0 disarms it. */
MOE_API void moe_debug_fail_next_cuda_calls(int32_t count);

/* Test hook: a gated grouped-FFN launch (moe_ready_gate) is refused with
 * MOE_ERR_CUDA when its kernel would hold more than `limit` registers per SM.
 * 0 (or less) restores the library's limit, 55,296. */
MOE_API void moe_debug_gated_regs_per_sm(int64_t limit);

#ifdef __cplusplus
}
#endif

#endif /* SPLIT_WEIGHT_B200_MOE_H */
