/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse MoE FFN layer forward.
 *
 * The layer (forward only, one GPU):
 *   RMS statistic  r_t = 1/sqrt(mean_i x_ti^2 + eps)
 *   router         l_te = r_t * sum_i x_ti gamma_i Wr_ie + b_e   (fp32)
 *   top-k gating   k largest l_te (ties -> lower e, slots largest first),
 *                  gate_tj = softmax_e(l_t)[idx_tj]  (optionally renormalised)
 *   dispatch       per-expert histogram, expert capacity, stable permutation
 *                  grouping assignments a = t*k+j by expert, token order inside
 *   experts        SwiGLU per expert with variable widths f_e:
 *                  h = silu(r_t*(xg_t W1_e)) * (r_t*(xg_t W3_e)),  y = h W2_e,
 *                  where xg_t = x_t * gamma
 *   combine        out_t = sum over kept slots of gate_tj * y_(t,j)
 *
 * Sources of each step:
 *  - CODA sparse-MoE thread (digg.com), RMSNorm paragraphs: the statistic r is
 *    commuted across the GEMM that follows the norm and applied in that GEMM's
 *    epilogue -- in the router right before the top-k, and in the first expert
 *    linear, to which r travels with the dispatched token.
 *  - Mixture of Experts glossary (inferensys.com): gating network, top-k and
 *    Switch (top-1) routing, expert capacity
 *    C = (T*k)/E * capacity_factor with excess tokens dropped, fused MoE
 *    kernels combining routing, permutation and expert matmuls.
 *  - nanoMOE variable-size-experts notes (hbfreed.com): expert widths as
 *    multiples of 128, concatenated weights W1 [d, F], W2 [F, d] with
 *    cumulative column offsets ("Weight Allocation", "Offset Calculation").
 *  - OmniMoE summary (gist.science), section 2.2 "Expert-Centric Scheduling":
 *    routing decisions grouped by expert, sorted by token inside a group,
 *    executed as a grouped GEMM.
 *
 * Conventions (all entry points):
 *  - Every tensor pointer is a DEVICE pointer owned by the caller; the library
 *    allocates nothing and keeps no state between calls.  Row-major layouts.
 *    bf16 tensors are passed as moe_bf16_t (raw bf16 bit patterns).
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t, NULL = the
 *    legacy default stream); the return value only reports argument checks and
 *    launch errors.  Errors detected on the device (an expert id out of range,
 *    a bounded wait that expired) are OR-ed into an error word in the
 *    workspace; read it with moe_get_device_error().  No kernel traps.
 *  - Arguments are validated before anything is launched; on error nothing is
 *    enqueued.  bf16 matrices must be 16-byte aligned, fp32/int32 arrays
 *    4-byte aligned, the workspace 256-byte aligned.
 *  - Limits: 1 <= k <= E <= 64, d_model a positive multiple of 128, every
 *    expert width a positive multiple of 128, T >= 0 (T = 0 is a no-op),
 *    T*k < 2^31.  With T = 0 every call validates cfg and returns MOE_OK;
 *    only counts/offsets outputs are written (zeros), other pointers may be NULL.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef uint16_t moe_bf16_t; /* raw bfloat16 bits */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* bad shape, null pointer, k > E, ...          */
  MOE_ERR_ALIGNMENT = 2,   /* a pointer is not aligned as required         */
  MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required   */
  MOE_ERR_UNSUPPORTED = 4, /* valid but outside this build's limits        */
  MOE_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed            */
  MOE_ERR_DEVICE = 6,      /* the device error word is non-zero            */
  MOE_ERR_NO_DEVICE = 7    /* no usable sm_100 device                      */
} moe_status_t;

/* Bits of the device error word (moe_get_device_error). */
#define MOE_DEVERR_EXPERT_ID 0x1u  /* an expert id outside [0, E) reached dispatch */
#define MOE_DEVERR_TIMEOUT 0x2u    /* a bounded pipeline wait gave up             */
#define MOE_DEVERR_TILE_TABLE 0x4u /* kept rows exceed the buffers they index     */

typedef struct {
  int32_t T;        /* tokens                                                */
  int32_t d_model;  /* hidden size d                                         */
  int32_t E;        /* experts                                               */
  int32_t k;        /* experts per token                                     */
  /* HOST array [E+1]: cumulative expert widths, ffn_offsets[0] = 0 and
   * ffn_offsets[e+1] - ffn_offsets[e] = f_e (a multiple of 128).  Expert e
   * owns columns [ffn_offsets[e], ffn_offsets[e+1]) of W1/W3 and the same rows
   * of W2 (nanoMOE notes, "Offset Calculation").  Read during the call only. */
  const int32_t* ffn_offsets;
  float capacity_factor; /* <= 0: dropless; else C = floor((T*k)/E * cf)   */
  float eps;             /* RMS epsilon, e.g. 1e-5                            */
  int32_t renormalize;   /* 0: gate = softmax over all E; 1: renormalised
                            over the k chosen experts                       */
} moe_config_t;

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(moe_status_t status);

/* Expert capacity C of `cfg` ((T*k)/E * capacity_factor rounded down, MoE
 * glossary "Expert Capacity"), or -1 when dropless or cfg is invalid. */
MOE_API int64_t moe_capacity(const moe_config_t* cfg);

/* Maximum number of kept assignments: T*k when dropless, else min(T*k, E*C). */
MOE_API int64_t moe_max_kept(const moe_config_t* cfg);

/* Expert column offsets for moe_config_t.ffn_offsets from a variable-size
 * expert list of n_groups (count, size) pairs (nanoMOE notes, "Expert Size
 * Computation" and "Offset Calculation"): each size is rounded up to a
 * multiple of 128 and repeated count times, in list order, and the offsets
 * are the running sums of those widths, starting at 0.  Host only, no
 * device work.  Writes E + 1 entries to offsets (E = the sum of the counts,
 * which must be at most max_experts) and returns E; returns -1 and writes
 * nothing on a null pointer, n_groups < 0, a count < 0, a size < 1, E >
 * max_experts or a total width above 2^31 - 1. */
MOE_API int32_t moe_expert_offsets(const int32_t* counts, const int32_t* sizes, int32_t n_groups,
                                   int32_t* offsets, int32_t max_experts);

/* Bytes of workspace every entry point below needs for `cfg` (0 if cfg is
 * invalid).  One workspace of this size serves all calls; it holds the device
 * error word, the dispatch scratch and, for moe_layer_fwd, every
 * intermediate (routing, permutation, permuted activations -- or, for
 * moe_layer_fwd_gather, x * gamma in token order in the same buffer -- the
 * SwiGLU activations H and the per-assignment expert outputs). */
MOE_API size_t moe_workspace_size(const moe_config_t* cfg);

/* Zero the workspace header (the device error word and the wait limit, which
 * then means the default).  Call once after allocating a workspace, before its
 * first use.  Asynchronous on `stream`. */
MOE_API moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, copy the device error word to *code and clear it.
 * Returns MOE_ERR_DEVICE if the word was non-zero, MOE_OK otherwise. */
MOE_API moe_status_t moe_get_device_error(void* ws, size_t ws_bytes, void* stream, uint32_t* code);

/* Limit of the bounded pipeline waits of the kernels that later run on this
 * workspace (any workspace of this library: forward, training, MXFP8 or
 * host-buffer), written into its header in stream order.  limit_ns = 0
 * restores the default of 4 s.  Every wait inside the router, the dispatch's
 * scan and the expert GEMMs that does not complete within the limit sets
 * MOE_DEVERR_TIMEOUT, stops its kernel's CTAs (both CTAs of a tensor-core
 * pair), lets every copy and matrix operation already in flight finish, and
 * returns; the layer's outputs
 * are then undefined, and later calls with the default limit are unaffected.
 * Normal use never needs this: it exists to exercise that path (a limit of a
 * few ns makes nearly every wait run out).  moe_workspace_init resets it. */
MOE_API moe_status_t moe_set_wait_limit(void* ws, size_t ws_bytes, uint32_t limit_ns, void* stream);

/* Route: RMS statistic, router GEMM with the statistic applied after the GEMM
 * and before the top-k (CODA thread), softmax and top-k gating (MoE glossary,
 * "Top-k Gating" / "Switch Routing").
 *   x        [T, d]   bf16   activations
 *   gamma    [d]      bf16   RMSNorm weight
 *   Wr       [d, E]   bf16   router weight
 *   bias     [E]      fp32   router logit bias, or NULL for none
 *   expert_idx [T, k] int32  out: chosen experts, largest logit first
 *   gate     [T, k]   fp32   out: softmax(l_t) at the chosen experts
 *   r        [T]      fp32   out: RMS statistic
 *   logits   [T, E]   fp32   out (optional, NULL to skip): router logits
 *   prob_mean [E]     fp32   out (optional, NULL to skip): mean softmax
 *                            probability of each expert over the T tokens,
 *                            reduced in the router's epilogue in a fixed order
 *                            (deterministic); input of moe_router_stats
 * Logits accumulate exact bf16*bf16 products; each is rounded once to fp32.
 * The workspace (at least moe_workspace_size(cfg) bytes) holds gamma*Wr in
 * tensor-core fragment order, the prob_mean partials and the error word. */
MOE_API moe_status_t moe_route(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                       const moe_bf16_t* Wr, const float* bias, int32_t* expert_idx, float* gate,
                       float* r, float* logits, float* prob_mean, void* ws, size_t ws_bytes,
                       void* stream);

/* Router load-balance metrics (MoE glossary, "Load Balancing": an auxiliary
 * loss on the spread of the routing probability across experts), computed on
 * the device from moe_route's prob_mean and moe_dispatch's counts / offsets:
 *   stats[0] = E * sum_e f_e * P_e   (Switch-style term, f_e = counts_e/(T*k))
 *   stats[1] = CV^2 of P_e over experts (population variance / mean^2)
 *   stats[2] = CV^2 of counts_e over experts
 *   stats[3] = fraction of the T*k assignments dropped by the capacity limit
 * stats [4] fp32 device output; asynchronous on `stream`. */
MOE_API moe_status_t moe_router_stats(const moe_config_t* cfg, const float* prob_mean,
                                      const int32_t* counts, const int32_t* expert_offsets,
                                      float* stats, void* stream);

/* Dispatch: histogram, capacity, expert-centric permutation (OmniMoE summary,
 * "Expert-Centric Scheduling"; MoE glossary, "Expert Capacity"), and the
 * permuted, gamma-scaled activations the expert GEMMs read.
 *   expert_idx [T, k]   int32  in
 *   x          [T, d]   bf16   in (activations, as given to moe_route)
 *   gamma      [d]      bf16   in
 *   counts     [E]      int32  out: assignments per expert (before capacity)
 *   expert_offsets [E+1] int32 out: exclusive running sum of kept counts
 *   perm       [T*k]    int32  out: perm[p], p < n_kept, is the assignment
 *                              a = t*k+j kept at position p (grouped by
 *                              expert, token order inside a group)
 *   inv_perm   [T*k]    int32  out: position of assignment a, -1 if dropped
 *   x_perm     [T*k, d] bf16   out: x_perm[p] = bf16(x_t * gamma), t = perm[p]/k
 * The number of kept assignments is expert_offsets[E]; rows of perm/x_perm at
 * and beyond it are left untouched. */
MOE_API moe_status_t moe_dispatch(const moe_config_t* cfg, const int32_t* expert_idx, const moe_bf16_t* x,
                          const moe_bf16_t* gamma, int32_t* counts, int32_t* expert_offsets,
                          int32_t* perm, int32_t* inv_perm, moe_bf16_t* x_perm, void* ws,
                          size_t ws_bytes, void* stream);

/* moe_dispatch for callers that cannot allocate device memory.
 * (No counterpart in the pages: this is a deployment variant.)
 * Some callers own no allocator: an inference engine that hands a plugin only
 * its input and output buffers, a runtime that forbids cudaMalloc after start-up
 * (it synchronises the device and can fail under memory pressure), or code that
 * runs inside another library's memory pool.  Such callers cannot provide the
 * workspace moe_dispatch needs for the scratch of its scan (a status word and
 * two count vectors per tile of 1024 assignments), so this variant keeps that
 * scratch in a fixed array inside the library (a file-scope __device__ array
 * of 516 KiB + 256 B, held by every GPU that loads the library until the
 * process exits).  It allocates nothing and takes no workspace; arguments and
 * results are those of moe_dispatch.
 *  - Limit: T*k <= 1048576 assignments (the array holds the scan of 1024
 *    tiles of 1024 assignments for up to 64 experts); larger problems return
 *    MOE_ERR_UNSUPPORTED before anything is enqueued.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture.  The address is kept for the life of the process: after
 *    cudaDeviceReset() on a device the library's module is loaded anew there
 *    and the kept address is stale, so do not use this entry point on a
 *    device after resetting it.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents; the call clears what must start at zero.  Calls that overlap on
 *    the GPU (e.g. on two streams at once) race on the array: serialise them.
 *  - The device error word also lives in the array and is not readable through
 *    moe_get_device_error: an expert id outside [0, E) is dropped
 *    (inv_perm = -1) and left out of counts, so sum(counts) < T*k reveals it.
 *    The scan's waits use the default limit of 4 s. */
MOE_API moe_status_t moe_dispatch_noalloc(const moe_config_t* cfg, const int32_t* expert_idx,
                                          const moe_bf16_t* x, const moe_bf16_t* gamma,
                                          int32_t* counts, int32_t* expert_offsets, int32_t* perm,
                                          int32_t* inv_perm, moe_bf16_t* x_perm, void* stream);

/* Experts: the two grouped GEMMs over the expert-centric order.
 *   x_perm   [T*k, d] bf16   in (moe_dispatch)
 *   r        [T]      fp32   in (moe_route): applied in GEMM 1's epilogue
 *   gate     [T, k]   fp32   in (moe_route): applied in GEMM 2's epilogue
 *   perm, expert_offsets     in (moe_dispatch)
 *   W1, W3   [d, F]   bf16   expert e = columns ffn_offsets[e] .. [e+1]
 *   W2       [F, d]   bf16   expert e = rows    ffn_offsets[e] .. [e+1]
 *   y        [T*k, d] bf16   out: y[p] = bf16(gate_a * FFN_e(x_t)), a = perm[p],
 *                            for p < expert_offsets[E] (expert-centric order)
 * Uses the workspace for H (the SwiGLU activations). */
MOE_API moe_status_t moe_experts_fwd(const moe_config_t* cfg, const moe_bf16_t* x_perm, const float* r,
                             const float* gate, const int32_t* perm,
                             const int32_t* expert_offsets, const moe_bf16_t* W1,
                             const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* y, void* ws,
                             size_t ws_bytes, void* stream);

/* The two halves of moe_experts_fwd, for callers that schedule them apart.
 * moe_experts_up runs GEMM 1 (x_perm x (W1 | W3), r and SwiGLU in the
 * epilogue) and leaves H in the workspace; moe_experts_down runs GEMM 2
 * (H x W2, gate in the epilogue) on that H and writes y.  Same arguments and
 * layouts as moe_experts_fwd; the workspace must be the same between the two
 * calls and must not be used by another call in between. */
MOE_API moe_status_t moe_experts_up(const moe_config_t* cfg, const moe_bf16_t* x_perm, const float* r,
                                    const int32_t* perm, const int32_t* expert_offsets,
                                    const moe_bf16_t* W1, const moe_bf16_t* W3, void* ws,
                                    size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_experts_down(const moe_config_t* cfg, const float* gate, const int32_t* perm,
                                      const int32_t* expert_offsets, const moe_bf16_t* W2,
                                      moe_bf16_t* y, void* ws, size_t ws_bytes, void* stream);

/* Combine: out_t = bf16(sum_j y[inv_perm[t*k+j]]) over kept slots, summed in
 * fp32 in slot order j = 0..k-1; a token with every slot dropped gets 0.
 *   y        [T*k, d] bf16   in (moe_experts_fwd)
 *   inv_perm [T*k]    int32  in (moe_dispatch)
 *   out      [T, d]   bf16   out */
MOE_API moe_status_t moe_combine(const moe_config_t* cfg, const moe_bf16_t* y, const int32_t* inv_perm,
                         moe_bf16_t* out, void* stream);

/* The whole layer: route -> dispatch -> experts -> combine, on one stream,
 * with no host synchronisation (the kept counts never leave the device).
 * With k = 1 there is no combine: the second GEMM writes each kept row
 * straight to its token's row of out (a sum of one term, MoE glossary "Top-k
 * Gating"), after a memset of out has cleared the rows of tokens a capacity
 * limit dropped ("Expert Capacity"); the result is bit-identical to the
 * combine.  The layer's kernels after the first are launched with
 * programmatic stream serialization (each waits for the one before it before
 * touching memory), so they order like ordinary launches on `stream`.
 *   out [T, d] bf16 out.  expert_idx/gate/r/counts/prob_mean: optional copies
 *   of the routing results (NULL to skip), shapes as in moe_route /
 *   moe_dispatch; stats [4]: optional router metrics (moe_router_stats). */
MOE_API moe_status_t moe_layer_fwd(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                           const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                           const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out,
                           int32_t* expert_idx, float* gate, float* r, int32_t* counts,
                           float* prob_mean, float* stats, void* ws, size_t ws_bytes, void* stream);

/* moe_layer_fwd with the row gather fused into GEMM 1's A-operand load (CODA
 * thread: r travels with the dispatched token into the first expert linear;
 * OmniMoE, section 2.2: tasks grouped by expert into a grouped GEMM).  No
 * permuted copy of x is made: the router also writes xg = bf16(x * gamma) in
 * token order into the workspace, and GEMM 1's producer gathers each A tile
 * from it, row p = token perm[p] / k, with four-row TMA gathers
 * (tile::gather4) -- rows bit-identical to moe_dispatch's x_perm, so out is
 * bit-identical to moe_layer_fwd.  It saves the permuted copy's write and
 * read (2 * T*k * d * 2 bytes per call) but on B200 runs slower than
 * moe_layer_fwd: each four-row gather costs the SM's copy engine about as
 * much as a whole 128-row tile load, which leaves GEMM 1 load-bound.  Same
 * arguments, workspace and errors as moe_layer_fwd. */
MOE_API moe_status_t moe_layer_fwd_gather(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                                          const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                                          const moe_bf16_t* W3, const moe_bf16_t* W2, moe_bf16_t* out,
                                          int32_t* expert_idx, float* gate, float* r, int32_t* counts,
                                          float* prob_mean, float* stats, void* ws, size_t ws_bytes,
                                          void* stream);

/* ---- the layer on HOST buffers: copies in and out pipelined with the compute
 *
 * moe_layer_fwd with x and out in host memory (pinned memory, e.g. from
 * cudaHostAlloc, lets the copies overlap; pageable memory works but does not
 * overlap).  Without a capacity limit a token's output depends only on that
 * token, so the batch is cut into n_chunks chunks (sizes in the ratio
 * 1 : 4 : ... : 4 : 1, since only the first copy in and the last copy out are
 * exposed) and the copy of chunk i+1 in and of chunk i-1 out run on the library's own
 * copy streams while the layer runs on chunk i: out is bit-identical to
 * moe_layer_fwd on the whole batch.  With a capacity limit (capacity_factor >
 * 0) the drops depend on every token's rank, so the batch is one chunk.
 * n_chunks <= 0 picks the default (3); at most 64, at most T.  Asynchronous on `stream`: when the
 * stream reaches this point, out_host holds the result; x_host and out_host
 * must stay valid until then.  The workspace (moe_host_workspace_size for the
 * same n_chunks) holds one chunk's layer workspace, whose first 256 bytes
 * carry the device error word (moe_get_device_error works on it), and the
 * double-buffered device staging of x and out.  Calls on one device are
 * serialised while they enqueue (the copy streams are per device). */
MOE_API size_t moe_host_workspace_size(const moe_config_t* cfg, int32_t n_chunks);
/* Chunks moe_layer_fwd_host will use for `cfg` and n_chunks (-1 if invalid). */
MOE_API int32_t moe_host_chunks(const moe_config_t* cfg, int32_t n_chunks);
MOE_API moe_status_t moe_layer_fwd_host(const moe_config_t* cfg, const moe_bf16_t* x_host,
                                        const moe_bf16_t* gamma, const moe_bf16_t* Wr, const float* bias,
                                        const moe_bf16_t* W1, const moe_bf16_t* W3, const moe_bf16_t* W2,
                                        moe_bf16_t* out_host, int32_t n_chunks, void* ws, size_t ws_bytes,
                                        void* stream);

/* ---- MXFP8 expert GEMMs
 *
 * CODA sparse-MoE thread (digg.com): with low-precision expert GEMMs, the
 * conversions of their inputs go into the epilogues of the producing kernels.
 * Format: OCP Microscaling MXFP8 -- blocks of 32 consecutive values along a
 * GEMM's reduction share an E8M0 scale 2^e with e = floor(log2 max|v|) - 8,
 * and each value is v * 2^-e as FP8 E4M3 (round to nearest even, saturating
 * at 448).  The layer is moe_layer_fwd's (router, dispatch, combine
 * unchanged) with: x*gamma quantised per token along d by the dispatch, W1/W3
 * along d and W2 along F by moe_quantize_weights_mx (once per set of
 * weights), and the SwiGLU output H quantised along the expert width in the
 * first expert GEMM's epilogue; both expert GEMMs run block-scaled on the
 * tensor cores with fp32 accumulation; y and out stay bf16.  Each expert's
 * rows are padded to a multiple of 128 in the workspace. */

/* Bytes of the quantised weights for cfg (0 if invalid): K-major E4M3 copies
 * of W1, W3 ([F, d]) and W2 ([d, F]), their scale blocks (the layout
 * moe_mx_part describes), and the same scales once more in the form the MX
 * GEMM loads them: each 512-byte block stored four times, two blocks per
 * 4 KB region (about 4x the scale bytes; internal, not a part). */
MOE_API size_t moe_mx_weights_size(const moe_config_t* cfg);
/* Quantise W1, W3 [d, F] and W2 [F, d] (bf16, device) into wq (device,
 * 256-byte aligned, moe_mx_weights_size bytes, caller-owned). */
MOE_API moe_status_t moe_quantize_weights_mx(const moe_config_t* cfg, const moe_bf16_t* W1,
                                             const moe_bf16_t* W3, const moe_bf16_t* W2, void* wq,
                                             size_t wq_bytes, void* stream);
/* Bytes of workspace for moe_layer_fwd_mx (0 if invalid). */
MOE_API size_t moe_mx_workspace_size(const moe_config_t* cfg);
/* Rows of its permuted buffers: max kept + 127 E, rounded up to 128. */
MOE_API int64_t moe_mx_rows(const moe_config_t* cfg);
/* The layer with MXFP8 expert GEMMs: arguments as moe_layer_fwd, with the
 * quantised weights wq in place of W1/W3/W2.  out [T, d] bf16. */
MOE_API moe_status_t moe_layer_fwd_mx(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                                      const moe_bf16_t* Wr, const float* bias, const void* wq,
                                      size_t wq_bytes, moe_bf16_t* out, void* ws, size_t ws_bytes,
                                      void* stream);
/* Device addresses of the MX buffers, for inspection: parts of wq (ids 0-5)
 * or of the workspace of the last moe_layer_fwd_mx (6-14).  Scale blocks:
 * 512 bytes per 128 rows x 128 k, block (r/128, k/128) at index
 * (r/128) * (K/128) + k/128, scale of (r, k) at byte
 * 16 (r % 32) + 4 ((r % 128) / 32) + (k % 128) / 32 of its block. */
typedef enum {
  MOE_MX_W1 = 0,      /* [F, d] E4M3                                          */
  MOE_MX_W3 = 1,      /* [F, d] E4M3                                          */
  MOE_MX_W2 = 2,      /* [d, F] E4M3                                          */
  MOE_MX_SF1 = 3,     /* (F/128) x (d/128) blocks of w1                       */
  MOE_MX_SF3 = 4,     /* (F/128) x (d/128) blocks of w3                       */
  MOE_MX_SF2 = 5,     /* (d/128) x (F/128) blocks of w2                       */
  MOE_MX_X8 = 6,      /* [rows, d] E4M3                                       */
  MOE_MX_XSF = 7,     /* (rows/128) x (d/128) blocks                          */
  MOE_MX_H8 = 8,      /* [rows, f_max] E4M3                                   */
  MOE_MX_HSF = 9,     /* (rows/128) x (f_max/128) blocks                      */
  MOE_MX_PERM = 10,   /* [rows] int32, -1 at padding                          */
  MOE_MX_OFFSETS = 11, /* [E+1] int32 (128-row segments)                      */
  MOE_MX_IDX = 12,    /* [T, k] int32                                         */
  MOE_MX_GATE = 13,   /* [T, k] fp32                                          */
  MOE_MX_R = 14       /* [T] fp32                                             */
} moe_mx_part_t;
MOE_API moe_status_t moe_mx_part(const moe_config_t* cfg, void* wq, void* ws, size_t ws_bytes, int32_t which,
                                 void** ptr);

/* ---- training: forward that saves what the backward reads, and the backward
 *
 * CODA sparse-MoE thread (digg.com): the RMSNorm backward is fused into the
 * backward of the linears that read the normalised token (the router and the
 * first expert linear), which needs each token's statistic r; r is therefore
 * saved by the forward and read by the backward's epilogues.  The gradient is
 * the derivative of the forward above (routing ids and capacity drops carry
 * none; the router receives gradient through the gates).
 *
 * The training workspace (size from moe_train_workspace_size) holds the device
 * error word (so moe_get_device_error works on it), r, the routing, the fp32
 * logits, the expert-centric permutation with every expert's row segment
 * padded to a multiple of 64 rows (padding rows are zero), x_perm, the
 * pre-activations U = r*(x*gamma)W1_e and V = r*(x*gamma)W3_e, H, and the
 * ungated expert outputs, plus the backward's scratch.  One workspace serves
 * one forward/backward pair: moe_layer_bwd reads what the last
 * moe_layer_fwd_train on the same workspace saved, with the same cfg and
 * inputs.  Limits beyond the forward's: none. */

/* Bytes of training workspace for `cfg` (0 if cfg is invalid). */
MOE_API size_t moe_train_workspace_size(const moe_config_t* cfg);

/* The layer forward of moe_layer_fwd (same arguments, same out to the bit),
 * saving the backward's inputs in the training workspace `tws`. */
MOE_API moe_status_t moe_layer_fwd_train(const moe_config_t* cfg, const moe_bf16_t* x,
                                         const moe_bf16_t* gamma, const moe_bf16_t* Wr,
                                         const float* bias, const moe_bf16_t* W1, const moe_bf16_t* W3,
                                         const moe_bf16_t* W2, moe_bf16_t* out, void* tws,
                                         size_t tws_bytes, void* stream);

/* Gradients of L = <dout, out> for the forward last run on `tws`:
 *   dout   [T, d] bf16 in
 *   dx     [T, d] fp32 out        dgamma [d]    fp32 out
 *   dWr    [d, E] fp32 out        dbias  [E]    fp32 out (written even when
 *                                                the forward had no bias)
 *   dW1, dW3 [d, F] fp32 out      dW2    [F, d] fp32 out
 * Every output is overwritten (experts that received no rows get zero weight
 * gradients).  x, gamma, Wr, bias, W1, W3, W2 are the forward's inputs.
 * Pointers: 16-byte aligned except bias/dbias/dgamma (4).  Asynchronous on
 * `stream`; errors as for moe_layer_fwd. */
MOE_API moe_status_t moe_layer_bwd(const moe_config_t* cfg, const moe_bf16_t* x, const moe_bf16_t* gamma,
                                   const moe_bf16_t* Wr, const float* bias, const moe_bf16_t* W1,
                                   const moe_bf16_t* W3, const moe_bf16_t* W2, const moe_bf16_t* dout,
                                   float* dx, float* dgamma, float* dWr, float* dbias, float* dW1,
                                   float* dW3, float* dW2, void* tws, size_t tws_bytes, void* stream);

/* Saved tensors of the training workspace, for inspection (device pointers
 * into `tws`, valid while it lives; NULL and MOE_ERR_INVALID_ARG for an
 * unknown id).  Rows of the permuted tensors: moe_train_rows(cfg). */
typedef enum {
  MOE_SAVED_R = 0,        /* [T] fp32                                        */
  MOE_SAVED_IDX = 1,      /* [T, k] int32                                    */
  MOE_SAVED_GATE = 2,     /* [T, k] fp32                                     */
  MOE_SAVED_LOGITS = 3,   /* [T, E] fp32                                     */
  MOE_SAVED_OFFSETS = 4,  /* [E+1] int32, padded row segments                */
  MOE_SAVED_PERM = 5,     /* [rows] int32, -1 at padding                     */
  MOE_SAVED_INV_PERM = 6, /* [T*k] int32, -1 when dropped                    */
  MOE_SAVED_U = 7,        /* [rows, f_max] bf16                              */
  MOE_SAVED_V = 8,        /* [rows, f_max] bf16                              */
  MOE_SAVED_H = 9,        /* [rows, f_max] bf16                              */
  MOE_SAVED_Y = 10,       /* [rows, d] bf16, ungated expert outputs          */
  MOE_SAVED_DGATE = 11,   /* [T*k] fp32 (after moe_layer_bwd; kept slots)    */
  MOE_SAVED_DR = 12,      /* [T] fp32 dL/dr (after moe_layer_bwd)            */
  MOE_SAVED_COUNTS = 13   /* [E] int32 routed assignments per expert         */
} moe_saved_t;
MOE_API moe_status_t moe_train_saved(const moe_config_t* cfg, void* tws, size_t tws_bytes,
                                     int32_t which, void** ptr);
/* Rows of the padded permuted buffers: max kept + E * 63. */
MOE_API int64_t moe_train_rows(const moe_config_t* cfg);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
