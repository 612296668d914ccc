/*
 * moe.h -- C ABI of the B200 (sm_100a) top-k routed SwiGLU Mixture-of-Experts layer.
 *
 * The operation (forward pass of one MoE layer, T tokens, hidden H, E experts, top-k,
 * expert intermediate I):
 *
 *   l[t,e]   = sum_h x[t,h] W_router[h,e] + b_router[e]                    router logits
 *   S_t      = the k experts with the largest l[t,.], largest first, equal logits by
 *              lower expert index                                          top-k
 *   w[t,j]   = exp(l[t,S_tj] - l[t,S_t0]) / sum_j' exp(l[t,S_tj'] - l[t,S_t0])
 *                                                                          softmax over the
 *                                                                          selected logits
 *   count[e] = #{(t,j) : S_tj = e};  offsets = exclusive prefix sum of count
 *   perm     : rows of expert e are offsets[e] .. offsets[e+1]-1, holding the tokens routed
 *              to e in ascending token order; inv_perm[t,j] = row of (t, S_tj)
 *   g | u    = x[t] W_gate_up[e]   (gate = columns [0,I), up = columns [I,2I))
 *   h        = silu(g) * u,  silu(z) = z / (1 + exp(-z))                    SwiGLU
 *   out[t]   = sum_j w[t,j] * (h_(t,S_tj) W_down[S_tj])                     combine
 *
 * Source: the layer is the mixture of SwiGLU experts with top-4 routing over 32 experts and
 * hidden size 2880 in the Persona Kappa forum post ("Architecture Summary" table, "Notable
 * Details") and the kappa-20b-131k model card ("Model Details" table); 128 experts in the
 * hearth-lean-loomed-v1 card (intro and "Why 12-16 streams can be slow on Vulkan", which also
 * describes the few-tokens-per-expert decode regime).  bf16 operands with fp32 accumulation
 * follow the forum post's "Techniques That Made It Fit" list.  The pages print no formula,
 * no tie rule and no interface: the formulas above are the plain reading, ties go to the
 * lower expert index, and the calls below are this library's own.
 *
 * Conventions for every call
 * --------------------------
 * - All tensors are row-major and live in device memory of the current CUDA device, owned
 *   by the caller.  bf16 = IEEE bfloat16.  Every pointer must be 16-byte aligned.
 *     x          [T, H]      bf16
 *     W_router   [H, E]      bf16
 *     b_router   [E]         fp32
 *     W_gate_up  [E, H, 2I]  bf16   (per expert: gate columns [0,I), up columns [I,2I))
 *     W_down     [E, I, H]   bf16
 *     out        [T, H]      fp32   (fully overwritten)
 * - Work is only enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).  A call
 *   whose experts take more than one kernel family may run the row tiles on a second stream
 *   of the handle, forked from and joined back into `stream` with events, so the call stays
 *   ordered on `stream`.  No call below synchronises, allocates device memory or reads device
 *   memory on the host, except moe_create / moe_destroy (allocate / free the handle's 4-byte
 *   device status word, its second stream and two events), moe_sync_status, moe_tune and
 *   moe_last_dispatch (which synchronise) and moe_profile_* (events).
 * - Errors are returned, never thrown or aborted on.  Argument errors are found on the host
 *   before anything is enqueued and leave every buffer untouched.  A failed launch returns
 *   MOE_ERR_CUDA.  Faults detected on the device (a bounded wait that ran out) set the
 *   handle's status word, which moe_sync_status reports.
 * - One handle may be used from one stream at a time; separate handles are independent.
 * - H and I must be multiples of 64 (2880 = 45 * 64 is not a multiple of 128), 1 <= k <= E
 *   <= 256, H, I <= 16384, 0 <= T <= 2^20 and T * k < 2^31.  NaN or infinite inputs give
 *   undefined results.
 */
#ifndef MOE_H_
#define MOE_H_

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

struct CUstream_st;
typedef struct CUstream_st* moe_stream_t;  /* the same object as cudaStream_t */

typedef struct moe_ctx* moe_t;             /* opaque handle: shapes, settings, status word */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,          /* bad argument: null / misaligned pointer, size out of range */
  MOE_ERR_UNSUPPORTED = 2,  /* valid request this build does not support on this device */
  MOE_ERR_WORKSPACE = 3,    /* workspace pointer null or smaller than moe_workspace_bytes */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (reported by sync_status) */
  MOE_ERR_DEVICE = 6        /* no usable sm_100 device */
} moe_status;

/* Which kernels multiply an expert's rows.  Three kernel families:
 *   weight streaming  tensor-core mma.sync with the weights split over K across all SMs
 *                     (stream-K): balances best when only a few experts are touched
 *   expert tiles      tcgen05 MMAs with an expert's weight columns as the M operand and its rows
 *                     as N, each weight block read once for up to 128 rows (256 rows per
 *                     tile once a call's mean load reaches 128 rows per expert)
 *   row tiles         2-SM tcgen05 grouped GEMM, 256 rows x 256 columns per CTA pair (prefill,
 *                     long sequences)
 * MOE_PATH_AUTO chooses on the device, from the call's histogram (no host sync): in calls of at
 * most crossover_T tokens the experts with at most stream_rows rows stream.  The other experts
 * take one tcgen05 family for the whole call by default: expert tiles if their mean row count
 * is below tile_rows, row tiles otherwise (the two persistent kernels cannot share an SM, so a
 * call that runs both pays for two partly filled passes over the GPU).  With per-expert
 * dispatch on (moe_set_dispatch) each of them takes expert tiles up to tile_rows rows and row
 * tiles above; when a call's counts put a few experts just across that boundary (an almost
 * uniform routing), they join the larger side instead of running as a second, half-filled
 * launch: the upper side joins the lower one if it holds no more experts and none has more
 * than 2 * tile_rows rows, else the lower side joins the upper one if it holds fewer experts
 * and none has tile_rows / 2 rows or less.  This is the mat-vec / mat-mat choice of the
 * hearth-lean-loomed-v1 card ("Why 12-16 streams can be slow on Vulkan"), made per call (and
 * per expert on request).  The other values force one family for every expert. */
typedef enum {
  MOE_PATH_AUTO = 0,    /* choice among the three families below from the call's counts */
  MOE_PATH_STREAM = 1,  /* every expert through the weight-streaming kernels */
  MOE_PATH_GEMM = 2,    /* every expert through the 2-SM row-tile grouped GEMM */
  MOE_PATH_TILE = 3     /* every expert through the expert-tile kernels */
} moe_path;

/* Create a handle for a layer of shape (E, H, I, k) on the current device.  Validates the
 * shape (see conventions; MOE_ERR_ARG otherwise), checks for an sm_100 device
 * (MOE_ERR_DEVICE), allocates the 4-byte device status word, creates a second stream and two
 * events (for calls whose kernel families run side by side) and looks up the device address of
 * the library's routing scratch array (moe_route_static).  *out receives the handle.
 * Two environment variables, read here, select kernel variants for measurement: MOE_ROW_TILE=512
 * (row tiles of 256 x 512 instead of 256 x 256) and MOE_TILE_ROWS=128 or 256 (rows per expert
 * tile for every call instead of by the call's mean load). */
MOE_API moe_status moe_create(int E, int H, int I, int k, moe_t* out);

/* Free the handle and its status word.  NULL is accepted.  Work still queued on a stream
 * that uses the handle must have completed. */
MOE_API moe_status moe_destroy(moe_t ctx);

/* Bytes of device workspace that moe_forward needs for T tokens with the handle's current
 * path setting (moe_set_path / moe_tune change it, so query after them).  moe_route needs
 * moe_route_workspace_bytes.  Returns 0 for a NULL handle or T < 0. */
MOE_API size_t moe_workspace_bytes(moe_t ctx, int T);
MOE_API size_t moe_route_workspace_bytes(moe_t ctx, int T);

/* Routing half of the layer: router logits, top-k, softmax over the selected logits,
 * histogram, offsets and the stable permutation.  Outputs (caller-owned device memory):
 *   topk_idx       [T, k] int32   selected experts, largest logit first
 *   topk_w         [T, k] fp32    routing weights (sum to 1 per token)
 *   expert_offsets [E + 1] int32  row offsets of the expert segments (offsets[E] = T*k)
 *   perm           [T * k] int32  token of each row
 *   inv_perm       [T, k] int32   row of each (token, slot)
 * workspace: at least moe_route_workspace_bytes(ctx, T) bytes, 16-byte aligned.
 * T = 0 writes expert_offsets = 0 and nothing else. */
MOE_API moe_status moe_route(moe_t ctx, int T, const void* x_bf16, const void* W_router_bf16,
                     const float* b_router, int32_t* topk_idx, float* topk_w,
                     int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                     void* workspace, size_t ws_bytes, moe_stream_t stream);

/* The whole layer: writes out [T, H] fp32 (every element).  workspace: at least
 * moe_workspace_bytes(ctx, T) bytes.  The kernel family of each expert is chosen on the device
 * (see moe_path); the host only leaves out families that no expert can reach (an expert holds
 * at most T rows), so the call never synchronises.  T = 0 is a no-op. */
MOE_API moe_status moe_forward(moe_t ctx, int T, const void* x_bf16, const void* W_router_bf16,
                       const float* b_router, const void* W_gate_up_bf16,
                       const void* W_down_bf16, float* out, void* workspace, size_t ws_bytes,
                       moe_stream_t stream);

/* The whole layer with MXFP4 expert weights (W4A16): the experts' native format (Persona
 * Kappa forum post, "Quantization-Aware Training": MXFP4 with bf16 activations), read as OCP
 * Microscaling FP4 -- E2M1 codes, blocks of 32 consecutive K elements of one weight column
 * sharing an E8M0 scale 2^(s - 127) (s = 255: NaN).  For a [K, N] expert matrix:
 *   codes  [N, K/2] uint8  row n = column n of the matrix; byte j holds element k = 2j in
 *                          bits 0-3 and k = 2j + 1 in bits 4-7
 *   scales [K/32, N] uint8 scale of block k/32 of column n
 * gu_codes [E, 2I, H/2] and gu_scales [E, H/32, 2I] hold W_gate_up [E, H, 2I] (gate columns
 * [0, I), up columns [I, 2I)); dn_codes [E, H, I/2] and dn_scales [E, I/32, H] hold W_down
 * [E, I, H].  x, W_router, b_router and out as in moe_forward; all pointers 16-byte aligned.
 * Two kernel families: MOE_PATH_AUTO streams the weights in calls of at most 176 tokens and
 * runs the MXFP4 expert-tile kernel above; MOE_PATH_STREAM forces streaming, MOE_PATH_TILE and
 * MOE_PATH_GEMM expert tiles (there is no MXFP4 row-tile GEMM).
 *   - expert tiles: the codes are widened to bf16 weights in shared memory (exact: an E2M1 value
 *     times 2^(s - 127) has two significant bits; bf16 holds it for 2 <= s <= 252, and for
 *     smaller s as a subnormal down to 2^-133) and multiplied with the bf16 activations on
 *     tcgen05 (fp32 accumulate): the pages' W4A16 as written.
 *   - weight streaming: the products take the E2M1 values (exact in f16) and the activations
 *     converted from bf16 to f16, exact for magnitudes 2^-14 .. 65504 (smaller ones keep fewer
 *     bits); each 32-element block's fp32 result is scaled by its E8M0 factor in fp32.  An
 *     input beyond 65504 in magnitude would become infinite there: the call then flags it and
 *     the next moe_sync_status returns MOE_ERR_UNSUPPORTED (use MOE_PATH_TILE for such inputs).
 * workspace: at least moe_workspace_bytes_mxfp4(ctx, T) bytes (it depends on the path setting).
 * T = 0 is a no-op. */
MOE_API size_t moe_workspace_bytes_mxfp4(moe_t ctx, int T);
MOE_API moe_status moe_forward_mxfp4(moe_t ctx, int T, const void* x_bf16,
                                     const void* W_router_bf16, const float* b_router,
                                     const void* gu_codes, const void* gu_scales,
                                     const void* dn_codes, const void* dn_scales, float* out,
                                     void* workspace, size_t ws_bytes, moe_stream_t stream);

/* ---- Expert parallelism: the device work on either side of the exchange ----------------
 * With the E experts split over G GPUs (E/G each), every GPU routes its own tokens with
 * moe_route (full E), puts the routed rows in expert order with moe_permute, sends each
 * expert's rows to the GPU that owns it (an all-to-all over NVLink, sizes from the
 * histogram: the rows of the owner's experts are one contiguous run of x_perm), runs
 * moe_experts on what it received with a handle made for its E/G experts, sends the results
 * back, and adds each token's k results with moe_combine.  The pages kept every expert on
 * each GPU (Persona Kappa forum post, "The Config": expert-parallel degree 1); the split
 * divides the expert weight bytes each GPU streams in decode by G.  The exchange is the
 * caller's (NCCL all-to-all); these calls only enqueue kernels on `stream`.
 *
 * moe_permute: x_perm [T*k, H] bf16 = x[perm[r]] and row_w [T*k] fp32 = the routing weight
 *   of row r (topk_w[t, j] where inv_perm[t, j] = r), from moe_route's perm, inv_perm and
 *   topk_w.  A perm entry outside [0, T) skips its row and makes moe_sync_status return
 *   MOE_ERR_ARG.
 * moe_experts: the expert half of the layer on R rows that arrive as S*E segments (E = this
 *   handle's experts): seg_counts [S, E] int32 in device memory holds the rows of expert e
 *   from source s; rows are stored source-major, experts ascending inside a source (what an
 *   all-to-all of per-owner runs of x_perm delivers).  Writes
 *     y_rows[r] = row_w[r] * (swiglu(x_rows[r] W_gate_up[e]) W_down[e])   fp32 [R, H]
 *   with e the expert of r's segment.  Each expert's kernel family follows the handle's
 *   path setting, from its rows summed over the sources.  Counts that do not sum to R make
 *   moe_sync_status return MOE_ERR_ARG (rows past R are never read or written).  S * E <=
 *   4096.  workspace: moe_experts_workspace_bytes(ctx, R, S).
 * moe_combine: out [T, H] fp32 = sum over j < k of y_rows[inv_perm[t, j]], in slot order
 *   (y_rows in the row order of this GPU's x_perm, as the exchange back returns it). */
MOE_API moe_status moe_permute(moe_t ctx, int T, const void* x_bf16, const int32_t* perm,
                               const int32_t* inv_perm, const float* topk_w, void* x_perm_bf16,
                               float* row_w, moe_stream_t stream);
MOE_API size_t moe_experts_workspace_bytes(moe_t ctx, int R, int S);
MOE_API moe_status moe_experts(moe_t ctx, int R, int S, const int32_t* seg_counts,
                               const void* x_rows_bf16, const float* row_w,
                               const void* W_gate_up_bf16, const void* W_down_bf16,
                               float* y_rows, void* workspace, size_t ws_bytes,
                               moe_stream_t stream);
MOE_API moe_status moe_combine(moe_t ctx, int T, const int32_t* inv_perm, const float* y_rows,
                               float* out, moe_stream_t stream);

/* Choose the path.  crossover_T >= 0 also sets the largest call (in tokens) in which AUTO uses
 * the weight-streaming family (default: the largest T whose touched experts' tiles fill less
 * than two waves of the GPU or leave their last wave under 85 % full: 5 for the 20b and 4 for
 * the 120b shape on 148 SMs; moe_tune measures it);
 * crossover_T < 0 keeps the current one.  MOE_ERR_ARG for an unknown path. */
MOE_API moe_status moe_set_path(moe_t ctx, moe_path path, int crossover_T);

/* Current path setting and streaming crossover (tokens). */
MOE_API moe_status moe_get_path(moe_t ctx, moe_path* path, int* crossover_T);

/* The AUTO thresholds, in rows of one expert: stream_rows (default 16, one streaming chunk),
 * tile_rows (default 192: up to there the expert tiles, with 256 rows per tile once a call's mean
 * load reaches 128 rows, beat the row tiles) and per_expert (default 0): 1 lets one call run
 * expert tiles and row tiles side by side (each expert by its own count, the row tiles on the
 * handle's second stream), 0 keeps the call's non-streamed experts in one of the two by their
 * mean count.  A negative value keeps the current setting. */
MOE_API moe_status moe_set_dispatch(moe_t ctx, int stream_rows, int tile_rows, int per_expert);
MOE_API moe_status moe_get_dispatch(moe_t ctx, int* stream_rows, int* tile_rows,
                                    int* per_expert);

/* Measure the AUTO settings on this device with the caller's layer: times the whole layer
 * (median of 5 calls after 2 warm-ups) with every expert forced through each family, at
 * T = 1, 2, 4, 8, 12, 16, 24, 32, 48, 64, ... up to T_max, streaming against expert tiles and
 * expert tiles against row tiles.  For each pair it takes the largest T at which the first
 * family was not slower (stopping once the second has been faster for a doubling of T): the
 * first gives the streaming crossover (tokens), the second the tile_rows threshold as the mean
 * rows per expert at that T, ceil(T * k / E).  x must hold T_max rows, out T_max rows;
 * workspace at least moe_tune_workspace_bytes(ctx, T_max).  Synchronises `stream`; the path
 * setting is left as it was.  *crossover_out (may be NULL) receives the streaming crossover;
 * moe_get_dispatch gives tile_rows. */
MOE_API size_t moe_tune_workspace_bytes(moe_t ctx, int T_max);
MOE_API moe_status moe_tune(moe_t ctx, int T_max, const void* x_bf16, const void* W_router_bf16,
                    const float* b_router, const void* W_gate_up_bf16,
                    const void* W_down_bf16, float* out, void* workspace, size_t ws_bytes,
                    moe_stream_t stream, int* crossover_out);

/* Which kernels the last moe_forward (mxfp4 = 0) or moe_forward_mxfp4 (mxfp4 = 1) call of T
 * tokens on this workspace ran: synchronises `stream`, then writes for each family (0 weight
 * streaming, 1 expert tiles, 2 row tiles) the number of work-list entries it processed, or -1
 * if the call did not launch that family.  An entry is a row chunk of one expert (up to 16, 128
 * or 256 rows).  The handle's path and thresholds must be those of that call.  For
 * diagnostics and tests; reads device memory. */
MOE_API moe_status moe_last_dispatch(moe_t ctx, int T, int mxfp4, const void* workspace,
                                     size_t ws_bytes, int32_t* entries, moe_stream_t stream);

/* Synchronise `stream`, then read and clear the handle's device status word.  Returns
 * MOE_ERR_TIMEOUT if a device-side bounded wait gave up since the last call, MOE_ERR_ARG if a
 * kernel met an index or count outside its buffers (moe_permute, moe_experts, moe_combine),
 * MOE_ERR_UNSUPPORTED if an MXFP4 streaming call met an input beyond f16's range, MOE_ERR_CUDA if
 * the stream reports an error, MOE_OK otherwise. */
MOE_API moe_status moe_sync_status(moe_t ctx, moe_stream_t stream);

/* Static text for a status code ("unknown status" for values outside the enum). */
MOE_API const char* moe_status_string(moe_status s);

/* Number of kernels this handle has launched since it was created (host counter). */
MOE_API uint64_t moe_launch_count(moe_t ctx);

/* Kernel timing for benchmarks.  moe_profile_begin(ctx, max_calls) creates CUDA events for up
 * to max_calls subsequent moe_forward calls; each of those records an event pair around every
 * kernel it launches, on the call's stream.  moe_profile_end synchronises, and writes for
 * each kernel kind i < n_kinds the total milliseconds into ms[i] and its launch count into
 * launches[i], then frees the events.  Kinds: 0 router, 1 routing finalize / scan / scatter,
 * 2 gather of the rows into expert order, 3 / 4 gate/up projection + SwiGLU / down projection
 * + combine on the weight-streaming kernels, 5 conversion of the input to f16 (MXFP4 path),
 * 6 / 7 the same projections on the expert-tile kernels, 8 / 9 on the row-tile grouped GEMM.
 * moe_profile_kind_name gives a kind's name. */
#define MOE_PROFILE_KINDS 10
MOE_API moe_status moe_profile_begin(moe_t ctx, int max_calls);
MOE_API moe_status moe_profile_end(moe_t ctx, float* ms, int* launches, int n_kinds);
MOE_API const char* moe_profile_kind_name(int kind);

/* Routing into the library's own device scratch, for callers that cannot allocate.
 *
 * No counterpart on the source pages: this is an interface convenience of this library.
 * moe_route needs a caller-allocated workspace; some callers cannot provide one because they
 * may not allocate device memory at call time (every device byte belongs to another
 * allocator or pool, or allocation after start-up is forbidden, or the caller is plain C
 * without an allocator).  moe_route_static takes moe_route's arguments minus the workspace
 * and allocates nothing: its scratch is a fixed array of moe_route_static_max_bytes() bytes
 * (2 MiB) compiled into the library, which every device that loads the library keeps until
 * the process exits.  moe_create looks up the array's device address (a runtime call that
 * allocates nothing) and keeps it in the handle.
 *   - Results: for T <= 64 identical to moe_route.  For T > 64 the router is not split over
 *     the hidden dimension (moe_route splits it when T is small enough to leave SMs idle), so
 *     the fp32 logit sums run in another order: topk_w can differ in the last bits, and a
 *     token whose k-th and (k+1)-th logits are within rounding of each other (a near tie)
 *     can select differently.  For the same reason it is slower than moe_route for T between
 *     65 and a few thousand (ceil(T/64) blocks each sum over all of H).
 *   - The handle's device must be the current device (MOE_ERR_ARG otherwise).
 *   - If the routing scratch for T does not fit in the array, the call returns
 *     MOE_ERR_WORKSPACE and enqueues nothing.  The scratch is ceil(H/256)*T*E*4 bytes of
 *     partial logits for T <= 64 and ceil(T/64)*E*4 bytes of per-block expert counts above
 *     that; with H = 2880 every T <= 64 fits for any E, and larger T fits for E = 32 up to
 *     T = 1,048,320, for E = 128 up to T = 262,016 and for E = 256 up to T = 130,944.
 *   - Every scratch word a call reads is written earlier in the same call, so no clearing is
 *     needed between calls.  All calls share the one array: two calls whose work overlaps on
 *     the GPU (different streams, or different handles on one device) race and give undefined
 *     results. */
MOE_API size_t moe_route_static_max_bytes(void);
MOE_API moe_status moe_route_static(moe_t ctx, int T, const void* x_bf16,
                                    const void* W_router_bf16, const float* b_router,
                                    int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                                    int32_t* perm, int32_t* inv_perm, moe_stream_t stream);

/* Self-test of the device timeout path: launches one kernel that waits on a barrier nothing
 * completes, with a limit of `limit_us` microseconds (1..1000000), after which it sets the
 * status word and returns.  The next moe_sync_status then returns MOE_ERR_TIMEOUT.  No memory
 * is touched apart from the status word. */
MOE_API moe_status moe_selftest_timeout(moe_t ctx, int limit_us, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
