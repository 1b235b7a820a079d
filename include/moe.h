/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse top-k MoE FFN: the forward
 * pass, the aux-loss-free balancer's bias update, and the backward pass (fp32
 * problems on SIMT kernels, bf16 problems on the tensor cores).
 *
 * The forward pass, step by step:
 *   route    : logits = x . gate_w^T, scores (softmax / sigmoid / sqrtsoftplus),
 *              top-k with an optional fp32 bias, optional renormalisation;
 *   dispatch : per-expert histogram, exclusive scan to segment offsets, stable
 *              permutation of token copies into contiguous per-expert segments;
 *   grouped SwiGLU : h = silu(x W_g^T) * (x W_u^T) per routed segment, then
 *              y = w * (h W_d^T), only over experts that received tokens;
 *   shared expert  : the same MLP over all tokens, optionally sigmoid-gated;
 *   combine  : out[t] = sum_j y[(t, j)] + shared[t], back in token order.
 *
 * Passages each call follows (page title, section):
 *   "mstar.model.components.moe" -- Router contract (hidden_states [T,H] in;
 *     routing_weights [T,k] and int64 selected_experts [T,k] out), TopKRouter
 *     (softmax top-k, norm_topk_prob), SparseMoeBlock (fused layout
 *     gate_up_proj [E,2I,H], down_proj [E,H,I]), SparseMoeBlockWithSharedExpert
 *     (out = routed(x) + sigmoid(shared_gate(x)) * shared_expert(x)).
 *   "Sparse MoE FFN for DFlash-family drafters" -- What's here: MoEGate
 *     (sqrtsoftplus scores, fp32 aux-loss-free bias used for selection only),
 *     GroupedExperts (stacked [E, out, in] weights), SparseMoE (one argsort into
 *     contiguous per-expert segments, grouped GEMM with no host syncs, one
 *     shared expert).
 *   "feat: Phase 43 -- Sparse/Grouped MoE Dispatch" -- Summary and Neural
 *     Network: only the assigned top-k experts are computed, tokens grouped per
 *     expert (arg_sort, index_select, index_add); empty expert groups skipped.
 *   "MoE: shared experts, parameterized V_TOPK routing, explicit stage
 *     attribution" -- 1. (routing at any expert count, "topk must be
 *     positive"), 3. Tests (ungated, sigmoid-gated and n_shared-fused shared
 *     experts), 4. (shared width is the fused width n_shared * I).
 *
 * Conventions for every call:
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     stated otherwise. The library never allocates, frees or synchronises,
 *     except moe_read_device_error / moe_check_device_error, which
 *     synchronise the given stream.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously. Outputs are valid once the stream has
 *     passed the call.
 *   - Row-major, densely packed tensors. x, the weights, x_perm and out have
 *     the problem dtype (fp32 or bf16). y_perm and shared_out are fp32 for
 *     every problem dtype: the only roundings to bf16 on the path are the
 *     SwiGLU activation h (an operand of the down GEMM) and the final output.
 *     Biases, routing weights and the shared gate values are fp32.
 *     selected_experts is int64; counts, offsets, sorted_pairs and pair_pos
 *     are int32.
 *   - Every pointer must be 16-byte aligned. H, I and I_shared must be
 *     multiples of 8 (16-byte rows for the TMA engine).
 *   - Arguments are validated on the host before any launch. On an error
 *     status nothing is launched and no output is written.
 *   - Bad data found on the device (an expert id outside [0, E) handed to
 *     moe_dispatch) does not fault: the pair is skipped, a flag in the
 *     workspace header is set, and moe_read_device_error reports it.
 *   - The workspace (size from moe_workspace_size) is caller-owned device
 *     memory. Zero its header once with moe_workspace_init. Calls on different
 *     streams need distinct workspaces. There is no global mutable state.
 *   - T == 0 is a valid no-op.
 *   - Limits: 1 <= k <= E <= 256.
 */
#ifndef STM_MOE_H
#define STM_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* the same type as cudaStream_t */
typedef struct CUevent_st *moe_event_t;   /* the same type as cudaEvent_t  */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = 1,  /* bad size, pointer, alignment or enum    */
  MOE_ERR_UNSUPPORTED = 2,       /* valid but not implemented combination  */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3,
  MOE_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed   */
  MOE_ERR_DEVICE_FLAG = 5        /* a kernel flagged bad data or a timeout */
} moe_status;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype;
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1, MOE_SCORE_SQRTSOFTPLUS = 2 } moe_score;
/* LOGIT: bias added to the router logits (enters the scores).
 * SELECT: bias added to the scores for choosing the top-k only; the routing
 * weights come from the unbiased scores (aux-loss-free balancing bias). */
typedef enum { MOE_BIAS_NONE = 0, MOE_BIAS_LOGIT = 1, MOE_BIAS_SELECT = 2 } moe_bias_mode;
typedef enum { MOE_SHARED_NONE = 0, MOE_SHARED_PLAIN = 1, MOE_SHARED_SIGMOID_GATED = 2 } moe_shared_kind;

/* Device-side error bits reported by moe_read_device_error. */
#define MOE_DEVERR_BAD_EXPERT_ID 1 /* selected_experts held an id outside [0,E) */
#define MOE_DEVERR_WAIT_TIMEOUT 2  /* a pipeline wait gave up (never expected)   */
#define MOE_DEVERR_SMEM_LAYOUT 4   /* a GEMM found its shared memory misaligned
                                      and computed nothing (never expected)   */

typedef struct moe_problem {
  int64_t T;        /* tokens                                               */
  int64_t H;        /* hidden size                                          */
  int64_t E;        /* routed experts                                       */
  int64_t k;        /* experts per token (top-k)                            */
  int64_t I;        /* routed expert intermediate size                      */
  int64_t I_shared; /* shared expert intermediate size (fused width), or 0  */
  int32_t dtype;    /* moe_dtype                                            */
  int32_t score;    /* moe_score                                            */
  int32_t bias_mode;   /* moe_bias_mode                                     */
  int32_t renormalize; /* nonzero: routing weights divided by their sum     */
  int32_t shared;      /* moe_shared_kind                                   */
  int32_t reserved;    /* must be 0                                         */
} moe_problem;

typedef struct moe_weights {
  const void *gate_w;         /* [E, H] router weight                            */
  const float *bias;          /* [E] fp32, or NULL when bias_mode == NONE        */
  const void *gate_up;        /* [E, 2I, H]: rows 0..I-1 gate, rows I..2I-1 up   */
  const void *down;           /* [E, H, I]                                       */
  const void *shared_gate_up; /* [2*I_shared, H] (gate rows first), or NULL      */
  const void *shared_down;    /* [H, I_shared], or NULL                          */
  const void *shared_gate;    /* [H] gate vector (SIGMOID_GATED only), or NULL   */
} moe_weights;

/* Stages timed through moe_forward_ex's stage events, in launch order. */
enum {
  MOE_STAGE_ROUTE = 0,
  MOE_STAGE_DISPATCH = 1,
  MOE_STAGE_GATE_UP = 2,
  MOE_STAGE_DOWN = 3,
  MOE_STAGE_SHARED = 4,
  MOE_STAGE_COMBINE = 5,
  MOE_NUM_STAGES = 6
};

/* Bytes of workspace moe_forward needs for problem p (each of the other
 * forward calls needs at most this much; moe_backward has its own size,
 * moe_backward_workspace_size). Host only. */
moe_status moe_workspace_size(const moe_problem *p, size_t *bytes);

/* Zero the workspace header (error flags). Call once after allocating it. */
moe_status moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream);

/* Router ("mstar.model.components.moe", Router contract and TopKRouter;
 * "Sparse MoE FFN for DFlash-family drafters", MoEGate).
 *   x [T,H], gate_w [E,H]; bias [E] fp32 or NULL (per p->bias_mode);
 *   shared_gate [H] or NULL: when given, shared_gamma [T] (fp32) receives
 *   sigmoid(x[t] . shared_gate).
 *   routing_weights [T,k] fp32 and selected_experts [T,k] int64 are written;
 *   slot j holds the (j+1)-th largest selection key, equal keys ordered by
 *   ascending expert index. */
moe_status moe_route(const moe_problem *p, const void *x, const void *gate_w, const float *bias,
                     const void *shared_gate, float *routing_weights, int64_t *selected_experts,
                     float *shared_gamma, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Router selection only, from given fp32 logits [T,E] (bias applied per
 * p->bias_mode). Lets tests compare selection bit-exactly on identical
 * logits. */
moe_status moe_topk_from_logits(const moe_problem *p, const float *logits, const float *bias,
                                float *routing_weights, int64_t *selected_experts, moe_stream_t stream);

/* Sorted-segment dispatch ("Sparse MoE FFN for DFlash-family drafters",
 * SparseMoE; "feat: Phase 43", sparse_grouped_dispatch).
 *   Pair q = t*k + j routes token t to expert selected_experts[q].
 *   counts [E]: pairs per expert. offsets [E+1]: exclusive prefix sum,
 *   offsets[E] = pairs dispatched. sorted_pairs [T*k]: pair at segment
 *   position p, ascending q inside each segment (stable). pair_pos [T*k]:
 *   inverse, -1 for a pair skipped because of a bad expert id.
 *   x_perm [T*k, H]: x_perm[p] = x[sorted_pairs[p] / k]; x and x_perm may
 *   both be NULL to compute the permutation only. */
moe_status moe_dispatch(const moe_problem *p, const int64_t *selected_experts, const void *x,
                        int32_t *counts, int32_t *offsets, int32_t *sorted_pairs, int32_t *pair_pos,
                        void *x_perm, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Sorted-segment dispatch that allocates nothing. The pages have no
 * counterpart to this call; it exists for callers that cannot give the
 * library a workspace because they may not allocate device memory: code
 * running while another thread captures a CUDA graph in global capture mode
 * (where cudaMalloc is an error), plug-ins inside a host framework whose
 * memory pool owns the GPU, and latency-critical paths that must not wait on
 * an allocator.
 *   Same arguments and results as moe_dispatch, minus the workspace: the
 *   per-block count matrix the dispatch kernels pass to each other lives in
 *   a static 1 MiB device array inside this library, and the histogram's
 *   completion ticket in a static 4-byte one (every GPU that loads the
 *   library holds both until the process exits). Problems needing more than
 *   2^18 count entries, ceil(T / max(1, 256 / k)) * E, are rejected with
 *   MOE_ERR_UNSUPPORTED before anything is launched.
 *   `stream` must belong to the current device: the arrays used are the
 *   current device's. The first call on a device looks up their device
 *   addresses (with that device current; a failed lookup is retried by the
 *   next call); make that first call before any stream capture. Calls
 *   allocate and free nothing; each clears the ticket (an async memset on
 *   `stream`) before its two kernels.
 *   Every call reuses the same arrays: calls whose work overlaps on the GPU
 *   (two streams, or two host threads) race and corrupt each other's
 *   results; serialise them. Nothing carried over from an earlier call is
 *   read. A pair with an expert id outside [0, E) is skipped (pair_pos -1)
 *   as in moe_dispatch, but no error flag is recorded. */
moe_status moe_dispatch_noalloc(const moe_problem *p, const int64_t *selected_experts, const void *x,
                                int32_t *counts, int32_t *offsets, int32_t *sorted_pairs, int32_t *pair_pos,
                                void *x_perm, moe_stream_t stream);

/* moe_dispatch for an array of slots some of which are empty: every id
 * outside [0, E) (for example -1) marks an empty slot, which is skipped
 * (pair_pos -1, no row copied) without an error flag. Arguments, workspace
 * and results as for moe_dispatch. Used by the expert-parallel exchange to
 * regroup the slots it received by local expert. */
moe_status moe_dispatch_slots(const moe_problem *p, const int64_t *selected_experts, const void *x,
                              int32_t *counts, int32_t *offsets, int32_t *sorted_pairs, int32_t *pair_pos,
                              void *x_perm, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Grouped SwiGLU over the routed segments ("mstar.model.components.moe",
 * SparseMoeBlock fused layout; "Sparse MoE FFN for DFlash-family drafters",
 * grouped GEMM with no host syncs).
 *   For each expert e with offsets[e] < offsets[e+1] and each row p in that
 *   segment: h = silu(x_perm[p] . gate^T) * (x_perm[p] . up^T) (h kept in
 *   the workspace, rounded to the problem dtype), then
 *   y_perm[p] = routing_weights[sorted_pairs[p]] * (h . down[e]^T), fp32
 *   [T*k, H]. routing_weights and sorted_pairs may both be NULL (scale 1).
 *   Experts with no rows are never read. The segment table stays on the
 *   device; no host synchronisation. */
moe_status moe_grouped_swiglu(const moe_problem *p, const void *x_perm, const int32_t *offsets,
                              const void *gate_up, const void *down, const float *routing_weights,
                              const int32_t *sorted_pairs, void *y_perm, void *ws, size_t ws_bytes,
                              moe_stream_t stream);

/* Shared expert over all T tokens ("mstar.model.components.moe",
 * SparseMoeBlockWithSharedExpert; "MoE: shared experts ...", 3. Tests).
 *   shared_out [T,H] fp32 = gamma[t] * SwiGLU(x[t]) with gamma =
 *   shared_gamma[t] when shared_gamma is not NULL, else 1. */
moe_status moe_shared_expert(const moe_problem *p, const void *x, const void *shared_gate_up,
                             const void *shared_down, const float *shared_gamma, void *shared_out,
                             void *ws, size_t ws_bytes, moe_stream_t stream);

/* Combine back to token order ("feat: Phase 43", index_add scatter).
 *   out[t] = round( sum_{j<k} y_perm[pair_pos[t*k+j]] + shared_out[t] ), with
 *   fp32 y_perm [T*k,H] and shared_out [T,H], the sum in fp32 in slot order,
 *   rounded once to the problem dtype; shared_out may be NULL; pairs with
 *   pair_pos < 0 contribute nothing. */
moe_status moe_combine(const moe_problem *p, const void *y_perm, const int32_t *pair_pos,
                       const void *shared_out, void *out, moe_stream_t stream);

/* Whole forward: route, dispatch, grouped SwiGLU, shared expert, combine.
 *   x [T,H] -> out [T,H]; routing_weights [T,k] and selected_experts [T,k] are
 *   also written (router contract). All intermediates live in ws. */
moe_status moe_forward(const moe_problem *p, const moe_weights *w, const void *x, void *out,
                       float *routing_weights, int64_t *selected_experts, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_forward with two options:
 *   aux_stream: when not NULL (and not `stream`) and the problem has a shared
 *     expert, that expert runs on aux_stream (fork / join through two events
 *     the call creates and releases):
 *     - a small shared expert (its gate_up GEMM has at most 74 128x128
 *       tiles, as for a decode batch) runs beside the whole routed path and
 *       `stream` waits for it before the combine; its sigmoid gate is then
 *       computed by its own small kernel;
 *     - a larger one occupies every SM while it runs, so it starts after the
 *       route (whose top-k kernel computes the gate) and runs beside the
 *       dispatch kernels only; `stream` waits for it before the routed gate_up
 *       GEMM. The dispatch stage's event interval then ends when both are
 *       done and the shared stage's interval is empty.
 *     All work is complete once `stream` has passed the call.
 *   stage_events: NULL, or MOE_NUM_STAGES + 1 caller-created events recorded
 *     on `stream` before each stage (MOE_STAGE_*) and after the last one; a
 *     NULL entry is skipped. While `stream` is being captured into a CUDA
 *     graph they are recorded as event record nodes (cudaEventRecordExternal),
 *     so every replay of the graph records them. */
moe_status moe_forward_ex(const moe_problem *p, const moe_weights *w, const void *x, void *out,
                          float *routing_weights, int64_t *selected_experts, void *ws, size_t ws_bytes,
                          moe_stream_t stream, moe_stream_t aux_stream, moe_event_t *stage_events);

/* Which implementation serves problem p's routed gate_up GEMM: 0 = SIMT
 * fp32; 1 = tcgen05/TMEM, one CTA per 128-row tile; 2 = tcgen05 CTA pairs
 * (cta_group::2) per 256-row tile, chosen when segments average at least 192
 * rows (the same threshold for the down GEMM). Host only. */
moe_status moe_gemm_path(const moe_problem *p, int32_t *path);

/* Number of kernel launches one forward of problem p makes (0 when T == 0):
 * moe_forward when two_streams == 0, moe_forward_ex with an aux_stream
 * otherwise. Host only. */
moe_status moe_launches_per_forward(const moe_problem *p, int32_t two_streams, int32_t *n);

/* Synchronise `stream`, read the workspace error bits into *code (host
 * pointer), clear them. Returns MOE_ERR_DEVICE_FLAG when any bit was set. */
moe_status moe_read_device_error(void *ws, int32_t *code, moe_stream_t stream);

/* The same call with the stream before the result pointer. */
moe_status moe_check_device_error(void *ws, moe_stream_t stream, int32_t *code);

/* Diagnostic of the bounded pipeline waits. Every mbarrier wait in the
 * tensor-core GEMMs gives up after a fixed budget of SM clocks, records
 * MOE_DEVERR_WAIT_TIMEOUT in the workspace header and lets the kernel return,
 * so a stalled pipeline is reported rather than hanging the GPU. This call
 * launches one thread that waits, through the same routine with a ~10 ms
 * budget, on an mbarrier nothing arrives on; afterwards moe_read_device_error
 * on `ws` reports MOE_DEVERR_WAIT_TIMEOUT and the context stays usable. The
 * pages have no counterpart to this call. */
moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, moe_stream_t stream);

/* Aux-loss-free balancing: the deferred sign-controller update of the fp32
 * selection bias ("Sparse MoE FFN for DFlash-family drafters", What's here:
 * MoEGate's bias moves by a sign controller from all-reduced expert loads,
 * never by gradients; a forward stashes its routing counts and the update is
 * applied before the next forward; a second apply changes nothing).
 *   moe_bias_stash: load_stash[e] += counts[e] for e < p->E. counts [E] int32
 *     as written by moe_dispatch / the forward; load_stash [E] int64, device,
 *     caller-owned, zeroed by the caller before first use.
 *   moe_bias_update: with L = load_stash (already summed over data-parallel
 *     ranks when there are several) and mean m = sum(L) / E, bias[e] += rate
 *     when L[e] < m, bias[e] -= rate when L[e] > m, unchanged when L[e] == m
 *     (one fp32 add; the comparison is exact, in integers); then load_stash is
 *     zeroed. bias [E] fp32, device. rate must be finite.
 * Only p->E is read from the problem. One 256-thread block each; async on
 * `stream`; pointers must be aligned to their element size. */
moe_status moe_bias_stash(const moe_problem *p, const int32_t *counts, int64_t *load_stash, moe_stream_t stream);
moe_status moe_bias_update(const moe_problem *p, int64_t *load_stash, float *bias, float rate,
                           moe_stream_t stream);

/* Device address of the per-expert counts [E] (int32) that the last
 * moe_forward / moe_forward_ex on `ws` wrote, for moe_bias_stash: it stays
 * valid, and the counts unchanged, until the next call that uses ws. Host
 * only; checks ws_bytes against the problem's workspace size. */
moe_status moe_forward_counts(const moe_problem *p, const void *ws, size_t ws_bytes, const int32_t **counts);

/* ---- Expert parallelism over peer memory -------------------------------------
 * The routed experts of one layer split over G ranks (rank r owns experts
 * [r*E/G, (r+1)*E/G); E divisible by G; the router and the shared expert are
 * replicated; every rank runs the same problem p, with T its own tokens).
 * Each rank owns an arena (moe_ep_arena_size bytes, device memory, zeroed
 * once before first use) that every rank can store to: on one node, CUDA IPC
 * mappings over NVLink; on one GPU, ordinary device memory. `arenas` is a
 * device array of the G arenas' base addresses (this rank's own among them,
 * at index `rank`), `own_arena` this rank's (as a host-side value). Every
 * transfer is a 16-byte store to a peer's arena; nothing is read on the
 * host, and the calls can be captured in a CUDA graph. The arena keeps the
 * rank's forward count (its epoch): step 2 advances it on the device, and
 * steps 3, 5 and 6 use it. Per forward, rank r:
 *   1. routes and dispatches its tokens over all E experts (moe_route,
 *      moe_dispatch: sorted rows, offsets [E+1], sorted_pairs);
 *   2. moe_ep_send: stores each sorted row of owner q's experts, with its
 *      routing weight and local expert id, into q's arena (slots
 *      [r*T*k, (r+1)*T*k) belong to source r), marks the rest of those slots
 *      empty (id -1), then publishes the new epoch into q's rows flag for
 *      source r;
 *   3. moe_ep_wait(which 0): waits for all G sources' rows flags;
 *   4. moe_dispatch_slots over the G*T*k slots of its arena (k 1, E/G
 *      experts, ids and rows from the arena), moe_grouped_swiglu with the
 *      arena's routing weights: y_sorted [G*T*k, H] fp32;
 *   5. moe_ep_return: stores each weighted row back into its source's arena
 *      at the source's sorted position, then publishes the epoch into each
 *      source's return flag for owner r;
 *   6. moe_ep_wait(which 1): waits for all G owners' return flags; the
 *      arena's y region [T*k, H] fp32 is then this rank's y_perm, which
 *      moe_combine (with the pair_pos of step 1) turns into the output.
 * A wait polls each flag at most max_polls times (about 256 ns apart); on
 * giving up it raises MOE_DEVERR_WAIT_TIMEOUT in *err (a workspace header's
 * error bits, or NULL) and returns, so the stream goes on (with wrong rows).
 * Per-row arithmetic is that of the one-GPU forward: the output equals
 * moe_forward's for the same tokens and weights. */

/* Bytes of one rank's arena for problem p on G ranks. Host only. */
moe_status moe_ep_arena_size(const moe_problem *p, int32_t G, size_t *bytes);
/* Byte offsets inside an arena of the rows flags u64[G], return flags u64[G],
 * the epoch u64, received rows x [G*T*k, H] (problem dtype), their routing
 * weights fp32 [G*T*k], their local expert ids int64 [G*T*k] and the
 * returned rows y fp32 [T*k, H] (any pointer may be NULL). Host only. */
moe_status moe_ep_arena_offsets(const moe_problem *p, int32_t G, size_t *rows_flag, size_t *ret_flag,
                                size_t *epoch, size_t *x, size_t *w, size_t *id, size_t *y);
/* Step 2. x_perm [T*k, H], offsets [E+1], sorted_pairs [T*k] from this
 * rank's moe_dispatch; routing_weights [T, k] fp32 and selected_experts
 * [T, k] int64 from its moe_route. Async on `stream`. */
moe_status moe_ep_send(const moe_problem *p, int32_t G, int32_t rank, void *const *arenas, void *own_arena,
                       const void *x_perm, const int32_t *offsets, const int32_t *sorted_pairs,
                       const float *routing_weights, const int64_t *selected_experts, moe_stream_t stream);
/* Steps 1 (its dispatch part) and 2 in one: moe_dispatch's histogram and
 * scan, then the ranking kernel stores each pair's token row straight into
 * its owner's arena (no x_perm is written), with its routing weight and
 * local id, marks the owners' empty slots and publishes the new epoch, as
 * moe_ep_send does. counts, offsets, sorted_pairs and pair_pos as from
 * moe_dispatch (pair_pos is the combine's); routing_weights [T, k] fp32 from
 * moe_route; workspace as for moe_dispatch. T = 0 returns
 * MOE_ERR_UNSUPPORTED (an empty batch sends through moe_ep_send). */
moe_status moe_ep_dispatch_send(const moe_problem *p, int32_t G, int32_t rank, void *const *arenas, void *own_arena,
                                const int64_t *selected_experts, const void *x, const float *routing_weights,
                                int32_t *counts, int32_t *offsets, int32_t *sorted_pairs, int32_t *pair_pos,
                                void *ws, size_t ws_bytes, moe_stream_t stream);
/* Steps 4 and 5 in one, bf16 problems (the tensor-core GEMMs): the
 * received slots regrouped by local expert (as moe_dispatch_slots), the
 * grouped gate_up and SwiGLU, and the down GEMM whose epilogue stores each
 * weighted fp32 row straight into its source's arena (the return
 * all-to-all fused with the GEMM: no local y, no separate copy), then the
 * epoch published into every source's return flag. gate_up [E/G, 2I, H] and
 * down [E/G, H, I]: this rank's experts. ws: a workspace of
 * moe_workspace_size bytes for the problem (G*T*k tokens, k 1, E/G experts,
 * no shared expert, no bias). fp32 problems return MOE_ERR_UNSUPPORTED. */
moe_status moe_ep_experts(const moe_problem *p, int32_t G, int32_t rank, void *const *arenas, void *own_arena,
                          const void *gate_up, const void *down, void *ws, size_t ws_bytes, moe_stream_t stream);
/* Steps 3 (which = 0: rows received) and 6 (which = 1: rows returned). */
moe_status moe_ep_wait(const moe_problem *p, int32_t G, void *own_arena, int32_t which, int64_t max_polls,
                       int32_t *err, moe_stream_t stream);
/* Step 5. y_sorted [G*T*k, H] fp32, offsets1 [E/G + 1] and sorted_pairs1
 * [G*T*k] from step 4. */
moe_status moe_ep_return(const moe_problem *p, int32_t G, int32_t rank, void *const *arenas, void *own_arena,
                         const float *y_sorted, const int32_t *offsets1, const int32_t *sorted_pairs1,
                         moe_stream_t stream);

/* ---- Tensor parallelism over peer memory --------------------------------------
 * Every expert's I (and I_shared) split over G ranks, the router replicated,
 * every rank given the same tokens ("mstar.model.components.moe", the
 * tensor-parallel MoE block); each rank's grouped SwiGLU over its slice gives
 * partial fp32 rows y_perm [T*k, H] (and a partial shared output [T, H])
 * whose sums over ranks are the whole ones. The reduction is fused with the
 * combine and runs on peer memory: arenas as for the expert-parallel exchange
 * (moe_tp_arena_size bytes each, zeroed once; each keeps its rank's epoch).
 * H must be a multiple of 8*G. Per forward, rank r:
 *   1. moe_tp_scatter: for every token, the sum of its k partial rows in slot
 *      order plus its partial shared row (fp32, the library's combine
 *      arithmetic), each 1/G column slice stored into that slice's owner's
 *      arena; then the new epoch published into every owner's part flag;
 *   2. moe_tp_wait(which 0): waits for all G sources' partial slices;
 *   3. moe_tp_gather: sums the G slices of its own columns in rank order,
 *      rounds once to the problem dtype, stores them into every rank's
 *      output region, publishes the epoch into every rank's out flag;
 *   4. moe_tp_wait(which 1): the arena's out region [T, H] (problem dtype)
 *      then holds the layer's output, until this rank's next moe_tp_scatter.
 * Waits as in the expert-parallel exchange (bounded; timeout flag). */
moe_status moe_tp_arena_size(const moe_problem *p, int32_t G, size_t *bytes);
/* Byte offsets of the part flags u64[G], out flags u64[G], the epoch u64,
 * the partial slices fp32 [G][T][H/G] and the output [T, H]. Host only. */
moe_status moe_tp_arena_offsets(const moe_problem *p, int32_t G, size_t *part_flag, size_t *out_flag,
                                size_t *epoch, size_t *part, size_t *out);
/* Step 1. y_perm [T*k, H] fp32 and pair_pos [T*k] as for moe_combine;
 * shared_out [T, H] fp32 or NULL. */
moe_status moe_tp_scatter(const moe_problem *p, int32_t G, int32_t rank, void *const *arenas, void *own_arena,
                          const float *y_perm, const int32_t *pair_pos, const float *shared_out, moe_stream_t stream);
/* Step 3. */
moe_status moe_tp_gather(const moe_problem *p, int32_t G, int32_t rank, void *const *arenas, void *own_arena,
                         moe_stream_t stream);
/* Steps 2 (which = 0) and 4 (which = 1). */
moe_status moe_tp_wait(const moe_problem *p, int32_t G, void *own_arena, int32_t which, int64_t max_polls,
                       int32_t *err, moe_stream_t stream);

/* Gradient outputs of moe_backward. All fp32, device, caller-owned, 16-byte
 * aligned, fully overwritten (never accumulated into). */
typedef struct moe_grads {
  float *dx;               /* [T, H]                                          */
  float *d_gate_w;         /* [E, H]                                          */
  float *d_bias;           /* [E] when bias_mode == LOGIT, else NULL          */
  float *d_gate_up;        /* [E, 2I, H]                                      */
  float *d_down;           /* [E, H, I]                                       */
  float *d_shared_gate_up; /* [2*I_shared, H] with a shared expert, else NULL */
  float *d_shared_down;    /* [H, I_shared] with a shared expert, else NULL   */
  float *d_shared_gate;    /* [H] when SIGMOID_GATED, else NULL               */
} moe_grads;

/* Backward of the whole forward ("Sparse MoE FFN for DFlash-family
 * drafters", What's here: the backward pass through the grouped GEMM; Tests:
 * grad parity against a per-expert loop). Gradients of sum(dout * out) for
 * out = moe_forward(x) with the expert choice held at selected_experts:
 * top-k selection is piecewise constant, so no gradient flows through the
 * choice, and none reaches a SELECT bias (it only ranks experts; the
 * balancer moves it). A LOGIT bias gets sum over tokens of dlogits.
 *   x [T,H], dout [T,H], weights as for moe_forward, selected_experts [T,k]
 *   int64 (normally the forward's). Routing weights, the per-expert
 *   activations and outputs are recomputed from x; nothing from the forward
 *   is needed besides the choice.
 *   fp32 problems run on SIMT kernels in fp32 throughout. bf16 problems
 *   (x, dout and the weights bf16) run the expert GEMMs on the tensor cores
 *   and the router's logits, weight gradient and dx on the tensor cores (bf16
 *   operands, fp32 accumulation; [dg du], w*dout, h and dlogits are rounded
 *   to bf16 where they become operands; the weights are read as stored, no
 *   transposed copy is made), the rest in fp32; the gradients are fp32 for
 *   both. Nothing in the call allocates or waits on the host: it can be
 *   captured in a CUDA graph. Every gradient element is an fp32 sum in a fixed
 *   order (no atomics; the fp32 router weight gradient adds row-chunk partial
 *   sums in chunk order): results are deterministic. A pair with an expert id outside [0, E) contributes
 *   nothing and sets MOE_DEVERR_BAD_EXPERT_ID in the workspace header.
 *   Workspace: moe_backward_workspace_size bytes (its header as for
 *   moe_forward, zeroed by moe_workspace_init). Async on `stream`. */
moe_status moe_backward_workspace_size(const moe_problem *p, size_t *bytes);
moe_status moe_backward(const moe_problem *p, const moe_weights *w, const void *x, const void *dout,
                        const int64_t *selected_experts, moe_grads *g, void *ws, size_t ws_bytes,
                        moe_stream_t stream);

/* Static description of a status code. */
const char *moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* STM_MOE_H */
