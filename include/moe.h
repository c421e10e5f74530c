/*
 * moe.h -- C ABI of a GShard Mixture-of-Experts layer on B200 (sm_100a): the layer on one GPU,
 * forward and backward, and its expert-parallel forward over G GPUs (moe_ep_*).
 *
 * The layer (sources: "GShard: Scaling Giant Neural Networks with Conditional
 * Computation", section "Mixture-of-Experts Implementation" and its "Expert
 * Capacity" paragraph; "GShard: Scaling Giant Models with Conditional
 * Computation and Automatic Sharding", paper-note summary paragraph; "GShard
 * (Expert Parallelism)", "In plain words"):
 *
 *   logits  l = x . W_g (+ b)                         fp32, [S, E]
 *   p       = Softmax(l);  lse = logsumexp(l)          per token
 *   e_0..e_{k-1} = the k largest logits, ties to the lower expert index
 *   g_r     = p[e_r] / sum_{r'} p[e_r']                "softmax-normalised top-k weights"
 *   C       = ceil(capacity_factor * k * S / E)        expert capacity
 *   slots   : rank-major -- all first choices in token order, then all second
 *             choices, ...; an assignment at position >= C of its expert is
 *             dropped (contributes zero, no renormalisation)
 *   xbuf[e, slot] = x[t]                               dispatch (on-device all-to-all)
 *   ybuf[e, :n_e] = relu(xbuf[e, :n_e] W1[e]) W2[e]    expert feed-forward networks
 *   y[t]    = sum_{r kept} g_r ybuf[e_r, slot_r]        combine (second all-to-all)
 *   l_aux   = E * sum_j f_j P_j,  z = mean_t lse_t^2   auxiliary losses
 *
 * with f_j = fraction of tokens whose first choice is j (before capacity) and
 * P_j = mean_t p[t, j].
 *
 * Conventions for every entry point:
 *  - Every pointer argument named *_dev or documented "device" is a CUDA device
 *    pointer on the current device, 16-byte aligned.  Host pointers are named so.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    All work is enqueued asynchronously on it unless stated otherwise.
 *  - Errors are returned as moe_status; nothing aborts or throws across the ABI.
 *    An asynchronous device fault or a device-side wait that timed out surfaces
 *    on the next synchronising call (moe_aux_loss, moe_check) as MOE_ERR_CUDA or
 *    MOE_ERR_TIMEOUT.
 *  - A handle may be used by one host thread / one stream at a time.
 */
#ifndef GSHARD_MOE_H
#define GSHARD_MOE_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* a null, misaligned or out-of-range argument */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the library handles (e.g. E > 256) */
  MOE_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed, or a device fault */
  MOE_ERR_OOM = 4,           /* device workspace allocation failed */
  MOE_ERR_STATE = 5,         /* call out of order (e.g. aux loss before any forward) */
  MOE_ERR_TIMEOUT = 6        /* a device-side bounded wait gave up */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef struct moe_layer* moe_handle;

/* Stage indices of moe_get_stage_times. */
enum { MOE_STAGE_ROUTER = 0, MOE_STAGE_SCAN = 1, MOE_STAGE_DISPATCH = 2, MOE_STAGE_FFN1 = 3,
       MOE_STAGE_FFN2 = 4, MOE_STAGE_COMBINE = 5, MOE_NUM_STAGES = 6 };

/*
 * moe_create -- build a layer handle and allocate its device workspace.
 *
 * S_max            largest token count a forward will be given (1 .. 2^30).  The
 *                  expert buffers' rows, E * round256(min(C(S_max), S_max)), and
 *                  S_max * k must stay below 2^31 (32-bit row indices and TMA
 *                  coordinates); larger sizes return MOE_ERR_UNSUPPORTED.
 * M, H             model and expert-hidden widths; multiples of 64.
 * E, k             number of experts and choices per token, 1 <= k <= E <= 256.
 * capacity_factor  > 0 and finite; C = ceil(capacity_factor * k * S / E) per forward.
 * act              dtype of x, W1, W2 and y (MOE_F32 or MOE_BF16).  Gating is fp32.
 * Wg_dev           [M, E] fp32 row-major gate weights (E contiguous).
 * gate_bias_dev    [E] fp32 added to the logits before the softmax, or NULL.
 * W1_dev           [E, M, H] act, row-major (H contiguous): first expert layer.
 * W2_dev           [E, H, M] act, row-major (M contiguous): second expert layer.
 *
 * Ownership: the weights and bias are BORROWED -- the caller keeps them alive
 * and unchanged until moe_destroy.  The handle owns its workspace (per-expert
 * buffers [E, min(C(S_max), S_max), M|H], routing tables and loss partials),
 * allocated here with one cudaMalloc; no later call allocates device memory
 * except moe_enable_backward.
 * Must be called with the target device current.  On error *out is NULL.
 */
MOE_API moe_status moe_create(moe_handle* out, int64_t S_max, int64_t M, int64_t H, int32_t E, int32_t k,
                      double capacity_factor, moe_dtype act, const float* Wg_dev,
                      const float* gate_bias_dev, const void* W1_dev, const void* W2_dev);

/*
 * moe_forward -- one layer forward of S tokens (0 <= S <= S_max), enqueued on `stream`.
 *
 * x_dev  [S, M] act, row-major (read only).     y_dev  [S, M] act, fully overwritten.
 * A token whose k assignments were all dropped gets y = 0.  S = 0 enqueues no
 * kernel and sets l_aux = z = 0.  No host synchronisation, no allocation.
 * Top-1 routing (k = 1, bf16) on a handle without moe_enable_backward: the combine is
 * fused into the second expert GEMM, whose epilogue stores g * row straight into the
 * token's row of y (the expert-output buffer is not written and no combine kernel runs).
 */
MOE_API moe_status moe_forward(moe_handle h, int64_t S, const void* x_dev, void* y_dev, void* stream);

/*
 * moe_forward_host -- the same forward from and to HOST memory: copies x_host
 * ([S, M] act) into a device staging buffer of the handle, runs the forward and
 * copies y back into y_host ([S, M] act).
 *
 * The three steps run on the handle's own copy-in, compute and copy-out streams
 * with two staging slots, so back-to-back calls overlap: call i+1's input copy
 * runs during call i's compute, and call i's output copy during call i+1's.
 * Ordering: `stream` is made to wait for this call's copy back of y (synchronise
 * `stream` before reading y_host).  A call that follows another kind of call on
 * the handle first waits for the work already enqueued on `stream`; a call that
 * follows a moe_forward_host does not, so it must not depend on device work the
 * caller enqueued on `stream` in between (its input is host memory).  x_host and
 * y_host must stay valid, and x_host unchanged, until `stream` passes this call.
 * Page-locked (pinned) buffers make the copies asynchronous.
 */
MOE_API moe_status moe_forward_host(moe_handle h, int64_t S, const void* x_host, void* y_host, void* stream);

/*
 * moe_aux_loss -- the auxiliary losses of the last forward, to host floats.
 * l_aux = E * sum_j f_j P_j ("N * sum_j f_j * P_j", paper-note summary, N read
 * as E); z = mean_t logsumexp(l_t)^2.  The caller applies loss weights.
 * Synchronises `stream`; returns MOE_ERR_STATE before the first forward and
 * reports pending device errors (MOE_ERR_CUDA / MOE_ERR_TIMEOUT).
 */
MOE_API moe_status moe_aux_loss(moe_handle h, float* l_aux_host, float* z_loss_host, void* stream);

/* moe_destroy -- free the workspace (synchronises the device).  NULL is accepted. */
MOE_API moe_status moe_destroy(moe_handle h);

/*
 * moe_check -- synchronise `stream` and report a pending device error from any
 * earlier call on this handle (MOE_ERR_TIMEOUT, MOE_ERR_CUDA), clearing it.
 */
MOE_API moe_status moe_check(moe_handle h, void* stream);

/* ---- inspection (device-to-device copies on `stream`, valid after a forward) ---- */

/* logits_dev [S, E] fp32: the logits the routing used (bias included). */
MOE_API moe_status moe_get_logits(moe_handle h, float* logits_dev, void* stream);

/*
 * Routing of the last forward / route call: eidx_dev [S, k] int32 expert ids
 * (best first), gate_dev [S, k] fp32 normalised gates, slot_dev [S, k] int32
 * slot within the expert or -1 if dropped, cnt_dev [E] int32 demand per expert
 * before capacity.  Any pointer may be NULL to skip it.
 */
MOE_API moe_status moe_get_routing(moe_handle h, int32_t* eidx_dev, float* gate_dev, int32_t* slot_dev,
                           int32_t* cnt_dev, void* stream);

/*
 * moe_route_from_logits -- run only the routing steps (softmax, top-k, gates,
 * loss partials, capacity scan, slot assignment) on given fp32 logits
 * [S, E] (as they enter the softmax, bias included).  Results are read with
 * moe_get_routing / moe_aux_loss.  Expert buffers are not touched.
 */
MOE_API moe_status moe_route_from_logits(moe_handle h, int64_t S, const float* logits_dev, void* stream);

/* Buffers of moe_get_expert_rows. */
enum { MOE_BUF_X = 0,   /* xbuf [E, Cbuf, M] act: the dispatched token rows */
       MOE_BUF_H = 1,   /* hbuf [E, Cbuf, H] act: relu(xbuf W1[e]) */
       MOE_BUF_Y = 2 }; /* ybuf [E, Cbuf, M] act: hbuf W2[e] */

/*
 * moe_get_expert_rows -- copy rows 0 .. nrows-1 of expert e's slots in one of the
 * per-expert buffers of the last moe_forward (which = MOE_BUF_X, MOE_BUF_H or
 * MOE_BUF_Y) to dst_dev, a device buffer of nrows rows of M (or H for MOE_BUF_H)
 * act elements.  Row i is the assignment the capacity scan gave slot i of expert
 * e; only rows below n_e = min(cnt[e], C) hold data.  0 <= nrows <= the handle's
 * rows per expert (min(C(S_max), S_max) rounded up to 256).  Device-to-device copy
 * on `stream`.  Returns MOE_ERR_STATE unless the last routing call was a moe_forward,
 * and for MOE_BUF_Y after a forward whose combine was fused (top-1 inference).
 */
MOE_API moe_status moe_get_expert_rows(moe_handle h, int32_t which, int32_t e, int64_t nrows,
                                       void* dst_dev, void* stream);

/* Capacity C this handle uses for S tokens (host arithmetic, no device work). */
MOE_API moe_status moe_get_capacity(moe_handle h, int64_t S, int64_t* C_out);

/*
 * Per-stage timing.  With profiling on, moe_forward records CUDA events on its
 * stream between its kernels; moe_get_stage_times synchronises and writes the
 * last forward's per-stage milliseconds (MOE_NUM_STAGES values, order of the
 * MOE_STAGE_* enum) to ms_host.
 */
MOE_API moe_status moe_set_profiling(moe_handle h, int32_t enable);
MOE_API moe_status moe_get_stage_times(moe_handle h, float* ms_host, int32_t n);

/* Flags of moe_set_routing_flags. */
enum { MOE_ROUTE_REROUTE = 1 };

/*
 * moe_set_routing_flags -- options of the following forward and route calls (default 0:
 * a choice over capacity is dropped).
 * MOE_ROUTE_REROUTE: a dropped choice gets one second chance at an alternative expert
 * ("GShard: Scaling Giant Neural Networks with Conditional Computation", "Expert
 * Capacity": overflow tokens are dropped or routed to alternative experts; the rule is
 * this library's reading).  After the rank-major capacity pass, the token's j-th
 * dropped choice (in choice-rank order) is offered its (k+j)-th ranked expert (largest
 * logit among those it neither chose nor was offered, ties to the lower index).  Offers
 * are taken in the capacity pass's order -- choice rank, then token -- into the room
 * the pass left (C minus its kept rows), each accepted offer taking the next free slot;
 * an offer that finds no room stays dropped.  A rerouted choice keeps its gate weight.
 * moe_get_routing then reports the final slot (at the serving expert) and
 * moe_get_serving_experts the serving expert.  A forward with this flag launches 8
 * kernels.  moe_backward of a rerouted forward differentiates that forward: a rerouted
 * choice's rows are at the serving expert, and its gate gradient goes to the expert it
 * chose (its weight g_r is that expert's normalised gate).
 * Returns MOE_ERR_INVALID_ARG for unknown bits.
 */
MOE_API moe_status moe_set_routing_flags(moe_handle h, uint32_t flags);

/*
 * moe_get_serving_experts -- dest_dev [S, k] int32: the expert that serves each choice
 * of the last forward / route call (the chosen expert unless the choice was rerouted;
 * for a dropped choice, the chosen one).  Device copy on `stream`.
 */
MOE_API moe_status moe_get_serving_experts(moe_handle h, int32_t* dest_dev, void* stream);

/* Number of kernels one moe_forward of S tokens launches. */
MOE_API int32_t moe_kernels_per_forward(moe_handle h, int64_t S);

/*
 * moe_selftest_wait_timeout -- launch a kernel whose bounded wait is made to run
 * out (it waits for a device flag that nothing sets, with a limit of
 * limit_us microseconds) and return what the host reads back: MOE_ERR_TIMEOUT
 * when the bound works.  Leaves the context usable.  Synchronises `stream`.
 */
MOE_API moe_status moe_selftest_wait_timeout(int32_t limit_us, void* stream);

/*
 * moe_assign_slots_noalloc -- the capacity slot assignment, with no device allocation.
 * (The pages have no counterpart: this is an interface for callers of this library.)
 *
 * For callers that cannot call cudaMalloc.  Examples: a serving process whose
 * memory pool already holds nearly all of HBM, or a runtime where every device
 * allocation must go through its own allocator.  It applies the layer's
 * capacity rule to expert ids the caller already has; the caller passes all
 * inputs and outputs.
 *
 * S tokens (>= 0), E experts (1..256), k choices (1..min(E, 8)), capacity C (>= 0).
 * eidx_dev  [S, k] int32 expert ids, best choice first (input).
 * slot_dev  [S, k] int32 output: for r = 0..k-1 and tokens in order, an
 *           assignment takes the next free slot of its expert while fewer than C
 *           are taken, else -1 (dropped); ids outside [0, E) get -1.
 * cnt_dev   [E] int32 output: assignments per expert before capacity.
 *
 * Scratch lives in one fixed 8 MiB device array inside the library, which
 * every GPU that loads the library holds until the process exits.  The call
 * needs round256(4*S*k) + 2*round256(4*k*ceil(S/64)*E) bytes of it and
 * returns MOE_ERR_UNSUPPORTED, with no device work, when that exceeds 8 MiB.
 * The first call on a device looks up the array's device address and the
 * device's SM count (with that device current) and caches them; make that
 * first call before any stream capture.  The cache does not survive
 * cudaDeviceReset: after a reset, do not call this entry point again in the
 * same process.  Every call shares the array and leaves its contents behind, so
 * calls whose work overlaps on the GPU (other streams, other host threads)
 * race.  Enqueued on `stream`; no host synchronisation.
 */
MOE_API moe_status moe_assign_slots_noalloc(int64_t S, int32_t E, int32_t k, int64_t C,
                                            const int32_t* eidx_dev, int32_t* slot_dev,
                                            int32_t* cnt_dev, void* stream);

/* ---- expert parallelism: one layer over G ranks, one GPU each ------------------ */

/*
 * The layer with its experts spread over G ranks ("GShard (Expert Parallelism)", "In
 * plain words": each device hosts some experts; tokens go to them by an all-to-all and
 * come back by a second one; the "WideEP" claim: 256 experts on 8 GPUs, 32 per GPU,
 * results returned by a second all-to-all).  Rank g holds a contiguous block of the
 * batch's tokens (ranks in order) and the experts [g*E/G, (g+1)*E/G) (E % G == 0);
 * every rank holds the whole gate W_g.
 *
 * Capacity and slots keep their one-device meaning over the whole batch:
 * C = ceil(capacity_factor * k * S_total / E), and slots are rank-major over the
 * concatenated tokens.  The result -- expert ids, slots, drops, outputs, losses -- is
 * the single-GPU layer's on the concatenated batch.
 *
 * The library computes; the caller moves bytes between ranks (NCCL, or any transport)
 * at three points of one forward:
 *   1. moe_ep_route(x) -> stats_dev       [ALL-GATHER the stats of every rank, to host]
 *   2. moe_ep_dispatch(stats_all) -> sendbuf, send_rows[G], recv_rows[G]
 *                                         [ALL-TO-ALL: sendbuf -> recvbuf, row counts given]
 *   3. moe_ep_experts(recvbuf)            [ALL-TO-ALL back: recvbuf -> sendbuf, counts reversed]
 *   4. moe_ep_combine(sendbuf) -> y;  moe_ep_aux_loss
 * Rows are M act elements.  Rank g's send buffer holds, for each destination rank in
 * order, the rows of its kept choices ordered by expert, then choice rank, then token;
 * the receiver gets each source's rows in that order, source after source, and
 * moe_ep_experts writes each expert output over the row it came from, so the second
 * exchange is the first one reversed.
 *
 * Two phases (moe_ep_set_phases, bf16): the exchanges split in two, so that they can
 * overlap the expert GEMMs -- send phase 1 while the experts compute phase 0, return
 * phase 0 while they compute phase 1.  Each expert's slots are split at
 * split_e = 256 * floor((n_e + 256) / 512) (n_e its kept rows over the batch): slots
 * below it travel in phase 0, the rest in phase 1.  Both buffers hold all phase-0 rows
 * first, then all phase-1 rows, each phase ordered as above, and the row counts per
 * peer come per phase ([2][G], phase-major).  One forward with overlap:
 *   moe_ep_route; all-gather; moe_ep_dispatch -> send_rows[2][G], recv_rows[2][G]
 *   exchange phase 0;  [exchange phase 1 | moe_ep_experts_phase(0)]
 *   [return phase 0 | moe_ep_experts_phase(1)];  return phase 1;  moe_ep_combine
 * Every GEMM tile lies within one phase, so rows, slots and outputs are bit for bit
 * those of the one-phase forward.
 *
 * Over peer memory (moe_ep_set_peers): when every rank's receive buffer is mapped on
 * every GPU (CUDA IPC, symmetric memory), moe_ep_dispatch_to_peers packs each kept row
 * straight into its owner's receive buffer at the row the all-to-all would have put it
 * (stores over NVLink, no send buffer), and moe_ep_combine_from_peers reads each expert
 * output from the owner's buffer, where moe_ep_experts wrote it.  Both exchanges become
 * part of those kernels.  The caller orders the ranks:
 *   moe_ep_route; all-gather; moe_ep_dispatch_to_peers   [every rank done, writes visible]
 *   moe_ep_experts(own receive buffer)                   [every rank done]
 *   moe_ep_combine_from_peers                            [every rank done before the next
 *                                                         forward's dispatch]
 * e.g. a stream synchronise and a barrier of the ranks at each bracket.  One phase only.
 */
typedef struct moe_ep_layer* moe_ep_handle;

/* Doubles per rank in the stats vector: k*E counts (rank-r demand of expert e at
 * [r*E + e]), E probability sums, the sum of lse^2, the rank's token count. */
MOE_API int32_t moe_ep_stats_len(int32_t E, int32_t k);

/*
 * moe_ep_plan -- the exchange plan of rank g (host arithmetic, no device work; the
 * entry points below use the same).  counts_host [G][k][E]: rank q's rank-r demand of
 * expert e; S_host [G]: tokens per rank.  Outputs: C_out (capacity of the batch),
 * send_rows_host [G] rows rank g sends to each rank, recv_rows_host [G] rows it
 * receives from each, and (optional, may be NULL) base_host [G][k][E] -- the first
 * global slot of each (rank q, choice rank r, expert e) run -- and kept_host [G][k][E],
 * the kept rows of each run.  MOE_ERR_INVALID_ARG for negative or inconsistent counts
 * (each rank's rank-r counts must sum to its token count).
 */
MOE_API moe_status moe_ep_plan(int32_t G, int32_t g, int32_t E, int32_t k, double capacity_factor,
                               const int64_t* counts_host, const int64_t* S_host, int64_t* C_out,
                               int64_t* send_rows_host, int64_t* recv_rows_host, int64_t* base_host,
                               int64_t* kept_host);

/*
 * moe_ep_phase_plan -- per-phase row counts of rank g (host arithmetic, as moe_ep_plan):
 * send_rows_host / recv_rows_host [phases][G] (phase-major) and, optional, split_host [E]
 * (the first phase-1 slot of each expert; n_e with one phase).  phases: 1 or 2, else
 * MOE_ERR_INVALID_ARG; invalid counts as moe_ep_plan.
 */
MOE_API moe_status moe_ep_phase_plan(int32_t G, int32_t g, int32_t E, int32_t k, double capacity_factor,
                                     const int64_t* counts_host, const int64_t* S_host, int32_t phases,
                                     int64_t* send_rows_host, int64_t* recv_rows_host, int64_t* split_host);

/*
 * moe_ep_create -- rank g's handle.  S_max: most tokens this rank routes in a forward;
 * S_total_max: most tokens of a batch over all ranks (sizes the expert buffers).
 * Wg_dev [M, E] and gate_bias_dev [E] (or NULL) as in moe_create; W1_local_dev
 * [E/G, M, H] and W2_local_dev [E/G, H, M]: this rank's experts.  Borrowed, as in
 * moe_create.  One cudaMalloc here; the forward allocates nothing.
 */
MOE_API moe_status moe_ep_create(moe_ep_handle* out, int32_t G, int32_t g, int64_t S_max,
                                 int64_t S_total_max, int64_t M, int64_t H, int32_t E, int32_t k,
                                 double capacity_factor, moe_dtype act, const float* Wg_dev,
                                 const float* gate_bias_dev, const void* W1_local_dev,
                                 const void* W2_local_dev);
MOE_API moe_status moe_ep_destroy(moe_ep_handle h);

/* Rows the caller's buffers need: send buffer S_max*k, receive buffer E/G * min(C, S_total_max). */
MOE_API moe_status moe_ep_buffer_rows(moe_ep_handle h, int64_t* send_rows_max, int64_t* recv_rows_max);

/* Exchanges in 1 (default) or 2 phases for the forwards that follow (see above).  Two
 * phases need bf16 activations (MOE_ERR_UNSUPPORTED otherwise); a forward in progress
 * must start again from moe_ep_dispatch. */
MOE_API moe_status moe_ep_set_phases(moe_ep_handle h, int32_t phases);

/* Step 1: router and the rank's own scan on S tokens (x_dev [S, M] act); writes the
 * rank's stats (moe_ep_stats_len doubles, 8-byte aligned device memory) on `stream`. */
MOE_API moe_status moe_ep_route(moe_ep_handle h, int64_t S, const void* x_dev, double* stats_dev,
                                void* stream);

/* Step 2: stats_all_host [G][moe_ep_stats_len] (every rank's stats, rank order) ->
 * plan, send_rows_host / recv_rows_host [phases][G], and the kept rows of x_dev (the
 * same x as step 1) packed into sendbuf_dev (>= sum(send_rows) rows).  Host arithmetic,
 * then one table upload and one kernel on `stream`. */
MOE_API moe_status moe_ep_dispatch(moe_ep_handle h, const double* stats_all_host, const void* x_dev,
                                   void* sendbuf_dev, int64_t* send_rows_host, int64_t* recv_rows_host,
                                   void* stream);

/* Step 3: the received rows (recvbuf_dev, sum(recv_rows) rows) into the local experts'
 * slots, both expert GEMMs, and each expert output written over its received row
 * (every phase, in order). */
MOE_API moe_status moe_ep_experts(moe_ep_handle h, void* recvbuf_dev, void* stream);

/* Step 3 for one phase (0 <= phase < phases): the phase's received rows (its region of
 * recvbuf_dev: after the sum of the earlier phases' recv_rows) through the experts, the
 * outputs written over them.  Needs only that phase's rows to have arrived.
 * MOE_ERR_INVALID_ARG for a phase out of range. */
MOE_API moe_status moe_ep_experts_phase(moe_ep_handle h, void* recvbuf_dev, int32_t phase, void* stream);

/* Step 4: y_dev [S, M] act from the returned rows in sendbuf_dev (fully overwritten;
 * a token whose choices were all dropped gets 0). */
MOE_API moe_status moe_ep_combine(moe_ep_handle h, const void* sendbuf_dev, void* y_dev, void* stream);

/* The receive buffer of every rank, as this GPU addresses it (recv_bufs_host [G] device
 * pointers, 16-byte aligned, each of moe_ep_buffer_rows' receive rows; entry g is this
 * rank's own), for the peer-memory forms below.  NULL forgets them.  Host only. */
MOE_API moe_status moe_ep_set_peers(moe_ep_handle h, const void* const* recv_bufs_host);

/* Step 2 over peer memory: as moe_ep_dispatch, with each kept row stored into its
 * owner's receive buffer instead of a send buffer.  MOE_ERR_STATE without peers or with
 * two phases. */
MOE_API moe_status moe_ep_dispatch_to_peers(moe_ep_handle h, const double* stats_all_host, const void* x_dev,
                                            int64_t* send_rows_host, int64_t* recv_rows_host, void* stream);

/* Step 4 over peer memory: y_dev [S, M] act, each kept choice's expert output read from
 * its owner's receive buffer (same sum and rounding as moe_ep_combine).  MOE_ERR_STATE
 * unless the last dispatch was moe_ep_dispatch_to_peers (and moe_ep_combine after one). */
MOE_API moe_status moe_ep_combine_from_peers(moe_ep_handle h, void* y_dev, void* stream);

/* l_aux and z of the whole batch, from the stats given to the last moe_ep_dispatch (host). */
MOE_API moe_status moe_ep_aux_loss(moe_ep_handle h, float* l_aux_host, float* z_loss_host);

/* This rank's routing of the last forward (device copies; any pointer may be NULL):
 * eidx / gate [S, k], slot [S, k] global slot or -1, spos [S, k] send-buffer row or -1
 * (slot and spos need step 2), logits [S, E]. */
MOE_API moe_status moe_ep_get_routing(moe_ep_handle h, int32_t* eidx_dev, float* gate_dev,
                                      int32_t* slot_dev, int32_t* spos_dev, float* logits_dev,
                                      void* stream);

/* Synchronise `stream` and report a pending device error of this handle (as moe_check). */
MOE_API moe_status moe_ep_check(moe_ep_handle h, void* stream);

/* ---- backward (training) ---------------------------------------------------- */

/*
 * moe_enable_backward -- allocate the workspace moe_backward needs (once per
 * handle; a second call does nothing).  Inference-only handles never pay for
 * these buffers:
 *   dY  [E, Cbuf, M] act  (gradient of the expert outputs; reused for dX_e)
 *   dP  [E, Cbuf, H] act  (gradient of the first layer's pre-activation)
 *   dl  [S_max, E] fp32 (logit gradient), dgate [S_max, k] fp32, and the
 *   split-K partials of the gate-weight gradient;
 *   bf16 only: the ReLU mask bits [H/32, E*Cbuf] uint32, one bit per element
 *   of the first layer's output (set when the stored bf16 value is > 0).
 * Training mode: every bf16 forward after this call also stores those bits
 * (1/16 of the bytes of h), and moe_backward's dP step reads them instead of
 * re-reading h.  A backward of a forward that ran before this call re-reads h;
 * both give bitwise-equal gradients.  Once any forward of the handle has been
 * captured into a CUDA graph without the bits (captured before this call), the
 * backward always re-reads h, since replays of that graph are invisible to the
 * host: capture training graphs after this call to keep the faster path.
 * Synchronous (cudaMalloc); call it outside stream capture.
 */
MOE_API moe_status moe_enable_backward(moe_handle h);

/*
 * moe_backward -- gradients of
 *     L = <dy, y> + a_aux * l_aux + a_z * z
 * ("GShard: Scaling Giant Neural Networks with Conditional Computation",
 * "Training Methodology": the auxiliary loss joins the task loss with a small
 * weight, here a_aux, and only experts that received tokens get a gradient)
 * for the last moe_forward of this handle (same S, same x; the forward's saved
 * routing and expert buffers are read, not changed, so moe_backward may run
 * more than once per forward).  Enqueued on `stream`, no host synchronisation.
 *
 * The routing -- expert choices, slots, drops -- and the first-choice
 * fractions f_j are piecewise constant and carry no gradient; every other step
 * is differentiated exactly:
 *   combine      dY_e[slot_r] = g_r dy[t],  dgate_r = <dy[t], y_e[slot_r]>
 *                (both zero for a dropped assignment)
 *   expert FFN   dW2[e] = relu(P_e)^T dY_e,  dP_e = (dY_e W2[e]^T) * [h_e > 0],
 *                dW1[e] = X_e^T dP_e,  dx[t] += sum_{r kept} (dP_e W1[e]^T)[slot_r]
 *   gates        dl[t, e_r] += g_r (dgate_r - sum_r' g_r' dgate_r')
 *   l_aux        dl[t] += a_aux E/S p_t (f - <p_t, f>)
 *   z-loss       dl[t] += a_z 2/S lse_t p_t
 *   gate GEMM    dx += dl W_g^T,  dW_g = x^T dl,  dbias = sum_t dl
 *
 * x_dev     [S, M] act: the forward's input (unchanged since).
 * dy_dev    [S, M] act: dL/dy.
 * dx_dev    [S, M] act, overwritten.
 * dWg_dev   [M, E] fp32, overwritten.      dbias_dev [E] fp32 overwritten, or NULL.
 * dW1_dev   [E, M, H] act, overwritten.    dW2_dev   [E, H, M] act, overwritten
 *           (experts that kept no token get zeros, or are skipped: see
 *           moe_set_backward_flags).
 * Returns MOE_ERR_STATE unless moe_enable_backward succeeded and the last call
 * that routed on this handle was a moe_forward of S tokens that kept its expert outputs
 * (a top-1 forward before moe_enable_backward fuses the combine and keeps none).  Every output
 * pointer must be 16-byte aligned and must not alias the inputs.
 */
MOE_API moe_status moe_backward(moe_handle h, int64_t S, const void* x_dev, const void* dy_dev,
                                float a_aux, float a_z, void* dx_dev, float* dWg_dev,
                                float* dbias_dev, void* dW1_dev, void* dW2_dev, void* stream);

/* Number of kernels one moe_backward of S tokens launches. */
MOE_API int32_t moe_kernels_per_backward(moe_handle h, int64_t S);

/* Flags of moe_set_backward_flags. */
enum { MOE_BWD_SKIP_EMPTY_EXPERTS = 1 };

/*
 * moe_set_backward_flags -- options of the following moe_backward calls (default 0).
 * MOE_BWD_SKIP_EMPTY_EXPERTS: dW1[e] and dW2[e] of an expert that kept no token in
 * the forward are not written (the caller's buffer keeps what it held), instead of
 * being set to zero.  Only the experts a batch activated get a gradient ("GShard:
 * Scaling Giant Neural Networks with Conditional Computation", "Training
 * Methodology", "Gradient Synchronization"); a caller that applies sparse updates
 * reads which experts those were from moe_get_routing's cnt (cnt[e] > 0).
 * Returns MOE_ERR_INVALID_ARG for unknown bits.
 */
MOE_API moe_status moe_set_backward_flags(moe_handle h, uint32_t flags);

/* Stage indices of moe_get_backward_stage_times. */
enum { MOE_BSTAGE_GATE = 0,     /* combine + gate backward: dY, dgate, dl */
       MOE_BSTAGE_PAD = 1,      /* clearing the 64-row padding of the reduced buffers */
       MOE_BSTAGE_DW2 = 2,      /* dW2 = h^T dY */
       MOE_BSTAGE_DP = 3,       /* dP = (dY W2^T) * [h > 0] */
       MOE_BSTAGE_DW1 = 4,      /* dW1 = X^T dP */
       MOE_BSTAGE_DXE = 5,      /* dX_e = dP W1^T */
       MOE_BSTAGE_DX = 6,       /* dx = gathered dX_e + dl W_g^T */
       MOE_BSTAGE_DWG = 7,      /* dW_g = x^T dl, dbias (split-K + ordered sum) */
       MOE_NUM_BWD_STAGES = 8 };

/*
 * With profiling on (moe_set_profiling), moe_backward records CUDA events on its
 * stream between its stages; this synchronises and writes the last backward's
 * per-stage milliseconds (MOE_NUM_BWD_STAGES values) to ms_host.
 */
MOE_API moe_status moe_get_backward_stage_times(moe_handle h, float* ms_host, int32_t n);

/* Name of a MOE_BSTAGE_* index ("gate_bwd", "dW2", ...), or "?" */
MOE_API const char* moe_backward_stage_name(int32_t stage);

/* Static description of a status code (never NULL). */
MOE_API const char* moe_status_string(moe_status s);

/* Name of a MOE_STAGE_* index ("router", "scan", ...), or "?" */
MOE_API const char* moe_stage_name(int32_t stage);

#ifdef __cplusplus
}
#endif

#endif /* GSHARD_MOE_H */
