/*
 * ep.h -- C ABI of libep_b200: MoE expert-parallel token dispatch and
 * combine on one B200 (sm_100a), with the EP world of R ranks held as R
 * logical partitions of one HBM.
 *
 * The calls follow the statement of the problem on these pages:
 *   - NCCL EP paper page (arXiv 2603.13606): long-lived groups and
 *     per-forward-pass handles (Table II, Fig. 2); LL mode with a 3D
 *     expert-major output and HT mode with a 2D concatenated output plus
 *     per-expert token counts (Table III, Figs. 3-4); the tensor roles
 *     TOKENS, TOPK_IDX, TOPK_WEIGHTS and FP8 quantization scales (Table IV);
 *     a dispatch call that takes the tokens, the top-k ids and weights and
 *     the handle, and returns the received rows, their expert ids and
 *     their weights (Table V); combine collects each token's expert results
 *     and sums them back into that token's row (Table II); routing state
 *     shared by the forward and backward passes (Fig. 5).
 *   - MoonEP news article (opensourceforu.com): a GPU planner that
 *     replicates hot experts online so that every rank receives a
 *     predictable load (para. 3), placement straight into expert-grouped rank
 *     positions with static shapes and no per-layer host sync (para. 4), at
 *     most E/R prefetch slots per rank in training, and a reduce buffer for
 *     the gradients of duplicated experts (para. 5).
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses owned by the caller;
 *     the library never frees them and keeps none of them after the call
 *     returns. Token rows (x, recv_x, expert outputs, gradients) must be
 *     16-byte aligned; every other pointer naturally aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call except ep_get_* is asynchronous and stream-ordered:
 *     it enqueues kernels and returns without a host synchronisation.
 *   - Arguments the host can check are checked before anything is launched;
 *     a failed check returns an error status and launches nothing.
 *   - Conditions only the device can see (a bad or repeated expert id, LL
 *     capacity overflow, a balanced plan that runs out of slots) never trap
 *     and never hang: the offending pairs are skipped (or, for the plan,
 *     kept on the owner rank) and a bit is set in the handle's status word,
 *     read by ep_get_status.
 *   - A handle is not thread-safe; calls on one handle must be ordered by
 *     the caller (one stream, or explicit events).
 *   - Kernels are launched with programmatic dependent launch. The routing
 *     and router kernels let the next kernel of the stream start early, and
 *     the dispatch kernels read their token rows x before waiting for the
 *     kernels ahead of them. So a kernel of the caller's that writes x and is
 *     itself launched with programmatic dependent launch must write x before
 *     it triggers its dependents (kernels without that attribute need
 *     nothing).
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ep_status {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1, /* a bad size, a NULL or misaligned pointer */
    EP_ERR_CUDA = 2,        /* a CUDA runtime call or a launch failed */
    EP_ERR_UNSUPPORTED = 3, /* a valid but unsupported combination */
    EP_ERR_NOT_PLANNED = 4, /* a data call before the first ep_plan */
    EP_ERR_NO_MEMORY = 5,   /* workspace allocation failed */
    EP_ERR_TOO_LARGE = 6    /* sizes beyond ep_route_noalloc's fixed scratch */
} ep_status_t;

/* Bits of the device status word (ep_get_status). */
#define EP_FLAG_BAD_EXPERT_ID 0x1 /* an id outside [0, E) other than -1 */
#define EP_FLAG_DUP_EXPERT_ID 0x2 /* a token chose the same expert twice */
#define EP_FLAG_CAPACITY 0x4      /* LL: an expert received more than ll_capacity rows */
#define EP_FLAG_PLAN_SLOTS 0x8    /* balanced plan ran out of replica slots */
#define EP_FLAG_WAIT_TIMEOUT 0x10 /* a kernel's bounded wait for its own copy gave up
                                     (after 2 s); that call's outputs are incomplete */

typedef enum ep_mode { EP_MODE_LL = 0, EP_MODE_HT = 1 } ep_mode_t;

/* Which piece of a handle's routing state ep_get_tensor exposes. */
typedef enum ep_tensor {
    EP_T_DEST_ROW = 0,       /* int32 [T*K]: receive-buffer row of pair (t,k), -1 if none */
    EP_T_EXPERT_COUNTS = 1,  /* int32 [E]: routed pairs per expert */
    EP_T_RECV_COUNTS = 2,    /* int32 [R*(E/R + S)] HT, [E] LL: rows per local slot */
    EP_T_RANK_LOAD = 3,      /* int32 [R]: rows received by each logical rank */
    EP_T_RANK_OFFSET = 4,    /* int32 [R+1]: first row of each rank's region */
    EP_T_REPLICA_EXPERT = 5, /* int32 [R*S]: expert held by replica slot (r,s), -1 empty */
    EP_T_DIRECT_COUNT = 6,   /* int32 [R]: direct-read pieces of each rank (direct_overflow) */
    EP_T_DIRECT_EXPERT = 7,  /* int32 [R*E]: expert of direct piece i of rank r at [r*E+i], -1 unused */
    EP_T_DIRECT_LEN = 8,     /* int32 [R*E]: rows of that piece */
    EP_T_SRC_ROW = 9         /* int32 [rows]: for each receive row that a pair targets, that
                                pair's index t*K+k (the inverse of EP_T_DEST_ROW); rows no
                                pair targets hold unspecified values */
} ep_tensor_t;

/* One EP configuration: fixed for the lifetime of a handle (static shapes,
 * MoonEP article para. 4). T tokens of H hidden values, E experts chosen
 * top-K per token, R logical ranks owning E/R consecutive experts each;
 * token t belongs to source rank t / (T/R) (contiguous blocks). */
typedef struct ep_config {
    int32_t num_tokens;            /* T >= 0 (T = 0 is an empty batch) */
    int32_t hidden;                /* H > 0, multiple of 8 (of 128 with fp8) */
    int32_t num_experts;           /* E in [1, 4096], multiple of R */
    int32_t topk;                  /* K in [1, min(E, 32)] */
    int32_t num_ranks;             /* R >= 1 */
    int32_t mode;                  /* ep_mode_t */
    int32_t ll_capacity;           /* LL: rows per expert (>= 1); ignored in HT */
    int32_t fp8;                   /* 1: dispatch casts to FP8 e4m3 + fp32 scales */
    int32_t balanced;              /* 1: balanced-replica plan (HT only; its tables must
                                      fit one CTA's shared memory: E up to about 1700
                                      with the default E/R slots a rank, about 2200 with
                                      two; beyond it ep_validate_config returns
                                      EP_ERR_UNSUPPORTED) */
    int32_t replica_slots;         /* S in [1, E/R] with balanced; 0 = E/R */
    int64_t grad_elems_per_expert; /* G for ep_reduce_replica_grads; 0 if unused */
    int32_t direct_overflow;       /* 1 (with balanced): inference plan, see ep_plan */
} ep_config_t;

typedef struct ep_handle ep_handle_t;

/* ---- host-only queries (no GPU needed) -------------------------------- */

/* Check a configuration without touching the GPU. */
ep_status_t ep_validate_config(const ep_config_t *cfg);

/* Rows of the receive buffer: T*K in HT (one row per (token, k) pair,
 * NCCL EP Table III "2D"), E*ll_capacity in LL (the 3D expert-major buffer
 * [R][E/R][ll_capacity] flattened, Table III "3D"). */
ep_status_t ep_recv_rows(const ep_config_t *cfg, int64_t *rows);

/* Number of int32 entries of recv_counts: R*(E/R + S) in HT (per rank: its
 * own experts in id order, then its S replica slots; S = 0 without a
 * balanced plan, giving the per-expert counts [E]), E in LL. */
ep_status_t ep_recv_counts_len(const ep_config_t *cfg, int64_t *len);

/* Shape of the receive buffer in elements (NCCL EP Table III): HT *ndim = 2,
 * dims = {rows, H} (rows = T*K, one per (token, k) pair, grouped by expert;
 * "2D with token counts"); LL *ndim = 4, dims = {R, E/R, ll_capacity, H}
 * ("3D expert-major"). An FP8 payload has the same shape in bytes, plus
 * scales [rows, H/128]. dims[i] for i >= *ndim are set to 1. */
ep_status_t ep_output_shape(const ep_config_t *cfg, int64_t dims[4], int32_t *ndim);

/* Device bytes ep_create will allocate for the handle's workspace. */
ep_status_t ep_workspace_bytes(const ep_config_t *cfg, size_t *bytes);

/* Number of kernels one ep_plan launches for this configuration: one for
 * batches of up to 1024 (token, k) pairs (with a balanced plan, when its
 * tables and the batch fit one CTA's shared memory), and for up to 32768
 * pairs, with or without a plan, when the current device can hold the
 * routing cluster (asked of the device; reported as not holdable where there
 * is no GPU), else three. Every other data call launches one kernel. */
ep_status_t ep_plan_kernel_count(const ep_config_t *cfg, int32_t *count);

/* "major.minor.patch" of the library. */
const char *ep_version(void);

/* Human-readable name of a status code. */
const char *ep_status_string(ep_status_t status);

/* ---- group / handle lifetime (NCCL EP Table II, Fig. 2) --------------- */

/* Validate cfg and allocate the handle and all of its device workspace once
 * (routing state, plan tables, status word), on the current CUDA device.
 * No later call allocates. On error *out is NULL. */
ep_status_t ep_create(const ep_config_t *cfg, ep_handle_t **out);

/* Free the handle and its workspace (synchronises the device first).
 * NULL is accepted. */
ep_status_t ep_destroy(ep_handle_t *h);

/* ---- forward ----------------------------------------------------------- */

/* Router top-K, the gating step that feeds ep_plan ("Ultra-Large MoE Models:
 * Open-Source Evolution and Heterogeneous Inference Adaptation", §2.1 top-K
 * routing and §3.1 the fused top-K routing operator). For every token t:
 *   topk_idx[t, 0..K)  the K experts with the largest logits[t, :], in
 *                      descending order of logit, a tie going to the lower id;
 *   topk_w[t, k]       = exp(l_k - l_0) / sum_j exp(l_j - l_0) over the chosen
 *                      logits l_k (= softmax over all E experts, renormalised
 *                      over the K chosen), fp32, summed in k order.
 * logits: device fp32 [T, E] row-major; outputs device int32 / fp32 [T, K].
 * Needs E <= 1024 and K <= min(E, 32), else EP_ERR_INVALID_ARG. Logits must be
 * finite. No handle; stream-ordered, no host sync. */
ep_status_t ep_router_topk(const float *logits, int32_t num_tokens, int32_t num_experts, int32_t topk,
                           int32_t *topk_idx, float *topk_w, void *stream);

/* Routing for one forward pass (NCCL EP Fig. 5: the state it builds is
 * reused by dispatch, combine and both backward calls until the next
 * ep_plan). Clears the status word, then on the device:
 *   counts   cnt[e] = routed pairs (t,k) with topk_idx[t,k] == e;
 *   slots    j(t,k) = earlier routed pairs (t',k') < (t,k) in row-major
 *            order with the same expert (stable, deterministic);
 *   layout   HT: rows grouped by expert id, so rank r's region holds
 *            experts r*E/R .. (r+1)*E/R-1; LL: row e*ll_capacity + j, pairs
 *            with j >= ll_capacity dropped (EP_FLAG_CAPACITY);
 *   plan     with cfg.balanced, the balanced-replica plan: each rank
 *            receives floor or ceil of L/R rows (L = routed pairs), hot
 *            experts spilling into at most S replica slots per rank
 *            (MoonEP article paras. 3 and 5). With cfg.direct_overflow (the
 *            inference plan, MoonEP para. 5: only a few slots per rank, and
 *            rows past them read the owner's weights in place), a rank
 *            with rows to take but no free slot takes them as a direct piece:
 *            its rows are computed with the owner's weights read in place,
 *            and it follows the rank's slots in its region (EP_T_DIRECT_*);
 *            loads are then always floor or ceil of L/R.
 * topk_idx: device int32 [T, K] row-major. -1 marks a masked choice (not
 * routed, no flag); other ids outside [0, E) and repeats within a token are
 * skipped and flagged. */
ep_status_t ep_plan(ep_handle_t *h, const int32_t *topk_idx, void *stream);

/* Dispatch (NCCL EP Table V): for every routed pair (t,k) with row
 * d = dest_row[t,k]:
 *   recv_x[d, :]   = x[t, :]                       (bf16 rows [rows, H]), or
 *   recv_x[d, :]   = e4m3(x[t, b-block] / s_b)     (fp8 rows [rows, H] bytes)
 *   recv_scales[d, b] = s_b = amax_b / 448         (fp32 [rows, H/128])
 *     with amax_b the max |x| of the b-th 128-element block of x[t], fp32
 *     division, round-to-nearest-even, saturation to +-448; an all-zero
 *     block gives s = 0 and codes +0 (NCCL EP Table IV FP8 scales);
 *   recv_w[d]      = topk_w[t,k]       (fp32 [rows]; may be NULL)
 *   recv_expert[d] = topk_idx[t,k]     (int32 [rows]; may be NULL)
 * and recv_counts (int32, ep_recv_counts_len entries; may be NULL) receives
 * the rows per local slot. Rows no pair targets (LL padding) are not
 * written. x: device bf16 [T, H]. topk_idx must be the array given to the
 * last ep_plan (it may be NULL when recv_expert is NULL). recv_scales must
 * be non-NULL iff cfg.fp8. The bf16 payload moves by bulk copies through
 * shared memory; their completion wait is bounded, and a wait that runs out
 * (2 s) sets EP_FLAG_WAIT_TIMEOUT instead of hanging. */
ep_status_t ep_dispatch(ep_handle_t *h, const void *x, const int32_t *topk_idx, const float *topk_w,
                        void *recv_x, float *recv_scales, float *recv_w, int32_t *recv_expert,
                        int32_t *recv_counts, void *stream);

/* Combine (NCCL EP Table II combine row, Table III per-token reduction):
 *   out[t, :] = bf16( fold_k acc = fmaf(topk_w[t,k], y[dest_row[t,k], :], acc) )
 * over k = 0..K-1 in order, acc starting at +0 in fp32, pairs without a row
 * skipped, one round-to-nearest-even at the end.
 * expert_out: device bf16 [rows, H]; topk_w: fp32 [T, K]; out: bf16 [T, H]. */
ep_status_t ep_combine(ep_handle_t *h, const void *expert_out, const float *topk_w, void *out, void *stream);

/* ---- backward (NCCL EP Fig. 5: same routing state, roles swapped) ------ */

/* Gradient of combine w.r.t. the expert outputs, a dispatch-shaped pass:
 *   grad_expert_out[dest_row[t,k], :] = bf16(topk_w[t,k] * grad_out[t, :])
 * (fp32 product, one bf16 rounding). grad_out: bf16 [T, H];
 * grad_expert_out: bf16 [rows, H]; rows without a pair are not written. */
ep_status_t ep_combine_backward(ep_handle_t *h, const void *grad_out, const float *topk_w, void *grad_expert_out,
                                void *stream);

/* Gradient of dispatch w.r.t. x, a combine-shaped pass (unweighted):
 *   grad_x[t, :] = bf16( sum_k grad_recv[dest_row[t,k], :] )
 * fp32 adds in k order from +0. Only bf16 dispatch has a gradient here (an
 * FP8 payload is forward-only). grad_recv: bf16 [rows, H]; grad_x: bf16 [T, H]. */
ep_status_t ep_dispatch_backward(ep_handle_t *h, const void *grad_recv, void *grad_x, void *stream);

/* Replica-gradient reduce (MoonEP article para. 5): for every expert e
 * that has replicas under the current plan,
 *   owner_grad[e, :] += replica_grad[r, s, :] for each slot (r, s) with
 *                       replica_expert[r, s] == e, in ascending (r, s) order,
 * fp32. replica_grad: device fp32 [R, S, G]; owner_grad: fp32 [E, G], updated
 * in place; G = cfg.grad_elems_per_expert. Needs cfg.balanced. */
ep_status_t ep_reduce_replica_grads(ep_handle_t *h, const float *replica_grad, float *owner_grad, void *stream);

/* Replica weight prefetch (MoonEP article paras. 3 and 5: the planner picks
 * redundant experts online and their weights are prefetched into dedicated
 * prefetch slots of the receiving ranks). For every replica slot (r, s) the
 * current plan fills with expert e:
 *   prefetch_slots[r, s, :] = expert_weights[e, :]   (bytes_per_expert bytes)
 * Empty slots are not written. expert_weights: device [E, bytes_per_expert];
 * prefetch_slots: device [R, S, bytes_per_expert]; both 16-byte aligned and
 * bytes_per_expert a positive multiple of 16, with R*S*(bytes_per_expert/8192
 * + 1) at most 2^30 (the copy's 8 KB items are counted in 32 bits), else
 * EP_ERR_INVALID_ARG. Reads the plan on the device: no host sync. Needs
 * cfg.balanced. */
ep_status_t ep_prefetch_replica_weights(ep_handle_t *h, const void *expert_weights, int64_t bytes_per_expert,
                                        void *prefetch_slots, void *stream);

/* ---- inspection (these synchronise the stream) ------------------------- */

/* Wait for `stream`, then copy the plan to host memory: replica_expert
 * [R*S] (-1 = empty slot; may be NULL; nothing is written when the handle
 * has no plan, S = 0) and rank_load [R] (may be NULL). */
ep_status_t ep_get_plan(ep_handle_t *h, int32_t *replica_expert_host, int32_t *rank_load_host, void *stream);

/* Wait for `stream`, then read the device status word (EP_FLAG_* bits set
 * since the last ep_plan). */
ep_status_t ep_get_status(ep_handle_t *h, int32_t *flags, void *stream);

/* Read-only device pointer and element count of one piece of the handle's
 * routing state (valid until the next ep_plan or ep_destroy). */
ep_status_t ep_get_tensor(const ep_handle_t *h, ep_tensor_t which, const void **dptr, int64_t *numel);

/* ---- expert parallelism across GPUs: one rank per GPU ------------------
 *
 * The same path with the R ranks of the EP world on R GPUs (NVLink 5 through
 * NVSwitch), or, for testing, on one GPU with R separate receive buffers. The
 * steps follow the pages' statement of the exchange:
 *   - counts:  every rank counts its own routed pairs per expert
 *              (ep_plan_local_counts); the caller all-gathers the R count rows
 *              (R*E int32, e.g. one NCCL all-gather) into world_counts;
 *   - plan:    every rank derives the same global layout from world_counts,
 *              and the global row of each of its own pairs (ep_plan_world);
 *              the stable order of an expert's rows is (source rank, t, k),
 *              so rank r's pairs of expert e follow the pairs of ranks < r;
 *   - send:    rows go straight into the owning rank's receive buffer
 *              (ep_dispatch_peers: NCCL EP Table II / Fig. 2, the send half of
 *              the staged mode; MoonEP article para. 4, placement straight into
 *              expert-grouped remote positions with no staging copy);
 *   - signal / wait: per-source completion flags (ep_signal_peers,
 *              ep_wait_peers: the receive half of the staged mode);
 *   - combine: each rank reads its tokens' K rows from the ranks holding them
 *              and reduces them locally (ep_combine_peers: NCCL EP Table III,
 *              per-token reduction at the receiver);
 *   - backward: the same two movements with roles swapped, and the replica
 *              gradients reduced into their owners across ranks.
 * Remote rows move with plain 16-byte stores and loads in the library's own
 * kernels (no bulk copy or cluster-wide broadcast load touches another GPU's
 * memory).
 *
 * A handle for this mode is created with cfg.num_tokens = this rank's tokens
 * (the same on every rank) and cfg.num_ranks = R, the number of GPUs; global
 * row g of the world's receive buffer (the layout ep_plan gives for the
 * concatenation of all ranks' tokens, rank order) belongs to the rank r with
 * rank_offset[r] <= g < rank_offset[r+1], at local row g - rank_offset[r].
 * After ep_plan_world the single-GPU data calls (ep_dispatch, ep_combine, the
 * backward calls, the replica reduce and prefetch) refuse the handle with
 * EP_ERR_UNSUPPORTED, and the peer calls refuse a handle planned by ep_plan.
 */

#define EP_MAX_PEERS 64

/* Per-rank buffers of an EP world, as device addresses this GPU can reach
 * (CUDA IPC or symmetric-memory mappings of the peers' buffers, or plain
 * allocations on one GPU). Entry r belongs to rank r; unused arrays are NULL. */
typedef struct ep_peer_table {
    int32_t num_ranks;                   /* R, as in the handle's configuration */
    int64_t capacity_rows;               /* rows of every rank's receive buffer */
    void *recv_x[EP_MAX_PEERS];          /* [capacity_rows, H] bf16, or e4m3 bytes with fp8;
                                            ep_combine_peers reads the expert outputs here */
    float *recv_scales[EP_MAX_PEERS];    /* [capacity_rows, H/128] fp32 with fp8, else NULL */
    float *recv_w[EP_MAX_PEERS];         /* [capacity_rows] fp32, or NULL */
    int32_t *recv_expert[EP_MAX_PEERS];  /* [capacity_rows] int32, or NULL */
    uint32_t *flags[EP_MAX_PEERS];       /* [R] uint32: rank r's completion flags, one per source rank */
} ep_peer_table_t;

/* Rows one rank's receive buffer must hold for any routing (host-only):
 * LL (E/R)*ll_capacity; HT with a balanced plan ceil(L/R) for L = R*T*K pairs
 * of the world (more only when the plan flags EP_FLAG_PLAN_SLOTS); HT without
 * a plan L, since all pairs may route to one rank. */
ep_status_t ep_world_recv_rows(const ep_config_t *cfg, int64_t *rows);

/* Count this rank's routed pairs per expert: counts (device int32 [E]) as in
 * EP_T_EXPERT_COUNTS, the same rules for masked, bad and repeated ids (the
 * status word is cleared first). Keeps the per-tile ranks that ep_plan_world
 * completes. Always the three-kernel routing path's first two kernels. */
ep_status_t ep_plan_local_counts(ep_handle_t *h, const int32_t *topk_idx, int32_t *counts, void *stream);

/* Complete the plan of this rank (`rank`, in [0, R)) from world_counts
 * (device int32 [R, E], row r = rank r's ep_plan_local_counts output), after
 * ep_plan_local_counts on the same handle and batch. Every rank computes the
 * same layout (with cfg.balanced, the same balanced plan of the world's
 * counts); EP_T_DEST_ROW then holds global rows, EP_T_RANK_OFFSET,
 * EP_T_RANK_LOAD, EP_T_RECV_COUNTS, EP_T_REPLICA_EXPERT and
 * EP_T_EXPERT_COUNTS describe the whole world, and EP_T_SRC_ROW is not kept.
 * Counts inconsistent with the batch give unspecified rows (never an access
 * outside the buffers: ep_dispatch_peers checks every row against
 * capacity_rows). */
ep_status_t ep_plan_world(ep_handle_t *h, const int32_t *world_counts, int32_t rank, void *stream);

/* The send phase: for every routed pair (t,k) of this rank with global row g
 * on rank r at local row l, the same values as ep_dispatch (bf16 copy, or the
 * FP8 cast with its scales, recv_w, recv_expert) written to
 * peers->recv_x[r] row l (and the other arrays likewise). A row at or beyond
 * peers->capacity_rows is skipped and EP_FLAG_CAPACITY raised. */
ep_status_t ep_dispatch_peers(ep_handle_t *h, const void *x, const int32_t *topk_idx, const float *topk_w,
                              const ep_peer_table_t *peers, void *stream);

/* After the kernels before it on `stream` (stream order), make their writes
 * visible to the whole system and set peers->flags[r][rank] = epoch on every
 * rank r, with release semantics. */
ep_status_t ep_signal_peers(ep_handle_t *h, const ep_peer_table_t *peers, uint32_t epoch, void *stream);

/* The receive phase: a kernel on `stream` waits until flags[s] (device
 * uint32 [R], this rank's flags) has reached `epoch` for every source s
 * (acquire semantics), so the kernels after it see every row the sources
 * wrote before signalling. The wait is bounded: after timeout_us (0 = 2 s)
 * it gives up, sets EP_FLAG_WAIT_TIMEOUT in the status word and returns. */
ep_status_t ep_wait_peers(ep_handle_t *h, const uint32_t *flags, uint32_t epoch, int64_t timeout_us,
                          void *stream);

/* Combine across ranks: out[t] as ep_combine computes it, each pair's row
 * read from peers->recv_x[r] at local row l (the expert outputs of rank r,
 * bf16). out: device bf16 [T, H] of this rank's tokens. */
ep_status_t ep_combine_peers(ep_handle_t *h, const ep_peer_table_t *peers, const float *topk_w, void *out,
                             void *stream);

/* The backward pass across ranks (NCCL EP Fig. 5: the routing state of the
 * forward pass serves the backward pass, roles swapped). The rows' tables use
 * only their recv_x entries: rank r's gradient rows, bf16 [capacity_rows, H].
 *   ep_combine_backward_peers: for every routed pair (t,k) of this rank with
 *     global row g on rank r at local row l,
 *       grad_rows->recv_x[r] row l = bf16(topk_w[t,k] * grad_out[t])
 *     (one fp32 product, one rounding; as ep_combine_backward). grad_out:
 *     this rank's bf16 [T, H]. Rows past capacity_rows are skipped and flagged.
 *   ep_dispatch_backward_peers: grad_x[t] = bf16(sum over k of the pair's row
 *     in grad_rows->recv_x[r], fp32 adds in k order from +0) (as
 *     ep_dispatch_backward). grad_x: this rank's bf16 [T, H].
 * Signal and wait between the ranks' phases as in the forward pass. */
ep_status_t ep_combine_backward_peers(ep_handle_t *h, const void *grad_out, const float *topk_w,
                                      const ep_peer_table_t *grad_rows, void *stream);
ep_status_t ep_dispatch_backward_peers(ep_handle_t *h, const ep_peer_table_t *grad_rows, void *grad_x,
                                       void *stream);

/* Replica-gradient reduce across ranks (MoonEP article para. 5): this rank
 * (the `rank` of its ep_plan_world) adds to each of its own experts e that has
 * replicas under the world's balanced plan the gradients of e's replica slots
 * (r, s), in ascending (r, s) order, read from replica_grads->recv_x[r] (rank
 * r's replica gradients, fp32 [S, G]) at slot s:
 *   owner_grad[e - rank*E/R, :] += replica_grads[r][s, :]   (fp32, in place)
 * owner_grad: this rank's fp32 [E/R, G], G = cfg.grad_elems_per_expert. Needs
 * cfg.balanced; the ranks' replica gradients must be complete (signal / wait). */
ep_status_t ep_reduce_replica_grads_peers(ep_handle_t *h, const ep_peer_table_t *replica_grads, float *owner_grad,
                                          void *stream);

/* Replica weight prefetch across ranks (MoonEP article paras. 3 and 5): for
 * each replica slot s of this rank that the world's balanced plan fills with
 * expert e, copy e's weights from its owner o = e / (E/R):
 *   prefetch_slots[s, :] = weights->recv_x[o][e - o*E/R, :]   (bytes_per_expert)
 * weights: a table whose recv_x[r] holds rank r's own experts' weights
 * [E/R, bytes_per_expert]; prefetch_slots: this rank's [S, bytes_per_expert].
 * Both 16-byte aligned, bytes_per_expert a positive multiple of 16. Empty
 * slots are not written. Needs cfg.balanced. */
ep_status_t ep_prefetch_replica_weights_peers(ep_handle_t *h, const ep_peer_table_t *weights,
                                              int64_t bytes_per_expert, void *prefetch_slots, void *stream);

/* CUDA IPC of one device buffer, for building a peer table across processes:
 * export gives a 64-byte handle of the allocation holding dev_ptr and the
 * pointer's offset inside it; import maps a peer's allocation into this
 * process (with peer access enabled) and returns the address at that offset
 * and the mapping's base (to release with ep_ipc_close). */
ep_status_t ep_ipc_export(const void *dev_ptr, uint8_t handle[64], int64_t *offset);
ep_status_t ep_ipc_import(const uint8_t handle[64], int64_t offset, void **dev_ptr, void **base);
ep_status_t ep_ipc_close(void *base);

/* ---- routing without allocation ---------------------------------------- */

/* Bytes of the fixed device scratch behind ep_route_noalloc (4 MiB); every
 * GPU that loads the library holds this much until the process exits. */
#define EP_NOALLOC_SCRATCH_BYTES (4 << 20)

/* The routing pass of ep_plan for the plain HT layout, for callers that
 * cannot allocate device memory: no handle, no cudaMalloc, no cudaFree and
 * no allocating library call. This has no counterpart on the pages; it
 * exists for hosts that reserve all device memory up front (for example a
 * serving engine whose memory pool owns nearly all of HBM, where an extra
 * allocation would fail, fragment the pool, or stall the device) and for
 * plugin environments that forbid allocation after initialisation.
 *
 * Computes, exactly as ep_plan does for an HT configuration without a plan:
 *   expert_counts[e] (device int32 [E]) = routed pairs of expert e;
 *   dest_row[t*K+k] (device int32 [T*K]) = sum of the counts of experts
 *     below e + the pair's stable index within e, or -1 if not routed;
 *   *flags (one device int32) = EP_FLAG_* bits (bad or repeated ids).
 * topk_idx: device int32 [T, K]; -1 marks a masked choice. T*K may be 0.
 *
 * Scratch lives in one static device array of EP_NOALLOC_SCRATCH_BYTES per
 * GPU. Sizes whose scratch would not fit (about T*K above 500k pairs, fewer
 * with many experts) return EP_ERR_TOO_LARGE and launch nothing; other
 * argument errors return EP_ERR_INVALID_ARG. The first call on a device
 * looks the array's device address up (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture. Every
 * call shares the array and it keeps the last call's contents (each call
 * writes every word it later reads, so nothing needs clearing), so calls
 * whose work overlaps on the GPU (other streams, other host threads) race:
 * order them. Asynchronous on `stream`, like ep_plan. */
ep_status_t ep_route_noalloc(const int32_t *topk_idx, int32_t num_tokens, int32_t topk, int32_t num_experts,
                             int32_t *dest_row, int32_t *expert_counts, int32_t *flags, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_H */
