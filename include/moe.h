/*
 * moe.h -- C ABI of a B200 (sm_100a) library for one Mixture-of-Experts layer forward on
 * one GPU:  route -> dispatch -> expert SwiGLU grouped GEMM -> combine -> load statistics.
 *
 * Sources (page title, section):
 *   [EP-serving] "Expert Parallelism for MoE Serving" (aiunderstanding.org): "Deep dive"
 *                (a router picks the top-k experts per token, often 1 or 2; tokens are
 *                shuffled to their experts, the FFN runs, results are shuffled back) and
 *                "Technical insight" (two all-to-alls per layer, dispatch and combine;
 *                capacity factors, expert buffers and dropping or padding tokens keep the
 *                GEMMs uniform); FAQ (capacity = max tokens per expert, pad or drop past it).
 *   [EP-checks]  "MoE expert parallelism needs measurements before launch" (airouter.kz):
 *                "Mean expert load proves almost nothing" (mu = sum n_e / E; the per-layer
 *                record of tokens_per_expert, p50, p95, max, max/mean, top-5% share,
 *                dropped_tokens), "Capacity factor changes quality, memory and the latency
 *                tail" (capacity = mean tokens per expert x factor for top-1; overflow
 *                dropped; drop_tokens=false = unlimited; drop rate per route),
 *                "Profile all-to-all separately from compute" (router, pack/permute,
 *                dispatch, expert compute, combine, unpack; EP=1 keeps experts local with
 *                no all-to-all).
 *   [MegaScale]  "MegaScale-Infer: expert parallelism" slides (polomodov.tech), slide 11
 *                (the exchange library makes no GPU->CPU copies and no GPU synchronisation).
 *
 * On one GPU the two all-to-alls of [EP-serving] become a local permutation (dispatch)
 * and its inverse with a gate-weighted sum (combine), as in the EP=1 control run of
 * [EP-checks].
 *
 * Conventions for every entry point
 *   - All tensors are row-major and contiguous.  Weights are stored "out x in", i.e. the
 *     reduction dimension is innermost.
 *   - Device pointers are CUDA global memory of the current device.  The caller owns and
 *     allocates every buffer, including the workspace; the library allocates nothing and
 *     keeps no state besides a per-thread error string and a process-wide wait limit.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *     the call returns without synchronising, except where a host output is requested.
 *     Following [MegaScale] slide 11, per-expert counts never travel to the host: every
 *     kernel reads them from device memory.
 *   - Pointers passed to the library must be 16-byte aligned; T, d_model and d_ff must be
 *     such that every row is a multiple of 16 bytes.
 *   - Errors: a host-side check fails with MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED /
 *     MOE_ERR_WORKSPACE before anything is enqueued; a CUDA launch error gives
 *     MOE_ERR_CUDA.  Errors found by kernels (an expert index out of range, a bounded
 *     device wait that ran out, an expert-parallel row past its receive buffer) are
 *     recorded in the workspace's status word and reported by moe_check_device_error().  moe_last_error() gives a message for the last failure
 *     on the calling thread.
 *   - Inputs are finite; NaN and Inf inputs give unspecified results.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 5
#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOPK 8

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, k > E ...   */
  MOE_ERR_UNSUPPORTED = 2,   /* a valid request this build does not implement           */
  MOE_ERR_WORKSPACE = 3,     /* ws_bytes smaller than moe_workspace_size() asks          */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed                        */
  MOE_ERR_TIMEOUT = 5,       /* a bounded device wait ran out (reported lazily)          */
  MOE_ERR_DEVICE_DATA = 6    /* a kernel met invalid data, e.g. expert index >= E        */
} moe_status_t;

typedef enum { MOE_GATE_SOFTMAX = 0, MOE_GATE_SIGMOID = 1 } moe_gating_t;
typedef enum { MOE_LAYOUT_COMPACT = 0, MOE_LAYOUT_PADDED = 1 } moe_layout_t;
typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;
typedef enum { MOE_BIAS_SCORE_AND_WEIGHT = 0, MOE_BIAS_SELECTION_ONLY = 1 } moe_bias_mode_t;
typedef enum {
  MOE_DROP_TOKEN_ORDER = 0,
  MOE_DROP_PICK_RANK = 1,
  MOE_DROP_SCORE = 2
} moe_drop_policy_t;

/*
 * One layer's shape and routing rule.
 *   T               tokens in the batch ([EP-checks] "First fix the workload unit": the
 *                   active tokens of this layer and batch), 1 .. 2^31 - 1, with T*k and
 *                   the row count also below 2^31
 *   d_model, d_ff   model and expert hidden widths (d_model a multiple of 8, d_ff of 4,
 *                   both at most 2^24; bf16 expert FFNs need multiples of 64)
 *   E, k            experts (1..256) and picks per token (1..min(E, 8)) [EP-serving]
 *   gating          MOE_GATE_SOFTMAX: w_j = exp(z_j - z_max) / sum over the k picks;
 *                   MOE_GATE_SIGMOID: w_j = s(z_j) / sum over the k picks of s(z)
 *   layout          MOE_LAYOUT_COMPACT: expert buckets back to back, Sum(kept) rows;
 *                   MOE_LAYOUT_PADDED: bucket e starts at row e*C, E*C rows (needs a
 *                   finite capacity) [EP-serving "Technical insight": pad or drop]
 *   dtype           element type of x, expert weights, x_perm, h, y_perm and out
 *                   (MOE_F32: fp32 everywhere, fp32 FMA arithmetic;
 *                    MOE_BF16: bf16 storage, fp32 accumulation on tensor cores).
 *                   The router weight, logit bias, logits and gate weights are fp32.
 *   capacity_factor cf > 0: capacity C = ceil(cf * T * k / E) slots per expert;
 *                   cf <= 0: dropless ([EP-checks] "Capacity factor ...").
 * Routing variants (all zero = the plain rule above):
 *   n_groups, topk_groups   group-limited routing ([EP-serving] "Real-world implementation":
 *                   DeepSeek-V3 limits the nodes a token's experts span).  With n_groups > 1
 *                   the experts form n_groups equal contiguous groups; a group's score is
 *                   the largest selection score of its experts; a token keeps the
 *                   topk_groups best groups (equal scores -> lower group index) and takes
 *                   its k experts from them only.  Needs E % n_groups == 0 and
 *                   topk_groups * E / n_groups >= k.
 *   bias_mode       MOE_BIAS_SCORE_AND_WEIGHT: the logit bias enters selection and weights;
 *                   MOE_BIAS_SELECTION_ONLY: selection uses fp32(z + b) while the gate
 *                   weights and the returned logits use the unbiased z (the bias-only
 *                   balancing [EP-serving] "Future" names as loss-free load balancing).
 *   drop_policy     MOE_DROP_TOKEN_ORDER: within an expert, slots go by token index;
 *                   MOE_DROP_PICK_RANK: all first picks (in token order) before all second
 *                   picks, and so on, so capacity drops later picks first ([EP-checks]
 *                   "Top-2 does not insure against hot experts": second choices measured
 *                   and dropped separately);
 *                   MOE_DROP_SCORE: an overflowing expert keeps its C picks of highest
 *                   selection score (the fp32 score the top-k used; equal scores -> lower
 *                   token; NaN below every number, -0 equal to +0); the kept picks take
 *                   slots in token order, so without overflow the rows are those of
 *                   MOE_DROP_TOKEN_ORDER.  Dispatch then needs the scores:
 *                   moe_dispatch_scored (moe_layer_forward passes them itself).
 */
typedef struct moe_config {
  int64_t T;
  int64_t d_model;
  int64_t d_ff;
  int32_t E;
  int32_t k;
  int32_t gating;   /* moe_gating_t */
  int32_t layout;   /* moe_layout_t */
  int32_t dtype;    /* moe_dtype_t  */
  float capacity_factor;
  int32_t n_groups;     /* 0 or 1: no group limit */
  int32_t topk_groups;
  int32_t bias_mode;    /* moe_bias_mode_t   */
  int32_t drop_policy;  /* moe_drop_policy_t */
} moe_config_t;

/*
 * Per-layer load statistics ([EP-checks] "Mean expert load proves almost nothing" and
 * "Capacity factor ...": per-layer and per-route drop rate).
 *   tokens_per_expert is the kept count of each expert (the caller's kept_counts array);
 *   p50/p95/p99/max/mean/max_to_mean/top5pct_share are over those E kept counts, empty
 *   experts included; percentiles use linear interpolation between order statistics;
 *   mean = Sum kept / E; top5pct_share = (sum of the ceil(0.05 E) largest) / Sum kept;
 *   dropped counts dropped (token, expert) assignments = T*k - Sum kept;
 *   dropped_by_rank[j] counts drops of the j-th pick (j < k; the rest are 0);
 *   routed_* describe demand before the capacity limit.  Unused fields are 0.
 */
typedef struct moe_load_stats {
  int32_t E;
  int32_t k;
  int64_t active_tokens;
  int64_t capacity;            /* -1: dropless */
  int64_t routed_total;
  int64_t kept_total;
  int64_t dropped;
  int64_t tokens_with_drop;
  int64_t tokens_fully_dropped;
  double p50;
  double p95;
  double p99;
  double max;
  double mean;
  double max_to_mean;
  double routed_max;
  double routed_max_to_mean;
  double top5pct_share;
  int64_t dropped_by_rank[MOE_MAX_TOPK];
} moe_load_stats_t;

/* Inputs of a whole layer (device pointers). */
typedef struct moe_layer_inputs {
  const void* x;             /* [T, d_model] dtype                                        */
  const float* w_router;     /* [d_model, E] fp32                                         */
  const float* logit_bias;   /* NULL, or fp32 rows of E values, see bias_row_stride       */
  int64_t bias_row_stride;   /* 0: one [E] vector for all tokens; >= E: row t at t*stride */
  const void* w_gate;        /* [E, d_ff, d_model] dtype                                  */
  const void* w_up;          /* [E, d_ff, d_model] dtype                                  */
  const void* w_down;        /* [E, d_model, d_ff] dtype                                  */
  const void* w_router_split;/* NULL, or the split router weight of moe_router_split for
                                w_router: the tensor-core router then reads it instead of
                                splitting w_router at every call (see moe_route_ex)          */
} moe_layer_inputs_t;

/* Outputs and intermediates of a whole layer (device pointers, caller-allocated). */
typedef struct moe_layer_buffers {
  float* logits;             /* [T, E] fp32, or NULL to keep them in the workspace        */
  int32_t* topk_idx;         /* [T, k] experts, best first                               */
  float* topk_w;             /* [T, k] gate weights                                      */
  int32_t* routed_counts;    /* [E] assignments routed to each expert                    */
  int32_t* kept_counts;      /* [E] assignments kept (= tokens_per_expert)               */
  int32_t* expert_offsets;   /* [E+1] first row of each bucket; [E] = rows in use/alloc  */
  int32_t* assign_row;       /* [T, k] row of x_perm holding pick j of token t; -1 dropped*/
  int32_t* token_of_row;     /* [max_rows] token of each row; -1 for unused rows          */
  void* x_perm;              /* [max_rows, d_model] dtype, or NULL: no permuted copy, the */
                             /* gate/up GEMM gathers rows of x (moe_expert_ffn_gather)   */
  void* h;                   /* [max_rows, d_ff] dtype                                   */
  void* y_perm;              /* [max_rows, d_model] dtype                                */
  void* out;                 /* [T, d_model] dtype                                       */
  moe_load_stats_t* stats;   /* device struct, or NULL to skip the statistics            */
} moe_layer_buffers_t;

/* ---------------------------------------------------------------- expert parallelism
 *
 * [EP-serving] "Deep dive" / "Technical insight": with expert parallelism each rank (one
 * GPU) owns a subset of the experts, and every MoE layer runs two all-to-alls: dispatch
 * sends each token's row to the owners of its experts, combine returns the results.
 * [EP-checks] "Capacity factor changes quality, memory and the latency tail": tokens past
 * the capacity are dropped before the exchange, so each rank routes, ranks and drops its
 * own tokens with moe_route + moe_dispatch (moe_dispatch_scored under MOE_DROP_SCORE; x_perm
 * may be NULL) exactly as on one GPU, and the EP result on a rank equals the single-GPU layer
 * on that rank's tokens.
 *
 * No collective library moves the rows: every rank can address every rank's count
 * matrix, receive buffer and result buffer (peer pointers through NVLink, opened with
 * moe_ipc_open; or plain pointers when ranks share one device), and the exchange is fused
 * into the kernels:
 *   1. moe_ep_put_counts   my kept_counts -> row `rank` of every rank's count matrix
 *   --- all ranks' step 1 complete (barrier) ---
 *   2. moe_ep_plan         send_row of my picks; my local bucket table
 *   3. moe_ep_dispatch     my token rows -> the owners' receive buffers
 *   --- all ranks' step 3 complete (barrier) ---
 *   4. moe_ep_expert_ffn   grouped GEMM of my experts over my receive buffer
 *   --- all ranks' step 4 complete (barrier) ---
 *   5. moe_ep_combine      out[t] from the owners' result buffers, in pick order
 *   6. moe_ep_stats        the per-layer rank / node / pair-traffic record
 *   --- all ranks' step 5 complete before anyone's next step 1 or 3 (barrier) ---
 * The barriers are the caller's (for instance a stream-ordered all-reduce of one element
 * across the ranks); when all ranks run on one device in one stream, stream order is the
 * barrier.  Every kernel here is stream-ordered and never waits on another rank.
 *
 * Receive layout of rank g (rows of d_model elements): g's experts in ascending index; in
 * each expert the rows of source rank 0, then 1, ...; in each source its slot order.
 */
typedef struct moe_ep_config {
  int32_t world;           /* ranks, 1 .. 64                                               */
  int32_t rank;            /* this rank, 0 .. world-1                                      */
  int32_t ranks_per_node;  /* rank r sits on node r / ranks_per_node (>= 1)                */
  int32_t n_local;         /* experts this rank owns (= count of expert_rank[e] == rank)   */
  const int32_t* expert_rank; /* device [E]: owner of each expert (same on every rank)     */
  int64_t recv_rows;       /* rows of every rank's receive / result buffer (same on all)   */
} moe_ep_config_t;

/* Per-layer record of [EP-checks] "Expert and GPU can be balanced differently", from the
 * count matrix (identical on every rank after step 1).  Loads count kept assignments;
 * bytes count rows x d_model x element size sent between different ranks in one dispatch
 * (the combine returns the same bytes).  Pair figures run over every ordered pair of
 * different ranks, empty pairs included; percentiles interpolate linearly (type 7). */
typedef struct moe_ep_stats {
  int32_t world, ranks_per_node, nodes, reserved;
  int64_t total_assignments;   /* kept assignments of all ranks                            */
  int64_t local_assignments;   /* token and expert on the same rank                        */
  int64_t remote_bytes;        /* bytes crossing between ranks                              */
  int64_t cross_node_bytes;    /* of those, between ranks of different nodes               */
  double local_fraction;       /* local / total                                            */
  double cross_node_fraction;  /* cross_node_bytes / remote_bytes                          */
  double pair_bytes_p50, pair_bytes_p99, pair_bytes_max;
  double rank_load_max, rank_load_mean, rank_load_max_minus_mean, rank_load_max_to_mean;
  double node_load_max_to_mean;
  int64_t rank_load[64];       /* assignments of the experts each rank owns                */
  int64_t node_load[64];
  int64_t bytes_sent[64];      /* remote bytes each rank sends in a dispatch               */
  int64_t bytes_recv[64];
} moe_ep_stats_t;

/* ---------------------------------------------------------------- sizes */

/* Bytes of workspace every entry point below needs for `cfg` (the maximum over them). */
moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* Enqueue the zeroing of the workspace's status word.  Call once after allocating. */
moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Capacity C = ceil(cf * T * k / E) for cf > 0, -1 when dropless, -2 on a bad cfg. */
int64_t moe_capacity(const moe_config_t* cfg);

/* Rows to allocate for x_perm, h, y_perm and token_of_row: T*k when dropless,
 * min(T*k, E*C) when COMPACT with a capacity, E*C when PADDED.  -2 on a bad cfg. */
int64_t moe_max_rows(const moe_config_t* cfg);

/* ---------------------------------------------------------------- stages */

/*
 * Router scoring, top-k selection and gate weights ([EP-serving] "Deep dive").
 *   z[t, e] = sum_i x[t, i] * w_router[i, e] + b[t, e]   (fp32 accumulation)
 *   topk_idx[t, :] = the k largest z[t, :], best first; equal z -> lower expert index
 *   topk_w[t, :]   = gate weights renormalised over the k picks (cfg->gating)
 * logits may be NULL (then z lives in the workspace).  Needs the workspace.
 * Precision of z: fp32 FMA on CUDA cores, except for bf16 layers with E > 32 and d_model a
 * multiple of 64, where z = x . hi + x . lo runs on the tensor cores with W_r split into two
 * bf16 terms (|z - exact| <= 1e-4 (1 + |z|)); with few 128-token tiles (fewer than half the
 * SMs) each tile's K steps are split over several blocks and their fp32 sums added in a
 * fixed order.  The top-k is always taken on the fp32 z that is returned, so picks, weights
 * and everything downstream follow z.
 */
moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* w_router,
                       const float* logit_bias, int64_t bias_row_stride, float* logits,
                       int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * The split router weight of the tensor-core router, made once instead of at every call.
 * The router weight is constant across the forwards of a layer, but moe_route splits it
 * again each time: W' [E, 2 d_model] bf16, row e = [hi(w_router[:, e]), lo(w_router[:, e])],
 * hi = bf16(w), lo = bf16(w - hi) (round to nearest even), 2 E d_model bf16 values, 16-byte
 * aligned device memory owned by the caller.
 * moe_router_split_size: *bytes = that size, or 0 when the layer shape never takes the
 *   tensor-core router (fp32 layers, E <= 32, d_model not a multiple of 64).
 * moe_router_split: enqueue the split on `stream`.  MOE_ERR_UNSUPPORTED when the size is 0,
 *   MOE_ERR_INVALID_ARG when split_bytes is smaller or a pointer is NULL or unaligned.
 * The pages have no such step: it moves work the router repeats out of the forward.
 */
moe_status_t moe_router_split_size(const moe_config_t* cfg, size_t* bytes);
moe_status_t moe_router_split(const moe_config_t* cfg, const float* w_router, void* w_split,
                              size_t split_bytes, void* stream);

/*
 * moe_route with an optional argument: w_router_split NULL is moe_route; otherwise it is the
 * moe_router_split output for w_router, which the tensor-core router reads instead of
 * splitting w_router (one kernel launch fewer; the result is bitwise the same).  The other
 * router paths (fp32, E <= 32, d_model not a multiple of 64) read w_router and ignore it, so
 * w_router is required either way.  A split that was not made from this w_router gives the logits of the
 * weight it was made from.
 */
moe_status_t moe_route_ex(const moe_config_t* cfg, const void* x, const float* w_router,
                          const void* w_router_split, const float* logit_bias,
                          int64_t bias_row_stride, float* logits, int32_t* topk_idx,
                          float* topk_w, void* ws, size_t ws_bytes, void* stream);

/*
 * Dispatch ([EP-serving] "Technical insight"; [EP-checks] "Profile all-to-all ...": pack
 * and permute; "Capacity factor ...": overflow dropped).  Assignments are ranked within
 * each expert in token order; slot < C is kept, the rest dropped.
 *   routed_counts[e], kept_counts[e] = min(routed, C), expert_offsets[e] = first row of
 *   bucket e (COMPACT: exclusive scan of kept; PADDED: e*C), expert_offsets[E] = rows.
 *   assign_row[t, j] = expert_offsets[e] + slot, or -1 if dropped.
 *   token_of_row[r] = token copied into row r; -1 for rows no assignment uses.
 *   x_perm[assign_row[t, j], :] = x[t, :] for every kept pick; unused rows untouched.
 * x_perm may be NULL (x may then be NULL too): only the counts, offsets, assign_row and
 * token_of_row are produced, for moe_expert_ffn_gather.
 * With MOE_DROP_SCORE this call returns MOE_ERR_INVALID_ARG: use moe_dispatch_scored.
 */
moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                          int32_t* routed_counts, int32_t* kept_counts,
                          int32_t* expert_offsets, int32_t* assign_row,
                          int32_t* token_of_row, void* x_perm, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * moe_dispatch with the selection scores, for MOE_DROP_SCORE ([EP-checks] "Top-2 does not
 * insure against hot experts": which assignments an overflowing expert keeps).  The score
 * of pick (t, e) is logits[t, e], plus logit_bias[t * bias_row_stride + e] (fp32, one
 * addition) when cfg->bias_mode is MOE_BIAS_SELECTION_ONLY; with MOE_BIAS_SCORE_AND_WEIGHT
 * the bias is already inside the logits and logit_bias is not read.  Pass the logits and
 * bias moe_route used, so that the drop decision follows the same score as the pick.
 *   logits           [T, E] fp32 device array (required with MOE_DROP_SCORE)
 *   logit_bias       NULL, or fp32 rows as in moe_route; bias_row_stride 0 or >= E
 * Outputs, ownership and x_perm as in moe_dispatch.  Each expert with routed > C keeps the
 * C picks of highest priority (score, then lower token); its kept picks take slots 0, 1,
 * ... in token order; the rest get assign_row -1.  Scratch for the ranking comes from the
 * workspace (moe_workspace_size counts it for MOE_DROP_SCORE).  Six kernels (five without
 * x_perm), no host synchronisation.  With the other drop policies the scores are not read
 * and the call equals moe_dispatch.  An expert index outside [0, E) is skipped and reported
 * through the workspace status.
 */
moe_status_t moe_dispatch_scored(const moe_config_t* cfg, const void* x,
                                 const int32_t* topk_idx, const float* logits,
                                 const float* logit_bias, int64_t bias_row_stride,
                                 int32_t* routed_counts, int32_t* kept_counts,
                                 int32_t* expert_offsets, int32_t* assign_row,
                                 int32_t* token_of_row, void* x_perm, void* ws,
                                 size_t ws_bytes, void* stream);

/*
 * moe_dispatch without a workspace.  The pages have no counterpart to this entry point; it
 * exists for callers that cannot allocate device memory when they dispatch, for example
 * code inside a serving engine whose memory pool owns the whole GPU, or a plugin host that
 * hands kernels only their input and output tensors.  cudaMalloc is not an option there:
 * it synchronises the device and may fail once the pool has taken the memory.
 *
 * Same arguments, results and ordering as moe_dispatch minus (ws, ws_bytes).  The scratch
 * it needs (a status record and ceil(T/256)*E int32 block counts) lives in one fixed
 * 1 MiB + 256 B array in device memory, which every GPU that loads this library keeps
 * until the process exits; the call allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).  Limits and behaviour:
 *   - ceil(T/256) * E * 4 bytes (times k with MOE_DROP_PICK_RANK) must fit in 1 MiB (e.g.
 *     T <= 262144 at E = 256); larger sizes return MOE_ERR_UNSUPPORTED with a message,
 *     before anything is enqueued.  MOE_DROP_SCORE (which needs the scores and more
 *     scratch) returns MOE_ERR_UNSUPPORTED.
 *   - The first call on each device looks up the array's device address with that device
 *     current; make that first call before any stream capture.
 *   - Every call shares the one array: two calls that run on the GPU at the same time
 *     (other streams, other host threads) race and give wrong results.  Order them.
 *   - Kernel-side errors go to a status record in the same fixed array, which starts at
 *     zero and keeps the first error since it was last read: an expert index outside
 *     [0, E) (the pick is skipped, like a dropped one) or a bounded wait in the permute
 *     that ran out (x_perm is then incomplete).  A call does not clear it;
 *     moe_static_scratch_check() reports and clears it, without allocating.
 */
moe_status_t moe_dispatch_static_scratch(const moe_config_t* cfg, const void* x,
                                         const int32_t* topk_idx, int32_t* routed_counts,
                                         int32_t* kept_counts, int32_t* expert_offsets,
                                         int32_t* assign_row, int32_t* token_of_row,
                                         void* x_perm, void* stream);

/*
 * The kernel-side errors of moe_dispatch_static_scratch on the current device, for the same
 * callers (no counterpart on the pages; nothing is allocated).  Synchronises `stream`
 * (enqueue order: after the dispatch calls to be checked), reads the fixed scratch's status
 * record and, if it holds an error, clears it.  Returns MOE_OK if no call recorded an error
 * since the last check, else MOE_ERR_DEVICE_DATA (invalid expert index; the flat index of
 * the first one is in moe_last_error()) or MOE_ERR_TIMEOUT (a bounded wait in the permute
 * ran out).  Like the dispatch calls it shares the one array: checks and dispatches that
 * overlap on the GPU race.  Its first use on a device may do the device's set-up (see
 * moe_dispatch_static_scratch).
 */
moe_status_t moe_static_scratch_check(void* stream);

/*
 * Expert SwiGLU FFN as a grouped GEMM over the variable-sized buckets ([EP-checks]
 * "Profile all-to-all ...": grouped GEMMs over many experts).  For each expert e and each
 * row r in [expert_offsets[e], expert_offsets[e] + kept_counts[e]):
 *   h[r, :]      = silu(x_perm[r] . w_gate[e]^T) * (x_perm[r] . w_up[e]^T),
 *                  silu(u) = u / (1 + exp(-u))
 *   y_perm[r, :] = h[r] . w_down[e]^T
 * Rows outside every bucket are not written.  bf16 needs d_model and d_ff to be multiples
 * of 64 (MOE_ERR_UNSUPPORTED otherwise).  Needs the workspace (status word).
 */
moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                            const int32_t* expert_offsets, const int32_t* kept_counts,
                            const void* w_gate, const void* w_up, const void* w_down, void* h,
                            void* y_perm, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_ffn without the permuted copy of x: the gate/up GEMM reads bucket row r as
 * x[token_of_row[r], :] (16-byte asynchronous copies straight from x into the GEMM's
 * swizzled operand tiles), so dispatch need not write
 * x_perm.  This is the dispatch half of the fused dispatch-compute-combine kernels that
 * [EP-serving] names as the direction of expert parallelism (its closing section on the
 * future of EP serving, in the Wolof edition of the page).  Results are identical to
 * moe_dispatch + moe_expert_ffn.  token_of_row is
 * moe_dispatch's output ([max_rows] int32); an entry outside [0, T) inside a bucket reads
 * row 0 instead (never out of range).  Other arguments, layouts and errors as
 * moe_expert_ffn.
 */
moe_status_t moe_expert_ffn_gather(const moe_config_t* cfg, const void* x,
                                   const int32_t* token_of_row, const int32_t* expert_offsets,
                                   const int32_t* kept_counts, const void* w_gate,
                                   const void* w_up, const void* w_down, void* h, void* y_perm,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_ffn followed by moe_combine, with the combine fused into the down GEMM: as
 * each bucket row's 256-column block of y_perm is stored, its token's counter for that
 * block is bumped, and the thread completing the count sums the token's kept rows of the
 * block in pick order (fp32) into out.  This is the combine half of the fused
 * dispatch-compute-combine kernels that [EP-serving] names as the direction of expert
 * parallelism (its closing section on the future of EP serving, Wolof edition); the
 * combine's memory traffic overlaps the tensor-core work.  out is bitwise what
 * moe_combine gives; y_perm and h are written as by moe_expert_ffn.  A rows come from
 * x_perm, or, when x_perm is NULL, straight from x through token_of_row (as
 * moe_expert_ffn_gather).  fp32 layers run moe_combine's kernel after the FFN instead.
 * Uses the workspace's counters; calls on one workspace must not overlap.
 */
moe_status_t moe_expert_ffn_combine(const moe_config_t* cfg, const void* x, const void* x_perm,
                                    const int32_t* token_of_row, const int32_t* expert_offsets,
                                    const int32_t* kept_counts, const void* w_gate,
                                    const void* w_up, const void* w_down, void* h,
                                    void* y_perm, const int32_t* assign_row,
                                    const float* topk_w, void* out, void* ws, size_t ws_bytes,
                                    void* stream);

/*
 * Combine ([EP-serving] "Deep dive": results shuffled back; [EP-checks]: combine, unpack):
 *   out[t, :] = sum over j = 0..k-1 with assign_row[t, j] >= 0 of
 *               topk_w[t, j] * y_perm[assign_row[t, j], :]
 * summed in pick order in fp32, so the result is bitwise reproducible run to run.  A
 * dropped pick contributes nothing (no renormalisation); a fully dropped token gets 0.
 */
moe_status_t moe_combine(const moe_config_t* cfg, const void* y_perm,
                         const int32_t* assign_row, const float* topk_w, void* out,
                         void* stream);

/*
 * Per-layer load statistics (moe_load_stats_t above) from the dispatch outputs, written to
 * the device struct dev_out.  If host_out is not NULL the struct is also copied to host
 * memory and the stream is synchronised (as by every call given a host output, and by the
 * two error checks); with host_out NULL nothing waits.
 */
moe_status_t moe_load_stats(const moe_config_t* cfg, const int32_t* routed_counts,
                            const int32_t* kept_counts, const int32_t* assign_row,
                            moe_load_stats_t* dev_out, moe_load_stats_t* host_out,
                            void* stream);

/*
 * The job's record over data-parallel replicas: every GPU runs the whole layer on its own
 * tokens (no exchange) and the job reports one record per layer ([EP-checks] "Mean expert
 * load proves almost nothing").  It is the record of the union of the replicas' picks: the
 * per-expert counts added up, the drop counters and token counts added up, and an expert's
 * capacity the sum of the replicas' capacities (-1 if any replica is dropless).
 *   routed_sum, kept_sum  [E] int32 device arrays: element-wise sums over the replicas of
 *                         their routed_counts and kept_counts (e.g. an all-reduce SUM of
 *                         E ints each); every sum must be below 2^31
 *   parts                 [n_parts] device array of the replicas' moe_load_stats_t records
 *                         (e.g. an all-gather of the records moe_load_stats wrote), n_parts >= 1
 * cfg gives E and k; T and the capacity come from the records.  dev_out and host_out as in
 * moe_load_stats (a host copy synchronises the stream).  One kernel.
 */
moe_status_t moe_load_stats_merge(const moe_config_t* cfg, const int32_t* routed_sum,
                                  const int32_t* kept_sum, const moe_load_stats_t* parts,
                                  int32_t n_parts, moe_load_stats_t* dev_out,
                                  moe_load_stats_t* host_out, void* stream);

/*
 * Second-choice counters ([EP-checks] "Top-2 does not insure against hot experts": the
 * share of tokens whose second choice differs from the first, where second choices go, and
 * the share of second assignments that never reached the experts), for every pick rank j
 * (j = 0 the first choice, j = 1 the second, ...):
 *   routed_by_rank[j * E + e]  picks of rank j that chose expert e         ([k, E] int32)
 *   kept_by_rank[j * E + e]    those of them kept (assign_row >= 0)        ([k, E] int32)
 *   differs_by_rank[j]         tokens whose pick j lies in another group   ([k] int32)
 *                              than their pick 0; differs_by_rank[0] = 0
 * group_of_expert: NULL (a group is one expert, so for distinct picks differs = T for
 * j >= 1), or an [E] int32 device array mapping experts to any grouping the caller wants to
 * watch: routing groups, owner ranks, nodes.  Shares over the T tokens: differs / T, and
 * 1 - Sum_e kept_by_rank[j, e] / T dropped.  topk_idx and assign_row as moe_route and
 * moe_dispatch produce them.  One kernel, integer counts (deterministic), no host
 * synchronisation; every output element is written.  An expert index outside [0, E) is
 * skipped and reported through the workspace status.
 */
moe_status_t moe_pick_rank_counts(const moe_config_t* cfg, const int32_t* topk_idx,
                                  const int32_t* assign_row, const int32_t* group_of_expert,
                                  int32_t* routed_by_rank, int32_t* kept_by_rank,
                                  int32_t* differs_by_rank, void* ws, size_t ws_bytes,
                                  void* stream);

/*
 * The whole layer: moe_route_ex (with in->w_router_split), moe_dispatch_scored (given the
 * logits the router wrote: bufs->logits, or the workspace's copy when that is NULL; with the
 * drop policies other than MOE_DROP_SCORE this is moe_dispatch), moe_expert_ffn,
 * moe_combine and (when bufs->stats is
 * not NULL) moe_load_stats, enqueued back to back on one stream without a host
 * synchronisation.  bufs->x_perm NULL: dispatch writes no permuted copy and the gate/up GEMM
 * gathers rows of x (moe_expert_ffn_gather).  Returns the first failing stage's status.
 */
moe_status_t moe_layer_forward(const moe_config_t* cfg, const moe_layer_inputs_t* in,
                               const moe_layer_buffers_t* bufs, void* ws, size_t ws_bytes,
                               void* stream);

/* ---------------------------------------------------------------- errors */

/* Synchronise `stream`, read and clear the workspace status word.  MOE_OK if no kernel
 * recorded an error since the last check; MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_DATA
 * otherwise (details in moe_last_error()). */
moe_status_t moe_check_device_error(void* ws, size_t ws_bytes, void* stream);

/* Message for the last failing call on this thread ("" if none). */
const char* moe_last_error(void);

/* Static name of a status code. */
const char* moe_status_string(moe_status_t status);

/* Limit, in nanoseconds, on every wait a kernel makes on an on-chip barrier before it gives
 * up, records MOE_ERR_TIMEOUT and returns (default 2e9).  0 restores the default. */
void moe_set_wait_limit_ns(uint64_t ns);

/* Which kernel runs the bf16 expert FFN of moe_expert_ffn / moe_layer_forward (permuted
 * rows, combine separate), for the whole process.  A choice of schedule, not of results:
 * all three compute each output as the same fp32 sum in the same K order and give bitwise
 * the same h and y_perm.
 *   MOE_FFN_TOKEN_MAJOR (the default): one CTA per 128-token x 256-column tile (a bucket's
 *     last tile of at most 64 tokens runs at M = 64).
 *   MOE_FFN_TOKEN_N: the MMA's M = 128 rows are weight rows (output features), its N is up
 *     to 256 of a bucket's tokens, and a bucket's last tile takes its remaining tokens
 *     rounded up to 16 -- a ragged bucket wastes at most 15 rows of tensor work.
 *   MOE_FFN_CTA_PAIRS: each 256-token x 256-column tile on a pair of CTAs on the two SMs of
 *     a TPC sharing one tensor-core MMA (a cluster of two), each CTA loading half of each
 *     operand: a third fewer bytes from L2 per FLOP; if no cluster of two fits on the
 *     device, MOE_FFN_TOKEN_MAJOR runs.
 * The expert-parallel FFN (moe_ep_expert_ffn) follows the same setting; the gathered-A and
 * fused-combine forms always run the token-major kernel.  Returns MOE_ERR_INVALID_ARG for
 * an unknown kind. */
typedef enum {
  MOE_FFN_TOKEN_MAJOR = 0,
  MOE_FFN_CTA_PAIRS = 1,
  MOE_FFN_TOKEN_N = 2
} moe_ffn_kernel_t;
moe_status_t moe_set_ffn_kernel(moe_ffn_kernel_t kind);

/* Self-test of the bounded wait: one block waits on an on-chip barrier that nothing
 * completes, with the current limit, records MOE_ERR_TIMEOUT in the workspace status
 * word and returns.  Used to check that a run-out wait leaves the context usable. */
moe_status_t moe_selftest_bounded_wait(void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- expert parallelism calls
 * All take the layer's moe_config_t (global E, this rank's T) and the moe_ep_config_t.
 * Pointer tables (`mats`, `recv`, `ybuf`) are DEVICE arrays of `world` device pointers,
 * indexed by rank, that this rank may dereference.  Errors as for the single-GPU calls;
 * a row that would land at or past recv_rows is skipped and reported by
 * moe_check_device_error as MOE_ERR_DEVICE_DATA. */

/* Rows a receive buffer needs so that no distribution of picks can overflow it: world x
 * min(T*min(k, n_local), n_local*C) (C = capacity; T*min(k, n_local) when dropless),
 * with T the largest per-rank token count.  recv_rows must be the same on every rank (the
 * kernels check a row against the sender's value), so pass the n_local of the rank that
 * owns the most experts.  Reads only the sizes of cfg and ep; -2 (and
 * the reason in moe_last_error) when they are invalid. */
int64_t moe_ep_recv_rows_bound(const moe_config_t* cfg, const moe_ep_config_t* ep);

/* Step 1.  mats[g] -> rank g's count matrix [world, E] int32; row `rank` receives
 * kept_counts [E] (moe_dispatch's output). */
moe_status_t moe_ep_put_counts(const moe_config_t* cfg, const moe_ep_config_t* ep,
                               const int32_t* kept_counts, int32_t* const* mats, void* stream);

/* Step 2.  From this rank's full count matrix [world, E]:
 *   send_row [T, k]         row of pick (t, j) in its owner's receive buffer, -1 dropped
 *                           (= the owner's bucket start for the expert + the rows of lower
 *                           source ranks + the pick's slot on this rank);
 *   recv_offsets [n_local+1] start of each local expert's bucket in this rank's buffer
 *                           ([n_local] = rows received); recv_counts [n_local] its rows.
 * Buckets are cut at recv_rows (reported by moe_check_device_error as MOE_ERR_DEVICE_DATA),
 * so the local GEMM never reaches past the buffer.
 * topk_idx, assign_row, expert_offsets: this rank's moe_route / moe_dispatch outputs. */
moe_status_t moe_ep_plan(const moe_config_t* cfg, const moe_ep_config_t* ep,
                         const int32_t* count_mat, const int32_t* topk_idx,
                         const int32_t* assign_row, const int32_t* expert_offsets,
                         int32_t* send_row, int32_t* recv_offsets, int32_t* recv_counts,
                         void* ws, size_t ws_bytes, void* stream);

/* Step 3.  recv[g][send_row[t, j], :] = x[t, :] for every kept pick, g = the owner of
 * topk_idx[t, j]; each row of x is read once.  recv buffers: [recv_rows, d_model] dtype. */
moe_status_t moe_ep_dispatch(const moe_config_t* cfg, const moe_ep_config_t* ep,
                             const void* x, const int32_t* topk_idx, const int32_t* send_row,
                             void* const* recv, void* ws, size_t ws_bytes, void* stream);

/* Step 4.  moe_expert_ffn over this rank's receive buffer with its n_local experts'
 * weights (w_gate_local, w_up_local [n_local, d_ff, d_model]; w_down_local [n_local,
 * d_model, d_ff], local expert i = the i-th expert this rank owns in ascending index):
 * h [recv_rows, d_ff], y_recv [recv_rows, d_model]. */
moe_status_t moe_ep_expert_ffn(const moe_config_t* cfg, const moe_ep_config_t* ep,
                               const void* recv_x, const int32_t* recv_offsets,
                               const int32_t* recv_counts, const void* w_gate_local,
                               const void* w_up_local, const void* w_down_local, void* h,
                               void* y_recv, void* ws, size_t ws_bytes, void* stream);

/* Step 5.  out[t, :] = sum over kept picks j, in pick order, of topk_w[t, j] *
 * ybuf[g][send_row[t, j], :] (g = owner), fp32 accumulation: bitwise what moe_combine
 * gives on one GPU. */
moe_status_t moe_ep_combine(const moe_config_t* cfg, const moe_ep_config_t* ep,
                            const void* const* ybuf, const int32_t* topk_idx,
                            const int32_t* send_row, const float* topk_w, void* out,
                            void* ws, size_t ws_bytes, void* stream);

/* Step 6.  The EP record from the count matrix; host_out non-NULL copies it to the host
 * and synchronises the stream. */
moe_status_t moe_ep_stats(const moe_config_t* cfg, const moe_ep_config_t* ep,
                          const int32_t* count_mat, moe_ep_stats_t* dev_out,
                          moe_ep_stats_t* host_out, void* stream);

/* Peer memory for multi-process EP.  moe_ipc_handle gives the IPC handle (64 bytes) of the
 * device allocation that contains dev_ptr and dev_ptr's byte offset in it (allocators hand
 * out pieces of larger allocations); another process maps the allocation with
 * moe_ipc_open and adds the offset, and unmaps it with moe_ipc_close.  Thin wrappers of
 * the CUDA IPC calls; MOE_ERR_CUDA on failure. */
moe_status_t moe_ipc_handle(const void* dev_ptr, unsigned char handle_out[64],
                            int64_t* offset_out);
moe_status_t moe_ipc_open(const unsigned char handle[64], void** dev_ptr_out);
moe_status_t moe_ipc_close(void* dev_ptr);

/* MOE_ABI_VERSION of the loaded library. */
int32_t moe_abi_version(void);

/* Number of kernels this library has launched in this process so far, over every device
 * and stream (a launch is counted when it is issued, not when it runs).  The difference of
 * two readings around a region counts the library's kernels in it.  Never fails. */
uint64_t moe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
