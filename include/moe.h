/*
 * moe.h - C ABI of the B200 (sm_100a) MoE-layer forward.
 *
 * One token-routed Mixture-of-Experts layer, forward only, on one GPU:
 *
 *   logits = x W_r (+ bias)                       router GEMM
 *   idx = top-k(logits), gate = softmax over k    top-k routing
 *   counts / offsets / permutation / send layout  expert-grouped dispatch
 *   x_perm[r] = x[row_token[r]]                   permute
 *   h = silu(x_perm W_g[e]) * (x_perm W_u[e])     grouped SwiGLU, gate/up
 *   y_perm = h W_d[e]                             grouped SwiGLU, down
 *   y[t] = sum_j gate[t,j] y_perm[slot_row[t*k+j]] combine
 *
 * Sources (page title, then section / table; the tags are used below):
 *  - [Layout] "MoE Pretraining: Parallelism Layout Changes the Model, Not Quality",
 *    Methodology / Models and Data: a router sends each token to a few of 16
 *    SwiGLU experts (top-4); Finding 3: routing margin and near-ties.
 *  - [Revisiting] "Revisiting MoE and Dense Speed-Accuracy Comparisons for LLM Training",
 *    2.1 Architecture (SwiGLU, Top-K routing) and Table 1 (weight layouts:
 *    router "ME" = [d, E]; FFN1 "EMH" = [E, d, f]; FFN2 "EHM" = [E, f, d]).
 *  - [Coupling] "Expert Coupling in MoE Pretraining: Reducing All-to-All Overhead with
 *    Correlated Placement and Token Shuffling", Abstract (experts spread over
 *    EP ranks; each token sent to each GPU once), Table I (distinct GPUs per
 *    token, deduplicated rows; tokens split evenly over the GPUs), Table III
 *    (notation).
 *
 * Conventions for every call:
 *  - All array arguments are DEVICE pointers owned by the caller, except
 *    `expert_rank_host` (host memory, read during the call).  The library
 *    never allocates, never frees, and never synchronises the stream except
 *    in moe_get_device_status.
 *  - Every call enqueues its kernels on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns without waiting.  The returned status
 *    covers host-side argument checks and launch errors.  Errors detected on
 *    the device (an expert index out of range, a bounded wait that gave up)
 *    are recorded in the workspace's status word; read it with
 *    moe_get_device_status.
 *  - Row-major layouts throughout.  Floating-point tensors are bf16 (dtype
 *    MOE_BF16, fp32 accumulation) or fp32 (MOE_F32) as the shape says;
 *    router logits and gates are always fp32; indices are int32.
 *  - Pointers to bf16/fp32 tensors must be 16-byte aligned; int32 arrays
 *    4-byte aligned (MOE_ERR_ALIGNMENT otherwise).
 *  - Results are deterministic: repeated calls with the same inputs give
 *    bit-identical outputs (no floating-point atomics anywhere).
 *  - Calls on different streams with different workspaces may run
 *    concurrently.  The library's only global state is the scratch of
 *    moe_dispatch_layout_static (see there), a per-device record of the
 *    kernels' shared-memory limits and the CTA-pair GEMM's count of resident
 *    clusters (the last device queried), kept under locks.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* bad shape, NULL pointer, bad expert->rank map */
  MOE_ERR_UNSUPPORTED = 2,    /* valid shape outside what the kernels cover */
  MOE_ERR_ALIGNMENT = 3,      /* pointer not aligned as required */
  MOE_ERR_WORKSPACE = 4,      /* workspace / packed buffer too small */
  MOE_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait gave up */
  MOE_ERR_DEVICE_INDEX = 7    /* an expert index outside [0, E) reached a kernel */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/*
 * Problem statement, in the pages' notation (Expert Coupling, Table III):
 * T tokens of width d, E experts of FFN width f, top-k routing, and the
 * number of simulated expert-parallel ranks `ep` (P in Table III).
 * Supported: 0 <= T, T*k < 2^31; 1 <= E <= 256; 1 <= k <= min(E, 16);
 * 1 <= ep <= E with E % ep == 0; d % 64 == 0 and f % 64 == 0 with
 * d * sizeof(dtype) <= 16384 (else MOE_ERR_UNSUPPORTED).
 */
typedef struct {
  int64_t T;
  int32_t d;
  int32_t E;
  int32_t k;
  int32_t f;
  int32_t ep;
  int32_t dtype; /* moe_dtype */
} moe_shape;

/*
 * Dispatch statistics, written to device memory by moe_dispatch_layout
 * (Expert Coupling, Table I):
 *  rows_sent          sum over tokens of the number of distinct ranks its k
 *                     experts live on (one send row per token and rank);
 *                     0 when ep == 1 (nothing is dispatched)
 *  dup_removed        T*k - rows_sent: rows that a per-(token, expert)
 *                     dispatch would send and the deduplicated one does not;
 *                     0 when ep == 1
 *  tokens_single_rank tokens whose k experts all live on one rank
 *  home_rank_rows     assignments whose expert lives on the token's home
 *                     rank floor(t * ep / T) (T/ep tokens per rank)
 *  max/min_expert_rows largest / smallest per-expert row count
 */
typedef struct {
  int64_t rows_sent;
  int64_t dup_removed;
  int64_t tokens_single_rank;
  int64_t home_rank_rows;
  int32_t max_expert_rows;
  int32_t min_expert_rows;
} moe_stats;

/*
 * Outputs of moe_dispatch_layout (all device memory, R = T*k):
 *  expert_counts [E]      rows routed to each expert
 *  expert_offsets[E+1]    exclusive prefix sum; expert e owns rows
 *                         [expert_offsets[e], expert_offsets[e+1])
 *  row_token     [R]      token of each expert-grouped row; inside an expert
 *                         the rows follow the flat assignment index t*k+j
 *                         (a stable counting sort)
 *  slot_row      [R]      row of assignment t*k+j (inverse of row_token)
 *  rank_counts   [ep]     send rows per rank (deduplicated)           (*)
 *  rank_offsets  [ep+1]   exclusive prefix sum of rank_counts          (*)
 *  send_token    [R]      token of each send row: grouped by rank, tokens
 *                         ascending inside a rank; only the first
 *                         rank_offsets[ep] entries are written          (*)
 *  slot_send_row [R]      send row carrying assignment t*k+j            (*)
 *  stats                  moe_stats (device), may be NULL
 * (*) built only when ep > 1 (these may be NULL when ep == 1).
 */
typedef struct {
  int32_t* expert_counts;
  int32_t* expert_offsets;
  int32_t* row_token;
  int32_t* slot_row;
  int32_t* rank_counts;
  int32_t* rank_offsets;
  int32_t* send_token;
  int32_t* slot_send_row;
  moe_stats* stats;
} moe_layout;

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status s);

/*
 * Scratch workspace for moe_route, moe_dispatch_layout and
 * moe_grouped_swiglu (at most a few hundred KB): the device status word,
 * per-bin totals, the decoupled-lookback status words and the fused
 * router's per-tile histograms.
 * The workspace must be zero-filled once before its first use (cudaMemset or
 * moe_workspace_init); every call leaves it ready for the next call of any
 * shape.  One workspace serves one stream at a time.
 */
MOE_API moe_status moe_scratch_size(const moe_shape* shape, size_t* bytes);

/*
 * Workspace for moe_forward: the scratch above followed by every
 * intermediate the forward needs and the caller did not pass in
 * moe_forward_buffers (logits, routing, layout, x_perm, h, y_perm).
 */
MOE_API moe_status moe_forward_workspace_size(const moe_shape* shape, size_t* bytes);

/* Zero-fill `bytes` of workspace on `stream` (a cudaMemsetAsync). */
MOE_API moe_status moe_workspace_init(void* ws, size_t bytes, moe_stream_t stream);

/*
 * Size of the packed weight buffer for `shape`.
 */
MOE_API moe_status moe_packed_weights_size(const moe_shape* shape, size_t* bytes);

/*
 * Rearrange the layer's weights once into the kernels' operand layout
 * (K-major, i.e. each output column's weights contiguous):
 *   router  W_r [d, E] ("ME")   -> W_r^T [E16, d], E16 = E rounded up to 16,
 *                                   extra rows zero
 *   W_g, W_u [E, d, f] ("EMH")  -> per expert [2f, d]: blocks of B output
 *                                   columns, gate rows then up rows
 *                                   (B = 128 if f % 128 == 0 else 64)
 *   W_d [E, f, d] ("EHM")       -> per expert W_d^T [d, f]
 * All inputs in the shape's dtype, device memory, row-major.  The packed
 * buffer is what moe_route, moe_grouped_swiglu and moe_forward read; it is
 * only valid for the shape it was packed for.  Either part may be left out:
 * w_router NULL packs the experts alone, w_gate, w_up and w_down all NULL
 * the router alone (the part left out is not written and must not be read:
 * an expert-parallel rank routes with the whole router and holds only its
 * own experts).
 */
MOE_API moe_status moe_pack_weights(const moe_shape* shape, const void* w_router,
                            const void* w_gate, const void* w_up,
                            const void* w_down, void* packed,
                            size_t packed_bytes, moe_stream_t stream);

/*
 * Router GEMM + top-k + gates.  Defined by: [Layout] Methodology / Models and
 * Data (a router picks the top-4 of the experts per token); [Revisiting] 2.1
 * (Top-K routing) and Table 1 (router "ME" = [d, E]).
 *  x        [T, d] tokens (dtype), or NULL: then `logits` is an INPUT and only
 *           the top-k step runs on it ("given logits" mode)
 *  packed   packed weights (moe_pack_weights); unused when x == NULL
 *  bias     [E] fp32 added to the logits before selection, or NULL
 *  logits   [T, E] fp32: l[t,e] = sum_i x[t,i] W_r[i,e] + bias[e]
 *  topk_idx [T, k] int32: the k experts with the largest logits, ordered
 *           by (logit descending, expert index ascending); equal logits
 *           (including -0.0 vs +0.0) resolve to the lower index
 *  topk_gate[T, k] fp32: softmax of the k chosen logits
 *           g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
 *  ws, ws_bytes scratch workspace (moe_scratch_size), for device errors
 * Logits must be finite (NaN gives unspecified routing).
 */
MOE_API moe_status moe_route(const moe_shape* shape, const void* x, const void* packed,
                     const float* bias, float* logits, int32_t* topk_idx,
                     float* topk_gate, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * The router and the expert FFN on weights in the pages' own layouts, for
 * callers that keep the weights as [d, E] ("ME") for the router and
 * [E, d, f] ("EMH") / [E, f, d] ("EHM") for the experts ("Revisiting MoE and
 * Dense Speed-Accuracy Comparisons", Table 1).  Each call first packs the
 * weights it reads into the workspace (the transposes moe_pack_weights does
 * once), then runs the packed path, so its results are bit-identical to
 * moe_route / moe_grouped_swiglu on moe_pack_weights output.  Packing on
 * every call moves every weight byte twice more: pack once with
 * moe_pack_weights where the weights do not change between calls.
 *  ws, ws_bytes  at least moe_unpacked_workspace_size bytes (the scratch
 *                workspace followed by room for the packed weights),
 *                zero-filled once before first use like the scratch
 */
MOE_API moe_status moe_unpacked_workspace_size(const moe_shape* shape, size_t* bytes);

/*
 * moe_route with W_r [d, E] ("ME") in the shape's dtype (device) in place of
 * the packed buffer; x must not be NULL.  Other arguments as in moe_route.
 */
MOE_API moe_status moe_route_unpacked(const moe_shape* shape, const void* x,
                                      const void* w_router, const float* bias, float* logits,
                                      int32_t* topk_idx, float* topk_gate, void* ws,
                                      size_t ws_bytes, moe_stream_t stream);

/*
 * moe_grouped_swiglu with W_g, W_u [E, d, f] ("EMH") and W_d [E, f, d]
 * ("EHM") in the shape's dtype (device) in place of the packed buffer.
 * Other arguments as in moe_grouped_swiglu.
 */
MOE_API moe_status moe_grouped_swiglu_unpacked(const moe_shape* shape, const void* x_perm,
                                               const int32_t* expert_offsets,
                                               const void* w_gate, const void* w_up,
                                               const void* w_down, void* h, void* y_perm,
                                               void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_route with a selection-only expert bias: the experts are chosen on the
 * fp32 sum logits + selection_bias (same key and tie-break as moe_route),
 * and the gates are the softmax of the chosen experts' logits WITHOUT the
 * selection bias, in the chosen order.  This is the auxiliary-loss-free
 * router: a per-expert bias that steers which experts are picked for load
 * balance without changing how their outputs are weighted ("Expert Coupling
 * in MoE Pretraining", Fig. 11: the auxiliary-loss-free router; "MoE
 * Pretraining: Parallelism Layout Changes the Model, Not Quality",
 * introduction: loss-free balancing counts).
 *  selection_bias [E] fp32, device (required; MOE_ERR_INVALID_ARG if NULL).
 *  Every other argument as in moe_route; `logits` holds x W_r + bias (the
 *  selection bias is not added to it).
 */
MOE_API moe_status moe_route_selection_bias(const moe_shape* shape, const void* x,
                                            const void* packed, const float* bias,
                                            const float* selection_bias, float* logits,
                                            int32_t* topk_idx, float* topk_gate, void* ws,
                                            size_t ws_bytes, moe_stream_t stream);

/*
 * Router statistics (moe_router_counts), written to device memory by
 * moe_router_stats.  They
 * are the quantities "MoE Pretraining: Parallelism Layout Changes the Model,
 * Not Quality" recommends monitoring (Practical Implications: the near-tie
 * share of the router, and how a run's routing differs from a recorded
 * routing table; Finding 3: routing flips happen at near-ties).
 *  tokens           T
 *  near_tie_tokens  tokens whose routing margin is below the threshold
 *  changed_tokens   tokens with at least one expert not in the recorded row
 *  changed_experts  sum over tokens of the number of distinct experts of
 *                   topk_idx[t] missing from recorded[t]
 *  changed_slots    entries (t, j) with topk_idx[t,j] != recorded[t,j]
 * (the last three are 0 when no recorded routing is given)
 */
typedef struct {
  int64_t tokens;
  int64_t near_tie_tokens;
  int64_t changed_tokens;
  int64_t changed_experts;
  int64_t changed_slots;
} moe_router_counts;

/*
 * Routing margin and router statistics ("MoE Pretraining: Parallelism
 * Layout Changes the Model, Not Quality", Finding 3 and Practical
 * Implications).  For each token, with s = its logits (+ selection_bias, the
 * fp32 sum moe_route_selection_bias selects on):
 *   margin[t] = (s_(k) - s_(k+1)) / (max_e s - min_e s)
 * where s_(r) is the r-th largest value, computed in double from the fp32
 * values; +inf when k == E, 0 when every value is equal.  A token is a
 * near-tie when margin[t] < threshold.
 *  logits         [T, E] fp32 (device), as moe_route writes it
 *  selection_bias [E] fp32 or NULL
 *  topk_idx       [T, k] int32, the routing to compare (may be NULL when
 *                 recorded_idx is NULL)
 *  recorded_idx   [T, k] int32 recorded routing table, or NULL
 *  threshold      >= 0 (1e-5 is the near-tie bound of the parity tests)
 *  margin         [T] double output, or NULL
 *  stats          one moe_router_counts in device memory (8-byte aligned),
 *                 overwritten
 */
MOE_API moe_status moe_router_stats(const moe_shape* shape, const float* logits,
                                    const float* selection_bias, const int32_t* topk_idx,
                                    const int32_t* recorded_idx, double threshold, double* margin,
                                    moe_router_counts* stats, moe_stream_t stream);

/*
 * Expert capacity ("Revisiting MoE and Dense Speed-Accuracy Comparisons for
 * LLM Training", 2.1: top-2 routing with an expert capacity factor).  Each
 * expert takes at most
 *   capacity = ceil(capacity_factor * T * k / E)
 * assignments (the factor times an expert's mean load).  The page gives no
 * drop order; the one taken here: every token's first choice is served
 * before any token's second choice, and so on (choice rank ascending),
 * tokens in index order within a rank; an assignment is kept while its
 * expert has taken fewer than `capacity`.
 *  topk_idx   [T, k] int32 (device)
 *  topk_gate  [T, k] fp32 or NULL (unit gates)
 *  keep       [T, k] int32 output: 1 kept, 0 dropped
 *  kept_gate  [T, k] fp32 output or NULL: the gate where kept, 0 where
 *             dropped; moe_forward_routed with these gates gives the layer
 *             output with the dropped assignments removed (a dropped
 *             assignment adds nothing and its gate is not redistributed)
 *  capacity   host int64 output or NULL: the per-expert capacity
 *  ws         scratch workspace (moe_scratch_size), for device errors
 * capacity_factor must be > 0.  An index outside [0, E) sets
 * MOE_ERR_DEVICE_INDEX; its keep / kept_gate entries read 0.
 */
MOE_API moe_status moe_capacity_keep(const moe_shape* shape, const int32_t* topk_idx,
                                     const float* topk_gate, double capacity_factor,
                                     int32_t* keep, float* kept_gate, int64_t* capacity,
                                     void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Expert-grouped dispatch layout and the deduplicated per-rank send layout
 * (see moe_layout).  Defined by: [Coupling] Abstract (each token is sent to
 * each GPU that holds one of its experts once), Table I (GPUs per token,
 * deduplicated rows), Table III (expert -> GPU placement).  Block-level histograms plus a decoupled-lookback scan
 * across blocks, then a stable scatter.
 *  topk_idx         [T, k] int32, device
 *  expert_rank_host [E] int32 in HOST memory: rank owning each expert; NULL
 *                   means contiguous placement e -> e / (E/ep).  Must be a
 *                   partition: every rank owns exactly E/ep experts
 *                   (MOE_ERR_INVALID_ARG otherwise).
 *  ws, ws_bytes     scratch workspace (moe_scratch_size)
 * An index outside [0, E) sets MOE_ERR_DEVICE_INDEX in the device status.
 */
MOE_API moe_status moe_dispatch_layout(const moe_shape* shape, const int32_t* topk_idx,
                               const int32_t* expert_rank_host,
                               const moe_layout* out, void* ws, size_t ws_bytes,
                               moe_stream_t stream);

/*
 * Co-selection counts of a routing ("Expert Coupling in MoE Pretraining",
 * Table III: W[e,e'], how often experts e and e' are selected by the same
 * token; the statistic its correlated placement is fit on):
 *   counts[e * E + e'] = number of ordered slot pairs (j, j'), j != j', of a
 *                        token with topk_idx[t,j] = e and topk_idx[t,j'] = e'
 * which, for a routing of distinct experts, is the number of tokens that
 * select both.  Integer counts, identical on every run.
 *  topk_idx [T, k] int32 (device); counts [E * E] uint64 (device, 8-byte
 *  aligned, overwritten); ws scratch workspace (moe_scratch_size).  A token
 *  with an index outside [0, E) adds nothing and sets MOE_ERR_DEVICE_INDEX.
 */
MOE_API moe_status moe_coselection_counts(const moe_shape* shape, const int32_t* topk_idx,
                                          uint64_t* counts, void* ws, size_t ws_bytes,
                                          moe_stream_t stream);

/*
 * Correlated expert placement fit on co-selection counts ("Expert Coupling
 * in MoE Pretraining", Abstract: experts often selected together are placed
 * on the same GPU; Table I caption: fit on other iterations than those it is
 * measured on).  Host code, no GPU: rank r = 0, 1, ... in turn takes the
 * unassigned expert with the largest row sum of counts, then, until it holds
 * E/ep experts, the unassigned expert with the largest total count with the
 * experts the rank already holds (ties: the lowest expert index).
 *  counts_host      [E * E] uint64 in HOST memory (moe_coselection_counts,
 *                   copied back)
 *  expert_rank_host [E] int32 HOST output: a partition with E/ep experts per
 *                   rank, ready for moe_dispatch_layout / moe_forward
 */
MOE_API moe_status moe_fit_placement(int32_t E, int32_t ep, const uint64_t* counts_host,
                                     int32_t* expert_rank_host);

/*
 * Permute (gather): x_perm[r] = x[row_token[r]] for r < T*k, whole rows
 * (the dispatch of token rows to their experts, [Coupling] Abstract),
 * moved by TMA bulk copies staged through shared memory (rows over 1 KB) or
 * by register copies (shorter rows).
 *  x [T, d], x_perm [T*k, d] (dtype); row_token [T*k] int32.
 * A row_token entry outside [0, T) is read as 0 (wrong values, no access
 * outside x); moe_dispatch_layout never produces one.
 */
MOE_API moe_status moe_permute(const moe_shape* shape, const void* x,
                       const int32_t* row_token, void* x_perm,
                       moe_stream_t stream);

/*
 * The same permute done in token order: x row t is read once and written to
 * its k rows x_perm[slot_row[t*k + j]] (slot_row [T*k] from
 * moe_dispatch_layout).  Equal output to moe_permute; it moves |x| + |x_perm|
 * bytes through DRAM even when x is much larger than L2, where the gather
 * re-reads each row of x once per expert that picks it.
 * A slot_row entry outside [0, T*k) is read as 0 (no access outside x_perm).
 */
MOE_API moe_status moe_permute_by_token(const moe_shape* shape, const void* x,
                                        const int32_t* slot_row, void* x_perm,
                                        moe_stream_t stream);

/*
 * Grouped SwiGLU experts over the expert-grouped rows ([Revisiting] 2.1
 * Architecture: SwiGLU experts; Table 1: FFN1 "EMH", FFN2 "EHM" layouts):
 *  h[r]      = silu(x_perm[r] W_g[e]) * (x_perm[r] W_u[e])   [T*k, f]
 *  y_perm[r] = h[r] W_d[e]                                   [T*k, d]
 * for expert e owning row r (expert_offsets [E+1], device, as produced by
 * moe_dispatch_layout).  bf16: tcgen05 tensor cores, fp32 accumulation in
 * tensor memory, h and y_perm rounded to bf16.  fp32: CUDA-core FMA.
 * Offsets are clamped to [0, T*k] and a negative group size counts as
 * empty, so a malformed offset array gives wrong rows but no access outside
 * x_perm, h or y_perm.
 *  ws, ws_bytes  scratch workspace (moe_scratch_size)
 */
MOE_API moe_status moe_grouped_swiglu(const moe_shape* shape, const void* x_perm,
                              const int32_t* expert_offsets, const void* packed,
                              void* h, void* y_perm, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/*
 * The permute fused into the grouped SwiGLU experts (bf16 only): the same
 * h and y_perm as moe_permute followed by moe_grouped_swiglu, but the
 * gate/up GEMM copies row r of its operand straight from x[row_token[r]]
 * into shared memory (cp.async, 16 bytes per lane), so x_perm is never
 * written or read.
 *  x [T, d]; row_token [T*k] (moe_dispatch_layout); other arguments as in
 *  moe_grouped_swiglu.  MOE_ERR_UNSUPPORTED for fp32.  A row_token entry
 *  outside [0, T) is read as 0.
 */
MOE_API moe_status moe_grouped_swiglu_gather(const moe_shape* shape, const void* x,
                                             const int32_t* row_token,
                                             const int32_t* expert_offsets,
                                             const void* packed, void* h, void* y_perm,
                                             void* ws, size_t ws_bytes,
                                             moe_stream_t stream);

/*
 * Gate-weighted combine (un-permute): each token's output is its k experts'
 * outputs weighted by its gates ([Revisiting] 2.1: Top-K routing;
 * [Layout] Models and Data):
 *   y[t] = sum_{j<k} gate[t,j] * y_perm[slot_row[t*k+j]]
 * summed in fp32 in ascending j, rounded once to the dtype.
 *  y_perm [T*k, d]; slot_row [T*k] int32; topk_gate [T, k] fp32 or NULL for
 *  unit gates; y [T, d].  A slot_row entry outside [0, T*k) is read as 0.
 */
MOE_API moe_status moe_combine(const moe_shape* shape, const void* y_perm,
                       const int32_t* slot_row, const float* topk_gate,
                       void* y, moe_stream_t stream);

/*
 * Optional caller-owned buffers of moe_forward's intermediates (device).
 * Any NULL member is placed in the workspace instead; pass NULL for the
 * whole struct to keep everything in the workspace.  After the call logits,
 * routing, layout and y_perm hold their values; x_perm and h are written
 * only by the paths that materialise them (x_perm: x above 96 MB or fp32;
 * h: the unfused expert GEMMs) and are otherwise left untouched.
 */
typedef struct {
  float* logits;      /* [T, E] */
  int32_t* topk_idx;  /* [T, k] */
  float* topk_gate;   /* [T, k] */
  moe_layout layout;  /* as moe_dispatch_layout */
  void* x_perm;       /* [T*k, d] */
  void* h;            /* [T*k, f] */
  void* y_perm;       /* [T*k, d] */
} moe_forward_buffers;

/*
 * The whole layer enqueued back to back on `stream`, with no host
 * synchronisation in between (the steps and their sources as in the entry
 * points above: [Layout] Models and Data, [Revisiting] 2.1, [Coupling]
 * Abstract).  bf16: one kernel for router GEMM + top-k +
 * gates + the per-tile dispatch histogram, the layout scatter, then the
 * expert FFN: for f in {64, 128} and d in {128, 256} one kernel for the
 * gate/up GEMM, SwiGLU (H kept on chip) and down GEMM (same arithmetic as
 * the separate GEMMs, so the same y_perm), otherwise the gate/up GEMM with
 * SwiGLU and the down GEMM; then the combine.  The permute is
 * fused into the gate/up operand load (as moe_grouped_swiglu_gather, x_perm
 * not written) while x is at most 96 MB, and a separate token-order permute
 * (moe_permute_by_token) runs otherwise.  fp32: moe_route,
 * moe_dispatch_layout, moe_permute, moe_grouped_swiglu and moe_combine in
 * turn.
 *  x [T, d]; packed weights; bias [E] or NULL; expert_rank_host as in
 *  moe_dispatch_layout; y [T, d]; buffers may be NULL;
 *  ws, ws_bytes  moe_forward_workspace_size bytes.
 */
MOE_API moe_status moe_forward(const moe_shape* shape, const void* x, const void* packed,
                       const float* bias, const int32_t* expert_rank_host,
                       void* y, const moe_forward_buffers* buffers, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/*
 * moe_forward with the router of moe_route_selection_bias: experts chosen on
 * logits + selection_bias, gates from the logits alone; the dispatch layout,
 * experts and combine follow that routing.  Same kernels as moe_forward.
 *  selection_bias [E] fp32, device (required).  Other arguments as in
 *  moe_forward.
 */
MOE_API moe_status moe_forward_selection_bias(const moe_shape* shape, const void* x,
                                              const void* packed, const float* bias,
                                              const float* selection_bias,
                                              const int32_t* expert_rank_host, void* y,
                                              const moe_forward_buffers* buffers, void* ws,
                                              size_t ws_bytes, moe_stream_t stream);

typedef struct CUevent_st* moe_event_t; /* same type as cudaEvent_t */
#define MOE_FORWARD_STAGES 6

/*
 * moe_forward that also records events[i] on `stream` just before stage i
 * (0 route, 1 dispatch layout, 2 permute, 3 gate/up GEMM, 4 down GEMM,
 * 5 combine) and events[6] after the last, so cudaEventElapsedTime between
 * neighbours gives each stage's device time inside the forward.  A stage
 * that a path fuses into another has no work between its two events.
 * events: MOE_FORWARD_STAGES + 1 caller-created events.
 */
MOE_API moe_status moe_forward_timed(const moe_shape* shape, const void* x,
                                     const void* packed, const float* bias,
                                     const int32_t* expert_rank_host, void* y,
                                     const moe_forward_buffers* buffers, void* ws,
                                     size_t ws_bytes, moe_event_t* events,
                                     moe_stream_t stream);

/*
 * The layer below the router on a routing the caller supplies: the
 * dispatch layout of topk_idx, then permute, expert FFN and combine with
 * topk_gate, as in moe_forward (same kernels, same results for the same
 * routing).  It replays a recorded routing table, which applications that
 * depend on specific experts need once routing is not reproducible ("MoE
 * Pretraining: Parallelism Layout Changes the Model, Not Quality",
 * Practical Implications: routing replay).  No logits are computed and the
 * router block of `packed` is not read.
 *  topk_idx [T, k] int32 (device): experts in [0, E); an entry outside
 *    that range sets MOE_ERR_DEVICE_INDEX in the device status word, as in
 *    moe_dispatch_layout.
 *  topk_gate [T, k] fp32 (device) or NULL for unit gates.
 *  Other arguments as in moe_forward; the logits, topk_idx and topk_gate
 *  members of `buffers` are not used.
 */
MOE_API moe_status moe_forward_routed(const moe_shape* shape, const void* x,
                                      const void* packed, const int32_t* topk_idx,
                                      const float* topk_gate,
                                      const int32_t* expert_rank_host, void* y,
                                      const moe_forward_buffers* buffers, void* ws,
                                      size_t ws_bytes, moe_stream_t stream);

/*
 * Expert parallelism: the layer over P = shape->ep ranks (GPUs), tokens split
 * over the ranks and the E experts placed on them by the expert -> rank map,
 * with the deduplicated dispatch of "Expert Coupling in MoE Pretraining"
 * (Abstract: each token is sent to each GPU that holds one of its experts
 * once; Table I: GPUs per token and the rows deduplication removes; Fig. 7:
 * baseline vs deduplicated dispatch).  One rank's forward:
 *   moe_route, moe_dispatch_layout (ep = P)   the send plan of its tokens
 *   moe_ep_pack                                its send rows
 *   (exchange: rank_counts of every rank, then the send rows all-to-all;
 *    the rows for rank r are rows [rank_offsets[r], rank_offsets[r+1]))
 *   moe_ep_expert_forward                      one return row per received row
 *   (reverse exchange of the return rows)
 *   moe_ep_home_combine                        y of its tokens
 * The exchange is the caller's (NCCL all-to-all, peer copies, ...): the
 * library moves no bytes between GPUs.
 */

/*
 * Send rows of one rank, grouped by destination rank (send row s goes to
 * the rank r with rank_offsets[r] <= s < rank_offsets[r+1]):
 *   send_x   [send_rows, d]  x[send_token[s]]
 *   send_idx [send_rows, k]  the token's k experts as the destination's
 *                            local expert ids (the expert's position among
 *                            that rank's experts, ascending), or E/P for an
 *                            expert another rank holds
 *   send_gate[send_rows, k]  the token's k gates (1 when topk_gate is NULL)
 *  shape: T local tokens, ep = P >= 2; topk_idx / topk_gate [T, k] (device);
 *  expert_rank_host as in moe_dispatch_layout; layout: the slot_send_row
 *  and rank_offsets of moe_dispatch_layout on the same routing and map;
 *  send_rows: rows the send buffers hold (rank_offsets[P], read back, or
 *  any bound; rows s >= send_rows are not written).  Each token's x row is
 *  read once and stored into each of its send rows.
 */
MOE_API moe_status moe_ep_pack(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                               const float* topk_gate, const int32_t* expert_rank_host,
                               const moe_layout* layout, void* send_x, int32_t* send_idx,
                               float* send_gate, int64_t send_rows, moe_stream_t stream);

/*
 * Workspace of moe_ep_expert_forward for shape (T = rows this rank
 * received, ep = P): layout scratch and the expert-grouped intermediates.
 */
MOE_API moe_status moe_ep_expert_workspace_size(const moe_shape* shape, size_t* bytes);

/*
 * The receiving rank's experts: the received rows' assignments to its E/P
 * experts are laid out by local expert (a stable counting sort, the slots
 * of other ranks' experts set aside), run through the grouped SwiGLU
 * experts, and each received row's return row is the gated sum of its
 * local experts' outputs:
 *   y_ret[i] = sum_{j : recv_idx[i,j] < E/P} recv_gate[i,j] * expert_{recv_idx[i,j]}(recv_x[i])
 * summed in fp32 in ascending j, rounded once to the dtype.
 *  shape: T = received rows, E = all experts, ep = P; recv_x [T, d],
 *  recv_idx [T, k], recv_gate [T, k] (the moe_ep_pack rows of every source
 *  rank, in any order); packed_local: moe_pack_weights output for a shape
 *  with E/P experts (this rank's experts, ascending); y_ret [T, d];
 *  ws, ws_bytes: moe_ep_expert_workspace_size bytes, zero-filled once (its
 *  device status word is read with moe_get_device_status).
 */
MOE_API moe_status moe_ep_expert_forward(const moe_shape* shape, const void* recv_x,
                                         const int32_t* recv_idx, const float* recv_gate,
                                         const void* packed_local, void* y_ret, void* ws,
                                         size_t ws_bytes, moe_stream_t stream);

/*
 * The home rank's output: y[t] = sum over the distinct send rows of token t
 * (one per destination rank, taken in slot order) of y_back[row], in fp32,
 * rounded once; y_back [send_rows, d] holds the return rows in send-row
 * order, slot_send_row [T, k] is moe_dispatch_layout's.
 */
MOE_API moe_status moe_ep_home_combine(const moe_shape* shape, const void* y_back,
                                       const int32_t* slot_send_row, int64_t send_rows, void* y,
                                       moe_stream_t stream);

/*
 * Peer-memory exchange: the pack fused with the dispatch all-to-all, and the
 * experts' return rows fused with the reverse one.  Each kernel stores its
 * rows straight into the other ranks' buffers, which the caller has mapped
 * into this process (this GPU's own memory, or another GPU's over NVLink
 * through a peer mapping: CUDA IPC, a symmetric-memory allocation, a
 * cudaDeviceEnablePeerAccess'd allocation).  Plain 16-byte stores only:
 * nothing reads a peer's memory.  The rows, their order within each block
 * and every value are those of moe_ep_pack + all-to-all and
 * moe_ep_expert_forward + reverse all-to-all; only where the bytes are
 * written changes.  Rank order of the blocks: source rank s's rows at rank
 * r start at row sum_{s' < s} counts[s'][r] of r's receive buffers (counts
 * = every rank's rank_counts, exchanged first), and return rows go back to
 * the send-row position they left from.
 * Between the phases every rank must have finished storing before any
 * rank reads: moe_ep_signal_wait on each rank (or a host barrier after a
 * stream synchronisation).
 */
typedef struct moe_ep_peer_dest {
  void* recv_x;       /* rank r's receive rows [.., d] (dtype) */
  int32_t* recv_idx;  /* rank r's receive local expert ids [.., k] */
  float* recv_gate;   /* rank r's receive gates [.., k] */
  int64_t row0;       /* first row of this rank's block there */
  int64_t rows;       /* rows of the block: rank_counts[r] of this rank */
} moe_ep_peer_dest;

/*
 * moe_ep_pack whose send rows for rank r (rows rank_offsets[r] ..
 * rank_offsets[r+1] of the send plan) are stored at rows dests_host[r].row0 ..
 * of rank r's receive buffers.  dests_host: P entries (host); a block of 0
 * rows needs no buffers.  Send rows past dests_host[r].rows are not stored
 * (size rows from the exchanged counts).  Other arguments as moe_ep_pack.
 */
MOE_API moe_status moe_ep_dispatch_peer(const moe_shape* shape, const void* x,
                                        const int32_t* topk_idx, const float* topk_gate,
                                        const int32_t* expert_rank_host,
                                        const moe_layout* layout,
                                        const moe_ep_peer_dest* dests_host, moe_stream_t stream);

typedef struct moe_ep_peer_return {
  void* y_back;  /* source rank s's return rows [.., d] (its send-row order) */
  int64_t row0;  /* where this rank's rows start there: rank_offsets[me] of s */
  int64_t rows;  /* rows this rank received from s: counts[s][me] */
} moe_ep_peer_return;

/*
 * moe_ep_expert_forward whose return rows go straight back: the received
 * rows are the blocks of the source ranks in rank order (rets_host[s].rows
 * rows each, summing to shape->T), and return row i of source s's block is
 * stored at row rets_host[s].row0 + i of s's y_back.  Invalid argument when
 * the blocks do not sum to shape->T.  Other arguments as
 * moe_ep_expert_forward.
 */
MOE_API moe_status moe_ep_expert_forward_peer(const moe_shape* shape, const void* recv_x,
                                              const int32_t* recv_idx, const float* recv_gate,
                                              const void* packed_local,
                                              const moe_ep_peer_return* rets_host, void* ws,
                                              size_t ws_bytes, moe_stream_t stream);

/*
 * The ranks' rendezvous on device: one kernel stores `epoch` into slot
 * `rank` of every rank's flag array (a system-scope release after all
 * earlier work of `stream`, so this rank's stores into peers' buffers are
 * visible first) and waits until every slot of its own array holds at least
 * `epoch` (system-scope acquire).  flags_host: P device pointers (host
 * array), each rank's array of P uint64 slots, zero-filled before the first
 * epoch; epochs start at 1 and grow by one per rendezvous.  The wait gives
 * up after one second and records MOE_ERR_DEVICE_TIMEOUT (detail: the first
 * rank missing) in the control block of `ws` (any workspace of this
 * library; read with moe_get_device_status).  Every rank must call it once
 * per epoch on its own GPU: kernels that wait for one another must run on
 * different GPUs at the same time.
 * No counterpart in the pages, which leave the exchange to the library
 * they run on.
 */
MOE_API moe_status moe_ep_signal_wait(uint64_t* const* flags_host, int32_t rank, int32_t P,
                                      uint64_t epoch, void* ws, moe_stream_t stream);

/*
 * Test hook: moe_ep_signal_wait with the wait limited to wait_limit_ns
 * (0 < wait_limit_ns <= one second).
 */
MOE_API moe_status moe_debug_ep_signal_wait(uint64_t* const* flags_host, int32_t rank,
                                            int32_t P, uint64_t epoch, void* ws,
                                            int64_t wait_limit_ns, moe_stream_t stream);

/*
 * Synchronise `stream`, read the device status word of workspace `ws`
 * (MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_INDEX) into *out and
 * reset it to MOE_OK.  Returns MOE_ERR_CUDA if the stream reports an error.
 */
MOE_API moe_status moe_get_device_status(void* ws, moe_stream_t stream, moe_status* out);

/*
 * Test hook for the bounded wait of moe_dispatch_layout's decoupled lookback:
 * identical to moe_dispatch_layout, except that the block holding lookback
 * ticket `stall_block` never publishes its histogram, and the waits give up
 * after `wait_limit_ns` nanoseconds (production calls use one second).
 * The call then reports MOE_ERR_DEVICE_TIMEOUT through the device status, the
 * layout outputs are unspecified, and the context stays usable.
 */
MOE_API moe_status moe_debug_dispatch_layout_stall(const moe_shape* shape,
                                           const int32_t* topk_idx,
                                           const int32_t* expert_rank_host,
                                           const moe_layout* out, void* ws,
                                           size_t ws_bytes, int32_t stall_block,
                                           int64_t wait_limit_ns,
                                           moe_stream_t stream);

/*
 * Test and measurement hook of moe_grouped_swiglu (row_token NULL: a_rows
 * is x_perm) and moe_grouped_swiglu_gather (row_token given: a_rows is x):
 * the same call with the tensor-core GEMM engine chosen by the caller.
 *  engine 0  the library's choice (what those calls run)
 *         1  one CTA per 128-row tile for both GEMMs (the gather by
 *            cp.async)
 *         2  CTA pairs on 256-row tiles (tcgen05 cta_group::2; the gather
 *            by TMA gather4) for both GEMMs where the shape allows it (bf16,
 *            256-column tiles), else as 1
 *         3  CTA pairs for the down GEMM only
 *         4  CTA pairs for the gate/up GEMM only
 * All engines sum every output in the same order, so h and y_perm are
 * bit-identical across engines.  MOE_ERR_INVALID_ARG for another engine.
 */
MOE_API moe_status moe_debug_grouped_swiglu_engine(const moe_shape* shape, const void* a_rows,
                                                   const int32_t* row_token,
                                                   const int32_t* expert_offsets,
                                                   const void* packed, void* h, void* y_perm,
                                                   void* ws, size_t ws_bytes, int32_t engine,
                                                   moe_stream_t stream);

/*
 * Test and measurement hook: moe_forward with options.
 *   MOE_FWD_COMBINE_IN_DOWN  the combine summed in the down GEMM's epilogue
 *     where that GEMM runs on CTA pairs (bf16, d % 256 == 0, f >= 1024;
 *     ignored elsewhere): after a tile's rows are stored, a per-(token,
 *     64-column block) arrival counter is incremented, and the last of a
 *     token's k arrivals sums the token's k rows of y_perm in slot order
 *     (fp32, gate-weighted, rounded once: the combine kernel's arithmetic,
 *     so y is bit-identical).  Measured slower than the separate combine on
 *     the large workload, so moe_forward does not use it.
 * Other bits: MOE_ERR_INVALID_ARG.  Arguments otherwise as moe_forward.
 */
#define MOE_FWD_COMBINE_IN_DOWN 1
MOE_API moe_status moe_debug_forward_options(const moe_shape* shape, const void* x,
                                             const void* packed, const float* bias,
                                             const int32_t* expert_rank_host, void* y,
                                             const moe_forward_buffers* buffers, void* ws,
                                             size_t ws_bytes, int32_t options,
                                             moe_stream_t stream);

/*
 * moe_dispatch_layout for callers that cannot allocate device memory.
 * The source pages have no counterpart of this call; it exists for callers
 * that may not call cudaMalloc or any other allocator where they call this
 * library (an operator inside a framework whose device memory is planned
 * ahead and which receives only its inputs and outputs, or a C caller with
 * no device allocator), and therefore cannot pass the workspace that
 * moe_dispatch_layout needs.
 *
 * Same inputs and outputs as moe_dispatch_layout, but no workspace: the
 * scratch lives in a 1 MiB array inside this library, one per GPU, held
 * from when the library's device code is loaded until the process exits.
 * Nothing is allocated and nothing is freed by this call.
 *  - Shapes whose scratch exceeds 1 MiB are rejected with MOE_ERR_WORKSPACE
 *    (the scratch is 4352 B + 8 B * ceil(T/128) * bins, the second part
 *    rounded up to 256 B, with bins = E + (ep > 1 ? ep : 0) + 2; e.g.
 *    E=64, ep=8 fits up to about 225k tokens, E=256, ep=256 about 32k).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before capturing any stream on that device.
 *  - Every call on a device shares the one array, and it keeps the previous
 *    call's contents: each call first clears the part that must start at
 *    zero (on `stream`).  Calls whose work overlaps on the GPU (different
 *    streams or threads at the same time on one device) race on the array
 *    and give wrong layouts; order them on one stream.
 *  - device_status: optional device int32 that receives this call's device
 *    status (MOE_OK, MOE_ERR_DEVICE_INDEX or MOE_ERR_DEVICE_TIMEOUT) when
 *    the layout kernels finish; NULL to skip.
 */
MOE_API moe_status moe_dispatch_layout_static(const moe_shape* shape,
                                              const int32_t* topk_idx,
                                              const int32_t* expert_rank_host,
                                              const moe_layout* out,
                                              int32_t* device_status,
                                              moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
