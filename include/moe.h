/*
 * moe.h - C ABI of the B200 (sm_100a) sparse noisy top-k Mixture-of-Experts
 * layer forward pass (libmoe.so).
 *
 * The layer, as the MoE pages define it:
 *   "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 1-12 and
 *   "nanoMoEの深層解剖" slides 11-40 (Router, MLPExperts, MOELayer):
 *     s_raw = W_g x (+ b_g)                      router logits, fp32
 *     s     = s_raw + sigma * eps                noise, eps supplied ~ N(0,1)
 *     keep the k largest s, -inf elsewhere       KeepTopK
 *     g     = softmax over the kept scores       gates
 *     capacity-limited dispatch (first choices of all tokens ranked before
 *       second choices, tokens in order; places >= C dropped)
 *     E_e(x) = W_down[e] ReLU(W_up[e] x)         expert FFN
 *     y     = sum over kept choices of g * E_e(x)
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers marked "device" are device memory owned by the caller; the
 *    library never allocates, frees or keeps them after the call returns.
 *  - Scratch memory comes from a caller-provided workspace whose size the
 *    matching *_workspace_size call returns (256-byte aligned start).
 *  - Every compute call is asynchronous on the caller's CUDA stream
 *    (cudaStream_t passed as void*; NULL is the legacy default stream).
 *  - Arrays are dense and row-major.  Every array must start on a 16-byte
 *    boundary.
 *  - moe_dtype selects the storage type of x, W_up, W_down, the gathered
 *    buffers and y.  W_g, b_g, noise, logits and gates are always fp32;
 *    index arrays are int32.
 *  - Return value: MOE_OK, or an error code with a message available from
 *    moe_last_error() (thread-local, valid until the next call on that
 *    thread).  Argument errors are detected on the host before anything is
 *    launched.  Kernel-side failures (a bounded wait that ran out, an index
 *    check) are recorded in a status word and returned by moe_check_status()
 *    (or moe_check_route_status() for moe_route).  No kernel traps.
 *  - The status word is the first 4 bytes of a workspace (or the word given to
 *    moe_route_ex).  Kernels only OR error bits into it; nothing but
 *    moe_check_status() clears it, so an error stays visible through any
 *    number of later calls until the caller reads it.  A fresh workspace's
 *    first 4 bytes must be zeroed once before its first use (cudaMemset, or a
 *    moe_check_status() call, which reads and then clears the word).
 *  - Preconditions: 1 <= k <= E <= 256; N >= 0; d, d_ff >= 1; inputs finite
 *    (NaN or Inf in the scores gives unspecified routing).
 *  - Ties in the top-k go to the lower expert index; the k kept experts of a
 *    token are listed in (score descending, index ascending) order, which
 *    defines the first, second, ... choice for capacity priority.
 */
#ifndef MOE_H_
#define MOE_H_

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

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Expert activation: ReLU (the walkthrough's STEP 9) or GELU, x * Phi(x) with
 * Phi the standard normal CDF (nanoMoE's MLPExperts, "nanoMoEの深層解剖" slide 32). */
typedef enum { MOE_ACT_RELU = 1, MOE_ACT_GELU = 2 } moe_activation;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad size, null required pointer, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2,   /* valid arguments this build cannot run */
    MOE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    MOE_ERR_DEVICE_CHECK = 5,  /* a kernel's own index check failed */
    MOE_ERR_TIMEOUT = 6        /* a kernel's bounded wait ran out */
} moe_status;

/* Expert capacity C = min(N, ceil(cf * N * k / E)) computed in double
 * ("nanoMoEの深層解剖" slide 14, get_capacity; the pages do not print its body,
 * this is the problem statement's formula).  cf = +INFINITY means no limit
 * (C = N).  Returns -1 if cf <= 0, cf is NaN, N < 0 or k, E are out of range. */
MOE_API int64_t moe_capacity(int64_t N, int E, int k, double cf);

/* Rows of the gathered (expert-major) buffers: min(N * k, E * C) rounded up
 * to a multiple of 128.  x_gathered and out_gathered hold this many rows.
 * Returns -1 on invalid arguments. */
MOE_API int64_t moe_gathered_rows(int64_t N, int E, int k, double cf);

/* ---------------------------------------------------------------- router */

/* Router: logits, optional noise, KeepTopK and softmax over the kept scores.
 * ("Mixture of Experts (MoE) 12段階…" STEP 2-6; "nanoMoEの深層解剖" slides 11-13.)
 *
 *  x          device [N, d] of dt
 *  W_g        device [E, d] fp32            router weights, one row per expert
 *  b_g        device [E] fp32 or NULL       router bias added in fp32 to W_g x
 *  noise      device [N, E] fp32 or NULL    eps ~ N(0,1); skipped if NULL or sigma == 0
 *  sigma      noise scale; s = fl32(s_raw + fl32(sigma * eps)) (two roundings, no FMA)
 *  logits_out device [N, E] fp32 or NULL    receives s_raw (bias included, before noise)
 *  topk_idx   device [N, k] int32           kept experts, first choice first
 *  gates      device [N, k] fp32            softmax of the kept scores, same order
 * The dot products accumulate in fp32.  bf16 tokens (d a multiple of 8,
 * E <= 160, k <= 32) run them on the tensor cores with each fp32 weight split
 * exactly into three bf16 parts, so every product is exact and only the fp32
 * accumulation rounds; other shapes run on CUDA cores.  Either way the top-k
 * and softmax are the same given the logits, and a token's results do not
 * depend on N or on its position in the batch.
 *
 * Every wait in the tensor-core router is bounded (1 s).  If one runs out, the
 * kernel writes expert -1 and gate 0 for the tokens it could not finish and
 * records MOE_ERR_TIMEOUT: moe_route in the library's own per-device status
 * word, read and cleared by moe_check_route_status(); moe_route_ex in the
 * caller's word.  Concurrent moe_route calls share the library's word, so a
 * caller that needs per-call attribution uses moe_route_ex. */
MOE_API moe_status moe_route(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                     const float *noise, float sigma, int64_t N, int d, int E, int k,
                     float *logits_out, int32_t *topk_idx, float *gates, void *stream);

/* Workspace bytes with which moe_route_ex takes moe_forward's router path. */
MOE_API size_t moe_route_workspace_size(int d, int E);

/* moe_route with a caller workspace.  ws (device, 16-byte aligned, nullable):
 *  - NULL: exactly moe_route (the library's status word);
 *  - ws_bytes >= 256: its first 4 bytes are the status word (zero before first
 *    use), read and cleared by moe_check_status(ws, ...);
 *  - ws_bytes >= moe_route_workspace_size(d, E), bf16 tokens: on batches that
 *    take the router's persistent form (many tokens), the router weights are
 *    also split into ws first and read from there, as in moe_forward; smaller
 *    batches split them in-kernel.  Same results either way. */
MOE_API moe_status moe_route_ex(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                                const float *noise, float sigma, int64_t N, int d, int E, int k,
                                float *logits_out, int32_t *topk_idx, float *gates, void *ws, size_t ws_bytes,
                                void *stream);

/* Synchronises `stream` after reading and clearing (on that stream) the
 * library's status word of moe_route calls on the current device.  Returns
 * MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_CHECK; *detail (nullable) receives
 * the raw word. */
MOE_API moe_status moe_check_route_status(void *stream, uint32_t *detail);

/* ---------------------------------------------------------------- dispatch */

/* Workspace bytes for moe_dispatch (per-block expert histograms). */
MOE_API size_t moe_dispatch_workspace_size(int64_t N, int E, int k);

/* Capacity-limited dispatch ("nanoMoEの深層解剖" slides 14-23, one_hot + cumsum
 * ranking with all first choices before all second choices, capacity cut;
 * slides 33-36 for the gathered expert batches).
 *
 *  topk_idx   device [N, k] int32 (from moe_route)
 *  x          device [N, d] of dt
 *  cf         capacity factor (see moe_capacity)
 *  slot       device [N, k] int32 out: place of (t, j) in expert topk_idx[t][j]'s
 *             queue, or -1 if dropped
 *  counts     device [E] int32 out: kept rows per expert (<= C)
 *  offsets    device [E + 1] int32 out: exclusive prefix sum of counts
 *  x_gathered device [moe_gathered_rows(), d] of dt out: row offsets[e] + slot
 *             holds x[t] for every kept (t, j) with topk_idx[t][j] = e.  Rows past
 *             offsets[E] are left unwritten.
 *  ws, ws_bytes  workspace, at least moe_dispatch_workspace_size() bytes
 * Results are deterministic (no atomics decide an order). */
MOE_API moe_status moe_dispatch(const int32_t *topk_idx, const void *x, moe_dtype dt, int64_t N, int d,
                        int E, int k, double cf, int32_t *slot, int32_t *counts,
                        int32_t *offsets, void *x_gathered, void *ws, size_t ws_bytes,
                        void *stream);

/* Dispatch without a caller workspace.  No counterpart in the pages: this is
 * for callers that cannot allocate device memory when they dispatch, such as a
 * host runtime that forbids cudaMalloc after start-up (a device allocation can
 * synchronise the GPU and stall the latency-critical path) or a plug-in whose
 * framework owns every byte of device memory and hands it no scratch.
 *
 * Same arguments, results and errors as moe_dispatch, minus ws/ws_bytes.  The
 * scratch (per-block histograms and totals) lives in one fixed 8 MiB device
 * array inside the library, which every GPU that loads the library holds until
 * the process exits; batches needing more (moe_dispatch_workspace_size() >
 * 8 MiB, i.e. about N * k * E > 2^29) get MOE_ERR_INVALID_ARG with a
 * message.  The call allocates nothing and calls no allocating routine.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) for that device, which loads the library's device
 *    code there if it is not loaded yet; make that first call before any
 *    stream capture on the device.  The address is kept per device and CUDA
 *    context: after cudaDeviceReset (a new context) the next call looks it up
 *    again, so make a first call again before capturing.
 *  - Every call shares the one array and leaves its contents behind; the
 *    passes overwrite every scratch entry they read, so nothing has to start
 *    at zero.
 *  - Calls whose kernels overlap on the GPU (other streams, other threads)
 *    race on the array: serialise them. */
MOE_API moe_status moe_dispatch_noalloc(const int32_t *topk_idx, const void *x, moe_dtype dt, int64_t N,
                                        int d, int E, int k, double cf, int32_t *slot, int32_t *counts,
                                        int32_t *offsets, void *x_gathered, void *stream);

/* ---------------------------------------------------------------- token-sharded batches */

/* One batch whose tokens are split over G GPUs in contiguous ranges, rank
 * order.  A queue place depends on every earlier token of the batch (all first
 * choices before all second choices, "nanoMoEの深層解剖" slides 17-20), so the
 * shards exchange their per-(choice, expert) counts once; everything else stays
 * on each GPU.  Per shard:
 *   moe_route                       (local tokens)
 *   moe_shard_count   -> counts_je  (this shard's [k][E] totals)
 *   all-gather counts_je over the G ranks (e.g. NCCL) into all_counts [G][k][E]
 *   moe_shard_base    -> base       (this shard's first place per (j, e))
 *   moe_shard_dispatch              (C = moe_capacity(N of the whole batch, ...))
 *   moe_expert_ffn, moe_combine     (unchanged, on the shard's rows)
 * The drop set equals the unsharded one; the combine output of every token is
 * the same as in an unsharded call.  `slot` here numbers each expert's kept
 * rows inside the shard (choice rank first, then token order).
 *
 * Workspace for the count/dispatch pair of one shard (the count pass leaves
 * per-block prefixes in it that the dispatch reads: give both calls the same
 * workspace and do not touch it in between). */
MOE_API size_t moe_shard_workspace_size(int64_t N_local, int E, int k);

/*  counts_je device [k][E] int32 out: this shard's number of j-th choices of e. */
MOE_API moe_status moe_shard_count(const int32_t *topk_idx, int64_t N_local, int E, int k, int32_t *counts_je,
                                   void *ws, size_t ws_bytes, void *stream);

/*  all_counts device [G][k][E] int32 (rank order); base device [k][E] int32 out:
 *  base[j][e] = sum over all shards of choices j' < j of e + sum over shards
 *  before `rank` of choice j of e. */
MOE_API moe_status moe_shard_base(const int32_t *all_counts, int G, int rank, int E, int k, int32_t *base,
                                  void *stream);

/*  As moe_dispatch for this shard's tokens, with C the whole batch's capacity,
 *  counts_je/ws from moe_shard_count and base from moe_shard_base.  x_gathered
 *  needs ceil(N_local * k / 128) * 128 rows. */
MOE_API moe_status moe_shard_dispatch(const int32_t *topk_idx, const void *x, moe_dtype dt, int64_t N_local,
                                      int d, int E, int k, int64_t C, const int32_t *counts_je,
                                      const int32_t *base, int32_t *slot, int32_t *counts, int32_t *offsets,
                                      void *x_gathered, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- experts */

/* Workspace bytes for moe_expert_ffn (status word + the hidden activations). */
MOE_API size_t moe_expert_ffn_workspace_size(int64_t rows, int d, int E, int d_ff, moe_dtype dt);

/* Expert FFN on the gathered rows ("Mixture of Experts (MoE) 12段階…" STEP 8-10;
 * "nanoMoEの深層解剖" slide 32, MLPExperts with ReLU in place of GELU):
 *   out[r] = W_down[e] ReLU(W_up[e] x_gathered[r])   for offsets[e] <= r < offsets[e] + counts[e]
 *
 *  x_gathered   device [rows, d] of dt
 *  offsets      device [E + 1] int32, counts device [E] int32 (from moe_dispatch)
 *  W_up         device [E, d_ff, d] of dt
 *  W_down       device [E, d, d_ff] of dt
 *  out_gathered device [rows, d] of dt; rows outside the kept ranges are unspecified
 *  rows         allocated rows of x_gathered/out_gathered (moe_gathered_rows())
 * bf16: tcgen05 tensor-core grouped GEMMs, fp32 accumulation, the hidden
 * activation rounded to bf16 after ReLU, out rounded to bf16.  Needs d and
 * d_ff multiples of 8; otherwise (and for fp32) CUDA-core fp32 kernels run.
 * Rows are read from device counts, so nothing waits on the host. */
MOE_API moe_status moe_expert_ffn(const void *x_gathered, const int32_t *offsets, const int32_t *counts,
                          const void *W_up, const void *W_down, moe_dtype dt, int64_t rows,
                          int d, int d_ff, int E, void *out_gathered, void *ws, size_t ws_bytes,
                          void *stream);

/* The nanoMoE expert variant ("nanoMoEの深層解剖" slide 32, MLPExperts):
 *   out[r] = W_down[e] act(W_up[e] x_gathered[r] + b_up[e]) + b_down[e]
 * activation: MOE_ACT_RELU or MOE_ACT_GELU (erf form); b_up device [E, d_ff]
 * fp32 and b_down device [E, d] fp32, each nullable.  Everything else as
 * moe_expert_ffn (which is this call with ReLU and no biases).  Dropout, which
 * the slides apply in training, is the identity in this forward pass. */
MOE_API moe_status moe_expert_ffn_ex(const void *x_gathered, const int32_t *offsets, const int32_t *counts,
                                     const void *W_up, const void *W_down, moe_dtype dt, int64_t rows, int d,
                                     int d_ff, int E, int activation, const float *b_up, const float *b_down,
                                     void *out_gathered, void *ws, size_t ws_bytes, void *stream);

/* The expert FFN of a training step: as moe_expert_ffn (ReLU, no biases), and
 * the hidden activations H [rows, d_ff] of dt (device, caller-owned) are kept
 * for moe_backward: H[r] = ReLU(W_up[e] x_gathered[r]) rounded to dt, rows
 * outside the kept ranges unspecified.  out_gathered is written in every plan
 * (the decode plan sums its K-split partials into it).  Same workspace as
 * moe_expert_ffn. */
MOE_API moe_status moe_expert_ffn_train(const void *x_gathered, const int32_t *offsets, const int32_t *counts,
                                        const void *W_up, const void *W_down, moe_dtype dt, int64_t rows, int d,
                                        int d_ff, int E, void *out_gathered, void *H, void *ws, size_t ws_bytes,
                                        void *stream);

/* ---------------------------------------------------------------- combine */

/* Gate-weighted combine back to token order ("Mixture of Experts (MoE) 12段階…"
 * STEP 11-12; "nanoMoEの深層解剖" slides 38-40):
 *   y[t] = sum over j with slot[t][j] >= 0 of gates[t][j] * out_gathered[offsets[e] + slot[t][j]]
 * accumulated in fp32 in j order; a token with every choice dropped gets a
 * zero row; gates are not renormalised after drops.
 *  y device [N, d] of dt. */
MOE_API moe_status moe_combine(const void *out_gathered, const int32_t *slot, const int32_t *topk_idx,
                       const int32_t *offsets, const float *gates, moe_dtype dt, int64_t N,
                       int d, int k, void *y, void *stream);

/* ---------------------------------------------------------------- load statistics */

/* Per-expert load of one routed batch ("nanoMoEの深層解剖" slide 14: the
 * router's used_capacity counts each expert's rows that survive the capacity
 * cut; STEP 4's noise exists to spread this load).  No gradient or loss form
 * is on the pages; these are the quantities a balancing loss would use.
 *  topk_idx   device [N, k] int32 (from moe_route); entries outside [0, E) are skipped
 *  gates      device [N, k] fp32 or NULL
 *  cf         capacity factor, as for moe_dispatch (C = moe_capacity(N, E, k, cf))
 *  load       device [E] int32 out: choices (t, j) that picked e, before the cut
 *  used       device [E] int32 out: min(load[e], C), equal to moe_dispatch's counts
 *  importance device [E] double out or NULL: the gates of load's choices summed,
 *             each gate rounded to the nearest multiple of 2^-32 (ties to even) and
 *             added exactly, so the result does not depend on the order of the adds
 *  ws, ws_bytes  workspace of at least moe_load_stats_workspace_size() bytes
 * E <= 256, N * k < 2^31.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_WORKSPACE, MOE_ERR_CUDA. */
MOE_API size_t moe_load_stats_workspace_size(void);
MOE_API moe_status moe_load_stats(const int32_t *topk_idx, const float *gates, int64_t N, int E, int k,
                                  double cf, int32_t *load, int32_t *used, double *importance, void *ws,
                                  size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- backward */

/* Workspace bytes for moe_backward. */
MOE_API size_t moe_backward_workspace_size(int64_t N, int d, int E, int d_ff, int k, int64_t rows, moe_dtype dt);

/* Gradients of L = sum over t, i of dy[t][i] y[t][i] for the routing of a
 * forward pass made with the staged calls (moe_route, moe_dispatch,
 * moe_expert_ffn_train, moe_combine), ReLU experts without biases.
 * ("Mixture of Experts (MoE) 12段階…" STEP 6: the -inf mask keeps the kept
 * experts' softmax differentiable; STEP 11: g_i E_i(x) carries the gradient
 * to the router; "nanoMoEの深層解剖" slide 10: the router is trained by
 * backpropagation.)  The top-k indices and slots carry no gradient.  For a
 * kept pair (t, j) of expert e and gathered row r:
 *   dg = dy_t . O_r,  dO_r = g_j dy_t,  dZ_r = (dO_r W_down[e]) * [H_r > 0],
 *   dX_r = dZ_r W_up[e],  dW_down[e] += dO_r^T H_r,  dW_up[e] += dZ_r^T x_gathered_r;
 * for every chosen pair (dropped ones too, with dg = 0, since the gates are
 * formed before the capacity cut): ds_j = g_j (dg_j - sum_l g_l dg_l),
 *   dW_g[e] += ds_j x_t,  db_g[e] += ds_j,  dx_t = sum_kept dX_r + sum_j ds_j W_g[e_j].
 * The noise is added to the scores, so these are also the gradients through
 * the pre-noise logits.
 *
 *  x, W_g, W_up, W_down, N, d, E, d_ff, k   the forward's inputs
 *  rows                     moe_gathered_rows() of the forward
 *  topk_idx, gates          device [N, k] from moe_route
 *  slot, offsets, counts    device, from moe_dispatch
 *  x_gathered               device [rows, d] of dt, from moe_dispatch
 *  H                        device [rows, d_ff] of dt, from moe_expert_ffn_train
 *  out_gathered             device [rows, d] of dt, from moe_expert_ffn_train
 *  dy                       device [N, d] of dt
 *  dx                       device [N, d] of dt out
 *  dW_g [E, d], db_g [E], dW_up [E, d_ff, d], dW_down [E, d, d_ff]   device fp32 out
 *                           (overwritten; an expert without rows gets zeros)
 *  ws, ws_bytes             workspace of moe_backward_workspace_size() bytes; its first
 *                           4 bytes are the status word (moe_check_status)
 * bf16 with d and d_ff multiples of 8: the four expert GEMMs run on the tensor
 * cores (fp32 accumulation; dO, dZ and the expert part of dx rounded to bf16
 * on the way, weight gradients in fp32); otherwise fp32 CUDA-core kernels.
 * Deterministic: no atomics decide a sum's order. */
MOE_API moe_status moe_backward(const void *x, moe_dtype dt, const float *W_g, const void *W_up,
                                const void *W_down, int64_t N, int d, int E, int d_ff, int k, int64_t rows,
                                const int32_t *topk_idx, const float *gates, const int32_t *slot,
                                const int32_t *offsets, const int32_t *counts, const void *x_gathered,
                                const void *H, const void *out_gathered, const void *dy, void *dx, float *dW_g,
                                float *db_g, float *dW_up, float *dW_down, void *ws, size_t ws_bytes,
                                void *stream);

/* ---------------------------------------------------------------- fused */

/* Workspace bytes for moe_forward. */
MOE_API size_t moe_workspace_size(int64_t N, int d, int E, int d_ff, int k, double cf, moe_dtype dt);

/* The whole layer: route, dispatch, expert FFN, combine, on one stream with no
 * host synchronisation.  Arguments as in the calls above; every intermediate
 * lives in ws.  logits_out/topk_out/gates_out/slot_out/counts_out (all nullable)
 * receive copies of the intermediates for inspection.
 *  y device [N, d] of dt. */
MOE_API moe_status moe_forward(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                       const float *noise, float sigma, int64_t N, int d, int E, int d_ff,
                       int k, double cf, const void *W_up, const void *W_down, void *y,
                       float *logits_out, int32_t *topk_out, float *gates_out,
                       int32_t *slot_out, int32_t *counts_out,
                       void *ws, size_t ws_bytes, void *stream);

/* moe_forward with the nanoMoE expert variant (see moe_expert_ffn_ex):
 * activation, b_up [E, d_ff] and b_down [E, d] (fp32, nullable).  moe_forward is
 * this call with MOE_ACT_RELU and no biases.  Same workspace size. */
MOE_API moe_status moe_forward_ex(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                                  const float *noise, float sigma, int64_t N, int d, int E, int d_ff,
                                  int k, double cf, const void *W_up, const void *W_down, int activation,
                                  const float *b_up, const float *b_down, void *y,
                                  float *logits_out, int32_t *topk_out, float *gates_out,
                                  int32_t *slot_out, int32_t *counts_out,
                                  void *ws, size_t ws_bytes, void *stream);

/* Number of kernels one moe_forward call with these arguments launches on its
 * stream (0 for N = 0, -1 for invalid arguments).  Useful to size CUDA-graph
 * captures and to account for launches. */
MOE_API int moe_forward_launches(int64_t N, int d, int E, int d_ff, int k, double cf, moe_dtype dt);

/* Whether moe_forward runs batches of at most 64 bf16 tokens (E <= 16, ReLU
 * experts without biases, the decode plan) as one cooperative kernel on every
 * SM instead of the decode plan's separate kernels.  Both give identical
 * bits.  on = 1 or 0 sets the choice for the process (calls already queued
 * keep theirs); on < 0 only queries.  Returns the previous setting.  Default:
 * off (on a B200 the separate kernels stream the expert weights faster), or on
 * when the environment variable MOE_FUSED_DECODE is a nonzero number.  The
 * workspace size does not depend on it; moe_forward_launches follows it. */
MOE_API int moe_set_fused_small_batch(int on);

/* ---------------------------------------------------------------- status */

/* Reads the status word at the start of a workspace given to moe_expert_ffn,
 * moe_forward or moe_debug_wait_timeout (or a word given to moe_route_ex),
 * clears it, both on `stream`, and synchronises the stream.  Returns MOE_OK,
 * MOE_ERR_TIMEOUT (a bounded wait in a kernel ran out since the word was last
 * cleared; that kernel skipped its remaining work and released its tensor
 * memory) or MOE_ERR_DEVICE_CHECK.  *detail (nullable) receives the raw word:
 * bit 0 timeout, bit 2 index check, bits 8-15 which wait ran out (ORed). */
MOE_API moe_status moe_check_status(void *ws, void *stream, uint32_t *detail);

/* Diagnostic for the bounded-wait machinery: launches one CTA that waits on
 * a shared-memory barrier nothing will ever complete, with a limit of
 * timeout_us microseconds, using the same wait routine as the tensor-core
 * kernels.  The kernel then ORs MOE_ERR_TIMEOUT's bit into the status word of
 * ws (>= 256 bytes) and returns.  No pages' counterpart; exists so that tests
 * can check that a wait which runs out ends cleanly and that its report
 * survives later calls on the same workspace. */
MOE_API moe_status moe_debug_wait_timeout(uint32_t timeout_us, void *ws, size_t ws_bytes, void *stream);

/* Number of streaming multiprocessors the library sizes its persistent grids
 * for on the current device (0 if no device). */
MOE_API int moe_num_sms(void);

MOE_API const char *moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
