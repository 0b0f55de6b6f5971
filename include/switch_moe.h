/*
 * switch_moe.h -- C ABI of the Switch-FFN layer (forward pass and its
 * backward) on one NVIDIA B200 (sm_100a).
 *
 * The layer is the one of "Switch Transformers: scaling to trillion-parameter
 * models" (cited below as [P1 section]):
 *   router logits h(x) = W_r . x and softmax gate p_i(x)
 *       [P1 "Switch Routing: From Top-k to k = 1", gate equation],
 *   routing math in float32 [P1 "Making Sparse Training Stable",
 *       selective precision],
 *   top-1 expert (k = 1), lowest index on ties,
 *   expert capacity C = ceil(T / N x capacity_factor)
 *       [P1 "Expert Capacity and the Capacity Factor", capacity equation],
 *   tokens take slots in batch order; overflow tokens are dropped and pass
 *       through on the residual; unused slots are padding [same section],
 *   N independent ReLU FFN experts E_e(x) = relu(x W1_e^T) W2_e^T
 *       [P1 "The Core Idea"],
 *   gate-scaled combine y = p_i(x) E_i(x) [P1 "Switch Routing", combine
 *       equation, one selected expert], block output x + y,
 *   load-balancing loss alpha . N . sum_i f_i P_i
 *       [P1 "The Load-Balancing Loss", loss and f/P equations].
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous, each aligned to at least 16 bytes.  The library never
 *     allocates or frees device memory.
 *   - Scratch lives in a caller-owned device workspace of at least
 *     switch_workspace_size() bytes (256-byte aligned).  Its first 256 bytes
 *     hold the device error word and a counter that the calls leave at zero;
 *     zero them once after allocating (a zero-filled allocation is fine).
 *     Calls that share a workspace must be ordered on one stream.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it; nothing synchronises the host
 *     except switch_get_device_error().
 *   - Host-detectable errors (bad arguments, unsupported shapes, workspace
 *     too small) return synchronously and launch nothing.  Launch failures
 *     return SWITCH_ERR_CUDA.  Device-side failures (a bounded wait that ran
 *     out) are recorded in the error word and read by
 *     switch_get_device_error().
 *   - T = 0 is a no-op that returns SWITCH_OK and writes nothing.
 *   - Inputs must be finite; results for NaN/Inf inputs are unspecified.
 *   - dtype SWITCH_BF16: x, w1, w2, y, x_disp and out are bf16, the router
 *     weight/bias/probabilities/gates are fp32, d_model and d_ff must be
 *     multiples of 64.  dtype SWITCH_F32: every floating tensor is fp32 and
 *     all arithmetic is fp32 FMA (no TF32).
 *   - Index tensors are int32, the drop mask is uint8 (0 kept / 1 dropped).
 *   - Expert weights are stored output-major per expert, like the weight of
 *     a linear layer: w1 [N, d_ff, d_model], w2 [N, d_model, d_ff], so that
 *     E_e(x) = relu(x . w1[e]^T) . w2[e]^T.  Router weight w_r [N, d_model].
 */
#ifndef SWITCH_MOE_H_
#define SWITCH_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SWITCH_OK = 0,
  SWITCH_ERR_INVALID_ARG = 1,          /* null pointer, bad size, misaligned */
  SWITCH_ERR_UNSUPPORTED = 2,          /* shape/dtype this build does not run */
  SWITCH_ERR_WORKSPACE_TOO_SMALL = 3,
  SWITCH_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed */
  SWITCH_ERR_TIMEOUT = 5,              /* device: a bounded wait ran out */
  SWITCH_ERR_DEVICE_BOUNDS = 6         /* device: an index out of range */
} switch_status_t;

typedef enum { SWITCH_F32 = 0, SWITCH_BF16 = 1 } switch_dtype_t;

/* Option bits of switch_config_t.flags (0 = the default fast path). */
enum {
  SWITCH_FLAG_ROUTER_SIMT = 1,       /* CUDA-core fp32 FMA router */
  SWITCH_FLAG_ROUTER_3TERM = 2,      /* tensor-core router, W_r split in 3 bf16 terms (default 2) */
  SWITCH_FLAG_UNFUSED_COMBINE = 4,   /* forward: write Y, then a separate combine kernel */
  SWITCH_FLAG_GATHER_IN_GEMM = 8,    /* bf16 expert FFN: GEMM1 gathers the routed rows of x
                                        itself (default: one copy kernel first lays them out
                                        expert by expert, then GEMM1 reads tiles by TMA) */
  SWITCH_FLAG_NO_RESIDUAL = 16,      /* forward: block output is y alone (dropped -> 0) */
  SWITCH_FLAG_GEMM_1SM = 32,         /* both expert GEMMs on single CTAs */
  SWITCH_FLAG_GEMM_PAIRS = 64,       /* GEMM1 on CTA pairs too (default: GEMM1 single CTAs,
                                        GEMM2 CTA pairs) */
  SWITCH_FLAG_ROWS_DISPATCHED = 128, /* switch_expert_ffn: x is the dispatched row buffer
                                        x_disp [N*C, d_model] from switch_dispatch */
  SWITCH_FLAG_TOP2 = 512,            /* top-k routing with k = 2 (see "Top-2 routing" below) */
  SWITCH_FLAG_TRAINING = 1024,       /* forward keeps what switch_layer_backward needs in the
                                        workspace; the backward then reads it instead of
                                        recomputing (see switch_layer_backward) */
  SWITCH_FLAG_GEMM1_ROWS_PAIRS = 2048 /* bf16 GEMM1 on CTA pairs with 256 dispatched rows x 256
                                        columns per tile, an expert's last 128 rows as a half
                                        tile (needs the row copy: not with
                                        SWITCH_FLAG_GATHER_IN_GEMM); the default already when
                                        128 < C <= 256 or d_model >= 2048 */
};

typedef struct {
  int64_t T;                /* tokens in the batch: one routing group, batch order */
  int32_t d_model;
  int32_t d_ff;
  int32_t n_experts;        /* 1 <= N <= 1024 */
  int32_t dtype;            /* switch_dtype_t */
  double capacity_factor;   /* > 0; taken at the exact value of the double */
  float alpha;              /* load-balancing loss coefficient */
  int32_t flags;            /* SWITCH_FLAG_* */
  int64_t spin_limit;       /* bounded-wait limit in SM cycles; 0 = default (~2 s) */
} switch_config_t;

/* Top-2 routing [P1 "Switch Routing: From Top-k to k = 1": the top-k set
 * T of largest gates, output sum_{i in T} p_i(x) E_i(x), p the softmax over
 * all N experts, not renormalised].  With SWITCH_FLAG_TOP2 (needs N >= 2):
 *   - every per-token routing array has 2T entries, route-major: entry t is
 *     the token's first choice, entry T + t its second (the largest other
 *     logit, lowest index on ties);
 *   - expert capacity is taken over the 2T assignments:
 *     C = switch_capacity(2 T, N, capacity_factor) (each expert receives
 *     tokens from two routes);
 *   - dispatch ranks the assignments in that order, so every first choice
 *     takes a slot before any second choice; slot_token holds tokens;
 *   - combine adds both kept routes: x + sum_r gate_r * y[idx_r, rank_r];
 *   - the load-balancing loss keeps f_i over the first choices;
 *   - the tensor-core router supports it for terms x round_up(N, 32) <= 256
 *     (else the fp32 FMA router runs); switch_dispatch needs idx (not
 *     probs); switch_dispatch_noalloc returns SWITCH_ERR_UNSUPPORTED.
 * Readings of the pages (first choices first, f over first choices) are the
 * library's; the pages fix only the top-k set, the gates and the sum. */

/* Expert capacity C = ceil(T x capacity_factor / N), computed exactly
 * [P1 "Expert Capacity and the Capacity Factor", capacity equation; the
 * page prints no rounding, rounding up is the reading taken].
 * Returns -1 for T < 0, N < 1 or capacity_factor <= 0 (or not finite). */
int64_t switch_capacity(int64_t T, int32_t n_experts, double capacity_factor);

/* Bytes of device workspace every entry point below accepts for `cfg`
 * (the maximum over them).  Writes *bytes; validates cfg. */
switch_status_t switch_workspace_size(const switch_config_t* cfg, size_t* bytes);

/* Router [P1 "Switch Routing", gate equation; top-1; fp32 routing math].
 *   x      [T, d_model]  bf16 or fp32 (cfg->dtype)
 *   w_r    [N, d_model]  fp32;  b_r [N] fp32 or NULL (added to the logits)
 *   idx    [T] int32 out: expert of the largest logit, lowest index on ties
 *   gate   [T] fp32  out: p_idx(x)
 *   (top-2: idx and gate [2T], see "Top-2 routing")
 *   probs  [T, N] fp32 out, or NULL: softmax probabilities
 * bf16 x runs on the tensor cores: bf16 x is exact, W_r is split into bf16
 * terms hi + lo (W_r to about 2^-17 relative; SWITCH_FLAG_ROUTER_3TERM adds
 * a third term, whose sum is W_r exactly), each term accumulated in its
 * own fp32 TMEM columns and the logits summed in fp32.  Measured max
 * relative error of the probabilities against a float64 reference: about
 * 4e-6 (two terms), 2e-6 (three).  Probabilities below 2^-126 are returned
 * as 0.  fp32 x (or SWITCH_FLAG_ROUTER_SIMT) uses fp32 FMA. */
switch_status_t switch_router(const switch_config_t* cfg, const void* x,
                              const float* w_r, const float* b_r, int32_t* idx,
                              float* gate, float* probs, void* ws, size_t ws_bytes,
                              void* stream);

/* Capacity-bounded dispatch [P1 "Expert Capacity and the Capacity
 * Factor": overflow dropped, padding slots].  Input: idx [T] int32, or, when
 * idx is NULL, probs [T, N] fp32 whose argmax (lowest index on ties) is the
 * expert.  Outputs (all required):
 *   rank       [T] int32: number of earlier tokens routed to the same expert
 *   drop       [T] uint8: rank >= C
 *   counts     [N] int32: tokens routed to each expert (before the cut)
 *   slot_token [N * C] int32: token in slot r of expert e at e*C + r, -1 for
 *              padding
 * Optional gather: if x_disp is non-NULL, x [T, d_model] must be given and
 * x_disp [N, C, d_model] receives x[slot_token] per slot, zeros in padding.
 * Deterministic: slot order never depends on thread timing.
 * Expert ids outside [0, N) set SWITCH_ERR_DEVICE_BOUNDS in the error word
 * (the token is then treated as dropped).  Top-2: idx, rank and drop have
 * 2T entries (see "Top-2 routing"), counts counts both routes. */
switch_status_t switch_dispatch(const switch_config_t* cfg, const int32_t* idx,
                                const float* probs, int32_t* rank, uint8_t* drop,
                                int32_t* counts, int32_t* slot_token, const void* x,
                                void* x_disp, void* ws, size_t ws_bytes, void* stream);

/* switch_dispatch for callers that cannot allocate device memory (the
 * pages have no counterpart: this is a deployment convenience).  A plugin
 * running inside another engine's enqueue step, or a serving loop with a
 * fixed memory budget that must not call cudaMalloc after start-up (it can
 * synchronise the device), cannot hand this library a workspace; this entry
 * point needs none.  Same inputs and outputs as switch_dispatch without the
 * optional gather (idx or probs in; rank, drop, counts, slot_token out; all
 * device pointers owned by the caller), bit-identical results.
 *   - Scratch: a 2 MiB array compiled into the library, held by every GPU
 *     that loads it until the process exits.  Limits: T <= 131072 and
 *     N * ceil(T / 128) <= 131072; larger sizes return SWITCH_ERR_UNSUPPORTED
 *     and launch nothing.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after a
 *     cudaDeviceReset() the library must be unloaded and loaded again before
 *     this entry point is called on that device.
 *   - All calls share the array: calls that overlap on the GPU (different
 *     streams with no ordering between them) race and give wrong results.
 *   - No device error word: expert ids outside [0, N) make the token dropped
 *     (rank -1, drop 1) without a report.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
switch_status_t switch_dispatch_noalloc(const switch_config_t* cfg, const int32_t* idx,
                                        const float* probs, int32_t* rank, uint8_t* drop,
                                        int32_t* counts, int32_t* slot_token, void* stream);

/* Expert FFNs over the capacity buffers [P1 "The Core Idea"]:
 *   y[e, r, :] = relu(x[slot_token[e*C + r]] . w1[e]^T) . w2[e]^T
 * for r < n_e = min(counts[e], C).  Rows r >= n_e of y are left untouched.
 *   x [T, d_model], w1 [N, d_ff, d_model], w2 [N, d_model, d_ff],
 *   y [N, C, d_model]; slot_token [N*C], counts [N] as from switch_dispatch.
 * With SWITCH_FLAG_ROWS_DISPATCHED, x is instead the dispatched buffer
 * x_disp [N*C, d_model] (row e*C + r = x[slot_token[e*C + r]]) that
 * switch_dispatch writes; slot_token is then not read (may be NULL).
 * bf16: tcgen05 grouped GEMM, fp32 accumulation, the hidden activation is
 * rounded once to bf16, y rounded once to bf16.  fp32: CUDA-core FMA. */
switch_status_t switch_expert_ffn(const switch_config_t* cfg, const void* x,
                                  const int32_t* slot_token, const int32_t* counts,
                                  const void* w1, const void* w2, void* y, void* ws,
                                  size_t ws_bytes, void* stream);

/* Combine [P1 "Switch Routing", combine equation with one expert; dropped
 * tokens pass through on the residual]:
 *   out[t] = x_residual[t] + (drop[t] ? 0 : gate[t] * y[idx[t], rank[t], :])
 * computed in fp32 and rounded once to the output dtype.  x_residual may be
 * NULL (no residual term).  y [N, C, d_model].  Top-2: both kept routes are
 * added (first route first), idx/rank/drop/gate [2T]. */
switch_status_t switch_combine(const switch_config_t* cfg, const void* x_residual,
                               const int32_t* idx, const int32_t* rank,
                               const uint8_t* drop, const float* gate, const void* y,
                               void* out, void* stream);

/* Load-balancing loss [P1 "The Load-Balancing Loss"]:
 *   f_i = counts_i / T, P_i = (1/T) sum_t probs[t, i],
 *   loss = alpha . N . sum_i f_i P_i.
 * counts [N] int32 (routed, dropped included), probs [T, N] fp32.
 * loss: device fp32 scalar; f, P: [N] fp32 or NULL.  Fixed-order
 * reductions: the result is bit-reproducible run to run. */
switch_status_t switch_aux_loss(const switch_config_t* cfg, const int32_t* counts,
                                const float* probs, float* loss, float* f, float* P,
                                void* ws, size_t ws_bytes, void* stream);

/* The whole layer on one stream with no host synchronisation:
 * router -> dispatch (and, bf16, one copy of the routed rows) -> expert FFN
 * (ReLU in GEMM1's epilogue) -> gate x expert output + residual (fused into
 * GEMM2's epilogue; a separate combine with SWITCH_FLAG_UNFUSED_COMBINE or
 * top-2) -> load-balancing loss.
 *   out [T, d_model] (same dtype as x)
 *   idx [T] int32, gate [T] fp32, counts [N] int32: optional outputs (NULL
 *   to skip); loss: device fp32 scalar or NULL.  Top-2: idx and gate [2T],
 *   counts over both routes.
 * Same results as the staged calls above in sequence. */
switch_status_t switch_layer_forward(const switch_config_t* cfg, const void* x,
                                     const float* w_r, const float* b_r,
                                     const void* w1, const void* w2, void* out,
                                     int32_t* idx, float* gate, int32_t* counts,
                                     float* loss, void* ws, size_t ws_bytes,
                                     void* stream);

/* Backward pass of switch_layer_forward (bf16 or fp32; top-1, or top-2 below): the gradient of
 *   J = sum(dout * out) + dloss * loss
 * with respect to x, w_r, b_r, w1 and w2, routing decisions held fixed (the
 * argmax and the capacity cut are piecewise constant; f_i likewise).  The
 * gradient reaches the router through the gate value p_idx(x) that scales
 * the expert output [P1 "Switch Routing: From Top-k to k = 1": the gate
 * value is what makes the router trainable] and through P_i of the
 * load-balancing loss [P1 "The Load-Balancing Loss"]:
 *   dgate[t] = dout[t] . E_idx(x_t)           (kept tokens; 0 if dropped)
 *   dW2_e = sum_t (gate dout)[t]^T H_t,  dA = (gate dout W2_e) where H > 0,
 *   dW1_e = sum_t dA_t^T x_t,  dx_t += dA_t W1_e,
 *   dp[t, i] = [i = idx_t] dgate[t] + dloss alpha N f_i / T,
 *   dh = p (dp - sum_j p_j dp_j),  dx += dh W_r,  dW_r = dh^T x,
 *   db_r = sum_t dh,  dx += dout (the residual branch, unless
 *   SWITCH_FLAG_NO_RESIDUAL).
 * Saved activations: without SWITCH_FLAG_TRAINING the call recomputes the
 * forward's routing, dispatch and hidden activations from its inputs (as
 * activation checkpointing does) and reads nothing a previous call left in
 * the workspace.  With SWITCH_FLAG_TRAINING, switch_layer_forward (given a
 * workspace of switch_backward_workspace_size() bytes) keeps the router
 * probabilities, the routing, the dispatched rows and H there, and this
 * call reads them instead: it must follow that forward call with the same
 * config, inputs and workspace, with no other call on the workspace in
 * between (backward calls may repeat: they leave that state unchanged).
 * Both ways give bit-identical gradients.
 *   x [T, d_model], w_r [N, d_model] fp32, b_r [N] fp32 or NULL,
 *   w1 [N, d_ff, d_model], w2 [N, d_model, d_ff] (as the forward);
 *   dout [T, d_model]: gradient of J with respect to out;
 *   dloss: host float, the weight of the loss in J;
 *   outputs: dx [T, d_model], dw_r [N, d_model] fp32, db_r [N] fp32 or
 *   NULL, dw1 [N, d_ff, d_model], dw2 [N, d_model, d_ff], dgate [T] fp32
 *   or NULL (the gate gradient above); x, w1, w2, dout, dx, dw1 and dw2 in
 *   cfg->dtype (bf16 or fp32).
 * Top-2 (SWITCH_FLAG_TOP2) [P1 "Switch Routing": out = x + sum over the
 * top-k set of p_i E_i(x), p the full softmax, not renormalised]: every kept
 * route r of token t (expert idx_r, gate p_{idx_r}) contributes its own
 * expert gradients and its own gate gradient
 *   dgate[r T + t] = dout[t] . E_{idx_r}(x_t)  (0 for a dropped route),
 *   dp[t, i] = sum over kept r with idx_r = i of dgate[r T + t]
 *              + dloss alpha N f_i / T,
 * f_i over the first choices (as the forward's loss); dx adds both kept
 * routes' dA W1_e rows (kept in fp32 per slot, then summed per token in
 * route order with the residual and dh W_r).  dgate is then [2 T] fp32,
 * route-major.  A route whose gate underflowed to 0 reports dgate 0 (its
 * dY is 0; p = 0 removes it from dh in any case).
 * Arithmetic: bf16 -- expert GEMMs on the tensor cores (bf16 operands,
 * fp32 accumulation; gate * dout, dA and the weight gradients rounded once
 * to bf16); router backward in fp32 FMA with fixed-order reductions (dW_r
 * and db_r bit-reproducible).  fp32 -- every product and sum in fp32 on
 * CUDA-core FMA tiles (the path of small full-precision configurations),
 * each output element one fixed-order loop, so all gradients are
 * bit-reproducible.  Workspace: switch_backward_workspace_size() bytes.
 * T = 0 writes nothing. */
switch_status_t switch_layer_backward(const switch_config_t* cfg, const void* x,
                                      const float* w_r, const float* b_r,
                                      const void* w1, const void* w2, const void* dout,
                                      float dloss, void* dx, float* dw_r, float* db_r,
                                      void* dw1, void* dw2, float* dgate, void* ws,
                                      size_t ws_bytes, void* stream);

/* Bytes of device workspace switch_layer_backward needs for `cfg` (more
 * than switch_workspace_size(); every other entry point accepts it too). */
switch_status_t switch_backward_workspace_size(const switch_config_t* cfg, size_t* bytes);

/* ------------------------------------------------------------------------
 * Expert parallelism [P1 "Distributed Implementation and the Three
 * Parallelisms", expert-parallelism row: each device holds some of the
 * experts and tokens travel to their expert's device and back].
 *
 * G ranks (one GPU each) hold N / G experts each -- rank h owns experts
 * h*N/G .. (h+1)*N/G - 1 -- and cfg->T tokens each (the same T on every
 * rank).  The global batch is the ranks' batches end to end in rank order
 * and is ONE routing group: capacity C = switch_capacity(G*T, N, cf), slot
 * order is global batch order, f_i and P_i are over all G*T tokens.  So the
 * outputs, counts and loss equal switch_layer_forward's on the
 * concatenated batch on one GPU (bit for bit when T is a multiple of 128;
 * otherwise the loss differs by fp32 summation order only).
 *
 * One forward step, on every rank, in this order:
 *   1. switch_ep_route      router + this rank's per-expert counts; writes
 *                           this rank's exchange record (record_bytes);
 *   2. [caller] all-gather the records of all ranks, in rank order, into
 *      `records` [G][record_bytes] (e.g. an NCCL all-gather on the stream);
 *   3. switch_ep_dispatch   global ranks and drops; stores every kept
 *                           token's row, source and gate straight into its
 *                           owner's receive buffer (peer pointers); writes
 *                           dropped tokens' outputs; the loss;
 *   4. [caller] barrier: every rank's step 3 has completed;
 *   5. switch_ep_experts    this rank's experts' GEMMs; the second GEMM's
 *                           epilogue stores x + gate * E(x) into each
 *                           token's output row on its home rank (peer
 *                           pointers);
 *   6. [caller] barrier before any rank reads its output.
 * Peer buffers: every rank's receive buffer (recv_bytes, 256-byte aligned)
 * and output [T, d_model] must be reachable from every rank's GPU (CUDA IPC
 * or symmetric memory over NVLink); the calls take host arrays of the G
 * device pointers, entry h being rank h's.  No copy reads another GPU's
 * memory: the exchange is made of plain stores, none of them multicast.
 * bf16 only, top-1 only, CTA-pair second GEMM (SWITCH_FLAG_GEMM_1SM and
 * SWITCH_FLAG_TOP2 return SWITCH_ERR_UNSUPPORTED), N % G == 0, G <= 16,
 * T < 2^26.  SWITCH_FLAG_NO_RESIDUAL and SWITCH_FLAG_GEMM_PAIRS apply.
 * T = 0 makes every call a no-op. */
typedef struct {
  int32_t world_size;       /* G: ranks of the expert-parallel group */
  int32_t rank;             /* this rank, 0 <= rank < G */
} switch_ep_t;

/* Bytes of this rank's workspace (ws_bytes; the same conventions as
 * switch_workspace_size's), of one exchange record (record_bytes) and of a
 * receive buffer (recv_bytes).  Any output pointer may be NULL. */
switch_status_t switch_ep_sizes(const switch_config_t* cfg, const switch_ep_t* ep,
                                size_t* ws_bytes, size_t* record_bytes, size_t* recv_bytes);

/* Step 1.  x [T, d_model] bf16, w_r [N, d_model] fp32, b_r [N] or NULL as
 * for switch_router; idx [T] int32 and gate [T] fp32: optional copies of
 * the top-1 choices and gates.  record: record_bytes of device memory
 * (16-byte aligned) receiving this rank's per-expert counts and
 * per-128-token sums of the router probabilities. */
switch_status_t switch_ep_route(const switch_config_t* cfg, const switch_ep_t* ep,
                                const void* x, const float* w_r, const float* b_r,
                                int32_t* idx, float* gate, void* record, void* ws,
                                size_t ws_bytes, void* stream);

/* Step 3 (after step 2).  records: [G][record_bytes], rank order.
 * recv_peers: host array of the G ranks' receive buffers.  out: this rank's
 * output [T, d_model] bf16; this call writes its dropped tokens' rows (x,
 * or 0 without the residual).  counts [N] int32 (routed tokens of the whole
 * batch, before the cut) and loss (device fp32 scalar): optional. */
switch_status_t switch_ep_dispatch(const switch_config_t* cfg, const switch_ep_t* ep,
                                   const void* x, const void* records, void* const* recv_peers,
                                   void* out, int32_t* counts, float* loss, void* ws,
                                   size_t ws_bytes, void* stream);

/* Step 5 (after step 4).  w1_local [N/G, d_ff, d_model] and w2_local
 * [N/G, d_model, d_ff] bf16: this rank's experts' weights (rows
 * rank*N/G .. of the full w1 / w2).  recv: this rank's receive buffer.
 * out_peers: host array of the G ranks' outputs [T, d_model].  Kept
 * tokens' output rows are written on their home ranks. */
switch_status_t switch_ep_experts(const switch_config_t* cfg, const switch_ep_t* ep,
                                  const void* w1_local, const void* w2_local, const void* recv,
                                  void* const* out_peers, void* ws, size_t ws_bytes,
                                  void* stream);

/* Synchronises `stream`, reads the workspace's device error word, clears
 * it, and returns the recorded status (SWITCH_OK if none).  *where_out and
 * *info_out (either may be NULL) receive the reporting kernel role and a
 * detail value. */
switch_status_t switch_get_device_error(void* ws, void* stream, int32_t* where_out,
                                        int64_t* info_out);

/* Static, human-readable name of a status code. */
const char* switch_status_string(switch_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SWITCH_MOE_H_ */
