/*
 * moe_layer.h -- C ABI of the B200 (sm_100a) sparse-MoE FFN layer library (libmoe_layer.so).
 *
 * One fine-grained sparse-MoE FFN layer as described in "Step 3.5 Flash: Open
 * Frontier-Level Intelligence with 11B Active Parameters" (section 2.2: 288 routed experts
 * plus one always-on shared expert, top-k = 8 per token; section 2.2.2: loss-free
 * balancing, top-K set S_t and routing probabilities p_{t,e}; section 3.2.4: fused MoE
 * gather/scatter with grouped GEMM; section 4.1.2: routed aggregation needs an explicit
 * scale) and in the parameter table of "Step 3.5 Flash 技术论文深度解读" (architecture
 * item 1: routed-expert hidden size 1280, balancing by a bias instead of an auxiliary
 * loss; training-stability item: SwiGLU experts with gate and up branches).
 *
 * The layer, for token t with input row x_t (d = d_model, E routed experts, k = top_k,
 * f = d_ff, G = E + n_shared expert weight sets):
 *   l[t,e]  = x_t . W_r[e]                              router logits (fp32 accumulation)
 *   s[t,e]  = l[t,e] + b[e]                             fp32 add; the bias only SELECTS
 *   S_t     = the k experts with the largest s; equal scores -> lower expert id first,
 *             -0.0 == +0.0, NaN below every number; slot j = rank j
 *   g[t,j]  = exp(l[t,S_t[j]] - m) / sum_j' exp(l[t,S_t[j']] - m), m = max over S_t
 *   FFN_e(x) = W_d[e] . (silu(W_g[e] . x) * (W_u[e] . x)),  silu(z) = z / (1 + exp(-z))
 *   out_t   = FFN_E(x_t) [shared, if n_shared] + routed_scale * sum_j g[t,j] FFN_{S_t[j]}(x_t)
 *
 * Ownership and memory: every device buffer (weights, x, out, routing outputs, workspace)
 * belongs to the caller.  The library never allocates device memory; it keeps the weight
 * pointers (which must outlive the handle) and host-side TMA descriptors.  All calls that
 * take a stream are asynchronous on that stream, never synchronise the host, and may be
 * captured into a CUDA graph.  Argument, size and alignment errors are returned before
 * anything is launched; a failed launch returns MOE_ERR_CUDA.  Device-side waits are
 * bounded: a wait that gives up records a flag in the workspace, which
 * moe_device_status() reports.
 *
 * Layouts (all row-major, innermost dimension contiguous):
 *   x        [n_tokens, d]          dtype            out   [n_tokens, d]  dtype
 *   w_router [E, d]                 dtype            bias  [E]            fp32
 *   w_gate   [G, f, d]              dtype            w_up  [G, f, d]      dtype
 *   w_down   [G, d, f]              dtype            (shared expert = index E)
 *   logits   [n_tokens, E] fp32     topk_idx [n_tokens, k] int32   topk_gate [n_tokens, k] fp32
 *   expert_counts [E] int32         expert_offsets [E + 1] int32 (exclusive prefix sum)
 *   perm     [n_tokens * k] int32   perm[expert_offsets[e] + r] = t * k + j for the r-th
 *                                   token (ascending t) that selected e, in slot j
 *   slot_row [n_tokens, k] int32    inverse of perm: slot_row[t, j] = position of (t, j)
 * For MOE_BF16 the tensor-core path needs d % 128 == 0, f % 128 == 0 and every device
 * pointer 16-byte aligned.  MOE_F32 runs exact fp32 SIMT arithmetic (no TF32).
 */
#ifndef MOE_LAYER_H
#define MOE_LAYER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, k > E, n_tokens > max_tokens ... */
  MOE_ERR_UNSUPPORTED = 2,   /* shape the kernels do not handle (see layout notes above) */
  MOE_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE = 4,     /* workspace null or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 5,          /* a CUDA runtime / driver call or a launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 6 /* a bounded device-side wait gave up (moe_device_status) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Layer shape.  max_tokens bounds n_tokens of every call; n_shared is 0 or 1;
 * routed_scale multiplies the gate-weighted routed sum (1.0 when the pages give no value). */
typedef struct {
  int max_tokens;
  int d_model;
  int n_experts;
  int top_k;
  int d_ff;
  int n_shared;
  moe_dtype dtype;
  float routed_scale;
} moe_config;

/* Caller-owned device pointers to the layer's weights (layouts above). */
typedef struct {
  const void *w_router;
  const float *router_bias; /* may be null: zero bias */
  const void *w_gate;
  const void *w_up;
  const void *w_down;
} moe_weights;

typedef struct moe_layer *moe_handle;

/* Validates the shape and the weight pointers, records them and encodes the weight TMA
 * descriptors on the current CUDA device.  Host only: no device allocation, no launch, no
 * synchronisation.  On success *out is a new handle (free it with moe_layer_destroy). */
moe_status moe_layer_init(const moe_config *cfg, const moe_weights *w, moe_handle *out);

/* Releases the host-side handle.  Does not touch any device buffer. */
moe_status moe_layer_destroy(moe_handle h);

/* Launch-plan options of a handle (host only; takes effect from the next call):
 *   MOE_OPTION_H_HANDOVER  1 (default): the bf16 forward's down-projection GEMM starts while
 *                          the up GEMM still runs and takes each expert group's h as soon as
 *                          that group's up units have stored it (per-group completion counts
 *                          in the workspace) -- used only when the init-time occupancy check
 *                          finds every persistent up grid co-resident on the device;
 *                          0: the down GEMM waits for the whole up GEMM (same results, bit
 *                          for bit; for callers that share the GPU's SMs with other
 *                          persistent work and want no cross-kernel waiting at all).
 *   MOE_OPTION_SHARED_SIDE_SMS  n >= 2: in bf16 forwards on CTA pairs (about 96 or more
 *                          tokens per expert), the shared expert -- which needs no routing --
 *                          runs its up and down GEMMs on a stream of the handle on n SMs
 *                          (rounded down to whole pairs) while the caller's stream routes the
 *                          tokens; the caller's stream waits for it (an event) before the
 *                          combine, so the call stays asynchronous on `stream` and the results
 *                          are the same bit for bit.  0 (default): everything on `stream`.
 *                          The first non-zero value creates the stream and two events on the
 *                          handle's device (make it before capturing a CUDA graph; a captured
 *                          forward records the fork and join into the graph).  Calls on one
 *                          handle from several host threads at once are not supported.
 *                          Not used by moe_forward_profiled or moe_forward_save.
 *   MOE_OPTION_ROW_GATHER_IN_GEMM  in bf16 forwards on CTA pairs with a shared expert, who
 *                          writes the expert-sorted copy of x: 2: the up GEMM itself (two
 *                          warps of each CTA, while the CTAs run the shared expert's units,
 *                          which read x directly and are claimed first); 1 (default): the
 *                          same when the shared expert's up units are at least one per CTA
 *                          pair of the device (d_ff/256 x ceil(T/256) >= SMs/2), else as 0;
 *                          0: a kernel of its own before the up GEMM.  Same results, bit for
 *                          bit.  Off while the shared expert runs on the side stream.
 *   MOE_OPTION_GEMM_CLOCK  1: the bf16 forward's expert GEMMs add each CTA's SM cycles and
 *                          %globaltimer nanoseconds from entry to exit to the workspace's
 *                          status block, for moe_gemm_clock (two 64-bit atomics per CTA);
 *                          0 (default): nothing recorded.  Results are the same either way.
 * MOE_ERR_INVALID_ARG for an unknown option or value. */
#define MOE_OPTION_H_HANDOVER 1
#define MOE_OPTION_SHARED_SIDE_SMS 2
#define MOE_OPTION_ROW_GATHER_IN_GEMM 3
#define MOE_OPTION_GEMM_CLOCK 4
moe_status moe_set_option(moe_handle h, int option, int value);

/* Bytes of device workspace a call with n_tokens tokens needs (0 on bad arguments).
 * The workspace holds the routing scratch, the expert-sorted activations, the SwiGLU
 * outputs h and the per-row expert outputs y between the kernels of one call. */
size_t moe_workspace_size(moe_handle h, int n_tokens);

/* Clears the workspace's device status word (call once after allocating a workspace). */
moe_status moe_workspace_init(moe_handle h, void *ws, size_t ws_bytes, void *stream);

/* Router, selection and permutation ("fused MoE gather/scatter", section 3.2.4): computes
 * logits (written to logits_out if non-null), topk_idx, topk_gate, expert_counts,
 * expert_offsets, perm and slot_row.  `stream` is a cudaStream_t (null = default). */
moe_status moe_route(moe_handle h, const void *x, int n_tokens, float *logits_out,
                     int *topk_idx, float *topk_gate, int *expert_counts, int *expert_offsets,
                     int *perm, int *slot_row, void *ws, size_t ws_bytes, void *stream);

/* Same as moe_route but starting from caller-supplied fp32 logits [n_tokens, E]: selection
 * and permutation are then fully determined by integer-exact rules, which makes the
 * routing outputs comparable bit for bit. */
moe_status moe_route_from_logits(moe_handle h, const float *logits, int n_tokens,
                                 int *topk_idx, float *topk_gate, int *expert_counts,
                                 int *expert_offsets, int *perm, int *slot_row, void *ws,
                                 size_t ws_bytes, void *stream);

/* The whole layer: out = shared + routed_scale * sum_j g_j FFN_{S_t[j]}(x_t).  bf16 runs
 * the expert contractions on tcgen05 tensor cores with fp32 accumulation; h (the operand
 * of the down projection) is rounded to bf16, the per-row expert outputs stay fp32 and the
 * combine sums them in a fixed order in fp32 before one rounding to the output type. */
moe_status moe_forward(moe_handle h, const void *x, int n_tokens, void *out, void *ws,
                       size_t ws_bytes, void *stream);

/* moe_forward that also records caller-created CUDA events (cudaEvent_t, passed as void*)
 * on `stream` around its kernel stages, for per-kernel timing with no profiler attached:
 *   events[0] before the router, then one event after each of the MOE_PROFILE_STAGES
 *   stages: 1 router logits, 2 top-k + gates + chunk histograms, 3 permutation scatter,
 *   4 row gather (bf16 with more than about 12 tokens per expert; empty when the expert-up
 *   kernel gathers the rows of x as it loads them, or, on CTA pairs with
 *   MOE_OPTION_ROW_GATHER_IN_GEMM, writes the sorted copy itself), 5 expert up + SwiGLU,
 *   6 expert down, 7 combine.
 *   For n_tokens <= 64 (bf16) stages 2-3 are one fused launch, timed as stage 2 (3 empty);
 *   with at most 288 experts and d_model <= 8192 stages 1-3 are one launch, timed as stage 1.
 * n_events must be at least MOE_PROFILE_STAGES + 1; otherwise MOE_ERR_INVALID_ARG. */
#define MOE_PROFILE_STAGES 7
moe_status moe_forward_profiled(moe_handle h, const void *x, int n_tokens, void *out,
                                void *ws, size_t ws_bytes, void *stream, void *const *events,
                                int n_events);

/* Number of kernel launches one moe_forward of n_tokens tokens makes on the handle's
 * configuration (the launch plan depends on n_tokens); -1 for a null handle or n_tokens
 * outside [0, max_tokens].  No device work. */
int moe_forward_launch_count(moe_handle h, int n_tokens);

/* Waits for `stream`, then reads and clears the workspace's device status word:
 * MOE_ERR_DEVICE_TIMEOUT if a bounded device wait gave up since the last query. */
moe_status moe_device_status(moe_handle h, void *ws, size_t ws_bytes, void *stream);

/* Effective SM clock of the expert GEMMs of the forwards run on this workspace with
 * MOE_OPTION_GEMM_CLOCK since the last call: mhz[0] the up GEMM's, mhz[1] the down GEMM's
 * (CTA-time-weighted SM cycles per microsecond of %globaltimer; 0 when none ran).  Waits for
 * `stream`, reads the sums and clears them.  Under a power or thermal cap this is the clock
 * the tensor cores actually ran at, which a sampling tool (nvidia-smi) may not resolve inside
 * a millisecond-long kernel.  MOE_ERR_INVALID_ARG on null arguments or a short workspace. */
moe_status moe_gemm_clock(moe_handle h, void *ws, size_t ws_bytes, double *mhz, void *stream);

/* Backward of moe_forward: gradients of <out, dout> with respect to x and the weights, for
 * the forward's own selection (recomputed here with the same kernels; the selection carries
 * no gradient -- the bias only selects, "Step 3.5 Flash 技术论文深度解读", architecture item
 * 1 note).  Chain rule through sections 2.2 / 2.2.2 / 4.1.2 of "Step 3.5 Flash: Open
 * Frontier-Level Intelligence with 11B Active Parameters": the gates are the softmax of the
 * selected unbiased router logits, so the router weights receive
 *   dl_j = g_j (dgate_j - sum_i g_i dgate_i),  dgate_j = routed_scale * (dout_t . y_j),
 * with y_j the unscaled output of the j-th selected expert.
 *   x, dout   [n_tokens, d] layer dtype          dx        [n_tokens, d] fp32 (overwritten)
 *   dw_router [E, d] fp32    dw_gate, dw_up [E + n_shared, f, d] fp32
 *   dw_down   [E + n_shared, d, f] fp32
 * The weight gradients ACCUMULATE (+=) into the caller's buffers, as over micro-batches;
 * rows of experts no token chose are not touched (zero the buffers before the first call).
 * ws: at least moe_backward_workspace_size(h, n_tokens) bytes, 256-byte aligned (it holds a
 * forward workspace at its start, which this call reuses).
 * bf16 layer: the matrix products run on the tensor cores with fp32 accumulation; da, db and
 * routed_scale * gate * h enter the second-stage products rounded to bf16 (each weight
 * gradient and dx term has one rounded operand), dgate and the router terms are computed
 * from fp32 values.  fp32 layer: fp32 throughout on CUDA cores.  Every sum runs in a fixed
 * order and each weight-gradient element receives one addition per call: deterministic.
 * Errors as moe_forward. */
size_t moe_backward_workspace_size(moe_handle h, int n_tokens);
moe_status moe_backward(moe_handle h, const void *x, int n_tokens, const void *dout, float *dx,
                        float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                        void *ws, size_t ws_bytes, void *stream);

/* Training pair (bf16 layer): a forward that keeps what the backward would otherwise
 * recompute, and the backward that uses it -- the per-submodule choice between recomputing
 * activations and keeping them ("Step 3.5 Flash: Open Frontier-Level Intelligence with 11B
 * Active Parameters", section 3.2.5, fine-grained selective checkpointing): moe_backward
 * recomputes the expert pre-activations, this pair keeps them.
 * moe_forward_save is moe_forward (same out, same workspace use) that also writes the fp32
 * pre-activations a = x W_gate^T and b = x W_up^T of every expert-sorted row to `saved`:
 *   saved  [2, P, f] fp32, a then b, P = n_tokens * (top_k + n_shared) rows: the routed rows
 *          in the routing's sorted order (expert-major, ascending token), then the shared
 *          expert's n_tokens rows; at least moe_saved_size(h, n_tokens) bytes, 16-byte aligned
 * moe_backward_saved is moe_backward for a moe_forward_save of the same x and n_tokens (and
 * unchanged weights and router bias, so the routing it recomputes is the same): it reads a
 * and b from `saved` instead of recomputing them (one grouped GEMM over the gate and up
 * weights less); its results are those of moe_backward.
 * MOE_ERR_UNSUPPORTED for the fp32 layer; MOE_ERR_INVALID_ARG for a null or short `saved`,
 * MOE_ERR_ALIGNMENT for a misaligned one; otherwise errors as moe_forward / moe_backward. */
size_t moe_saved_size(moe_handle h, int n_tokens);
moe_status moe_forward_save(moe_handle h, const void *x, int n_tokens, void *out, float *saved,
                            size_t saved_bytes, void *ws, size_t ws_bytes, void *stream);
moe_status moe_backward_saved(moe_handle h, const void *x, int n_tokens, const void *dout,
                              const float *saved, size_t saved_bytes, float *dx,
                              float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                              void *ws, size_t ws_bytes, void *stream);

/* Backward with options: `saved` as in moe_backward_saved (null: recompute, as moe_backward;
 * non-null needs the bf16 layer), and `flags`:
 *   MOE_BACKWARD_OVERWRITE  the weight gradients are SET to this call's gradients instead of
 *                           added (rows of experts no token chose are set to zero), so the
 *                           first micro-batch needs no zeroed buffers and, in the bf16 layer,
 *                           the gradient tiles are stored instead of read, added and written.
 * Results otherwise as moe_backward; MOE_ERR_INVALID_ARG for unknown flags. */
#define MOE_BACKWARD_OVERWRITE 1u
moe_status moe_backward_ex(moe_handle h, const void *x, int n_tokens, const void *dout,
                           const float *saved, size_t saved_bytes, unsigned flags, float *dx,
                           float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                           void *ws, size_t ws_bytes, void *stream);

/* Expert health signals ("Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active
 * Parameters", section 4.1.2: monitor per-expert activation and parameter norms; "Step 3.5
 * Flash 技术论文深度解读", training stability, expert collapse: per-expert activation RMS
 * norm and the min-to-median ratio of parameter Frobenius norms).  Call after moe_forward
 * with the same workspace and n_tokens (it reads that forward's expert activations):
 *   act_rms[g]    (g < E + n_shared) RMS of the SwiGLU activation of expert g over the
 *                 tokens routed to it (every token for the shared expert); 0 if none
 *   param_norm[g] Frobenius norm of W_gate[g], W_up[g] and W_down[g] together
 *   ratios[0]     median / max of act_rms over the routed experts some token chose
 *   ratios[1]     min / median of param_norm over the routed experts
 *                 (median of an even count: mean of the middle two; a ratio whose
 *                 denominator is 0 is reported as 0)
 * Device fp32 outputs; fp64 sums, deterministic.  Reads every expert weight once (about
 * 1.4 ms for 289 full-size experts).  Errors as moe_forward; MOE_ERR_INVALID_ARG for
 * n_tokens == 0 or a null output. */
moe_status moe_expert_health(moe_handle h, int n_tokens, float *act_rms, float *param_norm,
                             float *ratios, void *ws, size_t ws_bytes, void *stream);

/* Self-test of the failure-detection path: launches (asynchronously, on `stream`) one small
 * kernel whose two bounded waits -- on an mbarrier that nothing arrives on and on a flag in
 * the workspace status block that nothing sets -- give up after limit_us microseconds
 * (1 .. 2,000,000) exactly as the layer's waits do when a pipeline stalls; the next
 * moe_device_status() then returns MOE_ERR_DEVICE_TIMEOUT and clears the word.  Nothing
 * faults or traps and the context stays usable.  ws: a workspace of this handle (only its
 * status block is touched).  MOE_ERR_INVALID_ARG for a null handle/workspace or a limit out
 * of range; MOE_ERR_ALIGNMENT if ws is not 256-byte aligned. */
moe_status moe_selftest_wait_timeout(moe_handle h, void *ws, size_t ws_bytes, int limit_us,
                                     void *stream);

/* Balancing statistics of a routing result ("Step 3.5 Flash: Open Frontier-Level
 * Intelligence with 11B Active Parameters", section 2.2.2: EP-group balance loss; section
 * 5.2.3: routing confidence).  From fp32 logits [n_tokens, E] and topk_idx [n_tokens, k]
 * (the outputs of moe_route):
 *   p[t,e]     = softmax of token t's E unbiased logits (its routing probability)
 *   p_mean[e]  = mean_t p[t,e]                       [E] fp32, device
 *   f_sel[e]   = (selections of e) / (n_tokens * k)  [E] fp32, device
 *   scalars[0] = L_EP = G * sum_g f_g * p_g, where f_g, p_g sum f_sel, p_mean over group g
 *                of n_groups groups of E / n_groups consecutive experts (E % n_groups == 0)
 *   scalars[1] = routing confidence = mean_t sum_{e in S_t} p[t,e]
 * Deterministic; uses the workspace of moe_workspace_size(h, n_tokens). */
moe_status moe_router_stats(moe_handle h, const float *logits, const int *topk_idx,
                            int n_tokens, int n_groups, float *p_mean, float *f_sel,
                            float *scalars, void *ws, size_t ws_bytes, void *stream);

/* Loss-free balancing step on a bias vector (fp32 [E], device, updated in place) from the
 * expert_counts of a routing over n_tokens tokens: bias[e] += gamma * sign(n_tokens * k / E -
 * counts[e]) with sign(0) = 0.  The pages balance by adjusting this bias instead of an
 * auxiliary loss ("Step 3.5 Flash 技术论文深度解读", architecture item 1) but give no rule;
 * this sign step toward the mean load is the library's reading. */
moe_status moe_update_router_bias(moe_handle h, const int *expert_counts, int n_tokens,
                                  float gamma, float *bias, void *stream);

/* ------------------------------------------------------------------ expert parallelism
 * The layer split by experts over R ranks ("Step 3.5 Flash: Open Frontier-Level Intelligence
 * with 11B Active Parameters", section 3: the MoE layers run expert-parallel, EP8 within a
 * node over NVLink / NVSwitch; section 2.2.2: the routed experts form G EP groups whose load
 * the EP-group balance loss evens out).  Rank q holds EP group q, the E / R consecutive
 * routed experts [q E / R, (q + 1) E / R) (the grouping moe_router_stats uses), plus the
 * shared expert, and the full router: every rank routes its own tokens over all E experts.
 * The exchanges themselves (all-to-all, all-gather, reduce-scatter) are the caller's (the
 * Python package's expert_parallel module runs them over torch.distributed); these calls
 * are the device steps around them.  bf16 layers only.
 *
 * moe_layer_init_ep: a handle over the routed experts [expert_begin, expert_end) of a layer
 * of cfg->n_experts experts.  w->w_router [E, d] and router_bias [E] are the whole router;
 * w_gate, w_up [(expert_end - expert_begin) + n_shared, f, d] and w_down [.., d, f] hold
 * those experts in order, then the shared expert.  Such a handle routes (moe_route,
 * moe_route_from_logits, moe_router_stats) and runs moe_forward_partial within its range;
 * the whole-layer calls (moe_forward, the backward, moe_expert_health) return
 * MOE_ERR_UNSUPPORTED on it.  moe_layer_init's handle holds [0, E). */
moe_status moe_layer_init_ep(const moe_config *cfg, const moe_weights *w, int expert_begin,
                             int expert_end, moe_handle *out);

/* Part of the layer for n_tokens tokens, unrounded fp32:
 *   out[t] = routed_scale * sum over slots j of t with expert_begin <= idx[t,j] < expert_end
 *            of gate[t,j] FFN_{idx[t,j]}(x_t)
 *          + FFN_shared(x_t) if shared_begin <= t < shared_end (else nothing)
 * with the slots summed in j order and the shared expert last, in fp32.  The selection is
 * topk_idx / topk_gate [n_tokens, k] (device; global expert ids, e.g. routed on another
 * rank; ids outside [0, E) contribute nothing), or, with both null, the layer's own routing
 * of x.  [expert_begin, expert_end) must lie in the handle's experts (it may be empty:
 * shared expert only).  Summing the outputs of calls whose expert ranges partition [0, E)
 * and whose shared ranges partition the tokens gives the layer output before its rounding.
 * A given selection must name distinct experts within each token (as the router's does).
 * out [n_tokens, d] fp32, 16-byte aligned; ws as for moe_forward.  MOE_ERR_UNSUPPORTED for
 * the fp32 layer. */
moe_status moe_forward_partial(moe_handle h, const void *x, int n_tokens, const int *topk_idx,
                               const float *topk_gate, int expert_begin, int expert_end,
                               int shared_begin, int shared_end, float *out, void *ws,
                               size_t ws_bytes, void *stream);

/* Dispatch plan of an all-to-all exchange over n_ranks ranks (E % n_ranks == 0, at most 512
 * ranks) from the tokens' selections topk_idx [n_tokens, k]: token t goes once to every rank
 * q that holds one of its experts.  The (token, rank) pairs are sorted by bucket, ascending
 * token within a bucket: bucket q holds the tokens sent to rank q, bucket n_ranks + q the
 * tokens that send nothing to rank q.  Outputs (device int32):
 *   send_counts  [2 n_ranks]    tokens per bucket: entry q = rows sent to rank q
 *   send_offsets [2 n_ranks + 1] exclusive prefix of send_counts: rank q's rows of the send
 *                               buffer are [send_offsets[q], send_offsets[q + 1])
 *   send_perm    [n_tokens * n_ranks]  row r of the send buffer carries pair send_perm[r]
 *                               = t * n_ranks + q (the first send_offsets[n_ranks] rows)
 *   send_slot    [n_tokens * n_ranks]  inverse: row of pair (t, q), >= send_offsets[n_ranks]
 *                               when t sends nothing to q
 * Deterministic (no atomic decides a position).  Uses the workspace of
 * moe_workspace_size(h, n_tokens). */
moe_status moe_ep_plan(moe_handle h, const int *topk_idx, int n_tokens, int n_ranks,
                       int *send_counts, int *send_offsets, int *send_perm, int *send_slot,
                       void *ws, size_t ws_bytes, void *stream);

/* Send buffer of the plan: row r < send_offsets[n_ranks] gets token t = send_perm[r] /
 * n_ranks: x_send[r] = x[t] (layer dtype, [rows, d], 16-byte aligned), idx_send[r] =
 * topk_idx[t], gate_send[r] = topk_gate[t] ([rows, k]).  The buffers need room for
 * n_tokens * n_ranks rows (the largest possible send); rows past the send are not written. */
moe_status moe_ep_pack(moe_handle h, const void *x, const int *topk_idx, const float *topk_gate,
                       int n_tokens, int n_ranks, const int *send_perm, const int *send_offsets,
                       void *x_send, int *idx_send, float *gate_send, void *stream);

/* Output of the rank's own tokens:
 *   out[t] = round( sum_{q = 0 .. n_ranks - 1, t sent to q} back[send_slot[t n_ranks + q]]
 *                   + shared[t] )
 * in fp32 in this order, one rounding to the layer dtype.  back: the fp32 partial rows the
 * ranks returned, in the send buffer's row order ([send_offsets[n_ranks], d]; null: none,
 * send_slot and send_offsets unused); shared: fp32 [n_tokens, d] (e.g. the shared expert's
 * moe_forward_partial, or a reduce-scattered sum of partials; null: none). */
moe_status moe_ep_combine(moe_handle h, const float *back, const int *send_slot,
                          const int *send_offsets, const float *shared, int n_tokens,
                          int n_ranks, void *out, void *stream);

/* Static description of a status code. */
const char *moe_status_string(moe_status s);

/* Router logits without any caller workspace, for callers that cannot allocate device
 * memory: plugin or embedding hosts that hand the library only its input and output buffers,
 * and latency-critical decode loops that must not touch an allocator.  (No counterpart on
 * the pages: this is a deployment convenience, not part of the layer's method.)
 *
 * Computes logits_out[t, e] = x_t . W_r[e] (fp32, [n_tokens, E], row-major) with a split-K
 * kernel in a fixed summation order (deterministic).  Where moe_route uses the same kernel
 * (fp32 layers; bf16 layers with more than 288 experts or d_model > 8192) the values are
 * identical to moe_route's logits; bf16 decode batches of moe_route go through its one-launch
 * router, which sums in another fixed order, so there the two agree to fp32 rounding of the
 * dot product (each within d_model * 2^-24 * sum_i |x_i w_i| of the exact value).
 * Its scratch (split partial sums and arrival counters)
 * lives in a fixed 2 MiB buffer inside the library's own static device memory, which every
 * GPU that loads the library holds until the process exits.  Limits: 1 <= n_tokens <= 64 and
 * ceil(d_model / 256) * n_tokens * E * 4 bytes <= 2 MiB (for d_model = 4096, E = 288: up to
 * 64 tokens); larger requests return MOE_ERR_UNSUPPORTED before anything is launched.
 * The first call on each device looks up the buffer's device address (host-side set-up).
 * The address is kept for the life of the process: do not use the library across a device
 * reset (cudaDeviceReset), which may move the buffer.  The current device must be the one
 * the handle was created on (MOE_ERR_INVALID_ARG otherwise).  All calls on a device share
 * the one buffer: calls that may overlap on the GPU (different streams without ordering)
 * race and give wrong results; serialise them.  Asynchronous on `stream`. */
moe_status moe_router_logits_static(moe_handle h, const void *x, int n_tokens,
                                    float *logits_out, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_LAYER_H */
