/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of one sparse
 * Mixture-of-Experts layer with shared experts, sigmoid or softmax routing,
 * selection-only expert bias, optional group-limited top-K, optional capacity
 * dropping, SwiGLU experts and the aux-loss-free bias step.
 *
 * The layer computed (notation of the source pages):
 *
 *   y_t = h_t + sum_{j=1..E_s} SwiGLU^S_j(h_t) + sum_{i in I_t} g_{t,i} SwiGLU^R_i(h_t)
 *   SwiGLU(h) = (SiLU(h W_gate^T) * (h W_up^T)) W_down^T
 *   s_{t,i} = sigmoid(h_t . e_i)             (score_fn = MOE_SCORE_SIGMOID)
 *           = softmax_i(h_t . e_i)           (score_fn = MOE_SCORE_SOFTMAX, no bias)
 *   I_t = TopK({s_{t,i} + b_i}, K)  [within the topk_groups best groups]
 *   g_{t,i} = s_{t,i} / max(sum_{j in I_t} s_{t,j}, 1e-12)
 *   b_i <- b_i + gamma * sign(c_bar - c_i),  c_i = #{t : i in I_t},  c_bar = K T / E_r
 *   MaxVio = (max_i c_i - c_bar) / c_bar
 *
 * Sources: "Sparse Mixture-of-Experts (MoE): Routing Math, Load Balancing &
 * Expert Parallelism" (section 0 layer equation; section 2 biased selection,
 * unbiased gates and the sign step; section 3 capacity bound; section 4 MaxVio);
 * "Mixture of Experts: Routing and Load Balancing" (section 2 routing rule;
 * section 5 capacity admits tokens in order); "Load Balancing -- DeepSeek-V3"
 * (How it works: g' and g; Official code: bias before grouped top-k);
 * "GPUs, memory and failures" (worked bias example; the bias card).
 *
 * Conventions for every entry point
 *  - Pointers are DEVICE pointers unless stated otherwise; the caller owns
 *    every buffer (inputs, outputs and the workspace `ws`).  The library never
 *    allocates or frees device memory.  Arrays are dense, row-major, with no
 *    padding.  Activation and weight matrices (h, x, y, slot, shared_out, x_perm,
 *    the expert weights) must be 16-byte aligned; every other array 4-byte
 *    aligned; the workspace 256-byte aligned.
 *  - Activations and expert weights have the element type cfg->dtype
 *    (MOE_DTYPE_F32: float; MOE_DTYPE_BF16: bfloat16 bits in uint16).
 *    MOE_DTYPE_BF16_E4M3: activations bf16, expert weights e4m3 blobs: an
 *    [n, rows, cols] weight tensor is n*rows*cols bytes of e4m3 codes (1 sign,
 *    4 exponent bits with bias 7, 3 mantissa bits, largest finite 448) followed
 *    by n*rows float32 row scales (powers of two); weight (i, r, c) is
 *    code[(i*rows + r)*cols + c] * scale[i*rows + r].  moe_quantize_rows writes
 *    this layout from bf16 or fp32 weights; d_model, d_ffn and d_ffn_shared
 *    must be multiples of 16.
 *    Centroids e, biases b, scores and gates are always float32; indices and
 *    counts are int32.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *    enqueues work on it: no host synchronisation, no device->host copy.
 *  - Errors: arguments are validated on the host first; on any failure the call
 *    returns a non-zero moe_status and enqueues NOTHING
 *    (moe_last_error_detail() describes the failure).  MOE_ERR_CUDA reports a
 *    launch failure.  Faults the kernels detect themselves (a bounded wait that
 *    expired, an index out of range) never trap: they set the error word held in
 *    the workspace, read with moe_get_device_error() after the stream is
 *    synchronised; the outputs of that call are then undefined.
 *  - Shapes: d_model, d_ffn, d_ffn_shared must be multiples of 8 (16-byte
 *    rows); 1 <= K <= min(E_r, 32); E_r <= 1024; E_s <= 8; T >= 1;
 *    n_groups divides E_r; topk_groups * (E_r / n_groups) >= K; group_topn <=
 *    E_r / n_groups.  Larger shapes return MOE_ERR_UNSUPPORTED.
 *  - Determinism: for the same inputs every output is bitwise reproducible
 *    (no floating-point atomics; every sum runs in a fixed order).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 4

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad shape or inconsistent config   */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement       */
  MOE_ERR_WORKSPACE = 3,    /* ws is NULL, misaligned or smaller than required    */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed        */
  MOE_ERR_DEVICE = 5        /* the device error word is set (moe_get_device_error)*/
} moe_status;

enum { MOE_SCORE_SIGMOID = 0, MOE_SCORE_SOFTMAX = 1 };
enum {
  MOE_DTYPE_F32 = 0,
  MOE_DTYPE_BF16 = 1,
  /* bf16 activations (h, y, x, slots, shared_out) with e4m3 expert weights: each
   * weight pointer is an e4m3 blob (moe_quantize_rows), and the rows entering
   * the two expert GEMMs are quantized the same way inside the library */
  MOE_DTYPE_BF16_E4M3 = 2
};

/* device error word values (moe_get_device_error) */
enum {
  MOE_DEVERR_NONE = 0,
  MOE_DEVERR_WAIT_TIMEOUT = 1,   /* a pipeline barrier wait gave up (bounded spin) */
  MOE_DEVERR_INDEX = 2,          /* an expert index outside [0, E_r) was met       */
  MOE_DEVERR_RANGE = 3           /* a layer's fp16 slot row saturated (|v| > 65504) */
};

typedef struct {
  int32_t T;             /* tokens in the batch (h is [T, d_model])                    */
  int32_t d_model;       /* d                                                           */
  int32_t E_r;           /* routed experts                                              */
  int32_t E_s;           /* shared (always-on) experts, 0 allowed                       */
  int32_t K;             /* experts selected per token                                  */
  int32_t d_ffn;         /* routed expert width f                                       */
  int32_t d_ffn_shared;  /* shared expert width f_s (ignored when E_s = 0)              */
  int32_t score_fn;      /* MOE_SCORE_SIGMOID or MOE_SCORE_SOFTMAX                      */
  int32_t n_groups;      /* expert groups for group-limited top-K (1 = no limit)        */
  int32_t topk_groups;   /* groups kept per token                                       */
  int32_t group_topn;    /* a group's score = sum of its top group_topn keys (0 = none) */
  float capacity_factor; /* <= 0: dropless; else C = floor(T*K*CF/E_r) rows per expert  */
  int32_t dtype;         /* MOE_DTYPE_F32, MOE_DTYPE_BF16 or MOE_DTYPE_BF16_E4M3         */
  int32_t add_residual;  /* 1: y includes h_t                                           */
  int32_t train;         /* 1: moe_layer_forward keeps what moe_layer_backward needs in
                            the workspace (bf16 layers; d_model, d_ffn, d_ffn_shared
                            multiples of 64); 0: inference                             */
} moe_config;

/* Library ABI version (MOE_ABI_VERSION). */
int32_t moe_abi_version(void);

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status s);

/* Text describing the last failed validation in this thread (static buffer). */
const char* moe_last_error_detail(void);

/*
 * Required workspace bytes for moe_layer_forward with this config (an upper
 * bound for every other entry point with the same config).  *bytes is a HOST
 * pointer.  The workspace must be 256-byte aligned device memory; its first
 * 256 bytes are the library's control block (the device error word and the
 * GEMM unit counters), which the caller must zero once (cudaMemset) before
 * first use.
 */
moe_status moe_workspace_size(const moe_config* cfg, size_t* bytes);

/*
 * Router: affinity, selection and gates (steps a1-a4).
 *   h      [T, d]   activations (cfg->dtype); may be NULL when s_in is given.
 *   e      [E_r, d] float32 centroids; may be NULL when s_in is given.
 *   b      [E_r]    float32 selection bias, or NULL for b = 0 (ignored for softmax).
 *   s_in   [T, E_r] float32 scores to route from ("fed" mode: skips the affinity),
 *                   or NULL to compute s from h and e (fp32 logits).
 *   s_out  [T, E_r] float32: the scores used, or NULL.
 *   z_out  [T, E_r] float32: the fp32 logits h_t . e_i, or NULL (not written
 *                   in fed mode, when there are no logits).
 *   idx    [T, K]   int32 out: I_t in ascending expert index.
 *   gates  [T, K]   float32 out: g_{t,i} in the same order.
 *   counts [E_r]    int32 out: c_i (before any capacity drop), or NULL.
 * Selection keys are s + b in fp32; ties choose the lower expert (group) index.
 * Sources: "Sparse Mixture-of-Experts ...", section 2 equation; "Load
 * Balancing -- DeepSeek-V3", How it works / Official code.
 */
moe_status moe_route(const moe_config* cfg, const void* h, const float* e, const float* b,
                     const float* s_in, float* s_out, float* z_out, int32_t* idx, float* gates,
                     int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * Dispatch: a stable permutation of the (token, slot) pairs grouped by expert
 * (step a5).  Rows of expert i are offsets[i] .. offsets[i+1]-1, tokens ascending;
 * with capacity, at most C = floor(T*K*CF/E_r) rows per expert (lowest token
 * indices kept, "Sparse Mixture-of-Experts ...", section 3; "Mixture of
 * Experts: Routing and Load Balancing", section 5).
 *   idx      [T, K]      int32 in (from moe_route).
 *   gates    [T, K]      float32 in, or NULL (then row_gate is not written).
 *   h        [T, d]      activations, or NULL (then x_perm is not written).
 *   offsets  [E_r + 1]   int32 out.        kept [E_r] int32 out (rows kept).
 *   perm_tok [T*K]       int32 out: token of each row (first offsets[E_r] valid).
 *   row_of   [T, K]      int32 out: row of (t, k), -1 when dropped.
 *   row_gate [T*K]       float32 out: gate of each row, or NULL.
 *   x_perm   [T*K, d]    out: h[perm_tok[r]] for each row, or NULL.
 */
moe_status moe_permute(const moe_config* cfg, const int32_t* idx, const float* gates,
                       const void* h, int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                       int32_t* kept, float* row_gate, void* x_perm, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Grouped SwiGLU experts (steps a6-a7) over expert-contiguous rows:
 *   out[r] = row_scale[r] * SwiGLU_g(x[r])  for offsets[g] <= r < offsets[g+1].
 *   n_experts    number of weight sets (groups); offsets is [n_experts + 1] on the
 *                device; offsets[n_experts] <= max_rows (host-known bound).
 *   d_ffn        expert width f (cfg->d_model is the model width d).
 *   x            [max_rows, d];  w_gate, w_up [n_experts, f, d];  w_down [n_experts, d, f].
 *   row_scale    [max_rows] float32, or NULL for 1.
 *   out          [max_rows, d], cfg->dtype.  Rows >= offsets[n_experts] untouched.
 * bf16 runs on the tensor cores (tcgen05, fp32 accumulation in TMEM; the SwiGLU
 * product is rounded to bf16 before W_down); fp32 runs on CUDA cores in fp32.
 * bf16 inference with max_rows >= 512 * n_experts (many rows per expert, as in
 * a dropless layer with T*K/E_r >= 512) runs both GEMMs on CTA pairs (clusters
 * of two CTAs, tcgen05 cta_group::2, 256-row tiles): the same arithmetic, with
 * the tensor core's own summation order inside each 16-element step.
 */
/* Workspace bytes moe_expert_ffn needs for these arguments (*bytes: HOST pointer). */
/*
 * Row-tile height of the GEMMs moe_expert_ffn runs for these arguments
 * (*rows: HOST pointer): 256 when both GEMMs run on CTA pairs, 128 for the
 * single-CTA tensor-core GEMMs, the CUDA-core tile for fp32.  moe_layer_forward
 * makes the same choice with n_experts = E_r and max_rows = its routed rows
 * (T*K, or E_r times the capacity), except that a training forward
 * (cfg->train) keeps the single-CTA GEMMs.  Queries the current device's
 * cluster occupancy once; launches nothing.
 */
moe_status moe_expert_ffn_tile_rows(const moe_config* cfg, int32_t n_experts, int32_t max_rows,
                                    int32_t* rows);
moe_status moe_expert_ffn_workspace_size(const moe_config* cfg, int32_t n_experts, int32_t d_ffn,
                                         int32_t max_rows, size_t* bytes);

moe_status moe_expert_ffn(const moe_config* cfg, int32_t n_experts, int32_t d_ffn,
                          int32_t max_rows, const int32_t* offsets, const void* x,
                          const void* w_gate, const void* w_up, const void* w_down,
                          const float* row_scale, void* out, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * Combine (step a8):  y_t = add_residual*h_t + sum_j shared_out[j, t]
 *                           + sum_{k ascending, row_of[t,k] >= 0} slot[row_of[t,k]]
 * accumulated in fp32 in exactly that order and rounded once to cfg->dtype.
 *   slot       [rows, d]  gate-scaled routed expert outputs (cfg->dtype).
 *   shared_out [E_s, T, d] shared expert outputs, or NULL when E_s = 0.
 *   row_of     [T, K] int32.    y [T, d] out.
 */
moe_status moe_combine(const moe_config* cfg, const void* h, const void* slot,
                       const void* shared_out, const int32_t* row_of, void* y, void* stream);

/*
 * Bias step (step a9), once per training step after the batch's loads are
 * counted ("GPUs, memory and failures", the bias card; "Sparse
 * Mixture-of-Experts ...", section 2):
 *   b_i <- b_i + gamma * sign(K*T - E_r*c_i)   (sign(0) = 0; one fp32 add)
 *   counts [E_r] int32 in;  b [E_r] float32 in/out;
 *   max_vio: float32 device scalar out ((max c - c_bar)/c_bar), or NULL.
 */
moe_status moe_bias_update(const moe_config* cfg, const int32_t* counts, float gamma, float* b,
                           float* max_vio, void* stream);

/*
 * The whole layer (a1-a8, and a9 when update_bias != 0), on one stream with no
 * host synchronisation.
 *   h [T, d]; e [E_r, d] float32; b [E_r] float32 (read, and updated in place
 *   when update_bias); w_gate/w_up [E_r, f, d], w_down [E_r, d, f];
 *   ws_gate/ws_up [E_s, f_s, d], ws_down [E_s, d, f_s] (NULL when E_s = 0).
 *   y [T, d] out.  Optional outputs (NULL to skip): idx_out [T, K],
 *   gates_out [T, K], counts_out [E_r], kept_out [E_r], s_out [T, E_r],
 *   z_out [T, E_r] (fp32 logits; not written in fed mode),
 *   max_vio_out (device float32 scalar; written whenever non-NULL).
 *   s_in: optional fed scores [T, E_r] (skips the affinity; e may then be NULL).
 * With update_bias, the routing of THIS call uses the incoming b and the step
 * is applied afterwards (the bias is carried to the next step).
 * Inside the workspace a bf16 layer keeps the gate-weighted expert rows and
 * the shared experts' outputs in fp16 (11 significant bits, 2 bytes) until the
 * combine adds them in fp32: a value beyond +-65504 saturates and sets
 * MOE_DEVERR_RANGE.  The standalone moe_expert_ffn / moe_combine keep cfg->dtype.
 */
moe_status moe_layer_forward(const moe_config* cfg, const void* h, const float* e, float* b,
                             const void* w_gate, const void* w_up, const void* w_down,
                             const void* ws_gate, const void* ws_up, const void* ws_down,
                             const float* s_in, void* y, int32_t* idx_out, float* gates_out,
                             int32_t* counts_out, int32_t* kept_out, float* s_out, float* z_out,
                             int32_t update_bias, float gamma, float* max_vio_out,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Router losses and logging over one batch (training-time reductions over the
 * routing results; none of them changes the forward output):
 *   stats[0] Switch auxiliary loss  alpha_aux * sum_i f_i P_i,
 *            f_i = E_r/(K T) c_i, P_i = mean_t s'_{t,i}, s' = s / sum_j s_j
 *            ("Sparse Mixture-of-Experts ...", section 1 equation; for softmax
 *            routing s' = p);
 *   stats[1] router z-loss  c_z / T * sum_t (logsumexp_i z_{t,i})^2 (same
 *            section), 0 when z is NULL;
 *   stats[2] sequence-wise balance loss ("Load Balancing -- DeepSeek-V3", How
 *            it works): alpha_seq * sum_i f_i P_i within each sequence of
 *            seq_len tokens (f_i normalised by K*seq_len), averaged over the
 *            T/seq_len sequences; 0 when seq_len = 0;
 *   stats[3] entropy of the load shares c_i / (K T) ("GPUs, memory and
 *            failures", log_router);
 *   stats[4] MaxVio;  stats[5] dropped rate 1 - sum kept / (K T) (0 when kept
 *            is NULL).
 *   s [T, E_r] scores and z [T, E_r] logits (NULL allowed) as exported by
 *   moe_route / moe_layer_forward; idx [T, K]; kept [E_r] or NULL;
 *   stats: 6 float32 on the device.  seq_len must be 0 or divide T.
 *   ws: at least moe_router_stats_workspace_size bytes (its first 256 bytes
 *   are not used by this call).  Deterministic (no floating-point atomics).
 */
/*
 * Row gather for expert-parallel layouts (no counterpart step on the pages;
 * the regrouping that an all-to-all dispatch needs, "Sparse Mixture-of-Experts
 * ...", section 3 and "Mixture-of-Experts: Expert Parallelism, All-to-All
 * Routing, ...", expert parallelism): dst[r] = src[map[r]] for r < n_rows, a
 * zero row where map[r] < 0.  Rows are row_bytes long (a multiple of 4; src
 * and dst 16-byte aligned when it is a multiple of 16).  map[r] >= n_src is
 * reported through no error word here: the row is skipped (callers pass maps
 * they built).  Enqueues one kernel; no host synchronisation.
 */
moe_status moe_gather_rows(const void* src, int64_t n_src, int32_t row_bytes, const int32_t* map,
                           int64_t n_rows, void* dst, void* stream);

/*
 * Exchange plan of an expert-parallel layer ("Sparse Mixture-of-Experts ...",
 * section 3: dispatch to the experts' ranks, grouped GEMM over the local
 * experts, combine; "Mixture-of-Experts: Expert Parallelism, All-to-All
 * Routing, ...", all-to-all routing).  The E_r routed experts are split over
 * `world` ranks, rank r owning experts r*E_loc .. (r+1)*E_loc - 1
 * (E_loc = E_r / world); every rank has permuted its own kept rows with
 * moe_permute, so its rows for rank r are one contiguous range.
 *   offsets_all [world, E_r + 1] int32: every rank's moe_permute offsets
 *                (all-gathered), DEVICE.
 *   splits      [2 * world] int32 out: rows this rank sends to each rank, then
 *                rows it receives from each rank (the all-to-all split sizes).
 *   local_offsets [E_loc + 1] int32 out: rows of each local expert after the
 *                regroup.
 *   regroup     [max_recv] int32 out: regrouped row j comes from received
 *                row regroup[j] -- received rows arrive source by source, the
 *                regroup orders them expert by expert, sources ascending, each
 *                source's rows in their order.
 *   inverse     [max_recv] int32 out: inverse[regroup[j]] = j.
 *   dev_error   optional int32 DEVICE word: set to MOE_DEVERR_INDEX when the
 *                offsets decrease or more than max_recv rows would arrive (the
 *                maps are then not written; splits still are).
 * 1 <= world <= 64, 0 <= rank < world, E_r <= 1024 and divisible by world.
 * Enqueues one kernel; the caller copies `splits` to the host if its
 * all-to-all needs them there.
 */
moe_status moe_ep_plan(const int32_t* offsets_all, int32_t world, int32_t rank, int32_t E_r,
                       int32_t max_recv, int32_t* splits, int32_t* local_offsets, int32_t* regroup,
                       int32_t* inverse, int32_t* dev_error, void* stream);

/*
 * Backward of moe_layer_forward (train = 1): gradients of a loss L, given
 * dy = dL/dy [T, d] (bf16), with respect to h, the centroids e and every
 * expert weight, for the routing the forward chose.  The derivative of the
 * layer equation ("Sparse Mixture-of-Experts ...", section 0) per expert,
 * through the gates g = s / sum_{I_t} s (section 2: the selection uses s + b,
 * the gates s alone, so no gradient reaches the bias b, and the top-K choice
 * and capacity drops are held fixed).
 *
 *   h, e, weights: the forward's inputs; s [T, E_r] fp32 and idx [T, K] the
 *   scores and selections the forward exported (s_out, idx_out).
 *   ws: the workspace of the forward call just before, with the same cfg
 *   (train = 1) -- it still holds the permutation, x, U | V, A and the
 *   slots; this call overwrites its group tables.
 *   Outputs: dh [T, d] bf16 (residual + shared + routed + router terms, summed
 *   in fp32 in a fixed order); de [E_r, d] fp32; dW_gate, dW_up [E_r, f, d],
 *   dW_down [E_r, d, f] bf16 (zero for experts without kept rows); the shared
 *   experts' dWs_* likewise (NULL when E_s = 0).
 *   Deterministic (no floating-point atomics).
 */
moe_status moe_layer_backward(const moe_config* cfg, const void* h, const float* e, const float* s,
                              const int32_t* idx, const void* w_gate, const void* w_up,
                              const void* w_down, const void* ws_gate, const void* ws_up,
                              const void* ws_down, const void* dy, void* dh, float* de,
                              void* dw_gate, void* dw_up, void* dw_down, void* dws_gate,
                              void* dws_up, void* dws_down, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * Low-precision expert weights ("GPUs, memory and failures", serving notes:
 * lower-precision expert weights when serving is bound by streaming them; the pages
 * fix no format -- this is the library's): e4m3 codes with one power-of-two
 * scale per row, the smallest s with max_c |x[r][c]| / s <= 448 (at least
 * 2^-126; 1 for an all-zero row), each element x / s rounded to the nearest
 * e4m3 value, ties to the even code, saturating at +-448.
 *
 * moe_quantized_bytes: size of the blob for n_rows x cols (cols a positive
 *   multiple of 16): n_rows*cols code bytes + n_rows*4 scale bytes.
 * moe_quantize_rows: src [n_rows, cols] (src_dtype MOE_DTYPE_BF16 or
 *   MOE_DTYPE_F32, 16-byte aligned, finite values) -> dst blob (16-byte
 *   aligned, moe_quantized_bytes long).  Deterministic, bit-exact with the
 *   definition above.  For the e4m3 layers quantize each weight tensor as
 *   n_rows = experts * rows.
 */
moe_status moe_quantized_bytes(int64_t n_rows, int32_t cols, size_t* bytes);
moe_status moe_quantize_rows(const void* src, int32_t src_dtype, int64_t n_rows, int32_t cols, void* dst,
                             void* stream);

moe_status moe_router_stats_workspace_size(const moe_config* cfg, int32_t seq_len, size_t* bytes);
moe_status moe_router_stats(const moe_config* cfg, const float* s, const float* z, const int32_t* idx,
                            const int32_t* kept, int32_t seq_len, float alpha_aux, float c_z,
                            float alpha_seq, float* stats, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device
 * memory for one (a caller whose device memory all belongs to its own pool, a
 * caller enqueuing work while another thread captures a CUDA graph, a
 * latency-critical caller that cannot accept cudaMalloc's implicit
 * synchronisation).  The pages have no counterpart: this is a deployment
 * variant of moe_permute with the same arguments, outputs and results,
 * minus ws/ws_bytes.
 *   dev_error: optional int32 DEVICE word that receives MOE_DEVERR_INDEX if an
 *   expert index outside [0, E_r) is met (NULL: not reported).
 * Scratch: a fixed 2 MiB + 64 KiB array in the library's own device memory,
 * held on every GPU that loads the library until exit.  Shapes needing more
 * (2 * ceil(T/256) * E_r + E_r + 64 int32 words) return MOE_ERR_UNSUPPORTED
 * before anything is enqueued.  The first call in each CUDA context (once per
 * device for the primary context; again after cudaDeviceReset rebuilds it)
 * looks up the array's device address (cudaGetSymbolAddress) and must
 * therefore come before any stream capture.  All calls share the array and it keeps the last call's
 * contents (the call clears what must start at zero): calls whose work
 * overlaps on the GPU, e.g. on two streams, race and must be serialised by the
 * caller.  No cudaMalloc/cudaFree or allocating library routine is called.
 */
moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* idx, const float* gates,
                               const void* h, int32_t* offsets, int32_t* perm_tok,
                               int32_t* row_of, int32_t* kept, float* row_gate, void* x_perm,
                               int32_t* dev_error, void* stream);

/*
 * Profiling support.  When n_events > 0, every later moe_layer_forward call in
 * this thread records the caller's CUDA events (cudaEvent_t handles, created
 * and owned by the caller) on its stream at the phase boundaries:
 *   0 start; 1 after routing (a1-a4); 2 after dispatch (a5); 3 after the FFN
 *   group tables; 4 after the gate/up GEMM (a6); 5 after the down GEMM (a7);
 *   6 after the combine (a8); 7 after the bias step (a9).
 * Only the first n_events (<= 8) are recorded; n_events = 0 turns it off.
 */
moe_status moe_set_phase_events(void* const* events, int32_t n_events);

/*
 * Read (synchronously, via cudaMemcpy) the device error word of a workspace
 * after the stream that used it has been synchronised.  *code is a HOST
 * pointer.  Returns MOE_ERR_DEVICE when the word is non-zero, MOE_OK otherwise.
 */
moe_status moe_get_device_error(const void* ws, int32_t* code);

/*
 * Failure-detection self-test.  Enqueues one kernel whose only thread waits,
 * through the same bounded shared-memory-barrier wait every GEMM pipeline
 * stage uses, on a barrier that nothing ever arrives on.  After limit_ns
 * (1 ms .. 2 s) the wait gives up, writes MOE_DEVERR_WAIT_TIMEOUT into the
 * error word of ws (the first 256 bytes of a workspace) and the kernel
 * returns: no trap, no hang, the context stays usable.  Read the word with
 * moe_get_device_error after synchronising the stream.
 */
moe_status moe_selftest_bounded_wait(void* ws, int64_t limit_ns, void* stream);

/* Zero the device error word of a workspace (enqueued on stream). */
moe_status moe_clear_device_error(void* ws, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
