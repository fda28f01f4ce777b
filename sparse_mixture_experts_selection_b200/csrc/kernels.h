// Internal launchers of the MoE library (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

// Arguments of the grouped SwiGLU FFN over routed groups (rows
// grp_row0[g] .. +grp_rows[g] of x_r / act_r / out_r, weights of expert g) and
// shared groups (all T rows of x_s, rows j*T.. of act_s / out_s).
struct FfnArgs {
  int dtype, T, d, f_r, f_s, E_r, E_s, max_rows_r;
  const void *x_r, *x_s;
  const void *wg_r, *wu_r, *wd_r, *wg_s, *wu_s, *wd_s;
  const int *grp_rows, *grp_row0, *pre_gu, *pre_dn;
  const float* row_scale;
  void *act_r, *act_s, *out_r, *out_s;
  int* err;
  int* tile_counters;   // [2] unit counters of the two GEMMs, zeroed by groups_kernel
  // e4m3 expert weights (q8 = 1): x_r / x_s and the weights are e4m3 codes
  // (weights: blobs of codes followed by fp32 row scales), xs_r / xs_s the row
  // scales of x; the SwiGLU output act_* (bf16) is quantized into actq_* with
  // row scales as_* before the down GEMM
  int q8;
  const float *xs_r, *xs_s;
  void *actq_r, *actq_s;
  float *as_r, *as_s;
  // training forward: U | V of every row ([rows, 2f] bf16) for the backward
  void *uv_r, *uv_s;
  // 1: run both GEMMs on CTA pairs (tc_pair_rows()-row tiles; the group
  // tables were built with that tile height)
  int pair;
  // 1: the down GEMM writes out_r / out_s in fp16 (saturating, MOE_DEVERR_RANGE)
  // instead of bf16 -- the layer's internal slot and shared rows
  int out_f16;
};

void launch_router_logits(const void* h, int dtype, const float* e, float* z, int T, int d, int E,
                          cudaStream_t st);
// in: n_parts arrays [T, E] (logits partial sums, added in order) or the scores
void launch_select(const float* in, int n_parts, int in_is_scores, const float* bias, int score_fn,
                   float* s_out, float* z_out, int32_t* idx, float* gates, int* hist, int chunk_shift,
                   int T, int E, int K, int n_groups, int topk_groups, int group_topn, cudaStream_t st);
void launch_hist(const int32_t* idx, int* hist, int chunk_shift, int T, int K, int E, int* err,
                 cudaStream_t st);
void launch_counts(const int* hist, int n_chunks, int E, int* counts, cudaStream_t st);
void launch_scan(const int* hist, int n_chunks, int E, int cap, int* counts, int* kept,
                 int* offsets, int* chunk_base, cudaStream_t st);
void launch_groups(const int* offsets, int E_r, int E_s, int T, int bm, int merge_max, int nt_gu_r, int nt_gu_s,
                   int nt_dn_r, int nt_dn_s, int* grp_rows, int* grp_row0, int* pre_gu,
                   int* pre_dn, int max_rows, int* err, int* tile_counters, cudaStream_t st);
void launch_scatter(const int32_t* idx, const float* gates, const int* offsets,
                    const int* chunk_base, int cap, int T, int K, int E, int32_t* perm_tok,
                    int32_t* row_of, float* row_gate, int* err, cudaStream_t st);
// x_perm[r] = h[perm_tok[r]] (rows of d * elem_bytes bytes, a multiple of 16)
// for r < *n_rows_ptr; with s_src also s_dst[r] = s_src[perm_tok[r]]
void launch_gather(const void* h, const int32_t* perm_tok, const int* n_rows_ptr, void* x_perm,
                   int d, int elem_bytes, int max_rows, int n_tok, int* err, cudaStream_t st,
                   const float* s_src = nullptr, float* s_dst = nullptr);
// slot_f16: slot and shared rows are fp16 (a bf16 layer's internal rows)
void launch_combine(const void* h, const void* slot, const void* shared, const int32_t* row_of,
                    void* y, int T, int d, int K, int E_s, int add_residual, int dtype,
                    int n_slot_rows, cudaStream_t st, int slot_f16 = 0);
void launch_bias_update(const int* counts, float* b, float gamma, float* max_vio, int E, int K,
                        int T, cudaStream_t st);
void launch_gather_map(const void* src, const int32_t* map, int64_t n_rows, int64_t n_src, int row_bytes,
                       void* dst, int* err, cudaStream_t st);
void launch_bounded_wait_selftest(uint64_t limit_ns, int* err, cudaStream_t st);
// Tokens per partial sum of the per-sequence score means (router statistics).
constexpr int kStatsChunk = 64;
void launch_router_stats(const float* s, const float* z, const int32_t* idx, const int32_t* kept,
                         int T, int E, int K, int seq_len, int use_seq, float alpha_aux, float c_z,
                         float alpha_seq, float* rowsum, float* lse2, int* seq_counts, float* pseq,
                         float* stats, cudaStream_t st);

// e4m3 rows with one power-of-two scale per row (src_dtype 1 = bf16, else fp32;
// cols a multiple of 16).  Row r reads source row src_row[r] (< n_src) when
// src_row is given, else row r; rows at or beyond *n_rows_ptr (when given) are
// skipped.
void launch_quantize_rows(const void* src, int src_dtype, const int32_t* src_row, int n_src,
                          const int* n_rows_ptr, int64_t n_rows, int cols, uint8_t* codes,
                          float* scales, int* err, cudaStream_t st);

int simt_bm();
int simt_bn();
void launch_ffn_simt(const FfnArgs& a, int which, cudaStream_t st);

// Router logits on the tensor cores: split e into three bf16 terms (e3 =
// [3, E, d] bf16 scratch) and write fp32 partial logits zpart [ks, T, E] over
// ks split-K ranges (summed in order by the select kernel).
// At most kRouterMaxSplits partials (kRouterMaxSplitsSmallT for batches of
// at most kRouterSmallT tokens, where one row tile leaves most SMs idle unless
// the reduction is cut finer); the select kernel adds them in split order,
// loading 64 partial values per lane at a time.
constexpr int kRouterMaxSplits = 16;
constexpr int kRouterMaxSplitsSmallT = 64;
constexpr int kRouterSmallT = 1024;
constexpr int kRouterMaxKbPerSplit = 24;
inline int router_max_splits(int T) { return T <= kRouterSmallT ? kRouterMaxSplitsSmallT : kRouterMaxSplits; }
void router_split_plan(int T, int d, int E, int n_sms, int* ks, int* per);
cudaError_t launch_router_tc(const void* h, const float* e, void* e3, float* zpart, int T, int d,
                             int E, int* err, int* ks_out, cudaStream_t st);

// Backward of the grouped SwiGLU experts (tcgen05, bf16): which 0 = dU|dV from
// dO and W_d; 1 = dX from dU|dV and W_g, W_u; 2, 3, 4 = dW_d, dW_g, dW_u.
// Routed rows are the permuted rows (grp_rows / grp_row0 of the routed
// groups); shared groups cover all T tokens (rows j*T.. of their buffers).
struct BwdArgs {
  int T, d, f_r, f_s, E_r, E_s, max_rows_r;
  const void *dO_r, *dy;                 // g*dy per permuted row [R, d]; dy [T, d]
  const void *wg_r, *wu_r, *wd_r, *wg_s, *wu_s, *wd_s;
  const void *uv_r, *uv_s;               // saved U | V [rows, 2f]
  void *duv_r, *duv_s;                   // dU | dV [rows, 2f]
  void *dx_r, *dx_s;                     // dX [rows, d]
  const void *x_r, *h;                   // permuted rows x [R, d]; h [T, d]
  const void *act_r, *act_s;             // A = SiLU(U) V [rows, f]
  void *dwg_r, *dwu_r, *dwd_r, *dwg_s, *dwu_s, *dwd_s;
  const int *grp_rows, *grp_row0, *pre_da, *pre_dx;
  int* err;
};
cudaError_t launch_bwd_tc(const BwdArgs& a, int which, cudaStream_t st);
int bwd_merge_rows();   // backward dA / dX: tails of <= this many rows share the unit before

// Backward of routing and combine (bf16 activations): per permuted row dO and
// dL/dg; per token dz, dh; per expert de.
struct BwdRouteArgs {
  int T, d, E, K, E_s, score_fn, add_residual, max_rows;
  const uint16_t *dy, *slot, *dx_r, *dx_s, *h;
  const int32_t *perm_tok, *row_of, *idx;
  const int* n_rows_ptr;
  const float *row_gate, *s, *e;
  uint16_t *dO, *dh;
  float *dg_row, *dz, *de;
  const int32_t* sel_tok;    // sigmoid: every selected (t, j) by expert, tokens ascending
  const int* sel_off;        // [E + 1] its offsets
  int* err;
  int slot_f16;              // slot rows in fp16 (the layer's), else bf16
};
void launch_bwd_route(const BwdRouteArgs& a, cudaStream_t st);        // dO, dL/dg
void launch_zero_tail_rows(void* buf, const int* n_rows_ptr, int max_rows, int cols, cudaStream_t st);
void launch_bwd_gate_dh_de(const BwdRouteArgs& a, cudaStream_t st);   // dz, dh, de

int tc_bm();
int tc_merge_rows();   // tails of <= this many rows share the unit of the tile before
// CTA-pair GEMMs: rows per pair tile, and the mean routed rows per expert from
// which bf16 inference layers use them
int tc_pair_rows();
int tc_pair_min_rows();
int tc_pair_merge_rows();   // pair kernel: tails of <= this many rows share the unit before
bool tc_pair_available();   // the device co-schedules enough CTA pairs of the pair kernel
int tc_cols_gateup();
int tc_cols_down();
// which = 0: gate/up GEMM + SwiGLU epilogue; which = 1: down GEMM + gate scaling
cudaError_t launch_ffn_tc(const FfnArgs& a, int which, cudaStream_t st);

}  // namespace moe
