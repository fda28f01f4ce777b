// Host side of the C ABI declared in include/moe.h: argument validation,
// workspace layout and the launch sequence of each entry point.  Every entry
// point validates first and enqueues nothing on failure; none allocates.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local char g_detail[512] = "";

moe_status fail(moe_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

constexpr int kChunkShift = 8;          // histogram chunk = 256 tokens (the scatter block)
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
// bytes of an activation element (h, y, x_perm, A, slots): 2 for the bf16 and
// e4m3-weight layers (bf16; a layer's own slot rows fp16), 4 for fp32 layers
size_t elem_bytes(int dtype) { return dtype == MOE_DTYPE_F32 ? 4 : 2; }
int act_dtype(int dtype) { return dtype == MOE_DTYPE_F32 ? MOE_DTYPE_F32 : MOE_DTYPE_BF16; }
bool is_q8(int dtype) { return dtype == MOE_DTYPE_BF16_E4M3; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t capacity_rows(const moe_config& c) {
  const int64_t tk = (int64_t)c.T * c.K;
  if (!(c.capacity_factor > 0.0f)) return tk;
  double cap = std::floor((double)c.T * (double)c.K * (double)c.capacity_factor / (double)c.E_r);
  if (cap > (double)tk) return tk;
  return (int64_t)cap;
}

struct Layout {
  size_t err, scores, hist, chunk_base, counts, kept, offsets, grp_rows, grp_row0, pre_gu, pre_dn;
  size_t idx, gates, row_of, perm_tok, row_gate, maxvio, x_perm, act_r, act_s, slot_r, slot_s, e3;
  // e4m3-weight layers: row scales of x_perm (codes), the e4m3 copy of h and its
  // scales (shared experts), the e4m3 copies of A and their scales
  size_t xs, hq, hs, actq_r, actq_s, as_r, as_s;
  // training: U | V kept by the forward; the backward's dO, dL/dg, dz, dU | dV, dX
  size_t uv_r, uv_s, dO, dg_row, dz, duv_r, duv_s, dx_r, dx_s;
  // every selected (token, expert) pair by expert (dropped ones included)
  size_t sel_tok, sel_row_of, sel_off, sel_base, sel_counts, sel_kept;
  size_t total;
  int n_chunks;
  int64_t cap, R;
};

Layout make_layout(const moe_config& c) {
  Layout L{};
  const size_t es = elem_bytes(c.dtype);
  const int G = c.E_r + c.E_s;
  L.n_chunks = (c.T + (1 << kChunkShift) - 1) >> kChunkShift;
  L.cap = capacity_rows(c);
  int64_t R = std::min<int64_t>((int64_t)c.T * c.K, (int64_t)c.E_r * L.cap);
  L.R = R < 1 ? 1 : R;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  L.err = take(kAlign);
  // fp32 logits: split-K partial sums of the tensor-core router (bf16 layers)
  // or the CUDA-core logits (fp32 layers)
  const bool tcr = c.dtype != MOE_DTYPE_F32;          // tensor-core router
  L.scores = take((size_t)(tcr ? moe::router_max_splits(c.T) : 1) * c.T * c.E_r * 4);
  L.e3 = take(tcr ? (size_t)3 * c.E_r * c.d_model * 2 : 0);
  L.hist = take((size_t)L.n_chunks * c.E_r * 4);
  L.chunk_base = take((size_t)L.n_chunks * c.E_r * 4);
  L.counts = take((size_t)c.E_r * 4);
  L.kept = take((size_t)c.E_r * 4);
  L.offsets = take((size_t)(c.E_r + 1) * 4);
  L.grp_rows = take((size_t)G * 4);
  L.grp_row0 = take((size_t)G * 4);
  L.pre_gu = take((size_t)(G + 1) * 4);
  L.pre_dn = take((size_t)(G + 1) * 4);
  L.idx = take((size_t)c.T * c.K * 4);
  L.gates = take((size_t)c.T * c.K * 4);
  L.row_of = take((size_t)c.T * c.K * 4);
  L.perm_tok = take((size_t)L.R * 4);
  L.row_gate = take((size_t)L.R * 4);
  L.maxvio = take(4);
  const bool q8 = is_q8(c.dtype);
  const size_t fs = c.E_s ? c.d_ffn_shared : 0;
  L.x_perm = take((size_t)L.R * c.d_model * (q8 ? 1 : es));
  L.act_r = take((size_t)L.R * c.d_ffn * es);
  L.act_s = take((size_t)c.E_s * c.T * fs * es);
  L.slot_r = take((size_t)L.R * c.d_model * es);
  L.slot_s = take((size_t)c.E_s * c.T * c.d_model * es);
  L.xs = take(q8 ? (size_t)L.R * 4 : 0);
  L.hq = take(q8 ? (size_t)c.T * c.d_model : 0);
  L.hs = take(q8 ? (size_t)c.T * 4 : 0);
  L.actq_r = take(q8 ? (size_t)L.R * c.d_ffn : 0);
  L.actq_s = take(q8 ? (size_t)c.E_s * c.T * fs : 0);
  L.as_r = take(q8 ? (size_t)L.R * 4 : 0);
  L.as_s = take(q8 ? (size_t)c.E_s * c.T * 4 : 0);
  const bool tr = c.train != 0;
  const size_t rs = (size_t)c.E_s * c.T;
  L.uv_r = take(tr ? (size_t)L.R * 2 * c.d_ffn * 2 : 0);
  L.uv_s = take(tr ? rs * 2 * fs * 2 : 0);
  L.dO = take(tr ? (size_t)L.R * c.d_model * 2 : 0);
  L.dg_row = take(tr ? (size_t)L.R * 4 : 0);
  L.dz = take(tr ? (size_t)c.T * c.E_r * 4 : 0);
  L.duv_r = take(tr ? (size_t)L.R * 2 * c.d_ffn * 2 : 0);
  L.duv_s = take(tr ? rs * 2 * fs * 2 : 0);
  L.dx_r = take(tr ? (size_t)L.R * c.d_model * 2 : 0);
  L.dx_s = take(tr ? rs * c.d_model * 2 : 0);
  L.sel_tok = take(tr ? (size_t)c.T * c.K * 4 : 0);
  L.sel_row_of = take(tr ? (size_t)c.T * c.K * 4 : 0);
  L.sel_off = take(tr ? (size_t)(c.E_r + 1) * 4 : 0);
  L.sel_base = take(tr ? (size_t)L.n_chunks * c.E_r * 4 : 0);
  L.sel_counts = take(tr ? (size_t)c.E_r * 4 : 0);
  L.sel_kept = take(tr ? (size_t)c.E_r * 4 : 0);
  L.total = o;
  return L;
}

moe_status validate(const moe_config* cfg) {
  if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  const moe_config& c = *cfg;
  if (c.T < 1 || c.T > (1 << 24)) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [1, 2^24]", c.T);
  if (c.d_model < 8 || c.d_model % 8) return fail(MOE_ERR_INVALID_ARG, "d_model=%d must be a positive multiple of 8", c.d_model);
  if (c.E_r < 1) return fail(MOE_ERR_INVALID_ARG, "E_r=%d < 1", c.E_r);
  if (c.E_r > 1024) return fail(MOE_ERR_UNSUPPORTED, "E_r=%d > 1024", c.E_r);
  if (c.E_s < 0) return fail(MOE_ERR_INVALID_ARG, "E_s=%d < 0", c.E_s);
  if (c.E_s > 8) return fail(MOE_ERR_UNSUPPORTED, "E_s=%d > 8", c.E_s);
  if (c.K < 1 || c.K > c.E_r) return fail(MOE_ERR_INVALID_ARG, "K=%d outside [1, E_r=%d]", c.K, c.E_r);
  if (c.K > 32) return fail(MOE_ERR_UNSUPPORTED, "K=%d > 32", c.K);
  if (c.d_ffn < 8 || c.d_ffn % 8) return fail(MOE_ERR_INVALID_ARG, "d_ffn=%d must be a positive multiple of 8", c.d_ffn);
  if (c.E_s > 0 && (c.d_ffn_shared < 8 || c.d_ffn_shared % 8))
    return fail(MOE_ERR_INVALID_ARG, "d_ffn_shared=%d must be a positive multiple of 8", c.d_ffn_shared);
  if (c.score_fn != MOE_SCORE_SIGMOID && c.score_fn != MOE_SCORE_SOFTMAX)
    return fail(MOE_ERR_INVALID_ARG, "score_fn=%d", c.score_fn);
  if (c.dtype != MOE_DTYPE_F32 && c.dtype != MOE_DTYPE_BF16 && c.dtype != MOE_DTYPE_BF16_E4M3)
    return fail(MOE_ERR_INVALID_ARG, "dtype=%d", c.dtype);
  if (c.add_residual != 0 && c.add_residual != 1) return fail(MOE_ERR_INVALID_ARG, "add_residual=%d", c.add_residual);
  if (!std::isfinite(c.capacity_factor)) return fail(MOE_ERR_INVALID_ARG, "capacity_factor is not finite");
  if (c.n_groups < 1) return fail(MOE_ERR_INVALID_ARG, "n_groups=%d < 1", c.n_groups);
  if (c.group_topn < 0) return fail(MOE_ERR_INVALID_ARG, "group_topn=%d < 0", c.group_topn);
  if (c.n_groups > 1 && c.group_topn > 0) {
    if (c.E_r % c.n_groups) return fail(MOE_ERR_INVALID_ARG, "n_groups=%d does not divide E_r=%d", c.n_groups, c.E_r);
    const int gsz = c.E_r / c.n_groups;
    if (c.topk_groups < 1 || c.topk_groups > c.n_groups)
      return fail(MOE_ERR_INVALID_ARG, "topk_groups=%d outside [1, n_groups=%d]", c.topk_groups, c.n_groups);
    if ((int64_t)c.topk_groups * gsz < c.K)
      return fail(MOE_ERR_INVALID_ARG, "topk_groups*(E_r/n_groups)=%d < K=%d", c.topk_groups * gsz, c.K);
    if (c.group_topn > gsz) return fail(MOE_ERR_INVALID_ARG, "group_topn=%d > group size %d", c.group_topn, gsz);
    if (c.n_groups > 32) return fail(MOE_ERR_UNSUPPORTED, "n_groups=%d > 32", c.n_groups);
  }
  if (c.dtype != MOE_DTYPE_F32 && (c.d_model < 64 || c.d_ffn < 64 || (c.E_s > 0 && c.d_ffn_shared < 64)))
    return fail(MOE_ERR_UNSUPPORTED, "bf16 layers need d_model, d_ffn, d_ffn_shared >= 64");
  if (is_q8(c.dtype) && (c.d_model % 16 || c.d_ffn % 16 || (c.E_s > 0 && c.d_ffn_shared % 16)))
    return fail(MOE_ERR_UNSUPPORTED, "e4m3 weights need d_model, d_ffn, d_ffn_shared multiples of 16");
  if (c.train != 0 && c.train != 1) return fail(MOE_ERR_INVALID_ARG, "train=%d", c.train);
  if (c.train && c.dtype != MOE_DTYPE_BF16) return fail(MOE_ERR_UNSUPPORTED, "train needs MOE_DTYPE_BF16");
  if (c.train && (c.d_model % 64 || c.d_ffn % 64 || (c.E_s > 0 && c.d_ffn_shared % 64)))
    return fail(MOE_ERR_UNSUPPORTED, "train needs d_model, d_ffn, d_ffn_shared multiples of 64");
  return MOE_OK;
}

moe_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(MOE_ERR_WORKSPACE, "ws is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return fail(MOE_ERR_WORKSPACE, "ws is not 256-byte aligned");
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "ws_bytes=%zu < required %zu", ws_bytes, need);
  return MOE_OK;
}

moe_status cuda_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(e));
  return MOE_OK;
}

#define MOE_CHECK(x) do { moe_status s_ = (x); if (s_ != MOE_OK) return s_; } while (0)
#define MOE_NONNULL(p) do { if (!(p)) return fail(MOE_ERR_INVALID_ARG, #p " is NULL"); \
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, #p " is not 16-byte aligned"); } while (0)
#define MOE_ALIGNED(p) do { if ((p) && !aligned16(p)) return fail(MOE_ERR_INVALID_ARG, #p " is not 16-byte aligned"); } while (0)
#define MOE_ALIGNED4(p) do { if ((p) && (reinterpret_cast<uintptr_t>(p) & 3u)) return fail(MOE_ERR_INVALID_ARG, #p " is not 4-byte aligned"); } while (0)
#define MOE_NONNULL4(p) do { if (!(p)) return fail(MOE_ERR_INVALID_ARG, #p " is NULL"); MOE_ALIGNED4(p); } while (0)

template <typename T> T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

bool use_tensor_cores(int dtype) { return dtype != MOE_DTYPE_F32; }

// a1-a4: logits (tensor cores for bf16, CUDA cores for fp32) unless scores are
// fed, then activation, selection, gates and the per-chunk histogram.
moe_status run_route(const moe_config& c, const Layout& L, void* ws, const void* h, const float* e,
                     const float* b, const float* s_in, float* s_out, float* z_out, int32_t* idx,
                     float* gates, cudaStream_t st) {
  int* hist = at<int>(ws, L.hist);
  float* scores = at<float>(ws, L.scores);
  cudaMemsetAsync(hist, 0, (size_t)L.n_chunks * c.E_r * 4, st);
  int n_parts = 1;
  if (!s_in) {
    if (use_tensor_cores(c.dtype)) {
      cudaError_t er = moe::launch_router_tc(h, e, at<void>(ws, L.e3), scores, c.T, c.d_model, c.E_r,
                                             at<int>(ws, L.err), &n_parts, st);
      if (er != cudaSuccess) return fail(MOE_ERR_CUDA, "tensor-core router launch: %s", cudaGetErrorString(er));
    } else {
      moe::launch_router_logits(h, c.dtype, e, scores, c.T, c.d_model, c.E_r, st);
    }
  }
  moe::launch_select(s_in ? s_in : scores, n_parts, s_in != nullptr,
                     c.score_fn == MOE_SCORE_SIGMOID ? b : nullptr, c.score_fn, s_out,
                     s_in ? nullptr : z_out, idx, gates, hist, kChunkShift, c.T, c.E_r, c.K,
                     c.n_groups, c.topk_groups, c.group_topn, st);
  return cuda_status();
}

// Caller-provided CUDA events recorded at the phase boundaries of
// moe_layer_forward (profiling support; see moe_set_phase_events).
thread_local cudaEvent_t g_phase_events[8] = {};
thread_local int g_n_phase_events = 0;

void mark_phase(int i, cudaStream_t st) {
  if (i < g_n_phase_events && g_phase_events[i]) cudaEventRecord(g_phase_events[i], st);
}

// bf16 grouped FFNs whose experts average many rows (the rows the caller
// provisions per routed expert: T*K/E_r in a dropless layer) run their GEMMs
// on CTA pairs (256-row tiles), unless they keep U | V for a backward.
static bool ffn_on_pairs(const moe_config& c, bool keeps_uv, int n_experts, int64_t max_rows) {
  return use_tensor_cores(c.dtype) && !is_q8(c.dtype) && !keeps_uv && n_experts > 0 &&
         max_rows >= (int64_t)moe::tc_pair_min_rows() * n_experts && moe::tc_pair_available();
}

// Group tables + both GEMMs of the grouped FFN (phase marks 3 and 4 after the
// group tables and the gate/up GEMM when phase_base >= 0).
moe_status run_ffn(const moe_config& c, moe::FfnArgs& a, const int* offsets, int max_rows,
                   cudaStream_t st, int phase_base = -1) {
  const bool tc = use_tensor_cores(c.dtype);
  // the group tables follow the tile height of the GEMMs that will run
  a.pair = ffn_on_pairs(c, a.uv_r != nullptr, a.E_r, max_rows);
  const int bm = a.pair ? moe::tc_pair_rows() : tc ? moe::tc_bm() : moe::simt_bm();
  const int bn_gu = tc ? moe::tc_cols_gateup() : moe::simt_bn();
  const int bn_dn = tc ? moe::tc_cols_down() : moe::simt_bn();
  moe::launch_groups(offsets, a.E_r, a.E_s, a.T, bm, a.pair ? moe::tc_pair_merge_rows() : tc ? moe::tc_merge_rows() : 0, (a.f_r + bn_gu - 1) / bn_gu,
                     a.E_s ? (a.f_s + bn_gu - 1) / bn_gu : 0, (a.d + bn_dn - 1) / bn_dn,
                     (a.d + bn_dn - 1) / bn_dn, const_cast<int*>(a.grp_rows),
                     const_cast<int*>(a.grp_row0), const_cast<int*>(a.pre_gu),
                     const_cast<int*>(a.pre_dn), max_rows, a.err, a.tile_counters, st);
  if (phase_base >= 0) mark_phase(phase_base, st);
  for (int which = 0; which < 2; ++which) {
    if (tc) {
      cudaError_t e = moe::launch_ffn_tc(a, which, st);
      if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "tensor-core FFN launch: %s", cudaGetErrorString(e));
    } else {
      moe::launch_ffn_simt(a, which, st);
    }
    if (which == 0 && a.q8) {
      // the down GEMM multiplies e4m3 by e4m3: quantize the SwiGLU output rows
      moe::launch_quantize_rows(a.act_r, MOE_DTYPE_BF16, nullptr, 0, offsets + a.E_r, max_rows, a.f_r,
                                static_cast<uint8_t*>(a.actq_r), a.as_r, a.err, st);
      if (a.E_s)
        moe::launch_quantize_rows(a.act_s, MOE_DTYPE_BF16, nullptr, 0, nullptr, (int64_t)a.E_s * a.T, a.f_s,
                                  static_cast<uint8_t*>(a.actq_s), a.as_s, a.err, st);
    }
    if (phase_base >= 0 && which == 0) mark_phase(phase_base + 1, st);
  }
  return cuda_status();
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status moe_expert_ffn_tile_rows(const moe_config* cfg, int32_t n_experts, int32_t max_rows, int32_t* rows) {
  MOE_CHECK(validate(cfg));
  if (!rows) return fail(MOE_ERR_INVALID_ARG, "rows is NULL");
  if (n_experts < 1 || max_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_experts=%d max_rows=%d", n_experts, max_rows);
  const moe_config& c = *cfg;
  if (!use_tensor_cores(c.dtype)) {
    *rows = moe::simt_bm();
    return MOE_OK;
  }
  *rows = ffn_on_pairs(c, false, n_experts, max_rows) ? moe::tc_pair_rows() : moe::tc_bm();
  return MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_last_error_detail(void) { return g_detail; }

moe_status moe_workspace_size(const moe_config* cfg, size_t* bytes) {
  MOE_CHECK(validate(cfg));
  if (!bytes) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = make_layout(*cfg).total;
  return MOE_OK;
}

moe_status moe_expert_ffn_workspace_size(const moe_config* cfg, int32_t n_experts, int32_t d_ffn,
                                         int32_t max_rows, size_t* bytes) {
  MOE_CHECK(validate(cfg));
  if (!bytes) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  if (n_experts < 1 || n_experts > 1024) return fail(MOE_ERR_INVALID_ARG, "n_experts=%d outside [1, 1024]", n_experts);
  if (d_ffn < 8 || d_ffn % 8) return fail(MOE_ERR_INVALID_ARG, "d_ffn=%d must be a positive multiple of 8", d_ffn);
  if (max_rows < 0) return fail(MOE_ERR_INVALID_ARG, "max_rows=%d < 0", max_rows);
  if (is_q8(cfg->dtype) && d_ffn % 16) return fail(MOE_ERR_UNSUPPORTED, "e4m3 weights need d_ffn % 16 == 0");
  const size_t mr = (size_t)(max_rows < 1 ? 1 : max_rows);
  size_t o = 0;
  o = align_up(o + kAlign);                                  // error word
  o = align_up(o + (size_t)n_experts * 8);                    // grp_rows, grp_row0
  o = align_up(o + (size_t)(n_experts + 1) * 8);              // pre_gu, pre_dn
  o = align_up(o + mr * d_ffn * elem_bytes(cfg->dtype));     // A
  if (is_q8(cfg->dtype)) {
    o = align_up(o + mr * cfg->d_model);                      // e4m3 x
    o = align_up(o + mr * 4);                                 // its row scales
    o = align_up(o + mr * d_ffn);                             // e4m3 A
    o = align_up(o + mr * 4);                                 // its row scales
  }
  *bytes = o;
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const void* h, const float* e, const float* b,
                     const float* s_in, float* s_out, float* z_out, int32_t* idx, float* gates,
                     int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  MOE_CHECK(validate(cfg));
  const moe_config& c = *cfg;
  if (!s_in) { MOE_NONNULL(h); MOE_NONNULL4(e); }
  MOE_ALIGNED4(s_in); MOE_ALIGNED4(s_out); MOE_ALIGNED4(z_out); MOE_ALIGNED4(b); MOE_ALIGNED4(counts);
  MOE_NONNULL4(idx); MOE_NONNULL4(gates);
  const Layout L = make_layout(c);
  MOE_CHECK(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_CHECK(run_route(c, L, ws, h, e, b, s_in, s_out, z_out, idx, gates, st));
  if (counts) moe::launch_counts(at<int>(ws, L.hist), L.n_chunks, c.E_r, counts, st);
  return cuda_status();
}

moe_status moe_permute(const moe_config* cfg, const int32_t* idx, const float* gates,
                       const void* h, int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                       int32_t* kept, float* row_gate, void* x_perm, void* ws, size_t ws_bytes,
                       void* stream) {
  MOE_CHECK(validate(cfg));
  const moe_config& c = *cfg;
  MOE_NONNULL4(idx); MOE_NONNULL4(offsets); MOE_NONNULL4(perm_tok); MOE_NONNULL4(row_of); MOE_NONNULL4(kept);
  MOE_ALIGNED4(gates); MOE_ALIGNED(h); MOE_ALIGNED4(row_gate); MOE_ALIGNED(x_perm);
  if (row_gate && !gates) return fail(MOE_ERR_INVALID_ARG, "row_gate needs gates");
  if (x_perm && !h) return fail(MOE_ERR_INVALID_ARG, "x_perm needs h");
  const Layout L = make_layout(c);
  MOE_CHECK(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err = at<int>(ws, L.err);
  int* hist = at<int>(ws, L.hist);
  cudaMemsetAsync(hist, 0, (size_t)L.n_chunks * c.E_r * 4, st);
  moe::launch_hist(idx, hist, kChunkShift, c.T, c.K, c.E_r, err, st);
  moe::launch_scan(hist, L.n_chunks, c.E_r, (int)L.cap, at<int>(ws, L.counts), kept, offsets,
                   at<int>(ws, L.chunk_base), st);
  moe::launch_scatter(idx, gates, offsets, at<int>(ws, L.chunk_base), (int)L.cap, c.T, c.K, c.E_r,
                      perm_tok, row_of, row_gate, err, st);
  if (x_perm)
    moe::launch_gather(h, perm_tok, offsets + c.E_r, x_perm, c.d_model, (int)elem_bytes(c.dtype),
                       c.T * c.K, c.T, err, st);
  return cuda_status();
}

moe_status moe_expert_ffn(const moe_config* cfg, int32_t n_experts, int32_t d_ffn,
                          int32_t max_rows, const int32_t* offsets, const void* x,
                          const void* w_gate, const void* w_up, const void* w_down,
                          const float* row_scale, void* out, void* ws, size_t ws_bytes,
                          void* stream) {
  size_t need = 0;
  MOE_CHECK(moe_expert_ffn_workspace_size(cfg, n_experts, d_ffn, max_rows, &need));
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DTYPE_F32 && d_ffn < 64) return fail(MOE_ERR_UNSUPPORTED, "bf16 needs d_ffn >= 64");
  MOE_NONNULL4(offsets); MOE_NONNULL(x); MOE_NONNULL(w_gate); MOE_NONNULL(w_up); MOE_NONNULL(w_down);
  MOE_NONNULL(out); MOE_ALIGNED4(row_scale);
  MOE_CHECK(check_ws(ws, ws_bytes, need));
  if (max_rows == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  size_t o = kAlign;
  int* grp_rows = at<int>(ws, o);
  int* grp_row0 = grp_rows + n_experts;
  o = align_up(o + (size_t)n_experts * 8);
  int* pre_gu = at<int>(ws, o);
  int* pre_dn = pre_gu + n_experts + 1;
  o = align_up(o + (size_t)(n_experts + 1) * 8);
  moe::FfnArgs a{};
  a.dtype = c.dtype; a.T = c.T; a.d = c.d_model; a.f_r = d_ffn; a.f_s = d_ffn;
  a.E_r = n_experts; a.E_s = 0; a.max_rows_r = max_rows;
  a.x_r = x; a.x_s = x;
  a.wg_r = w_gate; a.wu_r = w_up; a.wd_r = w_down;
  a.wg_s = w_gate; a.wu_s = w_up; a.wd_s = w_down;
  a.grp_rows = grp_rows; a.grp_row0 = grp_row0; a.pre_gu = pre_gu; a.pre_dn = pre_dn;
  a.row_scale = row_scale;
  a.act_r = at<void>(ws, o); a.act_s = a.act_r;
  a.out_r = out; a.out_s = out;
  a.err = at<int>(ws, 0);
  a.tile_counters = at<int>(ws, 64);   // spare words of the error block
  if (is_q8(c.dtype)) {
    const size_t mr = (size_t)max_rows;
    o = align_up(o + mr * d_ffn * elem_bytes(c.dtype));
    uint8_t* xq = at<uint8_t>(ws, o); o = align_up(o + mr * c.d_model);
    float* xs = at<float>(ws, o);     o = align_up(o + mr * 4);
    a.actq_r = a.actq_s = at<void>(ws, o); o = align_up(o + mr * d_ffn);
    a.as_r = a.as_s = at<float>(ws, o);
    // rows 0 .. offsets[n_experts] of x, quantized for the e4m3 gate/up GEMM
    moe::launch_quantize_rows(x, MOE_DTYPE_BF16, nullptr, 0, offsets + n_experts, max_rows, c.d_model,
                              xq, xs, a.err, st);
    a.q8 = 1;
    a.x_r = a.x_s = xq;
    a.xs_r = a.xs_s = xs;
  }
  return run_ffn(c, a, offsets, max_rows, st);
}

moe_status moe_combine(const moe_config* cfg, const void* h, const void* slot,
                       const void* shared_out, const int32_t* row_of, void* y, void* stream) {
  MOE_CHECK(validate(cfg));
  const moe_config& c = *cfg;
  MOE_NONNULL(h); MOE_NONNULL(slot); MOE_NONNULL4(row_of); MOE_NONNULL(y);
  if (c.E_s > 0) MOE_NONNULL(shared_out);
  moe::launch_combine(h, slot, shared_out, row_of, y, c.T, c.d_model, c.K, c.E_s, c.add_residual,
                      act_dtype(c.dtype), 0x7FFFFFFF, static_cast<cudaStream_t>(stream));
  return cuda_status();
}

moe_status moe_bias_update(const moe_config* cfg, const int32_t* counts, float gamma, float* b,
                           float* max_vio, void* stream) {
  MOE_CHECK(validate(cfg));
  const moe_config& c = *cfg;
  MOE_NONNULL4(counts); MOE_NONNULL4(b); MOE_ALIGNED4(max_vio);
  if (!std::isfinite(gamma)) return fail(MOE_ERR_INVALID_ARG, "gamma is not finite");
  moe::launch_bias_update(counts, b, gamma, max_vio, c.E_r, c.K, c.T, static_cast<cudaStream_t>(stream));
  return cuda_status();
}

moe_status moe_layer_forward(const moe_config* cfg, const void* h, const float* e, float* b,
                             const void* w_gate, const void* w_up, const void* w_down,
                             const void* ws_gate, const void* ws_up, const void* ws_down,
                             const float* s_in, void* y, int32_t* idx_out, float* gates_out,
                             int32_t* counts_out, int32_t* kept_out, float* s_out, float* z_out,
                             int32_t update_bias, float gamma, float* max_vio_out,
                             void* ws, size_t ws_bytes, void* stream) {
  MOE_CHECK(validate(cfg));
  const moe_config& c = *cfg;
  MOE_NONNULL(h); MOE_NONNULL(w_gate); MOE_NONNULL(w_up); MOE_NONNULL(w_down); MOE_NONNULL(y);
  if (!s_in) MOE_NONNULL4(e);
  if (c.E_s > 0) { MOE_NONNULL(ws_gate); MOE_NONNULL(ws_up); MOE_NONNULL(ws_down); }
  if (update_bias) {
    MOE_NONNULL4(b);
    if (!std::isfinite(gamma)) return fail(MOE_ERR_INVALID_ARG, "gamma is not finite");
  }
  MOE_ALIGNED4(b); MOE_ALIGNED4(s_in); MOE_ALIGNED4(idx_out); MOE_ALIGNED4(gates_out);
  MOE_ALIGNED4(counts_out); MOE_ALIGNED4(kept_out); MOE_ALIGNED4(s_out); MOE_ALIGNED4(z_out);
  MOE_ALIGNED4(max_vio_out);
  const Layout L = make_layout(c);
  MOE_CHECK(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  int* err = at<int>(ws, L.err);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
  float* gates = gates_out ? gates_out : at<float>(ws, L.gates);
  int* counts = counts_out ? counts_out : at<int>(ws, L.counts);
  int* kept = kept_out ? kept_out : at<int>(ws, L.kept);
  int* offsets = at<int>(ws, L.offsets);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  int32_t* perm_tok = at<int32_t>(ws, L.perm_tok);
  float* row_gate = at<float>(ws, L.row_gate);
  const size_t es = elem_bytes(c.dtype);

  // a1-a4: affinity, selection, gates, per-chunk histogram
  mark_phase(0, st);
  MOE_CHECK(run_route(c, L, ws, h, e, b, s_in, s_out, z_out, idx, gates, st));
  // a5: counts, capacity, offsets, stable scatter, row gather
  mark_phase(1, st);
  moe::launch_scan(at<int>(ws, L.hist), L.n_chunks, c.E_r, (int)L.cap, counts, kept, offsets,
                   at<int>(ws, L.chunk_base), st);
  moe::launch_scatter(idx, gates, offsets, at<int>(ws, L.chunk_base), (int)L.cap, c.T, c.K, c.E_r,
                      perm_tok, row_of, row_gate, err, st);
  void* x_perm = at<void>(ws, L.x_perm);
  const bool q8 = is_q8(c.dtype);
  if (q8) {
    // quantize each token's row of h once (the shared experts' input), then
    // gather the e4m3 rows and their scales into expert order
    moe::launch_quantize_rows(h, MOE_DTYPE_BF16, nullptr, 0, nullptr, c.T, c.d_model,
                              at<uint8_t>(ws, L.hq), at<float>(ws, L.hs), err, st);
    moe::launch_gather(at<uint8_t>(ws, L.hq), perm_tok, offsets + c.E_r, x_perm, c.d_model, 1, (int)L.R,
                       c.T, err, st, at<float>(ws, L.hs), at<float>(ws, L.xs));
  } else {
    moe::launch_gather(h, perm_tok, offsets + c.E_r, x_perm, c.d_model, (int)es, (int)L.R, c.T, err, st);
  }
  mark_phase(2, st);
  // a6-a7: grouped SwiGLU experts (routed + shared) with gate-scaled outputs
  moe::FfnArgs a{};
  a.dtype = c.dtype; a.T = c.T; a.d = c.d_model; a.f_r = c.d_ffn;
  a.f_s = c.E_s ? c.d_ffn_shared : c.d_ffn;
  a.E_r = c.E_r; a.E_s = c.E_s; a.max_rows_r = (int)L.R;
  a.x_r = x_perm; a.x_s = h;
  a.wg_r = w_gate; a.wu_r = w_up; a.wd_r = w_down;
  a.wg_s = c.E_s ? ws_gate : w_gate; a.wu_s = c.E_s ? ws_up : w_up; a.wd_s = c.E_s ? ws_down : w_down;
  a.grp_rows = at<int>(ws, L.grp_rows); a.grp_row0 = at<int>(ws, L.grp_row0);
  a.pre_gu = at<int>(ws, L.pre_gu); a.pre_dn = at<int>(ws, L.pre_dn);
  a.row_scale = row_gate;
  a.act_r = at<void>(ws, L.act_r); a.act_s = c.E_s ? at<void>(ws, L.act_s) : a.act_r;
  a.out_r = at<void>(ws, L.slot_r); a.out_s = c.E_s ? at<void>(ws, L.slot_s) : a.out_r;
  a.err = err;
  a.tile_counters = err + 16;          // spare words of the error block
  if (c.train) { a.uv_r = at<void>(ws, L.uv_r); a.uv_s = c.E_s ? at<void>(ws, L.uv_s) : a.uv_r; }
  if (q8) {
    a.q8 = 1;
    a.x_s = at<void>(ws, L.hq);
    a.xs_r = at<float>(ws, L.xs);
    a.xs_s = at<float>(ws, L.hs);
    a.actq_r = at<void>(ws, L.actq_r); a.actq_s = c.E_s ? at<void>(ws, L.actq_s) : a.actq_r;
    a.as_r = at<float>(ws, L.as_r); a.as_s = c.E_s ? at<float>(ws, L.as_s) : a.as_r;
  }
  // the slot and shared rows stay inside the workspace: fp16 for a bf16
  // layer (three more significant bits than bf16 in the same bytes)
  a.out_f16 = use_tensor_cores(c.dtype) ? 1 : 0;
  MOE_CHECK(run_ffn(c, a, offsets, (int)L.R, st, 3));
  mark_phase(5, st);
  // a8: fixed-order combine with the residual
  moe::launch_combine(h, a.out_r, c.E_s ? a.out_s : nullptr, row_of, y, c.T, c.d_model, c.K, c.E_s,
                      c.add_residual, act_dtype(c.dtype), (int)L.R, st, a.out_f16);
  mark_phase(6, st);
  // a9: the bias step, after this batch's loads are counted
  if (update_bias || max_vio_out)
    moe::launch_bias_update(counts, update_bias ? b : nullptr, gamma, max_vio_out, c.E_r, c.K, c.T, st);
  mark_phase(7, st);
  return cuda_status();
}

moe_status moe_layer_backward(const moe_config* cfg, const void* h, const float* e, const float* s,
                              const int32_t* idx, const void* w_gate, const void* w_up,
                              const void* w_down, const void* ws_gate, const void* ws_up,
                              const void* ws_down, const void* dy, void* dh, float* de,
                              void* dw_gate, void* dw_up, void* dw_down, void* dws_gate,
                              void* dws_up, void* dws_down, void* ws, size_t ws_bytes, void* stream) {
  MOE_CHECK(validate(cfg));
  const moe_config& c = *cfg;
  if (!c.train) return fail(MOE_ERR_INVALID_ARG, "cfg->train must be 1 (forward and backward)");
  MOE_NONNULL(h); MOE_NONNULL4(e); MOE_NONNULL4(s); MOE_NONNULL4(idx);
  MOE_NONNULL(w_gate); MOE_NONNULL(w_up); MOE_NONNULL(w_down);
  MOE_NONNULL(dy); MOE_NONNULL(dh); MOE_NONNULL(de);
  MOE_NONNULL(dw_gate); MOE_NONNULL(dw_up); MOE_NONNULL(dw_down);
  if (c.E_s > 0) {
    MOE_NONNULL(ws_gate); MOE_NONNULL(ws_up); MOE_NONNULL(ws_down);
    MOE_NONNULL(dws_gate); MOE_NONNULL(dws_up); MOE_NONNULL(dws_down);
  }
  const Layout L = make_layout(c);
  MOE_CHECK(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err = at<int>(ws, L.err);
  const int* offsets = at<int>(ws, L.offsets);
  const int fs = c.E_s ? c.d_ffn_shared : c.d_ffn;
  const int R = (int)L.R;
  // group tables of the backward GEMMs: 128-row tiles (a last tile of <= 64 rows merged into the
  // one before), 256-column tiles of f (dA) and d (dX)
  moe::launch_groups(offsets, c.E_r, c.E_s, c.T, 128, moe::bwd_merge_rows(), (c.d_ffn + 255) / 256, (fs + 255) / 256,
                     (c.d_model + 255) / 256, (c.d_model + 255) / 256, at<int>(ws, L.grp_rows),
                     at<int>(ws, L.grp_row0), at<int>(ws, L.pre_gu), at<int>(ws, L.pre_dn), R, err, err + 16, st);
  moe::BwdRouteArgs ra{};
  ra.T = c.T; ra.d = c.d_model; ra.E = c.E_r; ra.K = c.K; ra.E_s = c.E_s; ra.score_fn = c.score_fn;
  ra.add_residual = c.add_residual; ra.max_rows = R;
  ra.dy = static_cast<const uint16_t*>(dy); ra.slot = at<uint16_t>(ws, L.slot_r);
  ra.dx_r = at<uint16_t>(ws, L.dx_r); ra.dx_s = at<uint16_t>(ws, L.dx_s);
  ra.h = static_cast<const uint16_t*>(h);
  ra.perm_tok = at<int32_t>(ws, L.perm_tok); ra.row_of = at<int32_t>(ws, L.row_of); ra.idx = idx;
  ra.n_rows_ptr = offsets + c.E_r;
  ra.row_gate = at<float>(ws, L.row_gate); ra.s = s; ra.e = e;
  ra.dO = at<uint16_t>(ws, L.dO); ra.dh = static_cast<uint16_t*>(dh);
  ra.dg_row = at<float>(ws, L.dg_row); ra.dz = at<float>(ws, L.dz); ra.de = de;
  ra.err = err;
  ra.slot_f16 = 1;                     // the forward (train = 1, bf16) wrote fp16 slot rows
  if (c.score_fn == MOE_SCORE_SIGMOID) {
    // the forward's per-chunk histogram, scanned without a capacity and
    // scattered stably: every selected pair by expert, tokens ascending
    const int all = c.T * c.K;
    moe::launch_scan(at<int>(ws, L.hist), L.n_chunks, c.E_r, all, at<int>(ws, L.sel_counts),
                     at<int>(ws, L.sel_kept), at<int>(ws, L.sel_off), at<int>(ws, L.sel_base), st);
    moe::launch_scatter(idx, nullptr, at<int>(ws, L.sel_off), at<int>(ws, L.sel_base), all, c.T, c.K, c.E_r,
                        at<int32_t>(ws, L.sel_tok), at<int32_t>(ws, L.sel_row_of), nullptr, err, st);
    ra.sel_tok = at<int32_t>(ws, L.sel_tok);
    ra.sel_off = at<int>(ws, L.sel_off);
  }
  moe::launch_bwd_route(ra, st);                      // dO = g dy, dL/dg per kept row
  moe::BwdArgs ba{};
  ba.T = c.T; ba.d = c.d_model; ba.f_r = c.d_ffn; ba.f_s = fs; ba.E_r = c.E_r; ba.E_s = c.E_s;
  ba.max_rows_r = R;
  ba.dO_r = ra.dO; ba.dy = dy;
  ba.wg_r = w_gate; ba.wu_r = w_up; ba.wd_r = w_down;
  ba.wg_s = c.E_s ? ws_gate : w_gate; ba.wu_s = c.E_s ? ws_up : w_up; ba.wd_s = c.E_s ? ws_down : w_down;
  ba.uv_r = at<void>(ws, L.uv_r); ba.uv_s = c.E_s ? at<void>(ws, L.uv_s) : ba.uv_r;
  ba.duv_r = at<void>(ws, L.duv_r); ba.duv_s = c.E_s ? at<void>(ws, L.duv_s) : ba.duv_r;
  ba.dx_r = at<void>(ws, L.dx_r); ba.dx_s = c.E_s ? at<void>(ws, L.dx_s) : ba.dx_r;
  ba.x_r = at<void>(ws, L.x_perm); ba.h = h;
  ba.act_r = at<void>(ws, L.act_r); ba.act_s = c.E_s ? at<void>(ws, L.act_s) : ba.act_r;
  ba.dwg_r = dw_gate; ba.dwu_r = dw_up; ba.dwd_r = dw_down;
  ba.dwg_s = dws_gate; ba.dwu_s = dws_up; ba.dwd_s = dws_down;
  ba.grp_rows = at<int>(ws, L.grp_rows); ba.grp_row0 = at<int>(ws, L.grp_row0);
  ba.pre_da = at<int>(ws, L.pre_gu); ba.pre_dx = at<int>(ws, L.pre_dn);
  ba.err = err;
  // operand B of the weight gradients (x, A) is read up to 63 rows past the
  // last routed row: keep those rows finite (zero)
  moe::launch_zero_tail_rows(at<void>(ws, L.x_perm), offsets + c.E_r, R, c.d_model, st);
  moe::launch_zero_tail_rows(at<void>(ws, L.act_r), offsets + c.E_r, R, c.d_ffn, st);
  for (int which = 0; which < 5; ++which) {
    cudaError_t er = moe::launch_bwd_tc(ba, which, st);
    if (er != cudaSuccess) return fail(MOE_ERR_CUDA, "backward GEMM %d: %s", which, cudaGetErrorString(er));
  }
  moe::launch_bwd_gate_dh_de(ra, st);                 // dz, dh, de
  return cuda_status();
}

moe_status moe_set_phase_events(void* const* events, int32_t n_events) {
  if (n_events < 0 || n_events > 8) return fail(MOE_ERR_INVALID_ARG, "n_events=%d outside [0, 8]", n_events);
  if (n_events > 0 && !events) return fail(MOE_ERR_INVALID_ARG, "events is NULL");
  for (int i = 0; i < 8; ++i) g_phase_events[i] = i < n_events ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  g_n_phase_events = n_events;
  return MOE_OK;
}

moe_status moe_get_device_error(const void* ws, int32_t* code) {
  if (!ws || !code) return fail(MOE_ERR_INVALID_ARG, "ws or code is NULL");
  int32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_status();
  *code = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

static size_t router_stats_bytes(const moe_config& c, int32_t seq_len) {
  const int S = seq_len > 0 ? seq_len : c.T;
  const size_t n_seq = (size_t)c.T / S;
  const size_t n_ch = ((size_t)S + moe::kStatsChunk - 1) / moe::kStatsChunk;
  return align_up(kAlign + align_up((size_t)c.T * 4) * 2 + align_up(n_seq * c.E_r * 4) +
                  align_up(n_seq * n_ch * c.E_r * 4));
}

moe_status moe_router_stats_workspace_size(const moe_config* cfg, int32_t seq_len, size_t* bytes) {
  MOE_CHECK(validate(cfg));
  if (!bytes) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  if (seq_len < 0 || (seq_len > 0 && cfg->T % seq_len))
    return fail(MOE_ERR_INVALID_ARG, "seq_len=%d must be 0 or divide T=%d", seq_len, cfg->T);
  *bytes = router_stats_bytes(*cfg, seq_len);
  return MOE_OK;
}

moe_status moe_router_stats(const moe_config* cfg, const float* s, const float* z, const int32_t* idx,
                            const int32_t* kept, int32_t seq_len, float alpha_aux, float c_z,
                            float alpha_seq, float* stats, void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  MOE_CHECK(moe_router_stats_workspace_size(cfg, seq_len, &need));
  const moe_config& c = *cfg;
  MOE_NONNULL4(s); MOE_NONNULL4(idx); MOE_NONNULL4(stats); MOE_ALIGNED4(z); MOE_ALIGNED4(kept);
  if (!std::isfinite(alpha_aux) || !std::isfinite(c_z) || !std::isfinite(alpha_seq))
    return fail(MOE_ERR_INVALID_ARG, "non-finite loss coefficient");
  MOE_CHECK(check_ws(ws, ws_bytes, need));
  const int S = seq_len > 0 ? seq_len : c.T;
  const size_t n_seq = (size_t)c.T / S;
  size_t o = kAlign;
  float* rowsum = at<float>(ws, o); o += align_up((size_t)c.T * 4);
  float* lse2 = at<float>(ws, o); o += align_up((size_t)c.T * 4);
  int* seq_counts = at<int>(ws, o); o += align_up(n_seq * c.E_r * 4);
  float* pchunk = at<float>(ws, o);
  moe::launch_router_stats(s, z, idx, kept, c.T, c.E_r, c.K, S, seq_len > 0, alpha_aux, c_z,
                           alpha_seq, rowsum, lse2, seq_counts, pchunk, stats,
                           static_cast<cudaStream_t>(stream));
  return cuda_status();
}

moe_status moe_gather_rows(const void* src, int64_t n_src, int32_t row_bytes, const int32_t* map,
                           int64_t n_rows, void* dst, void* stream) {
  if (n_rows < 0 || n_src < 0) return fail(MOE_ERR_INVALID_ARG, "negative row count");
  if (row_bytes < 4 || row_bytes % 4) return fail(MOE_ERR_INVALID_ARG, "row_bytes=%d must be a positive multiple of 4", row_bytes);
  if (n_rows == 0) return MOE_OK;
  MOE_NONNULL4(map);
  if (row_bytes % 16 == 0) { MOE_NONNULL(dst); MOE_ALIGNED(src); } else { MOE_NONNULL4(dst); MOE_ALIGNED4(src); }
  if (!src && n_src > 0) return fail(MOE_ERR_INVALID_ARG, "src is NULL");
  moe::launch_gather_map(src, map, n_rows, n_src, row_bytes, dst, nullptr, static_cast<cudaStream_t>(stream));
  return cuda_status();
}

moe_status moe_quantized_bytes(int64_t n_rows, int32_t cols, size_t* bytes) {
  if (!bytes) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  if (n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_rows=%lld < 0", (long long)n_rows);
  if (cols < 16 || cols % 16) return fail(MOE_ERR_INVALID_ARG, "cols=%d must be a positive multiple of 16", cols);
  *bytes = (size_t)n_rows * cols + (size_t)n_rows * 4;
  return MOE_OK;
}

moe_status moe_quantize_rows(const void* src, int32_t src_dtype, int64_t n_rows, int32_t cols, void* dst,
                             void* stream) {
  size_t unused = 0;
  MOE_CHECK(moe_quantized_bytes(n_rows, cols, &unused));
  if (src_dtype != MOE_DTYPE_F32 && src_dtype != MOE_DTYPE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "src_dtype=%d", src_dtype);
  MOE_NONNULL(src); MOE_NONNULL(dst);
  if (n_rows == 0) return MOE_OK;
  uint8_t* codes = static_cast<uint8_t*>(dst);
  moe::launch_quantize_rows(src, src_dtype, nullptr, 0, nullptr, n_rows, cols, codes,
                            reinterpret_cast<float*>(codes + (size_t)n_rows * cols), nullptr,
                            static_cast<cudaStream_t>(stream));
  return cuda_status();
}

moe_status moe_selftest_bounded_wait(void* ws, int64_t limit_ns, void* stream) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "ws is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return fail(MOE_ERR_WORKSPACE, "ws is not 256-byte aligned");
  if (limit_ns < 1000000 || limit_ns > 2000000000) return fail(MOE_ERR_INVALID_ARG, "limit_ns outside [1 ms, 2 s]");
  moe::launch_bounded_wait_selftest((uint64_t)limit_ns, at<int>(ws, 0), static_cast<cudaStream_t>(stream));
  return cuda_status();
}

moe_status moe_clear_device_error(void* ws, void* stream) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "ws is NULL");
  cudaMemsetAsync(ws, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream));
  return cuda_status();
}

}  // extern "C"
