// Routing, dispatch, combine and bias-step kernels of the MoE layer forward.
//
// Sources (web pages):
//  "Sparse Mixture-of-Experts (MoE): Routing Math, Load Balancing & Expert
//   Parallelism": section 0 layer equation (combine), section 2 equation
//   (I_t = TopK(s + b), g = s / sum s, c_i, c_bar, b += gamma sign(c_bar - c_i)),
//   section 3 capacity bound, section 4 MaxVio.
//  "Load Balancing -- DeepSeek-V3": How it works (g', g); Official code
//   (bias added before the grouped top-k).
//  "Mixture of Experts: Routing and Load Balancing": section 5 (capacity admits
//   tokens in the order they appear).
//  "GPUs, memory and failures": the bias card (update once per step).
#include <algorithm>
#include <cfloat>
#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// a1 (CUDA cores): z[t, i] = sum_k h[t, k] e[i, k] in fp32.
// Tile 64 tokens x 64 experts x 32 k, 256 threads, 4 x 4 outputs per thread.
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(256)
router_logits_simt_kernel(const TIn* __restrict__ h, const float* __restrict__ e,
                          float* __restrict__ z, int T, int d, int E) {
  constexpr int BT = 64, BE = 64, BK = 32;
  __shared__ float hs[BK][BT + 4];
  __shared__ float es[BK][BE + 4];
  const int t0 = blockIdx.x * BT, e0 = blockIdx.y * BE;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += BK) {
    for (int i = tid; i < BT * BK; i += 256) {
      int r = i / BK, c = i % BK;
      int t = t0 + r, k = k0 + c;
      hs[c][r] = (t < T && k < d) ? to_f32(h[(size_t)t * d + k]) : 0.f;
      int ex = e0 + r;
      es[c][r] = (ex < E && k < d) ? e[(size_t)ex * d + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < BK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = hs[k][ty * 4 + i]; b[i] = es[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int ex = e0 + tx * 4 + j;
      if (ex < E) z[(size_t)t * E + ex] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// a1-a4: scores, (group-limited) top-K, gates and the per-chunk histogram.
// One warp per token; lane l holds experts l, l+32, ... (KPL per lane).
// ---------------------------------------------------------------------------

// (key, index) order of the selection: larger key first, ties -> lower index.
__device__ __forceinline__ bool beats(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

__device__ __forceinline__ void warp_best(float& k, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float ok = __shfl_xor_sync(kFull, k, off);
    int oi = __shfl_xor_sync(kFull, i, off);
    if (beats(ok, oi, k, i)) { k = ok; i = oi; }
  }
}

template <int KPL>
__global__ void __launch_bounds__(256)
select_kernel(const float* __restrict__ in, int n_parts, int in_is_scores, const float* __restrict__ bias,
              int score_fn, float* __restrict__ s_out, float* __restrict__ z_out, int32_t* __restrict__ idx,
              float* __restrict__ gates, int* __restrict__ hist, int chunk_shift, int T, int E,
              int K, int n_groups, int topk_groups, int group_topn) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int t = blockIdx.x * (blockDim.x / kWarp) + warp;
  if (t >= T) return;
  const float* row = in + (size_t)t * E;

  float s[KPL], key[KPL];
  // logits from split-K partial sums, added in split order (deterministic):
  // each round loads PC partials of all KPL experts of this lane at once
  // (KPL * PC = 64 loads in flight), so a token with many partials -- small
  // batches are split finest -- waits for n_parts / PC load latencies, not
  // for KPL * n_parts / PC of them
  constexpr int PC = 64 / KPL > 0 ? 64 / KPL : 1;
#pragma unroll
  for (int j = 0; j < KPL; ++j) s[j] = 0.f;
  for (int q0 = 0; q0 < n_parts; q0 += PC) {
    float part[KPL][PC];
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int ex = j * kWarp + lane;
#pragma unroll
      for (int q = 0; q < PC; ++q)
        part[j][q] = (q0 + q < n_parts && ex < E) ? row[(size_t)(q0 + q) * T * E + ex] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
#pragma unroll
      for (int q = 0; q < PC; ++q)
        if (q0 + q < n_parts) s[j] = (q0 + q == 0) ? part[j][q] : __fadd_rn(s[j], part[j][q]);
    }
  }
#pragma unroll
  for (int j = 0; j < KPL; ++j)
    if (j * kWarp + lane >= E) s[j] = 0.f;
  if (!in_is_scores) {
    if (z_out) {
#pragma unroll
      for (int j = 0; j < KPL; ++j)
        if (j * kWarp + lane < E) z_out[(size_t)t * E + j * kWarp + lane] = s[j];
    }
    if (score_fn == MOE_SCORE_SIGMOID) {
#pragma unroll
      for (int j = 0; j < KPL; ++j) s[j] = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-s[j])));
    } else {
      float m = -FLT_MAX;
#pragma unroll
      for (int j = 0; j < KPL; ++j)
        if (j * kWarp + lane < E) m = fmaxf(m, s[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < KPL; ++j) {
        s[j] = (j * kWarp + lane < E) ? expf(s[j] - m) : 0.f;
        sum = __fadd_rn(sum, s[j]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(kFull, sum, off));
#pragma unroll
      for (int j = 0; j < KPL; ++j) s[j] = __fdiv_rn(s[j], sum);
    }
  }
  if (s_out) {
#pragma unroll
    for (int j = 0; j < KPL; ++j)
      if (j * kWarp + lane < E) s_out[(size_t)t * E + j * kWarp + lane] = s[j];
  }
  // selection key: s + b as one fp32 add (the bias only picks)
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    int ex = j * kWarp + lane;
    key[j] = ex < E ? __fadd_rn(s[j], bias ? bias[ex] : 0.0f) : -INFINITY;
  }

  // group limit: keep the topk_groups groups with the largest sum of their
  // group_topn largest keys (added in descending order); others ineligible
  uint32_t eligible = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j)
    if (j * kWarp + lane < E) eligible |= 1u << j;
  if (n_groups > 1 && group_topn > 0) {
    const int gsz = E / n_groups;
    int grp[KPL];                                  // group of each held expert
#pragma unroll
    for (int j = 0; j < KPL; ++j) grp[j] = (j * kWarp + lane) / gsz;
    float G[32];
    for (int g = 0; g < n_groups; ++g) {
      float acc;
      if (group_topn == 2) {
        // the two largest keys of the group by one pairwise warp reduction
        // (their sum does not depend on how ties among them are ordered)
        float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
        for (int j = 0; j < KPL; ++j) {
          if (j * kWarp + lane < E && grp[j] == g) {
            const float v = key[j];
            if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float o1 = __shfl_xor_sync(kFull, m1, off), o2 = __shfl_xor_sync(kFull, m2, off);
          const float hi = fmaxf(m1, o1), lo = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
          m1 = hi; m2 = lo;
        }
        acc = __fadd_rn(m1, m2);
      } else {
        // general case: the group_topn largest keys in descending order
        uint32_t used = 0;
        acc = 0.f;
        for (int r = 0; r < group_topn; ++r) {
          float bk = -INFINITY;
          int bi = 0x7FFFFFFF;
#pragma unroll
          for (int j = 0; j < KPL; ++j) {
            int ex = j * kWarp + lane;
            if (ex < E && grp[j] == g && !(used >> j & 1u) && beats(key[j], ex, bk, bi)) {
              bk = key[j];
              bi = ex;
            }
          }
          warp_best(bk, bi);
          if ((bi & (kWarp - 1)) == lane) used |= 1u << (bi / kWarp);
          acc = r == 0 ? bk : __fadd_rn(acc, bk);
        }
      }
      G[g] = acc;
    }
    uint32_t keep = 0;
    for (int r = 0; r < topk_groups; ++r) {
      int bg = -1;
      for (int g = 0; g < n_groups; ++g)
        if (!(keep >> g & 1u) && (bg < 0 || G[g] > G[bg])) bg = g;
      keep |= 1u << bg;
    }
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      if (j * kWarp + lane < E && !(keep >> grp[j] & 1u)) eligible &= ~(1u << j);
    }
  }

  // top-K among the eligible experts
  uint32_t taken = 0;
  for (int r = 0; r < K; ++r) {
    float bk = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      int ex = j * kWarp + lane;
      if ((eligible >> j & 1u) && !(taken >> j & 1u) && beats(key[j], ex, bk, bi)) {
        bk = key[j];
        bi = ex;
      }
    }
    warp_best(bk, bi);
    if ((bi & (kWarp - 1)) == lane) taken |= 1u << (bi / kWarp);
  }

  // gate denominator: sum of the selected s in ascending expert index, fp32
  float S = 0.f;
  bool first = true;
  int pos_of[KPL];
  int pos = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    uint32_t m = __ballot_sync(kFull, taken >> j & 1u);
    pos_of[j] = pos + __popc(m & ((1u << lane) - 1u));
    pos += __popc(m);
    while (m) {
      int l = __ffs(m) - 1;
      float v = __shfl_sync(kFull, s[j], l);
      S = first ? v : __fadd_rn(S, v);
      first = false;
      m &= m - 1;
    }
  }
  const float denom = fmaxf(S, 1e-12f);
  const int chunk = t >> chunk_shift;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    if (taken >> j & 1u) {
      int ex = j * kWarp + lane;
      idx[(size_t)t * K + pos_of[j]] = ex;
      gates[(size_t)t * K + pos_of[j]] = __fdiv_rn(s[j], denom);
      if (hist) atomicAdd(&hist[(size_t)chunk * E + ex], 1);
    }
  }
}

// Histogram of a given idx [T, K] per chunk of tokens (for moe_permute).
__global__ void hist_kernel(const int32_t* __restrict__ idx, int* __restrict__ hist,
                            int chunk_shift, int T, int K, int E, int* err) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * K) return;
  int t = i / K, ex = idx[i];
  if (ex < 0 || ex >= E) { set_device_error(err, MOE_DEVERR_INDEX); return; }
  atomicAdd(&hist[(size_t)(t >> chunk_shift) * E + ex], 1);
}

// counts[e] = sum over chunks of hist[c][e]
__global__ void counts_kernel(const int* __restrict__ hist, int n_chunks, int E, int* counts) {
  int ex = blockIdx.x * blockDim.x + threadIdx.x;
  if (ex >= E) return;
  int run = 0;
  for (int c = 0; c < n_chunks; ++c) run += hist[(size_t)c * E + ex];
  counts[ex] = run;
}

// Exclusive scan of one value per thread over a block of up to 1024 threads.
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
  int x = v;
#pragma unroll
  for (int off = 1; off < kWarp; off <<= 1) {
    int y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  if (lane == kWarp - 1) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int nw = (blockDim.x + kWarp - 1) / kWarp;
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < kWarp; off <<= 1) {
      int y = __shfl_up_sync(kFull, w, off);
      if (lane >= off) w += y;
    }
    warp_sums[lane] = w;    // inclusive
  }
  __syncthreads();
  int base = warp > 0 ? warp_sums[warp - 1] : 0;
  int nw = (blockDim.x + kWarp - 1) / kWarp;
  if (total) *total = warp_sums[nw - 1];
  __syncthreads();
  return base + x - v;
}

// a4/a5 bookkeeping (one block of 1024 threads, E <= 1024):
// counts, kept = min(counts, C), offsets = exclusive scan of kept, and the
// per-chunk base rank chunk_base[c][e] = sum_{c' < c} hist[c'][e].
__global__ void __launch_bounds__(1024)
scan_kernel(const int* __restrict__ hist, int n_chunks, int E, int cap, int* __restrict__ counts,
            int* __restrict__ kept, int* __restrict__ offsets, int* __restrict__ chunk_base) {
  pdl_wait();
  pdl_trigger();
  const int ex = threadIdx.x;
  int kv = 0;
  if (ex < E) {
    int run = 0;
    for (int c = 0; c < n_chunks; ++c) {
      int v = hist[(size_t)c * E + ex];
      chunk_base[(size_t)c * E + ex] = run;
      run += v;
    }
    if (counts) counts[ex] = run;
    kv = run < cap ? run : cap;
    kept[ex] = kv;
  }
  int total;
  int off = block_exclusive_scan(kv, &total);
  if (ex < E) offsets[ex] = off;
  if (ex == 0) offsets[E] = total;
}

// Group table of the grouped FFN: groups 0..E_r-1 are the routed experts
// (rows offsets[g] .. offsets[g+1]-1), groups E_r..E_r+E_s-1 the shared experts
// (T rows each, row base j*T); unit prefixes for the two GEMMs, with tiles of
// bm rows and nt_* column tiles per group.
__global__ void __launch_bounds__(1024)
groups_kernel(const int* __restrict__ offsets, int E_r, int E_s, int T, int bm, int merge_max, int nt_gu_r,
              int nt_gu_s, int nt_dn_r, int nt_dn_s, int* __restrict__ grp_rows,
              int* __restrict__ grp_row0, int* __restrict__ pre_gu, int* __restrict__ pre_dn,
              int max_rows, int* err, int* tile_counters) {
  pdl_wait();
  pdl_trigger();
  if (tile_counters && threadIdx.x < 2) tile_counters[threadIdx.x] = 0;   // GEMM unit counters
  const int G = E_r + E_s;
  // routed offsets must be non-decreasing within [0, max_rows]; otherwise no
  // unit is scheduled (the FFN writes nothing) and the error word is set
  int bad = 0;
  for (int g = threadIdx.x; g < E_r; g += blockDim.x)
    bad |= offsets[g + 1] < offsets[g];
  if (threadIdx.x == 0) bad |= offsets[0] < 0 || offsets[E_r] > max_rows;
  bad = __syncthreads_or(bad);
  if (bad && threadIdx.x == 0) set_device_error(err, MOE_DEVERR_INDEX);
  // G <= 1032: each thread handles up to two groups (g and g + 1024 folded)
  int carry_gu = 0, carry_dn = 0;
  for (int base = 0; base < G; base += blockDim.x) {
    int g = base + threadIdx.x;
    int rows = 0, row0 = 0, ugu = 0, udn = 0;
    if (g < G) {
      if (g < E_r) { row0 = offsets[g]; rows = bad ? 0 : offsets[g + 1] - row0; }
      else { rows = bad ? 0 : T; row0 = (g - E_r) * T; }
      // row units: one per bm-row tile; a last tile of <= merge_max rows
      // shares the unit of the tile before it (tensor-core GEMM)
      int mt = (rows + bm - 1) / bm;
      if (mt >= 2 && rows - (mt - 1) * bm <= merge_max) --mt;
      ugu = mt * (g < E_r ? nt_gu_r : nt_gu_s);
      udn = mt * (g < E_r ? nt_dn_r : nt_dn_s);
      grp_rows[g] = rows;
      grp_row0[g] = row0;
    }
    int tot_gu, tot_dn;
    int pgu = block_exclusive_scan(ugu, &tot_gu);
    int pdn = block_exclusive_scan(udn, &tot_dn);
    if (g < G) { pre_gu[g] = carry_gu + pgu; pre_dn[g] = carry_dn + pdn; }
    carry_gu += tot_gu;
    carry_dn += tot_dn;
  }
  if (threadIdx.x == 0) { pre_gu[G] = carry_gu; pre_dn[G] = carry_dn; }
}

// a5: stable scatter.  One block of 256 threads per chunk of 256 tokens; the
// rank of (t, e) among the chunk's tokens choosing e comes from per-warp lane
// masks, so rows stay in ascending token order within each expert.
__global__ void __launch_bounds__(256)
scatter_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gates,
               const int* __restrict__ offsets, const int* __restrict__ chunk_base, int cap,
               int T, int K, int E, int32_t* __restrict__ perm_tok, int32_t* __restrict__ row_of,
               float* __restrict__ row_gate, int* err) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t sm_scatter[];
  uint32_t* wmask = sm_scatter;                        // [8][E]
  int* wbase = reinterpret_cast<int*>(sm_scatter + 8 * E);   // [8][E]
  const int chunk = blockIdx.x, tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
  for (int i = tid; i < 8 * E; i += blockDim.x) wmask[i] = 0;
  __syncthreads();
  const int t = chunk * 256 + tid;
  const bool valid = t < T;
  if (valid) {
    for (int k = 0; k < K; ++k) {
      int ex = idx[(size_t)t * K + k];
      if (ex < 0 || ex >= E) { set_device_error(err, MOE_DEVERR_INDEX); continue; }
      atomicOr(&wmask[warp * E + ex], 1u << lane);
    }
  }
  __syncthreads();
  for (int ex = tid; ex < E; ex += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 8; ++w) { wbase[w * E + ex] = run; run += __popc(wmask[w * E + ex]); }
  }
  __syncthreads();
  if (valid) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
      int ex = idx[(size_t)t * K + k];
      int row = -1;
      if (ex >= 0 && ex < E) {
        int r = chunk_base[(size_t)chunk * E + ex] + wbase[warp * E + ex] +
                __popc(wmask[warp * E + ex] & lt);
        if (r < cap) {
          row = offsets[ex] + r;
          if (row >= offsets[ex + 1]) {           // self-check: rank past the expert's rows
            set_device_error(err, MOE_DEVERR_INDEX);
            row = -1;
          } else {
            perm_tok[row] = t;
            if (row_gate) row_gate[row] = gates[(size_t)t * K + k];
          }
        }
      }
      row_of[(size_t)t * K + k] = row;
    }
  }
}

// x_perm[r] = h[perm_tok[r]] for r < offsets[E] (one warp per row, 16-byte
// moves); with s_src, also s_dst[r] = s_src[perm_tok[r]] (row scales of e4m3 rows)
__global__ void gather_rows_kernel(const uint4* __restrict__ h, const int32_t* __restrict__ perm_tok,
                                   const int* __restrict__ n_rows_ptr, uint4* __restrict__ x_perm,
                                   int vec_per_row, int n_tok, int max_rows, int* err,
                                   const float* __restrict__ s_src, float* __restrict__ s_dst) {
  pdl_wait();
  pdl_trigger();
  const int n = min(*n_rows_ptr, max_rows);
  const int lane = threadIdx.x % kWarp;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
  const int nw = gridDim.x * blockDim.x / kWarp;
  for (int r = gw; r < n; r += nw) {
    const int t = perm_tok[r];
    if ((unsigned)t >= (unsigned)n_tok) {            // self-check: never read outside h
      if (lane == 0) set_device_error(err, MOE_DEVERR_INDEX);
      continue;
    }
    if (s_src && lane == 0) s_dst[r] = s_src[t];
    const uint4* src = h + (size_t)t * vec_per_row;
    uint4* dst = x_perm + (size_t)r * vec_per_row;
    // 4 independent 16-byte loads in flight per lane before the stores
    int v = lane;
    for (; v + 3 * kWarp < vec_per_row; v += 4 * kWarp) {
      const uint4 a = src[v], b = src[v + kWarp], c = src[v + 2 * kWarp], e = src[v + 3 * kWarp];
      dst[v] = a; dst[v + kWarp] = b; dst[v + 2 * kWarp] = c; dst[v + 3 * kWarp] = e;
    }
    for (; v < vec_per_row; v += kWarp) dst[v] = src[v];
  }
}

// The same gather on the TMA engine's untiled bulk copies: one thread per CTA
// streams whole rows h[perm_tok[r]] -> shared memory -> x_perm[r] through a
// ring of n_buf row buffers (rows r = blockIdx.x + j * gridDim.x): n_buf -
// kGatherStoresInFlight row loads and the shared-memory reads of up to
// kGatherStoresInFlight row stores are in flight per CTA, and every write
// leaves as whole lines.  Addresses and row_bytes are multiples of 16 (checked
// by the launcher).  A row whose token index is out of range is neither read
// nor written (MOE_DEVERR_INDEX); every wait is bounded.
constexpr bool kGatherBulk = true;
constexpr int kGatherRingBytes = 96 * 1024;   // ring bytes per CTA at most
constexpr int kGatherMaxBuf = 16;
constexpr int kGatherStoresInFlight = 2;

__device__ __forceinline__ void bulk_load_row(void* sdst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(sdst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_store_row(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(gdst), "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}

__global__ void __launch_bounds__(32) gather_rows_bulk_kernel(
    const uint8_t* __restrict__ h, const int32_t* __restrict__ perm_tok, const int* __restrict__ n_rows_ptr,
    uint8_t* __restrict__ x_perm, int row_bytes, int n_buf, int max_my, int n_tok, int max_rows, int* err,
    const float* __restrict__ s_src, float* __restrict__ s_dst) {
  // n_buf row buffers, n_buf barriers, then the token of each of this CTA's rows
  extern __shared__ __align__(128) uint8_t ring[];
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)n_buf * row_bytes);
  int32_t* tok = reinterpret_cast<int32_t*>(full + n_buf);
  __shared__ int abort_flag;
  const int lane = threadIdx.x;
  if (lane == 0) {
    for (int b = 0; b < n_buf; ++b) mbar_init(&full[b], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();
  pdl_trigger();
  const int n = min(*n_rows_ptr, max_rows);
  int my = n > (int)blockIdx.x ? (n - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  if (my > max_my) {                                   // cannot happen with the launcher's grid
    if (lane == 0) set_device_error(err, MOE_DEVERR_INDEX);
    my = max_my;
  }
  auto row_of_j = [&](int j) { return (int)blockIdx.x + j * (int)gridDim.x; };
  // all lanes fetch the tokens (and, for e4m3 rows, copy the row scales) so
  // that the issuing lane never waits on a global load
#pragma unroll 4
  for (int j = lane; j < my; j += kWarp) {
    const int r = row_of_j(j), t = perm_tok[r];
    tok[j] = t;
    if (s_src && (unsigned)t < (unsigned)n_tok) s_dst[r] = s_src[t];
  }
  __syncwarp();
  if (lane != 0) return;
  auto issue = [&](int j) {
    const int b = j % n_buf;
    const int t = tok[j];
    if ((unsigned)t >= (unsigned)n_tok) {             // self-check: never read outside h
      set_device_error(err, MOE_DEVERR_INDEX);
      mbar_arrive(&full[b]);                           // completes the phase with no bytes
      return;
    }
    mbar_arrive_expect_tx(&full[b], (uint32_t)row_bytes);
    bulk_load_row(ring + (size_t)b * row_bytes, h + (size_t)t * row_bytes, (uint32_t)row_bytes, &full[b]);
  };
  // row j + ahead goes into the buffer of row j - kGatherStoresInFlight, whose
  // store is the oldest of the kGatherStoresInFlight + 1 committed last
  const int ahead = n_buf - kGatherStoresInFlight;
  int issued = 0;
  for (; issued < my && issued < ahead; ++issued) issue(issued);
  for (int j = 0; j < my; ++j) {
    const int b = j % n_buf;
    if (!mbar_wait(&full[b], (uint32_t)(j / n_buf) & 1u, &abort_flag, err)) break;
    if ((unsigned)tok[j] < (unsigned)n_tok) {
      fence_proxy_async_smem();
      bulk_store_row(x_perm + (size_t)row_of_j(j) * row_bytes, ring + (size_t)b * row_bytes, (uint32_t)row_bytes);
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");   // one group per row, even an empty one
    if (issued < my) {
      asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kGatherStoresInFlight) : "memory");
      issue(issued++);
    }
  }
  // after an abandoned wait, the loads still in flight (the last `ahead`
  // issued at most) must land before the CTA exits
  if (abort_flag) {
    for (int j = max(0, issued - ahead); j < issued; ++j) {
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&full[j % n_buf], (uint32_t)(j / n_buf) & 1u) &&
             global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// dst[r] = src[map[r]] (map[r] < 0: a zero row) for r < n_rows; rows of
// row_words 32-bit words, moved 16 bytes at a time when row_words % 4 == 0.
__global__ void gather_map_kernel(const uint32_t* __restrict__ src, const int32_t* __restrict__ map,
                                  int64_t n_rows, int64_t n_src, int row_words, uint32_t* __restrict__ dst,
                                  int* err) {
  const int lane = threadIdx.x % kWarp;
  const int64_t nw = (int64_t)gridDim.x * blockDim.x / kWarp;
  for (int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / kWarp; r < n_rows; r += nw) {
    const int32_t m = map[r];
    if (m >= n_src) {                                  // self-check: never read outside src
      if (lane == 0 && err) set_device_error(err, MOE_DEVERR_INDEX);
      continue;
    }
    uint32_t* d = dst + r * row_words;
    if ((row_words & 3) == 0) {
      uint4* d4 = reinterpret_cast<uint4*>(d);
      const uint4* s4 = m >= 0 ? reinterpret_cast<const uint4*>(src + (int64_t)m * row_words) : nullptr;
      for (int v = lane; v < row_words / 4; v += kWarp) d4[v] = s4 ? s4[v] : make_uint4(0, 0, 0, 0);
    } else {
      const uint32_t* s1 = m >= 0 ? src + (int64_t)m * row_words : nullptr;
      for (int v = lane; v < row_words; v += kWarp) d[v] = s1 ? s1[v] : 0u;
    }
  }
}

// a8: y_t = res*h_t + sum_j shared[j,t] + sum_k slot[row_of[t,k]], fp32 in that order.
// S: element type of the slot and shared rows (T, or fp16 for a bf16 layer's own).
template <typename T, typename S = T>
__global__ void __launch_bounds__(128)
combine_kernel(const T* __restrict__ h, const S* __restrict__ slot, const S* __restrict__ shared,
               const int32_t* __restrict__ row_of, T* __restrict__ y, int n_tok, int d, int K,
               int E_s, int add_residual, int n_slot_rows) {
  pdl_wait();
  pdl_trigger();
  constexpr int VEC = 16 / sizeof(T);
  const int t = blockIdx.x;
  int rows[32];
  for (int k = 0; k < K; ++k) {
    int r = row_of[(size_t)t * K + k];
    rows[k] = r < n_slot_rows ? r : -1;       // self-check: never read past the slot rows
  }
  // blockIdx.y splits a token's row over several blocks when there are few tokens
  for (int c = (blockIdx.y * blockDim.x + threadIdx.x) * VEC; c < d; c += blockDim.x * gridDim.y * VEC) {
    float acc[VEC];
    {
      uint4 raw = *reinterpret_cast<const uint4*>(h + (size_t)t * d + c);
      const T* v = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = add_residual ? to_f32(v[i]) : 0.f;
    }
    for (int j = 0; j < E_s; ++j) {
      uint4 raw = *reinterpret_cast<const uint4*>(shared + ((size_t)j * n_tok + t) * d + c);
      const S* v = reinterpret_cast<const S*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], to_f32(v[i]));
    }
    for (int k = 0; k < K; ++k) {
      if (rows[k] < 0) continue;
      uint4 raw = *reinterpret_cast<const uint4*>(slot + (size_t)rows[k] * d + c);
      const S* v = reinterpret_cast<const S*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], to_f32(v[i]));
    }
    uint4 out;
    T* o = reinterpret_cast<T*>(&out);
#pragma unroll
    for (int i = 0; i < VEC; ++i) o[i] = from_f32<T>(acc[i]);
    *reinterpret_cast<uint4*>(y + (size_t)t * d + c) = out;
  }
}

// Combine with K fixed at compile time: the K row indices stay in registers
// and every row's 16-byte chunk is loaded before the sums, which run in the
// same fixed order as combine_kernel (h, shared j ascending, slots k
// ascending), so the results are bit-identical.  Six resident blocks per SM
// (registers capped at 80): more loads in flight per SM than the five the
// unconstrained register count allows (measured 10-12 % faster), without the
// spills that eight would cost.
template <typename T, int KT, typename S = T>
__global__ void __launch_bounds__(128, 6)
combine_k_kernel(const T* __restrict__ h, const S* __restrict__ slot, const S* __restrict__ shared,
                 const int32_t* __restrict__ row_of, T* __restrict__ y, int n_tok, int d, int E_s,
                 int add_residual, int n_slot_rows) {
  pdl_wait();
  pdl_trigger();
  constexpr int VEC = 16 / sizeof(T);
  const int t = blockIdx.x;
  int rows[KT];
#pragma unroll
  for (int k = 0; k < KT; ++k) {
    const int r = __ldg(row_of + (size_t)t * KT + k);
    rows[k] = r < n_slot_rows ? r : -1;       // self-check: never read past the slot rows
  }
  for (int c = (blockIdx.y * blockDim.x + threadIdx.x) * VEC; c < d; c += blockDim.x * gridDim.y * VEC) {
    uint4 sv[KT];
#pragma unroll
    for (int k = 0; k < KT; ++k)
      sv[k] = rows[k] >= 0 ? __ldg(reinterpret_cast<const uint4*>(slot + (size_t)rows[k] * d + c))
                           : make_uint4(0, 0, 0, 0);
    const uint4 hv = __ldg(reinterpret_cast<const uint4*>(h + (size_t)t * d + c));
    float acc[VEC];
    {
      const T* v = reinterpret_cast<const T*>(&hv);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = add_residual ? to_f32(v[i]) : 0.f;
    }
    for (int j = 0; j < E_s; ++j) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(shared + ((size_t)j * n_tok + t) * d + c));
      const S* v = reinterpret_cast<const S*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], to_f32(v[i]));
    }
#pragma unroll
    for (int k = 0; k < KT; ++k) {
      if (rows[k] < 0) continue;
      const S* v = reinterpret_cast<const S*>(&sv[k]);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], to_f32(v[i]));
    }
    uint4 out;
    T* o = reinterpret_cast<T*>(&out);
#pragma unroll
    for (int i = 0; i < VEC; ++i) o[i] = from_f32<T>(acc[i]);
    *reinterpret_cast<uint4*>(y + (size_t)t * d + c) = out;
  }
}

// a9: b_i += gamma * sign(K*T - E_r*c_i) (one fp32 add), and MaxVio.
__global__ void __launch_bounds__(1024)
bias_update_kernel(const int* __restrict__ counts, float* __restrict__ b, float gamma,
                   float* __restrict__ max_vio, int E, int K, int T) {
  pdl_wait();
  pdl_trigger();
  __shared__ int smax[32];
  const int ex = threadIdx.x;
  int c = ex < E ? counts[ex] : 0;
  if (ex < E && b) {
    long long diff = (long long)K * T - (long long)E * c;
    float step = diff > 0 ? gamma : (diff < 0 ? -gamma : 0.0f);
    b[ex] = __fadd_rn(b[ex], step);
  }
  int m = c;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(kFull, m, off));
  if (threadIdx.x % kWarp == 0) smax[threadIdx.x / kWarp] = m;
  __syncthreads();
  if (threadIdx.x == 0 && max_vio) {
    int mm = 0;
    for (int w = 0; w < (int)(blockDim.x / kWarp); ++w) mm = max(mm, smax[w]);
    double cbar = (double)K * (double)T / (double)E;
    max_vio[0] = (float)(((double)mm - cbar) / cbar);
  }
}

// ---------------------------------------------------------------------------
// Router losses and logging: Switch aux loss, router z-loss, sequence-wise
// balance loss, load entropy, MaxVio, dropped rate.  Deterministic: integer
// atomics only, every float sum in a fixed order.
// ---------------------------------------------------------------------------

// Per token: row sum of s (for s' = s / sum s), (logsumexp z)^2, and the
// per-sequence selection counts.
__global__ void __launch_bounds__(256)
stats_token_kernel(const float* __restrict__ s, const float* __restrict__ z,
                   const int32_t* __restrict__ idx, float* __restrict__ rowsum,
                   float* __restrict__ lse2, int* __restrict__ seq_counts, int T, int E, int K,
                   int seq_len) {
  const int lane = threadIdx.x % kWarp;
  const int t = blockIdx.x * (blockDim.x / kWarp) + threadIdx.x / kWarp;
  if (t >= T) return;
  float acc = 0.f;
  for (int i = lane; i < E; i += kWarp) acc = __fadd_rn(acc, s[(size_t)t * E + i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, off));
  if (z) {
    float m = -INFINITY;
    for (int i = lane; i < E; i += kWarp) m = fmaxf(m, z[(size_t)t * E + i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    float e = 0.f;
    for (int i = lane; i < E; i += kWarp) e = __fadd_rn(e, expf(z[(size_t)t * E + i] - m));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) e = __fadd_rn(e, __shfl_xor_sync(kFull, e, off));
    if (lane == 0) {
      const float lse = m + logf(e);
      lse2[t] = lse * lse;
    }
  }
  if (lane == 0) rowsum[t] = acc;
  if (lane < K) {
    const int ex = idx[(size_t)t * K + lane];
    if (ex >= 0 && ex < E) atomicAdd(&seq_counts[(size_t)(t / seq_len) * E + ex], 1);
  }
}

// Per (sequence b, chunk j of kStatsChunk tokens, expert i): the partial sum
// of s'_{t,i} over the chunk, so that a long sequence is spread over many
// blocks; the final kernel adds the chunks of a sequence in ascending order.
__global__ void __launch_bounds__(256)
stats_seq_kernel(const float* __restrict__ s, const float* __restrict__ rowsum,
                 float* __restrict__ pchunk, int E, int seq_len, int n_ch) {
  const int b = blockIdx.x / n_ch, j = blockIdx.x % n_ch;
  const int i = blockIdx.y * blockDim.x + threadIdx.x;
  if (i >= E) return;
  const size_t t0 = (size_t)b * seq_len + (size_t)j * kStatsChunk;
  const int n = min(kStatsChunk, seq_len - j * kStatsChunk);
  float acc = 0.f;
  for (int t = 0; t < n; ++t) acc = __fadd_rn(acc, __fdiv_rn(s[(t0 + t) * E + i], rowsum[t0 + t]));
  pchunk[(size_t)blockIdx.x * E + i] = acc;
}

// Block-wide sum of one value per thread in a fixed tree order.
__device__ double block_sum_fixed(double v) {
  __shared__ double part[32];
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  if (lane == 0) part[warp] = v;
  __syncthreads();
  double r = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < (int)(blockDim.x / kWarp); ++w) r += part[w];
  __syncthreads();
  return r;     // valid in thread 0
}

// Final reductions (one block of 1024 threads, one expert per thread).
__global__ void __launch_bounds__(1024)
stats_final_kernel(const float* __restrict__ pchunk, const int* __restrict__ seq_counts,
                   const float* __restrict__ lse2, const int32_t* __restrict__ kept, int T, int E,
                   int K, int seq_len, int n_ch, int use_seq, float alpha_aux, float c_z,
                   float alpha_seq, float* __restrict__ stats) {
  const int i = threadIdx.x;
  const int n_seq = T / seq_len;
  double c_i = 0.0, P_i = 0.0, seq_i = 0.0;
  if (i < E) {
    for (int b = 0; b < n_seq; ++b) {
      const double cb = seq_counts[(size_t)b * E + i];
      double pb = 0.0;
      for (int j = 0; j < n_ch; ++j) pb += pchunk[((size_t)b * n_ch + j) * E + i];
      pb /= seq_len;
      c_i += cb;
      P_i += pb;
      seq_i += (double)E / ((double)K * seq_len) * cb * pb;
    }
    P_i /= n_seq;
  }
  const double f_i = (double)E / ((double)K * T) * c_i;
  const double aux = block_sum_fixed(i < E ? f_i * P_i : 0.0);
  const double seq = block_sum_fixed(i < E ? seq_i : 0.0);
  const double share = c_i / ((double)K * T);
  const double ent = block_sum_fixed((i < E && share > 0.0) ? -share * log(fmax(share, 1e-9)) : 0.0);
  const double ksum = block_sum_fixed((i < E && kept) ? (double)kept[i] : 0.0);
  __shared__ int cmax_s;
  if (threadIdx.x == 0) cmax_s = 0;
  __syncthreads();
  if (i < E) atomicMax(&cmax_s, (int)c_i);
  double zsum = 0.0;
  for (int t = threadIdx.x; t < T && lse2; t += blockDim.x) zsum += lse2[t];
  const double zl = block_sum_fixed(zsum);
  __syncthreads();
  if (threadIdx.x == 0) {
    const double cbar = (double)K * T / E;
    stats[0] = (float)(alpha_aux * aux);
    stats[1] = lse2 ? (float)(c_z * zl / T) : 0.0f;
    stats[2] = use_seq ? (float)(alpha_seq * seq / n_seq) : 0.0f;
    stats[3] = (float)ent;
    stats[4] = (float)(((double)cmax_s - cbar) / cbar);
    stats[5] = kept ? (float)(1.0 - ksum / ((double)K * T)) : 0.0f;
  }
}

// Failure-detection self-test: one thread waits, through the same bounded
// mbarrier wait the GEMM pipelines use, on a barrier nothing arrives on.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_barrier_init();
  mbar_wait(&bar, 0, &abort_flag, err, limit_ns);     // never completes: times out
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

void launch_router_stats(const float* s, const float* z, const int32_t* idx, const int32_t* kept,
                         int T, int E, int K, int seq_len, int use_seq, float alpha_aux, float c_z,
                         float alpha_seq, float* rowsum, float* lse2, int* seq_counts, float* pchunk,
                         float* stats, cudaStream_t st) {
  const int n_seq = T / seq_len;
  const int n_ch = (seq_len + kStatsChunk - 1) / kStatsChunk;
  cudaMemsetAsync(seq_counts, 0, (size_t)n_seq * E * sizeof(int), st);
  stats_token_kernel<<<(T + 7) / 8, 256, 0, st>>>(s, z, idx, rowsum, z ? lse2 : nullptr, seq_counts,
                                                  T, E, K, seq_len);
  stats_seq_kernel<<<dim3(n_seq * n_ch, (E + 255) / 256), 256, 0, st>>>(s, rowsum, pchunk, E, seq_len,
                                                                       n_ch);
  stats_final_kernel<<<1, 1024, 0, st>>>(pchunk, seq_counts, z ? lse2 : nullptr, kept, T, E, K,
                                         seq_len, n_ch, use_seq, alpha_aux, c_z, alpha_seq, stats);
}

void launch_bounded_wait_selftest(uint64_t limit_ns, int* err, cudaStream_t st) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, err);
}
void launch_router_logits(const void* h, int dtype, const float* e, float* z, int T, int d, int E,
                          cudaStream_t st) {
  dim3 grid((T + 63) / 64, (E + 63) / 64);
  if (dtype == MOE_DTYPE_BF16)
    router_logits_simt_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)h, e, z, T, d, E);
  else
    router_logits_simt_kernel<float><<<grid, 256, 0, st>>>((const float*)h, e, z, T, d, E);
}

void launch_select(const float* in, int n_parts, int in_is_scores, const float* bias, int score_fn,
                   float* s_out, float* z_out, int32_t* idx, float* gates, int* hist, int chunk_shift,
                   int T, int E, int K, int n_groups, int topk_groups, int group_topn, cudaStream_t st) {
  const int warps = 8;
  dim3 grid((T + warps - 1) / warps);
  int kpl = (E + 31) / 32;
#define MOE_SEL(N) launch_pdl(select_kernel<N>, grid, dim3(warps * 32), 0, st, in, n_parts, in_is_scores, bias, \
      score_fn, s_out, z_out, idx, gates, hist, chunk_shift, T, E, K, n_groups, topk_groups, group_topn)
  if (kpl <= 1) MOE_SEL(1);
  else if (kpl <= 2) MOE_SEL(2);
  else if (kpl <= 4) MOE_SEL(4);
  else if (kpl <= 8) MOE_SEL(8);
  else if (kpl <= 16) MOE_SEL(16);
  else MOE_SEL(32);
#undef MOE_SEL
}

void launch_hist(const int32_t* idx, int* hist, int chunk_shift, int T, int K, int E, int* err,
                 cudaStream_t st) {
  int n = T * K;
  hist_kernel<<<(n + 255) / 256, 256, 0, st>>>(idx, hist, chunk_shift, T, K, E, err);
}

void launch_counts(const int* hist, int n_chunks, int E, int* counts, cudaStream_t st) {
  counts_kernel<<<(E + 255) / 256, 256, 0, st>>>(hist, n_chunks, E, counts);
}

void launch_scan(const int* hist, int n_chunks, int E, int cap, int* counts, int* kept,
                 int* offsets, int* chunk_base, cudaStream_t st) {
  launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, hist, n_chunks, E, cap, counts, kept, offsets, chunk_base);
}

void launch_groups(const int* offsets, int E_r, int E_s, int T, int bm, int merge_max, int nt_gu_r, int nt_gu_s,
                   int nt_dn_r, int nt_dn_s, int* grp_rows, int* grp_row0, int* pre_gu,
                   int* pre_dn, int max_rows, int* err, int* tile_counters, cudaStream_t st) {
  launch_pdl(groups_kernel, dim3(1), dim3(1024), 0, st, offsets, E_r, E_s, T, bm, merge_max, nt_gu_r, nt_gu_s,
             nt_dn_r, nt_dn_s, grp_rows, grp_row0, pre_gu, pre_dn, max_rows, err, tile_counters);
}

void launch_scatter(const int32_t* idx, const float* gates, const int* offsets,
                    const int* chunk_base, int cap, int T, int K, int E, int32_t* perm_tok,
                    int32_t* row_of, float* row_gate, int* err, cudaStream_t st) {
  int n_chunks = (T + 255) / 256;
  size_t smem = (size_t)16 * E * sizeof(uint32_t);      // 64 KB at E = 1024
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 16 * 1024 * 4);
    attr_done[dev] = true;
  }
  launch_pdl(scatter_kernel, dim3(n_chunks), dim3(256), smem, st, idx, gates, offsets, chunk_base, cap, T, K, E,
             perm_tok, row_of, row_gate, err);
}

void launch_gather(const void* h, const int32_t* perm_tok, const int* n_rows_ptr, void* x_perm,
                   int d, int elem_bytes, int max_rows, int n_tok, int* err, cudaStream_t st,
                   const float* s_src, float* s_dst) {
  const int row_bytes = d * elem_bytes;
  const int n_buf = std::min(kGatherMaxBuf, kGatherRingBytes / std::max(row_bytes, 16));
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  sms = std::max(sms, 1);
  const size_t ring = (size_t)n_buf * row_bytes + (size_t)n_buf * sizeof(uint64_t);
  // as many CTAs per SM as their rings fit in 224 KB (at most 6)
  const int per_sm = std::max(1, std::min(6, (224 * 1024) / (int)(ring + 1024 + 8 * 1024)));
  const int blocks = std::min(std::max(max_rows, 1), per_sm * sms);
  const int max_my = (std::max(max_rows, 1) + blocks - 1) / blocks;   // rows per CTA at most
  const size_t smem = ring + (size_t)max_my * sizeof(int32_t);
  if (kGatherBulk && n_buf >= kGatherStoresInFlight + 2 && row_bytes % 16 == 0 && max_my <= 2048 &&
      ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(x_perm)) & 15) == 0) {
    static bool attr_done[64] = {};
    if (dev < 64 && !attr_done[dev]) {
      cudaFuncSetAttribute(gather_rows_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kGatherRingBytes + kGatherMaxBuf * (int)sizeof(uint64_t) + 2048 * 4);
      attr_done[dev] = true;
    }
    launch_pdl(gather_rows_bulk_kernel, dim3(blocks), dim3(kWarp), smem, st, (const uint8_t*)h, perm_tok,
               n_rows_ptr, (uint8_t*)x_perm, row_bytes, n_buf, max_my, n_tok, max_rows, err, s_src, s_dst);
    return;
  }
  int vec = d * elem_bytes / 16;
  int warps = max_rows < 148 * 64 ? max_rows : 148 * 64;
  if (warps < 1) warps = 1;
  const int ldst_blocks = (warps * 32 + 255) / 256;
  launch_pdl(gather_rows_kernel, dim3(ldst_blocks), dim3(256), 0, st, (const uint4*)h, perm_tok, n_rows_ptr,
             (uint4*)x_perm, vec, n_tok, max_rows, err, s_src, s_dst);
}

void launch_combine(const void* h, const void* slot, const void* shared, const int32_t* row_of,
                    void* y, int T, int d, int K, int E_s, int add_residual, int dtype,
                    int n_slot_rows, cudaStream_t st, int slot_f16) {
  // enough blocks to fill the GPU even for decode-sized batches
  const int nvec = d * (dtype == MOE_DTYPE_BF16 ? 2 : 4) / 16;
  int split = (2 * 148 + T - 1) / T;
  const int max_split = (nvec + 127) / 128;
  split = split < 1 ? 1 : (split > max_split ? max_split : split);
  const dim3 grid(T, split);
  if (dtype == MOE_DTYPE_BF16 && slot_f16 && (K == 2 || K == 4 || K == 6 || K == 8)) {
    const bf16* hh = (const bf16*)h;
    const __half *sl = (const __half*)slot, *sh = (const __half*)shared;
    bf16* yy = (bf16*)y;
    auto kern = K == 8 ? combine_k_kernel<bf16, 8, __half> : K == 6 ? combine_k_kernel<bf16, 6, __half>
              : K == 4 ? combine_k_kernel<bf16, 4, __half> : combine_k_kernel<bf16, 2, __half>;
    launch_pdl(kern, grid, dim3(128), 0, st, hh, sl, sh, row_of, yy, T, d, E_s, add_residual, n_slot_rows);
  } else if (dtype == MOE_DTYPE_BF16 && slot_f16) {
    launch_pdl(combine_kernel<bf16, __half>, grid, dim3(128), 0, st, (const bf16*)h, (const __half*)slot,
               (const __half*)shared, row_of, (bf16*)y, T, d, K, E_s, add_residual, n_slot_rows);
  } else if (dtype == MOE_DTYPE_BF16 && (K == 2 || K == 4 || K == 6 || K == 8)) {
    const bf16 *hh = (const bf16*)h, *sl = (const bf16*)slot, *sh = (const bf16*)shared;
    bf16* yy = (bf16*)y;
    auto kern = K == 8 ? combine_k_kernel<bf16, 8> : K == 6 ? combine_k_kernel<bf16, 6>
              : K == 4 ? combine_k_kernel<bf16, 4> : combine_k_kernel<bf16, 2>;
    launch_pdl(kern, grid, dim3(128), 0, st, hh, sl, sh, row_of, yy, T, d, E_s, add_residual, n_slot_rows);
  } else if (dtype == MOE_DTYPE_BF16)
    launch_pdl(combine_kernel<bf16>, grid, dim3(128), 0, st, (const bf16*)h, (const bf16*)slot, (const bf16*)shared,
               row_of, (bf16*)y, T, d, K, E_s, add_residual, n_slot_rows);
  else
    launch_pdl(combine_kernel<float>, grid, dim3(128), 0, st, (const float*)h, (const float*)slot,
               (const float*)shared, row_of, (float*)y, T, d, K, E_s, add_residual, n_slot_rows);
}

void launch_gather_map(const void* src, const int32_t* map, int64_t n_rows, int64_t n_src, int row_bytes,
                       void* dst, int* err, cudaStream_t st) {
  if (n_rows <= 0) return;
  const int64_t warps = n_rows < 148 * 64 ? n_rows : 148 * 64;
  gather_map_kernel<<<(unsigned)((warps * kWarp + 255) / 256), 256, 0, st>>>(
      static_cast<const uint32_t*>(src), map, n_rows, n_src, row_bytes / 4, static_cast<uint32_t*>(dst), err);
}

void launch_bias_update(const int* counts, float* b, float gamma, float* max_vio, int E, int K,
                        int T, cudaStream_t st) {
  launch_pdl(bias_update_kernel, dim3(1), dim3(1024), 0, st, counts, b, gamma, max_vio, E, K, T);
}

}  // namespace moe
