// Grouped SwiGLU experts on CUDA cores, fp32 in and out with fp32
// accumulation: the path for float32 layers (the toy aux-loss-free workload),
// whose 1e-4 relative tolerance rules out reduced-precision tensor-core inputs.
//
// SwiGLU(h) = (SiLU(h W_gate^T) * (h W_up^T)) W_down^T -- "Sparse
// Mixture-of-Experts (MoE): Routing Math, Load Balancing & Expert
// Parallelism", section 0 (definition under the layer equation).
//
// Work units are (group, 32-row tile, 64-column tile); a unit's group comes
// from the device-side unit prefix written by groups_kernel, so the launch
// needs no host knowledge of the per-expert row counts.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSimtBM = 32, kSimtBN = 64, kSimtBK = 32;

__device__ __forceinline__ void decode_unit(const int* __restrict__ pre, const int* __restrict__ rows,
                                            int G, int u, int bm, int& g, int& mt, int& nt) {
  int lo = 0, hi = G;                       // pre[lo] <= u < pre[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (pre[mid] <= u) lo = mid; else hi = mid;
  }
  g = lo;
  int local = u - pre[g];
  int mtiles = (rows[g] + bm - 1) / bm;
  mt = local % mtiles;
  nt = local / mtiles;
}

template <typename T>
__global__ void __launch_bounds__(256)
ffn_gateup_simt_kernel(const T* __restrict__ x_r, const T* __restrict__ x_s,
                       const T* __restrict__ wg_r, const T* __restrict__ wu_r,
                       const T* __restrict__ wg_s, const T* __restrict__ wu_s,
                       const int* __restrict__ grp_rows, const int* __restrict__ grp_row0,
                       const int* __restrict__ pre, int G, int E_r, int d, int f_r, int f_s,
                       T* __restrict__ act_r, T* __restrict__ act_s) {
  __shared__ float xs[kSimtBM][kSimtBK + 1];
  __shared__ float gs[kSimtBN][kSimtBK + 1];
  __shared__ float us[kSimtBN][kSimtBK + 1];
  const int u = blockIdx.x;
  if (u >= pre[G]) return;
  int g, mt, nt;
  decode_unit(pre, grp_rows, G, u, kSimtBM, g, mt, nt);
  const bool sh = g >= E_r;
  const int rows = grp_rows[g], row0 = grp_row0[g];
  const int f = sh ? f_s : f_r;
  const T* X = sh ? x_s : x_r + (size_t)row0 * d;
  const T* Wg = sh ? wg_s + (size_t)(g - E_r) * f_s * d : wg_r + (size_t)g * f_r * d;
  const T* Wu = sh ? wu_s + (size_t)(g - E_r) * f_s * d : wu_r + (size_t)g * f_r * d;
  T* out = sh ? act_s + (size_t)row0 * f_s : act_r + (size_t)row0 * f_r;

  const int tid = threadIdx.x, r = tid / 8, c = tid % 8;
  float ag[8] = {}, au[8] = {};
  for (int k0 = 0; k0 < d; k0 += kSimtBK) {
    for (int i = tid; i < kSimtBM * kSimtBK; i += 256) {
      int rr = i / kSimtBK, kk = i % kSimtBK, m = mt * kSimtBM + rr;
      xs[rr][kk] = (m < rows && k0 + kk < d) ? to_f32(X[(size_t)m * d + k0 + kk]) : 0.f;
    }
    for (int i = tid; i < kSimtBN * kSimtBK; i += 256) {
      int cc = i / kSimtBK, kk = i % kSimtBK, n = nt * kSimtBN + cc;
      bool ok = n < f && k0 + kk < d;
      gs[cc][kk] = ok ? to_f32(Wg[(size_t)n * d + k0 + kk]) : 0.f;
      us[cc][kk] = ok ? to_f32(Wu[(size_t)n * d + k0 + kk]) : 0.f;
    }
    __syncthreads();
    for (int kk = 0; kk < kSimtBK; ++kk) {
      float xv = xs[r][kk];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ag[i] = fmaf(xv, gs[c + 8 * i][kk], ag[i]);
        au[i] = fmaf(xv, us[c + 8 * i][kk], au[i]);
      }
    }
    __syncthreads();
  }
  const int m = mt * kSimtBM + r;
  if (m >= rows) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int n = nt * kSimtBN + c + 8 * i;
    if (n < f) {
      float gv = ag[i];
      float a = __fdiv_rn(gv, 1.0f + expf(-gv)) * au[i];
      out[(size_t)m * f + n] = from_f32<T>(a);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
ffn_down_simt_kernel(const T* __restrict__ act_r, const T* __restrict__ act_s,
                     const T* __restrict__ wd_r, const T* __restrict__ wd_s,
                     const int* __restrict__ grp_rows, const int* __restrict__ grp_row0,
                     const int* __restrict__ pre, int G, int E_r, int d, int f_r, int f_s,
                     const float* __restrict__ row_scale, T* __restrict__ out_r,
                     T* __restrict__ out_s) {
  __shared__ float as[kSimtBM][kSimtBK + 1];
  __shared__ float ws[kSimtBN][kSimtBK + 1];
  const int u = blockIdx.x;
  if (u >= pre[G]) return;
  int g, mt, nt;
  decode_unit(pre, grp_rows, G, u, kSimtBM, g, mt, nt);
  const bool sh = g >= E_r;
  const int rows = grp_rows[g], row0 = grp_row0[g];
  const int f = sh ? f_s : f_r;
  const T* A = sh ? act_s + (size_t)row0 * f_s : act_r + (size_t)row0 * f_r;
  const T* W = sh ? wd_s + (size_t)(g - E_r) * d * f_s : wd_r + (size_t)g * d * f_r;
  T* out = (sh ? out_s : out_r) + (size_t)row0 * d;

  const int tid = threadIdx.x, r = tid / 8, c = tid % 8;
  float acc[8] = {};
  for (int k0 = 0; k0 < f; k0 += kSimtBK) {
    for (int i = tid; i < kSimtBM * kSimtBK; i += 256) {
      int rr = i / kSimtBK, kk = i % kSimtBK, m = mt * kSimtBM + rr;
      as[rr][kk] = (m < rows && k0 + kk < f) ? to_f32(A[(size_t)m * f + k0 + kk]) : 0.f;
    }
    for (int i = tid; i < kSimtBN * kSimtBK; i += 256) {
      int cc = i / kSimtBK, kk = i % kSimtBK, n = nt * kSimtBN + cc;
      ws[cc][kk] = (n < d && k0 + kk < f) ? to_f32(W[(size_t)n * f + k0 + kk]) : 0.f;
    }
    __syncthreads();
    for (int kk = 0; kk < kSimtBK; ++kk) {
      float av = as[r][kk];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(av, ws[c + 8 * i][kk], acc[i]);
    }
    __syncthreads();
  }
  const int m = mt * kSimtBM + r;
  if (m >= rows) return;
  const float scale = (!sh && row_scale) ? row_scale[row0 + m] : 1.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int n = nt * kSimtBN + c + 8 * i;
    if (n < d) out[(size_t)m * d + n] = from_f32<T>(acc[i] * scale);
  }
}

int simt_bm() { return kSimtBM; }
int simt_bn() { return kSimtBN; }

void launch_ffn_simt(const FfnArgs& a, int which, cudaStream_t st) {
  // host bound on units: every group's row tiles times its column tiles
  const int nt_gu_r = (a.f_r + kSimtBN - 1) / kSimtBN, nt_gu_s = (a.f_s + kSimtBN - 1) / kSimtBN;
  const int nt_dn = (a.d + kSimtBN - 1) / kSimtBN;
  long long mt_r = (a.max_rows_r + kSimtBM - 1) / kSimtBM + a.E_r;
  long long mt_s = (long long)a.E_s * ((a.T + kSimtBM - 1) / kSimtBM);
  long long u_gu = mt_r * nt_gu_r + mt_s * nt_gu_s;
  long long u_dn = (mt_r + mt_s) * nt_dn;
  const int G = a.E_r + a.E_s;
  if (a.dtype == MOE_DTYPE_BF16) {
    using T = bf16;
    if (which == 0)
    ffn_gateup_simt_kernel<T><<<(unsigned)u_gu, 256, 0, st>>>(
        (const T*)a.x_r, (const T*)a.x_s, (const T*)a.wg_r, (const T*)a.wu_r, (const T*)a.wg_s,
        (const T*)a.wu_s, a.grp_rows, a.grp_row0, a.pre_gu, G, a.E_r, a.d, a.f_r, a.f_s,
        (T*)a.act_r, (T*)a.act_s);
    else
    ffn_down_simt_kernel<T><<<(unsigned)u_dn, 256, 0, st>>>(
        (const T*)a.act_r, (const T*)a.act_s, (const T*)a.wd_r, (const T*)a.wd_s, a.grp_rows,
        a.grp_row0, a.pre_dn, G, a.E_r, a.d, a.f_r, a.f_s, a.row_scale, (T*)a.out_r, (T*)a.out_s);
  } else {
    using T = float;
    if (which == 0)
    ffn_gateup_simt_kernel<T><<<(unsigned)u_gu, 256, 0, st>>>(
        (const T*)a.x_r, (const T*)a.x_s, (const T*)a.wg_r, (const T*)a.wu_r, (const T*)a.wg_s,
        (const T*)a.wu_s, a.grp_rows, a.grp_row0, a.pre_gu, G, a.E_r, a.d, a.f_r, a.f_s,
        (T*)a.act_r, (T*)a.act_s);
    else
    ffn_down_simt_kernel<T><<<(unsigned)u_dn, 256, 0, st>>>(
        (const T*)a.act_r, (const T*)a.act_s, (const T*)a.wd_r, (const T*)a.wd_s, a.grp_rows,
        a.grp_row0, a.pre_dn, G, a.E_r, a.d, a.f_r, a.f_s, a.row_scale, (T*)a.out_r, (T*)a.out_s);
  }
}

}  // namespace moe
