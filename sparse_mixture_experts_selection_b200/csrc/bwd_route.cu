// Backward of the routing and combine steps (everything around the expert
// GEMMs), deterministic: every floating-point sum runs in a fixed order.
//
//   per permuted row r of (t, k):  dO_r = g * dy_t,  dL/dg = <dy_t, O_r>
//     (O_r = slot_r / g, the expert's unscaled output; the slot holds g * O_r)
//   per token: ds over I_t through g_k = s_k / max(S, 1e-12) ("Sparse
//     Mixture-of-Experts ...", section 2: gates from s alone, so the bias has
//     no gradient), then dz through sigmoid s(1 - s) or softmax;
//   dh_t = add_residual dy_t + sum_j dX^S_j,t + sum_{k kept} dX_{row(t,k)} + sum_i dz_{t,i} e_i
//   de_i = sum_t dz_{t,i} h_t
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

__device__ __forceinline__ void unpack8(uint4 q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One warp per permuted row: dO = g * dy (bf16) and dL/dg = <dy, slot> / g.
__global__ void __launch_bounds__(256)
bwd_rows_kernel(const uint16_t* __restrict__ dy, const int32_t* __restrict__ perm_tok,
                const float* __restrict__ row_gate, const uint16_t* __restrict__ slot,
                const int* __restrict__ n_rows_ptr, int max_rows, int T, int d,
                uint16_t* __restrict__ dO, float* __restrict__ dg_row, int* err) {
  const int lane = threadIdx.x % kWarp;
  const int wpb = blockDim.x / kWarp;
  const int n = min(*n_rows_ptr, max_rows);
  for (int r = blockIdx.x * wpb + threadIdx.x / kWarp; r < n; r += gridDim.x * wpb) {
    const int t = perm_tok[r];
    if (t < 0 || t >= T) {
      if (lane == 0) { set_device_error(err, MOE_DEVERR_INDEX); dg_row[r] = 0.0f; }
      continue;
    }
    const float g = row_gate[r];
    const uint16_t* dyr = dy + (size_t)t * d;
    const uint16_t* sr = slot + (size_t)r * d;
    uint16_t* out = dO + (size_t)r * d;
    float acc = 0.0f;
    for (int c = lane * 8; c < d; c += kWarp * 8) {
      float a[8], b[8];
      unpack8(*reinterpret_cast<const uint4*>(dyr + c), a);
      unpack8(*reinterpret_cast<const uint4*>(sr + c), b);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fmaf(a[i], b[i], acc);
      *reinterpret_cast<uint4*>(out + c) = make_uint4(pack2(g * a[0], g * a[1]), pack2(g * a[2], g * a[3]),
                                                       pack2(g * a[4], g * a[5]), pack2(g * a[6], g * a[7]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
    if (lane == 0) dg_row[r] = g != 0.0f ? acc / g : 0.0f;
  }
}

// One warp per token: dz [T, E] from dL/dg of the K slots (0 for dropped ones).
__global__ void __launch_bounds__(256)
bwd_gate_kernel(const float* __restrict__ s, const int32_t* __restrict__ idx,
                const int32_t* __restrict__ row_of, const float* __restrict__ dg_row, int score_fn,
                int T, int E, int K, float* __restrict__ dz) {
  const int lane = threadIdx.x % kWarp;
  const int t = blockIdx.x * (blockDim.x / kWarp) + threadIdx.x / kWarp;
  if (t >= T) return;
  const float* sr = s + (size_t)t * E;
  // every lane walks the K slots in order (same sums in every lane)
  float S = 0.0f;
  for (int k = 0; k < K; ++k) S += sr[idx[(size_t)t * K + k]];
  const float den = fmaxf(S, 1e-12f);
  float corr = 0.0f;
  if (S > 1e-12f) {
    for (int k = 0; k < K; ++k) {
      const int ro = row_of[(size_t)t * K + k];
      const float dg = ro >= 0 ? dg_row[ro] : 0.0f;
      corr += (sr[idx[(size_t)t * K + k]] / den) * dg;
    }
  }
  // ds of slot k, held by lane k
  float dsk = 0.0f, sk = 0.0f;
  int jk = -1;
  if (lane < K) {
    const int ro = row_of[(size_t)t * K + lane];
    const float dg = ro >= 0 ? dg_row[ro] : 0.0f;
    jk = idx[(size_t)t * K + lane];
    sk = sr[jk];
    dsk = (dg - corr) / den;
  }
  float* zr = dz + (size_t)t * E;
  if (score_fn == 0) {
    for (int j = lane; j < E; j += kWarp) zr[j] = 0.0f;
    __syncwarp();
    if (lane < K) zr[jk] = dsk * sk * (1.0f - sk);
  } else {
    // softmax: dz_j = p_j (ds_j - sum_k ds_k p_{I_k})
    float dot = 0.0f;
    for (int k = 0; k < K; ++k) {
      const float dk = __shfl_sync(kFull, dsk, k);
      const float pk = __shfl_sync(kFull, sk, k);
      dot += dk * pk;
    }
    // unselected j: ds_j = 0; the K selected entries are rewritten after
    for (int j = lane; j < E; j += kWarp) zr[j] = sr[j] * (0.0f - dot);
    __syncwarp();
    if (lane < K) zr[jk] = sk * (dsk - dot);
  }
}

// One block per token: dh = a dy + sum_j dX^S_j + sum_{k kept} dX_row + sum_i dz_i e_i.
__global__ void __launch_bounds__(256)
bwd_dh_kernel(const uint16_t* __restrict__ dy, const uint16_t* __restrict__ dx_r,
              const uint16_t* __restrict__ dx_s, const int32_t* __restrict__ row_of,
              const float* __restrict__ dz, const float* __restrict__ e, const int32_t* __restrict__ idx,
              int T, int d, int K, int E, int E_s, int add_residual, int n_rows, int sparse,
              uint16_t* __restrict__ dh) {
  const int t = blockIdx.x;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    float acc[8], v[8];
    unpack8(*reinterpret_cast<const uint4*>(dy + (size_t)t * d + c), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = add_residual ? v[i] : 0.0f;
    for (int j = 0; j < E_s; ++j) {
      unpack8(*reinterpret_cast<const uint4*>(dx_s + ((size_t)j * T + t) * d + c), v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
    }
    for (int k = 0; k < K; ++k) {
      const int ro = row_of[(size_t)t * K + k];
      if (ro < 0 || ro >= n_rows) continue;
      unpack8(*reinterpret_cast<const uint4*>(dx_r + (size_t)ro * d + c), v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
    }
    // router term: sigmoid routing has dz != 0 only on the K selected experts
    // (ascending, as idx stores them); softmax touches every expert
    const float* zr = dz + (size_t)t * E;
    const int nj = sparse ? K : E;
    for (int q = 0; q < nj; ++q) {
      const int j = sparse ? idx[(size_t)t * K + q] : q;
      const float z = zr[j];
      if (z == 0.0f) continue;
      const float4 e0 = *reinterpret_cast<const float4*>(e + (size_t)j * d + c);
      const float4 e1 = *reinterpret_cast<const float4*>(e + (size_t)j * d + c + 4);
      acc[0] = fmaf(z, e0.x, acc[0]); acc[1] = fmaf(z, e0.y, acc[1]);
      acc[2] = fmaf(z, e0.z, acc[2]); acc[3] = fmaf(z, e0.w, acc[3]);
      acc[4] = fmaf(z, e1.x, acc[4]); acc[5] = fmaf(z, e1.y, acc[5]);
      acc[6] = fmaf(z, e1.z, acc[6]); acc[7] = fmaf(z, e1.w, acc[7]);
    }
    *reinterpret_cast<uint4*>(dh + (size_t)t * d + c) =
        make_uint4(pack2(acc[0], acc[1]), pack2(acc[2], acc[3]), pack2(acc[4], acc[5]), pack2(acc[6], acc[7]));
  }
}

// de [E, d] = dz^T h: one block per (expert, 256 columns), tokens in order.
__global__ void __launch_bounds__(256)
bwd_de_kernel(const float* __restrict__ dz, const uint16_t* __restrict__ h, int T, int d, int E,
              float* __restrict__ de) {
  const int j = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  float acc = 0.0f;
  for (int t = 0; t < T; ++t) {
    const float z = __ldg(dz + (size_t)t * E + j);
    if (z == 0.0f) continue;
    if (c < d) acc = fmaf(z, __uint_as_float((uint32_t)h[(size_t)t * d + c] << 16), acc);
  }
  if (c < d) de[(size_t)j * d + c] = acc;
}

// de for sigmoid routing: dz is non-zero only on the selected pairs; the
// pairs of expert j (every selected (t, j), dropped ones included) are rows
// sel_off[j] .. sel_off[j+1] of sel_tok, in ascending token order.
__global__ void __launch_bounds__(256)
bwd_de_sparse_kernel(const float* __restrict__ dz, const uint16_t* __restrict__ h,
                     const int32_t* __restrict__ sel_tok, const int* __restrict__ sel_off, int T, int d,
                     int E, float* __restrict__ de) {
  const int j = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  float acc = 0.0f;
  const int r0 = sel_off[j], r1 = sel_off[j + 1];
  for (int r = r0; r < r1; ++r) {
    const int t = sel_tok[r];
    if (t < 0 || t >= T) continue;
    const float z = __ldg(dz + (size_t)t * E + j);
    if (c < d) acc = fmaf(z, __uint_as_float((uint32_t)h[(size_t)t * d + c] << 16), acc);
  }
  if (c < d) de[(size_t)j * d + c] = acc;
}

// Zero rows n .. n+63 (n = *n_rows_ptr, capped at max_rows) of a bf16 [max_rows, cols]
// buffer: the weight-gradient GEMMs read up to 63 lines past an expert's last
// row as operand B, which must be finite there.
__global__ void zero_tail_rows_kernel(uint16_t* __restrict__ buf, const int* __restrict__ n_rows_ptr,
                                      int max_rows, int cols) {
  const int n = min(*n_rows_ptr, max_rows);
  const int rows = min(64, max_rows - n);
  const size_t total = (size_t)rows * cols / 8;
  uint4* p = reinterpret_cast<uint4*>(buf + (size_t)n * cols);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x)
    p[i] = make_uint4(0, 0, 0, 0);
}

}  // namespace

void launch_zero_tail_rows(void* buf, const int* n_rows_ptr, int max_rows, int cols, cudaStream_t st) {
  zero_tail_rows_kernel<<<64, 256, 0, st>>>(static_cast<uint16_t*>(buf), n_rows_ptr, max_rows, cols);
}

void launch_bwd_route(const BwdRouteArgs& a, cudaStream_t st) {
  const int warps = a.max_rows < 148 * 64 ? (a.max_rows > 0 ? a.max_rows : 1) : 148 * 64;
  bwd_rows_kernel<<<(warps * kWarp + 255) / 256, 256, 0, st>>>(
      a.dy, a.perm_tok, a.row_gate, a.slot, a.n_rows_ptr, a.max_rows, a.T, a.d, a.dO, a.dg_row, a.err);
}

void launch_bwd_gate_dh_de(const BwdRouteArgs& a, cudaStream_t st) {
  bwd_gate_kernel<<<(a.T + 7) / 8, 256, 0, st>>>(a.s, a.idx, a.row_of, a.dg_row, a.score_fn, a.T, a.E, a.K, a.dz);
  const int sparse = a.score_fn == 0;
  bwd_dh_kernel<<<a.T, 256, 0, st>>>(a.dy, a.dx_r, a.dx_s, a.row_of, a.dz, a.e, a.idx, a.T, a.d, a.K, a.E,
                                     a.E_s, a.add_residual, a.max_rows, sparse, a.dh);
  if (sparse)
    bwd_de_sparse_kernel<<<dim3(a.E, (a.d + 255) / 256), 256, 0, st>>>(a.dz, a.h, a.sel_tok, a.sel_off, a.T,
                                                                       a.d, a.E, a.de);
  else
    bwd_de_kernel<<<dim3(a.E, (a.d + 255) / 256), 256, 0, st>>>(a.dz, a.h, a.T, a.d, a.E, a.de);
}

}  // namespace moe
