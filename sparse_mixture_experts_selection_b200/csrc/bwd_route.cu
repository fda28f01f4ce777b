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

// eight fp16 values of a 16-byte vector (the layer's slot rows)
__device__ __forceinline__ void unpack8_f16(uint4 q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

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

// One warp per permuted row: dO = g * dy (bf16) and dL/dg = <dy, slot> / g
// (slot rows in fp16 when SLOT_F16, the layer's own, else bf16).
template <bool SLOT_F16>
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
    // four 16-byte vectors of dy and of the slot in flight per lane; the
    // products are accumulated in column order
    constexpr int U = 4;
    for (int c0 = lane * 8; c0 < d; c0 += U * kWarp * 8) {
      uint4 qa[U], qb[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * kWarp * 8;
        qa[u] = c < d ? __ldg(reinterpret_cast<const uint4*>(dyr + c)) : make_uint4(0, 0, 0, 0);
        qb[u] = c < d ? __ldg(reinterpret_cast<const uint4*>(sr + c)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * kWarp * 8;
        if (c >= d) break;
        float a[8], b[8];
        unpack8(qa[u], a);
        if (SLOT_F16) unpack8_f16(qb[u], b); else unpack8(qb[u], b);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = fmaf(a[i], b[i], acc);
        *reinterpret_cast<uint4*>(out + c) = make_uint4(pack2(g * a[0], g * a[1]), pack2(g * a[2], g * a[3]),
                                                         pack2(g * a[4], g * a[5]), pack2(g * a[6], g * a[7]));
      }
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

// dh = a dy + sum_j dX^S_j + sum_{k kept} dX_row + sum_i dz_i e_i: block
// (t, y) covers 8-column vectors y*128 + tid, += 128 * gridDim.y of token t.
// The K routed rows are loaded KC at a time before they are added, so their
// loads are in flight together; the sums keep the order above.
constexpr int kDhChunk = 8;
__global__ void __launch_bounds__(128)
bwd_dh_kernel(const uint16_t* __restrict__ dy, const uint16_t* __restrict__ dx_r,
              const uint16_t* __restrict__ dx_s, const int32_t* __restrict__ row_of,
              const float* __restrict__ dz, const float* __restrict__ e, const int32_t* __restrict__ idx,
              int T, int d, int K, int E, int E_s, int add_residual, int n_rows, int sparse,
              uint16_t* __restrict__ dh) {
  const int t = blockIdx.x;
  const int nvec = d / 8;
  for (int v0 = blockIdx.y * blockDim.x + threadIdx.x; v0 < nvec; v0 += blockDim.x * gridDim.y) {
    const int c = v0 * 8;
    float acc[8], v[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(dy + (size_t)t * d + c)), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = add_residual ? v[i] : 0.0f;
    for (int j = 0; j < E_s; ++j) {
      unpack8(__ldg(reinterpret_cast<const uint4*>(dx_s + ((size_t)j * T + t) * d + c)), v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
    }
    for (int k0 = 0; k0 < K; k0 += kDhChunk) {
      uint4 xr[kDhChunk];
      bool ok[kDhChunk];
#pragma unroll
      for (int q = 0; q < kDhChunk; ++q) {
        const int ro = k0 + q < K ? __ldg(row_of + (size_t)t * K + k0 + q) : -1;
        ok[q] = ro >= 0 && ro < n_rows;
        xr[q] = ok[q] ? __ldg(reinterpret_cast<const uint4*>(dx_r + (size_t)ro * d + c)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < kDhChunk; ++q) {
        if (!ok[q]) continue;
        unpack8(xr[q], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += v[i];
      }
    }
    // router term: sigmoid routing has dz != 0 only on the K selected experts
    // (ascending, as idx stores them); softmax touches every expert
    const float* zr = dz + (size_t)t * E;
    const int nj = sparse ? K : E;
    for (int q = 0; q < nj; ++q) {
      const int j = sparse ? __ldg(idx + (size_t)t * K + q) : q;
      const float z = __ldg(zr + j);
      if (z == 0.0f) continue;
      const float4 e0 = __ldg(reinterpret_cast<const float4*>(e + (size_t)j * d + c));
      const float4 e1 = __ldg(reinterpret_cast<const float4*>(e + (size_t)j * d + c + 4));
      acc[0] = fmaf(z, e0.x, acc[0]); acc[1] = fmaf(z, e0.y, acc[1]);
      acc[2] = fmaf(z, e0.z, acc[2]); acc[3] = fmaf(z, e0.w, acc[3]);
      acc[4] = fmaf(z, e1.x, acc[4]); acc[5] = fmaf(z, e1.y, acc[5]);
      acc[6] = fmaf(z, e1.z, acc[6]); acc[7] = fmaf(z, e1.w, acc[7]);
    }
    *reinterpret_cast<uint4*>(dh + (size_t)t * d + c) =
        make_uint4(pack2(acc[0], acc[1]), pack2(acc[2], acc[3]), pack2(acc[4], acc[5]), pack2(acc[6], acc[7]));
  }
}

// de [E, d] = dz^T h, tokens in ascending order: block (j, y) covers 8-column
// vectors y*128 + tid of expert j.  SPARSE (sigmoid routing): dz is non-zero
// only on the selected pairs, and the pairs of expert j (every selected
// (t, j), dropped ones included) are rows sel_off[j] .. sel_off[j+1] of
// sel_tok in ascending token order; otherwise every token.  Four tokens'
// rows are loaded before they are accumulated (in order).
constexpr int kDeUnroll = 4;
template <bool SPARSE>
__global__ void __launch_bounds__(128)
bwd_de_kernel(const float* __restrict__ dz, const uint16_t* __restrict__ h, const int32_t* __restrict__ sel_tok,
              const int* __restrict__ sel_off, int T, int d, int E, float* __restrict__ de) {
  const int j = blockIdx.x;
  const int vi = blockIdx.y * blockDim.x + threadIdx.x;
  if (vi >= d / 8) return;
  const int c = vi * 8;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  const int r0 = SPARSE ? __ldg(sel_off + j) : 0;
  const int r1 = SPARSE ? __ldg(sel_off + j + 1) : T;
  for (int r = r0; r < r1; r += kDeUnroll) {
    float z[kDeUnroll];
    uint4 hv[kDeUnroll];
#pragma unroll
    for (int u = 0; u < kDeUnroll; ++u) {
      int t = r + u < r1 ? (SPARSE ? __ldg(sel_tok + r + u) : r + u) : -1;
      if (t >= T) t = -1;
      z[u] = t >= 0 ? __ldg(dz + (size_t)t * E + j) : 0.0f;
      hv[u] = (t >= 0 && z[u] != 0.0f) ? __ldg(reinterpret_cast<const uint4*>(h + (size_t)t * d + c))
                                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kDeUnroll; ++u) {
      if (z[u] == 0.0f) continue;
      float v[8];
      unpack8(hv[u], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(z[u], v[i], acc[i]);
    }
  }
  float4* out = reinterpret_cast<float4*>(de + (size_t)j * d + c);
  out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
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
  auto kern = a.slot_f16 ? bwd_rows_kernel<true> : bwd_rows_kernel<false>;
  kern<<<(warps * kWarp + 255) / 256, 256, 0, st>>>(
      a.dy, a.perm_tok, a.row_gate, a.slot, a.n_rows_ptr, a.max_rows, a.T, a.d, a.dO, a.dg_row, a.err);
}

void launch_bwd_gate_dh_de(const BwdRouteArgs& a, cudaStream_t st) {
  bwd_gate_kernel<<<(a.T + 7) / 8, 256, 0, st>>>(a.s, a.idx, a.row_of, a.dg_row, a.score_fn, a.T, a.E, a.K, a.dz);
  const int sparse = a.score_fn == 0;
  const int nvec = a.d / 8;
  int split = (2 * 148 + a.T - 1) / a.T;                // fill the GPU for short batches
  const int max_split = (nvec + 127) / 128;
  split = split < 1 ? 1 : (split > max_split ? max_split : split);
  bwd_dh_kernel<<<dim3(a.T, split), 128, 0, st>>>(a.dy, a.dx_r, a.dx_s, a.row_of, a.dz, a.e, a.idx, a.T, a.d, a.K,
                                                 a.E, a.E_s, a.add_residual, a.max_rows, sparse, a.dh);
  const dim3 g_de(a.E, (nvec + 127) / 128);
  if (sparse)
    bwd_de_kernel<true><<<g_de, 128, 0, st>>>(a.dz, a.h, a.sel_tok, a.sel_off, a.T, a.d, a.E, a.de);
  else
    bwd_de_kernel<false><<<g_de, 128, 0, st>>>(a.dz, a.h, nullptr, nullptr, a.T, a.d, a.E, a.de);
}

}  // namespace moe
