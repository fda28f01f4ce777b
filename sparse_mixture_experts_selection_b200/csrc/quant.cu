// e4m3 quantization of matrix rows (low-precision expert weights, and the rows
// entering the e4m3 GEMMs): one power-of-two scale per row, the smallest s with
// amax / s <= 448, then each element x / s rounded to the nearest e4m3 value
// (ties to the even code, saturating at 448).  Dividing by a power of two is
// exact, so the codes depend only on the row's values -- no division rounding
// and no dependence on how amax was reduced.
//
// "GPUs, memory and failures" (serving notes) suggests lower-precision expert
// weights when serving is bound by streaming them; the pages fix no format,
// so the per-row power-of-two e4m3 layout is this library's reading.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// e with 2^e the smallest power of two such that amax <= 448 * 2^e, i.e. with
// amax = M * 2^E (1 <= M < 2): e = E - 8 + [M > 1.75]; at least -126 (a normal
// fp32 scale); 0 for amax == 0.
__device__ __forceinline__ int pow2_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax) & 0x7FFFFFFFu;
  if (b == 0) return 0;
  int E;
  uint32_t mant;
  if ((b >> 23) == 0) {                        // subnormal amax
    const int p = 31 - __clz(b);
    E = p - 149;
    mant = (b << (23 - p)) & 0x7FFFFFu;
  } else {
    E = (int)(b >> 23) - 127;
    mant = b & 0x7FFFFFu;
  }
  const int e = E - 8 + (mant > 0x600000u ? 1 : 0);
  return e < -126 ? -126 : e;
}

// Eight (bf16) or four (fp32) elements of one 16-byte load.
__device__ __forceinline__ void load16(const uint16_t* p, float* v) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load16(const float* p, float* v) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}

template <typename TIn>
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const TIn* __restrict__ src, const int32_t* __restrict__ src_row, int n_src,
                     const int* __restrict__ n_rows_ptr, int64_t n_rows, int cols,
                     uint8_t* __restrict__ codes, float* __restrict__ scales, int* err) {
  constexpr int V = 16 / sizeof(TIn);          // elements per 16-byte load
  const int lane = threadIdx.x % kWarp;
  const int64_t wpb = blockDim.x / kWarp;
  int64_t n = n_rows;
  if (n_rows_ptr) {
    const int64_t m = *n_rows_ptr;
    if (m < n) n = m;
  }
  for (int64_t r = blockIdx.x * wpb + threadIdx.x / kWarp; r < n; r += (int64_t)gridDim.x * wpb) {
    int64_t sr = r;
    if (src_row) {
      const int t = src_row[r];
      if (t < 0 || t >= n_src) {               // corrupt permutation: report, write zeros
        if (lane == 0) { if (err) set_device_error(err, MOE_DEVERR_INDEX); scales[r] = 1.0f; }
        for (int c = lane * 16; c < cols; c += kWarp * 16)
          *reinterpret_cast<uint4*>(codes + r * cols + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      sr = t;
    }
    const TIn* row = src + sr * cols;
    float amax = 0.0f;
    for (int c = lane * V; c < cols; c += kWarp * V) {
      float v[V];
      load16(row + c, v);
#pragma unroll
      for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
    const int e = pow2_exponent(amax);
    const float inv = __uint_as_float((uint32_t)(127 - e) << 23);      // 2^-e, exact
    uint8_t* out = codes + r * cols;
    for (int c = lane * 16; c < cols; c += kWarp * 16) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; j += V) load16(row + c + j, v + j);
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * inv, v[4 * i + 1] * inv),
                                                     __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * inv, v[4 * i + 3] * inv),
                                                     __NV_SATFINITE, __NV_E4M3);
        w[i] = (lo & 0xFFFFu) | (hi << 16);
      }
      *reinterpret_cast<uint4*>(out + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (lane == 0) scales[r] = __uint_as_float((uint32_t)(e + 127) << 23);   // 2^e
  }
}

}  // namespace

void launch_quantize_rows(const void* src, int src_dtype, const int32_t* src_row, int n_src,
                          const int* n_rows_ptr, int64_t n_rows, int cols, uint8_t* codes,
                          float* scales, int* err, cudaStream_t st) {
  if (n_rows <= 0) return;
  const int64_t warps = n_rows < 148 * 64 ? n_rows : 148 * 64;
  const unsigned blocks = (unsigned)((warps * kWarp + 255) / 256);
  if (src_dtype == 1)
    quantize_rows_kernel<uint16_t><<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(src), src_row,
                                                           n_src, n_rows_ptr, n_rows, cols, codes, scales, err);
  else
    quantize_rows_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(src), src_row, n_src,
                                                        n_rows_ptr, n_rows, cols, codes, scales, err);
}

}  // namespace moe
