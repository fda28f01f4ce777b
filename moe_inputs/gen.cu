// Counter-based synthetic-input generator: the CUDA and multithreaded-host twin
// of moe_inputs/__init__.py (same draws, bit for bit).  It holds no arithmetic
// of the MoE method: only SplitMix64 draws turned into normal / uniform
// variates and rounded to fp32 or bf16.
//
//   draw n of stream (seed, tensor_id):  mix(key + (n + 1) * GOLDEN)
//   key = mix(mix(seed) + tensor_id * GOLDEN)
//   normal: Box-Muller of the draw's two 32-bit halves,
//           sqrt(-2 ln((hi + 1/2) 2^-32)) cos(2 pi lo 2^-32) * sigma, with ln
//           and cos evaluated by the same fixed series, in the same order of
//           individually rounded double operations, as moe_inputs/__init__.py
//   uniform: lo + width * (draw >> 11) * 2^-53                  (double, unfused)
//   double -> float RN, float -> bf16 RN-even by bit arithmetic.
// The host path is compiled with -ffp-contract=off and the device path calls
// the round-to-nearest intrinsics, so no multiply-add is fused on either side.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t x) {
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

__host__ __device__ inline uint16_t f32_to_bf16_bits(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  b = (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
  return (uint16_t)b;
}

__host__ __device__ inline double mul_rn(double a, double b) {
#ifdef __CUDA_ARCH__
  return __dmul_rn(a, b);
#else
  return a * b;
#endif
}

__host__ __device__ inline double add_rn(double a, double b) {
#ifdef __CUDA_ARCH__
  return __dadd_rn(a, b);
#else
  return a + b;
#endif
}

__host__ __device__ inline double div_rn(double a, double b) {
#ifdef __CUDA_ARCH__
  return __ddiv_rn(a, b);
#else
  return a / b;
#endif
}

__host__ __device__ inline double sqrt_rn(double a) {
#ifdef __CUDA_ARCH__
  return __dsqrt_rn(a);
#else
  return std::sqrt(a);
#endif
}

// one Horner step: p * w + c with the multiply and the add rounded separately
__host__ __device__ inline double hstep(double p, double w, double c) { return add_rn(mul_rn(p, w), c); }

// ln(hi + 1/2) - 32 ln 2: hi + 1/2 = m 2^e exactly, m in [sqrt(1/2), sqrt(2)),
// ln m = 2 s (1 + s^2/3 + ... + s^20/21), s = (m - 1)/(m + 1)
__host__ __device__ inline double ln_half_int(uint32_t hi) {
  int e;
  double m = frexp((double)hi + 0.5, &e);
  if (m < 0x1.6a09e667f3bcdp-1) {
    m = mul_rn(m, 2.0);
    e -= 1;
  }
  const double s = div_rn(add_rn(m, -1.0), add_rn(m, 1.0));
  const double z = mul_rn(s, s);
  double p = 0x1.8618618618618p-5;
  p = hstep(p, z, 0x1.af286bca1af28p-5);
  p = hstep(p, z, 0x1.e1e1e1e1e1e1ep-5);
  p = hstep(p, z, 0x1.1111111111111p-4);
  p = hstep(p, z, 0x1.3b13b13b13b14p-4);
  p = hstep(p, z, 0x1.745d1745d1746p-4);
  p = hstep(p, z, 0x1.c71c71c71c71cp-4);
  p = hstep(p, z, 0x1.2492492492492p-3);
  p = hstep(p, z, 0x1.999999999999ap-3);
  p = hstep(p, z, 0x1.5555555555555p-2);
  p = hstep(p, z, 0x1.0000000000000p+0);
  return add_rn(mul_rn(mul_rn(s, 2.0), p), mul_rn((double)(e - 32), 0x1.62e42fefa39efp-1));
}

// cos(2 pi lo 2^-32): quadrant q and angle f pi / 2^31 within it from the
// integer, folded into [0, pi/4]; Taylor series of cos and sin there
__host__ __device__ inline double cos_2pi_frac(uint32_t lo) {
  const uint32_t q = lo >> 30;
  const uint32_t f = lo & ((1u << 30) - 1u);
  const bool fold = f >= (1u << 29);
  const uint32_t g = fold ? (1u << 30) - f : f;
  const double th = mul_rn((double)g, 0x1.921fb54442d18p-30);
  const double w = mul_rn(th, th);
  double c = 0x1.e542ba4020225p-62;
  c = hstep(c, w, -0x1.6827863b97d97p-53);
  c = hstep(c, w, 0x1.ae7f3e733b81fp-45);
  c = hstep(c, w, -0x1.93974a8c07c9dp-37);
  c = hstep(c, w, 0x1.1eed8eff8d898p-29);
  c = hstep(c, w, -0x1.27e4fb7789f5cp-22);
  c = hstep(c, w, 0x1.a01a01a01a01ap-16);
  c = hstep(c, w, -0x1.6c16c16c16c17p-10);
  c = hstep(c, w, 0x1.5555555555555p-5);
  c = hstep(c, w, -0x1.0000000000000p-1);
  c = hstep(c, w, 0x1.0000000000000p+0);
  double sp = 0x1.71b8ef6dcf572p-66;
  sp = hstep(sp, w, -0x1.2f49b46814157p-57);
  sp = hstep(sp, w, 0x1.952c77030ad4ap-49);
  sp = hstep(sp, w, -0x1.ae7f3e733b81fp-41);
  sp = hstep(sp, w, 0x1.6124613a86d09p-33);
  sp = hstep(sp, w, -0x1.ae64567f544e4p-26);
  sp = hstep(sp, w, 0x1.71de3a556c734p-19);
  sp = hstep(sp, w, -0x1.a01a01a01a01ap-13);
  sp = hstep(sp, w, 0x1.1111111111111p-7);
  sp = hstep(sp, w, -0x1.5555555555555p-3);
  sp = hstep(sp, w, 0x1.0000000000000p+0);
  const double sn = mul_rn(th, sp);
  const double ca = fold ? sn : c, sa = fold ? c : sn;
  return q == 0 ? ca : q == 1 ? -sa : q == 2 ? -ca : sa;
}

__host__ __device__ inline float draw_value(uint64_t key, int64_t n, int kind, double p0, double p1) {
  uint64_t r = mix64(key + (uint64_t)(n + 1) * kGolden);
  double v;
  if (kind == 0) {
    const double rad = sqrt_rn(mul_rn(ln_half_int((uint32_t)(r >> 32)), -2.0));
    v = mul_rn(mul_rn(rad, cos_2pi_frac((uint32_t)(r & 0xFFFFFFFFu))), p0);
  } else {
    double u = mul_rn((double)(r >> 11), 0x1p-53);
    v = add_rn(p0, mul_rn(p1, u));
  }
  return (float)v;   // round to nearest
}

__global__ void fill_kernel(void* out, int64_t count, int dtype, int kind, uint64_t key,
                            int64_t start, double p0, double p1) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    float v = draw_value(key, start + i, kind, p0, p1);
    if (dtype == 1)
      reinterpret_cast<uint16_t*>(out)[i] = f32_to_bf16_bits(v);
    else
      reinterpret_cast<float*>(out)[i] = v;
  }
}

}  // namespace

extern "C" {

uint64_t moe_gen_stream_key(uint64_t seed, uint64_t tensor_id) {
  return mix64(mix64(seed) + tensor_id * kGolden);
}

// kind: 0 = normal (p0 = sigma), 1 = uniform (p0 = lo, p1 = hi - lo)
// dtype: 0 = float32, 1 = bf16.  Returns 0 or a cudaError_t.
int moe_gen_fill_device(void* out, int64_t count, int dtype, int kind, uint64_t seed,
                        uint64_t tensor_id, int64_t start, double p0, double p1,
                        cudaStream_t stream) {
  if (count <= 0) return 0;
  uint64_t key = moe_gen_stream_key(seed, tensor_id);
  int64_t blocks = (count + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  fill_kernel<<<(unsigned)blocks, 256, 0, stream>>>(out, count, dtype, kind, key, start, p0, p1);
  return (int)cudaGetLastError();
}

void moe_gen_fill_host(void* out, int64_t count, int dtype, int kind, uint64_t seed,
                       uint64_t tensor_id, int64_t start, double p0, double p1, int threads) {
  if (count <= 0) return;
  uint64_t key = moe_gen_stream_key(seed, tensor_id);
  if (threads < 1) threads = 1;
  auto work = [=](int64_t a, int64_t b) {
    for (int64_t i = a; i < b; ++i) {
      float v = draw_value(key, start + i, kind, p0, p1);
      if (dtype == 1)
        reinterpret_cast<uint16_t*>(out)[i] = f32_to_bf16_bits(v);
      else
        reinterpret_cast<float*>(out)[i] = v;
    }
  };
  std::vector<std::thread> pool;
  int64_t per = (count + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    int64_t a = t * per, b = a + per < count ? a + per : count;
    if (a < b) pool.emplace_back(work, a, b);
  }
  for (auto& th : pool) th.join();
}

}  // extern "C"
