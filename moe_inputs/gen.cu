// Counter-based synthetic-input generator: the CUDA and multithreaded-host twin
// of moe_inputs/__init__.py (same draws, bit for bit).  It holds no arithmetic
// of the MoE method: only SplitMix64 draws turned into normal / uniform
// variates and rounded to fp32 or bf16.
//
//   draw n of stream (seed, tensor_id):  mix(key + (n + 1) * GOLDEN)
//   key = mix(mix(seed) + tensor_id * GOLDEN)
//   normal: (sum of the four 16-bit fields - 131070) * scale   (one double multiply)
//   uniform: lo + width * (draw >> 11) * 2^-53                  (double, unfused)
//   double -> float RN, float -> bf16 RN-even by bit arithmetic.
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

__host__ __device__ inline float draw_value(uint64_t key, int64_t n, int kind, double p0, double p1) {
  uint64_t r = mix64(key + (uint64_t)(n + 1) * kGolden);
  double v;
  if (kind == 0) {
    int64_t s = (int64_t)(r & 0xFFFF) + (int64_t)((r >> 16) & 0xFFFF) +
                (int64_t)((r >> 32) & 0xFFFF) + (int64_t)(r >> 48);
    v = mul_rn((double)(s - 131070), p0);
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

// kind: 0 = normal (p0 = scale = sigma*sqrt(3)/65536), 1 = uniform (p0 = lo, p1 = hi - lo)
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
