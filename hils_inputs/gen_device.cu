// Device copy of the seeded input generator defined in hils_inputs/__init__.py
// (splitmix64 counter stream -> Box-Muller in float64 -> float32 RNE -> bf16 RNE).
// It holds no arithmetic of the attention method; it only fills input tensors.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t sm64(uint64_t z) {
  z += kGolden;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t b = __float_as_uint(f);
  uint32_t lsb = (b >> 16) & 1u;
  return (uint16_t)((b + 0x7FFFu + lsb) >> 16);
}

__global__ void gen_normal_kernel(uint64_t key, uint64_t start, uint64_t n, double stdv,
                                  int dtype, void* out) {
  const double two_pi = 6.283185307179586;
  for (uint64_t t = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; t < n;
       t += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t i = start + t;
    uint64_t a = sm64(key + (2 * i) * kGolden);
    uint64_t b = sm64(key + (2 * i + 1) * kGolden);
    double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53;
    double u2 = (double)(b >> 11) * 0x1.0p-53;
    double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
    float v = (float)(z * stdv);
    if (dtype == 0) {
      ((float*)out)[t] = v;
    } else {
      ((uint16_t*)out)[t] = f32_to_bf16_rne(v);
    }
  }
}

}  // namespace

extern "C" int hils_gen_normal(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n,
                               double stdv, int dtype, void* out, void* stream) {
  if (n == 0) return 0;
  uint64_t key = sm64(sm64(seed) ^ tid);
  int threads = 256;
  uint64_t blocks = (n + threads - 1) / threads;
  if (blocks > 148ull * 64) blocks = 148ull * 64;
  gen_normal_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(key, start, n, stdv,
                                                                            dtype, out);
  return (int)cudaGetLastError();
}
