// Seeded synthetic input generator: host (OpenMP) and device (CUDA) versions of
// the counter-based definition documented in qwen3_synth/__init__.py.
// It holds none of the decoder block's arithmetic; it only draws inputs.
#include <cstdint>
#include <cmath>
#include <cstring>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t word(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * kGamma); }

inline uint64_t stream_key(uint64_t seed, uint64_t tid) { return mix64(mix64(seed) + tid * kGamma); }

__host__ __device__ inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  uint64_t r = ((uint64_t)u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return (uint16_t)r;
}

__host__ __device__ inline uint16_t normal_bits(uint64_t key, uint64_t i, double mean, double sd) {
  const double two_m53 = 1.1102230246251565404e-16;  // 2^-53
  double u1 = (double)((word(key, 2 * i) >> 11) + 1) * two_m53;
  double u2 = (double)(word(key, 2 * i + 1) >> 11) * two_m53;
  const double two_pi = 6.283185307179586476925286766559;
#ifdef __CUDA_ARCH__
  double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
  float v = __double2float_rn(mean + sd * z);
#else
  double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
  float v = (float)(mean + sd * z);
#endif
  return f32_to_bf16_rne(v);
}

__host__ __device__ inline int32_t uniform_int(uint64_t key, uint64_t i, uint64_t upper) {
  uint64_t w = word(key, i);
  uint64_t t = (w >> 32) * upper + (((w & 0xFFFFFFFFull) * upper) >> 32);
  return (int32_t)(t >> 32);
}

__global__ void normal_kernel(uint16_t* dst, int64_t n0, int64_t n1, int64_t n2, int64_t s0, int64_t s1,
                              int64_t base, uint64_t key, double mean, double sd) {
  const int64_t total = n0 * n1 * n2;
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < total;
       j += (int64_t)gridDim.x * blockDim.x) {
    int64_t i2 = j % n2, r = j / n2, i1 = r % n1, i0 = r / n1;
    dst[i0 * s0 + i1 * s1 + i2] = normal_bits(key, (uint64_t)(base + j), mean, sd);
  }
}

__global__ void uniform_int_kernel(int32_t* dst, int64_t n, int64_t base, uint64_t key, uint64_t upper) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n; j += (int64_t)gridDim.x * blockDim.x)
    dst[j] = uniform_int(key, (uint64_t)(base + j), upper);
}

}  // namespace

extern "C" {

int qwen3synth_normal_bf16_host(uint16_t* dst, int64_t n0, int64_t n1, int64_t n2, int64_t s0, int64_t s1,
                                int64_t base, uint64_t seed, uint64_t tid, double mean, double sd) {
  if (!dst || n0 < 0 || n1 < 0 || n2 < 0) return -1;
  const uint64_t key = stream_key(seed, tid);
  const int64_t total = n0 * n1 * n2;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < total; ++j) {
    int64_t i2 = j % n2, r = j / n2, i1 = r % n1, i0 = r / n1;
    dst[i0 * s0 + i1 * s1 + i2] = normal_bits(key, (uint64_t)(base + j), mean, sd);
  }
  return 0;
}

int qwen3synth_normal_bf16_device(uint16_t* dst, int64_t n0, int64_t n1, int64_t n2, int64_t s0, int64_t s1,
                                  int64_t base, uint64_t seed, uint64_t tid, double mean, double sd,
                                  void* stream) {
  if (!dst || n0 < 0 || n1 < 0 || n2 < 0) return -1;
  const int64_t total = n0 * n1 * n2;
  if (total == 0) return 0;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  normal_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(dst, n0, n1, n2, s0, s1, base,
                                                                    stream_key(seed, tid), mean, sd);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int qwen3synth_uniform_int_host(int32_t* dst, int64_t n, int64_t base, uint64_t seed, uint64_t tid,
                                int64_t upper) {
  if (!dst || n < 0 || upper <= 0) return -1;
  const uint64_t key = stream_key(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) dst[j] = uniform_int(key, (uint64_t)(base + j), (uint64_t)upper);
  return 0;
}

int qwen3synth_uniform_int_device(int32_t* dst, int64_t n, int64_t base, uint64_t seed, uint64_t tid,
                                  int64_t upper, void* stream) {
  if (!dst || n < 0 || upper <= 0) return -1;
  if (n == 0) return 0;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  uniform_int_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(dst, n, base, stream_key(seed, tid),
                                                                         (uint64_t)upper);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

}  // extern "C"
