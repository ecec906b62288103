// Device twin of the host generator in synthetic/__init__.py: the same
// SplitMix64 words and Irwin-Hall deviates, bit for bit, so large seeded
// inputs can be made directly in device memory.  No NVFP4 arithmetic here.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kG = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t stream_key(uint64_t seed, uint64_t stream) { return mix(mix(seed + kG) + (stream + 1) * kG); }

__device__ __forceinline__ uint64_t word(uint64_t key, uint64_t i) { return mix(key + (i + 1) * kG); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t b = __float_as_uint(f);
  return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

__global__ void normal_bf16_kernel(uint64_t key, int64_t start, int64_t count, double sigma, int scale,
                                   uint16_t *out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < count; j += stride) {
    const uint64_t base = 3ull * (uint64_t)(start + j);
    int64_t s = 0;
#pragma unroll
    for (int w = 0; w < 3; ++w) {
      const uint64_t x = word(key, base + w);
      s += (int64_t)(x & 0xFFFF) + (int64_t)((x >> 16) & 0xFFFF) + (int64_t)((x >> 32) & 0xFFFF) + (int64_t)(x >> 48);
    }
    double z = (double)(s - 393210) * (1.0 / 65536.0);   // exact
    if (scale) z = __dmul_rn(z, sigma);
    out[j] = f32_to_bf16_rne(__double2float_rn(z));
  }
}

__global__ void bytes_kernel(uint64_t key, int64_t start_word, int64_t nwords, uint64_t *out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nwords; i += stride)
    out[i] = word(key, (uint64_t)(start_word + i));
}

__global__ void mx_exp_kernel(uint64_t key, int64_t start, int64_t count, int lo, uint8_t *out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
    out[i] = (uint8_t)(127 + lo + (int)(word(key, (uint64_t)(start + i)) >> 61));
}

unsigned grid(int64_t n) {
  int64_t b = (n + 255) / 256;
  return (unsigned)(b < 148 * 16 ? (b < 1 ? 1 : b) : 148 * 16);
}

}  // namespace

extern "C" {

// bf16 bits of N(0, sigma^2) deviates j = start .. start+count-1 of (seed, stream).
int synth_normal_bf16(uint64_t seed, uint64_t stream, int64_t start, int64_t count, double sigma,
                      void *out, cudaStream_t cs) {
  if (count <= 0) return 0;
  normal_bf16_kernel<<<grid(count), 256, 0, cs>>>(stream_key(seed, stream), start, count, sigma,
                                                   sigma != 1.0, (uint16_t *)out);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

// nwords SplitMix64 words from word index start_word, written as little-endian bytes.
int synth_words(uint64_t seed, uint64_t stream, int64_t start_word, int64_t nwords, void *out, cudaStream_t cs) {
  if (nwords <= 0) return 0;
  bytes_kernel<<<grid(nwords), 256, 0, cs>>>(stream_key(seed, stream), start_word, nwords, (uint64_t *)out);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

// UE8M0 bytes 127 + lo + (word >> 61).
int synth_mx_exponents(uint64_t seed, uint64_t stream, int64_t start, int64_t count, int lo, void *out,
                       cudaStream_t cs) {
  if (count <= 0) return 0;
  mx_exp_kernel<<<grid(count), 256, 0, cs>>>(stream_key(seed, stream), start, count, lo, (uint8_t *)out);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

}  // extern "C"
