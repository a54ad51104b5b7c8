// Seeded synthetic inputs on the device (weights, embeddings, prompts).
//
// Holds no arithmetic of the method.  Each element is an independent function
// of (stream key, element index): the splitmix64 output function (Steele, Lea
// and Flood, OOPSLA 2014) applied to key + golden * (index + 1).  Normal draws
// sum the four 16-bit fields of one hash (Irwin-Hall), centre them, and apply
// one fp32 round-to-nearest multiply and one fp32 add before rounding to fp16;
// token ids take ((hash >> 32) * vocab) >> 32.  The host-side generator used by
// the tests implements the same published definition independently.
#include "kernels.h"

namespace flexq {
namespace {

__device__ __forceinline__ uint64_t splitmix_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t element_hash(uint64_t key, uint64_t idx) {
  return splitmix_mix(key + 0x9E3779B97F4A7C15ull * (idx + 1));
}

__device__ __forceinline__ __half normal_from_hash(uint64_t hsh, float scale, float mean) {
  const uint32_t s = static_cast<uint32_t>(hsh & 0xFFFF) + static_cast<uint32_t>((hsh >> 16) & 0xFFFF) +
                     static_cast<uint32_t>((hsh >> 32) & 0xFFFF) + static_cast<uint32_t>(hsh >> 48);
  const float z = static_cast<float>(static_cast<int>(s) - 131070);
  return __float2half_rn(__fadd_rn(__fmul_rn(z, scale), mean));
}

__global__ void synth_normal_kernel(__half* __restrict__ out, size_t n, uint64_t key, size_t start,
                                    float scale, float mean) {
  const size_t base = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (base >= n) return;
  if (base + 8 <= n && (reinterpret_cast<uintptr_t>(out + base) & 15) == 0) {
    __align__(16) __half v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = normal_from_hash(element_hash(key, start + base + j), scale, mean);
    *reinterpret_cast<uint4*>(out + base) = *reinterpret_cast<uint4*>(v);
  } else {
    for (size_t i = base; i < n && i < base + 8; ++i)
      out[i] = normal_from_hash(element_hash(key, start + i), scale, mean);
  }
}

__global__ void synth_tokens_kernel(int32_t* __restrict__ out, size_t n, uint64_t key, size_t start,
                                    int vocab) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint64_t hsh = element_hash(key, start + i);
  out[i] = static_cast<int32_t>(((hsh >> 32) * static_cast<uint64_t>(vocab)) >> 32);
}

}  // namespace

cudaError_t launch_synth_normal(__half* out, size_t n, uint64_t key, size_t start, float scale,
                                float mean, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const size_t threads = (n + 7) / 8;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  synth_normal_kernel<<<blocks, 256, 0, s>>>(out, n, key, start, scale, mean);
  return launched();
}

cudaError_t launch_synth_tokens(int32_t* out, size_t n, uint64_t key, size_t start, int vocab,
                                cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
  synth_tokens_kernel<<<blocks, 256, 0, s>>>(out, n, key, start, vocab);
  return launched();
}

}  // namespace flexq
