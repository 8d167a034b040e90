// 64-bit fingerprint of a device buffer (e.g. the reference LM-head weights an
// offline scoring artifact was produced with).
//
// Word i (16 bytes, two 64-bit halves lo, hi; the tail is zero-padded) maps to
//   mix(mix(lo ^ mix(2i + 1)) + hi + 0x9E3779B97F4A7C15 * (i + 1))
// and the fingerprint is mix(bytes ^ sum_i of those, mod 2^64). mix is the
// splitmix64 finaliser (Steele, Lea and Flood, "Fast splittable pseudorandom
// number generators", OOPSLA 2014). A sum is independent of the reduction
// order, so the result is the same for any grid, run after run.
#include <cstdint>

#include "internal.h"

namespace dpo {

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t word_hash(uint64_t lo, uint64_t hi, uint64_t i) {
  return mix64(mix64(lo ^ mix64(2 * i + 1)) + hi + 0x9E3779B97F4A7C15ull * (i + 1));
}

__global__ void __launch_bounds__(256) k_fingerprint(const uint8_t* __restrict__ data,
                                                     unsigned long long bytes,
                                                     unsigned long long* __restrict__ acc) {
  const unsigned long long nwords = (bytes + 15) / 16;
  const unsigned long long full = bytes / 16;
  uint64_t s = 0;
  for (unsigned long long i = blockIdx.x * 256ull + threadIdx.x; i < nwords;
       i += static_cast<unsigned long long>(gridDim.x) * 256ull) {
    uint64_t lo = 0, hi = 0;
    if (i < full) {
      const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(data) + i);
      lo = v.x;
      hi = v.y;
    } else {
      uint8_t b[16] = {};
      for (unsigned long long k = i * 16; k < bytes; ++k) b[k - i * 16] = data[k];
      for (int k = 0; k < 8; ++k) lo |= static_cast<uint64_t>(b[k]) << (8 * k);
      for (int k = 0; k < 8; ++k) hi |= static_cast<uint64_t>(b[8 + k]) << (8 * k);
    }
    s += word_hash(lo, hi, i);
  }
  // warp sum, then one atomic per warp (addition mod 2^64 commutes: order-free)
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(acc, static_cast<unsigned long long>(s));
}

__global__ void k_fingerprint_final(unsigned long long bytes, unsigned long long* acc) {
  *acc = mix64(*acc ^ bytes);
}

cudaError_t launch_fingerprint(const void* data, unsigned long long bytes,
                               unsigned long long* out, int sms, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  if (bytes > 0) {
    const unsigned long long words = (bytes + 15) / 16;
    unsigned long long blocks = (words + 255) / 256;
    const unsigned long long cap = static_cast<unsigned long long>(sms) * 8;
    if (blocks > cap) blocks = cap;
    k_fingerprint<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint8_t*>(data), bytes, out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  k_fingerprint_final<<<1, 1, 0, st>>>(bytes, out);
  return cudaGetLastError();
}

}  // namespace dpo
