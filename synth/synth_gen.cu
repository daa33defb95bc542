// Device twin of synth.normal_bf16_bits: counter-based SplitMix64 draws mapped
// through a 65536-entry table of bf16 normal quantiles supplied by the caller.
// Input generation only; none of the attention method lives here.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__global__ void normal_bf16_kernel(uint16_t* __restrict__ out, uint64_t key, uint64_t start,
                                   uint64_t count, const uint16_t* __restrict__ table) {
  const uint16_t* __restrict__ t = table;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x * 8;
  for (uint64_t base = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; base < count;
       base += stride) {
    if (base + 8 <= count && ((reinterpret_cast<uintptr_t>(out + base) & 15) == 0)) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t lo = t[mix64(key + (start + base + 2 * j + 1) * kGamma) >> 48];
        uint32_t hi = t[mix64(key + (start + base + 2 * j + 2) * kGamma) >> 48];
        w[j] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(out + base) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      for (uint64_t i = base; i < base + 8 && i < count; ++i)
        out[i] = t[mix64(key + (start + i + 1) * kGamma) >> 48];
    }
  }
}

}  // namespace

extern "C" int synth_normal_bf16(void* out, uint64_t key, uint64_t start, uint64_t count,
                                 const void* table, void* stream) {
  if (count == 0) return 0;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint64_t blocks_needed = (count + 8 * 256 - 1) / (8 * 256);
  int blocks = (int)(blocks_needed < (uint64_t)sms * 8 ? blocks_needed : (uint64_t)sms * 8);
  normal_bf16_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)out, key, start, count, (const uint16_t*)table);
  return (int)cudaGetLastError();
}
