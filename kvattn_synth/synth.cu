// Seeded N(0,1) bf16 generator on the device: SplitMix64 words (Steele, Lea,
// Flood, OOPSLA 2014) used counter-style, fed to Box-Muller (1958).  Same
// definition as the numpy implementation in __init__.py of this module; it
// holds no attention arithmetic and serves only to fill large inputs in HBM.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed ^ mix64(stream + kGamma));
}

__device__ inline uint16_t normal_bits(uint64_t key, uint64_t e) {
  const uint64_t w1 = mix64(key + (2 * e + 1) * kGamma);
  const uint64_t w2 = mix64(key + (2 * e + 2) * kGamma);
  const double u1 = (double)(w1 >> 11) * 0x1.0p-53;
  const double u2 = (double)(w2 >> 11) * 0x1.0p-53;
  const double z = sqrt(-2.0 * log1p(-u1)) * cos(2.0 * 3.141592653589793 * u2);
  const float f = __double2float_rn(z);
  const uint32_t u = __float_as_uint(f);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

__global__ void normal_kernel(uint64_t key, uint64_t offset, uint64_t n, uint16_t* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = normal_bits(key, offset + i);
}

// cache [B,S,Hkv,d]; element (b,r,j,c) gets the draw of its flat index when
// r < start_pos[b], else 0.
__global__ void cache_fill_kernel(uint64_t key, int B, int S, int row_elems,
                                  const int32_t* start_pos, uint16_t* out) {
  const uint64_t n = (uint64_t)B * S * row_elems;
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t row = i / row_elems;
    const int b = (int)(row / S);
    const int r = (int)(row % S);
    out[i] = (r < start_pos[b]) ? normal_bits(key, i) : (uint16_t)0;
  }
}

int grid_for(uint64_t n) {
  uint64_t g = (n + 255) / 256;
  if (g > 148ull * 64) g = 148ull * 64;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" int kvsynth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, uint64_t n,
                                   void* out, void* cuda_stream) {
  if (n == 0) return 0;
  if (!out) return 1;
  normal_kernel<<<grid_for(n), 256, 0, (cudaStream_t)cuda_stream>>>(
      stream_key(seed, stream), offset, n, (uint16_t*)out);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

extern "C" int kvsynth_cache_fill(uint64_t seed, uint64_t stream, int B, int S, int Hkv, int d,
                                  const void* start_pos, void* out, void* cuda_stream) {
  if (B <= 0 || S <= 0 || Hkv <= 0 || d <= 0) return 1;
  if (!out || !start_pos) return 1;
  const uint64_t n = (uint64_t)B * S * Hkv * d;
  cache_fill_kernel<<<grid_for(n), 256, 0, (cudaStream_t)cuda_stream>>>(
      stream_key(seed, stream), B, S, Hkv * d, (const int32_t*)start_pos, (uint16_t*)out);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}
