// synth.cu -- device side of the seeded synthetic-input generator.
//
// Draws element n of tensor (seed, kind, layer) exactly as the host generator
// in synth.py does: SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) keyed per
// stream, mapped to INT9 / POW2W / NORMAL values, with optional layer
// correlation x_l = 0.9 x_{l-1} + 0.44 n_l in fp32 (separately rounded
// multiplies and add, no contraction).  Holds none of the attention method's
// arithmetic; it only produces inputs.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, int kind, int layer) {
  return mix64(seed * kGamma + ((uint64_t)kind << 40) + ((uint64_t)layer << 24) + 1ull);
}

__device__ inline float draw(uint64_t z, int dist, float c) {
  if (dist == 0) return (float)((int)(((z >> 32) * 9ull) >> 32) - 4);
  if (dist == 1) {
    float mag = ldexpf(1.0f, -(int)((z >> 61) & 3ull));
    return (z >> 63) ? -mag : mag;
  }
  int s = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) s += (int)((z >> (16 * i)) & 0xFFFFull);
  return __fmul_rn((float)(s - 131070), c);
}

__device__ inline float round_bf16(float x) {
  uint32_t u = __float_as_uint(x);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  return __uint_as_float(u);
}

__global__ void synth_fill_kernel(void* out, int64_t n, int64_t start, uint64_t seed,
                                  int kind, int dist, int layer, float c, int corr,
                                  int is_bf16) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (; i < n; i += stride) {
    uint64_t idx = (uint64_t)(start + i);
    int l0 = corr ? 0 : layer;
    float x = 0.0f;
    for (int l = l0; l <= layer; ++l) {
      uint64_t z = mix64(stream_key(seed, kind, l) + (idx + 1ull) * kGamma);
      float v = draw(z, dist, c);
      if (l == l0) {
        x = v;
      } else {
        x = __fadd_rn(__fmul_rn(0.9f, x), __fmul_rn(0.44f, v));
      }
      if (dist == 0) {
        x = fminf(fmaxf(rintf(x), -4.0f), 4.0f);
      } else if (is_bf16) {
        x = round_bf16(x);
      }
    }
    if (is_bf16) {
      ((uint16_t*)out)[i] = (uint16_t)(__float_as_uint(round_bf16(x)) >> 16);
    } else {
      ((float*)out)[i] = x;
    }
  }
}

}  // namespace

extern "C" int dsa_synth_fill(void* out, int64_t n, int64_t start, uint64_t seed, int kind,
                              int dist, int layer, float normal_scale, int corr, int is_bf16,
                              void* stream) {
  if (n <= 0) return 0;
  if (!out || dist < 0 || dist > 2 || layer < 0) return 1;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  synth_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      out, n, start, seed, kind, dist, layer, normal_scale, corr, is_bf16);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
