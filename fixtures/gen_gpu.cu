// Device mirror of the seeded input generators (fixtures/gen.py): SplitMix64
// counter streams, packed code words, exact inverse-CDF bf16 normals from a
// threshold table built on the host, and the derived group biases. Integer
// arithmetic only (plus one exact fp32 multiply), so the output is bit for bit
// the host generator's. Holds no arithmetic of the MoE forward itself.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__device__ __forceinline__ uint64_t stream_at(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * 0x9E3779B97F4A7C15ull);
}

// out[e*per + i] = low32 of output i of stream keys[e]
__global__ void codes_kernel(uint32_t* out, const uint64_t* keys, uint64_t per, uint64_t n) {
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < n; g += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t e = g / per, i = g - e * per;
    out[g] = (uint32_t)stream_at(keys[e], i);
  }
}

__device__ __forceinline__ uint16_t draw(uint32_t u, const uint32_t* thr, int nthr, const uint16_t* vals) {
  int lo = 0, hi = nthr;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(thr + mid) <= u) lo = mid + 1; else hi = mid;
  }
  return __ldg(vals + lo);
}

__global__ void normal_kernel(uint16_t* out, const uint64_t* keys, uint64_t per, uint64_t n, const uint32_t* thr,
                              int nthr, const uint16_t* vals, int signed_) {
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < n; g += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t e = g / per, i = g - e * per;
    const uint64_t z = stream_at(keys[e], i);
    uint16_t v = draw((uint32_t)z, thr, nthr, vals);
    if (signed_) v |= (uint16_t)((z >> 63) << 15);
    out[g] = v;
  }
}

__device__ __forceinline__ uint16_t rne_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return (uint16_t)u;
}

__global__ void bias_kernel(uint16_t* b, const uint16_t* s, uint64_t n, int bits) {
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < n; g += (uint64_t)gridDim.x * blockDim.x) {
    const float sv = __uint_as_float((uint32_t)s[g] << 16);
    b[g] = rne_bf16(__fmul_rn(bits == 4 ? -8.0f : -1.5f, sv));
  }
}

int grid_for(uint64_t n) {
  uint64_t b = (n + 255) / 256;
  return (int)(b > 148 * 32 ? 148 * 32 : (b ? b : 1));
}

}  // namespace

extern "C" {

int fx_codes(uint32_t* out, const uint64_t* keys, uint64_t per, uint64_t n, void* stream) {
  codes_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, keys, per, n);
  return (int)cudaGetLastError();
}

int fx_normal(uint16_t* out, const uint64_t* keys, uint64_t per, uint64_t n, const uint32_t* thr, int nthr,
              const uint16_t* vals, int signed_, void* stream) {
  normal_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, keys, per, n, thr, nthr, vals, signed_);
  return (int)cudaGetLastError();
}

int fx_bias(uint16_t* b, const uint16_t* s, uint64_t n, int bits, void* stream) {
  bias_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(b, s, n, bits);
  return (int)cudaGetLastError();
}

}
