// CUDA implementation of the seeded input generator of synth/__init__.py, for
// tensors too large to draw on the host (8B-class weights, microbenchmark
// activations). Same definitions, element for element:
//   raw(seed, i)  = splitmix64 finaliser of seed + (i + 1) * 0x9E3779B97F4A7C15
//   u(r)          = (r >> 11) * 2^-53
//   normal(j)     = sqrt(-2 ln(1 - u(raw(2j)))) * cos(2 pi u(raw(2j + 1)))   (float64)
//   weight        = float32(scale * normal), stored as float32 or rounded to bf16
// Holds none of the early-skipping method's arithmetic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t raw(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double u53(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

__device__ __forceinline__ double normal_at(uint64_t seed, uint64_t j) {
  const double ua = u53(raw(seed, 2ull * j));
  const double ub = u53(raw(seed, 2ull * j + 1ull));
  return sqrt(-2.0 * log1p(-ua)) * cos((2.0 * 3.141592653589793) * ub);
}

__global__ void normal_kernel(void* out, uint64_t n, uint64_t seed, uint64_t start, double scale,
                              double shift, int bf16) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const float v = (float)(shift + scale * normal_at(seed, start + i));
    if (bf16)
      reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(out)[i] = v;
  }
}

// Microbenchmark tensors (synth.micro_inputs): x ~ N(0,1); the cached state is
// x + 0.01 * N(0,1) on rows kept by a Bernoulli(1 - changed_frac) draw, a fresh
// N(0,1) row otherwise (normal indices n + i and 2n + i); float64 then float32.
__global__ void micro_kernel(void* x_out, void* h_out, uint64_t rows, uint64_t d, uint64_t seed,
                             double changed_frac, int bf16) {
  const uint64_t n = rows * d;
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t row = i / d;
    const double x = normal_at(seed, i);
    const bool changed = u53(raw(seed + 1, row)) < changed_frac;
    const double h = changed ? normal_at(seed, 2 * n + i) : x + 0.01 * normal_at(seed, n + i);
    const float xf = (float)x, hf = (float)h;
    if (bf16) {
      reinterpret_cast<__nv_bfloat16*>(x_out)[i] = __float2bfloat16_rn(xf);
      reinterpret_cast<__nv_bfloat16*>(h_out)[i] = __float2bfloat16_rn(hf);
    } else {
      reinterpret_cast<float*>(x_out)[i] = xf;
      reinterpret_cast<float*>(h_out)[i] = hf;
    }
  }
}

}  // namespace

extern "C" {

int synth_fill_micro(void* x_out, void* h_out, uint64_t rows, uint64_t d, uint64_t seed,
                     double changed_frac, int bf16, void* stream) {
  if (!x_out || !h_out || rows == 0 || d == 0) return 1;
  micro_kernel<<<148 * 64, 256, 0, (cudaStream_t)stream>>>(x_out, h_out, rows, d, seed, changed_frac, bf16);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}


// out[i] = float32(shift + scale * normal(start + i)) (bf16 != 0: rounded to bf16), i < n
int synth_fill_normal(void* out, uint64_t n, uint64_t seed, uint64_t start, double scale,
                      double shift, int bf16, void* stream) {
  if (!out || n == 0) return 1;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 64) blocks = 148 * 64;
  normal_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(out, n, seed, start, scale, shift, bf16);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // extern "C"
