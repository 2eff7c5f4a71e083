// attn_quantize_fp8: tensorwise dynamic scaling of a bf16 tensor to float8 e4m3
// (nanochat Admin & Developer Guide, 5 "Precision: Explicit dtype & FP8": one scale
// per tensor from its absolute maximum, forward tensors in e4m3).
//   amax = max |x|,  s = 448 / amax (1 when amax = 0),  codes = e4m3(x * s)
// with the division and the product in fp32 and the rounding to nearest even,
// saturating at +-448; the dequantization factor amax / 448 goes to device memory.
// Two launches: per-block maxima into a small workspace, then every block reduces
// them and writes its share of the codes. HBM-bound: 2 bytes read twice, 1 written.
#pragma once
#include "ptx.cuh"

namespace cswa {

constexpr int kQuantMaxBlocks = 1024;

__device__ __forceinline__ float block_max_256(float m, float* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float bf16_abs_max8(const uint4& v, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    m = fmaxf(m, fabsf(__uint_as_float(w[u] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[u] & 0xffff0000u)));
  }
  return m;
}

// per-block maxima of |x| over 8-element vectors (n8 of them)
__global__ void __launch_bounds__(256) quant_amax_kernel(const uint4* x, long long n8, float* part) {
  __shared__ float red[8];
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n8; i += (long long)gridDim.x * 256)
    m = bf16_abs_max8(x[i], m);
  m = block_max_256(m, red);
  if (threadIdx.x == 0) part[blockIdx.x] = m;
}

// codes = e4m3(x * s) after reducing the n_part per-block maxima
__global__ void __launch_bounds__(256) quant_e4m3_kernel(const uint4* x, long long n8, const float* part,
                                                           int n_part, uint2* out, float* descale) {
  __shared__ float red[8];
  float m = 0.f;
  for (int i = threadIdx.x; i < n_part; i += 256) m = fmaxf(m, part[i]);
  const float amax = block_max_256(m, red);
  const float s = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *descale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n8; i += (long long)gridDim.x * 256) {
    const uint4 v = x[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      f[2 * u] = __fmul_rn(__uint_as_float(w[u] << 16), s);
      f[2 * u + 1] = __fmul_rn(__uint_as_float(w[u] & 0xffff0000u), s);
    }
    out[i] = make_uint2(pack_e4m3x4(f[0], f[1], f[2], f[3]), pack_e4m3x4(f[4], f[5], f[6], f[7]));
  }
}

}  // namespace cswa
