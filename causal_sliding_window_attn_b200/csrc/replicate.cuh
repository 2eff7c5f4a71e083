// attn_kv_replicate: the batch-1 prefill cache of every layer broadcast to N sample
// rows (nanochat Admin & Developer Guide, 7 "KV cache" and "Generation flow": the
// prompt is prefilled once at batch 1, then its cache is copied to every row).
// HBM-bound: each vector of the prompt rows is read once and stored N times, so the
// traffic is the algorithmic (1 + N) x the prompt bytes. Grid-stride over vectors,
// kInFlight loads per thread before their stores.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct ReplicateParams {
  const uint8_t* src[2];  // k, v: (n_layers, 1, Tsrc, Hkv, D)
  uint8_t* dst[2];        //       (n_layers, N, Tmax, Hkv, D)
  long long vec_per_layer;       // prompt vectors of one layer: rows * row_bytes / vec
  long long src_layer, dst_layer, dst_sample;  // strides in vectors
  long long total;               // 2 * n_layers * vec_per_layer
  int N;
};

template <typename V>
__global__ void __launch_bounds__(256) kv_replicate_kernel(const ReplicateParams p) {
  constexpr int kInFlight = 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; i0 < p.total; i0 += kInFlight * stride) {
    V val[kInFlight];
    V* dst[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const long long i = i0 + u * stride;
      if (i < p.total) {
        const bool is_v = i >= p.total / 2;
        const long long r = is_v ? i - p.total / 2 : i;
        const long long l = r / p.vec_per_layer, e = r - l * p.vec_per_layer;
        const V* src = reinterpret_cast<const V*>(is_v ? p.src[1] : p.src[0]);
        val[u] = src[l * p.src_layer + e];
        dst[u] = reinterpret_cast<V*>(is_v ? p.dst[1] : p.dst[0]) + l * p.dst_layer + e;
      }
    }
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      if (i0 + u * stride < p.total)
        for (int n = 0; n < p.N; ++n) dst[u][n * p.dst_sample] = val[u];
    }
  }
}

}  // namespace cswa
