// Layer-stack helpers of the C ABI (see cswa_attn.h): the per-layer window rule and
// the batch-1 -> N KV-cache replication of nanochat's generation flow (nanochat Admin
// & Developer Guide, 3 "Sliding-window attention"; 7 "KV cache" and "Generation
// flow"). Host code only: the replication is stream-ordered copy-engine copies, no
// kernel, and nothing here allocates.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "cswa_attn.h"

namespace {

// Largest pitch a 2-D copy takes on the current device (looked up per call: cheap).
size_t max_pitch() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMaxPitch, dev) != cudaSuccess ||
      v <= 0)
    return 0;
  return (size_t)v;
}

bool disjoint(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x + na <= y || y + nb <= x;
}

}  // namespace

extern "C" {

int attn_layer_window(const char* pattern, int layer, int n_layer, int seq_len, int short_window) {
  if (!pattern || !pattern[0] || n_layer < 1 || layer < 0 || layer >= n_layer || seq_len < 1) return -2;
  const size_t len = std::strlen(pattern);
  for (size_t i = 0; i < len; ++i)
    if (pattern[i] != 'S' && pattern[i] != 'L') return -2;
  if (layer == n_layer - 1 || pattern[(size_t)layer % len] == 'L') return -1;  // the last layer is always L
  if (short_window > 0) return short_window;
  const long long quarter = ((long long)seq_len + 3) / 4;  // a quarter of the context, rounded up ...
  return (int)((quarter + 127) / 128 * 128);               // ... to a whole 128-row tile
}

attn_status_t attn_kv_replicate(const void* k_src, const void* v_src, void* k_dst, void* v_dst, int n_layers,
                                int rows, int Tmax_src, int N, int Tmax, int Hkv, int D, void* stream) {
  if (!k_src || !v_src || !k_dst || !v_dst || n_layers < 1 || rows < 0 || Tmax_src < 1 || N < 1 || Tmax < 1 ||
      Hkv < 1 || D < 1 || rows > Tmax_src || rows > Tmax)
    return ATTN_ERR_INVALID_ARG;
  const size_t row_bytes = (size_t)Hkv * D * 2;
  const size_t copy_bytes = (size_t)rows * row_bytes;     // the prompt rows of one (layer, sample)
  const size_t src_layer = (size_t)Tmax_src * row_bytes;  // batch-1 source: layer stride
  const size_t dst_batch = (size_t)Tmax * row_bytes;      // destination: sample stride ...
  const size_t dst_layer = (size_t)N * dst_batch;         // ... and layer stride
  const size_t src_bytes = (size_t)n_layers * src_layer, dst_bytes = (size_t)n_layers * dst_layer;
  if (!disjoint(k_dst, dst_bytes, v_dst, dst_bytes) || !disjoint(k_dst, dst_bytes, k_src, src_bytes) ||
      !disjoint(k_dst, dst_bytes, v_src, src_bytes) || !disjoint(v_dst, dst_bytes, k_src, src_bytes) ||
      !disjoint(v_dst, dst_bytes, v_src, src_bytes))
    return ATTN_ERR_INVALID_ARG;
  if (rows == 0) return ATTN_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool two_d = dst_batch <= max_pitch();
  const void* srcs[2] = {k_src, v_src};
  void* dsts[2] = {k_dst, v_dst};
  for (int x = 0; x < 2; ++x) {
    const uint8_t* s = static_cast<const uint8_t*>(srcs[x]);
    uint8_t* d = static_cast<uint8_t*>(dsts[x]);
    // sample 0 of every layer from the batch-1 cache ...
    for (int l = 0; l < n_layers; ++l)
      if (cudaMemcpyAsync(d + l * dst_layer, s + l * src_layer, copy_bytes, cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
        return ATTN_ERR_LAUNCH;
    // ... then the filled samples [0, m) are copied to [m, 2m): ceil(log2 N) rounds
    for (int m = 1; m < N;) {
      const int c = std::min(m, N - m);
      for (int l = 0; l < n_layers; ++l) {
        uint8_t* base = d + l * dst_layer;
        if (two_d) {
          if (cudaMemcpy2DAsync(base + (size_t)m * dst_batch, dst_batch, base, dst_batch, copy_bytes, c,
                                cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return ATTN_ERR_LAUNCH;
        } else {
          for (int i = 0; i < c; ++i)
            if (cudaMemcpyAsync(base + (size_t)(m + i) * dst_batch, base + (size_t)i * dst_batch, copy_bytes,
                                cudaMemcpyDeviceToDevice, st) != cudaSuccess)
              return ATTN_ERR_LAUNCH;
        }
      }
      m += c;
    }
  }
  return ATTN_OK;
}

}  // extern "C"
