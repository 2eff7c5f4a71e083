// Layer-stack helper of the C ABI (see cswa_attn.h): the per-layer window rule of
// nanochat's stacks (nanochat Admin & Developer Guide, 3 "Sliding-window attention").
// Host code only; the cache replication of the generation flow is a kernel
// (csrc/replicate.cuh, launched from csrc/cswa.cu).
#include <cstring>

#include "cswa_attn.h"

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

}  // extern "C"
