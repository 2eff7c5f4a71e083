// attn_decode: one new query token per sequence against a bf16 KV cache.
//
// Sequence b's token sits at position P = pos[b] and attends to the keys
// [max(0, P - W), P] of its cache (nanochat Admin & Developer Guide, 7 "KV
// cache": per-row positions, in-place append; 6: decode slices the window).
//
// Memory-bound split-K. Kernel 1 gives each CTA one (b, kv head, chunk of 128
// keys) and all G query heads of the group, so every cache byte is read once:
//   pass 1  scores: D/8 lanes per key row, one 16-byte load each, 16 rows in
//           flight per thread; s = <q, k> * scale * log2(e) into shared memory
//   pass 2  chunk max m and p = 2^(s - m), sum l
//   pass 3  acc = sum_j p_j v_j, 16-byte V loads, reduced across key groups
// and writes (acc, m, l) per query head. The chunk holding P reads k_new/v_new
// instead of the cache and writes them into it. Kernel 2 merges the chunks of
// each (b, h) with weights 2^(m_c - max m): o = sum acc / sum l, lse.
#pragma once
#include "ptx.cuh"

namespace cswa {

constexpr int kDecodeChunk = 128;

struct DecodeParams {
  const __nv_bfloat16* q;
  __nv_bfloat16* kc;
  __nv_bfloat16* vc;
  const __nv_bfloat16* kn;
  const __nv_bfloat16* vn;
  const int* pos;
  __nv_bfloat16* o;
  float* lse;
  float* ws;  // (B, Hq, n_chunks, D + 2)
  int Tmax, Hq, Hkv, G, window, n_chunks;
  float scale_log2;
};

__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 t = __bfloat1622float2(h[u]);
    f[2 * u] = t.x;
    f[2 * u + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 ld_stream(const __nv_bfloat16* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int D, int GMAX>
__global__ void __launch_bounds__(128) decode_chunk_kernel(const DecodeParams p) {
  constexpr int LK = D / 8;          // lanes per key row
  constexpr int KPP = 128 / LK;      // key rows per pass
  constexpr int PASSES = kDecodeChunk / KPP;
  constexpr int UNROLL = PASSES < 8 ? PASSES : 8;
  __shared__ float s_sc[GMAX][kDecodeChunk];
  __shared__ float s_red[GMAX][4];
  __shared__ float s_stat[GMAX][2];
  __shared__ float s_acc[KPP][GMAX][D];

  const int chunk = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int P = p.pos[b];
  if (P < 0 || P >= p.Tmax) {
    if (threadIdx.x == 0 && chunk == 0 && hk == 0) atomicOr(&g_status, kStatusBadPosition);
    return;
  }
  const int lo = p.window < 0 ? 0 : max(0, P - p.window);
  const int k_begin = lo + chunk * kDecodeChunk;
  if (k_begin > P) return;
  const int nk = min(P, k_begin + kDecodeChunk - 1) - k_begin + 1;
  const int tid = threadIdx.x, lr = tid % LK, sub = tid / LK, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;
  const bool append = p.kn != nullptr;

  float qf[GMAX][8];
#pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    if (g < G) {
      bf16x8_to_float(*reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + hk * G + g) * D + lr * 8),
                      qf[g]);
    }
  }
  auto row_ptr = [&](const __nv_bfloat16* cache, const __nv_bfloat16* fresh, int j) {
    return (append && j == P) ? fresh + ((size_t)b * p.Hkv + hk) * D + lr * 8
                              : cache + (((size_t)b * p.Tmax + j) * p.Hkv + hk) * D + lr * 8;
  };

  // pass 1: scores
  for (int ps = 0; ps < PASSES; ps += UNROLL) {
    uint4 kv[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int kc = (ps + u) * KPP + sub;
      kv[u] = kc < nk ? ld_stream(row_ptr(p.kc, p.kn, k_begin + kc)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float kf[8];
      bf16x8_to_float(kv[u], kf);
      const int kc = (ps + u) * KPP + sub;
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g < G) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) d = fmaf(qf[g][e], kf[e], d);
#pragma unroll
          for (int o = LK / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
          if (lr == 0 && kc < nk) s_sc[g][kc] = d * p.scale_log2;
        }
      }
    }
  }
  __syncthreads();

  // pass 2: chunk max and exponentials (thread tid owns key tid)
#pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    if (g < G) {
      float v = tid < nk ? s_sc[g][tid] : -INFINITY;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0) s_red[g][warp] = v;
    }
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    if (g < G) {
      const float m = fmaxf(fmaxf(s_red[g][0], s_red[g][1]), fmaxf(s_red[g][2], s_red[g][3]));
      const float e = tid < nk ? ex2_approx(s_sc[g][tid] - m) : 0.f;
      if (tid < nk) s_sc[g][tid] = e;
      float l = e;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (tid == 0) s_stat[g][0] = m;
      __syncwarp();
      if (lane == 0) s_acc[0][g][warp] = l;  // scratch for the sum
    }
  }
  __syncthreads();
  if (tid < G) s_stat[tid][1] = s_acc[0][tid][0] + s_acc[0][tid][1] + s_acc[0][tid][2] + s_acc[0][tid][3];
  __syncthreads();

  // pass 3: acc = sum_j p_j v_j
  float acc[GMAX][8];
#pragma unroll
  for (int g = 0; g < GMAX; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  for (int ps = 0; ps < PASSES; ps += UNROLL) {
    uint4 vv[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int kc = (ps + u) * KPP + sub;
      vv[u] = kc < nk ? ld_stream(row_ptr(p.vc, p.vn, k_begin + kc)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float vf[8];
      bf16x8_to_float(vv[u], vf);
      const int kc = (ps + u) * KPP + sub;
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g < G) {
          const float pj = kc < nk ? s_sc[g][kc] : 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pj, vf[e], acc[g][e]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < GMAX; ++g)
    if (g < G)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_acc[sub][g][lr * 8 + e] = acc[g][e];
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += 128) {
    const int g = idx / D, d = idx % D;
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < KPP; ++k) sum += s_acc[k][g][d];
    float* w = p.ws + (((size_t)b * p.Hq + hk * G + g) * p.n_chunks + chunk) * (D + 2);
    w[d] = sum;
    if (d == 0) {
      w[D] = s_stat[g][0];
      w[D + 1] = s_stat[g][1];
    }
  }
  // in-place append of the new token's key/value (only the chunk that holds P)
  if (append && P >= k_begin && P < k_begin + nk) {
    for (int idx = tid; idx < 2 * LK; idx += 128) {
      const int which = idx / LK, l = idx % LK;
      const __nv_bfloat16* src = (which ? p.vn : p.kn) + ((size_t)b * p.Hkv + hk) * D + l * 8;
      __nv_bfloat16* dst = (which ? p.vc : p.kc) + (((size_t)b * p.Tmax + P) * p.Hkv + hk) * D + l * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int P = p.pos[b];
  __nv_bfloat16* out = p.o + ((size_t)b * p.Hq + h) * D;
  if (P < 0 || P >= p.Tmax) {
    out[d] = __float2bfloat16(NAN);
    if (d == 0 && p.lse) p.lse[(size_t)b * p.Hq + h] = NAN;
    return;
  }
  const int lo = p.window < 0 ? 0 : max(0, P - p.window);
  const int nc = (P - lo + kDecodeChunk) / kDecodeChunk;
  const float* w = p.ws + ((size_t)b * p.Hq + h) * p.n_chunks * (D + 2);
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, w[c * (D + 2) + D]);
  float Lsum = 0.f, O = 0.f;
  for (int c = 0; c < nc; ++c) {
    const float f = ex2_approx(w[c * (D + 2) + D] - M);
    Lsum = fmaf(f, w[c * (D + 2) + D + 1], Lsum);
    O = fmaf(f, w[c * (D + 2) + d], O);
  }
  out[d] = __float2bfloat16(O / Lsum);
  if (d == 0 && p.lse) p.lse[(size_t)b * p.Hq + h] = (M + __log2f(Lsum)) * 0.69314718055994531f;
}

}  // namespace cswa
