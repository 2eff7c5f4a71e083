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

// d += a.lo * b.lo + a.hi * b.hi for packed bf16 pairs, accumulated in fp32 (the
// products of two bf16 values are exact in fp32): no conversion instructions.
__device__ __forceinline__ float fma_bf16x2_f32(uint32_t a, uint32_t b, float d) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\tfma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(d)
      : "r"(a), "r"(b));
  return d;
}
// d_lo += p * b.lo, d_hi += p * b.hi with p a bf16 value (in the low half of pp)
__device__ __forceinline__ void fma_bf16_pair_f32(uint32_t pp, uint32_t b, float& lo, float& hi) {
  asm("{\n\t.reg .b16 p, x, bl, bh;\n\tmov.b32 {p, x}, %2;\n\tmov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, p, bl, %0;\n\tfma.rn.f32.bf16 %1, p, bh, %1;\n\t}"
      : "+f"(lo), "+f"(hi)
      : "r"(pp), "r"(b));
}

// Sum of v[0..7] (one partial dot product per key) over the 16 lanes of a key-row
// group, as a transposing butterfly: 8 shuffles for 8 keys. Lane lr ends with the
// full sum of key (lr >> 1) & 7.
__device__ __forceinline__ float reduce8x16(float (&v)[8], int lr) {
  const bool b3 = lr & 8, b2 = lr & 4, b1 = lr & 2;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b3 ? v[i] : v[i + 4], keep = b3 ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b2 ? v[i] : v[i + 2], keep = b2 ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const float send = b1 ? v[0] : v[1], keep = b1 ? v[1] : v[0];
  float r = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  return r + __shfl_xor_sync(0xffffffffu, r, 1);
}

template <int D, int GMAX>
__global__ void __launch_bounds__(128) decode_chunk_kernel(const DecodeParams p) {
  constexpr int LK = D / 8;          // lanes per key row
  constexpr int KPP = 128 / LK;      // key rows per pass
  constexpr int PASSES = kDecodeChunk / KPP;
  constexpr int UNROLL = 8;          // key rows per thread in flight (the butterfly takes 8)
  static_assert(PASSES % UNROLL == 0, "passes per chunk");
  static_assert(LK == 16 || LK == 8, "lanes per key row");
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
  // chunks before the last hold 128 cache rows and not the new token: no bounds
  // checks, no row substitution
  const bool full = (k_begin + kDecodeChunk - 1 < P);
  const int tid = threadIdx.x, lr = tid % LK, sub = tid / LK, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;
  const bool append = p.kn != nullptr;
  const size_t row_stride = (size_t)p.Hkv * D;          // elements between consecutive keys
  const size_t pass_stride = row_stride * KPP;          // between a thread's consecutive rows
  const size_t cache_off = (((size_t)b * p.Tmax + k_begin + sub) * p.Hkv + hk) * D + lr * 8;
  const size_t fresh_off = ((size_t)b * p.Hkv + hk) * D + lr * 8;

  uint32_t qv[GMAX][4];
#pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    const uint4 t = (g < G) ? *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + hk * G + g) * D + lr * 8)
                            : make_uint4(0, 0, 0, 0);
    qv[g][0] = t.x, qv[g][1] = t.y, qv[g][2] = t.z, qv[g][3] = t.w;
  }
  // row kc of the chunk for this thread's pass u: cache row, or the new token at P
  auto load_row = [&](const __nv_bfloat16* cache, const __nv_bfloat16* fresh, int u) {
    const int kc = u * KPP + sub;
    if (full) return ld_stream(cache + cache_off + u * pass_stride);
    if (kc >= nk) return make_uint4(0, 0, 0, 0);
    if (append && k_begin + kc == P) return ld_stream(fresh + fresh_off);
    return ld_stream(cache + cache_off + u * pass_stride);
  };

  // pass 1: scores s = <q, k> * scale * log2(e)
  for (int ps = 0; ps < PASSES; ps += UNROLL) {
    uint4 kv[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) kv[u] = load_row(p.kc, p.kn, ps + u);
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < G) {
        float d[8];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          float t = 0.f;
          t = fma_bf16x2_f32(qv[g][0], kv[u].x, t);
          t = fma_bf16x2_f32(qv[g][1], kv[u].y, t);
          t = fma_bf16x2_f32(qv[g][2], kv[u].z, t);
          t = fma_bf16x2_f32(qv[g][3], kv[u].w, t);
          d[u] = t;
        }
        float sum;
        if (LK == 16) {
          sum = reduce8x16(d, lr);
          const int kc = (ps + ((lr >> 1) & 7)) * KPP + sub;
          if ((lr & 1) == 0 && kc < nk) s_sc[g][kc] = sum * p.scale_log2;
        } else {
          // 8 lanes per row: reduce each key separately
#pragma unroll
          for (int u = 0; u < UNROLL; ++u) {
            float t = d[u];
#pragma unroll
            for (int o = LK / 2; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            const int kc = (ps + u) * KPP + sub;
            if (lr == 0 && kc < nk) s_sc[g][kc] = t * p.scale_log2;
          }
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

  // pass 3: acc = sum_j p_j v_j, p_j rounded to bf16 (as the PV product of attn_fwd)
  float acc[GMAX][8];
#pragma unroll
  for (int g = 0; g < GMAX; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  for (int ps = 0; ps < PASSES; ps += UNROLL) {
    uint4 vv[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) vv[u] = load_row(p.vc, p.vn, ps + u);
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int kc = (ps + u) * KPP + sub;
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g < G) {
          const float pj = (full || kc < nk) ? s_sc[g][kc] : 0.f;
          const uint32_t pb = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(pj));
          fma_bf16_pair_f32(pb, vv[u].x, acc[g][0], acc[g][1]);
          fma_bf16_pair_f32(pb, vv[u].y, acc[g][2], acc[g][3]);
          fma_bf16_pair_f32(pb, vv[u].z, acc[g][4], acc[g][5]);
          fma_bf16_pair_f32(pb, vv[u].w, acc[g][6], acc[g][7]);
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

// Merge of the chunk partials of one (b, h): weights 2^(m_c - max m), o = sum of the
// weighted acc / sum of the weighted l, lse. The chunk statistics are spread over the
// block and reduced with shuffles; the weighted sum over chunks issues 8 loads at a
// time (all L2 hits), so the merge costs a few load latencies, not two per chunk.
constexpr int kDecodeMaxChunks = 4096;
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  static_assert(D % 32 == 0 && D >= 64, "block of D threads");
  constexpr int NW = D / 32;
  __shared__ float s_f[kDecodeMaxChunks];
  __shared__ float s_red[NW];
  __shared__ float s_bc;
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x, lane = d & 31, wp = d >> 5;
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
  // max of the chunk maxima
  float mx = -INFINITY;
  for (int c = d; c < nc; c += D) mx = fmaxf(mx, w[c * (D + 2) + D]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[wp] = mx;
  __syncthreads();
  if (d == 0) {
    float m = s_red[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) m = fmaxf(m, s_red[i]);
    s_bc = m;
  }
  __syncthreads();
  const float M = s_bc;
  // chunk weights and the weighted sum of l
  float ls = 0.f;
  for (int c = d; c < nc; c += D) {
    const float f = ex2_approx(w[c * (D + 2) + D] - M);
    s_f[c] = f;
    ls = fmaf(f, w[c * (D + 2) + D + 1], ls);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  __syncthreads();  // s_red is reused; s_f is complete
  if (lane == 0) s_red[wp] = ls;
  __syncthreads();
  float Lsum = 0.f;
#pragma unroll
  for (int i = 0; i < NW; ++i) Lsum += s_red[i];
  // o[d] = sum_c f_c acc_c[d] / Lsum, 8 chunks per round
  float O = 0.f;
  for (int c0 = 0; c0 < nc; c0 += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = (c0 + u < nc) ? w[(c0 + u) * (D + 2) + d] : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c0 + u < nc) O = fmaf(s_f[c0 + u], v[u], O);
  }
  out[d] = __float2bfloat16(O / Lsum);
  if (d == 0 && p.lse) p.lse[(size_t)b * p.Hq + h] = (M + __log2f(Lsum)) * 0.69314718055994531f;
}

}  // namespace cswa
