// attn_decode: one new query token per sequence against a bf16 KV cache.
//
// Sequence b's token sits at position P = pos[b] and attends to the keys
// [max(0, P - W), P] of its cache (nanochat Admin & Developer Guide, 7 "KV
// cache": per-row positions, in-place append; 6: decode slices the window).
//
// Memory-bound split-K in one launch. Each CTA takes one (b, kv head, chunk of 128
// keys) and all G query heads of the group (in sub-groups of up to 8), so every cache
// byte is read from HBM once:
//   pass 1  scores: D/8 lanes per key row, one 16-byte load each, 8 rows in flight
//           per thread; s = <q, k> * scale * log2(e) into shared memory
//   pass 2  chunk max m and p = 2^(s - m), sum l
//   pass 3  acc = sum_j p_j v_j, 16-byte V loads, reduced across key groups
// and writes (acc, m, l) per query head. The chunk holding P reads k_new/v_new
// instead of the cache and writes them into it. The last of a (b, kv head)'s chunk
// CTAs to finish (an arrival counter in the workspace) merges the chunks of each
// head with weights 2^(m_c - max m): o = sum acc / sum l, lse.
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
  float* ws;                      // (B, Hq, n_chunks, D + 2) partials
  unsigned long long* counters;   // (B, Hkv) arrival counters (see decode_arrive)
  unsigned epoch;                 // this call's tag for the counters (never 0)
  int Tmax, Hq, Hkv, G, window, n_chunks;
  float scale_log2;
};

constexpr int kDecodeMaxChunks = 4096;

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

// Arrival counter of a (sequence, KV head): the chunk CTAs of one call count themselves
// in; the last one merges. The counter is tagged with the call's epoch (high 32 bits)
// so that a stale or never-initialised counter reads as zero, and the merging CTA
// leaves it at (epoch, 0), which a replay of the same call (a CUDA graph) also
// reads as zero. Returns the CTA's arrival number (1-based), or 0 if the update did
// not go through within its retry limit (then nobody merges and the status word
// reports it).
__device__ __forceinline__ unsigned decode_arrive(unsigned long long* cnt, unsigned epoch) {
  unsigned long long old = atomicAdd(cnt, 0ull), nw = 0;
  for (int i = 0; i < (1 << 16); ++i) {
    const unsigned have = ((unsigned)(old >> 32) == epoch) ? (unsigned)old : 0u;
    nw = ((unsigned long long)epoch << 32) | (unsigned long long)(have + 1u);
    const unsigned long long prev = atomicCAS(cnt, old, nw);
    if (prev == old) return have + 1u;
    old = prev;
  }
  atomicOr(&g_status, kStatusTimeout);
  return 0u;
}

// resident CTAs per SM the register allocation must allow (65536 / (128 x registers))
constexpr int decode_min_blocks(int gmax) { return gmax == 1 ? 9 : gmax == 2 ? 7 : gmax == 4 ? 5 : 3; }

template <int D, int GMAX>
__global__ void __launch_bounds__(128, decode_min_blocks(GMAX)) decode_chunk_kernel(const DecodeParams p) {
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
  __shared__ unsigned s_last;
  __shared__ float s_mrg[2][4];  // the merge's block reductions (maximum, weighted sum)

  const int chunk = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lr = tid % LK, sub = tid / LK, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;
  const int P = p.pos[b];
  if (P < 0 || P >= p.Tmax) {
    // a position out of range: NaN outputs for the sequence's heads, and the status word
    if (chunk == 0) {
      for (int idx = tid; idx < G * D; idx += 128) {
        const int h = hk * G + idx / D;
        p.o[((size_t)b * p.Hq + h) * D + idx % D] = __float2bfloat16(NAN);
        if (idx % D == 0 && p.lse) p.lse[(size_t)b * p.Hq + h] = NAN;
      }
      if (tid == 0 && hk == 0) atomicOr(&g_status, kStatusBadPosition);
    }
    return;
  }
  const int lo = p.window < 0 ? 0 : max(0, P - p.window);
  const int k_begin = lo + chunk * kDecodeChunk;
  if (k_begin > P) return;  // not one of this sequence's chunks: it does not count in
  const int nk = min(P, k_begin + kDecodeChunk - 1) - k_begin + 1;
  // chunks before the last hold 128 cache rows and not the new token: no bounds
  // checks, no row substitution
  const bool full = (k_begin + kDecodeChunk - 1 < P);
  const bool append = p.kn != nullptr;
  const size_t row_stride = (size_t)p.Hkv * D;          // elements between consecutive keys
  const size_t pass_stride = row_stride * KPP;          // between a thread's consecutive rows
  const size_t cache_off = (((size_t)b * p.Tmax + k_begin + sub) * p.Hkv + hk) * D + lr * 8;
  const size_t fresh_off = ((size_t)b * p.Hkv + hk) * D + lr * 8;

  // row kc of the chunk for this thread's pass u: cache row, or the new token at P
  auto load_row = [&](const __nv_bfloat16* cache, const __nv_bfloat16* fresh, int u) {
    const int kc = u * KPP + sub;
    if (full) return ld_stream(cache + cache_off + u * pass_stride);
    if (kc >= nk) return make_uint4(0, 0, 0, 0);
    if (append && k_begin + kc == P) return ld_stream(fresh + fresh_off);
    return ld_stream(cache + cache_off + u * pass_stride);
  };

  // the group's query heads in sub-groups of GMAX (only the widest instantiation sees
  // groups larger than GMAX); a sub-group after the first reads the chunk's rows
  // again, from L2
  constexpr bool kWide = (GMAX == 8);
  for (int g0 = 0; g0 < (kWide ? G : 1); g0 += GMAX) {
    const int gn = kWide ? min(GMAX, G - g0) : G;
    uint32_t qv[GMAX][4];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      const uint4 t = (g < gn)
                          ? *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + hk * G + g0 + g) * D + lr * 8)
                          : make_uint4(0, 0, 0, 0);
      qv[g][0] = t.x, qv[g][1] = t.y, qv[g][2] = t.z, qv[g][3] = t.w;
    }

    // pass 1: scores s = <q, k> * scale * log2(e)
    for (int ps = 0; ps < PASSES; ps += UNROLL) {
      uint4 kv[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) kv[u] = load_row(p.kc, p.kn, ps + u);
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g < gn) {
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
          if (LK == 16) {
            const float sum = reduce8x16(d, lr);
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
      if (g < gn) {
        float v = tid < nk ? s_sc[g][tid] : -INFINITY;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) s_red[g][warp] = v;
      }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < gn) {
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
    if (tid < gn) s_stat[tid][1] = s_acc[0][tid][0] + s_acc[0][tid][1] + s_acc[0][tid][2] + s_acc[0][tid][3];
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
          if (g < gn) {
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
      if (g < gn)
#pragma unroll
        for (int e = 0; e < 8; ++e) s_acc[sub][g][lr * 8 + e] = acc[g][e];
    __syncthreads();
    for (int idx = tid; idx < gn * D; idx += 128) {
      const int g = idx / D, d = idx % D;
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < KPP; ++k) sum += s_acc[k][g][d];
      float* w = p.ws + (((size_t)b * p.Hq + hk * G + g0 + g) * p.n_chunks + chunk) * (D + 2);
      w[d] = sum;
      if (d == 0) {
        w[D] = s_stat[g][0];
        w[D + 1] = s_stat[g][1];
      }
    }
    __syncthreads();  // s_sc, s_stat and s_acc are reused by the next sub-group
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

  // ------------------------------------------------------------ merge by the last chunk CTA
  // Merge of the chunk partials of each head of the group: weights 2^(m_c - max m),
  // o = sum of the weighted acc / sum of the weighted l, lse; an online pass over the
  // chunks. Partials become visible through each CTA's fence before it counts in.
  const int nc = (P - lo) / kDecodeChunk + 1;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (decode_arrive(p.counters + (size_t)b * p.Hkv + hk, p.epoch) == (unsigned)nc) ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // per head: the chunk statistics first (one round of independent loads into shared
  // memory), then every dimension's weighted sum, its loads issued 8 chunks at a time
  float* s_f = &s_sc[0][0];  // chunk weights 2^(m_c - M), up to kDecodeChunk at a time
  for (int g = 0; g < G; ++g) {
    const int h = hk * G + g;
    const float* w = p.ws + ((size_t)b * p.Hq + h) * p.n_chunks * (D + 2);
    float M = -INFINITY, Ls = 0.f;
    // maximum over chunks (nc may exceed the block: strided, then a block reduction)
    float mx = -INFINITY;
    for (int c = tid; c < nc; c += 128) mx = fmaxf(mx, __ldcg(w + (size_t)c * (D + 2) + D));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_mrg[0][warp] = mx;
    __syncthreads();
    M = fmaxf(fmaxf(s_mrg[0][0], s_mrg[0][1]), fmaxf(s_mrg[0][2], s_mrg[0][3]));
    __syncthreads();
    float O = 0.f;
    for (int c0 = 0; c0 < nc; c0 += kDecodeChunk) {
      const int cn = min(kDecodeChunk, nc - c0);
      float ls = 0.f;
      if (tid < cn) {
        const float* wc = w + (size_t)(c0 + tid) * (D + 2);
        const float f = ex2_approx(__ldcg(wc + D) - M);
        s_f[tid] = f;
        ls = f * __ldcg(wc + D + 1);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
      if (lane == 0) s_mrg[1][warp] = ls;
      __syncthreads();
      Ls += (s_mrg[1][0] + s_mrg[1][1]) + (s_mrg[1][2] + s_mrg[1][3]);
      if (tid < D) {
        for (int c = 0; c < cn; c += 8) {
          float a[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] = (c + u < cn) ? __ldcg(w + (size_t)(c0 + c + u) * (D + 2) + tid) : 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (c + u < cn) O = fmaf(s_f[c + u], a[u], O);
        }
      }
      __syncthreads();  // s_f and s_mrg are rewritten by the next round
    }
    if (tid < D) p.o[((size_t)b * p.Hq + h) * D + tid] = __float2bfloat16(O / Ls);
    if (tid == 0 && p.lse) p.lse[(size_t)b * p.Hq + h] = (M + __log2f(Ls)) * 0.69314718055994531f;
  }
  if (tid == 0) p.counters[(size_t)b * p.Hkv + hk] = (unsigned long long)p.epoch << 32;  // (epoch, 0)
}

}  // namespace cswa
