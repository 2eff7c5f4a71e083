// attn_bwd: gradients of the causal sliding-window GQA attention on tcgen05 / TMEM.
//
// For o = attn_fwd(q, k, v) and an upstream gradient dO (the softmax backward
// of nanoGPT Administrator & Developer Guide, 8 "CausalSelfAttention", which
// nanochat runs through autograd -- nanochat feature spec, "Backward pass"):
//   Delta_i = dO_i . o_i,   P_ij = exp(scale q_i.k_j - lse_i) on the visible band,
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),
//   dQ = scale dS K,  dK = scale dS^T Q,
// dK and dV of a KV head summed over its G = Hq/Hkv query heads.
//
// Three kernels:
//   bwd_prep     Delta_i and lse_i * log2(e) per row into the workspace
//                (padded to 128-row tiles with Delta = 0, lse = +inf so padded
//                rows get P = 0), and zeroes the fp32 dQ accumulator.
//   bwd_main     one CTA per (128-key tile, KV head, batch). K and V stay in
//                shared memory; the CTA walks every (query head of the group,
//                128-row query tile) that sees the key tile. Per step:
//                  S^T  = K Q^T        (SS)   -> TMEM cols [0,128)
//                  dP^T = V dO^T       (SS)   -> TMEM cols [128,256)
//                  P^T  = exp2(S^T*c - lse)   written back as bf16 into [0,64)
//                  dV  += P^T dO       (TS)   -> TMEM (persistent)
//                  dS^T = P^T (dP^T - Delta)  bf16 into shared memory
//                  dK  += dS^T Q       (SS)   -> TMEM (persistent)
//                  dQ   = dS K         (SS, dS read MN-major) -> TMEM [128,128+D)
//                and dQ is added to the fp32 accumulator with vector atomics.
//                dK, dV are complete in the CTA (the whole group is walked here),
//                so they are written once, as bf16, with no atomics.
//   bwd_dq_cast  the fp32 dQ accumulator -> bf16 dq.
// Warp roles in bwd_main: 0 TMA, 1 MMA issuer, 2 TMEM allocator,
// 4-7 P/dS (thread = key row), 8-11 dQ drain (thread = query row).
#pragma once
#include "ptx.cuh"

namespace cswa {

struct BwdParams {
  const float* lse2;   // (B, Hq, Tpad): lse * log2(e), +inf on padded rows
  const float* delta;  // (B, Hq, Tpad)
  float* dq_acc;       // (B, T, Hq, D)
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int T, Tpad, Hq, G, window, n_tiles;
  float scale, scale_log2;
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int D>
struct BwdLayout {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kPanels = D / 64;
  static constexpr int kK = 0, kV = kTile, kQ = 2 * kTile, kDO = 4 * kTile, kDS = 6 * kTile;
  static constexpr int kStat = kDS + 32768;  // lse2[2][128], delta[2][128]
  static constexpr int kBar = kStat + 2048;
  static constexpr int kUsed = kBar + 256;
  static constexpr int kBytes = (kUsed + 1024 <= 232448) ? kUsed + 1024 : 232448;
  static constexpr uint32_t kTmemCols = 512;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // The layout needs a 1024-byte aligned base; report (never corrupt) if the
  // runtime placed dynamic shared memory so that the aligned layout overflows.
  if ((smem - smem_raw) + L::kUsed > L::kBytes) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusLayout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;   // [2]
  uint64_t* qd_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* dp_full = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* ds_full = bars + 8;
  uint64_t* dv_done = bars + 9;
  uint64_t* dq_full = bars + 10;
  uint64_t* dq_free = bars + 11;
  uint64_t* final_bar = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);
  float* s_lse = reinterpret_cast<float*>(smem + L::kStat);          // [2][128]
  float* s_delta = reinterpret_cast<float*>(smem + L::kStat + 1024);  // [2][128]

  const int warp = warp_id(), lane = lane_id();
  const int hk = blockIdx.x, b = blockIdx.y, n = blockIdx.z;
  const int W = p.window, G = p.G;
  const int k0 = n * 128;
  const int m_hi = (W < 0) ? p.n_tiles - 1 : min(p.n_tiles - 1, (k0 + 127 + W) / 128);
  const int m_cnt = m_hi - n + 1;
  const int n_iters = G * m_cnt;

  if (warp == 0 && lane == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 128);
    mbar_init(ds_full, 128);
    mbar_init(dv_done, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + L::kK, sV = sbase + L::kV, sDS = sbase + L::kDS;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
      for (int pn = 0; pn < L::kPanels; ++pn) {
        tma_load_4d(smem + L::kK + pn * 16384, &tm_k, kv_full, pn * 64, hk, k0, b);
        tma_load_4d(smem + L::kV + pn * 16384, &tm_v, kv_full, pn * 64, hk, k0, b);
      }
      int last_issue[2] = {-1, -1};
      for (int it = 0; it < n_iters; ++it) {
        const int st = it & 1;
        const int g = it / m_cnt, m = n + it % m_cnt;
        const int h = hk * G + g;
        if (!mbar_wait(&qd_empty[st], ((it >> 1) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&qd_full[st], 2 * L::kTile + 1024);
        for (int pn = 0; pn < L::kPanels; ++pn) {
          tma_load_4d(smem + L::kQ + st * L::kTile + pn * 16384, &tm_q, &qd_full[st], pn * 64, h, m * 128, b);
          tma_load_4d(smem + L::kDO + st * L::kTile + pn * 16384, &tm_do, &qd_full[st], pn * 64, h, m * 128,
                      b);
        }
        const size_t row0 = ((size_t)b * p.Hq + h) * p.Tpad + (size_t)m * 128;
        bulk_load(s_lse + st * 128, p.lse2 + row0, 512, &qd_full[st]);
        bulk_load(s_delta + st * 128, p.delta + row0, 512, &qd_full[st]);
        last_issue[st] = it;
      }
      if (*abort_flag) {
        volatile int dummy = 0;
        for (int st = 0; st < 2; ++st)
          if (last_issue[st] >= 0) mbar_wait(&qd_full[st], (last_issue[st] >> 1) & 1, &dummy);
        mbar_wait(kv_full, 0, &dummy);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idSP = idesc_bf16(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t idKV = idesc_bf16(128, D, false, true);     // dV (TS), dK: B MN-major
      constexpr uint32_t idQ = idesc_bf16(128, D, true, true);       // dQ: A and B MN-major
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      for (int it = 0; ok && it < n_iters; ++it) {
        const int st = it & 1;
        const uint32_t sQ = sbase + L::kQ + st * L::kTile, sDO = sbase + L::kDO + st * L::kTile;
        if (!(ok = mbar_wait(&qd_full[st], (it >> 1) & 1, abort_flag))) break;
        if (it > 0 && !(ok = mbar_wait(dv_done, (it - 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), idSP, kk > 0);
        }
        mma_commit(s_full);
        if (it > 0 && !(ok = mbar_wait(dq_free, (it - 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tdP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sDO + off, 16, 1024), idSP, kk > 0);
        }
        mma_commit(dp_full);
        if (!(ok = mbar_wait(p_full, it & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tdV, tS + kk * 8, sdesc_sw128(sDO + kk * 2048, 16384, 1024), idKV, (it > 0 || kk > 0));
        mma_commit(dv_done);
        if (!(ok = mbar_wait(ds_full, it & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tdK, sdesc_sw128(sDS + off, 16, 1024), sdesc_sw128(sQ + kk * 2048, 16384, 1024), idKV,
                 (it > 0 || kk > 0));
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tdQ, sdesc_sw128(sDS + kk * 2048, 16384, 1024), sdesc_sw128(sK + kk * 2048, 16384, 1024), idQ,
                 kk > 0);
        mma_commit(dq_full);
        mma_commit(&qd_empty[st]);
      }
      mma_commit(final_bar);
      volatile int dummy = 0;
      mbar_wait(final_bar, 0, &dummy);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ P and dS (thread = key row)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int j = k0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    uint8_t* ds_row = smem + L::kDS + r * 128;
    bool ok = true;
    for (int it = 0; it < n_iters; ++it) {
      const int st = it & 1;
      const int q0 = (n + it % m_cnt) * 128;
      const float* lse_s = s_lse + st * 128;
      const float* dl_s = s_delta + st * 128;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tS + lane_off + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tS + lane_off + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_ld_wait();
      const bool full = (k0 + 127 <= q0) && (W < 0 || q0 + 127 - k0 <= W);
      // P^T row in place as packed bf16 pairs; the same bf16 P feeds dV (TMEM) and dS
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int i = q0 + 2 * c;
        const bool v0 = full || ((j <= i) && (W < 0 || i - j <= W));
        const bool v1 = full || ((j <= i + 1) && (W < 0 || i + 1 - j <= W));
        const float p0 = v0 ? ex2_approx(fmaf(__uint_as_float(sr[2 * c]), sl2, -lse_s[2 * c])) : 0.f;
        const float p1 = v1 ? ex2_approx(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -lse_s[2 * c + 1])) : 0.f;
        sr[c] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_st32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);

      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, abort_flag));
      if (ok && it > 0) ok = __all_sync(0xffffffffu, mbar_wait(dq_full, (it - 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dp[32];
        tmem_ld32(tdP + lane_off + cc * 32, dp);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = cc * 32 + 2 * e;
          const float2 pp = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sr[cc * 16 + e]));
          const float d0 = pp.x * (__uint_as_float(dp[2 * e]) - dl_s[c0]);
          const float d1 = pp.y * (__uint_as_float(dp[2 * e + 1]) - dl_s[c0 + 1]);
          w[e] = pack_bf16x2(d0, d1);
        }
        // queries cc*32 .. cc*32+31 = 4 16-byte chunks of panel cc/2, chunks (cc&1)*4 ..
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = (cc & 1) * 4 + u;
          uint4* dst = reinterpret_cast<uint4*>(ds_row + (cc >> 1) * 16384 + ((chunk ^ (r & 7)) << 4));
          *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // ---------------------------------------------------------- dK epilogue
    ok = __all_sync(0xffffffffu, ok && mbar_wait(final_bar, 0, abort_flag));
    tc_fence_after();
    if (ok) {
      __nv_bfloat16* dst = p.dk + ((size_t)((size_t)b * p.T + j) * (p.Hq / G) + hk) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tdK + lane_off + c * 32, o);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * p.scale, __uint_as_float(o[2 * e + 1]) * p.scale);
        if (j < p.T) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) d4[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dQ drain (thread = query row)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_iters; ++it) {
      const int g = it / m_cnt;
      const int i = (n + it % m_cnt) * 128 + row;
      const int h = hk * G + g;
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float* dst = p.dq_acc + ((size_t)((size_t)b * p.T + i) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tdQ + lane_off + c * 32, o);
        tmem_ld_wait();
        if (i < p.T) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float4 v = make_float4(__uint_as_float(o[4 * u]) * p.scale, __uint_as_float(o[4 * u + 1]) * p.scale,
                                   __uint_as_float(o[4 * u + 2]) * p.scale, __uint_as_float(o[4 * u + 3]) * p.scale);
            atomicAdd(reinterpret_cast<float4*>(dst + c * 32 + 4 * u), v);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(dq_free);
    }
    // ---------------------------------------------------------- dV epilogue (thread = key row)
    ok = __all_sync(0xffffffffu, ok && mbar_wait(final_bar, 0, abort_flag));
    tc_fence_after();
    if (ok) {
      const int j = k0 + row;
      __nv_bfloat16* dst = p.dv + ((size_t)((size_t)b * p.T + j) * (p.Hq / G) + hk) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tdV + lane_off + c * 32, o);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
        if (j < p.T) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) d4[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Delta_i = dO_i . o_i and lse_i * log2(e) into the padded (B, Hq, Tpad) workspace
// arrays, and zeroes the dQ accumulator row: D/8 lanes per (b, t, h) row.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                             const float* lse, float* lse2, float* delta,
                                                             float* dq_acc, int B, int T, int Tpad, int Hq) {
  constexpr int LK = D / 8;
  const long long rows = (long long)B * Tpad * Hq;
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gtid / LK;
  const int lr = (int)(gtid % LK);
  const bool active = row < rows;
  // row enumerates (b, t, h) with t over the padded length
  const int h = active ? (int)(row % Hq) : 0;
  const long long bt = active ? row / Hq : 0;
  const int t = (int)(bt % Tpad), b = (int)(bt / Tpad);
  const bool real = active && t < T;
  float dsum = 0.f;
  if (real) {
    const size_t off = ((size_t)((size_t)b * T + t) * Hq + h) * D + lr * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(o + off);
    const uint4 gv = *reinterpret_cast<const uint4*>(dout + off);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 a = __bfloat1622float2(o2[u]), c = __bfloat1622float2(g2[u]);
      dsum = fmaf(a.x, c.x, fmaf(a.y, c.y, dsum));
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int s = LK / 2; s >= 1; s >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, s);
  if (active && lr == 0) {
    const size_t so = ((size_t)b * Hq + h) * Tpad + t;
    delta[so] = real ? dsum : 0.f;
    lse2[so] = real ? lse[((size_t)b * Hq + h) * T + t] * 1.4426950408889634f : INFINITY;
  }
}

__global__ void __launch_bounds__(256) attn_bwd_dq_cast_kernel(const float* acc, __nv_bfloat16* dq, long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  reinterpret_cast<uint4*>(dq)[i] =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
}

}  // namespace cswa
