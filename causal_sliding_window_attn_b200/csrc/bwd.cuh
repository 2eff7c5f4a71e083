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
//                128-row query tile) that sees the key tile. Per step, all
//                MMAs M = 128, N = 128 (the shape the tensor pipe runs at full
//                rate), TMEM regions R0, R1 of 128 columns each:
//                  S^T  = K Q^T         (SS)  -> R0
//                  P^T  = exp2(S^T c - lse)     bf16 back into R0
//                  dV  += P^T dO        (TS)  -> TMEM [256,256+D)
//                  dP^T = V dO^T        (SS)  -> R1
//                  dS^T = P^T (dP^T - Delta)    bf16 into shared memory
//                  dK  += dS^T Q        (SS)  -> TMEM [256+D,256+2D)
//                  dQ^T = K^T dS^T      (SS, both MN-major) -> R1
//                A drain warpgroup reads dQ^T out of TMEM and adds it to the
//                fp32 accumulator with 128-byte coalesced reductions.
//                dK, dV are complete in the CTA (the whole group is walked
//                here), so they are written once, as bf16, with no atomics.
//   bwd_dq_cast  the fp32 dQ accumulator (B, Hq, Tpad, D) -> bf16 dq (B, T, Hq, D).
// Warp roles in bwd_main: 0 TMA, 1 MMA issuer, 2 TMEM allocator,
// 4-7 P/dS + dK epilogue (thread = key row), 8-11 dQ drain + dV epilogue.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct BwdParams {
  const float* lse2;   // (B, Hq, Tpad): lse * log2(e), +inf on padded rows
  const float* delta;  // (B, Hq, Tpad)
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int T, Tpad, Hq, G, window, n_kv_tiles, n_q_tiles;  // tiles of 128 rows
  float scale, scale_log2;
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// 2-D tiled reduce-add shared -> global (fp32 add in L2), bulk-group completion.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* m, const void* src, int c0, int c1) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int D>
struct BwdLayout {
  static constexpr int kTile = 128 * D * 2;   // one 128-row bf16 tile (K, V, Q or dO)
  static constexpr int kPanel = 128 * 128;    // one 64-column panel of a 128-row tile
  static constexpr int kK = 0;
  static constexpr int kZero = kK + kTile;    // D = 64: zero panel after K (pads K^T to M = 128)
  static constexpr int kV = kZero + (D == 64 ? kPanel : 0);
  static constexpr int kQ = kV + kTile;       // [2]
  static constexpr int kDO = kQ + 2 * kTile;  // [2]
  static constexpr int kDS = kDO + 2 * kTile; // dS^T: 128 keys x 128 queries bf16, 2 panels
  static constexpr int kStat = kDS + 2 * kPanel;  // lse2[2][128], delta[2][128]
  static constexpr int kBar = kStat + 2048;
  static constexpr int kUsed = kBar + 256;
  static constexpr int kBytes = (kUsed + 1024 <= 232448) ? kUsed + 1024 : 232448;
  static_assert(kUsed <= 232448, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    float* __restrict__ dq_acc, const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // the layout needs a 1024-byte aligned base: report (never overrun) if the slack is too small
  if ((smem - smem_raw) + L::kUsed > L::kBytes) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusLayout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;   // [2]
  uint64_t* qd_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* dv_done = bars + 7;
  uint64_t* dp_full = bars + 8;
  uint64_t* ds_full = bars + 9;
  uint64_t* dq_full = bars + 10;
  uint64_t* dq_free = bars + 11;
  uint64_t* final_bar = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);
  float* s_lse = reinterpret_cast<float*>(smem + L::kStat);           // [2][128]
  float* s_delta = reinterpret_cast<float*>(smem + L::kStat + 1024);  // [2][128]

  const int warp = warp_id(), lane = lane_id();
  const int hk = blockIdx.x, b = blockIdx.y, n = blockIdx.z;
  const int W = p.window, G = p.G;
  const int k0 = n * 128;
  const int m_hi = (W < 0) ? p.n_q_tiles - 1 : min(p.n_q_tiles - 1, (k0 + 127 + W) / 128);
  const int m_cnt = m_hi - n + 1;
  const int n_iters = G * m_cnt;

  if (D == 64) {
    for (int i = threadIdx.x; i < L::kPanel / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(smem + L::kZero)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(dv_done, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 128);
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
  // R0: S^T, then P^T (bf16) in its first 64 columns; R1: dP^T, then dQ^T
  const uint32_t tR0 = tmem, tR1 = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  const uint32_t sbase = smem_u32(smem);
  auto iter_head = [&](int it) { return hk * G + it / m_cnt; };
  auto iter_q0 = [&](int it) { return (n + it % m_cnt) * 128; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
      for (int pn = 0; pn < D / 64; ++pn) {
        tma_load_4d(smem + L::kK + pn * L::kPanel, &tm_k, kv_full, pn * 64, hk, k0, b);
        tma_load_4d(smem + L::kV + pn * L::kPanel, &tm_v, kv_full, pn * 64, hk, k0, b);
      }
      int last_issue[2] = {-1, -1};
      for (int it = 0; it < n_iters; ++it) {
        const int st = it & 1;
        const int h = iter_head(it), q0 = iter_q0(it);
        CSWA_MARK(3, it, 0);
        if (!mbar_wait(&qd_empty[st], ((it >> 1) & 1) ^ 1, abort_flag)) break;
        CSWA_MARK(3, it, 1);
        mbar_arrive_expect_tx(&qd_full[st], 2 * L::kTile + 1024);
        for (int pn = 0; pn < D / 64; ++pn) {
          tma_load_4d(smem + L::kQ + st * L::kTile + pn * L::kPanel, &tm_q, &qd_full[st], pn * 64, h, q0, b);
          tma_load_4d(smem + L::kDO + st * L::kTile + pn * L::kPanel, &tm_do, &qd_full[st], pn * 64, h, q0, b);
        }
        const size_t row0 = ((size_t)b * p.Hq + h) * p.Tpad + q0;
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
      constexpr uint32_t idQ = idesc_bf16(128, 128, true, true);     // dQ^T: A and B MN-major
      // Descriptors are built once; an MMA only adds (byte offset >> 4) to the start field.
      const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024), dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);
      const uint64_t dK_mn = sdesc_sw128(sbase + L::kK, L::kPanel, 1024);
      const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024), dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kPanel, 1024);
      const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kPanel, 1024);
      const uint64_t dDS_k = sdesc_sw128(sbase + L::kDS, 16, 1024);
      const uint64_t dDS_mn = sdesc_sw128(sbase + L::kDS, L::kPanel, 1024);
      // step it reads Q/dO stage it & 1
      auto issue_S = [&](int it) {
        const uint32_t qo = (it & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
          mma_ss(tR0, dK_k + (off >> 4), dQ_k + ((qo + off) >> 4), idSP, kk > 0);
        }
        mma_commit(s_full);
      };
      auto issue_dP = [&](int it) {
        const uint32_t qo = (it & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
          mma_ss(tR1, dV_k + (off >> 4), dDO_k + ((qo + off) >> 4), idSP, kk > 0);
        }
        mma_commit(dp_full);
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag) && mbar_wait(&qd_full[0], 0, abort_flag);
      tc_fence_after();
      if (ok && n_iters > 0) {
        issue_S(0);
        issue_dP(0);
      }
      for (int it = 0; ok && it < n_iters; ++it) {
        const int st = it & 1;
        const uint32_t qo = st * L::kTile;
        CSWA_MARK(0, it, 0);
        if (!(ok = mbar_wait(p_full, it & 1, abort_flag))) break;
        CSWA_MARK(0, it, 1);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tdV, tR0 + kk * 8, dDO_mn + ((qo + kk * 2048) >> 4), idKV, (it > 0 || kk > 0));
        mma_commit(dv_done);
        if (it + 1 < n_iters) {
          // S^T of the next step overwrites P^T: wait until dV has read it
          if (!(ok = mbar_wait(&qd_full[st ^ 1], ((it + 1) >> 1) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(dv_done, it & 1, abort_flag))) break;
          tc_fence_after();
          issue_S(it + 1);
          CSWA_MARK(0, it, 2);
        }
        if (!(ok = mbar_wait(ds_full, it & 1, abort_flag))) break;
        CSWA_MARK(0, it, 3);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tdK, dDS_k + (((kk >> 2) * L::kPanel + (kk & 3) * 32) >> 4), dQ_mn + ((qo + kk * 2048) >> 4),
                 idKV, (it > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tR1, dK_mn + ((kk * 2048) >> 4), dDS_mn + ((kk * 2048) >> 4), idQ, kk > 0);
        CSWA_MARK(0, it, 4);
        mma_commit(dq_full);
        mma_commit(&qd_empty[st]);
        if (it + 1 < n_iters) {
          // dP^T of the next step goes where dQ^T is: wait until the drain has read it
          if (!(ok = mbar_wait(dq_free, it & 1, abort_flag))) break;
          tc_fence_after();
          issue_dP(it + 1);
          CSWA_MARK(0, it, 5);
        }
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
      const int q0 = iter_q0(it);
      const float* lse_s = s_lse + st * 128;
      const float* dl_s = s_delta + st * 128;
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 0);
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, it & 1, abort_flag));
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 1);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tR0 + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      tmem_ld_wait();
      const bool full = (k0 + 127 <= q0) && (W < 0 || q0 + 127 - k0 <= W);
      const int c_lo = j - q0;                       // query q0 + c sees key j iff c >= c_lo
      const int c_hi = (W < 0) ? 127 : j + W - q0;   //   and c <= c_hi
      // P^T row in place as packed bf16 pairs (the same bf16 P feeds dV and dS).
      // Masked entries get exponent -inf (ex2 -> 0): no branch around the exponential;
      // tiles inside the band skip the mask (a warp-uniform branch).
      const float4* lse4 = reinterpret_cast<const float4*>(lse_s);
      if (full) {
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const float4 l = lse4[c4];
          sr[2 * c4] = pack_bf16x2(ex2_approx(fmaf(__uint_as_float(sr[4 * c4]), sl2, -l.x)),
                                   ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 1]), sl2, -l.y)));
          sr[2 * c4 + 1] = pack_bf16x2(ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 2]), sl2, -l.z)),
                                       ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 3]), sl2, -l.w)));
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const float4 l = lse4[c4];
          const float lv[4] = {l.x, l.y, l.z, l.w};
          float pv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = 4 * c4 + u;
            const bool vis = (c >= c_lo) & (c <= c_hi);
            pv[u] = ex2_approx(vis ? fmaf(__uint_as_float(sr[c]), sl2, -lv[u]) : -INFINITY);
          }
          sr[2 * c4] = pack_bf16x2(pv[0], pv[1]);
          sr[2 * c4 + 1] = pack_bf16x2(pv[2], pv[3]);
        }
      }
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 6);
      tmem_st32(tR0 + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_st32(tR0 + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 2);

      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, abort_flag));
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 3);
      // dS^T of the previous step must have been consumed by dK and dQ^T
      if (ok && it > 0) ok = __all_sync(0xffffffffu, mbar_wait(dq_full, (it - 1) & 1, abort_flag));
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 4);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dp[32];
        tmem_ld32(tR1 + lane_off + cc * 32, dp);
        tmem_ld_wait();
        const float4* dl4 = reinterpret_cast<const float4*>(dl_s + cc * 32);
        uint32_t w[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 dl = dl4[e4];
          const float2 p0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sr[cc * 16 + 2 * e4]));
          const float2 p1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sr[cc * 16 + 2 * e4 + 1]));
          w[2 * e4] = pack_bf16x2(p0.x * (__uint_as_float(dp[4 * e4]) - dl.x),
                                  p0.y * (__uint_as_float(dp[4 * e4 + 1]) - dl.y));
          w[2 * e4 + 1] = pack_bf16x2(p1.x * (__uint_as_float(dp[4 * e4 + 2]) - dl.z),
                                      p1.y * (__uint_as_float(dp[4 * e4 + 3]) - dl.w));
        }
        // queries cc*32 .. cc*32+31 = 16-byte chunks (cc&1)*4 .. +3 of panel cc/2, 128-byte swizzle
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = (cc & 1) * 4 + u;
          *reinterpret_cast<uint4*>(ds_row + (cc >> 1) * L::kPanel + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
      if (warp == 4 && lane == 0) CSWA_MARK(1, it, 5);
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
    // ------------------------------------------------------------ dQ drain (thread = head-dim index)
    const int quarter = warp & 3;
    const int dd = quarter * 32 + lane;  // d index of this thread's TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_iters; ++it) {
      if (warp == 8 && lane == 0) CSWA_MARK(2, it, 0);
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, it & 1, abort_flag));
      if (warp == 8 && lane == 0) CSWA_MARK(2, it, 1);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tR1 + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(dq_free);
      // dQ[q0 + c][dd] += scale * dQ^T[dd][c]: a warp covers 32 consecutive d, one
      // 128-byte coalesced fp32 reduction per instruction
      if (dd < D) {
        float* dst = dq_acc + (((size_t)b * p.Hq + iter_head(it)) * p.Tpad + iter_q0(it)) * D + dd;
#pragma unroll
        for (int c = 0; c < 128; ++c) atomicAdd(dst + (size_t)c * D, __uint_as_float(v[c]) * p.scale);
      }
      if (warp == 8 && lane == 0) CSWA_MARK(2, it, 2);
    }
    // ---------------------------------------------------------- dV epilogue (thread = key row)
    ok = __all_sync(0xffffffffu, ok && mbar_wait(final_bar, 0, abort_flag));
    tc_fence_after();
    if (ok) {
      const int j = k0 + dd;
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
// arrays, and zeroes the padded dQ accumulator row: D/8 lanes per (b, t, h) row.
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
  }
  if (active) {
    float4* z = reinterpret_cast<float4*>(dq_acc + (((size_t)b * Hq + h) * Tpad + t) * D + lr * 8);
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

// dq (B, T, Hq, D) bf16 <- dq_acc (B, Hq, Tpad, D) fp32; one thread per 8 values.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_cast_kernel(const float* acc, __nv_bfloat16* dq, int T, int Tpad,
                                                                int Hq, long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const int d8 = (int)(i % (D / 8));
  const long long row = i / (D / 8);  // (b, t, h) of the output
  const int h = (int)(row % Hq);
  const long long bt = row / Hq;
  const int t = (int)(bt % T), b = (int)(bt / T);
  const float4* src = reinterpret_cast<const float4*>(acc + (((size_t)b * Hq + h) * Tpad + t) * D + d8 * 8);
  const float4 a = src[0], c = src[1];
  reinterpret_cast<uint4*>(dq)[i] =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
}

}  // namespace cswa
