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
//                rows get P = 0).
//   bwd_main     one CTA per (128-key tile, KV head, batch). K and V stay in
//                shared memory; the CTA walks every (query head of the group,
//                128-row query tile) that sees the key tile. Per step, all
//                MMAs M = 128, N = 128 (the shape the tensor pipe runs at full
//                rate), TMEM regions R0, R1 of 128 columns each:
//                  S^T  = K Q^T         (SS)  -> R0
//                  P^T  = exp2(S^T c - lse)     bf16 back over the S^T it came from
//                  dV  += P^T dO        (TS)  -> TMEM [256,256+D)
//                  dP^T = V dO^T        (SS)  -> R1
//                  dS^T = P^T (dP^T - Delta)    bf16 into shared memory
//                  dK  += dS^T Q        (SS)  -> TMEM [256+D,256+2D)
//                and the dS^T tile goes to the workspace with one TMA store.
//                Two warpgroups split the elementwise work by query columns.
//                dK, dV are complete in the CTA (the whole group is walked
//                here), so they are written once, as bf16, with no atomics.
//   bwd_dq       one CTA per (128-row query tile, query head, batch):
//                dQ = scale * sum over key tiles of dS K, accumulated in TMEM
//                from the stored dS^T tiles and K tiles, written once as bf16.
// Splitting dQ out keeps the per-step fp32 reductions of dQ out of the main
// kernel's load/store pipe, which its elementwise warps need.
// Warp roles in bwd_main: 0 TMA, 1 MMA issuer, 2 TMEM allocator, 3 dS store,
// 4-7 and 8-11 P/dS (thread = key row; columns 0-63 and 64-127), then the
// dK and dV epilogues.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct BwdParams {
  const float* lse2;   // (B, Hq, Tpad): lse * log2(e), +inf on padded rows
  const float* delta;  // (B, Hq, Tpad)
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  __nv_bfloat16* dq;
  int T, Tpad, Hq, G, window, n_tiles, span;  // tiles of 128 rows; span = query tiles per key tile
  long long tiles_per_bh;                     // stored dS^T tiles per (batch, query head)
  float scale, scale_log2;
};

// Query tiles that see key tile n: [n, n + min(n_tiles - n, span) - 1], where
// span = n_tiles (no window) or floor((127 + W) / 128) + 1. The dS^T tiles of
// one (batch, head) are stored key tile by key tile; this is where key tile n starts.
__host__ __device__ inline int bwd_span(int n_tiles, int window) {
  return window < 0 ? n_tiles : min(n_tiles, (127 + window) / 128 + 1);
}
__host__ __device__ inline long long ds_tiles_before(int n, int n_tiles, int span) {
  const int a = max(0, n_tiles - span);  // key tiles whose whole span fits
  if (n <= a) return (long long)n * span;
  const long long hi = n_tiles - a, lo = n_tiles - n + 1;  // sum of (n_tiles - n') for n' in [a, n)
  return (long long)a * span + (hi + lo) * (hi - lo + 1) / 2;
}

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
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
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
  static constexpr int kV = kK + kTile;
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
                    const __grid_constant__ CUtensorMap tm_ds, const BwdParams p) {
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
  uint64_t* ds_free = bars + 10;
  uint64_t* final_bar = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 13);
  float* s_lse = reinterpret_cast<float*>(smem + L::kStat);           // [2][128]
  float* s_delta = reinterpret_cast<float*>(smem + L::kStat + 1024);  // [2][128]

  const int warp = warp_id(), lane = lane_id();
  const int hk = blockIdx.x, b = blockIdx.y, n = blockIdx.z;
  const int W = p.window, G = p.G;
  const int k0 = n * 128;
  const int m_cnt = min(p.n_tiles - n, p.span);
  const int n_iters = G * m_cnt;

  if (warp == 0 && lane == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(dv_done, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 2);  // dK has read dS^T (MMA commit) + the TMA store has read it
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
  // R0: S^T, then P^T (bf16) in columns 0-31 and 64-95; R1: dP^T
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
      // Descriptors are built once; an MMA only adds (byte offset >> 4) to the start field.
      const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024), dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);
      const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024), dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kPanel, 1024);
      const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kPanel, 1024);
      const uint64_t dDS_k = sdesc_sw128(sbase + L::kDS, 16, 1024);
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
        for (int kk = 0; kk < 8; ++kk)  // P^T of queries 16kk..16kk+15: columns 64*(kk/4) + 8*(kk%4)
          mma_ts(tdV, tR0 + (kk >> 2) * 64 + (kk & 3) * 8, dDO_mn + ((qo + kk * 2048) >> 4), idKV,
                 (it > 0 || kk > 0));
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
        mma_commit(ds_free);
        mma_commit(&qd_empty[st]);
        CSWA_MARK(0, it, 4);
        // dP^T of the next step: the P/dS warps read this step's dP^T before ds_full
        if (it + 1 < n_iters) {
          issue_dP(it + 1);
          CSWA_MARK(0, it, 5);
        }
      }
      mma_commit(final_bar);
      volatile int dummy = 0;
      mbar_wait(final_bar, 0, &dummy);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ dS^T tile store
    if (lane == 0) {
      tma_prefetch_desc(&tm_ds);
      const long long base = ((long long)b * p.Hq) * p.tiles_per_bh + ds_tiles_before(n, p.n_tiles, p.span);
      for (int it = 0; it < n_iters; ++it) {
        if (!mbar_wait(ds_full, it & 1, abort_flag)) break;
        CSWA_MARK(3, it, 2);
        const int h = iter_head(it);
        const long long tile = base + (long long)h * p.tiles_per_bh + it % m_cnt;
        const int row = (int)(tile * 128);
        tma_store_2d(&tm_ds, smem + L::kDS, 0, row);
        tma_store_2d(&tm_ds, smem + L::kDS + L::kPanel, 64, row);
        bulk_commit();
        bulk_wait_read<0>();
        CSWA_MARK(3, it, 3);
        mbar_arrive(ds_free);
      }
      bulk_wait_all();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P and dS (thread = key row)
    // warps 4-7 take query columns 0-63, warps 8-11 columns 64-127 (warp 2 only allocates TMEM)
    const int half = (warp >= 8) ? 1 : 0;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int j = k0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    uint8_t* ds_row = smem + L::kDS + half * L::kPanel + r * 128;
    const bool tracer = (warp == 4 && lane == 0);
    const bool tracer1 = (warp == 8 && lane == 0);
    bool ok = true;
    for (int it = 0; it < n_iters; ++it) {
      const int st = it & 1;
      const int q0 = iter_q0(it) + 64 * half;  // first query of this thread's columns
      const float* lse_s = s_lse + st * 128 + 64 * half;
      const float* dl_s = s_delta + st * 128 + 64 * half;
      if (tracer) CSWA_MARK(1, it, 0);
      if (tracer1) CSWA_MARK(2, it, 0);
      // the lse/Delta rows of this stage come from a bulk copy: acquire them from its
      // own barrier (completion of S^T alone does not order that copy before our reads)
      ok = __all_sync(0xffffffffu, mbar_wait(&qd_full[st], (it >> 1) & 1, abort_flag) &&
                                       mbar_wait(s_full, it & 1, abort_flag));
      if (tracer) CSWA_MARK(1, it, 1);
      if (tracer1) CSWA_MARK(2, it, 1);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tR0 + lane_off + 64 * half + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tR0 + lane_off + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait();
      // debug dump layout: [it][half][r][kind][64]
#define DBG_SLOT(kind, c) ((((it * 2 + half) * 128 + r) * 5 + (kind)) * 64 + (c))
      if (it < 3) {
#pragma unroll
        for (int c = 0; c < 64; ++c) CSWA_DUMP(DBG_SLOT(0, c), __uint_as_float(sr[c]));
#pragma unroll
        for (int c = 0; c < 64; ++c) CSWA_DUMP(DBG_SLOT(1, c), lse_s[c]);
      }
      const bool full = (k0 + 127 <= q0) && (W < 0 || q0 + 63 - k0 <= W);
      const int c_lo = j - q0;                      // query q0 + c sees key j iff c >= c_lo
      const int c_hi = (W < 0) ? 63 : j + W - q0;   //   and c <= c_hi
      // P^T in place as packed bf16 pairs (the same bf16 P feeds dV and dS).
      // Masked entries get exponent -inf (ex2 -> 0): no branch around the exponential;
      // tiles inside the band skip the mask (a warp-uniform branch).
      const float4* lse4 = reinterpret_cast<const float4*>(lse_s);
      if (full) {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l = lse4[c4];
          sr[2 * c4] = pack_bf16x2(ex2_approx(fmaf(__uint_as_float(sr[4 * c4]), sl2, -l.x)),
                                   ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 1]), sl2, -l.y)));
          sr[2 * c4 + 1] = pack_bf16x2(ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 2]), sl2, -l.z)),
                                       ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 3]), sl2, -l.w)));
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
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
      if (tracer) CSWA_MARK(1, it, 6);
      if (tracer1) CSWA_MARK(2, it, 6);
      // P^T of this warpgroup's 64 queries goes over the first half of its own S^T
      // columns (64*half .. 64*half+31), which only this warpgroup has read
      tmem_st32(tR0 + lane_off + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      if (tracer) CSWA_MARK(1, it, 2);
      if (tracer1) CSWA_MARK(2, it, 2);

      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, abort_flag));
      if (tracer) CSWA_MARK(1, it, 3);
      if (tracer1) CSWA_MARK(2, it, 3);
      // dS^T of the previous step must have been read by dK and by its TMA store
      if (ok && it > 0) ok = __all_sync(0xffffffffu, mbar_wait(ds_free, (it - 1) & 1, abort_flag));
      if (tracer) CSWA_MARK(1, it, 4);
      if (tracer1) CSWA_MARK(2, it, 4);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dp[32];
        tmem_ld32(tR1 + lane_off + 64 * half + cc * 32, dp);
        tmem_ld_wait();
        const float4* dl4 = reinterpret_cast<const float4*>(dl_s + cc * 32);
        if (it < 3) {
#pragma unroll
          for (int e = 0; e < 32; ++e) CSWA_DUMP(DBG_SLOT(2, cc * 32 + e), __uint_as_float(dp[e]));
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 pp = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sr[cc * 16 + e]));
            CSWA_DUMP(DBG_SLOT(3, cc * 32 + 2 * e), pp.x);
            CSWA_DUMP(DBG_SLOT(3, cc * 32 + 2 * e + 1), pp.y);
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) CSWA_DUMP(DBG_SLOT(4, cc * 32 + e), dl_s[cc * 32 + e]);
        }
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
        // this warpgroup's panel, queries cc*32 .. cc*32+31 = 16-byte chunks cc*4 .. cc*4+3
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = cc * 4 + u;
          *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
      if (tracer) CSWA_MARK(1, it, 5);
      if (tracer1) CSWA_MARK(2, it, 5);
    }
    // ---------------------------------------------------------- dK (warps 4-7) / dV (8-11) epilogue
    ok = __all_sync(0xffffffffu, ok && mbar_wait(final_bar, 0, abort_flag));
    tc_fence_after();
    if (ok) {
      const uint32_t src = half ? tdV : tdK;
      const float mul = half ? 1.f : p.scale;
      __nv_bfloat16* dst = (half ? p.dv : p.dk) + ((size_t)((size_t)b * p.T + j) * (p.Hq / G) + hk) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(src + lane_off + c * 32, o);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * mul, __uint_as_float(o[2 * e + 1]) * mul);
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

// dQ = scale * sum_n dS(m, n) K_n for one 128-row query tile m of one query head,
// from the dS^T tiles bwd_main stored; accumulated in TMEM, written once as bf16.
template <int D>
struct DqLayout {
  static constexpr int kStages = 3;
  static constexpr int kDS = 32768;            // one dS^T tile (128 keys x 128 queries bf16)
  static constexpr int kK = 128 * D * 2;       // one K tile
  static constexpr int kStage = kDS + kK;
  static constexpr int kBar = kStages * kStage;
  static constexpr int kBytes = kBar + 256 + 1024;
  static constexpr uint32_t kTmemCols = D < 32 ? 32 : D;
};

template <int D>
__global__ void __launch_bounds__(256, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ds,
                       const BwdParams p) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* full = bars;                  // [kStages]
  uint64_t* empty = bars + L::kStages;    // [kStages]
  uint64_t* done = bars + 2 * L::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * L::kStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * L::kStages + 2);

  const int warp = warp_id(), lane = lane_id();
  const int h = blockIdx.x, b = blockIdx.y, m = blockIdx.z;
  const int hk = h / p.G;
  // key tiles n whose query range [n, n + span - 1] holds m
  const int n_lo = max(0, m - p.span + 1);
  const int steps = m - n_lo + 1;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
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
  const uint32_t sbase = smem_u32(smem);
  const long long bh_base = ((long long)b * p.Hq + h) * p.tiles_per_bh;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_ds);
      int last_issue[L::kStages];
      for (int s = 0; s < L::kStages; ++s) last_issue[s] = -1;
      for (int i = 0; i < steps; ++i) {
        const int st = i % L::kStages;
        const int n = n_lo + i;
        if (!mbar_wait(&empty[st], ((i / L::kStages) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], L::kDS + L::kK);
        const int row = (int)((bh_base + ds_tiles_before(n, p.n_tiles, p.span) + (m - n)) * 128);
        uint8_t* dst = smem + st * L::kStage;
        tma_load_2d(dst, &tm_ds, &full[st], 0, row);
        tma_load_2d(dst + 16384, &tm_ds, &full[st], 64, row);
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(dst + L::kDS + pn * 16384, &tm_k, &full[st], pn * 64, hk, n * 128, b);
        last_issue[st] = i;
      }
      if (*abort_flag) {
        volatile int dummy = 0;
        for (int s = 0; s < L::kStages; ++s)
          if (last_issue[s] >= 0) mbar_wait(&full[s], (last_issue[s] / L::kStages) & 1, &dummy);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id = idesc_bf16(128, D, true, true);  // A = dS (queries contiguous), B = K (d contiguous)
      bool ok = true;
      for (int i = 0; ok && i < steps; ++i) {
        const int st = i % L::kStages;
        if (!(ok = mbar_wait(&full[st], (i / L::kStages) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t sds = sbase + st * L::kStage, sk = sds + L::kDS;
        const uint64_t da = sdesc_sw128(sds, 16384, 1024), db = sdesc_sw128(sk, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(tmem, da + ((kk * 2048) >> 4), db + ((kk * 2048) >> 4), id, (i > 0 || kk > 0));
        mma_commit(&empty[st]);
      }
      mma_commit(done);
      volatile int dummy = 0;
      mbar_wait(done, 0, &dummy);
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int i = m * 128 + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag));
    tc_fence_after();
    if (ok) {
      __nv_bfloat16* dst = p.dq + ((size_t)((size_t)b * p.T + i) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + c * 32, o);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * p.scale, __uint_as_float(o[2 * e + 1]) * p.scale);
        if (i < p.T) {
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
// arrays: D/8 lanes per (b, t, h) row.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                             const float* lse, float* lse2, float* delta, int B,
                                                             int T, int Tpad, int Hq) {
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
#pragma unroll
  for (int s = LK / 2; s >= 1; s >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, s);
  if (active && lr == 0) {
    const size_t so = ((size_t)b * Hq + h) * Tpad + t;
    delta[so] = real ? dsum : 0.f;
    lse2[so] = real ? lse[((size_t)b * Hq + h) * T + t] * 1.4426950408889634f : INFINITY;
  }
}

}  // namespace cswa
