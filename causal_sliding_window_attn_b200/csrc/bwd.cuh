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
// Three kernels, all on the caller's stream:
//   bwd_prep     per query row: -lse_i/scale and -Delta_i as bf16 hi + lo pairs laid
//                out as one extra K = 16 step of an MMA (padded rows: a large negative
//                lse term, so P = 0 there); zeroes the fp32 dQ accumulator and the
//                work counter; for the fused block backward, the cos/sin table of the
//                rotary angles.
//   bwd_main     persistent, one CTA per SM, taking (128-key tile, KV head, batch)
//                items from a global counter. For an item, dK and dV accumulate in
//                tensor memory while the CTA walks every (query head of the group,
//                128-row query tile) that sees the key tile. Per step, every MMA has
//                M = 128 (the shape the tensor pipe runs at full rate):
//                  S^T' = K Q^T - lse/scale    (SS, + extension step)  -> X
//                  P^T  = exp2(c S^T')         bf16 pairs over X          (warpgroup A)
//                  dP^T'= V dO^T - Delta       (SS, + extension step)  -> Y
//                  dS^T = P^T dP^T'            bf16 tile in shared memory (warpgroup B)
//                  dV  += P^T dO               (TS: A from X)
//                  dK  += dS^T Q               (SS: the dS^T tile, K-major)
//                  dQ_m = dS K                 (SS: the same tile read MN-major) -> Y
//                and warpgroup B adds dQ_m into the fp32 accumulator with 16-byte
//                reductions in L2. dK and dV are complete in the CTA, so they are
//                written once, as bf16, with no atomics; with the fused prologue, the
//                dK epilogue applies the prologue backward on the way out.
//   bwd_dq       dq = scale * dQ accumulator as bf16 (with the fused prologue, the
//                prologue backward of q applied per row). HBM-bound.
// Tensor memory (512 columns): X = S^T / P^T, Y = dP^T / dQ_m, dV, dK. The one shared
// dS^T tile serves both dK and dQ_m. Warp roles in bwd_main: 0 TMA (K, Q ring),
// 1 MMA issuer (whole warp, one elected lane issues), 2 TMEM allocator and work
// scheduler, 3 TMA (V, dO), 4-7 warpgroup A (P; dV epilogue), 8-11 warpgroup B
// (dS, dQ reductions; dK epilogue). Thread i of a warpgroup owns TMEM lane i.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct BwdParams {
  // per (batch, query head, 128-row query tile): 512 bytes holding -lse/scale and
  // -Delta of the tile's rows as bf16 hi + lo pairs, laid out as the extra K = 16 step
  // of the S^T and dP^T MMAs reads them (see attn_bwd_prep_kernel)
  const uint8_t* ext_lse;
  const uint8_t* ext_delta;
  float* dq_acc;       // (B, T, Hq, D) fp32: sum of dS K over key tiles (zeroed by the prep kernel)
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int* item_counter;   // next work item of the main kernel (zeroed by the prep kernel)
  int T, Tpad, Hq, G, window, n_tiles, span;  // tiles of 128 rows; span = query tiles per key tile
  float scale, scale_log2;
  // fused prologue backward (dk with respect to the raw k); k_raw is null otherwise
  const __nv_bfloat16* k_raw;
  const float2* rope_cs;  // (T, D/2): (cos, sin) of t * omega_j
  float eps;
};

// Query tiles that see key tile n: [n, n + min(n_tiles - n, span) - 1], where
// span = n_tiles (no window) or floor((127 + W) / 128) + 1.
__host__ __device__ inline int bwd_span(int n_tiles, int window) {
  return window < 0 ? n_tiles : min(n_tiles, (127 + window) / 128 + 1);
}

// Work-item order of the persistent backward kernel. Items are (tile t, block blk)
// pairs, blk = (head, batch) block of n_blocks, t of n_tiles; a tile's weight falls
// as t grows. Blocks are taken 8 at a time (a super-block) and, inside one, the tile
// index is the slow one: the heaviest tiles of 8 blocks first, then the next ones.
// Handed out first come first served, this ends every super-block (and the whole
// run) with the lightest items, while the CTAs running at the same time share the
// tiles of those 8 blocks in L2.
__host__ __device__ inline void sb_order(int item, int n_tiles, int n_blocks, int& t, int& blk) {
  constexpr int kSB = 8;
  const int s = item / (kSB * n_tiles);
  const int w = min(kSB, n_blocks - kSB * s);
  const int r = item - kSB * n_tiles * s;
  t = r / w;
  blk = kSB * s + r % w;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Prologue backward of one row held whole by one thread (nanochat Admin & Developer
// Guide, 3: RMS-norm without weight, then RoPE). dy_chunk(c0, v) fills v with elements
// c0 .. c0+15 of the gradient with respect to the prologue output (fp32); x is the raw
// row (bf16), cs[j] = (cos, sin) of the row's angle for pair (j, j + D/2). Writes
//   dx = (g - xh (g . xh) / D) / r,  r = sqrt(mean(x^2) + eps),  xh = x / r,
// g = dy rotated by -phi, as bf16 to dst when `store` is set. dy is asked for twice per
// element (a dot product pass, then the output pass) so that no full row of it stays in
// registers. Every lane of a warp runs the same steps (dy_chunk may be warp-collective);
// a lane with nothing to store passes store = false and any valid x and cs rows.
template <int D, typename DyChunk>
__device__ __forceinline__ void prologue_bwd_row(DyChunk&& dy_chunk, const __nv_bfloat16* x,
                                                 const float2* cs, float eps, __nv_bfloat16* dst, bool store) {
  constexpr int H = D / 2;
  // the raw row: the sum of squares first, then re-read (from L1) chunk by chunk
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < D / 8; ++v) {
    const uint4 t = *reinterpret_cast<const uint4*>(x + 8 * v);
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float lo = __uint_as_float(w[u] << 16), hi = __uint_as_float(w[u] & 0xffff0000u);
      ss = fmaf(lo, lo, fmaf(hi, hi, ss));
    }
  }
  const float inv_r = rsqrtf(ss * (1.f / D) + eps);
  auto x16 = [&](int c0, float (&v)[16]) {
    const uint4 t0 = *reinterpret_cast<const uint4*>(x + c0), t1 = *reinterpret_cast<const uint4*>(x + c0 + 8);
    const uint32_t w[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      v[2 * u] = __uint_as_float(w[u] << 16) * inv_r;
      v[2 * u + 1] = __uint_as_float(w[u] & 0xffff0000u) * inv_r;
    }
  };
  float dot = 0.f;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const float proj = dot * (1.f / D);
#pragma unroll 1
    for (int c0 = 0; c0 < H; c0 += 16) {
      float a[16], b[16], xa[16], xb[16];
      dy_chunk(c0, a);      // elements c0 .. c0+15
      dy_chunk(H + c0, b);  // elements H + c0 .. H + c0 + 15
      x16(c0, xa);
      x16(H + c0, xb);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float2 t = cs[c0 + u];
        const float ga = fmaf(b[u], t.y, a[u] * t.x);
        const float gb = fmaf(-a[u], t.y, b[u] * t.x);
        if (pass == 0) {
          dot = fmaf(ga, xa[u], fmaf(gb, xb[u], dot));
        } else {
          a[u] = (ga - xa[u] * proj) * inv_r;
          b[u] = (gb - xb[u] * proj) * inv_r;
        }
      }
      if (pass == 1 && store) {
        uint32_t oa[8], ob[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          oa[u] = pack_bf16x2(a[2 * u], a[2 * u + 1]);
          ob[u] = pack_bf16x2(b[2 * u], b[2 * u + 1]);
        }
        uint4* da = reinterpret_cast<uint4*>(dst + c0);
        uint4* db = reinterpret_cast<uint4*>(dst + H + c0);
        da[0] = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        da[1] = make_uint4(oa[4], oa[5], oa[6], oa[7]);
        db[0] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
        db[1] = make_uint4(ob[4], ob[5], ob[6], ob[7]);
      }
    }
  }
}

template <int D>
struct BwdLayout {
  static constexpr int kQStages = 2;
  static constexpr int kTile = 128 * D * 2;   // one 128-row bf16 tile (K, V, Q or dO)
  static constexpr int kPanel = 128 * 128;    // one 64-column panel of a 128-row tile
  static constexpr int kK = 0;                            // [2]: consecutive items alternate
  static constexpr int kV = kK + 2 * kTile;
  static constexpr int kQ = kV + kTile;                   // [kQStages]
  static constexpr int kDO = kQ + kQStages * kTile;       // one stage
  static constexpr int kDS = kDO + kTile;                 // dS^T: 128 keys x 128 queries, two panels
  // per-row extension slots (512 bytes, see the prep kernel) of the Q stages, then of
  // the dO stage, then the constant key-side extension (a core of ones, a core of zeros)
  static constexpr int kExt = kDS + 2 * kPanel;
  static constexpr int kExtOnes = kExt + (kQStages + 1) * 512;
  static constexpr int kBar = kExtOnes + 256;
  static constexpr int kUsed = kBar + 256;
  static constexpr int kBytes = (kUsed + 1024 <= 232448) ? kUsed + 1024 : 232448;
  static_assert(kUsed <= 232448, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p, int n_items) {
  using L = BwdLayout<D>;
  constexpr int QS = L::kQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // the layout needs a 1024-byte aligned base: report (never overrun) if the slack is too small
  if ((smem - smem_raw) + L::kUsed > L::kBytes) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusLayout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* k_full = bars + 0;        // [2]
  uint64_t* k_empty = bars + 2;       // [2] the item's last S^T and dQ have read K
  uint64_t* v_full = bars + 4;
  uint64_t* v_empty = bars + 5;       // the item's last dP^T has read V
  uint64_t* q_full = bars + 6;        // [QS]
  uint64_t* q_empty = bars + 8;       // [QS] S^T and dK have read the Q stage
  uint64_t* do_full = bars + 10;
  uint64_t* do_empty = bars + 11;     // dP^T and dV have read dO
  uint64_t* s_full = bars + 12;       // S^T in X
  uint64_t* p_chunk = bars + 13;      // [4] P^T of queries 32c .. 32c+31 written over X
  uint64_t* dp_full = bars + 17;      // dP^T in Y
  uint64_t* ld_done = bars + 18;      // warpgroup B has read P^T: X may be overwritten
  uint64_t* ds_full = bars + 19;      // the dS^T tile is in shared memory
  uint64_t* dq_full = bars + 20;      // dK and dQ_m of the step have completed (dQ_m in Y)
  uint64_t* y_free = bars + 21;       // warpgroup B has read dQ_m
  uint64_t* final_bar = bars + 22;    // the item's dK and dV are complete in TMEM
  uint64_t* dv_free = bars + 23;      // the dV epilogue has read the accumulator
  uint64_t* dk_free = bars + 24;      // the dK epilogue has read the accumulator
  uint64_t* done_bar = bars + 25;     // every MMA of the CTA has completed
  uint64_t* item_full = bars + 26;    // the next work item's index is in item_slot
  uint64_t* item_empty = bars + 27;   // every role has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 28);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 29);
  volatile int* item_slot = reinterpret_cast<volatile int*>(bars + 30);

  const int warp = warp_id(), lane = lane_id();
  const int W = p.window, G = p.G;
  // Persistent: the CTAs share the (key tile n, KV head, batch) items through a global
  // counter, first come first served, in super-block order (see sb_order). Warp 2 claims
  // them and passes each index to the other roles through a one-deep slot. Every step
  // of every item consumes one Q stage and the dO stage, so a step counter g running
  // across the CTA's items gives all ring stages and per-step barrier phases.
  struct Item {
    int n, hk, b, m_cnt, n_iters;
  };
  auto item_of = [&](int item) {
    Item it;
    int blk;
    sb_order(item, p.n_tiles, n_items / p.n_tiles, it.n, blk);
    it.hk = blk % (p.Hq / G);
    it.b = blk / (p.Hq / G);
    it.m_cnt = min(p.n_tiles - it.n, p.span);
    it.n_iters = G * it.m_cnt;
    return it;
  };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    for (int c = 0; c < 4; ++c) mbar_init(&p_chunk[c], 128);
    mbar_init(dp_full, 1);
    mbar_init(ld_done, 128);
    mbar_init(ds_full, 128);
    mbar_init(dq_full, 1);
    mbar_init(y_free, 128);
    mbar_init(final_bar, 1);
    mbar_init(dv_free, 128);
    mbar_init(dk_free, 128);
    mbar_init(done_bar, 1);
    mbar_init(item_full, 1);
    mbar_init(item_empty, 11);  // warps 0, 1, 3 and the eight warps of the two warpgroups
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 3) {
    // Extension slots start at zero (an MMA reads up to 96 bytes past a slot, into
    // the next one or the constant cores, always multiplied by zero: those bytes must
    // hold finite values even before the first copy lands). The constant key-side
    // cores: rows of (1, 1, 0, 0, 0, 0, 0, 0), then zeros.
    uint32_t* e = reinterpret_cast<uint32_t*>(smem + L::kExt);
    for (int i = lane; i < (L::kExtOnes - L::kExt) / 4; i += 32) e[i] = 0u;
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + L::kExtOnes);
    for (int i = lane; i < 64; i += 32) ones[i] = (i < 32 && (i & 3) == 0) ? 0x3F803F80u : 0u;
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tX = tmem, tY = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  const uint32_t sbase = smem_u32(smem);
  // the k-th work item of this CTA (-1: none left, or the CTA gave up), read by a whole
  // warp; one lane releases the slot for the role
  auto take_item = [&](int k) {
    int v = mbar_wait(item_full, k & 1, abort_flag) ? *item_slot : -1;
    v = __shfl_sync(0xffffffffu, v, 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(item_empty);
    return v;
  };

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers
    // warp 0: K of each item (two stages: the next item's K loads while the current
    // item's dQ_m products still read its own) and the Q ring; warp 3: V of each item
    // and the dO stage. Each Q / dO load also takes the 512-byte row extension of its
    // tile: -lse/scale with Q, -Delta with dO. The whole warp takes the items (the
    // slot is read warp-wide); lane 0 issues.
    const bool qside = (warp == 0);
    int last_q[QS] = {-1, -1}, last_do = -1, last_k[2] = {-1, -1}, last_v = -1;
    if (lane == 0) {
      if (qside) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
      } else {
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
      }
    }
    int g = 0;
    bool ok = true;
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      if (lane == 0) {
        const Item I = item_of(item);
        if (qside) {
          const int kb = k & 1;
          if ((ok = mbar_wait(&k_empty[kb], ((k >> 1) & 1) ^ 1, abort_flag))) {
            mbar_arrive_expect_tx(&k_full[kb], L::kTile);
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(smem + L::kK + kb * L::kTile + pn * L::kPanel, &tm_k, &k_full[kb], pn * 64, I.hk,
                          I.n * 128, I.b);
            last_k[kb] = k;
          }
        } else {
          if ((ok = mbar_wait(v_empty, (k & 1) ^ 1, abort_flag))) {
            mbar_arrive_expect_tx(v_full, L::kTile);
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(smem + L::kV + pn * L::kPanel, &tm_v, v_full, pn * 64, I.hk, I.n * 128, I.b);
            last_v = k;
          }
        }
        for (int it = 0; ok && it < I.n_iters; ++it, ++g) {
          const int h = I.hk * G + it / I.m_cnt, q0 = (I.n + it % I.m_cnt) * 128;
          const size_t ext_off = (((size_t)I.b * p.Hq + h) * p.n_tiles + q0 / 128) * 512;
          if (qside) {
            const int st = g % QS;
            if (!(ok = mbar_wait(&q_empty[st], ((g / QS) & 1) ^ 1, abort_flag))) break;
            mbar_arrive_expect_tx(&q_full[st], L::kTile + 512);
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(smem + L::kQ + st * L::kTile + pn * L::kPanel, &tm_q, &q_full[st], pn * 64, h, q0, I.b);
            bulk_load(smem + L::kExt + st * 512, p.ext_lse + ext_off, 512, &q_full[st]);
            last_q[st] = g;
          } else {
            if (!(ok = mbar_wait(do_empty, (g & 1) ^ 1, abort_flag))) break;
            mbar_arrive_expect_tx(do_full, L::kTile + 512);
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(smem + L::kDO + pn * L::kPanel, &tm_do, do_full, pn * 64, h, q0, I.b);
            bulk_load(smem + L::kExt + QS * 512, p.ext_delta + ext_off, 512, do_full);
            last_do = g;
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    if (lane == 0) {
      // let every copy in flight land before the CTA's shared memory is released (at
      // once after a normal run; an abort raised by another role may leave some pending)
      for (int s = 0; s < QS; ++s)
        if (last_q[s] >= 0) mbar_drain(&q_full[s], (last_q[s] / QS) & 1);
      for (int s = 0; s < 2; ++s)
        if (last_k[s] >= 0) mbar_drain(&k_full[s], (last_k[s] >> 1) & 1);
      if (last_do >= 0) mbar_drain(do_full, last_do & 1);
      if (last_v >= 0) mbar_drain(v_full, last_v & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); one elected lane
    // issues the MMAs and commits. Per step g of an item, in issue order:
    //   dV(g)      chunk by chunk as warpgroup A publishes P^T(g)
    //   S^T(g+1)   into X once warpgroup B has read P^T(g) (dV(g) precedes it in the pipe)
    //   dK(g), dQ_m(g)  once the dS^T tile is written; dQ_m(g) into Y (dP^T(g) was read)
    //   dP^T(g+1)  into Y once warpgroup B has read dQ_m(g)
    // Every group is preceded by all of its waits, so the tensor pipe is fed in bursts.
    const uint32_t leader = elect_one();
    constexpr uint32_t idSP = idesc_bf16(128, 128, false, false);  // S^T, dP^T
    constexpr uint32_t idKV = idesc_bf16(128, D, false, true);     // dV (A from TMEM), dK: B MN-major
    constexpr uint32_t idQ = idesc_bf16(128, D, true, true);       // dQ_m: A = dS MN-major, B = K MN-major
    // Descriptors are built once; an MMA only adds (byte offset >> 4) to the start field.
    const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024), dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);
    const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024), dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);
    const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kPanel, 1024);
    const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kPanel, 1024);
    const uint64_t dK_mn = sdesc_sw128(sbase + L::kK, L::kPanel, 1024);
    const uint64_t dS_k = sdesc_sw128(sbase + L::kDS, 16, 1024);           // A of dK: keys x queries
    const uint64_t dS_mn = sdesc_sw128(sbase + L::kDS, L::kPanel, 1024);   // A of dQ_m: queries contiguous
    // The extra K = 16 step: A = rows of (1, 1, 0, ..., 0) for every key (one core
    // repeated along M: stride 0; the second K core is the zero core), B = the slot's
    // (hi, lo) rows, MN-major, 32 bytes per 8 queries. B's K rows 2..15 are multiplied
    // by zeros (the second K core repeats the first: stride 0).
    constexpr uint32_t idX = idesc_bf16(128, 128, false, true);
    const uint64_t dOnes = sdesc_noswz(sbase + L::kExtOnes, 128, 0);
    const uint64_t dX = sdesc_noswz(sbase + L::kExt, 0, 32);
    // S^T' = K Q^T - lse/scale and dP^T' = V dO^T - Delta: A = K or V, B = Q or dO, both
    // K-major over d, then the extension step with slot xslot
    auto issue_R = [&](uint32_t dst, uint64_t dA, uint32_t aoff, uint64_t dB, uint32_t boff, int xslot,
                       uint64_t* done) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
        mma_ss(dst, dA + ((aoff + off) >> 4), dB + ((boff + off) >> 4), idSP, kk > 0, leader);
      }
      mma_ss(dst, dOnes, dX + ((xslot * 512) >> 4), idX, 1, leader);
      mma_commit(done, leader);
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    int g0 = 0, k = 0;  // step counter at the item's first step; items done
    bool ok = true;
    for (;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      const Item I = item_of(item);
      const int kb = k & 1;
      const uint32_t koff = kb * L::kTile;
      // S^T and dP^T of the item's first step: X and Y must be free of the previous step
      if (!(ok = wait_all(&k_full[kb], (k >> 1) & 1) && wait_all(&q_full[g0 % QS], (g0 / QS) & 1) &&
                 (g0 == 0 || wait_all(ld_done, (g0 - 1) & 1))))
        break;
      tc_fence_after();
      issue_R(tX, dK_k, koff, dQ_k, (g0 % QS) * L::kTile, g0 % QS, s_full);
      if (!(ok = wait_all(v_full, k & 1) && wait_all(do_full, g0 & 1) && (g0 == 0 || wait_all(y_free, (g0 - 1) & 1))))
        break;
      tc_fence_after();
      issue_R(tY, dV_k, 0, dDO_k, 0, QS, dp_full);
      if (I.n_iters == 1) mma_commit(v_empty, leader);  // V is no longer read
      for (int it = 0; ok && it < I.n_iters; ++it) {
        const int g = g0 + it;
        const int qs = g % QS, q1 = (g + 1) % QS;
        const bool more = it + 1 < I.n_iters;
        if (lane == 0) CSWA_MARK(0, g, 0);
        // the accumulators are free once the epilogues have read the previous item's
        if (it == 0 && !(ok = wait_all(dv_free, (k & 1) ^ 1))) break;
        // dV(g) chunk by chunk as warpgroup A publishes P^T: chunk c holds queries
        // 32c .. 32c+31 (K steps 2c, 2c+1), as bf16 pairs in columns 16c .. 16c+15
        for (int c = 0; c < 4; ++c) {
          if (!(ok = wait_all(&p_chunk[c], g & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int kk = 2 * c + u;
            mma_ts(tdV, tX + kk * 8, dDO_mn + ((kk * 2048) >> 4), idKV, (it > 0 || kk > 0), leader);
          }
        }
        if (!ok) break;
        mma_commit(do_empty, leader);
        if (lane == 0) CSWA_MARK(0, g, 1);
        // S^T(g+1) overwrites P^T(g) after dV(g) (issue order) and after warpgroup B read it
        if (more) {
          if (!(ok = wait_all(ld_done, g & 1) && wait_all(&q_full[q1], ((g + 1) / QS) & 1))) break;
          tc_fence_after();
          issue_R(tX, dK_k, koff, dQ_k, q1 * L::kTile, q1, s_full);
        }
        if (lane == 0) CSWA_MARK(0, g, 2);
        if (!(ok = wait_all(ds_full, g & 1))) break;
        if (lane == 0) CSWA_MARK(0, g, 3);
        if (it == 0 && !(ok = wait_all(dk_free, (k & 1) ^ 1))) break;
        tc_fence_after();
        // dK += dS^T Q: A = the dS^T tile (keys x queries, K-major), B = Q (MN-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
          mma_ss(tdK, dS_k + (off >> 4), dQ_mn + ((qs * L::kTile + kk * 2048) >> 4), idKV, (it > 0 || kk > 0),
                 leader);
        }
        mma_commit(&q_empty[qs], leader);
        // dQ_m = dS K into Y (dP^T(g) was read before ds_full): A = the same tile read
        // MN-major (queries contiguous), B = K (MN-major); 16 keys per K step
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tY, dS_mn + ((kk * 2048) >> 4), dK_mn + ((koff + kk * 2048) >> 4), idQ, kk > 0, leader);
        mma_commit(dq_full, leader);
        if (lane == 0) CSWA_MARK(0, g, 4);
        if (!more) mma_commit(&k_empty[kb], leader);  // the item's last S^T and dQ_m have read K
        if (more) {
          if (!(ok = wait_all(y_free, g & 1) && wait_all(do_full, (g + 1) & 1))) break;
          tc_fence_after();
          issue_R(tY, dV_k, 0, dDO_k, 0, QS, dp_full);
          if (it + 2 == I.n_iters) mma_commit(v_empty, leader);  // the item's last dP^T
        }
        if (lane == 0) CSWA_MARK(0, g, 5);
      }
      if (!ok) break;
      mma_commit(final_bar, leader);  // dK and dV of the item are complete
      g0 += I.n_iters;
    }
    // every MMA issued above has finished before TMEM is released
    mma_commit(done_bar, leader);
    mbar_drain(done_bar, 0);
  } else if (warp == 2) {
    // ------------------------------------------------------------ work scheduler
    // claims the CTA's next item from the global counter once every role has read
    // the previous one; -1 when none is left
    if (lane == 0) {
      for (int k = 0;; ++k) {
        if (!mbar_wait(item_empty, (k & 1) ^ 1, abort_flag)) break;
        const int idx = atomicAdd(p.item_counter, 1);
        const int v = idx < n_items ? idx : -1;
        *item_slot = v;
        mbar_arrive(item_full);
        if (v < 0) break;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ warpgroup A: P^T, dV epilogue
    // thread r = key row r of the tile (TMEM lane r)
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    const float2 sl2v = make_float2(sl2, sl2);
    bool ok = true;
    int g0 = 0;
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      const Item I = item_of(item);
      const int k0 = I.n * 128;
      const int j = k0 + r;
      for (int it = 0; it < I.n_iters; ++it) {
        const int g = g0 + it;
        const int q0 = (I.n + it % I.m_cnt) * 128;
        if (r == 0) CSWA_MARK(1, g, 0);
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, g & 1, abort_flag));
        if (!ok) break;
        if (r == 0) CSWA_MARK(1, g, 1);
        tc_fence_after();
        // P = exp2(scale log2e (S - lse/scale)): the MMA has already added -lse/scale, so one
        // packed multiply per two columns; masked entries are 0 after the exp2. Tiles inside
        // the band skip the mask (a warp-uniform branch).
        const bool full = (k0 + 127 <= q0) && (W < 0 || q0 + 127 - k0 <= W);
        const int c_lo = j - q0;                      // query q0 + c sees key j iff c >= c_lo
        const int c_hi = (W < 0) ? 127 : j + W - q0;  //   and c <= c_hi
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sr[64];
          tmem_ld32(tX + lane_off + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(tX + lane_off + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;  // queries 32c .. 32c+31
            uint32_t pk[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int col = 32 * c + 2 * u;  // query index within the tile
              const float2 e = __fmul2_rn(make_float2(__uint_as_float(sr[col - 64 * half]),
                                                      __uint_as_float(sr[col - 64 * half + 1])),
                                          sl2v);
              float y0 = ex2_approx(e.x), y1 = ex2_approx(e.y);
              if (!full) {
                y0 = ((col >= c_lo) & (col <= c_hi)) ? y0 : 0.f;
                y1 = ((col + 1 >= c_lo) & (col + 1 <= c_hi)) ? y1 : 0.f;
              }
              pk[u] = pack_bf16x2(y0, y1);
            }
            // bf16 pairs of queries 32c .. 32c+31 into columns 16c .. 16c+15: their fp32
            // S^T (queries <= 32c + 31 < 64 (half + 1)) is already in registers
            tmem_st16(tX + lane_off + 16 * c, pk);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_chunk[c]);
          }
        }
        if (r == 0) CSWA_MARK(1, g, 2);
      }
      if (!ok) break;
      // ------------------------------------------------------ dV epilogue (key row j)
      ok = __all_sync(0xffffffffu, mbar_wait(final_bar, k & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      __nv_bfloat16* dst = p.dv + ((size_t)((size_t)I.b * p.T + j) * (p.Hq / G) + I.hk) * D;
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
      tc_fence_before();
      mbar_arrive(dv_free);
      g0 += I.n_iters;
    }
  } else {
    // ------------------------------------------------------------ warpgroup B: dS^T, dQ, dK epilogue
    // thread r = TMEM lane r: key row r for dP^T / P^T / dK, query row r for dQ_m
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // row r of each panel of the dS^T tile; 16-byte chunk c of a panel row sits at
    // ((c ^ (r & 7)) * 16): the 128-byte swizzle the MMA descriptors expect
    uint8_t* ds_row = smem + L::kDS + r * 128;
    const uint32_t swz = (uint32_t)(r & 7);
    bool ok = true;
    int g0 = 0;
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      const Item I = item_of(item);
      const int j = I.n * 128 + r;
      for (int it = 0; it < I.n_iters; ++it) {
        const int g = g0 + it;
        const int h = I.hk * G + it / I.m_cnt;
        const int q0 = (I.n + it % I.m_cnt) * 128;
        if (r == 0) CSWA_MARK(2, g, 0);
        ok = __all_sync(0xffffffffu,
                        mbar_wait(dp_full, g & 1, abort_flag) && mbar_wait(&p_chunk[3], g & 1, abort_flag));
        if (!ok) break;
        if (r == 0) CSWA_MARK(2, g, 1);
        tc_fence_after();
        // dS = P * (dP - Delta): the MMA has already subtracted Delta. P^T (bf16 pairs, 64
        // columns of X) first: once it is in registers X may take S^T of the next step.
        // Then dP^T in four batches of 32 queries; each batch is 4 chunks of 8 queries of
        // one panel of the tile.
        uint32_t pp[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld32(tX + lane_off + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&pp[32 * c]));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(ld_done);
        if (r == 0) CSWA_MARK(2, g, 2);
#pragma unroll
        for (int bt = 0; bt < 4; ++bt) {
          uint32_t dp[32];
          tmem_ld32(tY + lane_off + 32 * bt, dp);
          tmem_ld_wait();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t pw = pp[16 * bt + 4 * ch + u];
              const float2 pf = make_float2(__uint_as_float(pw << 16), __uint_as_float(pw & 0xffff0000u));
              const float2 d = __fmul2_rn(pf, make_float2(__uint_as_float(dp[8 * ch + 2 * u]),
                                                          __uint_as_float(dp[8 * ch + 2 * u + 1])));
              w[u] = pack_bf16x2(d.x, d.y);
            }
            // queries 32 bt + 8 ch .. : panel bt / 2, chunk 4 (bt & 1) + ch of the row
            const int chunk = 4 * (bt & 1) + ch;
            *reinterpret_cast<uint4*>(ds_row + (bt >> 1) * L::kPanel + ((chunk ^ swz) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();  // the generic-proxy stores become visible to the MMAs
        mbar_arrive(ds_full);
        if (r == 0) CSWA_MARK(2, g, 3);
        // dQ_m(g) = dS K of this step (query row r of tile q0) into the fp32 accumulator
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full, g & 1, abort_flag));
        if (!ok) break;
        if (r == 0) CSWA_MARK(2, g, 4);
        tc_fence_after();
        // in halves of D/2 columns: the first half's reductions go out before the second
        // half is read, and Y is released as soon as the last columns are in registers
        float* acc = p.dq_acc + ((size_t)((size_t)I.b * p.T + q0 + r) * p.Hq + h) * D;
        const bool in_seq = q0 + r < p.T;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t a[D / 2];
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tmem_ld32(tY + lane_off + (D / 2) * hf + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&a[32 * c]));
          tmem_ld_wait();
          if (hf == 1) {
            tc_fence_before();
            mbar_arrive(y_free);
            if (r == 0) CSWA_MARK(2, g, 5);
          }
          if (in_seq) {
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
              red_add_f32x4(acc + (D / 2) * hf + 4 * c, __uint_as_float(a[4 * c]), __uint_as_float(a[4 * c + 1]),
                            __uint_as_float(a[4 * c + 2]), __uint_as_float(a[4 * c + 3]));
          }
        }
        if (r == 0) CSWA_MARK(2, g, 6);
      }
      if (!ok) break;
      // ------------------------------------------------------ dK epilogue (key row j)
      ok = __all_sync(0xffffffffu, mbar_wait(final_bar, k & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const size_t row = ((size_t)I.b * p.T + j) * (p.Hq / G) + I.hk;
      __nv_bfloat16* dst = p.dk + row * D;
      if (p.k_raw) {
        // dk with respect to the raw k: the prologue backward on the way out
        const uint32_t src = tdK + lane_off;
        const float sc = p.scale;
        auto dy_chunk = [&](int c0, float (&v)[16]) {
          uint32_t t[16];
          tmem_ld16(src + c0, t);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u) v[u] = __uint_as_float(t[u]) * sc;
        };
        // tcgen05.ld is warp-collective: rows past T run the same steps on row T - 1's
        // inputs and store nothing
        const int jj = min(j, p.T - 1);
        const size_t row_in = ((size_t)I.b * p.T + jj) * (p.Hq / G) + I.hk;
        prologue_bwd_row<D>(dy_chunk, p.k_raw + row_in * D, p.rope_cs + (size_t)jj * (D / 2), p.eps, dst,
                            j < p.T);
      } else {
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
      tc_fence_before();
      mbar_arrive(dk_free);
      g0 += I.n_iters;
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Row extensions of the S^T and dP^T MMAs, the dQ accumulator's zeroing, and (for
// the fused prologue backward) the rotary cos/sin table.
// For each query row i (padded to 128-row tiles) x = -lse_i / scale and y = -Delta_i
// = -(dO_i . o_i) are split into bf16 pairs hi + lo (hi = bf16(x), lo = bf16(x - hi):
// together 16 significant bits), so that one extra K = 16 MMA step against key-side
// rows (1, 1, 0, ...) adds x (or y) to every entry of query column i in fp32. Padded
// rows get x = -1e30 (finite: the MMA also multiplies these bytes by zero; exp2 of it
// is 0) and y = 0. Per (batch, head, query tile) 512 bytes: for each group of 8 rows,
// 16 bytes of the 8 hi values then 16 bytes of the 8 lo values (the MN-major no-swizzle
// layout: one core row per K index). D/8 lanes per (b, t, h) row.
struct PrepParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  uint8_t* ext_lse;
  uint8_t* ext_delta;
  float* dq_acc;
  int* item_counter;
  float2* rope_cs;           // (T, D/2), or null
  long long row_blocks;      // blocks of the row part; the blocks after them fill rope_cs
  int B, T, Tpad, Hq;
  float inv_scale;
  // turns of rotary pair j per unit position as a 64-bit fixed-point fraction (as the
  // prologue kernel computes its angles)
  unsigned long long turns[64];
};

template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __grid_constant__ PrepParams p) {
  constexpr int LK = D / 8;
  if (blockIdx.x >= p.row_blocks) {
    // the cos/sin table of the rotary angles: entry (t, j) = angle t * omega_j
    const long long e = (blockIdx.x - p.row_blocks) * (long long)blockDim.x + threadIdx.x;
    if (e < (long long)p.T * (D / 2)) {
      const int t = (int)(e / (D / 2)), jj = (int)(e % (D / 2));
      const unsigned long long frac = (unsigned long long)(unsigned)t * p.turns[jj];
      const float ang = (float)(int)(unsigned)(frac >> 32) * 1.4629180792671596e-09f;  // 2 pi / 2^32
      float c, s;
      __sincosf(ang, &s, &c);
      p.rope_cs[e] = make_float2(c, s);
    }
    return;
  }
  // the main kernel that follows on the stream hands out its work items from this counter
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.item_counter = 0;
  const long long rows = (long long)p.B * p.Tpad * p.Hq;
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gtid / LK;
  const int lr = (int)(gtid % LK);
  const bool active = row < rows;
  // row enumerates (b, t, h) with t over the padded length (32-bit math when it fits)
  int h, t, b;
  if (rows < (1ll << 31)) {
    const unsigned r32 = active ? (unsigned)row : 0u;
    h = (int)(r32 % (unsigned)p.Hq);
    const unsigned bt = r32 / (unsigned)p.Hq;
    t = (int)(bt % (unsigned)p.Tpad), b = (int)(bt / (unsigned)p.Tpad);
  } else {
    h = active ? (int)(row % p.Hq) : 0;
    const long long bt = active ? row / p.Hq : 0;
    t = (int)(bt % p.Tpad), b = (int)(bt / p.Tpad);
  }
  const bool real = active && t < p.T;
  float dsum = 0.f;
  if (real) {
    const size_t off = ((size_t)((size_t)b * p.T + t) * p.Hq + h) * D + lr * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(p.o + off);
    const uint4 gv = *reinterpret_cast<const uint4*>(p.dout + off);
    float4* acc = reinterpret_cast<float4*>(p.dq_acc + off);
    acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
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
    // clamped to stay finite in bf16 (a huge 1/scale must not turn x into -inf)
    const float x =
        real ? fminf(fmaxf(-p.lse[((size_t)b * p.Hq + h) * p.T + t] * p.inv_scale, -3.0e38f), 3.0e38f) : -1e30f;
    const float y = real ? -dsum : 0.f;
    const int i = t & 127;
    const size_t at = (((size_t)b * p.Hq + h) * (p.Tpad / 128) + t / 128) * 512 + (i >> 3) * 32 + (i & 7) * 2;
    const __nv_bfloat16 xh = __float2bfloat16_rn(x), yh = __float2bfloat16_rn(y);
    *reinterpret_cast<__nv_bfloat16*>(p.ext_lse + at) = xh;
    *reinterpret_cast<__nv_bfloat16*>(p.ext_lse + at + 16) = __float2bfloat16_rn(x - __bfloat162float(xh));
    *reinterpret_cast<__nv_bfloat16*>(p.ext_delta + at) = yh;
    *reinterpret_cast<__nv_bfloat16*>(p.ext_delta + at + 16) = __float2bfloat16_rn(y - __bfloat162float(yh));
  }
}

// dq = scale * (dQ accumulator) as bf16; with kFused, the prologue backward of the
// raw q applied per row (rows t of every (b, h), position t). D/8 lanes per row,
// lane l owning elements 4l..4l+3 of both halves, so a rotation pair never leaves
// its lane; kRows rows per thread.
struct DqParams {
  const float* dq_acc;
  __nv_bfloat16* dq;
  const __nv_bfloat16* q_raw;  // kFused only
  const float2* rope_cs;       // kFused only
  long long rows;              // B * T * Hq
  int Hq, T;
  float scale, eps;
};

template <int D, bool kFused>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const DqParams p) {
  constexpr int LK = D / 8, H = D / 2, kRows = 2;
  constexpr int kRowsPerBlock = 256 / LK;
  const int lr = threadIdx.x % LK;
  const int j0 = 4 * lr;
#pragma unroll
  for (int u = 0; u < kRows; ++u) {
    const long long row = ((long long)blockIdx.x * kRows + u) * kRowsPerBlock + threadIdx.x / LK;
    const bool active = row < p.rows;  // uniform over the row's lanes
    const long long rr = active ? row : 0;
    const float* a = p.dq_acc + rr * D;
    const float4 va = *reinterpret_cast<const float4*>(a + j0);
    const float4 vb = *reinterpret_cast<const float4*>(a + H + j0);
    float ya[4] = {va.x * p.scale, va.y * p.scale, va.z * p.scale, va.w * p.scale};
    float yb[4] = {vb.x * p.scale, vb.y * p.scale, vb.z * p.scale, vb.w * p.scale};
    if constexpr (kFused) {
      const int t = (int)((rr / p.Hq) % p.T);
      const uint2 xa2 = *reinterpret_cast<const uint2*>(p.q_raw + rr * D + j0);
      const uint2 xb2 = *reinterpret_cast<const uint2*>(p.q_raw + rr * D + H + j0);
      const float4 c01 = *reinterpret_cast<const float4*>(p.rope_cs + (size_t)t * H + j0);
      const float4 c23 = *reinterpret_cast<const float4*>(p.rope_cs + (size_t)t * H + j0 + 2);
      const float cs_c[4] = {c01.x, c01.z, c23.x, c23.z}, cs_s[4] = {c01.y, c01.w, c23.y, c23.w};
      float xa[4], xb[4];
      {
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa2);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb2);
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const float2 fa = __bfloat1622float2(a2[v]), fb = __bfloat1622float2(b2[v]);
          xa[2 * v] = fa.x, xa[2 * v + 1] = fa.y, xb[2 * v] = fb.x, xb[2 * v + 1] = fb.y;
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < 4; ++v) ss = fmaf(xa[v], xa[v], fmaf(xb[v], xb[v], ss));
#pragma unroll
      for (int o = LK / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv_r = rsqrtf(ss * (1.f / D) + p.eps);
      float ga[4], gb[4], dot = 0.f;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        ga[v] = fmaf(yb[v], cs_s[v], ya[v] * cs_c[v]);
        gb[v] = fmaf(-ya[v], cs_s[v], yb[v] * cs_c[v]);
        dot = fmaf(ga[v], xa[v] * inv_r, fmaf(gb[v], xb[v] * inv_r, dot));
      }
#pragma unroll
      for (int o = LK / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float proj = dot * (1.f / D);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        ya[v] = (ga[v] - xa[v] * inv_r * proj) * inv_r;
        yb[v] = (gb[v] - xb[v] * inv_r * proj) * inv_r;
      }
    }
    if (active) {
      *reinterpret_cast<uint2*>(p.dq + rr * D + j0) = make_uint2(pack_bf16x2(ya[0], ya[1]), pack_bf16x2(ya[2], ya[3]));
      *reinterpret_cast<uint2*>(p.dq + rr * D + H + j0) =
          make_uint2(pack_bf16x2(yb[0], yb[1]), pack_bf16x2(yb[2], yb[3]));
    }
  }
}

}  // namespace cswa
