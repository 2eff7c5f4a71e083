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
//   bwd_prep     per query row, -lse_i/scale and -Delta_i as bf16 hi + lo pairs,
//                laid out as one extra K = 16 step of an MMA (padded rows: a
//                large negative lse term, so P = 0 there).
//   bwd_main     persistent, one CTA per SM, taking (128-key tile, KV head,
//                batch) items from a global counter. For an item, K and V stay in shared
//                memory and the CTA walks every (query head of the group, 128-row
//                query tile) that sees the key tile, with Q and dO in rings of 3
//                and 2 stages that run on across items; the next item's K and V
//                load during the current item's last step, and its first S^T and
//                dP^T are computed during the current item's dK/dV epilogue. Per step, all MMAs M = 128, N = 128 (the
//                shape the tensor pipe runs at full rate), TMEM regions R0, R1 of
//                128 columns each:
//                  S^T' = K Q^T - lse/scale     (SS, + extension step) -> R0
//                  P^T  = exp2(c S^T')          bf16 pairs written over R0
//                  dV  += P^T dO                (TS: A from TMEM) -> [256,256+D)
//                  dP^T'= V dO^T - Delta        (SS, + extension step) -> R1
//                  dS^T = P^T dP^T'             bf16 pairs written over R1
//                  dK  += dS^T Q                (TS) -> [256+D,256+2D)
//                The extension step adds the per-query terms inside the MMA, so
//                the elementwise warps read no per-column statistics at all.
//                The MMA warp issues dV(it) + S^T(it+1) and dK(it) + dP^T(it+1)
//                as bursts, so S^T and dP^T of the next step are computed while
//                the elementwise warps work on this one. dS^T leaves as bf16
//                tiles for bwd_dq (plain 512-byte coalesced stores). dK, dV are
//                complete in the CTA (the whole group is walked here), so they
//                are written once, as bf16, with no atomics: each goes through
//                the Q or dO ring stage of the item's last step (lent to the
//                epilogue until its TMA stores have read it) and leaves as TMA
//                stores of 32-row boxes.
//   bwd_dq       persistent, (128-row query tile, query head, batch) items:
//                dQ = scale * sum over key tiles of dS K, accumulated in TMEM
//                from the stored dS^T tiles (one bulk copy each) and K tiles,
//                written once as bf16 through a staging tile and TMA stores.
// Splitting dQ out keeps fp32 dQ reductions out of the main kernel, whose
// TMEM (512 columns) and shared memory are fully used. (A variant that reduced a
// per-step dQ tile into an fp32 accumulator in L2 instead -- 64 KB of 16-byte
// reductions per step -- measured slower on B200: the reductions drained at about
// 14 bytes per clock per SM.)
// For the block backward (attn_block_bwd) the dK epilogue and the dQ kernel's
// epilogue also apply the prologue backward, so dk and dq come out with respect to
// the raw k and q: the raw tile arrives by TMA in the staging buffer, the rotary
// angles are computed from the row's position, and the result overwrites the raw
// rows in place before the store.
// Warp roles in bwd_main: 0 TMA (K, V, Q ring), 1 MMA issuer (whole warp, one
// elected lane issues), 2 TMEM allocator and work scheduler, 3 TMA (dO ring),
// 4-7 and 8-11 P/dS (thread = key row; query columns 0-63 and 64-127), then
// the dK (4-7) and dV (8-11) epilogues.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct BwdParams {
  // per (batch, query head, 128-row query tile): 512 bytes holding -lse/scale and
  // -Delta of the tile's rows as bf16 hi + lo pairs, laid out as the extra K = 16 step
  // of the S^T and dP^T MMAs reads them (see attn_bwd_prep_kernel)
  const uint8_t* ext_lse;
  const uint8_t* ext_delta;
  __nv_bfloat16* ds;   // stored dS^T tiles (see ds_unit_offset)
  int* item_counter;   // [2] next work item of the main and dQ kernels (zeroed by the prep kernel)
  int T, Tpad, Hq, G, window, n_tiles, span;  // tiles of 128 rows; span = query tiles per key tile
  long long tiles_per_bh;                     // stored dS^T tiles per (batch, query head)
  // the call may run in passes over the (batch, KV head) blocks, blk = b * Hkv + hk: this
  // launch covers blocks blk0 .. blk0 + n_items / n_tiles - 1, and the stored dS^T tiles of
  // block blk0 start at the beginning of p.ds
  int blk0;
  float scale, scale_log2;
  // fused prologue backward (attn_block_bwd): dk and dq with respect to the raw k and
  // q (whose tensor maps the kernels take), the RMS-norm eps and the turns of rotary
  // pair j per unit position as 64-bit fixed-point fractions (see rope_cos_sin)
  int rope;
  float eps;
  unsigned long long turns[64];
};

// Query tiles that see key tile n: [n, n + min(n_tiles - n, span) - 1], where
// span = n_tiles (no window) or floor((127 + W) / 128) + 1. The dS^T tiles of
// one (batch, head) are stored key tile by key tile; this is where key tile n starts.
__host__ __device__ inline int bwd_span(int n_tiles, int window) {
  return window < 0 ? n_tiles : min(n_tiles, (127 + window) / 128 + 1);
}
// Byte offset, inside one stored 32 KB dS^T tile, of the 16-byte unit holding
// queries 8u .. 8u+7 (u in 0..15) of key row r: 8 KB per 32 keys, 512 bytes per 8
// queries, 16 bytes per key. A warp of 32 key rows thus writes 512 contiguous bytes
// per unit index, and the tile is the no-swizzle MN-major operand layout of the dQ
// MMA (core matrices of 8 keys x 8 queries: 128 bytes along K, 512 bytes along M).
__host__ __device__ inline uint32_t ds_unit_offset(int r, int u) {
  return (uint32_t)((r >> 5) * 8192 + u * 512 + (r & 31) * 16);
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
// Prologue backward of 16 rotary pairs (j0 .. j0+15, and j0 + D/2 ..) of one row held
// by one thread (nanochat Admin & Developer Guide, 3: RMS-norm without weight, then
// RoPE). With dy the gradient with respect to the prologue output and x the raw row:
//   g = dy rotated by -phi,  r = sqrt(mean(x^2) + eps),  xh = x / r,
//   dx = (g - xh (g . xh) / D) / r.
// rotate_back: g of the pairs from dy (both halves, fp32, in place).
template <int D>
__device__ __forceinline__ void rope_rotate_back(const unsigned long long* turns, unsigned pos, int j0,
                                                 float (&a)[16], float (&b)[16]) {
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    float c, sn;
    rope_cos_sin(pos, turns[j0 + u], c, sn);
    const float ga = fmaf(b[u], sn, a[u] * c);
    const float gb = fmaf(-a[u], sn, b[u] * c);
    a[u] = ga;
    b[u] = gb;
  }
}

// Work-item order of the persistent backward kernels. Items are (tile t, block blk)
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

// P/dS warps of the main kernel, in groups of 4 (one per TMEM lane quarter), each group
// taking 128 / (kBwdSoftmaxWarps / 4) query columns of the step. 16 (four per SM
// sub-partition, 32 columns each, 96 registers a thread) measured slower than 8.
constexpr int kBwdSoftmaxWarps = 8;
constexpr int kBwdThreads = (4 + kBwdSoftmaxWarps) * 32;

template <int D>
struct BwdLayout {
  static constexpr int kQStages = 3, kDOStages = 2;
  static constexpr int kTile = 128 * D * 2;   // one 128-row bf16 tile (K, V, Q or dO)
  static constexpr int kPanel = 128 * 128;    // one 64-column panel of a 128-row tile
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;                    // [kQStages]
  static constexpr int kDO = kQ + kQStages * kTile;        // [kDOStages]
  // per-row extension slots (512 bytes, see the prep kernel) of the Q stages, then of
  // the dO stages, then the constant key-side extension (a core of ones, a core of zeros)
  static constexpr int kExt = kDO + kDOStages * kTile;
  static constexpr int kExtOnes = kExt + (kQStages + kDOStages) * 512;
  static constexpr int kBar = kExtOnes + 256;
  static constexpr int kNumBars = 29;
  // the barriers, then three 4-byte slots (TMEM base, abort flag, work item)
  static constexpr int kUsed = kBar + kNumBars * 8 + 16;
  static constexpr int kBytes = (kUsed + 1024 <= 232448) ? kUsed + 1024 : 232448;
  static_assert(kUsed <= 232448, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
};

// tm_kr: the raw k (block backward only); tm_dk, tm_dv: the outputs, 32-row boxes.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_dk,
                    const __grid_constant__ CUtensorMap tm_dv, const __grid_constant__ BwdParams p, int n_items) {
  using L = BwdLayout<D>;
  constexpr int QS = L::kQStages, DS = L::kDOStages;
  // query columns of a step: kSGroups groups of kSCols, each group's P^T (and dS^T) packed
  // as bf16 pairs into the first kSCols / 2 of its own columns, published in kPChunks
  // chunks of 16 queries (one MMA K step each)
  constexpr int kSGroups = kBwdSoftmaxWarps / 4, kSCols = 128 / kSGroups, kPChunks = kSCols / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // the layout needs a 1024-byte aligned base: report (never overrun) if the slack is too small
  if ((smem - smem_raw) + L::kUsed > L::kBytes) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusLayout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;               // the item's last S^T and dP^T have read K and V
  uint64_t* q_full = bars + 2;                 // [QS]
  uint64_t* q_empty = q_full + QS;             // [QS]  dK has read the Q tile
  uint64_t* q_borrow = q_empty + QS;           // [QS]  the dK epilogue is done with a lent stage
  uint64_t* do_full = q_borrow + QS;           // [DS]
  uint64_t* do_empty = do_full + DS;           // [DS]  dV has read the dO tile
  uint64_t* do_borrow = do_empty + DS;         // [DS]  the dV epilogue is done with a lent stage
  uint64_t* s_full = do_borrow + DS;           // S^T in TMEM
  uint64_t* p_chunk = s_full + 1;              // [4] P^T chunk c of every column group written
  uint64_t* dp_full = p_chunk + 4;             // dP^T in TMEM
  uint64_t* ds_full = dp_full + 1;             // dS^T written over dP^T
  uint64_t* final_bar = ds_full + 1;           // the item's dK and dV are complete in TMEM
  uint64_t* acc_free = final_bar + 1;          // the epilogue has read them
  uint64_t* item_full = acc_free + 1;          // the next work item's index is in item_slot
  uint64_t* item_empty = item_full + 1;        // every role has read it
  uint64_t* kr_full = item_empty + 1;          // the raw k tile is in the lent Q stage
  static_assert(L::kNumBars == 2 + 3 * QS + 3 * DS + 9 + 2 + 1, "barrier count");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kr_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(kr_full + 1) + 1;
  volatile int* item_slot = reinterpret_cast<volatile int*>(kr_full + 1) + 2;

  const int warp = warp_id(), lane = lane_id();
  const int W = p.window, G = p.G;
  // Persistent: the CTAs share the (key tile n, KV head, batch) items through a
  // global counter (first come, first served: CTAs that finish early take more), in
  // super-block order (see sb_order): CTAs working at the same time read the same
  // few blocks' Q/dO tiles through L2, and the last items handed out are light. Warp 2
  // claims them and passes each index to the other roles through a one-deep slot.
  // Every step of every item consumes one stage of the Q ring and one of the dO
  // ring, so a step counter g running across the CTA's items gives all ring stages
  // and per-step barrier phases.
  struct Item {
    int n, hk, b, m_cnt, n_iters;
  };
  auto item_of = [&](int item) {
    Item it;
    int blk;
    sb_order(item, p.n_tiles, n_items / p.n_tiles, it.n, blk);
    blk += p.blk0;
    it.hk = blk % (p.Hq / G);
    it.b = blk / (p.Hq / G);
    it.m_cnt = min(p.n_tiles - it.n, p.span);
    it.n_iters = G * it.m_cnt;
    return it;
  };

  if (warp == 0 && lane == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&q_borrow[s], 4);  // the four dK epilogue warps
    }
    for (int s = 0; s < DS; ++s) {
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
      mbar_init(&do_borrow[s], 4);  // the four dV epilogue warps
    }
    mbar_init(s_full, 1);
    for (int c = 0; c < 4; ++c) mbar_init(&p_chunk[c], kBwdSoftmaxWarps * 32);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kBwdSoftmaxWarps * 32);
    mbar_init(final_bar, 1);
    mbar_init(acc_free, 256);
    mbar_init(item_full, 1);
    mbar_init(item_empty, 3 + kBwdSoftmaxWarps);  // warps 0, 1, 3 and the P/dS warps
    mbar_init(kr_full, 1);
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
  // S^T (P^T packed over it), dP^T (dS^T packed over it), dV, dK
  const uint32_t tR0 = tmem, tR1 = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

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
    // warp 0: K and V of each item and the Q ring; warp 3: the dO ring (its stages
    // free up at a different point of the step, so it waits on its own). Each stage
    // also takes the 512-byte row extension of its tile: -lse/scale with Q, -Delta
    // with dO. K and V of the next item load as soon as the current item's last S^T
    // and dP^T have read the previous ones. The stage of an item's last step is lent
    // to that item's dK (Q ring) or dV (dO ring) epilogue as its staging buffer: it
    // is loaded again only once the epilogue has released it (the borrow barrier).
    // The whole warp takes the items (the slot is read warp-wide); lane 0 issues.
    const bool qside = (warp == 0);
    const int nst = qside ? QS : DS;
    int last_issue[3] = {-1, -1, -1};
    int last_kv = -1;
    if (lane == 0) {
      if (qside) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      } else {
        tma_prefetch_desc(&tm_do);
      }
    }
    uint64_t* full = qside ? q_full : do_full;
    uint64_t* empty = qside ? q_empty : do_empty;
    uint64_t* borrow = qside ? q_borrow : do_borrow;
    uint32_t lent = 0, lent_par = 0;  // per stage: lent to an epilogue; parity of its next release
    const CUtensorMap* tm = qside ? &tm_q : &tm_do;
    const int base = qside ? L::kQ : L::kDO;
    const uint8_t* ext = qside ? p.ext_lse : p.ext_delta;
    uint8_t* ext_slot = smem + L::kExt + (qside ? 0 : QS * 512);
    int g = 0;
    bool ok = true;
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      if (lane == 0) {
        const Item I = item_of(item);
        if (qside) {
          if ((ok = mbar_wait(kv_empty, (k & 1) ^ 1, abort_flag))) {
            mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
            for (int pn = 0; pn < D / 64; ++pn) {
              tma_load_4d(smem + L::kK + pn * L::kPanel, &tm_k, kv_full, pn * 64, I.hk, I.n * 128, I.b);
              tma_load_4d(smem + L::kV + pn * L::kPanel, &tm_v, kv_full, pn * 64, I.hk, I.n * 128, I.b);
            }
            // the raw k rows the dK epilogue will load: on their way to L2 now
            if (p.rope)
              for (int pn = 0; pn < D / 64; ++pn) tma_prefetch_l2_4d(&tm_kr, pn * 64, I.hk, I.n * 128, I.b);
            last_kv = k;
          }
        }
        for (int it = 0; ok && it < I.n_iters; ++it, ++g) {
          const int st = g % nst;
          const int h = I.hk * G + it / I.m_cnt, q0 = (I.n + it % I.m_cnt) * 128;
          if (qside) CSWA_MARK(3, g, 0);
          if ((lent >> st) & 1u) {
            if (!(ok = mbar_wait(&borrow[st], (lent_par >> st) & 1u, abort_flag))) break;
            lent &= ~(1u << st);
            lent_par ^= 1u << st;
          }
          if (!(ok = mbar_wait(&empty[st], ((g / nst) & 1) ^ 1, abort_flag))) break;
          if (qside) CSWA_MARK(3, g, 1);
          mbar_arrive_expect_tx(&full[st], L::kTile + 512);
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_4d(smem + base + st * L::kTile + pn * L::kPanel, tm, &full[st], pn * 64, h, q0, I.b);
          bulk_load(ext_slot + st * 512, ext + (((size_t)I.b * p.Hq + h) * p.n_tiles + q0 / 128) * 512, 512,
                    &full[st]);
          last_issue[st] = g;
          if (it + 1 == I.n_iters) lent |= 1u << st;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    if (lane == 0) {
      // let every copy in flight land before the CTA's shared memory is released (at
      // once after a normal run; an abort raised by another role may leave some pending)
      for (int s = 0; s < nst; ++s)
        if (last_issue[s] >= 0) mbar_drain(&full[s], (last_issue[s] / nst) & 1);
      if (qside && last_kv >= 0) mbar_drain(kv_full, last_kv & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); one elected lane
    // issues the MMAs and commits.
    const uint32_t leader = elect_one();
    constexpr uint32_t idSP = idesc_bf16(128, 128, false, false);  // S^T, dP^T
    constexpr uint32_t idKV = idesc_bf16(128, D, false, true);     // dV, dK: A from TMEM, B MN-major
    // Descriptors are built once; an MMA only adds (byte offset >> 4) to the start field.
    const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024), dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);
    const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024), dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);
    const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kPanel, 1024);
    const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kPanel, 1024);
    // The extra K = 16 step: A = rows of (1, 1, 0, ..., 0) for every key (one core
    // repeated along M: stride 0; the second K core is the zero core), B = the slot's
    // (hi, lo) rows, MN-major, 32 bytes per 8 queries. B's K rows 2..15 are multiplied
    // by zeros (the second K core repeats the first: stride 0).
    constexpr uint32_t idX = idesc_bf16(128, 128, false, true);
    const uint64_t dOnes = sdesc_noswz(sbase + L::kExtOnes, 128, 0);
    const uint64_t dX = sdesc_noswz(sbase + L::kExt, 0, 32);
    // S^T' = K Q^T - lse/scale and dP^T' = V dO^T - Delta: A = K or V, B = Q or dO, both
    // K-major over d, then the extension step with slot xslot
    auto issue_R = [&](uint32_t dst, uint64_t dA, uint64_t dB, uint32_t boff, int xslot, uint64_t* done) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::kPanel + (kk & 3) * 32;
        mma_ss(dst, dA + (off >> 4), dB + ((boff + off) >> 4), idSP, kk > 0, leader);
      }
      mma_ss(dst, dOnes, dX + ((xslot * 512) >> 4), idX, 1, leader);
      mma_commit(done, leader);
    };
    // dK += dS^T Q: A = the bf16 pairs packed over dP^T (column group u's queries in its
    // first kSCols / 2 columns; K step kk = group kk / kPChunks, chunk kk % kPChunks), B = Q,
    // MN-major
    auto issue_acc = [&](uint32_t dst, uint32_t a_tmem, uint64_t dB, uint32_t boff, bool first) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(dst, a_tmem + (kk / kPChunks) * kSCols + (kk % kPChunks) * 8, dB + ((boff + kk * 2048) >> 4), idKV,
               (!first || kk > 0), leader);
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    const bool tracer = (lane == 0);
    (void)tracer;
    int g0 = 0, k = 0;  // step counter at the item's first step; items done
    bool ok = true;
    for (;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      const Item I = item_of(item);
      // S^T and dP^T of the item's first step, once its K, V, Q and dO are in
      if (!(ok = wait_all(kv_full, k & 1) && wait_all(&q_full[g0 % QS], (g0 / QS) & 1))) break;
      tc_fence_after();
      issue_R(tR0, dK_k, dQ_k, (g0 % QS) * L::kTile, g0 % QS, s_full);
      if (!(ok = wait_all(&do_full[g0 % DS], (g0 / DS) & 1))) break;
      tc_fence_after();
      issue_R(tR1, dV_k, dDO_k, (g0 % DS) * L::kTile, QS + g0 % DS, dp_full);
      if (I.n_iters == 1) mma_commit(kv_empty, leader);  // K and V are no longer read
      // Each step issues two bursts, each preceded by all of its waits (a barrier wait
      // between two groups would let the tensor pipe run dry): dV(it) + S^T(it+1) once
      // P^T(it) is written, dK(it) + dP^T(it+1) once dS^T(it) is written.
      for (int it = 0; ok && it < I.n_iters; ++it) {
        const int g = g0 + it;
        const int qs = g % QS, ds = g % DS;
        const int q1 = (g + 1) % QS, d1 = (g + 1) % DS;
        const bool more = it + 1 < I.n_iters;
        if (tracer) CSWA_MARK(0, g, 0);
        if (more && !(ok = wait_all(&q_full[q1], ((g + 1) / QS) & 1))) break;
        // the accumulators are free once the epilogue has read the previous item's
        if (it == 0 && !(ok = wait_all(acc_free, (k & 1) ^ 1))) break;
        // dV(it) chunk by chunk as the P/dS warps publish P^T: chunk c holds queries
        // 16c..16c+15 of each column group u, i.e. the K steps kPChunks * u + c
        for (int c = 0; c < kPChunks; ++c) {
          if (!(ok = wait_all(&p_chunk[c], g & 1))) break;
          if (tracer && c == 0) CSWA_MARK(0, g, 1);
          tc_fence_after();
#pragma unroll
          for (int u = 0; u < kSGroups; ++u) {
            const int kk = kPChunks * u + c;
            mma_ts(tdV, tR0 + u * kSCols + c * 8, dDO_mn + ((ds * L::kTile + kk * 2048) >> 4), idKV,
                   (it > 0 || kk > 0), leader);
          }
        }
        if (!ok) break;
        mma_commit(&do_empty[ds], leader);
        if (tracer) CSWA_MARK(0, g, 2);
        // S^T(it+1) overwrites P^T(it) only after dV(it) has read it: MMAs run in issue order
        if (more) issue_R(tR0, dK_k, dQ_k, q1 * L::kTile, q1, s_full);
        if (tracer) CSWA_MARK(0, g, 4);
        if (more && !(ok = wait_all(&do_full[d1], ((g + 1) / DS) & 1))) break;
        if (!(ok = wait_all(ds_full, g & 1))) break;
        if (tracer) CSWA_MARK(0, g, 5);
        tc_fence_after();
        issue_acc(tdK, tR1, dQ_mn, qs * L::kTile, it == 0);
        mma_commit(&q_empty[qs], leader);
        if (tracer) CSWA_MARK(0, g, 6);
        if (more) {
          issue_R(tR1, dV_k, dDO_k, d1 * L::kTile, QS + d1, dp_full);
          if (it + 2 == I.n_iters) mma_commit(kv_empty, leader);  // the item's last S^T and dP^T
        }
        if (tracer) CSWA_MARK(0, g, 7);
      }
      if (!ok) break;
      mma_commit(final_bar, leader);  // dK and dV of the item are complete
      g0 += I.n_iters;
    }
    // every MMA issued above has finished before TMEM is released. Items 0 .. k-1 each
    // committed one phase of final_bar, the last of which covers every MMA of a normal
    // run; after an abort, one more phase covers those issued since (final_bar gets no
    // other commit, so neither wait can find its phase already overtaken).
    if (k > 0) mbar_drain(final_bar, (k - 1) & 1);
    if (!ok) {
      mma_commit(final_bar, leader);
      mbar_drain(final_bar, k & 1);
    }
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
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P and dS (thread = key row)
    // warps 4-7 take query columns 0 .. kSCols-1, warps 8-11 the next kSCols (warp 2 only
    // allocates TMEM and schedules)
    const int half = (warp - 4) >> 2;  // column group; groups 0 and 1 also run the dK / dV epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t cols = lane_off + kSCols * half;  // this thread's S^T / dP^T columns
    const float sl2 = p.scale_log2;
    const bool tracer = ((warp == 4 || warp == 8) && lane == 0);
    const int trole = 1 + half;
    (void)tracer;
    (void)trole;
    // dS^T of the step (this warp's 32 keys x 64 queries) and where it goes in the
    // workspace tile the dQ kernel reads. It is stored right after the dS phase, while the
    // warp waits for the next S^T (the stores drain while nothing else runs on the warp,
    // and the registers are free again for the P phase). The tile is written as 16-byte
    // units (8 queries of one key) ordered so that every warp store covers 512 contiguous
    // bytes (see ds_unit_offset).
    uint32_t dsk[kSCols / 2];
    bool ok = true;
    int g0 = 0, k = 0;
    int kr_pending = -1;  // warp 4, lane 0: the item whose raw k load nobody has waited for yet
    // the ring stage this warp lent its last epilogue, returned once the TMA stores have
    // read it: during the next item's first P phase, so that the read overlaps the
    // exponentials (the dO stage after the first chunk, as the producer reloads it a step
    // ahead; the Q stage after the last)
    int lent_stage = -1;
    auto return_stage = [&]() {
      if (lane == 0) {
        bulk_wait_read0();
        mbar_arrive(half ? &do_borrow[lent_stage] : &q_borrow[lent_stage]);
      }
      lent_stage = -1;
    };
    for (;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      const Item I = item_of(item);
      const int k0 = I.n * 128;
      const int j = k0 + r;
      // the item's first stored dS^T tile (key tile n of batch b, query head 0)
      const long long tile0 = ((long long)I.b * p.Hq - (long long)p.blk0 * G) * p.tiles_per_bh +
                              ds_tiles_before(I.n, p.n_tiles, p.span);
      for (int it = 0; it < I.n_iters; ++it) {
        const int g = g0 + it;
        const int q0 = (I.n + it % I.m_cnt) * 128 + kSCols * half;  // first query of this thread's columns
        if (tracer) CSWA_MARK(trole, g, 0);
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, g & 1, abort_flag));
        if (tracer) CSWA_MARK(trole, g, 1);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[kSCols];
#pragma unroll
        for (int h32 = 0; h32 < kSCols; h32 += 32) tmem_ld32(tR0 + cols + h32, *reinterpret_cast<uint32_t(*)[32]>(&sr[h32]));
        tmem_ld_wait();
        if (tracer) CSWA_MARK(trole, g, 2);
        const bool full = (k0 + 127 <= q0) && (W < 0 || q0 + kSCols - 1 - k0 <= W);
        const int c_lo = j - q0;                              // query q0 + c sees key j iff c >= c_lo
        const int c_hi = (W < 0) ? kSCols - 1 : j + W - q0;   //   and c <= c_hi
        // P = exp2(scale log2e (S - lse/scale)): the MMA has already added -lse/scale, so
        // one packed multiply per two columns; masked entries are set to 0 after the exp2,
        // tiles inside the band skip the mask (a warp-uniform branch). P^T goes back to
        // TMEM in kPChunks chunks of 16 queries, each published on its own barrier so that
        // dV starts on the first while the rest is computed. Chunk c's bf16 pairs land in
        // the group's columns 8c..8c+7, whose fp32 S^T (queries <= 16c+15) is already in
        // registers.
        const float2 sl2v = make_float2(sl2, sl2);
        // Chunk c+1's exponentials are computed while chunk c's TMEM store completes: the
        // wait for a chunk's store, and its publication, come after the next chunk's math.
        uint32_t pkb[2][8];
        auto publish = [&](int c) {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_chunk[c]);
          if (tracer && c == 0) CSWA_MARK(trole, g, 3);
          if (lent_stage >= 0 && c == (half ? 0 : kPChunks - 1)) return_stage();
        };
#pragma unroll
        for (int c = 0; c < kPChunks; ++c) {
          uint32_t(&pk)[8] = pkb[c & 1];
#pragma unroll
          for (int c2 = 8 * c; c2 < 8 * c + 8; ++c2) {
            const float2 e = __fmul2_rn(make_float2(__uint_as_float(sr[2 * c2]), __uint_as_float(sr[2 * c2 + 1])), sl2v);
            float y[2] = {ex2_approx(e.x), ex2_approx(e.y)};
            if (!full) {
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int col = 2 * c2 + u;
                y[u] = ((col >= c_lo) & (col <= c_hi)) ? y[u] : 0.f;
              }
            }
            sr[2 * c2] = __float_as_uint(y[0]);
            sr[2 * c2 + 1] = __float_as_uint(y[1]);
            pk[c2 - 8 * c] = pack_bf16x2(y[0], y[1]);
          }
          if (c > 0) publish(c - 1);
          tmem_st8(tR0 + cols + 8 * c, pk);
        }
        publish(kPChunks - 1);
        const float* pf = reinterpret_cast<const float*>(sr);
        if (tracer) CSWA_MARK(trole, g, 4);

        ok = __all_sync(0xffffffffu, mbar_wait(dp_full, g & 1, abort_flag));
        if (!ok) break;
        if (tracer) CSWA_MARK(trole, g, 5);
        tc_fence_after();
        // dS = P * (dP - Delta): the MMA has already subtracted Delta; one packed multiply
        // per two columns, 32 columns at a time
#pragma unroll
        for (int hc = 0; hc < kSCols / 32; ++hc) {
          uint32_t dp[32];
          tmem_ld32(tR1 + cols + 32 * hc, dp);
          tmem_ld_wait();
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            const int c = 32 * hc + 2 * c2;
            const float2 d = __fmul2_rn(make_float2(pf[c], pf[c + 1]),
                                        make_float2(__uint_as_float(dp[2 * c2]), __uint_as_float(dp[2 * c2 + 1])));
            dsk[c / 2] = pack_bf16x2(d.x, d.y);
          }
        }
        if (tracer) CSWA_MARK(trole, g, 6);
        // over this thread's own (already read) dP^T columns
        if constexpr (kSCols == 64)
          tmem_st32(tR1 + cols, *reinterpret_cast<uint32_t(*)[32]>(dsk));
        else
          tmem_st16(tR1 + cols, *reinterpret_cast<uint32_t(*)[16]>(dsk));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(ds_full);
        if (tracer) CSWA_MARK(trole, g, 7);
        const long long tile = tile0 + (long long)(I.hk * G + it / I.m_cnt) * p.tiles_per_bh + it % I.m_cnt;
        uint8_t* const ds_dst =
            reinterpret_cast<uint8_t*>(p.ds) + (size_t)tile * 32768 + ds_unit_offset(r, (kSCols / 8) * half);
#pragma unroll
        for (int u = 0; u < kSCols / 8; ++u)
          *reinterpret_cast<uint4*>(ds_dst + u * 512) = make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]);
      }
      if (!ok) break;
      // column groups past the first two have no epilogue: on to the next item
      if (half >= 2) {
        g0 += I.n_iters;
        continue;
      }
      // ------------------------------------------------------ dK (warps 4-7) / dV (8-11) epilogue
      // Thread = key row j of the tile. The accumulator goes to bf16 in the ring stage
      // of the item's last step (the Q stage for dK, the dO stage for dV: lent by the
      // producers, whose last reader -- the last dK or dV MMA -- has completed), in the
      // 128-byte-swizzled layout of a TMA tile; each warp then stores its 32 rows with
      // one TMA store per 64-column panel (rows past T are not written) and returns the
      // stage once the stores have read it. dV is complete as soon as the last dV MMA
      // is (it released its dO stage), a step ahead of dK.
      const int g_last = g0 + I.n_iters - 1;
      const int st_last = half ? g_last % DS : g_last % QS;
      uint8_t* stage = smem + (half ? L::kDO : L::kQ) + st_last * L::kTile;
      // (profiling builds: epilogue marks of the CTA's first 8 items at steps 56-63)
      const int emark = 56 + (k & 7);
      (void)emark;
      if (tracer && k < 8) CSWA_MARK(trole, emark, 0);
      ok = __all_sync(0xffffffffu, half ? mbar_wait(&do_empty[st_last], (g_last / DS) & 1, abort_flag)
                                        : mbar_wait(final_bar, k & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      if (tracer && k < 8) CSWA_MARK(trole, emark, 1);
      const uint32_t src = (half ? tdV : tdK) + lane_off;
      if (!half && p.rope) {
        // dk with respect to the raw k: the prologue backward on the way out. The raw
        // tile goes into the stage now (it was on its way to L2 since the item began)
        // while dy is rotated back in TMEM; then the row statistics, then dx in place.
        if (warp == 4 && lane == 0) {
          mbar_arrive_expect_tx(kr_full, L::kTile);
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_4d(stage + pn * L::kPanel, &tm_kr, kr_full, pn * 64, I.hk, k0, I.b);
          kr_pending = k;
        }
        constexpr int H = D / 2;
#pragma unroll 1
        for (int j0 = 0; j0 < H; j0 += 16) {
          uint32_t ta[16], tb[16];
          tmem_ld16(src + j0, ta);
          tmem_ld16(src + H + j0, tb);
          tmem_ld_wait();
          float a[16], b[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) a[u] = __uint_as_float(ta[u]) * p.scale, b[u] = __uint_as_float(tb[u]) * p.scale;
          rope_rotate_back<D>(p.turns, (unsigned)j, j0, a, b);
#pragma unroll
          for (int u = 0; u < 16; ++u) ta[u] = __float_as_uint(a[u]), tb[u] = __float_as_uint(b[u]);
          tmem_st16(src + j0, ta);
          tmem_st16(src + H + j0, tb);
        }
        tmem_st_wait();
        ok = __all_sync(0xffffffffu, mbar_wait(kr_full, k & 1, abort_flag));
        if (!ok) break;
        if (warp == 4 && lane == 0) kr_pending = -1;
        float ss = 0.f, gx = 0.f;
#pragma unroll 1
        for (int j0 = 0; j0 < H; j0 += 16) {
          uint32_t ta[16], tb[16];
          tmem_ld16(src + j0, ta);
          tmem_ld16(src + H + j0, tb);
          float xa[16], xb[16];
          tile_ld16(stage, r, j0, xa);
          tile_ld16(stage, r, H + j0, xb);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            ss = fmaf(xa[u], xa[u], fmaf(xb[u], xb[u], ss));
            gx = fmaf(__uint_as_float(ta[u]), xa[u], fmaf(__uint_as_float(tb[u]), xb[u], gx));
          }
        }
        const float inv_r = rsqrtf(ss * (1.f / D) + p.eps);
        const float c1 = gx * inv_r * inv_r * (1.f / D);  // (g . xh) / D, applied to x / r
#pragma unroll 1
        for (int j0 = 0; j0 < H; j0 += 16) {
          uint32_t ta[16], tb[16];
          tmem_ld16(src + j0, ta);
          tmem_ld16(src + H + j0, tb);
          float xa[16], xb[16];
          tile_ld16(stage, r, j0, xa);
          tile_ld16(stage, r, H + j0, xb);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            xa[u] = (__uint_as_float(ta[u]) - xa[u] * c1) * inv_r;
            xb[u] = (__uint_as_float(tb[u]) - xb[u] * c1) * inv_r;
          }
          tile_st16(stage, r, j0, xa);
          tile_st16(stage, r, H + j0, xb);
        }
      } else {
        // 64 columns per TMEM round trip (four loads, one wait)
        const float mul = half ? 1.f : p.scale;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) {
          uint32_t t[4][16];
#pragma unroll
          for (int e = 0; e < 4; ++e) tmem_ld16(src + c0 + 16 * e, t[e]);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = __uint_as_float(t[e][u]) * mul;
            tile_st16(stage, r, c0 + 16 * e, v);
          }
        }
      }
      if (tracer && k < 8) CSWA_MARK(trole, emark, 2);
      // the accumulators may take the next item's first products
      tc_fence_before();
      mbar_arrive(acc_free);
      // the warp's 32 rows leave as TMA stores; the stage goes back to the producer
      // once they have read it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int pn = 0; pn < D / 64; ++pn)
          tma_store_4d(half ? &tm_dv : &tm_dk, stage + pn * L::kPanel + quarter * 4096, pn * 64, I.hk, k0 + 32 * quarter,
                       I.b);
        bulk_commit();
        if (tracer && k < 8) CSWA_MARK(trole, emark, 3);
      }
      lent_stage = st_last;
      g0 += I.n_iters;
    }
    if (lent_stage >= 0) return_stage();
    // before the CTA's shared memory goes: the stores have completed, and a raw k load
    // left behind by an abort has landed
    if (lane == 0) bulk_wait0();
    if (kr_pending >= 0) mbar_drain(kr_full, kr_pending & 1);
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// dQ = scale * sum_n dS(m, n) K_n for every 128-row query tile m of every query
// head, from the dS^T tiles bwd_main stored; accumulated in TMEM, written once as bf16.
// Persistent: one CTA per SM takes (m, h, b) items from a global counter (warp 3
// claims them). A 3-stage ring of (dS^T tile, K tile) runs on across items, and two
// TMEM accumulators let the epilogue of one item overlap the MMAs of the next. The
// epilogue (warps 4-7, thread = query row) turns the accumulator into bf16 rows of a
// staging tile that each warp stores with TMA (its 32 rows); for the block backward
// the warp first loads its 32 raw q rows there by TMA and writes dq in their place.
template <int D>
struct DqLayout {
  static constexpr int kStages = 3;
  static constexpr int kDS = 32768;            // one dS^T tile (128 keys x 128 queries bf16)
  static constexpr int kK = 128 * D * 2;       // one K tile
  static constexpr int kStage = kDS + kK;
  static constexpr int kX = kStages * kStage;  // the epilogue's staging tile (128 rows)
  static constexpr int kBar = kX + 128 * D * 2;
  static constexpr int kBytes = kBar + 256 + 1024;
  static constexpr uint32_t kTmemCols = 2 * D;  // two accumulators
};

// tm_qr: the raw q (block backward only), tm_dq: the output; both 32-row boxes.
template <int D>
__global__ void __launch_bounds__(256, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_qr,
                       const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ BwdParams p,
                       int n_items) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* full = bars;                   // [kStages]
  uint64_t* empty = bars + L::kStages;     // [kStages]
  uint64_t* acc_full = bars + 2 * L::kStages;       // [2] an item's dQ is in TMEM
  uint64_t* acc_empty = acc_full + 2;               // [2] the epilogue has read it
  uint64_t* final_bar = acc_empty + 2;
  uint64_t* item_full = final_bar + 1;     // the next work item's index is in item_slot
  uint64_t* item_empty = item_full + 1;    // every role has read it
  uint64_t* x_full = item_empty + 1;       // [4] an epilogue warp's raw q rows have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x_full + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(x_full + 5);
  volatile int* item_slot = reinterpret_cast<volatile int*>(x_full + 6);

  const int warp = warp_id(), lane = lane_id();
  // item -> (query tile m, head h, batch b) in super-block order with the heaviest
  // query tiles (the most key tiles) first, and the key tiles n whose query range
  // [n, n + span - 1] holds m; items are handed out first come first served. The blocks
  // go in the reverse of the main kernel's order: the dS^T tiles it wrote last are the
  // ones still in L2 when this kernel starts.
  auto item_of = [&](int item, int& m, int& h, int& b, int& n_lo, int& steps) {
    int t, blk;
    const int n_blocks = n_items / p.n_tiles;
    sb_order(item, p.n_tiles, n_blocks, t, blk);
    blk = n_blocks - 1 - blk + p.blk0 * p.G;  // the pass's query-head blocks: G per KV block
    m = p.n_tiles - 1 - t;
    h = blk % p.Hq;
    b = blk / p.Hq;
    n_lo = max(0, m - p.span + 1);
    steps = m - n_lo + 1;
  };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 128);
    }
    mbar_init(final_bar, 1);
    mbar_init(item_full, 1);
    mbar_init(item_empty, 6);  // warps 0, 1 and the four epilogue warps
    for (int q = 0; q < 4; ++q) mbar_init(&x_full[q], 1);
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
  // the k-th work item of this CTA (-1: none left, or the CTA gave up), read by a whole
  // warp; one lane releases the slot for the role
  auto take_item = [&](int k) {
    int v = mbar_wait(item_full, k & 1, abort_flag) ? *item_slot : -1;
    v = __shfl_sync(0xffffffffu, v, 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(item_empty);
    return v;
  };

  if (warp == 0) {
    // producer: the whole warp takes the items, lane 0 issues
    int last_issue[L::kStages];
    for (int s = 0; s < L::kStages; ++s) last_issue[s] = -1;
    if (lane == 0) tma_prefetch_desc(&tm_k);
    int g = 0;  // ring step counter across items
    bool ok = true;
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      if (lane == 0) {
        int m, h, b, n_lo, steps;
        item_of(item, m, h, b, n_lo, steps);
        const long long bh_base = ((long long)b * p.Hq + h - (long long)p.blk0 * p.G) * p.tiles_per_bh;
        for (int i = 0; i < steps; ++i, ++g) {
          const int st = g % L::kStages;
          const int n = n_lo + i;
          if (!(ok = mbar_wait(&empty[st], ((g / L::kStages) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&full[st], L::kDS + L::kK);
          const long long tile = bh_base + ds_tiles_before(n, p.n_tiles, p.span) + (m - n);
          uint8_t* dst = smem + st * L::kStage;
          bulk_load(dst, reinterpret_cast<const uint8_t*>(p.ds) + (size_t)tile * L::kDS, L::kDS, &full[st]);
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_4d(dst + L::kDS + pn * 16384, &tm_k, &full[st], pn * 64, h / p.G, n * 128, b);
          last_issue[st] = g;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    if (lane == 0) {
      // every copy in flight lands before the CTA's shared memory is released
      for (int s = 0; s < L::kStages; ++s)
        if (last_issue[s] >= 0) mbar_drain(&full[s], (last_issue[s] / L::kStages) & 1);
    }
  } else if (warp == 1) {
    // whole warp runs the loop, one elected lane issues
    const uint32_t leader = elect_one();
    constexpr uint32_t id = idesc_bf16(128, D, true, true);  // A = dS (queries contiguous), B = K (d contiguous)
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    int g = 0;
    bool ok = true;
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      int m, h, b, n_lo, steps;
      item_of(item, m, h, b, n_lo, steps);
      const int buf = k & 1;
      // the epilogue has drained this accumulator (item k - 2)
      if (!(ok = wait_all(&acc_empty[buf], ((k >> 1) & 1) ^ 1))) break;
      for (int i = 0; i < steps; ++i, ++g) {
        const int st = g % L::kStages;
        if (!(ok = wait_all(&full[st], (g / L::kStages) & 1))) break;
        tc_fence_after();
        const uint32_t sds = sbase + st * L::kStage, sk = sds + L::kDS;
        // A = dS (M = queries, K = keys) in the stored unit order: 128 bytes between
        // core matrices along K, 512 along M; 16 keys per MMA = (kk / 2) * 8 KB + (kk & 1) * 256
        const uint64_t da = sdesc_noswz(sds, 128, 512), db = sdesc_sw128(sk, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + buf * D, da + ((ds_unit_offset(16 * kk, 0)) >> 4), db + ((kk * 2048) >> 4), id,
                 (i > 0 || kk > 0), leader);
        mma_commit(&empty[st], leader);
      }
      if (!ok) break;
      mma_commit(&acc_full[buf], leader);
    }
    mma_commit(final_bar, leader);
    mbar_drain(final_bar, 0);
  } else if (warp == 3) {
    // work scheduler: claims the CTA's next item from the global counter once every
    // role has read the previous one; -1 when none is left
    if (lane == 0) {
      for (int k = 0;; ++k) {
        if (!mbar_wait(item_empty, (k & 1) ^ 1, abort_flag)) break;
        const int idx = atomicAdd(p.item_counter + 1, 1);
        const int v = idx < n_items ? idx : -1;
        *item_slot = v;
        mbar_arrive(item_full);
        if (v < 0) break;
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* xs = smem + L::kX;  // this warp's rows: 32 * quarter .. + 31 of each panel
    int x_pending = -1;          // lane 0: the item whose raw q load nobody has waited for yet
    for (int k = 0;; ++k) {
      const int item = take_item(k);
      if (item < 0) break;
      int m, h, b, n_lo, steps;
      item_of(item, m, h, b, n_lo, steps);
      const int buf = k & 1;
      const int i = m * 128 + row;
      if (lane == 0) {
        // the previous item's stores must have read the rows before they are reused
        bulk_wait_read0();
        if (p.rope) {
          mbar_arrive_expect_tx(&x_full[quarter], 32 * D * 2);
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_4d(xs + pn * 16384 + quarter * 4096, &tm_qr, &x_full[quarter], pn * 64, h, m * 128 + 32 * quarter,
                        b);
          x_pending = k;
        }
      }
      __syncwarp();
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (k >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t src = tmem + buf * D + lane_off;
      if (p.rope) {
        // dq with respect to the raw q: dy rotated back in TMEM, the row statistics, then
        // dx written over the raw row
        constexpr int H = D / 2;
#pragma unroll 1
        for (int j0 = 0; j0 < H; j0 += 16) {
          uint32_t ta[16], tb[16];
          tmem_ld16(src + j0, ta);
          tmem_ld16(src + H + j0, tb);
          tmem_ld_wait();
          float a[16], bb[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) a[u] = __uint_as_float(ta[u]) * p.scale, bb[u] = __uint_as_float(tb[u]) * p.scale;
          rope_rotate_back<D>(p.turns, (unsigned)i, j0, a, bb);
#pragma unroll
          for (int u = 0; u < 16; ++u) ta[u] = __float_as_uint(a[u]), tb[u] = __float_as_uint(bb[u]);
          tmem_st16(src + j0, ta);
          tmem_st16(src + H + j0, tb);
        }
        tmem_st_wait();
        if (!__all_sync(0xffffffffu, mbar_wait(&x_full[quarter], k & 1, abort_flag))) break;
        if (lane == 0) x_pending = -1;
        float ss = 0.f, gx = 0.f;
#pragma unroll 1
        for (int j0 = 0; j0 < H; j0 += 16) {
          uint32_t ta[16], tb[16];
          tmem_ld16(src + j0, ta);
          tmem_ld16(src + H + j0, tb);
          float xa[16], xb[16];
          tile_ld16(xs, row, j0, xa);
          tile_ld16(xs, row, H + j0, xb);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            ss = fmaf(xa[u], xa[u], fmaf(xb[u], xb[u], ss));
            gx = fmaf(__uint_as_float(ta[u]), xa[u], fmaf(__uint_as_float(tb[u]), xb[u], gx));
          }
        }
        const float inv_r = rsqrtf(ss * (1.f / D) + p.eps);
        const float c1 = gx * inv_r * inv_r * (1.f / D);
#pragma unroll 1
        for (int j0 = 0; j0 < H; j0 += 16) {
          uint32_t ta[16], tb[16];
          tmem_ld16(src + j0, ta);
          tmem_ld16(src + H + j0, tb);
          float xa[16], xb[16];
          tile_ld16(xs, row, j0, xa);
          tile_ld16(xs, row, H + j0, xb);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            xa[u] = (__uint_as_float(ta[u]) - xa[u] * c1) * inv_r;
            xb[u] = (__uint_as_float(tb[u]) - xb[u] * c1) * inv_r;
          }
          tile_st16(xs, row, j0, xa);
          tile_st16(xs, row, H + j0, xb);
        }
      } else {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) {
          uint32_t t[4][16];
#pragma unroll
          for (int e = 0; e < 4; ++e) tmem_ld16(src + c0 + 16 * e, t[e]);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = __uint_as_float(t[e][u]) * p.scale;
            tile_st16(xs, row, c0 + 16 * e, v);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int pn = 0; pn < D / 64; ++pn)
          tma_store_4d(&tm_dq, xs + pn * 16384 + quarter * 4096, pn * 64, h, m * 128 + 32 * quarter, b);
        bulk_commit();
      }
      (void)i;
    }
    if (lane == 0) {
      bulk_wait0();
      if (x_pending >= 0) mbar_drain(&x_full[quarter], x_pending & 1);
    }
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Row extensions of the S^T and dP^T MMAs. For each query row i (padded to 128-row
// tiles) x = -lse_i / scale and y = -Delta_i = -(dO_i . o_i) are split into bf16
// pairs hi + lo (hi = bf16(x), lo = bf16(x - hi): together 16 significant bits), so
// that one extra K = 16 MMA step against key-side rows (1, 1, 0, ...) adds x (or y)
// to every entry of query column i in fp32. Padded rows get x = -1e30 (finite: the
// MMA also multiplies these bytes by zero; exp2 of it is 0) and y = 0.
// Per (batch, head, query tile) 512 bytes: for each group g of 8 rows, 16 bytes of
// the 8 hi values then 16 bytes of the 8 lo values (the MN-major no-swizzle layout:
// one core row per K index). D/8 lanes per (b, t, h) row.
struct PrepParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  uint8_t* ext_lse;
  uint8_t* ext_delta;
  int* item_counter;
  int B, T, Tpad, Hq;
  int chunks;  // chunks of 2 * 256 / (D / 16) rows per batch
  float inv_scale;
};

template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __grid_constant__ PrepParams p) {
  // A chunk is kRows * kRowsPerPass consecutive (t, h) rows of one batch, t over the
  // padded length; the blocks (a few per SM, resident together) take the B * chunks
  // chunks in turn, so that no partial last wave of short blocks is left. LK lanes per
  // row, 16 elements each; every thread takes kRows rows (r0 + u * kRowsPerPass) of a
  // chunk with all their loads in flight before the sums, and forms o . dO with mixed
  // bf16 x bf16 -> fp32 FMAs (no conversions).
  constexpr int LK = D / 16;
  constexpr int kRows = 2, kRowsPerPass = 256 / LK;
  // the main and dQ kernels that follow on the stream hand out their work items from
  // these two counters
  if (blockIdx.x == 0 && threadIdx.x < 2) p.item_counter[threadIdx.x] = 0;
  const int T = p.T, Tpad = p.Tpad, Hq = p.Hq;
  const int rows = Tpad * Hq;  // < 2^31 (the host checks the stored tile rows, which bound it)
  const int lr = (int)threadIdx.x % LK;
  for (long long ch = blockIdx.x; ch < (long long)p.B * p.chunks; ch += gridDim.x) {
    const int b = (int)(ch / p.chunks);
    const int r0 = (int)(ch - (long long)b * p.chunks) * (kRows * kRowsPerPass) + (int)threadIdx.x / LK;
    int hh[kRows], tt[kRows];
    bool real[kRows];
    uint4 ov[kRows][2], gv[kRows][2];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int r = r0 + u * kRowsPerPass;
      tt[u] = r / Hq;
      hh[u] = r - tt[u] * Hq;
      real[u] = r < rows && tt[u] < T;
#pragma unroll
      for (int e = 0; e < 2; ++e) ov[u][e] = gv[u][e] = make_uint4(0, 0, 0, 0);
      if (real[u]) {
        const size_t off = ((size_t)((size_t)b * T + tt[u]) * Hq + hh[u]) * D + lr * 16;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          ov[u][e] = *reinterpret_cast<const uint4*>(p.o + off + 8 * e);
          gv[u][e] = *reinterpret_cast<const uint4*>(p.dout + off + 8 * e);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int r = r0 + u * kRowsPerPass;
      const int h = hh[u], t = tt[u];
      float dsum = 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        dsum = fma_bf16x2_f32(ov[u][e].x, gv[u][e].x, dsum);
        dsum = fma_bf16x2_f32(ov[u][e].y, gv[u][e].y, dsum);
        dsum = fma_bf16x2_f32(ov[u][e].z, gv[u][e].z, dsum);
        dsum = fma_bf16x2_f32(ov[u][e].w, gv[u][e].w, dsum);
      }
#pragma unroll
      for (int sh = LK / 2; sh >= 1; sh >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, sh);
      if (r < rows && lr == 0) {
        // clamped to stay finite in bf16 (a huge 1/scale must not turn x into -inf)
        const float x = real[u] ? fminf(fmaxf(-p.lse[((size_t)b * Hq + h) * T + t] * p.inv_scale, -3.0e38f), 3.0e38f)
                                : -1e30f;
        const float y = real[u] ? -dsum : 0.f;
        const int i = t & 127;
        const size_t at = (((size_t)b * Hq + h) * (Tpad / 128) + t / 128) * 512 + (i >> 3) * 32 + (i & 7) * 2;
        const __nv_bfloat16 xh = __float2bfloat16_rn(x), yh = __float2bfloat16_rn(y);
        *reinterpret_cast<__nv_bfloat16*>(p.ext_lse + at) = xh;
        *reinterpret_cast<__nv_bfloat16*>(p.ext_lse + at + 16) = __float2bfloat16_rn(x - __bfloat162float(xh));
        *reinterpret_cast<__nv_bfloat16*>(p.ext_delta + at) = yh;
        *reinterpret_cast<__nv_bfloat16*>(p.ext_delta + at + 16) = __float2bfloat16_rn(y - __bfloat162float(yh));
      }
    }
  }
}

}  // namespace cswa
