// attn_fwd: causal sliding-window GQA attention forward on tcgen05 / TMEM.
//
// Computes, per (batch b, query head h, query row i), over the visible keys
// j (j <= i and, for window W >= 0, i - j <= W) of KV head h / G:
//   o_i = softmax_j(scale * <q_i, k_j>) v_j,   lse_i = log sum_j exp(scale * <q_i, k_j>)
// (nanochat Admin & Developer Guide, 3 "Sliding-window attention" and 6 "Attention:
// FA3 with SDPA Fallback"; nanoGPT Administrator & Developer Guide, 8
// "CausalSelfAttention", manual path).
//
// One CTA owns two 128-row query tiles ("slots") of one (b, h): tiles 2p and
// 2p+1. It walks the union of their key-tile ranges inside the causal/window
// band; key tiles outside the band are never loaded. With an even group size G
// the training forward pairs two query heads of one KV group at the same query
// tile instead: both slots then see the same key tiles, and no key tile is
// walked by one slot alone (the first and last tiles of a tile pair are).
//   warp 0      TMA producer: Q once, then K and V tiles into 2-stage rings
//   warp 1      MMA issuer (whole warp, one elected lane issues): S_s = Q_s K^T (SS),
//               O_s += P_s V (TS)
//   warp 2      TMEM allocator
//   warps 4-7   softmax + epilogue for slot 0 (thread = query row)
//   warps 8-11  softmax + epilogue for slot 1
// TMEM (512 columns): S0 | S1 | O0 | O1. P_s (bf16) overwrites the first half
// of S_s in place and feeds the PV product straight from tensor memory.
// Softmax runs in the log2 domain; the running max is only moved (and O
// rescaled) when it grows by more than 2^8, which leaves the result exact.
//
// Chunked prefill (kCache): the queries are a chunk of T new tokens of each
// sequence, chunk row t at position pos[b] + t, and the keys and values are the
// sequence's KV cache, which already holds the chunk's own entries (nanochat Admin
// & Developer Guide, 6 "Attention: FA3 with SDPA Fallback": chunked / sliding-window
// inference over a cache; 7 "KV cache"). No cache row past the chunk's last token
// (unwritten, possibly NaN) may reach a product, since 0 * NaN would poison the
// rows that mask it. Two tile grids ensure that:
//  * chunk given (k_new / v_new): the grid is anchored at the chunk's START. Key
//    tile t >= 0 is read from k_new / v_new (rows past T are the TMA's zero fill),
//    t < 0 from the cache (the last such tile ends at pos[b] - 1). The kernel never
//    reads the cache at or past pos[b], so warp 3 copies the chunk into the cache
//    while the tiles are computed (the CTA of the group's first query head copies
//    its own query tiles' rows).
//  * chunk already in the cache: the grid is anchored at the chunk's END. Query
//    tile qt covers chunk rows 128 qt - shift .. with shift = 128 ceil(T/128) - T,
//    key tile t covers cache rows pos[b] - shift + 128 t .., so the last key row
//    loaded is the chunk's last token.
// Rows before the chunk or before position 0 come from the TMA's zero fill and are
// masked. The (sequence, pair) items are ranked by their key-tile count (read from
// pos on the device) and handed to the CTAs heaviest first, so the last wave of
// CTAs holds the lightest items.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int T, Hq, G, window;
  float scale_log2;  // scale * log2(e)
  int nq_tiles;
  int n_pairs;
  // chunked prefill only
  const int32_t* pos;  // (B) entries already in each cache = position of chunk row 0
  int Tmax;            // cache rows
  int shift;           // 128 * nq_tiles - T, or 0 when the chunk comes from kn / vn
  int B, Hkv;
  const uint4* kn;     // the chunk's k / v (B, T, Hkv, D), or null
  const uint4* vn;
  uint4* kc;           // the caches (B, Tmax, Hkv, D)
  uint4* vc;
  // fp8 forward only: the dequantization factors of q, k, v (device memory, 3 floats)
  const float* descale;
  // training forward with G even: the two slots are query heads 2x and 2x + 1 (one KV
  // group) at the same query tile, so that both walk the same key tiles (0: the slots
  // are query tiles 2p and 2p + 1 of one head)
  int head_pairs;
};

constexpr int kMaxRankedItems = 256;  // prefill items ranked by weight (more: pair order)

template <int D, bool kFp8 = false>
struct FwdLayout {
  static constexpr int kElem = kFp8 ? 1 : 2;  // bytes per element: e4m3 or bf16
  static constexpr int kTile = 128 * D * kElem;  // bytes of one 128-row tile
  static constexpr int kPanels = D * kElem / 128;  // 128-byte-wide panels per tile
  static constexpr int kQ0 = 0, kQ1 = kTile, kK0 = 2 * kTile, kV0 = 4 * kTile;
  static constexpr int kBar = 6 * kTile;
  static constexpr int kBytes = kBar + 256 + 1024;  // + barriers + alignment slack
  static constexpr uint32_t kTmemCols = 512;
};

constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D, bool kCache = false, bool kFp8 = false>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams p) {
  static_assert(!kFp8 || (D == 128 && !kCache), "the fp8 forward takes D = 128, training layout");
  using L = FwdLayout<D, kFp8>;
  constexpr int kPanelElems = 128 / L::kElem;  // elements across one 128-byte panel
  // the bf16 training forward writes o with TMA stores from the slot's Q tile (tm_o:
  // 32-row boxes); the prefill and the fp8 forward store rows directly
  constexpr bool kTmaO = !kCache && !kFp8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* k_empty = bars + 5;   // [2] S of the tile has read K
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* pv_done = bars + 11;  // [2]
  uint64_t* final_bar = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);
  uint64_t* v_empty = bars + 16;  // [2] PV of the tile has read V
  uint64_t* p_chunk = bars + 18;  // [2][4] P_s of keys 32c .. 32c+31 written over S_s

  const int warp = warp_id(), lane = lane_id();
  const int hp = p.head_pairs;
  const int h = hp ? 2 * blockIdx.x : blockIdx.x;  // the first slot's query head
  auto head_of = [&](int s) { return h + (hp ? s : 0); };
  int b = blockIdx.y;
  int pair = p.n_pairs - 1 - blockIdx.z;  // heaviest tiles first
  const int hk = h / p.G;
  const int W = p.window;
  // e0: position of tile row 0 (0 in training); shift: chunk row of a tile's first row
  // is 128 qt - shift (0 in training)
  int e0 = 0, shift = 0, P = 0;
  // first key tile of query tile q: the one holding its first row's oldest visible
  // key (an arithmetic shift: the floor also for the negative tiles of kCache)
  auto lo_of_at = [&](int base, int q) { return (((W < 0) ? 0 : max(0, base + q * 128 - W)) - base) >> 7; };
  if constexpr (kCache) {
    shift = p.shift;
    const int n_items = p.B * p.n_pairs;
    if (n_items <= kMaxRankedItems) {
      // rank the (sequence, pair) items by key tiles, heaviest first (ties: lower index
      // first); the CTA at launch rank blockIdx.z * B + blockIdx.y takes that rank's item
      int* w = reinterpret_cast<int*>(smem + L::kV0 + L::kTile);  // free until the first V load
      int* order = w + kMaxRankedItems;
      for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const int bi = i / p.n_pairs, pi = i - bi * p.n_pairs;
        const int Pi = p.pos[bi];
        int wt = -1;  // an item out of range only reports and leaves: last
        if (Pi >= 0 && Pi <= p.Tmax - p.T) {
          wt = 0;
          for (int s2 = 0; s2 < 2; ++s2) {
            const int q = 2 * pi + s2;
            if (q < p.nq_tiles) wt += q - lo_of_at(Pi - shift, q) + 1;
          }
        }
        w[i] = wt;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const int wi = w[i];
        int r = 0;
        for (int j = 0; j < n_items; ++j) r += (w[j] > wi) | ((w[j] == wi) & (j < i));
        order[r] = i;
      }
      __syncthreads();
      const int item = order[blockIdx.z * p.B + blockIdx.y];
      b = item / p.n_pairs;
      pair = item - b * p.n_pairs;
      __syncthreads();  // the scratch is V stage 1: read before anything else touches it
    }
    P = p.pos[b];
    if (P < 0 || P > p.Tmax - p.T) {  // uniform over the CTA: nothing allocated yet
      if (threadIdx.x == 0) atomicOr(&g_status, kStatusBadPosition);
      return;
    }
    e0 = P - shift;
  }
  auto lo_of = [&](int q) { return lo_of_at(e0, q); };

  int qt[2], lo[2], hi[2];
  bool has[2];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    qt[s] = hp ? pair : 2 * pair + s;
    has[s] = qt[s] < p.nq_tiles;
    hi[s] = qt[s];
    lo[s] = lo_of(qt[s]);
  }
  const int t_lo = lo[0];
  const int t_hi = has[1] ? hi[1] : hi[0];

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      for (int c = 0; c < 4; ++c) mbar_init(&p_chunk[4 * s + c], 128);
      mbar_init(&pv_done[s], 1);
    }
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
  // TMEM columns of slot s: S_s at 128*s, O_s at 256 + D*s
  auto tS = [&](int s) { return tmem + 128u * s; };
  auto tO = [&](int s) { return tmem + 256u + (uint32_t)D * s; };

  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (kCache && p.kn) {
        tma_prefetch_desc(&tm_kn);
        tma_prefetch_desc(&tm_vn);
      }
      mbar_arrive_expect_tx(q_full, (has[1] ? 2 : 1) * L::kTile);
      for (int s = 0; s < 2; ++s)
        if (has[s])
          for (int pn = 0; pn < L::kPanels; ++pn)
            tma_load_4d(smem + (s ? L::kQ1 : L::kQ0) + pn * 16384, &tm_q, q_full, pn * kPanelElems, head_of(s),
                        qt[s] * 128 - shift, b);
      // K and V stages are released separately (K once the S products have read it, V
      // once the PV products have), so K of the next tile loads a whole tile ahead
      int n = 0, last_k[2] = {-1, -1}, last_v[2] = {-1, -1};
      for (int t = t_lo; t <= t_hi; ++t, ++n) {
        const int st = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        // key tiles at or past the chunk's start come from k_new / v_new when given
        const bool fresh = kCache && p.kn && t >= 0;
        const CUtensorMap* mk = fresh ? &tm_kn : &tm_k;
        const CUtensorMap* mv = fresh ? &tm_vn : &tm_v;
        const int row = fresh ? t * 128 : e0 + t * 128;
        if (!mbar_wait(&k_empty[st], ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[st], L::kTile);
        for (int pn = 0; pn < L::kPanels; ++pn)
          tma_load_4d(smem + L::kK0 + st * L::kTile + pn * 16384, mk, &k_full[st], pn * kPanelElems, hk, row, b);
        last_k[st] = n;
        if (!mbar_wait(&v_empty[st], ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&v_full[st], L::kTile);
        for (int pn = 0; pn < L::kPanels; ++pn)
          tma_load_4d(smem + L::kV0 + st * L::kTile + pn * 16384, mv, &v_full[st], pn * kPanelElems, hk, row, b);
        last_v[st] = n;
      }
      // never leave with copies in flight: wait (bounded) for the last load of each
      // stage. After a normal run they were all consumed and these return at once; after
      // an abort (raised by any role, before or after this loop ended) they may not be.
      for (int st = 0; st < 2; ++st) {
        if (last_k[st] >= 0) mbar_drain(&k_full[st], (last_k[st] >> 1) & 1);
        if (last_v[st] >= 0) mbar_drain(&v_full[st], (last_v[st] >> 1) & 1);
      }
      mbar_drain(q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); one elected lane
    // issues. MMAs run in issue order, so S_s of the next key tile, issued after PV_s
    // of this one, never overwrites P_s before PV_s has read it, and the softmax warps,
    // which see S_s only through a commit issued after PV_s, find O_s stable.
    const uint32_t leader = elect_one();
    constexpr uint32_t idS = kFp8 ? idesc_e4m3(128, 128, false, false) : idesc_bf16(128, 128, false, false);
    constexpr uint32_t idO = kFp8 ? idesc_e4m3(128, D, false, true) : idesc_bf16(128, D, false, true);
    // a K step is 32 bytes of a row: 16 bf16 or 32 e4m3 elements
    constexpr int kKSteps = D * L::kElem / 32;       // steps of S = Q K^T
    constexpr int kPVSteps = 128 * L::kElem / 32;    // steps of O += P V (128 keys)
    // descriptors built once; each MMA adds (byte offset >> 4) to the start field
    const uint64_t dQ0 = sdesc_sw128(sbase + L::kQ0, 16, 1024), dQ1 = sdesc_sw128(sbase + L::kQ1, 16, 1024);
    const uint64_t dK0 = sdesc_sw128(sbase + L::kK0, 16, 1024);
    const uint64_t dV0 = sdesc_sw128(sbase + L::kV0, 16384, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    int cnt[2] = {0, 0};
    auto active = [&](int s, int t) { return has[s] && lo[s] <= t && t <= hi[s]; };
    auto issue_S = [&](int s, int st) {
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        if constexpr (kFp8)
          mma_ss_f8(tS(s), (s ? dQ1 : dQ0) + (off >> 4), dK0 + ((st * L::kTile + off) >> 4), idS, kk > 0, leader);
        else
          mma_ss(tS(s), (s ? dQ1 : dQ0) + (off >> 4), dK0 + ((st * L::kTile + off) >> 4), idS, kk > 0, leader);
      }
      mma_commit(&s_full[s], leader);
    };
    // Ping-pong: S_s of key tile t+1 follows PV_s of tile t at once, so each slot's
    // chain S -> softmax -> PV runs without waiting for the other slot's PV.
    bool ok = wait_all(q_full, 0) && wait_all(&k_full[0], 0);
    tc_fence_after();
    if (ok) {
      for (int s = 0; s < 2; ++s)
        if (active(s, t_lo)) issue_S(s, 0);
      mma_commit(&k_empty[0], leader);
    }
    int n = 0;
    const bool tracer = (lane == 0);
    (void)tracer;
    for (int t = t_lo; ok && t <= t_hi; ++t, ++n) {
      const int st = n & 1;
      const uint32_t ph = (n >> 1) & 1;
      const bool next = t + 1 <= t_hi;
      if (tracer) CSWA_MARK(0, n, 0);
      if (!(ok = wait_all(&v_full[st], ph))) break;
      if (next && !(ok = wait_all(&k_full[st ^ 1], ((n + 1) >> 1) & 1))) break;
      if (tracer) CSWA_MARK(0, n, 1);
      for (int s = 0; s < 2; ++s) {
        if (active(s, t)) {
          // PV_s chunk by chunk as the softmax warps publish P_s: chunk c holds keys
          // 32c .. 32c+31, as bf16 pairs in columns 16c .. 16c+15 (K steps 2c, 2c+1) or
          // as e4m3 quadruples in columns 8c .. 8c+7 (K step c); a K step reads 8 columns
          // of P and 32 bytes x its keys of V
          constexpr int kPer = kPVSteps / 4;
          for (int c = 0; c < 4; ++c) {
            if (!(ok = wait_all(&p_chunk[4 * s + c], cnt[s] & 1))) break;
            if (tracer && c == 0) CSWA_MARK(0, n, 2 + 3 * s);
            tc_fence_after();
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
              const int kk = kPer * c + u;
              const uint64_t bv = dV0 + ((st * L::kTile + kk * (32 / L::kElem) * 128) >> 4);
              if constexpr (kFp8)
                mma_ts_f8(tO(s), tS(s) + kk * 8, bv, idO, (cnt[s] > 0 || kk > 0), leader);
              else
                mma_ts(tO(s), tS(s) + kk * 8, bv, idO, (cnt[s] > 0 || kk > 0), leader);
            }
          }
          if (!ok) break;
          mma_commit(&pv_done[s], leader);
          ++cnt[s];
          if (tracer) CSWA_MARK(0, n, 3 + 3 * s);
        }
        tc_fence_after();
        if (next && active(s, t + 1)) issue_S(s, st ^ 1);
        if (tracer) CSWA_MARK(0, n, 4 + 3 * s);
      }
      if (!ok) break;
      mma_commit(&v_empty[st], leader);                 // V(t) read by both PVs
      if (next) mma_commit(&k_empty[st ^ 1], leader);  // K(t+1) read by both S
    }
    // every MMA issued above has finished before TMEM is released
    mma_commit(final_bar, leader);
    mbar_drain(final_bar, 0);
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ cache append (prefill)
    // Warps 2 and 3 of the group's first query head copy the chunk rows of the CTA's
    // own query tiles into the caches (each (b, KV head, row) exactly once), 8 vectors
    // of k and 8 of v in flight per lane. Nothing in this launch reads those cache
    // rows: the key tiles at or past pos[b] come from k_new / v_new.
    if constexpr (kCache) {
      if (p.kn && h % p.G == 0) {
        constexpr int V = D / 8;  // 16-byte vectors per row
        constexpr int kBatch = 8;
        const int tid = (warp - 2) * 32 + lane;
        const size_t rs = (size_t)p.Hkv * V;  // row stride in vectors
#pragma unroll 1
        for (int s2 = 0; s2 < 2; ++s2) {
          if (!has[s2]) continue;
          const int r0 = qt[s2] * 128, n = min(128, p.T - r0) * V;
          const uint4* ks = p.kn + ((size_t)((size_t)b * p.T + r0) * p.Hkv + hk) * V;
          const uint4* vs = p.vn + ((size_t)((size_t)b * p.T + r0) * p.Hkv + hk) * V;
          uint4* kd = p.kc + ((size_t)((size_t)b * p.Tmax + P + r0) * p.Hkv + hk) * V;
          uint4* vd = p.vc + ((size_t)((size_t)b * p.Tmax + P + r0) * p.Hkv + hk) * V;
#pragma unroll 1
          for (int e0b = 0; e0b < n; e0b += 64 * kBatch) {
            uint4 kr[kBatch], vr[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int e = e0b + u * 64 + tid;
              if (e < n) {
                const size_t off = (size_t)(e / V) * rs + (e % V);
                kr[u] = ks[off];
                vr[u] = vs[off];
              }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int e = e0b + u * 64 + tid;
              if (e < n) {
                const size_t off = (size_t)(e / V) * rs + (e % V);
                kd[off] = kr[u];
                vd[off] = vr[u];
              }
            }
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int s = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int my_qt = hp ? pair : 2 * pair + s;
    const int my_h = head_of(s);
    const int my_hi = my_qt;
    const int my_lo = lo_of(my_qt);
    const uint32_t tSs = tS(s) + lane_off, tOs = tO(s) + lane_off;
    if (my_qt < p.nq_tiles) {
      const int q0 = e0 + my_qt * 128;  // position of the tile's first row
      const int i = q0 + row;
      // fp8: the scores carry the quantization scales of q and k
      const float sl2 = kFp8 ? p.scale_log2 * (p.descale[0] * p.descale[1]) : p.scale_log2;
      // fp8: P is scaled by 2^8 before its e4m3 rounding (the exponent gets + 8) and must
      // stay below 448, so the running max moves whenever it grows
      constexpr float kThreshold = kFp8 ? 0.f : kRescaleThreshold;
      constexpr float kPBias = kFp8 ? 8.f : 0.f;
      float m_run = -INFINITY, l_run = 0.f;
      int cnt = 0;
      bool ok = true;
      const bool tracer = (quarter == 0 && lane == 0);
      (void)tracer;
      for (int t = my_lo; t <= my_hi; ++t, ++cnt) {
        if (tracer) CSWA_MARK(1 + s, cnt, 0);
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[s], cnt & 1, abort_flag));
        if (tracer) CSWA_MARK(1 + s, cnt, 1);
        if (!ok) break;
        tc_fence_after();
        uint32_t r[128];
        tmem_ld32(tSs + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(tSs + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld32(tSs + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
        tmem_ld32(tSs + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
        tmem_ld_wait();
        const int k0 = e0 + t * 128;
        const bool full = (k0 + 127 <= q0) && (W < 0 || q0 + 127 - k0 <= W) && (!kCache || k0 >= 0);
        // 4 independent 3-input max chains instead of one 128-long dependent chain
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (!full) {
          // visible columns of this row: [c_lo, c_hi] (empty when c_lo > c_hi)
          const int c_hi = i - k0;
          int c_lo = (W < 0) ? -1 : i - W - k0;
          if constexpr (kCache) c_lo = max(c_lo, -k0);  // no key before position 0
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool vis = (c <= c_hi) & (c >= c_lo);
            r[c] = vis ? r[c] : __float_as_uint(-INFINITY);
          }
        }
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], __uint_as_float(r[c + 4]), __uint_as_float(r[c + 5]));
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], __uint_as_float(r[c + 6]), __uint_as_float(r[c + 7]));
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        if (tracer) CSWA_MARK(1 + s, cnt, 2);
        const float m_tile = mx * sl2;
        bool rescale = false;
        float factor = 1.f;
        if (cnt == 0) {
          m_run = m_tile;
        } else if (m_tile > m_run + kThreshold) {
          factor = ex2_approx(m_run - m_tile);
          m_run = m_tile;
          l_run *= factor;
          rescale = true;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        // rescale O first, only when some row of the warp needs it (O is stable: this
        // tile's S was committed after the previous PV, so that PV has completed), so that
        // every P chunk published below may start its PV at once
        if (__any_sync(0xffffffffu, rescale)) {
          // 16 columns at a time: the row's 128 scores are still live in registers
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tOs + c * 16, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st16(tOs + c * 16, o);
          }
          tmem_st_wait();
        }
        // p = exp2(s * scale * log2e - m), two columns per packed FMA; row sum in packed adds.
        // Published in four chunks of 32 keys, each on its own barrier: chunk c's bf16 pairs
        // land in columns 16c .. 16c+15, whose fp32 S (keys < 32c + 32) is already in registers
        const float2 sl2v = make_float2(sl2, sl2), nm = make_float2(kPBias - m_use, kPBias - m_use);
        float2 ls4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if constexpr (kFp8) {
            // e4m3 quadruples of keys 32ch .. 32ch+31 into columns 8ch .. 8ch+7, whose fp32
            // S (keys < 8ch + 8) is already in registers
#pragma unroll
            for (int c = 8 * ch; c < 8 * ch + 8; ++c) {
              const float2 x0 =
                  __ffma2_rn(make_float2(__uint_as_float(r[4 * c]), __uint_as_float(r[4 * c + 1])), sl2v, nm);
              const float2 x1 =
                  __ffma2_rn(make_float2(__uint_as_float(r[4 * c + 2]), __uint_as_float(r[4 * c + 3])), sl2v, nm);
              const float2 p0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
              const float2 p1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
              ls4[c & 3] = __fadd2_rn(ls4[c & 3], __fadd2_rn(p0, p1));
              r[c] = pack_e4m3x4(p0.x, p0.y, p1.x, p1.y);
            }
            tmem_st8(tSs + 8 * ch, *reinterpret_cast<uint32_t(*)[8]>(&r[8 * ch]));
          } else {
#pragma unroll
            for (int c = 16 * ch; c < 16 * ch + 16; ++c) {
              const float2 x =
                  __ffma2_rn(make_float2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), sl2v, nm);
              const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              ls4[c & 3] = __fadd2_rn(ls4[c & 3], pp);
              r[c] = pack_bf16x2(pp.x, pp.y);
            }
            tmem_st16(tSs + 16 * ch, *reinterpret_cast<uint32_t(*)[16]>(&r[16 * ch]));
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_chunk[4 * s + ch]);
        }
        l_run += ((ls4[0].x + ls4[0].y) + (ls4[1].x + ls4[1].y)) + ((ls4[2].x + ls4[2].y) + (ls4[3].x + ls4[3].y));
        if (tracer) CSWA_MARK(1 + s, cnt, 4);
      }
      // ---------------------------------------------------------- epilogue
      if (ok && cnt > 0) ok = mbar_wait(&pv_done[s], (cnt - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok && kTmaO) {
        // O / l as bf16 rows of the slot's Q tile (every S of the slot has read it), in
        // the TMA layout; the warp stores its 32 rows (rows past T are not written)
        const int cr = my_qt * 128 + row;
        const float inv_l = 1.f / l_run;
        uint8_t* stg = smem + (s ? L::kQ1 : L::kQ0);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t t0[16], t1[16];
          tmem_ld16(tOs + c0, t0);
          tmem_ld16(tOs + c0 + 16, t1);
          tmem_ld_wait();
          float v0[16], v1[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) v0[u] = __uint_as_float(t0[u]) * inv_l, v1[u] = __uint_as_float(t1[u]) * inv_l;
          tile_st16(stg, row, c0, v0);
          tile_st16(stg, row, c0 + 16, v1);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int pn = 0; pn < D / 64; ++pn)
            tma_store_4d(&tm_o, stg + pn * 16384 + quarter * 4096, pn * 64, my_h, my_qt * 128 + 32 * quarter, b);
          bulk_commit();
        }
        if (cr < p.T) p.lse[((size_t)b * p.Hq + my_h) * p.T + cr] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      } else if (ok) {
        // tcgen05.ld is warp-collective: every lane loads, only rows of [0, T) store
        const int cr = my_qt * 128 - shift + row;  // output row (chunk row in kCache)
        const bool store = (cr < p.T) && (!kCache || cr >= 0);
        // fp8: O and l both carry P's 2^8, and O the quantization scale of v
        const float inv_l = (kFp8 ? p.descale[2] : 1.f) / l_run;
        __nv_bfloat16* dst = p.o + ((size_t)((size_t)b * p.T + cr) * p.Hq + my_h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tOs + c * 32, o);
          tmem_ld_wait();
          uint4 v[4];
          uint32_t* pv = reinterpret_cast<uint32_t*>(v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
          if (store) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = v[e];
          }
        }
        if (store && (!kCache || p.lse))
          p.lse[((size_t)b * p.Hq + my_h) * p.T + cr] = (m_run + __log2f(l_run) - kPBias) * 0.69314718055994531f;
      }
    }
  }

  // the o stores have completed before the CTA's shared memory goes
  if (kTmaO && warp >= 4 && lane == 0) bulk_wait0();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace cswa
