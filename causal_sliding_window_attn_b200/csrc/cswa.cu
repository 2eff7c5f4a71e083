// C ABI of the causal sliding-window GQA attention library (see cswa_attn.h):
// argument checks, TMA tensor-map encoding and kernel launches. Nothing here
// allocates device memory; every launch is asynchronous on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "cswa_attn.h"
#include "bwd.cuh"
#include "decode.cuh"
#include "fwd.cuh"
#include "prologue.cuh"
#include "quant.cuh"
#include "replicate.cuh"

using namespace cswa;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// BTHD tensor as a 4-D tensor map (D, H, T, B); box = one rows-high, 128-byte-wide
// panel (64 bf16 or 128 one-byte elements) x 1 x rows x 1, 128-byte swizzle, zero fill
// past T. elem = 2 (bf16) or 1 (e4m3 codes).
bool encode_bthd(CUtensorMap* m, const void* base, int B, int T, int H, int D, int rows = 128, int elem = 2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * elem, (cuuint64_t)H * D * elem, (cuuint64_t)T * H * D * elem};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / elem), 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SMs of the current device (looked up once per device)
int sm_count() {
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    counts[dev] = (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) ? n : 148;
  }
  return counts[dev];
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dims_ok(int B, int T, int Hq, int Hkv) {
  return B >= 1 && T >= 1 && Hq >= 1 && Hkv >= 1 && Hq % Hkv == 0 && (long long)B * T * Hq < (1ll << 40);
}
inline bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline attn_status_t launched() { return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH; }

constexpr float kLog2e = 1.4426950408889634f;
inline int tiles128(int T) { return (T + 127) / 128; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kMaxDevices = 64;

// cudaFuncSetAttribute acts on the current device only, so the dynamic shared-memory
// limits are raised once per (device, head dim): a process that drives several GPUs
// sets them on each before its first launch there.
template <int D>
bool set_smem_attrs() {
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (done[dev].load(std::memory_order_acquire)) return true;
  bool r = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                FwdLayout<D>::kBytes) == cudaSuccess;
  r = r && cudaFuncSetAttribute(attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BwdLayout<D>::kBytes) == cudaSuccess;
  r = r && cudaFuncSetAttribute(attn_fwd_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                FwdLayout<D>::kBytes) == cudaSuccess;
  r = r && cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                DqLayout<D>::kBytes) == cudaSuccess;
  if constexpr (D == 128)
    r = r && cudaFuncSetAttribute(attn_fwd_kernel<D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  FwdLayout<D, true>::kBytes) == cudaSuccess;
  if (r) done[dev].store(true, std::memory_order_release);
  return r;
}

// Rotary angle of pair j per unit position, omega_j / (2 pi) = base^(-2j/D) / (2 pi)
// turns, as a 64-bit fixed-point fraction: position p's angle in turns is p * U_j
// mod 2^64, exact for any 32-bit position.
void rope_turns(int D, float base, unsigned long long* turns) {
  for (int j = 0; j < D / 2; ++j) {
    const double u = std::exp2(-2.0 * (double)j / (double)D * std::log2((double)base)) *
                     0.15915494309189533576888376337251;  // turns per unit position
    turns[j] = (unsigned long long)(u * 18446744073709551616.0);
  }
}

template <int D, bool kBwd>
attn_status_t launch_rope(const RopeParams& p, long long n_pos, cudaStream_t st) {
  const long long blocks = (n_pos + kPosPerBlock - 1) / kPosPerBlock;
  if (blocks > 0x7fffffffll) return ATTN_ERR_INVALID_ARG;
  rope_qknorm_kernel<D, kBwd><<<(unsigned)blocks, 256, 0, st>>>(p);
  return launched();
}

attn_status_t rope_common(const void* x0, const void* x1, const void* dy0, const void* dy1, void* y0, void* y1,
                          const int32_t* pos, int B, int T, int Hq, int Hkv, int D, float base, float eps,
                          void* stream, bool bwd) {
  // the prologue treats q and k rows alike: no Hq/Hkv relation is needed here. A block's
  // row index reaches kPosPerBlock * H, which the kernel divides in float: H <= 65535
  // keeps it exact
  if (B < 1 || T < 1 || (x0 && (Hq < 1 || Hq > 65535)) || (x1 && (Hkv < 1 || Hkv > 65535)) ||
      (long long)B * T * (Hq + Hkv) >= (1ll << 40) ||
      !(base > 1.f) || !std::isfinite(base) || !(eps >= 0.f) || !std::isfinite(eps))
    return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!x0 && !x1) return ATTN_ERR_INVALID_ARG;
  if ((x0 && (!y0 || !aligned16(x0) || !aligned16(y0) || (bwd && (!dy0 || !aligned16(dy0))))) ||
      (x1 && (!y1 || !aligned16(x1) || !aligned16(y1) || (bwd && (!dy1 || !aligned16(dy1))))))
    return ATTN_ERR_INVALID_ARG;
  RopeParams p{};
  p.x[0] = static_cast<const __nv_bfloat16*>(x0);
  p.x[1] = static_cast<const __nv_bfloat16*>(x1);
  p.dy[0] = static_cast<const __nv_bfloat16*>(dy0);
  p.dy[1] = static_cast<const __nv_bfloat16*>(dy1);
  p.y[0] = static_cast<__nv_bfloat16*>(y0);
  p.y[1] = static_cast<__nv_bfloat16*>(y1);
  p.pos = pos;
  p.rows[0] = x0 ? (long long)B * T * Hq : 0;
  p.rows[1] = x1 ? (long long)B * T * Hkv : 0;
  p.T = T;
  p.H[0] = Hq;
  p.H[1] = Hkv;
  p.eps = eps;
  rope_turns(D, base, p.turns);
  cudaStream_t st = as_stream(stream);
  const long long n_pos = (long long)B * T;
  if (D == 64) return bwd ? launch_rope<64, true>(p, n_pos, st) : launch_rope<64, false>(p, n_pos, st);
  return bwd ? launch_rope<128, true>(p, n_pos, st) : launch_rope<128, false>(p, n_pos, st);
}

template <int D>
attn_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T, int Hq,
                         int Hkv, int window, float scale, cudaStream_t st) {
  CUtensorMap tq, tk, tv, to;
  if (!encode_bthd(&tq, q, B, T, Hq, D) || !encode_bthd(&tk, k, B, T, Hkv, D) || !encode_bthd(&tv, v, B, T, Hkv, D) ||
      !encode_bthd(&to, o, B, T, Hq, D, 32))
    return ATTN_ERR_LAUNCH;
  if (!set_smem_attrs<D>()) return ATTN_ERR_LAUNCH;
  FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.T = T;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.window = (window >= T) ? -1 : window;
  p.scale_log2 = scale * kLog2e;
  p.nq_tiles = tiles128(T);
  // G even: the slots are two query heads of one KV group at one query tile
  p.head_pairs = (p.G % 2 == 0) ? 1 : 0;
  p.n_pairs = p.head_pairs ? p.nq_tiles : (p.nq_tiles + 1) / 2;
  dim3 grid(p.head_pairs ? Hq / 2 : Hq, B, p.n_pairs);
  // the two chunk maps are unused in training: q's map stands in for them
  attn_fwd_kernel<D><<<grid, 384, FwdLayout<D>::kBytes, st>>>(tq, tk, tv, tq, tq, to, p);
  return launched();
}

// The fp8 forward: e4m3 codes of q, k, v (one byte per element, BTHD) and their three
// dequantization factors in device memory; D = 128.
attn_status_t launch_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* descale, void* o, float* lse,
                             int B, int T, int Hq, int Hkv, int window, float scale, cudaStream_t st) {
  constexpr int D = 128;
  CUtensorMap tq, tk, tv;
  if (!encode_bthd(&tq, q8, B, T, Hq, D, 128, 1) || !encode_bthd(&tk, k8, B, T, Hkv, D, 128, 1) ||
      !encode_bthd(&tv, v8, B, T, Hkv, D, 128, 1))
    return ATTN_ERR_LAUNCH;
  if (!set_smem_attrs<D>()) return ATTN_ERR_LAUNCH;
  FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.T = T;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.window = (window >= T) ? -1 : window;
  p.scale_log2 = scale * kLog2e;
  p.nq_tiles = tiles128(T);
  p.n_pairs = (p.nq_tiles + 1) / 2;
  p.descale = descale;
  dim3 grid(Hq, B, p.n_pairs);
  attn_fwd_kernel<D, false, true><<<grid, 384, FwdLayout<D, true>::kBytes, st>>>(tq, tk, tv, tq, tq, tq, p);
  return launched();
}

// Chunked prefill: the forward kernel in cache mode. q (B,T,Hq,D) is the chunk. With
// k_new / v_new (B,T,Hkv,D) the chunk's keys are read from them and copied into the
// caches (B,Tmax,Hkv,D) by the same launch; without, the caches already hold them at
// rows pos[b] .. pos[b]+T-1.
template <int D>
attn_status_t launch_prefill(const void* q, void* kc, void* vc, const void* kn, const void* vn, const int32_t* pos,
                             void* o, float* lse, int B, int T, int Tmax, int Hq, int Hkv, int window, float scale,
                             cudaStream_t st) {
  CUtensorMap tq, tk, tv, tkn, tvn;
  if (!encode_bthd(&tq, q, B, T, Hq, D) || !encode_bthd(&tk, kc, B, Tmax, Hkv, D) ||
      !encode_bthd(&tv, vc, B, Tmax, Hkv, D))
    return ATTN_ERR_LAUNCH;
  if (kn) {
    if (!encode_bthd(&tkn, kn, B, T, Hkv, D) || !encode_bthd(&tvn, vn, B, T, Hkv, D)) return ATTN_ERR_LAUNCH;
  } else {
    tkn = tq;  // unused
    tvn = tq;
  }
  if (!set_smem_attrs<D>()) return ATTN_ERR_LAUNCH;
  FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.T = T;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.window = (window >= Tmax) ? -1 : window;  // no position reaches Tmax
  p.scale_log2 = scale * kLog2e;
  p.nq_tiles = tiles128(T);
  p.n_pairs = (p.nq_tiles + 1) / 2;
  p.pos = pos;
  p.Tmax = Tmax;
  p.shift = kn ? 0 : 128 * p.nq_tiles - T;
  p.B = B;
  p.Hkv = Hkv;
  p.kn = static_cast<const uint4*>(kn);
  p.vn = static_cast<const uint4*>(vn);
  p.kc = static_cast<uint4*>(kc);
  p.vc = static_cast<uint4*>(vc);
  dim3 grid(Hq, B, p.n_pairs);
  attn_fwd_kernel<D, true><<<grid, 384, FwdLayout<D>::kBytes, st>>>(tq, tk, tv, tkn, tvn, tq, p);
  return launched();
}

// attn_bwd's (and attn_block_bwd's) workspace: the row extensions of the S^T and dP^T
// MMAs (-lse/scale and -Delta per query row, padded to 128-row tiles), the bf16 dS^T
// tiles of every (key tile, query tile) pair inside the window, and the two work counters.
struct BwdWorkspace {
  uint8_t* ext_lse;       // (B, Hq, Tpad / 128) x 512 bytes
  uint8_t* ext_delta;     // (B, Hq, Tpad / 128) x 512 bytes
  __nv_bfloat16* ds;      // stored dS^T tiles, 128 x 128 each
  int* counter;           // [2] work-item counters of the main and dQ kernels (zeroed by the prep kernel)
  long long tiles_per_bh;
  int span;
};
int eff_window(int window, int T) { return (window >= T) ? -1 : window; }
// Layout: the two row-extension arrays, the counters, then the dS^T tiles of as many
// (batch, KV head) blocks as one pass covers (kv_blocks; all B * Hkv of them when the
// caller's workspace allows a single pass).
size_t bwd_ws_parts(int B, int T, int Hq, int Hkv, int window, long long kv_blocks, BwdWorkspace* w, void* base) {
  const int nt = tiles128(T);
  const size_t Tpad = (size_t)nt * 128;
  const int span = bwd_span(nt, eff_window(window, T));
  const long long tiles = ds_tiles_before(nt, nt, span);
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* at = p ? p + off : nullptr;
    off += align256(bytes);
    return at;
  };
  uint8_t* e1 = take((size_t)B * Hq * Tpad * 4);
  uint8_t* e2 = take((size_t)B * Hq * Tpad * 4);
  uint8_t* cnt = take(256);
  uint8_t* ds = take((size_t)kv_blocks * (Hq / Hkv) * tiles * 32768);
  if (w) {
    w->ext_lse = e1;
    w->ext_delta = e2;
    w->ds = reinterpret_cast<__nv_bfloat16*>(ds);
    w->counter = reinterpret_cast<int*>(cnt);
    w->tiles_per_bh = tiles;
    w->span = span;
  }
  return off;
}
// (batch, KV head) blocks per pass that a workspace of ws_bytes holds, at most all of them
// and at most what keeps a pass's stored tile rows below 2^31; 0 if not even one fits
long long bwd_blocks_per_pass(int B, int T, int Hq, int Hkv, int window, size_t ws_bytes) {
  const long long total = (long long)B * Hkv;
  const size_t fixed = bwd_ws_parts(B, T, Hq, Hkv, window, 0, nullptr, nullptr);
  const int nt = tiles128(T);
  const long long per_block = (long long)(Hq / Hkv) * ds_tiles_before(nt, nt, bwd_span(nt, eff_window(window, T)));
  if (ws_bytes < fixed) return 0;
  long long n = std::min<long long>(total, (long long)((ws_bytes - fixed) / ((size_t)per_block * 32768)));
  n = std::min<long long>(n, ((1ll << 31) - 1) / (per_block * 128));
  // a partial pass must still fit its rounding to 256 bytes
  while (n > 0 && bwd_ws_parts(B, T, Hq, Hkv, window, n, nullptr, nullptr) > ws_bytes) --n;
  return n;
}

// The fused prologue backward of the block variant: raw q and k, and the rotary
// base and eps of the forward prologue (positions t). Null q_raw: plain attn_bwd.
struct RopeBwd {
  const void* q_raw;
  const void* k_raw;
  float base, eps;
};

template <int D>
attn_status_t launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B, int T,
                         int Hq, int Hkv, int window, float scale, const RopeBwd& rb, cudaStream_t st) {
  const int nt = tiles128(T);
  const int Tpad = nt * 128;
  const bool rope = rb.q_raw != nullptr;
  const long long total_blocks = (long long)B * Hkv;
  const long long nblk = bwd_blocks_per_pass(B, T, Hq, Hkv, window, ws_bytes);
  if (nblk <= 0) return ATTN_ERR_INVALID_ARG;
  BwdWorkspace w;
  bwd_ws_parts(B, T, Hq, Hkv, window, nblk, &w, ws);
  // operands (128-row boxes), the outputs (32-row boxes: one per epilogue warp), and
  // for the block backward the raw k (128 rows, one load per tile) and q (32 rows)
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq, tkr, tqr;
  if (!encode_bthd(&tq, q, B, T, Hq, D) || !encode_bthd(&tk, k, B, T, Hkv, D) ||
      !encode_bthd(&tv, v, B, T, Hkv, D) || !encode_bthd(&tdo, dO, B, T, Hq, D) ||
      !encode_bthd(&tdk, dk, B, T, Hkv, D, 32) || !encode_bthd(&tdv, dv, B, T, Hkv, D, 32) ||
      !encode_bthd(&tdq, dq, B, T, Hq, D, 32))
    return ATTN_ERR_LAUNCH;
  if (rope) {
    if (!encode_bthd(&tkr, rb.k_raw, B, T, Hkv, D) || !encode_bthd(&tqr, rb.q_raw, B, T, Hq, D, 32))
      return ATTN_ERR_LAUNCH;
  } else {
    tkr = tk;  // not read
    tqr = tdq;
  }
  if (!set_smem_attrs<D>()) return ATTN_ERR_LAUNCH;
  {
    PrepParams pp{};
    pp.o = static_cast<const __nv_bfloat16*>(o);
    pp.dout = static_cast<const __nv_bfloat16*>(dO);
    pp.lse = lse;
    pp.ext_lse = w.ext_lse;
    pp.ext_delta = w.ext_delta;
    pp.item_counter = w.counter;
    pp.B = B;
    pp.T = T;
    pp.Tpad = Tpad;
    pp.Hq = Hq;
    pp.inv_scale = 1.f / scale;
    // chunks of 2 * 256 / (D / 16) rows (D / 16 lanes per row, two rows per lane), taken
    // in turn by as many blocks as are resident at once
    const long long rows = (long long)Tpad * Hq, per_chunk = 2 * 256 / (D / 16);
    pp.chunks = (int)((rows + per_chunk - 1) / per_chunk);
    const long long n_chunks = (long long)B * pp.chunks;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_bwd_prep_kernel<D>, 256, 0) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    const unsigned blocks = (unsigned)std::min<long long>(n_chunks, (long long)per_sm * sm_count());
    attn_bwd_prep_kernel<D><<<blocks, 256, 0, st>>>(pp);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  }
  BwdParams p{};
  p.ext_lse = w.ext_lse;
  p.ext_delta = w.ext_delta;
  p.ds = w.ds;
  p.item_counter = w.counter;
  p.T = T;
  p.Tpad = Tpad;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.window = eff_window(window, T);
  p.n_tiles = nt;
  p.span = w.span;
  p.tiles_per_bh = w.tiles_per_bh;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.rope = rope ? 1 : 0;
  p.eps = rb.eps;
  if (rope) rope_turns(D, rb.base, p.turns);
  // One pass (a main and a dQ launch) per nblk (batch, KV head) blocks; the prep kernel
  // zeroed the work counters for the first, a memset does it for the others.
  for (long long blk0 = 0; blk0 < total_blocks; blk0 += nblk) {
    const long long n = std::min(nblk, total_blocks - blk0);
    if (blk0 > 0 && cudaMemsetAsync(w.counter, 0, 2 * sizeof(int), st) != cudaSuccess) return ATTN_ERR_LAUNCH;
    p.blk0 = (int)blk0;
    // persistent: one CTA per SM walks the pass's (key tile, KV head, batch) items
    const long long kv_items = (long long)nt * n;
    const int kv_grid = (int)std::min<long long>(kv_items, sm_count());
    attn_bwd_kernel<D><<<kv_grid, kBwdThreads, BwdLayout<D>::kBytes, st>>>(tq, tk, tv, tdo, tkr, tdk, tdv, p,
                                                                    (int)kv_items);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    const long long items = kv_items * p.G;
    const int grid = (int)std::min<long long>(items, sm_count());
    attn_bwd_dq_kernel<D><<<grid, 256, DqLayout<D>::kBytes, st>>>(tk, tqr, tdq, p, (int)items);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  }
  return launched();
}

template <int D, int GMAX>
attn_status_t launch_decode(const DecodeParams& p, int B, cudaStream_t st) {
  dim3 g1(p.n_chunks, p.Hkv, B);
  decode_chunk_kernel<D, GMAX><<<g1, 128, 0, st>>>(p);
  return launched();
}

int decode_chunks(int Tmax, int window) {
  const int span = (window < 0 || window >= Tmax) ? Tmax : window + 1;
  return (span + kDecodeChunk - 1) / kDecodeChunk;
}

// attn_decode's workspace: the fp32 split-K partials (B, Hq, chunks, D + 2), rounded up
// to 256 bytes, then one 8-byte arrival counter per (sequence, KV head) -- B * Hq of
// them, enough for any Hkv <= Hq.
size_t decode_ws_bytes(int B, int Hq, int D, int Tmax, int window) {
  return align256((size_t)B * Hq * decode_chunks(Tmax, window) * (D + 2) * 4) + (size_t)B * Hq * 8;
}

// Tag of one decode call for its arrival counters: a fresh value per call in this
// process (never 0, so zeroed memory never matches; a CUDA graph that captured a call
// replays its tag, which the counters' reset to (tag, 0) allows).
std::atomic<unsigned> g_decode_epoch{0};
unsigned next_decode_epoch() {
  unsigned e = g_decode_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
  if (e == 0) e = g_decode_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
  return e;
}

// ---------------------------------------------------------------- no-allocation decode
// Scratch for attn_decode_noalloc: the split-K partials live in this file-scope
// device array instead of a caller-provided workspace. Every GPU that loads the
// library holds it (kNoAllocScratchFloats * 4 bytes) until the process exits.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;  // 4 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// The device address of g_noalloc_scratch, looked up once per device with that
// device current (host code only sees a stand-in symbol, never the address).
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

attn_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return ATTN_ERR_LAUNCH;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return ATTN_OK;
}

attn_status_t bwd_common(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                         int T, int Hq, int Hkv, int D, int window, float scale, const RopeBwd& rb, void* stream) {
  if (!dims_ok(B, T, Hq, Hkv) || !scale_ok(scale)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
  const bool rope = rb.q_raw != nullptr;
  if (rope && (!rb.k_raw || !aligned16(rb.q_raw) || !aligned16(rb.k_raw) || !(rb.base > 1.f) ||
               !std::isfinite(rb.base) || !(rb.eps >= 0.f) || !std::isfinite(rb.eps)))
    return ATTN_ERR_INVALID_ARG;
  if (Hq > 65535 || B > 65535 || tiles128(T) > 65535) return ATTN_ERR_INVALID_ARG;
  // a pass's stored dS^T tile rows (one (batch, KV head) block at least), its work items
  // and the prep kernel's rows per batch (Tpad * Hq) are counted in 32 bits
  const int nt = tiles128(T);
  if ((long long)(Hq / Hkv) * ds_tiles_before(nt, nt, bwd_span(nt, eff_window(window, T))) * 128 >= (1ll << 31) ||
      (long long)nt * 128 * Hq >= (1ll << 31))
    return ATTN_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      bwd_blocks_per_pass(B, T, Hq, Hkv, window, ws_bytes) <= 0)
    return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D == 64 ? launch_bwd<64>(q, k, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, T, Hq, Hkv, window, scale,
                                  rb, st)
                 : launch_bwd<128>(q, k, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, T, Hq, Hkv, window, scale,
                                   rb, st);
}
}  // namespace

extern "C" {

attn_status_t attn_rope_qknorm(const void* q, const void* k, void* q_out, void* k_out, const int32_t* pos, int B,
                               int T, int Hq, int Hkv, int D, float rope_base, float eps, void* stream) {
  return rope_common(q, k, nullptr, nullptr, q_out, k_out, pos, B, T, Hq, Hkv, D, rope_base, eps, stream, false);
}

attn_status_t attn_rope_qknorm_bwd(const void* q, const void* k, const void* dq_hat, const void* dk_hat, void* dq,
                                   void* dk, const int32_t* pos, int B, int T, int Hq, int Hkv, int D,
                                   float rope_base, float eps, void* stream) {
  return rope_common(q, k, dq_hat, dk_hat, dq, dk, pos, B, T, Hq, Hkv, D, rope_base, eps, stream, true);
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T, int Hq,
                       int Hkv, int D, int window, float scale, void* stream) {
  if (!dims_ok(B, T, Hq, Hkv) || !scale_ok(scale)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(lse))
    return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D == 64 ? launch_fwd<64>(q, k, v, o, lse, B, T, Hq, Hkv, window, scale, st)
                 : launch_fwd<128>(q, k, v, o, lse, B, T, Hq, Hkv, window, scale, st);
}

size_t attn_bwd_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int window) {
  if (!dims_ok(B, T, Hq, Hkv) || (D != 64 && D != 128)) return 0;
  return bwd_ws_parts(B, T, Hq, Hkv, window, (long long)B * Hkv, nullptr, nullptr);
}

size_t attn_bwd_workspace_min_bytes(int B, int T, int Hq, int Hkv, int D, int window) {
  if (!dims_ok(B, T, Hq, Hkv) || (D != 64 && D != 128)) return 0;
  return bwd_ws_parts(B, T, Hq, Hkv, window, 1, nullptr, nullptr);
}

size_t attn_block_bwd_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int window) {
  return attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, window);
}


attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                       void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int T, int Hq, int Hkv,
                       int D, int window, float scale, void* stream) {
  const RopeBwd none{nullptr, nullptr, 0.f, 0.f};
  return bwd_common(q, k, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, T, Hq, Hkv, D, window, scale, none,
                    stream);
}

attn_status_t attn_block_bwd(const void* q, const void* k, const void* q_hat, const void* k_hat, const void* v,
                             const void* o, const void* dO, const float* lse, void* dq, void* dk, void* dv,
                             void* workspace, size_t ws_bytes, int B, int T, int Hq, int Hkv, int D, int window,
                             float scale, float rope_base, float eps, void* stream) {
  if (!q || !k) return ATTN_ERR_INVALID_ARG;
  const RopeBwd rb{q, k, rope_base, eps};
  return bwd_common(q_hat, k_hat, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, T, Hq, Hkv, D, window, scale, rb,
                    stream);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int D, int Tmax, int window) {
  if (B < 1 || Hq < 1 || Tmax < 1 || (D != 64 && D != 128)) return 0;
  return decode_ws_bytes(B, Hq, D, Tmax, window);
}

attn_status_t attn_decode(const void* q, void* kcache, void* vcache, const void* k_new, const void* v_new,
                          const int32_t* pos, void* o, float* lse, int B, int Tmax, int Hq, int Hkv, int D, int window,
                          float scale, void* workspace, size_t ws_bytes, void* stream) {
  if (!dims_ok(B, Tmax, Hq, Hkv) || !scale_ok(scale)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (!q || !kcache || !vcache || !pos || !o || !workspace || (k_new == nullptr) != (v_new == nullptr))
    return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, kcache, vcache, o, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
  if ((k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return ATTN_ERR_INVALID_ARG;
  if (ws_bytes < attn_decode_workspace_bytes(B, Hq, D, Tmax, window) || Hkv > 65535 || B > 65535 || Hq > 65535)
    return ATTN_ERR_INVALID_ARG;
  const size_t part_bytes = align256((size_t)B * Hq * decode_chunks(Tmax, window) * (D + 2) * 4);
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<__nv_bfloat16*>(kcache);
  p.vc = static_cast<__nv_bfloat16*>(vcache);
  p.kn = static_cast<const __nv_bfloat16*>(k_new);
  p.vn = static_cast<const __nv_bfloat16*>(v_new);
  p.pos = pos;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.ws = static_cast<float*>(workspace);
  p.counters = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + part_bytes);
  p.epoch = next_decode_epoch();
  p.Tmax = Tmax;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.window = window;
  p.n_chunks = decode_chunks(Tmax, window);
  if (p.n_chunks > kDecodeMaxChunks) return ATTN_ERR_UNSUPPORTED;  // more than 512k keys in view
  p.scale_log2 = scale * kLog2e;
  cudaStream_t st = as_stream(stream);
  const int gm = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8;
  if (D == 64) {
    switch (gm) {
      case 1: return launch_decode<64, 1>(p, B, st);
      case 2: return launch_decode<64, 2>(p, B, st);
      case 4: return launch_decode<64, 4>(p, B, st);
      default: return launch_decode<64, 8>(p, B, st);
    }
  }
  switch (gm) {
    case 1: return launch_decode<128, 1>(p, B, st);
    case 2: return launch_decode<128, 2>(p, B, st);
    case 4: return launch_decode<128, 4>(p, B, st);
    default: return launch_decode<128, 8>(p, B, st);
  }
}

// attn_decode without a workspace argument: the split-K partials go to the
// library's own device scratch (see cswa_attn.h for who needs this and the limits).
attn_status_t attn_decode_noalloc(const void* q, void* kcache, void* vcache, const void* k_new, const void* v_new,
                                  const int32_t* pos, void* o, float* lse, int B, int Tmax, int Hq, int Hkv, int D,
                                  int window, float scale, void* stream) {
  const size_t need = attn_decode_workspace_bytes(B, Hq, D, Tmax, window);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (need > kNoAllocScratchFloats * sizeof(float)) return ATTN_ERR_INVALID_ARG;  // beyond the fixed scratch
  void* scratch = nullptr;
  const attn_status_t st = noalloc_scratch(&scratch);
  if (st != ATTN_OK) return st;
  // every partial the merge reads is written earlier in the same call, and the arrival
  // counters are tagged per call (stale contents read as zero): nothing to clear
  return attn_decode(q, kcache, vcache, k_new, v_new, pos, o, lse, B, Tmax, Hq, Hkv, D, window, scale, scratch, need,
                     stream);
}

attn_status_t attn_prefill(const void* q, void* kcache, void* vcache, const void* k_new, const void* v_new,
                           const int32_t* pos, void* o, float* lse, int B, int T, int Tmax, int Hq, int Hkv, int D,
                           int window, float scale, void* stream) {
  if (!dims_ok(B, T, Hq, Hkv) || !dims_ok(B, Tmax, Hq, Hkv) || T > Tmax || !scale_ok(scale))
    return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!q || !kcache || !vcache || !pos || !o || (k_new == nullptr) != (v_new == nullptr)) return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, kcache, vcache, o};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
  if ((k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  return D == 64
             ? launch_prefill<64>(q, kcache, vcache, k_new, v_new, pos, o, lse, B, T, Tmax, Hq, Hkv, window, scale, st)
             : launch_prefill<128>(q, kcache, vcache, k_new, v_new, pos, o, lse, B, T, Tmax, Hq, Hkv, window, scale,
                                   st);
}

size_t attn_quantize_fp8_workspace_bytes(long long n) {
  if (n < 8 || n % 8) return 0;
  return (size_t)kQuantMaxBlocks * 4;
}

attn_status_t attn_quantize_fp8(const void* x, long long n, void* x8, float* descale, void* workspace,
                                size_t ws_bytes, void* stream) {
  if (n < 8 || n % 8 || !x || !x8 || !descale || !workspace || !aligned16(x) ||
      (reinterpret_cast<uintptr_t>(x8) & 7u) || (reinterpret_cast<uintptr_t>(descale) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 3u) || ws_bytes < attn_quantize_fp8_workspace_bytes(n))
    return ATTN_ERR_INVALID_ARG;
  const long long n8 = n / 8;
  const int blocks = (int)std::min<long long>((n8 + 255) / 256, kQuantMaxBlocks);
  cudaStream_t st = as_stream(stream);
  float* part = static_cast<float*>(workspace);
  quant_amax_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(x), n8, part);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  quant_e4m3_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(x), n8, part, blocks, static_cast<uint2*>(x8),
                                            descale);
  return launched();
}

attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* descale, void* o, float* lse,
                           int B, int T, int Hq, int Hkv, int D, int window, float scale, void* stream) {
  if (!dims_ok(B, T, Hq, Hkv) || !scale_ok(scale)) return ATTN_ERR_INVALID_ARG;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!q8 || !k8 || !v8 || !descale || !o || !lse || !aligned16(q8) || !aligned16(k8) || !aligned16(v8) ||
      !aligned16(o) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(descale) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  return launch_fwd_fp8(q8, k8, v8, descale, o, lse, B, T, Hq, Hkv, window, scale, as_stream(stream));
}

attn_status_t attn_kv_replicate(const void* k_src, const void* v_src, void* k_dst, void* v_dst, int n_layers,
                                int rows, int Tmax_src, int N, int Tmax, int Hkv, int D, void* stream) {
  if (!k_src || !v_src || !k_dst || !v_dst || n_layers < 1 || rows < 0 || Tmax_src < 1 || N < 1 || Tmax < 1 ||
      Hkv < 1 || D < 1 || rows > Tmax_src || rows > Tmax)
    return ATTN_ERR_INVALID_ARG;
  const size_t row_bytes = (size_t)Hkv * D * 2;
  const size_t src_layer = (size_t)Tmax_src * row_bytes;  // batch-1 source: layer stride
  const size_t dst_sample = (size_t)Tmax * row_bytes;     // destination: sample stride ...
  const size_t dst_layer = (size_t)N * dst_sample;        // ... and layer stride
  const size_t src_bytes = (size_t)n_layers * src_layer, dst_bytes = (size_t)n_layers * dst_layer;
  auto disjoint = [](const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x + na <= y || y + nb <= x;
  };
  if (!disjoint(k_dst, dst_bytes, v_dst, dst_bytes) || !disjoint(k_dst, dst_bytes, k_src, src_bytes) ||
      !disjoint(k_dst, dst_bytes, v_src, src_bytes) || !disjoint(v_dst, dst_bytes, k_src, src_bytes) ||
      !disjoint(v_dst, dst_bytes, v_src, src_bytes))
    return ATTN_ERR_INVALID_ARG;
  if (rows == 0) return ATTN_OK;
  // the widest vector every pointer and stride allows
  const uintptr_t align = reinterpret_cast<uintptr_t>(k_src) | reinterpret_cast<uintptr_t>(v_src) |
                          reinterpret_cast<uintptr_t>(k_dst) | reinterpret_cast<uintptr_t>(v_dst) | row_bytes;
  const int vec = (align % 16 == 0) ? 16 : (align % 4 == 0) ? 4 : 2;
  ReplicateParams p{};
  p.src[0] = static_cast<const uint8_t*>(k_src);
  p.src[1] = static_cast<const uint8_t*>(v_src);
  p.dst[0] = static_cast<uint8_t*>(k_dst);
  p.dst[1] = static_cast<uint8_t*>(v_dst);
  p.vec_per_layer = (long long)((size_t)rows * row_bytes / vec);
  p.src_layer = (long long)(src_layer / vec);
  p.dst_layer = (long long)(dst_layer / vec);
  p.dst_sample = (long long)(dst_sample / vec);
  p.total = 2 * (long long)n_layers * p.vec_per_layer;
  p.N = N;
  const long long blocks = std::min<long long>((p.total + 255) / 256, (long long)sm_count() * 8);
  cudaStream_t st = as_stream(stream);
  if (vec == 16)
    kv_replicate_kernel<uint4><<<(unsigned)blocks, 256, 0, st>>>(p);
  else if (vec == 4)
    kv_replicate_kernel<uint32_t><<<(unsigned)blocks, 256, 0, st>>>(p);
  else
    kv_replicate_kernel<uint16_t><<<(unsigned)blocks, 256, 0, st>>>(p);
  return launched();
}

attn_status_t attn_get_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (v && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (v & (kStatusTimeout | kStatusLayout)) return ATTN_ERR_TIMEOUT;
  if (v & kStatusBadPosition) return ATTN_ERR_DEVICE;
  return ATTN_OK;
}

attn_status_t attn_debug_set_wait_limit(unsigned long long ns, void* stream) {
  const unsigned long long v = ns ? ns : kWaitTimeoutNs;
  if (v > kWaitTimeoutNs) return ATTN_ERR_INVALID_ARG;
  // kernels already enqueued on `stream` keep the limit they started with
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  return cudaDeviceSynchronize() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

#ifdef CSWA_TRACE
// Profiling builds only: copies the pipeline trace marks (clock64 per CTA, role,
// step and tag; see CSWA_MARK) to host memory.
int attn_debug_trace_copy(void* dst, size_t bytes) {
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  return cudaMemcpyFromSymbol(dst, g_trace, bytes < sizeof(g_trace) ? bytes : sizeof(g_trace)) == cudaSuccess ? 0 : 3;
}
int attn_debug_trace_clear(void) {
  static unsigned long long zeros[1024] = {};
  for (size_t off = 0; off < sizeof(g_trace); off += sizeof(zeros))
    if (cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros), off) != cudaSuccess) return 3;
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : 3;
}
#endif

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported head dim or device";
    case ATTN_ERR_LAUNCH: return "CUDA launch or tensor-map encode failed";
    case ATTN_ERR_TIMEOUT: return "a device-side wait timed out";
    case ATTN_ERR_DEVICE: return "a device-side range check failed (decode or prefill position out of range)";
  }
  return "unknown status";
}

int attn_device_supported(void) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return 0;
  return (major == 10 && minor == 0) ? 1 : 0;
}

}  // extern "C"
