// attn_rope_qknorm (+ its backward): the fused QK RMS-norm + rotary prologue.
//
// For every (b, t, h) row x of q and of k (nanochat Admin & Developer Guide,
// 3 "The GPT Model (Internals)": RMS-normalised queries and keys with no
// learnable weight, rotary position embedding):
//   r = sqrt(mean(x^2) + eps),  xh = x / r,
//   y_j = xh_j cos(phi_j) - xh_{j+D/2} sin(phi_j),
//   y_{j+D/2} = xh_j sin(phi_j) + xh_{j+D/2} cos(phi_j),  phi_j = p * base^(-2j/D)
// with p = t + pos[b] (pos may be null). Backward, with g = rotation of dy by -phi:
//   dx = (g - xh (g . xh) / D) / r.
//
// HBM-bound elementwise work: D / (2 kRopeVec) lanes own one row, each holding both
// members of its rotation pairs (one load of kRopeVec values from each half per
// operand). The angles are computed once per position and shared by all its head rows.
#pragma once
#include "ptx.cuh"

namespace cswa {

struct RopeParams {
  const __nv_bfloat16* x[2];   // q rows, k rows (either may be null)
  const __nv_bfloat16* dy[2];  // backward only
  __nv_bfloat16* y[2];
  const int* pos;
  long long rows[2];  // B*T*Hq, B*T*Hkv (0 when the operand is absent)
  int T, H[2];
  float eps;
  // turns of pair j per unit position, as a 64-bit fixed-point fraction:
  // U_j = (base^(-2j/D) / (2 pi)) * 2^64, computed on the host in double precision
  unsigned long long turns[64];
};

// Each block owns kPosPerBlock consecutive (b, t) positions and every q and k
// head row at them (the block's q rows, and its k rows, are each one contiguous
// range). The angle of pair j at position p, in turns, is p * U_j mod 2^64 (exact
// for any 32-bit position); its top 32 bits, read as signed, give the reduced angle
// in [-pi, pi). A block first issues the loads of its first rows, then builds one
// cos/sin table per position in shared memory while they are in flight, and streams
// the rows: D / (2 kRopeVec) lanes per row, lane l owning elements kRopeVec l ..
// kRopeVec (l + 1) - 1 of each half (so a rotation pair never leaves its lane), kBatch
// rows per thread in flight.
constexpr int kPosPerBlock = 4;
// elements of each half a lane owns: 8 (two 16-byte loads per row and operand; measured
// against 4 with 8-byte loads and 8 positions per block: 0.0374 against 0.0394 ms for d20 q and k)
constexpr int kRopeVec = 8;

// kE consecutive bf16 values (8 or 16 bytes) as floats
template <int kE>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* src, bool active, float (&f)[kE]) {
  uint32_t w[kE / 2];
  if constexpr (kE == 4) {
    const uint2 v = active ? *reinterpret_cast<const uint2*>(src) : make_uint2(0, 0);
    w[0] = v.x, w[1] = v.y;
  } else {
    const uint4 v = active ? *reinterpret_cast<const uint4*>(src) : make_uint4(0, 0, 0, 0);
    w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
  }
#pragma unroll
  for (int u = 0; u < kE / 2; ++u) {
    f[2 * u] = __uint_as_float(w[u] << 16);
    f[2 * u + 1] = __uint_as_float(w[u] & 0xffff0000u);
  }
}
template <int kE>
__device__ __forceinline__ void store_bf16(__nv_bfloat16* dst, const float (&f)[kE]) {
  if constexpr (kE == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
}

template <int D, bool kBwd>
__global__ void __launch_bounds__(256, 4) rope_qknorm_kernel(const __grid_constant__ RopeParams p) {
  constexpr int kE = kRopeVec;
  constexpr int kLanesPerRow = D / (2 * kE);
  constexpr int kHalf = D / 2;
  constexpr int kRowsPerRound = 256 / kLanesPerRow;
  // rows per thread in flight: the forward keeps 4, the backward (twice the loads per
  // row, more live values) 2, so that 4 blocks fit per SM
  constexpr int kBatch = kBwd ? 2 : 4;
  __shared__ float4 cs4[kPosPerBlock][kHalf / 2];  // (cos_j, sin_j, cos_j+1, sin_j+1)

  const long long n_pos = p.rows[0] > 0 ? p.rows[0] / p.H[0] : p.rows[1] / p.H[1];  // B * T
  const long long pos0 = (long long)blockIdx.x * kPosPerBlock;
  const int Hq = p.rows[0] > 0 ? p.H[0] : 0;
  const int Hk = p.rows[1] > 0 ? p.H[1] : 0;
  const int n_pos_here = (int)min((long long)kPosPerBlock, n_pos - pos0);
  const int rows_q = n_pos_here * Hq, rows_k = n_pos_here * Hk;
  const int rows_all = rows_q + rows_k;
  const int lr = threadIdx.x % kLanesPerRow;
  const int row0 = threadIdx.x / kLanesPerRow;
  const int j0 = lr * kE;  // elements j0..j0+kE-1 and kHalf + j0..
  const float inv_hq = Hq ? 1.f / (float)Hq : 0.f, inv_hk = Hk ? 1.f / (float)Hk : 0.f;
  // every thread runs the same number of rounds so the row shuffles stay warp-uniform
  const int rounds = (kPosPerBlock * (Hq + Hk) + kRowsPerRound - 1) / kRowsPerRound;

  // block-local row -> (operand, element offset, position in block)
  auto locate = [&](int row, int& seg, size_t& off, int& pi) {
    seg = row >= rows_q;
    const int rr = seg ? row - rows_q : row;
    const int H = seg ? Hk : Hq;
    // rr < 2^20, so the float quotient truncates to the exact integer one
    pi = __float2int_rz(((float)rr + 0.5f) * (seg ? inv_hk : inv_hq));
    off = ((size_t)pos0 * H + rr) * D + j0;
  };

  for (int rd0 = 0; rd0 < rounds; rd0 += kBatch) {
    float xa[kBatch][kE], xb[kBatch][kE], ga[kBatch][kE], gb[kBatch][kE];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int row = (rd0 + u) * kRowsPerRound + row0;
      int seg, pi;
      size_t off;
      locate(row, seg, off, pi);
      const bool active = row < rows_all;
      load_bf16<kE>(p.x[seg] + off, active, xa[u]);
      load_bf16<kE>(p.x[seg] + off + kHalf, active, xb[u]);
      if (kBwd) {
        load_bf16<kE>(p.dy[seg] + off, active, ga[u]);
        load_bf16<kE>(p.dy[seg] + off + kHalf, active, gb[u]);
      }
    }
    if (rd0 == 0) {
      // the cos/sin table, built while the first loads are in flight
      for (int e = threadIdx.x; e < kPosPerBlock * kHalf; e += blockDim.x) {
        const int pi = e / kHalf, j = e % kHalf;
        const long long bt = pos0 + pi;
        float c = 1.f, sn = 0.f;
        if (bt < n_pos) {
          const int t = (int)(bt % p.T), b = (int)(bt / p.T);
          rope_cos_sin((unsigned)(t + (p.pos ? p.pos[b] : 0)), p.turns[j], c, sn);
        }
        reinterpret_cast<float2*>(&cs4[pi][0])[j] = make_float2(c, sn);
      }
      __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (rd0 + u >= rounds) break;  // uniform across the block
      const int row = (rd0 + u) * kRowsPerRound + row0;
      int seg, pi;
      size_t off;
      locate(row, seg, off, pi);
      const bool active = row < rows_all;
      if (!active) pi = 0;
      // a[i] = element j0 + i, bq[i] = element kHalf + j0 + i
      const float* a = xa[u];
      const float* bq = xb[u];
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < kE; ++v) ss = fmaf(a[v], a[v], fmaf(bq[v], bq[v], ss));
#pragma unroll
      for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv_r = rsqrtf(ss * (1.f / D) + p.eps);
      float c[kE], s[kE];
#pragma unroll
      for (int v = 0; v < kE / 2; ++v) {
        const float4 t = cs4[pi][j0 / 2 + v];
        c[2 * v] = t.x, s[2 * v] = t.y, c[2 * v + 1] = t.z, s[2 * v + 1] = t.w;
      }
      float oa[kE], ob[kE];
      if (!kBwd) {
#pragma unroll
        for (int v = 0; v < kE; ++v) {
          const float xa_ = a[v] * inv_r, xb_ = bq[v] * inv_r;
          oa[v] = fmaf(-xb_, s[v], xa_ * c[v]);
          ob[v] = fmaf(xa_, s[v], xb_ * c[v]);
        }
      } else {
        // g = rotation of dy by -phi
        const float* ga_ = ga[u];
        const float* gb_ = gb[u];
        float gra[kE], grb[kE], dot = 0.f;
#pragma unroll
        for (int v = 0; v < kE; ++v) {
          gra[v] = fmaf(gb_[v], s[v], ga_[v] * c[v]);
          grb[v] = fmaf(-ga_[v], s[v], gb_[v] * c[v]);
          dot = fmaf(gra[v], a[v] * inv_r, fmaf(grb[v], bq[v] * inv_r, dot));
        }
#pragma unroll
        for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float proj = dot * (1.f / D);
#pragma unroll
        for (int v = 0; v < kE; ++v) {
          oa[v] = (gra[v] - a[v] * inv_r * proj) * inv_r;
          ob[v] = (grb[v] - bq[v] * inv_r * proj) * inv_r;
        }
      }
      if (active) {
        store_bf16<kE>(p.y[seg] + off, oa);
        store_bf16<kE>(p.y[seg] + off + kHalf, ob);
      }
    }
  }
}

}  // namespace cswa
