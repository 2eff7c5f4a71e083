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
// HBM-bound elementwise work: D/8 lanes own one row, each holding both members
// of its rotation pairs (two 8-byte loads per operand). The angles are computed
// once per position and shared by all its head rows.
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
// the rows: D/8 lanes per row, lane l owning elements 4l..4l+3 of each half (so a
// rotation pair never leaves its lane), kBatch rows per thread in flight.
constexpr int kPosPerBlock = 8;

template <int D, bool kBwd>
__global__ void __launch_bounds__(256, 4) rope_qknorm_kernel(const __grid_constant__ RopeParams p) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kHalf = D / 2;
  constexpr int kRowsPerRound = 256 / kLanesPerRow;
  // rows per thread in flight: 4 (8 loads of 8 bytes); the backward, with twice the
  // loads per row and more live values, keeps 2 so that 4 blocks fit per SM
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
  const int j0 = lr * 4;  // elements j0..j0+3 and kHalf + j0..kHalf + j0+3
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
    uint2 xa[kBatch], xb[kBatch], ga[kBatch], gb[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int row = (rd0 + u) * kRowsPerRound + row0;
      int seg, pi;
      size_t off;
      locate(row, seg, off, pi);
      const bool active = row < rows_all;
      xa[u] = active ? *reinterpret_cast<const uint2*>(p.x[seg] + off) : make_uint2(0, 0);
      xb[u] = active ? *reinterpret_cast<const uint2*>(p.x[seg] + off + kHalf) : make_uint2(0, 0);
      if (kBwd) {
        ga[u] = active ? *reinterpret_cast<const uint2*>(p.dy[seg] + off) : make_uint2(0, 0);
        gb[u] = active ? *reinterpret_cast<const uint2*>(p.dy[seg] + off + kHalf) : make_uint2(0, 0);
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
          const unsigned long long pos = (unsigned long long)(unsigned)(t + (p.pos ? p.pos[b] : 0));
          const unsigned long long frac = pos * p.turns[j];
          const float ang = (float)(int)(unsigned)(frac >> 32) * 1.4629180792671596e-09f;  // 2 pi / 2^32
          __sincosf(ang, &sn, &c);
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
      // a[i] = element j0 + i, b[i] = element kHalf + j0 + i
      float a[4], bq[4];
      {
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa[u]);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb[u]);
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const float2 fa = __bfloat1622float2(a2[v]), fb = __bfloat1622float2(b2[v]);
          a[2 * v] = fa.x, a[2 * v + 1] = fa.y, bq[2 * v] = fb.x, bq[2 * v + 1] = fb.y;
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < 4; ++v) ss = fmaf(a[v], a[v], fmaf(bq[v], bq[v], ss));
#pragma unroll
      for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv_r = rsqrtf(ss * (1.f / D) + p.eps);
      const float4 t01 = cs4[pi][j0 / 2], t23 = cs4[pi][j0 / 2 + 1];
      const float c[4] = {t01.x, t01.z, t23.x, t23.z}, s[4] = {t01.y, t01.w, t23.y, t23.w};
      float oa[4], ob[4];
      if (!kBwd) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float xa_ = a[v] * inv_r, xb_ = bq[v] * inv_r;
          oa[v] = fmaf(-xb_, s[v], xa_ * c[v]);
          ob[v] = fmaf(xa_, s[v], xb_ * c[v]);
        }
      } else {
        // g = rotation of dy by -phi
        float ga_[4], gb_[4];
        {
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ga[u]);
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&gb[u]);
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const float2 fa = __bfloat1622float2(a2[v]), fb = __bfloat1622float2(b2[v]);
            ga_[2 * v] = fa.x, ga_[2 * v + 1] = fa.y, gb_[2 * v] = fb.x, gb_[2 * v + 1] = fb.y;
          }
        }
        float gra[4], grb[4], dot = 0.f;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          gra[v] = fmaf(gb_[v], s[v], ga_[v] * c[v]);
          grb[v] = fmaf(-ga_[v], s[v], gb_[v] * c[v]);
          dot = fmaf(gra[v], a[v] * inv_r, fmaf(grb[v], bq[v] * inv_r, dot));
        }
#pragma unroll
        for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float proj = dot * (1.f / D);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          oa[v] = (gra[v] - a[v] * inv_r * proj) * inv_r;
          ob[v] = (grb[v] - bq[v] * inv_r * proj) * inv_r;
        }
      }
      if (active) {
        *reinterpret_cast<uint2*>(p.y[seg] + off) = make_uint2(pack_bf16x2(oa[0], oa[1]), pack_bf16x2(oa[2], oa[3]));
        *reinterpret_cast<uint2*>(p.y[seg] + off + kHalf) =
            make_uint2(pack_bf16x2(ob[0], ob[1]), pack_bf16x2(ob[2], ob[3]));
      }
    }
  }
}

}  // namespace cswa
