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
// HBM-bound elementwise work: D/8 lanes own one row, 16 bytes each (one
// vector load per operand), the pair partner j + D/2 is a shuffle away. The
// angles are computed once per position and shared by all its head rows.
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
  double log2_base;
};

// Each block owns kPosPerBlock consecutive (b, t) positions and every q and k
// head row at them. It first builds one cos/sin table per position in shared
// memory -- the angle of pair j at position p, in turns, is p * u_j with
// u_j = omega_j / (2 pi), held as a 64-bit fixed-point fraction U_j = u_j 2^64,
// so p * U_j mod 2^64 is the exact fractional turn for any 32-bit position and
// its top 32 bits, read as signed, give the reduced angle in [-pi, pi) -- and
// then streams the rows: D/8 lanes per row, one 16-byte load per operand.
constexpr int kPosPerBlock = 8;

template <int D, bool kBwd>
__global__ void __launch_bounds__(256) rope_qknorm_kernel(const RopeParams p) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kHalf = D / 2;
  __shared__ unsigned long long turns[kHalf];
  __shared__ float2 cs[kPosPerBlock][kHalf];  // (cos, sin)

  const long long n_pos = p.rows[0] > 0 ? p.rows[0] / p.H[0] : p.rows[1] / p.H[1];  // B * T
  const long long pos0 = (long long)blockIdx.x * kPosPerBlock;
  const int Hq = p.rows[0] > 0 ? p.H[0] : 0;
  const int Hk = p.rows[1] > 0 ? p.H[1] : 0;

  for (int j = threadIdx.x; j < kHalf; j += blockDim.x) {
    const double u = exp2(-2.0 * (double)j / (double)D * p.log2_base) * 0.15915494309189533576888376337251;
    turns[j] = (unsigned long long)(u * 18446744073709551616.0);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kPosPerBlock * kHalf; e += blockDim.x) {
    const int pi = e / kHalf, j = e % kHalf;
    const long long bt = pos0 + pi;
    float c = 1.f, sn = 0.f;
    if (bt < n_pos) {
      const int t = (int)(bt % p.T), b = (int)(bt / p.T);
      const unsigned long long pos = (unsigned long long)(unsigned)(t + (p.pos ? p.pos[b] : 0));
      const unsigned long long frac = pos * turns[j];
      const float ang = (float)(int)(unsigned)(frac >> 32) * 1.4629180792671596e-09f;  // 2 pi / 2^32
      __sincosf(ang, &sn, &c);
    }
    cs[pi][j] = make_float2(c, sn);
  }
  __syncthreads();

  const int n_pos_here = (int)min((long long)kPosPerBlock, n_pos - pos0);
  const int rows_q = n_pos_here * Hq, rows_k = n_pos_here * Hk;
  const int tasks = (rows_q + rows_k) * kLanesPerRow;
  const int lr = threadIdx.x % kLanesPerRow;
  const bool second_half = lr >= kLanesPerRow / 2;
  const int j0 = (lr % (kLanesPerRow / 2)) * 8;
  // every thread runs the same trip count so the row shuffles stay warp-uniform
  const int trips = (kPosPerBlock * (Hq + Hk) * kLanesPerRow + blockDim.x - 1) / blockDim.x;
  for (int tr = 0; tr < trips; ++tr) {
    const int task = tr * blockDim.x + threadIdx.x;
    const bool active = task < tasks;
    const int row = task / kLanesPerRow;
    const int seg = (row >= rows_q) ? 1 : 0;
    const int rr = seg ? row - rows_q : row;                 // row within the segment, block-local
    const int H = seg ? Hk : Hq;
    const int pi = active ? rr / H : 0;
    const long long grow = (pos0 * H) + rr;                  // global row of the segment
    float x[8], g[8];
    if (active) {
      const uint4 xv = *reinterpret_cast<const uint4*>(p.x[seg] + grow * D + lr * 8);
      const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(x2[u]);
        x[2 * u] = f.x;
        x[2 * u + 1] = f.y;
      }
      if (kBwd) {
        const uint4 gv = *reinterpret_cast<const uint4*>(p.dy[seg] + grow * D + lr * 8);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(g2[u]);
          g[2 * u] = f.x;
          g[2 * u + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = g[u] = 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) ss = fmaf(x[u], x[u], ss);
#pragma unroll
    for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv_r = rsqrtf(ss * (1.f / D) + p.eps);
    float c[8], s[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float2 t = cs[pi][j0 + u];
      c[u] = t.x;
      s[u] = t.y;
    }
    float out[8];
    if (!kBwd) {
      float xh[8], partner[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) xh[u] = x[u] * inv_r;
#pragma unroll
      for (int u = 0; u < 8; ++u) partner[u] = __shfl_xor_sync(0xffffffffu, xh[u], kLanesPerRow / 2);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        out[u] = second_half ? fmaf(partner[u], s[u], xh[u] * c[u]) : fmaf(-partner[u], s[u], xh[u] * c[u]);
    } else {
      // g = rotation of dy by -phi
      float partner[8], gr[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) partner[u] = __shfl_xor_sync(0xffffffffu, g[u], kLanesPerRow / 2);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        gr[u] = second_half ? fmaf(-partner[u], s[u], g[u] * c[u]) : fmaf(partner[u], s[u], g[u] * c[u]);
      float dot = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) dot = fmaf(gr[u], x[u] * inv_r, dot);
#pragma unroll
      for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float proj = dot * (1.f / D);
#pragma unroll
      for (int u = 0; u < 8; ++u) out[u] = (gr[u] - x[u] * inv_r * proj) * inv_r;
    }
    if (active) {
      uint4 ov;
      uint32_t* o32 = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
      for (int u = 0; u < 4; ++u) o32[u] = pack_bf16x2(out[2 * u], out[2 * u + 1]);
      *reinterpret_cast<uint4*>(p.y[seg] + grow * D + lr * 8) = ov;
    }
  }
}

}  // namespace cswa
