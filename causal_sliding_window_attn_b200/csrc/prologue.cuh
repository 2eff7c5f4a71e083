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
// angle p * omega_j is reduced modulo 2*pi exactly in 64-bit fixed point, so
// the fp32 sin/cos see a small, accurate argument at any position.
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

// The angle of pair j at position p, in turns, is p * u_j with u_j = omega_j / (2 pi).
// u_j is held as a 64-bit fixed-point fraction U_j = u_j * 2^64, so that
// p * U_j mod 2^64 is the exact fractional part of p * u_j (to 2^-53 of u_j,
// from the fp64 value it was built from) for any 32-bit position; its top 32
// bits, read as a signed number, give the reduced angle in [-pi, pi).
template <int D>
__device__ __forceinline__ void rope_row_angles(const RopeParams& p, const unsigned long long* turns, int seg,
                                                long long r, int lane_in_row, float (&c)[8], float (&s)[8]) {
  const long long bt = r / p.H[seg];
  const int t = (int)(bt % p.T);
  const int b = (int)(bt / p.T);
  const unsigned long long pos = (unsigned long long)(unsigned)(t + (p.pos ? p.pos[b] : 0));
  constexpr int kHalfLanes = D / 16;
  const int j0 = (lane_in_row % kHalfLanes) * 8;  // first pair index of this lane
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const unsigned long long frac = pos * turns[j0 + u];
    const float ang = (float)(int)(unsigned)(frac >> 32) * 1.4629180792671596e-09f;  // 2 pi / 2^32
    __sincosf(ang, &s[u], &c[u]);
  }
}

// kBwd = false: y = prologue(x). kBwd = true: y = d prologue / dx applied to dy.
template <int D, bool kBwd>
__global__ void __launch_bounds__(256) rope_qknorm_kernel(const RopeParams p) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const long long total = p.rows[0] + p.rows[1];
  const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow;
  const int lr = lane % kLanesPerRow;
  const long long row = warp_global * kRowsPerWarp + sub;
  const bool active = row < total;
  const int seg = (active && row >= p.rows[0]) ? 1 : 0;
  const long long r = active ? (seg ? row - p.rows[0] : row) : 0;
  const bool second_half = lr >= kLanesPerRow / 2;

  // U_j = (base^(-2j/D) / (2 pi)) * 2^64, one table per block
  __shared__ unsigned long long turns[D / 2];
  for (int j = threadIdx.x; j < D / 2; j += blockDim.x) {
    const double u = exp2(-2.0 * (double)j / (double)D * p.log2_base) * 0.15915494309189533576888376337251;
    turns[j] = (unsigned long long)(u * 18446744073709551616.0);
  }
  __syncthreads();

  float x[8], g[8];
  if (active) {
    const uint4 xv = *reinterpret_cast<const uint4*>(p.x[seg] + r * D + lr * 8);
    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(x2[u]);
      x[2 * u] = f.x;
      x[2 * u + 1] = f.y;
    }
    if (kBwd) {
      const uint4 gv = *reinterpret_cast<const uint4*>(p.dy[seg] + r * D + lr * 8);
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
  if (active) {
    rope_row_angles<D>(p, turns, seg, r, lr, c, s);
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) c[u] = 1.f, s[u] = 0.f;
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
    *reinterpret_cast<uint4*>(p.y[seg] + r * D + lr * 8) = ov;
  }
}

}  // namespace cswa
