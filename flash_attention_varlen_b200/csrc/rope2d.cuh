// 2D rotary position embedding of the vision tower (device math shared by the rotation
// pass and the attention kernel's Q prologue).
//
// PR #279 (vision-tower port commit) names the width-first 2D RoPE order and the 1-based
// RoPE positions; the pages print no formula.  Reading taken, for head width D = 96:
//   * a token carries 1-based positions (pw, ph) = (x + 1, y + 1) in its image's patch grid;
//   * frequencies f_i = theta^(-2 i / (D / 2)), i = 0 .. D/4 - 1 (host-computed in double);
//   * angle a_d = pw * f_d for d < D/4 and ph * f_{d - D/4} for D/4 <= d < D/2 (width first);
//   * element d < D/2 pairs with d + D/2:
//       out[d] = x[d] cos a_d - x[d + D/2] sin a_d,  out[d + D/2] = x[d + D/2] cos a_d + x[d] sin a_d.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace vt {

constexpr int kRopeD = 96;
constexpr int kRopeFreqs = kRopeD / 4;  // 24 per axis

// sin and cos of x = pos * f.  The angle is reduced to r = x - 2 pi k in [-pi, pi] by a
// two-term split of 2 pi (the float nearest 2 pi, then the remainder 2 pi - that float),
// both applied with a fused multiply-add, and the hardware approximations are used on r,
// where their absolute error is about 2^-21.
__device__ __forceinline__ void rope_sincos(float x, float* s, float* c) {
  constexpr float kInv2Pi = 0.159154943091895335768883763372514362f;
  constexpr float k2PiHi = 6.28318548202514648437500f;       // float(2 pi)
  constexpr float k2PiLo = -1.74845553146951715e-07f;        // 2 pi - float(2 pi)
  const float k = rintf(x * kInv2Pi);
  float r = fmaf(-k, k2PiHi, x);
  r = fmaf(-k, k2PiLo, r);
  __sincosf(r, s, c);
}

// Rotate the 8 pairs of one 16-byte group by one axis position p: lo holds columns
// 8u .. 8u+7 of the first half (u < 6), hi the columns 48 + 8u .. 48 + 8u + 7, and f8 the
// group's 8 frequencies.  D/4 = 24 is a multiple of 8, so all 8 columns of a group lie on
// one axis: groups 0-2 take the width position with f_{8u+j}, groups 3-5 the height
// position with f_{8(u-3)+j}.  Values are bf16, rounded to nearest-even after rotation.
template <typename Freqs>
__device__ __forceinline__ void rope_rotate8(uint4& lo, uint4& hi, float p, const Freqs& f8) {
  uint32_t a[4] = {lo.x, lo.y, lo.z, lo.w};
  uint32_t b[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float x0[2], x1[2];
    x0[0] = __uint_as_float(a[e] << 16);
    x0[1] = __uint_as_float(a[e] & 0xFFFF0000u);
    x1[0] = __uint_as_float(b[e] << 16);
    x1[1] = __uint_as_float(b[e] & 0xFFFF0000u);
    float y0[2], y1[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      float sn, cs;
      rope_sincos(p * f8[2 * e + k], &sn, &cs);
      y0[k] = fmaf(x0[k], cs, -x1[k] * sn);
      y1[k] = fmaf(x1[k], cs, x0[k] * sn);
    }
    uint32_t p0, p1;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p0) : "f"(y0[1]), "f"(y0[0]));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p1) : "f"(y1[1]), "f"(y1[0]));
    a[e] = p0;
    b[e] = p1;
  }
  lo = make_uint4(a[0], a[1], a[2], a[3]);
  hi = make_uint4(b[0], b[1], b[2], b[3]);
}

// The same for group u of a token at 1-based positions (pw, ph), freq the D/4 frequencies.
__device__ __forceinline__ void rope_rotate_group(uint4& lo, uint4& hi, int u, float pw, float ph,
                                                  const float* freq) {
  rope_rotate8(lo, hi, u < 3 ? pw : ph, freq + 8 * (u < 3 ? u : u - 3));
}

}  // namespace vt
