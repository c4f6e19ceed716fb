// The 2D RoPE rotation pass: out = rope(x) for a bf16 [T, H, 96] tensor (out may be x).
//
// HBM-bound: each (token, head) row of 192 bytes is read and written once.  One thread owns
// one 16-byte group u < 6 of the first half of a token's rows (columns 8u .. 8u+7, paired
// with 48 + 8u .. 48 + 8u + 7) for every head, so each of its 8 angles is computed once per
// token and reused across the H heads.
#include <cmath>

#include "internal.h"
#include "rope2d.cuh"

namespace vt {
namespace {

__global__ void __launch_bounds__(256)
    rope2d_kernel(const uint4* x, uint4* out, const int32_t* __restrict__ pos, int32_t T,
                  int32_t H, const RopeFreqs f) {  // out may be x: each thread reads its groups first
  const int64_t items = static_cast<int64_t>(T) * 6;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
       it += stride) {
    const int64_t t = it / 6;
    const int u = static_cast<int>(it - t * 6);
    const int2 p = __ldg(reinterpret_cast<const int2*>(pos) + t);
    const float pw = static_cast<float>(p.x), ph = static_cast<float>(p.y);
    for (int h = 0; h < H; ++h) {
      const int64_t row = (t * H + h) * 12;  // 12 groups of 16 bytes per 96-column row
      uint4 lo = x[row + u], hi = x[row + 6 + u];
      rope_rotate_group(lo, hi, u, pw, ph, f.f);
      out[row + u] = lo;
      out[row + 6 + u] = hi;
    }
  }
}

}  // namespace

RopeFreqs rope_freqs(double theta) {
  RopeFreqs f;
  for (int i = 0; i < kRopeFreqs; ++i)
    f.f[i] = static_cast<float>(std::pow(theta, -2.0 * i / (kRopeD / 2)));
  return f;
}

cudaError_t launch_rope2d(const void* x, void* out, const int32_t* pos, int32_t T, int32_t H,
                          const RopeFreqs& f, int num_sms, cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(T) * 6;
  const int64_t blocks = (items + 255) / 256;
  const int grid = static_cast<int>(blocks < num_sms * 8 ? blocks : num_sms * 8);
  rope2d_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(x), static_cast<uint4*>(out),
                                          pos, T, H, f);
  return cudaGetLastError();
}

}  // namespace vt
