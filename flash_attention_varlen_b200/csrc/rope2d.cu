// The 2D RoPE rotation pass: out = rope(x) for a bf16 [T, H, 96] tensor (out may be x).
//
// HBM-bound: each (token, head) row of 192 bytes is read and written once.  One thread
// handles (token, head, group u < 6) items: the 16-byte group of columns 8u .. 8u+7 and its
// partner 48 + 8u .. 48 + 8u + 7.  Consecutive threads take consecutive groups of a row and
// consecutive rows, so a warp reads and writes contiguous bytes.  Blocks of 192 threads and
// a grid stride that is a multiple of 6 keep a thread on one group u, so its 8 frequencies
// sit in registers for all its items.  blockIdx.y picks the tensor when one launch rotates
// two (Q and K share the positions).
#include <cmath>

#include "internal.h"
#include "ptx.cuh"
#include "rope2d.cuh"

namespace vt {
namespace {

constexpr int kRopeBlock = 192;  // a multiple of the 6 groups of a row

struct RopeTensors {
  const uint4* x[kRopeMaxTensors];
  uint4* out[kRopeMaxTensors];  // out[i] may be x[i]: each thread reads its groups first
};

__global__ void __launch_bounds__(kRopeBlock)
    rope2d_kernel(const __grid_constant__ RopeTensors io, const int32_t* __restrict__ pos,
                  int32_t T, int32_t H, const __grid_constant__ RopeFreqs f) {
  // An attention kernel queued next may start its set-up now; it reads the rotated tensors
  // only after this grid has completed.
  griddep_launch_dependents();
  const uint4* x = io.x[blockIdx.y];
  uint4* out = io.out[blockIdx.y];
  const int u = static_cast<int>(threadIdx.x % 6);
  const int fb = 8 * (u < 3 ? u : u - 3);
  float f8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) f8[j] = f.f[fb + j];
  const int64_t items = static_cast<int64_t>(T) * H * 6;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kRopeBlock;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * kRopeBlock + threadIdx.x; it < items;
       it += stride) {
    const int64_t row = it / 6;  // token * H + head; it % 6 == u
    const int2 p = __ldg(reinterpret_cast<const int2*>(pos) + row / H);
    uint4 lo = x[row * 12 + u], hi = x[row * 12 + 6 + u];  // 12 groups of 16 bytes per row
    rope_rotate8(lo, hi, static_cast<float>(u < 3 ? p.x : p.y), f8);
    out[row * 12 + u] = lo;
    out[row * 12 + 6 + u] = hi;
  }
}

}  // namespace

RopeFreqs rope_freqs(double theta) {
  RopeFreqs f;
  for (int i = 0; i < kRopeFreqs; ++i)
    f.f[i] = static_cast<float>(std::pow(theta, -2.0 * i / (kRopeD / 2)));
  return f;
}

cudaError_t launch_rope2d(const void* const* x, void* const* out, int count, const int32_t* pos,
                          int32_t T, int32_t H, const RopeFreqs& f, int num_sms,
                          cudaStream_t stream) {
  if (count < 1 || count > kRopeMaxTensors) return cudaErrorInvalidValue;
  RopeTensors io = {};
  for (int i = 0; i < count; ++i) {
    io.x[i] = static_cast<const uint4*>(x[i]);
    io.out[i] = static_cast<uint4*>(out[i]);
  }
  const int64_t items = static_cast<int64_t>(T) * H * 6;
  const int64_t blocks = (items + kRopeBlock - 1) / kRopeBlock;
  const int64_t cap = static_cast<int64_t>(num_sms) * 64 / count;
  const dim3 grid(static_cast<unsigned>(blocks < cap ? blocks : cap), static_cast<unsigned>(count));
  rope2d_kernel<<<grid, kRopeBlock, 0, stream>>>(io, pos, T, H, f);
  return cudaGetLastError();
}

}  // namespace vt
