// f32-input varlen attention forward on the FP32 FMA pipes.
//
// The exactness arm of the library: the same block-diagonal softmax(QK^T s)V
// as the bf16 tensor-core kernel, in f32 throughout (no TF32), for inputs whose
// tolerance (1e-5 max-abs) a 10-bit-mantissa tensor path cannot meet.
//
// Work unit: 64 query rows of one (segment, head).  128 threads: two threads
// per query row, each owning 48 of the 96 columns of q and of the output
// accumulator; a score is the sum of the two halves (one shuffle).  Keys and
// values stream through shared memory in tiles of 32 rows; a running
// (online) softmax keeps the row max m and the row sum l.
#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = kF32BlockRows;  // 64
constexpr int kKeys = 32;
constexpr int kD = 96;
constexpr int kHalf = kD / 2;  // 48

struct F32Smem {
  float k[kKeys][kD];
  float v[kKeys][kD];
};

__global__ void __launch_bounds__(kThreads) attn_f32_kernel(const F32Args a) {
  __shared__ __align__(16) F32Smem sm;
  const int tid = threadIdx.x;
  const int r = tid >> 1, half = tid & 1;
  const int H = a.H;
  const int E = a.hdr->num_entries;
  const long long total_units = static_cast<long long>(E) * H;
  // the bf16 kernel's unit order: a snake over the CTAs, entry-major (longest segment
  // first) when the segments differ in length and head-major when they do not
  const bool entry_major = a.hdr->order != 0;
  const long long G = gridDim.x, cta = blockIdx.x;

  for (long long k = 0;; ++k) {
    const long long u = k * G + ((k & 1) ? G - 1 - cta : cta);
    if (u >= total_units) break;
    const int e = static_cast<int>(entry_major ? u / H : u % E);
    const int h = static_cast<int>(entry_major ? u % H : u / E);
    const WorkEntry we = a.entries[e];
    const int seg_start = we.seg_start, seg_end = we.seg_end;
    const int row = seg_start + we.qblock * kRows + r;
    const bool row_ok = row < seg_end;

    float q[kHalf], o[kHalf];
    const float* qp = a.q + (static_cast<size_t>(row) * H + h) * kD + half * kHalf;
#pragma unroll
    for (int i = 0; i < kHalf; i += 4) {
      float4 t = row_ok ? *reinterpret_cast<const float4*>(qp + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      q[i] = t.x; q[i + 1] = t.y; q[i + 2] = t.z; q[i + 3] = t.w;
      o[i] = o[i + 1] = o[i + 2] = o[i + 3] = 0.f;
    }
    float m = -INFINITY, l = 0.f;

    for (int kv0 = seg_start; kv0 < seg_end; kv0 += kKeys) {
      const int nvalid = min(kKeys, seg_end - kv0);
      __syncthreads();  // previous tile fully consumed
      for (int i = tid; i < kKeys * (kD / 4); i += kThreads) {
        const int kr = i / (kD / 4), c4 = (i % (kD / 4)) * 4;
        float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
        if (kr < nvalid) {
          const size_t off = (static_cast<size_t>(kv0 + kr) * H + h) * kD + c4;
          kk = *reinterpret_cast<const float4*>(a.k + off);
          vv = *reinterpret_cast<const float4*>(a.v + off);
        }
        *reinterpret_cast<float4*>(&sm.k[kr][c4]) = kk;
        *reinterpret_cast<float4*>(&sm.v[kr][c4]) = vv;
      }
      __syncthreads();

      float t[kKeys];
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        const float* kr = &sm.k[c][half * kHalf];
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kHalf; i += 4) {
          const float4 kk = *reinterpret_cast<const float4*>(kr + i);
          acc = fmaf(q[i], kk.x, acc);
          acc = fmaf(q[i + 1], kk.y, acc);
          acc = fmaf(q[i + 2], kk.z, acc);
          acc = fmaf(q[i + 3], kk.w, acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        t[c] = (c < nvalid) ? acc * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, t[c]);
      }
      const float m_new = fmaxf(m, tmax);
      const float alpha = exp2f(m - m_new);  // m = -inf on the first tile -> 0
      l *= alpha;
#pragma unroll
      for (int i = 0; i < kHalf; ++i) o[i] *= alpha;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        const float p = (c < nvalid) ? exp2f(t[c] - m_new) : 0.f;
        l += p;
        const float* vr = &sm.v[c][half * kHalf];
#pragma unroll
        for (int i = 0; i < kHalf; i += 4) {
          const float4 vv = *reinterpret_cast<const float4*>(vr + i);
          o[i] = fmaf(p, vv.x, o[i]);
          o[i + 1] = fmaf(p, vv.y, o[i + 1]);
          o[i + 2] = fmaf(p, vv.z, o[i + 2]);
          o[i + 3] = fmaf(p, vv.w, o[i + 3]);
        }
      }
      m = m_new;
    }

    if (row_ok) {
      const float inv_l = 1.0f / l;
      float* op = a.out + (static_cast<size_t>(row) * H + h) * kD + half * kHalf;
#pragma unroll
      for (int i = 0; i < kHalf; i += 4)
        *reinterpret_cast<float4*>(op + i) =
            make_float4(o[i] * inv_l, o[i + 1] * inv_l, o[i + 2] * inv_l, o[i + 3] * inv_l);
    }
  }
}

}  // namespace

size_t f32_smem_bytes() { return sizeof(F32Smem); }

cudaError_t launch_attn_f32(const F32Args& args, int grid, cudaStream_t stream) {
  attn_f32_kernel<<<grid, kThreads, 0, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace vt
