// Scheduling prepass for the varlen attention kernels.
//
// The segments of one call (cu_seqlens, on the device) are cut into work
// entries of `block_rows` query rows, ordered longest segment first.  The bf16
// kernel deals its units out in a snake over the CTAs, entry-major (longest
// first) when the segments differ in length and head-major when they do not (the
// header's order flag), and the f32 kernel walks its units the same way.  The
// cheap units come last and fill the tail
// (longest-processing-time-first list scheduling).  Lengths are validated here, before any loop depends on them, so
// a malformed cu_seqlens produces an empty work list and an error flag instead of
// out-of-range reads.
#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

constexpr int kThreads = 1024;
constexpr int kSortMax = 4096;  // calls with more segments keep their given order

__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += t;
  }
  return v;
}

__global__ void __launch_bounds__(kThreads)
    schedule_kernel(const int32_t* __restrict__ cu, int32_t n, int32_t T, int32_t block_rows,
                    int slot, WorkHeader* hdr, WorkEntry* entries) {
  __shared__ unsigned long long keys[kSortMax];
  __shared__ int warp_sums[32];
  __shared__ int chunk_total;
  __shared__ int len_min, len_max;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // The attention kernel that follows may launch now and set itself up while this runs;
  // it reads the work list only after this grid has completed.
  griddep_launch_dependents();
  if (tid == 0) {
    len_min = 0x7FFFFFFF;
    len_max = 0;
  }
  __syncthreads();

  // 1) validation: cu[0] == 0, cu[n] == T, non-decreasing.
  int bad = 0;
  if (tid == 0 && (cu[0] != 0 || cu[n] != T)) bad = 1;
  for (int s = tid; s < n; s += kThreads) {
    const int len = cu[s + 1] - cu[s];
    if (len < 0) bad = 1;
    if (len > 0) {  // the range of the non-empty lengths decides the unit order
      atomicMin(&len_min, len);
      atomicMax(&len_max, len);
    }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      hdr->status[slot] = kDevStatusBadSeqlens;
      hdr->status[slot ^ 1] = 0;
      hdr->num_entries = 0;
      hdr->order = 0;
    }
    return;
  }

  const bool do_sort = n <= kSortMax;
  int base = 0;
  for (int c0 = 0; c0 < n; c0 += kSortMax) {
    const int cn = min(kSortMax, n - c0);
    int padded = cn;
    if (do_sort) {
      padded = 1;
      while (padded < cn) padded <<= 1;
    }
    // key = (INT_MAX - len) << 32 | seg: ascending order = longest first, ties by index
    for (int i = tid; i < padded; i += kThreads) {
      if (i < cn) {
        const int s = c0 + i;
        const unsigned len = static_cast<unsigned>(cu[s + 1] - cu[s]);
        keys[i] = (static_cast<unsigned long long>(0x7FFFFFFFu - len) << 32) |
                  static_cast<unsigned>(s);
      } else {
        keys[i] = ~0ull;
      }
    }
    __syncthreads();
    if (do_sort) {  // bitonic sort, ascending
      for (int k = 2; k <= padded; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
          for (int i = tid; i < padded; i += kThreads) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const unsigned long long a = keys[i], b = keys[ixj];
              const bool up = (i & k) == 0;
              if ((a > b) == up) {
                keys[i] = b;
                keys[ixj] = a;
              }
            }
          }
          __syncthreads();
        }
      }
    }
    // 2) entries per segment, exclusive scan, then write.  Thread t owns items 4t..4t+3.
    int cnt[4], segs[4], starts[4], ends[4], local = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = tid * 4 + r;
      cnt[r] = 0;
      segs[r] = 0;
      starts[r] = ends[r] = 0;
      if (i < cn) {
        const int s = static_cast<int>(keys[i] & 0xFFFFFFFFull);
        starts[r] = cu[s];
        ends[r] = cu[s + 1];
        const int len = ends[r] - starts[r];
        segs[r] = s;
        cnt[r] = (len + block_rows - 1) / block_rows;
      }
      local += cnt[r];
    }
    const int incl = warp_inclusive_scan(local);
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int w = warp_sums[lane];
      const int wi = warp_inclusive_scan(w);
      warp_sums[lane] = wi - w;
      if (lane == 31) chunk_total = wi;
    }
    __syncthreads();
    int off = base + warp_sums[warp] + incl - local;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      for (int b = 0; b < cnt[r]; ++b) entries[off++] = WorkEntry{segs[r], b, starts[r], ends[r]};
    base += chunk_total;
    __syncthreads();
  }
  if (tid == 0) {
    hdr->num_entries = base;
    hdr->order = (do_sort && len_min < len_max) ? 1 : 0;  // unequal lengths: longest first
    hdr->status[slot] = 0;
    hdr->status[slot ^ 1] = 0;
  }
}

}  // namespace

cudaError_t launch_schedule(const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                            int32_t block_rows, int slot, WorkHeader* hdr, WorkEntry* entries,
                            cudaStream_t stream) {
  schedule_kernel<<<1, kThreads, 0, stream>>>(cu_seqlens, num_segments, total_tokens, block_rows,
                                              slot, hdr, entries);
  return cudaGetLastError();
}

}  // namespace vt
