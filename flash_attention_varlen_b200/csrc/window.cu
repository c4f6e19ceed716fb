// Window segmentation on the device: the permutation that makes each win x win block of
// an image's patch grid a contiguous segment, its cu_seqlens, and a row gather/scatter.
//
// The vision tower attends within windows of 32 x 32 patches in its window layers (issue
// #1545 (vllm.cpp), follow-up comment, the section on the resolved labelled uncertainties:
// the window side comes from the positional-embedding grid).  Its hidden states are put
// in window order once, before the first layer, and back in image order once, after the
// last (PR #279, vision-tower port commit: the inverse permutation comes before ln_post and
// the RoPE table is permuted alongside).  So the attention kernel reads packed, contiguous
// segments in every layer, and the permutation is two row copies per tower.
//
// Order (the pages name the two orders without printing them; the plain row-major reading):
// images packed one after another in row-major patch order; each image's blocks walked
// row-major over its block grid, with smaller blocks along the bottom and right edges of a
// grid that is not a multiple of win; the tokens of a block row-major inside it.
#include "internal.h"

namespace vt {
namespace {

// Position p of the window-ordered sequence -> packed image-order token.  Row r of blocks
// of an image covers rows [r win, r win + hr) of all w columns (hr = min(win, h - r win)),
// so it holds win * w tokens unless it is the last one; inside it, block c holds hr * win
// tokens unless it is the last one of the row.
__global__ void window_perm_kernel(const WindowImages g, int32_t* __restrict__ perm,
                                   int32_t* __restrict__ cu) {
  const int64_t T = g.token_base[g.n];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; p < T; p += stride) {
    int i = 0;
    while (g.token_base[i + 1] <= p) ++i;
    const int h = g.h[i], w = g.w[i], win = g.win;
    const int64_t q = p - g.token_base[i];
    const int r = static_cast<int>(q / (static_cast<int64_t>(win) * w));
    const int hr = min(win, h - r * win);
    const int64_t qr = q - static_cast<int64_t>(r) * win * w;
    const int c = static_cast<int>(qr / (static_cast<int64_t>(hr) * win));
    const int wc = min(win, w - c * win);
    const int qc = static_cast<int>(qr - static_cast<int64_t>(c) * hr * win);
    const int y = r * win + qc / wc, x = c * win + qc % wc;
    perm[p] = static_cast<int32_t>(g.token_base[i] + static_cast<int64_t>(y) * w + x);
  }
  // cu_seqlens: block k of image i starts where the blocks before it end
  const int64_t nwin = g.window_base[g.n];
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k <= nwin; k += stride) {
    if (k == nwin) {
      cu[k] = static_cast<int32_t>(T);
      continue;
    }
    int i = 0;
    while (g.window_base[i + 1] <= k) ++i;
    const int h = g.h[i], w = g.w[i], win = g.win;
    const int nc = (w + win - 1) / win;
    const int kk = static_cast<int>(k - g.window_base[i]);
    const int r = kk / nc, c = kk % nc;
    const int hr = min(win, h - r * win);
    cu[k] = static_cast<int32_t>(g.token_base[i] + static_cast<int64_t>(r) * win * w +
                                 static_cast<int64_t>(c) * hr * win);
  }
}

// Set (never cleared by a kernel) when a permute met an index outside [0, rows); the host
// reads and clears it (permute_rows_check).  One word per device, shared by all calls.
__device__ int g_permute_bad_index;

// dst[i] = src[idx[i]] (gather) or dst[idx[i]] = src[i] (scatter), rows of row_bytes
// (a multiple of 16), one warp per row, 16-byte accesses.  A row whose index lies outside
// [0, rows) is skipped before any access (nothing read or written for it) and raises the
// device's flag, so a bad index from the caller cannot reach outside the two buffers.
__global__ void permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                    const int32_t* __restrict__ idx, int32_t rows,
                                    int32_t row_vec, int32_t scatter) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += warps) {
    const int64_t j = __ldg(idx + r);
    if (j < 0 || j >= rows) {
      if (lane == 0) atomicOr(&g_permute_bad_index, 1);
      continue;
    }
    const int64_t s = scatter ? r : j, d = scatter ? j : r;
    const uint4* sp = src + s * row_vec;
    uint4* dp = dst + d * row_vec;
    for (int v = lane; v < row_vec; v += 32) dp[v] = __ldg(sp + v);
  }
}

}  // namespace

cudaError_t permute_rows_check(int* bad) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_permute_bad_index, sizeof(int));
  if (e != cudaSuccess) return e;
  *bad = v;
  if (v) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_permute_bad_index, &zero, sizeof(int));
  }
  return e;
}

cudaError_t launch_window_perm(const WindowImages& g, int32_t* perm, int32_t* cu,
                               int num_sms, cudaStream_t stream) {
  const int64_t work = g.token_base[g.n] > g.window_base[g.n] + 1 ? g.token_base[g.n]
                                                                  : g.window_base[g.n] + 1;
  const int64_t blocks = (work + 255) / 256;
  const int grid = static_cast<int>(blocks < num_sms * 8 ? blocks : num_sms * 8);
  window_perm_kernel<<<grid, 256, 0, stream>>>(g, perm, cu);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* idx, int32_t rows,
                                int32_t row_bytes, int32_t scatter, int num_sms,
                                cudaStream_t stream) {
  const int64_t blocks = (static_cast<int64_t>(rows) + 7) / 8;  // 8 warps (rows) per block
  const int grid = static_cast<int>(blocks < num_sms * 16 ? blocks : num_sms * 16);
  permute_rows_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(src),
                                                static_cast<uint4*>(dst), idx, rows,
                                                row_bytes / 16, scatter);
  return cudaGetLastError();
}

}  // namespace vt
