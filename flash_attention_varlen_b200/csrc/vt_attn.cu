// C-ABI entry points of libvtattn (declared in include/vt_attn.h).
//
// Host side only: argument validation, the per-(device, stream) scratch
// buffer that holds the work list, TMA descriptors for the bf16 kernel, and
// the two launches of a call (scheduling prepass, then the attention kernel).
#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "internal.h"
#include "ptx.cuh"
#include "vt_attn.h"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
constexpr int kHeadDim = 96;

struct DeviceInfo {
  bool init = false;
  int num_sms = 0;
  bool bf16_ready = false;
  bool f32_ready = false;
  bool swa_ready = false;
};

struct Scratch {
  void* ptr = nullptr;
  size_t bytes = 0;
  uint32_t calls = 0;  // forward calls queued on this scratch: their status slots alternate
  int last_slot = 0;   // status slot of the latest one
  // the split-key epilogue's workspace (rows' halves, then per-row flags) for up to
  // split_units units, and the id of the latest call that used it
  void* split_ptr = nullptr;
  long long split_units = 0;
  uint32_t split_calls = 0;
};

std::mutex g_mu;      // the per-stream work lists
std::mutex g_dev_mu;  // the per-device launch information
DeviceInfo g_dev[kMaxDevices];
std::map<std::pair<int, uintptr_t>, Scratch> g_scratch;

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// [T, H, D] bf16 viewed as (d, h, t); a box is 32 columns x 1 head x 128 rows, stored
// with the 64-byte swizzle (32 columns = 64 bytes per row) the MMA descriptors expect.
vt_status make_tensor_map(CUtensorMap* map, const void* base, int32_t T, int32_t H,
                          int32_t D = kHeadDim) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return VT_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(H) * D * 2};
  const cuuint32_t box[3] = {32, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VT_OK : VT_ERR_CUDA;
}

vt_status device_info(int dev, DeviceInfo** out) {
  if (dev < 0 || dev >= kMaxDevices) return VT_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return VT_ERR_CUDA;
    d.init = true;
  }
  *out = &d;
  return VT_OK;
}

// Scratch of at least `need` bytes for (dev, stream); grows by reallocation
// after draining the stream's earlier work that may still read the old buffer.
vt_status scratch_for(int dev, cudaStream_t stream, size_t need, Scratch** out) {
  Scratch& s = g_scratch[{dev, reinterpret_cast<uintptr_t>(stream)}];
  if (s.bytes < need) {
    size_t nb = need;
    if (nb < 2 * s.bytes) nb = 2 * s.bytes;
    if (nb < (64u << 10)) nb = 64u << 10;
    if (s.ptr) {
      if (cudaStreamSynchronize(stream) != cudaSuccess) return VT_ERR_CUDA;
      cudaFree(s.ptr);
      s.ptr = nullptr;
      s.bytes = 0;
    }
    if (cudaMalloc(&s.ptr, nb) != cudaSuccess) {
      s.ptr = nullptr;
      return VT_ERR_CUDA;
    }
    if (cudaMemsetAsync(s.ptr, 0, sizeof(vt::WorkHeader), stream) != cudaSuccess) return VT_ERR_CUDA;
    s.bytes = nb;
  }
  *out = &s;
  return VT_OK;
}

int block_rows_for(vt_dtype dtype) {
  return dtype == VT_DTYPE_BF16 ? vt::kBf16BlockRows : vt::kF32BlockRows;
}

}  // namespace

extern "C" {

vt_status vt_attn_validate_seqlens_host(const int32_t* cu, int32_t num_segments,
                                        int32_t total_tokens) {
  if (!cu) return VT_ERR_NULL;
  if (num_segments < 0 || total_tokens < 0) return VT_ERR_BAD_SEQLENS;
  if (cu[0] != 0 || cu[num_segments] != total_tokens) return VT_ERR_BAD_SEQLENS;
  for (int32_t s = 0; s < num_segments; ++s)
    if (cu[s + 1] < cu[s]) return VT_ERR_BAD_SEQLENS;
  return VT_OK;
}

size_t vt_attn_smem_bytes(int32_t D, vt_dtype dtype) {
  if (D != kHeadDim) return 0;
  if (dtype == VT_DTYPE_BF16) return vt::bf16_smem_bytes();
  if (dtype == VT_DTYPE_F32) return vt::f32_smem_bytes();
  return 0;
}

size_t vt_attn_workspace_bytes(int32_t num_segments, int32_t total_tokens, vt_dtype dtype) {
  if (num_segments < 0 || total_tokens < 0) return 0;
  if (dtype != VT_DTYPE_BF16 && dtype != VT_DTYPE_F32) return 0;
  return vt::scratch_bytes_for(total_tokens, num_segments, block_rows_for(dtype));
}

}  // extern "C"

namespace vt {

int block_rows_for_dtype(int dtype) { return block_rows_for(static_cast<vt_dtype>(dtype)); }

int check_fwd_args(const FwdCall& c, int32_t D, bool* no_work) {
  *no_work = false;
  if (c.dtype != VT_DTYPE_BF16 && c.dtype != VT_DTYPE_F32) return VT_ERR_INVALID_ARG;
  if (c.H < 1 || D < 1 || c.num_segments < 0 || c.total_tokens < 0) return VT_ERR_INVALID_ARG;
  if (!std::isfinite(c.scale)) return VT_ERR_INVALID_ARG;
  if (D != kHeadDim) return VT_ERR_UNSUPPORTED;
  if (c.num_segments == 0) {
    *no_work = true;
    return c.total_tokens == 0 ? VT_OK : VT_ERR_BAD_SEQLENS;
  }
  if (!c.cu_seqlens) return VT_ERR_NULL;
  if (c.total_tokens == 0) {  // every segment is empty: nothing to write
    *no_work = true;
    return VT_OK;
  }
  if (!c.q || !c.k || !c.v || !c.out) return VT_ERR_NULL;
  const uintptr_t align_or = reinterpret_cast<uintptr_t>(c.q) | reinterpret_cast<uintptr_t>(c.k) |
                             reinterpret_cast<uintptr_t>(c.v) | reinterpret_cast<uintptr_t>(c.out);
  if (align_or & 15u) return VT_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c.H) * D > (1 << 20)) return VT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(c.cu_seqlens) & 3u) return VT_ERR_INVALID_ARG;
  const size_t elem = c.dtype == VT_DTYPE_BF16 ? 2 : 4;
  const size_t bytes = static_cast<size_t>(c.total_tokens) * c.H * D * elem;
  if (ranges_overlap(c.out, bytes, c.q, bytes) || ranges_overlap(c.out, bytes, c.k, bytes) ||
      ranges_overlap(c.out, bytes, c.v, bytes))
    return VT_ERR_INVALID_ARG;
  return VT_OK;
}

int launch_fwd(const FwdCall& c, WorkHeader* hdr, WorkEntry* entries, int slot) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VT_ERR_CUDA;
  DeviceInfo* di = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    vt_status st = device_info(dev, &di);
    if (st != VT_OK) return st;
    if (c.dtype == VT_DTYPE_BF16 && !di->bf16_ready) {
      if (prepare_attn_bf16() != cudaSuccess) return VT_ERR_CUDA;
      di->bf16_ready = true;
    }
    if (c.dtype == VT_DTYPE_F32 && !di->f32_ready) {
      if (prepare_attn_f32() != cudaSuccess) return VT_ERR_CUDA;
      di->f32_ready = true;
    }
  }
  const int block_rows = block_rows_for_dtype(c.dtype);
  // A bf16 call with few segments needs no prepass: its kernel builds the work list.
  const bool inline_sched = c.dtype == VT_DTYPE_BF16 && c.num_segments <= kInlineSegments;
  if (!inline_sched && launch_schedule(c.cu_seqlens, c.num_segments, c.total_tokens, block_rows,
                                       slot, hdr, entries, c.stream) != cudaSuccess)
    return VT_ERR_CUDA;

  const long long max_units =
      static_cast<long long>(max_work_entries(c.total_tokens, c.num_segments, block_rows)) * c.H;
  if (c.dtype == VT_DTYPE_BF16) {
    CUtensorMap tq, tk, tv, to;
    vt_status st;
    if ((st = make_tensor_map(&tq, c.q, c.total_tokens, c.H)) != VT_OK) return st;
    if ((st = make_tensor_map(&tk, c.k, c.total_tokens, c.H)) != VT_OK) return st;
    if ((st = make_tensor_map(&tv, c.v, c.total_tokens, c.H)) != VT_OK) return st;
    if ((st = make_tensor_map(&to, c.out, c.total_tokens, c.H)) != VT_OK) return st;
    Bf16Args a;
    a.out = c.out;
    a.cu_seqlens = c.cu_seqlens;
    a.hdr = hdr;
    a.entries = entries;
    a.dev_status = &hdr->status[slot];
    a.next_status = &hdr->status[slot ^ 1];
    a.num_segments = c.num_segments;
    a.total_tokens = c.total_tokens;
    a.inline_sched = inline_sched ? 1 : 0;
    a.H = c.H;
    a.out_align32 = (reinterpret_cast<uintptr_t>(c.out) & 31u) == 0;
    const double log2e = 1.4426950408889634;
    a.scale_log2 = static_cast<float>(std::fabs(static_cast<double>(c.scale)) * log2e);
    a.idesc_qk = make_idesc_bf16(128, 128, false, false, c.scale < 0.0f);
    a.stall_test_cycles = c.stall_test_cycles;
    const bool split = c.part != nullptr;
    a.part = c.part;
    a.part_flag = c.part_flag;
    a.call_id = c.call_id;
    a.split_units_max = c.split_units_max;
    const long long units = split ? 2 * max_units : max_units;
    const int grid = static_cast<int>(units < di->num_sms ? units : di->num_sms);
    // Staged O stores pay off when a CTA runs several short units (window layers); with
    // one or two units per CTA the store's tail latency costs more than it hides.  The
    // host sees only T and n (cu_seqlens stays on the device), so the rule uses the mean.
    const int64_t rows_x_heads = static_cast<int64_t>(c.total_tokens) * c.H;
    const bool stage_o =
        static_cast<int64_t>(c.total_tokens) <= static_cast<int64_t>(kStageMaxMeanSegment) * c.num_segments &&
        rows_x_heads >= static_cast<int64_t>(kStageMinUnitsPerSm) * di->num_sms * kBf16BlockRows;
    const int epilogue = split ? kEpiSplit : stage_o ? kEpiStaged : kEpiRows;
    if (launch_attn_bf16(tq, tk, tv, to, a, grid, epilogue, c.stream) != cudaSuccess) return VT_ERR_CUDA;
  } else {
    F32Args a;
    a.q = static_cast<const float*>(c.q);
    a.k = static_cast<const float*>(c.k);
    a.v = static_cast<const float*>(c.v);
    a.out = static_cast<float*>(c.out);
    a.hdr = hdr;
    a.entries = entries;
    a.dev_status = &hdr->status[slot];
    a.H = c.H;
    a.T = c.total_tokens;
    a.scale_log2 = static_cast<float>(static_cast<double>(c.scale) * 1.4426950408889634);
    const int grid = static_cast<int>(max_units < di->num_sms ? max_units : di->num_sms);
    if (launch_attn_f32(a, grid, c.stream) != cudaSuccess) return VT_ERR_CUDA;
  }
  return VT_OK;
}

}  // namespace vt

namespace {

int sm_count();  // of the current device; 0 if it cannot be read

std::atomic<int32_t> g_split_keys{1};  // vt_attn_set_split_keys

// The forward of a validated call with the library-owned, per-(device, stream) work list.
vt_status fwd_impl(const vt::FwdCall& c) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  Scratch* sc = nullptr;
  const vt_status st = scratch_for(dev, c.stream,
                   vt::scratch_bytes_for(c.total_tokens, c.num_segments,
                                         vt::block_rows_for_dtype(c.dtype)),
                   &sc);
  if (st != VT_OK) return st;
  auto* hdr = static_cast<vt::WorkHeader*>(sc->ptr);
  vt::FwdCall call = c;
  // A bf16 call with at most half as many (entry, head) units as SMs splits each unit's
  // keys over two CTAs (two units) and combines them in the kernel's epilogue.  The kernel
  // counts the units from the work list and decides; the host only rules the split out
  // when even the fewest units the call can have, ceil(T / 256) per head, are too many,
  // or when no segment can be long enough to split.
  const long long fewest =
      (static_cast<long long>(c.total_tokens) + vt::kBf16BlockRows - 1) / vt::kBf16BlockRows * c.H;
  const int nsm = sm_count();
  if (c.dtype == VT_DTYPE_BF16 && g_split_keys.load(std::memory_order_relaxed) != 0 && nsm > 1 &&
      2 * fewest <= nsm &&
      c.total_tokens > (vt::kSplitMinKeyTiles - 1) * 128) {
    if (sc->split_units < nsm / 2) {
      if (sc->split_ptr) {
        if (cudaStreamSynchronize(c.stream) != cudaSuccess) return VT_ERR_CUDA;
        cudaFree(sc->split_ptr);
        sc->split_ptr = nullptr;
        sc->split_units = 0;
      }
      const long long cap = nsm / 2;  // covers every call that can split on this device
      const size_t part = vt::split_part_bytes(cap), flags = vt::split_flag_bytes(cap);
      if (cudaMalloc(&sc->split_ptr, part + flags) != cudaSuccess) {
        sc->split_ptr = nullptr;
        return VT_ERR_CUDA;
      }
      if (cudaMemsetAsync(static_cast<char*>(sc->split_ptr) + part, 0, flags, c.stream) !=
          cudaSuccess)
        return VT_ERR_CUDA;
      sc->split_units = cap;
    }
    if (++sc->split_calls == 0) sc->split_calls = 1;  // 0 is the flags' initial value
    call.part = static_cast<float*>(sc->split_ptr);
    call.part_flag = reinterpret_cast<uint32_t*>(static_cast<char*>(sc->split_ptr) +
                                                 vt::split_part_bytes(sc->split_units));
    call.call_id = sc->split_calls;
    call.split_units_max = static_cast<int32_t>(sc->split_units);
  }
  const int slot = static_cast<int>(sc->calls++ & 1u);
  sc->last_slot = slot;
  return static_cast<vt_status>(
      vt::launch_fwd(call, hdr, reinterpret_cast<vt::WorkEntry*>(hdr + 1), slot));
}

// The text decoder's attention: validated arguments, the prepass (128-row entries) and the
// kernel, on the stream's scratch.
vt_status swa_impl(const void* q, const void* k, const void* v, void* out, const int32_t* cu,
                   int32_t n, int32_t T, int32_t Hq, int32_t Hkv, float scale, int32_t window,
                   cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VT_ERR_CUDA;
  DeviceInfo* di = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    vt_status st = device_info(dev, &di);
    if (st != VT_OK) return st;
    if (!di->swa_ready) {
      if (vt::prepare_attn_swa() != cudaSuccess) return VT_ERR_CUDA;
      di->swa_ready = true;
    }
  }
  CUtensorMap tq, tk, tv;
  vt_status st;
  if ((st = make_tensor_map(&tq, q, T, Hq, vt::kSwaHeadDim)) != VT_OK) return st;
  if ((st = make_tensor_map(&tk, k, T, Hkv, vt::kSwaHeadDim)) != VT_OK) return st;
  if ((st = make_tensor_map(&tv, v, T, Hkv, vt::kSwaHeadDim)) != VT_OK) return st;
  std::lock_guard<std::mutex> lock(g_mu);
  Scratch* sc = nullptr;
  st = scratch_for(dev, stream, vt::scratch_bytes_for(T, n, vt::kSwaBlockRows), &sc);
  if (st != VT_OK) return st;
  auto* hdr = static_cast<vt::WorkHeader*>(sc->ptr);
  auto* entries = reinterpret_cast<vt::WorkEntry*>(hdr + 1);
  const int slot = static_cast<int>(sc->calls++ & 1u);
  sc->last_slot = slot;
  if (vt::launch_schedule(cu, n, T, vt::kSwaBlockRows, slot, hdr, entries, stream) != cudaSuccess)
    return VT_ERR_CUDA;
  vt::SwaArgs a;
  a.out = out;
  a.hdr = hdr;
  a.entries = entries;
  a.dev_status = &hdr->status[slot];
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.window = window;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  const long long units = vt::max_work_entries(T, n, vt::kSwaBlockRows) * static_cast<long long>(Hq);
  const long long cap = di->num_sms;  // one CTA per SM
  const int grid = static_cast<int>(units < cap ? units : cap);
  return vt::launch_attn_swa(tq, tk, tv, a, grid, stream) == cudaSuccess ? VT_OK : VT_ERR_CUDA;
}

vt::FwdCall make_call(const void* q, const void* k, const void* v, void* out,
                      const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                      int32_t H, float scale, vt_dtype dtype, void* stream_ptr, int32_t stall) {
  vt::FwdCall c;
  c.q = q;
  c.k = k;
  c.v = v;
  c.out = out;
  c.cu_seqlens = cu_seqlens;
  c.num_segments = num_segments;
  c.total_tokens = total_tokens;
  c.H = H;
  c.scale = scale;
  c.dtype = dtype;
  c.stream = static_cast<cudaStream_t>(stream_ptr);
  c.stall_test_cycles = stall;
  return c;
}

}  // namespace

extern "C" {

vt_status vt_attn_fwd(const void* q, const void* k, const void* v, void* out,
                      const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                      int32_t H, int32_t D, float scale, vt_dtype dtype, void* stream_ptr) {
  vt::FwdCall c = make_call(q, k, v, out, cu_seqlens, num_segments, total_tokens, H, scale, dtype,
                            stream_ptr, 0);
  bool no_work = false;
  const vt_status st = static_cast<vt_status>(vt::check_fwd_args(c, D, &no_work));
  if (st != VT_OK || no_work) return st;
  return fwd_impl(c);
}

vt_status vt_attn_selftest_wait_timeout(const void* q, const void* k, const void* v, void* out,
                                        const int32_t* cu_seqlens, int32_t num_segments,
                                        int32_t total_tokens, int32_t H, int32_t D, float scale,
                                        int32_t stall_cycles, void* stream_ptr) {
  if (stall_cycles < 1) return VT_ERR_INVALID_ARG;
  if (num_segments < 1 || total_tokens < 1) return VT_ERR_INVALID_ARG;  // a kernel must run
  vt::FwdCall c = make_call(q, k, v, out, cu_seqlens, num_segments, total_tokens, H, scale,
                            VT_DTYPE_BF16, stream_ptr, stall_cycles);
  bool no_work = false;
  const vt_status st = static_cast<vt_status>(vt::check_fwd_args(c, D, &no_work));
  if (st != VT_OK || no_work) return st;
  return fwd_impl(c);
}

}  // extern "C"

namespace {

// Host-side description of the images for the window kernels; checks sizes and limits.
vt_status window_images(const int32_t* grids, int32_t n_images, int32_t win, vt::WindowImages* g) {
  if (!grids) return VT_ERR_NULL;
  if (n_images < 1 || win < 1) return VT_ERR_INVALID_ARG;
  if (n_images > vt::kMaxWindowImages) return VT_ERR_UNSUPPORTED;
  g->n = n_images;
  g->win = win;
  g->token_base[0] = 0;
  g->window_base[0] = 0;
  for (int32_t i = 0; i < n_images; ++i) {
    const int32_t h = grids[2 * i], w = grids[2 * i + 1];
    if (h < 1 || w < 1) return VT_ERR_INVALID_ARG;
    g->h[i] = h;
    g->w[i] = w;
    g->token_base[i + 1] = g->token_base[i] + static_cast<int64_t>(h) * w;
    g->window_base[i + 1] = g->window_base[i] + static_cast<int64_t>((h + win - 1) / win) *
                                                    ((w + win - 1) / win);
    if (g->token_base[i + 1] > INT32_MAX) return VT_ERR_INVALID_ARG;
  }
  return VT_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace

extern "C" {

vt_status vt_window_count(const int32_t* grids, int32_t n_images, int32_t win,
                          int32_t* num_windows, int32_t* total_tokens) {
  vt::WindowImages g;
  const vt_status st = window_images(grids, n_images, win, &g);
  if (st != VT_OK) return st;
  if (num_windows) *num_windows = static_cast<int32_t>(g.window_base[n_images]);
  if (total_tokens) *total_tokens = static_cast<int32_t>(g.token_base[n_images]);
  return VT_OK;
}

vt_status vt_window_partition(const int32_t* grids, int32_t n_images, int32_t win, int32_t* perm,
                              int32_t* cu_seqlens, void* stream) {
  vt::WindowImages g;
  const vt_status st = window_images(grids, n_images, win, &g);
  if (st != VT_OK) return st;
  if (!perm || !cu_seqlens) return VT_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(perm) | reinterpret_cast<uintptr_t>(cu_seqlens)) & 3u)
    return VT_ERR_INVALID_ARG;
  const int nsm = sm_count();
  if (nsm < 1) return VT_ERR_CUDA;
  return vt::launch_window_perm(g, perm, cu_seqlens, nsm, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? VT_OK
             : VT_ERR_CUDA;
}

vt_status vt_permute_rows(const void* src, void* dst, const int32_t* index, int32_t num_rows,
                          int32_t row_bytes, int32_t scatter, void* stream) {
  if (num_rows < 0 || row_bytes < 16 || (row_bytes & 15)) return VT_ERR_INVALID_ARG;
  if (scatter != 0 && scatter != 1) return VT_ERR_INVALID_ARG;
  if (num_rows == 0) return VT_OK;
  if (!src || !dst || !index) return VT_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u)
    return VT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(index) & 3u) return VT_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(num_rows) * row_bytes;
  if (ranges_overlap(src, bytes, dst, bytes)) return VT_ERR_INVALID_ARG;
  const int nsm = sm_count();
  if (nsm < 1) return VT_ERR_CUDA;
  return vt::launch_permute_rows(src, dst, index, num_rows, row_bytes, scatter, nsm,
                                 static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? VT_OK
             : VT_ERR_CUDA;
}

vt_status vt_attn_fwd_rope2d(const void* q, const void* k, const void* v, void* out,
                             const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                             int32_t H, int32_t D, float scale, const int32_t* pos, float theta,
                             void* k_rot, void* stream_ptr) {
  vt::FwdCall c = make_call(q, k_rot, v, out, cu_seqlens, num_segments, total_tokens, H, scale,
                            VT_DTYPE_BF16, stream_ptr, 0);
  bool no_work = false;
  vt_status st = static_cast<vt_status>(vt::check_fwd_args(c, D, &no_work));
  if (st != VT_OK || no_work) return st;
  if (!std::isfinite(theta) || !(theta > 0.0f)) return VT_ERR_INVALID_ARG;
  if (!k || !pos) return VT_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(k) & 15u) || (reinterpret_cast<uintptr_t>(pos) & 7u))
    return VT_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(total_tokens) * H * D * 2;
  const size_t pos_bytes = static_cast<size_t>(total_tokens) * 2 * sizeof(int32_t);
  if (k != k_rot && (ranges_overlap(k, bytes, k_rot, bytes) || ranges_overlap(k, bytes, out, bytes)))
    return VT_ERR_INVALID_ARG;
  if (ranges_overlap(k_rot, bytes, q, bytes) || ranges_overlap(k_rot, bytes, v, bytes))
    return VT_ERR_INVALID_ARG;
  if (ranges_overlap(pos, pos_bytes, out, bytes) || ranges_overlap(pos, pos_bytes, k_rot, bytes))
    return VT_ERR_INVALID_ARG;
  const int nsm = sm_count();
  if (nsm < 1) return VT_ERR_CUDA;
  // One HBM-bound pass rotates Q into `out` and K into k_rot; the attention then reads its
  // Q from `out` and writes O over it.  Each unit of the kernel reads its own Q rows once,
  // before any of its O rows are stored, and no other unit reads those rows: rows a Q tile
  // carries past its segment's end belong to another unit, and their results are dropped.
  const void* src[2] = {q, k};
  void* dst[2] = {out, k_rot};
  if (vt::launch_rope2d(src, dst, 2, pos, total_tokens, H, vt::rope_freqs(theta), nsm,
                        static_cast<cudaStream_t>(stream_ptr)) != cudaSuccess)
    return VT_ERR_CUDA;
  c.q = out;
  return fwd_impl(c);
}

vt_status vt_attn_fwd_swa(const void* q, const void* k, const void* v, void* out,
                          const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                          int32_t Hq, int32_t Hkv, int32_t D, float scale, int32_t window,
                          void* stream_ptr) {
  if (Hq < 1 || Hkv < 1 || D < 1 || num_segments < 0 || total_tokens < 0 || window < 0)
    return VT_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || !std::isfinite(scale)) return VT_ERR_INVALID_ARG;
  if (D != vt::kSwaHeadDim) return VT_ERR_UNSUPPORTED;
  if (num_segments == 0) return total_tokens == 0 ? VT_OK : VT_ERR_BAD_SEQLENS;
  if (!cu_seqlens) return VT_ERR_NULL;
  if (total_tokens == 0) return VT_OK;
  if (!q || !k || !v || !out) return VT_ERR_NULL;
  const uintptr_t align_or = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                             reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
  if (align_or & 15u) return VT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) return VT_ERR_INVALID_ARG;
  if (static_cast<int64_t>(Hq) * D > (1 << 20)) return VT_ERR_INVALID_ARG;
  const size_t qbytes = static_cast<size_t>(total_tokens) * Hq * D * 2;
  const size_t kvbytes = static_cast<size_t>(total_tokens) * Hkv * D * 2;
  if (ranges_overlap(out, qbytes, q, qbytes) || ranges_overlap(out, qbytes, k, kvbytes) ||
      ranges_overlap(out, qbytes, v, kvbytes))
    return VT_ERR_INVALID_ARG;
  return swa_impl(q, k, v, out, cu_seqlens, num_segments, total_tokens, Hq, Hkv, scale, window,
                  static_cast<cudaStream_t>(stream_ptr));
}

vt_status vt_rope2d(const void* x, void* out, const int32_t* pos, int32_t total_tokens, int32_t H,
                    int32_t D, float theta, void* stream) {
  if (H < 1 || D < 1 || total_tokens < 0) return VT_ERR_INVALID_ARG;
  if (!std::isfinite(theta) || !(theta > 0.0f)) return VT_ERR_INVALID_ARG;
  if (D != kHeadDim) return VT_ERR_UNSUPPORTED;
  if (total_tokens == 0) return VT_OK;
  if (!x || !out || !pos) return VT_ERR_NULL;
  if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15u) ||
      (reinterpret_cast<uintptr_t>(pos) & 7u))
    return VT_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(total_tokens) * H * D * 2;
  if (x != out && ranges_overlap(x, bytes, out, bytes)) return VT_ERR_INVALID_ARG;
  if (ranges_overlap(pos, static_cast<size_t>(total_tokens) * 2 * sizeof(int32_t), out, bytes))
    return VT_ERR_INVALID_ARG;
  const int nsm = sm_count();
  if (nsm < 1) return VT_ERR_CUDA;
  return vt::launch_rope2d(&x, &out, 1, pos, total_tokens, H, vt::rope_freqs(theta), nsm,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? VT_OK
             : VT_ERR_CUDA;
}

vt_status vt_permute_rows_check(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return VT_ERR_CUDA;
  int bad = 0;
  if (vt::permute_rows_check(&bad) != cudaSuccess) return VT_ERR_CUDA;
  return bad ? VT_ERR_BAD_INDEX : VT_OK;
}

vt_status vt_attn_last_device_status(void* stream_ptr) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VT_ERR_CUDA;
  const int32_t* word = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_scratch.find({dev, reinterpret_cast<uintptr_t>(stream)});
    if (it == g_scratch.end() || !it->second.ptr) return VT_OK;
    word = static_cast<const vt::WorkHeader*>(it->second.ptr)->status + it->second.last_slot;
  }
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VT_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return VT_ERR_CUDA;
  if (status & vt::kDevStatusBadSeqlens) return VT_ERR_BAD_SEQLENS;
  if (status & vt::kDevStatusTimeout) return VT_ERR_DEVICE_TIMEOUT;
  return VT_OK;
}

const char* vt_attn_status_string(vt_status s) {
  switch (s) {
    case VT_OK: return "VT_OK";
    case VT_ERR_NULL: return "VT_ERR_NULL: a required pointer is NULL";
    case VT_ERR_INVALID_ARG: return "VT_ERR_INVALID_ARG: invalid size, dtype, scale, alignment or aliasing";
    case VT_ERR_UNSUPPORTED: return "VT_ERR_UNSUPPORTED: head dim other than 96 is not implemented";
    case VT_ERR_BAD_SEQLENS: return "VT_ERR_BAD_SEQLENS: cu_seqlens must start at 0, not decrease and end at total_tokens";
    case VT_ERR_CUDA: return "VT_ERR_CUDA: a CUDA call failed";
    case VT_ERR_DEVICE_TIMEOUT: return "VT_ERR_DEVICE_TIMEOUT: a kernel pipeline wait gave up";
    case VT_ERR_BAD_INDEX: return "VT_ERR_BAD_INDEX: a row index outside [0, num_rows) was skipped";
  }
  return "unknown vt_status";
}

int32_t vt_attn_version(void) { return 100; }

int32_t vt_attn_set_split_keys(int32_t enable) {
  return g_split_keys.exchange(enable != 0 ? 1 : 0);
}

}  // extern "C"
