// vt_attn_fwd_noalloc: the attention forward for callers that cannot allocate
// device memory.
//
// vt_attn_fwd keeps its work list in a buffer it allocates itself (once per
// stream, grown on demand).  Some callers cannot allow that: programs whose
// device memory is entirely owned by their own allocator or memory pool, programs
// that must not add the device-wide synchronisation cudaMalloc/cudaFree can
// cause, and programs that only allocate during start-up.  This entry point
// allocates nothing.  Its work list lives in a fixed array in the library's own
// device memory (kNoAllocScratchBytes, reserved on every GPU that loads the
// library until the process exits); the caller still provides q, k, v, out and
// cu_seqlens.
//
// The array's device address is looked up once per device, on the first call
// made with that device current; make that first call before capturing the
// stream into anything.  All calls share the one array: calls that overlap on the
// GPU (for example on two streams at once) race on it and must be serialised by
// the caller.  Each call rewrites what it reads (the scheduling prepass writes the
// header and every entry before the attention kernel reads them).
#include <cmath>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "vt_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB: header + 65528 entries
constexpr int kMaxDevicesNoAlloc = 64;
constexpr int kHeadDimNoAlloc = 96;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static_assert(sizeof(vt::WorkHeader) % 8 == 0, "entries follow the header");

struct NoAllocDevice {
  bool ready = false;
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int num_sms = 0;
  bool bf16_ready = false;
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kMaxDevicesNoAlloc];

using EncodeTiledFnNA = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnNA encode_fn_noalloc() {
  static EncodeTiledFnNA fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnNA>(p);
  });
  return fn;
}

// Same view of [T, H, 96] bf16 as the allocating entry point uses.
vt_status tensor_map_noalloc(CUtensorMap* map, const void* base, int32_t T, int32_t H) {
  EncodeTiledFnNA fn = encode_fn_noalloc();
  if (!fn) return VT_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDimNoAlloc), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDimNoAlloc) * 2,
                                 static_cast<cuuint64_t>(H) * kHeadDimNoAlloc * 2};
  const cuuint32_t box[3] = {32, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VT_OK : VT_ERR_CUDA;
}

// Per-device set-up on the first call: the array's device address and the SM count.
vt_status noalloc_device(int dev, NoAllocDevice** out) {
  if (dev < 0 || dev >= kMaxDevicesNoAlloc) return VT_ERR_CUDA;
  NoAllocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return VT_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return VT_ERR_CUDA;
    d.scratch = ptr;
    d.ready = true;
  }
  *out = &d;
  return VT_OK;
}

bool overlap_noalloc(const void* a, const void* b, size_t n) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + n && y < x + n;
}

}  // namespace

extern "C" vt_status vt_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                         const int32_t* cu_seqlens, int32_t num_segments,
                                         int32_t total_tokens, int32_t H, int32_t D, float scale,
                                         vt_dtype dtype, void* stream_ptr) {
  if (dtype != VT_DTYPE_BF16 && dtype != VT_DTYPE_F32) return VT_ERR_INVALID_ARG;
  if (H < 1 || D < 1 || num_segments < 0 || total_tokens < 0) return VT_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return VT_ERR_INVALID_ARG;
  if (D != kHeadDimNoAlloc) return VT_ERR_UNSUPPORTED;
  if (num_segments == 0) return total_tokens == 0 ? VT_OK : VT_ERR_BAD_SEQLENS;
  if (!cu_seqlens) return VT_ERR_NULL;
  if (total_tokens == 0) return VT_OK;
  if (!q || !k || !v || !out) return VT_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out)) & 15u)
    return VT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) return VT_ERR_INVALID_ARG;
  if (static_cast<int64_t>(H) * D > (1 << 20)) return VT_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(total_tokens) * H * D * (dtype == VT_DTYPE_BF16 ? 2 : 4);
  if (overlap_noalloc(out, q, bytes) || overlap_noalloc(out, k, bytes) ||
      overlap_noalloc(out, v, bytes))
    return VT_ERR_INVALID_ARG;

  // The work list must fit the fixed array: header + (ceil(T / rows) + n) entries.
  const int block_rows = dtype == VT_DTYPE_BF16 ? vt::kBf16BlockRows : vt::kF32BlockRows;
  if (vt::scratch_bytes_for(total_tokens, num_segments, block_rows) > kNoAllocScratchBytes)
    return VT_ERR_UNSUPPORTED;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VT_ERR_CUDA;
  NoAllocDevice* nd = nullptr;
  vt_status st = noalloc_device(dev, &nd);
  if (st != VT_OK) return st;

  auto* hdr = static_cast<vt::WorkHeader*>(nd->scratch);
  auto* entries = reinterpret_cast<vt::WorkEntry*>(hdr + 1);
  if (vt::launch_schedule(cu_seqlens, num_segments, total_tokens, block_rows, hdr, entries,
                          stream) != cudaSuccess)
    return VT_ERR_CUDA;

  const long long max_units =
      static_cast<long long>(vt::max_work_entries(total_tokens, num_segments, block_rows)) * H;
  if (dtype == VT_DTYPE_BF16) {
    if (!nd->bf16_ready) {
      if (vt::prepare_attn_bf16() != cudaSuccess) return VT_ERR_CUDA;
      nd->bf16_ready = true;
    }
    CUtensorMap tq, tk, tv;
    if ((st = tensor_map_noalloc(&tq, q, total_tokens, H)) != VT_OK) return st;
    if ((st = tensor_map_noalloc(&tk, k, total_tokens, H)) != VT_OK) return st;
    if ((st = tensor_map_noalloc(&tv, v, total_tokens, H)) != VT_OK) return st;
    vt::Bf16Args a;
    a.out = out;
    a.cu_seqlens = cu_seqlens;
    a.hdr = hdr;
    a.entries = entries;
    a.dev_status = &hdr->status;
    a.H = H;
    a.out_align32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    a.scale_log2 = static_cast<float>(std::fabs(static_cast<double>(scale)) * 1.4426950408889634);
    a.idesc_qk = vt::make_idesc_bf16(128, 128, false, false, scale < 0.0f);
    const int grid = static_cast<int>(max_units < nd->num_sms ? max_units : nd->num_sms);
    if (vt::launch_attn_bf16(tq, tk, tv, a, grid, stream) != cudaSuccess) return VT_ERR_CUDA;
  } else {
    vt::F32Args a;
    a.q = static_cast<const float*>(q);
    a.k = static_cast<const float*>(k);
    a.v = static_cast<const float*>(v);
    a.out = static_cast<float*>(out);
    a.cu_seqlens = cu_seqlens;
    a.hdr = hdr;
    a.entries = entries;
    a.H = H;
    a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    const long long cap = static_cast<long long>(nd->num_sms) * 16;
    const int grid = static_cast<int>(max_units < cap ? max_units : cap);
    if (vt::launch_attn_f32(a, grid, stream) != cudaSuccess) return VT_ERR_CUDA;
  }
  return VT_OK;
}
