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
#include <mutex>

#include "internal.h"
#include "vt_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB: header + 65528 entries
constexpr int kMaxDevicesNoAlloc = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static_assert(sizeof(vt::WorkHeader) % 8 == 0, "entries follow the header");

struct NoAllocDevice {
  bool ready = false;
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kMaxDevicesNoAlloc];
uint32_t g_noalloc_calls[kMaxDevicesNoAlloc];  // calls per device: their status slots alternate

// Per-device set-up on the first call made with that device current: the device address
// of the array.  In host code the name g_noalloc_scratch is only a host-side stand-in, so
// the kernels are given this address, never the name.  The address stays valid for the
// life of the device's context: a cudaDeviceReset (or anything else that destroys the
// primary context) invalidates it, together with the rest of the library's per-device
// state.
vt_status noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevicesNoAlloc) return VT_ERR_CUDA;
  NoAllocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return VT_ERR_CUDA;
    d.scratch = ptr;
    d.ready = true;
  }
  *out = d.scratch;
  return VT_OK;
}

}  // namespace

extern "C" vt_status vt_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                         const int32_t* cu_seqlens, int32_t num_segments,
                                         int32_t total_tokens, int32_t H, int32_t D, float scale,
                                         vt_dtype dtype, void* stream_ptr) {
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
  c.stall_test_cycles = 0;
  bool no_work = false;
  vt_status st = static_cast<vt_status>(vt::check_fwd_args(c, D, &no_work));
  if (st != VT_OK || no_work) return st;

  // The work list must fit the fixed array: header + (ceil(T / rows) + n) entries.
  if (vt::scratch_bytes_for(total_tokens, num_segments, vt::block_rows_for_dtype(dtype)) >
      kNoAllocScratchBytes)
    return VT_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VT_ERR_CUDA;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != VT_OK) return st;
  auto* hdr = static_cast<vt::WorkHeader*>(scratch);
  const int slot = static_cast<int>(g_noalloc_calls[dev]++ & 1u);  // status slots alternate
  return static_cast<vt_status>(
      vt::launch_fwd(c, hdr, reinterpret_cast<vt::WorkEntry*>(hdr + 1), slot));
}
