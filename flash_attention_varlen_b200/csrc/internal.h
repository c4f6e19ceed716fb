// Internal interfaces between the C-ABI layer (vt_attn.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace vt {

// Head of the per-stream scratch buffer.
struct alignas(128) WorkHeader {
  // kDevStatus* bit flags, one word per call parity: the call with slot k reports what
  // its device side finds in status[k] and clears status[k ^ 1], the word of the next
  // call on the same scratch, before that call can start
  int32_t status[2];
  int32_t num_entries;  // E: number of (segment, q-block) entries that follow (prepass)
  // Unit order of the bf16 kernel, set by the prepass: 0 = head-major (unit u = head u / E,
  // entry u % E), for segments of one length: the CTAs in flight share few heads' K/V in
  // L2; 1 = entry-major (entry u / H, head u % H), for segments of unequal length: the
  // units come longest first, which the snake assignment needs to balance the CTAs
  int32_t order;
  int32_t pad[28];
};
static_assert(sizeof(WorkHeader) == 128, "header size");

// A work entry: one block of `block_rows` query rows of one segment, stored
// decoded (the segment's bounds included) so a kernel reads it with a single
// 16-byte load it can issue a whole unit ahead.  The kernels expand entry e and
// head h into unit u = h * E + e.
struct alignas(16) WorkEntry {
  int32_t seg;
  int32_t qblock;
  int32_t seg_start;  // cu_seqlens[seg]
  int32_t seg_end;    // cu_seqlens[seg + 1]
};

// Entries that a call can produce at most: each ceil(L_s / R) <= (L_s + R - 1) / R, so the
// sum is at most floor((T + n (R - 1)) / R) (exact for one segment).
inline int64_t max_work_entries(int64_t total_tokens, int64_t num_segments, int block_rows) {
  return (total_tokens + num_segments * (block_rows - 1)) / block_rows;
}

inline size_t scratch_bytes_for(int64_t total_tokens, int64_t num_segments, int block_rows) {
  return sizeof(WorkHeader) +
         static_cast<size_t>(max_work_entries(total_tokens, num_segments, block_rows)) *
             sizeof(WorkEntry);
}

// Scheduling prepass (one CTA): validates cu_seqlens, orders segments by
// length (longest first) and writes the entry list.  Sets status[slot] to 0, or to
// kDevStatusBadSeqlens with num_entries 0 on a malformed cu_seqlens, and clears
// status[slot ^ 1].
cudaError_t launch_schedule(const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                            int32_t block_rows, int slot, WorkHeader* hdr, WorkEntry* entries,
                            cudaStream_t stream);

// The bf16 kernel builds the work list of a call with at most this many segments itself,
// in shared memory (same validation and order as the prepass), and no prepass runs.
constexpr int kInlineSegments = 32;

// 2D RoPE frequencies f_i = theta^(-2 i / (D / 2)), i < D / 4, for D = 96 (host-computed).
struct RopeFreqs {
  float f[24];
};
RopeFreqs rope_freqs(double theta);
// out[i] = rope(x[i]) for count (1 or 2) bf16 [T, H, 96] tensors in one launch (out[i] may
// equal x[i]); pos: int32 [T][2] 1-based (pw, ph), shared by the tensors.  The kernel lets
// a dependent launch (programmatic stream serialization) start early.
constexpr int kRopeMaxTensors = 2;
cudaError_t launch_rope2d(const void* const* x, void* const* out, int count, const int32_t* pos,
                          int32_t T, int32_t H, const RopeFreqs& f, int num_sms,
                          cudaStream_t stream);

// bf16 forward on tcgen05 tensor cores (sm_100a).
constexpr int kBf16BlockRows = 256;  // two 128-row Q tiles per unit
struct Bf16Args {
  void* out;
  const int32_t* cu_seqlens;
  const WorkHeader* hdr;
  const WorkEntry* entries;
  int* dev_status;   // this call's status word
  int* next_status;  // the next call's status word (cleared by this call when inline)
  int32_t num_segments, total_tokens;
  int32_t inline_sched;  // 1: no prepass ran; the kernel builds the work list itself
  int32_t H;
  int32_t out_align32;  // out is 32-byte aligned: rows go out as 256-bit stores
  float scale_log2;    // |scale| * log2(e)
  uint32_t idesc_qk;   // carries the sign of scale (negated A) for scale < 0
  // > 0 only in the failure-path self-test: the MMA thread first waits this many cycles
  // on a barrier that never completes (see vt_attn_selftest_wait_timeout)
  int32_t stall_test_cycles = 0;
  // split-key epilogue only: the halves' tiles (kPartF4 float4 columns of 128 rows each;
  // tile t's halves at 2 t and 2 t + 1), one flag per 32-row warp slice of a tile, and
  // this call's id (never 0)
  float* part = nullptr;
  uint32_t* part_flag = nullptr;
  uint32_t call_id = 0;
  int32_t split_units_max = 0;  // the kernel splits when the call's units are at most this
};
// The kernel's epilogue modes (one instantiation each): per-thread row stores; whole tiles
// staged in the Q buffers and stored by TMA; split-key units combined in the epilogue.
constexpr int kEpiRows = 0, kEpiStaged = 1, kEpiSplit = 2;
// Split-key units: segments of at least this many 128-key tiles are split (measured: with
// one key tile per half the combine, ~4 us, costs more than the half it saves).
constexpr int kSplitMinKeyTiles = 4;
// A split-key row: 96 unnormalised O values, then (m, l, 0, 0): 25 float4.
constexpr int kPartF4 = 25;
// Workspace of the split-key epilogue for up to `units` (entry, head) units: the rows'
// halves, then the flags (zeroed once when allocated; a flag holds the id of the last call
// that wrote it, so it needs no reset between calls).
// A unit has two 128-row tiles; tile (unit u, tile i) is 2 u + i, with two halves of
// kPartF4 * 128 float4 each and four flags (one per warp of 32 rows).
inline size_t split_part_bytes(long long units) {
  return static_cast<size_t>(units) * 2 * 2 * kPartF4 * 128 * 16;
}
inline size_t split_flag_bytes(long long units) {
  return static_cast<size_t>(units) * 2 * 4 * sizeof(uint32_t);
}
size_t bf16_smem_bytes();
cudaError_t prepare_attn_bf16();  // opt in to the kernel's dynamic shared memory (per device)
// `to` maps the output like tq maps Q (same shape, box and swizzle).  With stage_o, whole
// 128-row O tiles are staged in the unit's Q buffer and leave by TMA stores through it
// (worth it when a CTA runs several short units: the stores overlap the next unit);
// otherwise every row is stored by its thread.
cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const Bf16Args& args, int grid, int epilogue,
                             cudaStream_t stream);
// The staged epilogue is chosen for calls whose segments average at most this many tokens
// and that give each SM at least kStageMinUnitsPerSm units of 256 rows on average.
constexpr int kStageMaxMeanSegment = 2048;
constexpr int kStageMinUnitsPerSm = 3;

// f32 forward on tcgen05 tensor cores: each operand split into three bf16 parts
// (exactness arm).
constexpr int kF32BlockRows = 128;
struct F32Args {
  const float* q;
  const float* k;
  const float* v;
  float* out;
  const WorkHeader* hdr;
  const WorkEntry* entries;
  int* dev_status;
  int32_t H, T;
  float scale_log2;  // scale * log2(e), signed
};
size_t f32_smem_bytes();
cudaError_t prepare_attn_f32();  // opt in to the kernel's dynamic shared memory (per device)
cudaError_t launch_attn_f32(const F32Args& args, int grid, cudaStream_t stream);

// Text decoder attention: causal, a local window (0: none), grouped-query heads; bf16,
// head size 128.  Units are 256 query rows (two Q tiles) of one (segment, query head).
constexpr int kSwaBlockRows = 256;
constexpr int kSwaHeadDim = 128;
struct SwaArgs {
  void* out;
  const WorkHeader* hdr;
  const WorkEntry* entries;
  int* dev_status;
  int32_t Hq, Hkv, window;
  float scale_log2;  // scale * log2(e), signed
};
size_t swa_smem_bytes();
cudaError_t prepare_attn_swa();  // opt in to the kernel's dynamic shared memory (per device)
cudaError_t launch_attn_swa(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const SwaArgs& args, int grid, cudaStream_t stream);

// ---------------------------------------------------------------- host launcher
// One forward call as the entry points receive it (validated by check_fwd_args).
struct FwdCall {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  const int32_t* cu_seqlens;
  int32_t num_segments, total_tokens, H;
  float scale;
  int dtype;  // vt_dtype
  cudaStream_t stream;
  int32_t stall_test_cycles;  // > 0 only for the bf16 failure-path self-test
  // bf16 only: a workspace for split-key units (split_part_bytes / split_flag_bytes of
  // max_work_entries(...) * H units) and this call's id; null: no split-key units
  float* part = nullptr;
  uint32_t* part_flag = nullptr;
  uint32_t call_id = 0;
  int32_t split_units_max = 0;
};

// Host-side argument checks shared by every forward entry point; touches no device.
// Returns 0 (VT_OK) or a vt_status code.  *no_work is set when the call is valid but
// has nothing to compute (no segments, or no tokens).
int check_fwd_args(const FwdCall& c, int32_t D, bool* no_work);

// Query rows per work entry for a dtype (the kernel's unit of rows).
int block_rows_for_dtype(int dtype);

// Queues the scheduling prepass and the attention kernel of a validated call on
// c.stream, with the work list at (hdr, entries) in device memory that holds at
// least scratch_bytes_for(T, n, block_rows_for_dtype(dtype)) bytes.  The caller owns
// that memory and orders its reuse.  Returns 0 or a vt_status code.
// `slot` (0 or 1) is the call's status word in hdr; successive calls on one scratch
// alternate it.
int launch_fwd(const FwdCall& c, WorkHeader* hdr, WorkEntry* entries, int slot);

// Window segmentation (window.cu).  Images are passed by value: at most kMaxWindowImages.
constexpr int kMaxWindowImages = 64;
struct WindowImages {
  int32_t n, win;
  int32_t h[kMaxWindowImages], w[kMaxWindowImages];
  int64_t token_base[kMaxWindowImages + 1];   // packed image-order offset of each image
  int64_t window_base[kMaxWindowImages + 1];  // index of each image's first block
};
cudaError_t launch_window_perm(const WindowImages& g, int32_t* perm, int32_t* cu, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* idx, int32_t rows,
                                int32_t row_bytes, int32_t scatter, int num_sms,
                                cudaStream_t stream);
// Reads, then clears, the device's out-of-range-index flag of launch_permute_rows
// (synchronous; the current device).  *bad = 1 if some permute met such an index.
cudaError_t permute_rows_check(int* bad);

}  // namespace vt
