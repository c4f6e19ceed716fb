/*
 * vt_attn -- varlen block-diagonal attention forward for NVIDIA B200 (sm_100a).
 *
 * The operation (issue #1545 (vllm.cpp), "Why this one is bad" and "The fix";
 * PR #1579, "Numerics, both halves"): the non-causal scaled-dot-product
 * attention of a vision tower whose tokens are packed into independent
 * segments.  For every segment s = [cu[s], cu[s+1]), head h, query row i in s:
 *
 *     O[i,h,:] = sum_{j in s} softmax_j( scale * <Q[i,h,:], K[j,h,:]> ) V[j,h,:]
 *
 * i.e. softmax(Q_s K_s^T * scale) V_s per segment; tokens of different
 * segments never attend to each other (a block-diagonal mask given as row
 * slices).  In the perception encoder the pages describe, the segments are
 * the 32x32-patch windows of a window layer or the whole image of a full
 * layer; H = 16 heads of width D = 96.
 *
 * Layout of q, k, v and out: packed, contiguous, row-major [T, H, D]; element
 * (t, h, d) sits at index (t*H + h)*D + d.  All four have the same dtype.
 *
 * Ownership: the caller owns every buffer.  The library keeps, per
 * (device, stream), one small scratch buffer for its work list: it is
 * allocated on the first call on that stream and grown (never shrunk) when a
 * call needs more; make a first call on a stream before capturing it in a
 * CUDA graph.  A bf16 call with at most half as many (256-row block, head) units as
 * the device has SMs splits each unit's keys over two CTAs and combines the halves in
 * the kernel; its first such call on a stream also allocates, once, a workspace for
 * the halves (about 100 KB per SM).  Calls are stream-ordered; calls on different
 * streams use different scratch buffers.  The library keeps per-device state (launch
 * attributes, work lists, device addresses) for the life of the device's primary
 * context: a cudaDeviceReset invalidates it, so do not call the library again in a
 * process after resetting a device it has used.
 *
 * Errors: every entry point returns a status and never throws or aborts.
 * Argument errors are detected on the host before anything is launched.
 * cu_seqlens lives on the device, so its contents are validated on the device
 * (before any loop uses them); a malformed cu_seqlens makes the call write
 * nothing and is reported by vt_attn_last_device_status().
 */
#ifndef VT_ATTN_H_
#define VT_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VT_DTYPE_BF16 = 0, /* bfloat16 inputs/outputs, f32 accumulation (tensor cores) */
  VT_DTYPE_F32 = 1   /* float32 inputs/outputs, within 1e-5 of exact: tensor cores on
                        operands split into three bf16 parts, f32 softmax */
} vt_dtype;

typedef enum {
  VT_OK = 0,
  VT_ERR_NULL = 1,           /* a required pointer is NULL */
  VT_ERR_INVALID_ARG = 2,    /* bad size, dtype, scale, alignment or aliasing */
  VT_ERR_UNSUPPORTED = 3,    /* a valid request the library does not implement (D != 96) */
  VT_ERR_BAD_SEQLENS = 4,    /* cu_seqlens not 0 = cu[0] <= ... <= cu[n] = total_tokens */
  VT_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed */
  VT_ERR_DEVICE_TIMEOUT = 6, /* a kernel gave up waiting on its own pipeline (bug guard) */
  VT_ERR_BAD_INDEX = 7       /* vt_permute_rows met a row index outside [0, num_rows) */
} vt_status;

/*
 * Attention forward over packed variable-length segments.
 *
 *   q, k, v      device pointers, [total_tokens, H, D] of `dtype`, 16-byte aligned.
 *   out          device pointer, same shape and dtype; must not overlap q, k or v.
 *   cu_seqlens   device pointer to num_segments+1 int32 offsets:
 *                cu[0] = 0, non-decreasing, cu[num_segments] = total_tokens.
 *                Empty segments are allowed and produce no rows.
 *   num_segments >= 0; total_tokens >= 0 (both 0, or total_tokens 0: no work).
 *   H            heads, >= 1 (the encoder uses 16).
 *   D            head width; only 96 is implemented (VT_ERR_UNSUPPORTED otherwise).
 *   scale        any finite float (the encoder uses 1/sqrt(96)).
 *   stream       cudaStream_t as an opaque pointer (NULL = legacy default stream).
 *
 * Asynchronous: returns once the work is queued on `stream`.
 */
vt_status vt_attn_fwd(const void* q, const void* k, const void* v, void* out,
                      const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                      int32_t H, int32_t D, float scale, vt_dtype dtype, void* stream);

/*
 * vt_attn_fwd without any device allocation by the library.  (The source pages
 * have no counterpart to this entry point; it exists for callers, not for the
 * method.)
 *
 * For callers that cannot let a library allocate device memory: programs whose
 * device memory is owned entirely by their own allocator or pool, programs that
 * must not incur the device-wide synchronisation cudaMalloc/cudaFree may cause,
 * and programs that only allocate at start-up.  Arguments, layouts and results
 * are those of vt_attn_fwd; the work list lives in a fixed 1 MiB array in the
 * library's device memory (held on every GPU that loads the library until the
 * process exits) instead of a per-stream allocation.
 *
 * Limits and rules:
 *   - the work list must fit: 128 + 16 * floor((T + num_segments * (R - 1)) / R)
 *     <= 1 MiB, R = 256 for bf16, 128 for f32 (e.g. bf16 T = 16384 with 16 segments
 *     uses 1392 bytes); larger calls return VT_ERR_UNSUPPORTED and launch nothing;
 *   - the first call on a device looks up the array's device address for that
 *     device (make it with the device current, before capturing the stream into
 *     anything);
 *   - every call on a device shares the array, so calls that may overlap on the
 *     GPU (e.g. on two streams) race and must be serialised by the caller;
 *   - it never splits a unit's keys over two CTAs (its array has no room for that
 *     workspace), so on calls small enough for vt_attn_fwd to do so (at most half as
 *     many (256-row block, head) units as SMs) the two differ in rounding;
 *   - what the device side finds is not reported: vt_attn_last_device_status covers
 *     vt_attn_fwd's own work lists only.  A malformed cu_seqlens makes the call write
 *     nothing; a kernel wait that gives up (VT_ERR_DEVICE_TIMEOUT for vt_attn_fwd, a
 *     guard against a broken pipeline, never expected) leaves `out` partly written
 *     without a report.  Callers that need these checks use vt_attn_fwd.
 */
vt_status vt_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                              const int32_t* cu_seqlens, int32_t num_segments,
                              int32_t total_tokens, int32_t H, int32_t D, float scale,
                              vt_dtype dtype, void* stream);

/*
 * Pure host check of a host copy of cu_seqlens (num_segments+1 entries):
 * VT_OK, VT_ERR_NULL or VT_ERR_BAD_SEQLENS.  Touches no GPU.  The segments are the
 * block-diagonal mask as contiguous row slices (issue #1545 (vllm.cpp), "The fix"),
 * so they must tile [0, total_tokens): cu[0] = 0, non-decreasing, cu[n] =
 * total_tokens.  The check covers the whole array before any loop relies on it (PR
 * #279, vision-tower port commit: a coverage check placed after the slicing loop let
 * a bad input hang instead of fail).
 */
vt_status vt_attn_validate_seqlens_host(const int32_t* cu_seqlens_host, int32_t num_segments,
                                        int32_t total_tokens);

/*
 * Dynamic shared memory one CTA of the forward kernel for (D, dtype) uses, in
 * bytes; 0 for an unsupported combination.  Pure host arithmetic: the launch
 * shape contract, testable without a GPU (PR #1578 keeps the same kind of
 * host-side shared-memory contract next to its flash kernel).
 */
size_t vt_attn_smem_bytes(int32_t D, vt_dtype dtype);

/*
 * Bytes of scratch a call with these sizes needs (the work list).  Pure host.
 */
size_t vt_attn_workspace_bytes(int32_t num_segments, int32_t total_tokens, vt_dtype dtype);

/*
 * Synchronises `stream` and reports what the device side of the last
 * vt_attn_fwd call on it found: VT_OK, VT_ERR_BAD_SEQLENS or
 * VT_ERR_DEVICE_TIMEOUT (VT_ERR_CUDA if the synchronisation itself failed;
 * VT_OK if no call was made on this stream).
 */
vt_status vt_attn_last_device_status(void* stream);

/*
 * Failure-path self-test of the bf16 kernel's bounded waits.  Every wait in the
 * kernels is bounded.  In the vision-tower port commit of PR #279, a coverage
 * check placed after its loop let a bad input hang instead of fail; this call
 * exercises the bounded path on purpose, without a fault or a hang.
 *
 * Arguments are those of vt_attn_fwd for a valid bf16 problem (the same checks
 * apply; at least one token), plus stall_cycles >= 1.  The call launches the
 * bf16 forward, but in every CTA the MMA-issuing thread first waits on an
 * mbarrier that nothing arrives on.  After stall_cycles SM clock cycles the wait
 * gives up, raises the CTA's abort flag and records a timeout.  Every other role
 * then leaves its loop, the TMA copies already issued are drained, and TMEM is
 * released, as after a real stall.  No MMA is issued.
 *
 * Returns the launch status (VT_OK when launched).  A following
 * vt_attn_last_device_status(stream) returns VT_ERR_DEVICE_TIMEOUT.  `out` is
 * left unspecified.  The context stays usable, and the next vt_attn_fwd on the
 * stream resets the device status.  Ownership is as for vt_attn_fwd.
 */
vt_status vt_attn_selftest_wait_timeout(const void* q, const void* k, const void* v, void* out,
                                        const int32_t* cu_seqlens, int32_t num_segments,
                                        int32_t total_tokens, int32_t H, int32_t D, float scale,
                                        int32_t stall_cycles, void* stream);

/*
 * Window segmentation (the vision tower's window layers attend within 32 x 32-patch
 * windows of each image: issue #1545 (vllm.cpp), follow-up comment, the section on the
 * resolved labelled uncertainties).  The tower puts its hidden states in window order
 * once before its layers and back in image order once after them (PR #279,
 * vision-tower port commit).  The calls below build that order on the device and apply
 * it to [rows, ...] tensors.
 *
 * Order (the pages name the two orders without printing them; the plain row-major
 * reading):
 *   - images are packed one after another, each in row-major (y, x) patch order;
 *   - an image's win x win blocks are walked row-major over its block grid, with smaller
 *     blocks along the bottom and right edges when the grid is not a multiple of win;
 *   - the tokens of a block are taken row-major inside it.
 *
 * grids: host array of n_images (h, w) pairs, 1 <= n_images <= 64, h, w >= 1, win >= 1,
 * and the total token count must fit in int32 (else VT_ERR_INVALID_ARG /
 * VT_ERR_UNSUPPORTED for more than 64 images).
 *
 * vt_window_count (pure host): the number of blocks and of tokens; either output
 * pointer may be NULL.
 */
vt_status vt_window_count(const int32_t* grids, int32_t n_images, int32_t win,
                          int32_t* num_windows, int32_t* total_tokens);

/*
 * Writes, on `stream`, perm[p] (device, int32 [total_tokens]) = the packed image-order
 * token at position p of the window-ordered sequence, and cu_seqlens (device, int32
 * [num_windows + 1]) delimiting the blocks in that sequence (the cu_seqlens a window
 * layer passes to vt_attn_fwd).  Both buffers are the caller's, 4-byte aligned.
 */
vt_status vt_window_partition(const int32_t* grids, int32_t n_images, int32_t win,
                              int32_t* perm, int32_t* cu_seqlens, void* stream);

/*
 * Row permutation on `stream`: scatter == 0 gathers dst[i] = src[index[i]] (image order
 * to window order with index = perm); scatter == 1 scatters dst[index[i]] = src[i]
 * (back).  Rows are row_bytes long (a multiple of 16, e.g. H * D * 2 for bf16
 * [T, H, D]); src and dst are device pointers, 16-byte aligned, and must not overlap;
 * index holds num_rows distinct row numbers in [0, num_rows).  index lives on the
 * device, so its values are checked there: a row whose index lies outside
 * [0, num_rows) is skipped before any memory access (gather: dst row i keeps its
 * contents; scatter: nothing is written for it) and raises a per-device flag that
 * vt_permute_rows_check reports.
 */
vt_status vt_permute_rows(const void* src, void* dst, const int32_t* index, int32_t num_rows,
                          int32_t row_bytes, int32_t scatter, void* stream);

/*
 * Synchronises `stream`, then reports and clears the current device's out-of-range
 * flag of vt_permute_rows: VT_ERR_BAD_INDEX if any vt_permute_rows call on this device
 * since the previous check skipped a row (on any stream: the flag is one word per
 * device), else VT_OK; VT_ERR_CUDA if the synchronisation or the read failed.
 */
vt_status vt_permute_rows_check(void* stream);

/*
 * 2D rotary position embedding of the vision tower: out = rope(x) for a bf16
 * [total_tokens, H, D] tensor (PR #279, vision-tower port commit: the tower rotates Q and
 * K by a width-first 2D RoPE with 1-based positions, and the RoPE table travels with the
 * hidden states into window order).  The pages print no formula; the reading taken:
 *   pos        device int32 [total_tokens][2]: (pw, ph) = (x + 1, y + 1), the token's
 *              1-based column and row in its image's patch grid (in window order when the
 *              tokens are, e.g. gathered with vt_permute_rows);
 *   f_i        = theta^(-2 i / (D / 2)), i < D / 4 (computed on the host in double);
 *   angle a_d  = pw * f_d for d < D/4, ph * f_{d - D/4} for D/4 <= d < D/2 (width first);
 *   element d < D/2 pairs with d + D/2: (x_d, x_{d+D/2}) turns by a_d.
 * Arithmetic in f32 (sin/cos after reduction to [-pi, pi]); the result is rounded to bf16.
 *   x, out   device pointers, 16-byte aligned; out == x rotates in place, otherwise the
 *            two must not overlap; pos must not overlap out.
 *   D        only 96 (VT_ERR_UNSUPPORTED otherwise); H >= 1; theta finite and > 0 (the
 *            tower's base: 10000).
 * Asynchronous on `stream`; total_tokens == 0 is a no-op.
 */
vt_status vt_rope2d(const void* x, void* out, const int32_t* pos, int32_t total_tokens, int32_t H,
                    int32_t D, float theta, void* stream);

/*
 * Attention with the vision tower's 2D RoPE applied to Q and K first:
 *     O = attention(rope(Q), rope(K), V)   per segment, as vt_attn_fwd,
 * with rope() exactly as vt_rope2d defines it (bf16 only; D = 96).
 *   pos     device int32 [total_tokens][2], the tokens' 1-based (pw, ph) (in the same
 *           order as q, k, v: window order for a window layer).
 *   theta   RoPE base, finite and > 0 (the tower's: 10000).
 *   k_rot   caller-owned device buffer [total_tokens, H, D] bf16, 16-byte aligned, that
 *           receives rope(K) (the attention reads K from it); k_rot == k rotates K in
 *           place.  It must not overlap q, v or out.
 *   out     as for vt_attn_fwd; it also holds rope(Q) between the two steps below, so on
 *           an error reported by the device its contents are undefined.  pos must not
 *           overlap out or k_rot.
 * Two launches on `stream`: one HBM-bound pass (vt_rope2d's arithmetic) rotates Q into out
 * and K into k_rot; the attention kernel then reads Q from out and writes O over it (each
 * unit of the kernel reads its own Q rows before it stores those rows of O, and no other
 * unit needs them).  With at most 32 segments the attention kernel follows the pass
 * directly and, launched with programmatic stream serialization, sets itself up while the
 * pass ends.  Errors and asynchrony as for vt_attn_fwd.
 */
vt_status vt_attn_fwd_rope2d(const void* q, const void* k, const void* v, void* out,
                             const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                             int32_t H, int32_t D, float scale, const int32_t* pos, float theta,
                             void* k_rot, void* stream);

/*
 * The text decoder's attention (the Muse Glimmer next-steps document, "Architecture / Text
 * decoder": 32 query heads over 2 key/value heads, head size 128, a local window of 2048
 * tokens on the sliding layers): causal attention with an optional local window and
 * grouped-query heads, over packed segments.  For query token i of segment s and query
 * head h:
 *     O[i,h,:] = sum_j softmax_j(scale * <Q[i,h,:], K[j,g,:]>) V[j,g,:],
 *     j over the tokens of s with j <= i, and j > i - window when window > 0,
 *     g = h / (Hq / Hkv).
 *   q, out        device pointers, bf16 [total_tokens, Hq, D] row-major, 16-byte aligned.
 *   k, v          device pointers, bf16 [total_tokens, Hkv, D] row-major, 16-byte aligned.
 *   cu_seqlens    device pointer, int32 [num_segments + 1], validated on the device as for
 *                 vt_attn_fwd (a malformed one is reported by vt_attn_last_device_status).
 *   Hq, Hkv       Hq a multiple of Hkv (Hq == Hkv: ordinary multi-head attention).
 *   D             only 128 (VT_ERR_UNSUPPORTED otherwise).
 *   scale         any finite float (the decoder folds its query multiplier into it).
 *   window        >= 0; 0 means no window (a full-attention layer).
 * out must not overlap q, k or v.  bf16 in and out, f32 accumulation.  Asynchronous on
 * `stream`; the library's per-stream scratch is shared with vt_attn_fwd.  Returns as
 * vt_attn_fwd.
 */
vt_status vt_attn_fwd_swa(const void* q, const void* k, const void* v, void* out,
                          const int32_t* cu_seqlens, int32_t num_segments, int32_t total_tokens,
                          int32_t Hq, int32_t Hkv, int32_t D, float scale, int32_t window,
                          void* stream);

/*
 * Whether bf16 calls of vt_attn_fwd and vt_attn_fwd_rope2d may split a unit's keys over
 * two CTAs (enable != 0, the default) or never do (enable == 0).  A call with at most half
 * as many (256-row block, head) units as SMs normally sums each row of a segment of at
 * least four 128-key tiles in two halves, so its rows can differ in rounding from the
 * same segment inside a larger call (both within the bf16 bound against the definition).
 * With splitting off, a segment's output is the same bits whatever else the call packs,
 * at the cost of speed on small calls.  Process-wide; takes effect for calls queued after
 * it returns.  Returns the previous setting (1 or 0).
 */
int32_t vt_attn_set_split_keys(int32_t enable);

/* Static, human-readable name of a status code. */
const char* vt_attn_status_string(vt_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t vt_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VT_ATTN_H_ */
