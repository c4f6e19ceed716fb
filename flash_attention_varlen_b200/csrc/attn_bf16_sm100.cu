// bf16 varlen attention forward for B200 (sm_100a): TMA + tcgen05 + TMEM.
//
// Method: softmax(Q_s K_s^T * scale) V_s per packed segment s (issue #1545
// (vllm.cpp), "The fix": the block-diagonal mask is a set of per-segment row
// slices), computed flash-style with a running softmax (PR #1579, "Numerics,
// both halves"): scores are produced one 128-key tile at a time and never
// leave the SM.
//
// One CTA (persistent, one per SM) works through units of 256 query rows of
// one (segment, head): two 128-row Q tiles that share every K/V tile.
//
//   warps 8-11         : warp 8 loads K/V, warp 9 issues MMAs, warp 10 loads Q, warp 11
//                        stores finished O tiles (staged-epilogue instantiation only)
//   warp 8  (K/V loader): TMA loads of K/V tiles into a 2-stage ring (64-byte
//                        swizzled, 32-column chunks).
//   warp 10 (Q loader) : TMA loads of Q0/Q1 into a double buffer, so the next
//                        unit's Q arrives while the current unit still runs.
//   warp 9  (MMA)      : one thread issues tcgen05.mma:
//                          S_i = Q_i K_j^T     (SS, M128 N128 K96)  -> TMEM
//                          O_i += P_i [V_j | 1] (TS, M128 N112 K128; P read from TMEM)
//                        in the order S0 S1 | PV0 S0' | PV1 S1' | ... so that the
//                        tensor core works on one tile while the other is in softmax;
//                        one flat stream over all units of the CTA, so a tile's first
//                        S of the next unit follows its own last PV of this one.
//   warps 0-3, 4-7     : softmax warpgroups for Q0 and Q1, one thread per row:
//                        tcgen05.ld of the S row, row max (three-input max tree),
//                        p = 2^(s*c - m) (packed f32x2 FMA, then MUFU ex2 for two
//                        thirds of the pairs and a polynomial on the FMA pipe for
//                        the rest) with a deferred rescale (the running max m only
//                        moves when the new tile max exceeds it by more than a
//                        threshold, so O in TMEM is rarely touched), P packed to
//                        bf16 and written back over S in TMEM, then the epilogue
//                        O / l -> bf16, stored row by row by each thread; or, in the
//                        staged instantiation (calls of many short units), a whole
//                        128-row tile is staged in the unit's Q buffer (its QKs are
//                        done) and warp 11 sends it out with TMA stores, while the
//                        rows of a tile cut by its segment's end still go row by row.
//                        In the split-key instantiation (calls of at most half as
//                        many units as SMs) a unit may take half of its segment's key
//                        tiles; its rows are combined with the other half's through
//                        a workspace in global memory (see the epilogue).
//
// CTAs take their units in a longest-first snake order (see UnitStream).
//
// The row sum l is not accumulated by the softmax threads: each V stage carries
// a fourth 32-column chunk whose first column is all ones, so column 96 of O
// accumulates sum_j P_ij on the tensor core -- exactly the bf16-rounded weights
// the PV product used -- and is rescaled together with O.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,368), O1 [384,496)
// (O column 96 = l); P_i overlays the first 64 columns of S_i (two bf16 per
// 32-bit column).
//
// Keys past the end of a segment inside its last tile are masked (p = 0);
// query rows past the end are computed but not stored.  Every mbarrier wait is
// bounded and an abort flag lets all roles leave together.
#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

constexpr int kBM = 128;          // query rows per Q tile
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kD = 96;            // head width
constexpr int kKStages = 2;  // K ring depth
constexpr int kVStages = 2;  // V ring depth
constexpr int kQBufs = 2;    // Q is double-buffered: the next unit's Q lands during this one
constexpr int kDv = kD + 16;               // PV N: 96 value columns + ones column (+15 zero)
constexpr int kTileBytes = kBM * kD * 2;   // 24576: a 128-row Q or K tile
constexpr int kChunkBytes = 128 * 64;      // 8192: 128 rows x 32 bf16
constexpr int kVTileBytes = 4 * kChunkBytes;  // V tile + the ones chunk
constexpr int kThreads = 384;               // three warpgroups
// Registers: launched at 168 per thread (65536 / 384, rounded down to 8); the two
// softmax warpgroups raise theirs to 192 and the loader/MMA warpgroup drops to 120:
// 2*128*192 + 128*120 = 64512 = 384*168, so the increase always finds its registers.
constexpr uint32_t kRegsSoftmax = 192, kRegsOther = 120;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * 168, "register split");
constexpr int kWarpLoad = 8;       // K/V loader
constexpr int kWarpMma = 9;
constexpr int kWarpLoadQ = 10;     // Q loader (runs up to one unit ahead)
constexpr int kWarpStore = 11;     // TMA stores of the O tiles staged in the Q buffers
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
// The running max only moves when a tile's max exceeds it by more than this (log2
// units), so P stays below 2^3 between rescales.  Larger values save O rescales but
// let the dominant key's p be rounded to bf16 more often (its error does not cancel
// for a peaked softmax); 3 keeps a peaked (Q x 4) 1024-token row inside 1e-2 while
// random N(0,1) rows almost never rescale.
constexpr float kRescaleThreshold = 3.0f;
// Every kPolyEvery-th pair of scores of a 64-key half (10 of 32 pairs for 3) takes
// its exp2 on the FMA pipe (degree-3 minimax polynomial after Cody-Waite range
// reduction, relative error 7.5e-5, far below the bf16 rounding of P) instead of the
// MUFU, which is otherwise the busiest unit: one exp2 per 384 tensor FLOPs at head
// width 96, and the MUFU issues 16 per clock per SM.  0 disables.
constexpr int kPolyEvery = 3;
// P is handed to the PV product in two key halves: the product of the first 64 keys
// runs while the softmax still exponentiates the other 64.
constexpr int kPChunks = 2;

static_assert(kBf16BlockRows == 2 * kBM, "a unit is two Q tiles");
// waits of the MMA thread
__device__ __forceinline__ bool mma_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int* dev_status) {
  return mbar_wait_bounded(bar, parity, abort_flag, dev_status);
}

// The work list of a call with at most kInlineSegments segments, built in shared memory
// by the kernel itself (no prepass): its segments longest first, each as
// (segment, 0, start, end), and the prefix sums of their entry counts.
struct SchedTable {
  int4 seg[kInlineSegments];
  int32_t prefix[kInlineSegments + 1];
  int32_t n, E, order, bad;
};

struct Smem {
  uint8_t q[kQBufs][2][kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kVTileBytes];
  uint64_t q_full[kQBufs][2];
  uint64_t q_empty[kQBufs];
  uint64_t q_free[kQBufs];  // the O tiles staged in this Q buffer have been read out
  // tile i's 128 O rows are staged in Q buffer b.  One barrier per buffer: staging into b
  // again needs the Q of the unit two on, which is loaded only after b's stores were read,
  // so a barrier never runs a phase ahead of the store warp's wait.
  uint64_t o_staged[kQBufs][2];
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t s_full[2];
  uint64_t p_full[2][kPChunks];  // [Q tile][key chunk]: that chunk's P columns written
  uint64_t o_done[2];
  uint64_t drain;
  uint64_t never;  // nothing arrives on it: the failure-path self-test waits here
  uint32_t tmem_base;
  int abort_flag;
  SchedTable sched;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

struct Unit {
  int head, q0, seg_start, seg_end;
  int kv0, nkv;  // key tiles [kv0, kv0 + nkv) of the segment
  bool has_q1;
  int parts, split;  // split-key units: the unit's share (split of parts) of the key tiles
  uint32_t slot;     // split-key units: (entry, head) index, for the partial results
};

// Walks this CTA's units (one per 256 query rows of one segment and head).  The units are
// dealt to the CTAs in a snake: in round k, CTA c takes unit k G + c when k is even and
// k G + G - 1 - c when k is odd (G CTAs).  Their order comes from the prepass:
//  * segments of one length (a full layer; the windows of a window layer): head-major,
//    unit u = entry u % E of head u / E, so the CTAs in flight share the K/V of a few
//    heads in L2 (all heads at once would re-read K/V from HBM several times over);
//  * segments of unequal length (a batch of images): entry-major, unit u = entry u / H
//    of head u % H, so the units come longest segment first.  Dealt in a snake, each
//    round's expensive units pair with the next round's cheap ones: a
//    longest-processing-time-first approximation without an atomic counter (on eight
//    images of unequal size it balances the CTAs to within ~10-20%, where a plain
//    stride over head-major units left some with twice the mean).
// Each unit is decoded from its 16-byte entry, and the next unit's entry is loaded as soon
// as the current one is taken, so that load's latency is hidden behind a whole unit of
// work instead of stalling every role at each unit boundary.  With a shared-memory work
// table (a call of few segments) the entry is looked up there instead.  The unit count
// stays below 2^31 (tokens x heads in device memory).
//
// In the split-key instantiation, when the call's (entry, head) units fit the workspace
// (`split`: at most half as many as SMs), each becomes two units that take the first and
// the second half of the segment's key tiles; the two halves are combined in the
// epilogue.  A segment of fewer than kSplitMinKeyTiles key tiles is not split (the
// combine costs more than half its keys save): its second unit is empty and skipped by
// every role alike.
template <bool kSplit>
class UnitStream {
 public:
  __device__ __forceinline__ UnitStream(const WorkEntry* entries, const SchedTable* tab,
                                        uint32_t E, uint32_t total, uint32_t H, int order,
                                        bool split = false)
      : entries_(reinterpret_cast<const int4*>(entries)), tab_(tab), E_(E), H_(H),
        total_(total), entry_major_(order != 0), split_on_(kSplit && split) {
    locate();
  }
  __device__ __forceinline__ bool valid() const { return u_ < total_; }
  __device__ __forceinline__ Unit take() {
    Unit x;
    x.head = static_cast<int>(head_);
    x.seg_start = cur_.z;
    x.seg_end = cur_.w;
    x.q0 = x.seg_start + cur_.y * (2 * kBM);
    x.has_q1 = x.q0 + kBM < x.seg_end;
    const int nkv = (x.seg_end - x.seg_start + kBN - 1) / kBN;
    if (split_on_ && nkv >= kSplitMinKeyTiles) {
      const int first = (nkv + 1) / 2;
      x.parts = 2;
      x.split = static_cast<int>(split_);
      x.kv0 = split_ ? first : 0;
      x.nkv = split_ ? nkv - first : first;
    } else {
      x.parts = 1;
      x.split = 0;
      x.kv0 = 0;
      x.nkv = nkv;
    }
    x.slot = base_;
    ++k_;
    locate();
    return x;
  }

 private:
  __device__ __forceinline__ void locate() {
    const uint32_t c = blockIdx.x, G = gridDim.x;
#pragma unroll 1
    for (;;) {
      u_ = k_ * G + ((k_ & 1) ? G - 1 - c : c);
      if (u_ >= total_) return;
      find();
      // the second half of a segment too short to split is empty: skip it
      if (!split_on_ || split_ == 0 || cur_.w - cur_.z > (kSplitMinKeyTiles - 1) * kBN) return;
      ++k_;
    }
  }
  __device__ __forceinline__ void find() {
    base_ = split_on_ ? u_ >> 1 : u_;
    split_ = split_on_ ? u_ & 1u : 0u;
    uint32_t e;
    if (entry_major_) {
      e = base_ / H_;
      head_ = base_ - e * H_;
    } else {
      head_ = base_ / E_;
      e = base_ - head_ * E_;
    }
    if (tab_ != nullptr) {  // the last segment whose first entry is <= e
      int s = 0;
#pragma unroll 1
      while (s + 1 < tab_->n && tab_->prefix[s + 1] <= static_cast<int>(e)) ++s;
      cur_ = tab_->seg[s];
      cur_.y = static_cast<int>(e) - tab_->prefix[s];
    } else {
      cur_ = __ldg(entries_ + e);
    }
  }
  const int4* entries_;
  const SchedTable* tab_;
  uint32_t E_, H_, total_, k_ = 0, u_ = 0, head_ = 0, base_ = 0, split_ = 0;
  bool entry_major_;
  bool split_on_;
  int4 cur_ = make_int4(0, 0, 0, 0);
};

__device__ __forceinline__ void st_global_v8(void* ptr, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// The MMA thread shares its SM sub-partition with softmax warps that issue every
// cycle, so it must spend as few instructions per MMA as possible: descriptors are
// built once per tile base and each K16 step only adds a constant to the start
// address field (16-byte units; never carries out of the 14-bit field since
// shared addresses stay below 256 KB).

// S = Q K^T: both operands K-major (head dim contiguous), 64-byte swizzle,
// three 32-column chunks of 8 KB; K = 96 as six K16 steps.
__device__ __forceinline__ uint64_t qk_desc(uint32_t saddr) {
  return make_smem_desc(saddr, 16, 512, kSwizzle64B);
}
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc,
                                         uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const uint64_t off = static_cast<uint64_t>(((kk >> 1) * kChunkBytes + (kk & 1) * 32) >> 4);
    mma_ss(d_tmem, q_desc + off, k_desc + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P [V | 1]: P (128 x 128 bf16) from TMEM, V MN-major (head dim contiguous):
// 8-key groups 512 B apart (SBO), 32-column chunks 8 KB apart (LBO), N = 112 reaching
// into the ones chunk; eight K16 steps.
__device__ __forceinline__ uint64_t pv_desc(uint32_t saddr) {
  return make_smem_desc(saddr, kChunkBytes, 512, kSwizzle64B);
}
// One key chunk of the K loop (keys chunk * 128 / kPChunks onwards), so the product can
// start on the first keys while the softmax still computes the others.
__device__ __forceinline__ void issue_pv_chunk(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc,
                                               uint32_t idesc, int chunk, bool accumulate) {
  constexpr int kSteps = (kBN / 16) / kPChunks;  // K16 steps per chunk
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int kk = chunk * kSteps + s;
    mma_ts(d_tmem, p_tmem + kk * 8, v_desc + static_cast<uint64_t>((kk * 1024) >> 4), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

// O_i += P_i [V | 1] for one key tile, chunk by chunk as the softmax releases P.
__device__ __forceinline__ bool issue_pv(Smem& sm, int tile, uint32_t d_tmem, uint32_t p_tmem,
                                         uint64_t v_desc, uint32_t idesc, uint32_t parity,
                                         bool accumulate, volatile int* abort_flag, int* dev_status) {
#pragma unroll
  for (int c = 0; c < kPChunks; ++c) {
    if (!mma_wait(&sm.p_full[tile][c], parity, abort_flag, dev_status)) return false;
    tc_fence_after();
    issue_pv_chunk(d_tmem, p_tmem, v_desc, idesc, c, accumulate);
  }
  return true;
}

// Every lane waits; the outcome is made warp-uniform because the tcgen05.ld/st
// that follow are warp-collective.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* dev_status) {
  const bool ok = mbar_wait_bounded(bar, parity, abort_flag, dev_status);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, uint64_t* bar,
                                         int head, int row0) {
#pragma unroll
  for (int c = 0; c < kD / 32; ++c)
    tma_load_3d(static_cast<uint8_t*>(dst) + c * kChunkBytes, map, bar, c * 32, head, row0);
}

// Builds the shared-memory work table of a call with n <= kInlineSegments segments, by one
// warp: the same validation (cu[0] == 0, cu[n] == T, no negative length), the same
// longest-first order (ties by index) and the same unit order flag as the scheduling
// prepass, so the units, and the results, are identical to that path's.
__device__ __forceinline__ void build_sched_table(SchedTable& t, const int32_t* cu, int n, int T,
                                                  int lane) {
  constexpr unsigned kAll = 0xffffffffu;
  int start = 0, end = 0;
  bool bad = false;
  if (lane < n) {
    start = __ldg(cu + lane);
    end = __ldg(cu + lane + 1);
    bad = end < start || (lane == 0 && start != 0) || (lane == n - 1 && end != T);
  }
  bad = __any_sync(kAll, bad);
  const int len = end - start;
  // key = (INT_MAX - len) << 32 | segment: ascending order = longest first
  unsigned long long key =
      lane < n ? (static_cast<unsigned long long>(0x7FFFFFFFu - static_cast<unsigned>(len)) << 32) |
                     static_cast<unsigned>(lane)
               : ~0ull;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {  // bitonic sort over the warp, ascending
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long other = __shfl_xor_sync(kAll, key, j);
      const bool keep_min = ((lane & j) == 0) == ((lane & k) == 0);
      key = keep_min ? (other < key ? other : key) : (other < key ? key : other);
    }
  }
  const int seg = lane < n ? static_cast<int>(key & 0xFFFFFFFFu) : 0;  // at sorted position lane
  const int ss = __shfl_sync(kAll, start, seg), se = __shfl_sync(kAll, end, seg);
  const int cnt = lane < n ? (se - ss + kBf16BlockRows - 1) / kBf16BlockRows : 0;
  int incl = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(kAll, incl, d);
    if (lane >= d) incl += y;
  }
  const int E = __shfl_sync(kAll, incl, n - 1);
  // segments of unequal (non-empty) lengths: entry-major order, longest first
  const int lmin = __reduce_min_sync(kAll, lane < n && len > 0 ? len : 0x7FFFFFFF);
  const int lmax = __reduce_max_sync(kAll, lane < n && len > 0 ? len : 0);
  if (lane < n) {
    t.seg[lane] = make_int4(seg, 0, ss, se);
    t.prefix[lane + 1] = incl;
  }
  if (lane == 0) {
    t.prefix[0] = 0;
    t.n = n;
    t.bad = bad ? 1 : 0;
    t.E = bad ? 0 : E;
    t.order = lmin < lmax ? 1 : 0;
  }
}

// The MMA issuer (one thread).  It is kept out of line so that its loop is one compact
// piece of code: the thread sleeps in mbarrier waits between short bursts of MMA
// issue, and its wake-up latency is on the critical path of every key tile.
template <bool kSplit>
__device__ __noinline__ void mma_role(Smem& sm, const Bf16Args& a, uint32_t tmem, const SchedTable* tab,
                                      uint32_t E, uint32_t total, int order, bool split,
                                      volatile int* abort_flag, int* dev_status) {
  if (a.stall_test_cycles > 0) {
    // Failure-path self-test: this wait can never succeed, so it runs out after
    // stall_test_cycles, raises the CTA's abort flag and records a timeout; every other
    // role then leaves its loop exactly as after a real stall.  No MMA has been issued.
    if (!mbar_wait_bounded(&sm.never, 0, abort_flag, dev_status, a.stall_test_cycles)) return;
  }
  const uint32_t idesc_qk = a.idesc_qk;
  const uint32_t idesc_pv = make_idesc_bf16(kBM, kDv, false, true, false);
  // Q buffer b, tile i starts (2 b + i) * kTileBytes after q[0][0]
  const uint64_t dqbase = qk_desc(smem_u32(sm.q[0][0]));
  // stage s of the K (V) ring starts kTileBytes (kVTileBytes) after stage s-1
  const uint64_t dk0 = qk_desc(smem_u32(sm.k[0])), dv0 = pv_desc(smem_u32(sm.v[0]));
  auto dk = [&](uint32_t st) { return dk0 + static_cast<uint64_t>(st * (kTileBytes >> 4)); };  // K stage
  auto dv = [&](uint32_t st) { return dv0 + static_cast<uint64_t>(st * (kVTileBytes >> 4)); };
  auto dq = [&](uint32_t b, int tile) {
    return dqbase + static_cast<uint64_t>((2 * b + tile) * (kTileBytes >> 4));
  };
  uint32_t kv_it = 0, unit_it = 0, p_cnt0 = 0, p_cnt1 = 0;
  uint32_t q1_it0 = 0, q1_it1 = 0;  // Q1 loads consumed per buffer
  // Q of unit number n (buffer n % kQBufs) has landed
  uint64_t(*qbar)[2] = sm.q_full;
  auto wait_q = [&](const Unit& u, uint32_t n) {
    const uint32_t b = n % kQBufs;
    if (!mma_wait(&qbar[b][0], (n / kQBufs) & 1, abort_flag, dev_status)) return false;
    if (u.has_q1 && !mma_wait(&qbar[b][1], (b ? q1_it1 : q1_it0) & 1, abort_flag, dev_status))
      return false;
    return true;
  };
  // The issue order is one flat stream over all key tiles of all units of this CTA:
  //   PV0(j) | QK0(j+1) | PV1(j) | QK1(j+1)
  // where tile j+1 after a unit's last tile is the next unit's first.  So a Q tile's next S
  // is computed right after its own last PV of a unit (during that tile's epilogue), not
  // behind the other tile's last PV.  The K/V ring runs on across units as the loader fills it.
  UnitStream<kSplit> us(a.entries, tab, E, total, a.H, order, split);
  bool ok = us.valid();
  Unit x;
  if (ok) {
    x = us.take();
    ok = wait_q(x, 0);
  }
  if (ok) {
    const uint32_t st = 0, b = 0;
    ok = mma_wait(&sm.k_full[st], 0, abort_flag, dev_status);
    if (ok) {
      tc_fence_after();
      issue_qk(tmem + kColS0, dq(b, 0), dk(st), idesc_qk);
      mma_commit(&sm.s_full[0]);
      if (x.has_q1) {
        issue_qk(tmem + kColS1, dq(b, 1), dk(st), idesc_qk);
        mma_commit(&sm.s_full[1]);
      }
      mma_commit(&sm.k_empty[st]);
      if (x.nkv == 1) mma_commit(&sm.q_empty[b]);
    }
  }
  while (ok) {
    // S(x, 0) has been issued for both tiles
    const uint32_t b = unit_it % kQBufs, b2 = (unit_it + 1) % kQBufs;
    const bool has_next = us.valid();
    Unit y = x;
    if (has_next) y = us.take();
    for (int j = 0; j < x.nkv; ++j) {
      const uint32_t it = kv_it + j, st = it % kVStages;
      const bool last = j + 1 == x.nkv;
      const bool more = !last || has_next;  // a QK follows: this unit's next tile or y's first
      const uint32_t st1 = (it + 1) % kKStages;
      const uint32_t nb = last ? b2 : b;                  // Q buffer of that QK
      const bool next_q1 = last ? y.has_q1 : x.has_q1;    // ... and whether it has tile 1
      if (!mma_wait(&sm.v_full[st], (it / kVStages) & 1, abort_flag, dev_status)) { ok = false; break; }
      if (!issue_pv(sm, 0, tmem + kColO0, tmem + kColS0, dv(st), idesc_pv, p_cnt0 & 1, j > 0,
                    abort_flag, dev_status)) { ok = false; break; }
      ++p_cnt0;
      mma_commit(&sm.o_done[0]);
      // V_j is released as soon as its last PV has been issued (not behind the next QK)
      if (!x.has_q1) mma_commit(&sm.v_empty[st]);
      if (more) {
        if (last && !wait_q(y, unit_it + 1)) { ok = false; break; }
        if (!mma_wait(&sm.k_full[st1], ((it + 1) / kKStages) & 1, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        issue_qk(tmem + kColS0, dq(nb, 0), dk(st1), idesc_qk);
        mma_commit(&sm.s_full[0]);
      }
      if (x.has_q1) {
        if (!issue_pv(sm, 1, tmem + kColO1, tmem + kColS1, dv(st), idesc_pv, p_cnt1 & 1, j > 0,
                      abort_flag, dev_status)) { ok = false; break; }
        ++p_cnt1;
        mma_commit(&sm.o_done[1]);
        mma_commit(&sm.v_empty[st]);
      }
      if (more) {
        if (next_q1) {
          issue_qk(tmem + kColS1, dq(nb, 1), dk(st1), idesc_qk);
          mma_commit(&sm.s_full[1]);
        }
        mma_commit(&sm.k_empty[st1]);
        // release a Q buffer after the last QK that reads it
        if (!last && j + 2 == x.nkv) mma_commit(&sm.q_empty[b]);
        if (last && y.nkv == 1) mma_commit(&sm.q_empty[b2]);
      }
    }
    if (!ok || !has_next) break;
    kv_it += x.nkv;
    if (x.has_q1) { if (b) ++q1_it1; else ++q1_it0; }
    x = y;
    ++unit_it;
  }
  // All MMAs issued by this thread complete before TMEM is released.
  mma_commit(&sm.drain);
  mbar_wait_drain(&sm.drain, 0);
}

// The epilogue, fixed per instantiation:
//   kEpiRows   every row is stored by its thread; warp 11 idles;
//   kEpiStaged whole O tiles leave through the Q buffers and TMA stores (warp 11);
//   kEpiSplit  the split-key units: each half writes its unnormalised rows with (m, l) to
//              a workspace and the second half to finish combines the two.
// Separate instantiations, because the staging code alone, never run, moved the softmax
// loop's code enough to cost ~1.5% on long units.
template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                     const __grid_constant__ Bf16Args a) {
  constexpr bool kStageO = kEpi == kEpiStaged;
  constexpr bool kSplit = kEpi == kEpiSplit;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Set-up that reads nothing the scheduling prepass writes: with programmatic dependent
  // launch it overlaps the prepass.
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      for (int b = 0; b < kQBufs; ++b) {
        mbar_init(&sm.q_full[b][i], 1);
      }
      mbar_init(&sm.s_full[i], 1);
      for (int c = 0; c < kPChunks; ++c) mbar_init(&sm.p_full[i][c], kBM);
      mbar_init(&sm.o_done[i], 1);
    }
    for (int b = 0; b < kQBufs; ++b) {
      mbar_init(&sm.q_empty[b], 1);
      mbar_init(&sm.q_free[b], 1);
    }
    for (int b = 0; b < kQBufs; ++b)
      for (int i = 0; i < 2; ++i) mbar_init(&sm.o_staged[b][i], kBM);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.never, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  // Ones chunk of every V stage: row r holds bf16 1.0 in column 0 and zeros elsewhere,
  // in the 64-byte swizzle the MMA reads (16-byte unit u of row r is stored at unit
  // u ^ ((r >> 1) & 3)).  TMA never writes this chunk.
  for (int i = tid; i < kVStages * 128 * 4; i += kThreads) {
    const int st = i / (128 * 4), r = (i / 4) % 128, unit = i % 4;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (unit == ((r >> 1) & 3)) val.x = 0x3F80u;  // bf16 1.0 in the low half = column 0
    *reinterpret_cast<uint4*>(sm.v[st] + 3 * kChunkBytes + r * 64 + unit * 16) = val;
  }
  fence_proxy_async_smem();
  if (warp == kWarpMma) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int* dev_status = a.dev_status;

  // Inputs and the work list are read only after the previous kernel in the stream (the
  // prepass, when one runs) has completed.
  griddep_wait();
  const SchedTable* tab = nullptr;
  uint32_t E;
  int order;
  if (a.inline_sched) {
    if (warp == 0) build_sched_table(sm.sched, a.cu_seqlens, a.num_segments, a.total_tokens, lane);
    __syncthreads();
    tab = &sm.sched;
    E = static_cast<uint32_t>(sm.sched.E);
    order = sm.sched.order;
    if (blockIdx.x == 0 && tid == 0) {
      *a.next_status = 0;  // the next call on this scratch starts after this one ends
      if (sm.sched.bad) atomicOr(a.dev_status, kDevStatusBadSeqlens);
    }
  } else {
    E = static_cast<uint32_t>(a.hdr->num_entries);
    order = a.hdr->order;
  }
  // split-key units when this call's (entry, head) units fit the workspace: decided here,
  // from the work list itself, so the in-kernel and prepass work lists split alike
  const bool split = kSplit && E * static_cast<uint32_t>(a.H) <= static_cast<uint32_t>(a.split_units_max);
  const uint32_t total = E * static_cast<uint32_t>(a.H) * (split ? 2u : 1u);
  if (blockIdx.x >= total) {  // uniform over the CTA: no unit for it
    if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
    return;
  }

  if (warp >= 8) {
   setmaxnreg_dec<kRegsOther>();
   if (warp == kWarpLoad) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      uint32_t kv_it = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      for (UnitStream<kSplit> us(a.entries, tab, E, total, a.H, order, split); us.valid() && ok;) {
        const Unit x = us.take();
        for (int j = 0; j < x.nkv; ++j, ++kv_it) {
          const uint32_t sk = kv_it % kKStages, fk = kv_it / kKStages;
          const uint32_t sv = kv_it % kVStages, fv = kv_it / kVStages;
          const int row0 = x.seg_start + (x.kv0 + j) * kBN;
          if (fk > 0 && !mbar_wait_bounded(&sm.k_empty[sk], (fk - 1) & 1, abort_flag, dev_status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[sk], kTileBytes);
          tma_tile(sm.k[sk], &tk, &sm.k_full[sk], x.head, row0);
          ++k_issued;
          if (fv > 0 && !mbar_wait_bounded(&sm.v_empty[sv], (fv - 1) & 1, abort_flag, dev_status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.v_full[sv], kTileBytes);
          tma_tile(sm.v[sv], &tv, &sm.v_full[sv], x.head, row0);
          ++v_issued;
        }
      }
      {
        // Every copy this thread issued has landed before the CTA exits.  Normally the MMA
        // thread has already waited on each of them and these waits return at once; after
        // an abort the last fills of the ring may still be in flight.  Only the last
        // fills of each ring (one per stage) can be outstanding (each earlier one was waited
        // on before its stage was refilled).
        for (uint32_t f = (k_issued > kKStages ? k_issued - kKStages : 0); f < k_issued; ++f)
          mbar_wait_drain(&sm.k_full[f % kKStages], (f / kKStages) & 1);
        for (uint32_t f = (v_issued > kVStages ? v_issued - kVStages : 0); f < v_issued; ++f)
          mbar_wait_drain(&sm.v_full[f % kVStages], (f / kVStages) & 1);
      }
    }
   } else if (warp == kWarpLoadQ) {
    // ------------------------------------------------------------ Q loader
    if (lane == 0) {
      // per-buffer load counts (kept in scalars: a runtime-indexed array would go to local memory)
      uint32_t unit_it = 0, q0a = 0, q0b = 0, q1a = 0, q1b = 0;
      for (UnitStream<kSplit> us(a.entries, tab, E, total, a.H, order, split); us.valid(); ++unit_it) {
        const Unit x = us.take();
        const uint32_t b = unit_it % kQBufs, use = unit_it / kQBufs;
        // buffer b is free once every QK of the unit that used it before has completed and
        // the O tiles that unit staged in it have been stored
        if (use > 0 && (!mbar_wait_bounded(&sm.q_empty[b], (use - 1) & 1, abort_flag, dev_status) ||
                        (kStageO &&
                         !mbar_wait_bounded(&sm.q_free[b], (use - 1) & 1, abort_flag, dev_status))))
          break;
        mbar_arrive_expect_tx(&sm.q_full[b][0], kTileBytes);
        tma_tile(sm.q[b][0], &tq, &sm.q_full[b][0], x.head, x.q0);
        if (b) ++q0b; else ++q0a;
        if (x.has_q1) {
          mbar_arrive_expect_tx(&sm.q_full[b][1], kTileBytes);
          tma_tile(sm.q[b][1], &tq, &sm.q_full[b][1], x.head, x.q0 + kBM);
          if (b) ++q1b; else ++q1a;
        }
      }
      {
        // Every Q copy issued has landed before the CTA exits (see the K/V loader).
        if (q0a) mbar_wait_drain(&sm.q_full[0][0], (q0a - 1) & 1);
        if (q1a) mbar_wait_drain(&sm.q_full[0][1], (q1a - 1) & 1);
        if (kQBufs > 1 && q0b) mbar_wait_drain(&sm.q_full[kQBufs - 1][0], (q0b - 1) & 1);
        if (kQBufs > 1 && q1b) mbar_wait_drain(&sm.q_full[kQBufs - 1][1], (q1b - 1) & 1);
      }
    }
   } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      mma_role<kSplit>(sm, a, tmem, tab, E, total, order, split, abort_flag, dev_status);
    }
   } else if (kStageO && warp == kWarpStore) {
    // ------------------------------------------------------------ O tile stores
    // A whole 128-row O tile is staged by its softmax warpgroup in the unit's Q buffer
    // (free once the unit's last QK has run; same layout as the Q tile) and leaves by three
    // TMA stores.  Buffer b is released to the Q loader (q_free) once those stores have
    // read it; a unit with nothing staged releases it at once.  This thread first waits
    // for the unit's Q to land: the loader has then passed its q_free wait for the unit
    // that used b before, so each arrival completes the phase the loader waits on next.
    if (lane == 0) {
      uint32_t unit_it = 0, staged = 0;  // bit 2b + i: parity of (buffer b, tile i) stagings
      bool ok = true;
      for (UnitStream<kSplit> us(a.entries, tab, E, total, a.H, order, split); us.valid() && ok; ++unit_it) {
        const Unit x = us.take();
        const uint32_t b = unit_it % kQBufs;
        if (!mbar_wait_bounded(&sm.q_full[b][0], (unit_it / kQBufs) & 1, abort_flag, dev_status)) break;
        bool issued = false;
        for (int i = 0; i < (x.has_q1 ? 2 : 1); ++i) {
          const int row0 = x.q0 + i * kBM;
          if (row0 + kBM > x.seg_end) continue;  // a partial tile is stored row by row
          const uint32_t bit = 1u << (2 * b + i);
          if (!mbar_wait_bounded(&sm.o_staged[b][i], (staged & bit) ? 1u : 0u, abort_flag, dev_status)) {
            ok = false;
            break;
          }
          staged ^= bit;
#pragma unroll
          for (int c = 0; c < kD / 32; ++c)
            tma_store_3d(&to, sm.q[b][i] + c * kChunkBytes, c * 32, x.head, row0);
          issued = true;
        }
        if (!ok) break;
        if (issued) {
          bulk_commit_group();
          bulk_wait_read_all();
        }
        mbar_arrive(&sm.q_free[b]);
      }
      // Shared memory stays valid until every store has read it (stores issued before an
      // abort are still uncommitted); the grid's completion covers their global writes.
      bulk_commit_group();
      bulk_wait_read_all();
    }
   }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    setmaxnreg_inc<kRegsSoftmax>();
    const int wg = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (wg ? kColS1 : kColS0);
    const uint32_t tO = tmem + lane_base + (wg ? kColO1 : kColO0);
    const float c = a.scale_log2;
    uint32_t s_cnt = 0, o_base = 0, unit_it = 0;
    for (UnitStream<kSplit> us(a.entries, tab, E, total, a.H, order, split); us.valid();) {
      const Unit x = us.take();
      const uint32_t b = unit_it++ % kQBufs;
      if (wg == 1 && !x.has_q1) continue;
      const int row_tok = x.q0 + wg * kBM + r;
      float m = 0.f;
      bool ok = true;
      for (int j = 0; j < x.nkv; ++j) {
        if (!warp_wait(&sm.s_full[wg], s_cnt & 1, abort_flag, dev_status)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        const int nvalid = x.seg_end - (x.seg_start + (x.kv0 + j) * kBN);  // >= 1
        const bool masked = nvalid < kBN;
        float pm[8];
        // pass 1, row max: the row in two 64-column halves, eight independent
        // three-input max chains
#pragma unroll 1  // one copy of the half body: a smaller hot loop for the instruction cache
        for (int half = 0; half < 2; ++half) {
          uint32_t su[kBN / 2];
          float* sf = reinterpret_cast<float*>(su);
          tmem_ld32(tS + half * 64, su);
          tmem_ld32(tS + half * 64 + 32, su + 32);
          tmem_ld_wait();
          reg_fence<kBN / 2>(su);
          if (masked) {
#pragma unroll
            for (int i = 0; i < kBN / 2; ++i)
              if (half * 64 + i >= nvalid) sf[i] = -INFINITY;
          }
          if (half == 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q) pm[q] = fmaxf(sf[q], sf[q + 8]);
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) pm[q] = fmax3(pm[q], sf[q], sf[q + 8]);
          }
#pragma unroll
          for (int i = 16; i < kBN / 2; i += 16) {
#pragma unroll
            for (int q = 0; q < 8; ++q) pm[q] = fmax3(pm[q], sf[i + q], sf[i + 8 + q]);
          }
        }
        const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]),
                               fmaxf(pm[6], pm[7]));
        const float mt = mx * c;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m = mt;
        } else if (mt > m + kRescaleThreshold) {
          alpha = ex2_approx(m - mt);
          m = mt;
          rescale = true;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          // O (with its row-sum column) must hold PV_{j-1} before it is scaled (the commit
          // behind S_j already implies it; the wait makes it explicit).
          if (!warp_wait(&sm.o_done[wg], (o_base + j - 1) & 1, abort_flag, dev_status)) { ok = false; break; }
          tc_fence_after();
          // in 32-column chunks to keep the register footprint small
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int c0 = 0; c0 < kDv; c0 += 32) {
            uint32_t o[32];
            if (c0 + 32 <= kDv) tmem_ld32(tO + c0, o);
            else tmem_ld16(tO + c0, o);
            tmem_ld_wait();
            reg_fence<32>(o);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 y = fmul2(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
              o[i] = __float_as_uint(y.x);
              o[i + 1] = __float_as_uint(y.y);
            }
            if (c0 + 32 <= kDv) tmem_st32(tO + c0, o);
            else tmem_st16(tO + c0, o);
          }
        }
        // P in two key halves: the PV product of the first 64 keys starts while the
        // exponentials of the other 64 are computed
        // pass 2: reload each half of S, exponentiate, store its P half (P half 0
        // overwrites S columns 0-31 only after that half has been read)
        const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
#pragma unroll 1  // one copy of the half body: a smaller hot loop for the instruction cache
        for (int half = 0; half < 2; ++half) {
          uint32_t su[kBN / 2];
          const float* sf = reinterpret_cast<const float*>(su);
          tmem_ld32(tS + half * 64, su);
          tmem_ld32(tS + half * 64 + 32, su + 32);
          tmem_ld_wait();
          reg_fence<kBN / 2>(su);
          uint32_t p[kBN / 4];
#pragma unroll
          for (int i2 = 0; i2 < kBN / 4; ++i2) {
            const float2 t = ffma2(make_float2(sf[2 * i2], sf[2 * i2 + 1]), c2, nm2);
            if (kPolyEvery > 0 && i2 % kPolyEvery == kPolyEvery - 1) {
              const float2 e = exp2_poly2(t);  // FMA pipe: takes load off the MUFU
              p[i2] = pack_bf16x2(e.x, e.y);
            } else {
              p[i2] = pack_bf16x2(ex2_approx(t.x), ex2_approx(t.y));
            }
          }
          if (masked) {  // exact zeros past the segment end (also when scale is 0)
#pragma unroll
            for (int i2 = 0; i2 < kBN / 4; ++i2) {
              const int i = half * (kBN / 4) + i2;
              if (2 * i >= nvalid) p[i2] = 0u;
              else if (2 * i + 1 >= nvalid) p[i2] &= 0xFFFFu;
            }
          }
          tmem_st32(tS + half * (kBN / 4), p);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&sm.p_full[wg][half]);
        }
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> HBM (rows inside the segment only); l = O column 96
      if (!warp_wait(&sm.o_done[wg], (o_base + x.nkv - 1) & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      uint32_t o[kD + 1];
      tmem_ld32(tO + 0, o);
      tmem_ld32(tO + 32, o + 32);
      tmem_ld32(tO + 64, o + 64);
      tmem_ld1(tO + 96, o[96]);
      tmem_ld_wait();
      reg_fence<kD + 1>(o);
      const bool whole = kStageO && x.q0 + wg * kBM + kBM <= x.seg_end;  // staged for a TMA store
      if (kSplit && x.parts == 2) {
        // A split-key unit holds O and l over its half of the keys, both relative to
        // 2^m.  Each half writes its tile (per row: 96 values, m, l) as 25 float4 columns
        // of 128 rows, so a warp stores 512 contiguous bytes at a time.  Then, per warp,
        // lane 0 swaps this call's id into the warp's flag (release: the warp's rows are
        // visible first); the half that finds the id there finished second (acquire: the
        // other half's rows are visible) and combines the two into O.  The warp-uniform
        // flow keeps the shuffles and __syncwarp convergent.
        const size_t tile_id = static_cast<size_t>(x.slot) * 2 + wg;
        float4* mine = reinterpret_cast<float4*>(a.part) + (tile_id * 2 + x.split) * (kPartF4 * kBM) + r;
        const float4* other =
            reinterpret_cast<const float4*>(a.part) + (tile_id * 2 + (x.split ^ 1)) * (kPartF4 * kBM) + r;
        const float l_own = __uint_as_float(o[96]);
#pragma unroll
        for (int i = 0; i < kD / 4; ++i)
          __stcg(mine + i * kBM,
                 make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                             __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3])));
        __stcg(mine + (kD / 4) * kBM, make_float4(m, l_own, 0.f, 0.f));
        __syncwarp();
        uint32_t seen = 0;
        if (lane == 0) seen = atom_exch_acq_rel_gpu(a.part_flag + tile_id * 4 + (warp & 3), a.call_id);
        seen = __shfl_sync(0xffffffffu, seen, 0);
        __syncwarp();  // lane 0's acquire orders the other lanes' reads below too
        if (seen == a.call_id && row_tok < x.seg_end) {
          // the arithmetic runs on (first half, second half) whichever half combines,
          // so the result does not depend on which finished first
          const bool first = x.split == 0;
          const float4 ml = __ldcg(other + (kD / 4) * kBM);
          const float m0 = first ? m : ml.x, m1 = first ? ml.x : m;
          const float l0 = first ? l_own : ml.y, l1 = first ? ml.y : l_own;
          const float mm = fmaxf(m0, m1);
          const float a0 = exp2f(m0 - mm), a1 = exp2f(m1 - mm);
          const float inv = 1.0f / fmaf(a0, l0, a1 * l1);
          const float c0 = a0 * inv, c1 = a1 * inv;
          uint32_t w[kD / 2];
#pragma unroll
          for (int i = 0; i < kD / 4; ++i) {
            const float4 ov = __ldcg(other + i * kBM);
            const float4 ow = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                          __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
            const float4 h0 = first ? ow : ov, h1 = first ? ov : ow;
            w[2 * i] = pack_bf16x2(fmaf(c0, h0.x, c1 * h1.x), fmaf(c0, h0.y, c1 * h1.y));
            w[2 * i + 1] = pack_bf16x2(fmaf(c0, h0.z, c1 * h1.z), fmaf(c0, h0.w, c1 * h1.w));
          }
          uint8_t* row = static_cast<uint8_t*>(a.out) +
                         (static_cast<size_t>(row_tok) * a.H + x.head) * (kD * 2);
          if (a.out_align32) {
#pragma unroll
            for (int i = 0; i < kD / 16; ++i) st_global_v8(row + 32 * i, w + 8 * i);
          } else {
#pragma unroll
            for (int i = 0; i < kD / 8; ++i)
              reinterpret_cast<uint4*>(row)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      } else if (whole || row_tok < x.seg_end) {
        const float inv_l = 1.0f / __uint_as_float(o[96]);
        const float2 il2 = make_float2(inv_l, inv_l);
        uint32_t w[kD / 2];
#pragma unroll
        for (int i = 0; i < kD / 2; ++i) {
          const float2 y = fmul2(make_float2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), il2);
          w[i] = pack_bf16x2(y.x, y.y);
        }
        if (whole) {
          // the row into the tile's Q buffer, in the Q tile's layout (three 32-column chunks,
          // 16-byte unit u of row r at unit u ^ ((r >> 1) & 3)); the store warp sends it out
          uint8_t* tile = sm.q[b][wg] + r * 64;
          const uint32_t sw = (r >> 1) & 3;
#pragma unroll
          for (int c = 0; c < kD / 32; ++c) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t* g = w + 16 * c + 4 * u;
              *reinterpret_cast<uint4*>(tile + c * kChunkBytes + ((u ^ sw) << 4)) =
                  make_uint4(g[0], g[1], g[2], g[3]);
            }
          }
          fence_proxy_async_smem();  // generic-proxy writes, read by the TMA store
          mbar_arrive(&sm.o_staged[b][wg]);
        } else {
          uint8_t* row = static_cast<uint8_t*>(a.out) +
                         (static_cast<size_t>(row_tok) * a.H + x.head) * (kD * 2);
          // a row is 192 contiguous bytes: six 32-byte stores (whole sectors) when the
          // output is 32-byte aligned, else twelve 16-byte stores
          if (a.out_align32) {
#pragma unroll
            for (int i = 0; i < kD / 16; ++i) st_global_v8(row + 32 * i, w + 8 * i);
          } else {
#pragma unroll
            for (int i = 0; i < kD / 8; ++i)
              reinterpret_cast<uint4*>(row)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
      o_base += x.nkv;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t bf16_smem_bytes() { return kSmemBytes; }

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const Bf16Args& args, int grid,
                             int epilogue, cudaStream_t stream) {
  // Programmatic stream serialization: the kernel may launch while the scheduling prepass
  // before it still runs, and waits for it (griddepcontrol.wait) before reading its output.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (epilogue) {
    case kEpiRows: return cudaLaunchKernelEx(&cfg, attn_bf16_kernel<kEpiRows>, tq, tk, tv, to, args);
    case kEpiStaged: return cudaLaunchKernelEx(&cfg, attn_bf16_kernel<kEpiStaged>, tq, tk, tv, to, args);
    case kEpiSplit: return cudaLaunchKernelEx(&cfg, attn_bf16_kernel<kEpiSplit>, tq, tk, tv, to, args);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t prepare_attn_bf16() {
  const int bytes = static_cast<int>(kSmemBytes);
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<kEpiRows>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bf16_kernel<kEpiStaged>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bf16_kernel<kEpiSplit>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  return e;
}

}  // namespace vt
