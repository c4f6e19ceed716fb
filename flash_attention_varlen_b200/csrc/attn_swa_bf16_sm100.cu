// bf16 causal attention with a local window and grouped-query heads, head size 128, for
// B200 (sm_100a): the text decoder's attention (the Muse Glimmer next-steps document,
// "Architecture / Text decoder": 32 query heads over 2 key/value heads, head size 128, a
// local window of 2048 tokens on sliding layers, full causal attention on the others).
//
// Per packed segment, query i attends keys j of its segment with i - W < j <= i (W = 0: no
// window); query head h reads key/value head h / (Hq / Hkv).  Flash-style with a running
// softmax, as the vision kernel: scores never leave the SM.
//
// One CTA per SM works through units of 256 query rows of one (segment, query head): two
// 128-row Q tiles that share every K/V tile, as in the vision kernel, so the tensor core
// works on one tile while the other is in its softmax.  A unit visits only the key tiles its
// rows can see (from the window start of its first row to its last row), and each Q tile
// skips a key tile none of its rows can see.
//
//   warp 8 (loader)  : TMA loads of the two Q tiles and of each K and V tile into 2-stage
//                      rings (64-byte swizzle, four 32-column chunks).
//   warp 9 (MMA)     : one thread issues S_i = Q_i K^T (SS, M128 N128 K128) and
//                      O_i (+)= P_i V (TS, P from TMEM, N128) in the order
//                      S0 S1 | PV0 S0' | PV1 S1' | ...
//   warps 0-3, 4-7   : softmax for Q tiles 0 and 1, one thread per query row: the row's
//                      allowed keys of the tile, row max with a deferred rescale,
//                      p = 2^(s c - m) packed to bf16 over S in TMEM (in two 64-key halves,
//                      each handed to the PV as soon as it is stored), the row sum of the
//                      rounded p in f32; the epilogue O / l -> bf16 -> HBM.
//
// TMEM (512 columns): S0 [0,128), O0 [128,256), S1 [256,384), O1 [384,512); P_i overlays
// the first 64 columns of S_i.  Every mbarrier wait is bounded and an abort flag lets all
// roles leave together.
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

constexpr int kBM = 128;            // query rows per Q tile
constexpr int kUnitRows = kSwaBlockRows;  // 256: two Q tiles per unit
constexpr int kBN = 128;            // keys per tile
constexpr int kD = 128;
constexpr int kChunks = kD / 32;              // 32-column (64-byte) chunks per row
constexpr int kChunkBytes = 128 * 64;         // 128 rows x 32 bf16
constexpr int kTileBytes = kChunks * kChunkBytes;  // 32 KB
constexpr int kStages = 2;                    // K and V ring depth
constexpr int kThreads = 320;
constexpr int kWarpLoad = 8, kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;
// TMEM columns of Q tile i: S_i at 256 i, O_i at 256 i + 128
__host__ __device__ constexpr uint32_t col_s(int tile) { return 256u * tile; }
__host__ __device__ constexpr uint32_t col_o(int tile) { return 256u * tile + 128u; }
constexpr float kRescaleThreshold = 3.0f;  // log2 units, as the vision kernel

struct Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2][2], o_done[2];  // per Q tile (p_full: per 64-key half)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

struct Unit {
  int head, kv_head, q0, seg_start, seg_end;
  int j0, nkv;  // first key tile (from the segment start) and the tile count
  bool has_q1;  // the second Q tile holds rows of the segment
  // key tiles [first[i], last[i]] of the unit that Q tile i can see: a key tile none of
  // its rows can see (the last one for tile 0, a window-edge one for tile 1) is skipped
  int first[2], last[2];
};

// This CTA's units: a snake over the CTAs, entry-major with the query heads inner (the
// heads that share a key/value head run side by side and share its tiles in L2), segments
// longest first and, within a segment, its last row blocks (most keys) first.
struct Units {
  const WorkEntry* entries;
  long long total, G, cta;
  int Hq, group, window;
  __device__ bool get(long long k, Unit* x) const {
    const long long u = k * G + ((k & 1) ? G - 1 - cta : cta);
    if (u >= total) return false;
    const WorkEntry we = entries[u / Hq];
    x->head = static_cast<int>(u % Hq);
    x->kv_head = x->head / group;
    x->seg_start = we.seg_start;
    x->seg_end = we.seg_end;
    const int nblocks = (we.seg_end - we.seg_start + kUnitRows - 1) / kUnitRows;
    x->q0 = we.seg_start + (nblocks - 1 - we.qblock) * kUnitRows;
    x->has_q1 = x->q0 + kBM < we.seg_end;
    const int q_last = min(x->q0 + kUnitRows, we.seg_end) - 1;
    const int lo = window > 0 ? max(we.seg_start, x->q0 - window + 1) : we.seg_start;
    x->j0 = (lo - we.seg_start) / kBN;
    x->nkv = (q_last - we.seg_start) / kBN - x->j0 + 1;
    // tile 0: rows q0 .. min(q0 + 127, end - 1), from the unit's first key tile
    x->first[0] = 0;
    x->last[0] = (min(x->q0 + kBM, we.seg_end) - 1 - we.seg_start) / kBN - x->j0;
    // tile 1: rows q0 + 128 .., to the unit's last key tile
    const int lo1 = window > 0 ? max(we.seg_start, x->q0 + kBM - window + 1) : we.seg_start;
    x->first[1] = (lo1 - we.seg_start) / kBN - x->j0;
    x->last[1] = x->nkv - 1;
    return true;
  }
};

__device__ __forceinline__ uint64_t qk_desc(uint32_t saddr) {
  return make_smem_desc(saddr, 16, 512, kSwizzle64B);
}
__device__ __forceinline__ uint64_t pv_desc(uint32_t saddr) {
  return make_smem_desc(saddr, kChunkBytes, 512, kSwizzle64B);
}

__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int head,
                                         int row0) {
#pragma unroll
  for (int c = 0; c < kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, map, bar, c * 32, head, row0);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* dev_status) {
  const bool ok = mbar_wait_bounded(bar, parity, abort_flag, dev_status);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_swa_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ SwaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i][0], 128);
      mbar_init(&sm.p_full[i][1], 128);
      mbar_init(&sm.o_done[i], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
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

  // the work list is the prepass's: wait for it (programmatic dependent launch)
  griddep_wait();
  Units us;
  us.entries = a.entries;
  us.total = static_cast<long long>(a.hdr->num_entries) * a.Hq;
  us.G = gridDim.x;
  us.cta = blockIdx.x;
  us.Hq = a.Hq;
  us.group = a.Hq / a.Hkv;
  us.window = a.window;
  if (blockIdx.x >= us.total) {  // uniform over the CTA: no unit for it
    if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
    return;
  }

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      uint32_t nq = 0, nk = 0, nv = 0;  // Q pairs, K tiles and V tiles issued
      Unit x;
      bool ok = true;
      for (long long k = 0; ok && us.get(k, &x); ++k) {
        if (nq > 0 && !mbar_wait_bounded(&sm.q_empty, (nq - 1) & 1, abort_flag, dev_status)) break;
        mbar_arrive_expect_tx(&sm.q_full, x.has_q1 ? 2 * kTileBytes : kTileBytes);
        tma_tile(sm.q[0], &tq, &sm.q_full, x.head, x.q0);
        if (x.has_q1) tma_tile(sm.q[1], &tq, &sm.q_full, x.head, x.q0 + kBM);
        ++nq;
        for (int j = 0; j < x.nkv; ++j) {
          const int row0 = x.seg_start + (x.j0 + j) * kBN;
          const uint32_t sk = nk % kStages, sv = nv % kStages;
          if (nk >= kStages &&
              !mbar_wait_bounded(&sm.k_empty[sk], (nk / kStages - 1) & 1, abort_flag, dev_status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[sk], kTileBytes);
          tma_tile(sm.k[sk], &tk, &sm.k_full[sk], x.kv_head, row0);
          ++nk;
          if (nv >= kStages &&
              !mbar_wait_bounded(&sm.v_empty[sv], (nv / kStages - 1) & 1, abort_flag, dev_status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.v_full[sv], kTileBytes);
          tma_tile(sm.v[sv], &tv, &sm.v_full[sv], x.kv_head, row0);
          ++nv;
        }
      }
      // every copy issued lands before the CTA exits, aborted or not: the last use of each
      // ring stage
      if (nq > 0) mbar_wait_drain(&sm.q_full, (nq - 1) & 1);
      for (uint32_t s = 0; s < kStages; ++s) {
        if (nk > s) mbar_wait_drain(&sm.k_full[s], ((nk - 1 - s) / kStages) & 1);
        if (nv > s) mbar_wait_drain(&sm.v_full[s], ((nv - 1 - s) / kStages) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(kBM, kBN, false, false, a.scale_log2 < 0.0f);
      const uint32_t idesc_pv = make_idesc_bf16(kBM, kD, false, true, false);
      // descriptors: Q tile i starts i * kTileBytes after q[0]; ring stage s of K (V) starts
      // s * kTileBytes after k[0] (v[0])
      const uint64_t dq0 = qk_desc(smem_u32(sm.q[0])), dk0 = qk_desc(smem_u32(sm.k[0]));
      const uint64_t dv0 = pv_desc(smem_u32(sm.v[0]));
      constexpr uint64_t kTileStep = kTileBytes >> 4;
      auto issue_qk = [&](auto tile_c, uint32_t st) {
        constexpr int tile = decltype(tile_c)::value;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 1) * kChunkBytes + (kk & 1) * 32) >> 4);
          mma_ss(tmem + col_s(tile), dq0 + tile * kTileStep + off, dk0 + st * kTileStep + off, idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[tile]);
      };
      uint32_t nq = 0, kc = 0, vc = 0, pc0 = 0, pc1 = 0;
      // O_i (+)= P_i V for one key tile, each 64-key half as soon as the softmax stored it
      auto issue_pv = [&](auto tile_c, uint32_t sv, bool accumulate) {
        constexpr int tile = decltype(tile_c)::value;
        uint32_t& pc = tile == 0 ? pc0 : pc1;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait_bounded(&sm.p_full[tile][half], pc & 1, abort_flag, dev_status)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = half * 4; kk < half * 4 + 4; ++kk)
            mma_ts(tmem + col_o(tile), tmem + col_s(tile) + kk * 8,
                   dv0 + sv * kTileStep + static_cast<uint64_t>((kk * 1024) >> 4), idesc_pv,
                   (accumulate || kk > 0) ? 1u : 0u);
        }
        ++pc;
        mma_commit(&sm.o_done[tile]);
        return true;
      };
      using T0 = std::integral_constant<int, 0>;
      using T1 = std::integral_constant<int, 1>;
      Unit x;
      bool ok = true;
      for (long long k = 0; ok && us.get(k, &x); ++k, ++nq) {
        if (!mbar_wait_bounded(&sm.q_full, nq & 1, abort_flag, dev_status)) break;
        {
          const uint32_t st = kc % kStages;
          if (!mbar_wait_bounded(&sm.k_full[st], (kc / kStages) & 1, abort_flag, dev_status)) break;
          tc_fence_after();
          issue_qk(T0{}, st);  // tile 0 always sees the unit's first key tile
          if (x.has_q1 && x.first[1] == 0) issue_qk(T1{}, st);
          mma_commit(&sm.k_empty[st]);
          ++kc;
          if (x.nkv == 1) mma_commit(&sm.q_empty);
        }
        for (int j = 0; j < x.nkv; ++j, ++vc) {
          const uint32_t sv = vc % kStages;
          const bool more = j + 1 < x.nkv;
          const bool t1 = x.has_q1 && j >= x.first[1];  // tile 1 sees key tile j
          if (!mbar_wait_bounded(&sm.v_full[sv], (vc / kStages) & 1, abort_flag, dev_status)) { ok = false; break; }
          if (j <= x.last[0] && !issue_pv(T0{}, sv, j > 0)) { ok = false; break; }
          if (!t1) mma_commit(&sm.v_empty[sv]);
          const uint32_t st = kc % kStages;
          if (more) {
            if (!mbar_wait_bounded(&sm.k_full[st], (kc / kStages) & 1, abort_flag, dev_status)) { ok = false; break; }
            tc_fence_after();
            if (j + 1 <= x.last[0]) issue_qk(T0{}, st);
          }
          if (t1) {
            if (!issue_pv(T1{}, sv, j > x.first[1])) { ok = false; break; }
            mma_commit(&sm.v_empty[sv]);
          }
          if (more) {
            if (x.has_q1 && j + 1 >= x.first[1]) issue_qk(T1{}, st);
            mma_commit(&sm.k_empty[st]);
            ++kc;
            if (j + 2 == x.nkv) mma_commit(&sm.q_empty);
          }
        }
      }
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + col_s(wg), tO = tmem + lane_base + col_o(wg);
    const float c = fabsf(a.scale_log2);  // the sign of scale is in the QK descriptor
    uint32_t s_cnt = 0, o_base = 0;
    Unit x;
    for (long long k = 0; us.get(k, &x); ++k) {
      if (wg == 1 && !x.has_q1) continue;
      bool ok = true;
      const int i = x.q0 + wg * kBM + r;  // this thread's query row (token)
      const bool row_in = i < x.seg_end;
      // allowed keys of row i: [lo_i, i]; none for rows past the segment end
      const int lo_i = a.window > 0 ? max(x.seg_start, i - a.window + 1) : x.seg_start;
      float m = -INFINITY, l = 0.f;
      // (selected, not indexed by wg: an indexed read would put the unit in local memory)
      const int ja = wg ? x.first[1] : x.first[0], jb = wg ? x.last[1] : x.last[0];
      for (int j = ja; j <= jb; ++j) {
        if (!warp_wait(&sm.s_full[wg], s_cnt & 1, abort_flag, dev_status)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        const int kv0 = x.seg_start + (x.j0 + j) * kBN;
        // valid key columns [ka, kb) of this tile for this row
        const int ka = row_in ? max(lo_i - kv0, 0) : kBN;
        const int kb = row_in ? min(i - kv0 + 1, kBN) : 0;
        // tiles inside every row's allowed range (most of a window) skip the masking
        const bool need_mask = __any_sync(0xffffffffu, ka > 0 || kb < kBN);
        float pm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) pm[q] = -INFINITY;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t su[64];
          float* sf = reinterpret_cast<float*>(su);
          tmem_ld32(tS + half * 64, su);
          tmem_ld32(tS + half * 64 + 32, su + 32);
          tmem_ld_wait();
          reg_fence<64>(su);
          if (need_mask) {
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const int col = half * 64 + e;
              if (col < ka || col >= kb) sf[e] = -INFINITY;
            }
          }
#pragma unroll
          for (int e = 0; e < 64; e += 16) {
#pragma unroll
            for (int q = 0; q < 8; ++q) pm[q] = fmax3(pm[q], sf[e + q], sf[e + 8 + q]);
          }
        }
        const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]),
                               fmaxf(pm[6], pm[7]));
        const float mt = mx * c;
        float alpha = 1.f;
        if (mt > m + kRescaleThreshold) {  // never when the tile has no allowed key
          alpha = m == -INFINITY ? 0.f : ex2_approx(m - mt);
          m = mt;
        }
        // O holds this unit's earlier tiles from j = 1 on; S_j completing implies PV_{j-1}
        // has completed (one in-order MMA stream).  TMEM loads and stores are
        // warp-collective: the whole warp rescales when one of its rows needs it.
        if (j > ja && __any_sync(0xffffffffu, alpha != 1.f)) {
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int c0 = 0; c0 < kD; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_ld_wait();
            reg_fence<32>(o);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 y = fmul2(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
              o[e] = __float_as_uint(y.x);
              o[e + 1] = __float_as_uint(y.y);
            }
            tmem_st32(tO + c0, o);
          }
        }
        l *= alpha;
        const bool live = m != -INFINITY;
        const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t su[64];
          const float* sf = reinterpret_cast<const float*>(su);
          tmem_ld32(tS + half * 64, su);
          tmem_ld32(tS + half * 64 + 32, su + 32);
          tmem_ld_wait();
          reg_fence<64>(su);
          uint32_t p[32];
          float2 l2 = make_float2(0.f, 0.f);
          // Two copies of the loop: tiles inside every row's allowed range (most of them)
          // run one without the mask selects, which measured ~30% faster on the whole
          // kernel than a single loop testing need_mask per pair.  Every exponential
          // takes the MUFU: at head size 128 the tensor core's share of each key tile is
          // larger, the MUFU is not the limit, and the FMA-pipe polynomial of the vision
          // kernel only cost issue slots here.
          auto exps = [&](auto masked) {
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2) {
              const float2 tt = ffma2(make_float2(sf[2 * e2], sf[2 * e2 + 1]), c2, nm2);
              float2 pe = make_float2(ex2_approx(tt.x), ex2_approx(tt.y));
              if constexpr (decltype(masked)::value) {
                const int col = half * 64 + 2 * e2;
                if (!live || col < ka || col >= kb) pe.x = 0.f;
                if (!live || col + 1 < ka || col + 1 >= kb) pe.y = 0.f;
              }
              p[e2] = pack_bf16x2(pe.x, pe.y);
              // the row sum of the rounded weights the PV product uses
              l2 = fadd2(l2, make_float2(__uint_as_float(p[e2] << 16), __uint_as_float(p[e2] & 0xFFFF0000u)));
            }
          };
          if (need_mask) exps(std::true_type{});
          else exps(std::false_type{});
          l += l2.x + l2.y;
          tmem_st32(tS + half * 32, p);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&sm.p_full[wg][half]);
        }
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> HBM
      if (!warp_wait(&sm.o_done[wg], (o_base + (jb - ja)) & 1, abort_flag, dev_status)) break;
      o_base += jb - ja + 1;
      tc_fence_after();
      const float inv_l = 1.0f / l;
      uint8_t* row = static_cast<uint8_t*>(a.out) + (static_cast<size_t>(i) * a.Hq + x.head) * (kD * 2);
#pragma unroll
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c0, o);
        tmem_ld_wait();
        reg_fence<32>(o);
        if (row_in) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4*>(row + c0 * 2)[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      tc_fence_before();
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

size_t swa_smem_bytes() { return kSmemBytes; }

cudaError_t prepare_attn_swa() {
  return cudaFuncSetAttribute(attn_swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t launch_attn_swa(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const SwaArgs& args, int grid, cudaStream_t stream) {
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
  return cudaLaunchKernelEx(&cfg, attn_swa_kernel, tq, tk, tv, args);
}

}  // namespace vt
