// f32-input varlen attention forward on the tcgen05 tensor cores, by operand splitting.
//
// The exactness arm of the library (PR #1579, "Numerics, both halves": an f32 arm beside
// the bf16 one): the same block-diagonal softmax(Q_s K_s^T * scale) V_s as the bf16
// kernel, for f32 inputs and outputs, within 1e-5 of the exact result.  A bf16 factor
// keeps 8 significant bits, so every f32 operand x is split into three bf16 parts,
//     x0 = bf16(x),  x1 = bf16(x - x0),  x2 = bf16(x - x0 - x1)     (x ~ x0 + x1 + x2, 24 bits),
// and a product keeps the six part products of total order <= 2,
//     a b ~ a0 b0 + a0 b1 + a1 b0 + a0 b2 + a2 b0 + a1 b1,
// each a bf16 MMA (exact products, f32 accumulation in TMEM); the dropped terms are below
// 2^-24 of |a b|.  The MMAs are the bf16 kernel's forms (kind::f16, 64-byte swizzle).
// The tensor core's f32 accumulation loses more than round-to-nearest (measured: one S
// accumulator over all 36 MMAs put 1.5e-5 into O at scale -0.25), in proportion to the
// accumulator's magnitude and to the MMAs accumulated into it, so large sums are kept
// short: the big term a0 b0 of S goes into two accumulators of three K16 steps each and
// the five small terms into a third, added in f32 by the softmax; PV goes into a fresh
// accumulator per key tile, which the softmax folds into the running O in f32.
//
// One CTA (persistent) works through units of 128 query rows of one (segment, head); keys
// go by in tiles of 64.  Each key tile is serialised: this arm is about exactness, the
// bf16 kernel is the fast one.
//
//   warps 0-3 : load the f32 Q tile (once per unit) and each K and V tile from HBM with
//               coalesced 16-byte loads and write their three bf16 parts to shared memory
//               in the layout the MMA reads; then the softmax, one thread per query row:
//               S row from TMEM, exact f32 exp2 with the running max and row sum, O
//               rescaled in TMEM when the max moves, P split into three bf16 parts and
//               stored to TMEM; the epilogue O / l -> f32 -> HBM.
//   warp 4    : one thread issues, per key tile,
//                 S_b0 = Q_0 K_0^T over head columns 0-47, S_b1 over 48-95,
//                 S_x  = the five cross terms Q_i K_j^T     (SS, M128 N64, K16 steps)
//                 O_t  = sum of the six P_i V_j             (TS, M128 N96, K = 64)
//
// TMEM (512 columns allocated): S_b0 [0,64), S_b1 [64,128), S_x [128,192), P parts
// [192,224) [224,256) [256,288), O_t [288,384), running O [384,480).
// Keys past a segment's end get p = 0; query rows past it are computed but not stored.
// Every mbarrier wait is bounded and an abort flag lets all roles leave together.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

constexpr int kBM = kF32BlockRows;  // 128 query rows per unit
constexpr int kBN = 64;             // keys per tile
constexpr int kD = 96;
constexpr int kUnitsPerRow = kD / 8;             // 16-byte units (8 bf16) per row: 12
constexpr int kQChunk = kBM * 64;                // 8 KB: 128 rows x 32 bf16
constexpr int kKVChunk = kBN * 64;               // 4 KB: 64 rows x 32 bf16
constexpr int kQPart = 3 * kQChunk;              // 24 KB
constexpr int kKVPart = 3 * kKVChunk;            // 12 KB
constexpr int kThreads = 160;
constexpr int kWarpMma = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColSb0 = 0, kColSb1 = 64, kColSx = 128;  // S accumulators
constexpr uint32_t kColP = 192;                                // P part i at kColP + 32 i
constexpr uint32_t kColOt = 288, kColO = 384;                  // this tile's PV; running O
// the six (i, j) part pairs of total order <= 2: (0,0) (0,1) (1,0) (0,2) (2,0) (1,1)
__host__ __device__ constexpr int pair_a(int c) { return c == 2 || c == 5 ? 1 : c == 4 ? 2 : 0; }
__host__ __device__ constexpr int pair_b(int c) { return c == 1 || c == 5 ? 1 : c == 3 ? 2 : 0; }

struct Smem {
  uint8_t q[3][kQPart];
  uint8_t k[3][kKVPart];
  uint8_t v[3][kKVPart];
  uint64_t q_ready, kv_ready;  // parts written (128 arrivals each)
  uint64_t s_full, p_full;     // S computed; P stored (128 arrivals)
  uint64_t o_done;             // the PV of a key tile (and everything before it) completed
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

struct Unit {
  int head, q0, seg_start, seg_end, nkv;
};

// This CTA's units in the bf16 kernel's order: a snake over the CTAs, entry-major (longest
// segment first) when the segments differ in length and head-major when they do not.
struct Units {
  const WorkEntry* entries;
  long long total, G, cta;
  int E, H;
  bool entry_major;
  __device__ bool get(long long k, Unit* x) const {
    const long long u = k * G + ((k & 1) ? G - 1 - cta : cta);
    if (u >= total) return false;
    const int e = static_cast<int>(entry_major ? u / H : u % E);
    x->head = static_cast<int>(entry_major ? u % H : u / E);
    const WorkEntry we = entries[e];
    x->seg_start = we.seg_start;
    x->seg_end = we.seg_end;
    x->q0 = we.seg_start + we.qblock * kBM;
    x->nkv = (we.seg_end - we.seg_start + kBN - 1) / kBN;
    return true;
  }
};

// The three bf16 parts of x (round to nearest even at each step).
__device__ __forceinline__ void split3(float x, __nv_bfloat16& p0, __nv_bfloat16& p1,
                                       __nv_bfloat16& p2) {
  p0 = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(p0);
  p1 = __float2bfloat16_rn(r1);
  p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
}
__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

// Rows [row0, row0 + rows) of head h of an f32 [T, H, 96] tensor -> three bf16 part tiles
// in the MMA layout: three 32-column chunks of rows x 64 bytes, 16-byte unit u of row r
// stored at unit u ^ ((r >> 1) & 3) (64-byte swizzle).  Rows at or past T are zeros.
// Thread t of the 128 takes units t, t + 128, ... (12 per row: consecutive threads read
// consecutive 32-byte pieces of a row).
template <int kRows>
__device__ __forceinline__ void load_parts(const float* __restrict__ src, int T, int H, int h, int row0,
                                           uint8_t* part0, int part_stride, int t) {
  constexpr int kChunk = kRows * 64;
#pragma unroll 2
  for (int idx = t; idx < kRows * kUnitsPerRow; idx += 128) {
    const int r = idx / kUnitsPerRow, u = idx - r * kUnitsPerRow;
    const int row = row0 + r;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (row < T) {
      const float4* p = reinterpret_cast<const float4*>(src + (static_cast<size_t>(row) * H + h) * kD + u * 8);
      a = __ldg(p);
      b = __ldg(p + 1);
    }
    const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t w0[4], w1[4], w2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat16 e0, e1, e2, o0, o1, o2;
      split3(x[2 * i], e0, e1, e2);
      split3(x[2 * i + 1], o0, o1, o2);
      w0[i] = pack2(e0, o0);
      w1[i] = pack2(e1, o1);
      w2[i] = pack2(e2, o2);
    }
    const int off = (u >> 2) * kChunk + r * 64 + (((u & 3) ^ ((r >> 1) & 3)) << 4);
    *reinterpret_cast<uint4*>(part0 + off) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4*>(part0 + part_stride + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    *reinterpret_cast<uint4*>(part0 + 2 * part_stride + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
  }
}

// K-major operand (Q or K): 8-row groups 512 B apart; K16 step kk starts 32 B into the
// 64-byte rows of chunk kk / 2.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
  return make_smem_desc(saddr, 16, 512, kSwizzle64B);
}
__device__ __forceinline__ uint64_t kstep(int kk, int chunk_bytes) {
  return static_cast<uint64_t>(((kk >> 1) * chunk_bytes + (kk & 1) * 32) >> 4);
}
// V as the MN-major B operand of PV (N = 96 head columns, K = 64 keys): 8-key groups
// 512 B apart (SBO), 32-column chunks 4 KB apart (LBO); K16 step = 16 keys = 1024 B.
__device__ __forceinline__ uint64_t v_desc(uint32_t saddr) {
  return make_smem_desc(saddr, kKVChunk, 512, kSwizzle64B);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* dev_status) {
  const bool ok = mbar_wait_bounded(bar, parity, abort_flag, dev_status);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1) attn_f32split_kernel(const __grid_constant__ F32Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  Units us;
  us.entries = a.entries;
  us.E = a.hdr->num_entries;
  us.H = a.H;
  us.total = static_cast<long long>(us.E) * a.H;
  us.G = gridDim.x;
  us.cta = blockIdx.x;
  us.entry_major = a.hdr->order != 0;
  if (blockIdx.x >= us.total) return;  // uniform over the CTA

  if (tid == 0) {
    mbar_init(&sm.q_ready, 128);
    mbar_init(&sm.kv_ready, 128);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, 128);
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int* dev_status = a.dev_status;

  if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(kBM, kBN, false, false, false);
      const uint32_t idesc_pv = make_idesc_bf16(kBM, kD, false, true, false);
      uint64_t dq[3], dk[3], dv[3];
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        dq[i] = kmajor_desc(smem_u32(sm.q[i]));
        dk[i] = kmajor_desc(smem_u32(sm.k[i]));
        dv[i] = v_desc(smem_u32(sm.v[i]));
      }
      uint32_t t = 0, n = 0;
      Unit x;
      bool ok = true;
      for (long long k = 0; ok && us.get(k, &x); ++k, ++n) {
        if (!mbar_wait_bounded(&sm.q_ready, n & 1, abort_flag, dev_status)) break;
        for (int j = 0; j < x.nkv; ++j, ++t) {
          if (!mbar_wait_bounded(&sm.kv_ready, t & 1, abort_flag, dev_status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)  // big term, two accumulators of three steps
            mma_ss(tmem + (kk < 3 ? kColSb0 : kColSb1), dq[0] + kstep(kk, kQChunk),
                   dk[0] + kstep(kk, kKVChunk), idesc_qk, (kk % 3) > 0 ? 1u : 0u);
#pragma unroll
          for (int c = 1; c < 6; ++c) {         // the five cross terms
            const uint64_t qa = dq[pair_a(c)], kb = dk[pair_b(c)];
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
              mma_ss(tmem + kColSx, qa + kstep(kk, kQChunk), kb + kstep(kk, kKVChunk), idesc_qk,
                     (c > 1 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sm.s_full);
          if (!mbar_wait_bounded(&sm.p_full, t & 1, abort_flag, dev_status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            const uint32_t pa = tmem + kColP + 32 * pair_a(c);
            const uint64_t vb = dv[pair_b(c)];
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
              mma_ts(tmem + kColOt, pa + kk * 8, vb + static_cast<uint64_t>((kk * 1024) >> 4), idesc_pv,
                     (c > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sm.o_done);
        }
      }
      // all MMAs issued by this thread complete before TMEM is released
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ operands + softmax
    const int r = tid;  // query row of the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tRow = tmem + lane_base;
    const float c = a.scale_log2;  // signed
    // O = alpha O + O_t, in f32 (first tile of a unit: O = O_t); warp-collective
    auto fold = [&](float alpha, bool first) {
#pragma unroll
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t o[32], ot[32];
        tmem_ld32(tRow + kColOt + c0, ot);
        if (!first) tmem_ld32(tRow + kColO + c0, o);
        tmem_ld_wait();
        reg_fence<32>(ot);
        reg_fence<32>(o);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          o[i] = __float_as_uint(first ? __uint_as_float(ot[i])
                                       : fmaf(alpha, __uint_as_float(o[i]), __uint_as_float(ot[i])));
        tmem_st32(tRow + kColO + c0, o);
      }
      tmem_st_wait();
    };
    uint32_t t = 0;
    Unit x;
    for (long long k = 0; us.get(k, &x); ++k) {
      bool ok = true;
      // every MMA of the previous unit completed (its epilogue waited for that): Q is free
      load_parts<kBM>(a.q, a.T, a.H, x.head, x.q0, sm.q[0], kQPart, r);
      fence_proxy_async_smem();
      mbar_arrive(&sm.q_ready);
      float m = -INFINITY, l = 0.f, alpha_prev = 1.f;
      for (int j = 0; j < x.nkv; ++j, ++t) {
        if (j > 0) {
          // PV of the previous key tile completed: fold it into O; K and V parts are free
          if (!warp_wait(&sm.o_done, (t - 1) & 1, abort_flag, dev_status)) { ok = false; break; }
          tc_fence_after();
          fold(alpha_prev, j == 1);
        }
        const int row0 = x.seg_start + j * kBN;
        load_parts<kBN>(a.k, a.T, a.H, x.head, row0, sm.k[0], kKVPart, r);
        load_parts<kBN>(a.v, a.T, a.H, x.head, row0, sm.v[0], kKVPart, r);
        fence_proxy_async_smem();
        mbar_arrive(&sm.kv_ready);
        if (!warp_wait(&sm.s_full, t & 1, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        const int nvalid = x.seg_end - row0;  // >= 1
        float sv[kBN];
        float mx = -INFINITY;
#pragma unroll
        for (int h32 = 0; h32 < kBN; h32 += 32) {  // S = (S_b0 + S_b1) + S_x, 32 keys at a time
          uint32_t b0[32], b1[32], sx[32];
          tmem_ld32(tRow + kColSb0 + h32, b0);
          tmem_ld32(tRow + kColSb1 + h32, b1);
          tmem_ld32(tRow + kColSx + h32, sx);
          tmem_ld_wait();
          reg_fence<32>(b0);
          reg_fence<32>(b1);
          reg_fence<32>(sx);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sum = (__uint_as_float(b0[i]) + __uint_as_float(b1[i])) + __uint_as_float(sx[i]);
            sv[h32 + i] = h32 + i < nvalid ? sum * c : -INFINITY;
            mx = fmaxf(mx, sv[h32 + i]);
          }
        }
        const float m_new = fmaxf(m, mx);
        alpha_prev = j > 0 ? exp2f(m - m_new) : 1.f;  // scales O and l from earlier tiles
        l *= alpha_prev;
        m = m_new;
        uint32_t p0[kBN / 2], p1[kBN / 2], p2[kBN / 2];
#pragma unroll
        for (int i = 0; i < kBN / 2; ++i) {
          const float pe = exp2f(sv[2 * i] - m), po = exp2f(sv[2 * i + 1] - m);  // 0 past the end
          l += pe + po;
          __nv_bfloat16 e0, e1, e2, o0, o1, o2;
          split3(pe, e0, e1, e2);
          split3(po, o0, o1, o2);
          p0[i] = pack2(e0, o0);
          p1[i] = pack2(e1, o1);
          p2[i] = pack2(e2, o2);
        }
        tmem_st32(tRow + kColP, p0);
        tmem_st32(tRow + kColP + 32, p1);
        tmem_st32(tRow + kColP + 64, p2);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sm.p_full);
      }
      if (!ok) break;
      // epilogue: fold the last tile, then O / l -> f32 -> HBM (rows inside the segment only)
      if (!warp_wait(&sm.o_done, (t - 1) & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      fold(alpha_prev, x.nkv == 1);
      const int row_tok = x.q0 + r;
      const float inv_l = 1.0f / l;
      float* row = a.out + (static_cast<size_t>(row_tok) * a.H + x.head) * kD;
#pragma unroll
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tRow + kColO + c0, o);
        tmem_ld_wait();
        reg_fence<32>(o);
        if (row_tok < x.seg_end) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(row + c0 + i) =
                make_float4(__uint_as_float(o[i]) * inv_l, __uint_as_float(o[i + 1]) * inv_l,
                            __uint_as_float(o[i + 2]) * inv_l, __uint_as_float(o[i + 3]) * inv_l);
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

size_t f32_smem_bytes() { return kSmemBytes; }

cudaError_t prepare_attn_f32() {
  return cudaFuncSetAttribute(attn_f32split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t launch_attn_f32(const F32Args& args, int grid, cudaStream_t stream) {
  attn_f32split_kernel<<<grid, kThreads, kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace vt
