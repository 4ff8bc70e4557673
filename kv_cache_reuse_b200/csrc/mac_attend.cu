// mac_attend.cu -- Amend, Complete, miss fallback and the stable merge.
//
// "MAC-Attention: a Match-Amend-Complete Scheme for Fast and Accurate
// Attention Computation", page 1 (abstract): on a hit the amend stage
// corrects the reused attention by recomputing a small band of keys next to
// the match boundary, and the complete stage combines that result with fresh
// attention over the KV tail in a numerically stable merge; on a miss the
// step is split-KV decode attention over every key.  All three are
// the same computation -- attention of the current query group over a key
// range -- so one persistent kernel runs them over a flattened list of work
// items built by the match kernel.  A unit (sequence, KV head) with few fresh
// keys (every hit) is one whole item, done end to end by one CTA; a longer
// one is two split items,
//   [start, c_t)  -> folded into the unit's new prefix state
//   [c_t, p_t]    -> folded into the output only,
// cut wherever the CTAs' ranges cut them.  The items are laid end to end in a
// cost space (keys plus a fixed cost per item) split over the CTAs evenly, or
// on large steps in proportion to each SM's learned streaming rate, so a mix
// of hits (a few hundred keys) and misses (the whole context) keeps every SM
// equally busy.  With per-head matching each head masks the keys of the
// amend range below its own reuse boundary.
//
// Per CTA: eight warps; warp w owns boxes w, w+8, w+16, ... of every piece,
// where a box is 16 keys (it never crosses a page).  Each warp streams its
// own boxes through its own ring of shared-memory slots with TMA
// (cp.async.bulk.tensor, 128-byte swizzle, each CTA its own copies), keeping NST boxes
// in flight, so the warps never wait on one another inside a piece.
//
// A box is a small dense product on the tensor cores (mma.sync m16n8k16,
// bf16 in, fp32 accumulate), keys on the M side:
//   S^T[16 keys x 8] = K[16 x D] . Qx[D x 8]     (QK, D/16 k-steps)
//   O^T[D x 8]      += V^T[D x 16] . Px[16 x 8]  (PV, D/16 row tiles)
// The fp32 query (and the fp32 softmax weights) is split into a bf16 high
// part and a bf16 residual, so the products keep ~16 mantissa bits.  With up
// to 4 query heads per KV head the 8 columns are the group twice (high parts,
// then residuals; score = column h + column h+4; heads past the group are
// zero columns); with 5 to 8 heads each head has one column and the high and
// residual parts are two products into the same accumulator.  This is not
// about tensor throughput -- the work is HBM-bound (G flop per byte of K/V
// for G query heads) -- but about instruction issue: a box costs ~100 warp
// instructions instead of ~700 on the FP32 pipes, which keeps the miss path
// on the memory roofline and a hit's few boxes short.  K fragments come from
// ldmatrix, V^T fragments from ldmatrix.trans (the swizzle keeps both
// conflict-free); the weights reach their B-fragment layout through 64 bytes
// per head of shared memory per warp.
//
// Softmax runs in exp2 units (the query is pre-scaled by log2(e)/sqrt(D)).
// A whole item ends in the CTA: reused ring state (+) amend -> new ring
// entry, (+) tail -> out, lse.  A split piece ends in a partial (o
// unnormalised, m, l); the CTA that delivers a unit's last partial (atomic
// counter, no waiting) merges the reused state and the partials the same
// way.  The window's stored outputs are fp32 or bf16.
//
// Every wait is bounded (2 s on %globaltimer): on expiry the kernel sets
// MAC_DEV_TIMEOUT in the status word and leaves without hanging the GPU.
#include <limits.h>
#include <math.h>
#include <stdint.h>

#include <cuda_bf16.h>

#include "mac_internal.cuh"
#include "mac_match_dev.cuh"
#include "mac_attend_dev.cuh"

#include "../../include/mac.h"

namespace mac {
namespace {

constexpr int kRateMinBoxes = 256;  // a CTA's rate record needs this much streaming

// GP: the query group padded to 4 or 8 heads.  GP = 4 puts each head in
// two tile columns (bf16 high part, bf16 residual); GP = 8 gives each head
// one column and runs the high and residual parts as two products into the
// same accumulator.  The real group G = p.G <= GP sets the global layouts.
template <int D, int GP>
struct Cfg {
  static constexpr int KS = D / 16;               // k-steps of QK = row tiles of PV
  static constexpr int HALVES = D / 64;           // 128-byte swizzled halves of a key row
  static constexpr int NST = GP == 4 ? (D == 128 ? 3 : 6) : (D == 128 ? 2 : 4);  // boxes in flight per warp
  static constexpr int NQ = NST + 1;              // query buffers (pieces the issue cursor can be ahead)
  static constexpr int GD = GP * D;               // floats of a padded query group
  static constexpr int SF = GP * D + 2 * GP;      // a warp's state: o [GP][D], m [GP], l [GP]
  static constexpr int PB = kSubKeys * GP;        // floats of one weights exchange buffer
  static constexpr int WB = SF > 2 * PB ? SF : 2 * PB;  // per-warp scratch floats
  static constexpr int QW = GP == 4 ? 2 : 4;      // query B-fragment registers per k-step
  static_assert(WB % 4 == 0 && (NQ * GD) % 4 == 0, "warp slots hold 16-byte aligned runs");
};

template <int D, int GP>
struct __align__(1024) AttnSmem {
  using C = Cfg<D, GP>;
  // per warp: ring of (K box, V box), each [HALVES][16 keys][64 dims] bf16, 128-byte swizzle
  uint16_t kv[kConsumerWarps][C::NST][2][kSubKeys * D];
  float q[C::NQ][C::GD];              // queries of the upcoming pieces (heads >= G unused)
  float wbuf[kConsumerWarps][C::WB];  // weights exchange / piece combine
  unsigned long long full[kConsumerWarps][C::NST];
  unsigned long long empty[kConsumerWarps][C::NST];  // chunked groups: a box slot's C readers are done
  unsigned long long qfull[C::NQ];
  unsigned long long csync;
  unsigned long long rfull;          // reused ring state of the current whole-unit piece landed
  int abort_flag;
  int last_flag;
  int box_total;                     // boxes consumed by all warps (rate record)
  Segment items[kItemCache];         // the CTA's work items, from its first one on
  int nlocal;                        // one-launch step: whole units this CTA matched (in items)
  alignas(16) float ring[C::SF];     // that ring state: o [G][D], then m at GD, l at GD + GP
};

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D += A(16x16, row) . B(16x8, col), bf16 in, fp32 accumulate
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Byte offset of (key row, dim) in a box of [D/64][16][64] bf16 laid out by
// TMA with the 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r & 7).
__device__ __forceinline__ uint32_t box_off(int row, int dim) {
  return (uint32_t)((dim >> 6) * (kSubKeys * 128) + row * 128 + ((((dim >> 3) & 7) ^ (row & 7)) << 4) +
                    (dim & 7) * 2);
}

// The group size: GF when the kernel is built for one group size (4 or 8),
// else the run-time value (padded to GP in registers and shared memory).
template <int GF>
__device__ __forceinline__ int group_of(const AttendParams& p) {
  return GF > 0 ? GF : p.G;
}
// m and l of a ring entry are G-float runs at a multiple of G floats: bulk
// copies need 16-byte runs, so only groups of 4 and 8 move them that way.
template <int GF>
constexpr bool kBulkML = GF > 0 && GF % 4 == 0;


// ------------------------------------------------------------ consumer state
// Per warp, in mma fragment layout (lane = 4*gid + tig): the query columns
// as B fragments, O^T as C fragments (dims 16*dt + gid and + 8, columns
// 2*tig and 2*tig + 1), and the running max and sum of the two heads this
// lane's columns belong to, hh and hh + 1 (GP = 4: hh = 2*(tig & 1);
// GP = 8: hh = 2*tig).
template <int D, int GP>
struct Acc {
  uint32_t qb[Cfg<D, GP>::KS][Cfg<D, GP>::QW];
  float o[Cfg<D, GP>::KS][4];
  float m[2];
  float l[2];
};

// Load the query of a piece into B fragments.  GP = 4: column n = gid is
// head (gid & 3), its bf16 high part for gid < 4 and its bf16 residual
// otherwise.  GP = 8: column n = gid is head gid; qb[ks][0..1] hold the high
// parts, qb[ks][2..3] the residuals.  Heads >= G are zero columns.
template <int D, int GP>
__device__ __forceinline__ void load_query(Acc<D, GP>& A, const float* qs, int G) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int head = GP == 4 ? (gid & 3) : gid;
  const bool live = head < G;
  const float* qh = qs + head * D + 2 * tig;
#pragma unroll
  for (int ks = 0; ks < Cfg<D, GP>::KS; ++ks) {
    const float2 z = make_float2(0.f, 0.f);
    const float2 x01 = live ? *reinterpret_cast<const float2*>(qh + ks * 16) : z;
    const float2 x89 = live ? *reinterpret_cast<const float2*>(qh + ks * 16 + 8) : z;
    const uint32_t h0 = pack_bf16(x01.x, x01.y), h1 = pack_bf16(x89.x, x89.y);
    if constexpr (GP == 4) {
      A.qb[ks][0] = gid < 4 ? h0 : pack_bf16_residual(x01.x, x01.y, h0);
      A.qb[ks][1] = gid < 4 ? h1 : pack_bf16_residual(x89.x, x89.y, h1);
    } else {
      A.qb[ks][0] = h0;
      A.qb[ks][1] = h1;
      A.qb[ks][2] = pack_bf16_residual(x01.x, x01.y, h0);
      A.qb[ks][3] = pack_bf16_residual(x89.x, x89.y, h1);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) A.o[ks][i] = 0.f;
  }
  A.m[0] = A.m[1] = -INFINITY;
  A.l[0] = A.l[1] = 0.f;
}

// One 16-key box for one warp.  A box at the edge of its range (masked) has
// rows outside [k0, k1): their scores become -inf and their V rows are
// zeroed in shared memory (the rows may hold anything, NaN included, and
// 0 * NaN would poison the sum).
//
// PH (per-head matching): key rows below lo0 / lo1 are outside the ranges of
// this lane's heads hh / hh + 1 (inside their reused states): their scores
// become -inf for that head only (the rows are valid keys of the range).
template <int D, int GP, bool PH>
__device__ __forceinline__ void process_box(Acc<D, GP>& A, const uint16_t* kbox, uint16_t* vbox, float* pbuf,
                                            int key_box, int k0, int k1, bool masked, int lo0, int lo1) {
  constexpr int KS = Cfg<D, GP>::KS;
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int mj = lane >> 3, mr = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const uint32_t kb = smem_u32(kbox), vb = smem_u32(vbox);

  // S^T = K . Qx, two accumulator chains (GP = 4: alternate k-steps;
  // GP = 8: high parts into s, residuals into t)
  float s[4] = {0.f, 0.f, 0.f, 0.f}, t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(kb + box_off(mr + ((mj & 1) << 3), ks * 16 + ((mj >> 1) << 3)), a0, a1, a2, a3);
    if constexpr (GP == 4) {
      mma16816((ks & 1) ? t : s, a0, a1, a2, a3, A.qb[ks][0], A.qb[ks][1]);
    } else {
      mma16816(s, a0, a1, a2, a3, A.qb[ks][0], A.qb[ks][1]);
      mma16816(t, a0, a1, a2, a3, A.qb[ks][2], A.qb[ks][3]);
    }
  }
  // sc = (key gid, head hh), (gid, hh + 1), (gid + 8, hh), (gid + 8, hh + 1);
  // GP = 4: lanes tig and tig ^ 2 hold the high and residual columns
  float sc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sc[i] = s[i] + t[i];
    if constexpr (GP == 4) sc[i] += __shfl_xor_sync(kFull, sc[i], 2);
  }
  if (masked) {
    const int ka = key_box + gid, kc = ka + 8;
    if (ka < k0 || ka >= k1) sc[0] = sc[1] = -INFINITY;
    if (kc < k0 || kc >= k1) sc[2] = sc[3] = -INFINITY;
    // zero whole V rows (both halves) outside the range
    for (int i = lane; i < Cfg<D, GP>::HALVES * kSubKeys * 8; i += 32) {
      const int row = (i >> 3) & (kSubKeys - 1);
      if (key_box + row < k0 || key_box + row >= k1) reinterpret_cast<uint4*>(vbox)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if constexpr (PH) {
    const int ka = key_box + gid, kc = ka + 8;
    if (ka < lo0) sc[0] = -INFINITY;
    if (ka < lo1) sc[1] = -INFINITY;
    if (kc < lo0) sc[2] = -INFINITY;
    if (kc < lo1) sc[3] = -INFINITY;
  }
  // box max per head over its 16 keys (rows gid and gid + 8 of every lane)
  float bm0 = fmaxf(sc[0], sc[2]), bm1 = fmaxf(sc[1], sc[3]);
#pragma unroll
  for (int off = 4; off <= 16; off <<= 1) {
    bm0 = fmaxf(bm0, __shfl_xor_sync(kFull, bm0, off));
    bm1 = fmaxf(bm1, __shfl_xor_sync(kFull, bm1, off));
  }
  const float mn0 = fmaxf(A.m[0], bm0), mn1 = fmaxf(A.m[1], bm1);
  if (__any_sync(kFull, mn0 > A.m[0] || mn1 > A.m[1])) {
    const float a0 = ex2(A.m[0] - (mn0 == -INFINITY ? 0.f : mn0));
    const float a1 = ex2(A.m[1] - (mn1 == -INFINITY ? 0.f : mn1));
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      A.o[dt][0] *= a0;
      A.o[dt][1] *= a1;
      A.o[dt][2] *= a0;
      A.o[dt][3] *= a1;
    }
    A.l[0] *= a0;
    A.l[1] *= a1;
    A.m[0] = mn0;
    A.m[1] = mn1;
  }
  const float mu0 = A.m[0] == -INFINITY ? 0.f : A.m[0], mu1 = A.m[1] == -INFINITY ? 0.f : A.m[1];
  const float p0 = ex2(sc[0] - mu0), p1 = ex2(sc[1] - mu1), p2 = ex2(sc[2] - mu0), p3 = ex2(sc[3] - mu1);
  A.l[0] += p0 + p2;
  A.l[1] += p1 + p3;
  // weights P[key][head] ([16][GP] floats) through shared memory into the
  // B fragments of Px: b0 = keys 2*tig, 2*tig + 1; b1 = keys 2*tig + 8, + 9;
  // column gid
  const int hh = GP == 4 ? 2 * (tig & 1) : 2 * tig;
  if (GP == 8 || tig < 2) {
    *reinterpret_cast<float2*>(pbuf + gid * GP + hh) = make_float2(p0, p1);
    *reinterpret_cast<float2*>(pbuf + (gid + 8) * GP + hh) = make_float2(p2, p3);
  }
  __syncwarp();
  const int hc = GP == 4 ? (gid & 3) : gid;
  const float x0 = pbuf[(2 * tig) * GP + hc], x1 = pbuf[(2 * tig + 1) * GP + hc];
  const float x2 = pbuf[(2 * tig + 8) * GP + hc], x3 = pbuf[(2 * tig + 9) * GP + hc];
  const uint32_t h0 = pack_bf16(x0, x1), h1 = pack_bf16(x2, x3);
  // O^T += V^T . Px, one row tile of 16 dims per mma (GP = 8: the high and
  // the residual weights, two products into the same accumulator)
  if constexpr (GP == 4) {
    const uint32_t pb0 = gid < 4 ? h0 : pack_bf16_residual(x0, x1, h0);
    const uint32_t pb1 = gid < 4 ? h1 : pack_bf16_residual(x2, x3, h1);
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(vb + box_off(mr + ((mj >> 1) << 3), dt * 16 + ((mj & 1) << 3)), a0, a1, a2, a3);
      mma16816(A.o[dt], a0, a1, a2, a3, pb0, pb1);
    }
  } else {
    const uint32_t r0 = pack_bf16_residual(x0, x1, h0), r1 = pack_bf16_residual(x2, x3, h1);
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(vb + box_off(mr + ((mj >> 1) << 3), dt * 16 + ((mj & 1) << 3)), a0, a1, a2, a3);
      mma16816(A.o[dt], a0, a1, a2, a3, h0, h1);
      mma16816(A.o[dt], a0, a1, a2, a3, r0, r1);
    }
  }
}

// Bounded barrier of the 8 consumer warps (mbarrier with one arrival per warp).
template <typename SM>
__device__ __forceinline__ bool consumer_sync(SM& sm, uint32_t& phase, unsigned* status) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.csync);
  const bool ok = mbar_wait(&sm.csync, phase, &sm.abort_flag, status);
  phase ^= 1u;
  __syncwarp();
  return ok;
}

template <int D, int GP, int NH, typename SM>
__device__ __forceinline__ void combine_warps2(const SM& sm, int wA, int idx, int h, float& MA,
                                               float& LA, float& OA, float& MB, float& LB, float& OB);


// Store the warp's state in its shared-memory slot: o [GP][D] unnormalised,
// then m [GP] and l [GP].  GP = 4: lanes tig and tig ^ 2 hold the high and
// residual columns of the same heads.  Lanes of one tig hold different key
// rows for l.
template <int D, int GP>
__device__ __forceinline__ void warp_combine_store(Acc<D, GP>& A, float* wb) {
  constexpr int GD = Cfg<D, GP>::GD, KS = Cfg<D, GP>::KS;
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int hh = GP == 4 ? 2 * (tig & 1) : 2 * tig;
  __syncwarp();
  float l0 = A.l[0], l1 = A.l[1];
#pragma unroll
  for (int off = 4; off <= 16; off <<= 1) {
    l0 += __shfl_xor_sync(kFull, l0, off);
    l1 += __shfl_xor_sync(kFull, l1, off);
  }
  if constexpr (GP == 4) {
#pragma unroll
    for (int dt = 0; dt < KS; ++dt)
#pragma unroll
      for (int i = 0; i < 4; ++i) A.o[dt][i] += __shfl_xor_sync(kFull, A.o[dt][i], 2);
  }
  if (GP == 8 || tig < 2) {
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const int d0 = dt * 16 + gid;
      wb[hh * D + d0] = A.o[dt][0];
      wb[(hh + 1) * D + d0] = A.o[dt][1];
      wb[hh * D + d0 + 8] = A.o[dt][2];
      wb[(hh + 1) * D + d0 + 8] = A.o[dt][3];
    }
    if (gid == 0) {
      wb[GD + hh] = A.m[0];
      wb[GD + hh + 1] = A.m[1];
      wb[GD + GP + hh] = l0;
      wb[GD + GP + hh + 1] = l1;
    }
  }
}

// Merge the warps' states for element idx of head h, from slots laid out as
// o [NH][D], m [NH], l [NH]: warps below wA into (MA, LA, OA), the others
// into (MB, LB, OB); sums relative to 2^M.
template <int D, int GP, int NH, typename SM>
__device__ __forceinline__ void combine_warps2(const SM& sm, int wA, int idx, int h, float& MA,
                                               float& LA, float& OA, float& MB, float& LB, float& OB) {
  float m[kConsumerWarps], l[kConsumerWarps], o[kConsumerWarps];
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) {
    m[w] = sm.wbuf[w][NH * D + h];
    l[w] = sm.wbuf[w][NH * D + NH + h];
    o[w] = sm.wbuf[w][idx];
  }
  MA = MB = -INFINITY;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) {
    if (w < wA) MA = fmaxf(MA, m[w]);
    else MB = fmaxf(MB, m[w]);
  }
  const float MAu = MA == -INFINITY ? 0.f : MA, MBu = MB == -INFINITY ? 0.f : MB;
  LA = OA = LB = OB = 0.f;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) {
    const float a = ex2(m[w] - (w < wA ? MAu : MBu));
    if (w < wA) {
      LA += l[w] * a;
      OA += o[w] * a;
    } else {
      LB += l[w] * a;
      OB += o[w] * a;
    }
  }
}

// Finish of a unit from the eight warps' states in their shared-memory
// slots: warps [0, wA) hold set A (the amend range, or segment A's
// partials), warps [wA, 8) set B (the tail).  With a reused state (heads in
// hmask; o, m and l on chip in sm.ring) S = reused + A, else S = A; S is the
// unit's new ring entry in slot dst and S + B its output.
//
// Chunked groups (NC > 1, G = 8 NC heads per KV head): the call finishes the
// 8 heads of chunk ch, whose states the warps' slots and sm.ring hold; the
// global layouts are those of the whole group.
template <int D, int GP, int GF, int NC = 1, typename SM>
__device__ __forceinline__ void unit_epilogue(const AttendParams& p, SM& sm, int u, int wA, int hit,
                                              int hmask, int dst, int end, int ch = 0) {
  constexpr int GDP = Cfg<D, GP>::GD;
  const int G = NC > 1 ? GP : group_of<GF>(p), GD = G * D;  // heads of this call, and their elements
  const int Gt = NC > 1 ? GF : G, h0 = NC > 1 ? ch * GP : 0;  // heads of the unit; first head of the call
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  const int Wp1 = p.W + 1;
  constexpr int PER = (GDP + kConsumerWarps * 32 - 1) / (kConsumerWarps * 32);
  // cold code once per piece: a rolled loop fetches fewer instruction lines
#pragma unroll 1
  for (int k = 0; k < PER; ++k) {
    const int idx = threadIdx.x + k * kConsumerWarps * 32;
    if (idx >= GD) break;
    const int h = idx / D, d = idx - h * D;
    float MA, LA, OA, MB, LB, OB;
    combine_warps2<D, GP, GP>(sm, wA, idx, h, MA, LA, OA, MB, LB, OB);
    // new prefix state S = reused (hit) + amend
    const bool hh = hit && ((hmask >> h) & 1);
    const float rm = hh ? sm.ring[GDP + h] * kLog2e : -INFINITY;
    float M = fmaxf(MA, rm);
    const float Mu = M == -INFINITY ? 0.f : M;
    const float aA = ex2(MA - Mu);
    float L = LA * aA, O = OA * aA;
    if (hh) {
      const float a = ex2(rm - Mu), rl = sm.ring[GDP + GP + h];
      L += rl * a;
      O += ring_o_at(sm.ring, idx, p.ring_bf16) * rl * a;
    }
    const size_t ds = (size_t)u * Wp1 + dst;
    ring_o_put(p.ring_o, (ds * Gt + h0) * D + idx, L > 0.f ? __fdividef(O, L) : 0.f, p.ring_bf16);
    if (d == 0) {
      p.ring_m[ds * Gt + h0 + h] = L > 0.f ? M * kLn2 : -INFINITY;
      p.ring_l[ds * Gt + h0 + h] = L;
    }
    // output = S + tail
    const float M2 = fmaxf(M, MB);
    const float M2u = M2 == -INFINITY ? 0.f : M2;
    const float a0 = ex2(M - M2u), aB = ex2(MB - M2u);
    const float L2 = L * a0 + LB * aB, O2 = O * a0 + OB * aB;
    const size_t orow = (size_t)b * p.Hq + (size_t)kvh * Gt + h0 + h;
    p.out[orow * D + d] = __fdividef(O2, L2);  // L2 >= 1: every unit attends at least one key
    if (d == 0) p.lse[orow] = (M2 + __log2f(L2)) * kLn2;
  }
  if (threadIdx.x == 0 && ch == 0) p.ring_pos[(size_t)u * Wp1 + dst] = end - 1;
}

// Last arriver of a split unit: merge its partials.  Segment A's partials
// (with the reused state on a hit) give the new prefix state over [0, c_t),
// stored in the ring; that state and segment B's partials give the output.
// The warps share the partials out -- A's over warps [0, wA), B's over the
// rest, in proportion to their counts -- and each folds its own into one
// state (lane: four consecutive elements of every 128, KB partials per round
// of loads); the finish of a whole unit then combines the eight states.
template <int D, int GP, int GF, bool PH, int NC = 1>
__device__ __noinline__ bool merge_unit(const AttendParams& p, AttnSmem<D, GP>& sm, int u, uint32_t& sync_phase) {
  using C = Cfg<D, GP>;
  constexpr int NCH = C::GD / 128;                // 128-element runs of a padded group: 2, 4 or 8
  constexpr int KB = NCH <= 2 ? 8 : 16 / NCH;     // partials per round of loads
  // chunked groups (NC > 1): the unit's 8 NC heads are merged 8 at a time;
  // chunk ch of a partial is a run of partial_floats(8, D) floats at ch times that
  const int G = NC > 1 ? GP : group_of<GF>(p), GD = G * D, G4 = group4(G);  // heads of one chunk
  const int Gt = NC > 1 ? GF : G;                                           // heads of the unit
  const int PF = NC > 1 ? (int)partial_floats(Gt, D) : GD + 2 * G4;         // floats of one partial
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // plan and items may come from other CTAs of the same launch: read through L2
  const UnitPlan* const pp = p.plan + u;
  const int src_slot = __ldcg(&pp->src_slot), dst_slot = __ldcg(&pp->dst_slot), end = __ldcg(&pp->end);
  const int hmask = PH ? p.hplan[u].hmask : (__ldcg(&pp->hit) ? (1 << G) - 1 : 0);  // heads with a reused state
  const Segment sA = load_segment(p.seg + 2 * u), sB = load_segment(p.seg + 2 * u + 1);
  const int nA = sA.npieces, nB = sB.npieces, n = nA + nB;
  int wA = kConsumerWarps;
  if (nB > 0) {
    wA = nA > 0 ? (kConsumerWarps * nA + n / 2) / n : 0;
    if (nA > 0) wA = wA < 1 ? 1 : (wA > kConsumerWarps - 1 ? kConsumerWarps - 1 : wA);
  }
  const bool onA = warp < wA;
  const int cnt = onA ? nA : nB, stride = onA ? wA : kConsumerWarps - wA, first = onA ? warp : warp - wA;
#pragma unroll 1
  for (int ch = 0; ch < NC; ++ch) {
    const int h0 = ch * G;  // first head of this chunk in the unit
    const float* const part = p.part + (size_t)(onA ? sA.pbase : sB.pbase) * PF + (size_t)ch * (GD + 2 * G4);
    // the reused state on chip, in the layout of a whole unit's copy: each
    // head's o row (fp32 or bf16 as stored), then m at GP*D and l at GP*D + GP
    if (hmask != 0) {
      const size_t ub = (size_t)u * (p.W + 1);
      const int es = p.ring_bf16 ? 2 : 4, cph = D * es / 16;  // 16-byte chunks of one head's o
      const int h = tid / cph, c = tid - h * cph;
      if (h < G && ((hmask >> h) & 1)) {
        const int slot = PH ? p.hplan[u].hsrc[h] : src_slot;
        const uint4* src = reinterpret_cast<const uint4*>(
            ring_o_row(p.ring_o, ((ub + slot) * Gt + h0 + h) * D, p.ring_bf16));
        reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(sm.ring) + (size_t)h * D * es)[c] = __ldcg(src + c);
      }
      if (tid < 2 * G) {
        const int hh = tid < G ? tid : tid - G;
        if ((hmask >> hh) & 1) {
          const size_t e = (ub + (PH ? p.hplan[u].hsrc[hh] : src_slot)) * Gt + h0 + hh;
          sm.ring[C::GD + (tid < G ? hh : GP + hh)] = __ldcg(tid < G ? p.ring_m + e : p.ring_l + e);
        }
      }
    }
    float M[NCH], L[NCH], O[NCH][4];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      M[j] = -INFINITY;
      L[j] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) O[j][c] = 0.f;
    }
#pragma unroll 1
    for (int i0 = first; i0 < cnt; i0 += KB * stride) {
      float4 ov[KB][NCH];
      float mv[KB][NCH], lv[KB][NCH];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int i = i0 + k * stride;
        const float* q = part + (size_t)i * PF;
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          const int e = j * 128 + lane * 4, h = e / D;
          if (i < cnt && e < GD) {
            ov[k][j] = __ldcg(reinterpret_cast<const float4*>(q + e));
            mv[k][j] = __ldcg(q + GD + h);
            lv[k][j] = __ldcg(q + GD + G4 + h);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < KB; ++k)
#pragma unroll
        for (int j = 0; j < NCH; ++j)
          if (i0 + k * stride < cnt && j * 128 + lane * 4 < GD)
            fold_state<4>(M[j], L[j], O[j], mv[k][j], lv[k][j], &ov[k][j].x);
    }
    // this warp's state into its slot: o [GP][D], m [GP], l [GP]
    float* const wb = sm.wbuf[warp];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int e = j * 128 + lane * 4, h = e / D;
      if (e < GD) {
        *reinterpret_cast<float4*>(wb + e) = make_float4(O[j][0], O[j][1], O[j][2], O[j][3]);
        if (e - h * D == 0) {
          wb[C::GD + h] = M[j];
          wb[C::GD + GP + h] = L[j];
        }
      }
    }
    if (!consumer_sync(sm, sync_phase, p.status)) return false;
    unit_epilogue<D, GP, GF, NC>(p, sm, u, wA, hmask != 0, hmask, dst_slot, end, ch);
    // the warps' slots and the ring buffer are reused by the next chunk or piece
    if (!consumer_sync(sm, sync_phase, p.status)) return false;
  }
  if (tid == 0) p.unit_cnt[u] = 0;
  return true;
}

// End of a split piece: combine the 8 warps, write the partial, count it
// and, if it was the unit's last, merge the unit.
// Chunked groups: merge element e (head h) of chunk ch from the slots of the
// warps that hold that chunk (warps ch, ch + NC, ...), sums relative to 2^M.
template <int D, int GP, int NC>
__device__ __forceinline__ void combine_team(const AttnSmem<D, GP>& sm, int ch, int e, int h, float& M, float& L,
                                             float& O) {
  constexpr int NKL = kConsumerWarps / NC, GD = Cfg<D, GP>::GD;
  float m[NKL], l[NKL], o[NKL];
#pragma unroll
  for (int k = 0; k < NKL; ++k) {
    const int w = ch + NC * k;
    m[k] = sm.wbuf[w][GD + h];
    l[k] = sm.wbuf[w][GD + GP + h];
    o[k] = sm.wbuf[w][e];
  }
  M = m[0];
#pragma unroll
  for (int k = 1; k < NKL; ++k) M = fmaxf(M, m[k]);
  const float Mu = M == -INFINITY ? 0.f : M;
  L = O = 0.f;
#pragma unroll
  for (int k = 0; k < NKL; ++k) {
    const float a = ex2(m[k] - Mu);
    L += l[k] * a;
    O += o[k] * a;
  }
}

template <int D, int GP, int GF, bool PH, int NC = 1>
__device__ bool finalize_piece(const AttendParams& p, AttnSmem<D, GP>& sm, Acc<D, GP>& A, int unit, int pidx,
                               uint32_t& sync_phase) {
  const int G = group_of<GF>(p), GD = G * D, G4 = group4(G);
  warp_combine_store<D, GP>(A, sm.wbuf[threadIdx.x >> 5]);
  if (!consumer_sync(sm, sync_phase, p.status)) return false;
  float* dst = p.part + (size_t)pidx * (GD + 2 * G4);
  if constexpr (NC > 1) {
    // chunk ch of the partial: o [8][D], m [8], l [8] (the layout of an 8-head partial)
    constexpr int GDc = GP * D, PFc = GDc + 2 * GP;
#pragma unroll 1
    for (int idx = threadIdx.x; idx < GD; idx += kConsumerWarps * 32) {
      const int ch = idx / GDc, e = idx - ch * GDc, h = e / D;
      float M, L, O;
      combine_team<D, GP, NC>(sm, ch, e, h, M, L, O);
      float* dc = dst + (size_t)ch * PFc;
      dc[e] = O;
      if (e - h * D == 0) {
        dc[GDc + h] = M;
        dc[GDc + GP + h] = L;
      }
    }
  } else {
#pragma unroll 1
    for (int idx = threadIdx.x; idx < GD; idx += kConsumerWarps * 32) {
      const int h = idx / D;
      float MA, LA, OA, M, L, O;
      combine_warps2<D, GP, GP>(sm, 0, idx, h, MA, LA, OA, M, L, O);
      dst[idx] = O;
      if (idx - h * D == 0) {
        dst[GD + h] = M;
        dst[GD + G4 + h] = L;
      }
    }
  }
  // every thread's partial stores happen-before thread 0's fence through the
  // barrier; the fence publishes them device-wide before the count
  if (!consumer_sync(sm, sync_phase, p.status)) return false;
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(p.unit_cnt + unit, 1);
    sm.last_flag = (old == __ldcg(&p.plan[unit].expected) - 1);
  }
  if (!consumer_sync(sm, sync_phase, p.status)) return false;
  if (sm.last_flag) {
    __threadfence();
    if (p.counters != nullptr && threadIdx.x == 0) atomicAdd(p.counters + kCountMerged, 1ull);
    return merge_unit<D, GP, GF, PH, NC>(p, sm, unit, sync_phase);
  }
  return true;
}

// End of a whole-unit piece: warps [0, wA) hold the amend range [start, c_t),
// warps [wA, 8) the tail [c_t, p_t].  New prefix state = reused ring state
// (on a hit) + amend; output = new prefix + tail.  No partials, no counters.
// On a hit, the reused m and l come with o by bulk copy when GF is a multiple
// of 4 (16-byte runs), else thread t < 2G brings m (t < G) or l in rml.
// hmask: heads with a reused state (any of them when hit is set; per-head
// matching may leave some out).
template <int D, int GP, int GF>
__device__ bool finalize_unit(const AttendParams& p, AttnSmem<D, GP>& sm, Acc<D, GP>& A, int u, int wA, int hit,
                              int hmask, int dst, int end, float rml, uint32_t ring_phase, uint32_t& sync_phase) {
  constexpr int GDP = Cfg<D, GP>::GD;
  const int G = group_of<GF>(p);
  warp_combine_store<D, GP>(A, sm.wbuf[threadIdx.x >> 5]);
  if (!kBulkML<GF> && hit && (int)threadIdx.x < 2 * G &&
      ((hmask >> ((int)threadIdx.x < G ? (int)threadIdx.x : (int)threadIdx.x - G)) & 1))
    sm.ring[GDP + ((int)threadIdx.x < G ? (int)threadIdx.x : GP + (int)threadIdx.x - G)] = rml;
  if (!consumer_sync(sm, sync_phase, p.status)) return false;
  // the reused o was copied on chip at the start of the piece
  if (hit && !mbar_wait(&sm.rfull, ring_phase, &sm.abort_flag, p.status)) return false;
  unit_epilogue<D, GP, GF>(p, sm, u, wA, hit, hmask, dst, end);
  // the warps' slots are reused by the next piece
  return consumer_sync(sm, sync_phase, p.status);
}

// The boxes one warp takes from a piece: indices first, first + stride, ...
struct WarpRange {
  int kb0, k0, k1, nbox, first, stride;
};
__device__ __forceinline__ WarpRange warp_range(const Piece& pc, int warp) {
  WarpRange r;
  if (pc.whole && warp < pc.wA) {
    r.kb0 = pc.akb0;
    r.k0 = pc.a0;
    r.k1 = pc.a1;
    r.nbox = pc.anbox;
    r.first = warp;
    r.stride = pc.wA;
  } else {
    const int base = pc.whole ? pc.wA : 0;
    r.kb0 = pc.kb0;
    r.k0 = pc.k0;
    r.k1 = pc.k1;
    r.nbox = pc.nbox;
    r.first = warp - base;
    r.stride = kConsumerWarps - base;
  }
  return r;
}
// Chunked groups: the boxes of a split piece taken by key-lane kl of nkl.
__device__ __forceinline__ WarpRange team_range(const Piece& pc, int kl, int nkl) {
  WarpRange r;
  r.kb0 = pc.kb0;
  r.k0 = pc.k0;
  r.k1 = pc.k1;
  r.nbox = pc.nbox;
  r.first = kl;
  r.stride = nkl;
  return r;
}

// The cumulative range shares of the next weighted split from the SMs'
// rate records, by all threads of one CTA: unknown rates count as the mean,
// all are clamped to [1/2, 2] x mean, then scanned in fixed point (units of
// mean / 2^20, so the scan is exact).  Rates of other SMs may still be
// changing: any mix of old and new values is a valid split.
__device__ __noinline__ void rate_shares(const AttendParams& p) {
  __shared__ long long red[kConsumerWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, G = p.grid;
  const float r = tid < G ? __ldcg(p.rate + tid) : 0.f;
  long long v = r > 0.f ? ((long long)1 << 40) + (long long)(r * 1048576.0f) : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  long long tot = 0;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) tot += red[w];
  __syncthreads();
  const int known = (int)(tot >> 40);
  const double mean = known > 0 ? (double)(tot & (((long long)1 << 40) - 1)) / (1048576.0 * known) : 1.0;
  const double w = r > 0.f ? fmin(fmax((double)r, 0.5 * mean), 2.0 * mean) : mean;
  const long long wi = tid < G ? (long long)(w / mean * 1048576.0) : 0;
  long long x = wi;  // inclusive scan: lanes, then warps
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  long long before = 0, all = 0;
#pragma unroll
  for (int k = 0; k < kConsumerWarps; ++k) {
    if (k < warp) before += red[k];
    all += red[k];
  }
  if (tid < G) p.cw[tid] = (double)(before + x - wi) / (double)all;
  if (tid == 0) p.cw[G] = 1.0;
}

// NC: chunks of 8 heads per KV head (1 for groups of up to 8).  With NC > 1
// (G = 8 NC) warp w holds the heads [8 (w % NC), 8 (w % NC) + 8) over the
// boxes of key-lane w / NC: the NC warps of a key-lane read the same boxes
// from one ring of NST * NC slots, filled by the key-lane's first warp after
// every reader of the slot has released it (an mbarrier with NC arrivals), so
// each K/V byte crosses from HBM once for all 8 NC heads.  Such groups run
// split items only.
//
// FUSED (the one-launch step, mac_step.cu): the CTAs first run the match
// stage of their own units (unit u on CTA u mod grid), do every whole unit
// they matched on the spot (no other CTA is involved), then take the range
// of the step's split items that the last CTA to finish matching laid out
// (build_split_table) and stream it as the attention kernel does.  Needs all
// CTAs resident at once (a cooperative launch): a CTA waits, bounded, for
// the layout.
template <int D, int GP, int GF, bool PH, int NC, bool FUSED, bool RB>
__device__ __forceinline__ void attend_body(const AttendParams& p, const MatchParams& mp) {
  using C = Cfg<D, GP>;
  constexpr int NST = C::NST, NQ = C::NQ;
  constexpr int NKL = kConsumerWarps / NC, NSTT = NST * NC;  // key-lanes; box slots of one key-lane
  static_assert(NC == 1 || (GP == 8 && GF == 8 * NC && kConsumerWarps % NC == 0), "chunked groups of 8 heads");
  constexpr uint32_t kBoxBytes = kSubKeys * D * 2;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  // the swizzled TMA boxes need 1024-byte alignment of the shared window
  AttnSmem<D, GP>& sm =
      *reinterpret_cast<AttnSmem<D, GP>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = group_of<GF>(p), GD = G * D;  // real group: global layouts
  const int ch = warp % NC, kl = warp / NC;   // chunk of heads, key-lane (NC = 1: 0 and the warp)
  const bool issuer = ch == 0;                // fills the key-lane's box slots
  // box slot st of this key-lane: K box, V box (+ kSubKeys * D), its barriers
  auto kv_slot = [&](int st) -> uint16_t* {
    const int f = kl * NSTT + st;
    return sm.kv[f / NST][f % NST][0];
  };
  auto full_bar = [&](int st) -> unsigned long long* {
    const int f = kl * NSTT + st;
    return &sm.full[f / NST][f % NST];
  };
  auto empty_bar = [&](int st) -> unsigned long long* {
    const int f = kl * NSTT + st;
    return &sm.empty[f / NST][f % NST];
  };

  const int cta = blockIdx.x;
  if (tid == 32) {  // bring both TMA descriptors on chip while the match kernel runs
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmK)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmV)) : "memory");
  }
  if (tid == 0) {
    for (int w = 0; w < kConsumerWarps; ++w)
      for (int s = 0; s < NST; ++s) {
        mbar_init(&sm.full[w][s], 1);
        if (NC > 1) mbar_init(&sm.empty[w][s], NC);
      }
    for (int s = 0; s < NQ; ++s) mbar_init(&sm.qfull[s], 1);
    mbar_init(&sm.csync, kConsumerWarps);
    mbar_init(&sm.rfull, 1);
    sm.abort_flag = 0;
    sm.last_flag = 0;
    sm.box_total = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  unsigned smid;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
  const uint64_t pol = evict_first_policy();
  auto stamp = [&](int k) __attribute__((always_inline)) {
    if (p.trace != nullptr && tid == 0) p.trace[cta * kTracePoints + k] = globaltimer();
  };
  stamp(kTraceStart);

  // cursors, counters and barrier phases of this CTA; they carry over from
  // one walk to the next (the box slots' phases follow the box counts)
  int ipn = 0, nissued = 0, nq_issued = 0;    // issue side: pieces passed, boxes and queries issued
  Acc<D, GP> A;
  int cpn = 0, cons = 0, par = 0;             // consume side: pieces and boxes done
  uint32_t sync_phase = 0, ring_phase = 0;
  bool ring_pending = false;  // a reused-state copy was issued and not yet waited for
  bool ok = true;
  unsigned long long t_first = 0, t_last = 0;  // thread 0: first and last box of the timed walk
  int cons0 = 0;                               // boxes consumed before the timed walk
  auto range_of = [&](const Piece& pc) __attribute__((always_inline)) { return NC == 1 ? warp_range(pc, warp) : team_range(pc, kl, NKL); };

  // One walk over the items of `table` from first_seg on whose cost range
  // meets [lo, hi), as range `slot` of the table's split.
  // (forced inline: called twice, it must keep the accumulators in registers)
  auto walk = [&](const Segment* table, int nseg, int first_seg, long long lo, long long hi, int slot,
                  bool timed, bool local) __attribute__((always_inline)) {
  // issue cursor: this warp's (NC > 1: this key-lane's) boxes of every piece, NSTT ahead
  Walker wi{first_seg, lo, hi, sm.items, first_seg, table, nseg, local};
  Piece ip;
  WarpRange ir;
  bool ivalid = issuer && wi.next(slot, ip);
  if (ivalid) ir = range_of(ip);
  int ib = ivalid ? ir.first : 0;
  auto issue_advance = [&]() __attribute__((always_inline)) {
    while (ivalid && ib >= ir.nbox) {
      ivalid = wi.next(slot, ip);
      if (ivalid) {
        ir = range_of(ip);
        ib = ir.first;
      }
      ++ipn;
    }
  };
  auto issue_box = [&](int st) __attribute__((always_inline)) {
    // warp 0 always owns box 0 of its range in every piece: it brings the query
    // (chunked groups read their query straight from global memory instead)
    const bool qfirst = NC == 1 && warp == 0 && ib == 0;
    if (lane == 0) {
      if (qfirst) {
        const int qs = ipn % NQ;
        mbar_arrive_expect_tx(&sm.qfull[qs], GD * 4);
        bulk_load(sm.q[qs], p.qrot + (size_t)ip.unit * GD, GD * 4, &sm.qfull[qs]);
      }
      const int key = ir.kb0 + ib * kSubKeys;
      const int b = ip.unit / p.Hkv, kvh = ip.unit - b * p.Hkv;
      int c2, c3;
      if (p.page_size > 0) {
        c3 = p.block_table[(size_t)b * p.max_pages + key / p.page_size];
        c2 = key % p.page_size;
      } else {
        c2 = key;
        c3 = b;
      }
      unsigned long long* fb = full_bar(st);
      uint16_t* kbuf = kv_slot(st);
      mbar_arrive_expect_tx(fb, 2 * kBoxBytes);
#pragma unroll
      for (int hf = 0; hf < C::HALVES; ++hf) {
        tma_load_4d(kbuf + hf * kSubKeys * 64, &p.tmK, fb, 64 * hf, kvh, c2, c3, pol);
        tma_load_4d(kbuf + kSubKeys * D + hf * kSubKeys * 64, &p.tmV, fb, 64 * hf, kvh, c2, c3, pol);
      }
    }
    if (qfirst) ++nq_issued;
    ++nissued;
    ib += ir.stride;
    issue_advance();
  };
  issue_advance();
  // the first boxes of the walk go to the slots after the previous walk's last
  // (the consume side reads box n from slot n mod NSTT)
  for (int k = 0; k < NSTT && ivalid; ++k) issue_box(nissued % NSTT);

  // consume cursor
  Walker wc{first_seg, lo, hi, sm.items, first_seg, table, nseg, local};
  Piece cp;
  if (timed) cons0 = cons;
  while (ok && wc.next(slot, cp)) {
    if constexpr (NC == 1) {
      const int qs = cpn % NQ;
      if (!mbar_wait(&sm.qfull[qs], (uint32_t)(cpn / NQ) & 1u, &sm.abort_flag, p.status)) break;
      load_query<D, GP>(A, sm.q[qs], G);
    } else {
      // this warp's 8 heads of the unit's rotated query (written by the match kernel)
      load_query<D, GP>(A, p.qrot + ((size_t)cp.unit * GF + ch * GP) * D, GP);
    }
    const bool ring_copy = cp.whole && cp.hit;
    ring_pending = ring_copy;
    float rml = 0.f;  // m (thread t < G) or l (G <= t < 2G) of the reused state
    int hmask = ring_copy ? (1 << G) - 1 : 0;  // heads with a reused state
    int lo0 = 0, lo1 = 0;                      // per-head matching: first keys of this lane's heads
    if constexpr (PH) {
      // each head starts its fresh keys at its own reuse boundary (amend range
      // only; every head attends the whole tail)
      const HeadPlan* pp = p.hplan + cp.unit;
      if (ring_copy) hmask = pp->hmask;
      const bool onA = cp.whole ? warp < cp.wA : cp.segA;
      const int hh = GP == 4 ? 2 * ((lane & 3) & 1) : 2 * (lane & 3);
      lo0 = onA && hh < G ? pp->hstart[hh] : INT_MIN;
      lo1 = onA && hh + 1 < G ? pp->hstart[hh + 1] : INT_MIN;
    }
    if (PH && ring_copy) {
      // per-head matching: each reusing head's state comes from its own slot
      const size_t ub = (size_t)cp.unit * (p.W + 1);
      if (warp == 0) {
        const uint32_t ob = D * (p.ring_bf16 ? 2 : 4);  // bytes of one head's o
        if (lane == 0) mbar_arrive_expect_tx(&sm.rfull, __popc(hmask) * ob);
        __syncwarp();
        if (lane < G && ((hmask >> lane) & 1)) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          bulk_load(reinterpret_cast<unsigned char*>(sm.ring) + lane * ob,
                    ring_o_row(p.ring_o, ((ub + p.hplan[cp.unit].hsrc[lane]) * G + lane) * D, p.ring_bf16), ob,
                    &sm.rfull);
        }
      }
      if (tid < 2 * G) {
        const int h = tid < G ? tid : tid - G;
        if ((hmask >> h) & 1) {
          const size_t e = (ub + p.hplan[cp.unit].hsrc[h]) * G + h;
          rml = __ldcg(tid < G ? p.ring_m + e : p.ring_l + e);
        }
      }
    } else if (ring_copy) {
      // the merge at the end of the piece reads the reused ring state: copy
      // its o on chip now (the previous piece's merge is done with the
      // buffer); m and l travel in registers
      const size_t rs = (size_t)cp.unit * (p.W + 1) + cp.src;
      if (tid == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const uint32_t ob = GD * (p.ring_bf16 ? 2 : 4);  // bytes of the group's o
        mbar_arrive_expect_tx(&sm.rfull, ob + (kBulkML<GF> ? 2 * G * 4 : 0));
        bulk_load(sm.ring, ring_o_row(p.ring_o, rs * GD, p.ring_bf16), ob, &sm.rfull);
        if constexpr (kBulkML<GF>) {
          bulk_load(sm.ring + C::GD, p.ring_m + rs * G, G * 4, &sm.rfull);
          bulk_load(sm.ring + C::GD + GP, p.ring_l + rs * G, G * 4, &sm.rfull);
        }
      }
      if (!kBulkML<GF> && tid < 2 * G)
        rml = __ldcg(tid < G ? p.ring_m + rs * G + tid : p.ring_l + rs * G + (tid - G));
    }
    const WarpRange cr = range_of(cp);
    for (int bj = cr.first; bj < cr.nbox; bj += cr.stride) {
      const int st = cons % NSTT;
      const uint32_t ph = (uint32_t)(cons / NSTT) & 1u;
      if (!mbar_wait(full_bar(st), ph, &sm.abort_flag, p.status)) {
        ok = false;
        break;
      }
      if (timed && tid == 0 && cons == cons0) t_first = globaltimer();
      if (tid == 0 && cons == 0) stamp(kTraceFirstBox);
      const int key_box = cr.kb0 + bj * kSubKeys;
      float* pbuf = sm.wbuf[warp] + par * C::PB;
      uint16_t* kbuf = kv_slot(st);
      process_box<D, GP, PH>(A, kbuf, kbuf + kSubKeys * D, pbuf, key_box, cr.k0, cr.k1,
                             key_box < cr.k0 || key_box + kSubKeys > cr.k1, lo0, lo1);
      par ^= 1;
      ++cons;
      if constexpr (NC > 1) {
        // release the slot: this warp's reads (and its zeroing of rows outside
        // the range, identical in every reader) are done before the next copy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st));
        __syncwarp();
        if (ivalid && !mbar_wait(empty_bar(st), ph, &sm.abort_flag, p.status)) {
          ok = false;
          break;
        }
      } else {
        __syncwarp();
      }
      if (ivalid) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_box(st);
      }
    }
    if (!ok) break;
    if (timed && tid == 0) t_last = globaltimer();
    if (local) stamp(kTraceBoxesDone);
    bool fin;
    if constexpr (NC > 1)
      fin = finalize_piece<D, GP, GF, PH, NC>(p, sm, A, cp.unit, cp.pidx, sync_phase);
    else
      fin = cp.whole ? finalize_unit<D, GP, GF>(p, sm, A, cp.unit, cp.wA, cp.hit, hmask, cp.dst, cp.k1, rml,
                                                ring_phase, sync_phase)
                     : finalize_piece<D, GP, GF, PH>(p, sm, A, cp.unit, cp.pidx, sync_phase);
    if (ring_copy) ring_phase ^= 1u;
    ring_pending = false;
    if (!fin) {
      ok = false;
      break;
    }
    if (p.counters != nullptr && tid == 0) {
      atomicAdd(p.counters + kCountKeys, (unsigned long long)(cp.k1 - cp.k0 + (cp.whole ? cp.a1 - cp.a0 : 0)));
      atomicAdd(p.counters + kCountPieces, 1ull);
      if (cp.whole) atomicAdd(p.counters + kCountWhole, 1ull);
    }
    ++cpn;
  }
  };  // walk

  int weighted = 0;
  int first_seg = 0, slot = cta;
  long long lo = 0, hi = 0;
  if constexpr (FUSED) {
    // ---- the one-launch step: match, whole units on the spot, then the split range
    const int U = mp.B * mp.Hkv;
    using MS = MatchSmem<D, GP, false>;
    static_assert(sizeof(MS) <= sizeof(sm.kv), "match scratch lives in the box slots");
    MS& ms = *reinterpret_cast<MS*>(&sm.kv[0][0][0][0]);
    // this launch's epoch: read before the ticket (the layout advances it only
    // after every ticket), consumed after the match stage
    const unsigned epoch = tid == 0 ? ld_relaxed_u32(p.fsync + 1) : 0u;
    if (tid == 0) sm.nlocal = 0;
    __syncthreads();
    // match stage of this CTA's units; whole units become local items
#pragma unroll 1
    for (int u = cta; u < U; u += gridDim.x) {
      match_body<D, GP, GF, false, RB>(mp, u, ms);
      __syncthreads();
      if (tid == 0) {
        const UnitPlan pl = ms.s_plan;
        if (!(pl.bad || ms.s_bad_page) && pl.end - pl.start <= mp.unit_max && sm.nlocal < kItemCache) {
          Segment sg;
          sg.kind = kItemWhole;
          sg.flat = u;  // a local item carries its unit
          sg.len = pl.end - pl.start;
          sg.key0 = pl.start;
          sg.first_cta = cta;
          sg.pbase = pl.cut;
          sg.npieces = (pl.hit ? 1 : 0) | ((pl.hit && pl.src_slot >= 0 ? pl.src_slot & 0x7ff : 0) << 1) |
                       ((pl.dst_slot & 0x7ff) << 12);
          sm.items[sm.nlocal++] = sg;
        }
      }
    }
    stamp(kTraceMatched);
    // the box slots held the match scratch, and the bulk copies of this launch
    // read the rotated queries just written: order those generic writes (shared
    // and global) before any copy, then publish them device-wide
    asm volatile("fence.proxy.async;" ::: "memory");
    __syncthreads();
    // the last CTA lays out the split items once every other CTA has published
    // its plans (it holds a unit only when there are as many units as CTAs, so
    // the layout seldom waits behind a match or delays a whole unit)
    const int builder = (int)gridDim.x - 1;
    if (tid == 0) {
      p.smid_of[cta] = (int)smid;
      if (cta != builder) {
        // the block barrier above orders every thread's writes before this
        // thread's arrival, and a release is cumulative: the arrival publishes
        // them device-wide
        asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(p.fsync) : "memory");
      } else {
        const unsigned long long t0 = globaltimer();
        while ((int)ld_acquire_u32(p.fsync) != builder) {
          if (globaltimer() - t0 > kWaitLimitNs) {
            atomicOr(p.status, MAC_DEV_TIMEOUT);
            sm.abort_flag = 1;
            break;
          }
        }
      }
      if (p.trace) p.trace[cta * kTracePoints + kTraceTicket] = globaltimer();
    }
    __syncthreads();
    if (cta == builder) {
      // every other CTA's plans and SM id precede its arrival: lay out the split items
      __threadfence();
      static_assert(sizeof(SplitScratch) <= sizeof(sm.kv), "split scratch lives in the box slots");
      build_split_table(mp, U, (int)gridDim.x, p.smid_of, p.rank_of,
                        *reinterpret_cast<SplitScratch*>(&sm.kv[0][0][0][0]));
      asm volatile("fence.proxy.async;" ::: "memory");  // the scratch in the box slots, before copies
      __syncthreads();
      if (tid == 0) {
        p.fsync[0] = 0;
        // every thread's table writes, ordered by the barrier, are published by the release
        st_release_u32(p.fsync + 1, epoch + 1u);
        if (p.trace) p.trace[cta * kTracePoints + kTraceBuilt] = globaltimer();
      }
    }
    __syncthreads();
    // this CTA's whole units
    const int nlocal = sm.nlocal;
    if (nlocal > 0) walk(sm.items, nlocal, 0, 0, LLONG_MAX, cta, false, true);
    stamp(kTraceLocal);
    // the step's split table (bounded wait for the last CTA's layout)
    if (tid == 0 && ok) {
      const unsigned long long t0 = globaltimer();
      while (ld_acquire_u32(p.fsync + 1) != epoch + 1u) {
        if (globaltimer() - t0 > kWaitLimitNs) {
          atomicOr(p.status, MAC_DEV_TIMEOUT);
          sm.abort_flag = 1;
          break;
        }
      }
    }
    __syncthreads();
    // the split pieces' queries were written by other CTAs of this launch and
    // are read by bulk copies: order the acquire before those copies
    asm volatile("fence.proxy.async.global;" ::: "memory");
    stamp(kTraceTable);
    // (written by another CTA of this launch: read through L2)
    if (ok && !sm.abort_flag && __ldcg(&p.hdr->total) > 0) {
      weighted = __ldcg(&p.hdr->weighted);
      const int rank = __ldcg(p.rank_of + (weighted ? (int)smid : cta));
      if (rank >= 0) {
        slot = rank;
        lo = __ldcg(p.bounds + rank);
        hi = __ldcg(p.bounds + rank + 1);
        first_seg = __ldcg(p.first_seg + rank);
      }
    }
    ok = ok && !sm.abort_flag;
  } else {
    // launched with programmatic stream serialization: everything above
    // overlaps the match kernel; its results are visible after this wait
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // one round of loads: the split, then the CTA's items into shared memory
    const int n_cta = p.hdr->n_cta;
    weighted = p.hdr->weighted;
    const long long T = p.hdr->total;
    first_seg = p.first_seg[cta];
    // a weighted split: take the range of this SM (claimed in the same round
    // of loads), else the first free one
    int mine = 0;
    if (tid == 0 && p.claim != nullptr && (int)smid < p.grid) mine = atomicCAS(p.claim + smid, 0, 1) == 0;
    if (weighted) {
      if (tid == 0) {
        int c = mine ? (int)smid : -1;
        for (int k = 0; c < 0 && k < n_cta; ++k)
          if (atomicCAS(p.claim + k, 0, 1) == 0) c = k;
        sm.last_flag = c;
      }
      __syncthreads();
      slot = sm.last_flag;
      if (slot < 0) return;  // never: n_cta = grid ranges for grid CTAs
      lo = p.bounds[slot];
      hi = p.bounds[slot + 1];
      first_seg = p.first_seg[slot];
    } else {
      if (cta >= n_cta) return;
      lo = (long long)cta * T / n_cta;
      hi = (long long)(cta + 1) * T / n_cta;
    }
    stamp(kTraceTable);
  }
  if (ok && lo < hi) {
    if (tid < kItemCache && first_seg + tid < p.nseg) sm.items[tid] = load_segment(p.seg + first_seg + tid);
    __syncthreads();
    walk(p.seg, p.nseg, first_seg, lo, hi, slot, true, false);
    stamp(kTraceRange);
  }
  if (weighted && p.rate != nullptr) {
    // fold this SM's streaming rate (boxes per microsecond) into its record;
    // only CTAs that mostly streamed (at least kRateMinBoxes boxes) measure it
    if (lane == 0 && issuer) atomicAdd(&sm.box_total, cons - cons0);  // each box once, by the warp that filled it
    __syncthreads();
    const int boxes = sm.box_total;
    if (ok && tid == 0 && (int)smid < p.grid && boxes >= kRateMinBoxes && t_last > t_first + 2000) {
      const float r = (float)((double)boxes * 1000.0 / (double)(t_last - t_first));
      const float old = p.rate[smid];
      p.rate[smid] = old > 0.f ? 0.7f * old + 0.3f * r : r;
    }
    if (blockIdx.x == 0 && p.cw != nullptr && p.grid < kAttnThreads) rate_shares(p);
  }
  if (nissued > cons || !ok) {
    // aborting: let copies already issued land before the CTA leaves (bounded)
    if (lane == 0) {
      for (int k = cons; k < nissued; ++k) {
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(full_bar(k % NSTT), (uint32_t)(k / NSTT) & 1u) && globaltimer() - t0 < 100000000ull) {
        }
      }
      if (warp == 0) {
        // a reused-state copy of an unfinished hit piece may still be in flight
        const unsigned long long tr = globaltimer();
        while (ring_pending && !mbar_try_wait(&sm.rfull, ring_phase) && globaltimer() - tr < 100000000ull) {
        }
        for (int k = cpn; k < nq_issued; ++k) {
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(&sm.qfull[k % NQ], (uint32_t)(k / NQ) & 1u) && globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
    __syncwarp();
  }
  stamp(kTraceEnd);
}

template <int D, int GP, int GF, bool PH, int NC = 1>
__global__ void __launch_bounds__(kAttnThreads, 1) mac_attend_kernel(const __grid_constant__ AttendParams p) {
  attend_body<D, GP, GF, PH, NC, false, false>(p, MatchParams{});
}

// The whole decode step in one cooperative launch (groups of up to 8 heads,
// one decision per KV head): match, every whole unit by the CTA that matched
// it, then the split ranges.  RB: the window's queries are stored in bf16.
template <int D, int GP, int GF, bool RB>
__global__ void __launch_bounds__(kAttnThreads, 1)
    mac_step_kernel(const __grid_constant__ AttendParams p, const __grid_constant__ MatchParams mp) {
  attend_body<D, GP, GF, false, 1, true, RB>(p, mp);
}

// Failure-path self-test: one warp waits, through the kernels' bounded wait,
// on an mbarrier that nothing arrives on.  After the limit the wait sets
// MAC_DEV_TIMEOUT in the status word and the kernel returns.
__global__ void mac_wait_selftest_kernel(unsigned* status) {
  __shared__ unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort_flag, status);
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned* status, cudaStream_t s) {
  mac_wait_selftest_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

size_t attend_smem_bytes(int D, int G) {
  const bool g4 = group_pad(G) == 4;
  if (D == 128) return (g4 ? sizeof(AttnSmem<128, 4>) : sizeof(AttnSmem<128, 8>)) + 1024;
  return (g4 ? sizeof(AttnSmem<64, 4>) : sizeof(AttnSmem<64, 8>)) + 1024;
}

namespace {
// Kernel variants: exact groups of 4 and 8 (compile-time G), groups of 1-3
// and 5-7 padded to 4 and 8 (run-time G), and per-head matching (run-time G).
template <int D, int GP, int GF, bool PH, int NC = 1>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(mac_attend_kernel<D, GP, GF, PH, NC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)attend_smem_bytes(D, GP));
}
template <int D>
cudaError_t set_smem_all() {
  cudaError_t e = set_smem<D, 4, 4, false>();
  if (e == cudaSuccess) e = set_smem<D, 4, 0, false>();
  if (e == cudaSuccess) e = set_smem<D, 8, 8, false>();
  if (e == cudaSuccess) e = set_smem<D, 8, 0, false>();
  if (e == cudaSuccess) e = set_smem<D, 4, 0, true>();
  if (e == cudaSuccess) e = set_smem<D, 8, 0, true>();
  if (e == cudaSuccess) e = set_smem<D, 8, 16, false, 2>();
  if (e == cudaSuccess) e = set_smem<D, 8, 32, false, 4>();
  if (e == cudaSuccess) e = set_smem<D, 8, 64, false, 8>();
  return e;
}
// Per-head matching runs the run-time-group variants with per-head bounds.
template <int D>
cudaError_t launch_d(cudaLaunchConfig_t& cfg, const AttendParams& p) {
  const int G = p.G;
  cfg.dynamicSmemBytes = attend_smem_bytes(D, G);
  if (p.per_head) {
    if (G <= 4) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 4, 0, true>, p);
    return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 8, 0, true>, p);
  }
  if (G == 16) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 8, 16, false, 2>, p);
  if (G == 32) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 8, 32, false, 4>, p);
  if (G == 64) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 8, 64, false, 8>, p);
  if (G == 4) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 4, 4, false>, p);
  if (G == 8) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 8, 8, false>, p);
  if (G < 4) return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 4, 0, false>, p);
  return cudaLaunchKernelEx(&cfg, mac_attend_kernel<D, 8, 0, false>, p);
}
}  // namespace

namespace {
template <int D, bool RB>
const void* step_kernel(int G) {
  if (G == 4) return reinterpret_cast<const void*>(mac_step_kernel<D, 4, 4, RB>);
  if (G == 8) return reinterpret_cast<const void*>(mac_step_kernel<D, 8, 8, RB>);
  if (G < 4) return reinterpret_cast<const void*>(mac_step_kernel<D, 4, 0, RB>);
  return reinterpret_cast<const void*>(mac_step_kernel<D, 8, 0, RB>);
}
template <int D, bool RB>
cudaError_t step_launch_d(cudaLaunchConfig_t& cfg, const AttendParams& p, const MatchParams& mp) {
  const int G = p.G;
  if (G == 4) return cudaLaunchKernelEx(&cfg, mac_step_kernel<D, 4, 4, RB>, p, mp);
  if (G == 8) return cudaLaunchKernelEx(&cfg, mac_step_kernel<D, 8, 8, RB>, p, mp);
  if (G < 4) return cudaLaunchKernelEx(&cfg, mac_step_kernel<D, 4, 0, RB>, p, mp);
  return cudaLaunchKernelEx(&cfg, mac_step_kernel<D, 8, 0, RB>, p, mp);
}
}  // namespace

// Shared memory of one CTA of the one-launch step: the attention layout, but
// more than half of an SM, so that no SM ever holds two of its CTAs (the
// split's ranges are keyed by SM on large steps).
size_t step_smem_bytes(int D, int G) {
  static int half = -1;
  if (half < 0) {
    int dev = 0, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess)
      half = per_sm / 2 + 1024;
    else
      half = 0;
  }
  const size_t need = attend_smem_bytes(D, G);
  return need > (size_t)half ? need : (size_t)half;
}

namespace {
template <int D, int GP, int GF, bool RB>
cudaError_t step_smem_set(size_t bytes) {
  return cudaFuncSetAttribute(mac_step_kernel<D, GP, GF, RB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}
template <int D, bool RB>
cudaError_t step_smem_set_all(size_t b4, size_t b8) {
  cudaError_t e = step_smem_set<D, 4, 4, RB>(b4);
  if (e == cudaSuccess) e = step_smem_set<D, 4, 0, RB>(b4);
  if (e == cudaSuccess) e = step_smem_set<D, 8, 8, RB>(b8);
  if (e == cudaSuccess) e = step_smem_set<D, 8, 0, RB>(b8);
  return e;
}
}  // namespace

cudaError_t step_prepare(int D, int G, int* blocks_per_sm) {
  *blocks_per_sm = 0;
  if ((D != 64 && D != 128) || G < 1 || G > kMaxGroup) return cudaErrorInvalidValue;
  const size_t b4 = step_smem_bytes(D, 4), b8 = step_smem_bytes(D, 8);
  cudaError_t e = D == 128 ? step_smem_set_all<128, false>(b4, b8) : step_smem_set_all<64, false>(b4, b8);
  if (e == cudaSuccess) e = D == 128 ? step_smem_set_all<128, true>(b4, b8) : step_smem_set_all<64, true>(b4, b8);
  if (e != cudaSuccess) return e;
  // the launch needs every CTA resident at once: one per SM
  int nb = 0, nb2 = 0;
  const size_t smem = step_smem_bytes(D, G);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, D == 128 ? step_kernel<128, false>(G) : step_kernel<64, false>(G),
                                                    kAttnThreads, smem);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb2, D == 128 ? step_kernel<128, true>(G)
                                                                      : step_kernel<64, true>(G),
                                                      kAttnThreads, smem);
  *blocks_per_sm = nb < nb2 ? nb : nb2;
  return e;
}

cudaError_t launch_step(const AttendParams& p, const MatchParams& mp, int D, int grid, cudaStream_t s) {
  if ((D != 64 && D != 128) || p.G < 1 || p.G > kMaxGroup || p.per_head || mp.per_head)
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: they wait for the split table
  attr[0].val.cooperative = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = step_smem_bytes(D, p.G);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return mp.ring_bf16 ? step_launch_d<128, true>(cfg, p, mp) : step_launch_d<128, false>(cfg, p, mp);
  return mp.ring_bf16 ? step_launch_d<64, true>(cfg, p, mp) : step_launch_d<64, false>(cfg, p, mp);
}


cudaError_t attend_prepare(int D, int G) {
  if ((D != 64 && D != 128) || !group_ok(G)) return cudaErrorInvalidValue;
  if (D == 128 && G > kMaxGroup) {  // the tcgen05 path for groups of 16-64 heads
    cudaError_t e = attend_tc_prepare(G);
    if (e != cudaSuccess) return e;
  }
  return D == 128 ? set_smem_all<128>() : set_smem_all<64>();
}

cudaError_t launch_attend(const AttendParams& p, int D, int grid, cudaStream_t s) {
  if ((D != 64 && D != 128) || !group_ok(p.G) || (p.G > kMaxGroup && p.per_head)) return cudaErrorInvalidValue;
  // Programmatic stream serialization: the kernel may be scheduled while the
  // preceding match kernel drains; it calls griddepcontrol.wait before it
  // reads anything that kernel wrote.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128 && p.G > kMaxGroup && !p.per_head) return launch_attend_tc(p, grid, s);  // tcgen05 path
  return D == 128 ? launch_d<128>(cfg, p) : launch_d<64>(cfg, p);
}

}  // namespace mac
