// mac_attend_tc.cu -- attention for groups of 16, 32 and 64 query heads per
// KV head at head_dim 128 on the fifth-generation tensor cores (tcgen05.mma
// with tensor-memory accumulators), and the merge of its partial results.
// The work items, their cost-space split over the CTAs and the partial
// layout are those of the attention kernel (mac_attend.cu); the decode-step
// arithmetic is the same: softmax in exp2 units over the query pre-scaled by
// log2(e)/sqrt(D), partial states (o unnormalised, m, l) folded into the new
// prefix state (with the reused state on a hit) and the output.
#include <math.h>
#include <stdint.h>

#include <cuda_bf16.h>

#include "mac_internal.cuh"
#include "mac_attend_dev.cuh"

#include "../../include/mac.h"

namespace mac {
namespace {

// ============================================================ tcgen05 path
// Groups of 16, 32 or 64 query heads per KV head at head_dim 128: here the
// group is a real dense tile, so both products run on the fifth-generation
// tensor cores (tcgen05.mma, operands in shared memory, accumulators in
// tensor memory).  Per tile of 128 keys of one unit:
//   S^T [128 keys x N] = K [128 x D] . [Q_hi; Q_res]^T
//   O^T [D x N]       += V^T [D x 128 keys] . [P_hi | P_res]   (V read as stored,
//                                                               the MN-major operand)
// The query and the weights are split into a bf16 high part and a bf16
// residual (~16 mantissa bits, as in the box kernel), stacked along N: the
// columns of S and O are the G heads' high parts, then their residuals
// (padded to N = 64), and a head's value is the sum of its two columns.
// Warp 0 streams the K tiles and warp 2 the V tiles (16-key TMA boxes, each
// ring with its own barriers, so a K buffer returns to the stream as soon as
// its product is done), one thread of warp 1 issues the MMAs as their inputs
// arrive (S double-buffered in TMEM, O in TMEM), and the softmax warps from 4
// on (two per TMEM lane quadrant, four for groups of 64) each own a share of
// the heads for the 32 keys of their lanes: a thread holds one key's scores
// and its keys' running sums per head in registers; O is rescaled only when
// some head's maximum grows by more than 2^8 (weights stay below 256).  Every
// piece (a unit's keys in this CTA's range) ends in a partial in the
// chunk-major layout, and a second kernel (mac_tc_merge_kernel) merges each
// unit's partials with its reused state.
namespace tc {
constexpr int kKeys = 128;     // keys per tile: M of QK, K of PV
constexpr int kSoftWarp0 = 4;  // softmax warps from 4 on: warp w reads TMEM lanes 32 (w % 4) ..
// Softmax warps: four per TMEM lane quadrant for groups of 64 heads (16 heads
// each), two for smaller groups.
__host__ __device__ constexpr int soft_warps(int G) { return G >= 64 ? 16 : 8; }
__host__ __device__ constexpr int threads(int G) { return (kSoftWarp0 + soft_warps(G)) * 32; }
// Columns of S and of O: high parts and residuals of the G heads, at least 64.
__host__ __device__ constexpr int ncols(int G) { return 2 * G < 64 ? 64 : 2 * G; }
// Tiles in flight per ring and buffers of the weights P^T (shared memory:
// 2 + 3 tiles of K and V beside a 64-column query and two 64-column weight
// tiles; 2 + 3 beside 128-column ones and one weight tile).
__host__ __device__ constexpr int stages_k(int G) { return 2; }
__host__ __device__ constexpr int stages_v(int G) { return 3; }
__host__ __device__ constexpr int p_bufs(int G) { return G <= 32 ? 2 : 1; }
// Tensor memory: S[2] and O, N columns each, rounded to a power of two.
__host__ __device__ constexpr uint32_t tmem_cols(int G) { return 3 * ncols(G) <= 256 ? 256u : 512u; }
}  // namespace tc

// Shared memory of the tcgen05 kernel: the 128-byte-swizzled tiles first (each
// a multiple of 1 KB from a 1 KB-aligned base), then the small fields.
template <int G>
struct TcSmem {
  static constexpr int N = tc::ncols(G), SK = tc::stages_k(G), SV = tc::stages_v(G), NPB = tc::p_bufs(G);
  uint16_t k[SK][2][tc::kKeys * 64];  // [stage][half of D][128 keys][64 dims]
  uint16_t v[SV][2][tc::kKeys * 64];
  uint16_t q[2][N * 64];              // [half of D][N rows: Q_hi, Q_res, zero][64 dims]
  uint16_t pw[NPB][N / 64][tc::kKeys * 64];  // P^T: [buffer][64-column block][128 keys][64 columns]
  float m[G];                         // running maximum per head (log2 units)
  float red[4][G];                    // cross-warp reductions of the softmax warps
  unsigned long long full_k[SK], empty_k[SK], full_v[SV], empty_v[SV], s_full[2], s_empty[2];
  unsigned long long p_full[NPB], p_empty[NPB], q_full, drain;
  uint32_t tmem;
  int abort_flag;
  int last_flag;
};

// Byte offset of element (row, col) of a [rows][64] bf16 tile with the
// 128-byte swizzle (16-byte chunk c of row r at c ^ (r & 7)).
__device__ __forceinline__ uint32_t sw128_off(int row, int col64) {
  return (uint32_t)(row * 128 + ((((col64 >> 3) & 7) ^ (row & 7)) << 4) + (col64 & 7) * 2);
}
// Shared-memory matrix descriptor (tcgen05): start, leading and stride byte
// offsets, descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFF) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulate, bf16 A and B, the
// operands' majorness, N and M.
__host__ __device__ constexpr uint32_t umma_idesc(int a_mn, int b_mn, int N, int M) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred pa;\n\tsetp.ne.u32 pa, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pa;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Named barrier of the NT softmax threads, with an OR of one flag.
template <int NT>
__device__ __forceinline__ int softmax_sync_or(int flag) {
  int out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\tbar.red.or.pred po, 1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(flag), "n"(NT)
      : "memory");
  return out;
}
template <int NT>
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }

// A CTA role's walk over its pieces, tile by tile.
struct TileCursor {
  Walker w;
  Piece pc;
  int ntile, i, np;  // tiles of the piece, next tile in it, index of the piece
  bool live;
  __device__ __forceinline__ void open(int slot) {
    live = w.next(slot, pc);
    ntile = live ? (pc.k1 - pc.kb0 + tc::kKeys - 1) / tc::kKeys : 0;
    i = 0;
  }
  __device__ __forceinline__ void step(int slot) {
    if (++i >= ntile) {
      ++np;
      open(slot);
    }
  }
};

// n consecutive fp32 columns (n = 8, 16) of this warp's 32 TMEM lanes,
// issued without waiting (tmem_ld_wait completes them), and stored back.
template <int NCOL>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t* r);
template <int NCOL>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t* r);
template <>
__device__ __forceinline__ void tmem_ldn<8>(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_stn<8>(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ldn<16>(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_stn<16>(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}
template <int NR>
__device__ __forceinline__ void tmem_ld_wait(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < NR; ++j) asm volatile("" : "+r"(r[j]));
}
// Values of GH heads (8 or 16) of this thread's TMEM lane: the high-part
// columns at `hi` plus the residual columns at `res`.
template <int GH>
__device__ __forceinline__ void tmem_heads(uint32_t hi, uint32_t res, float* v) {
  static_assert(GH == 8 || GH == 16, "a softmax warp owns 8 or 16 heads");
  uint32_t r[2 * GH];
  tmem_ldn<GH>(hi, r);
  tmem_ldn<GH>(res, r + GH);
  tmem_ld_wait<2 * GH>(r);
#pragma unroll
  for (int j = 0; j < GH; ++j) v[j] = __uint_as_float(r[j]) + __uint_as_float(r[GH + j]);
}

// One ring of K or V tiles: boxes of 16 keys x 64 dims (two per key row of
// 128 dims) into stage t % S, never across a page; a tile's boxes past the
// piece's last key are not loaded.  Leaves once its copies have landed.
template <int S>
__device__ __forceinline__ void tc_stream(const AttendParams& p, const CUtensorMap* map, uint16_t (*ring)[2][tc::kKeys * 64],
                                          unsigned long long* full, unsigned long long* empty, TileCursor c, int slot,
                                          volatile int* abort_flag, uint64_t pol, unsigned long long* counters) {
  constexpr uint32_t kBox = 16 * 64 * 2;
  unsigned long long nkeys = 0, npieces = 0;
  int t = 0;
  while (c.live) {
    const int b = c.pc.unit / p.Hkv, kvh = c.pc.unit - b * p.Hkv;
    const int key0 = c.pc.kb0 + c.i * tc::kKeys, st = t % S;
    if (c.i == 0) {
      nkeys += (unsigned long long)(c.pc.k1 - c.pc.k0);
      ++npieces;
    }
    if (t >= S && !mbar_wait(&empty[st], (uint32_t)((t / S) - 1) & 1u, abort_flag, p.status)) break;
    const int left = (c.pc.k1 - key0 + kSubKeys - 1) / kSubKeys;
    const int nb = left < tc::kKeys / kSubKeys ? left : tc::kKeys / kSubKeys;
    mbar_arrive_expect_tx(&full[st], (uint32_t)nb * 2u * kBox);
    for (int j = 0; j < nb; ++j) {
      const int key = key0 + kSubKeys * j;
      int c2, c3;
      if (p.page_size > 0) {
        c3 = p.block_table[(size_t)b * p.max_pages + key / p.page_size];
        c2 = key % p.page_size;
      } else {
        c2 = key;
        c3 = b;
      }
      tma_load_4d(ring[st][0] + j * kSubKeys * 64, map, &full[st], 0, kvh, c2, c3, pol);
      tma_load_4d(ring[st][1] + j * kSubKeys * 64, map, &full[st], 64, kvh, c2, c3, pol);
    }
    ++t;
    c.step(slot);
  }
  // every copy issued has landed before the CTA leaves (bounded)
  for (int tt = t - S < 0 ? 0 : t - S; tt < t; ++tt) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&full[tt % S], (uint32_t)(tt / S) & 1u) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }
  if (counters != nullptr && npieces > 0) {
    atomicAdd(counters + kCountKeys, nkeys);
    atomicAdd(counters + kCountPieces, npieces);
  }
}

template <int GF>
__global__ void __launch_bounds__(tc::threads(GF), 1) mac_attend_tc_kernel(const __grid_constant__ AttendParams p) {
  constexpr int D = 128, G = GF, N = tc::ncols(G), SK = TcSmem<G>::SK, SV = TcSmem<G>::SV, NPB = TcSmem<G>::NPB;
  constexpr int SW = tc::soft_warps(G), NT = SW * 32;  // softmax warps and threads
  static_assert(G == 16 || G == 32 || G == 64, "groups of 16, 32 or 64 heads");
  constexpr int GDc = 8 * D, PFc = GDc + 16;  // one 8-head chunk of a partial: o [8][D], m [8], l [8]
  constexpr uint32_t kCols = tc::tmem_cols(G), kColO = 2 * N;  // S[0] at 0, S[1] at N, O at 2N
  constexpr uint32_t idesc_qk = umma_idesc(0, 0, N, tc::kKeys);
  constexpr uint32_t idesc_pv = umma_idesc(1, 1, N, tc::kKeys);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  TcSmem<G>& sm = *reinterpret_cast<TcSmem<G>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cta = blockIdx.x;
  if (tid == 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmK)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmV)) : "memory");
  }
  if (tid == 0) {
    for (int s_ = 0; s_ < SK; ++s_) {
      mbar_init(&sm.full_k[s_], 1);
      mbar_init(&sm.empty_k[s_], 1);
    }
    for (int s_ = 0; s_ < SV; ++s_) {
      mbar_init(&sm.full_v[s_], 1);
      mbar_init(&sm.empty_v[s_], 1);
    }
    for (int s_ = 0; s_ < 2; ++s_) {
      mbar_init(&sm.s_full[s_], 1);
      mbar_init(&sm.s_empty[s_], SW);
    }
    for (int s_ = 0; s_ < NPB; ++s_) {
      mbar_init(&sm.p_full[s_], SW);
      mbar_init(&sm.p_empty[s_], 1);
    }
    mbar_init(&sm.q_full, SW);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (p.trace != nullptr) p.trace[cta * kTracePoints + kTraceStart] = globaltimer();
  }
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the merge may be scheduled now: its CTAs take SMs as these CTAs leave,
  // and wait for this grid to complete before they read any partial
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the CTA's range of the cost space (as in the attention kernel)
  unsigned smid;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
  const int n_cta = p.hdr->n_cta, weighted = p.hdr->weighted;
  const long long T = p.hdr->total;
  int first_seg = p.first_seg[cta];
  int slot = cta;
  long long lo, hi;
  if (weighted) {
    if (tid == 0) {
      int c = (p.claim != nullptr && (int)smid < p.grid && atomicCAS(p.claim + smid, 0, 1) == 0) ? (int)smid : -1;
      for (int k = 0; c < 0 && k < n_cta; ++k)
        if (atomicCAS(p.claim + k, 0, 1) == 0) c = k;
      sm.last_flag = c;
    }
    __syncthreads();
    slot = sm.last_flag;
    if (slot < 0) return;
    lo = p.bounds[slot];
    hi = p.bounds[slot + 1];
    first_seg = p.first_seg[slot];
  } else {
    if (cta >= n_cta) return;
    lo = (long long)cta * T / n_cta;
    hi = (long long)(cta + 1) * T / n_cta;
  }
  // tensor memory for S[2] and O
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  volatile int* abort_flag = &sm.abort_flag;
  // every role walks the items from global memory (no shared copy: the base
  // puts them all past the cache)
  TileCursor cur;
  cur.w = Walker{first_seg, lo, hi, nullptr, first_seg - kItemCache, p.seg, p.nseg, false};
  cur.np = 0;
  cur.open(slot);

  if (warp == 0 || warp == 2) {
    // ---- the K stream (warp 0) and the V stream (warp 2)
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      if (warp == 0)
        tc_stream<SK>(p, &p.tmK, sm.k, sm.full_k, sm.empty_k, cur, slot, abort_flag, pol, p.counters);
      else
        tc_stream<SV>(p, &p.tmV, sm.v, sm.full_v, sm.empty_v, cur, slot, abort_flag, pol, nullptr);
    }
  } else if (warp == 1) {
    // ---- MMA issuer: QK of tile tq and PV of tile tp, whichever has its inputs
    if (lane == 0) {
      TileCursor cq = cur, cv = cur;
      int tq = 0, tp = 0;
      bool idle = false;
      unsigned long long idle0 = 0;
      while (cv.live) {
        bool prog = false;
        if (cq.live) {
          const int sb = tq & 1, st = tq % SK;
          if ((cq.i != 0 || mbar_test(&sm.q_full, (uint32_t)cq.np & 1u)) &&
              mbar_test(&sm.full_k[st], (uint32_t)(tq / SK) & 1u) &&
              (tq < 2 || mbar_test(&sm.s_empty[sb], (uint32_t)((tq >> 1) - 1) & 1u))) {
            tc_fence_after();
            if (tq == 0 && p.trace != nullptr) p.trace[cta * kTracePoints + kTraceFirstBox] = globaltimer();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const int half = ks >> 2, kin = ks & 3;
              const uint64_t a = umma_desc(smem_u32(sm.k[st][half]) + kin * 32, 16, 1024);
              const uint64_t b = umma_desc(smem_u32(sm.q[half]) + kin * 32, 16, 1024);
              umma(tmem + (uint32_t)(N * sb), a, b, idesc_qk, ks > 0 ? 1u : 0u);
            }
            umma_commit(&sm.s_full[sb]);
            umma_commit(&sm.empty_k[st]);
            ++tq;
            cq.step(slot);
            prog = true;
          }
        }
        if (tp < tq) {
          const int st = tp % SV, pb = tp % NPB;
          if (mbar_test(&sm.p_full[pb], (uint32_t)(tp / NPB) & 1u) &&
              mbar_test(&sm.full_v[st], (uint32_t)(tp / SV) & 1u)) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < tc::kKeys / 16; ++kk) {
              const uint64_t a = umma_desc(smem_u32(sm.v[st][0]) + kk * 2048, tc::kKeys * 128, 1024);
              const uint64_t b = umma_desc(smem_u32(sm.pw[pb][0]) + kk * 2048, tc::kKeys * 128, 1024);
              umma(tmem + kColO, a, b, idesc_pv, (cv.i > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&sm.empty_v[st]);
            umma_commit(&sm.p_empty[pb]);
            ++tp;
            cv.step(slot);
            prog = true;
          }
        }
        if (prog) {
          idle = false;
        } else {
          if (*abort_flag) break;
          const unsigned long long now = globaltimer();
          if (!idle) {
            idle = true;
            idle0 = now;
          } else if (now - idle0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(p.status, MAC_DEV_TIMEOUT);
            break;
          }
        }
      }
      // every MMA issued has completed before the tensor memory is released
      umma_commit(&sm.drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(&sm.drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  } else if (warp >= tc::kSoftWarp0) {
    // ---- softmax warps: warp 4 + 4 hh + wq owns TMEM lanes 32 wq .. 32 wq + 31
    // (the tile's keys) and heads [hh GH, hh GH + GH)
    constexpr int GH = G / (SW / 4);
    const int sw = warp - tc::kSoftWarp0, wq = sw & 3, hh = sw >> 2;
    const int ts = tid - tc::kSoftWarp0 * 32;  // 0 .. NT - 1
    const int k = 32 * wq + lane, hb = hh * GH;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * wq) << 16);
    if constexpr (2 * G < N) {
      // padding: columns 2G..N-1 of P^T and rows 2G..N-1 of the query stay zero
      if (hh == 0) {
#pragma unroll
        for (int pb = 0; pb < NPB; ++pb)
#pragma unroll
          for (int c = 2 * G / 8; c < 8; ++c)
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(sm.pw[pb][0]) + sw128_off(k, c * 8)) =
                make_uint4(0u, 0u, 0u, 0u);
      }
      for (int idx = ts; idx < 2 * (N - 2 * G); idx += NT) {
        const int row = 2 * G + (idx >> 1), half = idx & 1;
        unsigned char* qd = reinterpret_cast<unsigned char*>(sm.q[half]);
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(qd + sw128_off(row, c * 8)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // A failed wait flags the CTA's abort (every later wait then returns at
    // once) but the softmax warps still go through every tile and barrier of
    // their walk, so the named barriers always see all NT threads.
    bool ok = true;
    // per head of this warp: key sums, this key's scores and (16 heads at most,
    // 168 registers a thread) the running maxima; otherwise the maxima are read
    // from shared memory
    constexpr bool kMaxInRegs = GH <= 16 && SW == 8;
    float lsum[GH], sv[GH], mr[kMaxInRegs ? GH : 1];
#pragma unroll
    for (int j = 0; j < (kMaxInRegs ? GH : 1); ++j) mr[j] = -INFINITY;
    auto mget = [&](int j) __attribute__((always_inline)) {
      if constexpr (kMaxInRegs) return mr[j];
      else return sm.m[hb + j];
    };
    int t = 0;
    for (; cur.live; cur.i = cur.ntile - 1, cur.step(slot)) {
      const Piece& pc = cur.pc;
      // the piece's query: rows [0, G) high parts, [G, 2G) residuals; the
      // previous piece's products are done (every S and O of it was read)
      for (int idx = ts; idx < 4 * G; idx += NT) {
        const int row = idx >> 1, half = idx & 1, h = row < G ? row : row - G;
        const float* qsrc = p.qrot + ((size_t)pc.unit * G + h) * D + half * 64;
        unsigned char* qd = reinterpret_cast<unsigned char*>(sm.q[half]);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 a = *reinterpret_cast<const float4*>(qsrc + c * 8);
          const float4 b4 = *reinterpret_cast<const float4*>(qsrc + c * 8 + 4);
          uint4 vh;
          vh.x = pack_bf16(a.x, a.y);
          vh.y = pack_bf16(a.z, a.w);
          vh.z = pack_bf16(b4.x, b4.y);
          vh.w = pack_bf16(b4.z, b4.w);
          if (row >= G) {
            vh.x = pack_bf16_residual(a.x, a.y, vh.x);
            vh.y = pack_bf16_residual(a.z, a.w, vh.y);
            vh.z = pack_bf16_residual(b4.x, b4.y, vh.z);
            vh.w = pack_bf16_residual(b4.z, b4.w, vh.w);
          }
          *reinterpret_cast<uint4*>(qd + sw128_off(row, c * 8)) = vh;
        }
      }
      if (ts < G) sm.m[ts] = -INFINITY;
#pragma unroll
      for (int j = 0; j < GH; ++j) lsum[j] = 0.f;
#pragma unroll
      for (int j = 0; j < (kMaxInRegs ? GH : 1); ++j) mr[j] = -INFINITY;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full);
      for (int i = 0; i < cur.ntile; ++i, ++t) {
        const int sb = t & 1, st = t % SV;
        const int key = pc.kb0 + i * tc::kKeys + k;
        const bool valid = key >= pc.k0 && key < pc.k1;
        ok &= mbar_wait(&sm.s_full[sb], (uint32_t)(t >> 1) & 1u, abort_flag, p.status);
        __syncwarp();
        tc_fence_after();
        // this key's scores for the warp's heads: high-part plus residual column
        tmem_heads<GH>(lane_base + (uint32_t)(N * sb + hb), lane_base + (uint32_t)(N * sb + G + hb), sv);
#pragma unroll
        for (int j = 0; j < GH; ++j) sv[j] = valid ? sv[j] : -INFINITY;
        // S is in registers: its buffer takes the product of tile t + 2
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_empty[sb]);
        int grow = 0;
#pragma unroll
        for (int j = 0; j < GH; ++j) grow |= sv[j] > mget(j) + 8.f ? 1 : 0;
        if (softmax_sync_or<NT>(grow)) {
          // some head's maximum grew: new maxima, O and the sums rescaled
#pragma unroll
          for (int j = 0; j < GH; ++j) {
            float x = sv[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
            if (lane == 0) sm.red[wq][hb + j] = x;
          }
          softmax_sync<NT>();
          if (ts < G) {
            const float mo = sm.m[ts];
            const float mn = fmaxf(mo, fmaxf(fmaxf(sm.red[0][ts], sm.red[1][ts]), fmaxf(sm.red[2][ts], sm.red[3][ts])));
            sm.red[0][ts] = mo == -INFINITY ? 0.f : ex2(mo - mn);  // scale of the old sums
            sm.m[ts] = mn;
          }
          softmax_sync<NT>();
          if (i > 0) {
            // O holds the previous tile's product once that is done
            ok &= mbar_wait(&sm.p_empty[(t - 1) % NPB], (uint32_t)((t - 1) / NPB) & 1u, abort_flag, p.status);
            __syncwarp();
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {  // high-part columns, then residual columns
              const uint32_t ta = lane_base + kColO + (uint32_t)(part * G + hb);
              uint32_t r[GH];
              tmem_ldn<GH>(ta, r);
              tmem_ld_wait<GH>(r);
#pragma unroll
              for (int j = 0; j < GH; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * sm.red[0][hb + j]);
              tmem_stn<GH>(ta, r);
              asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            }
          }
#pragma unroll
          for (int j = 0; j < GH; ++j) lsum[j] *= sm.red[0][hb + j];
#pragma unroll
          for (int j = 0; j < (kMaxInRegs ? GH : 1); ++j) mr[j] = sm.m[hb + j];
          softmax_sync<NT>();
        }
        // this key's weights into row k of P^T buffer t % NPB (free once the
        // product of tile t - NPB is done): high parts at column h, residuals
        // at column G + h
        if (t >= NPB) ok &= mbar_wait(&sm.p_empty[t % NPB], (uint32_t)((t / NPB) - 1) & 1u, abort_flag, p.status);
        __syncwarp();
        tc_fence_after();
        unsigned char* const pw0 = reinterpret_cast<unsigned char*>(sm.pw[t % NPB][0]);
#pragma unroll
        for (int c = 0; c < GH / 8; ++c) {
          float x[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            x[j] = valid ? ex2(sv[c * 8 + j] - mget(c * 8 + j)) : 0.f;
            lsum[c * 8 + j] += x[j];
          }
          uint4 vh, vr;
          vh.x = pack_bf16(x[0], x[1]);
          vh.y = pack_bf16(x[2], x[3]);
          vh.z = pack_bf16(x[4], x[5]);
          vh.w = pack_bf16(x[6], x[7]);
          vr.x = pack_bf16_residual(x[0], x[1], vh.x);
          vr.y = pack_bf16_residual(x[2], x[3], vh.y);
          vr.z = pack_bf16_residual(x[4], x[5], vh.z);
          vr.w = pack_bf16_residual(x[6], x[7], vh.w);
          const int ch = hb + c * 8, cr = G + ch;
          *reinterpret_cast<uint4*>(pw0 + (ch >> 6) * (tc::kKeys * 128) + sw128_off(k, ch & 63)) = vh;
          *reinterpret_cast<uint4*>(pw0 + (cr >> 6) * (tc::kKeys * 128) + sw128_off(k, cr & 63)) = vr;
        }
        if (!valid && hh == 0) {
          // rows outside the piece: zero V (they may hold anything, NaN included)
          ok &= mbar_wait(&sm.full_v[st], (uint32_t)(t / SV) & 1u, abort_flag, p.status);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint4* vrow = reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(sm.v[st][hf]) + k * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) vrow[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[t % NPB]);
      }
      // the piece's partial: O (after its last product), running maxima, sums
      ok &= mbar_wait(&sm.p_empty[(t - 1) % NPB], (uint32_t)((t - 1) / NPB) & 1u, abort_flag, p.status);
      __syncwarp();
      tc_fence_after();
      float* dst = p.part + (size_t)pc.pidx * partial_floats(G, D);
      tmem_heads<GH>(lane_base + kColO + hb, lane_base + kColO + G + hb, sv);
#pragma unroll
      for (int j = 0; j < GH; ++j) {
        const int h = hb + j;  // element (h, d = k)
        dst[(h >> 3) * PFc + (h & 7) * D + k] = sv[j];
      }
#pragma unroll
      for (int j = 0; j < GH; ++j) {
        float v = lsum[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        if (lane == 0) sm.red[wq][hb + j] = v;
      }
      softmax_sync<NT>();
      if (ts < G) {
        float* dc = dst + (ts >> 3) * PFc;
        dc[GDc + (ts & 7)] = sm.m[ts];
        dc[GDc + 8 + (ts & 7)] = sm.red[0][ts] + sm.red[1][ts] + sm.red[2][ts] + sm.red[3][ts];
      }
      tc_fence_before();
      softmax_sync<NT>();
    }
    (void)ok;
  }
  // everyone is done with the tensor memory (the issuer drained its MMAs)
  // and the streams' copies have landed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && p.trace != nullptr) {
    const unsigned long long now = globaltimer();
    p.trace[cta * kTracePoints + kTraceRange] = now;
    p.trace[cta * kTracePoints + kTraceEnd] = now;
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
  }
}

// Merge of the tcgen05 path's partials, one CTA per unit (blockIdx.x) and
// pair of heads (blockIdx.y): warp w takes head w & 1 of the pair and every
// fourth partial from w >> 1 on (segment A's and B's in one sequence, KB in
// flight per lane), lane l the elements 4l .. 4l + 3; the four warps of a
// head then combine their states through shared memory.  Segment A's
// partials with the reused state (on a hit) give the new prefix state over
// [0, c_t), stored in ring slot dst; that state and segment B's partials give
// the output.
template <int GF>
__global__ void __launch_bounds__(kAttnThreads) mac_tc_merge_kernel(const __grid_constant__ AttendParams p) {
  constexpr int D = 128, G = GF, PFc = 8 * D + 16, KB = 10, NS = kAttnThreads / 64;  // NS warps per head
  __shared__ float4 so[2][NS][2][32];  // [head][warp][A|B][lane]: o
  __shared__ float sml[2][NS][2][2];   // [head][warp][A|B]: m, l
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int u = blockIdx.x, hp = threadIdx.x >> 5 & 1, part = threadIdx.x >> 6, lane = threadIdx.x & 31;
  const UnitPlan* const pp = p.plan + u;
  if (__ldcg(&pp->bad)) return;
  const Segment sA = load_segment(p.seg + 2 * u), sB = load_segment(p.seg + 2 * u + 1);
  const size_t PF = partial_floats(G, D);
  const int h = blockIdx.y * 2 + hp, ch = h >> 3, hl = h & 7, d0 = lane * 4;
  const int nA = sA.kind < 0 ? 0 : sA.npieces, nB = sB.kind < 0 ? 0 : sB.npieces;
  const float* const baseA = p.part + (size_t)sA.pbase * PF + (size_t)ch * PFc;
  const float* const baseB = p.part + (size_t)sB.pbase * PF + (size_t)ch * PFc;
  // segment A folds into (M, L, O), segment B into (MB, LB, OB)
  float M = -INFINITY, L = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
  float MB = -INFINITY, LB = 0.f, OB[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
  for (int i0 = part; i0 < nA + nB; i0 += KB * NS) {
    float4 ov[KB];
    float mv[KB], lv[KB];
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int i = i0 + k * NS;
      if (i < nA + nB) {
        const float* q = i < nA ? baseA + (size_t)i * PF : baseB + (size_t)(i - nA) * PF;
        ov[k] = __ldcg(reinterpret_cast<const float4*>(q + hl * D + d0));
        mv[k] = __ldcg(q + 8 * D + hl);
        lv[k] = __ldcg(q + 8 * D + 8 + hl);
      }
    }
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int i = i0 + k * NS;
      if (i < nA)
        fold_state<4>(M, L, O, mv[k], lv[k], &ov[k].x);
      else if (i < nA + nB)
        fold_state<4>(MB, LB, OB, mv[k], lv[k], &ov[k].x);
    }
  }
  so[hp][part][0][lane] = make_float4(O[0], O[1], O[2], O[3]);
  so[hp][part][1][lane] = make_float4(OB[0], OB[1], OB[2], OB[3]);
  if (lane == 0) {
    sml[hp][part][0][0] = M;
    sml[hp][part][0][1] = L;
    sml[hp][part][1][0] = MB;
    sml[hp][part][1][1] = LB;
  }
  __syncthreads();
  if (part != 0) return;
  // warps 0 and 1: the head's four states, in warp order
#pragma unroll
  for (int w = 1; w < NS; ++w) {
    float4 a = so[hp][w][0][lane], c = so[hp][w][1][lane];
    fold_state<4>(M, L, O, sml[hp][w][0][0], sml[hp][w][0][1], &a.x);
    fold_state<4>(MB, LB, OB, sml[hp][w][1][0], sml[hp][w][1][1], &c.x);
  }
  const int hit = __ldcg(&pp->hit), src = __ldcg(&pp->src_slot), dst = __ldcg(&pp->dst_slot), end = __ldcg(&pp->end);
  // new prefix state: segment A, plus the reused state on a hit
  const size_t Wp1 = (size_t)p.W + 1;
  if (hit) {
    const size_t e = ((size_t)u * Wp1 + src) * G + h;
    const float rm = __ldcg(p.ring_m + e) * kLog2e, rl = __ldcg(p.ring_l + e);
    const float Mn = fmaxf(M, rm), Mu = Mn == -INFINITY ? 0.f : Mn;
    const float a = ex2(M - Mu), c = ex2(rm - Mu);
    L = L * a + rl * c;
#pragma unroll
    for (int j = 0; j < 4; ++j) O[j] = O[j] * a + ring_o_at(p.ring_o, e * D + d0 + j, p.ring_bf16) * rl * c;
    M = Mn;
  }
  const size_t ds = (size_t)u * Wp1 + dst;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    ring_o_put(p.ring_o, (ds * G + h) * D + d0 + j, L > 0.f ? __fdividef(O[j], L) : 0.f, p.ring_bf16);
  if (lane == 0) {
    p.ring_m[ds * G + h] = L > 0.f ? M * kLn2 : -INFINITY;
    p.ring_l[ds * G + h] = L;
  }
  // output: the prefix state and segment B (the tail)
  const float M2 = fmaxf(M, MB), M2u = M2 == -INFINITY ? 0.f : M2;
  const float a0 = ex2(M - M2u), aB = ex2(MB - M2u);
  const float L2 = L * a0 + LB * aB;  // >= 1: every unit attends at least one key
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  const size_t orow = (size_t)b * p.Hq + (size_t)kvh * G + h;
  float4 o4;
  o4.x = __fdividef(O[0] * a0 + OB[0] * aB, L2);
  o4.y = __fdividef(O[1] * a0 + OB[1] * aB, L2);
  o4.z = __fdividef(O[2] * a0 + OB[2] * aB, L2);
  o4.w = __fdividef(O[3] * a0 + OB[3] * aB, L2);
  *reinterpret_cast<float4*>(p.out + orow * D + d0) = o4;
  if (lane == 0) p.lse[orow] = (M2 + __log2f(L2)) * kLn2;
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    p.ring_pos[(size_t)u * Wp1 + dst] = end - 1;
    if (p.counters != nullptr) atomicAdd(p.counters + kCountMerged, 1ull);
  }
}

}  // namespace

namespace {
template <int GF>
constexpr size_t tc_smem_bytes() { return sizeof(TcSmem<GF>) + 1024; }  // + alignment of the tiles to 1 KB
static_assert(tc_smem_bytes<16>() <= 232448 && tc_smem_bytes<32>() <= 232448 && tc_smem_bytes<64>() <= 232448,
              "the tcgen05 kernel's shared memory fits one CTA");
template <int GF>
cudaError_t tc_prepare() {
  return cudaFuncSetAttribute(mac_attend_tc_kernel<GF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)tc_smem_bytes<GF>());
}
template <int GF>
cudaError_t tc_launch(cudaLaunchConfig_t& cfg, const AttendParams& p, int U, cudaStream_t s) {
  cfg.dynamicSmemBytes = tc_smem_bytes<GF>();
  cfg.blockDim = dim3(tc::threads(GF));
  cudaError_t e = cudaLaunchKernelEx(&cfg, mac_attend_tc_kernel<GF>, p);
  cfg.blockDim = dim3(kAttnThreads);
  if (e != cudaSuccess) return e;
  // the merge may start while the products drain (it waits on them first)
  cfg.gridDim = dim3(U, GF / 2);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, mac_tc_merge_kernel<GF>, p);
}
}  // namespace

cudaError_t attend_tc_prepare(int G) {
  if (G == 16) return tc_prepare<16>();
  if (G == 32) return tc_prepare<32>();
  if (G == 64) return tc_prepare<64>();
  return cudaErrorInvalidValue;
}

cudaError_t launch_attend_tc(const AttendParams& p, int grid, cudaStream_t s) {
  // Programmatic stream serialization: the products may be scheduled while
  // the match kernel drains, the merge while the products drain; each waits
  // (griddepcontrol.wait) before it reads what its predecessor wrote.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int U = p.nseg / 2;
  if (p.G == 16) return tc_launch<16>(cfg, p, U, s);
  if (p.G == 32) return tc_launch<32>(cfg, p, U, s);
  if (p.G == 64) return tc_launch<64>(cfg, p, U, s);
  return cudaErrorInvalidValue;
}

}  // namespace mac
