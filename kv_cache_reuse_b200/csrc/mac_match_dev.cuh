// mac_match_dev.cuh -- device code of the match stage shared by the match
// kernels (mac_match.cu) and the one-launch step (mac_step.cu).
//
// "MAC-Attention: a Match-Amend-Complete Scheme for Fast and Accurate
// Attention Computation", page 1 (abstract): the match stage compares the
// current query, before RoPE, by L2 distance with a short window of recent
// queries whose attention results can be reused.  One CTA handles one (sequence, KV head)
// unit:
//   1. distance of the current pre-RoPE query group (G heads) to every
//      window entry: mean over heads of the squared L2 distance, summed in
//      fp32 as sum((a - b)^2) -- the expanded |a|^2 + |b|^2 - 2ab form would
//      cancel catastrophically for near-repeats;
//   2. argmin with ties to the more recent entry, hit iff the minimum is
//      strictly below tau; NaN distances never win (with per-head matching,
//      steps 1-3 run per query head: its own distance, entry and c_s, the
//      unit's fresh range starting at the smallest c_s);
//   3. key ranges: the reused prefix ends at c_s = max(0, p_s - band) (the
//      amend band starts there), the stored prefix of this step ends at
//      c_t = max(0, p_t - band), and the tail runs to p_t (band here is the
//      configured band minus the cut mode, so that with cut mode 1 the band
//      ends at the position itself);
//   4. RoPE of the query to rope_pos (fp64 angle), pre-scaled by
//      log2(e)/sqrt(D) so the attention kernel works in exp2 units;
//   5. the query enters the ring slot n mod (W+1) (W+1 slots: the slot
//      written is never one the window can read this step), in fp32 or
//      rounded to bf16.
// The last CTA to finish lays every unit's work items (one whole item, or
// two split key segments) end to end in a cost space (each non-empty item
// weighs its keys plus a fixed per-piece cost) and splits that space over
// the attention kernel's CTAs -- evenly, or on large steps in proportion to
// each SM's learned streaming rate -- so a batch mixing short hit ranges
// with whole-context misses is balanced by time rather than by keys.  No CTA
// waits for another: the last arrival does the work.
#pragma once
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include <cuda_bf16.h>

#include "mac_internal.cuh"

#include "../../include/mac.h"

namespace mac {
namespace {

constexpr double kLog2eD = 1.4426950408889634;
constexpr double kInvTwoPi = 0.15915494309189535;
constexpr double kTwoPiHi = 6.2831853069365025;    // 2*pi with the low 21 mantissa bits cleared
constexpr double kTwoPiLo = 2.430840202602477e-10;   // 2*pi - kTwoPiHi

// Four window elements: fp32 as they are, bf16 (two per 32-bit word, the
// first in the low half) widened exactly.
__device__ __forceinline__ float4 widen4(const float4& v) { return v; }
__device__ __forceinline__ float4 widen4(const uint2& v) {
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                     __uint_as_float(v.y & 0xffff0000u));
}
// Four fp32 values rounded to bf16 (nearest even), packed as widen4 reads them.
__device__ __forceinline__ uint2 narrow4(const float4& v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive scan of one value per thread over a block of kMatchThreads.
__device__ long long block_exclusive_scan(long long v, long long* total, long long* sbuf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sbuf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < kMatchThreads / 32 ? sbuf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kMatchThreads / 32) sbuf[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  long long before = warp > 0 ? sbuf[warp - 1] : 0;
  *total = sbuf[kMatchThreads / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// CTA holding cost-space offset x when the space [0, T) is split over N CTAs
// as [c*T/N, (c+1)*T/N): the largest c with floor(c*T/N) <= x.
// ceil(a / b) for 0 <= a < 2^62 and b > 0, without a 64-bit integer
// division: an fp64 estimate (off by at most a few units) corrected exactly.
__device__ __forceinline__ long long ceil_div(long long a, long long b, double rb) {
  long long q = (long long)((double)a * rb);
  while (q > 0 && q * b > a) --q;
  while ((q + 1) * b <= a) ++q;  // q = floor(a / b)
  return q + (q * b < a ? 1 : 0);
}
__device__ __forceinline__ int cta_of(long long x, long long T, int N, double rT) {
  return (int)ceil_div((x + 1) * (long long)N, T, rT) - 1;
}

static_assert(kMaxWindow + 1 <= 0x7ff, "ring slots must fit the 11-bit fields of a whole item");

// sin and cos of the RoPE angle pos * inv_freq, computed in fp64 and reduced
// to [-pi, pi] with a two-constant Cody-Waite reduction (2*pi = C1 + C2, C1
// carrying 32 significant bits so k*C1 is exact for |k| < 2^21) before sincos.
__device__ __forceinline__ void rope_sincos(int pos, double inv_freq, double* sn, double* cs) {
  const double ang = (double)pos * inv_freq;
  const double k = rint(ang * kInvTwoPi);
  double rr = ang;
  if (fabs(k) < 2097152.0) {
    rr = fma(-k, kTwoPiHi, ang);
    rr = fma(-k, kTwoPiLo, rr);
  }
  sincos(rr, sn, cs);
}

__device__ void build_segments(const MatchParams& p, int U, double cw_c) {
  __shared__ long long sbuf[kMatchThreads / 32];
  const int tid = threadIdx.x;
  const int nseg = 2 * U;
  const long long cost = p.piece_cost;
  // pass 1: item kinds, keys and cost-space offsets
  long long carry = 0;
  long long r_flat = 0;  // this thread's item, kept for pass 2 when nseg <= kMatchThreads
  int r_len = 0, r_kind = kItemEmpty;
  for (int base = 0; base < nseg; base += kMatchThreads) {
    const int s = base + tid;
    int len = 0, key0 = 0, kind = kItemEmpty, cut = 0, packed = 0;
    long long wlen = 0;
    if (s < nseg) {
      const UnitPlan* pl = p.plan + (s >> 1);
      const int bad = __ldcg(&pl->bad);
      if (!bad) {
        const int start = __ldcg(&pl->start), c = __ldcg(&pl->cut), end = __ldcg(&pl->end);
        if (end - start <= p.unit_max) {
          if ((s & 1) == 0) {  // the whole unit in slot 2u
            kind = kItemWhole;
            len = end - start;
            key0 = start;
            cut = c;
            // the CTA doing it also needs hit, reused slot and written slot
            const int hit = __ldcg(&pl->hit), src = __ldcg(&pl->src_slot), dst = __ldcg(&pl->dst_slot);
            // slots are below kMaxWindow + 1 <= 2^11: masked, neither field can spill into the other
            packed = (hit ? 1 : 0) | ((hit && src >= 0 ? src & 0x7ff : 0) << 1) | ((dst & 0x7ff) << 12);
          }
        } else {
          len = (s & 1) ? end - c : c - start;
          key0 = (s & 1) ? c : start;
          kind = len > 0 ? ((s & 1) ? kItemB : kItemA) : kItemEmpty;
        }
        if (kind != kItemEmpty) wlen = (long long)len + cost;
      }
    }
    long long tot;
    long long ex = block_exclusive_scan(wlen, &tot, sbuf);
    if (s < nseg) {
      const bool split = kind == kItemA || kind == kItemB;
      p.seg[s].flat = carry + ex + (split ? cost : 0);
      r_flat = carry + ex + (split ? cost : 0);
      r_len = kind == kItemEmpty ? 0 : len;
      r_kind = kind;
      p.seg[s].len = kind == kItemEmpty ? 0 : len;
      p.seg[s].key0 = key0;
      p.seg[s].kind = kind;
      p.seg[s].pbase = cut;  // whole items keep their cut here; split items overwrite it below
      if (kind == kItemWhole) p.seg[s].npieces = packed;
    }
    carry += tot;
  }
  const long long T = carry;
  int N = 0;
  if (T > 0) {
    long long want = (T + p.min_keys - 1) / p.min_keys;
    N = (int)(want < (long long)p.grid ? want : (long long)p.grid);
    if (N < 1) N = 1;
  }
  const double rT = T > 0 ? 1.0 / (double)T : 0.0;
  // weighted split: range c from the cumulative shares of the SMs' rates
  __shared__ long long sbound[kMatchThreads + 1];
  const bool weighted =
      p.cw != nullptr && N == p.grid && p.grid < kMatchThreads && T >= kWeightMinCost * (long long)p.grid;
  if (weighted) {
    if (tid <= N) sbound[tid] = tid == 0 ? 0 : (tid == N ? T : (long long)((double)T * cw_c));
    __syncthreads();
    if (tid <= N) p.bounds[tid] = sbound[tid];
  }
  if (p.claim != nullptr)
    for (int c = tid; c < p.grid; c += kMatchThreads) p.claim[c] = 0;
  // CTA holding offset x: the largest c with start(c) <= x (weighted: a
  // binary search of the range starts, at most 8 steps for 148 ranges)
  auto owner = [&](long long x) -> int {
    if (!weighted) return cta_of(x, T, N, rT);
    int lo = 0, hi = N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sbound[mid] <= x)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  };
  // first CTA whose range starts at or after x
  auto first_from = [&](long long x) -> long long {
    if (!weighted) return ceil_div(x * N, T, rT);
    return x <= 0 ? 0 : owner(x - 1) + 1;
  };
  __syncthreads();
  // pass 2: owning / first CTA, partial slots, and each CTA's first item
  long long pcarry = 0;
  for (int base = 0; base < nseg; base += kMatchThreads) {
    const int s = base + tid;
    int np = 0, first = 0, kind = kItemEmpty, len = 0;
    long long F = 0;
    if (s < nseg) {
      if (nseg <= kMatchThreads) {
        F = r_flat;
        len = r_len;
        kind = r_kind;
      } else {
        F = p.seg[s].flat;
        len = p.seg[s].len;
        kind = p.seg[s].kind;
      }
      if (kind == kItemA || kind == kItemB) {
        first = owner(F);
        np = owner(F + len - 1) - first + 1;
      } else if (kind == kItemWhole) {
        first = owner(F);
      }
    }
    long long tot;
    long long ex = block_exclusive_scan(np, &tot, sbuf);
    // units own items (2u, 2u+1): adjacent threads of one warp
    const int np_next = __shfl_down_sync(0xffffffffu, np, 1);
    if (s < nseg) {
      p.seg[s].first_cta = first;
      if (kind != kItemWhole) {
        p.seg[s].npieces = np;
        p.seg[s].pbase = (int)(pcarry + ex);
      }
      if ((s & 1) == 0) p.plan[s >> 1].expected = np + np_next;
      // CTAs whose range starts inside this item's cost extent [Fw, Fe)
      // begin their walk here (even split: lo_c = floor(c*T/N) lies in it
      // iff ceil(Fw*N/T) <= c < ceil(Fe*N/T))
      if (kind != kItemEmpty && N > 0) {
        const bool split = kind == kItemA || kind == kItemB;
        const long long Fw = split ? F - cost : F;
        const long long Fe = Fw + len + cost;
        const long long ca = first_from(Fw), cb = first_from(Fe);
        for (long long c = ca; c < cb && c < N; ++c) p.first_seg[c] = s;
      }
    }
    pcarry += tot;
  }
  if (tid == 0) {
    p.hdr->total = T;
    p.hdr->n_cta = N;
    p.hdr->weighted = weighted ? 1 : 0;
  }
}

// Block-wide sum of one double per thread; every thread gets the same value
// (the warps' parts are added in one fixed order).
__device__ double block_sum_d(double v, double* sbuf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sbuf[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kMatchThreads / 32; ++w) t += sbuf[w];
  return t;
}

// The split table of the one-launch step, built by the last CTA to finish
// matching (one CTA of kMatchThreads threads, grid <= kMatchThreads).  Every
// unit whose fresh range holds at most unit_max keys was done whole by the
// CTA that matched it (unit u on CTA u mod grid); only the other units' two
// key segments are laid end to end here, in a cost space where each weighs
// its keys plus the fixed piece cost.  The space is cut into one range per
// slot -- per SM on large steps (each SM's range sized by its learned
// streaming rate), per CTA otherwise -- such that each slot's whole-unit work
// (its keys plus an eighth of the piece cost) plus its range comes out
// proportional to its weight: with weights w_r and whole work h_r, range r
// holds max(0, w_r t - h_r) cost units, t chosen so
// the ranges add up to the split work (water filling).  Small steps use
// only the last ceil(S / min_keys) CTAs.  Empty ranges are dropped and the
// rest numbered in slot order (their rank): the items' first range and
// piece counts, the partial-result slots and first_seg are in rank space.
// Shared scratch of build_split_table (the caller places it in memory that
// is idle during the build).
struct SplitScratch {
  long long sbuf[kMatchThreads / 32];
  double dbuf[kMatchThreads / 32];
  unsigned long long wsum[kMatchThreads];  // whole-unit work of each CTA
  int cta_on[kMatchThreads];               // CTA resident on each SM
  long long sbound[kMatchThreads + 1];     // range starts, by rank
};

__device__ void build_split_table(const MatchParams& p, int U, int grid, const int* smid_of, int* rank_of,
                                  SplitScratch& sc) {
  long long* const sbuf = sc.sbuf;
  double* const dbuf = sc.dbuf;
  unsigned long long* const wsum = sc.wsum;
  int* const cta_on = sc.cta_on;
  long long* const sbound = sc.sbound;
  const int tid = threadIdx.x;
  const int nseg = 2 * U;
  const long long cost = p.piece_cost;
  // the SM map and (when the items fit one pass) the plans in one round of loads
  const int sm_ = tid < grid ? __ldcg(smid_of + tid) : -1;
  UnitPlan pre;
  pre.bad = 1;
  if (nseg <= kMatchThreads && tid < nseg) {
    const UnitPlan* pl = p.plan + (tid >> 1);
    pre.bad = __ldcg(&pl->bad);
    pre.start = __ldcg(&pl->start);
    pre.cut = __ldcg(&pl->cut);
    pre.end = __ldcg(&pl->end);
  }
  wsum[tid] = 0;
  cta_on[tid] = -1;
  __syncthreads();
  if (sm_ >= 0 && sm_ < grid) cta_on[sm_] = tid;
  __syncthreads();
  // ranges can be keyed by SM only if the CTAs sit on grid distinct SMs
  // with ids below grid (otherwise every slot is a CTA)
  const bool by_sm = __syncthreads_count(tid < grid && cta_on[tid] >= 0) == grid;
  // pass 1: the split items' keys and cost offsets; whole units' cost to their CTA
  long long carry = 0;
  long long r_flat = 0;
  int r_len = 0, r_kind = kItemEmpty;
  for (int base = 0; base < nseg; base += kMatchThreads) {
    const int s = base + tid;
    int len = 0, key0 = 0, kind = kItemEmpty, cut = 0;
    long long wlen = 0;
    if (s < nseg) {
      UnitPlan pl;
      if (nseg <= kMatchThreads) {
        pl = pre;
      } else {
        const UnitPlan* pp = p.plan + (s >> 1);
        pl.bad = __ldcg(&pp->bad);
        pl.start = __ldcg(&pp->start);
        pl.cut = __ldcg(&pp->cut);
        pl.end = __ldcg(&pp->end);
      }
      if (!pl.bad) {
        const int start = pl.start, c = pl.cut, end = pl.end;
        if (end - start <= p.unit_max) {
          // a whole unit delays its CTA's range by about its keys plus an eighth
          // of a piece's fixed cost (traced: a hit unit of ~270 keys holds its
          // CTA ~5 us, the time to stream ~430 keys on one SM)
          if ((s & 1) == 0) atomicAdd(&wsum[(s >> 1) % grid], (unsigned long long)(end - start + cost / 8));
        } else {
          len = (s & 1) ? end - c : c - start;
          key0 = (s & 1) ? c : start;
          kind = len > 0 ? ((s & 1) ? kItemB : kItemA) : kItemEmpty;
          cut = c;
        }
        if (kind != kItemEmpty) wlen = (long long)len + cost;
      }
    }
    long long tot;
    const long long ex = block_exclusive_scan(wlen, &tot, sbuf);
    if (s < nseg) {
      Segment sg;
      sg.flat = carry + ex + (kind != kItemEmpty ? cost : 0);
      sg.len = kind == kItemEmpty ? 0 : len;
      sg.key0 = key0;
      sg.first_cta = 0;
      sg.pbase = cut;
      sg.npieces = 0;
      sg.kind = kind;
      p.seg[s] = sg;
      r_flat = sg.flat;
      r_len = sg.len;
      r_kind = kind;
    }
    carry += tot;
  }
  const long long S = carry;
  __syncthreads();
  if (S == 0) {  // every unit whole (or invalid): no ranges
    if (tid < grid) rank_of[tid] = -1;
    if (tid == 0) {
      p.hdr->total = 0;
      p.hdr->n_cta = 0;
      p.hdr->weighted = 0;
    }
    return;
  }
  const bool weighted = by_sm && p.cw != nullptr && grid <= kMatchThreads && S >= kWeightMinCost * (long long)grid;
  int neff = grid;
  if (!weighted) {
    const long long want = (S + p.min_keys - 1) / p.min_keys;
    neff = want < (long long)grid ? (int)want : grid;
    if (neff < 1) neff = 1;
  }
  // slot r = tid: its weight and its CTA's whole-unit work
  const bool active = tid < grid && (weighted || tid >= grid - neff);
  double om = 0.0;
  double h = 0.0;
  if (tid < grid) {
    om = weighted ? __ldcg(p.cw + tid + 1) - __ldcg(p.cw + tid) : 1.0;
    if (!(om > 1e-9)) om = 1e-9;
    const int c = weighted ? cta_on[tid] : tid;
    h = c >= 0 ? (double)wsum[c] : 0.0;
  }
  // water filling: t = (S + sum of h over the filled slots) / (sum of their weights)
  bool in = active;
  double t = 0.0;
#pragma unroll 1
  for (int it = 0; it < 8; ++it) {
    const double sh = block_sum_d(in ? h : 0.0, dbuf);
    const double so = block_sum_d(in ? om : 0.0, dbuf);
    t = so > 0.0 ? ((double)S + sh) / so : 0.0;
    const bool next = active && om * t > h;
    const int changed = __syncthreads_or(next != in);  // the same answer in every thread
    in = next;
    if (!changed) break;
  }
  const long long ri = active ? (long long)fmax(0.0, om * t - h) : 0;
  long long tot_r;
  const long long pr = block_exclusive_scan(ri, &tot_r, sbuf);
  // integer range ends, scaled so that the last one is S exactly
  long long st_r = 0, en_r = 0;
  if (tid < grid) {
    if (tot_r > 0) {
      st_r = (long long)((__int128)pr * S / tot_r);
      en_r = (long long)((__int128)(pr + ri) * S / tot_r);
    } else if (tid == grid - 1) {  // nothing was filled (cannot happen for S > 0): one range
      en_r = S;
    }
  }
  const int nonempty = (tid < grid && en_r > st_r) ? 1 : 0;
  long long nr;
  const int rank = (int)block_exclusive_scan(nonempty, &nr, sbuf);
  const int N = (int)nr;
  if (tid < grid) rank_of[tid] = nonempty ? rank : -1;
  if (nonempty) sbound[rank] = st_r;
  if (tid == 0) {
    sbound[N] = S;
  }
  __syncthreads();
  for (int k = tid; k <= N; k += kMatchThreads) p.bounds[k] = sbound[k];
  // range (by rank) holding cost offset x: the largest r with start(r) <= x
  auto owner = [&](long long x) -> int {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sbound[mid] <= x)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  };
  auto first_from = [&](long long x) -> long long { return x <= 0 ? 0 : owner(x - 1) + 1; };
  // pass 2: first range, pieces and partial slots of each split item; each range's first item
  long long pcarry = 0;
  for (int base = 0; base < nseg; base += kMatchThreads) {
    const int s = base + tid;
    int np = 0, first = 0, kind = kItemEmpty, len = 0;
    long long F = 0;
    if (s < nseg) {
      if (nseg <= kMatchThreads) {
        F = r_flat;
        len = r_len;
        kind = r_kind;
      } else {
        F = p.seg[s].flat;
        len = p.seg[s].len;
        kind = p.seg[s].kind;
      }
      if (kind == kItemA || kind == kItemB) {
        first = owner(F);
        np = owner(F + len - 1) - first + 1;
      }
    }
    long long tot;
    const long long ex = block_exclusive_scan(np, &tot, sbuf);
    const int np_next = __shfl_down_sync(0xffffffffu, np, 1);  // items 2u, 2u+1: adjacent lanes
    if (s < nseg) {
      p.seg[s].first_cta = first;
      p.seg[s].npieces = np;
      p.seg[s].pbase = (int)(pcarry + ex);
      if ((s & 1) == 0) p.plan[s >> 1].expected = np + np_next;
      if (kind == kItemA || kind == kItemB) {
        const long long Fw = F - cost, Fe = F + len;
        const long long ca = first_from(Fw), cb = first_from(Fe);
        for (long long c = ca; c < cb && c < N; ++c) p.first_seg[c] = s;
      }
    }
    pcarry += tot;
  }
  if (tid == 0) {
    p.hdr->total = S;
    p.hdr->n_cta = N;
    p.hdr->weighted = weighted ? 1 : 0;
  }
}

// GP: the query group padded to 4 or 8 heads (register and shared-memory
// shapes); the real group G <= GP sets every global layout.  GF = G for the
// variants built for one group size (4, 8), 0 for a run-time G (p.G).
// PH: one decision per query head (per-head matching).  RB: the window's
// queries are stored in bf16.
// Shared memory of the match stage of one unit.
template <int D, int GP, bool PH>
struct MatchSmem {
  alignas(16) float sq[GP * D];
  float sdist[PH ? GP : 1][kMaxWindow];  // [decision][age]: one row, or one per head (PH)
  int spos[kMaxWindow];
  int sslot[kMaxWindow];
  int s_bad_page;
  int s_dhit[PH ? GP : 1], s_dpos[PH ? GP : 1], s_dslot[PH ? GP : 1];  // each decision's outcome
  UnitPlan s_plan;
};

// The match stage of unit u by the whole CTA (kMatchThreads threads): the
// decision, the unit's plan, the rotated query and the window's new query.
// Afterwards ms.s_plan holds the plan and ms.s_bad_page whether a page id
// was invalid.
// A hook that does nothing (the match kernels).
struct NoHook {
  __device__ __forceinline__ void operator()(int, int) const {}
};

template <int D, int GP, int GF, bool PH, bool RB, typename Hook = NoHook>
__device__ __forceinline__ void match_body(const MatchParams& p, int u, MatchSmem<D, GP, PH>& ms,
                                           const Hook& hook = Hook()) {
  using RT = std::conditional_t<RB, uint2, float4>;  // four window elements
  const int G = GF > 0 ? GF : p.G;
  const int GD = G * D;
  auto& sq = ms.sq;
  auto& sdist = ms.sdist;
  auto& spos = ms.spos;
  auto& sslot = ms.sslot;
  int& s_bad_page = ms.s_bad_page;
  auto& s_dhit = ms.s_dhit;
  auto& s_dpos = ms.s_dpos;
  auto& s_dslot = ms.s_dslot;
  UnitPlan& s_plan = ms.s_plan;
  __syncthreads();  // a previous unit's readers of this shared memory are done
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Wp1 = p.W + 1;

  // Every load below is independent of the others (no slot index waits for
  // the step counter): ring slots are read whole and mapped to ages later.
  constexpr int NW = kMatchThreads / 32;
  constexpr int BS = GP == 4 ? 5 : 3;  // slots per warp per batch of loads (8 warps x 5 >= W+1 for W <= 39)
  constexpr int F4 = GP * D / 4 / 32;  // float4 per lane per slot, at most
  const int n4 = GD / 4;               // groups of four elements of one slot
  RT r[BS][F4];
  int rpos[BS];
  auto load_batch = [&](int s0) {
#pragma unroll
    for (int k = 0; k < BS; ++k) {
      const int slot = s0 + k * NW;
      if (slot < Wp1) {
        const RT* rq = reinterpret_cast<const RT*>(p.ring_q) + ((size_t)u * Wp1 + slot) * n4;
#pragma unroll
        for (int f = 0; f < F4; ++f)
          if (lane + 32 * f < n4) r[k][f] = rq[lane + 32 * f];
        rpos[k] = p.ring_pos[(size_t)u * Wp1 + slot];
      }
    }
  };
  load_batch(warp);
  const size_t q0 = ((size_t)b * p.Hq + (size_t)kvh * G) * D / 4;  // first group of four of the query
  if (p.q_bf16) {
    const uint2* qsrc = reinterpret_cast<const uint2*>(p.q_pre) + q0;
    for (int i = tid; i < n4; i += kMatchThreads) reinterpret_cast<float4*>(sq)[i] = widen4(qsrc[i]);
  } else {
    const float4* qsrc = reinterpret_cast<const float4*>(p.q_pre) + q0;
    for (int i = tid; i < n4; i += kMatchThreads) reinterpret_cast<float4*>(sq)[i] = qsrc[i];
  }
  const int len = p.seq_lens[b];
  const int p_t = len - 1;
  const int n = p.steps[u];
  const int occ = n < p.W ? n : p.W;
  // RoPE angle of pair i = tid (D/2 <= 64 threads)
  double rot_sn = 0.0, rot_cs = 1.0;
  if (tid < D / 2) rope_sincos(p.rope_pos[b], p.inv_freq[tid], &rot_sn, &rot_cs);
  // the caller's work that needs the sequence length, issued while this
  // unit's loads are in flight (the one-launch step prefetches the K/V tail)
  hook(b, len);
  if (tid == 0) s_bad_page = 0;
  __syncthreads();
  const bool traced = p.trace != nullptr && tid == 0 && (int)blockIdx.x < p.grid;
  if (traced && p.trace[blockIdx.x * kTracePoints + kTraceLoaded] == 0)
    p.trace[blockIdx.x * kTracePoints + kTraceLoaded] = globaltimer_ns();

  // 1. distances: mean over the G heads of sum((q - q_s)^2), for the slots
  // holding the occ most recent entries (age j = 0 is step n - 1, in slot
  // (n - 1) mod (W+1); the age of slot s is (n - 1 - s) mod (W+1)).
  for (int s0 = warp; s0 < Wp1; s0 += BS * NW) {
    if (s0 != warp) load_batch(s0);
#pragma unroll
    for (int k = 0; k < BS; ++k) {
      const int slot = s0 + k * NW;
      if (slot < Wp1) {
        const int j = (((n - 1 - slot) % Wp1) + Wp1) % Wp1;
        if (PH && j < occ) {
          // one distance per head: float4 i of a slot belongs to head i / (D/4)
#pragma unroll
          for (int f = 0; f < F4; ++f) {
            const int i4 = lane + 32 * f;
            float a = 0.f;
            if (i4 < n4) {
              const float4 q = reinterpret_cast<const float4*>(sq)[i4], e = widen4(r[k][f]);
              const float dx = q.x - e.x, dy = q.y - e.y, dz = q.z - e.z, dw = q.w - e.w;
              a = fmaf(dx, dx, a);
              a = fmaf(dy, dy, a);
              a = fmaf(dz, dz, a);
              a = fmaf(dw, dw, a);
            }
#pragma unroll
            for (int o = D / 8; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);  // the head's D/4 lanes
            if (i4 < n4 && i4 % (D / 4) == 0) sdist[PH ? i4 / (D / 4) : 0][j] = a;
          }
          if (lane == 0) {
            spos[j] = rpos[k];
            sslot[j] = slot;
          }
        } else if (j < occ) {
          float acc = 0.f;
#pragma unroll
          for (int f = 0; f < F4; ++f) {
            if (lane + 32 * f >= n4) break;
            const float4 q = reinterpret_cast<const float4*>(sq)[lane + 32 * f], e = widen4(r[k][f]);
            const float dx = q.x - e.x, dy = q.y - e.y, dz = q.z - e.z, dw = q.w - e.w;
            acc = fmaf(dx, dx, acc);
            acc = fmaf(dy, dy, acc);
            acc = fmaf(dz, dz, acc);
            acc = fmaf(dw, dw, acc);
          }
          acc = warp_sum(acc);
          if (lane == 0) {
            // a power-of-two group divides exactly by its reciprocal
            sdist[0][j] = (GF == 4 || GF == 8) ? acc * (1.0f / (GF > 0 ? GF : 1)) : __fdiv_rn(acc, (float)G);
            spos[j] = rpos[k];
            sslot[j] = slot;
          }
        }
      }
    }
  }
  __syncthreads();

  // 2. argmin: smaller distance, then larger position, then the newer entry;
  // warp w takes decision w (the group's, or head w's with per-head matching)
  const int nd = PH ? G : 1;
  if (warp < nd) {
    float bd = INFINITY;
    int bp = 0, bj = -1;
    for (int j = lane; j < occ; j += 32) {
      const float d = sdist[warp][j];
      const int pos = spos[j];
      if (pos < p_t && (d < bd || (d == bd && bj >= 0 && (pos > bp || (pos == bp && j < bj))))) {
        bd = d;
        bp = pos;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, bd, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      const bool take = oj >= 0 && (bj < 0 || od < bd || (od == bd && (op > bp || (op == bp && oj < bj))));
      if (take) {
        bd = od;
        bp = op;
        bj = oj;
      }
    }
    if (lane == 0) {
      const int hit = (bj >= 0) && (bd < p.tau);
      s_dhit[warp] = hit;
      s_dpos[warp] = hit ? bp : -1;
      s_dslot[warp] = hit ? sslot[bj] : -1;
      if (!PH) {
        UnitPlan pl;
        pl.end = len;
        pl.cut = p_t - p.band > 0 ? p_t - p.band : 0;
        pl.hit = hit;
        pl.src_slot = hit ? sslot[bj] : -1;
        pl.start = hit ? (bp - p.band > 0 ? bp - p.band : 0) : 0;
        pl.dst_slot = n % Wp1;
        pl.bad = (len < 1 || len > p.capacity) ? 1 : 0;
        pl.expected = 0;
        s_plan = pl;
      }
    }
  }
  __syncthreads();
  if (PH) {
    // the unit reads the union of its heads' ranges: from the smallest first
    // fresh key; its reuse slot is the first reusing head's (-1: none)
    if (tid == 0) {
      UnitPlan pl;
      HeadPlan hp;
      pl.end = len;
      pl.cut = p_t - p.band > 0 ? p_t - p.band : 0;
      pl.dst_slot = n % Wp1;
      pl.bad = (len < 1 || len > p.capacity) ? 1 : 0;
      pl.expected = 0;
      int start = len, hmask = 0, src = -1;
      for (int d = 0; d < nd; ++d) {
        if (src < 0) src = s_dslot[d];
        const int st = s_dhit[d] ? (s_dpos[d] - p.band > 0 ? s_dpos[d] - p.band : 0) : 0;
        start = st < start ? st : start;
        hmask |= s_dhit[d] << d;
        hp.hstart[d] = st;
        hp.hsrc[d] = s_dslot[d];
      }
      pl.start = start;
      pl.hit = hmask != 0;
      pl.src_slot = src;
      hp.hmask = hmask;
      s_plan = pl;
      p.hplan[u] = hp;
    }
    __syncthreads();
  }

  if (traced && p.trace[blockIdx.x * kTracePoints + kTraceDecided] == 0)
    p.trace[blockIdx.x * kTracePoints + kTraceDecided] = globaltimer_ns();
  // paged KV: every page the step reads must be a valid pool page
  if (!s_plan.bad && p.page_size > 0) {
    const int pg0 = s_plan.start / p.page_size, pg1 = (s_plan.end - 1) / p.page_size;
    const int* row = p.block_table + (size_t)b * p.max_pages;
    for (int i = pg0 + tid; i <= pg1; i += kMatchThreads) {
      const int pg = row[i];
      if (pg < 0 || pg >= p.num_pages) s_bad_page = 1;
    }
  }
  __syncthreads();
  const int bad = s_plan.bad | s_bad_page;

  if (bad) {
    const float qnan = __int_as_float(0x7fc00000);
    for (int i = tid; i < GD; i += kMatchThreads) p.out[((size_t)b * p.Hq + (size_t)kvh * G) * D + i] = qnan;
    if (tid < G) p.lse[(size_t)b * p.Hq + kvh * G + tid] = qnan;
    if (tid < nd) {
      if (p.hit_mask) p.hit_mask[u * nd + tid] = 0;
      if (p.match_pos) p.match_pos[u * nd + tid] = -1;
    }
    if (tid == 0) {
      atomicOr(p.status, s_plan.bad ? MAC_DEV_BAD_SEQ_LEN : MAC_DEV_BAD_PAGE);
      UnitPlan pl = s_plan;
      pl.bad = 1;
      pl.hit = 0;
      p.plan[u] = pl;
    }
  } else {
    // 4. rotate pair i = tid (i, i + D/2) by the angle computed above
    const double scale = kLog2eD / sqrt((double)D);
    for (int i = tid; i < D / 2; i += kMatchThreads) {
      const double sn = rot_sn, cs = rot_cs;
      for (int h = 0; h < G; ++h) {
        const double x = sq[h * D + i], y = sq[h * D + i + D / 2];
        float* dst = p.qrot + ((size_t)u * G + h) * D;
        dst[i] = (float)((x * cs - y * sn) * scale);
        dst[i + D / 2] = (float)((y * cs + x * sn) * scale);
      }
    }
    // 5. this step's query enters the ring (bf16: rounded to nearest even)
    RT* rdst = reinterpret_cast<RT*>(p.ring_q) + ((size_t)u * Wp1 + s_plan.dst_slot) * n4;
    for (int i = tid; i < n4; i += kMatchThreads) {
      const float4 v = reinterpret_cast<const float4*>(sq)[i];
      if constexpr (RB)
        rdst[i] = narrow4(v);
      else
        rdst[i] = v;
    }
    if (tid < nd) {
      if (p.hit_mask) p.hit_mask[u * nd + tid] = (uint8_t)s_dhit[tid];
      if (p.match_pos) p.match_pos[u * nd + tid] = s_dpos[tid];
    }
    if (tid == 0) {
      p.steps[u] = n + 1;
      p.plan[u] = s_plan;
    }
  }
}

}  // namespace
}  // namespace mac
