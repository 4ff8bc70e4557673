// mac_match.cu -- Match stage of MAC-Attention and the step's work plan.
//
// "MAC-Attention: a Match-Amend-Complete Scheme for Fast and Accurate
// Attention Computation", page 1 (abstract): the match stage "performs
// pre-RoPE L2 matching over a short local window" of recent queries whose
// attention results can be reused.  One CTA handles one (sequence, KV head)
// unit:
//   1. distance of the current pre-RoPE query group (G heads) to every
//      window entry: mean over heads of the squared L2 distance, summed in
//      fp32 as sum((a - b)^2) -- the expanded |a|^2 + |b|^2 - 2ab form would
//      cancel catastrophically for near-repeats;
//   2. argmin with ties to the more recent entry, hit iff the minimum is
//      strictly below tau; NaN distances never win;
//   3. key ranges: the reused prefix ends at c_s = max(0, p_s - band) (the
//      amend band starts there), the stored prefix of this step ends at
//      c_t = max(0, p_t - band), and the tail runs to p_t (band here is the
//      configured band minus the cut mode, so that with cut mode 1 the band
//      ends at the position itself);
//   4. RoPE of the query to rope_pos (fp64 angle), pre-scaled by
//      log2(e)/sqrt(D) so the attention kernel works in exp2 units;
//   5. the query enters the ring slot n mod (W+1) (W+1 slots: the slot
//      written is never one the window can read this step).
// The attention kernel turns the plans into work items itself (every CTA
// computes the split from the plans).  CTA 0 also resets the attention
// CTAs' range claims and fixes the shares of this step's weighted split.
#include <math.h>
#include <stdint.h>

#include "mac_internal.cuh"

#include "../../include/mac.h"

namespace mac {
namespace {

constexpr double kLog2e = 1.4426950408889634;
constexpr double kInvTwoPi = 0.15915494309189535;
constexpr double kTwoPiHi = 6.2831853069365025;    // 2*pi with the low 21 mantissa bits cleared
constexpr double kTwoPiLo = 2.430840202602477e-10;   // 2*pi - kTwoPiHi

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive scan of one value per thread over a block of kMatchThreads.
template <int D>
__global__ void __launch_bounds__(kMatchThreads) mac_match_kernel(const MatchParams p) {
  constexpr int G = kGroup;
  constexpr int GD = G * D;
  __shared__ __align__(16) float sq[GD];
  __shared__ float sdist[kMaxWindow];
  __shared__ int spos[kMaxWindow];
  __shared__ int sslot[kMaxWindow];
  __shared__ int s_bad_page;
  __shared__ UnitPlan s_plan;

  // the attention kernel (launched with programmatic stream serialization)
  // may start its prologue now; it waits for this grid before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (blockIdx.x == 0) {
    // the attention launch that follows claims its ranges afresh, and splits
    // by the shares the last attention launch left (its CTA 0 writes the next
    // ones while this step's CTAs read these)
    if (p.claim != nullptr)
      for (int c = threadIdx.x; c < p.grid; c += kMatchThreads) p.claim[c] = 0;
    if (p.cw_next != nullptr)
      for (int c = threadIdx.x; c <= p.grid; c += kMatchThreads) p.cw[c] = __ldcg(p.cw_next + c);
  }
  const int u = blockIdx.x;
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Wp1 = p.W + 1;

  // Every load below is independent of the others (no slot index waits for
  // the step counter): ring slots are read whole and mapped to ages later.
  constexpr int NW = kMatchThreads / 32;
  constexpr int BS = 5;            // slots per warp per batch (8 warps x 5 >= W+1 for W <= 39)
  constexpr int F4 = GD / 4 / 32;  // float4 per lane per slot
  float4 r[BS][F4];
  int rpos[BS];
  auto load_batch = [&](int s0) {
#pragma unroll
    for (int k = 0; k < BS; ++k) {
      const int slot = s0 + k * NW;
      if (slot < Wp1) {
        const float4* rq = reinterpret_cast<const float4*>(p.ring_q + ((size_t)u * Wp1 + slot) * GD);
#pragma unroll
        for (int f = 0; f < F4; ++f) r[k][f] = rq[lane + 32 * f];
        rpos[k] = p.ring_pos[(size_t)u * Wp1 + slot];
      }
    }
  };
  load_batch(warp);
  const float4* qsrc = reinterpret_cast<const float4*>(p.q_pre + ((size_t)b * p.Hq + (size_t)kvh * G) * D);
  for (int i = tid; i < GD / 4; i += kMatchThreads) reinterpret_cast<float4*>(sq)[i] = qsrc[i];
  const int len = p.seq_lens[b];
  const int p_t = len - 1;
  const int n = p.steps[u];
  const int occ = n < p.W ? n : p.W;
  // RoPE angle of pair i = tid (D/2 <= 64 threads), reduced to [-pi, pi] with
  // a two-constant Cody-Waite reduction (2*pi = C1 + C2, C1 carrying 32
  // significant bits so k*C1 is exact for |k| < 2^21), then sincos in fp64.
  double rot_sn = 0.0, rot_cs = 1.0;
  if (tid < D / 2) {
    const double ang = (double)p.rope_pos[b] * p.inv_freq[tid];
    const double k = rint(ang * kInvTwoPi);
    double rr = ang;
    if (fabs(k) < 2097152.0) {
      rr = fma(-k, kTwoPiHi, ang);
      rr = fma(-k, kTwoPiLo, rr);
    }
    sincos(rr, &rot_sn, &rot_cs);
  }
  if (tid == 0) s_bad_page = 0;
  __syncthreads();

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
        if (j < occ) {
          float acc = 0.f;
#pragma unroll
          for (int f = 0; f < F4; ++f) {
            const float4 q = reinterpret_cast<const float4*>(sq)[lane + 32 * f];
            const float dx = q.x - r[k][f].x, dy = q.y - r[k][f].y, dz = q.z - r[k][f].z, dw = q.w - r[k][f].w;
            acc = fmaf(dx, dx, acc);
            acc = fmaf(dy, dy, acc);
            acc = fmaf(dz, dz, acc);
            acc = fmaf(dw, dw, acc);
          }
          acc = warp_sum(acc);
          if (lane == 0) {
            sdist[j] = acc * (1.0f / G);
            spos[j] = rpos[k];
            sslot[j] = slot;
          }
        }
      }
    }
  }
  __syncthreads();

  // 2. argmin: smaller distance, then larger position, then the newer entry
  if (warp == 0) {
    float bd = INFINITY;
    int bp = 0, bj = -1;
    for (int j = lane; j < occ; j += 32) {
      const float d = sdist[j];
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
      UnitPlan pl;
      pl.end = len;
      pl.cut = p_t - p.band > 0 ? p_t - p.band : 0;
      pl.hit = hit;
      pl.src_slot = hit ? sslot[bj] : -1;
      pl.start = hit ? (bp - p.band > 0 ? bp - p.band : 0) : 0;
      pl.dst_slot = n % Wp1;
      pl.bad = (len < 1 || len > p.capacity) ? 1 : 0;
      pl.pad = 0;
      s_plan = pl;
      spos[0] = hit ? bp : -1;  // matched position (slot 0 of spos no longer needed)
    }
  }
  __syncthreads();

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
    if (tid == 0) {
      atomicOr(p.status, s_plan.bad ? MAC_DEV_BAD_SEQ_LEN : MAC_DEV_BAD_PAGE);
      if (p.hit_mask) p.hit_mask[u] = 0;
      if (p.match_pos) p.match_pos[u] = -1;
      UnitPlan pl = s_plan;
      pl.bad = 1;
      pl.hit = 0;
      p.plan[u] = pl;
    }
  } else {
    // 4. rotate pair i = tid (i, i + D/2) by the angle computed above
    const double scale = kLog2e / sqrt((double)D);
    for (int i = tid; i < D / 2; i += kMatchThreads) {
      const double sn = rot_sn, cs = rot_cs;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const double x = sq[h * D + i], y = sq[h * D + i + D / 2];
        float* dst = p.qrot + ((size_t)u * G + h) * D;
        dst[i] = (float)((x * cs - y * sn) * scale);
        dst[i + D / 2] = (float)((y * cs + x * sn) * scale);
      }
    }
    // 5. this step's query enters the ring
    float4* rdst = reinterpret_cast<float4*>(p.ring_q + ((size_t)u * Wp1 + s_plan.dst_slot) * GD);
    for (int i = tid; i < GD / 4; i += kMatchThreads) rdst[i] = reinterpret_cast<const float4*>(sq)[i];
    if (tid == 0) {
      p.steps[u] = n + 1;
      if (p.hit_mask) p.hit_mask[u] = (uint8_t)s_plan.hit;
      if (p.match_pos) p.match_pos[u] = spos[0];
      p.plan[u] = s_plan;
    }
  }

}

}  // namespace

cudaError_t launch_match(const MatchParams& p, int D, cudaStream_t s) {
  const int U = p.B * p.Hkv;
  if (D == 128) {
    mac_match_kernel<128><<<U, kMatchThreads, 0, s>>>(p);
  } else if (D == 64) {
    mac_match_kernel<64><<<U, kMatchThreads, 0, s>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace mac
