// mac_match.cu -- the match kernels of MAC-Attention: one CTA per unit for
// groups of up to 8 heads, G/8 CTAs per unit for groups of 16-64 heads; the
// last CTA to finish builds the step's work plan for the attention kernel.
// The stage itself (distances, decision, plan, RoPE, window update) is in
// mac_match_dev.cuh.
#include "mac_match_dev.cuh"

namespace mac {
namespace {

template <int D, int GP, int GF, bool PH, bool RB>
__global__ void __launch_bounds__(kMatchThreads) mac_match_kernel(const MatchParams p) {
  __shared__ MatchSmem<D, GP, PH> ms;
  __shared__ int s_last;
  // the attention kernel (launched with programmatic stream serialization)
  // may start its prologue now; it waits for this grid before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the split's cumulative share of range tid, loaded now so the CTA that
  // builds the split does not wait for it
  const double cw_c = (p.cw != nullptr && (int)threadIdx.x <= p.grid) ? __ldcg(p.cw + threadIdx.x) : 0.0;
  const int tid = threadIdx.x;
  match_body<D, GP, GF, PH, RB>(p, blockIdx.x, ms);

  // last CTA to arrive builds the segment table for the attention kernel.
  // Only the plan (written by thread 0) is read by that CTA; everything else
  // goes to the attention kernel, which starts after this grid completes.
  if (tid == 0) {
    // the ticket's release publishes this CTA's plan; its acquire (for the
    // last CTA) orders the build's reads of the other plans
    int ticket;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(p.done) : "memory");
    s_last = (ticket == (int)gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  // no fence needed: every CTA's plan store precedes its ticket (a release),
  // the last ticket's acquire makes them visible to thread 0, and the block
  // barrier above orders this CTA's other threads after that acquire
  build_segments(p, (int)gridDim.x, cw_c);
  if (tid == 0) *p.done = 0;
}


// Groups of window slots each chunk's scan is split into (16-64-head groups):
// as many as the SMs allow, up to 4, with `ctas` = units x chunks.
__host__ __device__ inline int wide_slot_groups(int ctas, int grid) {
  const int s = ctas > 0 ? grid / ctas : 1;
  return s < 1 ? 1 : (s > 4 ? 4 : s);
}

// Groups of 16, 32 or 64 query heads per KV head (multi-query attention):
// NC = G / 8 chunks per unit, each split into S groups of window slots when
// the SMs allow (wide_slot_groups), CTA (u, c, g) holding the heads
// [8c, 8c + 8) and the slots of group g.  Each sums, for every window entry
// of its group, the squared L2 distance of its heads to the entry's (the
// window scan is spread over NC S SMs instead of one) and stores the part in
// dpart; group 0 rotates the chunk's queries and writes them to the step's
// ring slot.  The last of the unit's NC S CTAs to arrive (atomic ticket,
// nobody waits) adds the NC parts of each entry in chunk order -- the mean over the
// G heads -- and takes the decision exactly as the 8-head kernel does
// (argmin, ties to the larger position, then the newer entry; strict
// threshold; NaN never hits), then writes the plan; the last unit decided
// builds the step's work plan.  Per-head matching is not offered here.
template <int D, bool RB>
__global__ void __launch_bounds__(kMatchThreads) mac_match_wide_kernel(const MatchParams p) {
  using RT = std::conditional_t<RB, uint2, float4>;  // four window elements
  constexpr int GP = 8;                               // heads per CTA
  constexpr int GDc = GP * D;
  __shared__ __align__(16) float sq[GDc];
  __shared__ float sdist[kMaxWindow + 1];  // [slot] (the decider: the whole group's mean)
  __shared__ int spos[kMaxWindow + 1];
  __shared__ int s_bad_page, s_last, s_decider;
  __shared__ UnitPlan s_plan;
  __shared__ int s_hit, s_mpos;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const double cw_c = (p.cw != nullptr && (int)threadIdx.x <= p.grid) ? __ldcg(p.cw + threadIdx.x) : 0.0;
  const int G = p.G, NC = G / GP, S = wide_slot_groups(p.B * p.Hkv * NC, p.grid);
  const int u = blockIdx.x / (NC * S), cs = blockIdx.x - u * NC * S, c = cs / S, sg = cs - c * S;
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Wp1 = p.W + 1;
  constexpr int NW = kMatchThreads / 32;
  constexpr int BS = 3;                 // slots per warp per batch of loads
  constexpr int F4 = GDc / 4 / 32;      // float4 per lane per slot
  constexpr int n4 = GDc / 4;
  // this CTA's slots: group sg of S
  const int per = (Wp1 + S - 1) / S, sl0 = sg * per, sl1 = sl0 + per < Wp1 ? sl0 + per : Wp1;
  RT r[BS][F4];
  auto load_batch = [&](int s0) {
#pragma unroll
    for (int k = 0; k < BS; ++k) {
      const int slot = s0 + k * NW;
      if (slot < sl1) {
        const RT* rq = reinterpret_cast<const RT*>(p.ring_q) + (((size_t)u * Wp1 + slot) * G + (size_t)c * GP) * D / 4;
#pragma unroll
        for (int f = 0; f < F4; ++f) r[k][f] = rq[lane + 32 * f];
      }
    }
  };
  load_batch(sl0 + warp);
  const size_t q0 = ((size_t)b * p.Hq + (size_t)kvh * G + (size_t)c * GP) * D / 4;  // this chunk's heads
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
  const bool bad_len = len < 1 || len > p.capacity;
  double rot_sn = 0.0, rot_cs = 1.0;
  if (tid < D / 2) rope_sincos(p.rope_pos[b], p.inv_freq[tid], &rot_sn, &rot_cs);
  __syncthreads();

  // 1. this chunk's part of every occupied entry's distance: sum over its 8
  // heads of sum((q - q_s)^2), in fp32 (the difference form)
  for (int s0 = sl0 + warp; s0 < sl1; s0 += BS * NW) {
    if (s0 != sl0 + warp) load_batch(s0);
#pragma unroll
    for (int k = 0; k < BS; ++k) {
      const int slot = s0 + k * NW;
      if (slot < sl1) {
        const int j = (((n - 1 - slot) % Wp1) + Wp1) % Wp1;
        if (j < occ) {
          float acc = 0.f;
#pragma unroll
          for (int f = 0; f < F4; ++f) {
            const float4 q = reinterpret_cast<const float4*>(sq)[lane + 32 * f], e = widen4(r[k][f]);
            const float dx = q.x - e.x, dy = q.y - e.y, dz = q.z - e.z, dw = q.w - e.w;
            acc = fmaf(dx, dx, acc);
            acc = fmaf(dy, dy, acc);
            acc = fmaf(dz, dz, acc);
            acc = fmaf(dw, dw, acc);
          }
          acc = warp_sum(acc);
          if (lane == 0) p.dpart[((size_t)u * Wp1 + slot) * NC + c] = acc;
        }
      }
    }
  }
  // 2. rotate this chunk's heads (pair i = tid) and record them in the step's
  // ring slot (outside the window this step; skipped for an invalid length);
  // the chunk's first slot group does it
  if (sg == 0) {
    const double scale = kLog2eD / sqrt((double)D);
    for (int i = tid; i < D / 2; i += kMatchThreads) {
      for (int h = 0; h < GP; ++h) {
        const double x = sq[h * D + i], y = sq[h * D + i + D / 2];
        float* dst = p.qrot + ((size_t)u * G + (size_t)c * GP + h) * D;
        dst[i] = (float)((x * rot_cs - y * rot_sn) * scale);
        dst[i + D / 2] = (float)((y * rot_cs + x * rot_sn) * scale);
      }
    }
    if (!bad_len) {
      RT* rdst = reinterpret_cast<RT*>(p.ring_q) + (((size_t)u * Wp1 + n % Wp1) * G + (size_t)c * GP) * D / 4;
      for (int i = tid; i < n4; i += kMatchThreads) {
        const float4 v = reinterpret_cast<const float4*>(sq)[i];
        if constexpr (RB)
          rdst[i] = narrow4(v);
        else
          rdst[i] = v;
      }
    }
  }
  // every thread's stores are published before the unit's ticket
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    int ticket;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(p.ucnt + u) : "memory");
    s_decider = (ticket == NC * S - 1);
    if (s_decider) p.ucnt[u] = 0;
    s_bad_page = 0;
  }
  __syncthreads();
  if (!s_decider) return;
  __threadfence();  // the other chunks' parts, published before their tickets, are read below

  // 3. the decision (the last chunk CTA of the unit): mean over the G heads
  const float invG = 1.0f / (float)G;  // G = 16, 32, 64: exact
  for (int j = tid; j < occ; j += kMatchThreads) {
    const int slot = (((n - 1 - j) % Wp1) + Wp1) % Wp1;
    const float* dp = p.dpart + ((size_t)u * Wp1 + slot) * NC;
    float d = 0.f;
    for (int k = 0; k < NC; ++k) d += __ldcg(dp + k);
    sdist[j] = d * invG;
    spos[j] = p.ring_pos[(size_t)u * Wp1 + slot];
  }
  __syncthreads();
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
      pl.src_slot = hit ? (((n - 1 - bj) % Wp1) + Wp1) % Wp1 : -1;
      pl.start = hit ? (bp - p.band > 0 ? bp - p.band : 0) : 0;
      pl.dst_slot = n % Wp1;
      pl.bad = bad_len ? 1 : 0;
      pl.expected = 0;
      s_plan = pl;
      s_hit = hit;
      s_mpos = hit ? bp : -1;
    }
  }
  __syncthreads();
  if (!s_plan.bad && p.page_size > 0) {
    const int pg0 = s_plan.start / p.page_size, pg1 = (s_plan.end - 1) / p.page_size;
    const int* row = p.block_table + (size_t)b * p.max_pages;
    for (int i = pg0 + tid; i <= pg1; i += kMatchThreads) {
      const int pg = row[i];
      if (pg < 0 || pg >= p.num_pages) s_bad_page = 1;
    }
  }
  __syncthreads();
  if (s_plan.bad | s_bad_page) {
    const float qnan = __int_as_float(0x7fc00000);
    for (int i = tid; i < G * D; i += kMatchThreads) p.out[((size_t)b * p.Hq + (size_t)kvh * G) * D + i] = qnan;
    if (tid < G) p.lse[(size_t)b * p.Hq + kvh * G + tid] = qnan;
    if (tid == 0) {
      if (p.hit_mask) p.hit_mask[u] = 0;
      if (p.match_pos) p.match_pos[u] = -1;
      atomicOr(p.status, s_plan.bad ? MAC_DEV_BAD_SEQ_LEN : MAC_DEV_BAD_PAGE);
      UnitPlan pl = s_plan;
      pl.bad = 1;
      pl.hit = 0;
      p.plan[u] = pl;
    }
  } else if (tid == 0) {
    if (p.hit_mask) p.hit_mask[u] = (uint8_t)s_hit;
    if (p.match_pos) p.match_pos[u] = s_mpos;
    p.steps[u] = n + 1;
    p.plan[u] = s_plan;
  }

  // 4. the last unit decided builds the work plan (as in the 8-head kernel)
  if (tid == 0) {
    int ticket;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(p.done) : "memory");
    s_last = (ticket == p.B * p.Hkv - 1);
  }
  __syncthreads();
  if (!s_last) return;
  build_segments(p, p.B * p.Hkv, cw_c);
  if (tid == 0) *p.done = 0;
}

// Variants as for the attention kernel: exact groups of 4 and 8, run-time
// groups padded to 4 and 8, and per-head matching (run-time group).
template <int D, bool RB>
void launch_dr(const MatchParams& p, int U, cudaStream_t s) {
  if (p.per_head) {
    if (p.G <= 4)
      mac_match_kernel<D, 4, 0, true, RB><<<U, kMatchThreads, 0, s>>>(p);
    else
      mac_match_kernel<D, 8, 0, true, RB><<<U, kMatchThreads, 0, s>>>(p);
  } else if (p.G == 4) {
    mac_match_kernel<D, 4, 4, false, RB><<<U, kMatchThreads, 0, s>>>(p);
  } else if (p.G == 8) {
    mac_match_kernel<D, 8, 8, false, RB><<<U, kMatchThreads, 0, s>>>(p);
  } else if (p.G < 4) {
    mac_match_kernel<D, 4, 0, false, RB><<<U, kMatchThreads, 0, s>>>(p);
  } else {
    mac_match_kernel<D, 8, 0, false, RB><<<U, kMatchThreads, 0, s>>>(p);
  }
}
template <int D>
void launch_d(const MatchParams& p, int U, cudaStream_t s) {
  if (p.G > kMaxGroup) {  // 16, 32 or 64 heads: G / 8 CTAs per unit
    const int NC = group_chunks(p.G), grid = U * NC * wide_slot_groups(U * NC, p.grid);
    if (p.ring_bf16)
      mac_match_wide_kernel<D, true><<<grid, kMatchThreads, 0, s>>>(p);
    else
      mac_match_wide_kernel<D, false><<<grid, kMatchThreads, 0, s>>>(p);
  } else if (p.ring_bf16) {
    launch_dr<D, true>(p, U, s);
  } else {
    launch_dr<D, false>(p, U, s);
  }
}

}  // namespace

cudaError_t launch_match(const MatchParams& p, int D, cudaStream_t s) {
  const int U = p.B * p.Hkv;
  if (!group_ok(p.G) || (p.G > kMaxGroup && (p.per_head || p.dpart == nullptr || p.ucnt == nullptr)))
    return cudaErrorInvalidValue;
  if (D == 128)
    launch_d<128>(p, U, s);
  else if (D == 64)
    launch_d<64>(p, U, s);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace mac
