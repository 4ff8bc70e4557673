// mac_attend_dev.cuh -- device helpers shared by the attention kernels:
// mbarriers with bounded waits, TMA loads, bf16 packing, the window's stored
// outputs, the fold of partial states, and the walk over a CTA's work items.
#pragma once

#include <stdint.h>

#include <cuda_bf16.h>

#include "mac_internal.cuh"

#include "../../include/mac.h"

namespace mac {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

constexpr int kItemCache = 64;  // work items of one CTA kept in shared memory

__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of phase `parity` (a polling loop over several barriers
// uses it: try_wait may hold the thread for a while on one of them).
__device__ __forceinline__ bool mbar_test(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on phase `parity` of an mbarrier.  Returns false if the CTA
// is aborting or the wait exceeded kWaitLimitNs (then it flags the abort).
__device__ bool mbar_wait(unsigned long long* bar, uint32_t parity, volatile int* abort_flag,
                          unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, MAC_DEV_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, unsigned long long* bar, int c0,
                                            int c1, int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_u32(const int* ptr) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed_u32(const int* ptr) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(int* ptr, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
// A work item read through L2 (the one-launch step's items are written by
// another CTA of the same launch, so no SM may serve an old copy from L1).
static_assert(sizeof(Segment) == 32, "a work item is two 16-byte loads");
__device__ __forceinline__ Segment load_segment(const Segment* src) {
  const int4 a = __ldcg(reinterpret_cast<const int4*>(src)), b = __ldcg(reinterpret_cast<const int4*>(src) + 1);
  Segment sg;
  memcpy(reinterpret_cast<int4*>(&sg), &a, 16);
  memcpy(reinterpret_cast<int4*>(&sg) + 1, &b, 16);
  return sg;
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 values as bf16x2 (first in the low half), rounded to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// The bf16 residual pair of (a, b) after their bf16 rounding `hi`.
__device__ __forceinline__ uint32_t pack_bf16_residual(float a, float b, uint32_t hi) {
  return pack_bf16(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

// Stored outputs o of the window: fp32, or bf16 (rb) rounded to nearest even.
__device__ __forceinline__ float ring_o_at(const void* base, size_t i, bool rb) {
  return rb ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(base)[i] << 16)
            : reinterpret_cast<const float*>(base)[i];
}
__device__ __forceinline__ void ring_o_put(void* base, size_t i, float v, bool rb) {
  if (rb)
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(base)[i] = v;
}
__device__ __forceinline__ const unsigned char* ring_o_row(const void* base, size_t i, bool rb) {
  return reinterpret_cast<const unsigned char*>(base) + i * (rb ? 2 : 4);  // address of element i
}

// Fold one state (max m, sum l, outputs o relative to 2^m) into (M, L, O).
template <int N>
__device__ __forceinline__ void fold_state(float& M, float& L, float (&O)[N], float m, float l, const float* o) {
  const float Mn = fmaxf(M, m);
  const float Mu = Mn == -INFINITY ? 0.f : Mn;
  const float a = ex2(M - Mu), c = ex2(m - Mu);
  L = L * a + l * c;
#pragma unroll
  for (int j = 0; j < N; ++j) O[j] = O[j] * a + o[j] * c;
  M = Mn;
}

// The CTA's pieces, walked in order by every lane of every warp.  A split
// piece is part of one segment of a large unit; a whole-unit piece holds
// both segments of a small unit: A = [a0, a1) (may be empty), B = [k0, k1).
struct Piece {
  int unit, pidx, whole, segA;  // segA: a split piece of segment A (the amend / prefix range)
  int hit, src, dst;          // whole unit: plan of the unit (end = k1)
  int k0, k1, kb0, nbox;      // split: its keys; whole unit: segment B
  int a0, a1, akb0, anbox;    // whole unit: segment A
  int wA;                     // whole unit: warps on segment A
};

__device__ __forceinline__ int box_count(int k0, int k1) {
  const int kb0 = k0 & ~(kSubKeys - 1);
  return k1 > k0 ? (((k1 + kSubKeys - 1) & ~(kSubKeys - 1)) - kb0) / kSubKeys : 0;
}
struct Walker {
  int s;
  long long lo, hi;
  const Segment* cache;  // shared-memory copy of items [base, base + kItemCache)
  int base;
  const Segment* table;  // the items
  int nseg;
  bool local;            // a CTA's own whole units: flat holds the unit (else item 2u, 2u+1 is unit u)
  __device__ __forceinline__ bool next(int cta, Piece& pc) {
    while (s < nseg) {
      const Segment sg = (local || s - base < kItemCache) ? cache[s - base] : load_segment(table + s);
      const int cur = s++;
      if (sg.kind < 0) continue;
      if (!local && sg.flat >= hi) {  // this and every later item start past the range
        s = nseg;
        return false;
      }
      pc.unit = local ? (int)sg.flat : cur >> 1;
      if (sg.kind == kItemWhole) {
        if (sg.first_cta != cta) continue;  // owned by the CTA whose range holds its start
        const int start = sg.key0, cut = sg.pbase, end = sg.key0 + sg.len;
        pc.whole = 1;
        pc.segA = 0;
        pc.pidx = -1;
        pc.hit = sg.npieces & 1;
        pc.src = (sg.npieces >> 1) & 0x7ff;
        pc.dst = (sg.npieces >> 12) & 0x7ff;
        pc.a0 = start;
        pc.a1 = cut;
        pc.akb0 = start & ~(kSubKeys - 1);
        pc.anbox = box_count(start, cut);
        pc.k0 = cut;
        pc.k1 = end;
        pc.kb0 = cut & ~(kSubKeys - 1);
        pc.nbox = box_count(cut, end);
        const int nA = pc.anbox, nB = pc.nbox;
        int wA = 0;
        if (nA > 0) {
          wA = (kConsumerWarps * nA + (nA + nB) / 2) / (nA + nB);
          wA = wA < 1 ? 1 : (wA > kConsumerWarps - 1 ? kConsumerWarps - 1 : wA);
        }
        pc.wA = wA;
        return true;
      }
      const long long fa = lo > sg.flat ? lo : sg.flat;
      const long long fe = hi < sg.flat + sg.len ? hi : sg.flat + sg.len;
      if (fa >= fe) continue;  // the range holds only this segment's padding, or ends before it
      pc.whole = 0;
      pc.segA = sg.kind == kItemA;
      pc.wA = 0;
      pc.anbox = 0;
      pc.pidx = sg.pbase + (cta - sg.first_cta);
      pc.k0 = sg.key0 + (int)(fa - sg.flat);
      pc.k1 = sg.key0 + (int)(fe - sg.flat);
      pc.kb0 = pc.k0 & ~(kSubKeys - 1);
      pc.nbox = box_count(pc.k0, pc.k1);
      return true;
    }
    return false;
  }
};

}  // namespace
}  // namespace mac
