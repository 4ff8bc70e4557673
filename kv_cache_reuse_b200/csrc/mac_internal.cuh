// mac_internal.cuh -- device-side data layout shared by the MAC kernels and
// the host API of this library (not part of the public C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mac {

constexpr int kMaxGroup = 8;          // query heads per KV head held in one tensor-core tile: 1..8
constexpr int kMaxWideGroup = 64;     // larger groups: 16, 32 or 64 heads, as 2, 4 or 8 chunks of 8
constexpr int kSubKeys = 16;          // keys per TMA box (one box never crosses a page)
constexpr int kConsumerWarps = 8;     // attention warps that compute
constexpr int kKeysPerStage = 128;    // keys in flight per round of boxes (kConsumerWarps * 16)
constexpr int kAttnThreads = kConsumerWarps * 32;
constexpr int kMatchThreads = 256;
constexpr int kMaxWindow = 256;

// Per (sequence, KV head) plan written by the match kernel.  With per-head
// matching start is the smallest first fresh key over the unit's heads, hit
// says whether any head reuses a state, src_slot is the first reusing head's
// slot, and the heads' own decisions are in HeadPlan.
struct UnitPlan {
  int start;     // first key attended with the current query (c_s on a hit, 0 on a miss)
  int cut;       // c_t = max(0, p_t - band): end of the stored prefix state
  int end;       // p_t + 1
  int hit;       // 1 = reuse the state in ring slot src_slot
  int src_slot;  // ring slot of the matched entry (hit only)
  int dst_slot;  // ring slot receiving this step's entry
  int bad;       // 1 = invalid inputs: no work, NaN outputs, window unchanged
  int expected;  // partial results the unit's merge waits for
};

// Per-head matching: the decisions of a unit's query heads.
struct HeadPlan {
  int hmask;               // heads that reuse a state (bit h)
  int hstart[kMaxGroup];   // first key head h attends freshly (its c_s on a hit, 0 on a miss)
  int hsrc[kMaxGroup];     // ring slot of head h's reused state
};

// Work items, two slots per unit u.  A large unit (more than unit_max fresh
// keys) has two split items: 2u = [start, cut) (into the new prefix state) and
// 2u+1 = [cut, end) (tail, into the output only); each may be cut over several
// CTAs, whose partial results the unit's last CTA merges.  A small unit is
// one whole item in slot 2u, done end to end by one CTA, and slot 2u+1 is
// empty.  The items of all units are laid end to end in a cost space where a
// non-empty item weighs piece_cost + its keys (the fixed cost of a piece --
// query load, combine, merge -- expressed in keys), and that space is split
// evenly over the CTAs.  A split item's keys occupy [flat, flat + len) after
// its piece_cost of padding; a whole item starts at flat and belongs to the
// CTA whose range holds flat.
enum { kItemEmpty = -1, kItemA = 0, kItemB = 1, kItemWhole = 2 };
struct Segment {
  long long flat;  // split: cost offset of the first key; whole: cost offset of the item
  int len;         // keys (whole: end - start)
  int key0;        // first key (absolute position in the sequence)
  int first_cta;   // split: CTA holding `flat`; whole: the owning CTA
  int pbase;       // split: index of the first partial result; whole: the cut c_t
  int npieces;     // split: partial results (CTAs overlapping the keys);
                   // whole: hit | reused slot << 1 | written slot << 12
  int kind;        // kItem*
};

struct PlanHeader {
  long long total;  // size of the flattened cost space
  int n_cta;        // CTAs with work (<= grid)
  int weighted;     // 1: range c is [bounds[c], bounds[c+1]), sized by its SM's rate
};

// Weighted split.  HBM throughput differs between SMs, and the slow ones are
// the same from step to step.  On steps with at least kWeightMinCost cost
// units per CTA, range c of the split is sized in proportion to the learned
// streaming rate of SM c, and the CTA running on SM c takes range c (a CTA
// whose SM's range is already taken takes a free one).  At the end of such a
// step every CTA folds its measured rate into rate[its SM], and CTA 0 turns
// the rates into the cumulative shares cw[] that the next weighted step's
// split uses (cw[c] = share of ranges 0..c-1, cw[grid] = 1).
constexpr long long kWeightMinCost = 4096;

// Group sizes the kernels take: 1 to 8 heads per KV head in one tile, or
// 16, 32, 64 heads (multi-query attention sized groups) in chunks of 8.
__host__ __device__ inline bool group_ok(int G) {
  return (G >= 1 && G <= kMaxGroup) || G == 16 || G == 32 || G == 64;
}
// Chunks of 8 heads a group is processed in (1 for groups of up to 8).
__host__ __device__ inline int group_chunks(int G) { return G > kMaxGroup ? G / kMaxGroup : 1; }

// The kernels hold a query group padded to GP = 4 or 8 heads (the columns of
// their tensor-core tiles); heads G..GP-1 are zero and never stored.
__host__ __device__ inline int group_pad(int G) { return G <= 4 ? 4 : 8; }
// G rounded up to a multiple of 4 (keeps every partial 16-byte aligned).
__host__ __device__ inline int group4(int G) { return (G + 3) & ~3; }
// Layout of one partial result: o_acc [G][D] (unnormalised, relative to m),
// then m [G4] (log2 units) and l [G4], G4 = group4(G).
__host__ __device__ inline size_t partial_floats(int G, int D) { return (size_t)G * D + 2 * (size_t)group4(G); }

struct MatchParams {
  const void* q_pre;       // [B][Hq][D] fp32, or bf16 bits (q_bf16)
  const int* rope_pos;     // [B]
  const int* seq_lens;     // [B]
  const int* block_table;  // [B][max_pages] or null
  float* out;              // [B][Hq][D] (NaN for bad units)
  float* lse;              // [B][Hq]
  uint8_t* hit_mask;       // [U] ([U][G] with per-head matching) or null
  int* match_pos;          // [U] ([U][G] with per-head matching) or null
  void* ring_q;            // [U][W+1][G][D] fp32, or bf16 bits (ring_bf16)
  const int* ring_pos;     // [U][W+1]
  int* steps;              // [U]
  const double* inv_freq;  // [D/2]
  float* qrot;             // [U][G][D], RoPE'd and scaled by log2(e)/sqrt(D)
  UnitPlan* plan;          // [U]
  HeadPlan* hplan;         // [U], per-head matching only
  Segment* seg;            // [2U]
  PlanHeader* hdr;
  int* first_seg;          // [grid] first segment of each attention CTA's range
  const double* cw;        // [grid + 1] cumulative range shares, or null (even split)
  long long* bounds;       // [grid + 1] range starts of a weighted split
  int* claim;              // [grid] ranges taken by the attention CTAs (reset here)
  int* done;               // arrival counter of the match CTAs (reset by the last)
  float* dpart;            // chunked groups: [U][W+1][NC] each chunk's part of an entry's distance
  int* ucnt;               // chunked groups: [U] arrivals of a unit's chunk CTAs (reset by the last)
  unsigned long long* trace;  // [grid][kTracePoints] phase times (one-launch step), or null
  unsigned* status;
  int B, Hq, Hkv, G, W, band, page_size, max_pages, num_pages, capacity;  // band: b - cut_mode
  int per_head;   // 1: one match decision per query head
  int q_bf16;     // 1: q_pre holds bf16
  int ring_bf16;  // 1: window queries are stored in bf16
  float tau;
  int grid;       // CTAs of the attention kernel
  int min_keys;   // minimum cost-space units per attention CTA
  int piece_cost; // fixed cost of one piece, in keys
  int unit_max;   // units with at most this many fresh keys are whole items
};

struct AttendParams {
  CUtensorMap tmK;  // 4D (D, Hkv, rows, seqs|pages), box (D, 1, 16, 1)
  CUtensorMap tmV;
  const int* block_table;
  const float* qrot;
  const UnitPlan* plan;
  const HeadPlan* hplan;  // [U], per-head matching only
  const Segment* seg;
  const PlanHeader* hdr;
  const int* first_seg;  // [grid]
  const long long* bounds;  // [grid + 1]
  int* claim;        // [grid]
  float* rate;       // [grid] learned rate per SM, or null
  double* cw;        // [grid + 1] cumulative range shares (written by CTA 0)
  float* part;       // [max_parts][partial_floats(G, D)]
  int* unit_cnt;     // [U]
  int* smid_of;      // one-launch step: [grid] SM of each CTA
  int* rank_of;      // one-launch step: [grid] range of each split slot (-1: none)
  int* fsync;        // one-launch step: {CTAs that finished matching, epoch of the published split}
  unsigned long long* trace;     // [grid][kTracePoints] %globaltimer at each phase of the last step, or null
  unsigned long long* counters;  // [kCounters] step counters (added to), or null
  void* ring_o;      // [U][W+1][G][D] fp32, or bf16 bits (ring_bf16)
  float* ring_m;     // [U][W+1][G]
  float* ring_l;     // [U][W+1][G]
  int* ring_pos;     // [U][W+1]
  float* out;        // [B][Hq][D]
  float* lse;        // [B][Hq]
  unsigned* status;
  int Hq, Hkv, G, W, page_size, max_pages, nseg, grid;
  int per_head;      // 1: heads of a unit reuse states on their own (plan hmask, hstart, hsrc)
  int ring_bf16;     // 1: stored outputs o are bf16
};

struct AppendParams {
  uint16_t* K;
  uint16_t* V;
  const int* block_table;
  const int* seq_lens;
  const uint16_t* k_new;
  const uint16_t* v_new;
  unsigned* status;
  int B, Hkv, D, page_size, max_pages, num_pages, capacity;
};

// Observability.  Phases a CTA stamps (ns of %globaltimer) when tracing is
// on; a phase the CTA does not go through keeps 0.
enum {
  kTraceStart = 0,       // barriers initialised
  kTraceLoaded = 1,      // match: the first unit's query and window in registers
  kTraceDecided = 2,     // match: the first unit's decision taken
  kTraceMatched = 3,     // one-launch step: this CTA's units matched and recorded
  kTraceTicket = 4,      // one-launch step: this CTA's plans published
  kTraceFirstBox = 5,    // the CTA's first K/V box on chip
  kTraceBoxesDone = 6,   // one-launch step: the last box of this CTA's whole units consumed
  kTraceLocal = 7,       // one-launch step: this CTA's whole units done
  kTraceBuilt = 8,       // one-launch step, the laying-out CTA: split table published
  kTraceTable = 9,       // the split table seen (after the wait for it)
  kTraceRange = 10,      // this CTA's range of split items done
  kTraceEnd = 11,        // about to leave
  kTracePoints = 12
};
// Counters the kernels add to when they are on: keys attended with the
// current query (fresh keys), pieces walked, units done whole, split units
// merged.
enum { kCountKeys = 0, kCountPieces = 1, kCountWhole = 2, kCountMerged = 3, kCounters = 4 };

// Launchers (defined in the .cu files).
cudaError_t launch_match(const MatchParams& p, int D, cudaStream_t s);
cudaError_t launch_attend(const AttendParams& p, int D, int grid, cudaStream_t s);
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t attend_prepare(int D, int G);
// The tcgen05 path (mac_attend_tc.cu): groups of 16, 32 or 64 heads at head
// dim 128, one decision per KV head; products then merge, two launches.
cudaError_t attend_tc_prepare(int G);
cudaError_t launch_attend_tc(const AttendParams& p, int grid, cudaStream_t s);
// The one-launch step (groups of up to 8 heads, one decision per KV head):
// prepare sets its kernels' attributes and reports how many CTAs fit on an SM.
cudaError_t step_prepare(int D, int G, int* blocks_per_sm);
cudaError_t launch_step(const AttendParams& p, const MatchParams& mp, int D, int grid, cudaStream_t s);
cudaError_t launch_wait_selftest(unsigned* status, cudaStream_t s);
size_t attend_smem_bytes(int D, int G);

}  // namespace mac
