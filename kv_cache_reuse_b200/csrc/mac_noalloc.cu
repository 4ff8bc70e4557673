// mac_noalloc.cu -- dense split-KV decode attention that allocates nothing.
//
// For callers that cannot call cudaMalloc: inference-server plugins and
// embedded hosts that must take all device memory from their host
// framework's pre-planned pool (or whose memory budget is fixed when the
// model is loaded), and latency-critical paths where an allocation's implicit
// device synchronisation is not acceptable.  This entry point runs the
// library's match/plan and attention kernels in their miss-only
// configuration (window 0, so every unit attends all of its keys) with all of
// their scratch -- rotated queries, plan, segment table, partial results,
// counters, a one-slot dummy ring -- in one file-scope static __device__
// array below.  The caller passes the inputs and the outputs; nothing is
// allocated, freed, or taken from an allocating library routine.
//
// Limits: batch * num_kv_heads <= kMaxUnits (64), batch * num_q_heads <=
// kMaxQRows (256), head_dim 64 or 128, groups of 1 to 8 query heads, at most
// kMaxCtas (160) CTAs of the attention kernel.  The array costs about 2 MiB
// on every GPU that loads the library, for the life of the process.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "mac_internal.cuh"

#include "../../include/mac.h"

using namespace mac;

namespace {

constexpr int kMaxUnits = 64;
constexpr int kMaxQRows = 256;  // query heads over the batch (units x G)
constexpr int kMaxD = 128;
constexpr int kMaxCtas = 160;
constexpr int kMaxDevices = 64;

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
constexpr size_t kPartFloats = (size_t)kMaxGroup * kMaxD + 2 * kMaxGroup;  // partial_floats(G, D) at most
constexpr size_t kOffQrot = 0;
constexpr size_t kOffPlan = align256(kOffQrot + (size_t)kMaxQRows * kMaxD * 4);
constexpr size_t kOffSeg = align256(kOffPlan + kMaxUnits * sizeof(UnitPlan));
constexpr size_t kOffHdr = align256(kOffSeg + 2 * kMaxUnits * sizeof(Segment));
constexpr size_t kOffFirst = align256(kOffHdr + sizeof(PlanHeader));
constexpr size_t kOffPart = align256(kOffFirst + kMaxCtas * 4);
constexpr size_t kOffCnt = align256(kOffPart + (size_t)(kMaxCtas + 2 * kMaxUnits) * kPartFloats * 4);
// counters block, cleared on every call: unit_cnt[kMaxUnits], done, (unused), steps[kMaxUnits]
constexpr size_t kCntBytes = (2 * kMaxUnits + 2) * 4;
constexpr size_t kOffInv = align256(kOffCnt + kCntBytes);
constexpr size_t kOffRingQ = align256(kOffInv + (kMaxD / 2) * 8);
constexpr size_t kOffRingO = align256(kOffRingQ + (size_t)kMaxQRows * kMaxD * 4);
constexpr size_t kOffRingM = align256(kOffRingO + (size_t)kMaxQRows * kMaxD * 4);
constexpr size_t kOffRingL = align256(kOffRingM + kMaxQRows * 4);
constexpr size_t kOffRingPos = align256(kOffRingL + kMaxQRows * 4);
constexpr size_t kScratchBytes = align256(kOffRingPos + kMaxUnits * 4);

// The scratch.  In host code this name is only a stand-in for the symbol;
// its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_mac_static_scratch[kScratchBytes];

struct DeviceSetup {
  bool ready;
  unsigned char* base;  // device address of g_mac_static_scratch on this device
  int num_sms;
  int inv_D;            // head_dim and theta of the inverse frequencies in the scratch
  double inv_theta;
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, looked up once under g_mutex (by the first call's
// per-device set-up) and only read afterwards.
EncodeTiledFn g_encode = nullptr;

int encode_map(CUtensorMap* map, const void* base, int D, int Hkv, int rows, int outer) {
  const EncodeTiledFn fn = g_encode;
  if (!fn) return MAC_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows, (cuuint64_t)outer};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2, (cuuint64_t)rows * Hkv * D * 2};
  const cuuint32_t box[4] = {64u, 1u, (cuuint32_t)kSubKeys, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MAC_OK : MAC_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int mac_dense_decode_static(const float* q_pre, const int* rope_pos, const uint16_t* K,
                                       const uint16_t* V, const int* block_table, const int* seq_lens, float* out,
                                       float* lse, unsigned* device_status, int batch, int num_q_heads,
                                       int num_kv_heads, int head_dim, double rope_theta, int page_size,
                                       int max_seq, int max_pages_per_seq, int num_pages, void* stream) {
  // --- host-side checks: nothing is enqueued on failure
  if (!q_pre || !rope_pos || !K || !V || !seq_lens || !out || !lse || !device_status) return MAC_ERR_ARG;
  if (!aligned16(q_pre) || !aligned16(K) || !aligned16(V)) return MAC_ERR_ARG;
  if (batch < 1 || num_kv_heads < 1 || num_q_heads < 1 || !(rope_theta > 0.0)) return MAC_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0 || num_q_heads / num_kv_heads > kMaxGroup) return MAC_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return MAC_ERR_SHAPE;
  // beyond the static scratch
  if ((long long)batch * num_kv_heads > kMaxUnits || (long long)batch * num_q_heads > kMaxQRows) return MAC_ERR_SHAPE;
  if (page_size == 0) {
    if (max_seq < 1) return MAC_ERR_ARG;
  } else {
    if (page_size < 0 || page_size % kSubKeys != 0) return MAC_ERR_SHAPE;
    if (!block_table || max_pages_per_seq < 1 || num_pages < 1) return MAC_ERR_ARG;
  }

  // --- per-device set-up, once, with that device current (no allocation)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MAC_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MAC_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  DeviceSetup* ds = &g_setup[dev];
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!ds->ready) {
      if (!g_encode) {
        void* fp = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fp)
          return MAC_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fp);
      }
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_mac_static_scratch) != cudaSuccess || !ptr) return MAC_ERR_CUDA;
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MAC_ERR_CUDA;
      for (int g : {4, 8})
        if (attend_prepare(64, g) != cudaSuccess || attend_prepare(128, g) != cudaSuccess) return MAC_ERR_CUDA;
      ds->base = static_cast<unsigned char*>(ptr);
      ds->num_sms = sms;
      ds->inv_D = 0;
      ds->inv_theta = 0.0;
      ds->ready = true;
    }
    if (ds->inv_D != head_dim || ds->inv_theta != rope_theta) {
      // the upload reads a host array on this stack: it cannot be recorded
      // into a stream capture, so a change of frequencies during one is refused
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return MAC_ERR_CUDA;
      if (cs != cudaStreamCaptureStatusNone) return MAC_ERR_ARG;
      double inv[kMaxD / 2];
      for (int i = 0; i < head_dim / 2; ++i) inv[i] = pow(rope_theta, -2.0 * (double)i / (double)head_dim);
      // pageable source: the copy is complete when the call returns
      if (cudaMemcpyAsync(ds->base + kOffInv, inv, sizeof(double) * (head_dim / 2), cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
        return MAC_ERR_CUDA;
      ds->inv_D = head_dim;
      ds->inv_theta = rope_theta;
    }
  }
  unsigned char* base = ds->base;
  const int U = batch * num_kv_heads;
  const int grid = ds->num_sms < kMaxCtas ? ds->num_sms : kMaxCtas;
  int* cnt = reinterpret_cast<int*>(base + kOffCnt);
  unsigned* status = device_status;
  // counters start at zero on every call (the previous call's values persist)
  if (cudaMemsetAsync(cnt, 0, kCntBytes, st) != cudaSuccess) return MAC_ERR_CUDA;

  // --- plan: window 0 (never hits), band covering every key: one segment per unit
  MatchParams mp;
  mp.q_pre = q_pre;
  mp.rope_pos = rope_pos;
  mp.seq_lens = seq_lens;
  mp.block_table = page_size > 0 ? block_table : nullptr;
  mp.out = out;
  mp.lse = lse;
  mp.hit_mask = nullptr;
  mp.match_pos = nullptr;
  mp.ring_q = base + kOffRingQ;
  mp.q_bf16 = 0;
  mp.ring_bf16 = 0;
  mp.ring_pos = reinterpret_cast<const int*>(base + kOffRingPos);
  mp.steps = cnt + kMaxUnits + 2;
  mp.inv_freq = reinterpret_cast<const double*>(base + kOffInv);
  mp.qrot = reinterpret_cast<float*>(base + kOffQrot);
  mp.plan = reinterpret_cast<UnitPlan*>(base + kOffPlan);
  mp.hplan = nullptr;  // no per-head matching here
  mp.seg = reinterpret_cast<Segment*>(base + kOffSeg);
  mp.hdr = reinterpret_cast<PlanHeader*>(base + kOffHdr);
  mp.first_seg = reinterpret_cast<int*>(base + kOffFirst);
  mp.cw = nullptr;  // even split: no per-SM record
  mp.bounds = nullptr;
  mp.claim = nullptr;
  mp.done = cnt + kMaxUnits;
  mp.dpart = nullptr;  // groups of up to 8 heads only: one match CTA per unit
  mp.ucnt = nullptr;
  mp.trace = nullptr;
  mp.status = status;
  mp.B = batch;
  mp.Hq = num_q_heads;
  mp.Hkv = num_kv_heads;
  mp.G = num_q_heads / num_kv_heads;
  mp.per_head = 0;
  mp.W = 0;
  mp.band = 1 << 30;
  mp.page_size = page_size;
  mp.max_pages = max_pages_per_seq;
  mp.num_pages = num_pages;
  mp.capacity = page_size == 0 ? max_seq : max_pages_per_seq * page_size;
  mp.tau = 0.f;
  mp.grid = grid;
  mp.min_keys = 128;
  mp.piece_cost = 1024;
  mp.unit_max = 1024;
  if (launch_match(mp, head_dim, st) != cudaSuccess) return MAC_ERR_CUDA;

  // --- attention over every key, merge into out/lse (and the dummy ring)
  AttendParams ap;
  const int rows = page_size == 0 ? max_seq : page_size;
  const int outer = page_size == 0 ? batch : num_pages;
  int rc = encode_map(&ap.tmK, K, head_dim, num_kv_heads, rows, outer);
  if (rc != MAC_OK) return rc;
  rc = encode_map(&ap.tmV, V, head_dim, num_kv_heads, rows, outer);
  if (rc != MAC_OK) return rc;
  ap.block_table = page_size > 0 ? block_table : nullptr;
  ap.qrot = mp.qrot;
  ap.plan = mp.plan;
  ap.hplan = nullptr;
  ap.seg = mp.seg;
  ap.hdr = mp.hdr;
  ap.first_seg = mp.first_seg;
  ap.bounds = nullptr;
  ap.claim = nullptr;
  ap.rate = nullptr;
  ap.cw = nullptr;
  ap.part = reinterpret_cast<float*>(base + kOffPart);
  ap.unit_cnt = cnt;
  ap.smid_of = nullptr;  // two launches here, never the one-launch step
  ap.rank_of = nullptr;
  ap.fsync = nullptr;
  ap.trace = nullptr;
  ap.counters = nullptr;
  ap.ring_o = base + kOffRingO;
  ap.ring_bf16 = 0;
  ap.ring_m = reinterpret_cast<float*>(base + kOffRingM);
  ap.ring_l = reinterpret_cast<float*>(base + kOffRingL);
  ap.ring_pos = reinterpret_cast<int*>(base + kOffRingPos);
  ap.out = out;
  ap.lse = lse;
  ap.status = status;
  ap.Hq = num_q_heads;
  ap.Hkv = num_kv_heads;
  ap.G = num_q_heads / num_kv_heads;
  ap.per_head = 0;
  ap.W = 0;
  ap.page_size = page_size;
  ap.max_pages = max_pages_per_seq;
  ap.nseg = 2 * U;
  ap.grid = grid;
  return launch_attend(ap, head_dim, grid, st) == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
}
