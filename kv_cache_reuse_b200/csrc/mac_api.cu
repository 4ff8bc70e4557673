// mac_api.cu -- host side of the C ABI declared in include/mac.h: argument
// checks, state and scratch allocation, TMA descriptors, kernel launches,
// the KV append kernel, status and state export/import.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include <nvtx3/nvToolsExt.h>

#include "mac_internal.cuh"

#include "../../include/mac.h"

using namespace mac;

struct MacState {
  MacConfig cfg;
  int G, U, D, W, device, num_sms, grid, min_keys, piece_cost, unit_max, capacity;
  int ND;  // match decisions per unit: 1, or G with per-head matching
  int reproducible = 0;  // 1: even split on every step, no learned rates
  int QES, RES;  // bytes of a query element (input) and of a window q / o element
  size_t max_parts;
  // ring (library-owned state)
  unsigned char* ring_q = nullptr;  // fp32 or bf16 (ring_bf16) elements
  unsigned char* ring_o = nullptr;
  float* ring_m = nullptr;
  float* ring_l = nullptr;
  int* ring_pos = nullptr;
  int* steps = nullptr;
  // scratch
  float* qrot = nullptr;
  UnitPlan* plan = nullptr;
  HeadPlan* hplan = nullptr;  // per-head matching decisions
  Segment* seg = nullptr;
  PlanHeader* hdr = nullptr;
  int* first_seg = nullptr;
  float* rate = nullptr;        // learned streaming rate per SM (weighted split)
  long long* bounds = nullptr;  // range starts of a weighted split
  double* cw = nullptr;         // cumulative range shares of the next weighted split
  int* claim = nullptr;         // ranges taken by the attention CTAs
  float* part = nullptr;
  int* unit_cnt = nullptr;
  int* done = nullptr;
  float* dpart = nullptr;  // groups of 16-64 heads: each chunk's part of every entry's distance
  int* ucnt = nullptr;     // groups of 16-64 heads: chunk CTAs of a unit that arrived
  // the one-launch step
  int* smid_of = nullptr;  // [grid] SM of each CTA
  int* rank_of = nullptr;  // [grid] range of each split slot
  int* fsync = nullptr;    // {ticket, epoch}
  int one_launch_ok = 0;   // the configuration can run the step as one launch
  int one_launch = 1;      // ... and it does (mac_set_one_launch)
  // observability (mac_set_trace)
  unsigned long long* trace = nullptr;     // [grid][kTracePoints]
  unsigned long long* counters = nullptr;  // [kCounters]
  int tracing = 0;
  unsigned* status = nullptr;
  double* inv_freq = nullptr;
  // staging of mac_decode_step_host: one packed block each way, on the
  // device and in pinned host memory; the state's status word is the last
  // field of the output block, so one copy brings everything back
  unsigned char* dev_in = nullptr;    // q | pos | lens | k_new | v_new
  unsigned char* dev_out = nullptr;   // out | lse | hit | match_pos | status
  unsigned char* host_in = nullptr;
  unsigned char* host_out = nullptr;
  size_t off_q = 0, off_pos = 0, off_lens = 0, off_knew = 0, off_vnew = 0, in_bytes = 0, in_bytes_noappend = 0;
  size_t off_out = 0, off_lse = 0, off_hit = 0, off_mpos = 0, off_status = 0, out_bytes = 0;
  // the host step as a CUDA graph (copy in, append, match, attend, copy out),
  // captured for one set of cache pointers
  cudaStream_t cap_stream = nullptr;
  cudaGraphExec_t gexec = nullptr;
  const void* g_k = nullptr;
  const void* g_v = nullptr;
  const void* g_bt = nullptr;
  int g_append = -1;
  // TMA descriptors of the last K/V pointers seen
  const void* tm_k_ptr = nullptr;
  const void* tm_v_ptr = nullptr;
  CUtensorMap tmK, tmV;
};

namespace {

// A profiler range (NVTX) over an entry point or a host-side stage of one;
// without a profiler attached the calls do nothing.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T>
cudaError_t alloc(T** p, size_t count) {
  return cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T) + 16);
}

void drop_graph(MacState* s) {
  if (s->gexec) cudaGraphExecDestroy(s->gexec);
  s->gexec = nullptr;
  s->g_append = -1;
}

void free_all(MacState* s) {
  drop_graph(s);
  void* ptrs[] = {s->ring_q, s->ring_o, s->ring_m, s->ring_l, s->ring_pos, s->steps, s->qrot,     s->plan,   s->hplan,
                  s->seg,    s->hdr,    s->first_seg, s->rate, s->cw, s->bounds, s->claim, s->part, s->unit_cnt, s->done, s->dpart, s->ucnt, s->smid_of, s->rank_of, s->fsync, s->trace, s->counters, s->inv_freq, s->dev_in,
                  s->dev_out};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  if (s->host_in) cudaFreeHost(s->host_in);
  if (s->host_out) cudaFreeHost(s->host_out);
  if (s->cap_stream) cudaStreamDestroy(s->cap_stream);
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

int check_config(const MacConfig* c) {
  if (!c) return MAC_ERR_ARG;
  if (c->batch < 1 || c->num_kv_heads < 1 || c->num_q_heads < 1) return MAC_ERR_ARG;
  if (c->num_q_heads % c->num_kv_heads != 0 || !group_ok(c->num_q_heads / c->num_kv_heads)) return MAC_ERR_SHAPE;
  if (c->head_dim != 64 && c->head_dim != 128) return MAC_ERR_SHAPE;
  if (c->window < 1 || c->window > kMaxWindow) return MAC_ERR_SHAPE;
  if (c->band < 0 || c->cut_mode < 0 || c->cut_mode > 1) return MAC_ERR_ARG;
  if (c->match_per_head < 0 || c->match_per_head > 1) return MAC_ERR_ARG;
  // per-head matching holds a group in one tile: groups of up to 8 heads
  if (c->match_per_head && c->num_q_heads / c->num_kv_heads > kMaxGroup) return MAC_ERR_SHAPE;
  if (c->q_bf16 < 0 || c->q_bf16 > 1 || c->ring_bf16 < 0 || c->ring_bf16 > 1) return MAC_ERR_ARG;
  if (!(c->rope_theta > 0.0) || isnan(c->tau)) return MAC_ERR_ARG;
  if (c->page_size == 0) {
    if (c->max_seq < 1) return MAC_ERR_ARG;
  } else {
    if (c->page_size < 0 || c->page_size % kSubKeys != 0) return MAC_ERR_SHAPE;
    if (c->max_pages_per_seq < 1 || c->num_pages < 1) return MAC_ERR_ARG;
  }
  return MAC_OK;
}

int encode_kv_map(MacState* s, CUtensorMap* map, const void* base) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return MAC_ERR_CUDA;
  const MacConfig& c = s->cfg;
  const cuuint64_t D = (cuuint64_t)s->D, H = (cuuint64_t)c.num_kv_heads;
  cuuint64_t dims[4], strides[3];
  dims[0] = D;
  dims[1] = H;
  if (c.page_size == 0) {
    dims[2] = (cuuint64_t)c.max_seq;
    dims[3] = (cuuint64_t)c.batch;
  } else {
    dims[2] = (cuuint64_t)c.page_size;
    dims[3] = (cuuint64_t)c.num_pages;
  }
  strides[0] = D * 2;
  strides[1] = H * D * 2;
  strides[2] = dims[2] * H * D * 2;
  const cuuint32_t box[4] = {64u, 1u, (cuuint32_t)kSubKeys, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MAC_OK : MAC_ERR_CUDA;
}

__global__ void mac_append_kernel(const AppendParams p) {
  const int u = blockIdx.x;
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  const int pos = p.seq_lens[b] - 1;
  if (pos < 0 || pos >= p.capacity) {
    if (threadIdx.x == 0) atomicOr(p.status, MAC_DEV_BAD_SEQ_LEN);
    return;
  }
  size_t row;
  if (p.page_size > 0) {
    const int pg = p.block_table[(size_t)b * p.max_pages + pos / p.page_size];
    if (pg < 0 || pg >= p.num_pages) {
      if (threadIdx.x == 0) atomicOr(p.status, MAC_DEV_BAD_PAGE);
      return;
    }
    row = ((size_t)pg * p.page_size + (size_t)(pos % p.page_size)) * p.Hkv + kvh;
  } else {
    row = ((size_t)b * p.capacity + (size_t)pos) * p.Hkv + kvh;
  }
  const uint4* ks = reinterpret_cast<const uint4*>(p.k_new + (size_t)u * p.D);
  const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + (size_t)u * p.D);
  uint4* kd = reinterpret_cast<uint4*>(p.K + row * p.D);
  uint4* vd = reinterpret_cast<uint4*>(p.V + row * p.D);
  for (int i = threadIdx.x; i < p.D / 8; i += blockDim.x) {
    kd[i] = ks[i];
    vd[i] = vs[i];
  }
}

}  // namespace

namespace mac {
cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  mac_append_kernel<<<p.B * p.Hkv, 32, 0, s>>>(p);
  return cudaGetLastError();
}
}  // namespace mac

extern "C" {

const char* mac_error_string(int code) {
  switch (code) {
    case MAC_OK: return "ok";
    case MAC_ERR_ARG: return "invalid argument";
    case MAC_ERR_SHAPE: return "unsupported shape";
    case MAC_ERR_CUDA: return "CUDA call failed";
    case MAC_ERR_OOM: return "device allocation failed";
    case MAC_ERR_DEVICE: return "device-side fault flagged in the status word";
    default: return "unknown error";
  }
}

int mac_init_state(const MacConfig* cfg, MacState** out) {
  if (!out) return MAC_ERR_ARG;
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc != MAC_OK) return rc;
  MacState* s = new (std::nothrow) MacState();
  if (!s) return MAC_ERR_OOM;
  s->cfg = *cfg;
  s->G = cfg->num_q_heads / cfg->num_kv_heads;
  s->ND = cfg->match_per_head ? s->G : 1;
  s->QES = cfg->q_bf16 ? 2 : 4;
  s->RES = cfg->ring_bf16 ? 2 : 4;
  s->U = cfg->batch * cfg->num_kv_heads;
  s->D = cfg->head_dim;
  s->W = cfg->window;
  s->min_keys = 128;
  s->piece_cost = 1024;
  s->unit_max = 1024;
  s->capacity = cfg->page_size == 0 ? cfg->max_seq : cfg->max_pages_per_seq * cfg->page_size;
  if (cudaGetDevice(&s->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&s->num_sms, cudaDevAttrMultiProcessorCount, s->device) != cudaSuccess) {
    delete s;
    return MAC_ERR_CUDA;
  }
  s->grid = s->num_sms;  // one resident CTA per SM (shared-memory bound)
  s->max_parts = (size_t)s->grid + 2 * (size_t)s->U;
  const size_t U = s->U, W1 = s->W + 1, G = s->G, D = s->D, B = cfg->batch, Hq = cfg->num_q_heads;
  const size_t Hkv = cfg->num_kv_heads;
  cudaError_t e = cudaSuccess;
  auto A = [&](cudaError_t r) {
    if (e == cudaSuccess) e = r;
  };
  A(alloc(&s->ring_q, U * W1 * G * D * s->RES));
  A(alloc(&s->ring_o, U * W1 * G * D * s->RES));
  A(alloc(&s->ring_m, U * W1 * G));
  A(alloc(&s->ring_l, U * W1 * G));
  A(alloc(&s->ring_pos, U * W1));
  A(alloc(&s->steps, U));
  A(alloc(&s->qrot, U * G * D));
  A(alloc(&s->plan, U));
  A(alloc(&s->hplan, U));
  A(alloc(&s->seg, 2 * U));
  A(alloc(&s->hdr, 1));
  A(alloc(&s->first_seg, (size_t)s->grid));
  A(alloc(&s->rate, (size_t)s->grid));
  A(alloc(&s->bounds, (size_t)s->grid + 1));
  A(alloc(&s->cw, (size_t)s->grid + 1));
  A(alloc(&s->claim, (size_t)s->grid));
  A(alloc(&s->part, s->max_parts * partial_floats((int)G, (int)D)));
  A(alloc(&s->unit_cnt, U));
  A(alloc(&s->done, 1));
  A(alloc(&s->dpart, U * W1 * (size_t)group_chunks((int)G)));
  A(alloc(&s->ucnt, U));
  A(alloc(&s->smid_of, (size_t)s->grid));
  A(alloc(&s->rank_of, (size_t)s->grid));
  A(alloc(&s->fsync, 2));
  A(alloc(&s->trace, (size_t)s->grid * kTracePoints));
  A(alloc(&s->counters, (size_t)kCounters));
  A(alloc(&s->inv_freq, D / 2));
  s->off_q = 0;
  s->off_pos = up256(s->off_q + B * Hq * D * s->QES);
  s->off_lens = up256(s->off_pos + B * sizeof(int));
  s->off_knew = up256(s->off_lens + B * sizeof(int));
  s->in_bytes_noappend = s->off_knew;
  s->off_vnew = up256(s->off_knew + B * Hkv * D * 2);
  s->in_bytes = up256(s->off_vnew + B * Hkv * D * 2);
  s->off_out = 0;
  s->off_lse = up256(B * Hq * D * sizeof(float));
  s->off_hit = up256(s->off_lse + B * Hq * sizeof(float));
  s->off_mpos = up256(s->off_hit + U * s->ND);
  s->off_status = up256(s->off_mpos + U * s->ND * sizeof(int));
  s->out_bytes = s->off_status + 16;
  A(alloc(&s->dev_in, s->in_bytes));
  A(alloc(&s->dev_out, s->out_bytes));
  A(cudaMallocHost(reinterpret_cast<void**>(&s->host_in), s->in_bytes));
  A(cudaMallocHost(reinterpret_cast<void**>(&s->host_out), s->out_bytes));
  A(cudaStreamCreateWithFlags(&s->cap_stream, cudaStreamNonBlocking));
  if (e == cudaSuccess) s->status = reinterpret_cast<unsigned*>(s->dev_out + s->off_status);
  if (e != cudaSuccess) {
    free_all(s);
    delete s;
    return e == cudaErrorMemoryAllocation ? MAC_ERR_OOM : MAC_ERR_CUDA;
  }
  A(cudaMemset(s->ring_q, 0, U * W1 * G * D * s->RES));
  A(cudaMemset(s->ring_o, 0, U * W1 * G * D * s->RES));
  A(cudaMemset(s->ring_m, 0, U * W1 * G * sizeof(float)));
  A(cudaMemset(s->ring_l, 0, U * W1 * G * sizeof(float)));
  A(cudaMemset(s->ring_pos, 0, U * W1 * sizeof(int)));
  A(cudaMemset(s->steps, 0, U * sizeof(int)));
  A(cudaMemset(s->unit_cnt, 0, U * sizeof(int)));
  A(cudaMemset(s->done, 0, sizeof(int)));
  A(cudaMemset(s->ucnt, 0, U * sizeof(int)));
  A(cudaMemset(s->fsync, 0, 2 * sizeof(int)));
  A(cudaMemset(s->trace, 0, (size_t)s->grid * kTracePoints * sizeof(unsigned long long)));
  A(cudaMemset(s->counters, 0, kCounters * sizeof(unsigned long long)));
  A(cudaMemset(s->rate, 0, s->grid * sizeof(float)));
  A(cudaMemset(s->claim, 0, s->grid * sizeof(int)));
  {  // even shares until the first rates are measured
    double* cw = (double*)malloc(sizeof(double) * (s->grid + 1));
    for (int c = 0; c <= s->grid; ++c) cw[c] = (double)c / s->grid;
    A(cudaMemcpy(s->cw, cw, sizeof(double) * (s->grid + 1), cudaMemcpyHostToDevice));
    free(cw);
  }
  A(cudaMemset(s->dev_out, 0, s->out_bytes));
  A(cudaMemset(s->hdr, 0, sizeof(PlanHeader)));
  double* inv = (double*)malloc(sizeof(double) * (D / 2));
  for (size_t i = 0; i < D / 2; ++i) inv[i] = pow(cfg->rope_theta, -2.0 * (double)i / (double)D);
  A(cudaMemcpy(s->inv_freq, inv, sizeof(double) * (D / 2), cudaMemcpyHostToDevice));
  free(inv);
  A(attend_prepare((int)D, (int)G));
  // the one-launch step: groups of up to 8 heads, one decision per KV head,
  // every CTA resident at once (a cooperative launch of one CTA per SM) and
  // each CTA's whole units within its item cache
  if (e == cudaSuccess && G <= (size_t)kMaxGroup && !cfg->match_per_head && U <= 2 * (size_t)s->grid) {
    int coop = 0, nb = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, s->device) == cudaSuccess && coop &&
        step_prepare((int)D, (int)G, &nb) == cudaSuccess && nb >= 1)
      s->one_launch_ok = 1;
    cudaGetLastError();
  }
  A(cudaDeviceSynchronize());
  if (e != cudaSuccess) {
    free_all(s);
    delete s;
    return MAC_ERR_CUDA;
  }
  *out = s;
  return MAC_OK;
}

void mac_destroy(MacState* s) {
  if (!s) return;
  cudaDeviceSynchronize();
  free_all(s);
  delete s;
}

int mac_reset_seq(MacState* s, int b, void* stream) {
  if (!s || b < 0 || b >= s->cfg.batch) return MAC_ERR_ARG;
  const int H = s->cfg.num_kv_heads;
  cudaError_t e = cudaMemsetAsync(s->steps + (size_t)b * H, 0, sizeof(int) * H, (cudaStream_t)stream);
  return e == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
}

int mac_set_min_keys_per_cta(MacState* s, int keys) {
  if (!s || keys < 1) return MAC_ERR_ARG;
  s->min_keys = keys;
  drop_graph(s);
  return MAC_OK;
}

int mac_set_piece_cost(MacState* s, int keys) {
  if (!s || keys < 0) return MAC_ERR_ARG;
  s->piece_cost = keys;
  drop_graph(s);
  return MAC_OK;
}

int mac_set_whole_unit_keys(MacState* s, int keys) {
  if (!s || keys < 0) return MAC_ERR_ARG;
  s->unit_max = keys;
  drop_graph(s);
  return MAC_OK;
}

int mac_set_one_launch(MacState* s, int on) {
  if (!s || on < 0 || on > 1) return MAC_ERR_ARG;
  s->one_launch = on;
  drop_graph(s);
  return MAC_OK;
}

int mac_one_launch(const MacState* s) { return s && s->one_launch && s->one_launch_ok ? 1 : 0; }

int mac_set_trace(MacState* s, int on) {
  if (!s || on < 0 || on > 1) return MAC_ERR_ARG;
  s->tracing = on;
  drop_graph(s);
  return MAC_OK;
}

int mac_get_trace(MacState* s, unsigned long long* stamps, size_t n_stamps, unsigned long long* counters) {
  if (!s) return MAC_ERR_ARG;
  const size_t n = (size_t)s->grid * kTracePoints;
  if (stamps && n_stamps < n) return MAC_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MAC_ERR_CUDA;
  if (stamps && cudaMemcpy(stamps, s->trace, n * sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MAC_ERR_CUDA;
  if (counters) {
    if (cudaMemcpy(counters, s->counters, kCounters * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
        cudaSuccess)
      return MAC_ERR_CUDA;
  }
  if (cudaMemset(s->counters, 0, kCounters * sizeof(unsigned long long)) != cudaSuccess) return MAC_ERR_CUDA;
  return MAC_OK;
}

int mac_set_reproducible(MacState* s, int on) {
  if (!s || on < 0 || on > 1) return MAC_ERR_ARG;
  s->reproducible = on;
  drop_graph(s);
  return MAC_OK;
}

int mac_attend_grid(const MacState* s) { return s ? s->grid : 0; }

static int match_impl(MacState* s, float tau, const void* q_pre, const int* rope_pos, const int* block_table,
                      const int* seq_lens, float* out, float* lse, uint8_t* hit_mask, int* match_pos, void* stream);

int mac_match(MacState* s, const void* q_pre, const int* rope_pos, const int* block_table, const int* seq_lens,
              float* out, float* lse, uint8_t* hit_mask, int* match_pos, void* stream) {
  Range r("mac_match");
  if (!s) return MAC_ERR_ARG;
  return match_impl(s, s->cfg.tau, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask, match_pos, stream);
}

static int fill_match(MacState* s, float tau, const void* q_pre, const int* rope_pos, const int* block_table,
                      const int* seq_lens, float* out, float* lse, uint8_t* hit_mask, int* match_pos,
                      MatchParams& p) {
  if (!s || !q_pre || !rope_pos || !seq_lens || !out || !lse) return MAC_ERR_ARG;
  if (!aligned16(q_pre)) return MAC_ERR_ARG;
  if (s->cfg.page_size > 0 && !block_table) return MAC_ERR_ARG;
  p.q_pre = q_pre;
  p.q_bf16 = s->cfg.q_bf16;
  p.ring_bf16 = s->cfg.ring_bf16;
  p.rope_pos = rope_pos;
  p.seq_lens = seq_lens;
  p.block_table = s->cfg.page_size > 0 ? block_table : nullptr;
  p.out = out;
  p.lse = lse;
  p.hit_mask = hit_mask;
  p.match_pos = match_pos;
  p.ring_q = s->ring_q;
  p.ring_pos = s->ring_pos;
  p.steps = s->steps;
  p.inv_freq = s->inv_freq;
  p.qrot = s->qrot;
  p.plan = s->plan;
  p.hplan = s->hplan;
  p.seg = s->seg;
  p.hdr = s->hdr;
  p.first_seg = s->first_seg;
  p.cw = s->reproducible ? nullptr : s->cw;  // null: the even split on every step
  p.bounds = s->bounds;
  p.claim = s->claim;
  p.done = s->done;
  p.dpart = s->dpart;
  p.ucnt = s->ucnt;
  p.trace = s->tracing ? s->trace : nullptr;
  p.status = s->status;
  p.B = s->cfg.batch;
  p.Hq = s->cfg.num_q_heads;
  p.Hkv = s->cfg.num_kv_heads;
  p.G = s->G;
  p.W = s->W;
  p.band = s->cfg.band - s->cfg.cut_mode;  // c = max(0, p - band + cut_mode)
  p.per_head = s->cfg.match_per_head;
  p.ring_bf16 = s->cfg.ring_bf16;
  p.page_size = s->cfg.page_size;
  p.max_pages = s->cfg.max_pages_per_seq;
  p.num_pages = s->cfg.num_pages;
  p.capacity = s->capacity;
  p.tau = tau;
  p.grid = s->grid;
  p.min_keys = s->min_keys;
  p.piece_cost = s->piece_cost;
  p.unit_max = s->G > kMaxGroup ? 0 : s->unit_max;  // groups of 16-64 heads run split items only
  return MAC_OK;
}

static int match_impl(MacState* s, float tau, const void* q_pre, const int* rope_pos, const int* block_table,
                      const int* seq_lens, float* out, float* lse, uint8_t* hit_mask, int* match_pos, void* stream) {
  MatchParams p;
  const int rc = fill_match(s, tau, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask, match_pos, p);
  if (rc != MAC_OK) return rc;
  return launch_match(p, s->D, (cudaStream_t)stream) == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
}

static int fill_attend(MacState* s, const uint16_t* K, const uint16_t* V, const int* block_table, float* out,
                       float* lse, AttendParams& p) {
  if (!s || !K || !V || !out || !lse) return MAC_ERR_ARG;
  if (!aligned16(K) || !aligned16(V)) return MAC_ERR_ARG;
  if (s->cfg.page_size > 0 && !block_table) return MAC_ERR_ARG;
  if (K != s->tm_k_ptr) {
    int rc = encode_kv_map(s, &s->tmK, K);
    if (rc != MAC_OK) return rc;
    s->tm_k_ptr = K;
  }
  if (V != s->tm_v_ptr) {
    int rc = encode_kv_map(s, &s->tmV, V);
    if (rc != MAC_OK) return rc;
    s->tm_v_ptr = V;
  }
  p.tmK = s->tmK;
  p.tmV = s->tmV;
  p.block_table = s->cfg.page_size > 0 ? block_table : nullptr;
  p.qrot = s->qrot;
  p.plan = s->plan;
  p.hplan = s->hplan;
  p.seg = s->seg;
  p.hdr = s->hdr;
  p.first_seg = s->first_seg;
  p.bounds = s->bounds;
  p.claim = s->claim;
  p.rate = s->reproducible ? nullptr : s->rate;  // null: no rate is learned
  p.cw = s->reproducible ? nullptr : s->cw;
  p.part = s->part;
  p.unit_cnt = s->unit_cnt;
  p.ring_o = s->ring_o;
  p.ring_m = s->ring_m;
  p.ring_l = s->ring_l;
  p.ring_pos = s->ring_pos;
  p.out = out;
  p.lse = lse;
  p.status = s->status;
  p.Hq = s->cfg.num_q_heads;
  p.Hkv = s->cfg.num_kv_heads;
  p.G = s->G;
  p.W = s->W;
  p.page_size = s->cfg.page_size;
  p.max_pages = s->cfg.max_pages_per_seq;
  p.nseg = 2 * s->U;
  p.grid = s->grid;
  p.per_head = s->cfg.match_per_head;
  p.ring_bf16 = s->cfg.ring_bf16;
  p.smid_of = s->smid_of;
  p.rank_of = s->rank_of;
  p.fsync = s->fsync;
  p.trace = s->tracing ? s->trace : nullptr;
  p.counters = s->tracing ? s->counters : nullptr;
  return MAC_OK;
}

// With tracing on, a step's phase times start from zero (a phase a CTA does
// not reach stays 0).
static int clear_trace(MacState* s, cudaStream_t st) {
  if (!s->tracing) return MAC_OK;
  return cudaMemsetAsync(s->trace, 0, (size_t)s->grid * kTracePoints * sizeof(unsigned long long), st) ==
                 cudaSuccess
             ? MAC_OK
             : MAC_ERR_CUDA;
}

int mac_attend(MacState* s, const uint16_t* K, const uint16_t* V, const int* block_table, float* out, float* lse,
               void* stream) {
  Range r("mac_attend");
  AttendParams p;
  int rc = fill_attend(s, K, V, block_table, out, lse, p);
  if (rc == MAC_OK) rc = clear_trace(s, (cudaStream_t)stream);
  if (rc != MAC_OK) return rc;
  return launch_attend(p, s->D, s->grid, (cudaStream_t)stream) == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
}

int mac_decode_step(MacState* s, const void* q_pre, const int* rope_pos, const uint16_t* K, const uint16_t* V,
                    const int* block_table, const int* seq_lens, float* out, float* lse, uint8_t* hit_mask,
                    int* match_pos, void* stream) {
  Range r("mac_decode_step");
  if (!s || !K || !V) return MAC_ERR_ARG;
  if (!aligned16(K) || !aligned16(V)) return MAC_ERR_ARG;
  if (s->one_launch && s->one_launch_ok) {
    // match, every whole unit and the split ranges in one cooperative launch
    MatchParams mp;
    AttendParams ap;
    int rc = fill_match(s, s->cfg.tau, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask, match_pos, mp);
    if (rc == MAC_OK) rc = fill_attend(s, K, V, block_table, out, lse, ap);
    if (rc == MAC_OK) rc = clear_trace(s, (cudaStream_t)stream);
    if (rc != MAC_OK) return rc;
    return launch_step(ap, mp, s->D, s->grid, (cudaStream_t)stream) == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
  }
  int rc = mac_match(s, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask, match_pos, stream);
  if (rc != MAC_OK) return rc;
  return mac_attend(s, K, V, block_table, out, lse, stream);
}

int mac_append_kv(MacState* s, uint16_t* K, uint16_t* V, const int* block_table, const int* seq_lens,
                  const uint16_t* k_new, const uint16_t* v_new, void* stream) {
  Range r("mac_append_kv");
  if (!s || !K || !V || !seq_lens || !k_new || !v_new) return MAC_ERR_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(k_new) || !aligned16(v_new)) return MAC_ERR_ARG;
  if (s->cfg.page_size > 0 && !block_table) return MAC_ERR_ARG;
  AppendParams p;
  p.K = K;
  p.V = V;
  p.block_table = s->cfg.page_size > 0 ? block_table : nullptr;
  p.seq_lens = seq_lens;
  p.k_new = k_new;
  p.v_new = v_new;
  p.status = s->status;
  p.B = s->cfg.batch;
  p.Hkv = s->cfg.num_kv_heads;
  p.D = s->D;
  p.page_size = s->cfg.page_size;
  p.max_pages = s->cfg.max_pages_per_seq;
  p.num_pages = s->cfg.num_pages;
  p.capacity = s->capacity;
  return launch_append(p, (cudaStream_t)stream) == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
}

int mac_warm_start(MacState* s, int n, const void* q_pre, const int* rope_pos, const uint16_t* K, const uint16_t* V,
                   const int* block_table, const int* seq_lens, void* stream) {
  Range r("mac_warm_start");
  if (!s || n < 0 || n > s->W) return MAC_ERR_ARG;
  if (n > 0 && (!q_pre || !rope_pos || !seq_lens || !K || !V)) return MAC_ERR_ARG;
  if (n > 0 && (!aligned16(q_pre) || !aligned16(K) || !aligned16(V))) return MAC_ERR_ARG;
  if (s->cfg.page_size > 0 && n > 0 && !block_table) return MAC_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  // every window starts empty, then each position runs as a step with threshold 0
  if (cudaMemsetAsync(s->steps, 0, (size_t)s->U * sizeof(int), st) != cudaSuccess) return MAC_ERR_CUDA;
  const size_t B = s->cfg.batch, Hq = s->cfg.num_q_heads, D = s->D;
  float* out = reinterpret_cast<float*>(s->dev_out + s->off_out);  // outputs of these steps are not kept
  float* lse = reinterpret_cast<float*>(s->dev_out + s->off_lse);
  for (int j = 0; j < n; ++j) {
    int rc = match_impl(s, 0.f, static_cast<const unsigned char*>(q_pre) + (size_t)j * B * Hq * D * s->QES, rope_pos + (size_t)j * B, block_table,
                        seq_lens + (size_t)j * B, out, lse, nullptr, nullptr, stream);
    if (rc != MAC_OK) return rc;
    rc = mac_attend(s, K, V, block_table, out, lse, stream);
    if (rc != MAC_OK) return rc;
  }
  return MAC_OK;
}

// Enqueue one host step on `st`: copy the packed inputs in, append the new
// rows (optional), run the step, copy the packed outputs (and status) out.
static int enqueue_host_step(MacState* s, uint16_t* K, uint16_t* V, const int* block_table, bool append,
                             cudaStream_t st) {
  unsigned char* di = s->dev_in;
  unsigned char* dout = s->dev_out;
  if (cudaMemcpyAsync(di, s->host_in, append ? s->in_bytes : s->in_bytes_noappend, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return MAC_ERR_CUDA;
  const int* lens = reinterpret_cast<const int*>(di + s->off_lens);
  int rc;
  if (append) {
    rc = mac_append_kv(s, K, V, block_table, lens, reinterpret_cast<const uint16_t*>(di + s->off_knew),
                       reinterpret_cast<const uint16_t*>(di + s->off_vnew), st);
    if (rc != MAC_OK) return rc;
  }
  rc = mac_decode_step(s, di + s->off_q, reinterpret_cast<const int*>(di + s->off_pos),
                       K, V, block_table, lens, reinterpret_cast<float*>(dout + s->off_out),
                       reinterpret_cast<float*>(dout + s->off_lse), dout + s->off_hit,
                       reinterpret_cast<int*>(dout + s->off_mpos), st);
  if (rc != MAC_OK) return rc;
  return cudaMemcpyAsync(s->host_out, dout, s->out_bytes, cudaMemcpyDeviceToHost, st) == cudaSuccess ? MAC_OK
                                                                                                      : MAC_ERR_CUDA;
}

int mac_decode_step_host(MacState* s, const void* q_pre_h, const int* rope_pos_h, const int* seq_lens_h,
                         const uint16_t* k_new_h, const uint16_t* v_new_h, uint16_t* K, uint16_t* V,
                         const int* block_table, float* out_h, float* lse_h, uint8_t* hit_h, int* match_pos_h,
                         void* stream) {
  Range r("mac_decode_step_host");
  if (!s || !q_pre_h || !rope_pos_h || !seq_lens_h || !K || !V) return MAC_ERR_ARG;
  if ((k_new_h == nullptr) != (v_new_h == nullptr)) return MAC_ERR_ARG;
  if (!aligned16(K) || !aligned16(V)) return MAC_ERR_ARG;
  if (s->cfg.page_size > 0 && !block_table) return MAC_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t B = s->cfg.batch, Hq = s->cfg.num_q_heads, Hkv = s->cfg.num_kv_heads, D = s->D, U = s->U;
  const bool append = k_new_h != nullptr;
  // inputs into the pinned block (the graph copies the whole block in)
  memcpy(s->host_in + s->off_q, q_pre_h, B * Hq * D * s->QES);
  memcpy(s->host_in + s->off_pos, rope_pos_h, B * sizeof(int));
  memcpy(s->host_in + s->off_lens, seq_lens_h, B * sizeof(int));
  if (append) {
    memcpy(s->host_in + s->off_knew, k_new_h, B * Hkv * D * 2);
    memcpy(s->host_in + s->off_vnew, v_new_h, B * Hkv * D * 2);
  }
  const int* bt = s->cfg.page_size > 0 ? block_table : nullptr;
  if (!s->gexec || s->g_k != K || s->g_v != V || s->g_bt != bt || s->g_append != (int)append) {
    // (re)capture the step for these cache pointers
    drop_graph(s);
    cudaGraph_t graph = nullptr;
    bool ok = cudaStreamBeginCapture(s->cap_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    const int rc = ok ? enqueue_host_step(s, K, V, bt, append, s->cap_stream) : MAC_ERR_CUDA;
    if (ok) ok = cudaStreamEndCapture(s->cap_stream, &graph) == cudaSuccess && rc == MAC_OK;
    if (ok) ok = cudaGraphInstantiate(&s->gexec, graph, 0) == cudaSuccess;
    if (graph) cudaGraphDestroy(graph);
    if (!ok) {
      drop_graph(s);
      cudaGetLastError();
    } else {
      s->g_k = K;
      s->g_v = V;
      s->g_bt = bt;
      s->g_append = (int)append;
    }
  }
  if (s->gexec) {
    if (cudaGraphLaunch(s->gexec, st) != cudaSuccess) return MAC_ERR_CUDA;
  } else {
    const int rc = enqueue_host_step(s, K, V, bt, append, st);  // no graph: the same work, launched directly
    if (rc != MAC_OK) return rc;
  }
  {
    Range w("wait for the step");
    if (cudaStreamSynchronize(st) != cudaSuccess) return MAC_ERR_CUDA;
  }
  if (out_h) memcpy(out_h, s->host_out + s->off_out, B * Hq * D * sizeof(float));
  if (lse_h) memcpy(lse_h, s->host_out + s->off_lse, B * Hq * sizeof(float));
  if (hit_h) memcpy(hit_h, s->host_out + s->off_hit, U * s->ND);
  if (match_pos_h) memcpy(match_pos_h, s->host_out + s->off_mpos, U * s->ND * sizeof(int));
  unsigned status;
  memcpy(&status, s->host_out + s->off_status, sizeof status);
  return status ? MAC_ERR_DEVICE : MAC_OK;
}

int mac_selftest_wait_timeout(unsigned* device_status, void* stream) {
  if (!device_status) return MAC_ERR_ARG;
  return launch_wait_selftest(device_status, (cudaStream_t)stream) == cudaSuccess ? MAC_OK : MAC_ERR_CUDA;
}

int mac_get_status(MacState* s, int* device_status) {
  if (!s) return MAC_ERR_ARG;
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return MAC_ERR_CUDA;
  if (cudaMemcpy(&v, s->status, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return MAC_ERR_CUDA;
  if (cudaMemset(s->status, 0, sizeof(unsigned)) != cudaSuccess) return MAC_ERR_CUDA;
  if (device_status) *device_status = (int)v;
  return v ? MAC_ERR_DEVICE : MAC_OK;
}

size_t mac_state_bytes(const MacState* s) {
  if (!s) return 0;
  const size_t U = s->U, W1 = s->W + 1, G = s->G, D = s->D;
  return 8 * sizeof(int) + 2 * U * W1 * G * D * s->RES + 2 * U * W1 * G * sizeof(float) +
         U * W1 * sizeof(int) + U * sizeof(int);
}

static int copy_state(MacState* s, void* host, size_t bytes, bool to_host) {
  if (!s || !host || bytes < mac_state_bytes(s)) return MAC_ERR_ARG;
  const size_t U = s->U, W1 = s->W + 1, G = s->G, D = s->D;
  int hdr[8] = {0x4D414331, (int)U, (int)W1, (int)G, (int)D, s->cfg.ring_bf16, 0, 0};
  unsigned char* h = static_cast<unsigned char*>(host);
  if (to_host) {
    memcpy(h, hdr, sizeof hdr);
  } else {
    if (memcmp(h, hdr, sizeof hdr) != 0) return MAC_ERR_SHAPE;
  }
  h += sizeof hdr;
  const size_t es = s->RES;
  struct Part {
    void* dev;
    size_t bytes;
  } parts[] = {{s->ring_q, U * W1 * G * D * es}, {s->ring_o, U * W1 * G * D * es}, {s->ring_m, U * W1 * G * 4},
               {s->ring_l, U * W1 * G * 4},     {s->ring_pos, U * W1 * 4},      {s->steps, U * 4}};
  if (cudaDeviceSynchronize() != cudaSuccess) return MAC_ERR_CUDA;
  for (const Part& p : parts) {
    cudaError_t e = to_host ? cudaMemcpy(h, p.dev, p.bytes, cudaMemcpyDeviceToHost)
                            : cudaMemcpy(p.dev, h, p.bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return MAC_ERR_CUDA;
    h += p.bytes;
  }
  return MAC_OK;
}

int mac_export_state(const MacState* s, void* host_buf, size_t bytes) {
  return copy_state(const_cast<MacState*>(s), host_buf, bytes, true);
}

int mac_import_state(MacState* s, const void* host_buf, size_t bytes) {
  return copy_state(s, const_cast<void*>(host_buf), bytes, false);
}

}  // extern "C"
