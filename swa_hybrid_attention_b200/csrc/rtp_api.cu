// C ABI of librtp.so (declared in include/rtp.h): argument validation, the
// routing planner, TMA descriptor set-up and kernel dispatch.  No C++
// exception crosses the boundary; every entry point returns an rtp_status.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/rtp.h"
#include "internal.cuh"
#include "sm100.cuh"

using namespace rtp;

struct rtp_plan;
struct rtp_pipeline {
  rtp_attn_cfg cfg;
  int device = 0;
  int n_sparse = 0;
  std::vector<rtp_plan*> plans;  // one ranged plan per chunk of query rows
  std::vector<int> begin, end;
  cudaStream_t s_in = nullptr, s_out = nullptr;  // uploads, downloads
  std::vector<cudaEvent_t> ev_in, ev_out;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr;
};

struct rtp_plan {
  rtp_attn_cfg cfg;
  int device = 0;
  int num_sms = 148;
  int n_sparse = 0;
  int nqt = 0;  // 128-row query tiles
  int nqb = 0;  // query blocks of `block` rows
  int q_begin = 0, q_end = 0;  // query rows of this plan (whole sequence unless ranged)
  std::vector<uint8_t> kind;
  std::vector<int32_t> slot_heads;
  std::vector<int32_t> items_host;  // [n_items][4]
  long n_items = 0;
  long n_local = 0;  // items [0, n_local) see only keys at or after key_begin
  int key_begin = 0;
  void* d_mem = nullptr;
  int4* d_items = nullptr;
  int32_t* d_slot_heads = nullptr;
  float scale = 0.f;
};

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// An NVTX range named after the entry point for the duration of the call
// (visible in a profiler's timeline; no cost when none is attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
};

// Self-test of the bounded wait used by every kernel: an mbarrier nobody
// arrives on, waited for with a short limit.
__global__ void bounded_wait_selftest_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  __syncwarp();
}

// ---------------------------------------------------------------- status word
std::mutex g_status_mu;
uint32_t* g_status[64] = {nullptr};

uint32_t* status_word(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status[dev]) {
    uint32_t* p = nullptr;
    if (cudaMalloc(&p, sizeof(uint32_t)) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, sizeof(uint32_t)) != cudaSuccess) {
      cudaFree(p);
      return nullptr;
    }
    g_status[dev] = p;
  }
  return g_status[dev];
}

// The status word of `dev` if it has been created, else NULL (no allocation).
uint32_t* existing_status_word(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  return g_status[dev];
}

// ------------------------------------------------------------- TMA encoding
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 [slabs][slab_rows][128] viewed as a 3-D tensor of which the first
// `rows` rows of each slab are used (slab_rows = 0 means rows), 128-byte
// swizzled boxes of 64 columns x box_rows rows.  Rows past `rows` read as
// zero.
bool encode_bf16_3d(CUtensorMap* map, const void* base, long rows, long slabs, int box_rows, long slab_rows = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (slab_rows < rows) slab_rows = rows;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slabs)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                           static_cast<cuuint64_t>(kHeadDim) * 2 * static_cast<cuuint64_t>(slab_rows)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool cfg_common_ok(const rtp_attn_cfg* c) {
  if (!c) return false;
  if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1) return false;
  if (c->head_dim != kHeadDim || c->rank != kRank || c->n_sink != 1) return false;
  if (c->n_q_heads % c->n_kv_heads != 0) return false;
  const int g = c->n_q_heads / c->n_kv_heads;
  if (g > 16) return false;
  if (c->window < 1 || c->n_local < 1 || c->topk < 0) return false;
  if (c->block != 64 && c->block != 128) return false;
  if (!(c->scale >= 0.f) || !std::isfinite(c->scale)) return false;
  if (static_cast<long>(c->batch) * c->n_q_heads > (1L << 24)) return false;
  return true;
}

bool cfg_prefill_ok(const rtp_attn_cfg* c) {
  if (!cfg_common_ok(c)) return false;
  if ((c->n_q_heads / c->n_kv_heads) % 2 != 0) return false;
  if (c->seq < 1 || c->seq % c->block != 0) return false;
  if (c->seq > (1 << 30) / 2) return false;
  const long nb = c->seq / c->block;
  if (nb * 4 > 200 * 1024) return false;  // selection keys live in shared memory
  return true;
}

float effective_scale(const rtp_attn_cfg* c) {
  return c->scale > 0.f ? c->scale : 1.0f / std::sqrt(static_cast<float>(c->head_dim));
}

// Selected-list length for a query block t with at least... (see rtp.h):
// all blocks 0..t when there are at most topk candidates, else sink + topk +
// local.
long selected_count(long t, int topk, int n_local) {
  long ncand = std::max<long>(0, t - n_local);
  return ncand > topk ? 1L + topk + n_local : t + 1;
}

rtp_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RTP_OK : RTP_ERR_CUDA; }

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

// The indexer of a (possibly ranged) plan; q and k point at the plan's first
// row of slab 0 and consecutive (sequence, head) slabs are slab_rows apart.
rtp_status indexer_run(const rtp_plan* plan, const void* q, const void* k, int slab_rows, const float* proj,
                       float* centroids, float* qbar, void* stream) {
  if (plan->n_sparse == 0) return RTP_OK;
  if (!q || !k || !proj || !centroids || !qbar) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(proj) || !aligned16(centroids) || !aligned16(qbar))
    return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  IndexerArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.proj = proj;
  a.centroids = centroids;
  a.qbar = qbar;
  a.slot_heads = plan->d_slot_heads;
  a.batch = c.batch;
  a.seq = c.seq;
  a.n_q_heads = c.n_q_heads;
  a.n_kv_heads = c.n_kv_heads;
  a.group = c.n_q_heads / c.n_kv_heads;
  a.n_sparse = plan->n_sparse;
  a.block = c.block;
  a.blk0 = plan->q_begin / c.block;
  a.rows = slab_rows;
  a.n_blocks = plan->q_end / c.block - a.blk0;
  return cuda_status(launch_indexer(a, reinterpret_cast<cudaStream_t>(stream)));
}

// The prefill of a (possibly ranged) plan.  q and o point at the plan's first
// query row of slab 0, their slabs q_slab rows apart; k and v start at row 0,
// their slabs kv_slab rows apart.
// Work items [item_begin, item_end) of the plan's list (item_end < 0: to the
// end) run on at most max_ctas persistent CTAs (0: one per SM).
rtp_status prefill_run(const rtp_plan* plan, const void* q, int q_slab, const void* k, const void* v, int kv_slab,
                       const int32_t* sel, const int32_t* sel_cnt, void* o, void* stream, int sel_heads = 0,
                       long item_begin = 0, long item_end = -1, int max_ctas = 0) {
  if (item_end < 0) item_end = plan->n_items;
  if (item_begin < 0 || item_begin > item_end || item_end > plan->n_items || max_ctas < 0)
    return RTP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return RTP_ERR_INVALID_ARG;
  if (plan->n_sparse > 0 && (!sel || !sel_cnt)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (sel && !aligned16(sel)) return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  if (current_device() != plan->device) return RTP_ERR_INVALID_ARG;
  CUtensorMap mq, mk, mv;
  const int q_rows = plan->q_end - plan->q_begin;
  if (!encode_bf16_3d(&mq, q, q_rows, static_cast<long>(c.batch) * c.n_q_heads, 128, q_slab) ||
      !encode_bf16_3d(&mk, k, plan->q_end, static_cast<long>(c.batch) * c.n_kv_heads, 64, kv_slab) ||
      !encode_bf16_3d(&mv, v, plan->q_end, static_cast<long>(c.batch) * c.n_kv_heads, 64, kv_slab))
    return RTP_ERR_CUDA;
  PrefillArgs a;
  a.items = plan->d_items + item_begin;
  a.n_items = item_end - item_begin;
  a.sel = sel;
  a.cnt = sel_cnt;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.batch = c.batch;
  a.seq = c.seq;
  a.q_row0 = plan->q_begin;
  a.q_rows = q_rows;
  a.q_slab = q_slab;
  a.n_q_heads = c.n_q_heads;
  a.n_kv_heads = c.n_kv_heads;
  a.group = c.n_q_heads / c.n_kv_heads;
  a.n_sparse = plan->n_sparse;
  a.window = c.window;
  a.block = c.block;
  a.kmax = c.topk + 1 + c.n_local;
  a.nqb = plan->nqb;
  a.scale_log2 = plan->scale * kLog2e;
  a.status = status_word(plan->device);
  a.sel_heads = sel_heads;
  const int ctas = static_cast<int>(
      std::min<long>(a.n_items, max_ctas > 0 ? std::min(max_ctas, plan->num_sms) : plan->num_sms));
  if (ctas <= 0) return RTP_OK;
  return cuda_status(launch_prefill(a, mq, mk, mv, ctas, reinterpret_cast<cudaStream_t>(stream)));
}
rtp_status route_heads(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int q_begin, int q_end, int key_begin,
                       void* stream, rtp_plan** out);
}  // namespace

extern "C" {

const char* rtp_status_str(rtp_status s) {
  switch (s) {
    case RTP_OK: return "RTP_OK";
    case RTP_ERR_INVALID_ARG: return "RTP_ERR_INVALID_ARG";
    case RTP_ERR_UNSUPPORTED: return "RTP_ERR_UNSUPPORTED";
    case RTP_ERR_CUDA: return "RTP_ERR_CUDA";
    case RTP_ERR_TIMEOUT: return "RTP_ERR_TIMEOUT";
    case RTP_ERR_NO_MEMORY: return "RTP_ERR_NO_MEMORY";
  }
  return "RTP_ERR_UNKNOWN";
}

int rtp_version(void) { return (1 << 16) | 0; }

rtp_status rtp_route_heads(const rtp_attn_cfg* cfg, const uint8_t* kind_host, void* stream, rtp_plan** out) {
  if (!cfg) {
    if (out) *out = nullptr;
    return RTP_ERR_INVALID_ARG;
  }
  return rtp_route_heads_range(cfg, kind_host, 0, cfg->seq, stream, out);
}

rtp_status rtp_route_heads_range(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int q_begin, int q_end,
                                 void* stream, rtp_plan** out) {
  CallRange range_("rtp_route_heads_range");
  return route_heads(cfg, kind_host, q_begin, q_end, 0, stream, out);
}

rtp_status rtp_route_heads_split(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int q_begin, int q_end,
                                 int key_begin, void* stream, rtp_plan** out) {
  CallRange range_("rtp_route_heads_split");
  if (!cfg || key_begin < 0 || key_begin > q_begin) {
    if (out) *out = nullptr;
    return RTP_ERR_INVALID_ARG;
  }
  return route_heads(cfg, kind_host, q_begin, q_end, key_begin, stream, out);
}

long rtp_plan_num_local_items(const rtp_plan* plan) { return plan ? plan->n_local : -1; }

}  // extern "C"

namespace {
// The planner behind rtp_route_heads(_range/_split): work items of the query
// rows [q_begin, q_end), those whose visible keys all lie at or after
// key_begin first, each part longest first.
rtp_status route_heads(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int q_begin, int q_end, int key_begin,
                       void* stream, rtp_plan** out) {
  if (!out) return RTP_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg_prefill_ok(cfg) || !kind_host) return RTP_ERR_INVALID_ARG;
  if (q_begin < 0 || q_begin >= q_end || q_end > cfg->seq || q_begin % 128 != 0 ||
      (q_end % 128 != 0 && q_end != cfg->seq))
    return RTP_ERR_INVALID_ARG;
  for (int h = 0; h < cfg->n_kv_heads; ++h)
    if (kind_host[h] > RTP_HEAD_SPARSE) return RTP_ERR_INVALID_ARG;

  rtp_plan* p = new (std::nothrow) rtp_plan();
  if (!p) return RTP_ERR_NO_MEMORY;
  p->cfg = *cfg;
  p->scale = effective_scale(cfg);
  p->device = current_device();
  cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
  p->kind.assign(kind_host, kind_host + cfg->n_kv_heads);
  std::vector<int> slot_of(cfg->n_kv_heads, -1);
  for (int h = 0; h < cfg->n_kv_heads; ++h)
    if (kind_host[h] == RTP_HEAD_SPARSE) {
      slot_of[h] = static_cast<int>(p->slot_heads.size());
      p->slot_heads.push_back(h);
    }
  p->n_sparse = static_cast<int>(p->slot_heads.size());
  p->nqt = (cfg->seq + 127) / 128;
  p->nqb = cfg->seq / cfg->block;
  p->q_begin = q_begin;
  p->q_end = q_end;
  const int t_lo = q_begin / 128, t_hi = (q_end + 127) / 128;
  const int group = cfg->n_q_heads / cfg->n_kv_heads;
  const int pairs = group / 2;

  // Work items with their cost (KV tiles visited), then longest first.
  struct W {
    long cost;
    bool local;
    int32_t v[4];
  };
  std::vector<W> work;
  work.reserve(static_cast<size_t>(cfg->batch) * cfg->n_kv_heads * pairs * (t_hi - t_lo));
  for (int b = 0; b < cfg->batch; ++b)
    for (int h = 0; h < cfg->n_kv_heads; ++h)
      for (int t = t_lo; t < t_hi; ++t) {
        long cost;
        const int kind = kind_host[h];
        if (kind == RTP_HEAD_FULL) {
          cost = t + 1;
        } else if (kind == RTP_HEAD_SWA) {
          long first = 128L * t - cfg->window + 1;
          long lo = first <= 0 ? 0 : first / 128;
          cost = t - lo + 1;
        } else if (cfg->block == 128) {
          cost = selected_count(t, cfg->topk, cfg->n_local);
        } else {
          long c0 = selected_count(2L * t, cfg->topk, cfg->n_local);
          long c1 = 2L * t + 1 < p->nqb ? selected_count(2L * t + 1, cfg->topk, cfg->n_local) : 0;
          cost = (c0 + c1 + 1) / 2;
        }
        const int slot = kind == RTP_HEAD_SPARSE ? slot_of[h] : 0;
        // The earliest key the tile can see: the window's first row for a
        // streaming head; row 0 for a full head and for a sparse head (its
        // selection always holds the sink block).
        const long first_key = kind == RTP_HEAD_SWA ? std::max(0L, 128L * t - cfg->window + 1) : 0L;
        const bool local = first_key >= key_begin;
        for (int pr = 0; pr < pairs; ++pr)
          work.push_back(W{cost, local, {kind | (slot << 8), b * cfg->n_kv_heads + h, pr, t}});
      }
  std::stable_sort(work.begin(), work.end(), [](const W& a, const W& b) {
    if (a.local != b.local) return a.local;
    return a.cost > b.cost;
  });
  p->key_begin = key_begin;
  p->n_local = 0;
  for (const W& w : work) p->n_local += w.local ? 1 : 0;
  p->n_items = static_cast<long>(work.size());
  p->items_host.resize(work.size() * 4);
  for (size_t i = 0; i < work.size(); ++i) std::memcpy(&p->items_host[i * 4], work[i].v, sizeof(work[i].v));

  const size_t items_bytes = work.size() * sizeof(int4);
  const size_t slots_bytes = std::max<size_t>(1, p->slot_heads.size()) * sizeof(int32_t);
  if (cudaMalloc(&p->d_mem, items_bytes + 256 + slots_bytes) != cudaSuccess) {
    delete p;
    return RTP_ERR_NO_MEMORY;
  }
  p->d_items = reinterpret_cast<int4*>(p->d_mem);
  p->d_slot_heads = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p->d_mem) + ((items_bytes + 255) / 256) * 256);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(p->d_items, p->items_host.data(), items_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->slot_heads.empty())
    e = cudaMemcpyAsync(p->d_slot_heads, p->slot_heads.data(), p->slot_heads.size() * sizeof(int32_t),
                        cudaMemcpyHostToDevice, s);
  // The host arrays stay alive with the plan; make sure the upload finished
  // before the call returns so that a caller may use the plan on any stream.
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaFree(p->d_mem);
    delete p;
    return RTP_ERR_CUDA;
  }
  if (!status_word(p->device)) {
    cudaFree(p->d_mem);
    delete p;
    return RTP_ERR_NO_MEMORY;
  }
  *out = p;
  return RTP_OK;
}
}  // namespace

extern "C" {

void rtp_plan_destroy(rtp_plan* plan) {
  if (!plan) return;
  if (plan->d_mem) cudaFree(plan->d_mem);
  delete plan;
}

int rtp_plan_num_sparse(const rtp_plan* plan) { return plan ? plan->n_sparse : -1; }

long rtp_plan_num_items(const rtp_plan* plan) { return plan ? plan->n_items : -1; }

rtp_status rtp_plan_sparse_heads(const rtp_plan* plan, int32_t* slots_host) {
  if (!plan || (!slots_host && plan->n_sparse > 0)) return RTP_ERR_INVALID_ARG;
  if (plan->n_sparse > 0) std::memcpy(slots_host, plan->slot_heads.data(), plan->slot_heads.size() * sizeof(int32_t));
  return RTP_OK;
}

rtp_status rtp_plan_work_items(const rtp_plan* plan, int32_t* items_host) {
  if (!plan || !items_host) return RTP_ERR_INVALID_ARG;
  std::memcpy(items_host, plan->items_host.data(), plan->items_host.size() * sizeof(int32_t));
  return RTP_OK;
}

rtp_status rtp_indexer_project(const rtp_plan* plan, const void* q, const void* k, const float* proj,
                               float* centroids, float* qbar, void* stream) {
  CallRange range_("rtp_indexer_project");
  if (!plan) return RTP_ERR_INVALID_ARG;
  return indexer_run(plan, q, k, plan->q_end - plan->q_begin, proj, centroids, qbar, stream);
}


rtp_status rtp_block_select(const rtp_plan* plan, const float* qbar, const float* centroids, int32_t* sel,
                            int32_t* sel_cnt, void* stream) {
  CallRange range_("rtp_block_select");
  if (!plan) return RTP_ERR_INVALID_ARG;
  if (plan->n_sparse == 0) return RTP_OK;
  if (!qbar || !centroids || !sel || !sel_cnt) return RTP_ERR_INVALID_ARG;
  if (!aligned16(qbar) || !aligned16(centroids) || !aligned16(sel) || !aligned16(sel_cnt))
    return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  SelectArgs a = {};
  a.c_group = 1;
  a.qbar = qbar;
  a.centroids = centroids;
  a.sel = sel;
  a.cnt = sel_cnt;
  a.batch = c.batch;
  a.n_sparse = plan->n_sparse;
  a.nb = plan->nqb;
  a.topk = c.topk;
  a.n_local = c.n_local;
  a.kmax = c.topk + 1 + c.n_local;
  a.t0 = plan->q_begin / c.block;
  a.n_rows = plan->q_end / c.block - a.t0;
  return cuda_status(launch_select(a, reinterpret_cast<cudaStream_t>(stream)));
}

rtp_status rtp_block_select_dynamic(const rtp_plan* plan, const float* qbar, const float* centroids, float mass,
                                    int min_k, float beta, int32_t* sel, int32_t* sel_cnt, void* stream) {
  CallRange range_("rtp_block_select_dynamic");
  if (!plan) return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  if (!(mass > 0.f && mass <= 1.f) || !(beta >= 0.f) || !std::isfinite(beta)) return RTP_ERR_INVALID_ARG;
  if (min_k < 0 || min_k > c.topk) return RTP_ERR_INVALID_ARG;
  if (c.topk > kDynMaxCap) return RTP_ERR_UNSUPPORTED;
  if (plan->n_sparse == 0) return RTP_OK;
  if (!qbar || !centroids || !sel || !sel_cnt) return RTP_ERR_INVALID_ARG;
  if (!aligned16(qbar) || !aligned16(centroids) || !aligned16(sel) || !aligned16(sel_cnt))
    return RTP_ERR_INVALID_ARG;
  SelectArgs a = {};
  a.c_group = 1;
  a.qbar = qbar;
  a.centroids = centroids;
  a.sel = sel;
  a.cnt = sel_cnt;
  a.batch = c.batch;
  a.n_sparse = plan->n_sparse;
  a.nb = plan->nqb;
  a.topk = c.topk;
  a.n_local = c.n_local;
  a.kmax = c.topk + 1 + c.n_local;
  a.t0 = plan->q_begin / c.block;
  a.n_rows = plan->q_end / c.block - a.t0;
  a.mass = mass;
  a.min_k = min_k;
  a.beta_log2 = beta * kLog2e;
  return cuda_status(launch_select_dynamic(a, reinterpret_cast<cudaStream_t>(stream)));
}

rtp_status rtp_block_select_rowmax(const rtp_plan* plan, const void* q, const float* proj, const float* centroids,
                                   int32_t* sel, int32_t* sel_cnt, void* stream) {
  CallRange range_("rtp_block_select_rowmax");
  if (!plan) return RTP_ERR_INVALID_ARG;
  if (plan->n_sparse == 0) return RTP_OK;
  if (!q || !proj || !centroids || !sel || !sel_cnt) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(proj) || !aligned16(centroids) || !aligned16(sel) || !aligned16(sel_cnt))
    return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  SelectArgs a = {};
  a.c_group = 1;
  a.centroids = centroids;
  a.sel = sel;
  a.cnt = sel_cnt;
  a.batch = c.batch;
  a.n_sparse = plan->n_sparse;
  a.nb = plan->nqb;
  a.topk = c.topk;
  a.n_local = c.n_local;
  a.kmax = c.topk + 1 + c.n_local;
  a.t0 = plan->q_begin / c.block;
  a.n_rows = plan->q_end / c.block - a.t0;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.proj = proj;
  a.slot_heads = plan->d_slot_heads;
  a.n_q_heads = c.n_q_heads;
  a.n_kv_heads = c.n_kv_heads;
  a.group = c.n_q_heads / c.n_kv_heads;
  a.block = c.block;
  a.q_row0 = plan->q_begin;
  a.q_slab = plan->q_end - plan->q_begin;
  return cuda_status(launch_select_rowmax(a, reinterpret_cast<cudaStream_t>(stream)));
}

// Per-head selection: a whole-sequence plan with 128-key blocks and an even
// group (the prefill pairs the heads of a group).
static bool per_head_ok(const rtp_plan* plan) {
  const rtp_attn_cfg& c = plan->cfg;
  const int group = c.n_q_heads / c.n_kv_heads;
  return plan->q_begin == 0 && plan->q_end == c.seq && c.block == 128 && group % 2 == 0;
}

rtp_status rtp_indexer_project_heads(const rtp_plan* plan, const void* q, const float* proj, float* qbar_heads,
                                     void* stream) {
  CallRange range_("rtp_indexer_project_heads");
  if (!plan) return RTP_ERR_INVALID_ARG;
  if (!per_head_ok(plan)) return RTP_ERR_UNSUPPORTED;
  if (plan->n_sparse == 0) return RTP_OK;
  if (!q || !proj || !qbar_heads || !aligned16(q) || !aligned16(proj) || !aligned16(qbar_heads))
    return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  IndexerArgs a = {};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.proj = proj;
  a.qbar = qbar_heads;
  a.slot_heads = plan->d_slot_heads;
  a.batch = c.batch;
  a.seq = c.seq;
  a.n_q_heads = c.n_q_heads;
  a.n_kv_heads = c.n_kv_heads;
  a.group = c.n_q_heads / c.n_kv_heads;
  a.n_sparse = plan->n_sparse;
  a.block = c.block;
  a.blk0 = 0;
  a.rows = c.seq;
  a.n_blocks = c.seq / c.block;
  return cuda_status(launch_indexer_heads(a, reinterpret_cast<cudaStream_t>(stream)));
}

rtp_status rtp_block_select_heads(const rtp_plan* plan, const float* qbar_heads, const float* centroids,
                                  int32_t* sel, int32_t* sel_cnt, void* stream) {
  CallRange range_("rtp_block_select_heads");
  if (!plan) return RTP_ERR_INVALID_ARG;
  if (!per_head_ok(plan)) return RTP_ERR_UNSUPPORTED;
  if (plan->n_sparse == 0) return RTP_OK;
  if (!qbar_heads || !centroids || !sel || !sel_cnt) return RTP_ERR_INVALID_ARG;
  if (!aligned16(qbar_heads) || !aligned16(centroids) || !aligned16(sel) || !aligned16(sel_cnt))
    return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = plan->cfg;
  const int group = c.n_q_heads / c.n_kv_heads;
  SelectArgs a = {};
  a.c_group = group;  // selection row (slot, head) scores against the slot's centroids
  a.qbar = qbar_heads;
  a.centroids = centroids;
  a.sel = sel;
  a.cnt = sel_cnt;
  a.batch = c.batch;
  a.n_sparse = plan->n_sparse * group;
  a.nb = plan->nqb;
  a.topk = c.topk;
  a.n_local = c.n_local;
  a.kmax = c.topk + 1 + c.n_local;
  a.t0 = 0;
  a.n_rows = plan->nqb;
  return cuda_status(launch_select(a, reinterpret_cast<cudaStream_t>(stream)));
}

rtp_status rtp_hybrid_prefill_heads(const rtp_plan* plan, const void* q, const void* k, const void* v,
                                    const int32_t* sel, const int32_t* sel_cnt, void* o, void* stream) {
  CallRange range_("rtp_hybrid_prefill_heads");
  if (!plan) return RTP_ERR_INVALID_ARG;
  if (!per_head_ok(plan)) return RTP_ERR_UNSUPPORTED;
  return prefill_run(plan, q, plan->q_end - plan->q_begin, k, v, plan->q_end, sel, sel_cnt, o, stream, 1);
}

rtp_status rtp_hybrid_prefill(const rtp_plan* plan, const void* q, const void* k, const void* v,
                              const int32_t* sel, const int32_t* sel_cnt, void* o, void* stream) {
  CallRange range_("rtp_hybrid_prefill");
  if (!plan) return RTP_ERR_INVALID_ARG;
  return prefill_run(plan, q, plan->q_end - plan->q_begin, k, v, plan->q_end, sel, sel_cnt, o, stream);
}

rtp_status rtp_hybrid_prefill_items(const rtp_plan* plan, const void* q, const void* k, const void* v,
                                    const int32_t* sel, const int32_t* sel_cnt, void* o, long item_begin,
                                    long item_end, int max_ctas, void* stream) {
  CallRange range_("rtp_hybrid_prefill_items");
  if (!plan || item_end < 0) return RTP_ERR_INVALID_ARG;
  return prefill_run(plan, q, plan->q_end - plan->q_begin, k, v, plan->q_end, sel, sel_cnt, o, stream, 0,
                     item_begin, item_end, max_ctas);
}


// Decode workspace: sel [batch][n_kv][kmax] int32 | cnt [batch][n_kv] int32 |
// partials [spans of both lists][group][132] fp32, each 256-byte aligned.
// The spans (<= 128 keys each) form two lists ordered (sequence, head, span):
// list 0 = window and full heads plus each retrieval head's sink and local
// blocks (known before the selection), list 1 = the retrieval heads' top-k
// blocks.
namespace {
struct DecodeLayout {
  size_t sel_off, cnt_off, part_off, total;
  int kmax;
  int per_b[2];
  int span_off[2][kMaxDecodeKvHeads];
};

// Rows allocated per (sequence, KV head) in a decode-time cache: cfg->seq
// when it is at least cache_len, else exactly cache_len.
int decode_capacity(const rtp_attn_cfg* c, int cache_len) { return c->seq > cache_len ? c->seq : cache_len; }

// clu_end > 0: clustered retrieval heads (sink block + tail pieces fixed,
// topk chunks selected).
bool decode_layout(const rtp_attn_cfg* c, const uint8_t* kind, int cache_len, DecodeLayout& L, int clu_end = 0) {
  if (!cfg_common_ok(c) || !kind || cache_len < 1) return false;
  if (static_cast<long>(cache_len) / c->block * 4 > 200 * 1024) return false;
  if (c->n_kv_heads > kMaxDecodeKvHeads) return false;
  if (clu_end > 0 && (clu_end % c->block != 0 || clu_end <= c->block || clu_end > cache_len)) return false;
  const long t = (cache_len - 1) / c->block;  // block of the new token
  const long nfix = clu_end > 0 ? 1 + (cache_len - clu_end + 127) / 128  // sink + unclustered tail
                                : std::min<long>(t + 1, c->n_local + 1);   // sink + local blocks
  L.kmax = clu_end > 0 ? static_cast<int>(nfix) + c->topk : c->topk + 1 + c->n_local;
  long per_b[2] = {0, 0};
  for (int h = 0; h < c->n_kv_heads; ++h) {
    if (kind[h] > RTP_HEAD_SPARSE) return false;
    long s0 = 0, s1 = 0;
    if (kind[h] == RTP_HEAD_SPARSE) {
      s0 = nfix;
      s1 = L.kmax - nfix;
    } else if (kind[h] == RTP_HEAD_SWA) {
      s0 = (std::min(cache_len, c->window) + 127) / 128;
    } else {
      s0 = (cache_len + 127) / 128;
    }
    L.span_off[0][h] = static_cast<int>(per_b[0]);
    L.span_off[1][h] = static_cast<int>(per_b[1]);
    per_b[0] += s0;
    per_b[1] += s1;
  }
  if (per_b[0] > (1L << 30) || per_b[1] > (1L << 30)) return false;
  L.per_b[0] = static_cast<int>(per_b[0]);
  L.per_b[1] = static_cast<int>(per_b[1]);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t bk = static_cast<size_t>(c->batch) * c->n_kv_heads;
  const size_t spans = static_cast<size_t>(c->batch) * (per_b[0] + per_b[1]);
  const int group = c->n_q_heads / c->n_kv_heads;
  L.sel_off = 0;
  L.cnt_off = up(bk * L.kmax * sizeof(int32_t));
  L.part_off = L.cnt_off + up(bk * sizeof(int32_t));
  L.total = L.part_off + up(spans * group * kPartStride * sizeof(float));
  return true;
}

// SM count of the current device (looked up once per device).
int device_sms() {
  static std::mutex mu;
  static int sms[64] = {0};
  const int dev = current_device();
  if (dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    sms[dev] = n;
  }
  return sms[dev];
}

// The attention launch's schedule: one CTA per SM, no more CTAs than spans
// in the longer list.
bool decode_schedule(const rtp_attn_cfg* c, const DecodeLayout& L, DecodeArgs& a) {
  const int sms = device_sms();
  if (sms <= 0) return false;
  const long n0 = static_cast<long>(c->batch) * L.per_b[0], n1 = static_cast<long>(c->batch) * L.per_b[1];
  a.n_ctas = static_cast<int>(std::max(1L, std::min<long>(std::min(sms, 1024), std::max(n0, n1))));
  a.per_b[0] = L.per_b[0];
  a.per_b[1] = L.per_b[1];
  std::memset(a.span_off, 0, sizeof(a.span_off));
  for (int l = 0; l < 2; ++l) std::memcpy(a.span_off[l], L.span_off[l], sizeof(int) * c->n_kv_heads);
  return true;
}

// The arrays and sizes of a clustering description (cap = cache capacity).
bool cluster_args_ok(const rtp_attn_cfg* c, const uint8_t* kind, const rtp_clusters* cl, int cap) {
  if (!cfg_common_ok(c) || !kind || !cl || c->n_kv_heads > kMaxDecodeKvHeads || c->batch > 65535) return false;
  for (int h = 0; h < c->n_kv_heads; ++h)
    if (kind[h] > RTP_HEAD_SPARSE) return false;
  if (cl->clu_end <= c->block || cl->clu_end % c->block != 0 || cl->clu_end > cap) return false;
  const int n = cl->clu_end - c->block;
  if (cl->n_clusters < 1 || cl->n_clusters > kMaxClusters || cl->n_clusters > n) return false;
  if (!cl->centroids || !cl->members || !cl->offsets || !cl->chunk_centroids || !cl->chunk_start || !cl->chunk_len ||
      !cl->n_chunks)
    return false;
  // k_sorted / v_sorted: both given (cluster-ordered copy) or both NULL (in place)
  if ((cl->k_sorted == nullptr) != (cl->v_sorted == nullptr)) return false;
  return aligned16(cl->centroids) && aligned16(cl->k_sorted) && aligned16(cl->v_sorted) &&
         aligned16(cl->chunk_centroids);
}

// Argument checks and DecodeArgs of the decode entry points (cl: clustered
// mode, else contiguous blocks with `centroids`).
rtp_status prepare_decode(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* q,
                          const void* kcache, const void* vcache, const float* centroids, const float* proj,
                          const rtp_clusters* cl, void* o, int32_t* sel_out, int32_t* cnt_out, DecodeLayout& L,
                          DecodeArgs& a) {
  if (!cfg) return RTP_ERR_INVALID_ARG;
  if (!decode_layout(cfg, kind_host, cache_len, L, cl ? cl->clu_end : 0)) return RTP_ERR_INVALID_ARG;
  if (!q || !kcache || !vcache || !o) return RTP_ERR_INVALID_ARG;
  bool any_sparse = false;
  for (int h = 0; h < cfg->n_kv_heads; ++h) any_sparse |= kind_host[h] == RTP_HEAD_SPARSE;
  if (any_sparse && (!proj || (!cl && !centroids))) return RTP_ERR_INVALID_ARG;
  if (cl && !cluster_args_ok(cfg, kind_host, cl, decode_capacity(cfg, cache_len))) return RTP_ERR_INVALID_ARG;
  if ((sel_out == nullptr) != (cnt_out == nullptr)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if ((centroids && !aligned16(centroids)) || (proj && !aligned16(proj))) return RTP_ERR_INVALID_ARG;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kcache = static_cast<const __nv_bfloat16*>(kcache);
  a.vcache = static_cast<const __nv_bfloat16*>(vcache);
  a.centroids = centroids;
  a.proj = proj;
  a.o = static_cast<__nv_bfloat16*>(o);
  std::memset(a.kind, 0, sizeof(a.kind));
  std::memcpy(a.kind, kind_host, cfg->n_kv_heads);
  a.batch = cfg->batch;
  a.n_q_heads = cfg->n_q_heads;
  a.n_kv_heads = cfg->n_kv_heads;
  a.group = cfg->n_q_heads / cfg->n_kv_heads;
  a.cache_len = cache_len;
  a.cache_cap = decode_capacity(cfg, cache_len);
  a.nbc = a.cache_cap / cfg->block;
  a.window = cfg->window;
  a.block = cfg->block;
  a.topk = cfg->topk;
  a.n_local = cfg->n_local;
  a.kmax = L.kmax;
  a.scale_log2 = effective_scale(cfg) * kLog2e;
  a.clustered = cl ? 1 : 0;
  a.clu_end = cl ? cl->clu_end : 0;
  a.clu_rows = cl ? cl->clu_end - cfg->block : 0;
  a.max_chunks = cl ? a.clu_rows / 128 + cl->n_clusters : 0;
  a.k_sorted = cl ? static_cast<const __nv_bfloat16*>(cl->k_sorted) : nullptr;
  a.v_sorted = cl ? static_cast<const __nv_bfloat16*>(cl->v_sorted) : nullptr;
  a.members = cl ? cl->members : nullptr;
  a.gather = cl && !cl->k_sorted ? 1 : 0;
  a.chunk_centroids = cl ? cl->chunk_centroids : nullptr;
  a.chunk_start = cl ? cl->chunk_start : nullptr;
  a.chunk_len = cl ? cl->chunk_len : nullptr;
  a.n_chunks = cl ? cl->n_chunks : nullptr;
  if (!decode_schedule(cfg, L, a)) return RTP_ERR_CUDA;
  return RTP_OK;
}

// Scratch pointers, status word, TMA maps and the launch.
// `status`: the device word the kernels report in; NULL = the library's
// allocated status word of the current device.
rtp_status run_decode(DecodeArgs& a, const DecodeLayout& L, char* ws, int32_t* sel_out, int32_t* cnt_out,
                      uint32_t* status, const rtp_clusters* cl, void* stream) {
  a.sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(ws + L.sel_off);
  a.cnt = cnt_out ? cnt_out : reinterpret_cast<int32_t*>(ws + L.cnt_off);
  a.partial = reinterpret_cast<float*>(ws + L.part_off);
  a.status = status ? status : status_word(current_device());
  if (!a.status) return RTP_ERR_NO_MEMORY;
  const long slabs = static_cast<long>(a.batch) * a.n_kv_heads;
  CUtensorMap mk, mv, mks, mvs;
  if (!encode_bf16_3d(&mk, a.kcache, a.cache_len, slabs, 64, a.cache_cap) ||
      !encode_bf16_3d(&mv, a.vcache, a.cache_len, slabs, 64, a.cache_cap))
    return RTP_ERR_CUDA;
  if (cl && a.gather) {
    mks = mk;  // unused: gathered spans are copied with cp.async
    mvs = mv;
  } else if (cl) {
    if (!encode_bf16_3d(&mks, cl->k_sorted, a.clu_rows, slabs, 64) ||
        !encode_bf16_3d(&mvs, cl->v_sorted, a.clu_rows, slabs, 64))
      return RTP_ERR_CUDA;
  } else {
    mks = mk;
    mvs = mv;
  }
  return cuda_status(launch_decode(a, mk, mv, mks, mvs, reinterpret_cast<cudaStream_t>(stream)));
}

// Shared validation of the KV-cache maintenance calls; fills the common
// fields of CacheArgs.
rtp_status cache_args(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cap, const void* kcache,
                      const float* proj, float* centroids, CacheArgs& a) {
  if (!cfg_common_ok(cfg) || !kind_host || !kcache) return RTP_ERR_INVALID_ARG;
  if (cfg->n_kv_heads > kMaxDecodeKvHeads || cfg->batch > 65535 || cap < 1) return RTP_ERR_INVALID_ARG;
  bool any_sparse = false;
  for (int h = 0; h < cfg->n_kv_heads; ++h) {
    if (kind_host[h] > RTP_HEAD_SPARSE) return RTP_ERR_INVALID_ARG;
    any_sparse |= kind_host[h] == RTP_HEAD_SPARSE;
  }
  if (any_sparse && (!centroids || !proj)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(kcache) || (centroids && !aligned16(centroids)) || (proj && !aligned16(proj)))
    return RTP_ERR_INVALID_ARG;
  std::memset(a.kind, 0, sizeof(a.kind));
  std::memcpy(a.kind, kind_host, cfg->n_kv_heads);
  a.kcache = static_cast<__nv_bfloat16*>(const_cast<void*>(kcache));
  a.proj = proj;
  a.centroids = centroids;
  a.batch = cfg->batch;
  a.n_kv_heads = cfg->n_kv_heads;
  a.cache_cap = cap;
  a.block = cfg->block;
  a.k_new = a.v_new = nullptr;
  a.vcache = nullptr;
  a.pos = 0;
  a.n_blocks = 0;
  return RTP_OK;
}
}  // namespace

size_t rtp_decode_workspace_bytes(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len) {
  DecodeLayout L;
  if (!decode_layout(cfg, kind_host, cache_len, L)) return 0;
  return L.total;
}

size_t rtp_decode_clustered_workspace_bytes(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len,
                                            int clu_end) {
  DecodeLayout L;
  if (clu_end <= 0 || !decode_layout(cfg, kind_host, cache_len, L, clu_end)) return 0;
  return L.total;
}

rtp_status rtp_sparse_decode(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* q,
                             const void* kcache, const void* vcache, const float* centroids, const float* proj,
                             void* o, void* workspace, size_t ws_bytes, int32_t* sel_out, int32_t* cnt_out,
                             void* stream) {
  CallRange range_("rtp_sparse_decode");
  DecodeLayout L;
  DecodeArgs a;
  rtp_status st = prepare_decode(cfg, kind_host, cache_len, q, kcache, vcache, centroids, proj, nullptr, o, sel_out,
                                 cnt_out, L, a);
  if (st != RTP_OK) return st;
  if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return RTP_ERR_INVALID_ARG;
  return run_decode(a, L, static_cast<char*>(workspace), sel_out, cnt_out, nullptr, nullptr, stream);
}

rtp_status rtp_sparse_decode_clustered(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len,
                                       const void* q, const void* kcache, const void* vcache, const float* proj,
                                       const rtp_clusters* cl, void* o, void* workspace, size_t ws_bytes,
                                       int32_t* sel_out, int32_t* cnt_out, void* stream) {
  CallRange range_("rtp_sparse_decode_clustered");
  if (!cl) return RTP_ERR_INVALID_ARG;
  DecodeLayout L;
  DecodeArgs a;
  rtp_status st =
      prepare_decode(cfg, kind_host, cache_len, q, kcache, vcache, nullptr, proj, cl, o, sel_out, cnt_out, L, a);
  if (st != RTP_OK) return st;
  if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return RTP_ERR_INVALID_ARG;
  return run_decode(a, L, static_cast<char*>(workspace), sel_out, cnt_out, nullptr, cl, stream);
}

rtp_status rtp_sparse_decode_noalloc(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* q,
                                     const void* kcache, const void* vcache, const float* centroids,
                                     const float* proj, void* o, int32_t* sel_out, int32_t* cnt_out, void* stream) {
  CallRange range_("rtp_sparse_decode_noalloc");
  DecodeLayout L;
  DecodeArgs a;
  rtp_status st = prepare_decode(cfg, kind_host, cache_len, q, kcache, vcache, centroids, proj, nullptr, o, sel_out,
                                 cnt_out, L, a);
  if (st != RTP_OK) return st;
  if (L.total > kDecodeStaticScratchBytes) return RTP_ERR_INVALID_ARG;  // beyond the fixed scratch
  void* scratch = nullptr;
  uint32_t* status = nullptr;
  if (decode_static_scratch(&scratch, &status) != cudaSuccess || !scratch || !status) return RTP_ERR_CUDA;
  // the kernels report in the static status word, not the allocated one
  return run_decode(a, L, static_cast<char*>(scratch), sel_out, cnt_out, status, nullptr, stream);
}

size_t rtp_cache_cluster_workspace_bytes(const rtp_attn_cfg* cfg, int clu_end) {
  if (!cfg_common_ok(cfg) || clu_end <= cfg->block) return 0;
  const size_t bk = static_cast<size_t>(cfg->batch) * cfg->n_kv_heads;
  const size_t n = static_cast<size_t>(clu_end - cfg->block);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t n_seg = (n + kKmSegKeys - 1) / kKmSegKeys;
  return up(bk * n * kRank * sizeof(float)) + 2 * up(bk * n * sizeof(int32_t)) + up(bk * sizeof(int32_t)) +
         up(bk * n_seg * kMaxClusters * sizeof(int32_t));
}

rtp_status rtp_cache_cluster(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int iters, const void* kcache,
                             const void* vcache, const float* proj, const rtp_clusters* cl, void* workspace,
                             size_t ws_bytes, void* stream) {
  CallRange range_("rtp_cache_cluster");
  if (!cfg || !cl || iters < 1 || iters > 1000) return RTP_ERR_INVALID_ARG;
  if (!cluster_args_ok(cfg, kind_host, cl, decode_capacity(cfg, cl->clu_end))) return RTP_ERR_INVALID_ARG;
  if (!kcache || !vcache || !proj || !aligned16(kcache) || !aligned16(vcache) || !aligned16(proj))
    return RTP_ERR_INVALID_ARG;
  const size_t need = rtp_cache_cluster_workspace_bytes(cfg, cl->clu_end);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return RTP_ERR_INVALID_ARG;
  KmeansArgs a;
  std::memset(a.kind, 0, sizeof(a.kind));
  std::memcpy(a.kind, kind_host, cfg->n_kv_heads);
  a.kcache = static_cast<const __nv_bfloat16*>(kcache);
  a.vcache = static_cast<const __nv_bfloat16*>(vcache);
  a.proj = proj;
  a.batch = cfg->batch;
  a.n_kv_heads = cfg->n_kv_heads;
  a.cache_cap = decode_capacity(cfg, cl->clu_end);
  a.block = cfg->block;
  a.clu_end = cl->clu_end;
  a.n = cl->clu_end - cfg->block;
  a.nc = cl->n_clusters;
  a.max_chunks = a.n / 128 + a.nc;
  const size_t bk = static_cast<size_t>(cfg->batch) * cfg->n_kv_heads;
  a.X = static_cast<float*>(workspace);
  {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    char* w = static_cast<char*>(workspace) + up(bk * a.n * kRank * sizeof(float));
    a.assign = reinterpret_cast<int32_t*>(w);
    w += up(bk * a.n * sizeof(int32_t));
    a.amb_list = reinterpret_cast<int32_t*>(w);
    w += up(bk * a.n * sizeof(int32_t));
    a.amb_count = reinterpret_cast<int32_t*>(w);
    w += up(bk * sizeof(int32_t));
    a.seg = reinterpret_cast<int32_t*>(w);
    a.n_seg = (a.n + kKmSegKeys - 1) / kKmSegKeys;
  }
  a.centroids = cl->centroids;
  a.members = cl->members;
  a.offsets = cl->offsets;
  a.k_sorted = static_cast<__nv_bfloat16*>(cl->k_sorted);
  a.v_sorted = static_cast<__nv_bfloat16*>(cl->v_sorted);
  a.chunk_centroids = cl->chunk_centroids;
  a.chunk_start = cl->chunk_start;
  a.chunk_len = cl->chunk_len;
  a.n_chunks = cl->n_chunks;
  return cuda_status(launch_kmeans(a, iters, reinterpret_cast<cudaStream_t>(stream)));
}

rtp_status rtp_cache_centroids(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* kcache,
                               const float* proj, float* centroids, void* stream) {
  CallRange range_("rtp_cache_centroids");
  if (!cfg || cache_len < 1) return RTP_ERR_INVALID_ARG;
  CacheArgs a;
  const rtp_status st = cache_args(cfg, kind_host, decode_capacity(cfg, cache_len), kcache, proj, centroids, a);
  if (st != RTP_OK) return st;
  a.n_blocks = cache_len / cfg->block;
  return cuda_status(launch_cache_centroids(a, reinterpret_cast<cudaStream_t>(stream)));
}

rtp_status rtp_cache_append(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int pos, const void* k_new,
                            const void* v_new, void* kcache, void* vcache, const float* proj, float* centroids,
                            void* stream) {
  CallRange range_("rtp_cache_append");
  if (!cfg || pos < 0 || pos >= cfg->seq) return RTP_ERR_INVALID_ARG;
  CacheArgs a;
  const rtp_status st = cache_args(cfg, kind_host, cfg->seq, kcache, proj, centroids, a);
  if (st != RTP_OK) return st;
  if (!k_new || !v_new || !vcache || !aligned16(k_new) || !aligned16(v_new) || !aligned16(vcache))
    return RTP_ERR_INVALID_ARG;
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.vcache = static_cast<__nv_bfloat16*>(vcache);
  a.pos = pos;
  return cuda_status(launch_cache_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------- host pipeline
rtp_status rtp_pipeline_create(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int n_chunks, void* stream,
                               rtp_pipeline** out) {
  CallRange range_("rtp_pipeline_create");
  if (!out) return RTP_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg_prefill_ok(cfg) || !kind_host || n_chunks < 1 || n_chunks > 1024) return RTP_ERR_INVALID_ARG;
  const int tiles = (cfg->seq + 127) / 128;
  if (tiles < n_chunks) return RTP_ERR_INVALID_ARG;
  rtp_pipeline* pl = new (std::nothrow) rtp_pipeline();
  if (!pl) return RTP_ERR_NO_MEMORY;
  pl->cfg = *cfg;
  pl->device = current_device();
  auto fail = [&](rtp_status st) {
    rtp_pipeline_destroy(pl);
    return st;
  };
  // Chunk boundaries in tiles: equal chunks, except that with four or more
  // the last two are a half and a quarter of the others (what follows the
  // last upload -- that chunk's kernels and its download -- is the part of
  // the pipeline nothing overlaps); every chunk keeps at least one tile.
  std::vector<int> tb(n_chunks + 1, 0);
  {
    std::vector<double> w(n_chunks, 1.0);
    if (n_chunks >= 4) {
      w[n_chunks - 2] = 0.5;
      w[n_chunks - 1] = 0.25;
    }
    double total = 0.0, run = 0.0;
    for (double x : w) total += x;
    tb[n_chunks] = tiles;
    for (int c = 1; c < n_chunks; ++c) {
      run += w[c - 1];
      const int t = static_cast<int>(std::llround(run / total * tiles));
      tb[c] = std::min(std::max(t, tb[c - 1] + 1), tiles - (n_chunks - c));
    }
  }
  for (int c = 0; c < n_chunks; ++c) {
    const int b = 128 * tb[c];
    const int e = std::min(cfg->seq, 128 * tb[c + 1]);
    rtp_plan* p = nullptr;
    const rtp_status st = rtp_route_heads_range(cfg, kind_host, b, e, stream, &p);
    if (st != RTP_OK) return fail(st);
    pl->plans.push_back(p);
    pl->begin.push_back(b);
    pl->end.push_back(e);
  }
  pl->n_sparse = pl->plans[0]->n_sparse;
  if (cudaStreamCreateWithFlags(&pl->s_in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&pl->s_out, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&pl->ev_start, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&pl->ev_done, cudaEventDisableTiming) != cudaSuccess)
    return fail(RTP_ERR_CUDA);
  pl->ev_in.assign(n_chunks, nullptr);
  pl->ev_out.assign(n_chunks, nullptr);
  for (int c = 0; c < n_chunks; ++c)
    if (cudaEventCreateWithFlags(&pl->ev_in[c], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&pl->ev_out[c], cudaEventDisableTiming) != cudaSuccess)
      return fail(RTP_ERR_CUDA);
  *out = pl;
  return RTP_OK;
}

void rtp_pipeline_destroy(rtp_pipeline* pl) {
  if (!pl) return;
  for (rtp_plan* p : pl->plans) rtp_plan_destroy(p);
  for (cudaEvent_t e : pl->ev_in)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : pl->ev_out)
    if (e) cudaEventDestroy(e);
  if (pl->ev_start) cudaEventDestroy(pl->ev_start);
  if (pl->ev_done) cudaEventDestroy(pl->ev_done);
  if (pl->s_in) cudaStreamDestroy(pl->s_in);
  if (pl->s_out) cudaStreamDestroy(pl->s_out);
  delete pl;
}

rtp_status rtp_hybrid_prefill_host(rtp_pipeline* pl, const void* q_host, const void* k_host, const void* v_host,
                                   const float* proj, void* o_host, void* q_dev, void* k_dev, void* v_dev,
                                   void* o_dev, float* centroids, float* qbar, int32_t* sel, int32_t* sel_cnt,
                                   void* stream) {
  CallRange range_("rtp_hybrid_prefill_host");
  if (!pl || !q_host || !k_host || !v_host || !o_host || !q_dev || !k_dev || !v_dev || !o_dev)
    return RTP_ERR_INVALID_ARG;
  if (pl->n_sparse > 0 && (!proj || !centroids || !qbar || !sel || !sel_cnt)) return RTP_ERR_INVALID_ARG;
  if (current_device() != pl->device) return RTP_ERR_INVALID_ARG;
  const rtp_attn_cfg& c = pl->cfg;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t row = kHeadDim * sizeof(__nv_bfloat16);
  const size_t pitch = static_cast<size_t>(c.seq) * row;
  const size_t q_slabs = static_cast<size_t>(c.batch) * c.n_q_heads, kv_slabs = static_cast<size_t>(c.batch) * c.n_kv_heads;
  auto at = [&](const void* base, int r) { return static_cast<const char*>(base) + static_cast<size_t>(r) * row; };
  auto atw = [&](void* base, int r) { return static_cast<char*>(base) + static_cast<size_t>(r) * row; };
  // The copy streams start after the work already queued on `stream`.
  if (cudaEventRecord(pl->ev_start, s) != cudaSuccess || cudaStreamWaitEvent(pl->s_in, pl->ev_start) != cudaSuccess ||
      cudaStreamWaitEvent(pl->s_out, pl->ev_start) != cudaSuccess)
    return RTP_ERR_CUDA;
  for (size_t ci = 0; ci < pl->plans.size(); ++ci) {
    const rtp_plan* p = pl->plans[ci];
    const int b = pl->begin[ci], e = pl->end[ci];
    const size_t width = static_cast<size_t>(e - b) * row;
    // 1. this chunk's Q, K and V rows (every slab) to the device
    if (cudaMemcpy2DAsync(atw(q_dev, b), pitch, at(q_host, b), pitch, width, q_slabs, cudaMemcpyHostToDevice,
                          pl->s_in) != cudaSuccess ||
        cudaMemcpy2DAsync(atw(k_dev, b), pitch, at(k_host, b), pitch, width, kv_slabs, cudaMemcpyHostToDevice,
                          pl->s_in) != cudaSuccess ||
        cudaMemcpy2DAsync(atw(v_dev, b), pitch, at(v_host, b), pitch, width, kv_slabs, cudaMemcpyHostToDevice,
                          pl->s_in) != cudaSuccess ||
        cudaEventRecord(pl->ev_in[ci], pl->s_in) != cudaSuccess || cudaStreamWaitEvent(s, pl->ev_in[ci]) != cudaSuccess)
      return RTP_ERR_CUDA;
    // 2. its kernels: every earlier row is already on the device
    rtp_status st = RTP_OK;
    if (pl->n_sparse > 0) {
      st = indexer_run(p, atw(q_dev, b), atw(k_dev, b), c.seq, proj, centroids, qbar, stream);
      if (st == RTP_OK) st = rtp_block_select(p, qbar, centroids, sel, sel_cnt, stream);
    }
    if (st == RTP_OK) st = prefill_run(p, atw(q_dev, b), c.seq, k_dev, v_dev, c.seq, sel, sel_cnt, atw(o_dev, b), stream);
    if (st != RTP_OK) return st;
    // 3. its O rows back to the host
    if (cudaEventRecord(pl->ev_out[ci], s) != cudaSuccess || cudaStreamWaitEvent(pl->s_out, pl->ev_out[ci]) != cudaSuccess ||
        cudaMemcpy2DAsync(atw(o_host, b), pitch, at(o_dev, b), pitch, width, q_slabs, cudaMemcpyDeviceToHost,
                          pl->s_out) != cudaSuccess)
      return RTP_ERR_CUDA;
  }
  // `stream` completes when the last download does
  if (cudaEventRecord(pl->ev_done, pl->s_out) != cudaSuccess || cudaStreamWaitEvent(s, pl->ev_done) != cudaSuccess)
    return RTP_ERR_CUDA;
  return RTP_OK;
}

rtp_status rtp_selftest_bounded_wait(unsigned limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 10000) return RTP_ERR_INVALID_ARG;
  uint32_t* st = status_word(current_device());
  if (!st) return RTP_ERR_NO_MEMORY;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(st, static_cast<uint64_t>(limit_ms) * 1000000ull);
  if (cudaGetLastError() != cudaSuccess) return RTP_ERR_CUDA;
  return rtp_last_device_status(stream);
}

rtp_status rtp_last_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return RTP_ERR_CUDA;
  // Read (and clear) the words that exist on this device: the allocated one
  // once any entry point has created it, the static one of the
  // allocation-free decode once that has run.  Reading creates neither.
  uint32_t* words[2] = {existing_status_word(current_device()), decode_static_status_if_used()};
  uint32_t v = 0;
  for (uint32_t* w : words) {
    if (!w) continue;
    uint32_t x = 0;
    if (cudaMemcpy(&x, w, sizeof(x), cudaMemcpyDeviceToHost) != cudaSuccess) return RTP_ERR_CUDA;
    if (x != 0 && cudaMemset(w, 0, sizeof(uint32_t)) != cudaSuccess) return RTP_ERR_CUDA;
    v |= x;
  }
  if (v & RTP_DEVERR_TIMEOUT) return RTP_ERR_TIMEOUT;
  if (v) return RTP_ERR_INVALID_ARG;
  return RTP_OK;
}

}  // extern "C"
