// The C ABI of libmisa: argument checks, workspace planning, launches.
// Everything that computes runs in the kernels of pool.cu, route.cu,
// score.cu and topk.cu; this file only validates and sequences them.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <set>
#include <utility>
#include <vector>
#include <map>
#include <cstring>
#include <string>

#include "common.cuh"
#include "internal.h"

__device__ uint32_t g_misa_status;  // per-device status word (MISA_STATUS_* bits)

namespace misa {

namespace {
thread_local std::string g_last_error;
std::mutex g_mu;
uint32_t* g_status_ptr[64] = {nullptr};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::map<std::pair<const void*, int>, int> g_smem_set;  // (kernel, device) -> bytes set

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
// Default cap on the score buffer when sizing a workspace (queries are processed in chunks).
constexpr size_t kScoreBufferCap = size_t(2) << 30;
}  // namespace

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

int cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MISA_OK;
  set_error("%s: %s", what, cudaGetErrorString(e));
  return MISA_ERR_CUDA;
}

uint32_t* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_misa_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_status_ptr[dev];
}

int set_smem_limit(const void* kernel, int bytes) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_smem_set.find({kernel, dev});
  if (it != g_smem_set.end() && it->second >= bytes) return MISA_OK;
  // Only ever raise the limit: a lower value would reject later, larger launches.
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  g_smem_set[{kernel, dev}] = bytes;
  return MISA_OK;
}

int make_kmajor_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
        set_error("cuTensorMapEncodeTiled entry point unavailable");
        return MISA_ERR_CUDA;
      }
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  if (rows <= 0) rows = 1;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD * 2)};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d) rows=%lld box=%d", (int)r, (long long)rows,
              box_rows);
    return MISA_ERR_CUDA;
  }
  return MISA_OK;
}

namespace {
struct ProfRecord {
  const char* name;
  cudaEvent_t start, stop;
  int kernels;  // kernels launched inside the scope
};
thread_local bool t_prof_on = false;
thread_local std::vector<ProfRecord> t_prof;       // recorded, not yet collected
thread_local std::vector<cudaEvent_t> t_free_events;
// Device counters copied back while tracing (pinned host slot, event after the copy).
struct CountRecord {
  const char* name;
  int32_t* slot;
  cudaEvent_t done;
};
thread_local std::vector<CountRecord> t_counts;
thread_local std::vector<int32_t*> t_free_slots;

cudaEvent_t take_event() {
  if (!t_free_events.empty()) {
    cudaEvent_t e = t_free_events.back();
    t_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

int num_sms() {
  int dev = 0, n = kSms;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : kSms;
}

ProfScope::ProfScope(const char* name, cudaStream_t s) : slot(-1), st(s) {
  if (!t_prof_on) return;
  ProfRecord r{name, take_event(), take_event(), 1};
  if (!r.start || !r.stop) return;
  cudaEventRecord(r.start, st);
  t_prof.push_back(r);
  slot = (int)t_prof.size() - 1;
}

ProfScope::~ProfScope() {
  if (slot >= 0) cudaEventRecord(t_prof[slot].stop, st);
}

// A scope that launches more than one kernel adds the others to its record
// (the innermost open scope is the last one recorded).
void prof_add_kernels(int n) {
  if (t_prof_on && !t_prof.empty()) t_prof.back().kernels += n;
}

void prof_count(const char* name, const int* dev_count, cudaStream_t st) {
  if (!t_prof_on) return;
  int32_t* slot = nullptr;
  if (!t_free_slots.empty()) {
    slot = t_free_slots.back();
    t_free_slots.pop_back();
  } else if (cudaHostAlloc(reinterpret_cast<void**>(&slot), sizeof(int32_t),
                           cudaHostAllocDefault) != cudaSuccess) {
    return;
  }
  cudaEvent_t done = take_event();
  if (!done || cudaMemcpyAsync(slot, dev_count, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
                   cudaSuccess) {
    t_free_slots.push_back(slot);
    if (done) t_free_events.push_back(done);
    return;
  }
  cudaEventRecord(done, st);
  t_counts.push_back({name, slot, done});
}

// Argument checks, also used by the block-pruning entry point (blocks.cu).
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_problem(const misa_problem_t* p) {
  if (!p) { set_error("problem is NULL"); return MISA_ERR_INVALID_ARG; }
  if (p->head_dim != kD) {
    set_error("head_dim %d unsupported (must be 128)", p->head_dim);
    return MISA_ERR_UNSUPPORTED;
  }
  if (p->num_seqs < 1 || p->num_queries < 0 || p->num_heads < 1 || p->num_heads > 64 ||
      p->block < 1 || p->block > 4096 || p->max_seq_len < 1 || p->total_keys < 0 ||
      p->total_blocks < 0) {
    set_error("invalid problem sizes (S=%d T=%d H=%d B=%d max_len=%d)", p->num_seqs,
              p->num_queries, p->num_heads, p->block, p->max_seq_len);
    return MISA_ERR_INVALID_ARG;
  }
  if (p->total_keys >= (int64_t(1) << 31) || (int64_t)p->num_queries * 64 >= (int64_t(1) << 31)) {
    set_error("problem too large for 32-bit tensor coordinates");
    return MISA_ERR_UNSUPPORTED;
  }
  if (!p->key_offsets || !p->block_offsets || !p->query_offsets ||
      (p->num_queries > 0 && !p->q_pos)) {
    set_error("problem metadata pointer is NULL");
    return MISA_ERR_INVALID_ARG;
  }
  return MISA_OK;
}

int check_ptr(const void* ptr, size_t align, const char* name) {
  if (!ptr) { set_error("%s is NULL", name); return MISA_ERR_INVALID_ARG; }
  if (!aligned(ptr, align)) {
    set_error("%s is not %zu-byte aligned", name, align);
    return MISA_ERR_INVALID_ARG;
  }
  return MISA_OK;
}

bool pow2_le64(int x) { return x >= 1 && x <= 64 && (x & (x - 1)) == 0; }

namespace {

int64_t row_ld(const misa_problem_t* p) { return ((int64_t)p->max_seq_len + 3) / 4 * 4; }

// Group table: int4 [nq + S], the count word (16 bytes), first group of each
// sequence int [S].
size_t groups_bytes(int nq, int S) {
  return align_up(sizeof(int4) * (size_t)(nq + S) + 16 + sizeof(int) * (size_t)S);
}

// Failure counter (16 bytes) and list (one int per query), 256-byte aligned.
size_t fail_bytes(int nq) { return align_up(16 + sizeof(int32_t) * (size_t)nq); }

struct Carve {
  int4* groups;
  int* count;
  float* buf;
};

Carve carve(void* ws, int nq, int S) {
  Carve c;
  uint8_t* b = static_cast<uint8_t*>(ws);
  c.groups = reinterpret_cast<int4*>(b);
  c.count = reinterpret_cast<int*>(b + sizeof(int4) * (size_t)(nq + S));
  c.buf = reinterpret_cast<float*>(b + groups_bytes(nq, S));
  return c;
}

// Queries per chunk so that the group table and a [chunk, ld] fp32 score
// buffer fit in ws_bytes.
int chunk_queries(const misa_problem_t* p, int64_t ld, size_t ws_bytes) {
  const int T = p->num_queries;
  for (int c = T; c >= 1;) {
    const size_t need = groups_bytes(c, p->num_seqs) + align_up((size_t)c * ld * 4);
    if (need <= ws_bytes) return c;
    const size_t per = (size_t)ld * 4 + sizeof(int4);
    int guess = (int)(ws_bytes > groups_bytes(0, p->num_seqs) + 4096
                          ? (ws_bytes - groups_bytes(0, p->num_seqs) - 4096) / per
                          : 0);
    c = guess < c ? guess : c - 1;
  }
  return 0;
}

// Tensor-core router: power-of-two H with enough query groups to fill the GPU.
bool route_tc_applies(const misa_problem_t* p) {
  const int H = p->num_heads;
  if (H != 8 && H != 16 && H != 32 && H != 64) return false;
  return p->num_queries / route_tc_group_size(H) >= num_sms();
}

// CUDA-core router: group table, then the partial sums of split block ranges.
int route_max_groups(const misa_problem_t* p) {
  const int G = route_group_size(p->num_heads);
  return (p->num_queries + G - 1) / G + p->num_seqs;
}

size_t route_bytes(const misa_problem_t* p) {
  const int mg = route_max_groups(p);
  return groups_bytes(p->num_queries, p->num_seqs) +
         align_up(route_split_bytes(mg, route_split_count(*p, mg, num_sms())));
}

size_t route_tc_bytes(const misa_problem_t* p) {
  return groups_bytes(p->num_queries, p->num_seqs) + align_up(route_tc_split_bytes(*p));
}

// Streaming (fused top-k) scorer: used when every query scores its whole
// prefix in groups that fill the GPU, no score rows are requested, and m fits.
struct StreamPlan {
  bool use = false;
  int G = 0, grid = 0, max_groups = 0;
  int64_t cap = 0;
  size_t bytes = 0;           // selection inside the scoring kernel
  size_t bytes_deferred = 0;  // plus lists per query, selected by a second launch
};

StreamPlan stream_plan(const misa_problem_t* p, int m, int k, bool want_rows) {
  StreamPlan sp;
  if (want_rows || (m != 8 && m != 16 && m != 32 && m != 64) || k > 16384) return sp;
  sp.G = stream_group_size(m);
  const int T = p->num_queries;
  sp.max_groups = (T + sp.G - 1) / sp.G + p->num_seqs;
  const int sms = num_sms();
  if ((T / sp.G) < 2 * sms) return sp;  // too few groups: split the keys instead
  sp.grid = sms < sp.max_groups ? sms : sp.max_groups;
  sp.cap = stream_subcap(p->max_seq_len);
  sp.bytes = groups_bytes(T, p->num_seqs) + fail_bytes(T) +
             align_up(stream_cand_bytes(sp.grid, sp.cap, m));
  sp.bytes_deferred = sp.bytes + align_up(stream_deferred_bytes(T, sp.cap, k));
  sp.use = true;
  return sp;
}

int score_topk_impl(const misa_problem_t* p, const uint16_t* qsel, const float* wsel, int m,
                    const uint16_t* K, int k, int32_t* idx, float* val, float* scores_dbg,
                    int64_t scores_ld, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int T = p->num_queries;
  if (T == 0) return MISA_OK;
  const StreamPlan sp = stream_plan(p, m, k, scores_dbg != nullptr);
  if (sp.use && ws_bytes >= sp.bytes) {
    Carve c = carve(ws, T, p->num_seqs);
    int rc = launch_plan_groups(*p, 0, T, sp.G, c.groups, c.count, st);
    if (rc) return rc;
    StreamArgs a;
    a.p = p; a.qsel = qsel; a.wsel = wsel; a.m = m; a.K = K; a.groups = c.groups;
    a.group_count = c.count; a.max_groups = sp.max_groups; a.grid = sp.grid; a.k = k;
    // workspace: group table | failure counter + list | candidate buffers
    uint8_t* fb = reinterpret_cast<uint8_t*>(c.buf);
    a.fail_count = reinterpret_cast<int*>(fb);
    a.fail_list = reinterpret_cast<int32_t*>(fb + 16);
    a.cand = reinterpret_cast<uint2*>(fb + fail_bytes(T));
    a.subcap = sp.cap; a.idx = idx; a.val = val;
    if (ws_bytes >= sp.bytes_deferred) {
      // lists per query after the in-kernel buffers: [T][drows][128], counts, anchors
      uint8_t* db = reinterpret_cast<uint8_t*>(a.cand) + align_up(stream_cand_bytes(sp.grid, sp.cap, m));
      a.drows = stream_deferred_rows(k, sp.cap);
      a.dcand = reinterpret_cast<uint2*>(db);
      const size_t lists = align_up((size_t)T * a.drows * 128 * sizeof(uint2));
      a.dcnt = reinterpret_cast<int*>(db + lists);
      a.danchor = reinterpret_cast<int2*>(db + lists + align_up((size_t)T * 128 * sizeof(int)));
    }
    return launch_score_stream(a, st);
  }
  const int64_t ld = scores_dbg ? scores_ld : row_ld(p);
  int chunk = T;
  if (!scores_dbg) {
    chunk = chunk_queries(p, ld, ws_bytes);
    if (chunk < 1) {
      set_error("workspace of %zu bytes too small for one query row", ws_bytes);
      return MISA_ERR_WORKSPACE_TOO_SMALL;
    }
  } else if (ws_bytes < groups_bytes(T, p->num_seqs)) {
    set_error("workspace too small for the group table");
    return MISA_ERR_WORKSPACE_TOO_SMALL;
  }
  const int G = score_group_size(m);
  const int max_tiles = (p->max_seq_len + kTileKeys - 1) / kTileKeys;
  for (int q_lo = 0; q_lo < T; q_lo += chunk) {
    const int q_hi = q_lo + chunk < T ? q_lo + chunk : T;
    Carve c = carve(ws, q_hi - q_lo, p->num_seqs);
    float* I = scores_dbg ? scores_dbg + (int64_t)q_lo * scores_ld : c.buf;
    int rc = launch_plan_groups(*p, q_lo, q_hi, G, c.groups, c.count, st);
    if (rc) return rc;
    ScoreArgs a;
    a.p = p; a.qsel = qsel; a.wsel = wsel; a.m = m; a.K = K; a.cand = nullptr; a.k_cand = 0;
    a.groups = c.groups; a.group_count = c.count;
    a.max_groups = (q_hi - q_lo + G - 1) / G + p->num_seqs;
    a.G = G; a.q_lo = q_lo; a.I = I; a.ld = ld; a.max_tiles = max_tiles;
    rc = launch_score(a, st);
    if (rc) return rc;
    rc = launch_topk(*p, I, ld, nullptr, 0, q_lo, q_hi, k, idx, val, st);
    if (rc) return rc;
  }
  return MISA_OK;
}

__global__ void selftest_timeout_kernel(long long wait_ns, uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_barrier_init();
  // Nothing ever arrives on `bar`: the wait must run out and report.
  long long t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (!mbar_try_wait(&bar, 0)) {
    long long now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    if (now - t0 > wait_ns) {
      set_status(status, MISA_STATUS_TIMEOUT);
      break;
    }
  }
}

}  // namespace
// Workspace that misa_route uses for this problem on its fastest path (the
// tensor-core router where it applies, else the CUDA-core router with its
// pooled-block ranges).  The problem must have passed check_problem.
size_t route_path_bytes(const misa_problem_t* p) {
  return route_tc_applies(p) ? route_tc_bytes(p) : route_bytes(p);
}

// Whether tracing is on for the calling host thread.
bool tracing_enabled() { return t_prof_on; }

}  // namespace misa

using namespace misa;

extern "C" {

const char* misa_last_error_string(void) { return g_last_error.c_str(); }

size_t misa_workspace_size(const misa_problem_t* p, int32_t m, int32_t k, int32_t k_cand) {
  if (check_problem(p)) return 0;
  if (m < 1 || m > p->num_heads || k < 1 || k_cand < 0) {
    set_error("invalid m/k/k_cand");
    return 0;
  }
  const int T = p->num_queries, S = p->num_seqs;
  const int64_t ld = row_ld(p);
  size_t need = route_bytes(p);  // router
  if (route_tc_applies(p) && route_tc_bytes(p) > need) need = route_tc_bytes(p);
  // score / dense: chunk so the score buffer stays near kScoreBufferCap
  int64_t chunk = T;
  if ((size_t)chunk * ld * 4 > kScoreBufferCap) chunk = (int64_t)(kScoreBufferCap / ((size_t)ld * 4));
  if (chunk < 1) chunk = 1;
  size_t sc = groups_bytes((int)chunk, S) + align_up((size_t)chunk * ld * 4);
  if (sc > need) need = sc;
  if (k_cand > 0) {
    const size_t hr = groups_bytes(T, S) + align_up((size_t)T * k_cand * 4);
    if (hr > need) need = hr;
  }
  // streaming scorer for the routed heads (m) and for the dense indexer (H)
  const int ks = k_cand > k ? k_cand : k;
  for (int mm : {m, p->num_heads}) {
    const StreamPlan sp = stream_plan(p, mm, ks, false);
    if (sp.use && sp.bytes_deferred > need) need = sp.bytes_deferred;
  }
  return need;
}

int misa_block_offsets(const int64_t* key_offsets, int32_t num_seqs, int32_t block,
                       int64_t* block_offsets, misa_stream_t stream) {
  if (!key_offsets || !block_offsets || num_seqs < 1 || block < 1 || block > 4096) {
    set_error("misa_block_offsets: invalid arguments");
    return MISA_ERR_INVALID_ARG;
  }
  return launch_block_offsets(key_offsets, num_seqs, block, block_offsets,
                              static_cast<cudaStream_t>(stream));
}

int misa_pool_keys(const misa_problem_t* p, const uint16_t* K, float* Kbar,
                   misa_stream_t stream) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (p->total_blocks == 0) return MISA_OK;
  if ((rc = check_ptr(K, 16, "K")) || (rc = check_ptr(Kbar, 16, "Kbar"))) return rc;
  return launch_pool(*p, K, Kbar, static_cast<cudaStream_t>(stream));
}

int misa_pool_keys_from(const misa_problem_t* p, const uint16_t* K, float* Kbar,
                        const int32_t* from_pos, misa_stream_t stream) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (p->total_blocks == 0) return MISA_OK;
  if ((rc = check_ptr(K, 16, "K")) || (rc = check_ptr(Kbar, 16, "Kbar")) ||
      (rc = check_ptr(from_pos, 4, "from_pos")))
    return rc;
  return launch_pool_from(*p, K, Kbar, from_pos, static_cast<cudaStream_t>(stream));
}

int misa_route(const misa_problem_t* p, const uint16_t* q, const float* w, const uint16_t* K,
               const float* Kbar, int32_t m, int32_t* heads, uint16_t* q_r, float* w_r,
               float* router_scores, void* ws, size_t ws_bytes, misa_stream_t stream) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (m < 1 || m > p->num_heads) {
    set_error("m=%d outside 1..H=%d", m, p->num_heads);
    return MISA_ERR_INVALID_ARG;
  }
  if (p->num_queries == 0) return MISA_OK;
  if ((rc = check_ptr(q, 16, "q")) || (rc = check_ptr(w, 4, "w")) || (rc = check_ptr(K, 16, "K")) ||
      (rc = check_ptr(Kbar, 16, "Kbar")) || (rc = check_ptr(heads, 4, "heads")) ||
      (rc = check_ptr(q_r, 16, "q_r")) || (rc = check_ptr(w_r, 4, "w_r")) ||
      (rc = check_ptr(ws, 16, "workspace")))
    return rc;
  if (router_scores && !aligned(router_scores, 4)) {
    set_error("router_scores misaligned");
    return MISA_ERR_INVALID_ARG;
  }
  const int T = p->num_queries, S = p->num_seqs;
  if (ws_bytes < groups_bytes(T, S)) {
    set_error("workspace too small: %zu < %zu", ws_bytes, groups_bytes(T, S));
    return MISA_ERR_WORKSPACE_TOO_SMALL;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c = carve(ws, T, S);
  if (route_tc_applies(p) && ws_bytes >= route_tc_bytes(p)) {
    const int G = route_tc_group_size(p->num_heads);
    if ((rc = launch_plan_groups(*p, 0, T, G, c.groups, c.count, st))) return rc;
    RouteTcArgs a;
    a.p = p; a.q = q; a.w = w; a.K = K; a.Kbar = Kbar; a.m = m; a.heads = heads; a.q_r = q_r;
    a.w_r = w_r; a.router_scores = router_scores; a.groups = c.groups; a.group_count = c.count;
    a.max_groups = (T + G - 1) / G + S; a.split = c.buf;
    return launch_route_tc(a, st);
  }
  const int G = route_group_size(p->num_heads);
  const int mg = route_max_groups(p);
  // Split the block ranges only when the workspace holds the partial sums.
  int nsplit = route_split_count(*p, mg, num_sms());
  if (nsplit > 1 && ws_bytes < route_bytes(p)) nsplit = 1;
  // the plan also clears the split path's per-group completion counters
  int* done = nsplit > 1 ? route_split_counters(c.buf, mg, nsplit) : nullptr;
  if ((rc = launch_plan_groups(*p, 0, T, G, c.groups, c.count, st, done, done ? mg : 0)))
    return rc;
  return launch_route(*p, q, w, K, Kbar, m, heads, q_r, w_r, router_scores, c.groups, c.count,
                      mg, G, nsplit, nsplit > 1 ? c.buf : nullptr, st);
}

int misa_score_topk(const misa_problem_t* p, const uint16_t* q_r, const float* w_r, int32_t m,
                    const uint16_t* K, int32_t k, int32_t* idx, float* val, float* scores_dbg,
                    int64_t scores_ld, void* ws, size_t ws_bytes, misa_stream_t stream) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (!pow2_le64(m) || m > p->num_heads) {
    set_error("m=%d must be a power of two <= min(64, H)", m);
    return pow2_le64(m) ? MISA_ERR_INVALID_ARG : MISA_ERR_UNSUPPORTED;
  }
  if (k < 1 || k > 65536) { set_error("k=%d outside 1..65536", k); return MISA_ERR_INVALID_ARG; }
  if (p->num_queries == 0) return MISA_OK;
  if ((rc = check_ptr(q_r, 16, "q_r")) || (rc = check_ptr(w_r, 4, "w_r")) ||
      (rc = check_ptr(K, 16, "K")) || (rc = check_ptr(idx, 4, "idx")) ||
      (rc = check_ptr(val, 4, "val")) || (rc = check_ptr(ws, 16, "workspace")))
    return rc;
  if (scores_dbg && (scores_ld < p->max_seq_len || !aligned(scores_dbg, 4))) {
    set_error("scores_dbg needs scores_ld >= max_seq_len and 4-byte alignment");
    return MISA_ERR_INVALID_ARG;
  }
  return score_topk_impl(p, q_r, w_r, m, K, k, idx, val, scores_dbg, scores_ld, ws, ws_bytes,
                         static_cast<cudaStream_t>(stream));
}

int dsa_index_dense(const misa_problem_t* p, const uint16_t* q, const float* w,
                    const uint16_t* K, int32_t k, int32_t* idx, float* val, float* scores_dbg,
                    int64_t scores_ld, void* ws, size_t ws_bytes, misa_stream_t stream) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (!pow2_le64(p->num_heads)) {
    set_error("dense indexer needs H a power of two, got %d", p->num_heads);
    return MISA_ERR_UNSUPPORTED;
  }
  if (k < 1 || k > 65536) { set_error("k=%d outside 1..65536", k); return MISA_ERR_INVALID_ARG; }
  if (p->num_queries == 0) return MISA_OK;
  if ((rc = check_ptr(q, 16, "q")) || (rc = check_ptr(w, 4, "w")) || (rc = check_ptr(K, 16, "K")) ||
      (rc = check_ptr(idx, 4, "idx")) || (rc = check_ptr(val, 4, "val")) ||
      (rc = check_ptr(ws, 16, "workspace")))
    return rc;
  if (scores_dbg && (scores_ld < p->max_seq_len || !aligned(scores_dbg, 4))) {
    set_error("scores_dbg needs scores_ld >= max_seq_len and 4-byte alignment");
    return MISA_ERR_INVALID_ARG;
  }
  return score_topk_impl(p, q, w, p->num_heads, K, k, idx, val, scores_dbg, scores_ld, ws,
                         ws_bytes, static_cast<cudaStream_t>(stream));
}

int misa_hier_rerank(const misa_problem_t* p, const uint16_t* q, const float* w,
                     const uint16_t* K, const int32_t* cand, int32_t k_cand, int32_t k,
                     int32_t* idx, float* val, void* ws, size_t ws_bytes, misa_stream_t stream) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (!pow2_le64(p->num_heads)) {
    set_error("re-rank needs H a power of two, got %d", p->num_heads);
    return MISA_ERR_UNSUPPORTED;
  }
  if (k < 1 || k_cand < k || k_cand > 65536) {
    set_error("need 1 <= k <= k_cand <= 65536 (k=%d k_cand=%d)", k, k_cand);
    return MISA_ERR_INVALID_ARG;
  }
  const int T = p->num_queries, S = p->num_seqs;
  if (T == 0) return MISA_OK;
  if ((rc = check_ptr(q, 16, "q")) || (rc = check_ptr(w, 4, "w")) || (rc = check_ptr(K, 16, "K")) ||
      (rc = check_ptr(cand, 4, "cand")) || (rc = check_ptr(idx, 4, "idx")) ||
      (rc = check_ptr(val, 4, "val")) || (rc = check_ptr(ws, 16, "workspace")))
    return rc;
  const size_t need = groups_bytes(T, S) + align_up((size_t)T * k_cand * 4);
  if (ws_bytes < need) {
    set_error("workspace too small: %zu < %zu", ws_bytes, need);
    return MISA_ERR_WORKSPACE_TOO_SMALL;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c = carve(ws, T, S);
  // one query per group: the scoring kernel takes query rows directly (no plan)
  ScoreArgs a;
  a.p = p; a.qsel = q; a.wsel = w; a.m = p->num_heads; a.K = K; a.cand = cand;
  a.k_cand = k_cand; a.groups = nullptr; a.group_count = nullptr; a.max_groups = T;
  a.direct = true;
  a.G = 1; a.q_lo = 0; a.I = c.buf; a.ld = k_cand;
  a.max_tiles = (k_cand + kTileKeys - 1) / kTileKeys;
  if ((rc = launch_score(a, st))) return rc;
  return launch_topk(*p, c.buf, k_cand, cand, k_cand, 0, T, k, idx, val, st);
}

int misa_profile_enable(int32_t on) {
  t_prof_on = on != 0;
  return MISA_OK;
}

int misa_profile_collect(int32_t max_kernels, char* names, double* total_ms, int64_t* launches) {
  std::map<std::string, std::pair<double, int64_t>> acc;
  std::vector<std::string> order;
  for (auto& r : t_prof) {
    cudaError_t e = cudaEventSynchronize(r.stop);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.start, r.stop);
    if (e != cudaSuccess) return -cuda_fail(e, "misa_profile_collect");
    auto it = acc.find(r.name);
    if (it == acc.end()) {
      order.push_back(r.name);
      acc[r.name] = {ms, r.kernels};
    } else {
      it->second.first += ms;
      it->second.second += r.kernels;
    }
    t_free_events.push_back(r.start);
    t_free_events.push_back(r.stop);
  }
  t_prof.clear();
  for (auto& c : t_counts) {
    cudaError_t e = cudaEventSynchronize(c.done);
    if (e != cudaSuccess) return -cuda_fail(e, "misa_profile_collect");
    auto it = acc.find(c.name);
    if (it == acc.end()) {
      order.push_back(c.name);
      acc[c.name] = {0.0, *c.slot};
    } else {
      it->second.second += *c.slot;
    }
    t_free_slots.push_back(c.slot);
    t_free_events.push_back(c.done);
  }
  t_counts.clear();
  int n = 0;
  for (auto& name : order) {
    if (n >= max_kernels) break;
    if (names) {
      std::strncpy(names + 32 * n, name.c_str(), 31);
      names[32 * n + 31] = 0;
    }
    if (total_ms) total_ms[n] = acc[name].first;
    if (launches) launches[n] = acc[name].second;
    ++n;
  }
  return n;
}

int misa_stream_status(misa_stream_t stream, int32_t* device_status) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t* sp = status_ptr();
  if (!sp) { set_error("status word unavailable"); return MISA_ERR_CUDA; }
  uint32_t v = 0;
  e = cudaMemcpy(&v, sp, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  e = cudaMemset(sp, 0, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  if (device_status) *device_status = (int32_t)v;
  if (v & MISA_STATUS_TIMEOUT) { set_error("a device wait timed out"); return MISA_ERR_DEVICE_TIMEOUT; }
  if (v & MISA_STATUS_BOUNDS) { set_error("a device index was out of range"); return MISA_ERR_DEVICE_BOUNDS; }
  if (v & MISA_STATUS_BAD_INPUT) { set_error("bad input (position, candidate or a NaN score)"); return MISA_ERR_DEVICE_BAD_INPUT; }
  return MISA_OK;
}

int misa_selftest_timeout(int32_t wait_ms, misa_stream_t stream) {
  if (wait_ms < 1 || wait_ms > 5000) {
    set_error("wait_ms=%d outside 1..5000", wait_ms);
    return MISA_ERR_INVALID_ARG;
  }
  uint32_t* sp = status_ptr();
  if (!sp) { set_error("status word unavailable"); return MISA_ERR_CUDA; }
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (long long)wait_ms * 1000000ll, sp);
  return cuda_fail(cudaGetLastError(), "selftest_timeout_kernel");
}

}  // extern "C"
