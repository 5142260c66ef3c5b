// Host-side declarations shared by the translation units of libmisa.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/misa.h"

namespace misa {

constexpr int kD = 128;          // head dimension (fixed)
constexpr int kTileKeys = 128;   // keys per MMA tile (TMEM lanes)
constexpr int kSms = 148;

// One query group: queries [q_begin, q_end) of sequence `seq`, largest position max_pos.
// Stored as int4 {seq, q_begin, q_end, max_pos}.

void set_error(const char* fmt, ...);
int cuda_fail(cudaError_t e, const char* what);

// Device status word of the current device (a __device__ variable of libmisa).
uint32_t* status_ptr();

// cuTensorMapEncodeTiled through the runtime's driver entry point: 2-D bf16
// tensor [rows, 128] with a {64, box_rows} box and 128-byte swizzle.
int make_kmajor_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows);

int set_smem_limit(const void* kernel, int bytes);

// Launches `kern` with programmatic dependent launch: its CTAs may be
// scheduled while the previous kernel on `st` is still finishing.  Every
// kernel launched this way calls pdl_wait() (common.cuh) before it reads or
// writes global memory, so the result is the same as with plain stream order.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}
// SMs of the current device.
int num_sms();
// Workspace misa_route uses on its fastest path for a checked problem.
size_t route_path_bytes(const misa_problem_t* p);
// Whether tracing (misa_profile_enable) is on for the calling host thread.
bool tracing_enabled();

// Tracing: copies a device int32 counter back after the work queued on `st`
// so far; misa_profile_collect adds it under `name` (in the launch-count
// field).  No effect unless tracing is on.
void prof_count(const char* name, const int* dev_count, cudaStream_t st);

// Tracing: brackets one kernel launch with events on `st` when profiling is on.
struct ProfScope {
  ProfScope(const char* name, cudaStream_t st);
  ~ProfScope();
  int slot;
  cudaStream_t st;
};

// ---- pool.cu
int launch_block_offsets(const int64_t* key_offsets, int S, int B, int64_t* block_offsets,
                         cudaStream_t st);
// Build query groups of at most G queries over query rows [q_lo, q_hi).
// groups: int4 [q_hi-q_lo + S]; count: one int, followed 16 bytes later by
// int [S] of scratch (the first group of each sequence).
// zero / nzero: an int array that the plan also clears (the router's
// per-group completion counters), or nullptr.
int launch_plan_groups(const misa_problem_t& p, int q_lo, int q_hi, int G, int4* groups,
                       int* count, cudaStream_t st, int* zero = nullptr, int nzero = 0);
int launch_pool(const misa_problem_t& p, const uint16_t* K, float* Kbar, cudaStream_t st);
// Re-pool only the blocks of each sequence s that hold keys >= from_pos[s].
int launch_pool_from(const misa_problem_t& p, const uint16_t* K, float* Kbar,
                     const int32_t* from_pos, cudaStream_t st);

// ---- route.cu
int launch_route(const misa_problem_t& p, const uint16_t* q, const float* w, const uint16_t* K,
                 const float* Kbar, int m, int32_t* heads, uint16_t* q_r, float* w_r,
                 float* router_scores, const int4* groups, const int* group_count,
                 int max_groups, int G, int nsplit, float* partial, cudaStream_t st);
int route_group_size(int H);
// Pooled-block ranges per group for the CUDA-core router (1 = no split) and
// the workspace its partial sums take.
int route_split_count(const misa_problem_t& p, int max_groups, int sms);
size_t route_split_bytes(int max_groups, int nsplit);
// The per-group completion counters inside that scratch (cleared by the plan).
int* route_split_counters(float* partial, int max_groups, int nsplit);

// ---- route_tc.cu: the router as a tcgen05 GEMM (prefill-sized problems).
struct RouteTcArgs {
  const misa_problem_t* p;
  const uint16_t* q;
  const float* w;
  const uint16_t* K;
  const float* Kbar;
  int m;
  int32_t* heads;
  uint16_t* q_r;
  float* w_r;
  float* router_scores;
  const int4* groups;     // route_tc_group_size(H) queries per group
  const int* group_count;
  int max_groups;
  void* split;            // route_tc_split_bytes(p) of workspace
  float* Pm;              // set by launch_route_tc (inside split)
};
int launch_route_tc(const RouteTcArgs& a, cudaStream_t st);
int route_tc_group_size(int H);
size_t route_tc_split_bytes(const misa_problem_t& p);

// ---- score.cu
// I[(t - q_lo) * ld + s] = sum_{j<m} wsel[t,j] ReLU(qsel[t,j] . K[key(t,s)]) for the
// queries of the groups.  Contiguous mode (cand == nullptr): s = 0..q_pos[t].
// Gather mode: s = slot 0..k_cand-1 of cand[t, :], key = cand[t, s].
struct ScoreArgs {
  const misa_problem_t* p;
  const uint16_t* qsel;   // [T * m, 128] bf16
  const float* wsel;      // [T, m]
  int m;
  const uint16_t* K;      // [total_keys, 128] bf16
  const int32_t* cand;    // [T, k_cand] or nullptr
  int k_cand;
  const int4* groups;     // device group table
  const int* group_count; // device: number of valid groups
  int max_groups;         // host bound on the group count
  int G;                  // queries per group
  int q_lo;
  float* I;               // output rows
  int64_t ld;
  int max_tiles;          // host bound on key tiles per group
  bool direct = false;    // gather mode without a plan: group i is query row i
  bool row_by_group = false;  // groups of one query each; group i writes row i of I
};
int launch_score(const ScoreArgs& a, cudaStream_t st);

// ---- score_stream.cu: scoring with the top-k fused (every query's full prefix).
struct StreamArgs {
  const misa_problem_t* p;
  const uint16_t* qsel;   // [T * m, 128] bf16
  const float* wsel;      // [T, m]
  int m;                  // 8, 16, 32 or 64
  const uint16_t* K;
  const int4* groups;     // G = stream_group_size(m) queries per group
  const int* group_count;
  int max_groups;
  int grid;               // persistent CTAs (<= number of SMs)
  int k;
  uint2* cand;            // stream_cand_bytes(grid, subcap, m): candidate lists and counts
  int64_t subcap;         // stream_subcap(max_seq_len): rows of each list
  int32_t* idx;
  float* val;
  int32_t* fail_list;     // [T] queries whose sampled threshold did not verify
  int* fail_count;        // device counter for fail_list
  // Deferred selection (nullptr dcand: selection inside the scoring kernel):
  // one list per query row, stream_deferred_bytes(T, subcap, k) in all.
  uint2* dcand = nullptr;  // [T][drows][128]
  int* dcnt = nullptr;     // [T][128]
  int2* danchor = nullptr; // [T] {histogram base, top score bits}
  int drows = 0;           // stream_deferred_rows(k, subcap)
};
int launch_score_stream(const StreamArgs& a, cudaStream_t st);
size_t stream_deferred_bytes(int T, int64_t subcap, int k);
int stream_deferred_rows(int k, int64_t subcap);
int stream_group_size(int m);
size_t stream_cand_bytes(int grid, int64_t subcap, int m);
int64_t stream_subcap(int max_seq_len);
int score_group_size(int m);

// ---- topk.cu
// For query rows [q_lo, q_hi): select the top-k of I row (t - q_lo).
// Contiguous mode (tok == nullptr): elements 0..q_pos[t], token = element index.
// Token mode: elements 0..n_fixed-1 with token tok[t * n_fixed + e] (< 0 = absent).
// rows_list / rows_count (device, optional): row i of I belongs to query
// rows_list[i] for i < *rows_count; rows past the count are skipped (the
// grid still covers q_hi - q_lo rows).
int launch_topk(const misa_problem_t& p, const float* I, int64_t ld, const int32_t* tok,
                int n_fixed, int q_lo, int q_hi, int k, int32_t* idx, float* val,
                cudaStream_t st, const int32_t* rows_list = nullptr,
                const int* rows_count = nullptr);

}  // namespace misa
