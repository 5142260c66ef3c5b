// Block offsets, query-group planning and mean pooling of indexer keys.
//
// Pooling follows "MISA: Mixture of Indexer Sparse Attention for
// Long-Context LLM Inference", gist.science summary, "Methodologie: MISA"
// (Lightweight Block-Pooled Router): the prefix is split into
// M = ceil(L/B) blocks and each block is represented by the mean of its
// indexer keys.  HBM-bound: K is read once, 1/B of it is written back.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

// One CTA: block_offsets[s+1] = block_offsets[s] + ceil(L_s / B), chunked scan.
__global__ void block_offsets_kernel(const int64_t* __restrict__ ko, int S, int B,
                                     int64_t* __restrict__ bo, uint32_t* status) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  if (threadIdx.x == 0) { carry = 0; bo[0] = 0; }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int64_t v = 0;
    if (s < S) {
      const int64_t L = ko[s + 1] - ko[s];
      if (L < 0) { set_status(status, MISA_STATUS_BAD_INPUT); }
      v = L > 0 ? (L + B - 1) / B : 0;
    }
    int64_t x = v;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int64_t ws = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += y;
      }
      warp_sums[lane] = ws;  // inclusive over warps
    }
    __syncthreads();
    const int64_t before = carry + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (s < S) bo[s + 1] = before + x;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + x;
    __syncthreads();
  }
}

// One CTA: split every sequence's queries (restricted to [q_lo, q_hi)) into
// groups of at most G and record {seq, q_begin, q_end, max_pos}.  A scan over
// sequences gives each sequence its first group index; then every warp takes
// groups round-robin and reduces the positions of its group's queries.
// Positions outside their sequence are flagged and left out of max_pos.
__global__ void plan_groups_kernel(const int64_t* __restrict__ ko, const int32_t* __restrict__ qo,
                                   const int32_t* __restrict__ q_pos, int S, int q_lo, int q_hi,
                                   int G, int4* __restrict__ groups, int* __restrict__ count,
                                   uint32_t* status) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  __shared__ int s_first[1024], s_ng[1024], s_b[1024], s_e[1024];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int b = 0, e = 0, ng = 0;
    if (s < S) {
      b = max(qo[s], q_lo);
      e = min(qo[s + 1], q_hi);
      ng = e > b ? (e - b + G - 1) / G : 0;
    }
    int x = ng;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int ws = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += y;
      }
      warp_sums[lane] = ws;
    }
    __syncthreads();
    const int first = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - ng;
    s_first[threadIdx.x] = first;
    s_ng[threadIdx.x] = ng;
    s_b[threadIdx.x] = b;
    s_e[threadIdx.x] = e;
    __syncthreads();
    const int nseq = min((int)blockDim.x, S - base);
    for (int j = 0; j < nseq; ++j) {
      const int ngj = s_ng[j];
      if (ngj == 0) continue;
      const int sj = base + j, bj = s_b[j], ej = s_e[j], fj = s_first[j];
      const int64_t L = ko[sj + 1] - ko[sj];
      for (int g = warp; g < ngj; g += nwarps) {
        const int qb = bj + g * G, qe = min(qb + G, ej);
        int mp = -1;
        for (int t = qb + lane; t < qe; t += 32) {
          const int pos = q_pos[t];
          if (pos < 0 || pos >= L) set_status(status, MISA_STATUS_BAD_INPUT);
          else mp = max(mp, pos);
        }
        mp = __reduce_max_sync(0xffffffffu, mp);
        if (lane == 0) groups[fj + g] = make_int4(sj, qb, qe, mp);
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = first + ng;
    __syncthreads();
  }
  if (threadIdx.x == 0) *count = carry;
}

// One warp per pooled row; each lane owns 4 of the 128 dims.  fp64 sums so
// that the fp32 mean is the correctly rounded mean of the bf16 keys.
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ K,
                                                   const int64_t* __restrict__ ko,
                                                   const int64_t* __restrict__ bo, int S, int B,
                                                   int64_t total_blocks, int64_t total_keys,
                                                   float* __restrict__ Kbar, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= total_blocks) return;
  const int s = upper_segment<int64_t>(bo, S, row);
  const int64_t b = row - bo[s];
  const int64_t k0 = ko[s] + b * B;
  const int64_t k1 = min(k0 + (int64_t)B, ko[s + 1]);
  if (k0 < 0 || k1 > total_keys || k1 <= k0) {
    set_status(status, MISA_STATUS_BOUNDS);
    return;
  }
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  const uint2* src = reinterpret_cast<const uint2*>(K) + k0 * (kD / 4) + lane;
  int64_t n = k1 - k0;
  int64_t i = 0;
  for (; i + 4 <= n; i += 4) {
    uint2 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(src + (i + u) * (kD / 4));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc[0] += (double)__uint_as_float(v[u].x << 16);
      acc[1] += (double)__uint_as_float(v[u].x & 0xFFFF0000u);
      acc[2] += (double)__uint_as_float(v[u].y << 16);
      acc[3] += (double)__uint_as_float(v[u].y & 0xFFFF0000u);
    }
  }
  for (; i < n; ++i) {
    const uint2 v = __ldg(src + i * (kD / 4));
    acc[0] += (double)__uint_as_float(v.x << 16);
    acc[1] += (double)__uint_as_float(v.x & 0xFFFF0000u);
    acc[2] += (double)__uint_as_float(v.y << 16);
    acc[3] += (double)__uint_as_float(v.y & 0xFFFF0000u);
  }
  const double cnt = (double)n;
  float4 out;
  out.x = __double2float_rn(acc[0] / cnt);
  out.y = __double2float_rn(acc[1] / cnt);
  out.z = __double2float_rn(acc[2] / cnt);
  out.w = __double2float_rn(acc[3] / cnt);
  reinterpret_cast<float4*>(Kbar)[row * (kD / 4) + lane] = out;
}

}  // namespace

int launch_block_offsets(const int64_t* key_offsets, int S, int B, int64_t* block_offsets,
                         cudaStream_t st) {
  ProfScope ps("block_offsets", st);
  block_offsets_kernel<<<1, 1024, 0, st>>>(key_offsets, S, B, block_offsets, status_ptr());
  return cuda_fail(cudaGetLastError(), "block_offsets_kernel");
}

int launch_plan_groups(const misa_problem_t& p, int q_lo, int q_hi, int G, int4* groups,
                       int* count, cudaStream_t st) {
  ProfScope ps("plan_groups", st);
  plan_groups_kernel<<<1, 1024, 0, st>>>(p.key_offsets, p.query_offsets, p.q_pos, p.num_seqs,
                                         q_lo, q_hi, G, groups, count, status_ptr());
  return cuda_fail(cudaGetLastError(), "plan_groups_kernel");
}

int launch_pool(const misa_problem_t& p, const uint16_t* K, float* Kbar, cudaStream_t st) {
  if (p.total_blocks == 0) return MISA_OK;
  const int warps = 8;
  const int64_t grid = (p.total_blocks + warps - 1) / warps;
  ProfScope ps("pool_keys", st);
  pool_kernel<<<(unsigned)grid, warps * 32, 0, st>>>(K, p.key_offsets, p.block_offsets,
                                                    p.num_seqs, p.block, p.total_blocks,
                                                    p.total_keys, Kbar, status_ptr());
  return cuda_fail(cudaGetLastError(), "pool_kernel");
}

}  // namespace misa
