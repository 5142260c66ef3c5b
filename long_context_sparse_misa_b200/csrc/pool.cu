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

void prof_add_kernels(int n);  // abi.cu: counts an extra kernel of the open profiling scope
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

constexpr int kSmallPlanGroups = 256;  // plans up to this many groups take one CTA

// Query groups: every sequence's queries, restricted to [q_lo, q_hi), are cut
// into groups of at most G, recorded as {seq, q_begin, q_end, max_pos}.
// First a one-CTA scan over sequences gives each sequence the index of its
// first group (first[s]) and the group count; then one warp per group finds
// its sequence by binary search over first[] and reduces its queries'
// positions.  Positions outside their sequence are flagged and left out of
// max_pos.
__device__ __forceinline__ void group_scan(const int32_t* __restrict__ qo, int S, int q_lo,
                                           int q_hi, int G, int* __restrict__ first,
                                           int* __restrict__ count) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int base = 0; base < S; base += blockDim.x) {
    const int c0 = carry;
    const int s = base + threadIdx.x;
    int ng = 0;
    if (s < S) {
      const int b = max(qo[s], q_lo), e = min(qo[s + 1], q_hi);
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
    const int f = c0 + (warp > 0 ? warp_sums[warp - 1] : 0) + x - ng;
    if (s < S) first[s] = f;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = f + ng;
    __syncthreads();
  }
  if (threadIdx.x == 0) *count = carry;
}

__global__ void group_scan_kernel(const int32_t* __restrict__ qo, int S, int q_lo, int q_hi,
                                  int G, int* __restrict__ first, int* __restrict__ count,
                                  int* __restrict__ zero, int nzero) {
  pdl_wait_then_release();
  for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0;
  group_scan(qo, S, q_lo, q_hi, G, first, count);
}

// Group fg (by one warp).
__device__ __forceinline__ void group_fill(const int64_t* __restrict__ ko,
                                           const int32_t* __restrict__ qo,
                                           const int32_t* __restrict__ q_pos, int S, int q_lo,
                                           int q_hi, int G, const int* __restrict__ first, int fg,
                                           int4* __restrict__ groups, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = S - 1;  // last sequence j with first[j] <= fg
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (first[mid] <= fg) lo = mid; else hi = mid - 1;
  }
  const int j = lo;
  const int b = max(qo[j], q_lo), e = min(qo[j + 1], q_hi);
  const int qb = b + (fg - first[j]) * G, qe = min(qb + G, e);
  const int64_t L = ko[j + 1] - ko[j];
  int mp = -1;
  for (int t = qb + lane; t < qe; t += 32) {
    const int pos = q_pos[t];
    if (pos < 0 || pos >= L) set_status(status, MISA_STATUS_BAD_INPUT);
    else mp = max(mp, pos);
  }
  mp = __reduce_max_sync(0xffffffffu, mp);
  if (lane == 0) groups[fg] = make_int4(j, qb, qe, mp);
}

__global__ void group_fill_kernel(const int64_t* __restrict__ ko, const int32_t* __restrict__ qo,
                                  const int32_t* __restrict__ q_pos, int S, int q_lo, int q_hi,
                                  int G, const int* __restrict__ first,
                                  const int* __restrict__ count, int4* __restrict__ groups,
                                  uint32_t* status) {
  pdl_wait_then_release();
  const int fg = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  if (fg >= *count) return;
  group_fill(ko, qo, q_pos, S, q_lo, q_hi, G, first, fg, groups, status);
}

// Both steps in one CTA, for plans of few groups (a decode batch): the scan,
// a block barrier (the CTA's global writes are then visible to all its
// threads), and the warps take the groups round-robin.
__global__ void group_plan_small_kernel(const int64_t* __restrict__ ko,
                                        const int32_t* __restrict__ qo,
                                        const int32_t* __restrict__ q_pos, int S, int q_lo,
                                        int q_hi, int G, int* __restrict__ first,
                                        int* __restrict__ count, int4* __restrict__ groups,
                                        uint32_t* status, int* __restrict__ zero, int nzero) {
  pdl_wait_then_release();
  for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0;
  group_scan(qo, S, q_lo, q_hi, G, first, count);
  __syncthreads();
  // S <= kSmallPlanGroups here: the first groups of the sequences go to
  // shared memory for the warps' binary searches
  __shared__ int sfirst[kSmallPlanGroups];
  for (int s = threadIdx.x; s < S; s += blockDim.x) sfirst[s] = first[s];
  __syncthreads();
  const int n = *count;
  for (int fg = threadIdx.x >> 5; fg < n; fg += blockDim.x >> 5)
    group_fill(ko, qo, q_pos, S, q_lo, q_hi, G, sfirst, fg, groups, status);
}

// One warp per pooled row.  The two half-warps take alternate keys and each
// lane owns 8 of the 128 dims (one 16-byte load per key), with 8 loads in
// flight per lane; the halves are added at the end.  fp64 sums: every
// partial sum of at most 4096 bf16 keys is exact for keys within 2^33 of one
// another in magnitude, so the split does not change the result, and the
// fp32 mean is the correctly rounded mean of the bf16 keys.
__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4 v) {
  acc[0] += (double)__uint_as_float(v.x << 16);
  acc[1] += (double)__uint_as_float(v.x & 0xFFFF0000u);
  acc[2] += (double)__uint_as_float(v.y << 16);
  acc[3] += (double)__uint_as_float(v.y & 0xFFFF0000u);
  acc[4] += (double)__uint_as_float(v.z << 16);
  acc[5] += (double)__uint_as_float(v.z & 0xFFFF0000u);
  acc[6] += (double)__uint_as_float(v.w << 16);
  acc[7] += (double)__uint_as_float(v.w & 0xFFFF0000u);
}

// Mean of the keys of pooled row `row` of sequence s (block b), by one warp.
__device__ __forceinline__ void pool_row(const uint16_t* __restrict__ K, int64_t k0, int64_t k1,
                                         int64_t row, float* __restrict__ Kbar) {
  const int lane = threadIdx.x & 31;
  constexpr int kRow16 = kD / 8;  // 16-byte chunks per key
  const int half = lane >> 4, hl = lane & 15;
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  const uint4* src = reinterpret_cast<const uint4*>(K) + k0 * kRow16 + hl;
  const int64_t n = k1 - k0;
  int64_t i = half;
  for (; i + 14 < n; i += 16) {  // keys i, i+2, ..., i+14
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(src + (i + 2 * u) * kRow16);
#pragma unroll
    for (int u = 0; u < 8; ++u) add_bf16x8(acc, v[u]);
  }
  for (; i < n; i += 2) add_bf16x8(acc, __ldg(src + i * kRow16));
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 16);
  if (half == 0) {
    const double cnt = (double)n;
    float4 lo, hi;
    lo.x = __double2float_rn(acc[0] / cnt);
    lo.y = __double2float_rn(acc[1] / cnt);
    lo.z = __double2float_rn(acc[2] / cnt);
    lo.w = __double2float_rn(acc[3] / cnt);
    hi.x = __double2float_rn(acc[4] / cnt);
    hi.y = __double2float_rn(acc[5] / cnt);
    hi.z = __double2float_rn(acc[6] / cnt);
    hi.w = __double2float_rn(acc[7] / cnt);
    float4* dst = reinterpret_cast<float4*>(Kbar) + row * (kD / 4) + 2 * hl;
    dst[0] = lo;
    dst[1] = hi;
  }
}

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
    if (lane == 0) set_status(status, MISA_STATUS_BOUNDS);
    return;
  }
  pool_row(K, k0, k1, row, Kbar);
}

// Incremental form: one CTA per sequence re-pools only the blocks that hold
// keys at or after from_pos[s] (the keys appended since the last pooling);
// the other rows of Kbar are left as they are.  Warps take the blocks
// round-robin.
__global__ void __launch_bounds__(256) pool_from_kernel(const uint16_t* __restrict__ K,
                                                        const int64_t* __restrict__ ko,
                                                        const int64_t* __restrict__ bo, int B,
                                                        const int32_t* __restrict__ from_pos,
                                                        float* __restrict__ Kbar,
                                                        uint32_t* status) {
  pdl_wait_then_release();
  const int s = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int64_t L = ko[s + 1] - ko[s];
  const int64_t nblk = bo[s + 1] - bo[s];
  int64_t f = from_pos[s];
  if (f < 0) f = 0;
  if (f >= L) return;  // nothing new in this sequence
  if (nblk != (L + B - 1) / B) {
    if (threadIdx.x == 0) set_status(status, MISA_STATUS_BOUNDS);
    return;
  }
  const int64_t b0 = f / B;
  if (nblk - b0 >= nw) {
    for (int64_t b = b0 + warp; b < nblk; b += nw) {
      const int64_t k0 = ko[s] + b * B;
      const int64_t k1 = min(k0 + (int64_t)B, ko[s + 1]);
      pool_row(K, k0, k1, bo[s] + b, Kbar);
    }
    return;
  }
  // Fewer new blocks than warps (a decode step): the whole CTA pools each
  // block, 16 half-warps taking every 16th key, and the partial fp64 sums are
  // added per dim through shared memory.  The fp64 sums are exact (see
  // pool_row), so this split gives the same means as one warp per block.
  __shared__ double part[16][kD];
  const int hw = threadIdx.x >> 4, hl = lane & 15;
  constexpr int kRow16 = kD / 8;
  for (int64_t b = b0; b < nblk; ++b) {
    const int64_t k0 = ko[s] + b * B;
    const int64_t k1 = min(k0 + (int64_t)B, ko[s + 1]);
    const int64_t n = k1 - k0;
    const uint4* src = reinterpret_cast<const uint4*>(K) + k0 * kRow16 + hl;
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    int64_t i = hw;
    for (; i + 16 * 7 < n; i += 16 * 8) {  // keys i, i+16, ..., i+112
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(src + (i + 16 * u) * kRow16);
#pragma unroll
      for (int u = 0; u < 8; ++u) add_bf16x8(acc, v[u]);
    }
    for (; i < n; i += 16) add_bf16x8(acc, __ldg(src + i * kRow16));
    __syncthreads();  // the previous block's sums have been read
#pragma unroll
    for (int j = 0; j < 8; ++j) part[hw][8 * hl + j] = acc[j];
    __syncthreads();
    if (threadIdx.x < kD) {
      double t = 0.0;
#pragma unroll
      for (int h = 0; h < 16; ++h) t += part[h][threadIdx.x];
      Kbar[(bo[s] + b) * kD + threadIdx.x] = __double2float_rn(t / (double)n);
    }
  }
}

}  // namespace

int launch_block_offsets(const int64_t* key_offsets, int S, int B, int64_t* block_offsets,
                         cudaStream_t st) {
  ProfScope ps("block_offsets", st);
  block_offsets_kernel<<<1, 1024, 0, st>>>(key_offsets, S, B, block_offsets, status_ptr());
  return cuda_fail(cudaGetLastError(), "block_offsets_kernel");
}

int launch_plan_groups(const misa_problem_t& p, int q_lo, int q_hi, int G, int4* groups,
                       int* count, cudaStream_t st, int* zero, int nzero) {
  ProfScope ps("plan_groups", st);
  int* first = count + 4;  // [S] after the count word (see groups_bytes)
  const int64_t max_groups = (int64_t)(q_hi - q_lo + G - 1) / G + p.num_seqs;
  if (max_groups <= kSmallPlanGroups) {
    return cuda_fail(launch_pdl(group_plan_small_kernel, dim3(1), dim3(1024), 0, st,
                                p.key_offsets, p.query_offsets, p.q_pos, p.num_seqs, q_lo, q_hi,
                                G, first, count, groups, status_ptr(), zero, nzero),
                     "group_plan_small_kernel");
  }
  cudaError_t e = launch_pdl(group_scan_kernel, dim3(1), dim3(1024), 0, st, p.query_offsets,
                             p.num_seqs, q_lo, q_hi, G, first, count, zero, nzero);
  if (e != cudaSuccess) return cuda_fail(e, "group_scan_kernel");
  prof_add_kernels(1);  // the fill below is this scope's second kernel
  const int warps = 8;
  e = launch_pdl(group_fill_kernel, dim3((unsigned)((max_groups + warps - 1) / warps)),
                 dim3(warps * 32), 0, st, p.key_offsets, p.query_offsets, p.q_pos, p.num_seqs,
                 q_lo, q_hi, G, (const int*)first, (const int*)count, groups, status_ptr());
  return cuda_fail(e, "group_fill_kernel");
}

int launch_pool_from(const misa_problem_t& p, const uint16_t* K, float* Kbar,
                     const int32_t* from_pos, cudaStream_t st) {
  ProfScope ps("pool_keys", st);
  return cuda_fail(launch_pdl(pool_from_kernel, dim3(p.num_seqs), dim3(256), 0, st, K,
                              p.key_offsets, p.block_offsets, p.block, from_pos, Kbar,
                              status_ptr()),
                   "pool_from_kernel");
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
