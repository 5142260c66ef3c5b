// Per-query top-k selection over fp32 index scores.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
// Inference", gist.science summary, "Methodologie: MISA" (the final top-k
// tokens are selected from the routed heads' scores) and "Hierarchische
// Variant (MISA†)" (top-k of the re-scored candidates).
//
// Exact radix select, one CTA per query row.  Every element gets a 64-bit key
//     (order-preserving bits of the fp32 score) << 32 | (0xFFFFFFFF - token)
// so that a larger key means a higher score and, among equal scores, a lower
// token index; -0 is folded onto +0.  Digits of 11/11/10/11/11/10 bits are
// resolved from the top; a pass stops early as soon as the bin holding the
// k-th element is consumed exactly, which in practice happens after the
// first two score digits.  A last pass writes every element whose key prefix
// is at or above the threshold prefix: exactly min(k, n) of them.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kMaxBins = 2048;

struct Row {
  const float* I;
  const int32_t* tok;  // nullptr: token = element index
  int n;
  int pos;             // token limit (token mode)
};

__device__ __forceinline__ bool elem(const Row& r, int e, uint64_t& key, float& v, int& token) {
  v = r.I[e];
  if (r.tok) {
    token = r.tok[e];
    if (token < 0 || token > r.pos) return false;
  } else {
    token = e;
  }
  key = (static_cast<uint64_t>(order_key(v)) << 32) |
        static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(token));
  return true;
}

// Exclusive prefix sum over the CTA (thread order), returns this thread's offset.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t x, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = warp_tot[lane];
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;  // exclusive over warps
  }
  __syncthreads();
  const uint32_t r = warp_tot[warp] + inc - x;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kTopkThreads, 1)
    topk_kernel(const float* __restrict__ I, int64_t ld, const int32_t* __restrict__ tok,
                int n_fixed, const int64_t* __restrict__ ko, const int32_t* __restrict__ qo,
                const int32_t* __restrict__ q_pos, int S, int q_lo, int k,
                int32_t* __restrict__ idx_out, float* __restrict__ val_out, uint32_t* status) {
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t sel_bin, sel_above, sel_count, n_valid, out_cnt;

  const int t = q_lo + blockIdx.x;
  const int s = upper_segment<int32_t>(qo, S, t);
  const int64_t L = ko[s + 1] - ko[s];
  int pos = q_pos[t];
  if (pos < 0 || pos >= L) pos = -1;

  Row r;
  r.I = I + (int64_t)blockIdx.x * ld;
  r.tok = tok ? tok + (int64_t)t * n_fixed : nullptr;
  r.n = tok ? n_fixed : pos + 1;
  r.pos = pos;

  int32_t* idx = idx_out + (int64_t)t * k;
  float* val = val_out + (int64_t)t * k;

  constexpr int kShift[6] = {53, 42, 32, 21, 10, 0};
  constexpr int kWidth[6] = {11, 11, 10, 11, 11, 10};

  uint64_t prefix = 0;
  uint32_t remaining = (uint32_t)k;
  int shift = 64;  // 64: select every valid element
  bool done = false;
  if (threadIdx.x == 0) { n_valid = 0; out_cnt = 0; }
  if (!tok) {
    if (r.n <= k) done = true;
  }

  for (int p = 0; p < 6 && !done; ++p) {
    const int width = kWidth[p], sh = kShift[p];
    const int nb = 1 << width;
    const uint32_t mask = (uint32_t)nb - 1u;
    for (int b = threadIdx.x; b < nb; b += kTopkThreads) hist[b] = 0;
    __syncthreads();
    uint32_t local_valid = 0;
    for (int e = threadIdx.x; e < r.n; e += kTopkThreads) {
      uint64_t key; float v; int token;
      if (!elem(r, e, key, v, token)) continue;
      ++local_valid;
      if (p == 0 || (key >> (sh + width)) == prefix)
        atomicAdd(&hist[(uint32_t)(key >> sh) & mask], 1u);
    }
    if (p == 0 && tok) {
      atomicAdd(&n_valid, local_valid);
      __syncthreads();
      if (n_valid <= (uint32_t)k) { done = true; break; }  // uniform: every thread reads the same
    }
    __syncthreads();
    // Bins in descending order: thread i owns positions i*bpt .. i*bpt+bpt-1.
    const int bpt = nb / kTopkThreads;  // 1 or 2
    uint32_t c[2] = {0, 0};
    for (int j = 0; j < bpt; ++j) c[j] = hist[nb - 1 - (threadIdx.x * bpt + j)];
    const uint32_t above0 = block_exclusive_scan(c[0] + c[1], warp_tot);
    uint32_t above = above0;
    for (int j = 0; j < bpt; ++j) {
      if (above < remaining && above + c[j] >= remaining) {
        sel_bin = (uint32_t)(nb - 1 - (threadIdx.x * bpt + j));
        sel_above = above;
        sel_count = c[j];
      }
      above += c[j];
    }
    __syncthreads();
    remaining -= sel_above;
    prefix = (prefix << width) | sel_bin;
    shift = sh;
    if (sel_count == remaining) done = true;
    __syncthreads();
  }

  // Output every valid element whose key prefix is >= the threshold prefix.
  for (int e = threadIdx.x; e < r.n; e += kTopkThreads) {
    uint64_t key; float v; int token;
    if (!elem(r, e, key, v, token)) continue;
    if (shift == 64 || (key >> shift) >= prefix) {
      const uint32_t slot = atomicAdd(&out_cnt, 1u);
      if (slot < (uint32_t)k) {
        idx[slot] = token;
        val[slot] = v + 0.0f;
      } else {
        set_status(status, MISA_STATUS_BOUNDS);  // duplicate tokens in a candidate row
      }
    }
  }
  __syncthreads();
  for (int j = out_cnt + threadIdx.x; j < k; j += kTopkThreads) {
    idx[j] = -1;
    val[j] = -INFINITY;
  }
}

}  // namespace

int launch_topk(const misa_problem_t& p, const float* I, int64_t ld, const int32_t* tok,
                int n_fixed, int q_lo, int q_hi, int k, int32_t* idx, float* val,
                cudaStream_t st) {
  if (q_hi <= q_lo) return MISA_OK;
  ProfScope ps("topk", st);
  topk_kernel<<<q_hi - q_lo, kTopkThreads, 0, st>>>(I, ld, tok, n_fixed, p.key_offsets,
                                                    p.query_offsets, p.q_pos, p.num_seqs, q_lo,
                                                    k, idx, val, status_ptr());
  return cuda_fail(cudaGetLastError(), "topk_kernel");
}

}  // namespace misa
