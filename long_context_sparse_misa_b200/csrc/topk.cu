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
//
// Decode batches have few rows, each a long prefix.  There a row is split
// over a thread-block cluster: each CTA loads its slice of the row once into
// shared memory as 64-bit keys, builds its digit histogram there, and reads
// the other CTAs' histograms over distributed shared memory; every CTA then
// holds the same row histogram and takes the same decision, so the passes
// need no further exchange.  The output slots come from one counter in the
// first CTA of the cluster.
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
                int32_t* __restrict__ idx_out, float* __restrict__ val_out, uint32_t* status,
                const int32_t* __restrict__ rows_list, const int* __restrict__ rows_count) {
  pdl_wait_then_release();
  if (rows_list && (int)blockIdx.x >= *rows_count) return;
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t sel_bin, sel_above, sel_count, n_valid, out_cnt;

  const int t = rows_list ? rows_list[blockIdx.x] : q_lo + (int)blockIdx.x;
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
        // NaN ranks below every number, so it is selected only to fill a row
        // that has fewer numbers than the row needs
        if (v != v) set_status(status, MISA_STATUS_BAD_INPUT);
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

// ---------------------------------------------------------------- cluster form
constexpr int kClusterCap = 16384;  // keys per CTA held in shared memory
constexpr int kMaxCluster = 8;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster; orders shared-memory writes
// before the barrier against reads after it, cluster-wide.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ uint32_t dsmem_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t dsmem_atomic_add(uint32_t addr, uint32_t x) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(x)
               : "memory");
  return old;
}

__device__ __forceinline__ uint32_t block_sum(uint32_t x, uint32_t* warp_tot) {
  const uint32_t off = block_exclusive_scan(x, warp_tot);
  __shared__ uint32_t total;
  if (threadIdx.x == kTopkThreads - 1) total = off + x;
  __syncthreads();
  const uint32_t r = total;
  __syncthreads();
  return r;
}

// Grid: rows x C CTAs, cluster (C,1,1); C = gridDim.x / rows.
__global__ void __launch_bounds__(kTopkThreads, 1)
    topk_cluster_kernel(const float* __restrict__ I, int64_t ld, const int32_t* __restrict__ tok,
                        int n_fixed, const int64_t* __restrict__ ko,
                        const int32_t* __restrict__ qo, const int32_t* __restrict__ q_pos, int S,
                        int q_lo, int k, int C, int32_t* __restrict__ idx_out,
                        float* __restrict__ val_out, uint32_t* status,
                        const int32_t* __restrict__ rows_list,
                        const int* __restrict__ rows_count) {
  pdl_wait_then_release();
  extern __shared__ __align__(16) uint64_t keys[];  // [kClusterCap]; 0 = not a candidate
  __shared__ uint32_t hist[2][kMaxBins];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_valid, s_out;
  __shared__ uint32_t sel_bin, sel_above, sel_count;

  const uint32_t rank = cluster_ctarank();
  const int row = blockIdx.x / C;
  // (uniform over the cluster: every CTA of it has the same row)
  if (rows_list && row >= *rows_count) return;
  const int t = rows_list ? rows_list[row] : q_lo + row;
  const int s = upper_segment<int32_t>(qo, S, t);
  const int64_t L = ko[s + 1] - ko[s];
  int pos = q_pos[t];
  if (pos < 0 || pos >= L) pos = -1;

  Row r;
  r.I = I + (int64_t)row * ld;
  r.tok = tok ? tok + (int64_t)t * n_fixed : nullptr;
  r.n = tok ? n_fixed : pos + 1;
  r.pos = pos;
  int32_t* idx = idx_out + (int64_t)t * k;
  float* val = val_out + (int64_t)t * k;

  const int chunk = (((r.n + C - 1) / C) + 3) & ~3;
  if (chunk > kClusterCap) {  // uniform over the cluster: no CTA reaches a barrier
    if (rank == 0 && threadIdx.x == 0) set_status(status, MISA_STATUS_BOUNDS);
    return;
  }
  const int e0 = (int)rank * chunk;
  const int nloc = max(0, min(r.n, e0 + chunk) - e0);

  // Load the slice with 8 independent loads in flight per thread.
  uint32_t local_valid = 0;
  constexpr int kU = 8;
  for (int i0 = 0; i0 < nloc; i0 += kU * kTopkThreads) {
    float v[kU];
    int tk[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kTopkThreads + threadIdx.x;
      v[u] = 0.f;
      tk[u] = -1;
      if (i < nloc) {
        v[u] = r.I[e0 + i];
        tk[u] = r.tok ? r.tok[e0 + i] : e0 + i;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kTopkThreads + threadIdx.x;
      if (i >= nloc) continue;
      const bool ok = tk[u] >= 0 && (!r.tok || tk[u] <= r.pos);
      // A real key is never 0: its low word is 0xFFFFFFFF - token >= 2^31.
      keys[i] = ok ? (static_cast<uint64_t>(order_key(v[u])) << 32) |
                         static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(tk[u]))
                   : 0ull;
      local_valid += ok;
    }
  }
  const uint32_t cta_valid = block_sum(local_valid, warp_tot);
  if (threadIdx.x == 0) {
    s_valid = cta_valid;
    s_out = 0;
  }
  cluster_barrier();  // s_valid of every CTA and s_out of CTA 0 are set
  uint32_t n_valid = 0;
  for (int q = 0; q < C; ++q) n_valid += dsmem_ld(dsmem_addr(&s_valid, q));

  constexpr int kShift[6] = {53, 42, 32, 21, 10, 0};
  constexpr int kWidth[6] = {11, 11, 10, 11, 11, 10};
  uint64_t prefix = 0;
  uint32_t remaining = (uint32_t)k;
  int shift = 64;
  bool done = n_valid <= (uint32_t)k;

  for (int p = 0; p < 6 && !done; ++p) {
    const int width = kWidth[p], sh = kShift[p];
    const int nb = 1 << width;
    const uint32_t mask = (uint32_t)nb - 1u;
    uint32_t* h = hist[p & 1];
    // hist[p & 1] was last read remotely in pass p-2, before every CTA
    // arrived at pass p-1's cluster barrier: safe to clear.
    for (int b = threadIdx.x; b < nb; b += kTopkThreads) h[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nloc; i += kTopkThreads) {
      const uint64_t key = keys[i];
      if (key == 0ull) continue;
      if (p == 0 || (key >> (sh + width)) == prefix) atomicAdd(&h[(uint32_t)(key >> sh) & mask], 1u);
    }
    cluster_barrier();  // every CTA's histogram of this pass is complete
    const int bpt = nb / kTopkThreads;  // 1 or 2
    uint32_t c[2] = {0, 0};
    for (int j = 0; j < bpt; ++j) {
      const int bin = nb - 1 - (threadIdx.x * bpt + j);
      for (int q = 0; q < C; ++q) c[j] += dsmem_ld(dsmem_addr(h + bin, q));
    }
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

  // Output: this CTA's selected keys, at slots reserved from CTA 0's counter.
  uint32_t mine = 0;
  for (int i = threadIdx.x; i < nloc; i += kTopkThreads) {
    const uint64_t key = keys[i];
    mine += key != 0ull && (shift == 64 || (key >> shift) >= prefix);
  }
  const uint32_t off = block_exclusive_scan(mine, warp_tot);
  __shared__ uint32_t base;
  if (threadIdx.x == kTopkThreads - 1) base = dsmem_atomic_add(dsmem_addr(&s_out, 0), off + mine);
  __syncthreads();
  uint32_t slot = base + off;
  for (int i = threadIdx.x; i < nloc; i += kTopkThreads) {
    const uint64_t key = keys[i];
    if (key == 0ull || !(shift == 64 || (key >> shift) >= prefix)) continue;
    if (slot < (uint32_t)k) {
      idx[slot] = (int)(0xFFFFFFFFu - (uint32_t)key);
      val[slot] = key_to_float((uint32_t)(key >> 32));
      if ((uint32_t)(key >> 32) == 0u) set_status(status, MISA_STATUS_BAD_INPUT);  // a NaN
    } else {
      set_status(status, MISA_STATUS_BOUNDS);  // duplicate tokens in a candidate row
    }
    ++slot;
  }
  if (rank == 0) {
    const int filled = n_valid < (uint32_t)k ? (int)n_valid : k;
    for (int j = filled + threadIdx.x; j < k; j += kTopkThreads) {
      idx[j] = -1;
      val[j] = -INFINITY;
    }
  }
  cluster_barrier();  // CTA 0's counter stays alive until every CTA has used it
}

}  // namespace

// Cluster size for a top-k over `rows` rows of at most nmax elements: a power
// of two large enough to hold a row slice in shared memory, grown while all
// rows still fit one wave of CTAs; 1 = the one-CTA-per-row kernel.
int topk_cluster_size(int rows, int64_t nmax, int sms) {
  if (rows <= 0 || rows * 2 > sms || nmax < 4096) return 1;
  const int64_t need = (nmax + kClusterCap - 1) / kClusterCap;
  int c = 1;
  while (c < need) c <<= 1;
  while (c * 2 <= kMaxCluster && rows * c * 2 <= sms) c <<= 1;  // stay within one wave
  if (c > kMaxCluster || (int64_t)c * kClusterCap < nmax) return 1;
  return c;
}

int launch_topk(const misa_problem_t& p, const float* I, int64_t ld, const int32_t* tok,
                int n_fixed, int q_lo, int q_hi, int k, int32_t* idx, float* val,
                cudaStream_t st, const int32_t* rows_list, const int* rows_count) {
  if (q_hi <= q_lo) return MISA_OK;
  const int rows = q_hi - q_lo;
  const int64_t nmax = tok ? n_fixed : p.max_seq_len;
  const int C = topk_cluster_size(rows, nmax, num_sms());
  if (C > 1) {
    const int smem = kClusterCap * (int)sizeof(uint64_t);
    int rc = set_smem_limit((const void*)topk_cluster_kernel, smem);
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: the kernel waits on the previous one first
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    ProfScope ps(rows_list ? "rescan_topk" : "topk", st);
    cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, I, ld, tok, n_fixed,
                                       p.key_offsets, p.query_offsets, p.q_pos, p.num_seqs, q_lo,
                                       k, C, idx, val, status_ptr(), rows_list, rows_count);
    return cuda_fail(e, "topk_cluster_kernel");
  }
  ProfScope ps(rows_list ? "rescan_topk" : "topk", st);
  return cuda_fail(launch_pdl(topk_kernel, dim3(q_hi - q_lo), dim3(kTopkThreads), 0, st, I, ld,
                              tok, n_fixed, p.key_offsets, p.query_offsets, p.q_pos, p.num_seqs,
                              q_lo, k, idx, val, status_ptr(), rows_list, rows_count),
                   "topk_kernel");
}

}  // namespace misa
