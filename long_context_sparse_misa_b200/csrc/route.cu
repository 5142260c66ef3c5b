// Block-pooled head router.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// gist.science summary, "Methodologie: MISA" (Lightweight Block-Pooled
// Router): per-head affinities against the mean-pooled key blocks are
// aggregated into one importance score per head, and the top-h heads are
// kept.  The aggregation the pages leave open is read as
//     r[t,h] = w[t,h] * sum_{b < M_t} ReLU(q[t,h] . Kbar_t[b])
// (each head's own indexer term on the pooled keys, summed over the blocks
// the query can see; the last visible block is the causal partial mean of
// keys floor((t+1)/B)*B .. t).  Ties go to the lower head index.
//
// One CTA per query group (same sequence); thread = (query, head) row with
// its q row in registers; pooled blocks are staged through shared memory and
// read by broadcast.  fp32 arithmetic on CUDA cores.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kChunk = 32;  // pooled blocks per shared-memory stage

__global__ void __launch_bounds__(kRouteThreads, 1)
    route_kernel(const uint16_t* __restrict__ q, const float* __restrict__ w,
                 const uint16_t* __restrict__ K, const float* __restrict__ Kbar,
                 const int64_t* __restrict__ ko, const int64_t* __restrict__ bo,
                 const int32_t* __restrict__ q_pos, const int4* __restrict__ groups,
                 const int* __restrict__ group_count, int H, int B, int m, int G,
                 int32_t* __restrict__ heads, uint16_t* __restrict__ q_r, float* __restrict__ w_r,
                 float* __restrict__ router_scores, uint32_t* status) {
  extern __shared__ __align__(16) float smem_f[];
  float* kb = smem_f;                         // [kChunk][128]
  float* part = kb + kChunk * kD;             // [G][128]
  float* rs = part + G * kD;                  // [G][H]

  const int g = blockIdx.x;
  if (g >= *group_count) return;
  const int4 grp = groups[g];
  const int seq = grp.x, qb = grp.y, nq = grp.z - grp.y;
  const int tid = threadIdx.x;
  const int qq = tid / H, h = tid - qq * H;
  const bool active = qq < nq;
  const int t = qb + qq;
  const int64_t L = ko[seq + 1] - ko[seq];
  int pos = active ? q_pos[t] : -1;
  const bool valid = active && pos >= 0 && pos < L;
  if (!valid) pos = -1;
  const int n = pos + 1;
  const int nfull = n / B;
  const int max_full = (grp.w + 1) / B;

  float qreg[kD];
  if (valid) {
    const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t)t * H + h) * kD);
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
      const uint4 v = __ldg(src + i);
      qreg[8 * i + 0] = __uint_as_float(v.x << 16);
      qreg[8 * i + 1] = __uint_as_float(v.x & 0xFFFF0000u);
      qreg[8 * i + 2] = __uint_as_float(v.y << 16);
      qreg[8 * i + 3] = __uint_as_float(v.y & 0xFFFF0000u);
      qreg[8 * i + 4] = __uint_as_float(v.z << 16);
      qreg[8 * i + 5] = __uint_as_float(v.z & 0xFFFF0000u);
      qreg[8 * i + 6] = __uint_as_float(v.w << 16);
      qreg[8 * i + 7] = __uint_as_float(v.w & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kD; ++i) qreg[i] = 0.f;
  }

  // Full blocks: ReLU(q . Kbar_b) summed over b < nfull.
  float acc = 0.f;
  const float4* kbar4 = reinterpret_cast<const float4*>(Kbar + bo[seq] * kD);
  for (int c0 = 0; c0 < max_full; c0 += kChunk) {
    const int nb = min(kChunk, max_full - c0);
    __syncthreads();
    for (int i = tid; i < nb * (kD / 4); i += kRouteThreads)
      reinterpret_cast<float4*>(kb)[i] = __ldg(kbar4 + (int64_t)c0 * (kD / 4) + i);
    __syncthreads();
    const int lim = min(nb, nfull - c0);
    for (int b = 0; b < lim; ++b) {
      const float4* row = reinterpret_cast<const float4*>(kb + b * kD);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int i = 0; i < kD / 4; i += 2) {
        const float4 a = row[i], c = row[i + 1];
        d0 = fmaf(qreg[4 * i + 0], a.x, d0);
        d0 = fmaf(qreg[4 * i + 1], a.y, d0);
        d0 = fmaf(qreg[4 * i + 2], a.z, d0);
        d0 = fmaf(qreg[4 * i + 3], a.w, d0);
        d1 = fmaf(qreg[4 * i + 4], c.x, d1);
        d1 = fmaf(qreg[4 * i + 5], c.y, d1);
        d1 = fmaf(qreg[4 * i + 6], c.z, d1);
        d1 = fmaf(qreg[4 * i + 7], c.w, d1);
      }
      acc += fmaxf(d0 + d1, 0.f);
    }
  }

  // Causal partial block of every query of the group (mean of its visible keys).
  __syncthreads();
  for (int i = tid; i < G * kD; i += kRouteThreads) part[i] = 0.f;
  __syncthreads();
  for (int item = tid; item < nq * kD; item += kRouteThreads) {
    const int qi = item / kD, dim = item - qi * kD;
    const int p2 = q_pos[qb + qi];
    if (p2 < 0 || p2 >= L) continue;
    const int f2 = (p2 + 1) / B * B;
    if (f2 == p2 + 1) continue;
    const uint16_t* col = K + (ko[seq] + f2) * kD + dim;
    float s = 0.f;
    for (int key = f2; key <= p2; ++key) s += bf16_bits_to_float(col[(int64_t)(key - f2) * kD]);
    part[qi * kD + dim] = s / (float)(p2 + 1 - f2);
  }
  __syncthreads();
  if (valid && nfull * B != n) {
    const float4* row = reinterpret_cast<const float4*>(part + qq * kD);
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < kD / 4; ++i) {
      const float4 a = row[i];
      d = fmaf(qreg[4 * i + 0], a.x, d);
      d = fmaf(qreg[4 * i + 1], a.y, d);
      d = fmaf(qreg[4 * i + 2], a.z, d);
      d = fmaf(qreg[4 * i + 3], a.w, d);
    }
    acc += fmaxf(d, 0.f);
  }

  float r = -INFINITY;
  if (valid) {
    const float wt = __ldg(w + (int64_t)t * H + h);
    r = wt * acc;
    if (router_scores) router_scores[(int64_t)t * H + h] = r;
    if (r != r) {
      set_status(status, MISA_STATUS_BAD_INPUT);
      r = -INFINITY;
    }
  }
  if (active) rs[qq * H + h] = r;
  __syncthreads();

  // Top-m by (r desc, head asc): rank of this head among the query's heads.
  if (!valid) {
    if (active && h < m) {  // invalid query: deterministic padding
      heads[(int64_t)t * m + h] = -1;
      w_r[(int64_t)t * m + h] = 0.f;
      uint4* dst = reinterpret_cast<uint4*>(q_r + ((int64_t)t * m + h) * kD);
      for (int i = 0; i < kD / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  int rank = 0;
  for (int o = 0; o < H; ++o) {
    const float ro = rs[qq * H + o];
    rank += (ro > r) || (ro == r && o < h);
  }
  if (rank < m) {
    const int64_t dst_row = (int64_t)t * m + rank;
    heads[dst_row] = h;
    w_r[dst_row] = __ldg(w + (int64_t)t * H + h);
    const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t)t * H + h) * kD);
    uint4* dst = reinterpret_cast<uint4*>(q_r + dst_row * kD);
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) dst[i] = __ldg(src + i);
  }
}

}  // namespace

int route_group_size(int H) { return H >= kRouteThreads ? 1 : kRouteThreads / H; }

int launch_route(const misa_problem_t& p, const uint16_t* q, const float* w, const uint16_t* K,
                 const float* Kbar, int m, int32_t* heads, uint16_t* q_r, float* w_r,
                 float* router_scores, const int4* groups, const int* group_count,
                 int max_groups, int G, cudaStream_t st) {
  if (max_groups <= 0) return MISA_OK;
  const int smem = (kChunk * kD + G * kD + G * p.num_heads) * (int)sizeof(float);
  int rc = set_smem_limit((const void*)route_kernel, smem);
  if (rc) return rc;
  ProfScope ps("route", st);
  route_kernel<<<max_groups, kRouteThreads, smem, st>>>(
      q, w, K, Kbar, p.key_offsets, p.block_offsets, p.q_pos, groups, group_count,
      p.num_heads, p.block, m, G, heads, q_r, w_r, router_scores, status_ptr());
  return cuda_fail(cudaGetLastError(), "route_kernel");
}

}  // namespace misa
