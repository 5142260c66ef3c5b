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
//
// Decode batches have too few query groups to fill the GPU, and each group
// scans every pooled block of a long prefix.  There the pooled blocks are
// split into contiguous ranges: one CTA per (group, range), and one per group
// for its queries' causal partial blocks, write per-slot partial sums
// (route_mma_kernel, on warp-level tensor-core MMAs), and a second launch
// adds them in range order (a fixed order, so the result does not depend on
// scheduling) and takes the top-m.  The number of ranges is taken on the
// device from the actual group count, so that the (group, range) CTAs form
// one wave.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kChunk = 32;  // pooled blocks per shared-memory stage

// One CTA per query group does everything for it (problems whose groups fill
// the GPU, or without the scratch of the split path).
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_kernel(const uint16_t* __restrict__ q, const float* __restrict__ w,
                 const uint16_t* __restrict__ K, const float* __restrict__ Kbar,
                 const int64_t* __restrict__ ko, const int64_t* __restrict__ bo,
                 const int32_t* __restrict__ q_pos, const int4* __restrict__ groups,
                 const int* __restrict__ group_count, int H, int B, int m, int G,
                 int32_t* __restrict__ heads, uint16_t* __restrict__ q_r, float* __restrict__ w_r,
                 float* __restrict__ router_scores, uint32_t* status) {
  pdl_wait_then_release();
  extern __shared__ __align__(16) float smem_f[];
  float* kb = smem_f;                         // [kChunk][128]
  float* part = kb + kChunk * kD;             // [G][128]
  float* rs = part + G * kD;                  // [G][H]

  const int count = *group_count;
  const int g = (int)blockIdx.x;
  if (g >= count) return;
  constexpr bool do_full = true, do_tail = true;
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
  if (do_full) {
    const int b_lo = 0, b_hi = max_full;
    const float4* kbar4 = reinterpret_cast<const float4*>(Kbar + bo[seq] * kD);
    for (int c0 = b_lo; c0 < b_hi; c0 += kChunk) {
      const int nb = min(kChunk, b_hi - c0);
      __syncthreads();
      for (int i = tid; i < nb * (kD / 4); i += kRouteThreads)
        reinterpret_cast<float4*>(kb)[i] = __ldg(kbar4 + (int64_t)c0 * (kD / 4) + i);
      __syncthreads();
      const int lim = min(nb, nfull - c0);
      // Two blocks at a time (independent chains); each block's dot product
      // and the order of the ReLU sums are those of the one-block loop.
      int b = 0;
      for (; b + 1 < lim; b += 2) {
        const float4* r0 = reinterpret_cast<const float4*>(kb + b * kD);
        const float4* r1 = r0 + kD / 4;
        float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
        float e0 = 0.f, e1 = 0.f, e2 = 0.f, e3 = 0.f;
#pragma unroll
        for (int i = 0; i < kD / 4; i += 2) {
          const float4 a = r0[i], c = r0[i + 1], a1 = r1[i], c1 = r1[i + 1];
          ffma2(d0, d1, qreg[4 * i + 0], qreg[4 * i + 1], a.x, a.y);
          ffma2(e0, e1, qreg[4 * i + 0], qreg[4 * i + 1], a1.x, a1.y);
          ffma2(d0, d1, qreg[4 * i + 2], qreg[4 * i + 3], a.z, a.w);
          ffma2(e0, e1, qreg[4 * i + 2], qreg[4 * i + 3], a1.z, a1.w);
          ffma2(d2, d3, qreg[4 * i + 4], qreg[4 * i + 5], c.x, c.y);
          ffma2(e2, e3, qreg[4 * i + 4], qreg[4 * i + 5], c1.x, c1.y);
          ffma2(d2, d3, qreg[4 * i + 6], qreg[4 * i + 7], c.z, c.w);
          ffma2(e2, e3, qreg[4 * i + 6], qreg[4 * i + 7], c1.z, c1.w);
        }
        acc += relu_nan((d0 + d1) + (d2 + d3));
        acc += relu_nan((e0 + e1) + (e2 + e3));
      }
      for (; b < lim; ++b) {
        const float4* row = reinterpret_cast<const float4*>(kb + b * kD);
        float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
        for (int i = 0; i < kD / 4; i += 2) {
          // packed pairs: d0 takes dims 0 mod 4 and 2 mod 4 in order, d1
          // dims 1 and 3 mod 4, d2 / d3 the same on the next four
          const float4 a = row[i], c = row[i + 1];
          ffma2(d0, d1, qreg[4 * i + 0], qreg[4 * i + 1], a.x, a.y);
          ffma2(d0, d1, qreg[4 * i + 2], qreg[4 * i + 3], a.z, a.w);
          ffma2(d2, d3, qreg[4 * i + 4], qreg[4 * i + 5], c.x, c.y);
          ffma2(d2, d3, qreg[4 * i + 6], qreg[4 * i + 7], c.z, c.w);
        }
        acc += relu_nan((d0 + d1) + (d2 + d3));
      }
    }
  }
  // Causal partial block of every query of the group (mean of its visible keys).
  if (do_tail) {
    __syncthreads();
    for (int i = tid; i < G * kD; i += kRouteThreads) part[i] = 0.f;
    __syncthreads();
    // Queries whose partial blocks start at the same key share one staging of
    // its rows: up to 64 rows (16 KB, the pooled-block stage) per round trip,
    // then one thread per (query, pair of dims) adds its keys in order.
    const uint16_t* Kseq = K + ko[seq] * kD;
    uint16_t* rows = reinterpret_cast<uint16_t*>(kb);
    constexpr int kStageRows = kChunk * kD * 4 / (kD * 2);  // 64 bf16 rows
    int qi0 = 0;
    while (qi0 < nq) {
      // block-uniform: every thread reads the same positions
      const int p0 = q_pos[qb + qi0];
      const int f0 = (p0 + 1) / B * B;
      if (p0 < 0 || p0 >= L || p0 + 1 == f0) {
        ++qi0;
        continue;
      }
      int qi1 = qi0 + 1, cmax = p0 + 1 - f0;
      while (qi1 < nq && qi1 - qi0 < kRouteThreads / (kD / 2)) {  // <= 4 queries a pass
        const int p1 = q_pos[qb + qi1];
        if (p1 < 0 || p1 >= L || (p1 + 1) / B * B != f0) break;
        cmax = max(cmax, p1 + 1 - f0);
        ++qi1;
      }
      const int item = tid;  // (query qi0 + item / 64, dims 2*(item % 64) and +1)
      const int qi = qi0 + item / (kD / 2), dp = item % (kD / 2);
      int cnt = 0;
      if (qi < qi1) {
        const int p2 = q_pos[qb + qi];
        cnt = p2 + 1 - f0;  // 0 when this query's block is complete
        if (cnt < 0) cnt = 0;
      }
      float s0 = 0.f, s1 = 0.f;
      for (int c0 = 0; c0 < cmax; c0 += kStageRows) {
        const int nr = min(kStageRows, cmax - c0);
        __syncthreads();
        const uint4* src = reinterpret_cast<const uint4*>(Kseq + (int64_t)(f0 + c0) * kD);
        for (int i = tid; i < nr * (kD / 8); i += kRouteThreads)
          reinterpret_cast<uint4*>(rows)[i] = __ldg(src + i);
        __syncthreads();
        const uint32_t* col = reinterpret_cast<const uint32_t*>(rows) + dp;
        const int lim = min(cnt - c0, nr);
        for (int key = 0; key < lim; ++key) {
          const uint32_t v = col[key * (kD / 2)];
          s0 += __uint_as_float(v << 16);
          s1 += __uint_as_float(v & 0xFFFF0000u);
        }
      }
      if (cnt > 0) {
        part[qi * kD + 2 * dp] = s0 / (float)cnt;
        part[qi * kD + 2 * dp + 1] = s1 / (float)cnt;
      }
      qi0 = qi1;
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
      acc += relu_nan(d);
    }
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

// ---------------------------------------------------------------- ranges on tensor cores
// The ranges of a decode batch on warp-level tensor-core MMAs (mma.sync
// m16n8k16, bf16 inputs, fp32 accumulation).  CTA (group, y): y < ns sums
// range y of the full pooled blocks, y == ns the queries' causal partial
// blocks.  Each warp takes 16 (query, head) slots (A = their q rows, exact in
// bf16) against 8 pooled blocks at a time (B = Kbar as a bf16 pair hi + lo,
// hi + lo ~= Kbar to about 2^-16 relative, so q . Kbar = q . hi + q . lo).
// A CUDA-core loop with one thread per slot is bound by shared-memory operand
// traffic (every thread reads every pooled row); the MMA reads each row once
// per warp.  The ReLU sum over the range's blocks is taken on the
// accumulator fragments and added across the 4 lanes of a row at the end; the
// partial blocks are one more MMA against the group's partial means.  Each
// CTA stores one sum per slot; the group's last CTA adds them in range order
// and ranks the heads.
constexpr int kMmaBlock = 512;              // 16 warps x 16 slots = kRouteThreads
constexpr int kRowW = kD / 2 + 4;           // words per staged row: 64 bf16 pairs + 4 pad

__device__ __forceinline__ uint32_t bf16_pair(float a, float b) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
}

// hi / lo bf16 pairs of two fp32 values: hi = bf16(x), lo = bf16(x - hi).
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
  const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
  hi = bf16_pair(h0, h1);
  lo = bf16_pair(x0 - h0, x1 - h1);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// C = A (16 slots x 128 dims, fragments a[kk]) x B (128 dims x 8 rows of the
// staged hi / lo arrays, starting at row r0), both halves of the pair.
__device__ __forceinline__ void mma_rows(float (&c)[4], const uint32_t (&a)[kD / 16][4],
                                         const uint32_t* hi, const uint32_t* lo, int r0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  c[0] = c[1] = c[2] = c[3] = 0.f;
  const uint32_t* h = hi + (r0 + g) * kRowW + t;
  const uint32_t* l = lo + (r0 + g) * kRowW + t;
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    mma_bf16_16816(c, a[kk], h[8 * kk], h[8 * kk + 4]);
    mma_bf16_16816(c, a[kk], l[8 * kk], l[8 * kk + 4]);
  }
}

__global__ void __launch_bounds__(kMmaBlock, 1)
    route_mma_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ K,
                     const float* __restrict__ Kbar, const int64_t* __restrict__ ko,
                     const int64_t* __restrict__ bo, const int32_t* __restrict__ q_pos,
                     const int4* __restrict__ groups, const int* __restrict__ group_count,
                     int H, int B, int G, int nsplit_max, int sms, float* __restrict__ partial,
                     int* __restrict__ done, const float* __restrict__ w, int m,
                     int32_t* __restrict__ heads, uint16_t* __restrict__ q_r,
                     float* __restrict__ w_r, float* __restrict__ router_scores,
                     uint32_t* status) {
  pdl_wait_then_release();
  extern __shared__ __align__(16) uint32_t smem_w[];
  uint32_t* khi = smem_w;                          // [kChunk][kRowW]
  uint32_t* klo = khi + kChunk * kRowW;            // [kChunk][kRowW]
  float* part = reinterpret_cast<float*>(klo + kChunk * kRowW);  // [G][128]
  const int G8 = (G + 7) / 8 * 8;
  uint32_t* phi = reinterpret_cast<uint32_t*>(part + G * kD);     // [G8][kRowW]
  uint32_t* plo = phi + G8 * kRowW;                               // [G8][kRowW]

  const int count = *group_count;
  const int ns = max(1, min(nsplit_max, sms / max(count, 1) - 1));
  const int g_ = (int)blockIdx.x / (ns + 1);
  if (g_ >= count) return;
  const int y = (int)blockIdx.x - g_ * (ns + 1);
  const int4 grp = groups[g_];
  const int seq = grp.x, qb = grp.y, nq = grp.z - grp.y;
  const int64_t L = ko[seq + 1] - ko[seq];
  const int max_full = (grp.w + 1) / B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gi = lane >> 2, ti = lane & 3;

  // This lane's two slots (rows gi and gi + 8 of the warp's 16) and their
  // queries' full-block counts.
  const int sA = warp * 16 + gi, sB = sA + 8;
  int nA = 0, nB = 0, qA = -1, qB = -1;
  {
    const int a = sA / H, b = sB / H;
    if (a < nq) {
      const int p = q_pos[qb + a];
      if (p >= 0 && p < L) { nA = p + 1; qA = a; }
    }
    if (b < nq) {
      const int p = q_pos[qb + b];
      if (p >= 0 && p < L) { nB = p + 1; qB = b; }
    }
  }
  const int fA = nA / B, fB = nB / B;  // full blocks of the two slots' queries
  const bool warp_active = warp * 16 < nq * H;
  // A fragments: q rows of the warp's slots (zero rows for invalid slots).
  uint32_t afr[kD / 16][4];
  {
    const uint32_t* rowA =
        qA >= 0 ? reinterpret_cast<const uint32_t*>(q + ((int64_t)(qb + qA) * H + sA % H) * kD)
                : nullptr;
    const uint32_t* rowB =
        qB >= 0 ? reinterpret_cast<const uint32_t*>(q + ((int64_t)(qb + qB) * H + sB % H) * kD)
                : nullptr;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      afr[kk][0] = rowA ? __ldg(rowA + 8 * kk + ti) : 0u;
      afr[kk][1] = rowB ? __ldg(rowB + 8 * kk + ti) : 0u;
      afr[kk][2] = rowA ? __ldg(rowA + 8 * kk + 4 + ti) : 0u;
      afr[kk][3] = rowB ? __ldg(rowB + 8 * kk + 4 + ti) : 0u;
    }
  }
  float accA = 0.f, accB = 0.f;  // this lane's share of its two slots' sums

  if (y < ns) {
    // ---- range y of the full blocks
    const int range = (max_full + ns - 1) / ns;
    const int b_lo = y * range, b_hi = min(max_full, b_lo + range);
    const float2* kbar2 = reinterpret_cast<const float2*>(Kbar + bo[seq] * kD);
    for (int c0 = b_lo; c0 < b_hi; c0 += kChunk) {
      const int nb = min(kChunk, b_hi - c0);
      __syncthreads();
      for (int i = tid; i < kChunk * (kD / 2); i += kMmaBlock) {
        const int r = i / (kD / 2), w = i - r * (kD / 2);
        uint32_t hv = 0u, lv = 0u;
        if (r < nb) {
          const float2 x = __ldg(kbar2 + (int64_t)(c0 + r) * (kD / 2) + w);
          split_pair(x.x, x.y, hv, lv);
        }
        khi[r * kRowW + w] = hv;
        klo[r * kRowW + w] = lv;
      }
      __syncthreads();
      if (warp_active) {
        for (int nt = 0; nt * 8 < nb; ++nt) {
          float c[4];
          mma_rows(c, afr, khi, klo, nt * 8);
          const int b0 = c0 + nt * 8 + 2 * ti;  // blocks of columns 2ti, 2ti + 1
          accA += (b0 < fA ? relu_nan(c[0]) : 0.f) + (b0 + 1 < fA ? relu_nan(c[1]) : 0.f);
          accB += (b0 < fB ? relu_nan(c[2]) : 0.f) + (b0 + 1 < fB ? relu_nan(c[3]) : 0.f);
        }
      }
    }
  } else {
    // ---- the causal partial block of every query of the group
    for (int i = tid; i < G * kD; i += kMmaBlock) part[i] = 0.f;
    __syncthreads();
    // Queries whose partial blocks start at the same key share one staging
    // of its rows (64 rows per round trip, in the pooled-block stage); one
    // thread per (query, pair of dims) adds its keys in order.
    const uint16_t* Kseq = K + ko[seq] * kD;
    uint16_t* rows = reinterpret_cast<uint16_t*>(khi);
    constexpr int kStageRows = 64;  // 64 bf16 rows = 16 KB <= the two staged arrays
    int qi0 = 0;
    while (qi0 < nq) {
      const int p0 = q_pos[qb + qi0];  // block-uniform
      const int f0 = (p0 + 1) / B * B;
      if (p0 < 0 || p0 >= L || p0 + 1 == f0) {
        ++qi0;
        continue;
      }
      int qi1 = qi0 + 1, cmax = p0 + 1 - f0;
      while (qi1 < nq && qi1 - qi0 < kMmaBlock / (kD / 2)) {
        const int p1 = q_pos[qb + qi1];
        if (p1 < 0 || p1 >= L || (p1 + 1) / B * B != f0) break;
        cmax = max(cmax, p1 + 1 - f0);
        ++qi1;
      }
      const int qi = qi0 + tid / (kD / 2), dp = tid % (kD / 2);
      int cnt = 0;
      if (qi < qi1) cnt = max(0, q_pos[qb + qi] + 1 - f0);
      float s0 = 0.f, s1 = 0.f;
      for (int c0 = 0; c0 < cmax; c0 += kStageRows) {
        const int nr = min(kStageRows, cmax - c0);
        __syncthreads();
        const uint4* src = reinterpret_cast<const uint4*>(Kseq + (int64_t)(f0 + c0) * kD);
        for (int i = tid; i < nr * (kD / 8); i += kMmaBlock)
          reinterpret_cast<uint4*>(rows)[i] = __ldg(src + i);
        __syncthreads();
        const uint32_t* col = reinterpret_cast<const uint32_t*>(rows) + dp;
        const int lim = min(cnt - c0, nr);
        for (int key = 0; key < lim; ++key) {
          const uint32_t v = col[key * (kD / 2)];
          s0 += __uint_as_float(v << 16);
          s1 += __uint_as_float(v & 0xFFFF0000u);
        }
      }
      if (cnt > 0) {
        part[qi * kD + 2 * dp] = s0 / (float)cnt;
        part[qi * kD + 2 * dp + 1] = s1 / (float)cnt;
      }
      qi0 = qi1;
    }
    __syncthreads();
    for (int i = tid; i < G8 * (kD / 2); i += kMmaBlock) {
      const int r = i / (kD / 2), w = i - r * (kD / 2);
      uint32_t hv = 0u, lv = 0u;
      if (r < G) split_pair(part[r * kD + 2 * w], part[r * kD + 2 * w + 1], hv, lv);
      phi[r * kRowW + w] = hv;
      plo[r * kRowW + w] = lv;
    }
    __syncthreads();
    // C[slot, query row]: each slot takes the column of its own query, if
    // that query has a partial block.
    if (warp_active) {
      for (int nt = 0; nt * 8 < G; ++nt) {
        float c[4];
        mma_rows(c, afr, phi, plo, nt * 8);
        const int col0 = nt * 8 + 2 * ti;
        const bool pa = qA >= 0 && fA * B != nA, pb = qB >= 0 && fB * B != nB;
        if (pa && qA == col0) accA += relu_nan(c[0]);
        if (pa && qA == col0 + 1) accA += relu_nan(c[1]);
        if (pb && qB == col0) accB += relu_nan(c[2]);
        if (pb && qB == col0 + 1) accB += relu_nan(c[3]);
      }
    }
  }

  // Add the 4 lanes of each row; lane ti == 0 stores the slot sums.
  accA += __shfl_xor_sync(0xffffffffu, accA, 1);
  accA += __shfl_xor_sync(0xffffffffu, accA, 2);
  accB += __shfl_xor_sync(0xffffffffu, accB, 1);
  accB += __shfl_xor_sync(0xffffffffu, accB, 2);
  if (ti == 0) {
    const int64_t base = ((int64_t)g_ * (nsplit_max + 1) + y) * kRouteThreads;
    partial[base + sA] = accA;
    partial[base + sB] = accB;
  }

  // The last of the group's ns + 1 CTAs to get here adds the stored sums in
  // range order and ranks the group's heads (the counters are cleared by
  // the plan launch before this one).
  __shared__ int s_last;
  __threadfence();  // this CTA's sums are visible before it counts itself
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&done[g_], 1) == ns;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float* rs = reinterpret_cast<float*>(plo + G8 * kRowW);  // [G][H] router scores
  const int slot = tid, qq = slot / H, h = slot - qq * H;
  const bool active = slot < kRouteThreads && qq < nq;
  const int t = qb + qq;
  int pos = active ? q_pos[t] : -1;
  const bool valid = active && pos >= 0 && pos < L;
  float r = -INFINITY;
  if (valid) {
    float acc = 0.f;
    const float* pp = partial + (int64_t)g_ * (nsplit_max + 1) * kRouteThreads + slot;
    for (int j0 = 0; j0 <= ns; j0 += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = j0 + u <= ns ? __ldcg(pp + (int64_t)(j0 + u) * kRouteThreads) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (j0 + u <= ns) acc += v[u];
    }
    r = __ldg(w + (int64_t)t * H + h) * acc;
    if (router_scores) router_scores[(int64_t)t * H + h] = r;
    if (r != r) {
      set_status(status, MISA_STATUS_BAD_INPUT);
      r = -INFINITY;
    }
  }
  if (active) rs[qq * H + h] = r;
  __syncthreads();
  if (!active) return;
  // Top-m by (r desc, head asc): rank of this head among the query's heads.
  if (!valid) {
    if (h < m) {  // invalid query: deterministic padding
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

// Most ranges of pooled blocks per group (the device takes fewer when there
// are more groups): split only when the groups alone leave SMs idle, into
// ranges of about 16 blocks or more.
int route_split_count(const misa_problem_t& p, int max_groups, int sms) {
  if (max_groups <= 0 || max_groups >= sms) return 1;
  const int max_blocks = (int)(p.max_seq_len / p.block);
  const int by_work = (max_blocks + 15) / 16;
  const int n = by_work < sms ? by_work : sms;
  return n < 2 ? 1 : n;
}

// Per-slot partial sums [max_groups][nsplit + 1][256] fp32, then one
// completion counter per group.
size_t route_split_bytes(int max_groups, int nsplit) {
  return nsplit <= 1 ? 0
                     : (size_t)max_groups * (nsplit + 1) * kRouteThreads * sizeof(float) +
                           (size_t)max_groups * sizeof(int);
}

int* route_split_counters(float* partial, int max_groups, int nsplit) {
  return reinterpret_cast<int*>(partial + (size_t)max_groups * (nsplit + 1) * kRouteThreads);
}

int launch_route(const misa_problem_t& p, const uint16_t* q, const float* w, const uint16_t* K,
                 const float* Kbar, int m, int32_t* heads, uint16_t* q_r, float* w_r,
                 float* router_scores, const int4* groups, const int* group_count,
                 int max_groups, int G, int nsplit, float* partial, cudaStream_t st) {
  if (max_groups <= 0) return MISA_OK;
  const int smem = (kChunk * kD + G * kD + G * p.num_heads) * (int)sizeof(float);
  const int sms = num_sms();
  int rc;
  if (nsplit <= 1 || !partial) {
    if ((rc = set_smem_limit((const void*)route_kernel, smem))) return rc;
    ProfScope ps("route", st);
    return cuda_fail(launch_pdl(route_kernel, dim3(max_groups), dim3(kRouteThreads), smem, st,
                                q, w, K, Kbar, p.key_offsets, p.block_offsets, p.q_pos, groups,
                                group_count, p.num_heads, p.block, m, G, heads, q_r, w_r,
                                router_scores, status_ptr()),
                     "route_kernel");
  }
  // One CTA per (group, range) and one per group for its partial blocks: the
  // device uses the first count * (ns + 1) of the grid, at most
  // max(sms, 2 * count) since ns + 1 <= max(2, sms / count).  The last CTA
  // of each group to finish ranks its heads.
  ProfScope ps("route", st);
  const int ranged = (int)std::min<int64_t>((int64_t)max_groups * (nsplit + 1),
                                            std::max(sms, 2 * max_groups));
  const int G8 = (G + 7) / 8 * 8;
  const int msmem = (2 * kChunk * kRowW + 2 * G8 * kRowW) * (int)sizeof(uint32_t) +
                    G * kD * (int)sizeof(float) + kRouteThreads * (int)sizeof(float);
  if ((rc = set_smem_limit((const void*)route_mma_kernel, msmem))) return rc;
  return cuda_fail(launch_pdl(route_mma_kernel, dim3(ranged), dim3(kMmaBlock), msmem, st, q, K,
                              Kbar, p.key_offsets, p.block_offsets, p.q_pos, groups,
                              group_count, p.num_heads, p.block, G, nsplit, sms, partial,
                              route_split_counters(partial, max_groups, nsplit), w, m, heads,
                              q_r, w_r, router_scores, status_ptr()),
                   "route_mma_kernel");
}

}  // namespace misa
