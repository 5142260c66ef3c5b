// Block-pooled head router on tcgen05 tensor cores.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// gist.science summary, "Methodologie: MISA" (Lightweight Block-Pooled
// Router): per-head affinities against the mean-pooled key blocks,
// aggregated into one importance score per head; the top-h heads are kept.
// Reading of the aggregation (as in route.cu):
//     r[t,h] = w[t,h] * sum_{b < M_t} ReLU(q[t,h] . Kbar_t[b])
// over the floor((t+1)/B) full blocks plus the causal partial block.
//
// In prefill this is a GEMM: rows (t,h) of q against the pooled keys, then a
// ReLU-sum along the block axis.  One CTA takes a group of G queries (G*H <=
// 256 rows, same sequence): A = its q rows (resident, 128-byte swizzle), B =
// 256-block chunks of the pooled keys streamed by TMA, and two TMEM
// accumulators of 128 rows x 256 blocks (all 512 columns; N = 256 keeps the
// tensor pipe busier than four 128-column accumulators of 512 rows, measured
// 3% faster at 128K).  The fp32 pooled
// keys enter as a bf16 pair hi = bf16(Kbar), lo = bf16(Kbar - hi)
// accumulated into the same fp32 accumulator, which keeps ~16 mantissa bits
// of the pooled keys.  Eight epilogue warps, two per TMEM lane quarter:
// each owns one row of every accumulator per lane and half of each chunk's
// columns, so the block-axis ReLU-sum is inside the thread (the two halves
// are added in shared memory); an accumulator is released as soon as both
// halves are copied to registers.  The causal partial block
// of every key position (the running mean of its block up to that key) is
// computed beforehand by one warp per pooled block; the epilogue stages the
// group's rows of it (again as a bf16 hi + lo pair, 128-byte swizzle) and
// the MMA warp runs one more round of N = 16 columns, column j = query j's
// partial block, so that each (query, head) row's partial-block affinity is
// the accumulator element in its own query's column.  Persistent: one CTA
// per SM walks its groups; the next
// group's q rows load as soon as the current group's MMAs are done, and its
// MMAs start while the epilogue still ranks the current group's heads.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kEpiWarps = 8;           // two per TMEM lane quarter, one per half of a chunk
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kRows = 256;             // q rows per CTA (2 accumulators of 128)
constexpr int kChunk = 256;            // pooled blocks per chunk (accumulator columns)
constexpr int kStages = 2;             // each stage: one of hi/lo for one chunk (2048 MMA cycles)
constexpr int kStageBytes = kChunk * kD * 2;          // 32 KB
constexpr int kHalfBytes = kStageBytes / 2;
constexpr int kQHalfBytes = kRows * 128;              // 64 KB per 64-dim half
constexpr int kQBytes = 2 * kQHalfBytes;
constexpr int kMaxG = 16;                             // queries per group
constexpr int kPmHalfBytes = kMaxG * 128;             // partial-block rows, one 64-dim half
constexpr int kPmBytes = 2 * 2 * kPmHalfBytes;        // hi and lo, two halves each
constexpr int kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kPmBytes + kRows * 4 /*r*/ +
                           2 * kRows * 4 /*racc*/ + kMaxG * 4 /*pos*/ + 16 * 8 + 16;

struct Smem {
  uint8_t* q;
  uint8_t* k;
  uint8_t* pm;  // [hi, lo][2 halves][kMaxG rows][128 B]: running block means at the queries
  float* r;     // [kRows] partial-block affinity, then router score, of each row
  float* racc;  // [2][kRows] block-axis ReLU sums of each half of the chunks
  int* pos;     // [kMaxG] query positions of the group (-1: none)
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;  // [4]
  uint64_t* qfull;
  uint64_t* qempty;
  uint64_t* pmfull;
  uint64_t* drain;
  uint32_t* tmem_slot;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.q = p;
  s.k = p + kQBytes;
  s.pm = s.k + kStages * kStageBytes;  // 1024-byte aligned
  s.r = reinterpret_cast<float*>(s.pm + kPmBytes);
  s.racc = s.r + kRows;
  s.pos = reinterpret_cast<int*>(s.racc + 2 * kRows);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.pos + kMaxG);  // 8-byte aligned
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 1;
  s.qfull = s.tempty + 4;
  s.qempty = s.qfull + 1;
  s.pmfull = s.qempty + 1;
  s.drain = s.pmfull + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.drain + 1);
  s.abort = reinterpret_cast<int*>(s.tmem_slot + 1);
  return s;
}

// Kbar (fp32) -> hi, lo (bf16) with hi + lo ~= Kbar.
__global__ void split_kbar_kernel(const float* __restrict__ Kbar, int64_t n,
                                  __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float x = Kbar[i];
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  hi[i] = h;
  lo[i] = __float2bfloat16_rn(x - __bfloat162float(h));
}

// Running block means of the keys: Pm[key] = mean of the keys from the start
// of key's pooled block up to key, summed in key order (fp32).  One warp per
// pooled block; each lane owns 4 of the 128 dims; 8 keys' loads in flight.
__global__ void __launch_bounds__(256)
    prefix_means_kernel(const uint16_t* __restrict__ K, const int64_t* __restrict__ ko,
                        const int64_t* __restrict__ bo, int S, int B, int64_t total_blocks,
                        float* __restrict__ Pm) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= total_blocks) return;
  const int s = upper_segment<int64_t>(bo, S, row);
  const int64_t k0 = ko[s] + (row - bo[s]) * B;
  const int64_t k1 = min(k0 + (int64_t)B, ko[s + 1]);
  const uint2* src = reinterpret_cast<const uint2*>(K) + lane;
  float4* dst = reinterpret_cast<float4*>(Pm) + lane;
  float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
  for (int64_t kb = k0; kb < k1; kb += 8) {
    uint2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = kb + u < k1 ? __ldg(src + (kb + u) * (kD / 4)) : make_uint2(0u, 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t key = kb + u;
      if (key >= k1) break;
      r0 += __uint_as_float(v[u].x << 16);
      r1 += __uint_as_float(v[u].x & 0xFFFF0000u);
      r2 += __uint_as_float(v[u].y << 16);
      r3 += __uint_as_float(v[u].y & 0xFFFF0000u);
      const float cnt = (float)(key - k0 + 1);
      dst[key * (kD / 4)] = make_float4(r0 / cnt, r1 / cnt, r2 / cnt, r3 / cnt);
    }
  }
}

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap himap,
                    const __grid_constant__ CUtensorMap lomap, const uint16_t* __restrict__ q,
                    const float* __restrict__ w, const uint16_t* __restrict__ K,
                    const int64_t* __restrict__ ko, const int64_t* __restrict__ bo,
                    const int32_t* __restrict__ q_pos, const int4* __restrict__ groups,
                    const int* __restrict__ group_count, const float* __restrict__ Pm, int B,
                    int m,
                    int32_t* __restrict__ heads, uint16_t* __restrict__ q_r,
                    float* __restrict__ w_r, float* __restrict__ router_scores,
                    uint32_t* status) {
  constexpr int G = (kRows / H) < kMaxG ? (kRows / H) : kMaxG;
  constexpr int ROWS = G * H;                       // rows used (<= kRows)
  constexpr int NSUB = (ROWS + 127) / 128;          // accumulators used
  constexpr uint32_t kQTx = 2u * ((ROWS + 31) / 32) * 32u * 128u;
  extern __shared__ uint8_t smem_raw[];

  // Persistent: CTA b takes groups b, b + gridDim.x, ...; every role walks
  // the same sequence and skips the same groups (no valid query).
  const int count = *group_count;
  if ((int)blockIdx.x >= count) return;

  Smem s = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(s.tfull, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&s.tempty[i], kEpiWarps);
    mbar_init(s.qfull, 1);
    mbar_init(s.qempty, 1);
    mbar_init(s.pmfull, kEpiWarps);
    mbar_init(s.drain, 1);
    *s.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&himap);
      tma_prefetch_desc(&lomap);
      int it = 0, gl = 0;
      bool ok = true;
      for (int gs = blockIdx.x; ok && gs < count; gs += gridDim.x) {
        const int4 grp = groups[gs];
        if (grp.w < 0 || grp.z <= grp.y) continue;
        const int64_t blk0 = bo[grp.x];
        const int nchunks = ((grp.w + 1) / B + kChunk - 1) / kChunk;
        // The q rows are replaced once the previous group's MMAs are done.
        if (!(ok = mbar_wait(s.qempty, (gl & 1) ^ 1, s.abort, status))) break;
        mbar_arrive_expect_tx(s.qfull, kQTx);
        for (int h = 0; h < 2; ++h)
          for (int r0 = 0; r0 < ROWS; r0 += 32)
            tma_load_2d(&qmap, s.qfull, s.q + h * kQHalfBytes + r0 * 128, h * 64,
                        grp.y * H + r0);
        ++gl;
        for (int c = 0; ok && c < nchunks; ++c) {
          for (int part = 0; part < 2; ++part, ++it) {
            const int st = it % kStages;
            if (!(ok = mbar_wait(&s.empty[st], ((it / kStages) & 1) ^ 1, s.abort, status))) break;
            mbar_arrive_expect_tx(&s.full[st], kStageBytes);
            const CUtensorMap* mp = part == 0 ? &himap : &lomap;
            const int32_t row = (int32_t)(blk0 + (int64_t)c * kChunk);
            uint8_t* dst = s.k + st * kStageBytes;
            tma_load_2d(mp, &s.full[st], dst, 0, row);
            tma_load_2d(mp, &s.full[st], dst + kHalfBytes, 64, row);
          }
        }
      }
      for (int i = max(0, it - kStages); i < it; ++i)
        mbar_wait(&s.full[i % kStages], (i / kStages) & 1, s.abort, status, kDrainCycles, true);
      if (gl > 0) mbar_wait(s.qfull, (gl - 1) & 1, s.abort, status, kDrainCycles, true);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, kChunk);
      const uint32_t q_addr = smem_u32(s.q);
      int it = 0, cc = 0, gl = 0;
      bool ok = true;
      for (int gs = blockIdx.x; ok && gs < count; gs += gridDim.x) {
        const int4 grp = groups[gs];
        if (grp.w < 0 || grp.z <= grp.y) continue;
        const int nchunks = ((grp.w + 1) / B + kChunk - 1) / kChunk;
        if (!(ok = mbar_wait(s.qfull, gl & 1, s.abort, status))) break;
        tc_fence_after();
        for (int c = 0; ok && c < nchunks; ++c, ++cc) {
          for (int part = 0; ok && part < 2; ++part, ++it) {
            const int st = it % kStages;
            if (!(ok = mbar_wait(&s.full[st], (it / kStages) & 1, s.abort, status))) break;
            tc_fence_after();
            const uint32_t k_addr = smem_u32(s.k + st * kStageBytes);
#pragma unroll
            for (int sub = 0; sub < NSUB; ++sub) {
              // accumulator `sub` is free once the epilogue has read chunk cc-1
              if (part == 0 &&
                  !(ok = mbar_wait(&s.tempty[sub], (cc & 1) ^ 1, s.abort, status)))
                break;
              if (part == 0) tc_fence_after();
              const uint32_t d = tmem_base + sub * kChunk;
#pragma unroll
              for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t off = (kk & 3) * 32;
                const uint64_t a = sw128_kmajor_desc(q_addr + (kk >> 2) * kQHalfBytes +
                                                     sub * 128 * 128 + off);
                const uint64_t b = sw128_kmajor_desc(k_addr + (kk >> 2) * kHalfBytes + off);
                umma_bf16(d, a, b, idesc, (part > 0 || kk > 0) ? 1u : 0u);
              }
            }
            if (!ok) break;
            umma_commit(&s.empty[st]);
          }
          if (ok) umma_commit(s.tfull);
        }
        // Partial blocks: N = 16 columns (query j's running block mean, hi
        // then lo) into the first columns of every accumulator.
        if (ok && (ok = mbar_wait(s.pmfull, gl & 1, s.abort, status))) {
          tc_fence_after();
          const uint32_t pm_addr = smem_u32(s.pm);
          const uint32_t idesc16 = idesc_bf16_f32(128, kMaxG);
#pragma unroll
          for (int sub = 0; sub < NSUB; ++sub) {
            if (!(ok = mbar_wait(&s.tempty[sub], (cc & 1) ^ 1, s.abort, status))) break;
            tc_fence_after();
            const uint32_t d = tmem_base + sub * kChunk;
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
              for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t off = (kk & 3) * 32;
                const uint64_t a = sw128_kmajor_desc(q_addr + (kk >> 2) * kQHalfBytes +
                                                     sub * 128 * 128 + off);
                const uint64_t b = sw128_kmajor_desc(pm_addr + part * 2 * kPmHalfBytes +
                                                     (kk >> 2) * kPmHalfBytes + off);
                umma_bf16(d, a, b, idesc16, (part > 0 || kk > 0) ? 1u : 0u);
              }
          }
          if (ok) umma_commit(s.tfull);
          ++cc;
        }
        umma_commit(s.qempty);  // q rows free once this group's MMAs are done
        ++gl;
      }
      umma_commit(s.drain);
      mbar_wait(s.drain, 0, s.abort, status, kDrainCycles, true);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp e = warp - 2: TMEM lane quarter warp % 4, columns ch*128 ..
    // ch*128+127 of every 256-block chunk (ch = e / 4), read 64 at a time;
    // each thread sums the ReLU of its row's visible columns, and the two
    // halves are added in shared memory.
    const int et = threadIdx.x - 64;            // 0..kEpiThreads-1
    const int quarter = warp & 3;
    const int ch = (warp - 2) >> 2;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int cc = 0;
    bool ok = true;
    for (int gs = blockIdx.x; ok && gs < count; gs += gridDim.x) {
      const int4 grp = groups[gs];
      const int seq = grp.x, qb = grp.y, nq = grp.z - grp.y;
      if (grp.w < 0 || nq <= 0) {
        // no valid query: deterministic padding for every row of the group
        for (int i = et; i < nq * m; i += kEpiThreads) {
          heads[(int64_t)qb * m + i] = -1;
          w_r[(int64_t)qb * m + i] = 0.f;
        }
        for (int i = et; i < nq * m * (kD / 8); i += kEpiThreads)
          reinterpret_cast<uint4*>(q_r + (int64_t)qb * m * kD)[i] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const int64_t L = ko[seq + 1] - ko[seq];
      const int nchunks = ((grp.w + 1) / B + kChunk - 1) / kChunk;
      if (et < kMaxG) {
        int p = -1;
        if (et < nq) {
          p = q_pos[qb + et];
          if (p < 0 || p >= L) p = -1;
        }
        s.pos[et] = p;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      // The queries' running block means (partial block) as the B operand of
      // the partial round: row j = query j, a bf16 hi + lo pair of the fp32
      // mean, 128-byte swizzle (16-byte chunk c of row j at chunk c ^ (j & 7));
      // zero rows for queries without a partial block.  One thread per
      // (row, 8 dims).
      for (int i = et; i < kMaxG * (kD / 8); i += kEpiThreads) {
        const int j = i / (kD / 8), c = i - j * (kD / 8), half = c >> 3, c8 = c & 7;
        const int p = s.pos[j];
        float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
        if (p >= 0 && (p + 1) % B != 0) {
          const float4* src = reinterpret_cast<const float4*>(Pm + (ko[seq] + p) * kD) + 2 * c;
          x0 = __ldg(src);
          x1 = __ldg(src + 1);
        }
        const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * e]);
          const __nv_bfloat16 h1 = __float2bfloat16_rn(x[2 * e + 1]);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * e] - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(x[2 * e + 1] - __bfloat162float(h1));
          hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int off = half * kPmHalfBytes + j * 128 + ((c8 ^ (j & 7)) << 4);
        *reinterpret_cast<uint4*>(s.pm + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(s.pm + 2 * kPmHalfBytes + off) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      fence_proxy_async_smem();  // visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(s.pmfull);

      // Block-axis ReLU sums: this thread owns row sub*128 + quarter*32 + lane
      // of every accumulator, columns ch*128 .. ch*128+127 of each chunk.
      float acc[NSUB];
      int lim[NSUB];
#pragma unroll
      for (int sub = 0; sub < NSUB; ++sub) {
        acc[sub] = 0.f;
        const int row = sub * 128 + quarter * 32 + lane;
        const int qi = row / H;
        const int p = (row < ROWS && qi < nq) ? s.pos[qi] : -1;
        lim[sub] = (p + 1) / B - ch * (kChunk / 2);  // full blocks visible, from this half's first column
      }
      for (int c = 0; c < nchunks && ok; ++c, ++cc) {
        if (!(ok = warp_wait(s.tfull, cc & 1, s.abort, status))) break;
        tc_fence_after();
#pragma unroll
        for (int sub = 0; sub < NSUB; ++sub) {
          for (int hh = 0; hh < 2; ++hh) {
            float v[2][32];
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tmem_ld32(lane_addr + sub * kChunk + ch * (kChunk / 2) + hh * 64 + j * 32, v[j]);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 2; ++j) reg_fence32(v[j]);
            if (hh == 1) {  // this warp's columns of accumulator `sub` are in registers
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&s.tempty[sub]);
            }
            const int nvis = lim[sub] - c * kChunk - hh * 64;  // visible of these 64 columns
            if (nvis >= 64) {
              float a0 = 0.f, a1 = 0.f;
#pragma unroll
              for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int x = 0; x < 32; x += 2) {
                  a0 += relu_nan(v[j][x]);
                  a1 += relu_nan(v[j][x + 1]);
                }
              acc[sub] += a0 + a1;
            } else if (nvis > 0) {
              float a0 = 0.f;
#pragma unroll
              for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int x = 0; x < 32; ++x)
                  if (j * 32 + x < nvis) a0 += relu_nan(v[j][x]);
              acc[sub] += a0;
            }
          }
        }
      }
      if (!ok) break;
      // Partial round: row (query qi, head h) takes column qi.
      if (!(ok = warp_wait(s.tfull, cc & 1, s.abort, status))) break;
      tc_fence_after();
#pragma unroll
      for (int sub = 0; sub < NSUB; ++sub) {
        float v[16];
        if (ch == 0) {
          tmem_ld16(lane_addr + sub * kChunk, v);
          tmem_wait_ld();
          reg_fence16(v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tempty[sub]);
        const int row = sub * 128 + quarter * 32 + lane;
        if (ch == 0 && row < ROWS) {
          const int qi = row / H;
          float dp = 0.f;
#pragma unroll
          for (int j = 0; j < kMaxG; ++j) dp = j == qi ? v[j] : dp;
          s.r[row] = dp;
        }
      }
      ++cc;
#pragma unroll
      for (int sub = 0; sub < NSUB; ++sub) {
        const int row = sub * 128 + quarter * 32 + lane;
        if (row < ROWS) s.racc[ch * kRows + row] = acc[sub];
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");  // s.r (partial), s.racc complete

      for (int row = et; row < ROWS; row += kEpiThreads) {
        const int qi = row / H, h = row - qi * H;
        float r = -INFINITY;
        if (qi < nq && s.pos[qi] >= 0) {
          const int p = s.pos[qi];
          float total = s.racc[row] + s.racc[kRows + row];
          if ((p + 1) % B != 0) total += relu_nan(s.r[row]);  // partial block
          r = __ldg(w + (int64_t)(qb + qi) * H + h) * total;
          if (router_scores) router_scores[(int64_t)(qb + qi) * H + h] = r;
          if (r != r) {
            set_status(status, MISA_STATUS_BAD_INPUT);
            r = -INFINITY;
          }
        }
        s.r[row] = r;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      // Top-m per query by (r desc, head asc): rank of each head.
      for (int row = et; row < ROWS; row += kEpiThreads) {
        const int qi = row / H, h = row - qi * H;
        if (qi >= nq) continue;
        const int64_t t = qb + qi;
        if (s.pos[qi] < 0) {
          if (h < m) {
            heads[t * m + h] = -1;
            w_r[t * m + h] = 0.f;
            uint4* dst = reinterpret_cast<uint4*>(q_r + (t * m + h) * kD);
            for (int i = 0; i < kD / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
          }
          continue;
        }
        const float r = s.r[row];
        const float* rq = s.r + qi * H;
        int rank = 0;
#pragma unroll 8
        for (int o = 0; o < H; ++o) {
          const float ro = rq[o];
          rank += (ro > r) || (ro == r && o < h);
        }
        if (rank < m) {
          heads[t * m + rank] = h;
          w_r[t * m + rank] = __ldg(w + t * H + h);
          const uint4* src = reinterpret_cast<const uint4*>(q + (t * H + h) * kD);
          uint4* dst = reinterpret_cast<uint4*>(q_r + (t * m + rank) * kD);
#pragma unroll
          for (int i = 0; i < kD / 8; ++i) dst[i] = __ldg(src + i);
        }
      }
      // s.pos, s.racc and s.r are rewritten by the next group
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int H>
int launch_h(const RouteTcArgs& a, const CUtensorMap& qmap, const CUtensorMap& himap,
             const CUtensorMap& lomap, cudaStream_t st) {
  auto kern = route_tc_kernel<H>;
  int rc = set_smem_limit((const void*)kern, kSmemBytes);
  if (rc) return rc;
  ProfScope ps("route", st);
  const int grid = a.max_groups < num_sms() ? a.max_groups : num_sms();  // persistent
  kern<<<grid, kThreads, kSmemBytes, st>>>(
      qmap, himap, lomap, a.q, a.w, a.K, a.p->key_offsets, a.p->block_offsets, a.p->q_pos,
      a.groups, a.group_count, a.Pm, a.p->block, a.m, a.heads, a.q_r, a.w_r, a.router_scores,
      status_ptr());
  return cuda_fail(cudaGetLastError(), "route_tc_kernel");
}

}  // namespace

int route_tc_group_size(int H) {
  const int g = kRows / H;
  return g < kMaxG ? g : kMaxG;
}

size_t route_tc_split_bytes(const misa_problem_t& p) {
  // hi + lo bf16 copies of Kbar, then the running block means (fp32 per key)
  const size_t split = ((size_t)p.total_blocks * kD * 2 * 2 + 255) & ~size_t(255);
  return split + (size_t)p.total_keys * kD * 4;
}

int launch_route_tc(const RouteTcArgs& a, cudaStream_t st) {
  const misa_problem_t& p = *a.p;
  if (a.max_groups <= 0) return MISA_OK;
  const int64_t n = p.total_blocks * kD;
  __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(a.split);
  __nv_bfloat16* lo = hi + n;
  RouteTcArgs b = a;
  b.Pm = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.split) +
                                  (((size_t)n * 2 * 2 + 255) & ~size_t(255)));
  if (p.total_blocks > 0) {
    ProfScope ps("route_means", st);
    prefix_means_kernel<<<(unsigned)((p.total_blocks + 7) / 8), 256, 0, st>>>(
        a.K, p.key_offsets, p.block_offsets, p.num_seqs, p.block, p.total_blocks, b.Pm);
    int rc = cuda_fail(cudaGetLastError(), "prefix_means_kernel");
    if (rc) return rc;
  }
  if (n > 0) {
    ProfScope ps("route_split", st);
    split_kbar_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.Kbar, n, hi, lo);
    int rc = cuda_fail(cudaGetLastError(), "split_kbar_kernel");
    if (rc) return rc;
  }
  CUtensorMap qmap, himap, lomap;
  int rc = make_kmajor_map(&qmap, a.q, (int64_t)p.num_queries * p.num_heads, 32);
  if (rc) return rc;
  if ((rc = make_kmajor_map(&himap, hi, p.total_blocks, kChunk))) return rc;
  if ((rc = make_kmajor_map(&lomap, lo, p.total_blocks, kChunk))) return rc;
  switch (p.num_heads) {
    case 8: return launch_h<8>(b, qmap, himap, lomap, st);
    case 16: return launch_h<16>(b, qmap, himap, lomap, st);
    case 32: return launch_h<32>(b, qmap, himap, lomap, st);
    case 64: return launch_h<64>(b, qmap, himap, lomap, st);
    default:
      set_error("tensor-core router needs H in {8,16,32,64}, got %d", p.num_heads);
      return MISA_ERR_UNSUPPORTED;
  }
}

}  // namespace misa
