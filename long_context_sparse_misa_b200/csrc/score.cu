// Token-level indexer scoring on tcgen05 tensor cores.
//
// Computes, for every query t of a group and key s of its causal prefix,
//     I[t,s] = sum_{j<m} w[t,j] * ReLU(q[t,j] . k[s])
// With the routed heads this is MISA's sparse token scoring ("MISA: Mixture
// of Indexer Sparse Attention for Long-Context LLM Inference", gist.science
// summary, "Methodologie: MISA", Sparse Token Scoring); with all H heads it
// is the dense DSA indexer (abstract); in gather mode over candidate tokens
// it is the MISA-dagger re-scoring (same page, "Hierarchische Variant").
//
// Layout of one CTA (one query group x a range of 128-key tiles):
//   A operand = 128 keys x 128 dims, TMA-loaded (or cp.async-gathered) into a
//               128-byte-swizzled K-major tile, kStages deep;
//   B operand = the group's (query, head) rows, N = nq*m <= 256, resident;
//   D         = TMEM, 128 lanes (one key per lane) x N fp32 columns, two
//               buffers so the epilogue of tile i overlaps the MMAs of i+1.
// Keys on the lanes means the head reduction of a query is a sum over m
// adjacent columns inside one thread: the epilogue is ReLU, one FMA with the
// head weight, and a causal compare -- no shuffles and no [m x L] tensor.
//
// Roles: warp 0 producer, warp 1 TMEM owner + MMA issuer (one thread),
// warps 2..5 epilogue (TMEM lane quarter = warp % 4); in gather mode warps 6,
// 7 and 8 are three more producers.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kThreads = 192;
// Gather mode adds three producer warps (6, 7 and 8): the copies of a tile
// are issued by one warp, tiles go round-robin over the four producers, one
// per stage.
constexpr int kGatherThreads = 288;
constexpr int kGatherProducers = 4;
__host__ __device__ constexpr int threads_for(bool gather) {
  return gather ? kGatherThreads : kThreads;
}
constexpr int kStages = 4;
constexpr int kStageBytes = kTileKeys * kD * 2;          // 32 KB: two 16 KB 64-dim halves
constexpr int kHalfBytes = kStageBytes / 2;
constexpr int kMaxN = 256;                               // MMA N and TMEM columns per buffer
constexpr int kQHalfBytes = kMaxN * 128;                 // 32 KB per 64-dim half
constexpr int kQBytes = 2 * kQHalfBytes;
constexpr int kTmemCols = 2 * kMaxN;
constexpr int kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kMaxN * 4 /*w*/ +
                           kMaxN * 4 /*pos*/ + kMaxN * 4 /*row*/ + 32 * 8 /*barriers*/ + 16;

struct Smem {
  uint8_t* q;
  uint8_t* k;
  float* w;
  int* pos;
  int* row;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* qfull;
  uint64_t* drain;
  uint32_t* tmem_slot;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.q = base;
  s.k = base + kQBytes;
  s.w = reinterpret_cast<float*>(s.k + kStages * kStageBytes);
  s.pos = reinterpret_cast<int*>(s.w + kMaxN);
  s.row = s.pos + kMaxN;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.row + kMaxN);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 2;
  s.qfull = s.tempty + 2;
  s.drain = s.qfull + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.drain + 1);
  s.abort = reinterpret_cast<int*>(s.tmem_slot + 1);
  return s;
}

template <int MH, bool GATHER>
__global__ void __launch_bounds__(threads_for(GATHER), 1)
    score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                 const uint16_t* __restrict__ K, const float* __restrict__ wsel,
                 const int32_t* __restrict__ q_pos, const int64_t* __restrict__ ko,
                 const int32_t* __restrict__ cand, int k_cand, const int4* __restrict__ groups,
                 const int* __restrict__ group_count, int tiles_per_split, int q_lo,
                 float* __restrict__ I, int64_t ld, int64_t total_keys, uint32_t* status,
                 const int32_t* __restrict__ qo, int S, int direct_T, int row_by_group) {
  pdl_wait_then_release();
  constexpr int G = GATHER ? 1 : kMaxN / MH;
  static_assert(G * MH <= kMaxN, "group too wide");
  extern __shared__ uint8_t smem_raw[];

  // tiles_per_split > 0: CTA (x, y) takes group x, tiles from y * tiles_per_split.
  // tiles_per_split == 0: one wave of gridDim.x CTAs spread over the groups
  // that exist, gridDim.x / count consecutive CTAs per group.
  // direct_T > 0 (gather mode): no group table; group i is query row i.
  const int count = direct_T > 0 ? direct_T : *group_count;
  int gi = blockIdx.x, split = blockIdx.y, nsplit = 0;
  if (tiles_per_split == 0) {
    nsplit = count > 0 ? max(1, (int)gridDim.x / count) : 1;
    gi = blockIdx.x / nsplit;
    split = blockIdx.x % nsplit;
  }
  if (gi >= count) return;
  int4 grp;
  if (GATHER && direct_T > 0) {
    const int sq = upper_segment<int32_t>(qo, S, gi);
    const int64_t Lq = ko[sq + 1] - ko[sq];
    int pq = q_pos[gi];
    if (pq < 0 || pq >= Lq) {  // as the planner: flagged, and the row is left out
      if (split == 0 && threadIdx.x == 0) set_status(status, MISA_STATUS_BAD_INPUT);
      pq = -1;
    }
    grp = make_int4(sq, gi, gi + 1, pq);
  } else {
    grp = groups[gi];
  }
  const int seq = grp.x, qb = grp.y, nq = grp.z - grp.y, maxpos = grp.w;
  if (maxpos < 0 || nq <= 0) return;
  const int64_t key_base = ko[seq];
  const int ntiles = GATHER ? (k_cand + kTileKeys - 1) / kTileKeys
                            : (maxpos + 1 + kTileKeys - 1) / kTileKeys;
  const int tps = tiles_per_split > 0 ? tiles_per_split : (ntiles + nsplit - 1) / nsplit;
  const int tile0 = split * tps;
  if (tile0 >= ntiles) return;
  const int nt = min(ntiles, tile0 + tps) - tile0;
  const int NP = ((nq * MH + 31) / 32) * 32;  // MMA N (multiple of 32, <= 256)

  Smem s = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], GATHER ? 32 : 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 4);
    }
    mbar_init(s.qfull, 1);
    mbar_init(s.drain, 1);
    *s.abort = 0;
    fence_barrier_init();
  }
  // Contiguous mode: the producer thread starts the query rows and the first
  // kStages key tiles at once (the stages start empty), before the block-wide
  // set-up below, so the first loads overlap it.
  int pre = 0;
  if (!GATHER && threadIdx.x == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
    mbar_arrive_expect_tx(s.qfull, 2u * NP * 128u);
    for (int h = 0; h < 2; ++h)
      for (int r0 = 0; r0 < NP; r0 += 32)
        tma_load_2d(&qmap, s.qfull, s.q + h * kQHalfBytes + r0 * 128, h * 64, qb * MH + r0);
    pre = min(kStages, nt);
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&s.full[i], kStageBytes);
      const int32_t krow = (int32_t)(key_base + (int64_t)(tile0 + i) * kTileKeys);
      uint8_t* dst = s.k + i * kStageBytes;
      tma_load_2d(&kmap, &s.full[i], dst, 0, krow);
      tma_load_2d(&kmap, &s.full[i], dst + kHalfBytes, 64, krow);
    }
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 6) {
    // Per-column head weight and per-query causal limit / output row.
    for (int c = threadIdx.x - 64; c < kMaxN; c += 128) {
      const int qi = c / MH;
      s.w[c] = (c < nq * MH) ? relu_weight(wsel[(int64_t)(qb + qi) * MH + (c - qi * MH)]) : 0.f;
    }
    for (int qi = threadIdx.x - 64; qi < kMaxN; qi += 128) {
      int pos = -1;
      if (qi < nq) {
        pos = q_pos[qb + qi];
        const int64_t L = ko[seq + 1] - key_base;
        if (pos < 0 || pos >= L) pos = -1;
      }
      s.pos[qi] = pos;
      // row_by_group: one query per group, written to row gi (a list of queries)
      s.row[qi] = row_by_group ? gi + qi : qb + qi - q_lo;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;

  if (warp == 0 || warp >= 6) {
    // ------------------------------------------------------------ producer(s)
    if (!GATHER) {
      if (lane == 0) {
        int issued = pre;
        for (int i = pre; i < nt; ++i) {
          const int st = i % kStages;
          const uint32_t ph = (i / kStages) & 1;
          if (!mbar_wait(&s.empty[st], ph ^ 1, s.abort, status)) break;
          mbar_arrive_expect_tx(&s.full[st], kStageBytes);
          const int32_t krow = (int32_t)(key_base + (int64_t)(tile0 + i) * kTileKeys);
          uint8_t* dst = s.k + st * kStageBytes;
          tma_load_2d(&kmap, &s.full[st], dst, 0, krow);
          tma_load_2d(&kmap, &s.full[st], dst + kHalfBytes, 64, krow);
          issued = i + 1;
        }
        // Drain: the last load of every stage must have landed before the CTA exits.
        for (int i = max(0, issued - kStages); i < issued; ++i)
          mbar_wait(&s.full[i % kStages], (i / kStages) & 1, s.abort, status, kDrainCycles,
                    /*drain=*/true);
      }
    } else {
      // Gather mode: rows K[key_base + cand[t, slot]] for the 128 slots of a
      // tile, copied as 16-byte chunks into the swizzled layout, two whole
      // rows per warp instruction.  Producer p (warp 0, 6, 7, 8) takes tiles
      // p, p + 4, ...
      const int t = qb;
      const int pos = s.pos[0];
      const int prod = warp == 0 ? 0 : warp - 5;
      if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&qmap);
        mbar_arrive_expect_tx(s.qfull, 2u * NP * 128u);
        for (int h = 0; h < 2; ++h)
          for (int r0 = 0; r0 < NP; r0 += 32)
            tma_load_2d(&qmap, s.qfull, s.q + h * kQHalfBytes + r0 * 128, h * 64,
                        qb * MH + r0);
      }
      __syncwarp();
      // Each producer has one tile in flight: copy, wait for its copies,
      // signal; the producers overlap.  A tile's candidate indices are
      // loaded one tile ahead, so their latency overlaps the previous
      // tile's copies.
      auto tile_tokens = [&](int i, int (&tk)[4]) {
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int slot = (tile0 + i) * kTileKeys + lane * 4 + rr;
          tk[rr] = (i < nt && slot < k_cand) ? cand[(int64_t)t * k_cand + slot] : -1;
        }
      };
      int tok_cur[4];
      tile_tokens(prod, tok_cur);
      for (int i = prod; i < nt; i += kGatherProducers) {
        const int st = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        int tok_next[4];
        tile_tokens(i + kGatherProducers, tok_next);
        if (!warp_wait(&s.empty[st], ph ^ 1, s.abort, status)) break;
        uint8_t* dst = s.k + st * kStageBytes;
        // Two rows per copy instruction: lanes 0-15 take the 16 chunks of one
        // row, lanes 16-31 those of the next, so each instruction reads two
        // whole 256-byte rows (row r's token is held by lane r / 4, slot r % 4).
        const int c = lane & 15, half = c >> 3, cc = c & 7;
#pragma unroll 2
        for (int u = 0; u < kTileKeys / 4; ++u) {  // rows 4u .. 4u+3, held by lane u
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int tA = __shfl_sync(0xffffffffu, tok_cur[2 * v], u);
            const int tB = __shfl_sync(0xffffffffu, tok_cur[2 * v + 1], u);
            const int r = 4 * u + 2 * v + (lane >> 4);
            const int tok = (lane >> 4) ? tB : tA;
            const bool ok = tok >= 0 && tok <= pos && key_base + tok < total_keys;
            const uint16_t* src = K + (ok ? (key_base + tok) : 0) * kD + c * 8;
            cp_async_16(dst + half * kHalfBytes + r * 128 + ((cc ^ (r & 7)) << 4), src, ok);
          }
        }
        cp_async_commit();
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        mbar_arrive(&s.full[st]);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) tok_cur[rr] = tok_next[rr];
      }
      cp_async_wait_group<0>();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileKeys, NP);
      bool ok = mbar_wait(s.qfull, 0, s.abort, status);
      tc_fence_after();
      const uint32_t q_addr = smem_u32(s.q);
      for (int i = 0; ok && i < nt; ++i) {
        const int st = i % kStages;
        const int buf = i & 1;
        if (!mbar_wait(&s.full[st], (i / kStages) & 1, s.abort, status)) break;
        if (!mbar_wait(&s.tempty[buf], ((i >> 1) & 1) ^ 1, s.abort, status)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(s.k + st * kStageBytes);
        const uint32_t d = tmem_base + buf * kMaxN;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 bf16 = 32 B along K
          const uint64_t a = sw128_kmajor_desc(k_addr + (kk >> 2) * kHalfBytes + off);
          const uint64_t b = sw128_kmajor_desc(q_addr + (kk >> 2) * kQHalfBytes + off);
          umma_bf16(d, a, b, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s.empty[st]);
        umma_commit(&s.tfull[buf]);
      }
      // Every issued MMA must complete before TMEM is released.
      umma_commit(s.drain);
      mbar_wait(s.drain, 0, s.abort, status, kDrainCycles, /*drain=*/true);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int lrow = quarter * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int nwin = (NP + 63) / 64;
    for (int i = 0; i < nt; ++i) {
      const int buf = i & 1;
      if (!warp_wait(&s.tfull[buf], (i >> 1) & 1, s.abort, status)) break;
      tc_fence_after();
      const int slot = (tile0 + i) * kTileKeys + lrow;
      int key = slot;  // contiguous mode: token index within the sequence
      bool key_ok = true;
      if (GATHER) {
        key = slot < k_cand ? cand[(int64_t)qb * k_cand + slot] : -1;
        key_ok = key >= 0 && key <= s.pos[0] && key_base + key < total_keys;
        if (key >= 0 && !key_ok) set_status(status, MISA_STATUS_BAD_INPUT);
      }
      const uint32_t taddr = lane_addr + buf * kMaxN;
      for (int c = 0; c < nwin; ++c) {
        // 64-column window (the buffer has kMaxN columns, so reading past NP is harmless)
        float v[2][32];
        tmem_ld32(taddr + c * 64, v[0]);
        tmem_ld32(taddr + c * 64 + 32, v[1]);
        tmem_wait_ld();
        reg_fence32(v[0]);
        reg_fence32(v[1]);
        constexpr int QPW = 64 / MH;  // queries per 64-column window
#pragma unroll
        for (int qq = 0; qq < QPW; ++qq) {
          const int qi = c * QPW + qq;
          if (qi >= nq) break;
          const float sc = relu_wsum<MH>(
              [&](int j) {
                const int col = qq * MH + j;
                return v[col >> 5][col & 31];
              },
              s.w + qi * MH);
          if (GATHER) {
            if (slot < k_cand && s.row[0] >= 0)
              I[(int64_t)s.row[0] * ld + slot] = key_ok ? sc : -INFINITY;
          } else if (key <= s.pos[qi]) {
            I[(int64_t)s.row[qi] * ld + key] = sc;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int MH, bool GATHER>
int launch_one(const ScoreArgs& a, const CUtensorMap& kmap, const CUtensorMap& qmap, dim3 grid,
               int tps, cudaStream_t st) {
  auto kern = score_kernel<MH, GATHER>;
  int rc = set_smem_limit((const void*)kern, kSmemBytes);
  if (rc) return rc;
  ProfScope ps(GATHER ? "rerank_score" : (a.row_by_group ? "rescan_score" : "score"), st);
  return cuda_fail(launch_pdl(kern, grid, dim3(threads_for(GATHER)), kSmemBytes, st, kmap, qmap, a.K,
                              a.wsel, a.p->q_pos, a.p->key_offsets, a.cand, a.k_cand, a.groups,
                              a.group_count, tps, a.q_lo, a.I, a.ld, a.p->total_keys,
                              status_ptr(), a.p->query_offsets, a.p->num_seqs,
                              a.direct ? a.p->num_queries : 0, a.row_by_group ? 1 : 0),
                   "score_kernel");
}

template <bool GATHER>
int dispatch(const ScoreArgs& a, const CUtensorMap& kmap, const CUtensorMap& qmap, dim3 grid,
             int tps, cudaStream_t st) {
  switch (a.m) {
    case 1: return launch_one<1, GATHER>(a, kmap, qmap, grid, tps, st);
    case 2: return launch_one<2, GATHER>(a, kmap, qmap, grid, tps, st);
    case 4: return launch_one<4, GATHER>(a, kmap, qmap, grid, tps, st);
    case 8: return launch_one<8, GATHER>(a, kmap, qmap, grid, tps, st);
    case 16: return launch_one<16, GATHER>(a, kmap, qmap, grid, tps, st);
    case 32: return launch_one<32, GATHER>(a, kmap, qmap, grid, tps, st);
    case 64: return launch_one<64, GATHER>(a, kmap, qmap, grid, tps, st);
    default:
      set_error("score: head count %d is not a power of two <= 64", a.m);
      return MISA_ERR_UNSUPPORTED;
  }
}

}  // namespace

int score_group_size(int m) { return kMaxN / m; }

int launch_score(const ScoreArgs& a, cudaStream_t st) {
  if (a.max_groups <= 0 || a.max_tiles <= 0) return MISA_OK;
  CUtensorMap kmap, qmap;
  int rc = make_kmajor_map(&kmap, a.K, a.p->total_keys, kTileKeys);
  if (rc) return rc;
  rc = make_kmajor_map(&qmap, a.qsel, (int64_t)a.p->num_queries * a.m, 32);
  if (rc) return rc;
  // Prefill-sized problems: about 8 CTAs per SM over the whole causal work,
  // for balance.  Decode-sized problems (fewer groups than SMs): one wave of
  // one CTA per SM, so that each CTA streams a long key range through its
  // pipeline rather than paying its set-up for a few tiles in many waves;
  // the device splits the wave among the groups that the plan produced.
  const int sms = num_sms();
  if (a.max_groups < sms) {
    // The device divides the SMs among the groups it finds (tiles_per_split 0).
    dim3 grid(sms, 1);
    return a.cand ? dispatch<true>(a, kmap, qmap, grid, 0, st)
                  : dispatch<false>(a, kmap, qmap, grid, 0, st);
  }
  const int64_t work = (int64_t)a.max_groups * a.max_tiles;
  int tps = (int)((work + 8 * sms - 1) / (8 * sms));
  tps = max(1, min(tps, 64));
  const int splits = (a.max_tiles + tps - 1) / tps;
  if (splits > 65535) {
    set_error("score: %d key splits exceed the grid limit", splits);
    return MISA_ERR_UNSUPPORTED;
  }
  dim3 grid(a.max_groups, splits);
  return a.cand ? dispatch<true>(a, kmap, qmap, grid, tps, st)
                : dispatch<false>(a, kmap, qmap, grid, tps, st);
}

}  // namespace misa
