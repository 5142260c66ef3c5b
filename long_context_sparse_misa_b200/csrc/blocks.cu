// Routed heads x block pruning: the routed heads score the pooled key blocks,
// only the tokens of the best blocks (plus the query's own incomplete block)
// are scored at token level, and the top-k is taken among them.
//
// Sources: the HISA abstract on the thelatestinai.com papers page (a
// block-level coarse filter scores pooled block representations and drops
// irrelevant regions; the indexer then refines only inside the kept blocks),
// and the gist.science summary of "MISA: Mixture of Indexer Sparse Attention
// for Long-Context LLM Inference", "Probleemstelling" (HISA works on the
// token axis) and "Betekenis en Claims" (head-axis routing combines with any
// token-level scheme).  The two axes compose here: the heads that the MISA
// router keeps also run the block stage.
//
// Launch sequence of misa_block_score_topk (all with programmatic dependent
// launch, so the chain can be replayed as one CUDA graph):
//   block_score_kernel<m>   S[t,b] = sum_j w_r[t,j] ReLU(q_r[t,j] . Kbar[b]),
//                           full blocks b < floor((q_pos[t]+1)/B)
//   topk (token mode)       the n_blocks best blocks by (S desc, block asc)
//   block_expand_kernel     candidate tokens: the kept blocks' keys and the
//                           keys of the incomplete block up to q_pos[t]
//   score_kernel<m, gather> the routed heads score the candidates (tcgen05)
//   topk (token mode)       the final top-k by (score desc, token asc)
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace misa {

// Argument checks shared with the other entry points (abi.cu).
int check_problem(const misa_problem_t* p);
int check_ptr(const void* ptr, size_t align, const char* name);
bool pow2_le64(int x);

namespace {

constexpr int kBlkPerCta = 64;  // pooled blocks per CTA, one per thread
constexpr int kRowF4 = 33;      // shared row stride in float4: 128 floats + 4 of padding
constexpr int kExpandThreads = 256;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// CTA (t, y) scores pooled blocks y*kBlkPerCta .. +kBlkPerCta-1 for query t.  The
// blocks' fp32 rows are staged in shared memory with coalesced loads (rows
// padded to 33 float4, so the per-thread row reads hit distinct banks); the
// query's m routed rows are widened to fp32 once and read as broadcasts.
template <int M>
__global__ void __launch_bounds__(kBlkPerCta)
    block_score_kernel(const uint16_t* __restrict__ q_r, const float* __restrict__ w_r,
                       const float* __restrict__ Kbar, const int64_t* __restrict__ ko,
                       const int64_t* __restrict__ bo, const int32_t* __restrict__ qo,
                       const int32_t* __restrict__ q_pos, int S, int B, int ld,
                       float* __restrict__ Sb, int32_t* __restrict__ btok, uint32_t* status) {
  pdl_wait_then_release();
  extern __shared__ float4 smem4[];
  float4* kb = smem4;                        // [kBlkPerCta][kRowF4]
  float4* qs = smem4 + kBlkPerCta * kRowF4;  // [M][32]
  __shared__ float ws[M];

  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int s = upper_segment<int32_t>(qo, S, t);
  const int64_t L = ko[s + 1] - ko[s];
  int pos = q_pos[t];
  if (pos < 0 || pos >= L) {
    if (blockIdx.y == 0 && tid == 0) set_status(status, MISA_STATUS_BAD_INPUT);
    pos = -1;
  }
  const int full = (pos + 1) / B;  // full blocks the query sees (all inside the sequence)
  const int b0 = blockIdx.y * kBlkPerCta;
  const int nrows = max(0, min(full - b0, kBlkPerCta));

  if (nrows > 0) {
    // q_r row t: M x 128 bf16 = M x 16 uint4 of 8 values each
    const uint4* qsrc = reinterpret_cast<const uint4*>(q_r + (int64_t)t * M * kD);
    for (int e = tid; e < M * 16; e += kBlkPerCta) {
      const uint4 u = __ldg(qsrc + e);
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
      float f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(wd[i] << 16);
        f[2 * i + 1] = __uint_as_float(wd[i] & 0xFFFF0000u);
      }
      const int j = e >> 4, c = (e & 15) * 2;
      qs[j * 32 + c] = make_float4(f[0], f[1], f[2], f[3]);
      qs[j * 32 + c + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    for (int j = tid; j < M; j += kBlkPerCta) ws[j] = w_r[(int64_t)t * M + j];
    const float4* ksrc = reinterpret_cast<const float4*>(Kbar + (bo[s] + b0) * kD);
    for (int f = tid; f < nrows * 32; f += kBlkPerCta)
      kb[(f >> 5) * kRowF4 + (f & 31)] = __ldg(ksrc + f);
  }
  __syncthreads();

  const int b = b0 + tid;
  if (b >= ld) return;
  const int64_t o = (int64_t)t * ld + b;
  if (tid >= nrows) {
    Sb[o] = -INFINITY;
    btok[o] = -1;
    return;
  }
  float acc[M];
#pragma unroll
  for (int j = 0; j < M; ++j) acc[j] = 0.f;
  const float4* row = kb + tid * kRowF4;
#pragma unroll 4
  for (int c = 0; c < 32; ++c) {
    const float4 kv = row[c];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      const float4 qv = qs[j * 32 + c];
      acc[j] = fmaf(qv.x, kv.x, acc[j]);
      acc[j] = fmaf(qv.y, kv.y, acc[j]);
      acc[j] = fmaf(qv.z, kv.z, acc[j]);
      acc[j] = fmaf(qv.w, kv.w, acc[j]);
    }
  }
  float score = 0.f;
#pragma unroll
  for (int j = 0; j < M; ++j) score = fmaf(ws[j], relu_nan(acc[j]), score);
  Sb[o] = score;
  btok[o] = b;
}

// Candidate row of query t: slot i*B + j is key j of kept block blk[t,i]
// (-1 when that slot of blk is padding); slots nb*B .. nb*B+B-1 hold the
// incomplete block's keys floor((pos+1)/B)*B + j, those past pos as -1.
__global__ void __launch_bounds__(kExpandThreads)
    block_expand_kernel(const int32_t* __restrict__ blk, int nb, const int64_t* __restrict__ ko,
                        const int32_t* __restrict__ qo, const int32_t* __restrict__ q_pos, int S,
                        int B, int32_t* __restrict__ cand) {
  pdl_wait_then_release();
  const int t = blockIdx.x;
  const int s = upper_segment<int32_t>(qo, S, t);
  const int64_t L = ko[s + 1] - ko[s];
  int pos = q_pos[t];
  if (pos < 0 || pos >= L) pos = -1;
  const int full = (pos + 1) / B;
  const int kc = (nb + 1) * B;
  int32_t* out = cand + (int64_t)t * kc;
  for (int e = threadIdx.x; e < kc; e += kExpandThreads) {
    const int i = e / B, j = e - i * B;
    int tok;
    if (i < nb) {
      const int b = blk[(int64_t)t * nb + i];
      tok = (b >= 0 && b < full) ? b * B + j : -1;
    } else {
      tok = full * B + j;
      if (tok > pos) tok = -1;
    }
    out[e] = tok;
  }
}

template <int M>
int launch_block_scores(const misa_problem_t& p, const uint16_t* q_r, const float* w_r,
                        const float* Kbar, int ld, float* Sb, int32_t* btok, cudaStream_t st) {
  auto kern = block_score_kernel<M>;
  const int smem = (kBlkPerCta * kRowF4 + M * 32) * (int)sizeof(float4);
  int rc = set_smem_limit((const void*)kern, smem);
  if (rc) return rc;
  // x: query (up to 2^31 - 1), y: chunk of pooled blocks
  const int chunks = (ld + kBlkPerCta - 1) / kBlkPerCta;
  if (chunks > 65535) {
    set_error("block scores: %d pooled blocks per row exceed the grid limit", ld);
    return MISA_ERR_UNSUPPORTED;
  }
  dim3 grid(p.num_queries, chunks);
  ProfScope ps("block_score", st);
  return cuda_fail(launch_pdl(kern, grid, dim3(kBlkPerCta), (size_t)smem, st, q_r, w_r, Kbar,
                              p.key_offsets, p.block_offsets, p.query_offsets, p.q_pos,
                              p.num_seqs, p.block, ld, Sb, btok, status_ptr()),
                   "block_score_kernel");
}

struct BlockPlan {
  int ld;       // pooled blocks per score row: ceil(max_seq_len / B)
  int kc;       // candidates per query: (n_blocks + 1) * B
  size_t o_tok, o_bval, o_bidx, o_cand, o_rows, total;
};

BlockPlan block_plan(const misa_problem_t& p, int nb) {
  BlockPlan b;
  const size_t T = (size_t)p.num_queries;
  b.ld = (p.max_seq_len + p.block - 1) / p.block;
  b.kc = (nb + 1) * p.block;
  b.o_tok = align256(T * b.ld * 4);
  b.o_bval = b.o_tok + align256(T * b.ld * 4);
  b.o_bidx = b.o_bval + align256(T * nb * 4);
  b.o_cand = b.o_bidx + align256(T * nb * 4);
  b.o_rows = b.o_cand + align256(T * b.kc * 4);
  b.total = b.o_rows + align256(T * b.kc * 4);
  return b;
}

int check_block_args(const misa_problem_t* p, int nb) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (nb < 1 || (int64_t)(nb + 1) * p->block > 65536) {
    set_error("need n_blocks >= 1 and (n_blocks + 1) * block <= 65536 (n_blocks=%d block=%d)",
              nb, p->block);
    return MISA_ERR_INVALID_ARG;
  }
  return MISA_OK;
}

}  // namespace
}  // namespace misa

using namespace misa;

extern "C" size_t misa_block_workspace_size(const misa_problem_t* p, int32_t n_blocks) {
  if (check_block_args(p, n_blocks)) return 0;
  return block_plan(*p, n_blocks).total;
}

extern "C" int misa_block_score_topk(const misa_problem_t* p, const uint16_t* q_r,
                                     const float* w_r, int32_t m, const uint16_t* K,
                                     const float* Kbar, int32_t n_blocks, int32_t k, int32_t* idx,
                                     float* val, int32_t* blocks, void* ws, size_t ws_bytes,
                                     misa_stream_t stream) {
  int rc = check_block_args(p, n_blocks);
  if (rc) return rc;
  if (!pow2_le64(m) || m > p->num_heads) {
    set_error("m=%d must be a power of two <= min(64, H=%d)", m, p->num_heads);
    return MISA_ERR_UNSUPPORTED;
  }
  const BlockPlan b = block_plan(*p, n_blocks);
  if (k < 1 || k > b.kc) {
    set_error("need 1 <= k <= (n_blocks + 1) * block = %d (k=%d)", b.kc, k);
    return MISA_ERR_INVALID_ARG;
  }
  const int T = p->num_queries;
  if (T == 0) return MISA_OK;
  if ((rc = check_ptr(q_r, 16, "q_r")) || (rc = check_ptr(w_r, 4, "w_r")) ||
      (rc = check_ptr(K, 16, "K")) || (rc = check_ptr(Kbar, 16, "Kbar")) ||
      (rc = check_ptr(idx, 4, "idx")) || (rc = check_ptr(val, 4, "val")) ||
      (rc = check_ptr(ws, 256, "workspace")) || (blocks && (rc = check_ptr(blocks, 4, "blocks"))))
    return rc;
  if (ws_bytes < b.total) {
    set_error("workspace too small: %zu < %zu", ws_bytes, b.total);
    return MISA_ERR_WORKSPACE_TOO_SMALL;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* Sb = reinterpret_cast<float*>(base);
  int32_t* btok = reinterpret_cast<int32_t*>(base + b.o_tok);
  float* bval = reinterpret_cast<float*>(base + b.o_bval);
  int32_t* bidx = blocks ? blocks : reinterpret_cast<int32_t*>(base + b.o_bidx);
  int32_t* cand = reinterpret_cast<int32_t*>(base + b.o_cand);
  float* rows = reinterpret_cast<float*>(base + b.o_rows);

  switch (m) {
    case 1: rc = launch_block_scores<1>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
    case 2: rc = launch_block_scores<2>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
    case 4: rc = launch_block_scores<4>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
    case 8: rc = launch_block_scores<8>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
    case 16: rc = launch_block_scores<16>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
    case 32: rc = launch_block_scores<32>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
    default: rc = launch_block_scores<64>(*p, q_r, w_r, Kbar, b.ld, Sb, btok, st); break;
  }
  if (rc) return rc;
  if ((rc = launch_topk(*p, Sb, b.ld, btok, b.ld, 0, T, n_blocks, bidx, bval, st))) return rc;
  {
    ProfScope ps("block_expand", st);
    rc = cuda_fail(launch_pdl(block_expand_kernel, dim3(T), dim3(kExpandThreads), 0, st,
                              (const int32_t*)bidx, (int)n_blocks, p->key_offsets,
                              p->query_offsets, p->q_pos, p->num_seqs, p->block, cand),
                   "block_expand_kernel");
    if (rc) return rc;
  }
  // The routed heads score the candidates: one query per group, rows taken
  // directly (no plan), as in the MISA-dagger re-rank.
  ScoreArgs a;
  a.p = p; a.qsel = q_r; a.wsel = w_r; a.m = m; a.K = K; a.cand = cand;
  a.k_cand = b.kc; a.groups = nullptr; a.group_count = nullptr; a.max_groups = T;
  a.direct = true;
  a.G = 1; a.q_lo = 0; a.I = rows; a.ld = b.kc;
  a.max_tiles = (b.kc + kTileKeys - 1) / kTileKeys;
  if ((rc = launch_score(a, st))) return rc;
  return launch_topk(*p, rows, b.kc, cand, b.kc, 0, T, k, idx, val, st);
}
