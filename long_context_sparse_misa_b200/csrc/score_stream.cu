// Routed token scoring with the per-query top-k fused into the epilogue
// (prefill: every query scores its whole causal prefix).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// gist.science summary, "Methodologie: MISA" (Sparse Token Scoring: only the
// routed heads score the prefix; the top-k tokens come from those scores).
// The same kernel with m = H is the dense DSA indexer (abstract).
//
// Why fused: at 128K prefill the score matrix is 8.6e9 fp32 values (34 GB);
// writing and re-reading it costs more than the tensor-core work.  Here no
// score leaves the SM unless it can still be in its query's top-k.
//
// CTA (persistent, one per SM): query groups of G = 256/m queries taken
// longest-prefix first, in rounds over the CTAs that alternate direction.
// Per group: the group's
// (query, head) rows stay in shared memory (B operand, N = 256); 128-key
// tiles of K stream through a 4-stage TMA ring (A operand); tcgen05.mma
// accumulates 128 keys x 256 columns in TMEM, two buffers.
//
// Epilogue (16 warps, four per SM sub-partition so that their dependency
// chains overlap: TMEM lane quarter = warp % 4, column quarter = which of the
// four warps of that lane quarter, i.e. 64 columns = 64/m queries each), per
// tile: four 16-column tcgen05.ld, each issued before the previous chunk is
// summed, then per key and query I = sum_j w_j ReLU(acc_j) (the TMEM buffer
// is released after the warp's last load), the causal mask, and the
// streaming selection:
//   * probe: a group first scores every 24th tile of its prefix and keeps a
//     256-bin histogram per query (1/32-octave bins of the order-preserving
//     score key, from 7 octaves below the first scored tile's maximum to one
//     above; scores outside fall into the end bins, which can only lower the
//     threshold).  Two 16-bit counts per shared word.
//     The starting threshold tau_q is the lower edge of the bin holding the
//     r-th best sampled score, r = k*f + 4*sqrt(k*f) + 1 (f = sampled share
//     of the prefix), i.e. a few standard deviations below the expected k-th
//     best score.
//   * main pass over all tiles: a key is appended to query q's candidates
//     only if I >= tau_q.  Each (query, TMEM lane) has its own list, so no
//     lane needs a rank from the others: a passing lane stores at its list's
//     next-row pointer and advances it (a compare, a predicated store and a
//     predicated add, no vote).  Every kCheckTiles tiles a list that could
//     pass its capacity before the next check stops storing and is marked
//     full, which sends its query to the rescan.  A query's 128 lists are
//     stored row by row, so that a row of all lists is 1 KB contiguous.
//   * check and select: every key scoring at least tau_q was appended, so
//     if at least min(k, n) keys were appended (and no list ran past its
//     rows) the exact top-k is among them.  A warp then histograms the
//     candidates, takes those above the bin holding the k-th, and resolves
//     that bin with a warp-level radix select over (score, lower index
//     first).  By default the lists are kept per query row and a second
//     launch (select_deferred_kernel) checks and selects every query after
//     the pass, so no selection work holds up the tensor pipe.  With less
//     workspace the lists are double buffered per CTA and two selector warps
//     check and select each finished group while the epilogue warps stream
//     the next (when the selectors fall behind, the epilogue warps claim the
//     remaining queries of the older buffer before reusing it).  A query that
//     fails the check is listed and rescanned by a last launch without a
//     probe, with lists of one row per tile (selected inside that launch).
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kStages = 4;
constexpr int kStageBytes = kTileKeys * kD * 2;  // 32 KB
constexpr int kHalfBytes = kStageBytes / 2;
constexpr int kN = 256;                          // MMA N = group columns
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = 32 * kEpiWarps;
// Final selection, one group behind.  Registers are split evenly over the
// four SM sub-partitions (16K each) and warps go to them round-robin, so 20
// warps (five per sub-partition) is the most that fits at 96 registers.
constexpr int kSelWarps = 2;
// warp 0 TMA, warp 1 MMA, warps 2..17 epilogue, warps 18..19 selectors
constexpr int kThreads = 64 + kEpiThreads + 32 * kSelWarps;
// Rows per main-pass candidate list: about 21 are used at 128K with the
// probe threshold; a query whose threshold is no filter (short prefixes) or
// that runs past 128 rows goes to the rescan launch, whose lists hold every
// key.  (Letting such queries fill full-length lists makes their exact
// selection, one warp per query, far slower than the rescan.)
constexpr int kRowsCap = 128;
constexpr int kParts = kEpiWarps / 4;            // column parts per TMEM lane quarter
constexpr int kColsPerWarp = kN / kParts;
constexpr int kQHalfBytes = kN * 128;            // 32 KB per 64-dim half
constexpr int kQBytes = 2 * kQHalfBytes;
constexpr int kTmemCols = 2 * kN;
constexpr int kMaxG = 32;                        // queries per group (m >= 8)
constexpr int kBins = 256;
constexpr int kHistWords = kBins / 2;            // two 16-bit bin counts per word
constexpr int kBinShift = 18;                    // 14-bit score key prefix: 1/32 octave
constexpr int kHeadroom = 224;                   // distance bins below the tile's spread
constexpr int kSelBins = 256;
constexpr int kProbeStride = 24;                 // probe every 24th tile ...
constexpr int kProbeOff = 12;                    // ... starting at tile 12
constexpr int kProbeMinTiles = 16;               // only prefixes of >= 2048 keys
constexpr int kCheckTiles = 8;                   // list capacity checked every 8 tiles
constexpr int kRescanCap = 128;                  // failed queries rescanned as score rows

static_assert(kSelBins >= kBins, "final-select histogram");
constexpr int kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kN * 4 /*w*/ +
                           kMaxG * 4 * 7 /*pos,row,tau,maxkey,minkey,base,top*/ +
                           kMaxG * kHistWords * 4 /*hist*/ + kSelWarps * kSelBins * 4 /*select*/ +
                           2 * kMaxG * 4 * 4 /*selector copies of pos,row,base,top*/ +
                           2 * 4 * 3 /*selnq,selnext,seldone*/ +
                           32 * 8 /*barriers*/ + 16;

struct Smem {
  uint8_t* q;
  uint8_t* k;
  float* w;
  int* pos;
  int* row;
  float* tau;
  uint32_t* maxkey;  // first scored tile's maximum and minimum (order keys)
  uint32_t* minkey;
  int* base;    // histogram anchor per query (see Anchor)
  float* top;
  uint32_t* hist;
  uint32_t* sel;   // [kSelWarps][kSelBins]
  int* mpos;       // [2][kMaxG] the selectors' copies of pos, row and the anchor
  int* mrow;
  int* mbase;
  float* mtop;
  int* selnq;          // [2] queries of the group in each candidate buffer
  int* selnext;        // [2] next query to claim for selection
  int* seldone;        // [2] queries selected
  uint64_t* selready;  // [2] a group's candidates are complete
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* qfull;
  uint64_t* qempty;
  uint64_t* ebar;
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
  s.w = reinterpret_cast<float*>(s.k + kStages * kStageBytes);
  s.pos = reinterpret_cast<int*>(s.w + kN);
  s.row = s.pos + kMaxG;
  s.tau = reinterpret_cast<float*>(s.row + kMaxG);
  s.maxkey = reinterpret_cast<uint32_t*>(s.tau + kMaxG);
  s.minkey = s.maxkey + kMaxG;
  s.base = reinterpret_cast<int*>(s.minkey + kMaxG);
  s.top = reinterpret_cast<float*>(s.base + kMaxG);
  s.hist = reinterpret_cast<uint32_t*>(s.top + kMaxG);
  s.sel = s.hist + kMaxG * kHistWords;
  s.mpos = reinterpret_cast<int*>(s.sel + kSelWarps * kSelBins);
  s.mrow = s.mpos + 2 * kMaxG;
  s.mbase = s.mrow + 2 * kMaxG;
  s.mtop = reinterpret_cast<float*>(s.mbase + 2 * kMaxG);
  s.selnq = reinterpret_cast<int*>(s.mtop + 2 * kMaxG);
  s.selnext = s.selnq + 2;
  s.seldone = s.selnext + 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.seldone + 2);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 2;
  s.qfull = s.tempty + 2;
  s.qempty = s.qfull + 1;
  s.ebar = s.qempty + 1;
  s.drain = s.ebar + 1;
  s.selready = s.drain + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.selready + 2);
  s.abort = reinterpret_cast<int*>(s.tmem_slot + 1);
  return s;
}

// Histogram bins of one query (probe and exact selection).  The anchor is
// the query's first scored tile, with spread = its largest minus its
// smallest score.  A score v falls in 1/32-octave bins of its distance below
// the reference top = (largest score) + spread/4, top - v, over distances
// from spread/128 to 2 * spread (256 bins, higher bin = higher score); bin
// 255 also takes every score above top or within spread/128 of it, bin 0
// every score more than 2 * spread below it.  Measuring from the top of the
// tile's own range (not from zero) keeps fine bins near the k-th best score
// whatever its sign: with all H heads, a query whose head weights are mostly
// negative has its k-th best score near or below zero.  The quarter spread
// above the tile's maximum leaves room for the many prefixes whose k-th best
// score lies above the first tile's maximum.  Bin numbers grow with v (the
// subtraction and the order key are both monotonic), so a bin boundary is a
// valid threshold.
struct Anchor {
  float top;
  int base;  // order-key bin (key >> kBinShift) of distance spread/128
};

__device__ __forceinline__ Anchor make_anchor(uint32_t maxkey, uint32_t minkey) {
  Anchor a;
  if (maxkey == 0u || minkey > maxkey) {  // no valid score in the tile
    a.top = 0.f;
    a.base = static_cast<int>(order_key(1e-30f) >> kBinShift) - kHeadroom;
    return a;
  }
  const float hi = key_to_float(maxkey);
  const float spread = fmaxf(hi - key_to_float(minkey), 1e-30f);
  a.top = hi + 0.25f * spread;
  a.base = static_cast<int>(order_key(spread) >> kBinShift) - kHeadroom;
  return a;
}

__device__ __forceinline__ int dist_bin(float v, float top, int base) {
  const int j = static_cast<int>(order_key(top - v) >> kBinShift) - base;
  return kBins - 1 - (j < 0 ? 0 : (j >= kBins ? kBins - 1 : j));
}

// Lowest score of bin b (b > 0): top minus the upper distance edge of the bin.
__device__ __forceinline__ float bin_floor(int b, float top, int base) {
  const int j = kBins - 1 - b;
  return top - key_to_float(static_cast<uint32_t>(base + j + 1) << kBinShift);
}

// Columns C*16 .. C*16+15 of a warp's 64: the head-weighted ReLU sums in the
// order of relu_wsum (even heads into a0, odd into a1, then a0 + a1), with
// a query's running sums acc = {a0, a1} carried across chunks when it spans
// several.  The halved weights come four at a time (one 16-byte shared load
// into two 64-bit pairs), so neither operand of the packed FMA is repacked.
template <int MH, int C, int QH>
__device__ __forceinline__ void chunk_wsum(const float (&v)[16], const float* wcol,
                                           uint64_t& acc, float (&sc)[QH], int tile_dep) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    constexpr int kBase = C * 16;
    const int col = kBase + 4 * p;
    // The load is not volatile, so it may be scheduled early within the
    // tile; `tile_dep` (unused by the instruction) ties it to this tile so it
    // is never hoisted out of the tile loop or above the barrier after which
    // a group's weights are written.
    uint64_t wlo, whi;
    asm("ld.shared.v2.b64 {%0, %1}, [%2];"
        : "=l"(wlo), "=l"(whi)
        : "r"(smem_u32(wcol + col)), "r"(tile_dep));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c2 = col + 2 * h;
      if (c2 % MH == 0) acc = 0ull;  // {+0, +0}
      const float c0 = v[4 * p + 2 * h], c1 = v[4 * p + 2 * h + 1];
      ffma2_acc(acc, h ? whi : wlo, c0 + fabsf(c0), c1 + fabsf(c1));
      if ((c2 + 2) % MH == 0) sc[c2 / MH] = sum_pair(acc);
    }
  }
}

// Appends {v, key} at *p and advances p by one list row (128 entries) when
// v >= tau; one compare, one predicated store, one predicated add.  (No
// memory clobber: nothing in this thread reads the lists back before a
// barrier, and the barriers are compiler fences.)
__device__ __forceinline__ void append_if(uint2*& p, float v, float tau, int key) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ge.f32 q, %1, %2;\n\t"
      "@q st.global.v2.b32 [%0], {%3, %4};\n\t"
      "@q add.s64 %0, %0, 1024;\n\t}\n"
      : "+l"(p)
      : "f"(v), "f"(tau), "r"(__float_as_uint(v)), "r"(key));
}

// Barrier over the epilogue warps (bounded; warp-uniform result).
__device__ __forceinline__ bool ep_barrier(Smem& s, uint32_t& phase, uint32_t* status) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(s.ebar);
  const bool ok = warp_wait(s.ebar, phase, s.abort, status);
  phase ^= 1u;
  return ok;
}

// 64-bit selection key: score order first, then the lower token index.
__device__ __forceinline__ uint64_t sel_key(uint2 e) {
  return (static_cast<uint64_t>(order_key(__uint_as_float(e.x))) << 32) |
         static_cast<uint64_t>(0xFFFFFFFFu - e.y);
}

// Bin (of `nb` descending-ordered counts, `per` per lane) where the count
// from the top reaches `need`; returns bin, count above it and its count.
template <int PER, typename Count>
__device__ __forceinline__ void find_crossing_by(Count count, int nb, uint32_t need, int& bin,
                                                 uint32_t& above_out, uint32_t& cnt_out) {
  const int lane = threadIdx.x & 31;
  uint32_t c[PER], loc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    c[i] = count(nb - 1 - (lane * PER + i));
    loc += c[i];
  }
  uint32_t inc = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  uint32_t above = inc - loc;
  int mb = -1;
  uint32_t ma = 0, mc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    if (above < need && above + c[i] >= need) {
      mb = nb - 1 - (lane * PER + i);
      ma = above;
      mc = c[i];
    }
    above += c[i];
  }
  const uint32_t who = __ballot_sync(0xffffffffu, mb >= 0);
  if (!who) {
    bin = -1;
    above_out = cnt_out = 0;
    return;
  }
  const int src = __ffs(who) - 1;
  bin = __shfl_sync(0xffffffffu, mb, src);
  above_out = __shfl_sync(0xffffffffu, ma, src);
  cnt_out = __shfl_sync(0xffffffffu, mc, src);
}

template <int PER>
__device__ __forceinline__ void find_crossing(const uint32_t* hist, int nb, uint32_t need,
                                              int& bin, uint32_t& above_out, uint32_t& cnt_out) {
  find_crossing_by<PER>([&](int b) { return hist[b]; }, nb, need, bin, above_out, cnt_out);
}

// Same over a histogram of 16-bit counts packed two per word.
template <int PER>
__device__ __forceinline__ void find_crossing16(const uint32_t* words, int nb, uint32_t need,
                                                int& bin, uint32_t& above_out,
                                                uint32_t& cnt_out) {
  find_crossing_by<PER>([&](int b) { return (words[b >> 1] >> ((b & 1) * 16)) & 0xffffu; }, nb,
                        need, bin, above_out, cnt_out);
}

// Exact top-k of one query's candidates, by one warp.  The candidates sit in
// 128 lists (one per TMEM lane, i.e. per key row of a tile) stored row by
// row: entry r of list l at region[r * 128 + l]; list l holds cnt[l]
// entries.  Lane j reads lists j, j+32, j+64, j+96, so each load instruction
// reads 256 contiguous bytes.  Threshold-bin entries are compacted to the
// front of their own list, which only rewrites entries that the same lane
// has already read.
__device__ void final_select(uint2* region, const int* cnt, Anchor anc, int k, int32_t* idx,
                             float* val, uint32_t* selh) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  constexpr uint32_t kAll = 0xffffffffu;
  int c[4], z[4];
  int mine = 0, cm = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c[i] = cnt[lane + 32 * i];
    z[i] = 0;
    mine += c[i];
    cm = max(cm, c[i]);
  }
  const int n = __reduce_add_sync(kAll, mine);
  const int rows = __reduce_max_sync(kAll, cm);
  uint2* mine_col = region + lane;  // entry (r, list lane + 32 i) at mine_col[r * 128 + 32 * i]
  int out = 0;
  if (n <= k) {
    for (int r = 0; r < rows; ++r) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool p = r < c[i];
        uint2 e = make_uint2(0u, 0u);
        if (p) e = mine_col[(int64_t)r * 128 + 32 * i];
        const uint32_t b = __ballot_sync(kAll, p);
        const int o = out + __popc(b & lt);
        if (p) {
          idx[o] = static_cast<int32_t>(e.y);
          val[o] = __uint_as_float(e.x) + 0.0f;
        }
        out += __popc(b);
      }
    }
  } else {
    constexpr int kR = 4;  // rows per batch: 16 loads in flight per lane
    // Pass 0: histogram of the entries (bins relative to the query's anchor).
    // Its loads keep the default L2 policy, so that pass 1's re-read of the
    // same rows mostly hits L2; pass 1's are marked evict-first (last use).
    for (int i = lane; i < kBins; i += 32) selh[i] = 0u;
    __syncwarp();
    for (int r0 = 0; r0 < rows; r0 += kR) {
      uint32_t xv[kR][4];
#pragma unroll
      for (int u = 0; u < kR; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          xv[u][i] = r0 + u < c[i] ? __ldcg(&mine_col[(int64_t)(r0 + u) * 128 + 32 * i].x) : 0u;
#pragma unroll
      for (int u = 0; u < kR; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          red_add_shared_if(&selh[dist_bin(__uint_as_float(xv[u][i]), anc.top, anc.base)],
                            r0 + u < c[i]);
    }
    __syncwarp();
    int bstar;
    uint32_t A, Z;
    find_crossing<kBins / 32>(selh, kBins, (uint32_t)k, bstar, A, Z);
    uint32_t need = (uint32_t)k - A;
    __syncwarp();
    // Pass 1: entries above the threshold bin go out; threshold-bin entries
    // move to the front of their list.
    for (int r0 = 0; r0 < rows; r0 += kR) {
      uint2 ev[kR][4];
#pragma unroll
      for (int u = 0; u < kR; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          ev[u][i] = r0 + u < c[i] ? __ldcs(&mine_col[(int64_t)(r0 + u) * 128 + 32 * i])
                                   : make_uint2(0u, 0u);
#pragma unroll
      for (int u = 0; u < kR; ++u) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint2 e = ev[u][i];
          const int b = r0 + u < c[i] ? dist_bin(__uint_as_float(e.x), anc.top, anc.base) : -1;
          const uint32_t up = __ballot_sync(kAll, b > bstar);
          const int o = out + __popc(up & lt);
          st_global_u32_if(idx + o, e.y, b > bstar && o < k);
          st_global_u32_if(val + o, __float_as_uint(__uint_as_float(e.x) + 0.0f),
                           b > bstar && o < k);
          out += __popc(up);
          if (b == bstar) {
            mine_col[(int64_t)z[i] * 128 + 32 * i] = e;
            ++z[i];
          }
        }
      }
    }
    int zm = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) zm = max(zm, z[i]);
    const int zrows = __reduce_max_sync(kAll, zm);
    __syncwarp();
    // Pass 2: choose `need` of the Z threshold-bin entries by exact key.
    int shift = 64;
    uint64_t prefix = 0;
    if (need < Z) {
      for (int p = 0; p < 8; ++p) {
        const int sh = 56 - 8 * p;
        for (int i = lane; i < kSelBins; i += 32) selh[i] = 0;
        __syncwarp();
        for (int r = 0; r < zrows; ++r) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (r < z[i]) {
              const uint64_t key = sel_key(mine_col[(int64_t)r * 128 + 32 * i]);
              if (p == 0 || (key >> (sh + 8)) == prefix) atomicAdd(&selh[(key >> sh) & 255u], 1u);
            }
          }
        }
        __syncwarp();
        int bin;
        uint32_t ab, cn;
        find_crossing<8>(selh, kSelBins, need, bin, ab, cn);
        need -= ab;
        prefix = (prefix << 8) | static_cast<uint64_t>(bin);
        shift = sh;
        __syncwarp();
        if (cn == need) break;
      }
    }
    for (int r = 0; r < zrows; ++r) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool p = r < z[i];
        uint2 e = make_uint2(0u, 0u);
        if (p) e = mine_col[(int64_t)r * 128 + 32 * i];
        const bool take = p && (shift == 64 || (sel_key(e) >> shift) >= prefix);
        const uint32_t tb = __ballot_sync(kAll, take);
        const int o = out + __popc(tb & lt);
        if (take && o < k) {
          idx[o] = static_cast<int32_t>(e.y);
          val[o] = __uint_as_float(e.x) + 0.0f;
        }
        out += __popc(tb);
      }
    }
  }
  for (int j = out + lane; j < k; j += 32) {
    idx[j] = -1;
    val[j] = -INFINITY;
  }
}

// This CTA's j-th schedule slot.  Groups come longest first; the rounds of
// gridDim.x slots alternate direction (CTA b takes slot b, then the round's
// last-but-b, ...), so that every CTA's sum of group lengths is about equal.
__device__ __forceinline__ int sched_slot(int j) {
  const int g = (int)gridDim.x, b = (int)blockIdx.x;
  return j * g + ((j & 1) ? g - 1 - b : b);
}

// Which group a CTA takes at schedule slot gs: longest prefix first from the
// planner's table, or (fixup launch) one query from the failure list.
struct Sched {
  const int4* groups;
  const int* count;        // number of groups (or of failed queries)
  const int32_t* fail_in;  // fixup launch: failed query indices; else nullptr
  int32_t* fail_out;       // first launch: where failed queries are recorded
  int* fail_count;
  const int32_t* qo;       // query offsets (fixup: query -> sequence)
  const int32_t* q_pos;
  int S;
};

__device__ __forceinline__ int4 fetch_group(const Sched& sc, int count, int gs) {
  if (!sc.fail_in) return sc.groups[count - 1 - gs];
  const int t = sc.fail_in[gs];
  return make_int4(upper_segment<int32_t>(sc.qo, sc.S, t), t, t + 1, sc.q_pos[t]);
}

// Probe schedule: tiles kProbeOff, kProbeOff + kProbeStride, ... of groups
// whose longest prefix spans at least kProbeMinTiles tiles.
// At most kProbeMaxTiles, so that no 16-bit bin count can overflow.
constexpr int kProbeMaxTiles = 65535 / kTileKeys;
__device__ __forceinline__ int probe_tiles(bool probe, int ntiles) {
  if (!probe || ntiles < kProbeMinTiles) return 0;
  const int np = (ntiles - kProbeOff + kProbeStride - 1) / kProbeStride;
  return np < kProbeMaxTiles ? np : kProbeMaxTiles;
}

// MMA width N: the group's 256 (query, head) columns, or in the rescan
// launch (one query per group) only that query's MH heads (at least 16).
template <int MH>
__device__ __forceinline__ int mma_cols(bool probe) {
  return probe ? kN : (MH < 16 ? 16 : MH);
}

// Candidate list of (buffer b, query slot q) of this CTA: rows_cap rows of 128.
// Deferred selection (anchor != nullptr): one list per query row t instead,
// [T][rows_cap][128] with counts [T][128] and the query's histogram anchor,
// selected after the pass by select_deferred_kernel.
struct Lists {
  uint2* cand;   // [grid][2][slots][rows_cap][128], or [T][rows_cap][128]
  int* cnt;      // [grid][2][slots][128], or [T][128]
  int rows_cap;
  int slots;
  int2* anchor;  // [T] {base, top bits}: deferred selection; nullptr: selected in the kernel
  __device__ __forceinline__ uint2* list_t(int64_t t) const {
    return cand + t * rows_cap * 128;
  }
  __device__ __forceinline__ int* counts_t(int64_t t) const { return cnt + t * 128; }
  __device__ __forceinline__ int64_t id(int b, int q) const {
    return ((int64_t)blockIdx.x * 2 + b) * slots + q;
  }
  __device__ __forceinline__ uint2* list(int b, int q) const {
    return cand + id(b, q) * rows_cap * 128;
  }
  __device__ __forceinline__ int* counts(int b, int q) const { return cnt + id(b, q) * 128; }
};

// Verify one query of a handed-over group and select its exact top-k (one
// warp).  Every key scoring at least the starting threshold was appended, so
// min(k, n) appended entries (none dropped at a full list) prove that the
// exact top-k is among them; otherwise the query goes to the rescan launch.
__device__ void select_query(const Smem& s, const Lists& ls, const Sched& sc, int b, int qi,
                             int k, int32_t* idx_out, float* val_out, uint32_t* selh) {
  const int lane = threadIdx.x & 31;
  const int t = s.mrow[b * kMaxG + qi];
  const int p = s.mpos[b * kMaxG + qi];
  if (p < 0) {  // invalid position: padded row
    for (int j = lane; j < k; j += 32) {
      idx_out[(int64_t)t * k + j] = -1;
      val_out[(int64_t)t * k + j] = -INFINITY;
    }
    return;
  }
  const int* qcnt = ls.counts(b, qi);
  const int c0 = qcnt[lane], c1 = qcnt[lane + 32], c2 = qcnt[lane + 64], c3 = qcnt[lane + 96];
  const int napp = __reduce_add_sync(0xffffffffu, c0 + c1 + c2 + c3);
  const int cmax = __reduce_max_sync(0xffffffffu, max(max(c0, c1), max(c2, c3)));
  const int need = min(k, p + 1);
  if (napp < need || cmax > ls.rows_cap) {
    if (lane == 0 && sc.fail_out) sc.fail_out[atomicAdd(sc.fail_count, 1)] = t;
    return;
  }
  final_select(ls.list(b, qi), qcnt, Anchor{s.mtop[b * kMaxG + qi], s.mbase[b * kMaxG + qi]}, k,
               idx_out + (int64_t)t * k, val_out + (int64_t)t * k, selh);
}

// Claims queries of candidate buffer b and selects them until none is left.
__device__ void select_claimed(const Smem& s, const Lists& ls, const Sched& sc, int b, int nq,
                               int k, int32_t* idx_out, float* val_out, uint32_t* selh) {
  const int lane = threadIdx.x & 31;
  while (true) {
    int qi = 0;
    if (lane == 0) qi = atomicAdd(&s.selnext[b], 1);
    qi = __shfl_sync(0xffffffffu, qi, 0);
    if (qi >= nq) break;
    select_query(s, ls, sc, b, qi, k, idx_out, val_out, selh);
    __syncwarp();
    __threadfence_block();  // this warp's reads of the lists are done
    if (lane == 0) atomicAdd(&s.seldone[b], 1);
  }
}

// Bounded wait (warp-uniform) until *c >= target.
__device__ __forceinline__ bool wait_count(const int* c, int target, int* abort,
                                           uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const long long t0 = clock64();
  while (true) {
    int v = 0, give_up = 0;
    if (lane == 0) {
      v = *reinterpret_cast<const volatile int*>(c);
      if (v < target) {
        if (*reinterpret_cast<volatile int*>(abort)) {
          give_up = 1;
        } else if (clock64() - t0 > kWaitCycles) {
          *reinterpret_cast<volatile int*>(abort) = 1;
          set_status(status, MISA_STATUS_TIMEOUT);
          give_up = 1;
        }
      }
    }
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v >= target) return true;
    if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    __nanosleep(128);
  }
}

template <int MH>
// 20 warps at 96 registers each: one CTA per SM.
__global__ void __maxnreg__(96)
    score_stream_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap qmap, const float* __restrict__ wsel,
                        const int64_t* __restrict__ ko, Sched sc, int k, Lists ls,
                        int32_t* __restrict__ idx_out, float* __restrict__ val_out,
                        uint32_t* status) {
  constexpr int G = kN / MH;          // queries per group
  constexpr int QH = G / kParts;      // queries per epilogue warp (its column part)
  static_assert(MH >= 8 && MH <= 64 && G <= kMaxG && QH >= 1, "unsupported head count");
  extern __shared__ uint8_t smem_raw[];

  const int count = *sc.count;
  if ((int)blockIdx.x >= count) return;
  const bool probe = sc.fail_in == nullptr;   // the fixup launch scans without a probe
  const bool deferred = ls.anchor != nullptr;  // lists per query, selected after the launch

  Smem s = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], kEpiWarps);
    }
    mbar_init(s.qfull, 1);
    mbar_init(s.qempty, 1);
    mbar_init(s.ebar, kEpiWarps);
    mbar_init(s.drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.selready[i], kEpiWarps);
    }
    *s.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&qmap);
      int it = 0, gl = 0;
      bool ok = true;
      for (int j = 0, gs = blockIdx.x; ok && gs < count; gs = sched_slot(++j)) {
        const int4 grp = fetch_group(sc, count, gs);
        if (grp.w < 0) continue;  // no valid query in the group
        const int64_t key_base = ko[grp.x];
        const int ntiles = (grp.w + kTileKeys) / kTileKeys;
        const int np = probe_tiles(probe, ntiles);
        if (!(ok = mbar_wait(s.qempty, (gl & 1) ^ 1, s.abort, status))) break;
        const int qrows = (mma_cols<MH>(probe) + 31) / 32 * 32;  // query rows the MMAs read
        mbar_arrive_expect_tx(s.qfull, 2u * qrows * 128u);
        for (int h = 0; h < 2; ++h)
          for (int r0 = 0; r0 < qrows; r0 += 32)
            tma_load_2d(&qmap, s.qfull, s.q + h * kQHalfBytes + r0 * 128, h * 64,
                        grp.y * MH + r0);
        ++gl;
        for (int step = 0; step < np + ntiles; ++step, ++it) {
          const int tile = step < np ? kProbeOff + kProbeStride * step : step - np;
          const int st = it % kStages;
          if (!(ok = mbar_wait(&s.empty[st], ((it / kStages) & 1) ^ 1, s.abort, status))) break;
          mbar_arrive_expect_tx(&s.full[st], kStageBytes);
          const int32_t krow = (int32_t)(key_base + (int64_t)tile * kTileKeys);
          uint8_t* dst = s.k + st * kStageBytes;
          tma_load_2d(&kmap, &s.full[st], dst, 0, krow);
          tma_load_2d(&kmap, &s.full[st], dst + kHalfBytes, 64, krow);
        }
      }
      // Drain this CTA's copies before it exits.
      for (int i = max(0, it - kStages); i < it; ++i)
        mbar_wait(&s.full[i % kStages], (i / kStages) & 1, s.abort, status, kDrainCycles, true);
      if (gl > 0) mbar_wait(s.qfull, (gl - 1) & 1, s.abort, status, kDrainCycles, true);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileKeys, mma_cols<MH>(probe));
      const uint32_t q_addr = smem_u32(s.q);
      int it = 0, tb = 0, gl = 0;
      bool ok = true;
      for (int j = 0, gs = blockIdx.x; ok && gs < count; gs = sched_slot(++j)) {
        const int4 grp = fetch_group(sc, count, gs);
        if (grp.w < 0) continue;
        const int ntiles = (grp.w + kTileKeys) / kTileKeys;
        const int np = probe_tiles(probe, ntiles);
        if (!(ok = mbar_wait(s.qfull, gl & 1, s.abort, status))) break;
        tc_fence_after();
        for (int step = 0; step < np + ntiles; ++step, ++it, ++tb) {
          const int st = it % kStages, buf = tb & 1;
          if (!(ok = mbar_wait(&s.full[st], (it / kStages) & 1, s.abort, status))) break;
          if (!(ok = mbar_wait(&s.tempty[buf], ((tb >> 1) & 1) ^ 1, s.abort, status))) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(s.k + st * kStageBytes);
          const uint32_t d = tmem_base + buf * kN;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t a = sw128_kmajor_desc(k_addr + (kk >> 2) * kHalfBytes + off);
            const uint64_t b = sw128_kmajor_desc(q_addr + (kk >> 2) * kQHalfBytes + off);
            umma_bf16(d, a, b, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s.empty[st]);
          umma_commit(&s.tfull[buf]);
        }
        umma_commit(s.qempty);  // the group's rows may be replaced once these MMAs are done
        ++gl;
      }
      umma_commit(s.drain);
      mbar_wait(s.drain, 0, s.abort, status, kDrainCycles, true);
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;                  // 0..kEpiWarps-1
    const int quarter = warp & 3;            // TMEM lane quarter of this warp
    const int half = e >> 2;                 // column part: queries half*QH .. half*QH+QH-1
    const int lrow = quarter * 32 + lane;    // key row of the tile
    const int et = threadIdx.x - 64;         // 0..kEpiThreads-1
    int gl = 0;  // groups done by this warp (candidate buffer gl & 1)
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t ephase = 0;
    int tb = 0;
    bool ok = true;
    for (int j = 0, gs = blockIdx.x; ok && gs < count; gs = sched_slot(++j)) {
      const int4 grp = fetch_group(sc, count, gs);
      if (grp.w < 0) continue;
      const int seq = grp.x, qb = grp.y, nq = grp.z - grp.y;
      const int ntiles = (grp.w + kTileKeys) / kTileKeys;
      const int np = probe_tiles(probe, ntiles);
      const int64_t L = ko[seq + 1] - ko[seq];
      const int bsel = gl & 1;
      if (gl >= 2 && !deferred) {
        // The group two back used this candidate buffer: claim what the
        // selectors have not taken yet, then wait until all of it is done.
        // The probe histograms are free here and serve as select scratch.
        const int nqo = s.selnq[bsel];
        select_claimed(s, ls, sc, bsel, nqo, k, idx_out, val_out, s.hist + e * kSelBins);
        if (!(ok = wait_count(&s.seldone[bsel], nqo, s.abort, status))) break;
        if (!(ok = ep_barrier(s, ephase, status))) break;
      }
      // Group state: column weights, query limits, selection state.
      if (et < kN) {
        const int qi = et / MH;
        s.w[et] = qi < nq ? relu_weight(wsel[(int64_t)(qb + qi) * MH + (et - qi * MH)]) : 0.f;
      }
      if (et < G) {
        int p = -1;
        if (et < nq) {
          p = sc.q_pos[qb + et];
          if (p < 0 || p >= L) p = -1;
        }
        s.pos[et] = p;
        s.row[et] = qb + et;
        s.tau[et] = p >= 0 ? -INFINITY : INFINITY;  // padding / invalid slots never append
        s.maxkey[et] = 0u;
        s.minkey[et] = 0xFFFFFFFFu;
      }
      for (int i = et; i < G * kHistWords; i += kEpiThreads) s.hist[i] = 0u;
      // This lane's list of each of its warp's queries (row-major over the 128
      // lists of a query): qlist(qq) is the first row, nxt[qq] the next row
      // to write.  A list that comes within kCheckTiles rows of its capacity
      // (checked every kCheckTiles main-pass tiles, so no store can pass the
      // end) stops appending and is marked full (one row past capacity).
      uint2* const mylist =
          (deferred ? ls.list_t(qb + half * QH)
                    : ls.list(bsel, 0) + (int64_t)(half * QH) * ls.rows_cap * 128) +
          lrow;
      const int64_t qstride = 128 * (int64_t)ls.rows_cap;
      auto qlist = [&](int qq) { return mylist + qq * qstride; };
      uint2* nxt[QH];
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) nxt[qq] = qlist(qq);
      if (!(ok = ep_barrier(s, ephase, status))) break;
      int minpos = 0x7fffffff;  // smallest valid position of the group (-1 if any invalid)
      for (int qi = 0; qi < nq; ++qi) minpos = min(minpos, s.pos[qi]);
      float tauR[QH];  // this warp's copy of its queries' thresholds
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) tauR[qq] = s.tau[half * QH + qq];

      // One tile: wait for its accumulators, read the warp's 64 columns in
      // four 16-column TMEM loads (each issued before the previous chunk is
      // summed, so the load latency overlaps the arithmetic; the buffer is
      // released after the last load) and form this lane's score of each of
      // the warp's queries.  The tile loops below are specialised (probe
      // tiles, full main-pass tiles in runs of kCheckTiles, the diagonal
      // tiles) so that no per-tile branch sits around this body.
      // (In the rescan launch the MMAs fill only the first query's columns;
      // the other columns hold stale values, read but never used: those query
      // slots are padding, which never appends.)
      auto tile_scores = [&](float (&sc_)[QH]) -> bool {
        const int buf = tb & 1;
        if (!warp_wait(&s.tfull[buf], (tb >> 1) & 1, s.abort, status)) return false;
        tc_fence_after();
        const uint32_t taddr = lane_addr + buf * kN + half * kColsPerWarp;
        const float* wcol = s.w + half * kColsPerWarp;
        uint64_t acc = 0ull;
        float vA[16], vB[16];
        tmem_ld16(taddr, vA);
        tmem_wait_ld();
        reg_fence16(vA);
        tmem_ld16(taddr + 16, vB);
        chunk_wsum<MH, 0>(vA, wcol, acc, sc_, tb);
        tmem_wait_ld();
        reg_fence16(vB);
        tmem_ld16(taddr + 32, vA);
        chunk_wsum<MH, 1>(vB, wcol, acc, sc_, tb);
        tmem_wait_ld();
        reg_fence16(vA);
        tmem_ld16(taddr + 48, vB);
        chunk_wsum<MH, 2>(vA, wcol, acc, sc_, tb);
        tmem_wait_ld();
        reg_fence16(vB);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tempty[buf]);
        chunk_wsum<MH, 3>(vB, wcol, acc, sc_, tb);
        ++tb;
        return true;
      };
      // Anchor every query's histogram on the range of its first scored tile.
      auto anchor = [&](const float (&sc_)[QH], int key) -> bool {
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) {
          const int qi = half * QH + qq;
          const bool v = key <= s.pos[qi];
          const uint32_t kk = order_key(sc_[qq]);
          const uint32_t hi = __reduce_max_sync(0xffffffffu, v ? kk : 0u);
          const uint32_t lo = __reduce_min_sync(0xffffffffu, v ? kk : 0xFFFFFFFFu);
          if (lane == 0) {
            atomicMax(&s.maxkey[qi], hi);
            atomicMin(&s.minkey[qi], lo);
          }
        }
        if (!ep_barrier(s, ephase, status)) return false;
        // every warp of a half writes the same anchors for its queries
        if (lane < QH) {
          const Anchor a = make_anchor(s.maxkey[half * QH + lane], s.minkey[half * QH + lane]);
          s.base[half * QH + lane] = a.base;
          s.top[half * QH + lane] = a.top;
        }
        __syncwarp();
        return true;
      };
      // Streaming selection: a passing lane appends to its own list.  Tiles
      // wholly below every query's position need no causal compare.
      auto append_full = [&](const float (&sc_)[QH], int key) {
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) append_if(nxt[qq], sc_[qq], tauR[qq], key);
      };
      auto append_causal = [&](const float (&sc_)[QH], int key) {
#pragma unroll
        for (int qq = 0; qq < QH; ++qq)
          append_if(nxt[qq], sc_[qq], key <= s.pos[half * QH + qq] ? tauR[qq] : INFINITY, key);
      };
      // After main-pass tiles 0..i-1: each tile adds at most one row to a
      // list, so a list may hold up to `room` rows now and still take every
      // row of the tiles until the next check.  (Lists hold at least
      // min(8, tiles) rows, so none can fill before the first check; the
      // rescan launch's lists hold a row per tile and are not checked.)
      auto check_room = [&](int i) {
        if (!probe || i >= ntiles) return;
        const int room = ls.rows_cap - min(kCheckTiles, ntiles - i);
        // (the list starts are recomputed here rather than kept in registers
        // across the tile loops: the volatile copy keeps the compiler from
        // hoisting them)
        int64_t qs;
        asm volatile("mov.b64 %0, %1;" : "=l"(qs) : "l"(qstride));
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) {
          const uint2* start = mylist + qq * qs;
          if (nxt[qq] - start > (int64_t)room * 128) {
            tauR[qq] = INFINITY;
            nxt[qq] = const_cast<uint2*>(start) + (int64_t)(ls.rows_cap + 1) * 128;
          }
        }
      };

      // ---- probe tiles (kProbeOff + kProbeStride * j): histogram only
      for (int step = 0; step < np; ++step) {
        float sc_[QH];
        if (!(ok = tile_scores(sc_))) break;
        const int key = (kProbeOff + kProbeStride * step) * kTileKeys + lrow;
        if (step == 0 && !(ok = anchor(sc_, key))) break;
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) {
          const int qi = half * QH + qq;
          const int b = dist_bin(sc_[qq], s.top[qi], s.base[qi]);
          red_add_shared_val_if(&s.hist[qi * kHistWords + (b >> 1)], 1u << ((b & 1) * 16),
                                key <= s.pos[qi]);
        }
      }
      if (!ok) break;
      if (np > 0) {
        // Starting thresholds from the sample: the bin holding the r-th best
        // sampled score, r = k*f + 4*sqrt(k*f) + 1 (f: sampled share of the
        // query's prefix).  Verified at the end of the group.
        if (!(ok = ep_barrier(s, ephase, status))) break;
        for (int qi = e; qi < G; qi += kEpiWarps) {
          const int n = s.pos[qi] + 1;
          int ns = 0;
          for (int j = lane; j < np; j += 32) {
            const int rem = n - (kProbeOff + kProbeStride * j) * kTileKeys;
            ns += rem <= 0 ? 0 : (rem > kTileKeys ? kTileKeys : rem);
          }
          ns = __reduce_add_sync(0xffffffffu, ns);
          float t0 = s.pos[qi] >= 0 ? -INFINITY : INFINITY;
          if (n > k && ns > 0) {
            const float ks = (float)k * (float)ns / (float)n;
            const int r = (int)ceilf(ks + 4.f * sqrtf(ks)) + 1;
            if (r <= ns) {
              int bstar;
              uint32_t A, Z;
              find_crossing16<kBins / 32>(s.hist + qi * kHistWords, kBins, (uint32_t)r, bstar, A,
                                          Z);
              if (bstar > 0) t0 = bin_floor(bstar, s.top[qi], s.base[qi]);
            }
          }
          if (lane == 0) s.tau[qi] = t0;
          for (int b = lane; b < kHistWords; b += 32) s.hist[qi * kHistWords + b] = 0u;
        }
        if (!(ok = ep_barrier(s, ephase, status))) break;
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) tauR[qq] = s.tau[half * QH + qq];
      }

      // ---- main pass over tiles 0..ntiles-1
      const int nfull = min(ntiles, (minpos + 1) / kTileKeys);  // tiles below every position
      int i = 0;
      if (np == 0 && ntiles > 0) {
        // no probe: the first main tile anchors the histograms
        float sc_[QH];
        if (!(ok = tile_scores(sc_))) break;
        const int key = lrow;
        if (!(ok = anchor(sc_, key))) break;
        if (nfull > 0) append_full(sc_, key); else append_causal(sc_, key);
        i = 1;
      }
      while (ok && i < nfull) {
        const int iend = min(nfull, (i / kCheckTiles + 1) * kCheckTiles);
        for (; i < iend; ++i) {
          float sc_[QH];
          if (!(ok = tile_scores(sc_))) break;
          append_full(sc_, i * kTileKeys + lrow);
        }
        if (ok && i % kCheckTiles == 0) check_room(i);
      }
      for (; ok && i < ntiles; ++i) {
        float sc_[QH];
        if (!(ok = tile_scores(sc_))) break;
        append_causal(sc_, i * kTileKeys + lrow);
        if (i % kCheckTiles == kCheckTiles - 1) check_room(i + 1);
      }
      if (!ok) break;
      int cnt[QH];
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) cnt[qq] = static_cast<int>((nxt[qq] - qlist(qq)) >> 7);
      if (deferred) {
        // Leave the group's counts and histogram anchors for the selection
        // pass after this launch.
#pragma unroll
        for (int qq = 0; qq < QH; ++qq)
          if (half * QH + qq < nq) ls.counts_t(qb + half * QH + qq)[lrow] = cnt[qq];
        // (each half's lane-quarter-0 warp wrote these anchors itself)
        if (quarter == 0 && lane < QH && half * QH + lane < nq)
          ls.anchor[qb + half * QH + lane] =
              make_int2(s.base[half * QH + lane], __float_as_int(s.top[half * QH + lane]));
        ++gl;
        if (!(ok = ep_barrier(s, ephase, status))) break;
        continue;
      }
      // Hand the group to the selectors: counts, and (warp 0 of the
      // epilogue) the per-query positions, rows and histogram anchors.
#pragma unroll
      for (int qq = 0; qq < QH; ++qq)
        if (half * QH + qq < nq) ls.counts(bsel, half * QH + qq)[lrow] = cnt[qq];
      if (e == 0) {
        s.mpos[bsel * kMaxG + lane] = lane < G ? s.pos[lane] : -1;
        s.mrow[bsel * kMaxG + lane] = lane < G ? s.row[lane] : 0;
        s.mbase[bsel * kMaxG + lane] = lane < G ? s.base[lane] : 0;
        s.mtop[bsel * kMaxG + lane] = lane < G ? s.top[lane] : 0.f;
        if (lane == 0) {
          s.selnq[bsel] = nq;
          s.selnext[bsel] = 0;
          s.seldone[bsel] = 0;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.selready[bsel]);
      ++gl;
      if (!(ok = ep_barrier(s, ephase, status))) break;
    }
    // Help the selectors with the last groups (no more probing: the
    // histograms are free).
    for (int j = gl >= 2 ? gl - 2 : 0; ok && !deferred && j < gl; ++j)
      select_claimed(s, ls, sc, j & 1, s.selnq[j & 1], k, idx_out, val_out,
                     s.hist + e * kSelBins);
  } else {
    // ------------------------------------------------------------ selectors
    // Verify each query of the previous group and select its exact top-k
    // from the candidates, while the epilogue streams the next group.
    const int sw = warp - 2 - kEpiWarps;  // 0..kSelWarps-1
    uint32_t* selh = s.sel + sw * kSelBins;
    int gl = 0;
    bool ok = !deferred;  // deferred selection: nothing to do here
    for (int j = 0, gs = blockIdx.x; ok && gs < count; gs = sched_slot(++j)) {
      const int4 grp = fetch_group(sc, count, gs);
      if (grp.w < 0) continue;
      const int nq = grp.z - grp.y;
      const int bsel = gl & 1;
      if (!(ok = warp_wait(&s.selready[bsel], (gl >> 1) & 1, s.abort, status))) break;
      select_claimed(s, ls, sc, bsel, nq, k, idx_out, val_out, selh);
      ++gl;
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

// Deferred selection: one warp per query row, after the scoring launch.
// The same check and exact selection as select_query, on the query's own
// lists; queries that fail the check go to the rescan list.  Each warp takes
// queries t, t + nw, ... and loads the counts of the query two ahead while
// it selects the current one.  (Requesting the next query's lists into L2
// ahead of time measured slower: with 32 warps per SM the lists in flight
// exceed L2, and the prefetched rows were evicted before use.)
constexpr int kSelectThreads = 256;
constexpr int kSelectCtasPerSm = 4;

struct QCounts {
  int c0, c1, c2, c3;
};

__device__ __forceinline__ QCounts load_counts(const Lists& ls, int t, int T) {
  const int lane = threadIdx.x & 31;
  QCounts c = {0, 0, 0, 0};
  if (t < T) {
    const int* q = ls.counts_t(t);
    c.c0 = q[lane];
    c.c1 = q[lane + 32];
    c.c2 = q[lane + 64];
    c.c3 = q[lane + 96];
  }
  return c;
}

__global__ void __launch_bounds__(kSelectThreads, kSelectCtasPerSm)
    select_deferred_kernel(Lists ls, const int32_t* __restrict__ q_pos,
                           const int32_t* __restrict__ qo, const int64_t* __restrict__ ko, int S,
                           int T, int k, int32_t* __restrict__ idx_out,
                           float* __restrict__ val_out, int32_t* __restrict__ fail_out,
                           int* __restrict__ fail_count) {
  pdl_wait_then_release();
  __shared__ uint32_t selh_all[kSelectThreads / 32][kSelBins];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* selh = selh_all[warp];
  const int nw = (int)gridDim.x * (kSelectThreads / 32);
  int t = (int)blockIdx.x * (kSelectThreads / 32) + warp;
  QCounts cur = load_counts(ls, t, T), next = load_counts(ls, t + nw, T);
  for (; t < T; t += nw) {
    const QCounts after = load_counts(ls, t + 2 * nw, T);
    const int sq = upper_segment<int32_t>(qo, S, t);
    const int64_t L = ko[sq + 1] - ko[sq];
    const int p = q_pos[t];
    int32_t* idx = idx_out + (int64_t)t * k;
    float* val = val_out + (int64_t)t * k;
    if (p < 0 || p >= L) {  // invalid position: padded row (the pass skipped it)
      for (int j = lane; j < k; j += 32) {
        idx[j] = -1;
        val[j] = -INFINITY;
      }
    } else {
      const int napp = __reduce_add_sync(0xffffffffu, cur.c0 + cur.c1 + cur.c2 + cur.c3);
      const int cmax =
          __reduce_max_sync(0xffffffffu, max(max(cur.c0, cur.c1), max(cur.c2, cur.c3)));
      if (napp < min(k, p + 1) || cmax > ls.rows_cap) {
        if (lane == 0) fail_out[atomicAdd(fail_count, 1)] = t;
      } else {
        const int2 an = ls.anchor[t];
        final_select(ls.list_t(t), ls.counts_t(t), Anchor{__int_as_float(an.y), an.x}, k, idx,
                     val, selh);
      }
    }
    __syncwarp();
    cur = next;
    next = after;
  }
}

// Rows of a deferred list: twice the expected candidates per lane (about
// 1.4 k / 128 with the probe threshold) plus 16, within [32, 256] and no more
// than one row per tile; a fuller list sends its query to the rescan.  (The
// selection reads a list's expected rows in any case, so a large k - the
// MISA-dagger keep of k' = 8192, ~93 rows per lane - takes lists up to 196
// rows rather than send every query whose busiest lane passes 128 rows, 1% at
// 128K, to the far slower one-query rescan.)
constexpr int kDeferredRowsCap = 256;
int deferred_rows(int k, int64_t rows_full) {
  int64_t r = 2 * ((14 * (int64_t)k + 1279) / 1280) + 16;
  r = r < 32 ? 32 : (r > kDeferredRowsCap ? kDeferredRowsCap : r);
  return (int)(r < rows_full ? r : rows_full);
}

// Candidate storage (one workspace region, 256-byte aligned parts): the main
// pass's lists [grid][2][G][rows_main][128] and counts, the in-kernel
// rescan's lists [grid][2][1][rows_full][128] and counts, then the
// split rescan's score rows [kRescanCap][row_ld] fp32, its one-query groups
// int4 [kRescanCap] and two counters {queries rescanned by rows, rest}.
struct CandLayout {
  int rows_main, rows_full;
  int64_t row_ld;
  size_t main_lists, main_counts, fix_lists, fix_counts, rescan_rows, rescan_groups;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

CandLayout cand_layout(int grid, int64_t rows_full, int G) {
  CandLayout c;
  c.rows_full = (int)rows_full;
  c.rows_main = (int)(rows_full < kRowsCap ? rows_full : kRowsCap);
  c.row_ld = rows_full * kTileKeys;
  c.main_lists = align256((size_t)grid * 2 * G * c.rows_main * 128 * sizeof(uint2));
  c.main_counts = align256((size_t)grid * 2 * G * 128 * sizeof(int));
  c.fix_lists = align256((size_t)grid * 2 * c.rows_full * 128 * sizeof(uint2));
  c.fix_counts = align256((size_t)grid * 2 * 128 * sizeof(int));
  c.rescan_rows = align256((size_t)kRescanCap * c.row_ld * sizeof(float));
  c.rescan_groups = align256((size_t)kRescanCap * sizeof(int4) + 16);
  return c;
}

// The first kRescanCap failed queries become one-query groups for the split
// rescan (the decode-path scorer spreads each over several CTAs, then the
// top-k selects from the score rows); any further ones are counted for the
// in-kernel rescan.  One CTA.
__global__ void rescan_plan_kernel(const int32_t* __restrict__ fail_list,
                                   const int* __restrict__ fail_count,
                                   const int32_t* __restrict__ qo, int S,
                                   const int32_t* __restrict__ q_pos, int4* __restrict__ groups,
                                   int* __restrict__ counts) {
  pdl_wait_then_release();
  const int n = *fail_count;
  const int g = n < kRescanCap ? n : kRescanCap;
  for (int i = threadIdx.x; i < g; i += blockDim.x) {
    const int t = fail_list[i];
    groups[i] = make_int4(upper_segment<int32_t>(qo, S, t), t, t + 1, q_pos[t]);
  }
  if (threadIdx.x == 0) {
    counts[0] = g;
    counts[1] = n - g;
  }
}

template <int MH>
int launch_one(const StreamArgs& a, const CUtensorMap& kmap, const CUtensorMap& qmap,
               const Sched& sc, const Lists& ls, cudaStream_t st) {
  auto kern = score_stream_kernel<MH>;
  int rc = set_smem_limit((const void*)kern, kSmemBytes);
  if (rc) return rc;
  ProfScope ps(sc.fail_in ? "score_fixup" : "score", st);
  kern<<<a.grid, kThreads, kSmemBytes, st>>>(kmap, qmap, a.wsel, a.p->key_offsets, sc, a.k, ls,
                                            a.idx, a.val, status_ptr());
  return cuda_fail(cudaGetLastError(), "score_stream_kernel");
}

template <int MH>
int launch_pair(const StreamArgs& a, const CUtensorMap& kmap, const CUtensorMap& qmap,
                cudaStream_t st) {
  Sched sc;
  sc.groups = a.groups;
  sc.count = a.group_count;
  sc.fail_in = nullptr;
  sc.fail_out = a.fail_list;
  sc.fail_count = a.fail_count;
  sc.qo = a.p->query_offsets;
  sc.q_pos = a.p->q_pos;
  sc.S = a.p->num_seqs;
  const CandLayout cl = cand_layout(a.grid, a.subcap, kN / MH);
  uint8_t* base = reinterpret_cast<uint8_t*>(a.cand);
  Lists main_ls, fix_ls;
  main_ls.cand = reinterpret_cast<uint2*>(base);
  main_ls.cnt = reinterpret_cast<int*>(base + cl.main_lists);
  main_ls.rows_cap = cl.rows_main;
  main_ls.slots = kN / MH;
  fix_ls.cand = reinterpret_cast<uint2*>(base + cl.main_lists + cl.main_counts);
  fix_ls.cnt = reinterpret_cast<int*>(base + cl.main_lists + cl.main_counts + cl.fix_lists);
  fix_ls.rows_cap = cl.rows_full;
  fix_ls.slots = 1;
  main_ls.anchor = fix_ls.anchor = nullptr;
  cudaError_t e = cudaMemsetAsync(a.fail_count, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "reset failure count");
  int rc;
  if (a.dcand) {
    // Lists per query, selected by a second launch over all query rows.
    Lists dl;
    dl.cand = a.dcand;
    dl.cnt = a.dcnt;
    dl.rows_cap = a.drows;
    dl.slots = 0;
    dl.anchor = a.danchor;
    if ((rc = launch_one<MH>(a, kmap, qmap, sc, dl, st))) return rc;
    {
      ProfScope ps("select", st);
      const int grid = kSelectCtasPerSm * num_sms();  // one wave
      rc = cuda_fail(launch_pdl(select_deferred_kernel, dim3(grid), dim3(kSelectThreads), 0, st,
                                dl, a.p->q_pos, a.p->query_offsets, a.p->key_offsets,
                                a.p->num_seqs, a.p->num_queries, a.k, a.idx, a.val,
                                a.fail_list, a.fail_count),
                     "select_deferred_kernel");
      if (rc) return rc;
    }
  } else if ((rc = launch_one<MH>(a, kmap, qmap, sc, main_ls, st))) {
    return rc;
  }
  // Queries whose probe threshold did not verify are scored again without a
  // threshold.  The first kRescanCap: their full score rows by the split
  // decode-path scorer (several CTAs per query), then the top-k of each row.
  prof_count("#rescan_queries", a.fail_count, st);
  int4* rgroups = reinterpret_cast<int4*>(base + cl.main_lists + cl.main_counts + cl.fix_lists +
                                          cl.fix_counts + cl.rescan_rows);
  int* rcounts = reinterpret_cast<int*>(rgroups + kRescanCap);  // {by rows, rest}
  float* rrows = reinterpret_cast<float*>(base + cl.main_lists + cl.main_counts + cl.fix_lists +
                                          cl.fix_counts);
  {
    ProfScope ps("rescan_plan", st);
    rc = cuda_fail(launch_pdl(rescan_plan_kernel, dim3(1), dim3(128), 0, st,
                              (const int32_t*)a.fail_list, (const int*)a.fail_count,
                              a.p->query_offsets, a.p->num_seqs, a.p->q_pos, rgroups, rcounts),
                   "rescan_plan_kernel");
    if (rc) return rc;
  }
  ScoreArgs ra;
  ra.p = a.p; ra.qsel = a.qsel; ra.wsel = a.wsel; ra.m = a.m; ra.K = a.K; ra.cand = nullptr;
  ra.k_cand = 0; ra.groups = rgroups; ra.group_count = rcounts; ra.max_groups = kRescanCap;
  ra.G = 1; ra.q_lo = 0; ra.I = rrows; ra.ld = cl.row_ld; ra.max_tiles = cl.rows_full;
  ra.row_by_group = true;
  if ((rc = launch_score(ra, st))) return rc;
  if ((rc = launch_topk(*a.p, rrows, cl.row_ld, nullptr, 0, 0, kRescanCap, a.k, a.idx, a.val, st,
                        a.fail_list, rcounts)))
    return rc;
  // Any further ones: rescan inside the streaming kernel, one query per
  // group, with lists that hold every key.
  Sched fx = sc;
  fx.fail_in = a.fail_list + kRescanCap;
  fx.fail_out = nullptr;
  fx.count = rcounts + 1;
  return launch_one<MH>(a, kmap, qmap, fx, fix_ls, st);
}

}  // namespace

int stream_group_size(int m) { return kN / m; }

int64_t stream_subcap(int max_seq_len) {
  // rows of a lane's list: one per 128-key tile of the longest prefix
  return ((int64_t)max_seq_len + kTileKeys - 1) / kTileKeys;
}

size_t stream_cand_bytes(int grid, int64_t subcap, int m) {
  const CandLayout c = cand_layout(grid, subcap, kN / m);
  return c.main_lists + c.main_counts + c.fix_lists + c.fix_counts + c.rescan_rows +
         c.rescan_groups;
}

size_t stream_deferred_bytes(int T, int64_t subcap, int k) {
  const int rows = deferred_rows(k, subcap);
  return align256((size_t)T * rows * 128 * sizeof(uint2)) + align256((size_t)T * 128 * sizeof(int)) +
         align256((size_t)T * sizeof(int2));
}

int stream_deferred_rows(int k, int64_t subcap) { return deferred_rows(k, subcap); }

int launch_score_stream(const StreamArgs& a, cudaStream_t st) {
  if (a.max_groups <= 0) return MISA_OK;
  CUtensorMap kmap, qmap;
  int rc = make_kmajor_map(&kmap, a.K, a.p->total_keys, kTileKeys);
  if (rc) return rc;
  rc = make_kmajor_map(&qmap, a.qsel, (int64_t)a.p->num_queries * a.m, 32);
  if (rc) return rc;
  switch (a.m) {
    case 8: return launch_pair<8>(a, kmap, qmap, st);
    case 16: return launch_pair<16>(a, kmap, qmap, st);
    case 32: return launch_pair<32>(a, kmap, qmap, st);
    case 64: return launch_pair<64>(a, kmap, qmap, st);
    default:
      set_error("streaming scorer needs m in {8,16,32,64}, got %d", a.m);
      return MISA_ERR_UNSUPPORTED;
  }
}

}  // namespace misa
